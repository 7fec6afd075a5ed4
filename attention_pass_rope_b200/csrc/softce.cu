// Soft cross-entropy distillation loss of the draft passes ("DFlash/DSpark and EAGLE-3
// TTT draft co-training" roadmap, NeMo-RL issue 3698, "What I'm working on", item 3:
// chunked, vocabulary-split soft-CE with per-pass global normalisation; the loss's
// token_chunk_size, NeMo-RL PR 3725, merge note 3).
//
// Draft row r = (pass p, token t) has logits z = W h_r over the vocabulary and learns
// the teacher distribution q = softmax(y_u) of position u = t + p (0-based p) of its
// sequence; loss l_r = logsumexp(z) - sum_v q_v z_v.  Per pass L_p = w_p / N_p * sum l.
//
// Every GEMM here runs on one persistent tcgen05 kernel (128 x 256 output tiles, a
// 4-stage TMA ring of 64-deep K slices, a double-buffered fp32 accumulator in TMEM so
// that a tile's epilogue overlaps the next tile's products) with four epilogues:
//   STATS  forward logits z = h W^T: per (row, 256-column tile) the running maxima and
//          sums of the draft and teacher softmaxes and sum q~ z (never storing z);
//   DZ     the same logits recomputed in the backward: dz = c_r (softmax(z) - q),
//          rounded to bf16 and stored (one token chunk of rows at a time);
//   BF16   dh = dz W (W as an MN-major operand), stored as bf16;
//   ACC    dW += dz^T h (both operands MN-major), fp32 reduce-add by TMA;
//   STATSZ the forward's statistics, and the chunk's fp32 logits stored as well.
// Small kernels finish the job: teacher rows and pass counts, the merge of the tile
// statistics into lse and l, the per-pass sums, and (fused call) dz from stored logits.
//
// The fused call (ttt_softce_fwd_bwd) takes the loss's upstream gradient up front: per
// chunk of rows it runs the STATSZ GEMM, merges the statistics, turns the stored logits
// into dz with one memory pass, then dh and dW.  That is three GEMM passes where separate
// forward and backward calls need four (the backward recomputes the logits).
#include <cuda_bf16.h>

#include <cmath>

#include "../../include/ttt_attn.h"
#include "common.cuh"
#include "ttt_internal.h"

namespace ttt {
namespace {

constexpr int kBM = 128, kBN = 256, kBK = 64, kStages = 4;
constexpr int kATile = kBM * kBK * 2;            // 16 KB
constexpr int kBTile = kBN * kBK * 2;            // 32 KB
constexpr int kStageBytes = kATile + kBTile;     // 48 KB
constexpr int kSlab = 32 * 128;                  // one epilogue warp's staging slab: 32 rows x 128 B
constexpr int kOffSlab = kStages * kStageBytes;  // 192 KB
constexpr int kOffBar = kOffSlab + 8 * kSlab;    // two slabs per epilogue warp
constexpr int kSmemBytes = kOffBar + 256 + 1024; // barriers, then slack for the 1024-byte alignment
constexpr int kThreads = 192;                    // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr int kTmemCols = 512;                   // two 256-column accumulators
constexpr int kGroupM = 16;                      // output tiles are walked in bands of 16 row tiles
constexpr float kLog2e = 1.4426950408889634f;

static_assert(kSmemBytes <= 232448, "shared memory per CTA");

enum Epi { EPI_STATS = 0, EPI_DZ = 1, EPI_BF16 = 2, EPI_ACC = 3, EPI_STATSZ = 4 };

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int c0, int c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(c0), "r"(c1)
               : "memory");
}
__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap* map, const void* src, int c0, int c1) {
  asm volatile("cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(c0), "r"(c1)
               : "memory");
}

// Output tile of linear index t: bands of kGroupM row tiles, each band swept over all
// column tiles with its row tiles innermost, so that the CTAs in flight share a few
// row slabs and column slabs in L2.
__device__ __forceinline__ void tile_coords(int t, int nm, int nn, int& m, int& n) {
  const int band = t / (kGroupM * nn);
  const int first = band * kGroupM;
  const int gm = min(kGroupM, nm - first);
  const int local = t - band * kGroupM * nn;
  m = first + local % gm;
  n = local / gm;
}

// Reads 8 teacher logits (bf16) y[u][col .. col+8) as fp32; columns >= V read as -inf.
__device__ __forceinline__ void load_y8(const __nv_bfloat16* yrow, int col, int V, float (&o)[8]) {
  if (col < V) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(yrow + col));
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      o[2 * i] = __uint_as_float(ww[i] << 16);
      o[2 * i + 1] = __uint_as_float(ww[i] & 0xFFFF0000u);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = -INFINITY;
  }
}

// One 32-column slice of a row's logits v (fp32 bits) and of its teacher row: updates the
// running maxima (log2 units) and sums of the draft and teacher softmaxes and sum e^(y-m) z.
__device__ __forceinline__ void stats_update(const uint32_t (&v)[32], int col0, int V, const __nv_bfloat16* yrow,
                                             float& mz, float& sz, float& my, float& sy, float& ac) {
  float zl[32], yl[32];
#pragma unroll
  for (int g8 = 0; g8 < 4; ++g8) {
    float y8[8];
    load_y8(yrow, col0 + 8 * g8, V, y8);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int j = 8 * g8 + i;
      zl[j] = col0 + j < V ? __uint_as_float(v[j]) * kLog2e : -INFINITY;
      yl[j] = y8[i] * kLog2e;
    }
  }
  float cz = zl[0], cy = yl[0];
#pragma unroll
  for (int j = 1; j < 31; j += 2) {
    cz = max3f(cz, zl[j], zl[j + 1]);
    cy = max3f(cy, yl[j], yl[j + 1]);
  }
  cz = fmaxf(cz, zl[31]);
  cy = fmaxf(cy, yl[31]);
  const float nz = fmaxf(mz, cz), ny = fmaxf(my, cy);
  float ssz = 0.f, ssy = 0.f, sac = 0.f;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    ssz += exp2_approx(zl[j] - nz);
    const float e = exp2_approx(yl[j] - ny);
    ssy += e;
    sac = fmaf(e, col0 + j < V ? __uint_as_float(v[j]) : 0.f, sac);
  }
  const float fz = exp2_approx(mz - nz), fy = exp2_approx(my - ny);
  sz = fmaf(sz, fz, ssz);
  sy = fmaf(sy, fy, ssy);
  ac = fmaf(ac, fy, sac);
  mz = nz;
  my = ny;
}

template <int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    softce_gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                       const __grid_constant__ CUtensorMap map_out, const SoftceGemmArgs a) {
  constexpr bool A_MN = EPI == EPI_ACC;
  constexpr bool B_MN = EPI == EPI_BF16 || EPI == EPI_ACC;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;   // [2]
  uint64_t* acc_empty = acc_full + 2;     // [2]
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    mbar_init(acc_full + 0, 1);
    mbar_init(acc_full + 1, 1);
    mbar_init(acc_empty + 0, 4);  // one arrival per epilogue warp
    mbar_init(acc_empty + 1, 4);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Watchdog wd{abort_flag, a.status, a.budget_ns};

  const int nm = (a.M + kBM - 1) / kBM;
  const int nn = (a.N + kBN - 1) / kBN;
  const int ntiles = nm * nn;
  const int nk = (a.K + kBK - 1) / kBK;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&map_a);
      tma_prefetch_desc(&map_b);
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        int m, n;
        tile_coords(t, nm, nn, m, n);
        const int m0 = m * kBM, n0 = n * kBN;
        for (int kt = 0; kt < nk; ++kt, ++it) {
          const int s = it % kStages;
          if (it >= kStages && !wait_bounded(empty + s, ((it / kStages) - 1) & 1, wd, kSiteCeEmpty)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + s * kStageBytes;
          uint8_t* sb = sa + kATile;
          const int k0 = kt * kBK;
          mbar_arrive_expect_tx(full + s, kStageBytes);
          if (A_MN) {
            // A^T stored [K rows][M]: two 64-column chunks of 64 K rows
            tma_load_2d(sa, &map_a, full + s, m0, k0);
            tma_load_2d(sa + kATile / 2, &map_a, full + s, m0 + 64, k0);
          } else {
            tma_load_2d(sa, &map_a, full + s, k0, (EPI <= EPI_DZ || EPI == EPI_STATSZ ? a.row0 : 0) + m0);
          }
          if (B_MN) {
#pragma unroll
            for (int c = 0; c < 4; ++c) tma_load_2d(sb + c * (kBTile / 4), &map_b, full + s, n0 + 64 * c, k0);
          } else {
            tma_load_2d(sb, &map_b, full + s, k0, n0);
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN, A_MN, B_MN);
    // descriptor K advance per 16-deep MMA: 32 bytes along a K-major row, 16 rows of
    // 128 bytes down an MN-major chunk (encoded >> 4)
    constexpr uint32_t a_step = A_MN ? 128u : 2u;
    constexpr uint32_t b_step = B_MN ? 128u : 2u;
    int it = 0, local = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++local) {
      const int b = local & 1;
      if (local >= 2 && !wait_warp(acc_empty + b, ((local >> 1) - 1) & 1, wd, kSiteCeAccEmpty)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t dacc = tmem + b * kBN;
      for (int kt = 0; kt < nk; ++kt, ++it) {
        const int s = it % kStages;
        if (!wait_warp(full + s, (it / kStages) & 1, wd, kSiteCeFull)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + s * kStageBytes);
        const uint64_t ad = sdesc_sw128(sa, A_MN ? kATile / 2 : 16, 1024);
        const uint64_t bd = sdesc_sw128(sa + kATile, B_MN ? kBTile / 4 : 16, 1024);
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk)
          umma_ss_warp(dacc, ad + kk * a_step, bd + kk * b_step, idesc, (kt | kk) ? 1u : 0u);
        umma_commit_warp(empty + s);
      }
      if (!ok) break;
      umma_commit_warp(acc_full + b);
    }
    umma_commit_warp(drain);
    wait_drain(drain, 0, wd, kSiteCeDrain);
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (warps 2-5)
    const int q = warp & 3;            // TMEM lanes 32q .. 32q+31 = tile rows
    const int row = 32 * q + lane;
    uint8_t* slabs = smem + kOffSlab + (warp - 2) * 2 * kSlab;
    int nslab = 0;  // staging slabs this warp has filled (double-buffered)
    int local = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++local) {
      int m, n;
      tile_coords(t, nm, nn, m, n);
      const int m0 = m * kBM, n0 = n * kBN;
      const int b = local & 1;
      if (!wait_warp(acc_full + b, (local >> 1) & 1, wd, kSiteCeAccFull)) break;
      tc_fence_after();
      const uint32_t tacc = tmem + (static_cast<uint32_t>(32 * q) << 16) + b * kBN;
      const int r = m0 + row;  // output row of this thread

      if (EPI == EPI_STATS || EPI == EPI_STATSZ) {
        const int u = r < a.M ? __ldg(a.tidx + a.row0 + r) : -1;
        const __nv_bfloat16* yrow = static_cast<const __nv_bfloat16*>(a.y) + static_cast<int64_t>(u < 0 ? 0 : u) * a.V;
        float mz = -INFINITY, sz = 0.f, my = -INFINITY, sy = 0.f, ac = 0.f;
        for (int c = 0; c < kBN / 32; ++c) {
          const int col0 = n0 + 32 * c;
          if (col0 >= a.N) break;  // warp-uniform
          uint32_t v[32];
          __syncwarp();
          tmem_ld32(tacc + 32 * c, v);
          tmem_ld_wait();
          reg_fence32(v);
          if (EPI == EPI_STATSZ) {
            // the fp32 logits of this row out through a swizzled slab and a TMA store
            uint8_t* slab = slabs + (nslab & 1) * kSlab;
            if (lane == 0) bulk_wait_read1();
            __syncwarp();
            uint8_t* rowp = slab + lane * 128;
#pragma unroll
            for (int k = 0; k < 8; ++k)
              *reinterpret_cast<uint4*>(rowp + ((k ^ (lane & 7)) << 4)) =
                  make_uint4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&map_out, slab, col0, m0 + 32 * q);
              bulk_commit();
            }
            ++nslab;
          }
          if (u >= 0) stats_update(v, col0, a.V, yrow, mz, sz, my, sy, ac);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty + b);
        if (r < a.M) {
          float* st = a.stats + (static_cast<int64_t>(n) * 5) * a.R + a.row0 + r;
          st[0] = mz;
          st[a.R] = sz;
          st[2 * static_cast<int64_t>(a.R)] = my;
          st[3 * static_cast<int64_t>(a.R)] = sy;
          st[4 * static_cast<int64_t>(a.R)] = ac;
        }
      } else if (EPI == EPI_DZ || EPI == EPI_BF16) {
        float cf = 0.f, lz = 0.f, ly = 0.f;
        const __nv_bfloat16* yrow = static_cast<const __nv_bfloat16*>(a.y);
        if (EPI == EPI_DZ && r < a.M) {
          const int u = __ldg(a.tidx + a.row0 + r);
          if (u >= 0) {
            cf = __ldg(a.coef + a.row0 + r);
            lz = __ldg(a.lse + a.row0 + r) * kLog2e;
            ly = __ldg(a.lse + a.R + a.row0 + r) * kLog2e;
            yrow = static_cast<const __nv_bfloat16*>(a.y) + static_cast<int64_t>(u) * a.V;
          }
        }
        for (int c2 = 0; c2 < kBN / 64; ++c2) {
          const int col0 = n0 + 64 * c2;
          if (col0 >= a.N) break;  // warp-uniform
          uint8_t* slab = slabs + (nslab & 1) * kSlab;
          // the store that last read this slab (two slabs ago) has finished reading it
          if (lane == 0) bulk_wait_read1();
          __syncwarp();
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t v[32];
            __syncwarp();
            tmem_ld32(tacc + 64 * c2 + 32 * h, v);
            tmem_ld_wait();
            reg_fence32(v);
            uint32_t pk[16];
            if (EPI == EPI_DZ) {
              if (cf != 0.f) {
#pragma unroll
                for (int g8 = 0; g8 < 4; ++g8) {
                  float y8[8];
                  load_y8(yrow, col0 + 32 * h + 8 * g8, a.V, y8);
#pragma unroll
                  for (int i = 0; i < 8; i += 2) {
                    const int j = 8 * g8 + i;
                    const float p0 = exp2_approx(fmaf(__uint_as_float(v[j]), kLog2e, -lz));
                    const float p1 = exp2_approx(fmaf(__uint_as_float(v[j + 1]), kLog2e, -lz));
                    const float q0 = exp2_approx(fmaf(y8[i], kLog2e, -ly));
                    const float q1 = exp2_approx(fmaf(y8[i + 1], kLog2e, -ly));
                    pk[j >> 1] = pack_bf16x2(cf * (p0 - q0), cf * (p1 - q1));
                  }
                }
              } else {
#pragma unroll
                for (int j = 0; j < 16; ++j) pk[j] = 0u;
              }
            } else {
#pragma unroll
              for (int j = 0; j < 16; ++j) pk[j] = pack_bf16x2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
            }
            // 128-byte swizzle: 16-byte unit k of row `lane` sits at unit k ^ (lane & 7)
            uint8_t* rowp = slab + lane * 128;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int unit = 4 * h + k;
              *reinterpret_cast<uint4*>(rowp + ((unit ^ (lane & 7)) << 4)) =
                  make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&map_out, slab, col0, m0 + 32 * q);
            bulk_commit();
          }
          ++nslab;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty + b);
      } else {
        // EPI_ACC: 32 fp32 columns per slab, reduce-added into the fp32 output
        for (int c = 0; c < kBN / 32; ++c) {
          const int col0 = n0 + 32 * c;
          if (col0 >= a.N) break;  // warp-uniform
          uint8_t* slab = slabs + (nslab & 1) * kSlab;
          if (lane == 0) bulk_wait_read1();
          __syncwarp();
          uint32_t v[32];
          tmem_ld32(tacc + 32 * c, v);
          tmem_ld_wait();
          reg_fence32(v);
          uint8_t* rowp = slab + lane * 128;
#pragma unroll
          for (int k = 0; k < 8; ++k)
            *reinterpret_cast<uint4*>(rowp + ((k ^ (lane & 7)) << 4)) =
                make_uint4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_reduce_add_2d(&map_out, slab, col0, m0 + 32 * q);
            bulk_commit();
          }
          ++nslab;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty + b);
      }
    }
    if (lane == 0) bulk_wait0();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// Teacher row of every draft row of pass p = blockIdx.x, the pass's count N_p and, for
// the backward, each row's gradient coefficient grad * w_p / N_p (0 if invalid).
__global__ void __launch_bounds__(1024) softce_rows_kernel(int P, int T, const int32_t* cu, int nseq,
                                                           const uint8_t* mask, const float* pass_weight,
                                                           const float* pass_count, float grad, int32_t* tidx,
                                                           float* counts, float* coef) {
  __shared__ int warp_cnt[32];
  __shared__ float s_coef;
  const int p = blockIdx.x;
  int cnt = 0;
  for (int t = threadIdx.x; t < T; t += blockDim.x) {
    int end;
    if (cu) {
      int lo = 0, hi = nseq - 1;  // last sequence whose start is <= t
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(cu + mid) <= t)
          lo = mid;
        else
          hi = mid - 1;
      }
      end = __ldg(cu + lo + 1);
    } else {
      const int S = nseq > 1 ? T / nseq : T;
      end = (t / S + 1) * S;
    }
    const int u = t + p;
    const bool valid = u < end && u < T && (!mask || __ldg(mask + u) != 0);
    tidx[static_cast<int64_t>(p) * T + t] = valid ? u : -1;
    cnt += valid ? 1 : 0;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if ((threadIdx.x & 31) == 0) warp_cnt[threadIdx.x >> 5] = cnt;
  __syncthreads();
  if (threadIdx.x == 0) {
    int total = 0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) total += warp_cnt[w];
    const float n = pass_count ? pass_count[p] : static_cast<float>(total);
    counts[p] = n;
    const float w = pass_weight ? pass_weight[p] : 1.f;
    s_coef = n > 0.f ? grad * w / n : 0.f;
  }
  __syncthreads();
  if (coef) {
    const float c = s_coef;
    for (int t = threadIdx.x; t < T; t += blockDim.x) {
      const int64_t i = static_cast<int64_t>(p) * T + t;
      coef[i] = tidx[i] >= 0 ? c : 0.f;
    }
  }
}

// General form, step 1: the teacher position of every draft row (or -1) and the valid
// rows per group (int atomics: exact and order-free).
__global__ void __launch_bounds__(256) softce_rows_general_kernel(int R, int Ty, int G, const int32_t* row_teacher,
                                                                  const int32_t* row_group, const uint8_t* mask,
                                                                  int32_t* tidx, int* icount) {
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= R) return;
  const int u = row_teacher[r];
  const int g = row_group ? row_group[r] : 0;
  const bool valid = u >= 0 && u < Ty && g >= 0 && g < G && (!mask || __ldg(mask + u) != 0);
  tidx[r] = valid ? u : -1;
  if (valid) atomicAdd(icount + g, 1);
}

// General form, step 2: N_g (given or counted) and each row's coefficient g * w_g / N_g.
__global__ void __launch_bounds__(256) softce_coef_general_kernel(int R, int G, const int32_t* row_group,
                                                                  const int32_t* tidx, const int* icount,
                                                                  const float* weight, const float* given,
                                                                  float grad, float* counts, float* coef) {
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r < G) counts[r] = given ? given[r] : static_cast<float>(icount[r]);
  if (!coef || r >= R) return;
  if (tidx[r] < 0) {
    coef[r] = 0.f;
    return;
  }
  const int g = row_group ? row_group[r] : 0;
  const float n = given ? given[g] : static_cast<float>(icount[g]);
  const float w = weight ? weight[g] : 1.f;
  coef[r] = n > 0.f ? grad * w / n : 0.f;
}

// Merge of the per-tile statistics of every row: lse of the draft logits and of the
// teacher row, and the loss l = lse_z - (sum_v e^(y_v - M) z_v) / (sum_v e^(y_v - M)).
// A block takes 32 rows (threadIdx.x, so that every tile's 32 values are one coalesced
// load) and kCombineSlices threads per row that merge interleaved tiles, then one
// thread per row merges their results.
constexpr int kCombineSlices = 16;

__device__ __forceinline__ void merge_stats(float& Mz, float& Sz, float& My, float& Sy, float& A, float mz, float sz,
                                            float my, float sy, float ac) {
  const float nz = fmaxf(Mz, mz);
  if (nz != -INFINITY) {
    Sz = Sz * exp2f(Mz - nz) + sz * exp2f(mz - nz);
    Mz = nz;
  }
  const float ny = fmaxf(My, my);
  if (ny != -INFINITY) {
    const float f0 = exp2f(My - ny), f1 = exp2f(my - ny);
    Sy = Sy * f0 + sy * f1;
    A = A * f0 + ac * f1;
    My = ny;
  }
}

__global__ void __launch_bounds__(32 * kCombineSlices) softce_combine_kernel(int R, int ntn, int r0, int nrows,
                                                                             const int32_t* tidx, const float* stats,
                                                                             float* row_loss, float* lse) {
  __shared__ float part[5][kCombineSlices][33];
  const int i = blockIdx.x * 32 + threadIdx.x;
  const int r = r0 + i;
  const bool live = i < nrows && tidx[r] >= 0;
  float Mz = -INFINITY, Sz = 0.f, My = -INFINITY, Sy = 0.f, A = 0.f;
  if (live) {
    for (int n = threadIdx.y; n < ntn; n += kCombineSlices) {
      const float* st = stats + static_cast<int64_t>(n) * 5 * R + r;
      merge_stats(Mz, Sz, My, Sy, A, st[0], st[R], st[2 * static_cast<int64_t>(R)], st[3 * static_cast<int64_t>(R)],
                  st[4 * static_cast<int64_t>(R)]);
    }
  }
  part[0][threadIdx.y][threadIdx.x] = Mz;
  part[1][threadIdx.y][threadIdx.x] = Sz;
  part[2][threadIdx.y][threadIdx.x] = My;
  part[3][threadIdx.y][threadIdx.x] = Sy;
  part[4][threadIdx.y][threadIdx.x] = A;
  __syncthreads();
  if (threadIdx.y != 0 || i >= nrows) return;
  if (!live) {
    row_loss[r] = 0.f;
    lse[r] = 0.f;
    lse[static_cast<int64_t>(R) + r] = 0.f;
    return;
  }
  for (int k = 1; k < kCombineSlices; ++k)
    merge_stats(Mz, Sz, My, Sy, A, part[0][k][threadIdx.x], part[1][k][threadIdx.x], part[2][k][threadIdx.x],
                part[3][k][threadIdx.x], part[4][k][threadIdx.x]);
  constexpr float kLn2 = 0.6931471805599453f;
  const float lz = (Mz + log2f(Sz)) * kLn2;
  const float ly = (My + log2f(Sy)) * kLn2;
  row_loss[r] = lz - A / Sy;
  lse[r] = lz;
  lse[static_cast<int64_t>(R) + r] = ly;
}

// dz of rows r0 .. r0+nrows from their stored fp32 logits (fused call): one warp per row,
// four columns per lane and step; dz = c_r (2^(z log2e - lse_z log2e) - 2^(y log2e -
// lse_y log2e)) rounded to bf16, the same expression as the DZ epilogue (0 for a row with
// c_r = 0).  z and dz rows are ldz elements apart.
__global__ void __launch_bounds__(256) softce_dz_kernel(int R, int V, int ldz, int r0, int nrows,
                                                        const int32_t* tidx, const float* coef, const float* lse,
                                                        const __nv_bfloat16* y, const float* z, __nv_bfloat16* dz) {
  const int i = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (i >= nrows) return;
  const int r = r0 + i;
  const int u = tidx[r];
  const float cf = u >= 0 ? coef[r] : 0.f;
  uint2* out = reinterpret_cast<uint2*>(dz + static_cast<int64_t>(i) * ldz);
  if (cf == 0.f) {
    for (int c4 = lane; c4 < V / 4; c4 += 32) out[c4] = make_uint2(0u, 0u);
    return;
  }
  const float lz = lse[r] * kLog2e, ly = lse[static_cast<int64_t>(R) + r] * kLog2e;
  const float4* zr = reinterpret_cast<const float4*>(z + static_cast<int64_t>(i) * ldz);
  const uint2* yr = reinterpret_cast<const uint2*>(y + static_cast<int64_t>(u) * V);
#pragma unroll 4
  for (int c4 = lane; c4 < V / 4; c4 += 32) {
    const float4 zz = __ldcs(zr + c4);
    const uint2 yy = __ldg(yr + c4);
    const float zs[4] = {zz.x, zz.y, zz.z, zz.w};
    const float ys[4] = {__uint_as_float(yy.x << 16), __uint_as_float(yy.x & 0xFFFF0000u),
                         __uint_as_float(yy.y << 16), __uint_as_float(yy.y & 0xFFFF0000u)};
    float d[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      d[k] = cf * (exp2_approx(fmaf(zs[k], kLog2e, -lz)) - exp2_approx(fmaf(ys[k], kLog2e, -ly)));
    out[c4] = make_uint2(pack_bf16x2(d[0], d[1]), pack_bf16x2(d[2], d[3]));
  }
}

// Per-group sums in a fixed order: L_g = w_g / N_g * sum of the group's row losses, then
// L.  The TTT passes are the groups of T consecutive rows; in the general form (group
// array given, or `general` with every row in group 0) the rows of a group are gathered
// by a filtered pass over all R rows.
__global__ void __launch_bounds__(1024) softce_finalize_kernel(int P, int T, const float* row_loss,
                                                               const float* counts, const float* pass_weight,
                                                               float* loss, int R = 0, bool general = false,
                                                               const int32_t* row_group = nullptr) {
  __shared__ double part[32];
  double total = 0.0;
  for (int p = 0; p < P; ++p) {
    double s = 0.0;
    if (!general) {
      for (int t = threadIdx.x; t < T; t += blockDim.x) s += row_loss[static_cast<int64_t>(p) * T + t];
    } else {
      for (int r = threadIdx.x; r < R; r += blockDim.x)
        if ((row_group ? row_group[r] : 0) == p) s += row_loss[r];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
      double sum = 0.0;
      for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) sum += part[w];
      const float n = counts[p];
      const double w = pass_weight ? pass_weight[p] : 1.0;
      const double lp = n > 0.f ? w * sum / n : 0.0;
      loss[p] = static_cast<float>(lp);
      total += lp;
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) loss[P] = static_cast<float>(total);
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) !=
                                                 cudaSuccess)
    return 148;
  return n > 0 ? n : 148;
}

template <int EPI>
cudaError_t launch_gemm(const SoftceGemmArgs& a, const CUtensorMap& ma, const CUtensorMap& mb,
                        const CUtensorMap& mo, cudaStream_t stream) {
  const long long tiles =
      static_cast<long long>((a.M + kBM - 1) / kBM) * static_cast<long long>((a.N + kBN - 1) / kBN);
  if (tiles <= 0 || a.K <= 0) return cudaSuccess;
  if (tiles > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
  cudaError_t e = cudaFuncSetAttribute(softce_gemm_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmemBytes);
  if (e != cudaSuccess) return e;
  const int grid = static_cast<int>(tiles < sm_count() ? tiles : sm_count());
  softce_gemm_kernel<EPI><<<grid, kThreads, kSmemBytes, stream>>>(ma, mb, mo, a);
  return cudaGetLastError();
}

struct CePlan {
  int P, T, d, V, R, ntn, C, Vp;
  bool general;  // explicit teacher positions and groups (row_teacher)
  int G, Ty;     // normalisation groups, teacher rows
  size_t off_tidx, off_counts, off_coef, off_stats, off_z, off_dz, total;
};

constexpr size_t kCeAlign = 1024;
inline size_t ce_align(size_t x) { return (x + kCeAlign - 1) / kCeAlign * kCeAlign; }

// mode 0: forward, 1: backward, 2: the fused forward + backward
ttt_status ce_plan(const ttt_softce_desc* d, int mode, CePlan* out) {
  if (!d || mode < 0 || mode > 2) return TTT_ERR_INVALID_ARG;
  if (d->P < 1 || d->T < 0 || d->d < 8 || d->V < 8) return TTT_ERR_INVALID_ARG;
  // the TMA boxes are 64 hidden columns and 256 vocabulary rows: smaller tensors are not taken
  if (d->d % 8 != 0 || d->V % 8 != 0 || d->d < 64 || d->V < 256) return TTT_ERR_UNSUPPORTED;
  if (d->token_chunk_size < 0) return TTT_ERR_INVALID_ARG;
  const bool general = d->row_teacher != nullptr;
  if (general) {
    if (d->ngroups < 1 || d->teacher_rows < 0) return TTT_ERR_INVALID_ARG;
    if (d->ngroups > 1 && !d->row_group) return TTT_ERR_INVALID_ARG;
  } else {
    if (d->nseq < 0) return TTT_ERR_INVALID_ARG;
    if (d->cu_seqlens && d->nseq < 1) return TTT_ERR_INVALID_ARG;
    if (!d->cu_seqlens && d->nseq > 1 && d->T % d->nseq != 0) return TTT_ERR_INVALID_ARG;
  }
  const long long R = static_cast<long long>(d->P) * d->T;
  if (R >= (1LL << 31)) return TTT_ERR_UNSUPPORTED;
  CePlan pl{};
  pl.P = d->P;
  pl.T = d->T;
  pl.d = d->d;
  pl.V = d->V;
  pl.R = static_cast<int>(R);
  pl.general = general;
  pl.G = general ? d->ngroups : d->P;
  pl.Ty = general ? d->teacher_rows : d->T;
  pl.ntn = (d->V + kBN - 1) / kBN;
  const int chunk = d->token_chunk_size > 0 ? d->token_chunk_size : 4096;
  pl.C = static_cast<int>(R < chunk ? (R > 0 ? R : 1) : chunk);
  pl.Vp = (d->V + 63) / 64 * 64;
  pl.off_tidx = kCeAlign;  // the status word lives in the first block
  pl.off_counts = ce_align(pl.off_tidx + static_cast<size_t>(pl.R) * 4);
  // N_g as floats, then the int counts of the general form
  const size_t after_counts = ce_align(pl.off_counts + static_cast<size_t>(pl.G) * 8);
  const size_t stats_bytes = static_cast<size_t>(pl.ntn) * 5 * pl.R * 4;
  if (mode == 0) {
    pl.off_stats = after_counts;
    pl.total = pl.off_stats + stats_bytes;
  } else if (mode == 1) {
    pl.off_coef = after_counts;
    pl.off_dz = ce_align(pl.off_coef + static_cast<size_t>(pl.R) * 4);
    pl.total = pl.off_dz + static_cast<size_t>(pl.C) * pl.Vp * 2;
  } else {
    pl.off_coef = after_counts;
    pl.off_stats = ce_align(pl.off_coef + static_cast<size_t>(pl.R) * 4);
    pl.off_z = ce_align(pl.off_stats + stats_bytes);
    pl.off_dz = ce_align(pl.off_z + static_cast<size_t>(pl.C) * pl.Vp * 4);
    pl.total = pl.off_dz + static_cast<size_t>(pl.C) * pl.Vp * 2;
  }
  *out = pl;
  return TTT_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

struct CeEvents {
  const ttt_attn_events* ev;
  int k;
  cudaStream_t s;
  bool on;
  CeEvents(const ttt_attn_events* e, int kk, cudaStream_t st, bool enabled = true) : ev(e), k(kk), s(st), on(enabled) {
    if (on && ev && ev->start[k]) cudaEventRecord(static_cast<cudaEvent_t>(ev->start[k]), s);
  }
  ~CeEvents() {
    if (on && ev && ev->stop[k]) cudaEventRecord(static_cast<cudaEvent_t>(ev->stop[k]), s);
  }
};

#define CE_CHECK(expr)                          \
  do {                                          \
    const cudaError_t e_ = (expr);              \
    if (e_ != cudaSuccess) {                    \
      record_cuda_error(static_cast<int>(e_));  \
      return TTT_ERR_CUDA;                      \
    }                                           \
  } while (0)

constexpr CUtensorMapDataType kBf16 = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
constexpr CUtensorMapSwizzle kSw128 = CU_TENSOR_MAP_SWIZZLE_128B;

// Teacher rows, N_g and (coef non-NULL) the rows' gradient coefficients, for either form.
ttt_status launch_rows(const ttt_softce_desc* d, const CePlan& pl, float grad, uint8_t* ws, int32_t* tidx,
                       float* counts, float* coef, cudaStream_t stream) {
  CeEvents ev(d->events, TTT_SOFTCE_KERNEL_ROWS, stream);
  if (!pl.general) {
    softce_rows_kernel<<<pl.P, 1024, 0, stream>>>(pl.P, pl.T, d->cu_seqlens, d->nseq, d->loss_mask, d->pass_weight,
                                                 d->pass_count, grad, tidx, counts, coef);
    CE_CHECK(cudaGetLastError());
    return TTT_OK;
  }
  int* icount = reinterpret_cast<int*>(counts + pl.G);
  CE_CHECK(cudaMemsetAsync(icount, 0, sizeof(int) * pl.G, stream));
  softce_rows_general_kernel<<<(pl.R + 255) / 256, 256, 0, stream>>>(pl.R, pl.Ty, pl.G, d->row_teacher, d->row_group,
                                                                      d->loss_mask, tidx, icount);
  CE_CHECK(cudaGetLastError());
  const int n = pl.R > pl.G ? pl.R : pl.G;
  softce_coef_general_kernel<<<(n + 255) / 256, 256, 0, stream>>>(pl.R, pl.G, d->row_group, tidx, icount,
                                                                  d->pass_weight, d->pass_count, grad, counts, coef);
  CE_CHECK(cudaGetLastError());
  (void)ws;
  return TTT_OK;
}

}  // namespace
}  // namespace ttt

using namespace ttt;

extern "C" {

size_t ttt_softce_workspace_size(const ttt_softce_desc* desc, int for_backward) {
  CePlan pl;
  if (ce_plan(desc, for_backward, &pl) != TTT_OK) return 0;
  return pl.total;
}

ttt_status ttt_softce_fwd(const ttt_softce_desc* desc, const void* h, const void* W, const void* y,
                          float* row_loss, float* lse, float* loss, void* workspace, size_t workspace_bytes,
                          void* stream_) {
  CePlan pl;
  const ttt_status st = ce_plan(desc, 0, &pl);
  if (st != TTT_OK) return st;
  if (!loss) return TTT_ERR_INVALID_ARG;
  if (pl.R > 0 && (!h || !W || !y || !row_loss || !lse)) return TTT_ERR_INVALID_ARG;
  if (pl.R > 0 && (!aligned16(h) || !aligned16(W) || !aligned16(y))) return TTT_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < pl.total || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return TTT_ERR_WORKSPACE;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  CE_CHECK(cudaMemsetAsync(status, 0, sizeof(uint32_t), stream));
  if (pl.R == 0) {
    CE_CHECK(cudaMemsetAsync(loss, 0, sizeof(float) * (pl.G + 1), stream));
    return TTT_OK;
  }
  int32_t* tidx = reinterpret_cast<int32_t*>(ws + pl.off_tidx);
  float* counts = reinterpret_cast<float*>(ws + pl.off_counts);
  float* stats = reinterpret_cast<float*>(ws + pl.off_stats);
  {
    const ttt_status sr = launch_rows(desc, pl, 1.f, ws, tidx, counts, nullptr, stream);
    if (sr != TTT_OK) return sr;
  }
  CUtensorMap mh, mw;
  if (!encode_map_2d(&mh, kBf16, h, pl.d, pl.R, static_cast<uint64_t>(pl.d) * 2, 64, 128, kSw128) ||
      !encode_map_2d(&mw, kBf16, W, pl.d, pl.V, static_cast<uint64_t>(pl.d) * 2, 64, 256, kSw128))
    return TTT_ERR_CUDA;
  SoftceGemmArgs a{};
  a.M = pl.R;
  a.N = pl.V;
  a.K = pl.d;
  a.row0 = 0;
  a.R = pl.R;
  a.V = pl.V;
  a.tidx = tidx;
  a.y = y;
  a.stats = stats;
  a.status = status;
  a.budget_ns = wait_budget_ns();
  {
    CeEvents ev(desc->events, TTT_SOFTCE_KERNEL_LOGITS, stream);
    CE_CHECK(launch_gemm<EPI_STATS>(a, mh, mw, mh, stream));
  }
  {
    CeEvents ev(desc->events, TTT_SOFTCE_KERNEL_REDUCE, stream);
    softce_combine_kernel<<<(pl.R + 31) / 32, dim3(32, kCombineSlices), 0, stream>>>(pl.R, pl.ntn, 0, pl.R, tidx,
                                                                                      stats, row_loss, lse);
    CE_CHECK(cudaGetLastError());
    softce_finalize_kernel<<<1, 1024, 0, stream>>>(pl.G, pl.T, row_loss, counts, desc->pass_weight, loss, pl.R,
                                                   pl.general, desc->row_group);
    CE_CHECK(cudaGetLastError());
  }
  return TTT_OK;
}

ttt_status ttt_softce_bwd(const ttt_softce_desc* desc, const void* h, const void* W, const void* y,
                          const float* lse, float grad, void* dh, float* dW, void* workspace,
                          size_t workspace_bytes, void* stream_) {
  CePlan pl;
  const ttt_status st = ce_plan(desc, 1, &pl);
  if (st != TTT_OK) return st;
  if (pl.R > 0 && (!h || !W || !y || !lse || !dh)) return TTT_ERR_INVALID_ARG;
  if (pl.R > 0 && (!aligned16(h) || !aligned16(W) || !aligned16(y) || !aligned16(dh) || (dW && !aligned16(dW))))
    return TTT_ERR_INVALID_ARG;
  if (!std::isfinite(grad)) return TTT_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < pl.total || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return TTT_ERR_WORKSPACE;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  CE_CHECK(cudaMemsetAsync(status, 0, sizeof(uint32_t), stream));
  if (pl.R == 0) return TTT_OK;
  int32_t* tidx = reinterpret_cast<int32_t*>(ws + pl.off_tidx);
  float* counts = reinterpret_cast<float*>(ws + pl.off_counts);
  float* coef = reinterpret_cast<float*>(ws + pl.off_coef);
  uint8_t* dz = ws + pl.off_dz;
  {
    const ttt_status sr = launch_rows(desc, pl, grad, ws, tidx, counts, coef, stream);
    if (sr != TTT_OK) return sr;
  }
  const uint64_t hrow = static_cast<uint64_t>(pl.d) * 2, zrow = static_cast<uint64_t>(pl.Vp) * 2;
  CUtensorMap mh, mw_k, mw_mn, mdw;
  if (!encode_map_2d(&mh, kBf16, h, pl.d, pl.R, hrow, 64, 128, kSw128) ||
      !encode_map_2d(&mw_k, kBf16, W, pl.d, pl.V, hrow, 64, 256, kSw128) ||
      !encode_map_2d(&mw_mn, kBf16, W, pl.d, pl.V, hrow, 64, 64, kSw128))
    return TTT_ERR_CUDA;
  if (dW && !encode_map_2d(&mdw, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, dW, pl.d, pl.V, static_cast<uint64_t>(pl.d) * 4,
                           32, 32, kSw128))
    return TTT_ERR_CUDA;
  SoftceGemmArgs base{};
  base.R = pl.R;
  base.V = pl.V;
  base.tidx = tidx;
  base.y = y;
  base.lse = lse;
  base.coef = coef;
  base.status = status;
  base.budget_ns = wait_budget_ns();
  for (int r0 = 0; r0 < pl.R; r0 += pl.C) {
    const int c = pl.R - r0 < pl.C ? pl.R - r0 : pl.C;
    const bool first = r0 == 0;
    const uint8_t* hc = static_cast<const uint8_t*>(h) + static_cast<size_t>(r0) * hrow;
    uint8_t* dhc = static_cast<uint8_t*>(dh) + static_cast<size_t>(r0) * hrow;
    CUtensorMap mz_out, mz_k, mz_mn, mdh, mh_mn;
    if (!encode_map_2d(&mz_out, kBf16, dz, pl.V, c, zrow, 64, 32, kSw128) ||
        !encode_map_2d(&mz_k, kBf16, dz, pl.V, c, zrow, 64, 128, kSw128) ||
        !encode_map_2d(&mz_mn, kBf16, dz, pl.V, c, zrow, 64, 64, kSw128) ||
        !encode_map_2d(&mdh, kBf16, dhc, pl.d, c, hrow, 64, 32, kSw128) ||
        !encode_map_2d(&mh_mn, kBf16, hc, pl.d, c, hrow, 64, 64, kSw128))
      return TTT_ERR_CUDA;
    {
      CeEvents ev(desc->events, TTT_SOFTCE_KERNEL_DZ, stream, first);
      SoftceGemmArgs a = base;
      a.M = c;
      a.N = pl.V;
      a.K = pl.d;
      a.row0 = r0;
      CE_CHECK(launch_gemm<EPI_DZ>(a, mh, mw_k, mz_out, stream));
    }
    {
      CeEvents ev(desc->events, TTT_SOFTCE_KERNEL_DH, stream, first);
      SoftceGemmArgs a = base;
      a.M = c;
      a.N = pl.d;
      a.K = pl.V;
      CE_CHECK(launch_gemm<EPI_BF16>(a, mz_k, mw_mn, mdh, stream));
    }
    if (dW) {
      CeEvents ev(desc->events, TTT_SOFTCE_KERNEL_DW, stream, first);
      SoftceGemmArgs a = base;
      a.M = pl.V;
      a.N = pl.d;
      a.K = c;
      CE_CHECK(launch_gemm<EPI_ACC>(a, mz_mn, mh_mn, mdw, stream));
    }
  }
  return TTT_OK;
}

ttt_status ttt_softce_fwd_bwd(const ttt_softce_desc* desc, const void* h, const void* W, const void* y, float grad,
                              float* row_loss, float* lse, float* loss, void* dh, float* dW, void* workspace,
                              size_t workspace_bytes, void* stream_) {
  CePlan pl;
  const ttt_status st = ce_plan(desc, 2, &pl);
  if (st != TTT_OK) return st;
  if (!loss) return TTT_ERR_INVALID_ARG;
  if (pl.R > 0 && (!h || !W || !y || !row_loss || !lse || !dh)) return TTT_ERR_INVALID_ARG;
  if (pl.R > 0 && (!aligned16(h) || !aligned16(W) || !aligned16(y) || !aligned16(dh) || (dW && !aligned16(dW))))
    return TTT_ERR_INVALID_ARG;
  if (!std::isfinite(grad)) return TTT_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < pl.total || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return TTT_ERR_WORKSPACE;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  CE_CHECK(cudaMemsetAsync(status, 0, sizeof(uint32_t), stream));
  if (pl.R == 0) {
    CE_CHECK(cudaMemsetAsync(loss, 0, sizeof(float) * (pl.G + 1), stream));
    return TTT_OK;
  }
  int32_t* tidx = reinterpret_cast<int32_t*>(ws + pl.off_tidx);
  float* counts = reinterpret_cast<float*>(ws + pl.off_counts);
  float* coef = reinterpret_cast<float*>(ws + pl.off_coef);
  float* stats = reinterpret_cast<float*>(ws + pl.off_stats);
  float* zbuf = reinterpret_cast<float*>(ws + pl.off_z);
  uint8_t* dz = ws + pl.off_dz;
  {
    const ttt_status sr = launch_rows(desc, pl, grad, ws, tidx, counts, coef, stream);
    if (sr != TTT_OK) return sr;
  }
  const uint64_t hrow = static_cast<uint64_t>(pl.d) * 2, zrow = static_cast<uint64_t>(pl.Vp) * 2;
  CUtensorMap mh, mw_k, mw_mn, mdw;
  if (!encode_map_2d(&mh, kBf16, h, pl.d, pl.R, hrow, 64, 128, kSw128) ||
      !encode_map_2d(&mw_k, kBf16, W, pl.d, pl.V, hrow, 64, 256, kSw128) ||
      !encode_map_2d(&mw_mn, kBf16, W, pl.d, pl.V, hrow, 64, 64, kSw128))
    return TTT_ERR_CUDA;
  if (dW && !encode_map_2d(&mdw, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, dW, pl.d, pl.V, static_cast<uint64_t>(pl.d) * 4,
                           32, 32, kSw128))
    return TTT_ERR_CUDA;
  SoftceGemmArgs base{};
  base.R = pl.R;
  base.V = pl.V;
  base.tidx = tidx;
  base.y = y;
  base.stats = stats;
  base.status = status;
  base.budget_ns = wait_budget_ns();
  for (int r0 = 0; r0 < pl.R; r0 += pl.C) {
    const int c = pl.R - r0 < pl.C ? pl.R - r0 : pl.C;
    const bool first = r0 == 0;
    const uint8_t* hc = static_cast<const uint8_t*>(h) + static_cast<size_t>(r0) * hrow;
    uint8_t* dhc = static_cast<uint8_t*>(dh) + static_cast<size_t>(r0) * hrow;
    CUtensorMap mz_out, mz_k, mz_mn, mdh, mh_mn;
    if (!encode_map_2d(&mz_out, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, zbuf, pl.V, c, static_cast<uint64_t>(pl.Vp) * 4, 32,
                       32, kSw128) ||
        !encode_map_2d(&mz_k, kBf16, dz, pl.V, c, zrow, 64, 128, kSw128) ||
        !encode_map_2d(&mz_mn, kBf16, dz, pl.V, c, zrow, 64, 64, kSw128) ||
        !encode_map_2d(&mdh, kBf16, dhc, pl.d, c, hrow, 64, 32, kSw128) ||
        !encode_map_2d(&mh_mn, kBf16, hc, pl.d, c, hrow, 64, 64, kSw128))
      return TTT_ERR_CUDA;
    {
      CeEvents ev(desc->events, TTT_SOFTCE_KERNEL_LOGITS, stream, first);
      SoftceGemmArgs a = base;
      a.M = c;
      a.N = pl.V;
      a.K = pl.d;
      a.row0 = r0;
      CE_CHECK(launch_gemm<EPI_STATSZ>(a, mh, mw_k, mz_out, stream));
    }
    {
      CeEvents ev(desc->events, TTT_SOFTCE_KERNEL_REDUCE, stream, first);
      softce_combine_kernel<<<(c + 31) / 32, dim3(32, kCombineSlices), 0, stream>>>(pl.R, pl.ntn, r0, c, tidx, stats,
                                                                                   row_loss, lse);
      CE_CHECK(cudaGetLastError());
    }
    {
      CeEvents ev(desc->events, TTT_SOFTCE_KERNEL_DZ, stream, first);
      softce_dz_kernel<<<(c + 7) / 8, 256, 0, stream>>>(pl.R, pl.V, pl.Vp, r0, c, tidx, coef, lse,
                                                        static_cast<const __nv_bfloat16*>(y), zbuf,
                                                        reinterpret_cast<__nv_bfloat16*>(dz));
      CE_CHECK(cudaGetLastError());
    }
    {
      CeEvents ev(desc->events, TTT_SOFTCE_KERNEL_DH, stream, first);
      SoftceGemmArgs a = base;
      a.M = c;
      a.N = pl.d;
      a.K = pl.V;
      CE_CHECK(launch_gemm<EPI_BF16>(a, mz_k, mw_mn, mdh, stream));
    }
    if (dW) {
      CeEvents ev(desc->events, TTT_SOFTCE_KERNEL_DW, stream, first);
      SoftceGemmArgs a = base;
      a.M = pl.V;
      a.N = pl.d;
      a.K = c;
      CE_CHECK(launch_gemm<EPI_ACC>(a, mz_mn, mh_mn, mdw, stream));
    }
  }
  softce_finalize_kernel<<<1, 1024, 0, stream>>>(pl.G, pl.T, row_loss, counts, desc->pass_weight, loss, pl.R,
                                                 pl.general, desc->row_group);
  CE_CHECK(cudaGetLastError());
  return TTT_OK;
}

}  // extern "C"
