// Branch half of the two-part attention and the exact joint-LSE merge (forward),
// the softmax-gradient preprocess, and the branch backward with the final inverse
// RoPE of every gradient.
//
// "DFlash/DSpark and EAGLE-3 TTT draft co-training ..." (NeMo-RL issue 3698),
// "What I'm working on", items 1 and 4 (trunk+branch, exact joint-LSE merge);
// "bounded multi-pass EAGLE-3 TTT provider" (NeMo-RL PR 3725), self-review
// (staircase: the query of pass p at position i sees the branch keys of passes
// 2..p at the same position i only).
//
// These are memory-bound kernels with <= P-1 keys per query: one warp per
// (position, KV head) row group, each lane holding D/32 elements of a row, dot
// products finished with warp shuffles.  No tensor cores.
#include <algorithm>

#include "common.cuh"

namespace ttt {

namespace {

constexpr int kWarpsPerBlock = 8;

// Lane element map: lane holds E = D/64 consecutive elements of each half of the
// head dimension, d in [E*lane, E*lane+E) and [D/2 + E*lane, ...), so that each
// RoPE pair (d, d + D/2) is in one lane.
template <int D>
struct LaneMap {
  static constexpr int E = D / 64;
  __device__ static int d(int lane, int half, int e) { return half * (D / 2) + E * lane + e; }
};

template <int D>
__device__ __forceinline__ void load_bf16_row(const __nv_bfloat16* row, int lane, float (&x)[2][D / 64]) {
  constexpr int E = D / 64;
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    if constexpr (E == 2) {
      const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(row + LaneMap<D>::d(lane, hh, 0));
      x[hh][0] = __low2float(v);
      x[hh][1] = __high2float(v);
    } else {
      x[hh][0] = __bfloat162float(row[LaneMap<D>::d(lane, hh, 0)]);
    }
  }
}

template <int D>
__device__ __forceinline__ void load_f32_row(const float* row, int lane, float (&x)[2][D / 64]) {
  constexpr int E = D / 64;
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    if constexpr (E == 2) {
      const float2 v = *reinterpret_cast<const float2*>(row + LaneMap<D>::d(lane, hh, 0));
      x[hh][0] = v.x;
      x[hh][1] = v.y;
    } else {
      x[hh][0] = row[LaneMap<D>::d(lane, hh, 0)];
    }
  }
}

template <int D>
__device__ __forceinline__ void store_bf16_row(__nv_bfloat16* row, int lane, const float (&x)[2][D / 64]) {
  constexpr int E = D / 64;
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    if constexpr (E == 2) {
      *reinterpret_cast<__nv_bfloat162*>(row + LaneMap<D>::d(lane, hh, 0)) = __floats2bfloat162_rn(x[hh][0], x[hh][1]);
    } else {
      row[LaneMap<D>::d(lane, hh, 0)] = __float2bfloat16_rn(x[hh][0]);
    }
  }
}

// x <- R(pos)^T x (rotation by the negative angle), in place.
template <int D>
__device__ __forceinline__ void rotate_back(float (&x)[2][D / 64], const float (&c)[D / 64], const float (&s)[D / 64]) {
#pragma unroll
  for (int e = 0; e < D / 64; ++e) {
    const float x1 = x[0][e], x2 = x[1][e];
    x[0][e] = fmaf(x1, c[e], x2 * s[e]);
    x[1][e] = fmaf(x2, c[e], -x1 * s[e]);
  }
}

// ---------------------------------------------------------------------------
// a5: delta = rowsum(dO * O), written with -lse * log2(e) into the tile-aligned
// row-statistics array that the trunk backward fetches one 512-byte slot at a time;
// the same pass zeroes the fp32 dq~ accumulator rows that the trunk backward
// reduces into.  One block per (pass, sequence, 64-token tile, head), head fastest
// so that neighbouring blocks read neighbouring rows of O and dO.  Memory bound:
// D/8 lanes per row, 16-byte loads, every row of a warp in flight at once.
// ---------------------------------------------------------------------------
constexpr int kPreRows = 64;
constexpr int kPreThreads = 256;

template <int D>
__global__ void __launch_bounds__(kPreThreads)
    bwd_preprocess_kernel(Geometry g, const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dout,
                          const float* __restrict__ lse, float* __restrict__ ld, float* __restrict__ dq_acc,
                          int* __restrict__ tickets, int ntile, int* __restrict__ qlim, uint32_t* status) {
  constexpr int LPR = D / 8;                            // lanes per row
  constexpr int RPI = 32 / LPR;                         // rows per warp instruction
  constexpr int RPWARP = kPreRows / (kPreThreads / 32);  // rows per warp (8)
  constexpr int NU = RPWARP / RPI;
  __shared__ float sdelta[kPreRows];
  const int h = static_cast<int>(blockIdx.x % g.H);
  int rest = static_cast<int>(blockIdx.x / g.H);
  const int tile = rest % ntile;
  rest /= ntile;
  const int n = rest % g.si.nseq;
  const int p = rest / g.si.nseq;
  int start, len;
  seq_bounds(g.si, n, start, len);
  const int pos0 = tile * kPreRows;
  if (pos0 >= len) return;
  const int nvalid = min(kPreRows, len - pos0);
  const int T = g.si.T;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane / LPR, c = lane % LPR;

  uint4 a[NU], b[NU];
#pragma unroll
  for (int u = 0; u < NU; ++u) {
    const int i = warp * RPWARP + u * RPI + sub;
    if (i < nvalid) {
      const int64_t row = p * g.sq + (static_cast<int64_t>(start + pos0 + i) * g.H + h) * D;
      a[u] = __ldg(reinterpret_cast<const uint4*>(o + row) + c);
      b[u] = __ldg(reinterpret_cast<const uint4*>(dout + row) + c);
    } else {
      a[u] = make_uint4(0, 0, 0, 0);
      b[u] = make_uint4(0, 0, 0, 0);
    }
  }
  // zero this tile's dq~ accumulator rows (contiguous: nvalid rows of D floats)
  float4* z = reinterpret_cast<float4*>(dq_acc + ((static_cast<int64_t>(p) * g.H + h) * T + start + pos0) * D);
  for (int i = threadIdx.x; i < nvalid * D / 4; i += kPreThreads) z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int u = 0; u < NU; ++u) {
    const __nv_bfloat162* x = reinterpret_cast<const __nv_bfloat162*>(&a[u]);
    const __nv_bfloat162* y = reinterpret_cast<const __nv_bfloat162*>(&b[u]);
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 fx = __bfloat1622float2(x[e]), fy = __bfloat1622float2(y[e]);
      acc = fmaf(fx.x, fy.x, fmaf(fx.y, fy.y, acc));
    }
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (c == 0) sdelta[warp * RPWARP + u * RPI + sub] = acc;
  }
  __syncthreads();
  const int64_t slot_index = (static_cast<int64_t>(p) * g.H + h) * ld_slots(g.si) + ld_slot(start, n, pos0);
  float* slot = ld + slot_index * 128;
  if (threadIdx.x == 0) tickets[slot_index] = 0;
  if (qlim && h == 0 && threadIdx.x < nvalid) {
    // block-draft rows: the trunk-key limit of each row (its block's clamped anchor), and
    // the anchors' order, which the trunk backward's tile walk relies on
    int kstart, klen;
    seq_bounds(g.ksi, n, kstart, klen);
    const int r = pos0 + threadIdx.x;
    qlim[start + r] = block_row_limit(g, start, r, klen);
    if (r % g.Bs == 0 && r >= g.Bs && g.anchors[(start + r) / g.Bs] < g.anchors[(start + r) / g.Bs - 1])
      atomicCAS(status, 0u, kStatusBadAnchors);
  }
  if (threadIdx.x < nvalid) {
    const int i = threadIdx.x;
    slot[i] = lse[lse_index(g.si, g.H, p, h, n, start + pos0 + i, pos0 + i)] * -1.4426950408889634f;
    slot[64 + i] = sdelta[i];
  }
}

// ---------------------------------------------------------------------------
// a7 + a8: branch backward and finalisation.  One warp per (token, KV head):
//   for every pass p and group head h:
//     dq~ = dq_acc (trunk part) + sum_j dS_j k~_j        (j = passes 1..p, 0-based)
//     dS_j = P_j (dO . V_j - delta),  P_j = exp(sigma q~ . k~_j - lse)
//     dk~_j += dS_j q~,  dV_j += P_j dO                   (accumulated over p >= j, h)
//     dQ_p = R(i+p)^T (sigma dq~)
//   dK_j = R(i+j)^T (sigma dk~_j) and dV_j for the branch passes j >= 1 (dK_1 and dV_1
//   are written by the trunk backward).
// The kernel is bound by memory latency, so resident warps matter most: the group
// heads of a pass go kBranchHeads at a time (one: more heads per warp keep more rows
// in flight but cost registers, and 64 registers at four blocks per SM measured
// fastest).  Shared memory: the block's inverse frequencies (double), then per warp
// the cos/sin of positions i..i+P-1 and the branch-pass accumulators.
// ---------------------------------------------------------------------------
constexpr int kBranchHeads = 1;

template <int D>
__global__ void __launch_bounds__(kWarpsPerBlock * 32, 4)
    branch_bwd_kernel(Geometry g, const __nv_bfloat16* __restrict__ qr, const __nv_bfloat16* __restrict__ kr,
                      const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ dout,
                      const float* __restrict__ lse, const float* __restrict__ ld,
                      const float* __restrict__ dq_acc,
                      __nv_bfloat16* __restrict__ dq, __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv) {
  constexpr int E = D / 64;
  extern __shared__ __align__(16) unsigned char branch_smem[];
  double* inv_freq = reinterpret_cast<double*>(branch_smem);  // [D/2]
  const int NB = g.P - 1;  // branch passes
  const int per_warp = g.P * D + (NB > 0 ? NB : 1) * 2 * D;  // floats: cos/sin [P][2][D/2], acc [NB][2][D]
  for (int d = threadIdx.x; d < D / 2; d += blockDim.x)
    inv_freq[d] = pow(static_cast<double>(g.theta), -2.0 * d / D);
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  const int64_t w = static_cast<int64_t>(blockIdx.x) * kWarpsPerBlock + wib;
  const int T = g.si.T;
  if (w >= static_cast<int64_t>(T) * g.Hkv) return;
  const int tau = static_cast<int>(w / g.Hkv);
  const int kvh = static_cast<int>(w % g.Hkv);
  int n, pos;
  token_position(g.si, tau, n, pos);
  const int gsz = g.H / g.Hkv;
  float* cs = reinterpret_cast<float*>(branch_smem + (D / 2) * sizeof(double)) + static_cast<int64_t>(wib) * per_warp;
  float* acc = cs + g.P * D;  // [NB][2 (dk, dv)][D]; a lane touches only its own elements
  for (int p = 0; p < g.P; ++p)
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int d = LaneMap<D>::d(lane, 0, e);
      angle_cos_sin(pos + p, inv_freq[d], cs[p * D + d], cs[p * D + D / 2 + d]);
    }
  for (int j = 0; j < NB; ++j)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh)
#pragma unroll
      for (int e = 0; e < E; ++e) {
        acc[(j * 2 + 0) * D + LaneMap<D>::d(lane, hh, e)] = 0.f;
        acc[(j * 2 + 1) * D + LaneMap<D>::d(lane, hh, e)] = 0.f;
      }
  const int64_t dl_base = static_cast<int64_t>(ld_slots(g.si)) * 128;
  const int64_t dl_off = static_cast<int64_t>(ld_slot(tau - pos, n, pos)) * 128 + 64 + (pos & 63);

  for (int p = 0; p < g.P; ++p) {
    float c[E], sn[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      c[e] = cs[p * D + LaneMap<D>::d(lane, 0, e)];
      sn[e] = cs[p * D + D / 2 + LaneMap<D>::d(lane, 0, e)];
    }
    for (int h0 = 0; h0 < gsz; h0 += kBranchHeads) {
      float dqv[kBranchHeads][2][E], q[kBranchHeads][2][E], dO[kBranchHeads][2][E];
      float lse_v[kBranchHeads], dl[kBranchHeads];
#pragma unroll
      for (int u = 0; u < kBranchHeads; ++u) {
        const int h = kvh * gsz + h0 + u;
        if (h0 + u < gsz) {
          const int64_t hrow = (static_cast<int64_t>(p) * g.H + h) * T + tau;
          load_f32_row<D>(dq_acc + hrow * D, lane, dqv[u]);
          if (p > 0) {
            load_bf16_row<D>(qr + hrow * D, lane, q[u]);
            load_bf16_row<D>(dout + p * g.sq + (static_cast<int64_t>(tau) * g.H + h) * D, lane, dO[u]);
            lse_v[u] = lse[lse_index(g.si, g.H, p, h, n, tau, pos)];
            dl[u] = ld[(static_cast<int64_t>(p) * g.H + h) * dl_base + dl_off];
          }
        }
      }
      for (int j = 1; j <= p; ++j) {
        float kj[2][E], vj[2][E];
        load_bf16_row<D>(kr + ((static_cast<int64_t>(j) * g.Hkv + kvh) * T + tau) * D, lane, kj);
        load_bf16_row<D>(v + j * g.skv + (static_cast<int64_t>(tau) * g.Hkv + kvh) * D, lane, vj);
        float sdot[kBranchHeads], tdot[kBranchHeads];
#pragma unroll
        for (int u = 0; u < kBranchHeads; ++u) {
          sdot[u] = 0.f;
          tdot[u] = 0.f;
#pragma unroll
          for (int hh = 0; hh < 2; ++hh)
#pragma unroll
            for (int e = 0; e < E; ++e) {
              sdot[u] = fmaf(q[u][hh][e], kj[hh][e], sdot[u]);
              tdot[u] = fmaf(dO[u][hh][e], vj[hh][e], tdot[u]);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
#pragma unroll
          for (int u = 0; u < kBranchHeads; ++u) {
            sdot[u] += __shfl_xor_sync(0xffffffffu, sdot[u], o);
            tdot[u] += __shfl_xor_sync(0xffffffffu, tdot[u], o);
          }
        float ak[2][E] = {}, av[2][E] = {};
#pragma unroll
        for (int u = 0; u < kBranchHeads; ++u) {
          if (h0 + u >= gsz) continue;
          const float pj = __expf(sdot[u] * g.scale - lse_v[u]);
          const float dsj = pj * (tdot[u] - dl[u]);
#pragma unroll
          for (int hh = 0; hh < 2; ++hh)
#pragma unroll
            for (int e = 0; e < E; ++e) {
              dqv[u][hh][e] = fmaf(dsj, kj[hh][e], dqv[u][hh][e]);
              ak[hh][e] = fmaf(dsj, q[u][hh][e], ak[hh][e]);
              av[hh][e] = fmaf(pj, dO[u][hh][e], av[hh][e]);
            }
        }
        float* akp = acc + ((j - 1) * 2 + 0) * D;
        float* avp = acc + ((j - 1) * 2 + 1) * D;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
#pragma unroll
          for (int e = 0; e < E; ++e) {
            const int d = LaneMap<D>::d(lane, hh, e);
            akp[d] += ak[hh][e];
            avp[d] += av[hh][e];
          }
      }
#pragma unroll
      for (int u = 0; u < kBranchHeads; ++u) {
        if (h0 + u >= gsz) continue;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
#pragma unroll
          for (int e = 0; e < E; ++e) dqv[u][hh][e] *= g.scale;
        rotate_back<D>(dqv[u], c, sn);
        store_bf16_row<D>(dq + p * g.sq + (static_cast<int64_t>(tau) * g.H + kvh * gsz + h0 + u) * D, lane, dqv[u]);
      }
    }
  }
  // dK and dV of the branch passes (those of the trunk pass come from the trunk backward)
  for (int j = 1; j < g.P; ++j) {
    float c[E], sn[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      c[e] = cs[j * D + LaneMap<D>::d(lane, 0, e)];
      sn[e] = cs[j * D + D / 2 + LaneMap<D>::d(lane, 0, e)];
    }
    float kx[2][E], vx[2][E];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh)
#pragma unroll
      for (int e = 0; e < E; ++e) {
        kx[hh][e] = acc[((j - 1) * 2 + 0) * D + LaneMap<D>::d(lane, hh, e)] * g.scale;
        vx[hh][e] = acc[((j - 1) * 2 + 1) * D + LaneMap<D>::d(lane, hh, e)];
      }
    rotate_back<D>(kx, c, sn);
    const int64_t krow = j * g.skv + (static_cast<int64_t>(tau) * g.Hkv + kvh) * D;
    store_bf16_row<D>(dk + krow, lane, kx);
    store_bf16_row<D>(dv + krow, lane, vx);
  }
}

// ---------------------------------------------------------------------------
// bounded-wait self-test: wait on a barrier that nothing completes
// ---------------------------------------------------------------------------
__global__ void watchdog_selftest_kernel(uint32_t* status, uint64_t budget_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const Watchdog wd{&abort_flag, status, budget_ns};
    wait_bounded(&bar, 0, wd, kSiteSelftest);
  }
  __syncthreads();
}

inline unsigned blocks_for(int64_t warps) {
  return static_cast<unsigned>((warps + kWarpsPerBlock - 1) / kWarpsPerBlock);
}

}  // namespace

cudaError_t launch_bwd_preprocess(const Geometry& g, const void* o, const void* dout, const float* lse, float* ld,
                                  float* dq_acc, int* tickets, int* qlim, uint32_t* status, cudaStream_t stream) {
  if (g.si.T == 0 || g.si.nseq == 0 || g.si.max_len == 0) return cudaSuccess;
  const int ntile = (g.si.max_len + kPreRows - 1) / kPreRows;
  const long long blocks = static_cast<long long>(g.P) * g.si.nseq * ntile * g.H;
  if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
  auto* ob = static_cast<const __nv_bfloat16*>(o);
  auto* db = static_cast<const __nv_bfloat16*>(dout);
  if (g.D == 128)
    bwd_preprocess_kernel<128><<<static_cast<unsigned>(blocks), kPreThreads, 0, stream>>>(g, ob, db, lse, ld, dq_acc,
                                                                                       tickets, ntile, qlim, status);
  else
    bwd_preprocess_kernel<64><<<static_cast<unsigned>(blocks), kPreThreads, 0, stream>>>(g, ob, db, lse, ld, dq_acc,
                                                                                      tickets, ntile, qlim, status);
  return cudaGetLastError();
}

cudaError_t launch_branch_bwd(const Geometry& g, const void* qr, const void* kr, const void* v, const void* dout,
                              const float* lse, const float* ld, const float* dq_acc, void* dq, void* dk, void* dv,
                              cudaStream_t stream) {
  const int64_t warps = static_cast<int64_t>(g.si.T) * g.Hkv;
  if (warps == 0) return cudaSuccess;
  const int NB = g.P - 1 > 0 ? g.P - 1 : 1;
  const size_t smem = static_cast<size_t>(g.D / 2) * sizeof(double) +
                      static_cast<size_t>(kWarpsPerBlock) * (g.P * g.D + NB * 2 * g.D) * sizeof(float);
  auto* qb = static_cast<const __nv_bfloat16*>(qr);
  auto* kb = static_cast<const __nv_bfloat16*>(kr);
  auto* vb = static_cast<const __nv_bfloat16*>(v);
  auto* db = static_cast<const __nv_bfloat16*>(dout);
  auto* dqb = static_cast<__nv_bfloat16*>(dq);
  auto* dkb = static_cast<__nv_bfloat16*>(dk);
  auto* dvb = static_cast<__nv_bfloat16*>(dv);
  cudaError_t e;
  if (g.D == 128) {
    e = cudaFuncSetAttribute(branch_bwd_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    branch_bwd_kernel<128><<<blocks_for(warps), kWarpsPerBlock * 32, smem, stream>>>(g, qb, kb, vb, db, lse, ld,
                                                                                      dq_acc, dqb, dkb, dvb);
  } else {
    e = cudaFuncSetAttribute(branch_bwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    branch_bwd_kernel<64><<<blocks_for(warps), kWarpsPerBlock * 32, smem, stream>>>(g, qb, kb, vb, db, lse, ld,
                                                                                     dq_acc, dqb, dkb, dvb);
  }
  return cudaGetLastError();
}

cudaError_t launch_watchdog_selftest(uint32_t* status, uint64_t budget_ns, cudaStream_t stream) {
  watchdog_selftest_kernel<<<1, 32, 0, stream>>>(status, budget_ns);
  return cudaGetLastError();
}

}  // namespace ttt
