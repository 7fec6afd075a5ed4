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
                          int* __restrict__ tickets, int ntile, int* __restrict__ qlim, uint32_t* status,
                          const uint32_t* __restrict__ dq_zeroed) {
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
  // zero this tile's dq~ accumulator rows (contiguous: nvalid rows of D floats), unless
  // the forward has zeroed the whole accumulator already
  if (!dq_zeroed || *dq_zeroed != kDqZeroedMagic) {
    float4* z = reinterpret_cast<float4*>(dq_acc + ((static_cast<int64_t>(p) * g.H + h) * T + start + pos0) * D);
    for (int i = threadIdx.x; i < nvalid * D / 4; i += kPreThreads) z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
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
// a7 + a8: branch backward and finalisation.  One warp per token at a time, for each of
// its KV heads and every pass p and group head h:
//     dq~ = dq_acc (trunk part) + sum_j dS_j k~_j        (j = passes 1..p, 0-based)
//     dS_j = P_j (dO . V_j - delta),  P_j = exp(sigma q~ . k~_j - lse)
//     dk~_j += dS_j q~,  dV_j += P_j dO                   (accumulated over p >= j, h)
//     dQ_p = R(i+p)^T (sigma dq~)
//   dK_j = R(i+j)^T (sigma dk~_j) and dV_j for the branch passes j >= 1 (dK_1 and dV_1
//   are written by the trunk backward).
// A warp works through (KV head, pass) units -- the unit's dq~ rows, q~ rows, dO rows,
// lse and delta of the group's heads and the branch keys / values it needs -- and
// fetches the next unit into the other half of a two-stage shared-memory buffer with
// cp.async while it computes the current one (no registers hold data in flight).  The
// cos / sin of the token's positions i..i+P-1 are formed once and serve all its KV
// heads.  Each warp takes tokens w, w + W, ... (W = warps in the grid).  The kernel is
// bound by instruction issue (ncu: issue slots ~64 % busy with 4 warps per scheduler),
// then by memory latency.  Shared memory: the block's inverse frequencies (double),
// then per warp the cos/sin of positions i..i+P-1, the branch-pass accumulators and the
// stages.
// ---------------------------------------------------------------------------
struct BranchLayout {
  int cs, acc, stage, dqa, q, o, kj, vj, lse, dl, stage_bytes, warp_bytes;
};

// byte offsets inside one warp's shared-memory region (every part 16-byte aligned)
__host__ __device__ inline BranchLayout branch_layout(int D, int gsz, int P) {
  const int NB = P > 1 ? P - 1 : 1;
  BranchLayout L{};
  L.cs = 0;                                // float [P][D]: cos [D/2], sin [D/2]
  L.acc = L.cs + P * D * 4;                // float [NB][2][D]
  L.stage = L.acc + NB * 2 * D * 4;        // two stages
  L.dqa = 0;                               // float [gsz][D]
  L.q = L.dqa + gsz * D * 4;               // bf16 [gsz][D]
  L.o = L.q + gsz * D * 2;                 // bf16 [gsz][D]
  L.kj = L.o + gsz * D * 2;                // bf16 [NB][D]
  L.vj = L.kj + NB * D * 2;                // bf16 [NB][D]
  L.lse = L.vj + NB * D * 2;               // float [gsz]
  L.dl = L.lse + ((gsz * 4 + 15) / 16) * 16;  // float [gsz]
  L.stage_bytes = L.dl + ((gsz * 4 + 15) / 16) * 16;
  L.warp_bytes = L.stage + 2 * L.stage_bytes;
  return L;
}

constexpr int kBranchTokensPerWarp = 1;
constexpr int kBranchFreqBytes = 512;  // inverse frequencies (double [D/2]), padded

template <int D>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    branch_bwd_kernel(Geometry g, const __nv_bfloat16* __restrict__ qr, const __nv_bfloat16* __restrict__ kr,
                      const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ dout,
                      const float* __restrict__ lse, const float* __restrict__ ld,
                      const float* __restrict__ dq_acc,
                      __nv_bfloat16* __restrict__ dq, __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv,
                      int warps_per_block) {
  constexpr int E = D / 64;
  extern __shared__ __align__(16) unsigned char branch_smem[];
  double* inv_freq = reinterpret_cast<double*>(branch_smem);  // [D/2]
  for (int d = threadIdx.x; d < D / 2; d += blockDim.x) inv_freq[d] = pow(static_cast<double>(g.theta), -2.0 * d / D);
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  if (wib >= warps_per_block) return;
  const int gsz = g.H / g.Hkv;
  const int NB = g.P > 1 ? g.P - 1 : 1;
  const BranchLayout Lo = branch_layout(D, gsz, g.P);
  unsigned char* wsm = branch_smem + kBranchFreqBytes + static_cast<size_t>(wib) * Lo.warp_bytes;
  float* cs = reinterpret_cast<float*>(wsm + Lo.cs);
  float* acc = reinterpret_cast<float*>(wsm + Lo.acc);
  auto stage = [&](int st) { return wsm + Lo.stage + st * Lo.stage_bytes; };
  const int T = g.si.T;
  const int64_t W = static_cast<int64_t>(gridDim.x) * warps_per_block;
  const int64_t dl_base = static_cast<int64_t>(ld_slots(g.si)) * 128;

  // queue the copies of unit (token tau, KV head kvh, pass p) into stage st (one commit
  // group per unit)
  auto issue = [&](int tau, int kvh, int p, int st) {
    unsigned char* sb = stage(st);
    constexpr int RC32 = D / 4;  // 16-byte chunks of an fp32 row
    constexpr int RC16 = D / 8;  // 16-byte chunks of a bf16 row
    for (int c = lane; c < gsz * RC32; c += 32) {
      const int hh = c / RC32, k = c % RC32;
      const int64_t row = (static_cast<int64_t>(p) * g.H + kvh * gsz + hh) * T + tau;
      cp_async16(sb + Lo.dqa + (hh * D + 4 * k) * 4, dq_acc + row * D + 4 * k);
    }
    if (p > 0) {
      int n, pos;
      token_position(g.si, tau, n, pos);
      const int64_t dl_off = static_cast<int64_t>(ld_slot(tau - pos, n, pos)) * 128 + 64 + (pos & 63);
      for (int c = lane; c < gsz * RC16; c += 32) {
        const int hh = c / RC16, k = c % RC16;
        const int64_t row = (static_cast<int64_t>(p) * g.H + kvh * gsz + hh) * T + tau;
        cp_async16(sb + Lo.q + (hh * D + 8 * k) * 2, qr + row * D + 8 * k);
      }
      const __nv_bfloat16* orow = dout + p * g.sq + (static_cast<int64_t>(tau) * g.H + kvh * gsz) * D;
      for (int c = lane; c < gsz * RC16; c += 32) cp_async16(sb + Lo.o + c * 16, orow + 8 * c);
      for (int c = lane; c < p * RC16; c += 32) {
        const int j = 1 + c / RC16, k = c % RC16;
        cp_async16(sb + Lo.kj + ((j - 1) * D + 8 * k) * 2, kr + ((static_cast<int64_t>(j) * g.Hkv + kvh) * T + tau) * D + 8 * k);
        cp_async16(sb + Lo.vj + ((j - 1) * D + 8 * k) * 2,
                   v + j * g.skv + (static_cast<int64_t>(tau) * g.Hkv + kvh) * D + 8 * k);
      }
      if (lane < gsz) {
        const int h = kvh * gsz + lane;
        cp_async4(sb + Lo.lse + lane * 4, lse + lse_index(g.si, g.H, p, h, n, tau, pos));
        cp_async4(sb + Lo.dl + lane * 4, ld + (static_cast<int64_t>(p) * g.H + h) * dl_base + dl_off);
      }
    }
    cp_async_commit();
  };

  // one token per warp at a time, all its KV heads and passes: the token's cos / sin
  // serve all of them
  int tau = static_cast<int>(static_cast<int64_t>(blockIdx.x) * warps_per_block + wib);
  if (tau >= T) return;
  int st = 0;
  issue(tau, 0, 0, 0);
  while (true) {
    int n, pos;
    token_position(g.si, tau, n, pos);
    // cos / sin of this token's positions
    for (int p = 0; p < g.P; ++p)
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const int d = LaneMap<D>::d(lane, 0, e);
        angle_cos_sin(g.pos0 + pos + p, inv_freq[d], cs[p * D + d], cs[p * D + D / 2 + d]);
      }
    const int64_t next_tau = tau + W;
    for (int kvh = 0; kvh < g.Hkv; ++kvh) {
      // zeroed branch accumulators of this KV head
      for (int j = 0; j < NB; ++j)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
#pragma unroll
          for (int e = 0; e < E; ++e) {
            acc[(j * 2 + 0) * D + LaneMap<D>::d(lane, hh, e)] = 0.f;
            acc[(j * 2 + 1) * D + LaneMap<D>::d(lane, hh, e)] = 0.f;
          }
      for (int p = 0; p < g.P; ++p) {
        // fetch the next unit while this one is computed
        int nt = tau, nk = kvh, np = p + 1;
        if (np == g.P) {
          np = 0;
          if (++nk == g.Hkv) {
            nk = 0;
            nt = next_tau < T ? static_cast<int>(next_tau) : -1;
          }
        }
        if (nt >= 0) {
          issue(nt, nk, np, st ^ 1);
          cp_async_wait<1>();
        } else {
          cp_async_wait<0>();
        }
      __syncwarp();
      const unsigned char* sb = stage(st);
      const float* sdqa = reinterpret_cast<const float*>(sb + Lo.dqa);
      const __nv_bfloat16* sq = reinterpret_cast<const __nv_bfloat16*>(sb + Lo.q);
      const __nv_bfloat16* so = reinterpret_cast<const __nv_bfloat16*>(sb + Lo.o);
      const __nv_bfloat16* skj = reinterpret_cast<const __nv_bfloat16*>(sb + Lo.kj);
      const __nv_bfloat16* svj = reinterpret_cast<const __nv_bfloat16*>(sb + Lo.vj);
      const float* slse = reinterpret_cast<const float*>(sb + Lo.lse);
      const float* sdl = reinterpret_cast<const float*>(sb + Lo.dl);
      float c[E], sn[E];
#pragma unroll
      for (int e = 0; e < E; ++e) {
        c[e] = cs[p * D + LaneMap<D>::d(lane, 0, e)];
        sn[e] = cs[p * D + D / 2 + LaneMap<D>::d(lane, 0, e)];
      }
      if (p > 0 && p <= 2) {
        // up to two branch keys (P <= 3): their k~ / V rows are read once for the group's
        // heads, and the heads' dk~ / dV contributions are summed in registers before
        // they join the accumulators
        float kjr[2][2][E], vjr[2][2][E], akr[2][2][E], avr[2][2][E];
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          if (jj < p) {
            load_bf16_row<D>(skj + jj * D, lane, kjr[jj]);
            load_bf16_row<D>(svj + jj * D, lane, vjr[jj]);
          }
#pragma unroll
          for (int x = 0; x < 2; ++x)
#pragma unroll
            for (int e = 0; e < E; ++e) akr[jj][x][e] = avr[jj][x][e] = 0.f;
        }
        for (int hh = 0; hh < gsz; ++hh) {
          float dqv[2][E], q[2][E], dO[2][E];
          load_f32_row<D>(sdqa + hh * D, lane, dqv);
          load_bf16_row<D>(sq + hh * D, lane, q);
          load_bf16_row<D>(so + hh * D, lane, dO);
          const float lse_v = slse[hh], dl = sdl[hh];
#pragma unroll
          for (int jj = 0; jj < 2; ++jj) {
            if (jj >= p) continue;
            float sdot = 0.f, tdot = 0.f;
#pragma unroll
            for (int x = 0; x < 2; ++x)
#pragma unroll
              for (int e = 0; e < E; ++e) {
                sdot = fmaf(q[x][e], kjr[jj][x][e], sdot);
                tdot = fmaf(dO[x][e], vjr[jj][x][e], tdot);
              }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
              sdot += __shfl_xor_sync(0xffffffffu, sdot, o);
              tdot += __shfl_xor_sync(0xffffffffu, tdot, o);
            }
            const float pj = __expf(sdot * g.scale - lse_v);
            const float dsj = pj * (tdot - dl);
#pragma unroll
            for (int x = 0; x < 2; ++x)
#pragma unroll
              for (int e = 0; e < E; ++e) {
                dqv[x][e] = fmaf(dsj, kjr[jj][x][e], dqv[x][e]);
                akr[jj][x][e] = fmaf(dsj, q[x][e], akr[jj][x][e]);
                avr[jj][x][e] = fmaf(pj, dO[x][e], avr[jj][x][e]);
              }
          }
#pragma unroll
          for (int x = 0; x < 2; ++x)
#pragma unroll
            for (int e = 0; e < E; ++e) dqv[x][e] *= g.scale;
          rotate_back<D>(dqv, c, sn);
          store_bf16_row<D>(dq + p * g.sq + (static_cast<int64_t>(tau) * g.H + kvh * gsz + hh) * D, lane, dqv);
        }
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          if (jj >= p) continue;
          float* akp = acc + (jj * 2 + 0) * D;
          float* avp = acc + (jj * 2 + 1) * D;
#pragma unroll
          for (int x = 0; x < 2; ++x)
#pragma unroll
            for (int e = 0; e < E; ++e) {
              const int d = LaneMap<D>::d(lane, x, e);
              akp[d] += akr[jj][x][e];
              avp[d] += avr[jj][x][e];
            }
        }
      } else
      for (int hh = 0; hh < gsz; ++hh) {
        float dqv[2][E], q[2][E], dO[2][E];
        load_f32_row<D>(sdqa + hh * D, lane, dqv);
        if (p > 0) {
          load_bf16_row<D>(sq + hh * D, lane, q);
          load_bf16_row<D>(so + hh * D, lane, dO);
          const float lse_v = slse[hh], dl = sdl[hh];
          for (int j = 1; j <= p; ++j) {
            float kj[2][E], vj[2][E];
            load_bf16_row<D>(skj + (j - 1) * D, lane, kj);
            load_bf16_row<D>(svj + (j - 1) * D, lane, vj);
            float sdot = 0.f, tdot = 0.f;
#pragma unroll
            for (int x = 0; x < 2; ++x)
#pragma unroll
              for (int e = 0; e < E; ++e) {
                sdot = fmaf(q[x][e], kj[x][e], sdot);
                tdot = fmaf(dO[x][e], vj[x][e], tdot);
              }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
              sdot += __shfl_xor_sync(0xffffffffu, sdot, o);
              tdot += __shfl_xor_sync(0xffffffffu, tdot, o);
            }
            const float pj = __expf(sdot * g.scale - lse_v);
            const float dsj = pj * (tdot - dl);
            float* akp = acc + ((j - 1) * 2 + 0) * D;
            float* avp = acc + ((j - 1) * 2 + 1) * D;
#pragma unroll
            for (int x = 0; x < 2; ++x)
#pragma unroll
              for (int e = 0; e < E; ++e) {
                const int d = LaneMap<D>::d(lane, x, e);
                dqv[x][e] = fmaf(dsj, kj[x][e], dqv[x][e]);
                akp[d] = fmaf(dsj, q[x][e], akp[d]);
                avp[d] = fmaf(pj, dO[x][e], avp[d]);
              }
          }
        }
#pragma unroll
        for (int x = 0; x < 2; ++x)
#pragma unroll
          for (int e = 0; e < E; ++e) dqv[x][e] *= g.scale;
        rotate_back<D>(dqv, c, sn);
        store_bf16_row<D>(dq + p * g.sq + (static_cast<int64_t>(tau) * g.H + kvh * gsz + hh) * D, lane, dqv);
      }
      __syncwarp();  // every lane is done with stage st before it is refilled
      st ^= 1;
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
      for (int x = 0; x < 2; ++x)
#pragma unroll
        for (int e = 0; e < E; ++e) {
          kx[x][e] = acc[((j - 1) * 2 + 0) * D + LaneMap<D>::d(lane, x, e)] * g.scale;
          vx[x][e] = acc[((j - 1) * 2 + 1) * D + LaneMap<D>::d(lane, x, e)];
        }
      rotate_back<D>(kx, c, sn);
      const int64_t krow = j * g.skv + (static_cast<int64_t>(tau) * g.Hkv + kvh) * D;
      store_bf16_row<D>(dk + krow, lane, kx);
      store_bf16_row<D>(dv + krow, lane, vx);
    }
    __syncwarp();  // the accumulators are rewritten for the next KV head
    }
    __syncwarp();  // cos / sin are rewritten for the next token
    if (next_tau >= T) break;
    tau = static_cast<int>(next_tau);
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

}  // namespace

cudaError_t launch_bwd_preprocess(const Geometry& g, const void* o, const void* dout, const float* lse, float* ld,
                                  float* dq_acc, int* tickets, int* qlim, uint32_t* status,
                                  const uint32_t* dq_zeroed, cudaStream_t stream) {
  if (g.si.T == 0 || g.si.nseq == 0 || g.si.max_len == 0) return cudaSuccess;
  const int ntile = (g.si.max_len + kPreRows - 1) / kPreRows;
  const long long blocks = static_cast<long long>(g.P) * g.si.nseq * ntile * g.H;
  if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
  auto* ob = static_cast<const __nv_bfloat16*>(o);
  auto* db = static_cast<const __nv_bfloat16*>(dout);
  if (g.D == 128)
    bwd_preprocess_kernel<128><<<static_cast<unsigned>(blocks), kPreThreads, 0, stream>>>(
        g, ob, db, lse, ld, dq_acc, tickets, ntile, qlim, status, dq_zeroed);
  else
    bwd_preprocess_kernel<64><<<static_cast<unsigned>(blocks), kPreThreads, 0, stream>>>(
        g, ob, db, lse, ld, dq_acc, tickets, ntile, qlim, status, dq_zeroed);
  return cudaGetLastError();
}

cudaError_t launch_branch_bwd(const Geometry& g, const void* qr, const void* kr, const void* v, const void* dout,
                              const float* lse, const float* ld, const float* dq_acc, void* dq, void* dk, void* dv,
                              cudaStream_t stream) {
  const int64_t items = g.si.T;  // tokens
  if (items == 0) return cudaSuccess;
  const BranchLayout Lo = branch_layout(g.D, g.H / g.Hkv, g.P);
  // as many warps per block as 227 KB of shared memory holds (at most kWarpsPerBlock)
  const int wpb = static_cast<int>(std::min<int64_t>(kWarpsPerBlock, (227 * 1024 - kBranchFreqBytes) / Lo.warp_bytes));
  if (wpb < 1) return cudaErrorInvalidConfiguration;
  const size_t smem = kBranchFreqBytes + static_cast<size_t>(wpb) * Lo.warp_bytes;
  const int64_t per_block = static_cast<int64_t>(wpb) * kBranchTokensPerWarp;
  const int64_t blocks = (items + per_block - 1) / per_block;
  if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
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
    branch_bwd_kernel<128><<<static_cast<unsigned>(blocks), wpb * 32, smem, stream>>>(
        g, qb, kb, vb, db, lse, ld, dq_acc, dqb, dkb, dvb, wpb);
  } else {
    e = cudaFuncSetAttribute(branch_bwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    branch_bwd_kernel<64><<<static_cast<unsigned>(blocks), wpb * 32, smem, stream>>>(
        g, qb, kb, vb, db, lse, ld, dq_acc, dqb, dkb, dvb, wpb);
  }
  return cudaGetLastError();
}

cudaError_t launch_watchdog_selftest(uint32_t* status, uint64_t budget_ns, cudaStream_t stream) {
  watchdog_selftest_kernel<<<1, 32, 0, stream>>>(status, budget_ns);
  return cudaGetLastError();
}

}  // namespace ttt
