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
// a7 + a8: branch backward and finalisation.  One warp per (token, KV head) item:
//   for every pass p and group head h:
//     dq~ = dq_acc (trunk part) + sum_j dS_j k~_j        (j = passes 1..p, 0-based)
//     dS_j = P_j (dO . V_j - delta),  P_j = exp(sigma q~ . k~_j - lse)
//     dk~_j += dS_j q~,  dV_j += P_j dO                   (accumulated over p >= j, h)
//     dQ_p = R(i+p)^T (sigma dq~)
//   dK_j = R(i+j)^T (sigma dk~_j) and dV_j for the branch passes j >= 1 (dK_1 and dV_1
//   are written by the trunk backward).
// The kernel is bound by memory latency, so what counts is the bytes each warp keeps in
// flight.  A warp works through (item, pass) units -- the unit's dq~ rows, q~ rows, dO
// rows, lse and delta of the group's heads and the branch keys / values it needs -- and
// fetches the next unit into the other half of a two-stage shared-memory buffer with
// cp.async while it computes the current one (no registers hold data in flight).  The
// compute is instruction-bound: each half-warp takes one head's row (16 lanes, a row's
// dot products reduce in 4 shuffle steps), two rows per warp instruction.  Each
// warp takes items w, w + W, ... (W = warps in the grid) so that neighbouring warps read
// neighbouring rows.  Shared memory: the block's inverse frequencies (double), then per
// warp the cos/sin of positions i..i+P-1, the branch-pass accumulators and the stages.
// ---------------------------------------------------------------------------
struct BranchLayout {
  int cs, acc, stage, dqa, q, o, kj, vj, lse, dl, stage_bytes, warp_bytes;
};

// byte offsets inside one warp's shared-memory region (every part 16-byte aligned)
__host__ __device__ inline BranchLayout branch_layout(int D, int gsz, int P) {
  const int NB = P > 1 ? P - 1 : 1;
  BranchLayout L{};
  L.cs = 0;                                // float [P][D]: cos [D/2], sin [D/2]
  L.acc = L.cs + P * D * 4;                // float [2 half-warps][NB][2][D]
  L.stage = L.acc + 2 * NB * 2 * D * 4;    // two stages
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

constexpr int kBranchItemsPerWarp = 8;
constexpr int kBranchFreqBytes = 512;  // inverse frequencies (double [D/2]), padded

template <int D>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    branch_bwd_kernel(Geometry g, const __nv_bfloat16* __restrict__ qr, const __nv_bfloat16* __restrict__ kr,
                      const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ dout,
                      const float* __restrict__ lse, const float* __restrict__ ld,
                      const float* __restrict__ dq_acc,
                      __nv_bfloat16* __restrict__ dq, __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv,
                      int warps_per_block) {
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
  const int64_t nitems = static_cast<int64_t>(T) * g.Hkv;
  const int64_t W = static_cast<int64_t>(gridDim.x) * warps_per_block;
  const int64_t dl_base = static_cast<int64_t>(ld_slots(g.si)) * 128;

  // queue the copies of unit (item, p) into stage st (one commit group per unit)
  auto issue = [&](int64_t item, int p, int st) {
    const int tau = static_cast<int>(item / g.Hkv);
    const int kvh = static_cast<int>(item % g.Hkv);
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

  // compute mapping: half-warp hw takes one head's row at a time; its lane l16 holds
  // the EL elements [EL*l16, EL*l16+EL) of each half of the head dimension, so that every
  // RoPE pair (d, d + D/2) stays in one lane and a row's dot products reduce over 16 lanes
  constexpr int EL = D / 32;
  const int hw = lane >> 4, l16 = lane & 15;
  const int dlo = EL * l16, dhi = D / 2 + EL * l16;
  float* acc_h = acc + hw * NB * 2 * D;  // this half-warp's accumulators
  auto lds_f32 = [](const float* row, int d, float (&x)[EL]) {
    if constexpr (EL == 4) {
      const float4 v4 = *reinterpret_cast<const float4*>(row + d);
      x[0] = v4.x; x[1] = v4.y; x[2] = v4.z; x[3] = v4.w;
    } else {
      const float2 v2 = *reinterpret_cast<const float2*>(row + d);
      x[0] = v2.x; x[1] = v2.y;
    }
  };
  auto lds_bf16 = [](const __nv_bfloat16* row, int d, float (&x)[EL]) {
    if constexpr (EL == 4) {
      const uint2 u = *reinterpret_cast<const uint2*>(row + d);
      const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
      const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
      x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
    } else {
      const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(row + d));
      x[0] = a.x; x[1] = a.y;
    }
  };
  auto stg_bf16 = [](__nv_bfloat16* row, int d, const float (&x)[EL]) {
    if constexpr (EL == 4) {
      *reinterpret_cast<uint2*>(row + d) = make_uint2(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]));
    } else {
      *reinterpret_cast<uint32_t*>(row + d) = pack_bf16x2(x[0], x[1]);
    }
  };

  int64_t item = static_cast<int64_t>(blockIdx.x) * warps_per_block + wib;
  if (item >= nitems) return;
  int st = 0;
  issue(item, 0, 0);
  while (true) {
    const int tau = static_cast<int>(item / g.Hkv);
    const int kvh = static_cast<int>(item % g.Hkv);
    int n, pos;
    token_position(g.si, tau, n, pos);
    // cos / sin of this token's positions, zeroed branch accumulators (both copies)
    for (int e = lane; e < g.P * (D / 2); e += 32) {
      const int p = e / (D / 2), d = e % (D / 2);
      angle_cos_sin(pos + p, inv_freq[d], cs[p * D + d], cs[p * D + D / 2 + d]);
    }
    for (int e = lane; e < 2 * NB * 2 * D; e += 32) acc[e] = 0.f;
    __syncwarp();
    const int64_t next_item = item + W;
    for (int p = 0; p < g.P; ++p) {
      // fetch the next unit while this one is computed
      const bool more = p + 1 < g.P || next_item < nitems;
      if (more) {
        issue(p + 1 < g.P ? item : next_item, p + 1 < g.P ? p + 1 : 0, st ^ 1);
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
      float c[EL], sn[EL];
      lds_f32(cs + p * D, dlo, c);
      lds_f32(cs + p * D + D / 2, dlo, sn);
      for (int h2 = 0; h2 < gsz; h2 += 2) {
        const int hh = h2 + hw;
        const bool on = hh < gsz;  // an odd group leaves the second half-warp idle on its last pair
        const int hr = on ? hh : h2;
        float x1[EL], x2[EL];
        lds_f32(sdqa + hr * D, dlo, x1);
        lds_f32(sdqa + hr * D, dhi, x2);
        if (p > 0) {
          float q1[EL], q2[EL], o1[EL], o2[EL];
          lds_bf16(sq + hr * D, dlo, q1);
          lds_bf16(sq + hr * D, dhi, q2);
          lds_bf16(so + hr * D, dlo, o1);
          lds_bf16(so + hr * D, dhi, o2);
          const float lse_v = slse[hr], dl = sdl[hr];
          for (int j = 1; j <= p; ++j) {
            float k1[EL], k2[EL], v1[EL], v2[EL];
            lds_bf16(skj + (j - 1) * D, dlo, k1);
            lds_bf16(skj + (j - 1) * D, dhi, k2);
            lds_bf16(svj + (j - 1) * D, dlo, v1);
            lds_bf16(svj + (j - 1) * D, dhi, v2);
            float sdot = 0.f, tdot = 0.f;
#pragma unroll
            for (int e = 0; e < EL; ++e) {
              sdot = fmaf(q1[e], k1[e], fmaf(q2[e], k2[e], sdot));
              tdot = fmaf(o1[e], v1[e], fmaf(o2[e], v2[e], tdot));
            }
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) {
              sdot += __shfl_xor_sync(0xffffffffu, sdot, o);
              tdot += __shfl_xor_sync(0xffffffffu, tdot, o);
            }
            float pj = __expf(sdot * g.scale - lse_v);
            float dsj = pj * (tdot - dl);
            if (!on) pj = dsj = 0.f;
            float* ak = acc_h + ((j - 1) * 2 + 0) * D;
            float* av = acc_h + ((j - 1) * 2 + 1) * D;
            float a1[EL], a2[EL], b1[EL], b2[EL];
            lds_f32(ak, dlo, a1);
            lds_f32(ak, dhi, a2);
            lds_f32(av, dlo, b1);
            lds_f32(av, dhi, b2);
#pragma unroll
            for (int e = 0; e < EL; ++e) {
              x1[e] = fmaf(dsj, k1[e], x1[e]);
              x2[e] = fmaf(dsj, k2[e], x2[e]);
              a1[e] = fmaf(dsj, q1[e], a1[e]);
              a2[e] = fmaf(dsj, q2[e], a2[e]);
              b1[e] = fmaf(pj, o1[e], b1[e]);
              b2[e] = fmaf(pj, o2[e], b2[e]);
            }
            if constexpr (EL == 4) {
              *reinterpret_cast<float4*>(ak + dlo) = make_float4(a1[0], a1[1], a1[2], a1[3]);
              *reinterpret_cast<float4*>(ak + dhi) = make_float4(a2[0], a2[1], a2[2], a2[3]);
              *reinterpret_cast<float4*>(av + dlo) = make_float4(b1[0], b1[1], b1[2], b1[3]);
              *reinterpret_cast<float4*>(av + dhi) = make_float4(b2[0], b2[1], b2[2], b2[3]);
            } else {
              *reinterpret_cast<float2*>(ak + dlo) = make_float2(a1[0], a1[1]);
              *reinterpret_cast<float2*>(ak + dhi) = make_float2(a2[0], a2[1]);
              *reinterpret_cast<float2*>(av + dlo) = make_float2(b1[0], b1[1]);
              *reinterpret_cast<float2*>(av + dhi) = make_float2(b2[0], b2[1]);
            }
          }
        }
        if (on) {
          // dQ = R(pos + p)^T (sigma dq~)
          float y1[EL], y2[EL];
#pragma unroll
          for (int e = 0; e < EL; ++e) {
            const float a = x1[e] * g.scale, b = x2[e] * g.scale;
            y1[e] = fmaf(a, c[e], b * sn[e]);
            y2[e] = fmaf(b, c[e], -a * sn[e]);
          }
          __nv_bfloat16* out = dq + p * g.sq + (static_cast<int64_t>(tau) * g.H + kvh * gsz + hh) * D;
          stg_bf16(out, dlo, y1);
          stg_bf16(out, dhi, y2);
        }
      }
      __syncwarp();  // every lane is done with stage st before it is refilled
      st ^= 1;
    }
    // dK and dV of the branch passes: the two half-warps' sums, sigma and R^T for dK
    // (those of the trunk pass come from the trunk backward); half-warp hw takes the
    // branch passes j = 1 + hw, 3 + hw, ...
    for (int j = 1 + hw; j < g.P; j += 2) {
      const float* k0 = acc + ((j - 1) * 2 + 0) * D;
      const float* k1b = acc + NB * 2 * D + ((j - 1) * 2 + 0) * D;
      const float* v0 = acc + ((j - 1) * 2 + 1) * D;
      const float* v1b = acc + NB * 2 * D + ((j - 1) * 2 + 1) * D;
      float a1[EL], a2[EL], t1[EL], t2[EL], b1[EL], b2[EL], u1[EL], u2[EL], c[EL], sn[EL];
      lds_f32(k0, dlo, a1); lds_f32(k0, dhi, a2); lds_f32(k1b, dlo, t1); lds_f32(k1b, dhi, t2);
      lds_f32(v0, dlo, b1); lds_f32(v0, dhi, b2); lds_f32(v1b, dlo, u1); lds_f32(v1b, dhi, u2);
      lds_f32(cs + j * D, dlo, c);
      lds_f32(cs + j * D + D / 2, dlo, sn);
      float y1[EL], y2[EL], w1[EL], w2[EL];
#pragma unroll
      for (int e = 0; e < EL; ++e) {
        const float a = (a1[e] + t1[e]) * g.scale, b = (a2[e] + t2[e]) * g.scale;
        y1[e] = fmaf(a, c[e], b * sn[e]);
        y2[e] = fmaf(b, c[e], -a * sn[e]);
        w1[e] = b1[e] + u1[e];
        w2[e] = b2[e] + u2[e];
      }
      const int64_t krow = j * g.skv + (static_cast<int64_t>(tau) * g.Hkv + kvh) * D;
      stg_bf16(dk + krow, dlo, y1);
      stg_bf16(dk + krow, dhi, y2);
      stg_bf16(dv + krow, dlo, w1);
      stg_bf16(dv + krow, dhi, w2);
    }
    __syncwarp();  // cos / sin and the accumulators are rewritten for the next item
    item = next_item;
    if (item >= nitems) break;
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
  const int64_t items = static_cast<int64_t>(g.si.T) * g.Hkv;
  if (items == 0) return cudaSuccess;
  const BranchLayout Lo = branch_layout(g.D, g.H / g.Hkv, g.P);
  // as many warps per block as 227 KB of shared memory holds (at most kWarpsPerBlock)
  const int wpb = static_cast<int>(std::min<int64_t>(kWarpsPerBlock, (227 * 1024 - kBranchFreqBytes) / Lo.warp_bytes));
  if (wpb < 1) return cudaErrorInvalidConfiguration;
  const size_t smem = kBranchFreqBytes + static_cast<size_t>(wpb) * Lo.warp_bytes;
  const int64_t per_block = static_cast<int64_t>(wpb) * kBranchItemsPerWarp;
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
