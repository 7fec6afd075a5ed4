// a1: per-pass rotate-half RoPE of Q and K (all passes, one launch).
//
// "DFlash/DSpark and EAGLE-3 TTT draft co-training ..." (NeMo-RL issue 3698),
// "What I'm working on", item 1: per-pass RoPE offsets aligned with inference; the
// offset itself (pass p, position i -> i+p-1) and rotate-half ("bounded multi-pass
// EAGLE-3 TTT provider", self-review) fix the rotation.
//
// Memory bound: reads q [P][T][H][D] and k [P][T][Hkv][D] once (consecutive passes
// g.sq and g.skv elements apart), writes the rotated
// copies head-major (q~ [P][H][T][D], k~ [P][Hkv][T][D]) so that the attention
// kernels fetch a (head, 128-token) tile as one contiguous block.  cos/sin depend
// on (position, frequency) only: each CTA computes them once per token in double
// precision (argument up to ~4e4 rad) and shares them across all heads.
#include <cuda_bf16.h>

#include "common.cuh"

namespace ttt {

namespace {

constexpr int kRopeTok = 8;       // tokens per CTA
constexpr int kRopeThreads = 256;

template <int D>
__global__ void __launch_bounds__(kRopeThreads) rope_fwd_kernel(Geometry g, const __nv_bfloat16* __restrict__ q,
                                                                const __nv_bfloat16* __restrict__ k,
                                                                __nv_bfloat16* __restrict__ qr,
                                                                __nv_bfloat16* __restrict__ kr) {
  constexpr int HALF = D / 2;
  constexpr int PARTS = HALF / 8;  // threads per row (8 elements of each half each)
  __shared__ float2 cs_hi[kRopeTok][HALF], cs_lo[kRopeTok][HALF];

  const int n = blockIdx.y;
  const int p = blockIdx.z;
  int start, len;
  seq_bounds(g.si, n, start, len);
  const int i0 = blockIdx.x * kRopeTok;
  if (i0 >= len) return;
  const int ntok = min(kRopeTok, len - i0);

  for (int e = threadIdx.x; e < kRopeTok * HALF; e += blockDim.x) {
    const int tok = e / HALF, d = e % HALF;
    const double inv_freq = pow(static_cast<double>(g.theta), -2.0 * d / D);
    const double ang = static_cast<double>(g.pos0 + i0 + tok + p) * inv_freq;
    double s, c;
    sincos(ang, &s, &c);
    cos_sin_split(c, s, cs_hi[tok][d], cs_lo[tok][d]);
  }
  __syncthreads();

  // every thread keeps one (token, 8-element part) slot and walks the heads, so that it
  // reads its cos / sin from shared memory once
  static_assert(kRopeThreads % (kRopeTok * PARTS) == 0, "threads must cover whole slots");
  constexpr int kHeadLanes = kRopeThreads / (kRopeTok * PARTS);
  const int NH = g.H + g.Hkv;
  const int T = g.si.T;
  const int slot = threadIdx.x % (kRopeTok * PARTS);
  const int part = slot % PARTS;
  const int tok = slot / PARTS;
  if (tok >= ntok) return;
  const int d0 = part * 8;
  float2 rh[8], rl[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    rh[e] = cs_hi[tok][d0 + e];
    rl[e] = cs_lo[tok][d0 + e];
  }
  const int tau = start + i0 + tok;
  for (int head = threadIdx.x / (kRopeTok * PARTS); head < NH; head += kHeadLanes) {
    const __nv_bfloat16* src;
    __nv_bfloat16* dst;
    if (head < g.H) {
      src = q + p * g.sq + (static_cast<int64_t>(tau) * g.H + head) * D;
      dst = qr + ((static_cast<int64_t>(p) * g.H + head) * T + tau) * D;
    } else {
      const int hk = head - g.H;
      src = k + p * g.skv + (static_cast<int64_t>(tau) * g.Hkv + hk) * D;
      dst = kr + ((static_cast<int64_t>(p) * g.Hkv + hk) * T + tau) * D;
    }
    const uint4 a = *reinterpret_cast<const uint4*>(src + d0);
    const uint4 b = *reinterpret_cast<const uint4*>(src + HALF + d0);
    const __nv_bfloat16* xa = reinterpret_cast<const __nv_bfloat16*>(&a);
    const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(&b);
    uint4 oa, ob;
    __nv_bfloat16* ya = reinterpret_cast<__nv_bfloat16*>(&oa);
    __nv_bfloat16* yb = reinterpret_cast<__nv_bfloat16*>(&ob);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      ya[e] = rotate_round(xa[e], xb[e], rh[e], rl[e], false);
      yb[e] = rotate_round(xa[e], xb[e], rh[e], rl[e], true);
    }
    *reinterpret_cast<uint4*>(dst + d0) = oa;
    *reinterpret_cast<uint4*>(dst + HALF + d0) = ob;
  }
}

}  // namespace

cudaError_t launch_rope_fwd(const Geometry& g, const void* q, const void* k, void* qr, void* kr,
                            cudaStream_t stream) {
  dim3 grid((g.si.max_len + kRopeTok - 1) / kRopeTok, g.si.nseq, g.P);
  if (g.D == 128)
    rope_fwd_kernel<128><<<grid, kRopeThreads, 0, stream>>>(
        g, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
        static_cast<__nv_bfloat16*>(qr), static_cast<__nv_bfloat16*>(kr));
  else
    rope_fwd_kernel<64><<<grid, kRopeThreads, 0, stream>>>(
        g, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
        static_cast<__nv_bfloat16*>(qr), static_cast<__nv_bfloat16*>(kr));
  return cudaGetLastError();
}

}  // namespace ttt
