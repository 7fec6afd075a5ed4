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
// on (position, frequency) only: each CTA takes 4 tokens with all their passes, computes
// cos/sin once per position it needs (4 + P - 1 of them) in double precision (argument
// up to ~4e4 rad) and shares them across all heads.
#include <cuda_bf16.h>

#include "common.cuh"

namespace ttt {

namespace {

constexpr int kRopeTok = 4;       // tokens per CTA
constexpr int kRopeMaxP = 16;     // passes (positions i .. i+P-1 share one table)
constexpr int kRopeThreads = 256;

template <int D>
__global__ void __launch_bounds__(kRopeThreads) rope_fwd_kernel(Geometry g, const __nv_bfloat16* __restrict__ q,
                                                                const __nv_bfloat16* __restrict__ k,
                                                                __nv_bfloat16* __restrict__ qr,
                                                                __nv_bfloat16* __restrict__ kr) {
  constexpr int HALF = D / 2;
  constexpr int PARTS = HALF / 8;  // threads per row (8 elements of each half each)
  constexpr int NPOS = kRopeTok + kRopeMaxP - 1;
  __shared__ float2 cs_hi[NPOS][HALF], cs_lo[NPOS][HALF];
  __shared__ double inv_freq[HALF];

  const int n = blockIdx.y;
  int start, len;
  seq_bounds(g.si, n, start, len);
  const int i0 = blockIdx.x * kRopeTok;
  if (i0 >= len) return;
  const int ntok = min(kRopeTok, len - i0);

  // pass p of token i0+t is at position i0+t+p: the CTA's tokens and passes need the
  // ntok+P-1 positions from i0 on
  for (int d = threadIdx.x; d < HALF; d += blockDim.x)
    inv_freq[d] = pow(static_cast<double>(g.theta), -2.0 * d / D);
  __syncthreads();
  const int npos = ntok + g.P - 1;
  for (int e = threadIdx.x; e < npos * HALF; e += blockDim.x) {
    const int u = e / HALF, d = e % HALF;
    double sn, cn;
    sincos(static_cast<double>(g.pos0 + i0 + u) * inv_freq[d], &sn, &cn);
    cos_sin_split(cn, sn, cs_hi[u][d], cs_lo[u][d]);
  }
  __syncthreads();

  // every thread keeps one (token, 8-element part) slot and walks the (pass, head) rows
  // of that token, one row's loads ahead; a warp's threads share the row index, so the
  // pass (and the cos / sin it selects) changes warp-uniformly
  static_assert(kRopeThreads % (kRopeTok * PARTS) == 0, "threads must cover whole slots");
  constexpr int kHeadLanes = kRopeThreads / (kRopeTok * PARTS);
  const int NH = g.H + g.Hkv;
  const int nrows = g.P * NH;
  const int T = g.si.T;
  const int slot = threadIdx.x % (kRopeTok * PARTS);
  const int part = slot % PARTS;
  const int tok = slot / PARTS;
  if (tok >= ntok) return;
  const int d0 = part * 8;
  const int tau = start + i0 + tok;
  auto src_of = [&](int u) -> const __nv_bfloat16* {
    const int p = u / NH, head = u % NH;
    return head < g.H ? q + p * g.sq + (static_cast<int64_t>(tau) * g.H + head) * D
                      : k + p * g.skv + (static_cast<int64_t>(tau) * g.Hkv + (head - g.H)) * D;
  };
  int u = threadIdx.x / (kRopeTok * PARTS);
  if (u >= nrows) return;
  uint4 a, b;
  {
    const __nv_bfloat16* src = src_of(u);
    a = *reinterpret_cast<const uint4*>(src + d0);
    b = *reinterpret_cast<const uint4*>(src + HALF + d0);
  }
  int pcur = -1;
  float2 rh[8];
  const float2* rl = nullptr;
  for (; u < nrows; u += kHeadLanes) {
    const int p = u / NH, head = u % NH;
    if (p != pcur) {
      pcur = p;
#pragma unroll
      for (int e = 0; e < 8; ++e) rh[e] = cs_hi[tok + p][d0 + e];
      rl = &cs_lo[tok + p][d0];
    }
    uint4 an = a, bn = b;
    if (u + kHeadLanes < nrows) {
      const __nv_bfloat16* src = src_of(u + kHeadLanes);
      an = *reinterpret_cast<const uint4*>(src + d0);
      bn = *reinterpret_cast<const uint4*>(src + HALF + d0);
    }
    __nv_bfloat16* dst = head < g.H ? qr + ((static_cast<int64_t>(p) * g.H + head) * T + tau) * D
                                    : kr + ((static_cast<int64_t>(p) * g.Hkv + (head - g.H)) * T + tau) * D;
    uint4 oa, ob;
    rotate8_round(a, b, rh, rl, oa, ob);
    *reinterpret_cast<uint4*>(dst + d0) = oa;
    *reinterpret_cast<uint4*>(dst + HALF + d0) = ob;
    a = an;
    b = bn;
  }
}

}  // namespace

cudaError_t launch_rope_fwd(const Geometry& g, const void* q, const void* k, void* qr, void* kr,
                            cudaStream_t stream) {
  if (g.P > kRopeMaxP) return cudaErrorInvalidValue;
  dim3 grid((g.si.max_len + kRopeTok - 1) / kRopeTok, g.si.nseq);
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
