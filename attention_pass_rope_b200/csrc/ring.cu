// Context-parallel ring over the pass-1 trunk K/V: the per-step pieces.
//
// "DFlash/DSpark and EAGLE-3 TTT draft co-training ..." (NeMo-RL issue 3698), "What
// I'm working on", item 4: the pass-1 trunk K/V is what travels between ranks (a zigzag
// ring), and the partial results are joined by the exact log-sum-exp merge.  A rank holds
// chunks of the sequence (all passes of their queries, keys and values); in each ring
// step it computes the attention of its query chunks against a visiting chunk of trunk
// keys/values, causal by global position, as a partial (O, lse) over that chunk's keys,
// and merges it into its running result:
//   lse = logaddexp(lse_a, lse_b),  O = e^(lse_a - lse) O_a + e^(lse_b - lse) O_b.
// The branch keys (passes 2..p at the query's own position) are local; they join the
// partial of the step that meets the chunk's own trunk keys.  The exchange between ranks
// is the caller's (host side); every kernel here reads only this GPU's memory.
#include <cmath>

#include "../../include/ttt_attn.h"
#include "common.cuh"

namespace ttt {

namespace {

constexpr int kMergeWarps = 8;

// acc <- acc (+) part for every row (p, i, h); first: acc <- part.
__global__ void __launch_bounds__(kMergeWarps * 32)
    ring_merge_kernel(int rows, int D, int H, int Lq, float* __restrict__ o_acc, float* __restrict__ lse_acc,
                      const float* __restrict__ o_part, const float* __restrict__ lse_part, int first) {
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kMergeWarps + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int lane = threadIdx.x & 31;
  // row = (p * Lq + i) * H + h; lse layout [P][H][Lq]
  const int h = static_cast<int>(row % H);
  const int64_t pi = row / H;
  const int i = static_cast<int>(pi % Lq);
  const int64_t p = pi / Lq;
  const int64_t li = (p * H + h) * Lq + i;
  float* oa = o_acc + row * D;
  const float* ob = o_part + row * D;
  const float lb = lse_part[li];
  if (first) {
    for (int d = lane * 4; d < D; d += 128) *reinterpret_cast<float4*>(oa + d) = *reinterpret_cast<const float4*>(ob + d);
    if (lane == 0) lse_acc[li] = lb;
    return;
  }
  const float la = lse_acc[li];
  const float m = fmaxf(la, lb);
  float wa = 0.f, wb = 0.f, l = m;
  if (m != -INFINITY) {
    const float ea = expf(la - m), eb = expf(lb - m);
    l = m + logf(ea + eb);
    wa = expf(la - l);
    wb = expf(lb - l);
  }
  for (int d = lane * 4; d < D; d += 128) {
    const float4 x = *reinterpret_cast<const float4*>(oa + d);
    const float4 y = *reinterpret_cast<const float4*>(ob + d);
    *reinterpret_cast<float4*>(oa + d) = make_float4(wa * x.x + wb * y.x, wa * x.y + wb * y.y, wa * x.z + wb * y.z,
                                                     wa * x.w + wb * y.w);
  }
  __syncwarp();
  if (lane == 0) lse_acc[li] = l;
}

__global__ void __launch_bounds__(256) ring_finish_kernel(int64_t n, const float* __restrict__ o_acc,
                                                          __nv_bfloat16* __restrict__ o) {
  const int64_t i = (static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x) * 4;
  if (i >= n) return;
  const float4 x = *reinterpret_cast<const float4*>(o_acc + i);
  *reinterpret_cast<uint2*>(o + i) = make_uint2(pack_bf16x2(x.x, x.y), pack_bf16x2(x.z, x.w));
}

// Trunk dK / dV of a chunk from the accumulators that travelled around the ring and came
// home: dK_1[t] = sigma * R(pos0 + t)^T dk~[t] and dV_1[t], bf16 into the pass-1 rows of
// the chunk's public dk, dv.  One warp per (token, KV head); lane l takes the rotation
// pairs (d, d + D/2) for d = l, l + 32, ... < D/2.
__global__ void __launch_bounds__(256) ring_dkv_finish_kernel(Geometry g, int n, const float* __restrict__ dk_acc,
                                                              const float* __restrict__ dv_acc,
                                                              __nv_bfloat16* __restrict__ dk,
                                                              __nv_bfloat16* __restrict__ dv) {
  const int64_t item = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (item >= static_cast<int64_t>(n) * g.Hkv) return;
  const int lane = threadIdx.x & 31;
  const int t = static_cast<int>(item / g.Hkv), kvh = static_cast<int>(item % g.Hkv);
  const int D = g.D, half = D / 2;
  const float* ka = dk_acc + (static_cast<int64_t>(kvh) * n + t) * D;
  const float* va = dv_acc + (static_cast<int64_t>(kvh) * n + t) * D;
  __nv_bfloat16* kd = dk + (static_cast<int64_t>(t) * g.Hkv + kvh) * D;  // pass 1 of the public layout
  __nv_bfloat16* vd = dv + (static_cast<int64_t>(t) * g.Hkv + kvh) * D;
  for (int d = lane; d < half; d += 32) {
    float c, s;
    angle_cos_sin(g.pos0 + t, pow(static_cast<double>(g.theta), -2.0 * d / D), c, s);
    const float x1 = ka[d] * g.scale, x2 = ka[d + half] * g.scale;
    kd[d] = __float2bfloat16_rn(fmaf(x1, c, x2 * s));
    kd[d + half] = __float2bfloat16_rn(fmaf(x2, c, -x1 * s));
    vd[d] = __float2bfloat16_rn(va[d]);
    vd[d + half] = __float2bfloat16_rn(va[d + half]);
  }
}

}  // namespace

cudaError_t launch_ring_dkv_finish(const Geometry& g, int n, const float* dk_acc, const float* dv_acc, void* dk,
                                   void* dv, cudaStream_t stream) {
  const int64_t items = static_cast<int64_t>(n) * g.Hkv;
  if (items <= 0) return cudaSuccess;
  ring_dkv_finish_kernel<<<static_cast<unsigned>((items + 7) / 8), 256, 0, stream>>>(
      g, n, dk_acc, dv_acc, static_cast<__nv_bfloat16*>(dk), static_cast<__nv_bfloat16*>(dv));
  return cudaGetLastError();
}

cudaError_t launch_ring_merge(int rows, int D, int H, int Lq, float* o_acc, float* lse_acc, const float* o_part,
                              const float* lse_part, bool first, cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  ring_merge_kernel<<<(rows + kMergeWarps - 1) / kMergeWarps, kMergeWarps * 32, 0, stream>>>(
      rows, D, H, Lq, o_acc, lse_acc, o_part, lse_part, first ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_ring_finish(int64_t n, const float* o_acc, void* o, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  const int64_t threads = (n + 3) / 4;
  ring_finish_kernel<<<static_cast<unsigned>((threads + 255) / 256), 256, 0, stream>>>(
      n, o_acc, static_cast<__nv_bfloat16*>(o));
  return cudaGetLastError();
}

}  // namespace ttt
