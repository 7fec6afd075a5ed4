// Block-draft attention of DFlash/DSpark drafters: the rotation of the context keys and
// of the block tokens, and the backward of the block part.
//
// "DFlash/DSpark and EAGLE-3 TTT draft co-training for speculative decoding (Megatron
// backend)" (NeMo-RL issue 3698), "What I'm working on", item 2: a block drafter drafts
// a block made of an anchor and mask tokens, with bidirectional attention inside the
// block and the trunk truncated at the anchor; item 4: the same on the packed layout.
// A block b of Bs tokens starts at anchor a_b of its sequence: token j sits at position
// a_b + j.  Every token of the block sees the context keys 0..a_b (the trunk, computed by
// the trunk kernels with the anchor as the row's key limit) and all Bs keys of its own
// block (computed here and in the trunk forward's epilogue); the two parts are merged
// exactly through their log-sum-exps.
#include <cuda_bf16.h>

#include "common.cuh"

namespace ttt {

namespace {

constexpr int kRopeRows = 8;
constexpr int kRopeThreads = 256;

// Position of row tau of a rotation: a context token (its position in its sequence) or
// a block token (its block's clamped anchor + its index in the block).
struct RowPositions {
  bool block;
  __device__ int operator()(const Geometry& g, int tau) const {
    if (!block) {
      int n, pos;
      token_position(g.ksi, tau, n, pos);
      return pos;
    }
    int n, r;
    token_position(g.si, tau, n, r);
    int kstart, klen;
    seq_bounds(g.ksi, n, kstart, klen);
    return block_row_position(g, tau - r, r, klen);
  }
};

// dst_x[head][tau][:] = R(pos(tau)) src_x[tau][head][:] for the heads of up to two
// tensors that share the rows' positions (rotate-half RoPE, double math, bf16 out;
// outputs head-major so that a (head, 128-row) tile is one contiguous block for TMA).
template <int D>
__global__ void __launch_bounds__(kRopeThreads) rope_rows_kernel(Geometry g, int T, RowPositions posf,
                                                                 const __nv_bfloat16* __restrict__ src_a, int nha,
                                                                 __nv_bfloat16* __restrict__ dst_a,
                                                                 const __nv_bfloat16* __restrict__ src_b, int nhb,
                                                                 __nv_bfloat16* __restrict__ dst_b) {
  constexpr int HALF = D / 2;
  constexpr int PARTS = HALF / 8;
  __shared__ double2 cs[kRopeRows][HALF];
  const int r0 = blockIdx.x * kRopeRows;
  const int nrows = min(kRopeRows, T - r0);
  for (int e = threadIdx.x; e < kRopeRows * HALF; e += blockDim.x) {
    const int r = e / HALF, d = e % HALF;
    if (r >= nrows) continue;
    const double inv_freq = pow(static_cast<double>(g.theta), -2.0 * d / D);
    double s, c;
    sincos(static_cast<double>(posf(g, r0 + r)) * inv_freq, &s, &c);
    cs[r][d] = make_double2(c, s);
  }
  __syncthreads();
  const int NH = nha + nhb;
  for (int task = threadIdx.x; task < NH * kRopeRows * PARTS; task += blockDim.x) {
    const int part = task % PARTS;
    const int r = (task / PARTS) % kRopeRows;
    const int head = task / (PARTS * kRopeRows);
    if (r >= nrows) continue;
    const int tau = r0 + r;
    const __nv_bfloat16* src;
    __nv_bfloat16* dst;
    if (head < nha) {
      src = src_a + (static_cast<int64_t>(tau) * nha + head) * D;
      dst = dst_a + (static_cast<int64_t>(head) * T + tau) * D;
    } else {
      const int hb = head - nha;
      src = src_b + (static_cast<int64_t>(tau) * nhb + hb) * D;
      dst = dst_b + (static_cast<int64_t>(hb) * T + tau) * D;
    }
    const int d0 = part * 8;
    const uint4 av = *reinterpret_cast<const uint4*>(src + d0);
    const uint4 bv = *reinterpret_cast<const uint4*>(src + HALF + d0);
    const __nv_bfloat16* xa = reinterpret_cast<const __nv_bfloat16*>(&av);
    const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(&bv);
    uint4 oa, ob;
    __nv_bfloat16* ya = reinterpret_cast<__nv_bfloat16*>(&oa);
    __nv_bfloat16* yb = reinterpret_cast<__nv_bfloat16*>(&ob);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const double2 rr = cs[r][d0 + e];
      ya[e] = rotate_round(xa[e], xb[e], rr, false);
      yb[e] = rotate_round(xa[e], xb[e], rr, true);
    }
    *reinterpret_cast<uint4*>(dst + d0) = oa;
    *reinterpret_cast<uint4*>(dst + HALF + d0) = ob;
  }
}

// ---------------------------------------------------------------------------
// Backward of the block part, and the final dq of the block tokens.  One CTA per
// (block, KV head): for every query head h of the group and block tokens i, j:
//   P_ij = exp(sigma q~_i . k~_j - lse_i),  dS_ij = P_ij (dO_i . V_j - delta_i)
//   dq~_i = (trunk part, from the trunk backward) + sum_j dS_ij k~_j
//   dk~_j += sum_i dS_ij q~_i,  dV_j += sum_i P_ij dO_i         (over the group's heads)
// then dQ_i = sigma R(a+i)^T dq~_i, dK_j = sigma R(a+j)^T dk~_j, dV_j, all bf16.
// ---------------------------------------------------------------------------
constexpr int kBlockThreads = 128;

template <int D>
struct BlockSmem {
  static constexpr int LD = D + 1;  // padded rows: a column walk touches distinct banks
  static constexpr int kMaxBs = 16;
  // K, V, Q, dO, accK, accV rows; S and dP [Bs][Bs]; cos/sin [Bs][D/2]
  static constexpr size_t bytes(int Bs) {
    return (6 * static_cast<size_t>(Bs) * LD + 2 * static_cast<size_t>(Bs) * Bs + 2 * static_cast<size_t>(Bs) * (D / 2)) *
           sizeof(float);
  }
};

template <int D>
__global__ void __launch_bounds__(kBlockThreads)
    block_bwd_kernel(Geometry g, const __nv_bfloat16* __restrict__ qr, const __nv_bfloat16* __restrict__ kr,
                     const __nv_bfloat16* __restrict__ vb, const __nv_bfloat16* __restrict__ dout,
                     const float* __restrict__ lse, const float* __restrict__ ld, const float* __restrict__ dq_acc,
                     __nv_bfloat16* __restrict__ dq, __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv) {
  using SM = BlockSmem<D>;
  constexpr int LD = SM::LD;
  constexpr int HALF = D / 2;
  extern __shared__ __align__(16) float blk_smem[];
  const int Bs = g.Bs;
  float* sK = blk_smem;
  float* sV = sK + Bs * LD;
  float* sQ = sV + Bs * LD;
  float* sO = sQ + Bs * LD;  // dO
  float* aK = sO + Bs * LD;
  float* aV = aK + Bs * LD;
  float* sS = aV + Bs * LD;  // S, then P
  float* sP = sS + Bs * Bs;  // dP, then dS
  float* sC = sP + Bs * Bs;  // cos [Bs][D/2]
  float* sN = sC + Bs * HALF;  // sin

  const int b = static_cast<int>(blockIdx.x) / g.Hkv;
  const int kvh = static_cast<int>(blockIdx.x) % g.Hkv;
  const int T = g.si.T;  // block rows
  const int row0 = b * Bs;
  int n, pos0;
  token_position(g.si, row0, n, pos0);
  int kstart, klen;
  seq_bounds(g.ksi, n, kstart, klen);
  const int qstart = row0 - pos0;
  const int anchor = block_row_position(g, qstart, pos0, klen);  // position of token 0
  const int gsz = g.H / g.Hkv;
  const int nslots = ld_slots(g.si);
  const int tid = threadIdx.x;

  for (int e = tid; e < Bs * D; e += blockDim.x) {
    const int j = e / D, d = e % D;
    sK[j * LD + d] = __bfloat162float(kr[(static_cast<int64_t>(kvh) * T + row0 + j) * D + d]);
    sV[j * LD + d] = __bfloat162float(vb[(static_cast<int64_t>(row0 + j) * g.Hkv + kvh) * D + d]);
    aK[j * LD + d] = 0.f;
    aV[j * LD + d] = 0.f;
  }
  for (int e = tid; e < Bs * HALF; e += blockDim.x) {
    const int i = e / HALF, d = e % HALF;
    float c, s;
    angle_cos_sin(anchor + i, pow(static_cast<double>(g.theta), -2.0 * d / D), c, s);
    sC[i * HALF + d] = c;
    sN[i * HALF + d] = s;
  }

  for (int hh = 0; hh < gsz; ++hh) {
    const int h = kvh * gsz + hh;
    __syncthreads();  // previous head's readers of sQ / sO / sS / sP are done
    for (int e = tid; e < Bs * D; e += blockDim.x) {
      const int i = e / D, d = e % D;
      sQ[i * LD + d] = __bfloat162float(qr[(static_cast<int64_t>(h) * T + row0 + i) * D + d]);
      sO[i * LD + d] = __bfloat162float(dout[(static_cast<int64_t>(row0 + i) * g.H + h) * D + d]);
    }
    __syncthreads();
    // scores and dP of every (i, j) pair
    for (int e = tid; e < Bs * Bs; e += blockDim.x) {
      const int i = e / Bs, j = e % Bs;
      float s = 0.f, t = 0.f;
#pragma unroll 8
      for (int d = 0; d < D; ++d) {
        s = fmaf(sQ[i * LD + d], sK[j * LD + d], s);
        t = fmaf(sO[i * LD + d], sV[j * LD + d], t);
      }
      const int pos = pos0 + i;
      const float l = lse[lse_index(g.si, g.H, 0, h, n, row0 + i, pos)];
      const float delta = ld[(static_cast<int64_t>(h) * nslots + ld_slot(qstart, n, pos)) * 128 + 64 + (pos & 63)];
      const float p = __expf(s * g.scale - l);
      sS[e] = p;
      sP[e] = p * (t - delta);
    }
    __syncthreads();
    // dq of the block tokens: trunk part + block part, then sigma and R^T
    for (int e = tid; e < Bs * HALF; e += blockDim.x) {
      const int i = e / HALF, d = e % HALF;
      const float* acc = dq_acc + (static_cast<int64_t>(h) * T + row0 + i) * D;
      float x1 = acc[d], x2 = acc[d + HALF];
      for (int j = 0; j < Bs; ++j) {
        const float ds = sP[i * Bs + j];
        x1 = fmaf(ds, sK[j * LD + d], x1);
        x2 = fmaf(ds, sK[j * LD + d + HALF], x2);
      }
      x1 *= g.scale;
      x2 *= g.scale;
      const float c = sC[i * HALF + d], s = sN[i * HALF + d];
      __nv_bfloat16* out = dq + (static_cast<int64_t>(row0 + i) * g.H + h) * D;
      out[d] = __float2bfloat16_rn(fmaf(x1, c, x2 * s));
      out[d + HALF] = __float2bfloat16_rn(fmaf(x2, c, -x1 * s));
    }
    // dk~ and dV of the block keys, summed over the group's heads
    for (int e = tid; e < Bs * D; e += blockDim.x) {
      const int j = e / D, d = e % D;
      float xk = aK[j * LD + d], xv = aV[j * LD + d];
      for (int i = 0; i < Bs; ++i) {
        xk = fmaf(sP[i * Bs + j], sQ[i * LD + d], xk);
        xv = fmaf(sS[i * Bs + j], sO[i * LD + d], xv);
      }
      aK[j * LD + d] = xk;
      aV[j * LD + d] = xv;
    }
  }
  __syncthreads();
  for (int e = tid; e < Bs * HALF; e += blockDim.x) {
    const int j = e / HALF, d = e % HALF;
    const float x1 = aK[j * LD + d] * g.scale, x2 = aK[j * LD + d + HALF] * g.scale;
    const float c = sC[j * HALF + d], s = sN[j * HALF + d];
    __nv_bfloat16* ok = dk + (static_cast<int64_t>(row0 + j) * g.Hkv + kvh) * D;
    ok[d] = __float2bfloat16_rn(fmaf(x1, c, x2 * s));
    ok[d + HALF] = __float2bfloat16_rn(fmaf(x2, c, -x1 * s));
    __nv_bfloat16* ov = dv + (static_cast<int64_t>(row0 + j) * g.Hkv + kvh) * D;
    ov[d] = __float2bfloat16_rn(aV[j * LD + d]);
    ov[d + HALF] = __float2bfloat16_rn(aV[j * LD + d + HALF]);
  }
}

}  // namespace

cudaError_t launch_rope_rows(const Geometry& g, bool block_rows, int T, const void* src_a, int nha, void* dst_a,
                             const void* src_b, int nhb, void* dst_b, cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  const unsigned grid = static_cast<unsigned>((T + kRopeRows - 1) / kRopeRows);
  const RowPositions posf{block_rows};
  auto* a = static_cast<const __nv_bfloat16*>(src_a);
  auto* b = static_cast<const __nv_bfloat16*>(src_b);
  auto* da = static_cast<__nv_bfloat16*>(dst_a);
  auto* db = static_cast<__nv_bfloat16*>(dst_b);
  if (g.D == 128)
    rope_rows_kernel<128><<<grid, kRopeThreads, 0, stream>>>(g, T, posf, a, nha, da, b, nhb, db);
  else
    rope_rows_kernel<64><<<grid, kRopeThreads, 0, stream>>>(g, T, posf, a, nha, da, b, nhb, db);
  return cudaGetLastError();
}

cudaError_t launch_block_bwd(const Geometry& g, const void* qr, const void* kr, const void* vb, const void* dout,
                             const float* lse, const float* ld, const float* dq_acc, void* dq, void* dk, void* dv,
                             cudaStream_t stream) {
  const long long nblocks = static_cast<long long>(g.si.T / g.Bs) * g.Hkv;
  if (nblocks <= 0) return cudaSuccess;
  if (nblocks > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
  auto* q = static_cast<const __nv_bfloat16*>(qr);
  auto* k = static_cast<const __nv_bfloat16*>(kr);
  auto* v = static_cast<const __nv_bfloat16*>(vb);
  auto* o = static_cast<const __nv_bfloat16*>(dout);
  auto* a = static_cast<__nv_bfloat16*>(dq);
  auto* b = static_cast<__nv_bfloat16*>(dk);
  auto* c = static_cast<__nv_bfloat16*>(dv);
  cudaError_t e;
  if (g.D == 128) {
    const size_t smem = BlockSmem<128>::bytes(g.Bs);
    e = cudaFuncSetAttribute(block_bwd_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    block_bwd_kernel<128><<<static_cast<unsigned>(nblocks), kBlockThreads, smem, stream>>>(g, q, k, v, o, lse, ld,
                                                                                          dq_acc, a, b, c);
  } else {
    const size_t smem = BlockSmem<64>::bytes(g.Bs);
    e = cudaFuncSetAttribute(block_bwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    block_bwd_kernel<64><<<static_cast<unsigned>(nblocks), kBlockThreads, smem, stream>>>(g, q, k, v, o, lse, ld,
                                                                                         dq_acc, a, b, c);
  }
  return cudaGetLastError();
}

}  // namespace ttt
