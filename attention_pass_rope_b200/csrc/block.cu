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
// tensors that share the rows' positions (rotate-half RoPE rounded as in fp64, bf16 out;
// outputs head-major so that a (head, 128-row) tile is one contiguous block for TMA).
template <int D>
__global__ void __launch_bounds__(kRopeThreads) rope_rows_kernel(Geometry g, int T, RowPositions posf,
                                                                 const __nv_bfloat16* __restrict__ src_a, int nha,
                                                                 __nv_bfloat16* __restrict__ dst_a,
                                                                 const __nv_bfloat16* __restrict__ src_b, int nhb,
                                                                 __nv_bfloat16* __restrict__ dst_b) {
  constexpr int HALF = D / 2;
  constexpr int PARTS = HALF / 8;
  __shared__ float2 cs_hi[kRopeRows][HALF], cs_lo[kRopeRows][HALF];
  const int r0 = blockIdx.x * kRopeRows;
  const int nrows = min(kRopeRows, T - r0);
  for (int e = threadIdx.x; e < kRopeRows * HALF; e += blockDim.x) {
    const int r = e / HALF, d = e % HALF;
    if (r >= nrows) continue;
    const double inv_freq = pow(static_cast<double>(g.theta), -2.0 * d / D);
    double s, c;
    sincos(static_cast<double>(posf(g, r0 + r)) * inv_freq, &s, &c);
    cos_sin_split(c, s, cs_hi[r][d], cs_lo[r][d]);
  }
  __syncthreads();
  // every thread keeps one (row, 8-element part) slot and walks the heads, so that it
  // reads its cos / sin from shared memory once
  static_assert(kRopeThreads % (kRopeRows * PARTS) == 0, "threads must cover whole slots");
  constexpr int kHeadLanes = kRopeThreads / (kRopeRows * PARTS);
  const int NH = nha + nhb;
  const int slot = threadIdx.x % (kRopeRows * PARTS);
  const int part = slot % PARTS;
  const int r = slot / PARTS;
  if (r >= nrows) return;
  const int d0 = part * 8;
  float2 rh[8], rl[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    rh[e] = cs_hi[r][d0 + e];
    rl[e] = cs_lo[r][d0 + e];
  }
  const int tau = r0 + r;
  for (int head = threadIdx.x / (kRopeRows * PARTS); head < NH; head += kHeadLanes) {
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
    const uint4 av = *reinterpret_cast<const uint4*>(src + d0);
    const uint4 bv = *reinterpret_cast<const uint4*>(src + HALF + d0);
    uint4 oa, ob;
    rotate8_round(av, bv, rh, rl, oa, ob);
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
// The group's heads are stacked into up to 64 query rows (r = head * Bs + i) so that
// every product is a small matrix product over shared memory; each thread computes a
// register block of it (4x4 scores, 4 rows x 16 columns of dq, 4 keys x 8 columns of
// dk~ / dV), which keeps shared-memory traffic per multiply-add low.
// ---------------------------------------------------------------------------
constexpr int kBlockThreads = 128;
constexpr int kBlockRows = 64;  // stacked query rows per pass over the group's heads

template <int D>
struct BlockSmem {
  static constexpr int LD = D + 4;   // fp32 row stride (floats): 16-byte aligned rows, staggered banks
  static constexpr int LDH = D + 8;  // bf16 row stride (elements): 16-byte aligned rows, staggered banks
  static constexpr int BP = 16;      // block keys, padded
  // Q, dO bf16 [64][LDH] (at the end: dk~ / dV fp32 [16][LD] over them); K, V [16][LD];
  // P, dS [64][16]; cos, sin [16][D/2]; lse, delta [64]; then the inverse frequencies
  // (double [D/2]).  bf16 staging of Q and dO keeps three CTAs on an SM.
  static_assert(kBlockRows * LDH * 2 >= 16 * LD * 4, "dk~ / dV fit over the staged rows");
  static constexpr size_t kFloats = kBlockRows * LDH + 2 * BP * LD + 2 * kBlockRows * BP + 2 * BP * (D / 2) +
                                    2 * kBlockRows;
  static constexpr size_t bytes = kFloats * sizeof(float) + (D / 2) * sizeof(double);
};

__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ void fma4(float (&acc)[4], float a, const float4& b) {
  acc[0] = fmaf(a, b.x, acc[0]);
  acc[1] = fmaf(a, b.y, acc[1]);
  acc[2] = fmaf(a, b.z, acc[2]);
  acc[3] = fmaf(a, b.w, acc[3]);
}
__device__ __forceinline__ float dot4(const float4& a, const float4& b, float acc) {
  return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, fmaf(a.w, b.w, acc))));
}
__device__ __forceinline__ float4 bf4u(const uint2 u) {  // 4 bf16 (as loaded) -> float4
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
  return make_float4(a.x, a.y, b.x, b.y);
}
constexpr int kLoadBatch = 8;

template <int D>
__global__ void __launch_bounds__(kBlockThreads)
    block_bwd_kernel(Geometry g, const __nv_bfloat16* __restrict__ qr, const __nv_bfloat16* __restrict__ kr,
                     const __nv_bfloat16* __restrict__ vb, const __nv_bfloat16* __restrict__ dout,
                     const float* __restrict__ lse, const float* __restrict__ ld, const float* __restrict__ dq_acc,
                     __nv_bfloat16* __restrict__ dq, __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv) {
  using SM = BlockSmem<D>;
  constexpr int LD = SM::LD;
  constexpr int LDH = SM::LDH;
  constexpr int BP = SM::BP;
  constexpr int HALF = D / 2;
  extern __shared__ __align__(16) float blk_smem[];
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(blk_smem);  // [64][LDH]
  __nv_bfloat16* sO = sQ + kBlockRows * LDH;                        // [64][LDH] dO
  float* sK = reinterpret_cast<float*>(sO + kBlockRows * LDH);      // [16][LD]
  float* sV = sK + BP * LD;              // [16][LD]
  float* sP = sV + BP * LD;              // [64][16] scores, then P
  float* sD = sP + kBlockRows * BP;      // [64][16] dP, then dS
  float* sC = sD + kBlockRows * BP;      // [16][D/2] cos
  float* sN = sC + BP * HALF;            // [16][D/2] sin
  float* sL = sN + BP * HALF;            // [64] lse
  float* sDl = sL + kBlockRows;          // [64] delta
  double* sF = reinterpret_cast<double*>(blk_smem + SM::kFloats);  // [D/2] inverse frequencies

  const int Bs = g.Bs;
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
  const int hc = max(1, min(gsz, kBlockRows / Bs));  // heads per pass
  const int nslots = ld_slots(g.si);
  const int tid = threadIdx.x;

  // block keys / values (rows >= Bs zero), cos / sin of the block's positions
  {
    constexpr int kIt = (BP * (D / 4) + kBlockThreads - 1) / kBlockThreads;
    uint2 ka[kIt], va[kIt];
#pragma unroll
    for (int u = 0; u < kIt; ++u) {
      const int e = tid + u * kBlockThreads;
      const int j = e / (D / 4), d = 4 * (e % (D / 4));
      ka[u] = va[u] = make_uint2(0u, 0u);
      if (e < BP * (D / 4) && j < Bs) {
        ka[u] = *reinterpret_cast<const uint2*>(kr + (static_cast<int64_t>(kvh) * T + row0 + j) * D + d);
        va[u] = *reinterpret_cast<const uint2*>(vb + (static_cast<int64_t>(row0 + j) * g.Hkv + kvh) * D + d);
      }
    }
#pragma unroll
    for (int u = 0; u < kIt; ++u) {
      const int e = tid + u * kBlockThreads;
      if (e >= BP * (D / 4)) break;
      const int j = e / (D / 4), d = 4 * (e % (D / 4));
      *reinterpret_cast<float4*>(sK + j * LD + d) = bf4u(ka[u]);
      *reinterpret_cast<float4*>(sV + j * LD + d) = bf4u(va[u]);
    }
  }
  for (int d = tid; d < HALF; d += blockDim.x) sF[d] = pow(static_cast<double>(g.theta), -2.0 * d / D);
  __syncthreads();
  for (int e = tid; e < Bs * HALF; e += blockDim.x) {
    const int i = e / HALF, d = e % HALF;
    float c, s;
    angle_cos_sin(anchor + i, sF[d], c, s);
    sC[i * HALF + d] = c;
    sN[i * HALF + d] = s;
  }

  // dk~ / dV accumulators: thread -> (4 keys, 8 columns) of dk~ (tid < 64) or of dV
  const bool acc_v = tid >= 64;
  const int akb = (tid & 63) / (D / 8);        // key block (4 keys)
  const int acol = 8 * ((tid & 63) % (D / 8));  // 8 consecutive columns
  const bool acc_on = akb < BP / 4;
  float acc[4][8] = {};

  for (int h0 = 0; h0 < gsz; h0 += hc) {
    const int nh = min(hc, gsz - h0);
    const int R = nh * Bs;
    const int RP = (R + 3) & ~3;
    __syncthreads();  // the previous pass's readers of sQ / sO / sP / sD are done
    // kLoadBatch iterations' loads are issued before any of them is converted and stored,
    // so that a thread waits for one round trip per batch rather than per element group
    for (int e0 = tid; e0 < RP * (D / 4); e0 += kLoadBatch * kBlockThreads) {
      uint2 qa[kLoadBatch], oa[kLoadBatch];
#pragma unroll
      for (int u = 0; u < kLoadBatch; ++u) {
        const int e = e0 + u * kBlockThreads;
        const int r = e / (D / 4), d = 4 * (e % (D / 4));
        qa[u] = oa[u] = make_uint2(0u, 0u);
        if (e < RP * (D / 4) && r < R) {
          const int h = kvh * gsz + h0 + r / Bs, i = r % Bs;
          qa[u] = *reinterpret_cast<const uint2*>(qr + (static_cast<int64_t>(h) * T + row0 + i) * D + d);
          oa[u] = *reinterpret_cast<const uint2*>(dout + (static_cast<int64_t>(row0 + i) * g.H + h) * D + d);
        }
      }
#pragma unroll
      for (int u = 0; u < kLoadBatch; ++u) {
        const int e = e0 + u * kBlockThreads;
        if (e >= RP * (D / 4)) break;
        const int r = e / (D / 4), d = 4 * (e % (D / 4));
        *reinterpret_cast<uint2*>(sQ + r * LDH + d) = qa[u];
        *reinterpret_cast<uint2*>(sO + r * LDH + d) = oa[u];
      }
    }
    for (int r = tid; r < RP; r += blockDim.x) {
      float l = 0.f, dl = 0.f;
      if (r < R) {
        const int h = kvh * gsz + h0 + r / Bs, pos = pos0 + r % Bs;
        l = lse[lse_index(g.si, g.H, 0, h, n, row0 + r % Bs, pos)];
        dl = ld[(static_cast<int64_t>(h) * nslots + ld_slot(qstart, n, pos)) * 128 + 64 + (pos & 63)];
      }
      sL[r] = l;
      sDl[r] = dl;
    }
    __syncthreads();
    // scores (threads 0..63) and dP (64..127), 4x4 blocks of (rows, keys)
    {
      const int blk = tid & 63;
      const int rb = blk / (BP / 4), cb = blk % (BP / 4);
      if (4 * rb < RP) {
        const __nv_bfloat16* A = tid < 64 ? sQ : sO;
        const float* Bm = tid < 64 ? sK : sV;
        float s[4][4] = {};
#pragma unroll 4
        for (int d = 0; d < D; d += 4) {
          float4 a[4], bb[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) a[u] = bf4u(*reinterpret_cast<const uint2*>(A + (4 * rb + u) * LDH + d));
#pragma unroll
          for (int v = 0; v < 4; ++v) bb[v] = ld4(Bm + (4 * cb + v) * LD + d);
#pragma unroll
          for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int v = 0; v < 4; ++v) s[u][v] = dot4(a[u], bb[v], s[u][v]);
        }
        float* out = tid < 64 ? sP : sD;
#pragma unroll
        for (int u = 0; u < 4; ++u)
          *reinterpret_cast<float4*>(out + (4 * rb + u) * BP + 4 * cb) = make_float4(s[u][0], s[u][1], s[u][2], s[u][3]);
      }
    }
    __syncthreads();
    // P = exp(sigma s - lse), dS = P (dP - delta); padding rows and keys give 0
    for (int e = tid; e < RP * BP; e += blockDim.x) {
      const int r = e / BP, j = e % BP;
      float p = 0.f, ds = 0.f;
      if (r < R && j < Bs) {
        p = __expf(sP[e] * g.scale - sL[r]);
        ds = p * (sD[e] - sDl[r]);
      }
      sP[e] = p;
      sD[e] = ds;
    }
    __syncthreads();
    // dq of the rows: 4 rows x (8 + 8 paired) columns per item
    for (int item = tid; item < (RP / 4) * (HALF / 8); item += blockDim.x) {
      const int rb = item / (HALF / 8), c = 8 * (item % (HALF / 8));
      float lo[4][8] = {}, hi[4][8] = {};
      for (int j = 0; j < Bs; ++j) {
        const float4 k0 = ld4(sK + j * LD + c), k1 = ld4(sK + j * LD + c + 4);
        const float4 k2 = ld4(sK + j * LD + HALF + c), k3 = ld4(sK + j * LD + HALF + c + 4);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float ds = sD[(4 * rb + u) * BP + j];
          float (&l4a)[4] = *reinterpret_cast<float(*)[4]>(&lo[u][0]);
          float (&l4b)[4] = *reinterpret_cast<float(*)[4]>(&lo[u][4]);
          float (&h4a)[4] = *reinterpret_cast<float(*)[4]>(&hi[u][0]);
          float (&h4b)[4] = *reinterpret_cast<float(*)[4]>(&hi[u][4]);
          fma4(l4a, ds, k0);
          fma4(l4b, ds, k1);
          fma4(h4a, ds, k2);
          fma4(h4b, ds, k3);
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int r = 4 * rb + u;
        if (r >= R) continue;
        const int h = kvh * gsz + h0 + r / Bs, i = r % Bs;
        const float* acc_row = dq_acc + (static_cast<int64_t>(h) * T + row0 + i) * D;
        __nv_bfloat16* out = dq + (static_cast<int64_t>(row0 + i) * g.H + h) * D;
        uint32_t plo[4], phi[4];
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
          float y[2][2];
#pragma unroll
          for (int w = 0; w < 2; ++w) {
            const int d = c + e + w;
            const float x1 = (acc_row[d] + lo[u][e + w]) * g.scale;
            const float x2 = (acc_row[d + HALF] + hi[u][e + w]) * g.scale;
            const float cs = sC[i * HALF + d], sn = sN[i * HALF + d];
            y[0][w] = fmaf(x1, cs, x2 * sn);
            y[1][w] = fmaf(x2, cs, -x1 * sn);
          }
          plo[e >> 1] = pack_bf16x2(y[0][0], y[0][1]);
          phi[e >> 1] = pack_bf16x2(y[1][0], y[1][1]);
        }
        *reinterpret_cast<uint4*>(out + c) = make_uint4(plo[0], plo[1], plo[2], plo[3]);
        *reinterpret_cast<uint4*>(out + HALF + c) = make_uint4(phi[0], phi[1], phi[2], phi[3]);
      }
    }
    // dk~ (sum of dS q~) and dV (sum of P dO) over this pass's rows
    if (acc_on) {
      const float* W = acc_v ? sP : sD;  // P for dV, dS for dk~
      const __nv_bfloat16* X = acc_v ? sO : sQ;
      for (int r = 0; r < R; ++r) {
        const float4 w4 = ld4(W + r * BP + 4 * akb);
        const uint4 xr = *reinterpret_cast<const uint4*>(X + r * LDH + acol);
        const float4 x0 = bf4u(make_uint2(xr.x, xr.y)), x1 = bf4u(make_uint2(xr.z, xr.w));
        const float w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          float (&a0)[4] = *reinterpret_cast<float(*)[4]>(&acc[v][0]);
          float (&a1)[4] = *reinterpret_cast<float(*)[4]>(&acc[v][4]);
          fma4(a0, w[v], x0);
          fma4(a1, w[v], x1);
        }
      }
    }
  }
  // dk~ and dV to shared memory (over sQ / sO), then dK = sigma R^T dk~ and dV in bf16
  __syncthreads();
  float* fQ = reinterpret_cast<float*>(sQ);  // dk~ [16][LD] over the staged rows
  float* fO = reinterpret_cast<float*>(sO);  // dV [16][LD]
  if (acc_on) {
    float* dst = acc_v ? fO : fQ;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      *reinterpret_cast<float4*>(dst + (4 * akb + v) * LD + acol) =
          make_float4(acc[v][0], acc[v][1], acc[v][2], acc[v][3]);
      *reinterpret_cast<float4*>(dst + (4 * akb + v) * LD + acol + 4) =
          make_float4(acc[v][4], acc[v][5], acc[v][6], acc[v][7]);
    }
  }
  __syncthreads();
  for (int e = tid; e < Bs * HALF; e += blockDim.x) {
    const int j = e / HALF, d = e % HALF;
    const float x1 = fQ[j * LD + d] * g.scale, x2 = fQ[j * LD + d + HALF] * g.scale;
    const float c = sC[j * HALF + d], s = sN[j * HALF + d];
    __nv_bfloat16* ok = dk + (static_cast<int64_t>(row0 + j) * g.Hkv + kvh) * D;
    ok[d] = __float2bfloat16_rn(fmaf(x1, c, x2 * s));
    ok[d + HALF] = __float2bfloat16_rn(fmaf(x2, c, -x1 * s));
    __nv_bfloat16* ov = dv + (static_cast<int64_t>(row0 + j) * g.Hkv + kvh) * D;
    ov[d] = __float2bfloat16_rn(fO[j * LD + d]);
    ov[d + HALF] = __float2bfloat16_rn(fO[j * LD + d + HALF]);
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
    const size_t smem = BlockSmem<128>::bytes;
    e = cudaFuncSetAttribute(block_bwd_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    block_bwd_kernel<128><<<static_cast<unsigned>(nblocks), kBlockThreads, smem, stream>>>(g, q, k, v, o, lse, ld,
                                                                                          dq_acc, a, b, c);
  } else {
    const size_t smem = BlockSmem<64>::bytes;
    e = cudaFuncSetAttribute(block_bwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    block_bwd_kernel<64><<<static_cast<unsigned>(nblocks), kBlockThreads, smem, stream>>>(g, q, k, v, o, lse, ld,
                                                                                         dq_acc, a, b, c);
  }
  return cudaGetLastError();
}

}  // namespace ttt
