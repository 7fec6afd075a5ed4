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

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

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

template <int D>
__device__ __forceinline__ float dot_row(const float (&a)[2][D / 64], const float (&b)[2][D / 64]) {
  float s = 0.f;
#pragma unroll
  for (int hh = 0; hh < 2; ++hh)
#pragma unroll
    for (int e = 0; e < D / 64; ++e) s = fmaf(a[hh][e], b[hh][e], s);
  return warp_sum(s);
}

// cos/sin of position * theta^(-2d/D) for this lane's E frequencies (double-precision
// argument, the same recipe as the forward rotation).
template <int D>
__device__ __forceinline__ void lane_cos_sin(float theta, int pos, int lane, float (&c)[D / 64], float (&s)[D / 64]) {
#pragma unroll
  for (int e = 0; e < D / 64; ++e) {
    const int d = LaneMap<D>::d(lane, 0, e);
    const double ang = static_cast<double>(pos) * pow(static_cast<double>(theta), -2.0 * d / D);
    double sd, cd;
    sincos(ang, &sd, &cd);
    c[e] = static_cast<float>(cd);
    s[e] = static_cast<float>(sd);
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
// a5: delta = rowsum(dO * O).  Written, with lse * log2(e), into the tile-aligned
// row-statistics array that the trunk backward fetches one 512-byte slot at a time.
// Memory bound (reads O and dO once): D/8 lanes per row, one 16-byte load of each
// per lane, kUnroll rows per lane group in flight.
// ---------------------------------------------------------------------------
constexpr int kUnroll = 4;

template <int D>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    bwd_preprocess_kernel(Geometry g, const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dout,
                          const float* __restrict__ lse, float* __restrict__ ld) {
  constexpr int LPR = D / 8;    // lanes per row
  constexpr int RPW = 32 / LPR;  // rows per warp and step
  const int lane = threadIdx.x & 31;
  const int sub = lane / LPR, c = lane % LPR;
  const int T = g.si.T;
  const int64_t nrows = static_cast<int64_t>(g.P) * T * g.H;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kWarpsPerBlock;
  const int nslots = ld_slots(g.si);
  for (int64_t r0 = (static_cast<int64_t>(blockIdx.x) * kWarpsPerBlock + (threadIdx.x >> 5)) * RPW * kUnroll;
       r0 < nrows; r0 += nwarps * RPW * kUnroll) {
    uint4 a[kUnroll], b[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t row = r0 + u * RPW + sub;
      if (row < nrows) {
        a[u] = __ldg(reinterpret_cast<const uint4*>(o + row * D) + c);
        b[u] = __ldg(reinterpret_cast<const uint4*>(dout + row * D) + c);
      } else {
        a[u] = make_uint4(0, 0, 0, 0);
        b[u] = make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
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
      const int64_t row = r0 + u * RPW + sub;
      if (c == 0 && row < nrows) {
        const int h = static_cast<int>(row % g.H);
        const int64_t pt = row / g.H;
        const int tau = static_cast<int>(pt % T);
        const int p = static_cast<int>(pt / T);
        int n, pos;
        token_position(g.si, tau, n, pos);
        float* slot = ld + ((static_cast<int64_t>(p) * g.H + h) * nslots + ld_slot(tau - pos, n, pos)) * 128;
        slot[pos & 63] = lse[lse_index(g.si, g.H, p, h, n, tau, pos)] * -1.4426950408889634f;
        slot[64 + (pos & 63)] = acc;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// a7 + a8: branch backward and finalisation.  One warp per (token, KV head):
//   for every pass p and group head h:
//     dq~ = dq_acc (trunk part) + sum_j dS_j k~_j        (j = passes 1..p, 0-based)
//     dS_j = P_j (dO . V_j - delta),  P_j = exp(sigma q~ . k~_j - lse)
//     dk~_j += dS_j q~,  dV_j += P_j dO                   (accumulated over p >= j, h)
//     dQ_p = R(i+p)^T (sigma dq~)
//   dK_j = R(i+j)^T (sigma dk~_j)  for every pass (j = 0 takes dk~_1 from the trunk
//   backward), dV_j for j >= 1 (dV_1 is written by the trunk backward).
// Per-warp accumulators for the branch passes live in shared memory.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    branch_bwd_kernel(Geometry g, const __nv_bfloat16* __restrict__ qr, const __nv_bfloat16* __restrict__ kr,
                      const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ dout,
                      const float* __restrict__ lse, const float* __restrict__ ld,
                      const float* __restrict__ dq_acc, const float* __restrict__ dk1_acc,
                      __nv_bfloat16* __restrict__ dq, __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv) {
  extern __shared__ float acc_smem[];
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
  const int NB = g.P - 1;  // branch passes
  // [NB][2 (dk, dv)][D] per warp; lane touches only its own elements
  float* acc = acc_smem + static_cast<int64_t>(wib) * (NB > 0 ? NB : 1) * 2 * D;
  for (int j = 0; j < NB; ++j)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh)
#pragma unroll
      for (int e = 0; e < D / 64; ++e) {
        acc[(j * 2 + 0) * D + LaneMap<D>::d(lane, hh, e)] = 0.f;
        acc[(j * 2 + 1) * D + LaneMap<D>::d(lane, hh, e)] = 0.f;
      }

  for (int p = 0; p < g.P; ++p) {
    float cs_c[D / 64], cs_s[D / 64];
    lane_cos_sin<D>(g.theta, pos + p, lane, cs_c, cs_s);
    for (int hi = 0; hi < gsz; ++hi) {
      const int h = kvh * gsz + hi;
      const int64_t hrow = (static_cast<int64_t>(p) * g.H + h) * T + tau;
      float dqv[2][D / 64];
      load_f32_row<D>(dq_acc + hrow * D, lane, dqv);
      if (p > 0) {
        float q[2][D / 64], dO[2][D / 64];
        load_bf16_row<D>(qr + hrow * D, lane, q);
        load_bf16_row<D>(dout + ((static_cast<int64_t>(p) * T + tau) * g.H + h) * D, lane, dO);
        const int64_t li = lse_index(g.si, g.H, p, h, n, tau, pos);
        const float lse_v = lse[li];
        const float dl = ld[((static_cast<int64_t>(p) * g.H + h) * ld_slots(g.si) + ld_slot(tau - pos, n, pos)) * 128 +
                            64 + (pos & 63)];
        for (int j = 1; j <= p; ++j) {
          float kj[2][D / 64], vj[2][D / 64];
          load_bf16_row<D>(kr + ((static_cast<int64_t>(j) * g.Hkv + kvh) * T + tau) * D, lane, kj);
          load_bf16_row<D>(v + ((static_cast<int64_t>(j) * T + tau) * g.Hkv + kvh) * D, lane, vj);
          const float pj = __expf(dot_row<D>(q, kj) * g.scale - lse_v);
          const float dsj = pj * (dot_row<D>(dO, vj) - dl);
          float* ak = acc + ((j - 1) * 2 + 0) * D;
          float* av = acc + ((j - 1) * 2 + 1) * D;
#pragma unroll
          for (int hh = 0; hh < 2; ++hh)
#pragma unroll
            for (int e = 0; e < D / 64; ++e) {
              const int d = LaneMap<D>::d(lane, hh, e);
              dqv[hh][e] = fmaf(dsj, kj[hh][e], dqv[hh][e]);
              ak[d] = fmaf(dsj, q[hh][e], ak[d]);
              av[d] = fmaf(pj, dO[hh][e], av[d]);
            }
        }
      }
#pragma unroll
      for (int hh = 0; hh < 2; ++hh)
#pragma unroll
        for (int e = 0; e < D / 64; ++e) dqv[hh][e] *= g.scale;
      rotate_back<D>(dqv, cs_c, cs_s);
      store_bf16_row<D>(dq + ((static_cast<int64_t>(p) * T + tau) * g.H + h) * D, lane, dqv);
    }
  }
  // dK of every pass (trunk from the trunk backward), dV of the branch passes
  for (int j = 0; j < g.P; ++j) {
    float cs_c[D / 64], cs_s[D / 64];
    lane_cos_sin<D>(g.theta, pos + j, lane, cs_c, cs_s);
    float kx[2][D / 64];
    if (j == 0) {
      load_f32_row<D>(dk1_acc + (static_cast<int64_t>(kvh) * T + tau) * D, lane, kx);
    } else {
#pragma unroll
      for (int hh = 0; hh < 2; ++hh)
#pragma unroll
        for (int e = 0; e < D / 64; ++e) kx[hh][e] = acc[((j - 1) * 2 + 0) * D + LaneMap<D>::d(lane, hh, e)];
    }
#pragma unroll
    for (int hh = 0; hh < 2; ++hh)
#pragma unroll
      for (int e = 0; e < D / 64; ++e) kx[hh][e] *= g.scale;
    rotate_back<D>(kx, cs_c, cs_s);
    const int64_t krow = ((static_cast<int64_t>(j) * T + tau) * g.Hkv + kvh) * D;
    store_bf16_row<D>(dk + krow, lane, kx);
    if (j > 0) {
      float vx[2][D / 64];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh)
#pragma unroll
        for (int e = 0; e < D / 64; ++e) vx[hh][e] = acc[((j - 1) * 2 + 1) * D + LaneMap<D>::d(lane, hh, e)];
      store_bf16_row<D>(dv + krow, lane, vx);
    }
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
                                  cudaStream_t stream) {
  const int64_t rows = static_cast<int64_t>(g.P) * g.si.T * g.H;
  if (rows == 0) return cudaSuccess;
  const int rpw = 32 / (g.D / 8);
  const int64_t warps = (rows + rpw * kUnroll - 1) / (rpw * kUnroll);
  const unsigned blocks = static_cast<unsigned>(std::min<int64_t>(blocks_for(warps), 148 * 32));
  auto* ob = static_cast<const __nv_bfloat16*>(o);
  auto* db = static_cast<const __nv_bfloat16*>(dout);
  if (g.D == 128)
    bwd_preprocess_kernel<128><<<blocks, kWarpsPerBlock * 32, 0, stream>>>(g, ob, db, lse, ld);
  else
    bwd_preprocess_kernel<64><<<blocks, kWarpsPerBlock * 32, 0, stream>>>(g, ob, db, lse, ld);
  return cudaGetLastError();
}

cudaError_t launch_branch_bwd(const Geometry& g, const void* qr, const void* kr, const void* v, const void* dout,
                              const float* lse, const float* ld, const float* dq_acc, const float* dk1_acc,
                              void* dq, void* dk, void* dv, cudaStream_t stream) {
  const int64_t warps = static_cast<int64_t>(g.si.T) * g.Hkv;
  if (warps == 0) return cudaSuccess;
  const int NB = g.P - 1 > 0 ? g.P - 1 : 1;
  const size_t smem = static_cast<size_t>(kWarpsPerBlock) * NB * 2 * g.D * sizeof(float);
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
                                                                                      dq_acc, dk1_acc, dqb, dkb, dvb);
  } else {
    e = cudaFuncSetAttribute(branch_bwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    branch_bwd_kernel<64><<<blocks_for(warps), kWarpsPerBlock * 32, smem, stream>>>(g, qb, kb, vb, db, lse, ld,
                                                                                     dq_acc, dk1_acc, dqb, dkb, dvb);
  }
  return cudaGetLastError();
}

cudaError_t launch_watchdog_selftest(uint32_t* status, uint64_t budget_ns, cudaStream_t stream) {
  watchdog_selftest_kernel<<<1, 32, 0, stream>>>(status, budget_ns);
  return cudaGetLastError();
}

}  // namespace ttt
