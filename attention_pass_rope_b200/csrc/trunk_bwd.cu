// a6: trunk backward on the 5th-generation tensor cores.
//
// Gradient of the trunk half of the two-part attention ("DFlash/DSpark and EAGLE-3
// TTT draft co-training ...", NeMo-RL issue 3698, "What I'm working on", item 1),
// recomputing the probabilities from the MERGED log-sum-exp, so that the branch
// keys' share of each row's softmax is accounted for exactly:
//   P = exp(s - lse),  dP = dO V^T,  dS = P (dP - delta),  delta = rowsum(dO * O)
//   dV_1 += P^T dO,  dk~_1 += dS^T q~,  dq~ += dS k~_1      (sigma applied later)
//
// One CTA owns one 128-key tile of one KV head and walks every 64-row query tile at
// or after the tile's diagonal (the last one first) and, for each, every (pass, group
// head) query head, keeping dK and dV of its keys in TMEM for the whole walk (no
// atomics on dK/dV).
// Transposed products keep the key dimension on the TMEM lanes:
//   S^T  = K~ Q~^T        (M=128 keys, N=64 queries)      SS
//   dP^T = V dO^T         (M=128 keys, N=64)              SS
//   dV  += P^T dO         (M=128, N=D, K=64 queries)      TS  (P^T in TMEM, bf16)
//   dK  += dS^T Q~        (M=128, N=D, K=64)              SS  (dS^T in smem, bf16)
//   dQ^T = K~^T dS^T      (M=128 rows of d, N=64, K=128)  SS  (both MN-major)
// dQ^T goes TMEM -> registers -> smem (fp32, row-major [q][d], two staging buffers of
// 32 rows) and is added to the fp32 dq~ accumulator by bulk reduce-adds, in arrival
// order, or in key-tile order under TTT_FLAG_DETERMINISTIC_DQ (per-tile tickets).
//
// CTA = 16 warps: warp 0 TMA producer (+ lse/delta rows), warp 1 TMEM allocator and
// S^T/dP^T issuer, warp 2 dV/dK/dQ^T issuer, warps 4-7 and 8-11 the two halves (query
// columns 0-31 / 32-63) of the probability / dS step, warps 12-15 the dQ writer.
// S^T/dP^T of step n+1 are issued as soon as the P/dS warps have read step n's into
// registers, so they are complete before those warps finish step n, and the
// dV/dK/dQ^T products of step n run under the CUDA-core work of step n+1.  P^T and
// dS^T are double buffered for that reason; S^T/dP^T are single buffered.
#include "common.cuh"

namespace ttt {

namespace {

template <int D>
struct BwdCfg {
  static constexpr int BK = 128;  // keys per CTA
  static constexpr int BQ = 64;   // queries per step
  static constexpr int ST = 3;    // Q~/dO ring stages
  static constexpr int KCH = D / 64;
  static constexpr int KCHUNK = 128 * 128;   // 128 rows x 64 bf16
  static constexpr int QCHUNK = 64 * 128;    // 64 rows x 64 bf16
  static constexpr int KTILE = 2 * KCHUNK;   // K~ always 2 chunks (D=64: chunk 1 is zero padding)
  static constexpr int VTILE = KCH * KCHUNK;
  static constexpr int QTILE = KCH * QCHUNK;
  static constexpr int DSTILE = 128 * 128;   // 128 keys x 64 queries bf16
  static constexpr int DQSTAGE = 32 * D * 4;    // half a query tile of dQ, fp32
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + KTILE;
  static constexpr int OFF_Q = OFF_V + (VTILE < KCHUNK ? KCHUNK : VTILE);
  static constexpr int OFF_DO = OFF_Q + ST * QTILE;
  static constexpr int OFF_DS = OFF_DO + ST * QTILE;
  static constexpr int OFF_DQ = OFF_DS + 2 * DSTILE;
  static constexpr int OFF_LD = OFF_DQ + 2 * DQSTAGE;      // [ST][2][64] floats: lse*log2e, delta
  static constexpr int OFF_BAR = OFF_LD + ST * 2 * BQ * 4;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_USED = OFF_BAR + BAR_BYTES;
  static constexpr int SMEM = (SMEM_USED < 120 * 1024 ? 120 * 1024 : SMEM_USED) + 1024;
  static_assert(SMEM <= 227 * 1024, "dynamic shared memory above the per-block limit");
  static constexpr int COL_DV = 0;
  static constexpr int COL_DK = D;
  static constexpr int COL_S = 2 * D;
  static constexpr int COL_DP = 2 * D + 64;
  static constexpr int COL_DQ = 2 * D + 128;
  static constexpr int COL_PT = 2 * D + 192;  // two buffers of 32 columns
  static constexpr int TMEM_COLS = 512;
  static constexpr int THREADS = 512;
};

constexpr float kLog2e = 1.4426950408889634f;

struct IterInfo {
  int p, h, q0;
};

// Walk order: query tiles from the last one down to the diagonal (outer), the G =
// P * (H / Hkv) query heads of this KV head (inner).  CTAs of the same KV head that
// run at the same time then read the same q~/dO tiles and reduce into the same dq~
// rows within a short window, so both stay in L2.
__device__ __forceinline__ IterInfo decode_iter(int it, int nqt, int jq0, int G, int gsz, int kvh) {
  const int qh = it % G;
  IterInfo r;
  r.p = qh / gsz;
  r.h = kvh * gsz + qh % gsz;
  r.q0 = (jq0 + nqt - 1 - it / G) * 64;
  return r;
}

// First 64-row query tile of a block-draft sequence whose last row sees key k0
// (anchors non-decreasing within a sequence, so the tiles that see k0 are a suffix).
__device__ int first_tile_seeing(const Geometry& g, const int* qlim, int qstart, int qlen, int k0) {
  int lo = 0, hi = (qlen + 63) / 64;  // answer in [lo, hi]; hi = no tile
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    const int last = min(mid * 64 + 63, qlen - 1);
    if (__ldg(qlim + qstart + last) >= k0)
      hi = mid;
    else
      lo = mid + 1;
  }
  return lo;
}

// Last 64-row query tile of a block-draft sequence whose first row still sees a key of
// [k0, k1] (for a sliding-window layer the first key of a row is block_row_start of its
// limit, non-decreasing too, so the tiles that see the key tile are a range).
__device__ int last_tile_seeing(const Geometry& g, const int* qlim, int qstart, int qlen, int k1) {
  int lo = -1, hi = (qlen + 63) / 64 - 1;  // answer in [lo, hi]; -1 = no tile
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (block_row_start(g, __ldg(qlim + qstart + mid * 64)) <= k1)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

// dK of the trunk keys, finalised: sigma * R(pos)^T dk~ in bf16, for one key row held
// by the calling thread as 32-column chunks (c, c + D/2 pair the RoPE dimensions).
template <int D>
__device__ __forceinline__ void store_dk_row(__nv_bfloat16* dst, int pos, float theta, float scale,
                                             const uint32_t (&lo)[32], const uint32_t (&hi)[32], int c) {
  // inverse frequencies theta^(-2d/D) for d = 32c .. 32c+31: one pow, then a ratio
  const double ratio = pow(static_cast<double>(theta), -2.0 / D);
  double f = pow(static_cast<double>(theta), -2.0 * (32 * c) / D);
  uint32_t out_lo[16], out_hi[16];
#pragma unroll
  for (int e = 0; e < 32; e += 2) {
    float r[2][2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      float cs, sn;
      angle_cos_sin(pos, f, cs, sn);
      f *= ratio;
      const float x1 = __uint_as_float(lo[e + u]) * scale, x2 = __uint_as_float(hi[e + u]) * scale;
      r[0][u] = fmaf(x1, cs, x2 * sn);
      r[1][u] = fmaf(x2, cs, -x1 * sn);
    }
    out_lo[e >> 1] = pack_bf16x2(r[0][0], r[0][1]);
    out_hi[e >> 1] = pack_bf16x2(r[1][0], r[1][1]);
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    *reinterpret_cast<uint4*>(dst + 32 * c + 8 * q) =
        make_uint4(out_lo[4 * q], out_lo[4 * q + 1], out_lo[4 * q + 2], out_lo[4 * q + 3]);
    *reinterpret_cast<uint4*>(dst + D / 2 + 32 * c + 8 * q) =
        make_uint4(out_hi[4 * q], out_hi[4 * q + 1], out_hi[4 * q + 2], out_hi[4 * q + 3]);
  }
}

// MODE 0: TTT trunk (queries and keys are the same tokens, causal).  MODE 1: block-draft
// trunk (queries are block rows, keys the context; a query row sees the keys up to its
// block's anchor, a.qlim).  MODE 2: one step of the context-parallel ring (queries are a
// chunk of the sequence, keys a visiting chunk; row r sees key t iff t <= r +
// g.limit_off); the keys' dk~ and dV are added to fp32 accumulators that travel with the
// chunk, the dq~ of the rows as in MODE 0.  MODE 3: MODE 1 for a sliding-window layer (a
// row sees the keys from block_row_start of its limit up to the limit); a mode of its own
// so that the window's bounds cost nothing in the plain block-draft kernel.
template <int D, int MODE>
__global__ void __launch_bounds__(BwdCfg<D>::THREADS, 1)
    trunk_bwd_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                     const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_do,
                     const TrunkBwdArgs a) {
  using C = BwdCfg<D>;
  constexpr bool BLOCK = MODE == 1 || MODE == 3;
  constexpr bool WIN = MODE == 3;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);

  const Geometry& g = a.g;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) TTT_CTA_MARK(0);

  // ---- work item: (key tile jk, sequence n, KV head).  The (sequence, KV head) groups
  // go in bands of nb groups, about 256 CTAs per band; inside a band the smallest jk
  // (most work) comes first.  The CTAs resident at one time then belong to few groups,
  // so the q~/dO tiles they read and the dq~ rows they reduce into are shared in L2
  // (with every group in flight at once, a batch of many short sequences streams all
  // of it from DRAM), while the work per band still runs largest first.
  const int njk = (g.ksi.max_len + C::BK - 1) / C::BK;
  const int ngroups = g.si.nseq * g.Hkv;
  const int nb = max(1, 256 / njk);
  const int band = static_cast<int>(blockIdx.x) / (nb * njk);
  const int in_band = static_cast<int>(blockIdx.x) % (nb * njk);
  const int members = min(nb, ngroups - band * nb);
  const int jk = in_band / members;
  const int gi = band * nb + in_band % members;
  const int n = gi / g.Hkv;
  const int kvh = gi % g.Hkv;
  int seq_start, len, kstart, klen;
  seq_bounds(g.si, n, seq_start, len);  // query rows
  seq_bounds(g.ksi, n, kstart, klen);   // key rows (the same tokens in MODE 0)
  const int k0 = jk * C::BK;
  if (k0 >= klen) return;
  const int gsz = g.H / g.Hkv;
  const int G = g.P * gsz;
  const int off = MODE == 2 ? g.limit_off : 0;  // row r sees key t iff t <= r + off (MODE 0, 2)
  const int jq0 = BLOCK ? first_tile_seeing(g, a.qlim, seq_start, len, k0) : max(k0 - off, 0) / C::BQ;
  const int jq1 = WIN ? last_tile_seeing(g, a.qlim, seq_start, len, k0 + C::BK - 1) : (len + C::BQ - 1) / C::BQ - 1;
  const int nqt = max(jq1 - jq0 + 1, 0);
  const int NIT = G * nqt;
  if (threadIdx.x == 0) TTT_CTA_INFO(NIT);
  if (NIT <= 0) {
    if (MODE == 2) return;  // the accumulators keep what other steps added
    // block-draft keys that no query row sees: zero gradients
    for (int i = threadIdx.x; i < C::BK * (D / 8); i += blockDim.x) {
      const int r = i / (D / 8), c8 = i % (D / 8);
      if (k0 + r >= klen) continue;
      const int64_t row = (static_cast<int64_t>(kstart + k0 + r) * g.Hkv + kvh) * D + 8 * c8;
      *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.dk) + row) = make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.dv) + row) = make_uint4(0, 0, 0, 0);
    }
    return;
  }

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* kv_bar = bars + 0;
  uint64_t* qdo_full = bars + 1;            // [ST]
  uint64_t* qdo_empty = bars + 1 + C::ST;   // [ST]
  uint64_t* sdp_full = bars + 1 + 2 * C::ST;
  uint64_t* sdp_free = sdp_full + 1;
  uint64_t* ds_ready = sdp_free + 1;        // [2], by step parity
  uint64_t* mma_done = ds_ready + 2;        // [2]
  uint64_t* dq_full = mma_done + 2;
  uint64_t* dq_free = dq_full + 1;
  uint64_t* final_bar = dq_free + 1;
  uint64_t* drain = final_bar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  uint32_t* abort_flag = tmem_slot + 1;

  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sDO = smem + C::OFF_DO;
  uint8_t* sDS = smem + C::OFF_DS;
  float* sDQ = reinterpret_cast<float*>(smem + C::OFF_DQ);
  float* sLD = reinterpret_cast<float*>(smem + C::OFF_LD);

  if (D == 64) {
    // zero padding rows d = 64..127 of K~ (the dQ^T product runs with M = 128)
    uint4* z = reinterpret_cast<uint4*>(sK + C::KCHUNK);
    for (int i = threadIdx.x; i < C::KCHUNK / 16; i += blockDim.x) z[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  if (threadIdx.x == 0) {
    mbar_init(kv_bar, 1);
    for (int s = 0; s < C::ST; ++s) {
      mbar_init(qdo_full + s, 1);
      mbar_init(qdo_empty + s, 1);
    }
    mbar_init(sdp_full, 1);
    mbar_init(sdp_free, 8);   // one arrival per P/dS warp
    mbar_init(ds_ready + 0, 8);   // one arrival per P/dS warp
    mbar_init(ds_ready + 1, 8);
    mbar_init(mma_done + 0, 1);
    mbar_init(mma_done + 1, 1);
    mbar_init(dq_full, 1);
    mbar_init(dq_free, 4);    // one arrival per dQ-writer warp
    mbar_init(final_bar, 2);  // one commit per MMA-issuing warp
    mbar_init(drain, 2);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Watchdog wd{abort_flag, a.status, a.budget_ns};

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&map_q);
      tma_prefetch_desc(&map_k);
      tma_prefetch_desc(&map_v);
      tma_prefetch_desc(&map_do);
      mbar_arrive_expect_tx(kv_bar, 2 * C::KCH * C::KCHUNK);
      for (int c = 0; c < C::KCH; ++c) {
        tma_load_3d(sK + c * C::KCHUNK, &map_k, kv_bar, c * 64, kstart + k0, kvh);
        tma_load_3d(sV + c * C::KCHUNK, &map_v, kv_bar, c * 64, kvh, kstart + k0);
      }
    }
    if (lane == 0) {
      const int nslots = ld_slots(g.si);
      for (int it = 0; it < NIT; ++it) {
        const int s = it % C::ST;
        if (it >= C::ST && !wait_bounded(qdo_empty + s, ((it / C::ST) - 1) & 1, wd, kSiteBwdQdoEmpty)) break;
        TTT_TRACE(16, it);
        const IterInfo ii = decode_iter(it, nqt, jq0, G, gsz, kvh);
        mbar_arrive_expect_tx(qdo_full + s, 2 * C::QTILE + 2 * C::BQ * 4);
        for (int c = 0; c < C::KCH; ++c) {
          tma_load_3d(sQ + s * C::QTILE + c * C::QCHUNK, &map_q, qdo_full + s, c * 64, seq_start + ii.q0,
                      ii.p * g.H + ii.h);
          tma_load_4d(sDO + s * C::QTILE + c * C::QCHUNK, &map_do, qdo_full + s, c * 64, ii.h, seq_start + ii.q0,
                      ii.p);
        }
        const float* src =
            a.ld + ((static_cast<int64_t>(ii.p) * g.H + ii.h) * nslots + ld_slot(seq_start, n, ii.q0)) * 128;
        bulk_load(sLD + s * 2 * C::BQ, src, 2 * C::BQ * 4, qdo_full + s);
      }
    }
    __syncwarp();
  } else if (warp == 1 || warp == 2) {
    // ------------------------------------------------------------ MMA issuers
    // Warp 1 issues S^T/dP^T, warp 2 the dV/dK/dQ^T products.  An issuing thread blocks
    // until the tensor pipe accepts its instruction, and a barrier check queued behind
    // it costs a few hundred cycles even when the barrier has completed; with two
    // issuers one warp's checks are covered by the other's products.  The two streams
    // share no TMEM columns, and each commit tracks only its own warp's products
    // (every cross-stream dependency is ordered through the P/dS barriers).
    {
      constexpr uint32_t idSP = idesc_bf16_f32(128, C::BQ, false, false);
      constexpr uint32_t idDV = idesc_bf16_f32(128, D, false, true);
      constexpr uint32_t idDQ = idesc_bf16_f32(128, C::BQ, true, true);
      // Descriptors are built once; a k-step only adds a constant to the start-address
      // field (bits 0-13 hold address >> 4, and every operand lies below 256 KB).
      const uint64_t dK_k = sdesc_sw128(smem_u32(sK), 16, 1024);          // K~ as K-major A
      const uint64_t dK_mn = sdesc_sw128(smem_u32(sK), C::KCHUNK, 1024);  // K~ as MN-major A
      const uint64_t dV_k = sdesc_sw128(smem_u32(sV), 16, 1024);
      const uint64_t dQ_k = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dQ_mn = sdesc_sw128(smem_u32(sQ), C::QCHUNK, 1024);
      const uint64_t dO_k = sdesc_sw128(smem_u32(sDO), 16, 1024);
      const uint64_t dO_mn = sdesc_sw128(smem_u32(sDO), C::QCHUNK, 1024);
      const uint64_t dS_k = sdesc_sw128(smem_u32(sDS), 16, 1024);
      const uint64_t dS_mn = sdesc_sw128(smem_u32(sDS), C::KCHUNK, 1024);
      auto issue_sdp = [&](int it) {
        const uint32_t so = static_cast<uint32_t>(((it % C::ST) * C::QTILE) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ok_ = ((kk >> 2) * C::KCHUNK + (kk & 3) * 32) >> 4;
          const uint32_t oq_ = ((kk >> 2) * C::QCHUNK + (kk & 3) * 32) >> 4;
          umma_ss_warp(tmem + C::COL_S, dK_k + ok_, dQ_k + so + oq_, idSP, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ok_ = ((kk >> 2) * C::KCHUNK + (kk & 3) * 32) >> 4;
          const uint32_t oq_ = ((kk >> 2) * C::QCHUNK + (kk & 3) * 32) >> 4;
          umma_ss_warp(tmem + C::COL_DP, dV_k + ok_, dO_k + so + oq_, idSP, kk > 0 ? 1u : 0u);
        }
      };
      bool ok = true;
      if (warp == 1) {
        // S^T/dP^T(n+2) once the P/dS warps hold S^T/dP^T(n+1) in registers: it is
        // complete before they finish step n+1
        ok = wait_warp(kv_bar, 0, wd, kSiteBwdKv);
        for (int it = 0; ok && it < NIT; ++it) {
          if (it > 0 && !wait_warp(sdp_free, (it - 1) & 1, wd, kSiteBwdSdpFree)) break;
          if (!wait_warp(qdo_full + it % C::ST, (it / C::ST) & 1, wd, kSiteBwdQdoFull)) break;
          TTT_TRACE(12, it);
          tc_fence_after();
          issue_sdp(it);
          umma_commit_warp(sdp_full);
          TTT_TRACE(1, it);
        }
      } else {
        ok = wait_warp(kv_bar, 0, wd, kSiteBwdKv);
        for (int it = 0; ok && it < NIT; ++it) {
          const int s = it % C::ST;
          const int b = it & 1;
          if (!wait_warp(ds_ready + b, (it >> 1) & 1, wd, kSiteBwdDsReady)) break;
          TTT_TRACE(0, it);
          tc_fence_after();
          const uint32_t so = static_cast<uint32_t>((s * C::QTILE) >> 4);
          const uint32_t bo = static_cast<uint32_t>((b * C::DSTILE) >> 4);
          // dV += P^T dO   (P^T: TMEM, 64 queries = 32 packed columns)
#pragma unroll
          for (int kk = 0; kk < C::BQ / 16; ++kk)
            umma_ts_warp(tmem + C::COL_DV, tmem + C::COL_PT + 32 * b + kk * 8, dO_mn + so + ((kk * 2048) >> 4),
                         idDV, (it > 0 || kk > 0) ? 1u : 0u);
          // dK += dS^T Q~
#pragma unroll
          for (int kk = 0; kk < C::BQ / 16; ++kk)
            umma_ss_warp(tmem + C::COL_DK, dS_k + bo + ((kk * 32) >> 4), dQ_mn + so + ((kk * 2048) >> 4), idDV,
                         (it > 0 || kk > 0) ? 1u : 0u);
          umma_commit_warp(qdo_empty + s);  // last readers of this step's q~ / dO tiles
          TTT_TRACE(2, it);
          if (it > 0) {
            if (!wait_warp(dq_free, (it - 1) & 1, wd, kSiteBwdDqFree)) break;
            tc_fence_after();
          }
          TTT_TRACE(3, it);
          // dQ^T = K~^T dS^T
#pragma unroll
          for (int kk = 0; kk < C::BK / 16; ++kk)
            umma_ss_warp(tmem + C::COL_DQ, dK_mn + ((kk * 2048) >> 4), dS_mn + bo + ((kk * 2048) >> 4), idDQ,
                         kk > 0 ? 1u : 0u);
          umma_commit_warp(mma_done + b);
          umma_commit_warp(dq_full);
          TTT_TRACE(4, it);
        }
      }
      (void)ok;
      umma_commit_warp(final_bar);
      umma_commit_warp(drain);
      wait_drain(drain, 0, wd, kSiteBwdDrain);
    }
    __syncwarp();
  } else if (warp >= 4 && warp < 12) {
    // ------------------------------------------------------------ P / dS
    const int hf = (warp - 4) >> 2;  // query columns [32*hf, 32*hf+32)
    const int wq = warp & 3;
    const int r = wq * 32 + lane;    // key row
    const int kpos = k0 + r;
    const bool kvalid = kpos < klen;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const float sl2 = g.scale * kLog2e;
    bool ok = true;
    for (int it = 0; it < NIT; ++it) {
      const int s = it % C::ST;
      const int b = it & 1;
      const IterInfo ii = decode_iter(it, nqt, jq0, G, gsz, kvh);
      // warp-agreed waits: the TMEM loads and stores that follow are warp-wide instructions
      if (!wait_warp(sdp_full, it & 1, wd, kSiteBwdSdpFull) ||
          !wait_warp(qdo_full + s, (it / C::ST) & 1, wd, kSiteBwdQdoFull)) {
        ok = false;
        break;
      }
      if (lane == 0 && warp == 4) TTT_TRACE(5, it);
      if (lane == 0 && warp == 4 && it == 0) TTT_CTA_MARK(1);
      if (lane == 0 && warp == 8) TTT_TRACE(13, it);
      tc_fence_after();
      uint32_t sv[32], dp[32];
      tmem_ld32(lane_base + C::COL_S + 32 * hf, sv);
      tmem_ld32(lane_base + C::COL_DP + 32 * hf, dp);
      tmem_ld_wait();
      reg_fence32(sv);
      reg_fence32(dp);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sdp_free);
#ifdef TTT_KERNEL_TRACE
      if (lane == 0) {
        constexpr int kSlot[8] = {6, 22, 23, 17, 19, 18, 14, 15};
        TTT_TRACE(kSlot[warp - 4], it);
      }
#endif
      const float* ldp = sLD + s * 2 * C::BQ + 32 * hf;
      // interior tile: every (key, query) pair of this half is visible
      const int qlo = ii.q0 + 32 * hf;
      bool interior = false;
      if (qlo + 32 <= len && k0 + C::BK <= klen) {
        if (!BLOCK) {
          interior = qlo + off >= k0 + C::BK - 1;
        } else if (!WIN) {
          interior = __ldg(a.qlim + seq_start + qlo) >= k0 + C::BK - 1;
        } else {
          // the first row has the smallest limit, the last the largest window start; both
          // loads are issued before either is compared (no dependent round trip)
          const int l_first = __ldg(a.qlim + seq_start + qlo);
          const int l_last = __ldg(a.qlim + seq_start + qlo + 31);
          interior = l_first >= k0 + C::BK - 1 && block_row_start(g, l_last) <= k0;
        }
      }
      // P = 2^(s*scale*log2e - lse*log2e), dS = P (dP - delta), two columns per
      // instruction; the bf16 pairs are packed straight from the results
      const uint64_t sl2x2 = f2_pack(sl2, sl2);
      uint32_t pk[16], dk[16];
#pragma unroll
      for (int c0 = 0; c0 < 32; c0 += 8) {
        const ulonglong2 nl0 = *reinterpret_cast<const ulonglong2*>(ldp + c0);
        const ulonglong2 nl1 = *reinterpret_cast<const ulonglong2*>(ldp + c0 + 4);
        const ulonglong2 dl0 = *reinterpret_cast<const ulonglong2*>(ldp + C::BQ + c0);
        const ulonglong2 dl1 = *reinterpret_cast<const ulonglong2*>(ldp + C::BQ + c0 + 4);
        const uint64_t nl[4] = {nl0.x, nl0.y, nl1.x, nl1.y};
        const uint64_t dl[4] = {dl0.x, dl0.y, dl1.x, dl1.y};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int c = c0 + 2 * u;
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])), sl2x2, nl[u]), x0, x1);
          float p0 = exp2_approx(x0), p1 = exp2_approx(x1);
          const uint64_t t = f2_sub(f2_pack(__uint_as_float(dp[c]), __uint_as_float(dp[c + 1])), dl[u]);
          float d0, d1;
          f2_unpack(f2_mul(f2_pack(p0, p1), t), d0, d1);
          if (!interior) {
            // padding rows of the statistics are never written: select, do not multiply
            int lim0 = qlo + c + off, lim1 = qlo + c + 1 + off;
            if (BLOCK) {
              lim0 = qlo + c < len ? __ldg(a.qlim + seq_start + qlo + c) : -1;
              lim1 = qlo + c + 1 < len ? __ldg(a.qlim + seq_start + qlo + c + 1) : -1;
            }
            bool v0 = kvalid && qlo + c < len && kpos <= lim0;
            bool v1 = kvalid && qlo + c + 1 < len && kpos <= lim1;
            if (WIN) {
              v0 = v0 && kpos >= block_row_start(g, lim0);
              v1 = v1 && kpos >= block_row_start(g, lim1);
            }
            p0 = v0 ? p0 : 0.f;
            d0 = v0 ? d0 : 0.f;
            p1 = v1 ? p1 : 0.f;
            d1 = v1 ? d1 : 0.f;
          }
          pk[c >> 1] = pack_bf16x2(p0, p1);
          dk[c >> 1] = pack_bf16x2(d0, d1);
        }
      }
      if (lane == 0 && warp == 4) TTT_TRACE(8, it);
      // P^T / dS^T buffer b was last read by the products of step it-2
      if (it >= 2 && !wait_warp(mma_done + b, ((it >> 1) - 1) & 1, wd, kSiteBwdMmaDone)) {
        ok = false;
        break;
      }
      if (lane == 0 && warp == 4) TTT_TRACE(7, it);
      tc_fence_after();
      tmem_st16(lane_base + C::COL_PT + 32 * b + 16 * hf, pk);
      // dS^T row r, 128-byte swizzle: 16-byte chunk c of the row sits at c ^ (r & 7)
      uint8_t* row = sDS + b * C::DSTILE + r * 128;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int cc = 4 * hf + i;
        *reinterpret_cast<uint4*>(row + ((cc ^ (r & 7)) << 4)) =
            make_uint4(dk[4 * i], dk[4 * i + 1], dk[4 * i + 2], dk[4 * i + 3]);
      }
      tmem_st_wait();
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(ds_ready + b);
      if (lane == 0 && warp == 4) TTT_TRACE(9, it);

    }
    // ---- epilogue: dV (half 0) and dK (half 1) of this CTA's keys, final: dV in bf16,
    // dK = sigma * R(pos)^T dk~ in bf16 (the trunk keys' rotation at their own position)
    if (ok && wait_warp(final_bar, 0, wd, kSiteBwdFinal)) {
      tc_fence_after();
      if (lane == 0 && warp == 4) TTT_CTA_MARK(2);
      const int64_t tau = kstart + kpos;
      if (MODE == 2) {
        // ring step: add this CTA's raw dV / dk~ rows to the travelling accumulators
        float* acc = (hf == 0 ? a.dv_acc : a.dk_acc) + (static_cast<int64_t>(kvh) * klen + kpos) * D;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(lane_base + (hf == 0 ? C::COL_DV : C::COL_DK) + 32 * c, v);
          tmem_ld_wait();
          reg_fence32(v);
          if (!kvalid) continue;
          float4* dst = reinterpret_cast<float4*>(acc + 32 * c);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            float4 x = dst[e];
            x.x += __uint_as_float(v[4 * e]);
            x.y += __uint_as_float(v[4 * e + 1]);
            x.z += __uint_as_float(v[4 * e + 2]);
            x.w += __uint_as_float(v[4 * e + 3]);
            dst[e] = x;
          }
        }
      } else if (hf == 0) {
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(lane_base + C::COL_DV + 32 * c, v);
          tmem_ld_wait();
          reg_fence32(v);
          if (!kvalid) continue;
          __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.dv) + (tau * g.Hkv + kvh) * D + 32 * c;
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 w = make_uint4(pack_bf16x2(__uint_as_float(v[e]), __uint_as_float(v[e + 1])),
                                 pack_bf16x2(__uint_as_float(v[e + 2]), __uint_as_float(v[e + 3])),
                                 pack_bf16x2(__uint_as_float(v[e + 4]), __uint_as_float(v[e + 5])),
                                 pack_bf16x2(__uint_as_float(v[e + 6]), __uint_as_float(v[e + 7])));
            *reinterpret_cast<uint4*>(dst + e) = w;
          }
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < D / 64; ++c) {
          uint32_t lo[32], hi[32];
          tmem_ld32(lane_base + C::COL_DK + 32 * c, lo);
          tmem_ld32(lane_base + C::COL_DK + D / 2 + 32 * c, hi);
          tmem_ld_wait();
          reg_fence32(lo);
          reg_fence32(hi);
          if (!kvalid) continue;
          store_dk_row<D>(static_cast<__nv_bfloat16*>(a.dk) + (tau * g.Hkv + kvh) * D, kpos, g.theta, g.scale, lo,
                          hi, c);
        }
      }
    }
  } else if (warp >= 12) {
    // ------------------------------------------------------------ dQ writer
    const int wq = warp & 3;
    const int d = wq * 32 + lane;  // TMEM lane = head dimension
    const int tid = threadIdx.x - 384;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const int nslots = ld_slots(g.si);
    volatile uint32_t* go = abort_flag + 1;  // lead thread's dq_full outcome, shared through the barrier
    for (int it = 0; it < NIT; ++it) {
      const IterInfo ii = decode_iter(it, nqt, jq0, G, gsz, kvh);
      // one thread waits and the four warps agree on the outcome, so that all of them
      // take the same named barriers on every path
      if (tid == 0) *go = wait_bounded(dq_full, it & 1, wd, kSiteBwdDqFull) ? 1u : 0u;
      named_bar_sync(1, 128);
      if (!*go) break;
      if (tid == 0) TTT_TRACE(10, it);
      tc_fence_after();
      uint32_t v0[32], v1[32];
      tmem_ld32(lane_base + C::COL_DQ, v0);
      tmem_ld32(lane_base + C::COL_DQ + 32, v1);
      tmem_ld_wait();
      reg_fence32(v0);
      reg_fence32(v1);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dq_free);
      if (tid == 0) TTT_TRACE(20, it);
      // ordered mode: the key tiles of this query tile add their dq~ in key-tile order
      int* ticket = nullptr;
      bool ordered_ok = true;
      if (a.tickets && tid == 0) {
        ticket = a.tickets + (static_cast<int64_t>(ii.p) * g.H + ii.h) * nslots + ld_slot(seq_start, n, ii.q0);
        ordered_ok = wait_counter(ticket, jk, wd, kSiteBwdTicket);
        asm volatile("fence.proxy.async.global;" ::: "memory");
      }
      // two halves of 32 query rows, each through its own staging buffer; one bulk
      // group is committed per half (empty past the end of the sequence), so the group
      // that last read a buffer is always the second most recent one
#pragma unroll
      for (int hq = 0; hq < 2; ++hq) {
        float* stage = sDQ + hq * (C::DQSTAGE / 4);
        if (tid == 0) bulk_wait_read1();
        named_bar_sync(1, 128);
        if (d < D) {
#pragma unroll
          for (int q = 0; q < 32; ++q) stage[q * D + d] = __uint_as_float(hq == 0 ? v0[q] : v1[q]);
        }
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (tid == 0) {
          const int r0 = ii.q0 + 32 * hq;
          const int nrows = min(32, len - r0);
          if (nrows > 0 && ordered_ok) {
            float* dst = a.dq_acc + ((static_cast<int64_t>(ii.p) * g.H + ii.h) * g.si.T + seq_start + r0) * D;
            bulk_reduce_add_f32(dst, stage, static_cast<uint32_t>(nrows * D * 4));
          }
          bulk_commit();
        }
      }
      if (ticket && ordered_ok) {
        // this tile's additions are complete before the next key tile may start its own
        bulk_wait0();
        asm volatile("fence.proxy.async.global;" ::: "memory");
        __threadfence();
        atomicAdd(ticket, 1);
      }
      if (tid == 0) TTT_TRACE(21, it);
    }
    if (tid == 0) bulk_wait0();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) TTT_CTA_MARK(3);
  if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

template <int D, int MODE>
cudaError_t launch(const TrunkBwdArgs& a, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                   const CUtensorMap& mdo, cudaStream_t stream) {
  using C = BwdCfg<D>;
  cudaError_t e =
      cudaFuncSetAttribute(trunk_bwd_kernel<D, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const int njk = (a.g.ksi.max_len + C::BK - 1) / C::BK;
  const long long blocks = static_cast<long long>(njk) * a.g.ksi.nseq * a.g.Hkv;
  if (blocks <= 0) return cudaSuccess;
  if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
  trunk_bwd_kernel<D, MODE><<<static_cast<unsigned>(blocks), C::THREADS, C::SMEM, stream>>>(mq, mk, mv, mdo, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_trunk_bwd(const TrunkBwdArgs& a, const CUtensorMap& map_q, const CUtensorMap& map_k,
                             const CUtensorMap& map_v, const CUtensorMap& map_do, cudaStream_t stream) {
  if (a.g.ring > 0)
    return a.g.D == 128 ? launch<128, 2>(a, map_q, map_k, map_v, map_do, stream)
                        : launch<64, 2>(a, map_q, map_k, map_v, map_do, stream);
  if (a.g.Bs > 0 && a.g.window > 0)
    return a.g.D == 128 ? launch<128, 3>(a, map_q, map_k, map_v, map_do, stream)
                        : launch<64, 3>(a, map_q, map_k, map_v, map_do, stream);
  if (a.g.Bs > 0)
    return a.g.D == 128 ? launch<128, 1>(a, map_q, map_k, map_v, map_do, stream)
                        : launch<64, 1>(a, map_q, map_k, map_v, map_do, stream);
  return a.g.D == 128 ? launch<128, 0>(a, map_q, map_k, map_v, map_do, stream)
                      : launch<64, 0>(a, map_q, map_k, map_v, map_do, stream);
}

}  // namespace ttt

TTT_TRACE_READER(ttt_trace_read_bwd)
