// a2: trunk causal attention forward on the 5th-generation tensor cores.
//
// "DFlash/DSpark and EAGLE-3 TTT draft co-training ..." (NeMo-RL issue 3698),
// "What I'm working on", item 1: the trunk half of the two-part trunk+branch
// attention.  Every pass p and every query head of a GQA group attends to the SAME
// pass-1 keys with the SAME index-causal predicate (key t <= query i), so one CTA
// stacks two (pass, head) query tiles of one KV head and streams each K/V tile once
// for both.
//
// CTA = 12 warps:
//   warp 0      TMA producer: two Q tiles once, then K/V tiles into a 2-stage ring
//   warp 1      TMEM allocator and MMA issuer (one thread): S = Q K^T (SS form),
//               O += P V (TS form, P read from TMEM)
//   warps 4-7   softmax for query tile 0 (one TMEM lane = one query row per thread)
//   warps 8-11  softmax for query tile 1
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+D), O1 [256+D,256+2D);
// P_t (bf16, two per column) overwrites the first 64 columns of S_t.
// The online softmax keeps a running max per row and rescales O (in TMEM) only when
// the max grows by more than 2^8; the final normalisation uses the same max, so the
// result is exact up to rounding.
// Output: O_t (normalised, fp32, head-major) and lse_t (natural log) per row.
#include "common.cuh"

namespace ttt {

namespace {

template <int D>
struct FwdCfg {
  static constexpr int BM = 128;  // query rows per tile
  static constexpr int BN = 128;  // keys per KV tile
  static constexpr int NQ = 2;    // query tiles per CTA
  static constexpr int KST = 3;   // K ring stages
  static constexpr int VST = 2;   // V ring stages (V_j is read one iteration after K_j)
  static constexpr int KCH = D / 64;
  static constexpr int CHUNK = 128 * 128;         // one 64-column chunk of a 128-row tile
  static constexpr int TILE = KCH * CHUNK;        // 128 rows x D bf16
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + NQ * TILE;
  static constexpr int OFF_V = OFF_K + KST * TILE;
  static constexpr int OFF_BAR = OFF_V + VST * TILE;
  static constexpr int BAR_BYTES = 256;
  // D = 64 needs only 96 KB; ask for more so that one CTA holds the SM (and its TMEM).
  static constexpr int SMEM_USED = OFF_BAR + BAR_BYTES;
  static constexpr int SMEM = (SMEM_USED < 120 * 1024 ? 120 * 1024 : SMEM_USED) + 1024;
  static constexpr int COL_S0 = 0;
  static constexpr int COL_O0 = 256;
  static constexpr int TMEM_COLS = 512;
  static constexpr int THREADS = 384;
};

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

// MODE 0: TTT trunk+branch attention (epilogue keys: the branch keys of passes 2..p at
// the query's position).  MODE 1: block-draft attention (query rows are block tokens,
// trunk keys the context up to the block's anchor, epilogue keys the Bs keys of the
// row's own block).  MODE 2: one step of the context-parallel ring (query rows are a
// chunk of the sequence, trunk keys a visiting chunk, causal by global position; the
// branch keys only in the step that meets the chunk's own keys; fp32 partial output).
template <int MODE>
struct EpiKeys {
  static constexpr int kMax = MODE == 1 ? 16 : 15;  // P <= 16 passes; Bs <= 16
};

template <int D, int MODE>
__global__ void __launch_bounds__(FwdCfg<D>::THREADS, 1)
    trunk_fwd_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                     const __grid_constant__ CUtensorMap map_v, const TrunkFwdArgs a) {
  using C = FwdCfg<D>;
  constexpr int kMaxBranch = EpiKeys<MODE>::kMax;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);

  const Geometry& g = a.g;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work item: (query block jq, sequence n, KV head, pair of (pass, head) tiles),
  // largest jq first (longest causal rows first).
  const int gsz = g.H / g.Hkv;
  const int G = g.P * gsz;  // query heads per KV head
  const int npairs = (G + 1) >> 1;
  const int njq = (g.si.max_len + C::BM - 1) / C::BM;
  const int per_jq = g.si.nseq * g.Hkv * npairs;
  const int jq = njq - 1 - static_cast<int>(blockIdx.x) / per_jq;
  int rem = static_cast<int>(blockIdx.x) % per_jq;
  const int n = rem / (g.Hkv * npairs);
  rem %= g.Hkv * npairs;
  const int kvh = rem / npairs;
  const int pair = rem % npairs;
  int seq_start, len, kstart, klen;
  seq_bounds(g.si, n, seq_start, len);  // query rows
  seq_bounds(g.ksi, n, kstart, klen);   // key rows (the same tokens in MODE 0)
  if (jq * C::BM >= len) return;  // the whole CTA leaves before touching TMEM
  const int nq_tiles = (2 * pair + 1 < G) ? 2 : 1;
  const int q0 = jq * C::BM;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;             // [KST]
  uint64_t* k_empty = k_full + C::KST;     // [KST]
  uint64_t* v_full = k_empty + C::KST;     // [VST]
  uint64_t* v_empty = v_full + C::VST;     // [VST]
  uint64_t* s_full = v_empty + C::VST;     // [NQ]
  uint64_t* p_full = s_full + C::NQ;       // [NQ]
  uint64_t* o_final = p_full + C::NQ;      // [NQ]
  uint64_t* p_half = o_final + C::NQ;      // [NQ]: P of the first 64 keys written
  uint64_t* drain = p_half + C::NQ;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  uint32_t* abort_flag = tmem_slot + 1;
  int* nkv_slot = reinterpret_cast<int*>(abort_flag + 1);

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < C::KST; ++s) {
      mbar_init(k_full + s, 1);
      mbar_init(k_empty + s, 1);
    }
    for (int s = 0; s < C::VST; ++s) {
      mbar_init(v_full + s, 1);
      mbar_init(v_empty + s, 1);
    }
    for (int t = 0; t < C::NQ; ++t) {
      mbar_init(s_full + t, 1);
      mbar_init(p_full + t, 4);  // one arrival per softmax warp
      mbar_init(p_half + t, 4);
      mbar_init(o_final + t, 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
  if (MODE == 1 && warp == 2) {
    // key tiles to stream: up to the largest anchor among this tile's rows
    // (none for an empty context: the rows see their block's keys only)
    const int rows = min(C::BM, len - q0);
    int mx = -1;
    for (int r = lane * g.Bs; r < rows; r += 32 * g.Bs) mx = max(mx, block_row_limit(g, seq_start, q0 + r, klen));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) *nkv_slot = (mx + C::BN) / C::BN;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int nkv = MODE == 0 ? jq + 1
                  : MODE == 1 ? *nkv_slot
                              : min(q0 + min(C::BM, len - q0) - 1 + g.limit_off, klen - 1) / C::BN + 1;
  const Watchdog wd{abort_flag, a.status, a.budget_ns};

  int p_of[2], h_of[2];
  for (int t = 0; t < 2; ++t) {
    const int qh = min(2 * pair + t, G - 1);
    p_of[t] = qh / gsz;
    h_of[t] = kvh * gsz + qh % gsz;
  }

  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&map_q);
      tma_prefetch_desc(&map_k);
      tma_prefetch_desc(&map_v);
      mbar_arrive_expect_tx(q_full, nq_tiles * C::TILE);
      for (int t = 0; t < nq_tiles; ++t)
        for (int c = 0; c < C::KCH; ++c)
          tma_load_3d(sQ + t * C::TILE + c * C::CHUNK, &map_q, q_full, c * 64, seq_start + q0,
                      p_of[t] * g.H + h_of[t]);
      for (int j = 0; j < nkv; ++j) {
        const int krow = kstart + j * C::BN;
        const int ks = j % C::KST;
        if (j >= C::KST && !wait_bounded(k_empty + ks, ((j / C::KST) - 1) & 1, wd, kSiteFwdKvEmpty)) break;
        TTT_TRACE(14, j);
        mbar_arrive_expect_tx(k_full + ks, C::TILE);
        for (int c = 0; c < C::KCH; ++c)
          tma_load_3d(sK + ks * C::TILE + c * C::CHUNK, &map_k, k_full + ks, c * 64, krow, kvh);
        const int vs = j % C::VST;
        if (j >= C::VST && !wait_bounded(v_empty + vs, ((j / C::VST) - 1) & 1, wd, kSiteFwdKvEmpty)) break;
        mbar_arrive_expect_tx(v_full + vs, C::TILE);
        for (int c = 0; c < C::KCH; ++c)
          tma_load_3d(sV + vs * C::TILE + c * C::CHUNK, &map_v, v_full + vs, c * 64, kvh, krow);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    {
      constexpr uint32_t idS = idesc_bf16_f32(128, C::BN, false, false);
      constexpr uint32_t idO = idesc_bf16_f32(128, D, false, true);
      // Descriptors are built once; a k-step only adds a constant to the start-address
      // field (bits 0-13 hold address >> 4, and every operand lies below 256 KB).
      const uint64_t dq0 = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dk0 = sdesc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dv0 = sdesc_sw128(smem_u32(sV), C::CHUNK, 1024);
      auto issue_s = [&](int t, int s) {
        const uint64_t qd = dq0 + static_cast<uint32_t>((t * C::TILE) >> 4);
        const uint64_t kd = dk0 + static_cast<uint32_t>((s * C::TILE) >> 4);
        const uint32_t d_tmem = tmem + C::COL_S0 + 128 * t;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * C::CHUNK + (kk & 3) * 32) >> 4;
          umma_ss_warp(d_tmem, qd + off, kd + off, idS, kk > 0 ? 1u : 0u);
        }
      };
      // O += P V over keys [16*k0, 16*k1) of the tile
      auto issue_pv = [&](int t, int s, bool acc, int k0, int k1) {
        const uint64_t vd = dv0 + static_cast<uint32_t>((s * C::TILE) >> 4);
        const uint32_t d_tmem = tmem + C::COL_O0 + D * t;
        const uint32_t a_tmem = tmem + C::COL_S0 + 128 * t;
#pragma unroll
        for (int kk = k0; kk < k1; ++kk)
          umma_ts_warp(d_tmem, a_tmem + kk * 8, vd + ((kk * 2048) >> 4), idO, (acc || kk > 0) ? 1u : 0u);
      };
      bool ok = wait_warp(q_full, 0, wd, kSiteFwdQ);
      // Order per KV tile j: for each query tile t, O_t += P_t(j-1) V_{j-1}, then
      // S_t(j) = Q_t K_j^T.  The in-order tensor pipe finishes reading P_t(j-1) (which
      // overlays S_t) before S_t(j) overwrites it.
      for (int j = 0; ok && j <= nkv; ++j) {
        for (int t = 0; t < nq_tiles; ++t) {
          if (j > 0) {
            // the first half of O += P V as soon as P of the first 64 keys is written, the
            // second half when the whole of P is
            if (!wait_warp(p_half + t, (j - 1) & 1, wd, kSiteFwdPFull)) {
              ok = false;
              break;
            }
            if (t == 0 && !wait_warp(v_full + (j - 1) % C::VST, ((j - 1) / C::VST) & 1, wd, kSiteFwdKvFull)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_pv(t, (j - 1) % C::VST, j - 1 > 0, 0, C::BN / 32);
            if (!wait_warp(p_full + t, (j - 1) & 1, wd, kSiteFwdPFull)) {
              ok = false;
              break;
            }
            TTT_TRACE(0 + t, j);
            tc_fence_after();
            issue_pv(t, (j - 1) % C::VST, true, C::BN / 32, C::BN / 16);
            if (j == nkv) umma_commit_warp(o_final + t);
            if (t == nq_tiles - 1) umma_commit_warp(v_empty + (j - 1) % C::VST);
          }
          if (j < nkv) {
            if (t == 0 && !wait_warp(k_full + j % C::KST, (j / C::KST) & 1, wd, kSiteFwdKvFull)) {
              ok = false;
              break;
            }
            if (t == 0) TTT_TRACE(15, j);
            tc_fence_after();
            issue_s(t, j % C::KST);
            umma_commit_warp(s_full + t);
            TTT_TRACE(2 + t, j);
            if (t == nq_tiles - 1) umma_commit_warp(k_empty + j % C::KST);
          }
        }
      }
      // nothing may still be running on the tensor cores when TMEM is released
      umma_commit_warp(drain);
      wait_drain(drain, 0, wd, kSiteFwdDrain);
    }
    __syncwarp();
  } else if (warp >= 4 && warp < 4 + 4 * nq_tiles) {
    // ------------------------------------------------------------ softmax
    const int t = (warp - 4) >> 2;
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const int qpos = q0 + row;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const uint32_t colS = C::COL_S0 + 128 * t;
    const uint32_t colO = C::COL_O0 + D * t;
    const float sl2 = g.scale * kLog2e;
    // last visible key of this row: its own position (causal) or its block's anchor
    const int lim = MODE == 0   ? qpos
                    : MODE == 1 ? (qpos < len ? block_row_limit(g, seq_start, qpos, klen) : 0)
                                : min(qpos + g.limit_off, klen - 1);
    float m_run = -INFINITY;
    float l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      if (!wait_warp(s_full + t, j & 1, wd, kSiteFwdSFull)) {  // warp-agreed: TMEM access follows
        ok = false;
        break;
      }
      if (lane == 0 && wq == 0) TTT_TRACE(4 + t, j);
      tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(lane_base + colS + 32 * c, sr[c]);
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < 4; ++c) reg_fence32(sr[c]);
      const int k0 = j * C::BN;
      if (k0 + C::BN - 1 > lim) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (k0 + 32 * c + e > lim) sr[c][e] = __float_as_uint(-INFINITY);
      }
      // row max: 8 independent chains, then a tree
      float mxv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) mxv[u] = fmaxf(__uint_as_float(sr[0][u]), __uint_as_float(sr[0][u + 8]));
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        mxv[u] = fmaxf(mxv[u], fmaxf(__uint_as_float(sr[0][u + 16]), __uint_as_float(sr[0][u + 24])));
#pragma unroll
        for (int c = 1; c < 4; ++c)
          mxv[u] = fmaxf(fmaxf(mxv[u], __uint_as_float(sr[c][u])),
                         fmaxf(fmaxf(__uint_as_float(sr[c][u + 8]), __uint_as_float(sr[c][u + 16])),
                               __uint_as_float(sr[c][u + 24])));
      }
#pragma unroll
      for (int u = 4; u > 0; u >>= 1)
#pragma unroll
        for (int v = 0; v < u; ++v) mxv[v] = fmaxf(mxv[v], mxv[v + u]);
      const float m_new = fmaxf(m_run, mxv[0] * sl2);
      if (lane == 0 && wq == 0) TTT_TRACE(8 + t, j);
      const bool rescale = m_new > m_run + kRescaleThreshold;
      float alpha = 1.f;
      if (rescale) {
        alpha = exp2_approx(m_run - m_new);
        l_run *= alpha;
        m_run = m_new;
      }
      // a warp with a row whose O needs rescaling releases P only after the rescale (rare:
      // the running max grew by more than 2^8); the others release the first 64 keys early
      const bool warp_rescale = __any_sync(0xffffffffu, rescale && j > 0);
      float rsv[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      // P = 2^(s*scale*log2e - m), bf16 pairs into the first 64 columns of S_t; the first
      // 64 keys are released to the MMA warp before the last 64 are computed
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float p0 = exp2_approx(fmaf(__uint_as_float(sr[c][2 * e]), sl2, -m_run));
          const float p1 = exp2_approx(fmaf(__uint_as_float(sr[c][2 * e + 1]), sl2, -m_run));
          rsv[(2 * e) & 7] += p0;
          rsv[(2 * e + 1) & 7] += p1;
          pk[e] = pack_bf16x2(p0, p1);
        }
        tmem_st16(lane_base + colS + 16 * c, pk);
        if (c == 1 && !warp_rescale) {
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(p_half + t);
        }
      }
#pragma unroll
      for (int u = 4; u > 0; u >>= 1)
#pragma unroll
        for (int v = 0; v < u; ++v) rsv[v] += rsv[v + u];
      l_run += rsv[0];
      if (lane == 0 && wq == 0) TTT_TRACE(10 + t, j);
      if (warp_rescale) {
        // O of this row was complete up to tile j-1 when s_full fired (in-order MMAs), and
        // no O += P V of this tile runs before this warp releases P.  TMEM loads and
        // stores are warp-wide instructions: the whole warp runs them, rows that need no
        // rescaling with alpha = 1 (exact)
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(lane_base + colO + 32 * c, o);
          tmem_ld_wait();
          reg_fence32(o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(lane_base + colO + 32 * c, o);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (warp_rescale) mbar_arrive(p_half + t);
        mbar_arrive(p_full + t);
      }
      if (lane == 0 && wq == 0) TTT_TRACE(12 + t, j);
    }
    if (ok && (nkv == 0 || wait_warp(o_final + t, 0, wd, kSiteFwdOFinal))) {
      tc_fence_after();
      // ---- epilogue: branch keys (a3) and the exact joint-LSE merge (a4).
      // MODE 0: query (pass p, position qpos) also sees k~_j[tau], V_j[tau] of the branch
      // passes j = 1..p (0-based) at its own position.  MODE 1: a block token also sees
      // the Bs keys of its own block (bidirectional).  Scores on the CUDA cores.  The
      // trunk partial is (m_run, l_run, unnormalised O in TMEM), all in log2 units.
      const bool valid = qpos < len;
      const int p = p_of[t], h = h_of[t];
      const int tau = seq_start + qpos;
      const int T = g.si.T;
      const int nkeys = MODE == 0 ? p : MODE == 1 ? g.Bs : (g.ring == 2 ? p : 0);  // epilogue keys of this row
      const int bstart = MODE == 1 ? tau - qpos % g.Bs : 0;  // first row of the block
      // key u (0-based) of the epilogue: k~ row and V row
      auto krow_of = [&](int u) -> const uint4* {
        const int64_t r = MODE != 1 ? (static_cast<int64_t>(u + 1) * g.Hkv + kvh) * T + tau
                                    : static_cast<int64_t>(kvh) * T + bstart + u;
        return reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.kr) + r * D);
      };
      auto vrow_of = [&](int u) -> const __nv_bfloat16* {
        return MODE != 1 ? static_cast<const __nv_bfloat16*>(a.v) + (u + 1) * g.skv +
                               (static_cast<int64_t>(tau) * g.Hkv + kvh) * D
                         : static_cast<const __nv_bfloat16*>(a.v) +
                               (static_cast<int64_t>(bstart + u) * g.Hkv + kvh) * D;
      };
      float bs[kMaxBranch];
      float m = m_run;
#pragma unroll
      for (int j = 1; j <= kMaxBranch; ++j) {
        bs[j - 1] = -INFINITY;
        if (j <= nkeys && valid) {
          const uint4* kj = krow_of(j - 1);
          const uint8_t* qrow = sQ + t * C::TILE + row * 128;
          float acc = 0.f;
#pragma unroll 4
          for (int c8 = 0; c8 < D / 8; ++c8) {
            const uint4 qv = *reinterpret_cast<const uint4*>(qrow + (c8 >> 3) * C::CHUNK + (((c8 & 7) ^ (row & 7)) << 4));
            const uint4 kv = __ldg(kj + c8);
            const __nv_bfloat162* q2 = reinterpret_cast<const __nv_bfloat162*>(&qv);
            const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&kv);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const float2 a2 = __bfloat1622float2(q2[u]);
              const float2 b2 = __bfloat1622float2(k2[u]);
              acc = fmaf(a2.x, b2.x, fmaf(a2.y, b2.y, acc));
            }
          }
          bs[j - 1] = acc * sl2;
          m = fmaxf(m, bs[j - 1]);
        }
      }
      const float scale_t = exp2_approx(m_run - m);
      float l = l_run * scale_t;
#pragma unroll
      for (int j = 0; j < kMaxBranch; ++j) {
        bs[j] = exp2_approx(bs[j] - m);  // branch weights (0 for absent passes)
        l += bs[j];
      }
      const float inv_l = 1.f / l;
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(a.o) + p * g.sq + (static_cast<int64_t>(tau) * g.H + h) * D;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        if (nkv > 0) {  // CTA-uniform: no trunk key at all leaves O in TMEM unwritten
          tmem_ld32(lane_base + colO + 32 * c, o);
          tmem_ld_wait();
          reg_fence32(o);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = 0u;
        }
        if (valid) {
          float acc[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) acc[e] = __uint_as_float(o[e]) * scale_t;
#pragma unroll
          for (int j = 1; j <= kMaxBranch; ++j) {
            if (j <= nkeys) {
              const uint4* vj = reinterpret_cast<const uint4*>(vrow_of(j - 1) + 32 * c);
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4) {
                const uint4 vv = __ldg(vj + q4);
                const __nv_bfloat162* v2 = reinterpret_cast<const __nv_bfloat162*>(&vv);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                  const float2 f2 = __bfloat1622float2(v2[u]);
                  acc[8 * q4 + 2 * u] = fmaf(bs[j - 1], f2.x, acc[8 * q4 + 2 * u]);
                  acc[8 * q4 + 2 * u + 1] = fmaf(bs[j - 1], f2.y, acc[8 * q4 + 2 * u + 1]);
                }
              }
            }
          }
          if (MODE == 2) {
            float4* dst = reinterpret_cast<float4*>(a.o_part + ((static_cast<int64_t>(p) * T + tau) * g.H + h) * D +
                                                    32 * c);
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4)
              dst[q4] = make_float4(acc[4 * q4] * inv_l, acc[4 * q4 + 1] * inv_l, acc[4 * q4 + 2] * inv_l,
                                    acc[4 * q4 + 3] * inv_l);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
              dst[q4] = make_uint4(pack_bf16x2(acc[8 * q4] * inv_l, acc[8 * q4 + 1] * inv_l),
                                   pack_bf16x2(acc[8 * q4 + 2] * inv_l, acc[8 * q4 + 3] * inv_l),
                                   pack_bf16x2(acc[8 * q4 + 4] * inv_l, acc[8 * q4 + 5] * inv_l),
                                   pack_bf16x2(acc[8 * q4 + 6] * inv_l, acc[8 * q4 + 7] * inv_l));
          }
        }
      }
      if (valid) a.lse[lse_index(g.si, g.H, p, h, n, tau, qpos)] = (m + __log2f(l)) * kLn2;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

template <int D, int MODE>
cudaError_t launch(const TrunkFwdArgs& a, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                   cudaStream_t stream) {
  using C = FwdCfg<D>;
  cudaError_t e =
      cudaFuncSetAttribute(trunk_fwd_kernel<D, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const int G = a.g.P * (a.g.H / a.g.Hkv);
  const int npairs = (G + 1) / 2;
  const int njq = (a.g.si.max_len + C::BM - 1) / C::BM;
  const long long blocks = static_cast<long long>(njq) * a.g.si.nseq * a.g.Hkv * npairs;
  if (blocks <= 0) return cudaSuccess;
  if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
  trunk_fwd_kernel<D, MODE><<<static_cast<unsigned>(blocks), C::THREADS, C::SMEM, stream>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_trunk_fwd(const TrunkFwdArgs& a, const CUtensorMap& map_q, const CUtensorMap& map_k,
                             const CUtensorMap& map_v, cudaStream_t stream) {
  if (a.g.ring > 0)
    return a.g.D == 128 ? launch<128, 2>(a, map_q, map_k, map_v, stream) : launch<64, 2>(a, map_q, map_k, map_v, stream);
  if (a.g.Bs > 0)
    return a.g.D == 128 ? launch<128, 1>(a, map_q, map_k, map_v, stream) : launch<64, 1>(a, map_q, map_k, map_v, stream);
  return a.g.D == 128 ? launch<128, 0>(a, map_q, map_k, map_v, stream) : launch<64, 0>(a, map_q, map_k, map_v, stream);
}

}  // namespace ttt

TTT_TRACE_READER(ttt_trace_read_fwd)
