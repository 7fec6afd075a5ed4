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
//   warp 0      TMA producer: Q_0, K_0, Q_1, then K/V tiles into 3- and 2-stage rings,
//               then the epilogue keys' k~ / V tiles into the released stages
//   warp 1      TMEM allocator and MMA issuer (the whole warp runs the loop, one lane
//               issues): S = Q K^T (SS form), O += P V (TS form, P read from TMEM)
//   warps 2-3   zero an optional region (the backward's dq~ accumulator) meanwhile
//   warps 4-7   softmax for query tile 0 (one TMEM lane = one query row per thread)
//   warps 8-11  softmax for query tile 1
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+D), O1 [256+D,256+2D);
// P_t (bf16, two per column) overwrites the first 64 columns of S_t.
// The online softmax keeps a running max per row and rescales O (in TMEM) only when
// the max grows by more than 2^8; the final normalisation uses the same max, so the
// result is exact up to rounding.
// Output: O (bf16, public layout, full 32-row warp slices by TMA stores through the
// Q tile's shared memory) and lse (natural log) per row; MODE 2 writes fp32 partials.
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
constexpr int kEpiTiles = 2;               // epilogue keys staged through the ring stages

// MODE 0: TTT trunk+branch attention (epilogue keys: the branch keys of passes 2..p at
// the query's position).  MODE 1: block-draft attention (query rows are block tokens,
// trunk keys the context up to the block's anchor, epilogue keys the Bs keys of the
// row's own block).  MODE 2: one step of the context-parallel ring (query rows are a
// chunk of the sequence, trunk keys a visiting chunk, causal by global position; the
// branch keys only in the step that meets the chunk's own keys; fp32 partial output).
// The epilogue keys of a row (up to 15 branch passes, or Bs <= 16 block keys) join it
// one at a time, so their number is not bounded by the kernel.

template <int D, int MODE>
__global__ void __launch_bounds__(FwdCfg<D>::THREADS, 1)
    trunk_fwd_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                     const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_o,
                     const __grid_constant__ CUtensorMap map_ek, const __grid_constant__ CUtensorMap map_ev,
                     const TrunkFwdArgs a) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);

  const Geometry& g = a.g;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) TTT_CTA_MARK(0);

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
  // this CTA's share of a.zero_base (see TrunkFwdArgs), by threads [first, first + nthr)
  auto zero_share = [&](int first, int nthr) {
    if (a.dq_zeroed && blockIdx.x == 0 && static_cast<int>(threadIdx.x) == first)
      *a.dq_zeroed = a.zero_n16 > 0 ? kDqZeroedMagic : 0u;  // read by a later kernel only
    if (a.zero_n16 <= 0) return;
    const int64_t per = (a.zero_n16 + gridDim.x - 1) / gridDim.x;
    const int64_t lo = static_cast<int64_t>(blockIdx.x) * per;
    const int64_t hi = min(lo + per, a.zero_n16);
    for (int64_t i = lo + (static_cast<int>(threadIdx.x) - first); i < hi; i += nthr)
      a.zero_base[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  };
  if (jq * C::BM >= len) {  // the whole CTA leaves before touching TMEM
    zero_share(0, C::THREADS);
    return;
  }
  const int nq_tiles = (2 * pair + 1 < G) ? 2 : 1;
  const int q0 = jq * C::BM;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars + 0;             // [NQ]: one per query tile
  uint64_t* k_full = bars + C::NQ;         // [KST]
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
  int* jlo_slot = nkv_slot + 1;  // MODE 1: first key tile streamed

  if (threadIdx.x == 0) {
    for (int t = 0; t < C::NQ; ++t) mbar_init(q_full + t, 1);
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
    // key tiles to stream: up to the largest anchor among this tile's rows, from the
    // smallest first key (0, or a sliding window's start); none for an empty context
    // (the rows see their block's keys only).  One row per block suffices.
    const int rows = min(C::BM, len - q0);
    int mx = -1, mn = 0x7fffffff;
    for (int r = lane * g.Bs; r < rows; r += 32 * g.Bs) {
      const int lim = block_row_limit(g, seq_start, q0 + r, klen);
      mx = max(mx, lim);
      mn = min(mn, block_row_start(g, lim));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    }
    if (lane == 0) {
      const int jlo = mx < 0 ? 0 : mn / C::BN;
      *jlo_slot = jlo;
      *nkv_slot = (mx + C::BN) / C::BN - jlo;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int nkv = MODE == 0 ? jq + 1
                  : MODE == 1 ? *nkv_slot
                              : min(q0 + min(C::BM, len - q0) - 1 + g.limit_off, klen - 1) / C::BN + 1;
  const int jlo = MODE == 1 ? *jlo_slot : 0;  // key tile j of the stream is tile jlo + j
  const Watchdog wd{abort_flag, a.status, a.budget_ns};
  if (threadIdx.x == 0) TTT_CTA_INFO(nkv);

  int p_of[2], h_of[2];
  for (int t = 0; t < 2; ++t) {
    const int qh = min(2 * pair + t, G - 1);
    p_of[t] = qh / gsz;
    h_of[t] = kvh * gsz + qh % gsz;
  }
  // Epilogue keys whose k~ / V rows come as 128-row tiles into the ring stages once the
  // trunk stream has released them (nothing reuses them afterwards): MODE 0 / 2 the
  // branch passes 2 and 3 (key u = pass u+1 at the rows' own positions, the same for
  // both query tiles), k~ in K stages nkv, nkv+1 and V in V stage nkv and K stage nkv+2;
  // MODE 1 the tile's own block rows (k~ in K stage nkv, V in V stage nkv).  Further
  // keys are read from global memory.
  const int ne = MODE == 1   ? 1
                 : MODE == 2 && g.ring != 2 ? 0
                                            : min(max(p_of[0], nq_tiles > 1 ? p_of[1] : 0), kEpiTiles);

  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&map_q);
      tma_prefetch_desc(&map_k);
      tma_prefetch_desc(&map_v);
      if (ne > 0) {
        tma_prefetch_desc(&map_ek);
        tma_prefetch_desc(&map_ev);
      }
      // Q_0 first, then K_0, then Q_1: the first product S_0(0) needs only Q_0 and K_0
      auto load_q = [&](int t) {
        mbar_arrive_expect_tx(q_full + t, C::TILE);
        for (int c = 0; c < C::KCH; ++c)
          tma_load_3d(sQ + t * C::TILE + c * C::CHUNK, &map_q, q_full + t, c * 64, seq_start + q0,
                      p_of[t] * g.H + h_of[t]);
      };
      load_q(0);
      if (nkv == 0 && nq_tiles > 1) load_q(1);
      for (int j = 0; j < nkv; ++j) {
        const int krow = kstart + (jlo + j) * C::BN;
        const int ks = j % C::KST;
        if (j >= C::KST && !wait_bounded(k_empty + ks, ((j / C::KST) - 1) & 1, wd, kSiteFwdKvEmpty)) break;
        TTT_TRACE(14, j);
        mbar_arrive_expect_tx(k_full + ks, C::TILE);
        for (int c = 0; c < C::KCH; ++c)
          tma_load_3d(sK + ks * C::TILE + c * C::CHUNK, &map_k, k_full + ks, c * 64, krow, kvh);
        if (j == 0 && nq_tiles > 1) load_q(1);
        const int vs = j % C::VST;
        if (j >= C::VST && !wait_bounded(v_empty + vs, ((j / C::VST) - 1) & 1, wd, kSiteFwdKvEmpty)) break;
        mbar_arrive_expect_tx(v_full + vs, C::TILE);
        for (int c = 0; c < C::KCH; ++c)
          tma_load_3d(sV + vs * C::TILE + c * C::CHUNK, &map_v, v_full + vs, c * 64, kvh, krow);
      }
      // the epilogue tiles, each into a stage whose last trunk reader has completed
      const int erow = seq_start + q0;
      auto k_stage_load = [&](int j, const CUtensorMap* map, bool is_v, int u) -> bool {
        const int ks = j % C::KST;
        if (j >= C::KST && !wait_bounded(k_empty + ks, ((j / C::KST) - 1) & 1, wd, kSiteFwdKvEmpty)) return false;
        mbar_arrive_expect_tx(k_full + ks, C::TILE);
        for (int c = 0; c < C::KCH; ++c) {
          if (is_v)
            tma_load_4d(sK + ks * C::TILE + c * C::CHUNK, map, k_full + ks, c * 64, kvh, erow, u + 1);
          else
            tma_load_3d(sK + ks * C::TILE + c * C::CHUNK, map, k_full + ks, c * 64, erow,
                        MODE == 1 ? kvh : (u + 1) * g.Hkv + kvh);
        }
        return true;
      };
      bool eok = true;
      for (int u = 0; eok && u < ne; ++u) eok = k_stage_load(nkv + u, &map_ek, false, u);
      if (eok && ne > 0) {
        const int vs = nkv % C::VST;
        if (nkv < C::VST || wait_bounded(v_empty + vs, ((nkv / C::VST) - 1) & 1, wd, kSiteFwdKvEmpty)) {
          mbar_arrive_expect_tx(v_full + vs, C::TILE);
          for (int c = 0; c < C::KCH; ++c)
            tma_load_4d(sV + vs * C::TILE + c * C::CHUNK, &map_ev, v_full + vs, c * 64, kvh, erow, MODE == 1 ? 0 : 1);
        } else {
          eok = false;
        }
      }
      if (eok && ne > 1) k_stage_load(nkv + 2, &map_ev, true, 1);
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
      bool ok = true;
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
            if (j == 0 && !wait_warp(q_full + t, 0, wd, kSiteFwdQ)) {
              ok = false;
              break;
            }
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
  } else if (warp == 2 || warp == 3) {
    zero_share(64, 64);
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
    const int lo = MODE == 1 ? block_row_start(g, lim) : 0;  // first visible key of this row
    float m_run = -INFINITY;
    float l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      if (!wait_warp(s_full + t, j & 1, wd, kSiteFwdSFull)) {  // warp-agreed: TMEM access follows
        ok = false;
        break;
      }
      if (lane == 0 && wq == 0) TTT_TRACE(4 + t, j);
      if (lane == 0 && wq == 0 && t == 0 && j == 0) TTT_CTA_MARK(1);
      tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(lane_base + colS + 32 * c, sr[c]);
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < 4; ++c) reg_fence32(sr[c]);
      const int k0 = (jlo + j) * C::BN;
      if (k0 + C::BN - 1 > lim || k0 < lo) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (k0 + 32 * c + e > lim || k0 + 32 * c + e < lo) sr[c][e] = __float_as_uint(-INFINITY);
      }
      // row max: 8 independent chains of three-input maxima, then a tree
      float mxv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        mxv[u] = max3f(__uint_as_float(sr[0][u]), __uint_as_float(sr[0][u + 8]), __uint_as_float(sr[0][u + 16]));
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        mxv[u] = max3f(mxv[u], __uint_as_float(sr[0][u + 24]), __uint_as_float(sr[1][u]));
        mxv[u] = max3f(mxv[u], __uint_as_float(sr[1][u + 8]), __uint_as_float(sr[1][u + 16]));
        mxv[u] = max3f(mxv[u], __uint_as_float(sr[1][u + 24]), __uint_as_float(sr[2][u]));
        mxv[u] = max3f(mxv[u], __uint_as_float(sr[2][u + 8]), __uint_as_float(sr[2][u + 16]));
        mxv[u] = max3f(mxv[u], __uint_as_float(sr[2][u + 24]), __uint_as_float(sr[3][u]));
        mxv[u] = max3f(mxv[u], __uint_as_float(sr[3][u + 8]), __uint_as_float(sr[3][u + 16]));
        mxv[u] = fmaxf(mxv[u], __uint_as_float(sr[3][u + 24]));
      }
      mxv[0] = max3f(mxv[0], mxv[1], mxv[2]);
      mxv[3] = max3f(mxv[3], mxv[4], mxv[5]);
      mxv[6] = fmaxf(mxv[6], mxv[7]);
      mxv[0] = max3f(mxv[0], mxv[3], mxv[6]);
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
      uint64_t rs2[4] = {0ull, 0ull, 0ull, 0ull};  // paired row-sum accumulators
      // a row that has seen no key yet (a sliding window's leading tiles) exponentiates
      // against 0: its scores are all -inf, so its P is 0
      const float mneg = m_run == -INFINITY ? 0.f : -m_run;
      const uint64_t sl2x2 = f2_pack(sl2, sl2), negm2 = f2_pack(mneg, mneg);
      // P = 2^(s*scale*log2e - m), bf16 pairs into the first 64 columns of S_t; the first
      // 64 keys are released to the MMA warp before the last 64 are computed
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[c][2 * e]), __uint_as_float(sr[c][2 * e + 1])), sl2x2, negm2),
                    x0, x1);
          const float p0 = exp2_approx(x0);
          const float p1 = exp2_approx(x1);
          rs2[e & 3] = f2_add(rs2[e & 3], f2_pack(p0, p1));
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
      rs2[0] = f2_add(f2_add(rs2[0], rs2[1]), f2_add(rs2[2], rs2[3]));
      float rs_lo, rs_hi;
      f2_unpack(rs2[0], rs_lo, rs_hi);
      l_run += rs_lo + rs_hi;
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
    // the epilogue tiles this query tile reads (warp-agreed waits)
    const int nkeys = MODE == 0 ? p_of[t] : MODE == 1 ? g.Bs : (g.ring == 2 ? p_of[t] : 0);  // epilogue keys
    const int ne_t = MODE == 1 ? ne : min(nkeys, ne);
    auto epi_tiles_ready = [&]() -> bool {
      // with no trunk key no product waited for the Q tile: the scores below read it
      if (nkv == 0 && !wait_warp(q_full + t, 0, wd, kSiteFwdQ)) return false;
      for (int u = 0; u < ne_t; ++u)
        if (!wait_warp(k_full + (nkv + u) % C::KST, ((nkv + u) / C::KST) & 1, wd, kSiteFwdKvFull)) return false;
      if (ne_t > 0 && !wait_warp(v_full + nkv % C::VST, (nkv / C::VST) & 1, wd, kSiteFwdKvFull)) return false;
      if (ne_t > 1 && !wait_warp(k_full + (nkv + 2) % C::KST, ((nkv + 2) / C::KST) & 1, wd, kSiteFwdKvFull))
        return false;
      return true;
    };
    if (ok && (nkv == 0 || wait_warp(o_final + t, 0, wd, kSiteFwdOFinal)) && epi_tiles_ready()) {
      tc_fence_after();
      if (lane == 0 && wq == 0 && t == 0) TTT_CTA_MARK(2);
      // ---- epilogue: the epilogue keys (a3) and the exact joint-LSE merge (a4).
      // MODE 0: query (pass p, position qpos) also sees k~_j[tau], V_j[tau] of the branch
      // passes j = 1..p (0-based) at its own position.  MODE 1: a block token also sees
      // the Bs keys of its own block (bidirectional).  MODE 2: the branch keys, in the step
      // that meets the chunk's own keys only.  The trunk partial is (m_run, l_run,
      // unnormalised O in TMEM), in log2 units; the keys join it one at a time by the
      // same online rule (running max, rescaled sum and O), each key's k~ and V rows
      // fetched in one round of loads, its score on the CUDA cores against q~ in smem.
      const bool valid = qpos < len;
      const int p = p_of[t], h = h_of[t];
      const int tau = seq_start + qpos;
      const int T = g.si.T;
      const int bstart = MODE == 1 ? tau - qpos % g.Bs : 0;  // first row of the block
      // key u (0-based) of the epilogue: k~ row and V row
      auto krow_of = [&](int u) -> const uint4* {
        const int64_t r = MODE != 1 ? (static_cast<int64_t>(u + 1) * g.Hkv + kvh) * T + tau
                                    : static_cast<int64_t>(kvh) * T + bstart + u;
        return reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.kr) + r * D);
      };
      auto vrow_of = [&](int u) -> const uint4* {
        return reinterpret_cast<const uint4*>(
            MODE != 1 ? static_cast<const __nv_bfloat16*>(a.v) + (u + 1) * g.skv +
                            (static_cast<int64_t>(tau) * g.Hkv + kvh) * D
                      : static_cast<const __nv_bfloat16*>(a.v) + (static_cast<int64_t>(bstart + u) * g.Hkv + kvh) * D);
      };
      // this row of the Q tile (q~ in, the output row out: each thread touches only its
      // own row, and every product that read the tile completed before o_final)
      uint8_t* srow = sQ + t * C::TILE + row * 128;
      auto unit = [&](int c8) -> uint8_t* { return srow + (c8 >> 3) * C::CHUNK + (((c8 & 7) ^ (row & 7)) << 4); };
      // the warp's 32 rows all belong to the sequence: the output goes out by one tensor
      // store per 64 columns
      const bool warp_full = MODE != 2 && q0 + 32 * wq + 32 <= len;
      float m = m_run, l = l_run;
      bool o_live = nkv > 0;  // O in TMEM holds the trunk part (CTA-uniform)
      // O <- alpha O + w V (V absent: w = 0), in TMEM for keys before the last, to the
      // output (scaled by 1 / l) for the last
      // 16-byte unit c8 of row rr of a 128-row tile in a ring stage (128-byte swizzle)
      auto tile_unit = [&](const uint8_t* stage, int rr, int c8) -> const uint4* {
        return reinterpret_cast<const uint4*>(stage + (c8 >> 3) * C::CHUNK + rr * 128 + (((c8 & 7) ^ (rr & 7)) << 4));
      };
      // V row: from a staged tile (vsm, row rr), else from global memory (vgl; none: w = 0)
      auto fold = [&](float alpha, float w, const uint4* vgl, const uint8_t* vsm, int rr, bool last) {
        const float inv_l = 1.f / l;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          if (o_live) {
            tmem_ld32(lane_base + colO + 32 * c, o);
            tmem_ld_wait();
            reg_fence32(o);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = 0u;
          }
          float acc[32];
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const uint4 v4 = vsm   ? *tile_unit(vsm, rr, 4 * c + q4)
                             : vgl ? __ldg(vgl + 4 * c + q4)
                                   : make_uint4(0u, 0u, 0u, 0u);
            const __nv_bfloat162* v2 = reinterpret_cast<const __nv_bfloat162*>(&v4);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const float2 f2 = __bfloat1622float2(v2[u]);
              acc[8 * q4 + 2 * u] = fmaf(w, f2.x, __uint_as_float(o[8 * q4 + 2 * u]) * alpha);
              acc[8 * q4 + 2 * u + 1] = fmaf(w, f2.y, __uint_as_float(o[8 * q4 + 2 * u + 1]) * alpha);
            }
          }
          if (!last) {
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(acc[e]);
            tmem_st32(lane_base + colO + 32 * c, o);
          } else if (MODE == 2) {
            if (valid) {
              float4* dst = reinterpret_cast<float4*>(a.o_part + ((static_cast<int64_t>(p) * T + tau) * g.H + h) * D +
                                                      32 * c);
#pragma unroll
              for (int q4 = 0; q4 < 8; ++q4)
                dst[q4] = make_float4(acc[4 * q4] * inv_l, acc[4 * q4 + 1] * inv_l, acc[4 * q4 + 2] * inv_l,
                                      acc[4 * q4 + 3] * inv_l);
            }
          } else {
            uint4 out[4];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
              out[q4] = make_uint4(pack_bf16x2(acc[8 * q4] * inv_l, acc[8 * q4 + 1] * inv_l),
                                   pack_bf16x2(acc[8 * q4 + 2] * inv_l, acc[8 * q4 + 3] * inv_l),
                                   pack_bf16x2(acc[8 * q4 + 4] * inv_l, acc[8 * q4 + 5] * inv_l),
                                   pack_bf16x2(acc[8 * q4 + 6] * inv_l, acc[8 * q4 + 7] * inv_l));
            if (warp_full) {
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4) *reinterpret_cast<uint4*>(unit(4 * c + q4)) = out[q4];
            } else if (valid) {
              uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.o) + p * g.sq +
                                                    (static_cast<int64_t>(tau) * g.H + h) * D + 32 * c);
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4) dst[q4] = out[q4];
            }
          }
        }
        if (!last) {
          tmem_st_wait();
          o_live = true;
        }
      };
      for (int u = 0; u < nkeys; ++u) {
        // key u from a staged tile when it is there: MODE 0 / 2 the first ne keys (row =
        // this row), MODE 1 the block rows inside this tile
        const uint8_t* ksm = nullptr;
        const uint8_t* vsm = nullptr;
        int rr = row;
        if (MODE == 1) {
          rr = row - qpos % g.Bs + u;
          if (ne > 0 && rr >= 0 && rr < C::BM) {
            ksm = sK + (nkv % C::KST) * C::TILE;
            vsm = sV + (nkv % C::VST) * C::TILE;
          }
        } else if (u < ne) {
          ksm = sK + ((nkv + u) % C::KST) * C::TILE;
          vsm = u == 0 ? sV + (nkv % C::VST) * C::TILE : sK + ((nkv + 2) % C::KST) * C::TILE;
        }
        const uint4* vgl = nullptr;
        float acc0 = 0.f, acc1 = 0.f;
        auto dot_unit = [&](int c8, const uint4& kq) {
          const uint4 qv = *reinterpret_cast<const uint4*>(unit(c8));
          const __nv_bfloat162* q2 = reinterpret_cast<const __nv_bfloat162*>(&qv);
          const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&kq);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 a2 = __bfloat1622float2(q2[e]);
            const float2 b2 = __bfloat1622float2(k2[e]);
            if (e & 1)
              acc1 = fmaf(a2.x, b2.x, fmaf(a2.y, b2.y, acc1));
            else
              acc0 = fmaf(a2.x, b2.x, fmaf(a2.y, b2.y, acc0));
          }
        };
        if (ksm) {
#pragma unroll
          for (int c8 = 0; c8 < D / 8; ++c8) dot_unit(c8, *tile_unit(ksm, rr, c8));
        } else {
          uint4 kv[D / 8];
          if (valid) {
            const uint4* kj = krow_of(u);
            vgl = vrow_of(u);
#pragma unroll
            for (int c8 = 0; c8 < D / 8; ++c8) kv[c8] = __ldg(kj + c8);
          } else {
#pragma unroll
            for (int c8 = 0; c8 < D / 8; ++c8) kv[c8] = make_uint4(0u, 0u, 0u, 0u);
          }
#pragma unroll
          for (int c8 = 0; c8 < D / 8; ++c8) dot_unit(c8, kv[c8]);
        }
        const float s = valid ? (acc0 + acc1) * sl2 : -INFINITY;
        const float m_new = fmaxf(m, s);
        const float base = m_new == -INFINITY ? 0.f : m_new;  // a row that has seen no key yet
        const float alpha = exp2_approx(m - base), w = exp2_approx(s - base);
        l = l * alpha + w;
        m = m_new;
        fold(alpha, w, vgl, vsm, rr, u + 1 == nkeys);
      }
      if (nkeys == 0) fold(1.f, 0.f, nullptr, nullptr, row, true);
      if (warp_full) {
        // this warp's 32 output rows are in the tile's shared memory: one tensor store per
        // 64 columns, issued once they are visible to the async proxy
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
#pragma unroll
          for (int cc = 0; cc < C::KCH; ++cc)
            tma_store_4d(&map_o, sQ + t * C::TILE + cc * C::CHUNK + wq * 32 * 128, cc * 64, h, seq_start + q0 + 32 * wq,
                         p);
          bulk_commit();
          bulk_wait_read0();
        }
        __syncwarp();
      }
      if (valid) a.lse[lse_index(g.si, g.H, p, h, n, tau, qpos)] = (m + __log2f(l)) * kLn2;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) TTT_CTA_MARK(3);
  if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

template <int D, int MODE>
cudaError_t launch(const TrunkFwdArgs& a, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                   const CUtensorMap& mo, const CUtensorMap& mek, const CUtensorMap& mev, cudaStream_t stream) {
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
  trunk_fwd_kernel<D, MODE><<<static_cast<unsigned>(blocks), C::THREADS, C::SMEM, stream>>>(mq, mk, mv, mo, mek, mev, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_trunk_fwd(const TrunkFwdArgs& a, const CUtensorMap& map_q, const CUtensorMap& map_k,
                             const CUtensorMap& map_v, const CUtensorMap& map_o, const CUtensorMap& map_ek,
                             const CUtensorMap& map_ev, cudaStream_t stream) {
  const bool d128 = a.g.D == 128;
  if (a.g.ring > 0)
    return d128 ? launch<128, 2>(a, map_q, map_k, map_v, map_o, map_ek, map_ev, stream)
                : launch<64, 2>(a, map_q, map_k, map_v, map_o, map_ek, map_ev, stream);
  if (a.g.Bs > 0)
    return d128 ? launch<128, 1>(a, map_q, map_k, map_v, map_o, map_ek, map_ev, stream)
                : launch<64, 1>(a, map_q, map_k, map_v, map_o, map_ek, map_ev, stream);
  return d128 ? launch<128, 0>(a, map_q, map_k, map_v, map_o, map_ek, map_ev, stream)
              : launch<64, 0>(a, map_q, map_k, map_v, map_o, map_ek, map_ev, stream);
}

}  // namespace ttt

TTT_TRACE_READER(ttt_trace_read_fwd)
