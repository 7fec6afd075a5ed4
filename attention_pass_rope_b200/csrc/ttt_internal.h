// Internal declarations shared by the host launcher (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ttt {

// Status word values (first 32-bit word of the workspace).
constexpr uint32_t kStatusTimeoutBase = 0x7100'0000u;  // | site code

// Wait-site codes recorded on timeout (low bits of the status word).
enum WaitSite : uint32_t {
  kSiteSelftest = 1,
  kSiteFwdQ = 0x10,
  kSiteFwdKvFull = 0x11,
  kSiteFwdKvEmpty = 0x12,
  kSiteFwdSFull = 0x13,
  kSiteFwdPFull = 0x14,
  kSiteFwdOFinal = 0x15,
  kSiteFwdDrain = 0x16,
  kSiteBwdQdoFull = 0x20,
  kSiteBwdQdoEmpty = 0x21,
  kSiteBwdKv = 0x22,
  kSiteBwdSdpFull = 0x23,
  kSiteBwdDsReady = 0x24,
  kSiteBwdMmaDone = 0x25,
  kSiteBwdDqFull = 0x26,
  kSiteBwdDqFree = 0x27,
  kSiteBwdFinal = 0x28,
  kSiteBwdDrain = 0x29,
  kSiteBwdSdpFree = 0x2a,
  kSiteBwdTicket = 0x2b,
  kSiteCeFull = 0x40,
  kSiteCeEmpty = 0x41,
  kSiteCeAccFull = 0x42,
  kSiteCeAccEmpty = 0x43,
  kSiteCeDrain = 0x44,
};

// Where the sequences are: dense batches (cu_seqlens == nullptr) hold nseq = B
// sequences of length S back to back; packed batches read cu_seqlens.
struct SeqInfo {
  const int32_t* cu_seqlens;  // device, nullptr for dense
  int nseq;                   // B (dense) or number of sequences
  int S;                      // dense sequence length (0 for packed)
  int T;                      // total tokens (B*S or mult * cu_seqlens[nseq])
  int max_len;                // longest sequence
  int mult;                   // packed: row counts are mult * the cu_seqlens entries (1 for tokens)
};

// The attention has two index spaces: query rows (si) and key rows (ksi), one sequence
// of each per batch entry.  For the TTT attention they are the same tokens.  For the
// block-draft attention (Bs > 0) query row r of sequence n is token r % Bs of block
// (start_n + r) / Bs, and the keys are the context tokens: the row sees the context
// keys 0..anchor of its block (qlim; a sliding-window layer only the last `window` of
// them) and the Bs keys of its own block.
struct Geometry {
  SeqInfo si;   // query rows (TTT: tokens; block draft: block rows)
  SeqInfo ksi;  // key rows (TTT: = si; block draft: context tokens)
  int P, H, Hkv, D;
  float theta;
  float scale;  // softmax scale sigma
  int64_t sq;   // elements between passes of the public q, o, dout, dq
  int64_t skv;  // elements between passes of the public k, v, dk, dv
  int Bs;                    // block-draft: tokens per block (0: TTT attention)
  const int32_t* anchors;    // block-draft: device int32, anchor position of every block
  int window;                // block-draft: trunk keys a - window + 1 .. a of anchor a (0: all)
  // context-parallel ring step (ring > 0): the queries are one chunk of a sequence, the
  // keys another chunk of the same sequence; query row r sees key row t iff
  // t <= r + limit_off (global positions: limit_off = q_start - kv_start >= 0)
  int ring;                  // 0: not a ring step; 1: without, 2: with the branch keys
  int limit_off;
  int pos0;                  // RoPE position of the first row (global position of a chunk)
};

// Status word of an argument error that only the device can see (block-draft anchors
// not non-decreasing within a sequence); reported as TTT_ERR_INVALID_ARG.
constexpr uint32_t kStatusBadAnchors = 0x7200'0001u;

// ----------------------------------------------------------------- launchers
// All launchers enqueue on `stream` and return the launch error.

// a1: q~ = R(i+p) q (head-major [P][H][T][D]), k~ = R(i+p) k ([P][Hkv][T][D]), bf16.
cudaError_t launch_rope_fwd(const Geometry& g, const void* q, const void* k, void* qr, void* kr,
                            cudaStream_t stream);

struct TrunkFwdArgs {
  Geometry g;
  float* o_part;   // ring step: fp32 partial output [P][Tq][H][D] (normalised over the step's keys)
  const void* kr;  // bf16 k~ head-major [P][Hkv][T][D] (branch keys, passes >= 1)
  const void* v;   // bf16 V, public layout [P][T][Hkv][D] (branch values; passes g.skv apart)
  void* o;         // bf16 output, public layout [P][T][H][D] (passes g.sq apart)
  float* lse;      // fp32 merged lse, public layout
  uint32_t* status;
  uint64_t budget_ns;
  // optional: a region that the otherwise idle warps zero while the attention runs (the
  // backward's dq~ accumulator, when the workspace is the backward's); 16-byte units
  float4* zero_base;
  int64_t zero_n16;
  uint32_t* dq_zeroed;  // optional marker word: set to kDqZeroedMagic when zero_n16 > 0, else to 0
};

// Workspace word next to the status word: the forward has zeroed the backward's dq~
// accumulator in this workspace (a backward told that the workspace is untouched since
// the forward then skips that zeroing, and clears the word).
constexpr uint32_t kDqZeroedMagic = 0x01010101u;  // every byte 1 (a byte-wise memset)
constexpr size_t kDqZeroedOffset = 4;
// a2+a3+a4: trunk causal attention on tcgen05 with the branch keys and the exact
// joint-LSE merge in its epilogue.  Maps: q~ (3D {D, T, P*H}), k~_1 (3D {D, T, Hkv}),
// V_1 (3D {D, Hkv, T}), all 64-element (128-byte) swizzled boxes; map_o is the bf16
// output (4D {D, H, T, P}, passes g.sq apart, box {64, 1, 32, 1}) that full 32-row
// warp slices are stored through (MODE 2 writes fp32 directly and ignores it).
// map_ek / map_ev cover the epilogue keys' k~ and V (a.kr, a.v) as 128-row tiles:
// MODE 0 / 2 k~ 3D {D, rows, P*Hkv} and V 4D {D, Hkv, rows, P} (passes g.skv apart);
// MODE 1 k~ 3D {D, rows, Hkv} and V 4D {D, Hkv, rows, 1}.
cudaError_t launch_trunk_fwd(const TrunkFwdArgs& a, const CUtensorMap& map_q, const CUtensorMap& map_k,
                             const CUtensorMap& map_v, const CUtensorMap& map_o, const CUtensorMap& map_ek,
                             const CUtensorMap& map_ev, cudaStream_t stream);

// Row statistics of the backward, tile-aligned: for query head (p, h) and the 64-row
// query tile j of sequence n, slot = start_n / 64 + n + j holds 64 values of
// lse * log2(e) followed by 64 values of delta (512 bytes, one bulk copy).  Slots of
// consecutive sequences never overlap: start_n/64 + n + ceil(len_n/64) <=
// start_{n+1}/64 + n + 1.  Padding entries are never written.
__host__ __device__ inline int ld_slots(const SeqInfo& si) { return si.T / 64 + si.nseq + 1; }

// a5: delta = rowsum(dO * O); writes the tile-aligned (-lse*log2e, delta) rows and
// zeroes the fp32 dq~ accumulator [P][H][T][D] (unless dq_zeroed is given and holds
// kDqZeroedMagic) and the per-slot order tickets.
// Block-draft geometry (g.Bs > 0): also writes qlim (the trunk-key limit of every query
// row) and records kStatusBadAnchors in *status if a sequence's anchors decrease.
cudaError_t launch_bwd_preprocess(const Geometry& g, const void* o, const void* dout, const float* lse, float* ld,
                                  float* dq_acc, int* tickets, int* qlim, uint32_t* status,
                                  const uint32_t* dq_zeroed, cudaStream_t stream);

struct TrunkBwdArgs {
  Geometry g;
  const float* ld;     // tile-aligned (lse*log2e, delta) rows, see ld_slots
  float* dq_acc;       // fp32 [P][H][Tq][D], zeroed before the launch
  void* dk;            // bf16 public dk of the trunk keys (pass 0 / the context): written here
  void* dv;            // bf16 public dv of the trunk keys: written here
  int* tickets;        // nullptr, or per statistics slot: key tiles whose dq~ is added (ordered mode)
  const int* qlim;     // block-draft: trunk-key limit of every query row; nullptr otherwise
  uint32_t* status;
  uint64_t budget_ns;
  // ring step (g.ring > 0): the visiting chunk's dk~ (before sigma and the inverse
  // rotation) and dV as fp32 [Hkv][klen][D], added to (dk / dv are not written)
  float* dk_acc;
  float* dv_acc;
};
// a6: trunk backward on tcgen05; maps: q~ (box 64 rows), k~_1 (box 128 rows),
// V_1 (box 128 rows), dO (4D {D, H, T, P}, pass stride g.sq, box 64 rows).
cudaError_t launch_trunk_bwd(const TrunkBwdArgs& a, const CUtensorMap& map_q, const CUtensorMap& map_k,
                             const CUtensorMap& map_v, const CUtensorMap& map_do, cudaStream_t stream);

// a7+a8: branch backward, dq finalize (inverse RoPE), dk/dv of the branch passes.
cudaError_t launch_branch_bwd(const Geometry& g, const void* qr, const void* kr, const void* v,
                              const void* dout, const float* lse, const float* ld, const float* dq_acc,
                              void* dq, void* dk, void* dv, cudaStream_t stream);

// Block-draft: head-major rotated copies dst[head][tau][:] = R(pos(tau)) src[tau][head][:]
// of up to two tensors sharing the rows' positions: context tokens (block_rows = false,
// rows of g.ksi, position in the sequence) or block tokens (rows of g.si, position =
// the block's clamped anchor + the token's index in the block).
cudaError_t launch_rope_rows(const Geometry& g, bool block_rows, int T, const void* src_a, int nha, void* dst_a,
                             const void* src_b, int nhb, void* dst_b, cudaStream_t stream);

// Block-draft: backward of the block part, dq of the block tokens (adding the trunk part
// from dq_acc), dk and dv of the block tokens.
cudaError_t launch_block_bwd(const Geometry& g, const void* qr, const void* kr, const void* vb, const void* dout,
                             const float* lse, const float* ld, const float* dq_acc, void* dq, void* dk, void* dv,
                             cudaStream_t stream);

// Ring: running merge of partial results (acc <- acc (+) part by log-sum-exp; `first`
// copies), and the final bf16 output.  O rows are [P][Lq][H][D] fp32, lse [P][H][Lq].
// Ring backward: a chunk's trunk dK / dV from its returned fp32 accumulators
// ([Hkv][n][D], dk~ before sigma and the inverse rotation), bf16 into the pass-1 rows.
cudaError_t launch_ring_dkv_finish(const Geometry& g, int n, const float* dk_acc, const float* dv_acc, void* dk,
                                   void* dv, cudaStream_t stream);
cudaError_t launch_ring_merge(int rows, int D, int H, int Lq, float* o_acc, float* lse_acc, const float* o_part,
                              const float* lse_part, bool first, cudaStream_t stream);
cudaError_t launch_ring_finish(int64_t n, const float* o_acc, void* o, cudaStream_t stream);

cudaError_t launch_watchdog_selftest(uint32_t* status, uint64_t budget_ns, cudaStream_t stream);

// Arguments of the soft cross-entropy GEMM kernel (softce.cu).  Output tile rows are
// draft rows row0 + m (STATS, DZ) or the GEMM's own rows (BF16, ACC).
struct SoftceGemmArgs {
  int M, N, K;              // output rows, output columns, reduction depth
  int row0;                 // STATS / DZ: first draft row of this launch
  int R;                    // draft rows in all (the stride of stats and lse)
  int V;                    // vocabulary (teacher row length)
  const int32_t* tidx;      // [R] teacher row of every draft row, -1 = invalid
  const void* y;            // bf16 teacher logits [T][V]
  float* stats;             // STATS: [ceil(V/256)][5][R] per-tile softmax statistics
  const float* lse;         // DZ: [2][R] logsumexp of the draft and of the teacher row
  const float* coef;        // DZ: [R] gradient coefficient g * w_p / N_p (0 = invalid)
  uint32_t* status;
  uint64_t budget_ns;
};

// Helpers of api.cu that the other host entry points share.
// 2-D tensor map (dims and strides innermost first), box {b0, b1}.
bool encode_map_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t d0, uint64_t d1,
                   uint64_t s1_bytes, uint32_t b0, uint32_t b1, CUtensorMapSwizzle sw);
uint64_t wait_budget_ns();
void record_cuda_error(int code);

}  // namespace ttt
