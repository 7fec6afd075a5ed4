/*
 * ttt_attn.h — C ABI of libttt_attn.so: forward and backward of the multi-pass
 * EAGLE-3 test-time-training (TTT) trunk+branch attention on NVIDIA B200 (sm_100a).
 *
 * What is computed.  Sources: "DFlash/DSpark and EAGLE-3 TTT draft co-training for
 * speculative decoding (Megatron backend)" (NeMo-RL issue 3698), section "What I'm
 * working on", items 1 and 4; "bounded multi-pass EAGLE-3 TTT provider" (NeMo-RL
 * PR 3725), Summary and self-review.
 *
 *   For pass p = 1..P, query head h, sequence position i (0-based within its
 *   sequence), with kv(h) = h / (H / Hkv) and sigma the softmax scale:
 *     q~_p[i] = R(i+p-1) Q_p[i],  k~_p[i] = R(i+p-1) K_p[i]      (rotate-half RoPE)
 *     trunk keys:  k~_1[t], V_1[t]  for t = 0..i                   (causal)
 *     branch keys: k~_j[i], V_j[i]  for j = 2..p                   (staircase)
 *     s = sigma * q~_p[i] . k ;  lse_t, O_t over the trunk keys, lse_b, O_b over
 *     the branch keys (empty for p = 1: lse_b = -inf);
 *     lse = logaddexp(lse_t, lse_b),  O = e^(lse_t-lse) O_t + e^(lse_b-lse) O_b.
 *   This equals one softmax over the (i+1)+(p-1) visible keys.  The rotated q~ and
 *   k~ are evaluated in double precision and rounded to bf16 (through fp32) before the
 *   dot products, which run on bf16 tensor-core operands with fp32 accumulation.
 *   R(m) pairs dimension d with d + D/2 and rotates by m * theta^(-2d/D).
 *
 * Layouts (all pass-major, the trunk is index 0 along P, row-major):
 *   dense (TTT_LAYOUT_BSHD):  q, o, dout, dq  [P][B][S][H][D]    bf16
 *                             k, v, dk, dv    [P][B][S][Hkv][D]  bf16
 *                             lse             [P][B][H][S]       fp32 (natural log)
 *   packed (TTT_LAYOUT_THD):  q, o, dout, dq  [P][T][H][D], k, v, dk, dv [P][T][Hkv][D],
 *                             lse [P][H][T]; sequences given by cu_seqlens (int32,
 *                             device memory, nseq+1 entries, cu_seqlens[0] = 0,
 *                             non-decreasing, cu_seqlens[nseq] = T); positions restart
 *                             at 0 at every sequence start and no attention crosses
 *                             a sequence boundary.
 *   Within a pass every tensor is contiguous.  Consecutive passes of q, o, dout and dq
 *   are desc->pass_stride_q elements apart, those of k, v, dk and dv
 *   desc->pass_stride_kv elements apart (0 selects the packed value, T*H*D and
 *   T*Hkv*D; T = B*S for dense batches), so a caller that produces the passes one at a
 *   time can place them at a common stride in one allocation instead of
 *   concatenating them.  lse is always packed.
 *   Supported: D in {64, 128}; H a multiple of Hkv; 1 <= P <= 16.
 *
 * Ownership.  Every pointer is device memory owned by the caller, including the
 * workspace, whose size ttt_attn_workspace_size() returns.  The library allocates
 * nothing and keeps no per-call state between calls, with these exceptions: the
 * no-allocation forward (ttt_attn_fwd_noalloc) uses a fixed 32 MiB array in the
 * library's own device memory, held by every GPU that loads the library, whose device
 * address is looked up once per device and cached; the in-kernel wait limit
 * (ttt_attn_set_wait_budget_ns) and the last CUDA error (ttt_attn_last_cuda_error)
 * are process-wide.  Outputs must not alias inputs.
 *
 * Asynchrony and errors.  Calls enqueue work on `stream` (a cudaStream_t; NULL is
 * the legacy default stream) and return without synchronising.  Argument errors
 * are reported before anything is enqueued.  TTT_ERR_CUDA reports a launch error.
 * Every wait inside the kernels is bounded; a wait that runs out records its site
 * in the workspace status word and the kernel exits cleanly;
 * ttt_attn_device_status() synchronises the stream and reports it as
 * TTT_ERR_DEVICE_TIMEOUT.
 */
#ifndef TTT_ATTN_H_
#define TTT_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TTT_OK = 0,
  TTT_ERR_INVALID_ARG = 1,    /* null pointer, bad size, inconsistent shape */
  TTT_ERR_UNSUPPORTED = 2,    /* valid but not implemented (e.g. D = 96) */
  TTT_ERR_WORKSPACE = 3,      /* workspace missing, too small or misaligned */
  TTT_ERR_CUDA = 4,           /* a CUDA runtime/driver call failed */
  TTT_ERR_DEVICE_TIMEOUT = 5  /* a bounded in-kernel wait ran out */
} ttt_status;

typedef enum { TTT_LAYOUT_BSHD = 0, TTT_LAYOUT_THD = 1 } ttt_layout;

/* Optional per-kernel timing: when the descriptor points at one of these, each
 * kernel k of a call is bracketed by cudaEventRecord(start[k]) / (stop[k]) on the
 * call's stream (entries left NULL are skipped).  Indices: TTT_KERNEL_*. */
enum {
  TTT_KERNEL_ROPE_FWD = 0,
  TTT_KERNEL_TRUNK_FWD = 1,
  TTT_KERNEL_UNUSED_2 = 2, /* the branch keys and the merge run in the trunk forward's epilogue */
  TTT_KERNEL_ROPE_BWD = 3,
  TTT_KERNEL_BWD_PREPROCESS = 4,
  TTT_KERNEL_TRUNK_BWD = 5,
  TTT_KERNEL_BRANCH_BWD = 6,
  TTT_KERNEL_COUNT = 8
};
typedef struct {
  void* start[TTT_KERNEL_COUNT]; /* cudaEvent_t */
  void* stop[TTT_KERNEL_COUNT];  /* cudaEvent_t */
} ttt_attn_events;

typedef struct {
  int layout;          /* ttt_layout */
  int P;               /* TTT passes (1 = plain causal attention) */
  int B, S;            /* dense: batch and sequence length (ignored for THD) */
  int H, Hkv, D;       /* query heads, KV heads, head dimension */
  float rope_theta;    /* RoPE base, > 0 */
  float softmax_scale; /* 0 selects 1/sqrt(D) */
  const int32_t* cu_seqlens; /* THD only: device int32[nseq+1] */
  int nseq;            /* THD only: number of sequences */
  int total_tokens;    /* THD only: T = cu_seqlens[nseq] */
  int max_seqlen;      /* THD only: upper bound on every sequence length */
  const ttt_attn_events* events; /* optional, NULL for none */
  int flags;           /* TTT_FLAG_* bits, 0 for none; other bits are rejected */
  /* Elements between consecutive passes of q, o, dout, dq (pass_stride_q) and of k, v,
   * dk, dv (pass_stride_kv); 0 = packed.  A non-zero stride must be a multiple of 8
   * (16 bytes) and at least the packed value (passes never overlap); with P = 1 it is
   * ignored.  Source: the boundary of the "DFlash/DSpark and EAGLE-3 TTT draft
   * co-training" roadmap (NeMo-RL issue 3698), items 1 and 4: passes run one after
   * another and hand their q/k/v to the attention as they are produced. */
  int64_t pass_stride_q;
  int64_t pass_stride_kv;
} ttt_attn_desc;

/* Descriptor flags. */
typedef enum {
  /* ttt_attn_bwd: the workspace still holds the rotated q~ / k~ that ttt_attn_fwd
   * wrote for this descriptor and these q, k (same workspace, untouched since), so
   * the backward uses them instead of rotating q and k again.  The backward's
   * workspace layout starts with the forward's (ttt_attn_workspace_layout), so a
   * workspace sized for the backward and passed to both calls qualifies.  If the
   * promise is broken the gradients are wrong; nothing is read out of bounds.
   * A forward given a workspace of at least the backward's size also zeroes the
   * backward's dq~ accumulator in it (on warps the attention leaves idle) and marks
   * that in the word after the status word; a backward with this flag then skips
   * its own zeroing, and every backward clears the mark. */
  TTT_FLAG_ROTATED_IN_WORKSPACE = 1,
  /* ttt_attn_bwd: bitwise reproducible dq.  The trunk backward adds the fp32
   * partial dq~ of the key tiles of a query tile in key-tile order (each waits,
   * bounded, for its predecessor's sum) instead of in arrival order.  Everything
   * else in the library is already deterministic.  Slower: the dq~ additions of a
   * query tile are serialised.  Ignored by ttt_attn_fwd. */
  TTT_FLAG_DETERMINISTIC_DQ = 2
} ttt_flag;

/* Bytes of workspace that ttt_attn_fwd (for_backward = 0) or ttt_attn_bwd
 * (for_backward = 1) needs for `desc`; 0 if the descriptor is invalid.  The
 * workspace must be 256-byte aligned. */
size_t ttt_attn_workspace_size(const ttt_attn_desc* desc, int for_backward);

/* Forward.  q, k, v: bf16 pre-RoPE inputs (layouts above).  o: bf16 output, same
 * layout as q.  lse: fp32 merged log-sum-exp (natural log of the sum of
 * exp(sigma * q~.k) over the visible keys).  The workspace holds, after the call,
 * the rotated q~ / k~ (see ttt_attn_workspace_layout). */
ttt_status ttt_attn_fwd(const ttt_attn_desc* desc, const void* q, const void* k, const void* v, void* o,
                        float* lse, void* workspace, size_t workspace_bytes, void* stream);

/* Backward of the forward above, recomputing the probabilities from the merged
 * lse.  dout: bf16 gradient of o.  dq, dk, dv: bf16 gradients with respect to the
 * PRE-RoPE q, k and v (the RoPE rotation is transposed; its bf16 rounding is
 * treated as the identity).  o and lse must be the forward's outputs for the same
 * inputs.  dk/dv of the trunk pass collect every pass and query head of the
 * group; those of branch pass j collect passes p >= j at the same position. */
ttt_status ttt_attn_bwd(const ttt_attn_desc* desc, const void* q, const void* k, const void* v, const void* o,
                        const float* lse, const void* dout, void* dq, void* dk, void* dv, void* workspace,
                        size_t workspace_bytes, void* stream);

/* Forward for callers that cannot allocate device memory.  The pages describe no
 * such entry point; it is a deployment aid.  A caller such as a plugin in a host
 * framework that owns every device allocation, or a latency-critical loop where
 * cudaMalloc (which can synchronise the device) is not acceptable, has no way to
 * provide the workspace ttt_attn_fwd needs.  This call computes exactly what
 * ttt_attn_fwd computes (same arguments, same outputs) with its scratch in a fixed
 * 32 MiB array inside the library's own device memory, held by every GPU that
 * loads the library until the process exits.  It allocates nothing (no cudaMalloc,
 * cudaFree or allocating library call).  Returns TTT_ERR_WORKSPACE, before
 * enqueuing anything, when ttt_attn_workspace_size(desc, 0) exceeds 32 MiB.  The
 * first call on a device looks up the array's device address (cudaGetSymbolAddress)
 * with that device current; make that first call before any stream capture.  All
 * calls on a device share the array and it keeps the last call's contents (the
 * call clears what must start at zero); calls whose GPU work overlaps (unordered
 * streams) race on it, so order them on one stream. */
ttt_status ttt_attn_fwd_noalloc(const ttt_attn_desc* desc, const void* q, const void* k, const void* v, void* o,
                                float* lse, void* stream);

/* ttt_attn_device_status() for ttt_attn_fwd_noalloc, whose status word is the first
 * word of the library's scratch array on the current device (the caller has no pointer
 * to it): synchronises `stream`, returns TTT_OK or TTT_ERR_DEVICE_TIMEOUT (raw word in
 * *detail if non-NULL) and clears the word.  Allocates nothing.  Like the forward, its
 * first call on a device looks up the array's address. */
ttt_status ttt_attn_fwd_noalloc_status(void* stream, uint32_t* detail);

/* ttt_attn_watchdog_selftest() with its status word in that scratch array: lets a
 * caller of the no-allocation forward check that a wait that runs out is reported
 * through ttt_attn_fwd_noalloc_status(). */
ttt_status ttt_attn_noalloc_watchdog_selftest(uint64_t budget_ns, void* stream);

/* ------------------------------------------------------------------------------
 * Block-draft attention of DFlash/DSpark drafters.  Source: "DFlash/DSpark and EAGLE-3
 * TTT draft co-training ..." (NeMo-RL issue 3698), "What I'm working on", item 2
 * (anchor + mask-token block drafting: bidirectional in-block attention, trunk
 * truncated at the anchor) and item 4 (packed THD layout).
 *
 *   A block b of Bs tokens starts at the anchor position a_b of its sequence; its
 *   token j sits at position a_b + j and has its own q, k, v.  With kv(h) = h / (H/Hkv):
 *     q~ = R(a_b + j) q,  k~ = R(a_b + j) k (block tokens),  k~_ctx[t] = R(t) k_ctx[t]
 *     trunk keys: k~_ctx[t], v_ctx[t] for t = s_b..a_b          (truncated at the anchor;
 *                 s_b = 0, or max(0, a_b - window + 1) for a sliding-window layer)
 *     block keys: k~, v of the Bs tokens of block b             (bidirectional)
 *     lse = logaddexp(lse_trunk, lse_block), O = the exact merge of the two partial
 *     softmaxes, i.e. one softmax over the (a_b - s_b + 1) + Bs visible keys.
 *   Rotated q~ / k~ are rounded to bf16 before the dot products, as in the TTT call.
 *
 * Layouts (row-major, contiguous; NB = total blocks, Tc = total context tokens):
 *   dense (TTT_LAYOUT_BSHD): B sequences of S context tokens and nblk blocks each:
 *     k_ctx, v_ctx, dk_ctx, dv_ctx [B][S][Hkv][D];  qb, o, dout, dqb [B][nblk][Bs][H][D];
 *     kb, vb, dkb, dvb [B][nblk][Bs][Hkv][D];  anchors int32 [B][nblk];
 *     lse fp32 [B][H][nblk*Bs].
 *   packed (TTT_LAYOUT_THD): cu_ctx (context tokens) and cu_blocks (blocks), device
 *     int32[nseq+1] prefix sums: k_ctx.. [Tc][Hkv][D], qb.. [NB][Bs][H][D],
 *     kb.. [NB][Bs][Hkv][D], anchors [NB], lse [H][NB*Bs].
 *   anchors: device int32, each block's anchor position within its sequence, in
 *   [0, its context length) (values outside are clamped to it) and non-decreasing
 *   within a sequence (the backward relies on the order and reports a violation as
 *   TTT_ERR_INVALID_ARG through ttt_attn_device_status; the forward is exact for any
 *   order).  Supported: D in {64, 128}, H a multiple of Hkv, 1 <= Bs <= 16.
 * Ownership, asynchrony, errors and the workspace contract are those of the TTT calls
 * above; descriptor flags TTT_FLAG_ROTATED_IN_WORKSPACE and TTT_FLAG_DETERMINISTIC_DQ
 * mean the same (the forward's workspace layout is a prefix of the backward's).
 * ------------------------------------------------------------------------------ */
typedef struct {
  int layout;                /* ttt_layout */
  int B, S, nblk;            /* dense: sequences, context length, blocks per sequence */
  int H, Hkv, D;             /* query heads, KV heads, head dimension */
  int Bs;                    /* tokens per block, 1..16 */
  float rope_theta;          /* RoPE base, > 0 */
  float softmax_scale;       /* 0 selects 1/sqrt(D) */
  const int32_t* anchors;    /* device int32[NB] */
  const int32_t* cu_ctx;     /* THD: device int32[nseq+1], context tokens */
  const int32_t* cu_blocks;  /* THD: device int32[nseq+1], blocks */
  int nseq;                  /* THD: sequences */
  int total_ctx;             /* THD: Tc = cu_ctx[nseq] */
  int total_blocks;          /* THD: NB = cu_blocks[nseq] */
  int max_ctx;               /* THD: upper bound on every context length */
  int max_blocks;            /* THD: upper bound on every sequence's block count */
  const ttt_attn_events* events; /* optional: TTT_KERNEL_ROPE_FWD, _TRUNK_FWD, _ROPE_BWD,
                                    _BWD_PREPROCESS, _TRUNK_BWD, _BRANCH_BWD (block part) */
  int flags;                 /* TTT_FLAG_* bits */
  /* Sliding-window block layers ("DFlash/DSpark and EAGLE-3 TTT draft co-training",
   * NeMo-RL issue 3698, "What I'm working on", item 4): a block anchored at a sees only
   * the context keys a - window + 1 .. a (from 0 when that is negative); 0 = the whole
   * trunk 0..a.  >= 0. */
  int window;
} ttt_block_desc;

/* Workspace bytes of ttt_block_attn_fwd (for_backward = 0) or ttt_block_attn_bwd (1); 0
 * for an invalid descriptor.  256-byte aligned. */
size_t ttt_block_workspace_size(const ttt_block_desc* desc, int for_backward);

/* Sub-buffers: fwd [0] status word, [1] q~ of the block tokens bf16 [H][NB*Bs][D],
 * [2] k~_ctx bf16 [Hkv][Tc][D], [3] k~ of the block tokens bf16 [Hkv][NB*Bs][D];
 * bwd adds [4] row statistics (as for the TTT call, over the block rows), [5] dq~
 * accumulator fp32 [H][NB*Bs][D], [6] order tickets, [7] int32 trunk-key limit of
 * every block row.  Returns the number of entries (at most 8), 0 if invalid. */
int ttt_block_workspace_layout(const ttt_block_desc* desc, int for_backward, size_t* offsets);

/* Forward: o (bf16, like qb) and lse (fp32 natural log). */
ttt_status ttt_block_attn_fwd(const ttt_block_desc* desc, const void* k_ctx, const void* v_ctx, const void* qb,
                              const void* kb, const void* vb, void* o, float* lse, void* workspace,
                              size_t workspace_bytes, void* stream);

/* Backward, recomputing the probabilities from lse: gradients with respect to the
 * pre-RoPE inputs (bf16).  dk_ctx / dv_ctx of context keys no block sees are zero. */
ttt_status ttt_block_attn_bwd(const ttt_block_desc* desc, const void* k_ctx, const void* v_ctx, const void* qb,
                              const void* kb, const void* vb, const void* o, const float* lse, const void* dout,
                              void* dk_ctx, void* dv_ctx, void* dqb, void* dkb, void* dvb, void* workspace,
                              size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------------
 * Context-parallel ring over the pass-1 trunk K/V.  Source: "DFlash/DSpark and EAGLE-3
 * TTT draft co-training ..." (NeMo-RL issue 3698), "What I'm working on", item 4 (pass-1
 * trunk K/V on a zigzag ring, exact joint-LSE merge).
 *
 * The sequence is cut into chunks held by different ranks.  A rank rotates its query
 * chunks (ttt_ring_rotate: every pass of q and k at the chunk's global positions), and
 * in each ring step computes the attention of a local query chunk against a visiting
 * chunk of rotated pass-1 keys and of pass-1 values, causal by global position
 * (ttt_ring_step), merging the partial into a running result (ttt_ring_merge); the last
 * step writes the bf16 output (ttt_ring_finish).  The chunk that meets its own trunk
 * keys also takes the branch keys (include_branch).  After every visiting chunk whose
 * start is at or before the query chunk's has been merged, the result equals
 * ttt_attn_fwd's on the whole sequence (up to rounding).  Moving chunks between ranks
 * is the caller's (e.g. NCCL send/recv into this GPU's memory); these calls read this
 * GPU's memory only.  Rows: queries [P][q_len][H][D], local k/v [P][q_len][Hkv][D];
 * rotated local qr [P][H][q_len][D], kr [P][Hkv][q_len][D]; visiting keys
 * kr_visit [Hkv][kv_len][D] (rotated, i.e. pass 0 of the owner's kr) and values
 * v_visit [kv_len][Hkv][D]; partial and running outputs fp32 [P][q_len][H][D] with lse
 * fp32 [P][H][q_len]. */
typedef struct {
  int P, H, Hkv, D;
  float rope_theta;
  float softmax_scale;       /* 0 selects 1/sqrt(D) */
  int q_len, q_start;        /* local query chunk: rows, global position of its first row */
  int kv_len, kv_start;      /* visiting key chunk: rows, global position of its first row */
  int include_branch;        /* 1: this step also takes the branch keys (the local chunk's) */
} ttt_ring_desc;

/* qr, kr <- the rotated local chunk (positions q_start + i + p), head-major. */
ttt_status ttt_ring_rotate(const ttt_ring_desc* desc, const void* q, const void* k, void* qr, void* kr, void* stream);

/* One ring step: partial (o_part, lse_part) of the local queries over the visiting
 * chunk's keys (and the branch keys with include_branch).  Requires kv_start <= q_start
 * (a chunk that starts later holds no visible key: skip it).  kr_local / v_local (the
 * local chunk's rotated keys and public-layout values) are read only with
 * include_branch.  status: a device word for the bounded waits (read it with
 * ttt_attn_device_status). */
ttt_status ttt_ring_step(const ttt_ring_desc* desc, const void* qr, const void* kr_local, const void* v_local,
                         const void* kr_visit, const void* v_visit, float* o_part, float* lse_part, void* status,
                         void* stream);

/* o_acc, lse_acc <- their exact log-sum-exp merge with o_part, lse_part (first != 0:
 * copy). */
ttt_status ttt_ring_merge(const ttt_ring_desc* desc, float* o_acc, float* lse_acc, const float* o_part,
                          const float* lse_part, int first, void* stream);

/* o (bf16 [P][q_len][H][D]) <- o_acc; the lse is lse_acc itself. */
ttt_status ttt_ring_finish(const ttt_ring_desc* desc, const float* o_acc, void* o, void* stream);

/* Ring backward (same page and item).  With the final o, lse of a local chunk and its
 * dout:
 *   1. ttt_ring_bwd_prepare: delta = rowsum(dout * o) and the row statistics into the
 *      chunk's workspace, its fp32 dq~ accumulator zeroed (the workspace's first word
 *      is the status word of the bounded waits: ttt_attn_device_status);
 *   2. ttt_ring_bwd_step, once per visiting chunk the forward met (kv_start <= q_start):
 *      adds the chunk's trunk dq~ to the accumulator, and the visiting keys' dk~ (before
 *      sigma and the inverse rotation) and dV to dk_acc, dv_acc (fp32 [Hkv][kv_len][D]);
 *      these accumulators travel with the visiting chunk and come home after the ring
 *      (moving them is the caller's, as in the forward);
 *   3. ttt_ring_bwd_finish: the branch keys' part, dq (every pass) and the dK / dV of
 *      the branch passes (p >= 2) of the local chunk, bf16 in the public layout;
 *   4. ttt_ring_dkv_finish on a chunk's returned accumulators (desc describing that
 *      chunk: q_len, q_start): the pass-1 rows of its dk, dv.
 * After all of it the gradients equal ttt_attn_bwd's on the whole sequence (up to
 * rounding and the order of the fp32 additions).  Layouts as in the forward; dq, dout
 * [P][q_len][H][D], dk, dv [P][q_len][Hkv][D].  The calls read and write this GPU's
 * memory only. */
size_t ttt_ring_bwd_workspace_size(const ttt_ring_desc* desc);
ttt_status ttt_ring_bwd_prepare(const ttt_ring_desc* desc, const void* o, const float* lse, const void* dout,
                                void* workspace, size_t workspace_bytes, void* stream);
ttt_status ttt_ring_bwd_step(const ttt_ring_desc* desc, const void* qr, const void* dout, const void* kr_visit,
                             const void* v_visit, float* dk_acc, float* dv_acc, void* workspace,
                             size_t workspace_bytes, void* stream);
ttt_status ttt_ring_bwd_finish(const ttt_ring_desc* desc, const void* qr, const void* kr_local, const void* v_local,
                               const void* dout, const float* lse, void* dq, void* dk, void* dv, void* workspace,
                               size_t workspace_bytes, void* stream);
ttt_status ttt_ring_dkv_finish(const ttt_ring_desc* desc, const float* dk_acc, const float* dv_acc, void* dk,
                               void* dv, void* stream);

/* ------------------------------------------------------------------------------
 * Soft cross-entropy distillation loss of the draft passes.  Source: "DFlash/DSpark
 * and EAGLE-3 TTT draft co-training ..." (NeMo-RL issue 3698), "What I'm working on",
 * item 3 (the draft learns the target's distribution through a soft cross-entropy,
 * computed in token chunks and split over the vocabulary, normalised per pass over
 * the global batch) and item 2 (the draft rides the target's vocabulary head); the
 * loss's token_chunk_size, default 4096 tokens: "bounded multi-pass EAGLE-3 TTT
 * provider" (NeMo-RL PR 3725), merge note 3.
 *
 *   Draft row r = p*T + t (pass p = 0..P-1, token t of the packed tokens) has logits
 *   z_r = W h_r (fp32 sums of bf16 products).  Its teacher position u = t + p must lie
 *   in t's sequence and have loss_mask[u] != 0, else the row is invalid:
 *     l_r = logsumexp(z_r) - sum_v softmax(y_u)_v z_r,v   (0 for an invalid row),
 *     N_p = pass_count[p] if given, else the number of valid rows of pass p,
 *     L_p = w_p / N_p * sum_t l_{p,t}  (0 if N_p = 0),   L = sum_p L_p.
 *   Backward of grad * L: dz_r = grad * w_p / N_p * (softmax(z_r) - softmax(y_u)),
 *   rounded to bf16; dh_r = W^T dz_r; dW += sum_r dz_r h_r^T.  The teacher y is not
 *   differentiated.
 *
 * Layouts (device memory, row-major, 16-byte aligned): h bf16 [P][T][d], W bf16 [V][d],
 * y bf16 [T][V], dh bf16 [P][T][d], dW fp32 [V][d].  Supported: d and V multiples of
 * 8, d >= 64, V >= 256, P*T < 2^31.  Sequences: cu_seqlens (device int32[nseq+1]), or, when it is NULL,
 * nseq equal sequences of T / nseq tokens (nseq = 0 or 1: one sequence).
 * Ownership, asynchrony and errors are those of the attention calls: the caller owns
 * every buffer, the calls enqueue on `stream` and return at once, the workspace's
 * first word is the status word of the bounded in-kernel waits
 * (ttt_attn_device_status).
 * ------------------------------------------------------------------------------ */
typedef struct {
  int P;                         /* draft passes */
  int T;                         /* tokens, all sequences back to back */
  int d;                         /* hidden size */
  int V;                         /* vocabulary */
  const int32_t* cu_seqlens;     /* device int32[nseq+1], or NULL (see above) */
  int nseq;
  const uint8_t* loss_mask;      /* device uint8[T] over teacher positions; NULL: all counted */
  const float* pass_weight;      /* device float[P]: w_p; NULL: all 1 */
  const float* pass_count;       /* device float[P]: N_p (e.g. summed over ranks); NULL: counted here */
  int token_chunk_size;          /* backward: draft rows per chunk of dz; 0 selects 4096 */
  const ttt_attn_events* events; /* optional, indices TTT_SOFTCE_KERNEL_* */
  /* General form, for normalisation groups other than the passes (e.g. the slots of a
   * block drafter, issue 3698 item 3's per-slot normalisation).  When row_teacher is
   * non-NULL, draft row r (of P*T) learns teacher position row_teacher[r] and belongs to
   * normalisation group row_group[r] (NULL: every row in group 0); a row whose teacher
   * position lies outside [0, teacher_rows), whose group lies outside [0, ngroups) or
   * whose position is masked is invalid.  y then has teacher_rows rows, loss_mask
   * teacher_rows entries, pass_weight / pass_count ngroups entries, the loss ngroups + 1
   * values; cu_seqlens and nseq are not read. */
  const int32_t* row_teacher;    /* device int32[P*T], or NULL for the TTT passes */
  const int32_t* row_group;      /* device int32[P*T], or NULL */
  int ngroups;                   /* >= 1 with row_teacher; groups > 1 need row_group */
  int teacher_rows;              /* rows of y with row_teacher */
} ttt_softce_desc;

/* Kernel indices of the soft-CE calls in ttt_attn_events (the backward's chunked
 * kernels are timed at their first chunk). */
enum {
  TTT_SOFTCE_KERNEL_ROWS = 0,    /* teacher rows, pass counts (and coefficients) */
  TTT_SOFTCE_KERNEL_LOGITS = 1,  /* forward logits GEMM with the softmax statistics (fused: and the logits) */
  TTT_SOFTCE_KERNEL_REDUCE = 2,  /* merge of the statistics, per-pass sums (fused: the merge) */
  TTT_SOFTCE_KERNEL_DZ = 4,      /* backward: logits recomputed, dz (fused: dz from the stored logits) */
  TTT_SOFTCE_KERNEL_DH = 5,      /* dh = dz W */
  TTT_SOFTCE_KERNEL_DW = 6       /* dW += dz^T h */
};

/* Bytes of workspace for ttt_softce_fwd (for_backward = 0), ttt_softce_bwd (1) or
 * ttt_softce_fwd_bwd (2); 0 if the descriptor is invalid.  256-byte aligned.  Forward:
 * about 20 * P*T * ceil(V/256) bytes (the per-tile statistics); backward: about
 * 2 * chunk * V bytes (one chunk of dz); fused: both, plus 4 * chunk * V bytes (one chunk
 * of fp32 logits). */
size_t ttt_softce_workspace_size(const ttt_softce_desc* desc, int for_backward);

/* Forward.  Writes row_loss float[P*T] (l_r), lse float[2][P*T] (logsumexp of z_r,
 * then of the teacher row y_u; 0 for an invalid row; the backward reads it) and loss
 * float[G+1] (L_0 .. L_{G-1}, then L), G = P (or ngroups in the general form). */
ttt_status ttt_softce_fwd(const ttt_softce_desc* desc, const void* h, const void* W, const void* y,
                          float* row_loss, float* lse, float* loss, void* workspace, size_t workspace_bytes,
                          void* stream);

/* Backward of grad * L, given the forward's lse.  Writes dh; adds to dW unless dW is
 * NULL (then dW is not computed).  Visits the rows token_chunk_size at a time. */
ttt_status ttt_softce_bwd(const ttt_softce_desc* desc, const void* h, const void* W, const void* y,
                          const float* lse, float grad, void* dh, float* dW, void* workspace,
                          size_t workspace_bytes, void* stream);

/* Forward and backward in one sweep, for a caller that knows the loss's upstream gradient
 * `grad` before the forward (a loss's is usually 1).  Same outputs as ttt_softce_fwd
 * followed by ttt_softce_bwd with that grad, bit for bit.  Per chunk of token_chunk_size
 * rows it keeps the chunk's fp32 logits in the workspace and derives dz from them, so the
 * logits GEMM runs once instead of twice. */
ttt_status ttt_softce_fwd_bwd(const ttt_softce_desc* desc, const void* h, const void* W, const void* y, float grad,
                              float* row_loss, float* lse, float* loss, void* dh, float* dW, void* workspace,
                              size_t workspace_bytes, void* stream);

/* The error behind the most recent TTT_ERR_CUDA returned by any call in this
 * process: a cudaError_t value, or 100000 + the CUresult when encoding a TMA tensor
 * map failed; 0 if there was none.  Not reset by later successful calls. */
int ttt_attn_last_cuda_error(void);

/* Name of a code returned by ttt_attn_last_cuda_error (static string). */
const char* ttt_attn_cuda_error_name(int code);

/* Synchronises `stream` and returns TTT_OK if no bounded wait of the calls made
 * with this workspace ran out since the last check, TTT_ERR_DEVICE_TIMEOUT (and
 * the raw status word in *detail if non-NULL) otherwise, TTT_ERR_INVALID_ARG for an
 * argument error only the device could see (block-draft anchors out of order), or
 * TTT_ERR_CUDA.  The status word is cleared. */
ttt_status ttt_attn_device_status(void* workspace, void* stream, uint32_t* detail);

/* Workspace sub-buffers (byte offsets from the workspace base), for inspection of
 * the intermediate results by tests:
 *   fwd: [0] status word (bytes 0-3; bytes 4-7: the "dq~ accumulator zeroed" mark),
 *        [1] q~ bf16 [P][H][Tt][D], [2] k~ bf16 [P][Hkv][Tt][D];
 *   bwd: [0] status, [1] q~, [2] k~, [3] row statistics fp32: for query head (p, h)
 *        and the 64-row query tile j of sequence n, 128 floats at slot
 *        start_n/64 + n + j of row p*H + h (-lse * log2(e) of the 64 rows, then their
 *        delta = rowsum(dout * o)), T/64 + nseq + 1 slots per row,
 *        [4] dq~ accumulator fp32 [P][H][Tt][D], [5] int32 order tickets of the dq~
 *        additions, one per statistics slot.
 * Tt = B*S (dense) or T (packed).  Returns the number of entries written to
 * offsets (at most 8), or 0 for an invalid descriptor. */
int ttt_attn_workspace_layout(const ttt_attn_desc* desc, int for_backward, size_t* offsets);

/* Self-test of the bounded-wait machinery: launches one CTA that waits on an
 * mbarrier nothing will ever complete, with a limit of budget_ns nanoseconds.
 * The kernel gives up, records the timeout in the workspace status word and
 * exits; read it back with ttt_attn_device_status().  No other work is done. */
ttt_status ttt_attn_watchdog_selftest(void* workspace, size_t workspace_bytes, uint64_t budget_ns, void* stream);

/* Limit, in nanoseconds, for every in-kernel wait of later calls (default 2e9).
 * Process-wide setting. */
void ttt_attn_set_wait_budget_ns(uint64_t budget_ns);

const char* ttt_status_string(ttt_status status);

/* Library version, e.g. "0.3.0". */
const char* ttt_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TTT_ATTN_H_ */
