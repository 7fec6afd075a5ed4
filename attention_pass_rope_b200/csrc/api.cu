// C ABI of libttt_attn.so (declared in include/ttt_attn.h): argument validation,
// workspace layout, TMA descriptors and the launch sequence of the forward and
// backward passes on the caller's stream.  No allocation, no per-call state.
#include <atomic>
#include <cmath>
#include <cstring>

#include "../../include/ttt_attn.h"
#include "ttt_internal.h"

namespace ttt {
namespace {

std::atomic<uint64_t> g_wait_budget_ns{2000000000ull};

constexpr size_t kAlign = 1024;
inline size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct Plan {
  Geometry g;
  size_t off[8];
  int noff;
  size_t total;
};

bool ptr_aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Validate the descriptor and derive the geometry and workspace layout.
ttt_status make_plan(const ttt_attn_desc* d, int for_backward, Plan* out) {
  if (!d) return TTT_ERR_INVALID_ARG;
  Plan pl{};
  Geometry& g = pl.g;
  if (d->layout != TTT_LAYOUT_BSHD && d->layout != TTT_LAYOUT_THD) return TTT_ERR_INVALID_ARG;
  if (d->P < 1 || d->H < 1 || d->Hkv < 1 || d->D < 1) return TTT_ERR_INVALID_ARG;
  if (d->H % d->Hkv != 0) return TTT_ERR_INVALID_ARG;
  if (d->P > 16) return TTT_ERR_UNSUPPORTED;
  if (d->D != 64 && d->D != 128) return TTT_ERR_UNSUPPORTED;  // rotary needs an even D; kernels take 64/128
  if (!(d->rope_theta > 0.f) || !std::isfinite(d->rope_theta)) return TTT_ERR_INVALID_ARG;
  if (!(d->softmax_scale >= 0.f) || !std::isfinite(d->softmax_scale)) return TTT_ERR_INVALID_ARG;
  if (d->flags & ~static_cast<int>(TTT_FLAG_ROTATED_IN_WORKSPACE | TTT_FLAG_DETERMINISTIC_DQ))
    return TTT_ERR_INVALID_ARG;
  g.P = d->P;
  g.H = d->H;
  g.Hkv = d->Hkv;
  g.D = d->D;
  g.theta = d->rope_theta;
  g.scale = d->softmax_scale > 0.f ? d->softmax_scale : 1.0f / std::sqrt(static_cast<float>(d->D));
  if (d->layout == TTT_LAYOUT_BSHD) {
    if (d->B < 0 || d->S < 0) return TTT_ERR_INVALID_ARG;
    const long long T = static_cast<long long>(d->B) * d->S;
    if (T > (1LL << 30)) return TTT_ERR_UNSUPPORTED;
    g.si.cu_seqlens = nullptr;
    g.si.nseq = d->B;
    g.si.S = d->S;
    g.si.T = static_cast<int>(T);
    g.si.max_len = d->S;
  } else {
    if (d->nseq < 0 || d->total_tokens < 0 || d->max_seqlen < 0) return TTT_ERR_INVALID_ARG;
    if (d->total_tokens > 0 && (!d->cu_seqlens || d->nseq < 1 || d->max_seqlen < 1)) return TTT_ERR_INVALID_ARG;
    if (d->max_seqlen > d->total_tokens) return TTT_ERR_INVALID_ARG;
    if (d->total_tokens > (1 << 30)) return TTT_ERR_UNSUPPORTED;
    g.si.cu_seqlens = d->cu_seqlens;
    g.si.nseq = d->nseq;
    g.si.S = 0;
    g.si.T = d->total_tokens;
    g.si.max_len = d->max_seqlen;
  }
  g.si.mult = 1;
  g.ksi = g.si;  // queries and keys index the same tokens
  g.Bs = 0;
  g.anchors = nullptr;
  g.ring = 0;
  g.limit_off = 0;
  g.pos0 = 0;
  // index arithmetic in the kernels: P*H*T*D elements must fit comfortably in int64,
  // per-pass offsets in int32 where they are formed that way
  const long long rows = static_cast<long long>(g.P) * g.H * g.si.T;
  if (rows * g.D > (1LL << 40)) return TTT_ERR_UNSUPPORTED;
  // per-pass strides of the public tensors (0: packed); passes never overlap
  const int64_t packed_q = static_cast<int64_t>(g.si.T) * g.H * g.D;
  const int64_t packed_kv = static_cast<int64_t>(g.si.T) * g.Hkv * g.D;
  g.sq = packed_q;
  g.skv = packed_kv;
  if (g.P > 1) {
    if (d->pass_stride_q != 0) {
      if (d->pass_stride_q < packed_q || d->pass_stride_q % 8 != 0) return TTT_ERR_INVALID_ARG;
      g.sq = d->pass_stride_q;
    }
    if (d->pass_stride_kv != 0) {
      if (d->pass_stride_kv < packed_kv || d->pass_stride_kv % 8 != 0) return TTT_ERR_INVALID_ARG;
      g.skv = d->pass_stride_kv;
    }
    if (g.sq > (1LL << 44) / g.P || g.skv > (1LL << 44) / g.P) return TTT_ERR_UNSUPPORTED;
  }

  const size_t T = static_cast<size_t>(g.si.T);
  const size_t P = g.P, H = g.H, Hkv = g.Hkv, D = g.D;
  size_t o = 0;
  pl.off[0] = 0;
  o = align_up(256);
  pl.off[1] = o;  // q~
  o = align_up(o + P * H * T * D * 2);
  pl.off[2] = o;  // k~
  o = align_up(o + P * Hkv * T * D * 2);
  if (!for_backward) {
    pl.noff = 3;
  } else {
    pl.off[3] = o;  // tile-aligned row statistics (-lse*log2e, delta)
    o = align_up(o + P * H * static_cast<size_t>(ld_slots(g.si)) * 128 * 4);
    pl.off[4] = o;  // dq~ accumulator
    o = align_up(o + P * H * T * D * 4);
    pl.off[5] = o;  // order tickets of the dq~ additions, one per statistics slot
    o = align_up(o + P * H * static_cast<size_t>(ld_slots(g.si)) * 4);
    pl.noff = 6;
  }
  pl.total = o;
  *out = pl;
  return TTT_OK;
}

// Block-draft attention: validate, derive the two index spaces (block rows, context)
// and the workspace layout.
ttt_status make_block_plan(const ttt_block_desc* d, int for_backward, Plan* out) {
  if (!d) return TTT_ERR_INVALID_ARG;
  Plan pl{};
  Geometry& g = pl.g;
  if (d->layout != TTT_LAYOUT_BSHD && d->layout != TTT_LAYOUT_THD) return TTT_ERR_INVALID_ARG;
  if (d->H < 1 || d->Hkv < 1 || d->D < 1 || d->Bs < 1) return TTT_ERR_INVALID_ARG;
  if (d->H % d->Hkv != 0) return TTT_ERR_INVALID_ARG;
  if (d->Bs > 16) return TTT_ERR_UNSUPPORTED;
  if (d->window < 0) return TTT_ERR_INVALID_ARG;
  if (d->D != 64 && d->D != 128) return TTT_ERR_UNSUPPORTED;
  if (!(d->rope_theta > 0.f) || !std::isfinite(d->rope_theta)) return TTT_ERR_INVALID_ARG;
  if (!(d->softmax_scale >= 0.f) || !std::isfinite(d->softmax_scale)) return TTT_ERR_INVALID_ARG;
  if (d->flags & ~static_cast<int>(TTT_FLAG_ROTATED_IN_WORKSPACE | TTT_FLAG_DETERMINISTIC_DQ))
    return TTT_ERR_INVALID_ARG;
  g.P = 1;
  g.H = d->H;
  g.Hkv = d->Hkv;
  g.D = d->D;
  g.theta = d->rope_theta;
  g.scale = d->softmax_scale > 0.f ? d->softmax_scale : 1.0f / std::sqrt(static_cast<float>(d->D));
  g.Bs = d->Bs;
  g.anchors = d->anchors;
  g.window = d->window;
  g.ring = 0;
  g.limit_off = 0;
  g.pos0 = 0;
  if (d->layout == TTT_LAYOUT_BSHD) {
    if (d->B < 0 || d->S < 0 || d->nblk < 0) return TTT_ERR_INVALID_ARG;
    const long long Tc = static_cast<long long>(d->B) * d->S;
    const long long NQ = static_cast<long long>(d->B) * d->nblk * d->Bs;
    if (Tc > (1LL << 30) || NQ > (1LL << 30)) return TTT_ERR_UNSUPPORTED;
    if (d->nblk > 0 && d->S < 1) return TTT_ERR_INVALID_ARG;  // a block needs a context to anchor in
    g.ksi = SeqInfo{nullptr, d->B, d->S, static_cast<int>(Tc), d->S, 1};
    g.si = SeqInfo{nullptr, d->B, d->nblk * d->Bs, static_cast<int>(NQ), d->nblk * d->Bs, 1};
  } else {
    if (d->nseq < 0 || d->total_ctx < 0 || d->total_blocks < 0 || d->max_ctx < 0 || d->max_blocks < 0)
      return TTT_ERR_INVALID_ARG;
    if (d->total_blocks > 0 && (!d->cu_ctx || !d->cu_blocks || d->nseq < 1 || d->max_blocks < 1 || d->max_ctx < 1))
      return TTT_ERR_INVALID_ARG;
    if (d->max_ctx > d->total_ctx || d->max_blocks > d->total_blocks) return TTT_ERR_INVALID_ARG;
    const long long NQ = static_cast<long long>(d->total_blocks) * d->Bs;
    if (d->total_ctx > (1 << 30) || NQ > (1LL << 30)) return TTT_ERR_UNSUPPORTED;
    g.ksi = SeqInfo{d->cu_ctx, d->nseq, 0, d->total_ctx, d->max_ctx, 1};
    g.si = SeqInfo{d->cu_blocks, d->nseq, 0, static_cast<int>(NQ), d->max_blocks * d->Bs, d->Bs};
  }
  if (g.si.T > 0 && !g.anchors) return TTT_ERR_INVALID_ARG;
  g.sq = static_cast<int64_t>(g.si.T) * g.H * g.D;
  g.skv = static_cast<int64_t>(g.ksi.T) * g.Hkv * g.D;
  const size_t NQ = static_cast<size_t>(g.si.T), Tc = static_cast<size_t>(g.ksi.T);
  const size_t H = g.H, Hkv = g.Hkv, D = g.D;
  size_t o = 0;
  pl.off[0] = 0;
  o = align_up(256);
  pl.off[1] = o;  // q~ of the block tokens
  o = align_up(o + H * NQ * D * 2);
  pl.off[2] = o;  // k~ of the context
  o = align_up(o + Hkv * Tc * D * 2);
  pl.off[3] = o;  // k~ of the block tokens
  o = align_up(o + Hkv * NQ * D * 2);
  if (!for_backward) {
    pl.noff = 4;
  } else {
    pl.off[4] = o;  // row statistics over the block rows
    o = align_up(o + H * static_cast<size_t>(ld_slots(g.si)) * 128 * 4);
    pl.off[5] = o;  // dq~ accumulator
    o = align_up(o + H * NQ * D * 4);
    pl.off[6] = o;  // order tickets
    o = align_up(o + H * static_cast<size_t>(ld_slots(g.si)) * 4);
    pl.off[7] = o;  // trunk-key limit of every block row
    o = align_up(o + NQ * 4);
    pl.noff = 8;
  }
  pl.total = o;
  *out = pl;
  return TTT_OK;
}

// Ring step geometry: the local query chunk is one dense sequence of q_len rows (B = 1),
// the visiting keys another of kv_len rows.
ttt_status make_ring_geometry(const ttt_ring_desc* d, Geometry* out) {
  if (!d) return TTT_ERR_INVALID_ARG;
  if (d->P < 1 || d->H < 1 || d->Hkv < 1 || d->H % d->Hkv != 0) return TTT_ERR_INVALID_ARG;
  if (d->P > 16) return TTT_ERR_UNSUPPORTED;
  if (d->D != 64 && d->D != 128) return TTT_ERR_UNSUPPORTED;
  if (!(d->rope_theta > 0.f) || !std::isfinite(d->rope_theta)) return TTT_ERR_INVALID_ARG;
  if (!(d->softmax_scale >= 0.f) || !std::isfinite(d->softmax_scale)) return TTT_ERR_INVALID_ARG;
  if (d->q_len < 0 || d->kv_len < 0 || d->q_start < 0 || d->kv_start < 0) return TTT_ERR_INVALID_ARG;
  if (d->q_len > (1 << 28) || d->kv_len > (1 << 28)) return TTT_ERR_UNSUPPORTED;
  Geometry g{};
  g.P = d->P;
  g.H = d->H;
  g.Hkv = d->Hkv;
  g.D = d->D;
  g.theta = d->rope_theta;
  g.scale = d->softmax_scale > 0.f ? d->softmax_scale : 1.0f / std::sqrt(static_cast<float>(d->D));
  g.si = SeqInfo{nullptr, 1, d->q_len, d->q_len, d->q_len, 1};
  g.ksi = SeqInfo{nullptr, 1, d->kv_len, d->kv_len, d->kv_len, 1};
  g.sq = static_cast<int64_t>(d->q_len) * d->H * d->D;
  g.skv = static_cast<int64_t>(d->q_len) * d->Hkv * d->D;
  g.ring = d->include_branch ? 2 : 1;
  g.limit_off = d->q_start - d->kv_start;
  g.pos0 = d->q_start;
  *out = g;
  return TTT_OK;
}

// The error behind the most recent TTT_ERR_CUDA (cudaError_t, or kEncodeErrorBase +
// CUresult when a TMA descriptor could not be encoded).
std::atomic<int> g_last_cuda_error{0};
constexpr int kEncodeErrorBase = 100000;

// ---- TMA descriptors (driver entry point fetched through the runtime)
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// 3-D bf16 tensor map, 128-byte swizzle, box {64, b1, b2}; dims/strides innermost first.
bool make_map(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1_bytes,
              uint64_t s2_bytes, uint32_t b1, uint32_t b2) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) {
    g_last_cuda_error.store(static_cast<int>(cudaErrorSymbolNotFound));
    return false;
  }
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {s1_bytes, s2_bytes};
  const cuuint32_t box[3] = {64, b1, b2};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) g_last_cuda_error.store(kEncodeErrorBase + static_cast<int>(r));
  return r == CUDA_SUCCESS;
}

// 4-D bf16 tensor map, 128-byte swizzle, box {64, b1, b2, b3}; dims/strides innermost first.
bool make_map4(CUtensorMap* m, const void* base, const uint64_t (&dims)[4], const uint64_t (&strides_bytes)[3],
               const uint32_t (&box_outer)[3]) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) {
    g_last_cuda_error.store(static_cast<int>(cudaErrorSymbolNotFound));
    return false;
  }
  const cuuint64_t d4[4] = {dims[0], dims[1], dims[2], dims[3]};
  const cuuint64_t s3[3] = {strides_bytes[0], strides_bytes[1], strides_bytes[2]};
  const cuuint32_t box[4] = {64, box_outer[0], box_outer[1], box_outer[2]};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), d4, s3, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) g_last_cuda_error.store(kEncodeErrorBase + static_cast<int>(r));
  return r == CUDA_SUCCESS;
}

struct EventScope {
  const ttt_attn_events* ev;
  int k;
  cudaStream_t s;
  EventScope(const ttt_attn_events* e, int kk, cudaStream_t st) : ev(e), k(kk), s(st) {
    if (ev && ev->start[k]) cudaEventRecord(static_cast<cudaEvent_t>(ev->start[k]), s);
  }
  ~EventScope() {
    if (ev && ev->stop[k]) cudaEventRecord(static_cast<cudaEvent_t>(ev->stop[k]), s);
  }
};

#define TTT_CHECK_CUDA(expr)                                    \
  do {                                                          \
    const cudaError_t e_ = (expr);                              \
    if (e_ != cudaSuccess) {                                    \
      g_last_cuda_error.store(static_cast<int>(e_));           \
      return TTT_ERR_CUDA;                                      \
    }                                                           \
  } while (0)

// The launchers read a launch's error with cudaGetLastError(), which also returns a
// non-sticky status left on this host thread by the caller's own runtime calls
// (cudaErrorNotReady from an event or stream query, for example: autograd worker
// threads make such queries).  Each entry point clears it before its first CUDA
// call; a sticky error cannot be cleared and still fails the call.
inline void clear_stale_error() { (void)cudaGetLastError(); }

}  // namespace

bool encode_map_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t d0, uint64_t d1,
                   uint64_t s1_bytes, uint32_t b0, uint32_t b1, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) {
    g_last_cuda_error.store(static_cast<int>(cudaErrorSymbolNotFound));
    return false;
  }
  const cuuint64_t dims[2] = {d0, d1};
  const cuuint64_t strides[1] = {s1_bytes};
  const cuuint32_t box[2] = {b0, b1};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) g_last_cuda_error.store(kEncodeErrorBase + static_cast<int>(r));
  return r == CUDA_SUCCESS;
}

uint64_t wait_budget_ns() { return g_wait_budget_ns.load(); }

void record_cuda_error(int code) { g_last_cuda_error.store(code); }
}  // namespace ttt

using namespace ttt;

extern "C" {

size_t ttt_attn_workspace_size(const ttt_attn_desc* desc, int for_backward) {
  Plan pl;
  if (make_plan(desc, for_backward, &pl) != TTT_OK) return 0;
  return pl.total;
}

int ttt_attn_workspace_layout(const ttt_attn_desc* desc, int for_backward, size_t* offsets) {
  Plan pl;
  if (!offsets || make_plan(desc, for_backward, &pl) != TTT_OK) return 0;
  for (int i = 0; i < pl.noff; ++i) offsets[i] = pl.off[i];
  return pl.noff;
}

ttt_status ttt_attn_fwd(const ttt_attn_desc* desc, const void* q, const void* k, const void* v, void* o, float* lse,
                        void* workspace, size_t workspace_bytes, void* stream_) {
  Plan pl;
  ttt_status st = make_plan(desc, 0, &pl);
  if (st != TTT_OK) return st;
  const Geometry& g = pl.g;
  if (g.si.T == 0) return TTT_OK;
  if (!q || !k || !v || !o || !lse) return TTT_ERR_INVALID_ARG;
  if (!ptr_aligned(q, 16) || !ptr_aligned(k, 16) || !ptr_aligned(v, 16) || !ptr_aligned(o, 16) ||
      !ptr_aligned(lse, 4))
    return TTT_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < pl.total || !ptr_aligned(workspace, 256)) return TTT_ERR_WORKSPACE;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws + pl.off[0]);
  void* qr = ws + pl.off[1];
  void* kr = ws + pl.off[2];
  const uint64_t T = g.si.T, D = g.D;

  // The first runtime call also makes the current device's primary context current
  // on this thread, which the driver's tensor-map encoder needs (a thread that has
  // made no runtime call yet, such as an autograd worker, has none).
  clear_stale_error();
  TTT_CHECK_CUDA(cudaMemsetAsync(status, 0, sizeof(uint32_t), stream));
  CUtensorMap mq, mk, mv, mo, mek, mev;
  const uint64_t P = g.P, H = g.H, Hkv = g.Hkv;
  if (!make_map(&mq, qr, D, T, P * H, D * 2, T * D * 2, 128, 1) ||
      !make_map(&mk, kr, D, T, Hkv, D * 2, T * D * 2, 128, 1) ||
      !make_map(&mv, v, D, Hkv, T, D * 2, Hkv * D * 2, 1, 128) ||
      !make_map4(&mo, o, {D, H, T, P}, {D * 2, H * D * 2, static_cast<uint64_t>(g.sq) * 2}, {1, 32, 1}) ||
      !make_map(&mek, kr, D, T, P * Hkv, D * 2, T * D * 2, 128, 1) ||
      !make_map4(&mev, v, {D, Hkv, T, P}, {D * 2, Hkv * D * 2, static_cast<uint64_t>(g.skv) * 2}, {1, 128, 1}))
    return TTT_ERR_CUDA;
  {
    EventScope es(desc->events, TTT_KERNEL_ROPE_FWD, stream);
    TTT_CHECK_CUDA(launch_rope_fwd(g, q, k, qr, kr, stream));
  }
  {
    EventScope es(desc->events, TTT_KERNEL_TRUNK_FWD, stream);
    TrunkFwdArgs a{g, nullptr, kr, v, o, lse, status, g_wait_budget_ns.load()};
    // a workspace sized for the backward: its dq~ accumulator is zeroed here, by warps
    // that the attention leaves idle, instead of in the backward's preprocess
    Plan pb;
    const bool zero_dq = make_plan(desc, 1, &pb) == TTT_OK && workspace_bytes >= pb.total;
    if (zero_dq) {
      a.zero_base = reinterpret_cast<float4*>(ws + pb.off[4]);
      a.zero_n16 = static_cast<int64_t>(g.P) * g.H * static_cast<int64_t>(T) * static_cast<int64_t>(D) / 4;
    }
    a.dq_zeroed = reinterpret_cast<uint32_t*>(ws + kDqZeroedOffset);
    TTT_CHECK_CUDA(launch_trunk_fwd(a, mq, mk, mv, mo, mek, mev, stream));
  }
  return TTT_OK;
}

ttt_status ttt_attn_bwd(const ttt_attn_desc* desc, const void* q, const void* k, const void* v, const void* o,
                        const float* lse, const void* dout, void* dq, void* dk, void* dv, void* workspace,
                        size_t workspace_bytes, void* stream_) {
  Plan pl;
  ttt_status st = make_plan(desc, 1, &pl);
  if (st != TTT_OK) return st;
  const Geometry& g = pl.g;
  if (g.si.T == 0) return TTT_OK;
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return TTT_ERR_INVALID_ARG;
  if (!ptr_aligned(q, 16) || !ptr_aligned(k, 16) || !ptr_aligned(v, 16) || !ptr_aligned(o, 16) ||
      !ptr_aligned(dout, 16) || !ptr_aligned(dq, 16) || !ptr_aligned(dk, 16) || !ptr_aligned(dv, 16) ||
      !ptr_aligned(lse, 4))
    return TTT_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < pl.total || !ptr_aligned(workspace, 256)) return TTT_ERR_WORKSPACE;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws + pl.off[0]);
  void* qr = ws + pl.off[1];
  void* kr = ws + pl.off[2];
  float* ld = reinterpret_cast<float*>(ws + pl.off[3]);
  float* dq_acc = reinterpret_cast<float*>(ws + pl.off[4]);
  int* tickets = reinterpret_cast<int*>(ws + pl.off[5]);
  const bool deterministic = (desc->flags & TTT_FLAG_DETERMINISTIC_DQ) != 0;
  const uint64_t T = g.si.T, D = g.D;

  // first runtime call before the tensor-map encoder (see ttt_attn_fwd)
  clear_stale_error();
  TTT_CHECK_CUDA(cudaMemsetAsync(status, 0, sizeof(uint32_t), stream));
  CUtensorMap mq, mk, mv, mdo;
  if (!make_map(&mq, qr, D, T, static_cast<uint64_t>(g.P) * g.H, D * 2, T * D * 2, 64, 1) ||
      !make_map(&mk, kr, D, T, g.Hkv, D * 2, T * D * 2, 128, 1) ||
      !make_map(&mv, v, D, g.Hkv, T, D * 2, g.Hkv * D * 2, 1, 128) ||
      !make_map4(&mdo, dout, {D, static_cast<uint64_t>(g.H), T, static_cast<uint64_t>(g.P)},
                 {D * 2, g.H * D * 2, static_cast<uint64_t>(g.sq) * 2}, {1, 64, 1}))
    return TTT_ERR_CUDA;
  {
    // the events are recorded either way, so a timing caller sees ~0 when the
    // forward's rotated q~ / k~ are reused
    EventScope es(desc->events, TTT_KERNEL_ROPE_BWD, stream);
    if (!(desc->flags & TTT_FLAG_ROTATED_IN_WORKSPACE)) TTT_CHECK_CUDA(launch_rope_fwd(g, q, k, qr, kr, stream));
  }
  {
    EventScope es(desc->events, TTT_KERNEL_BWD_PREPROCESS, stream);
    // a workspace untouched since the forward may hold an already zeroed dq~ accumulator
    const uint32_t* dq_zeroed = (desc->flags & TTT_FLAG_ROTATED_IN_WORKSPACE)
                                    ? reinterpret_cast<const uint32_t*>(ws + kDqZeroedOffset)
                                    : nullptr;
    TTT_CHECK_CUDA(launch_bwd_preprocess(g, o, dout, lse, ld, dq_acc, tickets, nullptr, status, dq_zeroed, stream));
  }
  {
    EventScope es(desc->events, TTT_KERNEL_TRUNK_BWD, stream);
    TrunkBwdArgs a{g, ld, dq_acc, dk, dv, deterministic ? tickets : nullptr, nullptr, status, g_wait_budget_ns.load()};
    TTT_CHECK_CUDA(launch_trunk_bwd(a, mq, mk, mv, mdo, stream));
  }
  {
    EventScope es(desc->events, TTT_KERNEL_BRANCH_BWD, stream);
    TTT_CHECK_CUDA(launch_branch_bwd(g, qr, kr, v, dout, lse, ld, dq_acc, dq, dk, dv, stream));
  }
  // the accumulator now holds this call's sums
  TTT_CHECK_CUDA(cudaMemsetAsync(ws + kDqZeroedOffset, 0, sizeof(uint32_t), stream));
  return TTT_OK;
}

size_t ttt_block_workspace_size(const ttt_block_desc* desc, int for_backward) {
  Plan pl;
  if (make_block_plan(desc, for_backward, &pl) != TTT_OK) return 0;
  return pl.total;
}

int ttt_block_workspace_layout(const ttt_block_desc* desc, int for_backward, size_t* offsets) {
  Plan pl;
  if (!offsets || make_block_plan(desc, for_backward, &pl) != TTT_OK) return 0;
  for (int i = 0; i < pl.noff; ++i) offsets[i] = pl.off[i];
  return pl.noff;
}

ttt_status ttt_block_attn_fwd(const ttt_block_desc* desc, const void* k_ctx, const void* v_ctx, const void* qb,
                              const void* kb, const void* vb, void* o, float* lse, void* workspace,
                              size_t workspace_bytes, void* stream_) {
  Plan pl;
  ttt_status st = make_block_plan(desc, 0, &pl);
  if (st != TTT_OK) return st;
  const Geometry& g = pl.g;
  if (g.si.T == 0) return TTT_OK;
  if (!k_ctx || !v_ctx || !qb || !kb || !vb || !o || !lse) return TTT_ERR_INVALID_ARG;
  if (!ptr_aligned(k_ctx, 16) || !ptr_aligned(v_ctx, 16) || !ptr_aligned(qb, 16) || !ptr_aligned(kb, 16) ||
      !ptr_aligned(vb, 16) || !ptr_aligned(o, 16) || !ptr_aligned(lse, 4))
    return TTT_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < pl.total || !ptr_aligned(workspace, 256)) return TTT_ERR_WORKSPACE;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws + pl.off[0]);
  void* qr = ws + pl.off[1];
  void* kr_ctx = ws + pl.off[2];
  void* kr_blk = ws + pl.off[3];
  const uint64_t NQ = g.si.T, Tc = g.ksi.T, D = g.D;
  clear_stale_error();
  TTT_CHECK_CUDA(cudaMemsetAsync(status, 0, sizeof(uint32_t), stream));
  CUtensorMap mq, mk, mv, mo, mek, mev;
  const uint64_t H = g.H, Hkv = g.Hkv;
  if (!make_map(&mq, qr, D, NQ, H, D * 2, NQ * D * 2, 128, 1) ||
      !make_map(&mk, kr_ctx, D, Tc, Hkv, D * 2, Tc * D * 2, 128, 1) ||
      !make_map(&mv, v_ctx, D, Hkv, Tc, D * 2, Hkv * D * 2, 1, 128) ||
      !make_map4(&mo, o, {D, H, NQ, 1}, {D * 2, H * D * 2, NQ * H * D * 2}, {1, 32, 1}) ||
      !make_map(&mek, kr_blk, D, NQ, Hkv, D * 2, NQ * D * 2, 128, 1) ||
      !make_map4(&mev, vb, {D, Hkv, NQ, 1}, {D * 2, Hkv * D * 2, NQ * Hkv * D * 2}, {1, 128, 1}))
    return TTT_ERR_CUDA;
  {
    EventScope es(desc->events, TTT_KERNEL_ROPE_FWD, stream);
    TTT_CHECK_CUDA(launch_rope_rows(g, false, g.ksi.T, k_ctx, g.Hkv, kr_ctx, nullptr, 0, nullptr, stream));
    TTT_CHECK_CUDA(launch_rope_rows(g, true, g.si.T, qb, g.H, qr, kb, g.Hkv, kr_blk, stream));
  }
  {
    EventScope es(desc->events, TTT_KERNEL_TRUNK_FWD, stream);
    TrunkFwdArgs a{g, nullptr, kr_blk, vb, o, lse, status, g_wait_budget_ns.load()};
    TTT_CHECK_CUDA(launch_trunk_fwd(a, mq, mk, mv, mo, mek, mev, stream));
  }
  return TTT_OK;
}

ttt_status ttt_block_attn_bwd(const ttt_block_desc* desc, const void* k_ctx, const void* v_ctx, const void* qb,
                              const void* kb, const void* vb, const void* o, const float* lse, const void* dout,
                              void* dk_ctx, void* dv_ctx, void* dqb, void* dkb, void* dvb, void* workspace,
                              size_t workspace_bytes, void* stream_) {
  Plan pl;
  ttt_status st = make_block_plan(desc, 1, &pl);
  if (st != TTT_OK) return st;
  const Geometry& g = pl.g;
  if (g.si.T == 0 && g.ksi.T == 0) return TTT_OK;
  if (!k_ctx || !v_ctx || !o || !lse || !dout || !dk_ctx || !dv_ctx) return TTT_ERR_INVALID_ARG;
  if (g.si.T > 0 && (!qb || !kb || !vb || !dqb || !dkb || !dvb)) return TTT_ERR_INVALID_ARG;
  const void* ptrs[] = {k_ctx, v_ctx, qb, kb, vb, o, dout, dk_ctx, dv_ctx, dqb, dkb, dvb};
  for (const void* p : ptrs)
    if (!ptr_aligned(p, 16)) return TTT_ERR_INVALID_ARG;
  if (!ptr_aligned(lse, 4)) return TTT_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < pl.total || !ptr_aligned(workspace, 256)) return TTT_ERR_WORKSPACE;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws + pl.off[0]);
  void* qr = ws + pl.off[1];
  void* kr_ctx = ws + pl.off[2];
  void* kr_blk = ws + pl.off[3];
  float* ld = reinterpret_cast<float*>(ws + pl.off[4]);
  float* dq_acc = reinterpret_cast<float*>(ws + pl.off[5]);
  int* tickets = reinterpret_cast<int*>(ws + pl.off[6]);
  int* qlim = reinterpret_cast<int*>(ws + pl.off[7]);
  const bool deterministic = (desc->flags & TTT_FLAG_DETERMINISTIC_DQ) != 0;
  const uint64_t NQ = g.si.T, Tc = g.ksi.T, D = g.D;
  clear_stale_error();
  TTT_CHECK_CUDA(cudaMemsetAsync(status, 0, sizeof(uint32_t), stream));
  if (g.si.T == 0) {
    // no block: no context key is seen
    TTT_CHECK_CUDA(cudaMemsetAsync(dk_ctx, 0, Tc * g.Hkv * D * 2, stream));
    TTT_CHECK_CUDA(cudaMemsetAsync(dv_ctx, 0, Tc * g.Hkv * D * 2, stream));
    return TTT_OK;
  }
  CUtensorMap mq, mk, mv, mdo;
  if (!make_map(&mq, qr, D, NQ, g.H, D * 2, NQ * D * 2, 64, 1) ||
      !make_map(&mk, kr_ctx, D, Tc, g.Hkv, D * 2, Tc * D * 2, 128, 1) ||
      !make_map(&mv, v_ctx, D, g.Hkv, Tc, D * 2, g.Hkv * D * 2, 1, 128) ||
      !make_map4(&mdo, dout, {D, static_cast<uint64_t>(g.H), NQ, 1}, {D * 2, g.H * D * 2, NQ * g.H * D * 2},
                 {1, 64, 1}))
    return TTT_ERR_CUDA;
  {
    EventScope es(desc->events, TTT_KERNEL_ROPE_BWD, stream);
    if (!(desc->flags & TTT_FLAG_ROTATED_IN_WORKSPACE)) {
      TTT_CHECK_CUDA(launch_rope_rows(g, false, g.ksi.T, k_ctx, g.Hkv, kr_ctx, nullptr, 0, nullptr, stream));
      TTT_CHECK_CUDA(launch_rope_rows(g, true, g.si.T, qb, g.H, qr, kb, g.Hkv, kr_blk, stream));
    }
  }
  {
    EventScope es(desc->events, TTT_KERNEL_BWD_PREPROCESS, stream);
    TTT_CHECK_CUDA(launch_bwd_preprocess(g, o, dout, lse, ld, dq_acc, tickets, qlim, status, nullptr, stream));
  }
  {
    EventScope es(desc->events, TTT_KERNEL_TRUNK_BWD, stream);
    TrunkBwdArgs a{g, ld, dq_acc, dk_ctx, dv_ctx, deterministic ? tickets : nullptr, qlim, status,
                   g_wait_budget_ns.load()};
    TTT_CHECK_CUDA(launch_trunk_bwd(a, mq, mk, mv, mdo, stream));
  }
  {
    EventScope es(desc->events, TTT_KERNEL_BRANCH_BWD, stream);
    TTT_CHECK_CUDA(launch_block_bwd(g, qr, kr_blk, vb, dout, lse, ld, dq_acc, dqb, dkb, dvb, stream));
  }
  return TTT_OK;
}

ttt_status ttt_ring_rotate(const ttt_ring_desc* desc, const void* q, const void* k, void* qr, void* kr,
                           void* stream_) {
  Geometry g;
  const ttt_status st = make_ring_geometry(desc, &g);
  if (st != TTT_OK) return st;
  if (desc->q_len == 0) return TTT_OK;
  if (!q || !k || !qr || !kr) return TTT_ERR_INVALID_ARG;
  if (!ptr_aligned(q, 16) || !ptr_aligned(k, 16) || !ptr_aligned(qr, 16) || !ptr_aligned(kr, 16))
    return TTT_ERR_INVALID_ARG;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  clear_stale_error();
  TTT_CHECK_CUDA(launch_rope_fwd(g, q, k, qr, kr, stream));
  return TTT_OK;
}

ttt_status ttt_ring_step(const ttt_ring_desc* desc, const void* qr, const void* kr_local, const void* v_local,
                         const void* kr_visit, const void* v_visit, float* o_part, float* lse_part, void* status,
                         void* stream_) {
  Geometry g;
  const ttt_status st = make_ring_geometry(desc, &g);
  if (st != TTT_OK) return st;
  if (desc->q_len == 0) return TTT_OK;
  if (desc->kv_start > desc->q_start || desc->kv_len == 0) return TTT_ERR_INVALID_ARG;  // no visible key
  if (!qr || !kr_visit || !v_visit || !o_part || !lse_part || !status) return TTT_ERR_INVALID_ARG;
  if (desc->include_branch && desc->P > 1 && (!kr_local || !v_local)) return TTT_ERR_INVALID_ARG;
  if (!ptr_aligned(qr, 16) || !ptr_aligned(kr_visit, 16) || !ptr_aligned(v_visit, 16) || !ptr_aligned(o_part, 16) ||
      !ptr_aligned(lse_part, 4) || !ptr_aligned(status, 4) || (kr_local && !ptr_aligned(kr_local, 16)) ||
      (v_local && !ptr_aligned(v_local, 16)))
    return TTT_ERR_INVALID_ARG;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  const uint64_t Lq = desc->q_len, Lk = desc->kv_len, D = g.D;
  clear_stale_error();
  CUtensorMap mq, mk, mv, mek, mev;
  const uint64_t P = g.P, Hkv = g.Hkv;
  if (!make_map(&mq, qr, D, Lq, P * g.H, D * 2, Lq * D * 2, 128, 1) ||
      !make_map(&mk, kr_visit, D, Lk, Hkv, D * 2, Lk * D * 2, 128, 1) ||
      !make_map(&mv, v_visit, D, Hkv, Lk, D * 2, Hkv * D * 2, 1, 128))
    return TTT_ERR_CUDA;
  // the branch keys' tiles (this chunk's own passes 2..P); without them the maps are
  // never used and stand in as copies of the query map
  mek = mq;
  mev = mq;
  if (g.ring == 2 && g.P > 1 &&
      (!make_map(&mek, kr_local, D, Lq, P * Hkv, D * 2, Lq * D * 2, 128, 1) ||
       !make_map4(&mev, v_local, {D, Hkv, Lq, P}, {D * 2, Hkv * D * 2, static_cast<uint64_t>(g.skv) * 2},
                  {1, 128, 1})))
    return TTT_ERR_CUDA;
  TrunkFwdArgs a{g, o_part, kr_local, v_local, nullptr, lse_part, static_cast<uint32_t*>(status),
                 g_wait_budget_ns.load()};
  // fp32 partial output: the bf16 output map is not used
  TTT_CHECK_CUDA(launch_trunk_fwd(a, mq, mk, mv, mq, mek, mev, stream));
  return TTT_OK;
}

ttt_status ttt_ring_merge(const ttt_ring_desc* desc, float* o_acc, float* lse_acc, const float* o_part,
                          const float* lse_part, int first, void* stream_) {
  Geometry g;
  const ttt_status st = make_ring_geometry(desc, &g);
  if (st != TTT_OK) return st;
  if (desc->q_len == 0) return TTT_OK;
  if (!o_acc || !lse_acc || !o_part || !lse_part || !ptr_aligned(o_acc, 16) || !ptr_aligned(o_part, 16))
    return TTT_ERR_INVALID_ARG;
  const long long rows = static_cast<long long>(g.P) * desc->q_len * g.H;
  if (rows > 0x7FFFFFFFLL) return TTT_ERR_UNSUPPORTED;
  clear_stale_error();
  TTT_CHECK_CUDA(launch_ring_merge(static_cast<int>(rows), g.D, g.H, desc->q_len, o_acc, lse_acc, o_part, lse_part,
                                   first != 0, static_cast<cudaStream_t>(stream_)));
  return TTT_OK;
}

ttt_status ttt_ring_finish(const ttt_ring_desc* desc, const float* o_acc, void* o, void* stream_) {
  Geometry g;
  const ttt_status st = make_ring_geometry(desc, &g);
  if (st != TTT_OK) return st;
  if (desc->q_len == 0) return TTT_OK;
  if (!o_acc || !o || !ptr_aligned(o_acc, 16) || !ptr_aligned(o, 16)) return TTT_ERR_INVALID_ARG;
  clear_stale_error();
  TTT_CHECK_CUDA(launch_ring_finish(static_cast<int64_t>(g.P) * desc->q_len * g.H * g.D, o_acc, o,
                                    static_cast<cudaStream_t>(stream_)));
  return TTT_OK;
}

// ---- ring backward
namespace {
struct RingBwdPlan {
  size_t off[4];  // status, row statistics, dq~ accumulator, order tickets
  size_t total;
};
RingBwdPlan ring_bwd_plan(const Geometry& g) {
  RingBwdPlan pl{};
  const size_t T = static_cast<size_t>(g.si.T), P = g.P, H = g.H, D = g.D;
  const size_t slots = static_cast<size_t>(ld_slots(g.si));
  size_t o = 0;
  pl.off[0] = 0;
  o = align_up(256);
  pl.off[1] = o;
  o = align_up(o + P * H * slots * 128 * 4);
  pl.off[2] = o;
  o = align_up(o + P * H * T * D * 4);
  pl.off[3] = o;
  o = align_up(o + P * H * slots * 4);
  pl.total = o;
  return pl;
}
}  // namespace

size_t ttt_ring_bwd_workspace_size(const ttt_ring_desc* desc) {
  Geometry g;
  if (make_ring_geometry(desc, &g) != TTT_OK) return 0;
  return ring_bwd_plan(g).total;
}

ttt_status ttt_ring_bwd_prepare(const ttt_ring_desc* desc, const void* o, const float* lse, const void* dout,
                                void* workspace, size_t workspace_bytes, void* stream_) {
  Geometry g;
  const ttt_status st = make_ring_geometry(desc, &g);
  if (st != TTT_OK) return st;
  if (desc->q_len == 0) return TTT_OK;
  const RingBwdPlan pl = ring_bwd_plan(g);
  if (!o || !lse || !dout || !ptr_aligned(o, 16) || !ptr_aligned(dout, 16) || !ptr_aligned(lse, 4))
    return TTT_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < pl.total || !ptr_aligned(workspace, 256)) return TTT_ERR_WORKSPACE;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  clear_stale_error();
  TTT_CHECK_CUDA(cudaMemsetAsync(ws, 0, sizeof(uint32_t), stream));
  TTT_CHECK_CUDA(launch_bwd_preprocess(g, o, dout, lse, reinterpret_cast<float*>(ws + pl.off[1]),
                                       reinterpret_cast<float*>(ws + pl.off[2]), reinterpret_cast<int*>(ws + pl.off[3]),
                                       nullptr, reinterpret_cast<uint32_t*>(ws), nullptr, stream));
  return TTT_OK;
}

ttt_status ttt_ring_bwd_step(const ttt_ring_desc* desc, const void* qr, const void* dout, const void* kr_visit,
                             const void* v_visit, float* dk_acc, float* dv_acc, void* workspace, size_t workspace_bytes,
                             void* stream_) {
  Geometry g;
  const ttt_status st = make_ring_geometry(desc, &g);
  if (st != TTT_OK) return st;
  if (desc->q_len == 0 || desc->kv_len == 0) return TTT_OK;
  if (desc->kv_start > desc->q_start) return TTT_ERR_INVALID_ARG;  // no visible key
  const RingBwdPlan pl = ring_bwd_plan(g);
  if (!qr || !dout || !kr_visit || !v_visit || !dk_acc || !dv_acc) return TTT_ERR_INVALID_ARG;
  if (!ptr_aligned(qr, 16) || !ptr_aligned(dout, 16) || !ptr_aligned(kr_visit, 16) || !ptr_aligned(v_visit, 16) ||
      !ptr_aligned(dk_acc, 16) || !ptr_aligned(dv_acc, 16))
    return TTT_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < pl.total || !ptr_aligned(workspace, 256)) return TTT_ERR_WORKSPACE;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const uint64_t Lq = desc->q_len, Lk = desc->kv_len, D = g.D, P = g.P, H = g.H, Hkv = g.Hkv;
  clear_stale_error();
  CUtensorMap mq, mk, mv, mdo;
  if (!make_map(&mq, qr, D, Lq, P * H, D * 2, Lq * D * 2, 64, 1) ||
      !make_map(&mk, kr_visit, D, Lk, Hkv, D * 2, Lk * D * 2, 128, 1) ||
      !make_map(&mv, v_visit, D, Hkv, Lk, D * 2, Hkv * D * 2, 1, 128) ||
      !make_map4(&mdo, dout, {D, H, Lq, P}, {D * 2, H * D * 2, static_cast<uint64_t>(g.sq) * 2}, {1, 64, 1}))
    return TTT_ERR_CUDA;
  TrunkBwdArgs a{g, reinterpret_cast<const float*>(ws + pl.off[1]), reinterpret_cast<float*>(ws + pl.off[2]),
                 nullptr, nullptr, nullptr, nullptr, reinterpret_cast<uint32_t*>(ws), g_wait_budget_ns.load(),
                 dk_acc, dv_acc};
  TTT_CHECK_CUDA(launch_trunk_bwd(a, mq, mk, mv, mdo, stream));
  return TTT_OK;
}

ttt_status ttt_ring_bwd_finish(const ttt_ring_desc* desc, const void* qr, const void* kr_local, const void* v_local,
                               const void* dout, const float* lse, void* dq, void* dk, void* dv, void* workspace,
                               size_t workspace_bytes, void* stream_) {
  Geometry g;
  const ttt_status st = make_ring_geometry(desc, &g);
  if (st != TTT_OK) return st;
  if (desc->q_len == 0) return TTT_OK;
  const RingBwdPlan pl = ring_bwd_plan(g);
  if (!qr || !kr_local || !v_local || !dout || !lse || !dq || !dk || !dv) return TTT_ERR_INVALID_ARG;
  for (const void* p : {qr, kr_local, v_local, dout, static_cast<const void*>(dq), static_cast<const void*>(dk),
                        static_cast<const void*>(dv)})
    if (!ptr_aligned(p, 16)) return TTT_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < pl.total || !ptr_aligned(workspace, 256)) return TTT_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  clear_stale_error();
  TTT_CHECK_CUDA(launch_branch_bwd(g, qr, kr_local, v_local, dout, lse, reinterpret_cast<const float*>(ws + pl.off[1]),
                                   reinterpret_cast<const float*>(ws + pl.off[2]), dq, dk, dv,
                                   static_cast<cudaStream_t>(stream_)));
  return TTT_OK;
}

ttt_status ttt_ring_dkv_finish(const ttt_ring_desc* desc, const float* dk_acc, const float* dv_acc, void* dk,
                               void* dv, void* stream_) {
  Geometry g;
  const ttt_status st = make_ring_geometry(desc, &g);
  if (st != TTT_OK) return st;
  if (desc->q_len == 0) return TTT_OK;
  if (!dk_acc || !dv_acc || !dk || !dv || !ptr_aligned(dk, 16) || !ptr_aligned(dv, 16)) return TTT_ERR_INVALID_ARG;
  clear_stale_error();
  TTT_CHECK_CUDA(launch_ring_dkv_finish(g, desc->q_len, dk_acc, dv_acc, dk, dv, static_cast<cudaStream_t>(stream_)));
  return TTT_OK;
}

ttt_status ttt_attn_device_status(void* workspace, void* stream_, uint32_t* detail) {
  if (!workspace) return TTT_ERR_WORKSPACE;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  uint32_t word = 0;
  if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
      cudaStreamSynchronize(stream) != cudaSuccess)
    return TTT_ERR_CUDA;
  if (detail) *detail = word;
  if (word == 0) return TTT_OK;
  if (cudaMemsetAsync(workspace, 0, sizeof(uint32_t), stream) != cudaSuccess ||
      cudaStreamSynchronize(stream) != cudaSuccess)
    return TTT_ERR_CUDA;
  return word == kStatusBadAnchors ? TTT_ERR_INVALID_ARG : TTT_ERR_DEVICE_TIMEOUT;
}

ttt_status ttt_attn_watchdog_selftest(void* workspace, size_t workspace_bytes, uint64_t budget_ns, void* stream_) {
  if (!workspace || workspace_bytes < 256 || !ptr_aligned(workspace, 256)) return TTT_ERR_WORKSPACE;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  uint32_t* status = static_cast<uint32_t*>(workspace);
  clear_stale_error();
  TTT_CHECK_CUDA(cudaMemsetAsync(status, 0, sizeof(uint32_t), stream));
  TTT_CHECK_CUDA(launch_watchdog_selftest(status, budget_ns, stream));
  return TTT_OK;
}

void ttt_attn_set_wait_budget_ns(uint64_t budget_ns) {
  g_wait_budget_ns.store(budget_ns == 0 ? 1 : budget_ns);
}

const char* ttt_status_string(ttt_status s) {
  switch (s) {
    case TTT_OK: return "ok";
    case TTT_ERR_INVALID_ARG: return "invalid argument";
    case TTT_ERR_UNSUPPORTED: return "unsupported configuration";
    case TTT_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
    case TTT_ERR_CUDA: return "CUDA error";
    case TTT_ERR_DEVICE_TIMEOUT: return "bounded in-kernel wait ran out";
  }
  return "unknown status";
}

const char* ttt_attn_version(void) { return "0.3.0"; }

int ttt_attn_last_cuda_error(void) { return g_last_cuda_error.load(); }

const char* ttt_attn_cuda_error_name(int code) {
  if (code >= kEncodeErrorBase) return "tensor map encoding failed (CUresult = code - 100000)";
  return cudaGetErrorName(static_cast<cudaError_t>(code));
}

}  // extern "C"
