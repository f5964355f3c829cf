// C ABI of libbsa (declared in include/bsa.h): argument validation, workspace
// layout, TMA tensor maps and the sequence of launches for each call.  Every
// argument error is returned before anything is launched; the library
// allocates no device memory and synchronises only in bsa_get_device_status.
// It owns one non-blocking side stream per device (created on first use), on
// which the planner runs beside the fixed-m bound.
#include <atomic>
#include <cmath>
#include <cstring>
#include <algorithm>
#include <mutex>
#include <vector>

#include "internal.h"

namespace bsa {

namespace {
std::atomic<uint64_t> g_launches{0};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int64_t cdiv64(int64_t a, int64_t b) { return (a + b - 1) / b; }
}  // namespace

void count_launch(int n) { g_launches.fetch_add(static_cast<uint64_t>(n)); }

// No batch entries or no query rows: every check on the shape, mask and
// options still applies, then the call does nothing.
bool problem_is_empty(const bsa_problem *prob) {
  return prob != nullptr && (prob->B == 0 || prob->Sq == 0);
}

WsLayout compute_layout(const bsa_problem &p) {
  WsLayout L{};
  const int64_t B = p.B, H = p.H;
  L.nM = static_cast<int>(cdiv64(p.Sq, kTile));
  L.nN = static_cast<int>(cdiv64(p.Skv, kTile));
  const int64_t nM = L.nM, nN = L.nN;
  L.nnz_cap = B * nM * nN;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  L.status = take(kHdrWords * 4);
  L.tile_class = take(static_cast<size_t>(B * nM * nN));
  L.rank = take(4 * static_cast<size_t>(B * nM * nN));
  L.row_cnt = take(4 * static_cast<size_t>(B * nM));
  L.row_ptr = take(4 * static_cast<size_t>(B * nM + 1));
  L.row_ent = take(4 * static_cast<size_t>(L.nnz_cap));
  L.col_cnt = take(4 * static_cast<size_t>(B * nN));
  L.col_ptr = take(4 * static_cast<size_t>(B * nN + 1));
  L.col_ent = take(4 * static_cast<size_t>(L.nnz_cap));
  L.col_rank = take(4 * static_cast<size_t>(L.nnz_cap));
  L.perm = take(4 * static_cast<size_t>(nN));
  L.seg_q = take(4 * static_cast<size_t>(p.Sq));
  L.seg_kv = take(4 * static_cast<size_t>(p.Skv));
  L.qblk = take(16 * static_cast<size_t>(B * nM));
  L.kblk = take(16 * static_cast<size_t>(B * nN));
  // kmax, qmax, then the bound kernel's finished-block counter, adjacent
  L.kmax = take(8 * static_cast<size_t>(B * H) + 4);
  L.qmax = L.kmax + 4 * static_cast<size_t>(B * H);
  L.gate = take(4 * static_cast<size_t>(B * H));
  L.qnorm = take(4 * static_cast<size_t>(B * H * p.Sq));
  L.kbar = take(4 * static_cast<size_t>(B * H * p.D));
  L.ksum = take(8 * static_cast<size_t>(B * H * p.D));
  L.kcount = take(4 * static_cast<size_t>(B));
  L.qdot = take(4 * static_cast<size_t>(B * H * p.Sq));
  L.kbmax = take(4 * static_cast<size_t>(B * p.H_kv * nN));
  L.kmax_q = take(4 * static_cast<size_t>(B * H * nM));
  L.fwd_end = off;
  L.delta = take(4 * static_cast<size_t>(B * H * nM * kTile));
  L.dq_accum = take(4 * static_cast<size_t>(B * H * nM * kTile * p.D));
  L.sem = take(4 * 4 * static_cast<size_t>(B * H * nM));  // one per 32-row quarter of a q-block
  L.o_resid = take(static_cast<size_t>(B * H * p.Sq * p.D));  // one byte per element
  L.q16 = take(2 * static_cast<size_t>(B * H * p.Sq * p.D));
  L.do16 = take(2 * static_cast<size_t>(B * H * p.Sq * p.D));
  L.total = off;
  return L;
}

namespace {

// cuTensorMapEncodeTiled, fetched through the runtime so that the library
// needs no link-time dependency on libcuda.
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// 4-D map over a 16-bit [B, S, H, D] tensor (bf16, or fp16 for the backward's
// converted copies): dims (D, S, H, B), 64 x 128 boxes, 128-byte swizzle.
// Out-of-range rows read as zero.
bool make_map(CUtensorMap *map, const void *ptr, int B, int S, int H, int D,
              const int64_t *stride, bool fp16 = false) {
  auto enc = get_encode();
  if (enc == nullptr) return false;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(S),
                              static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(stride[1]) * 2,
                                 static_cast<cuuint64_t>(stride[2]) * 2,
                                 static_cast<cuuint64_t>(stride[0]) * 2};
  const cuuint32_t box[4] = {64, static_cast<cuuint32_t>(kTile), 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(map, fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                         const_cast<void *>(ptr), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The backward's tensor maps: Q and dO from the fp16 copies the Delta pass
// writes into the workspace (contiguous [B, Sq, H, D]), K and V from the
// caller's bf16 tensors (converted per kv column inside the kernel).
bool bwd_maps(const bsa_problem &p, const WsLayout &L, uint8_t *ws, const void *k, const void *v,
              CUtensorMap *tq, CUtensorMap *tk, CUtensorMap *tv, CUtensorMap *tdo) {
  const int64_t cs[3] = {static_cast<int64_t>(std::max(p.Sq, 1)) * p.H * p.D,
                         static_cast<int64_t>(p.H) * p.D, p.D};
  return make_map(tq, ws + L.q16, p.B, p.Sq, p.H, p.D, cs, true) &&
         make_map(tk, k, p.B, p.Skv, p.H_kv, p.D, p.k_stride) &&
         make_map(tv, v, p.B, p.Skv, p.H_kv, p.D, p.v_stride) &&
         make_map(tdo, ws + L.do16, p.B, p.Sq, p.H, p.D, cs, true);
}

// Resolve defaults (contiguous strides, scale) into a private copy.
bsa_status normalise(const bsa_problem *in, bsa_problem *out) {
  if (in == nullptr) return BSA_ERR_INVALID_ARG;
  *out = *in;
  bsa_problem &p = *out;
  if (p.B < 0 || p.H < 1 || p.Sq < 0 || p.Skv < 1) return BSA_ERR_INVALID_ARG;
  if (p.H_kv == 0) p.H_kv = p.H;
  if (p.H_kv < 1 || p.H % p.H_kv != 0) return BSA_ERR_INVALID_ARG;
  if (p.D != 64 && p.D != 128) return BSA_ERR_UNSUPPORTED;
  if (p.Sq > kMaxSeq || p.Skv > kMaxSeq) return BSA_ERR_UNSUPPORTED;
  const int64_t nM = cdiv64(p.Sq, kTile), nN = cdiv64(p.Skv, kTile);
  if (static_cast<int64_t>(p.B) * nM * nN >= (int64_t{1} << 30)) return BSA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(p.B) * p.H * nM >= (int64_t{1} << 31)) return BSA_ERR_UNSUPPORTED;
  auto fix = [&](int64_t *s, int64_t S, int64_t heads) -> bsa_status {
    if (s[0] == 0 && s[1] == 0 && s[2] == 0) {
      s[0] = std::max<int64_t>(S, 1) * heads * p.D;
      s[1] = heads * p.D;
      s[2] = p.D;
    }
    for (int i = 0; i < 3; ++i) {
      if (s[i] <= 0) return BSA_ERR_INVALID_ARG;
      if (s[i] % 8 != 0) return BSA_ERR_UNSUPPORTED;  // 16-byte aligned rows for TMA
    }
    return BSA_OK;
  };
  bsa_status st;
  if ((st = fix(p.q_stride, p.Sq, p.H)) != BSA_OK) return st;
  if ((st = fix(p.k_stride, p.Skv, p.H_kv)) != BSA_OK) return st;
  if ((st = fix(p.v_stride, p.Skv, p.H_kv)) != BSA_OK) return st;
  if ((st = fix(p.o_stride, p.Sq, p.H)) != BSA_OK) return st;
  if (!(p.scale > 0.f) || !std::isfinite(p.scale)) p.scale = 1.0f / std::sqrt(static_cast<float>(p.D));
  return BSA_OK;
}

bsa_status check_mask(const bsa_problem &p, const bsa_mask_spec *m, bsa_mask_spec *out) {
  std::memset(out, 0, sizeof(*out));
  out->dilation = 1;
  if (m == nullptr) return BSA_OK;
  *out = *m;
  const uint32_t known = BSA_MASK_SEGMENT_IDS | BSA_MASK_KV_VALID_LEN | BSA_MASK_VARLEN |
                         BSA_MASK_CAUSAL_WINDOW | BSA_MASK_PREFIX_LM;
  if (m->flags & ~known) return BSA_ERR_INVALID_ARG;
  const bool win = (m->flags & BSA_MASK_CAUSAL_WINDOW) != 0;
  // an empty problem's predicate arrays have no element, so may be null
  const bool need = !problem_is_empty(&p);
  if ((m->flags & BSA_MASK_PREFIX_LM) && (!win || (need && m->prefix_len == nullptr)))
    return BSA_ERR_INVALID_ARG;
  if (m->dilation < 0 || (m->dilation > 1 && !win)) return BSA_ERR_INVALID_ARG;
  out->dilation = m->dilation > 1 ? m->dilation : 1;
  out->reserved = 0;
  if (!(m->flags & BSA_MASK_PREFIX_LM)) out->prefix_len = nullptr;
  if ((m->flags & BSA_MASK_SEGMENT_IDS) && need && (m->seg_q == nullptr || m->seg_kv == nullptr))
    return BSA_ERR_INVALID_ARG;
  if ((m->flags & BSA_MASK_KV_VALID_LEN) && need && m->kv_valid_len == nullptr)
    return BSA_ERR_INVALID_ARG;
  if (m->flags & BSA_MASK_VARLEN) {
    if (m->flags & BSA_MASK_SEGMENT_IDS) return BSA_ERR_INVALID_ARG;
    if (m->cu_seqlens == nullptr || m->n_seqs < 1 || m->n_align_tail < 0 ||
        m->n_align_tail > m->n_seqs || p.B != 1 || p.Sq != p.Skv)
      return BSA_ERR_INVALID_ARG;
  }
  if ((m->flags & BSA_MASK_CAUSAL_WINDOW) && m->window < 0) return BSA_ERR_INVALID_ARG;
  if (!(m->flags & BSA_MASK_CAUSAL_WINDOW)) out->window = 0;
  if (!(m->flags & BSA_MASK_VARLEN)) {
    out->n_seqs = 0;
    out->n_align_tail = 0;
  }
  return BSA_OK;
}

bsa_status check_options(const bsa_options *o, int nN, bsa_options *out) {
  std::memset(out, 0, sizeof(*out));
  out->deterministic = 1;
  if (o == nullptr) return BSA_OK;
  *out = *o;
  if (o->softmax_mode != BSA_SOFTMAX_ONLINE && o->softmax_mode != BSA_SOFTMAX_FIXED_M_GATED)
    return BSA_ERR_INVALID_ARG;
  if (o->bwd_order < BSA_ORDER_ASC || o->bwd_order > BSA_ORDER_GREEDY) return BSA_ERR_INVALID_ARG;
  if (o->bound_mode != BSA_BOUND_NORM && o->bound_mode != BSA_BOUND_SMOOTHED && o->bound_mode != BSA_BOUND_BLOCK)
    return BSA_ERR_INVALID_ARG;
  if (o->bound_mode != BSA_BOUND_NORM && o->kmax_override != nullptr) return BSA_ERR_INVALID_ARG;
  if (o->o_residual < BSA_O_RESIDUAL_AUTO || o->o_residual > BSA_O_RESIDUAL_DROP) return BSA_ERR_INVALID_ARG;
  if (o->bwd_order == BSA_ORDER_PERM) {
    if (o->perm == nullptr) return BSA_ERR_INVALID_ARG;
    std::vector<char> seen(static_cast<size_t>(nN), 0);
    for (int t = 0; t < nN; ++t) {
      const int n = o->perm[t];
      if (n < 0 || n >= nN || seen[static_cast<size_t>(n)]) return BSA_ERR_INVALID_ARG;
      seen[static_cast<size_t>(n)] = 1;
    }
  }
  return BSA_OK;
}

PlanSignature signature(const bsa_problem &p, const bsa_mask_spec &m, const bsa_options &o) {
  PlanSignature s{};
  s.w[0] = p.B;
  s.w[1] = p.Sq;
  s.w[2] = p.Skv;
  s.w[3] = m.flags;
  s.w[4] = m.window;
  s.w[5] = o.bwd_order;
  s.w[6] = m.n_seqs;
  s.w[7] = m.dilation;
  return s;
}

MaskParams mask_params(const bsa_problem &p, const bsa_mask_spec &m, const WsLayout &L,
                       uint8_t *ws) {
  MaskParams mp{};
  mp.flags = m.flags;
  mp.window = m.window;
  mp.offset = p.Skv - p.Sq;
  mp.Sq = p.Sq;
  mp.Skv = p.Skv;
  mp.kv_valid_len = (m.flags & BSA_MASK_KV_VALID_LEN) ? m.kv_valid_len : nullptr;
  mp.prefix_len = (m.flags & BSA_MASK_PREFIX_LM) ? m.prefix_len : nullptr;
  mp.dilation = m.dilation > 1 ? m.dilation : 1;
  mp.dil_pattern = 0;
  for (int k = 0; mp.dilation > 1 && k < 32; k += mp.dilation) mp.dil_pattern |= 1u << k;
  mp.dil_r32 = 32 % mp.dilation;
  if (m.flags & BSA_MASK_SEGMENT_IDS) {
    mp.seg_q = m.seg_q;
    mp.seg_kv = m.seg_kv;
  } else if (m.flags & BSA_MASK_VARLEN) {
    mp.seg_q = reinterpret_cast<const int32_t *>(ws + L.seg_q);
    mp.seg_kv = reinterpret_cast<const int32_t *>(ws + L.seg_kv);
  }
  return mp;
}

bool have_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return false;
  return major == 10;
}

struct Prepared {
  bsa_problem p;
  bsa_mask_spec m;
  bsa_options o;
  WsLayout L;
  bool empty;  // nothing to compute: no workspace, pointer or device is touched
};

bsa_status prepare(const bsa_problem *prob, const bsa_mask_spec *mask, const bsa_options *opt,
                   void *ws, size_t ws_bytes, bool backward, Prepared *out) {
  bsa_status st = normalise(prob, &out->p);
  if (st != BSA_OK) return st;
  if ((st = check_mask(out->p, mask, &out->m)) != BSA_OK) return st;
  out->L = compute_layout(out->p);
  if ((st = check_options(opt, out->L.nN, &out->o)) != BSA_OK) return st;
  if (out->o.bound_mode == BSA_BOUND_SMOOTHED && out->p.H_kv * out->p.D > kMaxSmoothedHD)
    return BSA_ERR_UNSUPPORTED;
  out->empty = problem_is_empty(&out->p);
  if (out->empty) return BSA_OK;
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return BSA_ERR_INVALID_ARG;
  // the O residual lives in the backward part of the workspace
  const bool full = backward || out->o.o_residual == BSA_O_RESIDUAL_KEEP;
  if (ws_bytes < (full ? out->L.total : out->L.fwd_end)) return BSA_ERR_WORKSPACE_TOO_SMALL;
  if (!have_device()) return BSA_ERR_NO_DEVICE;
  return BSA_OK;
}

bsa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? BSA_OK : BSA_ERR_CUDA; }

// B >= 1 batches of keys but no query row: the gradient is dK = dV = 0, the
// one result of an empty problem that has elements.
bool keys_without_rows(const bsa_problem *prob) {
  return prob != nullptr && prob->B > 0 && prob->Sq == 0;
}

bsa_status check_kv_grads(const void *dk, const void *dv) {
  if (dk == nullptr || dv == nullptr) return BSA_ERR_INVALID_ARG;
  if (!aligned16(dk) || !aligned16(dv)) return BSA_ERR_UNSUPPORTED;
  return BSA_OK;
}

// The result of the backward calls for an empty problem (after `prepare`).
bsa_status empty_backward(const bsa_problem &p, void *dk, void *dv, bsa_stream_t stream) {
  if (!keys_without_rows(&p)) return BSA_OK;
  if (!have_device()) return BSA_ERR_NO_DEVICE;
  return cuda_status(launch_zero_kv_grads(p, dk, dv, reinterpret_cast<cudaStream_t>(stream)));
}


// ---------------------------------------------------------------- plan || bound
constexpr int kMaxSideDevices = 64;
std::mutex g_side_mu;
cudaStream_t g_side[kMaxSideDevices] = {};

// The library's side stream on the current device (non-blocking: it never
// orders itself against the legacy default stream; every use is joined by
// events).
cudaError_t side_stream(cudaStream_t *out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxSideDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_side_mu);
  if (g_side[dev] == nullptr) {
    // the highest priority, so that the planner's one CTA (a whole SM's
    // registers) is placed before the bound's CTAs fill every SM
    int lo = 0, hi = 0;
    e = cudaDeviceGetStreamPriorityRange(&lo, &hi);
    if (e != cudaSuccess) return e;
    e = cudaStreamCreateWithPriority(&g_side[dev], cudaStreamNonBlocking, hi);
    if (e != cudaSuccess) return e;
  }
  *out = g_side[dev];
  return cudaSuccess;
}

// The fork and join events of the calling host thread on the current device,
// created on first use and kept for the thread's lifetime: a stream wait takes
// an event's state when it is issued, so re-recording them in the next call is
// safe, and separate host threads never share a pair.  (Kept, not created and
// destroyed per call, so that a call inside a stream capture creates nothing.)
struct ThreadEvents {
  cudaEvent_t fork[kMaxSideDevices] = {}, join[kMaxSideDevices] = {};
  ~ThreadEvents() {
    for (int d = 0; d < kMaxSideDevices; ++d) {
      if (fork[d] != nullptr) cudaEventDestroy(fork[d]);
      if (join[d] != nullptr) cudaEventDestroy(join[d]);
    }
  }
};
thread_local ThreadEvents t_events;

cudaError_t thread_events(cudaEvent_t *fork, cudaEvent_t *join) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxSideDevices) return cudaErrorInvalidDevice;
  if (t_events.fork[dev] == nullptr &&
      (e = cudaEventCreateWithFlags(&t_events.fork[dev], cudaEventDisableTiming)) != cudaSuccess)
    return e;
  if (t_events.join[dev] == nullptr &&
      (e = cudaEventCreateWithFlags(&t_events.join[dev], cudaEventDisableTiming)) != cudaSuccess)
    return e;
  *fork = t_events.fork[dev];
  *join = t_events.join[dev];
  return cudaSuccess;
}

// The block-map plan and the fixed-m bound of one call.  The bound reads the
// planner's output only for varlen masks (the alignment rows' ids); otherwise
// the two are independent, and the planner (one CTA) runs on the side stream
// while the bound's row-norm pass (the rest of the GPU) runs on `s`: forked
// from and joined back into `s` by events, so work after the call on `s` sees
// both, and stream capture records the same fork and join.
cudaError_t plan_and_bound(const bsa_problem &p, const bsa_mask_spec &m, const bsa_options &o,
                           const void *q, const void *k, const WsLayout &L, uint8_t *ws,
                           cudaStream_t s) {
  const MaskParams mp = mask_params(p, m, L, ws);
  if (m.flags & BSA_MASK_VARLEN) {
    cudaError_t e = launch_plan(p, m, o, L, ws, s);
    if (e != cudaSuccess) return e;
    return launch_fixed_m_bound(p, mp, o, q, k, L, ws, s);
  }
  cudaStream_t side = nullptr;
  cudaError_t e = side_stream(&side);
  if (e != cudaSuccess) return e;
  cudaEvent_t fork = nullptr, join = nullptr;
  if ((e = thread_events(&fork, &join)) != cudaSuccess) return e;
  e = cudaEventRecord(fork, s);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(side, fork, 0);
  if (e == cudaSuccess) e = launch_plan(p, m, o, L, ws, side);
  if (e == cudaSuccess) e = cudaEventRecord(join, side);
  cudaError_t eb = cudaSuccess;
  if (e == cudaSuccess) eb = launch_fixed_m_bound(p, mp, o, q, k, L, ws, s);
  // join even when the bound failed to launch, so `s` never runs ahead of the plan
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s, join, 0);
  return e != cudaSuccess ? e : eb;
}

}  // namespace

// The forward call.  side_stream_ok = false keeps the plan and the bound on
// `stream` one after the other (the static-scratch entry makes no call that
// creates a stream or an event).
bsa_status attn_fwd_impl(const bsa_problem *prob, const bsa_mask_spec *mask,
                         const bsa_options *opt, const void *q, const void *k, const void *v,
                         void *out, float *lse, void *ws, size_t ws_bytes, bsa_stream_t stream,
                         bool side_stream_ok) {
  if (!problem_is_empty(prob)) {
    if (q == nullptr || k == nullptr || v == nullptr || out == nullptr || lse == nullptr)
      return BSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
        (reinterpret_cast<uintptr_t>(lse) & 3u))
      return BSA_ERR_UNSUPPORTED;
  }
  Prepared P;
  bsa_status st = prepare(prob, mask, opt, ws, ws_bytes, false, &P);
  if (st != BSA_OK || P.empty) return st;
  const bsa_problem &p = P.p;
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, q, p.B, p.Sq, p.H, p.D, p.q_stride) ||
      !make_map(&tk, k, p.B, p.Skv, p.H_kv, p.D, p.k_stride) ||
      !make_map(&tv, v, p.B, p.Skv, p.H_kv, p.D, p.v_stride))
    return BSA_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t *w = static_cast<uint8_t *>(ws);
  const bool need_bound = P.o.softmax_mode == BSA_SOFTMAX_FIXED_M_GATED && !P.o.bound_ready;
  if (!P.o.plan_ready && need_bound && side_stream_ok) {
    if ((st = cuda_status(plan_and_bound(p, P.m, P.o, q, k, P.L, w, s))) != BSA_OK) return st;
  } else {
    if (!P.o.plan_ready && (st = cuda_status(launch_plan(p, P.m, P.o, P.L, w, s))) != BSA_OK) return st;
    if (need_bound &&
        (st = cuda_status(launch_fixed_m_bound(p, mask_params(p, P.m, P.L, w), P.o, q, k, P.L, w, s))) != BSA_OK)
      return st;
  }
  const MaskParams mp = mask_params(p, P.m, P.L, w);
  // the residual is kept when asked for, or by default when the workspace can
  // serve a backward; the forward records in the header which `out` it is for
  bsa_options fo = P.o;
  const bool keep = P.o.o_residual == BSA_O_RESIDUAL_KEEP ||
                    (P.o.o_residual == BSA_O_RESIDUAL_AUTO && ws_bytes >= P.L.total);
  fo.o_residual = keep ? BSA_O_RESIDUAL_KEEP : BSA_O_RESIDUAL_DROP;
  return cuda_status(launch_fwd(p, mp, fo, signature(p, P.m, P.o), tq, tk, tv, q, out, lse, P.L, w, s));
}

}  // namespace bsa

using namespace bsa;

extern "C" {

bsa_status bsa_workspace_size(const bsa_problem *prob, const bsa_mask_spec *mask,
                              int32_t with_backward, size_t *bytes) {
  if (bytes == nullptr) return BSA_ERR_INVALID_ARG;
  bsa_problem p;
  bsa_status st = normalise(prob, &p);
  if (st != BSA_OK) return st;
  bsa_mask_spec m;
  if ((st = check_mask(p, mask, &m)) != BSA_OK) return st;
  const WsLayout L = compute_layout(p);
  *bytes = problem_is_empty(&p) ? 0 : with_backward ? L.total : L.fwd_end;
  return BSA_OK;
}

bsa_status bsa_workspace_layout(const bsa_problem *prob, const bsa_mask_spec *mask,
                                bsa_workspace_view *view) {
  if (view == nullptr) return BSA_ERR_INVALID_ARG;
  bsa_problem p;
  bsa_status st = normalise(prob, &p);
  if (st != BSA_OK) return st;
  bsa_mask_spec m;
  if ((st = check_mask(p, mask, &m)) != BSA_OK) return st;
  const WsLayout L = compute_layout(p);
  if (problem_is_empty(&p)) {
    std::memset(view, 0, sizeof(*view));
    view->nM = L.nM;
    view->nN = L.nN;
    return BSA_OK;
  }
  view->total_bytes = L.total;
  view->fwd_bytes = L.fwd_end;
  view->off_status = L.status;
  view->off_tile_class = L.tile_class;
  view->off_rank = L.rank;
  view->off_row_ptr = L.row_ptr;
  view->off_row_ent = L.row_ent;
  view->off_col_ptr = L.col_ptr;
  view->off_col_ent = L.col_ent;
  view->off_col_rank = L.col_rank;
  view->off_perm = L.perm;
  view->off_kmax = L.kmax;
  view->off_qmax = L.qmax;
  view->off_gate = L.gate;
  view->off_delta = L.delta;
  view->off_dq_accum = L.dq_accum;
  view->off_sem = L.sem;
  view->off_kbar = L.kbar;
  view->off_qdot = L.qdot;
  view->off_o_resid = L.o_resid;
  view->off_kblk = L.kbmax;
  view->off_kmax_q = L.kmax_q;
  view->nM = L.nM;
  view->nN = L.nN;
  return BSA_OK;
}

bsa_status bsa_plan_build(const bsa_problem *prob, const bsa_mask_spec *mask,
                          const bsa_options *opt, void *ws, size_t ws_bytes, bsa_stream_t stream) {
  Prepared P;
  bsa_status st = prepare(prob, mask, opt, ws, ws_bytes, false, &P);
  if (st != BSA_OK || P.empty) return st;
  return cuda_status(launch_plan(P.p, P.m, P.o, P.L, static_cast<uint8_t *>(ws),
                                 reinterpret_cast<cudaStream_t>(stream)));
}

bsa_status bsa_attn_fwd(const bsa_problem *prob, const bsa_mask_spec *mask,
                        const bsa_options *opt, const void *q, const void *k, const void *v,
                        void *out, float *lse, void *ws, size_t ws_bytes, bsa_stream_t stream) {
  return bsa::attn_fwd_impl(prob, mask, opt, q, k, v, out, lse, ws, ws_bytes, stream, true);
}

bsa_status bsa_attn_bwd(const bsa_problem *prob, const bsa_mask_spec *mask,
                        const bsa_options *opt, const void *q, const void *k, const void *v,
                        const void *out, const void *dout, const float *lse, void *dq, void *dk,
                        void *dv, void *ws, size_t ws_bytes, bsa_stream_t stream) {
  bsa_status st;
  if (keys_without_rows(prob)) {
    if ((st = check_kv_grads(dk, dv)) != BSA_OK) return st;
  } else if (!problem_is_empty(prob)) {
    if (q == nullptr || k == nullptr || v == nullptr || out == nullptr || dout == nullptr ||
        lse == nullptr || dq == nullptr || dk == nullptr || dv == nullptr)
      return BSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) ||
        !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
        (reinterpret_cast<uintptr_t>(lse) & 3u))
      return BSA_ERR_UNSUPPORTED;
  }
  Prepared P;
  if ((st = prepare(prob, mask, opt, ws, ws_bytes, true, &P)) != BSA_OK) return st;
  if (P.empty) return empty_backward(P.p, dk, dv, stream);
  const bsa_problem &p = P.p;
  CUtensorMap tq, tk, tv, tdo;
  if (!bwd_maps(p, P.L, static_cast<uint8_t *>(ws), k, v, &tq, &tk, &tv, &tdo)) return BSA_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t *w = static_cast<uint8_t *>(ws);
  if (!P.o.plan_ready) {
    if ((st = cuda_status(launch_plan(p, P.m, P.o, P.L, w, s))) != BSA_OK) return st;
  }
  const MaskParams mp = mask_params(p, P.m, P.L, w);
  return cuda_status(launch_bwd(p, mp, P.o, signature(p, P.m, P.o), tq, tk, tv, tdo, q, out, dout,
                                lse, dq, dk, dv, P.L, w, s));
}

bsa_status bsa_fixed_m_bound(const bsa_problem *prob, const bsa_mask_spec *mask,
                             const bsa_options *opt, const void *q, const void *k, void *ws,
                             size_t ws_bytes, bsa_stream_t stream) {
  if (!problem_is_empty(prob)) {
    if (q == nullptr || k == nullptr) return BSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k)) return BSA_ERR_UNSUPPORTED;
  }
  Prepared P;
  bsa_status st = prepare(prob, mask, opt, ws, ws_bytes, false, &P);
  if (st != BSA_OK || P.empty) return st;
  uint8_t *w = static_cast<uint8_t *>(ws);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (!P.o.plan_ready) {
    // the key-validity predicates of varlen masks come from the planner
    if ((st = cuda_status(launch_plan(P.p, P.m, P.o, P.L, w, s))) != BSA_OK) return st;
  }
  const MaskParams mp = mask_params(P.p, P.m, P.L, w);
  return cuda_status(launch_fixed_m_bound(P.p, mp, P.o, q, k, P.L, w, s));
}

bsa_status bsa_plan_and_bound(const bsa_problem *prob, const bsa_mask_spec *mask,
                              const bsa_options *opt, const void *q, const void *k, void *ws,
                              size_t ws_bytes, bsa_stream_t stream) {
  if (!problem_is_empty(prob)) {
    if (q == nullptr || k == nullptr) return BSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k)) return BSA_ERR_UNSUPPORTED;
  }
  Prepared P;
  bsa_status st = prepare(prob, mask, opt, ws, ws_bytes, false, &P);
  if (st != BSA_OK || P.empty) return st;
  return cuda_status(plan_and_bound(P.p, P.m, P.o, q, k, P.L, static_cast<uint8_t *>(ws),
                                    reinterpret_cast<cudaStream_t>(stream)));
}

bsa_status bsa_bwd_preprocess(const bsa_problem *prob, const bsa_mask_spec *mask,
                              const bsa_options *opt, const void *q, const void *out,
                              const void *dout, void *ws, size_t ws_bytes, bsa_stream_t stream) {
  if (!problem_is_empty(prob)) {
    if (q == nullptr || out == nullptr || dout == nullptr) return BSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(out) || !aligned16(dout)) return BSA_ERR_UNSUPPORTED;
  }
  Prepared P;
  bsa_status st = prepare(prob, mask, opt, ws, ws_bytes, true, &P);
  if (st != BSA_OK || P.empty) return st;
  return cuda_status(launch_bwd_preprocess(P.p, P.o, q, out, dout, P.L, static_cast<uint8_t *>(ws),
                                           reinterpret_cast<cudaStream_t>(stream)));
}

bsa_status bsa_bwd_main(const bsa_problem *prob, const bsa_mask_spec *mask,
                        const bsa_options *opt, const void *q, const void *k, const void *v,
                        const void *dout, const float *lse, void *dk, void *dv, void *ws,
                        size_t ws_bytes, bsa_stream_t stream) {
  bsa_status st;
  if (keys_without_rows(prob)) {
    if ((st = check_kv_grads(dk, dv)) != BSA_OK) return st;
  } else if (!problem_is_empty(prob)) {
    if (q == nullptr || k == nullptr || v == nullptr || dout == nullptr || lse == nullptr ||
        dk == nullptr || dv == nullptr)
      return BSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) || !aligned16(dk) ||
        !aligned16(dv) || (reinterpret_cast<uintptr_t>(lse) & 3u))
      return BSA_ERR_UNSUPPORTED;
  }
  Prepared P;
  if ((st = prepare(prob, mask, opt, ws, ws_bytes, true, &P)) != BSA_OK) return st;
  if (P.empty) return empty_backward(P.p, dk, dv, stream);
  const bsa_problem &p = P.p;
  CUtensorMap tq, tk, tv, tdo;
  if (!bwd_maps(p, P.L, static_cast<uint8_t *>(ws), k, v, &tq, &tk, &tv, &tdo)) return BSA_ERR_UNSUPPORTED;
  uint8_t *w = static_cast<uint8_t *>(ws);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (!P.o.plan_ready) {
    if ((st = cuda_status(launch_plan(p, P.m, P.o, P.L, w, s))) != BSA_OK) return st;
  }
  const MaskParams mp = mask_params(p, P.m, P.L, w);
  return cuda_status(launch_bwd_main(p, mp, P.o, signature(p, P.m, P.o), tq, tk, tv, tdo, lse, dk,
                                     dv, P.L, w, s));
}

bsa_status bsa_bwd_convert(const bsa_problem *prob, const bsa_mask_spec *mask, void *dq, void *ws,
                           size_t ws_bytes, bsa_stream_t stream) {
  if (!problem_is_empty(prob)) {
    if (dq == nullptr) return BSA_ERR_INVALID_ARG;
    if (!aligned16(dq)) return BSA_ERR_UNSUPPORTED;
  }
  Prepared P;
  bsa_status st = prepare(prob, mask, nullptr, ws, ws_bytes, true, &P);
  if (st != BSA_OK || P.empty) return st;
  return cuda_status(launch_bwd_convert(P.p, dq, P.L, static_cast<uint8_t *>(ws),
                                        reinterpret_cast<cudaStream_t>(stream)));
}

bsa_status bsa_get_device_status(void *ws, size_t ws_bytes, bsa_stream_t stream, int32_t clear) {
  if (ws == nullptr || ws_bytes < kHdrWords * 4) return BSA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t h[2] = {0, 0};
  if (cudaMemcpyAsync(h, ws, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return BSA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return BSA_ERR_CUDA;
  if (clear) {
    if (cudaMemsetAsync(ws, 0, sizeof(h), s) != cudaSuccess) return BSA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return BSA_ERR_CUDA;
  }
  if (h[kHdrStatus] != 0) return static_cast<bsa_status>(h[kHdrStatus]);
  if (h[kHdrGateWarn] != 0) return BSA_WARN_GATE_VIOLATION;
  return BSA_OK;
}

bsa_status bsa_fixed_rows(void *ws, size_t ws_bytes, bsa_stream_t stream, uint64_t *rows) {
  if (ws == nullptr || rows == nullptr || ws_bytes < kHdrWords * 4) return BSA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t n = 0;
  if (cudaMemcpyAsync(&n, static_cast<uint32_t *>(ws) + kHdrFixedRows, sizeof(n), cudaMemcpyDeviceToHost, s) !=
      cudaSuccess)
    return BSA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return BSA_ERR_CUDA;
  *rows = n;
  return BSA_OK;
}

const char *bsa_status_string(bsa_status status) {
  switch (status) {
    case BSA_OK: return "ok";
    case BSA_ERR_INVALID_ARG: return "invalid argument";
    case BSA_ERR_UNSUPPORTED: return "unsupported shape, dtype, stride or alignment";
    case BSA_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case BSA_ERR_CUDA: return "CUDA runtime error";
    case BSA_ERR_SEM_TIMEOUT: return "a bounded device wait timed out; results are incomplete";
    case BSA_ERR_PLAN_MISMATCH: return "workspace plan was built for another problem";
    case BSA_ERR_BAD_MASK_DATA: return "cu_seqlens is not a non-decreasing [0 .. Sq] sequence";
    case BSA_WARN_GATE_VIOLATION: return "a gated fixed-m row summed below 2^-100";
    case BSA_ERR_NO_DEVICE: return "no sm_100 device is current";
    case BSA_ERR_INPUT_RANGE:
      return "a backward input or dS entry lies beyond the fp16 range or is not finite";
  }
  return "unknown status";
}

uint64_t bsa_launch_count(void) { return g_launches.load(); }

}  // extern "C"
