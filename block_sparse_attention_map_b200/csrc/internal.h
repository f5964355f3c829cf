// Internal declarations shared by the library's translation units: the
// workspace layout, the mask parameters every kernel evaluates, and the
// launchers of each step of the hot path.
#pragma once

#include <cstddef>
#include <cstdint>
#include <utility>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/bsa.h"

namespace bsa {

constexpr int kTile = BSA_TILE;
constexpr uint32_t kFullBit = 1u << 30;
constexpr uint32_t kIndexMask = (1u << 30) - 1u;
constexpr uint32_t kPlanMagic = 0xB5A7C0DEu;
// Largest Sq and Skv accepted (bsa_problem).
constexpr int kMaxSeq = 1 << 21;
// Largest H * D of the k-smoothed bound: one block keeps the centers of all
// heads of a batch row in shared memory (fp32).
constexpr int kMaxSmoothedHD = 24576;

// Header words at the start of the workspace.
enum HeaderWord : int {
  kHdrStatus = 0,      // sticky bsa_status
  kHdrGateWarn = 1,    // rows of gated heads whose fixed-m sum fell below 2^-100
  kHdrFwdTicket = 2,   // forward work-unit ticket counter
  kHdrBwdTicket = 3,   // backward column ticket counter
  kHdrMagic = 4,       // plan signature: magic, B, Sq, Skv, flags, window, order, n_seqs
  kHdrB = 5,
  kHdrSq = 6,
  kHdrSkv = 7,
  kHdrFlags = 8,
  kHdrWindow = 9,
  kHdrOrder = 10,
  kHdrNSeqs = 11,
  kHdrDilation = 12,
  kHdrFixedRows = 13,  // query rows the forwards since the plan build ran with a pinned reference
  kHdrFwdDone = 14,    // forward CTAs finished; the last one puts both forward words back to 0
  kHdrBwdDone = 15,    // the same for the backward's column ticket
  kHdrDqMode = 16,     // the last Delta pass's dQ protocol: 1 semaphore-ordered, 2 atomic (0: none)
  kHdrPlanWords = 48,  // words [0, 48) are reset by every plan build
  // The fp16-Q record (kept across plan builds): the `q` pointer and strides
  // whose fp16 copy the last forward on this workspace wrote (pointer 0: none);
  // it is written only together with the O residual, whose record below holds
  // the problem.
  kHdrQ16Lo = 48,
  kHdrQ16Hi = 49,
  kHdrQ16Sb = 50,
  kHdrQ16Ss = 51,
  kHdrQ16Sh = 52,
  // The O-residual record (kept across plan builds): the `out` pointer whose
  // residual the last forward on this workspace kept (0: none) and the problem
  // it was kept for, whose layout places the residual.
  kHdrResidLo = 56,
  kHdrResidHi = 57,
  kHdrResidB = 58,
  kHdrResidH = 59,
  kHdrResidSq = 60,
  kHdrResidSkv = 61,
  kHdrResidD = 62,
  kHdrWords = 64
};

struct WsLayout {
  size_t status;                      // header (256 bytes)
  size_t tile_class, rank;            // dense [B, nM, nN]
  size_t row_cnt, row_ptr, row_ent;   // row CSR (forward)
  size_t col_cnt, col_ptr, col_ent, col_rank;  // column CSR (backward)
  size_t perm;                        // pi [nN]
  size_t seg_q, seg_kv;               // varlen-derived segment ids [Sq], [Skv]
  size_t qblk, kblk;                  // per-block segment summaries [B*nM*4], [B*nN*4]
  size_t kmax, qmax, gate;            // [B, H]
  size_t qnorm;                       // [B, H, Sq]
  size_t kbar, ksum, kcount, qdot;    // k-smoothing: center [B,H,D] fp32, its fixed-point
                                      // sums [B,H,D] int64, valid keys [B], q.c [B,H,Sq]
  size_t kbmax, kmax_q;               // per q-block bound: [B,H_kv,nN] key-block maxima,
                                      // [B,H,nM] each q-block's kmax (written by the forward)
  size_t fwd_end;
  size_t delta, dq_accum, sem;        // backward scratch
  size_t o_resid;                     // [B, Sq, H, D] O rounding residual, scaled e5m2 bytes
  size_t q16, do16;                   // [B, Sq, H, D] fp16 copies of Q and dO (backward)
  size_t total;
  int nM, nN;
  int64_t nnz_cap;
};

WsLayout compute_layout(const bsa_problem &p);

// Plan signature words (B, Sq, Skv, flags, window, order, n_seqs, dilation)
// the planner stores in the header and every kernel that reads the plan checks.
constexpr int kSigWords = 8;
constexpr int kSigOrderWord = 5;
struct PlanSignature {
  uint32_t w[kSigWords];
};

// Mask predicates as every kernel sees them.  Varlen masks arrive here as
// segment ids derived by the planner (alignment rows: -1 on the query side,
// -2 on the key side, so they never match anything).
struct MaskParams {
  uint32_t flags;
  int32_t window;       // 0 = plain causal (when the flag is set)
  int32_t offset;       // o = Skv - Sq (bottom-right alignment)
  int32_t Sq, Skv;
  const int32_t *seg_q;   // [B, Sq] or null
  const int32_t *seg_kv;  // [B, Skv] or null
  const int32_t *kv_valid_len;  // [B] or null
  const int32_t *prefix_len;    // [B] or null (only with the window flag)
  int32_t dilation;             // > 1: dilated window, else 1
  uint32_t dil_pattern;         // bits 0, d, 2d, ... below 32 (dilation > 1)
  int32_t dil_r32;              // 32 mod d
};

// Launchers (each returns cudaGetLastError() of its launches).
cudaError_t launch_plan(const bsa_problem &p, const bsa_mask_spec &m, const bsa_options &o,
                        const WsLayout &L, uint8_t *ws, cudaStream_t s);

cudaError_t launch_fixed_m_bound(const bsa_problem &p, const MaskParams &mp,
                                 const bsa_options &o, const void *q, const void *k,
                                 const WsLayout &L, uint8_t *ws, cudaStream_t s);

cudaError_t launch_fwd(const bsa_problem &p, const MaskParams &mp, const bsa_options &o,
                       const PlanSignature &sig, const CUtensorMap &tq, const CUtensorMap &tk,
                       const CUtensorMap &tv, const void *q, void *out, float *lse,
                       const WsLayout &L, uint8_t *ws, cudaStream_t s);

cudaError_t launch_bwd(const bsa_problem &p, const MaskParams &mp, const bsa_options &o,
                       const PlanSignature &sig, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                       const CUtensorMap &tdo, const void *q, const void *out, const void *dout,
                       const float *lse, void *dq, void *dk, void *dv, const WsLayout &L,
                       uint8_t *ws, cudaStream_t s);

cudaError_t launch_bwd_preprocess(const bsa_problem &p, const bsa_options &o, const void *q,
                                  const void *out, const void *dout, const WsLayout &L,
                                  uint8_t *ws, cudaStream_t s);

cudaError_t launch_bwd_main(const bsa_problem &p, const MaskParams &mp, const bsa_options &o,
                            const PlanSignature &sig, const CUtensorMap &tq, const CUtensorMap &tk,
                            const CUtensorMap &tv, const CUtensorMap &tdo, const float *lse,
                            void *dk, void *dv, const WsLayout &L, uint8_t *ws, cudaStream_t s);

cudaError_t launch_bwd_convert(const bsa_problem &p, void *dq, const WsLayout &L, uint8_t *ws,
                               cudaStream_t s);

// dK = dV = 0 (a problem with B >= 1 key rows but Sq == 0): one kernel.
cudaError_t launch_zero_kv_grads(const bsa_problem &p, void *dk, void *dv, cudaStream_t s);

void count_launch(int n = 1);

// Launch with programmatic stream serialization: the kernel may start while
// the stream's preceding kernel finishes, and must call pdl_wait() before it
// touches anything that kernel writes or reads.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// B == 0 or Sq == 0: the call checks its arguments and then does nothing.
bool problem_is_empty(const bsa_problem *prob);

// bsa_attn_fwd; side_stream_ok = false never forks work onto the library's side
// stream (no stream or event is created).
bsa_status attn_fwd_impl(const bsa_problem *prob, const bsa_mask_spec *mask,
                         const bsa_options *opt, const void *q, const void *k, const void *v,
                         void *out, float *lse, void *ws, size_t ws_bytes, bsa_stream_t stream,
                         bool side_stream_ok);

}  // namespace bsa
