/*
 * bsa.h -- C ABI of libbsa: block-sparse exact softmax attention for sm_100a.
 *
 * What the library computes (all of it in its own CUDA kernels):
 *
 *   O = softmax(scale * Q K^T + mask) V  and the per-row LSE,
 *   dQ, dK, dV of sum(O * dO) with a deterministic dQ accumulation.
 *
 * The mask is the AND of up to four predicates (segment ids, global KV padding,
 * varlen cu_seqlens with trailing alignment rows, causal sliding window).  A
 * block map classifies every 128 x 128 (q-block, kv-block) tile as EMPTY,
 * PARTIAL or FULL so that empty tiles are never touched and full tiles skip the
 * per-element mask.
 *
 * Sources (the pages this library restates):
 *  - "Fixed-m softmax for 2D-ring x Ulysses attention (WAN 2.2)" (maxdiffusion
 *    PR #452): exact softmax attention whose running max may be replaced by the
 *    Cauchy-Schwarz bound scale*||q_i||*max_j||k_j||, with a per-head gate that
 *    keeps online softmax where the bound cannot be proven safe.
 *  - "Let splash attention exceed 524,288 tokens when packing is off" (maxtext
 *    PR #4929): segment-id masks; constant ids equal no ids; a block mask.
 *  - maxdiffusion PR #404 review, padding-mask comment: KV padding only at the
 *    end of the global sequence, masked by global position.
 *  - sglang PR #47566, "Modifications": cu_seqlens with trailing alignment rows
 *    that real rows never see; alignment rows are zero in the output.
 *  - "Add more optimal dk order optional arg" (flash-attention PR #2512):
 *    deterministic block-sparse backward with per-m_block dQ semaphores,
 *    rank(m, n), kv-column orders (asc, desc, arbitrary permutation) and one
 *    rank-sorted list per kv column.
 *
 * Conventions for every call:
 *  - All tensor pointers are DEVICE pointers unless a field says "host".
 *  - Q, K, V, O, dO, dQ, dK, dV are bf16 [B, S, H, D] with the head dimension
 *    contiguous; other strides are given in elements (0 = contiguous BSHD).
 *    Pointers and strides must be 16-byte aligned.  D is 64 or 128.
 *  - LSE is fp32 [B, H, Sq], natural log; a row with no allowed key has
 *    LSE = -inf and O = 0.
 *  - The caller owns every buffer, including the workspace.  The library never
 *    allocates device memory, never synchronises (except in
 *    bsa_get_device_status) and issues all work on the given stream.  Pointers
 *    are borrowed for the duration of the call's stream work only.
 *  - Argument errors are returned before anything is launched and nothing is
 *    written.  Errors detected on the device (inconsistent cu_seqlens, a plan
 *    that does not match the problem, a semaphore wait that timed out) are
 *    recorded in the workspace's sticky status word; read it with
 *    bsa_get_device_status.  There is no CPU fallback and no second backend.
 */
#ifndef BSA_H_
#define BSA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BSA_API __attribute__((visibility("default")))
#else
#define BSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream; 0 is the legacy default stream. */
typedef struct CUstream_st *bsa_stream_t;

typedef enum bsa_status {
  BSA_OK = 0,
  BSA_ERR_INVALID_ARG = 1,         /* null pointer, bad size, inconsistent fields   */
  BSA_ERR_UNSUPPORTED = 2,         /* D not in {64,128}, misaligned pointer/stride   */
  BSA_ERR_WORKSPACE_TOO_SMALL = 3, /* ws_bytes below bsa_workspace_size()            */
  BSA_ERR_CUDA = 4,                /* a CUDA runtime call or launch failed           */
  BSA_ERR_SEM_TIMEOUT = 5,         /* device: a bounded wait gave up (work skipped)  */
  BSA_ERR_PLAN_MISMATCH = 6,       /* device: workspace plan built for another problem */
  BSA_ERR_BAD_MASK_DATA = 7,       /* device: cu_seqlens not [0 .. Sq] non-decreasing */
  BSA_WARN_GATE_VIOLATION = 8,     /* device: a gated fixed-m row summed below 2^-100 */
  BSA_ERR_NO_DEVICE = 9,           /* no sm_100 device current                        */
  BSA_ERR_INPUT_RANGE = 10         /* device: a backward input (Q, K, V, dO) or an
                                      entry of dS lies beyond the fp16 range
                                      (|x| >= 65504) or is not finite; the
                                      backward takes its products in fp16 */
} bsa_status;

/* Block-map tile edge (rows and keys). */
#define BSA_TILE 128

/* Tile classes stored in the block map. */
#define BSA_TILE_EMPTY 0
#define BSA_TILE_PARTIAL 1
#define BSA_TILE_FULL 2

/* bsa_mask_spec.flags */
#define BSA_MASK_SEGMENT_IDS 1u   /* seg_q[b,i] == seg_kv[b,j]                         */
#define BSA_MASK_KV_VALID_LEN 2u  /* j < kv_valid_len[b]                                */
#define BSA_MASK_VARLEN 4u        /* same cu_seqlens segment, neither in the alignment tail */
#define BSA_MASK_CAUSAL_WINDOW 8u /* i+o-W < j <= i+o, o = Skv-Sq (W = 0: j <= i+o);
                                     with dilation d > 1 also (i+o-j) mod d == 0      */
#define BSA_MASK_PREFIX_LM 16u    /* with BSA_MASK_CAUSAL_WINDOW: keys j < prefix_len[b]
                                     are seen by every row as well (OR with the window) */

/* bsa_options.softmax_mode */
#define BSA_SOFTMAX_ONLINE 0
#define BSA_SOFTMAX_FIXED_M_GATED 1

/* bsa_options.bound_mode: the pinned reference of BSA_SOFTMAX_FIXED_M_GATED
 * ("Fixed-m softmax for 2D-ring x Ulysses attention (WAN 2.2)", introduction and
 * "Notes": k-smoothing is possible when one device holds all of K).
 *   NORM      m_i = scale*||q_i||*kmax, kmax = max over valid keys of ||k_j||;
 *             gate 2*scale*qmax*kmax <= G.
 *   SMOOTHED  center c = mean of the valid keys, R = max over valid keys of
 *             ||k_j - c||, m_i = scale*(q_i.c + ||q_i||*R); gate 2*scale*qmax*R <= G.
 *             The workspace's kmax array then holds R.  c is summed in a fixed-point
 *             format (terms rounded to 2^-20, |k| clamped to 2^20), so it does not
 *             depend on the order of the additions; any c keeps m_i a bound. */
#define BSA_BOUND_NORM 0
#define BSA_BOUND_SMOOTHED 1
/*   BLOCK     the pages' per-segment kmax, read as: per q-block m, kmax_m = the
 *             largest ||k_j|| over the valid keys of the kv blocks the block map
 *             lets q-block m reach (its non-empty tiles), so segments, windows
 *             and documents each get the bound of the keys their rows can see;
 *             m_i = scale*||q_i||*kmax_m, and the gate is taken per row:
 *             2*scale*||q_i||*kmax_m <= G (else that row runs online).  The
 *             bound pass reads K only (one maximum per kv block and key head);
 *             the forward takes ||q_i|| from its Q tile.  kmax_override is
 *             rejected with it. */
#define BSA_BOUND_BLOCK 2

/* bsa_options.bwd_order: order pi of the kv columns for the dQ semaphores */
#define BSA_ORDER_ASC 0
#define BSA_ORDER_DESC 1
#define BSA_ORDER_PERM 2
/* The two orders the "dk order" page's benchmark table names without defining
 * them, under the readings this library takes:
 *   OUTSIDE_IN  0, nN-1, 1, nN-2, ... (both ends first, then inwards);
 *   GREEDY      columns placed one at a time; each step takes the unplaced
 *               column whose non-empty tiles would wait on the most already
 *               placed tiles of their row blocks the least in total (ties: the
 *               smaller column), computed on the GPU by bsa_plan_build from
 *               the tile classes of all batches (one block; nN steps). */
#define BSA_ORDER_OUTSIDE_IN 3
#define BSA_ORDER_GREEDY 4

typedef struct bsa_problem {
  int32_t B;       /* batch, >= 0; 1 for varlen                                   */
  int32_t H;       /* query heads (Q, O, LSE, dQ, dO), >= 1                       */
  int32_t Sq;      /* query rows per batch (varlen: total tokens T); 0 .. 2^21    */
  int32_t Skv;     /* keys per batch (varlen: T); 1 .. 2^21                       */
  int32_t D;       /* head dim, 64 or 128                                         */
  int32_t H_kv;    /* key/value heads (K, V, dK, dV); 0 = H.  H must be a multiple:
                      query head h reads kv head h / (H / H_kv) (grouped-query
                      attention; H_kv = 1 is multi-query).  dK and dV of a kv
                      head are summed over the query heads of its group.        */
  /* element strides (batch, seq, head); all zero = contiguous BSHD.  q_stride
   * is used for Q and dQ, k_stride for K and dK, v_stride for V and dV,
   * o_stride for O and dO. */
  int64_t q_stride[3];
  int64_t k_stride[3];
  int64_t v_stride[3];
  int64_t o_stride[3];
  float scale;     /* <= 0: 1/sqrt(D)                                             */
  int32_t reserved1;
} bsa_problem;
/* An EMPTY problem (B == 0 or Sq == 0: no output row) is valid.  Every call
 * checks its shape, mask and options as usual, then returns BSA_OK without
 * touching a tensor or mask-array pointer (null allowed), the workspace
 * (0 bytes, null allowed), the stream or the device, and launches nothing.
 * Its workspace size is 0 and its bsa_workspace_view is all zero except nM
 * and nN.  The one exception: with B >= 1 and Sq == 0, dK and dV have
 * elements and their gradient is zero, so bsa_attn_bwd and bsa_bwd_main need
 * valid 16-byte aligned dk and dv (else INVALID_ARG / UNSUPPORTED) and a
 * device, and zero both with one kernel on `stream`.  Skv == 0 is an argument
 * error: a row with no allowed key is expressed by the mask (its output is 0
 * and its LSE -inf). */

typedef struct bsa_mask_spec {
  uint32_t flags;              /* OR of BSA_MASK_*                                  */
  int32_t window;              /* BSA_MASK_CAUSAL_WINDOW: keys per row including
                                  the diagonal; 0 = unlimited causal                */
  const int32_t *seg_q;        /* device [B, Sq]  (BSA_MASK_SEGMENT_IDS)            */
  const int32_t *seg_kv;       /* device [B, Skv] (BSA_MASK_SEGMENT_IDS)            */
  const int32_t *kv_valid_len; /* device [B]      (BSA_MASK_KV_VALID_LEN)           */
  const int32_t *cu_seqlens;   /* device [n_seqs + 1], cu[0] = 0, cu[n_seqs] = Sq    */
  int32_t n_seqs;              /* segments in cu_seqlens (BSA_MASK_VARLEN)           */
  int32_t n_align_tail;        /* trailing segments that are alignment rows         */
  const int32_t *prefix_len;   /* device [B]      (BSA_MASK_PREFIX_LM)              */
  int32_t dilation;            /* BSA_MASK_CAUSAL_WINDOW: keep only the keys whose
                                  distance back from the diagonal is a multiple of
                                  it; 0 or 1 = every key.  > 1 needs the window flag */
  int32_t reserved;
} bsa_mask_spec;

typedef struct bsa_options {
  int32_t softmax_mode;        /* BSA_SOFTMAX_*                                     */
  float gate_limit;            /* fixed-m gate G: a head runs fixed-m iff
                                  2*scale*max_i||q_i||*kmax <= G; <= 0: 64          */
  const float *kmax_override;  /* device [B, H] or NULL: caller-supplied max_j||k_j||
                                  bound used as is                                  */
  int32_t bwd_order;           /* BSA_ORDER_*                                       */
  int32_t deterministic;       /* 1: semaphore-ordered dQ; 0: atomic dQ             */
  const int32_t *perm;         /* HOST [ceil(Skv/128)] permutation (BSA_ORDER_PERM)  */
  int64_t sem_timeout_ns;      /* bound of every dQ semaphore wait; <= 0: 1 s       */
  int32_t plan_ready;          /* 1: the workspace already holds the plan for this
                                  problem, mask and order (bsa_plan_build or an
                                  earlier fwd/bwd call); 0: build it first          */
  int32_t bound_ready;         /* fixed-m only. 1: the workspace already holds
                                  kmax/qmax/gate from bsa_fixed_m_bound for these
                                  q and k; 0: bsa_attn_fwd computes them first      */
  int32_t bound_mode;          /* BSA_BOUND_*; SMOOTHED with kmax_override or with
                                  H_kv*D > 24576 is rejected                        */
  int32_t o_residual;          /* BSA_O_RESIDUAL_*: the bf16 rounding residual of O
                                  (fp32 O - bf16 O, one byte per element: an
                                  e5m2 of the residual times 2^12), with which
                                  the backward's Delta = rowsum(dO o O) uses O
                                  at ~11 significant bits instead of the bf16
                                  output's 8.  AUTO (0) applies it whenever a
                                  backward shares the forward's workspace; see
                                  below.                                       */
} bsa_options;

/* bsa_options.o_residual.
 *   AUTO  bsa_attn_fwd writes the residual into the backward part of the
 *         workspace when ws_bytes covers a backward (bsa_workspace_size with
 *         with_backward = 1), and records the `out` pointer it belongs to in
 *         the workspace header; otherwise it records none.  bsa_attn_bwd /
 *         bsa_bwd_preprocess use the residual when the header's record names
 *         the same `out` pointer (a check made on the device, so no
 *         synchronisation), else Delta comes from the bf16 O.  bsa_plan_build
 *         clears the record.  The backward assumes `out` still holds what that
 *         forward wrote, as any attention backward does.
 *   KEEP  as AUTO, but the forward requires a workspace sized with_backward
 *         (else BSA_ERR_WORKSPACE_TOO_SMALL).
 *   DROP  no residual: the forward writes none (and clears the record), the
 *         backward takes Delta from the bf16 O.  Saves one O-sized write and
 *         read per step; Delta then carries the output's rounding, which on
 *         rows with very few allowed keys moves dQ / dK by up to ~1e-2. */
#define BSA_O_RESIDUAL_AUTO 0
#define BSA_O_RESIDUAL_KEEP 1
#define BSA_O_RESIDUAL_DROP 2


/* Where the plan and the scratch arrays sit inside the workspace (byte offsets),
 * for inspection and tests.  Filled by bsa_workspace_layout. */
typedef struct bsa_workspace_view {
  size_t total_bytes;          /* forward + backward workspace                       */
  size_t fwd_bytes;            /* enough for bsa_plan_build + bsa_attn_fwd           */
  size_t off_status;           /* uint32 sticky status word                          */
  size_t off_tile_class;       /* uint8  [B, nM, nN]  BSA_TILE_*                     */
  size_t off_rank;             /* int32  [B, nM, nN]  rank(m, n), -1 where EMPTY     */
  size_t off_row_ptr;          /* int32  [B*nM + 1]   row CSR offsets                */
  size_t off_row_ent;          /* int32  [nnz]        n | FULL << 30, ascending n    */
  size_t off_col_ptr;          /* int32  [B*nN + 1]   column CSR offsets             */
  size_t off_col_ent;          /* int32  [nnz]        m | FULL << 30, (rank, m) order */
  size_t off_col_rank;         /* int32  [nnz]        rank of each column entry      */
  size_t off_perm;             /* int32  [nN]         pi                             */
  size_t off_kmax;             /* fp32   [B, H]       fixed-m key-norm bound          */
  size_t off_qmax;             /* fp32   [B, H]       max query norm                 */
  size_t off_gate;             /* int32  [B, H]       1 = fixed-m, 0 = online        */
  size_t off_delta;            /* fp32   [B, H, nM*128]  backward Delta              */
  size_t off_dq_accum;         /* fp32   backward dQ accumulator                     */
  size_t off_sem;              /* int32  [B, H, nM, 4] dQ semaphores, one per 32-row
                                  quarter of each q-block                          */
  size_t off_kbar;             /* fp32   [B, H_kv, D] k-smoothing center             */
  size_t off_qdot;             /* fp32   [B, H, Sq]   q_i . center                   */
  size_t off_o_resid;          /* u8     [B, Sq, H, D] O - bf16(O) (o_residual)       */
  size_t off_kblk;             /* fp32   [B, H_kv, nN] per kv block max ||k_j|| (BLOCK) */
  size_t off_kmax_q;           /* fp32   [B, H, nM]   per q-block kmax (BLOCK)         */
  int32_t nM, nN;
} bsa_workspace_view;

/* Bytes of workspace a problem needs.  with_backward = 0 sizes the forward
 * only (plan + fixed-m bound); 1 adds Delta, the fp32 dQ accumulator and the
 * semaphores.  Pure host arithmetic; no CUDA call.
 * Errors: INVALID_ARG (null prob or bytes, a size or stride out of range, an
 * inconsistent mask spec), UNSUPPORTED (D not 64/128, a stride not a multiple
 * of 8 elements, a sequence over 2^21, a map over 2^30 tiles). */
BSA_API bsa_status bsa_workspace_size(const bsa_problem *prob, const bsa_mask_spec *mask,
                              int32_t with_backward, size_t *bytes);

/* Offsets of the plan and scratch arrays inside the workspace (host only).
 * Errors as for bsa_workspace_size. */
BSA_API bsa_status bsa_workspace_layout(const bsa_problem *prob, const bsa_mask_spec *mask,
                                bsa_workspace_view *view);

/* Block map and backward schedule (steps a1 and a6 of the hot path): tile
 * classes from the mask predicates, row lists for the forward, rank(m, n)
 * under the order pi and the rank-sorted column lists for the backward.
 * Runs as CUDA kernels on `stream`; resets the sticky status word. */
BSA_API bsa_status bsa_plan_build(const bsa_problem *prob, const bsa_mask_spec *mask,
                          const bsa_options *opt, void *ws, size_t ws_bytes,
                          bsa_stream_t stream);

/* Forward (step a3; "Fixed-m softmax ...", introduction and "Notes"): out
 * (bf16, o_stride layout) and lse (fp32 [B,H,Sq]).  With
 * BSA_SOFTMAX_FIXED_M_GATED it first computes kmax/qmax/gate per (b, h) and
 * runs the fixed-m body on heads that pass the gate, online softmax on the
 * others.  Rows in the varlen alignment tail are written as 0 / -inf.
 * Builds the plan first unless opt->plan_ready (the workspace then holds one
 * built for this problem, mask and order, which a signature check enforces).
 * Errors: INVALID_ARG (a null tensor or workspace, a workspace not 256-byte
 * aligned, an invalid option), UNSUPPORTED (a tensor not 16-byte aligned, lse
 * not 4-byte aligned, or as for bsa_workspace_size), WORKSPACE_TOO_SMALL,
 * NO_DEVICE (no sm_100 device current), CUDA (a launch failed). */
BSA_API bsa_status bsa_attn_fwd(const bsa_problem *prob, const bsa_mask_spec *mask,
                        const bsa_options *opt, const void *q, const void *k,
                        const void *v, void *out, float *lse, void *ws,
                        size_t ws_bytes, bsa_stream_t stream);

/* Backward (steps a4, a5, a7; "Add more optimal dk order optional arg", "What
 * does this do" and "Sliding window perf issue"): dq, dk, dv (bf16, q_stride /
 * k_stride / v_stride layouts) from q, k, v, the forward's out and lse and the
 * incoming gradient dout.  deterministic = 1 orders every dQ contribution by
 * the dQ semaphores (bit-identical results run to run); 0 uses atomic adds.
 * Needs a workspace sized with with_backward = 1.  Errors as for bsa_attn_fwd;
 * a semaphore wait that gives up is reported by bsa_get_device_status as
 * BSA_ERR_SEM_TIMEOUT. */
BSA_API bsa_status bsa_attn_bwd(const bsa_problem *prob, const bsa_mask_spec *mask,
                        const bsa_options *opt, const void *q, const void *k,
                        const void *v, const void *out, const void *dout,
                        const float *lse, void *dq, void *dk, void *dv, void *ws,
                        size_t ws_bytes, bsa_stream_t stream);

/* The stages of the hot path, one call each, for callers that schedule or time
 * them separately.  bsa_attn_fwd = [bsa_plan_build] + [bsa_fixed_m_bound] (both
 * at once as bsa_plan_and_bound when both are needed) + forward kernel; bsa_attn_bwd = [bsa_plan_build] + bsa_bwd_preprocess +
 * bsa_bwd_main + bsa_bwd_convert.  Each expects the workspace state the
 * previous stage leaves; arguments as for bsa_attn_fwd / bsa_attn_bwd. */

/* a2 ("Fixed-m softmax ...", introduction and "Notes"): kmax[b,h] = max over
 * valid keys of ||k_j|| (or opt->kmax_override), qmax[b,h] and per-row ||q_i||,
 * gate[b,h] = 2*scale*qmax*kmax <= G, all into the workspace. */
BSA_API bsa_status bsa_fixed_m_bound(const bsa_problem *prob, const bsa_mask_spec *mask,
                                     const bsa_options *opt, const void *q, const void *k,
                                     void *ws, size_t ws_bytes, bsa_stream_t stream);

/* a1 + a2 together: the block-map plan (as bsa_plan_build) and the fixed-m bound
 * (as bsa_fixed_m_bound), the result identical to calling the two in turn.  For
 * every mask but BSA_MASK_VARLEN (whose key validity the bound reads from the
 * plan) the planner runs on a non-blocking stream of the library's own, created
 * once per device (with a fork / join event pair per host thread, created on
 * first use), concurrently with the bound's pass over Q and K on `stream`:
 * the side stream waits for an event recorded on `stream` and `stream` waits for
 * the planner before the call returns, so all later work on `stream` sees both
 * results, and a stream capture on `stream` records the same fork and join.
 * bsa_attn_fwd takes this path when it has to build both.  Arguments and errors
 * as for bsa_fixed_m_bound (q, k device pointers, 16-byte aligned). */
BSA_API bsa_status bsa_plan_and_bound(const bsa_problem *prob, const bsa_mask_spec *mask,
                                      const bsa_options *opt, const void *q, const void *k,
                                      void *ws, size_t ws_bytes, bsa_stream_t stream);

/* a4: Delta_i = sum_d dO_id O_id (fp32) into the workspace (with the O
 * residual per opt->o_residual); zeroes the dQ semaphores (and, for the atomic
 * backward, the fp32 dQ accumulator); writes fp16 copies of q and dout into the
 * workspace, on which bsa_bwd_main takes its products (values beyond the fp16
 * range are reported as BSA_ERR_INPUT_RANGE). */
BSA_API bsa_status bsa_bwd_preprocess(const bsa_problem *prob, const bsa_mask_spec *mask,
                                      const bsa_options *opt, const void *q, const void *out,
                                      const void *dout, void *ws, size_t ws_bytes,
                                      bsa_stream_t stream);

/* a5 ("Add more optimal dk order optional arg", "Sliding window perf issue"):
 * dK, dV written (bf16); dQ contributions accumulated into the workspace in
 * the order pi when opt->deterministic.  Reads Q and dO from the fp16 copies
 * bsa_bwd_preprocess left in the workspace (q and dout are checked as usual),
 * K and V from k and v. */
BSA_API bsa_status bsa_bwd_main(const bsa_problem *prob, const bsa_mask_spec *mask,
                                const bsa_options *opt, const void *q, const void *k,
                                const void *v, const void *dout, const float *lse, void *dk,
                                void *dv, void *ws, size_t ws_bytes, bsa_stream_t stream);

/* a7: dQ = bf16(dQ accumulator); zero rows for q-blocks no kv column reaches.
 * After a semaphore-ordered bsa_bwd_main on the same stream, the blocks may
 * start while that kernel's last columns still run: each converts its 32 rows
 * once their dQ semaphore counts every contribution of the row list.  The
 * call's work still completes only after bsa_bwd_main's. */
BSA_API bsa_status bsa_bwd_convert(const bsa_problem *prob, const bsa_mask_spec *mask,
                                   void *dq, void *ws, size_t ws_bytes, bsa_stream_t stream);

/* Forward for callers that cannot allocate device memory: plugin code run by a
 * host framework that owns every device allocation and forbids cudaMalloc inside
 * its execution callback, or code that must not risk the implicit device-wide
 * synchronisation cudaMalloc / cudaFree may perform.  Same computation and
 * arguments as bsa_attn_fwd (inputs and outputs still come from the caller), but
 * no workspace: the plan and the fixed-m bound live in a fixed 32 MiB device
 * array inside the library, which every GPU that loads the library holds until
 * the process exits.  The source pages have no counterpart to this; it is a
 * deployment convenience.
 *  - Problems whose forward workspace (bsa_workspace_size, with_backward = 0)
 *    exceeds 32 MiB are rejected with BSA_ERR_WORKSPACE_TOO_SMALL before any
 *    launch.
 *  - No cudaMalloc, cudaFree or other allocating call is made (the plan and the
 *    bound run one after the other on `stream`, never on the library's side
 *    stream, so no stream or event is created either).  The first use on each
 *    device looks up the array's device address (with that device current),
 *    which under lazy module loading is also when the driver loads this
 *    library's device code and places the array: call bsa_static_scratch_init
 *    once per device before any stream capture or allocation-free section.
 *    The looked-up address is kept; after cudaDeviceReset on a device, this
 *    entry point must not be used there again in the same process.
 *  - Every call shares the one array and rebuilds the plan in it, so calls
 *    whose work overlaps on the GPU (different streams, or concurrent host
 *    threads) race and must be serialised by the caller.
 *  - opt->plan_ready and opt->bound_ready are ignored, and the O residual is
 *    never kept (no backward shares this array).  Device-side errors (a bad
 *    cu_seqlens, a bounded wait that gave up) land in the array's sticky status
 *    word: read it with bsa_static_scratch_status.  Argument errors are
 *    returned as usual. */
BSA_API bsa_status bsa_attn_fwd_static_scratch(const bsa_problem *prob,
                                               const bsa_mask_spec *mask,
                                               const bsa_options *opt, const void *q,
                                               const void *k, const void *v, void *out,
                                               float *lse, bsa_stream_t stream);

/* The allocation-free forward's set-up on the current device: looks up the
 * static array's device address (loading the library's device code there if
 * the driver loads it lazily).  Call once per device before the first
 * bsa_attn_fwd_static_scratch inside a stream capture or any section that must
 * not allocate.  No counterpart in the pages.  Errors: NO_DEVICE, CUDA. */
BSA_API bsa_status bsa_static_scratch_init(void);

/* Synchronises `stream`, then returns the sticky device status of the static
 * array bsa_attn_fwd_static_scratch uses on the current device: BSA_OK unless
 * the most recent such call recorded a device-side error (every call rebuilds
 * the plan in the array, which resets the word).  clear = 1 resets it.
 * Allocates nothing.  No counterpart in the pages.  Errors: NO_DEVICE, CUDA. */
BSA_API bsa_status bsa_static_scratch_status(bsa_stream_t stream, int32_t clear);

/* Synchronises `stream`, then returns the sticky device status of `ws`
 * (BSA_OK if no device-side error was recorded); clear = 1 resets it. */
BSA_API bsa_status bsa_get_device_status(void *ws, size_t ws_bytes, bsa_stream_t stream,
                                 int32_t clear);

/* Number of query rows that the forwards on `ws` since its last plan build
 * ran with the pinned fixed-m reference (rows of heads, q-blocks or, with
 * BSA_BOUND_BLOCK, single rows that passed the gate); the rest ran online
 * softmax.  Synchronises `stream`, like bsa_get_device_status.  Errors:
 * INVALID_ARG (null or too small a workspace), CUDA. */
BSA_API bsa_status bsa_fixed_rows(void *ws, size_t ws_bytes, bsa_stream_t stream, uint64_t *rows);

/* Static description of a status code. */
BSA_API const char *bsa_status_string(bsa_status status);

/* Number of this library's kernel launches issued by the whole process since
 * the library was loaded (all threads; for the bench's launch count). */
BSA_API uint64_t bsa_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* BSA_H_ */
