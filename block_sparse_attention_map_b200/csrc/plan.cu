// Block-map planner: steps a1 (tile classes from the mask predicates) and a6
// (kv-column order pi, rank(m, n), rank-sorted column lists) of the hot path.
//
// Sources: "Let splash attention exceed 524,288 tokens when packing is off"
// (maxtext PR #4929) for the segment-id mask and the block mask it implies;
// maxdiffusion PR #404 review for global KV padding; sglang PR #47566
// ("Modifications") for varlen alignment rows; "Add more optimal dk order
// optional arg" (flash-attention PR #2512, "Sliding window perf issue" and "A
// simplish fix") for rank(m, n), the kv-column orders and the unified column
// list walked in rank order; its benchmark ("The numbers") names the
// outside_in and greedy orders and the prefix_lm, dilated_sliding_window and
// document masks, whose readings are stated where they are built.
//
// The block map is shared by every head (masks are head independent) and kept
// as compact CSR lists, so its size is O(non-empty tiles) per batch row plus
// one byte per tile for the dense class array.
#include "internal.h"
#include "ptx.cuh"

namespace bsa {
namespace {

// Varlen: validate cu_seqlens and expand it into per-position segment ids;
// alignment rows get -1 (query side) / -2 (key side) so they match nothing.
__global__ void k_varlen_expand(const int32_t *__restrict__ cu, int n_seqs, int n_align_tail,
                                int T, int32_t *__restrict__ seg_q, int32_t *__restrict__ seg_kv,
                                uint32_t *status) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i == 0) {
    bool ok = cu[0] == 0 && cu[n_seqs] == T;
    for (int s = 0; s < n_seqs; ++s) ok = ok && cu[s] <= cu[s + 1];
    if (!ok) record_status(status, BSA_ERR_BAD_MASK_DATA);
  }
  if (i >= T) return;
  int lo = 0, hi = n_seqs;  // find s with cu[s] <= i < cu[s+1]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (cu[mid] <= i) lo = mid; else hi = mid;
  }
  const bool align = lo >= n_seqs - n_align_tail;
  seg_q[i] = align ? -1 : lo;
  seg_kv[i] = align ? -2 : lo;
}

// The planner's first launch with segment or varlen ids: the per-block
// summaries of both id arrays (a warp per block, q blocks first), and the row
// and column counts (and, unless hdr is null, the plan's header words) zeroed,
// in one grid rather than two summary launches and three memsets.  A summary
// is [min, max, #positions with a real id, #alignment positions] over the
// in-range positions of the block; with neg_is_align (varlen) negative ids
// mark alignment positions, while caller-supplied segment ids may take any
// int32 value.
__global__ void k_plan_prep(const int32_t *__restrict__ seg_q, const int32_t *__restrict__ seg_kv,
                            int Sq, int Skv, int nM, int nN, int B, int64_t bq, int64_t bk,
                            int neg_is_align, int4 *__restrict__ qb, int4 *__restrict__ kb,
                            uint32_t *__restrict__ hdr, int32_t *__restrict__ row_cnt,
                            int32_t *__restrict__ col_cnt) {
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t nthr = static_cast<int64_t>(gridDim.x) * blockDim.x;
  if (hdr != nullptr && tid < kHdrPlanWords) hdr[tid] = 0u;  // null: reset by the caller already
  for (int64_t i = tid; i < static_cast<int64_t>(B) * nM; i += nthr) row_cnt[i] = 0;
  for (int64_t i = tid; i < static_cast<int64_t>(B) * nN; i += nthr) col_cnt[i] = 0;
  const int warp = static_cast<int>(tid >> 5);
  const int lane = threadIdx.x & 31;
  const int nq = B * nM;
  if (warp >= nq + B * nN) return;
  const bool is_q = warp < nq;
  const int blk = is_q ? warp : warp - nq, nb = is_q ? nM : nN, S = is_q ? Sq : Skv;
  const int b = blk / nb, j = blk % nb;
  const int32_t *seg = is_q ? seg_q : seg_kv;
  const int64_t bs = is_q ? bq : bk;
  int mn = 0x7fffffff, mx = -0x7fffffff - 1, nreal = 0, nbad = 0;
  for (int t = lane; t < kTile; t += 32) {
    const int i = j * kTile + t;
    if (i >= S) break;
    const int v = seg[b * bs + i];
    if (neg_is_align && v < 0) { ++nbad; continue; }
    mn = min(mn, v);
    mx = max(mx, v);
    ++nreal;
  }
  for (int o = 16; o > 0; o >>= 1) {
    mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    nreal += __shfl_xor_sync(0xffffffffu, nreal, o);
    nbad += __shfl_xor_sync(0xffffffffu, nbad, o);
  }
  if (lane == 0) (is_q ? qb : kb)[blk] = make_int4(mn, mx, nreal, nbad);
}

struct ClassifyArgs {
  int B, nM, nN, Sq, Skv;
  uint32_t flags;
  int window, dilation;
  const int32_t *kv_valid_len;
  const int32_t *prefix_len;       // null unless BSA_MASK_PREFIX_LM
  const int4 *qblk, *kblk;         // null unless segment ids / varlen
  const int32_t *seg_q, *seg_kv;   // the ids the kernels compare (null: none)
  int64_t seg_q_bstride, seg_kv_bstride;
  uint8_t *cls;
  int32_t *row_cnt, *col_cnt;
};

// Tile class of (b, m, n): the AND-combination of one class per enabled
// predicate (EMPTY if any predicate is empty, FULL if all are full).  The
// window (with its prefix and its dilation), padding and out-of-range columns
// are classified exactly over the tile's in-range rows and columns, in closed
// form; segment ids only through bounds (per-block [min, max] id intervals).
// *exact is cleared when the PARTIAL answer may be wrong: a bound-only
// predicate, or two predicates that are each partial (their allowed parts may
// not meet).
__device__ __forceinline__ uint8_t tile_class(const ClassifyArgs &a, int b, int m, int n,
                                              bool *exact) {
  const int i0 = m * kTile, i1 = min(a.Sq, i0 + kTile) - 1;
  const int j0 = n * kTile, jv1 = min(a.Skv, j0 + kTile) - 1;
  uint8_t c = BSA_TILE_FULL;
  int npartial = 0;
  bool bound_only = false;
  if (j0 + kTile - 1 > jv1) c = BSA_TILE_PARTIAL;  // out-of-range keys must be masked
  if (a.flags & BSA_MASK_CAUSAL_WINDOW) {
    const int o = a.Skv - a.Sq, W = a.window;
    const int P = a.prefix_len != nullptr ? a.prefix_len[b] : 0;
    // the band i+o-W < j <= i+o over columns [ja, jv1]
    auto band_any = [&](int ja) {
      return ja <= jv1 && ja <= i1 + o && (W == 0 || jv1 >= i0 + o - W + 1);
    };
    auto band_all = [&](int ja) {
      return ja > jv1 || (jv1 <= i0 + o && (W == 0 || ja >= i1 + o - W + 1));
    };
    const bool pre_all = jv1 < P, pre_any = j0 < P;
    const int ja = max(j0, P);  // first column the prefix does not cover
    const bool any = pre_any || band_any(j0);
    bool all = pre_all || band_all(ja);
    if (!any) return BSA_TILE_EMPTY;
    if (a.dilation > 1 && !pre_all) {
      // the dilated band over the columns the prefix does not cover: every
      // distance t = i + o - j in [i0 + o - jv1, i1 + o - ja] occurs in the
      // tile (i and j each run over a range), so the tile holds a kept key iff
      // that range cut to the band [0, W) holds a multiple of d; it is never
      // full unless that part is a single element, which is checked element
      // by element
      bool dil_any = false;
      if (ja <= jv1) {
        const int d = a.dilation;
        const int lo = max(i0 + o - jv1, 0);
        const int hi = W > 0 ? min(i1 + o - ja, W - 1) : i1 + o - ja;
        dil_any = lo <= hi && (hi / d) * d >= lo;
      }
      if (!pre_any && !dil_any) return BSA_TILE_EMPTY;
      all = false;
      if (i0 == i1 && ja == jv1) bound_only = true;
    }
    if (!all) {
      c = BSA_TILE_PARTIAL;
      ++npartial;
    }
  }
  if (a.flags & BSA_MASK_KV_VALID_LEN) {
    const int L = a.kv_valid_len[b];
    if (j0 >= L) return BSA_TILE_EMPTY;
    if (jv1 >= L) {
      c = BSA_TILE_PARTIAL;
      ++npartial;
    }
  }
  if (a.qblk != nullptr) {
    const int4 q = a.qblk[b * a.nM + m];
    const int4 k = a.kblk[b * a.nN + n];
    if (q.z == 0 || k.z == 0 || q.y < k.x || k.y < q.x) return BSA_TILE_EMPTY;
    const bool one = q.x == q.y && k.x == k.y && q.x == k.x && q.w == 0 && k.w == 0;
    if (!one) {
      c = BSA_TILE_PARTIAL;
      bound_only = true;
    }
  }
  *exact = !bound_only && npartial <= 1;
  return c;
}

// allowed(i, j) for one in-range element, every enabled predicate: the
// element-level definition the kernels apply on PARTIAL tiles.
__device__ __forceinline__ bool allowed_elem(const ClassifyArgs &a, int b, int i, int j,
                                             int seg_i, int seg_j, int P, int L) {
  if (j >= L) return false;
  if (a.seg_q != nullptr && seg_i != seg_j) return false;
  if (a.flags & BSA_MASK_CAUSAL_WINDOW) {
    if (j < P) return true;
    const int t = i + (a.Skv - a.Sq) - j;
    if (t < 0 || (a.window > 0 && t >= a.window)) return false;
    if (a.dilation > 1 && t % a.dilation != 0) return false;
  }
  return true;
}

// Exact class of tile (b, m, n) by the whole warp, element by element: lane l
// takes columns l, l+32, l+64, l+96 of the tile and the warp walks the rows
// from both ends inwards (first, last, second, second-to-last, ...), stopping
// as soon as it has seen one allowed and one masked element (the tile is
// PARTIAL then, whatever the remaining rows hold): most tiles the bounds leave
// open settle within their first rows, including those whose rows change
// segment near one end (a varlen alignment tail, a document boundary).
__device__ uint8_t refine_tile(const ClassifyArgs &a, int b, int m, int n, int lane) {
  const int i0 = m * kTile, i1 = min(a.Sq, i0 + kTile) - 1;
  const int P = a.prefix_len != nullptr ? a.prefix_len[b] : 0;
  const int L = min((a.flags & BSA_MASK_KV_VALID_LEN) ? a.kv_valid_len[b] : a.Skv, a.Skv);
  bool any = false, all = true;
  int jj[4], sj[4];
  bool in[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    jj[c] = n * kTile + lane + 32 * c;
    in[c] = jj[c] < a.Skv;
    if (!in[c]) all = false;
    sj[c] = (a.seg_kv != nullptr && in[c]) ? a.seg_kv[b * a.seg_kv_bstride + jj[c]] : 0;
  }
  const int rows = i1 - i0 + 1;
#pragma unroll 1
  for (int k = 0; k < rows; ++k) {
    const int i = (k & 1) ? i1 - (k >> 1) : i0 + (k >> 1);
    const int seg_i = a.seg_q != nullptr ? a.seg_q[b * a.seg_q_bstride + i] : 0;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      if (!in[c]) continue;
      const bool ok = allowed_elem(a, b, i, jj[c], seg_i, sj[c], P, L);
      any |= ok;
      all &= ok;
    }
    // k runs over the same rows in every lane: the votes are warp-uniform
    if ((k & 3) == 3 && __any_sync(0xffffffffu, any) && !__all_sync(0xffffffffu, all))
      return BSA_TILE_PARTIAL;
  }
  any = __any_sync(0xffffffffu, any);
  all = __all_sync(0xffffffffu, all);
  return all ? BSA_TILE_FULL : (any ? BSA_TILE_PARTIAL : BSA_TILE_EMPTY);
}

// One warp per (b, m, 32 consecutive columns): classify those tiles (tiles the
// bounds cannot settle are classified element by element by the whole warp),
// and add the non-empty ones to their row's and columns' counts (zeroed
// before; order-independent integer sums).  A row with many tiles to refine
// (the boundary block of a varlen alignment tail meets every column) spreads
// over as many warps as it has column chunks.
__global__ void k_classify_chunks(ClassifyArgs a) {
  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int chunks = (a.nN + 31) >> 5;
  if (wid >= static_cast<int64_t>(a.B) * a.nM * chunks) return;
  const int row_id = static_cast<int>(wid / chunks), n0 = static_cast<int>(wid % chunks) * 32;
  const int b = row_id / a.nM, m = row_id % a.nM;
  uint8_t *row = a.cls + static_cast<int64_t>(row_id) * a.nN;
  const int n = n0 + lane;
  uint8_t c = BSA_TILE_EMPTY;
  bool exact = true;
  if (n < a.nN) c = tile_class(a, b, m, n, &exact);
  uint32_t todo = __ballot_sync(0xffffffffu, c == BSA_TILE_PARTIAL && !exact);
  while (todo != 0u) {
    const int src = __ffs(todo) - 1;
    todo &= todo - 1u;
    const uint8_t rc = refine_tile(a, b, m, n0 + src, lane);
    if (lane == src) c = rc;
  }
  if (n < a.nN) {
    row[n] = c;
    if (c != BSA_TILE_EMPTY) atomicAdd(a.col_cnt + b * a.nN + n, 1);
  }
  const int cnt = __popc(__ballot_sync(0xffffffffu, c != BSA_TILE_EMPTY));
  if (lane == 0 && cnt != 0) atomicAdd(a.row_cnt + row_id, cnt);
}

// Exclusive scans of row and column counts into CSR offsets (block 0: rows,
// block 1: columns); ptr[count] receives the total.  Block 0 then writes the
// plan signature that the forward and backward kernels check.
__global__ void k_scan2(const int32_t *__restrict__ c0, int32_t *__restrict__ p0, int n0,
                        const int32_t *__restrict__ c1, int32_t *__restrict__ p1, int n1,
                        uint32_t *hdr, uint32_t B, uint32_t Sq, uint32_t Skv, uint32_t flags,
                        uint32_t window, uint32_t order, uint32_t n_seqs, uint32_t dilation) {
  const int32_t *c = blockIdx.x == 0 ? c0 : c1;
  int32_t *p = blockIdx.x == 0 ? p0 : p1;
  const int n = blockIdx.x == 0 ? n0 : n1;
  __shared__ int32_t warp_tot[32];
  __shared__ int32_t carry;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < n; base += 1024) {
    const int i = base + threadIdx.x;
    const int32_t v = i < n ? c[i] : 0;
    int32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[wid] = x;
    __syncthreads();
    if (wid == 0) {
      int32_t t = warp_tot[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, t, o);
        if (lane >= o) t += y;
      }
      warp_tot[lane] = t;  // inclusive over warps
    }
    __syncthreads();
    const int32_t before = (wid > 0 ? warp_tot[wid - 1] : 0) + carry;
    if (i < n) p[i] = before + x - v;
    __syncthreads();
    if (threadIdx.x == 0) carry += warp_tot[31];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    p[n] = carry;
    if (blockIdx.x == 0) {
      hdr[kHdrB] = B;
      hdr[kHdrSq] = Sq;
      hdr[kHdrSkv] = Skv;
      hdr[kHdrFlags] = flags;
      hdr[kHdrWindow] = window;
      hdr[kHdrOrder] = order;
      hdr[kHdrNSeqs] = n_seqs;
      hdr[kHdrDilation] = dilation;
      __threadfence();
      hdr[kHdrMagic] = kPlanMagic;
    }
  }
}

// pi[t] for the orders with a closed form: ascending, descending, and
// outside-in (0, nN-1, 1, nN-2, ...).
__device__ __forceinline__ int closed_form_order(int order, int t, int nN) {
  if (order == BSA_ORDER_DESC) return nN - 1 - t;
  if (order == BSA_ORDER_OUTSIDE_IN) return (t & 1) ? nN - 1 - (t >> 1) : (t >> 1);
  return t;
}

__device__ __forceinline__ bool order_in_workspace(int order) {
  return order == BSA_ORDER_PERM || order == BSA_ORDER_GREEDY;
}

// The greedy order, one block: the columns are placed one at a time; w[n] is
// the presumed semaphore wait of column n if it came next, the number of
// (already placed column, row block) pairs that share a non-empty row block
// with it, summed over all batches.  Each step takes the smallest (w[n], n)
// among the unplaced columns, then adds one to w[n'] for every unplaced n'
// per row block the placed column reaches (a warp per row block).
static_assert(sizeof(int32_t) * (kMaxSeq / kTile) <= 64 * 1024,
              "the greedy order keeps one presumed wait per kv block in shared memory");
__global__ void __launch_bounds__(1024) k_greedy_order(const uint8_t *__restrict__ cls, int BnM,
                                                       int nN, int32_t *__restrict__ perm) {
  extern __shared__ int32_t w[];
  __shared__ unsigned long long red[32];
  __shared__ int chosen;
  constexpr int32_t kPlaced = 0x7fffffff;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int n = threadIdx.x; n < nN; n += blockDim.x) w[n] = 0;
  __syncthreads();
  for (int step = 0; step < nN; ++step) {
    unsigned long long best = ~0ull;
    for (int n = threadIdx.x; n < nN; n += blockDim.x) {
      const int32_t x = w[n];
      if (x != kPlaced) {
        const unsigned long long key = (static_cast<unsigned long long>(x) << 32) |
                                       static_cast<unsigned>(n);
        best = key < best ? key : best;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long y = __shfl_xor_sync(0xffffffffu, best, o);
      best = y < best ? y : best;
    }
    if (lane == 0) red[wid] = best;
    __syncthreads();
    if (wid == 0) {
      unsigned long long v = lane < nw ? red[lane] : ~0ull;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const unsigned long long y = __shfl_xor_sync(0xffffffffu, v, o);
        v = y < v ? y : v;
      }
      if (lane == 0) {
        const int c = static_cast<int>(v & 0xffffffffull);
        chosen = c;
        perm[step] = c;
        w[c] = kPlaced;
      }
    }
    __syncthreads();
    const int c = chosen;
    for (int bm = wid; bm < BnM; bm += nw) {
      const uint8_t *row = cls + static_cast<int64_t>(bm) * nN;
      if (row[c] == BSA_TILE_EMPTY) continue;
      for (int n = lane; n < nN; n += 32)
        if (row[n] != BSA_TILE_EMPTY && w[n] != kPlaced) atomicAdd(w + n, 1);
    }
    __syncthreads();
  }
}

// One warp per (b, m): the forward's row list (ascending n, FULL flag in bit
// 30) and rank(m, n): row m's non-empty columns numbered 0, 1, 2, ... in the
// order pi (-1 for empty tiles).  pi has a closed form, or is the caller's
// permutation or the greedy order already in the workspace; warp 0 writes it
// out for the closed forms.
__global__ void k_row_fill(const uint8_t *__restrict__ cls, int BnM, int nN, int order,
                           int32_t *__restrict__ perm, const int32_t *__restrict__ row_ptr,
                           uint32_t *__restrict__ row_ent, int32_t *__restrict__ rank) {
  const int wid = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= BnM) return;
  const uint8_t *row = cls + static_cast<int64_t>(wid) * nN;
  const bool in_ws = order_in_workspace(order);
  if (wid == 0 && !in_ws)
    for (int t = lane; t < nN; t += 32) perm[t] = closed_form_order(order, t, nN);
  int pos = row_ptr[wid];
  for (int n0 = 0; n0 < nN; n0 += 32) {
    const int n = n0 + lane;
    const uint8_t c = n < nN ? row[n] : BSA_TILE_EMPTY;
    const uint32_t bal = __ballot_sync(0xffffffffu, c != BSA_TILE_EMPTY);
    if (c != BSA_TILE_EMPTY)
      row_ent[pos + __popc(bal & ((1u << lane) - 1u))] = n | (c == BSA_TILE_FULL ? kFullBit : 0u);
    pos += __popc(bal);
  }
  int32_t *rk = rank + static_cast<int64_t>(wid) * nN;
  int r = 0;
  for (int t0 = 0; t0 < nN; t0 += 32) {
    const int t = t0 + lane;
    int n = -1;
    if (t < nN) n = in_ws ? perm[t] : closed_form_order(order, t, nN);
    const bool ne = n >= 0 && row[n] != BSA_TILE_EMPTY;
    const uint32_t bal = __ballot_sync(0xffffffffu, ne);
    if (n >= 0) rk[n] = ne ? r + __popc(bal & ((1u << lane) - 1u)) : -1;
    r += __popc(bal);
  }
}

// Column lists for the backward: the unified partial+full list of column n,
// sorted by (rank(m, n), m).  One block per (b, n): the column's entries are
// gathered in ascending m by a block-wide compaction, then each entry's
// position is the number of entries with a smaller key.
__global__ void k_col_fill(const uint8_t *__restrict__ cls, const int32_t *__restrict__ rank,
                           int nM, int nN, const int32_t *__restrict__ col_ptr,
                           uint32_t *__restrict__ col_ent, int32_t *__restrict__ col_rank) {
  extern __shared__ unsigned long long keys[];
  __shared__ int warp_cnt[32];
  __shared__ int base_cnt;
  const int bn = blockIdx.x;
  const int b = bn / nN, n = bn % nN;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  if (threadIdx.x == 0) base_cnt = 0;
  __syncthreads();
  for (int m0 = 0; m0 < nM; m0 += blockDim.x) {
    const int m = m0 + threadIdx.x;
    unsigned long long key = 0;
    bool ne = false;
    if (m < nM) {
      const int64_t t = (static_cast<int64_t>(b) * nM + m) * nN + n;
      const uint8_t k = cls[t];
      ne = k != BSA_TILE_EMPTY;
      if (ne)
        key = (static_cast<unsigned long long>(rank[t]) << 32) |
              (static_cast<unsigned long long>(m) << 1) | (k == BSA_TILE_FULL ? 1ull : 0ull);
    }
    const uint32_t bal = __ballot_sync(0xffffffffu, ne);
    if (lane == 0) warp_cnt[wid] = __popc(bal);
    __syncthreads();
    int before = base_cnt;
    for (int w = 0; w < wid; ++w) before += warp_cnt[w];
    if (ne) keys[before + __popc(bal & ((1u << lane) - 1u))] = key;
    __syncthreads();
    if (threadIdx.x == 0)
      for (int w = 0; w < nw; ++w) base_cnt += warp_cnt[w];
    __syncthreads();
  }
  const int c = base_cnt;
  const int base = col_ptr[bn];
  for (int e = threadIdx.x; e < c; e += blockDim.x) {
    const unsigned long long ke = keys[e];
    int pos = 0;
    for (int f = 0; f < c; ++f) pos += keys[f] < ke;
    const uint32_t m = static_cast<uint32_t>((ke & 0xffffffffull) >> 1);
    col_ent[base + pos] = m | ((ke & 1ull) ? kFullBit : 0u);
    col_rank[base + pos] = static_cast<int32_t>(ke >> 32);
  }
}

// Exclusive scan of n counts in shared memory into out[0..n] (out[n] = total),
// by the whole block: each thread sums a contiguous run, the runs' sums are
// scanned across the block, then each thread writes its run's offsets.
__device__ void block_scan_to(const int32_t *cnt, int n, int32_t *out, int32_t *scratch,
                              int32_t *out_s = nullptr) {
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int lo = min(n, static_cast<int>(threadIdx.x) * per), hi = min(n, lo + per);
  int32_t run = 0;
  for (int i = lo; i < hi; ++i) run += cnt[i];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int32_t x = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scratch[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int32_t t = lane < static_cast<int>(blockDim.x >> 5) ? scratch[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    scratch[lane] = t;  // inclusive over warps
  }
  __syncthreads();
  int32_t acc = (wid > 0 ? scratch[wid - 1] : 0) + x - run;
  for (int i = lo; i < hi; ++i) {
    out[i] = acc;
    if (out_s != nullptr) out_s[i] = acc;
    acc += cnt[i];
  }
  if (threadIdx.x == blockDim.x - 1) {
    out[n] = acc;
    if (out_s != nullptr) out_s[n] = acc;
  }
  __syncthreads();
}

// Offsets (in int32 words) of k_plan_fused's shared-memory arrays.
struct FusedPlanSmem {
  int rcnt, ccnt, scratch, gw, rptr, cptr, rank, cls, keys;
  __host__ __device__ FusedPlanSmem(int B, int nM, int nN) {
    const int BnM = B * nM, BnN = B * nN;
    rcnt = 0;
    ccnt = rcnt + BnM;
    scratch = ccnt + BnN;
    gw = scratch + 32;
    rptr = gw + nN;
    cptr = rptr + BnM + 1;
    rank = cptr + BnN + 1;
    cls = rank + BnM * nN;
    keys = (cls + (BnM * nN + 3) / 4 + 1) & ~1;  // 8-byte boundary for the u64 keys
  }
};

struct FusedPlanArgs {
  ClassifyArgs ca;  // row_cnt / col_cnt unused: the counts live in shared memory
  int order;
  int32_t *perm, *rank, *row_ptr, *col_ptr, *col_rank;
  uint32_t *row_ent, *col_ent, *hdr;
  uint32_t sig_flags, sig_window, sig_n_seqs, sig_dilation;
};

// The whole plan in one block, for small block maps without segment or varlen
// ids: header reset, tile classes with row and column counts, both CSR scans,
// pi (closed form or greedy), the row lists with rank(m, n), and the column
// lists sorted by (rank, m) (a warp per column, ranking its entries in shared
// memory).  Same results as the multi-kernel path.  The tile classes, ranks
// and CSR offsets the later phases read stay in shared memory (their global
// copies are written, never read back): the phases do not wait on global
// round trips, which another kernel streaming through HBM beside the planner
// would lengthen.  Held to 32 registers per thread (1024 x 32 = half an SM's
// registers) so that it fits on an SM beside the fixed-m bound's blocks, which
// run concurrently on the caller's stream.
__global__ void __launch_bounds__(1024, 2) k_plan_fused(FusedPlanArgs pa) {
  extern __shared__ int32_t shm[];
  const ClassifyArgs &a = pa.ca;
  const int B = a.B, nM = a.nM, nN = a.nN, BnM = B * nM, BnN = B * nN;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const FusedPlanSmem F(B, nM, nN);
  int32_t *rcnt = shm + F.rcnt;        // [BnM]
  int32_t *ccnt = shm + F.ccnt;        // [BnN]
  int32_t *scratch = shm + F.scratch;  // [32]
  int32_t *gw = shm + F.gw;            // [nN] greedy presumed waits
  int32_t *rptr = shm + F.rptr;        // [BnM + 1]
  int32_t *cptr = shm + F.cptr;        // [BnN + 1]
  int32_t *rank_s = shm + F.rank;      // [BnM * nN]
  uint8_t *cls_s = reinterpret_cast<uint8_t *>(shm + F.cls);  // [BnM * nN]
  unsigned long long *keys = reinterpret_cast<unsigned long long *>(shm + F.keys);  // [nw][nM]
  if (threadIdx.x < kHdrPlanWords) pa.hdr[threadIdx.x] = 0u;
  for (int i = threadIdx.x; i < BnN; i += blockDim.x) ccnt[i] = 0;
  __syncthreads();
  // tile classes, a warp per row block
  for (int row = wid; row < BnM; row += nw) {
    const int b = row / nM, m = row % nM;
    uint8_t *crow = a.cls + static_cast<int64_t>(row) * nN;
    int cnt = 0;
    for (int n0 = 0; n0 < nN; n0 += 32) {
      const int n = n0 + lane;
      uint8_t c = BSA_TILE_EMPTY;
      bool exact = true;
      if (n < nN) c = tile_class(a, b, m, n, &exact);
      uint32_t todo = __ballot_sync(0xffffffffu, c == BSA_TILE_PARTIAL && !exact);
      while (todo != 0u) {
        const int src = __ffs(todo) - 1;
        todo &= todo - 1u;
        const uint8_t rc = refine_tile(a, b, m, n0 + src, lane);
        if (lane == src) c = rc;
      }
      if (n < nN) {
        crow[n] = c;
        cls_s[row * nN + n] = c;
        if (c != BSA_TILE_EMPTY) atomicAdd(ccnt + b * nN + n, 1);
      }
      cnt += __popc(__ballot_sync(0xffffffffu, c != BSA_TILE_EMPTY));
    }
    if (lane == 0) rcnt[row] = cnt;
  }
  __syncthreads();
  block_scan_to(rcnt, BnM, pa.row_ptr, scratch, rptr);
  block_scan_to(ccnt, BnN, pa.col_ptr, scratch, cptr);
  // pi
  const bool in_ws = order_in_workspace(pa.order);
  if (pa.order == BSA_ORDER_GREEDY) {
    constexpr int32_t kPlaced = 0x7fffffff;
    __shared__ unsigned long long red[32];
    __shared__ int chosen;
    for (int n = threadIdx.x; n < nN; n += blockDim.x) gw[n] = 0;
    __syncthreads();
    for (int step = 0; step < nN; ++step) {
      unsigned long long best = ~0ull;
      for (int n = threadIdx.x; n < nN; n += blockDim.x) {
        const int32_t w = gw[n];
        if (w != kPlaced) {
          const unsigned long long key = (static_cast<unsigned long long>(w) << 32) | static_cast<unsigned>(n);
          best = key < best ? key : best;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const unsigned long long y = __shfl_xor_sync(0xffffffffu, best, o);
        best = y < best ? y : best;
      }
      if (lane == 0) red[wid] = best;
      __syncthreads();
      if (wid == 0) {
        unsigned long long v = lane < nw ? red[lane] : ~0ull;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const unsigned long long y = __shfl_xor_sync(0xffffffffu, v, o);
          v = y < v ? y : v;
        }
        if (lane == 0) {
          const int c = static_cast<int>(v & 0xffffffffull);
          chosen = c;
          pa.perm[step] = c;
          gw[c] = kPlaced;
        }
      }
      __syncthreads();
      const int c = chosen;
      for (int bm = wid; bm < BnM; bm += nw) {
        const uint8_t *crow = cls_s + bm * nN;
        if (crow[c] == BSA_TILE_EMPTY) continue;
        for (int n = lane; n < nN; n += 32)
          if (crow[n] != BSA_TILE_EMPTY && gw[n] != kPlaced) atomicAdd(gw + n, 1);
      }
      __syncthreads();
    }
  } else if (!in_ws) {
    for (int t = threadIdx.x; t < nN; t += blockDim.x) pa.perm[t] = closed_form_order(pa.order, t, nN);
  }
  __syncthreads();
  // row lists and rank(m, n), a warp per row block
  for (int row = wid; row < BnM; row += nw) {
    const uint8_t *crow = cls_s + row * nN;
    int pos = rptr[row];
    for (int n0 = 0; n0 < nN; n0 += 32) {
      const int n = n0 + lane;
      const uint8_t c = n < nN ? crow[n] : BSA_TILE_EMPTY;
      const uint32_t bal = __ballot_sync(0xffffffffu, c != BSA_TILE_EMPTY);
      if (c != BSA_TILE_EMPTY)
        pa.row_ent[pos + __popc(bal & ((1u << lane) - 1u))] = n | (c == BSA_TILE_FULL ? kFullBit : 0u);
      pos += __popc(bal);
    }
    int32_t *rk = pa.rank + static_cast<int64_t>(row) * nN;
    int32_t *rks = rank_s + row * nN;
    int r = 0;
    for (int t0 = 0; t0 < nN; t0 += 32) {
      const int t = t0 + lane;
      int n = -1;
      if (t < nN) n = in_ws ? pa.perm[t] : closed_form_order(pa.order, t, nN);
      const bool ne = n >= 0 && crow[n] != BSA_TILE_EMPTY;
      const uint32_t bal = __ballot_sync(0xffffffffu, ne);
      if (n >= 0) {
        const int32_t v = ne ? r + __popc(bal & ((1u << lane) - 1u)) : -1;
        rk[n] = v;
        rks[n] = v;
      }
      r += __popc(bal);
    }
  }
  __syncthreads();
  // column lists sorted by (rank, m), a warp per column
  unsigned long long *mykeys = keys + static_cast<int64_t>(wid) * nM;
  for (int bn = wid; bn < BnN; bn += nw) {
    const int b = bn / nN, n = bn % nN;
    int cnt = 0;
    for (int m0 = 0; m0 < nM; m0 += 32) {
      const int m = m0 + lane;
      unsigned long long key = 0;
      bool ne = false;
      if (m < nM) {
        const int t = (b * nM + m) * nN + n;
        const uint8_t k = cls_s[t];
        ne = k != BSA_TILE_EMPTY;
        if (ne)
          key = (static_cast<unsigned long long>(rank_s[t]) << 32) |
                (static_cast<unsigned long long>(m) << 1) | (k == BSA_TILE_FULL ? 1ull : 0ull);
      }
      const uint32_t bal = __ballot_sync(0xffffffffu, ne);
      if (ne) mykeys[cnt + __popc(bal & ((1u << lane) - 1u))] = key;
      cnt += __popc(bal);
    }
    __syncwarp();
    const int base = cptr[bn];
    for (int e = lane; e < cnt; e += 32) {
      const unsigned long long ke = mykeys[e];
      int pos = 0;
      for (int f = 0; f < cnt; ++f) pos += mykeys[f] < ke;
      pa.col_ent[base + pos] = static_cast<uint32_t>((ke & 0xffffffffull) >> 1) | ((ke & 1ull) ? kFullBit : 0u);
      pa.col_rank[base + pos] = static_cast<int32_t>(ke >> 32);
    }
    __syncwarp();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t *h = pa.hdr;
    h[kHdrB] = B;
    h[kHdrSq] = a.Sq;
    h[kHdrSkv] = a.Skv;
    h[kHdrFlags] = pa.sig_flags;
    h[kHdrWindow] = pa.sig_window;
    h[kHdrOrder] = pa.order;
    h[kHdrNSeqs] = pa.sig_n_seqs;
    h[kHdrDilation] = pa.sig_dilation;
    __threadfence();
    h[kHdrMagic] = kPlanMagic;
  }
}

// Shared memory of k_plan_fused, and whether the fused path applies.
inline size_t fused_plan_smem(int B, int nM, int nN) {
  const FusedPlanSmem F(B, nM, nN);
  return sizeof(int32_t) * static_cast<size_t>(F.keys) + sizeof(unsigned long long) * 32 * static_cast<size_t>(nM);
}

inline unsigned cdiv(int64_t a, int64_t b) { return static_cast<unsigned>((a + b - 1) / b); }

}  // namespace

cudaError_t launch_plan(const bsa_problem &p, const bsa_mask_spec &m, const bsa_options &o,
                        const WsLayout &L, uint8_t *ws, cudaStream_t s) {
  const int B = p.B, nM = L.nM, nN = L.nN;
  uint32_t *hdr = reinterpret_cast<uint32_t *>(ws + L.status);
  cudaError_t e;
  const bool ids = (m.flags & (BSA_MASK_VARLEN | BSA_MASK_SEGMENT_IDS)) != 0;
  const int64_t tiles = static_cast<int64_t>(B) * nM * nN;
  const size_t fsm = fused_plan_smem(B, nM, nN);
  if (!ids && tiles <= 16384 && fsm <= 200 * 1024) {
    // small map: everything in one block, one launch
    int32_t *perm = reinterpret_cast<int32_t *>(ws + L.perm);
    if (o.bwd_order == BSA_ORDER_PERM) {
      e = cudaMemcpyAsync(perm, o.perm, sizeof(int32_t) * nN, cudaMemcpyHostToDevice, s);
      if (e != cudaSuccess) return e;
    }
    FusedPlanArgs pa{};
    ClassifyArgs &ca = pa.ca;
    ca.B = B; ca.nM = nM; ca.nN = nN; ca.Sq = p.Sq; ca.Skv = p.Skv;
    ca.flags = m.flags;
    ca.window = m.window;
    ca.dilation = m.dilation;
    ca.kv_valid_len = m.kv_valid_len;
    ca.prefix_len = (m.flags & BSA_MASK_PREFIX_LM) ? m.prefix_len : nullptr;
    ca.cls = ws + L.tile_class;
    pa.order = o.bwd_order;
    pa.perm = perm;
    pa.rank = reinterpret_cast<int32_t *>(ws + L.rank);
    pa.row_ptr = reinterpret_cast<int32_t *>(ws + L.row_ptr);
    pa.col_ptr = reinterpret_cast<int32_t *>(ws + L.col_ptr);
    pa.col_rank = reinterpret_cast<int32_t *>(ws + L.col_rank);
    pa.row_ent = reinterpret_cast<uint32_t *>(ws + L.row_ent);
    pa.col_ent = reinterpret_cast<uint32_t *>(ws + L.col_ent);
    pa.hdr = hdr;
    pa.sig_flags = m.flags;
    pa.sig_window = static_cast<uint32_t>(m.window);
    pa.sig_n_seqs = static_cast<uint32_t>(m.n_seqs);
    pa.sig_dilation = static_cast<uint32_t>(m.dilation);
    if (fsm > 48 * 1024) {
      e = cudaFuncSetAttribute(k_plan_fused, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(fsm));
      if (e != cudaSuccess) return e;
    }
    k_plan_fused<<<1, 1024, fsm, s>>>(pa);
    count_launch();
    return cudaGetLastError();
  }
  const int4 *qblk = nullptr, *kblk = nullptr;
  const int32_t *seg_q_ids = nullptr, *seg_kv_ids = nullptr;
  int64_t seg_q_bs = 0, seg_kv_bs = 0;
  const bool varlen = m.flags & BSA_MASK_VARLEN;
  int32_t *rank = reinterpret_cast<int32_t *>(ws + L.rank);
  int32_t *row_cnt = reinterpret_cast<int32_t *>(ws + L.row_cnt);
  int32_t *row_ptr = reinterpret_cast<int32_t *>(ws + L.row_ptr);
  int32_t *col_cnt = reinterpret_cast<int32_t *>(ws + L.col_cnt);
  int32_t *col_ptr = reinterpret_cast<int32_t *>(ws + L.col_ptr);
  int32_t *perm = reinterpret_cast<int32_t *>(ws + L.perm);
  if (varlen || (m.flags & BSA_MASK_SEGMENT_IDS)) {
    const int32_t *sq = m.seg_q, *sk = m.seg_kv;
    int64_t bq = p.Sq, bk = p.Skv;
    if (varlen) {
      // the expansion records bad cu_seqlens in the status word: the header
      // is reset before it
      e = cudaMemsetAsync(hdr, 0, kHdrPlanWords * sizeof(uint32_t), s);
      if (e != cudaSuccess) return e;
      int32_t *dq = reinterpret_cast<int32_t *>(ws + L.seg_q);
      int32_t *dk = reinterpret_cast<int32_t *>(ws + L.seg_kv);
      k_varlen_expand<<<cdiv(p.Sq, 256), 256, 0, s>>>(m.cu_seqlens, m.n_seqs, m.n_align_tail,
                                                      p.Sq, dq, dk, hdr + kHdrStatus);
      count_launch();
      sq = dq;
      sk = dk;
      bq = bk = 0;
    }
    int4 *qb = reinterpret_cast<int4 *>(ws + L.qblk);
    int4 *kb = reinterpret_cast<int4 *>(ws + L.kblk);
    k_plan_prep<<<cdiv(static_cast<int64_t>(B) * (nM + nN) * 32, 256), 256, 0, s>>>(
        sq, sk, p.Sq, p.Skv, nM, nN, B, bq, bk, varlen, qb, kb, varlen ? nullptr : hdr, row_cnt, col_cnt);
    count_launch();
    qblk = qb;
    kblk = kb;
    seg_q_ids = sq;
    seg_kv_ids = sk;
    seg_q_bs = bq;
    seg_kv_bs = bk;
  } else {
    e = cudaMemsetAsync(hdr, 0, kHdrPlanWords * sizeof(uint32_t), s);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(col_cnt, 0, sizeof(int32_t) * B * nN, s);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(row_cnt, 0, sizeof(int32_t) * B * nM, s);
    if (e != cudaSuccess) return e;
  }
  if (o.bwd_order == BSA_ORDER_PERM) {
    e = cudaMemcpyAsync(perm, o.perm, sizeof(int32_t) * nN, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return e;
  }
  ClassifyArgs ca;
  ca.B = B; ca.nM = nM; ca.nN = nN; ca.Sq = p.Sq; ca.Skv = p.Skv;
  ca.flags = m.flags;
  ca.window = m.window;
  ca.dilation = m.dilation;
  ca.kv_valid_len = m.kv_valid_len;
  ca.prefix_len = (m.flags & BSA_MASK_PREFIX_LM) ? m.prefix_len : nullptr;
  ca.qblk = qblk;
  ca.kblk = kblk;
  ca.seg_q = seg_q_ids;
  ca.seg_kv = seg_kv_ids;
  ca.seg_q_bstride = seg_q_bs;
  ca.seg_kv_bstride = seg_kv_bs;
  ca.cls = ws + L.tile_class;
  ca.row_cnt = row_cnt;
  ca.col_cnt = col_cnt;
  k_classify_chunks<<<cdiv(static_cast<int64_t>(B) * nM * ((nN + 31) / 32) * 32, 256), 256, 0, s>>>(ca);
  k_scan2<<<2, 1024, 0, s>>>(row_cnt, row_ptr, B * nM, col_cnt, col_ptr, B * nN, hdr, B, p.Sq,
                             p.Skv, m.flags, m.window, o.bwd_order, m.n_seqs,
                             static_cast<uint32_t>(m.dilation));
  if (o.bwd_order == BSA_ORDER_GREEDY) {
    const size_t gsm = sizeof(int32_t) * static_cast<size_t>(nN);
    if (gsm > 48 * 1024) {
      e = cudaFuncSetAttribute(k_greedy_order, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(gsm));
      if (e != cudaSuccess) return e;
    }
    k_greedy_order<<<1, 1024, gsm, s>>>(ws + L.tile_class, B * nM, nN, perm);
    count_launch();
  }
  k_row_fill<<<cdiv(static_cast<int64_t>(B) * nM * 32, 256), 256, 0, s>>>(
      ws + L.tile_class, B * nM, nN, o.bwd_order, perm, row_ptr,
      reinterpret_cast<uint32_t *>(ws + L.row_ent), rank);
  const size_t smem = sizeof(unsigned long long) * static_cast<size_t>(nM);
  if (smem > 48 * 1024) {
    e = cudaFuncSetAttribute(k_col_fill, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  k_col_fill<<<B * nN, 256, smem, s>>>(ws + L.tile_class, rank, nM, nN, col_ptr,
                                       reinterpret_cast<uint32_t *>(ws + L.col_ent),
                                       reinterpret_cast<int32_t *>(ws + L.col_rank));
  count_launch(4);
  return cudaGetLastError();
}

}  // namespace bsa
