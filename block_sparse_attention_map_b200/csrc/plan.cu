// Block-map planner: steps a1 (tile classes from the mask predicates) and a6
// (kv-column order pi, rank(m, n), rank-sorted column lists) of the hot path.
//
// Sources: "Let splash attention exceed 524,288 tokens when packing is off"
// (maxtext PR #4929) for the segment-id mask and the block mask it implies;
// maxdiffusion PR #404 review for global KV padding; sglang PR #47566
// ("Modifications") for varlen alignment rows; "Add more optimal dk order
// optional arg" (flash-attention PR #2512, "Sliding window perf issue" and "A
// simplish fix") for rank(m, n), the kv-column orders and the unified column
// list walked in rank order.
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

// Per-block summary of segment ids: [min, max, #positions with a real id,
// #alignment positions] over the in-range positions of the block.  With
// neg_is_align (varlen) negative ids mark alignment positions; caller-supplied
// segment ids may take any int32 value.
__global__ void k_block_summary(const int32_t *__restrict__ seg, int S, int nblk, int B,
                                int64_t bstride, int neg_is_align, int4 *__restrict__ out) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= B * nblk) return;
  const int b = warp / nblk, blk = warp % nblk;
  int mn = 0x7fffffff, mx = -0x7fffffff - 1, nreal = 0, nbad = 0;
  for (int t = lane; t < kTile; t += 32) {
    const int i = blk * kTile + t;
    if (i >= S) break;
    const int v = seg[b * bstride + i];
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
  if (lane == 0) out[warp] = make_int4(mn, mx, nreal, nbad);
}

struct ClassifyArgs {
  int B, nM, nN, Sq, Skv;
  uint32_t flags;
  int window;
  const int32_t *kv_valid_len;
  const int4 *qblk, *kblk;  // null unless segment ids / varlen
  uint8_t *cls;
};

// Tile class per (b, m, n): the AND-combination of one class per enabled
// predicate (EMPTY if any predicate is empty, FULL if all are full).  Window,
// padding and out-of-range columns are classified analytically and exactly;
// segment ids through per-block [min, max] intervals, exact for
// non-decreasing ids and conservative (PARTIAL instead of EMPTY) otherwise.
__global__ void k_classify(ClassifyArgs a) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t total = static_cast<int64_t>(a.B) * a.nM * a.nN;
  if (idx >= total) return;
  const int n = static_cast<int>(idx % a.nN);
  const int m = static_cast<int>((idx / a.nN) % a.nM);
  const int b = static_cast<int>(idx / (static_cast<int64_t>(a.nN) * a.nM));
  const int i0 = m * kTile, i1 = min(a.Sq, i0 + kTile) - 1;
  const int j0 = n * kTile, jv1 = min(a.Skv, j0 + kTile) - 1;
  uint8_t c = BSA_TILE_FULL;
  if (j0 + kTile - 1 > jv1) c = BSA_TILE_PARTIAL;  // out-of-range keys must be masked
  if (a.flags & BSA_MASK_CAUSAL_WINDOW) {
    const int o = a.Skv - a.Sq, W = a.window;
    const bool any = (j0 <= i1 + o) && (W == 0 || jv1 >= i0 + o - W + 1);
    const bool all = (jv1 <= i0 + o) && (W == 0 || j0 >= i1 + o - W + 1);
    if (!any) { a.cls[idx] = BSA_TILE_EMPTY; return; }
    if (!all) c = BSA_TILE_PARTIAL;
  }
  if (a.flags & BSA_MASK_KV_VALID_LEN) {
    const int L = a.kv_valid_len[b];
    if (j0 >= L) { a.cls[idx] = BSA_TILE_EMPTY; return; }
    if (jv1 >= L) c = BSA_TILE_PARTIAL;
  }
  if (a.qblk != nullptr) {
    const int4 q = a.qblk[b * a.nM + m];
    const int4 k = a.kblk[b * a.nN + n];
    if (q.z == 0 || k.z == 0 || q.y < k.x || k.y < q.x) { a.cls[idx] = BSA_TILE_EMPTY; return; }
    const bool one = q.x == q.y && k.x == k.y && q.x == k.x && q.w == 0 && k.w == 0;
    if (!one) c = BSA_TILE_PARTIAL;
  }
  a.cls[idx] = c;
}

__global__ void k_make_perm(int nN, int order, int32_t *perm) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t < nN) perm[t] = (order == BSA_ORDER_DESC) ? (nN - 1 - t) : t;
}

// rank(m, n): walk row m's columns in the order pi; non-empty ones get 0, 1, 2, ...
__global__ void k_row_rank(const uint8_t *__restrict__ cls, const int32_t *__restrict__ perm,
                           int BnM, int nN, int32_t *__restrict__ rank,
                           int32_t *__restrict__ row_cnt) {
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= BnM) return;
  const uint8_t *row = cls + static_cast<int64_t>(r) * nN;
  int32_t *rk = rank + static_cast<int64_t>(r) * nN;
  int cnt = 0;
  for (int t = 0; t < nN; ++t) {
    const int n = perm[t];
    rk[n] = row[n] != BSA_TILE_EMPTY ? cnt++ : -1;
  }
  row_cnt[r] = cnt;
}

__global__ void k_col_count(const uint8_t *__restrict__ cls, int B, int nM, int nN,
                            int32_t *__restrict__ col_cnt) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= B * nN) return;
  const int b = t / nN, n = t % nN;
  int cnt = 0;
  for (int m = 0; m < nM; ++m) cnt += cls[(static_cast<int64_t>(b) * nM + m) * nN + n] != 0;
  col_cnt[t] = cnt;
}

// Exclusive scans of row and column counts into CSR offsets (block 0: rows,
// block 1: columns); ptr[count] receives the total.
__global__ void k_scan2(const int32_t *__restrict__ c0, int32_t *__restrict__ p0, int n0,
                        const int32_t *__restrict__ c1, int32_t *__restrict__ p1, int n1) {
  const int32_t *c = blockIdx.x == 0 ? c0 : c1;
  int32_t *p = blockIdx.x == 0 ? p0 : p1;
  const int n = blockIdx.x == 0 ? n0 : n1;
  __shared__ int32_t buf[1024];
  __shared__ int32_t carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < n; base += 1024) {
    const int i = base + threadIdx.x;
    const int32_t v = i < n ? c[i] : 0;
    buf[threadIdx.x] = v;
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) {
      const int32_t add = threadIdx.x >= o ? buf[threadIdx.x - o] : 0;
      __syncthreads();
      buf[threadIdx.x] += add;
      __syncthreads();
    }
    if (i < n) p[i] = carry + buf[threadIdx.x] - v;
    __syncthreads();
    if (threadIdx.x == 1023) carry += buf[1023];
    __syncthreads();
  }
  if (threadIdx.x == 0) p[n] = carry;
}

// Row lists for the forward: ascending n, FULL flag in bit 30.
__global__ void k_row_fill(const uint8_t *__restrict__ cls, int BnM, int nN,
                           const int32_t *__restrict__ row_ptr, uint32_t *__restrict__ row_ent) {
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= BnM) return;
  const uint8_t *row = cls + static_cast<int64_t>(r) * nN;
  int pos = row_ptr[r];
  for (int n = 0; n < nN; ++n) {
    const uint8_t c = row[n];
    if (c != BSA_TILE_EMPTY) row_ent[pos++] = n | (c == BSA_TILE_FULL ? kFullBit : 0u);
  }
}

// Column lists for the backward: the unified partial+full list of column n,
// sorted by (rank(m, n), m).  One block per (b, n); the column's entries are
// gathered into shared memory and each entry's position is the number of
// entries with a smaller key.
__global__ void k_col_fill(const uint8_t *__restrict__ cls, const int32_t *__restrict__ rank,
                          int nM, int nN, const int32_t *__restrict__ col_ptr,
                          uint32_t *__restrict__ col_ent, int32_t *__restrict__ col_rank) {
  extern __shared__ unsigned long long keys[];
  __shared__ int cnt;
  const int bn = blockIdx.x;
  const int b = bn / nN, n = bn % nN;
  if (threadIdx.x == 0) {
    int c = 0;
    for (int m = 0; m < nM; ++m) {
      const int64_t t = (static_cast<int64_t>(b) * nM + m) * nN + n;
      const uint8_t k = cls[t];
      if (k != BSA_TILE_EMPTY) {
        keys[c++] = (static_cast<unsigned long long>(rank[t]) << 32) |
                    (static_cast<unsigned long long>(m) << 1) | (k == BSA_TILE_FULL ? 1ull : 0ull);
      }
    }
    cnt = c;
  }
  __syncthreads();
  const int c = cnt;
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

__global__ void k_signature(uint32_t *hdr, int B, int Sq, int Skv, uint32_t flags, int window,
                            int order, int n_seqs) {
  hdr[kHdrB] = B;
  hdr[kHdrSq] = Sq;
  hdr[kHdrSkv] = Skv;
  hdr[kHdrFlags] = flags;
  hdr[kHdrWindow] = window;
  hdr[kHdrOrder] = order;
  hdr[kHdrNSeqs] = n_seqs;
  __threadfence();
  hdr[kHdrMagic] = kPlanMagic;
}

inline unsigned cdiv(int64_t a, int64_t b) { return static_cast<unsigned>((a + b - 1) / b); }

}  // namespace

cudaError_t launch_plan(const bsa_problem &p, const bsa_mask_spec &m, const bsa_options &o,
                        const WsLayout &L, uint8_t *ws, cudaStream_t s) {
  const int B = p.B, nM = L.nM, nN = L.nN;
  uint32_t *hdr = reinterpret_cast<uint32_t *>(ws + L.status);
  cudaError_t e = cudaMemsetAsync(hdr, 0, kHdrWords * sizeof(uint32_t), s);
  if (e != cudaSuccess) return e;

  const int4 *qblk = nullptr, *kblk = nullptr;
  const bool varlen = m.flags & BSA_MASK_VARLEN;
  if (varlen || (m.flags & BSA_MASK_SEGMENT_IDS)) {
    const int32_t *sq = m.seg_q, *sk = m.seg_kv;
    int64_t bq = p.Sq, bk = p.Skv;
    if (varlen) {
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
    k_block_summary<<<cdiv(static_cast<int64_t>(B) * nM * 32, 256), 256, 0, s>>>(sq, p.Sq, nM, B,
                                                                                bq, varlen, qb);
    k_block_summary<<<cdiv(static_cast<int64_t>(B) * nN * 32, 256), 256, 0, s>>>(sk, p.Skv, nN,
                                                                                B, bk, varlen, kb);
    count_launch(2);
    qblk = qb;
    kblk = kb;
  }

  ClassifyArgs ca;
  ca.B = B; ca.nM = nM; ca.nN = nN; ca.Sq = p.Sq; ca.Skv = p.Skv;
  ca.flags = m.flags;
  ca.window = m.window;
  ca.kv_valid_len = m.kv_valid_len;
  ca.qblk = qblk;
  ca.kblk = kblk;
  ca.cls = ws + L.tile_class;
  k_classify<<<cdiv(static_cast<int64_t>(B) * nM * nN, 256), 256, 0, s>>>(ca);
  count_launch();

  int32_t *perm = reinterpret_cast<int32_t *>(ws + L.perm);
  if (o.bwd_order == BSA_ORDER_PERM) {
    e = cudaMemcpyAsync(perm, o.perm, sizeof(int32_t) * nN, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return e;
  } else {
    k_make_perm<<<cdiv(nN, 256), 256, 0, s>>>(nN, o.bwd_order, perm);
    count_launch();
  }

  int32_t *rank = reinterpret_cast<int32_t *>(ws + L.rank);
  int32_t *row_cnt = reinterpret_cast<int32_t *>(ws + L.row_cnt);
  int32_t *row_ptr = reinterpret_cast<int32_t *>(ws + L.row_ptr);
  int32_t *col_cnt = reinterpret_cast<int32_t *>(ws + L.col_cnt);
  int32_t *col_ptr = reinterpret_cast<int32_t *>(ws + L.col_ptr);
  k_row_rank<<<cdiv(B * nM, 128), 128, 0, s>>>(ws + L.tile_class, perm, B * nM, nN, rank, row_cnt);
  k_col_count<<<cdiv(B * nN, 128), 128, 0, s>>>(ws + L.tile_class, B, nM, nN, col_cnt);
  k_scan2<<<2, 1024, 0, s>>>(row_cnt, row_ptr, B * nM, col_cnt, col_ptr, B * nN);
  k_row_fill<<<cdiv(B * nM, 128), 128, 0, s>>>(ws + L.tile_class, B * nM, nN, row_ptr,
                                               reinterpret_cast<uint32_t *>(ws + L.row_ent));
  const size_t smem = sizeof(unsigned long long) * static_cast<size_t>(nM);
  if (smem > 48 * 1024) {
    e = cudaFuncSetAttribute(k_col_fill, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  k_col_fill<<<B * nN, 256, smem, s>>>(ws + L.tile_class, rank, nM, nN, col_ptr,
                                       reinterpret_cast<uint32_t *>(ws + L.col_ent),
                                       reinterpret_cast<int32_t *>(ws + L.col_rank));
  k_signature<<<1, 1, 0, s>>>(hdr, B, p.Sq, p.Skv, m.flags, m.window, o.bwd_order, m.n_seqs);
  count_launch(6);
  return cudaGetLastError();
}

}  // namespace bsa
