// Forward pass (steps a2 and a3 of the hot path).
//
// a2  fixed-m bound: kmax[b,h] = max over valid keys of ||k_j||, qmax[b,h] and
//     per-row ||q_i||, and the per-head gate 2*scale*qmax*kmax <= G ("Fixed-m
//     softmax for 2D-ring x Ulysses attention (WAN 2.2)", introduction and
//     "Notes": heads whose bound cannot be proven safe keep online softmax).
//     With k-smoothing ("Notes": possible when one device holds all of K) the
//     keys are centred on their mean c first: kmax becomes the radius
//     max ||k_j - c||, and each row's reference gains the shift scale * q_i . c.
// a3  the tiled exact softmax attention main loop over each q-block's row list
//     of non-empty tiles.  Online softmax keeps the running max in registers
//     (one query row per thread) and rescales lazily; fixed-m pins the max to
//     scale*||q_i||*kmax before streaming and needs neither max nor rescale.
//
// sm_100a design: one CTA per SM, persistent over work units = pairs of
// q-blocks (A = 2g, B = 2g+1) of one (b, h).  The CTA walks the union of the
// two row lists, so each K/V tile is loaded once for both q-blocks.  With
// grouped-query attention head h reads the K/V of kv head h / (H / H_kv).
// Units are handed out by an atomic ticket, so an SM whose loads wait longer
// takes fewer of them.
//   warp 0      ticket + TMA producer: draws a unit, decodes it into a
//               two-slot shared ring the other roles read, then loads Q_A, Q_B
//               once per unit and K and V tiles through separate stage rings,
//               128-byte swizzled 64 x 128 boxes.
//   warp 1      owns TMEM (512 columns) and issues tcgen05.mma from one lane,
//               ping-ponging the two groups: PV_A(u), S_A(u+1), PV_B(u),
//               S_B(u+1), so one group's softmax overlaps the other's MMAs.
//               S = Q K^T is SS (both K-major); O += P V is TS (P read from
//               TMEM over the S columns, V an MN-major B operand).
//   warps 4-7   softmax of q-block A, warps 8-11 of q-block B: one query row
//               per thread (its TMEM lane).  PARTIAL tiles are masked through a
//               128-bit allowed-key mask (the window's key range thinned by
//               its dilation, OR the prefix, AND segment ids); online
//               mode takes the tile max in a first pass over TMEM and rescales
//               O lazily; the epilogue writes O / l_r (bf16), the O residual
//               and LSE, 32 bytes per store.
// TMEM columns: S_A [0,128) S_B [128,256) O_A [256,256+D) O_B [256+D,256+2D).
#include <cfloat>

#include "internal.h"
#include "ptx.cuh"

namespace bsa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: tolerate p up to 2^8
constexpr int kUnitWords = 10;  // a decoded unit in the shared ring: valid, b, h, bh, m[2], rs[2], re[2]

struct FwdParams {
  MaskParams mask;
  int B, H, Sq, Skv, nM, n_units;
  int n_pairs;   // units [0, n_pairs) are q-block pairs; the rest are single q-blocks
  int head_group;  // (b, h) interleaved in groups of this many (a divisor of B * H)
  int kv_group;  // query heads per key/value head (grouped-query attention)
  float scale, scale_log2;
  const int32_t *row_ptr;
  const uint32_t *row_ent;
  __nv_bfloat16 *out;
  int64_t o_sb, o_ss, o_sh;
  float *lse;
  int fixed_mode;
  int block_bound;     // per q-block bound: kmax_m from kblk, ||q_i|| from the Q tile, per-row gate
  float gate_limit;
  int Hk, nN;
  const float *kblk;   // [B, H_kv, nN] per kv block max ||k_j|| (block bound)
  float *kmax_q;       // [B, H, nM] each q-block's kmax, written for inspection (block bound)
  const float *kmax;   // [B, H] (the radius R with k-smoothing)
  const float *qnorm;  // [B, H, Sq]
  const float *qdot;   // [B, H, Sq] q_i . center with k-smoothing, else null
  uint8_t *o_resid;  // [B, Sq, H, D] O - bf16(O) as scaled e5m2 bytes, or null
  const __nv_bfloat16 *q;  // the caller's Q (recorded with its fp16 copy)
  int64_t q_sb, q_ss, q_sh;
  int o_v8;          // O rows and row strides are 32-byte aligned: one store per 16 columns
  __half *q16;       // [B, Sq, H, D] fp16 copy of Q for the backward (with the residual), or null
  const int32_t *gate; // [B, H]
  uint32_t *hdr;
  uint64_t timeout_ns;
  uint32_t sig[kSigWords];  // expected plan signature (B, Sq, Skv, flags, window, order, n_seqs, dilation)
  uint32_t sig_mask;   // which signature words must match
};

template <int D, int NQ, int NK, int NV>
struct FwdSmem {
  static constexpr int kTB = kTile * D * 2;
  static constexpr int kQ = 0;                         // Q ring (both groups' tiles, in load order)
  static constexpr int kK = NQ * kTB;                  // K ring
  static constexpr int kV = kK + NK * kTB;             // V ring
  static constexpr int kSeg = kV + NV * kTB;           // int32 [group][buffer][128]
  static constexpr int kBar = kSeg + 4 * kTile * 4;
  // bTkFull / bTkEmpty: the unit ring
  static constexpr int bQFull = 0, bQEmpty = NQ, bKFull = 2 * NQ, bKEmpty = bKFull + NK,
                       bVFull = bKEmpty + NK, bVEmpty = bVFull + NV, bSFull = bVEmpty + NV,
                       bPFull = bSFull + 2, bPVDone = bPFull + 2, bSegReady = bPVDone + 2,
                       bTkFull = bSegReady + 4, bTkEmpty = bTkFull + 2, bFinal = bTkEmpty + 2,
                       kNumBars = bFinal + 1;
  static constexpr int kUnit = kBar + kNumBars * 8;         // int32 [2][kUnitWords]
  static constexpr int kMisc = kUnit + 2 * kUnitWords * 4;  // tmem slot, abort flag
  static constexpr int kAlloc = kMisc + 16;
};

// Bounded wait that ignores the abort flag: used only to drain copies already
// in flight before the CTA exits.
__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(a, parity)) {
    if (globaltimer_ns() - t0 > 200000000ull) return;
  }
}

// One work unit: a pair of q-blocks (A = 2g, B = 2g+1) of one (b, h).  The
// (b, h) are taken in groups of head_group; within a group the units go with
// the pair index descending and every (b, h) of the group in turn.  Under
// causal, prefix and document masks a q-block's row list grows with m, so the
// long units go first and the short ones fill the last wave, and the group's
// heads share the work of each pair index (document forward 151 -> 116 us,
// prefix-LM 385 -> 310 us against (b, h)-major ascending order).  The group is
// as large as keeps its heads' K and V within half the L2 (every head at the
// window and document shapes; one at the video shape, whose heads' K and V
// would otherwise stream through the L2 together: 113 -> 137 ms).  The pairs
// that would make a last, partly filled wave are split into two single q-block
// units each (slot A only), so that wave takes about half as long.
struct FwdUnit {
  int b, h, bh, m[2], rs[2], re[2];
};

__device__ __forceinline__ FwdUnit decode_unit(const FwdParams &p, int u) {
  FwdUnit w;
  const int nP = (p.nM + 1) >> 1;
  int pu = u, only = -1;
  if (u >= p.n_pairs) {
    const int s = u - p.n_pairs;
    pu = p.n_pairs + (s >> 1);
    only = s & 1;
  }
  const int G = p.head_group, per_group = G * nP;
  const int r = pu % per_group;
  w.bh = (pu / per_group) * G + r % G;
  const int g = nP - 1 - r / G;
  w.b = w.bh / p.H;
  w.h = w.bh % p.H;
#pragma unroll
  for (int x = 0; x < 2; ++x) {
    w.m[x] = only < 0 ? 2 * g + x : (x == 0 ? 2 * g + only : p.nM);
    if (w.m[x] < p.nM) {
      w.rs[x] = p.row_ptr[w.b * p.nM + w.m[x]];
      w.re[x] = p.row_ptr[w.b * p.nM + w.m[x] + 1];
    } else {
      w.rs[x] = w.re[x] = 0;
    }
  }
  return w;
}

__device__ __forceinline__ void write_unit(int32_t *e, bool valid, const FwdUnit &w) {
  e[0] = valid ? 1 : 0;
  e[1] = w.b;
  e[2] = w.h;
  e[3] = w.bh;
  e[4] = w.m[0];
  e[5] = w.m[1];
  e[6] = w.rs[0];
  e[7] = w.rs[1];
  e[8] = w.re[0];
  e[9] = w.re[1];
}

// Read after the slot's full barrier (acquire); false once the tickets are spent.
__device__ __forceinline__ bool read_unit(const int32_t *e, FwdUnit &w) {
  w.b = e[1];
  w.h = e[2];
  w.bh = e[3];
  w.m[0] = e[4];
  w.m[1] = e[5];
  w.rs[0] = e[6];
  w.rs[1] = e[7];
  w.re[0] = e[8];
  w.re[1] = e[9];
  return e[0] != 0;
}

// Walks the union of the two row lists in ascending kv-block order.
struct UnionWalk {
  const uint32_t *ent;
  int i[2], e[2];
  __device__ __forceinline__ bool next(int &n, bool &in0, bool &in1) {
    const int n0 = i[0] < e[0] ? static_cast<int>(ent[i[0]] & kIndexMask) : INT_MAX;
    const int n1 = i[1] < e[1] ? static_cast<int>(ent[i[1]] & kIndexMask) : INT_MAX;
    if (n0 == INT_MAX && n1 == INT_MAX) return false;
    n = min(n0, n1);
    in0 = n0 == n;
    in1 = n1 == n;
    i[0] += in0;
    i[1] += in1;
    return true;
  }
};

template <int D, int NQ, int NK, int NV>
__global__ void __launch_bounds__(384, 1)
k_attn_fwd(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
           const __grid_constant__ CUtensorMap tv, const FwdParams p) {
  using L = FwdSmem<D, NQ, NK, NV>;
  extern __shared__ __align__(1024) uint8_t sm[];
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::kBar);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::kMisc);
  int *abort_flag = reinterpret_cast<int *>(sm + L::kMisc + 4);
  int32_t *seg_sm = reinterpret_cast<int32_t *>(sm + L::kSeg);
  int32_t *unit_ring = reinterpret_cast<int32_t *>(sm + L::kUnit);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < L::kNumBars; ++i) {
      uint32_t cnt = 1;
      if ((i >= L::bPFull && i < L::bPFull + 2) || (i >= L::bSegReady && i < L::bSegReady + 4))
        cnt = 128;
      // a Q slot is free once the unit's MMAs are done and, when the fp16
      // copy is written, warps 2-3 have read it
      if (i >= L::bQEmpty && i < L::bQEmpty + NQ && p.q16 != nullptr) cnt = 1 + 64;
      // the unit ring's readers: the MMA lane, the eight softmax warps and,
      // when the fp16 copy of Q is written, warps 2-3
      if (i >= L::bTkEmpty && i < L::bTkEmpty + 2) cnt = 1 + 8 + (p.q16 != nullptr ? 2 : 0);
      mbar_init(&bars[i], cnt);
    }
    *abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tq);
    tma_prefetch_desc(&tk);
    tma_prefetch_desc(&tv);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  Watchdog wd{abort_flag, p.hdr + kHdrStatus, p.timeout_ns};
  if (threadIdx.x == 0) {
    const volatile uint32_t *h = p.hdr;
    bool ok = h[kHdrMagic] == kPlanMagic;
    for (int i = 0; i < kSigWords; ++i) ok = ok && (!((p.sig_mask >> i) & 1u) || h[kHdrB + i] == p.sig[i]);
    if (!ok) wd.trip(BSA_ERR_PLAN_MISMATCH);
    // the swizzled tiles rely on a 1024-byte aligned dynamic shared window
    if ((smem_u32(sm) & 1023u) != 0u) wd.trip(BSA_ERR_UNSUPPORTED);
    if (blockIdx.x == 0) {
      // which output (none: 0) and problem the O residual belongs to, for the
      // backward's Delta
      const uint64_t tag = (ok && p.o_resid != nullptr) ? reinterpret_cast<uint64_t>(p.out) : 0ull;
      p.hdr[kHdrResidLo] = static_cast<uint32_t>(tag);
      p.hdr[kHdrResidHi] = static_cast<uint32_t>(tag >> 32);
      p.hdr[kHdrResidB] = p.B;
      p.hdr[kHdrResidH] = p.H;
      p.hdr[kHdrResidSq] = p.Sq;
      p.hdr[kHdrResidSkv] = p.Skv;
      p.hdr[kHdrResidD] = D;
      const uint64_t qtag = (ok && p.q16 != nullptr) ? reinterpret_cast<uint64_t>(p.q) : 0ull;
      p.hdr[kHdrQ16Lo] = static_cast<uint32_t>(qtag);
      p.hdr[kHdrQ16Hi] = static_cast<uint32_t>(qtag >> 32);
      p.hdr[kHdrQ16Sb] = static_cast<uint32_t>(p.q_sb);
      p.hdr[kHdrQ16Ss] = static_cast<uint32_t>(p.q_ss);
      p.hdr[kHdrQ16Sh] = static_cast<uint32_t>(p.q_sh);
    }
  }
  __syncthreads();
  // no early trigger for a backward's Delta pass: it launches as our CTAs
  // leave (an early trigger measured 2-8 us per step slower on the 8192
  // window, gqa and document workloads)

  constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, 0, 0);
  constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, 0, 1);
  constexpr int kTB = L::kTB;

  if (wd.aborted()) {
    // plan mismatch or misaligned shared memory: nothing to do
  } else if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t kv = 0, qi = 0, k_issued = 0, v_issued = 0;
      bool stop = false;
      for (uint32_t tc = 0; !stop; ++tc) {
        const uint32_t slot = tc & 1;
        if (tc >= 2 && !wd.wait(&bars[L::bTkEmpty + slot], ((tc >> 1) - 1) & 1)) break;
        const int u = static_cast<int>(atomicAdd(p.hdr + kHdrFwdTicket, 1u));
        const bool valid = u < p.n_units;
        FwdUnit w{};
        if (valid) w = decode_unit(p, u);
        write_unit(unit_ring + slot * kUnitWords, valid, w);
        mbar_arrive(&bars[L::bTkFull + slot]);
        if (!valid) break;
        const bool has[2] = {w.re[0] > w.rs[0], w.re[1] > w.rs[1]};
        if (!has[0] && !has[1]) continue;
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          if (!has[x]) continue;
          // Q tiles go through a ring of NQ slots in load order (A, B of each
          // unit): with NQ = 3 the next unit's Q_A loads during this unit, and
          // its Q_B as soon as this unit's Q_A is released
          const uint32_t qs = qi % NQ;
          if (qi >= NQ && !wd.wait(&bars[L::bQEmpty + qs], ((qi / NQ) - 1) & 1)) { stop = true; break; }
          mbar_arrive_expect_tx(&bars[L::bQFull + qs], kTB);
          for (int c = 0; c < D / 64; ++c)
            tma_load_4d(sm + L::kQ + qs * kTB + c * 16384, &tq, &bars[L::bQFull + qs], c * 64,
                        w.m[x] * kTile, w.h, w.b);
          ++qi;
        }
        if (stop) break;
        UnionWalk uw{p.row_ent, {w.rs[0], w.rs[1]}, {w.re[0], w.re[1]}};
        int n;
        bool i0, i1;
        while (uw.next(n, i0, i1)) {
          const uint32_t ks = kv % NK, vs = kv % NV;
          if (kv >= NK && !wd.wait(&bars[L::bKEmpty + ks], ((kv / NK) - 1) & 1)) { stop = true; break; }
          mbar_arrive_expect_tx(&bars[L::bKFull + ks], kTB);
          for (int c = 0; c < D / 64; ++c)
            tma_load_4d(sm + L::kK + ks * kTB + c * 16384, &tk, &bars[L::bKFull + ks], c * 64,
                        n * kTile, w.h / p.kv_group, w.b);
          ++k_issued;
          if (kv >= NV && !wd.wait(&bars[L::bVEmpty + vs], ((kv / NV) - 1) & 1)) { stop = true; break; }
          mbar_arrive_expect_tx(&bars[L::bVFull + vs], kTB);
          for (int c = 0; c < D / 64; ++c)
            tma_load_4d(sm + L::kV + vs * kTB + c * 16384, &tv, &bars[L::bVFull + vs], c * 64,
                        n * kTile, w.h / p.kv_group, w.b);
          ++v_issued;
          ++kv;
        }
      }
      if (wd.aborted()) {
        // let every issued copy land before the CTA's shared memory goes away
        for (uint32_t t = (k_issued > NK ? k_issued - NK : 0); t < k_issued; ++t)
          drain_wait(&bars[L::bKFull + t % NK], (t / NK) & 1);
        for (uint32_t t = (v_issued > NV ? v_issued - NV : 0); t < v_issued; ++t)
          drain_wait(&bars[L::bVFull + t % NV], (t / NV) & 1);
        for (uint32_t t = (qi > NQ ? qi - NQ : 0); t < qi; ++t)
          drain_wait(&bars[L::bQFull + t % NQ], (t / NQ) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t kv = 0, qm = 0, tcount[2] = {0, 0};
      bool stop = false;
      uint32_t q_addr[2] = {0, 0}, q_slot[2] = {0, 0};
      // S_x = Q_x K^T into the S columns of group x.  The previous PV_x still
      // reads P_x from those columns; tcgen05.mma ops issued by one thread
      // execute in issue order, so no completion wait is needed in between.
      auto issue_s = [&](int x, uint32_t kvi) -> bool {
        if (!wd.wait(&bars[L::bKFull + kvi % NK], (kvi / NK) & 1)) return false;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sm + L::kK + (kvi % NK) * kTB);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_ss(tmem + x * 128, sw128_desc(q_addr[x] + off, 16, 1024),
                 sw128_desc(k_addr + off, 16, 1024), kIdescS, kk > 0);
        }
        mma_commit(&bars[L::bSFull + x]);
        return true;
      };
      for (uint32_t tc = 0; !stop; ++tc) {
        const uint32_t slot = tc & 1;
        if (!wd.wait(&bars[L::bTkFull + slot], (tc >> 1) & 1)) break;
        FwdUnit w;
        const bool valid = read_unit(unit_ring + slot * kUnitWords, w);
        mbar_arrive(&bars[L::bTkEmpty + slot]);
        if (!valid) break;
        const bool has[2] = {w.re[0] > w.rs[0], w.re[1] > w.rs[1]};
        if (!has[0] && !has[1]) continue;
        for (int x = 0; x < 2; ++x) {
          if (!has[x]) continue;
          q_slot[x] = qm % NQ;
          q_addr[x] = smem_u32(sm + L::kQ + q_slot[x] * kTB);
          if (!wd.wait(&bars[L::bQFull + q_slot[x]], (qm / NQ) & 1)) stop = true;
          ++qm;
        }
        if (stop) break;
        bool first[2] = {true, true};
        UnionWalk uw{p.row_ent, {w.rs[0], w.rs[1]}, {w.re[0], w.re[1]}};
        int n;
        bool in_cur[2], in_nxt[2];
        uw.next(n, in_cur[0], in_cur[1]);
        uint32_t kv_cur = kv;
        for (int x = 0; x < 2 && !stop; ++x)
          if (in_cur[x] && !issue_s(x, kv_cur)) stop = true;
        if (stop) break;
        mma_commit(&bars[L::bKEmpty + kv_cur % NK]);
        for (;;) {
          const bool more = uw.next(n, in_nxt[0], in_nxt[1]);
          const uint32_t kv_nxt = kv_cur + 1;
          if (!wd.wait(&bars[L::bVFull + kv_cur % NV], (kv_cur / NV) & 1)) { stop = true; break; }
          for (int x = 0; x < 2; ++x) {
            if (in_cur[x]) {
              // O_x += P_x V  (P from TMEM over the S columns, V as an MN-major B operand)
              if (!wd.wait(&bars[L::bPFull + x], tcount[x] & 1)) { stop = true; break; }
              tc_fence_after();
              const uint32_t v_addr = smem_u32(sm + L::kV + (kv_cur % NV) * kTB);
#pragma unroll
              for (int kk = 0; kk < 8; ++kk)
                mma_ts(tmem + 256 + x * D, tmem + x * 128 + kk * 8,
                       sw128_desc(v_addr + kk * 2048, 16384, 1024), kIdescPV,
                       (!first[x] || kk > 0) ? 1u : 0u);
              mma_commit(&bars[L::bPVDone + x]);
              first[x] = false;
              ++tcount[x];
            }
            // the next S of this group as soon as its P has been consumed
            if (more && in_nxt[x] && !issue_s(x, kv_nxt)) { stop = true; break; }
          }
          if (stop) break;
          mma_commit(&bars[L::bVEmpty + kv_cur % NV]);
          if (!more) break;
          mma_commit(&bars[L::bKEmpty + kv_nxt % NK]);
          kv_cur = kv_nxt;
          in_cur[0] = in_nxt[0];
          in_cur[1] = in_nxt[1];
        }
        if (stop) break;
        kv = kv_cur + 1;
        for (int x = 0; x < 2; ++x)
          if (has[x]) mma_commit(&bars[L::bQEmpty + q_slot[x]]);
      }
      // every tcgen05 op this thread issued is complete before TMEM is freed
      mma_commit(&bars[L::bFinal]);
      drain_wait(&bars[L::bFinal], 0);
    }
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------------------ fp16 Q (warps 2, 3)
    // When the forward keeps the O residual (a backward is expected on this
    // workspace), each Q tile it loads is also written out as fp16 for the
    // backward's products, while it sits in shared memory: the backward's
    // Delta pass then need not read Q again.  16-byte pieces, a row's pieces
    // on consecutive threads; the slot is released to the producer only after
    // these reads (its empty barrier counts them).
    if (p.q16 != nullptr) {
      const int ct = threadIdx.x - 64;
      auto wwait = [&](uint64_t *bar, uint32_t parity) {
        return __all_sync(0xffffffffu, wd.wait(bar, parity)) != 0;
      };
      constexpr int kCpr = D / 8;  // 16-byte pieces per row
      uint32_t qm = 0, in_max = 0;
      bool stop = false;
      for (uint32_t tc = 0; !stop; ++tc) {
        const uint32_t slot = tc & 1;
        if (!wwait(&bars[L::bTkFull + slot], (tc >> 1) & 1)) break;
        FwdUnit w;
        const bool valid = read_unit(unit_ring + slot * kUnitWords, w);
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[L::bTkEmpty + slot]);
        if (!valid) break;
#pragma unroll 1
        for (int x = 0; x < 2; ++x) {
          if (w.re[x] <= w.rs[x]) continue;
          const uint32_t qs = qm % NQ, par = (qm / NQ) & 1;
          ++qm;
          if (!wwait(&bars[L::bQFull + qs], par)) { stop = true; break; }
          const uint8_t *tile = sm + L::kQ + qs * kTB;
#pragma unroll 4
          for (int idx = ct; idx < kTile * kCpr; idx += 64) {
            const int r = idx / kCpr, piece = idx % kCpr, c = piece >> 3, k8 = piece & 7;
            const int i = w.m[x] * kTile + r;
            const int4 v = *reinterpret_cast<const int4 *>(tile + c * 16384 + r * 128 + ((k8 ^ (r & 7)) << 4));
            if (i < p.Sq) {
              const uint32_t xw[4] = {static_cast<uint32_t>(v.x), static_cast<uint32_t>(v.y),
                                      static_cast<uint32_t>(v.z), static_cast<uint32_t>(v.w)};
              uint32_t hw[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                in_max = __vmaxu2(in_max, xw[e] & 0x7fff7fffu);
                hw[e] = bf16x2_to_f16x2(xw[e]);
              }
              *reinterpret_cast<int4 *>(p.q16 + ((static_cast<int64_t>(w.b) * p.Sq + i) * p.H + w.h) * D +
                                        piece * 8) = make_int4(hw[0], hw[1], hw[2], hw[3]);
            }
          }
          mbar_arrive(&bars[L::bQEmpty + qs]);
        }
      }
      // |x| >= 65536 (bf16 bits 0x4780), infinities and NaNs: beyond what fp16 holds
      if ((in_max & 0xffffu) >= 0x4780u || (in_max >> 16) >= 0x4780u)
        record_status(p.hdr + kHdrStatus, BSA_ERR_INPUT_RANGE);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax, group x
    const int x = (warp - 4) >> 2;  // 0: q-block 2g, 1: q-block 2g+1
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t t_s = tmem + lane_off + x * 128;
    const uint32_t t_o = tmem + lane_off + 256 + x * D;
    const MaskParams &mk = p.mask;
    const bool use_seg = mk.seg_q != nullptr;
    // every lane waits, then the warp agrees, so tcgen05 .sync.aligned ops
    // never run on a diverged warp even when the watchdog trips
    auto wwait = [&](uint64_t *bar, uint32_t parity) {
      return __all_sync(0xffffffffu, wd.wait(bar, parity)) != 0;
    };
    uint32_t tcount = 0, ps = 0, qm = 0;
    bool stop = false;
    for (uint32_t tc = 0; !stop; ++tc) {
      const uint32_t slot = tc & 1;
      if (!wwait(&bars[L::bTkFull + slot], (tc >> 1) & 1)) break;
      FwdUnit w;
      const bool valid = read_unit(unit_ring + slot * kUnitWords, w);
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[L::bTkEmpty + slot]);
      if (!valid) break;
      // the unit's Q tiles sit in the Q ring in load order (A, then B), as the
      // producer and the MMA warp count them
      const bool has0 = w.re[0] > w.rs[0], has1 = w.re[1] > w.rs[1];
      const uint32_t q_i = qm + (x == 1 && has0 ? 1u : 0u);
      qm += (has0 ? 1u : 0u) + (has1 ? 1u : 0u);
      if (w.m[x] >= p.nM) continue;
      const int rs = w.rs[x], re = w.re[x], nt = re - rs;
      const int b = w.b, h = w.h, bh = w.bh;
      const int i = w.m[x] * kTile + r;
      const bool row_ok = i < p.Sq;
      if (nt == 0) {
        if (row_ok) {
          __nv_bfloat16 *orow = p.out + b * p.o_sb + static_cast<int64_t>(i) * p.o_ss + h * p.o_sh;
          float *lse_p = p.lse + static_cast<int64_t>(bh) * p.Sq + i;
          const int4 z = make_int4(0, 0, 0, 0);
#pragma unroll
          for (int c = 0; c < D / 8; ++c) reinterpret_cast<int4 *>(orow)[c] = z;
          *lse_p = -INFINITY;
        }
        continue;
      }
      bool fixed = p.fixed_mode && !p.block_bound && p.gate[bh] != 0;
      float m_ref = -INFINITY, l = 0.f, l_r = 0.f;
      if (fixed)
        m_ref = row_ok ? p.scale_log2 * fmaf(p.qnorm[static_cast<int64_t>(bh) * p.Sq + i], p.kmax[bh],
                                             p.qdot != nullptr ? p.qdot[static_cast<int64_t>(bh) * p.Sq + i] : 0.f)
                       : 0.f;
      if (p.fixed_mode && p.block_bound) {
        // per q-block bound: kmax_m over the key blocks of this q-block's row
        // list (each warp reduces it), ||q_i|| from this row of the Q tile,
        // and the gate per row
        const int hk = h / p.kv_group;
        const float *kb = p.kblk + (static_cast<int64_t>(b) * p.Hk + hk) * p.nN;
        float km = 0.f;
        for (int jj = rs + lane; jj < re; jj += 32) km = fmaxf(km, kb[p.row_ent[jj] & kIndexMask]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) km = fmaxf(km, __shfl_xor_sync(0xffffffffu, km, o));
        if (!wwait(&bars[L::bQFull + q_i % NQ], (q_i / NQ) & 1)) { stop = true; break; }
        const uint8_t *qt = sm + L::kQ + (q_i % NQ) * kTB + r * 128;
        float ss = 0.f;
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
#pragma unroll
          for (int k8 = 0; k8 < 8; ++k8) {
            const int4 v = *reinterpret_cast<const int4 *>(qt + c * 16384 + ((k8 ^ (r & 7)) << 4));
            const uint32_t xw[4] = {static_cast<uint32_t>(v.x), static_cast<uint32_t>(v.y),
                                    static_cast<uint32_t>(v.z), static_cast<uint32_t>(v.w)};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f2 = unpack_bf16x2(xw[e]);
              ss = fmaf(f2.x, f2.x, fmaf(f2.y, f2.y, ss));
            }
          }
        }
        const float qn = sqrtf(ss);
        fixed = 2.f * p.scale * qn * km <= p.gate_limit;
        if (fixed) m_ref = p.scale_log2 * qn * km;
        if (r == 0) p.kmax_q[static_cast<int64_t>(bh) * p.nM + w.m[x]] = km;
      }
      if (p.fixed_mode) {
        const uint32_t nf = __popc(__ballot_sync(0xffffffffu, fixed && row_ok));
        if (lane == 0 && nf != 0u) atomicAdd(p.hdr + kHdrFixedRows, nf);
      }
      // row-constant part of the mask: allowed keys lie in [lo, hi] (the
      // window, thinned by the dilation) or in the prefix [0, pre_hi]
      int lo = 0, hi = p.Skv - 1, pre_hi = -1;
      if (mk.flags & BSA_MASK_KV_VALID_LEN) hi = min(hi, mk.kv_valid_len[b] - 1);
      if (mk.prefix_len != nullptr) pre_hi = min(hi, mk.prefix_len[b] - 1);
      if (mk.flags & BSA_MASK_CAUSAL_WINDOW) {
        hi = min(hi, i + mk.offset);
        if (mk.window > 0) lo = max(lo, i + mk.offset - mk.window + 1);
      }
      const int seg_i = (use_seg && row_ok) ? mk.seg_q[static_cast<int64_t>(b) * p.Sq + i] : INT_MIN;

      // the tile's list word is fetched one tile ahead, its latency under the
      // previous tile's softmax
      uint32_t ent_next = p.row_ent[rs];
      for (int j = rs; j < re; ++j, ++tcount) {
        const uint32_t ent = ent_next;
        if (j + 1 < re) ent_next = p.row_ent[j + 1];
        const int n = static_cast<int>(ent & kIndexMask);
        const bool full = (ent & kFullBit) != 0;
        // allowed-key bits of this tile for this row (range AND segment ids),
        // built before the S row occupies registers
        uint32_t allow[4] = {~0u, ~0u, ~0u, ~0u};
        if (!full) {
#pragma unroll
          for (int q = 0; q < 4; ++q) allow[q] = range_bits(lo - n * kTile, hi - n * kTile, q);
          if (mk.dilation > 1) {
            // keep key j iff (i + o - j) mod d == 0: bit k of word q is key
            // 128n + 32q + k, kept iff k == (i + o - 128n - 32q) mod d
            int ph = (i + mk.offset - n * kTile) % mk.dilation;
            if (ph < 0) ph += mk.dilation;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              allow[q] &= ph < 32 ? (mk.dil_pattern << ph) : 0u;
              ph -= mk.dil_r32;
              if (ph < 0) ph += mk.dilation;
            }
          }
          if (pre_hi >= 0) {
#pragma unroll
            for (int q = 0; q < 4; ++q) allow[q] |= range_bits(-n * kTile, pre_hi - n * kTile, q);
          }
          if (use_seg) {
            int32_t *segt = seg_sm + (x * 2 + (ps & 1)) * kTile;
            const int jj = n * kTile + r;
            segt[r] = jj < p.Skv ? mk.seg_kv[static_cast<int64_t>(b) * p.Skv + jj] : INT_MIN + 1;
            mbar_arrive(&bars[L::bSegReady + x * 2 + (ps & 1)]);
            if (!wwait(&bars[L::bSegReady + x * 2 + (ps & 1)], (ps >> 1) & 1)) { stop = true; break; }
            ++ps;
            const int4 *seg4 = reinterpret_cast<const int4 *>(segt);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint32_t bits = 0;
#pragma unroll
              for (int t = 0; t < 8; ++t) {
                const int4 v = seg4[q * 8 + t];
                bits |= (static_cast<uint32_t>(v.x == seg_i) << (4 * t)) |
                        (static_cast<uint32_t>(v.y == seg_i) << (4 * t + 1)) |
                        (static_cast<uint32_t>(v.z == seg_i) << (4 * t + 2)) |
                        (static_cast<uint32_t>(v.w == seg_i) << (4 * t + 3));
              }
              allow[q] &= bits;
            }
          }
        }
        if (!wwait(&bars[L::bSFull + x], tcount & 1)) { stop = true; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, !fixed)) {
          // pass 1: the tile's row max (masked); rows whose reference is
          // pinned never rise above it, so they take no rescale
          float mx = -INFINITY;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t sv[32];
            tmem_ld32(t_s + 32 * c, sv);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 32; ++q) {
              const float v = ((allow[c] >> q) & 1u) ? __uint_as_float(sv[q]) : -INFINITY;
              mx = fmaxf(mx, v);
            }
          }
          const float mt = mx * p.scale_log2;
          const bool need = mt > m_ref + kRescaleThreshold;
          const bool resc = need && l > 0.f;
          float alpha = 1.f;
          if (need) {
            alpha = fast_exp2(m_ref - mt);
            l *= alpha;
            l_r *= alpha;
            m_ref = mt;
          }
          if (__any_sync(0xffffffffu, resc)) {
            if (!wwait(&bars[L::bPVDone + x], (tcount - 1) & 1)) { stop = true; break; }
            tc_fence_after();
            const float a = resc ? alpha : 1.f;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t o[32];
              tmem_ld32(t_o + c * 32, o);
              tmem_wait_ld();
#pragma unroll
              for (int q = 0; q < 32; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * a);
              tmem_st32(t_o + c * 32, o);
            }
            tmem_wait_st();
          }
        }
        // pass 2: P = exp2(s * scale * log2e - m) in bf16, packed over the first 64 S columns
        const float mu = (m_ref == -INFINITY) ? 0.f : m_ref;
        const float2 sc2 = make_float2(p.scale_log2, p.scale_log2), nmu = make_float2(-mu, -mu);
        float2 rs2 = make_float2(0.f, 0.f), rr2 = make_float2(0.f, 0.f);
        // eight 16-column pieces; the next piece's TMEM load is in flight while
        // this one is computed (a wait covers every load issued before it)
        uint32_t svb[2][16];
        tmem_ld16(t_s, svb[0]);
        tmem_wait_ld();
#pragma unroll
        for (int sc = 0; sc < 8; ++sc) {
          if (sc + 1 < 8) tmem_ld16(t_s + 16 * (sc + 1), svb[(sc + 1) & 1]);
          const uint32_t *sv = svb[sc & 1];
          const uint32_t bits = allow[sc >> 1] >> (16 * (sc & 1));
          uint32_t pk[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float2 t = __ffma2_rn(
                make_float2(__uint_as_float(sv[2 * q]), __uint_as_float(sv[2 * q + 1])), sc2, nmu);
            float p0 = fast_exp2(t.x), p1 = fast_exp2(t.y);
            if (!full) {
              p0 = ((bits >> (2 * q)) & 1u) ? p0 : 0.f;
              p1 = ((bits >> (2 * q + 1)) & 1u) ? p1 : 0.f;
            }
            pk[q] = pack_bf16x2(p0, p1);
            // two row sums: l over the exact weights (for LSE) and l_r over the
            // bf16-rounded weights the PV product uses (normalising O by l_r
            // makes numerator and denominator carry the same rounding)
            rs2 = __fadd2_rn(rs2, make_float2(p0, p1));
            rr2 = __fadd2_rn(rr2, unpack_bf16x2(pk[q]));
          }
          // P piece -> TMEM columns [8sc, 8sc+8): only S columns already read
          tmem_st8(t_s + 8 * sc, pk);
          if (sc + 1 < 8) tmem_wait_ld();
        }
        const float rowsum = rs2.x + rs2.y, rowsum_r = rr2.x + rr2.y;
        l += rowsum;
        l_r += rowsum_r;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars[L::bPFull + x]);
      }
      if (stop) break;
      // epilogue: O / l_r -> bf16, the O residual, LSE
      if (!wwait(&bars[L::bPVDone + x], (tcount - 1) & 1)) break;
      tc_fence_after();
      const float inv = l_r > 0.f ? 1.f / l_r : 0.f;
      __nv_bfloat16 *orow = p.out + b * p.o_sb + static_cast<int64_t>(i) * p.o_ss + h * p.o_sh;
      uint8_t *rrow = p.o_resid != nullptr
                          ? p.o_resid + ((static_cast<int64_t>(b) * p.Sq + i) * p.H + h) * D : nullptr;
      // 16-column pieces of O, the next piece's TMEM load in flight while this
      // one is converted and stored (a wait covers every load issued before
      // it); a piece of O is one 32-byte store, two pieces' residual bytes
      // another
      uint32_t ob[2][16], rb[8];
      tmem_ld16(t_o, ob[0]);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < D / 16; ++c) {
        if (c + 1 < D / 16) tmem_ld16(t_o + (c + 1) * 16, ob[(c + 1) & 1]);
        const uint32_t *o = ob[c & 1];
        if (row_ok) {
          uint32_t wv[8];
#pragma unroll
          for (int q = 0; q < 8; ++q)
            wv[q] = pack_bf16x2(__uint_as_float(o[2 * q]) * inv, __uint_as_float(o[2 * q + 1]) * inv);
          if (p.o_v8) {
            st_global_v8(orow + c * 16, wv);
          } else {
            int4 *dst = reinterpret_cast<int4 *>(orow + c * 16);
            dst[0] = make_int4(wv[0], wv[1], wv[2], wv[3]);
            dst[1] = make_int4(wv[4], wv[5], wv[6], wv[7]);
          }
          if (rrow != nullptr) {
            // what the bf16 rounding of O dropped (exact in fp32), for the
            // backward's Delta; 16 one-byte residuals per piece
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float2 r0 = unpack_bf16x2(wv[2 * q]), r1 = unpack_bf16x2(wv[2 * q + 1]);
              rb[(c & 1) * 4 + q] =
                  pack_resid_e5m2x2(__uint_as_float(o[4 * q]) * inv - r0.x,
                                    __uint_as_float(o[4 * q + 1]) * inv - r0.y) |
                  (pack_resid_e5m2x2(__uint_as_float(o[4 * q + 2]) * inv - r1.x,
                                     __uint_as_float(o[4 * q + 3]) * inv - r1.y)
                   << 16);
            }
            if (c & 1) st_global_v8(rrow + (c - 1) * 16, rb);
          }
        }
        if (c + 1 < D / 16) tmem_wait_ld();
      }
      tc_fence_before();
      float *lse_p = p.lse + static_cast<int64_t>(bh) * p.Sq + i;
      if (row_ok) *lse_p = l > 0.f ? (m_ref + __log2f(l)) * kLn2 : -INFINITY;
      if (fixed && l > 0.f && l < 7.888609052210118e-31f /* 2^-100 */)
        atomicAdd(p.hdr + kHdrGateWarn, 1u);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0) release_ticket(p.hdr + kHdrFwdTicket, p.hdr + kHdrFwdDone);
}

// ---------------------------------------------------------------- fixed-m bound
// Norms of every (row, head) vector of K (blockIdx.y == 0) and Q (== 1): one
// thread per vector, consecutive threads on consecutive heads of a row, each
// keeping kU 16-byte chunks in flight.  Keys: the maximum per (b, h) over valid
// keys (padding and varlen alignment keys excluded), for every query head of
// the key head's group.  Queries: the per-row norm is stored and the maximum per
// (b, h) kept.  With k-smoothing (center != 0) the keys' norms are taken of
// k_j - c and the queries also store q_i . c, c being the mean valid key of
// the head from the fixed-point sums of k_key_sums.  The block that finishes
// last computes the per-head gate.
struct NormArgs {
  const __nv_bfloat16 *k, *q;
  int64_t ks[3], qs[3];
  int B, Skv, Sq, H, Hk, only_q, center;  // Hk: key heads (H / Hk query heads each)
  MaskParams mk;
  float *kmax, *qmax, *qnorm;
  long long *ksum;        // [B, Hk, D] fixed-point sums of the valid keys
  int *kcount;            // [B] valid keys
  float *kbar, *qdot;     // [B, Hk, D] center (written once per batch row), [B, H, Sq]
  uint32_t *done;         // blocks finished (zero before the launch)
  const float *kmax_override;
  float scale, limit;
  int32_t *gate;
};

constexpr float kFixScale = 1048576.f;  // fixed-point unit 2^-20 of the key sums

__device__ __forceinline__ bool key_is_valid(const MaskParams &mk, int b, int j) {
  bool valid = true;
  if (mk.flags & BSA_MASK_KV_VALID_LEN) valid = j < mk.kv_valid_len[b];
  if ((mk.flags & BSA_MASK_VARLEN) && mk.seg_kv != nullptr) valid = valid && mk.seg_kv[j] >= 0;
  return valid;
}

// k-smoothing, first pass: per (b, h, d) the sum over valid keys of k_jd, each
// term rounded to a multiple of 2^-20 (|k| clamped to 2^20) and added as an
// int64, so the total does not depend on the order of the additions; and per
// b the number of valid keys.  A block takes 64 rows of one batch row; a
// thread owns 8 dims of one head and walks the rows.
template <int D>
__global__ void __launch_bounds__(256) k_key_sums(const NormArgs a) {
  constexpr int kRows = 64;
  constexpr int G = D / 8;
  const int64_t blocks_per_b = (a.Skv + kRows - 1) / kRows;
  const int b = static_cast<int>(blockIdx.x / blocks_per_b);
  const int r0 = static_cast<int>(blockIdx.x % blocks_per_b) * kRows;
  const int r1 = min(a.Skv, r0 + kRows);
  if (threadIdx.x == 0) {
    int n = 0;
    for (int r = r0; r < r1; ++r) n += key_is_valid(a.mk, b, r) ? 1 : 0;
    if (n != 0) atomicAdd(a.kcount + b, n);
  }
  const int cols = a.Hk * G;
  for (int c = threadIdx.x; c < cols; c += blockDim.x) {
    const int h = c / G, g = c % G;
    long long acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0;
    const __nv_bfloat16 *base = a.k + b * a.ks[0] + h * a.ks[2] + g * 8;
#pragma unroll 4
    for (int r = r0; r < r1; ++r) {
      if (!key_is_valid(a.mk, b, r)) continue;
      const int4 v = *reinterpret_cast<const int4 *>(base + static_cast<int64_t>(r) * a.ks[1]);
      const __nv_bfloat162 *x = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(x[e]);
        acc[2 * e] += __float2ll_rn(fminf(fmaxf(f.x, -kFixScale), kFixScale) * kFixScale);
        acc[2 * e + 1] += __float2ll_rn(fminf(fmaxf(f.y, -kFixScale), kFixScale) * kFixScale);
      }
    }
    unsigned long long *dst = reinterpret_cast<unsigned long long *>(
        a.ksum + (static_cast<int64_t>(b) * a.Hk + h) * D + g * 8);
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if (acc[e] != 0) atomicAdd(dst + e, static_cast<unsigned long long>(acc[e]));
  }
}

// Per q-block bound, its only pass over the inputs: for each kv block n and key
// head, the largest ||k_j|| over the block's valid keys (padding and varlen
// alignment keys excluded; 0 when none is valid).  One warp per (b, hk, n,
// 32-key quarter): lane l takes key 32 c + l of the block, the row's 16-byte
// pieces all in flight; the warp's maximum goes into the block's slot with an
// integer atomic max (non-negative floats order like their bit patterns; the
// slots are zeroed before the launch).
template <int D>
__global__ void __launch_bounds__(256) k_key_block_max(const NormArgs a, float *__restrict__ kblk, int nN) {
  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= static_cast<int64_t>(a.B) * a.Hk * nN * 4) return;
  const int64_t blk = wid >> 2;
  const int c = static_cast<int>(wid & 3);
  const int n = static_cast<int>(blk % nN);
  const int hk = static_cast<int>((blk / nN) % a.Hk);
  const int b = static_cast<int>(blk / (static_cast<int64_t>(nN) * a.Hk));
  float mx = 0.f;
  const int j = n * kTile + lane + 32 * c;
  if (j < a.Skv && key_is_valid(a.mk, b, j)) {
    const int4 *src = reinterpret_cast<const int4 *>(a.k + b * a.ks[0] + static_cast<int64_t>(j) * a.ks[1] +
                                                     hk * a.ks[2]);
    int4 v[D / 8];
#pragma unroll
    for (int u = 0; u < D / 8; ++u) v[u] = __ldg(src + u);
    float acc = 0.f;
#pragma unroll
    for (int u = 0; u < D / 8; ++u) {
      const uint32_t xw[4] = {static_cast<uint32_t>(v[u].x), static_cast<uint32_t>(v[u].y),
                              static_cast<uint32_t>(v[u].z), static_cast<uint32_t>(v[u].w)};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f2 = unpack_bf16x2(xw[e]);
        acc = fmaf(f2.x, f2.x, acc);
        acc = fmaf(f2.y, f2.y, acc);
      }
    }
    mx = sqrtf(acc);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0 && mx > 0.f) atomicMax(reinterpret_cast<unsigned int *>(kblk) + blk, __float_as_uint(mx));
}

// k-smoothing, second pass: the centers c = sum * 2^-20 / (valid keys).
template <int D>
__global__ void __launch_bounds__(256) k_key_centers(const NormArgs a) {
  const int64_t n = static_cast<int64_t>(a.B) * a.Hk * D;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < n;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int b = static_cast<int>(t / (static_cast<int64_t>(a.Hk) * D));
    const double inv = 1.0 / (static_cast<double>(kFixScale) * max(1, a.kcount[b]));
    a.kbar[t] = static_cast<float>(static_cast<double>(a.ksum[t]) * inv);
  }
}

// D/32 threads per (row, head) vector, each with four 16-byte pieces in
// flight; a block takes kVPB consecutive vectors of one batch row (rows are
// contiguous over heads).  Per-head maxima are reduced in shared memory first,
// then one global atomic per head and block.
// CENTER: k-smoothing on (a.center != 0), a compile-time choice so that the
// plain norm's inner loop carries no per-element test of it
template <int D, bool CENTER>
__global__ void __launch_bounds__(256) k_row_norms(const NormArgs a) {
  constexpr int kT = D / 32;          // threads per vector, four 16-byte loads each
  constexpr int kVPB = 256 / kT;      // vectors per block and pass
  extern __shared__ unsigned int smax[];  // [H]
  __shared__ bool last_block;
  const int is_key = !a.only_q && blockIdx.y == 0;
  const __nv_bfloat16 *x = is_key ? a.k : a.q;
  const int S = is_key ? a.Skv : a.Sq;
  const int64_t sb = is_key ? a.ks[0] : a.qs[0], ss = is_key ? a.ks[1] : a.qs[1],
                sh = is_key ? a.ks[2] : a.qs[2];
  float *rowmax = is_key ? a.kmax : a.qmax;
  const int H = a.H;
  const int Hx = is_key ? a.Hk : H;  // heads of this tensor
  const int grp = H / a.Hk;          // query heads per key head
  const int bpb = static_cast<int>(gridDim.x / a.B);  // blocks per batch row
  const int b = static_cast<int>(blockIdx.x) / bpb, blk = static_cast<int>(blockIdx.x) % bpb;
  for (int h = threadIdx.x; h < H; h += blockDim.x) smax[h] = 0u;
  __syncthreads();
  // Grid-stride over the batch row's (row, head) vectors, consecutive vectors
  // on consecutive heads of a row (the tensor's memory order).  kPass vectors
  // per thread and pass keep 4 * kPass 16-byte loads in flight; the per-head
  // maxima gather in shared memory over the block's whole range, so the
  // global atomics and the fence below happen once per block.
  constexpr int kPass = 2;  // vectors per thread and pass, all loads in flight
  const int64_t nvec = static_cast<int64_t>(S) * Hx;
  const int64_t stride = static_cast<int64_t>(bpb) * kVPB;
  const int t = threadIdx.x % kT;
  // The thread's vectors v0 + k * stride as (row, head) pairs, stepped by a
  // carry instead of a division per vector (vector = row * Hx + head).
  const int64_t v0 = static_cast<int64_t>(blk) * kVPB + threadIdx.x / kT;
  const int d_row = static_cast<int>(stride / Hx), d_hh = static_cast<int>(stride % Hx);
  int row_k = static_cast<int>(v0 / Hx), hh_k = static_cast<int>(v0 % Hx);
  auto step = [&](int &rw, int &hd) {
    hd += d_hh;
    rw += d_row;
    if (hd >= Hx) {
      hd -= Hx;
      ++rw;
    }
  };
  for (int64_t base = static_cast<int64_t>(blk) * kVPB; base < nvec; base += kPass * stride) {
    int rws[kPass], hds[kPass];
#pragma unroll
    for (int j = 0; j < kPass; ++j) {
      rws[j] = row_k;
      hds[j] = hh_k;
      step(row_k, hh_k);
    }
    bool in[kPass];
    int4 w[kPass][4];
#pragma unroll
    for (int j = 0; j < kPass; ++j) {
      in[j] = rws[j] < S;  // the vector is below nvec; no early exit: the shuffles need every lane
      if (in[j]) {
        const int4 *src =
            reinterpret_cast<const int4 *>(x + b * sb + static_cast<int64_t>(rws[j]) * ss + hds[j] * sh) + 4 * t;
#pragma unroll
        for (int u = 0; u < 4; ++u) w[j][u] = __ldg(src + u);
      }
    }
#pragma unroll
    for (int j = 0; j < kPass; ++j) {
      const int row = rws[j], hh = hds[j];
      float acc = 0.f, dot = 0.f;
      if (in[j]) {
        const float *c = CENTER ? a.kbar + (static_cast<int64_t>(b) * a.Hk + (is_key ? hh : hh / grp)) * D + 32 * t
                                : nullptr;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t xw[4] = {static_cast<uint32_t>(w[j][u].x), static_cast<uint32_t>(w[j][u].y),
                                  static_cast<uint32_t>(w[j][u].z), static_cast<uint32_t>(w[j][u].w)};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float2 f = unpack_bf16x2(xw[q]);
            if (CENTER) {
              const float2 cc = *reinterpret_cast<const float2 *>(c + 8 * u + 2 * q);
              if (is_key) {
                f.x -= cc.x;
                f.y -= cc.y;
              } else {
                dot = fmaf(f.x, cc.x, dot);
                dot = fmaf(f.y, cc.y, dot);
              }
            }
            acc = fmaf(f.x, f.x, acc);
            acc = fmaf(f.y, f.y, acc);
          }
        }
      }
#pragma unroll
      for (int o = kT / 2; o > 0; o >>= 1) {
        acc += __shfl_xor_sync(0xffffffffu, acc, o);
        dot += __shfl_xor_sync(0xffffffffu, dot, o);
      }
      if (in[j] && t == 0) {
        const float nrm = sqrtf(acc);
        bool valid = true;
        if (is_key) {
          valid = key_is_valid(a.mk, b, row);
        } else {
          const int64_t idx = (static_cast<int64_t>(b) * H + hh) * S + row;
          a.qnorm[idx] = nrm;
          if (CENTER) a.qdot[idx] = dot;
        }
        if (valid) atomicMax(&smax[hh], __float_as_uint(nrm));
      }
    }
  }
  __syncthreads();
  // a key head's maximum goes to every query head of its group
  for (int h = threadIdx.x; h < Hx; h += blockDim.x)
    if (smax[h] != 0u) {
      if (is_key) {
        for (int i = 0; i < grp; ++i)
          atomicMax(reinterpret_cast<unsigned int *>(rowmax) + b * H + h * grp + i, smax[h]);
      } else {
        atomicMax(reinterpret_cast<unsigned int *>(rowmax) + b * H + h, smax[h]);
      }
    }
  // the last block to finish takes the gate decision for every (b, h)
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t n = gridDim.x * gridDim.y;
    last_block = atomicAdd(a.done, 1u) == n - 1u;
  }
  __syncthreads();
  if (!last_block) return;
  __threadfence();
  const int BH = a.B * H;
  for (int i = threadIdx.x; i < BH; i += blockDim.x) {
    const float km = a.kmax_override != nullptr ? a.kmax_override[i] : __ldcg(a.kmax + i);
    a.kmax[i] = km;
    a.gate[i] = (2.f * a.scale * __ldcg(a.qmax + i) * km <= a.limit) ? 1 : 0;
  }
  if (threadIdx.x == 0) *a.done = 0u;
}

int sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

template <int D, int NQ, int NK, int NV>
cudaError_t run_fwd(const FwdParams &fp, const CUtensorMap &tq, const CUtensorMap &tk,
                    const CUtensorMap &tv, cudaStream_t s) {
  using L = FwdSmem<D, NQ, NK, NV>;
  static_assert(L::kAlloc <= 232448, "shared memory budget");
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(k_attn_fwd<D, NQ, NK, NV>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  // the unit ticket is zero: the plan build clears it and every launch's
  // last CTA puts it back
  const int grid = std::min(fp.n_units, sm_count());
  k_attn_fwd<D, NQ, NK, NV><<<grid, 384, L::kAlloc, s>>>(tq, tk, tv, fp);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fixed_m_bound(const bsa_problem &p, const MaskParams &mp,
                                 const bsa_options &o, const void *q, const void *k,
                                 const WsLayout &L, uint8_t *ws, cudaStream_t s) {
  NormArgs na{};
  na.k = static_cast<const __nv_bfloat16 *>(k);
  na.q = static_cast<const __nv_bfloat16 *>(q);
  for (int i = 0; i < 3; ++i) {
    na.ks[i] = p.k_stride[i];
    na.qs[i] = p.q_stride[i];
  }
  na.B = p.B;
  na.Skv = p.Skv;
  na.Sq = p.Sq;
  na.H = p.H;
  na.Hk = p.H_kv;
  na.only_q = o.kmax_override != nullptr;  // a caller-supplied kmax needs no key pass
  na.center = o.bound_mode == BSA_BOUND_SMOOTHED;
  na.mk = mp;
  na.kmax = reinterpret_cast<float *>(ws + L.kmax);
  na.qmax = reinterpret_cast<float *>(ws + L.qmax);
  na.done = reinterpret_cast<uint32_t *>(ws + L.qmax) + p.B * p.H;
  na.qnorm = reinterpret_cast<float *>(ws + L.qnorm);
  na.ksum = reinterpret_cast<long long *>(ws + L.ksum);
  na.kcount = reinterpret_cast<int *>(ws + L.kcount);
  na.kbar = reinterpret_cast<float *>(ws + L.kbar);
  na.qdot = reinterpret_cast<float *>(ws + L.qdot);
  na.kmax_override = o.kmax_override;
  na.scale = p.scale;
  na.limit = o.gate_limit > 0.f ? o.gate_limit : 64.f;
  na.gate = reinterpret_cast<int32_t *>(ws + L.gate);
  if (o.bound_mode == BSA_BOUND_BLOCK) {
    // the per q-block bound reads K only; the forward takes the rest
    const int64_t warps = static_cast<int64_t>(p.B) * p.H_kv * L.nN * 4;
    const unsigned blocks = static_cast<unsigned>((warps * 32 + 255) / 256);
    float *kblk = reinterpret_cast<float *>(ws + L.kbmax);
    cudaError_t e0 = cudaMemsetAsync(kblk, 0, sizeof(float) * static_cast<size_t>(p.B) * p.H_kv * L.nN, s);
    if (e0 != cudaSuccess) return e0;
    if (p.D == 64) k_key_block_max<64><<<blocks, 256, 0, s>>>(na, kblk, L.nN);
    else k_key_block_max<128><<<blocks, 256, 0, s>>>(na, kblk, L.nN);
    count_launch();
    return cudaGetLastError();
  }
  // kmax, qmax and the finished-block counter are adjacent: one memset
  cudaError_t e = cudaMemsetAsync(na.kmax, 0, sizeof(float) * p.B * p.H * 2 + sizeof(uint32_t), s);
  if (e != cudaSuccess) return e;
  const size_t smem = sizeof(unsigned int) * p.H;
  if (na.center) {
    // ksum and kcount are adjacent regions: one memset
    e = cudaMemsetAsync(ws + L.ksum, 0, L.qdot - L.ksum, s);
    if (e != cudaSuccess) return e;
    const unsigned sblocks = static_cast<unsigned>(static_cast<int64_t>(p.B) * ((p.Skv + 63) / 64));
    const unsigned cblocks = static_cast<unsigned>((static_cast<int64_t>(p.B) * p.H_kv * p.D + 255) / 256);
    if (p.D == 64) {
      k_key_sums<64><<<sblocks, 256, 0, s>>>(na);
      k_key_centers<64><<<cblocks, 256, 0, s>>>(na);
    } else {
      k_key_sums<128><<<sblocks, 256, 0, s>>>(na);
      k_key_centers<128><<<cblocks, 256, 0, s>>>(na);
    }
    count_launch(2);
  }
  // blocks per batch row: about two per SM over the whole grid (each thread
  // keeps eight 16-byte loads in flight, which covers the memory latency), and
  // no more than the larger tensor's vectors fill at 256 / (D / 32) per block.
  // Two leave an SM's other half of threads and registers to the planner,
  // which runs beside this pass on the library's side stream; four measured
  // the same pass time but kept the planner waiting for a free SM.
  const int64_t vec = static_cast<int64_t>(std::max(p.Sq * p.H, p.Skv * p.H_kv));
  const int64_t vpb = 256 / (p.D / 32);
  const int64_t want = std::max<int64_t>(1, (2 * 148) / (static_cast<int64_t>(p.B) * (na.only_q ? 1 : 2)));
  const int bpb = static_cast<int>(std::min<int64_t>(want, (vec + vpb - 1) / vpb));
  const dim3 grid(static_cast<unsigned>(p.B * bpb), na.only_q ? 1u : 2u);
  if (p.D == 64) {
    if (na.center) k_row_norms<64, true><<<grid, 256, smem, s>>>(na);
    else k_row_norms<64, false><<<grid, 256, smem, s>>>(na);
  } else {
    if (na.center) k_row_norms<128, true><<<grid, 256, smem, s>>>(na);
    else k_row_norms<128, false><<<grid, 256, smem, s>>>(na);
  }
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_fwd(const bsa_problem &p, const MaskParams &mp, const bsa_options &o,
                       const PlanSignature &sig, const CUtensorMap &tq, const CUtensorMap &tk,
                       const CUtensorMap &tv, const void *q, void *out, float *lse,
                       const WsLayout &L, uint8_t *ws, cudaStream_t s) {
  FwdParams fp{};
  fp.q = static_cast<const __nv_bfloat16 *>(q);
  fp.mask = mp;
  fp.B = p.B;
  fp.H = p.H;
  fp.Sq = p.Sq;
  fp.Skv = p.Skv;
  fp.nM = L.nM;
  fp.kv_group = p.H / p.H_kv;
  {
    // split the pairs of a last wave that is at most half full into singles
    const int pairs = p.B * p.H * ((L.nM + 1) / 2);
    const int grid0 = std::min(pairs, sm_count());
    const int r = pairs % grid0;
    fp.n_pairs = (r != 0 && 2 * r <= grid0) ? pairs - r : pairs;
    fp.n_units = pairs + (pairs - fp.n_pairs);
    // the largest divisor of B * H whose heads' K and V (4 D Skv bytes each)
    // fit in 64 MB, half the L2
    const int BH = p.B * p.H;
    const int64_t per_head = 4ll * p.D * p.Skv;
    const int64_t fit = std::max<int64_t>(1, (int64_t{64} << 20) / per_head);
    fp.head_group = 1;
    for (int d = 1; d <= BH; ++d)
      if (BH % d == 0 && d <= fit) fp.head_group = d;
  }
  fp.scale = p.scale;
  fp.scale_log2 = p.scale * kLog2e;
  fp.row_ptr = reinterpret_cast<const int32_t *>(ws + L.row_ptr);
  fp.row_ent = reinterpret_cast<const uint32_t *>(ws + L.row_ent);
  fp.out = static_cast<__nv_bfloat16 *>(out);
  fp.o_sb = p.o_stride[0];
  fp.o_ss = p.o_stride[1];
  fp.o_sh = p.o_stride[2];
  fp.o_v8 = (reinterpret_cast<uintptr_t>(out) & 31u) == 0 && p.o_stride[0] % 16 == 0 &&
            p.o_stride[1] % 16 == 0 && p.o_stride[2] % 16 == 0;
  fp.lse = lse;
  fp.fixed_mode = o.softmax_mode == BSA_SOFTMAX_FIXED_M_GATED;
  fp.block_bound = o.bound_mode == BSA_BOUND_BLOCK;
  fp.gate_limit = o.gate_limit > 0.f ? o.gate_limit : 64.f;
  fp.Hk = p.H_kv;
  fp.nN = L.nN;
  fp.kblk = reinterpret_cast<const float *>(ws + L.kbmax);
  fp.kmax_q = reinterpret_cast<float *>(ws + L.kmax_q);
  fp.kmax = reinterpret_cast<const float *>(ws + L.kmax);
  fp.qnorm = reinterpret_cast<const float *>(ws + L.qnorm);
  fp.qdot = o.bound_mode == BSA_BOUND_SMOOTHED ? reinterpret_cast<const float *>(ws + L.qdot) : nullptr;
  fp.o_resid = o.o_residual == BSA_O_RESIDUAL_KEEP ? ws + L.o_resid : nullptr;
  // the fp16 copy of Q for the backward goes with the residual
  fp.q16 = fp.o_resid != nullptr ? reinterpret_cast<__half *>(ws + L.q16) : nullptr;
  fp.q_sb = p.q_stride[0];
  fp.q_ss = p.q_stride[1];
  fp.q_sh = p.q_stride[2];
  fp.gate = reinterpret_cast<const int32_t *>(ws + L.gate);
  fp.hdr = reinterpret_cast<uint32_t *>(ws + L.status);
  fp.timeout_ns = 2000000000ull;
  for (int i = 0; i < kSigWords; ++i) fp.sig[i] = sig.w[i];
  // the forward does not depend on the kv-column order
  fp.sig_mask = ((1u << kSigWords) - 1u) & ~(1u << kSigOrderWord);
  if (p.D == 64) return run_fwd<64, 3, 4, 4>(fp, tq, tk, tv, s);
  return run_fwd<128, 3, 2, 2>(fp, tq, tk, tv, s);
}

}  // namespace bsa
