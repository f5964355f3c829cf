// Backward pass (steps a4, a5 and a7 of the hot path).
//
// a4  preprocess: Delta_i = sum_d dO_id O_id (fp32) for every query row.
// a5  main loop per kv column n (CTA = (b, kv head, n)): K_n and V_n stay in shared
//     memory; for each q-block m of the column's rank-sorted list the CTA
//     recomputes S^T = K_n Q_m^T and dP^T = V_n dO_m^T, forms
//     P^T = exp(S^T - LSE) (masked on PARTIAL tiles) and dS^T = P^T o (dP^T - Delta),
//     accumulates dV += P^T dO_m and dK += dS^T Q_m in TMEM, computes
//     dQ_m part = dS K_n and adds it to the fp32 dQ accumulator.  With the
//     deterministic protocol the add for q-block m waits until the per-m_block
//     semaphore equals rank(m, n), then increments it, so every dQ row sums its
//     contributions in the fixed order pi (the semaphore is kept per 32-row
//     quarter of the block, one chain per dQ warp; "Add more optimal dk order optional
//     arg", flash-attention PR #2512, "Sliding window perf issue" and "A simplish
//     fix").  Columns are handed out by an atomic ticket in pi order, so a column
//     only ever waits on columns that some running CTA already holds.
// a7  convert: dQ = bf16(dQ accumulator).
//
// Grouped-query attention: a ticket is a kv column of one kv head; the CTA
// walks the column's list once per query head of the group, so dK_n and dV_n
// sum the group's contributions in TMEM and are written once.
// sm_100a roles (512 threads, one CTA per SM, persistent over tickets):
//   warp 0      ticket + TMA producer (K_n, V_n once per column; Q_m, dO_m per entry)
//   warp 1      TMEM owner and tcgen05.mma issuer (one lane)
//   warps 4..11 compute: one key row per thread (TMEM lane) and half of the 128
//               query columns per warp (two warps per lane quarter), the allowed-
//               query mask of PARTIAL tiles (a prefix key is seen by every query;
//               other keys by a query range thinned by the dilation, AND segment
//               ids), P^T back to TMEM as the
//               A operand of dV, dS^T to TMEM over the read dP^T columns (the A
//               operand of dK) and to shared memory (128-byte swizzle, read
//               MN-major as the A operand of dQ), dK/dV epilogue
//   warps 12..15 dQ: one query row per thread; each warp waits on and releases
//               its own quarter's semaphore around its vector reductions
// TMEM columns: S^T / P^T [0,128)  dP^T / dQ [128,256)  dV [256,256+D)  dK [256+D,256+2D)
#include <cfloat>

#include "internal.h"
#include "ptx.cuh"

namespace bsa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;

struct BwdParams {
  MaskParams mask;
  int B, H, Sq, Skv, nM, nN, n_tickets;
  int H_kv, kv_group;  // key/value heads; query heads per kv head
  float scale, scale_log2;
  const int32_t *col_ptr;
  const uint32_t *col_ent;
  const int32_t *col_rank;
  const int32_t *perm;
  const float *lse;    // [B, H, Sq]
  const float *delta;  // [B, H, nM*128]
  float *dq_accum;     // [B, H, nM, D/4, 128, 4]
  uint32_t *sem;       // [B, H, nM]
  __nv_bfloat16 *dk, *dv;
  int64_t k_sb, k_ss, k_sh, v_sb, v_ss, v_sh;
  int deterministic;
  uint32_t *hdr;
  uint64_t timeout_ns, sem_timeout_ns;
  uint32_t sig[kSigWords];
  uint32_t sig_mask;
};

template <int D, int NQ, int NDO>
struct BwdSmem {
  static constexpr int kTB = kTile * D * 2;
  static constexpr int kK = 0;
  static constexpr int kV = kK + kTB;
  static constexpr int kDS = kV + kTB;           // dS^T, 128 x 128 bf16
  static constexpr int kQ = kDS + 32768;
  static constexpr int kDO = kQ + NQ * kTB;
  static constexpr int kVec = kDO + NDO * kTB;   // -LSE*log2e [2][128], -Delta [2][128]
  static constexpr int kTk = kVec + 2 * 2 * kTile * 4;  // ticket ring int[2]
  static constexpr int kBar = kTk + 16;
  // kK and kV are two 32 KB buffers X[0], X[1] that swap the K and V roles
  // from one column to the next (column c: K in X[c & 1], V in the other)
  static constexpr int bTkFull = 0, bTkEmpty = 2, bKFull = 4, bVFull = 5, bXFree = 6, bQFull = 8,
                       bQEmpty = bQFull + NQ, bDOFull = bQEmpty + NQ, bDOEmpty = bDOFull + NDO,
                       bSFull = bDOEmpty + NDO, bDPFull = bSFull + 1, bPReady = bDPFull + 1,
                       bDSReady = bPReady + 1, bDSFree = bDSReady + 1, bDQFull = bDSFree + 1,
                       bDQFree = bDQFull + 1, bDKVFull = bDQFree + 1, bDKVFree = bDKVFull + 1,
                       bVecReady = bDKVFree + 1, bKConv = bVecReady + 2, bVConv = bKConv + 1,
                       bFinal = bVConv + 1, kNumBars = bFinal + 1;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kAlloc = kMisc + 16;
};

constexpr int kThreads = 512;
constexpr int kLaunchRegs = 65536 / kThreads;  // 128: the whole register file
constexpr int kConsumersPerTicket = 1 + 8 + 4 + 2;  // MMA lane, compute warps, dQ warps, converters
constexpr int kComputeThreads = 256;
constexpr int kConvThreads = 64;  // warps 2 and 3

__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(a, parity)) {
    if (globaltimer_ns() - t0 > 200000000ull) return;
  }
}

// Bounded acquire-spin on a dQ semaphore; gives up (false) on timeout or when
// another CTA has already recorded an error.
__device__ bool sem_wait(const uint32_t *sem, uint32_t target, uint64_t limit_ns,
                         uint32_t *status) {
  if (ld_acquire_gpu(sem) == target) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (ld_acquire_gpu(sem) == target) return true;
    if ((it & 63u) == 0u) {
      if (*reinterpret_cast<volatile uint32_t *>(status) != 0u) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        record_status(status, BSA_ERR_SEM_TIMEOUT);
        return false;
      }
    }
    __nanosleep(32);
  }
}

// A ticket is one kv column n of one (b, kv head hk).  Its work is the
// column's entry list once per query head of the group (h0 .. h0+g-1), walked
// as one flat sequence x = 0 .. tot-1: query head h0 + x / len, entry
// es + x % len.  dK_n and dV_n accumulate over the whole sequence.
struct Ticket {
  int valid, b, hk, h0, n, es, ee, len, tot;
  __device__ __forceinline__ int entry(int x) const { return es + x % len; }
  __device__ __forceinline__ int head(int x) const { return h0 + x / len; }
};

__device__ __forceinline__ Ticket decode_ticket(const BwdParams &p, int t) {
  Ticket k{};
  if (t < 0 || t >= p.n_tickets) return k;
  const int BHk = p.B * p.H_kv;
  const int pos = t / BHk, bhk = t % BHk;
  k.valid = 1;
  k.b = bhk / p.H_kv;
  k.hk = bhk % p.H_kv;
  k.h0 = k.hk * p.kv_group;
  k.n = p.perm[pos];
  k.es = p.col_ptr[k.b * p.nN + k.n];
  k.ee = p.col_ptr[k.b * p.nN + k.n + 1];
  k.len = k.ee - k.es;
  k.tot = k.len * p.kv_group;
  return k;
}

template <int D, int NQ, int NDO>
__global__ void __launch_bounds__(kThreads, 1)
k_attn_bwd(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
           const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo,
           const BwdParams p) {
  using L = BwdSmem<D, NQ, NDO>;
  extern __shared__ __align__(1024) uint8_t sm[];
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::kBar);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::kMisc);
  int *abort_flag = reinterpret_cast<int *>(sm + L::kMisc + 4);
  volatile int *tk_ring = reinterpret_cast<volatile int *>(sm + L::kTk);
  float *vec_nl = reinterpret_cast<float *>(sm + L::kVec);  // [2][128] -LSE*log2e
  float *vec_nd = vec_nl + 2 * kTile;                        // [2][128] -Delta

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kTB = L::kTB;

  if (threadIdx.x == 0) {
    for (int i = 0; i < L::kNumBars; ++i) {
      uint32_t cnt = 1;
      if (i == L::bTkEmpty || i == L::bTkEmpty + 1) cnt = kConsumersPerTicket;
      if (i == L::bPReady || i == L::bDSReady || i == L::bDKVFree || i == L::bVecReady ||
          i == L::bVecReady + 1)
        cnt = kComputeThreads;
      if (i == L::bDQFree) cnt = 128;
      if (i == L::bKConv || i == L::bVConv) cnt = kConvThreads;
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
    tma_prefetch_desc(&tdo);
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
  }
  __syncthreads();
  // launched as a programmatic dependent of the Delta pass: the setup above
  // touches only the plan header; Delta, the semaphores and the accumulator
  // are read after the pass has completed.  The dQ convert may then launch.
  pdl_wait();
  pdl_trigger();

  const uint32_t T_S = tmem, T_DP = tmem + 128, T_DV = tmem + 256, T_DK = tmem + 256 + D;
  // every operand is fp16: Q, K, V, dO converted in shared memory by the
  // converter warps, P^T and dS^T written as fp16 by the compute warps
  constexpr uint32_t kIdS = idesc_f16_f32(128, 128, 0, 0);      // S^T, dP^T: both K-major
  constexpr uint32_t kIdKV = idesc_f16_f32(128, D, 0, 1);       // dV (TS), dK: B MN-major
  constexpr uint32_t kIdQ = idesc_f16_f32(128, D, 1, 1);        // dQ: A and B MN-major

  // register budgets, set first thing in each warpgroup's branch: 96 for the
  // producer / MMA warpgroup, 128 for each compute warpgroup, 160 for the dQ
  // warpgroup (its rows are 128 fp32 values each): 96 + 128 + 128 + 160 =
  // 4 x 128, the launch's share
  const bool run = !wd.aborted();
  if (warp < 4) {
    regs_dec<96>();
    if (run && warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t tc = 0, cc = 0, ec = 0, kv_issued = 0, q_issued = 0, do_issued = 0;
      for (;; ++tc) {
        const uint32_t slot = tc & 1;
        if (tc >= 2 && !wd.wait(&bars[L::bTkEmpty + slot], ((tc >> 1) - 1) & 1)) break;
        const int t = static_cast<int>(atomicAdd(p.hdr + kHdrBwdTicket, 1u));
        tk_ring[slot] = t < p.n_tickets ? t : -1;
        mbar_arrive(&bars[L::bTkFull + slot]);
        const Ticket k = decode_ticket(p, t);
        if (!k.valid) break;
        if (k.ee == k.es) continue;
        bool stop = false;
        for (int x = 0; x < k.tot; ++x, ++ec) {
          const int e = k.entry(x), h = k.head(x);
          const int m = static_cast<int>(p.col_ent[e] & kIndexMask);
          const uint32_t qs = ec % NQ, ds = ec % NDO;
          if (ec >= NQ && !wd.wait(&bars[L::bQEmpty + qs], ((ec / NQ) - 1) & 1)) { stop = true; break; }
          mbar_arrive_expect_tx(&bars[L::bQFull + qs], kTB);
          for (int c = 0; c < D / 64; ++c)
            tma_load_4d(sm + L::kQ + qs * kTB + c * 16384, &tq, &bars[L::bQFull + qs], c * 64,
                        m * kTile, h, k.b);
          ++q_issued;
          if (x == 0) {
            // K_n goes where the previous column kept V, free once that
            // column's last dP^T is done, so it loads under the previous
            // column's last entry; V_n then goes where the previous K was,
            // free after the previous column's last dQ
            const int kb = cc & 1, vb = kb ^ 1;
            if (cc >= 1 && !wd.wait(&bars[L::bXFree + kb], (cc - 1) & 1)) { stop = true; break; }
            mbar_arrive_expect_tx(&bars[L::bKFull], kTB);
            for (int c = 0; c < D / 64; ++c)
              tma_load_4d(sm + L::kK + kb * kTB + c * 16384, &tk, &bars[L::bKFull], c * 64,
                          k.n * kTile, k.hk, k.b);
            if (cc >= 1 && !wd.wait(&bars[L::bXFree + vb], (cc - 1) & 1)) { stop = true; break; }
            mbar_arrive_expect_tx(&bars[L::bVFull], kTB);
            for (int c = 0; c < D / 64; ++c)
              tma_load_4d(sm + L::kK + vb * kTB + c * 16384, &tv, &bars[L::bVFull], c * 64,
                          k.n * kTile, k.hk, k.b);
            ++kv_issued;
          }
          if (ec >= NDO && !wd.wait(&bars[L::bDOEmpty + ds], ((ec / NDO) - 1) & 1)) { stop = true; break; }
          mbar_arrive_expect_tx(&bars[L::bDOFull + ds], kTB);
          for (int c = 0; c < D / 64; ++c)
            tma_load_4d(sm + L::kDO + ds * kTB + c * 16384, &tdo, &bars[L::bDOFull + ds], c * 64,
                        m * kTile, h, k.b);
          ++do_issued;
        }
        if (stop) break;
        ++cc;
      }
      if (wd.aborted()) {
        for (uint32_t t = (q_issued > NQ ? q_issued - NQ : 0); t < q_issued; ++t)
          drain_wait(&bars[L::bQFull + t % NQ], (t / NQ) & 1);
        for (uint32_t t = (do_issued > NDO ? do_issued - NDO : 0); t < do_issued; ++t)
          drain_wait(&bars[L::bDOFull + t % NDO], (t / NDO) & 1);
        if (kv_issued > 0) {
          drain_wait(&bars[L::bKFull], (kv_issued - 1) & 1);
          drain_wait(&bars[L::bVFull], (kv_issued - 1) & 1);
        }
      }
    }
    } else if (run && warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Per entry e: dV(e), S^T(e+1), dK(e), dQ(e), dP^T(e+1).  S^T(e+1) reuses the
    // columns dV(e) reads P^T from: tcgen05.mma ops issued by one thread run in
    // issue order, so it follows dV(e) without a wait and the next entry's
    // exponentials overlap this entry's dK and dQ.
    if (lane == 0) {
      uint32_t tc = 0, cc = 0, ec = 0;
      uint32_t k_addr = 0, v_addr = 0;  // this column's K and V buffers
      const uint32_t ds_addr = smem_u32(sm + L::kDS);
      auto issue_s = [&](uint32_t e_idx) -> bool {  // S^T = K_n Q_m^T
        const uint32_t qs = e_idx % NQ;
        if (!wd.wait(&bars[L::bQFull + qs], (e_idx / NQ) & 1)) return false;
        tc_fence_after();
        const uint32_t q_addr = smem_u32(sm + L::kQ + qs * kTB);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_ss(T_S, sw128_desc(k_addr + off, 16, 1024), sw128_desc(q_addr + off, 16, 1024),
                 kIdS, kk > 0);
        }
        mma_commit(&bars[L::bSFull]);
        return true;
      };
      auto issue_dp = [&](uint32_t e_idx) -> bool {  // dP^T = V_n dO_m^T
        const uint32_t ds = e_idx % NDO;
        if (!wd.wait(&bars[L::bDOFull + ds], (e_idx / NDO) & 1)) return false;
        // the dQ of the previous entry occupies these columns until read out
        if (e_idx >= 1 && !wd.wait(&bars[L::bDQFree], (e_idx - 1) & 1)) return false;
        tc_fence_after();
        const uint32_t do_addr = smem_u32(sm + L::kDO + ds * kTB);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_ss(T_DP, sw128_desc(v_addr + off, 16, 1024), sw128_desc(do_addr + off, 16, 1024),
                 kIdS, kk > 0);
        }
        mma_commit(&bars[L::bDPFull]);
        return true;
      };
      for (;; ++tc) {
        const uint32_t slot = tc & 1;
        if (!wd.wait(&bars[L::bTkFull + slot], (tc >> 1) & 1)) break;
        const int t = tk_ring[slot];
        mbar_arrive(&bars[L::bTkEmpty + slot]);
        const Ticket k = decode_ticket(p, t);
        if (!k.valid) break;
        if (k.ee == k.es) continue;
        const int kb = cc & 1, vb = kb ^ 1;
        k_addr = smem_u32(sm + L::kK + kb * kTB);
        v_addr = smem_u32(sm + L::kK + vb * kTB);
        if (!wd.wait(&bars[L::bKConv], cc & 1)) break;
        bool stop = !issue_s(ec);
        if (!stop && !wd.wait(&bars[L::bVConv], cc & 1)) stop = true;
        if (!stop && !issue_dp(ec)) stop = true;
        // V's last use is the column's last dP^T: its buffer takes the next K
        if (!stop && k.tot == 1) mma_commit(&bars[L::bXFree + vb]);
        for (int x = 0; x < k.tot && !stop; ++x, ++ec) {
          const uint32_t qs = ec % NQ, ds = ec % NDO;
          const bool first = x == 0, last = x == k.tot - 1;
          if (!wd.wait(&bars[L::bPReady], ec & 1)) { stop = true; break; }
          if (first && cc >= 1 && !wd.wait(&bars[L::bDKVFree], (cc - 1) & 1)) { stop = true; break; }
          tc_fence_after();
          // dV += P^T dO_m   (P^T from TMEM, dO as an MN-major B operand)
          const uint32_t do_addr = smem_u32(sm + L::kDO + ds * kTB);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(T_DV, T_S + kk * 8 + (kk >= 4 ? 32 : 0), sw128_desc(do_addr + kk * 2048, 16384, 1024), kIdKV,
                   (!first || kk > 0) ? 1u : 0u);
          mma_commit(&bars[L::bDOEmpty + ds]);
          if (!last && !issue_s(ec + 1)) { stop = true; break; }
          if (!wd.wait(&bars[L::bDSReady], ec & 1)) { stop = true; break; }
          tc_fence_after();
          // dK += dS^T Q_m, dS^T from TMEM (the compute warps wrote it over the
          // dP^T columns they had read, laid out like P^T), so only Q comes
          // from shared memory
          const uint32_t q_addr = smem_u32(sm + L::kQ + qs * kTB);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(T_DK, T_DP + kk * 8 + (kk >= 4 ? 32 : 0), sw128_desc(q_addr + kk * 2048, 16384, 1024),
                   kIdKV, (!first || kk > 0) ? 1u : 0u);
          mma_commit(&bars[L::bQEmpty + qs]);
          // dQ_m part = dS K_n (dS read MN-major from the shared dS^T tile) into
          // the dP^T columns: issued after dK, which reads dS^T from them
          // (tcgen05.mma ops of one thread run in issue order).  The dQ warps'
          // read of it gates the next dP^T, which shares those columns.
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(T_DP, sw128_desc(ds_addr + kk * 2048, 16384, 1024),
                   sw128_desc(k_addr + kk * 2048, 16384, 1024), kIdQ, kk > 0);
          mma_commit(&bars[L::bDQFull]);
          // K's last use is the column's last dQ: its buffer takes the next V
          if (last) mma_commit(&bars[L::bXFree + kb]);
          mma_commit(&bars[L::bDSFree]);
          if (last) {
            mma_commit(&bars[L::bDKVFull]);
          } else {
            if (!issue_dp(ec + 1)) {
              stop = true;
              break;
            }
            if (x + 1 == k.tot - 1) mma_commit(&bars[L::bXFree + vb]);
          }
        }
        if (stop) break;
        ++cc;
      }
      mma_commit(&bars[L::bFinal]);
      drain_wait(&bars[L::bFinal], 0);
    }
    } else if (run) {
    // ------------------------------------------------------------ converters (warps 2, 3)
    // Every product runs on fp16 operands, so that P and dS enter them with
    // fp16's 11 significant bits instead of bf16's 8.  Q_m and dO_m arrive as
    // fp16 already (the Delta pass wrote fp16 copies); K_n and V_n, loaded once
    // per kv column from the caller's bf16 tensors, are turned into fp16 in
    // place here as soon as their copies land.  Values beyond the fp16 range
    // are clamped and reported as BSA_ERR_INPUT_RANGE.
    const int ct = threadIdx.x - 64;  // 0 .. 63
    auto wwait = [&](uint64_t *bar, uint32_t parity) {
      return __all_sync(0xffffffffu, wd.wait(bar, parity)) != 0;
    };
    uint32_t in_max = 0;  // per 16-bit half: the largest |x| bit pattern seen
    auto convert = [&](uint8_t *tile, uint64_t *done) {
      constexpr int kChunks = kTB / 16;            // 16-byte pieces of the tile
      constexpr int kPer = kChunks / kConvThreads;  // per thread
      constexpr int kBatch = 8;
      static_assert(kPer % kBatch == 0, "converter batches");
      int4 *t4 = reinterpret_cast<int4 *>(tile);
#pragma unroll 1
      for (int i0 = 0; i0 < kPer; i0 += kBatch) {
        int4 v[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) v[u] = t4[(i0 + u) * kConvThreads + ct];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
          uint32_t w[4] = {static_cast<uint32_t>(v[u].x), static_cast<uint32_t>(v[u].y),
                           static_cast<uint32_t>(v[u].z), static_cast<uint32_t>(v[u].w)};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            in_max = __vmaxu2(in_max, w[q] & 0x7fff7fffu);
            w[q] = bf16x2_to_f16x2(w[q]);
          }
          t4[(i0 + u) * kConvThreads + ct] = make_int4(w[0], w[1], w[2], w[3]);
        }
      }
      fence_proxy_async_smem();  // the MMAs read the tile through the async proxy
      mbar_arrive(done);
    };
    uint32_t tc = 0, cc = 0;
    for (;; ++tc) {
      const uint32_t slot = tc & 1;
      if (!wwait(&bars[L::bTkFull + slot], (tc >> 1) & 1)) break;
      const int t = tk_ring[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[L::bTkEmpty + slot]);
      const Ticket k = decode_ticket(p, t);
      if (!k.valid) break;
      if (k.ee == k.es) continue;
      const int kb = cc & 1, vb = kb ^ 1;
      if (!wwait(&bars[L::bKFull], cc & 1)) break;
      convert(sm + L::kK + kb * kTB, &bars[L::bKConv]);
      if (!wwait(&bars[L::bVFull], cc & 1)) break;
      convert(sm + L::kK + vb * kTB, &bars[L::bVConv]);
      ++cc;
    }
    // |x| >= 65536 (bf16 bits 0x4780; bf16 has no value in (65280, 65536)),
    // infinities and NaNs: beyond what fp16 holds
    if ((in_max & 0xffffu) >= 0x4780u || (in_max >> 16) >= 0x4780u)
      record_status(p.hdr + kHdrStatus, BSA_ERR_INPUT_RANGE);
    }
  } else if (warp < 12) {
    if (run) {
    // ------------------------------------------------------------ compute (key rows)
    // two warps per TMEM lane quarter: `half` 0 takes query columns 0..63,
    // half 1 columns 64..127 (and the matching halves of the dK/dV rows)
    const int quarter = warp & 3, half = (warp - 4) >> 2;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const MaskParams &mk = p.mask;
    const bool use_seg = mk.seg_q != nullptr;
    auto wwait = [&](uint64_t *bar, uint32_t parity) {
      return __all_sync(0xffffffffu, wd.wait(bar, parity)) != 0;
    };
    const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
    // this half's P^T columns in TMEM (read as the A operand of dV): inside its
    // own S^T columns, which only this warp reads
    const uint32_t t_p = T_S + lane_off + 64 * half;
    uint32_t tc = 0, cc = 0, ec = 0;
    uint32_t ds_max = 0;  // per 16-bit half: the largest |dS| fp16 bit pattern written
    bool stop = false;
    for (;; ++tc) {
      const uint32_t slot = tc & 1;
      if (!wwait(&bars[L::bTkFull + slot], (tc >> 1) & 1)) break;
      const int t = tk_ring[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[L::bTkEmpty + slot]);
      const Ticket k = decode_ticket(p, t);
      if (!k.valid) break;
      const int j = k.n * kTile + r;
      const bool row_ok = j < p.Skv;
      if (k.ee == k.es) {
        if (row_ok) {
          __nv_bfloat16 *dk_row = p.dk + k.b * p.k_sb + static_cast<int64_t>(j) * p.k_ss + k.hk * p.k_sh;
          __nv_bfloat16 *dv_row = p.dv + k.b * p.v_sb + static_cast<int64_t>(j) * p.v_ss + k.hk * p.v_sh;
          const int4 z = make_int4(0, 0, 0, 0);
#pragma unroll
          for (int c = half * (D / 16); c < (half + 1) * (D / 16); ++c) {
            reinterpret_cast<int4 *>(dk_row)[c] = z;
            reinterpret_cast<int4 *>(dv_row)[c] = z;
          }
        }
        continue;
      }
      // queries this key may be seen by: [qlo, qhi], thinned by the dilation
      // unless the key lies in the prefix every query sees
      int qlo = 0, qhi = p.Sq - 1;
      if (!row_ok) qhi = -1;
      const bool in_prefix = mk.prefix_len != nullptr && j < mk.prefix_len[k.b];
      const bool dilated = mk.dilation > 1 && !in_prefix;
      if ((mk.flags & BSA_MASK_CAUSAL_WINDOW) && !in_prefix) {
        qlo = max(qlo, j - mk.offset);
        if (mk.window > 0) qhi = min(qhi, j - mk.offset + mk.window - 1);
      }
      if ((mk.flags & BSA_MASK_KV_VALID_LEN) && j >= mk.kv_valid_len[k.b]) qhi = -1;
      const int seg_j = (use_seg && row_ok) ? mk.seg_kv[static_cast<int64_t>(k.b) * p.Skv + j] : INT_MIN;
      uint8_t *ds_tile = sm + L::kDS;
      // The entry's list word and this thread's -LSE*log2e (half 0; -inf where
      // the row has no key or lies past Sq) or -Delta (half 1) of the q-block,
      // negated so the element loops are one packed FMA / add.  Fetched ahead
      // (the list word two entries ahead, the value one entry ahead, its
      // address then known) so that both global loads fall under the previous
      // entries' work instead of delaying this entry's staging.
      auto vec_of = [&](int xx, uint32_t ent_x) -> float {
        const int64_t bh_x = static_cast<int64_t>(k.b) * p.H + k.head(xx);
        const int i_x = static_cast<int>(ent_x & kIndexMask) * kTile + r;
        if (half == 0) {
          float v = -INFINITY;
          if (i_x < p.Sq) {
            const float lv = p.lse[bh_x * p.Sq + i_x];
            if (lv != -INFINITY) v = -lv * kLog2e;
          }
          return v;
        }
        return -p.delta[bh_x * p.nM * kTile + i_x];
      };
      uint32_t ent_a = k.tot > 0 ? p.col_ent[k.entry(0)] : 0u;  // entry x
      uint32_t ent_b = k.tot > 1 ? p.col_ent[k.entry(1)] : 0u;  // entry x + 1
      float vec_a = k.tot > 0 ? vec_of(0, ent_a) : 0.f;
      for (int x = 0; x < k.tot; ++x, ++ec) {
        const uint32_t ent = ent_a;
        const float vecv = vec_a;
        if (x + 1 < k.tot) vec_a = vec_of(x + 1, ent_b);
        ent_a = ent_b;
        if (x + 2 < k.tot) ent_b = p.col_ent[k.entry(x + 2)];
        const int m = static_cast<int>(ent & kIndexMask);
        const bool full = (ent & kFullBit) != 0;
        {
          if (half == 0)
            vec_nl[(ec & 1) * kTile + r] = vecv;
          else
            vec_nd[(ec & 1) * kTile + r] = vecv;
          mbar_arrive(&bars[L::bVecReady + (ec & 1)]);
        }
        // allowed-query bits of this half's two 32-query words for this key
        // row (range AND segment ids, the latter read through L1 as broadcasts)
        uint32_t allow[2] = {~0u, ~0u};
        if (!full) {
#pragma unroll
          for (int w = 0; w < 2; ++w)
            allow[w] = range_bits(qlo - m * kTile, qhi - m * kTile, 2 * half + w);
          if (dilated) {
            // keep query i iff (i + o - j) mod d == 0: bit k of word w is query
            // 128m + 32w + k, kept iff k == (j - o - 128m - 32w) mod d
            int ph = (j - mk.offset - m * kTile - 64 * half) % mk.dilation;
            if (ph < 0) ph += mk.dilation;
#pragma unroll
            for (int w = 0; w < 2; ++w) {
              allow[w] &= ph < 32 ? (mk.dil_pattern << ph) : 0u;
              ph -= mk.dil_r32;
              if (ph < 0) ph += mk.dilation;
            }
          }
          if (use_seg) {
            const int32_t *sq = mk.seg_q + static_cast<int64_t>(k.b) * p.Sq + m * kTile + 64 * half;
            const int lim = p.Sq - m * kTile - 64 * half;
#pragma unroll
            for (int w = 0; w < 2; ++w) {
              uint32_t bits = 0;
#pragma unroll 8
              for (int q = 0; q < 32; ++q) {
                const int ii = 32 * w + q;
                bits |= static_cast<uint32_t>(ii < lim && __ldg(sq + ii) == seg_j) << q;
              }
              allow[w] &= bits;
            }
          }
        }
        if (!wwait(&bars[L::bVecReady + (ec & 1)], (ec >> 1) & 1)) { stop = true; break; }
        const float4 *nl4p = reinterpret_cast<const float4 *>(vec_nl + (ec & 1) * kTile + 64 * half);
        const float4 *nd4p = reinterpret_cast<const float4 *>(vec_nd + (ec & 1) * kTile + 64 * half);
        // phase 1: P^T = exp2(S^T * scale * log2e - LSE*log2e) -> fp16 in TMEM
        // (the A operand of dV) and kept in registers for dS: P lies in [0, 1],
        // where fp16 keeps 11 significant bits to bf16's 8
        if (!wwait(&bars[L::bSFull], ec & 1)) { stop = true; break; }
        tc_fence_after();
        uint32_t pk[32];
        // four 16-column pieces, the next one's TMEM load in flight while this
        // one is computed
        uint32_t sb[2][16];
        tmem_ld16(T_S + lane_off + 64 * half, sb[0]);
        tmem_wait_ld();
#pragma unroll
        for (int sc = 0; sc < 4; ++sc) {
          if (sc + 1 < 4) tmem_ld16(T_S + lane_off + 64 * half + 16 * (sc + 1), sb[(sc + 1) & 1]);
          const uint32_t *s = sb[sc & 1];
          const uint32_t bits = allow[sc >> 1] >> (16 * (sc & 1));
          uint32_t pb[8];
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const float4 nl4 = nl4p[4 * sc + q4];
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              const int e0 = 4 * q4 + 2 * h2;
              const float2 nl = h2 ? make_float2(nl4.z, nl4.w) : make_float2(nl4.x, nl4.y);
              const float2 tt = __ffma2_rn(
                  make_float2(__uint_as_float(s[e0]), __uint_as_float(s[e0 + 1])), sc2, nl);
              float p0 = fast_exp2(tt.x), p1 = fast_exp2(tt.y);
              if (!full) {
                p0 = ((bits >> e0) & 1u) ? p0 : 0.f;
                p1 = ((bits >> (e0 + 1)) & 1u) ? p1 : 0.f;
              }
              pb[e0 >> 1] = pack_f16x2(p0, p1);
            }
          }
#pragma unroll
          for (int q = 0; q < 8; ++q) pk[8 * sc + q] = pb[q];
          // P^T piece (fp16) -> TMEM columns [8sc, 8sc+8) of this half's
          // region: S^T columns this warp has already read
          tmem_st8(t_p + 8 * sc, pb);
          if (sc + 1 < 4) tmem_wait_ld();
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars[L::bPReady]);
        // phase 2: dS^T = P^T o (dP^T - Delta) in fp32 from the fp16 P^T -> fp16,
        // into the shared tile (128-byte swizzle, K-major; the dQ MMA reads it
        // MN-major) and into TMEM over this half's dP^T columns, already read
        // (the A operand of dK, laid out like P^T for dV)
        if (ec >= 1 && !wwait(&bars[L::bDSFree], (ec - 1) & 1)) { stop = true; break; }
        if (!wwait(&bars[L::bDPFull], ec & 1)) { stop = true; break; }
        tc_fence_after();
        // four 16-column pieces; the next piece's TMEM load is in flight while
        // this one is computed (a wait covers every load issued before it)
        uint32_t dpb[2][16];
        tmem_ld16(T_DP + lane_off + 64 * half, dpb[0]);
        tmem_wait_ld();
#pragma unroll
        for (int sc = 0; sc < 4; ++sc) {
          if (sc + 1 < 4) tmem_ld16(T_DP + lane_off + 64 * half + 16 * (sc + 1), dpb[(sc + 1) & 1]);
          const uint32_t *dp = dpb[sc & 1];
          uint32_t dk2[8];
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const float4 nd4 = nd4p[4 * sc + q4];
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              const int e0 = 4 * q4 + 2 * h2;
              const float2 nd = h2 ? make_float2(nd4.z, nd4.w) : make_float2(nd4.x, nd4.y);
              const float2 pv = unpack_f16x2(pk[8 * sc + (e0 >> 1)]);
              const float2 dd = __fadd2_rn(
                  make_float2(__uint_as_float(dp[e0]), __uint_as_float(dp[e0 + 1])), nd);
              const float2 dsv = __fmul2_rn(pv, dd);
              dk2[e0 >> 1] = pack_f16x2_sat(dsv.x, dsv.y);
              ds_max = __vmaxu2(ds_max, dk2[e0 >> 1] & 0x7fff7fffu);
            }
          }
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int chunk = 8 * half + 2 * sc + u;  // 0..15: 8 queries each
            const int sub = chunk >> 3, cw = chunk & 7;
            uint8_t *dst = ds_tile + sub * 16384 + r * 128 + ((cw ^ (r & 7)) << 4);
            *reinterpret_cast<int4 *>(dst) =
                make_int4(dk2[4 * u], dk2[4 * u + 1], dk2[4 * u + 2], dk2[4 * u + 3]);
          }
          // piece -> TMEM columns [8sc, 8sc+8) of this half: dP^T columns
          // already read (the load in flight is of columns 16(sc+1) on)
          tmem_st8(T_DP + lane_off + 64 * half + 8 * sc, dk2);
          if (sc + 1 < 4) tmem_wait_ld();
        }
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bars[L::bDSReady]);
      }
      if (stop) break;
      // epilogue: this half's columns of dV, then dK (scaled) -> bf16, staged
      // through the 4 KB of the dS^T tile that only this warp writes (its 32
      // rows of sub-tile `half`; the column's MMAs are done with the tile once
      // DKVFull fires), then stored as whole 128-byte row segments: a warp
      // store covers 512 / D rows instead of 32 scattered 16-byte pieces
      if (!wwait(&bars[L::bDKVFull], cc & 1)) break;
      tc_fence_after();
      {
        constexpr int kCpr = D / 16;           // 16-byte chunks per half row
        constexpr int kRowsPerStore = 32 / kCpr;
        uint8_t *stg = ds_tile + half * 16384 + quarter * 4096;
        auto slot = [](int s_) { return s_ ^ ((s_ >> 3) & 7); };  // bank-conflict-free
#pragma unroll
        for (int which = 0; which < 2; ++which) {
          const uint32_t tsrc = (which ? T_DK : T_DV) + lane_off + 32 * half * (D / 64);
          const float mul = which ? p.scale : 1.f;
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            uint32_t a[32];
            tmem_ld32(tsrc + 32 * c, a);
            tmem_wait_ld();
            uint32_t w[16];
#pragma unroll
            for (int q = 0; q < 16; ++q)
              w[q] = pack_bf16x2(__uint_as_float(a[2 * q]) * mul, __uint_as_float(a[2 * q + 1]) * mul);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              *reinterpret_cast<int4 *>(stg + (slot(lane * kCpr + 4 * c + q) << 4)) =
                  make_int4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
          }
          if (which == 1) {
            tc_fence_before();
            mbar_arrive(&bars[L::bDKVFree]);
          }
          __syncwarp();
          __nv_bfloat16 *base = which ? p.dk + k.b * p.k_sb + k.hk * p.k_sh
                                      : p.dv + k.b * p.v_sb + k.hk * p.v_sh;
          const int64_t rs = which ? p.k_ss : p.v_ss;
#pragma unroll
          for (int it = 0; it < D / 16; ++it) {
            const int rr = it * kRowsPerStore + lane / kCpr, ch = lane % kCpr;
            const int jj = k.n * kTile + quarter * 32 + rr;
            const int4 v = *reinterpret_cast<const int4 *>(stg + (slot(rr * kCpr + ch) << 4));
            if (jj < p.Skv)
              *reinterpret_cast<int4 *>(base + static_cast<int64_t>(jj) * rs + half * (D / 2) + 8 * ch) = v;
          }
          __syncwarp();
        }
      }
      ++cc;
    }
    // a dS clamped at the fp16 limit 65504 (0x7bff): reported, not silent
    if ((ds_max & 0xffffu) >= 0x7bffu || (ds_max >> 16) >= 0x7bffu)
      record_status(p.hdr + kHdrStatus, BSA_ERR_INPUT_RANGE);
    }
  } else {
    regs_inc<160>();
    if (run) {
    // ------------------------------------------------------------ dQ (query rows)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    auto wwait = [&](uint64_t *bar, uint32_t parity) {
      return __all_sync(0xffffffffu, wd.wait(bar, parity)) != 0;
    };
    // dQ part of entry `ec`: TMEM -> registers (scaled), columns handed back
    // to the next dP^T.  Every column load is in flight at once, one wait.
    float acc[D];
    auto read_dq = [&]() {
      tc_fence_after();
      uint32_t raw[D];
#pragma unroll
      for (int c = 0; c < D / 32; ++c)
        tmem_ld32(T_DP + lane_off + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&raw[32 * c]));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&bars[L::bDQFree]);
#pragma unroll
      for (int q = 0; q < D; ++q) acc[q] = __uint_as_float(raw[q]) * p.scale;
    };
    uint32_t tc = 0, ec = 0;
    bool ahead = false;  // acc already holds entry ec's dQ part
    for (;; ++tc) {
      const uint32_t slot = tc & 1;
      if (!wwait(&bars[L::bTkFull + slot], (tc >> 1) & 1)) break;
      const int t = tk_ring[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[L::bTkEmpty + slot]);
      const Ticket k = decode_ticket(p, t);
      if (!k.valid) break;
      bool stop = false;
      for (int x = 0; x < k.tot; ++x, ++ec) {
        const int e = k.entry(x);
        const int64_t bh = static_cast<int64_t>(k.b) * p.H + k.head(x);
        const int m = static_cast<int>(p.col_ent[e] & kIndexMask);
        const uint32_t rank = static_cast<uint32_t>(p.col_rank[e]);
        if (!ahead) {
          if (!wwait(&bars[L::bDQFull], ec & 1)) { stop = true; break; }
          read_dq();
        }
        ahead = false;
        // one semaphore per 32-row quarter of the q-block: this warp's rows
        uint32_t *sem = p.sem + (bh * p.nM + m) * 4 + quarter;
        int ok = 1;
        if (p.deterministic) {
          if (lane == 0) ok = sem_wait(sem, rank, p.sem_timeout_ns, p.hdr + kHdrStatus) ? 1 : 0;
          ok = __shfl_sync(0xffffffffu, ok, 0);
          // the warp barrier orders every lane's adds below after lane 0's
          // acquire (a shuffle alone carries no memory ordering)
          __syncwarp();
        }
        if (ok) {
          float *base = p.dq_accum + (bh * p.nM + m) * (D / 4) * (kTile * 4);
          if (p.deterministic && rank == 0) {
            // the first contributor in the order pi initialises the accumulator
            // rows, so the deterministic path needs no zeroing pass
#pragma unroll
            for (int c = 0; c < D / 4; ++c)
              st_v4(base + (static_cast<int64_t>(c) * kTile + r) * 4, acc[4 * c], acc[4 * c + 1],
                    acc[4 * c + 2], acc[4 * c + 3]);
          } else {
#pragma unroll
            for (int c = 0; c < D / 4; ++c)
              red_add_v4(base + (static_cast<int64_t>(c) * kTile + r) * 4, acc[4 * c],
                         acc[4 * c + 1], acc[4 * c + 2], acc[4 * c + 3]);
          }
        }
        // if the column's next dQ part is already complete, take it out of TMEM
        // before this entry's adds are fenced: the next dP^T then need not wait
        // for the fence.  A single test, never a wait, so the turn below is
        // passed on no later than the TMEM read.
        if (x + 1 < k.tot &&
            __all_sync(0xffffffffu, mbar_try_wait(smem_u32(&bars[L::bDQFull]), (ec + 1) & 1))) {
          read_dq();
          ahead = true;
        }
        if (p.deterministic) {
          // Pass this quarter's turn on once the warp's adds are ordered before
          // it: each thread's adds precede its device-scope acq_rel fence, the
          // warp synchronises, and lane 0's release add on the semaphore is
          // cumulative over what it has observed.  Each warp runs its own
          // quarter's chain: a hop carries 16 KB, and no warp waits for another.
          asm volatile("fence.acq_rel.gpu;" ::: "memory");
          __syncwarp();
          if (lane == 0) red_release_gpu_add(sem, 1u);
          __syncwarp();
        }
      }
      if (stop) break;
    }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0) release_ticket(p.hdr + kHdrBwdTicket, p.hdr + kHdrBwdDone);
}

// ---------------------------------------------------------------- a4: Delta
constexpr int kDeltaRuns = 2;         // runs of consecutive rows per tile, loads all in flight
constexpr int kDeltaBlocksPerSm = 3;  // the persistent grid (2 and 4 measured slower)

struct DeltaArgs {
  const __nv_bfloat16 *o, *dout, *q;
  int64_t sb, ss, sh;     // O and dO strides
  int64_t qb, qs, qh;     // Q strides
  int B, Sq, H, Skv, rows_pad;
  const uint8_t *resid;   // [B, Sq, H, D] scaled e5m2 residual bytes
  uint32_t *hdr;
  float *delta;
  uint32_t *sem;
  int64_t n_sem;
  uint32_t *q16, *do16;   // [B, Sq, H, D] fp16 copies for the backward's products
  uint32_t dq_mode;       // recorded for the dQ convert: 1 semaphore-ordered, 2 atomic
};

template <int D, bool RESID>
__global__ void __launch_bounds__(256, 3) k_bwd_delta(const DeltaArgs a) {
  // D/8 threads per (b, h, i) row vector, 16 bytes of O, dO, Q (and the O
  // residual) each.  A tile is kDeltaRuns runs of 256 / (D/8) consecutive rows
  // of one head (the Delta layout), every run's loads in flight before any is
  // reduced; rows past Sq (the last q-block's padding) get Delta = 0.  The
  // same pass writes fp16 copies of Q and dO (the backward main kernel takes
  // every product on fp16 operands) and reports values beyond the fp16 range
  // as BSA_ERR_INPUT_RANGE.  The grid also zeroes the dQ semaphores.  RESID:
  // the O residual is added to O
  // (a compile-time choice, so that the plain pass carries no zero vector),
  // and only when the header records that the last forward on this workspace
  // kept the residual of this very `o` for this problem (else Delta comes from
  // the bf16 O alone).  A true residual never exceeds half a bf16 ulp of its
  // O element; a residual element above that is dropped, so that even a stale
  // record (a workspace reused after another forward wrote into the same
  // output buffer) moves Delta by no more than the bf16 O alone would.
  constexpr int TPV = D / 8;
  constexpr int VPB = 256 / TPV;
  // O comes from the forward, launched just before.  No early trigger: the
  // backward main kernel, one persistent CTA per SM, launches as this pass's
  // blocks leave (measured 368 -> 330 us per step on the 8192 window against
  // a trigger here, which let its CTAs take SMs during the pass)
  pdl_wait();
  // which dQ protocol the backward main kernel will follow: the convert polls
  // the semaphores only when they count every contribution
  if (blockIdx.x == 0 && threadIdx.x == 0) a.hdr[kHdrDqMode] = a.dq_mode;
  const int B = a.B, Sq = a.Sq, H = a.H, rows_pad = a.rows_pad;
  const uint32_t *hdr = a.hdr;
  bool use_resid = false;
  if (RESID) {
    const uint64_t tag = (static_cast<uint64_t>(hdr[kHdrResidHi]) << 32) | hdr[kHdrResidLo];
    use_resid = tag == reinterpret_cast<uint64_t>(a.o) && hdr[kHdrResidB] == static_cast<uint32_t>(B) &&
                hdr[kHdrResidH] == static_cast<uint32_t>(H) && hdr[kHdrResidSq] == static_cast<uint32_t>(Sq) &&
                hdr[kHdrResidSkv] == static_cast<uint32_t>(a.Skv) && hdr[kHdrResidD] == static_cast<uint32_t>(D);
  }
  // the forward that kept this residual also wrote the fp16 copy of Q, if its
  // record names this very q (pointer and strides): Q need not be read again
  bool have_q16 = false;
  if (RESID && use_resid) {
    const uint64_t qtag = (static_cast<uint64_t>(hdr[kHdrQ16Hi]) << 32) | hdr[kHdrQ16Lo];
    have_q16 = qtag == reinterpret_cast<uint64_t>(a.q) && hdr[kHdrQ16Sb] == static_cast<uint32_t>(a.qb) &&
               hdr[kHdrQ16Ss] == static_cast<uint32_t>(a.qs) && hdr[kHdrQ16Sh] == static_cast<uint32_t>(a.qh);
  }
  for (int64_t z = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; z < a.n_sem;
       z += static_cast<int64_t>(gridDim.x) * blockDim.x)
    a.sem[z] = 0u;
  const int t = threadIdx.x % TPV;
  // Persistent over tiles of kDeltaRuns runs of VPB consecutive rows of one
  // (b, h) (the Delta layout), two tiles in flight: the next tile's loads are
  // issued before this tile's conversions and dot products, so the memory
  // system always has a tile's loads outstanding.
  constexpr int kRowsPerTile = kDeltaRuns * VPB;
  const int tiles_per_bh = rows_pad / kRowsPerTile;
  const int n_tiles = B * H * tiles_per_bh;
  struct Loaded {
    int4 av[kDeltaRuns], cv[kDeltaRuns], qv[kDeltaRuns];
    uint2 rv[kDeltaRuns];
  };
  auto load = [&](int tile, Loaded &x) {
    const int bh = tile / tiles_per_bh;
    const int i0 = (tile - bh * tiles_per_bh) * kRowsPerTile + threadIdx.x / TPV;
    const int b = bh / H, h = bh % H;
#pragma unroll
    for (int j = 0; j < kDeltaRuns; ++j) {
      const int i = i0 + j * VPB;
      x.av[j] = x.cv[j] = x.qv[j] = make_int4(0, 0, 0, 0);
      x.rv[j] = make_uint2(0u, 0u);
      if (tile < n_tiles && i < Sq) {
        const int64_t off = b * a.sb + static_cast<int64_t>(i) * a.ss + h * a.sh + t * 8;
        x.av[j] = __ldg(reinterpret_cast<const int4 *>(a.o + off));
        x.cv[j] = __ldg(reinterpret_cast<const int4 *>(a.dout + off));
        if (!have_q16)
          x.qv[j] = __ldcs(reinterpret_cast<const int4 *>(a.q + b * a.qb + static_cast<int64_t>(i) * a.qs + h * a.qh + t * 8));
        if (use_resid)
          x.rv[j] = __ldg(reinterpret_cast<const uint2 *>(a.resid + ((static_cast<int64_t>(b) * Sq + i) * H + h) * D + t * 8));
      }
    }
  };
  uint32_t in_max = 0;
  auto process = [&](int tile, const Loaded &x) {
    const int bh = tile / tiles_per_bh;
    const int i0 = (tile - bh * tiles_per_bh) * kRowsPerTile + threadIdx.x / TPV;
    const int b = bh / H, h = bh % H;
#pragma unroll
    for (int j = 0; j < kDeltaRuns; ++j) {
      const int i = i0 + j * VPB;
      const bool row = i < Sq;
      // fp16 copies of Q and dO, contiguous [B, Sq, H, D], and the dot
      // product; dO is unpacked once for both
      const int64_t off = ((static_cast<int64_t>(b) * Sq + i) * H + h) * (D / 2) + t * 4;
      if (row && !have_q16) {
        const uint32_t xq[4] = {static_cast<uint32_t>(x.qv[j].x), static_cast<uint32_t>(x.qv[j].y),
                                static_cast<uint32_t>(x.qv[j].z), static_cast<uint32_t>(x.qv[j].w)};
        uint32_t hq[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          in_max = __vmaxu2(in_max, xq[q] & 0x7fff7fffu);
          hq[q] = bf16x2_to_f16x2(xq[q]);
        }
        *reinterpret_cast<int4 *>(a.q16 + off) = make_int4(hq[0], hq[1], hq[2], hq[3]);
      }
      const uint32_t xa[4] = {static_cast<uint32_t>(x.av[j].x), static_cast<uint32_t>(x.av[j].y),
                              static_cast<uint32_t>(x.av[j].z), static_cast<uint32_t>(x.av[j].w)};
      const uint32_t xc[4] = {static_cast<uint32_t>(x.cv[j].x), static_cast<uint32_t>(x.cv[j].y),
                              static_cast<uint32_t>(x.cv[j].z), static_cast<uint32_t>(x.cv[j].w)};
      // residual bytes of elements 2q, 2q+1: 16 bits of rv
      const uint32_t xr[4] = {x.rv[j].x & 0xffffu, x.rv[j].x >> 16, x.rv[j].y & 0xffffu, x.rv[j].y >> 16};
      float acc = 0.f, accr = 0.f;
      uint32_t hd[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 fo = unpack_bf16x2(xa[q]);
        const float2 fd = unpack_bf16x2(xc[q]);
        in_max = __vmaxu2(in_max, xc[q] & 0x7fff7fffu);
        hd[q] = pack_f16x2_sat(fd.x, fd.y);
        if (use_resid) {
          // the residual scaled by 2^12 (its stored form), kept when |r| is at
          // most half a bf16 ulp of its O element, 2^(e - 135) for O's exponent
          // field e: |r 2^12| <= 2^(e - 123), the float with exponent field e + 4
          const float2 fr = unpack_f16x2(e5m2x2_to_f16x2(xr[q]));
          const float hu0 = __uint_as_float(((xa[q] << 16) & 0x7f800000u) + (4u << 23));
          const float hu1 = __uint_as_float((xa[q] & 0x7f800000u) + (4u << 23));
          accr = fmaf(fabsf(fr.x) <= hu0 ? fr.x : 0.f, fd.x, accr);
          accr = fmaf(fabsf(fr.y) <= hu1 ? fr.y : 0.f, fd.y, accr);
        }
        acc = fmaf(fo.x, fd.x, acc);
        acc = fmaf(fo.y, fd.y, acc);
      }
      if (row) *reinterpret_cast<int4 *>(a.do16 + off) = make_int4(hd[0], hd[1], hd[2], hd[3]);
      if (use_resid) acc = fmaf(accr, kResidScaleInv, acc);
#pragma unroll
      for (int sft = TPV / 2; sft > 0; sft >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, sft);
      // rows past Sq get Delta = 0
      if (t == 0) a.delta[static_cast<int64_t>(bh) * rows_pad + i] = acc;
    }
  };
  Loaded x0, x1;
  int tile = blockIdx.x;
  load(tile, x0);
  // two stages unrolled, so the buffers swap roles without copies; the loop
  // bounds are uniform per block (every lane reaches the shuffles)
  while (tile < n_tiles) {
    load(tile + gridDim.x, x1);
    process(tile, x0);
    tile += gridDim.x;
    if (tile >= n_tiles) break;
    load(tile + gridDim.x, x0);
    process(tile, x1);
    tile += gridDim.x;
  }
  // |x| >= 65536 (bf16 bits 0x4780), infinities and NaNs: beyond what fp16 holds
  if ((in_max & 0xffffu) >= 0x4780u || (in_max >> 16) >= 0x4780u)
    record_status(a.hdr + kHdrStatus, BSA_ERR_INPUT_RANGE);
}

// ---------------------------------------------------------------- a7: dQ convert
struct ConvertArgs {
  const float *acc;        // the interleaved accumulator [B, H, nM, D/4, 128, 4]
  const uint32_t *sem;     // [B, H, nM, 4] dQ semaphores
  uint32_t *hdr;
  const int32_t *row_ptr;
  __nv_bfloat16 *dq;
  int64_t sb, ss, sh;
  int B, H, Sq, nM;
};

constexpr uint64_t kConvertPollNs = 50000000ull;  // then wait for the whole backward grid

__device__ __forceinline__ uint32_t ld_relaxed_gpu(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

// Polls a dQ semaphore (acquire, as the backward's contributors do) until it
// reaches target: 1 when it did; 0 after limit_ns or once a device error has
// been recorded, when the caller waits for the backward grid instead.
__device__ int sem_poll(const uint32_t *sem, uint32_t target, uint64_t limit_ns,
                        const uint32_t *status) {
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 0;; ++it) {
    if (ld_acquire_gpu(sem) == target) return 1;
    if ((it & 15u) == 15u) {
      if (*reinterpret_cast<const volatile uint32_t *>(status) != 0u) return 0;
      if (globaltimer_ns() - t0 > limit_ns) return 0;
    }
    __nanosleep(128);
  }
}

// A block per 32-row quarter of one q-block: the rows' slice of the
// interleaved accumulator (32 consecutive float4 per column group: contiguous)
// is read with every thread keeping its loads in flight, staged in shared
// memory, and written as whole bf16 rows.  Q-blocks that no kv column reaches
// get zeros.
//
// After a semaphore-ordered backward a block does not wait for the whole
// backward grid: the quarter's semaphore counts the contributions released so
// far, and once it equals the length of the q-block's row list the rows are
// final.  Blocks placed on SMs the backward's CTAs have left thus convert the
// q-blocks already complete while its last columns still run.  Blocks take
// the q-blocks in the order they complete (the highest first under the
// descending column order, else the lowest first), heads interleaved.  The
// block with the last index waits for the backward grid, so that the
// convert's completion still implies the backward's.
template <int D>
__global__ void __launch_bounds__(256) k_dq_convert(const ConvertArgs a) {
  constexpr int kC = D / 4, kRows = 32, kLD = D + 4;
  constexpr int kPer = kC * kRows / 256;  // float4 loads per thread
  __shared__ __align__(16) float tile[kRows * kLD];
  __shared__ int ready_s;
  // launched once every backward CTA has passed its own wait for the Delta
  // pass (and so for everything before it): the plan and the header words that
  // pass wrote are visible here.  One round trip for all the block decides on:
  // the header words, both candidate q-blocks' row lengths and (thread 0) their
  // semaphores, read relaxed; thread 0 then reads the one it uses again with
  // acquire, and the block barrier orders every thread's reads after that
  const int64_t BH = static_cast<int64_t>(a.B) * a.H;
  const int quarter = static_cast<int>(blockIdx.x & 3u);
  const int64_t u = blockIdx.x >> 2;
  const int64_t bh = u % BH;
  const int mr = static_cast<int>(u / BH);
  const int b = static_cast<int>(bh / a.H), h = static_cast<int>(bh % a.H);
  const int m_asc = mr, m_desc = a.nM - 1 - mr;
  const uint32_t mode = a.hdr[kHdrDqMode], order = a.hdr[kHdrOrder];
  const int32_t *rp = a.row_ptr + b * a.nM;
  const int ra0 = rp[m_asc], ra1 = rp[m_asc + 1], rd0 = rp[m_desc], rd1 = rp[m_desc + 1];
  const uint32_t *sem_a = a.sem + (bh * a.nM + m_asc) * 4 + quarter;
  const uint32_t *sem_d = a.sem + (bh * a.nM + m_desc) * 4 + quarter;
  uint32_t sv_a = 0, sv_d = 0;
  if (threadIdx.x == 0) {
    sv_a = ld_relaxed_gpu(sem_a);
    sv_d = ld_relaxed_gpu(sem_d);
  }
  const bool desc = order == static_cast<uint32_t>(BSA_ORDER_DESC);
  const int m = desc ? m_desc : m_asc;
  const int rl = desc ? rd1 - rd0 : ra1 - ra0;
  const bool empty = rl == 0;
  const int r0 = quarter * kRows;
  if (!empty) {
    if (threadIdx.x == 0) {
      int ready = 0;
      if (mode == 1u) {
        // the relaxed read saw the last release: one acquire read of the same
        // word then orders the block's reads after the contributions (measured
        // faster than a fence after the relaxed read)
        if ((desc ? sv_d : sv_a) == static_cast<uint32_t>(rl))
          ready = ld_acquire_gpu(desc ? sem_d : sem_a) == static_cast<uint32_t>(rl) ? 1 : 0;
        if (!ready) {
          ready = sem_poll(desc ? sem_d : sem_a, static_cast<uint32_t>(rl), kConvertPollNs, a.hdr + kHdrStatus);
        }
      }
      ready_s = ready;
    }
    __syncthreads();
    // atomic adds (final once the backward main kernel completed), or a poll
    // that gave up
    if (!ready_s) pdl_wait();
  }
  const float4 *src = reinterpret_cast<const float4 *>(a.acc) + (bh * a.nM + m) * kC * kTile;
  float4 v[kPer];
#pragma unroll
  for (int w = 0; w < kPer; ++w) {
    const int idx = threadIdx.x + w * 256;  // (column group, row) with rows fastest
    const int c = idx / kRows, rr = idx % kRows;
    // from L2: the contributions were reductions there
    v[w] = empty ? make_float4(0.f, 0.f, 0.f, 0.f) : __ldcg(src + c * kTile + r0 + rr);
  }
#pragma unroll
  for (int w = 0; w < kPer; ++w) {
    const int idx = threadIdx.x + w * 256;
    const int c = idx / kRows, rr = idx % kRows;
    *reinterpret_cast<float4 *>(tile + rr * kLD + 4 * c) = v[w];
  }
  __syncthreads();
  constexpr int kCPR = D / 8;  // 16-byte output pieces per row
  for (int idx = threadIdx.x; idx < kRows * kCPR; idx += 256) {
    const int rr = idx / kCPR, j = idx % kCPR;
    const int i = m * kTile + r0 + rr;
    if (i >= a.Sq) continue;
    const float *t = tile + rr * kLD + 8 * j;
    const int4 w = make_int4(pack_bf16x2(t[0], t[1]), pack_bf16x2(t[2], t[3]),
                             pack_bf16x2(t[4], t[5]), pack_bf16x2(t[6], t[7]));
    *reinterpret_cast<int4 *>(a.dq + b * a.sb + static_cast<int64_t>(i) * a.ss + h * a.sh + 8 * j) = w;
  }
  // the grid completes only after the backward main kernel
  if (blockIdx.x == gridDim.x - 1 && threadIdx.x == 0) pdl_wait();
}

// dK = dV = 0, the whole gradient of a problem with keys but no query row:
// the 16-byte pieces of both strided [B, Skv, H_kv, D] tensors, grid-stride.
__global__ void __launch_bounds__(256) k_zero_kv_grads(__nv_bfloat16 *__restrict__ dk,
                                                       __nv_bfloat16 *__restrict__ dv, int Skv,
                                                       int Hkv, int D, int64_t pieces, int64_t ksb,
                                                       int64_t kss, int64_t ksh, int64_t vsb,
                                                       int64_t vss, int64_t vsh) {
  const int cpr = D / 8;
  const int64_t step = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < 2 * pieces;
       idx += step) {
    const bool is_v = idx >= pieces;
    int64_t r = is_v ? idx - pieces : idx;
    const int c = static_cast<int>(r % cpr);
    r /= cpr;
    const int h = static_cast<int>(r % Hkv);
    r /= Hkv;
    const int64_t j = r % Skv, b = r / Skv;
    __nv_bfloat16 *row = is_v ? dv + b * vsb + j * vss + h * vsh : dk + b * ksb + j * kss + h * ksh;
    *reinterpret_cast<int4 *>(row + 8 * c) = make_int4(0, 0, 0, 0);
  }
}

int sm_count_bwd() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

template <int D, int NQ, int NDO>
cudaError_t run_bwd_main(const BwdParams &bp, const CUtensorMap &tq, const CUtensorMap &tk,
                         const CUtensorMap &tv, const CUtensorMap &tdo, cudaStream_t s) {
  using L = BwdSmem<D, NQ, NDO>;
  static_assert(L::kAlloc <= 232448, "shared memory budget");
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(k_attn_bwd<D, NQ, NDO>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
    if (e != cudaSuccess) return e;
    // the warpgroups' register budgets add up to kThreads x kLaunchRegs: a
    // kernel built with any other register count must not be launched, since
    // an increase beyond what the launch holds would never be granted
    cudaFuncAttributes fa{};
    e = cudaFuncGetAttributes(&fa, k_attn_bwd<D, NQ, NDO>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
    attr = true;
  }
  const int grid = std::max(1, std::min(bp.n_tickets, sm_count_bwd()));
  const cudaError_t e = launch_pdl(k_attn_bwd<D, NQ, NDO>, dim3(grid), dim3(kThreads), L::kAlloc, s,
                                   tq, tk, tv, tdo, bp);
  if (e != cudaSuccess) return e;
  count_launch();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_preprocess(const bsa_problem &p, const bsa_options &o, const void *q,
                                  const void *out, const void *dout, const WsLayout &L,
                                  uint8_t *ws, cudaStream_t s) {
  const int rows_pad = L.nM * kTile;
  const int64_t groups = static_cast<int64_t>(p.B) * p.H * rows_pad;
  float *delta = reinterpret_cast<float *>(ws + L.delta);
  const uint8_t *resid = o.o_residual != BSA_O_RESIDUAL_DROP ? ws + L.o_resid : nullptr;
  // kDeltaRuns runs of 256 / (D / 8) rows per tile; a persistent grid of
  // kDeltaBlocksPerSm blocks per SM walks the tiles
  const int64_t vpb = kDeltaRuns * (256 / (p.D / 8));
  const int64_t n_tiles = (groups + vpb - 1) / vpb;
  const unsigned blocks = static_cast<unsigned>(std::min<int64_t>(n_tiles, kDeltaBlocksPerSm * sm_count_bwd()));
  uint32_t *sem = reinterpret_cast<uint32_t *>(ws + L.sem);
  const int64_t n_sem = static_cast<int64_t>(p.B) * p.H * L.nM * 4;  // a quarter each
  // a programmatic dependent of the forward (which reads O first after it)
  auto kern = p.D == 64 ? (resid != nullptr ? k_bwd_delta<64, true> : k_bwd_delta<64, false>)
                        : (resid != nullptr ? k_bwd_delta<128, true> : k_bwd_delta<128, false>);
  DeltaArgs da{};
  da.o = static_cast<const __nv_bfloat16 *>(out);
  da.dout = static_cast<const __nv_bfloat16 *>(dout);
  da.q = static_cast<const __nv_bfloat16 *>(q);
  da.sb = p.o_stride[0];
  da.ss = p.o_stride[1];
  da.sh = p.o_stride[2];
  da.qb = p.q_stride[0];
  da.qs = p.q_stride[1];
  da.qh = p.q_stride[2];
  da.B = p.B;
  da.Sq = p.Sq;
  da.H = p.H;
  da.Skv = p.Skv;
  da.rows_pad = rows_pad;
  da.resid = resid;
  da.hdr = reinterpret_cast<uint32_t *>(ws + L.status);
  da.delta = delta;
  da.sem = sem;
  da.n_sem = n_sem;
  da.q16 = reinterpret_cast<uint32_t *>(ws + L.q16);
  da.do16 = reinterpret_cast<uint32_t *>(ws + L.do16);
  da.dq_mode = o.deterministic ? 1u : 2u;
  cudaError_t e = launch_pdl(kern, dim3(blocks), dim3(256), 0, s, da);
  if (e != cudaSuccess) return e;
  count_launch();
  if (!o.deterministic) {
    // atomic adds need a zeroed accumulator; the deterministic path initialises
    // it with the first contributor's stores instead
    e = cudaMemsetAsync(ws + L.dq_accum, 0, sizeof(float) * static_cast<size_t>(groups) * p.D, s);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

cudaError_t launch_bwd_main(const bsa_problem &p, const MaskParams &mp, const bsa_options &o,
                            const PlanSignature &sig, const CUtensorMap &tq, const CUtensorMap &tk,
                            const CUtensorMap &tv, const CUtensorMap &tdo, const float *lse,
                            void *dk, void *dv, const WsLayout &L, uint8_t *ws, cudaStream_t s) {
  BwdParams bp{};
  bp.mask = mp;
  bp.B = p.B;
  bp.H = p.H;
  bp.Sq = p.Sq;
  bp.Skv = p.Skv;
  bp.nM = L.nM;
  bp.nN = L.nN;
  bp.H_kv = p.H_kv;
  bp.kv_group = p.H / p.H_kv;
  bp.n_tickets = p.B * p.H_kv * L.nN;
  bp.scale = p.scale;
  bp.scale_log2 = p.scale * kLog2e;
  bp.col_ptr = reinterpret_cast<const int32_t *>(ws + L.col_ptr);
  bp.col_ent = reinterpret_cast<const uint32_t *>(ws + L.col_ent);
  bp.col_rank = reinterpret_cast<const int32_t *>(ws + L.col_rank);
  bp.perm = reinterpret_cast<const int32_t *>(ws + L.perm);
  bp.lse = lse;
  bp.delta = reinterpret_cast<const float *>(ws + L.delta);
  bp.dq_accum = reinterpret_cast<float *>(ws + L.dq_accum);
  bp.sem = reinterpret_cast<uint32_t *>(ws + L.sem);
  bp.dk = static_cast<__nv_bfloat16 *>(dk);
  bp.dv = static_cast<__nv_bfloat16 *>(dv);
  bp.k_sb = p.k_stride[0];
  bp.k_ss = p.k_stride[1];
  bp.k_sh = p.k_stride[2];
  bp.v_sb = p.v_stride[0];
  bp.v_ss = p.v_stride[1];
  bp.v_sh = p.v_stride[2];
  bp.deterministic = o.deterministic ? 1 : 0;
  bp.hdr = reinterpret_cast<uint32_t *>(ws + L.status);
  bp.timeout_ns = 2000000000ull;
  bp.sem_timeout_ns =
      o.sem_timeout_ns > 0 ? static_cast<uint64_t>(o.sem_timeout_ns) : 1000000000ull;
  for (int i = 0; i < kSigWords; ++i) bp.sig[i] = sig.w[i];
  bp.sig_mask = (1u << kSigWords) - 1u;
  // the column ticket is zero: the plan build clears it and every launch's
  // last CTA puts it back
  return (p.D == 64) ? run_bwd_main<64, 2, 2>(bp, tq, tk, tv, tdo, s)
                     : run_bwd_main<128, 2, 2>(bp, tq, tk, tv, tdo, s);
}

cudaError_t launch_bwd_convert(const bsa_problem &p, void *dq, const WsLayout &L, uint8_t *ws,
                               cudaStream_t s) {
  ConvertArgs a{};
  a.acc = reinterpret_cast<const float *>(ws + L.dq_accum);
  a.sem = reinterpret_cast<const uint32_t *>(ws + L.sem);
  a.hdr = reinterpret_cast<uint32_t *>(ws + L.status);
  a.row_ptr = reinterpret_cast<const int32_t *>(ws + L.row_ptr);
  a.dq = static_cast<__nv_bfloat16 *>(dq);
  a.sb = p.q_stride[0];
  a.ss = p.q_stride[1];
  a.sh = p.q_stride[2];
  a.B = p.B;
  a.H = p.H;
  a.Sq = p.Sq;
  a.nM = L.nM;
  const unsigned blocks = static_cast<unsigned>(static_cast<int64_t>(p.B) * p.H * L.nM * (kTile / 32));
  // a programmatic dependent of the backward main kernel
  const cudaError_t e = launch_pdl(p.D == 64 ? k_dq_convert<64> : k_dq_convert<128>, dim3(blocks), dim3(256), 0,
                                   s, a);
  if (e != cudaSuccess) return e;
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_zero_kv_grads(const bsa_problem &p, void *dk, void *dv, cudaStream_t s) {
  const int64_t pieces = static_cast<int64_t>(p.B) * p.Skv * p.H_kv * (p.D / 8);
  const int64_t want = (2 * pieces + 255) / 256;
  const unsigned blocks = static_cast<unsigned>(std::min<int64_t>(want, 8 * sm_count_bwd()));
  k_zero_kv_grads<<<blocks, 256, 0, s>>>(static_cast<__nv_bfloat16 *>(dk),
                                         static_cast<__nv_bfloat16 *>(dv), p.Skv, p.H_kv, p.D,
                                         pieces, p.k_stride[0], p.k_stride[1], p.k_stride[2],
                                         p.v_stride[0], p.v_stride[1], p.v_stride[2]);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_bwd(const bsa_problem &p, const MaskParams &mp, const bsa_options &o,
                       const PlanSignature &sig, const CUtensorMap &tq, const CUtensorMap &tk,
                       const CUtensorMap &tv, const CUtensorMap &tdo, const void *q, const void *out,
                       const void *dout, const float *lse, void *dq, void *dk, void *dv,
                       const WsLayout &L, uint8_t *ws, cudaStream_t s) {
  cudaError_t e = launch_bwd_preprocess(p, o, q, out, dout, L, ws, s);
  if (e != cudaSuccess) return e;
  e = launch_bwd_main(p, mp, o, sig, tq, tk, tv, tdo, lse, dk, dv, L, ws, s);
  if (e != cudaSuccess) return e;
  return launch_bwd_convert(p, dq, L, ws, s);
}

}  // namespace bsa
