// Forward pass (steps a2 and a3 of the hot path).
//
// a2  fixed-m bound: kmax[b,h] = max over valid keys of ||k_j||, qmax[b,h] and
//     per-row ||q_i||, and the per-head gate 2*scale*qmax*kmax <= G ("Fixed-m
//     softmax for 2D-ring x Ulysses attention (WAN 2.2)", introduction and
//     "Notes": heads whose bound cannot be proven safe keep online softmax).
// a3  the tiled exact softmax attention main loop over each q-block's row list
//     of non-empty tiles.  Online softmax keeps the running max in registers
//     (one query row per thread) and rescales lazily; fixed-m pins the max to
//     scale*||q_i||*kmax before streaming and needs neither max nor rescale.
//
// sm_100a design: one CTA per SM, persistent over work units (b, h, q-block).
//   warp 0      TMA producer: Q tile (double-buffered) and K/V tiles
//               (NS-stage ring), 128-byte swizzled boxes of 64 x 128.
//   warp 1      owns TMEM (512 columns) and issues tcgen05.mma from one lane:
//               S = Q K^T (SS, both K-major) into one of two S buffers, then
//               O += P V (TS: P read from TMEM, V as an MN-major B operand).
//   warps 2..5  softmax: tcgen05.ld of one S row per thread, mask on PARTIAL
//               tiles only, exp2, P packed to bf16 and tcgen05.st back over S,
//               lazy O rescale, epilogue O / l -> bf16 and LSE.
// TMEM columns: S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [256+D,256+2D).
#include <cfloat>

#include "internal.h"
#include "ptx.cuh"

namespace bsa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: tolerate p up to 2^8

struct FwdParams {
  MaskParams mask;
  int B, H, Sq, Skv, nM, n_units;
  float scale, scale_log2;
  const int32_t *row_ptr;
  const uint32_t *row_ent;
  __nv_bfloat16 *out;
  int64_t o_sb, o_ss, o_sh;
  float *lse;
  int fixed_mode;
  const float *kmax;   // [B, H]
  const float *qnorm;  // [B, H, Sq]
  const int32_t *gate; // [B, H]
  uint32_t *hdr;
  uint64_t timeout_ns;
  uint32_t sig[7];     // expected plan signature (B, Sq, Skv, flags, window, order, n_seqs)
  uint32_t sig_mask;   // which signature words must match
};

template <int D, int NS>
struct FwdSmem {
  static constexpr int kTileBytes = kTile * D * 2;
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + 2 * kTileBytes;
  static constexpr int kV = kK + NS * kTileBytes;
  static constexpr int kSeg = kV + NS * kTileBytes;     // int32 [2][128]
  static constexpr int kBar = kSeg + 2 * kTile * 4;     // mbarriers
  // barrier indices
  static constexpr int bQFull = 0, bQEmpty = 2, bKFull = 4, bKEmpty = 4 + NS, bVFull = 4 + 2 * NS,
                       bVEmpty = 4 + 3 * NS, bSFull = 4 + 4 * NS, bPFull = bSFull + 2,
                       bSFree = bPFull + 2, bODone = bSFree + 2, bOFree = bODone + 1,
                       bSegReady = bOFree + 2, bFinal = bSegReady + 2, kNumBars = bFinal + 1;
  static constexpr int kMisc = kBar + kNumBars * 8;      // tmem slot, abort flag
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kAlloc = kBytes + 1024;           // slack for 1024-byte alignment
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

template <int D, int NS>
__global__ void __launch_bounds__(192, 1)
k_attn_fwd(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
           const __grid_constant__ CUtensorMap tv, const FwdParams p) {
  using L = FwdSmem<D, NS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::kBar);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::kMisc);
  int *abort_flag = reinterpret_cast<int *>(sm + L::kMisc + 4);
  int32_t *seg_sm = reinterpret_cast<int32_t *>(sm + L::kSeg);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < L::kNumBars; ++i) {
      uint32_t cnt = 1;
      if (i == L::bPFull || i == L::bPFull + 1 || i == L::bOFree || i == L::bOFree + 1 ||
          i == L::bSegReady || i == L::bSegReady + 1)
        cnt = 128;
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
    for (int i = 0; i < 7; ++i) ok = ok && (!((p.sig_mask >> i) & 1u) || h[kHdrB + i] == p.sig[i]);
    if (!ok) wd.trip(BSA_ERR_PLAN_MISMATCH);
  }
  __syncthreads();

  const int nM = p.nM;
  constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, 0, 0);
  constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, 0, 1);
  constexpr int kTB = L::kTileBytes;

  if (wd.aborted()) {
    // plan mismatch: nothing to do
  } else if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t kv_it = 0, ul = 0, k_issued = 0, v_issued = 0, q_issued = 0;
      for (int u = blockIdx.x; u < p.n_units; u += gridDim.x) {
        const int bh = u / nM, m = u % nM, b = bh / p.H, h = bh % p.H;
        const int rs = p.row_ptr[b * nM + m], re = p.row_ptr[b * nM + m + 1];
        if (re == rs) continue;
        const int qb = ul & 1;
        if (ul >= 2 && !wd.wait(&bars[L::bQEmpty + qb], ((ul >> 1) - 1) & 1)) break;
        mbar_arrive_expect_tx(&bars[L::bQFull + qb], kTB);
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(sm + L::kQ + qb * kTB + c * 16384, &tq, &bars[L::bQFull + qb], c * 64,
                      m * kTile, h, b);
        ++q_issued;
        bool stop = false;
        for (int e = rs; e < re; ++e) {
          const int n = static_cast<int>(p.row_ent[e] & kIndexMask);
          const uint32_t st = kv_it % NS;
          const uint32_t use = kv_it / NS;
          if (kv_it >= NS && !wd.wait(&bars[L::bKEmpty + st], (use - 1) & 1)) { stop = true; break; }
          mbar_arrive_expect_tx(&bars[L::bKFull + st], kTB);
          for (int c = 0; c < D / 64; ++c)
            tma_load_4d(sm + L::kK + st * kTB + c * 16384, &tk, &bars[L::bKFull + st], c * 64,
                        n * kTile, h, b);
          ++k_issued;
          if (kv_it >= NS && !wd.wait(&bars[L::bVEmpty + st], (use - 1) & 1)) { stop = true; break; }
          mbar_arrive_expect_tx(&bars[L::bVFull + st], kTB);
          for (int c = 0; c < D / 64; ++c)
            tma_load_4d(sm + L::kV + st * kTB + c * 16384, &tv, &bars[L::bVFull + st], c * 64,
                        n * kTile, h, b);
          ++v_issued;
          ++kv_it;
        }
        ++ul;
        if (stop) break;
      }
      if (wd.aborted()) {
        // let every issued copy land before the CTA's shared memory goes away
        for (uint32_t t = (k_issued > NS ? k_issued - NS : 0); t < k_issued; ++t)
          drain_wait(&bars[L::bKFull + t % NS], (t / NS) & 1);
        for (uint32_t t = (v_issued > NS ? v_issued - NS : 0); t < v_issued; ++t)
          drain_wait(&bars[L::bVFull + t % NS], (t / NS) & 1);
        for (uint32_t t = (q_issued > 2 ? q_issued - 2 : 0); t < q_issued; ++t)
          drain_wait(&bars[L::bQFull + (t & 1)], (t >> 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t it = 0, ul = 0;
      for (int u = blockIdx.x; u < p.n_units; u += gridDim.x) {
        const int bh = u / nM, m = u % nM, b = bh / p.H;
        const int rs = p.row_ptr[b * nM + m], re = p.row_ptr[b * nM + m + 1];
        const int nt = re - rs;
        if (nt == 0) continue;
        const int qb = ul & 1, ob = ul & 1;
        if (!wd.wait(&bars[L::bQFull + qb], (ul >> 1) & 1)) break;
        tc_fence_after();
        const uint32_t q_addr = smem_u32(sm + L::kQ + qb * kTB);
        const uint32_t o_tmem = tmem + 256 + ob * D;
        bool stop = false;
        for (int j = 0; j <= nt && !stop; ++j) {
          if (j < nt) {
            const uint32_t t = it + j, s = t & 1, st = t % NS;
            if (!wd.wait(&bars[L::bKFull + st], (t / NS) & 1)) { stop = true; break; }
            if (t >= 2 && !wd.wait(&bars[L::bSFree + s], ((t >> 1) - 1) & 1)) { stop = true; break; }
            tc_fence_after();
            const uint32_t k_addr = smem_u32(sm + L::kK + st * kTB);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
              mma_ss(tmem + s * 128, sw128_desc(q_addr + off, 16, 1024),
                     sw128_desc(k_addr + off, 16, 1024), kIdescS, kk > 0);
            }
            mma_commit(&bars[L::bSFull + s]);
            mma_commit(&bars[L::bKEmpty + st]);
          }
          if (j >= 1) {
            const uint32_t t = it + j - 1, s = t & 1, st = t % NS;
            if (j == 1 && ul >= 2 && !wd.wait(&bars[L::bOFree + ob], ((ul >> 1) - 1) & 1)) {
              stop = true;
              break;
            }
            if (!wd.wait(&bars[L::bVFull + st], (t / NS) & 1)) { stop = true; break; }
            if (!wd.wait(&bars[L::bPFull + s], (t >> 1) & 1)) { stop = true; break; }
            tc_fence_after();
            const uint32_t v_addr = smem_u32(sm + L::kV + st * kTB);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              mma_ts(o_tmem, tmem + s * 128 + kk * 8, sw128_desc(v_addr + kk * 2048, 16384, 1024),
                     kIdescPV, (j > 1 || kk > 0) ? 1u : 0u);
            }
            mma_commit(&bars[L::bVEmpty + st]);
            mma_commit(&bars[L::bSFree + s]);
            mma_commit(&bars[L::bODone]);
          }
        }
        if (stop) break;
        mma_commit(&bars[L::bQEmpty + qb]);
        it += nt;
        ++ul;
      }
      // every tcgen05 op this thread issued is complete before TMEM is freed
      mma_commit(&bars[L::bFinal]);
      drain_wait(&bars[L::bFinal], 0);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const MaskParams &mk = p.mask;
    const bool use_seg = mk.seg_q != nullptr;
    // every lane waits, then the warp agrees, so tcgen05 .sync.aligned ops
    // never run on a diverged warp even when the watchdog trips
    auto wwait = [&](uint64_t *bar, uint32_t parity) {
      return __all_sync(0xffffffffu, wd.wait(bar, parity)) != 0;
    };
    uint32_t it = 0, ul = 0, ps = 0;
    bool stop = false;
    for (int u = blockIdx.x; u < p.n_units && !stop; u += gridDim.x) {
      const int bh = u / nM, m = u % nM, b = bh / p.H, h = bh % p.H;
      const int rs = p.row_ptr[b * nM + m], re = p.row_ptr[b * nM + m + 1];
      const int nt = re - rs;
      const int i = m * kTile + r;
      const bool row_ok = i < p.Sq;
      __nv_bfloat16 *orow = p.out + b * p.o_sb + static_cast<int64_t>(i) * p.o_ss + h * p.o_sh;
      float *lse_p = p.lse + (static_cast<int64_t>(bh)) * p.Sq + i;
      if (nt == 0) {
        if (row_ok) {
          const int4 z = make_int4(0, 0, 0, 0);
#pragma unroll
          for (int c = 0; c < D / 8; ++c) reinterpret_cast<int4 *>(orow)[c] = z;
          *lse_p = -INFINITY;
        }
        continue;
      }
      const int ob = ul & 1;
      const bool fixed = p.fixed_mode && p.gate[bh] != 0;
      float m_ref = -INFINITY, l = 0.f, l_r = 0.f;
      if (fixed) m_ref = row_ok ? p.scale_log2 * p.qnorm[static_cast<int64_t>(bh) * p.Sq + i] * p.kmax[bh] : 0.f;
      // row-constant part of the mask: allowed keys lie in [lo, hi]
      int lo = 0, hi = p.Skv - 1;
      if (mk.flags & BSA_MASK_CAUSAL_WINDOW) {
        hi = min(hi, i + mk.offset);
        if (mk.window > 0) lo = max(lo, i + mk.offset - mk.window + 1);
      }
      if (mk.flags & BSA_MASK_KV_VALID_LEN) hi = min(hi, mk.kv_valid_len[b] - 1);
      const int seg_i = (use_seg && row_ok) ? mk.seg_q[static_cast<int64_t>(b) * p.Sq + i] : INT_MIN;

      for (int j = 0; j < nt; ++j, ++it) {
        const uint32_t ent = p.row_ent[rs + j];
        const int n = static_cast<int>(ent & kIndexMask);
        const bool full = (ent & kFullBit) != 0;
        const uint32_t s = it & 1;
        // segment-id equality of this row against the tile's 128 keys, as a
        // 128-bit mask built before the S row occupies registers
        uint32_t seg_ok[4] = {~0u, ~0u, ~0u, ~0u};
        if (!full && use_seg) {
          int32_t *segt = seg_sm + (ps & 1) * kTile;
          const int jj = n * kTile + r;
          segt[r] = jj < p.Skv ? mk.seg_kv[static_cast<int64_t>(b) * p.Skv + jj] : INT_MIN + 1;
          mbar_arrive(&bars[L::bSegReady + (ps & 1)]);
          if (!wwait(&bars[L::bSegReady + (ps & 1)], (ps >> 1) & 1)) { stop = true; break; }
          ++ps;
          const int4 *seg4 = reinterpret_cast<const int4 *>(segt);
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            uint32_t bits = 0;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const int4 v = seg4[w * 8 + q];
              bits |= (static_cast<uint32_t>(v.x == seg_i) << (4 * q)) |
                      (static_cast<uint32_t>(v.y == seg_i) << (4 * q + 1)) |
                      (static_cast<uint32_t>(v.z == seg_i) << (4 * q + 2)) |
                      (static_cast<uint32_t>(v.w == seg_i) << (4 * q + 3));
            }
            seg_ok[w] = bits;
          }
        }
        if (!wwait(&bars[L::bSFull + s], (it >> 1) & 1)) { stop = true; break; }
        tc_fence_after();
        uint32_t x[128];
        const uint32_t t_s = tmem + lane_off + s * 128;
        tmem_ld32(t_s + 0, *reinterpret_cast<uint32_t(*)[32]>(&x[0]));
        tmem_ld32(t_s + 32, *reinterpret_cast<uint32_t(*)[32]>(&x[32]));
        tmem_ld32(t_s + 64, *reinterpret_cast<uint32_t(*)[32]>(&x[64]));
        tmem_ld32(t_s + 96, *reinterpret_cast<uint32_t(*)[32]>(&x[96]));
        tmem_wait_ld();
        float *f = reinterpret_cast<float *>(x);
        if (!full) {
          const int c_lo = lo - n * kTile, c_hi = hi - n * kTile;
#pragma unroll
          for (int c = 0; c < 128; ++c) {
            const bool ok = c >= c_lo && c <= c_hi && ((seg_ok[c >> 5] >> (c & 31)) & 1u);
            f[c] = ok ? f[c] : -INFINITY;
          }
        }
        if (!fixed) {
          float mx = -INFINITY;
#pragma unroll
          for (int c = 0; c < 128; ++c) mx = fmaxf(mx, f[c]);
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
            if (!wwait(&bars[L::bODone], (it - 1) & 1)) { stop = true; break; }
            tc_fence_after();
            const float a = resc ? alpha : 1.f;
            const uint32_t t_o = tmem + lane_off + 256 + ob * D;
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
        const float mu = (m_ref == -INFINITY) ? 0.f : m_ref;
        float rowsum = 0.f, rowsum_r = 0.f;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t pk[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float p0 = fast_exp2(fmaf(f[64 * half + 2 * c], p.scale_log2, -mu));
            const float p1 = fast_exp2(fmaf(f[64 * half + 2 * c + 1], p.scale_log2, -mu));
            pk[c] = pack_bf16x2(p0, p1);
            // two row sums: l over the exact weights (for LSE) and l_r over the
            // bf16-rounded weights the PV product uses (normalising O by l_r
            // makes numerator and denominator carry the same rounding)
            rowsum += p0 + p1;
            rowsum_r += __uint_as_float(pk[c] << 16) + __uint_as_float(pk[c] & 0xffff0000u);
          }
          // P (bf16 pairs) overwrites the first 64 columns of this S buffer
          tmem_st32(t_s + 32 * half, pk);
        }
        l += rowsum;
        l_r += rowsum_r;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars[L::bPFull + s]);
      }
      if (stop) break;
      // epilogue: O / l -> bf16, LSE
      if (!wwait(&bars[L::bODone], (it - 1) & 1)) break;
      tc_fence_after();
      const float inv = l_r > 0.f ? 1.f / l_r : 0.f;
      const uint32_t t_o = tmem + lane_off + 256 + ob * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(t_o + c * 32, o);
        tmem_wait_ld();
        if (row_ok) {
          uint32_t w[16];
#pragma unroll
          for (int q = 0; q < 16; ++q)
            w[q] = pack_bf16x2(__uint_as_float(o[2 * q]) * inv, __uint_as_float(o[2 * q + 1]) * inv);
          int4 *dst = reinterpret_cast<int4 *>(orow + c * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q) dst[q] = make_int4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(&bars[L::bOFree + ob]);
      if (row_ok) *lse_p = l > 0.f ? (m_ref + __log2f(l)) * kLn2 : -INFINITY;
      if (fixed && l > 0.f && l < 7.888609052210118e-31f /* 2^-100 */)
        atomicAdd(p.hdr + kHdrGateWarn, 1u);
      ++ul;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- fixed-m bound
// Norms of every (row, head) vector of Q or K.  Keys: running max per (b, h)
// over valid keys (padding and varlen alignment keys excluded).  Queries: the
// per-row norm is stored and the running max per (b, h) kept.
template <int D>
__global__ void __launch_bounds__(256) k_row_norms(const __nv_bfloat16 *__restrict__ x,
                                                   int64_t sb, int64_t ss, int64_t sh, int B,
                                                   int S, int H, int is_key, MaskParams mk,
                                                   float *__restrict__ rowmax,
                                                   float *__restrict__ qnorm) {
  constexpr int TPV = D / 8;  // threads per vector, 16 bytes each
  constexpr int kRows = 16;
  extern __shared__ unsigned int smax[];  // [H]
  for (int h = threadIdx.x; h < H; h += blockDim.x) smax[h] = 0u;
  __syncthreads();
  const int64_t blocks_per_b = (S + kRows - 1) / kRows;
  const int b = static_cast<int>(blockIdx.x / blocks_per_b);
  const int r0 = static_cast<int>(blockIdx.x % blocks_per_b) * kRows;
  const int g = threadIdx.x / TPV, t = threadIdx.x % TPV;
  const int groups = blockDim.x / TPV;
  // uniform trip count across the warp: the shuffles below need every lane
  for (int base = 0; base < kRows * H; base += groups) {
    const int pair = base + g;
    const int row = r0 + pair / H, h = pair % H;
    const bool in = pair < kRows * H && row < S;
    float acc = 0.f;
    if (in) {
      const int4 v = *reinterpret_cast<const int4 *>(x + b * sb + static_cast<int64_t>(row) * ss +
                                                    h * sh + t * 8);
      const __nv_bfloat162 *e = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = __bfloat1622float2(e[q]);
        acc = fmaf(f.x, f.x, acc);
        acc = fmaf(f.y, f.y, acc);
      }
    }
#pragma unroll
    for (int o = TPV / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (t == 0 && in) {
      const float nrm = sqrtf(acc);
      bool valid = true;
      if (is_key) {
        if (mk.flags & BSA_MASK_KV_VALID_LEN) valid = row < mk.kv_valid_len[b];
        if ((mk.flags & BSA_MASK_VARLEN) && mk.seg_kv != nullptr) valid = valid && mk.seg_kv[row] >= 0;
      } else {
        qnorm[(static_cast<int64_t>(b) * H + h) * S + row] = nrm;
      }
      if (valid) atomicMax(&smax[h], __float_as_uint(nrm));
    }
  }
  __syncthreads();
  for (int h = threadIdx.x; h < H; h += blockDim.x)
    if (smax[h] != 0u) atomicMax(reinterpret_cast<unsigned int *>(rowmax) + b * H + h, smax[h]);
}

__global__ void k_gate(int BH, float scale, float limit, const float *kmax_override,
                       float *kmax, const float *qmax, int32_t *gate) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= BH) return;
  const float km = kmax_override != nullptr ? kmax_override[t] : kmax[t];
  kmax[t] = km;
  gate[t] = (2.f * scale * qmax[t] * km <= limit) ? 1 : 0;
}

template <int D>
cudaError_t run_norms(const bsa_problem &p, const MaskParams &mp, const void *x,
                      const int64_t *st, int S, int is_key, float *rowmax, float *qnorm,
                      cudaStream_t s) {
  const int64_t blocks = static_cast<int64_t>(p.B) * ((S + 15) / 16);
  const size_t smem = sizeof(unsigned int) * p.H;
  k_row_norms<D><<<static_cast<unsigned>(blocks), 256, smem, s>>>(
      static_cast<const __nv_bfloat16 *>(x), st[0], st[1], st[2], p.B, S, p.H, is_key, mp,
      rowmax, qnorm);
  count_launch();
  return cudaGetLastError();
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

template <int D, int NS>
cudaError_t run_fwd(const FwdParams &fp, const CUtensorMap &tq, const CUtensorMap &tk,
                    const CUtensorMap &tv, cudaStream_t s) {
  using L = FwdSmem<D, NS>;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(k_attn_fwd<D, NS>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const int grid = std::min(fp.n_units, sm_count());
  k_attn_fwd<D, NS><<<grid, 192, L::kAlloc, s>>>(tq, tk, tv, fp);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fixed_m_bound(const bsa_problem &p, const MaskParams &mp,
                                 const bsa_options &o, const void *q, const void *k,
                                 const WsLayout &L, uint8_t *ws, cudaStream_t s) {
  float *kmax = reinterpret_cast<float *>(ws + L.kmax);
  float *qmax = reinterpret_cast<float *>(ws + L.qmax);
  float *qnorm = reinterpret_cast<float *>(ws + L.qnorm);
  cudaError_t e = cudaMemsetAsync(kmax, 0, sizeof(float) * p.B * p.H * 2, s);  // kmax, qmax
  if (e != cudaSuccess) return e;
  if (o.kmax_override == nullptr) {
    e = p.D == 64 ? run_norms<64>(p, mp, k, p.k_stride, p.Skv, 1, kmax, nullptr, s)
                  : run_norms<128>(p, mp, k, p.k_stride, p.Skv, 1, kmax, nullptr, s);
    if (e != cudaSuccess) return e;
  }
  e = p.D == 64 ? run_norms<64>(p, mp, q, p.q_stride, p.Sq, 0, qmax, qnorm, s)
                : run_norms<128>(p, mp, q, p.q_stride, p.Sq, 0, qmax, qnorm, s);
  if (e != cudaSuccess) return e;
  const float limit = o.gate_limit > 0.f ? o.gate_limit : 64.f;
  const int BH = p.B * p.H;
  k_gate<<<(BH + 127) / 128, 128, 0, s>>>(BH, p.scale, limit, o.kmax_override, kmax, qmax,
                                          reinterpret_cast<int32_t *>(ws + L.gate));
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_fwd(const bsa_problem &p, const MaskParams &mp, const bsa_options &o,
                       const PlanSignature &sig, const CUtensorMap &tq, const CUtensorMap &tk,
                       const CUtensorMap &tv, void *out, float *lse, const WsLayout &L,
                       uint8_t *ws, cudaStream_t s) {
  FwdParams fp{};
  fp.mask = mp;
  fp.B = p.B;
  fp.H = p.H;
  fp.Sq = p.Sq;
  fp.Skv = p.Skv;
  fp.nM = L.nM;
  fp.n_units = p.B * p.H * L.nM;
  fp.scale = p.scale;
  fp.scale_log2 = p.scale * kLog2e;
  fp.row_ptr = reinterpret_cast<const int32_t *>(ws + L.row_ptr);
  fp.row_ent = reinterpret_cast<const uint32_t *>(ws + L.row_ent);
  fp.out = static_cast<__nv_bfloat16 *>(out);
  fp.o_sb = p.o_stride[0];
  fp.o_ss = p.o_stride[1];
  fp.o_sh = p.o_stride[2];
  fp.lse = lse;
  fp.fixed_mode = o.softmax_mode == BSA_SOFTMAX_FIXED_M_GATED;
  fp.kmax = reinterpret_cast<const float *>(ws + L.kmax);
  fp.qnorm = reinterpret_cast<const float *>(ws + L.qnorm);
  fp.gate = reinterpret_cast<const int32_t *>(ws + L.gate);
  fp.hdr = reinterpret_cast<uint32_t *>(ws + L.status);
  fp.timeout_ns = 2000000000ull;
  for (int i = 0; i < 7; ++i) fp.sig[i] = sig.w[i];
  fp.sig_mask = 0x7Fu & ~(1u << 5);  // the forward does not depend on the kv-column order
  if (p.D == 64) return run_fwd<64, 3>(fp, tq, tk, tv, s);
  return run_fwd<128, 2>(fp, tq, tk, tv, s);
}

}  // namespace bsa
