// fa2_forward.cu -- exact attention forward pass for B200 (sm_100a).
//
// One CTA owns 256 query rows of one (batch, query head): two 128-row query
// tiles, Q0 and Q1, that take turns on the tensor cores.  The grid runs over
// (query block, head, batch) -- the sequence parallelism of "FlashAttention 2:
// Three Places the Chip Was Still Waiting", section 2.3 -- so a single long
// head still fills the machine.  Within the CTA, work is split by role rather
// than by data:
//
//   warps 0-3   softmax for Q0, one thread per query row (TMEM lane == row), so
//   warps 4-7   softmax for Q1   row statistics never leave a thread (the
//                                "partition on the index that survives to the
//                                output" rule, section 2.4)
//   warps 8-11  correction: rescales the O accumulator in TMEM when a row max
//               moved, and the epilogue (the single 1/l division, section 2.2)
//   warp 12     MMA issuer: tcgen05 S = Q K^T and O += P V into TMEM
//   warp 13     TMA producer: Q once, then K_j / V_j through a smem ring
//   warps 14-15 idle (they only complete the fourth warpgroup)
//
// TMEM columns: S0 | S1 | O0 | O1 (fp32).  P (bf16) is written by the softmax
// threads over the first half of their own S tile and consumed from TMEM by
// the PV MMA.  The overlap of loads, matrix products and softmax follows the
// producer/consumer idea of "FlashAttention-2 and -3: From Algebra to GPU
// Scheduling", "FlashAttention-3: overlap work on Hopper", rebuilt for
// tcgen05/TMEM.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "../../include/fa2.h"
#include "sm100_ptx.cuh"

namespace fa2 {

constexpr int kBlockM = 128;        // query rows per tile (one per TMEM lane)
constexpr int kBlockN = 128;        // keys per K/V tile
constexpr int kTiles = 2;           // query tiles per CTA
constexpr int kRowsPerCta = kBlockM * kTiles;
constexpr int kThreads = 512;
constexpr int kLaunchRegs = 128;    // 65536 / 512: the pool the register split below draws on
constexpr uint32_t kTmemCols = 512;
constexpr int kSwizzleBytes = 128;  // one swizzle atom row: 64 bf16
constexpr int kChunkBytes = kBlockM * kSwizzleBytes;  // 64 columns of a 128-row tile

// Register split (per thread): 2 softmax warpgroups x 192 + correction 48 +
// MMA/load warpgroup 80 = 512 = 4 x 128, i.e. exactly the launch pool.
constexpr int kRegsSoftmax = 192;
constexpr int kRegsCorrection = 48;
constexpr int kRegsOther = 80;
static_assert(2 * kRegsSoftmax + kRegsCorrection + kRegsOther == 4 * kLaunchRegs,
              "register split must equal the launch allocation");

enum Bar {
  BAR_Q = 0,         // [2] Q tile loaded (TMA tx)
  BAR_S = 2,         // [2] S tile complete (MMA commit)
  BAR_P = 4,         // [2] P written to TMEM and O rescaled (128 softmax + 128 correction threads)
  BAR_STATS = 6,     // [2] per-row rescale factor published (128 softmax threads)
  BAR_OFINAL = 8,    // [2] last PV complete (MMA commit)
  BAR_FSTATS = 10,   // [2] final row max / denominator published
  BAR_DONE = 12,     // all MMAs drained (MMA commit)
  BAR_KV_FULL = 13,  // [stages] K/V tile landed (TMA tx); then [stages] slot free (MMA commit)
};

template <int D>
struct Cfg {
  static constexpr int kChunks = D / 64;
  static constexpr int kTileBytes = kBlockM * D * 2;
  static constexpr int kStages = (D == 128) ? 4 : 8;
  static constexpr int kOffQ = 0;
  static constexpr int kOffKV = kOffQ + kTiles * kTileBytes;
  static constexpr int kOffAlpha = kOffKV + kStages * kTileBytes;
  static constexpr int kOffM = kOffAlpha + kTiles * kBlockM * 4;
  static constexpr int kOffL = kOffM + kTiles * kBlockM * 4;
  static constexpr int kNumBars = BAR_KV_FULL + 2 * kStages;
  static constexpr int kOffBar = kOffL + kTiles * kBlockM * 4;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kUsed = kOffMisc + 16;
  static constexpr int kSmemBytes = kUsed + 1024;  // slack for 1024-byte alignment
  // TMEM column of S_t (P_t reuses its first half) and of O_t
  __host__ __device__ static constexpr uint32_t col_s(int t) { return t ? 128u : 0u; }
  __host__ __device__ static constexpr uint32_t col_o(int t) { return 256u + (t ? D : 0); }
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(256 + 2 * D <= (int)kTmemCols, "TMEM budget");
};

struct Params {
  __nv_bfloat16* o;
  float* lse;
  int B, Hq, Hkv, Nq, Nk;
  int causal;
  int n_qblk;
  float c;            // |softmax_scale| * log2(e)
  int negate;         // softmax_scale < 0: compute S = -(Q K^T) so c stays >= 0
  unsigned long long limit_ns;
};

__device__ int g_status = 0;

// Number of K/V tiles query tile t of this CTA visits (0 if it has no valid row
// or no visible key).
__device__ __forceinline__ int kv_tiles_for(const Params& p, int r0) {
  if (r0 >= p.Nq) return 0;
  const int nkt = (p.Nk + kBlockN - 1) / kBlockN;
  if (!p.causal) return nkt;
  const int rlast = min(r0 + kBlockM - 1, p.Nq - 1);
  const long lim = (long)rlast + (long)p.Nk - (long)p.Nq;  // last visible key of the last row
  if (lim < 0) return 0;
  return min(nkt, (int)(lim / kBlockN) + 1);
}

// 2^x for a pair of fp32 values on the FMA pipe instead of the MUFU: a
// Cody-Waite split x = j + f with j = round(x), f in [-1/2, 1/2], then
// 2^f ~= c0 + f(c1 + f(c2 + f c3)) and 2^j applied by adding j to the exponent
// field.  The coefficients minimise the maximum relative error of the cubic on
// [-1/2, 1/2] (Remez exchange, fitted for this kernel): 7.5e-5, far below the
// 2^-9 rounding of the bf16 P it feeds.  Inputs are clamped at -125 so the
// result stays a normal number (2^-125 ~ 2e-38 stands in for anything
// smaller); callers use it only where no score is masked to -inf.
constexpr float kExp2C0 = 9.999280572e-01f;
constexpr float kExp2C1 = 6.932609677e-01f;
constexpr float kExp2C2 = 2.426111251e-01f;
constexpr float kExp2C3 = 5.517166853e-02f;
__device__ __forceinline__ void exp2_poly_pair(float x0, float x1, float& e0, float& e1) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23: adding it rounds to an integer
  const uint64_t x = f2_pack(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
  const uint64_t t = f2_add(x, f2_pack(kRound, kRound));         // low mantissa bits hold j
  const uint64_t jf = f2_add(t, f2_pack(-kRound, -kRound));      // j as a float
  const uint64_t f = f2_fma(jf, f2_pack(-1.f, -1.f), x);         // f = x - j
  uint64_t q = f2_fma(f2_pack(kExp2C3, kExp2C3), f, f2_pack(kExp2C2, kExp2C2));
  q = f2_fma(q, f, f2_pack(kExp2C1, kExp2C1));
  q = f2_fma(q, f, f2_pack(kExp2C0, kExp2C0));
  float q0, q1, t0, t1;
  f2_unpack(q, q0, q1);
  f2_unpack(t, t0, t1);
  e0 = __int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23));
  e1 = __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23));
}

// Pairs of each 32-column chunk whose exponentials go through exp2_poly_pair
// in unmasked tiles (the rest use the MUFU).  It moves work from the MUFU to
// the FMA pipe; measured on B200 it does not pay while the per-tile chain,
// not MUFU throughput, bounds the kernel (2 or 4 pairs: -4 to -8 % on causal
// 8k), so the default is 0.
#ifndef FA2_EMU_PAIRS
#define FA2_EMU_PAIRS 0
#endif
constexpr int kEmuPairs = FA2_EMU_PAIRS;

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    fa2_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const Params p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_addr(smem);
  float* sm_alpha = reinterpret_cast<float*>(smem + C::kOffAlpha);
  float* sm_m = reinterpret_cast<float*>(smem + C::kOffM);
  float* sm_l = reinterpret_cast<float*>(smem + C::kOffL);
  const uint32_t bar0 = sbase + C::kOffBar;
  auto bar = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- block -> (query block, head, batch); heaviest query blocks first ----
  const int hb_count = p.Hq * p.B;
  const int hb = blockIdx.x % hb_count;
  const int qb = p.n_qblk - 1 - static_cast<int>(blockIdx.x / hb_count);
  const int hq = hb % p.Hq;
  const int b = hb / p.Hq;
  const int hk = hq / (p.Hq / p.Hkv);
  const int row0 = qb * kRowsPerCta;  // first row of Q0; Q1 starts kBlockM later
  const int nt0 = kv_tiles_for(p, row0);
  const int nt1 = kv_tiles_for(p, row0 + kBlockM);
  const int n_kv = max(nt0, nt1);
  const int koff = p.Nk - p.Nq;  // causal diagonal offset

  // ---- setup ----
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int i = 0; i < BAR_KV_FULL; ++i) {
      uint32_t cnt = 1;
      if ((i >= BAR_STATS && i < BAR_STATS + 2) || (i >= BAR_FSTATS && i < BAR_FSTATS + 2))
        cnt = kBlockM;
      if (i >= BAR_P && i < BAR_P + 2) cnt = 2 * kBlockM;
      mbar_init(bar(i), cnt);
    }
    for (int s = 0; s < 2 * C::kStages; ++s) mbar_init(bar(BAR_KV_FULL + s), 1);
    fence_mbar_init();
  }
  if (warp == 12) {
    tmem_alloc(smem_addr(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  if (warp == 13 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitGuard g{abort_flag, &g_status, p.limit_ns};
  const bool aligned_ok = (sbase & 1023u) == 0;  // always true by construction

  // Register split, one instruction site per warpgroup.
  if (warp < 8) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
  } else if (warp < 12) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsCorrection));
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsOther));
  }

  if (warp < 8) {
    // =================== softmax: one thread per query row ===================
    const int t = warp >> 2;
    const int q4 = warp & 3;
    const int rt = q4 * 32 + lane;  // row within the tile == TMEM lane
    const int r0t = row0 + t * kBlockM;
    const int ntt = t ? nt1 : nt0;
    const int row = r0t + rt;
    const uint32_t tS = tmem + (static_cast<uint32_t>(q4 * 32) << 16) + C::col_s(t);
    const float c = p.c;
    float m_raw = -INFINITY;  // running max of the raw scores
    float m_sc = 0.f;         // m_raw * c (0 while no key was visible)
    float l = 0.f;            // running denominator, relative to m_sc
    for (int j = 0; j < ntt; ++j) {
      if (!mbar_wait(bar(BAR_S + t), j & 1, g, FA2_SITE_S_READY, j)) break;
      tc_fence_after();
      float s[kBlockN];
#pragma unroll
      for (int k = 0; k < kBlockN / 32; ++k) {
        uint32_t r[32];
        tmem_ld32(tS + 32 * k, r);
#pragma unroll
        for (int i = 0; i < 32; ++i) s[32 * k + i] = __uint_as_float(r[i]);
      }
      tmem_wait_ld();
      // causal diagonal / ragged key tail: only these tiles pay for masking
      const int kbase = j * kBlockN;
      const bool masked = (kbase + kBlockN > p.Nk) || (p.causal && kbase + kBlockN - 1 > r0t + koff);
      int lim = kBlockN - 1;  // last visible column of this tile for this row
      if (masked) {
        lim = min(lim, p.Nk - 1 - kbase);
        if (p.causal) lim = min(lim, row + koff - kbase);
#pragma unroll
        for (int i = 0; i < kBlockN; ++i)
          if (i > lim) s[i] = -INFINITY;
      }
      // row max: 8 independent chains of 3-input max (max is exact in any order)
      float mp[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mp[k] = fmaxf(s[2 * k], s[2 * k + 1]);
#pragma unroll
      for (int i = 16; i < kBlockN; i += 16)
#pragma unroll
        for (int k = 0; k < 8; ++k) mp[k] = fmax3(mp[k], s[i + 2 * k], s[i + 2 * k + 1]);
      const float mx = fmax3(fmax3(mp[0], mp[1], mp[2]), fmax3(mp[3], mp[4], mp[5]),
                             fmax3(mp[6], mp[7], m_raw));
      const float m_sc_new = (mx == -INFINITY) ? 0.f : mx * c;
      // rescale factor for what was accumulated so far: exactly 1 when the max
      // did not move (then O is left untouched), 0 when nothing was visible yet
      float alpha = 1.f;
      if (mx != m_raw) alpha = (m_raw == -INFINITY) ? 0.f : ex2_approx(m_sc - m_sc_new);
      if (j > 0) {
        // Publish the rescale factor; the correction warps apply it to O
        // while this thread computes the exponentials.
        sm_alpha[t * kBlockM + rt] = alpha;
        mbar_arrive(bar(BAR_STATS + t));
      }
      // p = 2^(s*c - m*c): one packed FMA per pair of scores, then ex2
      const uint64_t cc = f2_pack(c, c), nn = f2_pack(-m_sc_new, -m_sc_new);
      uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};  // packed partial row sums (+0.0f pairs)
      const uint32_t tP = tS;  // P (bf16) overwrites the first half of S
      auto exp_row = [&](auto emu_tag) {
        constexpr int kEmu = decltype(emu_tag)::value;
#pragma unroll
        for (int k = 0; k < kBlockN / 32; ++k) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int c0 = 32 * k + 2 * i;
            float x0, x1, e0, e1;
            f2_unpack(f2_fma(f2_pack(s[c0], s[c0 + 1]), cc, nn), x0, x1);
            if (i >= 16 - kEmu) {
              exp2_poly_pair(x0, x1, e0, e1);
            } else {
              e0 = ex2_approx(x0);
              e1 = ex2_approx(x1);
            }
            acc[i & 3] = f2_add(acc[i & 3], f2_pack(e0, e1));
            pk[i] = pack_bf16x2(e0, e1);
          }
          tmem_st16(tP + 16 * k, pk);
        }
      };
      if (masked)  // masked scores are -inf and must give exactly 0: MUFU only
        exp_row(std::integral_constant<int, 0>{});
      else
        exp_row(std::integral_constant<int, kEmuPairs>{});
      float sum[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) f2_unpack(acc[i], sum[2 * i], sum[2 * i + 1]);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(BAR_P + t));
      l = l * alpha + (((sum[0] + sum[1]) + (sum[2] + sum[3])) + ((sum[4] + sum[5]) + (sum[6] + sum[7])));
      m_raw = mx;
      m_sc = m_sc_new;
    }
    sm_m[t * kBlockM + rt] = (m_raw == -INFINITY) ? -INFINITY : m_sc;
    sm_l[t * kBlockM + rt] = l;
    mbar_arrive(bar(BAR_FSTATS + t));
  } else if (warp < 12) {
    // ============== correction (O rescale) and epilogue warps ==============
    const int q4 = warp & 3;
    const int rt = q4 * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    bool ok = true;
    for (int j = 0; j < n_kv && ok; ++j) {
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (j >= (t ? nt1 : nt0)) continue;
        if (j == 0) {  // nothing accumulated yet: O_t is ready for the first PV
          mbar_arrive(bar(BAR_P + t));
          continue;
        }
        if (!mbar_wait(bar(BAR_STATS + t), (j - 1) & 1, g, FA2_SITE_STATS_READY, j)) {
          ok = false;
          break;
        }
        const float alpha = sm_alpha[t * kBlockM + rt];
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
          // the previous PV into O_t completed before S_t(j) did, which the
          // softmax threads waited for before publishing alpha
          tc_fence_after();
          const uint32_t tO = tmem + lane_off + C::col_o(t);
          const uint64_t aa = f2_pack(alpha, alpha);
#pragma unroll 1
          for (int ch = 0; ch < D / 16; ++ch) {
            uint32_t r[16];
            tmem_ld16(tO + 16 * ch, r);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              float lo, hi;
              f2_unpack(f2_mul(f2_pack(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])), aa), lo, hi);
              r[2 * i] = __float_as_uint(lo);
              r[2 * i + 1] = __float_as_uint(hi);
            }
            tmem_st16(tO + 16 * ch, r);
          }
          tmem_wait_st();
        }
        tc_fence_before();
        mbar_arrive(bar(BAR_P + t));
      }
    }
    // epilogue: O / l -> bf16, LSE = ln(sum exp(scale * s))
#pragma unroll 1
    for (int t = 0; t < 2; ++t) {
      const int row = row0 + t * kBlockM + rt;
      const bool valid = row < p.Nq;
      float inv_l = 0.f, lse = -INFINITY;
      bool have_o = false;
      if ((t ? nt1 : nt0) > 0 && ok) {
        if (!mbar_wait(bar(BAR_OFINAL + t), 0, g, FA2_SITE_O_FINAL, t) ||
            !mbar_wait(bar(BAR_FSTATS + t), 0, g, FA2_SITE_FINAL_STATS, t)) {
          ok = false;
        } else {
          tc_fence_after();
          const float m_sc = sm_m[t * kBlockM + rt];
          const float l = sm_l[t * kBlockM + rt];
          if (l > 0.f) {
            inv_l = 1.f / l;
            lse = (m_sc + log2f(l)) * 0.69314718055994530942f;
          }
          have_o = true;
        }
      }
      __nv_bfloat16* orow = p.o + ((static_cast<size_t>(b) * p.Nq + row) * p.Hq + hq) * D;
      const uint32_t tO = tmem + lane_off + C::col_o(t);
#pragma unroll 1
      for (int ch = 0; ch < D / 16; ++ch) {
        uint32_t r[16];
        if (have_o) {
          tmem_ld16(tO + 16 * ch, r);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) r[i] = 0u;
        }
        uint4 w[2];
        uint32_t* wp = reinterpret_cast<uint32_t*>(w);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          wp[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * inv_l, __uint_as_float(r[2 * i + 1]) * inv_l);
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + 16 * ch);
          dst[0] = w[0];
          dst[1] = w[1];
        }
      }
      if (valid) p.lse[(static_cast<size_t>(b) * p.Hq + hq) * p.Nq + row] = lse;
    }
  } else if (warp == 12) {
    // ============================ MMA issuer warp ============================
    // The whole warp follows the schedule (warp-uniform waits and descriptor
    // arithmetic); one elected lane -- always the same one in a converged warp,
    // so its commits cover its own MMAs -- issues each group of tcgen05
    // instructions (8 MMAs and their commit) inside a single elected block.
    // Measured on B200: a group issued this way takes ~23 cycles per MMA and
    // runs ahead of the tensor core, while a per-MMA elect/warp-sync costs
    // 50-60 cycles each and a single divergent lane is slower still when the
    // softmax warps sharing this SM sub-partition keep the issue slots busy.
    if (aligned_ok) {
      const uint32_t idS = idesc_bf16_f32(kBlockM, kBlockN, false, p.negate != 0);
      const uint32_t idPV = idesc_bf16_f32(kBlockM, D, true, false);
      const uint32_t sQ = sbase + C::kOffQ;
      const uint32_t sKV = sbase + C::kOffKV;
      auto stage_of = [&](int it) { return it % C::kStages; };
      auto phase_of = [&](int it) { return static_cast<uint32_t>((it / C::kStages) & 1); };
      // The start-address field is the low 14 bits of the descriptor (address
      // >> 4, below 2^14 for any shared-memory address), so advancing along K
      // inside a tile is a plain add of (byte offset >> 4).
      const uint64_t dQ = sw128_desc(sQ, 16, 1024);             // K-major, 8-row groups 1 KiB apart
      const uint64_t dK = sw128_desc(sKV, 16, 1024);            // K-major
      const uint64_t dV = sw128_desc(sKV, kChunkBytes, 1024);   // MN-major: d-chunks 16 KiB apart
      auto commit = [&](uint32_t b) {
        if (elect_one()) umma_commit(b);
        __syncwarp();
      };
      // One elected block per tile and KV step: O_t += P_t V_j, then (if any)
      // S_t(j+1) = Q_t K_{j+1}^T, then the commits that publish completion.
      // S_t(j+1) overwrites the TMEM columns that held P_t(j); it is issued by
      // the same thread after the PV that reads them, and one thread's tcgen05
      // MMAs execute in issue order.
      auto issue_block = [&](int t, int j, bool pv, bool s_next, uint32_t c_pv1, uint32_t c_pv2,
                             uint32_t c_s1, uint32_t c_s2) {
        const uint32_t dS = tmem + C::col_s(t), dO = tmem + C::col_o(t);
        const uint64_t bV = dV + ((stage_of(2 * j + 1) * C::kTileBytes) >> 4);
        const uint64_t a0 = dQ + ((t * C::kTileBytes) >> 4);
        const uint64_t bK = dK + ((stage_of(2 * j + 2) * C::kTileBytes) >> 4);
        if (elect_one()) {
          if (pv) {
#pragma unroll
            for (int kk = 0; kk < kBlockN / 16; ++kk)
              umma_ts(dO, dS + kk * 8, bV + ((kk * 16 * kSwizzleBytes) >> 4), idPV,
                      (j > 0 || kk > 0) ? 1u : 0u);
            if (c_pv1) umma_commit(c_pv1);
            if (c_pv2) umma_commit(c_pv2);
          }
          if (s_next) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = ((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4;
              umma_ss(dS, a0 + off, bK + off, idS, kk > 0 ? 1u : 0u);
            }
            if (c_s1) umma_commit(c_s1);
            if (c_s2) umma_commit(c_s2);
          }
        }
        __syncwarp();
      };
      // S_t(0)
      auto issue_s0 = [&](int t, uint32_t c2) {
        const uint32_t dS = tmem + C::col_s(t);
        const uint64_t a0 = dQ + ((t * C::kTileBytes) >> 4);
        const uint64_t bK = dK + ((stage_of(0) * C::kTileBytes) >> 4);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = ((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4;
            umma_ss(dS, a0 + off, bK + off, idS, kk > 0 ? 1u : 0u);
          }
          umma_commit(bar(BAR_S + t));
          if (c2) umma_commit(c2);
        }
        __syncwarp();
      };
      auto free_of = [&](int it) { return bar(BAR_KV_FULL + C::kStages + stage_of(it)); };
      bool ok = true;
      if (nt0 > 0) ok = mbar_wait_warp(bar(BAR_Q + 0), 0, g, FA2_SITE_Q_LOADED, 0);
      if (ok && nt1 > 0) ok = mbar_wait_warp(bar(BAR_Q + 1), 0, g, FA2_SITE_Q_LOADED, 1);
      if (ok && n_kv > 0) {
        ok = mbar_wait_warp(bar(BAR_KV_FULL + stage_of(0)), phase_of(0), g, FA2_SITE_KV_LOADED, 0);
        if (ok) {
          tc_fence_after();
          if (nt0 > 0) issue_s0(0, nt1 > 0 ? 0u : free_of(0));
          if (nt1 > 0) issue_s0(1, free_of(0));
        }
      }
      for (int j = 0; j < n_kv && ok; ++j) {
        const int itV = 2 * j + 1, itK = 2 * j + 2;
        const bool next = (j + 1 < n_kv);
        // operands of this step (normally landed long ago); checked while the
        // tensor pipe still holds the previous block
        if (!mbar_wait_warp(bar(BAR_KV_FULL + stage_of(itV)), phase_of(itV), g, FA2_SITE_KV_LOADED, j)) break;
        if (next && !mbar_wait_warp(bar(BAR_KV_FULL + stage_of(itK)), phase_of(itK), g,
                                    FA2_SITE_KV_LOADED, j + 1))
          break;
        // tile 0: PV0(j) and S0(j+1); V_j / K_{j+1} are freed here when tile 1 has no use for them
        if (j < nt0) {
          if (!mbar_wait_warp(bar(BAR_P + 0), j & 1, g, FA2_SITE_P_READY, j)) break;
          tc_fence_after();
          issue_block(0, j, true, j + 1 < nt0, j == nt0 - 1 ? bar(BAR_OFINAL + 0) : 0u,
                      j >= nt1 ? free_of(itV) : 0u, bar(BAR_S + 0), j + 1 >= nt1 ? free_of(itK) : 0u);
        }
        // tile 1: PV1(j) and S1(j+1); the last use of V_j and K_{j+1}
        if (j < nt1) {
          if (!mbar_wait_warp(bar(BAR_P + 1), j & 1, g, FA2_SITE_P_READY, j)) break;
          tc_fence_after();
          issue_block(1, j, true, j + 1 < nt1, free_of(itV), j == nt1 - 1 ? bar(BAR_OFINAL + 1) : 0u,
                      bar(BAR_S + 1), free_of(itK));
        }
      }
      // drain: every MMA issued above has completed before TMEM is released
      // (not cut short by the abort flag: tensor-core work always finishes)
      volatile int no_abort = 0;
      const WaitGuard drain{&no_abort, &g_status, p.limit_ns};
      commit(bar(BAR_DONE));
      mbar_wait_warp(bar(BAR_DONE), 0, drain, FA2_SITE_MMA_DRAIN, 0);
    }
  } else if (warp == 13) {
    // ============================ TMA producer warp ============================
    if (aligned_ok) {
      const uint32_t sQ = sbase + C::kOffQ;
      const uint32_t sKV = sbase + C::kOffKV;
#pragma unroll 1
      for (int t = 0; t < 2; ++t) {
        if ((t ? nt1 : nt0) == 0) continue;
        if (elect_one()) {
          mbar_arrive_expect_tx(bar(BAR_Q + t), C::kTileBytes);
#pragma unroll
          for (int ch = 0; ch < C::kChunks; ++ch)
            tma_load_4d(sQ + t * C::kTileBytes + ch * kChunkBytes, &tmQ, bar(BAR_Q + t), ch * 64, hq,
                        row0 + t * kBlockM, b);
        }
        __syncwarp();
      }
      int issued = 0;
      bool ok = true;
      for (int it = 0; it < 2 * n_kv; ++it) {
        const int st = it % C::kStages;
        if (it >= C::kStages &&
            !mbar_wait_warp(bar(BAR_KV_FULL + C::kStages + st), ((it / C::kStages) & 1) ^ 1, g,
                            FA2_SITE_KV_FREE, it)) {
          ok = false;
          break;
        }
        if (elect_one()) {
          mbar_arrive_expect_tx(bar(BAR_KV_FULL + st), C::kTileBytes);
          const CUtensorMap* map = (it & 1) ? &tmV : &tmK;
#pragma unroll
          for (int ch = 0; ch < C::kChunks; ++ch)
            tma_load_4d(sKV + st * C::kTileBytes + ch * kChunkBytes, map, bar(BAR_KV_FULL + st),
                        ch * 64, hk, (it >> 1) * kBlockN, b);
        }
        __syncwarp();
        issued = it + 1;
      }
      if (!ok) {
        // Give the copies already in flight time to land before the CTA exits.
        volatile int no_abort = 0;
        const WaitGuard drain{&no_abort, &g_status, p.limit_ns};
        for (int it = (issued > C::kStages ? issued - C::kStages : 0); it < issued; ++it)
          mbar_wait_warp(bar(BAR_KV_FULL + it % C::kStages), (it / C::kStages) & 1, drain,
                         FA2_SITE_LOAD_DRAIN, it);
        if (nt0 > 0) mbar_wait_warp(bar(BAR_Q + 0), 0, drain, FA2_SITE_LOAD_DRAIN, 0);
        if (nt1 > 0) mbar_wait_warp(bar(BAR_Q + 1), 0, drain, FA2_SITE_LOAD_DRAIN, 1);
      }
    }
  }

  // ---- teardown: all TMEM traffic is finished before the columns are freed ----
  tc_fence_before();
  __syncthreads();
  if (warp == 12) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// One warp waits on an mbarrier nothing arrives on; the bounded wait runs out.
__global__ void selftest_timeout_kernel(unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar_storage;
  __shared__ int abort_storage;
  if (threadIdx.x == 0) {
    abort_storage = 0;
    mbar_init(smem_addr(&bar_storage), 1);
    fence_mbar_init();
  }
  __syncwarp();
  const WaitGuard g{&abort_storage, &g_status, limit_ns};
  mbar_wait(smem_addr(&bar_storage), 0, g, FA2_SITE_SELFTEST, 0);
  __syncwarp();
  if (threadIdx.x == 0) mbar_arrive(smem_addr(&bar_storage));  // leave the barrier consistent
}

// ------------------------------- host side -------------------------------

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// 4-D map over a bf16 [B, N, H, d] tensor with a (64 x 1 x 128 x 1) box and
// 128-byte swizzle: one box is 128 sequence rows x 64 channels of one head.
static bool encode_bnhd(CUtensorMap* map, const void* base, int B, int N, int H, int d) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(d) * 2,
                                 static_cast<cuuint64_t>(H) * d * 2,
                                 static_cast<cuuint64_t>(N) * H * d * 2};
  const cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(kBlockM), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static int validate_shape(int B, int Hq, int Hkv, int Nq, int Nk, int d) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || Nk <= 0 || Hq % Hkv != 0) return FA2_ERR_BAD_SHAPE;
  if (d != 64 && d != 128) return FA2_ERR_HEAD_DIM;
  // TMA: every byte stride below 2^40; the grid below 2^31 blocks.
  const long long lim = 1LL << 40;
  const long long q_bytes = 2LL * B * Nq * Hq * d;
  const long long kv_bytes = 2LL * B * Nk * Hkv * d;
  if (q_bytes >= lim || kv_bytes >= lim) return FA2_ERR_SIZE;
  const long long nblk = (static_cast<long long>(Nq) + kRowsPerCta - 1) / kRowsPerCta;
  if (nblk * Hq * B > INT_MAX) return FA2_ERR_SIZE;
  return FA2_OK;
}

template <int D>
static int launch(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                  int Hkv, int Nq, int Nk, int causal, float scale, cudaStream_t stream) {
  using C = Cfg<D>;
  static std::once_flag once;
  static int setup_status = FA2_OK;
  std::call_once(once, [] {
    cudaFuncAttributes attr;
    if (cudaFuncGetAttributes(&attr, fa2_fwd_kernel<D>) != cudaSuccess) {
      setup_status = FA2_ERR_LAUNCH;
      return;
    }
    if (attr.numRegs != kLaunchRegs) {  // the setmaxnreg split assumes exactly this pool
      setup_status = FA2_ERR_BUILD;
      return;
    }
    if (cudaFuncSetAttribute(fa2_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::kSmemBytes) != cudaSuccess)
      setup_status = FA2_ERR_LAUNCH;
  });
  if (setup_status != FA2_OK) return setup_status;

  CUtensorMap tq, tk, tv;
  if (!encode_bnhd(&tq, q, B, Nq, Hq, D) || !encode_bnhd(&tk, k, B, Nk, Hkv, D) ||
      !encode_bnhd(&tv, v, B, Nk, Hkv, D))
    return FA2_ERR_LAUNCH;

  Params p;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Nq = Nq;
  p.Nk = Nk;
  p.causal = causal ? 1 : 0;
  p.n_qblk = (Nq + kRowsPerCta - 1) / kRowsPerCta;
  // c is kept strictly positive so a masked score (-inf) always maps to
  // exp2(-inf) = 0; for softmax_scale == 0 every unmasked exponent is then
  // c * (s - m) ~ 1e-30 * O(1e4), which rounds to exp2(0) = 1 as required.
  p.c = std::fmax(std::fabs(scale) * 1.4426950408889634f, 1e-30f);
  p.negate = scale < 0.f ? 1 : 0;
  p.limit_ns = 1000000000ull;  // 1 s per wait; a healthy wait takes microseconds
  const unsigned grid = static_cast<unsigned>(p.n_qblk) * Hq * B;
  fa2_fwd_kernel<D><<<grid, kThreads, C::kSmemBytes, stream>>>(tq, tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? FA2_OK : FA2_ERR_LAUNCH;
}

static int check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA2_ERR_DEVICE;
  static int cached[64];
  static std::once_flag flags[64];
  if (dev < 0 || dev >= 64) return FA2_ERR_DEVICE;
  std::call_once(flags[dev], [dev] {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    cached[dev] = (major == 10 && minor == 0) ? FA2_OK : FA2_ERR_DEVICE;
  });
  return cached[dev];
}

}  // namespace fa2

using namespace fa2;

extern "C" int fa2_forward(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                           int Hq, int Hkv, int Nq, int Nk, int d, int causal, float softmax_scale,
                           void* stream) {
  if (!q || !k || !v || !o || !lse) return FA2_ERR_NULL_POINTER;
  const int sv = validate_shape(B, Hq, Hkv, Nq, Nk, d);
  if (sv != FA2_OK) return sv;
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
       reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(o)) & 15u)
    return FA2_ERR_ALIGNMENT;
  if (reinterpret_cast<uintptr_t>(lse) & 3u) return FA2_ERR_ALIGNMENT;
  if (!std::isfinite(softmax_scale)) return FA2_ERR_SCALE;
  const int dv = check_device();
  if (dv != FA2_OK) return dv;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d == 128) return launch<128>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, causal, softmax_scale, s);
  return launch<64>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, causal, softmax_scale, s);
}

extern "C" const char* fa2_status_string(int status) {
  switch (status) {
    case FA2_OK: return "ok";
    case FA2_ERR_NULL_POINTER: return "null pointer argument";
    case FA2_ERR_BAD_SHAPE: return "bad shape: sizes must be > 0 and Hq a multiple of Hkv";
    case FA2_ERR_HEAD_DIM: return "unsupported head dimension (64 or 128)";
    case FA2_ERR_ALIGNMENT: return "misaligned pointer (q/k/v/o need 16 bytes, lse 4 bytes)";
    case FA2_ERR_SCALE: return "softmax_scale is not finite";
    case FA2_ERR_DEVICE: return "current device is not an sm_100 (B200-class) GPU";
    case FA2_ERR_LAUNCH: return "CUDA call or kernel launch failed";
    case FA2_ERR_SIZE: return "problem exceeds the supported tensor or grid extent";
    case FA2_ERR_BUILD: return "kernel image does not match its register plan";
    default: return "unknown status";
  }
}

extern "C" int fa2_debug_status(void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int value = 0;
  const int zero = 0;
  if (cudaMemcpyFromSymbolAsync(&value, g_status, sizeof(int), 0, cudaMemcpyDeviceToHost, s) !=
      cudaSuccess)
    return -1;
  if (cudaStreamSynchronize(s) != cudaSuccess) return -1;
  if (cudaMemcpyToSymbolAsync(g_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, s) !=
      cudaSuccess)
    return -1;
  if (cudaStreamSynchronize(s) != cudaSuccess) return -1;
  return value;
}

extern "C" int fa2_selftest_timeout(void* stream, long long limit_ns) {
  if (limit_ns < 1000000LL || limit_ns > 10000000000LL) return FA2_ERR_SIZE;
  const int dv = check_device();
  if (dv != FA2_OK) return dv;
  selftest_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<unsigned long long>(limit_ns));
  return cudaGetLastError() == cudaSuccess ? FA2_OK : FA2_ERR_LAUNCH;
}

extern "C" long long fa2_num_blocks(int B, int H, int N, int rows_per_block) {
  if (B <= 0 || H <= 0 || N <= 0 || rows_per_block <= 0) return -1;
  const long long tiles = (static_cast<long long>(N) + rows_per_block - 1) / rows_per_block;
  return tiles * H * B;
}

extern "C" int fa2_launch_plan(int B, int Hq, int Hkv, int Nq, int Nk, int d, int* grid_blocks,
                               int* threads_per_block, int* smem_bytes, int* rows_per_block) {
  const int sv = validate_shape(B, Hq, Hkv, Nq, Nk, d);
  if (sv != FA2_OK) return sv;
  if (grid_blocks) *grid_blocks = static_cast<int>(fa2_num_blocks(B, Hq, Nq, kRowsPerCta));
  if (threads_per_block) *threads_per_block = kThreads;
  if (smem_bytes) *smem_bytes = (d == 128) ? Cfg<128>::kSmemBytes : Cfg<64>::kSmemBytes;
  if (rows_per_block) *rows_per_block = kRowsPerCta;
  return FA2_OK;
}
