// fa2_backward.cuh -- backward pass of exact attention (dQ, dK, dV) for sm_100a.
//
// Included by fa2_forward.cu, inside namespace fa2: one translation unit, so
// both passes share the bounded-wait status word and the helpers above.
//
// Given the forward's O and LSE and an upstream gradient dO, with
// P_ij = exp(scale * q_i . k_j - LSE_i) over the keys row i sees:
//
//   D_i   = dO_i . O_i                     (= sum_j P_ij dP_ij)
//   dV_j  = sum_i P_ij dO_i
//   dP_ij = dO_i . v_j,   dS_ij = P_ij (dP_ij - D_i)
//   dQ_i  = scale * sum_j dS_ij k_j,   dK_j = scale * sum_i dS_ij q_i
//
// ("FlashAttention 2: Three Places the Chip Was Still Waiting", section 2.5
// reports the forward+backward figures; the gradients are the chain rule on
// the forward's definition.)  As in the forward, nothing of size Nq x Nk is
// stored: P is recomputed tile by tile from the saved LSE.
//
// Work decomposition: one CTA per (128-key block, KV head, batch) owns dK and
// dV of its keys in tensor memory for the whole pass and walks every query
// tile of every query head of its group that sees any of its keys, so dK and
// dV need no atomics (GQA sums the group's heads in place).  dQ is the only
// output shared between CTAs: each CTA adds its 128 x d contribution per
// query tile into an fp32 accumulator -- half by vector reductions from
// registers, half by a TMA bulk reduction staged in the shared-memory slot of
// that tile's dO, which every MMA has finished reading once the dQ tile is
// complete -- and a last kernel rounds the accumulator to bf16 (scale is
// applied before the reduction).  Each CTA walks its query tiles starting at a different one
// (rotated by the key block), so the CTAs of one head running at the same
// time add into different dQ rows.
//
// Per query tile (tensor memory: S^T | dP^T | dV | dK):
//   MMA   S^T = K Q^T (SS), dP^T = V dO^T (SS)            -> "S ready"
//   WG0   P^T = exp2(S^T c - LSE_i log2 e), dS^T = P^T (dP^T - D_i),
//         both written back to tensor memory as bf16 over S^T / dP^T, and
//         dS^T into shared memory as the MN-major A operand of dQ -> "P ready"
//   MMA   dV += P^T dO (TS), dK += dS^T Q (TS), dQ_tile = dS K (SS, into the
//         S^T columns, after the dV MMA read P^T: one thread's MMAs run in
//         issue order)                                     -> "dQ ready"
//   WG0/1 read dQ_tile, scale          -> "dQ free": the next tile's S^T
//         may overwrite the columns; WG0 adds its half with red.global,
//         WG1 stages its half in the tile's dO slot  -> "half staged"
//   RED   warp 10 issues the bulk reduce-add of WG1's half and waits until
//         it has read the slot -> "slot read"; the producer refills the slot
//         (two tiles later) after that.
//
// Roles: warps 0-3 (WG0) and 4-7 (WG1) split the query columns of P / dS
// (one thread per key row) and of the dQ read-out (one thread per query
// row); warp 8 MMA issuer; warp 9 TMA producer; warp 10 dQ reducer (a bulk
// async-group can only be waited for by the thread that issued it, so the
// wait sits on a warp with nothing else to do); warp 11 idle.  No register
// split: 384 threads leave 168 registers each.

constexpr int kBwdThreads = 384;

// 4-D tiled bulk reduction: adds one box of shared memory into global memory
// (fp32 add, element-wise atomic with respect to other reductions), as part
// of this thread's current bulk async-group.
__device__ __forceinline__ void tma_reduce_add_4d(const void* map, uint32_t src, int c0, int c1, int c2,
                                                  int c3) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.4d.global.shared::cta.add.tile.bulk_group"
      " [%0, {%2, %3, %4, %5}], [%1];" ::"l"(reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
__device__ __forceinline__ void bulk_commit_group() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Every bulk operation this thread committed has finished reading shared memory.
__device__ __forceinline__ void bulk_wait_group_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Every bulk operation this thread committed has completed.
__device__ __forceinline__ void bulk_wait_group0() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
// Element-wise fp32 add of four consecutive floats into global memory.
__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

enum BwdBar {
  BB_KV = 0,        // K and V tiles of this CTA landed (TMA tx)
  BB_QFULL = 1,     // [2] Q tile + its LSE / D rows landed (32 producer lanes + TMA tx)
  BB_QFREE = 3,     // [2] Q slot free: its last MMA (dK) completed
  BB_OFULL = 5,     // [2] dO tile landed (TMA tx)
  BB_OFREE = 7,     // [2] dO slot free: its last MMA (dV) completed
  BB_SDP = 9,       // S^T and dP^T complete
  BB_PDS = 10,      // P^T, dS^T in tensor memory and dS in shared memory (128 WG0 threads)
  BB_DQ = 11,       // dQ tile complete
  BB_DQFREE = 12,   // dQ tile read out (128 WG1 threads)
  BB_DONE = 13,     // every MMA complete: dK, dV final
  BB_STAGED = 14,   // [2 slot] warpgroup 1's half of the dQ tile staged in the dO slot (128 threads)
  BB_STGREAD = 16,  // [2 slot] its bulk reduction has read the slot (1 thread)
  BB_COUNT = 18,
};

template <int D>
struct BCfg {
  static constexpr int kTileBytes = kBlockM * D * 2;  // 128 rows x d bf16
  static constexpr int kChunks = D / 64;
  static constexpr int kOStages = 2;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kTileBytes;
  static constexpr int kOffQ = kOffV + kTileBytes;                 // [2]
  static constexpr int kOffO = kOffQ + 2 * kTileBytes;             // [kOStages]
  static constexpr int kOffDS = kOffO + kOStages * kTileBytes;     // 128 keys x 128 queries bf16
  static constexpr int kOffLse = kOffDS + kBlockN * kBlockM * 2;   // [2][128] log2-domain LSE
  static constexpr int kOffDelta = kOffLse + 2 * kBlockM * 4;      // [2][128] D_i
  static constexpr int kOffBar = kOffDelta + 2 * kBlockM * 4;
  static constexpr int kOffMisc = kOffBar + BB_COUNT * 8;
  static constexpr int kUsed = kOffMisc + 16;
  // At d = 128 the tiles leave less than 1 KiB of the 227 KiB for aligning the
  // base to 1024 bytes; the kernel checks the slack it got (dynamic shared
  // memory normally starts 1024-aligned, so the slack is 0).
  static constexpr int kSmemBytes = (kUsed + 1024 < 232448) ? kUsed + 1024 : 232448;
  static constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 256 + D;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(kColDK + D <= 512, "TMEM budget");
};

// TMEM column (within the S^T or dP^T block) of the bf16 P^T / dS^T values of
// query chunk ch (32 queries, 16 columns): 0, 16, 64, 80.
__host__ __device__ constexpr uint32_t bf16_col(int ch) { return 16u * ch + (ch >= 2 ? 32u : 0u); }

struct BwdParams {
  const float* lse2;    // [B, Hq, Nq] LSE * log2 e (+inf for a row with no visible key)
  const float* delta;   // [B, Hq, Nq] D_i
  float* dq_acc;        // [B, Nq, Hq, d] fp32, zero before the main kernel
  __nv_bfloat16* dk;    // [B, Nk, Hkv, d]
  __nv_bfloat16* dv;    // [B, Nk, Hkv, d]
  int B, Hq, Hkv, Nq, Nk;
  int wl, wr;
  float scale;
  float c;              // scale * log2 e (any sign)
  uint32_t limit_ns;
};

// Query tiles [lo, hi] whose rows see any key of key block kb (hi < lo: none).
__host__ __device__ inline void query_tiles_for(const BwdParams& p, int kb, int& lo, int& hi) {
  const int koff = p.Nk - p.Nq;
  const int k0 = kb * kBlockN;
  const int k1 = (k0 + kBlockN - 1 < p.Nk - 1) ? k0 + kBlockN - 1 : p.Nk - 1;
  int first = (p.wr >= 0) ? k0 - p.wr - koff : 0;      // g_i + wr >= k0
  int last = (p.wl >= 0) ? k1 + p.wl - koff : p.Nq - 1;  // g_i - wl <= k1
  if (first < 0) first = 0;
  if (last > p.Nq - 1) last = p.Nq - 1;
  if (first > last) {
    lo = 0;
    hi = -1;
    return;
  }
  lo = first / kBlockM;
  hi = last / kBlockM;
}

// D_i = dO_i . O_i and the log2-domain LSE; zeroes the dQ accumulator.
// Each lane takes 8 consecutive elements (16 bytes of bf16) of a row, so a
// row is D / 8 lanes and every load and store is a 16-byte vector; the dot
// product is summed across the row's lanes.
template <int D>
__global__ void __launch_bounds__(256) fa2_bwd_prep_kernel(const __nv_bfloat16* __restrict__ o,
                                                           const __nv_bfloat16* __restrict__ dout,
                                                           const float* __restrict__ lse,
                                                           float* lse2, float* delta, float* dq_acc,
                                                           int B, int Hq, int Nq) {
  constexpr int kLanesPerRow = D / 8;
  constexpr int kRowsPerWarp = 32 / kLanesPerRow;
  const int lane = threadIdx.x % 32;
  const long long warp_id = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) / 32;
  const long long row = warp_id * kRowsPerWarp + lane / kLanesPerRow;  // enumerates [B, Nq, Hq]
  const int c8 = 8 * (lane % kLanesPerRow);                              // first element of the lane
  const bool valid = row < static_cast<long long>(B) * Nq * Hq;
  float acc = 0.f;
  if (valid) {
    const uint4 ov = __ldg(reinterpret_cast<const uint4*>(o + row * D + c8));
    const uint4 gv = __ldg(reinterpret_cast<const uint4*>(dout + row * D + c8));
    const uint32_t ow[4] = {ov.x, ov.y, ov.z, ov.w}, gw[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc = fmaf(__uint_as_float(ow[e] << 16), __uint_as_float(gw[e] << 16), acc);
      acc = fmaf(__uint_as_float(ow[e] & 0xffff0000u), __uint_as_float(gw[e] & 0xffff0000u), acc);
    }
    float4* qrow = reinterpret_cast<float4*>(dq_acc + row * D + c8);
    qrow[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    qrow[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int off = kLanesPerRow / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (valid && c8 == 0) {
    const int hq = static_cast<int>(row % Hq);
    const long long bi = row / Hq;
    const int i = static_cast<int>(bi % Nq), b = static_cast<int>(bi / Nq);
    const long long s = (static_cast<long long>(b) * Hq + hq) * Nq + i;
    const float l = lse[s];
    delta[s] = acc;
    lse2[s] = (l == -INFINITY) ? INFINITY : l * 1.4426950408889634f;
  }
}

// dQ = bf16(dQ accumulator).
__global__ void __launch_bounds__(256) fa2_bwd_dq_kernel(const float* __restrict__ dq_acc,
                                                         __nv_bfloat16* dq, long long n4) {
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= n4) return;
  const float4 v = reinterpret_cast<const float4*>(dq_acc)[idx];
  uint2 w;
  w.x = pack_bf16x2(v.x, v.y);
  w.y = pack_bf16x2(v.z, v.w);
  reinterpret_cast<uint2*>(dq)[idx] = w;
}


template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    fa2_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                   const __grid_constant__ CUtensorMap tmDQ, const BwdParams p) {
  using C = BCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_addr(smem);
  if (sbase + C::kUsed > smem_addr(smem_raw) + C::kSmemBytes) {  // uniform: every thread leaves
    if (threadIdx.x == 0) atomicCAS(&g_status, 0, (FA2_SITE_SMEM_ALIGN << 16) | 1);
    return;
  }
  const uint32_t bar0 = sbase + C::kOffBar;
  auto bar = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };
  float* sm_lse = reinterpret_cast<float*>(smem + C::kOffLse);
  float* sm_delta = reinterpret_cast<float*>(smem + C::kOffDelta);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int kb = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int group = p.Hq / p.Hkv;
  const int koff = p.Nk - p.Nq;
  int qt_lo, qt_hi;
  query_tiles_for(p, kb, qt_lo, qt_hi);
  const int n_qt = qt_hi - qt_lo + 1 > 0 ? qt_hi - qt_lo + 1 : 0;
  // iteration it: head hk*group + it / n_qt, query tile qt_lo + (it % n_qt + kb) % n_qt
  const int n_it = n_qt * group;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int i = 0; i < BB_COUNT; ++i) {
      uint32_t cnt = 1;
      if (i == BB_QFULL || i == BB_QFULL + 1) cnt = 32;
      if (i == BB_PDS || i == BB_DQFREE) cnt = 2 * kBlockM;
      if (i == BB_STAGED || i == BB_STAGED + 1) cnt = kBlockM;
      mbar_init(bar(i), cnt);
    }
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(smem_addr(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  if (warp == 9 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmO);
    tma_prefetch_desc(&tmDQ);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitGuard g{smem_addr(const_cast<int*>(abort_flag)), p.limit_ns};

  if (warp < 8) {
    // ===== WG0 / WG1: P^T and dS^T for query columns [64 wg, 64 wg + 64) of
    // every key row, then that half of the dQ tile's columns =====
    const int wg = warp >> 2;
    const int q4 = warp & 3;
    const int kr = q4 * 32 + lane;            // key row in the block == TMEM lane (dQ: query row)
    const int key = kb * kBlockN + kr;
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::kColS, tDP = tmem + lane_off + C::kColDP;
    const uint32_t sDS = sbase + C::kOffDS;
    bool ok = true;
    for (int it = 0; it < n_it && ok; ++it) {
      const int st = it & 1;
      const int hq = hk * group + it / n_qt;
      const int q0 = (qt_lo + (it % n_qt + kb) % n_qt) * kBlockM;
      if (!mbar_wait_warp(bar(BB_SDP), it & 1, g, FA2_SITE_S_READY, it)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // visible query columns of this key row: g_i - wl <= key <= g_i + wr
      // (a tile needs masking when some key lies right of some row's right
      // bound, left of some row's left bound, or past the sequences' ends)
      const int k0 = kb * kBlockN;
      const bool masked = (q0 + kBlockM > p.Nq) || (k0 + kBlockN > p.Nk) ||
                          (p.wr >= 0 && k0 + kBlockN - 1 > q0 + koff + p.wr) ||
                          (p.wl >= 0 && k0 < q0 + kBlockM - 1 + koff - p.wl);
      const uint32_t sL = sbase + C::kOffLse + 4u * st * kBlockM, sDl = sbase + C::kOffDelta + 4u * st * kBlockM;
#pragma unroll 1
      for (int ch = 2 * wg; ch < 2 * wg + 2; ++ch) {
        uint32_t rs[32], rd[32];
        tmem_ld32(tS + 32 * ch, rs);
        tmem_ld32(tDP + 32 * ch, rd);
        tmem_wait_ld();
        uint32_t pk[16], dk[16];
        // P and dS of the chunk; the visibility test is compiled only into
        // the copy that masked tiles run (predicating it into every tile
        // costs a fifth of the kernel's time)
        auto pds = [&](auto mk) {
          constexpr bool kMasked = decltype(mk)::value;
#pragma unroll
          for (int i4 = 0; i4 < 8; ++i4) {
            // log2 LSE and D of 4 query rows (broadcast shared-memory reads,
            // addressed in the shared window)
            float4 l4, d4;
            asm("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(l4.x), "=f"(l4.y), "=f"(l4.z), "=f"(l4.w)
                : "r"(sL + 4u * (32 * ch + 4 * i4)));
            asm("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(d4.x), "=f"(d4.y), "=f"(d4.z), "=f"(d4.w)
                : "r"(sDl + 4u * (32 * ch + 4 * i4)));
            const float lz[4] = {l4.x, l4.y, l4.z, l4.w}, dz[4] = {d4.x, d4.y, d4.z, d4.w};
            float pv[4], dsv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int qc = 32 * ch + 4 * i4 + e;  // query column in the tile
              float pe = ex2_approx(fmaf(__uint_as_float(rs[4 * i4 + e]), p.c, -lz[e]));
              if constexpr (kMasked) {
                const int gi = q0 + qc + koff;  // diagonal key of query row q0 + qc
                const bool vis = (q0 + qc < p.Nq) && (key < p.Nk) && (p.wl < 0 || key >= gi - p.wl) &&
                                 (p.wr < 0 || key <= gi + p.wr);
                if (!vis) pe = 0.f;
              }
              pv[e] = pe;
              dsv[e] = pe * (__uint_as_float(rd[4 * i4 + e]) - dz[e]);
            }
            pk[2 * i4] = pack_bf16x2(pv[0], pv[1]);
            pk[2 * i4 + 1] = pack_bf16x2(pv[2], pv[3]);
            dk[2 * i4] = pack_bf16x2(dsv[0], dsv[1]);
            dk[2 * i4 + 1] = pack_bf16x2(dsv[2], dsv[3]);
          }
        };
        if (masked)
          pds(std::true_type{});
        else
          pds(std::false_type{});
        // bf16 P^T / dS^T over S^T / dP^T columns this warpgroup has consumed:
        // chunk ch goes to columns bf16_col(ch) (0, 16, 64, 80), so neither
        // warpgroup overwrites scores the other has yet to read
        tmem_st16(tS + bf16_col(ch), pk);
        tmem_st16(tDP + bf16_col(ch), dk);
        // dS^T row into shared memory: queries [32 ch, 32 ch + 32) of key row
        // kr, MN-major SW128 (query chunk of 64 = 16 KiB block, 128 B per key)
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int q8 = 32 * ch + 8 * u;  // first of 8 queries in this 16-byte unit
          const int blk = q8 / 64, unit = (q8 % 64) / 8;
          const uint32_t addr = sDS + blk * (kBlockN * 128) + kr * 128 + ((unit ^ (kr & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(dk[4 * u]),
                       "r"(dk[4 * u + 1]), "r"(dk[4 * u + 2]), "r"(dk[4 * u + 3])
                       : "memory");
        }
      }
      if (!ok) break;
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(BB_PDS));

      // ---- this warpgroup's half of the dQ tile (lane = query row) ----
      if (!mbar_wait_warp(bar(BB_DQ), it & 1, g, FA2_SITE_O_FINAL, it)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // Read the half row (query row q0 + kr) into registers and hand the
      // columns back to the MMA at once; the reduction into the accumulator
      // then overlaps the next tile's products.
      uint32_t r[D / 2];
#pragma unroll
      for (int c = 0; c < D / 64; ++c)
        tmem_ld32(tS + wg * (D / 2) + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(r + 32 * c));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bar(BB_DQFREE));
      // Add this half row (scaled) into the fp32 accumulator.  The TMA unit
      // also brings in every tile's Q and dO, so the two halves take
      // different paths: warpgroup 0 uses vector reductions from registers
      // (the load/store path), warpgroup 1 a bulk (TMA) reduction.
      if (wg == 0) {
        const int row = q0 + kr;
        if (row < p.Nq) {
          float* dst = p.dq_acc + ((static_cast<size_t>(b) * p.Nq + row) * p.Hq + hq) * D;
#pragma unroll
          for (int i = 0; i < D / 8; ++i)
            red_add_v4(dst + 4 * i, __uint_as_float(r[4 * i]) * p.scale, __uint_as_float(r[4 * i + 1]) * p.scale,
                       __uint_as_float(r[4 * i + 2]) * p.scale, __uint_as_float(r[4 * i + 3]) * p.scale);
        }
      } else {
        // staged as D/64 boxes of 128 rows x 32 fp32 columns in the 128-byte
        // swizzle of the dQ tensor map, in the tile's dO slot (exactly one
        // half tile at d = 64 and 128): every MMA that read it completed
        // before the dQ tile did, and the producer loads tile it + 2 into it
        // only after the reduction has read it
        const uint32_t sstg = sbase + C::kOffO + (it & 1) * C::kTileBytes;
#pragma unroll
        for (int bx = 0; bx < D / 64; ++bx)
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const uint32_t addr = sstg + bx * (kBlockM * 128) + kr * 128 + ((u ^ (kr & 7)) << 4);
            const int c = 32 * bx + 4 * u;
            asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                         "f"(__uint_as_float(r[c]) * p.scale), "f"(__uint_as_float(r[c + 1]) * p.scale),
                         "f"(__uint_as_float(r[c + 2]) * p.scale), "f"(__uint_as_float(r[c + 3]) * p.scale)
                         : "memory");
          }
        fence_proxy_async_smem();
        mbar_arrive(bar(BB_STAGED + (it & 1)));
      }
    }
    // ---- epilogue: WG0 writes dV, WG1 dK (scaled), rows of this key block ----
    if (ok && n_it > 0 && !mbar_wait_warp(bar(BB_DONE), 0, g, FA2_SITE_MMA_DRAIN, 0)) ok = false;
    tc_fence_after();
    // (the TMEM loads run on the whole warp -- tcgen05.ld is warp-collective --
    // and only the stores are limited to keys inside the sequence)
    const bool valid = key < p.Nk;
    if (ok) {
      const size_t rowk = ((static_cast<size_t>(b) * p.Nk + (valid ? key : 0)) * p.Hkv + hk) * D;
      const int which = wg;
      {
        const uint32_t tcol = tmem + lane_off + (which ? C::kColDK : C::kColDV);
        const float mul = which ? p.scale : 1.f;
        __nv_bfloat16* dst = (which ? p.dk : p.dv) + rowk;
#pragma unroll 1
        for (int ch = 0; ch < D / 16; ++ch) {
          uint32_t r[16];
          if (n_it > 0) {
            tmem_ld16(tcol + 16 * ch, r);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) r[i] = 0u;
          }
          uint4 w0, w1;
          w0.x = pack_bf16x2(__uint_as_float(r[0]) * mul, __uint_as_float(r[1]) * mul);
          w0.y = pack_bf16x2(__uint_as_float(r[2]) * mul, __uint_as_float(r[3]) * mul);
          w0.z = pack_bf16x2(__uint_as_float(r[4]) * mul, __uint_as_float(r[5]) * mul);
          w0.w = pack_bf16x2(__uint_as_float(r[6]) * mul, __uint_as_float(r[7]) * mul);
          w1.x = pack_bf16x2(__uint_as_float(r[8]) * mul, __uint_as_float(r[9]) * mul);
          w1.y = pack_bf16x2(__uint_as_float(r[10]) * mul, __uint_as_float(r[11]) * mul);
          w1.z = pack_bf16x2(__uint_as_float(r[12]) * mul, __uint_as_float(r[13]) * mul);
          w1.w = pack_bf16x2(__uint_as_float(r[14]) * mul, __uint_as_float(r[15]) * mul);
          if (valid) {
            reinterpret_cast<uint4*>(dst + 16 * ch)[0] = w0;
            reinterpret_cast<uint4*>(dst + 16 * ch)[1] = w1;
          }
        }
      }
    }
  } else if (warp == 8) {
    // ============ MMA issuer ============
    const uint32_t sK = sbase + C::kOffK, sV = sbase + C::kOffV;
    const uint32_t idSS = idesc_bf16_f32_ab(kBlockN, kBlockM, false, false);  // S^T, dP^T: K-major A and B
    const uint32_t idTS = idesc_bf16_f32_ab(kBlockN, D, false, true);         // dV, dK: B (dO, Q) MN-major
    const uint32_t idDQ = idesc_bf16_f32_ab(kBlockM, D, true, true);          // dQ: A (dS) and B (K) MN-major
    const uint64_t dK_k = sw128_desc(sK, 16, 1024), dV_k = sw128_desc(sV, 16, 1024);
    const uint64_t dK_mn = sw128_desc(sK, kChunkBytes, 1024);
    const uint64_t dDS = sw128_desc(sbase + C::kOffDS, kBlockN * 128, 1024);
    auto commit = [&](uint32_t bb) {
      if (elect_one()) umma_commit(bb);
      __syncwarp();
    };
    bool ok = n_it > 0 && mbar_wait_warp(bar(BB_KV), 0, g, FA2_SITE_KV_LOADED, 0);
    // S^T(it) and dP^T(it): dP^T goes first, as soon as Q / dO have landed; S^T
    // also waits until the previous dQ tile has left the S^T columns.
    auto issue_s_dp = [&](int it) -> bool {
      const int qs = it & 1, os = it % C::kOStages;
      if (!mbar_wait_warp(bar(BB_QFULL + qs), (it >> 1) & 1, g, FA2_SITE_Q_LOADED, it) ||
          !mbar_wait_warp(bar(BB_OFULL + os), (it / C::kOStages) & 1, g, FA2_SITE_Q_LOADED, it))
        return false;
      tc_fence_after();
      const uint32_t sQ = sbase + C::kOffQ + qs * C::kTileBytes;
      const uint32_t sO = sbase + C::kOffO + os * C::kTileBytes;
      uint64_t aK = dK_k, aV = dV_k, bQ = sw128_desc(sQ, 16, 1024), bO = sw128_desc(sO, 16, 1024);
      asm volatile("" : "+l"(aK), "+l"(aV), "+l"(bQ), "+l"(bO));
      // K advances 32 B in a swizzle atom, then jumps to the next 64-column chunk
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          umma_ss(tmem + C::kColDP, aV, bO, idSS, kk > 0 ? 1u : 0u);
          const uint32_t step = ((kk & 3) == 3) ? (kChunkBytes - 3 * 32) >> 4 : 32 >> 4;
          aV += step;
          bO += step;
        }
      }
      __syncwarp();
      if (it > 0 && !mbar_wait_warp(bar(BB_DQFREE), (it - 1) & 1, g, FA2_SITE_O_RESCALED, it)) return false;
      tc_fence_after();
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          umma_ss(tmem + C::kColS, aK, bQ, idSS, kk > 0 ? 1u : 0u);
          const uint32_t step = ((kk & 3) == 3) ? (kChunkBytes - 3 * 32) >> 4 : 32 >> 4;
          aK += step;
          bQ += step;
        }
        umma_commit(bar(BB_SDP));
      }
      __syncwarp();
      return true;
    };
    if (ok) ok = issue_s_dp(0);
    for (int it = 0; it < n_it && ok; ++it) {
      const int qs = it & 1, os = it % C::kOStages;
      const uint32_t sQ = sbase + C::kOffQ + qs * C::kTileBytes;
      const uint32_t sO = sbase + C::kOffO + os * C::kTileBytes;
      if (!mbar_wait_warp(bar(BB_PDS), it & 1, g, FA2_SITE_P_READY, it)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint64_t bOm = sw128_desc(sO, kChunkBytes, 1024), bQm = sw128_desc(sQ, kChunkBytes, 1024);
      uint64_t aDS = dDS, bKm = dK_mn;
      asm volatile("" : "+l"(bOm), "+l"(bQm), "+l"(aDS), "+l"(bKm));
      if (elect_one()) {
        // dV += P^T dO and dK += dS^T Q: A from TMEM (8 columns per 16 queries),
        // B MN-major (16 query rows = 2 KiB per step)
#pragma unroll
        for (int kk = 0; kk < kBlockM / 16; ++kk) {
          umma_ts(tmem + C::kColDV, tmem + C::kColS + bf16_col(kk >> 1) + 8 * (kk & 1), bOm, idTS,
                  (it > 0 || kk > 0) ? 1u : 0u);
          bOm += (16 * kSwizzleBytes) >> 4;
        }
        umma_commit(bar(BB_OFREE + os));
#pragma unroll
        for (int kk = 0; kk < kBlockM / 16; ++kk) {
          umma_ts(tmem + C::kColDK, tmem + C::kColDP + bf16_col(kk >> 1) + 8 * (kk & 1), bQm, idTS,
                  (it > 0 || kk > 0) ? 1u : 0u);
          bQm += (16 * kSwizzleBytes) >> 4;
        }
        umma_commit(bar(BB_QFREE + qs));
        // dQ tile = dS K: A = dS (queries x keys, MN-major in shared memory),
        // B = K (keys x d, MN-major); 16 keys = 2 KiB per step in both
#pragma unroll
        for (int kk = 0; kk < kBlockN / 16; ++kk) {
          umma_ss(tmem + C::kColS, aDS, bKm, idDQ, kk > 0 ? 1u : 0u);
          aDS += (16 * kSwizzleBytes) >> 4;
          bKm += (16 * kSwizzleBytes) >> 4;
        }
        umma_commit(bar(BB_DQ));
      }
      __syncwarp();
      // the next tile's dP^T may start now (its columns were last read by the
      // dK MMA above, and MMAs of one thread run in issue order)
      if (it + 1 < n_it && !issue_s_dp(it + 1)) {
        ok = false;
        break;
      }
    }
    // drain: every MMA complete before dK / dV are read and TMEM is freed
    const WaitGuard drain{0u, p.limit_ns};
    if (n_it > 0) {
      commit(bar(BB_DONE));
      mbar_wait_warp(bar(BB_DONE), 0, drain, FA2_SITE_MMA_DRAIN, 0);
    }
  } else if (warp == 9) {
    // ============ TMA producer ============
    bool ok = n_it > 0;
    if (ok) {
      if (elect_one()) {
        mbar_arrive_expect_tx(bar(BB_KV), 2 * C::kTileBytes);
#pragma unroll
        for (int ch = 0; ch < C::kChunks; ++ch) {
          tma_load_4d(sbase + C::kOffK + ch * kChunkBytes, &tmK, bar(BB_KV), ch * 64, hk, kb * kBlockN, b);
          tma_load_4d(sbase + C::kOffV + ch * kChunkBytes, &tmV, bar(BB_KV), ch * 64, hk, kb * kBlockN, b);
        }
      }
      __syncwarp();
    }
    int it = 0;
    for (; it < n_it && ok; ++it) {
      const int qs = it & 1, os = it % C::kOStages;
      const int hq = hk * group + it / n_qt;
      const int q0 = (qt_lo + (it % n_qt + kb) % n_qt) * kBlockM;
      if (it >= 2 && !mbar_wait_warp(bar(BB_QFREE + qs), ((it >> 1) - 1) & 1, g, FA2_SITE_KV_FREE, it)) {
        ok = false;
        break;
      }
      // LSE (log2 domain) and D of the tile's rows; rows past Nq see nothing
      const size_t srow = (static_cast<size_t>(b) * p.Hq + hq) * p.Nq;
#pragma unroll
      for (int e = 0; e < kBlockM / 32; ++e) {
        const int r = e * 32 + lane, i = q0 + r;
        sm_lse[qs * kBlockM + r] = (i < p.Nq) ? p.lse2[srow + i] : INFINITY;
        sm_delta[qs * kBlockM + r] = (i < p.Nq) ? p.delta[srow + i] : 0.f;
      }
      if (elect_one()) {
        mbar_arrive_expect_tx(bar(BB_QFULL + qs), C::kTileBytes);
#pragma unroll
        for (int ch = 0; ch < C::kChunks; ++ch)
          tma_load_4d(sbase + C::kOffQ + qs * C::kTileBytes + ch * kChunkBytes, &tmQ, bar(BB_QFULL + qs),
                      ch * 64, hq, q0, b);
      } else {
        mbar_arrive(bar(BB_QFULL + qs));
      }
      __syncwarp();
      if (it >= C::kOStages &&
          (!mbar_wait_warp(bar(BB_OFREE + os), ((it / C::kOStages) - 1) & 1, g, FA2_SITE_KV_FREE, it) ||
           !mbar_wait_warp(bar(BB_STGREAD + os), ((it / C::kOStages) - 1) & 1, g, FA2_SITE_KV_FREE, it))) {
        ok = false;
        break;
      }
      if (elect_one()) {
        mbar_arrive_expect_tx(bar(BB_OFULL + os), C::kTileBytes);
#pragma unroll
        for (int ch = 0; ch < C::kChunks; ++ch)
          tma_load_4d(sbase + C::kOffO + os * C::kTileBytes + ch * kChunkBytes, &tmO, bar(BB_OFULL + os),
                      ch * 64, hq, q0, b);
      }
      __syncwarp();
    }
    if (!ok && n_it > 0) {
      // let the copies in flight land before the CTA exits
      const WaitGuard drain{0u, p.limit_ns};
      mbar_wait_warp(bar(BB_KV), 0, drain, FA2_SITE_LOAD_DRAIN, 0);
      for (int j = (it > 2 ? it - 2 : 0); j < it; ++j) {
        mbar_wait_warp(bar(BB_QFULL + (j & 1)), (j >> 1) & 1, drain, FA2_SITE_LOAD_DRAIN, j);
        mbar_wait_warp(bar(BB_OFULL + j % C::kOStages), (j / C::kOStages) & 1, drain, FA2_SITE_LOAD_DRAIN, j);
      }
    }
  } else if (warp == 10) {
    // ============ dQ reducer: warpgroup 1's staged half, one bulk reduction per tile ============
    if (lane == 0) {
      for (int it = 0; it < n_it; ++it) {
        const int hq = hk * group + it / n_qt;
        const int q0 = (qt_lo + (it % n_qt + kb) % n_qt) * kBlockM;
        const uint32_t sstg = sbase + C::kOffO + (it & 1) * C::kTileBytes;
        if (!mbar_wait(bar(BB_STAGED + (it & 1)), (it >> 1) & 1, g, FA2_SITE_O_RESCALED, it)) break;
#pragma unroll
        for (int bx = 0; bx < D / 64; ++bx)
          tma_reduce_add_4d(&tmDQ, sstg + bx * (kBlockM * 128), D / 2 + 32 * bx, hq, q0, b);
        bulk_commit_group();
        bulk_wait_group_read0();
        mbar_arrive(bar(BB_STGREAD + (it & 1)));
      }
      // every reduction complete before the CTA exits
      bulk_wait_group0();
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------- host side -------------------------------

// 4-D map over the fp32 dQ accumulator [B, Nq, Hq, d] with a (32 x 1 x 128 x
// 1) box and 128-byte swizzle: one box is 128 query rows x 32 columns of one
// head, the unit of the bulk reductions.
static bool encode_dq_acc(CUtensorMap* map, const float* base, int B, int N, int H, int d) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(d) * 4,
                                 static_cast<cuuint64_t>(H) * d * 4,
                                 static_cast<cuuint64_t>(N) * H * d * 4};
  const cuuint32_t box[4] = {32, 1, static_cast<cuuint32_t>(kBlockM), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<float*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
static int launch_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                      const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Nq,
                      int Nk, Window win, float scale, void* workspace, cudaStream_t stream) {
  using C = BCfg<D>;
  static std::once_flag flags[kMaxDevices];
  static int setup_status[kMaxDevices];
  const int st = once_per_device(flags, setup_status, [] {
    return cudaFuncSetAttribute(fa2_bwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                C::kSmemBytes) == cudaSuccess
               ? static_cast<int>(FA2_OK)
               : static_cast<int>(FA2_ERR_LAUNCH);
  });
  if (st != FA2_OK) return st;
  const long long rows = static_cast<long long>(B) * Nq * Hq;
  float* dq_acc = static_cast<float*>(workspace);
  float* lse2 = dq_acc + ((rows * D + 63) / 64) * 64;
  float* delta = lse2 + ((rows + 63) / 64) * 64;
  // D / 8 lanes per row, 256 threads per block
  const long long prep_threads = (rows * (D / 8) + 31) / 32 * 32;
  fa2_bwd_prep_kernel<D><<<static_cast<unsigned>((prep_threads + 255) / 256), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), lse, lse2, delta,
      dq_acc, B, Hq, Nq);
  if (cudaGetLastError() != cudaSuccess) return FA2_ERR_LAUNCH;
  CUtensorMap tq, tk, tv, tdo, tdq;
  if (!encode_bnhd(&tq, q, B, Nq, Hq, D) || !encode_bnhd(&tk, k, B, Nk, Hkv, D) ||
      !encode_bnhd(&tv, v, B, Nk, Hkv, D) || !encode_bnhd(&tdo, dout, B, Nq, Hq, D) ||
      !encode_dq_acc(&tdq, dq_acc, B, Nq, Hq, D))
    return FA2_ERR_LAUNCH;
  BwdParams p;
  p.lse2 = lse2;
  p.delta = delta;
  p.dq_acc = dq_acc;
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Nq = Nq;
  p.Nk = Nk;
  p.wl = win.wl;
  p.wr = win.wr;
  p.scale = scale;
  p.c = scale * 1.4426950408889634f;
  p.limit_ns = 1000000000u;
  const dim3 grid(static_cast<unsigned>((Nk + kBlockN - 1) / kBlockN), Hkv, B);
  fa2_bwd_kernel<D><<<grid, kBwdThreads, C::kSmemBytes, stream>>>(tq, tk, tv, tdo, tdq, p);
  if (cudaGetLastError() != cudaSuccess) return FA2_ERR_LAUNCH;
  const long long n4 = rows * D / 4;
  fa2_bwd_dq_kernel<<<static_cast<unsigned>((n4 + 255) / 256), 256, 0, stream>>>(
      dq_acc, static_cast<__nv_bfloat16*>(dq), n4);
  return cudaGetLastError() == cudaSuccess ? FA2_OK : FA2_ERR_LAUNCH;
}

// Bytes of backward workspace: the fp32 dQ accumulator, then LSE in log2
// units and D per row (each region rounded up to 64 floats).
static long long bwd_workspace_bytes(int B, int Hq, int Nq, int d) {
  const long long rows = static_cast<long long>(B) * Nq * Hq;
  return 4LL * (((rows * d + 63) / 64) * 64 + 2 * ((rows + 63) / 64) * 64);
}
