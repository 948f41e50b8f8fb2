// fa2_forward.cu -- exact attention forward pass for B200 (sm_100a).
//
// A unit of work is 256 query rows of one (batch, query head): two 128-row
// query tiles, Q0 and Q1, that take turns on the tensor cores.  fa2_forward
// runs one CTA per unit over (query block, head, batch) -- the sequence
// parallelism of "FlashAttention 2: Three Places the Chip Was Still Waiting",
// section 2.3 -- so a single long head still fills the machine; with at least
// two units per SM it runs one persistent CTA per SM over a host-made plan of
// whole units (a last, at most half-full wave as single-tile halves);
// fa2_forward_ws runs persistent CTAs over equal ranges of the units' work
// (stream-K) and merges split units in a second kernel, and fa2_forward_auto
// picks between the two; fa2_forward_local narrows each unit to the key tiles
// its sliding window can see.  The backward pass lives in fa2_backward.cuh,
// compiled into this translation unit.
// Within the CTA, work is split by role rather than by data:
//
//   warps 0-3   softmax for Q0, one thread per query row (TMEM lane == row), so
//   warps 4-7   softmax for Q1   row statistics never leave a thread (the
//                                "partition on the index that survives to the
//                                output" rule, section 2.4)
//   warps 8-11  correction: rescales the O accumulator in TMEM when a row's
//               reference max is raised, and the epilogue (the single 1/l
//               division, section 2.2)
//   warp 12     MMA issuer: tcgen05 S = Q K^T and O += P V into TMEM
//   warp 13     TMA producer: Q once, then K_j / V_j through a smem ring
//   warps 14-15 rows of units that see no key at all (O = 0, LSE = -inf)
//
// TMEM columns: S0 | S1 | O0 | O1 (fp32).  P (bf16) is written by the softmax
// threads over the first half of its own S tile and consumed from TMEM by
// the PV MMA, in two halves of 64 keys, each as soon as it is written.  The
// overlap of loads, matrix products and softmax follows the
// producer/consumer idea of "FlashAttention-2 and -3: From Algebra to GPU
// Scheduling", "FlashAttention-3: overlap work on Hopper", rebuilt for
// tcgen05/TMEM.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <queue>
#include <type_traits>
#include <utility>
#include <vector>

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

// Register split (per thread): 2 softmax warpgroups x 192 + correction/epilogue
// 48 + MMA/load warpgroup 80 = 512 = 4 x 128, i.e. exactly the launch pool.
// Each role compiles without spills in its budget.
constexpr int kRegsSoftmax = 192;
constexpr int kRegsCorrection = 48;
constexpr int kRegsOther = 80;
static_assert(2 * kRegsSoftmax + kRegsCorrection + kRegsOther == 4 * kLaunchRegs,
              "register split must equal the launch allocation");

enum Bar {
  BAR_Q = 0,         // Q tiles of the current piece loaded (TMA tx)
  BAR_QFREE = 1,     // the current piece's last S MMA completed: Q smem reusable (MMA commit)
  BAR_S = 2,         // [2] S tile complete (MMA commit)
  BAR_P = 4,         // [2] keys 64-127 of P written to TMEM (128 softmax threads)
  BAR_STATS = 6,     // [2] per-row rescale factor published (128 softmax threads)
  BAR_OFINAL = 8,    // [2] last PV of a piece complete (MMA commit)
  BAR_FSTATS = 10,   // [2] final row max / denominator of a piece published (128 softmax threads)
  BAR_FCONS = 12,    // [2] final statistics read by the epilogue (128 correction threads)
  BAR_DONE = 14,     // all MMAs drained (MMA commit)
  BAR_PH = 15,       // [2] keys 0-63 of P written and O rescaled (128 softmax + 128 correction threads)
  BAR_K0 = 17,       // the first K tile of a piece landed (TMA tx)
  BAR_KV_FULL = 18,  // [stages] a V slot's barrier: V_j and K_{j+1} landed (TMA tx; K slots' are
                     // unused); then [stages] slot free (MMA commit)
};

// Scheduling cost of a unit, in K/V-tile iterations, on top of its
// iterations: the pipeline fill (Q load, first S) and the epilogue a unit
// pays however short it is.  Stream-K cuts the summed costs into equal
// ranges, so SMs that get many short units (the tail of a causal order) get
// fewer iterations.
constexpr int kUnitCost = 2;

// Whether the calls without a workspace run whole units on persistent CTAs
// (when there are at least two per SM) rather than one block per unit.
// Measured on B200 (interleaved CUDA-event runs): causal 8k +1.3 %,
// non-causal 2k +3.7 %, GQA 4k +6 %, 1024-key local window +8 %, results bit
// for bit the same (each unit's arithmetic is unchanged).
#ifndef FA2_PERSISTENT_UNITS
#define FA2_PERSISTENT_UNITS 1
#endif
constexpr bool kPersistentUnits = FA2_PERSISTENT_UNITS != 0;

// Lazy rescaling: a row's exponentials and its O accumulator are taken
// relative to a reference max that is raised to the running max only when the
// running max exceeds it by more than this many log2 units (a factor of 256).
// O and the denominator l always share the reference, so the result is the
// same in exact arithmetic; every probability stays <= 2^8 and l <= 2^8 Nk,
// far inside fp32.  On random data the reference settles after the first tile
// and O is almost never touched again ("FlashAttention 2: Three Places the Chip
// Was Still Waiting", section 2.2: the correction factor is what remains in
// the loop once the division has moved out of it).
constexpr float kRescaleThreshold = 8.f;

// Persistent whole units: the host plans which CTA runs which unit and in
// what order, and passes the plan as a kernel parameter (no device memory).
// Up to kMaxTableUnits units on up to kMaxTableCtas CTAs; larger problems
// deal units round robin instead.
constexpr int kMaxTableCtas = 160;
constexpr int kMaxTableUnits = 8192;
// An entry is a unit index u = round * B * Hq + (b * Hq + hq), or -- with
// kHalfTile0 / kHalfTile1 added -- only that unit's first or second 128-row
// query tile (a half unit: the two halves of a unit may run on two CTAs).
constexpr int kUnitBits = 13;
constexpr int kHalfTile0 = 1 << kUnitBits, kHalfTile1 = 2 << kUnitBits;
static_assert(kMaxTableUnits <= (1 << kUnitBits), "unit index bits");
struct UnitTable {
  uint16_t start[kMaxTableCtas + 1];  // CTA c runs unit[start[c] .. start[c+1]) in that order
  uint16_t unit[kMaxTableUnits];      // entries as above
};
struct NoTable {};

// The split units of a stream-K launch, one entry per unit, as the host
// found them from the range boundaries: the partial buffer of its first piece
// (slot = first cut - 1; piece q is in slot + q), its number of pieces, and
// its coordinates.  The combine kernel runs one block row per entry.
struct CutList {
  int n;
  uint16_t slot[kMaxTableCtas];
  uint16_t np[kMaxTableCtas];
  uint16_t qb[kMaxTableCtas];
  int bh[kMaxTableCtas];  // b * Hq + hq
};

// Warps 14-15 (otherwise idle) write the rows of units with no visible key.
constexpr int kEmptyThreads = 64;

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
  static constexpr int kOffLR = kOffL + kTiles * kBlockM * 4;
  static constexpr int kNumBars = BAR_KV_FULL + 2 * kStages;
  static constexpr int kOffBar = kOffLR + kTiles * kBlockM * 4;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kUsed = kOffMisc + 16;
  static constexpr int kSmemBytes = kUsed + 1024;  // slack for 1024-byte alignment
  // TMEM column of S_t (P_t reuses its first half) and of O_t
  __host__ __device__ static constexpr uint32_t col_s(int t) { return t ? 128u : 0u; }
  __host__ __device__ static constexpr uint32_t col_o(int t) { return 256u + (t ? D : 0); }
  // floats of one stream-K partial: O as [2 tiles][D/16 chunks][128 rows][16],
  // then m [2][128], l [2][128] and the rounding term lr [2][128]
  static constexpr int kPieceFloats = kTiles * kBlockM * (D + 3);
  __host__ __device__ static constexpr int part_o(int t, int ch, int row) {
    return ((t * (D / 16) + ch) * kBlockM + row) * 16;
  }
  __host__ __device__ static constexpr int part_m(int t, int row) { return kTiles * kBlockM * D + t * kBlockM + row; }
  __host__ __device__ static constexpr int part_l(int t, int row) { return part_m(t, row) + kTiles * kBlockM; }
  __host__ __device__ static constexpr int part_lr(int t, int row) { return part_l(t, row) + kTiles * kBlockM; }
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(256 + 2 * D <= (int)kTmemCols, "TMEM budget");
};

struct Params {
  __nv_bfloat16* o;
  float* lse;
  int B, Hq, Hkv, Nq, Nk;
  int wl, wr;         // visibility window widths (see Window); causal is (-1, 0)
  int n_qblk;
  int r_empty;        // first round (heaviest first) of units with no visible key; n_qblk if none
  float c;            // |softmax_scale| * log2(e)
  int negate;         // softmax_scale < 0: compute S = -(Q K^T) so c stays >= 0
  uint32_t limit_ns;  // per bounded wait
  // work decomposition
  int streamk;        // 0: CTA i runs unit i whole; 1: CTA c runs cost positions [c*T/G, (c+1)*T/G)
  int pu;             // with the persistent kernel: whole units (no splits), from the plan when tab is set,
                      // else dealt round robin
  int tab;            // the persistent kernel's unit plan is valid
  int T;              // summed unit costs, kUnitCost + iterations per unit (< 2^31, checked on the host)
  int span;           // T / G
  int rem;            // T % G
  int G;              // CTAs of a stream-K launch
  float* ws;          // stream-K partials: [G CTAs][2: first / last piece of its range][piece floats]
};

// Visibility: key j is visible to query row i when g - wl <= j <= g + wr
// with g = i + Nk - Nq, the row's diagonal key (bottom-right alignment); a
// negative width leaves that side open.  Causal attention is (-1, 0), full
// attention (-1, -1), and a sliding (local) window ("FlashAttention-2"
// explainer, "The Downstream Story") bounds the left side too.
struct Window {
  int wl, wr;
};

// K/V tiles a 128-row query tile starting at row r0 can see: [lo, lo + count)
// (count 0 when no row of it sees any key).
// (32-bit arithmetic: the host keeps 2 (Nq + Nk) below 2^31 and clamps the
// widths below Nk / Nq.)
__host__ __device__ inline int tile_span(int Nq, int Nk, Window w, int r0, int& lo) {
  lo = 0;
  if (r0 >= Nq) return 0;
  const int koff = Nk - Nq;
  const int rl = (r0 + kBlockM - 1 < Nq - 1) ? r0 + kBlockM - 1 : Nq - 1;
  int first = (w.wl >= 0) ? r0 + koff - w.wl : 0;      // left bound of the first row
  int last = (w.wr >= 0) ? rl + koff + w.wr : Nk - 1;  // right bound of the last row
  if (first < 0) first = 0;
  if (last > Nk - 1) last = Nk - 1;
  if (first > last) return 0;
  lo = first / kBlockN;
  return last / kBlockN - lo + 1;
}

// A unit's K/V range: it starts at tile j0, the first tile either of its two
// query tiles sees, and query tile t needs its first n0 / n1 tiles.  A query
// tile whose window starts later meets fully masked tiles first; they cost an
// iteration and contribute nothing.
struct UnitSpan {
  int j0, n0, n1;
};
__host__ __device__ inline UnitSpan unit_span(int Nq, int Nk, Window w, int qb) {
  int lo0 = 0, lo1 = 0;
  const int c0 = tile_span(Nq, Nk, w, qb * kRowsPerCta, lo0);
  const int c1 = tile_span(Nq, Nk, w, qb * kRowsPerCta + kBlockM, lo1);
  UnitSpan u{0, 0, 0};
  if (c0 == 0 && c1 == 0) return u;
  u.j0 = (c0 > 0 && c1 > 0) ? (lo0 < lo1 ? lo0 : lo1) : (c0 > 0 ? lo0 : lo1);
  u.n0 = c0 > 0 ? lo0 + c0 - u.j0 : 0;
  u.n1 = c1 > 0 ? lo1 + c1 - u.j0 : 0;
  return u;
}

// K/V-tile iterations of a unit (query block qb).
__host__ __device__ inline int unit_tiles(int Nq, int Nk, Window w, int qb) {
  const UnitSpan u = unit_span(Nq, Nk, w, qb);
  return u.n0 > u.n1 ? u.n0 : u.n1;
}

__host__ __device__ inline Window window_of(const Params& p) { return Window{p.wl, p.wr}; }
inline Window causal_window(int causal) { return Window{-1, causal ? 0 : -1}; }

// Start of CTA c's iteration range, floor(c * T / G), in 32-bit arithmetic:
// c*T/G = c*span + c*rem/G with T = span*G + rem, c*span <= T < 2^31 and
// c*rem < G*G.
__host__ __device__ inline int range_start(int span, int rem, int G, int c) {
  return c * span + (c * rem) / G;
}

// ---------------------------------------------------------------------------
// Work decomposition, evaluated identically by every role of a CTA.
//
// Units are (256-row query block, query head, batch) in heaviest-first order:
// round r holds the B*Hq units of query block n_qblk-1-r, (batch, head)
// fastest; all units of a round need the same number of K/V tiles.  A piece
// is a contiguous range [jb, je) of one unit's K/V tiles run by one CTA.
//
// Stream-K: the iterations of all units, concatenated in that order, are cut
// into G equal ranges, one per CTA, so every SM gets the same number of
// K/V-tile iterations (no wave quantisation, no long-unit tail).  A unit cut
// by a range boundary is split; its pieces are merged through the workspace.
// ---------------------------------------------------------------------------
struct Piece {
  int b, hq, qb;
  int j0;           // first K/V tile of the unit (absolute); iterations count from it
  int jb, je;       // K/V tiles [jb, je) of the unit
  int nt0, nt1;     // K/V tiles of Q0 / Q1 over the whole unit
  int a0, a1;       // iterations of Q0 / Q1 in this piece
  int own;          // query tiles whose outputs this piece writes (bit t; a half unit owns one)
  int split;        // the unit is shared with other pieces
  int slot;         // CTA that runs the unit's first piece (the partial buffers count from it)
  int npieces;      // pieces of the unit
  int index;        // this piece's position in the unit
};

// Smallest c in [1, G] with B_c > y (G when no boundary lies above y): binary
// search over the CTAs' range starts.
__device__ __forceinline__ int first_boundary_above(const Params& p, int y) {
  int lo = 1, hi = p.G;  // answer in [lo, hi]
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (range_start(p.span, p.rem, p.G, mid) > y) hi = mid; else lo = mid + 1;
  }
  return lo;
}

// Cost positions: round r's units are laid out one after another, unit k of
// round r at [cum_r + k*w_r, cum_r + (k+1)*w_r) with w_r = kUnitCost + n_r
// (0 for a round of empty units); iteration j of the unit sits at position
// cum_r + k*w_r + kUnitCost + j.  CTA c runs the iterations whose positions
// fall in [B_c, B_{c+1}), B_c = floor(c*T/G).
//
// Order of a CTA's pieces: when its range ends inside a unit that continues
// on the next CTA, that piece (the unit's head) runs first and the rest in
// order.  The next CTA starts with the same unit's tail, so both pieces of a
// split unit finish early and its merge overlaps the remaining work instead
// of landing at the end of the kernel.
template <bool SK>  // SK: stream-K ranges; otherwise CTA u runs unit u whole
struct PieceIter {
  int HB, r, n, k_cur;
  int cum, x, x_end;  // cost before round r; the natural walk's range [x, x_end)
  int state;          // unit mode: 1 = unit pending; stream-K: 1 = head piece pending

  __device__ __forceinline__ static int cost(int n) { return n > 0 ? n + kUnitCost : 0; }

  __device__ __forceinline__ void fill(const Params& p, Piece& pc, int r_, int k, int jb, int je) const {
    pc.qb = p.n_qblk - 1 - r_;
    pc.b = k / p.Hq;
    pc.hq = k % p.Hq;
    pc.jb = jb;
    pc.je = je;
    const UnitSpan u = unit_span(p.Nq, p.Nk, window_of(p), pc.qb);
    pc.j0 = u.j0;
    pc.nt0 = u.n0;
    pc.nt1 = u.n1;
    pc.a0 = max(0, min(je, pc.nt0) - jb);
    pc.a1 = max(0, min(je, pc.nt1) - jb);
    pc.own = 3;
  }

  // (batch, head, query block) of the current piece, recomputed from the
  // iterator so a role need not keep them live through its inner loop.
  __device__ __forceinline__ void coords(const Params& p, Piece& pc) const {
    pc.qb = p.n_qblk - 1 - r;
    pc.b = k_cur / p.Hq;
    pc.hq = k_cur % p.Hq;
  }

  // Which pieces share the current piece's unit: the range boundaries B_c
  // (c = 1..G-1) that fall strictly inside the unit's iteration positions.
  __device__ __forceinline__ void split_info(const Params& p, Piece& pc) const {
    pc.split = 0;
    pc.slot = 0;
    pc.npieces = 1;
    pc.index = 0;
    if constexpr (!SK) return;
    if (p.pu) return;
    const int s_u = cum + k_cur * cost(n) + kUnitCost;                // position of iteration 0
    const int c_first = first_boundary_above(p, s_u);                // B_c > s_u
    const int c_last = first_boundary_above(p, s_u + n - 1) - 1;     // B_c <= s_u + n - 1
    if (c_last >= c_first) {
      pc.split = 1;
      pc.npieces = c_last - c_first + 2;
      pc.slot = c_first - 1;
      // pieces start at iteration 0 and at each inside boundary
      const int ci = first_boundary_above(p, s_u + pc.jb) - 1;  // last boundary <= s_u + jb
      pc.index = (ci < c_first) ? 0 : min(ci, c_last) - c_first + 1;
    }
  }

  // Round state (r, cum, n) of the round holding cost position `pos`.
  __device__ __forceinline__ void seek_round(const Params& p, int pos) {
    r = 0;
    cum = 0;
    n = unit_tiles(p.Nq, p.Nk, window_of(p), p.n_qblk - 1);
    while (pos >= cum + HB * cost(n)) {  // the end of a round is at most T < 2^31
      cum += HB * cost(n);
      ++r;
      n = unit_tiles(p.Nq, p.Nk, window_of(p), p.n_qblk - 1 - r);
    }
  }

  __device__ __forceinline__ void init(const Params& p) {
    HB = p.B * p.Hq;
    r = cum = n = k_cur = 0;
    x = x_end = 0;
    state = 1;
    if constexpr (!SK) return;
    if (p.pu) {  // x counts this CTA's waves of whole units
      state = 0;
      return;
    }
    x = range_start(p.span, p.rem, p.G, blockIdx.x);
    x_end = range_start(p.span, p.rem, p.G, blockIdx.x + 1);
    state = 0;
    if (x_end <= x) return;
    // the unit holding the range's last position, and whether it continues
    // past the range while the range also holds earlier units
    seek_round(p, x_end - 1);
    const int w = cost(n);
    const int k = (x_end - 1 - cum) / w;
    const int s_u = cum + k * w;
    if (s_u > x && x_end - 1 >= s_u + kUnitCost && x_end < s_u + w) {
      state = 1;
      k_cur = k;
      x_end = s_u;  // the natural walk stops where the head piece begins
    }
  }

  // plan: the persistent launch's unit plan (read when p.tab is set)
  __device__ __forceinline__ bool next(const Params& p, Piece& pc, const UnitTable* plan = nullptr) {
    if constexpr (!SK) {
      if (!state) return false;
      state = 0;
      const int u = blockIdx.x;
      r = u / HB;
      k_cur = u % HB;
      const int nn = unit_tiles(p.Nq, p.Nk, window_of(p), p.n_qblk - 1 - r);
      if (nn == 0) return false;  // nothing to compute: warps 14-15 write this unit's empty rows
      cum = 0;
      n = nn;
      fill(p, pc, r, k_cur, 0, nn);
      return true;
    }
    if (p.pu) {
      // Whole units dealt to the G CTAs wave by wave, in heaviest-first order,
      // alternating direction (wave w gives CTA c unit wG + c, or wG + G-1-c
      // when w is odd) so each CTA's heavy and light units pair up.
      const int u_count = p.r_empty * HB;  // units with some visible key
      const int c = static_cast<int>(blockIdx.x);
      int u, half = 0;
      if (p.tab) {
        const int i = plan->start[c] + x;
        if (i >= plan->start[c + 1]) return false;
        u = plan->unit[i] & ((1 << kUnitBits) - 1);
        half = plan->unit[i] >> kUnitBits;
      } else {
        u = x * p.G + ((x & 1) ? p.G - 1 - c : c);
      }
      ++x;
      if (u >= u_count) return false;
      r = u / HB;
      k_cur = u % HB;
      cum = 0;
      n = unit_tiles(p.Nq, p.Nk, window_of(p), p.n_qblk - 1 - r);
      fill(p, pc, r, k_cur, 0, n);
      // a half unit walks only its query tile's prefix of the unit's K/V
      // range (every K/V item the piece loads must be used, which frees it)
      if (half == 1) {  // first query tile only: the second is another CTA's
        pc.a1 = 0;
        pc.je = pc.jb + pc.a0;
        pc.own = 1;
      } else if (half == 2) {
        pc.a0 = 0;
        pc.je = pc.jb + pc.a1;
        pc.own = 2;
      }
      return true;
    }
    if (state) {  // the head piece: iterations [0, B_{c+1} - position of iteration 0)
      state = 0;
      const int end = range_start(p.span, p.rem, p.G, blockIdx.x + 1);
      fill(p, pc, r, k_cur, 0, end - (cum + k_cur * cost(n) + kUnitCost));
      return true;
    }
    if (x >= x_end) return false;
    if (x < cum) {
      seek_round(p, x);  // first piece after the head piece
    } else {
      while (x >= cum + HB * cost(n)) {
        cum += HB * cost(n);
        ++r;
        n = unit_tiles(p.Nq, p.Nk, window_of(p), p.n_qblk - 1 - r);
      }
    }
    const int w = cost(n);
    const int k = (x - cum) / w;
    const int base = cum + k * w + kUnitCost;  // position of iteration 0 of unit k
    const int jb = max(0, x - base), je = min(n, x_end - base);
    if (je <= jb) {  // the range ends inside this unit's fixed cost: no iteration left
      x = x_end;
      return false;
    }
    k_cur = k;
    fill(p, pc, r, k, jb, je);
    x = base + je;
    return true;
  }
};

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
// the FMA pipe.  Measured on B200 with the final kernel (interleaved runs,
// 2 of 16 pairs): within +-1 % on causal 8k, non-causal 2k, GQA 4k and long
// 32k, because the exponentials are not what bounds the per-tile chain (a
// timing probe without any exponential is only ~5 % faster); the default is
// 0.  Built and checked against the oracle with 2 pairs by the GPU tests.
#ifndef FA2_EMU_PAIRS
#define FA2_EMU_PAIRS 0
#endif
constexpr int kEmuPairs = FA2_EMU_PAIRS;

template <int D, bool SK>
__global__ void __launch_bounds__(kThreads, 1)
    fa2_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const Params p,
                   const __grid_constant__ std::conditional_t<SK, UnitTable, NoTable> plan) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_addr(smem);
  float* sm_alpha = reinterpret_cast<float*>(smem + C::kOffAlpha);
  float* sm_m = reinterpret_cast<float*>(smem + C::kOffM);
  float* sm_l = reinterpret_cast<float*>(smem + C::kOffL);
  float* sm_lr = reinterpret_cast<float*>(smem + C::kOffLR);
  const uint32_t bar0 = sbase + C::kOffBar;
  auto bar = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int koff = p.Nk - p.Nq;  // causal diagonal offset

  // ---- setup ----
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int i = 0; i < BAR_KV_FULL; ++i) {
      uint32_t cnt = 1;
      if ((i >= BAR_STATS && i < BAR_STATS + 2) || (i >= BAR_FSTATS && i < BAR_FSTATS + 2) ||
          (i >= BAR_FCONS && i < BAR_FCONS + 2) || (i >= BAR_P && i < BAR_P + 2))
        cnt = kBlockM;
      if (i >= BAR_PH && i < BAR_PH + 2) cnt = 2 * kBlockM;
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
  const WaitGuard g{smem_addr(const_cast<int*>(abort_flag)), p.limit_ns};
  const UnitTable* unit_plan = nullptr;  // the host's plan of whole units (read when p.tab is set)
  if constexpr (SK) unit_plan = &plan;
  const bool aligned_ok = (sbase & 1023u) == 0;  // always true by construction

  // Each warpgroup executes one register-split instruction (one site per
  // warpgroup) that directly dominates its role's code; every role then walks
  // the same sequence of pieces with its own iterator.
  if (warp < 8) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    PieceIter<SK> pit;
    pit.init(p);
    Piece pc;
    // =================== softmax: one thread per query row ===================
    const int t = warp >> 2;
    const int q4 = warp & 3;
    const int rt = q4 * 32 + lane;  // row within the tile == TMEM lane
    const uint32_t tS = tmem + (static_cast<uint32_t>(q4 * 32) << 16) + C::col_s(t);
    const float c = p.c;
    uint32_t s_cnt = 0;      // S_t completions consumed so far (all pieces)
    uint32_t piece_cnt = 0;  // pieces finished
    bool ok = true;
    while (ok && pit.next(p, pc, unit_plan)) {
      const int ntt = t ? pc.a1 : pc.a0;
      const int r0t = pc.qb * kRowsPerCta + t * kBlockM;
      const int row = r0t + rt;
      float m_raw = -INFINITY;  // reference max of the raw scores (-inf while no key was visible)
      float m_sc = 0.f;         // m_raw * c (0 while no key was visible)
      float l = 0.f;            // running denominator, relative to m_sc
      float lr = 0.f;           // bf16 rounding of each tile's largest probability, summed like l
      // this row's visible keys [lo_abs, hi_abs]; tiles j >= j_hi cross some
      // row's right bound or the key tail, tiles j < j_lo some row's left bound
      // (ints: the host keeps Nq + Nk below 2^30 and each window below N)
      const int hi_abs = (p.wr >= 0) ? min(row + koff + p.wr, p.Nk - 1) : p.Nk - 1;
      const int lo_abs = (p.wl >= 0) ? row + koff - p.wl : 0;
      const int j_hi = (((p.wr >= 0) ? min(r0t + koff + p.wr, p.Nk - 1) : p.Nk - 1) + 1) / kBlockN;
      const int j_lo = (p.wl >= 0) ? (r0t + kBlockM - 1 + koff - p.wl + kBlockN - 1) / kBlockN : 0;
      for (int jj = 0; jj < ntt; ++jj) {
        const int j = pc.j0 + pc.jb + jj;  // K/V tile (absolute)
        if (!mbar_wait_warp(bar(BAR_S + t), s_cnt & 1, g, FA2_SITE_S_READY, j)) {
          ok = false;
          break;
        }
        ++s_cnt;
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
        // window edges (the causal diagonal) and the ragged key tail: only
        // tiles some row's bound falls into pay for masking
        const int kbase = j * kBlockN;
        const bool masked = j >= j_hi || j < j_lo;
        if (masked) {
          // visible columns [lo_i, hi_i] of this tile for this row
          const int hi_i = max(min(hi_abs - kbase, kBlockN - 1), -1);
          const int lo_i = min(lo_abs - kbase, kBlockN);
          // one 32-bit visibility mask per 32 columns: a compact test, so the
          // code unmasked tiles branch around stays small
#pragma unroll
          for (int k = 0; k < kBlockN / 32; ++k) {
            const int lk = max(lo_i - 32 * k, 0), hk = min(hi_i - 32 * k, 31);
            uint32_t vk = 0u;
            if (hk >= lk) vk = (0xffffffffu >> (31 - hk)) & (0xffffffffu << lk);
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (!((vk >> i) & 1u)) s[32 * k + i] = -INFINITY;
          }
        }
        // row max: 8 independent chains of 3-input max (max is exact in any order)
        float mp[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mp[k] = fmaxf(s[2 * k], s[2 * k + 1]);
#pragma unroll
        for (int i = 16; i < kBlockN; i += 16)
#pragma unroll
          for (int k = 0; k < 8; ++k) mp[k] = fmax3(mp[k], s[i + 2 * k], s[i + 2 * k + 1]);
        const float tmx = fmax3(fmax3(mp[0], mp[1], mp[2]), fmax3(mp[3], mp[4], mp[5]), fmaxf(mp[6], mp[7]));
        const float mx = fmaxf(tmx, m_raw);
        // New reference: the running max, taken when nothing was visible yet or
        // when it exceeds the current reference by more than the threshold;
        // otherwise the reference stays and the rescale factor is exactly 1 (O
        // is left untouched).  alpha is 0 when nothing was visible yet.
        float m_ref = m_raw, m_sc_new = m_sc, alpha = 1.f;
        if (m_raw == -INFINITY) {
          if (mx != -INFINITY) {
            m_ref = mx;
            m_sc_new = mx * c;
            alpha = 0.f;
          }
        } else if (mx * c - m_sc > kRescaleThreshold) {
          m_ref = mx;
          m_sc_new = mx * c;
          alpha = ex2_approx(m_sc - m_sc_new);
        }
        if (jj > 0) {
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
            if (k == 1) {
              // keys 0-63 of P are in TMEM: the first half of the PV product
              // can start while the second half is computed
              tmem_wait_st();
              tc_fence_before();
              mbar_arrive(bar(BAR_PH + t));
            }
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
        {
          // the tile's largest probability as the PV product saw it (bf16) minus
          // its fp32 value, computed with the same fused multiply-add and exp2
          const float pm = (tmx == -INFINITY) ? 0.f : ex2_approx(fmaf(tmx, c, -m_sc_new));
          const float rm = __uint_as_float(pack_bf16x2(pm, 0.f) << 16);
          lr = lr * alpha + (rm - pm);
        }
        m_raw = m_ref;
        m_sc = m_sc_new;
      }
      if (!ok) break;
      // final statistics of this piece; the previous piece's must have been read
      if (piece_cnt > 0 &&
          !mbar_wait_warp(bar(BAR_FCONS + t), (piece_cnt - 1) & 1, g, FA2_SITE_FINAL_STATS, piece_cnt)) {
        ok = false;
        break;
      }
      sm_m[t * kBlockM + rt] = (m_raw == -INFINITY) ? -INFINITY : m_sc;
      sm_l[t * kBlockM + rt] = l;
      sm_lr[t * kBlockM + rt] = lr;
      mbar_arrive(bar(BAR_FSTATS + t));
      ++piece_cnt;
    }
  } else if (warp < 12) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsCorrection));
    PieceIter<SK> pit;
    pit.init(p);
    Piece pc;
    // ============== correction (O rescale) and epilogue warps ==============
    const int q4 = warp & 3;
    const int rt = q4 * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    // parities of the phases consumed so far: bit t = STATS_t, bit 2 + t =
    // OFINAL_t, bit 4 = FSTATS (one per piece)
    uint32_t ph = 0;
    bool ok = true;

    while (ok && pit.next(p, pc, unit_plan)) {
      const int n_p = pc.je - pc.jb;
      for (int jj = 0; jj < n_p && ok; ++jj) {
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (jj >= (t ? pc.a1 : pc.a0)) continue;
          if (jj == 0) {  // nothing accumulated yet: O_t (read by the last epilogue) is free
            tc_fence_before();
            mbar_arrive(bar(BAR_PH + t));
            continue;
          }
          if (!mbar_wait_warp(bar(BAR_STATS + t), (ph >> t) & 1, g, FA2_SITE_STATS_READY, pc.jb + jj)) {
            ok = false;
            break;
          }
          ph ^= 1u << t;
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
          mbar_arrive(bar(BAR_PH + t));
        }
      }
      if (!ok) break;
      pit.coords(p, pc);
      pit.split_info(p, pc);

      // ---- epilogue of the piece, tile by tile: a whole unit is normalised
      // and stored; a piece of a split unit publishes its partial instead ----
      float* part = nullptr;
      if (pc.split)
        part = p.ws + static_cast<size_t>(2 * (pc.slot + pc.index) + (pc.index == 0 ? 1 : 0)) *
                          C::kPieceFloats;
#pragma unroll 1
      for (int t = 0; t < 2; ++t) {
        const bool have = (t ? pc.a1 : pc.a0) > 0;  // warp-uniform: tcgen05.ld needs the whole warp
        if (have) {
          if (!mbar_wait_warp(bar(BAR_OFINAL + t), (ph >> (2 + t)) & 1, g, FA2_SITE_O_FINAL, t)) {
            ok = false;
            break;
          }
          ph ^= 4u << t;
        }
        if (!mbar_wait_warp(bar(BAR_FSTATS + t), (ph >> 4) & 1, g, FA2_SITE_FINAL_STATS, t)) {
          ok = false;
          break;
        }
        const float m_sc = sm_m[t * kBlockM + rt];
        const float l = sm_l[t * kBlockM + rt];
        const float lr = sm_lr[t * kBlockM + rt];
        mbar_arrive(bar(BAR_FCONS + t));
        tc_fence_after();
        const uint32_t tO = tmem + lane_off + C::col_o(t);
        if (!((pc.own >> t) & 1)) {
          // the other half of a split-in-two unit writes this query tile
        } else if (!pc.split) {
          // single division per row, bf16 O, LSE = ln(sum exp(scale * s))
          const int row = pc.qb * kRowsPerCta + t * kBlockM + rt;
          const bool valid = row < p.Nq;
          float inv_l = 0.f, lse = -INFINITY;
          if (l > 0.f) {
            inv_l = 1.f / (l + lr);
            lse = (m_sc + log2f(l)) * 0.69314718055994530942f;
          }
          __nv_bfloat16* orow = p.o + ((static_cast<size_t>(pc.b) * p.Nq + row) * p.Hq + pc.hq) * D;
#pragma unroll 1
          for (int ch = 0; ch < D / 16; ++ch) {
            uint32_t r[16];
            if (have) {
              tmem_ld16(tO + 16 * ch, r);
              tmem_wait_ld();
            } else {
#pragma unroll
              for (int i = 0; i < 16; ++i) r[i] = 0u;
            }
            uint4 w0, w1;
            w0.x = pack_bf16x2(__uint_as_float(r[0]) * inv_l, __uint_as_float(r[1]) * inv_l);
            w0.y = pack_bf16x2(__uint_as_float(r[2]) * inv_l, __uint_as_float(r[3]) * inv_l);
            w0.z = pack_bf16x2(__uint_as_float(r[4]) * inv_l, __uint_as_float(r[5]) * inv_l);
            w0.w = pack_bf16x2(__uint_as_float(r[6]) * inv_l, __uint_as_float(r[7]) * inv_l);
            w1.x = pack_bf16x2(__uint_as_float(r[8]) * inv_l, __uint_as_float(r[9]) * inv_l);
            w1.y = pack_bf16x2(__uint_as_float(r[10]) * inv_l, __uint_as_float(r[11]) * inv_l);
            w1.z = pack_bf16x2(__uint_as_float(r[12]) * inv_l, __uint_as_float(r[13]) * inv_l);
            w1.w = pack_bf16x2(__uint_as_float(r[14]) * inv_l, __uint_as_float(r[15]) * inv_l);
            if (valid) {
              uint4* dst = reinterpret_cast<uint4*>(orow + 16 * ch);
              dst[0] = w0;
              dst[1] = w1;
            }
          }
          if (valid) p.lse[(static_cast<size_t>(pc.b) * p.Hq + pc.hq) * p.Nq + row] = lse;
        } else {
          // partial: O unnormalised (fp32), in 16-column chunks of 128 rows so
          // a warp's store covers 32 consecutive rows (2 KiB contiguous)
          if (have) {
#pragma unroll 1
            for (int ch = 0; ch < D / 16; ++ch) {
              uint32_t r[16];
              tmem_ld16(tO + 16 * ch, r);
              tmem_wait_ld();
              float4* dst = reinterpret_cast<float4*>(part + C::part_o(t, ch, rt));
#pragma unroll
              for (int i = 0; i < 4; ++i)
                __stcg(dst + i, make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                            __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3])));
            }
          }
          __stcg(part + C::part_m(t, rt), m_sc);
          __stcg(part + C::part_l(t, rt), have ? l : 0.f);
          __stcg(part + C::part_lr(t, rt), have ? lr : 0.f);
        }
      }
      if (!ok) break;
      ph ^= 16u;
    }
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsOther));
    PieceIter<SK> pit;
    pit.init(p);
    Piece pc;
   if (warp == 12) {
    // ============================ MMA issuer warp ============================
    // The whole warp follows the schedule (warp-uniform waits and descriptor
    // arithmetic); one elected lane -- always the same one in a converged warp,
    // so its commits cover its own MMAs -- issues each group of tcgen05
    // instructions (MMAs and their commits) inside a single elected block.
    // Measured on B200: a group issued this way takes ~23 cycles per MMA and
    // runs ahead of the tensor core, while a per-MMA elect/warp-sync costs
    // 50-60 cycles each and a single divergent lane is slower still when the
    // softmax warps sharing this SM sub-partition keep the issue slots busy.
    if (aligned_ok) {
      const uint32_t idS = idesc_bf16_f32(kBlockM, kBlockN, false, p.negate != 0);
      const uint32_t idPV = idesc_bf16_f32(kBlockM, D, true, false);
      const uint32_t sQ = sbase + C::kOffQ;
      const uint32_t sKV = sbase + C::kOffKV;
      auto stage_of = [&](uint32_t it) { return static_cast<int>(it % C::kStages); };
      auto phase_of = [&](uint32_t it) { return (it / C::kStages) & 1u; };
      auto free_of = [&](uint32_t it) { return bar(BAR_KV_FULL + C::kStages + stage_of(it)); };
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
      // S_t = Q_t K^T with the K tile of ring item itK, then commits
      auto issue_s = [&](int t, uint32_t itK, uint32_t c1, uint32_t c2, uint32_t c3) {
        const uint32_t dS = tmem + C::col_s(t);
        const uint64_t a0 = dQ + ((t * C::kTileBytes) >> 4);
        const uint64_t bK = dK + ((stage_of(itK) * C::kTileBytes) >> 4);
        if (elect_one()) {
          // K advances 32 bytes inside a 128-byte swizzle atom, then jumps to
          // the next 64-column chunk.  (The empty asm makes the per-MMA
          // descriptors opaque, so the compiler derives them here instead of
          // keeping all of them live across the whole schedule.)
          uint64_t da = a0, db = bK;
          asm volatile("" : "+l"(da), "+l"(db));
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            umma_ss(dS, da, db, idS, kk > 0 ? 1u : 0u);
            const uint32_t step = ((kk & 3) == 3) ? (kChunkBytes - 3 * 32) >> 4 : 32 >> 4;
            da += step;
            db += step;
          }
          if (c1) umma_commit(c1);
          if (c2) umma_commit(c2);
          if (c3) umma_commit(c3);
        }
        __syncwarp();
      };
      // O_t (+)= P_t V over keys [16 k0, 16 k1) of the V tile of ring item itV, then commits
      auto issue_pv = [&](int t, uint32_t itV, bool acc, int k0, int k1, uint32_t c1, uint32_t c2) {
        const uint32_t dS = tmem + C::col_s(t), dO = tmem + C::col_o(t);
        const uint64_t bV = dV + ((stage_of(itV) * C::kTileBytes) >> 4);
        if (elect_one()) {
          uint64_t db = bV + static_cast<uint32_t>(k0) * ((16 * kSwizzleBytes) >> 4);
          asm volatile("" : "+l"(db));
#pragma unroll
          for (int kk = k0; kk < k1; ++kk) {
            umma_ts(dO, dS + kk * 8, db, idPV, (acc || kk > 0) ? 1u : 0u);
            db += (16 * kSwizzleBytes) >> 4;  // next 16 keys
          }
          if (c1) umma_commit(c1);
          if (c2) umma_commit(c2);
        }
        __syncwarp();
      };
      uint32_t itb = 0;           // ring item of the current piece's first K tile
      uint32_t q_cnt = 0;         // pieces whose Q was waited for
      uint32_t p_cnt[2] = {0, 0}; // P_t phases consumed
      bool ok = true;
      while (ok && pit.next(p, pc, unit_plan)) {
        const int n_p = pc.je - pc.jb;
        const int a0 = pc.a0, a1 = pc.a1;
        if (!mbar_wait_warp(bar(BAR_Q), q_cnt & 1, g, FA2_SITE_Q_LOADED, q_cnt)) break;
        ++q_cnt;
        auto itK = [&](int jj) { return itb + 2u * static_cast<uint32_t>(jj); };
        auto itV = [&](int jj) { return itb + 2u * static_cast<uint32_t>(jj) + 1u; };
        // S_t of the piece's first K/V tile; K is free after the last S on it
        if (!mbar_wait_warp(bar(BAR_K0), (q_cnt - 1) & 1, g, FA2_SITE_KV_LOADED, pc.jb)) break;
        tc_fence_after();
        // (one piece per CTA in unit mode: the Q buffer is never reloaded)
        const uint32_t qfree0 = (SK && n_p == 1) ? bar(BAR_QFREE) : 0u;
        if (a0 > 0) issue_s(0, itK(0), bar(BAR_S + 0), a1 > 0 ? 0u : free_of(itK(0)), a1 > 0 ? 0u : qfree0);
        if (a1 > 0) issue_s(1, itK(0), bar(BAR_S + 1), free_of(itK(0)), qfree0);
        for (int jj = 0; jj < n_p && ok; ++jj) {
          // operands of this step, V_j and K_{j+1}, behind one barrier (V_j's);
          // checked while the tensor pipe still holds the previous block
          if (!mbar_wait_warp(bar(BAR_KV_FULL + stage_of(itV(jj))), phase_of(itV(jj)), g,
                              FA2_SITE_KV_LOADED, pc.jb + jj))
            break;
          // the last S of the piece frees the Q buffer for the next piece
          const uint32_t qfree = (SK && jj + 2 == n_p) ? bar(BAR_QFREE) : 0u;
          // tile 0: PV0(j) and S0(j+1); V_j / K_{j+1} are freed here when tile 1 has no use for them
          if (jj < a0) {
            // keys 0-63 as soon as their P is written and O_0 is rescaled, then the rest
            if (!mbar_wait_warp(bar(BAR_PH + 0), p_cnt[0] & 1, g, FA2_SITE_O_RESCALED, pc.jb + jj)) break;
            tc_fence_after();
            issue_pv(0, itV(jj), jj > 0, 0, kBlockN / 32, 0u, 0u);
            if (!mbar_wait_warp(bar(BAR_P + 0), p_cnt[0] & 1, g, FA2_SITE_P_READY, pc.jb + jj)) break;
            ++p_cnt[0];
            tc_fence_after();
            issue_pv(0, itV(jj), true, kBlockN / 32, kBlockN / 16, jj == a0 - 1 ? bar(BAR_OFINAL + 0) : 0u,
                     jj >= a1 ? free_of(itV(jj)) : 0u);
            if (jj + 1 < a0)
              issue_s(0, itK(jj + 1), bar(BAR_S + 0), jj + 1 >= a1 ? free_of(itK(jj + 1)) : 0u,
                      jj + 1 >= a1 ? qfree : 0u);
          }
          // tile 1: PV1(j) and S1(j+1); the last use of V_j and K_{j+1}
          if (jj < a1) {
            if (!mbar_wait_warp(bar(BAR_PH + 1), p_cnt[1] & 1, g, FA2_SITE_O_RESCALED, pc.jb + jj)) break;
            tc_fence_after();
            issue_pv(1, itV(jj), jj > 0, 0, kBlockN / 32, 0u, 0u);
            if (!mbar_wait_warp(bar(BAR_P + 1), p_cnt[1] & 1, g, FA2_SITE_P_READY, pc.jb + jj)) break;
            ++p_cnt[1];
            tc_fence_after();
            issue_pv(1, itV(jj), true, kBlockN / 32, kBlockN / 16, free_of(itV(jj)),
                     jj == a1 - 1 ? bar(BAR_OFINAL + 1) : 0u);
            if (jj + 1 < a1) issue_s(1, itK(jj + 1), bar(BAR_S + 1), free_of(itK(jj + 1)), qfree);
          }
        }
        itb += 2u * static_cast<uint32_t>(n_p);
      }
      // drain: every MMA issued above has completed before TMEM is released
      // (not cut short by the abort flag: tensor-core work always finishes)
      const WaitGuard drain{0u, p.limit_ns};
      commit(bar(BAR_DONE));
      mbar_wait_warp(bar(BAR_DONE), 0, drain, FA2_SITE_MMA_DRAIN, 0);
    }
  } else if (warp == 13) {
    // ============================ TMA producer warp ============================
    if (aligned_ok) {
      const uint32_t sQ = sbase + C::kOffQ;
      const uint32_t sKV = sbase + C::kOffKV;
      uint32_t it = 0;       // ring items issued
      uint32_t pieces = 0;   // pieces whose Q was loaded
      bool ok = true;
      while (ok && pit.next(p, pc, unit_plan)) {
        const int hk = pc.hq / (p.Hq / p.Hkv);
        // Q of this piece, once the previous piece's last S MMA released the buffer
        if (pieces > 0 && !mbar_wait_warp(bar(BAR_QFREE), (pieces - 1) & 1, g, FA2_SITE_Q_LOADED, pieces)) {
          ok = false;
          break;
        }
        if (elect_one()) {
          const uint32_t bytes = (pc.a0 > 0 ? C::kTileBytes : 0) + (pc.a1 > 0 ? C::kTileBytes : 0);
          mbar_arrive_expect_tx(bar(BAR_Q), bytes);
#pragma unroll 1
          for (int t = 0; t < 2; ++t) {
            if ((t ? pc.a1 : pc.a0) == 0) continue;
#pragma unroll
            for (int ch = 0; ch < C::kChunks; ++ch)
              tma_load_4d(sQ + t * C::kTileBytes + ch * kChunkBytes, &tmQ, bar(BAR_Q), ch * 64, pc.hq,
                          pc.qb * kRowsPerCta + t * kBlockM, pc.b);
          }
        }
        __syncwarp();
        ++pieces;
        // Ring items K_0, V_0, K_1, V_1, ...: K_0 signals BAR_K0; V_j and K_{j+1}
        // (what the MMA step j needs) both signal V_j's barrier, so the MMA
        // warp waits once per step.
        uint32_t vbar = 0;  // barrier of the last V item
        for (int j = pc.j0 + pc.jb; j < pc.j0 + pc.je && ok; ++j) {  // absolute K/V tiles
#pragma unroll 1
          for (int kv = 0; kv < 2; ++kv, ++it) {
            const int st = static_cast<int>(it % C::kStages);
            if (it >= static_cast<uint32_t>(C::kStages) &&
                !mbar_wait_warp(bar(BAR_KV_FULL + C::kStages + st), ((it / C::kStages) & 1) ^ 1, g,
                                FA2_SITE_KV_FREE, static_cast<int>(it))) {
              ok = false;
              break;
            }
            const bool first_k = (kv == 0 && j == pc.j0 + pc.jb);
            uint32_t tb;
            if (kv == 1) {
              vbar = bar(BAR_KV_FULL + st);
              tb = vbar;
            } else {
              tb = first_k ? bar(BAR_K0) : vbar;
            }
            if (elect_one()) {
              if (kv == 1)
                mbar_arrive_expect_tx(tb, (j + 1 < pc.j0 + pc.je ? 2 : 1) * C::kTileBytes);
              else if (first_k)
                mbar_arrive_expect_tx(tb, C::kTileBytes);
              const CUtensorMap* map = kv ? &tmV : &tmK;
#pragma unroll
              for (int ch = 0; ch < C::kChunks; ++ch)
                tma_load_4d(sKV + st * C::kTileBytes + ch * kChunkBytes, map, tb, ch * 64, hk, j * kBlockN, pc.b);
            }
            __syncwarp();
          }
        }
      }
      if (!ok) {
        // Give the copies already in flight time to land before the CTA exits.
        const WaitGuard drain{0u, p.limit_ns};
        for (uint32_t i = (it > static_cast<uint32_t>(C::kStages) ? it - C::kStages : 0u); i < it; ++i)
          if (i & 1u)  // V items: their barrier also counts the next K tile
            mbar_wait_warp(bar(BAR_KV_FULL + i % C::kStages), (i / C::kStages) & 1, drain,
                           FA2_SITE_LOAD_DRAIN, static_cast<int>(i));
        if (pieces > 0) mbar_wait_warp(bar(BAR_K0), (pieces - 1) & 1, drain, FA2_SITE_LOAD_DRAIN, 0);
        if (pieces > 0) mbar_wait_warp(bar(BAR_Q), (pieces - 1) & 1, drain, FA2_SITE_LOAD_DRAIN, 0);
      }
    }
   } else {
    // ============== warps 14-15: rows of units with no visible key ==============
    // Units with no K/V tile at all (causal, Nq > Nk): O = 0, LSE = -inf.
    // They form a suffix of the unit order; stream-K CTAs share them round robin.
    const int et = threadIdx.x - (kThreads - kEmptyThreads);  // 0..63
    const int HB = p.B * p.Hq;
    const int r0 = p.r_empty;
    const int nz = (p.n_qblk - r0) * HB;
    const int z0 = SK ? static_cast<int>(blockIdx.x) : static_cast<int>(blockIdx.x) - r0 * HB;
    const int dz = SK ? p.G : nz;  // unit mode: CTA u owns unit u only
    for (int z = z0; z >= 0 && z < nz; z += dz) {
      const int rr = r0 + z / HB, k = z % HB, qb = p.n_qblk - 1 - rr;
      const int b = k / p.Hq, hq = k % p.Hq;
      for (int i = et; i < kRowsPerCta * (D / 8); i += kEmptyThreads) {
        const int row = qb * kRowsPerCta + i / (D / 8);
        if (row >= p.Nq) continue;
        reinterpret_cast<uint4*>(p.o + ((static_cast<size_t>(b) * p.Nq + row) * p.Hq + hq) * D)[i % (D / 8)] =
            make_uint4(0u, 0u, 0u, 0u);
        if (i % (D / 8) == 0) p.lse[(static_cast<size_t>(b) * p.Hq + hq) * p.Nq + row] = -INFINITY;
      }
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

// ---------------------------------------------------------------------------
// Split-KV merge: after the stream-K kernel, every unit cut by a range boundary
// has np partials (O unnormalised in fp32, row max m and denominator l over
// its own K/V range); they combine with the identity that makes the softmax
// statistics mergeable: m = max m_i, l = sum l_i 2^(m_i - m),
// O = sum O_i 2^(m_i - m) / l, LSE = (m + log2 l) ln 2 ("FlashAttention-2 and
// -3: From Algebra to GPU Scheduling", "Keep the unchanged mathematical target
// in view" and "Another use of mergeable statistics").  Pieces are summed in
// their order in the unit, so the result is deterministic.
//
// Grid: (boundary c that is the first cut of a split unit, listed by the
// host) x (64-row block of the unit's 256 rows) x (16-column chunk of d);
// 4 threads share a row, each owning 4 consecutive columns, so a warp reads
// 512 contiguous bytes.
// ---------------------------------------------------------------------------
constexpr int kCombineThreads = 256;
constexpr int kCombineRows = 64;

template <int D>
__global__ void __launch_bounds__(kCombineThreads)
    fa2_combine_kernel(const Params p, const __grid_constant__ CutList cuts) {
  using C = Cfg<D>;
  const int slot = cuts.slot[blockIdx.x], np = cuts.np[blockIdx.x], qb = cuts.qb[blockIdx.x];
  const int b = cuts.bh[blockIdx.x] / p.Hq, hq = cuts.bh[blockIdx.x] % p.Hq;

  const int rr = static_cast<int>(blockIdx.y) * kCombineRows + static_cast<int>(threadIdx.x) / 4;
  const int f4 = threadIdx.x % 4;
  const int ch = blockIdx.z;
  const int t = rr / kBlockM, rt = rr % kBlockM;
  const int row = qb * kRowsPerCta + rr;
  if (row >= p.Nq) return;
  auto part = [&](int q) {
    return p.ws + static_cast<size_t>(2 * (slot + q) + (q == 0 ? 1 : 0)) * C::kPieceFloats;
  };
  // One pass over the pieces in batches of kBatch, every load of a batch in
  // flight at once (statistics and O together); the accumulator follows the
  // running max across batches.  A unit is cut into about G / units pieces,
  // so this is one or two round trips to memory per thread.  (Batches of 16
  // take 154 registers, one block per SM, and measured no faster.)
  constexpr int kBatch = 8;
  float m_run = -INFINITY, l_tot = 0.f, lr_tot = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int q0 = 0; q0 < np; q0 += kBatch) {
    float mq[kBatch], lq[kBatch], lrq[kBatch];
    float4 f[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      lq[i] = 0.f;
      lrq[i] = 0.f;
      mq[i] = -INFINITY;
      f[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (q0 + i < np) {
        const float* base = part(q0 + i);
        lq[i] = __ldcg(base + C::part_l(t, rt));
        lrq[i] = __ldcg(base + C::part_lr(t, rt));
        mq[i] = __ldcg(base + C::part_m(t, rt));
        // a piece with l = 0 may not have written its O: loaded, then skipped
        f[i] = __ldcg(reinterpret_cast<const float4*>(base + C::part_o(t, ch, rt)) + f4);
      }
    }
    float mb = m_run;
#pragma unroll
    for (int i = 0; i < kBatch; ++i)
      if (lq[i] > 0.f) mb = fmaxf(mb, mq[i]);
    if (mb != m_run) {  // rescale what earlier batches accumulated
      const float sc = (m_run == -INFINITY) ? 0.f : ex2_approx(m_run - mb);
      l_tot *= sc;
      lr_tot *= sc;
      acc.x *= sc;
      acc.y *= sc;
      acc.z *= sc;
      acc.w *= sc;
      m_run = mb;
    }
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      if (!(lq[i] > 0.f)) continue;
      const float wq = ex2_approx(mq[i] - m_run);
      l_tot = fmaf(lq[i], wq, l_tot);
      lr_tot = fmaf(lrq[i], wq, lr_tot);
      acc.x = fmaf(wq, f[i].x, acc.x);
      acc.y = fmaf(wq, f[i].y, acc.y);
      acc.z = fmaf(wq, f[i].z, acc.z);
      acc.w = fmaf(wq, f[i].w, acc.w);
    }
  }
  const float m_tot = m_run;
  const float inv_l = (l_tot > 0.f) ? 1.f / (l_tot + lr_tot) : 0.f;
  __nv_bfloat16* orow = p.o + ((static_cast<size_t>(b) * p.Nq + row) * p.Hq + hq) * D;
  uint2 o2;
  o2.x = pack_bf16x2(acc.x * inv_l, acc.y * inv_l);
  o2.y = pack_bf16x2(acc.z * inv_l, acc.w * inv_l);
  reinterpret_cast<uint2*>(orow + 16 * ch)[f4] = o2;
  if (ch == 0 && f4 == 0)
    p.lse[(static_cast<size_t>(b) * p.Hq + hq) * p.Nq + row] =
        (l_tot > 0.f) ? (m_tot + log2f(l_tot)) * 0.69314718055994530942f : -INFINITY;
}

// One warp waits on an mbarrier nothing arrives on; the bounded wait runs out.
__global__ void selftest_timeout_kernel(uint32_t limit_ns) {
  __shared__ __align__(8) uint64_t bar_storage;
  __shared__ int abort_storage;
  if (threadIdx.x == 0) {
    abort_storage = 0;
    mbar_init(smem_addr(&bar_storage), 1);
    fence_mbar_init();
  }
  __syncwarp();
  const WaitGuard g{smem_addr(&abort_storage), limit_ns};
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
  if (static_cast<long long>(Nq) + Nk >= (1LL << 30)) return FA2_ERR_SIZE;  // window bounds stay in int
  const long long nblk = (static_cast<long long>(Nq) + kRowsPerCta - 1) / kRowsPerCta;
  if (nblk * Hq * B > INT_MAX) return FA2_ERR_SIZE;
  // one round of units (all heads and batches of a query block) must count
  // fewer than 2^31 K/V-tile iterations
  const long long nkt = (static_cast<long long>(Nk) + kBlockN - 1) / kBlockN;
  if (nkt * Hq * B >= (1LL << 31)) return FA2_ERR_SIZE;
  return FA2_OK;
}

// Host-side plan of the work decomposition (same unit order and sizes as the
// device iterator).
struct Plan {
  int n_qblk = 0;
  long long units = 0;  // (query block, head, batch) units
  long long iters = 0;  // K/V-tile iterations summed over all units
  long long T = 0;      // summed unit costs (kUnitCost + iterations per non-empty unit)
  int G = 0;            // stream-K CTAs (0 when there is nothing to compute)
  long long ws_bytes = 0;
};

static Plan make_plan(int B, int Hq, int Nq, int Nk, Window win, int d, int num_sms) {
  Plan pl;
  pl.n_qblk = (Nq + kRowsPerCta - 1) / kRowsPerCta;
  const long long HB = static_cast<long long>(B) * Hq;
  pl.units = HB * pl.n_qblk;
  for (int qb = 0; qb < pl.n_qblk; ++qb) {
    const int n = unit_tiles(Nq, Nk, win, qb);
    pl.iters += HB * n;
    pl.T += HB * (n > 0 ? n + kUnitCost : 0);
  }
  if (pl.iters == 0 || num_sms <= 0) return pl;
  pl.G = static_cast<int>(pl.iters < num_sms ? pl.iters : num_sms);
  // a CTA's range holds at most two pieces of split units (its first and its
  // last), so two partial buffers per CTA cover every split
  const long long piece_bytes = 4LL * kTiles * kBlockM * (d + 3);
  pl.ws_bytes = (pl.G > 1) ? 2LL * pl.G * piece_bytes : 0;
  return pl;
}

// Which schedule a call with a workspace should take.  Both are priced in
// K/V-tile iterations of one CTA, a unit costing its tiles + kUnitCost:
// whole units finish when the busiest SM does (longest-first list
// scheduling of the units, one per CTA); split-KV spreads the summed cost
// evenly over G CTAs and adds the merge.  A split-KV iteration measured
// 1.25-1.35x slower than a whole-unit one (partial outputs, the merge, short
// pieces), so split-KV is taken only when it predicts a clear win, and only
// with fewer units than two per SM (the persistent whole-unit schedule
// balances anything larger to within a few percent) ("FlashAttention-2 and
// -3: From Algebra to GPU Scheduling", "Another use of mergeable statistics":
// splitting keys buys parallelism when the queries alone give too little).
constexpr double kSplitMargin = 1.5;
constexpr int kMergeCost = 4;
struct ScheduleChoice {
  int split = 0;
  long long mk_units = 0, mk_split = 0;
};

static ScheduleChoice choose_schedule(int B, int Hq, int Nq, int Nk, Window win, int d, int sms) {
  ScheduleChoice ch;
  const Plan pl = make_plan(B, Hq, Nq, Nk, win, d, sms);
  if (pl.G <= 0 || sms <= 0) return ch;
  const long long HB = static_cast<long long>(B) * Hq;
  long long units_ne = 0;
  for (int qb = 0; qb < pl.n_qblk; ++qb)
    if (unit_tiles(Nq, Nk, win, qb) > 0) units_ne += HB;
  ch.mk_split = (pl.T + pl.G - 1) / pl.G + kMergeCost;
  if (units_ne >= 2LL * sms) {  // balanced persistent plan: about the average
    ch.mk_units = (pl.T + sms - 1) / sms;
    return ch;
  }
  std::vector<long long> cost;
  for (int qb = pl.n_qblk - 1; qb >= 0; --qb) {
    const int n = unit_tiles(Nq, Nk, win, qb);
    if (n > 0) cost.insert(cost.end(), static_cast<size_t>(HB), n + kUnitCost);
  }
  std::sort(cost.begin(), cost.end(), std::greater<long long>());
  std::priority_queue<long long, std::vector<long long>, std::greater<long long>> load;
  for (int i = 0; i < sms; ++i) load.push(0);
  for (long long c : cost) {
    const long long l = load.top() + c;
    load.pop();
    load.push(l);
    ch.mk_units = std::max(ch.mk_units, l);
  }
  ch.split = (kSplitMargin * static_cast<double>(ch.mk_split) < static_cast<double>(ch.mk_units)) ? 1 : 0;
  return ch;
}

// Plan of persistent whole units (UnitTable).  The heavier units are listed in
// groups of consecutive (batch, head) pairs -- whole GQA groups, about one
// wave of units per group -- heaviest first inside each group; the light
// units (at most 40 % of the heaviest unit's cost) follow, across all heads,
// heaviest first.  Each unit in turn goes to the CTA whose planned work (K/V
// tile iterations plus the fixed cost of a unit) is smallest.  The groups keep
// the CTAs running at any moment on a few neighbouring heads, whose K and V
// then stay in L2; the light tail evens out the CTAs' work at the end, where a
// purely head-ordered list would leave some heavy units last ("FlashAttention
// 2: Three Places the Chip Was Still Waiting", section 2.3: many more blocks
// than SMs; which of them share the cache is this library's choice).  Returns
// false when the problem exceeds the table.
static bool plan_units(int B, int Hq, int Hkv, int Nq, int Nk, Window win, int n_qblk, int r_empty,
                       int G, UnitTable& tab) {
  const long long HB = static_cast<long long>(B) * Hq;
  const long long units = HB * r_empty;
  if (G <= 0 || G > kMaxTableCtas || units <= 0 || units > kMaxTableUnits) return false;
  const int grp = Hq / Hkv;  // query heads sharing a KV head
  // heads per group: about one wave of units, a whole number of GQA groups
  long long hg = (static_cast<long long>(G) + r_empty - 1) / r_empty;
  hg = ((hg + grp - 1) / grp) * grp;
  if (hg > HB) hg = HB;
  std::vector<int> cost(r_empty);
  int cmax = 0;
  for (int r = 0; r < r_empty; ++r) {
    cost[r] = unit_tiles(Nq, Nk, win, n_qblk - 1 - r) + kUnitCost;
    cmax = std::max(cmax, cost[r]);
  }
  std::vector<int> heavy, light;  // rounds
  for (int r = 0; r < r_empty; ++r) (5 * cost[r] > 2 * cmax ? heavy : light).push_back(r);
  std::stable_sort(light.begin(), light.end(), [&](int a, int b) { return cost[a] > cost[b]; });
  // list scheduling: the next unit goes to the CTA with the least planned work
  // the list of units in dealing order
  std::vector<std::pair<int, long long>> order;  // (round, b * Hq + hq)
  for (long long k0 = 0; k0 < HB; k0 += hg)
    for (int r : heavy)
      for (long long k = k0; k < std::min(HB, k0 + hg); ++k) order.push_back({r, k});
  for (int r : light)
    for (long long k = 0; k < HB; ++k) order.push_back({r, k});
  // Units that would make a last, at most half-full wave are dealt as two
  // single-tile halves each, so twice as many CTAs share that wave: with R
  // units left after the full waves (2 R <= G), the slowest CTA finishes one
  // half unit after the full waves instead of one whole unit.  A half costs
  // its tiles x 5/8 + the fixed cost (one query tile's softmax and MMAs per
  // K/V tile, the K/V stream unchanged).
  const long long rest = units % G;
  long long n_half = (2 * rest <= G && units + rest <= kMaxTableUnits) ? rest : 0;
  using Slot = std::pair<long long, int>;  // (planned work, CTA)
  std::priority_queue<Slot, std::vector<Slot>, std::greater<Slot>> free_at;
  for (int c = 0; c < G; ++c) free_at.push({0, c});
  std::vector<std::vector<uint16_t>> lists(G);
  auto assign = [&](int entry, int c_work) {
    const Slot sl = free_at.top();
    free_at.pop();
    lists[sl.second].push_back(static_cast<uint16_t>(entry));
    free_at.push({sl.first + c_work, sl.second});
  };
  const long long first_half = static_cast<long long>(order.size()) - n_half;
  for (long long i = 0; i < static_cast<long long>(order.size()); ++i) {
    const int r = order[i].first;
    const int u = static_cast<int>(r * HB + order[i].second);
    const UnitSpan sp = unit_span(Nq, Nk, win, n_qblk - 1 - r);
    if (i >= first_half && sp.n0 > 0 && sp.n1 > 0) {
      const int hc = (cost[r] - kUnitCost) * 5 / 8 + kUnitCost;
      assign(u + kHalfTile0, hc);
      assign(u + kHalfTile1, hc);
    } else {
      assign(u, cost[r]);
    }
  }
  int pos = 0;
  for (int c = 0; c < G; ++c) {
    tab.start[c] = static_cast<uint16_t>(pos);
    for (uint16_t u : lists[c]) tab.unit[pos++] = u;
  }
  tab.start[G] = static_cast<uint16_t>(pos);
  return true;
}

// The boundaries c (1 <= c < G) of a stream-K launch that cut a unit for the
// first time, in the device's unit order (the same walk as PieceIter and the
// combine kernel's own check).  False when G exceeds the list.
static bool first_cuts(const Params& p, Window win, CutList& cuts) {
  cuts.n = 0;
  if (p.G - 1 > kMaxTableCtas) return false;
  const long long HB = static_cast<long long>(p.B) * p.Hq;
  auto cost = [](int n) { return n > 0 ? n + kUnitCost : 0; };
  long long cum = 0;
  int r = 0;
  int n = unit_tiles(p.Nq, p.Nk, win, p.n_qblk - 1);
  for (int c = 1; c < p.G; ++c) {
    const long long bc = range_start(p.span, p.rem, p.G, c);
    while (bc >= cum + HB * cost(n)) {  // boundaries increase with c: walk the rounds once
      cum += HB * cost(n);
      ++r;
      n = unit_tiles(p.Nq, p.Nk, win, p.n_qblk - 1 - r);
    }
    const long long w = cost(n);
    const long long k = (bc - cum) / w;
    const long long s0 = cum + k * w + kUnitCost;  // position of the unit's iteration 0
    const bool cuts_unit = bc > s0 && bc <= s0 + n - 1;
    const bool first = c == 1 || range_start(p.span, p.rem, p.G, c - 1) <= s0;
    if (!cuts_unit || !first) continue;
    // pieces: one per range that overlaps the unit's iterations [s0, s0 + n)
    int c_end = c;
    while (c_end + 1 < p.G && range_start(p.span, p.rem, p.G, c_end + 1) <= s0 + n - 1) ++c_end;
    const int i = cuts.n++;
    cuts.slot[i] = static_cast<uint16_t>(c - 1);
    cuts.np[i] = static_cast<uint16_t>(c_end - c + 2);
    cuts.qb[i] = static_cast<uint16_t>(p.n_qblk - 1 - r);
    cuts.bh[i] = static_cast<int>(k);
  }
  return true;
}

static int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

// Devices the per-device set-up below can track (device ordinals 0 .. 63).
constexpr int kMaxDevices = 64;

// Runs `setup` once per device (the current one) and returns its status on
// every later call.  Function attributes such as the dynamic shared-memory
// limit are per device, so a process that calls the library on several GPUs
// sets them up on each.
template <typename F>
static int once_per_device(std::once_flag (&flags)[kMaxDevices], int (&status)[kMaxDevices], F setup) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA2_ERR_DEVICE;
  std::call_once(flags[dev], [&] { status[dev] = setup(); });
  return status[dev];
}

template <int D>
static int launch(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                  int Hkv, int Nq, int Nk, Window win, float scale, void* workspace,
                  long long workspace_bytes, cudaStream_t stream, bool persistent_units) {
  using C = Cfg<D>;
  static std::once_flag flags[kMaxDevices];
  static int setup_status[kMaxDevices];
  const int st = once_per_device(flags, setup_status, [] {
    auto setup = [](auto* kern) {
      cudaFuncAttributes attr;
      if (cudaFuncGetAttributes(&attr, kern) != cudaSuccess) return static_cast<int>(FA2_ERR_LAUNCH);
      // the setmaxnreg split assumes exactly this pool
      if (attr.numRegs != kLaunchRegs) return static_cast<int>(FA2_ERR_BUILD);
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
          cudaSuccess)
        return static_cast<int>(FA2_ERR_LAUNCH);
      return static_cast<int>(FA2_OK);
    };
    const int s0 = setup(fa2_fwd_kernel<D, false>);
    return s0 != FA2_OK ? s0 : setup(fa2_fwd_kernel<D, true>);
  });
  if (st != FA2_OK) return st;

  Params p;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Nq = Nq;
  p.Nk = Nk;
  p.wl = win.wl;
  p.wr = win.wr;
  p.n_qblk = (Nq + kRowsPerCta - 1) / kRowsPerCta;
  p.r_empty = 0;
  while (p.r_empty < p.n_qblk && unit_tiles(Nq, Nk, win, p.n_qblk - 1 - p.r_empty) > 0) ++p.r_empty;
  // c is kept strictly positive so a masked score (-inf) always maps to
  // exp2(-inf) = 0; for softmax_scale == 0 every unmasked exponent is then
  // c * (s - m) ~ 1e-30 * O(1e4), which rounds to exp2(0) = 1 as required.
  p.c = std::fmax(std::fabs(scale) * 1.4426950408889634f, 1e-30f);
  p.negate = scale < 0.f ? 1 : 0;
  p.limit_ns = 1000000000u;  // 1 s per wait; a healthy wait takes microseconds
  p.streamk = 0;
  p.pu = 0;
  p.tab = 0;
  p.T = 0;
  p.span = 0;
  p.rem = 0;
  p.G = 1;
  p.ws = nullptr;
  unsigned grid = static_cast<unsigned>(p.n_qblk) * Hq * B;  // one unit per CTA
  const long long units_ne = static_cast<long long>(p.r_empty) * Hq * B;
  const int sms = sm_count();
  static thread_local UnitTable plan;  // kernel parameter of the persistent launch
  if (!workspace && persistent_units && sms > 0 && units_ne >= 2LL * sms) {
    // persistent CTAs over whole units: the next unit's Q and K/V stream in
    // while the current one drains, instead of a block exit and launch
    p.pu = 1;
    p.G = sms;
    grid = static_cast<unsigned>(sms);
    p.tab = plan_units(B, Hq, Hkv, Nq, Nk, win, p.n_qblk, p.r_empty, sms, plan) ? 1 : 0;
  }
  if (workspace) {
    const Plan pl = make_plan(B, Hq, Nq, Nk, win, D, sm_count());
    if (pl.G > 0) {  // otherwise every unit is empty: one CTA per unit writes it
      if (pl.T > INT_MAX) return FA2_ERR_SIZE;
      if (workspace_bytes < pl.ws_bytes) return FA2_ERR_WORKSPACE;
      p.streamk = 1;
      p.T = static_cast<int>(pl.T);
      p.G = pl.G;
      p.span = static_cast<int>(pl.T / pl.G);
      p.rem = static_cast<int>(pl.T % pl.G);
      p.ws = static_cast<float*>(workspace);
      grid = static_cast<unsigned>(pl.G);
    }
  }

  CUtensorMap tq, tk, tv;
  if (!encode_bnhd(&tq, q, B, Nq, Hq, D) || !encode_bnhd(&tk, k, B, Nk, Hkv, D) ||
      !encode_bnhd(&tv, v, B, Nk, Hkv, D))
    return FA2_ERR_LAUNCH;
  if (p.streamk || p.pu)
    fa2_fwd_kernel<D, true><<<grid, kThreads, C::kSmemBytes, stream>>>(tq, tk, tv, p, plan);
  else
    fa2_fwd_kernel<D, false><<<grid, kThreads, C::kSmemBytes, stream>>>(tq, tk, tv, p, NoTable{});
  if (cudaGetLastError() != cudaSuccess) return FA2_ERR_LAUNCH;
  if (p.streamk && p.G > 1) {
    CutList cuts;
    if (!first_cuts(p, win, cuts)) return FA2_ERR_SIZE;
    if (cuts.n > 0) {
      const dim3 cgrid(static_cast<unsigned>(cuts.n), kRowsPerCta / kCombineRows, D / 16);
      fa2_combine_kernel<D><<<cgrid, kCombineThreads, 0, stream>>>(p, cuts);
      if (cudaGetLastError() != cudaSuccess) return FA2_ERR_LAUNCH;
    }
  }
  return FA2_OK;
}

#include "fa2_backward.cuh"

static int check_device() {
  static std::once_flag flags[kMaxDevices];
  static int cached[kMaxDevices];
  return once_per_device(flags, cached, [] {
    int dev = 0, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return static_cast<int>(FA2_ERR_DEVICE);
    return (major == 10 && minor == 0) ? static_cast<int>(FA2_OK) : static_cast<int>(FA2_ERR_DEVICE);
  });
}

}  // namespace fa2

using namespace fa2;

// The checks of the forward entry points that need no CUDA call: pointers,
// shape, alignment (TMA needs 16-byte aligned q, k, v, o), the scale.
static int validate_args(const void* q, const void* k, const void* v, const void* o, const float* lse,
                         int B, int Hq, int Hkv, int Nq, int Nk, int d, float softmax_scale) {
  if (!q || !k || !v || !o || !lse) return FA2_ERR_NULL_POINTER;
  const int sv = validate_shape(B, Hq, Hkv, Nq, Nk, d);
  if (sv != FA2_OK) return sv;
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
       reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(o)) & 15u)
    return FA2_ERR_ALIGNMENT;
  if (reinterpret_cast<uintptr_t>(lse) & 3u) return FA2_ERR_ALIGNMENT;
  if (!std::isfinite(softmax_scale)) return FA2_ERR_SCALE;
  return FA2_OK;
}

static int forward_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                        int Hq, int Hkv, int Nq, int Nk, int d, Window win, float softmax_scale,
                        void* workspace, long long workspace_bytes, void* stream) {
  const int sa = validate_args(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, softmax_scale);
  if (sa != FA2_OK) return sa;
  if (reinterpret_cast<uintptr_t>(workspace) & 15u) return FA2_ERR_ALIGNMENT;
  if (workspace && workspace_bytes < 0) return FA2_ERR_WORKSPACE;
  const int dv = check_device();
  if (dv != FA2_OK) return dv;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d == 128)
    return launch<128>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, win, softmax_scale, workspace,
                       workspace_bytes, s, kPersistentUnits);
  return launch<64>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, win, softmax_scale, workspace,
                    workspace_bytes, s, kPersistentUnits);
}

extern "C" int fa2_forward(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                           int Hq, int Hkv, int Nq, int Nk, int d, int causal, float softmax_scale,
                           void* stream) {
  return forward_impl(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal_window(causal), softmax_scale,
                      nullptr, 0, stream);
}

extern "C" int fa2_forward_local(const void* q, const void* k, const void* v, void* o, float* lse,
                                 int B, int Hq, int Hkv, int Nq, int Nk, int d, int window_left,
                                 int window_right, float softmax_scale, void* stream) {
  if (window_left < -1 || window_right < -1) return FA2_ERR_WINDOW;
  // a width that reaches past every key of every row is no bound: g - wl <= 0
  // for all rows once wl >= Nk, and g + wr >= Nk - 1 once wr >= Nq
  Window w{window_left >= Nk ? -1 : window_left, window_right >= Nq ? -1 : window_right};
  return forward_impl(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, w, softmax_scale, nullptr, 0, stream);
}

extern "C" int fa2_forward_ws(const void* q, const void* k, const void* v, void* o, float* lse,
                              int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal,
                              float softmax_scale, void* workspace, long long workspace_bytes,
                              void* stream) {
  if (!workspace) return FA2_ERR_NULL_POINTER;
  return forward_impl(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal_window(causal), softmax_scale,
                      workspace, workspace_bytes, stream);
}

extern "C" int fa2_schedule_choice(int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal, int num_sms,
                                   int* split, long long* cost_units, long long* cost_split) {
  const int sv = validate_shape(B, Hq, Hkv, Nq, Nk, d);
  if (sv != FA2_OK) return sv;
  if (num_sms <= 0) return FA2_ERR_BAD_SHAPE;
  const ScheduleChoice ch = choose_schedule(B, Hq, Nq, Nk, causal_window(causal), d, num_sms);
  if (split) *split = ch.split;
  if (cost_units) *cost_units = ch.mk_units;
  if (cost_split) *cost_split = ch.mk_split;
  return FA2_OK;
}

extern "C" int fa2_forward_auto(const void* q, const void* k, const void* v, void* o, float* lse,
                                int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal,
                                float softmax_scale, void* workspace, long long workspace_bytes,
                                void* stream) {
  const int sv = validate_shape(B, Hq, Hkv, Nq, Nk, d);
  if (sv != FA2_OK) return sv;
  const ScheduleChoice ch = choose_schedule(B, Hq, Nq, Nk, causal_window(causal), d, sm_count());
  const bool split = ch.split && workspace;
  return forward_impl(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal_window(causal), softmax_scale,
                      split ? workspace : nullptr, split ? workspace_bytes : 0, stream);
}

// ---------------------------------------------------------------------------
// Allocation-free stream-K: the same two kernels as fa2_forward_ws, with the
// scratch taken from a fixed device array of this library instead of from
// the caller.  For callers that cannot allocate device memory on the call
// path and hold no buffer to lend: code running against a fixed, already
// reserved memory budget (a serving loop that must not grow its footprint
// per request), and code that cannot afford the device-wide synchronisation
// cudaMalloc / cudaFree may imply.  Nothing in the array needs to start at
// zero: every partial the combine kernel reads was written earlier in the
// same call.  One array per device serves every call, so calls that may
// overlap in time race on it.
// ---------------------------------------------------------------------------
constexpr size_t kStaticScratchBytes = FA2_STATIC_WS_BYTES;  // 2 partials x 156 SMs at d = 128 fit
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of the array on device `dev` (the current device), or
// nullptr if it cannot be obtained.  Only a successful lookup is kept: a
// failed one (for instance made while the stream was being captured) is
// retried by the next call.
static void* static_scratch(int dev) {
  static std::atomic<void*> addr[kMaxDevices];
  void* a = addr[dev].load(std::memory_order_acquire);
  if (a) return a;
  if (cudaGetSymbolAddress(&a, g_static_scratch) != cudaSuccess || !a) {
    cudaGetLastError();  // clear it, so a later launch check does not report it
    return nullptr;
  }
  addr[dev].store(a, std::memory_order_release);  // the same value whichever thread stores it
  return a;
}

extern "C" int fa2_forward_static_ws(const void* q, const void* k, const void* v, void* o, float* lse,
                                     int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal,
                                     float softmax_scale, void* stream) {
  // every argument check fa2_forward makes, in its order, before any CUDA call
  const int sv = validate_args(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, softmax_scale);
  if (sv != FA2_OK) return sv;
  const int dv = check_device();
  if (dv != FA2_OK) return dv;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA2_ERR_DEVICE;
  void* scratch = static_scratch(dev);
  if (!scratch) return FA2_ERR_LAUNCH;
  // a problem whose plan needs more than the array is refused (FA2_ERR_WORKSPACE)
  return forward_impl(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal_window(causal), softmax_scale,
                      scratch, static_cast<long long>(kStaticScratchBytes), stream);
}

extern "C" long long fa2_backward_workspace_size(int B, int Hq, int Nq, int d) {
  if (B <= 0 || Hq <= 0 || Nq <= 0 || (d != 64 && d != 128)) return -1;
  return bwd_workspace_bytes(B, Hq, Nq, d);
}

static int backward_impl(const void* q, const void* k, const void* v, const void* o,
                         const float* lse, const void* dout, void* dq, void* dk, void* dv, int B,
                         int Hq, int Hkv, int Nq, int Nk, int d, Window win, float softmax_scale,
                         void* workspace, long long workspace_bytes, void* stream) {
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv || !workspace)
    return FA2_ERR_NULL_POINTER;
  const int sv = validate_shape(B, Hq, Hkv, Nq, Nk, d);
  if (sv != FA2_OK) return sv;
  if (Hkv > 65535 || B > 65535) return FA2_ERR_SIZE;
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v) |
       reinterpret_cast<uintptr_t>(o) | reinterpret_cast<uintptr_t>(dout) | reinterpret_cast<uintptr_t>(dq) |
       reinterpret_cast<uintptr_t>(dk) | reinterpret_cast<uintptr_t>(dv) |
       reinterpret_cast<uintptr_t>(workspace)) & 15u)
    return FA2_ERR_ALIGNMENT;
  if (reinterpret_cast<uintptr_t>(lse) & 3u) return FA2_ERR_ALIGNMENT;
  if (!std::isfinite(softmax_scale)) return FA2_ERR_SCALE;
  if (workspace_bytes < bwd_workspace_bytes(B, Hq, Nq, d)) return FA2_ERR_WORKSPACE;
  const int dv_ = check_device();
  if (dv_ != FA2_OK) return dv_;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d == 128)
    return launch_bwd<128>(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, Nq, Nk, win, softmax_scale,
                           workspace, s);
  return launch_bwd<64>(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, Nq, Nk, win, softmax_scale,
                        workspace, s);
}

extern "C" int fa2_backward(const void* q, const void* k, const void* v, const void* o,
                            const float* lse, const void* dout, void* dq, void* dk, void* dv, int B,
                            int Hq, int Hkv, int Nq, int Nk, int d, int causal, float softmax_scale,
                            void* workspace, long long workspace_bytes, void* stream) {
  return backward_impl(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, causal_window(causal),
                       softmax_scale, workspace, workspace_bytes, stream);
}

extern "C" int fa2_backward_local(const void* q, const void* k, const void* v, const void* o,
                                  const float* lse, const void* dout, void* dq, void* dk, void* dv,
                                  int B, int Hq, int Hkv, int Nq, int Nk, int d, int window_left,
                                  int window_right, float softmax_scale, void* workspace,
                                  long long workspace_bytes, void* stream) {
  if (window_left < -1 || window_right < -1) return FA2_ERR_WINDOW;
  // widths reaching past every key are no bound (as in fa2_forward_local)
  const Window w{window_left >= Nk ? -1 : window_left, window_right >= Nq ? -1 : window_right};
  return backward_impl(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, w, softmax_scale,
                       workspace, workspace_bytes, stream);
}

extern "C" long long fa2_workspace_size(int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal) {
  if (validate_shape(B, Hq, Hkv, Nq, Nk, d) != FA2_OK) return -1;
  const int n = sm_count();
  if (n <= 0) return -1;
  const Plan pl = make_plan(B, Hq, Nq, Nk, causal_window(causal), d, n);
  return pl.T > INT_MAX ? -1 : pl.ws_bytes;
}

extern "C" int fa2_persistent_plan(int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal,
                                   int num_sms, int* start, int* units, int units_capacity) {
  const int sv = validate_shape(B, Hq, Hkv, Nq, Nk, d);
  if (sv != FA2_OK) return sv;
  if (!start || !units) return FA2_ERR_NULL_POINTER;
  if (num_sms <= 0) return FA2_ERR_BAD_SHAPE;
  const Window win = causal_window(causal);
  const int n_qblk = (Nq + kRowsPerCta - 1) / kRowsPerCta;
  int r_empty = 0;
  while (r_empty < n_qblk && unit_tiles(Nq, Nk, win, n_qblk - 1 - r_empty) > 0) ++r_empty;
  static thread_local UnitTable tab;
  if (!plan_units(B, Hq, Hkv, Nq, Nk, win, n_qblk, r_empty, num_sms, tab)) return FA2_ERR_SIZE;
  if (tab.start[num_sms] > units_capacity) return FA2_ERR_SIZE;
  for (int c = 0; c <= num_sms; ++c) start[c] = tab.start[c];
  for (int i = 0; i < tab.start[num_sms]; ++i) units[i] = tab.unit[i];
  return FA2_OK;
}

extern "C" int fa2_streamk_plan(int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal,
                                int num_sms, long long* total_iters, int* ctas,
                                long long* workspace_bytes) {
  const int sv = validate_shape(B, Hq, Hkv, Nq, Nk, d);
  if (sv != FA2_OK) return sv;
  if (num_sms <= 0) return FA2_ERR_BAD_SHAPE;
  const Plan pl = make_plan(B, Hq, Nq, Nk, causal_window(causal), d, num_sms);
  if (pl.T > INT_MAX) return FA2_ERR_SIZE;
  if (total_iters) *total_iters = pl.iters;
  if (ctas) *ctas = pl.G;
  if (workspace_bytes) *workspace_bytes = pl.ws_bytes;
  return FA2_OK;
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
    case FA2_ERR_WORKSPACE: return "workspace smaller than fa2_workspace_size reports";
    case FA2_ERR_WINDOW: return "window widths must be >= -1";
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
  if (limit_ns < 1000000LL || limit_ns > 4000000000LL) return FA2_ERR_SIZE;
  const int dv = check_device();
  if (dv != FA2_OK) return dv;
  selftest_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint32_t>(limit_ns));
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
