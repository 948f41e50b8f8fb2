/*
 * fa2.h -- C ABI of the B200 (sm_100a) exact attention forward and backward
 * passes.
 *
 * The forward computes, for every batch b, query head hq and query row i,
 *
 *     O[b,i,hq,:] = softmax_j( softmax_scale * q[b,i,hq,:] . k[b,j,hk,:] ) v[b,j,hk,:]
 *     LSE[b,hq,i] = ln sum_j exp( softmax_scale * q[b,i,hq,:] . k[b,j,hk,:] )
 *
 * over the keys j visible to row i, exactly (up to floating-point rounding):
 * the result of standard attention, computed tile by tile with a running row
 * maximum and denominator so the Nq x Nk score matrix never exists in memory.
 * Sources: "FlashAttention 2: Three Places the Chip Was Still Waiting",
 * section 1 ("New here?": tiling and online softmax, the answer is exact) and
 * section 2.2 (the accumulator stays unnormalised and is divided once per
 * query block); "FlashAttention-2 and -3: From Algebra to GPU Scheduling",
 * "Keep the unchanged mathematical target in view".
 *
 * Conventions the pages leave open, fixed here:
 *   - causal: key j is visible to query row i iff j <= i + (Nk - Nq)
 *     (bottom-right alignment; the usual j <= i when Nq == Nk);
 *   - GQA ("GQA-aware" variants, "FlashAttention-2" explainer, "The
 *     Downstream Story"): query head hq reads KV head hq / (Hq / Hkv), i.e.
 *     consecutive groups of Hq/Hkv query heads share one KV head;
 *   - a row with no visible key gets O = 0 and LSE = -inf;
 *   - LSE is the natural log and includes softmax_scale.
 *
 * and the backward (fa2_backward) its gradients.  All entry points are
 * thread-safe and allocate no device memory; the stream-K forward and the
 * backward take their scratch memory from the caller, or (stream-K only) from
 * a fixed array of the library (fa2_forward_static_ws, whose calls must not
 * overlap).
 */
#ifndef FA2_H
#define FA2_H

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by the host entry points. */
enum fa2_status_code {
  FA2_OK = 0,
  FA2_ERR_NULL_POINTER = 1,   /* a required pointer is NULL                          */
  FA2_ERR_BAD_SHAPE = 2,      /* B, Hq, Hkv, Nq or Nk <= 0, or Hq % Hkv != 0         */
  FA2_ERR_HEAD_DIM = 3,       /* d is not 64 or 128                                  */
  FA2_ERR_ALIGNMENT = 4,      /* q, k, v, o not 16-byte aligned, or lse not 4-byte   */
  FA2_ERR_SCALE = 5,          /* softmax_scale is NaN or infinite                    */
  FA2_ERR_DEVICE = 6,         /* current device is not compute capability 10.0      */
  FA2_ERR_LAUNCH = 7,         /* a CUDA runtime/driver call or the launch failed    */
  FA2_ERR_SIZE = 8,           /* a tensor or the grid exceeds the supported extent   */
  FA2_ERR_BUILD = 9,          /* the kernel image does not match its register plan  */
  FA2_ERR_WORKSPACE = 10,     /* workspace smaller than fa2_workspace_size reports   */
  FA2_ERR_WINDOW = 11         /* a window width below -1                             */
};

/*
 * fa2_forward -- enqueue one attention forward pass on `stream` (one kernel:
 * a block per unit of 256 query rows, or, with at least two units per SM,
 * one persistent block per SM that takes whole units round robin so the next
 * unit's loads overlap the current one's drain; same arithmetic either way).
 *
 *   q    device pointer, bf16 [B, Nq, Hq,  d], contiguous (d fastest); read only
 *   k    device pointer, bf16 [B, Nk, Hkv, d], contiguous; read only
 *   v    device pointer, bf16 [B, Nk, Hkv, d], contiguous; read only
 *   o    device pointer, bf16 [B, Nq, Hq,  d], contiguous; written (every element)
 *   lse  device pointer, fp32 [B, Hq, Nq],     contiguous; written (every element)
 *   B, Hq, Hkv, Nq, Nk   sizes, all > 0, Hq a multiple of Hkv
 *   d               head dimension, 64 or 128
 *   causal          0 = every key visible, nonzero = causal (see above)
 *   softmax_scale   any finite value (1/sqrt(d) is the usual choice)
 *   stream          cudaStream_t to launch on; NULL = the legacy default stream
 *
 * Ownership: the caller owns every buffer; the library keeps no reference after
 * the call returns.  o and lse must not overlap q, k or v (undefined otherwise).
 * The call is asynchronous: it validates the arguments (before any CUDA call,
 * so validation works without a GPU), builds the TMA descriptors, launches one
 * kernel and returns.  Errors are returned as fa2_status_code values; nothing
 * is thrown across the ABI.  A kernel that gave up on a wait (a bounded wait
 * that ran out; never expected in normal operation) leaves a nonzero code that
 * fa2_debug_status reports.
 */
int fa2_forward(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                int Hkv, int Nq, int Nk, int d, int causal, float softmax_scale, void* stream);

/*
 * fa2_forward_local -- local (sliding-window) attention: as fa2_forward, with
 * key j visible to query row i exactly when
 *
 *     g - window_left <= j <= g + window_right,   g = i + Nk - Nq
 *
 * (g is the row's diagonal key under the bottom-right alignment used for
 * causal attention).  A width of -1 leaves that side open: (-1, 0) is causal
 * attention, (-1, -1) full attention, (W, 0) a causal window of W + 1 keys.
 * The sliding-window variants fork from the same scheduling skeleton
 * ("FlashAttention-2" explainer, "The Downstream Story"); here the window
 * narrows each query block's range of K/V tiles (tiles wholly outside every
 * row's window are never loaded or multiplied) and only tiles that a row's
 * bound falls into pay for masking.  Rows that see no key get O = 0 and
 * LSE = -inf.  Returns FA2_ERR_WINDOW for a width below -1; otherwise as
 * fa2_forward.
 */
int fa2_forward_local(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                      int Hq, int Hkv, int Nq, int Nk, int d, int window_left, int window_right,
                      float softmax_scale, void* stream);

/*
 * fa2_forward_ws -- the same computation as fa2_forward, scheduled stream-K
 * over a caller-provided workspace.
 *
 * Units of work are (256-row query block, query head, batch); a unit costs one
 * iteration per K/V tile it visits.  fa2_forward launches one thread block per
 * unit, so the last wave of blocks and the longest causal unit leave SMs idle
 * (the occupancy problem of "FlashAttention 2: Three Places the Chip Was Still
 * Waiting", section 2.3, and "FlashAttention-2 and -3: From Algebra to GPU
 * Scheduling", "Why more parallelism has limits").  fa2_forward_ws instead
 * launches one persistent block per SM and cuts the summed unit costs (one
 * per K/V tile plus a fixed per-unit cost for the pipeline fill and the
 * epilogue; units heaviest first) into equal contiguous ranges, one per block.
 * A unit cut by a range boundary is computed in pieces over disjoint K/V
 * ranges; each piece writes its partial (O unnormalised in fp32, its row max
 * m and denominator l) to the workspace, and a second kernel, launched by the
 * same call on the same stream, merges the pieces of every split unit with
 * the identity that makes the softmax statistics mergeable (m = max m_i,
 * l = sum l_i e^(m_i - m), O = sum O_i e^(m_i - m) / l): the same page, "Keep
 * the unchanged mathematical target in view" and "Another use of mergeable
 * statistics".  This is the split-KV form of the forward pass; it also gives
 * a single long unit (a short query block against a long key sequence) the
 * whole GPU.  Partials stay in fp32 and are summed in a fixed order, so the
 * result is deterministic and equals fa2_forward's up to the order of
 * floating-point rounding.
 *
 *   workspace        device pointer, 16-byte aligned, at least
 *                    fa2_workspace_size(...) bytes for this problem on the
 *                    current device; scratch (no initialisation needed),
 *                    overwritten by every call
 *   workspace_bytes  size of `workspace` in bytes
 *   (other arguments as in fa2_forward)
 *
 * Returns FA2_ERR_NULL_POINTER for a NULL workspace, FA2_ERR_WORKSPACE
 * when workspace_bytes is smaller than required, and FA2_ERR_SIZE when the
 * summed unit costs reach 2^31 (far beyond any single call worth scheduling
 * this way; fa2_forward has no such limit).  Calls that may run at the same
 * time (streams without ordering between them) need separate workspaces;
 * calls ordered on one stream may share one.
 */
int fa2_forward_ws(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                   int Hkv, int Nq, int Nk, int d, int causal, float softmax_scale,
                   void* workspace, long long workspace_bytes, void* stream);

/*
 * fa2_forward_auto -- fa2_forward or fa2_forward_ws, whichever the library
 * predicts to be faster for this problem on the current device.  Both
 * schedules are priced in K/V-tile iterations of one block (a unit costs its
 * tiles plus the fixed per-unit cost): whole units finish when the busiest SM
 * does (longest-first list scheduling of the units, or the average when the
 * units number at least two per SM and the persistent plan balances them);
 * split-KV spreads the summed cost over one block per SM and adds the merge.
 * Split-KV is taken only when there are fewer than two units per SM and its
 * price times 1.5 is still below the whole-unit price (a split-KV iteration
 * measured 1.25-1.35x dearer: partial outputs, the merge, short pieces) --
 * a short query block against a long key sequence, where one block per unit
 * would leave most SMs idle ("FlashAttention-2 and -3: From Algebra to GPU
 * Scheduling", "Another use of mergeable statistics").
 *
 *   workspace        as in fa2_forward_ws, or NULL: then whole units always
 *   workspace_bytes  its size (at least fa2_workspace_size(...) when split-KV
 *                    is chosen)
 *   (other arguments as in fa2_forward)
 *
 * Returns what the chosen entry point returns (FA2_ERR_WORKSPACE when
 * split-KV is chosen and the workspace is too small).  The result equals
 * either schedule's up to the order of floating-point rounding.
 */
int fa2_forward_auto(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                     int Hkv, int Nq, int Nk, int d, int causal, float softmax_scale,
                     void* workspace, long long workspace_bytes, void* stream);

/*
 * fa2_workspace_size -- bytes of workspace fa2_forward_ws needs for this
 * problem on the current device: two partials of 2 x 128 x (d + 3) floats per
 * SM (0 when the work fits one block).  Returns -1 for an invalid shape (as fa2_forward validates it),
 * for a problem fa2_forward_ws refuses with FA2_ERR_SIZE, or when the device
 * cannot be queried.  Queries the device's SM count; makes no
 * other CUDA call.
 */
long long fa2_workspace_size(int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal);

/*
 * fa2_forward_static_ws -- fa2_forward_ws without a caller workspace: the
 * stream-K scratch is a fixed device array inside this library
 * (FA2_STATIC_WS_BYTES, 40 MiB per device, reserved when the library's device
 * code is loaded on that device), so the call allocates no device memory and
 * takes none from the caller.  The pages describe no such entry point; it has
 * no counterpart there.  It is for callers that cannot allocate on the call
 * path and hold no buffer to lend: code running inside a fixed, already
 * reserved memory budget, or code that cannot afford the device-wide
 * synchronisation that cudaMalloc / cudaFree may imply.
 *
 *   arguments, layouts and ownership as in fa2_forward.
 *
 * Nothing in the array needs to start at zero: every partial the merge reads
 * is written earlier in the same call.  Returns FA2_ERR_WORKSPACE when the
 * problem's fa2_workspace_size exceeds FA2_STATIC_WS_BYTES (it fits for
 * d = 64 and d = 128 on GPUs with up to 156 SMs), FA2_ERR_LAUNCH when the
 * array's device address cannot be obtained, and otherwise what
 * fa2_forward_ws returns.
 *
 * The array's address is looked up once per device (cudaGetSymbolAddress,
 * with that device current) on the first call on that device; make that first
 * call before capturing the stream into a CUDA graph.  A lookup that fails is
 * not remembered: the call returns FA2_ERR_LAUNCH and the next call tries
 * again.  Argument checks (pointers, shape, alignment, scale) come before any
 * CUDA call, as in fa2_forward.  All calls on a device
 * share the one array: calls that may overlap in time (unordered streams,
 * several host threads) race on it and give wrong results -- order them on
 * one stream.
 */
int fa2_forward_static_ws(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                          int Hq, int Hkv, int Nq, int Nk, int d, int causal,
                          float softmax_scale, void* stream);
#define FA2_STATIC_WS_BYTES (40LL << 20)

/*
 * fa2_backward -- gradients of the forward pass: given q, k, v, the forward's
 * o and lse, and an upstream gradient dout (bf16 [B, Nq, Hq, d], like o),
 * writes dq (bf16 [B, Nq, Hq, d]), dk and dv (bf16 [B, Nk, Hkv, d]):
 *
 *   P_ij = exp(softmax_scale q_i . k_j - lse_i) over the keys row i sees
 *   D_i  = dout_i . o_i,  dS_ij = P_ij (dout_i . v_j - D_i)
 *   dq_i = softmax_scale sum_j dS_ij k_j,  dk_j = softmax_scale sum_i dS_ij q_i,
 *   dv_j = sum_i P_ij dout_i    (dk, dv summed over each KV head's query group)
 *
 * the chain rule on the forward's definition, with P recomputed tile by tile
 * from lse so nothing of size Nq x Nk is stored; the pages report the
 * forward+backward figures of the method ("FlashAttention 2: Three Places the
 * Chip Was Still Waiting", section 2.5).  Three kernels on `stream`: D and
 * the log2 LSE per row (and zeroing of the dq accumulator), the main kernel
 * (one block per 128-key block, KV head and batch, tcgen05 MMAs; dq summed
 * in fp32, half of each tile by vector reductions and half by TMA bulk
 * reductions, so its last bits depend on the order in which blocks add),
 * and the bf16 rounding of dq.
 *
 *   workspace        device pointer, 16-byte aligned, at least
 *                    fa2_backward_workspace_size(B, Hq, Nq, d) bytes of
 *                    scratch: the fp32 dq accumulator and two floats per row
 *   causal, softmax_scale, sizes: as the forward call that produced o, lse
 *
 * Returns the fa2_forward codes, FA2_ERR_WORKSPACE for a short workspace and
 * FA2_ERR_SIZE when Hkv or B exceeds 65535.  Rows with no visible key
 * (lse = -inf) get dq = 0 and contribute nothing.
 */
int fa2_backward(const void* q, const void* k, const void* v, const void* o, const float* lse,
                 const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Nq,
                 int Nk, int d, int causal, float softmax_scale, void* workspace,
                 long long workspace_bytes, void* stream);

/*
 * fa2_backward_local -- fa2_backward for fa2_forward_local's window: key j is
 * visible to row i when g - window_left <= j <= g + window_right,
 * g = i + Nk - Nq (-1 leaves a side open).  o and lse must come from
 * fa2_forward_local with the same window.  FA2_ERR_WINDOW for a width below
 * -1; otherwise as fa2_backward.
 */
int fa2_backward_local(const void* q, const void* k, const void* v, const void* o, const float* lse,
                       const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv,
                       int Nq, int Nk, int d, int window_left, int window_right,
                       float softmax_scale, void* workspace, long long workspace_bytes,
                       void* stream);

/* Bytes of scratch fa2_backward needs (-1 for invalid arguments). */
long long fa2_backward_workspace_size(int B, int Hq, int Nq, int d);

/* Human-readable text for a status code (static storage, never NULL). */
const char* fa2_status_string(int status);

/*
 * fa2_debug_status -- synchronise `stream`, return the device status word of
 * the current device and reset it to 0.  0 means no kernel gave up on a wait;
 * otherwise the value is (site << 16) | (iteration & 0xffff), where site
 * names the wait (FA2_SITE_* below).  Returns -1 if a CUDA call failed.
 */
int fa2_debug_status(void* stream);

/* Wait sites reported by fa2_debug_status. */
enum fa2_wait_site {
  FA2_SITE_Q_LOADED = 1,
  FA2_SITE_KV_LOADED = 2,
  FA2_SITE_KV_FREE = 3,
  FA2_SITE_S_READY = 4,
  FA2_SITE_P_READY = 5,
  FA2_SITE_STATS_READY = 6,
  FA2_SITE_O_RESCALED = 7,
  FA2_SITE_O_FINAL = 8,
  FA2_SITE_FINAL_STATS = 9,
  FA2_SITE_MMA_DRAIN = 10,
  FA2_SITE_LOAD_DRAIN = 11,
  FA2_SITE_SMEM_ALIGN = 13,   /* backward: shared memory base too far from 1 KiB alignment; not run */
  FA2_SITE_SELFTEST = 15
};

/*
 * fa2_selftest_timeout -- launch a one-warp kernel that waits on an mbarrier
 * nothing ever arrives on, with the given limit in nanoseconds (1 ms .. 4 s),
 * through the same bounded-wait routine the attention kernel uses.  The wait
 * runs out, the kernel records FA2_SITE_SELFTEST and returns; read it with
 * fa2_debug_status.  Exercises the failure path without faulting the GPU.
 */
int fa2_selftest_timeout(void* stream, long long limit_ns);

/*
 * Host-only planning helpers (no CUDA calls).
 *
 * fa2_num_blocks: thread blocks of a grid that runs over (query tile, head,
 * batch), ceil(N / rows_per_block) * H * B -- the sequence-parallel grid of
 * "FlashAttention 2: Three Places the Chip Was Still Waiting", section 2.3.
 * Returns -1 on non-positive arguments.
 *
 * fa2_launch_plan: the work decomposition fa2_forward uses for a problem:
 * the number of units (256 query rows of one head and batch each, one thread
 * block apiece when there are fewer than two units per SM; otherwise one
 * persistent block per SM takes whole units, see fa2_persistent_plan),
 * threads per block, dynamic shared memory bytes and query rows per unit.
 * Returns an fa2_status_code (validation as in fa2_forward, minus pointers).
 */
long long fa2_num_blocks(int B, int H, int N, int rows_per_block);
int fa2_launch_plan(int B, int Hq, int Hkv, int Nq, int Nk, int d, int* grid_blocks,
                    int* threads_per_block, int* smem_bytes, int* rows_per_block);

/*
 * fa2_persistent_plan: which units the persistent blocks of fa2_forward run,
 * in which order, on a GPU with num_sms SMs (fa2_forward uses it when the
 * problem has at least two units with a visible key per SM).  Units are
 * grouped by neighbouring (batch, head) pairs -- whole GQA groups, about one
 * wave of units per group -- heaviest first inside a group, and each goes to
 * the block with the least planned work (K/V tiles plus a fixed cost per
 * unit), so that the blocks running at any moment share a few heads' K and V
 * in L2 ("FlashAttention 2: Three Places the Chip Was Still Waiting",
 * section 2.3 for the units; the order is this library's).  The plan is a
 * kernel parameter: nothing is allocated.
 *
 *   start   num_sms + 1 ints (host): block c runs units[start[c] .. start[c+1])
 *   units   units_capacity ints (host): unit u = round * B * Hq + b * Hq + hq,
 *           round = query blocks counted from the last; u + 8192 (u + 16384)
 *           stands for the unit's first (second) 128-row query tile alone.
 *           When the units left after the full waves of num_sms would fill at
 *           most half the blocks, each of them is listed as its two halves,
 *           so twice as many blocks share the last wave
 *
 * Returns FA2_OK; FA2_ERR_SIZE when the problem has more than 8192 units with
 * a visible key, num_sms exceeds 160 (fa2_forward then deals units round
 * robin, heaviest first) or units_capacity is too small; FA2_ERR_NULL_POINTER
 * for missing arrays; otherwise fa2_forward's validation status.  No CUDA call.
 */
int fa2_persistent_plan(int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal, int num_sms,
                        int* start, int* units, int units_capacity);

/*
 * fa2_streamk_plan: the stream-K schedule fa2_forward_ws would use on a GPU
 * with num_sms SMs: total K/V-tile iterations over all units, persistent
 * blocks launched (min(num_sms, total); 0 when every unit is empty) and the
 * workspace bytes.  Any output pointer may be NULL.  Returns an
 * fa2_status_code (validation as in fa2_forward, minus pointers;
 * FA2_ERR_BAD_SHAPE for num_sms <= 0, FA2_ERR_SIZE as fa2_forward_ws).
 */
int fa2_streamk_plan(int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal, int num_sms,
                     long long* total_iters, int* ctas, long long* workspace_bytes);

/*
 * fa2_schedule_choice: the choice fa2_forward_auto makes on a GPU with
 * num_sms SMs -- *split = 1 for split-KV (fa2_forward_ws), 0 for whole units
 * -- and the two prices it compares, in K/V-tile iterations of the busiest
 * block (*cost_split includes the merge).  Any output pointer may be NULL.
 * Returns an fa2_status_code (validation as in fa2_forward, minus pointers;
 * FA2_ERR_BAD_SHAPE for num_sms <= 0).  No CUDA call.
 */
int fa2_schedule_choice(int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal, int num_sms,
                        int* split, long long* cost_units, long long* cost_split);

#ifdef __cplusplus
}
#endif

#endif /* FA2_H */
