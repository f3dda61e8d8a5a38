/*
 * moe_layout.h -- C ABI of the B200 (sm_100a) MoE token dispatch / combine
 * library, libmoe_layout.so.
 *
 * The path: a routing layout built from top-k expert ids and an
 * expert-to-partition placement map, a dispatch permute that gathers token
 * rows into partition- and expert-contiguous receive buffers (optionally one
 * copy per (token, partition) and optionally cast to FP8 e4m3 with one fp32
 * scale per 128 columns), and a combine that gate-weights and sums the top-k
 * expert outputs back into token order.  The E_part destination partitions of
 * an expert-parallel all-to-all are contiguous regions of one receive buffer
 * in this GPU's memory.
 *
 * Conventions shared by every entry point
 *   - Every pointer argument except `prob` and `lay` (host structs) is a
 *     DEVICE pointer, owned and allocated by the caller; nothing is allocated,
 *     freed or kept by the library.  Row buffers (x, y, recv_x, recv_scale,
 *     out, z) and the workspace must be 16-byte aligned, int32 arrays 4-byte
 *     aligned.
 *   - Calls are asynchronous on `stream` (NULL = legacy default stream) and
 *     never synchronise with the host or copy device data back to it.  Two
 *     calls on different streams that share an output race.
 *   - The return value reports what the host can see before the launch:
 *     MOE_OK, MOE_ERR_ARG (invalid sizes, null or misaligned pointers),
 *     MOE_ERR_WORKSPACE (workspace too small) or MOE_ERR_CUDA (a launch
 *     failed; nothing is retried).  Problems that only the data reveals are
 *     recorded in the device status word `lay->status` (MOE_STATUS_* bits);
 *     the kernels never trap or assert, and skip what they cannot process.
 *   - Row-major layouts throughout.  bf16 is IEEE binary32's upper half.
 */
#ifndef MOE_LAYOUT_H
#define MOE_LAYOUT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream. */
typedef struct CUstream_st *moe_stream_t;

/* return codes */
#define MOE_OK 0
#define MOE_ERR_ARG 1
#define MOE_ERR_WORKSPACE 2
#define MOE_ERR_CUDA 3

/* bits of the device status word (lay->status[0]) */
#define MOE_STATUS_BAD_EXPERT 1 /* a top-k id outside [0, G): that pair is left out   */
#define MOE_STATUS_BAD_PART 2   /* a placement entry outside [0, E_part): its expert's
                                   pairs are left out                                   */
#define MOE_STATUS_BAD_ROW 4    /* dispatch / combine met a row index outside the
                                   receive capacity M*topk: that copy / term skipped    */
#define MOE_STATUS_BAD_COUNT 8  /* moe_ep_plan: a count negative, an offset past
                                   INT32_MAX (written as -1) or expert counts that do
                                   not add up to the partition count                    */

/* limits checked by every entry point */
#define MOE_MAX_G 1024
#define MOE_MAX_E_PART 64
#define MOE_MAX_TOPK 32
#define MOE_MAX_N (1 << 24) /* columns: keeps every grid and in-row index in range */

/*
 * Problem sizes, as the all-to-all benchmark of the Triton-distributed issue
 * #117 ("All2all performance comparison between Triton-distributed and
 * DeepEP", Benchmark Configuration) poses them:
 *   M       tokens (>= 0; M = 0 makes every call a no-op)
 *   N       hidden size, bf16 columns (1..MOE_MAX_N, multiple of 8; of 128
 *           with fp8)
 *   G       experts (1..MOE_MAX_G)
 *   topk    experts per token (1..MOE_MAX_TOPK); M*topk < 2^31
 *   E_part  destination partitions (1..MOE_MAX_E_PART)
 *   dedup   0: one dispatch row per routed (token, expert) pair;
 *           1: one dispatch row per distinct (token, partition) pair
 *              ("each token is sent to a GPU only once regardless of how many
 *              of its experts reside there", Zyphra correlated expert
 *              placement news item)
 *   fp8     0: dispatch rows are bf16 copies; 1: e4m3 bytes plus one fp32
 *           scale per 128 columns (the WITH_SCALE / scale_src / scale_dst
 *           arguments of the issue #117 all_to_all_kernel)
 */
typedef struct moe_problem {
    int32_t M, N, G, topk, E_part;
    int32_t dedup, fp8;
} moe_problem_t;

/*
 * Layout arrays (device, int32, caller-allocated at worst-case capacity so
 * that no count has to travel back to the host):
 *   expert_count  [G]        routed pairs per expert
 *   expert_offset [G+1]      first expert row of each expert; [G] = R_exp.
 *                            The expert-row space orders the routed pairs by
 *                            (partition, expert id, token, slot), so each
 *                            partition's experts are contiguous and each
 *                            expert's rows are in token order; within a
 *                            partition the per-expert ends are the `offs`
 *                            a grouped GEMM consumes (DeepSpeed PR #8180,
 *                            "Add Triton grouped-GEMM for MoE experts").
 *   part_count    [E_part]   dispatch rows per partition
 *   part_offset   [E_part+1] first dispatch row of each partition; [E_part] =
 *                            R_disp.  This is the scattered-V receive layout
 *                            of Purlin section 3.1 ("Layouts"): contiguous,
 *                            variable-sized partitions indexed by destination.
 *   exp_row       [M*topk]   expert row of pair (t, k), -1 if left out
 *   disp_token    [M*topk]   token of each dispatch row (first R_disp used)
 *   disp_row      [M*E_part] dedup only: dispatch row of (t, p) or -1; rows
 *                            of a partition are in token order.  Ignored
 *                            (may be NULL) without dedup, where the dispatch
 *                            rows are the expert rows.
 *   exp_to_disp   [M*topk]   dedup only: dispatch row holding the token of
 *                            each expert row (first R_exp used); may be NULL
 *                            without dedup.
 *   status        [1]        MOE_STATUS_* bits; written by the layout
 *                            (moe_layout, moe_layout_static,
 *                            moe_layout_dispatch), OR-ed into by the calls
 *                            that read the layout afterwards.
 * Entries beyond R_exp / R_disp are left untouched.
 */
typedef struct moe_layout {
    int32_t *expert_count;
    int32_t *expert_offset;
    int32_t *part_count;
    int32_t *part_offset;
    int32_t *exp_row;
    int32_t *disp_token;
    int32_t *disp_row;
    int32_t *exp_to_disp;
    int32_t *status;
} moe_layout_t;

/* ABI version of this header (bumped on any incompatible change). */
#define MOE_ABI_VERSION 1
int moe_abi_version(void);

/* Human-readable text of a return code; never NULL. */
const char *moe_status_string(int code);

/*
 * Bytes of device workspace moe_layout needs for `prob` (0 if prob is
 * invalid).  The workspace holds per-tile expert / partition histograms; it
 * need not be zeroed and may be reused once the call has completed.
 */
size_t moe_layout_workspace_size(const moe_problem_t *prob);

/*
 * Routing layout.  Split counts and their prefix sums feed an all-to-all
 * (Triton-distributed issue #117 test snippet: split_send_buf and
 * send_split_cumsum); here they are built on the device together with the
 * row index of every routed pair.
 *   topk_idx  [M, topk] int32  expert ids
 *   part_of   [G] int32        placement map: partition of each expert
 *   lay                         output arrays (host struct of device pointers)
 *   workspace, workspace_bytes  >= moe_layout_workspace_size(prob), 16-B aligned
 * Deterministic: the same inputs give the same bits on every call.
 */
int moe_layout(const moe_problem_t *prob, const int32_t *topk_idx,
               const int32_t *part_of, const moe_layout_t *lay,
               void *workspace, size_t workspace_bytes, moe_stream_t stream);

/*
 * Routing layout that allocates nothing -- the same computation and outputs as
 * moe_layout, for callers that cannot allocate device memory where they route
 * tokens (code inside a CUDA-graph capture that must not call cudaMalloc,
 * runtimes whose memory planner hands out no scratch, C hosts without an
 * allocator).  The pages have no counterpart of this entry point.
 *   Scratch: a device array of MOE_STATIC_SCRATCH_BYTES compiled into the
 *   library, held by every GPU that loads it until the process exits.
 *   Limit: a problem whose moe_layout_workspace_size() exceeds
 *   MOE_STATIC_SCRATCH_BYTES is rejected with MOE_ERR_WORKSPACE before any
 *   launch.  The layout uses at most 148 tiles of G + 2 ints each, plus
 *   E_part more with dedup (padded to 4), so every M fits when
 *   G + (dedup ? E_part : 0) <= 438 (G = 256, E_part = 8 always fits);
 *   larger G fit only for small M.
 *   The first call in each CUDA context looks up the array's device address
 *   (one cudaGetSymbolAddress with the device current): the process's first
 *   call on a device, and the first call after that device's context was
 *   destroyed and re-created (cudaDeviceReset).  The address is remembered
 *   per context, never reused for another one.  Make such a first call
 *   before any stream capture.  Every call shares the array: calls whose
 *   execution overlaps on the GPU (other streams, other threads) race --
 *   serialise them.  Nothing in the array needs to start at zero.
 *   Other arguments, errors and results as moe_layout.
 */
#define MOE_STATIC_SCRATCH_BYTES (256 * 1024)
int moe_layout_static(const moe_problem_t *prob, const int32_t *topk_idx,
                      const int32_t *part_of, const moe_layout_t *lay,
                      moe_stream_t stream);

/*
 * Dispatch permute (issue #117 all_to_all_kernel: data_src -> data_dst with
 * optional scale_src -> scale_dst).  Each token row of x is read once and
 * written to every dispatch row that holds it.
 *   x           [M, N] bf16
 *   lay         a layout of the same problem (exp_row, or disp_row with dedup)
 *   recv_x      [M*topk, N] bf16 (fp8 = 0) or uint8 e4m3 (fp8 = 1); rows
 *               [0, R_disp) are written
 *   recv_scale  fp8 only: [M*topk, N/128] fp32; block b of row r holds
 *               scale = amax / 448 of x[t, 128b .. 128b+127] (0 for an
 *               all-zero block, whose bytes are then 0), and byte j holds
 *               e4m3(x / scale), nearest-even, saturating at +-448.
 *               May be NULL with fp8 = 0.
 */
int moe_dispatch(const moe_problem_t *prob, const void *x,
                 const moe_layout_t *lay, void *recv_x, float *recv_scale,
                 moe_stream_t stream);

/*
 * Combine: out[t, :] = bf16( sum_k w[t,k] * y[exp_row[t,k], :] ), one owner
 * per output element, fp32 fused multiply-adds in slot order k = 0..topk-1
 * starting from +0, one rounding to bf16 (the ordered, exclusively owned
 * reduction of Purlin section 3.3, "SCORE").  Left-out pairs (exp_row = -1)
 * contribute nothing.
 *   y             [M*topk, N] bf16 expert outputs in expert-row space
 *   topk_weights  [M, topk] fp32 gates
 *   out           [M, N] bf16
 */
int moe_combine(const moe_problem_t *prob, const void *y,
                const float *topk_weights, const moe_layout_t *lay, void *out,
                moe_stream_t stream);

/*
 * Grouped-GEMM tile metadata of a layout (DeepSpeed PR #8180, "Key points":
 * the per-tile -> group mapping of a grouped GEMM computed on the device
 * from offs, so no device -> host copy).  Tiles hold block_m rows and never
 * straddle two experts: expert e owns ceil(expert_count[e] / block_m)
 * tiles, numbered in row order.  All arrays are device int32, caller-owned:
 *   tile_first  [G+1]: first tile of expert e (also defined for experts
 *               without rows); tile_first[G] = number of tiles
 *   tile_expert [cap]: expert of tile i
 *   tile_row    [cap]: first expert row of tile i
 *   tile_rows   [cap]: rows of tile i, 1..block_m
 * cap = moe_expert_tiles_capacity(prob, block_m) = ceil(M*topk/block_m) + G,
 * the most a layout of this problem needs; entries past tile_first[G] are
 * untouched.  Requests with block_m < 1, null or misaligned arrays, or a
 * capacity of 2^31 entries or more are MOE_ERR_ARG.
 */
typedef struct {
  int32_t block_m;
  int32_t *tile_first;
  int32_t *tile_expert;
  int32_t *tile_row;
  int32_t *tile_rows;
} moe_tiles_t;

size_t moe_expert_tiles_capacity(const moe_problem_t *prob, int32_t block_m);

/*
 * Layout and dispatch in one call: the same results, bit for bit, as
 * moe_layout followed by moe_dispatch with the same arguments, and the same
 * argument rules and return codes as those two calls (workspace included).
 * Small batches -- 1 <= M*topk <= the library's fused limit (4096 routed
 * pairs by default), where both steps are bound by latency (Triton-
 * distributed issue #117, "Results (Latency in us)", M = 2..512) -- run as
 * ONE kernel in which every block rebuilds the small layout in shared
 * memory and dispatches its own chunk of tokens, with no inter-block wait;
 * larger batches run the two calls' kernels.  The workspace is left
 * untouched by the one-kernel schedule.
 * tiles (NULL: none) also fills the grouped-GEMM tile metadata, from inside
 * the same kernels (no extra launch); the results equal moe_expert_tiles'.
 */
int moe_layout_dispatch(const moe_problem_t *prob, const int32_t *topk_idx,
                        const int32_t *part_of, const moe_layout_t *lay,
                        void *workspace, size_t workspace_bytes, const void *x,
                        void *recv_x, float *recv_scale, const moe_tiles_t *tiles,
                        moe_stream_t stream);

/* 1 if moe_layout_dispatch takes the one-kernel schedule for `prob`, else 0
 * (also 0 for an invalid problem). */
int moe_layout_dispatch_fused(const moe_problem_t *prob);

/*
 * The tile metadata (moe_tiles_t above) of a finished layout, as a kernel of
 * its own: for callers of moe_layout or moe_layout_static.  Call after the
 * layout on the same stream, with the same part_of.  Counts that cannot
 * come from a layout of this problem (more tiles than the capacity) write
 * only the capacity's tiles and raise MOE_STATUS_BAD_ROW.
 */
int moe_expert_tiles(const moe_problem_t *prob, const int32_t *part_of,
                     const moe_layout_t *lay, const moe_tiles_t *tiles,
                     moe_stream_t stream);

/*
 * Two-level combine of a deduplicated dispatch (prob->dedup = 1, else
 * MOE_ERR_ARG): the return path of per-partition dedup, where each
 * partition first reduces the outputs of a token's experts it holds and the
 * token then sums its partitions (Zyphra news item, correlated expert
 * placement: one copy of a token per GPU each way; Purlin section 3.3,
 * SCORE: one owner per output element, source-order accumulation).
 * Results differ from moe_combine by the extra bf16 rounding of each
 * partition's partial sum.
 *
 * moe_combine_partial -- partition side:
 *   z[disp_row[t,p], :] = bf16( sum over slots k of t whose expert is on
 *                         partition p, in slot order, of w[t,k] *
 *                         y[exp_row[t,k], :] )   (fp32 fma from +0)
 *   y             [M*topk, N] bf16 expert outputs in expert-row space
 *   topk_weights  [M, topk] fp32
 *   z             [M*topk, N] bf16 in dispatch-row space; rows [0, R_disp)
 *                 are written (the payload that returns to the tokens)
 * moe_combine_reduce -- token side:
 *   out[t, :] = bf16( sum over p = 0..E_part-1 with disp_row[t,p] >= 0 of
 *               z[disp_row[t,p], :] )   (fp32 additions from +0)
 *   out           [M, N] bf16
 * Both are asynchronous on `stream`; run moe_combine_partial before
 * moe_combine_reduce on one stream (or order them with an event).  z is the
 * caller's buffer, 16-byte aligned like y and out.  Row indices outside
 * [0, M*topk) in exp_row, exp_to_disp or disp_row are skipped and raise
 * MOE_STATUS_BAD_ROW in lay->status; the calls never trap.
 */
int moe_combine_partial(const moe_problem_t *prob, const void *y,
                        const float *topk_weights, const moe_layout_t *lay,
                        void *z, moe_stream_t stream);
int moe_combine_reduce(const moe_problem_t *prob, const void *z,
                       const moe_layout_t *lay, void *out, moe_stream_t stream);

/*
 * Expert-parallel exchange plan.  With the partitions on W ranks (E_part = W,
 * partition p = rank p), each rank's layout counts what it sends to every
 * rank; an all-gather of those counts (the split_send_buf -> split_recv_buf
 * exchange and send_split_cumsum of the Triton-distributed issue #117
 * all-to-all) gives every rank the matrix P[s][d] of the rows source s sends
 * to destination d.  This call turns that matrix into rank r's offsets for the
 * data exchange into Purlin's transposed-V layout (section 3.1: destination r
 * holds partition r of every source, in source-rank order):
 *   world, rank    W (1..MOE_MAX_E_PART) and r (0..W-1)
 *   part_counts    [W][W] int32, row s = the part_count of rank s's layout
 *   expert_counts  [W][G] int32, row s = the expert_count of rank s's layout,
 *                  or NULL.  Only without dedup, where dispatch rows are
 *                  expert rows.
 *   part_of        [G] int32 placement (expert -> rank); with expert_counts
 *   G              experts (1..MOE_MAX_G); ignored without expert_counts
 *   plan           device arrays, caller-allocated:
 *     send_offset  [W]    sum_{s<r} P[s][d]: where r's rows for d start in d's
 *                         receive buffer (a push, by peer stores)
 *     src_offset   [W]    sum_{d<r} P[s][d]: where s's rows for r start in s's
 *                         dispatch buffer (a pull, by peer loads)
 *     recv_count   [W]    P[s][r]
 *     recv_offset  [W+1]  sum_{s'<s} P[s'][r]: where s's rows land in r's
 *                         receive buffer; [W] = rows r receives
 *     recv_expert_count [G]    (with expert_counts) rows r receives per expert:
 *                              sum_s X[s][e] for the experts on r, else 0
 *     recv_block_offset [W][G] (with expert_counts) first row of the block of
 *                              source s's rows of expert e in r's receive
 *                              buffer, for the experts on r (-1 elsewhere):
 *                              recv_offset[s] + sum of X[s][f] over the experts
 *                              f < e on r.  The (source, expert) blocks a
 *                              grouped GEMM over the receive buffer consumes.
 *     status       [1]    0 or MOE_STATUS_BAD_COUNT
 * Sums are exact in 64 bits; an offset past INT32_MAX is written as -1 and
 * flagged.  One small kernel on `stream`; it reads only the given arrays.
 * MOE_ERR_ARG for world, rank or G out of range and null or misaligned arrays.
 * The data exchange itself (peer stores or loads over NVLink, or an NCCL
 * all-to-all with these counts) is the caller's.
 */
typedef struct moe_ep_plan {
    int32_t *send_offset;
    int32_t *src_offset;
    int32_t *recv_count;
    int32_t *recv_offset;
    int32_t *recv_expert_count;
    int32_t *recv_block_offset;
    int32_t *status;
} moe_ep_plan_t;

int moe_ep_plan(int32_t world, int32_t rank, int32_t G, const int32_t *part_counts,
                const int32_t *expert_counts, const int32_t *part_of,
                const moe_ep_plan_t *plan, moe_stream_t stream);

/*
 * Expert-parallel data plane: the dispatch and the combine with partition p
 * on rank p (E_part = W ranks), each rank's buffers addressed through a
 * device array of pointers -- peer mappings over NVLink (cudaIpc handles,
 * symmetric memory), or plain local buffers when the ranks share one GPU.
 * Rank r's dispatch rows of partition p (rows [part_offset[p],
 * part_offset[p+1]) of its layout) occupy rows [send_offset[p],
 * send_offset[p] + count) of rank p's receive buffer, in the same order:
 * Purlin's transposed-V layout (section 3.1), with send_offset from rank r's
 * moe_ep_plan.  Dispatch row r of partition p therefore lives at row
 * send_offset[p] + r - part_offset[p] of rank p's buffers, and the outputs
 * rank p computes in its receive order come back from the same row.
 *   rows       [W] device array of device pointers, one per rank, each
 *              16-byte aligned
 *   scales     [W] device array of device pointers to fp32 scale buffers
 *              (moe_ep_dispatch with fp8), else ignored; 4-byte aligned
 *   capacity   rows each rank's buffer holds; rows at or past it are never
 *              touched
 * A row outside a rank's capacity or its partition, or a null or misaligned
 * pointer in the array, is skipped and raises MOE_STATUS_BAD_ROW in
 * lay->status.  The kernels never wait on another rank: the caller orders
 * the steps (every rank's dispatch complete before any destination reads
 * its receive buffer; every destination's outputs complete before any
 * combine), e.g. with a barrier or an NCCL collective between them.
 */
typedef struct moe_ep_peers {
    void *const *rows;
    float *const *scales;
    int32_t capacity;
} moe_ep_peers_t;

/*
 * Push dispatch (Purlin section 3.2: push in the latency path; issue #117
 * all_to_all_kernel data_src -> data_dst, scale_src -> scale_dst): each
 * token row of x is read once and stored into every destination rank's
 * receive buffer (peers->rows), bf16 or, with fp8, e4m3 bytes plus one
 * scale per 128 columns into peers->scales.  The bytes of every row equal
 * those moe_dispatch writes.  x, lay and the argument rules as moe_dispatch;
 * send_offset [E_part] int32 (device) from moe_ep_plan.
 */
int moe_ep_dispatch(const moe_problem_t *prob, const void *x, const moe_layout_t *lay,
                    const int32_t *send_offset, const moe_ep_peers_t *peers,
                    moe_stream_t stream);

/*
 * Pull combine (prob->dedup = 0): out[t, :] = bf16( sum_k w[t,k] *
 * y[rank p(k)][send_offset[p] + exp_row[t,k] - part_offset[p], :] ), fp32
 * fused multiply-adds in slot order from +0 (Purlin section 3.3, SCORE), with
 * y the ranks' expert-output buffers (y_peers->rows, bf16, rows in each
 * rank's receive order).  Equal to moe_combine over the gathered rows.
 */
int moe_ep_combine(const moe_problem_t *prob, const moe_ep_peers_t *y_peers,
                   const float *topk_weights, const moe_layout_t *lay,
                   const int32_t *send_offset, void *out, moe_stream_t stream);

/*
 * Pull token-side sum of the two-level combine (prob->dedup = 1): out[t, :] =
 * bf16( sum over p with disp_row[t,p] >= 0, in partition order, of
 * z[rank p][send_offset[p] + disp_row[t,p] - part_offset[p], :] ), fp32 from
 * +0, with z the ranks' partition-side rows (z_peers->rows, bf16, each rank's
 * receive order).  Equal to moe_combine_reduce over the gathered rows.
 */
int moe_ep_combine_reduce(const moe_problem_t *prob, const moe_ep_peers_t *z_peers,
                          const moe_layout_t *lay, const int32_t *send_offset, void *out,
                          moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_LAYOUT_H */
