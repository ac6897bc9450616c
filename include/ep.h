/*
 * ep.h -- C ABI of the single-GPU MoE expert-parallel permutation engine.
 *
 * The engine runs the three data-parallel steps that surround the expert
 * GEMM of a Mixture-of-Experts layer, with the expert-parallel ranks modelled
 * as R virtual partitions of one GPU's memory:
 *
 *   ep_layout    routing metadata: per-expert and per-rank counts, padded
 *                expert-major offsets, is_token_in_rank, and the receive row
 *                of every (token, top-k slot);
 *   ep_dispatch  scatter of each token's hidden row into the expert-major
 *                receive buffer, as BF16 or as FP8 e4m3 with one fp32 scale
 *                per 128 channels;
 *   ep_combine   gather of the k expert outputs of each token, reduced with
 *                the routing weights in fp32, back into token order.
 *
 * Around them: ep_layout_dispatch (layout and dispatch in one launch for
 * decode-sized batches), token-range forms (ep_dispatch_range /
 * ep_combine_range), FP16 rows (EP_FMT_FP16, ep_dispatch_ex, ep_combine_ex),
 * the expert-parallel form with one receive buffer per rank
 * (ep_dispatch_ranks / ep_combine_ranks), GEMM-ready helpers (MN-major FP8
 * scales, ep_dispatch_weights, ep_zero_pad_rows), the backward of dispatch
 * and combine, and a layout entry point that needs no workspace
 * (ep_layout_static_scratch).
 *
 * Source of the operations.  "DeepEP是什麼？MoE Dispatch、Combine、
 * All-to-all與V2架構" (yololab.net), stage table of the section
 * "MoE為什麼需要All-to-all": dispatch takes tokens, top-k indices and weights
 * and yields hidden states arranged by expert; combine takes the expert
 * outputs and routing weights and yields results in the original token order.
 * The same page's ElasticBuffer section has the buffer own the "dispatch
 * layout" and be sized from max tokens, top-k, hidden and EP degree; the
 * DeepEP v2 release notes (donniechu.com, "Có gì mới trong v2") pair the
 * buffer with an EPHandle that carries dispatch state into combine.  Here the
 * caller owns every buffer, and the opaque ep_handle_t carries the layout.
 *
 * Layout rules (the pages name a "GEMM layout" without defining it; this is
 * the reading taken): expert e belongs to rank floor(e / (E/R)); one flat
 * receive buffer holds experts in index order; expert e's block starts at
 * expert_off[e] and is padded up to a multiple of block_m rows; inside a
 * block, rows are in (source token, slot) order; rank r's receive buffer is
 * rows [rank_off[r], rank_off[r+1]).  Pad rows are never written.
 *
 * Conventions.  All tensors are dense row-major.  "device" pointers must be
 * addresses of the current CUDA device's global memory; "host" pointers are
 * ordinary CPU memory.  Every call that takes a stream enqueues its work on
 * that stream (a cudaStream_t passed as void*, NULL = legacy default stream)
 * and returns without waiting, except the ones documented as synchronising.
 * The library never allocates device memory; the handle itself is a small
 * host allocation made by ep_handle_create.
 *
 * Buffer sizes.  The library sees a buffer's pointer and the row count
 * (capacity) passed with it, never the allocation: every write is bounded by
 * the capacities given, so each buffer must hold at least the rows and the
 * row width its documented shape implies for that capacity (an FP8 row is H
 * bytes, a BF16/FP16 row 2H; row-major scales [capacity][H/128] fp32; MN-major
 * [H/128][capacity]).  A smaller buffer, or a host pointer where a device one
 * is asked for, is outside this contract and the GPU faults.  The Python
 * binding checks type, shape and device of every tensor before the call.
 *
 * Errors.  Argument problems that the host can see are returned at once and
 * nothing is enqueued.  Problems only the GPU can see (an index outside
 * [-1, E), a receive row beyond the capacity given) set bits in a sticky
 * device error word inside the workspace; the offending rows are skipped,
 * nothing out of bounds is touched, and ep_handle_check reports them.  No
 * kernel traps.  The one device-side wait -- the grid barrier between the
 * phases of the single-launch layout, whose CTAs are co-resident by a
 * cooperative launch -- has an iteration limit and reports EP_ERR_TIMEOUT.
 *
 * Thread safety: calls on one handle must not run concurrently from several
 * host threads; distinct handles are independent.
 */
#ifndef EP_H_
#define EP_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct ep_handle_s* ep_handle_t;

typedef enum {
    EP_OK = 0,
    EP_ERR_INVALID_ARG = 1,          /* bad size, null pointer, unsupported shape */
    EP_ERR_ALIGNMENT = 2,            /* a pointer misses its required alignment */
    EP_ERR_WORKSPACE_TOO_SMALL = 3,  /* workspace_bytes < ep_workspace_bytes(...) */
    EP_ERR_CAPACITY = 4,             /* a receive row did not fit the buffer given */
    EP_ERR_BAD_INDEX = 5,            /* a top-k index outside [-1, E) */
    EP_ERR_CUDA = 6,                 /* a CUDA runtime call failed; see ep_last_error_message */
    EP_ERR_STATE = 7,                /* e.g. dispatch/combine before any ep_layout */
    EP_ERR_NO_MEMORY = 8,            /* host malloc of the handle failed */
    EP_ERR_TIMEOUT = 9               /* a device-side wait (the layout's grid barrier) gave up
                                        after its iteration limit; that call's outputs are
                                        invalid.  Reported by ep_handle_check, which also
                                        resets the barrier. */
} ep_status_t;

/* Element type of 16-bit hidden rows (x, y, out).  The yololab page lists
 * BF16, FP16 and FP8 as the precisions a deployment should test
 * ("DeepEP是什麼？…", section Benchmark矩陣); its FP8與低精度通訊 section
 * covers the FP8 form. */
typedef enum {
    EP_DTYPE_BF16 = 0,            /* bfloat16 */
    EP_DTYPE_FP16 = 1             /* IEEE-754 binary16 */
} ep_dtype_t;

typedef enum {
    EP_FMT_BF16 = 0,              /* receive rows are the bf16 input rows */
    EP_FMT_FP8_E4M3_1X128 = 1,    /* e4m3 rows + one fp32 scale per 128 channels,
                                     scales row-major [rows][H/128] */
    EP_FMT_FP8_E4M3_1X128_MN = 2, /* the same codes and scales, scales MN-major
                                     [H/128][recv_capacity_rows]: each block's scales
                                     contiguous over rows (recv_capacity_rows % 4 == 0,
                                     so every block's column starts 16-byte aligned) */
    EP_FMT_FP16 = 3               /* receive rows are the fp16 input rows */
} ep_fmt_t;

/* Most ranks a per-rank buffer table of ep_dispatch_ranks / ep_combine_ranks
 * may have. */
#define EP_MAX_RANK_TABLE 64

/* Views of the layout held in the workspace (see ep_handle_view). */
typedef enum {
    EP_VIEW_NUM_TOKENS_PER_EXPERT = 0, /* int32 [E]     slots routed to each expert */
    EP_VIEW_NUM_TOKENS_PER_RANK = 1,   /* int32 [R]     tokens with >= 1 slot on rank r */
    EP_VIEW_NUM_ROWS_PER_RANK = 2,     /* int32 [R]     non-pad receive rows of rank r */
    EP_VIEW_EXPERT_OFFSET = 3,         /* int32 [E+1]   padded block starts; [E] = P */
    EP_VIEW_RANK_OFFSET = 4,           /* int32 [R+1]   rank r owns rows [off[r], off[r+1]) */
    EP_VIEW_IS_TOKEN_IN_RANK = 5,      /* uint8 [T][R]  1 if token t sends to rank r */
    EP_VIEW_DST_ROW = 6,               /* int32 [T][k]  receive row of slot (t,j), -1 unused */
    EP_VIEW_RECV_SRC = 7,              /* int32 [P]     source token of each row, -1 on pad */
    EP_VIEW_TOTAL_RECV_ROWS = 8,       /* int32 [1]     P, the padded receive rows */
    EP_VIEW_ERROR_WORDS = 9            /* int32 [3]     diagnostics: the sticky error bits,
                                          then the layout grid barrier's count and
                                          generation (do not write while work is queued) */
} ep_view_t;

/* Limits of this build. */
#define EP_MAX_TOPK 32
#define EP_MAX_EXPERTS 8192
#define EP_MAX_BLOCK_M 4096

/* Bytes of device workspace a handle needs for up to max_tokens tokens
 * (host; pure arithmetic).  Returns 0 if the arguments are invalid:
 * max_tokens >= 0, 1 <= num_topk <= EP_MAX_TOPK,
 * 1 <= num_experts <= EP_MAX_EXPERTS, 1 <= num_ranks, num_experts % num_ranks
 * == 0, 1 <= block_m <= EP_MAX_BLOCK_M, and every row count below 2^31.
 * The pages size the buffer from max tokens, top-k, hidden size and EP degree
 * ("DeepEP是什麼？…", section ElasticBuffer); here the hidden rows live in the
 * caller's buffers, so the workspace holds only the layout and is sized from
 * the same quantities less the hidden size. */
size_t ep_workspace_bytes(int max_tokens, int num_topk, int num_experts, int num_ranks,
                          int block_m);

/* Upper bound on the padded receive rows P for T tokens (host, no sync):
 * T*k + min(E, T*k)*(block_m - 1), rounded down to a multiple of block_m.
 * Sizing recv buffers with it lets a whole step run without reading P back,
 * e.g. inside a CUDA graph.  Returns -1 for invalid arguments.  This is the
 * capacity headroom for uneven routing that the same ElasticBuffer section
 * asks for, taken at its worst case (every used expert one row short of a
 * full block). */
int64_t ep_recv_rows_upper_bound(int T, int num_topk, int num_experts, int block_m);

/* Create a handle over a caller-owned device workspace (host; makes no CUDA
 * call).  workspace: device pointer, 256-byte aligned, at least
 * ep_workspace_bytes(...) bytes, owned by the caller and kept alive, and not
 * used for anything else, until ep_handle_destroy.  On success *out receives
 * the handle; on failure *out is set to NULL.  The handle plays the part of
 * the pages' EPHandle, which carries dispatch state into combine (DeepEP v2
 * release notes, section Có gì mới trong v2). */
ep_status_t ep_handle_create(void* workspace, size_t workspace_bytes, int max_tokens,
                             int num_topk, int num_experts, int num_ranks, int block_m,
                             ep_handle_t* out);

/* Free the host-side handle (not the workspace).  NULL is ignored.  Work
 * already enqueued that uses the workspace is unaffected. */
void ep_handle_destroy(ep_handle_t h);

/* Dispatch layout (get_dispatch_layout).  topk_idx: device int64 [T][k],
 * 8-byte aligned (may be NULL when T == 0); each value is an expert in
 * [0, E) or -1 for an unused slot.  0 <= T <= max_tokens.  Fills every view
 * of ep_view_t.  The layout stays valid, and is what ep_dispatch and
 * ep_combine use, until the next ep_layout on this handle.  An index outside
 * [-1, E) sets EP_ERR_BAD_INDEX in the sticky error word and is treated as -1.
 * Source: the pages' ElasticBuffer manages a "dispatch layout" ("DeepEP是什麼？
 * …", section ElasticBuffer); the same page's stage table (section
 * MoE為什麼需要All-to-all) has dispatch turn tokens and top-k indices into
 * hidden states arranged by expert, with sorting and imbalance as its cost,
 * and its Load Imbalance section lists per-expert token counts and per-rank
 * traffic as the figures to watch.  The exact layout rules (expert-major,
 * block_m padding, (token, slot) order) are the reading stated at the top of
 * this header. */
ep_status_t ep_layout(ep_handle_t h, const int64_t* topk_idx, int T, void* stream);

/* Layout followed by dispatch, the low-latency path for decode-sized batches
 * (the pages' low-latency mode serves decode and small batches, where launch
 * latency matters most: "DeepEP是什麼？…", section 高吞吐與低延遲工作負載).
 * Same arguments, results and errors as ep_layout(h, topk_idx, T, stream)
 * followed by ep_dispatch(h, x, H, fmt, recv_x, recv_scales,
 * recv_capacity_rows, stream) (so x is bf16, or fp16 with EP_FMT_FP16).
 * When the batch is small (T*k <= 4096, E <= 1024, T*R <= 65536, and the
 * per-CTA count tables fit 200 KB of shared memory) and rows take 32-byte
 * vectors (H % 16 == 0; x, and for a row copy recv_x, 32-byte aligned),
 * both run in ONE launch: every CTA
 * computes the same layout in its shared memory, CTA 0 publishes it, and all
 * CTAs dispatch from their own copy -- no grid-wide wait.  Otherwise the two
 * launches of the separate calls run.  All arguments are checked before
 * anything is enqueued. */
ep_status_t ep_layout_dispatch(ep_handle_t h, const int64_t* topk_idx, int T, const void* x, int H,
                               ep_fmt_t fmt, void* recv_x, float* recv_scales,
                               int64_t recv_capacity_rows, void* stream);

/* Device pointer of a layout view inside the workspace (host; no CUDA call);
 * *count (if not NULL) receives its number of elements for the last layout
 * (P for EP_VIEW_RECV_SRC is only known on the device, so its count is the
 * capacity reserved for max_tokens).  Returns NULL for an unknown view. */
const void* ep_handle_view(ep_handle_t h, ep_view_t what, int64_t* count);

/* Copy the counts of the last layout to host memory and wait for the stream
 * (SYNCHRONISING).  Any output pointer may be NULL.  num_tokens_per_expert:
 * int32 [E]; num_tokens_per_rank: int32 [R]; num_rows_per_rank: int32 [R];
 * total_recv_rows: int32 [1] (P).  These are the per-expert token counts and
 * per-rank volumes that "DeepEP是什麼？…", section Load Imbalance, names as the
 * signs of a hot expert or a straggling rank. */
ep_status_t ep_handle_read_counts(ep_handle_t h, int32_t* num_tokens_per_expert,
                                  int32_t* num_tokens_per_rank, int32_t* num_rows_per_rank,
                                  int32_t* total_recv_rows, void* stream);

/* Dispatch the T tokens of the last layout.
 * x: device bf16 [T][H] (fp16 with EP_FMT_FP16), 16-byte aligned.
 * EP_FMT_BF16 / EP_FMT_FP16: H % 8 == 0; recv_x: device rows of x's type
 *   [recv_capacity_rows][H], 16-byte aligned; recv_scales ignored.
 *   recv_x[dst_row[t][j]] = x[t].
 * EP_FMT_FP8_E4M3_1X128: H % 128 == 0; recv_x: device e4m3 bytes
 *   [recv_capacity_rows][H], 16-byte aligned; recv_scales: device fp32
 *   [recv_capacity_rows][H/128], 16-byte aligned.  For every token and every
 *   block b of 128 channels: amax = max |x|, s = amax / 448 (fp32 division),
 *   q = e4m3(x / s) (fp32 division, round to nearest even, saturate to
 *   +-448); amax == 0 gives s = 0 and q = 0.  Written to every dst row.
 *   This is the reading taken of the FP8 section of the yololab page, which
 *   asks to confirm scale granularity and format without fixing them.
 * EP_FMT_FP8_E4M3_1X128_MN: the same codes and scales; recv_scales is
 *   MN-major, fp32 [H/128][recv_capacity_rows] (scale of row r, block b at
 *   b * recv_capacity_rows + r), recv_capacity_rows % 4 == 0.
 * Only the rows listed in dst_row are written; pad rows keep their contents.
 * A row >= recv_capacity_rows is skipped and sets EP_ERR_CAPACITY.
 * Source of the operation: the Dispatch row of the stage table in
 * "DeepEP是什麼？…", section MoE為什麼需要All-to-all (tokens and top-k indices
 * in, hidden states arranged by expert out); its bytes, T k H sizeof(dtype),
 * are those of "DeepEP 编址服务深度对抗分析", section 五.2. */
ep_status_t ep_dispatch(ep_handle_t h, const void* x, int H, ep_fmt_t fmt, void* recv_x,
                        float* recv_scales, int64_t recv_capacity_rows, void* stream);

/* ep_dispatch with the type of x named.  x_dtype EP_DTYPE_BF16: as
 * ep_dispatch.  x_dtype EP_DTYPE_FP16: x is device binary16 [T][H];
 * fmt EP_FMT_FP16 copies the rows (recv_x binary16 [recv_capacity_rows][H]);
 * the FP8 formats quantise the binary16 values, widened exactly to fp32, with
 * the same amax, scale and rounding as above.  A copy format must match
 * x_dtype (EP_FMT_BF16 with bf16, EP_FMT_FP16 with fp16), else
 * EP_ERR_INVALID_ARG.  ep_dispatch itself takes fp16 rows only with
 * EP_FMT_FP16.  FP16 is one of the precisions (BF16, FP16, FP8) the yololab
 * page's Benchmark矩陣 section asks a deployment to cover. */
ep_status_t ep_dispatch_ex(ep_handle_t h, const void* x, ep_dtype_t x_dtype, int H, ep_fmt_t fmt,
                           void* recv_x, float* recv_scales, int64_t recv_capacity_rows,
                           void* stream);

/* Combine into token order for the T tokens of the last layout.
 * y: device bf16 [y_rows][H] in the receive layout, 16-byte aligned, H % 8 == 0.
 * topk_weights: device fp32 [T][k], 4-byte aligned.
 * out: device bf16 [T][H], 16-byte aligned, must not overlap y.
 * out[t][h] = bf16_rn(acc), acc = 0 then, for j = 0..k-1 over the used
 * slots, acc = fma(w[t][j], y[dst_row[t][j]][h], acc) in fp32.  Weights are
 * used as given (no renormalisation); unused slots (-1) are skipped.
 * A row >= y_rows is skipped and sets EP_ERR_CAPACITY.
 * Source: the Combine row of the stage table in "DeepEP是什麼？…", section
 * MoE為什麼需要All-to-all (expert outputs and routing weights in, results in
 * the original token order out, by a reverse exchange and a reduction).  The
 * pages leave the reduction's arithmetic open; the fp32 chain in slot order
 * above is the reading taken. */
ep_status_t ep_combine(ep_handle_t h, const void* y, int64_t y_rows, const float* topk_weights,
                       int H, void* out, void* stream);

/* ep_combine with the type of y and out named: EP_DTYPE_BF16 is ep_combine;
 * EP_DTYPE_FP16 reads binary16 expert outputs (widened exactly), accumulates
 * in fp32 in the same order and rounds the result to nearest even binary16
 * (sums beyond the binary16 range become infinities).  Precisions: the yololab
 * page's Benchmark矩陣 section (BF16, FP16, FP8). */
ep_status_t ep_combine_ex(ep_handle_t h, const void* y, int64_t y_rows, const float* topk_weights,
                          int H, ep_dtype_t dtype, void* out, void* stream);

/* Dispatch / combine a contiguous range of the last layout's tokens,
 * [t_begin, t_begin + t_count), 0 <= t_begin <= t_begin + t_count <= T.
 * Same semantics, formats and errors as ep_dispatch / ep_combine restricted
 * to those tokens; x_rows, topk_weights_rows and out_rows point at the rows
 * of token t_begin (x_rows: bf16 [t_count][H], or fp16 with EP_FMT_FP16;
 * topk_weights_rows: fp32 [t_count][k]; out_rows: bf16 [t_count][H]).  recv_x, recv_scales and y are
 * the whole receive-layout buffers.  The ranges of one layout may run in any
 * order and on different streams: they write disjoint rows.  This lets a
 * caller overlap the transfer of token chunks (host copies, or an upstream
 * producer) with dispatch and combine of the chunks already present, the
 * pipelining of communication with computation that "DeepEP：让大模型「专家们」
 * 高效协作的通信高速公路" (section 技术架构：从NVSHMEM到NCCL Gin的演进) gives as
 * the aim of the V2 buffer interface. */
ep_status_t ep_dispatch_range(ep_handle_t h, int t_begin, int t_count, const void* x_rows, int H,
                              ep_fmt_t fmt, void* recv_x, float* recv_scales,
                              int64_t recv_capacity_rows, void* stream);
ep_status_t ep_combine_range(ep_handle_t h, int t_begin, int t_count, const void* y,
                             int64_t y_rows, const float* topk_weights_rows, int H,
                             void* out_rows, void* stream);

/* Expert-parallel form: one receive buffer per rank.
 *
 * The pages describe dispatch as an all-to-all that sends each token's row
 * to the GPUs holding its experts and combine as the reverse exchange plus
 * the weighted reduction ("DeepEP是什麼？…", section MoE為什麼需要All-to-all);
 * rank p holds experts [p E/R, (p+1) E/R).  With the top-k indices of all
 * ranks gathered in rank order (T = the sum of the ranks' token counts), the
 * layout of ep_layout over the concatenated tokens is the expert-parallel
 * layout: rank p's receive buffer is rows [rank_off[p], rank_off[p+1]) of it,
 * renumbered from 0, so row d of the layout is row d - rank_off[p] of rank
 * p's buffer.  These calls take that global layout and a table of the R
 * ranks' buffers -- on R GPUs each entry is a peer pointer (the writes and
 * reads are plain stores and loads; no TMA, no multicast) -- and move the
 * rows of the source's own tokens [t_begin, t_begin + t_count) of the global
 * order.  Semantics, arithmetic and errors are those of ep_dispatch_range /
 * ep_combine_range restricted to a rank's block and renumbered.
 *
 * ep_dispatch_ranks: x_rows device [t_count][H] (bf16, or fp16 with
 *   EP_FMT_FP16), 32-byte aligned, H % 16 == 0.  fmt EP_FMT_BF16 /
 *   EP_FMT_FP16 (row copy) or EP_FMT_FP8_E4M3_1X128 (bf16 rows; row-major
 *   scales).  recv_x: HOST array of R device pointers, rank p's receive
 *   buffer [recv_rows[p]][H] of the row type (copy: 32-byte aligned) or of
 *   e4m3 bytes (FP8: 16-byte aligned); recv_scales (FP8 only): HOST array of
 *   R device pointers to fp32 [recv_rows[p]][H/128], 4-byte aligned;
 *   recv_rows: HOST array of R capacities.  R = the handle's rank count,
 *   at most EP_MAX_RANK_TABLE.  A row past its rank's capacity is skipped and
 *   sets EP_ERR_CAPACITY.
 * ep_combine_ranks: y: HOST array of R device pointers, rank p's expert
 *   outputs [y_rows[p]][H] (bf16 or fp16 as dtype), 16-byte aligned, H % 8 ==
 *   0; topk_weights_rows device fp32 [t_count][k]; out_rows device [t_count][H]
 *   of dtype.  out[t] = rn16(fma chain over the used slots, j = 0..k-1). */
ep_status_t ep_dispatch_ranks(ep_handle_t h, int t_begin, int t_count, const void* x_rows, int H,
                              ep_fmt_t fmt, void* const* recv_x, float* const* recv_scales,
                              const int64_t* recv_rows, void* stream);
ep_status_t ep_combine_ranks(ep_handle_t h, int t_begin, int t_count, const void* const* y,
                             const int64_t* y_rows, const float* topk_weights_rows, int H,
                             ep_dtype_t dtype, void* out_rows, void* stream);

/* Mapping another process's buffer into this one (CUDA IPC), to fill the
 * rank tables above when the ranks are separate processes (one per GPU, or
 * several on one GPU).  The owner calls ep_ipc_export on a buffer; the
 * handle bytes and the offset travel to the other ranks by any means (the
 * Python binding all-gathers them over the process group); each of them
 * calls ep_ipc_open and puts *ptr into its table.  Host-side ordering is the
 * caller's: the writes of every rank's ep_dispatch_ranks must be finished
 * (stream synchronised, then a barrier across the ranks) before any rank
 * reads its receive buffer, and likewise around the expert outputs that
 * ep_combine_ranks reads.  The pages' dispatch and combine are this
 * exchange between GPUs ("DeepEP是什麼？…", section MoE為什麼需要All-to-all).
 *
 * ep_ipc_export: ptr is a device pointer inside an allocation made with
 *   cudaMalloc (not a pool or virtual-memory allocation); handle receives
 *   EP_IPC_HANDLE_BYTES bytes (host), *offset (host) the distance of ptr
 *   from the start of its allocation.  A pointer outside any device
 *   allocation returns EP_ERR_INVALID_ARG.
 * ep_ipc_open: opens a handle exported by another process (CUDA allows no
 *   process to open its own); *base (host) receives the mapping of the
 *   whole allocation, to be passed to ep_ipc_close, and *ptr (host) = base +
 *   offset.  One handle is opened once per process; buffers that share an
 *   allocation share its mapping.
 * ep_ipc_close: unmaps a base returned by ep_ipc_open.
 * CUDA failures return EP_ERR_CUDA with the message in
 * ep_last_error_message.  These calls enqueue nothing. */
#define EP_IPC_HANDLE_BYTES 64
ep_status_t ep_ipc_export(const void* ptr, void* handle, uint64_t* offset);
ep_status_t ep_ipc_open(const void* handle, uint64_t offset, void** base, void** ptr);
ep_status_t ep_ipc_close(void* base);

/* Backward of the two calls above, for the source's tokens [t_begin,
 * t_begin + t_count) of the global layout (rows bf16 or fp16 as dtype).
 * ep_dispatch_ranks_backward: grad_x_rows[t] = the fp32 sum, in slot order,
 *   of the slot rows of the ranks' gradient buffers grad_recv[p] (HOST table
 *   of R device pointers, 16-byte aligned, grad_rows[p] rows), rounded to
 *   dtype -- ep_combine_ranks with unit weights.  H % 8 == 0.
 * ep_combine_ranks_backward: for every used slot, rank p's grad_y[p] row =
 *   rn16(w * grad_out[t]) (one fp32 product) and grad_weights[t][j] = the
 *   fp32 dot product of grad_out[t] with the slot's row of y[p] (fixed
 *   reduction order: bitwise repeatable).  y and grad_y: HOST tables of R
 *   device pointers with y_rows / grad_y_rows rows, 32-byte aligned;
 *   grad_out_rows device [t_count][H], 32-byte aligned; H % 16 == 0.
 * Rows past a rank's capacity are skipped and set EP_ERR_CAPACITY. */
ep_status_t ep_dispatch_ranks_backward(ep_handle_t h, int t_begin, int t_count,
                                       const void* const* grad_recv, const int64_t* grad_rows,
                                       int H, ep_dtype_t dtype, void* grad_x_rows, void* stream);
ep_status_t ep_combine_ranks_backward(ep_handle_t h, int t_begin, int t_count,
                                      const void* grad_out_rows, const void* const* y,
                                      const int64_t* y_rows, const float* topk_weights_rows, int H,
                                      ep_dtype_t dtype, void* const* grad_y,
                                      const int64_t* grad_y_rows, float* grad_weights_rows,
                                      void* stream);

/* GEMM-ready receive layout.  The pages say the high-throughput and
 * low-latency kernels share one "GEMM layout" (DeepEP v2 release notes, "Có
 * gì mới trong v2") without defining it; these helpers complete the reading
 * taken here for an expert GEMM that consumes the receive buffer directly.
 *
 * ep_dispatch_weights: recv_weights[dst_row[t][j]] = topk_weights[t][j] for
 * every used slot of the last layout (device fp32 [T][k] in, device fp32
 * [recv_capacity_rows] out, 4-byte aligned; pad rows are not written), so the
 * expert op can scale its rows.  A row >= recv_capacity_rows sets
 * EP_ERR_CAPACITY.
 *
 * ep_zero_pad_rows: set every pad row of a buffer in the receive layout to
 * zero bytes (rows: device, capacity_rows rows of row_bytes bytes; 16-byte
 * stores when row_bytes % 16 == 0 and rows is 16-byte aligned), so a GEMM
 * over whole 128-row blocks reads zeros there.  Works for recv_x, row-major
 * scales, y or grad_y.  A pad row >= capacity_rows sets EP_ERR_CAPACITY. */
ep_status_t ep_dispatch_weights(ep_handle_t h, const float* topk_weights, float* recv_weights,
                                int64_t recv_capacity_rows, void* stream);
ep_status_t ep_zero_pad_rows(ep_handle_t h, void* rows, int64_t row_bytes, int64_t capacity_rows,
                             void* stream);

/* Backward of ep_dispatch for the last layout: grad_x[t] = sum over the used
 * slots of grad_recv[dst_row[t][j]], accumulated in fp32 in slot order
 * j = 0..k-1, rounded to bf16 (the forward sent x[t] to each of those rows).
 * grad_recv: device bf16 [grad_rows][H] in the receive layout (for an FP8
 * dispatch: the gradient with respect to the dequantised rows); grad_x:
 * device bf16 [T][H].  16-byte aligned, H % 8 == 0.  A row >= grad_rows is
 * skipped and sets EP_ERR_CAPACITY.
 *
 * The pages name training as a use (pomoai page, 核心使用场景; yololab page,
 * high-throughput mode) but define no gradients; these are the gradients of
 * the forward definitions. */
ep_status_t ep_dispatch_backward(ep_handle_t h, const void* grad_recv, int64_t grad_rows, int H,
                                 void* grad_x, void* stream);

/* Backward of ep_combine for the last layout, given grad_out (device bf16
 * [T][H]) and the forward's y (device bf16 [y_rows][H]) and topk_weights
 * (device fp32 [T][k]):
 *   grad_y[dst_row[t][j]][h] = bf16_rn(w[t][j] * grad_out[t][h])   (one fp32 product)
 *   grad_weights[t][j]       = sum_h grad_out[t][h] * y[dst_row[t][j]][h]   (fp32)
 * grad_y: device bf16 [grad_y_rows][H] in the receive layout (pad rows keep
 * their contents); grad_weights: device fp32 [T][k], 0 for unused slots.
 * The dot products use fused multiply-adds per thread and a fixed reduction
 * tree: bitwise repeatable, within the fp32 summation bound
 * H * 2^-24 * sum |grad_out * y| of the exact value.  16-byte aligned
 * bf16 arrays, 4-byte aligned fp32 arrays, H % 8 == 0.  A row beyond
 * y_rows or grad_y_rows is skipped (grad_weights 0) and sets
 * EP_ERR_CAPACITY. */
ep_status_t ep_combine_backward(ep_handle_t h, const void* grad_out, const void* y,
                                int64_t y_rows, const float* topk_weights, int H, void* grad_y,
                                int64_t grad_y_rows, float* grad_weights, void* stream);

/* The two backward calls with the type of the 16-bit rows named:
 * EP_DTYPE_BF16 is the calls above; EP_DTYPE_FP16 takes binary16 gradient and
 * expert-output rows (widened exactly) and writes binary16 grad_x / grad_y
 * (round to nearest even), with the same fp32 arithmetic and order; grad_w
 * stays fp32. */
ep_status_t ep_dispatch_backward_ex(ep_handle_t h, const void* grad_recv, int64_t grad_rows, int H,
                                    ep_dtype_t dtype, void* grad_x, void* stream);
ep_status_t ep_combine_backward_ex(ep_handle_t h, const void* grad_out, const void* y,
                                   int64_t y_rows, const float* topk_weights, int H,
                                   ep_dtype_t dtype, void* grad_y, int64_t grad_y_rows,
                                   float* grad_weights, void* stream);

/* Wait for the stream (SYNCHRONISING), read and clear the sticky device
 * error word.  Returns EP_ERR_TIMEOUT, EP_ERR_BAD_INDEX or EP_ERR_CAPACITY
 * (in that order of precedence when several are set) or EP_OK. */
ep_status_t ep_handle_check(ep_handle_t h, void* stream);

/* ------------------------------------------------------------------------
 * Dispatch layout without any caller-provided workspace.
 *
 * The pages have no counterpart of this call; it exists for callers that
 * cannot allocate device memory: processes whose device memory is owned up
 * front by a framework allocator or a pre-reserved pool that forbids more
 * cudaMalloc calls, and plug-ins that are handed only input and output
 * pointers.
 *
 * It computes exactly what ep_layout computes, into caller-provided output
 * arrays, with the same kernels.  Its only scratch (4 bytes x ceil(T/32) x
 * (E + R) counters) lives in a fixed array of EP_STATIC_SCRATCH_BYTES inside
 * this library, which every GPU that loads the library keeps until the
 * process exits.  Nothing is allocated: no cudaMalloc, no cudaFree, no
 * allocating library call.
 *
 *   - Larger requests (4 * ceil(T/32) * (E + R) > EP_STATIC_SCRATCH_BYTES)
 *     return EP_ERR_WORKSPACE_TOO_SMALL and enqueue nothing.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) and caches it; make that first call before any
 *     stream capture.  Devices with an ordinal above 63 are refused
 *     (EP_ERR_INVALID_ARG); CUDA failures return EP_ERR_CUDA with the
 *     message in ep_last_error_message.
 *   - Every call shares the one array per device and it keeps the last
 *     call's contents (nothing in it needs to start at zero).  Calls that
 *     overlap on the GPU -- on different streams without ordering, or from
 *     several host threads -- race on it and must be serialised by the caller.
 *
 * Outputs (device): num_tokens_per_expert int32 [E], num_tokens_per_rank
 * int32 [R], num_rows_per_rank int32 [R], expert_off int32 [E+1], rank_off
 * int32 [R+1], total_recv_rows int32 [1], is_token_in_rank uint8 [T][R],
 * dst_row int32 [T][k], recv_src int32 [recv_src_capacity] with
 * recv_src_capacity >= ep_recv_rows_upper_bound(T, k, E, block_m)
 * (else EP_ERR_CAPACITY), error_word int32 [1]: zeroed by this call, then
 * EP_ERR_BAD_INDEX's bit (1) is set if an index is outside [-1, E).
 * topk_idx: device int64 [T][k], 8-byte aligned.  Shape rules as for
 * ep_workspace_bytes. */
#define EP_STATIC_SCRATCH_BYTES (4u << 20)
ep_status_t ep_layout_static_scratch(const int64_t* topk_idx, int T, int num_topk,
                                     int num_experts, int num_ranks, int block_m,
                                     int32_t* num_tokens_per_expert, int32_t* num_tokens_per_rank,
                                     int32_t* num_rows_per_rank, int32_t* expert_off,
                                     int32_t* rank_off, int32_t* total_recv_rows,
                                     uint8_t* is_token_in_rank, int32_t* dst_row,
                                     int32_t* recv_src, int64_t recv_src_capacity,
                                     int32_t* error_word, void* stream);

/* Human-readable name of a status. */
const char* ep_strerror(ep_status_t status);

/* Text of the last CUDA error seen by this host thread inside the library
 * ("" if none). */
const char* ep_last_error_message(void);

#ifdef __cplusplus
}
#endif

#endif /* EP_H_ */
