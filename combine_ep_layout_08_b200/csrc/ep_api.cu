// ep_api.cu -- the C ABI declared in include/ep.h: argument checks, the
// workspace carve, the handle, and the kernel launches.  No device memory is
// allocated here; the handle is one small host allocation.  The split between
// a caller-sized workspace holding the dispatch layout and a handle carrying it
// from dispatch to combine follows the pages' ElasticBuffer ("DeepEP是什麼？
// …", section ElasticBuffer: sized from max tokens, top-k, hidden size and EP
// degree) and EPHandle (DeepEP v2 release notes, section Có gì mới trong v2);
// each operation's own source is stated with its declaration in ep.h.
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <mutex>

#include "ep_internal.cuh"

namespace ep {

namespace {
thread_local char g_last_error[256] = "";
}  // namespace

ep_status_t cuda_fail(cudaError_t e, const char* where)
{
    snprintf(g_last_error, sizeof g_last_error, "%s: %s (%s)", where, cudaGetErrorName(e),
             cudaGetErrorString(e));
    return EP_ERR_CUDA;
}

ep_status_t fail_message(ep_status_t st, const char* what)
{
    snprintf(g_last_error, sizeof g_last_error, "%s", what);
    return st;
}

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

Handle* as_handle(ep_handle_t h)
{
    Handle* p = reinterpret_cast<Handle*>(h);
    return (p && p->magic == kHandleMagic) ? p : nullptr;
}

bool valid_shape(int max_tokens, int k, int E, int R, int block_m)
{
    if (max_tokens < 0 || k < 1 || k > EP_MAX_TOPK || E < 1 || E > EP_MAX_EXPERTS || R < 1 ||
        R > E || E % R != 0 || block_m < 1 || block_m > EP_MAX_BLOCK_M)
        return false;
    // every row and entry index must fit in int32
    const int64_t entries = (int64_t)max_tokens * k;
    if (entries > INT32_MAX)
        return false;
    if (recv_rows_bound(max_tokens, k, E, block_m) > INT32_MAX)
        return false;
    if ((int64_t)max_tokens * R > INT64_C(1) << 40)
        return false;
    return true;
}

}  // namespace

int64_t recv_rows_bound(int64_t T, int64_t k, int64_t E, int64_t block_m)
{
    const int64_t n = T * k;
    const int64_t m = n < E ? n : E;
    const int64_t b = n + m * (block_m - 1);
    return b / block_m * block_m;
}

bool carve_workspace(int max_tokens, int k, int E, int R, int block_m, Carve* c)
{
    if (!valid_shape(max_tokens, k, E, R, block_m))
        return false;
    const int64_t nchunks = ((int64_t)max_tokens + kChunkTokens - 1) / kChunkTokens;
    const int64_t rows = recv_rows_bound(max_tokens, k, E, block_m);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = align_up(off + (bytes ? bytes : 1));
        return at;
    };
    c->chunk_counts = take(sizeof(int32_t) * (size_t)nchunks * E);
    c->chunk_rank = take(sizeof(int32_t) * (size_t)nchunks * R);
    c->cnt = take(sizeof(int32_t) * (size_t)E);
    c->expert_off = take(sizeof(int32_t) * (size_t)(E + 1));
    c->rank_off = take(sizeof(int32_t) * (size_t)(R + 1));
    c->tokens_per_rank = take(sizeof(int32_t) * (size_t)R);
    c->rows_per_rank = take(sizeof(int32_t) * (size_t)R);
    c->total_rows = take(sizeof(int32_t));
    c->err = take(3 * sizeof(int32_t));
    c->tile_acc = take(sizeof(int32_t) * tile_acc_words(E, R));
    c->is_token_in_rank = take((size_t)max_tokens * R);
    c->dst_row = take(sizeof(int32_t) * (size_t)max_tokens * k);
    c->recv_src = take(sizeof(int32_t) * (size_t)rows);
    c->total = off;
    return true;
}

cudaError_t persistent_grid(const void* kernel, int block_threads, size_t dyn_smem,
                            int max_per_sm, int* grid)
{
    // Cache per (kernel, device); a handful of kernels and devices at most.
    struct Entry {
        const void* kernel;
        int device, grid;
    };
    static Entry cache[64];
    static int used = 0;
    static std::mutex mu;

    int dev = 0;
    cudaError_t rc = cudaGetDevice(&dev);
    if (rc != cudaSuccess)
        return rc;
    {
        std::lock_guard<std::mutex> lock(mu);
        for (int i = 0; i < used; ++i)
            if (cache[i].kernel == kernel && cache[i].device == dev) {
                *grid = cache[i].grid;
                return cudaSuccess;
            }
    }
    int sms = 0, per_sm = 0;
    if ((rc = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return rc;
    if ((rc = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, block_threads,
                                                            dyn_smem)) != cudaSuccess)
        return rc;
    if (per_sm < 1)
        per_sm = 1;
    if (per_sm > max_per_sm)
        per_sm = max_per_sm;
    *grid = sms * per_sm;
    std::lock_guard<std::mutex> lock(mu);
    if (used < 64)
        cache[used++] = Entry{kernel, dev, *grid};
    return cudaSuccess;
}

}  // namespace ep

using ep::Handle;

namespace {

// Dispatch / combine of the tokens [t_begin, t_begin + t_count) of the last
// layout: the kernels see a shallow copy of the handle whose token count and
// dst_row start at the range.
// Argument checks of a dispatch of t_count tokens (no launch).
ep_status_t dispatch_check(int t_count, const void* x, ep_dtype_t x_dtype, int H, ep_fmt_t fmt,
                           const void* recv_x, const float* recv_scales,
                           int64_t recv_capacity_rows)
{
    if (H <= 0 || recv_capacity_rows < 0)
        return EP_ERR_INVALID_ARG;
    if (x_dtype != EP_DTYPE_BF16 && x_dtype != EP_DTYPE_FP16)
        return EP_ERR_INVALID_ARG;
    const bool fp8 = fmt == EP_FMT_FP8_E4M3_1X128 || fmt == EP_FMT_FP8_E4M3_1X128_MN;
    const bool copy = fmt == EP_FMT_BF16 || fmt == EP_FMT_FP16;
    if (!copy && !fp8)
        return EP_ERR_INVALID_ARG;
    if (copy && (fmt == EP_FMT_FP16) != (x_dtype == EP_DTYPE_FP16))
        return EP_ERR_INVALID_ARG;
    if (copy && H % 8 != 0)
        return EP_ERR_INVALID_ARG;
    if (fp8 && H % 128 != 0)
        return EP_ERR_INVALID_ARG;
    if (fmt == EP_FMT_FP8_E4M3_1X128_MN && recv_capacity_rows % 4 != 0)
        return EP_ERR_INVALID_ARG;
    if (t_count > 0 && (!x || (!recv_x && recv_capacity_rows > 0)))
        return EP_ERR_INVALID_ARG;
    if (fp8 && t_count > 0 && recv_capacity_rows > 0 && !recv_scales)
        return EP_ERR_INVALID_ARG;
    if (!ep::aligned(x, 16) || !ep::aligned(recv_x, 16) || !ep::aligned(recv_scales, 16))
        return EP_ERR_ALIGNMENT;
    return EP_OK;
}

// The input type the formats of ep_dispatch imply: fp16 for the fp16 copy.
ep_dtype_t implied_dtype(ep_fmt_t fmt)
{
    return fmt == EP_FMT_FP16 ? EP_DTYPE_FP16 : EP_DTYPE_BF16;
}

// Dispatch / combine of the tokens [t_begin, t_begin + t_count) of the last
// layout: the kernels see a shallow copy of the handle whose token count and
// dst_row start at the range.
ep_status_t dispatch_impl(Handle* h, int t_begin, int t_count, const void* x, ep_dtype_t x_dtype,
                          int H, ep_fmt_t fmt, void* recv_x, float* recv_scales,
                          int64_t recv_capacity_rows, void* stream, const char* what)
{
    if (!h)
        return EP_ERR_INVALID_ARG;
    if (!h->has_layout)
        return EP_ERR_STATE;
    if (t_begin < 0 || t_count < 0 || (int64_t)t_begin + t_count > h->T)
        return EP_ERR_INVALID_ARG;
    const ep_status_t st =
        dispatch_check(t_count, x, x_dtype, H, fmt, recv_x, recv_scales, recv_capacity_rows);
    if (st != EP_OK)
        return st;
    Handle sub = *h;
    sub.T = t_count;
    sub.dst_row = h->dst_row + (int64_t)t_begin * h->k;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool copy = fmt == EP_FMT_BF16 || fmt == EP_FMT_FP16;
    cudaError_t rc = copy  // a 2-byte row copy, whatever the 16-bit type
                         ? ep::launch_dispatch_bf16(sub, x, H, recv_x, recv_capacity_rows, s)
                         : ep::launch_dispatch_fp8(
                               sub, x, H, recv_x, recv_scales,
                               fmt == EP_FMT_FP8_E4M3_1X128_MN ? recv_capacity_rows : 0,
                               recv_capacity_rows, x_dtype == EP_DTYPE_FP16, s);
    return rc == cudaSuccess ? EP_OK : ep::cuda_fail(rc, what);
}

ep_status_t layout_check(Handle* h, const int64_t* topk_idx, int T)
{
    if (!h || T < 0 || T > h->max_tokens || (T > 0 && !topk_idx))
        return EP_ERR_INVALID_ARG;
    if (!ep::aligned(topk_idx, 8))
        return EP_ERR_ALIGNMENT;
    return EP_OK;
}

// The workspace starts with unknown contents: zero the error word and the
// grid barrier's words once, on the first layout of the handle.
ep_status_t clear_error_words_once(Handle* h, cudaStream_t s)
{
    if (h->err_cleared)
        return EP_OK;
    cudaError_t rc = cudaMemsetAsync(h->err, 0, 3 * sizeof(int32_t), s);
    if (rc == cudaSuccess)
        rc = cudaMemsetAsync(h->tile_acc, 0, sizeof(int32_t) * ep::tile_acc_words(h->E, h->R), s);
    if (rc != cudaSuccess)
        return ep::cuda_fail(rc, "clearing the error words");
    h->err_cleared = 1;
    return EP_OK;
}

ep_status_t combine_impl(Handle* h, int t_begin, int t_count, const void* y, int64_t y_rows,
                         const float* topk_weights, int H, ep_dtype_t dtype, void* out,
                         void* stream, const char* what)
{
    if (!h || H <= 0 || H % 8 != 0 || y_rows < 0)
        return EP_ERR_INVALID_ARG;
    if (dtype != EP_DTYPE_BF16 && dtype != EP_DTYPE_FP16)
        return EP_ERR_INVALID_ARG;
    if (!h->has_layout)
        return EP_ERR_STATE;
    if (t_begin < 0 || t_count < 0 || (int64_t)t_begin + t_count > h->T)
        return EP_ERR_INVALID_ARG;
    if (t_count > 0 && (!out || !topk_weights || (!y && y_rows > 0)))
        return EP_ERR_INVALID_ARG;
    if (!ep::aligned(y, 16) || !ep::aligned(out, 16) || !ep::aligned(topk_weights, 4))
        return EP_ERR_ALIGNMENT;
    Handle sub = *h;
    sub.T = t_count;
    sub.dst_row = h->dst_row + (int64_t)t_begin * h->k;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t rc = ep::launch_combine(sub, y, y_rows, topk_weights, H, out,
                                        dtype == EP_DTYPE_FP16, s);
    return rc == cudaSuccess ? EP_OK : ep::cuda_fail(rc, what);
}

}  // namespace

extern "C" {

size_t ep_workspace_bytes(int max_tokens, int num_topk, int num_experts, int num_ranks,
                          int block_m)
{
    ep::Carve c;
    if (!ep::carve_workspace(max_tokens, num_topk, num_experts, num_ranks, block_m, &c))
        return 0;
    return c.total;
}

int64_t ep_recv_rows_upper_bound(int T, int num_topk, int num_experts, int block_m)
{
    if (T < 0 || num_topk < 1 || num_experts < 1 || block_m < 1)
        return -1;
    return ep::recv_rows_bound(T, num_topk, num_experts, block_m);
}

ep_status_t ep_handle_create(void* workspace, size_t workspace_bytes, int max_tokens,
                             int num_topk, int num_experts, int num_ranks, int block_m,
                             ep_handle_t* out)
{
    if (!out)
        return EP_ERR_INVALID_ARG;
    *out = nullptr;
    ep::Carve c;
    if (!ep::carve_workspace(max_tokens, num_topk, num_experts, num_ranks, block_m, &c))
        return EP_ERR_INVALID_ARG;
    if (!workspace)
        return EP_ERR_INVALID_ARG;
    if (!ep::aligned(workspace, ep::kAlign))
        return EP_ERR_ALIGNMENT;
    if (workspace_bytes < c.total)
        return EP_ERR_WORKSPACE_TOO_SMALL;
    Handle* h = static_cast<Handle*>(calloc(1, sizeof(Handle)));
    if (!h)
        return EP_ERR_NO_MEMORY;
    char* base = static_cast<char*>(workspace);
    h->magic = ep::kHandleMagic;
    h->max_tokens = max_tokens;
    h->k = num_topk;
    h->E = num_experts;
    h->R = num_ranks;
    h->block_m = block_m;
    h->max_rows = ep::recv_rows_bound(max_tokens, num_topk, num_experts, block_m);
    h->max_chunks = ((int64_t)max_tokens + ep::kChunkTokens - 1) / ep::kChunkTokens;
    h->chunk_counts = reinterpret_cast<int32_t*>(base + c.chunk_counts);
    h->chunk_rank = reinterpret_cast<int32_t*>(base + c.chunk_rank);
    h->cnt = reinterpret_cast<int32_t*>(base + c.cnt);
    h->expert_off = reinterpret_cast<int32_t*>(base + c.expert_off);
    h->rank_off = reinterpret_cast<int32_t*>(base + c.rank_off);
    h->tokens_per_rank = reinterpret_cast<int32_t*>(base + c.tokens_per_rank);
    h->rows_per_rank = reinterpret_cast<int32_t*>(base + c.rows_per_rank);
    h->total_rows = reinterpret_cast<int32_t*>(base + c.total_rows);
    h->err = reinterpret_cast<int32_t*>(base + c.err);
    h->tile_acc = reinterpret_cast<int32_t*>(base + c.tile_acc);
    h->is_token_in_rank = reinterpret_cast<uint8_t*>(base + c.is_token_in_rank);
    h->dst_row = reinterpret_cast<int32_t*>(base + c.dst_row);
    h->recv_src = reinterpret_cast<int32_t*>(base + c.recv_src);
    h->T = -1;
    h->has_layout = 0;
    h->err_cleared = 0;
    *out = reinterpret_cast<ep_handle_t>(h);
    return EP_OK;
}

void ep_handle_destroy(ep_handle_t hh)
{
    Handle* h = ep::as_handle(hh);
    if (!h)
        return;
    h->magic = 0;
    free(h);
}

ep_status_t ep_layout(ep_handle_t hh, const int64_t* topk_idx, int T, void* stream)
{
    Handle* h = ep::as_handle(hh);
    ep_status_t st = layout_check(h, topk_idx, T);
    if (st != EP_OK)
        return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((st = clear_error_words_once(h, s)) != EP_OK)
        return st;
    cudaError_t rc = ep::launch_layout(*h, topk_idx, T, s);
    if (rc != cudaSuccess) {
        h->has_layout = 0;
        return ep::cuda_fail(rc, "ep_layout");
    }
    h->T = T;
    h->has_layout = 1;
    return EP_OK;
}

ep_status_t ep_layout_dispatch(ep_handle_t hh, const int64_t* topk_idx, int T, const void* x,
                               int H, ep_fmt_t fmt, void* recv_x, float* recv_scales,
                               int64_t recv_capacity_rows, void* stream)
{
    Handle* h = ep::as_handle(hh);
    ep_status_t st = layout_check(h, topk_idx, T);
    if (st != EP_OK)
        return st;
    const ep_dtype_t x_dtype = implied_dtype(fmt);
    if ((st = dispatch_check(T, x, x_dtype, H, fmt, recv_x, recv_scales, recv_capacity_rows)) !=
        EP_OK)
        return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool fp8 = fmt == EP_FMT_FP8_E4M3_1X128 || fmt == EP_FMT_FP8_E4M3_1X128_MN;
    const bool v32 = H % 16 == 0 && ep::aligned(x, 32) && (fp8 || ep::aligned(recv_x, 32));
    if (T > 0 && v32 && ep::fused_layout_dispatch_fits(*h, T)) {
        if ((st = clear_error_words_once(h, s)) != EP_OK)
            return st;
        cudaError_t rc = ep::launch_layout_dispatch(
            *h, topk_idx, T, x, H, fp8, recv_x, recv_scales,
            fmt == EP_FMT_FP8_E4M3_1X128_MN ? recv_capacity_rows : 0, recv_capacity_rows, s);
        if (rc != cudaSuccess) {
            h->has_layout = 0;
            return ep::cuda_fail(rc, "ep_layout_dispatch");
        }
        h->T = T;
        h->has_layout = 1;
        return EP_OK;
    }
    if ((st = ep_layout(hh, topk_idx, T, stream)) != EP_OK)
        return st;
    return dispatch_impl(h, 0, T, x, x_dtype, H, fmt, recv_x, recv_scales, recv_capacity_rows,
                         stream, "ep_layout_dispatch");
}

const void* ep_handle_view(ep_handle_t hh, ep_view_t what, int64_t* count)
{
    Handle* h = ep::as_handle(hh);
    if (!h)
        return nullptr;
    const int64_t T = h->has_layout ? h->T : 0;
    const void* p = nullptr;
    int64_t n = 0;
    switch (what) {
    case EP_VIEW_NUM_TOKENS_PER_EXPERT: p = h->cnt; n = h->E; break;
    case EP_VIEW_NUM_TOKENS_PER_RANK: p = h->tokens_per_rank; n = h->R; break;
    case EP_VIEW_NUM_ROWS_PER_RANK: p = h->rows_per_rank; n = h->R; break;
    case EP_VIEW_EXPERT_OFFSET: p = h->expert_off; n = h->E + 1; break;
    case EP_VIEW_RANK_OFFSET: p = h->rank_off; n = h->R + 1; break;
    case EP_VIEW_IS_TOKEN_IN_RANK: p = h->is_token_in_rank; n = T * h->R; break;
    case EP_VIEW_DST_ROW: p = h->dst_row; n = T * h->k; break;
    case EP_VIEW_RECV_SRC: p = h->recv_src; n = h->max_rows; break;
    case EP_VIEW_TOTAL_RECV_ROWS: p = h->total_rows; n = 1; break;
    case EP_VIEW_ERROR_WORDS: p = h->err; n = 3; break;
    default: return nullptr;
    }
    if (count)
        *count = n;
    return p;
}

ep_status_t ep_handle_read_counts(ep_handle_t hh, int32_t* num_tokens_per_expert,
                                  int32_t* num_tokens_per_rank, int32_t* num_rows_per_rank,
                                  int32_t* total_recv_rows, void* stream)
{
    Handle* h = ep::as_handle(hh);
    if (!h)
        return EP_ERR_INVALID_ARG;
    if (!h->has_layout)
        return EP_ERR_STATE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t rc = cudaSuccess;
    if (num_tokens_per_expert && rc == cudaSuccess)
        rc = cudaMemcpyAsync(num_tokens_per_expert, h->cnt, sizeof(int32_t) * h->E,
                             cudaMemcpyDeviceToHost, s);
    if (num_tokens_per_rank && rc == cudaSuccess)
        rc = cudaMemcpyAsync(num_tokens_per_rank, h->tokens_per_rank, sizeof(int32_t) * h->R,
                             cudaMemcpyDeviceToHost, s);
    if (num_rows_per_rank && rc == cudaSuccess)
        rc = cudaMemcpyAsync(num_rows_per_rank, h->rows_per_rank, sizeof(int32_t) * h->R,
                             cudaMemcpyDeviceToHost, s);
    if (total_recv_rows && rc == cudaSuccess)
        rc = cudaMemcpyAsync(total_recv_rows, h->total_rows, sizeof(int32_t),
                             cudaMemcpyDeviceToHost, s);
    if (rc == cudaSuccess)
        rc = cudaStreamSynchronize(s);
    return rc == cudaSuccess ? EP_OK : ep::cuda_fail(rc, "ep_handle_read_counts");
}



ep_status_t ep_dispatch(ep_handle_t hh, const void* x, int H, ep_fmt_t fmt, void* recv_x,
                        float* recv_scales, int64_t recv_capacity_rows, void* stream)
{
    Handle* h = ep::as_handle(hh);
    return dispatch_impl(h, 0, h ? std::max(h->T, 0) : 0, x, implied_dtype(fmt), H, fmt, recv_x,
                         recv_scales, recv_capacity_rows, stream, "ep_dispatch");
}

ep_status_t ep_dispatch_ex(ep_handle_t hh, const void* x, ep_dtype_t x_dtype, int H, ep_fmt_t fmt,
                           void* recv_x, float* recv_scales, int64_t recv_capacity_rows,
                           void* stream)
{
    Handle* h = ep::as_handle(hh);
    return dispatch_impl(h, 0, h ? std::max(h->T, 0) : 0, x, x_dtype, H, fmt, recv_x,
                         recv_scales, recv_capacity_rows, stream, "ep_dispatch_ex");
}

ep_status_t ep_dispatch_range(ep_handle_t hh, int t_begin, int t_count, const void* x_rows,
                              int H, ep_fmt_t fmt, void* recv_x, float* recv_scales,
                              int64_t recv_capacity_rows, void* stream)
{
    return dispatch_impl(ep::as_handle(hh), t_begin, t_count, x_rows, implied_dtype(fmt), H, fmt,
                         recv_x, recv_scales, recv_capacity_rows, stream, "ep_dispatch_range");
}

ep_status_t ep_combine(ep_handle_t hh, const void* y, int64_t y_rows, const float* topk_weights,
                       int H, void* out, void* stream)
{
    Handle* h = ep::as_handle(hh);
    return combine_impl(h, 0, h ? std::max(h->T, 0) : 0, y, y_rows, topk_weights, H,
                        EP_DTYPE_BF16, out, stream, "ep_combine");
}

ep_status_t ep_combine_ex(ep_handle_t hh, const void* y, int64_t y_rows, const float* topk_weights,
                          int H, ep_dtype_t dtype, void* out, void* stream)
{
    Handle* h = ep::as_handle(hh);
    return combine_impl(h, 0, h ? std::max(h->T, 0) : 0, y, y_rows, topk_weights, H, dtype, out,
                        stream, "ep_combine_ex");
}

ep_status_t ep_combine_range(ep_handle_t hh, int t_begin, int t_count, const void* y,
                             int64_t y_rows, const float* topk_weights_rows, int H,
                             void* out_rows, void* stream)
{
    return combine_impl(ep::as_handle(hh), t_begin, t_count, y, y_rows, topk_weights_rows, H,
                        EP_DTYPE_BF16, out_rows, stream, "ep_combine_range");
}

ep_status_t ep_dispatch_ranks(ep_handle_t hh, int t_begin, int t_count, const void* x_rows, int H,
                              ep_fmt_t fmt, void* const* recv_x, float* const* recv_scales,
                              const int64_t* recv_rows, void* stream)
{
    Handle* h = ep::as_handle(hh);
    if (!h || H <= 0 || H % 16 != 0)
        return EP_ERR_INVALID_ARG;
    if (!h->has_layout)
        return EP_ERR_STATE;
    if (t_begin < 0 || t_count < 0 || (int64_t)t_begin + t_count > h->T)
        return EP_ERR_INVALID_ARG;
    const bool fp8 = fmt == EP_FMT_FP8_E4M3_1X128;
    if (!fp8 && fmt != EP_FMT_BF16 && fmt != EP_FMT_FP16)
        return EP_ERR_INVALID_ARG;
    if (fp8 && H % 128 != 0)
        return EP_ERR_INVALID_ARG;
    if (h->R > EP_MAX_RANK_TABLE || !recv_x || !recv_rows || (fp8 && !recv_scales))
        return EP_ERR_INVALID_ARG;
    if (t_count > 0 && !x_rows)
        return EP_ERR_INVALID_ARG;
    if (!ep::aligned(x_rows, 32))
        return EP_ERR_ALIGNMENT;
    ep::RankTable tab = {};
    for (int p = 0; p < h->R; ++p) {
        if (recv_rows[p] < 0 || (recv_rows[p] > 0 && !recv_x[p]) ||
            (fp8 && recv_rows[p] > 0 && !recv_scales[p]))
            return EP_ERR_INVALID_ARG;
        if (!ep::aligned(recv_x[p], fp8 ? 16 : 32) || (fp8 && !ep::aligned(recv_scales[p], 4)))
            return EP_ERR_ALIGNMENT;
        tab.base[p] = recv_x[p];
        tab.scales[p] = fp8 ? recv_scales[p] : nullptr;
        tab.rows[p] = recv_rows[p];
    }
    Handle sub = *h;
    sub.T = t_count;
    sub.dst_row = h->dst_row + (int64_t)t_begin * h->k;
    cudaError_t rc = ep::launch_dispatch_ranks(sub, x_rows, H, fp8, false, tab,
                                               static_cast<cudaStream_t>(stream));
    return rc == cudaSuccess ? EP_OK : ep::cuda_fail(rc, "ep_dispatch_ranks");
}

ep_status_t ep_combine_ranks(ep_handle_t hh, int t_begin, int t_count, const void* const* y,
                             const int64_t* y_rows, const float* topk_weights_rows, int H,
                             ep_dtype_t dtype, void* out_rows, void* stream)
{
    Handle* h = ep::as_handle(hh);
    if (!h || H <= 0 || H % 8 != 0 || (dtype != EP_DTYPE_BF16 && dtype != EP_DTYPE_FP16))
        return EP_ERR_INVALID_ARG;
    if (!h->has_layout)
        return EP_ERR_STATE;
    if (t_begin < 0 || t_count < 0 || (int64_t)t_begin + t_count > h->T)
        return EP_ERR_INVALID_ARG;
    if (h->R > EP_MAX_RANK_TABLE || !y || !y_rows)
        return EP_ERR_INVALID_ARG;
    if (t_count > 0 && (!out_rows || !topk_weights_rows))
        return EP_ERR_INVALID_ARG;
    if (!ep::aligned(out_rows, 16) || !ep::aligned(topk_weights_rows, 4))
        return EP_ERR_ALIGNMENT;
    ep::RankTable tab = {};
    for (int p = 0; p < h->R; ++p) {
        if (y_rows[p] < 0 || (y_rows[p] > 0 && !y[p]))
            return EP_ERR_INVALID_ARG;
        if (!ep::aligned(y[p], 16))
            return EP_ERR_ALIGNMENT;
        tab.base[p] = const_cast<void*>(y[p]);
        tab.rows[p] = y_rows[p];
    }
    Handle sub = *h;
    sub.T = t_count;
    sub.dst_row = h->dst_row + (int64_t)t_begin * h->k;
    cudaError_t rc = ep::launch_combine_ranks(sub, topk_weights_rows, H, dtype == EP_DTYPE_FP16,
                                              tab, out_rows, static_cast<cudaStream_t>(stream));
    return rc == cudaSuccess ? EP_OK : ep::cuda_fail(rc, "ep_combine_ranks");
}

namespace {

// A host table of R (pointer, rows) pairs into a RankTable; alignment of
// every non-empty entry checked.
ep_status_t fill_rank_table(const Handle* h, const void* const* ptrs, const int64_t* rows,
                            int align, ep::RankTable* tab)
{
    if (h->R > EP_MAX_RANK_TABLE || !ptrs || !rows)
        return EP_ERR_INVALID_ARG;
    for (int p = 0; p < h->R; ++p) {
        if (rows[p] < 0 || (rows[p] > 0 && !ptrs[p]))
            return EP_ERR_INVALID_ARG;
        if (!ep::aligned(ptrs[p], align))
            return EP_ERR_ALIGNMENT;
        tab->base[p] = const_cast<void*>(ptrs[p]);
        tab->rows[p] = rows[p];
    }
    return EP_OK;
}

ep_status_t range_check(const Handle* h, int t_begin, int t_count)
{
    if (!h->has_layout)
        return EP_ERR_STATE;
    if (t_begin < 0 || t_count < 0 || (int64_t)t_begin + t_count > h->T)
        return EP_ERR_INVALID_ARG;
    return EP_OK;
}

}  // namespace

ep_status_t ep_dispatch_ranks_backward(ep_handle_t hh, int t_begin, int t_count,
                                       const void* const* grad_recv, const int64_t* grad_rows,
                                       int H, ep_dtype_t dtype, void* grad_x_rows, void* stream)
{
    Handle* h = ep::as_handle(hh);
    if (!h || H <= 0 || H % 8 != 0 || (dtype != EP_DTYPE_BF16 && dtype != EP_DTYPE_FP16))
        return EP_ERR_INVALID_ARG;
    ep_status_t st = range_check(h, t_begin, t_count);
    if (st != EP_OK)
        return st;
    if (t_count > 0 && !grad_x_rows)
        return EP_ERR_INVALID_ARG;
    if (!ep::aligned(grad_x_rows, 16))
        return EP_ERR_ALIGNMENT;
    ep::RankTable tab = {};
    if ((st = fill_rank_table(h, grad_recv, grad_rows, 16, &tab)) != EP_OK)
        return st;
    Handle sub = *h;
    sub.T = t_count;
    sub.dst_row = h->dst_row + (int64_t)t_begin * h->k;
    cudaError_t rc = ep::launch_combine_ranks(sub, nullptr, H, dtype == EP_DTYPE_FP16, tab,
                                              grad_x_rows, static_cast<cudaStream_t>(stream));
    return rc == cudaSuccess ? EP_OK : ep::cuda_fail(rc, "ep_dispatch_ranks_backward");
}

ep_status_t ep_combine_ranks_backward(ep_handle_t hh, int t_begin, int t_count,
                                      const void* grad_out_rows, const void* const* y,
                                      const int64_t* y_rows, const float* topk_weights_rows, int H,
                                      ep_dtype_t dtype, void* const* grad_y,
                                      const int64_t* grad_y_rows, float* grad_weights_rows,
                                      void* stream)
{
    Handle* h = ep::as_handle(hh);
    if (!h || H <= 0 || H % 16 != 0 || (dtype != EP_DTYPE_BF16 && dtype != EP_DTYPE_FP16))
        return EP_ERR_INVALID_ARG;
    ep_status_t st = range_check(h, t_begin, t_count);
    if (st != EP_OK)
        return st;
    if (t_count > 0 && (!grad_out_rows || !topk_weights_rows || !grad_weights_rows))
        return EP_ERR_INVALID_ARG;
    if (!ep::aligned(grad_out_rows, 32) || !ep::aligned(topk_weights_rows, 4) ||
        !ep::aligned(grad_weights_rows, 4))
        return EP_ERR_ALIGNMENT;
    ep::RankTable ytab = {}, gytab = {};
    if ((st = fill_rank_table(h, y, y_rows, 32, &ytab)) != EP_OK)
        return st;
    if ((st = fill_rank_table(h, const_cast<const void* const*>(grad_y), grad_y_rows, 32,
                              &gytab)) != EP_OK)
        return st;
    Handle sub = *h;
    sub.T = t_count;
    sub.dst_row = h->dst_row + (int64_t)t_begin * h->k;
    cudaError_t rc = ep::launch_combine_ranks_backward(
        sub, grad_out_rows, topk_weights_rows, H, dtype == EP_DTYPE_FP16, ytab, gytab,
        grad_weights_rows, static_cast<cudaStream_t>(stream));
    return rc == cudaSuccess ? EP_OK : ep::cuda_fail(rc, "ep_combine_ranks_backward");
}

ep_status_t ep_dispatch_weights(ep_handle_t hh, const float* topk_weights, float* recv_weights,
                                int64_t recv_capacity_rows, void* stream)
{
    Handle* h = ep::as_handle(hh);
    if (!h || recv_capacity_rows < 0)
        return EP_ERR_INVALID_ARG;
    if (!h->has_layout)
        return EP_ERR_STATE;
    if (h->T > 0 && (!topk_weights || (!recv_weights && recv_capacity_rows > 0)))
        return EP_ERR_INVALID_ARG;
    if (!ep::aligned(topk_weights, 4) || !ep::aligned(recv_weights, 4))
        return EP_ERR_ALIGNMENT;
    cudaError_t rc = ep::launch_dispatch_weights(*h, topk_weights, recv_weights,
                                                 recv_capacity_rows,
                                                 static_cast<cudaStream_t>(stream));
    return rc == cudaSuccess ? EP_OK : ep::cuda_fail(rc, "ep_dispatch_weights");
}

ep_status_t ep_zero_pad_rows(ep_handle_t hh, void* rows, int64_t row_bytes, int64_t capacity_rows,
                             void* stream)
{
    Handle* h = ep::as_handle(hh);
    if (!h || row_bytes <= 0 || capacity_rows < 0)
        return EP_ERR_INVALID_ARG;
    if (!h->has_layout)
        return EP_ERR_STATE;
    if (!rows && capacity_rows > 0)
        return EP_ERR_INVALID_ARG;
    cudaError_t rc = ep::launch_zero_pad_rows(*h, rows, row_bytes, capacity_rows,
                                              static_cast<cudaStream_t>(stream));
    return rc == cudaSuccess ? EP_OK : ep::cuda_fail(rc, "ep_zero_pad_rows");
}

ep_status_t ep_dispatch_backward_ex(ep_handle_t hh, const void* grad_recv, int64_t grad_rows,
                                    int H, ep_dtype_t dtype, void* grad_x, void* stream)
{
    Handle* h = ep::as_handle(hh);
    if (!h || H <= 0 || H % 8 != 0 || grad_rows < 0 ||
        (dtype != EP_DTYPE_BF16 && dtype != EP_DTYPE_FP16))
        return EP_ERR_INVALID_ARG;
    if (!h->has_layout)
        return EP_ERR_STATE;
    if (h->T > 0 && (!grad_x || (!grad_recv && grad_rows > 0)))
        return EP_ERR_INVALID_ARG;
    if (!ep::aligned(grad_recv, 16) || !ep::aligned(grad_x, 16))
        return EP_ERR_ALIGNMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t rc = ep::launch_combine(*h, grad_recv, grad_rows, nullptr, H, grad_x,
                                        dtype == EP_DTYPE_FP16, s);
    return rc == cudaSuccess ? EP_OK : ep::cuda_fail(rc, "ep_dispatch_backward");
}

ep_status_t ep_dispatch_backward(ep_handle_t hh, const void* grad_recv, int64_t grad_rows, int H,
                                 void* grad_x, void* stream)
{
    return ep_dispatch_backward_ex(hh, grad_recv, grad_rows, H, EP_DTYPE_BF16, grad_x, stream);
}

ep_status_t ep_combine_backward_ex(ep_handle_t hh, const void* grad_out, const void* y,
                                   int64_t y_rows, const float* topk_weights, int H,
                                   ep_dtype_t dtype, void* grad_y, int64_t grad_y_rows,
                                   float* grad_weights, void* stream)
{
    Handle* h = ep::as_handle(hh);
    if (!h || H <= 0 || H % 8 != 0 || y_rows < 0 || grad_y_rows < 0 ||
        (dtype != EP_DTYPE_BF16 && dtype != EP_DTYPE_FP16))
        return EP_ERR_INVALID_ARG;
    if (!h->has_layout)
        return EP_ERR_STATE;
    if (h->T > 0 && (!grad_out || !topk_weights || !grad_weights || (!y && y_rows > 0) ||
                     (!grad_y && grad_y_rows > 0)))
        return EP_ERR_INVALID_ARG;
    if (!ep::aligned(grad_out, 16) || !ep::aligned(y, 16) || !ep::aligned(grad_y, 16) ||
        !ep::aligned(topk_weights, 4) || !ep::aligned(grad_weights, 4))
        return EP_ERR_ALIGNMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t rc = ep::launch_combine_backward(*h, grad_out, y, y_rows, topk_weights, H, grad_y,
                                                 grad_y_rows, grad_weights,
                                                 dtype == EP_DTYPE_FP16, s);
    return rc == cudaSuccess ? EP_OK : ep::cuda_fail(rc, "ep_combine_backward");
}

ep_status_t ep_combine_backward(ep_handle_t hh, const void* grad_out, const void* y,
                                int64_t y_rows, const float* topk_weights, int H, void* grad_y,
                                int64_t grad_y_rows, float* grad_weights, void* stream)
{
    return ep_combine_backward_ex(hh, grad_out, y, y_rows, topk_weights, H, EP_DTYPE_BF16,
                                  grad_y, grad_y_rows, grad_weights, stream);
}

ep_status_t ep_handle_check(ep_handle_t hh, void* stream)
{
    Handle* h = ep::as_handle(hh);
    if (!h)
        return EP_ERR_INVALID_ARG;
    if (!h->err_cleared)
        return EP_OK;  // nothing has run on this handle yet
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t word = 0;
    cudaError_t rc = cudaMemcpyAsync(&word, h->err, sizeof word, cudaMemcpyDeviceToHost, s);
    if (rc == cudaSuccess)
        rc = cudaStreamSynchronize(s);
    // Clear the error word; after a barrier time-out also reset the barrier
    // (its count is left mid-way) and the single-launch layout's sums.
    if (rc == cudaSuccess)
        rc = cudaMemsetAsync(h->err, 0, ((word & ep::kErrTimeout) ? 3 : 1) * sizeof(int32_t), s);
    if (rc == cudaSuccess && (word & ep::kErrTimeout) && h->tile_acc)
        rc = cudaMemsetAsync(h->tile_acc, 0, sizeof(int32_t) * ep::tile_acc_words(h->E, h->R), s);
    if (rc == cudaSuccess)
        rc = cudaStreamSynchronize(s);
    if (rc != cudaSuccess)
        return ep::cuda_fail(rc, "ep_handle_check");
    if (word & ep::kErrTimeout)
        return EP_ERR_TIMEOUT;
    if (word & ep::kErrBadIndex)
        return EP_ERR_BAD_INDEX;
    if (word & (ep::kErrDispatchCap | ep::kErrCombineCap))
        return EP_ERR_CAPACITY;
    return EP_OK;
}

const char* ep_strerror(ep_status_t status)
{
    switch (status) {
    case EP_OK: return "EP_OK";
    case EP_ERR_INVALID_ARG: return "EP_ERR_INVALID_ARG: invalid argument";
    case EP_ERR_ALIGNMENT: return "EP_ERR_ALIGNMENT: pointer misaligned";
    case EP_ERR_WORKSPACE_TOO_SMALL: return "EP_ERR_WORKSPACE_TOO_SMALL: workspace too small";
    case EP_ERR_CAPACITY: return "EP_ERR_CAPACITY: receive row beyond buffer capacity";
    case EP_ERR_BAD_INDEX: return "EP_ERR_BAD_INDEX: top-k index outside [-1, E)";
    case EP_ERR_CUDA: return "EP_ERR_CUDA: CUDA runtime error";
    case EP_ERR_STATE: return "EP_ERR_STATE: no layout on this handle";
    case EP_ERR_NO_MEMORY: return "EP_ERR_NO_MEMORY: host allocation failed";
    case EP_ERR_TIMEOUT: return "EP_ERR_TIMEOUT: a device-side wait gave up; that call's outputs are invalid";
    }
    return "unknown ep_status_t";
}

const char* ep_last_error_message(void) { return ep::g_last_error; }

}  // extern "C"
