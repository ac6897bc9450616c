// ep_internal.cuh -- shared definitions of the CUDA library (not installed).
//
// The handle, the workspace carve, the sticky error bits and the launchers
// each kernel file exports to the C-ABI layer (ep_api.cu).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ep.h"

namespace ep {

constexpr uint32_t kHandleMagic = 0x45504c38u;  // "EPL8"

// Sticky device error bits (one int32 in the workspace).
constexpr int kErrBadIndex = 1;      // top-k index outside [-1, E)
constexpr int kErrDispatchCap = 2;   // dispatch row >= recv capacity
constexpr int kErrCombineCap = 4;    // combine row >= y rows
constexpr int kErrTimeout = 8;       // a grid barrier gave up waiting

// The layout works on chunks of kChunkTokens consecutive tokens, one warp
// per chunk: the (token, slot) entries of a chunk are contiguous in topk_idx.
constexpr int kChunkTokens = 32;

// The single-launch layout groups its tiles; at most kTileMaxGroups groups of
// at most kTileMaxGroups tiles.
constexpr int kTileMaxGroups = 32;
// Words of the single-launch layout's sums (an epoch word and two buffers of
// group rows and per-rank sums); zero when the handle is first used.
size_t tile_acc_words(int E, int R);

struct Handle {
    uint32_t magic;
    int max_tokens, k, E, R, block_m;
    int64_t max_rows;  // capacity of recv_src: the padded-row bound at max_tokens
    int64_t max_chunks;
    // device pointers into the caller's workspace
    int32_t* chunk_counts;   // [max_chunks][E]  per-chunk expert counts, then prefixes
    int32_t* chunk_rank;     // [max_chunks][R]  per-chunk token-per-rank counts
    int32_t* cnt;            // [E]
    int32_t* expert_off;     // [E+1]
    int32_t* rank_off;       // [R+1]
    int32_t* tokens_per_rank;// [R]
    int32_t* rows_per_rank;  // [R]
    int32_t* total_rows;     // [1]
    int32_t* err;            // [3] sticky error bits, then the grid barrier's count and generation
    int32_t* tile_acc;       // [tile_acc_words] the single-launch layout's sums (may be null)
    uint8_t* is_token_in_rank;  // [max_tokens][R]
    int32_t* dst_row;        // [max_tokens][k]
    int32_t* recv_src;       // [max_rows]
    // state of the last layout
    int T;
    int has_layout;
    int err_cleared;  // the sticky error word has been zeroed once on the device
};

// Workspace carve: offsets of each array, 256-byte aligned.  Returns the
// total size, or 0 if the sizes overflow.
struct Carve {
    size_t chunk_counts, chunk_rank, cnt, expert_off, rank_off, tokens_per_rank,
        rows_per_rank, total_rows, err, tile_acc, is_token_in_rank, dst_row, recv_src, total;
};

int64_t recv_rows_bound(int64_t T, int64_t k, int64_t E, int64_t block_m);

// Record a CUDA error for ep_last_error_message and return EP_ERR_CUDA.
ep_status_t cuda_fail(cudaError_t e, const char* where);
// Record a message for ep_last_error_message and return st.
ep_status_t fail_message(ep_status_t st, const char* what);
bool carve_workspace(int max_tokens, int k, int E, int R, int block_m, Carve* c);

// Programmatic dependent launch (sm_90+): every kernel of the library is
// launched with programmatic stream serialization allowed and calls
// pdl_wait() -- it returns once the preceding kernel in the stream has
// completed and its memory is visible -- and then pdl_trigger(), which lets
// the next kernel's CTAs be scheduled while this one drains.  Before
// pdl_wait() a kernel writes nothing but its own shared memory and issues
// nothing but L2 prefetch hints (whose addresses may come from a read whose
// value is used for nothing else), so a kernel may follow any other work.
// 16-bit input values packed two to a 32-bit word: bfloat16 (kHalf = false,
// the upper half of a binary32, widened by a shift) or IEEE binary16
// (kHalf = true, widened exactly by the conversion instruction); and binary32
// rounded to nearest even into that type.
template <bool kHalf>
__device__ __forceinline__ float lo16(uint32_t w)
{
    if constexpr (kHalf)
        return __half2float(__ushort_as_half((unsigned short)(w & 0xffffu)));
    else
        return __uint_as_float(w << 16);
}

template <bool kHalf>
__device__ __forceinline__ float hi16(uint32_t w)
{
    if constexpr (kHalf)
        return __half2float(__ushort_as_half((unsigned short)(w >> 16)));
    else
        return __uint_as_float(w & 0xffff0000u);
}

template <bool kHalf>
__device__ __forceinline__ uint32_t pack16x2(float lo, float hi)
{
    uint32_t a, b;
    if constexpr (kHalf) {
        a = __half_as_ushort(__float2half_rn(lo));
        b = __half_as_ushort(__float2half_rn(hi));
    } else {
        a = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
        b = __bfloat16_as_ushort(__float2bfloat16_rn(hi));
    }
    return a | (b << 16);
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), unsigned grid, unsigned block, size_t smem,
                       cudaStream_t s, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Launchers (each returns the cudaError_t of its launches).
// allow_fused: the single cooperative layout kernel may be used (needs the
// grid barrier words at h.err[1..2], zero-initialised).
cudaError_t launch_layout(const Handle& h, const int64_t* topk_idx, int T, cudaStream_t s,
                          bool allow_fused = true);
// Layout + dispatch in one launch for small batches (fused_layout_dispatch_fits);
// the dispatch side needs the 256-bit path (H % 16 == 0, x / recv_x 32-byte aligned).
bool fused_layout_dispatch_fits(const Handle& h, int T);
cudaError_t launch_layout_dispatch(const Handle& h, const int64_t* topk_idx, int T, const void* x,
                                   int H, bool fp8, void* recv_x, float* recv_scales,
                                   int64_t scales_ld, int64_t cap_rows, cudaStream_t s);
cudaError_t launch_dispatch_bf16(const Handle& h, const void* x, int H, void* recv_x,
                                 int64_t cap_rows, cudaStream_t s);
cudaError_t launch_dispatch_fp8(const Handle& h, const void* x, int H, void* recv_q,
                                float* recv_scales, int64_t scales_ld, int64_t cap_rows,
                                bool half, cudaStream_t s);  // scales_ld 0: row-major scales;
                                                             // half: x is binary16
cudaError_t launch_dispatch_weights(const Handle& h, const float* w, float* recv_w,
                                    int64_t cap_rows, cudaStream_t s);
cudaError_t launch_zero_pad_rows(const Handle& h, void* rows, int64_t row_bytes, int64_t cap_rows,
                                 cudaStream_t s);
cudaError_t launch_combine(const Handle& h, const void* y, int64_t y_rows, const float* w,
                           int H, void* out, bool half,
                           cudaStream_t s);  // w == nullptr: unit weights; half: y, out binary16
cudaError_t launch_combine_backward(const Handle& h, const void* grad_out, const void* y,
                                    int64_t y_rows, const float* w, int H, void* grad_y,
                                    int64_t grad_y_rows, float* grad_w, bool half,
                                    cudaStream_t s);  // half: the rows are binary16

// Per-rank receive buffers of the expert-parallel entry points, passed by
// value: base[p] (rows of the layout's rank-p block, renumbered from 0),
// scales[p] (FP8 row-major scales, or null) and rows[p] (capacity in rows).
struct RankTable {
    void* base[EP_MAX_RANK_TABLE];
    float* scales[EP_MAX_RANK_TABLE];
    int64_t rows[EP_MAX_RANK_TABLE];
};

cudaError_t launch_dispatch_ranks(const Handle& h, const void* x, int H, bool fp8, bool half,
                                  const RankTable& tab, cudaStream_t s);
cudaError_t launch_combine_ranks(const Handle& h, const float* w, int H, bool half,
                                 const RankTable& tab, void* out,
                                 cudaStream_t s);  // w == nullptr: unit weights
cudaError_t launch_combine_ranks_backward(const Handle& h, const void* grad_out, const float* w,
                                          int H, bool half, const RankTable& ytab,
                                          const RankTable& gytab, float* grad_w, cudaStream_t s);

// Persistent-grid size: min(resident blocks per SM from the occupancy API,
// max_per_sm) x the SM count of the current device, cached per kernel and
// device.
cudaError_t persistent_grid(const void* kernel, int block_threads, size_t dyn_smem,
                            int max_per_sm, int* grid);

}  // namespace ep
