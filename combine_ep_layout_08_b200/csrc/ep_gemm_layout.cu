// ep_gemm_layout.cu -- helpers that make the receive buffer directly usable
// by an expert GEMM.  The pages say the high-throughput and low-latency
// kernels share one "GEMM layout" (DeepEP v2 release notes, "Có gì mới trong
// v2") without defining it; with the expert-major, 128-row-padded reading of
// ep.h these complete it: the routing weight of every receive row, and zeroed
// pad rows for a GEMM that runs over whole blocks.  (The MN-major FP8 scale
// layout is a dispatch format, in ep_dispatch.cu.)
#include <algorithm>

#include "ep_internal.cuh"

namespace ep {
namespace {

constexpr int kThreads = 256;
constexpr int64_t kMaxGrid = 1 << 20;

// recv_w[dst_row[t][j]] = w[t][j]: one thread per (token, slot).
__global__ void __launch_bounds__(kThreads)
dispatch_weights_kernel(const float* __restrict__ w, const int32_t* __restrict__ dst_row,
                        int64_t entries, float* __restrict__ recv_w, int64_t cap_rows,
                        int32_t* err)
{
    pdl_wait();
    pdl_trigger();
    for (int64_t f = (int64_t)blockIdx.x * kThreads + threadIdx.x; f < entries;
         f += (int64_t)gridDim.x * kThreads) {
        const int32_t d = dst_row[f];
        if (d < 0)
            continue;
        if (d >= cap_rows) {
            atomicOr(err, kErrDispatchCap);
            continue;
        }
        recv_w[d] = w[f];
    }
}

// Zero the pad rows [off[e] + cnt[e], off[e+1]) of a row buffer: grid
// (x, y = expert), one warp per pad row (an expert has at most block_m - 1);
// 16-byte stores when rows are 16-byte multiples.
__global__ void __launch_bounds__(kThreads)
zero_pad_rows_kernel(const int32_t* __restrict__ expert_off, const int32_t* __restrict__ cnt,
                     uint8_t* __restrict__ rows, int64_t row_bytes, int64_t cap_rows,
                     int32_t* err)
{
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int e = blockIdx.y;
    const int64_t a = (int64_t)expert_off[e] + cnt[e], b = expert_off[e + 1];
    const int64_t r = a + (int64_t)blockIdx.x * (kThreads / 32) + warp;
    if (r >= b)
        return;
    if (r >= cap_rows) {
        if (lane == 0)
            atomicOr(err, kErrDispatchCap);
        return;
    }
    uint8_t* row = rows + r * row_bytes;
    if ((row_bytes % 16 == 0) && (((uintptr_t)rows & 15u) == 0)) {
        for (int64_t i = 16 * lane; i < row_bytes; i += 16 * 32)
            *reinterpret_cast<int4*>(row + i) = make_int4(0, 0, 0, 0);
    } else {
        for (int64_t i = lane; i < row_bytes; i += 32) row[i] = 0;
    }
}

}  // namespace

cudaError_t launch_dispatch_weights(const Handle& h, const float* w, float* recv_w,
                                    int64_t cap_rows, cudaStream_t s)
{
    const int64_t entries = (int64_t)h.T * h.k;
    if (entries == 0)
        return cudaSuccess;
    const unsigned grid = (unsigned)std::min<int64_t>(kMaxGrid, (entries + kThreads - 1) / kThreads);
    return launch_pdl(dispatch_weights_kernel, grid, kThreads, 0, s, w, h.dst_row, entries, recv_w,
                      cap_rows, h.err);
}

cudaError_t launch_zero_pad_rows(const Handle& h, void* rows, int64_t row_bytes, int64_t cap_rows,
                                 cudaStream_t s)
{
    if (h.block_m < 2)
        return cudaSuccess;  // no padding
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((h.block_m - 1 + kThreads / 32 - 1) / (kThreads / 32)),
                       (unsigned)h.E);
    cfg.blockDim = dim3(kThreads);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, zero_pad_rows_kernel, (const int32_t*)h.expert_off,
                              (const int32_t*)h.cnt, static_cast<uint8_t*>(rows), row_bytes,
                              cap_rows, h.err);
}

}  // namespace ep
