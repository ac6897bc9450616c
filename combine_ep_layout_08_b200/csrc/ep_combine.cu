// ep_combine.cu -- combine on sm_100a: gather of the k expert outputs of each
// token and weighted reduction back into token order.
//
// Combine takes the expert outputs and routing weights and returns results
// in the original token order ("DeepEP是什麼？MoE Dispatch、Combine、
// All-to-all與V2架構", stage table of section "MoE為什麼需要All-to-all",
// row Combine: reverse all-to-all plus reduction); it moves the same
// batch x top_k x hidden x sizeof(dtype) bytes as dispatch ("DeepEP 编址服务
// 深度对抗分析", section 五.2).  Reduction semantics (stated in ep.h): fp32
// accumulator, one fused multiply-add per used slot in slot order
// j = 0..k-1, round-to-nearest-even to bf16 (or, for FP16 expert outputs,
// to binary16) at the end.
//
// With a null weight pointer every weight is 1 (fma(1, y, acc) rounds like
// acc + y): that is the backward of dispatch, grad_x[t] = sum of the k rows.
//
// HBM-bound: k row reads (k x 2H bytes) and one row write per token.  Work
// unit: one warp x (token, 32 x U 16-byte vectors of the row).  When every
// slot of the token is used and in range (the common case), all k x U loads
// of a lane are issued before the first multiply-add; the chain itself is
// still evaluated in slot order.  The persistent grid and 512-channel units
// measured best (one unit per warp, 256- or 1024-channel units, and three
// CTAs per SM were slower).  Before the dependent-launch wait each warp
// prefetches the rows of its first unit into L2 (1.1 us less per step at
// the DeepSeek-V3 shape).
#include "ep_internal.cuh"

namespace ep {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kThreads = 256;
constexpr int kU = 2;  // 16-byte vectors per lane per unit

template <bool kHalf>
__device__ __forceinline__ void fma8(float (&acc)[8], float w, const uint4& v)
{
    acc[0] = __fmaf_rn(w, lo16<kHalf>(v.x), acc[0]);
    acc[1] = __fmaf_rn(w, hi16<kHalf>(v.x), acc[1]);
    acc[2] = __fmaf_rn(w, lo16<kHalf>(v.y), acc[2]);
    acc[3] = __fmaf_rn(w, hi16<kHalf>(v.y), acc[3]);
    acc[4] = __fmaf_rn(w, lo16<kHalf>(v.z), acc[4]);
    acc[5] = __fmaf_rn(w, hi16<kHalf>(v.z), acc[5]);
    acc[6] = __fmaf_rn(w, lo16<kHalf>(v.w), acc[6]);
    acc[7] = __fmaf_rn(w, hi16<kHalf>(v.w), acc[7]);
}

// A hint that brings a line into L2; it returns no data, so it may be issued
// before the dependent-launch wait.
__device__ __forceinline__ void prefetch_l2(const void* p)
{
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// A load the compiler may not merge with a later load of the same address.
__device__ __forceinline__ int32_t ld_early(const int32_t* p)
{
    int32_t v;
    asm volatile("ld.global.cg.b32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

template <int KMAX, bool kHalf>
__device__ __forceinline__ void combine_unit_all_valid(const uint4* __restrict__ y, int64_t vpr,
                                                       int k, int d, float w, int64_t v0,
                                                       float (&acc)[kU][8])
{
    // Issue every load first (k <= KMAX), then reduce in slot order.
    uint4 v[KMAX][kU];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
        if (j < k) {
            const int dj = __shfl_sync(kFull, d, j);
            const uint4* row = y + (int64_t)dj * vpr;
#pragma unroll
            for (int i = 0; i < kU; ++i)
                if (v0 + 32 * i < vpr)
                    v[j][i] = __ldcs(row + v0 + 32 * i);
        }
    }
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
        if (j < k) {
            const float wj = __shfl_sync(kFull, w, j);
#pragma unroll
            for (int i = 0; i < kU; ++i)
                if (v0 + 32 * i < vpr)
                    fma8<kHalf>(acc[i], wj, v[j][i]);
        }
    }
}

template <bool kHalf>
__global__ void __launch_bounds__(kThreads)
combine_kernel(const uint4* __restrict__ y, int64_t y_rows, const float* __restrict__ weights,
               int T, int k, int64_t vpr, const int32_t* __restrict__ dst_row,
               uint4* __restrict__ out, int32_t* err)
{
    const int lane = threadIdx.x & 31;
    const int64_t wg = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * kThreads) >> 5;
    const int64_t unit_vec = 32 * kU;
    const int64_t upr = (vpr + unit_vec - 1) / unit_vec;
    const int64_t units = (int64_t)T * upr;
    // Before the wait: the expert-output rows of this warp's first unit into
    // L2.  The rows come from dst_row as it reads now (the layout was written
    // before the kernel ahead of this one started); whatever it reads, only
    // prefetch addresses depend on it, checked against y_rows.
    if (wg < units) {
        const int64_t t0 = wg / upr;
        const int64_t v0 = (wg - t0 * upr) * unit_vec + lane;
        const int d0 = lane < k ? ld_early(dst_row + t0 * k + lane) : -1;
        for (int j = 0; j < k; ++j) {
            const int dj = __shfl_sync(kFull, d0, j);
            if (dj >= 0 && dj < y_rows)
#pragma unroll
                for (int i = 0; i < kU; ++i)
                    if (v0 + 32 * i < vpr)
                        prefetch_l2(y + (int64_t)dj * vpr + v0 + 32 * i);
        }
    }
    pdl_wait();
    pdl_trigger();

    for (int64_t u = wg; u < units; u += nw) {
        const int64_t t = u / upr;
        const int64_t v0 = (u - t * upr) * unit_vec + lane;
        int d = -1;
        float w = 0.0f;
        if (lane < k) {
            d = __ldg(dst_row + t * k + lane);
            w = weights ? __ldg(weights + t * k + lane) : 1.0f;  // null: unit weights
        }
        if (d >= y_rows) {
            atomicOr(err, kErrCombineCap);
            d = -1;
        }
        const bool all_valid = __all_sync(kFull, lane >= k || d >= 0);

        float acc[kU][8];
#pragma unroll
        for (int i = 0; i < kU; ++i)
#pragma unroll
            for (int c = 0; c < 8; ++c) acc[i][c] = 0.0f;

        if (all_valid && k <= 8) {
            combine_unit_all_valid<8, kHalf>(y, vpr, k, d, w, v0, acc);
        } else {
            for (int j = 0; j < k; ++j) {
                const int dj = __shfl_sync(kFull, d, j);
                const float wj = __shfl_sync(kFull, w, j);
                if (dj < 0)
                    continue;
                const uint4* row = y + (int64_t)dj * vpr;
                uint4 v[kU];
#pragma unroll
                for (int i = 0; i < kU; ++i)
                    if (v0 + 32 * i < vpr)
                        v[i] = __ldcs(row + v0 + 32 * i);
#pragma unroll
                for (int i = 0; i < kU; ++i)
                    if (v0 + 32 * i < vpr)
                        fma8<kHalf>(acc[i], wj, v[i]);
            }
        }

        uint4* o = out + t * vpr;
#pragma unroll
        for (int i = 0; i < kU; ++i)
            if (v0 + 32 * i < vpr) {
                uint4 r;
                r.x = pack16x2<kHalf>(acc[i][0], acc[i][1]);
                r.y = pack16x2<kHalf>(acc[i][2], acc[i][3]);
                r.z = pack16x2<kHalf>(acc[i][4], acc[i][5]);
                r.w = pack16x2<kHalf>(acc[i][6], acc[i][7]);
                o[v0 + 32 * i] = r;
            }
    }
}

}  // namespace

cudaError_t launch_combine(const Handle& h, const void* y, int64_t y_rows, const float* w,
                           int H, void* out, bool half, cudaStream_t s)
{
    if (h.T == 0)
        return cudaSuccess;
    auto kern = half ? combine_kernel<true> : combine_kernel<false>;
    int grid = 0;
    cudaError_t rc = persistent_grid((const void*)kern, kThreads, 0, 8, &grid);
    if (rc != cudaSuccess)
        return rc;
    return launch_pdl(kern, grid, kThreads, 0, s, static_cast<const uint4*>(y), y_rows, w, h.T,
                      h.k, (int64_t)H / 8, h.dst_row, static_cast<uint4*>(out), h.err);
}

}  // namespace ep
