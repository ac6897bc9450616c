// ep_backward.cu -- gradients of dispatch and combine on sm_100a.
//
// The pages name training as a use of expert-parallel dispatch/combine
// ("DeepEP：让大模型「专家们」高效协作的通信高速公路", section 核心使用场景;
// "DeepEP是什麼？…", high-throughput mode for training and prefill) without
// defining gradients.  These are the gradients of the forward definitions:
//
//   dispatch backward: grad_x[t] = sum over used slots of grad_recv[dst_row[t][j]],
//     fp32 in slot order j = 0..k-1, rounded to the 16-bit type (bf16 or
//     fp16) -- the combine kernel with unit weights (ep_combine.cu);
//   combine backward:  grad_y[dst_row[t][j]] = rn16(w[t][j] * grad_out[t])
//                      grad_w[t][j] = sum_h grad_out[t][h] * y[dst_row[t][j]][h]
//     (this file).
//
// combine_backward_v32_kernel (rows in 32-byte vectors, the common case) is
// described where it is defined.  combine_backward_kernel (16-byte rows):
// one CTA per token.  Each thread takes 16-byte
// vectors of the row (8 channels), reads grad_out once and the k rows of y,
// writes the k scaled rows of grad_y and keeps k fp32 partial dot products
// (fused multiply-adds, its channels in order).  The partials are reduced
// with a fixed xor-shuffle tree inside each warp and then in warp order, so
// the result is bitwise repeatable (its rounding differs from a sequential
// sum by at most the fp32 summation bound).  Slots are taken 8 at a time.
// HBM traffic per token: 2H + 2kH read, 2kH written (+ 4k bytes of grad_w).
#include <cuda_bf16.h>

#include <algorithm>

#include "ep_dispatch_units.cuh"
#include "ep_internal.cuh"

namespace ep {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kMaxThreads = 256;
constexpr int kSlotBatch = 8;

template <bool kHalf>
__global__ void __launch_bounds__(kMaxThreads)
combine_backward_kernel(const uint4* __restrict__ grad_out, const uint4* __restrict__ y,
                        int64_t y_rows, const float* __restrict__ weights, int T, int k,
                        int64_t vpr, const int32_t* __restrict__ dst_row,
                        uint4* __restrict__ grad_y, int64_t grad_y_rows,
                        float* __restrict__ grad_w, int32_t* err)
{
    __shared__ int32_t s_row[EP_MAX_TOPK];
    __shared__ float s_w[EP_MAX_TOPK];
    __shared__ float s_red[kMaxThreads / 32][kSlotBatch];
    pdl_wait();
    pdl_trigger();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = blockDim.x >> 5;
    const int64_t t = blockIdx.x;
    if (t >= T)
        return;
    if ((int)threadIdx.x < k) {
        int32_t d = dst_row[t * k + threadIdx.x];
        if (d >= y_rows || d >= grad_y_rows) {
            atomicOr(err, kErrCombineCap);
            d = -1;
        }
        s_row[threadIdx.x] = d;
        s_w[threadIdx.x] = weights[t * k + threadIdx.x];
    }
    __syncthreads();
    const uint4* g_row = grad_out + t * vpr;

    for (int j0 = 0; j0 < k; j0 += kSlotBatch) {
        const int nj = min(kSlotBatch, k - j0);
        float part[kSlotBatch];
#pragma unroll
        for (int jj = 0; jj < kSlotBatch; ++jj) part[jj] = 0.0f;
        for (int64_t v = threadIdx.x; v < vpr; v += blockDim.x) {
            const uint4 gv = g_row[v];
            const float g[8] = {lo16<kHalf>(gv.x), hi16<kHalf>(gv.x), lo16<kHalf>(gv.y), hi16<kHalf>(gv.y),
                                lo16<kHalf>(gv.z), hi16<kHalf>(gv.z), lo16<kHalf>(gv.w), hi16<kHalf>(gv.w)};
            uint4 yv[kSlotBatch];
#pragma unroll
            for (int jj = 0; jj < kSlotBatch; ++jj) {
                const int d = jj < nj ? s_row[j0 + jj] : -1;
                if (d >= 0)
                    yv[jj] = __ldcs(y + (int64_t)d * vpr + v);
            }
#pragma unroll
            for (int jj = 0; jj < kSlotBatch; ++jj) {
                const int d = jj < nj ? s_row[j0 + jj] : -1;
                if (d < 0)
                    continue;
                const float f[8] = {lo16<kHalf>(yv[jj].x), hi16<kHalf>(yv[jj].x), lo16<kHalf>(yv[jj].y),
                                    hi16<kHalf>(yv[jj].y), lo16<kHalf>(yv[jj].z), hi16<kHalf>(yv[jj].z),
                                    lo16<kHalf>(yv[jj].w), hi16<kHalf>(yv[jj].w)};
#pragma unroll
                for (int c = 0; c < 8; ++c) part[jj] = __fmaf_rn(g[c], f[c], part[jj]);
                const float w = s_w[j0 + jj];
                uint4 o;
                o.x = pack16x2<kHalf>(__fmul_rn(w, g[0]), __fmul_rn(w, g[1]));
                o.y = pack16x2<kHalf>(__fmul_rn(w, g[2]), __fmul_rn(w, g[3]));
                o.z = pack16x2<kHalf>(__fmul_rn(w, g[4]), __fmul_rn(w, g[5]));
                o.w = pack16x2<kHalf>(__fmul_rn(w, g[6]), __fmul_rn(w, g[7]));
                grad_y[(int64_t)d * vpr + v] = o;
            }
        }
        // fixed-order reduction: xor tree in the warp, then warps in order
#pragma unroll
        for (int jj = 0; jj < kSlotBatch; ++jj)
            for (int o = 16; o > 0; o >>= 1) part[jj] += __shfl_xor_sync(kFull, part[jj], o);
        if (lane == 0)
#pragma unroll
            for (int jj = 0; jj < kSlotBatch; ++jj) s_red[warp][jj] = part[jj];
        __syncthreads();
        if ((int)threadIdx.x < nj) {
            float sum = 0.0f;
            for (int w = 0; w < nwarps; ++w) sum += s_red[w][threadIdx.x];
            grad_w[t * k + j0 + threadIdx.x] = s_row[j0 + threadIdx.x] >= 0 ? sum : 0.0f;
        }
        __syncthreads();
    }
}

// 32-byte vectors, one warp per token (rows 32-byte aligned, H % 16 == 0):
// the token's row is walked in 512-channel units, one vector per lane.  Per
// unit the lane loads grad_out's vector and the vectors of the (up to 8)
// slots of the batch before using any, writes the scaled vectors of grad_y
// (one fp32 product, bf16 round to nearest even: bit-exact) and adds its 16
// products per slot to that slot's partial dot (units in order, channels in
// order).  A fixed xor-shuffle tree then sums the 32 partials of each slot,
// so grad_w is bitwise repeatable; no block barrier is needed.
template <bool kHalf>
__global__ void __launch_bounds__(256)
combine_backward_v32_kernel(const units::Vec32* __restrict__ grad_out,
                            const units::Vec32* __restrict__ y, int64_t y_rows,
                            const float* __restrict__ weights, int T, int k, int64_t vpr,
                            const int32_t* __restrict__ dst_row, units::Vec32* __restrict__ grad_y,
                            int64_t grad_y_rows, float* __restrict__ grad_w, int32_t* err)
{
    using units::Vec32;
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (t >= T)
        return;
    int d = -1;
    float w = 0.0f;
    if (lane < k) {
        d = __ldg(dst_row + t * k + lane);
        w = __ldg(weights + t * k + lane);
        if (d >= y_rows || d >= grad_y_rows) {
            atomicOr(err, kErrCombineCap);
            d = -1;
        }
    }
    const int64_t upr = (vpr + 31) / 32;
    const Vec32* g_row = grad_out + t * vpr;
    for (int j0 = 0; j0 < k; j0 += kSlotBatch) {
        const int nj = min(kSlotBatch, k - j0);
        int dj[kSlotBatch];
        float wj[kSlotBatch], part[kSlotBatch];
#pragma unroll
        for (int jj = 0; jj < kSlotBatch; ++jj) {
            dj[jj] = __shfl_sync(kFull, d, (j0 + jj) & 31);
            wj[jj] = __shfl_sync(kFull, w, (j0 + jj) & 31);
            if (jj >= nj)
                dj[jj] = -1;
            part[jj] = 0.0f;
        }
        for (int64_t u = 0; u < upr; ++u) {
            const int64_t v = u * 32 + lane;
            if (v >= vpr)
                continue;  // only the last unit is ragged; no shuffles below
            const Vec32 gv = units::ld32_once(g_row + v);
            Vec32 yv[kSlotBatch];
#pragma unroll
            for (int jj = 0; jj < kSlotBatch; ++jj)
                if (dj[jj] >= 0)
                    yv[jj] = units::ld32_once(y + (int64_t)dj[jj] * vpr + v);
            float g[16];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                g[2 * c] = lo16<kHalf>(gv.w[c]);
                g[2 * c + 1] = hi16<kHalf>(gv.w[c]);
            }
#pragma unroll
            for (int jj = 0; jj < kSlotBatch; ++jj) {
                if (dj[jj] < 0)
                    continue;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    part[jj] = __fmaf_rn(g[2 * c], lo16<kHalf>(yv[jj].w[c]), part[jj]);
                    part[jj] = __fmaf_rn(g[2 * c + 1], hi16<kHalf>(yv[jj].w[c]), part[jj]);
                }
                Vec32 o;
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    o.w[c] = pack16x2<kHalf>(__fmul_rn(wj[jj], g[2 * c]), __fmul_rn(wj[jj], g[2 * c + 1]));
                units::st32(grad_y + (int64_t)dj[jj] * vpr + v, o);
            }
        }
        // fixed-order reduction over the lanes
#pragma unroll
        for (int jj = 0; jj < kSlotBatch; ++jj)
            for (int o = 16; o > 0; o >>= 1) part[jj] += __shfl_xor_sync(kFull, part[jj], o);
#pragma unroll
        for (int jj = 0; jj < kSlotBatch; ++jj)
            if (lane == jj && jj < nj)
                grad_w[t * k + j0 + jj] = dj[jj] >= 0 ? part[jj] : 0.0f;
    }
}

}  // namespace

cudaError_t launch_combine_backward(const Handle& h, const void* grad_out, const void* y,
                                    int64_t y_rows, const float* w, int H, void* grad_y,
                                    int64_t grad_y_rows, float* grad_w, bool half, cudaStream_t s)
{
    if (h.T == 0)
        return cudaSuccess;
    if (H % 16 == 0 && ((uintptr_t)grad_out & 31u) == 0 && ((uintptr_t)y & 31u) == 0 &&
        ((uintptr_t)grad_y & 31u) == 0) {
        const unsigned grid = (unsigned)((h.T + 7) / 8);  // one warp per token
        auto kern = half ? combine_backward_v32_kernel<true> : combine_backward_v32_kernel<false>;
        return launch_pdl(kern, grid, 256u, 0, s, static_cast<const units::Vec32*>(grad_out),
                          static_cast<const units::Vec32*>(y), y_rows, w, h.T, h.k,
                          (int64_t)H / 16, h.dst_row, static_cast<units::Vec32*>(grad_y),
                          grad_y_rows, grad_w, h.err);
    }
    const int64_t vpr = H / 8;
    const int threads = (int)std::min<int64_t>(kMaxThreads, 32 * ((vpr + 31) / 32));
    auto kern = half ? combine_backward_kernel<true> : combine_backward_kernel<false>;
    return launch_pdl(kern, (unsigned)h.T, (unsigned)threads, 0, s,
                      static_cast<const uint4*>(grad_out), static_cast<const uint4*>(y), y_rows, w,
                      h.T, h.k, vpr, h.dst_row, static_cast<uint4*>(grad_y), grad_y_rows, grad_w,
                      h.err);
}

}  // namespace ep
