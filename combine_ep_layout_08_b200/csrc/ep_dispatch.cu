// ep_dispatch.cu -- dispatch on sm_100a: scatter of token rows into the
// expert-major receive buffer, as a BF16 copy or with fused FP8 e4m3 1x128
// quantisation.
//
// Dispatch sends every token to its top-k experts ("DeepEP是什麼？MoE
// Dispatch、Combine、All-to-all與V2架構", stage table of section
// "MoE為什麼需要All-to-all"); the volume of the stage is
// batch x top_k x hidden x sizeof(dtype) ("DeepEP 编址服务深度对抗分析",
// section 五.2), i.e. one row write per (token, slot).  FP8 lowers the bytes
// written (yololab page, FP8 section); its scale granularity and formula are
// the reading stated in ep.h.
//
// Both kernels are HBM-bound streams (read 2H bytes per token, write k rows).
// Work unit: one warp x (token, 2 KiB of bf16 input = 1024 channels); each
// lane loads four 16-byte vectors up front (x is read once, with an
// evict-first hint), then writes them to the k destination rows with
// coalesced stores; consecutive lanes write consecutive bytes of a row.  The
// grid is persistent (resident CTAs x SM count) and strides over units, so a
// token's row is spread over several warps and the tail is small.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "ep_internal.cuh"

namespace ep {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kThreads = 256;
constexpr int kU = 4;               // 16-byte input vectors per lane per unit
constexpr int kUnitVec = 32 * kU;   // input vectors (8 channels each) per unit

__device__ __forceinline__ uint4 ld_once(const uint4* p) { return __ldcs(p); }

__global__ void __launch_bounds__(kThreads)
dispatch_bf16_kernel(const uint4* __restrict__ x, int T, int k, int64_t vpr,
                     const int32_t* __restrict__ dst_row, uint4* __restrict__ recv,
                     int64_t cap_rows, int32_t* err)
{
    const int lane = threadIdx.x & 31;
    const int64_t wg = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * kThreads) >> 5;
    const int64_t upr = (vpr + kUnitVec - 1) / kUnitVec;
    const int64_t units = (int64_t)T * upr;

    for (int64_t u = wg; u < units; u += nw) {
        const int64_t t = u / upr;
        const int64_t v0 = (u - t * upr) * kUnitVec + lane;
        int d = lane < k ? __ldg(dst_row + t * k + lane) : -1;
        if (d >= cap_rows) {
            atomicOr(err, kErrDispatchCap);
            d = -1;
        }
        const uint4* xs = x + t * vpr;
        uint4 v[kU];
#pragma unroll
        for (int i = 0; i < kU; ++i)
            if (v0 + 32 * i < vpr)
                v[i] = ld_once(xs + v0 + 32 * i);
        for (int j = 0; j < k; ++j) {
            const int dj = __shfl_sync(kFull, d, j);
            if (dj < 0)
                continue;
            uint4* dst = recv + (int64_t)dj * vpr;
#pragma unroll
            for (int i = 0; i < kU; ++i)
                if (v0 + 32 * i < vpr)
                    dst[v0 + 32 * i] = v[i];
        }
    }
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d)
{
    const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
    const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
    return lo | (hi << 16);
}

// FP8: a unit's lane vector i covers channels 8 v .. 8 v + 7 with
// v = unit * 128 + 32 i + lane, so lanes 0-15 hold block 2i of the unit and
// lanes 16-31 block 2i + 1; the block amax is a 16-lane xor reduction.  The
// 8 scales of a unit are gathered into lanes 0-7 and written as one 32-byte
// run per destination row.
__global__ void __launch_bounds__(kThreads)
dispatch_fp8_kernel(const uint4* __restrict__ x, int T, int k, int H,
                    const int32_t* __restrict__ dst_row, uint8_t* __restrict__ recv_q,
                    float* __restrict__ recv_scales, int64_t cap_rows, int32_t* err)
{
    const int lane = threadIdx.x & 31;
    const int64_t wg = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * kThreads) >> 5;
    const int64_t vpr = H / 8;
    const int nblk = H / 128;
    const int64_t upr = (vpr + kUnitVec - 1) / kUnitVec;
    const int64_t units = (int64_t)T * upr;

    for (int64_t u = wg; u < units; u += nw) {
        const int64_t t = u / upr;
        const int64_t unit = u - t * upr;
        const int64_t v0 = unit * kUnitVec + lane;
        int d = lane < k ? __ldg(dst_row + t * k + lane) : -1;
        if (d >= cap_rows) {
            atomicOr(err, kErrDispatchCap);
            d = -1;
        }
        const uint4* xs = x + t * vpr;
        uint4 a[kU];
#pragma unroll
        for (int i = 0; i < kU; ++i)
            a[i] = (v0 + 32 * i < vpr) ? ld_once(xs + v0 + 32 * i) : make_uint4(0, 0, 0, 0);

        uint2 q[kU];
        float sc[kU];
#pragma unroll
        for (int i = 0; i < kU; ++i) {
            float f[8] = {bf16_lo(a[i].x), bf16_hi(a[i].x), bf16_lo(a[i].y), bf16_hi(a[i].y),
                          bf16_lo(a[i].z), bf16_hi(a[i].z), bf16_lo(a[i].w), bf16_hi(a[i].w)};
            float m = 0.0f;
#pragma unroll
            for (int c = 0; c < 8; ++c) m = fmaxf(m, fabsf(f[c]));
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 8));
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 4));
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 2));
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 1));
            if (m == 0.0f) {
                sc[i] = 0.0f;
                q[i] = make_uint2(0u, 0u);
            } else {
                const float s = __fdiv_rn(m, 448.0f);
                sc[i] = s;
                q[i].x = e4m3x4(__fdiv_rn(f[0], s), __fdiv_rn(f[1], s), __fdiv_rn(f[2], s),
                                __fdiv_rn(f[3], s));
                q[i].y = e4m3x4(__fdiv_rn(f[4], s), __fdiv_rn(f[5], s), __fdiv_rn(f[6], s),
                                __fdiv_rn(f[7], s));
            }
        }
        // lane L < 8 takes the scale of block 2 (L/2) + (L%2) of the unit
        float my_scale = 0.0f;
#pragma unroll
        for (int i = 0; i < kU; ++i) {
            const float s0 = __shfl_sync(kFull, sc[i], 0);
            const float s1 = __shfl_sync(kFull, sc[i], 16);
            if (lane == 2 * i)
                my_scale = s0;
            if (lane == 2 * i + 1)
                my_scale = s1;
        }
        const int64_t blk = unit * (2 * kU) + lane;
        const bool sc_ok = lane < 2 * kU && blk < nblk;

        for (int j = 0; j < k; ++j) {
            const int dj = __shfl_sync(kFull, d, j);
            if (dj < 0)
                continue;
            uint2* dq = reinterpret_cast<uint2*>(recv_q + (int64_t)dj * H);
#pragma unroll
            for (int i = 0; i < kU; ++i)
                if (v0 + 32 * i < vpr)
                    dq[v0 + 32 * i] = q[i];
            if (sc_ok)
                recv_scales[(int64_t)dj * nblk + blk] = my_scale;
        }
    }
}

}  // namespace

cudaError_t launch_dispatch_bf16(const Handle& h, const void* x, int H, void* recv_x,
                                 int64_t cap_rows, cudaStream_t s)
{
    if (h.T == 0)
        return cudaSuccess;
    int grid = 0;
    cudaError_t rc = persistent_grid((const void*)dispatch_bf16_kernel, kThreads, 0, 8, &grid);
    if (rc != cudaSuccess)
        return rc;
    dispatch_bf16_kernel<<<grid, kThreads, 0, s>>>(
        static_cast<const uint4*>(x), h.T, h.k, (int64_t)H / 8, h.dst_row,
        static_cast<uint4*>(recv_x), cap_rows, h.err);
    return cudaGetLastError();
}

cudaError_t launch_dispatch_fp8(const Handle& h, const void* x, int H, void* recv_q,
                                float* recv_scales, int64_t cap_rows, cudaStream_t s)
{
    if (h.T == 0)
        return cudaSuccess;
    int grid = 0;
    cudaError_t rc = persistent_grid((const void*)dispatch_fp8_kernel, kThreads, 0, 8, &grid);
    if (rc != cudaSuccess)
        return rc;
    dispatch_fp8_kernel<<<grid, kThreads, 0, s>>>(static_cast<const uint4*>(x), h.T, h.k, H,
                                                  h.dst_row, static_cast<uint8_t*>(recv_q),
                                                  recv_scales, cap_rows, h.err);
    return cudaGetLastError();
}

}  // namespace ep
