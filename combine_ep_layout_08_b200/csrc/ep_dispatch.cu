// ep_dispatch.cu -- dispatch on sm_100a: scatter of token rows into the
// expert-major receive buffer, as a copy of the 16-bit rows (BF16 or FP16)
// or with fused FP8 e4m3 1x128 quantisation of BF16 or FP16 rows.
//
// Dispatch sends every token to its top-k experts ("DeepEP是什麼？MoE
// Dispatch、Combine、All-to-all與V2架構", stage table of section
// "MoE為什麼需要All-to-all"); the volume of the stage is
// batch x top_k x hidden x sizeof(dtype) ("DeepEP 编址服务深度对抗分析",
// section 五.2), i.e. one row write per (token, slot).  FP8 lowers the bytes
// written (yololab page, FP8 section); its scale granularity and formula are
// the reading stated in ep.h.
//
// Both kernels are HBM-bound streams (read 2H bytes per token, write k rows),
// and dispatch is write-dominated (k row writes per row read).  Work unit: one
// warp x (token, 512 channels for the copy, 1024 channels = 8 FP8 blocks for
// FP8); each lane loads its vectors of the unit up front (x is read once: no
// L1 allocation), then writes them to the k destination rows; consecutive
// lanes write consecutive bytes of a row, so every store instruction covers
// whole 32-byte sectors.  (Halving the FP8 unit measured slower at every
// batch size tried, 4096 and 8192 tokens.)
// The main kernels move 32-byte vectors (sm_100's 256-bit ld/st.global.v8),
// halving the store instructions of 16-byte vectors; 16-byte kernels remain
// for rows that are not 32-byte multiples.  Before the dependent-launch wait
// each warp of the main kernels prefetches its unit of x into L2 (x does not
// depend on the layout; a prefetch returns no data), so the loads after the
// wait find it there: measured 1.5 us less per launch at 8192 tokens.  The
// first wave's warps also prefetch the x of the next few waves (about 36 MB,
// evict_last) while the layout ahead still runs and HBM is otherwise idle:
// 4-5 us less per step at 8192 tokens (BF16) and at the DeepSeek-V3 shape
// (FP8); with the default L2 priority the row stores evicted those lines
// before use and the step got slower.  The grid gives every warp one
// unit (a grid-stride loop covers grids beyond kMaxGrid): measured on B200,
// a persistent single wave, in which every warp loads and then stores in
// lock step with all the others, reaches ~5.4 TB/s; two waves 5.8; one unit
// per warp, whose CTAs start and retire staggered, 6.1 TB/s.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "ep_dispatch_units.cuh"

#include <algorithm>

#include "ep_internal.cuh"

namespace ep {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kThreads = 256;
constexpr int kU = 4;               // 16-byte input vectors per lane per unit
constexpr int kUnitVec = 32 * kU;   // input vectors (8 channels each) per unit

__device__ __forceinline__ uint4 ld_once(const uint4* p) { return __ldcs(p); }

using units::Vec32;
using units::kUnitVec32;
using units::kUnitVec32Fp8;
constexpr int64_t kMaxGrid = 1 << 20;

// A hint that brings a line into L2; it reads nothing, so it may be issued
// before the dependent-launch wait (the data it fetches is never used
// directly: the loads after the wait see the memory as it is then).
__device__ __forceinline__ void prefetch_l2(const void* p)
{
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// The same with the L2 eviction priority evict_last, so that the row stores
// streaming through L2 meanwhile do not push the line out before it is read.
__device__ __forceinline__ void prefetch_l2_last(const void* p)
{
    asm volatile("prefetch.global.L2::evict_last [%0];" ::"l"(p));
}

// Before the dependent-launch wait: the x of this warp's first unit into L2,
// and, for the warps of the first wave (warp index < stride), the units
// stride, 2 stride, ..., waves x stride ahead of it, which the later waves
// of the grid will read (evict_last).  A unit is kVecs 32-byte vectors per
// lane of one token row (upr units per row).  Prefetches return no data:
// the loads after the wait read the memory as it is then.
template <int kVecs>
__device__ __forceinline__ void prefetch_x(const Vec32* x, int64_t vpr, int64_t upr,
                                           int64_t nunits, int64_t stride, int waves)
{
    const int64_t wg0 = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    for (int w = 0; w <= waves; ++w) {
        if (w > 0 && wg0 >= stride)
            break;
        const int64_t u = wg0 + (int64_t)w * stride;
        if (u >= nunits)
            break;
        const int64_t t = u / upr;
        const int64_t v = (u - t * upr) * (32 * kVecs) + lane;
#pragma unroll
        for (int i = 0; i < kVecs; ++i)
            if (v + 32 * i < vpr) {
                if (w == 0)
                    prefetch_l2(x + t * vpr + v + 32 * i);
                else
                    prefetch_l2_last(x + t * vpr + v + 32 * i);
            }
    }
}

// BF16 dispatch with 32-byte vectors; vpr = H / 16.
__global__ void __launch_bounds__(kThreads, 8)
dispatch_bf16_v32_kernel(const Vec32* __restrict__ x, int T, int k, int64_t vpr,
                         const int32_t* __restrict__ dst_row, Vec32* __restrict__ recv,
                         int64_t cap_rows, int32_t* err, int64_t pf_stride, int pf_waves)
{
    const int64_t upr0 = (vpr + kUnitVec32 - 1) / kUnitVec32;
    prefetch_x<1>(x, vpr, upr0, (int64_t)T * upr0, pf_stride, pf_waves);
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int64_t wg = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * kThreads) >> 5;
    const int64_t upr = (vpr + kUnitVec32 - 1) / kUnitVec32;
    const int64_t nunits = (int64_t)T * upr;
    for (int64_t u = wg; u < nunits; u += nw) {
        const int64_t t = u / upr;
        int d = lane < k ? __ldg(dst_row + t * k + lane) : -1;
        if (d >= cap_rows) {
            atomicOr(err, kErrDispatchCap);
            d = -1;
        }
        units::bf16_unit(x + t * vpr, vpr, u - t * upr, d, k, recv);
    }
}

__global__ void __launch_bounds__(kThreads)
dispatch_bf16_kernel(const uint4* __restrict__ x, int T, int k, int64_t vpr,
                     const int32_t* __restrict__ dst_row, uint4* __restrict__ recv,
                     int64_t cap_rows, int32_t* err)
{
    pdl_wait();
    pdl_trigger();
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

using units::e4m3x4;
using units::scale_index;

// FP8: a unit's lane vector i covers channels 8 v .. 8 v + 7 with
// v = unit * 128 + 32 i + lane, so lanes 0-15 hold block 2i of the unit and
// lanes 16-31 block 2i + 1; the block amax is a 16-lane xor reduction.  The
// 8 scales of a unit are gathered into lanes 0-7 and written as one 32-byte
// run per destination row.
template <bool kHalf>
__global__ void __launch_bounds__(kThreads)
dispatch_fp8_kernel(const uint4* __restrict__ x, int T, int k, int H,
                    const int32_t* __restrict__ dst_row, uint8_t* __restrict__ recv_q,
                    float* __restrict__ recv_scales, int64_t scales_ld, int64_t cap_rows,
                    int32_t* err)
{
    pdl_wait();
    pdl_trigger();
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
            float f[8] = {lo16<kHalf>(a[i].x), hi16<kHalf>(a[i].x), lo16<kHalf>(a[i].y),
                          hi16<kHalf>(a[i].y), lo16<kHalf>(a[i].z), hi16<kHalf>(a[i].z),
                          lo16<kHalf>(a[i].w), hi16<kHalf>(a[i].w)};
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
                float v[8];
                units::div_n_by_scale<8>(f, s, v);
                q[i].x = e4m3x4(v[0], v[1], v[2], v[3]);
                q[i].y = e4m3x4(v[4], v[5], v[6], v[7]);
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
                recv_scales[scale_index(dj, blk, nblk, scales_ld)] = my_scale;
        }
    }
}


// FP8 with 32-byte input vectors (units::fp8_unit); vpr = H / 16.
template <bool kHalf>
__global__ void __launch_bounds__(kThreads)
dispatch_fp8_v32_kernel(const Vec32* __restrict__ x, int T, int k, int H,
                        const int32_t* __restrict__ dst_row, uint8_t* __restrict__ recv_q,
                        float* __restrict__ recv_scales, int64_t scales_ld, int64_t cap_rows,
                        int32_t* err, int64_t pf_stride, int pf_waves)
{
    {
        const int64_t vpr0 = H / 16;
        const int64_t upr0 = (vpr0 + kUnitVec32Fp8 - 1) / kUnitVec32Fp8;
        prefetch_x<units::kU32Fp8>(x, vpr0, upr0, (int64_t)T * upr0, pf_stride, pf_waves);
    }
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int64_t wg = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * kThreads) >> 5;
    const int64_t vpr = H / 16;
    const int64_t upr = (vpr + kUnitVec32Fp8 - 1) / kUnitVec32Fp8;
    const int64_t nunits = (int64_t)T * upr;
    for (int64_t u = wg; u < nunits; u += nw) {
        const int64_t t = u / upr;
        int d = lane < k ? __ldg(dst_row + t * k + lane) : -1;
        if (d >= cap_rows) {
            atomicOr(err, kErrDispatchCap);
            d = -1;
        }
        units::fp8_unit<units::kU32Fp8, kHalf>(x + t * vpr, vpr, u - t * upr, d, k, H, recv_q,
                                               recv_scales, scales_ld);
    }
}

bool aligned32(const void* p) { return ((uintptr_t)p & 31u) == 0; }

// x bytes the first wave prefetches ahead (about what HBM delivers while the
// layout kernel ahead of the dispatch runs; 29-39 MB measured best at the
// 8k and DeepSeek-V3 shapes, 47 MB and more slower).
constexpr int64_t kPrefetchBudget = 36ll << 20;
constexpr int64_t kMaxPrefetchWaves = 8;  // bounds the loop where few CTAs fit per SM

// The first wave's size in warps (the CTAs resident per SM beside one CTA of
// the kernel ahead, x the SMs) and how many waves ahead of it to prefetch.
cudaError_t prefetch_plan(const void* kernel, int64_t unit_x_bytes, int64_t* stride, int* waves)
{
    int full = 0;
    cudaError_t rc = persistent_grid(kernel, kThreads, 0, 1 << 16, &full);
    if (rc != cudaSuccess)
        return rc;
    int dev = 0, sms = 1;
    if ((rc = cudaGetDevice(&dev)) != cudaSuccess ||
        (rc = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return rc;
    const int64_t ctas = std::max<int64_t>(sms, full - sms);
    *stride = ctas * (kThreads / 32);
    *waves = (int)std::min<int64_t>(kMaxPrefetchWaves,
                                    std::max<int64_t>(0, kPrefetchBudget / (*stride * unit_x_bytes) - 1));
    return cudaSuccess;
}

// One unit per warp: ceil(units / warps per CTA) CTAs, capped at kMaxGrid.
unsigned unit_grid(int64_t T, int64_t vec_per_row, int64_t unit_vec)
{
    const int64_t units = T * ((vec_per_row + unit_vec - 1) / unit_vec);
    const int64_t warps = kThreads / 32;
    return (unsigned)std::min<int64_t>(kMaxGrid, std::max<int64_t>(1, (units + warps - 1) / warps));
}

}  // namespace

cudaError_t launch_dispatch_bf16(const Handle& h, const void* x, int H, void* recv_x,
                                 int64_t cap_rows, cudaStream_t s)
{
    if (h.T == 0)
        return cudaSuccess;
    if (H % 16 == 0 && aligned32(x) && aligned32(recv_x)) {
        int64_t pf_stride = 0;
        int pf_waves = 0;
        cudaError_t rc = prefetch_plan((const void*)dispatch_bf16_v32_kernel,
                                       kUnitVec32 * (int64_t)sizeof(Vec32), &pf_stride, &pf_waves);
        if (rc != cudaSuccess)
            return rc;
        return launch_pdl(dispatch_bf16_v32_kernel, unit_grid(h.T, H / 16, kUnitVec32), kThreads,
                          0, s, static_cast<const Vec32*>(x), h.T, h.k, (int64_t)H / 16,
                          h.dst_row, static_cast<Vec32*>(recv_x), cap_rows, h.err, pf_stride,
                          pf_waves);
    }
    return launch_pdl(dispatch_bf16_kernel, unit_grid(h.T, H / 8, kUnitVec), kThreads, 0, s,
                      static_cast<const uint4*>(x), h.T, h.k, (int64_t)H / 8, h.dst_row,
                      static_cast<uint4*>(recv_x), cap_rows, h.err);
}

cudaError_t launch_dispatch_fp8(const Handle& h, const void* x, int H, void* recv_q,
                                float* recv_scales, int64_t scales_ld, int64_t cap_rows,
                                bool half, cudaStream_t s)
{
    if (h.T == 0)
        return cudaSuccess;
    if (aligned32(x)) {
        auto kern = half ? dispatch_fp8_v32_kernel<true> : dispatch_fp8_v32_kernel<false>;
        int64_t pf_stride = 0;
        int pf_waves = 0;
        cudaError_t rc = prefetch_plan((const void*)kern, kUnitVec32Fp8 * (int64_t)sizeof(Vec32),
                                       &pf_stride, &pf_waves);
        if (rc != cudaSuccess)
            return rc;
        return launch_pdl(kern, unit_grid(h.T, H / 16, kUnitVec32Fp8), kThreads, 0, s,
                          static_cast<const Vec32*>(x), h.T, h.k, H, h.dst_row,
                          static_cast<uint8_t*>(recv_q), recv_scales, scales_ld, cap_rows,
                          h.err, pf_stride, pf_waves);
    }
    auto kern = half ? dispatch_fp8_kernel<true> : dispatch_fp8_kernel<false>;
    return launch_pdl(kern, unit_grid(h.T, H / 8, kUnitVec), kThreads, 0, s,
                      static_cast<const uint4*>(x), h.T, h.k, H, h.dst_row,
                      static_cast<uint8_t*>(recv_q), recv_scales, scales_ld, cap_rows, h.err);
}

}  // namespace ep
