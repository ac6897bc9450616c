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
// Both kernels are HBM-bound streams (read 2H bytes per token, write k rows),
// and dispatch is write-dominated (k row writes per row read).  Work unit: one
// warp x (token, 2 KiB of bf16 input = 1024 channels); each lane loads its
// vectors of the unit up front (x is read once: no L1 allocation), then
// writes them to the k destination rows; consecutive lanes write consecutive
// bytes of a row, so every store instruction covers whole 32-byte sectors.
// The main kernels move 32-byte vectors (sm_100's 256-bit ld/st.global.v8),
// halving the store instructions of 16-byte vectors; 16-byte kernels remain
// for rows that are not 32-byte multiples.  The grid gives every warp one
// unit (a grid-stride loop covers grids beyond kMaxGrid): measured on B200,
// a persistent single wave, in which every warp loads and then stores in
// lock step with all the others, reaches ~5.4 TB/s; two waves 5.8; one unit
// per warp, whose CTAs start and retire staggered, 6.1 TB/s.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include <algorithm>

#include "ep_internal.cuh"

namespace ep {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kThreads = 256;
constexpr int kU = 4;               // 16-byte input vectors per lane per unit
constexpr int kUnitVec = 32 * kU;   // input vectors (8 channels each) per unit

__device__ __forceinline__ uint4 ld_once(const uint4* p) { return __ldcs(p); }

// 32-byte vector and its 256-bit global load (read-once, no L1 allocation)
// and store.
struct alignas(32) Vec32 {
    uint32_t w[8];
};

__device__ __forceinline__ Vec32 ld32_once(const Vec32* p)
{
    Vec32 r;
    asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r.w[0]), "=r"(r.w[1]), "=r"(r.w[2]), "=r"(r.w[3]), "=r"(r.w[4]),
                   "=r"(r.w[5]), "=r"(r.w[6]), "=r"(r.w[7])
                 : "l"(p));
    return r;
}

__device__ __forceinline__ void st32(Vec32* p, const Vec32& v)
{
    asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(v.w[0]),
                 "r"(v.w[1]), "r"(v.w[2]), "r"(v.w[3]), "r"(v.w[4]), "r"(v.w[5]), "r"(v.w[6]),
                 "r"(v.w[7])
                 : "memory");
}

constexpr int kU32 = 1;                 // 32-byte vectors per lane per BF16 unit
constexpr int kUnitVec32 = 32 * kU32;   // 32 vectors x 16 channels = 512 channels
constexpr int kU32Fp8 = 2;              // FP8 unit: 64 vectors = 1024 channels = 8 blocks
constexpr int kUnitVec32Fp8 = 32 * kU32Fp8;
constexpr int64_t kMaxGrid = 1 << 20;

// BF16 dispatch with 32-byte vectors; vpr = H / 16.
__global__ void __launch_bounds__(kThreads, 8)
dispatch_bf16_v32_kernel(const Vec32* __restrict__ x, int T, int k, int64_t vpr,
                         const int32_t* __restrict__ dst_row, Vec32* __restrict__ recv,
                         int64_t cap_rows, int32_t* err)
{
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int64_t wg = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * kThreads) >> 5;
    const int64_t upr = (vpr + kUnitVec32 - 1) / kUnitVec32;
    const int64_t units = (int64_t)T * upr;

    for (int64_t u = wg; u < units; u += nw) {
        const int64_t t = u / upr;
        const int64_t v0 = (u - t * upr) * kUnitVec32 + lane;
        int d = lane < k ? __ldg(dst_row + t * k + lane) : -1;
        if (d >= cap_rows) {
            atomicOr(err, kErrDispatchCap);
            d = -1;
        }
        const Vec32* xs = x + t * vpr;
        Vec32 v[kU32];
#pragma unroll
        for (int i = 0; i < kU32; ++i)
            if (v0 + 32 * i < vpr)
                v[i] = ld32_once(xs + v0 + 32 * i);
        for (int j = 0; j < k; ++j) {
            const int dj = __shfl_sync(kFull, d, j);
            if (dj < 0)
                continue;
            Vec32* dst = recv + (int64_t)dj * vpr;
#pragma unroll
            for (int i = 0; i < kU32; ++i)
                if (v0 + 32 * i < vpr)
                    st32(dst + v0 + 32 * i, v[i]);
        }
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

// Scale of (row, block): row-major [row][nblk] when ld == 0, else MN-major
// [block][ld] (each block's scales contiguous over rows, for GEMMs that read
// scales along M).
__device__ __forceinline__ int64_t scale_index(int64_t row, int64_t blk, int nblk, int64_t ld)
{
    return ld == 0 ? row * nblk + blk : blk * ld + row;
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
                recv_scales[scale_index(dj, blk, nblk, scales_ld)] = my_scale;
        }
    }
}


// FP8 with 32-byte input vectors: lane vector i of a unit covers channels
// 16 v .. 16 v + 15 with v = unit * 64 + 32 i + lane, so each 128-channel
// block is one group of 8 lanes (xor 4, 2, 1 reduction) and a unit's blocks
// 4i .. 4i + 3 sit in lane groups 0-3 of vector i.  Each lane writes its 16
// codes as one 16-byte store; the unit's 8 scales are gathered into lanes 0-7
// and written as one 32-byte run per destination row.
__global__ void __launch_bounds__(kThreads)
dispatch_fp8_v32_kernel(const Vec32* __restrict__ x, int T, int k, int H,
                        const int32_t* __restrict__ dst_row, uint8_t* __restrict__ recv_q,
                        float* __restrict__ recv_scales, int64_t scales_ld, int64_t cap_rows,
                        int32_t* err)
{
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int64_t wg = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * kThreads) >> 5;
    const int64_t vpr = H / 16;
    const int nblk = H / 128;
    const int64_t upr = (vpr + kUnitVec32Fp8 - 1) / kUnitVec32Fp8;
    const int64_t units = (int64_t)T * upr;

    for (int64_t u = wg; u < units; u += nw) {
        const int64_t t = u / upr;
        const int64_t unit = u - t * upr;
        const int64_t v0 = unit * kUnitVec32Fp8 + lane;
        int d = lane < k ? __ldg(dst_row + t * k + lane) : -1;
        if (d >= cap_rows) {
            atomicOr(err, kErrDispatchCap);
            d = -1;
        }
        const Vec32* xs = x + t * vpr;
        Vec32 a[kU32Fp8];
#pragma unroll
        for (int i = 0; i < kU32Fp8; ++i) {
            if (v0 + 32 * i < vpr) {
                a[i] = ld32_once(xs + v0 + 32 * i);
            } else {
#pragma unroll
                for (int c = 0; c < 8; ++c) a[i].w[c] = 0u;
            }
        }

        uint4 q[kU32Fp8];
        float sc[kU32Fp8];
#pragma unroll
        for (int i = 0; i < kU32Fp8; ++i) {
            float f[16];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                f[2 * c] = bf16_lo(a[i].w[c]);
                f[2 * c + 1] = bf16_hi(a[i].w[c]);
            }
            float m = 0.0f;
#pragma unroll
            for (int c = 0; c < 16; ++c) m = fmaxf(m, fabsf(f[c]));
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 4));
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 2));
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 1));
            if (m == 0.0f) {
                sc[i] = 0.0f;
                q[i] = make_uint4(0u, 0u, 0u, 0u);
            } else {
                const float s = __fdiv_rn(m, 448.0f);
                sc[i] = s;
                q[i].x = e4m3x4(__fdiv_rn(f[0], s), __fdiv_rn(f[1], s), __fdiv_rn(f[2], s),
                                __fdiv_rn(f[3], s));
                q[i].y = e4m3x4(__fdiv_rn(f[4], s), __fdiv_rn(f[5], s), __fdiv_rn(f[6], s),
                                __fdiv_rn(f[7], s));
                q[i].z = e4m3x4(__fdiv_rn(f[8], s), __fdiv_rn(f[9], s), __fdiv_rn(f[10], s),
                                __fdiv_rn(f[11], s));
                q[i].w = e4m3x4(__fdiv_rn(f[12], s), __fdiv_rn(f[13], s), __fdiv_rn(f[14], s),
                                __fdiv_rn(f[15], s));
            }
        }
        // lane L < 8 takes the scale of block L of the unit: vector L / 4,
        // lane group L % 4 (leader lane 8 (L % 4))
        float my_scale = 0.0f;
#pragma unroll
        for (int i = 0; i < kU32Fp8; ++i) {
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                const float sv = __shfl_sync(kFull, sc[i], 8 * g);
                if (lane == 4 * i + g)
                    my_scale = sv;
            }
        }
        const int64_t blk = unit * (4 * kU32Fp8) + lane;
        const bool sc_ok = lane < 4 * kU32Fp8 && blk < nblk;

        for (int j = 0; j < k; ++j) {
            const int dj = __shfl_sync(kFull, d, j);
            if (dj < 0)
                continue;
            uint4* dq = reinterpret_cast<uint4*>(recv_q + (int64_t)dj * H);
#pragma unroll
            for (int i = 0; i < kU32Fp8; ++i)
                if (v0 + 32 * i < vpr)
                    dq[v0 + 32 * i] = q[i];
            if (sc_ok)
                recv_scales[scale_index(dj, blk, nblk, scales_ld)] = my_scale;
        }
    }
}

bool aligned32(const void* p) { return ((uintptr_t)p & 31u) == 0; }

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
    if (H % 16 == 0 && aligned32(x) && aligned32(recv_x))
        return launch_pdl(dispatch_bf16_v32_kernel, unit_grid(h.T, H / 16, kUnitVec32), kThreads,
                          0, s, static_cast<const Vec32*>(x), h.T, h.k, (int64_t)H / 16,
                          h.dst_row, static_cast<Vec32*>(recv_x), cap_rows, h.err);
    return launch_pdl(dispatch_bf16_kernel, unit_grid(h.T, H / 8, kUnitVec), kThreads, 0, s,
                      static_cast<const uint4*>(x), h.T, h.k, (int64_t)H / 8, h.dst_row,
                      static_cast<uint4*>(recv_x), cap_rows, h.err);
}

cudaError_t launch_dispatch_fp8(const Handle& h, const void* x, int H, void* recv_q,
                                float* recv_scales, int64_t scales_ld, int64_t cap_rows,
                                cudaStream_t s)
{
    if (h.T == 0)
        return cudaSuccess;
    if (aligned32(x))
        return launch_pdl(dispatch_fp8_v32_kernel, unit_grid(h.T, H / 16, kUnitVec32Fp8),
                          kThreads, 0, s, static_cast<const Vec32*>(x), h.T, h.k, H, h.dst_row,
                          static_cast<uint8_t*>(recv_q), recv_scales, scales_ld, cap_rows,
                          h.err);
    return launch_pdl(dispatch_fp8_kernel, unit_grid(h.T, H / 8, kUnitVec), kThreads, 0, s,
                      static_cast<const uint4*>(x), h.T, h.k, H, h.dst_row,
                      static_cast<uint8_t*>(recv_q), recv_scales, scales_ld, cap_rows, h.err);
}

}  // namespace ep
