// ep_dispatch_units.cuh -- the per-unit bodies of the 256-bit dispatch
// kernels, shared by ep_dispatch.cu and the fused layout + dispatch kernel.
// The operation is dispatch as the stage table of "DeepEP是什麼？…" (section
// MoE為什麼需要All-to-all) defines it, with the FP8 form read from that page's
// FP8與低精度通訊 section (one fp32 scale per 128 channels, s = amax / 448).
// A unit is one warp's share of one token row: BF16 512 channels (32 lanes x
// one 32-byte vector), FP8 512 kU channels (32 lanes x kU 32-byte vectors =
// 4 kU blocks of 128; kU = 2 in the dispatch kernels, 1 in the fused
// small-batch kernel, where more and shorter units spread the latency).  `d` is this lane's destination row for slot j = lane
// (lanes >= k, unused slots and rows beyond the capacity pass -1).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "ep_internal.cuh"

namespace ep {
namespace units {

constexpr unsigned kFull = 0xffffffffu;

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

constexpr int kUnitVec32 = 32;      // BF16 unit: 32 vectors x 16 channels = 512 channels
constexpr int kU32Fp8 = 2;          // FP8 unit of the dispatch kernels: 2 vectors per lane
constexpr int kUnitVec32Fp8 = 32 * kU32Fp8;  // 64 vectors = 1024 channels = 8 blocks

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

// BF16: the lane's 32-byte vector of the unit is read once and written to
// each of the k destination rows; consecutive lanes write consecutive bytes.
// bf16_store takes the vector already loaded (v = the lane's vector index in
// the row).
__device__ __forceinline__ void bf16_store(const Vec32& val, int64_t v, int64_t vpr, int d, int k,
                                           Vec32* __restrict__ recv)
{
    for (int j = 0; j < k; ++j) {
        const int dj = __shfl_sync(kFull, d, j);
        if (dj >= 0 && v < vpr)
            st32(recv + (int64_t)dj * vpr + v, val);
    }
}

__device__ __forceinline__ void bf16_unit(const Vec32* __restrict__ xs, int64_t vpr, int64_t unit,
                                          int d, int k, Vec32* __restrict__ recv)
{
    const int lane = threadIdx.x & 31;
    const int64_t v = unit * kUnitVec32 + lane;
    Vec32 val;
    if (v < vpr)
        val = ld32_once(xs + v);
    bf16_store(val, v, vpr, d, k, recv);
}

// FP8: lane vector i of the unit covers channels 16 v .. 16 v + 15 with
// v = unit * 32 kU + 32 i + lane, so each 128-channel block is one group of 8
// lanes (xor 4, 2, 1 reduction) and the unit's blocks 4i .. 4i + 3 sit in
// lane groups 0-3 of vector i.  Each lane writes its 16 codes as one 16-byte
// store; the unit's 4 kU scales are gathered into lanes 0 .. 4 kU - 1 and
// written as one run per destination row (row-major scales).  xs: the token
// x / s rounded to nearest even (binary32) for the quantiser's scale
// s = amax / 448 and |x| <= amax, given r = 1 / s rounded to nearest:
// q0 = x r, then one correction with the exact remainder x - q0 s (one FMA),
// q = q0 + (x - q0 s) r.  This is Markstein's division (P. Markstein,
// "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34(1), 1990), three operations per element
// instead of a full division.  Checked on the host for every pair of
// BF16 or FP16 values (amax, x) with |x| <= amax and s >= kFastScaleMin:
// the quotient equals IEEE division's, except quotients of magnitude at most
// 2^-10 on both sides, which convert to the same E4M3 zero (of x's sign,
// hence the copysign).  Smaller or non-finite scales take IEEE division.
constexpr float kFastScaleMin = 0x1p-100f;

__device__ __forceinline__ bool fast_scale(float s)
{
    return s >= kFastScaleMin && s <= 3.40282347e38f;
}

__device__ __forceinline__ float div_by_scale(float x, float s, float r)
{
    const float q0 = __fmul_rn(x, r);
    const float rem = __fmaf_rn(-q0, s, x);
    return copysignf(__fmaf_rn(rem, r, q0), x);
}

// N quotients x / s (s > 0), as IEEE division gives them where it matters
// for E4M3 (see div_by_scale).
template <int N>
__device__ __forceinline__ void div_n_by_scale(const float (&f)[N], float s, float (&v)[N])
{
    if (fast_scale(s)) {
        const float r = __frcp_rn(s);
#pragma unroll
        for (int c = 0; c < N; ++c) v[c] = div_by_scale(f[c], s, r);
    } else {
#pragma unroll
        for (int c = 0; c < N; ++c) v[c] = __fdiv_rn(f[c], s);
    }
}

// row in 32-byte vectors, vpr = H / 16.
// The lane's kU vectors of the unit, zero past the end of the row.
template <int kU>
__device__ __forceinline__ void fp8_load(const Vec32* __restrict__ xs, int64_t vpr, int64_t unit,
                                         Vec32 (&a)[kU])
{
    const int lane = threadIdx.x & 31;
    const int64_t v0 = unit * (32 * kU) + lane;
#pragma unroll
    for (int i = 0; i < kU; ++i) {
        if (v0 + 32 * i < vpr) {
            a[i] = ld32_once(xs + v0 + 32 * i);
        } else {
#pragma unroll
            for (int c = 0; c < 8; ++c) a[i].w[c] = 0u;
        }
    }
}

// Quantise the loaded vectors (bfloat16, or binary16 when kHalf): the lane's
// codes q and, in lanes 0 .. 4 kU - 1, the scale of the unit's block L.
template <int kU, bool kHalf = false>
__device__ __forceinline__ void fp8_quantize(const Vec32 (&a)[kU], uint4 (&q)[kU],
                                             float& my_scale)
{
    const int lane = threadIdx.x & 31;
    float sc[kU];
#pragma unroll
    for (int i = 0; i < kU; ++i) {
        float f[16];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            f[2 * c] = lo16<kHalf>(a[i].w[c]);
            f[2 * c + 1] = hi16<kHalf>(a[i].w[c]);
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
            float v[16];
            div_n_by_scale<16>(f, s, v);
            q[i].x = e4m3x4(v[0], v[1], v[2], v[3]);
            q[i].y = e4m3x4(v[4], v[5], v[6], v[7]);
            q[i].z = e4m3x4(v[8], v[9], v[10], v[11]);
            q[i].w = e4m3x4(v[12], v[13], v[14], v[15]);
        }
    }
    // lane L < 8 takes the scale of block L of the unit: vector L / 4, lane
    // group L % 4 (leader lane 8 (L % 4))
    my_scale = 0.0f;
#pragma unroll
    for (int i = 0; i < kU; ++i) {
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            const float sv = __shfl_sync(kFull, sc[i], 8 * g);
            if (lane == 4 * i + g)
                my_scale = sv;
        }
    }
}

// Quantise the loaded vectors and write codes and scales to the k rows.
template <int kU, bool kHalf = false>
__device__ __forceinline__ void fp8_store(const Vec32 (&a)[kU], int64_t vpr, int64_t unit, int d,
                                          int k, int H, uint8_t* __restrict__ recv_q,
                                          float* __restrict__ recv_scales, int64_t scales_ld)
{
    const int lane = threadIdx.x & 31;
    const int nblk = H / 128;
    const int64_t v0 = unit * (32 * kU) + lane;
    uint4 q[kU];
    float my_scale;
    fp8_quantize<kU, kHalf>(a, q, my_scale);
    const int64_t blk = unit * (4 * kU) + lane;
    const bool sc_ok = lane < 4 * kU && blk < nblk;
    for (int j = 0; j < k; ++j) {
        const int dj = __shfl_sync(kFull, d, j);
        if (dj < 0)
            continue;
        uint4* dq = reinterpret_cast<uint4*>(recv_q + (int64_t)dj * H);
#pragma unroll
        for (int i = 0; i < kU; ++i)
            if (v0 + 32 * i < vpr)
                dq[v0 + 32 * i] = q[i];
        if (sc_ok)
            recv_scales[scale_index(dj, blk, nblk, scales_ld)] = my_scale;
    }
}

template <int kU = kU32Fp8, bool kHalf = false>
__device__ __forceinline__ void fp8_unit(const Vec32* __restrict__ xs, int64_t vpr, int64_t unit,
                                         int d, int k, int H, uint8_t* __restrict__ recv_q,
                                         float* __restrict__ recv_scales, int64_t scales_ld)
{
    Vec32 a[kU];
    fp8_load<kU>(xs, vpr, unit, a);
    fp8_store<kU, kHalf>(a, vpr, unit, d, k, H, recv_q, recv_scales, scales_ld);
}

}  // namespace units
}  // namespace ep
