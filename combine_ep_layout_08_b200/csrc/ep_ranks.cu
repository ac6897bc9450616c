// ep_ranks.cu -- dispatch and combine with the receive layout split into one
// buffer per rank: the expert-parallel form of the path.
//
// The pages describe dispatch as an all-to-all that sends each token to the
// GPUs holding its top-k experts, and combine as the reverse exchange plus
// the weighted reduction ("DeepEP是什麼？MoE Dispatch、Combine、All-to-all與V2
// 架構", stage table of section "MoE為什麼需要All-to-all"); each rank holds
// E / R experts (same page, same section).  With every rank's topk_idx
// gathered in rank order, the layout over the concatenated tokens IS the
// expert-parallel layout: rank p's receive buffer is rows [rank_off[p],
// rank_off[p+1]) of it, renumbered from 0.  So these kernels take the global
// layout (ep_layout over all ranks' tokens) and a table of R receive
// buffers -- on R GPUs, peer pointers into each rank's buffer -- and write
// (dispatch) or read (combine) row d at base[p] + (d - rank_off[p]) rows,
// p = the rank whose block holds d.  The source rank passes its own token
// range [t_begin, t_begin + t_count) of the global order.
//
// Data movement per row is that of ep_dispatch / ep_combine; the only extra
// work is finding p (a binary search of rank_off in shared memory, once per
// slot) and carrying a 64-bit row pointer per slot instead of a row index.
#include <algorithm>

#include "ep_dispatch_units.cuh"
#include "ep_internal.cuh"

namespace ep {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kThreads = 256;

using units::Vec32;

// A 16-byte read-only load that skips L1 (the expert outputs are read once
// per slot and not written while the kernel runs).
__device__ __forceinline__ uint4 ld16_once(const void* p)
{
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// rank_off of the layout (R + 1 words) into shared memory.
__device__ __forceinline__ void load_rank_off(const int32_t* rank_off, int R, int32_t* s_roff)
{
    for (int r = threadIdx.x; r <= R; r += blockDim.x) s_roff[r] = rank_off[r];
    __syncthreads();
}

// The rank whose block holds row d: the largest p with rank_off[p] <= d
// (empty ranks share their offset with the next rank and are skipped by
// taking the largest such p).
__device__ __forceinline__ int rank_of_row(const int32_t* s_roff, int R, int32_t d)
{
    int lo = 0, hi = R - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_roff[mid] <= d)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

// Lane j < k: the row of slot j as (rank, row in that rank's buffer), or
// rank -1 for an unused slot or a row past its rank's capacity (flagged).
__device__ __forceinline__ int slot_rank(const int32_t* __restrict__ dst_row, int64_t t, int k,
                                         const int32_t* s_roff, int R, const RankTable& tab,
                                         int32_t err_bit, int32_t* err, int64_t* local)
{
    const int lane = threadIdx.x & 31;
    int p = -1;
    *local = 0;
    if (lane < k) {
        const int32_t d = __ldg(dst_row + t * k + lane);
        if (d >= 0) {
            p = rank_of_row(s_roff, R, d);
            *local = (int64_t)d - s_roff[p];
            if (*local >= tab.rows[p]) {
                atomicOr(err, err_bit);
                p = -1;
            }
        }
    }
    return p;
}

// BF16 / FP16 row copy, 32-byte vectors, one 512-channel unit per warp.
__global__ void __launch_bounds__(kThreads)
dispatch_ranks_copy_kernel(const Vec32* __restrict__ x, int T, int k, int64_t vpr,
                           const int32_t* __restrict__ dst_row, const int32_t* __restrict__ rank_off,
                           int R, RankTable tab, int32_t* err)
{
    extern __shared__ int32_t s_roff[];
    pdl_wait();
    pdl_trigger();
    load_rank_off(rank_off, R, s_roff);
    const int lane = threadIdx.x & 31;
    const int64_t wg = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * kThreads) >> 5;
    const int64_t upr = (vpr + units::kUnitVec32 - 1) / units::kUnitVec32;
    for (int64_t u = wg; u < (int64_t)T * upr; u += nw) {
        const int64_t t = u / upr;
        int64_t local;
        const int p = slot_rank(dst_row, t, k, s_roff, R, tab, kErrDispatchCap, err, &local);
        const uint64_t rowp =
            p >= 0 ? (uint64_t)(static_cast<Vec32*>(tab.base[p]) + local * vpr) : 0ull;
        const int64_t v = (u - t * upr) * units::kUnitVec32 + lane;
        Vec32 val;
        if (v < vpr)
            val = units::ld32_once(x + t * vpr + v);
        for (int j = 0; j < k; ++j) {
            const uint64_t rj = __shfl_sync(kFull, rowp, j);
            if (rj != 0ull && v < vpr)
                units::st32(reinterpret_cast<Vec32*>(rj) + v, val);
        }
    }
}

// FP8 e4m3 1x128 (row-major scales), 32-byte input vectors, one 512-channel
// unit (4 blocks) per warp: the quantisation of units::fp8_store, writing
// through per-slot row pointers.
template <bool kHalf>
__global__ void __launch_bounds__(kThreads)
dispatch_ranks_fp8_kernel(const Vec32* __restrict__ x, int T, int k, int H,
                          const int32_t* __restrict__ dst_row, const int32_t* __restrict__ rank_off,
                          int R, RankTable tab, int32_t* err)
{
    extern __shared__ int32_t s_roff[];
    pdl_wait();
    pdl_trigger();
    load_rank_off(rank_off, R, s_roff);
    const int lane = threadIdx.x & 31;
    const int64_t wg = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * kThreads) >> 5;
    const int64_t vpr = H / 16;
    const int nblk = H / 128;
    const int64_t upr = (vpr + 31) / 32;
    for (int64_t u = wg; u < (int64_t)T * upr; u += nw) {
        const int64_t t = u / upr;
        const int64_t unit = u - t * upr;
        int64_t local;
        const int p = slot_rank(dst_row, t, k, s_roff, R, tab, kErrDispatchCap, err, &local);
        const uint64_t qrow =
            p >= 0 ? (uint64_t)(static_cast<uint8_t*>(tab.base[p]) + local * H) : 0ull;
        const uint64_t srow = p >= 0 ? (uint64_t)(tab.scales[p] + local * nblk) : 0ull;
        Vec32 a[1];
        units::fp8_load<1>(x + t * vpr, vpr, unit, a);
        uint4 q[1];
        float my_scale;
        units::fp8_quantize<1, kHalf>(a, q, my_scale);
        const int64_t v = unit * 32 + lane;
        const int64_t blk = unit * 4 + lane;
        const bool sc_ok = lane < 4 && blk < nblk;
        for (int j = 0; j < k; ++j) {
            const uint64_t qj = __shfl_sync(kFull, qrow, j);
            const uint64_t sj = __shfl_sync(kFull, srow, j);
            if (qj == 0ull)
                continue;
            if (v < vpr)
                reinterpret_cast<uint4*>(qj)[v] = q[0];
            if (sc_ok)
                reinterpret_cast<float*>(sj)[blk] = my_scale;
        }
    }
}

// Combine: the rows of each token's slots gathered from the ranks' y buffers
// (16-byte vectors, 512-channel units, persistent grid), fp32 fused
// multiply-add in slot order j = 0..k-1, rounded to the 16-bit type --
// ep_combine's arithmetic.  All loads of a unit are issued before the first
// multiply-add.
template <bool kHalf>
__global__ void __launch_bounds__(kThreads)
combine_ranks_kernel(const float* __restrict__ weights, int T, int k, int64_t vpr,
                     const int32_t* __restrict__ dst_row, const int32_t* __restrict__ rank_off,
                     int R, RankTable tab, uint4* __restrict__ out, int32_t* err)
{
    extern __shared__ int32_t s_roff[];
    pdl_wait();
    pdl_trigger();
    load_rank_off(rank_off, R, s_roff);
    constexpr int kU = 2;  // 16-byte vectors per lane per unit
    constexpr int kBatch = 8;
    const int lane = threadIdx.x & 31;
    const int64_t wg = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * kThreads) >> 5;
    const int64_t upr = (vpr + 32 * kU - 1) / (32 * kU);
    for (int64_t u = wg; u < (int64_t)T * upr; u += nw) {
        const int64_t t = u / upr;
        const int64_t v0 = (u - t * upr) * (32 * kU) + lane;
        // null weights: unit weights (the backward of dispatch)
        const float w = lane < k ? (weights ? __ldg(weights + t * k + lane) : 1.0f) : 0.0f;
        int64_t local;
        const int p = slot_rank(dst_row, t, k, s_roff, R, tab, kErrCombineCap, err, &local);
        const uint64_t rowp =
            p >= 0 ? (uint64_t)(static_cast<const uint4*>(tab.base[p]) + local * vpr) : 0ull;
        float acc[kU][8];
#pragma unroll
        for (int i = 0; i < kU; ++i)
#pragma unroll
            for (int c = 0; c < 8; ++c) acc[i][c] = 0.0f;
        for (int j0 = 0; j0 < k; j0 += kBatch) {
            // all row pointers of the batch first, then all loads, then the
            // multiply-adds in slot order
            uint64_t rj[kBatch];
            float wj[kBatch];
#pragma unroll
            for (int jj = 0; jj < kBatch; ++jj) {
                rj[jj] = __shfl_sync(kFull, rowp, (j0 + jj) & 31);
                wj[jj] = __shfl_sync(kFull, w, (j0 + jj) & 31);
                if (j0 + jj >= k)
                    rj[jj] = 0ull;
            }
            uint4 val[kBatch][kU];
#pragma unroll
            for (int jj = 0; jj < kBatch; ++jj)
#pragma unroll
                for (int i = 0; i < kU; ++i)
                    if (rj[jj] != 0ull && v0 + 32 * i < vpr)
                        val[jj][i] = ld16_once(reinterpret_cast<const uint4*>(rj[jj]) + v0 + 32 * i);
#pragma unroll
            for (int jj = 0; jj < kBatch; ++jj) {
                if (rj[jj] == 0ull)
                    continue;
#pragma unroll
                for (int i = 0; i < kU; ++i) {
                    if (v0 + 32 * i >= vpr)
                        continue;
                    const uint4 y = val[jj][i];
                    const uint32_t wd[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        acc[i][2 * c] = __fmaf_rn(wj[jj], lo16<kHalf>(wd[c]), acc[i][2 * c]);
                        acc[i][2 * c + 1] =
                            __fmaf_rn(wj[jj], hi16<kHalf>(wd[c]), acc[i][2 * c + 1]);
                    }
                }
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

// Backward of the per-rank combine, one warp per token (32-byte vectors):
// grad_y of slot j, in its rank's grad_y buffer, = rn16(w[t][j] * grad_out[t])
// (one fp32 product: bit-exact), and grad_w[t][j] = the fp32 dot product of
// grad_out[t] with the slot's expert-output row, read from its rank's y
// buffer -- units in order, channels in order within the lane, then a fixed
// xor-shuffle tree over the lanes (bitwise repeatable).  ytab and gytab hold
// the ranks' y and grad_y buffers.
template <bool kHalf>
__global__ void __launch_bounds__(kThreads, 2)
combine_ranks_backward_kernel(const Vec32* __restrict__ grad_out, const float* __restrict__ weights,
                              int T, int k, int64_t vpr, const int32_t* __restrict__ dst_row,
                              const int32_t* __restrict__ rank_off, int R, RankTable ytab,
                              RankTable gytab, float* __restrict__ grad_w, int32_t* err)
{
    extern __shared__ int32_t s_roff[];
    pdl_wait();
    pdl_trigger();
    load_rank_off(rank_off, R, s_roff);
    constexpr int kBatch = 8;
    const int lane = threadIdx.x & 31;
    const int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (t >= T)
        return;
    float w = 0.0f;
    uint64_t yrow = 0ull, gyrow = 0ull;
    if (lane < k) {
        w = __ldg(weights + t * k + lane);
        const int32_t d = __ldg(dst_row + t * k + lane);
        if (d >= 0) {
            const int p = rank_of_row(s_roff, R, d);
            const int64_t local = (int64_t)d - s_roff[p];
            if (local >= ytab.rows[p] || local >= gytab.rows[p]) {
                atomicOr(err, kErrCombineCap);
            } else {
                yrow = (uint64_t)(static_cast<const Vec32*>(ytab.base[p]) + local * vpr);
                gyrow = (uint64_t)(static_cast<Vec32*>(gytab.base[p]) + local * vpr);
            }
        }
    }
    const int64_t upr = (vpr + 31) / 32;
    const Vec32* g_row = grad_out + t * vpr;
    for (int j0 = 0; j0 < k; j0 += kBatch) {
        const int nj = min(kBatch, k - j0);
        uint64_t yj[kBatch], gj[kBatch];
        float wj[kBatch], part[kBatch];
#pragma unroll
        for (int jj = 0; jj < kBatch; ++jj) {
            yj[jj] = __shfl_sync(kFull, yrow, (j0 + jj) & 31);
            gj[jj] = __shfl_sync(kFull, gyrow, (j0 + jj) & 31);
            wj[jj] = __shfl_sync(kFull, w, (j0 + jj) & 31);
            if (jj >= nj)
                yj[jj] = 0ull;
            part[jj] = 0.0f;
        }
        for (int64_t u = 0; u < upr; ++u) {
            const int64_t v = u * 32 + lane;
            if (v >= vpr)
                continue;  // only the last unit is ragged; no shuffles below
            const Vec32 gv = units::ld32_once(g_row + v);
            Vec32 yv[kBatch];
#pragma unroll
            for (int jj = 0; jj < kBatch; ++jj)
                if (yj[jj] != 0ull)
                    yv[jj] = units::ld32_once(reinterpret_cast<const Vec32*>(yj[jj]) + v);
            float g[16];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                g[2 * c] = lo16<kHalf>(gv.w[c]);
                g[2 * c + 1] = hi16<kHalf>(gv.w[c]);
            }
#pragma unroll
            for (int jj = 0; jj < kBatch; ++jj) {
                if (yj[jj] == 0ull)
                    continue;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    part[jj] = __fmaf_rn(g[2 * c], lo16<kHalf>(yv[jj].w[c]), part[jj]);
                    part[jj] = __fmaf_rn(g[2 * c + 1], hi16<kHalf>(yv[jj].w[c]), part[jj]);
                }
                Vec32 o;
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    o.w[c] = pack16x2<kHalf>(__fmul_rn(wj[jj], g[2 * c]),
                                             __fmul_rn(wj[jj], g[2 * c + 1]));
                units::st32(reinterpret_cast<Vec32*>(gj[jj]) + v, o);
            }
        }
#pragma unroll
        for (int jj = 0; jj < kBatch; ++jj)
            for (int o = 16; o > 0; o >>= 1) part[jj] += __shfl_xor_sync(kFull, part[jj], o);
#pragma unroll
        for (int jj = 0; jj < kBatch; ++jj)
            if (lane == jj && jj < nj)
                grad_w[t * k + j0 + jj] = yj[jj] != 0ull ? part[jj] : 0.0f;
    }
}

unsigned warp_grid(int64_t units)
{
    const int64_t warps = kThreads / 32;
    return (unsigned)std::min<int64_t>(1 << 20, std::max<int64_t>(1, (units + warps - 1) / warps));
}

}  // namespace

cudaError_t launch_dispatch_ranks(const Handle& h, const void* x, int H, bool fp8, bool half,
                                  const RankTable& tab, cudaStream_t s)
{
    if (h.T == 0)
        return cudaSuccess;
    const size_t smem = sizeof(int32_t) * (size_t)(h.R + 1);
    const int64_t vpr = H / 16;
    if (!fp8)
        return launch_pdl(dispatch_ranks_copy_kernel, warp_grid(h.T * ((vpr + 31) / 32)), kThreads,
                          smem, s, static_cast<const Vec32*>(x), h.T, h.k, vpr, h.dst_row,
                          h.rank_off, h.R, tab, h.err);
    auto kern = half ? dispatch_ranks_fp8_kernel<true> : dispatch_ranks_fp8_kernel<false>;
    return launch_pdl(kern, warp_grid(h.T * ((vpr + 31) / 32)), kThreads, smem, s,
                      static_cast<const Vec32*>(x), h.T, h.k, H, h.dst_row, h.rank_off, h.R, tab,
                      h.err);
}

cudaError_t launch_combine_ranks_backward(const Handle& h, const void* grad_out, const float* w,
                                          int H, bool half, const RankTable& ytab,
                                          const RankTable& gytab, float* grad_w, cudaStream_t s)
{
    if (h.T == 0)
        return cudaSuccess;
    const size_t smem = sizeof(int32_t) * (size_t)(h.R + 1);
    auto kern = half ? combine_ranks_backward_kernel<true> : combine_ranks_backward_kernel<false>;
    const unsigned grid = (unsigned)((h.T + 7) / 8);  // one warp per token
    return launch_pdl(kern, grid, kThreads, smem, s, static_cast<const Vec32*>(grad_out), w, h.T,
                      h.k, (int64_t)H / 16, h.dst_row, h.rank_off, h.R, ytab, gytab, grad_w,
                      h.err);
}

cudaError_t launch_combine_ranks(const Handle& h, const float* w, int H, bool half,
                                 const RankTable& tab, void* out, cudaStream_t s)
{
    if (h.T == 0)
        return cudaSuccess;
    const size_t smem = sizeof(int32_t) * (size_t)(h.R + 1);
    auto kern = half ? combine_ranks_kernel<true> : combine_ranks_kernel<false>;
    int grid = 0;
    cudaError_t rc = persistent_grid((const void*)kern, kThreads, smem, 4, &grid);
    if (rc != cudaSuccess)
        return rc;
    return launch_pdl(kern, grid, kThreads, smem, s, w, h.T, h.k, (int64_t)H / 8, h.dst_row,
                      h.rank_off, h.R, tab, static_cast<uint4*>(out), h.err);
}

}  // namespace ep
