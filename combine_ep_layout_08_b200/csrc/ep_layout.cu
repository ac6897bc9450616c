// ep_layout.cu -- get_dispatch_layout on sm_100a.
//
// The layout is a stable counting sort of the flat (token, slot) entries of
// topk_idx by expert, followed by per-expert padding to block_m rows.  The
// pages name the sorting and the imbalance as the costs of dispatch ("DeepEP
// 是什麼？MoE Dispatch、Combine、All-to-all與V2架構", stage table of section
// "MoE為什麼需要All-to-all", column 瓶頸) and place the "dispatch layout" in
// the buffer object (same page, section ElasticBuffer); the reading of the
// layout itself is stated in ep.h.
//
// Positions must be deterministic (order inside an expert block is by source
// token, then slot), so they are never taken from atomics.  Three launches:
//   K1 count   one warp per chunk of 32 tokens: shared-memory histogram of
//              the chunk's experts, is_token_in_rank bytes, per-chunk count
//              of tokens per rank;
//   K2 scan    per expert, exclusive prefix of the chunk counts over chunks
//              (in place), per-expert totals and per-rank token totals;
//   K3 assign  every CTA scans the padded expert sizes into expert_off; each
//              warp replays its chunk in order, ranking equal experts inside
//              each group of 32 entries with __match_any_sync, to give
//              dst_row and recv_src; pad rows of recv_src are set to -1.
// Integer shared-memory atomics are used only for counts, whose sums do not
// depend on order.
#include <algorithm>

#include "ep_internal.cuh"

namespace ep {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kScanThreads = 1024;
constexpr size_t kSmemBudget = 200 * 1024;

__device__ __forceinline__ unsigned lanemask_lt()
{
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

__device__ __forceinline__ int32_t pad_up(int32_t c, int32_t b) { return ((c + b - 1) / b) * b; }

// K1.  Shared memory per warp: hist[E], rank_hist[R], entry_rank[32 k].
__global__ void layout_count_kernel(const int64_t* __restrict__ topk_idx, int T, int k, int E,
                                    int R, int epr, int64_t nchunks,
                                    int32_t* __restrict__ chunk_counts,
                                    int32_t* __restrict__ chunk_rank,
                                    uint8_t* __restrict__ is_token_in_rank, int32_t* err)
{
    extern __shared__ int32_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int per_warp = E + R + kChunkTokens * k;
    int32_t* hist = smem + (size_t)warp * per_warp;
    int32_t* rhist = hist + E;
    int32_t* erank = rhist + R;

    const int64_t c = (int64_t)blockIdx.x * (blockDim.x >> 5) + warp;
    if (c >= nchunks)
        return;  // the whole warp leaves; no block barrier follows
    const int64_t t0 = c * kChunkTokens;
    const int ntok = (int)min((int64_t)kChunkTokens, (int64_t)T - t0);
    const int nent = ntok * k;

    for (int e = lane; e < E; e += 32) hist[e] = 0;
    for (int r = lane; r < R; r += 32) rhist[r] = 0;
    __syncwarp();

    const int64_t* src = topk_idx + t0 * k;
    int bad = 0;
    for (int f = lane; f < nent; f += 32) {
        const int64_t v = src[f];
        int e = -1;
        if (v >= 0 && v < E)
            e = (int)v;
        else if (v != -1)
            bad = 1;
        erank[f] = e >= 0 ? e / epr : -1;
        if (e >= 0)
            atomicAdd(&hist[e], 1);
    }
    if (__any_sync(kFull, bad) && lane == 0)
        atomicOr(err, kErrBadIndex);
    __syncwarp();

    // is_token_in_rank bytes of the chunk, p = t * R + r: consecutive lanes
    // write consecutive bytes.
    for (int p = lane; p < ntok * R; p += 32) {
        const int t = p / R, r = p - t * R;
        int hit = 0;
        for (int j = 0; j < k; ++j) hit |= (erank[t * k + j] == r);
        is_token_in_rank[(t0 + t) * R + r] = (uint8_t)hit;
        if (hit)
            atomicAdd(&rhist[r], 1);
    }
    __syncwarp();

    for (int e = lane; e < E; e += 32) chunk_counts[c * E + e] = hist[e];
    for (int r = lane; r < R; r += 32) chunk_rank[c * R + r] = rhist[r];
}

// K2.  Blocks [0, ceil(E/32)) own 32 experts each, the rest 32 ranks each;
// lane = column, warp w = a contiguous range of chunks.
__global__ void __launch_bounds__(kScanThreads)
layout_scan_kernel(int32_t* __restrict__ chunk_counts, const int32_t* __restrict__ chunk_rank,
                   int E, int R, int64_t nchunks, int32_t* __restrict__ cnt,
                   int32_t* __restrict__ tokens_per_rank)
{
    __shared__ int32_t part[32][33];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int eblocks = (E + 31) / 32;
    const bool is_expert = (int)blockIdx.x < eblocks;
    const int ncol = is_expert ? E : R;
    const int col = (is_expert ? (int)blockIdx.x : (int)blockIdx.x - eblocks) * 32 + lane;
    const bool colok = col < ncol;
    const int32_t* M = is_expert ? chunk_counts : chunk_rank;

    const int64_t rpw = (nchunks + 31) / 32;
    const int64_t r0 = min(nchunks, (int64_t)warp * rpw);
    const int64_t r1 = min(nchunks, r0 + rpw);

    int32_t sum = 0;
    if (colok)
        for (int64_t r = r0; r < r1; ++r) sum += M[r * ncol + col];
    part[warp][lane] = sum;
    __syncthreads();

    int32_t pre = 0, total = 0;
    for (int w = 0; w < 32; ++w) {
        const int32_t v = part[w][lane];
        pre += (w < warp) ? v : 0;
        total += v;
    }
    if (is_expert && colok) {
        int32_t run = pre;
        for (int64_t r = r0; r < r1; ++r) {
            const int32_t v = chunk_counts[r * ncol + col];
            chunk_counts[r * ncol + col] = run;
            run += v;
        }
    }
    if (warp == 0 && colok) {
        if (is_expert)
            cnt[col] = total;
        else
            tokens_per_rank[col] = total;
    }
}

// K3.  Shared memory: off[E+1], warp totals[32], then run[E] per warp.
__global__ void layout_assign_kernel(const int64_t* __restrict__ topk_idx, int T, int k, int E,
                                     int R, int epr, int block_m, int64_t nchunks,
                                     const int32_t* __restrict__ chunk_prefix,
                                     const int32_t* __restrict__ cnt,
                                     int32_t* __restrict__ expert_off_g,
                                     int32_t* __restrict__ rank_off_g,
                                     int32_t* __restrict__ rows_per_rank_g,
                                     int32_t* __restrict__ total_rows_g,
                                     int32_t* __restrict__ dst_row,
                                     int32_t* __restrict__ recv_src)
{
    extern __shared__ int32_t smem[];
    int32_t* off = smem;
    int32_t* wsum = off + E + 1;
    int32_t* run_all = wsum + 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = blockDim.x >> 5;
    const int nthr = blockDim.x;

    // Block-wide exclusive scan of pad(cnt[e]): contiguous segment per thread.
    const int seg = (E + nthr - 1) / nthr;
    const int e0 = min(E, (int)threadIdx.x * seg), e1 = min(E, e0 + seg);
    int32_t local = 0;
    for (int e = e0; e < e1; ++e) local += pad_up(cnt[e], block_m);
    int32_t incl = local;
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t v = __shfl_up_sync(kFull, incl, o);
        if (lane >= o)
            incl += v;
    }
    if (lane == 31)
        wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int32_t v = lane < nwarps ? wsum[lane] : 0;
        int32_t inc = v;
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t u = __shfl_up_sync(kFull, inc, o);
            if (lane >= o)
                inc += u;
        }
        if (lane < nwarps)
            wsum[lane] = inc - v;
    }
    __syncthreads();
    int32_t run = wsum[warp] + incl - local;
    for (int e = e0; e < e1; ++e) {
        off[e] = run;
        run += pad_up(cnt[e], block_m);
    }
    if ((int)threadIdx.x == nthr - 1)
        off[E] = run;
    __syncthreads();

    if (blockIdx.x == 0) {
        for (int e = threadIdx.x; e <= E; e += nthr) expert_off_g[e] = off[e];
        for (int r = threadIdx.x; r <= R; r += nthr) rank_off_g[r] = off[r * epr];
        for (int r = threadIdx.x; r < R; r += nthr) {
            int32_t s = 0;
            for (int e = r * epr; e < (r + 1) * epr; ++e) s += cnt[e];
            rows_per_rank_g[r] = s;
        }
        if (threadIdx.x == 0)
            *total_rows_g = off[E];
    }

    // Pad rows of the experts this CTA owns.
    for (int e = blockIdx.x; e < E; e += gridDim.x)
        for (int32_t r = off[e] + cnt[e] + (int32_t)threadIdx.x; r < off[e + 1]; r += nthr)
            recv_src[r] = -1;

    const int64_t c = (int64_t)blockIdx.x * nwarps + warp;
    if (c >= nchunks)
        return;  // no block barrier follows
    int32_t* runc = run_all + (size_t)warp * E;
    for (int e = lane; e < E; e += 32) runc[e] = off[e] + chunk_prefix[c * E + e];
    __syncwarp();

    const int64_t t0 = c * kChunkTokens;
    const int ntok = (int)min((int64_t)kChunkTokens, (int64_t)T - t0);
    const int nent = ntok * k;
    const int64_t* src = topk_idx + t0 * k;
    const unsigned lt = lanemask_lt();
    for (int g = 0; g < nent; g += 32) {
        const int f = g + lane;
        int e = -2;  // lanes past the chunk end
        if (f < nent) {
            const int64_t v = src[f];
            e = (v >= 0 && v < E) ? (int)v : -1;
        }
        const unsigned peers = __match_any_sync(kFull, e);
        int pos = -1;
        if (e >= 0)
            pos = runc[e] + __popc(peers & lt);
        __syncwarp();
        if (e >= 0 && (peers & lt) == 0)
            runc[e] += __popc(peers);
        __syncwarp();
        if (f < nent) {
            dst_row[t0 * k + f] = pos;
            if (pos >= 0)
                recv_src[pos] = (int32_t)(t0 + f / k);
        }
    }
}

int warps_for(size_t per_warp_bytes, size_t fixed_bytes)
{
    size_t w = 4;
    while (w > 1 && fixed_bytes + w * per_warp_bytes > kSmemBudget) --w;
    return (int)w;
}

cudaError_t set_smem(const void* fn, size_t bytes)
{
    if (bytes <= 48 * 1024)
        return cudaSuccess;
    return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

}  // namespace

cudaError_t launch_layout(const Handle& h, const int64_t* topk_idx, int T, cudaStream_t s)
{
    const int k = h.k, E = h.E, R = h.R, epr = h.E / h.R;
    const int64_t nchunks = ((int64_t)T + kChunkTokens - 1) / kChunkTokens;
    cudaError_t rc;

    if (nchunks > 0) {
        const size_t per_warp = sizeof(int32_t) * (size_t)(E + R + kChunkTokens * k);
        const int w1 = warps_for(per_warp, 0);
        const size_t smem1 = per_warp * w1;
        if ((rc = set_smem((const void*)layout_count_kernel, smem1)) != cudaSuccess)
            return rc;
        const unsigned g1 = (unsigned)((nchunks + w1 - 1) / w1);
        layout_count_kernel<<<g1, 32 * w1, smem1, s>>>(topk_idx, T, k, E, R, epr, nchunks,
                                                       h.chunk_counts, h.chunk_rank,
                                                       h.is_token_in_rank, h.err);
        if ((rc = cudaGetLastError()) != cudaSuccess)
            return rc;
    }

    const unsigned g2 = (unsigned)((E + 31) / 32 + (R + 31) / 32);
    layout_scan_kernel<<<g2, kScanThreads, 0, s>>>(h.chunk_counts, h.chunk_rank, E, R, nchunks,
                                                   h.cnt, h.tokens_per_rank);
    if ((rc = cudaGetLastError()) != cudaSuccess)
        return rc;

    const size_t fixed3 = sizeof(int32_t) * (size_t)(E + 1 + 32);
    const size_t per_warp3 = sizeof(int32_t) * (size_t)E;
    const int w3 = warps_for(per_warp3, fixed3);
    const size_t smem3 = fixed3 + per_warp3 * w3;
    if ((rc = set_smem((const void*)layout_assign_kernel, smem3)) != cudaSuccess)
        return rc;
    const unsigned g3 = (unsigned)std::max<int64_t>(1, (nchunks + w3 - 1) / w3);
    layout_assign_kernel<<<g3, 32 * w3, smem3, s>>>(
        topk_idx, T, k, E, R, epr, h.block_m, nchunks, h.chunk_counts, h.cnt, h.expert_off,
        h.rank_off, h.rows_per_rank, h.total_rows, h.dst_row, h.recv_src);
    return cudaGetLastError();
}

}  // namespace ep
