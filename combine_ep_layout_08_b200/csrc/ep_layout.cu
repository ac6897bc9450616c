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
// token, then slot), so they are never taken from atomics: integer
// shared-memory atomics only build histograms, whose sums do not depend on
// order.  Entries are grouped in chunks of 32 tokens, one warp per chunk.
//
// Large batches, three launches:
//   K1 count   per chunk: shared-memory histogram of the chunk's experts,
//              is_token_in_rank bytes, per-chunk count of tokens per rank;
//   K2 scan    per expert, exclusive prefix of the chunk counts over chunks
//              (in place), per-expert totals and per-rank token totals;
//   K3 assign  every CTA scans the padded expert sizes into expert_off; each
//              warp replays its chunk in order, ranking equal experts inside
//              each group of 32 entries by lane (a ballot per key bit), to give
//              dst_row and recv_src; pad rows of recv_src are set to -1.
// Large batches, one launch (the default): layout_tile_kernel runs the three
// phases in one cooperative launch, one tile of tokens per CTA, its CTAs
// separated by a single grid barrier (every CTA then sums all tiles' counts
// itself); the three kernels remain for shapes whose tiles do not fit in
// shared memory and for the static-scratch entry point.
// Small batches (T k <= 4096, E <= 1024, shared memory permitting) run with
// one entry per thread in CTAs of 1024 threads that each compute the whole
// layout (layout_small_kernel).
//
// The work is latency-bound (at 8K tokens the layout reads 0.5 MB), so each
// kernel issues all of its global loads before it uses any of them, and every
// kernel is launched with programmatic dependent launch: it may start while
// its predecessor drains, and waits (griddepcontrol.wait) before it touches
// memory.
#include <algorithm>
#include <atomic>

#include "ep_dispatch_units.cuh"
#include "ep_internal.cuh"

namespace ep {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kScanThreads = 1024;
constexpr size_t kSmemBudget = 200 * 1024;
constexpr int kBatch = 8;  // entries per lane loaded before any is used

__device__ __forceinline__ unsigned lanemask_lt()
{
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Lanes of the warp whose key equals this lane's, for keys in [-1, 2^nbits - 1)
// (nbits uniform over the warp): the AND over the key bits of the matching
// ballot -- nbits ballots, where __match_any_sync slows down with the number
// of distinct keys (up to 32 here).
__device__ __forceinline__ unsigned match_key(int key, int nbits)
{
    const unsigned v = (unsigned)(key + 1);
    unsigned m = kFull;
    for (int b = 0; b < nbits; ++b) {
        const unsigned bit = (v >> b) & 1u;
        const unsigned bal = __ballot_sync(kFull, bit);
        m &= bit ? bal : ~bal;
    }
    return m;
}

__device__ __forceinline__ int32_t pad_up(int32_t c, int32_t b) { return ((c + b - 1) / b) * b; }

// An expert in [0, E), or -1 for an unused slot; anything else is flagged.
__device__ __forceinline__ int to_expert(int64_t v, int E, int& bad)
{
    if (v >= 0 && v < E)
        return (int)v;
    if (v != -1)
        bad = 1;
    return -1;
}

// Block-wide exclusive scan of pad(cnt[e]) into off[0..E] (shared memory).
// cnt may live in global or shared memory.  Uses wsum[32] as scratch.
__device__ void scan_padded(const int32_t* cnt, int E, int block_m, int32_t* off, int32_t* wsum)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = blockDim.x >> 5, nthr = blockDim.x;
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
}

// One warp: is_token_in_rank bytes of a chunk from the entries' ranks
// (erank[t * k + j], -1 for unused); byte p = t * R + r goes to lane p % 32,
// so consecutive lanes write consecutive bytes.  Tokens-per-rank counts are
// added to rhist.  With R <= 32 each token's ranks are first folded into a
// bitmask held by lane t, lane r counts the masks holding rank r (one shuffle
// per token), and each byte is one shuffle; larger R tests the k entries per
// byte.
__device__ __forceinline__ void chunk_rank_bytes(const int32_t* erank, int ntok, int k, int R,
                                                 int64_t t0, uint8_t* is_token_in_rank,
                                                 int32_t* rhist)
{
    const int lane = threadIdx.x & 31;
    const int total = ntok * R;
    const int dt = 32 / R, dr = 32 - (32 / R) * R;  // (t, r) step for p += 32
    int t = lane / R, r = lane - (lane / R) * R;
    if (R <= 32) {
        uint32_t mask = 0;
        if (lane < ntok)
            for (int j = 0; j < k; ++j) {
                const int q = erank[lane * k + j];
                if (q >= 0)
                    mask |= 1u << q;
            }
        // lane q counts the tokens whose mask holds rank q
        int c = 0;
        for (int u = 0; u < ntok; ++u) c += (int)((__shfl_sync(kFull, mask, u) >> lane) & 1u);
        if (lane < R && c)
            atomicAdd(&rhist[lane], c);
        for (int p0 = 0; p0 < total; p0 += 32) {
            const uint32_t m = __shfl_sync(kFull, mask, t & 31);
            if (p0 + lane < total)
                is_token_in_rank[(t0 + t) * R + r] = (uint8_t)((m >> r) & 1u);
            t += dt;
            r += dr;
            if (r >= R) {
                r -= R;
                ++t;
            }
        }
    } else {
        for (int p = lane; p < total; p += 32) {
            int hit = 0;
            for (int j = 0; j < k; ++j) hit |= (erank[t * k + j] == r);
            is_token_in_rank[(t0 + t) * R + r] = (uint8_t)hit;
            if (hit)
                atomicAdd(&rhist[r], 1);
            r += 32;
            while (r >= R) {
                r -= R;
                ++t;
            }
        }
    }
}

// One warp: recv_src[a, b) = -1 (an expert's pad rows), with 16-byte stores
// over the 4-aligned middle when the array is 16-byte aligned (vec).
__device__ __forceinline__ void fill_pad(int32_t* recv_src, int32_t a, int32_t b, bool vec)
{
    const int lane = threadIdx.x & 31;
    if (!vec || b - a < 8) {
        for (int32_t r = a + lane; r < b; r += 32) recv_src[r] = -1;
        return;
    }
    const int32_t a4 = (a + 3) & ~3, b4 = b & ~3;
    if (lane < a4 - a)
        recv_src[a + lane] = -1;
    if (lane < b - b4)
        recv_src[b4 + lane] = -1;
    const int4 m1 = make_int4(-1, -1, -1, -1);
    for (int32_t r = a4 + 4 * lane; r < b4; r += 128) *reinterpret_cast<int4*>(recv_src + r) = m1;
}

// One warp: replay a chunk's entries (ents in smem, -1 unused) in order and
// give each its row.  runc[e] holds the next free row of expert e for this
// chunk and is advanced here.
__device__ __forceinline__ void chunk_assign(const int32_t* ents, int nent, int k, int E,
                                             int64_t t0, int32_t* runc, int32_t* dst_row,
                                             int32_t* recv_src)
{
    const int lane = threadIdx.x & 31;
    const unsigned lt = lanemask_lt();
    const int ebits = 32 - __clz((unsigned)E);  // keys e + 1 in [0, E]
    for (int g = 0; g < nent; g += 32) {
        const int f = g + lane;
        const int e = f < nent ? ents[f] : -1;  // lanes past the chunk end: no expert
        const unsigned peers = match_key(e, ebits);
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

// One warp: load a chunk's entries (all loads of a batch issued first),
// validate them into ents[] and, if erank is given, their ranks; count them
// into hist (shared-memory atomics) if hist is given.  rank = floor(e / epr)
// is (e * rank_magic) >> 32 with rank_magic = ceil(2^32 / epr): exact for
// e, epr <= 2^13 (the error e * (rank_magic - 2^32/epr) / 2^32 < 2^-19 stays
// below the 1/epr gap to the next integer).
__device__ __forceinline__ int load_chunk(const int64_t* __restrict__ src, int nent, int E,
                                          uint64_t rank_magic, int32_t* ents, int32_t* erank,
                                          int32_t* hist)
{
    const int lane = threadIdx.x & 31;
    int bad = 0;
    for (int base = 0; base < nent; base += 32 * kBatch) {
        int64_t v[kBatch];
#pragma unroll
        for (int m = 0; m < kBatch; ++m) {
            const int f = base + m * 32 + lane;
            v[m] = f < nent ? src[f] : -1;
        }
#pragma unroll
        for (int m = 0; m < kBatch; ++m) {
            const int f = base + m * 32 + lane;
            if (f < nent) {
                const int e = to_expert(v[m], E, bad);
                if (ents)
                    ents[f] = e;
                if (erank)
                    erank[f] = e >= 0 ? (int32_t)(((uint64_t)e * rank_magic) >> 32) : -1;
                if (hist && e >= 0)
                    atomicAdd(&hist[e], 1);
            }
        }
    }
    return __any_sync(kFull, bad);
}

// K1.  Shared memory per warp: hist[E], rank_hist[R], entry_rank[32 k].
__global__ void layout_count_kernel(const int64_t* __restrict__ topk_idx, int T, int k, int E,
                                    int R, uint64_t rank_magic, int64_t nchunks,
                                    int32_t* __restrict__ chunk_counts,
                                    int32_t* __restrict__ chunk_rank,
                                    uint8_t* __restrict__ is_token_in_rank, int32_t* err)
{
    extern __shared__ int32_t smem[];
    pdl_wait();
    pdl_trigger();
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
    const int bad = load_chunk(topk_idx + t0 * k, nent, E, rank_magic, nullptr, erank, hist);
    if (bad && lane == 0)
        atomicOr(err, kErrBadIndex);
    __syncwarp();
    chunk_rank_bytes(erank, ntok, k, R, t0, is_token_in_rank, rhist);
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
    pdl_wait();
    pdl_trigger();
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

    // all loads of the range first (in registers when it is short)
    int32_t vals[kBatch];
    int32_t sum = 0;
    const bool short_range = (r1 - r0) <= kBatch;
    if (short_range) {
#pragma unroll
        for (int m = 0; m < kBatch; ++m)
            vals[m] = (colok && r0 + m < r1) ? M[(r0 + m) * ncol + col] : 0;
#pragma unroll
        for (int m = 0; m < kBatch; ++m) sum += vals[m];
    } else if (colok) {
        for (int64_t r = r0; r < r1; ++r) sum += M[r * ncol + col];
    }
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
        if (short_range) {
#pragma unroll
            for (int m = 0; m < kBatch; ++m)
                if (r0 + m < r1) {
                    chunk_counts[(r0 + m) * ncol + col] = run;
                    run += vals[m];
                }
        } else {
            for (int64_t r = r0; r < r1; ++r) {
                const int32_t v = chunk_counts[r * ncol + col];
                chunk_counts[r * ncol + col] = run;
                run += v;
            }
        }
    }
    if (warp == 0 && colok) {
        if (is_expert)
            cnt[col] = total;
        else
            tokens_per_rank[col] = total;
    }
}

// K3.  Shared memory: off[E+1], wsum[32], then per warp run[E] + ents[32 k].
__global__ void layout_assign_kernel(const int64_t* __restrict__ topk_idx, int T, int k, int E,
                                     int R, int epr, uint64_t rank_magic, int block_m,
                                     int64_t nchunks,
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
    pdl_wait();
    pdl_trigger();
    int32_t* off = smem;
    int32_t* wsum = off + E + 1;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = blockDim.x >> 5;
    const int nthr = blockDim.x;
    int32_t* runc = wsum + 32 + (size_t)warp * (E + kChunkTokens * k);
    int32_t* ents = runc + E;

    const int64_t c = (int64_t)blockIdx.x * nwarps + warp;
    const bool has_chunk = c < nchunks;
    const int64_t t0 = c * kChunkTokens;
    const int ntok = has_chunk ? (int)min((int64_t)kChunkTokens, (int64_t)T - t0) : 0;
    const int nent = ntok * k;

    // Loads that do not depend on each other, issued together: this warp's
    // row of chunk prefixes (into runc), its entries (into ents) and, in
    // scan_padded, the expert totals.
    if (has_chunk) {
        for (int base = 0; base < E; base += 32 * kBatch) {
            int32_t v[kBatch];
#pragma unroll
            for (int m = 0; m < kBatch; ++m) {
                const int e = base + m * 32 + lane;
                v[m] = e < E ? chunk_prefix[c * E + e] : 0;
            }
#pragma unroll
            for (int m = 0; m < kBatch; ++m) {
                const int e = base + m * 32 + lane;
                if (e < E)
                    runc[e] = v[m];
            }
        }
        int ignored = load_chunk(topk_idx + t0 * k, nent, E, rank_magic, ents, nullptr, nullptr);
        (void)ignored;  // bad indices were flagged by the count pass
    }
    scan_padded(cnt, E, block_m, off, wsum);

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
    // Pad rows: one warp per expert over the whole grid.
    const bool vec = ((uintptr_t)recv_src & 15u) == 0;
    for (int64_t e = (int64_t)blockIdx.x * nwarps + warp; e < E; e += (int64_t)gridDim.x * nwarps)
        fill_pad(recv_src, off[e] + cnt[e], off[e + 1], vec);

    if (!has_chunk)
        return;  // no block barrier follows
    for (int e = lane; e < E; e += 32) runc[e] += off[e];
    __syncwarp();
    chunk_assign(ents, nent, k, E, t0, runc, dst_row, recv_src);
}

// Small batches (T k <= kSmallEntries, E <= kSmallMaxE): CTAs of 1024
// threads take the entries 1024 at a time (a round, at most kSmallRounds),
// one per thread, kept in registers.  Entry f of round q belongs to virtual
// warp v = f / 32 = 32 q + warp.  Every CTA of the grid computes the whole
// layout in its own shared memory (deterministic, so all agree) and CTA 0
// writes it out; the pad rows of recv_src -- most of the bytes at decode
// sizes -- are spread over the CTAs, since one SM alone stores only some
// tens of GB/s.  Shared-memory atomics are avoided on the common path: many
// warps adding to the same few counters back up the shared-memory pipe.
// Five block barriers:
//   1  tables zeroed (before the dependent-launch wait: shared memory only),
//      topk_idx loaded, is_token_in_rank zeroed;
//   2  per round, equal experts inside the warp (ballots over the key bits);
//      the first lane of a group stores the group size in vtab[e][v]; entry
//      ranks and is_token_in_rank bytes.  When k divides 32 a token's slots
//      share the warp: an entry is the first of its token in its rank when no
//      lower slot of the token has its rank, and the first lane of each rank
//      group of such entries stores their number in ttab[r][v] (R <= 128);
//   3  per expert, tpe threads scan vtab[e][*] over the virtual warps in place
//      (exclusive), the last of them holding cnt[e]; padded and plain counts
//      scanned across the warp; tokens per rank summed from ttab (or, for
//      other shapes, counted with shared atomics);
//   4  each warp scans the 32 warp totals itself and stores off[e] and the
//      unpadded offsets uoff[e] (rows per rank are their differences);
//   5  position = off[e] + vtab[e][v] + rank among the equal lanes.
// Shared memory: vtab uint16 [E][nv] (nv = 32 rounds), ttab uint16 [R][nv]
// when R <= kSmallTabR, then 32-bit words cnt[E], off[E+1], uoff[E+1],
// wsum[2][32], rhist[R], erank[1024 rounds].
constexpr int kSmallThreads = 1024;
constexpr int kSmallRounds = 4;
constexpr int kSmallEntries = kSmallThreads * kSmallRounds;
constexpr int kSmallMaxE = 1024;
constexpr int64_t kSmallMaxRankBytes = 65536;  // T x R bytes of is_token_in_rank
constexpr int kSmallTabR = 128;                // largest R with a tokens-per-rank table

__host__ __device__ inline int small_rounds(int64_t nent)
{
    return nent <= kSmallThreads ? 1 : (int)((nent + kSmallThreads - 1) / kSmallThreads);
}

__host__ __device__ inline size_t small_ttab_halves(int R, int rounds)
{
    return R <= kSmallTabR ? (size_t)R * 32 * rounds : 0;
}

__host__ __device__ inline size_t small_smem_bytes(int E, int R, int rounds)
{
    return 2 * ((size_t)E * 32 * rounds + small_ttab_halves(R, rounds)) +
           sizeof(int32_t) * ((size_t)E + 2 * ((size_t)E + 1) + 64 + R + (size_t)kSmallThreads * rounds);
}

bool small_fits(int64_t T, int k, int E, int R)
{
    const int64_t nent = T * k;
    return nent <= kSmallEntries && E <= kSmallMaxE && T * R <= kSmallMaxRankBytes &&
           small_smem_bytes(E, R, small_rounds(nent)) <= kSmemBudget;
}

// Per-launch constants of the small kernel, computed on the host so that the
// kernel's 1024 threads shift instead of dividing (k and block_m are powers
// of two in practice; other values take the division).
struct SmallPlan {
    int rounds;   // rounds of 1024 entries
    int nv;       // virtual warps, 32 rounds
    int tpe_log;  // log2 of the threads per expert in the count scan
    int ebits;    // bit width of E: match keys e + 1 in [0, E]
    int rbits;    // bit width of R
    int k_log;    // log2 k when k is a power of two, else -1
    int bm_log;   // log2 block_m when a power of two, else -1
};

int log2_if_pow2(int v)
{
    if (v <= 0 || (v & (v - 1)) != 0)
        return -1;
    int l = 0;
    while ((1 << l) < v) ++l;
    return l;
}

int bits_of(unsigned v)
{
    int n = 0;
    while (n < 32 && (v >> n) != 0u) ++n;
    return n;
}

SmallPlan make_small_plan(int T, int k, int E, int R, int block_m)
{
    SmallPlan pl;
    pl.rounds = small_rounds((int64_t)T * k);
    pl.nv = 32 * pl.rounds;
    int tpe = 1;  // a power of two with tpe E <= 1024 and nv / tpe a multiple of 8
    while (2 * tpe * E <= kSmallThreads && (pl.nv / (2 * tpe)) % 8 == 0) tpe *= 2;
    pl.tpe_log = log2_if_pow2(tpe);
    pl.ebits = bits_of((unsigned)E);
    pl.rbits = bits_of((unsigned)R);
    pl.k_log = log2_if_pow2(k);
    pl.bm_log = log2_if_pow2(block_m);
    return pl;
}

// The dispatch half of the fused small-batch kernel (layout + dispatch in
// one launch): what ep_dispatch would be given.
struct FusedDispatch {
    const void* x;
    int H;
    int fp8;             // 0: BF16 copy; 1: FP8 e4m3 1x128
    void* recv_x;
    float* recv_scales;
    int64_t scales_ld;   // FP8: 0 row-major scales, else MN-major leading dimension
    int64_t cap_rows;
};

__device__ __forceinline__ int32_t sum_u16x8(int4 v)
{
    const uint32_t w[4] = {(uint32_t)v.x, (uint32_t)v.y, (uint32_t)v.z, (uint32_t)v.w};
    int32_t s = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) s += (int32_t)(w[i] & 0xffffu) + (int32_t)(w[i] >> 16);
    return s;
}

// Exclusive prefix of 8 packed uint16 counts starting at acc; returns the
// running sum after them.
__device__ __forceinline__ int32_t exscan_u16x8(int4& v, int32_t acc)
{
    uint32_t w[4] = {(uint32_t)v.x, (uint32_t)v.y, (uint32_t)v.z, (uint32_t)v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int32_t lo = (int32_t)(w[i] & 0xffffu), hi = (int32_t)(w[i] >> 16);
        w[i] = (uint32_t)acc | ((uint32_t)(acc + lo) << 16);
        acc += lo + hi;
    }
    v = make_int4((int)w[0], (int)w[1], (int)w[2], (int)w[3]);
    return acc;
}

// kR: rounds the kernel is compiled for (kSmallRounds; the fused launch of a
// one-round batch, every decode batch, takes kR = 1: measured 2 % faster in
// CUDA graphs; the layout-only kernel was slower so, and keeps kSmallRounds).
// kFused = false: the layout alone.  kFused = true: then every warp of the
// grid dispatches (token, unit) pieces with the positions in its own shared
// memory -- no grid-wide wait.
template <bool kFused, int kR = kSmallRounds>
__global__ void __launch_bounds__(kSmallThreads)
layout_small_kernel(const int64_t* __restrict__ topk_idx, int T, int k, int E, int R, int epr,
                    uint64_t rank_magic, int block_m, int32_t* __restrict__ cnt_g,
                    int32_t* __restrict__ expert_off_g, int32_t* __restrict__ rank_off_g,
                    int32_t* __restrict__ tokens_per_rank_g,
                    int32_t* __restrict__ rows_per_rank_g, int32_t* __restrict__ total_rows_g,
                    uint8_t* __restrict__ is_token_in_rank, int32_t* __restrict__ dst_row,
                    int32_t* __restrict__ recv_src, int32_t* err, FusedDispatch fd,
                    SmallPlan pl)
{
    extern __shared__ __align__(16) unsigned char small_smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool leader = blockIdx.x == 0;
    const int nent = T * k;
    const int rounds = pl.rounds, nv = pl.nv;
    const bool tok_in_warp = (32 % k) == 0;
    auto token_of = [&](int f) { return pl.k_log >= 0 ? f >> pl.k_log : f / k; };
    const bool use_ttab = tok_in_warp && R <= kSmallTabR;
    uint16_t* vtab = reinterpret_cast<uint16_t*>(small_smem);  // [E][nv]
    uint16_t* ttab = vtab + (size_t)E * nv;                     // [R][nv] when use_ttab
    int32_t* cnt = reinterpret_cast<int32_t*>(ttab + small_ttab_halves(R, rounds));
    int32_t* off = cnt + E;
    int32_t* uoff = off + E + 1;
    int32_t* wsum = uoff + E + 1;  // [2][32]: padded, plain
    int32_t* rhist = wsum + 64;
    int32_t* erank = rhist + R;    // entry ranks, then (fused) positions

    // 1: shared tables zeroed before the wait (no global memory touched)
    {
        int4* z = reinterpret_cast<int4*>(vtab);
        const int n16 = (int)(((size_t)E * nv + small_ttab_halves(R, rounds)) / 8);
        for (int i = tid; i < n16; i += kSmallThreads) z[i] = make_int4(0, 0, 0, 0);
    }
    for (int r = tid; r < R; r += kSmallThreads) rhist[r] = 0;
    pdl_wait();
    pdl_trigger();
    // fused: this warp's first dispatch piece is loaded now, so that its
    // latency hides behind the layout (x does not depend on it)
    const int64_t G = gridDim.x;
    const int64_t vpr = kFused ? fd.H / 16 : 0;
    const int64_t upr = kFused ? (vpr + 31) / 32 : 1;  // 512-channel pieces, BF16 and FP8
    const int64_t npieces = kFused ? (int64_t)T * upr : 0;
    const bool narrow = npieces < (int64_t(1) << 31);  // 32-bit division suffices
    auto token_of_piece = [&](int64_t u) {
        return narrow ? (int64_t)((uint32_t)u / (uint32_t)upr) : u / upr;
    };
    const int64_t u0 = (int64_t)warp * G + blockIdx.x;
    const units::Vec32* xv = static_cast<const units::Vec32*>(fd.x);
    units::Vec32 cur[1];
    if (kFused && u0 < npieces) {
        const int64_t t = token_of_piece(u0);
        units::fp8_load<1>(xv + t * vpr, vpr, u0 - t * upr, cur);
    }
    int64_t raw[kR];
#pragma unroll
    for (int q = 0; q < kR; ++q) {
        const int f = q * kSmallThreads + tid;
        raw[q] = (q < rounds && f < nent) ? topk_idx[f] : -1;
    }
    if (leader) {
        const int64_t bytes = (int64_t)T * R;
        uint8_t* itr = is_token_in_rank;
        if (((uintptr_t)itr & 15u) == 0) {
            for (int64_t i = (int64_t)tid * 16; i + 16 <= bytes; i += 16 * kSmallThreads)
                *reinterpret_cast<int4*>(itr + i) = make_int4(0, 0, 0, 0);
            for (int64_t i = (bytes & ~int64_t(15)) + tid; i < bytes; i += kSmallThreads) itr[i] = 0;
        } else {
            for (int64_t i = tid; i < bytes; i += kSmallThreads) itr[i] = 0;
        }
    }
    int e_r[kR];
    int bad = 0;
#pragma unroll
    for (int q = 0; q < kR; ++q) e_r[q] = to_expert(raw[q], E, bad);
    if (__syncthreads_or(bad) && tid == 0 && leader)
        atomicOr(err, kErrBadIndex);

    // 2: equal experts (and ranks) inside each warp
    const unsigned lt = lanemask_lt();
    int rin[kR];
#pragma unroll
    for (int q = 0; q < kR; ++q) {
        rin[q] = 0;
        if (q < rounds) {
            const int f = q * kSmallThreads + tid;
            const int v = q * 32 + warp;
            const int e = e_r[q];
            const unsigned peers = match_key(e, pl.ebits);
            rin[q] = __popc(peers & lt);
            const int rk = e >= 0 ? (int)(((uint64_t)e * rank_magic) >> 32) : -1;
            if (e >= 0 && rin[q] == 0)
                vtab[(size_t)e * nv + v] = (uint16_t)__popc(peers);
            if (leader && use_ttab) {
                const unsigned rpeers = match_key(rk, pl.rbits);
                const int j = lane & (k - 1);  // k divides 32: a power of two
                const bool first = rk >= 0 && (rpeers & (((1u << j) - 1u) << (lane - j))) == 0;
                const unsigned grp = rpeers & __ballot_sync(kFull, first);
                if (first && (grp & lt) == 0)
                    ttab[(size_t)rk * nv + v] = (uint16_t)__popc(grp);
            }
            if (f < nent) {
                erank[f] = rk;
                if (leader && rk >= 0)
                    is_token_in_rank[(int64_t)token_of(f) * R + rk] = 1;
            }
        }
    }
    __syncthreads();

    // 3: per expert, tpe consecutive threads over nv / tpe virtual warps each
    const int tpe = 1 << pl.tpe_log;
    const int x = tid >> pl.tpe_log, p = tid & (tpe - 1);
    const int chunk = nv >> pl.tpe_log;  // a multiple of 8 halfwords: whole int4s
    int32_t padded = 0, plain = 0;
    {
        int4* row = reinterpret_cast<int4*>(vtab + (size_t)x * nv + p * chunk);
        int32_t part = 0;
        if (x < E)
            for (int i = 0; i < chunk / 8; ++i) part += sum_u16x8(row[i]);
        int32_t incl = part;
        for (int o = 1; o < tpe; o <<= 1) {
            const int32_t u = __shfl_up_sync(kFull, incl, o, tpe);
            if (p >= o)
                incl += u;
        }
        if (x < E) {
            int32_t acc = incl - part;
            for (int i = 0; i < chunk / 8; ++i) {
                int4 v = row[i];
                acc = exscan_u16x8(v, acc);
                row[i] = v;
            }
            if (p == tpe - 1) {
                cnt[x] = incl;
                plain = incl;
                padded = pl.bm_log >= 0 ? ((incl + block_m - 1) >> pl.bm_log) << pl.bm_log
                                        : pad_up(incl, block_m);
            }
        }
    }
    int32_t pincl = padded, uincl = plain;
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t u = __shfl_up_sync(kFull, pincl, o);
        const int32_t w2 = __shfl_up_sync(kFull, uincl, o);
        if (lane >= o) {
            pincl += u;
            uincl += w2;
        }
    }
    if (lane == 31) {
        wsum[warp] = pincl;
        wsum[32 + warp] = uincl;
    }
    if (leader && use_ttab) {
        for (int r = tid; r < R; r += kSmallThreads) {
            const int4* trow = reinterpret_cast<const int4*>(ttab + (size_t)r * nv);
            int32_t sum = 0;
            for (int i = 0; i < nv / 8; ++i) sum += sum_u16x8(trow[i]);
            rhist[r] = sum;
        }
    } else if (leader) {
#pragma unroll
        for (int q = 0; q < kR; ++q) {
            const int f = q * kSmallThreads + tid;
            if (q < rounds && f < nent && e_r[q] >= 0) {
                const int rk = erank[f];
                const int t = token_of(f), j = f - t * k;
                bool first = true;
                for (int jj = 0; jj < j; ++jj) first &= (erank[t * k + jj] != rk);
                if (first)
                    atomicAdd(&rhist[rk], 1);
            }
        }
    }
    __syncthreads();

    // 4: expert offsets, padded and plain
    {
        const int32_t v = wsum[lane], v2 = wsum[32 + lane];
        int32_t inc = v, inc2 = v2;
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t u = __shfl_up_sync(kFull, inc, o);
            const int32_t u2 = __shfl_up_sync(kFull, inc2, o);
            if (lane >= o) {
                inc += u;
                inc2 += u2;
            }
        }
        const int32_t base = __shfl_sync(kFull, inc - v, warp);
        const int32_t base2 = __shfl_sync(kFull, inc2 - v2, warp);
        if (x < E && p == tpe - 1) {
            off[x] = base + pincl - padded;
            uoff[x] = base2 + uincl - plain;
            if (x == E - 1) {
                off[E] = base + pincl;
                uoff[E] = base2 + uincl;
            }
        }
    }
    __syncthreads();

    // 5: outputs (CTA 0), pad rows (all CTAs), positions
    if (leader) {
        for (int e = tid; e < E; e += kSmallThreads) cnt_g[e] = cnt[e];
        for (int e = tid; e <= E; e += kSmallThreads) expert_off_g[e] = off[e];
        for (int r = tid; r <= R; r += kSmallThreads) rank_off_g[r] = off[r * epr];
        for (int r = tid; r < R; r += kSmallThreads) {
            rows_per_rank_g[r] = uoff[(r + 1) * epr] - uoff[r * epr];
            tokens_per_rank_g[r] = rhist[r];
        }
        if (tid == 0)
            *total_rows_g = off[E];
    }
    {
        const bool vec = ((uintptr_t)recv_src & 15u) == 0;
        const int G = (int)gridDim.x;
        for (int64_t e = blockIdx.x + (int64_t)warp * G; e < E; e += (int64_t)G * (kSmallThreads / 32))
            fill_pad(recv_src, off[e] + cnt[e], off[e + 1], vec);
    }
#pragma unroll
    for (int q = 0; q < kR; ++q) {
        const int f = q * kSmallThreads + tid;
        if (q < rounds && f < nent) {
            const int e = e_r[q];
            const int pos = e >= 0 ? off[e] + vtab[(size_t)e * nv + q * 32 + warp] + rin[q] : -1;
            if (kFused)
                erank[f] = pos;  // the ranks were last read before barrier 3
            if (leader) {
                dst_row[f] = pos;
                if (pos >= 0)
                    recv_src[pos] = token_of(f);
            }
        }
    }
    if (!kFused)
        return;

    // dispatch: (token, 512-channel piece) pairs dealt to the CTAs in turn,
    // so that the row stores spread over every SM; each warp loads its next
    // piece after storing the current one
    __syncthreads();
    const int64_t stride = G * (kSmallThreads / 32);
    for (int64_t u = u0; u < npieces; u += stride) {
        const int64_t t = token_of_piece(u);
        int d = lane < k ? erank[t * k + lane] : -1;
        if (d >= fd.cap_rows) {
            atomicOr(err, kErrDispatchCap);
            d = -1;
        }
        if (fd.fp8)
            units::fp8_store<1>(cur, vpr, u - t * upr, d, k, fd.H,
                                static_cast<uint8_t*>(fd.recv_x), fd.recv_scales, fd.scales_ld);
        else
            units::bf16_store(cur[0], (u - t * upr) * 32 + lane, vpr, d, k,
                              static_cast<units::Vec32*>(fd.recv_x));
        const int64_t un = u + stride;
        if (un < npieces) {
            const int64_t tn = token_of_piece(un);
            units::fp8_load<1>(xv + tn * vpr, vpr, un - tn * upr, cur);
        }
    }
}

// Decode batches (T <= SMs, E <= 512, within the small-batch limits): layout
// and dispatch in one launch with one CTA per token.  A CTA needs the expert
// totals of the whole batch (for the padded offsets) but the positions of its
// own token's k slots only: slot (t, j) of expert e goes to row
// off[e] + #{entries before t k + j with expert e}, counted with one
// warp-wide sum per slot over the batch's entries, instead of the full
// per-warp grouping the other small kernel does in every CTA.  The CTA's
// 32 warps work in two groups that meet at block barrier 1 and at barrier 3:
//   layout warps 0-15 (named barrier 1):
//     1  entries loaded (up to kR per thread) and the token's experts
//        published (after the counters were zeroed, before the
//        dependent-launch wait);
//     2  the histogram of all entries and of those of the tokens before
//        this CTA's token (shared atomics: order-free sums);
//     3  the token's positions (warp w takes slots w, w + 16: the padded
//        counts of the experts below the slot's, the slot's expert's
//        entries before the token, its equal slots before it), released to
//        the dispatch group at once;
//     4  padded and plain exclusive scans over the experts (thread e =
//        expert e); then is_token_in_rank, the pad rows of the experts this
//        CTA owns, (the leader) the totals and offsets, and for R > 32 the
//        tokens on rank c (c + G, ...) counted in CTA c, the entries that
//        are their token's first slot on that rank;
//   dispatch warps 16-31 (named barrier 2): warp 16 + p loads 512-channel
//     piece p of the token's row before the layout starts and quantises it
//     (FP8) while the layout warps work; for R <= 32 one CTA's dispatch
//     group also counts the tokens per rank meanwhile (one rank mask per
//     token, one ballot per rank);
//   5  (barrier 3: the layout warps that wrote positions and the dispatch
//      group) the rows stored to the k positions, while the layout group
//      does step 4.
// When T + 1 CTAs fit on the SMs, an extra CTA without a token of its own
// takes the leader's and the counter's work, so that no token's stores wait
// for them.
// Dynamic shared memory: ent[T k] (the entries, for the first-slot test).
constexpr int kDecLayoutWarps = 16;
constexpr int kDecThreads = 32 * kDecLayoutWarps;  // threads of each group
constexpr int kDecMaxE = kDecThreads;               // one expert per layout thread

__device__ __forceinline__ void named_sync(int id, int nthreads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// The same from code paths that differ between the warps taking part (the
// non-aligned form: they reach it at different instructions).
__device__ __forceinline__ void named_sync_unaligned(int id, int nthreads)
{
    asm volatile("barrier.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}



// Number of threads of the named barrier's group whose predicate is true.
__device__ __forceinline__ int named_count(int id, int nthreads, bool pred)
{
    int n;
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %1, 0;\n\t"
                 "bar.red.popc.u32 %0, %2, %3, p;\n\t}"
                 : "=r"(n)
                 : "r"((unsigned)pred), "r"(id), "r"(nthreads)
                 : "memory");
    return n;
}

template <int kR>
__global__ void __launch_bounds__(kSmallThreads)
decode_layout_dispatch_kernel(const int64_t* __restrict__ topk_idx, int T, int k, int E, int R,
                              int epr, uint64_t rank_magic, int block_m, int bm_log, int k_log,
                              int32_t* __restrict__ cnt_g, int32_t* __restrict__ expert_off_g,
                              int32_t* __restrict__ rank_off_g,
                              int32_t* __restrict__ tokens_per_rank_g,
                              int32_t* __restrict__ rows_per_rank_g,
                              int32_t* __restrict__ total_rows_g,
                              uint8_t* __restrict__ is_token_in_rank,
                              int32_t* __restrict__ dst_row, int32_t* __restrict__ recv_src,
                              int32_t* err, FusedDispatch fd)
{
    extern __shared__ __align__(16) int32_t ent[];  // [T k]
    __shared__ int32_t cnt[kDecMaxE], cnt_before[kDecMaxE];
    __shared__ int32_t off[kDecMaxE + 1], uoff[kDecMaxE + 1];
    __shared__ int32_t wsum[2][kDecLayoutWarps];
    __shared__ int32_t rpart[kDecLayoutWarps][32];  // per-warp tokens per rank (R <= 32)
    __shared__ int32_t tgt_e[EP_MAX_TOPK], tgt_pos[EP_MAX_TOPK];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool layout_group = warp < kDecLayoutWarps;
    const int t = blockIdx.x;
    const bool has_token = t < T;  // else the extra CTA (grid T + 1): no token of its own
    const bool extra = (int)gridDim.x > T;
    // the leader writes the totals and offsets; the counter's dispatch group
    // counts the tokens per rank when R <= 32 (both the extra CTA if there is one)
    const bool leader = extra ? t == T : t == T - 1;
    const bool counter = extra ? t == T : t == max(T - 2, 0);
    const int nent = T * k;
    auto padded = [&](int32_t c) {
        return bm_log >= 0 ? ((c + block_m - 1) >> bm_log) << bm_log : pad_up(c, block_m);
    };
    const int64_t vpr = fd.H / 16;
    const int64_t upr = (vpr + 31) / 32;  // 512-channel pieces of the row
    const int piece = warp - kDecLayoutWarps;
    // barrier 3: the layout warps that write positions, then the dispatch group
    const int pos_warps = min(k, kDecLayoutWarps);
    const int release_threads = 32 * (pos_warps + kDecLayoutWarps);

    // 1
    if (layout_group)
        for (int e = tid; e < E; e += kDecThreads) {
            cnt[e] = 0;
            cnt_before[e] = 0;
        }
    pdl_wait();
    pdl_trigger();
    units::Vec32 cur[1];
    int e_r[kR];
    if (!layout_group) {
        if (piece < upr && has_token)
            units::fp8_load<1>(static_cast<const units::Vec32*>(fd.x) + (int64_t)t * vpr, vpr,
                               piece, cur);
    } else {
        int bad = 0;
#pragma unroll
        for (int q = 0; q < kR; ++q) {
            const int f = q * kDecThreads + tid;
            e_r[q] = f < nent ? to_expert(topk_idx[f], E, bad) : -1;
            if (f < nent) {
                ent[f] = e_r[q];
                if (f >= t * k && f < t * k + k)
                    tgt_e[f - t * k] = e_r[q];
            }
        }
        if (__any_sync(kFull, bad) && lane == 0 && leader)
            atomicOr(err, kErrBadIndex);
    }
    __syncthreads();

    if (layout_group) {
        // 2
        // The entries are read back from shared memory from here on: the
        // registers of the global loads would be reloaded from global memory
        // when the compiler rematerialises them (read-only data), an L2 round
        // trip per use.
        int e_s[kR];
#pragma unroll
        for (int q = 0; q < kR; ++q) {
            const int f = q * kDecThreads + tid;
            e_s[q] = f < nent ? ent[f] : -1;
        }
        // the histogram of all entries and of the entries of the tokens
        // before t (shared atomics: order-free sums)
        const int before = t * k;
#pragma unroll
        for (int q = 0; q < kR; ++q)
            if (e_s[q] >= 0) {
                atomicAdd(&cnt[e_s[q]], 1);
                if (q * kDecThreads + tid < before)
                    atomicAdd(&cnt_before[e_s[q]], 1);
            }
        named_sync(1, kDecThreads);

        // 3: the token's positions, released to the dispatch group at once.
        // Warp w takes slots w, w + 16: slot j of expert e lands at the padded
        // counts of the experts below e (summed here from the histogram; the
        // full scans follow, off the stores' path), plus the entries of e in
        // the tokens before t, plus the slots j' < j of token t with expert e.
        if (warp < pos_warps && has_token) {
            const int my_e = lane < k ? tgt_e[lane] : -1;
            for (int j = warp; j < k; j += kDecLayoutWarps) {
                const int e = tgt_e[j];
                int32_t below = 0;
#pragma unroll 4
                for (int f = lane; f < e; f += 32) below += padded(cnt[f]);
                below = __reduce_add_sync(kFull, below);
                const int dup = __popc(__ballot_sync(kFull, lane < j && my_e == e));
                if (lane == 0) {
                    const int32_t p = e >= 0 ? below + cnt_before[e] + dup : -1;
                    tgt_pos[j] = p;
                    dst_row[(int64_t)t * k + j] = p;
                    if (p >= 0)
                        recv_src[p] = t;
                }
            }
            named_sync_unaligned(3, release_threads);  // the positions are in shared memory
        }

        // 4: padded and plain exclusive scans, thread e owns expert e
        const int32_t c_e = tid < E ? cnt[tid] : 0, p_e = padded(c_e);
        int32_t pin = p_e, uin = c_e;
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t a = __shfl_up_sync(kFull, pin, o), b = __shfl_up_sync(kFull, uin, o);
            if (lane >= o) {
                pin += a;
                uin += b;
            }
        }
        if (lane == 31) {
            wsum[0][warp] = pin;
            wsum[1][warp] = uin;
        }
        named_sync(1, kDecThreads);
        {
            const int32_t v = lane < kDecLayoutWarps ? wsum[0][lane] : 0;
            const int32_t v2 = lane < kDecLayoutWarps ? wsum[1][lane] : 0;
            int32_t inc = v, inc2 = v2;
            for (int o = 1; o < kDecLayoutWarps; o <<= 1) {
                const int32_t a = __shfl_up_sync(kFull, inc, o), b = __shfl_up_sync(kFull, inc2, o);
                if (lane >= o) {
                    inc += a;
                    inc2 += b;
                }
            }
            const int32_t base = __shfl_sync(kFull, inc - v, warp);
            const int32_t base2 = __shfl_sync(kFull, inc2 - v2, warp);
            if (tid < E) {
                off[tid] = base + pin - p_e;
                uoff[tid] = base2 + uin - c_e;
                if (tid == E - 1) {
                    off[E] = base + pin;
                    uoff[E] = base2 + uin;
                }
            }
        }
        named_sync(1, kDecThreads);

        for (int r = tid; r < R && has_token; r += kDecThreads) {
            uint8_t hit = 0;
            for (int j = 0; j < k; ++j)
                hit |= (tgt_e[j] >= 0 && (int)(((uint64_t)tgt_e[j] * rank_magic) >> 32) == r);
            is_token_in_rank[(int64_t)t * R + r] = hit;
        }
        const bool vec = ((uintptr_t)recv_src & 15u) == 0;
        for (int e = blockIdx.x + warp * (int)gridDim.x; e < E; e += (int)gridDim.x * kDecLayoutWarps)
            fill_pad(recv_src, off[e] + cnt[e], off[e + 1], vec);
        if (leader) {
            for (int e = tid; e < E; e += kDecThreads) cnt_g[e] = cnt[e];
            for (int e = tid; e <= E; e += kDecThreads) expert_off_g[e] = off[e];
            for (int r = tid; r <= R; r += kDecThreads) rank_off_g[r] = off[r * epr];
            for (int r = tid; r < R; r += kDecThreads)
                rows_per_rank_g[r] = uoff[(r + 1) * epr] - uoff[r * epr];
            if (tid == 0)
                *total_rows_g = off[E];
        }
        // tokens per rank for R > 32: CTA c counts rank c (c + G, ...), the
        // entries that are their token's first slot on that rank (R <= 32:
        // the dispatch group of one CTA, below)
        if (R > 32) {
            for (int r = blockIdx.x; r < R; r += (int)gridDim.x) {  // uniform over the group
                int32_t n = 0;
#pragma unroll
                for (int q = 0; q < kR; ++q) {
                    const int f = q * kDecThreads + tid;
                    bool first = false;
                    if (f < nent && e_s[q] >= 0 &&
                        (int)(((uint64_t)e_s[q] * rank_magic) >> 32) == r) {
                        const int tok = k_log >= 0 ? f >> k_log : f / k;
                        first = true;
                        for (int g = tok * k; g < f; ++g)
                            first &= ent[g] < 0 ||
                                     (int)(((uint64_t)ent[g] * rank_magic) >> 32) != r;
                    }
                    n += named_count(1, kDecThreads, first);
                }
                if (tid == 0)
                    tokens_per_rank_g[r] = n;
            }
        }
    } else {
        // the dispatch group: the codes of its piece, then the stores
        uint4 q8[1];
        float my_scale = 0.0f;
        if (fd.fp8 && piece < upr)
            units::fp8_quantize<1>(cur, q8, my_scale);
        if (R <= 32 && counter) {
            // tokens per rank while the positions are computed: thread t
            // builds token t's rank mask, each warp counts the masks holding
            // rank r with one ballot per rank
            const int dw = warp - kDecLayoutWarps;
            int32_t mine = 0;  // lane r: this warp's tokens on rank r
            for (int t0 = dw * 32; t0 < T; t0 += kDecThreads) {
                const int tt = t0 + lane;
                uint32_t mask = 0;
                if (tt < T)
                    for (int j = 0; j < k; ++j) {
                        const int e = ent[tt * k + j];
                        if (e >= 0)
                            mask |= 1u << (int)(((uint64_t)e * rank_magic) >> 32);
                    }
                for (int r = 0; r < R; ++r) {
                    const int c = __popc(__ballot_sync(kFull, (mask >> r) & 1u));
                    if (lane == r)
                        mine += c;
                }
            }
            if (lane < R)
                rpart[dw][lane] = mine;
            named_sync(2, kDecThreads);
            const int dt = tid - kDecThreads;
            if (dt < R) {
                int32_t n = 0;
                for (int w = 0; w * 32 < T && w < kDecLayoutWarps; ++w) n += rpart[w][dt];
                tokens_per_rank_g[dt] = n;
            }
        }
        if (!has_token)
            return;
        named_sync_unaligned(3, release_threads);  // 5: the positions are in shared memory

        if (piece < upr) {
            int d = lane < k ? tgt_pos[lane] : -1;
            if (d >= fd.cap_rows) {
                atomicOr(err, kErrDispatchCap);
                d = -1;
            }
            const int64_t v = (int64_t)piece * 32 + lane;
            if (fd.fp8) {
                const int nblk = fd.H / 128;
                const int64_t blk = (int64_t)piece * 4 + lane;
                const bool sc_ok = lane < 4 && blk < nblk;
                uint8_t* rq = static_cast<uint8_t*>(fd.recv_x);
                for (int j0 = 0; j0 < k; j0 += 8) {  // the rows of 8 slots, then their stores
                    int dj[8];
#pragma unroll
                    for (int jj = 0; jj < 8; ++jj) dj[jj] = __shfl_sync(kFull, d, (j0 + jj) & 31);
#pragma unroll
                    for (int jj = 0; jj < 8; ++jj) {
                        if (j0 + jj >= k || dj[jj] < 0)
                            continue;
                        if (v < vpr)
                            reinterpret_cast<uint4*>(rq + (int64_t)dj[jj] * fd.H)[v] = q8[0];
                        if (sc_ok)
                            fd.recv_scales[units::scale_index(dj[jj], blk, nblk, fd.scales_ld)] =
                                my_scale;
                    }
                }
            } else {
                units::bf16_store(cur[0], v, vpr, d, k, static_cast<units::Vec32*>(fd.recv_x));
            }
        }
    }
}

// ------------------------------------------------------------------ fused
// Grid barrier over the CTAs of a cooperative launch (all co-resident).
// bar[0] is an arrival counter that only grows (32-bit wrap-around, compared
// by signed difference); bar[1] is its value when the current launch began.
// Each CTA reads the base at its start; the barrier waits until the counter
// reaches base + G; the last arrival stores the next launch's base (every
// CTA read the old one before arriving).  Waiters watch the counter itself:
// the last arrival's add is the release, one L2 round trip earlier than a
// separate release flag.  Graph replays need no host state, and G may
// differ between launches.  The same last arrival advances an epoch word
// that every CTA read at its start.  The poll is bounded: past kSpinLimit
// polls the CTA sets kErrTimeout and the caller abandons the launch
// (ep_handle_check then resets the words).
constexpr uint32_t kSpinLimit = 1u << 22;  // polls of one L2 read each

__device__ __forceinline__ int32_t ld_acquire(const int32_t* p)
{
    int32_t v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ int32_t atom_add_acq_rel(int32_t* p, int32_t v)
{
    int32_t old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;"
                 : "=r"(old)
                 : "l"(p), "r"(v)
                 : "memory");
    return old;
}

__device__ __forceinline__ int32_t signed_gap(int32_t a, int32_t b)
{
    return (int32_t)((uint32_t)a - (uint32_t)b);
}

// The barrier comes in two halves, so that a CTA can work between its
// arrival and its wait.  barrier_arrive: one thread, after a block barrier,
// so that its release covers the CTA's writes; the last arrival stores the
// next launch's base and advances the epoch word.  barrier_wait: every
// thread; the same thread polls (bounded), the others wait at a block
// barrier.
__device__ __forceinline__ void barrier_arrive(int32_t* bar, int32_t target, int32_t* epoch_word,
                                               int32_t next_epoch)
{
    const int32_t old = atom_add_acq_rel(bar, 1);
    if (signed_gap(old, target) == -1) {
        asm volatile("st.relaxed.gpu.global.b32 [%0], %1;" ::"l"(bar + 1), "r"(target) : "memory");
        asm volatile("st.relaxed.gpu.global.b32 [%0], %1;" ::"l"(epoch_word), "r"(next_epoch)
                     : "memory");
    }
}

__device__ bool barrier_wait(int32_t* bar, int32_t target, int32_t* err, bool poller)
{
    __shared__ int ok;
    if (poller) {
        int good = 1;
        uint32_t polls = 0;
        while (signed_gap(ld_acquire(bar), target) < 0) {
            if (++polls > kSpinLimit) {
                good = 0;
                break;
            }
        }
        if (!good)
            atomicOr(err, kErrTimeout);
        ok = good;
    }
    __syncthreads();
    return ok != 0;
}

// Large batches in one cooperative launch with a single grid barrier.  One
// tile per CTA: kTileWarps warps of wt consecutive tokens each, wt chosen on
// the host so that the tiles cover the SMs once.  Tiles form groups of gs
// consecutive tiles.  Counts travel as uint16 pairs packed in 32-bit words
// (a row of ldw = ceil(E / 8) * 4 words), which the host bounds: a group
// holds fewer than 2^16 entries.
//   phase 1  each warp loads its tokens' entries into shared memory and
//            counts them into its own histogram row (shared atomics); the
//            tile's expert counts go to its row of tile_rows and are added
//            (red.add of the packed pairs: no carry crosses a half) to its
//            group's row, its tokens-per-rank counts to per-rank sums;
//            is_token_in_rank bytes;
//   barrier  the only grid-wide wait;
//   phase 2  every CTA reads all group rows (their sum is the expert totals;
//            the rows of the groups before its own are most of its prefix)
//            and the rows of the tiles before it in its group, with 16-byte
//            loads all requested before any is used: about 2 sqrt(tiles) rows
//            instead of one per tile.  One pass over the experts then sums the
//            partial rows and scans the padded totals into expert_off (in
//            every CTA, so no second grid-wide wait is needed); CTA 0 writes
//            the totals, the offsets and the tokens per rank;
//   phase 3  position = the tile's first row of the expert + the entry's
//            place inside the tile's block of it, which each warp computed
//            while it waited at the barrier (its warp prefix plus its rank
//            among the equal experts before it, entries replayed in order);
//            the pad rows of recv_src are set to -1.
// The sums are double-buffered by launch: the epoch word's parity picks the
// buffer a launch adds into, and the launch clears the other one for the
// next launch (which starts after this one has finished); the last arrival
// at the barrier advances the epoch, after every CTA has read it.
// Shared memory (words, 16-byte aligned part first): part[nrg][nc][16]
// (phase-2 partial sums, nc = ldw / 4), ents[W][wt k], erank[W][wt k] (entry
// ranks, then their places in the tile), run[W][E] (warp histograms, then
// warp prefixes), off[E+1], pre[E], tot[E], wsum[32], rhist[R], rtot[R].
constexpr int kTileWarps = 8;                    // warps that own tokens
constexpr int kTileThreads = 32 * kTileWarps;
constexpr int kTileBlock = kTileThreads + 32;    // + one warp that holds the grid barrier
constexpr int kRowBatch = 4;   // rows per thread requested together in phase 2
constexpr int kMaxGroups = kTileMaxGroups;

__host__ __device__ inline int tile_ldw(int E) { return ((E + 7) / 8) * 4; }

__host__ __device__ inline size_t tile_smem_words(int wt, int k, int E, int R)
{
    const int nc = tile_ldw(E) / 4, nrg = kTileThreads / nc;
    return (size_t)nrg * nc * 16 + 2 * (size_t)kTileWarps * wt * k + (size_t)kTileWarps * E +
           (size_t)(E + 1) + 2 * (size_t)E + 32 + 2 * (size_t)R;
}

__device__ __forceinline__ void red_add(int32_t* p, int32_t v)
{
    asm volatile("red.relaxed.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__global__ void __launch_bounds__(kTileBlock, 1)
layout_tile_kernel(const int64_t* __restrict__ topk_idx, int T, int k, int E, int R, int epr,
                   uint64_t rank_magic, int block_m, int bm_log, int k_log, int wt, int ntiles, int gs,
                   int ngroups, uint32_t* __restrict__ tile_rows, int32_t* __restrict__ acc,
                   int32_t* __restrict__ cnt_g, int32_t* __restrict__ expert_off_g,
                   int32_t* __restrict__ rank_off_g, int32_t* __restrict__ tokens_per_rank_g,
                   int32_t* __restrict__ rows_per_rank_g, int32_t* __restrict__ total_rows_g,
                   uint8_t* __restrict__ is_token_in_rank, int32_t* __restrict__ dst_row,
                   int32_t* __restrict__ recv_src, int32_t* err)
{
    extern __shared__ __align__(16) int32_t smem[];
    pdl_wait();
    pdl_trigger();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool worker = warp < kTileWarps;  // else the barrier warp
    const int went = wt * k;
    const int ldw = tile_ldw(E), nc = ldw >> 2, nrg = kTileThreads / nc;
    const int tile = blockIdx.x, grp = tile / gs;
    int32_t* bar = err + 1;
    int32_t* epoch_word = acc;
    // acc: epoch word (padded to 16 bytes), then per buffer kMaxGroups group
    // rows of ldw words and R tokens-per-rank sums
    const size_t buf_words = (size_t)kMaxGroups * ldw + (size_t)((R + 3) & ~3);
    int32_t* bufs = acc + 4;
    auto padded = [&](int32_t c) {
        return bm_log >= 0 ? ((c + block_m - 1) >> bm_log) << bm_log : pad_up(c, block_m);
    };

    int32_t* part = smem;
    int32_t* ents_all = part + nrg * nc * 16;
    int32_t* erank_all = ents_all + kTileWarps * went;
    int32_t* run_all = erank_all + kTileWarps * went;
    int32_t* off = run_all + kTileWarps * E;
    int32_t* pre = off + E + 1;
    int32_t* tot = pre + E;
    int32_t* wsum = tot + E;
    int32_t* rhist = wsum + 32;
    int32_t* rtot = rhist + R;
    int32_t* ents = ents_all + warp * went;
    int32_t* run = run_all + warp * E;

    // A barrier that timed out earlier leaves its words inconsistent until
    // ep_handle_check resets them: refuse to take part (every CTA reads the
    // same word).  Every CTA reads the barrier base and the epoch before it
    // arrives, so before the last arrival stores the next ones.  The words
    // are requested here and used after the loads of phase 1.
    __shared__ int stale;
    __shared__ int32_t bar_base, epoch;
    int32_t err_word = 0, base_word = 0, epoch_w = 0;
    if (tid == 0) {
        err_word = *(volatile int32_t*)err;
        base_word = *(volatile int32_t*)(bar + 1);
        epoch_w = *(volatile int32_t*)epoch_word;
    }

    // ---- phase 1
    if (worker) {
        for (int e = lane; e < E; e += 32) run[e] = 0;
        for (int r = tid; r < R; r += kTileThreads) rhist[r] = 0;
    }
    __syncthreads();
    const int64_t t0 = ((int64_t)tile * kTileWarps + warp) * wt;
    const int ntok = worker ? (int)max((int64_t)0, min((int64_t)wt, (int64_t)T - t0)) : 0;
    if (ntok > 0) {
        int32_t* erank = erank_all + warp * went;
        const int bad = load_chunk(topk_idx + t0 * k, ntok * k, E, rank_magic, ents, erank, run);
        if (bad && lane == 0)
            atomicOr(err, kErrBadIndex);
        __syncwarp();
        for (int tb = 0; tb < ntok; tb += 32)
            chunk_rank_bytes(erank + tb * k, min(32, ntok - tb), k, R, t0 + tb, is_token_in_rank,
                             rhist);
    }
    if (tid == 0) {
        stale = (err_word & kErrTimeout) != 0;
        bar_base = base_word;
        epoch = epoch_w;
    }
    __syncthreads();
    int32_t* cur = bufs + (size_t)(epoch & 1) * buf_words;  // this launch's sums
    int32_t* nxt = bufs + (size_t)((epoch & 1) ^ 1) * buf_words;
    if (worker) {
        uint32_t* grow = reinterpret_cast<uint32_t*>(cur) + (size_t)grp * ldw;
        for (int i = tid; i < ldw; i += kTileThreads) {
            uint32_t c[2] = {0u, 0u};
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int e = 2 * i + h;
                if (e < E)
                    for (int w = 0; w < kTileWarps; ++w) {  // exclusive prefix over the warps
                        const int32_t n = run_all[w * E + e];
                        run_all[w * E + e] = (int32_t)c[h];
                        c[h] += (uint32_t)n;
                    }
            }
            const uint32_t pk = c[0] | (c[1] << 16);
            tile_rows[(size_t)tile * ldw + i] = pk;
            if (pk)
                red_add(reinterpret_cast<int32_t*>(grow + i), (int32_t)pk);
        }
        int32_t* rsum = cur + (size_t)kMaxGroups * ldw;
        for (int r = tid; r < R; r += kTileThreads)
            if (rhist[r])
                red_add(rsum + r, rhist[r]);
    }
    if (stale)
        return;
    __syncthreads();
    if (tid == kTileThreads)  // the barrier warp: its wait for the atomic stalls no token work
        barrier_arrive(bar, bar_base + (int32_t)gridDim.x, epoch_word, epoch + 1);
    // While the other tiles arrive: each warp replays its entries in order and
    // gives each its position inside the tile's block of its expert (the warp
    // prefix plus its rank among the equal experts before it), into lpos.
    int32_t* lpos = erank_all + warp * went;
    if (ntok > 0) {
        const int nent = ntok * k;
        const int ebits = 32 - __clz((unsigned)E);  // keys e + 1 in [0, E]
        const unsigned lt = lanemask_lt();
        for (int g = 0; g < nent; g += 32) {
            const int f = g + lane;
            const int e = f < nent ? ents[f] : -1;
            const unsigned peers = match_key(e, ebits);
            int32_t pos = -1;
            if (e >= 0)
                pos = run[e] + __popc(peers & lt);
            __syncwarp();
            if (e >= 0 && (peers & lt) == 0)
                run[e] += __popc(peers);
            __syncwarp();
            if (f < nent)
                lpos[f] = pos;
        }
    }
    if (!barrier_wait(bar, bar_base + (int32_t)gridDim.x, err, tid == kTileThreads))
        return;

    // ---- phase 2: totals and this tile's prefix
    {
        const int c = tid % nc, g = tid / nc;
        const int gfirst = grp * gs;
        const int nr = ngroups + (tile - gfirst);  // group rows, then tiles before this one
        int32_t apre[8], atot[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) apre[i] = atot[i] = 0;
        if (g < nrg) {
            const uint32_t* grows = reinterpret_cast<const uint32_t*>(cur);
            for (int j0 = g; j0 < nr; j0 += nrg * kRowBatch) {
                int4 v[kRowBatch];
#pragma unroll
                for (int m = 0; m < kRowBatch; ++m) {
                    const int j = j0 + m * nrg;
                    const uint32_t* row = j < ngroups ? grows + (size_t)j * ldw
                                                      : tile_rows + (size_t)(gfirst + j - ngroups) * ldw;
                    v[m] = j < nr ? __ldcg(reinterpret_cast<const int4*>(row) + c)
                                  : make_int4(0, 0, 0, 0);
                }
#pragma unroll
                for (int m = 0; m < kRowBatch; ++m) {
                    const int j = j0 + m * nrg;
                    const int32_t in_tot = j < ngroups ? -1 : 0;
                    const int32_t in_pre = (j < grp || j >= ngroups) ? -1 : 0;
                    const uint32_t wv[4] = {(uint32_t)v[m].x, (uint32_t)v[m].y, (uint32_t)v[m].z,
                                            (uint32_t)v[m].w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int32_t lo = (int32_t)(wv[i] & 0xffffu), hi = (int32_t)(wv[i] >> 16);
                        atot[2 * i] += lo & in_tot;
                        atot[2 * i + 1] += hi & in_tot;
                        apre[2 * i] += lo & in_pre;
                        apre[2 * i + 1] += hi & in_pre;
                    }
                }
            }
            int4* pp = reinterpret_cast<int4*>(part + (g * nc + c) * 16);
            pp[0] = make_int4(apre[0], apre[1], apre[2], apre[3]);
            pp[1] = make_int4(apre[4], apre[5], apre[6], apre[7]);
            pp[2] = make_int4(atot[0], atot[1], atot[2], atot[3]);
            pp[3] = make_int4(atot[4], atot[5], atot[6], atot[7]);
        }
        if (blockIdx.x == 0 && worker) {
            const int32_t* rsum = cur + (size_t)kMaxGroups * ldw;
            for (int r = tid; r < R; r += kTileThreads) rtot[r] = __ldcg(rsum + r);
        }
        // clear the other buffer for the next launch (no one reads it now)
        if (worker)
            for (int64_t i = (int64_t)blockIdx.x * kTileThreads + tid; i < (int64_t)buf_words;
                 i += (int64_t)gridDim.x * kTileThreads)
                nxt[i] = 0;
    }
    __syncthreads();
    // One pass over the experts, thread tid owning [e0, e1) (empty for the
    // barrier warp): the partial rows summed, the padded totals scanned across
    // the block (each warp scans the warp sums itself), and the tile's first
    // row per expert.
    {
        const int seg = (E + kTileThreads - 1) / kTileThreads;
        const int e0 = min(E, tid * seg), e1 = min(E, e0 + seg);
        int32_t local = 0;
        for (int e = e0; e < e1; ++e) {
            const int cc = e >> 3, j = e & 7;
            int32_t p = 0, s = 0;
            for (int g = 0; g < nrg; ++g) {
                const int32_t* q = part + (g * nc + cc) * 16;
                p += q[j];
                s += q[8 + j];
            }
            pre[e] = p;
            tot[e] = s;
            local += padded(s);
        }
        int32_t incl = local;
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t u = __shfl_up_sync(kFull, incl, o);
            if (lane >= o)
                incl += u;
        }
        if (lane == 31)
            wsum[warp] = incl;
        __syncthreads();
        const int32_t wv = lane < kTileWarps ? wsum[lane] : 0;
        int32_t winc = wv;
        for (int o = 1; o < kTileWarps; o <<= 1) {
            const int32_t u = __shfl_up_sync(kFull, winc, o);
            if (lane >= o)
                winc += u;
        }
        int32_t at = __shfl_sync(kFull, winc - wv, warp) + incl - local;
        for (int e = e0; e < e1; ++e) {
            off[e] = at;
            pre[e] += at;  // the tile's first row of expert e
            at += padded(tot[e]);
        }
        if (tid == kTileThreads - 1)
            off[E] = at;
    }
    __syncthreads();
    if (blockIdx.x == 0 && worker) {
        for (int e = tid; e < E; e += kTileThreads) cnt_g[e] = tot[e];
        for (int e = tid; e <= E; e += kTileThreads) expert_off_g[e] = off[e];
        for (int r = tid; r <= R; r += kTileThreads) rank_off_g[r] = off[r * epr];
        for (int r = tid; r < R; r += kTileThreads) {
            int32_t s = 0;
            for (int e = r * epr; e < (r + 1) * epr; ++e) s += tot[e];
            rows_per_rank_g[r] = s;
            tokens_per_rank_g[r] = rtot[r];
        }
        if (tid == 0)
            *total_rows_g = off[E];
    }

    // ---- phase 3
    if (ntok > 0) {
        const int nent = ntok * k;
        for (int f = lane; f < nent; f += 32) {
            const int e = ents[f];
            const int32_t pos = e >= 0 ? pre[e] + lpos[f] : -1;
            dst_row[t0 * k + f] = pos;
            if (pos >= 0)
                recv_src[pos] = (int32_t)(t0 + (k_log >= 0 ? f >> k_log : f / k));
        }
    }
    const bool vec = ((uintptr_t)recv_src & 15u) == 0;
    if (worker)
        for (int64_t e = (int64_t)blockIdx.x * kTileWarps + warp; e < E;
             e += (int64_t)gridDim.x * kTileWarps)
            fill_pad(recv_src, off[e] + tot[e], off[e + 1], vec);
}

uint64_t rank_magic_for(int epr) { return ((uint64_t(1) << 32) + (uint64_t)epr - 1) / (uint64_t)epr; }

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

// 0: not yet tried; 1: cooperative launches also take programmatic dependent
// launch; -1: they refused it (cooperative alone).
std::atomic<int> g_coop_pdl{0};

}  // namespace

size_t tile_acc_words(int E, int R)
{
    return 4 + 2 * ((size_t)kMaxGroups * tile_ldw(E) + (size_t)((R + 3) & ~3));
}

// The single-launch layout: tiles of kTileWarps x wt tokens, one per CTA,
// at most one CTA per SM, cooperative so that all CTAs are resident.
// Returns cudaErrorCooperativeLaunchTooLarge when the shape does not suit it
// (the caller then runs the three kernels).
cudaError_t launch_fused(const Handle& h, const int64_t* topk_idx, int T, cudaStream_t s)
{
    const int k = h.k, E = h.E, R = h.R, epr = h.E / h.R;
    const int ldw = tile_ldw(E);
    if (ldw / 4 > kTileThreads || !h.tile_acc)
        return cudaErrorCooperativeLaunchTooLarge;
    cudaError_t rc;
    int dev = 0, sms = 0;
    if ((rc = cudaGetDevice(&dev)) != cudaSuccess ||
        (rc = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return rc;
    // tokens per warp: the tiles cover the SMs once, and a tile holds at least
    // kChunkTokens tokens (so the tile rows fit in the chunk count matrix)
    int64_t wt = ((int64_t)T + (int64_t)kTileWarps * sms - 1) / ((int64_t)kTileWarps * sms);
    wt = std::max<int64_t>(wt, kChunkTokens / kTileWarps);
    const int64_t ntiles = ((int64_t)T + kTileWarps * wt - 1) / (kTileWarps * wt);
    if (ntiles > (int64_t)kMaxGroups * kMaxGroups || ntiles * ldw > h.max_chunks * (int64_t)E)
        return cudaErrorCooperativeLaunchTooLarge;
    int gs = 1;  // group size: about sqrt(tiles), so that groups and tiles per group balance
    while ((int64_t)gs * gs < ntiles) ++gs;
    const int ngroups = (int)((ntiles + gs - 1) / gs);
    if ((int64_t)gs * kTileWarps * wt * k > 65535)  // a group's count of one expert in 16 bits
        return cudaErrorCooperativeLaunchTooLarge;
    const size_t smem = sizeof(int32_t) * tile_smem_words((int)wt, k, E, R);
    if (smem > kSmemBudget)
        return cudaErrorCooperativeLaunchTooLarge;
    if ((rc = set_smem((const void*)layout_tile_kernel, smem)) != cudaSuccess)
        return rc;
    int per_sm = 0;
    if ((rc = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, layout_tile_kernel,
                                                            kTileBlock, smem)) != cudaSuccess)
        return rc;
    if (per_sm < 1 || ntiles > (int64_t)sms * per_sm)
        return cudaErrorCooperativeLaunchTooLarge;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)ntiles);
    cfg.blockDim = dim3(kTileBlock);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    auto launch = [&](int nattrs) {
        cfg.numAttrs = nattrs;
        return cudaLaunchKernelEx(&cfg, layout_tile_kernel, topk_idx, T, k, E, R, epr,
                                  rank_magic_for(epr), h.block_m, log2_if_pow2(h.block_m),
                                  log2_if_pow2(k), (int)wt, (int)ntiles, gs, ngroups,
                                  reinterpret_cast<uint32_t*>(h.chunk_counts), h.tile_acc, h.cnt,
                                  h.expert_off, h.rank_off, h.tokens_per_rank, h.rows_per_rank,
                                  h.total_rows, h.is_token_in_rank, h.dst_row, h.recv_src, h.err);
    };
    if (g_coop_pdl.load() >= 0) {
        rc = launch(2);
        if (rc == cudaSuccess) {
            g_coop_pdl = 1;
            return rc;
        }
        if (g_coop_pdl.load() == 1 || (rc != cudaErrorInvalidValue && rc != cudaErrorNotSupported))
            return rc;
        (void)cudaGetLastError();  // refused: cooperative launches without PDL from now on
        g_coop_pdl = -1;
    }
    return launch(1);
}

cudaError_t launch_layout(const Handle& h, const int64_t* topk_idx, int T, cudaStream_t s,
                          bool allow_fused)
{
    const int k = h.k, E = h.E, R = h.R, epr = h.E / h.R;
    const int64_t nchunks = ((int64_t)T + kChunkTokens - 1) / kChunkTokens;
    cudaError_t rc;

    // one entry per thread when the batch is small; one warp per expert's pad
    // rows, so ceil(E / 32) CTAs, each computing the same layout
    if (small_fits(T, k, E, R)) {
        const size_t smem = small_smem_bytes(E, R, small_rounds((int64_t)T * k));
        if ((rc = set_smem((const void*)layout_small_kernel<false>, smem)) != cudaSuccess)
            return rc;
        int dev = 0, sms = 0;
        if ((rc = cudaGetDevice(&dev)) != cudaSuccess ||
            (rc = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return rc;
        const unsigned grid = (unsigned)std::max(1, std::min(sms, (E + 31) / 32));
        return launch_pdl(layout_small_kernel<false>, grid, kSmallThreads, smem, s, topk_idx, T,
                          k, E, R, epr, rank_magic_for(epr), h.block_m, h.cnt, h.expert_off,
                          h.rank_off, h.tokens_per_rank, h.rows_per_rank, h.total_rows,
                          h.is_token_in_rank, h.dst_row, h.recv_src, h.err, FusedDispatch{},
                          make_small_plan(T, k, E, R, h.block_m));
    }

    if (allow_fused && nchunks > 0) {
        rc = launch_fused(h, topk_idx, T, s);
        if (rc != cudaErrorCooperativeLaunchTooLarge && rc != cudaErrorNotSupported)
            return rc;
        (void)cudaGetLastError();  // clear the refused launch; use three kernels
    }

    if (nchunks > 0) {
        const size_t per_warp = sizeof(int32_t) * (size_t)(E + R + kChunkTokens * k);
        const int w1 = warps_for(per_warp, 0);
        const size_t smem1 = per_warp * w1;
        if ((rc = set_smem((const void*)layout_count_kernel, smem1)) != cudaSuccess)
            return rc;
        const unsigned g1 = (unsigned)((nchunks + w1 - 1) / w1);
        if ((rc = launch_pdl(layout_count_kernel, g1, 32 * w1, smem1, s, topk_idx, T, k, E, R,
                             rank_magic_for(epr), nchunks, h.chunk_counts, h.chunk_rank, h.is_token_in_rank,
                             h.err)) != cudaSuccess)
            return rc;
    }

    const unsigned g2 = (unsigned)((E + 31) / 32 + (R + 31) / 32);
    if ((rc = launch_pdl(layout_scan_kernel, g2, kScanThreads, 0, s, h.chunk_counts,
                         h.chunk_rank, E, R, nchunks, h.cnt, h.tokens_per_rank)) != cudaSuccess)
        return rc;

    const size_t fixed3 = sizeof(int32_t) * (size_t)(E + 1 + 32);
    const size_t per_warp3 = sizeof(int32_t) * (size_t)(E + kChunkTokens * k);
    const int w3 = warps_for(per_warp3, fixed3);
    const size_t smem3 = fixed3 + per_warp3 * w3;
    if ((rc = set_smem((const void*)layout_assign_kernel, smem3)) != cudaSuccess)
        return rc;
    const unsigned g3 = (unsigned)std::max<int64_t>(1, (nchunks + w3 - 1) / w3);
    return launch_pdl(layout_assign_kernel, g3, 32 * w3, smem3, s, topk_idx, T, k, E, R, epr,
                      rank_magic_for(epr), h.block_m, nchunks, h.chunk_counts, h.cnt, h.expert_off, h.rank_off,
                      h.rows_per_rank, h.total_rows, h.dst_row, h.recv_src);
}

bool fused_layout_dispatch_fits(const Handle& h, int T)
{
    return small_fits(T, h.k, h.E, h.R);
}

cudaError_t launch_layout_dispatch(const Handle& h, const int64_t* topk_idx, int T, const void* x,
                                   int H, bool fp8, void* recv_x, float* recv_scales,
                                   int64_t scales_ld, int64_t cap_rows, cudaStream_t s)
{
    const int k = h.k, E = h.E, R = h.R, epr = h.E / h.R;
    {
        // one CTA per token when the batch fits on the SMs once
        int dev = 0, sms = 0;
        cudaError_t rc;
        if ((rc = cudaGetDevice(&dev)) != cudaSuccess ||
            (rc = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return rc;
        const int rounds = (int)(((int64_t)T * k + kDecThreads - 1) / kDecThreads);
        const size_t dsmem = sizeof(int32_t) * (size_t)T * k;
        if (T <= sms && E <= kDecMaxE && dsmem <= 64 * 1024 &&
            (H / 16 + 31) / 32 <= kSmallThreads / 32 - kDecLayoutWarps) {
            FusedDispatch fd{x, H, fp8 ? 1 : 0, recv_x, recv_scales, scales_ld, cap_rows};
            auto go = [&](auto kern) {
                cudaError_t r2 = set_smem((const void*)kern, dsmem);
                if (r2 != cudaSuccess)
                    return r2;
                const unsigned grid = (unsigned)(T + 1 <= sms ? T + 1 : T);  // + the extra CTA
                return launch_pdl(kern, grid, kSmallThreads, dsmem, s, topk_idx, T, k, E,
                                  R, epr, rank_magic_for(epr), h.block_m,
                                  log2_if_pow2(h.block_m), log2_if_pow2(k), h.cnt, h.expert_off,
                                  h.rank_off, h.tokens_per_rank, h.rows_per_rank, h.total_rows,
                                  h.is_token_in_rank, h.dst_row, h.recv_src, h.err, fd);
            };
            switch (rounds) {
            case 0:
            case 1: return go(decode_layout_dispatch_kernel<1>);
            case 2: return go(decode_layout_dispatch_kernel<2>);
            case 3: return go(decode_layout_dispatch_kernel<3>);
            case 4: return go(decode_layout_dispatch_kernel<4>);
            case 5: return go(decode_layout_dispatch_kernel<5>);
            case 6: return go(decode_layout_dispatch_kernel<6>);
            case 7: return go(decode_layout_dispatch_kernel<7>);
            default: return go(decode_layout_dispatch_kernel<8>);
            }
        }
    }
    const size_t smem = small_smem_bytes(E, R, small_rounds((int64_t)T * k));
    cudaError_t rc;
    const bool one_round = small_rounds((int64_t)T * k) == 1;
    auto kern = one_round ? layout_small_kernel<true, 1> : layout_small_kernel<true>;
    if ((rc = set_smem((const void*)kern, smem)) != cudaSuccess)
        return rc;
    int dev = 0, sms = 0;
    if ((rc = cudaGetDevice(&dev)) != cudaSuccess ||
        (rc = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return rc;
    // one CTA per SM: the layout is replicated (cheap at these sizes) so that
    // the dispatch -- FP8 division and row stores -- spreads over the GPU
    const unsigned grid = (unsigned)std::max(1, sms);
    FusedDispatch fd{x, H, fp8 ? 1 : 0, recv_x, recv_scales, scales_ld, cap_rows};
    return launch_pdl(kern, grid, kSmallThreads, smem, s, topk_idx, T, k, E,
                      R, epr, rank_magic_for(epr), h.block_m, h.cnt, h.expert_off, h.rank_off,
                      h.tokens_per_rank, h.rows_per_rank, h.total_rows, h.is_token_in_rank,
                      h.dst_row, h.recv_src, h.err, fd, make_small_plan(T, k, E, R, h.block_m));
}

}  // namespace ep
