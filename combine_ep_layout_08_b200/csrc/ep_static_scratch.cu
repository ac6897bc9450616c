// ep_static_scratch.cu -- ep_layout_static_scratch: the dispatch layout for
// callers that cannot allocate device memory.  The pages ask for a stated
// policy when a buffer cannot be allocated ("DeepEP是什麼？…", section
// ElasticBuffer); this entry point takes allocation out of the call.
//
// Some callers have no way to hand the library a workspace: processes whose
// device memory is owned up front by a framework allocator or a pre-reserved
// pool that forbids further cudaMalloc calls, and embedded or plug-in
// contexts that only receive input and output pointers.
// This entry point needs nothing from them beyond those pointers: the layout's
// only scratch (the per-chunk expert and rank count matrices) lives in a
// fixed-size array of this library's own device memory, declared below, which
// every GPU that loads the library holds until the process exits.
//
// The same three layout kernels as ep_layout run; only the home of their
// scratch differs.  Host code cannot pass the array's name to a kernel (on the
// host it is a stand-in symbol, not a device address), so the device address
// is looked up once per device with cudaGetSymbolAddress and cached.
#include <cuda_runtime.h>

#include <mutex>

#include "ep_internal.cuh"

// The scratch array itself (file scope, one per device that loads the library).
static __device__ __align__(256) int32_t g_layout_scratch[EP_STATIC_SCRATCH_BYTES / sizeof(int32_t)];

namespace ep {
namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int32_t* g_scratch_addr[kMaxDevices] = {};

// Device address of g_layout_scratch on the current device (set-up on the
// first call per device).  Returns EP_OK or the status to report, with its
// message recorded for ep_last_error_message.
ep_status_t scratch_address(int32_t** out)
{
    int dev = 0;
    cudaError_t rc = cudaGetDevice(&dev);
    if (rc != cudaSuccess)
        return cuda_fail(rc, "ep_layout_static_scratch: cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices)
        return fail_message(EP_ERR_INVALID_ARG,
                            "ep_layout_static_scratch: device ordinals above 63 are not served");
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        rc = cudaGetSymbolAddress(&p, g_layout_scratch);
        if (rc != cudaSuccess)
            return cuda_fail(rc, "ep_layout_static_scratch: cudaGetSymbolAddress");
        g_scratch_addr[dev] = static_cast<int32_t*>(p);
    }
    *out = g_scratch_addr[dev];
    return EP_OK;
}

}  // namespace
}  // namespace ep

extern "C" ep_status_t ep_layout_static_scratch(
    const int64_t* topk_idx, int T, int num_topk, int num_experts, int num_ranks, int block_m,
    int32_t* num_tokens_per_expert, int32_t* num_tokens_per_rank, int32_t* num_rows_per_rank,
    int32_t* expert_off, int32_t* rank_off, int32_t* total_recv_rows,
    uint8_t* is_token_in_rank, int32_t* dst_row, int32_t* recv_src,
    int64_t recv_src_capacity, int32_t* error_word, void* stream)
{
    ep::Carve c;
    if (!ep::carve_workspace(T, num_topk, num_experts, num_ranks, block_m, &c))
        return EP_ERR_INVALID_ARG;
    // scratch: 4 bytes x ceil(T/32) chunks x (E + R) counters
    const int64_t nchunks = ((int64_t)T + ep::kChunkTokens - 1) / ep::kChunkTokens;
    if ((int64_t)sizeof(int32_t) * nchunks * ((int64_t)num_experts + num_ranks) >
        (int64_t)EP_STATIC_SCRATCH_BYTES)
        return EP_ERR_WORKSPACE_TOO_SMALL;
    if (!num_tokens_per_expert || !num_tokens_per_rank || !num_rows_per_rank || !expert_off ||
        !rank_off || !total_recv_rows || !error_word)
        return EP_ERR_INVALID_ARG;
    if (T > 0 && (!topk_idx || !is_token_in_rank || !dst_row))
        return EP_ERR_INVALID_ARG;
    const int64_t need_rows = ep::recv_rows_bound(T, num_topk, num_experts, block_m);
    if (recv_src_capacity < need_rows || (need_rows > 0 && !recv_src))
        return EP_ERR_CAPACITY;
    if ((uintptr_t)topk_idx % 8 != 0)
        return EP_ERR_ALIGNMENT;

    int32_t* scratch = nullptr;
    const ep_status_t st = ep::scratch_address(&scratch);
    if (st != EP_OK)
        return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t rc = cudaMemsetAsync(error_word, 0, sizeof(int32_t), s);
    if (rc != cudaSuccess)
        return ep::cuda_fail(rc, "ep_layout_static_scratch: clearing the error word");

    // A handle on the stack: scratch from the static array, every output
    // from the caller.  Nothing in the scratch needs to start at zero: the
    // count kernel writes every chunk row before the scan reads it.
    ep::Handle h = {};
    h.magic = ep::kHandleMagic;
    h.max_tokens = T;
    h.k = num_topk;
    h.E = num_experts;
    h.R = num_ranks;
    h.block_m = block_m;
    h.max_rows = need_rows;
    h.max_chunks = nchunks;
    h.chunk_counts = scratch;
    h.chunk_rank = scratch + h.max_chunks * num_experts;
    h.cnt = num_tokens_per_expert;
    h.expert_off = expert_off;
    h.rank_off = rank_off;
    h.tokens_per_rank = num_tokens_per_rank;
    h.rows_per_rank = num_rows_per_rank;
    h.total_rows = total_recv_rows;
    h.err = error_word;
    h.is_token_in_rank = is_token_in_rank;
    h.dst_row = dst_row;
    h.recv_src = recv_src;
    h.T = T;
    h.has_layout = 1;
    h.err_cleared = 1;
    rc = ep::launch_layout(h, topk_idx, T, s, /*allow_fused=*/false);
    return rc == cudaSuccess ? EP_OK : ep::cuda_fail(rc, "ep_layout_static_scratch");
}
