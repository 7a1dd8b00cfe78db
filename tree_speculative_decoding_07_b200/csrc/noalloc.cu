// noalloc.cu -- tv_tree_attention_static: tree attention for callers that
// cannot allocate device memory.
//
// Some callers of this library have no way to hand it a workspace: a host
// process that gives all device memory to a fixed pool at start-up, a plugin
// inside a serving runtime whose hot path must not call the CUDA allocator
// (cudaMalloc can synchronise the device and stall every stream), or code
// recorded into a CUDA graph where a fresh allocation per call is not
// possible.  For them this entry point runs exactly the same kernels as
// tv_tree_attention, with the scratch memory taken from a file-scope device
// array that every GPU which loads the library holds until the process exits.
#include <mutex>

#include "kernels.h"
#include "tv_common.cuh"

namespace {

// Fixed scratch.  Tensor-core calls (bf16, head_dim 128) merge their KV splits
// through the cluster's shared memory and need none.  CUDA-core calls with
// several KV splits keep fp32 partial outputs and their log-sum-exp for every
// (split, query row): 4 * (head_dim + 1) bytes each.  The split count is chosen
// so splits x query rows stay within 32 rows per SM (4,736 on a 148-SM B200),
// i.e. at most about 2.4 MB at head_dim 128 and 1.2 MB at 64; 2 MiB covers
// every head_dim-64 call and head_dim-128 calls up to about 4,000
// (split, row) pairs, and larger ones are refused with TV_ERR_WORKSPACE.
__device__ __align__(256) unsigned char g_scratch[TV_STATIC_SCRATCH_BYTES];

constexpr int MAX_DEVICES = 64;
std::mutex g_mutex;
void* g_scratch_addr[MAX_DEVICES] = {};

// Device address of g_scratch on the current device.  In host code the name
// g_scratch is only a host-side stand-in, so the address is looked up once per
// device, with that device current, and cached.
tv_status scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return TV_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return TV_ERR_CUDA;
        }
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return TV_OK;
}

}  // namespace

extern "C" tv_status tv_tree_attention_static(const tv_attn_desc* desc, const void* q, const void* paged_k,
                                              const void* paged_v, const int32_t* block_table,
                                              const int32_t* prefix_lens, const int32_t* parent_idx, void* out,
                                              int32_t* dev_status, void* stream) {
    tv_attn_plan plan;
    tv_status s = tv_tree_attention_plan(desc, &plan);
    if (s != TV_OK) return s;
    if (plan.workspace_bytes > (size_t)TV_STATIC_SCRATCH_BYTES) return TV_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (plan.workspace_bytes) {
        s = scratch_address(&scratch);
        if (s != TV_OK) return s;
        // every partial the merge reads is written earlier in the same call, so
        // nothing in the array needs clearing
    }
    return tv_tree_attention(desc, q, paged_k, paged_v, block_table, prefix_lens, parent_idx, out, scratch,
                             plan.workspace_bytes ? (size_t)TV_STATIC_SCRATCH_BYTES : 0, dev_status, stream);
}
