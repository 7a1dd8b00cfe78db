// commit.cu -- the step after verification: the accepted path joins the cached
// prefix (blog "Speculative decoding x tree attention", section "KV cache
// management and prefix sharing"; glossary "Tree-based speculative decoding",
// section "KV cache management challenges": after verification every tree
// entry off the accepted path is dropped, and paged caches do it through
// block-table operations).
//
// Tree node j of sequence b sits at logical position L_b + j.  The root stays
// at L_b; accepted node path[k] moves to L_b + 1 + k; the new length is
// L_b + 1 + len.  A move whose source already is its destination (path[k] ==
// k + 1) is skipped.
//
// One CTA per (sequence, KV head).  Every CTA of a sequence validates the path,
// the length and the block ids of the tree's span the same way, so either all
// of them move their head's rows or none does.  A destination can be another
// move's source (path [2, 5]: node 5 goes where node 2 was), so each CTA reads
// all of its rows into shared memory before it writes any.
#include "kernels.h"
#include "tv_common.cuh"

namespace tv {
namespace {

constexpr int CM_THREADS = 256;

__global__ void __launch_bounds__(CM_THREADS) commit_kernel(const CommitArgs a) {
    extern __shared__ uint4 stage[];
    const int b = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
    const int N = a.N;
    const int L = a.prefix_lens[b];
    const int n = a.len[b];
    bool bad_count;
    const int nodes = seq_nodes(a.counts, b, N, bad_count);  // this sequence's tree nodes
    const int32_t* path = a.path + (size_t)b * N;
    const int32_t* bt = a.block_table + (size_t)b * a.max_blocks;
    const bool lead = h == 0 && tid == 0;
    if (n < 0 || (nodes == 0 && n == 0 && !bad_count)) {
        // flagged by the walk, or no tree this step: nothing is committed
        if (lead) a.new_prefix_lens[b] = L;
        return;
    }
    // validation, identical in every CTA of the sequence
    int bad = 0;
    if (bad_count || L < 0 || n > nodes - 1 || (long long)L + nodes > (long long)a.max_blocks * TV_BLOCK)
        bad = TV_ERR_INVALID_ARG;
    if (!bad)
        for (int k = tid; k < n; k += CM_THREADS) {
            const int prev = k == 0 ? 0 : path[k - 1];
            if (path[k] <= prev || path[k] >= nodes) bad = TV_ERR_TREE;
        }
    if (!bad)
        for (int bi = L / TV_BLOCK + tid; bi <= (L + nodes - 1) / TV_BLOCK; bi += CM_THREADS) {
            const int id = bt[bi];
            if (id < 0 || id >= a.num_blocks) bad = TV_ERR_BLOCK_TABLE;
        }
    __shared__ int s_bad;
    if (tid == 0) s_bad = 0;
    __syncthreads();
    if (bad) atomicMax(&s_bad, bad);
    __syncthreads();
    if (s_bad) {
        if (lead) {
            a.new_prefix_lens[b] = L;
            report(a.status, s_bad);
        }
        return;
    }
    // rows of this head: n positions x {K, V}, cpr 16-byte chunks each
    const int cpr = a.row_bytes / 16;
    const int total = n * 2 * cpr;
    const size_t pos_stride = (size_t)a.Hkv * a.row_bytes;  // bytes per cache position
    auto row_off = [&](int t) {
        return ((size_t)bt[t / TV_BLOCK] * TV_BLOCK + t % TV_BLOCK) * pos_stride + (size_t)h * a.row_bytes;
    };
    for (int i = tid; i < total; i += CM_THREADS) {
        const int k = i / (2 * cpr), c = (i / cpr) & 1, off = i % cpr;
        if (path[k] == k + 1) continue;  // already in place
        const uint8_t* cache = static_cast<const uint8_t*>(c == 0 ? a.k : a.v);
        stage[i] = reinterpret_cast<const uint4*>(cache + row_off(L + path[k]))[off];
    }
    __syncthreads();
    for (int i = tid; i < total; i += CM_THREADS) {
        const int k = i / (2 * cpr), c = (i / cpr) & 1, off = i % cpr;
        if (path[k] == k + 1) continue;
        uint8_t* cache = static_cast<uint8_t*>(c == 0 ? a.k : a.v);
        reinterpret_cast<uint4*>(cache + row_off(L + 1 + k))[off] = stage[i];
    }
    if (lead) a.new_prefix_lens[b] = L + 1 + n;
}

}  // namespace

size_t commit_smem_bytes(int N, int row_bytes) {
    const size_t rows = N > 1 ? (size_t)(N - 1) * 2 : 1;
    return rows * (size_t)row_bytes;
}

cudaError_t launch_commit(const CommitArgs& a, cudaStream_t st) {
    const size_t smem = commit_smem_bytes(a.N, a.row_bytes);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(commit_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    commit_kernel<<<dim3(a.B, a.Hkv), CM_THREADS, smem, st>>>(a);
    return cudaGetLastError();
}

}  // namespace tv
