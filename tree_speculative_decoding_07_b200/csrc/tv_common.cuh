// tv_common.cuh -- small device/host helpers shared by the libtreeverify kernels.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "treeverify.h"

#define TV_MAX_NODES_ATTN 128
#define TV_BLOCK 16

namespace tv {

// Record the first data-dependent error; later ones are dropped.
__device__ __forceinline__ void report(int32_t* status, int32_t code) {
    if (status) atomicCAS(status, 0, code);
}

template <typename T> struct Elem;
template <> struct Elem<float> {
    static __device__ __forceinline__ float load(const float* p) { return *p; }
    static __device__ __forceinline__ void store(float* p, float v) { *p = v; }
};
template <> struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float load(const __nv_bfloat16* p) { return __bfloat162float(*p); }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
};

// A tree is well formed when node 0 is the root (parent -1) and every other
// node's parent precedes it; then ancestor walks terminate and the nodes are
// in topological order.
// Nodes of sequence b: counts[b], or N when no counts are given.  A count
// outside [0, N] sets `bad` and yields N (the caller reports the error and
// writes no valid output for the sequence).
__device__ __forceinline__ int seq_nodes(const int32_t* counts, int b, int N, bool& bad) {
    if (!counts) {
        bad = false;
        return N;
    }
    const int n = counts[b];
    bad = n < 0 || n > N;
    return bad ? N : n;
}

// Parent of node i of sequence b; a NULL parent array means a chain.
__device__ __forceinline__ int32_t parent_at(const int32_t* parent, int b, int N, int i) {
    return parent ? parent[(size_t)b * N + i] : i - 1;
}

__device__ __forceinline__ bool parent_ok(const int32_t* parent, int i) {
    int p = parent[i];
    return i == 0 ? p == -1 : (p >= 0 && p < i);
}

// Tokens of sequence b handled by KV split s (of `splits`): balanced,
// 16-token aligned ranges over [0, total).
__device__ __forceinline__ void split_range(int total, int splits, int s, int& t0, int& t1) {
    int per = (total + splits - 1) / splits;
    per = (per + TV_BLOCK - 1) / TV_BLOCK * TV_BLOCK;
    t0 = min(total, s * per);
    t1 = min(total, t0 + per);
}

}  // namespace tv
