// select.cu -- the dynamic draft tree selected on the GPU (tv_tree_select_device).
//
// EAGLE-2's dynamic tree (LLM Primer VI ch. 9, 9.2): the draft grows many
// candidate paths and the tree that is verified is chosen among them.  The
// choice is the glossary's budget-constrained optimisation (the tree's
// expected accepted tokens under a node budget) with the draft's own path
// probability as each candidate's acceptance estimate: a candidate's score is
// the product of its draft probabilities along the path, and candidates are
// taken by descending score (equal scores: lower index first), each only once
// its parent is in, until the tree holds `budget` nodes with the root.
//
// With probabilities in [0, 1] a parent's score is at least its child's, and a
// parent's index is below its child's, so every parent comes before its
// children in that order: the taken set is exactly the first K = min(budget -
// 1, M) candidates of the order, and node k + 1 is the candidate of rank k.
// One CTA per sequence computes the scores in index order (a parent is always
// scored before its child), ranks every candidate by counting the candidates
// ahead of it, and writes the tree.  Scores are fp64 products formed in the
// order of the path, root first, so they equal a sequential evaluation bit
// for bit; the tree's value is their sum in node order.
#include "kernels.h"
#include "tv_common.cuh"

namespace tv {
namespace {

constexpr int SEL_THREADS = 512;

__global__ void __launch_bounds__(SEL_THREADS) select_tree_kernel(SelectArgs a) {
    extern __shared__ double sel_dyn[];
    double* score = sel_dyn;                                            // [max_cand]
    int32_t* par = reinterpret_cast<int32_t*>(score + a.max_cand);      // [max_cand]
    int32_t* rank = par + a.max_cand;                                   // [max_cand]; first a scored flag
    int32_t* node_cand = rank + a.max_cand;                             // [budget]
    __shared__ int s_bad;
    const int b = blockIdx.x, tid = threadIdx.x, T = blockDim.x;
    const int o = a.offsets[b];
    const int M = a.offsets[b + 1] - o;
    int32_t* out_par = a.parent_idx + (size_t)b * a.budget;
    int32_t* out_tok = a.tree_tokens + (size_t)b * a.budget;
    int32_t* out_idx = a.cand_index + (size_t)b * a.budget;
    if (tid == 0) s_bad = 0;
    __syncthreads();
    if (M < 0 || M > a.max_cand || o < 0) {
        // a count this launch was not sized for: nothing is selected for the sequence
        for (int j = tid; j < a.budget; j += T) out_par[j] = out_tok[j] = out_idx[j] = -1;
        if (tid == 0) {
            a.node_counts[b] = -1;
            a.expected[b] = 0.0;
            report(a.status, M < 0 || o < 0 ? TV_ERR_INVALID_ARG : TV_ERR_UNSUPPORTED);
        }
        return;
    }
    for (int c = tid; c < M; c += T) {
        const int p = a.cand_parent[o + c];
        const float pr = a.cand_prob[o + c];
        par[c] = p;
        rank[c] = 0;
        if (p < -1 || p >= c) atomicMax(&s_bad, TV_ERR_TREE);
        if (!(pr >= 0.f && pr <= 1.f)) atomicMax(&s_bad, TV_ERR_INVALID_ARG);
    }
    __syncthreads();
    if (s_bad) {
        for (int j = tid; j < a.budget; j += T) out_par[j] = out_tok[j] = out_idx[j] = -1;
        if (tid == 0) {
            a.node_counts[b] = -1;
            a.expected[b] = 0.0;
            report(a.status, s_bad);
        }
        return;
    }
    // ---- scores, in chunks of T candidates in index order: every parent of a chunk
    // lies in an earlier chunk or earlier in this one, so a few read / write rounds
    // per chunk score it (rank[] flags the scored ones meanwhile)
    for (int c0 = 0; c0 < M; c0 += T) {
        const int c = c0 + tid;
        bool done = c >= M;
        for (;;) {
            double v = 0.0;
            bool ready = false;
            if (!done) {
                const int p = par[c];
                const double pr = (double)a.cand_prob[o + c];
                if (p < 0) {
                    v = 1.0 * pr;
                    ready = true;
                } else if (p < c0 || rank[p]) {
                    v = score[p] * pr;
                    ready = true;
                }
            }
            __syncthreads();
            if (ready) {
                score[c] = v;
                rank[c] = 1;
                done = true;
            }
            if (!__syncthreads_or(!done)) break;
        }
    }
    // ---- ranks: the candidates ahead of c in (score descending, index ascending)
    const int K = min(a.budget - 1, M);
    for (int c = tid; c < M; c += T) {
        const double s = score[c];
        int r = 0;
        for (int c2 = 0; c2 < M; ++c2) {
            const double s2 = score[c2];
            r += (s2 > s || (s2 == s && c2 < c)) ? 1 : 0;
        }
        rank[c] = r;
        if (r < K) node_cand[r] = c;
    }
    __syncthreads();
    // ---- the tree: node 0 the root, node k + 1 the candidate of rank k
    for (int j = tid; j < a.budget; j += T) {
        if (j == 0) {
            out_par[0] = -1;
            out_tok[0] = -1;
            out_idx[0] = -1;
        } else if (j <= K) {
            const int c = node_cand[j - 1];
            const int p = par[c];
            out_par[j] = p < 0 ? 0 : rank[p] + 1;
            out_tok[j] = a.cand_token[o + c];
            out_idx[j] = c;
        } else {
            out_par[j] = out_tok[j] = out_idx[j] = -1;
        }
    }
    if (tid == 0) {
        double total = 0.0;
        for (int k = 0; k < K; ++k) total += score[node_cand[k]];
        a.expected[b] = total;
        a.node_counts[b] = K + 1;
    }
}

}  // namespace

size_t select_smem_bytes(int max_cand, int budget) {
    return (size_t)max_cand * (sizeof(double) + 2 * sizeof(int32_t)) + (size_t)budget * sizeof(int32_t);
}

cudaError_t launch_select(const SelectArgs& a, cudaStream_t st) {
    const size_t smem = select_smem_bytes(a.max_cand, a.budget);
    cudaError_t e = cudaFuncSetAttribute(select_tree_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    select_tree_kernel<<<a.B, SEL_THREADS, smem, st>>>(a);
    return cudaGetLastError();
}

}  // namespace tv
