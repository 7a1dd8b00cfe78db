// kernels.h -- launch interfaces between the host API (api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace tv {

struct AttnArgs {
    const void* q;
    const void* k;
    const void* v;
    const int32_t* block_table;
    const int32_t* prefix_lens;
    const int32_t* parent;  // [B][N]; NULL: every tree is a chain (parent of node i is i - 1)
    const int32_t* counts;  // [B] nodes per sequence (0..N); NULL: N for every sequence
    void* out;
    float* o_part;      // CUDA-core path: [splits][B][N][Hq][D] fp32 partial outputs (normalised)
    float* lse_part;    // CUDA-core path: [splits][B][N][Hq] log2-domain log-sum-exp of each partial
    int32_t* status;
    int B, N, Hq, Hkv, G, D, max_blocks, num_blocks, splits, row_tiles;
    int blocks_per_split;  // tensor-core path: split s covers logical blocks [s * bps, (s + 1) * bps)
    float scale_log2;   // softmax_scale * log2(e)
};

// CUDA-core split-KV kernel (fp32 or bf16 storage, fp32 math) + LSE combine.
cudaError_t launch_attn_simt(const AttnArgs& a, bool bf16, cudaStream_t st, int* launches);
int simt_rows_per_tile();

// Tensor-core (tcgen05 / TMEM / TMA) bf16 kernel, head_dim 128.
cudaError_t launch_attn_tc(const AttnArgs& a, cudaStream_t st, int* launches);
int tc_rows_per_tile();
int tc_max_splits();
int tc_pick_splits(int64_t groups, int64_t max_blocks, int sms);

struct SampleArgs {
    const float* p;
    const float* q;
    const int32_t* tokens;
    const int32_t* parent;  // [B][N]; NULL: every tree is a chain
    const int32_t* counts;  // [B] nodes per sequence (0..N); NULL: N for every sequence
    const float* uniforms;
    int32_t* path;
    int32_t* len;
    int32_t* bonus;
    int32_t* status;
    int B, N, V;
    int cluster, threads, slice, smem_bytes;
    int vec4;           // rows start 16-byte aligned and V % 4 == 0
    int logits;         // p and q hold the two models' logits: the walk applies the row softmax
    int gather;         // every child's p(x), q(x) and uniform are gathered into shared memory first
};

cudaError_t launch_verify_sample(const SampleArgs& a, cudaStream_t st, int* launches);

// KV commit of the accepted path (one launch).
struct CommitArgs {
    void* k;
    void* v;
    const int32_t* block_table;
    const int32_t* prefix_lens;
    const int32_t* path;   // [B][N] accepted node indices, root excluded
    const int32_t* len;    // [B] accepted lengths (< 0: flagged, no commit)
    const int32_t* counts; // [B] tree nodes per sequence (0..N); NULL: N for every sequence
    int32_t* new_prefix_lens;
    int32_t* status;
    int B, N, Hkv, row_bytes, max_blocks, num_blocks;
};
cudaError_t launch_commit(const CommitArgs& a, cudaStream_t st);
size_t commit_smem_bytes(int N, int row_bytes);
int sample_max_cluster();
size_t sample_static_smem();

// Top-k branching: child tokens from each parent's draft distribution (one launch).
struct FillArgs {
    const float* q;          // [B][N][V] draft distributions (or logits: the order is the same)
    const int32_t* parent;   // [B][N]; NULL: chains
    const int32_t* rank;     // [B][N] child ranks; NULL: a child's position among its siblings
    const int32_t* counts;   // [B] nodes per sequence; NULL: N
    int32_t* tokens;         // [B][N] written for children only
    int32_t* status;
    int B, N, V;
    int cluster, slice, smem_bytes, vec4;
};
void fill_topk_plan(int V, int* cluster, int* slice, int* smem_bytes);
cudaError_t launch_fill_topk(const FillArgs& a, cudaStream_t st);

// Budget-constrained tree shape (host).  Returns the node count.
int tree_shape_dp(const double* accept, int k, int budget, int max_depth, int32_t* parent, int32_t* rank,
                  double* value);

// The budget whose best tree maximises the step speedup (host).  Returns the node count.
int tree_shape_for_cost(const double* accept, int k, int max_budget, int max_depth, double draft_cost, double alpha,
                        int32_t* parent, int32_t* rank, double* value, double* speedup);

// SpecInfer's token-tree merge of several drafts' sequences (host).  Returns the
// node count, -1 if it would exceed max_nodes.
int tree_merge(int num_seqs, const int32_t* offsets, const int32_t* tokens, int max_nodes, int32_t* parent_idx,
               int32_t* tree_tokens, int32_t* node_of);

// Dynamic tree selection from a candidate set (host).  Returns the node count, -1 if not topological.
int tree_select(const int32_t* cand_parent, const int32_t* cand_token, const double* cand_prob, int M, int budget,
                int32_t* parent_idx, int32_t* tree_tokens, int32_t* cand_index, double* value);

// Dynamic tree selection on the device: one CTA per sequence (one launch).
struct SelectArgs {
    const int32_t* offsets;      // [B + 1] candidate ranges
    const int32_t* cand_parent;  // parent candidate (local to the sequence), -1 for a child of the root
    const int32_t* cand_token;
    const float* cand_prob;
    int32_t* parent_idx;         // [B][budget]
    int32_t* tree_tokens;        // [B][budget]
    int32_t* cand_index;         // [B][budget]
    int32_t* node_counts;        // [B]
    double* expected;            // [B]
    int32_t* status;
    int B, budget, max_cand;
};
size_t select_smem_bytes(int max_cand, int budget);
cudaError_t launch_select(const SelectArgs& a, cudaStream_t st);

}  // namespace tv
