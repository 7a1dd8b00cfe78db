// api.cu -- host side of libtreeverify: argument checks, launch planning and
// the extern "C" entry points declared in include/treeverify.h.
#include <math.h>
#include <stdint.h>

#include "kernels.h"
#include "tv_common.cuh"

namespace {

int device_sms() {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess)
        return sms;
    cudaGetLastError();
    return 148;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// shared memory a block may opt in to on sm_100 (227 KB)
constexpr int SMEM_PER_BLOCK_OPTIN = 232448;

tv_status check_attn_desc(const tv_attn_desc* d) {
    if (!d) return TV_ERR_INVALID_ARG;
    if (d->batch < 1 || d->num_nodes < 1 || d->num_q_heads < 1 || d->num_kv_heads < 1) return TV_ERR_INVALID_ARG;
    if (d->num_q_heads % d->num_kv_heads) return TV_ERR_INVALID_ARG;
    if (d->num_nodes > TV_MAX_NODES_ATTN) return TV_ERR_UNSUPPORTED;
    if (d->head_dim != 64 && d->head_dim != 128) return TV_ERR_UNSUPPORTED;
    if (d->block_size != TV_BLOCK) return TV_ERR_UNSUPPORTED;
    if (d->max_blocks_per_seq < 1 || d->num_blocks < 1) return TV_ERR_INVALID_ARG;
    if (d->dtype != TV_BF16 && d->dtype != TV_F32) return TV_ERR_INVALID_ARG;
    if (!(d->softmax_scale >= 0.f) || isinf(d->softmax_scale)) return TV_ERR_INVALID_ARG;
    if ((int64_t)d->max_blocks_per_seq * TV_BLOCK > INT32_MAX / 2) return TV_ERR_UNSUPPORTED;
    return TV_OK;
}

// Which kernel runs and how the KV range is split.
//  - bf16 with head_dim 128 runs on the tensor cores: 128-row query tiles;
//    the KV splits of a tile form one thread-block cluster and merge their
//    partial results through each other's shared memory (no workspace).
//  - everything else runs on the CUDA cores: 32-row tiles, splits merged by
//    a second kernel through a global workspace.
// Splits are chosen so the main launch covers the SMs about once, and never
// below 256 tokens per split on the tensor cores (64 on the CUDA cores, whose
// tiles stream 32 tokens at a time).
void make_plan(const tv_attn_desc* d, tv_attn_plan* p) {
    const int G = d->num_q_heads / d->num_kv_heads;
    const int rows = G * d->num_nodes;
    const int sms = device_sms();
    const int64_t max_tokens = (int64_t)d->max_blocks_per_seq * TV_BLOCK;
    const bool tc = d->dtype == TV_BF16 && d->head_dim == 128;
    p->kernel = tc ? 0 : 1;
    const int tile_rows = tc ? tv::tc_rows_per_tile() : tv::simt_rows_per_tile();
    p->row_tiles = (rows + tile_rows - 1) / tile_rows;
    const int64_t base = (int64_t)d->batch * d->num_kv_heads * p->row_tiles;
    int64_t splits;
    if (tc) {
        splits = tv::tc_pick_splits(base, d->max_blocks_per_seq, sms);
    } else {
        splits = base >= sms ? 1 : (sms / base);
        const int64_t by_len = (max_tokens + 63) / 64;  // at least two 32-token chunks per split
        if (splits > by_len) splits = by_len;
        if (splits < 1) splits = 1;
        if (splits > 64) splits = 64;
    }
    p->num_splits = (int32_t)splits;
    p->grid_ctas = (int32_t)(base * splits);
    p->launches = (!tc && splits > 1) ? 2 : 1;
    size_t ws = 0;
    if (!tc && splits > 1) {
        const size_t rows_all = (size_t)d->batch * d->num_nodes * d->num_q_heads;
        ws = align256(sizeof(float) * splits * rows_all * d->head_dim) + align256(sizeof(float) * splits * rows_all);
    }
    p->workspace_bytes = ws;
}

tv_status check_sample_desc(const tv_sample_desc* d) {
    if (!d) return TV_ERR_INVALID_ARG;
    if (d->batch < 1 || d->num_nodes < 1 || d->vocab < 1) return TV_ERR_INVALID_ARG;
    if (d->num_nodes > 1024) return TV_ERR_UNSUPPORTED;
    if (d->vocab > 16 * 13824) return TV_ERR_UNSUPPORTED;
    if ((int64_t)d->batch * 16 > INT32_MAX) return TV_ERR_UNSUPPORTED;
    return TV_OK;
}

// One cluster per sequence; each CTA caches a slice of about 8K entries of
// two rows' p and q (two buffers: the current node's row and the next one's
// prefetch, 16 bytes per entry) so a 128K-entry row spreads over 16 SMs.
void make_sample_plan(const tv_sample_desc* d, tv_sample_plan* p) {
    const int max_c = tv::sample_max_cluster();
    int c = (d->vocab + 8191) / 8192;
    if (c > max_c) c = max_c;
    if (c < 1) c = 1;
    int slice = (d->vocab + c - 1) / c;
    slice = (slice + 3) / 4 * 4;
    int threads = ((slice + 7) / 8 + 31) / 32 * 32;
    if (threads < 64) threads = 64;
    if (threads > 512) threads = 512;
    p->cluster_ctas = c;
    p->threads = threads;
    p->slice = slice;
    // the two row buffers, then (when they fit) the gathered child values: p(x),
    // q(x), the uniform and the first child of every node, 16 bytes per node
    const size_t rows = 4 * sizeof(float) * (size_t)slice;
    const size_t gathered = 16 * (size_t)d->num_nodes;
    const bool gather = rows + gathered + tv::sample_static_smem() + 1024 <= (size_t)SMEM_PER_BLOCK_OPTIN;
    p->smem_bytes = (int32_t)(rows + (gather ? gathered : 0));
    p->launches = 1;
}

// the walk gathers the child values into shared memory when the plan made room
bool sample_gathers(const tv_sample_plan& p) { return (size_t)p.smem_bytes > 4 * sizeof(float) * (size_t)p.slice; }

}  // namespace

namespace {
tv_status verify_sample_common(const tv_sample_desc* desc, const float* p, const float* q, const int32_t* tree_tokens,
                               const int32_t* parent_idx, const float* uniforms, int32_t* accepted_path,
                               int32_t* accepted_len, int32_t* bonus_token, int32_t* dev_status, void* stream,
                               bool logits) {
    tv_status s = check_sample_desc(desc);
    if (s != TV_OK) return s;
    if (!p || !q || !tree_tokens || !uniforms || !accepted_path || !accepted_len || !bonus_token)
        return TV_ERR_INVALID_ARG;
    tv_sample_plan plan;
    make_sample_plan(desc, &plan);
    tv::SampleArgs a = {};
    a.p = p; a.q = q; a.tokens = tree_tokens; a.parent = parent_idx; a.counts = desc->node_counts;
    a.uniforms = uniforms;
    a.path = accepted_path; a.len = accepted_len; a.bonus = bonus_token; a.status = dev_status;
    a.B = desc->batch; a.N = desc->num_nodes; a.V = desc->vocab;
    a.cluster = plan.cluster_ctas; a.threads = plan.threads; a.slice = plan.slice; a.smem_bytes = plan.smem_bytes;
    a.vec4 = (desc->vocab % 4 == 0) && !(reinterpret_cast<uintptr_t>(p) & 15) && !(reinterpret_cast<uintptr_t>(q) & 15);
    a.logits = logits ? 1 : 0;
    a.gather = sample_gathers(plan) ? 1 : 0;
    int launches = 0;
    cudaError_t e = tv::launch_verify_sample(a, static_cast<cudaStream_t>(stream), &launches);
    return e == cudaSuccess ? TV_OK : TV_ERR_CUDA;
}
}  // namespace

extern "C" {

int32_t tv_version(void) { return 100; }

const char* tv_status_string(int32_t s) {
    switch (s) {
        case TV_OK: return "ok";
        case TV_ERR_INVALID_ARG: return "invalid argument";
        case TV_ERR_UNSUPPORTED: return "unsupported configuration";
        case TV_ERR_TREE: return "malformed tree (parent not before child, bad root, or token out of range)";
        case TV_ERR_BLOCK_TABLE: return "block table entry out of range or sequence longer than the table";
        case TV_ERR_WORKSPACE: return "workspace missing or too small";
        case TV_ERR_CUDA: return "CUDA runtime error";
        case TV_ERR_TIMEOUT: return "bounded device wait ran out";
        default: return "unknown status";
    }
}

tv_status tv_tree_attention_plan(const tv_attn_desc* desc, tv_attn_plan* plan) {
    tv_status s = check_attn_desc(desc);
    if (s != TV_OK) return s;
    if (!plan) return TV_ERR_INVALID_ARG;
    make_plan(desc, plan);
    return TV_OK;
}

size_t tv_tree_attention_workspace_size(const tv_attn_desc* desc) {
    if (check_attn_desc(desc) != TV_OK) return 0;
    tv_attn_plan p;
    make_plan(desc, &p);
    return p.workspace_bytes;
}

tv_status tv_tree_attention(const tv_attn_desc* desc, const void* q, const void* paged_k, const void* paged_v,
                            const int32_t* block_table, const int32_t* prefix_lens, const int32_t* parent_idx,
                            void* out, void* workspace, size_t workspace_bytes, int32_t* dev_status,
                            void* stream) {
    tv_status s = check_attn_desc(desc);
    if (s != TV_OK) return s;
    if (!q || !paged_k || !paged_v || !block_table || !prefix_lens || !out) return TV_ERR_INVALID_ARG;
    tv_attn_plan plan;
    make_plan(desc, &plan);
    if (plan.kernel == 0) {
        // the tensor-core path reads q, K and V with 16-byte vector loads / TMA
        const uintptr_t mis = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(paged_k) |
                              reinterpret_cast<uintptr_t>(paged_v) | reinterpret_cast<uintptr_t>(out);
        if (mis & 15) return TV_ERR_INVALID_ARG;
    }
    if (plan.workspace_bytes) {
        if (!workspace || workspace_bytes < plan.workspace_bytes) return TV_ERR_WORKSPACE;
        if (reinterpret_cast<uintptr_t>(workspace) & 255) return TV_ERR_WORKSPACE;
    }
    tv::AttnArgs a = {};
    a.q = q; a.k = paged_k; a.v = paged_v;
    a.block_table = block_table; a.prefix_lens = prefix_lens; a.parent = parent_idx;
    a.counts = desc->node_counts; a.out = out; a.status = dev_status;
    a.B = desc->batch; a.N = desc->num_nodes; a.Hq = desc->num_q_heads; a.Hkv = desc->num_kv_heads;
    a.G = a.Hq / a.Hkv; a.D = desc->head_dim; a.max_blocks = desc->max_blocks_per_seq;
    a.num_blocks = desc->num_blocks; a.splits = plan.num_splits; a.row_tiles = plan.row_tiles;
    const float scale = desc->softmax_scale > 0.f ? desc->softmax_scale : 1.0f / sqrtf((float)desc->head_dim);
    a.scale_log2 = scale * 1.4426950408889634f;
    a.blocks_per_split = (desc->max_blocks_per_seq + a.splits - 1) / a.splits;
    if (plan.workspace_bytes) {
        const size_t rows_all = (size_t)a.B * a.N * a.Hq;
        a.o_part = static_cast<float*>(workspace);
        a.lse_part = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                              align256(sizeof(float) * a.splits * rows_all * a.D));
    }
    int launches = 0;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = plan.kernel == 0 ? tv::launch_attn_tc(a, st, &launches)
                                     : tv::launch_attn_simt(a, desc->dtype == TV_BF16, st, &launches);
    return e == cudaSuccess ? TV_OK : TV_ERR_CUDA;
}

tv_status tv_verify_sample_plan(const tv_sample_desc* desc, tv_sample_plan* plan) {
    tv_status s = check_sample_desc(desc);
    if (s != TV_OK) return s;
    if (!plan) return TV_ERR_INVALID_ARG;
    make_sample_plan(desc, plan);
    return TV_OK;
}

size_t tv_verify_sample_workspace_size(const tv_sample_desc* desc) {
    (void)desc;
    return 0;
}

tv_status tv_commit_path(const tv_attn_desc* desc, void* paged_k, void* paged_v, const int32_t* block_table,
                         const int32_t* prefix_lens, const int32_t* accepted_path, const int32_t* accepted_len,
                         int32_t* new_prefix_lens, int32_t* dev_status, void* stream) {
    tv_status s = check_attn_desc(desc);
    if (s != TV_OK) return s;
    if (!paged_k || !paged_v || !block_table || !prefix_lens || !accepted_path || !accepted_len || !new_prefix_lens)
        return TV_ERR_INVALID_ARG;
    // other CTAs still read a sequence's prefix length while its new length is written
    if (static_cast<const void*>(new_prefix_lens) == static_cast<const void*>(prefix_lens)) return TV_ERR_INVALID_ARG;
    // rows move as 16-byte pieces
    if ((reinterpret_cast<uintptr_t>(paged_k) | reinterpret_cast<uintptr_t>(paged_v)) & 15) return TV_ERR_INVALID_ARG;
    tv::CommitArgs a = {};
    a.k = paged_k; a.v = paged_v; a.block_table = block_table; a.prefix_lens = prefix_lens;
    a.path = accepted_path; a.len = accepted_len; a.counts = desc->node_counts;
    a.new_prefix_lens = new_prefix_lens; a.status = dev_status;
    a.B = desc->batch; a.N = desc->num_nodes; a.Hkv = desc->num_kv_heads;
    a.row_bytes = desc->head_dim * (desc->dtype == TV_BF16 ? 2 : 4);
    a.max_blocks = desc->max_blocks_per_seq; a.num_blocks = desc->num_blocks;
    return tv::launch_commit(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? TV_OK : TV_ERR_CUDA;
}


tv_status tv_tree_fill_topk(const tv_sample_desc* desc, const float* q, const int32_t* parent_idx,
                            const int32_t* rank, int32_t* tree_tokens, int32_t* dev_status, void* stream) {
    tv_status s = check_sample_desc(desc);
    if (s != TV_OK) return s;
    if (!q || !tree_tokens) return TV_ERR_INVALID_ARG;
    tv::FillArgs a = {};
    a.q = q; a.parent = parent_idx; a.rank = rank; a.counts = desc->node_counts; a.tokens = tree_tokens;
    a.status = dev_status;
    a.B = desc->batch; a.N = desc->num_nodes; a.V = desc->vocab;
    tv::fill_topk_plan(a.V, &a.cluster, &a.slice, &a.smem_bytes);
    if ((int64_t)a.cluster * a.B * a.N > INT32_MAX) return TV_ERR_UNSUPPORTED;
    a.vec4 = (a.V % 4 == 0) && !(reinterpret_cast<uintptr_t>(q) & 15);
    return tv::launch_fill_topk(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? TV_OK : TV_ERR_CUDA;
}

tv_status tv_tree_shape(const double* accept, int32_t num_ranks, int32_t budget, int32_t max_depth,
                        int32_t* parent_idx, int32_t* rank, int32_t* num_nodes, double* expected_accepted) {
    if (!accept || !parent_idx || !rank || !num_nodes || !expected_accepted) return TV_ERR_INVALID_ARG;
    if (num_ranks < 1 || budget < 1 || max_depth < 0) return TV_ERR_INVALID_ARG;
    if (num_ranks > 32 || budget > 256) return TV_ERR_UNSUPPORTED;
    for (int i = 0; i < num_ranks; ++i)
        if (!(accept[i] >= 0.0 && accept[i] <= 1.0)) return TV_ERR_INVALID_ARG;
    *num_nodes = tv::tree_shape_dp(accept, num_ranks, budget, max_depth, parent_idx, rank, expected_accepted);
    return TV_OK;
}

tv_status tv_tree_shape_for_cost(const double* accept, int32_t num_ranks, int32_t max_budget, int32_t max_depth,
                                 double draft_cost, double alpha, int32_t* parent_idx, int32_t* rank,
                                 int32_t* num_nodes, double* expected_accepted, double* speedup) {
    if (!accept || !parent_idx || !rank || !num_nodes || !expected_accepted || !speedup) return TV_ERR_INVALID_ARG;
    if (num_ranks < 1 || max_budget < 1 || max_depth < 0) return TV_ERR_INVALID_ARG;
    if (!(draft_cost >= 0.0) || !(alpha >= 0.0) || isinf(draft_cost) || isinf(alpha)) return TV_ERR_INVALID_ARG;
    if (num_ranks > 32 || max_budget > 256) return TV_ERR_UNSUPPORTED;
    for (int i = 0; i < num_ranks; ++i)
        if (!(accept[i] >= 0.0 && accept[i] <= 1.0)) return TV_ERR_INVALID_ARG;
    *num_nodes = tv::tree_shape_for_cost(accept, num_ranks, max_budget, max_depth, draft_cost, alpha, parent_idx, rank,
                                         expected_accepted, speedup);
    return TV_OK;
}

tv_status tv_tree_merge(int32_t num_seqs, const int32_t* seq_offsets, const int32_t* tokens, int32_t max_nodes,
                        int32_t* parent_idx, int32_t* tree_tokens, int32_t* node_of_token, int32_t* num_nodes) {
    if (num_seqs < 0 || !seq_offsets || !parent_idx || !tree_tokens || !num_nodes || max_nodes < 1)
        return TV_ERR_INVALID_ARG;
    if (seq_offsets[0] != 0) return TV_ERR_INVALID_ARG;
    for (int k = 0; k < num_seqs; ++k)
        if (seq_offsets[k + 1] < seq_offsets[k]) return TV_ERR_INVALID_ARG;
    const int32_t total = seq_offsets[num_seqs];
    if (total > 0 && (!tokens || !node_of_token)) return TV_ERR_INVALID_ARG;
    for (int32_t j = 0; j < total; ++j)
        if (tokens[j] < 0) return TV_ERR_INVALID_ARG;
    const int n = tv::tree_merge(num_seqs, seq_offsets, tokens, max_nodes, parent_idx, tree_tokens, node_of_token);
    if (n < 0) return TV_ERR_UNSUPPORTED;
    *num_nodes = n;
    return TV_OK;
}

tv_status tv_tree_select(const int32_t* cand_parent, const int32_t* cand_token, const double* cand_prob,
                         int32_t num_candidates, int32_t budget, int32_t* parent_idx, int32_t* tree_tokens,
                         int32_t* cand_index, int32_t* num_nodes, double* expected_accepted) {
    if (!parent_idx || !tree_tokens || !cand_index || !num_nodes || !expected_accepted) return TV_ERR_INVALID_ARG;
    if (num_candidates < 0 || budget < 1) return TV_ERR_INVALID_ARG;
    if (num_candidates > 0 && (!cand_parent || !cand_token || !cand_prob)) return TV_ERR_INVALID_ARG;
    if (num_candidates > (1 << 20) || budget > 1024) return TV_ERR_UNSUPPORTED;
    for (int c = 0; c < num_candidates; ++c)
        if (!(cand_prob[c] >= 0.0 && cand_prob[c] <= 1.0)) return TV_ERR_INVALID_ARG;
    const int n = tv::tree_select(cand_parent, cand_token, cand_prob, num_candidates, budget, parent_idx, tree_tokens,
                                  cand_index, expected_accepted);
    if (n < 0) return TV_ERR_TREE;
    *num_nodes = n;
    return TV_OK;
}

tv_status tv_tree_select_batch(int32_t batch, const int32_t* cand_offsets, const int32_t* cand_parent,
                               const int32_t* cand_token, const double* cand_prob, int32_t budget,
                               int32_t* parent_idx, int32_t* tree_tokens, int32_t* cand_index, int32_t* node_counts,
                               double* expected_accepted) {
    if (batch < 1 || !cand_offsets || !node_counts || !parent_idx || !tree_tokens || !cand_index ||
        !expected_accepted)
        return TV_ERR_INVALID_ARG;
    if (budget < 1) return TV_ERR_INVALID_ARG;
    if (budget > 1024) return TV_ERR_UNSUPPORTED;
    if (cand_offsets[0] != 0) return TV_ERR_INVALID_ARG;
    for (int b = 0; b < batch; ++b)
        if (cand_offsets[b + 1] < cand_offsets[b]) return TV_ERR_INVALID_ARG;
    // every sequence is checked before any output is written
    for (int b = 0; b < batch; ++b) {
        const int32_t o = cand_offsets[b], m = cand_offsets[b + 1] - o;
        for (int c = 0; c < m; ++c) {
            if (!cand_parent || !cand_token || !cand_prob) return TV_ERR_INVALID_ARG;
            if (!(cand_prob[o + c] >= 0.0 && cand_prob[o + c] <= 1.0)) return TV_ERR_INVALID_ARG;
            if (cand_parent[o + c] < -1 || cand_parent[o + c] >= c) return TV_ERR_TREE;
        }
    }
    for (int b = 0; b < batch; ++b) {
        const int32_t o = cand_offsets[b], m = cand_offsets[b + 1] - o;
        int32_t n = 0;
        tv_status s = tv_tree_select(m ? cand_parent + o : nullptr, m ? cand_token + o : nullptr,
                                     m ? cand_prob + o : nullptr, m, budget, parent_idx + (size_t)b * budget,
                                     tree_tokens + (size_t)b * budget, cand_index + (size_t)b * budget, &n,
                                     expected_accepted + b);
        if (s != TV_OK) return s;
        node_counts[b] = n;
    }
    return TV_OK;
}

tv_status tv_tree_select_device(int32_t batch, int32_t max_candidates, const int32_t* cand_offsets,
                                const int32_t* cand_parent, const int32_t* cand_token, const float* cand_prob,
                                int32_t budget, int32_t* parent_idx, int32_t* tree_tokens, int32_t* cand_index,
                                int32_t* node_counts, double* expected_accepted, int32_t* dev_status, void* stream) {
    if (batch < 1 || max_candidates < 0 || budget < 1) return TV_ERR_INVALID_ARG;
    if (!cand_offsets || !parent_idx || !tree_tokens || !cand_index || !node_counts || !expected_accepted)
        return TV_ERR_INVALID_ARG;
    if (max_candidates > 0 && (!cand_parent || !cand_token || !cand_prob)) return TV_ERR_INVALID_ARG;
    if (budget > 1024 || max_candidates > TV_SELECT_MAX_CANDIDATES) return TV_ERR_UNSUPPORTED;
    tv::SelectArgs a = {};
    a.offsets = cand_offsets; a.cand_parent = cand_parent; a.cand_token = cand_token; a.cand_prob = cand_prob;
    a.parent_idx = parent_idx; a.tree_tokens = tree_tokens; a.cand_index = cand_index; a.node_counts = node_counts;
    a.expected = expected_accepted; a.status = dev_status;
    a.B = batch; a.budget = budget; a.max_cand = max_candidates;
    return tv::launch_select(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? TV_OK : TV_ERR_CUDA;
}

tv_status tv_verify_sample(const tv_sample_desc* desc, const float* p, const float* q, const int32_t* tree_tokens,
                           const int32_t* parent_idx, const float* uniforms, int32_t* accepted_path,
                           int32_t* accepted_len, int32_t* bonus_token, void* workspace, size_t workspace_bytes,
                           int32_t* dev_status, void* stream) {
    (void)workspace;
    (void)workspace_bytes;
    return verify_sample_common(desc, p, q, tree_tokens, parent_idx, uniforms, accepted_path, accepted_len,
                                bonus_token, dev_status, stream, false);
}

tv_status tv_verify_sample_logits(const tv_sample_desc* desc, const float* target_logits, const float* draft_logits,
                                  const int32_t* tree_tokens, const int32_t* parent_idx, const float* uniforms,
                                  int32_t* accepted_path, int32_t* accepted_len, int32_t* bonus_token,
                                  void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream) {
    (void)workspace;
    (void)workspace_bytes;
    return verify_sample_common(desc, target_logits, draft_logits, tree_tokens, parent_idx, uniforms, accepted_path,
                                accepted_len, bonus_token, dev_status, stream, true);
}

}  // extern "C"
