/*
 * treeverify.h -- C ABI of libtreeverify, the target model's verification
 * step of tree-based speculative decoding on one NVIDIA B200 (sm_100a).
 *
 * The step has two parts, each one call:
 *
 *  tv_tree_attention  every draft-tree node attends to its sequence's cached
 *                     prefix and to its own root path, in one pass.  Defined
 *                     by the glossary page "Tree-based speculative decoding"
 *                     (jisaku.com), section "Tree attention": the mask
 *                     M[i][j] = 1 iff node j is node i or one of its
 *                     ancestors; its 5-node instance is the blog "Speculative
 *                     decoding x tree attention" (radar-34b), section 3,
 *                     figure "Tree Attention Verification Matrix".
 *
 *  tv_verify_sample   the lossless acceptance walk.  Defined by the same blog,
 *                     section 2, table "Rejection Sampling Acceptance
 *                     Condition" (accept x with probability min(1, p(x)/q(x)),
 *                     on rejection resample from max(0, p - q) normalised) and
 *                     the glossary's section "SpecInfer" (the tree is verified
 *                     root-down, depth first; a rejected child hands the
 *                     renormalised residual to its next sibling).
 *
 * Around the step:
 *
 *  tv_verify_sample_logits  the same walk on the two models' logits, the row
 *                     softmax formed inside the walk.
 *  tv_commit_path     after verification, the accepted path joins the cached
 *                     prefix (blog, "KV cache management and prefix sharing";
 *                     glossary, "KV cache management challenges").
 *  tv_tree_shape, tv_tree_fill_topk, tv_tree_select(_device)  building the
 *                     tree that is verified (glossary, tree-structure
 *                     optimisation: top-k branching and budget-constrained
 *                     optimisation; LLM Primer VI ch. 9, 9.2: EAGLE-2's
 *                     dynamic tree).
 *
 * Ragged batches (trees of different sizes in one call) go through the
 * descriptors' node_counts; a NULL parent_idx means chains (linear
 * speculation).
 *
 * Conventions shared by all calls
 *  - Every array pointer is a caller-owned DEVICE pointer unless stated
 *    otherwise (tv_tree_shape and tv_tree_select work on host arrays);
 *    descriptors and plan structs are host memory.  The library
 *    never allocates device memory and never synchronises the stream.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Work is enqueued asynchronously on it.
 *  - Host-checkable errors (shapes, dtype, null pointers, workspace size)
 *    return a status before anything is launched.
 *  - Data-dependent errors (a malformed tree, a block id or token id out of
 *    range) are written by the kernels to `*dev_status` (a device int32 the
 *    caller zeroes; may be NULL) with the first error code winning; the
 *    affected sequence gets sentinel outputs (NaN attention rows, -1 tokens)
 *    and the kernels exit normally.  Kernels never trap.
 *  - Results are deterministic: the same inputs give bit-identical outputs.
 */
#ifndef TREEVERIFY_H
#define TREEVERIFY_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TV_API __attribute__((visibility("default")))
#else
#define TV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    TV_OK = 0,
    TV_ERR_INVALID_ARG = 1,   /* bad descriptor field, null pointer, bad size */
    TV_ERR_UNSUPPORTED = 2,   /* valid but not supported by the library (e.g. head_dim) */
    TV_ERR_TREE = 3,          /* device: parent_idx not topological, or token out of range */
    TV_ERR_BLOCK_TABLE = 4,   /* device: block id outside [0, num_blocks) */
    TV_ERR_WORKSPACE = 5,     /* workspace null or smaller than the *_workspace_size value */
    TV_ERR_CUDA = 6,          /* a CUDA runtime call failed (launch configuration etc.) */
    TV_ERR_TIMEOUT = 7        /* device: a bounded wait ran out */
} tv_status;

typedef enum { TV_BF16 = 0, TV_F32 = 1 } tv_dtype;

/*
 * Tree attention problem.
 *   q, out      [batch][num_nodes][num_q_heads][head_dim], dtype, contiguous
 *   paged_k/v   [num_blocks][block_size][num_kv_heads][head_dim], dtype
 *   block_table [batch][max_blocks_per_seq] int32: logical block j of
 *               sequence b lives in physical block block_table[b][j]
 *   prefix_lens [batch] int32: L_b, committed tokens before the tree
 *   parent_idx  [batch][num_nodes] int32: parent_idx[b][0] = -1 (the root,
 *               i.e. the last committed token), 0 <= parent_idx[b][i] < i;
 *               NULL means every tree is a chain (parent of node i is i - 1:
 *               linear speculation, whose mask is plain causal)
 *   node_counts (descriptor field) [batch] int32 device array, or NULL: the
 *               number n_b of tree nodes of sequence b, 0 <= n_b <= num_nodes
 *               (ragged trees in one call; num_nodes is the capacity and the
 *               row stride).  Nodes n_b .. num_nodes-1 are padding: their
 *               parent_idx entries are ignored and their `out` rows are not
 *               written; n_b = 0 leaves the sequence out of this step.  A count
 *               outside [0, num_nodes] gives the sequence NaN rows and
 *               TV_ERR_INVALID_ARG in *dev_status.  NULL = num_nodes for all b.
 * Node i's key/value sit at logical position L_b + i of the paged cache;
 * the caller writes them before the call.  Query head h reads KV head
 * h / (num_q_heads / num_kv_heads).  Row (b, i, h) of `out` is softmax
 * attention of q[b][i][h] over positions t < L_b and the positions L_b + j
 * of the nodes j on i's root path, with scores scaled by softmax_scale
 * (0 means 1/sqrt(head_dim)).  Cache slots at positions >= L_b + num_nodes
 * inside an allocated block are never used.  For bf16 with head_dim 128
 * (the tensor-core path) q, paged_k, paged_v and out must be 16-byte
 * aligned, else TV_ERR_INVALID_ARG.
 */
typedef struct {
    int32_t batch;
    int32_t num_nodes;           /* 1..128 */
    int32_t num_q_heads;
    int32_t num_kv_heads;        /* divides num_q_heads */
    int32_t head_dim;            /* 64 or 128 */
    int32_t block_size;          /* 16 */
    int32_t max_blocks_per_seq;  /* >= ceil((L_b + num_nodes) / block_size) for every b */
    int32_t num_blocks;          /* physical blocks in paged_k / paged_v */
    int32_t dtype;               /* tv_dtype of q, paged_k, paged_v and out */
    float softmax_scale;         /* 0 => 1/sqrt(head_dim) */
    const int32_t *node_counts;  /* device [batch] nodes per sequence, or NULL (= num_nodes each) */
} tv_attn_desc;

/* How a call will run (host-side query; launches nothing). */
typedef struct {
    int32_t kernel;              /* 0 = tensor-core (tcgen05) bf16 path, 1 = CUDA-core path */
    int32_t num_splits;          /* KV splits per (sequence, KV head, row tile); on the tensor-core
                                    path the splits of a row tile form one thread-block cluster */
    int32_t row_tiles;           /* 128-row query tiles per (sequence, KV head) */
    int32_t grid_ctas;           /* CTAs in the main launch */
    int32_t launches;            /* kernel launches per call */
    size_t workspace_bytes;      /* same value as tv_tree_attention_workspace_size */
} tv_attn_plan;

TV_API tv_status tv_tree_attention_plan(const tv_attn_desc *desc, tv_attn_plan *plan);

/* Device workspace the call needs, in bytes (0 when none: always so on the
 * tensor-core path, whose KV splits merge inside a thread-block cluster).
 * Ownership stays with the caller; it must be 256-byte aligned and may be
 * reused across calls that are ordered on one stream (a call reads only what
 * it wrote there itself).  Calls that share a workspace must not overlap. */
TV_API size_t tv_tree_attention_workspace_size(const tv_attn_desc *desc);

TV_API tv_status tv_tree_attention(const tv_attn_desc *desc, const void *q, const void *paged_k,
                            const void *paged_v, const int32_t *block_table,
                            const int32_t *prefix_lens, const int32_t *parent_idx, void *out,
                            void *workspace, size_t workspace_bytes, int32_t *dev_status,
                            void *stream);

/*
 * Tree attention without a caller-provided workspace.  (The pages describe
 * no such call; it exists for callers of this library.)
 *
 * Same inputs, outputs, layouts and results as tv_tree_attention, for callers
 * that cannot allocate device memory when they call: a process that hands all
 * device memory to a fixed pool at start-up, a serving-runtime plugin whose
 * hot path must not call the CUDA allocator (cudaMalloc may synchronise the
 * device), or work recorded into a CUDA graph.  The scratch memory comes from
 * a fixed device array of TV_STATIC_SCRATCH_BYTES inside the library, which
 * every GPU that loads the library holds until the process exits; nothing is
 * allocated or freed by this call.  Tensor-core calls (bf16, head_dim 128) need
 * no scratch; CUDA-core calls with several KV splits need
 * tv_tree_attention_workspace_size() bytes of it.
 *  - Returns TV_ERR_WORKSPACE, before launching anything, when the problem
 *    needs more scratch than TV_STATIC_SCRATCH_BYTES (fp32 or bf16 at
 *    head_dim 128 on the CUDA cores with more than about 4,000 (KV split,
 *    query row) pairs).
 *  - The first call on each device looks up the array's device address (with
 *    that device current); make that first call before any stream capture.
 *  - All calls share the one array per device, and it keeps the previous
 *    call's contents (every value a call reads it has written itself):
 *    calls that can overlap on the GPU, from any stream or thread, race on it
 *    and must be serialised by the caller.
 */
#define TV_STATIC_SCRATCH_BYTES (2u << 20)

TV_API tv_status tv_tree_attention_static(const tv_attn_desc *desc, const void *q, const void *paged_k,
                                          const void *paged_v, const int32_t *block_table,
                                          const int32_t *prefix_lens, const int32_t *parent_idx,
                                          void *out, int32_t *dev_status, void *stream);

/*
 * Acceptance walk problem.
 *   p, q         [batch][num_nodes][vocab] float32 probabilities:
 *                p[b][u] = target distribution after node u's path,
 *                q[b][u] = draft distribution node u's children were drawn from
 *   tree_tokens  [batch][num_nodes] int32 draft token of each node (the
 *                root's entry is ignored)
 *   parent_idx   [batch][num_nodes] int32 as for tv_tree_attention (NULL:
 *                chains)
 *   node_counts  (descriptor field) as for tv_tree_attention: children at or
 *                past n_b do not exist; n_b = 0 gives accepted_len 0, bonus
 *                -1 and an all -1 path (no tree this step)
 *   uniforms     [batch][num_nodes] float32 in [0,1): uniforms[b][c] (c >= 1)
 *                is node c's acceptance draw, uniforms[b][0] the bonus draw
 * Walk: from the root, children of the current node u are tried in
 * ascending index; child c with token x is accepted iff
 * uniforms[b][c] < P(x) / q[b][u][x], P being p[b][u] renormalised after
 * each rejected sibling to max(0, P - q[b][u]) / sum(max(0, P - q[b][u]))
 * (q(x) = 0 accepts iff P(x) > 0; a zero residual keeps P).  Acceptance
 * descends into c.  When no child is accepted (or u is a leaf) the bonus
 * token is the first index whose running sum of P exceeds
 * uniforms[b][0] * sum(P) (the last positive index if rounding leaves none).
 * Outputs:
 *   accepted_path [batch][num_nodes] int32: accepted node indices, root
 *                 excluded, in walk order, padded with -1
 *   accepted_len  [batch] int32, bonus_token [batch] int32
 * A malformed tree or token gives accepted_len = -1, bonus = -1 and
 * TV_ERR_TREE in *dev_status (a node count outside [0, num_nodes]:
 * TV_ERR_INVALID_ARG).
 */
typedef struct {
    int32_t batch;
    int32_t num_nodes;           /* 1..1024 */
    int32_t vocab;               /* 1..221184 (16 CTAs x 13824 entries) */
    const int32_t *node_counts;  /* device [batch] nodes per sequence, or NULL (= num_nodes each) */
} tv_sample_desc;

typedef struct {
    int32_t cluster_ctas;        /* CTAs cooperating on one sequence's rows */
    int32_t threads;             /* threads per CTA */
    int32_t slice;               /* vocabulary entries held per CTA */
    int32_t smem_bytes;          /* dynamic shared memory per CTA */
    int32_t launches;            /* kernel launches per call */
} tv_sample_plan;

TV_API tv_status tv_verify_sample_plan(const tv_sample_desc *desc, tv_sample_plan *plan);

TV_API size_t tv_verify_sample_workspace_size(const tv_sample_desc *desc);

TV_API tv_status tv_verify_sample(const tv_sample_desc *desc, const float *p, const float *q,
                           const int32_t *tree_tokens, const int32_t *parent_idx,
                           const float *uniforms, int32_t *accepted_path, int32_t *accepted_len,
                           int32_t *bonus_token, void *workspace, size_t workspace_bytes,
                           int32_t *dev_status, void *stream);

/*
 * The acceptance walk on the two models' logits instead of their
 * distributions (the fused-logits form of tv_verify_sample).  Blog
 * "Speculative decoding x tree attention", section 2, and glossary
 * "Tree-based speculative decoding", section "SpecInfer": p and q are the
 * target and draft models' output distributions, i.e. the row softmax of
 * their logits.
 *
 * Same descriptor, tree, uniforms, outputs, errors and stream behaviour as
 * tv_verify_sample; target_logits and draft_logits are fp32 [B][N][V] device
 * arrays (row u: the logits after node u's path), and p = softmax(target row),
 * q = softmax(draft row) at temperature 1.  Each row the walk visits is read
 * once and turned into its softmax in shared memory (row max, fp64 sum of
 * exp(l - max), both cluster-wide); p and q are never written to memory.  The
 * exponentials are fp32, so a decision can differ from an exact-arithmetic walk
 * only when its uniform lies within about 1e-6 of the threshold.  A logit of
 * -inf (a masked token) has probability 0; every row the walk visits needs at
 * least one finite logit (an all -inf row has no softmax and its result is
 * undefined).
 */
TV_API tv_status tv_verify_sample_logits(const tv_sample_desc *desc, const float *target_logits,
                                         const float *draft_logits, const int32_t *tree_tokens,
                                         const int32_t *parent_idx, const float *uniforms,
                                         int32_t *accepted_path, int32_t *accepted_len, int32_t *bonus_token,
                                         void *workspace, size_t workspace_bytes, int32_t *dev_status,
                                         void *stream);

/*
 * Commit the accepted path into the KV cache: the step after verification.
 * Blog "Speculative decoding x tree attention", section "KV cache management and
 * prefix sharing", and glossary "Tree-based speculative decoding", section "KV
 * cache management challenges": once the tree is verified, every tree entry off
 * the accepted path is dropped, which paged caches do through block-table
 * operations rather than by compacting memory.
 *
 * For each sequence b, tree node j sits at logical position prefix_lens[b] + j
 * (the layout tv_tree_attention reads).  With n = accepted_len[b] >= 0 and the
 * node indices accepted_path[b][0 .. n) (root excluded, strictly increasing, as
 * tv_verify_sample writes them), the K and V rows of node accepted_path[b][k]
 * move to position prefix_lens[b] + 1 + k for every KV head; the root stays at
 * prefix_lens[b]; new_prefix_lens[b] = prefix_lens[b] + 1 + n.  Positions from
 * the new length on hold nothing live: blocks wholly past it may be returned
 * to the caller's allocator (the block table is not changed).  accepted_len[b]
 * < 0 (a sequence the walk flagged) leaves the sequence unchanged.  With
 * desc->node_counts, the tree of sequence b has n_b nodes: path entries must
 * lie in [1, n_b), the span checked is L_b .. L_b + n_b - 1, and n_b = 0 with
 * accepted_len 0 commits nothing.
 *
 * Arguments: desc as for tv_tree_attention (batch, num_nodes, num_kv_heads,
 * head_dim, block_size 16, max_blocks_per_seq, num_blocks and dtype are used;
 * num_q_heads and softmax_scale are only validated).  paged_k / paged_v: device
 * caches [num_blocks][16][Hkv][D], 16-byte aligned, updated in place; the
 * blocks holding a sequence's tree span must belong to that sequence alone.
 * block_table [B][max_blocks_per_seq], prefix_lens [B], accepted_path [B][N],
 * accepted_len [B]: device int32, read.  new_prefix_lens [B]: device int32,
 * written; must not be prefix_lens (it is read while written).  dev_status: a
 * device int32 or NULL.  One launch on `stream`; no workspace; nothing is
 * allocated.
 * Errors: a bad descriptor, a null or misaligned pointer, or new_prefix_lens ==
 * prefix_lens return before launching.  A path that is not strictly increasing
 * inside [1, N), a length over N - 1, a prefix too long for the table, or a
 * block id out of range in the tree's span leaves that sequence unchanged
 * (new length = old) and writes TV_ERR_TREE, TV_ERR_INVALID_ARG or
 * TV_ERR_BLOCK_TABLE to *dev_status.
 */
TV_API tv_status tv_commit_path(const tv_attn_desc *desc, void *paged_k, void *paged_v,
                                const int32_t *block_table, const int32_t *prefix_lens,
                                const int32_t *accepted_path, const int32_t *accepted_len,
                                int32_t *new_prefix_lens, int32_t *dev_status, void *stream);

/*
 * Building the draft tree: top-k branching.  Glossary "Tree-based speculative
 * decoding", section on tree-structure optimisation, "Top-k branching": each
 * node expands the draft model's k most probable tokens as its children.
 *
 * For every node u of every sequence b that has children, child c receives the
 * rank[b][c]-th most probable token of q[b][u] (rank 0 = the most probable;
 * equal values rank the lower token id first; -0.0 ranks below +0.0):
 * tree_tokens[b][c] = that token id.  Only the rows of nodes with children are
 * read; the root's entry and padding entries of tree_tokens are not written.
 *   desc         batch, num_nodes (capacity, <= 1024), vocab, node_counts as for
 *                tv_verify_sample
 *   q            [batch][num_nodes][vocab] float32 device: u's draft
 *                distribution, or its logits (same order); no NaN
 *   parent_idx   [batch][num_nodes] int32 device, or NULL (chains)
 *   rank         [batch][num_nodes] int32 device, or NULL: then a child's rank is
 *                its position among its siblings in ascending node index
 *   tree_tokens  [batch][num_nodes] int32 device, written for children
 * A node may have at most 32 children and ranks lie in [0, 32) and below
 * vocab; otherwise that node's children get token -1.  A malformed tree (or a
 * bad node count) sets every child entry of the sequence to -1.  Both write
 * TV_ERR_TREE (TV_ERR_INVALID_ARG for a count) to *dev_status.  One launch on
 * `stream`; nothing is allocated.
 */
TV_API tv_status tv_tree_fill_topk(const tv_sample_desc *desc, const float *q, const int32_t *parent_idx,
                                   const int32_t *rank, int32_t *tree_tokens, int32_t *dev_status,
                                   void *stream);

/*
 * Building the draft tree: the budget-constrained shape.  Glossary, same
 * section, "Budget-constrained optimisation": under a node budget, allocate the
 * branches so that the whole tree's expected number of accepted tokens is
 * largest; dynamic programming solves it (as Sequoia does at run time).
 *
 * Model: accept[r] is the probability that a node's rank-r candidate is
 * accepted, the same at every depth (positional acceptance); a node's children
 * have ranks 0 .. m-1 with m <= num_ranks; a tree's value is the sum over its
 * non-root nodes of the product of accept[rank] along the root path (the
 * expected accepted tokens; one more token, the bonus, is always emitted).  The
 * call returns a tree of at most `budget` nodes (root included) and depth at
 * most max_depth (0 = no cap) with the largest value.  Ties go to the smaller
 * subtree sizes in rank order and then to the smaller tree.
 *   accept             num_ranks host doubles in [0, 1]
 *   parent_idx, rank   host int32 arrays of `budget` entries, written: nodes
 *                      numbered by depth, then by the ranks along their path
 *                      (parents before children, siblings in rank order, so
 *                      the output feeds tv_tree_fill_topk and the verifier);
 *                      root parent -1 and rank -1; entries past the tree -1
 *   num_nodes          host int32, written: the tree's size
 *   expected_accepted  host double, written: the tree's value
 * Host computation only (no device work): num_ranks <= 32, budget <= 256,
 * else TV_ERR_UNSUPPORTED; a null pointer, budget < 1, max_depth < 0 or an
 * accept value outside [0, 1]: TV_ERR_INVALID_ARG.
 */
TV_API tv_status tv_tree_shape(const double *accept, int32_t num_ranks, int32_t budget, int32_t max_depth,
                               int32_t *parent_idx, int32_t *rank, int32_t *num_nodes,
                               double *expected_accepted);

/*
 * Building the draft tree from several drafts: SpecInfer's token tree.
 * Glossary "Tree-based speculative decoding", section "SpecInfer": each draft
 * model (SSM) generates its own candidate sequence, and the sequences are
 * merged into one token tree in which candidates with a common prefix share
 * those nodes.
 *
 * Sequence k is tokens[seq_offsets[k] .. seq_offsets[k+1]) (token ids >= 0;
 * seq_offsets has num_seqs + 1 entries, starts at 0 and does not decrease).
 * Node 0 is the root (the last committed token: parent -1, token -1); walking
 * each sequence from the root in input order, every (node, token) pair not
 * seen before becomes the next node, so parents come before children and
 * siblings appear in the order the drafts proposed them (the order the walk
 * tries them).  Outputs (host int32): parent_idx and tree_tokens of max_nodes
 * entries (the rest -1), node_of_token[j] = the node of tokens[j], *num_nodes.
 * Host computation only.  Errors: null pointers, max_nodes < 1, bad offsets or
 * a negative token: TV_ERR_INVALID_ARG (nothing written); a tree larger than
 * max_nodes: TV_ERR_UNSUPPORTED (the outputs then hold a partial tree).
 */
TV_API tv_status tv_tree_merge(int32_t num_seqs, const int32_t *seq_offsets, const int32_t *tokens,
                               int32_t max_nodes, int32_t *parent_idx, int32_t *tree_tokens,
                               int32_t *node_of_token, int32_t *num_nodes);

/*
 * The tree size that pays.  LLM Primer VI ch. 9, 9.3: a step's speedup over
 * plain decoding is E[emitted tokens] / (T_draft/T_decode + 1 + alpha N), with
 * alpha the verification overhead per position (0.05-0.15) and N the draft
 * tokens, so an engine that fixes N misses the optimum; the glossary: Sequoia
 * sizes the tree for the hardware.
 *
 * For every budget n = 1 .. max_budget the best tree of tv_tree_shape (same
 * accept, num_ranks, max_depth) is scored by (1 + E) / (draft_cost + 1 +
 * alpha (size - 1)), E its expected accepted tokens (the 1 is the bonus
 * token), draft_cost = T_draft / T_decode; the call returns the tree with the
 * largest speedup (the smallest on ties) in the same format as tv_tree_shape,
 * with *speedup.  Arrays hold max_budget entries.  Host computation only;
 * errors as tv_tree_shape's, and draft_cost or alpha negative or not finite:
 * TV_ERR_INVALID_ARG.
 */
TV_API tv_status tv_tree_shape_for_cost(const double *accept, int32_t num_ranks, int32_t max_budget,
                                        int32_t max_depth, double draft_cost, double alpha,
                                        int32_t *parent_idx, int32_t *rank, int32_t *num_nodes,
                                        double *expected_accepted, double *speedup);

/*
 * Building the draft tree: the dynamic tree (EAGLE-2's dynamic draft-tree
 * expansion, LLM Primer VI ch. 9, 9.2: the target chooses among many draft
 * paths, not one guess), selected as the glossary's budget-constrained
 * optimisation (the whole tree's expected accepted tokens under a node budget)
 * with the draft's own probabilities as the acceptance estimate.
 *
 * Candidates 0 .. num_candidates-1 were grown by the caller (for example by
 * tv_tree_fill_topk level by level): cand_parent[c] < c is c's parent
 * candidate, or -1 for a child of the root; cand_token[c] its token;
 * cand_prob[c] in [0, 1] the draft probability of that token given its
 * parent's path.  A candidate's score is the product of cand_prob along its
 * path.  Candidates are taken by descending score, equal scores by lower
 * index, each only if its parent is already taken (with probabilities <= 1
 * this is the best-scoring ancestor-closed set), until the tree holds
 * `budget` nodes including the root.
 * Outputs (host arrays of `budget` entries, the rest set to -1): node 0 is
 * the root (parent -1, token -1, candidate -1); nodes 1.. are the taken
 * candidates in the order taken (so parents come first and siblings run from
 * the best score down, the order the walk tries them in): parent_idx,
 * tree_tokens (feed tv_tree_attention and tv_verify_sample; the root's token
 * is the caller's last committed token), cand_index (which candidate each
 * node is); *num_nodes; *expected_accepted = the sum of the taken scores.
 * Host computation only.  Errors: null outputs, budget < 1, a negative count
 * or a probability outside [0, 1]: TV_ERR_INVALID_ARG; candidates that are
 * not topological: TV_ERR_TREE; more than 2^20 candidates or a budget over
 * 1024: TV_ERR_UNSUPPORTED.
 */
TV_API tv_status tv_tree_select(const int32_t *cand_parent, const int32_t *cand_token, const double *cand_prob,
                                int32_t num_candidates, int32_t budget, int32_t *parent_idx,
                                int32_t *tree_tokens, int32_t *cand_index, int32_t *num_nodes,
                                double *expected_accepted);

/*
 * tv_tree_select for a whole batch, laid out for the ragged calls: sequence b's
 * candidates are entries cand_offsets[b] .. cand_offsets[b+1]-1 of the
 * candidate arrays (parent indices local to the sequence), and its tree goes
 * to row b of parent_idx, tree_tokens and cand_index ([batch][budget] host
 * int32), its size to node_counts[b] and its value to expected_accepted[b].
 * The outputs are the arrays tv_tree_attention, tv_verify_sample and
 * tv_commit_path take (num_nodes = budget, desc.node_counts = node_counts on
 * the device).  Every sequence is checked before anything is written; the
 * errors are tv_tree_select's, and cand_offsets must start at 0 and not
 * decrease (TV_ERR_INVALID_ARG).
 */
TV_API tv_status tv_tree_select_batch(int32_t batch, const int32_t *cand_offsets, const int32_t *cand_parent,
                                      const int32_t *cand_token, const double *cand_prob, int32_t budget,
                                      int32_t *parent_idx, int32_t *tree_tokens, int32_t *cand_index,
                                      int32_t *node_counts, double *expected_accepted);

/*
 * tv_tree_select_batch on the device: the same trees, bit for bit, from
 * candidate arrays that already sit in GPU memory (where the draft model
 * grew them), so the selection between drafting and verification needs no
 * round trip to the host.  Section and selection rule as tv_tree_select.
 *   cand_offsets  [batch + 1] int32: sequence b's candidates are entries
 *                 cand_offsets[b] .. cand_offsets[b+1]-1 of the candidate
 *                 arrays (at most max_candidates of them)
 *   cand_parent, cand_token  int32, cand_prob float32 in [0, 1], as for
 *                 tv_tree_select (parent indices local to the sequence)
 * Outputs (device): parent_idx, tree_tokens, cand_index [batch][budget]
 * int32 (-1 past the tree), node_counts [batch] int32, expected_accepted
 * [batch] float64 (the sum of the taken scores, scores formed in fp64 from
 * the fp32 probabilities).  One launch on `stream`, one CTA per sequence,
 * dynamic shared memory of 16 bytes per candidate slot plus 4 per budget
 * slot; no workspace.  Host-checked: batch >= 1, budget in [1, 1024],
 * max_candidates in [0, TV_SELECT_MAX_CANDIDATES], non-null arrays
 * (TV_ERR_INVALID_ARG / TV_ERR_UNSUPPORTED).  Device-checked, per sequence
 * (its node count becomes -1, its rows -1, the code goes to *dev_status):
 * candidates not topological (TV_ERR_TREE), a probability outside [0, 1] or
 * decreasing offsets (TV_ERR_INVALID_ARG), more than max_candidates
 * (TV_ERR_UNSUPPORTED).  Ranking is quadratic in the candidates of a sequence
 * (about a microsecond per thousand candidates squared over 512 threads).
 */
#define TV_SELECT_MAX_CANDIDATES 8192

TV_API tv_status tv_tree_select_device(int32_t batch, int32_t max_candidates, const int32_t *cand_offsets,
                                       const int32_t *cand_parent, const int32_t *cand_token,
                                       const float *cand_prob, int32_t budget, int32_t *parent_idx,
                                       int32_t *tree_tokens, int32_t *cand_index, int32_t *node_counts,
                                       double *expected_accepted, int32_t *dev_status, void *stream);

/* Static string for a status code. */
TV_API const char *tv_status_string(int32_t status);

/* Library version: major * 10000 + minor * 100 + patch. */
TV_API int32_t tv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TREEVERIFY_H */
