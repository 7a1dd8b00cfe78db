// treebuild.cu -- building the draft tree the verifier checks (glossary
// "Tree-based speculative decoding", section on tree-structure optimisation):
//
//  * top-k branching: each node expands the draft model's k most probable
//    tokens as its children.  fill_topk_kernel gives child c of node u the
//    rank(c)-th most probable token of u's draft distribution (ties to the
//    lower token id), reading only the rows of nodes that have children.
//  * budget-constrained optimisation: under a node budget, allocate branches so
//    the whole tree's expected accepted tokens is largest, by dynamic
//    programming (tree_shape_dp, host code: the table is small).
//
// fill_topk_kernel: one thread-block cluster per (sequence, node).  Each CTA of
// the cluster reads its slice of the node's row once, every thread keeping its
// own top K (K = kk rounded up to a power of two, kk = the largest child rank +
// 1) of 64-bit keys in registers (value bits mapped to an unsigned order in the
// high half, the complemented token id in the low half, so equal values rank
// the lower id first); kk block-wide rounds then pick the CTA's top kk, which
// go to the lead CTA's shared memory; the lead CTA merges the C * kk keys and
// writes the children's tokens.  Clusters of leaves leave after reading the
// tree.
#include <cooperative_groups.h>

#include <algorithm>
#include <unordered_map>
#include <vector>

#include "kernels.h"
#include "tv_common.cuh"

namespace cg = cooperative_groups;

namespace tv {
namespace {

constexpr int FT_THREADS = 256;
constexpr int FT_MAX_K = 32;        // largest child rank + 1
// at most 8 CTAs per row: 16-CTA clusters measured at 31 clusters in flight on
// the whole GPU, which left the 46 expanding rows of a 64-node tree two waves deep
constexpr int FT_MAX_CLUSTER = 8;

// float -> unsigned with the same order (negative values below positive ones)
__device__ __forceinline__ uint32_t ordered_bits(float v) {
    const uint32_t u = __float_as_uint(v);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ unsigned long long make_key(float v, int idx) {
    return ((unsigned long long)ordered_bits(v) << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)idx);
}

__device__ __forceinline__ int key_index(unsigned long long k) {
    return (int)(0xFFFFFFFFu - (uint32_t)(k & 0xFFFFFFFFull));
}

__device__ __forceinline__ unsigned long long warp_max_u64(unsigned long long v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        const unsigned long long w = __shfl_xor_sync(0xffffffffu, v, o);
        v = w > v ? w : v;
    }
    return v;
}

struct FillShared {
    int32_t parent[1024];
    int32_t kid[FT_MAX_K];                                   // children of the node, ascending
    int32_t kid_rank[FT_MAX_K];
    unsigned long long warp_best[FT_THREADS / 32];
    unsigned long long mine[FT_MAX_K];                       // this CTA's top kk
    unsigned long long all[FT_MAX_CLUSTER * FT_MAX_K];       // lead CTA: every CTA's top kk
    int nkids, kk;
    int bad;        // the whole sequence is malformed (count or tree): no child entry is valid
    int bad_node;   // this node's children cannot be expanded (too many, or a bad rank)
};

// Insert key into a descending list of K keys held in registers (the smallest
// falls off); keys that do not beat the last entry are skipped cheaply.
template <int K>
__device__ __forceinline__ void list_insert(unsigned long long (&L)[K], unsigned long long x, unsigned long long below) {
    if (x <= L[K - 1] || x >= below) return;
#pragma unroll
    for (int j = 0; j < K; ++j) {
        const unsigned long long hi = L[j] > x ? L[j] : x;
        x = L[j] > x ? x : L[j];
        L[j] = hi;
    }
}

// The CTA's next `take` keys (take <= K) below `below` among src[0, cnt) (token
// ids lo + i), into sh.mine[r0, r0 + take): one pass over global memory with a
// K-entry list per thread, then `take` rounds in which every thread offers its
// best remaining key and the block-wide winner drops it.  Keys of 0 mean "none"
// (the slice has fewer entries).
template <int K>
__device__ void slice_topk(const float* src, int cnt, int lo, bool vec4, int take, int r0, unsigned long long below,
                           FillShared& sh) {
    unsigned long long L[K];
#pragma unroll
    for (int j = 0; j < K; ++j) L[j] = 0ull;
    const int tid = threadIdx.x;
    if (vec4) {
        const float4* s4 = reinterpret_cast<const float4*>(src);
        const int n4 = cnt >> 2;
        int i = tid;
        for (; i + FT_THREADS < n4; i += 2 * FT_THREADS) {
            const float4 v0 = __ldg(s4 + i), v1 = __ldg(s4 + i + FT_THREADS);
            const int e0 = lo + 4 * i, e1 = e0 + 4 * FT_THREADS;
            list_insert<K>(L, make_key(v0.x, e0), below);
            list_insert<K>(L, make_key(v0.y, e0 + 1), below);
            list_insert<K>(L, make_key(v0.z, e0 + 2), below);
            list_insert<K>(L, make_key(v0.w, e0 + 3), below);
            list_insert<K>(L, make_key(v1.x, e1), below);
            list_insert<K>(L, make_key(v1.y, e1 + 1), below);
            list_insert<K>(L, make_key(v1.z, e1 + 2), below);
            list_insert<K>(L, make_key(v1.w, e1 + 3), below);
        }
        for (; i < n4; i += FT_THREADS) {
            const float4 v = __ldg(s4 + i);
            const int e = lo + 4 * i;
            list_insert<K>(L, make_key(v.x, e), below);
            list_insert<K>(L, make_key(v.y, e + 1), below);
            list_insert<K>(L, make_key(v.z, e + 2), below);
            list_insert<K>(L, make_key(v.w, e + 3), below);
        }
        for (int e = (cnt & ~3) + tid; e < cnt; e += FT_THREADS) list_insert<K>(L, make_key(__ldg(src + e), lo + e), below);
    } else {
        for (int e = tid; e < cnt; e += FT_THREADS) list_insert<K>(L, make_key(__ldg(src + e), lo + e), below);
    }
    const int warp = tid >> 5, lane = tid & 31;
    for (int r = 0; r < take; ++r) {
        const unsigned long long w = warp_max_u64(L[0]);
        if (lane == 0) sh.warp_best[warp] = w;
        __syncthreads();
        const unsigned long long best = warp_max_u64(lane < FT_THREADS / 32 ? sh.warp_best[lane] : 0ull);
        if (tid == 0) sh.mine[r0 + r] = best;
        if (best != 0ull && L[0] == best) {  // keys are unique: one thread drops its head
#pragma unroll
            for (int j = 0; j + 1 < K; ++j) L[j] = L[j + 1];
            L[K - 1] = 0ull;
        }
        __syncthreads();  // warp_best is reused for the next rank
    }
}

__global__ void __launch_bounds__(FT_THREADS) fill_topk_kernel(const FillArgs a) {
    __shared__ FillShared sh;
    cg::cluster_group cluster = cg::this_cluster();
    const int C = a.cluster;
    const int crank = C > 1 ? (int)cluster.block_rank() : 0;
    const int row = blockIdx.x / C;            // (sequence, node)
    const int b = row / a.N, u = row % a.N;
    const int tid = threadIdx.x;
    const int N = a.N;

    bool bad_count;
    const int n = seq_nodes(a.counts, b, N, bad_count);
    for (int i = tid; i < n; i += FT_THREADS) sh.parent[i] = parent_at(a.parent, b, N, i);
    if (tid == 0) {
        sh.nkids = 0;
        sh.bad = bad_count ? TV_ERR_INVALID_ARG : 0;
        sh.bad_node = 0;
    }
    __syncthreads();
    int bad_local = 0;
    for (int i = tid; i < n; i += FT_THREADS)
        if (!parent_ok(sh.parent, i)) bad_local = TV_ERR_TREE;
    if (bad_local) atomicMax(&sh.bad, bad_local);
    // children of u in ascending index, by one warp (ballots keep the order)
    if (tid < 32 && !bad_count && u < n) {
        int found = 0;
        for (int c0 = u + 1; c0 < n; c0 += 32) {
            const int c = c0 + tid;
            const bool kid = c < n && sh.parent[c] == u;
            const unsigned m = __ballot_sync(0xffffffffu, kid);
            const int pos = found + __popc(m & ((1u << tid) - 1u));
            if (kid && pos < FT_MAX_K) {
                sh.kid[pos] = c;
                sh.kid_rank[pos] = a.rank ? a.rank[(size_t)b * N + c] : pos;
            }
            found += __popc(m);
        }
        if (tid == 0) sh.nkids = found;
    }
    __syncthreads();
    const int nk = sh.nkids;
    if (tid == 0 && !sh.bad) {
        int kk = 0, err = nk > FT_MAX_K ? TV_ERR_TREE : 0;
        for (int j = 0; j < min(nk, FT_MAX_K); ++j) {
            const int r = sh.kid_rank[j];
            if (r < 0 || r >= FT_MAX_K || r >= a.V) err = TV_ERR_TREE;
            kk = max(kk, r + 1);
        }
        sh.kk = kk;
        sh.bad_node = err;
    }
    __syncthreads();
    if (sh.bad) {
        // a malformed sequence: every cluster of it sees the same, and the root's
        // cluster alone clears all of its child entries and reports
        if (u == 0 && crank == 0) {
            for (int c = 1 + tid; c < min(n, N); c += FT_THREADS) a.tokens[(size_t)b * N + c] = -1;
            if (tid == 0) report(a.status, sh.bad);
        }
        return;
    }
    if (sh.bad_node) {
        // this node's children (all of them, also past the first 32) get -1
        if (crank == 0) {
            for (int c = u + 1 + tid; c < n; c += FT_THREADS)
                if (sh.parent[c] == u) a.tokens[(size_t)b * N + c] = -1;
            if (tid == 0) report(a.status, sh.bad_node);
        }
        return;
    }
    if (u >= n || nk == 0) return;  // no such node, or a leaf: nothing to expand (cluster-uniform)
    const int kk = sh.kk;

    // ---- the top kk keys of this CTA's slice of u's draft row, read once
    {
        const int lo = min(a.V, crank * a.slice);
        const int cnt = min(a.V, lo + a.slice) - lo;
        const float* src = a.q + ((size_t)b * N + u) * (size_t)a.V + lo;
        const bool v4 = a.vec4 != 0;
        if (kk <= 1) {
            slice_topk<1>(src, cnt, lo, v4, kk, 0, ~0ull, sh);
        } else if (kk <= 2) {
            slice_topk<2>(src, cnt, lo, v4, kk, 0, ~0ull, sh);
        } else if (kk <= 4) {
            slice_topk<4>(src, cnt, lo, v4, kk, 0, ~0ull, sh);
        } else {
            // eight ranks per pass over the slice (more than eight children is rare)
            unsigned long long below = ~0ull;
            for (int r0 = 0; r0 < kk; r0 += 8) {
                const int take = min(8, kk - r0);
                slice_topk<8>(src, cnt, lo, v4, take, r0, below, sh);
                below = sh.mine[r0 + take - 1];
                if (below == 0ull) {  // the slice ran out: the remaining ranks are empty
                    for (int r = r0 + take + threadIdx.x; r < kk; r += FT_THREADS) sh.mine[r] = 0ull;
                    __syncthreads();
                    break;
                }
            }
        }
    }
    // ---- gather every CTA's keys in the lead CTA
    if (C > 1) {
        cluster.sync();  // every CTA of the cluster is running before shared memory is shared
        unsigned long long* dst = cluster.map_shared_rank(sh.all, 0);
        for (int r = tid; r < kk; r += FT_THREADS) dst[crank * FT_MAX_K + r] = sh.mine[r];
        cluster.sync();  // the stores are visible to the lead CTA
        if (crank != 0) return;
    } else {
        for (int r = tid; r < kk; r += FT_THREADS) sh.all[r] = sh.mine[r];
        __syncthreads();
    }
    // ---- lead CTA: merge C * kk keys, rank by rank, and write the children's tokens
    if (tid < 32) {
        unsigned long long prev = ~0ull;
        const int total = C * FT_MAX_K;
        for (int r = 0; r < kk; ++r) {
            unsigned long long best = 0ull;
            for (int i = tid; i < total; i += 32) {
                const int cr = i / FT_MAX_K, j = i % FT_MAX_K;
                if (j >= kk || cr >= C) continue;
                const unsigned long long k = sh.all[i];
                if (k < prev && k > best) best = k;
            }
            best = warp_max_u64(best);
            if (tid == 0) sh.mine[r] = best;
            prev = best;
        }
        __syncwarp();
        for (int j = tid; j < nk; j += 32) {
            const unsigned long long k = sh.mine[sh.kid_rank[j]];
            a.tokens[(size_t)b * N + sh.kid[j]] = k ? key_index(k) : -1;
        }
    }
}

}  // namespace

void fill_topk_plan(int V, int* cluster, int* slice, int* smem_bytes) {
    int c = (V + 16383) / 16384;
    if (c > FT_MAX_CLUSTER) c = FT_MAX_CLUSTER;
    if (c < 1) c = 1;
    int s = (V + c - 1) / c;
    s = (s + 3) / 4 * 4;
    *cluster = c;
    *slice = s;
    *smem_bytes = 0;  // the slice is scanned straight from global memory
}

cudaError_t launch_fill_topk(const FillArgs& a, cudaStream_t st) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    cfg.gridDim = dim3((unsigned)a.cluster * (unsigned)a.B * (unsigned)a.N, 1, 1);
    cfg.blockDim = dim3(FT_THREADS, 1, 1);
    cfg.dynamicSmemBytes = a.smem_bytes;
    cfg.stream = st;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = a.cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = a.cluster > 1 ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, fill_topk_kernel, a);
}

// ---------------------------------------------------------------- budget DP

// F[d][n]: best expected accepted tokens of a subtree of exactly n nodes with at
// most d levels below its root; G[i][s]: best value of the children of ranks
// i.. holding s nodes in all:  G[i][s] = max_t accept[i] (1 + F[d-1][t]) +
// G[i+1][s-t], F[d][n] = G[0][n-1].  Ties go to the smallest t, and among equal
// totals to the smallest tree.  Nodes are numbered by depth, then by the ranks
// along their path.
namespace {

struct ShapeTable {
    int budget, D;
    std::vector<std::vector<double>> F;        // F[d][n]
    std::vector<std::vector<int32_t>> choice;  // choice[d][i * budget + s] = t
};

void shape_table(const double* accept, int k, int budget, int D, ShapeTable& T) {
    const double NEG = -INFINITY;
    T.budget = budget;
    T.D = D;
    T.F.assign(D + 1, std::vector<double>(budget + 1, NEG));
    T.choice.assign(D + 1, std::vector<int32_t>());
    std::vector<double> G((size_t)(k + 1) * budget);
    for (int d = 0; d <= D; ++d) {
        T.F[d][1] = 0.0;
        if (d == 0) continue;
        std::vector<int32_t>& ch = T.choice[d];
        ch.assign((size_t)(k + 1) * budget, 0);
        std::fill(G.begin(), G.end(), NEG);
        G[(size_t)k * budget + 0] = 0.0;
        for (int i = k - 1; i >= 0; --i) {
            double* gi = &G[(size_t)i * budget];
            const double* gn = &G[(size_t)(i + 1) * budget];
            gi[0] = 0.0;
            for (int s = 1; s < budget; ++s) {
                double best = NEG;
                int arg = 0;
                for (int t = 1; t <= s; ++t) {
                    const double f = T.F[d - 1][t], g = gn[s - t];
                    if (f == NEG || g == NEG) continue;
                    const double grow = 1.0 + f;
                    const double take = accept[i] * grow;
                    const double v = take + g;
                    if (v > best) {
                        best = v;
                        arg = t;
                    }
                }
                gi[s] = best;
                ch[(size_t)i * budget + s] = arg;
            }
        }
        for (int nn = 2; nn <= budget; ++nn) T.F[d][nn] = G[nn - 1];
    }
}

bool path_less(const std::vector<int>& x, const std::vector<int>& y) {
    if (x.size() != y.size()) return x.size() < y.size();
    return x < y;
}

// The n-node tree of the table, numbered by depth, then by the ranks along the path.
int shape_rebuild(const ShapeTable& T, int n_nodes, int32_t* parent, int32_t* rank) {
    std::vector<std::vector<int>> paths;
    struct Item { std::vector<int> path; int d, n; };
    std::vector<Item> stack{{{}, T.D, n_nodes}};
    while (!stack.empty()) {
        Item it = stack.back();
        stack.pop_back();
        paths.push_back(it.path);
        int s = it.n - 1, i = 0;
        while (s > 0) {
            const int t = T.choice[it.d][(size_t)i * T.budget + s];
            std::vector<int> p = it.path;
            p.push_back(i);
            stack.push_back({p, it.d - 1, t});
            s -= t;
            ++i;
        }
    }
    std::sort(paths.begin(), paths.end(), path_less);
    const int n = (int)paths.size();
    for (int j = 0; j < T.budget; ++j) {
        parent[j] = -1;
        rank[j] = -1;
    }
    for (int j = 1; j < n; ++j) {
        std::vector<int> up(paths[j].begin(), paths[j].end() - 1);
        // the parent's path is shorter, so it sits before j in the sorted list
        parent[j] = (int)(std::lower_bound(paths.begin(), paths.begin() + j, up, path_less) - paths.begin());
        rank[j] = paths[j].back();
    }
    return n;
}

int depth_levels(int budget, int max_depth) {
    return (max_depth <= 0 || max_depth > budget - 1) ? budget - 1 : max_depth;
}

}  // namespace

int tree_shape_dp(const double* accept, int k, int budget, int max_depth, int32_t* parent, int32_t* rank,
                  double* value) {
    ShapeTable T;
    shape_table(accept, k, budget, depth_levels(budget, max_depth), T);
    int n_best = 1;
    for (int nn = 2; nn <= budget; ++nn)
        if (T.F[T.D][nn] > T.F[T.D][n_best]) n_best = nn;
    *value = T.F[T.D][n_best];
    return shape_rebuild(T, n_best, parent, rank);
}

// The size whose best tree gives the largest step speedup
// (1 + E) / (draft_cost + 1 + alpha (n - 1)); the smallest such size on ties.
int tree_shape_for_cost(const double* accept, int k, int max_budget, int max_depth, double draft_cost, double alpha,
                        int32_t* parent, int32_t* rank, double* value, double* speedup) {
    ShapeTable T;
    shape_table(accept, k, max_budget, depth_levels(max_budget, max_depth), T);
    int n_best = 1;
    double best = -INFINITY;
    for (int nn = 1; nn <= max_budget; ++nn) {
        const double f = T.F[T.D][nn];
        if (f == -INFINITY) continue;
        const double gain = 1.0 + f;
        const double cost = draft_cost + 1.0 + alpha * (double)(nn - 1);
        const double sp = gain / cost;
        if (sp > best) {
            best = sp;
            n_best = nn;
        }
    }
    *value = T.F[T.D][n_best];
    *speedup = best;
    return shape_rebuild(T, n_best, parent, rank);
}

// ---------------------------------------------------------------- token-tree merge

// Sequences k = 0.. (tokens[offsets[k] .. offsets[k+1])) merge into one tree:
// node 0 is the root; walking a sequence from the root, each (node, token)
// pair not seen before becomes a new node, so common prefixes share nodes and
// nodes appear in input order.  Returns the node count, or -1 when it would
// exceed max_nodes (nothing past max_nodes is written).
int tree_merge(int num_seqs, const int32_t* offsets, const int32_t* tokens, int max_nodes, int32_t* parent_idx,
               int32_t* tree_tokens, int32_t* node_of) {
    std::unordered_map<uint64_t, int32_t> child;
    parent_idx[0] = -1;
    tree_tokens[0] = -1;
    int n = 1;
    for (int k = 0; k < num_seqs; ++k) {
        int32_t u = 0;
        for (int32_t j = offsets[k]; j < offsets[k + 1]; ++j) {
            const uint64_t key = ((uint64_t)(uint32_t)u << 32) | (uint32_t)tokens[j];
            auto it = child.find(key);
            if (it == child.end()) {
                if (n >= max_nodes) return -1;
                parent_idx[n] = u;
                tree_tokens[n] = tokens[j];
                it = child.emplace(key, n).first;
                ++n;
            }
            u = it->second;
            node_of[j] = u;
        }
    }
    for (int j = n; j < max_nodes; ++j) {
        parent_idx[j] = -1;
        tree_tokens[j] = -1;
    }
    return n;
}

// ---------------------------------------------------------------- dynamic selection

// Candidates 0..M-1 are topological (parent < index, -1 = a child of the root);
// score = product of prob along the path.  Take candidates by descending score,
// equal scores by lower index, each only if its parent is already taken, until
// the tree holds `budget` nodes with the root.  Returns the node count, or -1
// when the candidates are not topological.
int tree_select(const int32_t* cand_parent, const int32_t* cand_token, const double* cand_prob, int M, int budget,
                int32_t* parent_idx, int32_t* tree_tokens, int32_t* cand_index, double* value) {
    std::vector<double> score(M);
    for (int c = 0; c < M; ++c) {
        const int p = cand_parent[c];
        if (p < -1 || p >= c) return -1;
        const double up = p >= 0 ? score[p] : 1.0;
        score[c] = up * cand_prob[c];
    }
    std::vector<int> order(M);
    for (int c = 0; c < M; ++c) order[c] = c;
    std::sort(order.begin(), order.end(), [&](int x, int y) {
        if (score[x] != score[y]) return score[x] > score[y];
        return x < y;
    });
    std::vector<int> node_of(M, -1);
    for (int j = 0; j < budget; ++j) {
        parent_idx[j] = -1;
        tree_tokens[j] = -1;
        cand_index[j] = -1;
    }
    int n = 1;
    double total = 0.0;
    for (int k = 0; k < M && n < budget; ++k) {
        const int c = order[k];
        const int p = cand_parent[c];
        if (p >= 0 && node_of[p] < 0) continue;
        node_of[c] = n;
        parent_idx[n] = p >= 0 ? node_of[p] : 0;
        tree_tokens[n] = cand_token[c];
        cand_index[n] = c;
        ++n;
    }
    for (int j = 1; j < n; ++j) total += score[cand_index[j]];
    *value = total;
    return n;
}

}  // namespace tv
