// attn_tc.cu -- tensor-core tree attention for bf16, head_dim 128 (sm_100a).
//
// Every draft-tree node attends to its sequence's cached prefix and to its own
// root path (glossary "Tree-based speculative decoding", section "Tree
// attention": M[i][j] = 1 iff node j is node i or an ancestor of i).
//
// Decomposition.  The G query heads that share a KV head, times the N tree
// nodes, form the query rows of one (sequence, KV head): row r is node r / G,
// head r % G, so each K/V row is read once for all G heads.  A CTA owns one
// 128-row tile of those rows and one KV split: a fixed range of logical
// blocks of the block table (known at launch, so the block ids are fetched
// before the sequence's length arrives).  The S splits of a row tile form one
// thread-block cluster; when all have finished their tokens, each stages its
// normalised partial rows (bf16) and their log-sum-exp in its idle V ring, and
// after a cluster barrier each CTA reads the rows it owns (an equal share per
// CTA) from every CTA's staging in place (distributed shared memory) and
// combines them (flash-decoding log-sum-exp merge).  No global workspace is used.
//
// Warp roles (384 threads):
//   warp 0      TMA producer of K tiles, warp 3 of V tiles: the rows of 8 paged
//               blocks per 128-token tile (one 2 KB box per block and 64-column
//               half, 128-byte swizzle) into 3-deep K and V rings.  Block ids
//               reach them through a shared-memory ring filled by cp.async
//               several tiles ahead.  In a split of few tiles the V copies
//               wait for the first V tile, so they do not compete with the K
//               tiles the first score tiles need.
//   warp 1      S = Q K^T issuer: tcgen05.mma kind::f16, M 128, N 128, 8 x K16,
//               into the TMEM S buffer, reused as soon as both softmax groups
//               have read the previous tile's scores into registers.  Q is
//               staged in TMEM by the softmax threads (one row each), so the
//               MMA takes it from there (the TMEM-A form) and reads only the
//               K tile from shared memory: with both operands in shared memory
//               each of these MMAs took ~86 cycles against ~68 for the P V
//               MMAs, which read one.
//   warp 2      O_x += P_x V issuer (one per softmax group, over that group's 64
//               tokens), and owner of the TMEM allocation (all 512 columns:
//               S, P, Q, O_A, O_B).  The two issuers sit on different SM
//               sub-partitions.
//   warps 4-7   softmax group A: columns 0..63 of every S tile
//   warps 8-11  softmax group B: columns 64..127
// Each softmax thread owns one query row (its TMEM lane).  The two groups
// keep separate running maxima / sums and separate O accumulators, merged at
// the end like two splits.  (Making the two warps that share an SM
// sub-partition take turns at the exponentials, through named barriers,
// measured 4 % slower on the l8b step.)  Scores are scaled into the log2
// domain by the same FFMA that subtracts the running max; the O rescale in
// TMEM is skipped while the max grows by at most 2^8.  P is written as bf16 pairs into a TMEM P buffer of its
// own, once this group's P V of the previous tile has read it, and P V takes it
// from there (the TMEM-A form of the MMA); since P does not overwrite the
// scores, S = Q K^T of tile j + 1 runs while the softmax of tile j is still
// computing.  The tree mask is a 128-bit ancestor set per node (anc(i) =
// anc(parent(i)) | {i}), shifted into column space once per tile; prefix-only
// tiles skip it.
//
// Every mbarrier wait is bounded (about two seconds of clock); on expiry the
// CTA records TV_ERR_TIMEOUT, stops issuing work, drains its copies and MMAs,
// frees its TMEM, and still takes part in the merge with NaN rows, so every CTA
// of the cluster reaches the merge's two cluster barriers.
#include <mutex>

#include "tc_device.cuh"

namespace tv {
namespace {

constexpr int TC_THREADS = 384;
constexpr int HALF_N = TN / 2;   // tokens per softmax group
constexpr int KST = 3;           // K ring depth
constexpr int VST = 3;           // V ring depth
constexpr int SHORT_SPLIT_TILES = 8;  // splits of at most this many tiles hold their V ring at first
constexpr uint32_t SK_OFF = 0;             // K ring: KST x 32 KB
constexpr uint32_t SV_OFF = SK_OFF + KST * 32768u;  // V ring: VST x 32 KB
constexpr uint32_t SMEM_BYTES = SV_OFF + VST * 32768u + 1024;
constexpr uint32_t TMEM_COLS = 512;        // S [0,128), P [128,192), Q [192,256), O_A [256,384), O_B [384,512)
constexpr uint32_t P_COL = 128;            // P: 64 columns of bf16 pairs, group x at x * 32
constexpr uint32_t Q_COL = 192;            // Q: 64 columns of bf16 pairs (dims 2c, 2c + 1 in column c)
constexpr uint32_t O_COL = 256;

// mbarrier slots, derived from the ring depths
constexpr int BAR_K_FULL = 0;                    // KST: K tile landed (TMA transaction count)
constexpr int BAR_K_EMPTY = BAR_K_FULL + KST;    // KST: S = Q K^T done with the K slot
constexpr int BAR_V_FULL = BAR_K_EMPTY + KST;    // VST: V tile landed
constexpr int BAR_V_EMPTY = BAR_V_FULL + VST;    // VST: P V done with the V slot
constexpr int BAR_S_FULL = BAR_V_EMPTY + VST;    // S of the next tile written
constexpr int BAR_S_FREE = BAR_S_FULL + 1;       // both groups have read S (256 arrivals)
constexpr int BAR_P_FULL = BAR_S_FREE + 1;       // 2: group's P written (and O rescaled)
constexpr int BAR_O_DONE = BAR_P_FULL + 2;       // 2: group's P V done
constexpr int BAR_Q_READY = BAR_O_DONE + 2;      // Q staged
constexpr int BAR_DRAIN_QK = BAR_Q_READY + 1;    // all S = Q K^T MMAs done
constexpr int BAR_DRAIN_PV = BAR_DRAIN_QK + 1;   // all P V MMAs done
constexpr int BAR_COUNT = BAR_DRAIN_PV + 1;
static_assert(BAR_COUNT == 2 * KST + 2 * VST + 9, "barrier slots overlap");
static_assert(TM * PROW_BYTES <= VST * TILE_BYTES, "staged partial rows exceed the V ring");

__global__ void __launch_bounds__(TC_THREADS, 1)
    attn_tc_kernel(const __grid_constant__ AttnArgs a, const __grid_constant__ CUtensorMap tmk,
                   const __grid_constant__ CUtensorMap tmv) {
    extern __shared__ uint8_t dsmem[];
    __shared__ __align__(8) uint64_t bars[BAR_COUNT];
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort, s_bad;
    __shared__ int32_t s_par[TV_MAX_NODES_ATTN];
    __shared__ __align__(16) int32_t s_ids[2][ID_RING * BLK_PER_TILE];  // block ids, per producer

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int split = blockIdx.x, tile = blockIdx.y;
    const int b = blockIdx.z / a.Hkv, kvh = blockIdx.z % a.Hkv;
    const int N = a.N, G = a.G, S = a.splits;
    // the prefix length and the sequence's node count decide where the tokens end:
    // both loads are issued before any set-up
    const int L = a.prefix_lens[b];
    bool bad_count;
    const int n = seq_nodes(a.counts, b, N, bad_count);
    // row tiles past a short tree have no rows; every split of such a tile (the
    // whole cluster) leaves here, so no merge waits on it
    if (!bad_count && tile * TM >= G * n) return;
    const uint32_t raw = smem_u32(dsmem);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* base_ptr = dsmem + (base - raw);
    auto sK = [&](int s) { return base + SK_OFF + (uint32_t)s * TILE_BYTES; };
    auto sV = [&](int s) { return base + SV_OFF + (uint32_t)s * TILE_BYTES; };
    const uint32_t bar0 = smem_u32(&bars[0]);
    auto k_full = [&](int s) { return bar0 + 8u * (BAR_K_FULL + s); };
    auto k_empty = [&](int s) { return bar0 + 8u * (BAR_K_EMPTY + s); };
    auto v_full = [&](int s) { return bar0 + 8u * (BAR_V_FULL + s); };
    auto v_empty = [&](int s) { return bar0 + 8u * (BAR_V_EMPTY + s); };
    const uint32_t s_full = bar0 + 8u * BAR_S_FULL, s_free = bar0 + 8u * BAR_S_FREE;
    auto p_full = [&](int x) { return bar0 + 8u * (BAR_P_FULL + x); };
    auto o_done = [&](int x) { return bar0 + 8u * (BAR_O_DONE + x); };
    const uint32_t q_ready = bar0 + 8u * BAR_Q_READY;
    const uint32_t drain_qk = bar0 + 8u * BAR_DRAIN_QK, drain_pv = bar0 + 8u * BAR_DRAIN_PV;
    volatile int* abort_flag = &s_abort;
    // results of the softmax groups, consumed by the split merge after the role blocks
    uint32_t pk[32];   // this thread's 64 outputs of its row, as bf16 pairs
    float lse = -INFINITY;
    const int X = warp >= 4 ? (warp - 4) >> 2 : 0;          // softmax group: tokens X*64 .. X*64+63 of a tile
    const int r = ((warp & 3) << 5) + lane;                  // query row in the tile (softmax warps)

    // ---- prologue
    // The softmax threads request their row's 64 query values and one parent index
    // first of all, so these global-memory latencies overlap the set-up below and the
    // block-id loads instead of following them (Q goes to TMEM after the barrier).
    const int gr = tile * TM + r;
    const bool row_ok = warp >= 4 && gr < G * n;
    const int node = row_ok ? gr / G : 0;
    const int head = kvh * G + (row_ok ? gr % G : 0);
    uint32_t qw[32];
    {
        const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.q) +
                                                          (((size_t)b * N + node) * a.Hq + head) * HD + X * 64);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const uint4 v = row_ok ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
            qw[4 * c] = v.x;
            qw[4 * c + 1] = v.y;
            qw[4 * c + 2] = v.z;
            qw[4 * c + 3] = v.w;
        }
    }
    const int32_t par_i = (warp >= 4 && tid - 128 < n) ? parent_at(a.parent, b, N, tid - 128) : 0;
    // The producer warps request the tensor maps and their first block ids before
    // anything else (a thread that also initialised the barriers issued them only after
    // its cluster-scope fence); warp 1, idle until the barrier below, initialises the
    // barriers, and warp 2 allocates TMEM.
    if ((warp == 0 || warp == 3) && lane == 0) prefetch_tensormap(warp == 0 ? &tmk : &tmv);
    // This split's logical blocks are [blk0, blk_end) of the block table, fixed at
    // launch, so their ids are fetched without waiting for the prefix length.
    // They reach the producers through a shared-memory ring that cp.async fills
    // ID_AHEAD tiles ahead of use, so no tile's copies wait on a block-table load
    // (a register loaded one tile earlier would stall every iteration for one
    // global-memory latency).  The first copies start before the barrier,
    // overlapping barrier set-up and TMEM allocation.
    const int blk0 = min(a.max_blocks, split * a.blocks_per_split);
    const int blk_end = min(a.max_blocks, blk0 + a.blocks_per_split);
    const int32_t* bt = a.block_table + (size_t)b * a.max_blocks;
    const int prod = warp == 0 ? 0 : 1;
    auto prefetch_ids = [&](int jt) {
        const int bi = blk0 + jt * BLK_PER_TILE + lane;
        if (lane < BLK_PER_TILE && bi < blk_end)
            cp_async_4(smem_u32(&s_ids[prod][(jt % ID_RING) * BLK_PER_TILE + lane]), bt + bi);
        cp_async_commit();  // one group per tile on every lane, empty or not
    };
    if (warp == 0 || warp == 3)
        for (int jt = 0; jt < ID_AHEAD; ++jt) prefetch_ids(jt);
    if (tid == 32) {
        s_abort = 0;
        s_bad = 0;
        for (int s = 0; s < KST; ++s) {
            mbar_init(k_full(s), 1);
            mbar_init(k_empty(s), 1);
        }
        for (int s = 0; s < VST; ++s) {
            mbar_init(v_full(s), 1);
            mbar_init(v_empty(s), 1);
        }
        mbar_init(s_full, 1);
        mbar_init(s_free, 256);
        for (int x = 0; x < 2; ++x) {
            mbar_init(p_full(x), 128);
            mbar_init(o_done(x), 1);
        }
        mbar_init(q_ready, 256);
        mbar_init(drain_qk, 1);
        mbar_init(drain_pv, 1);
        fence_barrier_init();
    }
    if (warp == 2) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        tc_fence_before();
    }
    __syncthreads();
    // a kernel launched after this one with programmatic stream serialisation may
    // start its set-up now; it waits for this grid before reading anything
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    // the split's tokens: [t0, t1) of the sequence's L + n
    const int total = L + n;
    const bool bad_len = L < 0 || (total + TV_BLOCK - 1) / TV_BLOCK > a.max_blocks;
    const int t0 = blk0 * TV_BLOCK;
    const int t1 = max(t0, min(blk_end * TV_BLOCK, bad_len ? 0 : total));
    const int ntiles = (t1 - t0 + TN - 1) / TN;
    const int used_blk = (t1 + TV_BLOCK - 1) / TV_BLOCK;  // blocks holding this split's tokens end here

    if (warp == 0 || warp == 3) {
        // ---------------- TMA producers: warp 0 streams K tiles, warp 3 V tiles
        const bool is_k = warp == 0;
        const CUtensorMap* map = is_k ? &tmk : &tmv;
        const int depth = is_k ? KST : VST;
        int issued = 0;
        bool bad_id = false;
        for (int j = 0; j < ntiles; ++j) {
            const int s = j % depth;
            if (j >= depth && !warp_wait(is_k ? k_empty(s) : v_empty(s), ((j - depth) / depth) & 1, abort_flag)) break;
            // this lane's id copies for tile j are complete; the warp barrier makes
            // every lane's copies visible to lane 0
            cp_async_wait<ID_AHEAD - 1>();
            __syncwarp();
            if (lane == 0) {
                // blocks of the tile that hold tokens of the split (the last tile may
                // hold fewer than 8); the others repeat its last block, whose rows past the
                // split are masked (K) and zeroed (V) like any rows past the split (a copy
                // of all 8 blocks with a constant byte count measured faster than
                // issuing only the ones in range)
                const int nb = min(BLK_PER_TILE, used_blk - (blk0 + j * BLK_PER_TILE));
                int cur[BLK_PER_TILE];
                const int32_t* ring = &s_ids[prod][(j % ID_RING) * BLK_PER_TILE];
#pragma unroll
                for (int k = 0; k < BLK_PER_TILE; ++k) {
                    int id = ring[k < nb ? k : nb - 1];
                    if (id < 0 || id >= a.num_blocks) {
                        bad_id = true;
                        id = 0;
                    }
                    cur[k] = id;
                }
                const uint32_t full = is_k ? k_full(s) : v_full(s);
                const uint32_t dst = is_k ? sK(s) : sV(s);
                mbar_expect_tx(full, TILE_BYTES);
#pragma unroll
                for (int k = 0; k < BLK_PER_TILE; ++k)
#pragma unroll
                    for (int h = 0; h < 2; ++h)
                        tma_load_4d(dst + h * HALF_BYTES + k * 2048u, map, full, 0, kvh * 2 + h, 0, cur[k]);
            }
            __syncwarp();
            // the slot refilled here last held tile j + ID_AHEAD - ID_RING, read before
            prefetch_ids(j + ID_AHEAD);
            ++issued;
            // A split of a few tiles is bound by its first tiles' latency: its V copies wait
            // until the first V tile has landed, so they do not queue beside the K tiles the
            // first S = Q K^T tiles need (l8b with L2 flushed: 23.0 us against 24.6 with
            // both rings held after their first tile, and 24.1 with neither).  A long split
            // streams both rings from the start (2-3 % faster on l70b and long).
            if (j == 0 && !is_k && ntiles > 1 && ntiles <= SHORT_SPLIT_TILES &&
                !warp_wait(v_full(0), 0, abort_flag))
                break;
        }
        asm volatile("cp.async.wait_all;" ::: "memory");  // no id copy lands after the ring is abandoned
        if (bad_id) s_bad = TV_ERR_BLOCK_TABLE;
        if (*abort_flag && lane == 0) {
            // let copies already in flight land before the CTA retires
            for (int j = max(0, issued - depth); j < issued; ++j) {
                const long long c0 = clock64();
                const uint32_t full = is_k ? k_full(j % depth) : v_full(j % depth);
                while (!mbar_try(full, (j / depth) & 1) && clock64() - c0 < (WAIT_LIMIT >> 4)) {
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- S = Q K^T issuer (one thread).  The two MMA streams are issued
        // from warps on different SM sub-partitions: a thread issuing tcgen05.mma shares
        // its sub-partition's issue slots with two softmax warps, and one thread issuing
        // all sixteen MMAs of a tile was slower than the tile's softmax.
        if (ntiles > 0 && lane == 0) {
            bool ok = mbar_wait(q_ready, 0, abort_flag);
            bool issued_any = false;
            // descriptors of the tiles' first 16-column step; the other steps add a
            // constant to the address field (addresses stay below 2^18 bytes)
            const uint64_t dk0 = sdesc(sK(0), 16, 1024);
            for (int j = 0; ok && j < ntiles; ++j) {
                const int ks = j % KST;
                // the S buffer is free once both groups have read tile j - 1's scores (they
                // cannot read tile j's before this commit, so the phases stay in step)
                if (j >= 1) ok = mbar_wait(s_free, (j - 1) & 1, abort_flag);
                if (ok) ok = mbar_wait(k_full(ks), (j / KST) & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint64_t dk = dk0 + (uint64_t)((ks * TILE_BYTES) >> 4);
#pragma unroll
                for (int k = 0; k < HD / 16; ++k) {
                    const uint32_t off = ((k >> 2) * HALF_BYTES + (k & 3) * 32u) >> 4;
                    mma_bf16_ts(tmem, tmem + Q_COL + k * 8, dk + off, IDESC_QK, k > 0 ? 1u : 0u);
                }
                mma_commit(s_full);
                mma_commit(k_empty(ks));
                issued_any = true;
            }
            if (issued_any) {
                // every MMA issued by this thread has finished before TMEM is released
                mma_commit(drain_qk);
                const long long c0 = clock64();
                while (!mbar_try(drain_qk, 0) && clock64() - c0 < WAIT_LIMIT) {
                }
            }
        }
        __syncwarp();
    } else if (warp == 2) {
        // ---------------- O += P V issuer (one thread)
        if (ntiles > 0 && lane == 0) {
            bool ok = true, issued_any = false;
            const uint64_t dv0 = sdesc(sV(0), HALF_BYTES, 1024);
            for (int t = 0; ok && t < ntiles; ++t) {
                const int vs = t % VST;
                ok = mbar_wait(v_full(vs), (t / VST) & 1, abort_flag);
                const uint64_t dv = dv0 + (uint64_t)((vs * TILE_BYTES) >> 4);
                for (int x = 0; ok && x < 2; ++x) {
                    ok = mbar_wait(p_full(x), t & 1, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int k = 0; k < HALF_N / 16; ++k)
                        mma_bf16_ts(tmem + O_COL + x * HD, tmem + P_COL + x * 32 + k * 8,
                                    dv + (uint64_t)(((x * 4 + k) * 2048u) >> 4), IDESC_PV, (t > 0 || k > 0) ? 1u : 0u);
                    mma_commit(o_done(x));
                    issued_any = true;
                }
                if (!ok) break;
                mma_commit(v_empty(vs));
            }
            if (issued_any) {
                mma_commit(drain_pv);
                const long long c0 = clock64();
                while (!mbar_try(drain_pv, 0) && clock64() - c0 < WAIT_LIMIT) {
                }
            }
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ---------------- softmax groups: one thread per query row / TMEM lane
        const int st = tid - 128;  // 0..255
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        if (st < n) s_par[st] = par_i;  // n <= TV_MAX_NODES_ATTN < 256
        asm volatile("bar.sync 1, 256;" ::: "memory");
        for (int i = st; i < n; i += 256)
            if (!parent_ok(s_par, i)) s_bad = TV_ERR_TREE;
        if (st == 0 && bad_len) s_bad = TV_ERR_BLOCK_TABLE;
        if (st == 0 && bad_count) s_bad = TV_ERR_INVALID_ARG;
        uint32_t an0 = 0, an1 = 0, an2 = 0, an3 = 0;
        if (row_ok && !a.parent) {
            // a chain: node i's ancestors are nodes 0..i (the causal tail), no walk needed
            an0 = below(node + 1, 0);
            an1 = below(node + 1, 1);
            an2 = below(node + 1, 2);
            an3 = below(node + 1, 3);
        } else if (row_ok) {
            int steps = 0;
            for (int jn = node; jn >= 0 && jn < N && steps <= N; jn = s_par[jn], ++steps) {
                const uint32_t bit = 1u << (jn & 31);
                const int w = jn >> 5;
                an0 |= w == 0 ? bit : 0u;
                an1 |= w == 1 ? bit : 0u;
                an2 |= w == 2 ? bit : 0u;
                an3 |= w == 3 ? bit : 0u;
            }
        }
        {
            tmem_st_x32(tmem + lane_base + Q_COL + X * 32, qw);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(q_ready);
        }
        float m_run = -INFINITY, l_run = 0.f;  // running max in the scaled log2 domain, running sum
        const float sl = a.scale_log2;
        bool live = true;  // warp-uniform: every wait of this warp so far succeeded
        for (int j = 0; j < ntiles; ++j) {
            live = live && warp_wait(s_full, j & 1, abort_flag);
            float x[HALF_N];
            const int tstart = t0 + j * TN;
            const int lim = t1 - tstart;   // tile columns >= lim lie past the split
            const int tree0 = L - tstart;  // tile columns >= tree0 are tree nodes
            // after a failed wait the loads, exponentials and stores below still run (on
            // whatever the buffers hold; the CTA's output is NaN then), only the waits and
            // hand-offs to other roles are skipped
            tc_fence_after();
#pragma unroll
            for (int c32 = 0; c32 < HALF_N / 32; ++c32) {
                uint32_t rr[32];
                tmem_ld_x32(tmem + lane_base + X * HALF_N + c32 * 32, rr);
#pragma unroll
                for (int i = 0; i < 32; ++i) x[c32 * 32 + i] = __uint_as_float(rr[i]);
            }
            // the scores are in registers (the loads waited): the next tile's S = Q K^T may
            // overwrite the buffer
            tc_fence_before();
            if (live) mbar_arrive(s_free);
            if (lim < TN || tree0 < TN) {
                uint32_t cm[2];
#pragma unroll
                for (int w = 0; w < 2; ++w)
                    cm[w] = (below(tree0, 2 * X + w) | shifted_word(an0, an1, an2, an3, tree0, 2 * X + w)) &
                            below(lim, 2 * X + w);
#pragma unroll
                for (int i = 0; i < HALF_N; ++i)
                    if (!((cm[i >> 5] >> (i & 31)) & 1u)) x[i] = -INFINITY;
            }
            const float mt = max_tree(x) * sl;
            float f = 1.f;
            if (mt > m_run + 8.f) {  // grow the reference max (also the first finite tile)
                if (m_run != -INFINITY) f = ex2(m_run - mt);
                m_run = mt;
            }
            const float mu = m_run == -INFINITY ? 0.f : m_run;
            // one P buffer: this group's P V of the previous tile has read it before it is
            // overwritten (the same wait also frees O for the rescale below)
            if (j > 0 && live) live = warp_wait(o_done(X), (j - 1) & 1, abort_flag);
            // exponentials, packed as bf16 pairs (token 2i in the low half of column i), into
            // this group's 32 columns of P buffer j % 2; P V of tile j - 2, which read them,
            // finished before this group released P of tile j - 1 (the o_done wait below)
            float s4[4] = {0.f, 0.f, 0.f, 0.f};
            {
                uint32_t pp[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float e0 = ex2(fmaf(x[2 * i], sl, -mu));
                    const float e1 = ex2(fmaf(x[2 * i + 1], sl, -mu));
                    s4[(2 * i) & 3] += e0;
                    s4[(2 * i + 1) & 3] += e1;
                    pp[i] = pack_bf16(e0, e1);
                }
                tmem_st_x32(tmem + lane_base + P_COL + X * 32, pp);
            }
            if (!live) continue;
            l_run = l_run * f + ((s4[0] + s4[1]) + (s4[2] + s4[3]));
            if (lim < TN) {
                // value rows past the split end repeat another block or hold data
                // past the sequence: clear this group's ones
                const int tok = X * HALF_N + (r & 63);
                if (tok >= lim) {
                    const int vs = j % VST;
                    mbar_wait(v_full(vs), (j / VST) & 1, abort_flag);
                    const uint32_t row = sV(vs) + (r >> 6) * HALF_BYTES + tok * 128;
#pragma unroll
                    for (int c = 0; c < 8; ++c) st_shared_v4(row + c * 16, make_uint4(0, 0, 0, 0));
                }
                fence_proxy_async();
            }
            // this group's previous P V must be complete before O is rescaled and
            // before P V of this tile is released (every phase is waited, in order)
            if (!live) continue;
            // tcgen05.ld / st are warp-collective (.sync.aligned): the whole warp rescales
            // when any of its rows needs it (rows whose max did not move multiply by 1)
            if (j > 0 && __any_sync(0xffffffffu, f != 1.f)) {
                tc_fence_after();
#pragma unroll
                for (int c4 = 0; c4 < HD / 32; ++c4) {
                    uint32_t rr[32];
                    tmem_ld_x32(tmem + lane_base + O_COL + X * HD + c4 * 32, rr);
#pragma unroll
                    for (int i = 0; i < 32; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * f);
                    tmem_st_x32(tmem + lane_base + O_COL + X * HD + c4 * 32, rr);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(p_full(X));
        }
        // ---- epilogue: merge the two groups' halves into this CTA's partial output
        asm volatile("bar.sync 1, 256;" ::: "memory");
        bool fail = __any_sync(0xffffffffu, *abort_flag != 0);
        if (ntiles > 0 && !fail) fail = !warp_wait(o_done(X), (ntiles - 1) & 1, abort_flag);
        // per-row (max, sum) of each group, exchanged through the first K slot: every
        // K copy was consumed by an S = Q K^T that finished before the loops ended
        float* pm = reinterpret_cast<float*>(base_ptr + SK_OFF);
        auto s_m = [&](int g) { return pm + g * (HALF_BYTES / 4); };
        auto s_l = [&](int g) { return pm + g * (HALF_BYTES / 4) + TM; };
        s_m(X)[r] = m_run;
        s_l(X)[r] = l_run;
        asm volatile("bar.sync 1, 256;" ::: "memory");
        const bool bad = __any_sync(0xffffffffu, *abort_flag != 0 || s_bad != 0);
        const float mA = s_m(0)[r], mB = s_m(1)[r];
        const float m = fmaxf(mA, mB);
        const float wA = mA == -INFINITY ? 0.f : ex2(mA - m);
        const float wB = mB == -INFINITY ? 0.f : ex2(mB - m);
        const float l = wA * s_l(0)[r] + wB * s_l(1)[r];
        const float inv = l > 0.f ? 1.f / l : 0.f;
        lse = bad ? NAN : (l > 0.f ? m + log2f(l) : -INFINITY);
        const bool have_o = ntiles > 0 && !bad;
        tc_fence_after();
#pragma unroll
        for (int c32 = 0; c32 < 2; ++c32) {
            uint32_t ra[32], rb[32];
            if (have_o) {
                tmem_ld_x32(tmem + lane_base + O_COL + X * 64 + c32 * 32, ra);
                tmem_ld_x32(tmem + lane_base + O_COL + HD + X * 64 + c32 * 32, rb);
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float o0 = have_o ? (wA * __uint_as_float(ra[2 * i]) + wB * __uint_as_float(rb[2 * i])) * inv
                                        : (bad ? NAN : 0.f);
                const float o1 = have_o ? (wA * __uint_as_float(ra[2 * i + 1]) + wB * __uint_as_float(rb[2 * i + 1])) *
                                              inv
                                        : (bad ? NAN : 0.f);
                pk[c32 * 16 + i] = pack_bf16(o0, o1);
            }
        }
        tc_fence_before();
        if (S == 1 && row_ok) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) +
                                                  (((size_t)b * N + node) * a.Hq + head) * HD + X * 64);
#pragma unroll
            for (int q8 = 0; q8 < 8; ++q8)
                dst[q8] = make_uint4(pk[4 * q8], pk[4 * q8 + 1], pk[4 * q8 + 2], pk[4 * q8 + 3]);
        } else if (S > 1) {
            // stage this row's partial in the V ring (every P V has finished: both groups
            // waited for their last one before the barrier above): row r at r * PROW_BYTES,
            // group X's 64 outputs at byte X * 128, the log-sum-exp at byte 256
            const uint32_t row = base + SV_OFF + (uint32_t)r * PROW_BYTES;
#pragma unroll
            for (int q8 = 0; q8 < 8; ++q8)
                st_shared_v4(row + X * HD + q8 * 16, make_uint4(pk[4 * q8], pk[4 * q8 + 1], pk[4 * q8 + 2], pk[4 * q8 + 3]));
            if (X == 0) st_shared_v4(row + 2 * HD, make_uint4(__float_as_uint(lse), 0u, 0u, 0u));
        }
    }

    __syncthreads();  // every role finished; all TMEM reads completed; the rings are idle
    if (warp == 2) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
    }
    if (S > 1) {
        // ---- merge the KV splits of this row tile through the cluster's shared memory.
        // Rows [k R, k R + R) belong to CTA k (split k).  Every CTA has staged its 128
        // partial rows in its V ring; after one cluster barrier (release / acquire) each
        // CTA reads its rows from every CTA's staging in place and combines them, and a
        // second one keeps every CTA resident until all have read its rows.  (Copying the
        // rows to their owners first, once every owner reported its ring idle, took ~2.3 us
        // after the last split arrived on l8b, against ~1 us for this.)
        const int R = (TM + S - 1) / S;
        const uint32_t stage = base + SV_OFF;
        asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
        asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
        switch (S) {
            case 2: merge_rows<TM, TC_THREADS, 2>(a, stage, R, split, tile, b, kvh, tid, G * n); break;
            case 3: merge_rows<TM, TC_THREADS, 3>(a, stage, R, split, tile, b, kvh, tid, G * n); break;
            case 4: merge_rows<TM, TC_THREADS, 4>(a, stage, R, split, tile, b, kvh, tid, G * n); break;
            case 5: merge_rows<TM, TC_THREADS, 5>(a, stage, R, split, tile, b, kvh, tid, G * n); break;
            case 6: merge_rows<TM, TC_THREADS, 6>(a, stage, R, split, tile, b, kvh, tid, G * n); break;
            case 7: merge_rows<TM, TC_THREADS, 7>(a, stage, R, split, tile, b, kvh, tid, G * n); break;
            case 8: merge_rows<TM, TC_THREADS, 8>(a, stage, R, split, tile, b, kvh, tid, G * n); break;
            case 9: merge_rows<TM, TC_THREADS, 9>(a, stage, R, split, tile, b, kvh, tid, G * n); break;
            case 10: merge_rows<TM, TC_THREADS, 10>(a, stage, R, split, tile, b, kvh, tid, G * n); break;
            case 11: merge_rows<TM, TC_THREADS, 11>(a, stage, R, split, tile, b, kvh, tid, G * n); break;
            case 12: merge_rows<TM, TC_THREADS, 12>(a, stage, R, split, tile, b, kvh, tid, G * n); break;
            case 13: merge_rows<TM, TC_THREADS, 13>(a, stage, R, split, tile, b, kvh, tid, G * n); break;
            case 14: merge_rows<TM, TC_THREADS, 14>(a, stage, R, split, tile, b, kvh, tid, G * n); break;
            case 15: merge_rows<TM, TC_THREADS, 15>(a, stage, R, split, tile, b, kvh, tid, G * n); break;
            default: merge_rows<TM, TC_THREADS, 16>(a, stage, R, split, tile, b, kvh, tid, G * n); break;
        }
        asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
        asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
    }
    if (tid == 0) {
        if (s_bad) report(a.status, s_bad);
        if (s_abort) report(a.status, TV_ERR_TIMEOUT);
    }
}

// Per-device launch facts, looked up once per device with that device current:
// whether the kernel's shared-memory and cluster-size attributes are set, and
// how many clusters of each split count the device holds at once.
struct TcDeviceInfo {
    int state = 0;                    // 0 unknown, 1 ready, -1 unusable
    int clusters[MAX_SPLITS + 1] = {};  // [s]: clusters of s CTAs resident at once (s = 1: CTAs)
};
constexpr int MAX_DEVICES = 64;
std::mutex g_info_mutex;
TcDeviceInfo g_info[MAX_DEVICES];

const TcDeviceInfo* tc_device_info() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) {
        cudaGetLastError();
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(g_info_mutex);
    TcDeviceInfo& d = g_info[dev];
    if (d.state == 0) {
        d.state = -1;
        if (cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES) ==
                cudaSuccess &&
            cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess) {
            d.state = 1;
            int per_sm = 0, sms = 0;
            if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
                cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, attn_tc_kernel, TC_THREADS, SMEM_BYTES) ==
                    cudaSuccess)
                d.clusters[1] = per_sm * sms;
            for (int s = 2; s <= MAX_SPLITS; ++s) {
                cudaLaunchConfig_t cfg = {};
                cudaLaunchAttribute attr[1];
                cfg.gridDim = dim3(s, 1, 1);
                cfg.blockDim = dim3(TC_THREADS, 1, 1);
                cfg.dynamicSmemBytes = SMEM_BYTES;
                attr[0].id = cudaLaunchAttributeClusterDimension;
                attr[0].val.clusterDim.x = s;
                attr[0].val.clusterDim.y = 1;
                attr[0].val.clusterDim.z = 1;
                cfg.attrs = attr;
                cfg.numAttrs = 1;
                int c = 0;
                if (cudaOccupancyMaxActiveClusters(&c, attn_tc_kernel, &cfg) != cudaSuccess) c = 0;
                d.clusters[s] = c;
            }
        }
        cudaGetLastError();
    }
    return &d;
}

}  // namespace

int tc_rows_per_tile() { return TM; }
int tc_max_splits() { return MAX_SPLITS; }

// KV splits per row tile (the splits of a tile form one cluster).  Splitting
// pays only while the grid fills less than half of the GPU.  Among 2..16
// splits (at least 256 tokens each) take the one with the fewest tiles on the
// longest path: waves of clusters the device holds at once, times the tiles
// of one split.  Without a device (host-only planning) every SM is assumed to
// hold one CTA and a cluster of s CTAs to need s SMs.
int tc_pick_splits(int64_t groups, int64_t max_blocks, int sms) {
    const TcDeviceInfo* info = tc_device_info();
    const bool known = info && info->state == 1 && info->clusters[1] > 0;
    const int64_t cap = known ? info->clusters[1] : sms;
    if (groups * 2 > cap) return 1;
    const int64_t tiles1 = (max_blocks + BLK_PER_TILE - 1) / BLK_PER_TILE;
    int best = 1;
    int64_t best_cost = tiles1 * ((groups + cap - 1) / cap);
    for (int s = 2; s <= MAX_SPLITS; ++s) {
        if (max_blocks < (int64_t)s * 16) break;  // at least 256 tokens per split
        const int64_t per_wave = known ? info->clusters[s] : sms / s;
        if (per_wave <= 0) continue;
        const int64_t bps = (max_blocks + s - 1) / s;
        const int64_t cost = ((groups + per_wave - 1) / per_wave) * ((bps + BLK_PER_TILE - 1) / BLK_PER_TILE);
        if (cost < best_cost) {
            best_cost = cost;
            best = s;
        }
    }
    return best;
}

cudaError_t launch_attn_tc(const AttnArgs& a, cudaStream_t st, int* launches) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    if (a.D != HD || a.splits < 1 || a.splits > MAX_SPLITS || a.blocks_per_split < 1) return cudaErrorInvalidValue;
    CUtensorMap mk, mv;
    if (!make_kv_map(fn, &mk, a.k, a.Hkv, a.num_blocks) || !make_kv_map(fn, &mv, a.v, a.Hkv, a.num_blocks))
        return cudaErrorInvalidValue;
    const TcDeviceInfo* info = tc_device_info();
    if (!info || info->state != 1) return cudaErrorInvalidDeviceFunction;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attrs[1];
    cfg.gridDim = dim3(a.splits, a.row_tiles, a.B * a.Hkv);
    cfg.blockDim = dim3(TC_THREADS, 1, 1);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = st;
    // the splits of a row tile merge through each other's shared memory: one cluster
    attrs[0].id = cudaLaunchAttributeClusterDimension;
    attrs[0].val.clusterDim.x = a.splits;
    attrs[0].val.clusterDim.y = 1;
    attrs[0].val.clusterDim.z = 1;
    cfg.attrs = attrs;
    cfg.numAttrs = a.splits > 1 ? 1 : 0;
    *launches = 1;
    return cudaLaunchKernelEx(&cfg, attn_tc_kernel, a, mk, mv);
}

}  // namespace tv
