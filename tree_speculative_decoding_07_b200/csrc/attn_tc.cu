// attn_tc.cu -- tensor-core tree attention for bf16, head_dim 128 (sm_100a).
//
// Every draft-tree node attends to its sequence's cached prefix and to its own
// root path (glossary "Tree-based speculative decoding", section "Tree
// attention": M[i][j] = 1 iff node j is node i or an ancestor of i).
//
// Decomposition.  The G query heads that share a KV head, times the N tree
// nodes, form the query rows of one (sequence, KV head): row r is node r / G,
// head r % G.  A CTA owns one 128-row tile of those rows and one KV split;
// the splits of a tile form a thread-block cluster and merge their partial
// results through distributed shared memory at the end (flash-decoding
// log-sum-exp merge), so nothing goes through global scratch memory.
//
// Per 128-token KV tile (8 paged blocks of 16 tokens):
//   producer warp   TMA-loads the K and V rows of the 8 blocks (one 2 KB box
//                   per block and 64-column half, 128-byte swizzle) into a
//                   two-stage ring; block ids come from the block table.
//   MMA warp        S = Q K^T (tcgen05.mma kind::f16, M 128, N 128, K 16 x 8)
//                   into one of two TMEM S buffers, then O += P V into the
//                   TMEM accumulator once the softmax warps published P.
//   softmax warps   one thread per query row (TMEM lane): read the row of S,
//                   scale, apply the tree mask on the tree block, keep an
//                   online max / sum in the log2 domain (the O rescale in
//                   TMEM is skipped while the max grows by at most 2^8), write
//                   P as bf16 into shared memory in the MMA's swizzled layout.
// The tree mask is a 128-bit ancestor set per node, built from parent_idx in
// the prologue (anc(i) = anc(parent(i)) | {i}) and shifted into column space
// once per tile.
//
// Every wait on an mbarrier is bounded (about two seconds of clock); on expiry
// the CTA records TV_ERR_TIMEOUT, stops issuing work, writes NaN rows, frees
// its TMEM and still takes part in the cluster barriers so no peer is left
// waiting.
#include <cuda.h>
#include <cooperative_groups.h>

#include "tv_common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace tv {
namespace {

constexpr int TC_THREADS = 256;
constexpr int TM = 128;          // query rows per CTA (TMEM lanes)
constexpr int TN = 128;          // KV tokens per tile
constexpr int HD = 128;          // head dim
constexpr int BLK_PER_TILE = TN / TV_BLOCK;
constexpr int STAGES = 2;
constexpr int MAX_CLUSTER = 8;
constexpr uint32_t SQ_OFF = 0;           // Q: 2 x [128 rows][128 B], swizzled
constexpr uint32_t SP_OFF = 32768;       // P: 2 x [128 rows][128 B], swizzled
constexpr uint32_t SKV_OFF = 65536;      // stage s: K at +0 (32 KB), V at +32 KB
constexpr uint32_t STAGE_BYTES = 65536;
constexpr uint32_t HALF_BYTES = 16384;   // one 64-column half of a 128-row operand
constexpr uint32_t TILE_TX_BYTES = 2 * 2 * BLK_PER_TILE * 2048;  // K and V, 2 halves, 8 blocks
constexpr uint32_t SMEM_BYTES = SKV_OFF + STAGES * STAGE_BYTES + 1024;
constexpr int OPITCH = HD + 4;           // floats per row when staging partial outputs
constexpr uint32_t TMEM_COLS = 512;      // S0 [0,128), S1 [128,256), O [256,384)
constexpr uint32_t O_COL = 256;
constexpr long long WAIT_LIMIT = 1ll << 32;  // clock cycles (~2 s)

// instruction descriptor, kind::f16: D fp32, A/B bf16, A K-major,
// B K-major (S = Q K^T) or MN-major (O += P V), M = 128, N = 128
constexpr uint32_t IDESC_QK = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(TN >> 3) << 17) | ((uint32_t)(TM >> 4) << 24);
constexpr uint32_t IDESC_PV = IDESC_QK | (1u << 16);

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// shared-memory matrix descriptor, 128-byte swizzle, sm_100 version bits
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait on one phase.  Returns false once the CTA is aborting.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
    if (mbar_try(bar, parity)) return true;
    const long long t0 = clock64();
    for (;;) {
        if (mbar_try(bar, parity)) return true;
        if (*abort_flag) return false;
        if (clock64() - t0 > WAIT_LIMIT) {
            *abort_flag = 1;
            return false;
        }
    }
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1,
                                            int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], [%2];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void tmem_ld_x32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_st_x32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n"
                 :
                 : "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
                 : "memory");
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint32_t word_sel(uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, int i) {
    return i == 0 ? a0 : i == 1 ? a1 : i == 2 ? a2 : i == 3 ? a3 : 0u;
}

// Bits [32w, 32w + 32) of the 128-bit set a shifted left by s (s may be
// negative): result bit k is bit (32w + k - s) of a, zero outside [0, 128).
__device__ __forceinline__ uint32_t shifted_word(uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, int s, int w) {
    const int base = 32 * w - s;
    const int wi = base >> 5;  // floor division
    const int sh = base & 31;
    const uint32_t lo = word_sel(a0, a1, a2, a3, wi);
    const uint32_t hi = word_sel(a0, a1, a2, a3, wi + 1);
    return sh == 0 ? lo : __funnelshift_r(lo, hi, sh);
}

// mask of bit positions k in [0, 32) with 32w + k < n
__device__ __forceinline__ uint32_t below(int n, int w) {
    const int m = n - 32 * w;
    return m <= 0 ? 0u : m >= 32 ? 0xffffffffu : ((1u << m) - 1u);
}

// Warp-uniform bounded wait: every lane polls, the warp proceeds only if all saw the phase.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
    const bool ok = mbar_wait(bar, parity, abort_flag);
    return __all_sync(0xffffffffu, ok);
}

__global__ void __launch_bounds__(TC_THREADS, 1)
    attn_tc_kernel(const AttnArgs a, const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv) {
    extern __shared__ uint8_t dsmem[];
    __shared__ __align__(8) uint64_t bars[12];
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort, s_bad;
    __shared__ int32_t s_par[TV_MAX_NODES_ATTN];
    __shared__ float s_lse[TM];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int split = blockIdx.x, tile = blockIdx.y;
    const int b = blockIdx.z / a.Hkv, kvh = blockIdx.z % a.Hkv;
    const int N = a.N, G = a.G, S = a.splits;
    const uint32_t raw = smem_u32(dsmem);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* base_ptr = dsmem + (base - raw);
    const uint32_t sQ = base + SQ_OFF, sP = base + SP_OFF, sKV = base + SKV_OFF;
    const uint32_t bar0 = smem_u32(&bars[0]);
    auto kv_full = [&](int s) { return bar0 + 8u * (0 + s); };
    auto kv_empty = [&](int s) { return bar0 + 8u * (2 + s); };
    auto s_full = [&](int s) { return bar0 + 8u * (4 + s); };
    auto s_free = [&](int s) { return bar0 + 8u * (6 + s); };
    const uint32_t p_full = bar0 + 8u * 8, o_done = bar0 + 8u * 9, q_ready = bar0 + 8u * 10;
    const uint32_t mma_drain = bar0 + 8u * 11;
    volatile int* abort_flag = &s_abort;

    const int L = a.prefix_lens[b];
    const int total = L + N;

    // ---- prologue: tree check, barriers, TMEM
    if (tid == 0) {
        s_abort = 0;
        s_bad = (L < 0 || (total + TV_BLOCK - 1) / TV_BLOCK > a.max_blocks) ? TV_ERR_BLOCK_TABLE : 0;
    }
    for (int i = tid; i < N; i += TC_THREADS) s_par[i] = a.parent[(size_t)b * N + i];
    if (tid == 32) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(kv_full(s), 1);
            mbar_init(kv_empty(s), 1);
            mbar_init(s_full(s), 1);
            mbar_init(s_free(s), 128);
        }
        mbar_init(p_full, 128);
        mbar_init(o_done, 1);
        mbar_init(q_ready, 128);
        mbar_init(mma_drain, 1);
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
    for (int i = tid; i < N; i += TC_THREADS)
        if (!parent_ok(s_par, i)) s_bad = TV_ERR_TREE;
    tc_fence_after();
    __syncthreads();
    const uint32_t tmem = s_tmem;
    const bool bad0 = s_bad != 0;
    int t0, t1;
    split_range(total, S, split, t0, t1);
    if (bad0) t1 = t0;
    const int ntiles = (t1 - t0 + TN - 1) / TN;
    const int last_blk = (t1 - 1) / TV_BLOCK;

    if (warp == 0) {
        // ---------------- TMA producer
        const int32_t* bt = a.block_table + (size_t)b * a.max_blocks;
        auto fetch = [&](int j) {
            int id = 0;
            if (lane < BLK_PER_TILE) {
                int bi = (t0 + j * TN) / TV_BLOCK + lane;
                if (bi > last_blk) bi = last_blk;
                id = bt[bi];
                if (id < 0 || id >= a.num_blocks) {
                    s_bad = TV_ERR_BLOCK_TABLE;
                    id = 0;
                }
            }
            return id;
        };
        int ids = ntiles > 0 ? fetch(0) : 0;
        int issued = 0;
        for (int j = 0; j < ntiles; ++j) {
            const int stage = j & 1;
            if (j >= STAGES && !warp_wait(kv_empty(stage), ((j - STAGES) >> 1) & 1, abort_flag)) break;
            int cur[BLK_PER_TILE];
#pragma unroll
            for (int k = 0; k < BLK_PER_TILE; ++k) cur[k] = __shfl_sync(0xffffffffu, ids, k);
            if (lane == 0) {
                const uint32_t full = kv_full(stage);
                mbar_expect_tx(full, TILE_TX_BYTES);
                const uint32_t sK = sKV + stage * STAGE_BYTES, sV = sK + 32768u;
#pragma unroll
                for (int k = 0; k < BLK_PER_TILE; ++k) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        tma_load_4d(sK + h * HALF_BYTES + k * 2048u, &tmk, full, 0, kvh * 2 + h, 0, cur[k]);
                        tma_load_4d(sV + h * HALF_BYTES + k * 2048u, &tmv, full, 0, kvh * 2 + h, 0, cur[k]);
                    }
                }
            }
            ++issued;
            __syncwarp();
            if (j + 1 < ntiles) ids = fetch(j + 1);
        }
        if (*abort_flag) {
            // let copies already in flight land before the CTA retires
            for (int j = max(0, issued - STAGES); j < issued; ++j) {
                const long long t_0 = clock64();
                while (!mbar_try(kv_full(j & 1), (j >> 1) & 1) && clock64() - t_0 < (WAIT_LIMIT >> 4)) {
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (one thread)
        if (ntiles > 0 && lane == 0) {
            bool ok = mbar_wait(q_ready, 0, abort_flag);
            bool issued_any = false;
            for (int j = 0; ok && j <= ntiles; ++j) {
                if (j < ntiles) {
                    const int stage = j & 1, sb = j & 1;
                    ok = mbar_wait(kv_full(stage), (j >> 1) & 1, abort_flag);
                    if (ok && j >= 2) ok = mbar_wait(s_free(sb), ((j - 2) >> 1) & 1, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t sK = sKV + stage * STAGE_BYTES;
#pragma unroll
                    for (int k = 0; k < HD / 16; ++k) {
                        const uint32_t off = (k >> 2) * HALF_BYTES + (k & 3) * 32u;
                        mma_bf16(tmem + sb * TN, sdesc(sQ + off, 16, 1024), sdesc(sK + off, 16, 1024), IDESC_QK,
                                 k > 0 ? 1u : 0u);
                    }
                    mma_commit(s_full(sb));
                    issued_any = true;
                }
                if (j >= 1) {
                    const int t = j - 1, stage = t & 1;
                    ok = mbar_wait(p_full, t & 1, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t sV = sKV + stage * STAGE_BYTES + 32768u;
#pragma unroll
                    for (int k = 0; k < TN / 16; ++k) {
                        const uint32_t off = (k >> 2) * HALF_BYTES + (k & 3) * 32u;
                        mma_bf16(tmem + O_COL, sdesc(sP + off, 16, 1024), sdesc(sV + k * 2048u, HALF_BYTES, 1024),
                                 IDESC_PV, (t > 0 || k > 0) ? 1u : 0u);
                    }
                    mma_commit(o_done);
                    mma_commit(kv_empty(stage));
                }
            }
            if (issued_any) {
                // every MMA issued by this thread has finished before TMEM is released
                mma_commit(mma_drain);
                const long long t_0 = clock64();
                while (!mbar_try(mma_drain, 0) && clock64() - t_0 < WAIT_LIMIT) {
                }
            }
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ---------------- softmax: one thread per query row / TMEM lane
        const int r = tid - 128;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const int gr = tile * TM + r;
        const bool row_ok = gr < G * N;
        const int node = row_ok ? gr / G : 0;
        const int head = kvh * G + (row_ok ? gr % G : 0);
        uint32_t an0 = 0, an1 = 0, an2 = 0, an3 = 0;
        if (!bad0 && row_ok)
            for (int jn = node; jn >= 0; jn = s_par[jn]) {
                const uint32_t bit = 1u << (jn & 31);
                const int w = jn >> 5;
                an0 |= w == 0 ? bit : 0u;
                an1 |= w == 1 ? bit : 0u;
                an2 |= w == 2 ? bit : 0u;
                an3 |= w == 3 ? bit : 0u;
            }
        {
            const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.q) +
                                                              (((size_t)b * N + node) * a.Hq + head) * HD);
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const uint4 v = row_ok ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
                st_shared_v4(sQ + (c >> 3) * HALF_BYTES + r * 128 + (((c & 7) ^ (r & 7)) << 4), v);
            }
            fence_proxy_async();
            mbar_arrive(q_ready);
        }
        float m_run = -INFINITY, l_run = 0.f;
        const float sl = a.scale_log2;
        for (int j = 0; j < ntiles; ++j) {
            const int sb = j & 1, stage = j & 1;
            if (!warp_wait(s_full(sb), (j >> 1) & 1, abort_flag)) break;
            tc_fence_after();
            float x[TN];
#pragma unroll
            for (int c4 = 0; c4 < TN / 32; ++c4) {
                uint32_t rr[32];
                tmem_ld_x32(tmem + lane_base + sb * TN + c4 * 32, rr);
#pragma unroll
                for (int i = 0; i < 32; ++i) x[c4 * 32 + i] = __uint_as_float(rr[i]);
            }
            tc_fence_before();
            mbar_arrive(s_free(sb));
            const int tstart = t0 + j * TN;
            const int lim = t1 - tstart;  // columns >= lim lie past the split
            const int tree0 = L - tstart; // columns >= tree0 are tree nodes (node = column - tree0)
            float mt = -INFINITY;
            if (lim >= TN && tree0 >= TN) {
#pragma unroll
                for (int c = 0; c < TN; ++c) {
                    x[c] *= sl;
                    mt = fmaxf(mt, x[c]);
                }
            } else {
                uint32_t cm[4];
#pragma unroll
                for (int w = 0; w < 4; ++w)
                    cm[w] = (below(tree0, w) | shifted_word(an0, an1, an2, an3, tree0, w)) & below(lim, w);
#pragma unroll
                for (int c = 0; c < TN; ++c) {
                    const bool ok = (cm[c >> 5] >> (c & 31)) & 1u;
                    x[c] = ok ? x[c] * sl : -INFINITY;
                    mt = fmaxf(mt, x[c]);
                }
            }
            // the previous P V must be done: it frees P and settles O
            if (j > 0 && !warp_wait(o_done, (j - 1) & 1, abort_flag)) break;
            if (mt > m_run + 8.f) {
                if (m_run != -INFINITY) {
                    const float f = ex2(m_run - mt);
                    l_run *= f;
                    if (j > 0) {
                        tc_fence_after();
#pragma unroll
                        for (int c4 = 0; c4 < HD / 32; ++c4) {
                            uint32_t rr[32];
                            tmem_ld_x32(tmem + lane_base + O_COL + c4 * 32, rr);
#pragma unroll
                            for (int i = 0; i < 32; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * f);
                            tmem_st_x32(tmem + lane_base + O_COL + c4 * 32, rr);
                        }
                        tmem_wait_st();
                    }
                }
                m_run = mt;
            }
            const float mu = m_run == -INFINITY ? 0.f : m_run;
            float ls = 0.f;
#pragma unroll
            for (int cc = 0; cc < TN / 8; ++cc) {
                float p[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    p[e] = ex2(x[cc * 8 + e] - mu);
                    ls += p[e];
                }
                uint4 v;
                v.x = pack_bf16(p[0], p[1]);
                v.y = pack_bf16(p[2], p[3]);
                v.z = pack_bf16(p[4], p[5]);
                v.w = pack_bf16(p[6], p[7]);
                st_shared_v4(sP + (cc >> 3) * HALF_BYTES + r * 128 + (((cc & 7) ^ (r & 7)) << 4), v);
            }
            l_run += ls;
            if (lim < TN && r >= lim) {
                // value rows past the split end may hold stale data: clear them before P V
                mbar_wait(kv_full(stage), (j >> 1) & 1, abort_flag);
                const uint32_t sV = sKV + stage * STAGE_BYTES + 32768u;
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int c = 0; c < 8; ++c) st_shared_v4(sV + h * HALF_BYTES + r * 128 + c * 16, make_uint4(0, 0, 0, 0));
            }
            fence_proxy_async();
            tc_fence_before();
            mbar_arrive(p_full);
        }
        // ---- epilogue: normalise this CTA's partial output
        asm volatile("bar.sync 1, 128;" ::: "memory");
        bool fail = *abort_flag != 0;
        if (ntiles > 0 && !fail) fail = !warp_wait(o_done, (ntiles - 1) & 1, abort_flag);
        asm volatile("bar.sync 1, 128;" ::: "memory");
        // one decision per warp: tcgen05.ld below is warp-collective
        const bool bad = __any_sync(0xffffffffu, *abort_flag != 0 || s_bad != 0);
        tc_fence_after();
        const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
        const float lse = l_run > 0.f ? m_run + log2f(l_run) : -INFINITY;
        const bool have_o = ntiles > 0 && !bad;
        if (S == 1) {
            __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.out) + (((size_t)b * N + node) * a.Hq + head) * HD;
#pragma unroll
            for (int c4 = 0; c4 < HD / 32; ++c4) {
                uint32_t rr[32];
                if (have_o) {
                    tmem_ld_x32(tmem + lane_base + O_COL + c4 * 32, rr);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) rr[i] = 0u;
                }
                if (row_ok) {
#pragma unroll
                    for (int q8 = 0; q8 < 4; ++q8) {
                        float o[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) o[e] = bad ? NAN : __uint_as_float(rr[q8 * 8 + e]) * inv;
                        uint4 v;
                        v.x = pack_bf16(o[0], o[1]);
                        v.y = pack_bf16(o[2], o[3]);
                        v.z = pack_bf16(o[4], o[5]);
                        v.w = pack_bf16(o[6], o[7]);
                        reinterpret_cast<uint4*>(dst + c4 * 32)[q8] = v;
                    }
                }
            }
        } else {
            float* stage_o = reinterpret_cast<float*>(base_ptr + SKV_OFF);
#pragma unroll
            for (int c4 = 0; c4 < HD / 32; ++c4) {
                uint32_t rr[32];
                if (have_o) {
                    tmem_ld_x32(tmem + lane_base + O_COL + c4 * 32, rr);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) rr[i] = 0u;
                }
#pragma unroll
                for (int q4 = 0; q4 < 8; ++q4) {
                    float4 v;
                    v.x = __uint_as_float(rr[q4 * 4 + 0]) * inv;
                    v.y = __uint_as_float(rr[q4 * 4 + 1]) * inv;
                    v.z = __uint_as_float(rr[q4 * 4 + 2]) * inv;
                    v.w = __uint_as_float(rr[q4 * 4 + 3]) * inv;
                    *reinterpret_cast<float4*>(stage_o + r * OPITCH + c4 * 32 + q4 * 4) = v;
                }
            }
            s_lse[r] = bad ? NAN : lse;
        }
        tc_fence_before();
    }

    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
    }
    if (S > 1) {
        // ---- merge the splits of this row tile through distributed shared memory
        cg::cluster_group cluster = cg::this_cluster();
        cluster.sync();
        const float* stage_o = reinterpret_cast<const float*>(base_ptr + SKV_OFF);
        const int R = (TM + S - 1) / S;
        const int r0 = split * R;
        for (int item = tid; item < R * (HD / 4); item += TC_THREADS) {
            const int r = r0 + item / (HD / 4), c4 = item % (HD / 4);
            const int gr = tile * TM + r;
            if (r >= TM || gr >= G * N) continue;
            float mx = -INFINITY;
            bool nan = false;
            for (int s = 0; s < S; ++s) {
                const float l = *cluster.map_shared_rank(&s_lse[r], s);
                nan |= isnan(l);
                mx = fmaxf(mx, l);
            }
            float den = 0.f;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int s = 0; s < S; ++s) {
                const float l = *cluster.map_shared_rank(&s_lse[r], s);
                if (l == -INFINITY || nan) continue;
                const float w = ex2(l - mx);
                const float4 v = *reinterpret_cast<const float4*>(
                    cluster.map_shared_rank(stage_o + r * OPITCH + c4 * 4, s));
                den += w;
                acc.x = fmaf(w, v.x, acc.x);
                acc.y = fmaf(w, v.y, acc.y);
                acc.z = fmaf(w, v.z, acc.z);
                acc.w = fmaf(w, v.w, acc.w);
            }
            const bool dead = nan || den == 0.f;
            const float id = dead ? 0.f : 1.f / den;
            const int node = gr / G, head = kvh * G + gr % G;
            uint2 o;
            o.x = pack_bf16(dead ? NAN : acc.x * id, dead ? NAN : acc.y * id);
            o.y = pack_bf16(dead ? NAN : acc.z * id, dead ? NAN : acc.w * id);
            *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(a.out) + (((size_t)b * N + node) * a.Hq + head) * HD +
                                      c4 * 4) = o;
        }
        cluster.sync();  // peers may still read this CTA's shared memory until here
    }
    if (tid == 0) {
        if (s_bad) report(a.status, s_bad);
        if (s_abort) report(a.status, TV_ERR_TIMEOUT);
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        cudaGetLastError();
    }
    return fn;
}

// Paged cache [num_blocks][16][Hkv][128] bf16 seen as a 4-D tensor
// (64 columns, Hkv * 2 column halves, 16 slots, blocks); one box is the 16
// slots of one block for one half-head: 16 rows of 128 bytes.
bool make_kv_map(EncodeTiledFn fn, CUtensorMap* m, const void* ptr, int Hkv, int num_blocks) {
    const cuuint64_t dims[4] = {64, (cuuint64_t)(2 * Hkv), (cuuint64_t)TV_BLOCK, (cuuint64_t)num_blocks};
    const cuuint64_t strides[3] = {128, (cuuint64_t)Hkv * HD * 2, (cuuint64_t)TV_BLOCK * Hkv * HD * 2};
    const cuuint32_t box[4] = {64, 1, TV_BLOCK, 1};
    const cuuint32_t es[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

int tc_rows_per_tile() { return TM; }
int tc_max_cluster() { return MAX_CLUSTER; }

cudaError_t launch_attn_tc(const AttnArgs& a, cudaStream_t st, int* launches) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    if (a.D != HD || a.splits < 1 || a.splits > MAX_CLUSTER) return cudaErrorInvalidValue;
    CUtensorMap mk, mv;
    if (!make_kv_map(fn, &mk, a.k, a.Hkv, a.num_blocks) || !make_kv_map(fn, &mv, a.v, a.Hkv, a.num_blocks))
        return cudaErrorInvalidValue;
    static cudaError_t attr =
        cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (attr != cudaSuccess) return attr;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attrs[1];
    cfg.gridDim = dim3(a.splits, a.row_tiles, a.B * a.Hkv);
    cfg.blockDim = dim3(TC_THREADS, 1, 1);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = st;
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
