// tc_device.cuh -- pieces shared by the tensor-core attention kernels for
// sm_100a: mbarrier waits, TMA and cp.async copies, tcgen05 MMA and TMEM
// access, the tree-mask words, the split merge, and the host-side tensor map
// over the paged KV cache.
#pragma once

#include <cuda.h>

#include "tv_common.cuh"
#include "kernels.h"

namespace tv {
namespace {

constexpr int TM = 128;          // query rows per Q tile (TMEM lanes)
constexpr int TN = 128;          // KV tokens per tile
constexpr int HD = 128;          // head dim
constexpr int BLK_PER_TILE = TN / TV_BLOCK;
constexpr int MAX_SPLITS = 16;
constexpr int ID_RING = 8;       // tiles of block ids held per producer
constexpr int ID_AHEAD = 6;      // tiles between an id copy's issue and its use
constexpr uint32_t TILE_BYTES = 32768;     // one K or V tile: 2 halves x 128 rows x 128 B
constexpr uint32_t HALF_BYTES = 16384;
// one split's partial row in the workspace: 128 normalised outputs as bf16, the
// row's log-sum-exp as fp32 at byte 256, padding to a 16-byte multiple
constexpr int PROW_BYTES = 272;
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

// 4-byte asynchronous global -> shared copy (no register holds the value)
__device__ __forceinline__ void cp_async_4(uint32_t dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
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
// D (TMEM) += A (TMEM, bf16 pairs per 32-bit column) * B (shared memory descriptor)
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n"
        ::"r"(d_tmem), "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
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

// address of the same shared-memory location in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
// loads from another CTA's shared memory (a shared::cluster address from mapa)
__device__ __forceinline__ uint4 ld_cluster_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared::cluster.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}
__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
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

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
// Combine this CTA's share of one ROWS-row tile, rows [split * R, split * R + own),
// from the S partials (rows of PROW_BYTES: 128 bf16 outputs, then the fp32
// log-sum-exp): out = sum_s 2^(lse_s - m) o_s / sum_s 2^(lse_s - m), m = max_s lse_s.
// Each item is 8 columns of one row, so a thread issues all its loads at once; `stage` is
// the shared-memory address at which every CTA of the cluster staged its partial rows
// (row r at r * PROW_BYTES), read in place from each CTA (distributed shared memory).
template <int ROWS, int THREADS, int S_>
__device__ __forceinline__ void merge_rows(const AttnArgs& a, uint32_t stage, int R, int split, int tile, int b,
                                           int kvh, int tid, int nrows) {
    constexpr int NC = HD / 8;
    const int own = max(0, min(ROWS, (split + 1) * R) - split * R);
    for (int item = tid; item < own * NC; item += THREADS) {
        const int rr = item / NC, cc = item % NC;
        const int gr = tile * ROWS + split * R + rr;
        if (gr >= nrows) continue;  // rows of nodes past the sequence's tree
        float ls[S_];
        uint4 v[S_];
#pragma unroll
        for (int k = 0; k < S_; ++k) {
            const uint32_t prow = mapa_shared(stage + (uint32_t)(split * R + rr) * PROW_BYTES, (uint32_t)k);
            ls[k] = ld_cluster_f32(prow + 2 * HD);
            v[k] = ld_cluster_v4(prow + 16u * cc);
        }
        float mx = -INFINITY;
        bool nan = false;
#pragma unroll
        for (int k = 0; k < S_; ++k) {
            nan |= isnan(ls[k]);
            mx = fmaxf(mx, ls[k]);
        }
        float den = 0.f;
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
        for (int k = 0; k < S_; ++k) {
            const float w = ls[k] == -INFINITY ? 0.f : ex2(ls[k] - mx);
            den += w;
            const uint32_t wd[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                acc[2 * e] = fmaf(w, __uint_as_float(wd[e] << 16), acc[2 * e]);
                acc[2 * e + 1] = fmaf(w, __uint_as_float(wd[e] & 0xFFFF0000u), acc[2 * e + 1]);
            }
        }
        const bool dead = nan || !(den > 0.f);
        const float id = dead ? 0.f : 1.f / den;
        const int node = gr / a.G, head = kvh * a.G + gr % a.G;
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) pk[e] = pack_bf16(dead ? NAN : acc[2 * e] * id, dead ? NAN : acc[2 * e + 1] * id);
        *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) + (((size_t)b * a.N + node) * a.Hq + head) * HD +
                                  cc * 8) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
}

template <int NV>
__device__ __forceinline__ float max_tree(const float (&v)[NV]) {
    float m[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) m[k] = v[k];
#pragma unroll
    for (int i = 8; i < NV; ++i) m[i & 7] = fmaxf(m[i & 7], v[i]);
    return fmaxf(fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3])), fmaxf(fmaxf(m[4], m[5]), fmaxf(m[6], m[7])));
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
}  // namespace tv
