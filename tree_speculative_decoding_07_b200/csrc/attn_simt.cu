// attn_simt.cu -- CUDA-core split-KV tree attention (fp32 math).
//
// The fp32 path of tv_tree_attention (a 1e-5 relative tolerance rules out
// TF32 tensor-core math) and the path for shapes the tensor-core kernel does
// not cover.  Every node attends to the prefix and to its own root path
// (glossary page "Tree-based speculative decoding", section "Tree attention":
// M[i][j] = 1 iff j is i or an ancestor of i).
//
// Work decomposition: one CTA per (KV split, 32-row query tile, sequence x
// KV head).  Query rows of one KV head are (node, head-in-group) pairs,
// node-major, so the G query heads sharing a KV head read each K/V row once.
// Tokens are streamed in chunks of 32 through shared memory, one token per
// lane; each warp owns 8 query rows and keeps an online softmax (running max
// and sum in the log2 domain) plus D/32 output columns per lane.  A chunk is
// loaded in 4-element pieces, every thread issuing all of its loads before it
// stores any; the warp's 8 rows are computed together (8 independent dot
// products per token, 8 x D/32 independent accumulations per value row).
#include "tv_common.cuh"
#include "kernels.h"

namespace tv {
namespace {

constexpr int SIMT_WARPS = 4;
constexpr int SIMT_RPW = 8;                       // query rows per warp
constexpr int SIMT_ROWS = SIMT_WARPS * SIMT_RPW;  // query rows per CTA
constexpr int CHUNK = 32;                         // tokens per step (one per lane)

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// four consecutive elements as fp32: one 16-byte (fp32) or 8-byte (bf16) load when
// VEC, else four scalar loads
template <typename T, bool VEC> struct Load4;
template <> struct Load4<float, true> {
    static __device__ __forceinline__ float4 get(const float* p) { return __ldg(reinterpret_cast<const float4*>(p)); }
};
template <> struct Load4<__nv_bfloat16, true> {
    static __device__ __forceinline__ float4 get(const __nv_bfloat16* p) {
        const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
        return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u), __uint_as_float(u.y << 16),
                           __uint_as_float(u.y & 0xFFFF0000u));
    }
};
template <typename T> struct Load4<T, false> {
    static __device__ __forceinline__ float4 get(const T* p) {
        return make_float4(Elem<T>::load(p), Elem<T>::load(p + 1), Elem<T>::load(p + 2), Elem<T>::load(p + 3));
    }
};

template <typename T, int D, bool VEC>
__global__ void __launch_bounds__(SIMT_WARPS * 32) attn_simt_kernel(AttnArgs a) {
    constexpr int DPL = D / 32;
    extern __shared__ float simt_smem[];
    float (*Qs)[D] = reinterpret_cast<float (*)[D]>(simt_smem);
    float (*Ks)[D + 1] = reinterpret_cast<float (*)[D + 1]>(simt_smem + SIMT_ROWS * D);
    float (*Vs)[D] = reinterpret_cast<float (*)[D]>(simt_smem + SIMT_ROWS * D + CHUNK * (D + 1));
    __shared__ uint32_t anc[TV_MAX_NODES_ATTN][4];
    __shared__ int32_t par[TV_MAX_NODES_ATTN];
    __shared__ int s_bad;

    const T* __restrict__ qg = static_cast<const T*>(a.q);
    const T* __restrict__ kg = static_cast<const T*>(a.k);
    const T* __restrict__ vg = static_cast<const T*>(a.v);
    const int split = blockIdx.x, tile = blockIdx.y;
    const int b = blockIdx.z / a.Hkv, kvh = blockIdx.z % a.Hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int N = a.N, G = a.G;
    const int L = a.prefix_lens[b];
    bool bad_count;
    const int n = seq_nodes(a.counts, b, N, bad_count);  // this sequence's tree nodes
    const int total = L + n;
    const int rows_total = G * n;
    const int r0 = tile * SIMT_ROWS;
    if (!bad_count && r0 >= rows_total) return;  // a row tile past a short tree

    if (tid == 0)
        s_bad = bad_count ? TV_ERR_INVALID_ARG
                          : (L < 0 || (total + TV_BLOCK - 1) / TV_BLOCK > a.max_blocks) ? TV_ERR_BLOCK_TABLE : 0;
    for (int i = tid; i < n; i += blockDim.x) par[i] = parent_at(a.parent, b, N, i);
    __syncthreads();
    for (int i = tid; i < n; i += blockDim.x)
        if (!parent_ok(par, i)) s_bad = TV_ERR_TREE;
    __syncthreads();
    const bool tree_bad = s_bad != 0;
    for (int i = tid; i < n; i += blockDim.x) {
        uint32_t m0 = 0, m1 = 0, m2 = 0, m3 = 0;
        if (!tree_bad)
            for (int j = i; j >= 0; j = par[j]) {
                uint32_t bit = 1u << (j & 31);
                int w = j >> 5;
                m0 |= w == 0 ? bit : 0u; m1 |= w == 1 ? bit : 0u;
                m2 |= w == 2 ? bit : 0u; m3 |= w == 3 ? bit : 0u;
            }
        anc[i][0] = m0; anc[i][1] = m1; anc[i][2] = m2; anc[i][3] = m3;
    }
    for (int e = tid; e < SIMT_ROWS * D; e += blockDim.x) {
        const int r = e / D, d = e % D, gr = r0 + r;
        float val = 0.f;
        if (gr < rows_total) {
            const int node = gr / G, h = kvh * G + gr % G;
            val = Elem<T>::load(qg + (((size_t)b * N + node) * a.Hq + h) * D + d) * a.scale_log2;
        }
        Qs[r][d] = val;
    }

    int t0, t1;
    split_range(total, a.splits, split, t0, t1);
    if (tree_bad) t1 = t0;

    float m_run[SIMT_RPW], l_run[SIMT_RPW], acc[SIMT_RPW][DPL];
#pragma unroll
    for (int rr = 0; rr < SIMT_RPW; ++rr) {
        m_run[rr] = -INFINITY;
        l_run[rr] = 0.f;
#pragma unroll
        for (int dd = 0; dd < DPL; ++dd) acc[rr][dd] = 0.f;
    }

    constexpr int PER = CHUNK * D / 4 / (SIMT_WARPS * 32);  // 4-element pieces per thread and chunk
    for (int c0 = t0; c0 < t1; c0 += CHUNK) {
        __syncthreads();  // previous chunk fully consumed (and Qs/anc written on entry)
        {
            float4 kq[PER], vq[PER];
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                const int e = tid + i * SIMT_WARPS * 32;
                const int t = e / (D / 4), d = (e % (D / 4)) * 4, pos = c0 + t;
                kq[i] = make_float4(0.f, 0.f, 0.f, 0.f);
                vq[i] = kq[i];
                if (pos < t1) {
                    const int blk = a.block_table[(size_t)b * a.max_blocks + pos / TV_BLOCK];
                    if (blk < 0 || blk >= a.num_blocks) {
                        s_bad = TV_ERR_BLOCK_TABLE;
                    } else {
                        const size_t off = (((size_t)blk * TV_BLOCK + pos % TV_BLOCK) * a.Hkv + kvh) * D + d;
                        kq[i] = Load4<T, VEC>::get(kg + off);
                        vq[i] = Load4<T, VEC>::get(vg + off);
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                const int e = tid + i * SIMT_WARPS * 32;
                const int t = e / (D / 4), d = (e % (D / 4)) * 4;
                Ks[t][d] = kq[i].x;
                Ks[t][d + 1] = kq[i].y;
                Ks[t][d + 2] = kq[i].z;
                Ks[t][d + 3] = kq[i].w;
                *reinterpret_cast<float4*>(&Vs[t][d]) = vq[i];
            }
        }
        __syncthreads();
        const int pos = c0 + lane;
        const bool in_range = pos < t1;
        // scores of the warp's 8 rows for this lane's token
        float sc[SIMT_RPW];
#pragma unroll
        for (int rr = 0; rr < SIMT_RPW; ++rr) sc[rr] = 0.f;
#pragma unroll 8
        for (int d = 0; d < D; ++d) {
            const float kd = Ks[lane][d];
#pragma unroll
            for (int rr = 0; rr < SIMT_RPW; ++rr) sc[rr] = fmaf(Qs[warp * SIMT_RPW + rr][d], kd, sc[rr]);
        }
        float pr[SIMT_RPW];
#pragma unroll
        for (int rr = 0; rr < SIMT_RPW; ++rr) {
            const int gr = r0 + warp * SIMT_RPW + rr;
            const bool row = gr < rows_total;  // warp-uniform
            bool ok = in_range && row;
            if (ok && pos >= L) {
                const int j = pos - L;
                ok = (anc[gr / G][j >> 5] >> (j & 31)) & 1u;
            }
            const float sv = ok ? sc[rr] : -INFINITY;
            const float m_new = fmaxf(m_run[rr], warp_max(sv));
            // nothing visible yet for this row: its state stays as it was
            const bool live = m_new != -INFINITY;
            pr[rr] = (ok && live) ? exp2f(sv - m_new) : 0.f;
            const float corr = live ? exp2f(m_run[rr] - m_new) : 1.f;
            l_run[rr] = live ? l_run[rr] * corr + warp_sum(pr[rr]) : l_run[rr];
#pragma unroll
            for (int dd = 0; dd < DPL; ++dd) acc[rr][dd] *= corr;
            m_run[rr] = live ? m_new : m_run[rr];
        }
#pragma unroll 4
        for (int t = 0; t < CHUNK; ++t) {
            float vt[DPL];
#pragma unroll
            for (int dd = 0; dd < DPL; ++dd) vt[dd] = Vs[t][lane + 32 * dd];
#pragma unroll
            for (int rr = 0; rr < SIMT_RPW; ++rr) {
                const float pt = __shfl_sync(0xffffffffu, pr[rr], t);
#pragma unroll
                for (int dd = 0; dd < DPL; ++dd) acc[rr][dd] = fmaf(pt, vt[dd], acc[rr][dd]);
            }
        }
    }
    __syncthreads();
    const int bad = s_bad;
    if (bad && tid == 0) report(a.status, bad);

#pragma unroll
    for (int rr = 0; rr < SIMT_RPW; ++rr) {
        const int gr = r0 + warp * SIMT_RPW + rr;
        if (gr >= rows_total) break;
        const int node = gr / G, h = kvh * G + gr % G;
        const size_t row = ((size_t)b * N + node) * a.Hq + h;
        const float inv = l_run[rr] > 0.f ? 1.f / l_run[rr] : 0.f;
        const float lse = l_run[rr] > 0.f ? m_run[rr] + log2f(l_run[rr]) : -INFINITY;
        if (a.splits == 1) {
            T* og = static_cast<T*>(a.out) + row * D;
#pragma unroll
            for (int dd = 0; dd < DPL; ++dd) Elem<T>::store(og + lane + 32 * dd, bad ? NAN : acc[rr][dd] * inv);
        } else {
            const size_t prow = (size_t)split * a.B * N * a.Hq + row;
            float* op = a.o_part + prow * D;
#pragma unroll
            for (int dd = 0; dd < DPL; ++dd) op[lane + 32 * dd] = bad ? NAN : acc[rr][dd] * inv;
            if (lane == 0) a.lse_part[prow] = bad ? NAN : lse;
        }
    }
}

// out = sum_s 2^(lse_s - lse_max) o_s / sum_s 2^(lse_s - lse_max); one CTA per row.
template <typename T>
__global__ void attn_combine_kernel(AttnArgs a) {
    const size_t row = blockIdx.x;
    const size_t rows = (size_t)a.B * a.N * a.Hq;
    {
        const int b = (int)(row / ((size_t)a.N * a.Hq)), node = (int)((row / a.Hq) % a.N);
        bool bad_count;
        if (node >= seq_nodes(a.counts, b, a.N, bad_count)) return;  // no such node in this sequence
    }
    float mx = -INFINITY;
    bool nan = false;
    for (int s = 0; s < a.splits; ++s) {
        const float l = a.lse_part[s * rows + row];
        nan |= isnan(l);
        mx = fmaxf(mx, l);
    }
    T* og = static_cast<T*>(a.out) + row * a.D;
    for (int d = threadIdx.x; d < a.D; d += blockDim.x) {
        float num = 0.f, den = 0.f;
        for (int s = 0; s < a.splits; ++s) {
            const float l = a.lse_part[s * rows + row];
            if (l == -INFINITY) continue;
            const float w = exp2f(l - mx);
            den += w;
            num = fmaf(w, a.o_part[(s * rows + row) * a.D + d], num);
        }
        Elem<T>::store(og + d, (nan || den == 0.f) ? NAN : num / den);
    }
}

constexpr size_t simt_smem_bytes(int D) {
    return sizeof(float) * ((size_t)SIMT_ROWS * D + (size_t)CHUNK * (D + 1) + (size_t)CHUNK * D);
}

template <typename T, int D, bool VEC>
cudaError_t launch_vec(const AttnArgs& a, cudaStream_t st) {
    cudaError_t attr = cudaFuncSetAttribute(attn_simt_kernel<T, D, VEC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            (int)simt_smem_bytes(D));
    if (attr != cudaSuccess) return attr;
    dim3 grid(a.splits, a.row_tiles, a.B * a.Hkv);
    attn_simt_kernel<T, D, VEC><<<grid, SIMT_WARPS * 32, simt_smem_bytes(D), st>>>(a);
    return cudaGetLastError();
}

// vector loads need the caches aligned to 4 elements (16 bytes fp32, 8 bytes bf16)
template <typename T, int D>
cudaError_t launch_dim(const AttnArgs& a, cudaStream_t st) {
    const uintptr_t m = reinterpret_cast<uintptr_t>(a.k) | reinterpret_cast<uintptr_t>(a.v);
    return (m % (4 * sizeof(T))) == 0 ? launch_vec<T, D, true>(a, st) : launch_vec<T, D, false>(a, st);
}

template <typename T>
cudaError_t launch_typed(const AttnArgs& a, cudaStream_t st, int* launches) {
    cudaError_t e = a.D == 128 ? launch_dim<T, 128>(a, st) : launch_dim<T, 64>(a, st);
    *launches = 1;
    if (e != cudaSuccess || a.splits == 1) return e;
    attn_combine_kernel<T><<<a.B * a.N * a.Hq, a.D, 0, st>>>(a);
    *launches = 2;
    return cudaGetLastError();
}

}  // namespace

int simt_rows_per_tile() { return SIMT_ROWS; }

cudaError_t launch_attn_simt(const AttnArgs& a, bool bf16, cudaStream_t st, int* launches) {
    return bf16 ? launch_typed<__nv_bfloat16>(a, st, launches) : launch_typed<float>(a, st, launches);
}

}  // namespace tv
