// sample.cu -- the lossless acceptance walk of tree verification.
//
// Rule (blog "Speculative decoding x tree attention", section 2, table
// "Rejection Sampling Acceptance Condition"): draft x is accepted when
// r < min(1, p(x)/q(x)); on rejection the next token comes from
// max(0, p - q) / sum max(0, p - q).  Trees (glossary "Tree-based speculative
// decoding", section "SpecInfer") are walked root-down; a rejected child
// hands the renormalised residual to its next sibling, and when every child
// fails the bonus token is drawn from the final residual.
//
// Residuals are never materialised.  After j rejections at a node the
// current distribution is max(0, p - c*q) / Z with c = 0, Z = 1 before the
// first rejection (plain p) and, per rejection, c <- c + Z,
// Z <- sum_x max(0, p(x) - c*q(x)).  This equals the explicit renormalisation:
// where max(0, p - c q) > 0, (p - c q)/Z - q = (p - (c + Z) q)/Z, and where it
// is 0 both forms are <= 0.  A zero Z keeps (c, Z).
//
// Layout: one thread-block cluster of C CTAs per sequence.  CTA k holds the
// vocabulary slice [k*S, (k+1)*S) of the current node's p and q rows in
// shared memory, loaded once per node when first needed; every later sibling
// pass and the final draw read the cached slice.  Each normaliser is an fp64
// reduction (per thread, warp shuffle, CTA, then the C partials read through
// distributed shared memory in rank order), so every CTA obtains the same
// bits and takes the same branch without further communication.
#include <cooperative_groups.h>

#include "tv_common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace tv {
namespace {

constexpr int MAX_NODES = 1024;
constexpr int MAX_THREADS = 512;
constexpr int MAX_CLUSTER = 16;

struct SampleShared {
    int16_t parent[MAX_NODES];
    int16_t child_start[MAX_NODES];
    int16_t child_count[MAX_NODES];
    int16_t child_list[MAX_NODES];
    int32_t token[MAX_NODES];
    double ch_p[32], ch_q[32], ch_u[32];
    int32_t ch_node[32];
    double warp_part[MAX_THREADS / 32];
    double cta_part[2];           // this CTA's partial, double-buffered by pass parity
    double all_part[MAX_CLUSTER]; // every CTA's partial of the latest pass
    int bad;
    int found;
};

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// residual mass of one element: p itself while c == 0, else max(0, p - c q)
__device__ __forceinline__ double resid(float p, float q, double c) {
    return c == 0.0 ? (double)p : fmax(0.0, fma(-c, (double)q, (double)p));
}

struct Walker {
    const SampleArgs& a;
    SampleShared& sh;
    float* ps;
    float* qs;
    int rank, C, lo, n, tid, lane, warp, nwarps;
    int pass;

    // Sum over the whole row of resid(p, q, c); every CTA returns the same value.
    __device__ double cluster_sum(double c) {
        double acc = 0.0;
        for (int i = tid; i < n; i += blockDim.x) acc += resid(ps[i], qs[i], c);
        acc = warp_sum_d(acc);
        if (lane == 0) sh.warp_part[warp] = acc;
        __syncthreads();
        const int slot = pass & 1;
        ++pass;
        if (tid == 0) {
            double s = 0.0;
            for (int w = 0; w < nwarps; ++w) s += sh.warp_part[w];
            sh.cta_part[slot] = s;
        }
        if (C == 1) {
            __syncthreads();
            if (tid == 0) sh.all_part[0] = sh.cta_part[slot];
            __syncthreads();
            return sh.all_part[0];
        }
        cg::cluster_group cluster = cg::this_cluster();
        cluster.sync();  // every CTA's partial of this pass is written
        if (tid < C) sh.all_part[tid] = *cluster.map_shared_rank(&sh.cta_part[slot], tid);
        __syncthreads();
        double total = 0.0;
        for (int k = 0; k < C; ++k) total += sh.all_part[k];
        // A later pass writes the other slot; the pass after that rewrites this
        // slot only once every CTA has passed the next cluster.sync, i.e. after
        // all remote reads of this pass.
        return total;
    }

    __device__ void load_row(int u) {
        const size_t base = ((size_t)(blockIdx.x / C) * a.N + u) * (size_t)a.V + lo;
        const float* pr = a.p + base;
        const float* qr = a.q + base;
        if (a.vec4) {
            const int n4 = n >> 2;
            const float4* p4 = reinterpret_cast<const float4*>(pr);
            const float4* q4 = reinterpret_cast<const float4*>(qr);
            float4* ps4 = reinterpret_cast<float4*>(ps);
            float4* qs4 = reinterpret_cast<float4*>(qs);
#pragma unroll 4
            for (int i = tid; i < n4; i += blockDim.x) {
                ps4[i] = __ldg(p4 + i);
                qs4[i] = __ldg(q4 + i);
            }
            for (int i = (n4 << 2) + tid; i < n; i += blockDim.x) {
                ps[i] = __ldg(pr + i);
                qs[i] = __ldg(qr + i);
            }
        } else {
#pragma unroll 4
            for (int i = tid; i < n; i += blockDim.x) {
                ps[i] = __ldg(pr + i);
                qs[i] = __ldg(qr + i);
            }
        }
        __syncthreads();
    }
};

__global__ void __launch_bounds__(MAX_THREADS) verify_sample_kernel(SampleArgs a) {
    extern __shared__ float4 sample_dyn[];
    __shared__ SampleShared sh;
    const int C = a.cluster;
    const int rank = C > 1 ? (int)cg::this_cluster().block_rank() : 0;
    const int b = blockIdx.x / C;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
    const int N = a.N;
    const int lo = min(a.V, rank * a.slice);
    const int n = min(a.V, lo + a.slice) - lo;
    float* ps = reinterpret_cast<float*>(sample_dyn);
    float* qs = ps + a.slice;

    // ---- tree: validate, child lists in ascending index order
    if (tid == 0) sh.bad = 0;
    for (int i = tid; i < N; i += blockDim.x) {
        sh.parent[i] = (int16_t)max(-1, min(a.parent[(size_t)b * N + i], MAX_NODES - 1));
        sh.token[i] = a.tokens[(size_t)b * N + i];
        sh.child_count[i] = 0;
    }
    __syncthreads();
    for (int i = tid; i < N; i += blockDim.x) {
        const int p = a.parent[(size_t)b * N + i];
        const bool ok = (i == 0) ? p == -1 : (p >= 0 && p < i && sh.token[i] >= 0 && sh.token[i] < a.V);
        if (!ok) sh.bad = 1;
    }
    __syncthreads();
    const bool bad = sh.bad != 0;
    if (!bad) {
        if (tid == 0) {
            for (int c = 1; c < N; ++c) sh.child_count[sh.parent[c]]++;
            int s = 0;
            for (int v = 0; v < N; ++v) { sh.child_start[v] = (int16_t)s; s += sh.child_count[v]; }
        }
        __syncthreads();
        // child c goes to slot start(parent) + (number of earlier siblings)
        for (int c = 1 + tid; c < N; c += blockDim.x) {
            const int p = sh.parent[c];
            int r = 0;
            for (int j = p + 1; j < c; ++j) r += sh.parent[j] == p;
            sh.child_list[sh.child_start[p] + r] = (int16_t)c;
        }
        __syncthreads();
    }

    Walker w{a, sh, ps, qs, rank, C, lo, n, tid, lane, warp, nwarps, 0};
    int32_t* path_out = a.path + (size_t)b * N;

    if (bad) {
        if (rank == 0) {
            for (int i = tid; i < N; i += blockDim.x) path_out[i] = -1;
            if (tid == 0) {
                a.len[b] = -1;
                a.bonus[b] = -1;
                report(a.status, TV_ERR_TREE);
            }
        }
        if (C > 1) cg::this_cluster().sync();
        return;
    }

    // ---- walk from the root
    int u = 0, len = 0;
    int loaded = -1;  // node whose row slice sits in ps/qs
    double cur_c = 0.0, cur_z = 1.0;
    for (;;) {
        cur_c = 0.0;
        cur_z = 1.0;
        int accepted = -1;
        const int cs = sh.child_start[u], cc = sh.child_count[u];
        for (int g0 = 0; g0 < cc && accepted < 0; g0 += 32) {
            // gather up to 32 children's scalars at once
            __syncthreads();
            if (warp == 0 && g0 + lane < cc) {
                const int c = sh.child_list[cs + g0 + lane];
                const int x = sh.token[c];
                const size_t row = ((size_t)b * N + u) * (size_t)a.V;
                sh.ch_node[lane] = c;
                sh.ch_p[lane] = (double)__ldg(a.p + row + x);
                sh.ch_q[lane] = (double)__ldg(a.q + row + x);
                sh.ch_u[lane] = (double)__ldg(a.uniforms + (size_t)b * N + c);
            }
            __syncthreads();
            const int gn = min(32, cc - g0);
            for (int k = 0; k < gn; ++k) {
                const double px = sh.ch_p[k], qx = sh.ch_q[k], r = sh.ch_u[k];
                const double num = cur_c == 0.0 ? px : fmax(0.0, fma(-cur_c, qx, px));
                const bool acc = qx > 0.0 ? (r < num / (cur_z * qx)) : (num > 0.0);
                if (acc) { accepted = sh.ch_node[k]; break; }
                if (loaded != u) { w.load_row(u); loaded = u; }
                const double c_new = cur_c + cur_z;
                const double z_new = w.cluster_sum(c_new);
                if (z_new > 0.0) { cur_c = c_new; cur_z = z_new; }
            }
        }
        if (accepted >= 0) {
            if (rank == 0 && tid == 0) path_out[len] = accepted;
            ++len;
            u = accepted;
            continue;
        }
        break;
    }

    // ---- bonus token: first index whose running residual mass exceeds u0 * total
    if (loaded != u) { w.load_row(u); loaded = u; }
    const double total = w.cluster_sum(cur_c);  // also leaves every CTA's partial in all_part
    const double target = (double)__ldg(a.uniforms + (size_t)b * N) * total;
    // first CTA whose inclusive prefix exceeds the target; the last CTA with
    // mass if rounding leaves none
    int owner = -1, last_pos_cta = -1;
    double before = 0.0, run = 0.0;
    for (int k = 0; k < C; ++k) {
        const double pk = sh.all_part[k];
        if (pk > 0.0) last_pos_cta = k;
        if (owner < 0) {
            if (run + pk > target) { owner = k; before = run; }
            run += pk;
        }
    }
    const bool fallback = owner < 0;
    if (fallback) owner = last_pos_cta;

    if (rank == owner) {
        // warp segments of the slice, contiguous, 32-aligned
        const int segw = ((n + nwarps - 1) / nwarps + 31) / 32 * 32;
        const int s0 = min(n, warp * segw), s1 = min(n, s0 + segw);
        double ws = 0.0;
        for (int i = s0 + lane; i < s1; i += 32) ws += resid(ps[i], qs[i], cur_c);
        ws = warp_sum_d(ws);
        if (lane == 0) sh.warp_part[warp] = ws;
        if (tid == 0) sh.found = -1;
        __syncthreads();
        __shared__ int s_warp;
        __shared__ double s_before;
        if (tid == 0) {
            int wsel = -1, wlast = -1;
            double rb = before, rr = before;
            for (int k = 0; k < nwarps; ++k) {
                if (sh.warp_part[k] > 0.0) wlast = k;
                if (wsel < 0 && !fallback) {
                    if (rr + sh.warp_part[k] > target) { wsel = k; rb = rr; }
                    rr += sh.warp_part[k];
                }
            }
            if (wsel < 0) { wsel = wlast; rb = -INFINITY; }  // rounding: last positive element
            s_warp = wsel;
            s_before = rb;
        }
        __syncthreads();
        if (warp == s_warp) {
            const bool take_last = s_before == -INFINITY;
            double rr = s_before;
            int pick = -1, lastp = -1;
            for (int i0 = s0; i0 < s1; i0 += 32) {
                const int i = i0 + lane;
                const double v = i < s1 ? resid(ps[i], qs[i], cur_c) : 0.0;
                double sc = v;  // inclusive scan over the lanes
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const double t = __shfl_up_sync(0xffffffffu, sc, o);
                    if (lane >= o) sc += t;
                }
                const unsigned pos = __ballot_sync(0xffffffffu, v > 0.0);
                if (pos) lastp = i0 + 31 - __clz(pos);
                if (!take_last) {
                    const unsigned hit = __ballot_sync(0xffffffffu, rr + sc > target);
                    if (hit) { pick = i0 + __ffs(hit) - 1; break; }
                    rr += __shfl_sync(0xffffffffu, sc, 31);
                }
            }
            if (pick < 0) pick = lastp;  // rounding left no crossing inside the segment
            if (lane == 0) sh.found = pick;
        }
        __syncthreads();
        if (tid == 0) {
            a.bonus[b] = sh.found >= 0 ? lo + sh.found : -1;
            a.len[b] = len;
        }
        for (int i = len + tid; i < N; i += blockDim.x) path_out[i] = -1;
    } else if (owner < 0 && rank == 0) {
        // no mass anywhere (all-zero distribution)
        if (tid == 0) { a.bonus[b] = -1; a.len[b] = len; }
        for (int i = len + tid; i < N; i += blockDim.x) path_out[i] = -1;
    }
    if (C > 1) cg::this_cluster().sync();  // keep shared memory alive for remote readers
}

}  // namespace

int sample_max_cluster() {
    static int best = -1;
    if (best >= 0) return best;
    best = 8;
    if (cudaFuncSetAttribute(verify_sample_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        cfg.gridDim = dim3(16, 1, 1);
        cfg.blockDim = dim3(MAX_THREADS, 1, 1);
        cfg.dynamicSmemBytes = 96 * 1024;
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 16;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        cudaFuncSetAttribute(verify_sample_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 96 * 1024);
        int clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&clusters, verify_sample_kernel, &cfg) == cudaSuccess && clusters > 0)
            best = 16;
    }
    cudaGetLastError();
    return best;
}

cudaError_t launch_verify_sample(const SampleArgs& a, cudaStream_t st, int* launches) {
    cudaError_t e = cudaFuncSetAttribute(verify_sample_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         a.smem_bytes);
    if (e != cudaSuccess) return e;
    if (a.cluster > 8) {
        e = cudaFuncSetAttribute(verify_sample_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    cfg.gridDim = dim3((unsigned)a.cluster * (unsigned)a.B, 1, 1);
    cfg.blockDim = dim3(a.threads, 1, 1);
    cfg.dynamicSmemBytes = a.smem_bytes;
    cfg.stream = st;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = a.cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = a.cluster > 1 ? 1 : 0;
    *launches = 1;
    return cudaLaunchKernelEx(&cfg, verify_sample_kernel, a);
}

}  // namespace tv
