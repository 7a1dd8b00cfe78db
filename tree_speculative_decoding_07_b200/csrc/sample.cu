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
// Layout: one thread-block cluster of C CTAs per sequence; CTA k owns the
// vocabulary slice [k*S, (k+1)*S).  When the walk arrives at a node every CTA
// starts a bulk copy of its slice of that node's p and q rows into one of two
// shared-memory buffers, so the row is usually resident by the time a
// rejection needs it.  Each normaliser is an fp64 reduction: per lane over a
// contiguous per-warp segment, warp shuffle, CTA, then every CTA pushes its
// partial to all peers with st.async, which completes on the receiver's own
// mbarrier; every CTA adds the C partials in rank order, so all obtain the
// same bits and take the same branches.  The first pass over a row keeps each
// lane's entries in registers as fp64 (segments of up to four 128-entry
// steps), so later passes on that row do only the fp64 arithmetic.  The bonus
// draw reuses the per-CTA and per-warp partials of the last pass: the owning
// CTA and warp are located from them, the owning CTA scans that warp's
// segment, and one thread finds the element among its few.
//
// Children.  Every CTA first gathers, for every child c of the tree, the
// draft token's entries p(x_c), q(x_c) of its parent's rows and its uniform
// into shared memory (one round of independent loads), so no acceptance test
// waits on a global load.  With those values the walk knows, on arriving at a
// node, whether its first child passes the plain test u_c < p(x)/q(x); while
// it does, the walk moves on without that node's row, and the row load is
// started only for the node where the first test fails (its residual is
// needed) or the leaf where the walk ends (its bonus draw).  The logits form
// needs every visited row's softmax before any test, so it loads each
// visited row.  When the vocabulary slice leaves no shared memory for the
// gathered values, each node's children are gathered when the walk reaches it.
//
// Exit.  No CTA retires while a peer may still write to its shared memory:
// every CTA arrives on every peer's exit barrier and waits (bounded) on its
// own.  A CTA whose bounded wait ran out stops exchanging (no pushes, no
// waits), so its peers time out once and stop too; the status word records
// TV_ERR_TIMEOUT.
#include <cooperative_groups.h>
#include <mutex>

#include "tv_common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace tv {
namespace {

constexpr int MAX_NODES = 1024;
constexpr int MAX_THREADS = 512;
constexpr int MAX_CLUSTER = 16;
constexpr long long WAIT_LIMIT = 1ll << 32;  // clock cycles (~2 s)

struct SampleShared {
    int32_t parent[MAX_NODES];
    int32_t token[MAX_NODES];
    double ch_p[32], ch_q[32], ch_u[32];
    int32_t ch_node[32];
    int ch_n;      // children gathered in this batch
    int ch_next;   // index where the scan for the next batch resumes (N when done)
    double warp_part[MAX_THREADS / 32];
    double warp_part2[MAX_THREADS / 32];
    double peer[2][MAX_CLUSTER];   // values from every CTA of the cluster, by exchange parity
    double peer2[2][MAX_CLUSTER];  // second values of two-value exchanges
    // logits mode: the softmax of the row in buffer x is p = exp(l - row_mp[x]) * row_zp_inv[x]
    double row_zp_inv[2], row_zq_inv[2];
    float row_mp[2], row_mq[2];
    unsigned long long peer_bar[2];
    unsigned long long row_bar[2];
    unsigned long long exit_bar;
    int timeout;
    int found;
    int found_t;
    int wsel;
    double wbefore;
    float u0;                       // the bonus draw's uniform, read at launch
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
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
// bounded wait on one phase; false (and the timeout flag set) when it runs out,
// and false at once when an earlier wait of this CTA ran out
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* timeout) {
    if (mbar_try(bar, parity)) return true;
    if (*timeout) return false;
    const long long t0 = clock64();
    for (;;) {
        if (mbar_try(bar, parity)) return true;
        if (clock64() - t0 > WAIT_LIMIT) {
            *timeout = 1;
            return false;
        }
    }
}
// arrive on the mbarrier at this shared::cluster address (any CTA of the cluster);
// relaxed: the exit barrier orders nothing but "this CTA sends no more values"
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ bool mbar_try_cluster(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ uint32_t mapa(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
// remote store of one double that completes 8 bytes on the receiver's mbarrier
__device__ __forceinline__ void st_async_f64(uint32_t remote_addr, double v, uint32_t remote_bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b64 [%0], %1, [%2];" ::"r"(remote_addr),
                 "l"(__double_as_longlong(v)), "r"(remote_bar)
                 : "memory");
}
// bring [src, src + bytes) into L2 (16-byte aligned, a multiple of 16 bytes); no data
// reaches the CTA, so it may run before the previous kernel has finished
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(src)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void prefetch_line_l2(const void* p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<uint64_t>(p)) : "memory");
}
// bulk copy global -> this CTA's shared memory, completing on a local mbarrier
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
                 : "memory");
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
// inclusive prefix sums over lanes 0..15 (lane k gets v_0 + ... + v_k, summed as a tree;
// lanes 16..31 get values that are not used)
__device__ __forceinline__ double half_scan_d(double v, int lane) {
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) {
        const double t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
    }
    return v;
}
// The first of n (<= 16) running totals that exceeds a target, from one value per lane:
// `first` is that lane (-1 if none), `last_pos` the last lane with a positive value, and
// `before` the running total of the lanes before `first` (0 for lane 0).  Every lane of
// the warp gets the same results.
struct Crossing {
    int first, last_pos;
    double before;
};
__device__ __forceinline__ Crossing first_crossing(double v, int n, double base, double target, int lane) {
    const double inc = half_scan_d(lane < n ? v : 0.0, lane);
    const unsigned cross = __ballot_sync(0xffffffffu, lane < n && base + inc > target);
    const unsigned pos = __ballot_sync(0xffffffffu, lane < n && v > 0.0);
    Crossing r;
    r.first = cross ? __ffs((int)cross) - 1 : -1;
    r.last_pos = pos ? 31 - __clz((int)pos) : -1;
    const double prev = __shfl_sync(0xffffffffu, inc, r.first > 0 ? r.first - 1 : 0);
    r.before = base + (r.first > 0 ? prev : 0.0);
    return r;
}
// Sum and maximum over 16 values (a cluster's CTAs, a CTA's warps: both at most 16).
// Both half-warps hold the 16 values, so four butterfly levels give every lane the
// result, with the same pairings, hence the same bits, as a 32-lane butterfly over the
// values padded with the identity.
static_assert(MAX_CLUSTER <= 16 && MAX_THREADS / 32 <= 16, "the half-warp reductions take at most 16 values");
__device__ __forceinline__ double half_sum_d(double v) {
#pragma unroll
    for (int o = 8; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ double half_max_d(double v) {
#pragma unroll
    for (int o = 8; o; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_max_f(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// max(0, d) for the residual terms: the sign is read from the high word, because
// the fp64 max instruction runs at an eighth of the fp64 add / fma rate
__device__ __forceinline__ double pos_part(double d) { return __double2hiint(d) >= 0 ? d : 0.0; }

// residual mass of one element: p itself while c == 0, else max(0, p - c q)
__device__ __forceinline__ double resid(float p, float q, double c) {
    return c == 0.0 ? (double)p : pos_part(fma(-c, (double)q, (double)p));
}

struct Walker {
    SampleShared& sh;
    float* buf;      // [2][2][slice]: buffer x holds p at buf + 2*x*slice, q right after
    const float* p;
    const float* q;
    int V, N, slice;
    int b, rank, C, lo, n, tid, lane, warp, nwarps, segw;
    bool bulk;
    int passes;        // cluster exchanges so far
    uint32_t pending;  // bit x: a copy into buffer x is in flight
    uint32_t phase;    // bit x: parity of the next phase of buffer x's barrier
    // The lane's whole steps of one buffer's row, converted to fp64 by the first pass
    // over that row (rows of at most four steps per lane): later passes on the same row
    // neither read shared memory nor convert again.  Steps past the slice hold zeros.
    int cached = -1;   // buffer whose row rp / rq hold, -1 for none
    double rp[4][4], rq[4][4];

    __device__ float* ps(int x) const { return buf + (size_t)2 * x * slice; }
    __device__ float* qs(int x) const { return ps(x) + slice; }
    __device__ uint32_t row_bar(int x) const { return smem_u32(&sh.row_bar[x]); }

    // Wait until buffer x holds its row (collective).  Always waits (bounded), even
    // after a timeout elsewhere: no copy may land in a buffer that is reused or in a
    // CTA that has retired.
    __device__ void wait_row(int x) {
        if (!((pending >> x) & 1u)) return;
        const uint32_t par = (phase >> x) & 1u;
        if (!mbar_try(row_bar(x), par)) {
            const long long t0 = clock64();
            while (!mbar_try(row_bar(x), par)) {
                if (clock64() - t0 > WAIT_LIMIT) {
                    sh.timeout = 1;
                    break;
                }
            }
        }
        phase ^= 1u << x;
        pending &= ~(1u << x);
    }

    // Start loading this CTA's slice of node u's p and q rows into buffer x (collective).
    __device__ __forceinline__ void issue_row(int x, int u) {
        wait_row(x);  // the buffer's previous copy must have landed before it is reused
        if (cached == x) cached = -1;
        const size_t base = ((size_t)b * N + u) * (size_t)V + lo;
        if (bulk) {
            if (tid == 0) {
                mbar_expect_tx(row_bar(x), (uint32_t)(8 * n));
                if (n > 0) {
                    bulk_load(smem_u32(ps(x)), p + base, (uint32_t)(4 * n), row_bar(x));
                    bulk_load(smem_u32(qs(x)), q + base, (uint32_t)(4 * n), row_bar(x));
                }
            }
        } else {
            float* pd = ps(x);
            float* qd = qs(x);
            for (int i = tid; i < n; i += blockDim.x) {
                pd[i] = __ldg(p + base + i);
                qd[i] = __ldg(q + base + i);
            }
            __syncthreads();
            if (tid == 0) mbar_expect_tx(row_bar(x), 0);
        }
        pending |= 1u << x;
    }

    // Sum over the whole row of resid(p, q, c) from buffer x; every CTA returns
    // the same value.  Leaves this CTA's per-warp partials in sh.warp_part and
    // every CTA's partial in sh.peer[parity of the pass].
    __device__ __forceinline__ double cluster_pass(int x, double c) {
        const float* pr = ps(x);
        const float* qr = qs(x);
        const int s0 = min(n, warp * segw), s1 = min(n, s0 + segw);
        double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
        // four consecutive elements per lane and step (16-byte shared loads; segw is a
        // multiple of 128 and the slices start 16-byte aligned); a lane's last,
        // incomplete step at the end of the row is done element by element
        int i = s0 + 4 * lane;
        if (c == 0.0) {
            for (; i + 3 < s1; i += 128) {
                const float4 pv = *reinterpret_cast<const float4*>(pr + i);
                a0 += (double)pv.x;
                a1 += (double)pv.y;
                a2 += (double)pv.z;
                a3 += (double)pv.w;
            }
        } else if (segw <= 4 * 128) {
            if (cached != x) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    float4 pv = make_float4(0.f, 0.f, 0.f, 0.f), qv = pv;
                    if (i + 128 * k + 3 < s1) {
                        pv = *reinterpret_cast<const float4*>(pr + i + 128 * k);
                        qv = *reinterpret_cast<const float4*>(qr + i + 128 * k);
                    }
                    rp[k][0] = pv.x;
                    rp[k][1] = pv.y;
                    rp[k][2] = pv.z;
                    rp[k][3] = pv.w;
                    rq[k][0] = qv.x;
                    rq[k][1] = qv.y;
                    rq[k][2] = qv.z;
                    rq[k][3] = qv.w;
                }
                cached = x;
            }
            // the same sums in the same order as from shared memory: a zero step adds +0.0
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                a0 += pos_part(fma(-c, rq[k][0], rp[k][0]));
                a1 += pos_part(fma(-c, rq[k][1], rp[k][1]));
                a2 += pos_part(fma(-c, rq[k][2], rp[k][2]));
                a3 += pos_part(fma(-c, rq[k][3], rp[k][3]));
            }
            while (i + 3 < s1) i += 128;
        } else {
            for (; i + 3 < s1; i += 128) {
                const float4 pv = *reinterpret_cast<const float4*>(pr + i);
                const float4 qv = *reinterpret_cast<const float4*>(qr + i);
                a0 += pos_part(fma(-c, (double)qv.x, (double)pv.x));
                a1 += pos_part(fma(-c, (double)qv.y, (double)pv.y));
                a2 += pos_part(fma(-c, (double)qv.z, (double)pv.z));
                a3 += pos_part(fma(-c, (double)qv.w, (double)pv.w));
            }
        }
        for (int e = i; e < s1 && e < i + 4; ++e) a0 += resid(pr[e], qr[e], c);
        const double wsum = warp_sum_d((a0 + a1) + (a2 + a3));
        if (lane == 0) sh.warp_part[warp] = wsum;
        __syncthreads();
        // this CTA's partial: a fixed shuffle tree over its warps (warp 0's value is sent)
        const double s = warp == 0 ? half_sum_d((lane & 15) < nwarps ? sh.warp_part[lane & 15] : 0.0) : 0.0;
        double total, unused;
        exchange(1, s, 0.0, false, total, unused);
        return total;
    }

    // One cluster-wide exchange of nv (1 or 2) values: warp 0 holds this CTA's values
    // v0, v1 and sends them to every CTA of the cluster (one lane per receiver, by
    // st.async completing on the receiver's own mbarrier); every warp then combines
    // the C values with the same shuffle tree -- sums, or maxima when take_max -- so
    // all CTAs and all warps obtain the same bits and take the same branches.  The
    // per-CTA values stay in sh.peer / sh.peer2 at the parity of the exchange.  Once a
    // wait of this CTA has run out it neither sends nor waits any more.
    __device__ __forceinline__ void exchange(int nv, double v0, double v1, bool take_max, double& r0, double& r1) {
        const int par = passes & 1;
        const uint32_t use = (uint32_t)(passes >> 1);
        ++passes;
        if (warp == 0) {
            if (C == 1) {
                if (lane == 0) {
                    sh.peer[par][0] = v0;
                    sh.peer2[par][0] = v1;
                }
            } else if (!sh.timeout) {
                const uint32_t bar = smem_u32(&sh.peer_bar[par]);
                if (lane == 0) mbar_expect_tx(bar, (uint32_t)(8 * nv * C));
                if (lane < C) {
                    st_async_f64(mapa(smem_u32(&sh.peer[par][rank]), lane), v0, mapa(bar, lane));
                    if (nv == 2) st_async_f64(mapa(smem_u32(&sh.peer2[par][rank]), lane), v1, mapa(bar, lane));
                }
            }
        }
        if (C == 1) {
            __syncthreads();
        } else {
            mbar_wait(smem_u32(&sh.peer_bar[par]), use & 1, &sh.timeout);
        }
        const double id = take_max ? -INFINITY : 0.0;
        const int k = lane & 15;
        const double x0 = k < C ? sh.peer[par][k] : id;
        r0 = take_max ? half_max_d(x0) : half_sum_d(x0);
        if (nv == 2) {
            const double x1 = k < C ? sh.peer2[par][k] : id;
            r1 = take_max ? half_max_d(x1) : half_sum_d(x1);
        } else {
            r1 = 0.0;
        }
    }

    // Logits mode: buffer x holds this CTA's slice of one node's target and draft
    // logits.  Turn them in place into the row softmax: e = exp(l - M) in fp32 with M
    // the row max, Z the fp64 sum of e over the whole row (both cluster-wide), and
    // p = (float)(e * (1 / Z)); keep M and 1 / Z for the children's p(x), q(x), which
    // the gather computes with the same expression so they equal the converted row.
    __device__ void prep_row(int x) {
        if (cached == x) cached = -1;  // the row is rewritten in place
        float* pl = ps(x);
        float* ql = qs(x);
        float mp = -INFINITY, mq = -INFINITY;
        for (int i = tid; i < n; i += blockDim.x) {
            mp = fmaxf(mp, pl[i]);
            mq = fmaxf(mq, ql[i]);
        }
        mp = warp_max_f(mp);
        mq = warp_max_f(mq);
        if (lane == 0) {
            sh.warp_part[warp] = (double)mp;
            sh.warp_part2[warp] = (double)mq;
        }
        __syncthreads();
        double Mp, Mq;
        {
            const int k = lane & 15;
            const double v0 = warp == 0 ? half_max_d(k < nwarps ? sh.warp_part[k] : -INFINITY) : 0.0;
            const double v1 = warp == 0 ? half_max_d(k < nwarps ? sh.warp_part2[k] : -INFINITY) : 0.0;
            exchange(2, v0, v1, true, Mp, Mq);
        }
        const float mpf = (float)Mp, mqf = (float)Mq;
        double sp = 0.0, sq = 0.0;
        for (int i = tid; i < n; i += blockDim.x) {
            const float ep = expf(pl[i] - mpf), eq = expf(ql[i] - mqf);
            pl[i] = ep;
            ql[i] = eq;
            sp += (double)ep;
            sq += (double)eq;
        }
        sp = warp_sum_d(sp);
        sq = warp_sum_d(sq);
        __syncthreads();  // warp 0 has read the max partials before its exchange
        if (lane == 0) {
            sh.warp_part[warp] = sp;
            sh.warp_part2[warp] = sq;
        }
        __syncthreads();
        double Zp, Zq;
        {
            const int k = lane & 15;
            const double v0 = warp == 0 ? half_sum_d(k < nwarps ? sh.warp_part[k] : 0.0) : 0.0;
            const double v1 = warp == 0 ? half_sum_d(k < nwarps ? sh.warp_part2[k] : 0.0) : 0.0;
            exchange(2, v0, v1, false, Zp, Zq);
        }
        const double zpi = Zp > 0.0 ? 1.0 / Zp : 0.0, zqi = Zq > 0.0 ? 1.0 / Zq : 0.0;
        for (int i = tid; i < n; i += blockDim.x) {
            pl[i] = (float)((double)pl[i] * zpi);
            ql[i] = (float)((double)ql[i] * zqi);
        }
        if (tid == 0) {
            sh.row_mp[x] = mpf;
            sh.row_mq[x] = mqf;
            sh.row_zp_inv[x] = zpi;
            sh.row_zq_inv[x] = zqi;
        }
        __syncthreads();
    }
};

template <bool LOGITS>
__global__ void __launch_bounds__(MAX_THREADS) verify_sample_kernel(const __grid_constant__ SampleArgs a) {
    extern __shared__ float4 sample_dyn[];
    __shared__ SampleShared sh;
    const int C = a.cluster;
    const int rank = C > 1 ? (int)cg::this_cluster().block_rank() : 0;
    const int b = blockIdx.x / C;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
    const int N = a.N;
    const int lo = min(a.V, rank * a.slice);
    const int n = min(a.V, lo + a.slice) - lo;
    float* const rows = reinterpret_cast<float*>(sample_dyn);
    // the gathered child values follow the two row buffers (a.gather): p(x_c) and
    // q(x_c) of child c's token in its parent's rows (the raw logits in logits mode),
    // c's uniform, and each node's first child (nn when it has none)
    float* const g_p = rows + 4 * (size_t)a.slice;
    float* const g_q = g_p + N;
    float* const g_u = g_q + N;
    int* const g_first = reinterpret_cast<int*>(g_u + N);

    if (tid == 0) {
        sh.timeout = 0;
        for (int x = 0; x < 2; ++x) {
            mbar_init(smem_u32(&sh.row_bar[x]), 1);
            mbar_init(smem_u32(&sh.peer_bar[x]), 1);
        }
        mbar_init(smem_u32(&sh.exit_bar), (uint32_t)C);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // Launched with a programmatic dependency, the kernel may start while the previous
    // kernel still runs: warm L2 (and the address translations) for what the walk
    // reads first -- this CTA's slice of the root's p and q rows, and the sequence's
    // tree, tokens and uniforms.  Only prefetches happen before the wait below: the
    // data is read after it, so a write by the previous kernel is still seen.
    if (tid == 0 && a.vec4 && n > 0) {
        const size_t row = (size_t)b * N * (size_t)a.V + lo;  // node 0's row
        bulk_prefetch_l2(a.p + row, (uint32_t)(4 * n));
        bulk_prefetch_l2(a.q + row, (uint32_t)(4 * n));
    }
    if (rank == 0 && tid < 96) {
        const int arr = tid / 32, line = tid % 32;  // parents, tokens, uniforms: 32 lines of 128 B each
        const char* base = arr == 0 ? reinterpret_cast<const char*>(a.parent)
                                    : arr == 1 ? reinterpret_cast<const char*>(a.tokens)
                                               : reinterpret_cast<const char*>(a.uniforms);
        if (base && 128 * line < 4 * N) prefetch_line_l2(base + 4 * (size_t)b * N + 128 * line);
    }
    __syncthreads();
    // the kernel may have been launched while the previous one on the stream was still
    // running (programmatic dependent launch): its inputs are read only after that
    // kernel has completed and its memory is visible
    asm volatile("griddepcontrol.wait;" ::: "memory");

    Walker w{sh, rows, a.p, a.q, a.V, N, a.slice, b, rank, C, lo, n, tid, lane, warp, nwarps,
             ((n + nwarps - 1) / nwarps + 127) / 128 * 128, a.vec4 != 0, 0, 0u, 0u};
    // the root's row is needed unless its first child is accepted: start it now
    w.issue_row(0, 0);

    // ---- tree and tokens; a malformed sequence gets -1 outputs
    bool bad_count;
    const int nn = seq_nodes(a.counts, b, N, bad_count);  // this sequence's tree nodes
    for (int i = tid; i < nn; i += blockDim.x) {
        sh.parent[i] = parent_at(a.parent, b, N, i);
        sh.token[i] = a.tokens[(size_t)b * N + i];
        if (a.gather) g_first[i] = nn;
    }
    if (tid == 0) sh.u0 = __ldg(a.uniforms + (size_t)b * N);
    __syncthreads();
    // Every child's draft-token entries and uniform are requested now, before the cluster
    // barrier, so their latency overlaps it.  Each entry's parent and token are checked one
    // by one: a malformed tree's values are never used, but no load may leave the rows.
    // (Up to two children per thread; a tree with more falls back to loading them after
    // the checks below.)
    constexpr int GPT = 2;
    const bool early = a.gather && nn <= GPT * (int)blockDim.x;
    float gp[GPT], gq[GPT], gu[GPT];
#pragma unroll
    for (int k = 0; k < GPT; ++k) {
        gp[k] = gq[k] = gu[k] = 0.f;
        const int c = tid + 1 + k * (int)blockDim.x;
        if (early && c < nn) {
            const int pu = sh.parent[c], tk = sh.token[c];
            if (pu >= 0 && pu < c && tk >= 0 && tk < a.V) {
                const size_t at = ((size_t)b * N + pu) * (size_t)a.V + tk;
                gp[k] = __ldg(a.p + at);
                gq[k] = __ldg(a.q + at);
                gu[k] = __ldg(a.uniforms + (size_t)b * N + c);
            }
        }
    }
    // every CTA's barriers must exist before a peer pushes to them (the first pass)
    if (C > 1) cg::this_cluster().sync();
    bool bad_local = false;
    for (int i = tid; i < nn; i += blockDim.x) {
        const int p = sh.parent[i];
        bad_local |= (i == 0) ? p != -1 : (p < 0 || p >= i || sh.token[i] < 0 || sh.token[i] >= a.V);
    }
    int32_t* path_out = a.path + (size_t)b * N;
    if (__syncthreads_or(bad_local) || bad_count || nn == 0) {
        // a malformed sequence gets -1 outputs; an empty one (no tree this step)
        // accepts nothing and draws no token
        if (rank == 0) {
            for (int i = tid; i < N; i += blockDim.x) path_out[i] = -1;
            if (tid == 0) {
                const bool empty = nn == 0 && !bad_count;
                a.len[b] = empty ? 0 : -1;
                a.bonus[b] = -1;
                if (!empty) report(a.status, bad_count ? TV_ERR_INVALID_ARG : TV_ERR_TREE);
            }
        }
    } else {
        if (early) {
#pragma unroll
            for (int k = 0; k < GPT; ++k) {
                const int c = tid + 1 + k * (int)blockDim.x;
                if (c < nn) {
                    g_p[c] = gp[k];
                    g_q[c] = gq[k];
                    g_u[c] = gu[k];
                    atomicMin(&g_first[sh.parent[c]], c);
                }
            }
            __syncthreads();
        } else if (a.gather) {
            // every child's draft-token entries and uniform, in one round of loads
            for (int c = tid + 1; c < nn; c += blockDim.x) {
                const int pu = sh.parent[c];
                const size_t at = ((size_t)b * N + pu) * (size_t)a.V + sh.token[c];
                g_p[c] = __ldg(a.p + at);
                g_q[c] = __ldg(a.q + at);
                g_u[c] = __ldg(a.uniforms + (size_t)b * N + c);
                atomicMin(&g_first[pu], c);
            }
            __syncthreads();
        }

        // ---- walk from the root
        int u = 0, len = 0, x = 0;
        double cur_c = 0.0, cur_z = 1.0;
        int last_pass_node = -1;
        double last_pass_c = -1.0;
        // From a node the walk has just reached (its distribution is still plain p),
        // follow every first child that passes its plain test; returns the node where
        // that stops, whose row the walk needs.  Every thread computes the same steps.
        auto descend = [&](int v) {
            if constexpr (!LOGITS) {
                while (a.gather) {
                    const int c = g_first[v];
                    if (c >= nn) break;
                    const double px = g_p[c], qx = g_q[c], r = g_u[c];
                    if (!(qx > 0.0 ? (r * qx < px) : (px > 0.0))) break;
                    if (rank == 0 && tid == 0) path_out[len] = c;
                    ++len;
                    v = c;
                }
            }
            return v;
        };
        u = descend(0);
        if (u != 0) {
            // the root's row (buffer 0) was not needed; this node's is
            x = 1;
            w.issue_row(x, u);
        }
        for (;;) {
            cur_c = 0.0;
            cur_z = 1.0;
            int accepted = -1;
            int scan = u + 1;
            if (LOGITS) {
                // even the first child's test needs the row's softmax normalisers
                w.wait_row(x);
                w.prep_row(x);
            }
            while (accepted < 0 && scan < nn) {
                // warp 0 collects the next (up to 32) children of u in ascending order with
                // their draft tokens' p, q and acceptance draws
                if (warp == 0) {
                    int found = 0, next = nn;
                    for (int c0 = scan; c0 < nn; c0 += 32) {
                        const int c = c0 + lane;
                        const bool kid = c < nn && sh.parent[c] == u;
                        const unsigned m = __ballot_sync(0xffffffffu, kid);
                        const int pos = found + __popc(m & ((1u << lane) - 1u));
                        if (kid && pos < 32) sh.ch_node[pos] = c;
                        if (found + __popc(m) > 32) {
                            // resume after the last child taken from this chunk
                            unsigned mm = m;
                            for (int t = 0; t < 32 - found; ++t) mm &= mm - 1u;
                            next = c0 + __ffs(mm) - 1;
                            found = 32;
                            break;
                        }
                        found += __popc(m);
                    }
                    __syncwarp();
                    if (lane < found) {
                        const int c = sh.ch_node[lane];
                        const size_t at = ((size_t)b * N + u) * (size_t)a.V + sh.token[c];
                        const float vp = a.gather ? g_p[c] : __ldg(a.p + at);
                        const float vq = a.gather ? g_q[c] : __ldg(a.q + at);
                        const float vu = a.gather ? g_u[c] : __ldg(a.uniforms + (size_t)b * N + c);
                        if (LOGITS) {
                            const float ep = expf(vp - sh.row_mp[x]);
                            const float eq = expf(vq - sh.row_mq[x]);
                            sh.ch_p[lane] = (double)(float)((double)ep * sh.row_zp_inv[x]);
                            sh.ch_q[lane] = (double)(float)((double)eq * sh.row_zq_inv[x]);
                        } else {
                            sh.ch_p[lane] = (double)vp;
                            sh.ch_q[lane] = (double)vq;
                        }
                        sh.ch_u[lane] = (double)vu;
                    }
                    if (lane == 0) {
                        sh.ch_n = found;
                        sh.ch_next = next;
                    }
                }
                __syncthreads();
                const int gn = sh.ch_n;
                for (int k = 0; k < gn; ++k) {
                    const double px = sh.ch_p[k], qx = sh.ch_q[k], r = sh.ch_u[k];
                    // r < num / (Z q(x)), compared without the fp64 division
                    const double num = cur_c == 0.0 ? px : pos_part(fma(-cur_c, qx, px));
                    const bool acc = qx > 0.0 ? (r * (cur_z * qx) < num) : (num > 0.0);
                    if (acc) {
                        accepted = sh.ch_node[k];
                        break;
                    }
                    w.wait_row(x);
                    const double c_new = cur_c + cur_z;
                    const double z_new = w.cluster_pass(x, c_new);
                    last_pass_node = u;
                    last_pass_c = c_new;
                    if (z_new > 0.0) {
                        cur_c = c_new;
                        cur_z = z_new;
                    }
                }
                scan = sh.ch_next;
                __syncthreads();  // ch_* are rewritten by the next batch
            }
            if (accepted < 0) break;
            if (rank == 0 && tid == 0) path_out[len] = accepted;
            ++len;
            u = descend(accepted);
            x ^= 1;
            w.issue_row(x, u);  // the row of the node where the walk goes on, into the other buffer
        }

        // ---- bonus token: first index whose running residual mass exceeds u0 * total
        w.wait_row(x);
        double total;
        if (last_pass_node == u && last_pass_c == cur_c) {
            total = cur_z;  // the last pass summed exactly this distribution; reuse its partials
        } else {
            total = w.cluster_pass(x, cur_c);
        }
        const int par = (w.passes - 1) & 1;
        const double target = (double)sh.u0 * total;
        // the CTA whose slice holds the crossing: every warp scans the C slice totals of the
        // last pass (one per lane), so every thread of every CTA gets the same owner
        const Crossing oc = first_crossing(lane < C ? sh.peer[par][lane] : 0.0, C, 0.0, target, lane);
        const bool fallback = oc.first < 0;
        const int owner = fallback ? oc.last_pos : oc.first;
        const double before = oc.before;

        if (rank == owner) {
            const float* pr = w.ps(x);
            const float* qr = w.qs(x);
            if (warp == 0) {
                // first warp segment whose running sum crosses the target; the last one
                // with mass if rounding leaves none (or the CTA was taken as a fallback)
                const Crossing wc = first_crossing(lane < nwarps ? sh.warp_part[lane] : 0.0, nwarps, before,
                                                   fallback ? INFINITY : target, lane);
                if (lane == 0) {
                    sh.wsel = wc.first >= 0 ? wc.first : wc.last_pos;
                    sh.wbefore = wc.first >= 0 ? wc.before : -INFINITY;  // -inf: the segment's last positive element
                    sh.found = -1;
                    sh.found_t = INT_MAX;
                }
            }
            __syncthreads();
            // the whole CTA scans the selected segment: each thread a run of at most a
            // few elements, then an inclusive scan over the threads (lanes, then warps)
            const int s0 = sh.wsel < 0 ? n : min(n, sh.wsel * w.segw), s1 = min(n, s0 + w.segw);
            const int per = (s1 - s0 + (int)blockDim.x - 1) / (int)blockDim.x;
            const int e0 = min(s1, s0 + tid * per), e1 = min(s1, e0 + per);
            double mine = 0.0;
            int mylast = -1;
            for (int i = e0; i < e1; ++i) {
                const double v = resid(pr[i], qr[i], cur_c);
                mine += v;
                if (v > 0.0) mylast = i;
            }
            double incl = mine;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const double t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            if (lane == 31) sh.warp_part2[warp] = incl;
            __syncthreads();
            {
                // this warp's offset: the running total of the warps before it
                const double inc = half_scan_d(lane < nwarps ? sh.warp_part2[lane] : 0.0, lane);
                const double prev = __shfl_sync(0xffffffffu, inc, warp > 0 ? warp - 1 : 0);
                incl += warp > 0 ? prev : 0.0;
            }
            const bool take_last = sh.wbefore == -INFINITY;
            // the first thread whose inclusive running sum exceeds the target holds the draw
            if (!take_last && sh.wbefore + incl > target) atomicMin(&sh.found_t, tid);
            if (mylast >= 0) atomicMax(&sh.found, mylast);  // the segment's last positive element
            __syncthreads();
            const int ft = sh.found_t;
            if (ft != INT_MAX && tid == ft) {
                double rsum = sh.wbefore + incl - mine;
                int pick = -1;
                for (int i = e0; i < e1; ++i) {
                    const double v = resid(pr[i], qr[i], cur_c);
                    if (v > 0.0) pick = i;
                    rsum += v;
                    if (rsum > target && v > 0.0) break;
                }
                sh.found = pick;
            }
            __syncthreads();
            if (tid == 0) {
                a.bonus[b] = sh.found >= 0 ? lo + sh.found : -1;
                a.len[b] = len;
            }
            for (int i = len + tid; i < N; i += blockDim.x) path_out[i] = -1;
        } else if (owner < 0 && rank == 0) {
            // no mass anywhere (an all-zero distribution)
            if (tid == 0) {
                a.bonus[b] = -1;
                a.len[b] = len;
            }
            for (int i = len + tid; i < N; i += blockDim.x) path_out[i] = -1;
        }
    }

    // ---- exit: no copy may still be landing in this CTA's shared memory, and no
    // peer may still send to it, when it retires
    w.wait_row(0);
    w.wait_row(1);
    if (C > 1) {
        __syncthreads();
        if (tid == 0) {
            const uint32_t bar = smem_u32(&sh.exit_bar);
            for (int k = 0; k < C; ++k) mbar_arrive_remote(mapa(bar, (uint32_t)k));
            const long long t0 = clock64();
            while (!mbar_try_cluster(bar, 0)) {
                if (clock64() - t0 > WAIT_LIMIT) {
                    sh.timeout = 1;
                    break;
                }
            }
            if (sh.timeout) {
                // exchanges were abandoned: give values a peer pushed before it stopped
                // time to land before this CTA's shared memory is released
                const long long t1 = clock64();
                while (clock64() - t1 < (1ll << 20)) {
                }
            }
        }
        __syncthreads();
    }
    if (tid == 0 && sh.timeout) report(a.status, TV_ERR_TIMEOUT);
}

}  // namespace

size_t sample_static_smem() { return sizeof(SampleShared); }

// The largest cluster (16 CTAs, else the portable 8) that the device can hold, found once per
// device: the answer and the function attributes set to find it belong to the current device.
namespace {
constexpr int MAX_DEVICES = 64;
std::mutex g_cluster_mutex;
int g_max_cluster[MAX_DEVICES] = {};  // 0: not yet found
}  // namespace

int sample_max_cluster() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) {
        cudaGetLastError();
        return 8;
    }
    std::lock_guard<std::mutex> lock(g_cluster_mutex);
    if (g_max_cluster[dev]) return g_max_cluster[dev];
    int best = 8;
    if (cudaFuncSetAttribute(verify_sample_kernel<false>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
            cudaSuccess &&
        cudaFuncSetAttribute(verify_sample_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, 160 * 1024) ==
            cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        cfg.gridDim = dim3(16, 1, 1);
        cfg.blockDim = dim3(MAX_THREADS, 1, 1);
        cfg.dynamicSmemBytes = 160 * 1024;
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 16;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&clusters, verify_sample_kernel<false>, &cfg) == cudaSuccess && clusters > 0)
            best = 16;
    }
    cudaGetLastError();
    g_max_cluster[dev] = best;
    return best;
}

cudaError_t launch_verify_sample(const SampleArgs& a, cudaStream_t st, int* launches) {
    void (*kern)(SampleArgs) = a.logits ? verify_sample_kernel<true> : verify_sample_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, a.smem_bytes);
    if (e != cudaSuccess) return e;
    if (a.cluster > 8) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    cfg.gridDim = dim3((unsigned)a.cluster * (unsigned)a.B, 1, 1);
    cfg.blockDim = dim3(a.threads, 1, 1);
    cfg.dynamicSmemBytes = a.smem_bytes;
    cfg.stream = st;
    // launch set-up may overlap the previous kernel's tail; the kernel waits for that
    // kernel (griddepcontrol.wait) before reading any input
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = a.cluster;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = a.cluster > 1 ? 2 : 1;
    *launches = 1;
    return cudaLaunchKernelEx(&cfg, kern, a);
}

}  // namespace tv
