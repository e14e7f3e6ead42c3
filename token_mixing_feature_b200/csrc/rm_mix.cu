// Fused token mixing + residual + LayerNorm, the final LayerNorm + mean
// pooling, and row LayerNorm statistics.
//
// Token mixing with H = T heads (fun-rec chapter "Rankmixer: 硬件效率优化",
// section Token Mixing机制) sends chunk h of token t to position t*dh of output
// token h (dh = D / T).  Every output row of a sample reads a slice of every
// input row, so the sample is the unit of work: a persistent CTA stages whole
// samples ([T, D], contiguous) in shared memory with one cp.async.bulk each,
// into a two-slot ring when two samples fit (the next sample's copy overlaps
// the current one's arithmetic) and one slot otherwise (then two CTAs per SM
// overlap each other).  The permutation is applied through shared-memory
// addressing with 16-byte vectors, so X is read from HBM once and S written
// once, with no transpose pass; one warp owns one output row.
//
// The previous block's LayerNorm (PRE) uses row statistics produced where the
// row was written (the grouped GEMM's epilogue, the MoE combine, or
// row_stats_kernel) as partial (mean, M2) pairs over P column slices, merged
// here with Chan's pairwise formula -- no extra pass over the rows.
//
// mix_ln:  Xh = PRE ? LN_pre(X) : X                       (per token row)
//          Z[h, t*dh + j] = Xh[t, h*dh + j] + Xh[h, t*dh + j]
//          S[h, :] = LN1(Z[h, :])             (one warp per output row)
//          or, without the Add & Norm after mixing, S[h, t*dh + j] = Xh[t, h*dh + j]
// ln_pool: pooled[b, :] = (1/T) sum_t LN(X[b, t, :])  (ascending t)
#include <cuda_bf16.h>

#include "rm_device.cuh"

namespace rm {
namespace {

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

template <int N>
__device__ __forceinline__ void load_params(const float* __restrict__ p, float (&o)[N]) {
#pragma unroll
    for (int q = 0; q < N / 4; ++q) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(p) + q);
        o[4 * q + 0] = v.x;
        o[4 * q + 1] = v.y;
        o[4 * q + 2] = v.z;
        o[4 * q + 3] = v.w;
    }
}

// Two-slot ring of whole samples in shared memory (slot state kept in bit
// masks so nothing is indexed dynamically).
template <typename E>
struct SampleRing {
    unsigned char* base;   // slot s at base + s * bytes
    uint32_t bar0;         // mbarrier of slot s at bar0 + 8 * s
    int nbuf;
    uint32_t bytes;
    uint32_t outstanding;  // bit s: a copy into slot s was issued and not yet waited for
    uint32_t parity;       // bit s: parity of slot s's next completion

    __device__ __forceinline__ E* buf(int slot) const { return reinterpret_cast<E*>(base + (size_t)slot * bytes); }
    __device__ __forceinline__ uint32_t bar(int slot) const { return bar0 + 8u * (uint32_t)slot; }

    __device__ void issue(int slot, const E* src) {   // thread 0 only
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(bar(slot), bytes);
        bulk_load(smem_u32(buf(slot)), src, bytes, bar(slot));
        outstanding |= 1u << slot;
    }
    // thread 0 only: wait for the copy in `slot`; false if it ran out.
    __device__ bool wait(int slot, const WaitCtx& wc, int site) {
        const bool ok = mbar_wait(bar(slot), (parity >> slot) & 1u, wc, site, false);
        if (ok) {
            outstanding &= ~(1u << slot);
            parity ^= 1u << slot;
        }
        return ok;
    }
    // thread 0 only: let every copy still in flight land before the CTA exits.
    __device__ void drain(const WaitCtx& wc, int site) {
        for (int s = 0; s < nbuf; ++s)
            if ((outstanding >> s) & 1u) mbar_wait(bar(s), (parity >> s) & 1u, wc, site, false);
    }
};

// Carves the ring and the per-row statistics out of dynamic shared memory.
template <typename E>
__device__ __forceinline__ SampleRing<E> make_ring(unsigned char* smem, int TD, int nbuf, float*& mean_s,
                                                   float*& rstd_s, int T) {
    SampleRing<E> r;
    r.bytes = (uint32_t)((size_t)TD * sizeof(E));
    r.nbuf = nbuf;
    r.base = smem;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)nbuf * r.bytes);
    r.bar0 = smem_u32(bars);
    r.outstanding = 0;
    r.parity = 0;
    mean_s = reinterpret_cast<float*>(bars + 2);
    rstd_s = mean_s + T;
    return r;
}

// Merge partial statistics (count, mean, M2) b into a (Chan et al.).
__device__ __forceinline__ void stats_merge(float& na, float& ma, float& qa, float nb, float mb, float qb) {
    if (nb == 0.f) return;
    if (na == 0.f) {
        na = nb;
        ma = mb;
        qa = qb;
        return;
    }
    const float n = na + nb, d = mb - ma, f = nb / n;
    ma += d * f;
    qa += qb + d * d * na * f;
    na = n;
}

// Mean and 1/sqrt(var + eps) of row `row` from its P partials (each over
// D/P columns); the warp merges lane-strided partials, then a fixed
// shfl_down tree (deterministic).  Result valid in every lane.
__device__ __forceinline__ void row_mean_rstd(const float2* __restrict__ part, int P, int D, long long row, float eps,
                                              float& mean, float& rstd) {
    const int lane = threadIdx.x & 31;
    const float per = (float)D / (float)P;
    float n = 0.f, m = 0.f, q = 0.f;
    for (int p = lane; p < P; p += 32) {
        const float2 v = __ldg(part + row * P + p);
        stats_merge(n, m, q, per, v.x, v.y);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float nb = __shfl_down_sync(0xffffffffu, n, o);
        const float mb = __shfl_down_sync(0xffffffffu, m, o);
        const float qb = __shfl_down_sync(0xffffffffu, q, o);
        if (lane < o) stats_merge(n, m, q, nb, mb, qb);
    }
    mean = __shfl_sync(0xffffffffu, m, 0);
    rstd = rsqrtf(__shfl_sync(0xffffffffu, q, 0) / D + eps);
}

// Columns c0 .. c0+V-1 of output row h, mixed term: source token t = c / dh,
// column h*dh + c - t*dh.  `mixed` holds columns [h0*dh, (h0+R)*dh) of every
// row t with row stride rs = R*dh, so the element is mixed[t*rs + hoff + j]
// with hoff = (h-h0)*dh.  MV = elements per contiguous piece: V (one 16-byte
// load), V/2 (8-byte loads) or 1.
template <typename E, int MV>
__device__ __forceinline__ void load_mixed(const E* mixed, int rs, int hoff, int dh, int c0, Vec16<E>& o) {
    constexpr int V = Vec16<E>::N;
    if constexpr (MV == V) {
        const int t = c0 / dh;
        o.u = *reinterpret_cast<const uint4*>(mixed + (size_t)t * rs + hoff + (c0 - t * dh));
    } else if constexpr (MV * sizeof(E) == 8) {
#pragma unroll
        for (int sv = 0; sv < V / MV; ++sv) {
            const int c = c0 + sv * MV, t = c / dh;
            const uint2 q = *reinterpret_cast<const uint2*>(mixed + (size_t)t * rs + hoff + (c - t * dh));
            if (sv == 0) {
                o.u.x = q.x;
                o.u.y = q.y;
            } else {
                o.u.z = q.x;
                o.u.w = q.y;
            }
        }
    } else {
        int t = c0 / dh, j = c0 - t * dh;
#pragma unroll
        for (int e = 0; e < V; ++e) {
            o.e[e] = mixed[(size_t)t * rs + hoff + j];
            if (++j == dh) {
                j = 0;
                ++t;
            }
        }
    }
}

// In-place LayerNorm of the staged sample (row statistics already in shared
// memory).  Thread i owns column vector i % nv and walks the rows of its row
// group, so each thread loads its columns' gamma/beta once per sample.
template <typename E>
__device__ __forceinline__ void normalize_in_place(E* xs, int T, int D, const float* __restrict__ g,
                                                   const float* __restrict__ bta, const float* mean_s,
                                                   const float* rstd_s) {
    constexpr int V = Vec16<E>::N;
    const int nv = D / V;
    const int groups = max(1, (int)blockDim.x / nv);
    const int grp = threadIdx.x / nv;
    if (grp >= groups) return;
    for (int v = threadIdx.x - grp * nv; v < nv; v += (groups == 1 ? blockDim.x : nv)) {
        const int c0 = v * V;
        float gg[V], bb[V];
        load_params(g + c0, gg);
        load_params(bta + c0, bb);
        for (int t = grp; t < T; t += groups) {
            uint4* p = reinterpret_cast<uint4*>(xs + (size_t)t * D + c0);
            Vec16<E> x;
            x.u = *p;
            const float m = mean_s[t], r = rstd_s[t];
#pragma unroll
            for (int e = 0; e < V; ++e) x.e[e] = from_f<E>(fmaf((to_f(x.e[e]) - m) * r, gg[e], bb[e]));
            *p = x.u;
        }
    }
}

template <typename E, bool PRE, int MV, int NV, bool ADDNORM>
__global__ void __launch_bounds__(NV >= 16 ? 256 : 512) mix_ln_kernel(
    const E* __restrict__ X, const float* __restrict__ pre_g, const float* __restrict__ pre_b,
    const float2* __restrict__ pstats, int P, const float* __restrict__ g1, const float* __restrict__ b1,
    E* __restrict__ S, int B, int T, int D, float eps, int nbuf, DeviceErr err, uint64_t budget_ns) {
    constexpr int V = Vec16<E>::N;
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ int abort_flag, s_ok;
    const int TD = T * D;
    float *mean_s, *rstd_s;
    SampleRing<E> ring = make_ring<E>(smem, TD, nbuf, mean_s, rstd_s, T);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    const WaitCtx wc{&abort_flag, budget_ns, err};
    if (tid == 0) {
        mbar_init(ring.bar(0), 1);
        mbar_init(ring.bar(1), 1);
        abort_flag = 0;
        fence_mbar_init();
        if (blockIdx.x < B) ring.issue(0, X + (size_t)blockIdx.x * TD);
    }
    __syncthreads();
    const int dh = D / T;
    const int nv = D / V;
    // Whole-vector pieces: the mixed vector i of output row h sits at
    // moff[i] + h*dh (its source token t = c0/dh does not depend on h).
    int moff[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int c0 = (lane + 32 * i) * V, t = c0 / dh;
        moff[i] = t * (D - dh) + c0;
    }
    int it = 0;
    for (int b = blockIdx.x; b < B; b += gridDim.x, ++it) {
        const int cur = nbuf == 2 ? (it & 1) : 0;
        const int nb = b + gridDim.x;
        if (PRE) {   // statistics of this sample's rows, from the producer's partials
            for (int t = warp; t < T; t += nw) {
                float m, r;
                row_mean_rstd(pstats, P, D, (long long)b * T + t, eps, m, r);
                if (lane == 0) {
                    mean_s[t] = m;
                    rstd_s[t] = r;
                }
            }
        }
        if (tid == 0) {
            if (nbuf == 2 && nb < B) ring.issue(cur ^ 1, X + (size_t)nb * TD);
            s_ok = ring.wait(cur, wc, SITE_MIX_LN);
        }
        __syncthreads();
        if (!s_ok) break;
        E* xs = ring.buf(cur);
        if (PRE) {
            // the previous block's LayerNorm, applied once per element, in place
            normalize_in_place(xs, T, D, pre_g, pre_b, mean_s, rstd_s);
            __syncthreads();
        }
        E* srow = S + (size_t)b * TD;
        for (int h = warp; h < T; h += nw) {
            const int hoff = h * dh;
            if (!ADDNORM) {   // S = TokenMixing(Xh): a permutation of the staged sample
                for (int v = lane; v < nv; v += 32) {
                    Vec16<E> o;
                    load_mixed<E, MV>(xs, D, hoff, dh, v * V, o);
                    *reinterpret_cast<uint4*>(srow + (size_t)h * D + v * V) = o.u;
                }
                continue;
            }
            float z[NV][V];
            float s = 0.f;
#pragma unroll
            for (int i = 0; i < NV; ++i) {
                const int v = lane + 32 * i;
                if (v < nv) {
                    const int c0 = v * V;
                    Vec16<E> xr, xm;
                    xr.u = *reinterpret_cast<const uint4*>(xs + (size_t)h * D + c0);
                    if constexpr (MV == V)
                        xm.u = *reinterpret_cast<const uint4*>(xs + moff[i] + hoff);
                    else
                        load_mixed<E, MV>(xs, D, hoff, dh, c0, xm);
#pragma unroll
                    for (int e = 0; e < V; ++e) {
                        z[i][e] = to_f(xm.e[e]) + to_f(xr.e[e]);
                        s += z[i][e];
                    }
                }
            }
            const float mu = warp_sum(s) / D;
            float q = 0.f;
#pragma unroll
            for (int i = 0; i < NV; ++i) {
                if (lane + 32 * i < nv) {
#pragma unroll
                    for (int e = 0; e < V; ++e) {
                        const float d = z[i][e] - mu;
                        q = fmaf(d, d, q);
                    }
                }
            }
            const float rstd = rsqrtf(warp_sum(q) / D + eps);
#pragma unroll
            for (int i = 0; i < NV; ++i) {
                const int v = lane + 32 * i;
                if (v < nv) {
                    const int c0 = v * V;
                    float gg[V], bb[V];
                    load_params(g1 + c0, gg);
                    load_params(b1 + c0, bb);
                    Vec16<E> o;
#pragma unroll
                    for (int e = 0; e < V; ++e) o.e[e] = from_f<E>(fmaf((z[i][e] - mu) * rstd, gg[e], bb[e]));
                    *reinterpret_cast<uint4*>(srow + (size_t)h * D + c0) = o.u;
                }
            }
        }
        __syncthreads();   // the slot and the statistics are free again
        if (nbuf == 1 && tid == 0 && nb < B) ring.issue(0, X + (size_t)nb * TD);
    }
    if (tid == 0) ring.drain(wc, SITE_MIX_LN);
}

// pooled[b, c] = gamma[c] * (1/T) sum_t (x[t, c] - m_t) r_t + beta[c]; Xout
// (optional) receives LN(x).  Persistent CTAs stage whole samples in the same
// shared-memory ring as mix_ln (one bulk copy per sample: far more bytes in
// flight than per-thread loads).  The threads form `groups` row groups of
// nv = D/V column-vector threads; group q sums rows q, q+groups, ... and the
// groups' partial sums are added in ascending q (deterministic).
constexpr int kPoolThreads = 512;
constexpr size_t kMaxSmemPerCta = 227 * 1024;

template <typename E>
__global__ void __launch_bounds__(kPoolThreads) ln_pool_kernel(const E* __restrict__ X,
                                                              const float2* __restrict__ pstats, int P,
                                                              const float* __restrict__ g,
                                                              const float* __restrict__ bta,
                                                              float* __restrict__ pooled, E* __restrict__ Xout,
                                                              int B, int T, int D, float eps, int nbuf, int groups,
                                                              DeviceErr err, uint64_t budget_ns) {
    constexpr int V = Vec16<E>::N;
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ int abort_flag, s_ok;
    const int TD = T * D;
    float *mean_s, *rstd_s;
    SampleRing<E> ring = make_ring<E>(smem, TD, nbuf, mean_s, rstd_s, T);
    float* part = rstd_s + T;   // [groups][D] partial sums of (x - m_t) r_t
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    const WaitCtx wc{&abort_flag, budget_ns, err};
    if (tid == 0) {
        mbar_init(ring.bar(0), 1);
        mbar_init(ring.bar(1), 1);
        abort_flag = 0;
        fence_mbar_init();
        if (blockIdx.x < B) ring.issue(0, X + (size_t)blockIdx.x * TD);
    }
    __syncthreads();
    const int nv = D / V;
    const int grp = tid / nv, v = tid - grp * nv, c0 = v * V;
    const float invT = 1.0f / T;
    float gg[V], bb[V];
    if (Xout && grp < groups) {
        load_params(g + c0, gg);
        load_params(bta + c0, bb);
    }
    int it = 0;
    for (int b = blockIdx.x; b < B; b += gridDim.x, ++it) {
        const int cur = nbuf == 2 ? (it & 1) : 0;
        const int nb = b + gridDim.x;
        for (int t = warp; t < T; t += nw) {
            float m, r;
            row_mean_rstd(pstats, P, D, (long long)b * T + t, eps, m, r);
            if (lane == 0) {
                mean_s[t] = m;
                rstd_s[t] = r;
            }
        }
        if (tid == 0) {
            if (nbuf == 2 && nb < B) ring.issue(cur ^ 1, X + (size_t)nb * TD);
            s_ok = ring.wait(cur, wc, SITE_LN_POOL);
        }
        __syncthreads();
        if (!s_ok) break;
        const E* xs = ring.buf(cur);
        if (grp < groups) {
            float acc[V];
#pragma unroll
            for (int e = 0; e < V; ++e) acc[e] = 0.f;
            for (int t = grp; t < T; t += groups) {
                Vec16<E> x;
                x.u = *reinterpret_cast<const uint4*>(xs + (size_t)t * D + c0);
                const float mt = mean_s[t], rt = rstd_s[t];
                Vec16<E> o;
#pragma unroll
                for (int e = 0; e < V; ++e) {
                    const float u = (to_f(x.e[e]) - mt) * rt;
                    acc[e] += u;
                    if (Xout) o.e[e] = from_f<E>(fmaf(u, gg[e], bb[e]));
                }
                if (Xout) *reinterpret_cast<uint4*>(Xout + (size_t)b * TD + (size_t)t * D + c0) = o.u;
            }
            float4* dst = reinterpret_cast<float4*>(part + (size_t)grp * D + c0);
#pragma unroll
            for (int q = 0; q < V / 4; ++q)
                dst[q] = make_float4(acc[4 * q], acc[4 * q + 1], acc[4 * q + 2], acc[4 * q + 3]);
        }
        __syncthreads();
        for (int c = tid; c < D; c += blockDim.x) {
            float a = part[c];
            for (int q = 1; q < groups; ++q) a += part[(size_t)q * D + c];
            pooled[(size_t)b * D + c] = fmaf(__ldg(g + c), a * invT, __ldg(bta + c));
        }
        __syncthreads();   // slot, statistics and partials are free again
        if (nbuf == 1 && tid == 0 && nb < B) ring.issue(0, X + (size_t)nb * TD);
    }
    if (tid == 0) ring.drain(wc, SITE_LN_POOL);
}

// (mean, M2) of every row over all D columns (P = 1), one warp per row, one
// pass of sums shifted by the row's first element.
template <typename E>
__global__ void __launch_bounds__(256) row_stats_kernel(const E* __restrict__ X, float2* __restrict__ out,
                                                       long long rows, int D) {
    constexpr int V = Vec16<E>::N;
    const int lane = threadIdx.x & 31;
    const long long r = blockIdx.x * (long long)(blockDim.x >> 5) + (threadIdx.x >> 5);
    if (r >= rows) return;
    const E* x = X + r * D;
    const float K = to_f(x[0]);
    float s1 = 0.f, s2 = 0.f;
    for (int v = lane; v < D / V; v += 32) {
        Vec16<E> u;
        u.u = __ldg(reinterpret_cast<const uint4*>(x) + v);
#pragma unroll
        for (int e = 0; e < V; ++e) {
            const float d = to_f(u.e[e]) - K;
            s1 += d;
            s2 = fmaf(d, d, s2);
        }
    }
    s1 = warp_sum(s1);
    s2 = warp_sum(s2);
    if (lane == 0) out[r] = make_float2(K + s1 / D, fmaxf(s2 - s1 * s1 / D, 0.f));
}

// One slot per CTA once a sample is large enough that two CTAs (each with its
// own slot) fit an SM only that way: the co-resident CTA overlaps the loads.
inline void ring_shape(int T, int D, size_t esz, size_t extra_floats, int* nbuf, size_t* smem) {
    const size_t one = (size_t)T * D * esz;
    const size_t extra = 2 * sizeof(uint64_t) + sizeof(float) * (2 * (size_t)T + extra_floats);
    *nbuf = one <= 56 * 1024 ? 2 : 1;
    *smem = (size_t)(*nbuf) * one + extra;
}

template <typename E, bool PRE, int MV, int NVV, bool ADDNORM>
cudaError_t mix_ln_go(const E* X, const float* pg, const float* pb, RowStats ps, const float* g1, const float* b1,
                      E* S, int B, int T, int D, float eps, int num_sms, DeviceErr err, uint64_t budget,
                      cudaStream_t s) {
    int nbuf;
    size_t smem;
    ring_shape(T, D, sizeof(E), 0, &nbuf, &smem);
    // one slot: 256 threads so that two CTAs fit an SM's registers as well
    const int threads = (NVV >= 16 || nbuf == 1 || T < 16) ? 256 : 512;
    auto k = mix_ln_kernel<E, PRE, MV, NVV, ADDNORM>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, threads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const long long g = (long long)num_sms * per_sm;
    const int grid = (int)(g < B ? g : B);
    k<<<grid, threads, smem, s>>>(X, pg, pb, ps.part, ps.P, g1, b1, S, B, T, D, eps, nbuf, err, budget);
    return cudaGetLastError();
}

template <typename E, bool PRE, int MV>
cudaError_t mix_ln_nv(int nvl, int addnorm, const E* X, const float* pg, const float* pb, RowStats ps,
                      const float* g1, const float* b1, E* S, int B, int T, int D, float eps, int num_sms,
                      DeviceErr err, uint64_t budget, cudaStream_t s) {
    if (!addnorm) return mix_ln_go<E, PRE, MV, 1, false>(X, pg, pb, ps, g1, b1, S, B, T, D, eps, num_sms, err, budget, s);
    if (nvl <= 1) return mix_ln_go<E, PRE, MV, 1, true>(X, pg, pb, ps, g1, b1, S, B, T, D, eps, num_sms, err, budget, s);
    if (nvl <= 2) return mix_ln_go<E, PRE, MV, 2, true>(X, pg, pb, ps, g1, b1, S, B, T, D, eps, num_sms, err, budget, s);
    if (nvl <= 4) return mix_ln_go<E, PRE, MV, 4, true>(X, pg, pb, ps, g1, b1, S, B, T, D, eps, num_sms, err, budget, s);
    if (nvl <= 6) return mix_ln_go<E, PRE, MV, 6, true>(X, pg, pb, ps, g1, b1, S, B, T, D, eps, num_sms, err, budget, s);
    if (nvl <= 8) return mix_ln_go<E, PRE, MV, 8, true>(X, pg, pb, ps, g1, b1, S, B, T, D, eps, num_sms, err, budget, s);
    return cudaErrorInvalidValue;
}

template <typename E>
cudaError_t mix_ln_typed(const void* X, const float* pg, const float* pb, RowStats ps, const float* g1,
                         const float* b1, void* S, int B, int T, int D, float eps, int addnorm, int num_sms,
                         DeviceErr err, uint64_t budget, cudaStream_t s) {
    constexpr int V = Vec16<E>::N;
    const int nvl = (D / V + 31) / 32;
    const int dh = D / T;
    const int mv = dh % V == 0 ? V : (dh % (V / 2) == 0 ? V / 2 : 1);
    const E* x = static_cast<const E*>(X);
    E* y = static_cast<E*>(S);
#define RM_MIX_MV(PREV, MVV) \
    mix_ln_nv<E, PREV, MVV>(nvl, addnorm, x, pg, pb, ps, g1, b1, y, B, T, D, eps, num_sms, err, budget, s)
#define RM_MIX_PRE(PREV) (mv == V ? RM_MIX_MV(PREV, V) : mv == V / 2 ? RM_MIX_MV(PREV, V / 2) : RM_MIX_MV(PREV, 1))
    const cudaError_t e = pg ? RM_MIX_PRE(true) : RM_MIX_PRE(false);
#undef RM_MIX_PRE
#undef RM_MIX_MV
    return e;
}

template <typename E>
cudaError_t ln_pool_go(const void* X, RowStats stats, const float* g, const float* b, float* pooled, void* Xout, int B,
                       int T, int D, float eps, int num_sms, DeviceErr err, uint64_t budget, cudaStream_t s) {
    constexpr int V = Vec16<E>::N;
    const int nv = D / V;
    if (nv < 1 || nv > kPoolThreads) return cudaErrorInvalidValue;
    int groups = kPoolThreads / nv;
    if (groups > T) groups = T;
    int nbuf;
    size_t smem;
    ring_shape(T, D, sizeof(E), (size_t)groups * D, &nbuf, &smem);
    while (groups > 1 && smem > kMaxSmemPerCta) {   // large samples: fewer row groups
        --groups;
        ring_shape(T, D, sizeof(E), (size_t)groups * D, &nbuf, &smem);
    }
    auto k = ln_pool_kernel<E>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, kPoolThreads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const long long gr = (long long)num_sms * per_sm;
    const int grid = (int)(gr < B ? gr : B);
    k<<<grid, kPoolThreads, smem, s>>>(static_cast<const E*>(X), stats.part, stats.P, g, b, pooled, static_cast<E*>(Xout),
                                       B, T, D, eps, nbuf, groups, err, budget);
    return cudaGetLastError();
}

}  // namespace

// Largest D per dtype the register-cached mix kernel supports (8 vectors per lane).
int mix_ln_max_d(int dtype) { return 32 * 8 * (dtype == RM_BF16 ? 8 : 4); }

cudaError_t launch_mix_ln(int dtype, const void* X, const float* pre_g, const float* pre_b, RowStats pre_stats,
                          const float* g1, const float* b1, void* S, int B, int T, int D, float eps, int addnorm,
                          int num_sms, DeviceErr err, uint64_t budget_ns, cudaStream_t s) {
    if (pre_g && !pre_stats.part) return cudaErrorInvalidValue;
    if (dtype == RM_BF16)
        return mix_ln_typed<__nv_bfloat16>(X, pre_g, pre_b, pre_stats, g1, b1, S, B, T, D, eps, addnorm, num_sms,
                                           err, budget_ns, s);
    return mix_ln_typed<float>(X, pre_g, pre_b, pre_stats, g1, b1, S, B, T, D, eps, addnorm, num_sms, err,
                               budget_ns, s);
}

cudaError_t launch_ln_pool(int dtype, const void* X, RowStats stats, const float* g, const float* b, float* pooled,
                           void* Xout, int B, int T, int D, float eps, int num_sms, DeviceErr err, uint64_t budget_ns,
                           cudaStream_t s) {
    if (dtype == RM_BF16)
        return ln_pool_go<__nv_bfloat16>(X, stats, g, b, pooled, Xout, B, T, D, eps, num_sms, err, budget_ns, s);
    return ln_pool_go<float>(X, stats, g, b, pooled, Xout, B, T, D, eps, num_sms, err, budget_ns, s);
}

cudaError_t launch_row_stats(int dtype, const void* X, float2* out, long long rows, int D, cudaStream_t s) {
    const int grid = (int)((rows + 7) / 8);
    if (dtype == RM_BF16)
        row_stats_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(X), out, rows, D);
    else
        row_stats_kernel<float><<<grid, 256, 0, s>>>(static_cast<const float*>(X), out, rows, D);
    return cudaGetLastError();
}

}  // namespace rm
