// Fused token mixing + residual + LayerNorm, and the final LayerNorm + mean
// pooling.
//
// Token mixing with H = T heads (fun-rec chapter "Rankmixer: 硬件效率优化",
// section Token Mixing机制) sends chunk h of token t to position t*dh of output
// token h (dh = D / T), so every output row draws on every input row of the
// same sample.  Both kernels therefore stage one whole sample [T, D] in shared
// memory and apply the permutation through shared-memory addressing: X is read
// from HBM once and S is written once; no transpose pass touches HBM.
//
// Persistent CTAs walk the samples b = blockIdx.x, +gridDim.x, ...; one thread
// streams the next sample into the other half of a two-slot ring with a 1-D
// bulk copy (cp.async.bulk, completion on an mbarrier) while the CTA works on
// the current one.  All shared-memory and global accesses of the row phases
// are 16-byte vectors (8 bf16 or 4 fp32), consecutive lanes on consecutive
// columns.
//
// mix_ln:  Xh = PRE ? LN_pre(X) : X          (previous block's LN, row-wise)
//          Z[h, t*dh + j] = Xh[t, h*dh + j] + Xh[h, t*dh + j]
//          S[h, :] = LN1(Z[h, :])             (one warp per output row h)
//          or, without the Add & Norm after mixing, S[h, t*dh + j] = Xh[t, h*dh + j]
// ln_pool: Xh = LN(X);  pooled[b, :] = (1/T) sum_t Xh[t, :]  (ascending t)
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

// Mean and 1/sqrt(var + eps) of every row of the staged sample, one warp per
// row, from a single pass of sums shifted by the row's first element
// (var = E[(x-K)^2] - E[x-K]^2, which stays accurate while K is near the mean).
template <typename E>
__device__ __forceinline__ void row_stats(const E* xs, int T, int D, float eps, float* mean_s, float* rstd_s) {
    constexpr int V = Vec16<E>::N;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int nv = D / V;
    for (int t = warp; t < T; t += nw) {
        const E* r = xs + (size_t)t * D;
        const float K = to_f(r[0]);
        float s1 = 0.f, s2 = 0.f;
        for (int v = lane; v < nv; v += 32) {
            Vec16<E> x;
            x.u = *reinterpret_cast<const uint4*>(r + v * V);
#pragma unroll
            for (int e = 0; e < V; ++e) {
                const float d = to_f(x.e[e]) - K;
                s1 += d;
                s2 += d * d;
            }
        }
        s1 = warp_sum(s1);
        s2 = warp_sum(s2);
        if (lane == 0) {
            const float m1 = s1 / D;
            const float var = fmaxf(s2 / D - m1 * m1, 0.f);
            mean_s[t] = K + m1;
            rstd_s[t] = rsqrtf(var + eps);
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

template <typename E, bool PRE, bool CONTIG, int NV, bool ADDNORM>
__global__ void __launch_bounds__(NV >= 16 ? 256 : 512) mix_ln_kernel(const E* __restrict__ X, const float* __restrict__ pre_g,
                                                    const float* __restrict__ pre_b, const float* __restrict__ g1,
                                                    const float* __restrict__ b1, E* __restrict__ S, int B, int T,
                                                    int D, float eps, int nbuf, DeviceErr err, uint64_t budget_ns) {
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
    int it = 0;
    for (int b = blockIdx.x; b < B; b += gridDim.x, ++it) {
        const int cur = nbuf == 2 ? (it & 1) : 0;
        const int nb = b + gridDim.x;
        if (tid == 0) {
            if (nbuf == 2 && nb < B) ring.issue(cur ^ 1, X + (size_t)nb * TD);
            s_ok = ring.wait(cur, wc, SITE_MIX_LN);
        }
        __syncthreads();
        if (!s_ok) break;
        E* xs = ring.buf(cur);
        if (PRE) {
            // the previous block's LayerNorm, applied once per element, in place
            row_stats(xs, T, D, eps, mean_s, rstd_s);
            __syncthreads();
            normalize_in_place(xs, T, D, pre_g, pre_b, mean_s, rstd_s);
            __syncthreads();
        }
        E* srow = S + (size_t)b * TD;
        if (!ADDNORM) {
            // S = TokenMixing(Xh): a permutation of the (normalised) staged sample
            for (int h = warp; h < T; h += nw) {
                for (int v = lane; v < nv; v += 32) {
                    const int c0 = v * V;
                    Vec16<E> o;
                    if (CONTIG) {
                        const int t = c0 / dh, k0 = h * dh + (c0 - t * dh);
                        o.u = *reinterpret_cast<const uint4*>(xs + (size_t)t * D + k0);
                    } else {
                        int t = c0 / dh, j = c0 - t * dh;
#pragma unroll
                        for (int e = 0; e < V; ++e) {
                            o.e[e] = xs[(size_t)t * D + h * dh + j];
                            if (++j == dh) {
                                j = 0;
                                ++t;
                            }
                        }
                    }
                    *reinterpret_cast<uint4*>(srow + (size_t)h * D + c0) = o.u;
                }
            }
        }
        for (int h = warp; ADDNORM && h < T; h += nw) {
            float z[NV][V];
            float s = 0.f;
#pragma unroll
            for (int i = 0; i < NV; ++i) {
                const int v = lane + 32 * i;
                if (v < nv) {
                    const int c0 = v * V;
                    Vec16<E> xr;
                    xr.u = *reinterpret_cast<const uint4*>(xs + (size_t)h * D + c0);
                    if (CONTIG) {
                        // the V columns c0.. come from one source token t, contiguous there
                        const int t = c0 / dh, k0 = h * dh + (c0 - t * dh);
                        Vec16<E> xm;
                        xm.u = *reinterpret_cast<const uint4*>(xs + (size_t)t * D + k0);
#pragma unroll
                        for (int e = 0; e < V; ++e) {
                            z[i][e] = to_f(xm.e[e]) + to_f(xr.e[e]);
                            s += z[i][e];
                        }
                    } else {
                        int t = c0 / dh, j = c0 - t * dh;
#pragma unroll
                        for (int e = 0; e < V; ++e) {
                            z[i][e] = to_f(xs[(size_t)t * D + h * dh + j]) + to_f(xr.e[e]);
                            s += z[i][e];
                            if (++j == dh) {
                                j = 0;
                                ++t;
                            }
                        }
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

// Partial column sums of the pooling pass: row groups of ln_pool.
constexpr int kPoolGroups = 2;

template <typename E>
__global__ void __launch_bounds__(512) ln_pool_kernel(const E* __restrict__ X, const float* __restrict__ g,
                                                     const float* __restrict__ bta, float* __restrict__ pooled,
                                                     E* __restrict__ Xout, int B, int T, int D, float eps, int nbuf,
                                                     DeviceErr err, uint64_t budget_ns) {
    constexpr int V = Vec16<E>::N;
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ int abort_flag, s_ok;
    const int TD = T * D;
    float *mean_s, *rstd_s;
    SampleRing<E> ring = make_ring<E>(smem, TD, nbuf, mean_s, rstd_s, T);
    float* part = rstd_s + T;   // [kPoolGroups][D] partial sums of (x - m_t) r_t
    const int tid = threadIdx.x;
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
    const int groups = min(kPoolGroups, max(1, (int)blockDim.x / nv));
    const int grp = tid / nv;
    const float invT = 1.0f / T;
    int it = 0;
    for (int b = blockIdx.x; b < B; b += gridDim.x, ++it) {
        const int cur = nbuf == 2 ? (it & 1) : 0;
        const int nb = b + gridDim.x;
        if (tid == 0) {
            if (nbuf == 2 && nb < B) ring.issue(cur ^ 1, X + (size_t)nb * TD);
            s_ok = ring.wait(cur, wc, SITE_LN_POOL);
        }
        __syncthreads();
        if (!s_ok) break;
        const E* xs = ring.buf(cur);
        row_stats(xs, T, D, eps, mean_s, rstd_s);
        __syncthreads();
        // sum over this group's rows of (x - m_t) r_t, per column
        if (grp < groups) {
            for (int v = tid - grp * nv; v < nv; v += (groups == 1 ? blockDim.x : nv)) {
                const int c0 = v * V;
                float acc[V], gg[V], bb[V];
                if (Xout) {
                    load_params(g + c0, gg);
                    load_params(bta + c0, bb);
                }
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
#pragma unroll
                for (int e = 0; e < V; ++e) part[grp * D + c0 + e] = acc[e];
            }
        }
        __syncthreads();
        // pooled = (gamma * sum_t u_t + T beta) / T, partials added in group order
        for (int c = tid; c < D; c += blockDim.x) {
            float acc = 0.f;
            for (int q = 0; q < groups; ++q) acc += part[q * D + c];
            pooled[(size_t)b * D + c] = fmaf(__ldg(g + c), acc * invT, __ldg(bta + c));
        }
        __syncthreads();
        if (nbuf == 1 && tid == 0 && nb < B) ring.issue(0, X + (size_t)nb * TD);
    }
    if (tid == 0) ring.drain(wc, SITE_LN_POOL);
}

// Ring slots and dynamic shared memory for one sample of T*D elements.
// One slot per CTA once a sample is large enough that two CTAs (each with its
// own slot) fit an SM only that way: the co-resident CTA overlaps the loads.
inline void ring_shape(int T, int D, size_t esz, size_t extra_floats, int* nbuf, size_t* smem) {
    const size_t one = (size_t)T * D * esz;
    const size_t extra = 2 * sizeof(uint64_t) + sizeof(float) * (2 * (size_t)T + extra_floats);
    *nbuf = one <= 56 * 1024 ? 2 : 1;
    *smem = (size_t)(*nbuf) * one + extra;
}

template <typename K>
cudaError_t persistent_launch(K kernel, int threads, size_t smem, int B, int num_sms, cudaStream_t s, int* grid) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    long long g = (long long)num_sms * per_sm;
    *grid = (int)(g < B ? g : B);
    return cudaSuccess;
}

template <typename E, bool PRE, bool CONTIG, int NVV, bool ADDNORM = true>
cudaError_t mix_ln_go(const E* X, const float* pg, const float* pb, const float* g1, const float* b1, E* S, int B,
                      int T, int D, float eps, int num_sms, DeviceErr err, uint64_t budget, cudaStream_t s) {
    int nbuf;
    size_t smem;
    ring_shape(T, D, sizeof(E), 0, &nbuf, &smem);
    // one slot: 256 threads so that two CTAs fit an SM's registers as well
    const int threads = (NVV >= 16 || nbuf == 1 || T < 16) ? 256 : 512;
    auto k = mix_ln_kernel<E, PRE, CONTIG, NVV, ADDNORM>;
    int grid = 0;
    cudaError_t e = persistent_launch(k, threads, smem, B, num_sms, s, &grid);
    if (e != cudaSuccess) return e;
    k<<<grid, threads, smem, s>>>(X, pg, pb, g1, b1, S, B, T, D, eps, nbuf, err, budget);
    return cudaGetLastError();
}

template <typename E, bool PRE, bool CONTIG>
cudaError_t mix_ln_nv(int nvl, const E* X, const float* pg, const float* pb, const float* g1, const float* b1, E* S,
                      int B, int T, int D, float eps, int num_sms, DeviceErr err, uint64_t budget, cudaStream_t s) {
    if (nvl <= 1) return mix_ln_go<E, PRE, CONTIG, 1>(X, pg, pb, g1, b1, S, B, T, D, eps, num_sms, err, budget, s);
    if (nvl <= 2) return mix_ln_go<E, PRE, CONTIG, 2>(X, pg, pb, g1, b1, S, B, T, D, eps, num_sms, err, budget, s);
    if (nvl <= 4) return mix_ln_go<E, PRE, CONTIG, 4>(X, pg, pb, g1, b1, S, B, T, D, eps, num_sms, err, budget, s);
    if (nvl <= 8) return mix_ln_go<E, PRE, CONTIG, 8>(X, pg, pb, g1, b1, S, B, T, D, eps, num_sms, err, budget, s);
    if (nvl <= 16) return mix_ln_go<E, PRE, CONTIG, 16>(X, pg, pb, g1, b1, S, B, T, D, eps, num_sms, err, budget, s);
    return cudaErrorInvalidValue;
}

template <typename E>
cudaError_t mix_ln_typed(const void* X, const float* pg, const float* pb, const float* g1, const float* b1, void* S,
                         int B, int T, int D, float eps, int addnorm, int num_sms, DeviceErr err, uint64_t budget,
                         cudaStream_t s) {
    constexpr int V = Vec16<E>::N;
    const int nvl = (D / V + 31) / 32;
    const bool contig = ((D / T) % V) == 0;
    const E* x = static_cast<const E*>(X);
    E* y = static_cast<E*>(S);
    if (!addnorm) {
        if (pg)
            return contig ? mix_ln_go<E, true, true, 1, false>(x, pg, pb, g1, b1, y, B, T, D, eps, num_sms, err, budget, s)
                          : mix_ln_go<E, true, false, 1, false>(x, pg, pb, g1, b1, y, B, T, D, eps, num_sms, err, budget, s);
        return contig ? mix_ln_go<E, false, true, 1, false>(x, pg, pb, g1, b1, y, B, T, D, eps, num_sms, err, budget, s)
                      : mix_ln_go<E, false, false, 1, false>(x, pg, pb, g1, b1, y, B, T, D, eps, num_sms, err, budget, s);
    }
    if (pg)
        return contig ? mix_ln_nv<E, true, true>(nvl, x, pg, pb, g1, b1, y, B, T, D, eps, num_sms, err, budget, s)
                      : mix_ln_nv<E, true, false>(nvl, x, pg, pb, g1, b1, y, B, T, D, eps, num_sms, err, budget, s);
    return contig ? mix_ln_nv<E, false, true>(nvl, x, pg, pb, g1, b1, y, B, T, D, eps, num_sms, err, budget, s)
                  : mix_ln_nv<E, false, false>(nvl, x, pg, pb, g1, b1, y, B, T, D, eps, num_sms, err, budget, s);
}

template <typename E>
cudaError_t ln_pool_typed(const void* X, const float* g, const float* b, float* pooled, void* Xout, int B, int T,
                          int D, float eps, int num_sms, DeviceErr err, uint64_t budget, cudaStream_t s) {
    int nbuf;
    size_t smem;
    ring_shape(T, D, sizeof(E), (size_t)kPoolGroups * D, &nbuf, &smem);
    auto k = ln_pool_kernel<E>;
    int grid = 0;
    cudaError_t e = persistent_launch(k, 512, smem, B, num_sms, s, &grid);
    if (e != cudaSuccess) return e;
    k<<<grid, 512, smem, s>>>(static_cast<const E*>(X), g, b, pooled, static_cast<E*>(Xout), B, T, D, eps, nbuf, err,
                              budget);
    return cudaGetLastError();
}

}  // namespace

// Largest D per dtype the register-cached mix kernel supports (16 vectors per lane).
int mix_ln_max_d(int dtype) { return 32 * 16 * (dtype == RM_BF16 ? 8 : 4); }

cudaError_t launch_mix_ln(int dtype, const void* X, const float* pre_g, const float* pre_b, const float* g1,
                          const float* b1, void* S, int B, int T, int D, float eps, int addnorm, int num_sms,
                          DeviceErr err, uint64_t budget_ns, cudaStream_t s) {
    if (dtype == RM_BF16)
        return mix_ln_typed<__nv_bfloat16>(X, pre_g, pre_b, g1, b1, S, B, T, D, eps, addnorm, num_sms, err, budget_ns,
                                           s);
    return mix_ln_typed<float>(X, pre_g, pre_b, g1, b1, S, B, T, D, eps, addnorm, num_sms, err, budget_ns, s);
}

cudaError_t launch_ln_pool(int dtype, const void* X, const float* g, const float* b, float* pooled, void* Xout, int B,
                           int T, int D, float eps, int num_sms, DeviceErr err, uint64_t budget_ns, cudaStream_t s) {
    if (dtype == RM_BF16)
        return ln_pool_typed<__nv_bfloat16>(X, g, b, pooled, Xout, B, T, D, eps, num_sms, err, budget_ns, s);
    return ln_pool_typed<float>(X, g, b, pooled, Xout, B, T, D, eps, num_sms, err, budget_ns, s);
}

}  // namespace rm
