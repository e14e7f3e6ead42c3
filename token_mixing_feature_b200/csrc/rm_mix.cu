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

template <int NP>
__device__ __forceinline__ void load_pairs(const float* __restrict__ p, float2 (&o)[NP]) {
#pragma unroll
    for (int q = 0; q < NP / 2; ++q) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(p) + q);
        o[2 * q] = make_float2(v.x, v.y);
        o[2 * q + 1] = make_float2(v.z, v.w);
    }
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

// Ring of whole samples in shared memory.  Slot s holds one sample's T rows
// at a row stride of rs >= D elements; it fills from one cp.async.bulk copy
// (rs == D) or T row copies issued by the lanes of warp 0, on the slot's
// mbarrier.  Slot bookkeeping lives in bit masks in lane 0 of warp 0.
constexpr int kMaxSlots = 4;

template <typename E>
struct SampleRing {
    unsigned char* base;   // slot s at base + s * slot_bytes
    uint32_t bar0;         // mbarrier of slot s at bar0 + 8 * s
    int nslots, T, D, rs;
    uint32_t slot_bytes;
    uint32_t outstanding;  // bit s: a copy into slot s was issued and not yet waited for
    uint32_t parity;       // bit s: parity of slot s's next completion

    __device__ __forceinline__ E* buf(int slot) const { return reinterpret_cast<E*>(base + (size_t)slot * slot_bytes); }
    __device__ __forceinline__ uint32_t bar(int slot) const { return bar0 + 8u * (uint32_t)slot; }

    // all lanes of warp 0: sample src [T, D] (contiguous) into `slot`
    __device__ void issue(int slot, const E* src) {
        const int lane = threadIdx.x & 31;
        const uint32_t row_bytes = (uint32_t)(D * sizeof(E));
        if (lane == 0) {
            mbar_arrive_expect_tx(bar(slot), row_bytes * (uint32_t)T);
            outstanding |= 1u << slot;
        }
        __syncwarp();
        fence_proxy_async_smem();   // earlier generic accesses to the slot come first
        const uint32_t dst = smem_u32(buf(slot));
        if (rs == D) {   // unpadded rows: the sample is one contiguous copy
            if (lane == 0) bulk_load(dst, src, row_bytes * (uint32_t)T, bar(slot));
            return;
        }
        for (int r = lane; r < T; r += 32)
            bulk_load(dst + (uint32_t)(r * rs) * (uint32_t)sizeof(E), src + (size_t)r * D, row_bytes, bar(slot));
    }
    // thread 0 only: wait for the copies into `slot`; false if the wait ran out.
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
        for (int s = 0; s < nslots; ++s)
            if ((outstanding >> s) & 1u) mbar_wait(bar(s), (parity >> s) & 1u, wc, site, false);
    }
};

// Bytes of one ring slot (128-byte multiple).
inline __host__ __device__ size_t slot_bytes_of(int T, int rs, size_t esz) {
    return ((size_t)T * rs * esz + 127) / 128 * 128;
}

// Carves the ring (nslots slots), its barriers and the per-row statistics
// (mean_s[T], rstd_s[T]) out of dynamic shared memory; returns the first
// float after them.
template <typename E>
__device__ __forceinline__ float* make_ring(SampleRing<E>& r, unsigned char* smem, int T, int D, int rs, int nslots,
                                            float*& mean_s, float*& rstd_s) {
    r.slot_bytes = (uint32_t)slot_bytes_of(T, rs, sizeof(E));
    r.nslots = nslots;
    r.T = T;
    r.D = D;
    r.rs = rs;
    r.base = smem;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)nslots * r.slot_bytes);
    r.bar0 = smem_u32(bars);
    r.outstanding = 0;
    r.parity = 0;
    mean_s = reinterpret_cast<float*>(bars + kMaxSlots);
    rstd_s = mean_s + T;
    return rstd_s + T;
}

// Row stride of the staged sample for the mixing kernel: D plus a pad that
// makes consecutive token rows start (dh - D) * esz bytes apart modulo 128,
// so the 16-byte pieces that consecutive lanes gather from consecutive token
// rows fall in consecutive banks.  Only for whole-vector pieces.
inline int mix_row_stride(int D, int dh, size_t esz) {
    const long long bytes = (long long)dh * (long long)esz;
    if (bytes % 16) return D;
    long long pad = ((long long)(dh - D) * (long long)esz) % 128;
    if (pad < 0) pad += 128;
    return D + (int)(pad / (long long)esz);
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

// Threads of the mixing kernel form `groups` row groups of nv = D/V
// column-vector threads: thread (grp, v) owns columns [v*V, v*V + V) of rows
// grp, grp + groups, ... in the element-wise passes, so the source offset of
// its mixed vector and its gamma/beta stay in registers.
constexpr int kMixMaxThreads = 384;

// In-place LayerNorm of the staged sample (row statistics in shared memory),
// in fp32 pairs: y = ((x r) - m r) gamma + beta.
template <typename E>
__device__ __forceinline__ void normalize_in_place(E* xs, int T, int rs, int c0, int grp, int groups,
                                                   const float* __restrict__ g, const float* __restrict__ bta,
                                                   const float* mean_s, const float* rstd_s) {
    constexpr int NP = Vec16<E>::N / 2;
    float2 gp[NP], bp[NP];
    load_pairs(g + c0, gp);
    load_pairs(bta + c0, bp);
#pragma unroll 2
    for (int t = grp; t < T; t += groups) {
        uint4* p = reinterpret_cast<uint4*>(xs + (size_t)t * rs + c0);
        float2 x[NP];
        unpack_pairs(*p, x);
        const float r = rstd_s[t];
        const float2 r2 = f2(r), mr2 = f2(-mean_s[t] * r);
#pragma unroll
        for (int j = 0; j < NP; ++j) x[j] = f2_fma(f2_fma(x[j], r2, mr2), gp[j], bp[j]);
        *p = pack_pairs(x);
    }
}

// Mixed vector of output row h at column c0 of a sample staged at row stride
// rs: whole-vector pieces come from a precomputed h-independent offset
// moff = t (rs - dh) + c0 (source token t = c0/dh), others piecewise.
template <typename E, int MV>
__device__ __forceinline__ void mixed_vec(const E* xs, int rs, int dh, int h, int c0, int moff, Vec16<E>& o) {
    constexpr int V = Vec16<E>::N;
    if constexpr (MV == V)
        o.u = *reinterpret_cast<const uint4*>(xs + moff + h * dh);
    else
        load_mixed<E, MV>(xs, rs, h * dh, dh, c0, o);
}

template <typename E, bool PRE, int MV, int NV, bool ADDNORM>
__global__ void __launch_bounds__(kMixMaxThreads, 2) mix_ln_kernel(
    const E* __restrict__ X, const float* __restrict__ pre_g, const float* __restrict__ pre_b,
    const float2* __restrict__ pstats, int P, const float* __restrict__ g1, const float* __restrict__ b1,
    E* __restrict__ S, int B, int T, int D, float eps, int rs, int nslots, int groups, DeviceErr err,
    uint64_t budget_ns) {
    constexpr int V = Vec16<E>::N;
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ int abort_flag, s_ok;
    const int TD = T * D;
    float *mean_s, *rstd_s;
    SampleRing<E> ring;
    make_ring<E>(ring, smem, T, D, rs, nslots, mean_s, rstd_s);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    const WaitCtx wc{&abort_flag, budget_ns, err};
    if (tid == 0) {
        for (int k = 0; k < nslots; ++k) mbar_init(ring.bar(k), 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (warp == 0)
        for (int k = 0; k < nslots; ++k) {
            const long long bk = blockIdx.x + (long long)k * gridDim.x;
            if (bk < B) ring.issue(k, X + (size_t)bk * TD);
        }
    const int dh = D / T;
    const int nv = D / V;
    const int grp = tid / nv, c0 = (tid - grp * nv) * V;
    const bool active = grp < groups;
    const int moff = (c0 / dh) * (rs - dh) + c0;   // used when MV == V
    constexpr int NP = V / 2;
    float2 g1p[NP], b1p[NP];
    if (ADDNORM && active) {
        load_pairs(g1 + c0, g1p);
        load_pairs(b1 + c0, b1p);
    }
    // statistics pass: lane l of a warp takes vectors l, l + 32, ... of a row
    int moffA[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int c = (lane + 32 * i) * V;
        moffA[i] = (c / dh) * (rs - dh) + c;
    }
    int it = 0;
    for (int b = blockIdx.x; b < B; b += gridDim.x, ++it) {
        const int cur = it % nslots;
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
        if (tid == 0) s_ok = ring.wait(cur, wc, SITE_MIX_LN);
        __syncthreads();
        if (!s_ok) break;
        E* xs = ring.buf(cur);
        if (PRE) {
            // the previous block's LayerNorm, applied once per element, in place
            if (active) normalize_in_place(xs, T, rs, c0, grp, groups, pre_g, pre_b, mean_s, rstd_s);
            __syncthreads();
        }
        E* srow = S + (size_t)b * TD;
        if (ADDNORM) {
            // pass A: mean and rstd of Z[h, :] = mix[h, :] + Xh[h, :], one warp
            // per row, sums shifted by the row's first element
            for (int h = warp; h < T; h += nw) {
                const float K = to_f(xs[h * dh]) + to_f(xs[(size_t)h * rs]);
                const float2 nK = f2(-K);
                float2 a1 = f2(0.f), a2 = f2(0.f);
#pragma unroll
                for (int i = 0; i < NV; ++i) {
                    const int v = lane + 32 * i;
                    if (v < nv) {
                        Vec16<E> xm;
                        mixed_vec<E, MV>(xs, rs, dh, h, v * V, moffA[i], xm);
                        float2 pm[NP], pr[NP];
                        unpack_pairs(xm.u, pm);
                        unpack_pairs(*reinterpret_cast<const uint4*>(xs + (size_t)h * rs + v * V), pr);
#pragma unroll
                        for (int j = 0; j < NP; ++j) {
                            const float2 d = f2_add(f2_add(pm[j], pr[j]), nK);
                            a1 = f2_add(a1, d);
                            a2 = f2_fma(d, d, a2);
                        }
                    }
                }
                const float s1 = warp_sum(a1.x + a1.y);
                const float s2 = warp_sum(a2.x + a2.y);
                if (lane == 0) {
                    const float m1 = s1 / D;
                    mean_s[h] = K + m1;
                    rstd_s[h] = rsqrtf(fmaxf(s2 / D - m1 * m1, 0.f) + eps);
                }
            }
            __syncthreads();
        }
        // pass B: element-wise, thread (grp, v) over rows grp, grp + groups, ...
        if (active) {
#pragma unroll 2
            for (int h = grp; h < T; h += groups) {
                Vec16<E> xm;
                mixed_vec<E, MV>(xs, rs, dh, h, c0, moff, xm);
                uint4 o = xm.u;   // without Add & Norm: S = TokenMixing(Xh), a permutation
                if (ADDNORM) {
                    float2 pm[NP], pr[NP];
                    unpack_pairs(xm.u, pm);
                    unpack_pairs(*reinterpret_cast<const uint4*>(xs + (size_t)h * rs + c0), pr);
                    const float r = rstd_s[h];
                    const float2 r2 = f2(r), mr2 = f2(-mean_s[h] * r);
#pragma unroll
                    for (int j = 0; j < NP; ++j) pm[j] = f2_fma(f2_fma(f2_add(pm[j], pr[j]), r2, mr2), g1p[j], b1p[j]);
                    o = pack_pairs(pm);
                }
                *reinterpret_cast<uint4*>(srow + (size_t)h * D + c0) = o;
            }
        }
        __syncthreads();   // the slot and the statistics are free again
        const long long nb = b + (long long)nslots * gridDim.x;
        if (warp == 0 && nb < B) ring.issue(cur, X + (size_t)nb * TD);
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
__global__ void __launch_bounds__(kPoolThreads, 2) ln_pool_kernel(const E* __restrict__ X,
                                                              const float2* __restrict__ pstats, int P,
                                                              const float* __restrict__ g,
                                                              const float* __restrict__ bta,
                                                              float* __restrict__ pooled, E* __restrict__ Xout,
                                                              int B, int T, int D, float eps, int nslots,
                                                              int groups, DeviceErr err, uint64_t budget_ns) {
    constexpr int V = Vec16<E>::N;
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ int abort_flag, s_ok;
    const int TD = T * D;
    float *mean_s, *rstd_s;
    SampleRing<E> ring;
    float* part = make_ring<E>(ring, smem, T, D, D, nslots, mean_s, rstd_s);   // [groups][D] partial sums
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    const WaitCtx wc{&abort_flag, budget_ns, err};
    if (tid == 0) {
        for (int k = 0; k < nslots; ++k) mbar_init(ring.bar(k), 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (warp == 0)
        for (int k = 0; k < nslots; ++k) {
            const long long bk = blockIdx.x + (long long)k * gridDim.x;
            if (bk < B) ring.issue(k, X + (size_t)bk * TD);
        }
    const int nv = D / V;
    const int grp = tid / nv, v = tid - grp * nv, c0 = v * V;
    const float invT = 1.0f / T;
    constexpr int NP = V / 2;
    float2 gp[NP], bp[NP];
    if (Xout && grp < groups) {
        load_pairs(g + c0, gp);
        load_pairs(bta + c0, bp);
    }
    int it = 0;
    for (int b = blockIdx.x; b < B; b += gridDim.x, ++it) {
        const int cur = it % nslots;
        for (int t = warp; t < T; t += nw) {
            float m, r;
            row_mean_rstd(pstats, P, D, (long long)b * T + t, eps, m, r);
            if (lane == 0) {
                mean_s[t] = m;
                rstd_s[t] = r;
            }
        }
        if (tid == 0) s_ok = ring.wait(cur, wc, SITE_LN_POOL);
        __syncthreads();
        if (!s_ok) break;
        const E* xs = ring.buf(cur);
        if (grp < groups) {
            float2 acc[NP];
#pragma unroll
            for (int j = 0; j < NP; ++j) acc[j] = f2(0.f);
#pragma unroll 2
            for (int t = grp; t < T; t += groups) {
                float2 x[NP];
                unpack_pairs(*reinterpret_cast<const uint4*>(xs + (size_t)t * D + c0), x);
                const float rt = rstd_s[t];
                const float2 r2 = f2(rt), mr2 = f2(-mean_s[t] * rt);
#pragma unroll
                for (int j = 0; j < NP; ++j) {
                    x[j] = f2_fma(x[j], r2, mr2);   // (x - m_t) r_t
                    acc[j] = f2_add(acc[j], x[j]);
                }
                if (Xout) {
#pragma unroll
                    for (int j = 0; j < NP; ++j) x[j] = f2_fma(x[j], gp[j], bp[j]);
                    *reinterpret_cast<uint4*>(Xout + (size_t)b * TD + (size_t)t * D + c0) = pack_pairs(x);
                }
            }
            float4* dst = reinterpret_cast<float4*>(part + (size_t)grp * D + c0);
#pragma unroll
            for (int q = 0; q < NP / 2; ++q)
                dst[q] = make_float4(acc[2 * q].x, acc[2 * q].y, acc[2 * q + 1].x, acc[2 * q + 1].y);
        }
        __syncthreads();
        for (int c = tid; c < D; c += blockDim.x) {
            float a = part[c];
            for (int q = 1; q < groups; ++q) a += part[(size_t)q * D + c];
            pooled[(size_t)b * D + c] = fmaf(__ldg(g + c), a * invT, __ldg(bta + c));
        }
        __syncthreads();   // slot, statistics and partials are free again
        const long long nb = b + (long long)nslots * gridDim.x;
        if (warp == 0 && nb < B) ring.issue(cur, X + (size_t)nb * TD);
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

// Ring slots (up to kMaxSlots, at least 1) and dynamic shared memory for
// samples of T rows at row stride rs, plus extra_floats floats after the
// per-row statistics.  Two CTAs share an SM whenever one slot each fits:
// measured in the stack, two independent CTAs (one computes while the other
// waits for its copy) beat one CTA with a deeper ring.
inline void ring_shape(int T, int rs, size_t esz, size_t extra_floats, int* nslots, size_t* smem) {
    const size_t one = slot_bytes_of(T, rs, esz);
    const size_t fixed = 8 * kMaxSlots + sizeof(float) * (2 * (size_t)T + extra_floats);
    const size_t full = 227 * 1024 - 1024;    // static shared memory and slack
    const size_t half = full / 2 - 1024;
    const size_t avail = one + fixed <= half ? half : full;
    long long n = avail > fixed ? (long long)((avail - fixed) / one) : 0;
    if (n > kMaxSlots) n = kMaxSlots;
    if (n < 1) n = 1;
    *nslots = (int)n;
    *smem = (size_t)n * one + fixed;
}

// Row groups: the largest divisor of T (so every group gets the same rows)
// with groups * nv <= kMixMaxThreads.
inline int mix_groups(int T, int nv) {
    int g = kMixMaxThreads / nv;
    if (g > T) g = T;
    while (g > 1 && T % g) --g;
    return g < 1 ? 1 : g;
}

template <typename E, bool PRE, int MV, int NVV, bool ADDNORM>
cudaError_t mix_ln_go(const E* X, const float* pg, const float* pb, RowStats ps, const float* g1, const float* b1,
                      E* S, int B, int T, int D, float eps, int num_sms, DeviceErr err, uint64_t budget,
                      cudaStream_t s) {
    constexpr int V = Vec16<E>::N;
    const int nv = D / V;
    if (nv < 1 || nv > kMixMaxThreads) return cudaErrorInvalidValue;
    const int groups = mix_groups(T, nv);
    int threads = (groups * nv + 31) / 32 * 32;
    if (threads < 64) threads = 64;
    const int rs = MV == V ? mix_row_stride(D, D / T, sizeof(E)) : D;
    int nslots;
    size_t smem;
    ring_shape(T, rs, sizeof(E), 0, &nslots, &smem);
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
    k<<<grid, threads, smem, s>>>(X, pg, pb, ps.part, ps.P, g1, b1, S, B, T, D, eps, rs, nslots, groups, err,
                                  budget);
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
    int nslots;
    size_t smem;
    ring_shape(T, D, sizeof(E), (size_t)groups * D, &nslots, &smem);
    while (groups > 1 && smem > kMaxSmemPerCta) {   // large samples: fewer row groups
        --groups;
        ring_shape(T, D, sizeof(E), (size_t)groups * D, &nslots, &smem);
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
                                       B, T, D, eps, nslots, groups, err, budget);
    return cudaGetLastError();
}

}  // namespace

// Largest D per dtype the mixing kernel supports (8 vectors per lane in its
// statistics pass).
int mix_ln_max_d(int dtype) { return 32 * 8 * (dtype == RM_BF16 ? 8 : 4); }

// Whether one staged sample (padded for the mixing gather) plus the kernels'
// per-row and pooling scratch fits a CTA's shared memory.
bool mix_ln_sample_fits(int dtype, int T, int D) {
    const size_t esz = dtype == RM_BF16 ? 2 : 4;
    const int V = (int)(16 / esz);
    const int dh = D / T;
    const int rs = dh % V == 0 ? mix_row_stride(D, dh, esz) : D;
    const size_t fixed = 8 * kMaxSlots + sizeof(float) * (2 * (size_t)T + (size_t)D);   // one pooling group
    return slot_bytes_of(T, rs, esz) + fixed <= 227 * 1024 - 1024;
}

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
