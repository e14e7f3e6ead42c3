// Memory-bound kernels of the RankMixer stack: token mixing, LayerNorm, the
// fused mix + residual + LayerNorm pass, the final LayerNorm + mean pooling,
// Pad-Split tokenisation and the sigmoid head.
//
// Token mixing with H = T (fun-rec chapter "Rankmixer: 硬件效率优化", section
// Token Mixing机制: SplitHead into H chunks of D/H, then Concat chunk h of
// every token) maps output element (b, h, t*dh + j) to input element
// (b, t, h*dh + j), dh = D/T.  It is a permutation within one sample, so the
// kernels below stage one whole sample [T, D] in shared memory (read once,
// coalesced) and apply the permutation through shared-memory addressing; no
// transpose pass ever touches HBM.
#include <cuda_bf16.h>

#include "rm_device.cuh"

namespace rm {
namespace {

constexpr int kThreads = 256;

inline int grid_for(long long work, int per_block) {
    long long g = (work + per_block - 1) / per_block;
    if (g < 1) g = 1;
    if (g > 148LL * 16) g = 148LL * 16;
    return (int)g;
}

// ------------------------------------------------------------- token mixing
// One thread per V consecutive output elements; V > 1 only when dh % V == 0,
// so a vector never straddles two source tokens and is contiguous in X.
template <typename E, int V>
__global__ void __launch_bounds__(kThreads) token_mix_kernel(const E* __restrict__ X, E* __restrict__ Y,
                                                             long long nvec, int T, int D, int dh) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < nvec;
         i += (long long)gridDim.x * blockDim.x) {
        const long long o = i * V;
        const long long row = o / D;         // b*T + h
        const int c = (int)(o - row * D);
        const long long b = row / T;
        const int h = (int)(row - b * T);
        const int t = c / dh, j = c - t * dh;
        const E* src = X + (b * T + t) * D + (long long)h * dh + j;
        if constexpr (V == 1) {
            Y[o] = *src;
        } else {
            *reinterpret_cast<uint4*>(Y + o) = __ldg(reinterpret_cast<const uint4*>(src));
        }
    }
}

// ------------------------------------------------------------- row LayerNorm
// One warp per row: out = LN(A + R).  Mean, then the centred second moment,
// as two passes (the row stays in L1).
template <typename E>
__global__ void __launch_bounds__(kThreads) layernorm_kernel(const E* A, const E* R, const float* __restrict__ g,
                                                             const float* __restrict__ bta, E* out, long long rows,
                                                             int D, float eps) {
    constexpr int V = Vec16<E>::N;
    const int lane = threadIdx.x & 31;
    const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
    const int nv = D / V;
    for (long long r = blockIdx.x * (long long)(blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
        const uint4* a4 = reinterpret_cast<const uint4*>(A + r * D);
        const uint4* r4 = R ? reinterpret_cast<const uint4*>(R + r * D) : nullptr;
        float s = 0.f;
        for (int v = lane; v < nv; v += 32) {
            Vec16<E> x, y;
            x.u = a4[v];
            if (r4) y.u = r4[v];
#pragma unroll
            for (int e = 0; e < V; ++e) s += to_f(x.e[e]) + (r4 ? to_f(y.e[e]) : 0.f);
        }
        const float mu = warp_sum(s) / D;
        float q = 0.f;
        for (int v = lane; v < nv; v += 32) {
            Vec16<E> x, y;
            x.u = a4[v];
            if (r4) y.u = r4[v];
#pragma unroll
            for (int e = 0; e < V; ++e) {
                const float d = to_f(x.e[e]) + (r4 ? to_f(y.e[e]) : 0.f) - mu;
                q += d * d;
            }
        }
        const float rstd = rsqrtf(warp_sum(q) / D + eps);
        uint4* o4 = reinterpret_cast<uint4*>(out + r * D);
        for (int v = lane; v < nv; v += 32) {
            Vec16<E> x, y, o;
            x.u = a4[v];
            if (r4) y.u = r4[v];
#pragma unroll
            for (int e = 0; e < V; ++e) {
                const int c = v * V + e;
                const float z = to_f(x.e[e]) + (r4 ? to_f(y.e[e]) : 0.f);
                o.e[e] = from_f<E>(__ldg(g + c) * ((z - mu) * rstd) + __ldg(bta + c));
            }
            o4[v] = o.u;
        }
    }
}

// Load sample b ([T, D] contiguous) into shared memory with 16-byte vectors.
template <typename E>
__device__ __forceinline__ void load_sample(const E* X, E* xs, long long b, int TD) {
    const uint4* src = reinterpret_cast<const uint4*>(X + b * TD);
    uint4* dst = reinterpret_cast<uint4*>(xs);
    const int n = TD * (int)sizeof(E) / 16;
    for (int i = threadIdx.x; i < n; i += blockDim.x) dst[i] = __ldg(src + i);
}

// Mean and reciprocal std of every token row of the staged sample.
template <typename E>
__device__ __forceinline__ void row_stats(const E* xs, int T, int D, float eps, float* mean_s, float* rstd_s) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    for (int t = warp; t < T; t += nw) {
        const E* r = xs + t * D;
        float s = 0.f;
        for (int c = lane; c < D; c += 32) s += to_f(r[c]);
        const float mu = warp_sum(s) / D;
        float q = 0.f;
        for (int c = lane; c < D; c += 32) {
            const float d = to_f(r[c]) - mu;
            q += d * d;
        }
        q = warp_sum(q);
        if (lane == 0) {
            mean_s[t] = mu;
            rstd_s[t] = rsqrtf(q / D + eps);
        }
    }
}

// ---------------------------------------------------------- fused mix + LN
// One CTA per sample.  Xh = PRE ? LN_pre(X) : X per token row (the previous
// block's second LayerNorm, applied on load), then
//   Z[h, c] = Xh[t, h*dh + j] + Xh[h, c],  c = t*dh + j
//   S[h, :] = LN1(Z[h, :])
// One warp per output row h; each lane keeps its NV vectors of Z in registers.
template <typename E, bool PRE, bool CONTIG, int NV>
__global__ void __launch_bounds__(kThreads) mix_ln_kernel(const E* __restrict__ X, const float* __restrict__ pre_g,
                                                          const float* __restrict__ pre_b,
                                                          const float* __restrict__ g1,
                                                          const float* __restrict__ b1, E* __restrict__ S,
                                                          int T, int D, float eps) {
    constexpr int V = Vec16<E>::N;
    extern __shared__ __align__(16) unsigned char smem[];
    E* xs = reinterpret_cast<E*>(smem);
    float* mean_s = reinterpret_cast<float*>(smem + (size_t)T * D * sizeof(E));
    float* rstd_s = mean_s + T;
    const long long b = blockIdx.x;
    const int TD = T * D;
    load_sample(X, xs, b, TD);
    __syncthreads();
    if (PRE) {
        row_stats(xs, T, D, eps, mean_s, rstd_s);
        __syncthreads();
    }
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int dh = D / T;
    const int nv = D / V;
    E* srow_base = S + b * TD;
    for (int h = warp; h < T; h += nw) {
        float z[NV][V];
        float s = 0.f;
        const float mh = PRE ? mean_s[h] : 0.f, rh = PRE ? rstd_s[h] : 1.f;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            const int v = lane + 32 * i;
            if (v < nv) {
                const int c0 = v * V;
                int t = c0 / dh, j = c0 - t * dh;
#pragma unroll
                for (int e = 0; e < V; ++e) {
                    if (!CONTIG && e > 0) {
                        if (++j == dh) { j = 0; ++t; }
                    }
                    const int jj = CONTIG ? j + e : j;
                    const int k = h * dh + jj;          // column of the source token
                    const int c = c0 + e;
                    float xm = to_f(xs[t * D + k]);
                    float xr = to_f(xs[h * D + c]);
                    if (PRE) {
                        xm = (xm - mean_s[t]) * rstd_s[t] * __ldg(pre_g + k) + __ldg(pre_b + k);
                        xr = (xr - mh) * rh * __ldg(pre_g + c) + __ldg(pre_b + c);
                    }
                    z[i][e] = xm + xr;
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
                    q += d * d;
                }
            }
        }
        const float rstd = rsqrtf(warp_sum(q) / D + eps);
        uint4* out4 = reinterpret_cast<uint4*>(srow_base + (long long)h * D);
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            const int v = lane + 32 * i;
            if (v < nv) {
                Vec16<E> o;
#pragma unroll
                for (int e = 0; e < V; ++e) {
                    const int c = v * V + e;
                    o.e[e] = from_f<E>(__ldg(g1 + c) * ((z[i][e] - mu) * rstd) + __ldg(b1 + c));
                }
                out4[v] = o.u;
            }
        }
    }
}

// ------------------------------------------------------- final LN + pooling
// One CTA per sample: Xh = LN(X) per token row; pooled[b, d] = (1/T) sum_t
// Xh[t, d] summed in ascending t; Xout (optional) receives Xh.
template <typename E>
__global__ void __launch_bounds__(kThreads) ln_pool_kernel(const E* __restrict__ X, const float* __restrict__ g,
                                                           const float* __restrict__ bta, float* __restrict__ pooled,
                                                           E* __restrict__ Xout, int T, int D, float eps) {
    extern __shared__ __align__(16) unsigned char smem[];
    E* xs = reinterpret_cast<E*>(smem);
    float* mean_s = reinterpret_cast<float*>(smem + (size_t)T * D * sizeof(E));
    float* rstd_s = mean_s + T;
    const long long b = blockIdx.x;
    const int TD = T * D;
    load_sample(X, xs, b, TD);
    __syncthreads();
    row_stats(xs, T, D, eps, mean_s, rstd_s);
    __syncthreads();
    const float invT = 1.0f / T;
    for (int d = threadIdx.x; d < D; d += blockDim.x) {
        const float gd = __ldg(g + d), bd = __ldg(bta + d);
        float acc = 0.f;
        for (int t = 0; t < T; ++t) {
            const float xh = gd * ((to_f(xs[t * D + d]) - mean_s[t]) * rstd_s[t]) + bd;
            acc += xh;
            if (Xout) Xout[b * TD + (long long)t * D + d] = from_f<E>(xh);
        }
        pooled[b * D + d] = acc * invT;
    }
}

// ------------------------------------------------------------------ Pad-Split
template <typename E>
__global__ void __launch_bounds__(kThreads) padsplit_kernel(PadSplitArgs a, E* __restrict__ X0, long long B,
                                                            int width) {
    constexpr int V = Vec16<E>::N;
    const int wv = width / V;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < B * wv;
         i += (long long)gridDim.x * blockDim.x) {
        const long long b = i / wv;
        const int c = (int)(i - b * wv) * V;
        int gi = 0;
        while (gi < a.n && c >= a.col0[gi + 1]) ++gi;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (gi < a.n) {
            const int w = a.col0[gi + 1] - a.col0[gi];
            const E* src = reinterpret_cast<const E*>(a.src[gi]) + b * w + (c - a.col0[gi]);
            v = __ldg(reinterpret_cast<const uint4*>(src));
        }
        *reinterpret_cast<uint4*>(X0 + b * width + c) = v;
    }
}

// ----------------------------------------------------------------------- head
template <typename E>
__global__ void __launch_bounds__(kThreads) head_kernel(const float* __restrict__ pooled, const E* __restrict__ w,
                                                        const float* __restrict__ bias, float* __restrict__ prob,
                                                        int B, int D) {
    const int lane = threadIdx.x & 31;
    const int b = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (b >= B) return;
    float s = 0.f;
    for (int d = lane; d < D; d += 32) s += pooled[(long long)b * D + d] * to_f(w[d]);
    s = warp_sum(s);
    if (lane == 0) prob[b] = 1.0f / (1.0f + expf(-(s + bias[0])));
}

// ------------------------------------------------------------ wait self-test
// A single thread waits on an mbarrier that nobody arrives at; the bounded
// wait must run out, record RM_ERR_DEVICE_TIMEOUT and return.
__global__ void selftest_wait_kernel(DeviceErr err, uint64_t budget_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x != 0) return;
    abort_flag = 0;
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
    WaitCtx w{&abort_flag, budget_ns, err};
    mbar_wait(smem_u32(&bar), 0, w, SITE_SELFTEST);
}

template <typename E, bool PRE, bool CONTIG>
cudaError_t mix_ln_dispatch_nv(int nvl, const E* X, const float* pg, const float* pb, const float* g1,
                               const float* b1, E* S, int B, int T, int D, float eps, size_t smem,
                               cudaStream_t s) {
#define RM_MIXLN_CASE(NVV)                                                                           \
    if (nvl <= NVV) {                                                                                \
        auto k = mix_ln_kernel<E, PRE, CONTIG, NVV>;                                                 \
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); \
        if (e != cudaSuccess) return e;                                                              \
        k<<<B, kThreads, smem, s>>>(X, pg, pb, g1, b1, S, T, D, eps);                                \
        return cudaGetLastError();                                                                   \
    }
    RM_MIXLN_CASE(1)
    RM_MIXLN_CASE(2)
    RM_MIXLN_CASE(4)
    RM_MIXLN_CASE(8)
    RM_MIXLN_CASE(16)
#undef RM_MIXLN_CASE
    return cudaErrorInvalidValue;
}

template <typename E>
cudaError_t mix_ln_typed(const void* X, const float* pg, const float* pb, const float* g1, const float* b1,
                         void* S, int B, int T, int D, float eps, cudaStream_t s) {
    constexpr int V = Vec16<E>::N;
    const int dh = D / T;
    const int nv = D / V;
    const int nvl = (nv + 31) / 32;
    const size_t smem = (size_t)T * D * sizeof(E) + 2 * sizeof(float) * T;
    const bool contig = (dh % V) == 0;
    const E* x = static_cast<const E*>(X);
    E* y = static_cast<E*>(S);
    if (pg) {
        return contig ? mix_ln_dispatch_nv<E, true, true>(nvl, x, pg, pb, g1, b1, y, B, T, D, eps, smem, s)
                      : mix_ln_dispatch_nv<E, true, false>(nvl, x, pg, pb, g1, b1, y, B, T, D, eps, smem, s);
    }
    return contig ? mix_ln_dispatch_nv<E, false, true>(nvl, x, pg, pb, g1, b1, y, B, T, D, eps, smem, s)
                  : mix_ln_dispatch_nv<E, false, false>(nvl, x, pg, pb, g1, b1, y, B, T, D, eps, smem, s);
}

}  // namespace

// Largest D per dtype the register-cached mix kernel supports (16 vectors per lane).
int mix_ln_max_d(int dtype) { return 32 * 16 * (dtype == RM_BF16 ? 8 : 4); }

cudaError_t launch_token_mix(int dtype, const void* X, void* Y, int B, int T, int D, cudaStream_t s) {
    const int dh = D / T;
    const long long n = (long long)B * T * D;
    if (dtype == RM_BF16) {
        using E = __nv_bfloat16;
        if (dh % 8 == 0) {
            token_mix_kernel<E, 8><<<grid_for(n / 8, kThreads), kThreads, 0, s>>>(
                (const E*)X, (E*)Y, n / 8, T, D, dh);
        } else {
            token_mix_kernel<E, 1><<<grid_for(n, kThreads), kThreads, 0, s>>>((const E*)X, (E*)Y, n, T, D, dh);
        }
    } else {
        if (dh % 4 == 0) {
            token_mix_kernel<float, 4><<<grid_for(n / 4, kThreads), kThreads, 0, s>>>(
                (const float*)X, (float*)Y, n / 4, T, D, dh);
        } else {
            token_mix_kernel<float, 1><<<grid_for(n, kThreads), kThreads, 0, s>>>((const float*)X, (float*)Y,
                                                                                n, T, D, dh);
        }
    }
    return cudaGetLastError();
}

cudaError_t launch_layernorm(int dtype, const void* A, const void* R, const float* g, const float* b, void* out,
                             long long rows, int D, float eps, cudaStream_t s) {
    const int grid = grid_for(rows, kThreads / 32);
    if (dtype == RM_BF16) {
        using E = __nv_bfloat16;
        layernorm_kernel<E><<<grid, kThreads, 0, s>>>((const E*)A, (const E*)R, g, b, (E*)out, rows, D, eps);
    } else {
        layernorm_kernel<float><<<grid, kThreads, 0, s>>>((const float*)A, (const float*)R, g, b, (float*)out,
                                                           rows, D, eps);
    }
    return cudaGetLastError();
}

cudaError_t launch_mix_ln(int dtype, const void* X, const float* pre_g, const float* pre_b, const float* g1,
                          const float* b1, void* S, int B, int T, int D, float eps, cudaStream_t s) {
    if (dtype == RM_BF16) return mix_ln_typed<__nv_bfloat16>(X, pre_g, pre_b, g1, b1, S, B, T, D, eps, s);
    return mix_ln_typed<float>(X, pre_g, pre_b, g1, b1, S, B, T, D, eps, s);
}

cudaError_t launch_ln_pool(int dtype, const void* X, const float* g, const float* b, float* pooled, void* Xout,
                           int B, int T, int D, float eps, cudaStream_t s) {
    const size_t esz = dtype == RM_BF16 ? 2 : 4;
    const size_t smem = (size_t)T * D * esz + 2 * sizeof(float) * T;
    if (dtype == RM_BF16) {
        using E = __nv_bfloat16;
        auto k = ln_pool_kernel<E>;
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        k<<<B, kThreads, smem, s>>>((const E*)X, g, b, pooled, (E*)Xout, T, D, eps);
    } else {
        auto k = ln_pool_kernel<float>;
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        k<<<B, kThreads, smem, s>>>((const float*)X, g, b, pooled, (float*)Xout, T, D, eps);
    }
    return cudaGetLastError();
}

cudaError_t launch_padsplit(int dtype, const PadSplitArgs& a, void* X0, int B, int width, cudaStream_t s) {
    const long long n = (long long)B * width / (dtype == RM_BF16 ? 8 : 4);
    if (dtype == RM_BF16)
        padsplit_kernel<__nv_bfloat16><<<grid_for(n, kThreads), kThreads, 0, s>>>(a, (__nv_bfloat16*)X0, B, width);
    else
        padsplit_kernel<float><<<grid_for(n, kThreads), kThreads, 0, s>>>(a, (float*)X0, B, width);
    return cudaGetLastError();
}

cudaError_t launch_head(int dtype, const float* pooled, const void* w, const float* bias, float* prob, int B,
                        int D, cudaStream_t s) {
    const int grid = (B + kThreads / 32 - 1) / (kThreads / 32);
    if (dtype == RM_BF16)
        head_kernel<__nv_bfloat16><<<grid, kThreads, 0, s>>>(pooled, (const __nv_bfloat16*)w, bias, prob, B, D);
    else
        head_kernel<float><<<grid, kThreads, 0, s>>>(pooled, (const float*)w, bias, prob, B, D);
    return cudaGetLastError();
}

cudaError_t launch_selftest_wait(DeviceErr err, uint64_t budget_ns, cudaStream_t s) {
    selftest_wait_kernel<<<1, 32, 0, s>>>(err, budget_ns);
    return cudaGetLastError();
}

}  // namespace rm
