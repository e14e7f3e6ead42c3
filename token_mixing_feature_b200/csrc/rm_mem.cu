// Memory-bound kernels of the RankMixer stack: standalone token mixing and
// row LayerNorm (the unfused variants behind rm_token_mix / rm_layernorm),
// Pad-Split tokenisation, the sigmoid head, and the wait self-test.
//
// Token mixing with H = T (fun-rec chapter "Rankmixer: 硬件效率优化", section
// Token Mixing机制: SplitHead into H chunks of D/H, then Concat chunk h of
// every token) maps output element (b, h, t*dh + j) to input element
// (b, t, h*dh + j), dh = D/T.
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
    pdl_enter();
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
            Y[o] = __ldcg(src);
        } else {
            *reinterpret_cast<uint4*>(Y + o) = __ldcg(reinterpret_cast<const uint4*>(src));
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
    pdl_enter();
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

// ------------------------------------------------------------------ Pad-Split
template <typename E>
__global__ void __launch_bounds__(kThreads) padsplit_kernel(PadSplitArgs a, E* __restrict__ X0, long long B,
                                                            int width) {
    pdl_enter();
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
            v = __ldcg(reinterpret_cast<const uint4*>(src));
        }
        *reinterpret_cast<uint4*>(X0 + b * width + c) = v;
    }
}

// ----------------------------------------------------------------------- head
template <typename E>
__global__ void __launch_bounds__(kThreads) head_kernel(const float* __restrict__ pooled, const E* __restrict__ w,
                                                        const float* __restrict__ bias, float* __restrict__ prob,
                                                        int B, int D) {
    pdl_enter();
    const int lane = threadIdx.x & 31;
    const int b = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (b >= B) return;
    float s = 0.f;
    for (int d = lane; d < D; d += 32) s += __ldcg(pooled + (long long)b * D + d) * to_f(w[d]);
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

}  // namespace

cudaError_t launch_token_mix(int dtype, const void* X, void* Y, int B, int T, int D, cudaStream_t s) {
    const int dh = D / T;
    const long long n = (long long)B * T * D;
    if (dtype == RM_BF16) {
        using E = __nv_bfloat16;
        if (dh % 8 == 0)
            return launch_pdl(token_mix_kernel<E, 8>, grid_for(n / 8, kThreads), kThreads, 0, s, (const E*)X, (E*)Y,
                              n / 8, T, D, dh);
        return launch_pdl(token_mix_kernel<E, 1>, grid_for(n, kThreads), kThreads, 0, s, (const E*)X, (E*)Y, n, T, D,
                          dh);
    }
    if (dh % 4 == 0)
        return launch_pdl(token_mix_kernel<float, 4>, grid_for(n / 4, kThreads), kThreads, 0, s, (const float*)X,
                          (float*)Y, n / 4, T, D, dh);
    return launch_pdl(token_mix_kernel<float, 1>, grid_for(n, kThreads), kThreads, 0, s, (const float*)X, (float*)Y, n,
                      T, D, dh);
}

cudaError_t launch_layernorm(int dtype, const void* A, const void* R, const float* g, const float* b, void* out,
                             long long rows, int D, float eps, cudaStream_t s) {
    const int grid = grid_for(rows, kThreads / 32);
    if (dtype == RM_BF16) {
        using E = __nv_bfloat16;
        return launch_pdl(layernorm_kernel<E>, grid, kThreads, 0, s, (const E*)A, (const E*)R, g, b, (E*)out, rows, D,
                          eps);
    }
    return launch_pdl(layernorm_kernel<float>, grid, kThreads, 0, s, (const float*)A, (const float*)R, g, b,
                      (float*)out, rows, D, eps);
}

cudaError_t launch_padsplit(int dtype, const PadSplitArgs& a, void* X0, int B, int width, cudaStream_t s) {
    const long long n = (long long)B * width / (dtype == RM_BF16 ? 8 : 4);
    if (dtype == RM_BF16)
        return launch_pdl(padsplit_kernel<__nv_bfloat16>, grid_for(n, kThreads), kThreads, 0, s, a,
                          (__nv_bfloat16*)X0, (long long)B, width);
    return launch_pdl(padsplit_kernel<float>, grid_for(n, kThreads), kThreads, 0, s, a, (float*)X0, (long long)B,
                      width);
}

cudaError_t launch_head(int dtype, const float* pooled, const void* w, const float* bias, float* prob, int B,
                        int D, cudaStream_t s) {
    const int grid = (B + kThreads / 32 - 1) / (kThreads / 32);
    if (dtype == RM_BF16)
        return launch_pdl(head_kernel<__nv_bfloat16>, grid, kThreads, 0, s, pooled, (const __nv_bfloat16*)w, bias,
                          prob, B, D);
    return launch_pdl(head_kernel<float>, grid, kThreads, 0, s, pooled, (const float*)w, bias, prob, B, D);
}

cudaError_t launch_selftest_wait(DeviceErr err, uint64_t budget_ns, cudaStream_t s) {
    selftest_wait_kernel<<<1, 32, 0, s>>>(err, budget_ns);
    return cudaGetLastError();
}

}  // namespace rm
