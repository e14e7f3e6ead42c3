// fp32 T-grouped GEMM on CUDA cores (tensor cores off), for fp32 handles.
//     out[g, m, n] = epilogue( sum_k A[g, m, k] * W[g, n, k] )
// Same operand addressing and epilogues as the tcgen05 kernel, in fp32
// throughout: 64 x 64 output tiles, K slices of 16 staged in shared memory,
// a 4 x 4 register block per thread, FFMA accumulation in ascending k.
#include "rm_device.cuh"

namespace rm {
namespace {

constexpr int TM = 64, TN = 64, TK = 16;

template <int EPI>
__global__ void __launch_bounds__(256) gemm_simt_kernel(GroupedGemm p) {
    pdl_enter();
    __shared__ float As[TK][TM + 4];
    __shared__ float Ws[TK][TN + 4];
    const int g = blockIdx.z;
    const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const float* A = static_cast<const float*>(p.A) + (long long)g * p.a_gstride;
    const float* W = static_cast<const float*>(p.W) + (long long)g * p.N * p.K;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < p.K; k0 += TK) {
        for (int i = threadIdx.x; i < TM * TK; i += 256) {
            const int r = i / TK, kk = i - r * TK;
            const int m = m0 + r, n = n0 + r, k = k0 + kk;
            As[kk][r] = (m < p.M && k < p.K) ? A[(long long)m * p.a_ld + k] : 0.f;
            Ws[kk][r] = (n < p.N && k < p.K) ? W[(long long)n * p.K + k] : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < TK; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = Ws[kk][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
    float* out = static_cast<float*>(p.out) + (long long)g * p.o_gstride;
    const float* resid = static_cast<const float*>(p.resid);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + ty * 4 + i;
        if (m >= p.M) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + tx * 4 + j;
            if (n >= p.N) continue;
            float v = acc[i][j] + p.bias[(long long)g * p.N + n];
            if (EPI == EPI_GELU_TANH) {
                v = 0.5f * v * (1.0f + tanhf(0.7978845608028654f * (v + 0.044715f * v * v * v)));
            } else if (EPI == EPI_GELU_ERF) {
                v = 0.5f * v * (1.0f + erff(v * 0.7071067811865476f));
            } else if (EPI == EPI_RELU) {
                v = fmaxf(v, 0.0f);
            } else if (EPI == EPI_BIAS_RESID) {
                if (resid) v += resid[(long long)g * p.r_gstride + (long long)m * p.r_ld + n];
            }
            out[(long long)m * p.o_ld + n] = v;
        }
    }
}

}  // namespace

cudaError_t launch_gemm_simt(const GroupedGemm& p, cudaStream_t s) {
    if (p.grp_cnt || p.epi == EPI_BIAS_GATE) return cudaErrorInvalidValue;
    if (p.M == 0) return cudaSuccess;
    dim3 grid((p.N + TN - 1) / TN, (p.M + TM - 1) / TM, p.G);
    switch (p.epi) {
        case EPI_GELU_TANH: return launch_pdl(gemm_simt_kernel<EPI_GELU_TANH>, grid, 256, 0, s, p);
        case EPI_GELU_ERF: return launch_pdl(gemm_simt_kernel<EPI_GELU_ERF>, grid, 256, 0, s, p);
        case EPI_RELU: return launch_pdl(gemm_simt_kernel<EPI_RELU>, grid, 256, 0, s, p);
        default: return launch_pdl(gemm_simt_kernel<EPI_BIAS_RESID>, grid, 256, 0, s, p);
    }
}

}  // namespace rm
