// e4m3 (fp8) quantisation for the stack with fp8 weights: every row of a
// [rows][K] bf16 array gets its own scale, absmax / 448 (448 is e4m3's largest
// finite value; an all-zero row gets scale 1), and its elements become
// e4m3(x / scale) with saturation.  Used for the FFN weights (one scale per
// output channel) and for the activations S and H (one scale per token row),
// so that the tensor cores' kind::f8f6f4 products dequantise as
// acc * ascale[row] * wscale[column] in the GEMM epilogue.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include <algorithm>

#include "rm_device.cuh"

namespace rm {
namespace {

constexpr int kThreads = 256;
constexpr float kE4M3Max = 448.0f;

// One CTA per row: every thread holds NV of the row's 16-byte vectors in
// registers (one read from HBM), the CTA reduces the absmax (warp butterflies,
// then the warps' maxima in shared memory), and the row leaves as e4m3 bytes.
template <int NV>
__global__ void __launch_bounds__(kThreads) quant_rows_kernel(const __nv_bfloat16* __restrict__ src,
                                                              uint8_t* __restrict__ dst, float* __restrict__ scale,
                                                              int K) {
    pdl_enter();
    __shared__ float wmax[kThreads / 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const long long r = blockIdx.x;
    const int nv = K / 8;
    const uint4* row = reinterpret_cast<const uint4*>(src + r * K);
    uint4 x[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int v = threadIdx.x + i * blockDim.x;
        if (v < nv) x[i] = __ldcg(row + v);
    }
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        if (threadIdx.x + i * blockDim.x < nv) {
            float2 p[4];
            unpack_pairs(x[i], p);
#pragma unroll
            for (int q = 0; q < 4; ++q) m = fmaxf(m, fmaxf(fabsf(p[q].x), fabsf(p[q].y)));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) wmax[warp] = m;
    __syncthreads();
    m = 0.f;
    for (int w = 0; w < nw; ++w) m = fmaxf(m, wmax[w]);
    const float sc = m > 0.f ? m / kE4M3Max : 1.0f;
    const float inv = 1.0f / sc;
    if (threadIdx.x == 0) scale[r] = sc;
    uint2* out = reinterpret_cast<uint2*>(dst + r * K);
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int v = threadIdx.x + i * blockDim.x;
        if (v < nv) {
            float2 p[4];
            unpack_pairs(x[i], p);
            uint32_t w[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
                    make_float2(p[2 * h].x * inv, p[2 * h].y * inv), __NV_SATFINITE, __NV_E4M3);
                const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
                    make_float2(p[2 * h + 1].x * inv, p[2 * h + 1].y * inv), __NV_SATFINITE, __NV_E4M3);
                w[h] = (uint32_t)lo | ((uint32_t)hi << 16);
            }
            out[v] = make_uint2(w[0], w[1]);
        }
    }
}

}  // namespace

cudaError_t launch_quant_rows(const void* src, void* dst, float* scale, long long rows, int K, cudaStream_t s) {
    if (K % 16 || rows > 0x7fffffffLL) return cudaErrorInvalidValue;
    const int nv = K / 8;
    // threads: the row's vectors up to 256, rounded to whole warps; NV vectors each
    const int threads = std::min(kThreads, (nv + 31) / 32 * 32);
    const int per = (nv + threads - 1) / threads;
    const auto* x = static_cast<const __nv_bfloat16*>(src);
    auto* d = static_cast<uint8_t*>(dst);
    const int grid = (int)rows;
    switch (per) {
        case 1: return launch_pdl(quant_rows_kernel<1>, grid, threads, 0, s, x, d, scale, K);
        case 2: return launch_pdl(quant_rows_kernel<2>, grid, threads, 0, s, x, d, scale, K);
        case 3: return launch_pdl(quant_rows_kernel<3>, grid, threads, 0, s, x, d, scale, K);
        case 4: return launch_pdl(quant_rows_kernel<4>, grid, threads, 0, s, x, d, scale, K);
        default:
            if (per <= 8) return launch_pdl(quant_rows_kernel<8>, grid, threads, 0, s, x, d, scale, K);
            return cudaErrorInvalidValue;   // rows of more than 16384 elements
    }
}

}  // namespace rm
