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

// RPC rows per CTA: every thread holds NV of each row's 16-byte vectors in
// registers (one read from HBM; all RPC rows' loads issued before the first
// use), the CTA reduces each row's absmax (warp butterflies, then the warps'
// maxima in shared memory), and the rows leave as e4m3 bytes.  Short rows
// take several per CTA so that more bytes are in flight per SM.
template <int NV, int RPC>
__global__ void __launch_bounds__(kThreads) quant_rows_kernel(const __nv_bfloat16* __restrict__ src,
                                                              uint8_t* __restrict__ dst, float* __restrict__ scale,
                                                              long long rows, int K) {
    pdl_enter();
    __shared__ float wmax[RPC][kThreads / 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const long long r0 = (long long)blockIdx.x * RPC;
    const int nv = K / 8;
    uint4 x[RPC][NV];
#pragma unroll
    for (int j = 0; j < RPC; ++j) {
        const uint4* row = reinterpret_cast<const uint4*>(src + (r0 + j) * K);
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            const int v = threadIdx.x + i * blockDim.x;
            if (r0 + j < rows && v < nv) x[j][i] = __ldcg(row + v);
        }
    }
    float m[RPC];
#pragma unroll
    for (int j = 0; j < RPC; ++j) {
        m[j] = 0.f;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            if (r0 + j < rows && threadIdx.x + i * blockDim.x < nv) {
                float2 p[4];
                unpack_pairs(x[j][i], p);
#pragma unroll
                for (int q = 0; q < 4; ++q) m[j] = fmaxf(m[j], fmaxf(fabsf(p[q].x), fabsf(p[q].y)));
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m[j] = fmaxf(m[j], __shfl_xor_sync(0xffffffffu, m[j], o));
        if (lane == 0) wmax[j][warp] = m[j];
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < RPC; ++j) {
        const long long r = r0 + j;
        if (r >= rows) break;
        float mm = 0.f;
        for (int w = 0; w < nw; ++w) mm = fmaxf(mm, wmax[j][w]);
        const float sc = mm > 0.f ? mm / kE4M3Max : 1.0f;
        const float inv = 1.0f / sc;
        if (threadIdx.x == 0) scale[r] = sc;
        uint2* out = reinterpret_cast<uint2*>(dst + r * K);
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            const int v = threadIdx.x + i * blockDim.x;
            if (v < nv) {
                float2 p[4];
                unpack_pairs(x[j][i], p);
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
    if (per == 1) {   // rows of up to 2048 elements: four to a CTA
        const int grid = (int)((rows + 3) / 4);
        return launch_pdl(quant_rows_kernel<1, 4>, grid, threads, 0, s, x, d, scale, rows, K);
    }
    const int grid = (int)rows;
    switch (per) {
        case 2: return launch_pdl(quant_rows_kernel<2, 1>, grid, threads, 0, s, x, d, scale, rows, K);
        case 3: return launch_pdl(quant_rows_kernel<3, 1>, grid, threads, 0, s, x, d, scale, rows, K);
        case 4: return launch_pdl(quant_rows_kernel<4, 1>, grid, threads, 0, s, x, d, scale, rows, K);
        default:
            if (per <= 8) return launch_pdl(quant_rows_kernel<8, 1>, grid, threads, 0, s, x, d, scale, rows, K);
            return cudaErrorInvalidValue;   // rows of more than 16384 elements
    }
}

}  // namespace rm
