// e4m3 (fp8) quantisation for the stack with fp8 weights: every row of a
// [rows][K] bf16 array gets its own scale, absmax / 448 (448 is e4m3's largest
// finite value; an all-zero row gets scale 1), and its elements become
// e4m3(x / scale) with saturation.  Used for the FFN weights (one scale per
// output channel) and for the activations S and H (one scale per token row),
// so that the tensor cores' kind::f8f6f4 products dequantise as
// acc * ascale[row] * wscale[column] in the GEMM epilogue.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "rm_device.cuh"

namespace rm {
namespace {

constexpr int kThreads = 256;
constexpr float kE4M3Max = 448.0f;

// One warp per row: absmax over the row, then the row again (from L2),
// converted four pairs at a time.
__global__ void __launch_bounds__(kThreads) quant_rows_kernel(const __nv_bfloat16* __restrict__ src,
                                                              uint8_t* __restrict__ dst, float* __restrict__ scale,
                                                              long long rows, int K) {
    pdl_enter();
    const int lane = threadIdx.x & 31;
    const long long r = blockIdx.x * (long long)(blockDim.x >> 5) + (threadIdx.x >> 5);
    if (r >= rows) return;   // warp-uniform
    const int nv = K / 8;
    const uint4* row = reinterpret_cast<const uint4*>(src + r * K);
    float m = 0.f;
    for (int v = lane; v < nv; v += 32) {
        float2 p[4];
        unpack_pairs(__ldcg(row + v), p);
#pragma unroll
        for (int q = 0; q < 4; ++q) m = fmaxf(m, fmaxf(fabsf(p[q].x), fabsf(p[q].y)));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float sc = m > 0.f ? m / kE4M3Max : 1.0f;
    const float inv = 1.0f / sc;
    if (lane == 0) scale[r] = sc;
    uint2* out = reinterpret_cast<uint2*>(dst + r * K);
    for (int v = lane; v < nv; v += 32) {
        float2 p[4];
        unpack_pairs(__ldcg(row + v), p);
        uint32_t w[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const __nv_fp8x2_storage_t lo =
                __nv_cvt_float2_to_fp8x2(make_float2(p[2 * h].x * inv, p[2 * h].y * inv), __NV_SATFINITE, __NV_E4M3);
            const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
                make_float2(p[2 * h + 1].x * inv, p[2 * h + 1].y * inv), __NV_SATFINITE, __NV_E4M3);
            w[h] = (uint32_t)lo | ((uint32_t)hi << 16);
        }
        out[v] = make_uint2(w[0], w[1]);
    }
}

}  // namespace

cudaError_t launch_quant_rows(const void* src, void* dst, float* scale, long long rows, int K, cudaStream_t s) {
    if (K % 16) return cudaErrorInvalidValue;
    const int grid = (int)((rows + kThreads / 32 - 1) / (kThreads / 32));
    return launch_pdl(quant_rows_kernel, grid, kThreads, 0, s, static_cast<const __nv_bfloat16*>(src),
                      static_cast<uint8_t*>(dst), scale, rows, K);
}

}  // namespace rm
