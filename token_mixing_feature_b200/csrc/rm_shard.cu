// Token-sharded stack forward: each of G ranks owns Tl = T / G consecutive
// tokens (their rows of every sample and their per-token FFN weights), and
// the token mixing becomes an all-to-all between the ranks.  The pages draw
// the analogy ("特征交叉 —— RankMixer 精读笔记": the mixing "和 all-to-all 操作的
// 逻辑一样"; "重新理解 RankMixer" section 3.3 on model sharding).
//
// With H = T heads, output token h of a sample takes chunk h of every input
// token t: S_pre[b, h, t dh + j] = Xh[b, t, h dh + j].  Rank q holds tokens t
// in [q Tl, (q + 1) Tl); the chunks h of its rows that rank r needs are the
// contiguous column range [r Tl dh, (r + 1) Tl dh) of each row (D / G
// columns), so rank q's send buffer is [G dest][B][Tl src token][D / G] and
// an equal-split all-to-all delivers recv[q src][b][tq][hr dh + j] to rank r.
//
//   pack:    Xh = LN2(V + S) (the previous block's output) or X0, for the
//            rank's own rows; Xh kept for the residual, its column ranges
//            scattered into the send buffer
//   mix_ln:  S[b, hr, t dh + j] = LN1(recv[t / Tl][b][t % Tl][hr dh + j]
//                                     + Xh[b, hr, t dh + j])
//   pool:    pooled_part[b] = gamma2 * mean over own t of xhat2 + beta2; the
//            mean over all T tokens is the mean of the G ranks' parts
//
// One warp per row in every kernel: the row's 16-byte vectors stay in
// registers, LayerNorm statistics are exact two-pass sums over the warp.
#include <cuda_bf16.h>

#include "rm_device.cuh"

namespace rm {
namespace {

constexpr int kThreads = 256;

// Two-pass mean and 1/sqrt(var + eps) of a row held as NVL vectors of 8
// values per lane (nv vectors in all).
template <int NVL>
__device__ __forceinline__ float2 row_stats(const float2 (&z)[NVL][4], int nv, int D, float eps) {
    const int lane = threadIdx.x & 31;
    float2 a = f2(0.f);
#pragma unroll
    for (int i = 0; i < NVL; ++i)
        if (lane + 32 * i < nv)
#pragma unroll
            for (int q = 0; q < 4; ++q) a = f2_add(a, z[i][q]);
    const float mean = warp_sum(a.x + a.y) / D;
    const float2 nm = f2(-mean);
    float2 a2 = f2(0.f);
#pragma unroll
    for (int i = 0; i < NVL; ++i)
        if (lane + 32 * i < nv)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float2 d = f2_add(z[i][q], nm);
                a2 = f2_fma(d, d, a2);
            }
    return make_float2(mean, rsqrtf(warp_sum(a2.x + a2.y) / D + eps));
}

// Rows (b, tq) of the rank: Z = Za + Zb (Zb may be null), Xh = LN(Z) with
// (g, bt) when g is given, else Z; Xh written to Xh[row] and its D / G column
// ranges to send[r][b][tq][:].
template <int NVL>
__global__ void __launch_bounds__(kThreads) shard_pack_kernel(const __nv_bfloat16* __restrict__ Za,
                                                              const __nv_bfloat16* __restrict__ Zb,
                                                              const float* __restrict__ g,
                                                              const float* __restrict__ bt, float eps,
                                                              __nv_bfloat16* __restrict__ Xh,
                                                              __nv_bfloat16* __restrict__ send, int B, int Tl, int D,
                                                              int G) {
    pdl_enter();
    const int lane = threadIdx.x & 31;
    const long long row = blockIdx.x * (long long)(blockDim.x >> 5) + (threadIdx.x >> 5);
    if (row >= (long long)B * Tl) return;   // warp-uniform
    const int b = (int)(row / Tl), tq = (int)(row - (long long)b * Tl);
    const int nv = D / 8, seg = D / G;
    float2 z[NVL][4];
#pragma unroll
    for (int i = 0; i < NVL; ++i) {
        const int v = lane + 32 * i;
        if (v < nv) {
            unpack_pairs(__ldcg(reinterpret_cast<const uint4*>(Za + row * D) + v), z[i]);
            if (Zb) {
                float2 y[4];
                unpack_pairs(__ldcg(reinterpret_cast<const uint4*>(Zb + row * D) + v), y);
#pragma unroll
                for (int q = 0; q < 4; ++q) z[i][q] = f2_add(z[i][q], y[q]);
            }
        }
    }
    if (g) {
        const float2 st = row_stats<NVL>(z, nv, D, eps);
        const float2 r2 = f2(st.y), mr2 = f2(-st.x * st.y);
#pragma unroll
        for (int i = 0; i < NVL; ++i) {
            const int v = lane + 32 * i;
            if (v < nv) {
                const float4 g0 = __ldg(reinterpret_cast<const float4*>(g) + 2 * v);
                const float4 g1 = __ldg(reinterpret_cast<const float4*>(g) + 2 * v + 1);
                const float4 b0 = __ldg(reinterpret_cast<const float4*>(bt) + 2 * v);
                const float4 b1 = __ldg(reinterpret_cast<const float4*>(bt) + 2 * v + 1);
                const float2 gp[4] = {make_float2(g0.x, g0.y), make_float2(g0.z, g0.w), make_float2(g1.x, g1.y),
                                      make_float2(g1.z, g1.w)};
                const float2 bp[4] = {make_float2(b0.x, b0.y), make_float2(b0.z, b0.w), make_float2(b1.x, b1.y),
                                      make_float2(b1.z, b1.w)};
#pragma unroll
                for (int q = 0; q < 4; ++q) z[i][q] = f2_fma(f2_fma(z[i][q], r2, mr2), gp[q], bp[q]);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < NVL; ++i) {
        const int v = lane + 32 * i;
        if (v < nv) {
            const uint4 o = pack_pairs(z[i]);   // the block output, rounded to bf16 as a stored one would be
            reinterpret_cast<uint4*>(Xh + row * D)[v] = o;
            const int c0 = 8 * v, r = c0 / seg;
            reinterpret_cast<uint4*>(send + (((long long)r * B + b) * Tl + tq) * seg + (c0 - r * seg))[0] = o;
        }
    }
}

// Output rows (b, hr) of the rank: Z[t dh + j] = recv[t / Tl][b][t % Tl][hr dh
// + j] + Xh[b, hr, t dh + j], S = LN1(Z).  dh % 8 == 0 (whole 16-byte pieces).
template <int NVL>
__global__ void __launch_bounds__(kThreads) shard_mix_ln_kernel(const __nv_bfloat16* __restrict__ recv,
                                                                const __nv_bfloat16* __restrict__ Xh,
                                                                const float* __restrict__ g,
                                                                const float* __restrict__ bt, float eps,
                                                                __nv_bfloat16* __restrict__ S, int B, int Tl, int D,
                                                                int G) {
    pdl_enter();
    const int lane = threadIdx.x & 31;
    const long long row = blockIdx.x * (long long)(blockDim.x >> 5) + (threadIdx.x >> 5);
    if (row >= (long long)B * Tl) return;   // warp-uniform
    const int b = (int)(row / Tl), hr = (int)(row - (long long)b * Tl);
    const int nv = D / 8, seg = D / G, dh = D / (Tl * G);
    uint4 xm[NVL], xr[NVL];
#pragma unroll
    for (int i = 0; i < NVL; ++i) {
        const int v = lane + 32 * i;
        if (v < nv) {
            const int c0 = 8 * v, t = c0 / dh, q = t / Tl, tq = t - q * Tl;
            xm[i] = __ldcg(reinterpret_cast<const uint4*>(recv + (((long long)q * B + b) * Tl + tq) * seg + hr * dh +
                                                          (c0 - t * dh)));
            xr[i] = __ldcg(reinterpret_cast<const uint4*>(Xh + row * D) + v);
        }
    }
    float2 z[NVL][4];
#pragma unroll
    for (int i = 0; i < NVL; ++i) {
        if (lane + 32 * i < nv) {
            float2 y[4];
            unpack_pairs(xm[i], z[i]);
            unpack_pairs(xr[i], y);
#pragma unroll
            for (int q = 0; q < 4; ++q) z[i][q] = f2_add(z[i][q], y[q]);
        }
    }
    const float2 st = row_stats<NVL>(z, nv, D, eps);
    const float2 r2 = f2(st.y), mr2 = f2(-st.x * st.y);
#pragma unroll
    for (int i = 0; i < NVL; ++i) {
        const int v = lane + 32 * i;
        if (v < nv) {
            const float4 g0 = __ldg(reinterpret_cast<const float4*>(g) + 2 * v);
            const float4 g1 = __ldg(reinterpret_cast<const float4*>(g) + 2 * v + 1);
            const float4 b0 = __ldg(reinterpret_cast<const float4*>(bt) + 2 * v);
            const float4 b1 = __ldg(reinterpret_cast<const float4*>(bt) + 2 * v + 1);
            const float2 gp[4] = {make_float2(g0.x, g0.y), make_float2(g0.z, g0.w), make_float2(g1.x, g1.y),
                                  make_float2(g1.z, g1.w)};
            const float2 bp[4] = {make_float2(b0.x, b0.y), make_float2(b0.z, b0.w), make_float2(b1.x, b1.y),
                                  make_float2(b1.z, b1.w)};
#pragma unroll
            for (int q = 0; q < 4; ++q) z[i][q] = f2_fma(f2_fma(z[i][q], r2, mr2), gp[q], bp[q]);
            reinterpret_cast<uint4*>(S + row * D)[v] = pack_pairs(z[i]);
        }
    }
}

// pooled_part[b, :] = g * (1/Tl) sum over the rank's tokens of xhat(V + S) + bt.
// CTA = one sample; warp w takes its tokens w, w + 8, ...; the warps' column
// sums are added in warp order through shared memory (deterministic).
template <int NVL>
__global__ void __launch_bounds__(kThreads) shard_pool_kernel(const __nv_bfloat16* __restrict__ V,
                                                              const __nv_bfloat16* __restrict__ Sres,
                                                              const float* __restrict__ g,
                                                              const float* __restrict__ bt, float eps,
                                                              float* __restrict__ pooled_part, int B, int Tl, int D) {
    pdl_enter();
    extern __shared__ float colsum[];   // [warps][D]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int b = blockIdx.x;
    const int nv = D / 8;
    float2 acc[NVL][4];
#pragma unroll
    for (int i = 0; i < NVL; ++i)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[i][q] = f2(0.f);
    for (int tq = warp; tq < Tl; tq += nw) {
        const long long row = (long long)b * Tl + tq;
        float2 z[NVL][4];
#pragma unroll
        for (int i = 0; i < NVL; ++i) {
            const int v = lane + 32 * i;
            if (v < nv) {
                float2 y[4];
                unpack_pairs(__ldcg(reinterpret_cast<const uint4*>(V + row * D) + v), z[i]);
                unpack_pairs(__ldcg(reinterpret_cast<const uint4*>(Sres + row * D) + v), y);
#pragma unroll
                for (int q = 0; q < 4; ++q) z[i][q] = f2_add(z[i][q], y[q]);
            }
        }
        const float2 st = row_stats<NVL>(z, nv, D, eps);
        const float2 r2 = f2(st.y), mr2 = f2(-st.x * st.y);
#pragma unroll
        for (int i = 0; i < NVL; ++i)
            if (lane + 32 * i < nv)
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[i][q] = f2_add(acc[i][q], f2_fma(z[i][q], r2, mr2));
    }
#pragma unroll
    for (int i = 0; i < NVL; ++i) {
        const int v = lane + 32 * i;
        if (v < nv)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                colsum[warp * D + 8 * v + 2 * q] = acc[i][q].x;
                colsum[warp * D + 8 * v + 2 * q + 1] = acc[i][q].y;
            }
    }
    __syncthreads();
    const float inv = 1.0f / Tl;
    for (int d = threadIdx.x; d < D; d += blockDim.x) {
        float s = 0.f;
        for (int w = 0; w < nw; ++w) s += colsum[w * D + d];
        pooled_part[(long long)b * D + d] = fmaf(__ldg(g + d), s * inv, __ldg(bt + d));
    }
}

}  // namespace

#define RM_SHARD_NVL(NV, CALL) \
    ((NV) <= 32 ? CALL(1) : (NV) <= 64 ? CALL(2) : (NV) <= 128 ? CALL(4) : (NV) <= 256 ? CALL(8) : cudaErrorInvalidValue)

cudaError_t launch_shard_pack(const void* Za, const void* Zb, const float* g, const float* bt, float eps, void* Xh,
                              void* send, int B, int Tl, int D, int G, cudaStream_t s) {
    const long long rows = (long long)B * Tl;
    const int grid = (int)((rows + kThreads / 32 - 1) / (kThreads / 32));
    const auto* a = static_cast<const __nv_bfloat16*>(Za);
    const auto* c = static_cast<const __nv_bfloat16*>(Zb);
    auto* xh = static_cast<__nv_bfloat16*>(Xh);
    auto* sd = static_cast<__nv_bfloat16*>(send);
#define RM_PACK(N) launch_pdl(shard_pack_kernel<N>, grid, kThreads, 0, s, a, c, g, bt, eps, xh, sd, B, Tl, D, G)
    return RM_SHARD_NVL(D / 8, RM_PACK);
#undef RM_PACK
}

cudaError_t launch_shard_mix_ln(const void* recv, const void* Xh, const float* g, const float* bt, float eps, void* S,
                                int B, int Tl, int D, int G, cudaStream_t s) {
    const long long rows = (long long)B * Tl;
    const int grid = (int)((rows + kThreads / 32 - 1) / (kThreads / 32));
    const auto* rc = static_cast<const __nv_bfloat16*>(recv);
    const auto* xh = static_cast<const __nv_bfloat16*>(Xh);
    auto* so = static_cast<__nv_bfloat16*>(S);
#define RM_MIXS(N) launch_pdl(shard_mix_ln_kernel<N>, grid, kThreads, 0, s, rc, xh, g, bt, eps, so, B, Tl, D, G)
    return RM_SHARD_NVL(D / 8, RM_MIXS);
#undef RM_MIXS
}

cudaError_t launch_shard_pool(const void* V, const void* Sres, const float* g, const float* bt, float eps,
                              float* pooled_part, int B, int Tl, int D, cudaStream_t s) {
    const size_t smem = sizeof(float) * (size_t)(kThreads / 32) * D;
    const auto* v = static_cast<const __nv_bfloat16*>(V);
    const auto* r = static_cast<const __nv_bfloat16*>(Sres);
#define RM_POOL(N)                                                                                                 \
    [&]() -> cudaError_t {                                                                                         \
        cudaError_t e = cudaFuncSetAttribute(shard_pool_kernel<N>, cudaFuncAttributeMaxDynamicSharedMemorySize,   \
                                             (int)smem);                                                            \
        if (e != cudaSuccess) return e;                                                                            \
        return launch_pdl(shard_pool_kernel<N>, B, kThreads, smem, s, v, r, g, bt, eps, pooled_part, B, Tl, D);     \
    }()
    return RM_SHARD_NVL(D / 8, RM_POOL);
#undef RM_POOL
}

#undef RM_SHARD_NVL

}  // namespace rm
