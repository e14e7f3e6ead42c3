// One training step of a dense bf16 RankMixer stack: forward with the
// tensors the backward pass needs, loss, and the gradient of every parameter
// and of the stack input.
//
// Forward (fun-rec chapter "Rankmixer: 硬件效率优化", section RankMixer整体架构,
// per block l):
//     Z1 = TokenMixing(X) + X,   S = LN1(Z1) = g1 * xhat1 + b1_ln
//     U  = S W1_t^T + b1_t,      Hh = act(U),   V = Hh W2_t^T + b2_t
//     Y  = V + S,                X' = LN2(Y) = g2 * xhat2 + b2_ln
// then pooled = mean_t X_L, logit = pooled . w + c, and the task loss
//     L = (1/B) sum_b [softplus(logit_b) - y_b logit_b]
// (mean binary cross-entropy of the sigmoid head; the pages name L_task
// without defining it, section Sparse MoE扩展).
//
// Backward, block by block in reverse, by the chain rule on those equations:
//     dX' -> dY          LayerNorm backward (ln2_bwd_kernel); the last block's
//                        dX' is dpooled / T on every token (the pooling's
//                        transpose)
//     dHh = dY W2_t,     dU = dHh * act'(U)      (grouped GEMM, N-major W2)
//     dW2_t = dY_t^T Hh_t,  db2_t = sum_b dY      (grouped GEMM over the batch)
//     dS  = dU W1_t + dY                          (grouped GEMM, N-major W1)
//     dW1_t = dU_t^T S_t,   db1_t = sum_b dU
//     dZ1 = LN1 backward of dS (ln1_bwd_kernel), and since the token mixing
//     with H = T is a permutation that is its own inverse, its transpose is
//     itself: dX = dZ1 + TokenMixing(dZ1).
// LayerNorm parameter gradients are column sums over every row:
// dg = sum dX' * xhat, db = sum dX'.
//
// Every column sum is computed as partial sums over fixed row blocks followed
// by an ordered reduction, so results are deterministic run to run.
#include <cuda_bf16.h>

#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <new>

#include "rm_device.cuh"

namespace rm {
namespace {

constexpr int kThreads = 256;
constexpr int kLnRows = 8;          // rows per block-wide reduction in the LayerNorm backward
constexpr int kMaxSampleBlock = 64; // samples per CTA of the LayerNorm backward
constexpr int kColRows = 16;        // rows per partial of the column sums
constexpr int kRedWarps = 32;       // sample / slice warps of the ordered column reductions

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}
__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
    return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                      pack_bf16x2(f[6], f[7]));
}
__device__ __forceinline__ void load8f(const float* p, float (&f)[8]) {
    const float4 a = __ldcg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldcg(reinterpret_cast<const float4*>(p) + 1);
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}
__device__ __forceinline__ void load8_param(const float* __restrict__ p, float (&f)[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}
__device__ __forceinline__ void store8f(float* p, const float (&f)[8]) {
    reinterpret_cast<float4*>(p)[0] = make_float4(f[0], f[1], f[2], f[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(f[4], f[5], f[6], f[7]);
}

// ------------------------------------------------------------ head and loss
// One warp per sample: logit, dL/dlogit = (sigmoid(logit) - y) / B and the
// sample's loss term softplus(logit) - y logit.
__global__ void __launch_bounds__(kThreads) head_logit_kernel(const float* pooled, const __nv_bfloat16* __restrict__ w,
                                                             const float* __restrict__ bias,
                                                             const float* __restrict__ labels, float* dlogit,
                                                             float* lterm, int B, int D) {
    pdl_enter();
    const int lane = threadIdx.x & 31;
    const int b = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (b >= B) return;
    float s = 0.f;
    for (int d = lane; d < D; d += 32) s += __ldcg(pooled + (long long)b * D + d) * __bfloat162float(w[d]);
    s = warp_sum(s);
    if (lane == 0) {
        const float logit = s + bias[0];
        const float y = labels[b];
        const float p = 1.0f / (1.0f + expf(-logit));
        dlogit[b] = (p - y) / (float)B;
        lterm[b] = fmaxf(logit, 0.f) + log1pf(expf(-fabsf(logit))) - y * logit;
    }
}

// dw[n] = sum_b dlogit_b pooled[b, n] and gpool[b, n] = dlogit_b w[n] / T,
// the gradient of every token row of the last block's output.  CTA = 32
// columns; warp w takes samples b = w, w + kRedWarps, ... in ascending order
// and the warp sums are added in warp order.  Warp 0 of CTA 0 adds up the
// loss and dc: lane l over b = l, l + 32, ..., then a fixed butterfly.
__global__ void __launch_bounds__(32 * kRedWarps) head_grad_kernel(const float* pooled,
                                                                  const __nv_bfloat16* __restrict__ w,
                                                                  const float* dlogit, const float* lterm, float* dw,
                                                                  float* dc, float* loss, float* gpool, int B, int D,
                                                                  float invT) {
    pdl_enter();
    __shared__ float red[kRedWarps][33];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int n = blockIdx.x * 32 + lane;
    float acc = 0.f;
    if (n < D) {
        const float wn = __bfloat162float(w[n]) * invT;
        for (int b = warp; b < B; b += kRedWarps) {
            const float g = __ldcg(dlogit + b);
            acc = fmaf(g, __ldcg(pooled + (long long)b * D + n), acc);
            gpool[(long long)b * D + n] = g * wn;
        }
    }
    red[warp][lane] = acc;
    __syncthreads();
    if (warp == 0 && n < D) {
        float t = 0.f;
#pragma unroll
        for (int q = 0; q < kRedWarps; ++q) t += red[q][lane];
        dw[n] = t;
    }
    if (blockIdx.x == 0 && warp == 0) {
        float l = 0.f, c = 0.f;
        for (int b = lane; b < B; b += 32) {
            l += __ldcg(lterm + b);
            c += __ldcg(dlogit + b);
        }
        l = warp_sum(l);
        c = warp_sum(c);
        if (lane == 0) {
            *loss = l / (float)B;
            *dc = c;
        }
    }
}

// ------------------------------------------------------- LayerNorm backward
// dY = rstd * (g*G - mean(g*G) - xhat * mean(g*G*xhat)) for the rows (b, t),
// b in one block of SB samples, t = blockIdx.y, with xhat = (Y - mean) * rstd
// recomputed from Y and its partial statistics.  Thread v owns the 8 columns
// [8v, 8v + 8) of every row and accumulates, over its rows, the partial
// column sums of G * xhat (dgamma), G (dbeta) and dY (the token's second
// bias).  Rows go in groups of kLnRows: one pass for the rows' sums (one
// block-wide reduction per group), a second pass, reading the rows again,
// for dY.  G is dX' [B, T, D] (bf16), or with FROM_POOL gpool [B, D] (fp32,
// the same row for every token).
template <bool FROM_POOL>
__device__ __forceinline__ void ln2_bwd_load(const __nv_bfloat16* G, const float* gpool, const __nv_bfloat16* Y,
                                             long long b, long long row, int D, int c0, float (&g)[8], float (&y)[8]) {
    if (FROM_POOL) load8f(gpool + b * D + c0, g);
    else unpack8(__ldcg(reinterpret_cast<const uint4*>(G + row * D + c0)), g);
    unpack8(__ldcg(reinterpret_cast<const uint4*>(Y + row * D + c0)), y);
}

template <bool FROM_POOL>
__global__ void __launch_bounds__(kThreads) ln2_bwd_kernel(const __nv_bfloat16* G, const float* gpool,
                                                          const __nv_bfloat16* Y, const float2* ystats, int P,
                                                          const float* __restrict__ gamma, float eps,
                                                          __nv_bfloat16* dY, float* part_g, float* part_b,
                                                          float* part_db, int B, int T, int D, int SB) {
    pdl_enter();
    __shared__ float mean_s[kMaxSampleBlock], rstd_s[kMaxSampleBlock];
    __shared__ float red[2][kThreads / 32][2 * kLnRows];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int t = blockIdx.y, sb = blockIdx.x, nsb = gridDim.x;
    const int b0 = sb * SB, nb = min(SB, B - b0);
    const float n = (float)D / (float)P;
    for (int i = warp; i < nb; i += nw) {   // row statistics from the producer's partials
        const long long row = (long long)(b0 + i) * T + t;
        const float2 v = lane < P ? __ldcg(ystats + row * P + lane) : make_float2(0.f, 0.f);
        const float mean = warp_sum(v.x) / (float)P;
        const float d = v.x - mean;
        const float q = warp_sum(lane < P ? fmaf(n * d, d, v.y) : 0.f);
        if (lane == 0) {
            mean_s[i] = mean;
            rstd_s[i] = rsqrtf(q / D + eps);
        }
    }
    __syncthreads();
    const int nv = D / 8, v = threadIdx.x;
    const bool active = v < nv;
    const int c0 = 8 * v;
    float gm[8], ag[8], ab[8], adb[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) ag[e] = ab[e] = adb[e] = 0.f;
    if (active) load8_param(gamma + c0, gm);
    const float invD = 1.0f / (float)D;
    int par = 0;
    for (int i0 = 0; i0 < nb; i0 += kLnRows, par ^= 1) {
        // pass 1: the rows' sums of g*G and g*G*xhat, and the column partials
        float cs[2 * kLnRows];
#pragma unroll
        for (int k = 0; k < kLnRows; ++k) {
            const int i = i0 + k;
            float s1 = 0.f, s2 = 0.f;
            if (active && i < nb) {
                float g[8], y[8];
                ln2_bwd_load<FROM_POOL>(G, gpool, Y, b0 + i, (long long)(b0 + i) * T + t, D, c0, g, y);
                const float m = mean_s[i], r = rstd_s[i];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float xh = (y[e] - m) * r;
                    const float gx = g[e] * gm[e];
                    s1 += gx;
                    s2 = fmaf(gx, xh, s2);
                    ag[e] = fmaf(g[e], xh, ag[e]);
                    ab[e] += g[e];
                }
            }
            cs[2 * k] = s1;
            cs[2 * k + 1] = s2;
        }
#pragma unroll
        for (int q = 0; q < 2 * kLnRows; ++q) cs[q] = warp_sum(cs[q]);
        if (lane == 0)
#pragma unroll
            for (int q = 0; q < 2 * kLnRows; ++q) red[par][warp][q] = cs[q];
        __syncthreads();
#pragma unroll
        for (int q = 0; q < 2 * kLnRows; ++q) {
            float a = 0.f;
            for (int w = 0; w < nw; ++w) a += red[par][w][q];
            cs[q] = a * invD;
        }
        // pass 2: the rows again (from L1 / L2), dY out
#pragma unroll
        for (int k = 0; k < kLnRows; ++k) {
            const int i = i0 + k;
            if (active && i < nb) {
                const long long row = (long long)(b0 + i) * T + t;
                float g[8], y[8], dy[8];
                ln2_bwd_load<FROM_POOL>(G, gpool, Y, b0 + i, row, D, c0, g, y);
                const float m = mean_s[i], r = rstd_s[i];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float xh = (y[e] - m) * r;
                    dy[e] = r * (g[e] * gm[e] - cs[2 * k] - xh * cs[2 * k + 1]);
                    adb[e] += dy[e];
                }
                *reinterpret_cast<uint4*>(dY + row * D + c0) = pack8(dy);
            }
        }
    }
    if (active) {
        const long long o = ((long long)t * nsb + sb) * D + c0;
        store8f(part_g + o, ag);
        store8f(part_b + o, ab);
        store8f(part_db + o, adb);
    }
}

// --------------------------------------------------------------- column sums
// part[(g * nrb + rb) * N + n] = sum over rows r of block rb of A[g, r, n],
// and part2 the same sum of A[g, r, n] * X2[g, r, n] (X2 may be null);
// A element (g, r, n) at A + g*gs + r*ld + n.  Thread = 8 columns.
__global__ void __launch_bounds__(kThreads) colsum_kernel(const __nv_bfloat16* A, const __nv_bfloat16* X2,
                                                         float* part, float* part2, int R, int N, long long gs,
                                                         long long ld, int RB) {
    pdl_enter();
    const int v = blockIdx.x * blockDim.x + threadIdx.x;
    if (8 * v >= N) return;
    const int rb = blockIdx.y, nrb = gridDim.y, g = blockIdx.z;
    const int r0 = rb * RB, r1 = min(R, r0 + RB);
    float a[8], a2[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) a[e] = a2[e] = 0.f;
    for (int r = r0; r < r1; r += 4) {   // up to four rows' loads in flight, summed in row order
        uint4 xa[4], xb[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            if (r + q < r1) {
                const long long off = g * gs + (long long)(r + q) * ld + 8 * v;
                xa[q] = __ldcg(reinterpret_cast<const uint4*>(A + off));
                if (X2) xb[q] = __ldcg(reinterpret_cast<const uint4*>(X2 + off));
            }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            if (r + q < r1) {
                float x[8];
                unpack8(xa[q], x);
                if (X2) {
                    float y[8];
                    unpack8(xb[q], y);
#pragma unroll
                    for (int e = 0; e < 8; ++e) a2[e] = fmaf(x[e], y[e], a2[e]);
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) a[e] += x[e];
            }
        }
    }
    const long long o = ((long long)g * nrb + rb) * N + 8 * v;
    store8f(part + o, a);
    if (X2) store8f(part2 + o, a2);
}

// The same over variable row ranges: part[(g * nrb + rb) * N + n] = sum over
// rows r of block rb of [0, cnt[g]) of A[(off[g] + r) * ld + n] (the
// sparse-MoE experts' compacted rows; blocks past cnt[g] write zeros).
__global__ void __launch_bounds__(kThreads) colsum_var_kernel(const __nv_bfloat16* A, float* part,
                                                             const int* __restrict__ off,
                                                             const int* __restrict__ cnt, int N, long long ld,
                                                             int RB) {
    pdl_enter();
    const int v = blockIdx.x * blockDim.x + threadIdx.x;
    if (8 * v >= N) return;
    const int rb = blockIdx.y, nrb = gridDim.y, g = blockIdx.z;
    const int c = __ldcg(cnt + g);
    const long long base = __ldcg(off + g);
    const int r0 = rb * RB, r1 = min(c, r0 + RB);
    float a[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) a[e] = 0.f;
    for (int r = r0; r < r1; r += 4) {   // up to four rows' loads in flight, summed in row order
        uint4 xa[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
            if (r + q < r1) xa[q] = __ldcg(reinterpret_cast<const uint4*>(A + (base + r + q) * ld + 8 * v));
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            if (r + q < r1) {
                float x[8];
                unpack8(xa[q], x);
#pragma unroll
                for (int e = 0; e < 8; ++e) a[e] += x[e];
            }
        }
    }
    store8f(part + ((long long)g * nrb + rb) * N + 8 * v, a);
}

// out[g * N + n] = sum_{j < J} part[(g * J + j) * N + n].  CTA = (32
// columns, group g) x W warps (W = blockDim.x / 32, about J / 8 from the
// host, at most kRedWarps); warp w sums the slices j = w, w + W, ... of its
// lane's column in ascending j, then one warp adds the warp sums in warp order
// (a fixed order for a given shape: deterministic).
__global__ void __launch_bounds__(32 * kRedWarps) reduce_parts_kernel(const float* part, float* out, int G, int J,
                                                                      int N) {
    pdl_enter();
    __shared__ float red[kRedWarps][33];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, W = blockDim.x >> 5;
    const int n = blockIdx.x * 32 + lane, g = blockIdx.y;
    float a = 0.f;
    if (n < N) {
        const float* p = part + (long long)g * J * N + n;
        int j = warp;
        for (; j + 3 * W < J; j += 4 * W) {   // four loads in flight
            const float x0 = __ldcg(p + (long long)j * N), x1 = __ldcg(p + (long long)(j + W) * N);
            const float x2 = __ldcg(p + (long long)(j + 2 * W) * N);
            const float x3 = __ldcg(p + (long long)(j + 3 * W) * N);
            a += x0;
            a += x1;
            a += x2;
            a += x3;
        }
        for (; j < J; j += W) a += __ldcg(p + (long long)j * N);
    }
    red[warp][lane] = a;
    __syncthreads();
    if (warp == 0 && n < N) {
        float t = 0.f;
        for (int w = 0; w < W; ++w) t += red[w][lane];
        out[(long long)g * N + n] = t;
    }
}

// scratch[(g * gridDim.z + c) * N + n] = sum of slices [c*CH, min(J, c*CH + CH))
// of column n of group g, in the same warp-split order as reduce_parts_kernel.
__global__ void __launch_bounds__(32 * kRedWarps) reduce_chunks_kernel(const float* part, float* scratch, int G, int J,
                                                                       int N, int CH) {
    pdl_enter();
    __shared__ float red[kRedWarps][33];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, W = blockDim.x >> 5;
    const int n = blockIdx.x * 32 + lane, g = blockIdx.y, c = blockIdx.z;
    const int j0 = c * CH, j1 = min(J, j0 + CH);
    float a = 0.f;
    if (n < N) {
        const float* p = part + (long long)g * J * N + n;
        for (int j = j0 + warp; j < j1; j += W) a += __ldcg(p + (long long)j * N);
    }
    red[warp][lane] = a;
    __syncthreads();
    if (warp == 0 && n < N) {
        float t = 0.f;
        for (int w = 0; w < W; ++w) t += red[w][lane];
        scratch[((long long)g * gridDim.z + c) * N + n] = t;
    }
}

// Ordered reduction of J slices per column: about eight slices per warp.
// When the (column block, group) grid is too small to fill the GPU and J is
// large, the slices are first reduced in fixed chunks of kRedChunk into
// `scratch` (ceil(J / kRedChunk) x G x N floats), then those chunk sums in
// order: a fixed order for a given shape (deterministic).
constexpr int kRedChunk = 64;
inline cudaError_t launch_reduce_parts(const float* part, float* out, int G, int J, int N, cudaStream_t s,
                                       float* scratch = nullptr) {
    const long long ctas = (long long)((N + 31) / 32) * G;
    if (scratch && ctas < 2 * 148 && J > 2 * kRedChunk) {
        const int JS = (J + kRedChunk - 1) / kRedChunk;
        // chunk c of group g: slices [c*kRedChunk, ...) of g -> scratch[(g*JS + c)*N + n]
        const int W = std::min(kRedWarps, kRedChunk / 8);
        cudaError_t e = launch_pdl(reduce_chunks_kernel, dim3((N + 31) / 32, G, JS), dim3(32 * W), 0, s, part,
                                   scratch, G, J, N, kRedChunk);
        if (e != cudaSuccess) return e;
        part = scratch;
        J = JS;
    }
    const int W = std::min(kRedWarps, std::max(1, (J + 7) / 8));
    return launch_pdl(reduce_parts_kernel, dim3((N + 31) / 32, G), dim3(32 * W), 0, s, part, out, G, J, N);
}

// ---------------------------------------------- LN1 backward + mixing transpose
// Per sample (persistent CTAs, two per SM): one warp per row h reads the
// row's dS and xhat1 from global memory and computes
//     dZ = rstd1 * (g1*dS - mean(g1*dS) - xhat1 * mean(g1*dS*xhat1))
// into shared memory (rows padded for the mixing gather); then
//     dX[t] = dZ[t] + TokenMixing(dZ)[t]
// leaves through the same 16-byte gather as the forward mixing (thread =
// row group x 16-byte column vector).  Only dZ is staged, since every other
// input is row-local.
constexpr int kBwdMixThreads = 256;

template <int NV>
__global__ void __launch_bounds__(kBwdMixThreads, 2) ln1_bwd_mix_kernel(const __nv_bfloat16* dS,
                                                                       const __nv_bfloat16* xhat, const float* rstd1,
                                                                       const float* __restrict__ gamma,
                                                                       __nv_bfloat16* dX, int B, int T, int D, int rs,
                                                                       int groups, DeviceErr err,
                                                                       uint64_t budget_ns) {
    pdl_enter();
    extern __shared__ __align__(128) unsigned char smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    const int TD = T * D, dh = D / T, nv = D / 8;
    const uint32_t dz_a = smem_u32(smem);   // [T][rs] bf16
    const float invD = 1.0f / (float)D;
    // element pass layout: thread (grp, v) over rows grp, grp + groups, ...
    const int grp = tid / nv, c0 = (tid - grp * nv) * 8;
    const bool active = grp < groups;
    // source of the mixed vector at column c0 of output row h: token t = c0 / dh,
    // element t*rs + h*dh + (c0 - t*dh) of the staged sample (16-byte pieces: dh % 8 == 0)
    const int msrc = (c0 / dh) * (rs - dh) + c0;
    for (int b = blockIdx.x; b < B; b += gridDim.x) {
        const __nv_bfloat16* dsb = dS + (size_t)b * TD;
        const __nv_bfloat16* xhb = xhat + (size_t)b * TD;
        for (int h = warp; h < T; h += nw) {
            uint4 du[NV], xu[NV];
#pragma unroll
            for (int i = 0; i < NV; ++i) {   // every load of the row in flight at once
                const int v = lane + 32 * i;
                if (v < nv) {
                    du[i] = __ldcg(reinterpret_cast<const uint4*>(dsb + (size_t)h * D) + v);
                    xu[i] = __ldcg(reinterpret_cast<const uint4*>(xhb + (size_t)h * D) + v);
                }
            }
            const float r = __ldcg(rstd1 + (long long)b * T + h);
            float s1 = 0.f, s2 = 0.f;
#pragma unroll
            for (int i = 0; i < NV; ++i) {
                if (lane + 32 * i < nv) {
                    float d[8], x[8], g[8];
                    unpack8(du[i], d);
                    unpack8(xu[i], x);
                    load8_param(gamma + 8 * (lane + 32 * i), g);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float gx = d[e] * g[e];
                        s1 += gx;
                        s2 = fmaf(gx, x[e], s2);
                    }
                }
            }
            s1 = warp_sum(s1) * invD;
            s2 = warp_sum(s2) * invD;
#pragma unroll
            for (int i = 0; i < NV; ++i) {
                const int v = lane + 32 * i;
                if (v < nv) {
                    float d[8], x[8], g[8], dz[8];
                    unpack8(du[i], d);
                    unpack8(xu[i], x);
                    load8_param(gamma + 8 * v, g);
#pragma unroll
                    for (int e = 0; e < 8; ++e) dz[e] = r * (d[e] * g[e] - s1 - x[e] * s2);
                    sts128(dz_a + (uint32_t)((h * rs + 8 * v) * 2), pack8(dz));
                }
            }
        }
        __syncthreads();
        if (active) {
            __nv_bfloat16* out = dX + (size_t)b * TD;
            for (int r = grp; r < T; r += groups) {
                float a[8], m[8];
                unpack8(lds128(dz_a + (uint32_t)((r * rs + c0) * 2)), a);
                unpack8(lds128(dz_a + (uint32_t)((msrc + r * dh) * 2)), m);
#pragma unroll
                for (int e = 0; e < 8; ++e) a[e] += m[e];
                *reinterpret_cast<uint4*>(out + (size_t)r * D + c0) = pack8(a);
            }
        }
        __syncthreads();   // the staged dZ is free again
    }
    (void)err;
    (void)budget_ns;
}

int mix_pad_stride(int D, int dh) {
    // consecutive token rows start (dh - D) * 2 bytes apart modulo 128, so the
    // 16-byte pieces consecutive threads gather fall in consecutive banks
    long long pad = ((long long)(dh - D) * 2) % 128;
    if (pad < 0) pad += 128;
    return D + (int)(pad / 2);
}

size_t ln1_bwd_smem(int T, int D, int rs) {
    (void)D;
    return ((size_t)T * rs * 2 + 127) / 128 * 128;
}

inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace
}  // namespace rm

// ==================================================================== host
struct rm_trainer {
    rm_config cfg;
    int num_sms;
    int stat_P;
    int nsb, SB;             // LayerNorm-backward sample blocks
    unsigned char* ws;
    size_t ws_bytes;
    int* err;
    uint64_t budget_ns;
    // per block
    unsigned char **S, **XH1, **U, **H, **Y;
    float** RS1;
    float2** ystats;
    // per block, sparse MoE (Ne > 0): routing and compaction (slot lists
    // padded per expert to a multiple of 64), DTSI's second router's gates,
    // and the compacted expert rows (S, activation input U, hidden H, gated
    // output)
    rm::MoeWork* moe;
    float** gates_inf;
    long long rows_max;      // compacted rows allocated per array
    float lambda;            // L_reg weight
    // shared
    float *pooled, *dlogit, *lterm, *gpool;
    unsigned char *dY, *dU, *dS, *dX;
    float *pg, *pb, *pdb, *pcol, *pcol2;
    float* rscratch;         // chunk sums of the two-stage ordered reductions
    float* lreg_part;        // chunk sums of L_reg
    float* sk_ws;
    int* sk_cnt;
    // shared, sparse MoE backward
    unsigned char *dEg, *dUg, *dSg;
    float *dR, *dRinf, *prt, *prt_b;
    int* cnt_scratch;
};

namespace {

using rm::round_up;

rm::DeviceErr terr(rm_trainer* t) { return rm::DeviceErr{t->err, t->err + 1}; }

template <typename P>
P* carve(unsigned char* base, size_t& off, size_t bytes) {
    P* p = reinterpret_cast<P*>(base + off);
    off += round_up(bytes, 256);
    return p;
}

bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

rm_status cuda_st(cudaError_t e) { return e == cudaSuccess ? RM_OK : RM_ERR_CUDA; }

}  // namespace

namespace {

// Backward of one sparse-MoE FFN given dL/dY in t->dY (fun-rec "Rankmixer:
// 硬件效率优化", section Sparse MoE扩展): the gates' and the experts'
// gradients over the compacted (padded) slot lists, the experts' weight
// gradients as variable-K grouped products, the routers' gradients (L_reg on
// the routing gates, or on DTSI's second router), and dL/dS into t->dS.
cudaError_t moe_backward(rm_trainer* t, const rm_block_weights& w, const rm_block_grads& gr, int l, int B,
                         cudaStream_t s) {
    const rm_config& c = t->cfg;
    const int T = c.T, D = c.D, Hd = c.hidden, Ne = c.n_experts, G = T * Ne;
    const rm::DeviceErr err = terr(t);
    const uint64_t budget = t->budget_ns;
    const rm::MoeWork& mw = t->moe[l];
    const float* ginf = w.Wr_infer ? t->gates_inf[l] : nullptr;
    float* dRinf = ginf ? t->dRinf : nullptr;
    cudaError_t e = rm::launch_moe_bwd_gate(t->dY, mw, ginf, t->lambda, t->dEg, t->dR, dRinf, B, T, D, Ne, s);
    if (e != cudaSuccess) return e;
    // dU_j = (de_j W2_j) * act'(U_j) over the expert's slots
    rm::GroupedGemm gh{};
    gh.G = G; gh.M = 0; gh.N = Hd; gh.K = D;
    gh.A = t->dEg; gh.a_ld = D; gh.a_rows_total = t->rows_max;
    gh.W = w.W2; gh.w_mn = true; gh.w_gstride = (long long)D * Hd; gh.w_ld = Hd;
    gh.out = t->dUg; gh.o_ld = Hd;
    gh.resid = t->U[l]; gh.r_ld = Hd;
    gh.epi = rm::dact_epi_for_act(c.act);
    gh.var_cg = 1;
    gh.grp_cnt = mw.cnt_pad; gh.grp_off = mw.offsets; gh.mtile_prefix = mw.mtile_prefix;
    if ((e = rm::launch_gemm_tc(gh, err, budget, t->num_sms, s)) != cudaSuccess) return e;
    // dW2_j = de_j^T H_j (fp32), K = the expert's padded slot count
    rm::GroupedGemm gw2{};
    gw2.G = G; gw2.M = D; gw2.N = Hd; gw2.K = 64;
    gw2.A = t->dEg; gw2.a_mn = true; gw2.a_ld = D; gw2.a_rows_total = t->rows_max;
    gw2.W = mw.Hg; gw2.w_mn = true; gw2.w_ld = Hd;
    gw2.out = gr.W2; gw2.o_gstride = (long long)D * Hd; gw2.o_ld = Hd;
    gw2.epi = rm::EPI_F32;
    gw2.vark = true; gw2.vark_cnt = mw.cnt_pad; gw2.grp_off = mw.offsets;
    if ((e = rm::launch_gemm_tc(gw2, err, budget, t->num_sms, s)) != cudaSuccess) return e;
    // db2_j, db1_j: column sums over the expert's slots (padding rows are zero)
    const int nrb_g = (B + 64 + rm::kColRows - 1) / rm::kColRows;
    e = rm::launch_pdl(rm::colsum_var_kernel, dim3((D / 8 + rm::kThreads - 1) / rm::kThreads, nrb_g, G),
                       dim3(rm::kThreads), 0, s, (const __nv_bfloat16*)t->dEg, t->pcol, (const int*)mw.offsets,
                       (const int*)mw.cnt_pad, D, (long long)D, rm::kColRows);
    if (e != cudaSuccess) return e;
    if ((e = rm::launch_reduce_parts((const float*)t->pcol, gr.b2, G, nrb_g, D, s)) != cudaSuccess) return e;
    // dS_j = dU_j W1_j (plain bf16 rows)
    rm::GroupedGemm gs{};
    gs.G = G; gs.M = 0; gs.N = D; gs.K = Hd;
    gs.A = t->dUg; gs.a_ld = Hd; gs.a_rows_total = t->rows_max;
    gs.W = w.W1; gs.w_mn = true; gs.w_gstride = (long long)Hd * D; gs.w_ld = D;
    gs.out = t->dSg; gs.o_ld = D;
    gs.epi = rm::EPI_BIAS_GATE;   // no bias, no gate: the product itself
    gs.var_cg = 1;
    gs.grp_cnt = mw.cnt_pad; gs.grp_off = mw.offsets; gs.mtile_prefix = mw.mtile_prefix;
    if ((e = rm::launch_gemm_tc(gs, err, budget, t->num_sms, s)) != cudaSuccess) return e;
    // dW1_j = dU_j^T S_j (fp32)
    rm::GroupedGemm gw1{};
    gw1.G = G; gw1.M = Hd; gw1.N = D; gw1.K = 64;
    gw1.A = t->dUg; gw1.a_mn = true; gw1.a_ld = Hd; gw1.a_rows_total = t->rows_max;
    gw1.W = mw.Sg; gw1.w_mn = true; gw1.w_ld = D;
    gw1.out = gr.W1; gw1.o_gstride = (long long)Hd * D; gw1.o_ld = D;
    gw1.epi = rm::EPI_F32;
    gw1.vark = true; gw1.vark_cnt = mw.cnt_pad; gw1.grp_off = mw.offsets;
    if ((e = rm::launch_gemm_tc(gw1, err, budget, t->num_sms, s)) != cudaSuccess) return e;
    e = rm::launch_pdl(rm::colsum_var_kernel, dim3((Hd / 8 + rm::kThreads - 1) / rm::kThreads, nrb_g, G),
                       dim3(rm::kThreads), 0, s, (const __nv_bfloat16*)t->dUg, t->pcol, (const int*)mw.offsets,
                       (const int*)mw.cnt_pad, Hd, (long long)Hd, rm::kColRows);
    if (e != cudaSuccess) return e;
    if ((e = rm::launch_reduce_parts((const float*)t->pcol, gr.b1, G, nrb_g, Hd, s)) != cudaSuccess) return e;
    // router gradients: dWr[t, j] = sum_b dR[b, t, j] s_bt, dbr[t, j] = sum_b dR[b, t, j]
    const int nrb_b = (B + rm::kColRows - 1) / rm::kColRows;
    for (int pass = 0; pass < (ginf ? 2 : 1); ++pass) {
        const float* dR = pass ? dRinf : t->dR;
        e = rm::launch_router_grad(t->S[l], dR, t->prt, t->prt_b, B, T, D, Ne, rm::kColRows, s);
        if (e != cudaSuccess) return e;
        if ((e = rm::launch_reduce_parts((const float*)t->prt, pass ? gr.Wr_infer : gr.Wr, T, nrb_b, Ne * D, s)) !=
            cudaSuccess)
            return e;
        if ((e = rm::launch_reduce_parts((const float*)t->prt_b, pass ? gr.br_infer : gr.br, T, nrb_b, Ne, s,
                                         t->rscratch)) !=
            cudaSuccess)
            return e;
    }
    // dS = dY (the residual) + sum_j dS_j + the routers' terms
    return rm::launch_moe_bwd_combine(t->dY, t->dSg, mw, t->dR, w.Wr, dRinf, w.Wr_infer, t->dS, B, T, D, Ne, s);
}

}  // namespace

extern "C" {

static void free_trainer(rm_trainer* t) {
    if (!t) return;
    if (t->ws) cudaFree(t->ws);
    delete[] t->S;
    delete[] t->RS1;
    delete[] t->ystats;
    delete[] t->moe;
    delete[] t->gates_inf;
    delete t;
}

rm_status rm_train_create(const rm_config* cfg, rm_trainer** out) {
    if (!cfg || !out) return RM_ERR_INVALID_ARG;
    *out = nullptr;
    const rm_config c = *cfg;
    if (c.B_max < 8 || c.T < 1 || c.D < 1 || c.hidden < 1 || c.L < 1 || c.n_experts < 0) return RM_ERR_INVALID_ARG;
    if (c.dtype != RM_BF16 || !c.mix_addnorm || c.n_experts > 32) return RM_ERR_UNSUPPORTED;
    if (c.act != RM_ACT_GELU_TANH && c.act != RM_ACT_GELU_ERF && c.act != RM_ACT_RELU) return RM_ERR_INVALID_ARG;
    if (c.T > 64 || c.D % c.T || c.D % 64 || c.hidden % 64 || c.D > 2048 || (c.D / c.T) % 8) return RM_ERR_UNSUPPORTED;
    if (!rm::mix_ln_sample_fits(RM_BF16, c.T, c.D)) return RM_ERR_UNSUPPORTED;
    const int rs = rm::mix_pad_stride(c.D, c.D / c.T);
    if (rm::ln1_bwd_smem(c.T, c.D, rs) > 227 * 1024 - 1024) return RM_ERR_UNSUPPORTED;
    const int Ne = c.n_experts;
    const int G = c.T * Ne;
    // (T <= 64 and Ne <= 32: at most 2048 expert groups, the grouped GEMM's limit)
    rm_trainer* t = new (std::nothrow) rm_trainer();
    if (!t) return RM_ERR_OOM;
    t->cfg = c;
    t->budget_ns = 1000000000ull;
    t->lambda = 0.f;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&t->num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        free_trainer(t);
        return RM_ERR_CUDA;
    }
    // the sparse-MoE combine writes whole-row statistics; the dense second
    // projection writes one partial per 64 columns
    t->stat_P = Ne ? 1 : c.D / 64;
    t->SB = 32;
    t->nsb = (c.B_max + t->SB - 1) / t->SB;
    const size_t L = (size_t)c.L, BTD = (size_t)c.B_max * c.T * c.D;
    const size_t TBH = Ne ? 0 : (size_t)c.T * c.B_max * c.hidden;
    const size_t BTN = (size_t)c.B_max * c.T * Ne;                 // (sample, token, expert) entries
    t->rows_max = (long long)BTN + 64LL * G;                        // padded slot lists
    const size_t RM = (size_t)t->rows_max;
    const size_t nrb_rows = (size_t)((c.B_max * c.T + rm::kColRows - 1) / rm::kColRows);
    const size_t nrb_b = (size_t)((c.B_max + rm::kColRows - 1) / rm::kColRows);
    const size_t nrb_g = (size_t)((c.B_max + 64 + rm::kColRows - 1) / rm::kColRows);   // rows per expert <= B + 63
    size_t col_parts = std::max(nrb_rows * c.D, nrb_b * (size_t)c.T * c.hidden);
    if (Ne) col_parts = std::max(col_parts, nrb_g * (size_t)G * std::max(c.D, c.hidden));
    t->S = new (std::nothrow) unsigned char*[5 * L];
    t->RS1 = new (std::nothrow) float*[L];
    t->ystats = new (std::nothrow) float2*[L];
    t->moe = new (std::nothrow) rm::MoeWork[L];
    t->gates_inf = new (std::nothrow) float*[L];
    if (!t->S || !t->RS1 || !t->ystats || !t->moe || !t->gates_inf) {
        free_trainer(t);
        return RM_ERR_OOM;
    }
    t->XH1 = t->S + L;
    t->U = t->S + 2 * L;
    t->H = t->S + 3 * L;
    t->Y = t->S + 4 * L;
    size_t off = 0;
    for (int pass = 0; pass < 2; ++pass) {
        unsigned char* base = pass ? t->ws : nullptr;
        off = 0;
        t->err = carve<int>(base, off, 2 * sizeof(int));
        for (size_t l = 0; l < L; ++l) {
            t->S[l] = carve<unsigned char>(base, off, BTD * 2);
            t->XH1[l] = carve<unsigned char>(base, off, BTD * 2);
            t->RS1[l] = carve<float>(base, off, (size_t)c.B_max * c.T * 4);
            t->U[l] = carve<unsigned char>(base, off, TBH * 2);
            t->H[l] = carve<unsigned char>(base, off, TBH * 2);
            t->Y[l] = carve<unsigned char>(base, off, BTD * 2);
            t->ystats[l] = carve<float2>(base, off, (size_t)c.B_max * c.T * t->stat_P * 8);
            rm::MoeWork& m = t->moe[l];
            m = rm::MoeWork{};
            t->gates_inf[l] = nullptr;
            if (Ne) {
                m.gates = carve<float>(base, off, BTN * 4);
                m.counts = carve<int>(base, off, (size_t)G * 4);
                m.offsets = carve<int>(base, off, (size_t)G * 4);
                m.cnt_pad = carve<int>(base, off, (size_t)G * 4);
                m.mtile_prefix = carve<int>(base, off, (size_t)(G + 1) * 4);
                m.totals = carve<int>(base, off, 2 * 4);
                m.slot_row = carve<int>(base, off, RM * 4);
                m.slot_gate = carve<float>(base, off, RM * 4);
                m.slot_of = carve<int>(base, off, BTN * 4);
                m.Sg = carve<unsigned char>(base, off, RM * c.D * 2);
                m.Hg = carve<unsigned char>(base, off, RM * c.hidden * 2);
                m.Eg = carve<unsigned char>(base, off, RM * c.D * 2);
                t->U[l] = carve<unsigned char>(base, off, RM * c.hidden * 2);   // the experts' activation input
                t->gates_inf[l] = carve<float>(base, off, BTN * 4);
            }
        }
        t->pooled = carve<float>(base, off, (size_t)c.B_max * c.D * 4);
        t->dlogit = carve<float>(base, off, (size_t)c.B_max * 4);
        t->lterm = carve<float>(base, off, (size_t)c.B_max * 4);
        t->gpool = carve<float>(base, off, (size_t)c.B_max * c.D * 4);
        t->dY = carve<unsigned char>(base, off, BTD * 2);
        t->dU = carve<unsigned char>(base, off, TBH * 2);
        t->dS = carve<unsigned char>(base, off, BTD * 2);
        t->dX = carve<unsigned char>(base, off, BTD * 2);
        t->pg = carve<float>(base, off, (size_t)c.T * t->nsb * c.D * 4);
        t->pb = carve<float>(base, off, (size_t)c.T * t->nsb * c.D * 4);
        t->pdb = carve<float>(base, off, (size_t)c.T * t->nsb * c.D * 4);
        t->pcol = carve<float>(base, off, col_parts * 4);
        t->pcol2 = carve<float>(base, off, col_parts * 4);
        {
            const size_t ch = (size_t)rm::kRedChunk;
            const size_t r1 = (nrb_rows + ch - 1) / ch * c.D, r2 = ((size_t)c.T * t->nsb + ch - 1) / ch * c.D;
            const size_t r3 = (nrb_b + ch - 1) / ch * (size_t)c.T * std::max(Ne, 1);
            t->rscratch = carve<float>(base, off, std::max(std::max(r1, r2), r3) * 4);
        }
        t->lreg_part = carve<float>(base, off, 256 * 4);
        t->sk_cnt = carve<int>(base, off, rm::gemm_tc_split_cnt_ints(t->num_sms) * sizeof(int));
        t->sk_ws = carve<float>(base, off, rm::gemm_tc_split_ws_bytes(t->num_sms));
        if (Ne) {
            t->dEg = carve<unsigned char>(base, off, RM * c.D * 2);
            t->dUg = carve<unsigned char>(base, off, RM * c.hidden * 2);
            t->dSg = carve<unsigned char>(base, off, RM * c.D * 2);
            t->dR = carve<float>(base, off, BTN * 4);
            t->dRinf = carve<float>(base, off, BTN * 4);
            t->prt = carve<float>(base, off, (size_t)c.T * nrb_b * Ne * c.D * 4);
            t->prt_b = carve<float>(base, off, (size_t)c.T * nrb_b * Ne * 4);
            t->cnt_scratch = carve<int>(base, off, (size_t)G * 4);
        }
        if (pass == 0) {
            t->ws_bytes = off;
            if (cudaMalloc(&t->ws, off) != cudaSuccess) {
                cudaGetLastError();
                t->ws = nullptr;
                free_trainer(t);
                return RM_ERR_OOM;
            }
        }
    }
    if (cudaMemset(t->ws, 0, t->ws_bytes) != cudaSuccess) {
        free_trainer(t);
        return RM_ERR_CUDA;
    }
    *out = t;
    return RM_OK;
}

rm_status rm_train_destroy(rm_trainer* t) {
    if (!t) return RM_ERR_INVALID_ARG;
    cudaDeviceSynchronize();
    free_trainer(t);
    return RM_OK;
}

rm_status rm_train_set_reg(rm_trainer* t, float lambda) {
    if (!t || !(lambda >= 0.f)) return RM_ERR_INVALID_ARG;
    t->lambda = lambda;
    return RM_OK;
}

size_t rm_train_workspace_bytes(const rm_trainer* t) { return t ? t->ws_bytes : 0; }

rm_status rm_train_sync_status(rm_trainer* t, rm_stream_t stream) {
    if (!t) return RM_ERR_INVALID_ARG;
    int word = 0;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return RM_ERR_CUDA;
    if (cudaMemcpy(&word, t->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return RM_ERR_CUDA;
    return (rm_status)word;
}

rm_status rm_train_step(rm_trainer* t, const rm_block_weights* blocks, const void* X0, const void* head_w,
                        const float* head_b, const float* labels, const rm_block_grads* grads, void* dX0,
                        float* dhead_w, float* dhead_b, float* loss, float* pooled_out, int B, rm_stream_t stream) {
    if (!t || !blocks || !grads || !aligned16(X0) || !aligned16(head_w) || !head_b || !aligned16(labels) ||
        !aligned16(dhead_w) || !dhead_b || !loss)
        return RM_ERR_INVALID_ARG;
    const rm_config& c = t->cfg;
    if (B < 8 || B > c.B_max || B % 8) return RM_ERR_INVALID_ARG;
    if (dX0 && !aligned16(dX0)) return RM_ERR_INVALID_ARG;
    if (pooled_out && !aligned16(pooled_out)) return RM_ERR_INVALID_ARG;
    for (int l = 0; l < c.L; ++l) {
        const rm_block_weights& w = blocks[l];
        const rm_block_grads& g = grads[l];
        if (!aligned16(w.W1) || !aligned16(w.b1) || !aligned16(w.W2) || !aligned16(w.b2) || !aligned16(w.ln1_g) ||
            !aligned16(w.ln1_b) || !aligned16(w.ln2_g) || !aligned16(w.ln2_b))
            return RM_ERR_INVALID_ARG;
        if (!aligned16(g.W1) || !aligned16(g.b1) || !aligned16(g.W2) || !aligned16(g.b2) || !aligned16(g.ln1_g) ||
            !aligned16(g.ln1_b) || !aligned16(g.ln2_g) || !aligned16(g.ln2_b))
            return RM_ERR_INVALID_ARG;
        if (c.n_experts) {   // routers (and DTSI's second router, when given)
            if (!aligned16(w.Wr) || !w.br || !aligned16(g.Wr) || !g.br) return RM_ERR_INVALID_ARG;
            if (w.Wr_infer && (!aligned16(w.Wr_infer) || !w.br_infer || !aligned16(g.Wr_infer) || !g.br_infer))
                return RM_ERR_INVALID_ARG;
        }
    }
    cudaStream_t s = stream;
    const int T = c.T, D = c.D, Hd = c.hidden, L = c.L, P = t->stat_P, Ne = c.n_experts, G = T * Ne;
    const rm::DeviceErr err = terr(t);
    const uint64_t budget = t->budget_ns;
    cudaError_t e = cudaSuccess;
#define RM_TRY(x)                          \
    do {                                   \
        e = (x);                           \
        if (e != cudaSuccess) return RM_ERR_CUDA; \
    } while (0)

    // ------------------------------------------------------------ forward
    for (int l = 0; l < L; ++l) {
        const rm_block_weights& w = blocks[l];
        const rm_block_weights* prev = l ? &blocks[l - 1] : nullptr;
        RM_TRY(rm::launch_mix_ln(RM_BF16, l ? (const void*)t->Y[l - 1] : X0, prev ? prev->ln2_g : nullptr,
                                 prev ? prev->ln2_b : nullptr, rm::RowStats{l ? t->ystats[l - 1] : nullptr, P},
                                 w.ln1_g, w.ln1_b, t->S[l], B, T, D, c.ln_eps, 1, t->num_sms, err, budget, s,
                                 t->XH1[l], t->RS1[l]));
        if (Ne) {
            // sparse MoE: route (slot lists padded per expert to a multiple of
            // 64), DTSI's second router, gather, the expert projections (the
            // first also stores its activation input), combine
            rm::MoeWork& mw = t->moe[l];
            RM_TRY(rm::launch_moe_route(t->S[l], w.Wr, w.br, mw, B, T, D, Ne, s, 128));
            if (w.Wr_infer)
                RM_TRY(rm::launch_moe_route_only(t->S[l], w.Wr_infer, w.br_infer, t->gates_inf[l], t->cnt_scratch, B, T,
                                                 D, Ne, s));
            RM_TRY(rm::launch_moe_gather(t->S[l], mw, B, T, D, Ne, s));
            rm::GroupedGemm e1{};
            e1.G = G; e1.M = 0; e1.N = Hd; e1.K = D;
            e1.A = mw.Sg; e1.a_ld = D; e1.a_rows_total = t->rows_max;
            e1.W = w.W1;
            e1.out = mw.Hg; e1.o_ld = Hd;
            e1.resid = t->U[l]; e1.r_ld = Hd;   // the activation input, stored
            e1.bias = static_cast<const float*>(w.b1);
            e1.epi = rm::epi_for_act(c.act);
            e1.var_cg = 1;
            e1.grp_cnt = mw.cnt_pad; e1.grp_off = mw.offsets; e1.mtile_prefix = mw.mtile_prefix;
            RM_TRY(rm::launch_gemm_tc(e1, err, budget, t->num_sms, s));
            rm::GroupedGemm e2 = e1;
            e2.N = D; e2.K = Hd;
            e2.A = mw.Hg; e2.a_ld = Hd;
            e2.W = w.W2;
            e2.out = mw.Eg; e2.o_ld = D;
            e2.resid = nullptr; e2.r_ld = 0;
            e2.bias = static_cast<const float*>(w.b2);
            e2.gate = mw.slot_gate;
            e2.epi = rm::EPI_BIAS_GATE;
            RM_TRY(rm::launch_gemm_tc(e2, err, budget, t->num_sms, s));
            RM_TRY(rm::launch_moe_combine(mw, t->S[l], t->Y[l], t->ystats[l], B, T, D, Ne, s));
            continue;
        }
        rm::GroupedGemm g1{};
        g1.G = T; g1.M = B; g1.N = Hd; g1.K = D;
        g1.A = t->S[l]; g1.a_gstride = D; g1.a_ld = (long long)T * D;
        g1.W = w.W1;
        g1.out = t->H[l]; g1.o_gstride = (long long)B * Hd; g1.o_ld = Hd;
        g1.resid = t->U[l]; g1.r_gstride = (long long)B * Hd; g1.r_ld = Hd;   // the activation input, stored
        g1.bias = static_cast<const float*>(w.b1);
        g1.epi = rm::epi_for_act(c.act);
        RM_TRY(rm::launch_gemm_tc(g1, err, budget, t->num_sms, s));
        rm::GroupedGemm g2{};
        g2.G = T; g2.M = B; g2.N = D; g2.K = Hd;
        g2.A = t->H[l]; g2.a_gstride = (long long)B * Hd; g2.a_ld = Hd;
        g2.W = w.W2;
        g2.out = t->Y[l]; g2.o_gstride = D; g2.o_ld = (long long)T * D;
        g2.bias = static_cast<const float*>(w.b2);
        g2.resid = t->S[l]; g2.r_gstride = D; g2.r_ld = (long long)T * D;
        g2.epi = rm::EPI_BIAS_RESID;
        g2.stats = t->ystats[l]; g2.s_gstride = P; g2.s_ld = (long long)T * P;
        g2.sk_ws = t->sk_ws; g2.sk_cnt = t->sk_cnt;
        RM_TRY(rm::launch_gemm_tc(g2, err, budget, t->num_sms, s));
    }
    const rm_block_weights& last = blocks[L - 1];
    RM_TRY(rm::launch_ln_pool(RM_BF16, t->Y[L - 1], rm::RowStats{t->ystats[L - 1], P}, last.ln2_g, last.ln2_b,
                              t->pooled, nullptr, B, T, D, c.ln_eps, t->num_sms, err, budget, s));
    if (pooled_out)
        RM_TRY(cudaMemcpyAsync(pooled_out, t->pooled, (size_t)B * D * 4, cudaMemcpyDeviceToDevice, s));

    // ------------------------------------------------------- loss and head
    const __nv_bfloat16* hw = static_cast<const __nv_bfloat16*>(head_w);
    RM_TRY(rm::launch_pdl(rm::head_logit_kernel, dim3((B + 7) / 8), dim3(rm::kThreads), 0, s,
                          (const float*)t->pooled, hw, head_b, labels, t->dlogit, t->lterm, B, D));
    RM_TRY(rm::launch_pdl(rm::head_grad_kernel, dim3((D + 31) / 32), dim3(32 * rm::kRedWarps), 0, s,
                          (const float*)t->pooled, hw, (const float*)t->dlogit, (const float*)t->lterm, dhead_w,
                          dhead_b, loss, t->gpool, B, D, 1.0f / T));
    if (Ne && t->lambda > 0.f)   // + lambda L_reg: the regularised gates of every MoE block, in block order
        for (int l = 0; l < L; ++l)
            RM_TRY(rm::launch_add_scaled_sum(blocks[l].Wr_infer ? t->gates_inf[l] : t->moe[l].gates,
                                             (long long)B * T * Ne, t->lambda, loss, t->lreg_part, s));

    // ------------------------------------------------------------ backward
    const int nsb = (B + t->SB - 1) / t->SB;
    const int nv = D / 8;
    const int lnb_threads = (nv + 31) / 32 * 32;
    if (lnb_threads > rm::kThreads) return RM_ERR_UNSUPPORTED;
    for (int l = L - 1; l >= 0; --l) {
        const rm_block_weights& w = blocks[l];
        const rm_block_grads& gr = grads[l];
        const __nv_bfloat16* Yl = reinterpret_cast<const __nv_bfloat16*>(t->Y[l]);
        __nv_bfloat16* dY = reinterpret_cast<__nv_bfloat16*>(t->dY);
        // LN2 backward: dY, and the partial sums of dgamma2, dbeta2, db2
        if (l == L - 1)
            RM_TRY(rm::launch_pdl(rm::ln2_bwd_kernel<true>, dim3(nsb, T), dim3(lnb_threads), 0, s,
                                  (const __nv_bfloat16*)nullptr, (const float*)t->gpool, Yl,
                                  (const float2*)t->ystats[l], P, w.ln2_g, c.ln_eps, dY, t->pg, t->pb, t->pdb, B, T,
                                  D, t->SB));
        else
            RM_TRY(rm::launch_pdl(rm::ln2_bwd_kernel<false>, dim3(nsb, T), dim3(lnb_threads), 0, s,
                                  (const __nv_bfloat16*)t->dX, (const float*)nullptr, Yl, (const float2*)t->ystats[l],
                                  P, w.ln2_g, c.ln_eps, dY, t->pg, t->pb, t->pdb, B, T, D, t->SB));
        RM_TRY(rm::launch_reduce_parts((const float*)t->pg, gr.ln2_g, 1, T * nsb, D, s, t->rscratch));
        RM_TRY(rm::launch_reduce_parts((const float*)t->pb, gr.ln2_b, 1, T * nsb, D, s, t->rscratch));
        if (Ne) {
            RM_TRY(moe_backward(t, w, gr, l, B, s));
        } else {
        RM_TRY(rm::launch_reduce_parts((const float*)t->pdb, gr.b2, T, nsb, D, s));
        // dU = (dY W2_t) * act'(U)
        rm::GroupedGemm gh{};
        gh.G = T; gh.M = B; gh.N = Hd; gh.K = D;
        gh.A = t->dY; gh.a_gstride = D; gh.a_ld = (long long)T * D;
        gh.W = w.W2; gh.w_mn = true; gh.w_gstride = (long long)D * Hd; gh.w_ld = Hd;
        gh.out = t->dU; gh.o_gstride = (long long)B * Hd; gh.o_ld = Hd;
        gh.resid = t->U[l]; gh.r_gstride = (long long)B * Hd; gh.r_ld = Hd;
        gh.epi = rm::dact_epi_for_act(c.act);
        gh.sk_ws = t->sk_ws; gh.sk_cnt = t->sk_cnt;
        RM_TRY(rm::launch_gemm_tc(gh, err, budget, t->num_sms, s));
        // dW2_t = dY_t^T Hh_t (fp32)
        rm::GroupedGemm gw2{};
        gw2.G = T; gw2.M = D; gw2.N = Hd; gw2.K = B;
        gw2.A = t->dY; gw2.a_mn = true; gw2.a_gstride = D; gw2.a_ld = (long long)T * D;
        gw2.W = t->H[l]; gw2.w_mn = true; gw2.w_gstride = (long long)B * Hd; gw2.w_ld = Hd; gw2.w_from_kernel = true;
        gw2.out = gr.W2; gw2.o_gstride = (long long)D * Hd; gw2.o_ld = Hd;
        gw2.epi = rm::EPI_F32;
        gw2.sk_ws = t->sk_ws; gw2.sk_cnt = t->sk_cnt;
        RM_TRY(rm::launch_gemm_tc(gw2, err, budget, t->num_sms, s));
        // db1_t = sum_b dU
        const int nrb_b = (B + rm::kColRows - 1) / rm::kColRows;
        RM_TRY(rm::launch_pdl(rm::colsum_kernel, dim3((Hd / 8 + rm::kThreads - 1) / rm::kThreads, nrb_b, T),
                              dim3(rm::kThreads), 0, s, (const __nv_bfloat16*)t->dU, (const __nv_bfloat16*)nullptr,
                              t->pcol, (float*)nullptr, B, Hd, (long long)B * Hd, (long long)Hd, rm::kColRows));
        RM_TRY(rm::launch_reduce_parts((const float*)t->pcol, gr.b1, T, nrb_b, Hd, s));
        // dS = dU W1_t + dY
        rm::GroupedGemm gs{};
        gs.G = T; gs.M = B; gs.N = D; gs.K = Hd;
        gs.A = t->dU; gs.a_gstride = (long long)B * Hd; gs.a_ld = Hd;
        gs.W = w.W1; gs.w_mn = true; gs.w_gstride = (long long)Hd * D; gs.w_ld = D;
        gs.out = t->dS; gs.o_gstride = D; gs.o_ld = (long long)T * D;
        gs.resid = t->dY; gs.r_gstride = D; gs.r_ld = (long long)T * D;
        gs.epi = rm::EPI_BIAS_RESID;
        gs.sk_ws = t->sk_ws; gs.sk_cnt = t->sk_cnt;
        RM_TRY(rm::launch_gemm_tc(gs, err, budget, t->num_sms, s));
        // dW1_t = dU_t^T S_t (fp32)
        rm::GroupedGemm gw1{};
        gw1.G = T; gw1.M = Hd; gw1.N = D; gw1.K = B;
        gw1.A = t->dU; gw1.a_mn = true; gw1.a_gstride = (long long)B * Hd; gw1.a_ld = Hd;
        gw1.W = t->S[l]; gw1.w_mn = true; gw1.w_gstride = D; gw1.w_ld = (long long)T * D; gw1.w_from_kernel = true;
        gw1.out = gr.W1; gw1.o_gstride = (long long)Hd * D; gw1.o_ld = D;
        gw1.epi = rm::EPI_F32;
        gw1.sk_ws = t->sk_ws; gw1.sk_cnt = t->sk_cnt;
        RM_TRY(rm::launch_gemm_tc(gw1, err, budget, t->num_sms, s));
        }
        // dgamma1 = sum dS * xhat1, dbeta1 = sum dS over every row
        const int nrb = (B * T + rm::kColRows - 1) / rm::kColRows;
        RM_TRY(rm::launch_pdl(rm::colsum_kernel, dim3((D / 8 + rm::kThreads - 1) / rm::kThreads, nrb, 1),
                              dim3(rm::kThreads), 0, s, (const __nv_bfloat16*)t->dS,
                              (const __nv_bfloat16*)t->XH1[l], t->pcol, t->pcol2, B * T, D, 0LL, (long long)D,
                              rm::kColRows));
        RM_TRY(rm::launch_reduce_parts((const float*)t->pcol2, gr.ln1_g, 1, nrb, D, s, t->rscratch));
        RM_TRY(rm::launch_reduce_parts((const float*)t->pcol, gr.ln1_b, 1, nrb, D, s, t->rscratch));
        // LN1 backward and the mixing's transpose: dX (the stack input's gradient for l = 0)
        __nv_bfloat16* dXo = (l == 0 && dX0) ? static_cast<__nv_bfloat16*>(dX0)
                                             : reinterpret_cast<__nv_bfloat16*>(t->dX);
        const int rs = rm::mix_pad_stride(D, D / T);
        const size_t smem = rm::ln1_bwd_smem(T, D, rs);
        const int groups = [&] {
            int g = rm::kBwdMixThreads / nv;
            if (g > T) g = T;
            if (g < 1) g = 1;
            return g;
        }();
        const int nvl = (nv + 31) / 32;
        auto go = [&](auto kern) -> cudaError_t {
            cudaError_t ee = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (ee != cudaSuccess) return ee;
            const int grid = std::min(B, 2 * t->num_sms);
            return rm::launch_pdl(kern, dim3(grid), dim3(rm::kBwdMixThreads), smem, s, (const __nv_bfloat16*)t->dS,
                                  (const __nv_bfloat16*)t->XH1[l], (const float*)t->RS1[l], w.ln1_g, dXo, B, T, D, rs,
                                  groups, err, budget);
        };
        switch (nvl) {
            case 1: RM_TRY(go(rm::ln1_bwd_mix_kernel<1>)); break;
            case 2: RM_TRY(go(rm::ln1_bwd_mix_kernel<2>)); break;
            case 3: RM_TRY(go(rm::ln1_bwd_mix_kernel<3>)); break;
            case 4: RM_TRY(go(rm::ln1_bwd_mix_kernel<4>)); break;
            case 5: RM_TRY(go(rm::ln1_bwd_mix_kernel<5>)); break;
            case 6: RM_TRY(go(rm::ln1_bwd_mix_kernel<6>)); break;
            case 7: RM_TRY(go(rm::ln1_bwd_mix_kernel<7>)); break;
            default: RM_TRY(go(rm::ln1_bwd_mix_kernel<8>)); break;
        }
    }
#undef RM_TRY
    return RM_OK;
}

}  // extern "C"
