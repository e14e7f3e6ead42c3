// Sparse-MoE routing for the per-token FFN: ReLU gates, deterministic
// compaction of active (sample, token, expert) entries into per-expert row
// lists, row gather, and the fixed-order combine.
//
// ReLU routing (fun-rec chapter "Rankmixer: 硬件效率优化", section Sparse
// MoE扩展): G[b, t, j] = ReLU(h_t(s)), v = sum_j G[b, t, j] e_{t,j}(s), with
// no softmax and no top-k, so each token activates a data-dependent number
// of experts; an expert whose gate is 0 contributes nothing and is not
// evaluated.  Router h_t is linear: logits = Wr_t s + br_t.
//
// Everything stays on the device: counts, offsets and the expert GEMMs' tile
// list are produced here and read by the grouped GEMM without a host round
// trip.  Expert g = t * Ne + j owns slots [offsets[g], offsets[g] + counts[g])
// in ascending sample order.
#include <cuda_bf16.h>

#include "rm_device.cuh"

namespace rm {
namespace {

constexpr int kThreads = 256;

// One warp per (b, t) row of S.  NE is the compile-time capacity (>= Ne).
template <int NE>
__global__ void __launch_bounds__(kThreads) route_kernel(const __nv_bfloat16* __restrict__ S,
                                                         const float* __restrict__ Wr,
                                                         const float* __restrict__ br, float* __restrict__ gates,
                                                         int* __restrict__ counts, long long rows, int T, int D,
                                                         int Ne) {
    const int lane = threadIdx.x & 31;
    const long long r = blockIdx.x * (long long)(blockDim.x >> 5) + (threadIdx.x >> 5);
    if (r >= rows) return;
    const int t = (int)(r % T);
    const __nv_bfloat16* srow = S + r * D;
    const float* w = Wr + (long long)t * Ne * D;
    float acc[NE];
#pragma unroll
    for (int j = 0; j < NE; ++j) acc[j] = 0.f;
    for (int v = lane; v < D / 8; v += 32) {
        Vec16<__nv_bfloat16> x;
        x.u = __ldg(reinterpret_cast<const uint4*>(srow) + v);
        float xf[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) xf[e] = __bfloat162float(x.e[e]);
#pragma unroll
        for (int j = 0; j < NE; ++j) {
            if (j < Ne) {
                const float4* w4 = reinterpret_cast<const float4*>(w + (long long)j * D + v * 8);
                const float4 a = __ldg(w4), b = __ldg(w4 + 1);
                acc[j] += xf[0] * a.x + xf[1] * a.y + xf[2] * a.z + xf[3] * a.w + xf[4] * b.x + xf[5] * b.y +
                          xf[6] * b.z + xf[7] * b.w;
            }
        }
    }
#pragma unroll
    for (int j = 0; j < NE; ++j) {
        if (j < Ne) {
            const float logit = warp_sum(acc[j]) + __ldg(br + (long long)t * Ne + j);
            const float gate = logit > 0.f ? logit : 0.f;
            if (lane == 0) {
                gates[r * Ne + j] = gate;
                if (gate > 0.f) atomicAdd(counts + (long long)t * Ne + j, 1);
            }
        }
    }
}

__device__ __forceinline__ int warp_isum(int v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// One CTA of 1024 threads per expert g = t * Ne + j: its slot offset and
// m-tile prefix (sums over the experts before it), then the list of samples
// b (ascending) whose gate is > 0.
__global__ void __launch_bounds__(1024) compact_kernel(const float* __restrict__ gates,
                                                       const int* __restrict__ counts, int* __restrict__ offsets,
                                                       int* __restrict__ mtile_prefix, int* __restrict__ totals,
                                                       int* __restrict__ slot_row, float* __restrict__ slot_gate,
                                                       int* __restrict__ slot_of, int B, int T, int Ne) {
    __shared__ int s_off;
    __shared__ int s_warp[32];
    const int G = T * Ne;
    const int g = blockIdx.x;
    const int t = g / Ne, j = g - t * Ne;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (warp == 0) {
        int off = 0, mt = 0;
        for (int q = lane; q < g; q += 32) {
            const int c = counts[q];
            off += c;
            mt += (c + 127) / 128;
        }
        off = warp_isum(off);
        mt = warp_isum(mt);
        if (lane == 0) {
            s_off = off;
            offsets[g] = off;
            mtile_prefix[g] = mt;
            if (g == G - 1) {
                const int c = counts[g];
                mtile_prefix[G] = mt + (c + 127) / 128;
                totals[0] = off + c;
                totals[1] = mt + (c + 127) / 128;
            }
        }
    }
    __syncthreads();
    const int off = s_off;
    int base = 0;
    for (int b0 = 0; b0 < B; b0 += 1024) {
        const int b = b0 + threadIdx.x;
        const long long e = ((long long)b * T + t) * Ne + j;
        const float gate = b < B ? gates[e] : 0.f;
        const bool act = gate > 0.f;
        const unsigned m = __ballot_sync(0xffffffffu, act);
        const int before = __popc(m & ((1u << lane) - 1u));
        if (lane == 0) s_warp[warp] = __popc(m);
        __syncthreads();
        int wbase = 0, blk = 0;
        for (int q = 0; q < 32; ++q) {
            const int c = s_warp[q];
            if (q < warp) wbase += c;
            blk += c;
        }
        if (b < B) {
            if (act) {
                const int slot = off + base + wbase + before;
                slot_row[slot] = b * T + t;
                slot_gate[slot] = gate;
                slot_of[e] = slot;
            } else {
                slot_of[e] = -1;
            }
        }
        base += blk;
        __syncthreads();
    }
}

// Sg[slot] = S[slot_row[slot]]: one warp per active slot, 16-byte vectors.
__global__ void __launch_bounds__(kThreads) gather_kernel(const __nv_bfloat16* __restrict__ S,
                                                          const int* __restrict__ slot_row,
                                                          const int* __restrict__ totals,
                                                          __nv_bfloat16* __restrict__ Sg, int D) {
    const int lane = threadIdx.x & 31;
    const int n = totals[0];
    const int nv = D / 8;
    for (long long s = blockIdx.x * (long long)(blockDim.x >> 5) + (threadIdx.x >> 5); s < n;
         s += (long long)gridDim.x * (blockDim.x >> 5)) {
        const uint4* src = reinterpret_cast<const uint4*>(S + (long long)slot_row[s] * D);
        uint4* dst = reinterpret_cast<uint4*>(Sg + s * D);
        for (int v = lane; v < nv; v += 32) dst[v] = __ldg(src + v);
    }
}

// out[r] = resid[r] + sum over j ascending of Eg[slot_of[r, j]] (active only),
// summed in fp32.  One warp per (b, t) row.
__global__ void __launch_bounds__(kThreads) combine_kernel(const __nv_bfloat16* __restrict__ Eg,
                                                           const int* __restrict__ slot_of,
                                                           const __nv_bfloat16* __restrict__ resid,
                                                           __nv_bfloat16* __restrict__ out, long long rows, int D,
                                                           int Ne) {
    const int lane = threadIdx.x & 31;
    const long long r = blockIdx.x * (long long)(blockDim.x >> 5) + (threadIdx.x >> 5);
    if (r >= rows) return;
    const int nv = D / 8;
    for (int v = lane; v < nv; v += 32) {
        float acc[8];
        if (resid) {
            Vec16<__nv_bfloat16> x;
            x.u = __ldg(reinterpret_cast<const uint4*>(resid + r * D) + v);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = __bfloat162float(x.e[e]);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = 0.f;
        }
        for (int j = 0; j < Ne; ++j) {
            const int slot = __ldg(slot_of + r * Ne + j);
            if (slot < 0) continue;
            Vec16<__nv_bfloat16> x;
            x.u = __ldg(reinterpret_cast<const uint4*>(Eg + (long long)slot * D) + v);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] += __bfloat162float(x.e[e]);
        }
        uint4 o;
        o.x = pack_bf16x2(acc[0], acc[1]);
        o.y = pack_bf16x2(acc[2], acc[3]);
        o.z = pack_bf16x2(acc[4], acc[5]);
        o.w = pack_bf16x2(acc[6], acc[7]);
        reinterpret_cast<uint4*>(out + r * D)[v] = o;
    }
}

}  // namespace

cudaError_t launch_moe_route(const void* S, const float* Wr, const float* br, const MoeWork& w, int B, int T,
                             int D, int Ne, cudaStream_t s) {
    cudaError_t e = cudaMemsetAsync(w.counts, 0, sizeof(int) * T * Ne, s);
    if (e != cudaSuccess) return e;
    const long long rows = (long long)B * T;
    const int grid = (int)((rows + kThreads / 32 - 1) / (kThreads / 32));
    const auto* Sb = static_cast<const __nv_bfloat16*>(S);
    if (Ne <= 1) route_kernel<1><<<grid, kThreads, 0, s>>>(Sb, Wr, br, w.gates, w.counts, rows, T, D, Ne);
    else if (Ne <= 2) route_kernel<2><<<grid, kThreads, 0, s>>>(Sb, Wr, br, w.gates, w.counts, rows, T, D, Ne);
    else if (Ne <= 4) route_kernel<4><<<grid, kThreads, 0, s>>>(Sb, Wr, br, w.gates, w.counts, rows, T, D, Ne);
    else if (Ne <= 8) route_kernel<8><<<grid, kThreads, 0, s>>>(Sb, Wr, br, w.gates, w.counts, rows, T, D, Ne);
    else if (Ne <= 16) route_kernel<16><<<grid, kThreads, 0, s>>>(Sb, Wr, br, w.gates, w.counts, rows, T, D, Ne);
    else route_kernel<32><<<grid, kThreads, 0, s>>>(Sb, Wr, br, w.gates, w.counts, rows, T, D, Ne);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    compact_kernel<<<T * Ne, 1024, 0, s>>>(w.gates, w.counts, w.offsets, w.mtile_prefix, w.totals, w.slot_row,
                                           w.slot_gate, w.slot_of, B, T, Ne);
    return cudaGetLastError();
}

cudaError_t launch_moe_gather(const void* S, const MoeWork& w, int B, int T, int D, int Ne, cudaStream_t s) {
    (void)B;
    (void)T;
    (void)Ne;
    gather_kernel<<<148 * 8, kThreads, 0, s>>>(static_cast<const __nv_bfloat16*>(S), w.slot_row, w.totals,
                                               static_cast<__nv_bfloat16*>(w.Sg), D);
    return cudaGetLastError();
}

cudaError_t launch_moe_combine(const MoeWork& w, const void* resid, void* out, int B, int T, int D, int Ne,
                               cudaStream_t s) {
    const long long rows = (long long)B * T;
    const int grid = (int)((rows + kThreads / 32 - 1) / (kThreads / 32));
    combine_kernel<<<grid, kThreads, 0, s>>>(static_cast<const __nv_bfloat16*>(w.Eg), w.slot_of,
                                             static_cast<const __nv_bfloat16*>(resid),
                                             static_cast<__nv_bfloat16*>(out), rows, D, Ne);
    return cudaGetLastError();
}

}  // namespace rm
