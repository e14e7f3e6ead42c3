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

#include <algorithm>

#include "rm_device.cuh"

namespace rm {
namespace {

constexpr int kThreads = 256;

// Router logits, ReLU gates and per-expert active counts.  CTA (t, chunk)
// stages router t's weights Wr_t [Ne][D] in shared memory once (before the
// launch wait: no kernel of the forward pass writes router weights) and
// serves `rows` samples b (chosen on the host so the grid fills the SMs in
// one wave).  A warp takes RW = max(1, 16 / NE) rows (b, t) of S at a time:
// lane l multiplies the 8-column vectors l, l + 32, ... of those rows (all
// their 16-byte loads issued before the first multiply) with all NE experts,
// in paired fp32 accumulators, so each staged weight vector feeds RW rows and
// each S vector NE experts.  The weights are staged split by halves of each
// 8-column vector ([Ne][2][D/8] float4s), so the lanes' 16-byte shared loads
// are consecutive (conflict-free).  The NA = RW x NE partial dot products per
// lane (16 or 32) are reduced across the warp by a transposing butterfly,
// after which lane l holds the logit of entry l % NA (row (l % NA) / NE,
// expert l % NE).  Active counts are summed in shared memory and added to the
// global counts once per CTA.

// acc[i] summed over the warp (N = 16 or 32); afterwards acc[0] of lane l
// is the sum of everyone's acc[l % N].
template <int N>
__device__ __forceinline__ void warp_reduce_transpose(float (&acc)[N]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = N / 2; o >= 1; o >>= 1) {
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < o; ++i) {
            const float send = upper ? acc[i] : acc[i + o];
            const float keep = upper ? acc[i + o] : acc[i];
            acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
    if constexpr (N == 16) acc[0] += __shfl_xor_sync(0xffffffffu, acc[0], 16);
}

// 16-byte S vectors per row and lane per pass: two for up to two rows per
// warp pass, else one; three CTAs per SM for NE = 8 or 16 (two for 32).
template <int NE>
__global__ void __launch_bounds__(kThreads, NE == 32 ? 2 : (NE >= 8 ? 3 : 1)) route_kernel(const __nv_bfloat16* __restrict__ S,
                                                            const float* __restrict__ Wr,
                                                            const float* __restrict__ br, float* __restrict__ gates,
                                                            int* __restrict__ counts, int B, int T, int D, int Ne,
                                                            int rows) {
    pdl_trigger();
    constexpr int RW = NE < 16 ? 16 / NE : 1;   // rows per warp pass
    constexpr int NA = RW * NE;                 // dot products per lane: 16 or 32
    constexpr int KV = RW <= 2 ? 2 : 1;
    extern __shared__ __align__(16) float4 wsm4[];   // [Ne][2][D/8]
    __shared__ int cnt[NE];
    const int t = blockIdx.x;
    const int b0 = blockIdx.y * rows;
    const int bend = min(B, b0 + rows);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int nv = D / 8;   // 8-column vectors per row
    {
        const float4* src = reinterpret_cast<const float4*>(Wr + (size_t)t * Ne * D);
        const int nq = D / 4;
        for (int i = threadIdx.x; i < Ne * nq; i += blockDim.x) {
            const int j = i / nq, q = i - j * nq;   // columns 4q .. 4q+3 of expert j: half q & 1 of vector q / 2
            wsm4[(2 * j + (q & 1)) * nv + (q >> 1)] = __ldg(src + i);
        }
        if (threadIdx.x < NE) cnt[threadIdx.x] = 0;
    }
    const int ia = lane % NA;
    const int jl = ia % NE, rl = ia / NE;   // this lane's (row, expert) after the reduction
    const float bias = jl < Ne ? __ldg(br + (long long)t * Ne + jl) : 0.f;
    pdl_wait();
    __syncthreads();
    for (int bw = b0 + warp * RW; bw < bend; bw += nw * RW) {
        float2 acc2[NA];   // [row q][expert j], even / odd columns
#pragma unroll
        for (int i = 0; i < NA; ++i) acc2[i] = f2(0.f);
        for (int v0 = 0; v0 < nv; v0 += 32 * KV) {
            uint4 xs[RW][KV];
#pragma unroll
            for (int q = 0; q < RW; ++q) {
                const int b = bw + q;
                const uint4* row = reinterpret_cast<const uint4*>(S + ((long long)b * T + t) * D);
#pragma unroll
                for (int k = 0; k < KV; ++k) {
                    const int v = v0 + lane + 32 * k;
                    xs[q][k] = (b < bend && v < nv) ? __ldcg(row + v) : make_uint4(0u, 0u, 0u, 0u);
                }
            }
#pragma unroll
            for (int k = 0; k < KV; ++k) {
                const int v = v0 + lane + 32 * k;
                if (v < nv) {
                    float2 xf[RW][4];
#pragma unroll
                    for (int q = 0; q < RW; ++q) unpack_pairs(xs[q][k], xf[q]);
#pragma unroll
                    for (int j = 0; j < NE; ++j) {
                        if (j < Ne) {
                            const float4 w0 = wsm4[(2 * j) * nv + v], w1 = wsm4[(2 * j + 1) * nv + v];
                            const float2 wp[4] = {make_float2(w0.x, w0.y), make_float2(w0.z, w0.w),
                                                  make_float2(w1.x, w1.y), make_float2(w1.z, w1.w)};
#pragma unroll
                            for (int q = 0; q < RW; ++q) {
                                float2 a = acc2[q * NE + j];
#pragma unroll
                                for (int e = 0; e < 4; ++e) a = f2_fma(xf[q][e], wp[e], a);
                                acc2[q * NE + j] = a;
                            }
                        }
                    }
                }
            }
        }
        float acc[NA];
#pragma unroll
        for (int i = 0; i < NA; ++i) acc[i] = acc2[i].x + acc2[i].y;
        warp_reduce_transpose<NA>(acc);
        const int b = bw + rl;
        if (lane < NA && jl < Ne && b < bend) {
            const float logit = acc[0] + bias;
            const float gate = logit > 0.f ? logit : 0.f;
            gates[((long long)b * T + t) * Ne + jl] = gate;
            if (gate > 0.f) atomicAdd(&cnt[jl], 1);
        }
    }
    __syncthreads();
    if (threadIdx.x < Ne && cnt[threadIdx.x]) atomicAdd(counts + (long long)t * Ne + threadIdx.x, cnt[threadIdx.x]);
}

__device__ __forceinline__ int warp_isum(int v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// One CTA of 1024 threads per expert g = t * Ne + j: its slot offset and
// m-tile prefix (sums over the experts before it), then the list of samples
// b (ascending) whose gate is > 0.  With cnt_pad (training), every expert's
// list is padded to a multiple of 64 slots, at least 64 (the expert's
// K range in the weight-gradient products): offsets, m-tiles and totals count
// the padded lists, cnt_pad receives the padded counts, and the padding slots
// get row -1 and gate 0.
__device__ __forceinline__ int padded_count(int c) { return c < 64 ? 64 : (c + 63) / 64 * 64; }

__global__ void __launch_bounds__(1024) compact_kernel(const float* __restrict__ gates,
                                                       const int* __restrict__ counts, int* __restrict__ offsets,
                                                       int* __restrict__ mtile_prefix, int* __restrict__ totals,
                                                       int* __restrict__ slot_row, float* __restrict__ slot_gate,
                                                       int* __restrict__ slot_of, int* __restrict__ cnt_pad, int B,
                                                       int T, int Ne, int tile_rows) {
    pdl_enter();
    __shared__ int s_off;
    __shared__ int s_warp[32];
    const int G = T * Ne;
    const int g = blockIdx.x;
    const int t = g / Ne, j = g - t * Ne;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const bool pad = cnt_pad != nullptr;
    auto rows_of = [&](int c) { return pad ? padded_count(c) : c; };
    if (warp == 0) {
        int off = 0, mt = 0;
        for (int q = lane; q < g; q += 32) {
            const int c = rows_of(__ldcg(counts + q));
            off += c;
            mt += (c + tile_rows - 1) / tile_rows;
        }
        off = warp_isum(off);
        mt = warp_isum(mt);
        if (lane == 0) {
            s_off = off;
            offsets[g] = off;
            mtile_prefix[g] = mt;
            if (pad) cnt_pad[g] = rows_of(__ldcg(counts + g));
            if (g == G - 1) {
                const int c = rows_of(__ldcg(counts + g));
                mtile_prefix[G] = mt + (c + tile_rows - 1) / tile_rows;
                totals[0] = off + c;
                totals[1] = mt + (c + tile_rows - 1) / tile_rows;
            }
        }
    }
    __syncthreads();
    const int off = s_off;
    if (pad) {   // the padding slots after the expert's active entries
        const int c = __ldcg(counts + g);
        for (int q = c + threadIdx.x; q < padded_count(c); q += blockDim.x) {
            slot_row[off + q] = -1;
            slot_gate[off + q] = 0.f;
        }
    }
    int base = 0;
    for (int b0 = 0; b0 < B; b0 += 1024) {
        const int b = b0 + threadIdx.x;
        const long long e = ((long long)b * T + t) * Ne + j;
        const float gate = b < B ? __ldcg(gates + e) : 0.f;
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

// Sg[slot] = S[slot_row[slot]] (zeros for a padding slot, row -1): one warp
// per slot, 16-byte vectors.
__global__ void __launch_bounds__(kThreads) gather_kernel(const __nv_bfloat16* __restrict__ S,
                                                          const int* __restrict__ slot_row,
                                                          const int* __restrict__ totals,
                                                          __nv_bfloat16* __restrict__ Sg, int D) {
    pdl_enter();
    const int lane = threadIdx.x & 31;
    const int n = __ldcg(totals);
    const int nv = D / 8;
    for (long long s = blockIdx.x * (long long)(blockDim.x >> 5) + (threadIdx.x >> 5); s < n;
         s += (long long)gridDim.x * (blockDim.x >> 5)) {
        const int row = __ldcg(slot_row + s);
        uint4* dst = reinterpret_cast<uint4*>(Sg + s * D);
        if (row < 0) {
            for (int v = lane; v < nv; v += 32) dst[v] = make_uint4(0u, 0u, 0u, 0u);
            continue;
        }
        const uint4* src = reinterpret_cast<const uint4*>(S + (long long)row * D);
        for (int v0 = lane; v0 < nv; v0 += 128) {   // up to four loads in flight per lane
            uint4 t[4];
#pragma unroll
            for (int k = 0; k < 4; ++k)
                if (v0 + 32 * k < nv) t[k] = __ldcg(src + v0 + 32 * k);
#pragma unroll
            for (int k = 0; k < 4; ++k)
                if (v0 + 32 * k < nv) dst[v0 + 32 * k] = t[k];
        }
    }
}

// out[r] = resid[r] + sum over j ascending of Eg[slot_of[r, j]] (active only),
// summed in fp32 pairs.  One warp per (b, t) row: the row's expert slots are
// read once (lane j holds slot j), lane l keeps vectors l, l + 32, ... of the
// row (NVL of them) in registers, and each active expert's vectors are loaded
// together.  stats (optional) = (mean, M2) of the stored row, from sums
// shifted by the row's first stored value.
template <int NVL>
__global__ void __launch_bounds__(kThreads) combine_kernel(const __nv_bfloat16* __restrict__ Eg,
                                                           const int* __restrict__ slot_of,
                                                           const __nv_bfloat16* __restrict__ resid,
                                                           __nv_bfloat16* __restrict__ out, float2* __restrict__ stats,
                                                           long long rows, int D, int Ne) {
    pdl_enter();
    const int lane = threadIdx.x & 31;
    const long long r = blockIdx.x * (long long)(blockDim.x >> 5) + (threadIdx.x >> 5);
    if (r >= rows) return;   // warp-uniform
    const int nv = D / 8;
    const int myslot = lane < Ne ? __ldcg(slot_of + r * Ne + lane) : -1;
    const unsigned act = __ballot_sync(0xffffffffu, myslot >= 0);
    float2 acc[NVL][4];
#pragma unroll
    for (int i = 0; i < NVL; ++i) {
        const int v = lane + 32 * i;
        if (resid && v < nv) {
            unpack_pairs(__ldcg(reinterpret_cast<const uint4*>(resid + r * D) + v), acc[i]);
        } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[i][e] = f2(0.f);
        }
    }
    for (unsigned m = act; m; m &= m - 1) {   // active experts, ascending j
        const int slot = __shfl_sync(0xffffffffu, myslot, __ffs(m) - 1);
        const uint4* src = reinterpret_cast<const uint4*>(Eg + (long long)slot * D);
        uint4 x[NVL];
#pragma unroll
        for (int i = 0; i < NVL; ++i)
            if (lane + 32 * i < nv) x[i] = __ldcg(src + lane + 32 * i);
#pragma unroll
        for (int i = 0; i < NVL; ++i) {
            if (lane + 32 * i < nv) {
                float2 p[4];
                unpack_pairs(x[i], p);
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[i][e] = f2_add(acc[i][e], p[e]);
            }
        }
    }
    uint4 o[NVL];
#pragma unroll
    for (int i = 0; i < NVL; ++i) {
        o[i] = pack_pairs(acc[i]);
        if (lane + 32 * i < nv) reinterpret_cast<uint4*>(out + r * D)[lane + 32 * i] = o[i];
    }
    if (stats) {
        const float K = __shfl_sync(0xffffffffu, __uint_as_float(o[0].x << 16), 0);   // stored element 0
        const float2 nK = f2(-K);
        float2 a1 = f2(0.f), a2 = f2(0.f);
#pragma unroll
        for (int i = 0; i < NVL; ++i) {
            if (lane + 32 * i < nv) {
                float2 p[4];
                unpack_pairs(o[i], p);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 d = f2_add(p[e], nK);
                    a1 = f2_add(a1, d);
                    a2 = f2_fma(d, d, a2);
                }
            }
        }
        const float s1 = warp_sum(a1.x + a1.y);
        const float s2 = warp_sum(a2.x + a2.y);
        if (lane == 0) stats[r] = make_float2(K + s1 / D, fmaxf(s2 - s1 * s1 / D, 0.f));
    }
}

}  // namespace

cudaError_t launch_moe_route(const void* S, const float* Wr, const float* br, const MoeWork& w, int B, int T,
                             int D, int Ne, cudaStream_t s, int tile_rows) {
    cudaError_t e = cudaMemsetAsync(w.counts, 0, sizeof(int) * T * Ne, s);
    if (e != cudaSuccess) return e;
    const size_t smem = sizeof(float) * (size_t)Ne * D;
    const auto* Sb = static_cast<const __nv_bfloat16*>(S);
    int num_sms = 0, dev = 0;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    // Rows per CTA: the (T x chunks) grid fills the resident CTA slots once;
    // a multiple of the rows a CTA's warps take per pass (8 warps x max(1, 16/NE)).
#define RM_ROUTE(NEV)                                                                                    \
    {                                                                                                    \
        e = cudaFuncSetAttribute(route_kernel<NEV>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); \
        if (e != cudaSuccess) return e;                                                                  \
        int occ = 0;                                                                                     \
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, route_kernel<NEV>, kThreads, smem);      \
        if (e != cudaSuccess) return e;                                                                  \
        const int per_pass = (kThreads / 32) * (NEV < 16 ? 16 / NEV : 1);                                \
        const long long slots = (long long)num_sms * (occ > 0 ? occ : 1);                                \
        long long chunks = slots / T;                                                                    \
        if (chunks < 1) chunks = 1;                                                                      \
        long long rows = (B + chunks - 1) / chunks;                                                      \
        rows = (rows + per_pass - 1) / per_pass * per_pass;                                              \
        const dim3 grid(T, (unsigned)((B + rows - 1) / rows));                                           \
        e = launch_pdl(route_kernel<NEV>, grid, kThreads, smem, s, Sb, Wr, br, w.gates, w.counts, B, T, D, Ne, \
                       (int)rows);                                                                       \
        if (e != cudaSuccess) return e;                                                                  \
    }
    if (Ne <= 1) RM_ROUTE(1)
    else if (Ne <= 2) RM_ROUTE(2)
    else if (Ne <= 4) RM_ROUTE(4)
    else if (Ne <= 8) RM_ROUTE(8)
    else if (Ne <= 16) RM_ROUTE(16)
    else RM_ROUTE(32)
#undef RM_ROUTE
    if (tile_rows == 0) return cudaSuccess;   // gates only (DTSI's second router)
    return launch_pdl(compact_kernel, T * Ne, 1024, 0, s, w.gates, w.counts, w.offsets, w.mtile_prefix, w.totals,
                      w.slot_row, w.slot_gate, w.slot_of, w.cnt_pad, B, T, Ne, tile_rows);
}

cudaError_t launch_moe_gather(const void* S, const MoeWork& w, int B, int T, int D, int Ne, cudaStream_t s) {
    (void)B;
    (void)T;
    (void)Ne;
    return launch_pdl(gather_kernel, 148 * 8, kThreads, 0, s, static_cast<const __nv_bfloat16*>(S), w.slot_row,
                      w.totals, static_cast<__nv_bfloat16*>(w.Sg), D);
}

cudaError_t launch_moe_combine(const MoeWork& w, const void* resid, void* out, float2* stats, int B, int T, int D,
                               int Ne, cudaStream_t s) {
    const long long rows = (long long)B * T;
    const int grid = (int)((rows + kThreads / 32 - 1) / (kThreads / 32));
    const int nvl = (D / 8 + 31) / 32;
    const auto* eg = static_cast<const __nv_bfloat16*>(w.Eg);
    const auto* rs = static_cast<const __nv_bfloat16*>(resid);
    auto* o = static_cast<__nv_bfloat16*>(out);
    if (nvl <= 1) return launch_pdl(combine_kernel<1>, grid, kThreads, 0, s, eg, w.slot_of, rs, o, stats, rows, D, Ne);
    if (nvl <= 2) return launch_pdl(combine_kernel<2>, grid, kThreads, 0, s, eg, w.slot_of, rs, o, stats, rows, D, Ne);
    if (nvl <= 4) return launch_pdl(combine_kernel<4>, grid, kThreads, 0, s, eg, w.slot_of, rs, o, stats, rows, D, Ne);
    if (nvl <= 8) return launch_pdl(combine_kernel<8>, grid, kThreads, 0, s, eg, w.slot_of, rs, o, stats, rows, D, Ne);
    return cudaErrorInvalidValue;
}

}  // namespace rm

// ------------------------------------------------------ training (backward)
// Gradients of v = sum_j G_j e_j (fun-rec "Rankmixer: 硬件效率优化", section
// Sparse MoE扩展, ReLU routing) for the active entries, and of the routers
// G = ReLU(Wr s + br): dG_j = dV . e_j, de_j = G_j dV, dR_j = dG_j [R_j > 0]
// (+ lambda for L_reg on these gates), DTSI's second router dR_inf_j =
// lambda [R_inf_j > 0].
namespace rm {
namespace {

// One warp per row r = (b, t): dV's vectors stay in registers; for each
// active expert j (ascending) the gated output row Eg = G_j e_j gives
// dG_j = dV . Eg / G_j (a fixed-order warp sum), and de_j = G_j dV is
// written to the expert's slot.  Lane j writes dR[r, j] (0 when inactive)
// and, under DTSI, dRinf[r, j].
template <int NVL>
__global__ void __launch_bounds__(kThreads) moe_bwd_gate_kernel(
    const __nv_bfloat16* __restrict__ dV, const __nv_bfloat16* __restrict__ Eg, const int* __restrict__ slot_of,
    const float* __restrict__ slot_gate, const float* __restrict__ gates_inf, float lambda,
    __nv_bfloat16* __restrict__ dEg, float* __restrict__ dR, float* __restrict__ dRinf, long long rows, int D,
    int Ne) {
    pdl_enter();
    const int lane = threadIdx.x & 31;
    const long long r = blockIdx.x * (long long)(blockDim.x >> 5) + (threadIdx.x >> 5);
    if (r >= rows) return;   // warp-uniform
    const int nv = D / 8;
    const int myslot = lane < Ne ? __ldcg(slot_of + r * Ne + lane) : -1;
    const unsigned act = __ballot_sync(0xffffffffu, myslot >= 0);
    float2 dv[NVL][4];
#pragma unroll
    for (int i = 0; i < NVL; ++i) {
        const int v = lane + 32 * i;
        if (v < nv) unpack_pairs(__ldcg(reinterpret_cast<const uint4*>(dV + r * D) + v), dv[i]);
    }
    float my_dr = 0.f;
    for (unsigned m = act; m; m &= m - 1) {   // active experts, ascending j
        const int j = __ffs(m) - 1;
        const int slot = __shfl_sync(0xffffffffu, myslot, j);
        const float gate = __ldcg(slot_gate + slot);
        const uint4* src = reinterpret_cast<const uint4*>(Eg + (long long)slot * D);
        uint4 x[NVL];
#pragma unroll
        for (int i = 0; i < NVL; ++i)
            if (lane + 32 * i < nv) x[i] = __ldcg(src + lane + 32 * i);
        float2 a = f2(0.f);
        uint4* dst = reinterpret_cast<uint4*>(dEg + (long long)slot * D);
#pragma unroll
        for (int i = 0; i < NVL; ++i) {
            if (lane + 32 * i < nv) {
                float2 e[4], de[4];
                unpack_pairs(x[i], e);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    a = f2_fma(dv[i][q], e[q], a);
                    de[q] = f2_mul(dv[i][q], f2(gate));
                }
                dst[lane + 32 * i] = pack_pairs(de);
            }
        }
        const float dG = warp_sum(a.x + a.y) / gate;
        if (lane == j) my_dr = dG + (gates_inf ? 0.f : lambda);
    }
    if (lane < Ne) {
        dR[r * Ne + lane] = my_dr;
        if (dRinf) dRinf[r * Ne + lane] = __ldcg(gates_inf + r * Ne + lane) > 0.f ? lambda : 0.f;
    }
}

// Zero the rows of the padding slots (row -1) of a compacted [slots, D] array.
__global__ void __launch_bounds__(kThreads) zero_pad_rows_kernel(__nv_bfloat16* __restrict__ dst,
                                                                 const int* __restrict__ slot_row,
                                                                 const int* __restrict__ totals, int D) {
    pdl_enter();
    const int lane = threadIdx.x & 31;
    const int n = __ldcg(totals);
    const int nv = D / 8;
    for (long long s = blockIdx.x * (long long)(blockDim.x >> 5) + (threadIdx.x >> 5); s < n;
         s += (long long)gridDim.x * (blockDim.x >> 5)) {
        if (__ldcg(slot_row + s) >= 0) continue;   // warp-uniform
        uint4* d = reinterpret_cast<uint4*>(dst + s * D);
        for (int v = lane; v < nv; v += 32) d[v] = make_uint4(0u, 0u, 0u, 0u);
    }
}

// dS[r] = dZ[r] + sum over active j (ascending) of dSg[slot(r, j)]
//         + sum_j dR[r, j] Wr[t, j, :] + sum_j dRinf[r, j] Wrinf[t, j, :]
// (one warp per row, fp32 pairs, fixed order; zero router terms skipped).
template <int NVL>
__global__ void __launch_bounds__(kThreads) moe_bwd_combine_kernel(
    const __nv_bfloat16* __restrict__ dZ, const __nv_bfloat16* __restrict__ dSg, const int* __restrict__ slot_of,
    const float* __restrict__ dR, const float* __restrict__ Wr, const float* __restrict__ dRinf,
    const float* __restrict__ Wrinf, __nv_bfloat16* __restrict__ dS, long long rows, int T, int D, int Ne) {
    pdl_enter();
    const int lane = threadIdx.x & 31;
    const long long r = blockIdx.x * (long long)(blockDim.x >> 5) + (threadIdx.x >> 5);
    if (r >= rows) return;   // warp-uniform
    const int t = (int)(r % T);
    const int nv = D / 8;
    const int myslot = lane < Ne ? __ldcg(slot_of + r * Ne + lane) : -1;
    const unsigned act = __ballot_sync(0xffffffffu, myslot >= 0);
    float2 acc[NVL][4];
#pragma unroll
    for (int i = 0; i < NVL; ++i) {
        const int v = lane + 32 * i;
        if (v < nv) unpack_pairs(__ldcg(reinterpret_cast<const uint4*>(dZ + r * D) + v), acc[i]);
    }
    for (unsigned m = act; m; m &= m - 1) {
        const int slot = __shfl_sync(0xffffffffu, myslot, __ffs(m) - 1);
        const uint4* src = reinterpret_cast<const uint4*>(dSg + (long long)slot * D);
        uint4 x[NVL];
#pragma unroll
        for (int i = 0; i < NVL; ++i)
            if (lane + 32 * i < nv) x[i] = __ldcg(src + lane + 32 * i);
#pragma unroll
        for (int i = 0; i < NVL; ++i) {
            if (lane + 32 * i < nv) {
                float2 p[4];
                unpack_pairs(x[i], p);
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[i][q] = f2_add(acc[i][q], p[q]);
            }
        }
    }
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {   // the routing router, then DTSI's second router
        const float* d = pass ? dRinf : dR;
        const float* W = pass ? Wrinf : Wr;
        if (!d) continue;
        const float my = lane < Ne ? __ldcg(d + r * Ne + lane) : 0.f;
        for (int j = 0; j < Ne; ++j) {
            const float dr = __shfl_sync(0xffffffffu, my, j);
            if (dr == 0.f) continue;   // warp-uniform
            const float* w = W + ((long long)t * Ne + j) * D;
#pragma unroll
            for (int i = 0; i < NVL; ++i) {
                const int v = lane + 32 * i;
                if (v < nv) {
                    const float4 w0 = __ldg(reinterpret_cast<const float4*>(w) + 2 * v);
                    const float4 w1 = __ldg(reinterpret_cast<const float4*>(w) + 2 * v + 1);
                    const float2 wp[4] = {make_float2(w0.x, w0.y), make_float2(w0.z, w0.w), make_float2(w1.x, w1.y),
                                          make_float2(w1.z, w1.w)};
#pragma unroll
                    for (int q = 0; q < 4; ++q) acc[i][q] = f2_fma(f2(dr), wp[q], acc[i][q]);
                }
            }
        }
    }
#pragma unroll
    for (int i = 0; i < NVL; ++i)
        if (lane + 32 * i < nv) reinterpret_cast<uint4*>(dS + r * D)[lane + 32 * i] = pack_pairs(acc[i]);
}

// Router weight-gradient partials over blocks of RB samples: part[((t * nrb +
// rb) * Ne + j) * D + d] = sum_{b in block rb} dR[b, t, j] S[b, t, d], and
// part_b[(t * nrb + rb) * Ne + j] = sum_b dR[b, t, j] (both in ascending b).
// Thread = 8 columns; experts in passes of 8; rows whose dR is zero skipped.
__global__ void __launch_bounds__(kThreads) router_grad_kernel(const __nv_bfloat16* __restrict__ S,
                                                               const float* __restrict__ dR, float* __restrict__ part,
                                                               float* __restrict__ part_b, int B, int T, int D, int Ne,
                                                               int RB) {
    pdl_enter();
    const int v = blockIdx.x * blockDim.x + threadIdx.x;
    const int rb = blockIdx.y, nrb = gridDim.y, t = blockIdx.z;
    const int b0 = rb * RB, b1 = min(B, b0 + RB);
    const bool col = 8 * v < D;
    for (int j0 = 0; j0 < Ne; j0 += 8) {
        float a[8][8];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj)
#pragma unroll
            for (int e = 0; e < 8; ++e) a[jj][e] = 0.f;
        for (int bq = b0; bq < b1; bq += 4) {   // four rows' loads in flight, summed in row order
            float dr[4][8];
            uint4 sv[4];
            bool any[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int b = bq + q;
                const long long row = (long long)b * T + t;
                any[q] = false;
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    dr[q][jj] = (b < b1 && j0 + jj < Ne) ? __ldg(dR + row * Ne + j0 + jj) : 0.f;
                    any[q] |= dr[q][jj] != 0.f;
                }
                if (any[q] && col) sv[q] = __ldcg(reinterpret_cast<const uint4*>(S + row * D) + v);
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                if (!any[q] || !col) continue;
                float2 sp[4];
                unpack_pairs(sv[q], sp);
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    if (dr[q][jj] != 0.f) {
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            a[jj][2 * e] = fmaf(dr[q][jj], sp[e].x, a[jj][2 * e]);
                            a[jj][2 * e + 1] = fmaf(dr[q][jj], sp[e].y, a[jj][2 * e + 1]);
                        }
                    }
                }
            }
        }
        if (col) {
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                if (j0 + jj < Ne) {
                    float4* o = reinterpret_cast<float4*>(part + (((long long)t * nrb + rb) * Ne + j0 + jj) * D + 8 * v);
                    o[0] = make_float4(a[jj][0], a[jj][1], a[jj][2], a[jj][3]);
                    o[1] = make_float4(a[jj][4], a[jj][5], a[jj][6], a[jj][7]);
                }
            }
        }
    }
    if (blockIdx.x == 0 && threadIdx.x < Ne) {
        float sb = 0.f;
        for (int b = b0; b < b1; ++b) sb += __ldg(dR + ((long long)b * T + t) * Ne + threadIdx.x);
        part_b[((long long)t * nrb + rb) * Ne + threadIdx.x] = sb;
    }
}

// loss[0] += lambda * sum of x[0 .. n), in a fixed order: CTA p sums chunk
// p of kSumChunks equal chunks (thread i over elements i, i + 256, ..., then
// a fixed tree) into part[p]; one warp adds the chunk sums (lane l over
// chunks l, l + 32, ..., then a fixed butterfly).
constexpr int kSumChunks = 256;

__global__ void __launch_bounds__(256) sum_chunks_kernel(const float* __restrict__ x, long long n,
                                                         float* __restrict__ part) {
    pdl_enter();
    __shared__ float red[8];
    const long long chunk = (n + gridDim.x - 1) / gridDim.x;
    const long long i0 = blockIdx.x * chunk, i1 = min(n, i0 + chunk);
    float a = 0.f;
    for (long long i = i0 + threadIdx.x; i < i1; i += blockDim.x) a += __ldcg(x + i);
    a = warp_sum(a);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
    __syncthreads();
    if (threadIdx.x == 0) {
        float t = 0.f;
        for (int w = 0; w < 8; ++w) t += red[w];
        part[blockIdx.x] = t;
    }
}

__global__ void __launch_bounds__(32) add_scaled_parts_kernel(const float* __restrict__ part, int np, float lambda,
                                                               float* __restrict__ loss) {
    pdl_enter();
    float a = 0.f;
    for (int i = threadIdx.x; i < np; i += 32) a += __ldcg(part + i);
    a = warp_sum(a);
    if (threadIdx.x == 0) loss[0] += lambda * a;
}

}  // namespace

cudaError_t launch_moe_route_only(const void* S, const float* Wr, const float* br, float* gates, int* counts_scratch,
                                  int B, int T, int D, int Ne, cudaStream_t s) {
    MoeWork w{};
    w.gates = gates;
    w.counts = counts_scratch;
    return launch_moe_route(S, Wr, br, w, B, T, D, Ne, s, 0);
}

cudaError_t launch_moe_bwd_gate(const void* dV, const MoeWork& w, const float* gates_inf, float lambda, void* dEg,
                                float* dR, float* dRinf, int B, int T, int D, int Ne, cudaStream_t s) {
    const long long rows = (long long)B * T;
    const int grid = (int)((rows + kThreads / 32 - 1) / (kThreads / 32));
    const int nvl = (D / 8 + 31) / 32;
    const auto* dv = static_cast<const __nv_bfloat16*>(dV);
    const auto* eg = static_cast<const __nv_bfloat16*>(w.Eg);
    auto* de = static_cast<__nv_bfloat16*>(dEg);
    cudaError_t e;
#define RM_GATE(N)                                                                                                  \
    e = launch_pdl(moe_bwd_gate_kernel<N>, grid, kThreads, 0, s, dv, eg, w.slot_of, w.slot_gate, gates_inf, lambda, \
                   de, dR, dRinf, rows, D, Ne)
    if (nvl <= 1) RM_GATE(1);
    else if (nvl <= 2) RM_GATE(2);
    else if (nvl <= 4) RM_GATE(4);
    else if (nvl <= 8) RM_GATE(8);
    else return cudaErrorInvalidValue;
#undef RM_GATE
    if (e != cudaSuccess) return e;
    return launch_pdl(zero_pad_rows_kernel, 148 * 8, kThreads, 0, s, de, w.slot_row, w.totals, D);
}

cudaError_t launch_moe_bwd_combine(const void* dZ, const void* dSg, const MoeWork& w, const float* dR, const float* Wr,
                                   const float* dRinf, const float* Wrinf, void* dS, int B, int T, int D, int Ne,
                                   cudaStream_t s) {
    const long long rows = (long long)B * T;
    const int grid = (int)((rows + kThreads / 32 - 1) / (kThreads / 32));
    const int nvl = (D / 8 + 31) / 32;
    const auto* dz = static_cast<const __nv_bfloat16*>(dZ);
    const auto* dsg = static_cast<const __nv_bfloat16*>(dSg);
    auto* ds = static_cast<__nv_bfloat16*>(dS);
#define RM_CMB(N)                                                                                                  \
    return launch_pdl(moe_bwd_combine_kernel<N>, grid, kThreads, 0, s, dz, dsg, w.slot_of, dR, Wr, dRinf, Wrinf, ds, \
                      rows, T, D, Ne)
    if (nvl <= 1) RM_CMB(1);
    if (nvl <= 2) RM_CMB(2);
    if (nvl <= 4) RM_CMB(4);
    if (nvl <= 8) RM_CMB(8);
#undef RM_CMB
    return cudaErrorInvalidValue;
}

cudaError_t launch_router_grad(const void* S, const float* dR, float* part, float* part_b, int B, int T, int D, int Ne,
                               int RB, cudaStream_t s) {
    const int nrb = (B + RB - 1) / RB;
    const int nv = D / 8;
    const int threads = nv < kThreads ? std::max(32, (nv + 31) / 32 * 32) : kThreads;
    const dim3 grid((unsigned)((nv + threads - 1) / threads), (unsigned)nrb, (unsigned)T);
    return launch_pdl(router_grad_kernel, grid, threads, 0, s, static_cast<const __nv_bfloat16*>(S), dR, part, part_b,
                      B, T, D, Ne, RB);
}

cudaError_t launch_add_scaled_sum(const float* x, long long n, float lambda, float* loss, float* part,
                                  cudaStream_t s) {
    cudaError_t e = launch_pdl(sum_chunks_kernel, kSumChunks, 256, 0, s, x, n, part);
    if (e != cudaSuccess) return e;
    return launch_pdl(add_scaled_parts_kernel, 1, 32, 0, s, (const float*)part, kSumChunks, lambda, loss);
}

}  // namespace rm
