// Fused token mixing + residual + LayerNorm, the final LayerNorm + mean
// pooling, and row LayerNorm statistics.
//
// Token mixing with H = T heads (fun-rec chapter "Rankmixer: 硬件效率优化",
// section Token Mixing机制) sends chunk h of token t to position t*dh of output
// token h (dh = D / T).  Every output row of a sample reads a slice of every
// input row, so the sample is the unit of work: persistent CTAs (two per SM)
// stage whole samples -- or chunks of several small samples -- in a
// shared-memory ring of 1-4 slots with cp.async.bulk, so the next chunk's
// copy overlaps the current one's arithmetic.  The permutation is applied
// through shared-memory addressing with 16-byte vectors (rows padded so the
// pieces consecutive lanes gather fall in consecutive banks), so X is read
// from HBM once and S written once, with no transpose pass.
//
// The mixing kernel computes each output row's LN1 statistics with LPR =
// 8/16/32 lanes per row (pass A), then writes the normalised rows with one
// thread per (row group, 16-byte column vector) that keeps gamma / beta in
// registers (pass B).  The previous block's LayerNorm (PRE) uses row
// statistics produced where the row was written (the grouped GEMM's epilogue,
// the MoE combine, or row_stats_kernel) as partial (mean, M2) pairs over P
// equal column slices; those partials travel into the ring slot with the rows
// (one more bulk copy), so no thread waits on a global load for them.
//
// mix_ln:  Xh = PRE ? LN_pre(X) : X                       (per token row)
//          Z[h, t*dh + j] = Xh[t, h*dh + j] + Xh[h, t*dh + j]
//          S[h, :] = LN1(Z[h, :])
//          or, without the Add & Norm after mixing, S[h, t*dh + j] = Xh[t, h*dh + j]
// ln_pool: pooled[b, :] = (1/T) sum_t LN(X[b, t, :])  (one thread per sample
//          and 16-byte column vector, rows summed in ascending t)
#include <cuda_bf16.h>

#include <algorithm>

#include "rm_device.cuh"

namespace rm {
namespace {

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

template <int NP>
__device__ __forceinline__ void load_pairs(const float* __restrict__ p, float2 (&o)[NP]) {
#pragma unroll
    for (int q = 0; q < NP / 2; ++q) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(p) + q);
        o[2 * q] = make_float2(v.x, v.y);
        o[2 * q + 1] = make_float2(v.z, v.w);
    }
}

template <int N>
__device__ __forceinline__ void load_params(const float* __restrict__ p, float (&o)[N]) {
#pragma unroll
    for (int q = 0; q < N / 4; ++q) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(p) + q);
        o[4 * q + 0] = v.x;
        o[4 * q + 1] = v.y;
        o[4 * q + 2] = v.z;
        o[4 * q + 3] = v.w;
    }
}

// Ring of whole samples in shared memory.  Slot s holds one chunk's rows at a
// row stride of rs >= D elements, and (when the kernel merges LayerNorm
// partials) the chunk's partial statistics after them; it fills from one
// cp.async.bulk copy of the rows (rs == D) or one copy per row issued by the
// lanes of warp 0, plus one copy of the partials, all on the slot's mbarrier.
// Slot bookkeeping lives in bit masks in lane 0 of warp 0.
//
// Partials: the chunk's P * rows float2 pairs are contiguous in global memory
// but need not start on a 16-byte boundary, so the copy starts at the
// boundary below and ends at the one above; the partial array must be
// readable up to the 16-byte boundary past its end (its workspace region is
// padded to 256 bytes).  stats() returns the chunk's first pair in the slot.
constexpr int kMaxSlots = 4;

template <typename E>
struct SampleRing {
    unsigned char* base;   // slot s at base + s * slot_bytes
    uint32_t bar0;         // mbarrier of slot s at bar0 + 8 * s
    int nslots, D, rs;
    uint32_t slot_bytes;
    uint32_t stats_off;    // byte offset of the staged partials in a slot; 0: none staged
    const float2* part;    // partials [rows][P] in global memory (stats_off != 0)
    int P;
    uint32_t outstanding;  // bit s: a copy into slot s was issued and not yet waited for
    uint32_t parity;       // bit s: parity of slot s's next completion

    __device__ __forceinline__ E* buf(int slot) const { return reinterpret_cast<E*>(base + (size_t)slot * slot_bytes); }
    __device__ __forceinline__ uint32_t bar(int slot) const { return bar0 + 8u * (uint32_t)slot; }
    __device__ __forceinline__ const float2* stats(int slot, long long row0) const {
        const uintptr_t a = reinterpret_cast<uintptr_t>(part + row0 * P);
        return reinterpret_cast<const float2*>(base + (size_t)slot * slot_bytes + stats_off + (a & 15u));
    }

    // all lanes of warp 0: `rows` contiguous rows [rows, D] from src (global
    // rows row0 ...) into `slot`, with their partials if staged
    __device__ void issue(int slot, const E* src, int rows, long long row0) {
        const int lane = threadIdx.x & 31;
        const uint32_t row_bytes = (uint32_t)(D * sizeof(E));
        uint32_t sbytes = 0;
        const void* ssrc = nullptr;
        if (stats_off) {
            const uintptr_t a = reinterpret_cast<uintptr_t>(part + row0 * P);
            const uintptr_t e = a + (uintptr_t)rows * (uintptr_t)P * sizeof(float2);
            const uintptr_t a16 = a & ~static_cast<uintptr_t>(15), e16 = (e + 15) & ~static_cast<uintptr_t>(15);
            ssrc = reinterpret_cast<const void*>(a16);
            sbytes = (uint32_t)(e16 - a16);
        }
        if (lane == 0) {
            mbar_arrive_expect_tx(bar(slot), row_bytes * (uint32_t)rows + sbytes);
            outstanding |= 1u << slot;
        }
        __syncwarp();
        fence_proxy_async_smem();   // earlier generic accesses to the slot come first
        const uint32_t dst = smem_u32(buf(slot));
        if (sbytes && lane == 31) bulk_load(dst + stats_off, ssrc, sbytes, bar(slot));
        if (rs == D) {   // unpadded rows: one contiguous copy
            if (lane == 0) bulk_load(dst, src, row_bytes * (uint32_t)rows, bar(slot));
            return;
        }
        for (int r = lane; r < rows; r += 32)
            bulk_load(dst + (uint32_t)(r * rs) * (uint32_t)sizeof(E), src + (size_t)r * D, row_bytes, bar(slot));
    }
    // thread 0 only: wait for the copies into `slot`; false if the wait ran out.
    __device__ bool wait(int slot, const WaitCtx& wc, int site) {
        const bool ok = mbar_wait(bar(slot), (parity >> slot) & 1u, wc, site, false);
        if (ok) {
            outstanding &= ~(1u << slot);
            parity ^= 1u << slot;
        }
        return ok;
    }
    // thread 0 only: let every copy still in flight land before the CTA exits.
    __device__ void drain(const WaitCtx& wc, int site) {
        for (int s = 0; s < nslots; ++s)
            if ((outstanding >> s) & 1u) mbar_wait(bar(s), (parity >> s) & 1u, wc, site, false);
    }
};

// Bytes of the rows part of a slot (128-byte multiple) and of its staged
// partials (rows * P pairs plus 16 bytes of alignment slack, 16-byte multiple).
inline __host__ __device__ size_t rows_bytes_of(int rows, int rs, size_t esz) {
    return ((size_t)rows * rs * esz + 127) / 128 * 128;
}
inline __host__ __device__ size_t stats_bytes_of(int rows, int P) {
    return P > 0 ? ((size_t)rows * P * 8 + 16 + 15) / 16 * 16 : 0;
}
inline __host__ __device__ size_t slot_bytes_of(int rows, int rs, size_t esz, int P) {
    return (rows_bytes_of(rows, rs, esz) + stats_bytes_of(rows, P) + 127) / 128 * 128;
}

// Carves the ring (nslots slots of `rows` rows, with partials when P > 0), its
// barriers and the per-row statistics (mean_s[rows], rstd_s[rows]) out of
// dynamic shared memory.
template <typename E>
__device__ __forceinline__ void make_ring(SampleRing<E>& r, unsigned char* smem, int rows, int D, int rs,
                                          int nslots, const float2* part, int P, float*& mean_s,
                                          float*& rstd_s) {
    r.slot_bytes = (uint32_t)slot_bytes_of(rows, rs, sizeof(E), part ? P : 0);
    r.stats_off = part ? (uint32_t)rows_bytes_of(rows, rs, sizeof(E)) : 0u;
    r.part = part;
    r.P = P;
    r.nslots = nslots;
    r.D = D;
    r.rs = rs;
    r.base = smem;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)nslots * r.slot_bytes);
    r.bar0 = smem_u32(bars);
    r.outstanding = 0;
    r.parity = 0;
    mean_s = reinterpret_cast<float*>(bars + kMaxSlots);
    rstd_s = mean_s + rows;
}

// Row stride of the staged sample for the mixing kernel: D plus a pad that
// makes consecutive token rows start (dh - D) * esz bytes apart modulo 128,
// so the 16-byte pieces that consecutive lanes gather from consecutive token
// rows fall in consecutive banks.  Only for whole-vector pieces.
inline int mix_row_stride(int D, int dh, size_t esz) {
    const long long bytes = (long long)dh * (long long)esz;
    if (bytes % 16) return D;
    long long pad = ((long long)(dh - D) * (long long)esz) % 128;
    if (pad < 0) pad += 128;
    return D + (int)(pad / (long long)esz);
}

// Mean and 1/sqrt(var + eps) of a row from its P partials (mean_p, M2_p),
// each over the same n = D/P columns.  With equal counts the pairwise
// (Chan et al.) combination reduces to mean = (1/P) sum_p mean_p and
// M2 = sum_p M2_p + n sum_p (mean_p - mean)^2: two warp sums in a fixed
// butterfly order (deterministic), no divisions; P <= 32.
// Row statistics of the R rows of a chunk into mean_s/rstd_s, all warps of
// the CTA, from the partials staged in shared memory with the chunk.
__device__ __forceinline__ void chunk_stats(const float2* part, int P, int D, int R, float eps, float* mean_s,
                                            float* rstd_s) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const float n = (float)D / (float)P;
    for (int r = warp; r < R; r += nw) {
        const float2 v = lane < P ? part[(size_t)r * P + lane] : make_float2(0.f, 0.f);
        const float mean = warp_sum(v.x) / (float)P;
        const float d = v.x - mean;
        const float q = warp_sum(lane < P ? fmaf(n * d, d, v.y) : 0.f);
        if (lane == 0) {
            mean_s[r] = mean;
            rstd_s[r] = rsqrtf(q / D + eps);
        }
    }
}

// Columns c0 .. c0+V-1 of output row h, mixed term: source token t = c / dh,
// column h*dh + c - t*dh.  `mixed` holds columns [h0*dh, (h0+R)*dh) of every
// row t with row stride rs = R*dh, so the element is mixed[t*rs + hoff + j]
// with hoff = (h-h0)*dh.  MV = elements per contiguous piece: V (one 16-byte
// load), V/2 (8-byte loads) or 1.
template <typename E, int MV>
__device__ __forceinline__ void load_mixed(const E* mixed, int rs, int hoff, int dh, int c0, Vec16<E>& o) {
    constexpr int V = Vec16<E>::N;
    if constexpr (MV == V) {
        const int t = c0 / dh;
        o.u = *reinterpret_cast<const uint4*>(mixed + (size_t)t * rs + hoff + (c0 - t * dh));
    } else if constexpr (MV * sizeof(E) == 8) {
#pragma unroll
        for (int sv = 0; sv < V / MV; ++sv) {
            const int c = c0 + sv * MV, t = c / dh;
            const uint2 q = *reinterpret_cast<const uint2*>(mixed + (size_t)t * rs + hoff + (c - t * dh));
            if (sv == 0) {
                o.u.x = q.x;
                o.u.y = q.y;
            } else {
                o.u.z = q.x;
                o.u.w = q.y;
            }
        }
    } else {
        int t = c0 / dh, j = c0 - t * dh;
#pragma unroll
        for (int e = 0; e < V; ++e) {
            o.e[e] = mixed[(size_t)t * rs + hoff + j];
            if (++j == dh) {
                j = 0;
                ++t;
            }
        }
    }
}

// Threads of the mixing kernel form `groups` row groups of nv = D/V
// column-vector threads: thread (grp, v) owns columns [v*V, v*V + V) of rows
// grp, grp + groups, ... in the element-wise passes, so the source offset of
// its mixed vector and its gamma/beta stay in registers.
constexpr int kMixMaxThreads = 384;

// In-place LayerNorm of the staged sample (row statistics in shared memory),
// in fp32 pairs: y = ((x r) - m r) gamma + beta.
template <typename E>
__device__ __forceinline__ void normalize_in_place(uint32_t xs_a, int rows, int rs, int c0, int grp, int groups,
                                                   const float* __restrict__ g, const float* __restrict__ bta,
                                                   uint32_t mean_a, uint32_t rstd_a) {
    constexpr int NP = Vec16<E>::N / 2;
    float2 gp[NP], bp[NP];
    load_pairs(g + c0, gp);
    load_pairs(bta + c0, bp);
    uint32_t pa = xs_a + (uint32_t)((grp * rs + c0) * (int)sizeof(E));
    const uint32_t pstep = (uint32_t)(groups * rs * (int)sizeof(E));
#pragma unroll 4
    for (int t = grp; t < rows; t += groups, pa += pstep) {
        float2 x[NP];
        unpack_pairs(lds128(pa), x);
        const float r = lds_f32(rstd_a + 4u * (uint32_t)t);
        const float2 r2 = f2(r), mr2 = f2(-lds_f32(mean_a + 4u * (uint32_t)t) * r);
#pragma unroll
        for (int j = 0; j < NP; ++j) x[j] = f2_fma(f2_fma(x[j], r2, mr2), gp[j], bp[j]);
        sts128(pa, pack_pairs(x));
    }
}

// Source offsets of the mixed vector at column c0 (h-independent): piece k
// (16 bytes if MV == V, else 8 bytes at c = c0 + k*V/2) comes from token
// t = c/dh at element t (rs - dh) + c + h*dh of the staged sample.
struct MixOff {
    int a, b;
};
template <typename E, int MV>
__device__ __forceinline__ MixOff mix_off(int c0, int dh, int rs) {
    constexpr int V = Vec16<E>::N;
    MixOff m;
    m.a = (c0 / dh) * (rs - dh) + c0;
    const int c1 = c0 + V / 2;
    m.b = MV * 2 == V ? (c1 / dh) * (rs - dh) + c1 : 0;
    return m;
}

// Mixed vector of output row h at column c0 of a sample staged at row stride
// rs, from precomputed offsets (16- or 8-byte pieces) or element by element.
template <typename E, int MV>
__device__ __forceinline__ void mixed_vec(const E* xs, int rs, int dh, int h, int c0, MixOff mo, Vec16<E>& o) {
    constexpr int V = Vec16<E>::N;
    if constexpr (MV == V) {
        o.u = *reinterpret_cast<const uint4*>(xs + mo.a + h * dh);
    } else if constexpr (MV * 2 == V) {
        const uint2 q0 = *reinterpret_cast<const uint2*>(xs + mo.a + h * dh);
        const uint2 q1 = *reinterpret_cast<const uint2*>(xs + mo.b + h * dh);
        o.u = make_uint4(q0.x, q0.y, q1.x, q1.y);
    } else {
        load_mixed<E, MV>(xs, rs, h * dh, dh, c0, o);
    }
}

// SAVE (training): also write the normalised rows xhat_out and the rows'
// 1/sqrt(var + eps) rstd_out, the LN1 backward's inputs.
template <typename E, bool PRE, int MV, int NV, bool ADDNORM, int LPR, bool SAVE>
__global__ void __launch_bounds__(kMixMaxThreads, 2) mix_ln_kernel(
    const E* __restrict__ X, const float* __restrict__ pre_g, const float* __restrict__ pre_b,
    const float2* __restrict__ pstats, int P, const float* __restrict__ g1, const float* __restrict__ b1,
    E* __restrict__ S, int B, int T, int D, float eps, int rs, int spb, int nslots, int groups, DeviceErr err,
    uint64_t budget_ns, E* __restrict__ xhat_out, float* __restrict__ rstd_out) {
    pdl_enter();
    constexpr int V = Vec16<E>::N;
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ int abort_flag, s_ok;
    const int TD = T * D;
    const int nchunks = (B + spb - 1) / spb;   // chunk c: samples [c*spb, c*spb + spb) in one slot
    float *mean_s, *rstd_s;
    SampleRing<E> ring;
    make_ring<E>(ring, smem, spb * T, D, rs, nslots, PRE ? pstats : nullptr, P, mean_s, rstd_s);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    const WaitCtx wc{&abort_flag, budget_ns, err};
    if (tid == 0) {
        for (int k = 0; k < nslots; ++k) mbar_init(ring.bar(k), 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    auto chunk_rows = [&](long long c) { return (int)(min((long long)spb, B - c * spb) * T); };
    if (warp == 0)
        for (int k = 0; k < nslots; ++k) {
            const long long ck = blockIdx.x + (long long)k * gridDim.x;
            if (ck < nchunks) ring.issue(k, X + (size_t)ck * spb * TD, chunk_rows(ck), ck * spb * T);
        }
    const int dh = D / T;
    const int nv = D / V;
    const int grp = tid / nv, c0 = (tid - grp * nv) * V;
    const bool active = grp < groups;
    const MixOff moff = mix_off<E, MV>(c0, dh, rs);
    constexpr int NP = V / 2;
    float2 g1p[NP], b1p[NP];
    if (ADDNORM && active) {
        load_pairs(g1 + c0, g1p);
        load_pairs(b1 + c0, b1p);
    }
    // statistics pass: a warp takes 32/LPR rows at a time; lane l of the
    // row's LPR lanes takes vectors l, l + LPR, ... of it
    constexpr int RPW = 32 / LPR;
    const int sl = lane % LPR, sub = lane / LPR;
    MixOff moffA[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) moffA[i] = mix_off<E, MV>((sl + LPR * i) * V, dh, rs);
    const int sstride = T * rs;   // elements between the staged samples of a chunk
    int it = 0;
    for (long long c = blockIdx.x; c < nchunks; c += gridDim.x, ++it) {
        const int cur = it % nslots;
        const int R = chunk_rows(c);
        const long long row0 = c * spb * T;   // global row of the chunk's first row
        if (tid == 0) s_ok = ring.wait(cur, wc, SITE_MIX_LN);
        __syncthreads();
        if (!s_ok) break;
        E* xs = ring.buf(cur);
        if (PRE) {
            // the previous block's LayerNorm, from the partials staged with the
            // chunk, applied once per element, in place
            chunk_stats(ring.stats(cur, row0), P, D, R, eps, mean_s, rstd_s);
            __syncthreads();
            if (active)
                normalize_in_place<E>(smem_u32(xs), R, rs, c0, grp, groups, pre_g, pre_b, smem_u32(mean_s),
                                      smem_u32(rstd_s));
            __syncthreads();
        }
        E* srow = S + (size_t)row0 * D;
        if (ADDNORM) {
            // pass A: mean and rstd of Z[h, :] = mix[h, :] + Xh[h, :], LPR lanes
            // per row, sums shifted by the row's first element
            for (int r0 = warp * RPW; r0 < R; r0 += nw * RPW) {
                const int r = min(r0 + sub, R - 1);   // lanes past the last row repeat it, unwritten
                const int s = r / T, h = r - s * T;
                const E* xsm = xs + (size_t)s * sstride;   // this row's sample
                const float K = to_f(xsm[h * dh]) + to_f(xs[(size_t)r * rs]);
                const float2 nK = f2(-K);
                float2 a1 = f2(0.f), a2 = f2(0.f);
#pragma unroll
                for (int i = 0; i < NV; ++i) {
                    const int v = sl + LPR * i;
                    if (v < nv) {
                        Vec16<E> xm;
                        mixed_vec<E, MV>(xsm, rs, dh, h, v * V, moffA[i], xm);
                        float2 pm[NP], pr[NP];
                        unpack_pairs(xm.u, pm);
                        unpack_pairs(*reinterpret_cast<const uint4*>(xs + (size_t)r * rs + v * V), pr);
#pragma unroll
                        for (int j = 0; j < NP; ++j) {
                            const float2 d = f2_add(f2_add(pm[j], pr[j]), nK);
                            a1 = f2_add(a1, d);
                            a2 = f2_fma(d, d, a2);
                        }
                    }
                }
                float s1 = a1.x + a1.y, s2 = a2.x + a2.y;
#pragma unroll
                for (int o = LPR / 2; o > 0; o >>= 1) {   // within the row's lanes
                    s1 += __shfl_xor_sync(0xffffffffu, s1, o);
                    s2 += __shfl_xor_sync(0xffffffffu, s2, o);
                }
                if (sl == 0 && r0 + sub < R) {
                    const float m1 = s1 / D;
                    const float rstd = rsqrtf(fmaxf(s2 / D - m1 * m1, 0.f) + eps);
                    mean_s[r] = K + m1;
                    rstd_s[r] = rstd;
                    if (SAVE) rstd_out[row0 + r] = rstd;
                }
            }
            __syncthreads();
        }
        // pass B: element-wise, thread (grp, v) over rows grp, grp + groups, ...
        // (groups divides T, so h wraps to the next sample exactly)
        if (active) {
            int h = grp;
            const E* xsm = xs;
#pragma unroll 2
            for (int r = grp; r < R; r += groups) {
                Vec16<E> xm;
                mixed_vec<E, MV>(xsm, rs, dh, h, c0, moff, xm);
                uint4 o = xm.u;   // without Add & Norm: S = TokenMixing(Xh), a permutation
                if (ADDNORM) {
                    float2 pm[NP], pr[NP];
                    unpack_pairs(xm.u, pm);
                    unpack_pairs(*reinterpret_cast<const uint4*>(xs + (size_t)r * rs + c0), pr);
                    const float rr = rstd_s[r];
                    const float2 r2 = f2(rr), mr2 = f2(-mean_s[r] * rr);
#pragma unroll
                    for (int j = 0; j < NP; ++j) pm[j] = f2_fma(f2_add(pm[j], pr[j]), r2, mr2);   // xhat
                    if (SAVE)   // training: the normalised row, kept for the backward pass
                        *reinterpret_cast<uint4*>(xhat_out + (size_t)(row0 + r) * D + c0) = pack_pairs(pm);
#pragma unroll
                    for (int j = 0; j < NP; ++j) pm[j] = f2_fma(pm[j], g1p[j], b1p[j]);
                    o = pack_pairs(pm);
                }
                *reinterpret_cast<uint4*>(srow + (size_t)r * D + c0) = o;
                h += groups;
                if (h >= T) {
                    h -= T;
                    xsm += sstride;
                }
            }
        }
        __syncthreads();   // the slot and the statistics are free again
        const long long nc = c + (long long)nslots * gridDim.x;
        if (warp == 0 && nc < nchunks) ring.issue(cur, X + (size_t)nc * spb * TD, chunk_rows(nc), nc * spb * T);
    }
    if (tid == 0) ring.drain(wc, SITE_MIX_LN);
}

// pooled[b, c] = gamma[c] * (1/T) sum_t (x[t, c] - m_t) r_t + beta[c]; Xout
// (optional) receives LN(x).  CTA = spc samples: its rows' statistics are
// merged from the producer's partials (one warp per row) into shared memory;
// then thread u takes (sample u / nv, 16-byte column vector u % nv) and sums
// that column over the sample's T rows in ascending t (deterministic), with
// eight rows' loads in flight at a time straight from global memory (no
// staging: each element is read once, and many small CTAs keep enough loads
// in flight to cover the memory latency).
constexpr int kPoolThreads = 256;
constexpr int kPoolRowsInFlight = 8;

template <typename E>
__global__ void __launch_bounds__(kPoolThreads, 3) ln_pool_kernel(const E* X, const float2* pstats, int P,
                                                              const float* __restrict__ g,
                                                              const float* __restrict__ bta, float* __restrict__ pooled,
                                                              E* __restrict__ Xout, int B, int T, int D, float eps,
                                                              int spc) {
    pdl_enter();
    constexpr int V = Vec16<E>::N;
    constexpr int NP = V / 2;
    extern __shared__ float rowstat[];   // mean [spc * T], rstd [spc * T]
    float* mean_s = rowstat;
    float* rstd_s = rowstat + spc * T;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    const long long b0 = (long long)blockIdx.x * spc;
    const int ns = (int)min((long long)spc, B - b0);
    const int R = ns * T;
    const float n = (float)D / (float)P;
    for (int r = warp; r < R; r += 8 * nw) {   // eight rows' partials in flight per warp
        float2 v[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int rr = r + k * nw;
            v[k] = (rr < R && lane < P) ? __ldcg(pstats + (b0 * T + rr) * P + lane) : make_float2(0.f, 0.f);
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int rr = r + k * nw;
            if (rr < R) {   // warp-uniform
                const float mean = warp_sum(v[k].x) / (float)P;
                const float d = v[k].x - mean;
                const float q = warp_sum(lane < P ? fmaf(n * d, d, v[k].y) : 0.f);
                if (lane == 0) {
                    mean_s[rr] = mean;
                    rstd_s[rr] = rsqrtf(q / D + eps);
                }
            }
        }
    }
    __syncthreads();
    const int nv = D / V;
    const float invT = 1.0f / T;
    for (int u = tid; u < ns * nv; u += blockDim.x) {
        const int sm = u / nv, c0 = (u - sm * nv) * V;
        const E* col = X + (size_t)(b0 + sm) * T * D + c0;
        float2 gp[NP], bp[NP];
        load_pairs(g + c0, gp);
        load_pairs(bta + c0, bp);
        float2 acc[NP];
#pragma unroll
        for (int j = 0; j < NP; ++j) acc[j] = f2(0.f);
        for (int t0 = 0; t0 < T; t0 += kPoolRowsInFlight) {
            uint4 xv[kPoolRowsInFlight];
#pragma unroll
            for (int k = 0; k < kPoolRowsInFlight; ++k)
                if (t0 + k < T) xv[k] = __ldcg(reinterpret_cast<const uint4*>(col + (size_t)(t0 + k) * D));
#pragma unroll
            for (int k = 0; k < kPoolRowsInFlight; ++k) {
                const int t = t0 + k;
                if (t < T) {
                    float2 x[NP];
                    unpack_pairs(xv[k], x);
                    const float rt = rstd_s[sm * T + t];
                    const float2 r2 = f2(rt), mr2 = f2(-mean_s[sm * T + t] * rt);
#pragma unroll
                    for (int j = 0; j < NP; ++j) {
                        x[j] = f2_fma(x[j], r2, mr2);   // (x - m_t) r_t
                        acc[j] = f2_add(acc[j], x[j]);
                    }
                    if (Xout) {
#pragma unroll
                        for (int j = 0; j < NP; ++j) x[j] = f2_fma(x[j], gp[j], bp[j]);
                        *reinterpret_cast<uint4*>(Xout + ((size_t)(b0 + sm) * T + t) * D + c0) = pack_pairs(x);
                    }
                }
            }
        }
        float4* dst = reinterpret_cast<float4*>(pooled + (size_t)(b0 + sm) * D + c0);
#pragma unroll
        for (int q = 0; q < NP / 2; ++q) {
            const float2 p0 = f2_fma(gp[2 * q], f2_mul(acc[2 * q], f2(invT)), bp[2 * q]);
            const float2 p1 = f2_fma(gp[2 * q + 1], f2_mul(acc[2 * q + 1], f2(invT)), bp[2 * q + 1]);
            dst[q] = make_float4(p0.x, p0.y, p1.x, p1.y);
        }
    }
}

// (mean, M2) of every row over all D columns (P = 1), one warp per row, one
// pass of sums shifted by the row's first element.
template <typename E>
__global__ void __launch_bounds__(256) row_stats_kernel(const E* __restrict__ X, float2* __restrict__ out,
                                                       long long rows, int D) {
    pdl_enter();
    constexpr int V = Vec16<E>::N;
    const int lane = threadIdx.x & 31;
    const long long r = blockIdx.x * (long long)(blockDim.x >> 5) + (threadIdx.x >> 5);
    if (r >= rows) return;
    const E* x = X + r * D;
    const float K = to_f(x[0]);
    float s1 = 0.f, s2 = 0.f;
    for (int v = lane; v < D / V; v += 32) {
        Vec16<E> u;
        u.u = __ldcg(reinterpret_cast<const uint4*>(x) + v);
#pragma unroll
        for (int e = 0; e < V; ++e) {
            const float d = to_f(u.e[e]) - K;
            s1 += d;
            s2 = fmaf(d, d, s2);
        }
    }
    s1 = warp_sum(s1);
    s2 = warp_sum(s2);
    if (lane == 0) out[r] = make_float2(K + s1 / D, fmaxf(s2 - s1 * s1 / D, 0.f));
}

// Samples per ring slot: small samples travel in chunks of about 48 KB (the
// nearest whole number of samples), so the per-chunk synchronisation and
// statistics are amortised while two CTAs with two slots each fit an SM.
constexpr size_t kChunkTargetBytes = 48 * 1024;
inline int samples_per_chunk(int T, int rs, size_t esz, int B) {
    const size_t one = (size_t)T * rs * esz;
    long long spb = (long long)((kChunkTargetBytes + one / 2) / one);
    if (spb > B) spb = B;
    return spb < 1 ? 1 : (int)spb;
}

// Ring slots (up to kMaxSlots, at least 1) and dynamic shared memory for
// chunks of `rows` rows at row stride rs, with P staged partials per row (P =
// 0: none), plus the per-row statistics and extra_floats floats, for `per_sm`
// CTAs per SM (two, each with as many slots as fit, whenever one slot each
// fits: measured in the stack, two independent CTAs -- one computes while the
// other waits for its copy -- beat one CTA with a deeper ring).
inline void ring_shape(int rows, int rs, size_t esz, int P, int per_sm, int* nslots, size_t* smem,
                       size_t extra_floats = 0) {
    const size_t one = slot_bytes_of(rows, rs, esz, P);
    const size_t fixed = 8 * kMaxSlots + sizeof(float) * (2 * (size_t)rows + extra_floats) + 32;
    const size_t full = 227 * 1024 - 1024;    // static shared memory and slack
    const size_t half = full / 2 - 1024;
    const size_t avail = per_sm > 1 && one + fixed <= half ? half : full;
    long long n = avail > fixed ? (long long)((avail - fixed) / one) : 0;
    if (n > kMaxSlots) n = kMaxSlots;
    if (n < 1) n = 1;
    *nslots = (int)n;
    *smem = (size_t)n * one + fixed;
}

// Row groups: the largest divisor of T (so every group gets the same rows)
// with groups * nv <= cap threads.
inline int mix_groups_cap(int T, int nv, int cap) {
    int g = cap / nv;
    if (g > T) g = T;
    while (g > 1 && T % g) --g;
    return g < 1 ? 1 : g;
}
inline int mix_groups(int T, int nv) { return mix_groups_cap(T, nv, kMixMaxThreads); }

template <typename E, bool PRE, int MV, int NVV, bool ADDNORM, int LPR, bool SAVE>
cudaError_t mix_ln_go(const E* X, const float* pg, const float* pb, RowStats ps, const float* g1, const float* b1,
                      E* S, int B, int T, int D, float eps, int num_sms, DeviceErr err, uint64_t budget,
                      cudaStream_t s, E* xhat_out, float* rstd_out) {
    constexpr int V = Vec16<E>::N;
    const int nv = D / V;
    if (nv < 1 || nv > kMixMaxThreads) return cudaErrorInvalidValue;
    const int groups = mix_groups(T, nv);
    int threads = (groups * nv + 31) / 32 * 32;
    if (threads < 64) threads = 64;
    const int rs = MV == V ? mix_row_stride(D, D / T, sizeof(E)) : D;
    const int spb = samples_per_chunk(T, rs, sizeof(E), B);
    int nslots;
    size_t smem;
    ring_shape(spb * T, rs, sizeof(E), PRE ? ps.P : 0, 2, &nslots, &smem);
    auto k = mix_ln_kernel<E, PRE, MV, NVV, ADDNORM, LPR, SAVE>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, threads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const long long nchunks = (B + spb - 1) / spb;
    const long long g = (long long)num_sms * per_sm;
    const int grid = (int)(g < nchunks ? g : nchunks);
    return launch_pdl(k, grid, threads, smem, s, X, pg, pb, ps.part, ps.P, g1, b1, S, B, T, D, eps, rs, spb, nslots,
                      groups, err, budget, xhat_out, rstd_out);
}

// Lanes per row of the statistics pass: 8 for rows of <= 64 vectors, 16 for
// <= 128, else 32, so each lane takes at most 8 vectors (NV) and a warp works
// on 32/LPR rows at once.
template <typename E, bool PRE, int MV>
cudaError_t mix_ln_nv(int nv, int addnorm, const E* X, const float* pg, const float* pb, RowStats ps,
                      const float* g1, const float* b1, E* S, int B, int T, int D, float eps, int num_sms,
                      DeviceErr err, uint64_t budget, cudaStream_t s, E* xo, float* ro) {
    // the training outputs exist for bf16 rows of whole 16-byte pieces only
    constexpr bool kSaveOk = sizeof(E) == 2 && MV == Vec16<E>::N;
#define RM_MIX_GO(NVV, AN, LPRV)                                                                                    \
    ((kSaveOk && AN && xo)                                                                                          \
         ? mix_ln_go<E, PRE, MV, NVV, AN, LPRV, kSaveOk && AN>(X, pg, pb, ps, g1, b1, S, B, T, D, eps, num_sms, err, \
                                                              budget, s, xo, ro)                                   \
         : mix_ln_go<E, PRE, MV, NVV, AN, LPRV, false>(X, pg, pb, ps, g1, b1, S, B, T, D, eps, num_sms, err, budget, \
                                                      s, nullptr, nullptr))
    if (!addnorm) return RM_MIX_GO(1, false, 32);
    if (nv <= 64) {
        const int nvl = (nv + 7) / 8;
        switch (nvl) {
            case 1: return RM_MIX_GO(1, true, 8);
            case 2: return RM_MIX_GO(2, true, 8);
            case 3: return RM_MIX_GO(3, true, 8);
            case 4: return RM_MIX_GO(4, true, 8);
            case 5: return RM_MIX_GO(5, true, 8);
            case 6: return RM_MIX_GO(6, true, 8);
            default: return RM_MIX_GO(8, true, 8);
        }
    }
    if (nv <= 128) {
        const int nvl = (nv + 15) / 16;
        return nvl <= 5 ? RM_MIX_GO(5, true, 16) : nvl <= 6 ? RM_MIX_GO(6, true, 16) : RM_MIX_GO(8, true, 16);
    }
    if (nv <= 256) {
        const int nvl = (nv + 31) / 32;
        return nvl <= 5 ? RM_MIX_GO(5, true, 32) : nvl <= 6 ? RM_MIX_GO(6, true, 32) : RM_MIX_GO(8, true, 32);
    }
#undef RM_MIX_GO
    return cudaErrorInvalidValue;
}

template <typename E>
cudaError_t mix_ln_typed(const void* X, const float* pg, const float* pb, RowStats ps, const float* g1,
                         const float* b1, void* S, int B, int T, int D, float eps, int addnorm, int num_sms,
                         DeviceErr err, uint64_t budget, cudaStream_t s, void* xhat_out, float* rstd_out) {
    constexpr int V = Vec16<E>::N;
    const int nv = D / V;
    const int dh = D / T;
    const int mv = dh % V == 0 ? V : (dh % (V / 2) == 0 ? V / 2 : 1);
    const E* x = static_cast<const E*>(X);
    E* y = static_cast<E*>(S);
#define RM_MIX_MV(PREV, MVV) \
    mix_ln_nv<E, PREV, MVV>(nv, addnorm, x, pg, pb, ps, g1, b1, y, B, T, D, eps, num_sms, err, budget, s, \
                            static_cast<E*>(xhat_out), rstd_out)
#define RM_MIX_PRE(PREV) (mv == V ? RM_MIX_MV(PREV, V) : mv == V / 2 ? RM_MIX_MV(PREV, V / 2) : RM_MIX_MV(PREV, 1))
    const cudaError_t e = pg ? RM_MIX_PRE(true) : RM_MIX_PRE(false);
#undef RM_MIX_PRE
#undef RM_MIX_MV
    return e;
}

template <typename E>
cudaError_t ln_pool_go(const void* X, RowStats stats, const float* g, const float* b, float* pooled, void* Xout, int B,
                       int T, int D, float eps, cudaStream_t s) {
    constexpr int V = Vec16<E>::N;
    const int nv = D / V;
    if (nv < 1 || nv > kPoolThreads) return cudaErrorInvalidValue;
    int spc = kPoolThreads / nv;   // samples per CTA
    if (spc > B) spc = B;
    if (spc < 1) spc = 1;
    const int threads = std::max(64, (spc * nv + 31) / 32 * 32);
    const size_t smem = sizeof(float) * 2 * (size_t)spc * T;
    const int grid = (B + spc - 1) / spc;
    return launch_pdl(ln_pool_kernel<E>, grid, threads, smem, s, static_cast<const E*>(X), stats.part, stats.P, g,
                      b, pooled, static_cast<E*>(Xout), B, T, D, eps, spc);
}

}  // namespace

// Largest D per dtype the mixing kernel supports (8 vectors per lane in its
// statistics pass).
int mix_ln_max_d(int dtype) { return 32 * 8 * (dtype == RM_BF16 ? 8 : 4); }

// Whether one staged sample (padded for the mixing gather) with its staged
// LayerNorm partials (D/64 per row for bf16 rows of a multiple of 64 columns,
// else 1) and per-row statistics fits a CTA's shared memory.
bool mix_ln_sample_fits(int dtype, int T, int D) {
    const size_t esz = dtype == RM_BF16 ? 2 : 4;
    const int V = (int)(16 / esz);
    const int dh = D / T;
    const int rs = dh % V == 0 ? mix_row_stride(D, dh, esz) : D;
    const int P = (dtype == RM_BF16 && D % 64 == 0) ? D / 64 : 1;   // LayerNorm partials per row
    const size_t fixed = 8 * kMaxSlots + sizeof(float) * 2 * (size_t)T + 32;
    return slot_bytes_of(T, rs, esz, P) + fixed <= 227 * 1024 - 1024;
}

cudaError_t launch_mix_ln(int dtype, const void* X, const float* pre_g, const float* pre_b, RowStats pre_stats,
                          const float* g1, const float* b1, void* S, int B, int T, int D, float eps, int addnorm,
                          int num_sms, DeviceErr err, uint64_t budget_ns, cudaStream_t s, void* xhat_out,
                          float* rstd_out) {
    if (pre_g && (!pre_stats.part || pre_stats.P < 1 || pre_stats.P > 32)) return cudaErrorInvalidValue;
    if ((xhat_out || rstd_out) && (!addnorm || !xhat_out || !rstd_out || dtype != RM_BF16 || (D / T) % 8))
        return cudaErrorInvalidValue;
    if (dtype == RM_BF16)
        return mix_ln_typed<__nv_bfloat16>(X, pre_g, pre_b, pre_stats, g1, b1, S, B, T, D, eps, addnorm, num_sms,
                                           err, budget_ns, s, xhat_out, rstd_out);
    return mix_ln_typed<float>(X, pre_g, pre_b, pre_stats, g1, b1, S, B, T, D, eps, addnorm, num_sms, err,
                               budget_ns, s, xhat_out, rstd_out);
}

cudaError_t launch_ln_pool(int dtype, const void* X, RowStats stats, const float* g, const float* b, float* pooled,
                           void* Xout, int B, int T, int D, float eps, int num_sms, DeviceErr err, uint64_t budget_ns,
                           cudaStream_t s) {
    (void)num_sms;   // (a grid of ceil(B / samples per CTA) small CTAs; no waits)
    (void)err;
    (void)budget_ns;
    if (!stats.part || stats.P < 1 || stats.P > 32) return cudaErrorInvalidValue;
    if (dtype == RM_BF16)
        return ln_pool_go<__nv_bfloat16>(X, stats, g, b, pooled, Xout, B, T, D, eps, s);
    return ln_pool_go<float>(X, stats, g, b, pooled, Xout, B, T, D, eps, s);
}

cudaError_t launch_row_stats(int dtype, const void* X, float2* out, long long rows, int D, cudaStream_t s) {
    const int grid = (int)((rows + 7) / 8);
    if (dtype == RM_BF16)
        return launch_pdl(row_stats_kernel<__nv_bfloat16>, grid, 256, 0, s, static_cast<const __nv_bfloat16*>(X), out,
                          rows, D);
    return launch_pdl(row_stats_kernel<float>, grid, 256, 0, s, static_cast<const float*>(X), out, rows, D);
}

}  // namespace rm
