// T-grouped bf16 GEMM on the 5th-generation tensor cores (tcgen05) of sm_100a.
//
// The per-token FFN of RankMixer (fun-rec chapter "Rankmixer: 硬件效率优化",
// section Per-Token FFN) applies T independent weight sets, one per token.
// Executed for a batch it is the grouped product [T, B, D] @ [T, D, kD] ->
// [T, B, kD] of "重新理解 RankMixer：扩参为什么有效，又为什么划算？" section 3.2,
// followed by [T, B, kD] @ [T, kD, D].  This kernel computes
//     out[g, m, n] = epilogue( sum_k A[g, m, k] * W[g, n, k] )
// for every group g, with A rows addressed through strides (so the token-t
// rows of S [B, T, D] are read in place) and W stored [G][N][K].
//
// Structure (persistent; dense problems use CTA pairs, cluster of 2, with
// 256 x BN tiles and tcgen05.mma.cta_group::2; expert groups use single CTAs
// with 128 x BN tiles):
//   warp 0      TMA producer: A and W tiles (64-wide K slices, 128-byte
//               swizzle) into a STAGES-deep shared-memory ring.
//   warp 1      MMA issuer: one thread issues tcgen05.mma (K=16 per
//               instruction) into a double-buffered fp32 accumulator in tensor
//               memory and releases ring slots / accumulators with
//               tcgen05.commit.
//   warps 2..9  epilogue: tcgen05.ld of the accumulator, bias + GELU / ReLU,
//               bias + residual (+ LayerNorm partials), or gate * (acc + bias),
//               bf16 out (TMA stores of 64-column chunks for dense tiles).
//               Two warps per 32-lane TMEM quarter.
// The last partial wave of dense tiles is split along K (split-K tail).
// Every mbarrier wait is bounded (rm_device.cuh); a wait that runs out records
// RM_ERR_DEVICE_TIMEOUT, stops the CTA's other roles, drains in-flight copies
// and MMAs, frees tensor memory and returns.
#include <cuda.h>
#include <cuda_bf16.h>

#include <cstdio>
#include <cstdlib>
#include <cstring>

#include "rm_device.cuh"
#include "rm_tmap.h"

namespace rm {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;       // bf16 elements per 128-byte swizzle row
constexpr int UMMA_K = 16;   // K per tcgen05.mma of kind::f16
constexpr int kEpiWarps = 8;
constexpr int kThreads = (2 + kEpiWarps) * 32;
constexpr int kMaxVarGroups = 2048 + 1;   // entries of the variable-row tile prefix (G <= 2048)

struct KParams {
    int G, M, N, K;
    int var_rows;
    int a_g_inner;            // A map coordinate order (k, g, m) if 1, else (k, m, g)
    int o_g_inner;            // out / resid map coordinate order (n, g, m) if 1, else (n, m, g)
    __nv_bfloat16* out;
    long long o_gstride, o_ld;
    const float* bias;
    const __nv_bfloat16* resid;
    long long r_gstride, r_ld;
    const float* gate;
    const int* grp_cnt;
    const int* grp_off;
    const int* mtile_prefix;
    float2* stats;            // LayerNorm partials of stored rows (dense EPI_BIAS_RESID), or null
    long long s_gstride, s_ld;
    // Split-K tail (dense only): tiles [full_tiles, tiles) are each computed
    // as nsplit K-slices by different CTAs; fp32 partials go to sk_ws and the
    // last slice to finish (per-warp arrival counters sk_cnt) sums them in
    // slice order and runs the epilogue.  nsplit = 1: no split items.
    long long full_tiles;
    int nsplit;
    float* sk_ws;
    int* sk_cnt;
    int save_pre;             // activation epilogues: also store bf16(acc + bias), the activation's input, via tmR
    int w_from_kernel;        // W (B operand) written by an earlier kernel: no loads before the launch wait
    int w_g_inner;            // W map coordinate order (k|n, g, n|k) if 1, else (k|n, n|k, g)
    // Variable-K groups (weight gradients of the sparse-MoE experts): dense
    // G x M x N tiles whose K rows are rows [grp_off[g], grp_off[g] + grp_cnt[g])
    // of the compacted A and W operands (grp_cnt a multiple of 64, the padding
    // rows zero); group coordinate 0 in both maps.
    int vark;
    // e4m3 operands (EPI_F8_*): dequantisation scales of A's rows and W's rows
    const float* ascale;
    long long as_gstride, as_ld;
    const float* wscale;
    DeviceErr err;
    unsigned long long budget_ns;
};

// Tile shapes.  CG = 1: one CTA computes a 128 x BN tile.  CG = 2: a CTA pair
// (cluster of 2) computes a 256 x BN tile with 2-SM MMAs; each CTA loads its
// 128 rows of A and BN/2 rows of B and holds its 128 accumulator rows.
template <int BN, int CG, bool VAR>
struct Cfg {
    static constexpr int BN_LOCAL = BN / CG;   // W rows this CTA loads per tile
    static constexpr int TM = BM * CG;         // output rows per tile
    static constexpr int A_BYTES = BM * BK * 2;
    static constexpr int B_BYTES = BN_LOCAL * BK * 2;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    // Dense tiles leave the epilogue through a 32 x 64 bf16 staging buffer per
    // epilogue warp (TMA stores); variable-row tiles store rows directly.
    static constexpr int STAGING_BYTES = VAR ? 0 : kEpiWarps * 4096;
    // as many ring stages as fit next to the staging buffers, the 1 KB
    // alignment slack and the barriers (227 KB per CTA)
    // variable-row tiles keep the tile prefix table (G + 1 ints) in shared memory
    static constexpr int TABLE_BYTES = VAR ? kMaxVarGroups * 4 + 16 : 0;
    static constexpr int STAGES_RAW = (227 * 1024 - 1024 - 512 - STAGING_BYTES - TABLE_BYTES) / STAGE_BYTES;
    static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
    static constexpr int TMEM_COLS = 2 * BN <= 128 ? 128 : (2 * BN <= 256 ? 256 : 512);
    static constexpr int NBARS = 2 * STAGES + 5 + kEpiWarps;
    static constexpr int BAR_BYTES = 8 * NBARS + 16;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + STAGING_BYTES + BAR_BYTES + TABLE_BYTES;
    static_assert(BN % 64 == 0 || VAR, "dense tiles leave in 64-column chunks");
    static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "BN");
    static_assert(B_BYTES % 1024 == 0, "stage alignment");
    static_assert(CG == 1 || CG == 2, "CTA group");
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

struct Tile {
    int g;        // weight group
    int ag;       // A map group coordinate
    int arow;     // A map row coordinate of this CTA's first row
    int rows;     // valid rows of this CTA's 128 (may be <= 0)
    int n0;       // first output column of the tile
    long long orow0;  // out / resid row index of this CTA's first row (group-local in dense mode)
};

// mt: the variable-row tile prefix (mtile_prefix, staged in shared memory).
template <int CG>
__device__ __forceinline__ Tile decode_tile(const KParams& p, long long idx, int nblk, int mblk, int bn,
                                            int rank, const int* mt = nullptr) {
    Tile t;
    if (!p.var_rows) {
        const long long per_g = (long long)nblk * mblk;
        t.g = (int)(idx / per_g);
        const int r = (int)(idx - (long long)t.g * per_g);
        const int nb = r / mblk, mb = r - nb * mblk;
        const int m0 = mb * (BM * CG) + rank * BM;
        t.ag = p.vark ? 0 : t.g;
        t.arow = m0;
        t.rows = min(BM, p.M - m0);
        t.n0 = nb * bn;
        t.orow0 = m0;
    } else {   // tiles of BM * CG rows; rank r of a pair takes rows [r*BM, r*BM + BM) of it
        int lo = 0, hi = p.G;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if ((long long)mt[mid] * nblk <= idx) lo = mid; else hi = mid;
        }
        const int p0 = mt[lo];
        const int nt = mt[lo + 1] - p0;
        const int local = (int)(idx - (long long)p0 * nblk);
        const int nb = local / nt, mb = local - nb * nt;
        const int m0 = mb * (BM * CG) + rank * BM;
        const int off = __ldcg(p.grp_off + lo);
        t.g = lo;
        t.ag = 0;
        t.arow = off + m0;
        t.rows = min(BM, __ldcg(p.grp_cnt + lo) - m0);   // <= 0: the odd CTA of a pair past the group's end
        t.n0 = nb * bn;
        t.orow0 = off + m0;
    }
    return t;
}

// Work item idx -> tile index, K-block range and (for split items) the tail
// tile's ordinal and this item's slice.  Items below full_tiles are whole tiles.
struct Item {
    long long tile;
    int kb_lo, kb_hi;
    int koff;    // K offset of the tile's group (variable-K groups), else 0
    int tj;      // tail tile ordinal (split items), else -1
    int slice;
};

__device__ __forceinline__ Item decode_item(const KParams& p, long long idx, int num_kb, long long per_g = 1) {
    Item it;
    it.koff = 0;
    if (idx < p.full_tiles || p.nsplit == 1) {
        it.tile = idx;
        it.kb_lo = 0;
        it.kb_hi = num_kb;
        it.tj = -1;
        it.slice = 0;
        if (p.vark) {   // this group's K rows
            const int g = (int)(idx / per_g);
            it.kb_hi = __ldcg(p.grp_cnt + g) / BK;
            it.koff = __ldcg(p.grp_off + g);
        }
    } else {
        const long long j = idx - p.full_tiles;
        it.tj = (int)(j / p.nsplit);
        it.slice = (int)(j - (long long)it.tj * p.nsplit);
        it.tile = p.full_tiles + it.tj;
        it.kb_lo = (int)((long long)it.slice * num_kb / p.nsplit);
        it.kb_hi = (int)((long long)(it.slice + 1) * num_kb / p.nsplit);
    }
    return it;
}

// Operand layouts in shared memory (one ring stage): K-major operands are
// single TMA boxes of 64 K x rows (128-byte swizzled rows of K); M- or
// N-major operands (AMN / BMN, the backward products) are boxes of 64 rows x
// 64 K, one 8 KB box per 64 rows, each K row a 128-byte swizzled run of 64
// rows.
constexpr uint32_t kMnChunkBytes = 64 * BK * 2;

// A ring stage's operand tile of `rows` rows starting at row r0 and K column
// kc, from map tm whose coordinate order is (k|r, g, r|k) with g_inner, else
// (k|r, r|k, g).  pair: completion counted on the even CTA's barrier.
template <bool MN, int ROWS, bool PAIR>
__device__ __forceinline__ void load_operand(uint32_t dst, const CUtensorMap* tm, uint32_t bar, int kc, int r0, int g,
                                             int g_inner) {
    if constexpr (!MN) {
        if (PAIR) {
            if (g_inner) tma_load_3d_pair(dst, tm, bar, kc, g, r0);
            else tma_load_3d_pair(dst, tm, bar, kc, r0, g);
        } else {
            if (g_inner) tma_load_3d(dst, tm, bar, kc, g, r0);
            else tma_load_3d(dst, tm, bar, kc, r0, g);
        }
    } else {
#pragma unroll
        for (int c = 0; c < ROWS / 64; ++c) {
            const uint32_t d = dst + (uint32_t)c * kMnChunkBytes;
            const int r = r0 + 64 * c;
            if (PAIR) {
                if (g_inner) tma_load_3d_pair(d, tm, bar, r, g, kc);
                else tma_load_3d_pair(d, tm, bar, r, kc, g);
            } else {
                if (g_inner) tma_load_3d(d, tm, bar, r, g, kc);
                else tma_load_3d(d, tm, bar, r, kc, g);
            }
        }
    }
}

// Derivative of the FFN activation at u (the backward products' epilogue).
template <int EPI>
__device__ __forceinline__ float dact(float u) {
    if constexpr (EPI == EPI_DACT_RELU) {
        return u > 0.f ? 1.f : 0.f;
    } else if constexpr (EPI == EPI_DACT_ERF) {
        // d/du [u Phi(u)] = Phi(u) + u phi(u)
        return 0.5f * (1.0f + erff(u * 0.7071067811865476f)) + u * 0.3989422804014327f * __expf(-0.5f * u * u);
    } else {
        // tanh form: g(u) = u/2 (1 + tanh(a)), a = c (u + 0.044715 u^3), c = sqrt(2/pi)
        // g'(u) = (1 + tanh(a))/2 + u/2 (1 - tanh(a)^2) c (1 + 3 * 0.044715 u^2)
        const float c = 0.7978845608028654f;
        const float a = c * fmaf(0.044715f * u * u, u, u);
        float th;
        asm("tanh.approx.f32 %0, %1;" : "=f"(th) : "f"(a));
        return fmaf(0.5f * u * c * fmaf(3.0f * 0.044715f, u * u, 1.0f), 1.0f - th * th, 0.5f * (1.0f + th));
    }
}

// The derivative at a pair of points: the tanh form in paired fp32
// instructions (two elements an instruction, tanh from the SFU), the other
// activations element by element.
template <int EPI>
__device__ __forceinline__ float2 dact_pair(float2 u) {
    if constexpr (EPI == EPI_DACT_TANH) {
        const float c = 0.7978845608028654f;
        const float2 u2 = f2_mul(u, u);
        const float2 a = f2_mul(u, f2_fma(u2, f2(c * 0.044715f), f2(c)));      // c (u + 0.044715 u^3)
        float2 th;
        asm("tanh.approx.f32 %0, %1;" : "=f"(th.x) : "f"(a.x));
        asm("tanh.approx.f32 %0, %1;" : "=f"(th.y) : "f"(a.y));
        const float2 hd = f2_mul(f2_mul(u, f2(0.5f)), f2_fma(u2, f2(3.0f * 0.044715f * c), f2(c)));
        const float2 sech2 = f2_fma(th, make_float2(-th.x, -th.y), f2(1.0f));   // 1 - tanh^2
        return f2_fma(hd, sech2, f2_fma(th, f2(0.5f), f2(0.5f)));
    } else {
        return make_float2(dact<EPI>(u.x), dact<EPI>(u.y));
    }
}

template <int BN, int EPI, int CG, bool VAR, bool AMN = false, bool BMN = false>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmR,
                   const KParams p) {
    using C = Cfg<BN, CG, VAR>;
    static_assert(!(VAR && AMN), "variable-row groups read a K-major A");
    static_assert(!BMN || C::BN_LOCAL % 64 == 0, "N-major W tiles are whole 64-row boxes");
    constexpr bool DACT = EPI == EPI_DACT_TANH || EPI == EPI_DACT_ERF || EPI == EPI_DACT_RELU;
    constexpr bool F32OUT = EPI == EPI_F32;
    // e4m3 operands: the bf16 epilogue EB after dequantisation; a ring stage
    // holds KE = 128 one-byte K elements per row instead of 64 bf16
    constexpr bool F8 = EPI >= EPI_F8_GELU_TANH;
    constexpr int EB = EPI == EPI_F8_GELU_TANH ? EPI_GELU_TANH
                       : EPI == EPI_F8_GELU_ERF ? EPI_GELU_ERF
                       : EPI == EPI_F8_RELU ? EPI_RELU
                       : EPI == EPI_F8_BIAS_RESID ? EPI_BIAS_RESID : EPI;
    constexpr int KE = F8 ? 128 : BK;
    static_assert(!(F8 && (VAR || AMN || BMN || CG == 0)), "e4m3 operands: dense, K-major");
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    unsigned char* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(smem);
    const uint32_t staging0 = sbase + C::STAGES * C::STAGE_BYTES;   // 1024-aligned
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES + C::STAGING_BYTES);
    const uint32_t full0 = smem_u32(bars);
    const uint32_t empty0 = full0 + 8 * C::STAGES;
    const uint32_t tfull0 = empty0 + 8 * C::STAGES;
    const uint32_t tempty0 = tfull0 + 16;
    const uint32_t drain_bar = tempty0 + 16;
    const uint32_t rbar0 = drain_bar + 8;      // one per epilogue warp: residual tile loads
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBARS);
    int* mt_table = reinterpret_cast<int*>(smem + C::STAGES * C::STAGE_BYTES + C::STAGING_BYTES + C::BAR_BYTES);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = CG == 2 ? cluster_ctarank() : 0u;
    const bool leader = rank == 0;
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull0 + 8 * a, 1);
            mbar_init(tempty0 + 8 * a, CG * kEpiWarps * 32);
        }
        mbar_init(drain_bar, 1);
        for (int w = 0; w < kEpiWarps; ++w) mbar_init(rbar0 + 8 * w, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
        if (!VAR) prefetch_tmap(&tmO);
    }
    if (warp == 0) {
        if (CG == 2) {
            tmem_alloc_pair(smem_u32(tmem_slot), C::TMEM_COLS);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (CG == 2) cluster_sync_all();   // the peer's barriers exist before anyone signals them
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // The set-up above overlaps the previous kernel's tail (programmatic
    // launch).  Every thread waits for that kernel before it touches data an
    // earlier kernel wrote; only the producer's first weight tiles come before
    // the wait (no kernel writes weights).
    pdl_trigger();
    if (VAR) {   // the tile count and prefix come from the routing kernels
        pdl_wait();
        for (int i = threadIdx.x; i <= p.G; i += blockDim.x) mt_table[i] = __ldcg(p.mtile_prefix + i);
        __syncthreads();
    }

    const WaitCtx wc{abort_flag, p.budget_ns, p.err};
    const int nblk = (p.N + BN - 1) / BN;
    const int mblk = (p.M + C::TM - 1) / C::TM;
    const int num_kb = (p.K + KE - 1) / KE;
    const long long total = p.var_rows ? (long long)mt_table[p.G] * nblk
                                       : p.full_tiles + ((long long)p.G * nblk * mblk - p.full_tiles) * p.nsplit;
    const long long unit = blockIdx.x / CG, nunits = gridDim.x / CG;
    const long long per_g = (long long)nblk * mblk;   // tiles per group (dense decode)

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            int stage = 0;
            uint32_t phase = 0, issued = 0, issued_phase = 0;
            bool ok = true;
            // Weight (B) tiles of the first tile's first stages, before the wait.
            int npre = 0;
            if (!VAR && !p.w_from_kernel && !p.vark && unit < total) {
                const Item it0 = decode_item(p, unit, num_kb);
                const Tile t0 = decode_tile<CG>(p, it0.tile, nblk, mblk, BN, (int)rank, mt_table);
                const int nb0 = t0.n0 + (int)rank * C::BN_LOCAL;
                npre = min(C::STAGES, it0.kb_hi - it0.kb_lo);
                for (int k = 0; k < npre; ++k) {   // fresh ring: every slot is free
                    const uint32_t fb = full0 + 8 * k;
                    if (leader) mbar_arrive_expect_tx(fb, CG * C::STAGE_BYTES);
                    const uint32_t sb = sbase + k * C::STAGE_BYTES + C::A_BYTES;
                    const int kc = (it0.kb_lo + k) * KE;
                    load_operand<BMN, C::BN_LOCAL, CG == 2>(sb, &tmB, CG == 2 ? mapa_shared(fb, 0) : fb, kc, nb0,
                                                            t0.g, p.w_g_inner);
                }
            }
            pdl_wait();
            bool first = true;
            for (long long idx = unit; idx < total && ok; idx += nunits) {
                const Item item = decode_item(p, idx, num_kb, per_g);
                const Tile t = decode_tile<CG>(p, item.tile, nblk, mblk, BN, (int)rank, mt_table);
                const int nb0 = t.n0 + (int)rank * C::BN_LOCAL;
                const int wg = p.vark ? 0 : t.g;   // W map group coordinate
                for (int kb = item.kb_lo; kb < item.kb_hi; ++kb) {
                    const bool pre = first && kb - item.kb_lo < npre;   // B already issued
                    if (!pre && !mbar_wait(empty0 + 8 * stage, phase ^ 1u, wc, SITE_TC_PRODUCER)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = full0 + 8 * stage;
                    if (leader && !pre) mbar_arrive_expect_tx(fb, CG * C::STAGE_BYTES);
                    const uint32_t sa = sbase + stage * C::STAGE_BYTES;
                    const int kc = kb * KE + item.koff;
                    // the pair counts bytes on the even CTA's barrier
                    const uint32_t fbl = CG == 2 ? mapa_shared(fb, 0) : fb;
                    load_operand<AMN, BM, CG == 2>(sa, &tmA, fbl, kc, t.arow, t.ag, p.a_g_inner);
                    if (!pre) load_operand<BMN, C::BN_LOCAL, CG == 2>(sa + C::A_BYTES, &tmB, fbl, kc, nb0, wg, p.w_g_inner);
                    issued |= 1u << stage;
                    issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
                }
                first = false;
            }
            // Every issued copy must land before the CTA's shared memory goes
            // away (for a pair, the even CTA's barrier counts both CTAs' bytes).
            if (leader)
                for (int s = 0; s < C::STAGES; ++s)
                    if (issued & (1u << s))
                        mbar_wait(full0 + 8 * s, (issued_phase >> s) & 1u, wc, SITE_TC_DRAIN, false);
        }
        __syncwarp();
    } else if (warp == 1) {
        pdl_wait();   // (reads no global memory; keeps every thread ordered after the previous kernel)
        if (lane == 0 && leader) {
            // ------------------------------------------------ MMA issuer
            constexpr uint32_t idesc = F8 ? idesc_e4m3_f32(C::TM, BN) : idesc_bf16_f32(C::TM, BN, AMN, BMN);
            // per K = 16 step: 32 bytes along a K-major row, or 16 K rows (2 KB)
            // of an M/N-major tile; descriptors count 16-byte units
            constexpr uint64_t a_step = AMN ? 128 : 2, b_step = BMN ? 128 : 2;
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true, any = false;
            int it = 0;
            for (long long idx = unit; idx < total && ok; idx += nunits, ++it) {
                const int acc = it & 1;
                const uint32_t aph = (uint32_t)(it >> 1) & 1u;
                if (!mbar_wait(tempty0 + 8 * acc, aph ^ 1u, wc, SITE_TC_MMA_TMEM)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                const Item item = decode_item(p, idx, num_kb, per_g);
                for (int kb = item.kb_lo; kb < item.kb_hi; ++kb) {
                    if (!mbar_wait(full0 + 8 * stage, phase, wc, SITE_TC_MMA_FULL)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = sbase + stage * C::STAGE_BYTES;
                    const uint64_t adesc = AMN ? smem_desc_mn_sw128(sa, kMnChunkBytes) : smem_desc_k_sw128(sa);
                    const uint64_t bdesc = BMN ? smem_desc_mn_sw128(sa + C::A_BYTES, kMnChunkBytes)
                                               : smem_desc_k_sw128(sa + C::A_BYTES);
#pragma unroll
                    for (int k = 0; k < BK / UMMA_K; ++k) {
                        const uint32_t accum = (kb != item.kb_lo || k != 0) ? 1u : 0u;
                        if constexpr (F8) {   // (a K step of 32 bytes, as for bf16)
                            if (CG == 2)
                                tc_mma_f8_pair(d_tmem, adesc + a_step * k, bdesc + b_step * k, idesc, accum);
                            else
                                tc_mma_f8(d_tmem, adesc + a_step * k, bdesc + b_step * k, idesc, accum);
                        } else {
                            if (CG == 2)
                                tc_mma_f16_pair(d_tmem, adesc + a_step * k, bdesc + b_step * k, idesc, accum);
                            else
                                tc_mma_f16(d_tmem, adesc + a_step * k, bdesc + b_step * k, idesc, accum);
                        }
                    }
                    if (CG == 2) tc_commit_pair_mc(empty0 + 8 * stage, 0x3);
                    else tc_commit(empty0 + 8 * stage);
                    any = true;
                    if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                if (CG == 2) tc_commit_pair_mc(tfull0 + 8 * acc, 0x3);
                else tc_commit(tfull0 + 8 * acc);
            }
            // Every issued MMA must complete before tensor memory is released.
            if (any) {
                if (CG == 2) tc_commit_pair(drain_bar);
                else tc_commit(drain_bar);
                mbar_wait(drain_bar, 0, wc, SITE_TC_DRAIN, false);
            }
        }
        __syncwarp();
    } else if constexpr (!VAR) {
        pdl_wait();
        // ------------------------------------- epilogue, dense: TMA stores
        // Each warp owns 32 accumulator rows (its TMEM lane quarter) and half
        // of the BN columns, in 64-column chunks: tcgen05.ld -> registers ->
        // bias / GELU / residual -> bf16 into a 128-byte-swizzled 32 x 64
        // staging buffer -> one TMA bulk store (float output instead goes
        // through the buffer as a transpose and leaves as whole 128-byte
        // lines from the registers).  The residual tile arrives in the same
        // buffer by TMA first.  The accumulator is released right after the
        // tile's last tcgen05.ld.
        const int ew = warp - 2;
        const int quarter = warp & 3;
        const int half = ew >> 2;
        // 64-column chunks alternate between the two halves (chunk k -> half
        // k % 2), so every chunk, and the LayerNorm partial of its 64 columns,
        // belongs to one warp; CH = chunks of the larger share.
        constexpr int CH = (BN / 64 + 1) / 2;
        const uint32_t tempty_leader = CG == 2 ? mapa_shared(tempty0, 0) : tempty0;
        const uint32_t stg = staging0 + (uint32_t)ew * 4096u;
        const uint32_t rbar = rbar0 + 8u * (uint32_t)ew;
        uint32_t rphase = 0;
        const bool has_resid = (EB == EPI_BIAS_RESID || DACT) && p.resid != nullptr;
        const uint32_t my_row = stg + (uint32_t)lane * 128u;
        const uint32_t swz = (uint32_t)(lane & 7);
        int it = 0;
        for (long long idx = unit; idx < total; idx += nunits, ++it) {
            const Item item = decode_item(p, idx, num_kb);
            const Tile t = decode_tile<CG>(p, item.tile, nblk, mblk, BN, (int)rank, mt_table);
            const int acc = it & 1;
            const uint32_t aph = (uint32_t)(it >> 1) & 1u;
            if (!mbar_wait(tfull0 + 8 * acc, aph, wc, SITE_TC_EPILOGUE)) break;
            tc_fence_after();
            const int wrow0 = (int)t.orow0 + quarter * 32;
            const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BN);
            const float* bias_g = p.bias ? p.bias + (long long)t.g * p.N : nullptr;
            const bool split = item.tj >= 0;
            // this warp's block (CH chunks of 32 x 64) of slice s of tail tile tj: [chunk][16 float4][lane]
            const long long wsblk = split ? (((long long)item.tj * p.nsplit) * CG + rank) * kEpiWarps + ew : 0;
            const long long wstride = (long long)CG * kEpiWarps * (CH * 512);   // float4s between slices
            float4* wsw = split ? reinterpret_cast<float4*>(p.sk_ws) + wsblk * (CH * 512) : nullptr;
            if (split) {
                // dump this slice's partial sums, release the accumulator, count the arrival
#pragma unroll 1
                for (int c = 64 * half; c < BN; c += 128) {
                    float v[64];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        float w16[16];
                        tmem_ld16(tbase + (uint32_t)(c + 16 * q), w16);
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[16 * q + e] = w16[e];
                    }
                    tmem_ld_wait();
                    float4* dst = wsw + (long long)item.slice * wstride + ((c - 64 * half) / 128) * 16 * 32 + lane;
#pragma unroll
                    for (int q = 0; q < 16; ++q) __stcg(dst + q * 32, make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]));
                }
                tc_fence_before();
                if (CG == 2 && !leader) mbar_arrive_cluster_relaxed(tempty_leader + 8u * (uint32_t)acc);
                else mbar_arrive(tempty0 + 8 * acc);
                __threadfence();
                __syncwarp();
                int* cnt = p.sk_cnt + ((long long)item.tj * CG + rank) * kEpiWarps + ew;
                int last = 0;
                if (lane == 0) {
                    int old;
                    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;" : "=r"(old) : "l"(cnt) : "memory");
                    last = old == p.nsplit - 1;
                    if (last) *cnt = 0;   // ready for the next launch
                }
                last = __shfl_sync(0xffffffffu, last, 0);
                if (!last) continue;
                __threadfence();
            }
            bool ok = true;
#pragma unroll 1
            for (int c = 64 * half; c < BN; c += 128) {
                const int n = t.n0 + c;
                const bool live = n < p.N;   // warp-uniform
                if (!F32OUT) {   // (float output: transposed line stores below)
                    if (lane == 0) bulk_wait_read_all();   // the previous store has read the buffer
                    __syncwarp();
                }
                if (has_resid && live && lane == 0) {
                    mbar_arrive_expect_tx(rbar, 4096);
                    if (p.o_g_inner) tma_load_3d(stg, &tmR, rbar, n, t.g, wrow0);
                    else tma_load_3d(stg, &tmR, rbar, n, wrow0, t.g);
                }
                float v[64];
                if (split) {
                    // the tile's sum over its K slices, always in slice order
                    const float4* src = wsw + ((c - 64 * half) / 128) * 16 * 32 + lane;
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        const float4 a = __ldcg(src + q * 32);
                        v[4 * q] = a.x;
                        v[4 * q + 1] = a.y;
                        v[4 * q + 2] = a.z;
                        v[4 * q + 3] = a.w;
                    }
#pragma unroll 1
                    for (int sl = 1; sl < p.nsplit; ++sl) {
#pragma unroll
                        for (int q = 0; q < 16; ++q) {
                            const float4 a = __ldcg(src + sl * wstride + q * 32);
                            v[4 * q] += a.x;
                            v[4 * q + 1] += a.y;
                            v[4 * q + 2] += a.z;
                            v[4 * q + 3] += a.w;
                        }
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        float w16[16];
                        tmem_ld16(tbase + (uint32_t)(c + 16 * q), w16);
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[16 * q + e] = w16[e];
                    }
                    tmem_ld_wait();
                }
                if (!split && c + 128 >= BN) {   // this warp's last chunk: the accumulator may be reused
                    tc_fence_before();
                    if (CG == 2 && !leader) mbar_arrive_cluster_relaxed(tempty_leader + 8u * (uint32_t)acc);
                    else mbar_arrive(tempty0 + 8 * acc);
                }
                if (!live) continue;
                if constexpr (F8) {   // dequantise: acc * ascale[row] * wscale[g][n + e]
                    const int mrow = wrow0 + lane;
                    const float sa =
                        mrow < p.M ? __ldg(p.ascale + (long long)t.g * p.as_gstride + (long long)mrow * p.as_ld) : 0.f;
                    const float4* ws4 = reinterpret_cast<const float4*>(p.wscale + (long long)t.g * p.N + n);
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        if (n + 4 * q < p.N) {
                            const float4 w = __ldg(ws4 + q);
                            v[4 * q] *= sa * w.x;
                            v[4 * q + 1] *= sa * w.y;
                            v[4 * q + 2] *= sa * w.z;
                            v[4 * q + 3] *= sa * w.w;
                        }
                    }
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    if (bias_g && n + 16 * q < p.N) {
                        const float4* b4 = reinterpret_cast<const float4*>(bias_g + n + 16 * q);
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            const float4 bb = __ldg(b4 + r);
                            const int e = 16 * q + 4 * r;
                            const float2 lo = f2_add(make_float2(v[e], v[e + 1]), make_float2(bb.x, bb.y));
                            const float2 hi = f2_add(make_float2(v[e + 2], v[e + 3]), make_float2(bb.z, bb.w));
                            v[e] = lo.x;
                            v[e + 1] = lo.y;
                            v[e + 2] = hi.x;
                            v[e + 3] = hi.y;
                        }
                    }
                }
                if ((EB == EPI_RELU || EB == EPI_GELU_TANH || EB == EPI_GELU_ERF) && p.save_pre) {
                    // the activation's input, kept for the backward pass: its own
                    // store through the staging buffer, before the activation
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(my_row + ((((uint32_t)j) ^ swz) << 4)),
                                     "r"(pack_bf16x2(v[8 * j], v[8 * j + 1])), "r"(pack_bf16x2(v[8 * j + 2], v[8 * j + 3])),
                                     "r"(pack_bf16x2(v[8 * j + 4], v[8 * j + 5])), "r"(pack_bf16x2(v[8 * j + 6], v[8 * j + 7]))
                                     : "memory");
                    fence_proxy_async_shared();
                    __syncwarp();
                    if (lane == 0) {
                        if (p.o_g_inner) tma_store_3d(&tmR, stg, n, t.g, wrow0);
                        else tma_store_3d(&tmR, stg, n, wrow0, t.g);
                        bulk_commit_group();
                        bulk_wait_read_all();
                    }
                    __syncwarp();
                }
                if (EB == EPI_RELU) {
#pragma unroll
                    for (int e = 0; e < 64; ++e) v[e] = fmaxf(v[e], 0.0f);
                } else if (EB == EPI_GELU_TANH) {
#pragma unroll
                    for (int e = 0; e < 64; e += 2) {
                        const float2 y = gelu_tanh_pair(make_float2(v[e], v[e + 1]));
                        v[e] = y.x;
                        v[e + 1] = y.y;
                    }
                } else if (EB == EPI_GELU_ERF) {
#pragma unroll
                    for (int e = 0; e < 64; ++e) v[e] = 0.5f * v[e] * (1.0f + erff(v[e] * 0.7071067811865476f));
                } else if (EB == EPI_BIAS_RESID || DACT) {
                    if (has_resid) {
                        if (!mbar_wait(rbar, rphase, wc, SITE_TC_EPILOGUE)) {
                            ok = false;
                            break;
                        }
                        rphase ^= 1u;
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            uint4 u;
                            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                         : "=r"(u.x), "=r"(u.y), "=r"(u.z), "=r"(u.w)
                                         : "r"(my_row + ((((uint32_t)j) ^ swz) << 4)));
                            float2 rp[4];
                            unpack_pairs(u, rp);
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 a = make_float2(v[8 * j + 2 * e], v[8 * j + 2 * e + 1]);
                                const float2 y = DACT ? f2_mul(a, dact_pair<EPI>(rp[e]))
                                                      : f2_add(a, rp[e]);
                                v[8 * j + 2 * e] = y.x;
                                v[8 * j + 2 * e + 1] = y.y;
                            }
                        }
                    }
                }
                if constexpr (F32OUT) {
                    // Two 32-column float halves, transposed through the
                    // staging buffer: the lanes write their rows, then read
                    // back four whole rows per instruction (8 lanes x 16 bytes
                    // a row) and store them as full 128-byte lines.  No bulk
                    // store to wait for, so a warp's stores are not limited
                    // to one 4 KB buffer in flight.
                    float* obase = reinterpret_cast<float*>(p.out) + (long long)t.g * p.o_gstride;
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int n2 = n + 32 * hh;
                        if (n2 >= p.N) break;   // warp-uniform; N is a multiple of 32
                        __syncwarp();          // every lane has read the previous half
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const float* q = v + 32 * hh + 4 * j;
                            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                                             my_row + ((((uint32_t)j) ^ swz) << 4)),
                                         "r"(__float_as_uint(q[0])), "r"(__float_as_uint(q[1])),
                                         "r"(__float_as_uint(q[2])), "r"(__float_as_uint(q[3]))
                                         : "memory");
                        }
                        __syncwarp();
                        const uint32_t ju = (uint32_t)(lane & 7);
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const int r = 4 * i + (lane >> 3);
                            uint32_t x0, x1, x2, x3;
                            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                         : "=r"(x0), "=r"(x1), "=r"(x2), "=r"(x3)
                                         : "r"(stg + (uint32_t)r * 128u + ((ju ^ (uint32_t)(r & 7)) << 4))
                                         : "memory");
                            if (wrow0 + r < p.M)
                                __stcs(reinterpret_cast<float4*>(obase + (long long)(wrow0 + r) * p.o_ld + n2 +
                                                                 4 * (int)ju),
                                       make_float4(__uint_as_float(x0), __uint_as_float(x1), __uint_as_float(x2),
                                                   __uint_as_float(x3)));
                        }
                    }
                    continue;
                }
                uint32_t w[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) w[j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
                if (EB == EPI_BIAS_RESID && p.stats != nullptr && wrow0 + lane < p.M) {
                    // LayerNorm partials of the stored (rounded) 64 values: (mean, M2)
                    float2 a1 = f2(0.f);
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        a1 = f2_add(a1, make_float2(__uint_as_float(w[j] << 16), __uint_as_float(w[j] & 0xffff0000u)));
                    const float mean = (a1.x + a1.y) * (1.0f / 64.0f);
                    const float2 nm = f2(-mean);
                    float2 a2 = f2(0.f);
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const float2 d = f2_add(make_float2(__uint_as_float(w[j] << 16), __uint_as_float(w[j] & 0xffff0000u)), nm);
                        a2 = f2_fma(d, d, a2);
                    }
                    const float q = a2.x + a2.y;
                    p.stats[(long long)t.g * p.s_gstride + (long long)(wrow0 + lane) * p.s_ld + (n >> 6)] =
                        make_float2(mean, q);
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(my_row + ((((uint32_t)j) ^ swz) << 4)),
                                 "r"(w[4 * j]), "r"(w[4 * j + 1]), "r"(w[4 * j + 2]), "r"(w[4 * j + 3])
                                 : "memory");
                }
                fence_proxy_async_shared();
                __syncwarp();
                if (lane == 0) {
                    if (p.o_g_inner) tma_store_3d(&tmO, stg, n, t.g, wrow0);
                    else tma_store_3d(&tmO, stg, n, wrow0, t.g);
                    bulk_commit_group();
                }
            }
            if (!ok) break;
        }
        if (lane == 0) bulk_wait_all();
        __syncwarp();
    } else {
        // (the wait for the routing kernels came before the tile count)
        // ------------------------------ epilogue, variable rows: row stores
        const int ew = warp - 2;
        const int quarter = warp & 3;          // TMEM lanes this warp may access
        const int half = ew >> 2;              // which half of the BN columns
        const int row = quarter * 32 + lane;
        constexpr int HALF = BN / 2;
        // the pair's accumulator-free barrier lives on the even CTA
        const uint32_t tempty_leader = CG == 2 ? mapa_shared(tempty0, 0) : tempty0;
        int it = 0;
        for (long long idx = unit; idx < total; idx += nunits, ++it) {
            const Tile t = decode_tile<CG>(p, idx, nblk, mblk, BN, (int)rank, mt_table);
            const int acc = it & 1;
            const uint32_t aph = (uint32_t)(it >> 1) & 1u;
            if (!mbar_wait(tfull0 + 8 * acc, aph, wc, SITE_TC_EPILOGUE)) break;
            tc_fence_after();
            const bool row_ok = row < t.rows;
            const long long orow = t.orow0 + row;
            const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BN);
            const float* bias_g = p.bias ? p.bias + (long long)t.g * p.N : nullptr;
            __nv_bfloat16* out_row = p.out + (long long)t.g * p.o_gstride + orow * p.o_ld;
            // bf16 row of the same shape as out: the activation input (DACT, loaded)
            // or the pre-activation values (save_pre, stored)
            const long long rrow = orow * p.r_ld;
            float gate = 1.f;
            if (EPI == EPI_BIAS_GATE && row_ok && p.gate) gate = __ldcg(p.gate + orow);
            // DACT: the activation input of the row, one 16-column chunk ahead
            uint4 un[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
            if (DACT && row_ok && t.n0 + half * HALF < p.N) {
                const uint4* u4 = reinterpret_cast<const uint4*>(p.resid + rrow + t.n0 + half * HALF);
                un[0] = __ldcg(u4);
                un[1] = __ldcg(u4 + 1);
            }
#pragma unroll 1
            for (int c = half * HALF; c < (half + 1) * HALF; c += 16) {
                const uint4 uc[2] = {un[0], un[1]};
                if (DACT && row_ok && c + 16 < (half + 1) * HALF && t.n0 + c + 16 < p.N) {
                    const uint4* u4 = reinterpret_cast<const uint4*>(p.resid + rrow + t.n0 + c + 16);
                    un[0] = __ldcg(u4);
                    un[1] = __ldcg(u4 + 1);
                }
                float v[16];
                tmem_ld16(tbase + (uint32_t)c, v);
                tmem_ld_wait();
                const int n = t.n0 + c;
                if (row_ok && n < p.N) {
                    if (bias_g) {
                        const float4* b4 = reinterpret_cast<const float4*>(bias_g + n);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const float4 bb = __ldg(b4 + q);
                            const float2 lo = f2_add(make_float2(v[4 * q], v[4 * q + 1]), make_float2(bb.x, bb.y));
                            const float2 hi = f2_add(make_float2(v[4 * q + 2], v[4 * q + 3]), make_float2(bb.z, bb.w));
                            v[4 * q] = lo.x;
                            v[4 * q + 1] = lo.y;
                            v[4 * q + 2] = hi.x;
                            v[4 * q + 3] = hi.y;
                        }
                    }
                    if ((EPI == EPI_RELU || EPI == EPI_GELU_TANH || EPI == EPI_GELU_ERF) && p.save_pre) {
                        uint4* pre = reinterpret_cast<uint4*>(const_cast<__nv_bfloat16*>(p.resid) + rrow + n);
                        pre[0] = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                                            pack_bf16x2(v[6], v[7]));
                        pre[1] = make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]),
                                            pack_bf16x2(v[12], v[13]), pack_bf16x2(v[14], v[15]));
                    }
                    if (EPI == EPI_RELU) {
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] = fmaxf(v[e], 0.0f);
                    } else if (EPI == EPI_GELU_TANH) {
#pragma unroll
                        for (int e = 0; e < 16; e += 2) {
                            const float2 y = gelu_tanh_pair(make_float2(v[e], v[e + 1]));
                            v[e] = y.x;
                            v[e + 1] = y.y;
                        }
                    } else if (EPI == EPI_GELU_ERF) {
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] = 0.5f * v[e] * (1.0f + erff(v[e] * 0.7071067811865476f));
                    } else if (DACT) {   // acc * act'(U), U the stored activation input of the row
#pragma unroll
                        for (int q = 0; q < 2; ++q) {
                            float2 up[4];
                            unpack_pairs(uc[q], up);
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 y = f2_mul(make_float2(v[8 * q + 2 * e], v[8 * q + 2 * e + 1]),
                                                        dact_pair<EPI>(up[e]));
                                v[8 * q + 2 * e] = y.x;
                                v[8 * q + 2 * e + 1] = y.y;
                            }
                        }
                    } else if (EPI == EPI_BIAS_GATE) {
#pragma unroll
                        for (int e = 0; e < 16; e += 2) {
                            const float2 y = f2_mul(make_float2(v[e], v[e + 1]), f2(gate));
                            v[e] = y.x;
                            v[e + 1] = y.y;
                        }
                    }
                    uint4 o0, o1;
                    o0.x = pack_bf16x2(v[0], v[1]);
                    o0.y = pack_bf16x2(v[2], v[3]);
                    o0.z = pack_bf16x2(v[4], v[5]);
                    o0.w = pack_bf16x2(v[6], v[7]);
                    o1.x = pack_bf16x2(v[8], v[9]);
                    o1.y = pack_bf16x2(v[10], v[11]);
                    o1.z = pack_bf16x2(v[12], v[13]);
                    o1.w = pack_bf16x2(v[14], v[15]);
                    uint4* dst = reinterpret_cast<uint4*>(out_row + n);
                    dst[0] = o0;
                    dst[1] = o1;
                }
            }
            tc_fence_before();
            if (CG == 2 && !leader) mbar_arrive_cluster_relaxed(tempty_leader + 8u * (uint32_t)acc);
            else mbar_arrive(tempty0 + 8 * acc);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (CG == 2) cluster_sync_all();   // the pair's MMAs and copies are done before either CTA leaves
    if (warp == 0) {
        tc_fence_after();
        if (CG == 2) tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
        else tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

// ----------------------------------------------------------------- host side
struct Maps {
    CUtensorMap a, b, o, r;
};

template <int BN, int EPI, int CG, bool VAR, bool AMN = false, bool BMN = false>
cudaError_t launch_typed(const Maps& m, const KParams& kp, int grid, cudaStream_t s) {
    using C = Cfg<BN, CG, VAR>;
    auto k = gemm_tc_kernel<BN, EPI, CG, VAR, AMN, BMN>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CG;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, k, m.a, m.b, m.o, m.r, kp);
}

// Operand layouts of the backward products: (K-major A, N-major W) for the
// activation gradients, (M-major A, N-major W) for the weight gradients.
template <int BN, int CG>
cudaError_t launch_bn_mn(int epi, bool a_mn, const Maps& m, const KParams& kp, int grid, cudaStream_t s) {
    if constexpr ((BN / CG) % 64 != 0) {
        return cudaErrorInvalidValue;
    } else {
        if (a_mn) {
            if (epi == EPI_F32) return launch_typed<BN, EPI_F32, CG, false, true, true>(m, kp, grid, s);
            return cudaErrorInvalidValue;
        }
        switch (epi) {
            case EPI_DACT_TANH: return launch_typed<BN, EPI_DACT_TANH, CG, false, false, true>(m, kp, grid, s);
            case EPI_DACT_ERF: return launch_typed<BN, EPI_DACT_ERF, CG, false, false, true>(m, kp, grid, s);
            case EPI_DACT_RELU: return launch_typed<BN, EPI_DACT_RELU, CG, false, false, true>(m, kp, grid, s);
            case EPI_BIAS_RESID: return launch_typed<BN, EPI_BIAS_RESID, CG, false, false, true>(m, kp, grid, s);
        }
        return cudaErrorInvalidValue;
    }
}

// Variable-row groups with an N-major W (the sparse-MoE experts' activation
// gradients): acc x act'(U), or plain acc (EPI_BIAS_GATE without bias and gate).
template <int BN>
cudaError_t launch_bn_var_mn(int epi, const Maps& m, const KParams& kp, int grid, cudaStream_t s) {
    if constexpr (BN % 64 != 0) {
        return cudaErrorInvalidValue;
    } else {
        switch (epi) {
            case EPI_DACT_TANH: return launch_typed<BN, EPI_DACT_TANH, 1, true, false, true>(m, kp, grid, s);
            case EPI_DACT_ERF: return launch_typed<BN, EPI_DACT_ERF, 1, true, false, true>(m, kp, grid, s);
            case EPI_DACT_RELU: return launch_typed<BN, EPI_DACT_RELU, 1, true, false, true>(m, kp, grid, s);
            case EPI_BIAS_GATE: return launch_typed<BN, EPI_BIAS_GATE, 1, true, false, true>(m, kp, grid, s);
        }
        return cudaErrorInvalidValue;
    }
}

template <int BN, int CG, bool VAR>
cudaError_t launch_bn(int epi, const Maps& m, const KParams& kp, int grid, cudaStream_t s) {
    switch (epi) {
        case EPI_GELU_TANH: return launch_typed<BN, EPI_GELU_TANH, CG, VAR>(m, kp, grid, s);
        case EPI_GELU_ERF: return launch_typed<BN, EPI_GELU_ERF, CG, VAR>(m, kp, grid, s);
        case EPI_RELU: return launch_typed<BN, EPI_RELU, CG, VAR>(m, kp, grid, s);
        case EPI_BIAS_RESID:
            if constexpr (!VAR) return launch_typed<BN, EPI_BIAS_RESID, CG, VAR>(m, kp, grid, s);
            break;
        case EPI_BIAS_GATE:
            if constexpr (VAR) return launch_typed<BN, EPI_BIAS_GATE, CG, VAR>(m, kp, grid, s);
            break;
        case EPI_F8_GELU_TANH:
            if constexpr (!VAR) return launch_typed<BN, EPI_F8_GELU_TANH, CG, VAR>(m, kp, grid, s);
            break;
        case EPI_F8_GELU_ERF:
            if constexpr (!VAR) return launch_typed<BN, EPI_F8_GELU_ERF, CG, VAR>(m, kp, grid, s);
            break;
        case EPI_F8_RELU:
            if constexpr (!VAR) return launch_typed<BN, EPI_F8_RELU, CG, VAR>(m, kp, grid, s);
            break;
        case EPI_F8_BIAS_RESID:
            if constexpr (!VAR) return launch_typed<BN, EPI_F8_BIAS_RESID, CG, VAR>(m, kp, grid, s);
            break;
    }
    return cudaErrorInvalidValue;
}

}  // namespace

// Tile width for N: the candidate with the best product of column fill, a
// per-width tensor-core efficiency measured on B200 with 2-SM tiles at
// K = 1536..6144 (BN 256 : 192 : 128 = 1 : 0.88 : 0.74), and a damped wave
// fill over the SMs (a partial last wave costs less than its share, since the
// tiles of that wave see less L2 contention).
// K slices per tail tile: the last partial wave's `tail` tiles are spread
// over the otherwise idle units, each slice keeping >= 8 K blocks.
static int split_slices(long long tiles, int units, int num_kb) {
    const long long tail = tiles % units;
    if (tail == 0) return 1;
    long long S = units / tail;
    if (S > 8) S = 8;
    while (S > 1 && num_kb / S < 8) --S;
    return (int)S;
}

static cudaError_t launch_gemm_tc_nosplit(const GroupedGemm& g, DeviceErr err, uint64_t budget_ns, int num_sms,
                                   cudaStream_t s) {
    GroupedGemm h = g;
    h.sk_ws = nullptr;
    h.sk_cnt = nullptr;
    return launch_gemm_tc(h, err, budget_ns, num_sms, s);
}

static int gemm_tc_pick_bn(int G, int M, int N, int K, bool var_rows, int num_sms, int cg, bool split,
                           bool w_mn = false) {
    const int cands[4] = {256, 192, 160, 128};
    const double mma_eff[4] = {1.0, 0.88, 0.8, 0.74};
    int best = 256;
    double best_s = -1.0;
    for (int i = 0; i < 4; ++i) {
        const int bn = cands[i];
        if (!var_rows && bn % 64) continue;   // dense tiles leave in 64-column chunks
        if (w_mn && (bn / cg) % 64) continue;  // N-major W tiles are whole 64-row boxes
        const long long nblk = (N + bn - 1) / bn;
        const double col_fill = (double)N / (double)(nblk * bn);
        double wave_fill = 1.0;
        if (!var_rows) {
            const long long units = num_sms / cg;
            const long long tiles = (long long)G * ((M + BM * cg - 1) / (BM * cg)) * nblk;
            const long long waves = (tiles + units - 1) / units;
            wave_fill = (double)tiles / (double)(waves * units);
            if (split) {   // the tail wave costs about 1/S of a wave
                const int S = split_slices(tiles, (int)units, (K + BK - 1) / BK);
                if (S > 1) wave_fill = (double)tiles / ((double)(tiles / units) * units + (double)units / S);
            }
        }
        const double sc = col_fill * mma_eff[i] * (0.5 + 0.5 * wave_fill);
        if (sc > best_s + 1e-9) {
            best_s = sc;
            best = bn;
        }
    }
    return best;
}

cudaError_t launch_gemm_tc(const GroupedGemm& g, DeviceErr err, uint64_t budget_ns, int num_sms, cudaStream_t s) {
    if (g.K % 8 || g.N % 16 || g.G < 1 || g.M < 0 || g.K < 1) return cudaErrorInvalidValue;
    const bool var = g.grp_cnt != nullptr;
    if (var && g.G + 1 > kMaxVarGroups) return cudaErrorInvalidValue;
    const bool dact = g.epi == EPI_DACT_TANH || g.epi == EPI_DACT_ERF || g.epi == EPI_DACT_RELU;
    const bool f32out = g.epi == EPI_F32;
    const bool mn = g.a_mn || g.w_mn;
    const bool vark = g.vark;
    // layouts the kernel is instantiated for
    if (var && (vark || g.a_mn || (g.w_mn && !dact && g.epi != EPI_BIAS_GATE) || (dact && !g.w_mn)))
        return cudaErrorInvalidValue;
    if (!var && mn && (!g.w_mn || (g.a_mn != f32out) || (!g.a_mn && !dact && g.epi != EPI_BIAS_RESID)))
        return cudaErrorInvalidValue;
    if (vark && (!g.a_mn || !g.w_mn || !f32out || !g.grp_off || !g.vark_cnt)) return cudaErrorInvalidValue;
    const bool f8 = g.epi >= EPI_F8_GELU_TANH;
    if (f8 && (var || vark || mn || !g.ascale || !g.wscale || g.K % 16)) return cudaErrorInvalidValue;
    const uint64_t ae = f8 ? 1 : 2;   // bytes per A / W element
    if (f32out && !mn) return cudaErrorInvalidValue;
    if (dact && !mn) return cudaErrorInvalidValue;
    if (dact && !g.resid) return cudaErrorInvalidValue;
    if (g.a_mn && g.M % 8) return cudaErrorInvalidValue;   // 16-byte rows of an M-major A
    if (f32out && g.N % 32) return cudaErrorInvalidValue;
    KParams kp{};
    kp.G = g.G;
    kp.M = g.M;
    kp.N = g.N;
    kp.K = g.K;
    kp.var_rows = var ? 1 : 0;
    kp.vark = vark ? 1 : 0;
    kp.out = static_cast<__nv_bfloat16*>(g.out);
    kp.o_gstride = var ? 0 : g.o_gstride;
    kp.o_ld = g.o_ld;
    kp.bias = g.bias;
    kp.resid = static_cast<const __nv_bfloat16*>(g.resid);
    kp.r_gstride = var ? 0 : g.r_gstride;
    kp.r_ld = g.r_ld;
    kp.gate = g.gate;
    kp.grp_cnt = vark ? g.vark_cnt : g.grp_cnt;
    kp.grp_off = g.grp_off;
    kp.mtile_prefix = g.mtile_prefix;
    kp.stats = g.stats;
    kp.s_gstride = g.s_gstride;
    kp.s_ld = g.s_ld;
    if (g.stats && (var || (g.epi != EPI_BIAS_RESID && g.epi != EPI_F8_BIAS_RESID) || g.N % 64))
        return cudaErrorInvalidValue;
    kp.full_tiles = 0;
    kp.nsplit = 1;
    kp.sk_ws = g.sk_ws;
    kp.sk_cnt = g.sk_cnt;
    kp.w_from_kernel = (g.w_from_kernel || vark) ? 1 : 0;
    // activation epilogues with resid set: resid receives the pre-activation values
    kp.save_pre = (g.resid && (g.epi == EPI_GELU_TANH || g.epi == EPI_GELU_ERF || g.epi == EPI_RELU)) ? 1 : 0;
    kp.w_g_inner = 0;
    kp.ascale = g.ascale;
    kp.as_gstride = g.as_gstride;
    kp.as_ld = g.as_ld;
    kp.wscale = g.wscale;
    kp.err = err;
    kp.budget_ns = budget_ns;

    // 2-SM (256-row) tiles for dense problems with more than one 128-row block;
    // the variable-row (MoE) groups keep 128-row tiles.
    int cg = var ? (g.var_cg == 2 && !g.w_mn ? 2 : 1) : (g.M > BM ? 2 : 1);
    int bn = gemm_tc_pick_bn(g.G, g.M, g.N, g.K, var, num_sms, cg, g.sk_ws && g.sk_cnt, g.w_mn);
    // Tuning overrides (same kernel, other tile shape): RM_GEMM_CG=1|2, RM_GEMM_BN=256|192|160|128.
    if (const char* e = getenv("RM_GEMM_CG")) {
        const int v = atoi(e);
        if ((v == 1 || (v == 2 && !var)) ) cg = v;
    }
    if (const char* e = getenv("RM_GEMM_BN")) {
        const int v = atoi(e);
        if (v == 256 || v == 192 || v == 128 || (var && v == 160)) bn = v;
    }
    if (g.w_mn && (bn / cg) % 64) bn = 128 * cg > 256 ? 256 : 128 * cg;
    Maps m;
    memset(&m, 0, sizeof(m));
    bool ok;
    if (var) {
        // compacted rows [rows_total, K]
        ok = make_map(&m.a, g.A, g.K, g.a_rows_total, 1, g.a_ld * 2, g.a_rows_total * g.a_ld * 2, BM, 1);
        kp.a_g_inner = 0;
    } else if (vark) {
        // compacted rows [rows_total, M], M-major: K runs over the rows (group coordinate 0)
        ok = make_map(&m.a, g.A, g.M, g.a_rows_total, 1, g.a_ld * 2, g.a_rows_total * g.a_ld * 2, BK, 1);
        kp.a_g_inner = 0;
    } else if (g.a_mn) {
        // M-major A: element (g, m, k) at g*a_gstride + k*a_ld + m; boxes of 64 rows x 64 K
        if (g.a_gstride <= g.a_ld) {
            ok = make_map(&m.a, g.A, g.M, g.G, g.K, g.a_gstride * 2, g.a_ld * 2, 1, BK);
            kp.a_g_inner = 1;
        } else {
            ok = make_map(&m.a, g.A, g.M, g.K, g.G, g.a_ld * 2, g.a_gstride * 2, BK, 1);
            kp.a_g_inner = 0;
        }
    } else if (g.a_gstride <= g.a_ld) {
        // group stride inside the row stride, e.g. S [B, T, D]: dims (K, G, M)
        ok = make_map_e(&m.a, g.A, g.K, g.G, g.M, g.a_gstride * ae, g.a_ld * ae, 1, BM, (int)ae);
        kp.a_g_inner = 1;
    } else {
        // groups outermost, e.g. H [T, B, kD]: dims (K, M, G)
        ok = make_map_e(&m.a, g.A, g.K, g.M, g.G, g.a_ld * ae, g.a_gstride * ae, BM, 1, (int)ae);
        kp.a_g_inner = 0;
    }
    const long long w_ld = g.w_ld ? g.w_ld : g.K, w_gs = g.w_ld ? g.w_gstride : (long long)g.N * g.K;
    if (vark) {
        // compacted rows [rows_total, N], N-major: K runs over the rows (group coordinate 0)
        ok = ok && make_map(&m.b, g.W, g.N, g.a_rows_total, 1, w_ld * 2, g.a_rows_total * w_ld * 2, BK, 1);
    } else if (g.w_mn) {
        // N-major W: element (g, n, k) at g*w_gstride + k*w_ld + n; boxes of 64 rows x 64 K
        if (w_gs <= w_ld) {
            ok = ok && make_map(&m.b, g.W, g.N, g.G, g.K, w_gs * 2, w_ld * 2, 1, BK);
            kp.w_g_inner = 1;
        } else {
            ok = ok && make_map(&m.b, g.W, g.N, g.K, g.G, w_ld * 2, w_gs * 2, BK, 1);
        }
    } else {
        ok = ok && make_map_e(&m.b, g.W, g.K, g.N, g.G, w_ld * ae, w_gs * ae, (uint32_t)(bn / cg), 1, (int)ae);
    }
    if (!var) {
        // output (and residual) tiles of 32 rows x 64 columns (32 for float
        // output), same orientation as A
        const uint64_t osz = f32out ? 4 : 2;
        if (g.o_gstride <= g.o_ld) {
            ok = ok && make_map(&m.o, g.out, g.N, g.G, g.M, g.o_gstride * osz, g.o_ld * osz, 1, 32, f32out);
            kp.o_g_inner = 1;
        } else {
            ok = ok && make_map(&m.o, g.out, g.N, g.M, g.G, g.o_ld * osz, g.o_gstride * osz, 32, 1, f32out);
            kp.o_g_inner = 0;
        }
        if (g.resid) {   // residual / activation input tile (loaded), or the pre-activation output (stored)
            if ((g.r_gstride <= g.r_ld) != (kp.o_g_inner == 1)) return cudaErrorInvalidValue;
            ok = ok && (kp.o_g_inner ? make_map(&m.r, g.resid, g.N, g.G, g.M, g.r_gstride * 2, g.r_ld * 2, 1, 32)
                                     : make_map(&m.r, g.resid, g.N, g.M, g.G, g.r_ld * 2, g.r_gstride * 2, 32, 1));
        }
    }
    if (!ok) return cudaErrorInvalidValue;

    int units = num_sms / cg;
    if (!var) {
        const long long tiles = (long long)g.G * ((g.M + BM * cg - 1) / (BM * cg)) * ((g.N + bn - 1) / bn);
        if (tiles == 0) return cudaSuccess;
        const int ke = f8 ? 128 : BK;   // K elements per ring stage
        const int num_kb = (g.K + ke - 1) / ke;
        const int S = (g.sk_ws && g.sk_cnt && !vark) ? split_slices(tiles, units, num_kb) : 1;
        if (const char* e = getenv("RM_GEMM_SPLIT"))   // tuning override: 0 disables the split tail
            if (atoi(e) == 0 && S > 1) return launch_gemm_tc_nosplit(g, err, budget_ns, num_sms, s);
        const long long tail = S > 1 ? tiles % units : 0;
        kp.full_tiles = tiles - tail;
        kp.nsplit = S;
        const long long items = kp.full_tiles + tail * S;
        if (items < units) units = (int)items;
        if (getenv("RM_GEMM_LOG"))
            fprintf(stderr, "gemm_tc G=%d M=%d N=%d K=%d epi=%d cg=%d bn=%d tiles=%lld tail=%lld slices=%d grid=%d\n",
                    g.G, g.M, g.N, g.K, g.epi, cg, bn, tiles, tail, S, units * cg);
    }
    const int grid = units * cg;
    if (var && g.w_mn) {
        switch (bn) {
            case 256: return launch_bn_var_mn<256>(g.epi, m, kp, grid, s);
            case 192: return launch_bn_var_mn<192>(g.epi, m, kp, grid, s);
            default: return launch_bn_var_mn<128>(g.epi, m, kp, grid, s);
        }
    }
    if (var) {
        if (cg == 2) {
            switch (bn) {
                case 256: return launch_bn<256, 2, true>(g.epi, m, kp, grid, s);
                case 192: return launch_bn<192, 2, true>(g.epi, m, kp, grid, s);
                case 160: return launch_bn<160, 2, true>(g.epi, m, kp, grid, s);
                default: return launch_bn<128, 2, true>(g.epi, m, kp, grid, s);
            }
        }
        switch (bn) {
            case 256: return launch_bn<256, 1, true>(g.epi, m, kp, grid, s);
            case 192: return launch_bn<192, 1, true>(g.epi, m, kp, grid, s);
            case 160: return launch_bn<160, 1, true>(g.epi, m, kp, grid, s);
            default: return launch_bn<128, 1, true>(g.epi, m, kp, grid, s);
        }
    }
    if (mn) {
        if (cg == 2) return bn == 256 ? launch_bn_mn<256, 2>(g.epi, g.a_mn, m, kp, grid, s)
                                      : launch_bn_mn<128, 2>(g.epi, g.a_mn, m, kp, grid, s);
        switch (bn) {
            case 256: return launch_bn_mn<256, 1>(g.epi, g.a_mn, m, kp, grid, s);
            case 192: return launch_bn_mn<192, 1>(g.epi, g.a_mn, m, kp, grid, s);
            default: return launch_bn_mn<128, 1>(g.epi, g.a_mn, m, kp, grid, s);
        }
    }
    if (cg == 2) {
        switch (bn) {
            case 256: return launch_bn<256, 2, false>(g.epi, m, kp, grid, s);
            case 192: return launch_bn<192, 2, false>(g.epi, m, kp, grid, s);
            default: return launch_bn<128, 2, false>(g.epi, m, kp, grid, s);
        }
    }
    switch (bn) {
        case 256: return launch_bn<256, 1, false>(g.epi, m, kp, grid, s);
        case 192: return launch_bn<192, 1, false>(g.epi, m, kp, grid, s);
        default: return launch_bn<128, 1, false>(g.epi, m, kp, grid, s);
    }
}

size_t gemm_tc_split_ws_bytes(int num_sms) { return (size_t)num_sms * BM * 256 * sizeof(float); }
size_t gemm_tc_split_cnt_ints(int num_sms) { return (size_t)num_sms * kEpiWarps; }

}  // namespace rm
