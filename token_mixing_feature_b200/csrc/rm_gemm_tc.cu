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
// Structure (one CTA per SM, persistent over 128 x BN output tiles):
//   warp 0      TMA producer: A and W tiles (64-wide K slices, 128-byte
//               swizzle) into a STAGES-deep shared-memory ring.
//   warp 1      MMA issuer: one thread issues tcgen05.mma (M=128, N=BN, K=16)
//               into a double-buffered fp32 accumulator in tensor memory and
//               releases ring slots / accumulators with tcgen05.commit.
//   warps 2..9  epilogue: tcgen05.ld of the accumulator, bias + GELU, bias +
//               residual, or gate * (acc + bias), bf16 stores.  Two warps per
//               32-lane TMEM quarter, each taking half of the columns.
// Every mbarrier wait is bounded (rm_device.cuh); a wait that runs out records
// RM_ERR_DEVICE_TIMEOUT, stops the CTA's other roles, drains in-flight copies
// and MMAs, frees tensor memory and returns.
#include <cuda.h>
#include <cuda_bf16.h>

#include <mutex>

#include "rm_device.cuh"

namespace rm {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;       // bf16 elements per 128-byte swizzle row
constexpr int UMMA_K = 16;   // K per tcgen05.mma of kind::f16
constexpr int kEpiWarps = 8;
constexpr int kThreads = (2 + kEpiWarps) * 32;

struct KParams {
    int G, M, N, K;
    int var_rows;
    int a_g_inner;            // A map coordinate order (k, g, m) if 1, else (k, m, g)
    __nv_bfloat16* out;
    long long o_gstride, o_ld;
    const float* bias;
    const __nv_bfloat16* resid;
    long long r_gstride, r_ld;
    const float* gate;
    const int* grp_cnt;
    const int* grp_off;
    const int* mtile_prefix;
    DeviceErr err;
    unsigned long long budget_ns;
};

template <int BN>
struct Cfg {
    static constexpr int A_BYTES = BM * BK * 2;
    static constexpr int B_BYTES = BN * BK * 2;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int STAGES_RAW = (216 * 1024) / STAGE_BYTES;
    static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
    static constexpr int TMEM_COLS = 2 * BN <= 128 ? 128 : (2 * BN <= 256 ? 256 : 512);
    static constexpr int BAR_BYTES = 8 * (2 * STAGES + 5) + 16;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + BAR_BYTES;
    static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "BN");
    static_assert(B_BYTES % 1024 == 0, "stage alignment");
};

struct Tile {
    int g;        // weight group
    int ag;       // A map group coordinate
    int arow;     // A map row coordinate of the tile's first row
    int rows;     // valid rows in this tile (<= BM)
    int n0;
    long long orow0;  // out / resid row index of the first row (group-local in dense mode)
};

__device__ __forceinline__ Tile decode_tile(const KParams& p, long long idx, int nblk, int mblk) {
    Tile t;
    if (!p.var_rows) {
        const long long per_g = (long long)nblk * mblk;
        t.g = (int)(idx / per_g);
        const int r = (int)(idx - (long long)t.g * per_g);
        const int nb = r / mblk, mb = r - nb * mblk;
        const int m0 = mb * BM;
        t.ag = t.g;
        t.arow = m0;
        t.rows = min(BM, p.M - m0);
        t.n0 = nb;
        t.orow0 = m0;
    } else {
        int lo = 0, hi = p.G;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if ((long long)__ldg(p.mtile_prefix + mid) * nblk <= idx) lo = mid; else hi = mid;
        }
        const int p0 = __ldg(p.mtile_prefix + lo);
        const int mt = __ldg(p.mtile_prefix + lo + 1) - p0;
        const int local = (int)(idx - (long long)p0 * nblk);
        const int nb = local / mt, mb = local - nb * mt;
        const int m0 = mb * BM;
        const int off = __ldg(p.grp_off + lo);
        t.g = lo;
        t.ag = 0;
        t.arow = off + m0;
        t.rows = min(BM, __ldg(p.grp_cnt + lo) - m0);
        t.n0 = nb;
        t.orow0 = off + m0;
    }
    return t;
}

__device__ __forceinline__ float gelu_tanh_approx(float x) {
    // 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))), tanh from the SFU.
    const float u = 0.7978845608028654f * fmaf(0.044715f * x * x, x, x);
    float th;
    asm("tanh.approx.f32 %0, %1;" : "=f"(th) : "f"(u));
    return 0.5f * x * (1.0f + th);
}

template <int BN, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const KParams p) {
    using C = Cfg<BN>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    unsigned char* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(smem);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
    const uint32_t full0 = smem_u32(bars);
    const uint32_t empty0 = full0 + 8 * C::STAGES;
    const uint32_t tfull0 = empty0 + 8 * C::STAGES;
    const uint32_t tempty0 = tfull0 + 16;
    const uint32_t drain_bar = tempty0 + 16;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * C::STAGES + 5);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull0 + 8 * a, 1);
            mbar_init(tempty0 + 8 * a, kEpiWarps * 32);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const WaitCtx wc{abort_flag, p.budget_ns, p.err};
    const int nblk = (p.N + BN - 1) / BN;
    const int mblk = (p.M + BM - 1) / BM;
    const int num_kb = (p.K + BK - 1) / BK;
    const long long total = p.var_rows ? (long long)__ldg(p.mtile_prefix + p.G) * nblk
                                       : (long long)p.G * nblk * mblk;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            int stage = 0;
            uint32_t phase = 0, issued = 0, issued_phase = 0;
            bool ok = true;
            for (long long idx = blockIdx.x; idx < total && ok; idx += gridDim.x) {
                const Tile t = decode_tile(p, idx, nblk, mblk);
                const int n0 = t.n0 * BN;
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(empty0 + 8 * stage, phase ^ 1u, wc, SITE_TC_PRODUCER)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = full0 + 8 * stage;
                    mbar_arrive_expect_tx(fb, C::STAGE_BYTES);
                    const uint32_t sa = sbase + stage * C::STAGE_BYTES;
                    const int kc = kb * BK;
                    if (p.a_g_inner) tma_load_3d(sa, &tmA, fb, kc, t.ag, t.arow);
                    else tma_load_3d(sa, &tmA, fb, kc, t.arow, t.ag);
                    tma_load_3d(sa + C::A_BYTES, &tmB, fb, kc, n0, t.g);
                    issued |= 1u << stage;
                    issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            // Every issued copy must land before the CTA's shared memory goes away.
            for (int s = 0; s < C::STAGES; ++s)
                if (issued & (1u << s)) mbar_wait(full0 + 8 * s, (issued_phase >> s) & 1u, wc, SITE_TC_DRAIN, false);
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer
            constexpr uint32_t idesc = idesc_bf16_f32(BM, BN);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true, any = false;
            int it = 0;
            for (long long idx = blockIdx.x; idx < total && ok; idx += gridDim.x, ++it) {
                const int acc = it & 1;
                const uint32_t aph = (uint32_t)(it >> 1) & 1u;
                if (!mbar_wait(tempty0 + 8 * acc, aph ^ 1u, wc, SITE_TC_MMA_TMEM)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(full0 + 8 * stage, phase, wc, SITE_TC_MMA_FULL)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = sbase + stage * C::STAGE_BYTES;
                    const uint64_t adesc = smem_desc_k_sw128(sa);
                    const uint64_t bdesc = smem_desc_k_sw128(sa + C::A_BYTES);
#pragma unroll
                    for (int k = 0; k < BK / UMMA_K; ++k) {
                        // advance the start address by k * 32 bytes (16-byte units)
                        tc_mma_f16(d_tmem, adesc + (uint64_t)(2 * k), bdesc + (uint64_t)(2 * k), idesc,
                                   (kb | k) != 0 ? 1u : 0u);
                    }
                    tc_commit(empty0 + 8 * stage);
                    any = true;
                    if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                tc_commit(tfull0 + 8 * acc);
            }
            // Every issued MMA must complete before tensor memory is released.
            if (any) {
                tc_commit(drain_bar);
                mbar_wait(drain_bar, 0, wc, SITE_TC_DRAIN, false);
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------- epilogue
        const int ew = warp - 2;
        const int quarter = warp & 3;          // TMEM lanes this warp may access
        const int half = ew >> 2;              // which half of the BN columns
        const int row = quarter * 32 + lane;
        constexpr int HALF = BN / 2;
        int it = 0;
        for (long long idx = blockIdx.x; idx < total; idx += gridDim.x, ++it) {
            const Tile t = decode_tile(p, idx, nblk, mblk);
            const int acc = it & 1;
            const uint32_t aph = (uint32_t)(it >> 1) & 1u;
            if (!mbar_wait(tfull0 + 8 * acc, aph, wc, SITE_TC_EPILOGUE)) break;
            tc_fence_after();
            const bool row_ok = row < t.rows;
            const long long orow = t.orow0 + row;
            const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BN);
            const float* bias_g = p.bias + (long long)t.g * p.N;
            __nv_bfloat16* out_row = p.out + (long long)t.g * p.o_gstride + orow * p.o_ld;
            float gate = 0.f;
            if (EPI == EPI_BIAS_GATE && row_ok) gate = __ldg(p.gate + orow);
#pragma unroll 1
            for (int c = half * HALF; c < (half + 1) * HALF; c += 16) {
                float v[16];
                tmem_ld16(tbase + (uint32_t)c, v);
                tmem_ld_wait();
                const int n = t.n0 * BN + c;
                if (row_ok && n < p.N) {
                    const float4* b4 = reinterpret_cast<const float4*>(bias_g + n);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float4 bb = __ldg(b4 + q);
                        v[4 * q + 0] += bb.x;
                        v[4 * q + 1] += bb.y;
                        v[4 * q + 2] += bb.z;
                        v[4 * q + 3] += bb.w;
                    }
                    if (EPI == EPI_GELU_TANH) {
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] = gelu_tanh_approx(v[e]);
                    } else if (EPI == EPI_GELU_ERF) {
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] = 0.5f * v[e] * (1.0f + erff(v[e] * 0.7071067811865476f));
                    } else if (EPI == EPI_BIAS_RESID) {
                        if (p.resid) {
                            const uint4* r4 = reinterpret_cast<const uint4*>(
                                p.resid + (long long)t.g * p.r_gstride + orow * p.r_ld + n);
#pragma unroll
                            for (int q = 0; q < 2; ++q) {
                                Vec16<__nv_bfloat16> r;
                                r.u = __ldg(r4 + q);
#pragma unroll
                                for (int e = 0; e < 8; ++e) v[8 * q + e] += __bfloat162float(r.e[e]);
                            }
                        }
                    } else {  // EPI_BIAS_GATE
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] *= gate;
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
            mbar_arrive(tempty0 + 8 * acc);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

// ----------------------------------------------------------------- host side
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// 3-D bf16 tensor map: dims d0 (contiguous), d1, d2 with byte strides s1, s2;
// box (64, b1, b2), 128-byte swizzle, zero fill out of bounds.
bool make_map(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1, uint64_t s2,
              uint32_t b1, uint32_t b2) {
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {s1, s2};
    cuuint32_t box[3] = {(cuuint32_t)BK, b1, b2};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int BN, int EPI>
cudaError_t launch_typed(const CUtensorMap& ma, const CUtensorMap& mb, const KParams& kp, int grid,
                         cudaStream_t s) {
    auto k = gemm_tc_kernel<BN, EPI>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<BN>::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    k<<<grid, kThreads, Cfg<BN>::SMEM_BYTES, s>>>(ma, mb, kp);
    return cudaGetLastError();
}

template <int BN>
cudaError_t launch_bn(int epi, const CUtensorMap& ma, const CUtensorMap& mb, const KParams& kp, int grid,
                      cudaStream_t s) {
    switch (epi) {
        case EPI_GELU_TANH: return launch_typed<BN, EPI_GELU_TANH>(ma, mb, kp, grid, s);
        case EPI_GELU_ERF: return launch_typed<BN, EPI_GELU_ERF>(ma, mb, kp, grid, s);
        case EPI_BIAS_RESID: return launch_typed<BN, EPI_BIAS_RESID>(ma, mb, kp, grid, s);
        case EPI_BIAS_GATE: return launch_typed<BN, EPI_BIAS_GATE>(ma, mb, kp, grid, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

// Tile width for N: the candidate with the best product of column fill, wave
// fill over the SMs, and a per-width tensor-core efficiency (wider tiles read
// less shared memory per MMA).
int gemm_tc_pick_bn(int G, int M, int N, bool var_rows, int num_sms) {
    const int cands[4] = {256, 192, 160, 128};
    const double mma_eff[4] = {1.0, 0.95, 0.92, 0.86};
    int best = 256;
    double best_s = -1.0;
    for (int i = 0; i < 4; ++i) {
        const int bn = cands[i];
        const long long nblk = (N + bn - 1) / bn;
        const double col_fill = (double)N / (double)(nblk * bn);
        double wave_fill = 1.0;
        if (!var_rows) {
            const long long tiles = (long long)G * ((M + BM - 1) / BM) * nblk;
            const long long waves = (tiles + num_sms - 1) / num_sms;
            wave_fill = (double)tiles / (double)(waves * num_sms);
        }
        const double sc = col_fill * wave_fill * mma_eff[i];
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
    KParams kp{};
    kp.G = g.G;
    kp.M = g.M;
    kp.N = g.N;
    kp.K = g.K;
    kp.var_rows = var ? 1 : 0;
    kp.out = static_cast<__nv_bfloat16*>(g.out);
    kp.o_gstride = var ? 0 : g.o_gstride;
    kp.o_ld = g.o_ld;
    kp.bias = g.bias;
    kp.resid = static_cast<const __nv_bfloat16*>(g.resid);
    kp.r_gstride = var ? 0 : g.r_gstride;
    kp.r_ld = g.r_ld;
    kp.gate = g.gate;
    kp.grp_cnt = g.grp_cnt;
    kp.grp_off = g.grp_off;
    kp.mtile_prefix = g.mtile_prefix;
    kp.err = err;
    kp.budget_ns = budget_ns;

    const int bn = gemm_tc_pick_bn(g.G, g.M, g.N, var, num_sms);
    CUtensorMap ma, mb;
    bool ok;
    if (var) {
        // compacted rows [rows_total, K]
        ok = make_map(&ma, g.A, g.K, g.a_rows_total, 1, g.a_ld * 2, g.a_rows_total * g.a_ld * 2, BM, 1);
        kp.a_g_inner = 0;
    } else if (g.a_gstride <= g.a_ld) {
        // group stride inside the row stride, e.g. S [B, T, D]: dims (K, G, M)
        ok = make_map(&ma, g.A, g.K, g.G, g.M, g.a_gstride * 2, g.a_ld * 2, 1, BM);
        kp.a_g_inner = 1;
    } else {
        // groups outermost, e.g. H [T, B, kD]: dims (K, M, G)
        ok = make_map(&ma, g.A, g.K, g.M, g.G, g.a_ld * 2, g.a_gstride * 2, BM, 1);
        kp.a_g_inner = 0;
    }
    ok = ok && make_map(&mb, g.W, g.K, g.N, g.G, (uint64_t)g.K * 2, (uint64_t)g.N * g.K * 2, (uint32_t)bn, 1);
    if (!ok) return cudaErrorInvalidValue;

    int grid = num_sms;
    if (!var) {
        const long long tiles = (long long)g.G * ((g.M + BM - 1) / BM) * ((g.N + bn - 1) / bn);
        if (tiles == 0) return cudaSuccess;
        if (tiles < grid) grid = (int)tiles;
    }
    switch (bn) {
        case 256: return launch_bn<256>(g.epi, ma, mb, kp, grid, s);
        case 192: return launch_bn<192>(g.epi, ma, mb, kp, grid, s);
        case 160: return launch_bn<160>(g.epi, ma, mb, kp, grid, s);
        default: return launch_bn<128>(g.epi, ma, mb, kp, grid, s);
    }
}

}  // namespace rm
