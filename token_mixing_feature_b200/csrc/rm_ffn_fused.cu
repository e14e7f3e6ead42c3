// Fused per-token FFN for narrow tokens on the 5th-generation tensor cores
// (tcgen05) of sm_100a: both projections in one kernel, the hidden
// activation kept on chip.
//
// RankMixer's Per-Token FFN (fun-rec chapter "Rankmixer: 硬件效率优化",
// section Per-Token FFN) gives token t its own two-layer FFN:
//     V[m, t, :] = GELU(S[m, t, :] W1_t^T + b1_t) W2_t^T + b2_t  (+ S[m, t, :])
// with W1 stored [T][kD][D] and W2 [T][D][kD].  The two-GEMM path writes
// the hidden [T, B, kD] to HBM and reads it back.  When D <= 320 the output
// block of a 256-row tile fits in tensor memory next to one hidden chunk and
// its accumulator, so this kernel walks the hidden dimension in chunks of 128
// columns instead:
//     acc1  = S_tile W1_t[chunk]^T                   (tcgen05, tensor memory)
//     Hc    = bf16(act(acc1 + b1_t[chunk]))          (epilogue warps -> tensor memory)
//     acc2 += Hc W2_t[:, chunk]^T                    (tcgen05, A operand in tensor memory)
// and after the last chunk stores V = bf16(acc2 + b2_t (+ S)) with the
// LayerNorm partials (mean, M2) of every 64-column slice of each stored row:
// the same outputs, rounded the same way, as the two-GEMM path.
//
// Structure: persistent CTA pairs (cluster of 2) with 2-SM MMAs own 256-row
// tiles (128 rows per CTA); the tile's S rows stay in shared memory for all
// chunks.
//   warp 0      TMA: the S tile, then W1 chunks through ring 1
//   warp 1      MMA issuer: the first projection of chunk c + 1 is issued
//               before the second projection of chunk c, so the tensor pipe
//               works on one while the epilogue turns the other's
//               accumulator into the next hidden chunk
//   warps 2..9  epilogue: hidden chunks (tcgen05.ld -> bias + activation ->
//               bf16 pairs -> tcgen05.st), then the previous tile's output
//               rows once the next tile's first hidden chunk is written
//   warp 10     TMA: W2 chunks through ring 2
// Tensor memory (512 columns): acc2 in columns [0, D), the bf16 hidden chunk
// in [320, 384) (two values per column: the second projection's A operand),
// acc1 in [384, 512).  The S tile and the weights sit in shared memory; the
// hidden chunk never leaves tensor memory.
// Every mbarrier wait is bounded (rm_device.cuh); a wait that runs out
// records RM_ERR_DEVICE_TIMEOUT, stops the CTA's other roles, drains
// in-flight copies and MMAs, frees tensor memory and returns.
#include <cuda.h>
#include <cuda_bf16.h>

#include <cstdlib>

#include "rm_device.cuh"
#include "rm_tmap.h"

namespace rm {
namespace {

constexpr int BM = 128;          // rows per CTA
constexpr int BK = 64;           // bf16 per 128-byte swizzle row
constexpr int UMMA_K = 16;       // K per tcgen05.mma of kind::f16
constexpr int HC = 128;          // hidden columns per chunk
constexpr int kEpiWarps = 8;
constexpr int kThreads = (3 + kEpiWarps) * 32;
constexpr int kW2Warp = 2 + kEpiWarps;
constexpr int H_COL = 320;       // tensor-memory column of the bf16 hidden chunk (HC / 2 columns)
constexpr int ACC1_COL = 384;    // tensor-memory column of the hidden-chunk accumulator
constexpr int TMEM_COLS = 512;
constexpr int BLK_BYTES = BM * BK * 2;   // one swizzled [128 x 64] operand block

struct FParams {
    int G, M, hidden;
    int epi;                  // EPI_GELU_TANH, EPI_GELU_ERF or EPI_RELU
    const float* b1;          // [G][hidden]
    const float* b2;          // [G][D]
    __nv_bfloat16* out;
    long long o_gstride, o_ld;
    const __nv_bfloat16* resid;
    long long r_gstride, r_ld;
    float2* stats;
    long long s_gstride, s_ld;
    DeviceErr err;
    unsigned long long budget_ns;
};

// Shared-memory plan for width D.  The second projection's D output columns
// are one MMA (D <= 256) or two of D/2 (N <= 256, a multiple of 32 with A in
// tensor memory); for a 2-SM MMA each CTA holds half of the B rows of each,
// so a ring-2 stage is this CTA's halves of both, one K block deep.
template <int D>
struct FCfg {
    static constexpr int KB1 = D / BK;                        // K blocks of the first projection
    static constexpr int NSUB = D > 256 ? 2 : 1;
    static constexpr int NSUBN = D / NSUB;                    // N of one second-projection MMA
    static constexpr int A_BYTES = KB1 * BLK_BYTES;           // this CTA's 128 S rows
    static constexpr int W1_STAGE = (HC / 2) * BK * 2;        // this CTA's 64 W1 rows, one K block
    static constexpr int W2_SUB = (NSUBN / 2) * BK * 2;       // this CTA's W2 rows of one MMA, one K block
    static constexpr int W2_STAGE = NSUB * W2_SUB;
    static constexpr int R2 = 4;
    static constexpr int BAR_BYTES = 512;
    static constexpr int R1_RAW = (227 * 1024 - 1024 - BAR_BYTES - A_BYTES - R2 * W2_STAGE) / W1_STAGE;
    static constexpr int R1 = R1_RAW > 16 ? 16 : R1_RAW;
    static constexpr int NBARS = 2 * R1 + 2 * R2 + 9;
    static constexpr int SMEM_BYTES = 1024 + A_BYTES + R1 * W1_STAGE + R2 * W2_STAGE + BAR_BYTES;
    static_assert(D % 64 == 0 && D >= 64 && D <= H_COL, "D");
    static_assert(NSUBN % 32 == 0 && NSUBN <= 256 && (NSUBN / 2) % 8 == 0, "second-projection MMA width");
    static_assert(W2_SUB % 1024 == 0 && W1_STAGE % 1024 == 0, "swizzle atoms stay 1024-byte aligned");
    static_assert(R1 >= 4, "ring 1 depth");
    static_assert(8 * NBARS + 8 <= BAR_BYTES, "barrier area");
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    ffn_fused_kernel(const __grid_constant__ CUtensorMap tmS, const __grid_constant__ CUtensorMap tmW1,
                     const __grid_constant__ CUtensorMap tmW2, const __grid_constant__ FParams p) {
    using C = FCfg<D>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    unsigned char* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
    const uint32_t sA = smem_u32(smem);
    const uint32_t sW1 = sA + C::A_BYTES;
    const uint32_t sW2 = sW1 + C::R1 * C::W1_STAGE;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::A_BYTES + C::R1 * C::W1_STAGE + C::R2 * C::W2_STAGE);
    const uint32_t full1 = smem_u32(bars);
    const uint32_t empty1 = full1 + 8 * C::R1;
    const uint32_t full2 = empty1 + 8 * C::R1;
    const uint32_t empty2 = full2 + 8 * C::R2;
    const uint32_t fullA = empty2 + 8 * C::R2;    // S tile landed (pair's bytes, on the even CTA)
    const uint32_t emptyA = fullA + 8;            // S tile no longer read (both CTAs)
    const uint32_t acc1_full = emptyA + 8;        // hidden-chunk accumulator ready (both CTAs)
    const uint32_t acc1_empty = acc1_full + 8;    // ... read by every epilogue warp of the pair (even CTA)
    const uint32_t h_full = acc1_empty + 8;       // hidden chunk stored in tensor memory (even CTA)
    const uint32_t h_empty = h_full + 8;          // ... consumed by the second projection (both CTAs)
    const uint32_t acc2_full = h_empty + 8;       // tile's output accumulator complete (both CTAs)
    const uint32_t acc2_empty = acc2_full + 8;    // ... read by every epilogue warp of the pair (even CTA)
    const uint32_t drain_bar = acc2_empty + 8;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBARS);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    constexpr uint32_t kPairEpiWarps = 2 * kEpiWarps;   // one arrival per epilogue warp of the pair
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::R1; ++s) {
            mbar_init(full1 + 8 * s, 1);
            mbar_init(empty1 + 8 * s, 1);
        }
        for (int s = 0; s < C::R2; ++s) {
            mbar_init(full2 + 8 * s, 1);
            mbar_init(empty2 + 8 * s, 1);
        }
        mbar_init(fullA, 1);
        mbar_init(emptyA, 1);
        mbar_init(acc1_full, 1);
        mbar_init(acc1_empty, kPairEpiWarps);
        mbar_init(h_full, kPairEpiWarps);
        mbar_init(h_empty, 1);
        mbar_init(acc2_full, 1);
        mbar_init(acc2_empty, kPairEpiWarps);
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmS);
        prefetch_tmap(&tmW1);
        prefetch_tmap(&tmW2);
    }
    if (warp == 0) {
        tmem_alloc_pair(smem_u32(tmem_slot), TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();   // the peer's barriers exist before anyone signals them
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // The set-up above overlaps the previous kernel's tail (programmatic
    // launch); only weight copies are issued before waiting for it.
    pdl_trigger();

    const WaitCtx wc{abort_flag, p.budget_ns, p.err};
    const int mblk = (p.M + 2 * BM - 1) / (2 * BM);
    const long long tiles = (long long)p.G * mblk;
    const int NC = p.hidden / HC;
    const long long unit = blockIdx.x >> 1, nunits = gridDim.x >> 1;

    if (warp == 0 || warp == kW2Warp) {
        if (lane == 0) {
            // ------------------------------------------ TMA producers
            // warp 0: S tiles + ring 1 (W1 chunks, KB1 K blocks each);
            // warp 10: ring 2 (W2 chunks, HC / BK K blocks each).  Each ring
            // is filled in the order the MMA issuer consumes it.
            const bool w1 = warp == 0;
            const int R = w1 ? C::R1 : C::R2;
            const uint32_t full0 = w1 ? full1 : full2;
            const uint32_t empty0 = w1 ? empty1 : empty2;
            const int stage_bytes = w1 ? C::W1_STAGE : C::W2_STAGE;
            const int per_chunk = w1 ? C::KB1 : HC / BK;
            const int per_tile = NC * per_chunk;
            auto load_w = [&](int q, int g, int stage) {   // K block q of the tile's weight stream
                const uint32_t fb = full0 + 8 * stage;
                if (leader) mbar_arrive_expect_tx(fb, 2 * stage_bytes);
                const uint32_t fbl = mapa_shared(fb, 0);   // the pair counts bytes on the even CTA
                const int c = q / per_chunk, kb = q - c * per_chunk;
                const uint32_t dst = (w1 ? sW1 : sW2) + stage * stage_bytes;
                if (w1) {
                    tma_load_3d_pair(dst, &tmW1, fbl, kb * BK, c * HC + (int)rank * (HC / 2), g);
                } else {
#pragma unroll
                    for (int sub = 0; sub < C::NSUB; ++sub)
                        tma_load_3d_pair(dst + sub * C::W2_SUB, &tmW2, fbl, c * HC + kb * BK,
                                         sub * C::NSUBN + (int)rank * (C::NSUBN / 2), g);
                }
            };
            int stage = 0;
            uint32_t phase = 0, issued = 0, issued_phase = 0;
            int a_loads = 0;
            bool ok = true;
            int npre = 0;
            if (unit < tiles) {   // fresh ring: the first stages are free
                npre = min(R, per_tile);
                for (int q = 0; q < npre; ++q) {
                    load_w(q, (int)(unit / mblk), q);
                    issued |= 1u << q;
                }
            }
            pdl_wait();
            int j = 0;
            for (long long idx = unit; idx < tiles && ok; idx += nunits, ++j) {
                const int g = (int)(idx / mblk);
                if (w1) {
                    const int m0 = (int)(idx - (long long)g * mblk) * (2 * BM) + (int)rank * BM;
                    if (!mbar_wait(emptyA, ((uint32_t)j & 1u) ^ 1u, wc, SITE_TC_PRODUCER)) break;
                    if (leader) mbar_arrive_expect_tx(fullA, 2 * C::A_BYTES);
                    const uint32_t fal = mapa_shared(fullA, 0);
                    for (int kb = 0; kb < C::KB1; ++kb) tma_load_3d_pair(sA + kb * BLK_BYTES, &tmS, fal, kb * BK, g, m0);
                    ++a_loads;
                }
                for (int q = 0; q < per_tile; ++q) {
                    if (!(j == 0 && q < npre)) {
                        if (!mbar_wait(empty0 + 8 * stage, phase ^ 1u, wc, SITE_TC_PRODUCER)) {
                            ok = false;
                            break;
                        }
                        load_w(q, g, stage);
                    }
                    issued |= 1u << stage;
                    issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == R) { stage = 0; phase ^= 1u; }
                }
            }
            // Every issued copy must land before the CTA's shared memory goes
            // away (for a pair, the even CTA's barrier counts both CTAs' bytes).
            if (leader) {
                for (int s = 0; s < R; ++s)
                    if (issued & (1u << s))
                        mbar_wait(full0 + 8 * s, (issued_phase >> s) & 1u, wc, SITE_TC_DRAIN, false);
                if (a_loads > 0) mbar_wait(fullA, (uint32_t)(a_loads - 1) & 1u, wc, SITE_TC_DRAIN, false);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        pdl_wait();   // (reads no global memory; keeps every thread ordered after the previous kernel)
        if (lane == 0 && leader) {
            // ------------------------------------------------ MMA issuer
            constexpr uint32_t idesc1 = idesc_bf16_f32(2 * BM, HC);
            constexpr uint32_t idesc2 = idesc_bf16_f32(2 * BM, C::NSUBN);
            const uint32_t t_acc1 = tmem_base + ACC1_COL;
            const uint32_t t_acc2 = tmem_base;
            const uint32_t t_h = tmem_base + H_COL;
            int s1 = 0, s2 = 0;
            uint32_t ph1 = 0, ph2 = 0;
            bool ok = true, any = false;
            // second projection of hidden chunk c2 (k2-th chunk of this pair, tile ordinal j2)
            auto second = [&](int c2, int j2, long long k2) -> bool {
                if (c2 == 0 && !mbar_wait(acc2_empty, ((uint32_t)j2 & 1u) ^ 1u, wc, SITE_TC_MMA_TMEM)) return false;
                if (!mbar_wait(h_full, (uint32_t)k2 & 1u, wc, SITE_TC_MMA_FULL)) return false;
                tc_fence_after();
                for (int kb = 0; kb < HC / BK; ++kb) {
                    if (!mbar_wait(full2 + 8 * s2, ph2, wc, SITE_TC_MMA_FULL)) return false;
                    tc_fence_after();
                    const uint32_t sb = sW2 + s2 * C::W2_STAGE;
#pragma unroll
                    for (int k = 0; k < BK / UMMA_K; ++k) {
                        const uint32_t accum = (c2 != 0 || kb != 0 || k != 0) ? 1u : 0u;
                        // hidden columns [64 kb + 16 k, + 16): 8 packed tensor-memory columns
                        const uint32_t a_tmem = t_h + (uint32_t)(32 * kb + 8 * k);
#pragma unroll
                        for (int sub = 0; sub < C::NSUB; ++sub)
                            tc_mma_f16_pair_ts(t_acc2 + (uint32_t)(sub * C::NSUBN), a_tmem,
                                               smem_desc_k_sw128(sb + sub * C::W2_SUB) + (uint64_t)(2 * k), idesc2, accum);
                    }
                    tc_commit_pair_mc(empty2 + 8 * s2, 0x3);
                    if (++s2 == C::R2) { s2 = 0; ph2 ^= 1u; }
                }
                tc_commit_pair_mc(h_empty, 0x3);
                if (c2 == NC - 1) tc_commit_pair_mc(acc2_full, 0x3);
                return true;
            };
            long long k = 0;    // hidden chunks started by this pair
            int j = 0;
            int pend_c = -1, pend_j = 0;
            long long pend_k = 0;
            for (long long idx = unit; idx < tiles && ok; idx += nunits, ++j) {
                if (!mbar_wait(fullA, (uint32_t)j & 1u, wc, SITE_TC_MMA_FULL)) break;
                for (int c = 0; c < NC; ++c, ++k) {
                    // first projection of chunk c into acc1
                    if (!mbar_wait(acc1_empty, ((uint32_t)k & 1u) ^ 1u, wc, SITE_TC_MMA_TMEM)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    for (int kb = 0; kb < C::KB1; ++kb) {
                        if (!mbar_wait(full1 + 8 * s1, ph1, wc, SITE_TC_MMA_FULL)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint64_t adesc = smem_desc_k_sw128(sA + kb * BLK_BYTES);
                        const uint64_t bdesc = smem_desc_k_sw128(sW1 + s1 * C::W1_STAGE);
#pragma unroll
                        for (int kk = 0; kk < BK / UMMA_K; ++kk)
                            tc_mma_f16_pair(t_acc1, adesc + (uint64_t)(2 * kk), bdesc + (uint64_t)(2 * kk), idesc1,
                                            (kb != 0 || kk != 0) ? 1u : 0u);
                        tc_commit_pair_mc(empty1 + 8 * s1, 0x3);
                        any = true;
                        if (++s1 == C::R1) { s1 = 0; ph1 ^= 1u; }
                    }
                    if (!ok) break;
                    tc_commit_pair_mc(acc1_full, 0x3);
                    if (c == NC - 1) tc_commit_pair_mc(emptyA, 0x3);
                    // then the second projection of the previous chunk
                    if (pend_c >= 0 && !second(pend_c, pend_j, pend_k)) {
                        ok = false;
                        break;
                    }
                    pend_c = c;
                    pend_j = j;
                    pend_k = k;
                }
            }
            if (ok && pend_c >= 0) second(pend_c, pend_j, pend_k);
            // Every issued MMA must complete before tensor memory is released.
            if (any) {
                tc_commit_pair(drain_bar);
                mbar_wait(drain_bar, 0, wc, SITE_TC_DRAIN, false);
            }
        }
        __syncwarp();
    } else {
        pdl_wait();
        // --------------------------------------------------------- epilogue
        // Warp w reads TMEM lanes 32 (w % 4) .. + 31 (this CTA's rows) and
        // half (w - 2) / 4 of the columns: hidden columns [64 half, 64 half
        // + 64) of each chunk (stored as tensor-memory columns H_COL + 32 half
        // .. + 31), and output slices of 64 columns alternating between the
        // halves.
        const int ew = warp - 2;
        const int quarter = warp & 3;
        const int half = ew >> 2;
        const int rl = quarter * 32 + lane;
        const uint32_t lane_tmem = tmem_base + ((uint32_t)(quarter * 32) << 16);
        // Waits give one answer per warp (the signals below converge the warp).
        auto warp_wait = [&](uint32_t bar, uint32_t parity) -> bool {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, wc, SITE_TC_EPILOGUE));
        };
        // One arrival per warp: each lane's tcgen05 loads or stores are
        // complete and fenced, then the warp converges and lane 0 signals the
        // pair's even CTA (from the odd CTA without release semantics: the
        // arrival publishes no memory writes).
        auto arrive_even = [&](uint32_t bar) {
            __syncwarp();
            if (lane == 0) {
                if (leader) mbar_arrive(bar);
                else mbar_arrive_cluster_relaxed(mapa_shared(bar, 0));
            }
        };
        // hidden chunk c of group g (the k-th chunk of this pair)
        auto hidden_chunk = [&](int g, int c, long long k) -> bool {
            // the chunk's biases first (weights: no wait needed), then its accumulator
            const float4* b4 = reinterpret_cast<const float4*>(p.b1 + (long long)g * p.hidden + c * HC + 64 * half);
            float4 bias[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) bias[r] = __ldg(b4 + r);
            if (!warp_wait(acc1_full, (uint32_t)k & 1u)) return false;
            tc_fence_after();
            float v[64];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float w16[16];
                tmem_ld16(lane_tmem + (uint32_t)(ACC1_COL + 64 * half + 16 * q), w16);
#pragma unroll
                for (int e = 0; e < 16; ++e) v[16 * q + e] = w16[e];
            }
            tmem_ld_wait();
            tc_fence_before();
            arrive_even(acc1_empty);
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                const float4 bb = bias[r];
                const float2 lo = f2_add(make_float2(v[4 * r], v[4 * r + 1]), make_float2(bb.x, bb.y));
                const float2 hi = f2_add(make_float2(v[4 * r + 2], v[4 * r + 3]), make_float2(bb.z, bb.w));
                v[4 * r] = lo.x;
                v[4 * r + 1] = lo.y;
                v[4 * r + 2] = hi.x;
                v[4 * r + 3] = hi.y;
            }
            if (p.epi == EPI_RELU) {
#pragma unroll
                for (int e = 0; e < 64; ++e) v[e] = fmaxf(v[e], 0.0f);
            } else if (p.epi == EPI_GELU_ERF) {
#pragma unroll
                for (int e = 0; e < 64; ++e) v[e] = 0.5f * v[e] * (1.0f + erff(v[e] * 0.7071067811865476f));
            } else {
#pragma unroll
                for (int e = 0; e < 64; e += 2) {
                    const float2 y = gelu_tanh_pair(make_float2(v[e], v[e + 1]));
                    v[e] = y.x;
                    v[e + 1] = y.y;
                }
            }
            uint32_t w[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) w[e] = pack_bf16x2(v[2 * e], v[2 * e + 1]);
            // the previous chunk's second projection has read the operand
            if (!warp_wait(h_empty, ((uint32_t)k & 1u) ^ 1u)) return false;
            tmem_st32(lane_tmem + (uint32_t)(H_COL + 32 * half), w);
            tmem_st_wait();
            tc_fence_before();
            arrive_even(h_full);
            return true;
        };
        // output rows of tile jt (group g, this CTA's first row m0)
        auto output_tile = [&](int jt, int g, int m0) -> bool {
            if (!warp_wait(acc2_full, (uint32_t)jt & 1u)) return false;
            tc_fence_after();
            const int row = m0 + rl;
            const bool row_ok = row < p.M;
            const float* bias_g = p.b2 + (long long)g * D;
            bool released = false;
#pragma unroll 1
            for (int c = 64 * half; c < D; c += 128) {
                float v[64];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float w16[16];
                    tmem_ld16(lane_tmem + (uint32_t)(c + 16 * q), w16);
#pragma unroll
                    for (int e = 0; e < 16; ++e) v[16 * q + e] = w16[e];
                }
                tmem_ld_wait();
                if (c + 128 >= D) {   // this thread's last slice: the accumulator may be reused
                    tc_fence_before();
                    arrive_even(acc2_empty);
                    released = true;
                }
                if (!row_ok) continue;
                const float4* b4 = reinterpret_cast<const float4*>(bias_g + c);
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    const float4 bb = __ldg(b4 + r);
                    const float2 lo = f2_add(make_float2(v[4 * r], v[4 * r + 1]), make_float2(bb.x, bb.y));
                    const float2 hi = f2_add(make_float2(v[4 * r + 2], v[4 * r + 3]), make_float2(bb.z, bb.w));
                    v[4 * r] = lo.x;
                    v[4 * r + 1] = lo.y;
                    v[4 * r + 2] = hi.x;
                    v[4 * r + 3] = hi.y;
                }
                if (p.resid) {
                    const uint4* r4 =
                        reinterpret_cast<const uint4*>(p.resid + (long long)g * p.r_gstride + (long long)row * p.r_ld + c);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        float2 rp[4];
                        unpack_pairs(__ldcg(r4 + e), rp);
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float2 y = f2_add(make_float2(v[8 * e + 2 * i], v[8 * e + 2 * i + 1]), rp[i]);
                            v[8 * e + 2 * i] = y.x;
                            v[8 * e + 2 * i + 1] = y.y;
                        }
                    }
                }
                uint32_t w[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) w[e] = pack_bf16x2(v[2 * e], v[2 * e + 1]);
                if (p.stats) {
                    // LayerNorm partials of the stored (rounded) 64 values: (mean, M2)
                    float2 a1 = f2(0.f);
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        a1 = f2_add(a1, make_float2(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xffff0000u)));
                    const float mean = (a1.x + a1.y) * (1.0f / 64.0f);
                    const float2 nm = f2(-mean);
                    float2 a2 = f2(0.f);
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const float2 d =
                            f2_add(make_float2(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xffff0000u)), nm);
                        a2 = f2_fma(d, d, a2);
                    }
                    p.stats[(long long)g * p.s_gstride + (long long)row * p.s_ld + (c >> 6)] =
                        make_float2(mean, a2.x + a2.y);
                }
                uint4* dst = reinterpret_cast<uint4*>(p.out + (long long)g * p.o_gstride + (long long)row * p.o_ld + c);
#pragma unroll
                for (int e = 0; e < 8; ++e) dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
            }
            if (!released) {   // no output slice in this half (D = 64)
                tc_fence_before();
                arrive_even(acc2_empty);
            }
            return true;
        };
        long long k = 0;
        int j = 0, pg = 0, pm0 = 0;
        bool ok = true;
        for (long long idx = unit; idx < tiles && ok; idx += nunits, ++j) {
            const int g = (int)(idx / mblk);
            const int m0 = (int)(idx - (long long)g * mblk) * (2 * BM) + (int)rank * BM;
            for (int c = 0; c < NC; ++c, ++k) {
                if (!hidden_chunk(g, c, k)) {
                    ok = false;
                    break;
                }
                // the previous tile's rows, once this tile's first hidden chunk is on its way
                if (c == 0 && j > 0 && !output_tile(j - 1, pg, pm0)) {
                    ok = false;
                    break;
                }
            }
            pg = g;
            pm0 = m0;
        }
        if (ok && j > 0) output_tile(j - 1, pg, pm0);
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();   // the pair's MMAs and copies are done before either CTA leaves
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, TMEM_COLS);
    }
}

template <int D>
cudaError_t launch_d(const CUtensorMap& mS, const CUtensorMap& mW1, const CUtensorMap& mW2, const FParams& fp,
                     int grid, cudaStream_t s) {
    using C = FCfg<D>;
    auto k = ffn_fused_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, k, mS, mW1, mW2, fp);
}

}  // namespace

bool ffn_fused_supported(int D, int hidden) {
    return D % 64 == 0 && D >= 64 && D <= H_COL && hidden % HC == 0 && hidden >= HC;
}

// Opt-in (RM_FFN_FUSED=1).  Measured on B200 at the Pad-Split size (D 320,
// kD 1280, 16 tokens x 4096 samples) it takes 171 us per block against
// 78 + 74 us for the two grouped GEMMs: a chunk's first projection (20 MMAs
// of N = 128) runs at ~60 % of its nominal rate, and 256 tiles fill 3.46
// waves of the 74 CTA pairs.
bool ffn_fused_preferred(int G, int M, int D, int hidden, int num_sms) {
    (void)G;
    (void)M;
    (void)num_sms;
    if (!ffn_fused_supported(D, hidden)) return false;
    const char* e = getenv("RM_FFN_FUSED");
    return e && atoi(e) != 0;
}

cudaError_t launch_ffn_fused(const FusedFfn& f, DeviceErr err, uint64_t budget_ns, int num_sms, cudaStream_t s) {
    if (!ffn_fused_supported(f.D, f.hidden) || f.G < 1 || f.M < 0) return cudaErrorInvalidValue;
    if (f.epi != EPI_GELU_TANH && f.epi != EPI_GELU_ERF && f.epi != EPI_RELU) return cudaErrorInvalidValue;
    if (f.a_gstride > f.a_ld) return cudaErrorInvalidValue;   // S rows [M][G][D]: group inside the row stride
    const long long tiles = (long long)f.G * ((f.M + 2 * BM - 1) / (2 * BM));
    if (tiles == 0) return cudaSuccess;
    FParams fp{};
    fp.G = f.G;
    fp.M = f.M;
    fp.hidden = f.hidden;
    fp.epi = f.epi;
    fp.b1 = f.b1;
    fp.b2 = f.b2;
    fp.out = static_cast<__nv_bfloat16*>(f.out);
    fp.o_gstride = f.o_gstride;
    fp.o_ld = f.o_ld;
    fp.resid = static_cast<const __nv_bfloat16*>(f.resid);
    fp.r_gstride = f.r_gstride;
    fp.r_ld = f.r_ld;
    fp.stats = f.stats;
    fp.s_gstride = f.s_gstride;
    fp.s_ld = f.s_ld;
    fp.err = err;
    fp.budget_ns = budget_ns;
    const int nsub = f.D > 256 ? 2 : 1;
    CUtensorMap mS, mW1, mW2;
    bool ok = make_map(&mS, f.A, f.D, f.G, f.M, f.a_gstride * 2, f.a_ld * 2, 1, BM);
    ok = ok && make_map(&mW1, f.W1, f.D, f.hidden, f.G, (uint64_t)f.D * 2, (uint64_t)f.hidden * f.D * 2, HC / 2, 1);
    ok = ok && make_map(&mW2, f.W2, f.hidden, f.D, f.G, (uint64_t)f.hidden * 2, (uint64_t)f.D * f.hidden * 2,
                        (uint32_t)(f.D / nsub / 2), 1);
    if (!ok) return cudaErrorInvalidValue;
    long long units = num_sms / 2;
    if (tiles < units) units = tiles;
    const int grid = (int)(2 * units);
    switch (f.D) {
        case 64: return launch_d<64>(mS, mW1, mW2, fp, grid, s);
        case 128: return launch_d<128>(mS, mW1, mW2, fp, grid, s);
        case 192: return launch_d<192>(mS, mW1, mW2, fp, grid, s);
        case 256: return launch_d<256>(mS, mW1, mW2, fp, grid, s);
        default: return launch_d<320>(mS, mW1, mW2, fp, grid, s);
    }
}

}  // namespace rm
