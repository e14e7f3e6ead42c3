// Internal interface between the C ABI (rm_api.cu) and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/rankmixer.h"

namespace rm {

// Device error word and site id (both in device memory, owned by a handle).
struct DeviceErr {
    int* word;
    int* site;
};

// Wait-site ids recorded with RM_ERR_DEVICE_TIMEOUT.
enum WaitSite : int {
    SITE_TC_PRODUCER = 1,
    SITE_TC_MMA_FULL = 2,
    SITE_TC_MMA_TMEM = 3,
    SITE_TC_EPILOGUE = 4,
    SITE_TC_DRAIN = 5,
    SITE_MIX_LN = 6,
    SITE_LN_POOL = 7,
    SITE_TRAIN_MIX = 8,
    SITE_SELFTEST = 9,
};

// ---- memory-bound kernels (rm_mem.cu); E = 0 float, 1 bf16 -------------
cudaError_t launch_token_mix(int dtype, const void* X, void* Y, int B, int T, int D, cudaStream_t s);
cudaError_t launch_layernorm(int dtype, const void* A, const void* R, const float* g, const float* b,
                             void* out, long long rows, int D, float eps, cudaStream_t s);
// ---- rm_mix.cu ------------------------------------------------------------
// LayerNorm statistics of rows (row = b*T + t) in partial form: part[row*P + p]
// = (mean, M2) over the D/P columns of slice p, as written by the producer.
struct RowStats {
    float2* part;
    int P;
};
// S = LN1(TokenMixing(Xh) + Xh), Xh = pre_g ? LN_pre(X) : X (per token row,
// statistics from pre_stats); with addnorm == 0, S = TokenMixing(Xh).
// Training (addnorm only): xhat_out [B, T, D] receives the normalised rows
// (Z - mean) * rstd and rstd_out [B*T] the rows' 1/sqrt(var + eps).
cudaError_t launch_mix_ln(int dtype, const void* X, const float* pre_g, const float* pre_b, RowStats pre_stats,
                          const float* g1, const float* b1, void* S, int B, int T, int D, float eps, int addnorm,
                          int num_sms, DeviceErr err, uint64_t budget_ns, cudaStream_t s, void* xhat_out = nullptr,
                          float* rstd_out = nullptr);
// pooled[b] = mean_t LN(X[b, t]) (statistics given); Xout (optional) = LN(X).
cudaError_t launch_ln_pool(int dtype, const void* X, RowStats stats, const float* g, const float* b, float* pooled,
                           void* Xout, int B, int T, int D, float eps, int num_sms, DeviceErr err,
                           uint64_t budget_ns, cudaStream_t s);
// out[row] = (mean, M2) of each row over all D columns (P = 1).
cudaError_t launch_row_stats(int dtype, const void* X, float2* out, long long rows, int D, cudaStream_t s);
int mix_ln_max_d(int dtype);
bool mix_ln_sample_fits(int dtype, int T, int D);
struct PadSplitArgs {
    const void* src[32];
    int col0[33];   // first padded column of each group; col0[n] = sum of widths
    int n;
};
cudaError_t launch_padsplit(int dtype, const PadSplitArgs& a, void* X0, int B, int width,
                            cudaStream_t s);
cudaError_t launch_head(int dtype, const float* pooled, const void* w, const float* bias, float* prob,
                        int B, int D, cudaStream_t s);
cudaError_t launch_selftest_wait(DeviceErr err, uint64_t budget_ns, cudaStream_t s);

// ---- grouped GEMMs ------------------------------------------------------
// out[g, m, n] = epi( sum_k A[g, m, k] * W[g, n, k] )  (W stored [G][N][K]).
enum Epilogue : int {
    EPI_GELU_TANH = 0,   // bf16( GELU_tanh(acc + bias) )
    EPI_GELU_ERF = 1,    // bf16( GELU_erf(acc + bias) )
    EPI_BIAS_RESID = 2,  // bf16( acc [+ bias] [+ resid] )
    EPI_BIAS_GATE = 3,   // bf16( gate[row] * (acc + bias) )
    EPI_RELU = 4,        // bf16( max(acc + bias, 0) )
    // backward products (dense only): resid holds the activation's input U
    EPI_DACT_TANH = 5,   // bf16( acc * GELU_tanh'(U) )
    EPI_DACT_ERF = 6,    // bf16( acc * GELU_erf'(U) )
    EPI_DACT_RELU = 7,   // bf16( acc * [U > 0] )
    EPI_F32 = 8,         // float( acc )   (out is float)
    // e4m3 operands (kind::f8f6f4; dense, K-major): acc is first dequantised,
    // acc * ascale[row] * wscale[g][n], then as the bf16 epilogue named
    EPI_F8_GELU_TANH = 9,
    EPI_F8_GELU_ERF = 10,
    EPI_F8_RELU = 11,
    EPI_F8_BIAS_RESID = 12,
};
inline int f8_epi_for_act(int act) {
    return act == RM_ACT_GELU_ERF ? EPI_F8_GELU_ERF : act == RM_ACT_RELU ? EPI_F8_RELU : EPI_F8_GELU_TANH;
}
inline int epi_for_act(int act) { return act == RM_ACT_GELU_ERF ? EPI_GELU_ERF : act == RM_ACT_RELU ? EPI_RELU : EPI_GELU_TANH; }
inline int dact_epi_for_act(int act) {
    return act == RM_ACT_GELU_ERF ? EPI_DACT_ERF : act == RM_ACT_RELU ? EPI_DACT_RELU : EPI_DACT_TANH;
}

struct GroupedGemm {
    int G, M, N, K;
    // A operand: element (g, m, k) at A + g*a_gstride + m*a_ld + k (elements),
    // or, with a_mn (M-major A, dense only), at A + g*a_gstride + k*a_ld + m.
    const void* A;
    long long a_gstride, a_ld;
    long long a_rows_total;   // variable-row mode: rows allocated in A (and out)
    bool a_mn;
    // W operand: [G][N][K] contiguous when w_ld == 0; else element (g, n, k)
    // at W + g*w_gstride + n*w_ld + k, or, with w_mn (N-major, dense only),
    // at W + g*w_gstride + k*w_ld + n.
    const void* W;
    long long w_gstride, w_ld;
    bool w_mn;
    // W was written by an earlier kernel on the stream (activations in a
    // weight-gradient product): its tiles are loaded only after the
    // programmatic-launch wait.  False for model weights.
    bool w_from_kernel;
    // out element (g, m, n) at out + g*o_gstride + m*o_ld + n (bf16; float
    // for EPI_F32).
    void* out;
    long long o_gstride, o_ld;
    const float* bias;        // [G][N]; may be null for EPI_BIAS_RESID; unused by EPI_DACT_* / EPI_F32
    // bf16, same indexing as out, strides below: EPI_BIAS_RESID the residual
    // (may be null); EPI_DACT_* the activation input U; activation epilogues
    // (dense, may be null): receives bf16(acc + bias), the activation input.
    const void* resid;
    long long r_gstride, r_ld;
    const float* gate;        // EPI_BIAS_GATE: [rows] in variable-row mode
    int epi;
    // Optional LayerNorm partial statistics of the stored (rounded) output rows,
    // EPI_BIAS_RESID dense only, N % 64 == 0: (mean, M2) of columns
    // [64c, 64c + 64) of row (g, m) at stats + g*s_gstride + m*s_ld + c.
    float2* stats;
    long long s_gstride, s_ld;
    // Variable-row mode (sparse MoE): group g owns rows [grp_off[g], grp_off[g] + grp_cnt[g])
    // of A and out (g strides unused); mtile_prefix[g] = sum_{g' < g} ceil(cnt / (128 var_cg)).
    // var_cg = 2: CTA pairs with 256-row tiles (each CTA 128 rows); else 1.
    int var_cg;
    const int* grp_cnt;
    const int* grp_off;
    const int* mtile_prefix;  // [G + 1]
    // Variable-K mode (the sparse-MoE experts' weight gradients, a_mn and w_mn,
    // EPI_F32): dense G x M x N output tiles; group g's K runs over rows
    // [grp_off[g], grp_off[g] + vark_cnt[g]) of the compacted A [rows][M] and
    // W [rows][N] (a_ld, w_ld their row strides; vark_cnt a multiple of 64,
    // at least 64, the padding rows zero).  grp_cnt must be null.
    bool vark;
    const int* vark_cnt;
    // e4m3 operands (EPI_F8_*): A and W hold one byte per element; row (g, m)
    // of A has scale ascale[g*as_gstride + m*as_ld], row (g, n) of W wscale[g*N + n].
    const float* ascale;
    long long as_gstride, as_ld;
    const float* wscale;
    // Optional split-K workspace for the dense tcgen05 path (both null: no
    // split).  sk_ws holds gemm_tc_split_ws_bytes(num_sms) bytes; sk_cnt holds
    // gemm_tc_split_cnt_ints(num_sms) ints, zero before the first use (the
    // kernel leaves them zero when it completes).
    float* sk_ws;
    int* sk_cnt;
};

size_t gemm_tc_split_ws_bytes(int num_sms);
size_t gemm_tc_split_cnt_ints(int num_sms);

cudaError_t launch_gemm_tc(const GroupedGemm& p, DeviceErr err, uint64_t budget_ns, int num_sms,
                           cudaStream_t s);
cudaError_t launch_gemm_simt(const GroupedGemm& p, cudaStream_t s);   // fp32, CUDA cores

// ---- sparse MoE routing (rm_moe.cu) ----------------------------------------
struct MoeWork {
    float* gates;          // [B, T, Ne]
    int* counts;           // [T*Ne]
    int* offsets;          // [T*Ne]
    int* mtile_prefix;     // [T*Ne + 1]: prefix of ceil(count / tile rows) over the experts
    int* totals;           // [2]: active entries, m-tiles
    int* slot_row;         // [B*T*Ne]: slot -> row b*T + t of S
    float* slot_gate;      // [B*T*Ne]
    int* slot_of;          // [B, T, Ne]: slot or -1
    void* Sg;              // [B*T*Ne, D] bf16 gathered rows
    void* Hg;              // [B*T*Ne, hidden] bf16
    void* Eg;              // [B*T*Ne, D] bf16 gate-scaled expert outputs
    // training: every expert's slot list padded to a multiple of 64, at least
    // 64 (padded counts here; rows -1 and gates 0 in the padding); null: none
    int* cnt_pad = nullptr;    // [T*Ne]
};
cudaError_t launch_moe_route(const void* S, const float* Wr, const float* br, const MoeWork& w, int B,
                             int T, int D, int Ne, cudaStream_t s, int tile_rows = 128);
// out[r] = resid[r] + sum_j Eg[slot_of[r, j]]; stats (may be null) = (mean, M2)
// of each stored row (P = 1).
cudaError_t launch_moe_gather(const void* S, const MoeWork& w, int B, int T, int D, int Ne,
                              cudaStream_t s);
cudaError_t launch_moe_combine(const MoeWork& w, const void* resid, void* out, float2* stats, int B, int T, int D,
                               int Ne, cudaStream_t s);
// Training (sparse-MoE backward).  Gates of a router alone (no compaction);
// counts_scratch [T*Ne] ints.
cudaError_t launch_moe_route_only(const void* S, const float* Wr, const float* br, float* gates, int* counts_scratch,
                                  int B, int T, int D, int Ne, cudaStream_t s);
// dEg[slot] = G dV[row], dR[r, j] = dV . e_j [active] (+ lambda unless gates_inf),
// dRinf[r, j] = lambda [gates_inf > 0] (gates_inf / dRinf may be null); the
// padding slots' rows of dEg are zeroed.
cudaError_t launch_moe_bwd_gate(const void* dV, const MoeWork& w, const float* gates_inf, float lambda, void* dEg,
                                float* dR, float* dRinf, int B, int T, int D, int Ne, cudaStream_t s);
// dS[r] = dZ[r] + sum_j dSg[slot(r, j)] + sum_j dR[r, j] Wr[t, j] + sum_j dRinf[r, j] Wrinf[t, j].
cudaError_t launch_moe_bwd_combine(const void* dZ, const void* dSg, const MoeWork& w, const float* dR, const float* Wr,
                                   const float* dRinf, const float* Wrinf, void* dS, int B, int T, int D, int Ne,
                                   cudaStream_t s);
// Router weight-gradient partials over blocks of RB samples (see rm_moe.cu).
cudaError_t launch_router_grad(const void* S, const float* dR, float* part, float* part_b, int B, int T, int D, int Ne,
                               int RB, cudaStream_t s);
// loss[0] += lambda * sum of x[0 .. n), in a fixed order; part: 256 floats of scratch.
cudaError_t launch_add_scaled_sum(const float* x, long long n, float lambda, float* loss, float* part,
                                  cudaStream_t s);

// e4m3 rows (rm_fp8.cu): dst[r][k] = e4m3(src[r][k] / scale[r]), scale[r] =
// absmax of row r / 448 (1 for a zero row); src bf16 [rows][K], K % 16 == 0.
cudaError_t launch_quant_rows(const void* src, void* dst, float* scale, long long rows, int K, cudaStream_t s);

// Token-sharded forward (rm_shard.cu): G ranks of Tl = T / G tokens each.
cudaError_t launch_shard_pack(const void* Za, const void* Zb, const float* g, const float* bt, float eps, void* Xh,
                              void* send, int B, int Tl, int D, int G, cudaStream_t s);
cudaError_t launch_shard_mix_ln(const void* recv, const void* Xh, const float* g, const float* bt, float eps, void* S,
                                int B, int Tl, int D, int G, cudaStream_t s);
cudaError_t launch_shard_pool(const void* V, const void* Sres, const float* g, const float* bt, float eps,
                              float* pooled_part, int B, int Tl, int D, cudaStream_t s);

}  // namespace rm
