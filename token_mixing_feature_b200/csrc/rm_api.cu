// C ABI of librankmixer (declared in include/rankmixer.h): handle and
// workspace management, host-side validation, and the launch sequences of the
// RankMixer block and stack forward passes.
//
// Block (fun-rec chapter "Rankmixer: 硬件效率优化", section RankMixer整体架构):
//     S  = LN1(TokenMixing(X) + X)
//     X' = LN2(F(S) + S),   F = per-token FFN or sparse-MoE FFN
// Stack launch sequence, all on one stream, no host synchronisation:
//     block l:  mix_ln(Y_{l-1} -> S; applies LN2 of block l-1 on load, and
//               LN1 of block l)  ->  FFN GEMM1 (bias + GELU) -> H
//               ->  FFN GEMM2 (bias + residual S) -> Y_l (pre-LN2)
//     end:      ln_pool(Y_{L-1}: LN2 of block L-1, mean over tokens) -> pooled
// so every block's second LayerNorm is applied where the next pass reads the
// row anyway, at no extra HBM traffic.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <new>

#include "rm_internal.h"

struct rm_handle {
    rm_config cfg;
    int device;
    int num_sms;
    size_t esz;
    unsigned char* ws;
    size_t ws_bytes;
    void* S;
    void* H;
    void* Y;
    void* X0buf;
    float* pooledbuf;
    // asynchronous host entry: second buffer set, copy streams and events
    // (created on first use), slot of the next call
    void* X0buf2;
    float* pooledbuf2;
    cudaStream_t h2d, d2h;
    cudaEvent_t ev_copied[2], ev_computed[2], ev_read[2];
    bool pipe_ready;
    int host_slot;
    float2* ystats;   // LayerNorm partials of the pre-LN block outputs Y [B_max*T][stat_P]
    int stat_P;
    float* sk_ws;     // split-K partial tiles of the dense tcgen05 GEMMs (null for fp32 / MoE)
    int* sk_cnt;      // their arrival counters (zero between launches)
    rm::MoeWork moe;
    // e4m3 stack (allocated on its first call): the quantised S and H and their
    // per-row scales
    void* f8ws;
    void* S8;
    void* H8;
    float* sS;
    float* sH;
    int* err;       // [0] error word, [1] site
    unsigned long long budget_ns;
    int last_site;
    // launch profiling (rm_profile_begin / rm_profile_end)
    cudaEvent_t* ev;      // 2 per recorded launch
    int* ev_kind;
    int ev_cap;
    int ev_n;
    bool prof;
};

namespace {

using rm::DeviceErr;

inline bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned16_or_null(const void* p) { return !p || (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

rm_status cuda_status(cudaError_t e) { return e == cudaSuccess ? RM_OK : RM_ERR_CUDA; }

DeviceErr derr(rm_handle* h) { return DeviceErr{h->err, h->err + 1}; }

// Brackets one kernel launch with a CUDA event pair on its stream while
// profiling is on (no effect otherwise).
struct ProfScope {
    rm_handle* h;
    cudaStream_t s;
    int idx;
    ProfScope(rm_handle* hh, int kind, cudaStream_t ss) : h(hh), s(ss), idx(-1) {
        if (h->prof && h->ev_n < h->ev_cap) {
            idx = h->ev_n++;
            h->ev_kind[idx] = kind;
            cudaEventRecord(h->ev[2 * idx], s);
        }
    }
    ~ProfScope() {
        if (idx >= 0) cudaEventRecord(h->ev[2 * idx + 1], s);
    }
};

void free_events(rm_handle* h) {
    if (h->ev) {
        for (int i = 0; i < 2 * h->ev_cap; ++i) cudaEventDestroy(h->ev[i]);
        free(h->ev);
        free(h->ev_kind);
    }
    h->ev = nullptr;
    h->ev_kind = nullptr;
    h->ev_cap = h->ev_n = 0;
    h->prof = false;
}

rm_status check_batch(const rm_handle* h, int B) {
    if (!h) return RM_ERR_INVALID_ARG;
    if (B < 1 || B > h->cfg.B_max) return RM_ERR_INVALID_ARG;
    return RM_OK;
}

rm_status check_block_weights(const rm_handle* h, const rm_block_weights* w, bool need_ln) {
    if (!w) return RM_ERR_INVALID_ARG;
    if (!aligned16(w->W1) || !aligned16(w->W2) || !aligned16(w->b1) || !aligned16(w->b2)) return RM_ERR_INVALID_ARG;
    if (need_ln && h->cfg.mix_addnorm && (!aligned16(w->ln1_g) || !aligned16(w->ln1_b))) return RM_ERR_INVALID_ARG;
    if (need_ln && (!aligned16(w->ln2_g) || !aligned16(w->ln2_b))) return RM_ERR_INVALID_ARG;
    if (h->cfg.n_experts > 0 && (!aligned16(w->Wr) || !aligned16(w->br))) return RM_ERR_INVALID_ARG;
    return RM_OK;
}

// V = F(S) (+ resid when resid != nullptr); F the dense per-token FFN.  With
// stats != nullptr the second projection's epilogue also writes the LayerNorm
// partials of V (h->stat_P slices per row); *stats_done tells whether it did.
rm_status run_pffn(rm_handle* h, const rm_block_weights* w, const void* S, void* V, const void* resid, int B,
                   cudaStream_t s, float2* stats = nullptr, bool* stats_done = nullptr) {
    const rm_config& c = h->cfg;
    rm::GroupedGemm g1{};
    g1.G = c.T;
    g1.M = B;
    g1.N = c.hidden;
    g1.K = c.D;
    g1.A = S;
    g1.a_gstride = c.D;
    g1.a_ld = (long long)c.T * c.D;
    g1.W = w->W1;
    g1.out = h->H;
    g1.o_gstride = (long long)B * c.hidden;
    g1.o_ld = c.hidden;
    g1.bias = static_cast<const float*>(w->b1);
    g1.epi = rm::epi_for_act(c.act);

    rm::GroupedGemm g2{};
    g2.G = c.T;
    g2.M = B;
    g2.N = c.D;
    g2.K = c.hidden;
    g2.A = h->H;
    g2.a_gstride = (long long)B * c.hidden;
    g2.a_ld = c.hidden;
    g2.W = w->W2;
    g2.out = V;
    g2.o_gstride = c.D;
    g2.o_ld = (long long)c.T * c.D;
    g2.bias = static_cast<const float*>(w->b2);
    g2.resid = resid;
    g2.r_gstride = c.D;
    g2.r_ld = (long long)c.T * c.D;
    g2.epi = rm::EPI_BIAS_RESID;
    g1.sk_ws = g2.sk_ws = h->sk_ws;
    g1.sk_cnt = g2.sk_cnt = h->sk_cnt;
    const bool gemm_stats = stats && c.dtype == RM_BF16 && c.D % 64 == 0;
    if (gemm_stats) {
        g2.stats = stats;
        g2.s_gstride = h->stat_P;
        g2.s_ld = (long long)c.T * h->stat_P;
    }
    if (stats_done) *stats_done = gemm_stats;

    cudaError_t e;
    {
        ProfScope ps(h, RM_K_GEMM1, s);
        e = c.dtype == RM_BF16 ? rm::launch_gemm_tc(g1, derr(h), h->budget_ns, h->num_sms, s)
                               : rm::launch_gemm_simt(g1, s);
    }
    if (e == cudaSuccess) {
        ProfScope ps(h, RM_K_GEMM2, s);
        e = c.dtype == RM_BF16 ? rm::launch_gemm_tc(g2, derr(h), h->budget_ns, h->num_sms, s)
                               : rm::launch_gemm_simt(g2, s);
    }
    return cuda_status(e);
}

// Expert tiles: single CTAs with 128-row tiles, or CTA pairs with 256-row
// tiles (tuning override RM_MOE_PAIR=1; the routing's tile prefix follows).
bool moe_pair_tiles() {
    static const bool on = [] {
        const char* e = getenv("RM_MOE_PAIR");
        return e && atoi(e) == 1;
    }();
    return on;
}

// V = sum_j ReLU-gate * expert(S) (+ resid); gates_out optional copy of G;
// stats (optional) receives the LayerNorm statistics of V (one slice per row).
rm_status run_moe(rm_handle* h, const rm_block_weights* w, const void* S, void* V, const void* resid,
                  float* gates_out, int B, cudaStream_t s, float2* stats = nullptr) {
    const rm_config& c = h->cfg;
    const int Ne = c.n_experts;
    const int G = c.T * Ne;
    const long long rows_total = (long long)c.B_max * c.T * Ne;
    cudaError_t e;
    {
        ProfScope ps(h, RM_K_MOE_ROUTE, s);
        e = rm::launch_moe_route(S, w->Wr, w->br, h->moe, B, c.T, c.D, Ne, s, moe_pair_tiles() ? 256 : 128);
    }
    if (e == cudaSuccess) {
        ProfScope ps(h, RM_K_MOE_GATHER, s);
        e = rm::launch_moe_gather(S, h->moe, B, c.T, c.D, Ne, s);
    }
    rm::GroupedGemm g1{};
    g1.G = G;
    g1.M = 0;
    g1.N = c.hidden;
    g1.K = c.D;
    g1.A = h->moe.Sg;
    g1.a_ld = c.D;
    g1.a_rows_total = rows_total;
    g1.W = w->W1;
    g1.out = h->moe.Hg;
    g1.o_ld = c.hidden;
    g1.bias = static_cast<const float*>(w->b1);
    g1.epi = rm::epi_for_act(c.act);
    g1.var_cg = moe_pair_tiles() ? 2 : 1;
    g1.grp_cnt = h->moe.counts;
    g1.grp_off = h->moe.offsets;
    g1.mtile_prefix = h->moe.mtile_prefix;
    rm::GroupedGemm g2 = g1;
    g2.N = c.D;
    g2.K = c.hidden;
    g2.A = h->moe.Hg;
    g2.a_ld = c.hidden;
    g2.W = w->W2;
    g2.out = h->moe.Eg;
    g2.o_ld = c.D;
    g2.bias = static_cast<const float*>(w->b2);
    g2.gate = h->moe.slot_gate;
    g2.epi = rm::EPI_BIAS_GATE;
    if (e == cudaSuccess) {
        ProfScope ps(h, RM_K_GEMM1, s);
        e = rm::launch_gemm_tc(g1, derr(h), h->budget_ns, h->num_sms, s);
    }
    if (e == cudaSuccess) {
        ProfScope ps(h, RM_K_GEMM2, s);
        e = rm::launch_gemm_tc(g2, derr(h), h->budget_ns, h->num_sms, s);
    }
    if (e == cudaSuccess) {
        ProfScope ps(h, RM_K_MOE_COMBINE, s);
        e = rm::launch_moe_combine(h->moe, resid, V, stats, B, c.T, c.D, Ne, s);
    }
    if (e == cudaSuccess && gates_out)
        e = cudaMemcpyAsync(gates_out, h->moe.gates, sizeof(float) * (size_t)B * c.T * Ne, cudaMemcpyDeviceToDevice, s);
    return cuda_status(e);
}

// V = F(S) + resid; with stats, also the LayerNorm statistics of V in
// h->stat_P slices per row (from the producing epilogue when it can, else by
// a row-statistics pass).
rm_status run_ffn(rm_handle* h, const rm_block_weights* w, const void* S, void* V, const void* resid, int B,
                  cudaStream_t s, float2* stats = nullptr) {
    if (h->cfg.n_experts > 0) return run_moe(h, w, S, V, resid, nullptr, B, s, stats);
    bool done = false;
    rm_status st = run_pffn(h, w, S, V, resid, B, s, stats, &done);
    if (st != RM_OK || !stats || done) return st;
    ProfScope ps(h, RM_K_LAYERNORM, s);
    return cuda_status(rm::launch_row_stats(h->cfg.dtype, V, stats, (long long)B * h->cfg.T, h->cfg.D, s));
}

rm_status run_stack(rm_handle* h, const rm_block_weights* blocks, const void* X0, float* pooled, void* Xlast,
                    int B, cudaStream_t s) {
    const rm_config& c = h->cfg;
    for (int l = 0; l < c.L; ++l) {
        const rm_block_weights* w = &blocks[l];
        const rm_block_weights* prev = l ? &blocks[l - 1] : nullptr;
        const rm::RowStats ys{h->ystats, h->stat_P};
        cudaError_t e;
        {
            ProfScope ps(h, RM_K_MIX_LN, s);
            e = rm::launch_mix_ln(c.dtype, l ? h->Y : X0, prev ? prev->ln2_g : nullptr,
                                  prev ? prev->ln2_b : nullptr, ys, w->ln1_g, w->ln1_b, h->S, B, c.T, c.D, c.ln_eps,
                                  c.mix_addnorm, h->num_sms, derr(h), h->budget_ns, s);
        }
        if (e != cudaSuccess) return RM_ERR_CUDA;
        rm_status st = run_ffn(h, w, h->S, h->Y, h->S, B, s, h->ystats);
        if (st != RM_OK) return st;
    }
    const rm_block_weights* last = &blocks[c.L - 1];
    ProfScope ps(h, RM_K_LN_POOL, s);
    return cuda_status(rm::launch_ln_pool(c.dtype, h->Y, rm::RowStats{h->ystats, h->stat_P}, last->ln2_g,
                                          last->ln2_b, pooled, Xlast, B, c.T, c.D, c.ln_eps, h->num_sms, derr(h),
                                          h->budget_ns, s));
}

template <typename T>
T* carve(unsigned char* base, size_t& off, size_t bytes) {
    T* p = reinterpret_cast<T*>(base + off);
    off += round_up(bytes, 256);
    return p;
}

}  // namespace

extern "C" {

const char* rm_status_string(rm_status s) {
    switch (s) {
        case RM_OK: return "ok";
        case RM_ERR_INVALID_ARG: return "invalid argument";
        case RM_ERR_UNSUPPORTED: return "unsupported shape or mode";
        case RM_ERR_CUDA: return "CUDA runtime error";
        case RM_ERR_OOM: return "device workspace allocation failed";
        case RM_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait ran out";
        case RM_ERR_DEVICE_BOUNDS: return "a device-side bounds check failed";
    }
    return "unknown status";
}

rm_status rm_create(const rm_config* cfg, rm_handle** out) {
    if (!out) return RM_ERR_INVALID_ARG;
    *out = nullptr;
    if (!cfg) return RM_ERR_INVALID_ARG;
    const rm_config c = *cfg;
    if (c.B_max < 1 || c.T < 1 || c.D < 1 || c.hidden < 1 || c.L < 1 || c.n_experts < 0) return RM_ERR_INVALID_ARG;
    if (c.dtype != RM_F32 && c.dtype != RM_BF16) return RM_ERR_INVALID_ARG;
    if (c.act != RM_ACT_GELU_TANH && c.act != RM_ACT_GELU_ERF && c.act != RM_ACT_RELU) return RM_ERR_INVALID_ARG;
    if (c.mix_addnorm != 0 && c.mix_addnorm != 1) return RM_ERR_INVALID_ARG;
    if (!(c.ln_eps > 0.f)) return RM_ERR_INVALID_ARG;
    if (c.T > 64 || c.n_experts > 32 || c.D % c.T) return RM_ERR_UNSUPPORTED;
    const size_t esz = c.dtype == RM_BF16 ? 2 : 4;
    if (c.dtype == RM_BF16 && (c.D % 16 || c.hidden % 16)) return RM_ERR_UNSUPPORTED;
    if (c.dtype == RM_F32 && (c.D % 4 || c.hidden % 4)) return RM_ERR_UNSUPPORTED;
    if (c.n_experts > 0 && c.dtype != RM_BF16) return RM_ERR_UNSUPPORTED;
    if ((size_t)c.n_experts * c.D * sizeof(float) > 160 * 1024) return RM_ERR_UNSUPPORTED;   // router staged in smem
    if (c.D > rm::mix_ln_max_d(c.dtype)) return RM_ERR_UNSUPPORTED;
    if (!rm::mix_ln_sample_fits(c.dtype, c.T, c.D)) return RM_ERR_UNSUPPORTED;   // a sample is staged in smem

    rm_handle* h = new (std::nothrow) rm_handle();
    if (!h) return RM_ERR_OOM;
    h->cfg = c;
    h->esz = esz;
    h->budget_ns = 1000000000ull;
    if (cudaGetDevice(&h->device) != cudaSuccess ||
        cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device) != cudaSuccess) {
        delete h;
        return RM_ERR_CUDA;
    }
    const size_t BTD = (size_t)c.B_max * c.T * c.D;
    const size_t slots = (size_t)c.B_max * c.T * (c.n_experts > 0 ? c.n_experts : 0);
    const size_t G = (size_t)c.T * c.n_experts;
    size_t off = 0;
    // First pass computes the size, second pass carves the allocation.
    for (int pass = 0; pass < 2; ++pass) {
        unsigned char* base = pass ? h->ws : nullptr;
        off = 0;
        h->err = carve<int>(base, off, 2 * sizeof(int));
        h->S = carve<unsigned char>(base, off, BTD * esz);
        h->Y = carve<unsigned char>(base, off, BTD * esz);
        h->X0buf = carve<unsigned char>(base, off, BTD * esz);
        h->pooledbuf = carve<float>(base, off, (size_t)c.B_max * c.D * sizeof(float));
        h->X0buf2 = carve<unsigned char>(base, off, BTD * esz);
        h->pooledbuf2 = carve<float>(base, off, (size_t)c.B_max * c.D * sizeof(float));
        h->stat_P = (c.dtype == RM_BF16 && c.n_experts == 0 && c.D % 64 == 0) ? c.D / 64 : 1;
        h->ystats = carve<float2>(base, off, (size_t)c.B_max * c.T * h->stat_P * sizeof(float2));
        h->H = c.n_experts == 0 ? carve<unsigned char>(base, off, (size_t)c.T * c.B_max * c.hidden * esz) : nullptr;
        const bool split = c.dtype == RM_BF16 && c.n_experts == 0;
        h->sk_cnt = split ? carve<int>(base, off, rm::gemm_tc_split_cnt_ints(h->num_sms) * sizeof(int)) : nullptr;
        h->sk_ws = split ? carve<float>(base, off, rm::gemm_tc_split_ws_bytes(h->num_sms)) : nullptr;
        if (c.n_experts > 0) {
            rm::MoeWork& m = h->moe;
            m.gates = carve<float>(base, off, slots * sizeof(float));
            m.counts = carve<int>(base, off, G * sizeof(int));
            m.offsets = carve<int>(base, off, G * sizeof(int));
            m.mtile_prefix = carve<int>(base, off, (G + 1) * sizeof(int));
            m.totals = carve<int>(base, off, 2 * sizeof(int));
            m.slot_row = carve<int>(base, off, slots * sizeof(int));
            m.slot_gate = carve<float>(base, off, slots * sizeof(float));
            m.slot_of = carve<int>(base, off, slots * sizeof(int));
            m.Sg = carve<unsigned char>(base, off, slots * c.D * esz);
            m.Hg = carve<unsigned char>(base, off, slots * c.hidden * esz);
            m.Eg = carve<unsigned char>(base, off, slots * c.D * esz);
        }
        if (pass == 0) {
            h->ws_bytes = off;
            if (cudaMalloc(reinterpret_cast<void**>(&h->ws), off) != cudaSuccess) {
                cudaGetLastError();
                delete h;
                return RM_ERR_OOM;
            }
        }
    }
    if (cudaMemset(h->err, 0, 2 * sizeof(int)) != cudaSuccess ||
        (h->sk_cnt && cudaMemset(h->sk_cnt, 0, rm::gemm_tc_split_cnt_ints(h->num_sms) * sizeof(int)) != cudaSuccess)) {
        cudaFree(h->ws);
        delete h;
        return RM_ERR_CUDA;
    }
    *out = h;
    return RM_OK;
}

rm_status rm_destroy(rm_handle* h) {
    if (!h) return RM_ERR_INVALID_ARG;
    int cur = 0;
    cudaGetDevice(&cur);
    cudaSetDevice(h->device);
    cudaDeviceSynchronize();
    free_events(h);
    if (h->pipe_ready) {
        cudaStreamDestroy(h->h2d);
        cudaStreamDestroy(h->d2h);
        for (int i = 0; i < 2; ++i) {
            cudaEventDestroy(h->ev_copied[i]);
            cudaEventDestroy(h->ev_computed[i]);
            cudaEventDestroy(h->ev_read[i]);
        }
    }
    cudaError_t e = cudaFree(h->ws);
    if (h->f8ws) cudaFree(h->f8ws);
    cudaSetDevice(cur);
    delete h;
    return cuda_status(e);
}

size_t rm_workspace_bytes(const rm_handle* h) { return h ? h->ws_bytes : 0; }

rm_status rm_token_mix(rm_handle* h, const void* X, void* Y, int B, rm_stream_t stream) {
    rm_status st = check_batch(h, B);
    if (st != RM_OK) return st;
    if (!aligned16(X) || !aligned16(Y) || X == Y) return RM_ERR_INVALID_ARG;
    ProfScope ps(h, RM_K_TOKEN_MIX, stream);
    return cuda_status(rm::launch_token_mix(h->cfg.dtype, X, Y, B, h->cfg.T, h->cfg.D, stream));
}

rm_status rm_layernorm(rm_handle* h, const void* A, const void* R, const float* gamma, const float* beta,
                       void* out, int rows, rm_stream_t stream) {
    if (!h || rows < 1 || (long long)rows > (long long)h->cfg.B_max * h->cfg.T) return RM_ERR_INVALID_ARG;
    if (!aligned16(A) || !aligned16_or_null(R) || !aligned16(gamma) || !aligned16(beta) || !aligned16(out))
        return RM_ERR_INVALID_ARG;
    ProfScope ps(h, RM_K_LAYERNORM, stream);
    return cuda_status(rm::launch_layernorm(h->cfg.dtype, A, R, gamma, beta, out, rows, h->cfg.D, h->cfg.ln_eps,
                                            stream));
}

rm_status rm_pffn_forward(rm_handle* h, const rm_block_weights* w, const void* S, void* V, int B,
                          rm_stream_t stream) {
    rm_status st = check_batch(h, B);
    if (st != RM_OK) return st;
    if (h->cfg.n_experts > 0) return RM_ERR_UNSUPPORTED;
    if ((st = check_block_weights(h, w, false)) != RM_OK) return st;
    if (!aligned16(S) || !aligned16(V)) return RM_ERR_INVALID_ARG;
    return run_pffn(h, w, S, V, nullptr, B, stream);
}

rm_status rm_moe_forward(rm_handle* h, const rm_block_weights* w, const void* S, void* V, float* gates, int B,
                         rm_stream_t stream) {
    rm_status st = check_batch(h, B);
    if (st != RM_OK) return st;
    if (h->cfg.n_experts == 0) return RM_ERR_UNSUPPORTED;
    if ((st = check_block_weights(h, w, false)) != RM_OK) return st;
    if (!aligned16(S) || !aligned16(V) || !aligned16_or_null(gates)) return RM_ERR_INVALID_ARG;
    return run_moe(h, w, S, V, nullptr, gates, B, stream);
}

rm_status rm_block_forward(rm_handle* h, const rm_block_weights* w, const void* X, void* Xout, int B,
                           rm_stream_t stream) {
    rm_status st = check_batch(h, B);
    if (st != RM_OK) return st;
    if ((st = check_block_weights(h, w, true)) != RM_OK) return st;
    if (!aligned16(X) || !aligned16(Xout)) return RM_ERR_INVALID_ARG;
    const rm_config& c = h->cfg;
    cudaError_t e;
    {
        ProfScope ps(h, RM_K_MIX_LN, stream);
        e = rm::launch_mix_ln(c.dtype, X, nullptr, nullptr, rm::RowStats{nullptr, 0}, w->ln1_g, w->ln1_b, h->S, B,
                              c.T, c.D, c.ln_eps, c.mix_addnorm, h->num_sms, derr(h), h->budget_ns, stream);
    }
    if (e != cudaSuccess) return RM_ERR_CUDA;
    if ((st = run_ffn(h, w, h->S, h->Y, h->S, B, stream)) != RM_OK) return st;
    ProfScope ps(h, RM_K_LAYERNORM, stream);
    return cuda_status(rm::launch_layernorm(c.dtype, h->Y, nullptr, w->ln2_g, w->ln2_b, Xout, (long long)B * c.T,
                                            c.D, c.ln_eps, stream));
}

rm_status rm_stack_forward(rm_handle* h, const rm_block_weights* blocks, const void* X0, float* pooled, void* Xlast,
                           int B, rm_stream_t stream) {
    rm_status st = check_batch(h, B);
    if (st != RM_OK) return st;
    if (!blocks || !aligned16(X0) || !aligned16(pooled) || !aligned16_or_null(Xlast)) return RM_ERR_INVALID_ARG;
    for (int l = 0; l < h->cfg.L; ++l)
        if ((st = check_block_weights(h, &blocks[l], true)) != RM_OK) return st;
    return run_stack(h, blocks, X0, pooled, Xlast, B, stream);
}

rm_status rm_quantize_fp8(const void* src, void* dst, float* scale, long long rows, int K, rm_stream_t stream) {
    if (!aligned16(src) || !aligned16(dst) || !scale || rows < 0 || K < 16 || K % 16) return RM_ERR_INVALID_ARG;
    if (K > 16384 || rows > 0x7fffffffLL) return RM_ERR_UNSUPPORTED;   // one CTA per row, <= 8 vectors a thread
    if (rows == 0) return RM_OK;
    return cuda_status(rm::launch_quant_rows(src, dst, scale, rows, K, stream));
}

rm_status rm_stack_forward_fp8(rm_handle* h, const rm_block_weights* blocks, const rm_fp8_weights* q, const void* X0,
                               float* pooled, int B, rm_stream_t stream) {
    rm_status st = check_batch(h, B);
    if (st != RM_OK) return st;
    const rm_config& c = h->cfg;
    if (c.dtype != RM_BF16 || c.n_experts != 0 || c.D % 64 || c.hidden % 16) return RM_ERR_UNSUPPORTED;
    if (!blocks || !q || !aligned16(X0) || !aligned16(pooled)) return RM_ERR_INVALID_ARG;
    for (int l = 0; l < c.L; ++l) {
        if ((st = check_block_weights(h, &blocks[l], true)) != RM_OK) return st;
        if (!aligned16(q[l].W1q) || !aligned16(q[l].W2q) || !aligned16(q[l].W1s) || !aligned16(q[l].W2s))
            return RM_ERR_INVALID_ARG;
    }
    const size_t rows = (size_t)c.B_max * c.T;
    if (!h->f8ws) {   // first call: the quantised activations and their scales
        const size_t s8 = round_up(rows * c.D, 256), h8 = round_up(rows * c.hidden, 256),
                     sc = round_up(rows * sizeof(float), 256);
        if (cudaMalloc(&h->f8ws, s8 + h8 + 2 * sc) != cudaSuccess) {
            cudaGetLastError();
            h->f8ws = nullptr;
            return RM_ERR_OOM;
        }
        unsigned char* b = static_cast<unsigned char*>(h->f8ws);
        h->S8 = b;
        h->H8 = b + s8;
        h->sS = reinterpret_cast<float*>(b + s8 + h8);
        h->sH = reinterpret_cast<float*>(b + s8 + h8 + sc);
    }
    cudaStream_t s = stream;
    for (int l = 0; l < c.L; ++l) {
        const rm_block_weights* w = &blocks[l];
        const rm_block_weights* prev = l ? &blocks[l - 1] : nullptr;
        cudaError_t e;
        {
            ProfScope ps(h, RM_K_MIX_LN, s);
            e = rm::launch_mix_ln(c.dtype, l ? h->Y : X0, prev ? prev->ln2_g : nullptr, prev ? prev->ln2_b : nullptr,
                                  rm::RowStats{h->ystats, h->stat_P}, w->ln1_g, w->ln1_b, h->S, B, c.T, c.D,
                                  c.ln_eps, c.mix_addnorm, h->num_sms, derr(h), h->budget_ns, s);
        }
        // S rows (b, t) and H rows (t, b), each with its own scale
        if (e == cudaSuccess) e = rm::launch_quant_rows(h->S, h->S8, h->sS, (long long)B * c.T, c.D, s);
        rm::GroupedGemm g1{};
        g1.G = c.T; g1.M = B; g1.N = c.hidden; g1.K = c.D;
        g1.A = h->S8; g1.a_gstride = c.D; g1.a_ld = (long long)c.T * c.D;
        g1.W = q[l].W1q;
        g1.out = h->H; g1.o_gstride = (long long)B * c.hidden; g1.o_ld = c.hidden;
        g1.bias = static_cast<const float*>(w->b1);
        g1.epi = rm::f8_epi_for_act(c.act);
        g1.ascale = h->sS; g1.as_gstride = 1; g1.as_ld = c.T;
        g1.wscale = q[l].W1s;
        g1.sk_ws = h->sk_ws; g1.sk_cnt = h->sk_cnt;
        if (e == cudaSuccess) {
            ProfScope ps(h, RM_K_GEMM1, s);
            e = rm::launch_gemm_tc(g1, derr(h), h->budget_ns, h->num_sms, s);
        }
        if (e == cudaSuccess) e = rm::launch_quant_rows(h->H, h->H8, h->sH, (long long)c.T * B, c.hidden, s);
        rm::GroupedGemm g2{};
        g2.G = c.T; g2.M = B; g2.N = c.D; g2.K = c.hidden;
        g2.A = h->H8; g2.a_gstride = (long long)B * c.hidden; g2.a_ld = c.hidden;
        g2.W = q[l].W2q;
        g2.out = h->Y; g2.o_gstride = c.D; g2.o_ld = (long long)c.T * c.D;
        g2.bias = static_cast<const float*>(w->b2);
        g2.resid = h->S; g2.r_gstride = c.D; g2.r_ld = (long long)c.T * c.D;
        g2.epi = rm::EPI_F8_BIAS_RESID;
        g2.stats = h->ystats; g2.s_gstride = h->stat_P; g2.s_ld = (long long)c.T * h->stat_P;
        g2.ascale = h->sH; g2.as_gstride = B; g2.as_ld = 1;
        g2.wscale = q[l].W2s;
        g2.sk_ws = h->sk_ws; g2.sk_cnt = h->sk_cnt;
        if (e == cudaSuccess) {
            ProfScope ps(h, RM_K_GEMM2, s);
            e = rm::launch_gemm_tc(g2, derr(h), h->budget_ns, h->num_sms, s);
        }
        if (e != cudaSuccess) return RM_ERR_CUDA;
    }
    const rm_block_weights* last = &blocks[c.L - 1];
    ProfScope ps(h, RM_K_LN_POOL, s);
    return cuda_status(rm::launch_ln_pool(c.dtype, h->Y, rm::RowStats{h->ystats, h->stat_P}, last->ln2_g,
                                          last->ln2_b, pooled, nullptr, B, c.T, c.D, c.ln_eps, h->num_sms, derr(h),
                                          h->budget_ns, s));
}

rm_status rm_stack_forward_host(rm_handle* h, const rm_block_weights* blocks, const void* X0_host,
                                float* pooled_host, int B, rm_stream_t stream) {
    rm_status st = check_batch(h, B);
    if (st != RM_OK) return st;
    if (!blocks || !X0_host || !pooled_host) return RM_ERR_INVALID_ARG;
    for (int l = 0; l < h->cfg.L; ++l)
        if ((st = check_block_weights(h, &blocks[l], true)) != RM_OK) return st;
    const size_t in_bytes = (size_t)B * h->cfg.T * h->cfg.D * h->esz;
    if (cudaMemcpyAsync(h->X0buf, X0_host, in_bytes, cudaMemcpyHostToDevice, stream) != cudaSuccess)
        return RM_ERR_CUDA;
    if ((st = run_stack(h, blocks, h->X0buf, h->pooledbuf, nullptr, B, stream)) != RM_OK) return st;
    if (cudaMemcpyAsync(pooled_host, h->pooledbuf, (size_t)B * h->cfg.D * sizeof(float), cudaMemcpyDeviceToHost,
                        stream) != cudaSuccess)
        return RM_ERR_CUDA;
    return cuda_status(cudaStreamSynchronize(stream));
}

rm_status rm_stack_forward_host_async(rm_handle* h, const rm_block_weights* blocks, const void* X0_host,
                                      float* pooled_host, int B, rm_stream_t stream) {
    rm_status st = check_batch(h, B);
    if (st != RM_OK) return st;
    if (!blocks || !X0_host || !pooled_host) return RM_ERR_INVALID_ARG;
    for (int l = 0; l < h->cfg.L; ++l)
        if ((st = check_block_weights(h, &blocks[l], true)) != RM_OK) return st;
    if (!h->pipe_ready) {
        int cur = 0;
        if (cudaGetDevice(&cur) != cudaSuccess || cur != h->device) return RM_ERR_INVALID_ARG;
        bool ok = cudaStreamCreateWithFlags(&h->h2d, cudaStreamNonBlocking) == cudaSuccess &&
                  cudaStreamCreateWithFlags(&h->d2h, cudaStreamNonBlocking) == cudaSuccess;
        for (int i = 0; i < 2 && ok; ++i)
            ok = cudaEventCreateWithFlags(&h->ev_copied[i], cudaEventDisableTiming) == cudaSuccess &&
                 cudaEventCreateWithFlags(&h->ev_computed[i], cudaEventDisableTiming) == cudaSuccess &&
                 cudaEventCreateWithFlags(&h->ev_read[i], cudaEventDisableTiming) == cudaSuccess;
        if (!ok) return RM_ERR_CUDA;
        h->pipe_ready = true;
    }
    const int s = h->host_slot;
    h->host_slot ^= 1;
    void* xb = s ? h->X0buf2 : h->X0buf;
    float* pb = s ? h->pooledbuf2 : h->pooledbuf;
    const size_t in_bytes = (size_t)B * h->cfg.T * h->cfg.D * h->esz;
    const size_t out_bytes = (size_t)B * h->cfg.D * sizeof(float);
    // input slot s is free once the stack that last read it has run
    if (cudaStreamWaitEvent(h->h2d, h->ev_computed[s], 0) != cudaSuccess ||
        cudaMemcpyAsync(xb, X0_host, in_bytes, cudaMemcpyHostToDevice, h->h2d) != cudaSuccess ||
        cudaEventRecord(h->ev_copied[s], h->h2d) != cudaSuccess)
        return RM_ERR_CUDA;
    // the stack waits for its input and for the previous read-back of output slot s
    if (cudaStreamWaitEvent(stream, h->ev_copied[s], 0) != cudaSuccess ||
        cudaStreamWaitEvent(stream, h->ev_read[s], 0) != cudaSuccess)
        return RM_ERR_CUDA;
    if ((st = run_stack(h, blocks, xb, pb, nullptr, B, stream)) != RM_OK) return st;
    if (cudaEventRecord(h->ev_computed[s], stream) != cudaSuccess ||
        cudaStreamWaitEvent(h->d2h, h->ev_computed[s], 0) != cudaSuccess ||
        cudaMemcpyAsync(pooled_host, pb, out_bytes, cudaMemcpyDeviceToHost, h->d2h) != cudaSuccess ||
        cudaEventRecord(h->ev_read[s], h->d2h) != cudaSuccess)
        return RM_ERR_CUDA;
    return RM_OK;
}

rm_status rm_host_wait(rm_handle* h) {
    if (!h) return RM_ERR_INVALID_ARG;
    if (!h->pipe_ready) return RM_OK;
    // every call's read-back is ordered after its stack, which follows its copy in
    return cuda_status(cudaStreamSynchronize(h->d2h));
}

// ---- token-sharded forward (one rank's share; the caller runs the all-to-all)
namespace {
rm_status check_shard(const rm_handle* h, int B, int world) {
    if (!h) return RM_ERR_INVALID_ARG;
    const rm_config& c = h->cfg;
    if (B < 1 || B > c.B_max || world < 1) return RM_ERR_INVALID_ARG;
    if (c.dtype != RM_BF16 || c.n_experts != 0 || c.D % 8 || c.D > 2048) return RM_ERR_UNSUPPORTED;
    const long long T = (long long)c.T * world;
    if (c.D % world || (c.D / world) % 8 || c.D % T || (c.D / T) % 8) return RM_ERR_UNSUPPORTED;
    return RM_OK;
}
}  // namespace

rm_status rm_tokshard_pack(rm_handle* h, const void* Za, const void* Zb, const float* ln_g, const float* ln_b,
                           void* Xh, void* send, int B, int world, rm_stream_t stream) {
    rm_status st = check_shard(h, B, world);
    if (st != RM_OK) return st;
    if (!aligned16(Za) || !aligned16_or_null(Zb) || !aligned16(Xh) || !aligned16(send)) return RM_ERR_INVALID_ARG;
    if ((ln_g == nullptr) != (ln_b == nullptr) || !aligned16_or_null(ln_g) || !aligned16_or_null(ln_b))
        return RM_ERR_INVALID_ARG;
    return cuda_status(rm::launch_shard_pack(Za, Zb, ln_g, ln_b, h->cfg.ln_eps, Xh, send, B, h->cfg.T, h->cfg.D,
                                             world, stream));
}

rm_status rm_tokshard_mix_ln(rm_handle* h, const void* recv, const void* Xh, const float* ln1_g, const float* ln1_b,
                             void* S, int B, int world, rm_stream_t stream) {
    rm_status st = check_shard(h, B, world);
    if (st != RM_OK) return st;
    if (!h->cfg.mix_addnorm) return RM_ERR_UNSUPPORTED;
    if (!aligned16(recv) || !aligned16(Xh) || !aligned16(S) || !aligned16(ln1_g) || !aligned16(ln1_b))
        return RM_ERR_INVALID_ARG;
    ProfScope ps(h, RM_K_MIX_LN, stream);
    return cuda_status(rm::launch_shard_mix_ln(recv, Xh, ln1_g, ln1_b, h->cfg.ln_eps, S, B, h->cfg.T, h->cfg.D, world,
                                               stream));
}

rm_status rm_tokshard_pool(rm_handle* h, const void* V, const void* S, const float* ln2_g, const float* ln2_b,
                           float* pooled_part, int B, rm_stream_t stream) {
    rm_status st = check_shard(h, B, 1);
    if (st != RM_OK) return st;
    if (!aligned16(V) || !aligned16(S) || !aligned16(ln2_g) || !aligned16(ln2_b) || !aligned16(pooled_part))
        return RM_ERR_INVALID_ARG;
    ProfScope ps(h, RM_K_LN_POOL, stream);
    return cuda_status(
        rm::launch_shard_pool(V, S, ln2_g, ln2_b, h->cfg.ln_eps, pooled_part, B, h->cfg.T, h->cfg.D, stream));
}

rm_status rm_padsplit_tokenize(rm_handle* h, const void* const* groups, const int* widths, int n_groups, void* X0,
                               int B, rm_stream_t stream) {
    rm_status st = check_batch(h, B);
    if (st != RM_OK) return st;
    if (!groups || !widths || n_groups < 1 || n_groups > 32 || !aligned16(X0)) return RM_ERR_INVALID_ARG;
    rm::PadSplitArgs a{};
    a.n = n_groups;
    a.col0[0] = 0;
    const int width = h->cfg.T * h->cfg.D;
    for (int i = 0; i < n_groups; ++i) {
        if (widths[i] < 1 || widths[i] % 8 || !aligned16(groups[i])) return RM_ERR_INVALID_ARG;
        a.src[i] = groups[i];
        a.col0[i + 1] = a.col0[i] + widths[i];
        if (a.col0[i + 1] > width) return RM_ERR_INVALID_ARG;
    }
    ProfScope ps(h, RM_K_PADSPLIT, stream);
    return cuda_status(rm::launch_padsplit(h->cfg.dtype, a, X0, B, width, stream));
}

rm_status rm_head_forward(rm_handle* h, const void* w, const float* bias, const float* pooled, float* prob, int B,
                          rm_stream_t stream) {
    rm_status st = check_batch(h, B);
    if (st != RM_OK) return st;
    if (!aligned16(w) || !bias || !aligned16(pooled) || !prob) return RM_ERR_INVALID_ARG;
    ProfScope ps(h, RM_K_HEAD, stream);
    return cuda_status(rm::launch_head(h->cfg.dtype, pooled, w, bias, prob, B, h->cfg.D, stream));
}

rm_status rm_sync_status(rm_handle* h, rm_stream_t stream) {
    if (!h) return RM_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return RM_ERR_CUDA;
    int v[2] = {0, 0};
    if (cudaMemcpy(v, h->err, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return RM_ERR_CUDA;
    if (v[0] != 0) {
        h->last_site = v[1];
        if (cudaMemset(h->err, 0, sizeof(v)) != cudaSuccess) return RM_ERR_CUDA;
        // a GEMM that stopped early may have left split-K arrival counts behind
        if (h->sk_cnt && cudaMemset(h->sk_cnt, 0, rm::gemm_tc_split_cnt_ints(h->num_sms) * sizeof(int)) != cudaSuccess)
            return RM_ERR_CUDA;
    }
    return static_cast<rm_status>(v[0]);
}

int rm_last_error_site(const rm_handle* h) { return h ? h->last_site : 0; }

rm_status rm_set_wait_budget(rm_handle* h, unsigned long long ns) {
    if (!h || ns == 0) return RM_ERR_INVALID_ARG;
    h->budget_ns = ns;
    return RM_OK;
}

rm_status rm_selftest_wait_timeout(rm_handle* h, rm_stream_t stream) {
    if (!h) return RM_ERR_INVALID_ARG;
    return cuda_status(rm::launch_selftest_wait(derr(h), h->budget_ns, stream));
}

rm_status rm_profile_begin(rm_handle* h, int max_launches) {
    if (!h || max_launches < 1) return RM_ERR_INVALID_ARG;
    if (h->ev_cap < max_launches) {
        free_events(h);
        h->ev = static_cast<cudaEvent_t*>(calloc(2 * (size_t)max_launches, sizeof(cudaEvent_t)));
        h->ev_kind = static_cast<int*>(calloc((size_t)max_launches, sizeof(int)));
        if (!h->ev || !h->ev_kind) {
            free(h->ev);
            free(h->ev_kind);
            h->ev = nullptr;
            h->ev_kind = nullptr;
            return RM_ERR_OOM;
        }
        for (int i = 0; i < 2 * max_launches; ++i) {
            if (cudaEventCreate(&h->ev[i]) != cudaSuccess) {
                h->ev_cap = i / 2;   // free_events destroys 2 * ev_cap events
                for (int j = 2 * h->ev_cap; j < i; ++j) cudaEventDestroy(h->ev[j]);
                free_events(h);
                return RM_ERR_CUDA;
            }
        }
        h->ev_cap = max_launches;
    }
    h->ev_n = 0;
    h->prof = true;
    return RM_OK;
}

rm_status rm_profile_end(rm_handle* h, float* ms_by_kind, int* launches_by_kind, int n_kinds) {
    if (!h || n_kinds < 0) return RM_ERR_INVALID_ARG;
    h->prof = false;
    for (int k = 0; k < n_kinds; ++k) {
        if (ms_by_kind) ms_by_kind[k] = 0.f;
        if (launches_by_kind) launches_by_kind[k] = 0;
    }
    for (int i = 0; i < h->ev_n; ++i) {
        if (cudaEventSynchronize(h->ev[2 * i + 1]) != cudaSuccess) return RM_ERR_CUDA;
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, h->ev[2 * i], h->ev[2 * i + 1]) != cudaSuccess) return RM_ERR_CUDA;
        const int k = h->ev_kind[i];
        if (k >= 0 && k < n_kinds) {
            if (ms_by_kind) ms_by_kind[k] += ms;
            if (launches_by_kind) launches_by_kind[k] += 1;
        }
    }
    h->ev_n = 0;
    return RM_OK;
}

const char* rm_kernel_name(int kind) {
    static const char* names[RM_K_COUNT] = {"mix_ln", "gemm1", "gemm2", "ln_pool", "layernorm", "token_mix",
                                            "moe_route", "moe_gather", "moe_combine", "padsplit", "head"};
    return kind >= 0 && kind < RM_K_COUNT ? names[kind] : "unknown";
}

}  // extern "C"
