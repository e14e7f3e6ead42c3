/*
 * rankmixer.h -- C ABI of librankmixer.so, the B200 (sm_100a) forward pass of
 * a stack of RankMixer blocks.
 *
 * Model (fun-rec chapter "Rankmixer: 硬件效率优化", section RankMixer整体架构):
 *     S_{n-1} = LN(TokenMixing(X_{n-1}) + X_{n-1})
 *     X_n     = LN(PFFN(S_{n-1}) + S_{n-1})
 * for n = 1..L, then mean pooling over the T tokens.
 *
 * Conventions shared by every entry point:
 *   - Tensor pointers are DEVICE pointers owned by the caller, unless an entry
 *     point says "host".  They must be 16-byte aligned.
 *   - Activations are row-major [B, T, D]: token t of sample b starts at
 *     element (b*T + t)*D.  Element type is the handle's dtype (RM_BF16 =
 *     bfloat16, RM_F32 = float).  pooled outputs are always float.
 *   - Weight matrices (handle dtype) are stored per token, output-major (the
 *     orientation of the product W1 s_t in the Per-Token FFN equation):
 *       dense  W1 [T][kD][D]      W2 [T][D][kD]      b1 [T][kD]  b2 [T][D]
 *       MoE    W1 [T][Ne][kD][D]  W2 [T][Ne][D][kD]  b1 [T][Ne][kD]  b2 [T][Ne][D]
 *              Wr [T][Ne][D]      br [T][Ne]
 *     Biases, router and LayerNorm parameters are float.  LayerNorm
 *     parameters are [D], one pair per LN instance, shared by all tokens.
 *   - Calls are asynchronous on the given stream (NULL = legacy default
 *     stream) and never synchronise the host, except rm_sync_status and
 *     rm_stack_forward_host.  Argument errors are returned before anything is
 *     launched.  Faults detected on the device (a bounded wait that ran out)
 *     set the handle's device error word, read by rm_sync_status.
 *   - A handle owns its device workspace (allocated by rm_create); the
 *     forward calls allocate nothing.  One handle must not be used from two
 *     streams or threads at the same time.
 *   - Requirements: D % T == 0 (H = T heads of width D/T), D % 16 == 0 and
 *     hidden % 16 == 0 for RM_BF16 (D % 4 == 0 for RM_F32), 1 <= B <= B_max,
 *     1 <= T <= 64, n_experts <= 32, n_experts * D <= 40960, D <= 2048 (bf16) or 1024 (fp32), and
 *     one sample (T * D elements, rows padded by < 128 bytes) plus T * (8 + 8 * P) + D * 8 bytes
 *     within 226 KB of shared memory (P = D / 64 for RM_BF16 when D % 64 == 0, else 1).  Violations return RM_ERR_INVALID_ARG or RM_ERR_UNSUPPORTED.
 *   - RM_F32 handles compute on CUDA cores only (no tensor cores).  RM_BF16
 *     handles run the FFN products on tcgen05 tensor cores with fp32
 *     accumulation; S, the FFN hidden and the pre-LN rows are stored bf16.
 */
#ifndef RANKMIXER_H
#define RANKMIXER_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
/* Same type as cudaStream_t. */
typedef struct CUstream_st *rm_stream_t;

typedef enum {
    RM_OK = 0,
    RM_ERR_INVALID_ARG = 1,     /* null/misaligned pointer, bad size            */
    RM_ERR_UNSUPPORTED = 2,     /* shape or mode this build does not implement  */
    RM_ERR_CUDA = 3,            /* a CUDA runtime call failed                   */
    RM_ERR_OOM = 4,             /* workspace allocation failed in rm_create     */
    RM_ERR_DEVICE_TIMEOUT = 5,  /* a bounded device-side wait ran out           */
    RM_ERR_DEVICE_BOUNDS = 6    /* a device-side bounds check failed            */
} rm_status;

typedef enum { RM_F32 = 0, RM_BF16 = 1 } rm_dtype;

/* FFN activation: GELU (tanh form or exact erf form), or ReLU (the activation
 * of the Mixer backbone timed in Appendix B of "重新理解 RankMixer"). */
typedef enum { RM_ACT_GELU_TANH = 0, RM_ACT_GELU_ERF = 1, RM_ACT_RELU = 2 } rm_act;

typedef struct {
    int B_max;       /* largest batch any call will pass                         */
    int T;           /* tokens per sample (= heads H)                            */
    int D;           /* token width                                              */
    int hidden;      /* FFN hidden width kD (per expert for MoE)                 */
    int L;           /* blocks in a stack                                        */
    int n_experts;   /* 0 = dense per-token FFN; else experts per token (Ne)     */
    rm_dtype dtype;
    float ln_eps;    /* LayerNorm epsilon, inside the square root (e.g. 1e-5)    */
    int act;         /* rm_act                                                   */
    int mix_addnorm; /* 1: S = LN(TokenMixing(X) + X), the block equation;        */
                     /* 0: S = TokenMixing(X), the variant without Add & Norm     */
                     /*    after mixing ("淘宝闪购-爆品团精排 Scaling Up 迭代实践", 3.5) */
} rm_config;

typedef struct {
    const void *W1, *b1, *W2, *b2;             /* see layout above; b1, b2 float */
    const float *ln1_g, *ln1_b;                /* LN after token mixing [D]      */
    const float *ln2_g, *ln2_b;                /* LN after the FFN [D]           */
    const float *Wr, *br;                      /* MoE router (NULL when dense)   */
    /* DTSI's second router h_infer (training only, may be NULL): its gates
     * carry L_reg; the forward routes with Wr, br.  Same shapes as Wr, br. */
    const float *Wr_infer, *br_infer;
} rm_block_weights;

typedef struct rm_handle rm_handle;

/* Create a handle on the current CUDA device and allocate its workspace for
 * batches up to cfg->B_max.  *out receives the handle (NULL on error).
 * Returns RM_ERR_OOM if the workspace does not fit. */
rm_status rm_create(const rm_config *cfg, rm_handle **out);

/* Release the workspace and the handle.  Waits for the handle's work. */
rm_status rm_destroy(rm_handle *h);

/* Bytes of device workspace the handle owns. */
size_t rm_workspace_bytes(const rm_handle *h);

/* Token mixing with H = T (section Token Mixing机制 of the fun-rec chapter:
 * SplitHead, then Concat per head):
 *     Y[b, h, t*dh + j] = X[b, t, h*dh + j],   dh = D / T.
 * A pure permutation; X and Y [B, T, D] must not overlap. */
rm_status rm_token_mix(rm_handle *h, const void *X, void *Y, int B, rm_stream_t stream);

/* Row LayerNorm, out = LN(A + R) over D for rows = B*T rows (R may be NULL).
 * gamma/beta [D] float.  A, R, out [rows, D] in the handle dtype; out may
 * alias A. */
rm_status rm_layernorm(rm_handle *h, const void *A, const void *R, const float *gamma,
                       const float *beta, void *out, int rows, rm_stream_t stream);

/* Per-token FFN (section Per-Token FFN of the fun-rec chapter):
 *     V[b, t] = W2_t GELU(W1_t S[b, t] + b1_t) + b2_t
 * S, V [B, T, D]; uses w->W1, b1, W2, b2.  No residual, no LayerNorm.
 * bf16 runs two grouped tcgen05 GEMMs (the hidden [T, B, hidden] in the
 * handle's workspace). */
rm_status rm_pffn_forward(rm_handle *h, const rm_block_weights *w, const void *S, void *V,
                          int B, rm_stream_t stream);

/* Sparse-MoE per-token FFN with ReLU routing (section Sparse MoE扩展 of the
 * fun-rec chapter; "特征交叉 —— RankMixer 精读笔记", PFFN paragraph):
 *     G[b, t, j] = ReLU(Wr_t[j] . S[b, t] + br_t[j])
 *     V[b, t]    = sum over j with G > 0 of G[b, t, j] * FFN_{t,j}(S[b, t])
 * Experts whose gate is 0 are not evaluated.  gates (may be NULL) receives G
 * [B, T, Ne] float.  Needs an MoE handle (n_experts > 0) of dtype RM_BF16. */
rm_status rm_moe_forward(rm_handle *h, const rm_block_weights *w, const void *S, void *V,
                         float *gates, int B, rm_stream_t stream);

/* One RankMixer block: Xout = LN2(F(S) + S), S = LN1(TokenMixing(X) + X)
 * (S = TokenMixing(X) when cfg.mix_addnorm is 0), F the dense or MoE
 * per-token FFN.  X, Xout [B, T, D]; may alias. */
rm_status rm_block_forward(rm_handle *h, const rm_block_weights *w, const void *X, void *Xout,
                           int B, rm_stream_t stream);

/* The stack: cfg.L blocks (blocks[0..L-1]) from X0, then the mean over the
 * T tokens of the last block's output (section RankMixer整体架构):
 *     pooled[b, :] = (1/T) sum_t X_L[b, t, :]          pooled [B, D] float
 * Xlast (may be NULL) receives X_L [B, T, D].  X0 is not modified. */
rm_status rm_stack_forward(rm_handle *h, const rm_block_weights *blocks, const void *X0,
                           float *pooled, void *Xlast, int B, rm_stream_t stream);

/* rm_stack_forward for callers whose X0 and pooled live in HOST memory
 * (pinned memory gives full copy speed).  Copies X0 into the handle's
 * workspace, runs the stack, copies pooled back, and synchronises the stream
 * before returning.  Weights stay device pointers. */
rm_status rm_stack_forward_host(rm_handle *h, const rm_block_weights *blocks,
                                const void *X0_host, float *pooled_host, int B,
                                rm_stream_t stream);

/* Asynchronous form of rm_stack_forward_host for back-to-back batches (a
 * serving runtime facility; the pages define no such call).  Returns after
 * enqueueing: X0_host is copied into one of two device input buffers on the
 * handle's own copy stream, the stack runs on `stream` once that copy and the
 * previous read-back of the same buffer pair are done, and pooled is copied
 * into pooled_host on a second copy stream.  So the input copy of call i+1
 * overlaps the stack of call i.  X0_host must stay unchanged and pooled_host
 * unread until rm_host_wait returns.  All asynchronous calls of a handle use
 * the same `stream`, with the handle's device current.  Host buffers should
 * be pinned (pageable memory makes the copies synchronous). */
rm_status rm_stack_forward_host_async(rm_handle *h, const rm_block_weights *blocks,
                                      const void *X0_host, float *pooled_host, int B,
                                      rm_stream_t stream);

/* Blocks until every rm_stack_forward_host_async call of the handle has
 * written its pooled_host.  RM_ERR_CUDA if a copy or launch failed; device
 * errors are read by rm_sync_status. */
rm_status rm_host_wait(rm_handle *h);

/* Pad-Split tokenisation ("淘宝闪购-爆品团精排 Scaling Up 迭代实践", section
 * 3.4: concatenate all feature-group embeddings, zero-pad, split into equal
 * tokens, no projection):
 *     X0[b, :] = [groups[0][b, :] ; ... ; groups[n-1][b, :] ; 0 ... 0]
 * groups: HOST array of n_groups DEVICE pointers, groups[i] [B, widths[i]]
 * in the handle dtype; widths: host array.  sum(widths) <= T*D, every width a
 * multiple of 8; n_groups <= 32.  X0 [B, T*D]. */
rm_status rm_padsplit_tokenize(rm_handle *h, const void *const *groups, const int *widths,
                               int n_groups, void *X0, int B, rm_stream_t stream);

/* Prediction head on the pooled vector: prob[b] = sigmoid(pooled[b] . w + bias).
 * w [D] in the handle dtype, bias: device pointer to one float, pooled [B, D]
 * float, prob [B] float. */
rm_status rm_head_forward(rm_handle *h, const void *w, const float *bias, const float *pooled,
                          float *prob, int B, rm_stream_t stream);

/* Synchronise the stream, then return and clear the device error word
 * (RM_OK, RM_ERR_DEVICE_TIMEOUT or RM_ERR_DEVICE_BOUNDS), or RM_ERR_CUDA. */
rm_status rm_sync_status(rm_handle *h, rm_stream_t stream);

/* Detail of the last device error: the site id of the wait that ran out. */
int rm_last_error_site(const rm_handle *h);

/* Budget, in nanoseconds, of every bounded device-side wait launched with
 * this handle from now on (default 1e9, 1 second). */
rm_status rm_set_wait_budget(rm_handle *h, unsigned long long ns);

/* Diagnostic: launch a kernel whose single wait is on an mbarrier that no one
 * ever arrives at, so the wait runs out after the handle's wait budget and the
 * kernel records RM_ERR_DEVICE_TIMEOUT.  Exists to test the timeout path. */
rm_status rm_selftest_wait_timeout(rm_handle *h, rm_stream_t stream);

/* ---- per-token FFN without device allocation ----------------------------
 * The pages have no counterpart to this entry point; it exists for callers
 * that cannot allocate device memory (code running where cudaMalloc is off
 * limits, e.g. inside another runtime's memory pool or with all device memory
 * reserved up front), so they cannot create a handle.
 *
 * Computes the same V = PFFN(S) as rm_pffn_forward (same kernels, same
 * layouts; dtype and act as in rm_config), with no handle.  Its only scratch,
 * the FFN hidden activations [T, B, hidden], lives in a fixed device array of
 * RM_STATIC_SCRATCH_BYTES inside the library, which every GPU that loads the
 * library holds until the process exits; the caller passes inputs and outputs
 * only, and the call allocates nothing.
 *   - Returns RM_ERR_INVALID_ARG, before launching anything, if
 *     T * B * hidden * sizeof(element) > RM_STATIC_SCRATCH_BYTES - 256, and
 *     RM_ERR_UNSUPPORTED if T > 64.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture.
 *   - Every call uses the same array: calls that overlap on the GPU (other
 *     streams, other host threads on the same device) race on it.
 *   - device_status (device pointer to one int, may be NULL) receives, in
 *     stream order, RM_OK or RM_ERR_DEVICE_TIMEOUT for this call. */
#define RM_STATIC_SCRATCH_BYTES (16u << 20)
rm_status rm_pffn_forward_static(const rm_block_weights *w, const void *S, void *V, int B, int T,
                                 int D, int hidden, rm_dtype dtype, int act, int *device_status,
                                 rm_stream_t stream);

/* ---- stack with e4m3 (fp8) FFN weights ------------------------------------
 * Lower-precision serving of the dense bf16 stack (8-bit serving is only
 * mentioned, in section 4.1 of the least reliable of the pages; the scheme
 * here is this library's own): the FFN
 * weights are quantised once to e4m3 with one fp32 scale per output channel,
 * and in every block S and the FFN hidden H are quantised per token row, so
 * both FFN projections run on the tensor cores' kind::f8f6f4 path and
 * dequantise in their epilogues (acc * scale_row * scale_channel, then the
 * bias, GELU / residual and LayerNorm partials as in the bf16 stack).
 * e4m3 keeps 3 mantissa bits: results differ from the bf16 stack by a few
 * percent relative L2 (the tests derive their bound from that rounding).
 *
 * rm_quantize_fp8: dst[r][k] = e4m3(src[r][k] / scale[r]) with scale[r] =
 *   max_k |src[r][k]| / 448 (1 for an all-zero row), src bf16 [rows][K],
 *   dst one byte per element, K % 16 == 0 (else RM_ERR_INVALID_ARG), K <=
 *   16384 and rows < 2^31 (else RM_ERR_UNSUPPORTED).  For W1 [T][kD][D] call it with
 *   rows = T*kD, K = D; for W2 [T][D][kD] with rows = T*D, K = kD.
 * rm_stack_forward_fp8: as rm_stack_forward (pooled output only) with the
 *   quantised weights of every block in q[l] (the biases, LayerNorm
 *   parameters come from blocks[l]); dense bf16 handles with D % 64 == 0 and
 *   hidden % 16 == 0, else RM_ERR_UNSUPPORTED.  The first call allocates the
 *   quantised activations (B_max*T*(D + kD) bytes + scales). */
typedef struct {
    const void *W1q, *W2q;          /* e4m3 [T][kD][D], [T][D][kD]     */
    const float *W1s, *W2s;         /* scales [T][kD], [T][D]          */
} rm_fp8_weights;
rm_status rm_quantize_fp8(const void *src, void *dst, float *scale, long long rows, int K, rm_stream_t stream);
rm_status rm_stack_forward_fp8(rm_handle *h, const rm_block_weights *blocks, const rm_fp8_weights *q, const void *X0,
                               float *pooled, int B, rm_stream_t stream);

/* ---- token-sharded forward (one rank's share) ------------------------------
 * G ranks each own Tl = T / G consecutive tokens: their rows of every sample
 * [B, Tl, D] and their per-token FFN weights.  The token mixing with H = T
 * then needs chunk h of every token's row on the rank owning token h: an
 * all-to-all between the ranks ("特征交叉 —— RankMixer 精读笔记": the mixing
 * works like an all-to-all; "重新理解 RankMixer" section 3.3, model sharding).
 * The handle is created with cfg->T = Tl (the rank's tokens).  Per block:
 *   rm_tokshard_pack: Xh = LN(Za + Zb) with (ln_g, ln_b) (the previous
 *     block's LN2 of V + S), or Za alone (ln_g = ln_b = Zb = NULL: the stack
 *     input); Xh [B, Tl, D] is written (kept for the residual) and its
 *     column range [r D/G, (r+1) D/G) of each row to send + r * B*Tl*D/G,
 *     laid out [r][b][tq][D/G], for an equal-split all-to-all of send into
 *     recv (B*Tl*D elements each, bf16);
 *   rm_tokshard_mix_ln: S = LN1(TokenMixing(Xh) + Xh) for the rank's tokens,
 *     the mixed pieces read from recv ([q][b][tq][D/G]);
 *   rm_pffn_forward on S with the rank's token weights (W1 + rank*Tl*kD*D, ...);
 *   after the last block rm_tokshard_pool: pooled_part [B, D] float = ln2_g *
 *     mean over the rank's tokens of xhat(V + S) + ln2_b; the pooled output
 *     is the mean of the G ranks' parts.
 * Supported: bf16, dense FFN, Add & Norm after mixing, D % G == 0,
 * (D / G) % 8 == 0, (D / T) % 8 == 0, D <= 2048; else RM_ERR_UNSUPPORTED. */
rm_status rm_tokshard_pack(rm_handle *h, const void *Za, const void *Zb, const float *ln_g, const float *ln_b,
                           void *Xh, void *send, int B, int world, rm_stream_t stream);
rm_status rm_tokshard_mix_ln(rm_handle *h, const void *recv, const void *Xh, const float *ln1_g, const float *ln1_b,
                             void *S, int B, int world, rm_stream_t stream);
rm_status rm_tokshard_pool(rm_handle *h, const void *V, const void *S, const float *ln2_g, const float *ln2_b,
                           float *pooled_part, int B, rm_stream_t stream);

/* ---- training step (dense and sparse-MoE bf16 stacks) ---------------------
 * One training step of a stack of L dense RankMixer blocks with the sigmoid
 * head: the forward pass (keeping what the backward pass needs), the task loss
 * and the gradient of the loss with respect to every parameter and to the
 * stack input.  The pages give the FLOPs of a RankMixer training step
 * ("重新理解 RankMixer", Table 1) and name the task loss without defining it
 * (fun-rec "Rankmixer: 硬件效率优化", section Sparse MoE扩展: L = L_task +
 * lambda L_reg); this library takes the mean binary cross-entropy of the
 * sigmoid head,
 *     L = (1/B) sum_b [softplus(logit_b) - y_b logit_b],
 *     logit_b = head_w . mean_t X_L[b, t] + head_b,
 * and the gradients are the chain rule through the block equations (the
 * token mixing with H = T is its own transpose).
 *
 * A trainer owns its device workspace (per block: S, the normalised mixed
 * rows, their 1/sqrt(var + eps), the FFN activation input and output, the
 * pre-LN rows and their statistics; plus the backward buffers), allocated by
 * rm_train_create for batches up to cfg->B_max.  Supported: dtype RM_BF16,
 * n_experts 0 (dense) or 1..32 (sparse MoE with ReLU routing), mix_addnorm 1,
 * D % 64 == 0, hidden % 64 == 0, (D / T) % 8 == 0, D <= 2048, plus the
 * forward's limits.  Otherwise RM_ERR_UNSUPPORTED.  Sparse-MoE blocks keep
 * their routing, their compacted expert rows (each expert's slot list padded
 * to a multiple of 64 with zero rows) and the experts' activation inputs, and
 * the backward pass computes, per active (sample, token, expert) entry,
 * dG = dV . e_j and de_j = G_j dV, the experts' gradients over their slots
 * (the weight gradients as products whose K runs over the expert's slots),
 * and the routers' gradients through ReLU (fun-rec "Rankmixer: 硬件效率优化",
 * section Sparse MoE扩展). */
typedef struct rm_trainer rm_trainer;

/* Gradient outputs of one block (device pointers, float, the parameters'
 * shapes and layouts): W1 [T][kD][D], b1 [T][kD], W2 [T][D][kD], b2 [T][D],
 * ln1_g, ln1_b, ln2_g, ln2_b [D]; sparse MoE: W1 [T][Ne][kD][D], b1
 * [T][Ne][kD], W2 [T][Ne][D][kD], b2 [T][Ne][D], the router's Wr [T][Ne][D]
 * and br [T][Ne], and DTSI's second router's Wr_infer, br_infer (when the
 * block's weights give one; else unused, may be NULL).  Every entry is
 * overwritten (not added to). */
typedef struct {
    float *W1, *b1, *W2, *b2;
    float *ln1_g, *ln1_b, *ln2_g, *ln2_b;
    float *Wr, *br, *Wr_infer, *br_infer;
} rm_block_grads;

rm_status rm_train_create(const rm_config *cfg, rm_trainer **out);
/* Weight lambda of L_reg (default 0; lambda >= 0, else RM_ERR_INVALID_ARG):
 * the loss becomes L_task + lambda * (sum over the batch's tokens and experts
 * of the regularised gates of every MoE block: DTSI's second router's where a
 * block gives one, else the routing gates).  fun-rec "Rankmixer: 硬件效率优化",
 * section Sparse MoE扩展 (L = L_task + lambda L_reg, DTSI-MoE). */
rm_status rm_train_set_reg(rm_trainer *t, float lambda);
rm_status rm_train_destroy(rm_trainer *t);
size_t rm_train_workspace_bytes(const rm_trainer *t);

/* One step on B samples (8 <= B <= B_max, B % 8 == 0):
 *   X0 [B, T, D] bf16 input; head_w [D] bf16, head_b [1] float; labels [B]
 *   float (0 or 1); grads [L] outputs; dX0 [B, T, D] bf16 (may be NULL):
 *   dL/dX0; dhead_w [D], dhead_b [1], loss [1] float outputs; pooled_out
 *   [B, D] float (may be NULL): the forward's pooled output.
 * Asynchronous on the stream; device-side faults (a bounded wait that ran
 * out) set the trainer's error word, read by rm_train_sync_status. */
rm_status rm_train_step(rm_trainer *t, const rm_block_weights *blocks, const void *X0, const void *head_w,
                        const float *head_b, const float *labels, const rm_block_grads *grads, void *dX0,
                        float *dhead_w, float *dhead_b, float *loss, float *pooled_out, int B,
                        rm_stream_t stream);

/* Synchronise the stream and return the trainer's device error word. */
rm_status rm_train_sync_status(rm_trainer *t, rm_stream_t stream);

/* ---- launch profiling ----------------------------------------------------
 * Kernel kinds launched by the forward entry points: */
typedef enum {
    RM_K_MIX_LN = 0,      /* token mixing + residual + LayerNorm (prev. LN2 on load) */
    RM_K_GEMM1 = 1,       /* FFN first projection + bias + GELU (grouped GEMM)       */
    RM_K_GEMM2 = 2,       /* FFN second projection + bias (+ residual / gate)        */
    RM_K_LN_POOL = 3,     /* last LayerNorm + mean pooling                           */
    RM_K_LAYERNORM = 4,
    RM_K_TOKEN_MIX = 5,
    RM_K_MOE_ROUTE = 6,   /* router + ReLU gates + compaction                        */
    RM_K_MOE_GATHER = 7,
    RM_K_MOE_COMBINE = 8,
    RM_K_PADSPLIT = 9,
    RM_K_HEAD = 10,
    RM_K_COUNT = 11
} rm_kernel_kind;

/* Start recording a CUDA event pair around each kernel launch made through h
 * (on the launch stream), for up to max_launches launches; later launches
 * are not recorded.  Restarts any recording in progress. */
rm_status rm_profile_begin(rm_handle *h, int max_launches);

/* Stop recording, wait for the recorded events, and return per kind the
 * summed elapsed milliseconds and the number of recorded launches (arrays of
 * n_kinds entries, indexed by rm_kernel_kind; either may be NULL). */
rm_status rm_profile_end(rm_handle *h, float *ms_by_kind, int *launches_by_kind, int n_kinds);

/* Name of a kernel kind ("gemm1", ...), or "unknown". */
const char *rm_kernel_name(int kind);

/* Static description of a status code. */
const char *rm_status_string(rm_status s);

#ifdef __cplusplus
}
#endif

#endif /* RANKMIXER_H */
