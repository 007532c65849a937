/*
 * libsparseattn — block-sparse attention with in-softmax block approximation,
 * for NVIDIA B200 (sm_100a).
 *
 * The method (sources, by page title):
 *   [PISA]  "PISA - Atenção Esparsa por Partes para Transformers de Difusão
 *            Eficientes", §2 "Algoritmo Central" and "Implementação de Hardware"
 *   [SLA2]  "SLA2: Sparse-Linear Attention with Learnable Routing and QAT",
 *            §2A (mixture), §2B (router), §2C (low-precision sparse branch)
 *   [SALAD] "SALAD: Achieve High-Sparsity Attention via Efficient Linear
 *            Attention Tuning for Video Diffusion Transformer", §2 (ReLU
 *            linear branch in parallel with the sparse one)
 *   [SPLA]  "SPLA - Block Sparse Plus Linear Attention para Modelagem de
 *            Contexto Longo", §2.1 (second-order block score), §2.2
 *            (subtraction form of the residual linear term; decode is bound
 *            by KV loading)
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers to memory the caller owns; the
 *     library allocates nothing and frees nothing.  Dense activations are
 *     row-major and contiguous: [B, H, N, d] means d is the fastest axis.
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL is the legacy default stream).  The return value reports host-side
 *     argument validation and the launch; a fault inside a kernel surfaces at
 *     the caller's next synchronisation as usual.
 *   - On any status other than SA_OK nothing has been launched, except for
 *     SA_ERR_CUDA (a launch failed; earlier launches of the same call may have
 *     run).  sa_last_error() then returns a message for the calling thread.
 *   - Supported: d in {64, 128}; block in {64, 128}; N a multiple of block;
 *     0 <= topk <= N/block; pointers 16-byte aligned.
 *   - Nothing is thrown across this interface.
 */
#ifndef SPARSEATTN_H
#define SPARSEATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SA_OK = 0,
  SA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, topk out of range */
  SA_ERR_UNSUPPORTED = 2,   /* valid request this build does not implement */
  SA_ERR_ALIGNMENT = 3,     /* a pointer is not 16-byte aligned */
  SA_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
  SA_ERR_WORKSPACE = 5      /* workspace missing or smaller than required */
} sa_status;

typedef enum { SA_FP32 = 0, SA_BF16 = 1 } sa_dtype;

typedef enum {
  SA_ROUTE_DOT = 0,      /* q̄_i · k̄_j on mean-pooled blocks [SLA2 §2B] */
  SA_ROUTE_PROJ = 1,     /* (q̄_i P_q) · (k̄_j P_k), learnable router [SLA2 §2B] */
  SA_ROUTE_TAYLOR2 = 2,  /* s q̄·k̄_j + log1p(½ s² Σ_c q̄_c² var_jc), the log of
                            exp(q·k̄)(1 + ½ qᵀ diag(Var k) q) [SPLA §2.1] */
  SA_ROUTE_COV = 3       /* s q̄·k̄_j + log1p(s ‖q̄_i‖ M_j / block): the block's
                            zero-order mass plus the bound s‖q‖M_j on the
                            first-order term the hybrid order leaves out,
                            M_j = ‖H_j − H̄‖₂ (stats->covnorm)
                            [PISA §2 "Roteamento Consciente de Covariância"] */
} sa_route_mode;

typedef enum {
  SA_TAIL_DROP = 0,        /* unselected blocks contribute nothing */
  SA_TAIL_ZERO_ORDER = 1,  /* PISA zero-order block term inside numerator
                              and denominator [PISA §2 "Algoritmo Central"] */
  SA_TAIL_LINEAR_MIX = 2,  /* O = α⊙O_s + (1−α)⊙O_l, O_l = ReLU linear
                              attention over the unselected blocks
                              [SLA2 §2A, SALAD §2, SPLA §2.2] */
  SA_TAIL_FIRST_ORDER = 3, /* PISA hybrid order: the zero-order terms plus
                              the global first-order correction of the
                              numerator, (s q) H̄ Σ_{j∈U} e^{s q·k̄_j}
                              [PISA §2 "Algoritmo Central"] */
  SA_TAIL_RESIDUAL_LINEAR = 4  /* decode only: o = O_s + RMSNorm(o_rla),
                              O_s the DROP output, o_rla = φ(q)ᵀ Σ_{n∈U}
                              φ(k_n) v_nᵀ with φ = exp, formed as
                              φ(q)ᵀ S_all − Σ_{n∈S} (φ(q)·φ(k_n)) v_n from
                              the tiles the exact pass loads; RMSNorm(x) =
                              x / sqrt(mean(x²) + 1e-6), unit gain
                              [SPLA §2.2 subtraction form, §2.3] */
} sa_tail_mode;

/* Shape of a prefill problem: Q, K, V, O are [B, H, N, d]; query blocks and
 * KV blocks both hold `block` consecutive tokens (nb = N / block of each). */
typedef struct {
  int32_t B, H, N, d, block;
} sa_shape;

/* Shape of a GQA decode problem: q and o are [B, Hq, d] (one token per
 * sequence), the caches are [B, Hkv, N, d]; query head h reads KV head
 * h / (Hq / Hkv). */
typedef struct {
  int32_t B, Hq, Hkv, N, d, block;
} sa_decode_shape;

/* Block statistics, float32 device arrays owned by the caller.  A NULL field
 * is not computed by sa_block_pool and must not be needed by a later call.
 * nqb = nb = N / block.  [PISA "Implementação de Hardware", pre-computation;
 * SLA2 §2B pooling; SPLA §2.1 block mean and diagonal covariance] */
typedef struct {
  float* qmean;     /* [B,H,nqb,d] mean of each query block                 */
  float* kmean;     /* [B,H,nb,d]  mean of each key block (centroid k̄_j)    */
  float* vsum;      /* [B,H,nb,d]  sum of each value block Σ_n v_{j,n}       */
  float* kvar;      /* [B,H,nb,d]  per-channel population variance of keys */
  float* zrelu;     /* [B,H,nb,d]  Σ_{n∈j} relu(k_n)                         */
  float* htot;      /* [B,H,d,d]   Σ_n relu(k_n) v_nᵀ over all tokens        */
  float* ztot;      /* [B,H,d]     Σ_n relu(k_n) over all tokens             */
  uint16_t* kmean_bf16;  /* [B,H,nb,d] bf16 copy of kmean (tensor-core tail) */
  uint16_t* vmean_bf16;  /* [B,H,nb,d] bf16 of vsum / block (tensor-core tail) */
  float* hbar;      /* [B,H,d,d]   H̄ = (1/nb) Σ_j Σ_{n∈j} (k_n − k̄_j) v_nᵀ, the
                       mean first-order block statistic of PISA's hybrid
                       order [PISA §2]; row c, column e                     */
  uint16_t* hbarT_bf16;  /* [B,H,d,d] bf16 of H̄ᵀ (row e, column c; the
                       tensor-core first-order tail)                        */
  float* covnorm;   /* [B,H,nb]    M_j = ‖H_j − H̄‖₂, the spectral norm of each
                       block's first-order deviation from the mean (Lanczos
                       on the Gram matrix to 1e-6 relative)
                       [PISA §2 "Roteamento Consciente de Covariância"]    */
  float* sexp;      /* [B,H,d,d]   S_all = Σ_n φ(k_n) v_nᵀ over all tokens, φ = exp
                       (bf16-rounded on the tensor-core path, as the decode
                       kernel rounds φ(k) of the selected blocks)
                       [SPLA §2.2, the residual linear state]              */
  uint16_t* kvar_bf16;   /* [B,H,nb,d] bf16 copy of kvar (the decode's bf16
                       statistics; with kmean_bf16 and vmean_bf16 they are
                       half the bytes of the float32 kmean, kvar, vsum)    */
} sa_block_stats;

/* Block statistics of Q (optional), K and V.
 * Q: [B,H,N,d] or NULL (then stats->qmean is ignored); K, V: [B,H,N,d];
 * dtype: element type of Q, K, V.  Every non-NULL field of *stats is written
 * (the bf16 copies are the round-to-nearest-even bf16 of the float32 values);
 * kmean and vsum are required.  htot, ztot and hbar are sums over all tokens
 * of a head and are overwritten (no accumulation across calls); hbarT_bf16
 * and covnorm need hbar.
 * Errors: SA_ERR_INVALID_ARG (null K/V/stats/kmean/vsum, bad shape),
 *         SA_ERR_UNSUPPORTED (d or block not supported), SA_ERR_ALIGNMENT. */
sa_status sa_block_pool(const void* Q, const void* K, const void* V, sa_dtype dtype,
                        sa_shape shape, const sa_block_stats* stats, void* stream);

/* Router: scores every (query block i, KV block j) pair and keeps the topk
 * best KV blocks per query block [SLA2 §2B; PISA S_i; SPLA §2.1].
 * stats: needs qmean and kmean (+ kvar for TAYLOR2, covnorm for COV).  proj_q, proj_k: [d,d]
 * float32 row-major (x P means Σ_r x_r P[r][c]); required for PROJ, ignored
 * otherwise.  scale: softmax scale s (used by TAYLOR2 and COV; COV also
 * divides by shape.block).
 * block_idx: [B,H,nqb,topk] int32 output, ascending; a tie in score goes to
 * the smaller block index (may be NULL when topk == 0).  scores: [B,H,nqb,nb] float32 output or NULL.
 * Errors: SA_ERR_INVALID_ARG, SA_ERR_UNSUPPORTED (nb > 4096), SA_ERR_ALIGNMENT. */
sa_status sa_route(const sa_block_stats* stats, sa_shape shape, sa_route_mode mode,
                   const float* proj_q, const float* proj_k, float scale, int32_t topk,
                   int32_t* block_idx, float* scores, void* stream);

/* Sparse prefill forward [PISA §2; SLA2 §2A]:
 * for query row t of block i with selected set S_i = block_idx[b,h,i,:] and
 * unselected set U_i,
 *   DROP:        o_t = Σ_{n∈S} e^{s q·k_n} v_n / Σ_{n∈S} e^{s q·k_n}  (0 if S empty)
 *   ZERO_ORDER:  o_t = (Σ_{n∈S} e^{s q·k_n} v_n + Σ_{j∈U} e^{s q·k̄_j} vsum_j)
 *                    / (Σ_{n∈S} e^{s q·k_n}     + Σ_{j∈U} block·e^{s q·k̄_j})
 *   FIRST_ORDER: ZERO_ORDER with the numerator's first-order block term
 *                added through the head's mean statistic H̄ (stats->hbar):
 *                o_t = (N_t^ZO + (s q_t)ᵀ H̄ · Σ_{j∈U} e^{s q·k̄_j}) / D_t^ZO
 *                (the denominator's first-order term is zero: a block's key
 *                deviations from k̄_j sum to zero)
 *   LINEAR_MIX:  o_t = α_h ⊙ O_s + (1−α_h) ⊙ O_l,  O_s the DROP output,
 *                O_l = relu(q)ᵀ(H_tot − Σ_{j∈S} h_j) / (relu(q)·(z_tot − Σ_{j∈S} z_j) + 1e-6),
 *                h_j = Σ_{n∈j} relu(k_n) v_nᵀ (accumulated from the tiles the
 *                kernel already loads, SPLA §2.2's subtraction form);
 *                O_l = 0 when every block is selected (U_i empty).
 * Q, K, V, O: [B,H,N,d] of `dtype` (O has the same dtype).  block_idx:
 * [B,H,nqb,topk] int32, each row ascending without repeats, entries in
 * [0, nb).  alpha: [H,d] float32 (LINEAR_MIX only).  stats: ZERO_ORDER needs
 * kmean, vsum (and kmean_bf16, vmean_bf16 for the bf16 tensor-core path);
 * FIRST_ORDER needs those and hbar (+ hbarT_bf16 for the tensor-core path);
 * LINEAR_MIX needs zrelu, htot, ztot.
 * Errors: SA_ERR_INVALID_ARG, SA_ERR_UNSUPPORTED, SA_ERR_ALIGNMENT. */
sa_status sa_sparse_attn_fwd(const void* Q, const void* K, const void* V, sa_dtype dtype,
                             sa_shape shape, const int32_t* block_idx, int32_t topk,
                             sa_tail_mode tail, const float* alpha,
                             const sa_block_stats* stats, float scale, void* O,
                             void* stream);

/* sa_sparse_attn_fwd that also writes each query row's log-sum-exp of its
 * logits in log2 units: lse2[b,h,t] = log2 D_t, D_t the denominator of PISA
 * "Algoritmo Central" (Σ over the row's exact keys of e^{s q_t·k_n} plus,
 * for ZERO_ORDER, Σ over the unselected blocks of block·e^{s q_t·k̄_j}; for
 * DROP the first sum alone), +inf for a row without keys.  sa_sparse_attn_bwd_lse takes it to skip the
 * recomputation of the row statistics.  lse2: float32 [B,H,N], caller-owned,
 * 16-byte aligned.  Only the bf16 tensor-core kernel produces it: d = 128,
 * block 128, SA_TAIL_DROP, SA_TAIL_ZERO_ORDER or SA_TAIL_FIRST_ORDER (with
 * stats->kmean_bf16 and vmean_bf16, + hbarT_bf16 for FIRST_ORDER; the
 * first-order term changes the numerator only, so D_t is the zero-order one);
 * anything else returns SA_ERR_UNSUPPORTED.
 * Errors: those of sa_sparse_attn_fwd; SA_ERR_INVALID_ARG without lse2. */
sa_status sa_sparse_attn_fwd_lse(const void* Q, const void* K, const void* V, sa_dtype dtype,
                                 sa_shape shape, const int32_t* block_idx, int32_t topk,
                                 sa_tail_mode tail, const sa_block_stats* stats, float scale,
                                 void* O, float* lse2, void* stream);

/* Bytes of workspace sa_sparse_attn_bwd needs (0 on bad arguments). */
size_t sa_sparse_attn_bwd_workspace_size(sa_shape shape, int32_t topk);

/* Backward of sa_sparse_attn_fwd for the DROP, ZERO_ORDER and FIRST_ORDER
 * tails: given the forward's inputs, its output O and the output cotangent dO,
 * writes dQ, dK, dV (float32 [B,H,N,d], overwritten).  The forward is softmax
 * attention of query block i to its exact keys k_n (n in the selected
 * blocks) and, for ZERO_ORDER, one pseudo-key per unselected block j (key
 * k̄_j, value vsum_j / block, logit bias ln block), so with
 * p = exp(s q·k + bias − lse), δ_t = dO_t·o_t and ds = p (dO·v − δ):
 *   dQ = s Σ ds k,   dK_key = s Σ ds q,   dV_key = Σ p dO,
 * and each pseudo-key's gradients are spread over its block's tokens
 * divided by block (k̄ and vsum / block are means of the block's k and v).
 * FIRST_ORDER [PISA §2 "Algoritmo Central", hybrid order] adds λ_t f_t to the
 * zero-order output, f_t = s H̄ᵀ q_t, λ_t = Σ_{pseudo-keys} p / block: the
 * pseudo-keys' value seen by row t is v̄_j + f_t / block, and with
 * G = s Σ_t λ_t q_t dO_tᵀ the gradients gain dq_t += s λ_t H̄ dO_t,
 * dk_m += G (v_m − v̄_j) / nb and dv_m += Gᵀ (k_m − k̄_j) / nb for every
 * token m of block j (through H̄ = (1/nb) Σ_j Σ_{m∈j} (k_m − k̄_j) v_mᵀ); it
 * runs for bf16, d = 128, block 128 only (SA_ERR_UNSUPPORTED otherwise) and
 * needs stats->kmean, vsum, kmean_bf16, vmean_bf16 and hbar.
 * Q, K, V, O, dO of `dtype`; block_idx, topk, tail, stats (kmean, vsum for
 * ZERO_ORDER) and scale as given to the forward.  workspace: at least
 * sa_sparse_attn_bwd_workspace_size() bytes, 16-byte aligned.  bf16 with
 * d = 128 runs on the tensor cores (tcgen05 with TMEM accumulators for
 * block 128, warp-level MMAs for block 64; p and ds rounded to bf16 for the
 * second products, as the forward rounds p); fp32 and d = 64 run on CUDA
 * cores in fp32.  The sums over query blocks run in a fixed order (no
 * atomics), so the result does not depend on scheduling.
 * Errors: SA_ERR_INVALID_ARG, SA_ERR_UNSUPPORTED (other tails), SA_ERR_ALIGNMENT,
 *         SA_ERR_WORKSPACE. */
sa_status sa_sparse_attn_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                             sa_dtype dtype, sa_shape shape, const int32_t* block_idx, int32_t topk,
                             sa_tail_mode tail, const sa_block_stats* stats, float scale, float* dQ,
                             float* dK, float* dV, void* workspace, size_t workspace_bytes, void* stream);

/* sa_sparse_attn_bwd given the forward's lse2 (sa_sparse_attn_fwd_lse, same
 * inputs): the bf16 tensor-core path for block 128 then forms the scores
 * once per tile instead of twice; other paths recompute the statistics and
 * ignore lse2.  lse2: float32 [B,H,N], 16-byte aligned, required.
 * Errors: those of sa_sparse_attn_bwd; SA_ERR_INVALID_ARG without lse2. */
sa_status sa_sparse_attn_bwd_lse(const void* Q, const void* K, const void* V, const void* O,
                                 const void* dO, const float* lse2, sa_dtype dtype, sa_shape shape,
                                 const int32_t* block_idx, int32_t topk, sa_tail_mode tail,
                                 const sa_block_stats* stats, float scale, float* dQ, float* dK,
                                 float* dV, void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of workspace sa_sparse_attn_bwd_linear_mix needs (0 on bad arguments
 * or a shape it does not run: d and block must be 128). */
size_t sa_sparse_attn_bwd_linear_mix_workspace_size(sa_shape shape, int32_t topk);

/* Backward of sa_sparse_attn_fwd with SA_TAIL_LINEAR_MIX [SLA2 §2A; SALAD §2]:
 * O = α⊙O_s + (1−α)⊙O_l, O_s the softmax attention over the selected blocks
 * and O_l = φ(q)ᵀ H_U / (φ(q)·z_U + 1e-6) the ReLU linear attention over the
 * unselected ones (H_U = H_tot − Σ_{j∈S} h_j, z_U likewise; O_l = 0 when
 * every block is selected).  With g = dO_t and g_l = (1−α)⊙g:
 *   softmax branch: the DROP backward of the cotangent α⊙g, its
 *     δ_s = (α⊙g)·O_s = g·O − g_l·O_l formed from O and the recomputed O_l;
 *   linear branch: dnum = g_l / den, dden = −(g_l·O_l) / den,
 *     dq += 1[q > 0] ⊙ (H_U dnum + z_U dden), and per key block j, with
 *     dh_j = Σ_{query blocks i not selecting j} Σ_{t∈i} φ(q_t) dnumᵀ (and dz_j
 *     likewise), dk_n += 1[k_n > 0] ⊙ (dh_j v_n + dz_j), dv_n += dh_jᵀ φ(k_n).
 * Q, K, V, O, dO: bf16 [B,H,N,d] (O the forward's output); block_idx, topk,
 * alpha [H,d] and stats (htot, ztot, zrelu) as given to the forward.
 * dQ, dK, dV: float32 [B,H,N,d], overwritten.  workspace: at least
 * sa_sparse_attn_bwd_linear_mix_workspace_size() bytes, 16-byte aligned (it
 * holds the per-block h_j and per-query-block dH_U as bf16 d x d tiles).
 * bf16, d = 128, block 128 only (the softmax branch runs on the tcgen05
 * backward, the linear branch on mma.sync); sums run in a fixed order.
 * Errors: SA_ERR_INVALID_ARG, SA_ERR_UNSUPPORTED, SA_ERR_ALIGNMENT,
 *         SA_ERR_WORKSPACE. */
sa_status sa_sparse_attn_bwd_linear_mix(const void* Q, const void* K, const void* V, const void* O,
                                        const void* dO, sa_dtype dtype, sa_shape shape,
                                        const int32_t* block_idx, int32_t topk, const float* alpha,
                                        const sa_block_stats* stats, float scale, float* dQ, float* dK,
                                        float* dV, void* workspace, size_t workspace_bytes, void* stream);

/* Per-block e4m3 quantisation [SLA2 §2C, low-precision sparse branch]:
 * X: bf16 [BH][N][d] (BH = batch x heads); codes: uint8 [BH][N][d] e4m3fn bit
 * patterns; scales: float [BH][ceil(N/block)] with σ = absmax/448 of each block
 * of `block` rows (1 for an all-zero block; the last block may be ragged);
 * scale_max: float [BH] (max of the head's σ) or NULL.  code = e4m3(x / σ)
 * with the correctly rounded fp32 division, round-to-nearest-even and
 * saturation to ±448.  d and block in {64, 128}.
 * Errors: SA_ERR_INVALID_ARG, SA_ERR_UNSUPPORTED, SA_ERR_ALIGNMENT. */
sa_status sa_quantize_e4m3(const void* X, int64_t BH, int32_t N, int32_t d, int32_t block, uint8_t* codes,
                           float* scales, float* scale_max, void* stream);

/* e4m3 operands of sa_sparse_attn_fwd_fp8 (all device pointers; block 128). */
typedef struct {
  const uint8_t* q;            /* [B,H,N,d] codes of Q                          */
  const uint8_t* k;            /* [B,H,N,d] codes of K                          */
  const uint8_t* v;            /* [B,H,N,d] codes of V                          */
  const float* q_scale;        /* [B,H,N/128]                                   */
  const float* k_scale;        /* [B,H,N/128]                                   */
  const float* v_scale;        /* [B,H,N/128]                                   */
  const float* v_scale_max;    /* [B,H] max of v_scale over the head            */
  const uint8_t* kbar;         /* [B,H,nb,d] codes of kmean_bf16 (ZERO_ORDER)   */
  const uint8_t* vbar;         /* [B,H,nb,d] codes of vmean_bf16 (ZERO_ORDER)   */
  const float* kbar_scale;     /* [B,H,ceil(nb/128)] scales of 128-centroid tiles */
  const float* vbar_scale;     /* [B,H,ceil(nb/128)]                            */
} sa_fp8_operands;

/* Sparse prefill with the SLA2 §2C low-precision sparse branch: the same
 * DROP / ZERO_ORDER attention as sa_sparse_attn_fwd with e4m3 Q, K, V (and
 * centroid tiles, produced by sa_quantize_e4m3 from kmean_bf16 / vmean_bf16),
 * logits σ_Q σ_K (Q̂·K̂ᵀ), P quantised to e4m3 on the tensor cores, fp32
 * accumulation, row sums from the unquantised P.  O: bf16 [B,H,N,d].
 * d = block = 128.
 * Errors: SA_ERR_INVALID_ARG, SA_ERR_UNSUPPORTED, SA_ERR_ALIGNMENT, SA_ERR_CUDA. */
sa_status sa_sparse_attn_fwd_fp8(const sa_fp8_operands* ops, sa_shape shape, const int32_t* block_idx,
                                 int32_t topk, sa_tail_mode tail, float scale, void* O, void* stream);

/* Bytes of workspace sa_decode_fwd needs for this shape and topk (0 on bad
 * arguments). */
size_t sa_decode_workspace_size(sa_decode_shape shape, int32_t topk);

/* GQA decode of one query token per sequence [SPLA §2.1, §2.2; PISA §2]:
 * routes each (sequence, KV head) group with the TAYLOR2 score summed over the
 * group's query heads (a logsumexp of the log scores), keeps topk blocks, and
 * evaluates ZERO_ORDER (or DROP) attention for every query head of the group.
 * Split over the KV axis; partial (max, sum, acc) states are merged.
 * q: [B,Hq,d]; Kcache, Vcache: [B,Hkv,N,d], all of `dtype` (bf16 only);
 * the group Hq / Hkv is 1, 2, 4 or 8.
 * stats: the block statistics of the caches (sa_block_pool with Q = NULL),
 * read in one of two precisions:
 *   - float32: kmean, kvar and vsum (all three required);
 *   - bf16, when stats->kmean is NULL: kmean_bf16, kvar_bf16 and, for
 *     SA_TAIL_ZERO_ORDER, vmean_bf16 (= vsum / block).  Half the statistics
 *     bytes; the scores and the tail are computed in float32 from the bf16
 *     values.
 * block_idx_out: [B,Hkv,topk] int32 or NULL; scores_out: [B,Hkv,nb] float32
 * or NULL.  O: [B,Hq,d] of `dtype`.  workspace: device scratch of at least
 * sa_decode_workspace_size() bytes, 256-byte aligned; its contents on entry
 * do not matter.
 * Errors: SA_ERR_INVALID_ARG, SA_ERR_UNSUPPORTED, SA_ERR_ALIGNMENT,
 *         SA_ERR_WORKSPACE. */
sa_status sa_decode_fwd(const void* q, const void* Kcache, const void* Vcache, sa_dtype dtype,
                        sa_decode_shape shape, const sa_block_stats* stats, int32_t topk,
                        float scale, sa_tail_mode tail, int32_t* block_idx_out,
                        float* scores_out, void* O, void* workspace, size_t workspace_bytes,
                        void* stream);

/* Size of the scratch array that sa_decode_fwd_static uses: 8 MiB.  It holds
 * the route scores, the kept indices and the per-split partial states of one
 * call; the 16-sequence x 8-KV-head x 131072-token decode with topk 64 needs
 * about 7.1 MiB. */
#define SA_DECODE_STATIC_SCRATCH_BYTES (8u << 20)

/* sa_decode_fwd for callers that cannot allocate device memory.
 * Not part of the method: the pages have no counterpart to it.
 *
 * Some callers have no device allocator they may use: a plugin or
 * foreign-function host that only passes the tensors it was given and has no
 * way to request a workspace, or a serving loop that must not call cudaMalloc
 * because it can synchronise the whole device.  This entry point takes the
 * same arguments as sa_decode_fwd minus the workspace and allocates nothing:
 * its scratch is a static device array of SA_DECODE_STATIC_SCRATCH_BYTES that
 * every GPU loading the library holds until the process exits.  Inputs and
 * outputs are still the caller's.
 *   - A problem whose sa_decode_workspace_size() exceeds
 *     SA_DECODE_STATIC_SCRATCH_BYTES is rejected with SA_ERR_WORKSPACE before
 *     anything runs.
 *   - The first call in each CUDA context looks up the array's device
 *     address (cudaGetSymbolAddress, with that context current) and caches
 *     it under the context's unique id (cuCtxGetId).  A device's primary
 *     context is one such context; so is the new primary context after
 *     cudaDeviceReset and any context the caller creates and makes current,
 *     each with an array of its own.  Make the first call in a context before
 *     any stream capture in it.  Later calls in that context do no set-up.
 *   - Every call on a device shares the one array and it keeps the last
 *     call's contents (nothing in it needs clearing: each call writes every
 *     entry before reading it).  Calls whose executions overlap on the GPU
 *     (different streams, no ordering between them) race on the array and
 *     corrupt each other's results: serialise them.
 * Errors: as sa_decode_fwd, plus SA_ERR_WORKSPACE for a problem too large for
 * the static scratch and SA_ERR_CUDA if the symbol lookup fails. */
sa_status sa_decode_fwd_static(const void* q, const void* Kcache, const void* Vcache, sa_dtype dtype,
                               sa_decode_shape shape, const sa_block_stats* stats, int32_t topk,
                               float scale, sa_tail_mode tail, int32_t* block_idx_out,
                               float* scores_out, void* O, void* stream);

/* ---- Sparse feature attention ["Scaling Attention via Feature Sparsity",
 * §2: top-k feature codes of Q and K; FlashSFA's exact online softmax over
 * the overlap of the supports] ---------------------------------------------
 *
 * Sparse feature codes: for every row of X ([rows][d] bf16) the kf
 * coordinates of largest |x|, a tie in magnitude going to the smaller
 * channel index, in ascending channel order: vals [rows][kf] bf16 (signed
 * values), idx [rows][kf] uint8 (channels).  dense: [rows][d] bf16 or NULL;
 * when given, the zero-filled row (x at the kept channels, 0 elsewhere).
 * d in {64, 128}; 1 <= kf <= min(d, 32).  X and dense 16-byte aligned.
 * Errors: SA_ERR_INVALID_ARG, SA_ERR_UNSUPPORTED, SA_ERR_ALIGNMENT. */
sa_status sa_sfa_encode(const void* X, int64_t rows, int32_t d, int32_t kf, void* vals, uint8_t* idx,
                        void* dense, void* stream);

/* Zero-filled rows dense [rows][d] bf16 from codes (vals, idx) as written by
 * sa_sfa_encode (e.g. a key cache kept as codes).  Same limits. */
sa_status sa_sfa_densify(const void* vals, const uint8_t* idx, int64_t rows, int32_t d, int32_t kf,
                         void* dense, void* stream);

/* Bytes of workspace sa_sfa_attn_fwd needs (0 on a bad shape). */
size_t sa_sfa_workspace_size(sa_shape shape);

/* Sparse feature attention forward, non-causal: for every query row t,
 *   o_t = Σ_n e^{s a_tn} v_n / Σ_n e^{s a_tn},  a_tn = Σ_{c ∈ supp(q_t) ∩ supp(k_n)} q_tc k_nc,
 * which is the dot product of the zero-filled sparse rows.  Qs, Ks: the
 * zero-filled codes of Q and K ([B,H,N,d], from sa_sfa_encode or
 * sa_sfa_densify); V: [B,H,N,d] dense; all of `dtype`; O: [B,H,N,d] of
 * `dtype`.  shape.block is the tile of the online softmax (128 with d = 128
 * and bf16 takes the tensor-core kernel).  workspace: at least
 * sa_sfa_workspace_size(shape) bytes, 16-byte aligned.
 * Errors: SA_ERR_INVALID_ARG, SA_ERR_UNSUPPORTED, SA_ERR_ALIGNMENT,
 *         SA_ERR_WORKSPACE. */
sa_status sa_sfa_attn_fwd(const void* Qs, const void* Ks, const void* V, sa_dtype dtype, sa_shape shape,
                          float scale, void* O, void* workspace, size_t workspace_bytes, void* stream);

/* Reads and clears the library's device-side error word (synchronous: waits
 * for work already queued on the legacy default stream).  Non-zero means a
 * kernel gave up on an internal wait (bit 0: a bounded barrier wait timed
 * out, about two seconds) and returned without writing its output; the CUDA
 * context stays usable.  Kernels never trap on their own errors. */
sa_status sa_device_error(uint32_t* code);

/* Message for the last non-SA_OK status returned on the calling thread. */
const char* sa_last_error(void);

/* Library version string. */
const char* sa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SPARSEATTN_H */
