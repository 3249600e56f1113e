/*
 * surelock.h -- C ABI of libsurelock.so: the SureLock decoding step on B200 (sm_100a).
 *
 * SureLock ("Stopping Computation for Converged Tokens in Masked Diffusion-LM
 * Decoding", Oba, Bollegala, Kaneko, Okazaki) keeps two disjoint sets of
 * positions while a masked diffusion LM denoises: the active set A_t, which the
 * denoiser computes, and the locked set L_t, whose rows skip the query
 * projection and the FFN but keep their attention keys/values cached so that
 * active rows still attend to them (Paper-Notes, "Method: overall framework" and
 * "Key design: permanent locking"; Abstract).  A position locks once its
 * posterior is stable: D_t = KL(p_t || p_{t-1}) <= eps at an unmasked position
 * (Paper-Notes, "lock criterion: step-to-step KL"; Abstract), optionally also
 * requiring u_t = 1 - max_v p_t(v) <= q_m(u_t), a quantile of u over the active
 * tokens (Paper-Notes, "optional confidence gate"; gist.science/it section 2,
 * "Filtro di Confidenza").  The active set only shrinks (Paper-Notes, "Key
 * findings").
 *
 * Conventions for every entry point:
 *  - Pointers named d_* are device pointers (cudaMalloc'd or torch-allocated on
 *    the current device); h_* are host pointers.  `stream` is a cudaStream_t
 *    passed as void* (NULL = the legacy default stream).
 *  - Work is enqueued asynchronously on `stream`.  Argument and state errors are
 *    detected on the host before anything is enqueued and return SL_ERR_INVALID
 *    or SL_ERR_STATE; CUDA launch errors return SL_ERR_CUDA.  sl_last_error()
 *    returns a message for the calling thread's last non-OK status.
 *  - Layouts are row-major.  Weights are [out_features, in_features].  Token
 *    positions of sequence b are b * n_ctx + i, i in [0, n_ctx).
 *  - Ownership: the caller owns weights, tokens, logits and per-row outputs;
 *    the model only borrows weight pointers (they must outlive it).  Objects
 *    created here (model, KV cache, active list, sampler) own their device
 *    memory and free it on destroy.
 *  - An object is used from one stream at a time.
 */
#ifndef SURELOCK_H
#define SURELOCK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SL_MAX_BATCH 64

typedef enum sl_status {
  SL_OK = 0,
  SL_ERR_INVALID = 1,     /* bad argument: null pointer, size out of range, unsupported shape */
  SL_ERR_CUDA = 2,        /* a CUDA runtime call or launch failed */
  SL_ERR_OOM = 3,         /* device or pinned allocation failed */
  SL_ERR_UNSUPPORTED = 4, /* valid request the library does not implement */
  SL_ERR_TIMEOUT = 5,     /* a kernel gave up a bounded wait and flagged it */
  SL_ERR_STATE = 6        /* call out of order (e.g. stepping a finished sampler) */
} sl_status;

typedef enum sl_dtype { SL_F32 = 0, SL_BF16 = 1 } sl_dtype;

/* Denoiser shape.  head_dim * n_heads must equal d_model.  dtype selects fp32
 * weights/activations/cache/logits (SIMT path) or bf16 (tensor-core path;
 * d_model, d_ffn and vocab must be multiples of 128, head_dim 128). */
typedef struct sl_config {
  int n_layers, d_model, n_heads, head_dim, d_ffn, vocab, mask_id;
  float rms_eps, rope_theta;
  int dtype; /* sl_dtype */
} sl_config;

/* One transformer block: RMSNorm gains [d], Wq/Wk/Wv/Wo [d, d], W_gate/W_up [f, d],
 * W_down [d, f]; all in the model dtype. */
typedef struct sl_layer_weights {
  const void *attn_norm, *wq, *wk, *wv, *wo, *ffn_norm, *w_gate, *w_up, *w_down;
} sl_layer_weights;

/* tok_emb [V, d], final_norm [d], lm_head [V, d]; layers: host array of n_layers. */
typedef struct sl_weights {
  const void *tok_emb, *final_norm, *lm_head;
  const sl_layer_weights *layers;
} sl_weights;

typedef struct sl_model sl_model;
typedef struct sl_kv_cache sl_kv_cache;
typedef struct sl_active sl_active;
typedef struct sl_sampler sl_sampler;

/* Message for the calling thread's last non-OK status (thread-local, owned by
 * the library; valid until the thread's next failing call; "" if none). */
const char *sl_last_error(void);
/* Library version string (static, owned by the library). */
const char *sl_version(void);

/* ---------------------------------------------------------------- model --- */

/* The denoiser whose steps the method runs on the active rows only: a
 * bidirectional masked-diffusion transformer (the pages evaluate LLaDA-8B;
 * Paper-Notes, "Method: overall framework": the model is applied to the
 * active set A_t while the locked set L_t is served from the cache).  The
 * pages give no model details beyond that; the layer layout here (RMSNorm,
 * rotary attention, SwiGLU FFN, untied LM head) is the LLaDA-style reading.
 * Borrows the caller's device weights (they must outlive the model; nothing
 * is copied) and builds the per-model launch state (TMA descriptors for the
 * bf16 path).  Fails with SL_ERR_INVALID on an inconsistent config (no work
 * is enqueued), SL_ERR_OOM if its small device state cannot be allocated. */
sl_status sl_model_create(const sl_config *cfg, const sl_weights *w, sl_model **out);
/* Frees the model's launch state (not the borrowed weights).  Caches and
 * samplers created from it must be destroyed first.  NULL is a no-op. */
void sl_model_destroy(sl_model *m);

/* --------------------------------------------------------------- KV cache --- */

/* The cache C of the pages (Paper-Notes, "permanent locking": K^all[L_t] <-
 * C.k[L_t]; gist.science/it section 2 "Azione di Blocco": K and V of a locked
 * token are kept for every layer).  Per layer, k and v are [batch][n_ctx][d_model]
 * in the model dtype (head h occupies columns h*head_dim .. +head_dim; k is stored
 * after the rotary embedding).  The object also owns the activation workspace
 * for up to batch * n_ctx active rows.  Contents start at zero. */
sl_status sl_kv_cache_create(const sl_model *m, int batch, int n_ctx, sl_kv_cache **out);
sl_status sl_kv_cache_reset(sl_kv_cache *c, void *stream);
/* Device pointers of layer `layer`'s k and v (for inspection and teacher forcing). */
sl_status sl_kv_cache_view(const sl_kv_cache *c, int layer, void **d_k, void **d_v);
void sl_kv_cache_destroy(sl_kv_cache *c);

/* ------------------------------------------------------------ active set --- */

/* The active set A_t of the pages (Paper-Notes, "Method: overall framework":
 * each step splits the positions into the active set A_t, which is computed,
 * and the locked set L_t, which is not; "permanent locking": a position never
 * leaves L_t, so A_t only shrinks).  For a batch: on the device, a flat
 * ascending list of positions rows[0..M) (entry b*n_ctx + i) and per-sequence
 * offsets seq_off[0..batch] (seq_off[batch] = M).  The host keeps a mirror of
 * the per-sequence counts, refreshed by sl_active_counts.  batch in
 * [1, SL_MAX_BATCH], n_ctx > 0, else SL_ERR_INVALID; SL_ERR_OOM if the device
 * or pinned buffers cannot be allocated.  Owns its memory (sl_active_destroy). */
sl_status sl_active_create(int batch, int n_ctx, sl_active **out);
/* A_0 = {0..n_ctx-1} for every sequence: at the first step nothing is locked
 * (Paper-Notes, "Method: overall framework"). */
sl_status sl_active_reset(sl_active *a, void *stream);
/* Teacher forcing: h_counts[batch], h_pos = the concatenated ascending local
 * positions (i in [0, n_ctx)) of every sequence.  SL_ERR_INVALID if a list is
 * not strictly ascending or out of range. */
sl_status sl_active_load(sl_active *a, const int32_t *h_counts, const int32_t *h_pos, void *stream);
/* Per-sequence counts |A_t^b| = M_t of the pages (Paper-Notes, "Key
 * findings": M_t falls monotonically over the decode) into h_counts[batch];
 * waits for the last update enqueued on the active set to finish. */
sl_status sl_active_counts(sl_active *a, int32_t *h_counts);
/* Device pointers of rows[] and seq_off[] (owned by the active set). */
sl_status sl_active_view(const sl_active *a, int32_t **d_rows, int32_t **d_seq_off);
void sl_active_destroy(sl_active *a);

/* --------------------------------------------------------- the hot path --- */

/* One denoiser pass on the active rows only (Abstract: locked positions skip
 * the query projection and FFN; attention cost O(M N d) instead of O(N^2 d),
 * gist.science/nl section 2 "Complexiteitsvermindering"):
 *   h = E[x[rows]]; per layer: a = RMSNorm(h); q,k,v = a Wq^T, a Wk^T, a Wv^T;
 *   RoPE(q, k) at the absolute position; C.k/C.v[layer][rows] <- k, v;
 *   h += Attn(q, C.k[layer][seq], C.v[layer][seq]) Wo^T  (all n_ctx keys);
 *   b = RMSNorm(h); h += (silu(b Wg^T) * (b Wu^T)) Wd^T;
 *   logits[rows] = RMSNorm(h) W_out^T.
 * d_tokens: [batch][n_ctx] int32 ids x_t.  d_logits: [batch][n_ctx][vocab] in the
 * model dtype; only the active rows are written.  The cache must have been
 * created for the same batch and n_ctx as the active set.  Under the
 * SL_ABLATE_NO_KV_CACHE ablation the attention sees the active rows' keys only. */
sl_status sl_step(sl_model *m, sl_kv_cache *c, sl_active *a, const int32_t *d_tokens,
                  void *d_logits, void *stream);

typedef struct sl_lock_params {
  float eps;             /* KL threshold; eps <= 0 disables locking */
  float gate_q;          /* confidence-gate quantile in [0,1]; < 0 = gate off */
  int has_prev;          /* 0 at t = 0: no previous posterior, nothing locks */
  int scripted_target;   /* < 0: the KL test.  >= 0: scripted mode, lock eligible
                            rows in ascending (D, position) order until each
                            sequence has this many active rows */
  int gate_only;         /* ablation (Paper-Notes, ablation table, "confidence gate
                            only"): lock_j = !masked[row_j] && has_prev &&
                            u_j <= thr_b, eps and D play no part; needs gate_q >= 0
                            (SL_ERR_INVALID otherwise).  Ignored in scripted mode. */
} sl_lock_params;

/* The sure test on the active rows (Paper-Notes, "lock criterion" and
 * "optional confidence gate"; Abstract: the test applies to positions that are
 * no longer masked):
 *   lse_j = logsumexp(z_cur[row_j]);  log p = z - lse
 *   D_j = max(0, sum_v p_cur (log p_cur - log p_prev))
 *       = max(0, E_pcur[z_cur - z_prev] - lse_cur + lse_prev)
 *   u_j = 1 - max_v p_cur(v);  conf_j / argmax_j over v != mask_id (lowest id on ties)
 *   thr_b = sorted(u over A_t^b)[floor(gate_q (M_b - 1))]
 *   lock_j = eps > 0 && !masked[row_j] && has_prev && D_j <= eps && (gate off || u_j <= thr_b)
 * d_logits_cur/prev: [batch*n_ctx][vocab] (dtype), read at the active rows;
 * d_lse_prev / d_lse_cur: [batch*n_ctx] fp32 (lse_cur written at active rows);
 * d_masked: [batch*n_ctx] u8 mask flags at the start of the step.
 * Outputs indexed by active-row index j in [0, M): d_kl, d_unc, d_conf (fp32),
 * d_argmax (int32), d_lock (u8).  Needs vocab % 8 == 0 for bf16. */
sl_status sl_kl_lock(sl_active *a, int vocab, int mask_id, int logits_dtype,
                     const void *d_logits_cur, const void *d_logits_prev,
                     const float *d_lse_prev, float *d_lse_cur, const uint8_t *d_masked,
                     const sl_lock_params *p, float *d_kl, float *d_unc, float *d_conf,
                     int32_t *d_argmax, uint8_t *d_lock, void *stream);

/* sl_step and the statistics half of sl_kl_lock in one pass: the LM-head GEMM
 * rounds each logit to the model dtype, stores it at its row as sl_step does,
 * and in the same epilogue takes, per (row, vocab tile), the running max, the
 * sum of exp(z - max), the sum of exp(z - max) (z - z_prev) against
 * d_logits_prev and the best value over v != mask_id; a per-row merge then
 * writes lse_cur, D, u, conf and argmax exactly as sl_kl_lock defines them, on
 * the stored logits, without reading them back.  This fuses the LM head with
 * the sure test, which the pages name as future work (gist.science/nl section
 * 5: fused kernels; gist.science/it section 4: kernel fusion to turn the FLOP
 * savings into wall-clock).  Arguments as sl_step and sl_kl_lock: d_logits_prev
 * and d_lse_prev [batch*n_ctx][vocab] / [batch*n_ctx] are read at the active
 * rows when has_prev (otherwise they may be NULL and D = +inf); outputs d_kl,
 * d_unc, d_conf, d_argmax by active-row index, d_lse_cur at the rows'
 * positions.  fp32 models run sl_step followed by a separate statistics pass
 * (same results).  Follow with sl_lock_decide for the lock flags. */
sl_status sl_step_stats(sl_model *m, sl_kv_cache *c, sl_active *a, const int32_t *d_tokens,
                        void *d_logits, const void *d_logits_prev, const float *d_lse_prev,
                        int has_prev, float *d_lse_cur, float *d_kl, float *d_unc,
                        float *d_conf, int32_t *d_argmax, void *stream);

/* The decision half of sl_kl_lock, from statistics already computed (by
 * sl_step_stats or sl_kl_lock): per sequence the gate threshold
 * thr_b = sorted(u over A_t^b)[floor(gate_q (M_b - 1))], then
 * lock_j = eps > 0 && !masked[row_j] && has_prev && D_j <= eps && (gate off ||
 * u_j <= thr_b), or the scripted / gate-only variants of sl_lock_params
 * (Paper-Notes, "lock criterion" and "optional confidence gate").  d_kl, d_unc
 * and d_lock are indexed by active-row index. */
sl_status sl_lock_decide(sl_active *a, const uint8_t *d_masked, const sl_lock_params *p,
                         const float *d_kl, const float *d_unc, uint8_t *d_lock, void *stream);

/* Sampler step: among the masked active rows with local position in
 * [block_lo, block_hi), unmask the k with the highest confidence (ties to the
 * lower position): tokens[row] = argmax, masked[row] = 0.  This is the
 * unmodified sampler the pages compare against (Abstract: the baseline is this
 * sampler with locking switched off). */
sl_status sl_unmask_topk(sl_active *a, const float *d_conf, const int32_t *d_argmax,
                         int block_lo, int block_hi, int k, int32_t *d_tokens,
                         uint8_t *d_masked, void *stream);

/* Stable compaction: A_{t+1} = [row_j in A_t : !lock_j] in ascending order, and
 * locked[row] = 1, lock_t[row] = step for each locked row (Paper-Notes,
 * "permanent locking": the active set only shrinks).  d_lock is indexed by
 * active-row index; d_locked/d_lock_t are [batch*n_ctx]. */
sl_status sl_compact_active(sl_active *a, const uint8_t *d_lock, uint8_t *d_locked,
                            int32_t *d_lock_t, int step, void *stream);

/* One transformer block of layer `layer` on the active rows, the body of
 * sl_step's layer loop: d_h [M][d_model] fp32 holds the block inputs of the
 * active rows (in active-list order) and is overwritten with the block outputs;
 * C.k/C.v[layer] rows of the active positions receive the fresh k, v.  Frozen
 * block inputs of locked rows are never touched (gist.science/it section 2,
 * "Azione di Blocco"). */
sl_status sl_layer_forward(sl_model *m, sl_kv_cache *c, sl_active *a, int layer, float *d_h,
                           void *stream);

/* Attention of the active rows over all n_ctx cached keys of their sequence in
 * layer `layer` (over the active rows' keys only under SL_ABLATE_NO_KV_CACHE):
 * d_q [M][d_model] (after the rotary embedding), d_o [M][d_model], both in the
 * model dtype. */
sl_status sl_attention(sl_model *m, sl_kv_cache *c, sl_active *a, int layer, const void *d_q,
                       void *d_o, void *stream);

/* The tensor-core GEMM of the bf16 path, C = A[M,K] * B[N,K]^T (bf16 operands,
 * fp32 accumulation), exposed for kernel-level checks and benchmarks.
 *   SL_GEMM_STORE : out bf16 [.][ldo], row r written to row d_row_map[r] (or r)
 *   SL_GEMM_RESID : out fp32 [M][ldo] += C (added in L2 by TMA reduce-add)
 *   SL_GEMM_SWIGLU: d_b = W_gate [F][K], d_b2 = W_up [F][K], N = 2F;
 *                   out bf16 [M][ldo] = silu(A W_gate^T) * (A W_up^T)
 *   SL_GEMM_ACCUM : out fp32 [M][ldo] += C (atomic; with d_b2, gate/up halves
 *                   accumulate into columns [0,F) and [F,2F))
 * bn (64/128/192/256) and splits (>= 1, RESID/ACCUM only; -1 = stream-K: every SM
 * or CTA pair takes an equal share of the tiles x 64-wide K-blocks and adds
 * its partial tiles atomically) pick the tiling; variant
 * picks the kernel: 0 = one CTA per 128 x bn tile, 1 = one CTA per 256 x bn
 * tile (two accumulators share each weight tile), 2 = a CTA pair per 256 x bn
 * tile with 2-SM tensor-core instructions (bn 128, 192 or 256), 3 = swapped
 * operands for few rows (M <= 256, bn 128, splits >= 1, RESID or ACCUM): each
 * CTA multiplies 128 weight rows by all M rows (C^T = B A^T, the tensor-core
 * work following M rounded up to 32 instead of a padded 256-row tile) and adds
 * the transposed tile into out.  bn = 0 lets the library choose everything.  K % 64 == 0, N % bn == 0, pointers 16-byte
 * aligned, ldo >= the output columns (N, or F for SWIGLU) with 16-byte rows
 * (ldo % 4 == 0 for fp32 outputs, % 8 for bf16); SL_ERR_INVALID otherwise. */
enum { SL_GEMM_STORE = 0, SL_GEMM_RESID = 1, SL_GEMM_SWIGLU = 2, SL_GEMM_ACCUM = 3 };
sl_status sl_gemm_bf16(int epi, const void *d_a, int M, int K, const void *d_b, const void *d_b2,
                       int N, void *d_out, int ldo, const int32_t *d_row_map, int bn, int splits,
                       int variant, void *stream);

/* The per-row statistics of sl_kl_lock (lse, D, u, conf, argmax; no gate and
 * no lock flags) for callers that cannot allocate device memory: hosts whose
 * device memory is owned by another runtime's pool (a serving engine that
 * reserves nearly all of HBM at start-up, so cudaMalloc would fail), and code
 * that must not trigger cudaMalloc's implicit device synchronisation.  It
 * allocates nothing: the split-reduction scratch is a static device array
 * built into this library (about 560 KB per GPU that loads it, kept until the
 * process exits).  The pages have no counterpart; this is a library-level
 * entry point.
 *   d_rows [M]: flat positions of the rows to test, as in sl_active.
 *   Outputs as sl_kl_lock: d_kl, d_unc, d_conf, d_argmax by row index j,
 *   d_lse_cur at position d_rows[j].  has_prev = 0 writes D = +inf.
 * Limits: 0 <= M <= 8192 (SL_ERR_INVALID otherwise); vocab % 8 == 0.
 * The first call on a device looks up the scratch array's device address
 * (cudaGetSymbolAddress, once per device); make that first call before any
 * stream capture.  All calls share the one scratch array, so calls whose
 * kernels overlap on the GPU (other streams, other threads) race and corrupt
 * each other's results: serialise them. */
sl_status sl_kl_stats_noalloc(const int32_t *d_rows, int M, int vocab, int mask_id,
                              int logits_dtype, const void *d_logits_cur,
                              const void *d_logits_prev, const float *d_lse_prev,
                              float *d_lse_cur, int has_prev, float *d_kl, float *d_unc,
                              float *d_conf, int32_t *d_argmax, void *stream);

/* Autotune the tensor-core GEMM tilings of this model on this device: every
 * valid (tile width, 128/256-row tiles, K split) of the five projection GEMMs
 * (fused QKV, output projection, fused gate/up, down projection, LM head) is
 * timed at each row-count bucket up to max_rows, and later sl_step /
 * sl_layer_forward calls use the fastest (untuned sizes use an analytic cost
 * model).  Runs synchronously on `stream` (seconds at most); overwrites the
 * cache's KV and workspace contents, so call it before a decode starts.
 * A no-op for fp32 models. */
sl_status sl_model_autotune(sl_model *m, sl_kv_cache *c, int max_rows, void *stream);
/* The tiling sl_step would use for GEMM `kind` (0 QKV, 1 output projection,
 * 2 gate/up, 3 down, 4 LM head) at M rows; *splits and *variant as for
 * sl_gemm_bf16. */
sl_status sl_model_tuning(const sl_model *m, int kind, int M, int *bn, int *splits, int *variant);
/* Pin the attention layout of sl_step / sl_attention on this model:
 * queries_per_cta 128 or 256 (the tensor-core kernel with one or two 128-query
 * tiles per CTA), or 16, 32 or 64 (the mma.sync kernel; its four warps then
 * split every 64-key tile 4, 2 or 1 ways), and the split of the key range
 * across CTAs (1..16, rounded so that every split holds key tiles); 0 leaves
 * either to the library's cost model (the tensor-core kernel).
 * SL_ERR_INVALID for other values. */
sl_status sl_model_set_attention(sl_model *m, int queries_per_cta, int splits);
/* Pin the key tile of the tensor-core attention (queries_per_cta 0, 128 or
 * 256): 64 or 128 keys per tile (128 with one query tile per CTA only; a pin
 * that no layout satisfies makes the step fail with SL_ERR_CUDA), 0 = cost
 * model.  SL_ERR_INVALID for other values. */
sl_status sl_model_set_attention_keys(sl_model *m, int key_tile);
/* Pin the tiling of GEMM `kind` for the row-count bucket that holds M (the
 * buckets of sl_model_autotune); arguments as for sl_gemm_bf16.  Returns
 * SL_ERR_INVALID for a tiling the GEMM cannot use (the LM head takes no K
 * split and no swapped operands; swapped operands need a bucket of at most 256
 * rows).  bf16 models only. */
sl_status sl_model_set_tuning(sl_model *m, int kind, int M, int bn, int splits, int variant);

/* Ablations of the method (Paper-Notes, ablation table), a bit set; 0 (the
 * default) is the method itself.
 *   SL_ABLATE_NO_KV_CACHE  "no KV cache": the queries of sl_step, sl_layer_forward
 *       and sl_attention attend to the keys of their sequence's active rows only;
 *       the cached K/V of locked rows are not read.  Same FLOPs, locked tokens'
 *       information is lost to the active ones.
 *   SL_ABLATE_GATE_ONLY    "confidence gate only": the model's samplers lock with
 *       the gate alone (sl_lock_params.gate_only); the sampler then needs
 *       gate_q >= 0, else sl_sampler_step returns SL_ERR_INVALID.
 * Unknown bits: SL_ERR_INVALID.  Takes effect from the next call on the model. */
#define SL_ABLATE_NO_KV_CACHE 1
#define SL_ABLATE_GATE_ONLY 2
sl_status sl_model_set_ablation(sl_model *m, int flags);

/* Whether this model's samplers take the sure test's statistics from the LM
 * head's epilogue (sl_step_stats; enable = 1, the default) or from a separate
 * pass over the stored logits (sl_step then sl_kl_lock; enable = 0).  Same
 * results either way; a switch for comparing the two. */
sl_status sl_model_set_head_fusion(sl_model *m, int enable);

/* ---------------------------------------------------------------- sampler --- */

/* Semi-autoregressive SureLock decode driven by the library: prompt_len given
 * tokens then gen_len [MASK] tokens; gen region split in blocks of block_len,
 * steps/(gen_len/block_len) steps per block, tokens_per_step unmasked per step
 * (the unmodified sampler the pages compare against, Abstract: their baseline
 * is this sampler with locking switched off; here the sure test of sl_kl_lock
 * runs between steps). */
typedef struct sl_sampler_params {
  int prompt_len, gen_len, steps, block_len, tokens_per_step;
  float eps;             /* KL threshold; eps <= 0 disables locking */
  float gate_q;          /* confidence-gate quantile in [0,1]; < 0 = gate off */
  int scripted;          /* 1: scripted lock schedule, M decays linearly to 10% of N */
} sl_sampler_params;

/* Device buffers owned by a sampler (for inspection / teacher forcing). */
typedef struct sl_sampler_state {
  int32_t *tokens;       /* [B][N] */
  uint8_t *masked;       /* [B][N] */
  uint8_t *locked;       /* [B][N] */
  int32_t *lock_t;       /* [B][N], -1 if unlocked */
  void *logits[2];       /* [B][N][V] ping-pong, step t writes logits[t % 2] */
  float *lse[2];         /* [B][N] */
  float *kl, *unc, *conf;/* [B*N] by the index of the rows the step computed */
  int32_t *argmax;       /* [B*N] */
  uint8_t *lock;         /* [B*N] */
  sl_kv_cache *cache;
  sl_active *active;
  int t;                 /* next step to run */
  int batch, n_ctx;
  sl_active *computed;   /* K/V reuse on: the rows the last step between refreshes
                            computed (refresh steps compute `active` and leave it
                            as it was); NULL if reuse was never switched on */
} sl_sampler_state;

/* Creates a sampler for `batch` sequences (1..SL_MAX_BATCH) of n_ctx =
 * prompt_len + gen_len positions, with its own KV cache, active set, token,
 * flag and logit buffers (two [batch][n_ctx][vocab] logit buffers in the model
 * dtype).  SL_ERR_INVALID if gen_len does not split into blocks or steps into
 * blocks, or gate_q > 1; SL_ERR_UNSUPPORTED for block_len > 2048; SL_ERR_OOM if
 * the buffers do not fit.  The model must outlive the sampler. */
sl_status sl_sampler_create(sl_model *m, int batch, const sl_sampler_params *p, sl_sampler **out);
/* Reset state for a new decode from device prompts [batch][prompt_len]. */
sl_status sl_sampler_start(sl_sampler *s, const int32_t *d_prompts, void *stream);
/* SureLock composed with cross-step K/V reuse for the active rows, which the
 * pages call orthogonal to locking and stackable with it (Paper-Notes,
 * "permanent locking" design motivation, where dLLM-Cache is the per-step
 * selective counterpart, and "loss / training strategy"; gist.science/it
 * section 4, "Ortogonalita"); the scheme is this library's reading:
 * period R = 1 (the default) is SureLock alone.  With R > 1, step t computes
 * all active rows when t mod R = 0 (a refresh step).  Between refreshes it
 * computes the active rows that are masked, or were masked at the start of the
 * previous step (so a row is computed once more after its unmasking); each
 * other active row keeps its cached K/V, its last logits and lse (carried into
 * the step's logit buffer), is not tested and stays active.  The sure test,
 * the confidence gate's quantile and the unmasking run over the computed rows;
 * kl, unc, conf, argmax and lock are indexed by them.  The first call with
 * R > 1 allocates a second active list and 3 bytes per position.
 * SL_ERR_INVALID: R < 1, or R > 1 on a scripted sampler (its lock count is
 * defined over the whole active set); SL_ERR_STATE while a decode is in
 * progress (started and t < steps); SL_ERR_OOM.  sl_sampler_step returns
 * SL_ERR_INVALID if R > 1 and the model has the no-KV-cache ablation. */
sl_status sl_sampler_set_kv_reuse(sl_sampler *s, int period);
/* One denoising step t: sl_step_stats and sl_lock_decide (or sl_step and
 * sl_kl_lock, see sl_model_set_head_fusion), sl_unmask_topk, sl_compact_active
 * (with K/V reuse, on the computed rows; see sl_sampler_set_kv_reuse). */
sl_status sl_sampler_step(sl_sampler *s, void *stream);
/* Whole decode from host prompts [batch][prompt_len] to host tokens
 * [batch][n_ctx]; both copies are inside the call. */
sl_status sl_sampler_generate(sl_sampler *s, const int32_t *h_prompts, int32_t *h_tokens,
                              void *stream);
/* The sampler's buffers and step counter; the pointers stay owned by the
 * sampler and valid until it is destroyed. */
sl_status sl_sampler_get_state(const sl_sampler *s, sl_sampler_state *out);
void sl_sampler_destroy(sl_sampler *s);

/* ------------------------------------------------------------ diagnostics --- */

/* Per kernel class device time, measured with CUDA events around every launch
 * of that class while timing is enabled on the model, and the algorithmic work
 * of those launches (bytes: operands read + results written once; flops:
 * 2 per multiply-add). */
enum { SL_K_GEMM = 0, SL_K_ATTN = 1, SL_K_LOCK = 2, SL_K_OTHER = 3, SL_K_COUNT = 4 };
typedef struct sl_timing {
  double ms[SL_K_COUNT];
  double bytes[SL_K_COUNT];
  double flops[SL_K_COUNT];
  long long launches[SL_K_COUNT];
  long long kernels;     /* kernels this library launched (all classes, all objects) */
} sl_timing;
sl_status sl_timing_enable(sl_model *m, int enable);
/* Synchronises the recorded events, returns the sums since the last reset. */
sl_status sl_timing_read(sl_model *m, sl_timing *out, int reset);

/* Device error word, set by a kernel that gave up a bounded wait or met a
 * token id outside [0, vocab) (that row is embedded as zeros, never read from
 * out of range): returns SL_ERR_TIMEOUT or SL_ERR_STATE respectively (and
 * clears the word if `clear`), SL_OK if nothing was recorded.  Synchronises
 * the device. */
sl_status sl_device_check(int clear);

/* Test hooks for the failure path of the bounded waits.  Neither raises a GPU
 * fault: they only make a wait run out, after which the kernel records
 * SL_ERR_TIMEOUT in the device error word, drains its copies, frees its TMEM
 * and returns, and the context stays usable.
 *   sl_debug_set_wait_limit: every later tensor-core GEMM and attention launch
 *     (sl_step, sl_step_stats, sl_layer_forward, sl_attention, sl_gemm_bf16,
 *     autotuning) gives up a barrier wait after `ns` nanoseconds instead of
 *     the default 2 s; 0 restores the default.
 *     SL_ERR_INVALID outside [1 ms, 2 s].  Process-wide.
 *   sl_debug_inject_lost_load: the next tensor-core GEMM launch on the 1-SM
 *     kernels has its first CTA leave out the operand copies of its first
 *     pipeline stage, so the MMA warp's wait for them runs out (one-shot). */
sl_status sl_debug_set_wait_limit(unsigned long long ns);
sl_status sl_debug_inject_lost_load(void);

#ifdef __cplusplus
}
#endif
#endif /* SURELOCK_H */
