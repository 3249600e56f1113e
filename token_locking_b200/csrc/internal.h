// Internal declarations shared by the library's translation units.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>
#include <vector>

#include "surelock.h"

namespace sl {

// ------------------------------------------------------------------ errors --
sl_status fail(sl_status st, const char *fmt, ...);
sl_status cuda_fail(cudaError_t e, const char *what);
int *device_error_word();   // per-device int, allocated on first use; nullptr on failure
void note_launch(int n = 1); // count kernels launched by this library
long long launches_total();

#define SL_CUDA(call)                                  \
  do {                                                 \
    cudaError_t _e = (call);                           \
    if (_e != cudaSuccess) return ::sl::cuda_fail(_e, #call); \
  } while (0)

// Launch with programmatic stream serialisation (see pdl_wait/pdl_trigger).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                            cudaStream_t s, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  note_launch();
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// The same with a cluster of 2 CTAs along x (CTA pairs for 2-SM MMAs).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_k_cluster2(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                     cudaStream_t s, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  note_launch();
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ----------------------------------------------------- epilogue selection --
enum GemmEpi : int {
  EPI_STORE = 0,      // out[row_map ? row_map[r] : r][col_off + c] = acc   (dtype)
  EPI_RESID = 1,      // resid[r][c] += acc   (fp32; atomic when split over K)
  EPI_SWIGLU = 2,     // out[r][c] = silu(gate) * up      (dtype; tile = gate|up halves)
  EPI_ACCUM = 3,      // ws[r][col] += acc  (fp32 atomics, split-K workspace)
  EPI_QKV = 4,        // fused Q|K|V: RoPE(q) -> q_out[r], RoPE(k), v -> cache rows row_map[r]
  EPI_HEAD = 5        // LM head: as EPI_STORE (bf16 logits at rows row_map[r]) plus the sure
                      // test's statistics of each (row, vocab tile) on the stored values
};

// ------------------------------------------------------------------ layers.cu
// Out-of-range token ids embed as zeros and set DEV_BAD_INDEX in *err.
cudaError_t launch_gather_embed(int dtype, const int32_t *tokens, const int32_t *rows, int M,
                                const void *emb, int d, int vocab, float *h, int *err,
                                cudaStream_t s);
cudaError_t launch_rmsnorm(int dtype, const float *h, const void *g, int d, float eps, int M,
                           void *out, cudaStream_t s);
// qkv_in: [M][3d] (in_f32 ? float : dtype).  q_out [M][d] dtype; ck/cv: the layer's
// cache [B*n_ctx][d]; rope: [n_ctx][head_dim/2] (cos, sin).  zero_in: clear the
// fp32 input after reading (split-K workspace).
cudaError_t launch_rope_scatter(int dtype, const void *qkv_in, bool in_f32, bool zero_in, int M,
                                const int32_t *rows, int n_ctx, int n_heads, int head_dim,
                                const float2 *rope, void *q_out, void *ck, void *cv,
                                cudaStream_t s);
// act[r][c] = silu(ws[r][c]) * ws[r][F + c]; ws fp32 [M][2F] (zeroed after use) or dtype.
cudaError_t launch_swiglu(int dtype, const void *ws, bool in_f32, bool zero_in, int M, int F,
                          void *act, cudaStream_t s);
// fp32 SIMT GEMM: C = A[M,K] * B[N,K]^T with EPI_STORE (ldc, col_off, row_map) or EPI_RESID.
cudaError_t launch_gemm_f32(int epi, const float *A, int M, int K, const float *B, int N,
                            float *C, int ldc, int col_off, const int32_t *row_map,
                            cudaStream_t s);
// fp32 attention, head_dim <= 64: o[j] = softmax(q_j K_b^T / sqrt(dh)) V_b;
// with stamp non-null, over the keys n with stamp[b * n_ctx + n] == gen only.
cudaError_t launch_attn_f32(const float *q, const float *ck, const float *cv,
                            const int32_t *rows, int M, int n_ctx, int n_heads, int head_dim,
                            float *o, cudaStream_t s, const int32_t *stamp = nullptr,
                            int gen = 0);
// stamp[rows[j]] = gen for j < M: marks the active rows' keys visible.
cudaError_t launch_key_stamp(const int32_t *rows, int M, int gen, int32_t *stamp,
                             cudaStream_t s);

// -------------------------------------------------------------------- attn.cu
// Query tiles per sequence for the bf16 attention kernel.
struct AttnSeqs {
  int batch;
  int seq_start[SL_MAX_BATCH];   // first active-row index of the sequence
  int seq_count[SL_MAX_BATCH];   // active rows of the sequence
};
size_t attn_bf16_workspace_bytes(int max_rows, int n_heads, int max_splits);
// force_q (16/32/64) and force_splits (>= 1) pin the layout; 0 = cost model.
// [pf, pf + pf_bytes) is prefetched into L2 while the attention runs.
cudaError_t launch_attn_bf16(const void *q, const void *ck, const void *cv, const AttnSeqs &seqs,
                             int M, int n_ctx, int n_heads, void *o, float *ws, int max_splits,
                             int num_sms, cudaStream_t s, int force_q = 0,
                             int force_splits = 0, const void *pf = nullptr,
                             size_t pf_bytes = 0, const int32_t *stamp = nullptr,
                             int gen = 0);

// ----------------------------------------------------------------- attn_tc.cu
// Tensor-core attention (head_dim 128, bf16): q_map over q [M][d] with
// 128-row boxes, the layer's cache k/v [B*n_ctx][d] with 128-row boxes (for
// 128-key tiles) and 64-row boxes (for 64-key tiles); ws as for
// launch_attn_bf16; tickets [M][n_heads] zero
// between calls.  force_q 128 or 256 pins one or two query tiles per CTA,
// force_bn 64 or 128 the key tile (128 with one query tile only) and
// force_splits >= 1 the key split (0 = cost model).
struct TmaMat;
struct AttnTcPlan {
  int qt = 0, bn = 0, splits = 0, kt_per_split = 0, ktiles = 0, units = 0;
};
AttnTcPlan attn_tc_plan(const AttnSeqs &seqs, int n_heads, int n_ctx, int num_sms,
                        int max_splits, int force_q, int force_splits, int force_bn = 0);
size_t attn_tc_tickets_bytes(int max_rows, int n_heads);
cudaError_t launch_attn_tc(const TmaMat &q_map, const TmaMat &k_map128, const TmaMat &v_map128,
                           const TmaMat &k_map64, const TmaMat &v_map64, const AttnSeqs &seqs,
                           int M, int n_ctx, int n_heads, void *o, float *ws,
                           unsigned int *tickets, int max_splits, int num_sms, int *err,
                           unsigned long long wait_ns, cudaStream_t s, int force_q = 0,
                           int force_splits = 0, int force_bn = 0, const void *pf = nullptr,
                           size_t pf_bytes = 0, const int32_t *stamp = nullptr, int gen = 0);

// ----------------------------------------------------------------- gemm_tc.cu
// A bf16 K-major operand in global memory with its TMA descriptor.
struct TmaMat {
  CUtensorMap map;
  const void *ptr;
  int rows, cols;        // cols = K (contiguous)
  int box_rows;          // rows per TMA box
};
bool tma_encode(TmaMat *m, const void *ptr, int rows, int cols, int box_rows);
bool tma_encode_out(TmaMat *m, const void *ptr, int rows, int cols, int ld, bool f32);

struct TcGemmArgs {
  int epi;               // GemmEpi
  const TmaMat *A;       // activations [rows >= M][K]
  const TmaMat *B[3];    // weight segments, each [n_i][K]; SWIGLU: B[0]=gate, B[1]=up
  int n_seg[3];          // rows of each segment (STORE/ACCUM may use up to 3; others 1)
  int M, N, K;           // N = total output columns (SWIGLU: 2F)
  int splits;            // K splits (EPI_RESID / EPI_ACCUM only); -1: stream-K
  int bn;                // 64, 128 or 256
  int b_swiglu;          // B tile = BN/2 gate rows (B[0]) | BN/2 up rows (B[1])
  int msub;              // 1: 128-row units; 2: 256-row units (two accumulators per B tile)
  int pair;              // 1: CTA-pair kernel (2-SM MMA, 256-row units, B maps with BN/2 boxes)
  const TmaMat *OUT;     // RESID/ACCUM (fp32) or SWIGLU (bf16) output descriptor from
                         // tma_encode_out: tiles leave by TMA reduce-add / store (optional)
  void *out;             // STORE/SWIGLU: dtype out; RESID: fp32 resid; ACCUM: fp32 ws
  int ldo;               // leading dimension of out (elements)
  const int32_t *row_map;// STORE: output row index per A row (or null); QKV: flat positions
  // QKV: rotary table [n_ctx][64], q out [M][d], this layer's cache k/v [B*n_ctx][d]
  const float2 *rope;
  int n_ctx;
  void *q_out, *ck, *cv;
  // HEAD: previous step's logits (same row positions; null = no previous
  // posterior), per (row, vocab tile) records (max, sum e, sum e (z - z_prev),
  // best value) and best index over v != mask_id; records [M][N / bn]
  const void *prev;
  float4 *stat;
  int *stat_idx;
  int mask_id;
  // failure-detection test hooks: barrier wait limit in ns (0 = WAIT_LIMIT_NS),
  // and CTA 0 leaving out its first stage's operand copies (1-SM kernel only)
  unsigned long long wait_ns;
  int lost_load;
  // ACCUM split-K tile fix-up (see accum_fixup in gemm_tc.cu): tickets
  // [ceil(M / 32)][N / bn] zero between uses; QKV uses row_map, rope, n_ctx,
  // q_out, ck, cv; gate/up writes SiLU(gate) * up to fix_act [M][N / 2]
  unsigned int *fix_ctr;
  void *fix_act;
  // swapped operands (M <= 256, bn = 128, RESID / ACCUM): the weight tile is the
  // MMA's 128-row operand and the M rows its N dimension (gemm_swap_kernel)
  int swap;
};
cudaError_t launch_gemm_tc(const TcGemmArgs &a, int num_sms, int *err, cudaStream_t s);

// ------------------------------------------------------------------ lock.cu
struct LockStatsArgs {
  int dtype;
  const void *cur, *prev;        // [rows][V]
  const float *lse_prev;
  float *lse_cur;
  const int32_t *rows;           // active rows (flat positions)
  int M, V, mask_id, has_prev;
  float *kl, *unc, *conf;
  int32_t *argmax;
  float4 *part;                  // [M * splits * 2] partial records
  unsigned int *counters;        // [M], zero between calls
  int splits;
};
cudaError_t launch_lock_stats(const LockStatsArgs &a, cudaStream_t s);
int lock_stats_splits(int M, int V, int num_sms);

cudaError_t launch_lock_decide(const int32_t *seq_off, int batch, const int32_t *rows,
                               const float *kl, const float *unc, const uint8_t *masked,
                               float eps, float gate_q, int has_prev, int scripted_target,
                               uint8_t *lock, cudaStream_t s);
cudaError_t launch_compact(int32_t *rows, int32_t *seq_off, int batch, const uint8_t *lock,
                           uint8_t *locked, int32_t *lock_t, int step, cudaStream_t s);
cudaError_t launch_unmask(const int32_t *seq_off, int batch, const int32_t *rows, int n_ctx,
                          const float *conf, const int32_t *argmax, int lo, int hi, int k,
                          int32_t *tokens, uint8_t *masked, cudaStream_t s);
// Merge of the LM-head epilogue's per-tile records into the sure test's row
// statistics (the outputs of lock_stats): one warp per row.
cudaError_t launch_head_stats_merge(const float4 *stat, const int *stat_idx, int n_tiles,
                                    const int32_t *rows, int M, int has_prev,
                                    const float *lse_prev, float *lse_cur, float *kl, float *unc,
                                    float *conf, int32_t *argmax, cudaStream_t s);
cudaError_t launch_active_fill(int32_t *rows, int32_t *seq_off, int batch, int n_ctx,
                               cudaStream_t s);
// K/V reuse for active rows: the computed list of a step between refreshes,
// the reused rows' logits and lse carried forward, and the computed rows' lock
// flags mapped onto the active list.
cudaError_t launch_reuse_select(const int32_t *rows, const int32_t *seq_off, int batch,
                                const uint8_t *masked, const uint8_t *masked_before,
                                int32_t *out_rows, int32_t *out_off, cudaStream_t s);
cudaError_t launch_reuse_carry(const int32_t *rows, const int32_t *seq_off, int batch,
                               int m_active, const uint8_t *masked,
                               const uint8_t *masked_before, const void *prev, void *cur,
                               const float *lse_prev, float *lse_cur, size_t row_bytes,
                               cudaStream_t s);
cudaError_t launch_reuse_lock_map(const int32_t *c_rows, const int32_t *c_off,
                                  const uint8_t *c_lock, const int32_t *a_rows,
                                  const int32_t *a_off, int batch, uint8_t *by_pos,
                                  uint8_t *a_lock, cudaStream_t s);

}  // namespace sl
