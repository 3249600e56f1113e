// Row-wise kernels of the denoiser on the active rows, and the fp32 SIMT
// GEMM/attention used by fp32 models.
//
// The gather, norm, rotary, scatter and SwiGLU kernels are memory-bound: one
// CTA per active row, 16-byte vector accesses on the bf16 path.
#include "common.cuh"
#include "internal.h"

namespace sl {

// ---------------------------------------------------------------- gather ---
// h[j, :] = E[tokens[rows[j]], :]  (fp32 residual stream).  Only the M active
// rows are embedded: locked rows keep a frozen block input and are not
// recomputed (gist.science/it section 2, "Azione di Blocco").
// A token id outside [0, vocab) is never used as an address: the row is
// embedded as zeros and DEV_BAD_INDEX goes into the device error word (the
// first error wins), which sl_device_check reports.
template <typename T>
__global__ void gather_embed_kernel(const int32_t *__restrict__ tokens,
                                    const int32_t *__restrict__ rows, int M,
                                    const T *__restrict__ emb, int d, int vocab,
                                    float *__restrict__ h, int *__restrict__ err) {
  int j = blockIdx.x;
  if (j >= M) return;
  pdl_wait();
  pdl_trigger();
  const int tok = tokens[rows[j]];
  float *o = h + (size_t)j * d;
  if (tok < 0 || tok >= vocab) {
    if (threadIdx.x == 0 && err) atomicCAS(err, DEV_OK, DEV_BAD_INDEX);
    for (int c = threadIdx.x; c < d; c += blockDim.x) o[c] = 0.f;
    return;
  }
  const T *e = emb + (size_t)tok * d;
  for (int c = threadIdx.x; c < d; c += blockDim.x) o[c] = to_f(e[c]);
}

cudaError_t launch_gather_embed(int dtype, const int32_t *tokens, const int32_t *rows, int M,
                                const void *emb, int d, int vocab, float *h, int *err,
                                cudaStream_t s) {
  cudaError_t e = cudaSuccess;
  if (M <= 0) return cudaSuccess;
  if (dtype == SL_BF16) {
    e = launch_k(gather_embed_kernel<bf16>, M, 256, 0, s, tokens, rows, M, (const bf16 *)emb, d,
                 vocab, h, err);
  } else {
    e = launch_k(gather_embed_kernel<float>, M, 256, 0, s, tokens, rows, M, (const float *)emb, d,
                 vocab, h, err);
  }
  return e;
}

// --------------------------------------------------------------- rmsnorm ---
// out = h / sqrt(mean(h^2) + eps) * g, rounded to the model dtype.
template <typename T>
__global__ void rmsnorm_kernel(const float *__restrict__ h, const T *__restrict__ g, int d,
                               float eps, int M, T *__restrict__ out) {
  int j = blockIdx.x;
  if (j >= M) return;
  pdl_wait();
  pdl_trigger();
  const float *x = h + (size_t)j * d;
  float ss = 0.f;
  for (int c = threadIdx.x; c < d; c += blockDim.x) ss += x[c] * x[c];
  __shared__ float red[32];
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    v = warp_sum(v);
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  float r = rsqrtf(red[0] / (float)d + eps);
  T *o = out + (size_t)j * d;
  for (int c = threadIdx.x; c < d; c += blockDim.x) o[c] = from_f<T>(x[c] * r * to_f(g[c]));
}

// bf16 output: one CTA of 256 threads per row, the row held in registers as
// VPT float4 per thread, so the row is read once and the sum of squares needs a
// single block reduction.
template <int VPT>
__global__ void __launch_bounds__(256) rmsnorm_bf16_kernel(const float *__restrict__ h,
                                                           const bf16 *__restrict__ g, int d,
                                                           float eps, int M,
                                                           bf16 *__restrict__ out) {
  const int j = blockIdx.x;
  if (j >= M) return;
  pdl_wait();
  pdl_trigger();
  const float4 *x = reinterpret_cast<const float4 *>(h + (size_t)j * d);
  const int n4 = d >> 2;
  float4 v[VPT];
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < VPT; ++k) {
    const int i = threadIdx.x + k * 256;
    v[k] = i < n4 ? x[i] : make_float4(0.f, 0.f, 0.f, 0.f);
    ss += v[k].x * v[k].x + v[k].y * v[k].y + v[k].z * v[k].z + v[k].w * v[k].w;
  }
  __shared__ float red[8];
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) tot += red[w];
  const float r = rsqrtf(tot / (float)d + eps);
  const uint2 *g2 = reinterpret_cast<const uint2 *>(g);
  uint2 *o2 = reinterpret_cast<uint2 *>(out + (size_t)j * d);
#pragma unroll
  for (int k = 0; k < VPT; ++k) {
    const int i = threadIdx.x + k * 256;
    if (i < n4) {
      union { uint2 u; __nv_bfloat162 b[2]; } gg, oo;
      gg.u = g2[i];
      const float2 g0 = __bfloat1622float2(gg.b[0]), g1 = __bfloat1622float2(gg.b[1]);
      oo.b[0] = __floats2bfloat162_rn(v[k].x * r * g0.x, v[k].y * r * g0.y);
      oo.b[1] = __floats2bfloat162_rn(v[k].z * r * g1.x, v[k].w * r * g1.y);
      o2[i] = oo.u;
    }
  }
}

cudaError_t launch_rmsnorm(int dtype, const float *h, const void *g, int d, float eps, int M,
                           void *out, cudaStream_t s) {
  if (dtype == SL_BF16 && d % 4 == 0 && d <= 8 * 1024) {
    if (M <= 0) return cudaSuccess;
    const int vpt = (d / 4 + 255) / 256;
    const bf16 *gb = (const bf16 *)g;
    bf16 *ob = (bf16 *)out;
    if (vpt <= 1) return launch_k(rmsnorm_bf16_kernel<1>, M, 256, 0, s, h, gb, d, eps, M, ob);
    if (vpt <= 2) return launch_k(rmsnorm_bf16_kernel<2>, M, 256, 0, s, h, gb, d, eps, M, ob);
    if (vpt <= 4) return launch_k(rmsnorm_bf16_kernel<4>, M, 256, 0, s, h, gb, d, eps, M, ob);
    return launch_k(rmsnorm_bf16_kernel<8>, M, 256, 0, s, h, gb, d, eps, M, ob);
  }
  cudaError_t err = cudaSuccess;
  if (M <= 0) return cudaSuccess;
  int th = d >= 1024 ? 512 : 128;
  if (dtype == SL_BF16) {
    err = launch_k(rmsnorm_kernel<bf16>, M, th, 0, s, h, (const bf16 *)g, d, eps, M, (bf16 *)out);
  } else {
    err = launch_k(rmsnorm_kernel<float>, M, th, 0, s, h, (const float *)g, d, eps, M, (float *)out);
  }
  return err;
}

// ------------------------------------------------------- rotary + scatter ---
// From the projection output [M][3d] (q | k | v): q_out[j] = RoPE(q_j),
// C.k[rows[j]] = RoPE(k_j), C.v[rows[j]] = v_j.  RoPE is rotate-half on the
// pair (i, i + dh/2) at the absolute position rows[j] % n_ctx; the (cos, sin)
// table is precomputed in double precision on the host.  Writing the fresh k,v
// of active rows into the cache is the "K^all[A_t]" half of the pages'
// K^all[L_t] <- C.k[L_t] (Paper-Notes, "permanent locking").  One thread per
// (row, pair) so that a few rows still spread over every SM; used after a
// split-K projection (input = the fp32 partial-sum workspace, cleared here for
// the next split-K GEMM) and on the fp32 path.
template <typename Tin, typename T>
__global__ void __launch_bounds__(256) rope_scatter_kernel(
    Tin *__restrict__ qkv, bool zero_in, int M, const int32_t *__restrict__ rows, int n_ctx,
    int n_heads, int dh, const float2 *__restrict__ rope, T *__restrict__ q_out,
    T *__restrict__ ck, T *__restrict__ cv) {
  // grid: x = chunks of 256 pairs within a row (3 * d / 2 pairs), y = row
  const int j = blockIdx.y;
  const int d = n_heads * dh;
  const int half = dh >> 1;
  const int per_seg = d >> 1;
  const int pr_all = blockIdx.x * 256 + threadIdx.x;
  pdl_wait();
  pdl_trigger();
  if (pr_all < 3 * per_seg) {
    const int seg = pr_all / per_seg;
    const int pr = pr_all - seg * per_seg;
    const int hh = pr / half, i = pr - hh * half;
    const int c0 = hh * dh + i, c1 = c0 + half;
    Tin *in = qkv + (size_t)j * 3 * d + seg * d;
    const float x0 = to_f(in[c0]), x1 = to_f(in[c1]);
    if (zero_in) {
      in[c0] = Tin(0.f);
      in[c1] = Tin(0.f);
    }
    const int p = rows[j];
    T *dst = seg == 0 ? q_out + (size_t)j * d : (seg == 1 ? ck : cv) + (size_t)p * d;
    if (seg < 2) {
      const float2 cs = rope[(size_t)(p % n_ctx) * half + i];
      dst[c0] = from_f<T>(x0 * cs.x - x1 * cs.y);
      dst[c1] = from_f<T>(x1 * cs.x + x0 * cs.y);
    } else {
      dst[c0] = from_f<T>(x0);
      dst[c1] = from_f<T>(x1);
    }
  }
}

// The same from the fp32 split-K workspace into bf16, eight pairs per thread:
// 16-byte loads of both halves, the (cos, sin) table and the clearing stores,
// 16-byte bf16 stores (head_dim % 16 == 0).
__global__ void __launch_bounds__(256) rope_scatter_ws_kernel(
    float *__restrict__ ws, int M, const int32_t *__restrict__ rows, int n_ctx, int n_heads,
    int dh, const float2 *__restrict__ rope, bf16 *__restrict__ q_out, bf16 *__restrict__ ck,
    bf16 *__restrict__ cv) {
  const int j = blockIdx.y;
  const int d = n_heads * dh;
  const int half = dh >> 1;
  const int groups = half >> 3;                      // 8-pair groups per head
  const int t = blockIdx.x * 256 + threadIdx.x;      // (segment, head, group)
  pdl_wait();
  pdl_trigger();
  if (t >= 3 * n_heads * groups) return;
  const int seg = t / (n_heads * groups);
  const int rem = t - seg * n_heads * groups;
  const int hh = rem / groups, i0 = (rem - hh * groups) * 8;
  const int c0 = hh * dh + i0, c1 = c0 + half;
  float4 *in0 = reinterpret_cast<float4 *>(ws + (size_t)j * 3 * d + seg * d + c0);
  float4 *in1 = reinterpret_cast<float4 *>(ws + (size_t)j * 3 * d + seg * d + c1);
  const float4 a0 = in0[0], a1 = in0[1], b0 = in1[0], b1 = in1[1];
  const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
  in0[0] = z;
  in0[1] = z;
  in1[0] = z;
  in1[1] = z;
  const float x0[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
  const float x1[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
  const int p = rows[j];
  bf16 *dst = seg == 0 ? q_out + (size_t)j * d : (seg == 1 ? ck : cv) + (size_t)p * d;
  Pack8 lo, hi;
  if (seg < 2) {
    const float4 *tab = reinterpret_cast<const float4 *>(rope + (size_t)(p % n_ctx) * half + i0);
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      const float4 cs = tab[e >> 1];                 // (cos, sin) of pairs e and e + 1
      lo.h[e] = __float2bfloat16_rn(x0[e] * cs.x - x1[e] * cs.y);
      hi.h[e] = __float2bfloat16_rn(x1[e] * cs.x + x0[e] * cs.y);
      lo.h[e + 1] = __float2bfloat16_rn(x0[e + 1] * cs.z - x1[e + 1] * cs.w);
      hi.h[e + 1] = __float2bfloat16_rn(x1[e + 1] * cs.z + x0[e + 1] * cs.w);
    }
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      lo.h[e] = __float2bfloat16_rn(x0[e]);
      hi.h[e] = __float2bfloat16_rn(x1[e]);
    }
  }
  *reinterpret_cast<uint4 *>(dst + c0) = lo.u;
  *reinterpret_cast<uint4 *>(dst + c1) = hi.u;
}

cudaError_t launch_rope_scatter(int dtype, const void *qkv_in, bool in_f32, bool zero_in, int M,
                                const int32_t *rows, int n_ctx, int n_heads, int head_dim,
                                const float2 *rope, void *q_out, void *ck, void *cv,
                                cudaStream_t s) {
  if (M <= 0) return cudaSuccess;
  if (M > 65535) return cudaErrorInvalidValue;
  if (dtype == SL_BF16 && in_f32 && zero_in && head_dim % 16 == 0) {
    const int threads = 3 * n_heads * (head_dim / 16);
    return launch_k(rope_scatter_ws_kernel, dim3((threads + 255) / 256, M), 256, 0, s,
                    (float *)qkv_in, M, rows, n_ctx, n_heads, head_dim, rope, (bf16 *)q_out,
                    (bf16 *)ck, (bf16 *)cv);
  }
  const dim3 grid((3 * n_heads * head_dim / 2 + 255) / 256, M);
  if (dtype == SL_BF16) {
    if (in_f32)
      return launch_k(rope_scatter_kernel<float, bf16>, grid, 256, 0, s, (float *)qkv_in, zero_in,
                      M, rows, n_ctx, n_heads, head_dim, rope, (bf16 *)q_out, (bf16 *)ck,
                      (bf16 *)cv);
    return launch_k(rope_scatter_kernel<bf16, bf16>, grid, 256, 0, s, (bf16 *)qkv_in, false, M,
                    rows, n_ctx, n_heads, head_dim, rope, (bf16 *)q_out, (bf16 *)ck, (bf16 *)cv);
  }
  return launch_k(rope_scatter_kernel<float, float>, grid, 256, 0, s, (float *)qkv_in, zero_in, M,
                  rows, n_ctx, n_heads, head_dim, rope, (float *)q_out, (float *)ck, (float *)cv);
}

// ----------------------------------------------------------------- swiglu ---
// act[j][c] = silu(g[j][c]) * u[j][c] from a [M][2F] buffer (gate | up); grid
// x = chunks of 1024 columns (4 per thread), y = row; the fp32 workspace is
// cleared for the next split-K GEMM.
template <typename Tin, typename T>
__global__ void __launch_bounds__(256) swiglu_kernel(Tin *__restrict__ ws, bool zero_in, int M,
                                                     int F, T *__restrict__ act) {
  const int j = blockIdx.y;
  pdl_wait();
  pdl_trigger();
  Tin *g = ws + (size_t)j * 2 * F;
  T *o = act + (size_t)j * F;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int c = blockIdx.x * 1024 + k * 256 + threadIdx.x;
    if (c < F) {
      const float gv = to_f(g[c]), uv = to_f(g[F + c]);
      if (zero_in) {
        g[c] = Tin(0.f);
        g[F + c] = Tin(0.f);
      }
      o[c] = from_f<T>(silu_f(gv) * uv);
    }
  }
}

// The same from the fp32 split-K workspace into bf16, eight columns per thread
// (F % 8 == 0): 16-byte loads and clearing stores, one 16-byte bf16 store.
__global__ void __launch_bounds__(256) swiglu_ws_kernel(float *__restrict__ ws, int M, int F,
                                                        bf16 *__restrict__ act) {
  const int j = blockIdx.y;
  const int c = (blockIdx.x * 256 + threadIdx.x) * 8;
  pdl_wait();
  pdl_trigger();
  if (c >= F) return;
  float4 *g = reinterpret_cast<float4 *>(ws + (size_t)j * 2 * F + c);
  float4 *u = reinterpret_cast<float4 *>(ws + (size_t)j * 2 * F + F + c);
  const float4 g0 = g[0], g1 = g[1], u0 = u[0], u1 = u[1];
  const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
  g[0] = z;
  g[1] = z;
  u[0] = z;
  u[1] = z;
  const float gv[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
  const float uv[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
  Pack8 o;
#pragma unroll
  for (int e = 0; e < 8; ++e) o.h[e] = __float2bfloat16_rn(silu_f(gv[e]) * uv[e]);
  *reinterpret_cast<uint4 *>(act + (size_t)j * F + c) = o.u;
}

cudaError_t launch_swiglu(int dtype, const void *ws, bool in_f32, bool zero_in, int M, int F,
                          void *act, cudaStream_t s) {
  if (M <= 0) return cudaSuccess;
  if (M > 65535) return cudaErrorInvalidValue;
  if (dtype == SL_BF16 && in_f32 && zero_in && F % 8 == 0)
    return launch_k(swiglu_ws_kernel, dim3((F / 8 + 255) / 256, M), 256, 0, s, (float *)ws, M, F,
                    (bf16 *)act);
  const dim3 grid((F + 1023) / 1024, M);
  if (dtype == SL_BF16) {
    if (in_f32)
      return launch_k(swiglu_kernel<float, bf16>, grid, 256, 0, s, (float *)ws, zero_in, M, F,
                      (bf16 *)act);
    return launch_k(swiglu_kernel<bf16, bf16>, grid, 256, 0, s, (bf16 *)ws, false, M, F,
                    (bf16 *)act);
  }
  return launch_k(swiglu_kernel<float, float>, grid, 256, 0, s, (float *)ws, zero_in, M, F,
                  (float *)act);
}

// -------------------------------------------------------- fp32 SIMT GEMM ---
// C[M,N] = A[M,K] B[N,K]^T, 64x64 tiles, 16x16 threads with 4x4 outputs each.
// Used only for fp32 models (tiny shapes); bf16 models run on tcgen05.
constexpr int FT = 64, FK = 16;

__global__ void __launch_bounds__(256) gemm_f32_kernel(int epi, const float *__restrict__ A, int M,
                                                       int K, const float *__restrict__ B, int N,
                                                       float *__restrict__ C, int ldc, int col_off,
                                                       const int32_t *__restrict__ row_map) {
  __shared__ float As[FK][FT + 1];
  __shared__ float Bs[FK][FT + 1];
  pdl_wait();
  int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  int m0 = blockIdx.y * FT, n0 = blockIdx.x * FT;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += FK) {
    for (int e = threadIdx.x; e < FT * FK; e += 256) {
      int r = e / FK, kk = e % FK;
      int gm = m0 + r, gn = n0 + r, gk = k0 + kk;
      As[kk][r] = (gm < M && gk < K) ? A[(size_t)gm * K + gk] : 0.f;
      Bs[kk][r] = (gn < N && gk < K) ? B[(size_t)gn * K + gk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < FK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int i = 0; i < 4; ++i) b[i] = Bs[kk][tx * 4 + i];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) acc[i][jj] = fmaf(a[i], b[jj], acc[i][jj]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int gm = m0 + ty * 4 + i;
    if (gm >= M) continue;
    int orow = row_map ? row_map[gm] : gm;
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      int gn = n0 + tx * 4 + jj;
      if (gn >= N) continue;
      float *dst = C + (size_t)orow * ldc + col_off + gn;
      if (epi == EPI_RESID) *dst += acc[i][jj];
      else *dst = acc[i][jj];
    }
  }
  pdl_trigger();
}

cudaError_t launch_gemm_f32(int epi, const float *A, int M, int K, const float *B, int N,
                            float *C, int ldc, int col_off, const int32_t *row_map,
                            cudaStream_t s) {
  cudaError_t err = cudaSuccess;
  if (M <= 0) return cudaSuccess;
  dim3 grid((N + FT - 1) / FT, (M + FT - 1) / FT);
  err = launch_k(gemm_f32_kernel, grid, 256, 0, s, epi, A, M, K, B, N, C, ldc, col_off, row_map);
  return err;
}

// ------------------------------------------------------------ key stamps ---
// The no-KV-cache ablation (the pages' ablation table: locked tokens cannot be
// attended): the keys a query may see are its sequence's active rows.  Each
// call stamps stamp[row] = gen at the active rows with a new generation, and the
// attention kernels take a key as visible iff its stamp equals gen, so rows
// that left the active set drop out without a clearing pass.
__global__ void key_stamp_kernel(const int32_t *__restrict__ rows, int M, int gen,
                                 int32_t *__restrict__ stamp) {
  pdl_wait();
  pdl_trigger();
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j < M) stamp[rows[j]] = gen;
}

cudaError_t launch_key_stamp(const int32_t *rows, int M, int gen, int32_t *stamp,
                             cudaStream_t s) {
  if (M <= 0) return cudaSuccess;
  return launch_k(key_stamp_kernel, (M + 255) / 256, 256, 0, s, rows, M, gen, stamp);
}

// --------------------------------------------------------- fp32 attention ---
// One warp per (active row, head).  Keys of the row's sequence are processed in
// chunks of 32 (one key per lane) with an online softmax; each lane keeps a
// partial output over its keys, reduced across the warp at the end.  With
// `stamp` non-null only keys whose stamp equals `gen` take part.
template <int DH>
__global__ void attn_f32_kernel(const float *__restrict__ q, const float *__restrict__ ck,
                                const float *__restrict__ cv, const int32_t *__restrict__ rows,
                                int M, int n_ctx, int n_heads, const int32_t *__restrict__ stamp,
                                int gen, float *__restrict__ o) {
  int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  int lane = threadIdx.x & 31;
  if (warp >= M * n_heads) return;
  pdl_wait();
  int j = warp / n_heads, hh = warp % n_heads;
  int d = n_heads * DH;
  int b = rows[j] / n_ctx;
  const float *qv = q + (size_t)j * d + hh * DH;
  float qr[DH];
#pragma unroll
  for (int i = 0; i < DH; ++i) qr[i] = qv[i];
  const float scale = rsqrtf((float)DH);
  float m = -INFINITY, l = 0.f;
  float acc[DH];
#pragma unroll
  for (int i = 0; i < DH; ++i) acc[i] = 0.f;
  for (int n0 = 0; n0 < n_ctx; n0 += 32) {
    int n = n0 + lane;
    const bool live = n < n_ctx && (stamp == nullptr || stamp[(size_t)b * n_ctx + n] == gen);
    float sc = -INFINITY;
    const size_t kr = ((size_t)b * n_ctx + n) * d + hh * DH;
    if (live) {
      float dot = 0.f;
#pragma unroll
      for (int i = 0; i < DH; ++i) dot = fmaf(qr[i], ck[kr + i], dot);
      sc = dot * scale;
    }
    float cm = warp_max(sc);
    float mn = fmaxf(m, cm);
    // a chunk with no visible key while nothing has been seen leaves m = -inf
    float corr = (m == -INFINITY) ? 0.f : __expf(m - mn);
    float pe = live ? __expf(sc - mn) : 0.f;
    l = l * corr + warp_sum(pe);
#pragma unroll
    for (int i = 0; i < DH; ++i) acc[i] *= corr;
    if (live) {
#pragma unroll
      for (int i = 0; i < DH; ++i) acc[i] = fmaf(pe, cv[kr + i], acc[i]);
    }
    m = mn;
  }
  float *ov = o + (size_t)j * d + hh * DH;
#pragma unroll
  for (int i = 0; i < DH; ++i) {
    float v = warp_sum(acc[i]);
    if (lane == 0) ov[i] = v / l;
  }
  pdl_trigger();
}

cudaError_t launch_attn_f32(const float *q, const float *ck, const float *cv,
                            const int32_t *rows, int M, int n_ctx, int n_heads, int head_dim,
                            float *o, cudaStream_t s, const int32_t *stamp, int gen) {
  cudaError_t err = cudaSuccess;
  if (M <= 0) return cudaSuccess;
  int warps = M * n_heads;
  int blocks = (warps * 32 + 255) / 256;
  switch (head_dim) {
    case 8: err = launch_k(attn_f32_kernel<8>, blocks, 256, 0, s, q, ck, cv, rows, M, n_ctx, n_heads, stamp, gen, o); break;
    case 16: err = launch_k(attn_f32_kernel<16>, blocks, 256, 0, s, q, ck, cv, rows, M, n_ctx, n_heads, stamp, gen, o); break;
    case 32: err = launch_k(attn_f32_kernel<32>, blocks, 256, 0, s, q, ck, cv, rows, M, n_ctx, n_heads, stamp, gen, o); break;
    case 64: err = launch_k(attn_f32_kernel<64>, blocks, 256, 0, s, q, ck, cv, rows, M, n_ctx, n_heads, stamp, gen, o); break;
    default: return cudaErrorInvalidValue;
  }
  return err;
}

}  // namespace sl
