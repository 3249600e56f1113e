// The sure test, the confidence gate, compaction of the active set and the
// sampler's unmasking step: the step-to-step KL test D_t = KL(p_t || p_{t-1})
// <= eps at unmasked positions (Paper-Notes, "lock criterion"; Abstract), the
// optional gate u_t = 1 - max p_t <= q_m(u_t) over the active tokens
// (Paper-Notes, "optional confidence gate"; gist.science/it section 2,
// "Filtro di Confidenza"), and the active set that only shrinks (Paper-Notes,
// "permanent locking").
//
// lock_stats: one streaming read of the current and previous logits of every
//   active row.  Each CTA reduces a contiguous vocab chunk of one row with an
//   online max / sum-exp / sum-exp-weighted difference plus the argmax over
//   v != [MASK]; the last CTA of the row (atomic ticket) merges the chunk
//   records and writes D, u, conf, argmax and lse.  HBM-bound.
// lock_decide: per sequence, the gate threshold as an exact order statistic
//   (block-wide radix select on the float bits of u), or the scripted lock
//   schedule (radix select on (D, position)); writes the lock flags.
// compact: stable block-wide ballot/prefix-sum compaction of the active list.
// unmask: top-k confidence among the masked rows of the current block.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace sl {

// ----------------------------------------------------------- lock_stats ----
struct Stat {
  float m;    // running max over all v (includes [MASK])
  float s;    // sum exp(z - m)
  float t;    // sum exp(z - m) * (z - z_prev)
  float bv;   // best value over v != mask_id
  int bi;     // its lowest index
};

// x * c, where a factor c that underflowed to 0 also drops an infinite x (a
// term whose weight is 0 contributes nothing, as 0 log 0 = 0 in the KL).
__device__ __forceinline__ float scaled(float x, float c) { return c == 0.f ? 0.f : x * c; }

__device__ __forceinline__ void stat_merge(Stat &a, const Stat &b) {
  float m = fmaxf(a.m, b.m);
  float ca = (a.m == -INFINITY) ? 0.f : __expf(a.m - m);
  float cb = (b.m == -INFINITY) ? 0.f : __expf(b.m - m);
  a.s = a.s * ca + b.s * cb;
  a.t = scaled(a.t, ca) + scaled(b.t, cb);
  a.m = m;
  if (b.bv > a.bv || (b.bv == a.bv && b.bi < a.bi)) { a.bv = b.bv; a.bi = b.bi; }
}

__device__ __forceinline__ Stat stat_shfl(const Stat &x, int o) {
  Stat y;
  y.m = __shfl_xor_sync(0xffffffffu, x.m, o);
  y.s = __shfl_xor_sync(0xffffffffu, x.s, o);
  y.t = __shfl_xor_sync(0xffffffffu, x.t, o);
  y.bv = __shfl_xor_sync(0xffffffffu, x.bv, o);
  y.bi = __shfl_xor_sync(0xffffffffu, x.bi, o);
  return y;
}

template <typename T> struct Vec8;
template <> struct Vec8<bf16> {
  static __device__ __forceinline__ void load(const bf16 *p, float *o) {
    Pack8 v;
    v.u = __ldcs(reinterpret_cast<const uint4 *>(p));
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(v.h2[i]);
      o[2 * i] = f.x;
      o[2 * i + 1] = f.y;
    }
  }
};
template <> struct Vec8<float> {
  static __device__ __forceinline__ void load(const float *p, float *o) {
    float4 a = __ldcs(reinterpret_cast<const float4 *>(p));
    float4 b = __ldcs(reinterpret_cast<const float4 *>(p) + 1);
    o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
    o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
  }
};

__device__ __forceinline__ void stat_add8(Stat &st, const float *z, const float *zp, int v0,
                                          int mask_id, bool has_prev) {
  float cm = z[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) cm = fmaxf(cm, z[i]);
  if (cm > st.m) {
    float c = (st.m == -INFINITY) ? 0.f : __expf(st.m - cm);
    st.s *= c;
    st.t = scaled(st.t, c);
    st.m = cm;
  }
  // A -inf logit has probability 0 and adds nothing to s or t (0 log 0 = 0 in
  // the KL); while every logit seen so far is -inf, st.m is -inf too and the
  // exponent would be -inf - -inf, so that case is skipped outright.
  // The group's terms are summed first and added to the running sums once, so
  // a row's many small terms do not each round against a sum near 1.
  const bool live = st.m != -INFINITY;
  float gs = 0.f, gt = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float e = live ? __expf(z[i] - st.m) : 0.f;
    gs += e;
    if (has_prev && e > 0.f) gt = fmaf(e, z[i] - zp[i], gt);
    int v = v0 + i;
    if (v != mask_id && z[i] > st.bv) { st.bv = z[i]; st.bi = v; }
  }
  st.s += gs;
  st.t += gt;
}

constexpr int LOCK_THREADS = 256;

template <typename T>
__global__ void __launch_bounds__(LOCK_THREADS) lock_stats_kernel(LockStatsArgs a) {
  const int j = blockIdx.x / a.splits;
  const int sidx = blockIdx.x - j * a.splits;
  if (j >= a.M) return;
  pdl_wait();
  const int V = a.V;
  const int p = a.rows[j];
  const T *cur = reinterpret_cast<const T *>(a.cur) + (size_t)p * V;
  const T *prv = reinterpret_cast<const T *>(a.prev) + (size_t)p * V;
  const bool hp = a.has_prev != 0;

  // vocab chunk of this CTA, in units of 8 elements
  const int nvec = V >> 3;
  const int per = (nvec + a.splits - 1) / a.splits;
  const int vb = sidx * per;
  const int ve = min(nvec, vb + per);

  Stat st{-INFINITY, 0.f, 0.f, -INFINITY, 0x7fffffff};
  float z0[8], p0[8], z1[8], p1[8];
  int v = vb + threadIdx.x;
  for (; v + LOCK_THREADS < ve; v += 2 * LOCK_THREADS) {
    Vec8<T>::load(cur + (size_t)v * 8, z0);
    Vec8<T>::load(cur + (size_t)(v + LOCK_THREADS) * 8, z1);
    if (hp) {
      Vec8<T>::load(prv + (size_t)v * 8, p0);
      Vec8<T>::load(prv + (size_t)(v + LOCK_THREADS) * 8, p1);
    }
    stat_add8(st, z0, p0, v * 8, a.mask_id, hp);
    stat_add8(st, z1, p1, (v + LOCK_THREADS) * 8, a.mask_id, hp);
  }
  if (v < ve) {
    Vec8<T>::load(cur + (size_t)v * 8, z0);
    if (hp) Vec8<T>::load(prv + (size_t)v * 8, p0);
    stat_add8(st, z0, p0, v * 8, a.mask_id, hp);
  }
  // tail (V % 8) handled by the last chunk's first threads
  if (sidx == a.splits - 1) {
    for (int e = nvec * 8 + threadIdx.x; e < V; e += LOCK_THREADS) {
      float z = to_f(cur[e]);
      if (z == -INFINITY) continue;       // probability 0: no term in s, t or the argmax
      float zp = hp ? to_f(prv[e]) : 0.f;
      Stat one{z, 1.f, hp ? (z - zp) : 0.f, (e != a.mask_id) ? z : -INFINITY,
               (e != a.mask_id) ? e : 0x7fffffff};
      stat_merge(st, one);
    }
  }

  pdl_trigger();
  // block reduction
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    Stat y = stat_shfl(st, o);
    stat_merge(st, y);
  }
  __shared__ Stat red[LOCK_THREADS / 32];
  __shared__ bool last;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = st;
  __syncthreads();
  if (warp == 0) {
    st = lane < LOCK_THREADS / 32 ? red[lane] : Stat{-INFINITY, 0.f, 0.f, -INFINITY, 0x7fffffff};
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      Stat y = stat_shfl(st, o);
      stat_merge(st, y);
    }
  }
  if (a.splits > 1) {
    if (threadIdx.x == 0) {
      float4 *rec = a.part + ((size_t)j * a.splits + sidx) * 2;
      rec[0] = make_float4(st.m, st.s, st.t, st.bv);
      rec[1] = make_float4(__int_as_float(st.bi), 0.f, 0.f, 0.f);
      __threadfence();
      unsigned int ticket = atomicAdd(&a.counters[j], 1u);
      last = (ticket == (unsigned)a.splits - 1);
    }
    __syncthreads();
    if (!last) return;
    __threadfence();
    if (warp != 0) return;
    st = Stat{-INFINITY, 0.f, 0.f, -INFINITY, 0x7fffffff};
    for (int q = lane; q < a.splits; q += 32) {
      const float4 *rec = a.part + ((size_t)j * a.splits + q) * 2;
      float4 r0 = __ldcg(rec);
      float4 r1 = __ldcg(rec + 1);
      Stat y{r0.x, r0.y, r0.z, r0.w, __float_as_int(r1.x)};
      stat_merge(st, y);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      Stat y = stat_shfl(st, o);
      stat_merge(st, y);
    }
    if (lane == 0) a.counters[j] = 0u;   // ready for the next call
  } else if (warp != 0) {
    return;
  }
  if (lane == 0) {
    const float lse = st.m + logf(st.s);
    a.lse_cur[p] = lse;
    float D = INFINITY;
    if (hp) D = fmaxf(0.f, st.t / st.s - lse + a.lse_prev[p]);
    a.kl[j] = D;
    a.unc[j] = fmaxf(0.f, 1.f - 1.f / st.s);     // 1 - exp(max z - lse)
    a.conf[j] = __expf(st.bv - lse);
    a.argmax[j] = st.bi;
  }
}

// ------------------------------------------------------ head_stats_merge ----
// The LM-head GEMM's epilogue leaves one record per (row, vocab tile) of the
// stored logits: (max, sum e, sum e (z - z_prev), best value) and the best
// index over v != mask_id.  One warp per active row merges them into the same
// outputs as lock_stats.
__global__ void __launch_bounds__(256) head_stats_merge_kernel(
    const float4 *__restrict__ stat, const int *__restrict__ stat_idx, int n_tiles,
    const int32_t *__restrict__ rows, int M, int has_prev, const float *__restrict__ lse_prev,
    float *__restrict__ lse_cur, float *__restrict__ kl, float *__restrict__ unc,
    float *__restrict__ conf, int32_t *__restrict__ argmax) {
  const int j = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  pdl_wait();
  pdl_trigger();
  if (j >= M) return;
  Stat st{-INFINITY, 0.f, 0.f, -INFINITY, 0x7fffffff};
  const float4 *rec = stat + (size_t)j * n_tiles;
  const int *rid = stat_idx + (size_t)j * n_tiles;
  for (int q = lane; q < n_tiles; q += 32) {
    const float4 r = __ldcs(rec + q);
    Stat y{r.x, r.y, r.z, r.w, __ldcs(rid + q)};
    stat_merge(st, y);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    Stat y = stat_shfl(st, o);
    stat_merge(st, y);
  }
  if (lane == 0) {
    const int p = rows[j];
    const float lse = st.m + logf(st.s);
    lse_cur[p] = lse;
    kl[j] = has_prev ? fmaxf(0.f, st.t / st.s - lse + lse_prev[p]) : INFINITY;
    unc[j] = fmaxf(0.f, 1.f - 1.f / st.s);
    conf[j] = __expf(st.bv - lse);
    argmax[j] = st.bi;
  }
}

cudaError_t launch_head_stats_merge(const float4 *stat, const int *stat_idx, int n_tiles,
                                    const int32_t *rows, int M, int has_prev,
                                    const float *lse_prev, float *lse_cur, float *kl, float *unc,
                                    float *conf, int32_t *argmax, cudaStream_t s) {
  if (M <= 0) return cudaSuccess;
  const int blocks = (M * 32 + 255) / 256;
  return launch_k(head_stats_merge_kernel, blocks, 256, 0, s, stat, stat_idx, n_tiles, rows, M,
                  has_prev, lse_prev, lse_cur, kl, unc, conf, argmax);
}

int lock_stats_splits(int M, int V, int num_sms) {
  if (M <= 0) return 1;
  int target = 4 * num_sms;
  int splits = (target + M - 1) / M;
  int max_by_len = (V / 8) / 256;                 // keep >= 256 vectors per CTA
  if (max_by_len < 1) max_by_len = 1;
  if (splits > max_by_len) splits = max_by_len;
  if (splits > 64) splits = 64;
  if (splits < 1) splits = 1;
  return splits;
}

cudaError_t launch_lock_stats(const LockStatsArgs &a, cudaStream_t s) {
  cudaError_t err = cudaSuccess;
  if (a.M <= 0) return cudaSuccess;
  const long blocks = (long)a.splits * a.M;
  if (blocks > 0x7fffffffL) return cudaErrorInvalidValue;
  dim3 grid((unsigned)blocks);
  if (a.dtype == SL_BF16) { err = launch_k(lock_stats_kernel<bf16>, grid, LOCK_THREADS, 0, s, a); } else { err = launch_k(lock_stats_kernel<float>, grid, LOCK_THREADS, 0, s, a); }
  return err;
}

// ---------------------------------------------------------- radix select ---
// Exact k-th smallest (0-based) key among the n keys key(i) with valid(i),
// 8 bits per pass from the most significant digit.  All threads of the block
// must call it; returns the key value.
constexpr int DEC_THREADS = 1024;

template <typename K, typename KeyFn>
__device__ K block_select(int n, int rank, KeyFn keyfn, unsigned int *hist, K *sh_prefix,
                          int *sh_rank) {
  constexpr int BITS = sizeof(K) * 8;
  K prefix = 0, pmask = 0;
  for (int shift = BITS - 8; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      bool ok;
      K key = keyfn(i, ok);
      if (ok && (key & pmask) == prefix) atomicAdd(&hist[(int)((key >> shift) & 0xff)], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      unsigned int loc = 0;
      for (int q = 0; q < 8; ++q) loc += hist[lane * 8 + q];
      unsigned int inc = loc;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        unsigned int y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
      }
      unsigned int excl = inc - loc;
      int r = rank;
      bool mine = (unsigned)r >= excl && (unsigned)r < inc;
      if (mine) {
        unsigned int c = excl;
        for (int q = 0; q < 8; ++q) {
          unsigned int hcount = hist[lane * 8 + q];
          if ((unsigned)r < c + hcount) {
            *sh_prefix = prefix | ((K)(lane * 8 + q) << shift);
            *sh_rank = r - (int)c;
            break;
          }
          c += hcount;
        }
      }
    }
    __syncthreads();
    prefix = *sh_prefix;
    rank = *sh_rank;
    pmask |= ((K)0xff << shift);
    __syncthreads();
  }
  return prefix;
}

__global__ void __launch_bounds__(DEC_THREADS) lock_decide_kernel(
    const int32_t *__restrict__ seq_off, const int32_t *__restrict__ rows,
    const float *__restrict__ kl, const float *__restrict__ unc,
    const uint8_t *__restrict__ masked, float eps, float gate_q, int has_prev,
    int scripted_target, uint8_t *__restrict__ lock) {
  __shared__ unsigned int hist[256];
  __shared__ unsigned long long sh_p64;
  __shared__ unsigned int sh_p32;
  __shared__ int sh_rank;
  __shared__ int sh_cnt;
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.x;
  const int s0 = seq_off[b], s1 = seq_off[b + 1];
  const int Mb = s1 - s0;
  if (Mb <= 0) return;

  if (scripted_target >= 0) {
    // Scripted schedule: lock the n_lock eligible rows with the smallest (D, position).
    int n_lock = Mb - scripted_target;
    if (!has_prev || n_lock <= 0) {
      for (int i = threadIdx.x; i < Mb; i += blockDim.x) lock[s0 + i] = 0;
      return;
    }
    if (threadIdx.x == 0) sh_cnt = 0;
    __syncthreads();
    int cnt = 0;
    for (int i = threadIdx.x; i < Mb; i += blockDim.x) cnt += masked[rows[s0 + i]] ? 0 : 1;
    atomicAdd(&sh_cnt, cnt);
    __syncthreads();
    const int n_elig = sh_cnt;
    auto key64 = [&](int i, bool &ok) -> unsigned long long {
      int p = rows[s0 + i];
      ok = masked[p] == 0;
      return ((unsigned long long)__float_as_uint(kl[s0 + i]) << 32) | (unsigned)p;
    };
    unsigned long long kth = ~0ull;
    if (n_lock < n_elig)
      kth = block_select<unsigned long long>(Mb, n_lock - 1, key64, hist, &sh_p64, &sh_rank);
    for (int i = threadIdx.x; i < Mb; i += blockDim.x) {
      bool ok;
      unsigned long long k = key64(i, ok);
      lock[s0 + i] = (ok && k <= kth) ? 1 : 0;
    }
    return;
  }

  if (!(eps > 0.f) || !has_prev) {
    for (int i = threadIdx.x; i < Mb; i += blockDim.x) lock[s0 + i] = 0;
    return;
  }
  float thr = INFINITY;
  if (gate_q >= 0.f) {
    // q-quantile of u over the sequence's active rows, lower order statistic.
    int r = (int)floor((double)gate_q * (double)(Mb - 1));
    auto key32 = [&](int i, bool &ok) -> unsigned int {
      ok = true;
      return __float_as_uint(unc[s0 + i]);   // u >= 0: bit order = value order
    };
    unsigned int kth = block_select<unsigned int>(Mb, r, key32, hist, &sh_p32, &sh_rank);
    thr = __uint_as_float(kth);
  }
  for (int i = threadIdx.x; i < Mb; i += blockDim.x) {
    int j = s0 + i;
    bool l = masked[rows[j]] == 0 && kl[j] <= eps && unc[j] <= thr;
    lock[j] = l ? 1 : 0;
  }
}

cudaError_t launch_lock_decide(const int32_t *seq_off, int batch, const int32_t *rows,
                               const float *kl, const float *unc, const uint8_t *masked,
                               float eps, float gate_q, int has_prev, int scripted_target,
                               uint8_t *lock, cudaStream_t s) {
  cudaError_t err = cudaSuccess;
  err = launch_k(lock_decide_kernel, batch, DEC_THREADS, 0, s, seq_off, rows, kl, unc, masked, eps, gate_q,
                                                    has_prev, scripted_target, lock);
  return err;
}

// ------------------------------------------------------------- compaction ---
// A_{t+1} = [rows_j : !lock_j], stable, in place; one CTA walks the sequences
// in order so that the flat list and its offsets stay consistent.
__global__ void __launch_bounds__(DEC_THREADS) compact_kernel(
    int32_t *__restrict__ rows, int32_t *__restrict__ seq_off, int batch,
    const uint8_t *__restrict__ lock, uint8_t *__restrict__ locked, int32_t *__restrict__ lock_t,
    int step) {
  __shared__ int old_off[SL_MAX_BATCH + 1];
  __shared__ int wsum[DEC_THREADS / 32];
  __shared__ int total;
  pdl_wait();
  pdl_trigger();
  for (int i = threadIdx.x; i <= batch; i += blockDim.x) old_off[i] = seq_off[i];
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int out = 0;
  for (int b = 0; b < batch; ++b) {
    const int s0 = old_off[b], s1 = old_off[b + 1];
    const int start = out;
    for (int c0 = s0; c0 < s1; c0 += blockDim.x) {
      const int j = c0 + threadIdx.x;
      bool keep = false;
      int p = 0;
      if (j < s1) {
        p = rows[j];
        if (lock[j]) {
          locked[p] = 1;
          lock_t[p] = step;
        } else {
          keep = true;
        }
      }
      unsigned int bal = __ballot_sync(0xffffffffu, keep);
      int wpre = __popc(bal & ((1u << lane) - 1u));
      if (lane == 0) wsum[warp] = __popc(bal);
      __syncthreads();
      if (warp == 0) {
        int v = lane < (int)(blockDim.x >> 5) ? wsum[lane] : 0;
        int inc = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          int y = __shfl_up_sync(0xffffffffu, inc, o);
          if (lane >= o) inc += y;
        }
        wsum[lane] = inc - v;          // exclusive
        if (lane == 31) total = inc;
      }
      __syncthreads();
      if (keep) rows[out + wsum[warp] + wpre] = p;
      out += total;
      __syncthreads();
    }
    if (threadIdx.x == 0) seq_off[b] = start;
  }
  if (threadIdx.x == 0) seq_off[batch] = out;
}

cudaError_t launch_compact(int32_t *rows, int32_t *seq_off, int batch, const uint8_t *lock,
                           uint8_t *locked, int32_t *lock_t, int step, cudaStream_t s) {
  cudaError_t err = cudaSuccess;
  err = launch_k(compact_kernel, 1, DEC_THREADS, 0, s, rows, seq_off, batch, lock, locked, lock_t, step);
  return err;
}

// --------------------------------------------------------------- unmask ----
constexpr int UNMASK_MAX_CAND = 2048;

__global__ void __launch_bounds__(256) unmask_kernel(
    const int32_t *__restrict__ seq_off, const int32_t *__restrict__ rows, int n_ctx,
    const float *__restrict__ conf, const int32_t *__restrict__ argmax, int lo, int hi, int k,
    int32_t *__restrict__ tokens, uint8_t *__restrict__ masked) {
  __shared__ int cj[UNMASK_MAX_CAND];
  __shared__ int ncand;
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.x;
  const int s0 = seq_off[b], s1 = seq_off[b + 1];
  if (threadIdx.x == 0) ncand = 0;
  __syncthreads();
  for (int j = s0 + threadIdx.x; j < s1; j += blockDim.x) {
    int p = rows[j];
    int i = p - b * n_ctx;
    if (i >= lo && i < hi && masked[p]) {
      int slot = atomicAdd(&ncand, 1);
      if (slot < UNMASK_MAX_CAND) cj[slot] = j;
    }
  }
  __syncthreads();
  const int n = min(ncand, UNMASK_MAX_CAND);
  for (int c = threadIdx.x; c < n; c += blockDim.x) {
    const int j = cj[c];
    const float cf = conf[j];
    const int p = rows[j];
    int better = 0;
    for (int c2 = 0; c2 < n && better < k; ++c2) {
      const int j2 = cj[c2];
      const float f2 = conf[j2];
      better += (f2 > cf || (f2 == cf && rows[j2] < p)) ? 1 : 0;
    }
    if (better < k) {
      tokens[p] = argmax[j];
      masked[p] = 0;
    }
  }
}

cudaError_t launch_unmask(const int32_t *seq_off, int batch, const int32_t *rows, int n_ctx,
                          const float *conf, const int32_t *argmax, int lo, int hi, int k,
                          int32_t *tokens, uint8_t *masked, cudaStream_t s) {
  cudaError_t err = cudaSuccess;
  if (hi - lo > UNMASK_MAX_CAND) return cudaErrorInvalidValue;
  err = launch_k(unmask_kernel, batch, 256, 0, s, seq_off, rows, n_ctx, conf, argmax, lo, hi, k, tokens,
                                      masked);
  return err;
}

// ------------------------------------------------------------ active fill ---
__global__ void active_fill_kernel(int32_t *rows, int32_t *seq_off, int batch, int n_ctx) {
  pdl_wait();
  pdl_trigger();
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  int total = batch * n_ctx;
  if (i < total) rows[i] = i;
  if (i <= batch) seq_off[i] = i * n_ctx;
}

cudaError_t launch_active_fill(int32_t *rows, int32_t *seq_off, int batch, int n_ctx,
                               cudaStream_t s) {
  cudaError_t err = cudaSuccess;
  int total = batch * n_ctx;
  int n = total > batch + 1 ? total : batch + 1;
  err = launch_k(active_fill_kernel, (n + 255) / 256, 256, 0, s, rows, seq_off, batch, n_ctx);
  return err;
}

// ----------------------------------------------- K/V reuse for active rows --
// Between the refresh steps of the reuse, a step computes the active rows that
// are masked now or were masked at the start of the previous step (a row is
// computed once more after its unmasking, so that its cached K/V carry its
// token).  The other active rows keep their cache entries and last posterior.

__device__ __forceinline__ bool reuse_computed(const uint8_t *masked,
                                               const uint8_t *masked_before, int p) {
  return (masked[p] | masked_before[p]) != 0;
}

// C_t = [rows_j : computed(rows_j)], stable, into a second list; one CTA walks
// the sequences in order, as the compaction does.
__global__ void __launch_bounds__(DEC_THREADS) reuse_select_kernel(
    const int32_t *__restrict__ rows, const int32_t *__restrict__ seq_off, int batch,
    const uint8_t *__restrict__ masked, const uint8_t *__restrict__ masked_before,
    int32_t *__restrict__ out_rows, int32_t *__restrict__ out_off) {
  __shared__ int wsum[DEC_THREADS / 32];
  __shared__ int total;
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int out = 0;
  for (int b = 0; b < batch; ++b) {
    const int s0 = seq_off[b], s1 = seq_off[b + 1];
    if (threadIdx.x == 0) out_off[b] = out;
    for (int c0 = s0; c0 < s1; c0 += blockDim.x) {
      const int j = c0 + threadIdx.x;
      int p = 0;
      bool keep = false;
      if (j < s1) {
        p = rows[j];
        keep = reuse_computed(masked, masked_before, p);
      }
      const unsigned int bal = __ballot_sync(0xffffffffu, keep);
      const int wpre = __popc(bal & ((1u << lane) - 1u));
      if (lane == 0) wsum[warp] = __popc(bal);
      __syncthreads();
      if (warp == 0) {
        const int v = lane < (int)(blockDim.x >> 5) ? wsum[lane] : 0;
        int inc = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, inc, o);
          if (lane >= o) inc += y;
        }
        wsum[lane] = inc - v;
        if (lane == 31) total = inc;
      }
      __syncthreads();
      if (keep) out_rows[out + wsum[warp] + wpre] = p;
      out += total;
      __syncthreads();
    }
  }
  if (threadIdx.x == 0) out_off[batch] = out;
}

// The reused rows' logits and lse carried from the previous step's buffers to
// this step's, so that the ping-pong pair always holds every row's last
// posterior (bandwidth-bound copy of 16-byte vectors; blockIdx.y strides over
// the active rows, blockIdx.x over one row's vectors).
constexpr int REUSE_CARRY_THREADS = 256;
constexpr int REUSE_CARRY_VEC = 4;   // 16-byte vectors per thread per pass

__global__ void __launch_bounds__(REUSE_CARRY_THREADS) reuse_carry_kernel(
    const int32_t *__restrict__ rows, const int32_t *__restrict__ seq_off, int batch,
    const uint8_t *__restrict__ masked, const uint8_t *__restrict__ masked_before,
    const uint4 *__restrict__ prev, uint4 *__restrict__ cur, const float *__restrict__ lse_prev,
    float *__restrict__ lse_cur, int row_vecs) {
  pdl_wait();
  pdl_trigger();
  const int M = seq_off[batch];
  for (int j = blockIdx.y; j < M; j += gridDim.y) {
    const int p = rows[j];
    if (reuse_computed(masked, masked_before, p)) continue;
    const uint4 *src = prev + (size_t)p * row_vecs;
    uint4 *dst = cur + (size_t)p * row_vecs;
    const int span = REUSE_CARRY_THREADS * REUSE_CARRY_VEC;
    for (int i0 = blockIdx.x * span; i0 < row_vecs; i0 += gridDim.x * span) {
      uint4 v[REUSE_CARRY_VEC];
#pragma unroll
      for (int u = 0; u < REUSE_CARRY_VEC; ++u) {
        const int i = i0 + u * REUSE_CARRY_THREADS + threadIdx.x;
        if (i < row_vecs) v[u] = src[i];
      }
#pragma unroll
      for (int u = 0; u < REUSE_CARRY_VEC; ++u) {
        const int i = i0 + u * REUSE_CARRY_THREADS + threadIdx.x;
        if (i < row_vecs) dst[i] = v[u];
      }
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) lse_cur[p] = lse_prev[p];
  }
}

// Lock flags of the computed rows (by computed-row index) onto the active list
// (by active-row index) through a per-position byte array that is zero
// between calls: scatter, then gather and clear.  One CTA, so the barrier
// between the two passes is __syncthreads.
__global__ void __launch_bounds__(DEC_THREADS) reuse_lock_map_kernel(
    const int32_t *__restrict__ c_rows, const int32_t *__restrict__ c_off,
    const uint8_t *__restrict__ c_lock, const int32_t *__restrict__ a_rows,
    const int32_t *__restrict__ a_off, int batch, uint8_t *__restrict__ by_pos,
    uint8_t *__restrict__ a_lock) {
  pdl_wait();
  pdl_trigger();
  const int mc = c_off[batch], ma = a_off[batch];
  for (int j = threadIdx.x; j < mc; j += blockDim.x) by_pos[c_rows[j]] = c_lock[j];
  __syncthreads();
  for (int j = threadIdx.x; j < ma; j += blockDim.x) {
    const int p = a_rows[j];
    a_lock[j] = by_pos[p];
    by_pos[p] = 0;
  }
}

cudaError_t launch_reuse_select(const int32_t *rows, const int32_t *seq_off, int batch,
                                const uint8_t *masked, const uint8_t *masked_before,
                                int32_t *out_rows, int32_t *out_off, cudaStream_t s) {
  return launch_k(reuse_select_kernel, 1, DEC_THREADS, 0, s, rows, seq_off, batch, masked,
                  masked_before, out_rows, out_off);
}

cudaError_t launch_reuse_carry(const int32_t *rows, const int32_t *seq_off, int batch,
                               int m_active, const uint8_t *masked,
                               const uint8_t *masked_before, const void *prev, void *cur,
                               const float *lse_prev, float *lse_cur, size_t row_bytes,
                               cudaStream_t s) {
  if (m_active <= 0) return cudaSuccess;
  if (row_bytes % 16 != 0 || ((uintptr_t)prev & 15) || ((uintptr_t)cur & 15))
    return cudaErrorInvalidValue;
  const int row_vecs = (int)(row_bytes / 16);
  const int span = REUSE_CARRY_THREADS * REUSE_CARRY_VEC;
  dim3 grid((row_vecs + span - 1) / span, m_active < 65535 ? m_active : 65535);
  return launch_k(reuse_carry_kernel, grid, REUSE_CARRY_THREADS, 0, s, rows, seq_off, batch,
                  masked, masked_before, static_cast<const uint4 *>(prev),
                  static_cast<uint4 *>(cur), lse_prev, lse_cur, row_vecs);
}

cudaError_t launch_reuse_lock_map(const int32_t *c_rows, const int32_t *c_off,
                                  const uint8_t *c_lock, const int32_t *a_rows,
                                  const int32_t *a_off, int batch, uint8_t *by_pos,
                                  uint8_t *a_lock, cudaStream_t s) {
  return launch_k(reuse_lock_map_kernel, 1, DEC_THREADS, 0, s, c_rows, c_off, c_lock, a_rows,
                  a_off, batch, by_pos, a_lock);
}

}  // namespace sl

// ---------------------------------------------------- no-allocation variant --
// The per-row sure-test statistics for callers that cannot allocate device
// memory.  The chunk records and tickets that the split reduction needs live
// in this file-scope array instead of a workspace: NOALLOC_MAX_RECORDS
// (row, vocab-chunk) records of two float4 each, followed by one ticket
// counter per row for up to NOALLOC_MAX_ROWS rows (about 560 KB per GPU that
// loads the library, held until the process exits).
namespace sl {
namespace {
constexpr int NOALLOC_MAX_ROWS = 8192;
constexpr int NOALLOC_MAX_RECORDS = 16384;
constexpr int NOALLOC_FLOAT4S = NOALLOC_MAX_RECORDS * 2 + NOALLOC_MAX_ROWS / 4;
static __device__ __align__(256) float4 g_noalloc_scratch[NOALLOC_FLOAT4S];

// Host-side device address of g_noalloc_scratch, resolved once per device.
// In host code the symbol itself is only a stand-in, never a device pointer.
struct NoallocSlot {
  bool ready;
  float4 *ptr;
};
NoallocSlot g_noalloc_slots[64];
std::mutex g_noalloc_mu;
}  // namespace
}  // namespace sl

extern "C" sl_status sl_kl_stats_noalloc(const int32_t *d_rows, int M, int vocab, int mask_id,
                                         int logits_dtype, const void *d_logits_cur,
                                         const void *d_logits_prev, const float *d_lse_prev,
                                         float *d_lse_cur, int has_prev, float *d_kl,
                                         float *d_unc, float *d_conf, int32_t *d_argmax,
                                         void *stream) {
  using namespace sl;
  if (M < 0 || M > NOALLOC_MAX_ROWS)
    return fail(SL_ERR_INVALID, "sl_kl_stats_noalloc: M = %d outside [0, %d], the size of its "
                "built-in scratch", M, NOALLOC_MAX_ROWS);
  if (M == 0) return SL_OK;
  if (!d_rows || !d_logits_cur || !d_lse_cur || !d_kl || !d_unc || !d_conf || !d_argmax)
    return fail(SL_ERR_INVALID, "sl_kl_stats_noalloc: null argument");
  if (has_prev && (!d_logits_prev || !d_lse_prev))
    return fail(SL_ERR_INVALID, "sl_kl_stats_noalloc: has_prev needs previous logits and lse");
  if (vocab <= 0 || vocab % 8 != 0)
    return fail(SL_ERR_INVALID, "sl_kl_stats_noalloc: vocab must be a positive multiple of 8");
  if (mask_id < -1 || mask_id >= vocab)
    return fail(SL_ERR_INVALID, "sl_kl_stats_noalloc: bad mask_id");
  if (logits_dtype != SL_F32 && logits_dtype != SL_BF16)
    return fail(SL_ERR_INVALID, "sl_kl_stats_noalloc: bad dtype");
  if (((uintptr_t)d_logits_cur & 15) || (d_logits_prev && ((uintptr_t)d_logits_prev & 15)))
    return fail(SL_ERR_INVALID, "sl_kl_stats_noalloc: logits must be 16-byte aligned");
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "sl_kl_stats_noalloc: cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(SL_ERR_UNSUPPORTED, "sl_kl_stats_noalloc: device %d", dev);
  float4 *scratch = nullptr;
  {
    std::lock_guard<std::mutex> g(g_noalloc_mu);
    NoallocSlot &slot = g_noalloc_slots[dev];
    if (!slot.ready) {
      e = cudaGetSymbolAddress((void **)&slot.ptr, g_noalloc_scratch);
      if (e != cudaSuccess) return cuda_fail(e, "sl_kl_stats_noalloc: cudaGetSymbolAddress");
      slot.ready = true;
    }
    scratch = slot.ptr;
  }
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int splits = lock_stats_splits(M, vocab, sms);
  if (splits > NOALLOC_MAX_RECORDS / M) splits = NOALLOC_MAX_RECORDS / M;
  if (splits < 1) splits = 1;
  unsigned int *tickets = reinterpret_cast<unsigned int *>(scratch + NOALLOC_MAX_RECORDS * 2);
  cudaStream_t s = (cudaStream_t)stream;
  // tickets must start at zero; the array keeps whatever the last call left
  e = cudaMemsetAsync(tickets, 0, (size_t)M * sizeof(unsigned int), s);
  if (e != cudaSuccess) return cuda_fail(e, "sl_kl_stats_noalloc: clearing tickets");
  LockStatsArgs a;
  a.dtype = logits_dtype;
  a.cur = d_logits_cur;
  a.prev = d_logits_prev;
  a.lse_prev = d_lse_prev;
  a.lse_cur = d_lse_cur;
  a.rows = d_rows;
  a.M = M;
  a.V = vocab;
  a.mask_id = mask_id;
  a.has_prev = has_prev ? 1 : 0;
  a.kl = d_kl;
  a.unc = d_unc;
  a.conf = d_conf;
  a.argmax = d_argmax;
  a.part = scratch;
  a.counters = tickets;
  a.splits = splits;
  e = launch_lock_stats(a, s);
  if (e != cudaSuccess) return cuda_fail(e, "sl_kl_stats_noalloc: launch");
  return SL_OK;
}

