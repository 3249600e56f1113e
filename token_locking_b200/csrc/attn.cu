// Attention of the M active queries over all N cached keys of their sequence,
// bf16 in, fp32 softmax/accumulation (head_dim 128).
//
// The pages reduce per-step attention from O(N^2 d) to O(M N d) by issuing
// queries for the active rows only while keys/values of every position are
// read from the cache C (Abstract; Paper-Notes, "permanent locking":
// K^all[L_t] <- C.k[L_t]).  One CTA owns 16 * QW queries of one (sequence,
// head) and a range of 64-key tiles, which stream through a 3-deep
// shared-memory ring (cp.async) with an online softmax.  Its four warps are
// QW query warps x 4/QW key warps: with few active rows per sequence (the
// late denoising steps) the warps split every key tile between them instead
// of idling on empty query rows, and merge their (max, sum, output) states
// through shared memory at the end.  Only when the CTAs cannot fill the GPU
// and the key range is long is it also split across CTAs, with a second
// kernel merging those partial records, one warp per (row, head).
//
// The MASK instantiation serves the no-KV-cache ablation: a key takes part
// only if its stamp equals the step's generation (the active rows' keys); the
// others score -inf exactly like the ragged tail beyond n_ctx.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace sl {

constexpr int AT_K = 64;       // keys per tile
constexpr int AT_D = 128;      // head dim
constexpr int AT_THREADS = 128;
constexpr int AT_STAGES = 3;   // K/V tiles in flight
constexpr int ATTN_MAX_SPLITS = 16;    // cross-CTA split-KV partials merged by attn_combine

template <int QW>
struct AtCfg {
  static constexpr int KW = 4 / QW;          // warps sharing each key tile
  static constexpr int TQ = 16 * QW;         // queries per CTA
  static constexpr int KS = AT_K / KW;       // keys of a tile per warp: 64, 32 or 16
  static constexpr int Q_BYTES = TQ * AT_D * 2;
  static constexpr int KV_BYTES = AT_K * AT_D * 2;   // one K (or V) tile
  static constexpr int SMEM = Q_BYTES + AT_STAGES * 2 * KV_BYTES;
  // merge scratch (reuses the K/V ring): per partial warp 32 lanes x (64 + 4) floats
  static constexpr int PART_FLOATS = 68;
  static_assert(QW * (KW - 1) * 32 * (PART_FLOATS + 4) * 4 <= AT_STAGES * 2 * KV_BYTES,
                "merge scratch must fit in the K/V ring");
};

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
// 16-byte chunk c of row r in a [rows][128] bf16 tile, XOR-swizzled.
__device__ __forceinline__ uint32_t tile_off(int r, int c) {
  return (uint32_t)(r * 256 + ((c ^ (r & 7)) << 4));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
  int sz = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(sz));
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N> __device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                        uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1,
                                          uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void mma16816(float *c, const uint32_t *a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

struct AttnParams {
  const bf16 *q;         // [M][d]
  const bf16 *ck, *cv;   // [B*n_ctx][d]
  bf16 *o;               // [M][d]
  float *ws_o;           // [splits][M][H][128]
  float *ws_ml;          // [splits][M][H][2]
  AttnSeqs seqs;
  int M, n_ctx, n_heads, splits, kblocks;
  const void *pf;        // the next GEMM's weights, prefetched into L2 (optional)
  size_t pf_bytes;
  const int32_t *stamp;  // [B*n_ctx] key stamps (MASK instantiation only)
  int gen;               // stamp value of a visible key
};

template <int QW, bool MASK>
__global__ void __launch_bounds__(AT_THREADS) attn_bf16_kernel(const __grid_constant__ AttnParams p) {
  using C = AtCfg<QW>;
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sQ = smem_u32(smem);
  const uint32_t sKV = sQ + C::Q_BYTES;      // stage s: K tile, then V tile
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int qw = warp / C::KW, kw = warp % C::KW;
  const int h = blockIdx.y, split = blockIdx.z;
  const int d = p.n_heads * AT_D;

  // locate (sequence, query tile)
  int tile = blockIdx.x, b = 0, q0 = 0, qn = 0;
  for (; b < p.seqs.batch; ++b) {
    int nt = (p.seqs.seq_count[b] + C::TQ - 1) / C::TQ;
    if (tile < nt) break;
    tile -= nt;
  }
  if (b >= p.seqs.batch) return;
  q0 = p.seqs.seq_start[b] + tile * C::TQ;
  qn = min(C::TQ, p.seqs.seq_count[b] - tile * C::TQ);

  const int per = (p.kblocks + p.splits - 1) / p.splits;
  const int kb0 = split * per;
  const int kb1 = min(p.kblocks, kb0 + per);
  const int ntiles = max(0, kb1 - kb0);

  const bf16 *kbase = p.ck + (size_t)b * p.n_ctx * d + h * AT_D;
  const bf16 *vbase = p.cv + (size_t)b * p.n_ctx * d + h * AT_D;
  if (tid == 0) {
    const int cta = (blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
    l2_prefetch_share(p.pf, p.pf_bytes, cta, gridDim.x * gridDim.y * gridDim.z);
  }
  pdl_wait();

  for (int e = tid; e < C::TQ * 16; e += AT_THREADS) {
    int r = e >> 4, c = e & 15;
    bool ok = r < qn;
    const bf16 *src = p.q + (size_t)(q0 + (ok ? r : 0)) * d + h * AT_D + c * 8;
    cp_async16(sQ + tile_off(r, c), src, ok);
  }
  auto load_kv = [&](int kb, int stage) {
    const uint32_t sK = sKV + stage * 2 * C::KV_BYTES;
    const uint32_t sV = sK + C::KV_BYTES;
    for (int e = tid; e < AT_K * 16; e += AT_THREADS) {
      int r = e >> 4, c = e & 15;
      int key = kb * AT_K + r;
      bool ok = key < p.n_ctx;
      size_t off = (size_t)(ok ? key : 0) * d + c * 8;
      cp_async16(sK + tile_off(r, c), kbase + off, ok);
      cp_async16(sV + tile_off(r, c), vbase + off, ok);
    }
  };
  // groups: {Q, tile 0}, {tile 1}, then one per iteration (possibly empty)
#pragma unroll
  for (int i = 0; i < AT_STAGES - 1; ++i) {
    if (i < ntiles) load_kv(kb0 + i, i);
    cp_commit();
  }

  const float sl2 = 1.4426950408889634f * rsqrtf((float)AT_D);   // log2(e)/sqrt(dh)
  float o_acc[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) o_acc[i][0] = o_acc[i][1] = o_acc[i][2] = o_acc[i][3] = 0.f;
  float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
  uint32_t qf[8][4];
  const int g = lane >> 2, c4 = lane & 3;
  constexpr int NT = C::KS / 8;     // 8-key score tiles per warp

  for (int i = 0; i < ntiles; ++i) {
    const int kb = kb0 + i, stage = i % AT_STAGES;
    if (i + AT_STAGES - 1 < ntiles) load_kv(kb + AT_STAGES - 1, (i + AT_STAGES - 1) % AT_STAGES);
    cp_commit();
    cp_wait<AT_STAGES - 1>();
    __syncthreads();
    if (i == 0) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        int r = qw * 16 + (lane & 15);
        int c = 2 * kk + (lane >> 4);
        ldsm_x4(sQ + tile_off(r, c), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
      }
    }
    const uint32_t sK = sKV + stage * 2 * C::KV_BYTES;
    const uint32_t sV = sK + C::KV_BYTES;
    float s[NT][4];
#pragma unroll
    for (int t = 0; t < NT; ++t) s[t][0] = s[t][1] = s[t][2] = s[t][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
      for (int nt = 0; nt < NT; nt += 2) {
        int r = kw * C::KS + nt * 8 + (lane & 7) + ((lane >> 4) << 3);
        int c = 2 * kk + ((lane >> 3) & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(sK + tile_off(r, c), b0, b1, b2, b3);
        mma16816(s[nt], qf[kk], b0, b1);
        mma16816(s[nt + 1], qf[kk], b2, b3);
      }
    }
    // online softmax (base 2) on rows g and g+8 of this warp's 16 queries
    float tmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        int key = kb * AT_K + kw * C::KS + nt * 8 + 2 * c4 + (e & 1);
        bool live = key < p.n_ctx;
        if constexpr (MASK) live = live && p.stamp[(size_t)b * p.n_ctx + key] == p.gen;
        float v = live ? s[nt][e] * sl2 : -INFINITY;
        s[nt][e] = v;
        tmax[e >> 1] = fmaxf(tmax[e >> 1], v);
      }
    }
    float corr[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      tmax[r] = fmaxf(tmax[r], __shfl_xor_sync(0xffffffffu, tmax[r], 1));
      tmax[r] = fmaxf(tmax[r], __shfl_xor_sync(0xffffffffu, tmax[r], 2));
      float mn = fmaxf(m_r[r], tmax[r]);
      corr[r] = (m_r[r] == -INFINITY) ? 0.f : exp2f(m_r[r] - mn);
      m_r[r] = mn;
    }
    float rs[2] = {0.f, 0.f};
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float mm = m_r[e >> 1];
        float pv = (mm == -INFINITY) ? 0.f : exp2f(s[nt][e] - mm);
        s[nt][e] = pv;
        rs[e >> 1] += pv;
      }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      rs[r] += __shfl_xor_sync(0xffffffffu, rs[r], 1);
      rs[r] += __shfl_xor_sync(0xffffffffu, rs[r], 2);
      l_r[r] = l_r[r] * corr[r] + rs[r];
    }
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      o_acc[t][0] *= corr[0]; o_acc[t][1] *= corr[0];
      o_acc[t][2] *= corr[1]; o_acc[t][3] *= corr[1];
    }
    // O += P V over this warp's keys of the tile
#pragma unroll
    for (int kc = 0; kc < NT / 2; ++kc) {
      uint32_t pa[4];
      pa[0] = pack_bf16(s[2 * kc][0], s[2 * kc][1]);
      pa[1] = pack_bf16(s[2 * kc][2], s[2 * kc][3]);
      pa[2] = pack_bf16(s[2 * kc + 1][0], s[2 * kc + 1][1]);
      pa[3] = pack_bf16(s[2 * kc + 1][2], s[2 * kc + 1][3]);
#pragma unroll
      for (int dt = 0; dt < 16; dt += 2) {
        int r = kw * C::KS + kc * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
        int c = dt + (lane >> 4);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(sV + tile_off(r, c), b0, b1, b2, b3);
        mma16816(o_acc[dt], pa, b0, b1);
        mma16816(o_acc[dt + 1], pa, b2, b3);
      }
    }
    __syncthreads();      // the stage is refilled by the next iteration's load
  }
  cp_wait<0>();
  pdl_trigger();

  if constexpr (C::KW > 1) {
    // key warps 1.. hand their (max, sum, output) states to key warp 0 of the
    // same query warp through the (now idle) K/V ring
    __syncthreads();
    float *part = reinterpret_cast<float *>(smem + C::Q_BYTES);
    float4 *ml = reinterpret_cast<float4 *>(part + QW * (C::KW - 1) * 32 * C::PART_FLOATS);
    if (kw > 0) {
      const int slot = (qw * (C::KW - 1) + kw - 1) * 32 + lane;
      float4 *dst = reinterpret_cast<float4 *>(part + slot * C::PART_FLOATS);
#pragma unroll
      for (int t = 0; t < 16; ++t) dst[t] = make_float4(o_acc[t][0], o_acc[t][1], o_acc[t][2], o_acc[t][3]);
      ml[slot] = make_float4(m_r[0], m_r[1], l_r[0], l_r[1]);
    }
    __syncthreads();
    if (kw > 0) return;
#pragma unroll 1
    for (int j = 1; j < C::KW; ++j) {
      const int slot = (qw * (C::KW - 1) + j - 1) * 32 + lane;
      const float4 pm = ml[slot];
      const float om[2] = {pm.x, pm.y}, ol[2] = {pm.z, pm.w};
      float c1[2], c2[2];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const float mx = fmaxf(m_r[r], om[r]);
        c1[r] = (m_r[r] == -INFINITY) ? 0.f : exp2f(m_r[r] - mx);
        c2[r] = (om[r] == -INFINITY) ? 0.f : exp2f(om[r] - mx);
        l_r[r] = l_r[r] * c1[r] + ol[r] * c2[r];
        m_r[r] = mx;
      }
      const float4 *src = reinterpret_cast<const float4 *>(part + slot * C::PART_FLOATS);
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        const float4 v = src[t];
        o_acc[t][0] = o_acc[t][0] * c1[0] + v.x * c2[0];
        o_acc[t][1] = o_acc[t][1] * c1[0] + v.y * c2[0];
        o_acc[t][2] = o_acc[t][2] * c1[1] + v.z * c2[1];
        o_acc[t][3] = o_acc[t][3] * c1[1] + v.w * c2[1];
      }
    }
  }

  // epilogue: rows g and g+8 of this query warp's 16
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    int qr = qw * 16 + g + 8 * r;
    if (qr >= qn) continue;
    int j = q0 + qr;
    if (p.splits == 1) {
      float inv = l_r[r] > 0.f ? 1.f / l_r[r] : 0.f;
      bf16 *dst = p.o + (size_t)j * d + h * AT_D;
#pragma unroll
      for (int dt = 0; dt < 16; ++dt) {
        *reinterpret_cast<uint32_t *>(dst + dt * 8 + 2 * c4) =
            pack_bf16(o_acc[dt][2 * r] * inv, o_acc[dt][2 * r + 1] * inv);
      }
    } else {
      size_t rec = ((size_t)split * p.M + j) * p.n_heads + h;
      float *dst = p.ws_o + rec * AT_D;
#pragma unroll
      for (int dt = 0; dt < 16; ++dt)
        *reinterpret_cast<float2 *>(dst + dt * 8 + 2 * c4) =
            make_float2(o_acc[dt][2 * r], o_acc[dt][2 * r + 1]);
      if (c4 == 0) *reinterpret_cast<float2 *>(p.ws_ml + rec * 2) = make_float2(m_r[r], l_r[r]);
    }
  }
}

// Merge split-KV partials: one warp per (row, head), 4 dims per lane.
__global__ void attn_combine_kernel(const float *__restrict__ ws_o, const float *__restrict__ ws_ml,
                                    int M, int n_heads, int splits, bf16 *__restrict__ o) {
  const int w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= M * n_heads) return;
  pdl_wait();
  pdl_trigger();
  const int j = w / n_heads, h = w % n_heads;
  float m[ATTN_MAX_SPLITS], l[ATTN_MAX_SPLITS];
  float mx = -INFINITY;
#pragma unroll
  for (int sp = 0; sp < ATTN_MAX_SPLITS; ++sp) {
    m[sp] = -INFINITY;
    l[sp] = 0.f;
    if (sp < splits) {
      const float2 ml = *reinterpret_cast<const float2 *>(ws_ml + (((size_t)sp * M + j) * n_heads + h) * 2);
      m[sp] = ml.x;
      l[sp] = ml.y;
      mx = fmaxf(mx, ml.x);
    }
  }
  float L = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int sp = 0; sp < ATTN_MAX_SPLITS; ++sp) {
    if (sp < splits) {
      const float c = (m[sp] == -INFINITY) ? 0.f : exp2f(m[sp] - mx);
      L += l[sp] * c;
      const float4 v = *reinterpret_cast<const float4 *>(
          ws_o + (((size_t)sp * M + j) * n_heads + h) * AT_D + lane * 4);
      acc.x += v.x * c; acc.y += v.y * c; acc.z += v.z * c; acc.w += v.w * c;
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  bf16 *dst = o + (size_t)j * n_heads * AT_D + h * AT_D + lane * 4;
  *reinterpret_cast<uint2 *>(dst) =
      make_uint2(pack_bf16(acc.x * inv, acc.y * inv), pack_bf16(acc.z * inv, acc.w * inv));
}

size_t attn_bf16_workspace_bytes(int max_rows, int n_heads, int max_splits) {
  return (size_t)max_splits * max_rows * n_heads * (AT_D + 2) * sizeof(float);
}


template <int QW, bool MASK>
static cudaError_t run_attn(const AttnParams &p, int tiles, cudaStream_t s) {
  using C = AtCfg<QW>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(attn_bf16_kernel<QW, MASK>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  return launch_k(attn_bf16_kernel<QW, MASK>, dim3(tiles, p.n_heads, p.splits), AT_THREADS,
                  C::SMEM, s, p);
}

template <bool MASK>
static cudaError_t run_attn_qw(int qw, const AttnParams &p, int tiles, cudaStream_t s) {
  return qw == 4 ? run_attn<4, MASK>(p, tiles, s)
                 : qw == 2 ? run_attn<2, MASK>(p, tiles, s) : run_attn<1, MASK>(p, tiles, s);
}

cudaError_t launch_attn_bf16(const void *q, const void *ck, const void *cv, const AttnSeqs &seqs,
                             int M, int n_ctx, int n_heads, void *o, float *ws, int max_splits,
                             int num_sms, cudaStream_t s, int force_q, int force_splits,
                             const void *pf, size_t pf_bytes, const int32_t *stamp, int gen) {
  cudaError_t err = cudaSuccess;
  if (M <= 0) return cudaSuccess;
  // Queries per CTA (16 * qw) and cross-CTA key split from a small cost model:
  // mma.sync instructions per warp (16 queries x its share of the keys), about
  // 15 ns each once two CTAs share every SM; the K/V re-reads from L2, one per
  // query tile; and a fixed cost for the merge kernel of a split.
  const int kblocks = (n_ctx + AT_K - 1) / AT_K;
  int qw = 4, splits = 1, tiles = 0;
  double best = 1e30;
  const int max_sp = std::min(std::max(kblocks / 4, 1), std::min(max_splits, ATTN_MAX_SPLITS));
  for (int cq : {4, 2, 1}) {
    int nt = 0;
    for (int b = 0; b < seqs.batch; ++b) nt += (seqs.seq_count[b] + 16 * cq - 1) / (16 * cq);
    if (nt == 0) return cudaSuccess;
    for (int sp = 1; sp <= max_sp; ++sp) {
      const double warps = 4.0 * nt * n_heads * sp;
      const double per_warp = 2.0 * ((double)kblocks * AT_K / sp) / (4 / cq);
      const double t_mma = per_warp * std::max(1.0, warps / (8.0 * num_sms)) * 15e-9;
      const double t_l2 = (double)nt * n_heads * n_ctx * AT_D * 4.0 / 8e12;
      const double t = std::max(t_mma, t_l2) + (sp > 1 ? 3e-6 : 0.0);
      if (force_q && 16 * cq != force_q) continue;
      if (force_splits && sp != std::min(force_splits, max_sp)) continue;
      if (t < best - 1e-12) {
        best = t;
        qw = cq;
        splits = sp;
        tiles = nt;
      }
    }
  }
  AttnParams p;
  p.q = (const bf16 *)q;
  p.ck = (const bf16 *)ck;
  p.cv = (const bf16 *)cv;
  p.o = (bf16 *)o;
  p.ws_o = ws;
  p.ws_ml = ws + (size_t)splits * M * n_heads * AT_D;
  p.seqs = seqs;
  p.M = M;
  p.n_ctx = n_ctx;
  p.n_heads = n_heads;
  p.splits = splits;
  p.kblocks = kblocks;
  p.pf = pf;
  p.pf_bytes = pf_bytes;
  p.stamp = stamp;
  p.gen = gen;
  err = stamp ? run_attn_qw<true>(qw, p, tiles, s) : run_attn_qw<false>(qw, p, tiles, s);
  if (err != cudaSuccess || splits == 1) return err;
  const int warps = M * n_heads;
  return launch_k(attn_combine_kernel, (warps * 32 + 255) / 256, 256, 0, s, (const float *)p.ws_o,
                  (const float *)p.ws_ml, M, n_heads, splits, (bf16 *)o);
}

}  // namespace sl
