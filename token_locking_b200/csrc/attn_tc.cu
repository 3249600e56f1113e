// Attention of the M active queries over all N cached keys of their sequence
// on the 5th-generation tensor cores (tcgen05 + TMEM), K/V tiles fed by TMA.
//
// The pages cut a step's attention from O(N^2 d) to O(M N d) by issuing
// queries for the active rows only, while the keys and values of every
// position come from the cache C, frozen at the lock step for locked rows
// (Abstract; Paper-Notes, "permanent locking": K^all[L_t] <- C.k[L_t];
// gist.science/nl section 2, "Complexiteitsvermindering").
//
// One CTA owns a tile of 128 queries of one (sequence, head) and a range of
// 128-key tiles (the whole key range, or a share of it when the tiles alone
// cannot fill the GPU):
//   warp 0      TMA producer: the Q tile once, then K and V tiles through a
//               two-stage ring (two 64-column boxes each, 128-byte swizzle)
//   warp 1      TMEM owner and single-thread MMA issue:
//                 S_t = Q K_t^T  (M=128, N=128 keys, K=128 dims; both K-major)
//                 into one of two TMEM score buffers, one tile ahead, and
//                 O += P_t V_t   (M=128, N=128 dims, K=128 keys; P K-major from
//                 shared memory, V MN-major straight from its TMA tile)
//   warps 2..5  softmax: thread i owns query row i (its TMEM lane), so the row
//               max and sum need no shuffles.  Scores are scaled into base 2;
//               the running max is raised lazily (only when a tile's max
//               exceeds it by more than 2^8, rescaling O in TMEM), the bf16
//               probabilities go to shared memory for the P V product.
// A split key range leaves unnormalised partial rows and (max, sum) in a
// workspace; the thread that completes a row's last split (atomic ticket per
// row and head) merges them, so no second kernel is needed.
// Every barrier wait is bounded; a wait that runs out records the failure in
// the device error word and the CTA winds down (copies drained, TMEM freed).
#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"

namespace sl {

namespace {
constexpr int TA_BM = 128;                    // queries per tile (TMEM lanes)
constexpr int TA_BN = 128;                    // keys per tile
constexpr int TA_D = 128;                     // head dim
constexpr int TA_STAGES = 2;                  // K/V tiles in flight
constexpr int TA_BOX = 128 * 128;             // one [128 rows][64 bf16] swizzled box, bytes
constexpr int TA_Q_OFF = 0;                   // Q: dims 0-63 box, dims 64-127 box
constexpr int TA_KV_OFF = 2 * TA_BOX;         // stage s: K box 0, K box 1, V box 0, V box 1
constexpr int TA_STAGE = 4 * TA_BOX;
constexpr int TA_P_OFF = TA_KV_OFF + TA_STAGES * TA_STAGE;   // P: keys 0-63 box, keys 64-127 box
constexpr int TA_BAR_OFF = TA_P_OFF + 2 * TA_BOX;
constexpr int TA_SMEM = TA_BAR_OFF + 256 + 1024;             // barriers + 1 KB alignment slack
constexpr uint32_t TA_TMEM_COLS = 512;        // S buffers at 0 and 128, O at 256
constexpr uint32_t TA_COL_S = 0, TA_COL_O = 256;
constexpr int TA_THREADS = 192;
constexpr float TA_RESCALE = 8.f;             // raise the running max when exceeded by 2^8
static_assert(TA_SMEM <= 232448, "attention tile exceeds the shared memory of a CTA");

// barrier slots
enum : int { B_Q = 0, B_KVF = 1, B_KVE = 3, B_SF = 5, B_SE = 7, B_PF = 9, B_OR = 10, B_DRAIN = 11,
             B_COUNT = 12 };
}  // namespace

struct TaParams {
  CUtensorMap q_map;     // q [M][d], box 64 x 128 rows
  CUtensorMap k_map;     // this layer's C.k [B*n_ctx][d], box 64 x 128 rows
  CUtensorMap v_map;     // C.v, same
  bf16 *o;               // [M][d]
  float *ws_o;           // [splits][M][H][128] unnormalised partial rows
  float *ws_ml;          // [splits][M][H][2] (max in base 2, sum)
  unsigned int *tickets; // [M][H], zero between calls
  AttnSeqs seqs;
  int M, n_ctx, n_heads, splits, kt_per_split, ktiles;
  const int32_t *stamp;  // [B*n_ctx] key stamps (MASK instantiation only)
  int gen;
  const void *pf;        // the next GEMM's weights, prefetched into L2 (optional)
  size_t pf_bytes;
  int *err;
  unsigned long long wait_ns;
};

__device__ __forceinline__ uint32_t pack2_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

// All 32 lanes wait; the outcome is made uniform across the warp so that the
// warp-collective tcgen05 loads and stores that follow never run on a partial
// warp.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                          unsigned long long lim) {
  const bool ok = mbar_wait(bar, parity, abort_flag, lim);
  return __all_sync(0xffffffffu, ok);
}

template <bool MASK>
__global__ void __launch_bounds__(TA_THREADS, 1) attn_tc_kernel(const __grid_constant__ TaParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = s_addr(smem);
  const uint32_t bar0 = sbase + TA_BAR_OFF;
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + TA_BAR_OFF + 8 * B_COUNT);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned long long lim = p.wait_ns;

  // (sequence, query tile) of this CTA; uniform, so an empty CTA leaves at once
  int tile = blockIdx.x, b = 0;
  for (; b < p.seqs.batch; ++b) {
    const int nt = (p.seqs.seq_count[b] + TA_BM - 1) / TA_BM;
    if (tile < nt) break;
    tile -= nt;
  }
  if (b >= p.seqs.batch) return;
  const int q0 = p.seqs.seq_start[b] + tile * TA_BM;
  const int qn = min(TA_BM, p.seqs.seq_count[b] - tile * TA_BM);
  const int h = blockIdx.y, split = blockIdx.z;
  const int kt0 = split * p.kt_per_split;
  const int T = max(0, min(p.ktiles, kt0 + p.kt_per_split) - kt0);
  const int d = p.n_heads * TA_D;

  if (threadIdx.x == 0) {
    mbar_init(bar(B_Q), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(B_KVF + s), 1);
      mbar_init(bar(B_KVE + s), 1);
      mbar_init(bar(B_SF + s), 1);
      mbar_init(bar(B_SE + s), 4);         // the four softmax warps
    }
    mbar_init(bar(B_PF), 4);
    mbar_init(bar(B_OR), 1);
    mbar_init(bar(B_DRAIN), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    tma_prefetch_desc(&p.q_map);
    tma_prefetch_desc(&p.k_map);
    tma_prefetch_desc(&p.v_map);
    const int cta = (blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
    l2_prefetch_share(p.pf, p.pf_bytes, cta, gridDim.x * gridDim.y * gridDim.z);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     s_addr(tmem_slot)),
                 "r"(TA_TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      pdl_wait();                            // q and this step's fresh K/V
      bool ok = true;
      mbar_expect_tx(bar(B_Q), 2 * TA_BOX);
      tma_load_2d(sbase + TA_Q_OFF, &p.q_map, h * TA_D, q0, bar(B_Q));
      tma_load_2d(sbase + TA_Q_OFF + TA_BOX, &p.q_map, h * TA_D + 64, q0, bar(B_Q));
      int last_st = -1;
      uint32_t last_ph = 0;
      for (int t = 0; t < T; ++t) {
        const int st = t & 1;
        const uint32_t ph = (uint32_t)(t >> 1) & 1u;
        if (!mbar_wait(bar(B_KVE + st), ph ^ 1u, abort_flag, lim)) { ok = false; break; }
        mbar_expect_tx(bar(B_KVF + st), TA_STAGE);
        const int y = b * p.n_ctx + (kt0 + t) * TA_BN;
        const uint32_t sk = sbase + TA_KV_OFF + st * TA_STAGE;
        tma_load_2d(sk, &p.k_map, h * TA_D, y, bar(B_KVF + st));
        tma_load_2d(sk + TA_BOX, &p.k_map, h * TA_D + 64, y, bar(B_KVF + st));
        tma_load_2d(sk + 2 * TA_BOX, &p.v_map, h * TA_D, y, bar(B_KVF + st));
        tma_load_2d(sk + 3 * TA_BOX, &p.v_map, h * TA_D + 64, y, bar(B_KVF + st));
        last_st = st;
        last_ph = ph;
      }
      pdl_trigger();
      if (!ok) {
        atomicExch(p.err, DEV_TIMEOUT_PRODUCER);
        *abort_flag = 1;
      }
      // every issued copy lands before the CTA can exit
      volatile int never = 0;
      mbar_wait(bar(B_Q), 0, &never, lim);
      if (last_st >= 0) mbar_wait(bar(B_KVF + last_st), last_ph, &never, lim);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_bf16_f32<TA_BN>();
      constexpr uint32_t id_o = idesc_bf16_f32_bmn<TA_D>();
      const uint32_t sq = sbase + TA_Q_OFF;
      auto issue_s = [&](int t) {
        const int st = t & 1;
        const uint32_t sk = sbase + TA_KV_OFF + st * TA_STAGE;
        const uint32_t dt = tmem_base + TA_COL_S + (uint32_t)(st * TA_BN);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t a = smem_desc_sw128(sq + (kk >> 2) * TA_BOX) + 2 * (kk & 3);
          const uint64_t bd = smem_desc_sw128(sk + (kk >> 2) * TA_BOX) + 2 * (kk & 3);
          tc_mma(dt, a, bd, id_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(B_SF + st));
      };
      bool ok = mbar_wait(bar(B_Q), 0, abort_flag, lim);
      if (ok && T > 0) ok = mbar_wait(bar(B_KVF), 0, abort_flag, lim);
      if (ok && T > 0) {
        tc_fence_after();
        issue_s(0);
      }
      for (int t = 0; ok && t < T; ++t) {
        if (t + 1 < T) {
          const int st = (t + 1) & 1;
          const uint32_t ph = (uint32_t)((t + 1) >> 1) & 1u;
          if (!mbar_wait(bar(B_KVF + st), ph, abort_flag, lim) ||
              !mbar_wait(bar(B_SE + st), ph ^ 1u, abort_flag, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_s(t + 1);
        }
        if (!mbar_wait(bar(B_PF), (uint32_t)t & 1u, abort_flag, lim)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sv = sbase + TA_KV_OFF + (t & 1) * TA_STAGE + 2 * TA_BOX;
        const uint32_t sp = sbase + TA_P_OFF;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t a = smem_desc_sw128(sp + (kk >> 2) * TA_BOX) + 2 * (kk & 3);
          const uint64_t bd = smem_desc_sw128_mn(sv + kk * 2048, TA_BOX, 1024);
          tc_mma(tmem_base + TA_COL_O, a, bd, id_o, (t > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(bar(B_KVE + (t & 1)));   // K_t and V_t consumed
        tc_commit(bar(B_OR));              // O holds tiles 0..t; P may be rewritten
      }
      if (!ok) {
        atomicExch(p.err, DEV_TIMEOUT_MMA);
        *abort_flag = 1;
      }
      tc_commit(bar(B_DRAIN));
      volatile int never = 0;
      mbar_wait(bar(B_DRAIN), 0, &never, lim);
    }
  } else {
    // --------------------------------------------------------- softmax
    pdl_wait();                              // o may still be read by an earlier kernel
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;       // query row of this thread (TMEM lane)
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t t_o = tmem_base + lane_off + TA_COL_O;
    const float sl2 = 1.4426950408889634f * rsqrtf((float)TA_D);   // log2(e) / sqrt(dh)
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    float s[TA_BN];
    for (int t = 0; t < T; ++t) {
      const int st = t & 1;
      if (!warp_wait(bar(B_SF + st), (uint32_t)(t >> 1) & 1u, abort_flag, lim)) { ok = false; break; }
      tc_fence_after();
      const uint32_t ts = tmem_base + lane_off + TA_COL_S + (uint32_t)(st * TA_BN);
      tmem_ld32_nw(ts, s);
      tmem_ld32_nw(ts + 32, s + 32);
      tmem_ld32_nw(ts + 64, s + 64);
      tmem_ld32_nw(ts + 96, s + 96);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_SE + st));
      const int key0 = (kt0 + t) * TA_BN;
      float mt = -INFINITY;
#pragma unroll
      for (int i = 0; i < TA_BN; ++i) {
        const int key = key0 + i;
        bool live = key < p.n_ctx;
        if constexpr (MASK) live = live && p.stamp[(size_t)b * p.n_ctx + key] == p.gen;
        s[i] = live ? s[i] * sl2 : -INFINITY;
        mt = fmaxf(mt, s[i]);
      }
      const float m_new = fmaxf(m, mt);
      const bool resc = t > 0 && m_new > m + TA_RESCALE;
      const float m_use = (t == 0 || resc) ? m_new : m;
      const float alpha = resc ? ((m == -INFINITY) ? 0.f : ex2_approx(m - m_new)) : 1.f;
      float rs = 0.f;
#pragma unroll
      for (int i = 0; i < TA_BN; ++i) {
        const float pv = (m_use == -INFINITY) ? 0.f : ex2_approx(s[i] - m_use);
        s[i] = pv;
        rs += pv;
      }
      if (t > 0) {
        // P V of the previous tile done: P may be overwritten, O is current
        if (!warp_wait(bar(B_OR), (uint32_t)(t - 1) & 1u, abort_flag, lim)) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, resc)) {
#pragma unroll 1
          for (int c = 0; c < TA_D; c += 32) {
            float o[32];
            tmem_ld32_nw(t_o + c, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] *= alpha;
            tmem_st32(t_o + c, o);
          }
          tmem_wait_st();
        }
      }
      l = l * alpha + rs;
      m = m_use;
      // P row -> shared memory, K-major with the 128-byte swizzle of a TMA tile
      const uint32_t prow = sbase + TA_P_OFF + (uint32_t)r * 128u;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        st_shared_v4(prow + (c >> 3) * TA_BOX + ((uint32_t)((c & 7) ^ (r & 7)) << 4),
                     pack2_bf16(s[8 * c], s[8 * c + 1]), pack2_bf16(s[8 * c + 2], s[8 * c + 3]),
                     pack2_bf16(s[8 * c + 4], s[8 * c + 5]), pack2_bf16(s[8 * c + 6], s[8 * c + 7]));
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_PF));
    }
    if (ok && T > 0) ok = warp_wait(bar(B_OR), (uint32_t)(T - 1) & 1u, abort_flag, lim);
    if (ok && T > 0) {
      tc_fence_after();
      tmem_ld32_nw(t_o, s);
      tmem_ld32_nw(t_o + 32, s + 32);
      tmem_ld32_nw(t_o + 64, s + 64);
      tmem_ld32_nw(t_o + 96, s + 96);
      tmem_wait_ld();
      const int j = q0 + r;                  // active-row index of this query
      if (r < qn) {
        if (p.splits == 1) {
          const float inv = l > 0.f ? 1.f / l : 0.f;
          uint4 *dst = reinterpret_cast<uint4 *>(p.o + (size_t)j * d + h * TA_D);
#pragma unroll
          for (int c = 0; c < 16; ++c)
            dst[c] = make_uint4(pack2_bf16(s[8 * c] * inv, s[8 * c + 1] * inv),
                                pack2_bf16(s[8 * c + 2] * inv, s[8 * c + 3] * inv),
                                pack2_bf16(s[8 * c + 4] * inv, s[8 * c + 5] * inv),
                                pack2_bf16(s[8 * c + 6] * inv, s[8 * c + 7] * inv));
        } else {
          const size_t rec = ((size_t)split * p.M + j) * p.n_heads + h;
          float4 *dst = reinterpret_cast<float4 *>(p.ws_o + rec * TA_D);
#pragma unroll
          for (int c = 0; c < 32; ++c)
            dst[c] = make_float4(s[4 * c], s[4 * c + 1], s[4 * c + 2], s[4 * c + 3]);
          *reinterpret_cast<float2 *>(p.ws_ml + rec * 2) = make_float2(m, l);
          __threadfence();
          unsigned int *tk = p.tickets + (size_t)j * p.n_heads + h;
          const unsigned int ticket = atomicAdd(tk, 1u);
          if (ticket == (unsigned)p.splits - 1) {
            // this thread completed the row: merge every split's partial
            __threadfence();
            float mx = -INFINITY;
            for (int q = 0; q < p.splits; ++q) {
              const float2 ml = __ldcg(reinterpret_cast<const float2 *>(
                  p.ws_ml + (((size_t)q * p.M + j) * p.n_heads + h) * 2));
              mx = fmaxf(mx, ml.x);
            }
#pragma unroll
            for (int e = 0; e < TA_D; ++e) s[e] = 0.f;
            float L = 0.f;
            for (int q = 0; q < p.splits; ++q) {
              const size_t rq = ((size_t)q * p.M + j) * p.n_heads + h;
              const float2 ml = __ldcg(reinterpret_cast<const float2 *>(p.ws_ml + rq * 2));
              const float c = (ml.x == -INFINITY) ? 0.f : ex2_approx(ml.x - mx);
              L += ml.y * c;
              const float4 *src = reinterpret_cast<const float4 *>(p.ws_o + rq * TA_D);
#pragma unroll
              for (int e = 0; e < 32; ++e) {
                const float4 v = __ldcg(src + e);
                s[4 * e] += v.x * c;
                s[4 * e + 1] += v.y * c;
                s[4 * e + 2] += v.z * c;
                s[4 * e + 3] += v.w * c;
              }
            }
            const float inv = L > 0.f ? 1.f / L : 0.f;
            uint4 *dst2 = reinterpret_cast<uint4 *>(p.o + (size_t)j * d + h * TA_D);
#pragma unroll
            for (int c = 0; c < 16; ++c)
              dst2[c] = make_uint4(pack2_bf16(s[8 * c] * inv, s[8 * c + 1] * inv),
                                   pack2_bf16(s[8 * c + 2] * inv, s[8 * c + 3] * inv),
                                   pack2_bf16(s[8 * c + 4] * inv, s[8 * c + 5] * inv),
                                   pack2_bf16(s[8 * c + 6] * inv, s[8 * c + 7] * inv));
            *tk = 0u;                          // ready for the next call
          }
        }
      }
    }
    if (!ok && lane == 0) {
      atomicExch(p.err, DEV_TIMEOUT_EPI);
      *abort_flag = 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(TA_TMEM_COLS)
                 : "memory");
  }
}

template <bool MASK>
static cudaError_t run_attn_tc(const TaParams &p, dim3 grid, cudaStream_t s) {
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<MASK>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, TA_SMEM);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  return launch_k(attn_tc_kernel<MASK>, grid, TA_THREADS, TA_SMEM, s, p);
}

// Key splits of the tcgen05 attention from a small cost model: CTAs run one
// wave after another (one per SM, shared memory bound); a CTA costs a fixed
// set-up and drain plus a per-key-tile time, and a split adds the merge.
int attn_tc_splits(int q_tiles, int n_heads, int n_ctx, int num_sms, int max_splits) {
  const int ktiles = (n_ctx + TA_BN - 1) / TA_BN;
  int best_s = 1;
  double best = 1e30;
  for (int sp = 1; sp <= std::min(ktiles, std::min(max_splits, 16)); ++sp) {
    const int per = (ktiles + sp - 1) / sp;
    const int s_eff = (ktiles + per - 1) / per;
    if (s_eff != sp) continue;
    const long ctas = (long)q_tiles * n_heads * sp;
    const long waves = (ctas + num_sms - 1) / num_sms;
    const double t = waves * (2.0 + 0.6 * per) + (sp > 1 ? 1.0 : 0.0);
    if (t < best - 1e-9) {
      best = t;
      best_s = sp;
    }
  }
  return best_s;
}

size_t attn_tc_tickets_bytes(int max_rows, int n_heads) {
  return (size_t)max_rows * n_heads * sizeof(unsigned int);
}

cudaError_t launch_attn_tc(const TmaMat &q_map, const TmaMat &k_map, const TmaMat &v_map,
                           const AttnSeqs &seqs, int M, int n_ctx, int n_heads, void *o,
                           float *ws, unsigned int *tickets, int max_splits, int num_sms,
                           int *err, unsigned long long wait_ns, cudaStream_t s, int force_splits,
                           const void *pf, size_t pf_bytes, const int32_t *stamp, int gen) {
  if (M <= 0) return cudaSuccess;
  int q_tiles = 0;
  for (int b = 0; b < seqs.batch; ++b) q_tiles += (seqs.seq_count[b] + TA_BM - 1) / TA_BM;
  if (q_tiles == 0) return cudaSuccess;
  const int ktiles = (n_ctx + TA_BN - 1) / TA_BN;
  int splits = force_splits > 0 ? std::min(force_splits, std::min(ktiles, max_splits))
                                : attn_tc_splits(q_tiles, n_heads, n_ctx, num_sms, max_splits);
  const int per = (ktiles + splits - 1) / splits;
  splits = (ktiles + per - 1) / per;          // no empty split
  TaParams p;
  memset(&p, 0, sizeof(p));
  p.q_map = q_map.map;
  p.k_map = k_map.map;
  p.v_map = v_map.map;
  p.o = (bf16 *)o;
  p.ws_o = ws;
  p.ws_ml = ws + (size_t)splits * M * n_heads * TA_D;
  p.tickets = tickets;
  p.seqs = seqs;
  p.M = M;
  p.n_ctx = n_ctx;
  p.n_heads = n_heads;
  p.splits = splits;
  p.kt_per_split = per;
  p.ktiles = ktiles;
  p.stamp = stamp;
  p.gen = gen;
  p.pf = pf;
  p.pf_bytes = pf_bytes;
  p.err = err;
  p.wait_ns = wait_ns ? wait_ns : WAIT_LIMIT_NS;
  const dim3 grid(q_tiles, n_heads, splits);
  return stamp ? run_attn_tc<true>(p, grid, s) : run_attn_tc<false>(p, grid, s);
}

}  // namespace sl
