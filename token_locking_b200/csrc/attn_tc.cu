// Attention of the M active queries over all N cached keys of their sequence
// on the 5th-generation tensor cores (tcgen05 + TMEM), K/V tiles fed by TMA.
//
// The pages cut a step's attention from O(N^2 d) to O(M N d) by issuing
// queries for the active rows only, while the keys and values of every
// position come from the cache C, frozen at the lock step for locked rows
// (Abstract; Paper-Notes, "permanent locking": K^all[L_t] <- C.k[L_t];
// gist.science/nl section 2, "Complexiteitsvermindering").
//
// One CTA owns QT tiles of 128 queries of one (sequence, head) and a range of
// BN-key tiles (the whole key range, or a share of it when the tiles alone
// cannot fill the GPU):
//   warp 0      TMA producer: the Q tiles once, then K and V tiles through an
//               ST-stage ring (64-column boxes, 128-byte swizzle)
//   warp 1      TMEM owner and single-thread MMA issue, per key tile t and
//               query tile j:
//                 S_j = Q_j K_t^T  (M=128, N=BN keys, K=128 dims; both K-major
//                 from shared memory) into a TMEM score buffer of tile j, one
//                 key tile ahead, then
//                 O_j += P_j V_t   (M=128, N=128 dims, K=BN keys; P K-major
//                 from TMEM, V MN-major straight from its TMA tile)
//   warps 2..   one softmax warpgroup per query tile: thread i owns query row
//               i (its TMEM lane), so the row max and sum need no shuffles.
//               Scores are scaled into base 2; the running max is raised
//               lazily (only when a tile's max exceeds it by more than 2^8,
//               rescaling O in TMEM); the bf16 probabilities go back to TMEM
//               into one of two P buffers, so the P V product of tile t runs
//               while the exponentials of tile t + 1 are taken, and the
//               product reads P from TMEM, sparing shared memory the P traffic.
// What bounds one CTA is latency, not a pipe or a memory path: every key tile
// passes from the TMA producer to the MMA warp (scores), to the softmax
// warpgroup (P), and back to the MMA warp (P V), about a microsecond of
// handoffs per tile whatever the work in it; a CTA also spends ~6 us starting
// (TMEM, first copies) and draining (O out).  So the default layout is small
// enough for two CTAs per SM, which then run two independent tile chains that
// hide each other's handoffs, start-up and drain.  Two query tiles per CTA
// (QT = 2) share every K/V tile instead, halving the K/V bytes per FLOP, with
// one score buffer per query tile (64-key tiles): the scores of tile t + 1 are
// issued as soon as the softmax has loaded those of tile t.
// A K/V stage is released only when the P V products of its tile have
// completed, so the copy of tile t + ST starts then and must land before the
// scores of that tile can be issued: the ring is deep enough to cover the TMA
// latency (about a microsecond) with the work of the tiles in between.
// Layouts (query tiles / key tile / ring depth / score buffers): 1 / 128 / 3 /
// 2 and 2 / 64 / 5 / 1 use most of an SM's shared memory and all 512 TMEM
// columns (one CTA per SM); 1 / 64 / 2 / 1 needs 97 KB and 256 columns, so two
// CTAs share an SM and each hides the other's barrier handoffs, start-up and
// drain.
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
constexpr int TA_D = 128;                     // head dim
constexpr int TA_HBOX = 128 * 128;            // [128 rows][64 bf16] swizzled box, bytes
constexpr float TA_RESCALE = 8.f;             // raise the running max when exceeded by 2^8

template <int QT, int BN, int ST, int SB>
struct TaCfg {
  static constexpr int KBOX = BN * 128;                  // [BN rows][64 dims] box of K or V
  static constexpr int STAGE = 4 * KBOX;                 // K box 0, K box 1, V box 0, V box 1
  static constexpr int Q_OFF = 0;                        // per query tile two dims boxes
  static constexpr int KV_OFF = QT * 2 * TA_HBOX;
  static constexpr int BAR_OFF = KV_OFF + ST * STAGE;
  // barriers: Q, k_full[ST], k_empty[ST], v_full[ST], v_empty[ST] (a stage's
  // K half is released when the scores of its tile are done, its V half when
  // the P V products are), per query tile (s_full[2], s_free[2], p_full[2],
  // pv_done[2]), drain
  static constexpr int B_Q = 0, B_KF = 1, B_KE = 1 + ST, B_VF = 1 + 2 * ST, B_VE = 1 + 3 * ST;
  static constexpr int B_TILE = 1 + 4 * ST;
  static constexpr int B_DRAIN = B_TILE + 8 * QT, B_COUNT = B_DRAIN + 1;
  static constexpr int SMEM = BAR_OFF + 8 * B_COUNT + 16 + 1024;   // + slot/flag + alignment
  static constexpr int THREADS = 64 + 128 * QT;
  // TMEM: SB score buffers of tile j at (SB j + b) BN, O of tile j at
  // O_COL + 128 j, the two bf16 P buffers of tile j (BN / 2 columns each, two
  // keys per column) at P_COL + (2 j + u) BN / 2
  static constexpr uint32_t O_COL = QT * SB * BN;
  static constexpr uint32_t P_COL = O_COL + QT * 128;
  // two CTAs per SM when both fit: half of TMEM and of shared memory each
  static constexpr int CTAS_PER_SM = (P_COL + QT * BN <= 256 && SMEM <= 232448 / 2 - 1024) ? 2 : 1;
  static constexpr uint32_t TMEM_COLS = CTAS_PER_SM == 2 ? 256 : 512;
  static_assert(P_COL + QT * BN <= TMEM_COLS, "TMEM columns");
  static_assert(SMEM <= 232448, "shared memory of a CTA");
  static_assert(BN % 64 == 0 && BN <= 256, "key tile");
  static_assert(SB == 1 || SB == 2, "score buffers");
};
}  // namespace

struct TaParams {
  CUtensorMap q_map;     // q [M][d], box 64 x 128 rows
  CUtensorMap k_map;     // this layer's C.k [B*n_ctx][d], box 64 x BN rows
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

// Loads 32 fp32 columns per call; n = BN / 32 calls then one wait.
template <int BN>
__device__ __forceinline__ void tmem_ld_row(uint32_t taddr, float *s) {
#pragma unroll
  for (int c = 0; c < BN; c += 32) tmem_ld32_nw(taddr + c, s + c);
  tmem_wait_ld();
}

template <int QT, int BN, int ST, int SB, bool MASK>
__global__ void __launch_bounds__(TaCfg<QT, BN, ST, SB>::THREADS, TaCfg<QT, BN, ST, SB>::CTAS_PER_SM)
    attn_tc_kernel(const __grid_constant__ TaParams p) {
  using C = TaCfg<QT, BN, ST, SB>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = s_addr(smem);
  const uint32_t bar0 = sbase + C::BAR_OFF;
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  auto tbar = [&](int j, int k) { return bar0 + 8u * (uint32_t)(C::B_TILE + 8 * j + k); };
  // per query tile: 0,1 s_full[b]; 2,3 s_free[b]; 4,5 p_full[u]; 6,7 pv_done[u]
  // (b = score buffer of key tile t, u = t & 1).  With two score buffers each
  // completes once every other key tile; with one, s_full[0] and s_free[0]
  // complete once per key tile.
  auto sbuf = [](int t) { return SB == 2 ? (t & 1) : 0; };
  auto spar = [](int t) { return (uint32_t)(SB == 2 ? (t >> 1) : t) & 1u; };
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::BAR_OFF + 8 * C::B_COUNT);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned long long lim = p.wait_ns;

  // (sequence, query tiles) of this CTA; uniform, so an empty CTA leaves at once
  int unit = blockIdx.x, b = 0;
  for (; b < p.seqs.batch; ++b) {
    const int nt = ((p.seqs.seq_count[b] + TA_BM - 1) / TA_BM + QT - 1) / QT;
    if (unit < nt) break;
    unit -= nt;
  }
  if (b >= p.seqs.batch) return;
  const int q0 = p.seqs.seq_start[b] + unit * QT * TA_BM;
  const int qn_all = min(QT * TA_BM, p.seqs.seq_count[b] - unit * QT * TA_BM);
  const int nj = (qn_all + TA_BM - 1) / TA_BM;          // query tiles present (1..QT)
  const int h = blockIdx.y, split = blockIdx.z;
  const int kt0 = split * p.kt_per_split;
  const int T = max(0, min(p.ktiles, kt0 + p.kt_per_split) - kt0);
  const int d = p.n_heads * TA_D;

  if (threadIdx.x == 0) {
    mbar_init(bar(C::B_Q), 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(bar(C::B_KF + s), 1);
      mbar_init(bar(C::B_KE + s), 1);
      mbar_init(bar(C::B_VF + s), 1);
      mbar_init(bar(C::B_VE + s), 1);
    }
    for (int j = 0; j < QT; ++j)
      for (int u = 0; u < 2; ++u) {
        mbar_init(tbar(j, u), 1);            // MMA commit
        mbar_init(tbar(j, 2 + u), 4);        // the tile's four softmax warps
        mbar_init(tbar(j, 4 + u), 4);
        mbar_init(tbar(j, 6 + u), 1);
      }
    mbar_init(bar(C::B_DRAIN), 1);
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
                 "r"(C::TMEM_COLS)
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
      mbar_expect_tx(bar(C::B_Q), nj * 2 * TA_HBOX);
      for (int j = 0; j < nj; ++j) {
        const uint32_t sq = sbase + C::Q_OFF + j * 2 * TA_HBOX;
        tma_load_2d(sq, &p.q_map, h * TA_D, q0 + j * TA_BM, bar(C::B_Q));
        tma_load_2d(sq + TA_HBOX, &p.q_map, h * TA_D + 64, q0 + j * TA_BM, bar(C::B_Q));
      }
      // K of tile t + ST goes into stage t % ST once the scores of tile t are
      // done, V once its P V products are: K runs ahead of V
      int nk = 0, nv = 0;                    // K and V copies issued
      for (int t = 0; t < T; ++t) {
        const int st = t % ST;
        const uint32_t ph = (uint32_t)(t / ST) & 1u;
        const int y = b * p.n_ctx + (kt0 + t) * BN;
        const uint32_t sk = sbase + C::KV_OFF + st * C::STAGE;
        if (!mbar_wait(bar(C::B_KE + st), ph ^ 1u, abort_flag, lim)) { ok = false; break; }
        mbar_expect_tx(bar(C::B_KF + st), 2 * C::KBOX);
        tma_load_2d(sk, &p.k_map, h * TA_D, y, bar(C::B_KF + st));
        tma_load_2d(sk + C::KBOX, &p.k_map, h * TA_D + 64, y, bar(C::B_KF + st));
        ++nk;
        if (!mbar_wait(bar(C::B_VE + st), ph ^ 1u, abort_flag, lim)) { ok = false; break; }
        mbar_expect_tx(bar(C::B_VF + st), 2 * C::KBOX);
        tma_load_2d(sk + 2 * C::KBOX, &p.v_map, h * TA_D, y, bar(C::B_VF + st));
        tma_load_2d(sk + 3 * C::KBOX, &p.v_map, h * TA_D + 64, y, bar(C::B_VF + st));
        ++nv;
      }
      pdl_trigger();
      if (!ok) {
        atomicExch(p.err, DEV_TIMEOUT_PRODUCER);
        *abort_flag = 1;
      }
      // every issued copy lands before the CTA can exit: the last copy into
      // each stage of each ring (copies complete in any order)
      volatile int never = 0;
      mbar_wait(bar(C::B_Q), 0, &never, lim);
      for (int st = 0; st < ST; ++st) {
        if (st < nk) {
          const int tl = st + ((nk - 1 - st) / ST) * ST;   // last tile copied into stage st
          mbar_wait(bar(C::B_KF + st), (uint32_t)(tl / ST) & 1u, &never, lim);
        }
        if (st < nv) {
          const int tl = st + ((nv - 1 - st) / ST) * ST;
          mbar_wait(bar(C::B_VF + st), (uint32_t)(tl / ST) & 1u, &never, lim);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_bf16_f32<BN>();
      constexpr uint32_t id_o = idesc_bf16_f32_bmn<TA_D>();
      auto issue_s = [&](int t, int j) {
        const uint32_t sq = sbase + C::Q_OFF + j * 2 * TA_HBOX;
        const uint32_t sk = sbase + C::KV_OFF + (t % ST) * C::STAGE;
        const uint32_t dt = tmem_base + (uint32_t)((j * SB + sbuf(t)) * BN);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t a = smem_desc_sw128(sq + (kk >> 2) * TA_HBOX) + 2 * (kk & 3);
          const uint64_t bd = smem_desc_sw128(sk + (kk >> 2) * C::KBOX) + 2 * (kk & 3);
          tc_mma(dt, a, bd, id_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(tbar(j, sbuf(t)));
      };
      auto issue_pv = [&](int t, int j) {
        const uint32_t sv = sbase + C::KV_OFF + (t % ST) * C::STAGE + 2 * C::KBOX;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          // P of key tile t from its TMEM buffer: 16 keys = 8 columns per step
          const uint64_t bd = smem_desc_sw128_mn(sv + kk * 2048, C::KBOX, 1024);
          const uint32_t pa =
              tmem_base + C::P_COL + (uint32_t)((2 * j + (t & 1)) * (BN / 2) + kk * 8);
          tc_mma_ts(tmem_base + C::O_COL + 128 * j, pa, bd, id_o, (t > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(tbar(j, 6 + (t & 1)));
      };
      bool ok = mbar_wait(bar(C::B_Q), 0, abort_flag, lim);
      if (ok && T > 0) ok = mbar_wait(bar(C::B_KF), 0, abort_flag, lim);
      if (ok && T > 0) {
        tc_fence_after();
        for (int j = 0; j < nj; ++j) issue_s(0, j);
        tc_commit(bar(C::B_KE));             // K_0 free once these scores are done
      }
      for (int t = 0; ok && t < T; ++t) {
        if (t + 1 < T) {
          const int st = (t + 1) % ST;
          if (!mbar_wait(bar(C::B_KF + st), (uint32_t)((t + 1) / ST) & 1u, abort_flag, lim)) {
            ok = false;
            break;
          }
          for (int j = 0; ok && j < nj; ++j) {
            // the score buffer of key tile t + 1 was last read at key tile
            // t + 1 - SB (its s_free phase before the current one)
            if (!mbar_wait(tbar(j, 2 + sbuf(t + 1)), spar(t + 1) ^ 1u, abort_flag, lim)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_s(t + 1, j);
          }
          if (!ok) break;
          tc_commit(bar(C::B_KE + st));      // K_{t+1} consumed by every tile
        }
        if (!mbar_wait(bar(C::B_VF + t % ST), (uint32_t)(t / ST) & 1u, abort_flag, lim)) {
          ok = false;
          break;
        }
        for (int j = 0; ok && j < nj; ++j) {
          if (!mbar_wait(tbar(j, 4 + (t & 1)), (uint32_t)(t >> 1) & 1u, abort_flag, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_pv(t, j);
        }
        if (!ok) break;
        tc_commit(bar(C::B_VE + t % ST));    // V_t consumed by every tile
      }
      if (!ok) {
        atomicExch(p.err, DEV_TIMEOUT_MMA);
        *abort_flag = 1;
      }
      tc_commit(bar(C::B_DRAIN));
      volatile int never = 0;
      mbar_wait(bar(C::B_DRAIN), 0, &never, lim);
    }
  } else {
    // ---------------------------------------------------------- softmax
    const int j = (warp - 2) >> 2;           // query tile of this warpgroup
    if (j < nj) {
      pdl_wait();                            // o may still be read by an earlier kernel
      const int quarter = warp & 3;
      const int r = quarter * 32 + lane;     // query row of this thread (TMEM lane)
      const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
      const uint32_t t_o = tmem_base + lane_off + C::O_COL + 128 * j;
      const int qn = min(TA_BM, qn_all - j * TA_BM);
      const float sl2 = 1.4426950408889634f * rsqrtf((float)TA_D);   // log2(e) / sqrt(dh)
      float m = -INFINITY, l = 0.f;
      bool ok = true;
      float s[BN];
      for (int t = 0; t < T; ++t) {
        const int u = t & 1;
        if (!warp_wait(tbar(j, sbuf(t)), spar(t), abort_flag, lim)) { ok = false; break; }
        tc_fence_after();
        tmem_ld_row<BN>(tmem_base + lane_off + (uint32_t)((j * SB + sbuf(t)) * BN), s);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tbar(j, 2 + sbuf(t)));
        const int key0 = (kt0 + t) * BN;
        // row max of the raw scores (the scale is positive) as eight independent
        // partials: a single running value would chain BN dependent instructions
        float mx[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) mx[e] = -INFINITY;
        if (key0 + BN <= p.n_ctx && !MASK) {
#pragma unroll
          for (int i = 0; i < BN; ++i) mx[i & 7] = fmaxf(mx[i & 7], s[i]);
        } else {
#pragma unroll
          for (int i = 0; i < BN; ++i) {
            const int key = key0 + i;
            bool live = key < p.n_ctx;
            if constexpr (MASK) live = live && p.stamp[(size_t)b * p.n_ctx + key] == p.gen;
            s[i] = live ? s[i] : -INFINITY;
            mx[i & 7] = fmaxf(mx[i & 7], s[i]);
          }
        }
        const float mt = sl2 * fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                     fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
        const float m_new = fmaxf(m, mt);
        const bool resc = t > 0 && m_new > m + TA_RESCALE;
        const float m_use = (t == 0 || resc) ? m_new : m;
        const float alpha = resc ? ((m == -INFINITY) ? 0.f : ex2_approx(m - m_new)) : 1.f;
        float sm[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        const float m_sub = (m_use == -INFINITY) ? 0.f : m_use;   // all scores -inf: p = 0
        // p = 2^(s log2(e) / sqrt(dh) - m): the scale and the shift in one FMA
#pragma unroll
        for (int i = 0; i < BN; ++i) {
          const float pv = ex2_approx(fmaf(s[i], sl2, -m_sub));
          s[i] = pv;
          sm[i & 7] += pv;
        }
        const float rs = ((sm[0] + sm[1]) + (sm[2] + sm[3])) + ((sm[4] + sm[5]) + (sm[6] + sm[7]));
        // O must be current before a rescale, and the P buffer about to be
        // written must have been read, last by the P V product of tile t - 2
        const bool any_resc = __any_sync(0xffffffffu, resc);
        const int t_prev = any_resc ? t - 1 : t - 2;
        if (t_prev >= 0) {
          const int ub = t_prev & 1;
          if (!warp_wait(tbar(j, 6 + ub), (uint32_t)(t_prev >> 1) & 1u, abort_flag, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (any_resc) {
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
        // P row -> this lane of the tile's P buffer u, two bf16 keys per column
        {
          const uint32_t tp = tmem_base + lane_off + C::P_COL + (uint32_t)((2 * j + u) * (BN / 2));
#pragma unroll
          for (int c = 0; c < BN / 64; ++c) {
            uint32_t pk[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) pk[e] = pack2_bf16(s[64 * c + 2 * e], s[64 * c + 2 * e + 1]);
            tmem_st32_u(tp + 32 * c, pk);
          }
          tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tbar(j, 4 + u));
      }
      if (ok && T > 0)
        ok = warp_wait(tbar(j, 6 + ((T - 1) & 1)), (uint32_t)((T - 1) >> 1) & 1u, abort_flag, lim);
      if (ok && T > 0) {
        tc_fence_after();
        const int jr = q0 + j * TA_BM + r;     // active-row index of this query
        bf16 *orow = p.o + (size_t)jr * d + h * TA_D;
        // O leaves in two 64-column halves (fewer live registers)
        if (p.splits == 1) {
          const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
          for (int c0 = 0; c0 < TA_D; c0 += 64) {
            tmem_ld_row<64>(t_o + c0, s);
            if (r < qn) {
              uint4 *dst = reinterpret_cast<uint4 *>(orow + c0);
#pragma unroll
              for (int c = 0; c < 8; ++c)
                dst[c] = make_uint4(pack2_bf16(s[8 * c] * inv, s[8 * c + 1] * inv),
                                    pack2_bf16(s[8 * c + 2] * inv, s[8 * c + 3] * inv),
                                    pack2_bf16(s[8 * c + 4] * inv, s[8 * c + 5] * inv),
                                    pack2_bf16(s[8 * c + 6] * inv, s[8 * c + 7] * inv));
            }
          }
        } else {
          const size_t rec = ((size_t)split * p.M + jr) * p.n_heads + h;
#pragma unroll 1
          for (int c0 = 0; c0 < TA_D; c0 += 64) {
            tmem_ld_row<64>(t_o + c0, s);
            if (r < qn) {
              float4 *dst = reinterpret_cast<float4 *>(p.ws_o + rec * TA_D + c0);
#pragma unroll
              for (int c = 0; c < 16; ++c)
                dst[c] = make_float4(s[4 * c], s[4 * c + 1], s[4 * c + 2], s[4 * c + 3]);
            }
          }
          if (r < qn) {
            *reinterpret_cast<float2 *>(p.ws_ml + rec * 2) = make_float2(m, l);
            __threadfence();
            unsigned int *tk = p.tickets + (size_t)jr * p.n_heads + h;
            const unsigned int ticket = atomicAdd(tk, 1u);
            if (ticket == (unsigned)p.splits - 1) {
              // this thread completed the row: merge every split's partial
              __threadfence();
              float mx = -INFINITY, L = 0.f;
              for (int q = 0; q < p.splits; ++q) {
                const float2 ml = __ldcg(reinterpret_cast<const float2 *>(
                    p.ws_ml + (((size_t)q * p.M + jr) * p.n_heads + h) * 2));
                mx = fmaxf(mx, ml.x);
              }
              for (int q = 0; q < p.splits; ++q) {
                const float2 ml = __ldcg(reinterpret_cast<const float2 *>(
                    p.ws_ml + (((size_t)q * p.M + jr) * p.n_heads + h) * 2));
                L += ml.y * ((ml.x == -INFINITY) ? 0.f : ex2_approx(ml.x - mx));
              }
              const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll 1
              for (int c0 = 0; c0 < TA_D; c0 += 64) {
#pragma unroll
                for (int e = 0; e < 64; ++e) s[e] = 0.f;
                for (int q = 0; q < p.splits; ++q) {
                  const size_t rq = ((size_t)q * p.M + jr) * p.n_heads + h;
                  const float2 ml = __ldcg(reinterpret_cast<const float2 *>(p.ws_ml + rq * 2));
                  const float c = (ml.x == -INFINITY) ? 0.f : ex2_approx(ml.x - mx);
                  const float4 *src = reinterpret_cast<const float4 *>(p.ws_o + rq * TA_D + c0);
#pragma unroll
                  for (int e = 0; e < 16; ++e) {
                    const float4 v = __ldcg(src + e);
                    s[4 * e] += v.x * c;
                    s[4 * e + 1] += v.y * c;
                    s[4 * e + 2] += v.z * c;
                    s[4 * e + 3] += v.w * c;
                  }
                }
                uint4 *dst2 = reinterpret_cast<uint4 *>(orow + c0);
#pragma unroll
                for (int c = 0; c < 8; ++c)
                  dst2[c] = make_uint4(pack2_bf16(s[8 * c] * inv, s[8 * c + 1] * inv),
                                       pack2_bf16(s[8 * c + 2] * inv, s[8 * c + 3] * inv),
                                       pack2_bf16(s[8 * c + 4] * inv, s[8 * c + 5] * inv),
                                       pack2_bf16(s[8 * c + 6] * inv, s[8 * c + 7] * inv));
              }
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
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(C::TMEM_COLS)
                 : "memory");
  }
}

template <int QT, int BN, int ST, int SB, bool MASK>
static cudaError_t run_attn_tc(const TaParams &p, dim3 grid, cudaStream_t s) {
  using C = TaCfg<QT, BN, ST, SB>;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<QT, BN, ST, SB, MASK>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    // all of the SM's unified L1 as shared memory, so that two CTAs fit
    e = cudaFuncSetAttribute(attn_tc_kernel<QT, BN, ST, SB, MASK>,
                             cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  return launch_k(attn_tc_kernel<QT, BN, ST, SB, MASK>, grid, C::THREADS, C::SMEM, s, p);
}

// Layout and key split of the tensor-core attention from a small cost model:
// CTAs run in waves (one or two per SM, bound by shared memory and TMEM); a
// CTA costs a fixed set-up and drain plus a time per (128-query tile x 128
// keys) of work that depends on the layout; a split adds the merge.
namespace {
struct TaLayout {
  int qt, bn, per_sm;   // query tiles and key tile of a CTA, CTAs resident per SM
  double c_unit;        // us per 128 x 128 block of work of one CTA at the power-capped clock
};
// measured on batch 4 x 512 and 2048 queries over 2048 keys; a CTA's start-up
// (first Q/K/V copies, TMEM allocation) and drain (O out) cost ~6 us; a key
// split costs as much again plus its partial rows: every split of every query
// row and head writes 128 fp32 values and the merge reads them back, at an
// effective ~1.8 TB/s (measured: two splits take 91 / 134 / 245 us at batch 4 x
// 256 / 384 / 768 queries against 46 / 85 / 126 us unsplit)
constexpr TaLayout kTaLayouts[] = {{1, 128, 1, 1.3}, {1, 64, 2, 2.2}, {2, 64, 1, 1.9}};
constexpr double kTaCtaFixed = 6.0, kTaSplitCost = 6.0, kTaSplitBytesPerUs = 1.8e6;
}  // namespace

AttnTcPlan attn_tc_plan(const AttnSeqs &seqs, int n_heads, int n_ctx, int num_sms,
                        int max_splits, int force_q, int force_splits, int force_bn) {
  AttnTcPlan best{};
  double best_t = 1e30;
  for (const TaLayout &ly : kTaLayouts) {
    const int qt = ly.qt, bn = ly.bn;
    if (force_q && force_q != 128 * qt) continue;
    if (force_bn && force_bn != bn) continue;
    const int ktiles = (n_ctx + bn - 1) / bn;
    int units = 0, tiles = 0;
    for (int b = 0; b < seqs.batch; ++b) {
      const int qtb = (seqs.seq_count[b] + TA_BM - 1) / TA_BM;
      units += (qtb + qt - 1) / qt;
      tiles += qtb;
    }
    if (units == 0) return best;
    const double fill = (double)tiles / ((double)units * qt);   // query tiles present per slot
    long rows = 0;                                              // query rows of the launch
    for (int b = 0; b < seqs.batch; ++b) rows += seqs.seq_count[b];
    const int max_sp = std::min(ktiles, std::min(max_splits, 16));
    for (int req = 1; req <= max_sp; ++req) {
      // a requested split rounds to the count that covers the key tiles evenly
      // (no empty split); a pinned request is taken as that count
      if (force_splits && req != std::min(force_splits, max_sp)) continue;
      const int per = (ktiles + req - 1) / req;
      const int sp = (ktiles + per - 1) / per;
      if (!force_splits && sp != req) continue;
      const long ctas = (long)units * n_heads * sp;
      const long waves = (ctas + (long)num_sms * ly.per_sm - 1) / ((long)num_sms * ly.per_sm);
      const double work = (double)per * bn / 128.0 * qt * fill;
      const double split_bytes = sp > 1 ? (double)rows * n_heads * sp * TA_D * 4.0 * 2.0 : 0.0;
      const double t = waves * (kTaCtaFixed + ly.c_unit * work) +
                       (sp > 1 ? kTaSplitCost + split_bytes / kTaSplitBytesPerUs : 0.0);
      if (t < best_t * 0.97) {                 // a clear gain, else the earlier layout
        best_t = t;
        best.qt = qt;
        best.bn = bn;
        best.splits = sp;
        best.kt_per_split = per;
        best.ktiles = ktiles;
        best.units = units;
      }
    }
  }
  return best;
}

size_t attn_tc_tickets_bytes(int max_rows, int n_heads) {
  return (size_t)max_rows * n_heads * sizeof(unsigned int);
}

cudaError_t launch_attn_tc(const TmaMat &q_map, const TmaMat &k_map128, const TmaMat &v_map128,
                           const TmaMat &k_map64, const TmaMat &v_map64, const AttnSeqs &seqs,
                           int M, int n_ctx, int n_heads, void *o, float *ws,
                           unsigned int *tickets, int max_splits, int num_sms, int *err,
                           unsigned long long wait_ns, cudaStream_t s, int force_q,
                           int force_splits, int force_bn, const void *pf, size_t pf_bytes,
                           const int32_t *stamp, int gen) {
  if (M <= 0) return cudaSuccess;
  if (force_q != 0 && force_q != 128 && force_q != 256) return cudaErrorInvalidValue;
  if (force_bn != 0 && force_bn != 64 && force_bn != 128) return cudaErrorInvalidValue;
  int q_tiles = 0;
  for (int b = 0; b < seqs.batch; ++b) q_tiles += (seqs.seq_count[b] + TA_BM - 1) / TA_BM;
  if (q_tiles == 0) return cudaSuccess;
  const AttnTcPlan pl = attn_tc_plan(seqs, n_heads, n_ctx, num_sms, max_splits, force_q,
                                     force_splits, force_bn);
  if (pl.units == 0) return cudaErrorInvalidConfiguration;     // never silently skip work
  TaParams p;
  memset(&p, 0, sizeof(p));
  p.q_map = q_map.map;
  p.k_map = pl.bn == 64 ? k_map64.map : k_map128.map;
  p.v_map = pl.bn == 64 ? v_map64.map : v_map128.map;
  p.o = (bf16 *)o;
  p.ws_o = ws;
  p.ws_ml = ws + (size_t)pl.splits * M * n_heads * TA_D;
  p.tickets = tickets;
  p.seqs = seqs;
  p.M = M;
  p.n_ctx = n_ctx;
  p.n_heads = n_heads;
  p.splits = pl.splits;
  p.kt_per_split = pl.kt_per_split;
  p.ktiles = pl.ktiles;
  p.stamp = stamp;
  p.gen = gen;
  p.pf = pf;
  p.pf_bytes = pf_bytes;
  p.err = err;
  p.wait_ns = wait_ns ? wait_ns : WAIT_LIMIT_NS;
  const dim3 grid(pl.units, n_heads, pl.splits);
  if (pl.qt == 2)
    return stamp ? run_attn_tc<2, 64, 5, 1, true>(p, grid, s)
                 : run_attn_tc<2, 64, 5, 1, false>(p, grid, s);
  if (pl.bn == 64)
    return stamp ? run_attn_tc<1, 64, 2, 1, true>(p, grid, s)
                 : run_attn_tc<1, 64, 2, 1, false>(p, grid, s);
  return stamp ? run_attn_tc<1, 128, 3, 2, true>(p, grid, s)
               : run_attn_tc<1, 128, 3, 2, false>(p, grid, s);
}

}  // namespace sl
