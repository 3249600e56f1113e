// Projection / FFN / LM-head GEMMs of the active rows on the 5th-generation
// tensor cores (tcgen05 + TMEM), operands staged by TMA.
//
//   C[M, N] = A[M, K] * B[N, K]^T      A = bf16 activations of the M active rows,
//                                      B = bf16 weights [out, in] (both K-major)
//
// Locked rows skip the query projection and the FFN (Abstract; Paper-Notes,
// "permanent locking"), so every GEMM here runs on the M active rows only:
// O(M d^2) work per layer (gist.science/nl section 2).
//
// Design (sm_100a, one CTA per SM, persistent):
//   warp 0      TMA producer: A tile 128x64 and B tile BNx64 per stage, 128B swizzle
//   warp 1      TMEM allocation + single-thread tcgen05.mma issue (M=128, N=BN, K=16)
//   warps 2..5  epilogue: tcgen05.ld 32x32b of the fp32 accumulator, fused
//               output transform (bf16 store with optional row scatter, fp32
//               residual add, SiLU(gate)*up, or fp32 split-K accumulation)
// Two TMEM accumulators (2 x BN columns) let the epilogue of one tile overlap
// the main loop of the next.  Every barrier wait is bounded; on timeout the
// kernel records it in the device error word and winds down.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"

namespace sl {

// ------------------------------------------------------------- host: TMA ---
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (PFN_cuTensorMapEncodeTiled_v12000)p;
  }
  return fn;
}

bool tma_encode(TmaMat *m, const void *ptr, int rows, int cols, int box_rows) {
  auto fn = encode_fn();
  if (!fn || rows <= 0 || cols % 64 != 0 || ((uintptr_t)ptr & 15) != 0) return false;
  cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(&m->map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), gdim,
                  gstride, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  m->ptr = ptr;
  m->rows = rows;
  m->cols = cols;
  m->box_rows = box_rows;
  return r == CUDA_SUCCESS;
}

// Output descriptor for the TMA epilogue: [rows][cols] with leading dimension
// ld (elements), 32-row boxes of 128 bytes (32 fp32 or 64 bf16 columns), 128-byte
// swizzle.  Rows past `rows` are clipped by the copy engine.
bool tma_encode_out(TmaMat *m, const void *ptr, int rows, int cols, int ld, bool f32) {
  auto fn = encode_fn();
  const int esz = f32 ? 4 : 2, box_cols = f32 ? 32 : 64;
  if (!fn || rows <= 0 || cols % box_cols != 0 || ld < cols || ((size_t)ld * esz) % 16 != 0 ||
      ((uintptr_t)ptr & 15) != 0)
    return false;
  cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)ld * esz};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(&m->map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                  2, const_cast<void *>(ptr), gdim, gstride, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  m->ptr = ptr;
  m->rows = rows;
  m->cols = cols;
  m->box_rows = 32;
  return r == CUDA_SUCCESS;
}

// --- CTA-pair (cluster of 2) helpers for the 2-SM MMA variant
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// shared::cluster address of the same shared-memory offset in CTA `rank`
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
  uint32_t out;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(saddr), "r"(rank));
  return out;
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
// TMA load into this CTA's shared memory whose completion is counted on the
// pair leader's barrier (cluster address); no multicast.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *map, int x, int y,
                                                 uint32_t leader_bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(leader_bar)
      : "memory");
}
__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// arrive on the barrier at this offset in both CTAs of the pair once the
// issued MMAs complete
__device__ __forceinline__ void tc_commit_pair_both(uint32_t bar) {
  const uint16_t mask = 0x3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar), "h"(mask)
      : "memory");
}
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

// ---------------------------------------------------------------- kernel ---
struct TcParams {
  CUtensorMap a;
  CUtensorMap b[3];
  CUtensorMap out_map;     // TMA epilogue destination (tma_out)
  int seg0, seg1;          // output column boundaries of segments 0 and 1
  int b_swiglu;            // 1: B tile = gate rows | up rows (halves of BN)
  int M, N, K;
  int m_tiles, n_tiles, splits, kb_per_split, kblocks, units;
  int stream_k;            // 1: balanced split of the tile x K-block space (see WorkIter)
  int tma_out;             // 1: RESID/ACCUM/SWIGLU tiles leave through out_map (see epilogue)
  void *out;
  int ldo;
  int ffn;                 // SWIGLU/ACCUM-swiglu: F (columns of one half)
  const int32_t *row_map;  // STORE: output row per A row; QKV: flat position per row
  int *err;
  // HEAD epilogue: previous logits (or null), per (row, vocab tile) records
  const bf16 *prev;
  float4 *stat;
  int *stat_idx;
  int mask_id;
  unsigned long long wait_ns;  // limit of every barrier wait (WAIT_LIMIT_NS by default)
  int lost_load;           // test hook: CTA 0 leaves out its first stage's copies
  int fixup;               // ACCUM: the split-K tile fix-up (see accum_fixup)
  unsigned int *fix_ctr;   // [ceil(M / 32)][n_tiles] arrival tickets, zero between uses
  bf16 *fix_act;           // gate/up fix-up output [M][ffn]
  // QKV epilogue: rotary table [n_ctx][64] (cos, sin), q out [M][d], cache k/v
  const float2 *rope;
  int n_ctx, dmodel;
  bf16 *q_out, *ck, *cv;
};

constexpr int GROUP_M = 16;
__host__ __device__ constexpr uint32_t tmem_cols_pow2(uint32_t n) {
  uint32_t c = 32;
  while (c < n) c <<= 1;
  return c;
}
// Epilogue staging: each of the 4 epilogue warps owns one 32-row x 128-byte box
// (128-byte swizzled, as the output descriptors expect).
constexpr int EPI_STAGING_BYTES = 4 * 4096;

// Unit u of m_tiles x n_tiles x splits: groups of GROUP_M row tiles walk the
// column tiles together, row tile fastest, so a weight tile is read from HBM
// once and re-read by the group's row tiles from L2.
__device__ __forceinline__ void decode_unit(const TcParams &p, int u, int splits, int &mt, int &nt,
                                            int &sp) {
  const int per_group = GROUP_M * p.n_tiles * splits;
  const int g = u / per_group;
  const int r = u - g * per_group;
  const int first_m = g * GROUP_M;
  const int gm = min(GROUP_M, p.m_tiles - first_m);
  mt = first_m + r % gm;
  const int nn = r / gm;
  nt = nn / splits;
  sp = nn - nt * splits;
}

// The work of one worker (a CTA, or a CTA pair) as a sequence of (output tile,
// K-block range) items; the producer, MMA and epilogue roles each walk the
// same sequence.  Grid-stride mode: units w, w + nw, ... of the m_tiles x
// n_tiles x splits units.  Stream-K mode: the worker's equal share
// [w I / nw, (w + 1) I / nw) of the I = tiles x kblocks iteration space, cut
// where it passes from one tile to the next, so that every worker runs the
// same number of K-blocks whatever the tile count (partial tiles are summed
// atomically by the epilogue).
struct WorkIter {
  long long pos, end, total;
  int step, nw;
  int ncontrib;            // partial tiles summed into the current item's tile
  __device__ __forceinline__ WorkIter(const TcParams &p, int w, int nw_) : nw(nw_) {
    if (p.stream_k) {
      total = (long long)p.m_tiles * p.n_tiles * p.kblocks;
      pos = total * w / nw;
      end = total * (w + 1) / nw;
      step = 0;
    } else {
      total = p.units;
      pos = w;
      end = p.units;
      step = nw;
    }
  }
  // Stream-K: the worker whose share holds iteration x (every share is
  // non-empty: the grid never exceeds the iteration count).
  __device__ __forceinline__ long long owner(long long x) const {
    return ((x + 1) * nw - 1) / total;
  }
  __device__ __forceinline__ bool next(const TcParams &p, int &mt, int &nt, int &kb0, int &kb1) {
    if (pos >= end) return false;
    int sp;
    if (p.stream_k) {
      const int t = (int)(pos / p.kblocks);
      kb0 = (int)(pos - (long long)t * p.kblocks);
      kb1 = (int)min((long long)p.kblocks, (long long)kb0 + (end - pos));
      pos = (long long)t * p.kblocks + kb1;
      decode_unit(p, t, 1, mt, nt, sp);
      const long long first = (long long)t * p.kblocks;
      ncontrib = (int)(owner(first + p.kblocks - 1) - owner(first) + 1);
    } else {
      decode_unit(p, (int)pos, p.splits, mt, nt, sp);
      kb0 = sp * p.kb_per_split;
      kb1 = min(p.kblocks, kb0 + p.kb_per_split);
      pos += step;
      ncontrib = p.splits;
    }
    return true;
  }
};

template <int BN, int STAGES, int MSUB>
struct TcSmem {
  static constexpr int A_BYTES = MSUB * 128 * 64 * 2;   // MSUB 128-row A tiles per stage
  static constexpr int B_BYTES = BN * 64 * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int EPI_OFF = STAGES * STAGE_BYTES;          // epilogue staging, 4 warps x 4 KB
  static constexpr int BAR_OFF = EPI_OFF + EPI_STAGING_BYTES;
  static constexpr int TOTAL = BAR_OFF + 256 + 1024;   // barriers + alignment slack
};

// B tile of K-block kb for output tile nt: BN rows of one weight segment, or
// BN/2 gate rows followed by the matching BN/2 up rows.
template <int BN>
__device__ __forceinline__ void load_b(const TcParams &p, uint32_t sb, int nt, int kb,
                                       uint32_t bar) {
  if (p.b_swiglu) {
    const int f0 = nt * (BN / 2);
    tma_load_2d(sb, &p.b[0], kb * 64, f0, bar);
    tma_load_2d(sb + (BN / 2) * 128, &p.b[1], kb * 64, f0, bar);
  } else {
    const int c0 = nt * BN;
    if (c0 < p.seg0) tma_load_2d(sb, &p.b[0], kb * 64, c0, bar);
    else if (c0 < p.seg1) tma_load_2d(sb, &p.b[1], kb * 64, c0 - p.seg0, bar);
    else tma_load_2d(sb, &p.b[2], kb * 64, c0 - p.seg1, bar);
  }
}

// Put 128 bytes of row `lane` into the warp's staging box (16-byte chunk j at
// j ^ (row % 8): the 128-byte swizzle, and conflict-free per 8 lanes) once the
// previous bulk copy out of the box has read it.
__device__ __forceinline__ void stage_wait(int lane) {
  if (lane == 0) bulk_wait_read0();
  __syncwarp();
}
__device__ __forceinline__ void stage_chunk(uint32_t stg, int lane, int j, uint32_t a, uint32_t b,
                                            uint32_t c, uint32_t d) {
  st_shared_v4(stg + lane * 128 + ((j ^ (lane & 7)) << 4), a, b, c, d);
}
__device__ __forceinline__ void stage_done() {
  fence_proxy_async_smem();
  __syncwarp();
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const uint32_t l = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
  const uint32_t h = __bfloat16_as_ushort(__float2bfloat16_rn(hi));
  return l | (h << 16);
}

// Split-K tile fix-up: once every partial tile of this warp's 32 rows has been
// added into the fp32 workspace (per row group and column tile, an arrival
// ticket counts the contributors), the warp that adds the last one applies
// the projection's finishing step to those rows itself and clears the
// workspace for the next split GEMM: RoPE of q and k and the cache scatter of
// k, v (fused Q|K|V), or SiLU(gate) * up (fused gate/up).  This replaces a
// separate finalize kernel and its launch boundary.
template <int BN>
__device__ __forceinline__ void accum_fixup(const TcParams &p, int row0, int nt, int ncontrib,
                                            int lane) {
  int last = 0;
  if (lane == 0) {
    bulk_wait0();                                  // this warp's reduce-adds are done
    asm volatile("fence.proxy.async.global;" ::: "memory");
    __threadfence();
    unsigned int *ctr = p.fix_ctr + (size_t)(row0 >> 5) * p.n_tiles + nt;
    last = atomicAdd(ctr, 1u) == (unsigned)(ncontrib - 1);
    if (last) *ctr = 0u;                           // ready for the next launch
  }
  last = __shfl_sync(0xffffffffu, last, 0);
  if (!last) return;
  __threadfence();
  const int r = row0 + lane;
  if (r >= p.M) return;
  float *wrow = reinterpret_cast<float *>(p.out) + (size_t)r * p.ldo;
  const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
  if (p.b_swiglu) {
    const int f0 = nt * (BN / 2);
#pragma unroll 1
    for (int c = 0; c < BN / 2; c += 8) {
      float4 *g = reinterpret_cast<float4 *>(wrow + f0 + c);
      float4 *u = reinterpret_cast<float4 *>(wrow + p.ffn + f0 + c);
      const float4 g0 = __ldcg(g), g1 = __ldcg(g + 1), u0 = __ldcg(u), u1 = __ldcg(u + 1);
      g[0] = z4; g[1] = z4; u[0] = z4; u[1] = z4;
      const float gv[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
      const float uv[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
      Pack8 o;
#pragma unroll
      for (int e = 0; e < 8; ++e) o.h[e] = __float2bfloat16_rn(silu_f(gv[e]) * uv[e]);
      *reinterpret_cast<uint4 *>(p.fix_act + (size_t)r * p.ffn + f0 + c) = o.u;
    }
    return;
  }
  // fused Q|K|V: the tile holds whole heads of one segment
  const int col0 = nt * BN;
  const int seg = col0 / p.dmodel;                 // 0 q, 1 k, 2 v
  const int pos_flat = p.row_map[r];
  const int pos = pos_flat % p.n_ctx;
  bf16 *dst_row = seg == 0 ? p.q_out + (size_t)r * p.dmodel
                           : (seg == 1 ? p.ck : p.cv) + (size_t)pos_flat * p.dmodel;
#pragma unroll 1
  for (int hd = 0; hd < BN / 128; ++hd) {
    const int cw = col0 + hd * 128;                // workspace column of the head
    const int cs = cw - seg * p.dmodel;            // its column in the segment
#pragma unroll 1
    for (int i0 = 0; i0 < 64; i0 += 8) {
      float4 *a = reinterpret_cast<float4 *>(wrow + cw + i0);
      float4 *b = reinterpret_cast<float4 *>(wrow + cw + 64 + i0);
      const float4 a0 = __ldcg(a), a1 = __ldcg(a + 1), b0 = __ldcg(b), b1 = __ldcg(b + 1);
      a[0] = z4; a[1] = z4; b[0] = z4; b[1] = z4;
      const float x0[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float x1[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
      Pack8 lo, hi;
      if (seg < 2) {
        const float4 *tab = reinterpret_cast<const float4 *>(p.rope + (size_t)pos * 64 + i0);
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
          const float4 cs4 = __ldg(tab + (e >> 1));    // (cos, sin) of pairs e and e + 1
          lo.h[e] = __float2bfloat16_rn(x0[e] * cs4.x - x1[e] * cs4.y);
          hi.h[e] = __float2bfloat16_rn(x1[e] * cs4.x + x0[e] * cs4.y);
          lo.h[e + 1] = __float2bfloat16_rn(x0[e + 1] * cs4.z - x1[e + 1] * cs4.w);
          hi.h[e + 1] = __float2bfloat16_rn(x1[e + 1] * cs4.z + x0[e + 1] * cs4.w);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          lo.h[e] = __float2bfloat16_rn(x0[e]);
          hi.h[e] = __float2bfloat16_rn(x1[e]);
        }
      }
      *reinterpret_cast<uint4 *>(dst_row + cs + i0) = lo.u;
      *reinterpret_cast<uint4 *>(dst_row + cs + 64 + i0) = hi.u;
    }
  }
}

// TMA epilogue of RESID / ACCUM (fp32 reduce-add) and SWIGLU (bf16 store): the
// warp's 32 rows x 32 (64) columns go through its staging box and leave as one
// bulk tensor copy, whole 128-byte lines; boxes past the live rows are skipped.
template <int BN, int EPI>
__device__ __forceinline__ void epilogue_tile_tma(const TcParams &p, uint32_t taddr, int row0,
                                                  int nt, uint32_t stg, int lane,
                                                  int ncontrib = 0) {
  if (row0 >= p.M) return;
  float v[32];
  if (EPI == EPI_SWIGLU) {
    const int f0 = nt * (BN / 2);
#pragma unroll 1
    for (int c = 0; c < BN / 2; c += 64) {
      stage_wait(lane);
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        float g[32];
        tmem_ld32(taddr + c + 32 * h, g);
        tmem_ld32(taddr + BN / 2 + c + 32 * h, v);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            w[e] = pack_bf16(silu_f(g[8 * j + 2 * e]) * v[8 * j + 2 * e],
                             silu_f(g[8 * j + 2 * e + 1]) * v[8 * j + 2 * e + 1]);
          stage_chunk(stg, lane, 4 * h + j, w[0], w[1], w[2], w[3]);
        }
      }
      stage_done();
      if (lane == 0) {
        tma_store_2d(&p.out_map, f0 + c, row0, stg);
        bulk_commit();
      }
    }
  } else {
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      tmem_ld32(taddr + c, v);
      int col = nt * BN + c;
      if (EPI == EPI_ACCUM && p.b_swiglu) {   // gate into [0, F), up into [F, 2F)
        const int half = BN / 2, f0 = nt * half;
        col = (c < half) ? (f0 + c) : (p.ffn + f0 + (c - half));
      }
      stage_wait(lane);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        stage_chunk(stg, lane, j, __float_as_uint(v[4 * j]), __float_as_uint(v[4 * j + 1]),
                    __float_as_uint(v[4 * j + 2]), __float_as_uint(v[4 * j + 3]));
      stage_done();
      if (lane == 0) {
        tma_reduce_add_2d(&p.out_map, col, row0, stg);
        bulk_commit();
      }
    }
    if (EPI == EPI_ACCUM && p.fixup) accum_fixup<BN>(p, row0, nt, ncontrib, lane);
  }
}

// Per-thread epilogue of one 128-row accumulator tile (STORE, QKV, and SWIGLU
// without an output descriptor): TMEM lane quarter of the calling warp (taddr
// carries the lane offset), A row r, output tile nt; each thread writes its row.
template <int BN, int EPI>
__device__ __forceinline__ void epilogue_tile(const TcParams &p, uint32_t taddr, int r, int nt) {
  const bool live = r < p.M;
  float v[32];
  if (EPI == EPI_SWIGLU) {
    const int f0 = nt * (BN / 2);
#pragma unroll 1
    for (int c = 0; c < BN / 2; c += 32) {
      float g[32];
      tmem_ld32(taddr + c, g);
      tmem_ld32(taddr + BN / 2 + c, v);
      if (live) {
        bf16 *dst = reinterpret_cast<bf16 *>(p.out) + (size_t)r * p.ldo + f0 + c;
#pragma unroll
        for (int i = 0; i < 32; i += 8) {
          Pack8 pk;
#pragma unroll
          for (int e = 0; e < 8; ++e) pk.h[e] = __float2bfloat16_rn(silu_f(g[i + e]) * v[i + e]);
          *reinterpret_cast<uint4 *>(dst + i) = pk.u;
        }
      }
    }
  } else if (EPI == EPI_QKV) {
    // whole heads per tile: pair (i, i + 64) of a head is rotated together
    const int col0 = nt * BN;
    const int seg = col0 / p.dmodel;              // 0 q, 1 k, 2 v
    const int pos_flat = live ? p.row_map[r] : 0;
    const int pos = pos_flat % p.n_ctx;
#pragma unroll 1
    for (int hd = 0; hd < BN / 128; ++hd) {
      const int cbase = col0 - seg * p.dmodel + hd * 128;   // column of the head in its segment
#pragma unroll 1
      for (int j = 0; j < 2; ++j) {
        float x2[32];
        tmem_ld32(taddr + hd * 128 + 32 * j, v);
        tmem_ld32(taddr + hd * 128 + 64 + 32 * j, x2);
        if (!live) continue;
        bf16 *dst;
        if (seg == 0) dst = p.q_out + (size_t)r * p.dmodel + cbase;
        else if (seg == 1) dst = p.ck + (size_t)pos_flat * p.dmodel + cbase;
        else dst = p.cv + (size_t)pos_flat * p.dmodel + cbase;
        if (seg < 2) {
          const float4 *tab =
              reinterpret_cast<const float4 *>(p.rope + (size_t)pos * 64 + 32 * j);
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float4 cs = __ldg(tab + (e >> 1));   // (cos, sin) of e and e+1
            const float a0 = v[e], b0 = x2[e], a1 = v[e + 1], b1 = x2[e + 1];
            v[e] = a0 * cs.x - b0 * cs.y;
            x2[e] = b0 * cs.x + a0 * cs.y;
            v[e + 1] = a1 * cs.z - b1 * cs.w;
            x2[e + 1] = b1 * cs.z + a1 * cs.w;
          }
        }
#pragma unroll
        for (int i = 0; i < 32; i += 8) {
          Pack8 lo, hi;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            lo.h[e] = __float2bfloat16_rn(v[i + e]);
            hi.h[e] = __float2bfloat16_rn(x2[i + e]);
          }
          *reinterpret_cast<uint4 *>(dst + 32 * j + i) = lo.u;
          *reinterpret_cast<uint4 *>(dst + 64 + 32 * j + i) = hi.u;
        }
      }
    }
  } else if (EPI == EPI_HEAD) {
    // Logits of the row's BN vocab entries, rounded to bf16 and stored; the
    // sure test's statistics are taken on the stored values, so they equal
    // what a separate pass over the stored logits would find: running max m,
    // sum of e = exp(z - m), sum of e (z - z_prev), and the best value over
    // v != mask_id with its lowest index.
    const int orow = live ? p.row_map[r] : 0;
    bf16 *dst = reinterpret_cast<bf16 *>(p.out) + (size_t)orow * p.ldo + nt * BN;
    const bf16 *zpr = p.prev ? p.prev + (size_t)orow * p.ldo + nt * BN : nullptr;
    float m = -INFINITY, se = 0.f, st = 0.f, bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      tmem_ld32(taddr + c, v);
      if (!live) continue;
      float cm = -INFINITY;
#pragma unroll
      for (int i = 0; i < 32; i += 8) {
        Pack8 pk;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          pk.h[e] = __float2bfloat16_rn(v[i + e]);
          v[i + e] = __bfloat162float(pk.h[e]);
          cm = fmaxf(cm, v[i + e]);
        }
        *reinterpret_cast<uint4 *>(dst + c + i) = pk.u;
      }
      if (cm > m) {
        const float sc = (m == -INFINITY) ? 0.f : __expf(m - cm);
        se *= sc;
        st = sc == 0.f ? 0.f : st * sc;
        m = cm;
      }
      float zp[32];
      if (zpr) {
#pragma unroll
        for (int i = 0; i < 32; i += 8) {
          Pack8 pk;
          pk.u = __ldcs(reinterpret_cast<const uint4 *>(zpr + c + i));
#pragma unroll
          for (int e = 0; e < 8; ++e) zp[i + e] = __bfloat162float(pk.h[e]);
        }
      }
      // the chunk's terms are summed in groups of 8, then added to the running
      // sums, so that small terms do not each round against a sum near 1
#pragma unroll
      for (int i = 0; i < 32; i += 8) {
        float gs = 0.f, gt = 0.f;
#pragma unroll
        for (int e8 = 0; e8 < 8; ++e8) {
          const float e = (m == -INFINITY) ? 0.f : __expf(v[i + e8] - m);
          gs += e;
          if (zpr && e > 0.f) gt = fmaf(e, v[i + e8] - zp[i + e8], gt);
          const int vi = nt * BN + c + i + e8;
          if (vi != p.mask_id && v[i + e8] > bv) { bv = v[i + e8]; bi = vi; }
        }
        se += gs;
        st += gt;
      }
    }
    if (live) {
      const size_t rec = (size_t)r * p.n_tiles + nt;
      p.stat[rec] = make_float4(m, se, st, bv);
      p.stat_idx[rec] = bi;
    }
  } else {
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      tmem_ld32(taddr + c, v);
      if (!live) continue;
      // EPI_STORE
      const int orow = p.row_map ? p.row_map[r] : r;
      bf16 *dst = reinterpret_cast<bf16 *>(p.out) + (size_t)orow * p.ldo + nt * BN + c;
#pragma unroll
      for (int i = 0; i < 32; i += 8) {
        Pack8 pk;
#pragma unroll
        for (int e = 0; e < 8; ++e) pk.h[e] = __float2bfloat16_rn(v[i + e]);
        *reinterpret_cast<uint4 *>(dst + i) = pk.u;
      }
    }
  }
}

// MSUB = 1: one 128-row tile of A per unit; MSUB = 2: two (256 rows) sharing
// each B tile, accumulated in two TMEM accumulators (halves the weight-tile
// re-reads when 128 < M <= 256).  Accumulators are double-buffered when
// 2 * MSUB * BN TMEM columns fit in 512.
template <int BN, int STAGES, int EPI, int MSUB>
__global__ void __launch_bounds__(192, 1) gemm_tc_kernel(const __grid_constant__ TcParams p) {
  using L = TcSmem<BN, STAGES, MSUB>;
  constexpr int ACC_BUFS = (2 * MSUB * BN <= 512) ? 2 : 1;
  constexpr int ACC_COLS = MSUB * BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = s_addr(smem);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::BAR_OFF);
  // bars: full[STAGES], empty[STAGES], tfull[2], tempty[2], drain
  const uint32_t bar0 = s_addr(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::BAR_OFF + 8 * (2 * STAGES + 5));
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // tcgen05.alloc takes a power of two >= 32 columns
  constexpr uint32_t TMEM_COLS = tmem_cols_pow2(ACC_BUFS * ACC_COLS);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 4);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    tma_prefetch_desc(&p.a);
    tma_prefetch_desc(&p.b[0]);
  }
  __syncthreads();                       // barrier initialisation visible to every role
  // TMEM is allocated after the producer has started: a CTA that becomes
  // resident while the previous kernel's CTA on the SM still holds the TMEM
  // streams its first weight tiles while it waits for the allocation.
  uint32_t tmem_base = 0;
  if (warp >= 1) {
    if (warp == 1) {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       s_addr(tmem_slot)),
                   "r"(TMEM_COLS)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    named_bar_sync(1, 160);              // MMA warp + 4 epilogue warps
    tc_fence_after();
    tmem_base = *tmem_slot;
  }

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      // Weight tiles do not depend on the previous kernel: issue the B loads of
      // the first stages of this CTA's first unit before waiting on it, so the
      // weight stream starts while the previous kernel drains.
      // Test hook (lost_load): CTA 0 never issues the copies of its first
      // stage, so the MMA warp's wait for them runs out and the kernel winds
      // down through its error path; nothing is read or written out of place.
      const bool lost = p.lost_load && blockIdx.x == 0;
      int npre = 0;
      WorkIter first_it(p, blockIdx.x, gridDim.x);
      int mt, nt, kb0, kb1;
      if (first_it.next(p, mt, nt, kb0, kb1)) {
        npre = min(STAGES, kb1 - kb0);
        for (int i = 0; i < npre; ++i) {
          if (lost && i == 0) continue;
          const uint32_t sb = sbase + i * L::STAGE_BYTES + L::A_BYTES;
          mbar_expect_tx(full_bar(i), L::STAGE_BYTES);
          load_b<BN>(p, sb, nt, kb0 + i, full_bar(i));
        }
      }
      pdl_wait();
      int stage = 0;
      uint32_t phase = 0;
      int last_stage = -1;
      uint32_t last_phase = 0;
      bool ok = true;
      bool first = true;
      WorkIter it(p, blockIdx.x, gridDim.x);
      while (ok && it.next(p, mt, nt, kb0, kb1)) {
        for (int kb = kb0; kb < kb1; ++kb) {
          const bool pre = first && (kb - kb0) < npre;
          if (!pre) {
            if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, p.wait_ns)) {
              ok = false;
              break;
            }
            mbar_expect_tx(full_bar(stage), L::STAGE_BYTES);
          }
          const uint32_t sa = sbase + stage * L::STAGE_BYTES;
          if (!(lost && first && kb == kb0)) {
#pragma unroll
            for (int sub = 0; sub < MSUB; ++sub)
              tma_load_2d(sa + sub * 16384, &p.a, kb * 64, (mt * MSUB + sub) * 128,
                          full_bar(stage));
            if (!pre) load_b<BN>(p, sa + L::A_BYTES, nt, kb, full_bar(stage));
            last_stage = stage;
            last_phase = phase;
          }
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        first = false;
      }
      pdl_trigger();
      if (!ok) {
        atomicExch(p.err, DEV_TIMEOUT_PRODUCER);
        *abort_flag = 1;
      }
      // make sure the last issued copy has landed before the CTA can exit
      if (last_stage >= 0) {
        volatile int never = 0;
        mbar_wait(full_bar(last_stage), last_phase, &never, p.wait_ns);
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32<BN>();
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      WorkIter it(p, blockIdx.x, gridDim.x);
      int mt, nt, kb0, kb1;
      while (ok && it.next(p, mt, nt, kb0, kb1)) {
        if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, abort_flag, p.wait_ns)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * ACC_COLS);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag, p.wait_ns)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = sbase + stage * L::STAGE_BYTES;
          const uint32_t sb = sa + L::A_BYTES;
          const uint64_t bdesc = smem_desc_sw128(sb);
#pragma unroll
          for (int sub = 0; sub < MSUB; ++sub) {
            const uint64_t adesc = smem_desc_sw128(sa + sub * 16384);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              tc_mma(d_tmem + sub * BN, adesc + 2 * k, bdesc + 2 * k, idesc,
                     (kb > kb0 || k > 0) ? 1u : 0u);
          }
          tc_commit(empty_bar(stage));
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(tfull_bar(acc));
        if (++acc == ACC_BUFS) { acc = 0; acc_phase ^= 1u; }
      }
      if (!ok) {
        atomicExch(p.err, DEV_TIMEOUT_MMA);
        *abort_flag = 1;
      }
      // wait for every issued MMA to finish before TMEM can be released
      tc_commit(drain_bar);
      volatile int never = 0;
      mbar_wait(drain_bar, 0, &never, p.wait_ns);
    }
  } else {
    // ---------------------------------------------------------- epilogue
    pdl_wait();                             // outputs may be in use by the previous kernel
    const int q = warp & 3;                 // TMEM lane quarter of this warp
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    WorkIter it(p, blockIdx.x, gridDim.x);
    int mt, nt, kb0, kb1;
    while (it.next(p, mt, nt, kb0, kb1)) {
      if (!mbar_wait(tfull_bar(acc), acc_phase, abort_flag, p.wait_ns)) { ok = false; break; }
      tc_fence_after();
#pragma unroll 1
      for (int sub = 0; sub < MSUB; ++sub) {
      const int r = (mt * MSUB + sub) * 128 + q * 32 + lane;
      const uint32_t taddr = tmem_base + (uint32_t)(acc * ACC_COLS + sub * BN) +
                             ((uint32_t)(q * 32) << 16);
      if constexpr (EPI == EPI_RESID || EPI == EPI_ACCUM)
        epilogue_tile_tma<BN, EPI>(p, taddr, r - lane, nt, sbase + L::EPI_OFF + q * 4096, lane,
                                   it.ncontrib);
      else if (EPI == EPI_SWIGLU && (BN / 2) % 64 == 0 && p.tma_out)
        epilogue_tile_tma<BN, EPI>(p, taddr, r - lane, nt, sbase + L::EPI_OFF + q * 4096, lane);
      else
        epilogue_tile<BN, EPI>(p, taddr, r, nt);
      }   // sub
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty_bar(acc));
      if (++acc == ACC_BUFS) { acc = 0; acc_phase ^= 1u; }

    }
    if (lane == 0) bulk_wait0();          // staged tiles written before the CTA exits
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
                 "r"(TMEM_COLS)
                 : "memory");
  }
}

// ------------------------------------------------ swapped-operand kernel ---
// D^T = W X^T for few rows (M <= 256): the weight tile is the MMA's 128-row A
// operand and the M active rows are its N dimension (rounded up to 32), so the
// tensor-core work follows M instead of a 256-row padded tile.  TMEM then holds
// output features on its lanes and rows on its columns; the epilogue reads 32
// rows of a lane's feature at a time, writes them transposed into the warp's
// 32-row x 128-byte staging box (same 128-byte swizzle as the other fp32
// epilogues) and adds the box into the fp32 destination with a TMA reduce:
// the residual stream (RESID) or a zeroed workspace whose finishing pass
// (RoPE + cache scatter, SiLU(gate) * up) runs as its own kernel (ACCUM).
// A stage holds the unit's two 128-row activation boxes (rows past M read as
// zeros) and 128 weight rows (64 gate + 64 up rows for the gate/up GEMM).
template <int STAGES>
struct SwSmem {
  static constexpr int A_BYTES = 2 * 128 * 64 * 2;     // 256 activation rows
  static constexpr int B_BYTES = 128 * 64 * 2;         // 128 weight rows
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int EPI_OFF = STAGES * STAGE_BYTES;
  static constexpr int BAR_OFF = EPI_OFF + EPI_STAGING_BYTES;
  static constexpr int TOTAL = BAR_OFF + 256 + 1024;
};

template <int STAGES, int EPI>
__global__ void __launch_bounds__(192, 1) gemm_swap_kernel(const __grid_constant__ TcParams p) {
  using L = SwSmem<STAGES>;
  constexpr int ACC_COLS = 256;                        // up to 256 rows per accumulator
  constexpr uint32_t TMEM_COLS = 512;                  // two accumulators
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = s_addr(smem);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::BAR_OFF);
  const uint32_t bar0 = s_addr(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::BAR_OFF + 8 * (2 * STAGES + 5));
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int np = min(256, (p.M + 31) & ~31);           // MMA N: rows rounded up to 32

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 4);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    tma_prefetch_desc(&p.a);
    tma_prefetch_desc(&p.b[0]);
  }
  __syncthreads();
  uint32_t tmem_base = 0;
  if (warp >= 1) {
    if (warp == 1) {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       s_addr(tmem_slot)),
                   "r"(TMEM_COLS)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    named_bar_sync(1, 160);
    tc_fence_after();
    tmem_base = *tmem_slot;
  }

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      // the first unit's weight tiles before the wait on the previous kernel
      int npre = 0;
      WorkIter first_it(p, blockIdx.x, gridDim.x);
      int mt, nt, kb0, kb1;
      if (first_it.next(p, mt, nt, kb0, kb1)) {
        npre = min(STAGES, kb1 - kb0);
        for (int i = 0; i < npre; ++i) {
          mbar_expect_tx(full_bar(i), L::STAGE_BYTES);
          load_b<128>(p, sbase + i * L::STAGE_BYTES + L::A_BYTES, nt, kb0 + i, full_bar(i));
        }
      }
      pdl_wait();
      int stage = 0;
      uint32_t phase = 0;
      int last_stage = -1;
      uint32_t last_phase = 0;
      bool ok = true, first = true;
      WorkIter it(p, blockIdx.x, gridDim.x);
      while (ok && it.next(p, mt, nt, kb0, kb1)) {
        for (int kb = kb0; kb < kb1; ++kb) {
          const bool pre = first && (kb - kb0) < npre;
          if (!pre) {
            if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, p.wait_ns)) {
              ok = false;
              break;
            }
            mbar_expect_tx(full_bar(stage), L::STAGE_BYTES);
          }
          const uint32_t sa = sbase + stage * L::STAGE_BYTES;
          tma_load_2d(sa, &p.a, kb * 64, 0, full_bar(stage));
          tma_load_2d(sa + 16384, &p.a, kb * 64, 128, full_bar(stage));
          if (!pre) load_b<128>(p, sa + L::A_BYTES, nt, kb, full_bar(stage));
          last_stage = stage;
          last_phase = phase;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        first = false;
      }
      pdl_trigger();
      if (!ok) {
        atomicExch(p.err, DEV_TIMEOUT_PRODUCER);
        *abort_flag = 1;
      }
      if (last_stage >= 0) {
        volatile int never = 0;
        mbar_wait(full_bar(last_stage), last_phase, &never, p.wait_ns);
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------------- MMA
    if (lane == 0) {
      // M = 128 weight rows, N = np activation rows (a multiple of 32 <= 256)
      const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(np >> 3) << 17) |
                             ((uint32_t)(128 >> 4) << 24);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      WorkIter it(p, blockIdx.x, gridDim.x);
      int mt, nt, kb0, kb1;
      while (ok && it.next(p, mt, nt, kb0, kb1)) {
        if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, abort_flag, p.wait_ns)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * ACC_COLS);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag, p.wait_ns)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = sbase + stage * L::STAGE_BYTES;
          const uint64_t wdesc = smem_desc_sw128(sa + L::A_BYTES);   // weights: the A operand
          const uint64_t xdesc = smem_desc_sw128(sa);                // rows: the B operand
#pragma unroll
          for (int k = 0; k < 4; ++k)
            tc_mma(d_tmem, wdesc + 2 * k, xdesc + 2 * k, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
          tc_commit(empty_bar(stage));
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(tfull_bar(acc));
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (!ok) {
        atomicExch(p.err, DEV_TIMEOUT_MMA);
        *abort_flag = 1;
      }
      tc_commit(drain_bar);
      volatile int never = 0;
      mbar_wait(drain_bar, 0, &never, p.wait_ns);
    }
  } else {
    // ---------------------------------------------------------- epilogue
    pdl_wait();
    const int q = warp & 3;                 // TMEM lane quarter: features q*32 .. q*32+31
    const uint32_t stg = sbase + L::EPI_OFF + q * 4096;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    WorkIter it(p, blockIdx.x, gridDim.x);
    int mt, nt, kb0, kb1;
    while (it.next(p, mt, nt, kb0, kb1)) {
      if (!mbar_wait(tfull_bar(acc), acc_phase, abort_flag, p.wait_ns)) { ok = false; break; }
      tc_fence_after();
      // destination column of this warp's 32 features
      int col = nt * 128 + q * 32;
      if (p.b_swiglu) {                     // gate features into [0, F), up into [F, 2F)
        const int f0 = nt * 64;
        col = q < 2 ? f0 + q * 32 : p.ffn + f0 + (q - 2) * 32;
      }
      const uint32_t taddr = tmem_base + (uint32_t)(acc * ACC_COLS) + ((uint32_t)(q * 32) << 16);
#pragma unroll 1
      for (int r0 = 0; r0 < np && r0 < p.M; r0 += 32) {
        float v[32];
        tmem_ld32(taddr + r0, v);            // rows r0 .. r0+31 of this lane's feature
        stage_wait(lane);
        // element (row i, feature lane) of the 32 x 32 fp32 box: 16-byte chunk
        // lane / 4 of row i, swizzled by row i % 8
#pragma unroll
        for (int i = 0; i < 32; ++i)
          asm volatile("st.shared.f32 [%0], %1;" ::"r"(stg + i * 128 +
                                                         ((((uint32_t)lane >> 2) ^ (i & 7)) << 4) +
                                                         ((lane & 3) << 2)),
                       "f"(v[i])
                       : "memory");
        stage_done();
        if (lane == 0) {
          tma_reduce_add_2d(&p.out_map, col, r0, stg);
          bulk_commit();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty_bar(acc));
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    if (lane == 0) bulk_wait0();
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
                 "r"(TMEM_COLS)
                 : "memory");
  }
}

// ------------------------------------------------------ CTA-pair kernel ---
// The same GEMM with 2-SM tensor-core instructions: a cluster of two CTAs
// computes a 256 x BN tile; each CTA stages its own 128 rows of A and its half
// (BN/2 rows) of the weight tile, the pair leader issues tcgen05.mma.cta_group::2
// (M = 256) over both CTAs' shared memory, and each CTA's TMEM holds the
// accumulator of its 128 rows.  Per SM this halves the weight-tile traffic
// from L2 and the shared-memory operand reads of the 1-SM kernel.
template <int BN, int STAGES, int EPI>
__global__ void __launch_bounds__(192, 1) gemm_tc2_kernel(const __grid_constant__ TcParams p) {
  constexpr int A_BYTES = 128 * 64 * 2;
  constexpr int B_BYTES = (BN / 2) * 64 * 2;
  constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  constexpr int EPI_OFF = STAGES * STAGE_BYTES;
  constexpr int BAR_OFF = EPI_OFF + EPI_STAGING_BYTES;
  constexpr uint32_t TMEM_COLS = tmem_cols_pow2(2 * BN);
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = s_addr(smem);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + BAR_OFF);
  const uint32_t bar0 = s_addr(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + BAR_OFF + 8 * (2 * STAGES + 5));
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 8);     // 4 epilogue warps in each CTA
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    tma_prefetch_desc(&p.a);
    tma_prefetch_desc(&p.b[0]);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     s_addr(tmem_slot)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      auto load_b_half = [&](uint32_t sb, int nt, int kb, uint32_t bar) {
        if (p.b_swiglu) {
          tma_load_2d_pair(sb, &p.b[rank], kb * 64, nt * (BN / 2), bar);
        } else {
          const int c0 = nt * BN + (int)rank * (BN / 2);
          if (c0 < p.seg0) tma_load_2d_pair(sb, &p.b[0], kb * 64, c0, bar);
          else if (c0 < p.seg1) tma_load_2d_pair(sb, &p.b[1], kb * 64, c0 - p.seg0, bar);
          else tma_load_2d_pair(sb, &p.b[2], kb * 64, c0 - p.seg1, bar);
        }
      };
      int npre = 0;
      WorkIter first_it(p, pair, n_pairs);
      int mt, nt, kb0, kb1;
      if (first_it.next(p, mt, nt, kb0, kb1)) {
        npre = min(STAGES, kb1 - kb0);
        for (int i = 0; i < npre; ++i) {
          if (leader) mbar_expect_tx(full_bar(i), 2 * STAGE_BYTES);
          load_b_half(sbase + i * STAGE_BYTES + A_BYTES, nt, kb0 + i, map_to_rank(full_bar(i), 0));
        }
      }
      pdl_wait();
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true, first = true;
      WorkIter it(p, pair, n_pairs);
      while (ok && it.next(p, mt, nt, kb0, kb1)) {
        for (int kb = kb0; kb < kb1; ++kb) {
          const bool pre = first && (kb - kb0) < npre;
          if (!pre) {
            if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, p.wait_ns)) { ok = false; break; }
            if (leader) mbar_expect_tx(full_bar(stage), 2 * STAGE_BYTES);
          }
          const uint32_t sa = sbase + stage * STAGE_BYTES;
          const uint32_t lbar = map_to_rank(full_bar(stage), 0);
          tma_load_2d_pair(sa, &p.a, kb * 64, mt * 256 + (int)rank * 128, lbar);
          if (!pre) load_b_half(sa + A_BYTES, nt, kb, lbar);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        first = false;
      }
      pdl_trigger();
      if (!ok) {
        atomicExch(p.err, DEV_TIMEOUT_PRODUCER);
        *abort_flag = 1;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------- MMA (pair leader)
    if (lane == 0 && leader) {
      constexpr uint32_t idesc = idesc_bf16_f32<BN, 256>();
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      WorkIter it(p, pair, n_pairs);
      int mt, nt, kb0, kb1;
      while (ok && it.next(p, mt, nt, kb0, kb1)) {
        if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, abort_flag, p.wait_ns)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag, p.wait_ns)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = sbase + stage * STAGE_BYTES;
          const uint64_t adesc = smem_desc_sw128(sa);
          const uint64_t bdesc = smem_desc_sw128(sa + A_BYTES);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            tc_mma_pair(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
          tc_commit_pair_both(empty_bar(stage));
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit_pair_both(tfull_bar(acc));
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (!ok) {
        atomicExch(p.err, DEV_TIMEOUT_MMA);
        *abort_flag = 1;
      }
      tc_commit_pair(drain_bar);
      volatile int never = 0;
      mbar_wait(drain_bar, 0, &never, p.wait_ns);
    }
  } else {
    // ------------------------------------------------- epilogue (both CTAs)
    pdl_wait();
    const int q = warp & 3;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    WorkIter it(p, pair, n_pairs);
    int mt, nt, kb0, kb1;
    while (it.next(p, mt, nt, kb0, kb1)) {
      if (!mbar_wait(tfull_bar(acc), acc_phase, abort_flag, p.wait_ns)) { ok = false; break; }
      tc_fence_after();
      const int r = mt * 256 + (int)rank * 128 + q * 32 + lane;
      const uint32_t taddr = tmem_base + (uint32_t)(acc * BN) + ((uint32_t)(q * 32) << 16);
      if constexpr (EPI == EPI_RESID || EPI == EPI_ACCUM)
        epilogue_tile_tma<BN, EPI>(p, taddr, r - lane, nt, sbase + EPI_OFF + q * 4096, lane,
                                   it.ncontrib);
      else if (EPI == EPI_SWIGLU && (BN / 2) % 64 == 0 && p.tma_out)
        epilogue_tile_tma<BN, EPI>(p, taddr, r - lane, nt, sbase + EPI_OFF + q * 4096, lane);
      else
        epilogue_tile<BN, EPI>(p, taddr, r, nt);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(map_to_rank(tempty_bar(acc), 0));
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    if (lane == 0) bulk_wait0();          // staged tiles written before the CTA exits
    if (!ok && lane == 0) {
      atomicExch(p.err, DEV_TIMEOUT_EPI);
      *abort_flag = 1;
    }
  }

  // neither CTA leaves while the pair's MMAs may still read its shared memory
  // or its epilogue may still signal the leader
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(TMEM_COLS)
                 : "memory");
  }
}

// ------------------------------------------------------------------ host ---
template <int BN, int STAGES, int EPI, int MSUB>
static cudaError_t run_tc(const TcParams &p, int grid, cudaStream_t s) {
  cudaError_t err = cudaSuccess;
  using L = TcSmem<BN, STAGES, MSUB>;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<BN, STAGES, EPI, MSUB>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::TOTAL);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  err = launch_k(gemm_tc_kernel<BN, STAGES, EPI, MSUB>, grid, 192, L::TOTAL, s, p);
  return err;
}

// `pairs` CTA pairs, capped at the number of pairs the GPU holds at once
// (a GPC with an odd number of usable SMs leaves one SM out of the pairing).
template <int BN, int STAGES, int EPI>
static cudaError_t run_tc2(const TcParams &p, int pairs, cudaStream_t s) {
  constexpr int SMEM = STAGES * (16384 + (BN / 2) * 128) + EPI_STAGING_BYTES + 256 + 1024;
  static int max_pairs = 0;
  if (max_pairs == 0) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tc2_kernel<BN, STAGES, EPI>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs);
    cfg.blockDim = dim3(192);
    cfg.dynamicSmemBytes = SMEM;
    cudaLaunchAttribute at;
    at.id = cudaLaunchAttributeClusterDimension;
    at.val.clusterDim.x = 2;
    at.val.clusterDim.y = 1;
    at.val.clusterDim.z = 1;
    cfg.attrs = &at;
    cfg.numAttrs = 1;
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, gemm_tc2_kernel<BN, STAGES, EPI>, &cfg);
    if (e != cudaSuccess) return e;
    if (n <= 0) return cudaErrorInvalidConfiguration;
    max_pairs = n;
  }
  if (pairs > max_pairs) pairs = max_pairs;
  return launch_k_cluster2(gemm_tc2_kernel<BN, STAGES, EPI>, 2 * pairs, 192, SMEM, s, p);
}

template <int STAGES, int EPI>
static cudaError_t run_swap(const TcParams &p, int grid, cudaStream_t s) {
  using L = SwSmem<STAGES>;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(gemm_swap_kernel<STAGES, EPI>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::TOTAL);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  return launch_k(gemm_swap_kernel<STAGES, EPI>, grid, 192, L::TOTAL, s, p);
}

template <int BN, int STAGES>
static cudaError_t run_epi2(int epi, const TcParams &p, int pairs, cudaStream_t s) {
  switch (epi) {
    case EPI_STORE: return run_tc2<BN, STAGES, EPI_STORE>(p, pairs, s);
    case EPI_RESID: return run_tc2<BN, STAGES, EPI_RESID>(p, pairs, s);
    case EPI_SWIGLU: return run_tc2<BN, STAGES, EPI_SWIGLU>(p, pairs, s);
    case EPI_ACCUM: return run_tc2<BN, STAGES, EPI_ACCUM>(p, pairs, s);
    case EPI_QKV: return run_tc2<BN, STAGES, EPI_QKV>(p, pairs, s);
    case EPI_HEAD: return run_tc2<BN, STAGES, EPI_HEAD>(p, pairs, s);
  }
  return cudaErrorInvalidValue;
}

template <int BN, int STAGES, int MSUB>
static cudaError_t run_epi(int epi, const TcParams &p, int grid, cudaStream_t s) {
  switch (epi) {
    case EPI_STORE: return run_tc<BN, STAGES, EPI_STORE, MSUB>(p, grid, s);
    case EPI_RESID: return run_tc<BN, STAGES, EPI_RESID, MSUB>(p, grid, s);
    case EPI_SWIGLU: return run_tc<BN, STAGES, EPI_SWIGLU, MSUB>(p, grid, s);
    case EPI_ACCUM: return run_tc<BN, STAGES, EPI_ACCUM, MSUB>(p, grid, s);
    case EPI_QKV: return run_tc<BN, STAGES, EPI_QKV, MSUB>(p, grid, s);
    case EPI_HEAD: return run_tc<BN, STAGES, EPI_HEAD, MSUB>(p, grid, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_gemm_tc(const TcGemmArgs &a, int num_sms, int *err, cudaStream_t s) {
  if (a.M <= 0) return cudaSuccess;
  const int bn = a.bn;
  if (a.swap) {
    // swapped operands: 128 weight rows per tile, at most 256 rows, the fp32
    // reduce epilogues only (no fix-up, no stream-K)
    if (bn != 128 || a.M > 256 || a.K % 64 != 0 || a.N % 128 != 0 || a.pair || a.fix_ctr ||
        (a.epi != EPI_RESID && a.epi != EPI_ACCUM) || !a.OUT || a.splits < 1)
      return cudaErrorInvalidValue;
    if (a.b_swiglu && (a.N % 2 != 0 || (a.N / 2) % 64 != 0)) return cudaErrorInvalidValue;
    TcParams p;
    memset(&p, 0, sizeof(p));
    p.a = a.A->map;
    for (int i = 0; i < 3; ++i)
      if (a.B[i]) p.b[i] = a.B[i]->map;
    p.b_swiglu = a.b_swiglu ? 1 : 0;
    p.seg0 = a.n_seg[0];
    p.seg1 = a.n_seg[0] + a.n_seg[1];
    if (!a.b_swiglu && p.seg0 == 0) p.seg0 = a.N;
    if (p.seg1 < p.seg0) p.seg1 = p.seg0;
    p.M = a.M;
    p.N = a.N;
    p.K = a.K;
    p.m_tiles = 1;
    p.n_tiles = a.N / 128;
    p.kblocks = a.K / 64;
    int splits = a.splits > p.kblocks ? p.kblocks : a.splits;
    p.kb_per_split = (p.kblocks + splits - 1) / splits;
    p.splits = (p.kblocks + p.kb_per_split - 1) / p.kb_per_split;
    p.units = p.n_tiles * p.splits;
    p.out_map = a.OUT->map;
    p.tma_out = 1;
    p.out = a.out;
    p.ldo = a.ldo;
    p.ffn = a.N / 2;
    p.err = err;
    p.wait_ns = a.wait_ns ? a.wait_ns : WAIT_LIMIT_NS;
    const int grid = p.units < num_sms ? p.units : num_sms;
    return a.epi == EPI_RESID ? run_swap<4, EPI_RESID>(p, grid, s)
                              : run_swap<4, EPI_ACCUM>(p, grid, s);
  }
  if ((bn != 64 && bn != 128 && bn != 192 && bn != 256) || a.K % 64 != 0 || a.N % bn != 0)
    return cudaErrorInvalidValue;
  const bool swiglu_b = a.b_swiglu != 0;
  if (a.epi == EPI_SWIGLU && !swiglu_b) return cudaErrorInvalidValue;
  TcParams p;
  memset(&p, 0, sizeof(p));
  p.a = a.A->map;
  for (int i = 0; i < 3; ++i)
    if (a.B[i]) p.b[i] = a.B[i]->map;
  p.b_swiglu = swiglu_b ? 1 : 0;
  p.seg0 = a.n_seg[0];
  p.seg1 = a.n_seg[0] + a.n_seg[1];
  if (!swiglu_b && p.seg0 == 0) p.seg0 = a.N;    // single segment
  if (p.seg1 < p.seg0) p.seg1 = p.seg0;
  p.M = a.M;
  p.N = a.N;
  p.K = a.K;
  const bool pair_mma = a.pair != 0;
  if (pair_mma && bn < 128) return cudaErrorInvalidValue;
  const int msub = (a.msub == 2 || pair_mma) ? 2 : 1;   // a pair owns 256 rows
  p.m_tiles = (a.M + 128 * msub - 1) / (128 * msub);
  p.n_tiles = a.N / bn;
  p.kblocks = a.K / 64;
  // splits < 0: stream-K (partial sums must be summable: RESID and ACCUM only)
  const bool stream_k = a.splits < 0 && (a.epi == EPI_RESID || a.epi == EPI_ACCUM);
  int splits = a.splits < 1 ? 1 : a.splits;
  if (a.epi == EPI_STORE || a.epi == EPI_QKV || a.epi == EPI_SWIGLU || a.epi == EPI_HEAD)
    splits = 1;
  if (a.epi == EPI_HEAD && (!a.row_map || !a.stat || !a.stat_idx)) return cudaErrorInvalidValue;
  if (a.epi == EPI_QKV && (bn % 128 != 0 || !a.row_map || !a.rope || !a.q_out || !a.ck || !a.cv ||
                           (a.N % 3) != 0 || ((a.N / 3) % 128) != 0))
    return cudaErrorInvalidValue;
  if (splits > p.kblocks) splits = p.kblocks;
  p.kb_per_split = (p.kblocks + splits - 1) / splits;
  p.splits = (p.kblocks + p.kb_per_split - 1) / p.kb_per_split;   // no empty split
  p.units = p.m_tiles * p.n_tiles * p.splits;
  p.stream_k = stream_k ? 1 : 0;
  if ((a.epi == EPI_RESID || a.epi == EPI_ACCUM) && !a.OUT) return cudaErrorInvalidValue;
  if (a.OUT && (a.epi == EPI_RESID || a.epi == EPI_ACCUM ||
                (a.epi == EPI_SWIGLU && (bn / 2) % 64 == 0))) {
    p.out_map = a.OUT->map;
    p.tma_out = 1;
  }
  // stream-K: one worker per SM (CTA pair), never more than there are K-blocks
  const long long sk_iters = (long long)p.m_tiles * p.n_tiles * p.kblocks;
  p.out = a.out;
  p.ldo = a.ldo;
  p.ffn = a.N / 2;
  p.row_map = a.row_map;
  p.err = err;
  p.wait_ns = a.wait_ns ? a.wait_ns : WAIT_LIMIT_NS;
  p.lost_load = a.lost_load && !pair_mma ? 1 : 0;
  if (a.epi == EPI_ACCUM && a.fix_ctr) {
    // the fix-up needs whole heads per Q|K|V tile and the gate/up output
    if (!swiglu_b && (bn % 128 != 0 || !a.row_map || !a.rope || !a.q_out || !a.ck || !a.cv ||
                      a.N % 3 != 0))
      return cudaErrorInvalidValue;
    if (swiglu_b && !a.fix_act) return cudaErrorInvalidValue;
    p.fixup = 1;
    p.fix_ctr = a.fix_ctr;
    p.fix_act = (bf16 *)a.fix_act;
  }
  p.rope = a.rope;
  p.n_ctx = a.n_ctx;
  p.dmodel = (a.epi == EPI_QKV || (p.fixup && !swiglu_b)) ? a.N / 3 : 0;
  p.prev = (const bf16 *)a.prev;
  p.stat = a.stat;
  p.stat_idx = a.stat_idx;
  p.mask_id = a.mask_id;
  p.q_out = (bf16 *)a.q_out;
  p.ck = (bf16 *)a.ck;
  p.cv = (bf16 *)a.cv;
  if (pair_mma) {
    const long long work = stream_k ? sk_iters : p.units;
    const int pairs = work < num_sms / 2 ? (int)work : num_sms / 2;
    if (bn == 256) return run_epi2<256, 6>(a.epi, p, pairs, s);
    if (bn == 192) return run_epi2<192, 7>(a.epi, p, pairs, s);
    return run_epi2<128, 6>(a.epi, p, pairs, s);
  }
  const long long work = stream_k ? sk_iters : p.units;
  int grid = work < num_sms ? (int)work : num_sms;
  if (msub == 2) {
    switch (bn) {
      case 256: return run_epi<256, 3, 2>(a.epi, p, grid, s);
      case 192: return run_epi<192, 3, 2>(a.epi, p, grid, s);
      case 128: return run_epi<128, 4, 2>(a.epi, p, grid, s);
      default: return run_epi<64, 5, 2>(a.epi, p, grid, s);
    }
  }
  switch (bn) {
    case 256: return run_epi<256, 4, 1>(a.epi, p, grid, s);
    case 192: return run_epi<192, 5, 1>(a.epi, p, grid, s);
    case 128: return run_epi<128, 6, 1>(a.epi, p, grid, s);
    default: return run_epi<64, 8, 1>(a.epi, p, grid, s);
  }
}

}  // namespace sl
