// Host-only check of the GEMM tiling planner (no GPU needed).
//
// The library's analytic planner chooses, for each projection GEMM of a step,
// the tile width, the rows per unit, the kernel variant and the K split.  The
// launch path accepts only some of those: a fused Q|K|V tile takes its weight
// rows from one of Wq, Wk, Wv (its width divides d_model) and, unsplit, rotates
// whole 128-column heads; a SwiGLU tile's gate and up halves divide d_ffn; a
// CTA pair needs tiles of at least 128 columns; the LM head writes logits rows
// and takes no K split; stream-K runs only where partial sums can be added.
// This program sweeps model shapes, row counts and SM counts and checks that
// every plan the planner returns satisfies them, and does the same for the
// layout and key split the tensor-core attention plans (a plan must exist for
// any launch with queries, and every split must hold key tiles).  It includes
// the runtime's source so that it sees the planners as the library compiles
// them.
#include "api.cu"

#include <cstdio>

static int g_fail = 0;
static long g_checked = 0;

#define CHECK(cond, ...)                                              \
  do {                                                                \
    if (!(cond)) {                                                    \
      if (++g_fail <= 25) {                                           \
        printf("FAIL (%s) ", #cond);                                  \
        printf(__VA_ARGS__);                                          \
        printf("\n");                                                 \
      }                                                               \
    }                                                                 \
  } while (0)

struct Shape {
  const char *name;
  int d, f, V;
};

static void check_plan(const Shape &sh, int kind, int M, int ns, const Plan &pl) {
  ++g_checked;
  const int d = sh.d, f = sh.f, V = sh.V;
  const int N = kind == G_QKV ? 3 * d : kind == G_GU ? 2 * f : kind == G_HD ? V : d;
  const int K = kind == G_DN ? f : d;
  const char *kn[] = {"QKV", "O", "GU", "DN", "HD"};
#define CTX "%s %s M=%d sms=%d -> bn=%d splits=%d msub=%d pair=%d", sh.name, kn[kind], M, ns, \
            pl.bn, pl.splits, pl.msub, pl.pair
  CHECK(pl.bn == 64 || pl.bn == 128 || pl.bn == 192 || pl.bn == 256, CTX);
  if (pl.bn <= 0) return;
  CHECK(N % pl.bn == 0, CTX);
  CHECK(pl.msub == 1 || pl.msub == 2, CTX);
  CHECK(!pl.pair || pl.msub == 2, CTX);
  CHECK(!pl.pair || pl.bn >= 128, CTX);
  CHECK(pl.splits == -1 || (pl.splits >= 1 && pl.splits <= K / 64), CTX);
  const int v = plan_variant(pl);
  Plan back{pl.bn, pl.splits, 1, 0.0};
  plan_set_variant(back, v);
  CHECK(back.msub == pl.msub && back.pair == pl.pair && back.swap == pl.swap, CTX);
  // swapped operands: projections of at most 256 rows, 128 weight rows per tile
  CHECK(!pl.swap || (pl.bn == 128 && M <= 256 && kind != G_HD && pl.splits >= 1), CTX);
  switch (kind) {
    case G_QKV:
      CHECK(d % pl.bn == 0, CTX);                           // one of Wq, Wk, Wv per tile
      CHECK(pl.splits != 1 || pl.bn % 128 == 0, CTX);       // whole heads in the RoPE epilogue
      break;
    case G_GU:
      CHECK(f % (pl.bn / 2) == 0, CTX);                     // gate and up halves
      break;
    case G_HD:
      CHECK(pl.splits == 1, CTX);                           // logits are stored, not summed
      break;
    default:
      break;
  }
#undef CTX
}

int main() {
  const Shape shapes[] = {
      {"llada8b", 4096, 12288, 126464}, {"mini256", 256, 512, 1024},
      {"mini768", 768, 768, 1024},      {"d512", 512, 1536, 32000},
      {"d2048", 2048, 5632, 32000},     {"d1024", 1024, 2816, 50304},
      {"d3072", 3072, 8192, 128256},    {"d1536", 1536, 4096, 65536},
  };
  const int sms[] = {148, 132, 20, 2};
  for (const Shape &sh : shapes) {
    sl_model m;
    memset(&m.cfg, 0, sizeof(m.cfg));
    m.cfg.n_layers = 1;
    m.cfg.d_model = sh.d;
    m.cfg.n_heads = sh.d / 128;
    m.cfg.head_dim = 128;
    m.cfg.d_ffn = sh.f;
    m.cfg.vocab = sh.V;
    m.cfg.dtype = SL_BF16;
    for (int ns : sms) {
      for (int M = 1; M <= 8192; M += (M < 320 ? 1 : (M < 2048 ? 29 : 211))) {
        for (int kind = 0; kind < G_KINDS; ++kind) check_plan(sh, kind, M, ns, plan_kind(&m, kind, M, ns));
      }
    }
  }
  // the tensor-core attention's layout and key split: a plan exists whenever
  // some sequence has queries; one or two query tiles per CTA as pinned; every
  // split holds at least one key tile and together they cover all of them
  {
    const int counts_set[][4] = {{1, 0, 0, 0}, {5, 0, 0, 0}, {128, 1, 0, 0}, {129, 128, 1, 0},
                                 {300, 0, 0, 0}, {2048, 2048, 2048, 2048}, {0, 40, 0, 0},
                                 {257, 384, 130, 7}};
    const int nctx_set[] = {64, 130, 384, 640, 2048, 2500, 4000};
    for (const auto &cs : counts_set)
      for (int batch = 1; batch <= 4; ++batch)
        for (int n_ctx : nctx_set)
          for (int ns : sms)
            for (int fq : {0, 128, 256})
              for (int fb : {0, 64, 128})
              for (int fs = 0; fs <= 17; ++fs) {
                AttnSeqs seqs{};
                seqs.batch = batch;
                int tiles = 0, off = 0;
                for (int b = 0; b < batch; ++b) {
                  const int c = cs[b] > n_ctx ? n_ctx : cs[b];
                  seqs.seq_start[b] = off;
                  seqs.seq_count[b] = c;
                  off += c;
                  tiles += (c + 127) / 128;
                }
                const AttnTcPlan pl = attn_tc_plan(seqs, 32, n_ctx, ns, 16, fq, fs, fb);
                ++g_checked;
#define ACTX "attn batch=%d n_ctx=%d sms=%d fq=%d fb=%d fs=%d -> qt=%d bn=%d splits=%d per=%d kt=%d units=%d",              batch, n_ctx, ns, fq, fb, fs, pl.qt, pl.bn, pl.splits, pl.kt_per_split, pl.ktiles, pl.units
                if (fq == 256 && fb == 128) {          // no such layout: no plan
                  CHECK(pl.units == 0, ACTX);
                  continue;
                }
                if (tiles == 0) {
                  CHECK(pl.units == 0, ACTX);
                  continue;
                }
                CHECK(pl.units > 0, ACTX);
                if (pl.units <= 0) continue;
                CHECK(pl.qt == 1 || pl.qt == 2, ACTX);
                CHECK(fq == 0 || fq == 128 * pl.qt, ACTX);
                CHECK(fb == 0 || fb == pl.bn, ACTX);
                CHECK(pl.bn == 64 || (pl.bn == 128 && pl.qt == 1), ACTX);
                CHECK(pl.ktiles == (n_ctx + pl.bn - 1) / pl.bn, ACTX);
                CHECK(pl.splits >= 1 && pl.splits <= 16, ACTX);
                CHECK(pl.kt_per_split * pl.splits >= pl.ktiles, ACTX);
                CHECK(pl.kt_per_split * (pl.splits - 1) < pl.ktiles, ACTX);   // no empty split
                int units = 0;
                for (int b = 0; b < batch; ++b)
                  units += ((seqs.seq_count[b] + 127) / 128 + pl.qt - 1) / pl.qt;
                CHECK(units == pl.units, ACTX);
#undef ACTX
              }
  }
  // row-count buckets of the autotuner: every M maps to the smallest bound >= M
  for (int M = 1; M <= 131072; M = M < 512 ? M + 1 : M + 97) {
    const int b = tune_bucket(M);
    CHECK(b >= 0 && kTuneBounds[b] >= M && (b == 0 || kTuneBounds[b - 1] < M), "bucket of M=%d", M);
  }
  CHECK(tune_bucket(131073) == -1, "beyond the last bucket");
  printf("planner_check: %ld plans checked, %d failures\n", g_checked, g_fail);
  return g_fail == 0 ? 0 : 1;
}
