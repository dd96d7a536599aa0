// Host-only check of the launch planners against the invariants the kernels
// rely on (tile coverage, one consumer per 16-byte vector, shared memory within
// the attribute the launches set, accumulator and ticket sizes the workspace
// holds).  Built and run by tests/test_plans_cpu.py; it calls no CUDA API, so
// it needs no GPU.
#include <cstdio>

#include "qs.h"
#include "qs_internal.cuh"

namespace qs {
GemvPlan plan_gemv_mma(int T, int d_out, int rows_bound, int mats);
GemvPlan plan_qgemv_mma(int T, int d_out, int rows_bound);
}  // namespace qs

static int g_fails = 0;
static long g_checked = 0;
#define CHECK(cond, ...)                                  \
  do {                                                    \
    ++g_checked;                                          \
    if (!(cond)) {                                        \
      if (++g_fails <= 20) {                              \
        std::printf("FAIL %s: ", #cond);                  \
        std::printf(__VA_ARGS__);                         \
        std::printf("\n");                                \
      }                                                   \
    }                                                     \
  } while (0)

constexpr size_t kSmemAttr = 200 * 1024;   // dynamic shared memory the GEMV launches allow
constexpr int kTicketSlots = 4096 - 8;      // gemv ticket slots of the workspace

static int round4(int t) { return (t + 3) & ~3; }

static void check_gemv(int T, int d_out, int rows, int mats, int eb) {
  const qs::GemvPlan p = qs::plan_gemv(T, d_out, rows, mats, eb);
  const char* f = "T=%d d_out=%d rows=%d mats=%d eb=%d";
  CHECK(p.groups * p.TT >= T && (p.groups - 1) * p.TT < T, f, T, d_out, rows, mats, eb);
  CHECK(p.S >= 1 && p.S <= 256 && p.copies >= 1 && p.copies <= 8, f, T, d_out, rows, mats, eb);
  CHECK(p.smem <= kSmemAttr, f, T, d_out, rows, mats, eb);
  CHECK(p.tickets == p.groups * p.n_ct && p.tickets <= kTicketSlots, f, T, d_out, rows, mats, eb);
  if (p.mma) {
    CHECK(eb == 2 && d_out % 16 == 0 && T >= 3, f, T, d_out, rows, mats, eb);
    CHECK(p.TT == 4 || p.TT == 8, f, T, d_out, rows, mats, eb);
    CHECK(p.vec_tile % 2 == 0 && p.vec_tile / 2 <= 8 * 12, f, T, d_out, rows, mats, eb);
    CHECK((long)p.n_ct * p.vec_tile * 16 >= (long)d_out * 2 &&
              (long)(p.n_ct - 1) * p.vec_tile * 16 < (long)d_out * 2,
          f, T, d_out, rows, mats, eb);
    CHECK(p.threads == 8 * 32 + 32 && p.rps == 16 && p.nst >= 2 && p.nst <= 4, f, T, d_out, rows,
          mats, eb);
    CHECK(p.smem == (size_t)p.nst * 16 * (p.vec_tile * 16 + 16) + (size_t)p.rcap * 4 * (1 + p.TT),
          f, T, d_out, rows, mats, eb);
    CHECK(p.parts_elems == (size_t)p.copies * mats * d_out * round4(T), f, T, d_out, rows, mats, eb);
    // one CTA per SM exactly for stages of 40 KB or more; the shared memory of
    // the occupancy the plan is sized for fits an SM (228 KB, 1 KB per CTA
    // reserved, a few KB of static shared memory), and the grid is resident
    const long stage = 16L * (p.vec_tile * 16 + 16);
    CHECK(p.cta_sm == (stage >= 40L * 1024 ? 1 : 2), f, T, d_out, rows, mats, eb);
    CHECK(p.cta_sm == 1 ? p.smem <= kSmemAttr : p.smem <= 108u * 1024, f, T, d_out, rows, mats, eb);
    CHECK((long)p.n_ct * mats * p.S <= 148L * p.cta_sm || p.S == 1, f, T, d_out, rows, mats, eb);
  } else {
    const int vec_row = (int)((long)d_out * eb / 16);
    CHECK(p.TT == 1 || p.TT == 2 || p.TT == 4 || p.TT == 8, f, T, d_out, rows, mats, eb);
    CHECK((long)p.n_ct * p.vec_tile >= vec_row && (long)(p.n_ct - 1) * p.vec_tile < vec_row, f, T,
          d_out, rows, mats, eb);
    CHECK(p.threads % 32 == 0 && p.threads - 32 >= p.vec_tile && p.threads <= 384 + 32, f, T,
          d_out, rows, mats, eb);
    CHECK(p.rps >= 1 && p.nst >= 3 && p.nst <= 32, f, T, d_out, rows, mats, eb);
    CHECK(p.smem == (size_t)p.nst * p.rps * p.vec_tile * 16 + (size_t)p.rcap * 4 * (1 + p.TT), f,
          T, d_out, rows, mats, eb);
    CHECK(p.parts_elems == (size_t)p.copies * mats * T * d_out, f, T, d_out, rows, mats, eb);
  }
}

static void check_qgemv(int T, int d_out, int rows) {
  const qs::GemvPlan p = qs::plan_qgemv(T, d_out, rows);
  const char* f = "T=%d d_out=%d rows=%d";
  const int row_words = d_out / 16;
  CHECK(p.groups * p.TT >= T && (p.groups - 1) * p.TT < T, f, T, d_out, rows);
  CHECK(p.vec_tile % 4 == 0 && p.vec_tile >= 4, f, T, d_out, rows);          // 16-byte copies
  CHECK((long)p.n_ct * p.vec_tile >= row_words && (long)(p.n_ct - 1) * p.vec_tile < row_words, f,
        T, d_out, rows);
  CHECK(p.S >= 1 && p.S <= 256 && p.copies == 1, f, T, d_out, rows);
  CHECK(p.smem <= kSmemAttr, f, T, d_out, rows);
  CHECK(p.tickets == p.groups * p.n_ct && p.tickets <= kTicketSlots, f, T, d_out, rows);
  if (p.mma) {
    CHECK(T >= 8 && (p.TT == 8 || p.TT == 16 || p.TT == 24 || p.TT == 32), f, T, d_out, rows);
    CHECK(p.vec_tile <= 8 * (12 / (p.TT / 8)), f, T, d_out, rows);
    CHECK(p.threads == 8 * 32 + 32 && p.rps == 32 && p.nst >= 2 && p.nst <= 16, f, T, d_out, rows);
    CHECK(p.rcap % 32 == 0, f, T, d_out, rows);                           // whole 32-row stages
    CHECK(p.smem == (size_t)p.nst * 32 * (p.vec_tile * 4 + 16) + (size_t)p.rcap * (4 + p.TT), f,
          T, d_out, rows);
    CHECK(p.parts_elems == (size_t)d_out * round4(T), f, T, d_out, rows);
  } else {
    const int lpt = p.TT == 1 ? 8 : (p.TT == 2 ? 16 : (p.TT == 4 ? 8 : 4));   // QTune
    CHECK(T < 8 && (p.TT == 1 || p.TT == 2 || p.TT == 4 || p.TT == 8), f, T, d_out, rows);
    CHECK(p.threads % 32 == 0 && (long)(p.threads - 32) * lpt >= (long)p.vec_tile * 8 &&
              p.threads <= 192 + 32,
          f, T, d_out, rows);
    CHECK(p.rps >= 1 && p.rps <= 16 && p.nst >= 3 && p.nst <= 32, f, T, d_out, rows);
    CHECK(p.smem == (size_t)p.nst * p.rps * p.vec_tile * 4 + (size_t)p.rcap * (4 + p.TT), f, T,
          d_out, rows);
    CHECK(p.parts_elems == (size_t)T * d_out, f, T, d_out, rows);
  }
}

// The workspace of (op, T, d_in, d_out, k) must hold the accumulators of every
// chunk's plan, for this k and any other.
static void check_layout(int op, int T, int d_in, int d_out, int k) {
  qs::WsLayout L;
  const char* f = "op=%d T=%d d_in=%d d_out=%d k=%d";
  CHECK(qs::ws_layout(op, T, d_in, d_out, k, &L), f, op, T, d_in, d_out, k);
  const int Tc = T < QS_PREFILL_MIN_T ? T : QS_PREFILL_MIN_T;
  for (int t = 1; t <= Tc; ++t) {
    for (int kk : {0, 1, k, d_in}) {
      if (kk > d_in) continue;
      const long tk = (long)t * kk;
      const int rb = (int)(tk < d_in ? tk : d_in);
      if (op == QS_OP_SPARSE_LINEAR) {
        for (int eb : {2, 4})
          if (d_out % (16 / eb) == 0)
            CHECK(qs::plan_gemv(t, d_out, rb, 1, eb).parts_elems <= L.parts1_elems, f, op, T, d_in,
                  d_out, kk);
      } else if (op == QS_OP_QUANT_SPARSE_LINEAR) {
        CHECK(qs::plan_qgemv(t, d_out, rb).parts_elems <= L.parts1_elems, f, op, T, d_in, d_out, kk);
      }
    }
  }
  if (op == QS_OP_SPARSE_FFN || op == QS_OP_SPARSE_FFN_GATE_FIRST) {
    // up and gate together (two matrices), or the gate alone (gate first)
    const int mats = op == QS_OP_SPARSE_FFN ? 2 : 1;
    for (int t = 1; t <= Tc; ++t)
      for (int eb : {2, 4}) {
        const long tk = (long)t * k;
        const int rb_h = (int)(tk < d_out ? tk : d_out);
        const qs::GemvPlan p1 = qs::plan_gemv(t, d_out, d_in, mats, eb);
        const qs::GemvPlan p2 = qs::plan_gemv(t, d_in, rb_h, 1, eb);
        CHECK(p1.parts_elems <= L.parts1_elems, f, op, T, d_in, d_out, k);
        CHECK(p2.parts_elems <= L.parts2_elems, f, op, T, d_in, d_out, k);
        // both projections' tickets fit the GEMV ticket slots
        CHECK(p1.tickets + p2.tickets <= kTicketSlots, f, op, T, d_in, d_out, k);
      }
  }
}

int main() {
  const int gemv_outs[] = {8, 16, 64, 96, 136, 160, 264, 512, 1024, 1552, 4096, 8200, 11008, 14336,
                           16384, 49152};
  const int rows_list[] = {1, 7, 31, 100, 1597, 2867, 5425, 16384, 49152};
  for (int T = 1; T <= 64; ++T)
    for (int d_out : gemv_outs)
      for (int rows : rows_list)
        for (int mats = 1; mats <= 2; ++mats)
          for (int eb : {2, 4})
            if (d_out % (16 / eb) == 0) check_gemv(T, d_out, rows, mats, eb);
  const int quant_outs[] = {64, 128, 320, 4096, 11008, 14336, 49152};
  for (int T = 1; T <= 64; ++T)
    for (int d_out : quant_outs)
      for (int rows : rows_list) check_qgemv(T, d_out, rows);
  const int shapes[][3] = {{512, 512, 256}, {4096, 11008, 2867}, {11008, 4096, 7705},
                           {4096, 14336, 1433}, {300, 64, 117}, {1000, 264, 500}, {77, 136, 38}};
  for (int T : {1, 2, 3, 8, 13, 64, 66, 200})
    for (const auto& s : shapes) {
      check_layout(QS_OP_SPARSE_LINEAR, T, s[0], s[1], s[2]);
      if (s[1] % 64 == 0) check_layout(QS_OP_QUANT_SPARSE_LINEAR, T, s[0], s[1], s[2]);
      if (s[2] <= s[1]) check_layout(QS_OP_SPARSE_FFN, T, s[0], s[1], s[2]);
      if (s[2] <= s[1]) check_layout(QS_OP_SPARSE_FFN_GATE_FIRST, T, s[0], s[1], s[2]);
    }
  // the batched-decode up/gate plans of the two FFN shapes: 2.75 KB tiles of
  // the Llama shape run one CTA per SM with four stages, the 2 KB tiles of the
  // dReLU shape two CTAs per SM (both measured faster that way)
  {
    const qs::GemvPlan ll = qs::plan_gemv(8, 11008, 4096, 2, 2);
    CHECK(ll.mma && ll.vec_tile == 172 && ll.cta_sm == 1 && ll.nst == 4 && ll.n_ct * 2 * ll.S == 144,
          "llama up/gate T=8 %d", 0);
    const qs::GemvPlan dr = qs::plan_gemv(4, 14336, 4096, 2, 2);
    CHECK(dr.mma && dr.vec_tile == 128 && dr.cta_sm == 2 && dr.nst == 2, "drelu up/gate T=4 %d", 0);
    const qs::GemvPlan q1 = qs::plan_qgemv(1, 11008, 1597);
    CHECK(!q1.mma && q1.vec_tile == 172 && q1.threads == 192 + 32, "int8 4096->11008 T=1 %d", 0);
  }
  std::printf("%ld checks, %d failed\n", g_checked, g_fails);
  return g_fails == 0 ? 0 : 1;
}
