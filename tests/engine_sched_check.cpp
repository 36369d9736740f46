// Host check of the decode engine's stage geometry (engine_sched.h), built and run by
// tests/test_engine_schedule.py.  For every row length K (multiples of 128 up to 49152) and
// token count T (1..16) it checks that the planned stage fits its ring slot, that a chunk is
// whole 64-byte steps and one TMA box row, that the staged activations fit, and -- walking
// the stage order the producer and the consumers share for 0..40 tiles and one or two
// tensors -- that every (tile, tensor, chunk) is streamed exactly once, that every partial
// sum is flushed exactly once per activation chunk, and that no weight or activation read
// leaves its buffer.
#include <cstdio>
#include <vector>

#include "engine_sched.h"

using namespace bitnet;

int main() {
  int bad = 0, cases = 0;
  auto fail = [&](int K, int T, const char* what) {
    if (bad < 20) std::printf("FAIL K=%d T=%d: %s\n", K, T, what);
    ++bad;
  };
  for (int K = 128; K <= 49152; K += 128) {
    for (int T = 1; T <= 16; ++T) {
      ++cases;
      EngGeom g;
      if (!eng_plan(K, T, ENG_SLOT_MAX, ENG_ACT_MAX, g)) {
        fail(K, T, "no geometry");
        continue;
      }
      const int RB = K / 4;
      if (g.RB != RB) fail(K, T, "RB");
      if (g.slot_bytes > ENG_SLOT_MAX) fail(K, T, "slot too large");
      if (T * g.x_pitch > ENG_ACT_MAX) fail(K, T, "activations do not fit");
      if (g.full_rows) {
        if (g.CB != RB || g.n_chunks != 1 || g.n_ac != 1 || g.rs < 1 || g.rs > ENG_MAX_RS) fail(K, T, "full-row fields");
        if (ENG_SLOT_WARPS % g.rs) fail(K, T, "tiles per stage do not divide the consumer warps");
        if (16 * g.rs * RB + 64 > g.slot_bytes) fail(K, T, "full-row slot");
      } else {
        if (g.rs != 1 || g.CB % 64 || g.CB > ENG_BOX_MAX_BYTES || g.CB < 64) fail(K, T, "chunk size");
        if ((long)g.n_chunks * g.CB < RB || (long)(g.n_chunks - 1) * g.CB >= RB) fail(K, T, "chunk count");
        if (16 * g.CB + 64 > g.slot_bytes) fail(K, T, "chunked slot");
        if (g.ac_chunks < 1 || (long)g.n_ac * g.ac_chunks < g.n_chunks || (long)(g.n_ac - 1) * g.ac_chunks >= g.n_chunks)
          fail(K, T, "activation chunks");
      }
      // walk the stage order
      for (int NT = 1; NT <= 2; ++NT) {
        for (int nt = 0; nt <= 40; ++nt) {
          std::vector<int> seen(nt * NT * g.n_chunks, 0), flushes(nt * NT * g.n_ac, 0);
          int stages = 0;
          for (int ac = 0; ac < g.n_ac; ++ac) {
            const int wc0 = ac * g.ac_chunks, wc1 = (wc0 + g.ac_chunks < g.n_chunks) ? wc0 + g.ac_chunks : g.n_chunks;
            const int k0 = 4 * wc0 * g.CB, k1 = (4 * wc1 * g.CB < K) ? 4 * wc1 * g.CB : K;
            const int staged = (k1 - k0 + 255) / 256 * 256;  // activation bytes per token staged (zero-padded)
            if (staged + 64 > g.x_pitch) fail(K, T, "staged chunk exceeds the pitch");
            for (int tg0 = 0; tg0 < nt; tg0 += g.rs) {
              const int ntg = (g.rs < nt - tg0) ? g.rs : nt - tg0;
              for (int u = 0; u < NT; ++u) {
                for (int wc = wc0; wc < wc1; ++wc) {
                  ++stages;
                  const int cbytes = (g.CB < RB - wc * g.CB) ? g.CB : RB - wc * g.CB;
                  const int S = (cbytes + 63) / 64;
                  const int xoff = 256 * (wc - wc0) * (g.CB / 64);
                  if (xoff + 256 * S > staged) fail(K, T, "activation read past the staged chunk");
                  for (int tl = 0; tl < ntg; ++tl) {
                    // last byte read: row 15 of tile tl, step S-1, lane r = 3
                    const long last = (long)(tl * 16 + 15) * g.CB + 64L * (S - 1) + 48 + 16;
                    if (last > g.slot_bytes) fail(K, T, "weight read past the slot");
                    seen[((tg0 + tl) * NT + u) * g.n_chunks + wc]++;
                    if (wc == wc1 - 1) flushes[((tg0 + tl) * NT + u) * g.n_ac + ac]++;
                  }
                }
              }
            }
          }
          if (stages != eng_stage_count(g, nt, NT)) fail(K, T, "stage count");
          for (int v : seen)
            if (v != 1) fail(K, T, "a (tile, tensor, chunk) not streamed exactly once");
          for (int v : flushes)
            if (v != 1) fail(K, T, "a partial sum not flushed exactly once");
        }
      }
    }
  }
  if (bad) {
    std::printf("%d failures in %d cases\n", bad, cases);
    return 1;
  }
  std::printf("OK %d cases\n", cases);
  return 0;
}
