// Host check of the decode engine's stage schedule (engine_sched.h), built and run by
// tests/test_engine_schedule.py.  For every CTA tile count and chunk count in a grid it
// checks that the producer's sequence holds every (tile, chunk) exactly once, that each
// group's share of a tile is a contiguous ascending chunk range closed by one `last`
// flag, and that every group's closed-form stage list (EngOwnStages) is exactly its
// stages of the producer's sequence, with their sequence positions.
#include <cstdio>
#include <vector>

#include "engine_sched.h"

struct Stage {
  int grp, tile, c;
  bool last;
};

int main() {
  int bad = 0, cases = 0;
  for (int nt = 0; nt <= 48; ++nt) {
    for (int nch = 1; nch <= 16; ++nch) {
      ++cases;
      bitnet::EngSched sc(nt, nch);
      std::vector<Stage> seq;
      int grp, tile, c;
      bool last;
      while (sc.next(grp, tile, c, last)) seq.push_back({grp, tile, c, last});
      auto fail = [&](const char* what) {
        if (bad < 20) std::printf("FAIL nt=%d nch=%d: %s\n", nt, nch, what);
        ++bad;
      };
      if ((int)seq.size() != nt * nch) fail("sequence length");
      if ((int)seq.size() != bitnet::EngSched(nt, nch).total()) fail("total()");
      std::vector<int> seen(nt * nch, 0);
      for (const Stage& st : seq) {
        if (st.tile < 0 || st.tile >= nt || st.c < 0 || st.c >= nch) {
          fail("stage out of range");
          continue;
        }
        if (st.grp < 0 || st.grp >= sc.ng) fail("group out of range");
        ++seen[st.tile * nch + st.c];
      }
      for (int v : seen)
        if (v != 1) fail("(tile, chunk) not exactly once");
      for (int g = 0; g < sc.ng; ++g) {
        // the group's stages in the producer's order, with positions
        std::vector<int> pos;
        for (int i = 0; i < (int)seq.size(); ++i)
          if (seq[i].grp == g) pos.push_back(i);
        // contiguous ascending chunks per tile, `last` at the end of each run
        for (size_t k = 0; k < pos.size(); ++k) {
          const Stage& st = seq[pos[k]];
          const bool run_ends = k + 1 == pos.size() || seq[pos[k + 1]].tile != st.tile;
          if (st.last != run_ends) fail("last flag");
          if (!run_ends && seq[pos[k + 1]].c != st.c + 1) fail("chunks of a run not consecutive");
        }
        bitnet::EngOwnStages own(sc, g);
        int p, t2, c2;
        bool l2;
        size_t k = 0;
        while (own.next(p, t2, c2, l2)) {
          if (k >= pos.size()) {
            fail("own stages: too many");
            break;
          }
          const Stage& st = seq[pos[k]];
          if (p != pos[k] || t2 != st.tile || c2 != st.c || l2 != st.last) fail("own stage differs");
          ++k;
        }
        if (k != pos.size()) fail("own stages: too few");
      }
    }
  }
  std::printf("%s: %d cases, %d failures\n", bad ? "FAIL" : "OK", cases, bad);
  return bad != 0;
}
