// Stage schedule of a decode-engine GEMV phase (see engine.cuh): which CTA-local tile and
// K-chunk every stage of the weight ring holds, in the order the producer warp issues them,
// and each consumer group's own stages in closed form.  No CUDA dependency, so the host
// test of the schedule compiles it as plain C++.
//
// A phase gives a CTA nt tiles (16 weight rows each) of nch K-chunks.  The consumer warps
// form ng groups; a group owns a tile for all of its chunks.  Tiles are dealt to the
// groups in rounds of ng (stage order: chunk-major within a round, group-minor); the
// `left` tiles of a last, partial round are each split into s contiguous chunk ranges
// (units), unit u going to group u, and their stages run step-major over the units.
#pragma once

#if defined(__CUDACC__)
#define ENG_HD __host__ __device__ __forceinline__
#else
#define ENG_HD inline
#endif

namespace bitnet {

ENG_HD int eng_groups(int nt) { return nt >= 5 ? 5 : (nt >= 3 ? 3 : 1); }

struct EngSched {
  int nch, ng, R, s, units, maxlen;
  int a, b, q;
  bool rem;
  ENG_HD EngSched(int nt, int nch_) : nch(nch_), a(0), b(0), q(0), rem(false) {
    ng = eng_groups(nt);
    R = nt / ng;
    const int left = nt - R * ng;
    s = left == 0 ? 1 : (nch >= 2 ? (ng / left < nch ? ng / left : nch) : 1);
    units = left * s;
    maxlen = (nch + s - 1) / s;
  }
  // Chunk range [cb, ce) of unit u of the last round.
  ENG_HD int unit_begin(int u) const { return nch * (u % s) / s; }
  ENG_HD int unit_end(int u) const { return nch * (u % s + 1) / s; }
  // Stages of the whole phase.
  ENG_HD int total() const {
    int n = R * ng * nch;
    for (int u = 0; u < units; ++u) n += unit_end(u) - unit_begin(u);
    return n;
  }
  // Next stage: owning group, tile (local index), chunk, and whether it is the last chunk
  // of the group's share of the tile.  False at the end.
  ENG_HD bool next(int& grp, int& tile, int& c, bool& last) {
    while (true) {
      if (!rem) {
        if (a >= R) {
          rem = true;
          a = 0;
          q = 0;
          continue;
        }
        grp = q;
        tile = a * ng + q;
        c = b;
        last = b == nch - 1;
        if (++q == ng) {
          q = 0;
          if (++b == nch) {
            b = 0;
            ++a;
          }
        }
        return true;
      }
      if (a >= maxlen || units == 0) return false;
      const int u = q, i = a;
      if (++q == units) {
        q = 0;
        ++a;
      }
      const int cb = unit_begin(u), ce = unit_end(u);
      if (cb + i < ce) {
        grp = u;
        tile = R * ng + u / s;
        c = cb + i;
        last = c == ce - 1;
        return true;
      }
    }
  }
};

// The stages of group `grp` in sequence order, with their index `pos` in the producer's
// sequence: in the full rounds every ng-th stage (tile r * ng + grp, chunks 0 .. nch-1); in
// the last round unit grp, whose stage i sits at i * units + grp while every unit still has
// a chunk i (i < lmin), else after the units of the last round that do.
struct EngOwnStages {
  int ng, nch, grp, R, s, units, own_full, own_rem, ucb, lmin, rank;
  int j, rr, cc;
  ENG_HD EngOwnStages(const EngSched& sc, int grp_)
      : ng(sc.ng), nch(sc.nch), grp(grp_), R(sc.R), s(sc.s), units(sc.units), own_full(sc.R * sc.nch),
        own_rem(0), ucb(0), lmin(0), rank(0), j(0), rr(0), cc(0) {
    if (grp < units) {
      ucb = sc.unit_begin(grp);
      own_rem = sc.unit_end(grp) - ucb;
      lmin = nch / s;
      for (int u = 0; u < grp; ++u)
        if (sc.unit_end(u) - sc.unit_begin(u) > lmin) ++rank;
    }
  }
  ENG_HD bool next(int& pos, int& tile, int& c, bool& last) {
    if (j >= own_full + own_rem) return false;
    if (j < own_full) {
      c = cc;
      tile = rr * ng + grp;
      pos = (rr * nch + cc) * ng + grp;
      last = cc == nch - 1;
      if (++cc == nch) {
        cc = 0;
        ++rr;
      }
    } else {
      const int i = j - own_full;
      c = ucb + i;
      tile = R * ng + grp / s;
      pos = R * ng * nch + (i < lmin ? i * units + grp : lmin * units + rank);
      last = i == own_rem - 1;
    }
    ++j;
    return true;
  }
};

}  // namespace bitnet
