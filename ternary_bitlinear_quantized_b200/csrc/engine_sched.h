// Stage geometry of a decode-engine product phase (see engine.cuh), shared by the host
// planner, the producer warp and the consumer warps.  No CUDA dependency, so the host test
// compiles it as plain C++.
//
// A stage (one ring slot) holds weights of ONE tensor: `rs` 16-row tiles x `CB` bytes of each
// row (rs divides the 15 consumer warps; each tile is worked on by 15 / rs of them).  Two modes:
//   full rows  (CB == RB, the whole row): the tiles' rows are one contiguous byte range of
//              the I2_S tensor, fetched with one 1-D bulk copy per run of tiles of the same
//              tensor (large contiguous copies stream at close to the HBM peak);
//   chunked    (rs == 1, CB < RB): one 2-D TMA box of 16 rows x CB bytes (8-byte elements,
//              zero fill past the row end) per stage, for rows too long for a slot or for
//              activations too large to stage whole.
// The activations of the phase are staged in shared memory in chunks of `ac_chunks` weight
// chunks (the whole row in full-row mode).  Stage order on a CTA that owns tiles [0, nt):
//   for ac < n_ac:  for tg0 = 0, rs, 2 rs, .. < nt:  for u < NT:  for wc in chunks of ac:
// (NT = 2 for the FFN's gate/up pair, whose stages alternate gate and up; else 1).  The
// consumers' partial sums of a tile persist over the chunks of one activation chunk and one
// tensor and are flushed after its last chunk.
#pragma once

#if defined(__CUDACC__)
#define ENG_HD __host__ __device__ __forceinline__
#else
#define ENG_HD inline
#endif

namespace bitnet {

constexpr int ENG_BOX_MAX_BYTES = 2048;     // a TMA box row: 256 elements of 8 bytes
constexpr int ENG_SLOT_MAX = 40 * 1024 + 64;  // bytes of one ring slot at most (a stage + slack)
constexpr int ENG_ACT_MAX = 72 * 1024;        // shared memory for the staged activations
constexpr int ENG_STAGE_TARGET = 40 * 1024;  // full-row stages group tiles up to this size
constexpr int ENG_MAX_RS = 5;                // tiles per full-row stage at most
constexpr int ENG_SLOT_WARPS = 15;           // consumer warps sharing a slot; rs divides it, so
                                             // each tile of a stage gets ENG_SLOT_WARPS / rs warps

struct EngGeom {
  int RB;           // bytes per weight row (K / 4)
  int rs;           // 16-row tiles per stage (full-row mode), 1 in chunked mode
  int CB;           // bytes of each row per stage (== RB in full-row mode, a multiple of 64 otherwise)
  int full_rows;    // 1: full-row mode
  int n_chunks;     // chunks per row
  int ac_chunks;    // chunks per activation chunk
  int n_ac;         // activation chunks
  int x_pitch;      // shared-memory bytes per token of a staged activation chunk
  int slot_bytes;   // shared-memory bytes a stage occupies (with 64 bytes of slack for a
                    // 32-byte half step read past the last row)
};

// Bytes per token of a staged activation chunk of n in-features: whole 256-in-feature
// steps (zero-padded), plus 64 so that consecutive tokens fall in different banks.
ENG_HD int eng_x_pitch_for(int n) { return ((n + 255) / 256) * 256 + 64; }

// Plan a phase of K in-features for T tokens: slot_max bytes per ring slot at most,
// act_max bytes of shared memory for the staged activations (all T tokens).  Returns false
// if no geometry fits.
ENG_HD bool eng_plan(int K, int T, int slot_max, int act_max, EngGeom& g) {
  g.RB = K / 4;
  const int RB = g.RB;
  if (16 * RB + 64 <= slot_max && T * eng_x_pitch_for(K) <= act_max) {
    g.full_rows = 1;
    g.CB = RB;
    // tiles per stage: the largest divisor of ENG_SLOT_WARPS (5, 3 or 1) that keeps the
    // stage within ENG_STAGE_TARGET and the slot
    int rs = 1;
    for (int c = ENG_MAX_RS; c > 1; --c)
      if (ENG_SLOT_WARPS % c == 0 && 16 * c * RB <= ENG_STAGE_TARGET && 16 * c * RB + 64 <= slot_max) {
        rs = c;
        break;
      }
    g.rs = rs;
    g.n_chunks = 1;
    g.ac_chunks = 1;
    g.n_ac = 1;
    g.x_pitch = eng_x_pitch_for(K);
    g.slot_bytes = 16 * rs * RB + 64;
    return true;
  }
  g.full_rows = 0;
  g.rs = 1;
  // Largest chunk (multiple of 64 bytes, at most one TMA box row) whose stage and whose
  // activations (one chunk per activation chunk at least) fit; then even chunks.
  int cmax = ENG_BOX_MAX_BYTES;
  while (cmax >= 64 && (16 * cmax + 64 > slot_max || T * eng_x_pitch_for(4 * cmax) > act_max)) cmax -= 64;
  if (cmax < 64) return false;
  const int n = (RB + cmax - 1) / cmax;
  int cb = (RB + n - 1) / n;
  cb = (cb + 63) / 64 * 64;
  if (cb > cmax) cb = cmax;
  g.CB = cb;
  g.n_chunks = (RB + cb - 1) / cb;
  int ac = 1;
  while (ac < g.n_chunks && T * eng_x_pitch_for(4 * cb * (ac + 1)) <= act_max) ++ac;
  g.ac_chunks = ac;
  g.n_ac = (g.n_chunks + ac - 1) / ac;
  g.x_pitch = eng_x_pitch_for(4 * cb * ac);
  g.slot_bytes = 16 * cb + 64;
  return true;
}

// Number of stages of a phase on a CTA with nt tiles.
ENG_HD int eng_stage_count(const EngGeom& g, int nt, int NT) {
  const int groups = (nt + g.rs - 1) / g.rs;
  return groups * NT * g.n_chunks;
}

}  // namespace bitnet
