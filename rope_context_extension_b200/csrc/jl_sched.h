// Tile schedule of the fused prefill (host and device): which 128-key blocks
// a 128-row query block visits, in which order, and with which operands.
//
// The pages define the pair classes (Jet-Long review, "Method"; gist.science
// summary, "Methodologie §1"): a causal pair (i, j) is local when
// i - j < w0 and scored with base RoPE, and remote otherwise.  A 128 x 128
// tile holding both kinds is visited twice (a local and a remote pass with
// complementary masks).  The kernel runs these functions per CTA; the host
// exports the same functions' tile counts (jl_prefill_tile_classes) so the
// schedule can be checked without a GPU.
#pragma once

#include "jl_positions.h"

namespace jl {

// Pass kinds: kBifocal (local passes, then remote passes: the fused method),
// or one of the three calls of the inclusion-exclusion formulation (Jet-Long
// review, "Method"): kWindowBase (A: pairs with 0 <= i - j < w0, base rows),
// kCausalRemote (B: every causal pair, corrected rows), kWindowRemote (C: the
// window of A, corrected rows).
enum : int { kBifocal = 0, kWindowBase = 1, kCausalRemote = 2, kWindowRemote = 3 };

// Pass schedule of one query block whose first query position is `off` and
// last one `last` (off + 127, or the sequence's last row; keys in 128-key
// blocks nb).  Block nb spans i - j in [off - 128 nb - 127, last - 128 nb].
// Local passes run on the key blocks nb_max, nb_max - 1, ... that hold a pair
// with 0 <= i - j < w0; remote passes on nb_rem_max, ..., 0 (the blocks with a
// pair i - j >= w0).
struct Sched {
  int n_loc, n_rem, nb_max, nb_rem_max;
};

JL_HD int sched_max(int a, int b) {
#if defined(__CUDA_ARCH__)
  return max(a, b);
#else
  return a > b ? a : b;
#endif
}

JL_HD int floor_div128(int x) { return x >= 0 ? x / 128 : -((127 - x) / 128); }

template <int kind>
JL_HD Sched make_sched(int off, int last, int w0, bool all_local) {
  Sched s;
  s.nb_max = (off + 127) / 128;  // last block holding a causal key
  if (kind == kCausalRemote) {
    s.n_loc = 0;
    s.nb_rem_max = s.nb_max;
    s.n_rem = s.nb_max + 1;
    return s;
  }
  if (all_local) {
    s.n_loc = s.nb_max + 1;
    s.n_rem = 0;
    s.nb_rem_max = -1;
    return s;
  }
  if (w0 > 0) {
    const int nb_loc_min = sched_max(0, floor_div128(off - 127 - w0) + 1);  // 128 nb > off - 127 - w0
    s.n_loc = sched_max(0, s.nb_max - nb_loc_min + 1);
  } else {
    s.n_loc = 0;
  }
  s.nb_rem_max = floor_div128(last - w0);  // 128 nb <= last - w0
  s.n_rem = kind == kBifocal ? sched_max(0, s.nb_rem_max + 1) : 0;
  return s;
}

JL_HD int pass_block(const Sched& s, int p) { return p < s.n_loc ? s.nb_max - p : s.nb_rem_max - (p - s.n_loc); }

// Does pass p read the corrected (remote-position) Q / K rows?
template <int kind>
JL_HD bool pass_remote_ops(const Sched& s, int p) {
  return kind == kBifocal ? p >= s.n_loc : (kind != kWindowBase);
}

// Which pairs of the tile pass p keeps: 0 band (0 <= i-j < w0), 1 beyond the
// band (i-j >= w0), 2 every causal pair (i-j >= 0).
template <int kind>
JL_HD int pass_mask_kind(const Sched& s, int p) {
  if (kind == kCausalRemote) return 2;
  return p < s.n_loc ? 0 : 1;
}

}  // namespace jl
