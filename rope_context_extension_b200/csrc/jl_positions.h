// Integer position algebra of Dynamic Bifocal RoPE (host and device).
//
//  * group size      G = max(1, ceil(L / w_pretrained))     Jet-Long review, "Method";
//                                                           gist.science summary, "Methodologie §1"
//  * key remote pos  f(j) = floor(j / G)                    same passages
//  * query remote    p_q(i) = floor(i / G) + shift, with shift = w0 - floor(w0 / G)
//                    (Self-Extend-style reading, remote distances continue from w0)
//                    or shift = 0 (f on both sides); the pages leave this unstated.
//  * local pair      i - j < w0 (exact base RoPE); every other causal pair is remote.
//  * correction      dq(i) = p_q(i) - i, dk(j) = f(j) - j: R(dk) R(j) k = R(f(j)) k
//                    because RoPE rotations compose additively (gist.science summary,
//                    "§2 On-the-Fly Correctie Rotatie").
#pragma once

#include <stdint.h>

#if defined(__CUDACC__)
#define JL_HD __host__ __device__ __forceinline__
#else
#define JL_HD inline
#endif

namespace jl {

JL_HD int64_t group_size(int64_t L, int64_t w_pretrained) {
  const int64_t g = (L + w_pretrained - 1) / w_pretrained;
  return g < 1 ? 1 : g;
}

// mode: 0 = no query shift, 1 = Self-Extend-style shift.
JL_HD int64_t query_shift(int64_t w0, int64_t G, int mode) { return mode == 1 ? w0 - w0 / G : 0; }

JL_HD int64_t key_remote(int64_t j, int64_t G) { return j / G; }

JL_HD int64_t query_remote(int64_t i, int64_t G, int64_t shift) { return i / G + shift; }

// True when no remote pair can exist, so every causal pair is scored with base
// RoPE: G = 1 (exact base model) or the band covers the whole sequence.
JL_HD bool all_local(int64_t L, int64_t w0, int64_t G) { return G == 1 || w0 >= L; }

}  // namespace jl
