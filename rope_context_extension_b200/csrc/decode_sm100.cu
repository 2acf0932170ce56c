// Fused Dynamic Bifocal RoPE decode for sm_100a: one new query token per
// sequence (at position L - 1) against a cache of base-rotated keys.
//
// The cache holds keys rotated at their absolute positions and is never
// rewritten (Jet-Long review, "Method"; gist.science summary, "§2 On-the-Fly
// Correctie Rotatie").  Keys with (L - 1) - j < w0 are scored with the query as
// given; every other key is scored with the correction rotations applied in
// registers: the query is rotated by dq = p_q(L-1) - (L-1) and key j by
// dk(j) = f(j) - j.
//
// Split-KV layout: grid (splits, Hkv, B); each CTA streams a contiguous run of
// tiles (16 keys per consumer warp) of one KV head through a TMA ring (128-byte
// swizzled so ldmatrix is conflict-free) and scores all r = Hq / Hkv query
// heads of that KV head at once with mma.sync m16n8k16 (heads on the M axis,
// 16 keys per warp).  The base query's A fragments sit in shared memory (the
// same for every warp), which keeps the consumers at 164 registers.
//
// Correction rotation of keys, per warp tile of 16 keys starting at j0:
//   dk(j) = dk(j0) - e(j) with e(j) in [0, 15]; the query side carries
//   R(dq - dk(j0)) q (kept in fp32, advanced by one fixed small rotation per
//   tile), and the key side only needs R(-e(j)) from a 16-row table, applied
//   to the key fragments in registers before the product.  Every angle with a
//   large argument is formed and reduced in fp64 once per CTA.  Corrected
//   operands enter the products as bf16 hi + lo pairs, so the remote scores
//   carry about 16 significant bits, like the unrotated local ones.
//
// Partials (running max, sum, unnormalised O) go to caller scratch; the last
// CTA of each (batch, KV head) - found with an atomic ticket, no spinning -
// merges them with a warp-shuffle log-sum-exp combine.
#include "jl_kernels.cuh"

namespace jl {

namespace {

// Consumer warps per CTA (16 keys each per stage), ring depth and register cap.
// The register file is split evenly over the four SM sub-partitions (16384
// registers each) and a CTA's warps are dealt out over them, so at 168
// registers a sub-partition holds three warps: one CTA of 11 consumer warps +
// the TMA warp per SM (two 176-key stages, 2 x 88 KB).  The consumers are
// bound by the latency of the in-register correction, so warps per SM is what
// counts: measured at B 8 / 128K, 11 warps in one CTA stream the cache about 8%
// faster than two CTAs of 4 (and 10% faster at B 1).
#ifndef JL_DEC_WARPS
#define JL_DEC_WARPS 11
#endif
#ifndef JL_DEC_STAGES
#define JL_DEC_STAGES 2
#endif
#ifndef JL_DEC_MAXNREG
#define JL_DEC_MAXNREG 168
#endif
constexpr int kDecWarps = JL_DEC_WARPS;
constexpr int kDecKeys = 16 * kDecWarps;  // keys per stage
constexpr int kDecStages = JL_DEC_STAGES;
constexpr int kDecThreads = 32 * (kDecWarps + 1);  // consumer warps + 1 TMA warp
static_assert(kDecWarps >= 1 && kDecWarps <= 11, "consumer warps");
constexpr int kMaxR = 8;       // query heads per KV head handled (M rows used)

template <int D>
struct DecCfg {
  static constexpr int kChunks = D / 64;
  static constexpr int kTileBytes = kDecKeys * D * 2;  // one of K or V
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kERow = (D / 2 + 8) * 8;        // bytes per E row (padded)
  static constexpr int kEOff = kDecStages * kStageBytes;
  static constexpr int kFOff = kEOff + 16 * kERow;
  static constexpr int kQ0Off = kFOff + 2 * (D / 2) * 8;  // [warps][D/2] initial query factors
  static constexpr int kQBOff = kQ0Off + kDecWarps * (D / 2) * 8;  // [D/16][2][32 lanes] base query fragments
  static constexpr int kBarOff = kQBOff + (D / 16) * 2 * 32 * 4;
  static constexpr int kSmem = kBarOff + 128 + 1024;
  static constexpr int kNT = D / 8;                    // t values per lane
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// bf16x2 word -> packed fp32x2 (exact)
__device__ __forceinline__ uint64_t bf16x2_to_f2(uint32_t w) { return f2_pack(bf16lo_to_f32(w), bf16hi_to_f32(w)); }

// Packed pair v = (a, b) -> bf16x2 hi = round(a, b) and lo = round((a, b) - hi).
__device__ __forceinline__ void split_f2_bf16(uint64_t v, uint32_t& hi, uint32_t& lo) {
  float a, b;
  f2_unpack(v, a, b);
  hi = pack_bf16x2(a, b);
  const uint64_t r = f2_sub(v, bf16x2_to_f2(hi));
  float ra, rb;
  f2_unpack(r, ra, rb);
  lo = pack_bf16x2(ra, rb);
}

// Rotate the bf16 pairs (x, y) of two adjacent RoPE pairs by the factors
// f = (c0, c1, s0, s1) and return the results as hi / lo bf16 parts:
// x' = x c - y s, y' = y c + x s.
__device__ __forceinline__ void rot_split_bf16(uint32_t xw, uint32_t yw, const float4& f, uint32_t& xh, uint32_t& xl,
                                               uint32_t& yh, uint32_t& yl) {
  const uint64_t x = bf16x2_to_f2(xw), y = bf16x2_to_f2(yw);
  const uint64_t c = f2_pack(f.x, f.y), sn = f2_pack(f.z, f.w);
  const uint64_t xr = f2_sub(f2_mul(x, c), f2_mul(y, sn));
  const uint64_t yr = f2_fma(x, sn, f2_mul(y, c));
  split_f2_bf16(xr, xh, xl);
  split_f2_bf16(yr, yh, yl);
}

__device__ __forceinline__ void named_sync_consumers() {
  asm volatile("bar.sync 1, %0;" ::"n"(32 * kDecWarps) : "memory");
}

template <int D>
__global__ void __maxnreg__(JL_DEC_MAXNREG)
    bifocal_decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                          const __grid_constant__ DecodeArgs args) {
  using C = DecCfg<D>;
  constexpr int H2 = D / 2;
  constexpr int KS = D / 16;   // k-steps of the score product
  constexpr int KS2 = D / 32;  // k-steps holding the first half of each pair
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kBarOff + 64);
  volatile int* ticket_slot = reinterpret_cast<volatile int*>(smem + C::kBarOff + 68);
  auto full_bar = [&](int s) -> uint32_t { return smem_addr(&bars[s]); };
  auto empty_bar = [&](int s) -> uint32_t { return smem_addr(&bars[kDecStages + s]); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int r = args.r;
  // This sequence's length and the position algebra that follows from it
  // (group size, query shift, local band), per CTA so that every sequence of
  // a varlen batch gets its own G.
  int L = args.L;
  if (args.seq_lens != nullptr) {
    L = args.seq_lens[b];
    if (L < 1 || (int64_t)L > args.cache_len) {
      if (threadIdx.x == 0 && args.dev_error) atomicExch(args.dev_error, kDevBadLength);
      L = L < 1 ? 1 : (int)args.cache_len;
    }
  }
  // Key row j of this call sits at position j + key_off; the query at Lpos - 1
  // (Lpos = the sequence's total length; a sequence-split decode gives each
  // GPU one key range of the cache and the global length).
  const int key_off = args.key_off;
  const int Lpos = args.L_total > 0 ? args.L_total : L;
  const int G = (int)group_size(Lpos, args.w_pretrained);
  const bool all_local = jl::all_local(Lpos, args.w0, G);
  const int64_t dq = query_remote(Lpos - 1, G, query_shift(args.w0, G, args.qshift)) - (Lpos - 1);
  const uint32_t g_magic = G < 16 ? (uint32_t)((((uint64_t)1 << 32) + (uint64_t)G - 1) / (uint64_t)G) : 0u;
  const int ntiles_b = (L + kDecKeys - 1) / kDecKeys;
  const int t_begin = (int)(((int64_t)split * ntiles_b) / args.splits);
  const int t_end = (int)(((int64_t)(split + 1) * ntiles_b) / args.splits);
  const int ntile = t_end - t_begin;  // may be 0 for short sequences of a varlen batch
  const int local_from = all_local ? 0 : Lpos - args.w0 - key_off;  // rows j >= local_from are local

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), kDecWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();
  if (warp == kDecWarps) {
    // ------------------------------------------------------------ TMA producer
    // (starts streaming at once; the consumers build their tables meanwhile)
    if (lane == 0) {
      tma_prefetch_map(&tm_k);
      tma_prefetch_map(&tm_v);
      int last = -1;
      bool ok = true;
      for (int i = 0; i < ntile; ++i) {
        const int s = i % kDecStages;
        const uint32_t ph = (uint32_t)(i / kDecStages) & 1u;
        if (!(ok = mbar_wait(empty_bar(s), ph ^ 1u, abort_flag, args.dev_error))) break;
        const int key0 = (t_begin + i) * kDecKeys;
        mbar_arrive_expect_tx(full_bar(s), (uint32_t)C::kStageBytes);
        const uint32_t st = sbase + s * C::kStageBytes;
        for (int c = 0; c < C::kChunks; ++c) {
          tma_load_4d(st + c * (kDecKeys * 128), &tm_k, full_bar(s), c * 64, g, key0, b);
          tma_load_4d(st + C::kTileBytes + c * (kDecKeys * 128), &tm_v, full_bar(s), c * 64, g, key0, b);
        }
        last = i;
      }
      if (!ok) {
        for (int i = max(0, last - kDecStages + 1); i <= last; ++i) {
          const uint64_t t0 = global_timer_ns();
          while (!mbar_try_wait(full_bar(i % kDecStages), (uint32_t)(i / kDecStages) & 1u))
            if (global_timer_ns() - t0 > 100000000ull) break;
        }
      }
    }
    return;
  }
  constexpr int kCons = 32 * kDecWarps;  // consumer threads
  // Correction tables (the consumers fill and use them):
  //   E[e][t]  rotation by -e (e in [0, 16)) applied to keys within a warp tile
  //   F[k][t]  advance of the query factor from one warp tile to the next
  //            (kDecKeys keys later), k = (number of new groups) - floor(kDecKeys / G)
  //   Q0[w][t] rotation by dq - dk(j0) for warp w's first tile
  float2* E = reinterpret_cast<float2*>(smem + C::kEOff);
  float2* F = reinterpret_cast<float2*>(smem + C::kFOff);
  float2* Q0 = reinterpret_cast<float2*>(smem + C::kQ0Off);
  if (!all_local) {
    const int q64 = kDecKeys / G;
    for (int idx = threadIdx.x; idx < (18 + kDecWarps) * H2; idx += kCons) {
      const int row = idx / H2, t = idx % H2;
      int64_t turns;  // the angle in units of theta_t (an integer)
      if (row < 16) {
        turns = -row;
      } else if (row < 18) {
        turns = -(q64 + (row - 16) - kDecKeys);  // -(dk(j0 + kDecKeys) - dk(j0))
      } else {
        const int64_t j0 = (int64_t)t_begin * kDecKeys + 16 * (row - 18) + key_off;  // position
        turns = dq - (j0 / G - j0);
      }
      double sn, cs;
      sincos_int_angle(turns, args.u_hi[t], args.u_lo[t], &sn, &cs);
      // E and F rows hold (c_t, c_t+1, s_t, s_t+1) for even t; Q0 rows (c_t, s_t)
      float* dst = row < 16 ? reinterpret_cast<float*>(E) + row * (C::kERow / 4)
                            : reinterpret_cast<float*>(F) + (row - 16) * D;
      if (row < 18) {
        dst[(t >> 1) * 4 + (t & 1)] = (float)cs;
        dst[(t >> 1) * 4 + 2 + (t & 1)] = (float)sn;
      } else {
        Q0[(row - 18) * H2 + t] = make_float2((float)cs, (float)sn);
      }
    }
  }
  // The base query as A fragments of mma m16n8k16 (heads on M rows 0-7),
  // identical for every consumer warp: [k-step][a1 / a3][lane] holds the bf16
  // pair at dims 16 ks + 2 (lane % 4) (+ 8) of head lane / 4.
  uint32_t* QB = reinterpret_cast<uint32_t*>(smem + C::kQBOff);
  for (int idx = threadIdx.x; idx < KS * 2 * 32; idx += kCons) {
    const int ks = idx / 64, hf = (idx / 32) & 1, l = idx & 31;
    const int hr = l >> 2;
    uint32_t w = 0u;
    if (hr < r) {
      const __nv_bfloat16* qp = args.q + ((size_t)b * args.Hq + g * r + hr) * D + 16 * ks + 8 * hf + 2 * (l & 3);
      w = *reinterpret_cast<const uint32_t*>(qp);
    }
    QB[idx] = w;
  }
  named_sync_consumers();

  // -------------------------------------------------------------- consumers
  const int c4 = lane & 3;        // column group of the mma fragments
  const int hrow = lane >> 2;     // query head (M row) of this lane
  const bool head_ok = hrow < r;

  // The fp32 query copy in the lane's t-set: t = 16 ks + 2 c4 + {0, 1, 8, 9},
  // ks < D/32 (the base fragments stay in shared memory for local tiles).
  float qre[C::kNT], qim[C::kNT];
#pragma unroll
  for (int ks = 0; ks < KS2; ++ks) {
    const uint32_t x0 = QB[(ks * 2 + 0) * 32 + lane], x1 = QB[(ks * 2 + 1) * 32 + lane];
    const uint32_t y0 = QB[((ks + KS2) * 2 + 0) * 32 + lane], y1 = QB[((ks + KS2) * 2 + 1) * 32 + lane];
    qre[4 * ks + 0] = bf16lo_to_f32(x0);
    qre[4 * ks + 1] = bf16hi_to_f32(x0);
    qre[4 * ks + 2] = bf16lo_to_f32(x1);
    qre[4 * ks + 3] = bf16hi_to_f32(x1);
    qim[4 * ks + 0] = bf16lo_to_f32(y0);
    qim[4 * ks + 1] = bf16hi_to_f32(y0);
    qim[4 * ks + 2] = bf16lo_to_f32(y1);
    qim[4 * ks + 3] = bf16hi_to_f32(y1);
  }
  // q^c = R(dq - dk(j0)) q for this warp's first 16-key tile.
  if (!all_local) {
#pragma unroll
    for (int e = 0; e < C::kNT; ++e) {
      const int t = 16 * (e >> 2) + 2 * c4 + (e & 1) + ((e & 2) ? 8 : 0);
      const float2 f = Q0[warp * H2 + t];
      const float x = qre[e], y = qim[e];
      qre[e] = x * f.x - y * f.y;
      qim[e] = y * f.x + x * f.y;
    }
  }

  // O is accumulated transposed, O^T[dim][head] += V^T[dim][key] P^T[key][head]:
  // V^T comes from ldmatrix.trans, and P^T's B fragment is exactly the score
  // C fragment of this lane, so no shuffle is needed.  Lane holds dims
  // 16 mt + lane/4 (+8) for heads 2 c4 and 2 c4 + 1.
  float oacc[D / 16][4];
#pragma unroll
  for (int n = 0; n < D / 16; ++n) oacc[n][0] = oacc[n][1] = oacc[n][2] = oacc[n][3] = 0.f;
  float m_used = -INFINITY, l_part = 0.f;
  const float sl2 = args.scale_log2;
  bool ok = true;

  // Group arithmetic of this warp's tile start j0, advanced by kDecKeys keys per
  // tile without divisions: j0 = qd G + rm.
  int j0 = t_begin * kDecKeys + 16 * warp;  // row in this call's cache
  int qd = (j0 + key_off) / G, rm = (j0 + key_off) - qd * G;  // of the position j0 + key_off
  const int q64 = kDecKeys / G, r64 = kDecKeys - q64 * G;
  // floor(x / G) for 0 <= x < G + 16 (one multiply-high; exact there)
  auto div_small = [&](int x) -> int {
    return G >= 16 ? (x >= G ? 1 : 0) : (int)__umulhi((unsigned)x, g_magic);
  };

  for (int i = 0; i < ntile; ++i) {
    const int s = i % kDecStages;
    const uint32_t ph = (uint32_t)(i / kDecStages) & 1u;
    if (i > 0) {
      j0 += kDecKeys;
      qd += q64;
      rm += r64;
      int fidx = 0;
      if (rm >= G) {
        rm -= G;
        ++qd;
        fidx = 1;
      }
      // advance q^c from the previous tile's j0 to this one
      if (!all_local) {
        const float4* Fr = reinterpret_cast<const float4*>(F) + fidx * (H2 / 2);
#pragma unroll
        for (int e = 0; e < C::kNT; e += 2) {
          const int t = 16 * (e >> 2) + 2 * c4 + ((e & 2) ? 8 : 0);  // even
          const float4 f = Fr[t >> 1];
          const uint64_t c = f2_pack(f.x, f.y), sn = f2_pack(f.z, f.w);
          const uint64_t x = f2_pack(qre[e], qre[e + 1]), y = f2_pack(qim[e], qim[e + 1]);
          const uint64_t xr = f2_sub(f2_mul(x, c), f2_mul(y, sn));
          const uint64_t yr = f2_fma(x, sn, f2_mul(y, c));
          f2_unpack(xr, qre[e], qre[e + 1]);
          f2_unpack(yr, qim[e], qim[e + 1]);
        }
      }
    }

    ok = mbar_wait(full_bar(s), ph, abort_flag, args.dev_error);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) break;

    if (j0 < L) {
      const uint32_t kst = sbase + s * C::kStageBytes;
      const uint32_t vst = kst + C::kTileBytes;
      const bool t_local = all_local || j0 >= local_from;
      const bool t_remote = !all_local && (j0 + 15 < local_from);

      float sloc[2][4], sah[2][4], sal[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int k = 0; k < 4; ++k) sloc[nt][k] = sah[nt][k] = sal[nt][k] = 0.f;

      // correction rows of this lane's two keys (one per 8-key n-tile):
      // dk(j0 + u) = dk(j0) - e(u), e(u) = u - (floor((j0 + u)/G) - floor(j0/G))
      const float4* Er[2];
      if (!t_local) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const int u = 8 * nt + (lane >> 2);
          const int e = u - div_small(rm + u);
          Er[nt] = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(E) + e * (C::kERow / 4));
        }
      }

      // Key fragments are loaded a pair of k-steps at a time: k-step kp holds
      // the first coordinate of RoPE pairs t in [16kp, 16kp + 16) and k-step
      // kp + D/32 the second, so each pair is complete in registers.
#pragma unroll
      for (int kp = 0; kp < KS2; ++kp) {
        uint32_t klo[4], khi[4];
        {
          const int mi = lane >> 3;
          const int kr = 16 * warp + (mi >> 1) * 8 + (lane & 7);
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const int ks = kp + hf * KS2;
            const int u = 2 * (ks & 3) + (mi & 1);
            const uint32_t addr = kst + (ks >> 2) * (kDecKeys * 128) + kr * 128 + ((u ^ (kr & 7)) << 4);
            if (hf == 0)
              ldsm_x4(addr, klo[0], klo[1], klo[2], klo[3]);
            else
              ldsm_x4(addr, khi[0], khi[1], khi[2], khi[3]);
          }
        }
        if (!t_remote) {  // local or straddling: base query, keys as stored
          const uint32_t alo[4] = {QB[(kp * 2) * 32 + lane], 0u, QB[(kp * 2 + 1) * 32 + lane], 0u};
          const uint32_t ahi[4] = {QB[((kp + KS2) * 2) * 32 + lane], 0u, QB[((kp + KS2) * 2 + 1) * 32 + lane], 0u};
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            mma_bf16(sloc[nt], alo, klo[2 * nt], klo[2 * nt + 1]);
            mma_bf16(sloc[nt], ahi, khi[2 * nt], khi[2 * nt + 1]);
          }
        }
        if (!t_local) {  // remote or straddling: corrected query and keys
          // The corrected operands are carried as bf16 hi + lo pairs (about 16
          // significant bits): the query's hi part sits in M rows 0-7 and its
          // lo part in rows 8-15 (unused by the r <= 8 heads), so two products
          // per k-step (keys hi, keys lo; separate accumulators to shorten the
          // dependency chains) give (q_hi + q_lo) . (k_hi + k_lo) once rows
          // h and h + 8 of both accumulators are added.
          uint32_t kah[4], kal[4], kbh[4], kbl[4];
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            const float4 f01 = Er[nt][(16 * kp + 2 * c4) >> 1];
            const float4 f23 = Er[nt][(16 * kp + 8 + 2 * c4) >> 1];
            rot_split_bf16(klo[2 * nt], khi[2 * nt], f01, kah[2 * nt], kal[2 * nt], kbh[2 * nt], kbl[2 * nt]);
            rot_split_bf16(klo[2 * nt + 1], khi[2 * nt + 1], f23, kah[2 * nt + 1], kal[2 * nt + 1], kbh[2 * nt + 1],
                           kbl[2 * nt + 1]);
          }
          uint32_t alo[4], ahi[4];
          split_f2_bf16(f2_pack(qre[4 * kp + 0], qre[4 * kp + 1]), alo[0], alo[1]);
          split_f2_bf16(f2_pack(qre[4 * kp + 2], qre[4 * kp + 3]), alo[2], alo[3]);
          split_f2_bf16(f2_pack(qim[4 * kp + 0], qim[4 * kp + 1]), ahi[0], ahi[1]);
          split_f2_bf16(f2_pack(qim[4 * kp + 2], qim[4 * kp + 3]), ahi[2], ahi[3]);
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            mma_bf16(sah[nt], alo, kah[2 * nt], kah[2 * nt + 1]);
            mma_bf16(sal[nt], alo, kal[2 * nt], kal[2 * nt + 1]);
            mma_bf16(sah[nt], ahi, kbh[2 * nt], kbh[2 * nt + 1]);
            mma_bf16(sal[nt], ahi, kbl[2 * nt], kbl[2 * nt + 1]);
          }
        }
      }

      // scores in log2 units with band selection and the tail mask
      float x[2][2];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int j = j0 + 8 * nt + 2 * c4 + k;
          const bool loc = all_local || j >= local_from;
          const float rem = (sah[nt][k] + sah[nt][k + 2]) + (sal[nt][k] + sal[nt][k + 2]);
          float v = (loc ? sloc[nt][k] : rem) * sl2;
          if (j >= L) v = -INFINITY;
          x[nt][k] = v;
        }
      float mt = fmaxf(fmaxf(x[0][0], x[0][1]), fmaxf(x[1][0], x[1][1]));
      mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
      mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
      const float m_new = fmaxf(m_used, mt);
      float alpha = 1.f;
      bool resc = false;
      if (m_new > m_used + 8.f) {
        alpha = (m_used == -INFINITY) ? 0.f : ex2_approx(m_used - m_new);
        resc = m_used != -INFINITY;
        l_part *= alpha;
        m_used = m_new;
      }
      if (__any_sync(0xffffffffu, resc)) {
        // this lane's O^T columns are heads 2 c4 and 2 c4 + 1
        const float a0 = __shfl_sync(0xffffffffu, alpha, 8 * c4);
        const float a1 = __shfl_sync(0xffffffffu, alpha, 8 * c4 + 4);
#pragma unroll
        for (int n = 0; n < D / 16; ++n) {
          oacc[n][0] *= a0;
          oacc[n][1] *= a1;
          oacc[n][2] *= a0;
          oacc[n][3] *= a1;
        }
      }
      const float msub = (m_used == -INFINITY) ? 0.f : m_used;
      float p[2][2];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          p[nt][k] = ex2_approx(x[nt][k] - msub);
          l_part += p[nt][k];
        }
      const uint32_t pb0 = pack_bf16x2(p[0][0], p[0][1]);  // keys 2 c4 + {0, 1}, head lane/4
      const uint32_t pb1 = pack_bf16x2(p[1][0], p[1][1]);  // keys 8 + 2 c4 + {0, 1}
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) {
        const int mi = lane >> 3;
        const int kr = 16 * warp + (mi >> 1) * 8 + (lane & 7);
        const int u = 2 * (mt & 3) + (mi & 1);
        const uint32_t addr = vst + (mt >> 2) * (kDecKeys * 128) + kr * 128 + ((u ^ (kr & 7)) << 4);
        uint32_t va[4];
        ldsm_x4_t(addr, va[0], va[1], va[2], va[3]);
        mma_bf16(oacc[mt], va, pb0, pb1);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty_bar(s));
  }

  // ---------------------------------------------------------- CTA merge
  l_part += __shfl_xor_sync(0xffffffffu, l_part, 1);
  l_part += __shfl_xor_sync(0xffffffffu, l_part, 2);
  named_sync_consumers();  // every warp is done with the stage buffers
  float* mw = reinterpret_cast<float*>(smem);  // [warps][kMaxR]
  float* lw = mw + kDecWarps * kMaxR;          // [warps][kMaxR]
  float* ow = lw + kDecWarps * kMaxR;          // [warps][kMaxR][D]
  if (head_ok && c4 == 0) {
    mw[warp * kMaxR + hrow] = m_used;
    lw[warp * kMaxR + hrow] = l_part;
  }
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int h = 2 * c4 + (k & 1);
      const int d = 16 * mt + (lane >> 2) + ((k & 2) ? 8 : 0);
      if (h < r) ow[(warp * kMaxR + h) * D + d] = oacc[mt][k];
    }
  }
  named_sync_consumers();
  const size_t pbase = (((size_t)b * args.Hkv + g) * args.splits + split) * r;
  for (int idx = threadIdx.x; idx < r * D; idx += 32 * kDecWarps) {
    const int h = idx / D, d = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, mw[w * kMaxR + h]);
    float o = 0.f, l = 0.f;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) {
      const float mwv = mw[w * kMaxR + h];
      const float wt = (mwv == -INFINITY) ? 0.f : ex2_approx(mwv - M);
      o += wt * ow[(w * kMaxR + h) * D + d];
      l += wt * lw[w * kMaxR + h];
    }
    args.part_o[(pbase + h) * D + d] = o;
    if (d == 0) args.part_ml[pbase + h] = make_float2(M, l);
  }

  // ---------------------------------------------------------- last CTA merges
  __threadfence();
  named_sync_consumers();
  if (threadIdx.x == 0) {
    const int prev = atomicAdd(&args.counters[b * args.Hkv + g], 1);
    *ticket_slot = (prev == args.splits - 1) ? 1 : 0;
  }
  named_sync_consumers();
  if (*ticket_slot == 0) return;
  __threadfence();
  const size_t sbase_p = ((size_t)b * args.Hkv + g) * args.splits;
  const int S = args.splits;
  // Per head: the global max and sum over the splits (lanes over splits), then
  // each split's weight 2^(m_s - M) / l in shared memory (the stage area is
  // free); then every consumer thread reduces its (head, dim) outputs over the
  // splits with independent loads in flight.
  float* wts = reinterpret_cast<float*>(smem);  // [r][S]
  for (int h = warp; h < r; h += kDecWarps) {
    float M = -INFINITY;
    for (int sp = lane; sp < S; sp += 32) M = fmaxf(M, __ldcg(&args.part_ml[(sbase_p + sp) * r + h]).x);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float l = 0.f;
    for (int sp = lane; sp < S; sp += 32) {
      const float2 ml = __ldcg(&args.part_ml[(sbase_p + sp) * r + h]);
      l += (ml.x == -INFINITY) ? 0.f : ml.y * ex2_approx(ml.x - M);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    const float inv = l > 0.f ? 1.f / l : 0.f;
    for (int sp = lane; sp < S; sp += 32) {
      const float mx = __ldcg(&args.part_ml[(sbase_p + sp) * r + h]).x;
      wts[h * S + sp] = (mx == -INFINITY) ? 0.f : ex2_approx(mx - M) * inv;
    }
    if (lane == 0 && args.lse != nullptr)
      args.lse[(size_t)b * args.Hq + g * r + h] = (M + __log2f(l)) * 0.69314718055994531f;
  }
  named_sync_consumers();
  for (int idx = threadIdx.x; idx < r * D; idx += kCons) {
    const int h = idx / D, d = idx % D;
    const float* po = args.part_o + (sbase_p * r + h) * D + d;  // split sp at + sp * r * D
    float acc = 0.f;
#pragma unroll 8
    for (int sp = 0; sp < S; ++sp) acc += wts[h * S + sp] * __ldcg(po + (size_t)sp * r * D);
    args.o[((size_t)b * args.Hq + g * r + h) * D + d] = __float2bfloat16_rn(acc);
  }
  if (threadIdx.x == 0) args.counters[b * args.Hkv + g] = 0;  // ready for the next call
}

template <int D>
cudaError_t set_decode_attrs() {
  auto k = bifocal_decode_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, DecCfg<D>::kSmem);
  if (e != cudaSuccess) return e;
  // shared memory is the whole carve-out: two CTAs (~110 KB each) per SM
  return cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
}

}  // namespace

int decode_tile_keys() { return kDecKeys; }

int decode_ctas_per_sm() {
  static int cached = 0;
  if (cached > 0) return cached;
  int n = 0;
  if (set_decode_attrs<128>() != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, bifocal_decode_kernel<128>, kDecThreads,
                                                    DecCfg<128>::kSmem) != cudaSuccess ||
      n < 1)
    n = 1;
  cached = n;
  return n;
}

cudaError_t launch_decode(const CUtensorMap& tm_k, const CUtensorMap& tm_v, const DecodeArgs& a, int D,
                          cudaStream_t stream) {
  dim3 grid(a.splits, a.Hkv, a.B);
  cudaError_t e;
  if (D == 128) {
    if ((e = set_decode_attrs<128>()) != cudaSuccess) return e;
    bifocal_decode_kernel<128><<<grid, kDecThreads, DecCfg<128>::kSmem, stream>>>(tm_k, tm_v, a);
  } else {
    if ((e = set_decode_attrs<64>()) != cudaSuccess) return e;
    bifocal_decode_kernel<64><<<grid, kDecThreads, DecCfg<64>::kSmem, stream>>>(tm_k, tm_v, a);
  }
  return cudaGetLastError();
}

}  // namespace jl
