// Fused Dynamic Bifocal RoPE prefill for sm_100a, with remote scores carried at
// about 22 significant bits (the library's default prefill path).
//
// A causal (query i, key j) pair with i - j < w0 is scored with the base-rotated
// Q and K (exact base RoPE); every other causal pair with R(p_q(i)) q and
// R(f(j)) k (Jet-Long review, "Method"; gist.science summary, "Methodologie
// §1").  The inputs are rotated at their absolute positions, so the remote rows
// are R(dq_i) Q_i and R(dk_j) K_j with dq_i = p_q(i) - i, dk_j = f(j) - j: RoPE
// rotations compose additively (gist.science summary, "§2 On-the-Fly Correctie
// Rotatie").  Nothing is written back to the inputs:
//   * a rotation warpgroup rotates the block's query rows once, in fp32
//     registers, into TMEM as fp16 hi + lo (hi = fp16(x), lo = fp16(x - hi);
//     Q_hi and Q_lo are the A operands);
//   * the key tiles' hi / lo rows come either from the correction pass
//     (rope_rotate.cu, once per KV head, fp32 math; the default, kRotK =
//     false) or from the same warpgroup, which then reads each key row of a
//     remote tile from global memory one tile ahead, rotates it in registers
//     and writes hi / lo into shared memory in the 128-byte-swizzled K-major
//     layout the tensor core reads (kRotK = true; no scratch, but measured
//     3.7x slower at 128K on B200: the per-tile row loads, the second
//     unrolled code region and the per-tile synchronisation cost more than
//     the correction pass, which serves every query head of a KV head at
//     once);
//   * a remote score tile is S = Q_hi K_hi + Q_hi K_lo + Q_lo K_hi (fp32
//     accumulate): a score's rounding error is about 2^-21 of |q| |k|
//     instead of 2^-11 for one fp16 product (which is what a key of large norm
//     that dominates a softmax row turns into an LSE error).
// In-kernel correction angles theta_t * d come from a factor R(theta_t (d_x0 -
// 16 a)) for the row set's first row x0 (fp64: one sincos per CTA, its whole
// turns removed exactly first, then an fp64 recurrence from one key tile to the
// next) times a table R(-theta_t b), with d = d_x0 - (16 a + b) inside the set.
//
// Each 128 x 128 (query block, key block) tile is visited once per score set it
// needs (remote passes first, then local passes; a tile straddling the band
// edge gets both, with complementary masks), all feeding one online softmax.
//
// CTA = one 128-row query block of one query head.  Warp roles (384 threads):
//   warp 0      TMA producer: V and (pre-rotated) K, 2 stages each
//   warp 1      tcgen05 MMA issuer; owns the TMEM allocation (512 columns)
//   warps 4-7   softmax (thread = query row = TMEM lane)
//   warps 8-11  rotation: query rows into TMEM (and key tiles with kRotK)
// TMEM columns: S double buffer at 0 / 128 (P, bf16, overwrites the first 64
// columns of its S), O at 256, Q_hi (or the base Q) at 256 + D, Q_lo at
// 256 + 3D/2.  MMA order S(0) S(1) PV(0) S(2) PV(1) S(3) ...: the tensor core
// computes the next tile's scores while the softmax works on this one.
#include "jl_kernels.cuh"

namespace jl {

namespace {

constexpr int kHThreads = 384;
constexpr int kHStages = 2;
constexpr int kHLaunchRegs = 168;  // 65536 / 384, rounded down to a multiple of 8
// Registers per thread of each warpgroup after setmaxnreg.  With key tiles
// rotated in the kernel the rotation warpgroup holds two key rows in flight
// and needs as many as the softmax; otherwise it only sets up the query
// operands, and the producer / MMA warpgroup gets the difference (the MMA
// thread's loop then keeps all its state in registers).
template <bool kRotK>
struct HRegs {
  static constexpr int kProducer = kRotK ? 104 : 152;  // warpgroup 0: TMA producer, MMA issuer
  static constexpr int kSoftmax = 200;                 // warpgroup 1
  static constexpr int kRotation = kRotK ? 200 : 152;  // warpgroup 2
  static_assert(128 * (kProducer + kSoftmax + kRotation) <= kHThreads * kHLaunchRegs,
                "register split exceeds the launch pool");
};
constexpr int kSlab = 128 * 128;  // one 128-row x 128-byte swizzled slab

template <int D>
struct HCfg {
  static constexpr int kChunks = D / 64;  // 64-element (128 B) slabs per row
  static constexpr int kTile = 128 * D * 2;
  static constexpr int kKOff = 0;                               // [stage][hi | lo]
  static constexpr int kVOff = kKOff + kHStages * 2 * kTile;    // [stage]
  static constexpr int kT1Off = kVOff + kHStages * kTile;       // R(-theta_t b): [t/2][b][t&1] float2
  static constexpr int kT1Bytes = (D / 2) * 16 * 8;
  static constexpr int kCOff = kT1Off + kT1Bytes;               // [buffer][t/2][a][t&1] float2
  static constexpr int kCBytes = (D / 2) * 8 * 8;               // buffers 0, 1: key tiles; 2: query block
  static constexpr int kBarOff = kCOff + 3 * kCBytes;
  static constexpr int kUsed = kBarOff + 256;
  // At least 120 KB so only one CTA is resident per SM (each allocates 512
  // TMEM columns).
  static constexpr int kSmem = (kUsed < 120 * 1024 ? 120 * 1024 : kUsed) + 1024;
};

// barrier slots
// Every barrier the MMA thread commits to or waits on costs tensor-pipe time
// (the issuing thread has no slack between products), so each signal serves
// every consumer that can use it: the score commit of a pass also frees the
// key stage it read, and the P V commit also tells the softmax that O holds
// that pass's product.  Stage s, S buffer s and V stage s all belong to the
// passes p with p % 2 == s.
//
// With pre-rotated keys (the default) the MMA thread waits once per pass:
// hReady[s] gathers everything pass p (p % 2 == s) needs before its P V and
// the next score products of the same parity.  Phase 0 of hReady[s] holds
// K(s) and V(s) for the first two passes (the softmax arrives once at the
// start); phase n >= 1 is pass p = 2 (n - 1) + s: P(p) written (128 softmax
// arrivals), V(p) and K(p + 2) landed (the producer's arrival comes with
// K(p + 2), or alone when there is none).  Each party registers on phase n
// only after something it waited for shows phase n - 1 complete: the
// producer's K(p + 2) follows S(p), V(p)'s bytes follow P V of pass p - 2,
// and P(p) follows S(p), all issued after the MMA thread's wait on phase n - 1.
// With keys corrected in the kernel, hReady[s] is "key tile p in shared
// memory" (128 rotation-thread arrivals) and V and P have barriers of their own.
enum {
  hReady = 0,         // [parity]: the pass barrier above (key tile p with in-kernel keys)
  hVFull = 2,         // [stage] (in-kernel keys only)
  hVEmpty = 4,        // [stage]: O += P V of the stage's latest pass has completed
  hSFull = 6,         // [S buffer]: scores complete; the key stage they read is free
  hPFull = 8,         // [S buffer]: P written over S (in-kernel keys only)
  hQReady = 10,       // the query operands are in TMEM (phase 0: first pass kind, 1: after the switch)
  hQEmpty = 11,       // the last product reading the first query operands has completed
  hCReady = 12,       // rotation warpgroup: factor table of the next tile written
  hOFinal = 13,
  hDrain = 14,
  hNumBars = 15
};
static_assert(hNumBars * 8 <= 192, "barrier block overflow");

__device__ __forceinline__ bool h_drain_wait(uint32_t bar, uint32_t parity) {
  // Only after an abort: wait (up to ~100 ms) for async work already in flight
  // so the CTA never exits while a copy or an MMA still targets it.
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > 100000000ull) return false;
  }
  return true;
}

struct HPass {
  int nb;       // key block
  bool remote;  // corrected operands (hi + lo) or base operands
  int mask;     // 0: band 0 <= i-j < w0, 1: beyond the band i-j >= w0, 2: every causal pair
};

// Pass p of a query block: the fused method visits its remote passes first
// (key blocks nb_rem_max .. 0), then its local passes (nb_max down); the
// inclusion-exclusion calls visit one kind only.
template <int kind>
__device__ __forceinline__ HPass hilo_pass(const Sched& s, int p) {
  HPass r;
  if (kind == kBifocal) {
    if (p < s.n_rem) {
      r.nb = s.nb_rem_max - p;
      r.remote = true;
      r.mask = 1;
    } else {
      r.nb = s.nb_max - (p - s.n_rem);
      r.remote = false;
      r.mask = 0;
    }
  } else {
    r.nb = s.nb_max - p;
    r.remote = kind != kWindowBase;
    r.mask = kind == kCausalRemote ? 2 : 0;
  }
  return r;
}

__device__ __forceinline__ void tmem_st4(uint32_t taddr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// 16-byte global load that does not allocate in L1: the key rows stream
// through once per tile, and L1 (what shared memory leaves of it) is kept for
// the softmax's spilled registers.
__device__ __forceinline__ uint4 ldg_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// x rounded to fp16 (hi) and the rounding residual rounded to fp16 (lo), for
// two values; hi + lo carries about 22 significant bits.
__device__ __forceinline__ void split_f16x2(float a, float b, uint32_t& hi, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(a, b);
  const float2 hf = __half22float2(h);
  const __half2 l = __floats2half2_rn(a - hf.x, b - hf.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

// Bit 15 / 31 of the result is set when that fp16 half of h is inf or NaN.
__device__ __forceinline__ uint32_t f16x2_nonfinite_bits(uint32_t h) { return (h & 0x7FFF7FFFu) + 0x04000400u; }

// Rotates one row of D bf16 values (half-split pairs (t, t + D/2), D/2 words of
// two consecutive dims each) by R(theta_t (base - delta)) with the factor
// C[t][delta >> 4] * T1[t][delta & 15] (C = R(theta_t (base - 16 a)), T1 =
// R(-theta_t b)), and hands each 8-dim unit U (flat index over the row) of the
// fp16 hi and lo results to emit(U, hi[4], lo[4]).  Non-finite hi halves are
// recorded in *range.
template <int D, typename Emit>
__device__ __forceinline__ void rotate_row_hilo(const uint32_t (&raw)[D / 2], const float2* Cb, const float2* T1s,
                                                int delta, uint32_t& range, Emit&& emit) {
  constexpr int H2 = D / 2;
  const int a = delta >> 4, bb = delta & 15;
#pragma unroll
  for (int u = 0; u < H2 / 8; ++u) {
    uint32_t hx[4], lx[4], hy[4], ly[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int t = 8 * u + 2 * k;
      const float4 cf = *reinterpret_cast<const float4*>(&Cb[((t >> 1) * 8 + a) * 2]);
      const float4 tf = *reinterpret_cast<const float4*>(&T1s[((t >> 1) * 16 + bb) * 2]);
      const float c0 = cf.x * tf.x - cf.y * tf.y, s0 = cf.x * tf.y + cf.y * tf.x;
      const float c1 = cf.z * tf.z - cf.w * tf.w, s1 = cf.z * tf.w + cf.w * tf.z;
      const uint32_t xw = raw[t / 2], yw = raw[(t + H2) / 2];
      const float x0 = bf16lo_to_f32(xw), x1 = bf16hi_to_f32(xw);
      const float y0 = bf16lo_to_f32(yw), y1 = bf16hi_to_f32(yw);
      // (x, y) -> (x cos - y sin, y cos + x sin)
      split_f16x2(x0 * c0 - y0 * s0, x1 * c1 - y1 * s1, hx[k], lx[k]);
      split_f16x2(y0 * c0 + x0 * s0, y1 * c1 + x1 * s1, hy[k], ly[k]);
      range |= f16x2_nonfinite_bits(hx[k]) | f16x2_nonfinite_bits(hy[k]);
    }
    emit(u, hx, lx);
    emit(u + H2 / 8, hy, ly);
  }
}

template <int D, bool kRotK, int kKind>
__global__ void __launch_bounds__(kHThreads, 1)
    bifocal_prefill_hilo_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                                const __grid_constant__ CUtensorMap tm_kh, const __grid_constant__ CUtensorMap tm_kl,
                                const __grid_constant__ PrefillHiloArgs args) {
  using C = HCfg<D>;
  constexpr int H2 = D / 2;
  constexpr uint32_t kColO = 256, kColQA = 256 + D, kColQB = 256 + D + D / 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kBarOff + 192);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kBarOff + 196);
  auto bar = [&](int i) -> uint32_t { return smem_addr(&bars[i]); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Work order (CTAs launch in increasing linear index): the CTAs of one KV
  // head's query heads run together, heaviest query blocks first, so the CTAs
  // resident at any time read the same K / V rows and find them in L2.
  const int r = args.r;
  int lin = (int)(blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z));
  const int hg = lin % r;
  lin /= r;
  const int mb = args.num_mb - 1 - lin % args.num_mb;
  lin /= args.num_mb;
  const int kvh = lin % args.Hkv;
  const int b = lin / args.Hkv;
  const int hq = kvh * r + hg;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kHStages; ++s) {
      mbar_init(bar(hReady + s), kRotK ? 128 : 129);
      mbar_init(bar(hVFull + s), 1);
      mbar_init(bar(hVEmpty + s), 1);
      mbar_init(bar(hSFull + s), 1);
      mbar_init(bar(hPFull + s), 128);
    }
    mbar_init(bar(hQReady), 128);
    mbar_init(bar(hQEmpty), 1);
    mbar_init(bar(hCReady), 128);
    mbar_init(bar(hOFinal), 1);
    mbar_init(bar(hDrain), 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), 512u);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int off = args.q_off + mb * 128;                             // position of this block's first query
  const int last = min(off + 127, args.q_off + args.Lq - 1);         // its last query row
  const Sched sc = make_sched<kKind>(off, last, args.w0, false);
  const int npass = sc.n_loc + sc.n_rem;
  const bool q_switch = kKind == kBifocal && sc.n_loc > 0 && sc.n_rem > 0;
  const int p_switch = sc.n_rem;  // first local pass (fused method)

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(HRegs<kRotK>::kProducer));
    if (warp == 0 && lane == 0) {
      // ------------------------------------------------------------ producer
      tma_prefetch_map(&tm_v);
      if (!kRotK) {
        tma_prefetch_map(&tm_k);
        tma_prefetch_map(&tm_kh);
        tma_prefetch_map(&tm_kl);
      }
      int k_last = -1, v_last = -1;
      bool ok = true;
      for (int p = 0; p < npass; ++p) {
        const int s = p & 1;
        const uint32_t ph = (uint32_t)(p >> 1) & 1u;
        const HPass ps = hilo_pass<kKind>(sc, p);
        const uint32_t vdst = sbase + C::kVOff + s * C::kTile;
        if constexpr (!kRotK) {
          // K(p): its stage is free once S(p - 2) has completed; it belongs to
          // the phase of pass p - 2 (phase 0 for p < 2, together with V(p))
          if (!(ok = mbar_wait(bar(hSFull + s), ph ^ 1u, abort_flag, args.dev_error))) break;
          const uint32_t khi = sbase + C::kKOff + s * 2 * C::kTile;
          const uint32_t kbytes = (uint32_t)((ps.remote ? 2 : 1) * C::kTile);
          mbar_arrive_expect_tx(bar(hReady + s), p < 2 ? kbytes + (uint32_t)C::kTile : kbytes);
          for (int c = 0; c < C::kChunks; ++c) {
            if (ps.remote) {
              tma_load_4d(khi + c * kSlab, &tm_kh, bar(hReady + s), c * 64, kvh, ps.nb * 128, b);
              tma_load_4d(khi + C::kTile + c * kSlab, &tm_kl, bar(hReady + s), c * 64, kvh, ps.nb * 128, b);
            } else {
              tma_load_4d(khi + c * kSlab, &tm_k, bar(hReady + s), c * 64, kvh, ps.nb * 128, b);
            }
          }
          k_last = p;
          // V(p): its stage is free once P V of pass p - 2 has completed, and
          // by then the phase of pass p is open
          if (p >= 2) {
            if (!(ok = mbar_wait(bar(hVEmpty + s), ph ^ 1u, abort_flag, args.dev_error))) break;
            mbar_expect_tx(bar(hReady + s), (uint32_t)C::kTile);
          }
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_4d(vdst + c * kSlab, &tm_v, bar(hReady + s), c * 64, kvh, ps.nb * 128, b);
          v_last = p;
          if (p + 2 >= npass) {
            // no K(p + 2): pass p's phase gets the producer's arrival now
            if (p < 2 && !(ok = mbar_wait(bar(hReady + s), 0u, abort_flag, args.dev_error))) break;
            mbar_arrive(bar(hReady + s));
          }
        } else {
          if (!(ok = mbar_wait(bar(hVEmpty + s), ph ^ 1u, abort_flag, args.dev_error))) break;
          mbar_arrive_expect_tx(bar(hVFull + s), (uint32_t)C::kTile);
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_4d(vdst + c * kSlab, &tm_v, bar(hVFull + s), c * 64, kvh, ps.nb * 128, b);
          v_last = p;
        }
      }
      if (!ok) {
        // Let every copy already issued land before the CTA can exit.  (With
        // pre-rotated keys a pass barrier also waits for softmax arrivals
        // that an abort may never bring, so those waits end on their bound.)
        for (int p = max(0, k_last - kHStages + 1); p <= k_last; ++p)
          h_drain_wait(bar(hReady + (p & 1)), (uint32_t)(p >> 1) & 1u);
        for (int p = max(0, v_last - kHStages + 1); p <= v_last; ++p) {
          if constexpr (kRotK)
            h_drain_wait(bar(hVFull + (p & 1)), (uint32_t)(p >> 1) & 1u);
          else if (p >= 2)
            h_drain_wait(bar(hReady + (p & 1)), (uint32_t)((p >> 1) + 1) & 1u);
        }
      }
    } else if (warp == 1 && lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      const uint32_t id_loc = make_idesc_16bit(128, 128, false, false);  // bf16 Q K
      const uint32_t id_rem = make_idesc_16bit(128, 128, false, true);   // fp16 Q_hi / Q_lo, K_hi / K_lo
      const uint32_t id_pv = make_idesc_16bit(128, D, true, false);      // bf16 P V
      // Shared-memory matrix descriptors, built once: K_hi of each stage (K_lo
      // is one tile further) and V of each stage.  A k-step of 16 elements
      // moves the start address by 32 B inside a 128-byte slab and by a slab
      // every four steps; the address field holds bytes >> 4.
      const uint64_t dk_hi0 = make_sdesc_sw128(sbase + C::kKOff, 16, 1024);
      const uint64_t dk_hi1 = make_sdesc_sw128(sbase + C::kKOff + 2 * C::kTile, 16, 1024);
      const uint64_t dv0 = make_sdesc_sw128(sbase + C::kVOff, kSlab, 1024);
      const uint64_t dv1 = make_sdesc_sw128(sbase + C::kVOff + C::kTile, kSlab, 1024);
      auto kstep_off = [](int ks) -> uint64_t { return (uint64_t)(((ks >> 2) * kSlab + (ks & 3) * 32) >> 4); };
      // passes with corrected (hi + lo) operands: the fused method's remote
      // passes come first; the single-kind calls use one operand kind
      const int n_hilo = kKind == kBifocal ? sc.n_rem : (kKind != kWindowBase ? npass : 0);
      // Score products of pass q into S buffer q % 2, then its commit (the
      // softmax may read S; the key stage is free).
      // The score products into S buffer s (= the pass's parity, a constant at
      // every call on the hot path): remote passes Q_hi K_hi + Q_hi K_lo +
      // Q_lo K_hi into one accumulator, local passes one bf16 product.
      auto s_mmas_hilo = [&](int s) {
        const uint32_t d = tmem + (uint32_t)(128 * s);
        // descriptors of the stage's K_hi / K_lo tiles (k-step offsets are
        // added below as compile-time constants: one add per MMA)
        const uint64_t dkh = s == 0 ? dk_hi0 : dk_hi1;
        const uint64_t dkl = dkh + (uint64_t)(C::kTile >> 4);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          mma_ts(d, tmem + kColQA + (uint32_t)(ks * 8), dkh + kstep_off(ks), id_rem, ks > 0 ? 1u : 0u);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          mma_ts(d, tmem + kColQA + (uint32_t)(ks * 8), dkl + kstep_off(ks), id_rem, 1u);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          mma_ts(d, tmem + kColQB + (uint32_t)(ks * 8), dkh + kstep_off(ks), id_rem, 1u);
      };
      auto s_mmas_local = [&](int s) {
        const uint32_t d = tmem + (uint32_t)(128 * s);
        const uint64_t dkh = s == 0 ? dk_hi0 : dk_hi1;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          mma_ts(d, tmem + kColQA + (uint32_t)(ks * 8), dkh + kstep_off(ks), id_loc, ks > 0 ? 1u : 0u);
      };
      // Score products of pass q with its commit (the softmax may read S; the
      // key stage is free), and the query operands' release after the last
      // remote pass.
      auto s_products = [&](int q, int s) {
        if (q < n_hilo)
          s_mmas_hilo(s);
        else
          s_mmas_local(s);
        tc_commit(bar(hSFull + s));
        if (q_switch && q == p_switch - 1) tc_commit(bar(hQEmpty));
      };
      // O += P V of pass p, then its commit (V stage free; O holds the pass).
      auto pv_products = [&](int p, int s) {  // s = p % 2
        const uint64_t dv = s == 0 ? dv0 : dv1;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          // V is MN-major here: 64-dim slabs kSlab apart, 8-key groups 1024 B
          // apart, 16 keys (2048 B) per k-step.
          mma_ts(tmem + kColO, tmem + (uint32_t)(128 * s + ks * 8), dv + (uint64_t)((ks * 2048) >> 4), id_pv,
                 (p > 0 || ks > 0) ? 1u : 0u);
        }
        tc_commit(bar(hVEmpty + s));
      };
      // the query operands of pass q (the first pass kind, or the base rows
      // after the switch) must be in TMEM
      auto wait_q = [&](int q) -> bool {
        if (q == 0 || (q_switch && q == p_switch))
          return mbar_wait(bar(hQReady), q == 0 ? 0u : 1u, abort_flag, args.dev_error);
        return true;
      };
      bool ok = true;
      if constexpr (!kRotK) {
        // MMA order S(0) S(1) PV(0) S(2) PV(1) ...: one wait per pass, on the
        // pass barrier that holds P(p), V(p) and K(p + 2).
        for (int q = 0; q < 2 && q < npass && ok; ++q) {
          ok = wait_q(q) && mbar_wait(bar(hReady + q), 0u, abort_flag, args.dev_error);
          if (!ok) break;
          tc_fence_after();
          s_products(q, q);
        }
        // One step per pass: wait, P V(p), then S(p + 2).  The passes run in
        // segments whose steps test nothing at run time (remote score
        // products, local ones, none), with the one or two steps around the
        // switch of query operands in between; each segment is unrolled by
        // two so that each copy's parity (S buffer, stage, barrier addresses)
        // is a constant.  Every instruction between two products on this
        // thread costs tensor time.
        auto pass_wait = [&](int p, int s) -> bool {
          if (!mbar_wait(bar(hReady + s), (uint32_t)((p >> 1) + 1) & 1u, abort_flag, args.dev_error)) return false;
          tc_fence_after();
          pv_products(p, s);
          return true;
        };
        auto step_hilo = [&](int p, int s) -> bool {
          if (!pass_wait(p, s)) return false;
          s_mmas_hilo(s);
          tc_commit(bar(hSFull + s));
          return true;
        };
        auto step_local = [&](int p, int s) -> bool {
          if (!pass_wait(p, s)) return false;
          s_mmas_local(s);
          tc_commit(bar(hSFull + s));
          return true;
        };
        auto step_any = [&](int p, int s) -> bool {
          if (!pass_wait(p, s)) return false;
          if (p + 2 < npass) {
            if (q_switch && p + 2 == p_switch) {
              if (!wait_q(p + 2)) return false;
              tc_fence_after();
            }
            s_products(p + 2, s);
          }
          return true;
        };
        auto run = [&](int p0, int p1, auto&& body) {
          int p = p0;
          if (ok && p < p1 && (p & 1)) ok = body(p++, 1);
          for (; p + 1 < p1 && ok; p += 2) ok = body(p, 0) && body(p + 1, 1);
          if (ok && p < p1) ok = body(p, 0);
        };
        // iterations p issue S(p + 2) while p < npass - 2; it is remote while
        // p + 2 < n_hilo; with a switch, p_switch = n_hilo and the steps that
        // release the remote query operands (p_switch - 3) and wait for the
        // base ones (p_switch - 2) test at run time
        const int n_s = max(npass - 2, 0);
        auto clampi = [&](int x) { return min(max(x, 0), n_s); };
        const int a_end = clampi(q_switch ? n_hilo - 3 : n_hilo - 2);
        const int b_end = clampi(q_switch ? n_hilo - 1 : n_hilo - 2);
        run(0, a_end, step_hilo);
        run(a_end, b_end, step_any);
        run(b_end, n_s, step_local);
        run(n_s, npass, pass_wait);
      } else {
        auto issue_s = [&](int q) -> bool {
          if (!wait_q(q)) return false;
          if (!mbar_wait(bar(hReady + (q & 1)), (uint32_t)(q >> 1) & 1u, abort_flag, args.dev_error)) return false;
          tc_fence_after();
          s_products(q, q & 1);
          return true;
        };
        // O += P V once the softmax has written all of P.
        auto issue_pv = [&](int p) -> bool {
          const int s = p & 1;
          const uint32_t ph = (uint32_t)(p >> 1) & 1u;
          if (!mbar_wait(bar(hVFull + s), ph, abort_flag, args.dev_error)) return false;
          if (!mbar_wait(bar(hPFull + s), ph, abort_flag, args.dev_error)) return false;
          tc_fence_after();
          pv_products(p, s);
          return true;
        };
        if (npass > 0) {
          ok = issue_s(0);
          if (ok && npass > 1) ok = issue_s(1);
          for (int p = 0; p < npass && ok; ++p) {
            ok = issue_pv(p);
            if (ok && p + 2 < npass) ok = issue_s(p + 2);
          }
        }
      }
      // Every product issued must have completed before TMEM is released.
      if (ok) {
        tc_commit(bar(hOFinal));
        h_drain_wait(bar(hOFinal), 0);
      } else {
        tc_commit(bar(hDrain));
        h_drain_wait(bar(hDrain), 0);
      }
    }
  } else if (warp < 8) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(HRegs<kRotK>::kSoftmax));
    // ------------------------------------------------------------ softmax
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t o_addr = tmem + lane_off + kColO;
    const float sl2 = args.scale_log2;
    const int w0 = args.w0;
    float m_used = -INFINITY;
    float l_sum = 0.f;
    bool ok = true;
    if constexpr (!kRotK) {
      // phase 0 of both pass barriers (the first two passes) has no P
      mbar_arrive(bar(hReady + 0));
      mbar_arrive(bar(hReady + 1));
    }

    for (int p = 0; p < npass; ++p) {
      const int s = p & 1;
      const uint32_t ph = (uint32_t)(p >> 1) & 1u;
      ok = mbar_wait(bar(hSFull + s), ph, abort_flag, args.dev_error);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const HPass ps = hilo_pass<kKind>(sc, p);
      const int mkind = ps.mask;
      const int dd0 = off - 128 * ps.nb;  // i - j at row 0, column 0
      const uint32_t s_addr = tmem + lane_off + (uint32_t)(128 * s);

      // S in two 64-column halves: the first half's mask and partial row max
      // run while the second half's load is in flight.
      uint32_t sr[4][32];
      tmem_ld32(s_addr, sr[0]);
      tmem_ld32(s_addr + 32, sr[1]);
      tmem_ld_wait(sr[0]);
      tmem_ld_wait(sr[1]);
      tmem_ld32(s_addr + 64, sr[2]);
      tmem_ld32(s_addr + 96, sr[3]);

      float x[128];  // raw scores (fp32 accumulator values)
      const bool need_mask = mkind == 1 ? (dd0 - 127 < w0)
                             : mkind == 0 ? (dd0 - 127 < 0 || dd0 + 127 >= w0)
                                          : (dd0 - 127 < 0);
      const int dd = dd0 + row;  // i - j = dd - col
      float m4[4];
      auto take = [&](int c0) {
#pragma unroll
        for (int c = c0; c < c0 + 2; ++c)
#pragma unroll
          for (int k = 0; k < 32; ++k) x[c * 32 + k] = __uint_as_float(sr[c][k]);
        if (need_mask) {
#pragma unroll
          for (int col = c0 * 32; col < c0 * 32 + 64; ++col) {
            const int rel = dd - col;
            const bool keep = mkind == 1 ? (rel >= w0) : mkind == 0 ? (rel >= 0 && rel < w0) : (rel >= 0);
            if (!keep) x[col] = -INFINITY;
          }
        }
      };
      take(0);
#pragma unroll
      for (int j = 0; j < 4; ++j) m4[j] = fmaxf(x[j], x[4 + j]);
#pragma unroll
      for (int col = 8; col < 64; col += 8)
#pragma unroll
        for (int j = 0; j < 4; ++j) m4[j] = fmax3(m4[j], x[col + j], x[col + 4 + j]);
      // (the partial maxima are tied to this wait, so they are taken while the
      // second half of S is in flight)
      asm volatile("tcgen05.wait::ld.sync.aligned;" : "+f"(m4[0]), "+f"(m4[1]), "+f"(m4[2]), "+f"(m4[3])::"memory");
      tmem_ld_wait(sr[2]);
      tmem_ld_wait(sr[3]);
      take(2);
#pragma unroll
      for (int col = 64; col < 128; col += 8)
#pragma unroll
        for (int j = 0; j < 4; ++j) m4[j] = fmax3(m4[j], x[col + j], x[col + 4 + j]);
      const float mt = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * sl2;
      const float m_new = fmaxf(m_used, mt);
      float alpha = 1.f;
      bool rescale_o = false;
      // Lazy rescaling: keep the exponent offset until the row max has grown
      // by more than 2^8; p <= 256 stays exact enough in fp32 / bf16.
      if (m_new > m_used + 8.f) {
        if (m_used != -INFINITY) {
          alpha = ex2_approx(m_used - m_new);
          rescale_o = true;
        } else {
          alpha = 0.f;
        }
        l_sum *= alpha;
        m_used = m_new;
      }
      const float msub = (m_used == -INFINITY) ? 0.f : m_used;
      // O must be rescaled before this pass's P V: in the (rare) passes that
      // need it, P is released after the rescale.
      const bool resc = __any_sync(0xffffffffu, rescale_o) && p > 0;
      const uint64_t sc2 = f2_pack(sl2, sl2), nm2 = f2_pack(-msub, -msub);
      uint64_t acc[2] = {0ull, 0ull};
      auto pair_exp = [&](int half, int k) -> uint32_t {
        const uint64_t ev = f2_fma(f2_pack(x[half * 64 + 2 * k], x[half * 64 + 2 * k + 1]), sc2, nm2);
        float e0, e1;
        f2_unpack(ev, e0, e1);
        const float p0 = ex2_approx(e0), p1 = ex2_approx(e1);
        acc[k & 1] = f2_add(acc[k & 1], f2_pack(p0, p1));
        return pack_bf16x2(p0, p1);
      };
      {
        uint32_t pk[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) pk[k] = pair_exp(0, k);
        tmem_st32(s_addr, pk);
      }
      {
        uint32_t pk[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) pk[k] = pair_exp(1, k);
        tmem_st32(s_addr + 32, pk);
        if (resc) {
          // O must hold the previous pass's product first.
          bool okw = mbar_wait(bar(hVEmpty + ((p - 1) & 1)), (uint32_t)((p - 1) >> 1) & 1u, abort_flag,
                               args.dev_error);
          okw = __all_sync(0xffffffffu, okw);
          if (!okw) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t ov[32];
            tmem_ld32(o_addr + c * 32, ov);
            tmem_ld_wait(ov);
#pragma unroll
            for (int k = 0; k < 32; ++k) ov[k] = __float_as_uint(__uint_as_float(ov[k]) * alpha);
            tmem_st32(o_addr + c * 32, ov);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar(kRotK ? hPFull + s : hReady + s));
      }
      {
        float a0, a1;
        f2_unpack(f2_add(acc[0], acc[1]), a0, a1);
        l_sum += a0 + a1;
      }
    }

    if (ok) {
      ok = mbar_wait(bar(hOFinal), 0, abort_flag, args.dev_error);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      const int i = mb * 128 + row;  // row of this chunk's Q / O / LSE
      const float inv = (l_sum > 0.f && npass > 0) ? 1.f / l_sum : 0.f;
      const size_t obase = (((size_t)b * args.Lq + i) * args.Hq + hq) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ov[32];
        tmem_ld32(o_addr + c * 32, ov);  // (never written when npass == 0; inv is 0 then)
        tmem_ld_wait(ov);
        if (i < args.Lq) {
          if (args.o_f32 != nullptr) {
            float4* dst = reinterpret_cast<float4*>(args.o_f32 + obase + c * 32);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const float4 w = npass > 0 ? make_float4(__uint_as_float(ov[4 * k]) * inv,
                                                       __uint_as_float(ov[4 * k + 1]) * inv,
                                                       __uint_as_float(ov[4 * k + 2]) * inv,
                                                       __uint_as_float(ov[4 * k + 3]) * inv)
                                         : make_float4(0.f, 0.f, 0.f, 0.f);
              dst[k] = w;
            }
          } else {
            uint32_t w[16];
#pragma unroll
            for (int k = 0; k < 16; ++k)
              w[k] = npass > 0
                         ? pack_bf16x2(__uint_as_float(ov[2 * k]) * inv, __uint_as_float(ov[2 * k + 1]) * inv)
                         : 0u;  // no key at all: O = 0, LSE = -inf
            uint4* dst = reinterpret_cast<uint4*>(args.o + obase + c * 32);
#pragma unroll
            for (int k = 0; k < 4; ++k) dst[k] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
          }
        }
      }
      if (args.lse != nullptr && i < args.Lq) {
        const float m = (m_used == -INFINITY) ? 0.f : m_used;
        args.lse[((size_t)b * args.Hq + hq) * args.Lq + i] =
            l_sum > 0.f ? (m + __log2f(l_sum)) * 0.69314718055994531f : -INFINITY;
      }
    }
  } else {
    if constexpr (kRotK)
      asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(HRegs<kRotK>::kRotation));
    else
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(HRegs<kRotK>::kRotation));
    // ------------------------------------------------------------ rotation
    const int wq = warp & 3;
    const int e = wq * 32 + lane;  // query row of the block / key row of the tile
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    float2* T1s = reinterpret_cast<float2*>(smem + C::kT1Off);
    float2* Cs = reinterpret_cast<float2*>(smem + C::kCOff);
    constexpr int kCElems = H2 * 8;  // float2 per factor buffer
    const int64_t G = args.G;
    uint32_t range = 0;
    bool ok = true;

    // Factor buffer `buf` for a row set whose first row's correction is
    // `base` (dk_j0 or dq_i0): C[t][a] = R(theta_t (base - 16 a)).  One fp64
    // sincos per (t, thread); 256 / D threads share a t.
    auto fill_c = [&](int buf, int64_t base) {
      constexpr int TPT = 256 / D;
      constexpr int APT = 8 / TPT;
      const int t = e / TPT;
      const int a0 = (e % TPT) * APT;
      double sn, cs;
      sincos_int_angle(base, args.u_hi[t], args.u_lo[t], &sn, &cs);
      const float cb = (float)cs, sb = (float)sn;
#pragma unroll
      for (int j = 0; j < APT; ++j) {
        const float2 m = args.t16[t * 8 + a0 + j];
        Cs[buf * kCElems + ((t >> 1) * 8 + a0 + j) * 2 + (t & 1)] = make_float2(cb * m.x - sb * m.y, cb * m.y + sb * m.x);
      }
    };
    // Position offset of row e of a row set starting at position x0 from the
    // set's first row: f(x0 + e) - f(x0) - e = -delta, delta in [0, 127].
    auto delta_of = [&](int64_t x0) -> int { return e - (int)((x0 % G + e) / G); };

    uint32_t raw[H2];  // one row of bf16 pairs
    auto load_row = [&](const __nv_bfloat16* src, bool valid) {
      const uint4* s4 = reinterpret_cast<const uint4*>(src);
#pragma unroll
      for (int w = 0; w < H2 / 4; ++w) {
        const uint4 v = valid ? ldg_stream(s4 + w) : make_uint4(0u, 0u, 0u, 0u);
        raw[4 * w] = v.x;
        raw[4 * w + 1] = v.y;
        raw[4 * w + 2] = v.z;
        raw[4 * w + 3] = v.w;
      }
    };
    const int qi = mb * 128 + e;  // this thread's query row in the chunk
    const __nv_bfloat16* qrow = args.q + (((size_t)b * args.Lq + qi) * args.Hq + hq) * D;
    // The query operands of the base (local) passes: the base row, as bf16.
    auto write_base_q = [&]() {
#pragma unroll
      for (int U = 0; U < D / 8; ++U)
        tmem_st4(tmem + lane_off + kColQA + 4 * U, raw[4 * U], raw[4 * U + 1], raw[4 * U + 2], raw[4 * U + 3]);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(hQReady));
    };

    // Tables (R(-theta_t b) from the arguments) and the query block's factors.
    for (int i = e; i < H2 * 16; i += 128) {
      const int t = i >> 4, bb = i & 15;
      T1s[((t >> 1) * 16 + bb) * 2 + (t & 1)] = args.t1[i];
    }
    const int64_t dq0 = off / G + args.shift - off;  // dq at the block's first query
    fill_c(2, dq0);
    mbar_arrive(bar(hCReady));
    ok = mbar_wait(bar(hCReady), 0, abort_flag, args.dev_error);

    // Query operands of the first pass kind.
    if (ok && npass > 0) {
      load_row(qrow, qi < args.Lq);
      if (hilo_pass<kKind>(sc, 0).remote) {
        rotate_row_hilo<D>(raw, Cs + 2 * kCElems, T1s, delta_of(off), range,
                           [&](int U, const uint32_t (&h)[4], const uint32_t (&l)[4]) {
                             tmem_st4(tmem + lane_off + kColQA + 4 * U, h[0], h[1], h[2], h[3]);
                             tmem_st4(tmem + lane_off + kColQB + 4 * U, l[0], l[1], l[2], l[3]);
                           });
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar(hQReady));
      } else {
        write_base_q();
      }
    }

    if (kRotK) {
      // Key tiles.  Each thread rotates key row e of a tile; the rows of the
      // next two tiles are kept in flight in two register buffers, so a
      // tile's loads overlap the rotation of the one before it.
      auto load_k = [&](uint32_t (&dst)[H2], int p) {
        const HPass ps = hilo_pass<kKind>(sc, p);
        const int j = ps.nb * 128 + e;
        const bool valid = j < args.k_rows;
        const uint4* s4 = reinterpret_cast<const uint4*>(
            args.k + (((size_t)b * args.k_rows + (valid ? j : 0)) * args.Hkv + kvh) * D);
#pragma unroll
        for (int w = 0; w < H2 / 4; ++w) {
          const uint4 v = valid ? ldg_stream(s4 + w) : make_uint4(0u, 0u, 0u, 0u);
          dst[4 * w] = v.x;
          dst[4 * w + 1] = v.y;
          dst[4 * w + 2] = v.z;
          dst[4 * w + 3] = v.w;
        }
      };
      // Per-tile factor base R(theta_t dk_j0) for this thread's t, carried in
      // fp64 from one remote tile to the next (key blocks descend by one:
      // dk_j0 grows by 128 - ceil(128 / G) or 128 - floor(128 / G)); one fp64
      // sincos for the first remote tile of the CTA.
      constexpr int TPT = 256 / D;
      constexpr int APT = 8 / TPT;
      const int ft = e / TPT;
      const int fa0 = (e % TPT) * APT;
      const double uh = args.u_hi[ft], ul = args.u_lo[ft];
      const int64_t s_lo = 128 - (128 + G - 1) / G;
      double st_s[2], st_c[2];
      sincos_int_angle(s_lo, uh, ul, &st_s[0], &st_c[0]);
      sincos_int_angle(s_lo + 1, uh, ul, &st_s[1], &st_c[1]);
      double kb_c = 1.0, kb_s = 0.0;
      int64_t prev_dk0 = 0;
      bool have_base = false;
      auto fill_k = [&](int p) {
        const HPass ps = hilo_pass<kKind>(sc, p);
        if (ps.remote) {
          const int64_t j0 = (int64_t)ps.nb * 128;
          const int64_t dk0 = j0 / G - j0;
          if (!have_base) {
            sincos_int_angle(dk0, uh, ul, &kb_s, &kb_c);
            have_base = true;
          } else {
            const int i = (int)(dk0 - prev_dk0 - s_lo);  // 0 or 1
            const double c = kb_c * st_c[i] - kb_s * st_s[i];
            kb_s = kb_c * st_s[i] + kb_s * st_c[i];
            kb_c = c;
          }
          prev_dk0 = dk0;
          const float cb = (float)kb_c, sb = (float)kb_s;
#pragma unroll
          for (int jj = 0; jj < APT; ++jj) {
            const float2 m = args.t16[ft * 8 + fa0 + jj];
            Cs[(p & 1) * kCElems + ((ft >> 1) * 8 + fa0 + jj) * 2 + (ft & 1)] =
                make_float2(cb * m.x - sb * m.y, cb * m.y + sb * m.x);
          }
        }
        mbar_arrive(bar(hCReady));  // tile p's factors (if any) are written
      };
      const uint32_t rowoff = (uint32_t)(e * 128);
      const uint32_t sw = (uint32_t)(e & 7);
      auto unit_addr = [&](uint32_t slot, int U) -> uint32_t {
        return slot + (uint32_t)((U >> 3) * kSlab) + rowoff + ((((uint32_t)U & 7u) ^ sw) << 4);
      };
      // Rotate (or, for a local pass, copy) tile p from `src` into its stage.
      auto process = [&](const uint32_t (&src)[H2], int p) -> bool {
        const int s = p & 1;
        const HPass ps = hilo_pass<kKind>(sc, p);
        // every thread's factors for tile p, then the stage's previous reader
        if (!mbar_wait(bar(hCReady), (uint32_t)(p + 1) & 1u, abort_flag, args.dev_error)) return false;
        if (!mbar_wait(bar(hSFull + s), ((uint32_t)(p >> 1) & 1u) ^ 1u, abort_flag, args.dev_error)) return false;
        const uint32_t khi = sbase + C::kKOff + s * 2 * C::kTile;
        if (ps.remote) {
          const int64_t j0 = (int64_t)ps.nb * 128;
          rotate_row_hilo<D>(src, Cs + (p & 1) * kCElems, T1s, delta_of(j0), range,
                             [&](int U, const uint32_t (&h)[4], const uint32_t (&l)[4]) {
                               sts128(unit_addr(khi, U), h[0], h[1], h[2], h[3]);
                               sts128(unit_addr(khi + C::kTile, U), l[0], l[1], l[2], l[3]);
                             });
        } else {
#pragma unroll
          for (int U = 0; U < D / 8; ++U)
            sts128(unit_addr(khi, U), src[4 * U], src[4 * U + 1], src[4 * U + 2], src[4 * U + 3]);
        }
        fence_proxy_async_smem();  // the tensor core reads these rows through the async proxy
        mbar_arrive(bar(hReady + s));
        if (q_switch && p == p_switch) {
          // The remote query operands have been read for the last time: put
          // the base rows in their place.
          if (!mbar_wait(bar(hQEmpty), 0, abort_flag, args.dev_error)) return false;
          tc_fence_after();
          const uint4* q4 = reinterpret_cast<const uint4*>(qrow);
#pragma unroll
          for (int U = 0; U < D / 8; ++U) {
            const uint4 w = qi < args.Lq ? ldg_stream(q4 + U) : make_uint4(0u, 0u, 0u, 0u);
            tmem_st4(tmem + lane_off + kColQA + 4 * U, w.x, w.y, w.z, w.w);
          }
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(bar(hQReady));
        }
        if (p + 1 < npass) fill_k(p + 1);
        return true;
      };
      uint32_t rawB[H2];
      if (ok && npass > 0) {
        load_k(raw, 0);
        fill_k(0);
        if (npass > 1) load_k(rawB, 1);
      }
      for (int p = 0; p < npass && ok; p += 2) {
        if (!(ok = process(raw, p))) break;
        if (p + 2 < npass) load_k(raw, p + 2);
        if (p + 1 >= npass) break;
        if (!(ok = process(rawB, p + 1))) break;
        if (p + 3 < npass) load_k(rawB, p + 3);
      }
    } else if (ok && q_switch) {
      ok = mbar_wait(bar(hQEmpty), 0, abort_flag, args.dev_error);
      if (ok) {
        tc_fence_after();
        load_row(qrow, qi < args.Lq);
        write_base_q();
      }
    }
    // A corrected value beyond fp16's range (|x| >= 65520) makes the result
    // invalid; report it.
    if ((range & 0x80008000u) != 0u && args.dev_error != nullptr) atomicExch(args.dev_error, kDevRange);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512u);
}

template <int D, bool kRotK, int kKind>
cudaError_t launch_hilo_t(const CUtensorMap& tm_k, const CUtensorMap& tm_v, const CUtensorMap& tm_kh,
                          const CUtensorMap& tm_kl, const PrefillHiloArgs& a, cudaStream_t stream) {
  auto k = bifocal_prefill_hilo_kernel<D, kRotK, kKind>;
  // The setmaxnreg split inside the kernel assumes the launch register count.
  cudaFuncAttributes attr;
  cudaError_t e = cudaFuncGetAttributes(&attr, k);
  if (e != cudaSuccess) return e;
  if (attr.numRegs != kHLaunchRegs) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, HCfg<D>::kSmem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.Hq, a.num_mb, a.B);
  k<<<grid, kHThreads, HCfg<D>::kSmem, stream>>>(tm_k, tm_v, tm_kh, tm_kl, a);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_hilo_d(const CUtensorMap& tm_k, const CUtensorMap& tm_v, const CUtensorMap& tm_kh,
                          const CUtensorMap& tm_kl, const PrefillHiloArgs& a, bool rot_k, cudaStream_t stream) {
  if (rot_k) {
    if (a.kind != kBifocal) return cudaErrorInvalidValue;
    return launch_hilo_t<D, true, kBifocal>(tm_k, tm_v, tm_kh, tm_kl, a, stream);
  }
  switch (a.kind) {
    case kWindowBase: return launch_hilo_t<D, false, kWindowBase>(tm_k, tm_v, tm_kh, tm_kl, a, stream);
    case kCausalRemote: return launch_hilo_t<D, false, kCausalRemote>(tm_k, tm_v, tm_kh, tm_kl, a, stream);
    case kWindowRemote: return launch_hilo_t<D, false, kWindowRemote>(tm_k, tm_v, tm_kh, tm_kl, a, stream);
    default: return launch_hilo_t<D, false, kBifocal>(tm_k, tm_v, tm_kh, tm_kl, a, stream);
  }
}

}  // namespace

cudaError_t launch_prefill_hilo(const CUtensorMap& tm_k, const CUtensorMap& tm_v, const CUtensorMap& tm_kh,
                                const CUtensorMap& tm_kl, const PrefillHiloArgs& a, int D, bool rot_k,
                                cudaStream_t stream) {
  return D == 128 ? launch_hilo_d<128>(tm_k, tm_v, tm_kh, tm_kl, a, rot_k, stream)
                  : launch_hilo_d<64>(tm_k, tm_v, tm_kh, tm_kl, a, rot_k, stream);
}

}  // namespace jl
