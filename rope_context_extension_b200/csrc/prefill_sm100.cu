// Fused Dynamic Bifocal RoPE prefill for sm_100a.
//
// Causal GQA attention where a (query i, key j) pair with i - j < w0 is scored
// with the base-rotated Q and K (exact base RoPE), and every other causal pair
// with the remote-rotated rows R(p_q(i)) q and R(f(j)) k (Jet-Long review,
// "Method"; gist.science summary, "Methodologie §1").  The remote rows come
// from the correction pass in rope_rotate.cu, in fp16; local products are
// bf16 x bf16, remote ones fp16 x fp16, P V is bf16 x bf16, all fp32-accumulated.
// This is the fast, lower-precision path (one fp16 product per remote score,
// about 2^-11 relative operand error); prefill_hilo_sm100.cu is the default.
// With every pair local (G = 1 or w0 >= L) it is plain causal RoPE attention
// on the bf16 inputs, exact up to accumulation order, and serves that case for
// every precision.
//
// Instead of the pages' three FlashAttention calls merged by inclusion-exclusion,
// each 128x128 (query block, key block) tile is classified by its range of
// i - j: wholly local, wholly remote, or straddling the band edge.  A tile is
// visited once per score set it needs ("pass"): local passes read Q / K, remote
// passes read Q_rem / K_rem, and a straddling tile gets one pass of each with
// complementary masks.  Both passes feed the same online softmax, so no score
// is counted twice and nothing is subtracted.
//
// CTA = one 128-row query block of NH (1 or 2) query heads that share a KV head.
// Warp roles (384 threads):
//   warp 0      TMA producer: Q (base, later remote) and a 2-stage K / V ring
//   warp 1      tcgen05 MMA issuer; owns the TMEM allocation
//   warps 4-7   softmax for head 0 (thread = query row = TMEM lane)
//   warps 8-11  softmax for head 1
// TMEM columns: S_h at 128 h, O_h at 128 NH + D h.  P (bf16) overwrites the
// first 64 columns of S_h and is the A operand of O_h += P V from TMEM.
// Per pass the MMA order is S0(i), PV1(i-1), S1(i), PV0(i): each softmax group
// works on its S while the tensor core runs the other head's two products.
#include "jl_kernels.cuh"

namespace jl {

namespace {

constexpr int kBM = 128;  // query rows per block
constexpr int kBN = 128;  // keys per tile
constexpr int kStages = 2;
constexpr int kThreads = 384;
constexpr int kLaunchRegs = 168;  // 65536 / 384, rounded down to a multiple of 8
constexpr int kLowRegs = 104;     // warpgroup 0: TMA producer, MMA issuer
constexpr int kHighRegs = 200;    // warpgroups 1-2: softmax
static_assert(128 * kLowRegs + 256 * kHighRegs <= kThreads * kLaunchRegs, "register split exceeds the launch pool");
constexpr int kChunkBytes = 128 * 128;  // one 128-row x 128-byte swizzled slab

template <int D>
struct Cfg {
  static constexpr int kChunks = D / 64;  // 64-element (128 B) slabs per row
  static constexpr int kTileBytes = kBM * D * 2;
  static constexpr int kKSlots = 1;   // tiles per K stage
  static constexpr int kVStages = kStages;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + 2 * kTileBytes;
  static constexpr int kVOff = kKOff + kStages * kKSlots * kTileBytes;
  static constexpr int kBarOff = kVOff + kVStages * kTileBytes;
  static constexpr int kUsed = kBarOff + 256;
  // Ask for enough shared memory that only one CTA fits per SM: each CTA
  // allocates up to 512 TMEM columns.
  static constexpr int kSmem = (kUsed < 120 * 1024 ? 120 * 1024 : kUsed) + 1024;
};

// barrier slots
enum {
  kQFull = 0,
  kQEmpty = 1,
  kKFull = 2,
  kKEmpty = kKFull + kStages,
  kVFull = kKEmpty + kStages,
  kVEmpty = kVFull + kStages,
  kSFull = kVEmpty + kStages,  // 2
  kPFull = kSFull + 2,         // 4: [head][64-key half of P]
  kOFinal = kPFull + 4,
  kDrain = kOFinal + 1,
  kNumBars = kDrain + 1
};
static_assert(kNumBars * 8 <= 192, "barrier block overflow");

__device__ __forceinline__ bool drain_wait(uint32_t bar, uint32_t parity) {
  // Used only after an abort: wait (up to ~100 ms) for async work already in
  // flight so the CTA never exits while a copy or an MMA still targets it.
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > 100000000ull) return false;
  }
  return true;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    bifocal_prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_qr,
                           const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_kr,
                           const __grid_constant__ CUtensorMap tm_v, const PrefillArgs args) {
  constexpr int kKind = kBifocal;
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kBarOff + 192);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kBarOff + 196);
  auto bar = [&](int i) -> uint32_t { return smem_addr(&bars[i]); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int NH = args.nh;
  // Work order (CTAs launch in increasing linear index): the CTAs of one KV
  // head's query heads run together, heaviest query blocks first, so the CTAs
  // resident at any time stream the same K / V rows and re-read them from L2.
  const int hpk = args.r / NH;  // CTAs (query-head groups) per KV head and block
  int lin = (int)(blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z));
  const int hg = lin % hpk;
  lin /= hpk;
  const int mb = args.num_mb - 1 - lin % args.num_mb;
  lin /= args.num_mb;
  const int kvh = lin % args.Hkv;
  const int b = lin / args.Hkv;
  const int hq0 = (kvh * hpk + hg) * NH;
  const uint32_t ncols = NH == 2 ? 512u : 256u;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar(kQFull), 1);
    mbar_init(bar(kQEmpty), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(kKFull + s), 1);
      mbar_init(bar(kKEmpty + s), 1);
    }
    for (int s = 0; s < C::kVStages; ++s) {
      mbar_init(bar(kVFull + s), 1);
      mbar_init(bar(kVEmpty + s), 1);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(bar(kSFull + h), 1);
      mbar_init(bar(kPFull + 2 * h), 128);
      mbar_init(bar(kPFull + 2 * h + 1), 128);
    }
    mbar_init(bar(kOFinal), 1);
    mbar_init(bar(kDrain), 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;


  const int off = args.q_off + mb * kBM;  // position of this block's first query
  const int last = min(off + kBM - 1, args.q_off + args.Lq - 1);  // last query row of the block
  const Sched sc = make_sched<kKind>(off, last, args.w0, args.all_local != 0);
  const int npass = sc.n_loc + sc.n_rem;
  const bool q_switch = sc.n_loc > 0 && sc.n_rem > 0;
  const int w0 = args.w0;

  // Register split: the producer / MMA warpgroup needs few registers, the two
  // softmax warpgroups hold a 128-column score row each.  The launch gives
  // 384 x kLaunchRegs; 128 x kLowRegs + 256 x kHighRegs stays within it (the
  // host refuses to launch if the compiled register count differs).  Each
  // warpgroup changes its budget once, at the top of its own branch.
  if (warp < 4) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kLowRegs));
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_map(&tm_q);
      tma_prefetch_map(&tm_qr);
      tma_prefetch_map(&tm_k);
      tma_prefetch_map(&tm_kr);
      tma_prefetch_map(&tm_v);
      // Q region: one tile per head (NH heads).
      auto load_q = [&](bool remote) {
        const CUtensorMap* m = remote ? &tm_qr : &tm_q;
        mbar_arrive_expect_tx(bar(kQFull), (uint32_t)(NH * C::kTileBytes));
        for (int hh = 0; hh < NH; ++hh)
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_4d(sbase + C::kQOff + hh * C::kTileBytes + c * kChunkBytes, m, bar(kQFull), c * 64,
                        hq0 + hh, mb * kBM, b);
      };
      // A query block with no pass (a window call with w0 = 0) loads nothing.
      if (npass > 0) load_q(pass_remote_ops<kKind>(sc, 0));
      int q_loads = npass > 0 ? 1 : 0;
      int k_last = -1, v_last = -1;  // last passes whose K / V copies were issued
      bool ok = true;
      for (int p = 0; p < npass; ++p) {
        const int s = p % kStages;
        const uint32_t ph = (uint32_t)(p / kStages) & 1u;
        const int sv = p % C::kVStages;
        const uint32_t phv = (uint32_t)(p / C::kVStages) & 1u;
        const bool remote = pass_remote_ops<kKind>(sc, p);
        const int nb = pass_block(sc, p);
        if (q_switch && p == sc.n_loc) {
          if (!(ok = mbar_wait(bar(kQEmpty), 0, abort_flag, args.dev_error))) break;
          load_q(true);
          ++q_loads;
        }
        if (!(ok = mbar_wait(bar(kKEmpty + s), ph ^ 1u, abort_flag, args.dev_error))) break;
        const uint32_t kdst = sbase + C::kKOff + s * C::kKSlots * C::kTileBytes;
        mbar_arrive_expect_tx(bar(kKFull + s), (uint32_t)C::kTileBytes);
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_4d(kdst + c * kChunkBytes, remote ? &tm_kr : &tm_k, bar(kKFull + s), c * 64, kvh, nb * kBN, b);
        k_last = p;
        if (!(ok = mbar_wait(bar(kVEmpty + sv), phv ^ 1u, abort_flag, args.dev_error))) break;
        mbar_arrive_expect_tx(bar(kVFull + sv), (uint32_t)C::kTileBytes);
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_4d(sbase + C::kVOff + sv * C::kTileBytes + c * kChunkBytes, &tm_v, bar(kVFull + sv), c * 64,
                      kvh, nb * kBN, b);
        v_last = p;
      }
      if (!ok) {
        // Let every copy already issued land before the CTA can exit.
        if (q_loads > 0) drain_wait(bar(kQFull), (uint32_t)(q_loads - 1) & 1u);
        for (int p = max(0, k_last - kStages + 1); p <= k_last; ++p)
          drain_wait(bar(kKFull + p % kStages), (uint32_t)(p / kStages) & 1u);
        for (int p = max(0, v_last - C::kVStages + 1); p <= v_last; ++p)
          drain_wait(bar(kVFull + p % C::kVStages), (uint32_t)(p / C::kVStages) & 1u);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id_s_loc = make_idesc_16bit(kBM, kBN, false, false);  // bf16 Q K
      const uint32_t id_s_rem = make_idesc_16bit(kBM, kBN, false, true);   // fp16 Q_rem K_rem
      const uint32_t id_pv = make_idesc_16bit(kBM, D, true, false);        // bf16 P V
      bool ok = npass == 0 || mbar_wait(bar(kQFull), 0, abort_flag, args.dev_error);
      auto s_col = [&](int h) -> uint32_t { return (uint32_t)(h * 128); };
      auto o_col = [&](int h) -> uint32_t { return (uint32_t)(NH * 128 + h * D); };

      // Shared-memory matrix descriptors, built once (Q of each head, K and V of
      // each stage); a k-step adds a compile-time offset (bytes >> 4).
      const uint64_t dq0 = make_sdesc_sw128(sbase + C::kQOff, 16, 1024);
      const uint64_t dq1 = make_sdesc_sw128(sbase + C::kQOff + C::kTileBytes, 16, 1024);
      const uint64_t dk0 = make_sdesc_sw128(sbase + C::kKOff, 16, 1024);
      const uint64_t dk1 = make_sdesc_sw128(sbase + C::kKOff + C::kKSlots * C::kTileBytes, 16, 1024);
      const uint64_t dv0 = make_sdesc_sw128(sbase + C::kVOff, kChunkBytes, 1024);
      const uint64_t dv1 = make_sdesc_sw128(sbase + C::kVOff + C::kTileBytes, kChunkBytes, 1024);
      auto kstep_off = [](int ks) -> uint64_t {
        return (uint64_t)(((ks >> 2) * kChunkBytes + (ks & 3) * 32) >> 4);
      };
      auto issue_s = [&](int h, int p, int s) -> bool {  // s = p % 2
        const uint32_t ph = (uint32_t)(p >> 1) & 1u;
        if (h == 0) {
          if (q_switch && p == sc.n_loc && !mbar_wait(bar(kQFull), 1, abort_flag, args.dev_error)) return false;
          if (!mbar_wait(bar(kKFull + s), ph, abort_flag, args.dev_error)) return false;
          tc_fence_after();
        }
        const uint64_t dq = h == 0 ? dq0 : dq1;
        const uint64_t dk = s == 0 ? dk0 : dk1;
        const bool remote = pass_remote_ops<kKind>(sc, p);
        const uint32_t id_s = remote ? id_s_rem : id_s_loc;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          mma_ss(tmem + s_col(h), dq + kstep_off(ks), dk + kstep_off(ks), id_s, ks > 0 ? 1u : 0u);
        tc_commit(bar(kSFull + h));
        if (h == NH - 1) {
          tc_commit(bar(kKEmpty + s));
          if (q_switch && p == sc.n_loc - 1) tc_commit(bar(kQEmpty));
        }
        return true;
      };
      // O_h += P V in two 64-key halves, each issued as soon as the softmax
      // has written that half of P, so the first half's product runs while
      // the second half's exponentials are taken.
      auto issue_pv = [&](int h, int p, int s) -> bool {  // s = p % 2
        const uint32_t ph = (uint32_t)(p >> 1) & 1u;
        if (h == 0 && !mbar_wait(bar(kVFull + s), ph, abort_flag, args.dev_error)) return false;
        const uint64_t dv = s == 0 ? dv0 : dv1;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          if (!mbar_wait(bar(kPFull + 2 * h + half), (uint32_t)p & 1u, abort_flag, args.dev_error)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kBN / 32; ++kk) {
            const int ks = half * (kBN / 32) + kk;
            // V tile is MN-major for this product: 64-dim slabs kChunkBytes apart
            // (leading offset), 8-key groups 1024 B apart (stride offset).
            mma_ts(tmem + o_col(h), tmem + s_col(h) + (uint32_t)(ks * 8),
                   dv + (uint64_t)((ks * 2048) >> 4), id_pv,
                   (p > 0 || ks > 0) ? 1u : 0u);
          }
        }
        if (h == NH - 1) tc_commit(bar(kVEmpty + s));
        return true;
      };

      if (ok && npass > 0) {
        if (NH == 2) {
          // unrolled by two passes so that each copy's stage parity is a constant
          auto pass2 = [&](int p, int s) -> bool {
            return issue_s(0, p, s) && issue_pv(1, p - 1, s ^ 1) && issue_s(1, p, s) && issue_pv(0, p, s);
          };
          ok = issue_s(0, 0, 0) && issue_s(1, 0, 0) && issue_pv(0, 0, 0);
          int p = 1;
          for (; p + 1 < npass && ok; p += 2) ok = pass2(p, 1) && pass2(p + 1, 0);
          if (ok && p < npass) ok = pass2(p, 1);
          if (ok) ok = issue_pv(1, npass - 1, (npass - 1) & 1);
        } else {
          auto pass1 = [&](int p, int s) -> bool { return issue_s(0, p, s) && issue_pv(0, p, s); };
          int p = 0;
          for (; p + 1 < npass && ok; p += 2) ok = pass1(p, 0) && pass1(p + 1, 1);
          if (ok && p < npass) ok = pass1(p, 0);
        }
      }
      // Every product issued must have completed before TMEM is released.
      if (ok) {
        tc_commit(bar(kOFinal));
        drain_wait(bar(kOFinal), 0);
      } else {
        tc_commit(bar(kDrain));
        drain_wait(bar(kDrain), 0);
      }
    }
  }
  } else {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kHighRegs));
  if (((warp - 4) >> 2) < NH) {
    // ------------------------------------------------------------ softmax
    const int h = (warp - 4) >> 2;
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const int hq = hq0 + h;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t s_addr = tmem + lane_off + (uint32_t)(h * 128);
    const uint32_t o_addr = tmem + lane_off + (uint32_t)(NH * 128 + h * D);
    const float sl2 = args.scale_log2;
    float m_used = -INFINITY;
    float l_sum = 0.f;
    bool ok = true;

    for (int p = 0; p < npass; ++p) {
      ok = mbar_wait(bar(kSFull + h), (uint32_t)p & 1u, abort_flag, args.dev_error);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const int mkind = pass_mask_kind<kKind>(sc, p);
      const int dd0 = off - 128 * pass_block(sc, p);  // i - j at row 0, column 0

      // S in two 64-column halves: the first half's mask and partial row max
      // run while the second half's load is in flight (tcgen05.wait::ld
      // waits for every outstanding load, so the second pair is issued after
      // the first wait).
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
      // Row max over four independent chains of three-input maxima (the scale
      // is positive, so the max of the raw scores scales to the max of the
      // scaled ones).
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

      // O_h must be rescaled before either half of this pass's P V; in the
      // (rare) passes that need it, both halves of P are released after it.
      const bool resc = __any_sync(0xffffffffu, rescale_o) && p > 0;
      // p = 2^(s * scale * log2 e - m): one packed FMA per pair, the row sum in
      // two packed accumulators.
      const uint64_t sc2 = f2_pack(sl2, sl2), nm2 = f2_pack(-msub, -msub);
      uint64_t acc[2] = {0ull, 0ull};
      // One pair of P: 2^(s * scale * log2 e - m) for columns 64 half + 2k, +1.
      auto pair_exp = [&](int half, int k) -> uint32_t {
        const uint64_t ev = f2_fma(f2_pack(x[half * 64 + 2 * k], x[half * 64 + 2 * k + 1]), sc2, nm2);
        float e0, e1;
        f2_unpack(ev, e0, e1);
        const float p0 = ex2_approx(e0), p1 = ex2_approx(e1);  // on the MUFU
        acc[k & 1] = f2_add(acc[k & 1], f2_pack(p0, p1));
        return pack_bf16x2(p0, p1);
      };
      // P half 0 is stored, then half 1's first eight pairs are taken while
      // that store lands (6-8 measured best); half 0 is released after them,
      // half 1 at the end.  In a pass that rescales O both are released after
      // the rescale.
      {
        uint32_t pk[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) pk[k] = pair_exp(0, k);
        tmem_st32(s_addr, pk);
      }
      {
        uint32_t pk[32];
#pragma unroll
        for (int k = 0; k < 8; ++k) pk[k] = pair_exp(1, k);
        if (!resc) {
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(bar(kPFull + 2 * h));
        }
#pragma unroll
        for (int k = 8; k < 32; ++k) pk[k] = pair_exp(1, k);
        tmem_st32(s_addr + 32, pk);
        if (resc) {
          // O_h(p-1) is final here: its product was issued before S_h(p).
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
        if (resc) mbar_arrive(bar(kPFull + 2 * h));
        mbar_arrive(bar(kPFull + 2 * h + 1));
      }
      {
        float a0, a1;
        f2_unpack(f2_add(acc[0], acc[1]), a0, a1);
        l_sum += a0 + a1;
      }
    }

    if (ok) {
      ok = mbar_wait(bar(kOFinal), 0, abort_flag, args.dev_error);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      const int i = mb * kBM + row;  // row of this chunk's Q / O / LSE
      const float inv = (l_sum > 0.f && npass > 0) ? 1.f / l_sum : 0.f;
      __nv_bfloat16* orow = args.o + (((size_t)b * args.Lq + i) * args.Hq + hq) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ov[32];
        tmem_ld32(o_addr + c * 32, ov);  // (never written when npass == 0; inv is 0 then)
        tmem_ld_wait(ov);
        uint32_t w[16];
#pragma unroll
        for (int k = 0; k < 16; ++k)
          w[k] = npass > 0 ? pack_bf16x2(__uint_as_float(ov[2 * k]) * inv, __uint_as_float(ov[2 * k + 1]) * inv)
                           : 0u;  // no key at all: O = 0, LSE = -inf
        if (i < args.Lq) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int k = 0; k < 4; ++k) dst[k] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
        }
      }
      if (args.lse != nullptr && i < args.Lq) {
        const float m = (m_used == -INFINITY) ? 0.f : m_used;
        args.lse[((size_t)b * args.Hq + hq) * args.Lq + i] =
            l_sum > 0.f ? (m + __log2f(l_sum)) * 0.69314718055994531f : -INFINITY;
      }
    }
  }

  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, ncols);
}

template <int D>
cudaError_t launch_prefill_t(const CUtensorMap& tm_q, const CUtensorMap& tm_qr, const CUtensorMap& tm_k,
                             const CUtensorMap& tm_kr, const CUtensorMap& tm_v, const PrefillArgs& a,
                             cudaStream_t stream) {
  auto k = bifocal_prefill_kernel<D>;
  // The setmaxnreg split inside the kernel assumes the launch register count.
  cudaFuncAttributes attr;
  cudaError_t e = cudaFuncGetAttributes(&attr, k);
  if (e != cudaSuccess) return e;
  if (attr.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<D>::kSmem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.Hq / a.nh, a.num_mb, a.B);
  k<<<grid, kThreads, Cfg<D>::kSmem, stream>>>(tm_q, tm_qr, tm_k, tm_kr, tm_v, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const CUtensorMap& tm_q, const CUtensorMap& tm_qr, const CUtensorMap& tm_k,
                           const CUtensorMap& tm_kr, const CUtensorMap& tm_v, const PrefillArgs& a, int D,
                           cudaStream_t stream) {
  return D == 128 ? launch_prefill_t<128>(tm_q, tm_qr, tm_k, tm_kr, tm_v, a, stream)
                  : launch_prefill_t<64>(tm_q, tm_qr, tm_k, tm_kr, tm_v, a, stream);
}

}  // namespace jl
