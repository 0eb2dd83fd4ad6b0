// fa_fwd.cuh -- forward pass of exact attention on sm_100a.
//
// What it computes (hysenlabs FlashAttention API page, outputs section;
// Qiita Flash Attention tutorial, sections 4.2-4.3; abeam.tech FlashAttention
// summary, "computing softmax blockwise correctly"): for each query row,
//   O = sum_j softmax_j(scale * q . k_j) v_j,   LSE = ln sum_j exp(scale * q . k_j)
// by walking the visible key/value tiles once with a running row max m and a
// running sum l; when m grows, l and the partial O are rescaled by
// exp(m_old - m_new), and O is divided by l once at the end.  S and P live in
// tensor memory and never reach HBM.
//
// Design on B200 (one CTA per SM, warp-specialised):
//   * TMA warp      : Q tile(s) once, then K_j / V_j through a KST-deep ring.
//   * MMA warp      : one thread issues tcgen05.mma: S = Q K_j^T (both operands
//                     from shared memory, fp32 into TMEM) and O += P V_j (P
//                     read straight from TMEM, V from shared memory).
//   * softmax warps : one warpgroup per 128-row Q tile; thread r owns TMEM
//                     lane r, i.e. a whole score row, so the row max and row
//                     sum need no shuffles.  exp2 with the scale folded into
//                     one FMA; P is written back into TMEM as bf16 over its S.
// With two Q tiles per CTA (d <= 128) the tensor core computes one tile's
// S/PV while the other tile's softmax runs.  For d = 256 (one Q tile) the two
// S slots alternate between consecutive key tiles instead.
//
// In tiles without masked keys, NPOLY of every 8 pairs of exponentials are
// computed on the FMA pipe (exp2_poly_pair) rather than the MUFU unit, which
// would otherwise bound the softmax; tiles with masked keys use MUFU ex2 only,
// which returns exact zeros for -inf.
//
// The running max is only moved (and O rescaled) when the tile max exceeds
// it by more than 2^8 in the exp2 domain; otherwise the old reference is kept.
// Every P stays <= 2^8, the result is the same exact softmax (the reference
// cancels in O / l), and most O rescales are skipped.
#pragma once
#include "fa_common.cuh"

namespace fa {

struct FwdParams {
  int B, Nq, Nk, Hq, Hkv, group;  // group = Hq / Hkv
  float scale_log2;               // softmax scale * log2(e)
  MaskSpec mask;
  int n_qgroups;                  // CTAs along the query axis
  int head_chunk;                 // heads per scheduling chunk (see ChunkedOrder)
  float* lse;                     // [B, Hq, Nq]; packed sequences: [Hq, total_q]
  // packed sequences (null when dense): sequence b holds query rows
  // [cu_q[b], cu_q[b+1]) and key rows [cu_k[b], cu_k[b+1]) of tensors seen
  // as one batch; Nq / Nk are then the longest sequence's lengths
  const int* cu_q;
  const int* cu_k;
  int total_q;
  uint16_t* o;               // O, for the plain stores of a packed sequence's last tile
  // block-sparse attention (BS kernels): a byte per 128 x 128 (query block,
  // key block) of batch b, query head h at bmask + b * bm_sb + h * bm_sh,
  // rows of bm_cols key blocks; zero = the block is skipped
  const uint8_t* bmask;
  long long bm_sb, bm_sh;
  int bm_cols;
  unsigned long long wait_limit_ns;
  // test only (fa_test_withhold_next_load): the producer of CTA 0 issues no
  // key/value load after its first ring stages, so the MMA thread's bounded
  // wait for the next one runs out; 0 in every ordinary launch
  int test_withhold;
};

template <int D_, int NQT_, int BN_, int KST_, int NPOLY_ = 2, bool SPLITP_ = false>
struct FwdCfg {
  static constexpr bool F16 = false;  // elements are bf16 (AsF16<> flips it to fp16)
  static constexpr int D = D_, NQT = NQT_, BN = BN_, KST = KST_;
  // NQT == 2 only: P reaches the tensor core in two key halves, so the first
  // half's PV overlaps the softmax of the second (one more wait point per
  // tile in the MMA thread; pays off when the PV is short, i.e. small d)
  static constexpr bool SPLITP = SPLITP_ && NQT_ == 2;
  // of every 8 score pairs of an unmasked tile, NPOLY take exp2 on the FMA
  // pipe (exp2_poly_pair), the rest on the MUFU unit
  static constexpr int NPOLY = NPOLY_;
  static constexpr int BM = 128;
  static constexpr int NCHUNK = D / 64;      // 128-byte swizzle chunks across d
  static constexpr int QCHUNK = BM * 128;    // bytes of one 64-column chunk of a Q tile
  static constexpr int KCHUNK = BN * 128;
  static constexpr int QTILE = NCHUNK * QCHUNK;
  static constexpr int KTILE = NCHUNK * KCHUNK;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + NQT * QTILE;
  static constexpr int OFF_V = OFF_K + KST * KTILE;
  static constexpr int OFF_BAR = OFF_V + KST * KTILE;
  // bar_q, k_full[KST] (with NQT == 2 it signals K and V of the tile together),
  // k_empty[KST], v_full[KST], v_empty[KST], s_full[2], p_full[4], o_done[2], drain
  // (p_full: NQT == 2, [2t + half] for the key halves of Q tile t, [2t]
  // alone without SPLITP; NQT == 1, [slot])
  static constexpr int NBAR = 1 + 4 * KST + 8 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + slack to align the base to 1 KiB
  // softmax warpgroups first, then one producer warpgroup (TMA warp, MMA
  // warp, two idle warps) so registers can move to the softmax warpgroups
  static constexpr int NWARPS = 4 * NQT + 4;
  static constexpr int NTHREADS = 32 * NWARPS;
  static constexpr int TMA_WARP = 4 * NQT;
  static constexpr int MMA_WARP = 4 * NQT + 1;
  // registers per thread: at launch (65536 / NTHREADS, rounded down to 8),
  // producer share, softmax share; the shares add up to the launch total.
  // The MMA thread keeps only base descriptors live (FwdIssueS / FwdIssuePV),
  // so the producer warpgroup gets by with 40 and the softmax warpgroups get
  // 232 (two Q tiles): with more registers their exp / pack stream schedules
  // with more instruction-level parallelism.
  static constexpr int REG_LAUNCH = (65536 / NTHREADS) / 8 * 8;
  static constexpr int REG_PRODUCER = 40;
  static constexpr int REG_MATH =
      ((NTHREADS * REG_LAUNCH - 128 * REG_PRODUCER) / (128 * NQT)) / 8 * 8 > 248
          ? 248
          : ((NTHREADS * REG_LAUNCH - 128 * REG_PRODUCER) / (128 * NQT)) / 8 * 8;
  static_assert(NQT * 128 * REG_MATH + 128 * REG_PRODUCER <= NTHREADS * REG_LAUNCH, "register split");
  static constexpr int COL_S = 0;        // S slot s: columns [s*BN, s*BN+BN); its P: first BN/2
  static constexpr int COL_O = 2 * BN;   // O of Q tile t: columns [COL_O + t*D, +D)
  static constexpr int TMEM_USED = 2 * BN + NQT * D;
  static constexpr int TMEM_COLS = TMEM_USED <= 128 ? 128 : TMEM_USED <= 256 ? 256 : 512;
  static_assert(TMEM_USED <= 512, "TMEM budget");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(D % 64 == 0 && BN % 64 == 0, "tile shapes");
  static_assert(NQT == 1 || NQT == 2, "one or two Q tiles per CTA");
};

// Unrolled MMA sequences with compile-time descriptor offsets (mma_ss_at /
// mma_ts_at): S = Q K^T over d in steps of 16, and O (+)= P V over the key
// tile in steps of 16.
template <class C, int KK = 0>
struct FwdIssueS {
  static __device__ __forceinline__ void run(uint32_t d_tmem, uint64_t qa, uint64_t kb, uint32_t id) {
    if constexpr (KK < C::D / 16) {
      constexpr uint32_t oq = ((KK >> 2) * C::QCHUNK + (KK & 3) * 32) >> 4;
      constexpr uint32_t ok = ((KK >> 2) * C::KCHUNK + (KK & 3) * 32) >> 4;
      mma_ss_at<oq, ok>(d_tmem, qa, kb, id, KK > 0 ? 1u : 0u);
      FwdIssueS<C, KK + 1>::run(d_tmem, qa, kb, id);
    }
  }
};
template <class C, int KK = 0, int KEND = C::BN / 16>
struct FwdIssuePV {
  static __device__ __forceinline__ void run(uint32_t d_tmem, uint32_t a_tmem, uint64_t vb, uint32_t id,
                                             bool acc) {
    if constexpr (KK < KEND) {
      mma_ts_at<KK * 8, KK * 128>(d_tmem, a_tmem, vb, id, (acc || KK > 0) ? 1u : 0u);
      FwdIssuePV<C, KK + 1, KEND>::run(d_tmem, a_tmem, vb, id, acc);
    }
  }
};

// P for score columns [C0, C1) of one row: 2^(s * scale_log2 - mb) packed to
// bf16 pairs into pk[C0/2 ..], row sums accumulated into two fp32 pairs.
// EDGE: the tile has masked (-inf) scores, so MUFU ex2 only (exact zeros);
// otherwise NPOLY of every 8 pairs use exp2_poly_pair.
template <class C, int C0, int C1, bool EDGE>
__device__ __forceinline__ void fwd_exp_cols(const float* sc, uint64_t scale2, uint64_t shift2,
                                             uint32_t* pk, uint64_t& acc0, uint64_t& acc1) {
#pragma unroll
  for (int c = C0; c < C1; c += 2) {
    const uint64_t x2 = f2_fma(f2_pack(sc[c], sc[c + 1]), scale2, shift2);
    float p0, p1;
    if (!EDGE && (c / 2) % 8 < C::NPOLY) {
      exp2_poly_pair(x2, p0, p1);
    } else {
      float x0, x1;
      f2_unpack(x2, x0, x1);
      p0 = ex2_approx(x0);
      p1 = ex2_approx(x1);
    }
    pk[c / 2] = pack2<C::F16>(p0, p1);
    if ((c / 2) & 1)
      acc1 = f2_add(acc1, f2_pack(p0, p1));
    else
      acc0 = f2_add(acc0, f2_pack(p0, p1));
  }
}

// VL: packed variable-length sequences (FwdParams::cu_q / cu_k); BS: a block
// mask (FwdParams::bmask).  The dense instantiation compiles without either.
template <class C, bool VL = false, bool BS = false>
__global__ void __launch_bounds__(C::NTHREADS, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                  const FwdParams p) {
  constexpr int D = C::D, NQT = C::NQT, BN = C::BN, KST = C::KST, BM = C::BM;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* bar_q = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + KST;
  uint64_t* v_full = k_empty + KST;
  uint64_t* v_empty = v_full + KST;
  uint64_t* s_full = v_empty + KST;  // [2]
  uint64_t* p_full = s_full + 2;     // [4]
  uint64_t* o_done = p_full + 4;     // [2]
  uint64_t* bar_drain = o_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  const uint32_t sQ = sbase + C::OFF_Q, sK = sbase + C::OFF_K, sV = sbase + C::OFF_V;

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  // ---- work unit: (batch b, head h, query group g), heaviest (latest, for
  // causal) query groups first within L2-sized chunks of heads
  const ChunkedOrder order(blockIdx.x, p.B * p.Hq, p.n_qgroups, p.head_chunk);
  const int bh = order.head;
  const int g = p.n_qgroups - 1 - order.rank;
  const int h = bh % p.Hq, hk = h / p.group;
  const int r0 = g * NQT * BM;
  // dense: batch b of the tensors; packed: sequence b at row offsets
  // q_off / k_off of one-batch tensors (tb = 0), its own lengths and masks
  int b = bh / p.Hq, q_off = 0, k_off = 0;
  MaskSpec mask = p.mask;
  if constexpr (VL) {
    q_off = __ldg(p.cu_q + b);
    k_off = __ldg(p.cu_k + b);
    mask.Nq = __ldg(p.cu_q + b + 1) - q_off;
    mask.Nk = __ldg(p.cu_k + b + 1) - k_off;
    if (r0 >= mask.Nq) return;  // this sequence has no query group g
  }
  const int nq = mask.Nq;
  const int tb = VL ? 0 : b;
  const int r_last = min(nq - 1, r0 + NQT * BM - 1);
  const int key_lo = mask.lo(r0), key_hi = mask.hi(r_last);
  const int j_begin = key_lo / BN;
  int n_kv = (key_hi >= key_lo) ? (key_hi / BN - j_begin + 1) : 0;

  // Block-sparse: the TMA warp lists the key tiles of that range whose mask
  // block is set for either Q tile (bit 30 + t: set for Q tile t), compacted
  // with warp ballots, before the block-wide sync; every role then walks the
  // list instead of the range.
  uint32_t* tile_list = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC + 16);
  volatile int* list_count = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);
  if constexpr (BS) {
    if (warp == C::TMA_WARP) {
      const uint8_t* m0 = p.bmask + b * p.bm_sb + h * p.bm_sh + static_cast<long long>(r0 / 128) * p.bm_cols;
      const bool two = NQT == 2 && r0 + BM < nq;
      int cnt = 0;
      for (int c0 = 0; c0 < n_kv; c0 += 32) {
        const int it = c0 + lane;
        uint32_t a0 = 0, a1 = 0;
        if (it < n_kv) {
          const int blk = ((j_begin + it) * BN) / 128;
          a0 = __ldg(m0 + blk) != 0;
          if (two) a1 = __ldg(m0 + p.bm_cols + blk) != 0;
        }
        const unsigned bal = __ballot_sync(0xffffffffu, (a0 | a1) != 0);
        if (a0 | a1)
          tile_list[cnt + __popc(bal & ((1u << lane) - 1u))] =
              static_cast<uint32_t>(j_begin + it) | (a0 << 30) | (a1 << 31);
        cnt += __popc(bal);
      }
      n_kv = cnt;
      if (lane == 0) *list_count = cnt;
      __syncwarp();
    }
  }
  auto tile_of = [&](int it) {
    if constexpr (BS)
      return static_cast<int>(tile_list[it] & 0x3fffffffu);
    else
      return j_begin + it;
  };

  // Copies of key tile `it` into ring stage it % KST (K and V on one barrier
  // with two Q tiles, on their own barriers with one)
  auto load_k = [&](int it) {
    const int s = it % KST, krow = k_off + tile_of(it) * BN;
    uint64_t* bar = &k_full[s];
    mbar_expect_tx(bar, (NQT == 2 ? 2 : 1) * C::KTILE);
    for (int c = 0; c < C::NCHUNK; ++c) {
      tma_load_4d(sK + s * C::KTILE + c * C::KCHUNK, &tm_k, bar, c * 64, hk, krow, tb);
      if (NQT == 2) tma_load_4d(sV + s * C::KTILE + c * C::KCHUNK, &tm_v, bar, c * 64, hk, krow, tb);
    }
  };
  auto load_v = [&](int it) {  // NQT == 1 only
    const int s = it % KST, krow = k_off + tile_of(it) * BN;
    mbar_expect_tx(&v_full[s], C::KTILE);
    for (int c = 0; c < C::NCHUNK; ++c)
      tma_load_4d(sV + s * C::KTILE + c * C::KCHUNK, &tm_v, &v_full[s], c * 64, hk, krow, tb);
  };
  // The TMA thread sets up the barriers and issues Q and the first KST key
  // tiles (no stage to wait for yet) before the block-wide sync, so the
  // copies overlap the TMEM allocation and the sync.
  const int n_pre = min(n_kv, KST);
  if (warp == C::TMA_WARP && lane == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < KST; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&o_done[s], 1);
    }
    for (int i = 0; i < 4; ++i) mbar_init(&p_full[i], BM);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    if (n_kv > 0) {
      mbar_expect_tx(bar_q, NQT * C::QTILE);
      for (int t = 0; t < NQT; ++t)
        for (int c = 0; c < C::NCHUNK; ++c)
          tma_load_4d(sQ + t * C::QTILE + c * C::QCHUNK, &tm_q, bar_q, c * 64, h, q_off + r0 + t * BM, tb);
      for (int it = 0; it < n_pre; ++it) {
        load_k(it);
        if (NQT == 1) load_v(it);
      }
    }
    tma_prefetch_desc(&tm_o);
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(smem_addr(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if constexpr (BS) n_kv = *list_count;

  if (warp == C::TMA_WARP) {
    // ------------------------------------------------------------ producer
    setmaxnreg_dec<C::REG_PRODUCER>();
    if (lane == 0 && n_kv > 0) {
      // Q and key tiles 0 .. n_pre-1 were issued before the block-wide sync
      int nk = n_pre, nv = NQT == 1 ? n_pre : 0;
      for (int it = n_pre; it < n_kv; ++it) {
        if (p.test_withhold && blockIdx.x == 0) break;  // test only: key tile `it` is never loaded
        const int s = it % KST, use = it / KST;
        // the stage is free once the last MMA reading the tile held there
        // before has completed (NQT == 2: K_j and V_j share the stage)
        if (!mbar_wait(&k_empty[s], (use - 1) & 1, abort_flag, &g_status, p.wait_limit_ns)) break;
        load_k(it);
        ++nk;
        if constexpr (NQT == 1) {
          if (!mbar_wait(&v_empty[s], (use - 1) & 1, abort_flag, &g_status, p.wait_limit_ns)) break;
          load_v(it);
          ++nv;
        }
      }
      // every copy issued must land before the CTA may exit
      mbar_drain(bar_q, 0, p.wait_limit_ns);
      for (int s = 0; s < KST; ++s) {
        if (nk > s) mbar_drain(&k_full[s], ((nk - 1 - s) / KST) & 1, p.wait_limit_ns);
        if (nv > s) mbar_drain(&v_full[s], ((nv - 1 - s) / KST) & 1, p.wait_limit_ns);
      }
    }
  } else if (warp == C::MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    setmaxnreg_dec<C::REG_PRODUCER>();
    if (lane == 0 && n_kv > 0) {
      constexpr uint32_t ID_QK = idesc_kind_f16<C::F16>(128, BN, false, false);
      constexpr uint32_t ID_PV = idesc_kind_f16<C::F16>(128, D, false, true);
      // Descriptors are built once; every MMA only adds a compile-time offset
      // (in 16-byte units) to the start-address field.  The issuing thread
      // must stay ahead of the tensor core, so it does as little as possible
      // between MMAs and checks barriers at as few points as it can.
      const uint64_t dq0 = sdesc_sw128(sQ, 16, 1024);
      const uint64_t dk0 = sdesc_sw128(sK, 16, 1024);
      const uint64_t dv0 = sdesc_sw128(sV, C::KCHUNK, 1024);
      auto wait = [&](uint64_t* bar, uint32_t par) {
        const bool ok = mbar_wait(bar, par, abort_flag, &g_status, p.wait_limit_ns);
        tc_fence_after();
        return ok;
      };
      // S[slot] = Q_t K_s^T
      auto issue_s = [&](int slot, int t, int s) {
        FwdIssueS<C>::run(tmem + C::COL_S + slot * BN, dq0 + static_cast<uint64_t>((t * C::QTILE) >> 4),
                          dk0 + static_cast<uint64_t>((s * C::KTILE) >> 4), ID_QK);
      };
      // O_t (+)= P[slot] V_s, over the whole key tile or one half of it
      auto issue_pv = [&](int slot, int t, int s, bool acc) {
        FwdIssuePV<C>::run(tmem + C::COL_O + t * D, tmem + C::COL_S + slot * BN,
                           dv0 + static_cast<uint64_t>((s * C::KTILE) >> 4), ID_PV, acc);
      };
      auto issue_pv_lo = [&](int slot, int t, int s, bool acc) {
        FwdIssuePV<C, 0, BN / 32>::run(tmem + C::COL_O + t * D, tmem + C::COL_S + slot * BN,
                                       dv0 + static_cast<uint64_t>((s * C::KTILE) >> 4), ID_PV, acc);
      };
      auto issue_pv_hi = [&](int slot, int t, int s) {
        FwdIssuePV<C, BN / 32, BN / 16>::run(tmem + C::COL_O + t * D, tmem + C::COL_S + slot * BN,
                                             dv0 + static_cast<uint64_t>((s * C::KTILE) >> 4), ID_PV, true);
      };
      bool ok = wait(bar_q, 0) && wait(&k_full[0], 0);
      if (ok) {
        if constexpr (NQT == 2) {
          // per key tile j: PV_0(j), S_0(j+1), PV_1(j), S_1(j+1); the two Q
          // tiles' softmax warpgroups alternate with the tensor core.  With
          // SPLITP, P arrives in two key halves, and the first half's PV
          // runs while the softmax still computes the second.
          issue_s(0, 0, 0);
          tc_commit(&s_full[0]);
          issue_s(1, 1, 0);
          tc_commit(&s_full[1]);
          for (int it = 0; it < n_kv && ok; ++it) {
            const int s = it % KST, s1 = (it + 1) % KST;
            const bool more = it + 1 < n_kv;
            const uint32_t par = it & 1;
            if (!(ok = wait(&p_full[0], par))) break;
            if (more && !(ok = wait(&k_full[s1], ((it + 1) / KST) & 1))) break;
            if constexpr (C::SPLITP) {
              issue_pv_lo(0, 0, s, it > 0);
              if (!(ok = wait(&p_full[1], par))) break;
              issue_pv_hi(0, 0, s);
            } else {
              issue_pv(0, 0, s, it > 0);
            }
            if (more) {
              issue_s(0, 0, s1);
              tc_commit(&s_full[0]);
            } else {
              tc_commit(&o_done[0]);  // tile 0's epilogue may start
            }
            if (!(ok = wait(&p_full[2], par))) break;
            if constexpr (C::SPLITP) {
              issue_pv_lo(1, 1, s, it > 0);
              if (!(ok = wait(&p_full[3], par))) break;
              issue_pv_hi(1, 1, s);
            } else {
              issue_pv(1, 1, s, it > 0);
            }
            tc_commit(&k_empty[s]);  // K_j and V_j are no longer read
            if (more) {
              issue_s(1, 1, s1);
              tc_commit(&s_full[1]);
            } else {
              tc_commit(&o_done[1]);
            }
          }
        } else {
          // one Q tile: S slots alternate between consecutive key tiles
          issue_s(0, 0, 0);
          tc_commit(&s_full[0]);
          tc_commit(&k_empty[0]);
          if (n_kv > 1) {
            if ((ok = wait(&k_full[1 % KST], (1 / KST) & 1))) {
              issue_s(1, 0, 1 % KST);
              tc_commit(&s_full[1]);
              tc_commit(&k_empty[1 % KST]);
            }
          }
          for (int it = 0; it < n_kv && ok; ++it) {
            const int slot = it & 1, s = it % KST;
            if (!(ok = wait(&p_full[slot], (it >> 1) & 1))) break;
            if (!(ok = wait(&v_full[s], (it / KST) & 1))) break;
            issue_pv(slot, 0, s, it > 0);
            tc_commit(&o_done[0]);
            tc_commit(&v_empty[s]);
            if (it + 2 < n_kv) {
              const int s2 = (it + 2) % KST;
              if (!(ok = wait(&k_full[s2], ((it + 2) / KST) & 1))) break;
              issue_s(slot, 0, s2);
              tc_commit(&s_full[slot]);
              tc_commit(&k_empty[s2]);
            }
          }
        }
      }
    }
    if (lane == 0) {  // all MMAs this thread issued are complete before TMEM is released
      tc_commit(bar_drain);
      mbar_drain(bar_drain, 0, p.wait_limit_ns);
    }
    __syncwarp();
  } else if (warp < C::TMA_WARP) {
    // ------------------------------------------------------------ softmax
    setmaxnreg_inc<C::REG_MATH>();
    const int t = warp / 4;          // Q tile of this warpgroup
    const int r = threadIdx.x % BM;  // row within the tile == TMEM lane
    const int row = r0 + t * BM + r;
    const int lo = mask.lo(row), hi = mask.hi(row);
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp % 4) * 32) << 16);
    const float sl2 = p.scale_log2;
    float m_ref = -INFINITY;  // reference max, exp2 domain (scale folded in)
    float l = 0.f;
    bool ok = true;
    for (int it = 0; it < n_kv; ++it) {
      const int slot = (NQT == 2) ? t : (it & 1);
      const uint32_t par = (NQT == 2) ? (it & 1) : ((it >> 1) & 1);
      ok = mbar_wait(&s_full[slot], par, abort_flag, &g_status, p.wait_limit_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t col_s = C::COL_S + slot * BN;
      uint32_t sv[BN];
#pragma unroll
      for (int cc = 0; cc < BN / 32; ++cc) tmem_ld_x32(lane_base + col_s + cc * 32, &sv[cc * 32]);
#pragma unroll
      for (int cc = 0; cc < BN / 32; ++cc) tmem_ld_wait_x32(&sv[cc * 32]);
      float* sc = reinterpret_cast<float*>(sv);
      const int k0 = tile_of(it) * BN;
      int tlo = lo, thi = hi;
      if constexpr (BS) {
        if (!((tile_list[it] >> (30 + t)) & 1u)) {  // block off for this Q tile: no key visible
          tlo = 1;
          thi = 0;
        }
      }
      const bool edge = k0 < tlo || k0 + BN - 1 > thi;
      if (edge) {
#pragma unroll
        for (int c = 0; c < BN; ++c) {
          const int key = k0 + c;
          if (key < tlo || key > thi) sc[c] = -INFINITY;
        }
      }
      float mx0 = fmaxf(sc[0], sc[1]), mx1 = fmaxf(sc[2], sc[3]);
      float mx2 = fmaxf(sc[4], sc[5]), mx3 = fmaxf(sc[6], sc[7]);
#pragma unroll
      for (int c = 8; c < BN; c += 8) {
        mx0 = fmax3(mx0, sc[c], sc[c + 1]);
        mx1 = fmax3(mx1, sc[c + 2], sc[c + 3]);
        mx2 = fmax3(mx2, sc[c + 4], sc[c + 5]);
        mx3 = fmax3(mx3, sc[c + 6], sc[c + 7]);
      }
      const float m_tile = fmax3(mx0, mx1, fmaxf(mx2, mx3)) * sl2;
      const float m_new = fmaxf(m_ref, m_tile);
      const bool grow = m_new > m_ref + 8.0f;
      float alpha = 1.f;
      if (grow) {
        alpha = ex2_approx(m_ref - m_new);
        m_ref = m_new;
      }
      const float mb = (m_ref == -INFINITY) ? 0.f : m_ref;
      uint32_t pk[BN / 2];
      const uint64_t scale2 = f2_pack(sl2, sl2), shift2 = f2_pack(-mb, -mb);
      uint64_t acc0 = 0, acc1 = 0;  // running row sums, two pairs of fp32 lanes
      const uint32_t col_o = C::COL_O + t * D;
      auto rescale_o = [&]() {
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t ov[32];
          tmem_ld_x32(lane_base + col_o + cc * 32, ov);
          tmem_ld_wait_x32(ov);
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
          tmem_st_x32(lane_base + col_o + cc * 32, ov);
        }
      };
      if constexpr (C::SPLITP) {
        // O of this tile is current (PV of the previous key tile completed
        // before S of this one, which was committed after it): rescale it
        // before the first half of P goes to the tensor core
        if (it > 0 && __any_sync(0xffffffffu, grow)) rescale_o();
        if (edge)
          fwd_exp_cols<C, 0, BN / 2, true>(sc, scale2, shift2, pk, acc0, acc1);
        else
          fwd_exp_cols<C, 0, BN / 2, false>(sc, scale2, shift2, pk, acc0, acc1);
#pragma unroll
        for (int cc = 0; cc < BN / 128; ++cc) tmem_st_x32(lane_base + col_s + cc * 32, &pk[cc * 32]);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_full[2 * t]);
        if (edge)
          fwd_exp_cols<C, BN / 2, BN, true>(sc, scale2, shift2, pk, acc0, acc1);
        else
          fwd_exp_cols<C, BN / 2, BN, false>(sc, scale2, shift2, pk, acc0, acc1);
#pragma unroll
        for (int cc = BN / 128; cc < BN / 64; ++cc) tmem_st_x32(lane_base + col_s + cc * 32, &pk[cc * 32]);
        float rs0, rs1;
        f2_unpack(f2_add(acc0, acc1), rs0, rs1);
        l = l * alpha + (rs0 + rs1);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_full[2 * t + 1]);
      } else {
        if (edge)
          fwd_exp_cols<C, 0, BN, true>(sc, scale2, shift2, pk, acc0, acc1);
        else
          fwd_exp_cols<C, 0, BN, false>(sc, scale2, shift2, pk, acc0, acc1);
        float rs0, rs1;
        f2_unpack(f2_add(acc0, acc1), rs0, rs1);
        l = l * alpha + (rs0 + rs1);
#pragma unroll
        for (int cc = 0; cc < BN / 64; ++cc) tmem_st_x32(lane_base + col_s + cc * 32, &pk[cc * 32]);
        // NQT == 1: PV of the previous key tile must be complete before O is
        // rescaled.  The wait is taken at every step, not only when
        // rescaling: a parity wait is only unambiguous while the barrier is
        // at most one phase ahead of the waiter, and this keeps the waiter in
        // lock step.  (NQT == 2: that PV completed before S of this tile.)
        if (NQT == 1 && it > 0) {
          ok = mbar_wait(&o_done[0], (it - 1) & 1, abort_flag, &g_status, p.wait_limit_ns);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
        }
        if (it > 0 && __any_sync(0xffffffffu, grow)) rescale_o();
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_full[NQT == 2 ? 2 * t : slot]);
      }
    }
    // ---- epilogue: O / l -> bf16 -> shared (reusing this tile's Q buffer) -> TMA store
    if (ok && n_kv > 0) {
      // NQT == 2: one commit per tile after its last PV (phase 0), so each
      // tile's epilogue starts as soon as its own O is final;
      // NQT == 1: one commit per PV, the last one is phase n_kv - 1
      ok = mbar_wait(&o_done[NQT == 2 ? t : 0], NQT == 2 ? 0u : static_cast<uint32_t>((n_kv - 1) & 1), abort_flag,
                     &g_status, p.wait_limit_ns);
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
    }
    const uint32_t sQt = sQ + t * C::QTILE;
    const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
    if (ok) {
#pragma unroll 1
      for (int c = 0; c < C::NCHUNK; ++c) {
        uint32_t ov[64];
        if (n_kv > 0) {
          tmem_ld_x32(lane_base + C::COL_O + t * D + c * 64, ov);
          tmem_ld_x32(lane_base + C::COL_O + t * D + c * 64 + 32, ov + 32);
          tmem_ld_wait_x32(ov);
          tmem_ld_wait_x32(ov + 32);
        } else {
#pragma unroll
          for (int i = 0; i < 64; ++i) ov[i] = 0u;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float* f = reinterpret_cast<const float*>(ov + 8 * u);
          st_shared_v4(sQt + c * C::QCHUNK + sw128_offset(r, u),
                       pack2<C::F16>(f[0] * inv_l, f[1] * inv_l), pack2<C::F16>(f[2] * inv_l, f[3] * inv_l),
                       pack2<C::F16>(f[4] * inv_l, f[5] * inv_l), pack2<C::F16>(f[6] * inv_l, f[7] * inv_l));
        }
      }
      fence_proxy_async_smem();
    }
    named_bar_sync(1 + t, BM);
    const bool aborted = *abort_flag != 0;
    const int t_row0 = r0 + t * BM;
    if (!VL || t_row0 + BM <= nq) {
      // whole tile (or dense, where TMA clips the tensor's last tile itself)
      if (r == 0 && !aborted && t_row0 < nq) {
        for (int c = 0; c < C::NCHUNK; ++c)
          tma_store_4d(&tm_o, sQt + c * C::QCHUNK, c * 64, h, q_off + t_row0, tb);
        tma_store_commit();
        tma_store_wait_read();
      }
    } else if (!aborted) {
      // last tile of a packed sequence: rows past its end belong to the next
      // sequence, so only the valid rows are stored, 16 bytes at a time
      store_rows_sw128(sQt, C::QCHUNK, nq - t_row0, D, p.o, q_off + t_row0, p.total_q, p.Hq, h, D, 0, r, BM);
    }
    if (!aborted && row < nq && (!VL || (q_off + row >= 0 && q_off + row < p.total_q))) {
      const float mb = (m_ref == -INFINITY) ? 0.f : m_ref;
      const size_t lse_row = VL ? static_cast<size_t>(h) * p.total_q + q_off + row
                                : (static_cast<size_t>(b) * p.Hq + h) * p.Nq + row;
      p.lse[lse_row] = (l > 0.f) ? (mb + log2f(l)) * kLn2 : -INFINITY;
    }
  } else {
    setmaxnreg_dec<C::REG_PRODUCER>();  // idle members of the producer warpgroup
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == C::MMA_WARP) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace fa
