// fa_decode.cuh -- forward pass for a few query rows against a long key/value
// sequence (decoding with a KV cache), split over the keys.
//
// Same result as fa_fwd: O = softmax(scale Q K^T) V and LSE per query row,
// with the masks and the GQA head mapping of fa_fwd (hysenlabs FlashAttention
// API page, option list and changelog v2.2 on the KV-cache decoding path).
// The work of one step is dominated by reading K and V once from HBM, and
// with Nq small the (batch, head, query tile) units are too few to fill the
// GPU, so the keys are split as well:
//
//   fa_decode_kernel  CTA (query tile, split, batch, kv head): the G = Hq/Hkv
//       query heads of one key/value head and `qpt` query rows of each are
//       packed into the rows of one 128-row Q tile (row rr = query rr / G,
//       head rr % G), so K and V are streamed once per group, not once per
//       query head.  The CTA walks its contiguous share of the visible key
//       tiles with the online softmax of fa_fwd (S = Q K^T and O += P V on
//       tcgen05, S/P/O in tensor memory).
//   When the packed rows fill only 32 (or 64) TMEM lanes, the rows are stored
//   4 (or 2) times in the Q tile.  Copy c then owns key columns
//   [c * BN / NC, (c + 1) * BN / NC) of every key tile: its softmax warp
//   computes exponentials for those columns only and leaves P zero elsewhere,
//   so each copy runs an independent online softmax over its own subset of the
//   keys and the exponentials per thread drop NC-fold.  The epilogue merges
//   the copies with the blockwise softmax rule (abeam.tech FlashAttention
//   summary, "computing softmax blockwise correctly"): with per-copy row
//   statistics (m_c, l_c) and outputs O_c, M = max m_c,
//   L = sum_c 2^(m_c - M) l_c and O = sum_c 2^(m_c - M) O_c / L.
//   With more than one split, every CTA stores its normalised partial output
//   and LSE, then counts itself done on its unit's counter; the CTA that
//   completes the count merges all splits of the unit the same way, in
//   natural-log form: lse = ln sum_s exp(lse_s), O = sum_s exp(lse_s - lse)
//   O_s, summed in split order whichever CTA does it, so the result does not
//   depend on the order the CTAs finish.  No CTA waits for another.
#pragma once
#include "fa_fwd.cuh"

namespace fa {

struct DecodeParams {
  int B, Nq, Nk, Hq, Hkv, group;  // group = Hq / Hkv
  int qpt;                        // query rows per tile; rows per tile RT = qpt * group <= 128
  int n_qtiles;                   // ceil(Nq / qpt)
  int n_splits;                   // most key splits of a (batch, kv head, query tile) unit
  int split_tiles;                // key tiles per split; a unit with n visible key tiles
                                  // uses ceil(n / split_tiles) splits (at least 1)
  float scale_log2;
  MaskSpec mask;                  // with Nk = the key capacity; per batch see below
  const int* seqlens;             // [B] cached keys per sequence, or null (all Nk)
  int n_new;                      // keys appended after seqlens[b] by this call
  uint16_t* o;               // [B, Nq, Hq, d]
  float* lse;                     // [B, Hq, Nq]
  float* part_o;                  // [units, n_splits, RT, d] normalised partial O (n_splits > 1)
  float* part_lse;                // [units, n_splits, RT]    natural-log partial LSE
  unsigned long long* counters;   // [units] finished splits: call tag << 32 | count
  unsigned int tag;               // nonzero, different for consecutive calls
  unsigned long long wait_limit_ns;
};

// RCP: TMEM lanes (rows) one copy of the packed rows spans: 32, 64 or 128.
template <int D_, int BN_, int KST_, int RCP_>
struct DecCfg {
  static constexpr bool F16 = false;  // elements are bf16 (AsF16<> flips it to fp16)
  static constexpr int D = D_, BN = BN_, KST = KST_, RCP = RCP_;
  static constexpr int BM = 128;
  static constexpr int NC = BM / RCP;        // copies of the packed rows
  static constexpr int CW = BN / NC;         // key columns per copy and tile
  static constexpr int WPC = RCP / 32;       // softmax warps per copy
  static constexpr int NCHUNK = D / 64;
  static constexpr int QCHUNK = BM * 128;
  static constexpr int KCHUNK = BN * 128;
  static constexpr int QTILE = NCHUNK * QCHUNK;
  static constexpr int KTILE = NCHUNK * KCHUNK;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + QTILE;
  static constexpr int OFF_V = OFF_K + KST * KTILE;
  static constexpr int OFF_BAR = OFF_V + KST * KTILE;
  // k_full[KST], k_empty[KST], v_full[KST], v_empty[KST], s_full[2], p_full[2], o_done, drain
  static constexpr int NBAR = 4 * KST + 6;
  static constexpr int OFF_STAT = OFF_BAR + NBAR * 8;   // m[128], l[128]
  static constexpr int OFF_MISC = OFF_STAT + 2 * BM * 4;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  // epilogue staging of the copies' weighted O rows, over the Q/K/V buffers
  static constexpr int STAGE_LD = D + 4;     // floats per staged row (4 pad: no bank conflicts)
  static constexpr int STAGE_FLOATS = BM * STAGE_LD;
  static_assert(STAGE_FLOATS * 4 <= OFF_BAR, "epilogue staging fits the tile buffers");
  // warps 0-3 softmax (TMEM lane quarter = warp), 4 TMA, 5 MMA
  static constexpr int NTHREADS = 192;
  static constexpr int TMA_WARP = 4, MMA_WARP = 5;
  // TMEM columns: S slots [0, 2 BN), P slots [2 BN, 3 BN) (bf16 pairs, BN/2
  // columns each), O [3 BN, 3 BN + D)
  static constexpr int COL_S = 0, COL_P = 2 * BN, COL_O = 3 * BN;
  static constexpr int TMEM_USED = 3 * BN + D;
  static constexpr int TMEM_COLS = TMEM_USED <= 128 ? 128 : TMEM_USED <= 256 ? 256 : 512;
  static_assert(TMEM_USED <= 512, "TMEM budget");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(CW >= 16 && CW % 16 == 0, "columns per copy");
};

// CW fp32 scores of this thread's TMEM lane, starting at column address taddr
template <int CW>
__device__ __forceinline__ void dec_load_cols(uint32_t taddr, uint32_t* sv) {
  if constexpr (CW == 16) {
    tmem_ld_x16(taddr, sv);
    tmem_ld_wait_x16(sv);
  } else {
#pragma unroll
    for (int cc = 0; cc < CW / 32; ++cc) tmem_ld_x32(taddr + cc * 32, &sv[cc * 32]);
#pragma unroll
    for (int cc = 0; cc < CW / 32; ++cc) tmem_ld_wait_x32(&sv[cc * 32]);
  }
}

// N packed bf16 pairs to TMEM (N = CW / 2)
template <int N>
__device__ __forceinline__ void dec_store_cols(uint32_t taddr, const uint32_t* pk) {
  if constexpr (N == 8) {
    tmem_st_x8(taddr, pk);
  } else if constexpr (N == 16) {
    tmem_st_x16(taddr, pk);
  } else {
#pragma unroll
    for (int cc = 0; cc < N / 32; ++cc) tmem_st_x32(taddr + cc * 32, &pk[cc * 32]);
  }
}

// Counts one more finished split on a unit's counter and returns true for the
// split that completes the count (and resets the counter to zero for the next
// call).  The counter holds (call tag << 32 | splits counted); a value with
// another call's tag counts as zero, so the workspace needs no clearing.  A
// compare-and-swap retry loop, bounded: each failed attempt means another
// split of the unit got its count in.
__device__ __forceinline__ bool decode_claim_last(unsigned long long* ctr, unsigned int tag, int n_splits) {
  unsigned long long old = *reinterpret_cast<volatile unsigned long long*>(ctr);
  for (int tries = 0; tries < (1 << 20); ++tries) {
    const unsigned long long base = (old >> 32) == tag ? old : static_cast<unsigned long long>(tag) << 32;
    const unsigned long long want = base + 1;
    const unsigned long long seen = atomicCAS(ctr, old, want);
    if (seen == old) {
      const bool last = static_cast<int>(want & 0xffffffffull) == n_splits;
      if (last) atomicExch(ctr, 0ull);
      return last;
    }
    old = seen;
  }
  atomicExch(&g_status, kDevTimeout);
  return false;
}

template <class C>
__global__ void __launch_bounds__(C::NTHREADS, 1)
    fa_decode_kernel(const uint16_t* __restrict__ q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const DecodeParams p) {
  constexpr int D = C::D, BN = C::BN, KST = C::KST, BM = C::BM, RCP = C::RCP, NC = C::NC, CW = C::CW;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* k_full = bars;
  uint64_t* k_empty = k_full + KST;
  uint64_t* v_full = k_empty + KST;
  uint64_t* v_empty = v_full + KST;
  uint64_t* s_full = v_empty + KST;  // [2]
  uint64_t* p_full = s_full + 2;     // [2]
  uint64_t* o_done = p_full + 2;
  uint64_t* bar_drain = o_done + 1;
  float* stat_m = reinterpret_cast<float*>(smem + C::OFF_STAT);
  float* stat_l = stat_m + BM;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  volatile int* last_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);
  float* stage = reinterpret_cast<float*>(smem);
  const uint32_t sQ = sbase + C::OFF_Q, sK = sbase + C::OFF_K, sV = sbase + C::OFF_V;

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  // ---- work unit: query tile fastest, so the tiles sharing a key range run together
  const int qt = blockIdx.x % p.n_qtiles;
  const int split = (blockIdx.x / p.n_qtiles) % p.n_splits;
  const int bk = blockIdx.x / (p.n_qtiles * p.n_splits);  // b * Hkv + hk
  const int b = bk / p.Hkv, hk = bk % p.Hkv;
  const int G = p.group;
  const int RT = p.qpt * G;
  const int i_first = qt * p.qpt;
  const int i_last = min(p.Nq - 1, i_first + p.qpt - 1);
  // keys of this sequence: the whole capacity, or its cached length plus the
  // keys appended by this call (clamped to the capacity); the causal diagonal
  // and the window are aligned to that length
  MaskSpec mask = p.mask;
  if (p.seqlens != nullptr) mask.Nk = max(0, min(p.Nk, __ldg(p.seqlens + b) + p.n_new));
  const int key_lo = mask.lo(i_first), key_hi = mask.hi(i_last);
  const int j_all = key_lo / BN;
  const int n_all = (key_hi >= key_lo) ? (key_hi / BN - j_all + 1) : 0;
  // this unit's splits: a fixed number of key tiles each, so a sequence with
  // fewer keys (ragged cache lengths) takes fewer CTAs; the others leave at once
  int split_tiles = p.split_tiles;
  int ns = max(1, (n_all + split_tiles - 1) / split_tiles);
  if (ns > p.n_splits) {  // more tiles than the launch planned for: spread them over its splits
    split_tiles = (n_all + p.n_splits - 1) / p.n_splits;
    ns = max(1, (n_all + split_tiles - 1) / split_tiles);
  }
  if (split >= ns) return;
  const int t_begin = split * split_tiles;
  const int n_kv = min(n_all, t_begin + split_tiles) - t_begin;
  const int j_begin = j_all + t_begin;

  auto load_k = [&](int it) {
    const int s = it % KST, krow = (j_begin + it) * BN;
    mbar_expect_tx(&k_full[s], C::KTILE);
    for (int c = 0; c < C::NCHUNK; ++c)
      tma_load_4d(sK + s * C::KTILE + c * C::KCHUNK, &tm_k, &k_full[s], c * 64, hk, krow, b);
  };
  auto load_v = [&](int it) {
    const int s = it % KST, krow = (j_begin + it) * BN;
    mbar_expect_tx(&v_full[s], C::KTILE);
    for (int c = 0; c < C::NCHUNK; ++c)
      tma_load_4d(sV + s * C::KTILE + c * C::KCHUNK, &tm_v, &v_full[s], c * 64, hk, krow, b);
  };
  const int n_pre = min(n_kv, KST);
  if (warp == C::TMA_WARP && lane == 0) {
    for (int s = 0; s < KST; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], BM);
    }
    mbar_init(o_done, 1);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    for (int it = 0; it < n_pre; ++it) {
      load_k(it);
      load_v(it);
    }
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(smem_addr(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp < 4) {
    // packed Q rows -> every copy of the Q tile (128-byte swizzle, 16-byte
    // units); rows past the tile or past Nq are zero
    constexpr int UPR = D / 8;  // 16-byte units per row
    for (int x = threadIdx.x; x < RCP * UPR; x += 128) {
      const int rr = x / UPR, u = x % UPR;
      const int i = i_first + rr / G;
      uint4 val = make_uint4(0u, 0u, 0u, 0u);
      if (rr < RT && i < p.Nq) {
        const int hq = hk * G + rr % G;
        val = __ldg(reinterpret_cast<const uint4*>(q + ((static_cast<size_t>(b) * p.Nq + i) * p.Hq + hq) * D) + u);
      }
#pragma unroll
      for (int c = 0; c < NC; ++c)
        st_shared_v4(sQ + (u / 8) * C::QCHUNK + sw128_offset(c * RCP + rr, u % 8), val.x, val.y, val.z, val.w);
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == C::TMA_WARP) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && n_kv > 0) {
      int nk = n_pre, nv = n_pre;
      for (int it = n_pre; it < n_kv; ++it) {
        const int s = it % KST, use = it / KST;
        if (!mbar_wait(&k_empty[s], (use - 1) & 1, abort_flag, &g_status, p.wait_limit_ns)) break;
        load_k(it);
        ++nk;
        if (!mbar_wait(&v_empty[s], (use - 1) & 1, abort_flag, &g_status, p.wait_limit_ns)) break;
        load_v(it);
        ++nv;
      }
      for (int s = 0; s < KST; ++s) {
        if (nk > s) mbar_drain(&k_full[s], ((nk - 1 - s) / KST) & 1, p.wait_limit_ns);
        if (nv > s) mbar_drain(&v_full[s], ((nv - 1 - s) / KST) & 1, p.wait_limit_ns);
      }
    }
  } else if (warp == C::MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_kv > 0) {
      constexpr uint32_t ID_QK = idesc_kind_f16<C::F16>(128, BN, false, false);
      constexpr uint32_t ID_PV = idesc_kind_f16<C::F16>(128, D, false, true);
      const uint64_t dq0 = sdesc_sw128(sQ, 16, 1024);
      const uint64_t dk0 = sdesc_sw128(sK, 16, 1024);
      const uint64_t dv0 = sdesc_sw128(sV, C::KCHUNK, 1024);
      auto wait = [&](uint64_t* bar, uint32_t par) {
        const bool ok = mbar_wait(bar, par, abort_flag, &g_status, p.wait_limit_ns);
        tc_fence_after();
        return ok;
      };
      auto issue_s = [&](int slot, int s) {
        FwdIssueS<C>::run(tmem + C::COL_S + slot * BN, dq0, dk0 + static_cast<uint64_t>((s * C::KTILE) >> 4), ID_QK);
      };
      auto issue_pv = [&](int slot, int s, bool acc) {
        FwdIssuePV<C>::run(tmem + C::COL_O, tmem + C::COL_P + slot * (BN / 2),
                           dv0 + static_cast<uint64_t>((s * C::KTILE) >> 4), ID_PV, acc);
      };
      // S slots alternate between consecutive key tiles; S of tile it + 2
      // goes in as soon as PV of tile it is issued
      bool ok = wait(&k_full[0], 0);
      if (ok) {
        issue_s(0, 0);
        tc_commit(&s_full[0]);
        tc_commit(&k_empty[0]);
        if (n_kv > 1 && (ok = wait(&k_full[1 % KST], (1 / KST) & 1))) {
          issue_s(1, 1 % KST);
          tc_commit(&s_full[1]);
          tc_commit(&k_empty[1 % KST]);
        }
      }
      for (int it = 0; it < n_kv && ok; ++it) {
        const int slot = it & 1, s = it % KST;
        if (!(ok = wait(&p_full[slot], (it >> 1) & 1))) break;
        if (!(ok = wait(&v_full[s], (it / KST) & 1))) break;
        issue_pv(slot, s, it > 0);
        tc_commit(o_done);
        tc_commit(&v_empty[s]);
        if (it + 2 < n_kv) {
          const int s2 = (it + 2) % KST;
          if (!(ok = wait(&k_full[s2], ((it + 2) / KST) & 1))) break;
          issue_s(slot, s2);
          tc_commit(&s_full[slot]);
          tc_commit(&k_empty[s2]);
        }
      }
    }
    if (lane == 0) {
      tc_commit(bar_drain);
      mbar_drain(bar_drain, 0, p.wait_limit_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int c = warp / C::WPC;                  // copy of this warp
    const int rr = (warp % C::WPC) * 32 + lane;   // packed row within the copy
    const int tl = warp * 32 + lane;              // TMEM lane = c * RCP + rr
    const int i = i_first + rr / G;
    const bool row_ok = rr < RT && i < p.Nq;
    const int lo = row_ok ? mask.lo(i) : 1, hi = row_ok ? mask.hi(i) : 0;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const float sl2 = p.scale_log2;
    if constexpr (NC > 1) {
      // P stays zero outside this copy's columns for the whole CTA
      uint32_t zero[32];
#pragma unroll
      for (int x = 0; x < 32; ++x) zero[x] = 0u;
#pragma unroll
      for (int cc = 0; cc < BN / 32; ++cc) tmem_st_x32(lane_base + C::COL_P + cc * 32, zero);
    }
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int it = 0; it < n_kv; ++it) {
      const int slot = it & 1;
      ok = mbar_wait(&s_full[slot], (it >> 1) & 1, abort_flag, &g_status, p.wait_limit_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      uint32_t sv[CW];
      dec_load_cols<CW>(lane_base + C::COL_S + slot * BN + c * CW, sv);
      float* sc = reinterpret_cast<float*>(sv);
      const int k0 = (j_begin + it) * BN + c * CW;
      if (k0 < lo || k0 + CW - 1 > hi) {
#pragma unroll
        for (int x = 0; x < CW; ++x)
          if (k0 + x < lo || k0 + x > hi) sc[x] = -INFINITY;
      }
      float mx0 = sc[0], mx1 = sc[1];
#pragma unroll
      for (int x = 2; x < CW; x += 2) {
        mx0 = fmaxf(mx0, sc[x]);
        mx1 = fmaxf(mx1, sc[x + 1]);
      }
      const float m_new = fmaxf(m_ref, fmaxf(mx0, mx1) * sl2);
      const bool grow = m_new > m_ref + 8.0f;
      float alpha = 1.f;
      if (grow) {
        alpha = ex2_approx(m_ref - m_new);
        m_ref = m_new;
      }
      const float mb = (m_ref == -INFINITY) ? 0.f : m_ref;
      uint32_t pk[CW / 2];
      float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
      for (int x = 0; x < CW; x += 2) {
        const float p0 = ex2_approx(fmaf(sc[x], sl2, -mb));
        const float p1 = ex2_approx(fmaf(sc[x + 1], sl2, -mb));
        pk[x / 2] = pack2<C::F16>(p0, p1);
        rs0 += p0;
        rs1 += p1;
      }
      l = l * alpha + (rs0 + rs1);
      dec_store_cols<CW / 2>(lane_base + C::COL_P + slot * (BN / 2) + c * (CW / 2), pk);
      // PV of the previous tile must be complete before O is rescaled; the
      // wait is taken every step so the parity stays unambiguous
      if (it > 0) {
        ok = mbar_wait(o_done, (it - 1) & 1, abort_flag, &g_status, p.wait_limit_ns);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, grow)) {
#pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t ov[32];
            tmem_ld_x32(lane_base + C::COL_O + cc * 32, ov);
            tmem_ld_wait_x32(ov);
#pragma unroll
            for (int x = 0; x < 32; ++x) ov[x] = __float_as_uint(__uint_as_float(ov[x]) * alpha);
            tmem_st_x32(lane_base + C::COL_O + cc * 32, ov);
          }
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[slot]);
    }
    if (ok && n_kv > 0) {
      ok = mbar_wait(o_done, static_cast<uint32_t>((n_kv - 1) & 1), abort_flag, &g_status, p.wait_limit_ns);
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
    }
    // ---- epilogue: merge the copies (statistics through shared memory, the
    // weighted O rows staged over the now idle tile buffers), then store
    stat_m[tl] = m_ref;
    stat_l[tl] = l;
    named_bar_sync(1, BM);
    float M = -INFINITY;
#pragma unroll
    for (int x = 0; x < NC; ++x) M = fmaxf(M, stat_m[x * RCP + rr]);
    float L = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int x = 0; x < NC; ++x) {
        const float mx = stat_m[x * RCP + rr];
        if (mx != -INFINITY) L += stat_l[x * RCP + rr] * ex2_approx(mx - M);
      }
    }
    const float wgt = (L > 0.f && m_ref != -INFINITY) ? ex2_approx(m_ref - M) / L : 0.f;
    float* srow = stage + static_cast<size_t>(tl) * C::STAGE_LD;
#pragma unroll 1
    for (int cc = 0; cc < D / 32; ++cc) {
      uint32_t ov[32];
      if (ok && n_kv > 0) {
        tmem_ld_x32(lane_base + C::COL_O + cc * 32, ov);
        tmem_ld_wait_x32(ov);
      } else {
#pragma unroll
        for (int x = 0; x < 32; ++x) ov[x] = 0u;
      }
#pragma unroll
      for (int x = 0; x < 32; x += 4)
        *reinterpret_cast<float4*>(srow + cc * 32 + x) =
            make_float4(__uint_as_float(ov[x]) * wgt, __uint_as_float(ov[x + 1]) * wgt,
                        __uint_as_float(ov[x + 2]) * wgt, __uint_as_float(ov[x + 3]) * wgt);
    }
    named_bar_sync(1, BM);
    const bool aborted = *abort_flag != 0;
    if (!aborted) {
      const long long unit = static_cast<long long>(bk) * p.n_qtiles + qt;
      if (ns == 1) {
        constexpr int UPR = D / 8;
        for (int x = threadIdx.x; x < RT * UPR; x += BM) {
          const int r2 = x / UPR, col = (x % UPR) * 8;
          const int i2 = i_first + r2 / G;
          if (i2 >= p.Nq) continue;
          float f[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) f[e] = 0.f;
#pragma unroll
          for (int x2 = 0; x2 < NC; ++x2) {
            const float* sr = stage + static_cast<size_t>(x2 * RCP + r2) * C::STAGE_LD + col;
            const float4 a = *reinterpret_cast<const float4*>(sr);
            const float4 a2 = *reinterpret_cast<const float4*>(sr + 4);
            f[0] += a.x; f[1] += a.y; f[2] += a.z; f[3] += a.w;
            f[4] += a2.x; f[5] += a2.y; f[6] += a2.z; f[7] += a2.w;
          }
          const int hq = hk * G + r2 % G;
          *reinterpret_cast<uint4*>(p.o + ((static_cast<size_t>(b) * p.Nq + i2) * p.Hq + hq) * D + col) =
              make_uint4(pack2<C::F16>(f[0], f[1]), pack2<C::F16>(f[2], f[3]), pack2<C::F16>(f[4], f[5]),
                         pack2<C::F16>(f[6], f[7]));
        }
        if (c == 0 && row_ok)
          p.lse[(static_cast<size_t>(b) * p.Hq + hk * G + rr % G) * p.Nq + i] =
              (L > 0.f) ? (M + log2f(L)) * kLn2 : -INFINITY;
      } else {
        constexpr int UPR = D / 4;
        const size_t pbase = (static_cast<size_t>(unit) * p.n_splits + split) * RT;
        for (int x = threadIdx.x; x < RT * UPR; x += BM) {
          const int r2 = x / UPR, col = (x % UPR) * 4;
          float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int x2 = 0; x2 < NC; ++x2) {
            const float4 a =
                *reinterpret_cast<const float4*>(stage + static_cast<size_t>(x2 * RCP + r2) * C::STAGE_LD + col);
            f.x += a.x; f.y += a.y; f.z += a.z; f.w += a.w;
          }
          *reinterpret_cast<float4*>(p.part_o + (pbase + r2) * D + col) = f;
        }
        if (c == 0 && rr < RT) p.part_lse[pbase + rr] = (L > 0.f) ? (M + log2f(L)) * kLn2 : -INFINITY;
        // publish the partial result; the split that completes the unit's
        // count merges all of them
        __threadfence();
        named_bar_sync(1, BM);
        if (threadIdx.x == 0) *last_flag = decode_claim_last(p.counters + unit, p.tag, ns) ? 1 : 0;
        named_bar_sync(1, BM);
        if (*last_flag && ns * RT <= C::STAGE_FLOATS) {
          // the unit's partial LSEs (contiguous, [split][row]) into shared
          // memory in one parallel pass, then turned into merge weights
          __threadfence();
          const size_t ubase = static_cast<size_t>(unit) * p.n_splits * RT;  // split s, row r: ubase + s RT + r
          const int nsr = ns * RT;
          for (int x = threadIdx.x; x < nsr; x += BM) stage[x] = __ldcg(p.part_lse + ubase + x);
          named_bar_sync(1, BM);
          if (threadIdx.x < RT) {
            const int r2 = threadIdx.x;
            float mx = -INFINITY;
            for (int s = 0; s < ns; ++s) mx = fmaxf(mx, stage[s * RT + r2]);
            float sum = 0.f;
            if (mx != -INFINITY) {
              for (int s = 0; s < ns; ++s) {
                const float ls = stage[s * RT + r2];
                if (ls != -INFINITY) sum += ex2_approx((ls - mx) * kLog2e);
              }
            }
            const float Lr = (mx == -INFINITY) ? -INFINITY : mx + logf(sum);
            stat_l[r2] = Lr;
            const int i2 = i_first + r2 / G;
            if (i2 < p.Nq) p.lse[(static_cast<size_t>(b) * p.Hq + hk * G + r2 % G) * p.Nq + i2] = Lr;
          }
          named_bar_sync(1, BM);
          for (int x = threadIdx.x; x < nsr; x += BM) {
            const float ls = stage[x], Lr = stat_l[x % RT];
            stage[x] = (ls == -INFINITY || Lr == -INFINITY) ? 0.f : ex2_approx((ls - Lr) * kLog2e);
          }
          named_bar_sync(1, BM);
          constexpr int UPR8 = D / 8;
          for (int x = threadIdx.x; x < RT * UPR8; x += BM) {
            const int r2 = x / UPR8, col = (x % UPR8) * 8;
            const int i2 = i_first + r2 / G;
            if (i2 >= p.Nq) continue;
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = 0.f;
#pragma unroll 4
            for (int s = 0; s < ns; ++s) {
              const float w = stage[s * RT + r2];
              const size_t row = ubase + static_cast<size_t>(s) * RT + r2;
              const float4 a = __ldcg(reinterpret_cast<const float4*>(p.part_o + row * D + col));
              const float4 a2 = __ldcg(reinterpret_cast<const float4*>(p.part_o + row * D + col + 4));
              f[0] = fmaf(w, a.x, f[0]); f[1] = fmaf(w, a.y, f[1]);
              f[2] = fmaf(w, a.z, f[2]); f[3] = fmaf(w, a.w, f[3]);
              f[4] = fmaf(w, a2.x, f[4]); f[5] = fmaf(w, a2.y, f[5]);
              f[6] = fmaf(w, a2.z, f[6]); f[7] = fmaf(w, a2.w, f[7]);
            }
            const int hq = hk * G + r2 % G;
            *reinterpret_cast<uint4*>(p.o + ((static_cast<size_t>(b) * p.Nq + i2) * p.Hq + hq) * D + col) =
                make_uint4(pack2<C::F16>(f[0], f[1]), pack2<C::F16>(f[2], f[3]), pack2<C::F16>(f[4], f[5]),
                           pack2<C::F16>(f[6], f[7]));
          }
        } else if (*last_flag) {
          // more partial rows than the staging buffer holds: the same merge,
          // reading the LSEs straight from global memory
          __threadfence();
          const size_t ubase = static_cast<size_t>(unit) * p.n_splits * RT;
          if (threadIdx.x < RT) {
            const int r2 = threadIdx.x;
            float mx = -INFINITY;
            for (int s = 0; s < ns; ++s) mx = fmaxf(mx, __ldcg(p.part_lse + ubase + static_cast<size_t>(s) * RT + r2));
            float sum = 0.f;
            if (mx != -INFINITY) {
              for (int s = 0; s < ns; ++s) {
                const float ls = __ldcg(p.part_lse + ubase + static_cast<size_t>(s) * RT + r2);
                if (ls != -INFINITY) sum += ex2_approx((ls - mx) * kLog2e);
              }
            }
            const float Lr = (mx == -INFINITY) ? -INFINITY : mx + logf(sum);
            stat_l[r2] = Lr;
            const int i2 = i_first + r2 / G;
            if (i2 < p.Nq) p.lse[(static_cast<size_t>(b) * p.Hq + hk * G + r2 % G) * p.Nq + i2] = Lr;
          }
          named_bar_sync(1, BM);
          constexpr int UPR8 = D / 8;
          for (int x = threadIdx.x; x < RT * UPR8; x += BM) {
            const int r2 = x / UPR8, col = (x % UPR8) * 8;
            const int i2 = i_first + r2 / G;
            if (i2 >= p.Nq) continue;
            const float Lr = stat_l[r2];
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = 0.f;
            if (Lr != -INFINITY) {
              for (int s = 0; s < ns; ++s) {
                const size_t row = ubase + static_cast<size_t>(s) * RT + r2;
                const float ls = __ldcg(p.part_lse + row);
                if (ls == -INFINITY) continue;
                const float w = ex2_approx((ls - Lr) * kLog2e);
                const float4 a = __ldcg(reinterpret_cast<const float4*>(p.part_o + row * D + col));
                const float4 a2 = __ldcg(reinterpret_cast<const float4*>(p.part_o + row * D + col + 4));
                f[0] = fmaf(w, a.x, f[0]); f[1] = fmaf(w, a.y, f[1]);
                f[2] = fmaf(w, a.z, f[2]); f[3] = fmaf(w, a.w, f[3]);
                f[4] = fmaf(w, a2.x, f[4]); f[5] = fmaf(w, a2.y, f[5]);
                f[6] = fmaf(w, a2.z, f[6]); f[7] = fmaf(w, a2.w, f[7]);
              }
            }
            const int hq = hk * G + r2 % G;
            *reinterpret_cast<uint4*>(p.o + ((static_cast<size_t>(b) * p.Nq + i2) * p.Hq + hq) * D + col) =
                make_uint4(pack2<C::F16>(f[0], f[1]), pack2<C::F16>(f[2], f[3]), pack2<C::F16>(f[4], f[5]),
                           pack2<C::F16>(f[6], f[7]));
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == C::MMA_WARP) tmem_dealloc(tmem, C::TMEM_COLS);
}

// In-place append of the new keys and values to the caches: row t of
// sequence b goes to cache row seqlens[b] + t (rows at or past the capacity
// Nk are dropped).  One thread per 16 bytes of a row of K and of V.
__global__ void __launch_bounds__(256)
    fa_kvcache_append_kernel(uint16_t* __restrict__ k_cache, uint16_t* __restrict__ v_cache,
                             const uint16_t* __restrict__ k_new, const uint16_t* __restrict__ v_new,
                             const int* __restrict__ seqlens, int B, int n_new, int Nk, int Hkv, int d) {
  const int upr = d / 8;  // 16-byte units per row
  const long long total = static_cast<long long>(B) * n_new * Hkv * upr;
  for (long long x = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; x < total;
       x += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int u = static_cast<int>(x % upr);
    const long long row = x / upr;  // (b, t, h)
    const int h = static_cast<int>(row % Hkv);
    const long long bt = row / Hkv;
    const int t = static_cast<int>(bt % n_new);
    const int b = static_cast<int>(bt / n_new);
    const int dst = __ldg(seqlens + b) + t;
    if (dst < 0 || dst >= Nk) continue;
    const size_t src_off = static_cast<size_t>(row) * d + u * 8;
    const size_t dst_off = ((static_cast<size_t>(b) * Nk + dst) * Hkv + h) * d + u * 8;
    *reinterpret_cast<uint4*>(k_cache + dst_off) = __ldg(reinterpret_cast<const uint4*>(k_new + src_off));
    *reinterpret_cast<uint4*>(v_cache + dst_off) = __ldg(reinterpret_cast<const uint4*>(v_new + src_off));
  }
}

}  // namespace fa
