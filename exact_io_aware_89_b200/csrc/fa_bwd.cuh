// fa_bwd.cuh -- backward pass of exact attention on sm_100a.
//
// The pages fix only the strategy (abeam.tech FlashAttention summary,
// "backward uses recomputation": keep the softmax statistics of the forward,
// recompute attention blockwise instead of storing P).  The formulas are the
// calculus of the loss L = sum(dO * O):
//   P_ij  = exp(scale * q_i.k_j - LSE_i)         (recomputed from the saved LSE)
//   D_i   = sum_c dO_ic O_ic
//   dP_ij = dO_i . v_j,   dS_ij = P_ij (dP_ij - D_i)
//   dV_j  = sum_i P_ij dO_i,  dK_j = scale sum_i dS_ij q_i,  dQ_i = scale sum_j dS_ij k_j
//
// Three launches on the caller's stream:
//   1. fa_bwd_prep_*      : D_i and lse2_i = LSE_i * log2(e) into the workspace
//                           (rows padded to a multiple of 256; padding rows get
//                           lse2 = +inf so every P there is exactly 0).
//   2. fa_bwd_dq_kernel   : query-stationary.  Per key tile: S = Q K^T and
//                           dP = dO V^T (tcgen05, TMEM), dS in registers, dS
//                           written back into TMEM as bf16, dQ += dS K with dS
//                           read from TMEM.  dQ is accumulated in fp32 in TMEM
//                           by one CTA in a fixed order, so it is deterministic
//                           with no atomics and no extra workspace.
//   3. fa_bwd_dkdv_kernel : key-stationary.  Per (query head of the group,
//                           query tile): S^T = K Q^T and dP^T = V dO^T, then
//                           P^T and dS^T (bf16, in TMEM over their sources),
//                           dV += P^T dO and dK += dS^T Q.  dK/dV for a GQA group
//                           are summed inside one CTA, in a fixed order.
// Every contraction is a tcgen05 tile GEMM fed by TMA.
#pragma once
#include "fa_common.cuh"

namespace fa {

// =====================================================================
// 1. preprocess: D = rowsum(dO * O), lse2 = LSE * log2(e)
// =====================================================================
// fp32 inputs (the fp32 entry points): one warp per (b, i, h) row; ws layout:
// D [B, Hq, Nq_pad] then lse2 [B, Hq, Nq_pad]
template <typename T>
__global__ void __launch_bounds__(256) fa_bwd_prep_kernel(const T* __restrict__ o,
                                                          const T* __restrict__ dout,
                                                          const float* __restrict__ lse,
                                                          float* __restrict__ ws, int B, int Nq,
                                                          int Hq, int d, int Nq_pad) {
  const long long warp_id = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) / 32;
  const int lane = threadIdx.x % 32;
  const long long rows_pad = static_cast<long long>(B) * Hq * Nq_pad;
  if (warp_id >= rows_pad) return;
  const int i = static_cast<int>(warp_id % Nq_pad);
  const long long bh = warp_id / Nq_pad;
  const int h = static_cast<int>(bh % Hq);
  const int b = static_cast<int>(bh / Hq);
  float* Dp = ws + warp_id;
  float* L2p = ws + rows_pad + warp_id;
  if (i >= Nq) {
    if (lane == 0) {
      *Dp = 0.f;
      *L2p = INFINITY;
    }
    return;
  }
  const size_t base = ((static_cast<size_t>(b) * Nq + i) * Hq + h) * d;
  float acc = 0.f;
  for (int c = lane; c < d; c += 32) acc += static_cast<float>(o[base + c]) * static_cast<float>(dout[base + c]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) {
    *Dp = acc;
    const float L = lse[(static_cast<size_t>(b) * Hq + h) * Nq + i];
    // a row with no visible key (LSE = -inf) has P = 0 everywhere
    *L2p = (L == -INFINITY) ? INFINITY : L * kLog2e;
  }
}

// bf16 or fp16 (F16): G = d / 8 lanes per row, each loading 8 elements of O and of dO with
// one 16-byte load; the G partial dot products are added with shuffles inside
// the lane group (groups are aligned within the warp, G divides 32).  Each
// lane group handles RPG rows, with all their loads issued before any use, so
// that enough bytes are in flight to approach HBM bandwidth.  Same outputs
// and layout as fa_bwd_prep_kernel; rows_pad must be a multiple of
// RPG * 256 / G (it is a multiple of 256).
template <int G, int RPG, bool VL = false, bool F16 = false>
__global__ void __launch_bounds__(256) fa_bwd_prep_h16_kernel(const uint16_t* __restrict__ o,
                                                               const uint16_t* __restrict__ dout,
                                                               const float* __restrict__ lse,
                                                               float* __restrict__ ws, int B, int Nq,
                                                               int Hq, int Nq_pad,
                                                               const int* __restrict__ cu_q = nullptr,
                                                               int total_q = 0) {
  static_assert(G == 8 || G == 16 || G == 32, "d = 64, 128 or 256");
  constexpr int D = G * 8;
  constexpr int GROUPS = 256 / G;  // lane groups per block
  const int grp = threadIdx.x / G;
  const int sub = threadIdx.x % G;
  const long long rows_pad = static_cast<long long>(B) * Hq * Nq_pad;
  uint4 ov[RPG], gv[RPG];
  long long row[RPG];
  bool live[RPG];
  long long grow_[RPG];  // row of O / dO / LSE: (b, i) dense, cu_q[b] + i packed
#pragma unroll
  for (int k = 0; k < RPG; ++k) {
    row[k] = (static_cast<long long>(blockIdx.x) * RPG + k) * GROUPS + grp;
    const int i = static_cast<int>(row[k] % Nq_pad);
    const long long bh = row[k] / Nq_pad;
    live[k] = row[k] < rows_pad && i < Nq;
    grow_[k] = (bh / Hq) * Nq + i;
    if (VL && live[k]) {
      const int b = static_cast<int>(bh / Hq);
      const int q0 = __ldg(cu_q + b);
      grow_[k] = static_cast<long long>(q0) + i;
      live[k] = i < __ldg(cu_q + b + 1) - q0 && grow_[k] >= 0 && grow_[k] < total_q;
    }
    if (live[k]) {
      const size_t base = (static_cast<size_t>(grow_[k]) * Hq + bh % Hq) * D + sub * 8;
      ov[k] = __ldg(reinterpret_cast<const uint4*>(o + base));
      gv[k] = __ldg(reinterpret_cast<const uint4*>(dout + base));
    }
  }
#pragma unroll
  for (int k = 0; k < RPG; ++k) {
    float acc = 0.f;
    if (live[k]) {
      const uint32_t* op = reinterpret_cast<const uint32_t*>(&ov[k]);
      const uint32_t* gp = reinterpret_cast<const uint32_t*>(&gv[k]);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        acc = fmaf(h16_to_f32<F16>(op[u] & 0xFFFFu), h16_to_f32<F16>(gp[u] & 0xFFFFu), acc);
        acc = fmaf(h16_to_f32<F16>(op[u] >> 16), h16_to_f32<F16>(gp[u] >> 16), acc);
      }
    }
#pragma unroll
    for (int off = G / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (sub == 0 && row[k] < rows_pad) {
      if (!live[k]) {  // padding row: D = 0 and lse2 = +inf, so every P there is 0
        ws[row[k]] = 0.f;
        ws[rows_pad + row[k]] = INFINITY;
      } else {
        ws[row[k]] = acc;
        // LSE is [B, Hq, Nq] dense, [Hq, total_q] packed
        const long long bh = row[k] / Nq_pad;
        const float L = VL ? lse[(bh % Hq) * static_cast<long long>(total_q) + grow_[k]]
                                        : lse[bh * Nq + row[k] % Nq_pad];
        // a row with no visible key (LSE = -inf) has P = 0 everywhere
        ws[rows_pad + row[k]] = (L == -INFINITY) ? INFINITY : L * kLog2e;
      }
    }
  }
}

struct BwdParams {
  int B, Nq, Nk, Hq, Hkv, group;
  float scale;        // softmax scale (dQ, dK carry it)
  float scale_log2;   // scale * log2(e)
  MaskSpec mask;
  int Nq_pad;
  const float* D;     // [B, Hq, Nq_pad]
  const float* lse2;  // [B, Hq, Nq_pad]
  int n_qgroups;      // dq kernel: CTAs along the query axis
  int n_kvtiles;      // dkdv kernel: CTAs along the key axis
  int head_chunk;     // dq kernel: heads per scheduling chunk
  int head_chunk_kv;  // dkdv kernel: key/value heads per scheduling chunk
  // packed sequences (null when dense): sequence b is query rows [cu_q[b],
  // cu_q[b+1]) and key rows [cu_k[b], cu_k[b+1]) of one-batch tensors; Nq / Nk
  // are then the longest lengths, and D / lse2 stay [B, Hq, Nq_pad] (rows past
  // a sequence's end are padding: D = 0, lse2 = +inf)
  const int* cu_q;
  const int* cu_k;
  int total_q, total_k;
  uint16_t* dq;  // outputs, for the plain stores of a packed sequence's last tile
  uint16_t* dk;
  uint16_t* dv;
  // block-sparse (BS kernels): a byte per 128 x 128 (query block, key block)
  // of batch b, query head h at bmask + b * bm_sb + h * bm_sh, rows of
  // bm_cols key blocks; zero = the block is skipped
  const uint8_t* bmask;
  long long bm_sb, bm_sh;
  int bm_cols;
  unsigned long long wait_limit_ns;
};

// =====================================================================
// 2. dQ: query-stationary
// =====================================================================
template <int D_, int NQT_, int BN_, int KST_>
struct DqCfg {
  static constexpr bool F16 = false;  // elements are bf16 (AsF16<> flips it to fp16)
  static constexpr int D = D_, NQT = NQT_, BN = BN_, KST = KST_;
  static constexpr int BM = 128;
  static constexpr bool ONE_TILE = false;
  static constexpr int NCHUNK = D / 64;
  static constexpr int QCHUNK = BM * 128;
  static constexpr int KCHUNK = BN * 128;
  static constexpr int QTILE = NCHUNK * QCHUNK;
  static constexpr int KTILE = NCHUNK * KCHUNK;
  static constexpr int OFF_Q = 0;                             // Q tiles  [NQT]
  static constexpr int OFF_DO = OFF_Q + NQT * QTILE;          // dO tiles [NQT]
  static constexpr int OFF_K = OFF_DO + NQT * QTILE;          // K stages [KST]
  static constexpr int OFF_V = OFF_K + KST * KTILE;           // V stages [KST]
  static constexpr int OFF_BAR = OFF_V + KST * KTILE;
  static constexpr int NBAR = 1 + 2 * KST + 2 * NQT + 1 + 1;  // q_full, kv_full/empty, sp_full/ds_full, dq_done, drain
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr int NWARPS = 4 * NQT + 2;
  static constexpr int NTHREADS = 32 * NWARPS;
  static constexpr int TMA_WARP = 4 * NQT;
  static constexpr int MMA_WARP = 4 * NQT + 1;
  // TMEM: tile t: S at t*2*BN, dP at t*2*BN + BN (dS overlays dP's first BN/2), dQ at 2*BN*NQT + t*D
  static constexpr int COL_DQ = 2 * BN * NQT;
  static constexpr int TMEM_USED = COL_DQ + NQT * D;
  static constexpr int TMEM_COLS = TMEM_USED <= 128 ? 128 : TMEM_USED <= 256 ? 256 : 512;
  static_assert(TMEM_USED <= 512, "TMEM budget");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

template <class C, bool VL = false, bool BS = false>
__global__ void __launch_bounds__(C::NTHREADS, 1)
    fa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                     const __grid_constant__ CUtensorMap tm_dq, const BwdParams p) {
  constexpr int D = C::D, NQT = C::NQT, BN = C::BN, KST = C::KST, BM = C::BM;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + KST;
  uint64_t* sp_full = kv_empty + KST;  // [NQT]
  uint64_t* ds_full = sp_full + NQT;   // [NQT]
  uint64_t* dq_done = ds_full + NQT;
  uint64_t* bar_drain = dq_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  const uint32_t sQ = sbase + C::OFF_Q, sdO = sbase + C::OFF_DO, sK = sbase + C::OFF_K,
                 sV = sbase + C::OFF_V;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  // heaviest query groups first within L2-sized chunks of heads
  const ChunkedOrder order(blockIdx.x, p.B * p.Hq, p.n_qgroups, p.head_chunk);
  const int bh = order.head;
  const int g = p.n_qgroups - 1 - order.rank;
  const int b = bh / p.Hq, h = bh % p.Hq, hk = h / p.group;
  const int r0 = g * NQT * BM;
  const SeqView sq(p.mask, VL ? p.cu_q : nullptr, p.cu_k, b);
  const int nq = sq.mask.Nq;
  if (VL && r0 >= nq) return;  // this packed sequence has no query group g
  const int r_last = min(nq - 1, r0 + NQT * BM - 1);
  const int key_lo = sq.mask.lo(r0), key_hi = sq.mask.hi(r_last);
  const int j_begin = key_lo / BN;
  int n_kv = (key_hi >= key_lo) ? (key_hi / BN - j_begin + 1) : 0;
  // block-sparse: the key tiles of that range whose mask block is set for
  // this query block, listed by the TMA warp before the block-wide sync
  uint32_t* tile_list = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC + 16);
  volatile int* list_count = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);
  if constexpr (BS) {
    if (warp == C::TMA_WARP) {
      const uint8_t* mrow = p.bmask + b * p.bm_sb + h * p.bm_sh + static_cast<long long>(r0 / 128) * p.bm_cols;
      const int cnt = warp_compact(n_kv, tile_list, [&](int it) { return __ldg(mrow + (j_begin + it) * BN / 128) != 0; });
      if (lane == 0) *list_count = cnt;
      __syncwarp();
    }
  }
  auto tile_of = [&](int it) {
    if constexpr (BS)
      return j_begin + static_cast<int>(tile_list[it]);
    else
      return j_begin + it;
  };

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < KST; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int t = 0; t < NQT; ++t) {
      mbar_init(&sp_full[t], 1);
      mbar_init(&ds_full[t], BM);
    }
    mbar_init(dq_done, 1);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
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
    if (lane == 0 && n_kv > 0) {
      mbar_expect_tx(q_full, 2 * NQT * C::QTILE);
      for (int t = 0; t < NQT; ++t)
        for (int c = 0; c < C::NCHUNK; ++c) {
          tma_load_4d(sQ + t * C::QTILE + c * C::QCHUNK, &tm_q, q_full, c * 64, h, sq.q_off + r0 + t * BM, sq.tb);
          tma_load_4d(sdO + t * C::QTILE + c * C::QCHUNK, &tm_do, q_full, c * 64, h, sq.q_off + r0 + t * BM, sq.tb);
        }
      int n_issued = 0;
      for (int it = 0; it < n_kv; ++it) {
        const int s = it % KST, use = it / KST;
        const int krow = tile_of(it) * BN;
        if (use > 0 && !mbar_wait(&kv_empty[s], (use - 1) & 1, abort_flag, &g_status, p.wait_limit_ns))
          break;
        mbar_expect_tx(&kv_full[s], 2 * C::KTILE);
        for (int c = 0; c < C::NCHUNK; ++c) {
          tma_load_4d(sK + s * C::KTILE + c * C::KCHUNK, &tm_k, &kv_full[s], c * 64, hk, sq.k_off + krow, sq.tb);
          tma_load_4d(sV + s * C::KTILE + c * C::KCHUNK, &tm_v, &kv_full[s], c * 64, hk, sq.k_off + krow, sq.tb);
        }
        ++n_issued;
      }
      mbar_drain(q_full, 0, p.wait_limit_ns);
      for (int s = 0; s < KST; ++s)
        if (n_issued > s) mbar_drain(&kv_full[s], ((n_issued - 1 - s) / KST) & 1, p.wait_limit_ns);
    }
  } else if (warp == C::MMA_WARP) {
    if (lane == 0 && n_kv > 0) {
      constexpr uint32_t ID_S = idesc_kind_f16<C::F16>(128, BN, false, false);
      constexpr uint32_t ID_DQ = idesc_kind_f16<C::F16>(128, D, false, true);
      auto wait = [&](uint64_t* bar, uint32_t par) {
        const bool ok = mbar_wait(bar, par, abort_flag, &g_status, p.wait_limit_ns);
        tc_fence_after();
        return ok;
      };
      // Descriptors are built once; each MMA adds a compile-time offset (in
      // 16-byte units).  The issuing thread has to keep ahead of the tensor
      // core, so it does little besides issuing.
      const uint64_t dq_q = sdesc_sw128(sQ, 16, 1024), dq_do = sdesc_sw128(sdO, 16, 1024);
      const uint64_t dq_k = sdesc_sw128(sK, 16, 1024), dq_v = sdesc_sw128(sV, 16, 1024);
      const uint64_t dq_kmn = sdesc_sw128(sK, C::KCHUNK, 1024);
      // S_t = Q_t K_s^T and dP_t = dO_t V_s^T
      auto issue_sdp = [&](int t, int s) {
        const uint32_t d_s = tmem + t * 2 * BN, d_dp = d_s + BN;
        const uint64_t qa = dq_q + static_cast<uint64_t>((t * C::QTILE) >> 4);
        const uint64_t da = dq_do + static_cast<uint64_t>((t * C::QTILE) >> 4);
        const uint64_t kb = dq_k + static_cast<uint64_t>((s * C::KTILE) >> 4);
        const uint64_t vb = dq_v + static_cast<uint64_t>((s * C::KTILE) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t qo = ((kk >> 2) * C::QCHUNK + (kk & 3) * 32) >> 4;
          const uint32_t ko = ((kk >> 2) * C::KCHUNK + (kk & 3) * 32) >> 4;
          mma_ss(d_s, qa + qo, kb + ko, ID_S, kk > 0);
          mma_ss(d_dp, da + qo, vb + ko, ID_S, kk > 0);
        }
      };
      // dQ_t (+)= dS_t K_s, dS from TMEM (bf16 over dP_t), K as MN-major B
      auto issue_dq = [&](int t, int s, bool acc) {
        const uint32_t d_dq = tmem + C::COL_DQ + t * D;
        const uint32_t a_ds = tmem + t * 2 * BN + BN;
        const uint64_t kb = dq_kmn + static_cast<uint64_t>((s * C::KTILE) >> 4);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          mma_ts(d_dq, a_ds + kk * 8, kb + static_cast<uint64_t>(kk * 128), ID_DQ,
                 (acc || kk > 0) ? 1u : 0u);
      };
      bool ok = wait(q_full, 0) && wait(&kv_full[0], 0);
      if (ok) {
        for (int t = 0; t < NQT; ++t) {
          issue_sdp(t, 0);
          tc_commit(&sp_full[t]);
        }
        for (int it = 0; it < n_kv && ok; ++it) {
          const int s = it % KST, s1 = (it + 1) % KST;
          const bool more = it + 1 < n_kv;
          for (int t = 0; t < NQT && ok; ++t) {
            if (!(ok = wait(&ds_full[t], it & 1))) break;
            // with two or more stages the next key tile's wait shares this
            // wait point; with one stage it has to follow this tile's release
            if (KST > 1 && t == 0 && more && !(ok = wait(&kv_full[s1], ((it + 1) / KST) & 1))) break;
            issue_dq(t, s, it > 0);
            if (t == NQT - 1) tc_commit(&kv_empty[s]);
            if (more) {
              if (KST == 1 && t == 0 && !(ok = wait(&kv_full[s1], ((it + 1) / KST) & 1))) break;
              issue_sdp(t, s1);
              tc_commit(&sp_full[t]);
            }
          }
        }
        tc_commit(dq_done);
      }
    }
    if (lane == 0) {
      tc_commit(bar_drain);
      mbar_drain(bar_drain, 0, p.wait_limit_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ dS warpgroups (thread = query row)
    const int t = warp / 4;
    const int r = threadIdx.x % BM;
    const int row = r0 + t * BM + r;
    const int lo = sq.mask.lo(row), hi = sq.mask.hi(row);
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp % 4) * 32) << 16);
    const size_t srow = (static_cast<size_t>(b) * p.Hq + h) * p.Nq_pad + row;  // row < Nq_pad
    const float lse2 = p.lse2[srow];
    const float Drow = p.D[srow];
    const float sl2 = p.scale_log2;
    bool ok = true;
    for (int it = 0; it < n_kv; ++it) {
      ok = mbar_wait(&sp_full[t], it & 1, abort_flag, &g_status, p.wait_limit_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      uint32_t sv[BN], dv[BN];
      const uint32_t col_s = t * 2 * BN, col_dp = col_s + BN;
#pragma unroll
      for (int cc = 0; cc < BN / 32; ++cc) {
        tmem_ld_x32(lane_base + col_s + cc * 32, &sv[cc * 32]);
        tmem_ld_x32(lane_base + col_dp + cc * 32, &dv[cc * 32]);
      }
#pragma unroll
      for (int cc = 0; cc < BN / 32; ++cc) {
        tmem_ld_wait_x32(&sv[cc * 32]);
        tmem_ld_wait_x32(&dv[cc * 32]);
      }
      float* sc = reinterpret_cast<float*>(sv);
      const float* dp = reinterpret_cast<const float*>(dv);
      const int k0 = tile_of(it) * BN;
      if (k0 < lo || k0 + BN - 1 > hi) {
#pragma unroll
        for (int c = 0; c < BN; ++c) {
          const int key = k0 + c;
          if (key < lo || key > hi) sc[c] = -INFINITY;
        }
      }
      uint32_t pk[BN / 2];
#pragma unroll
      for (int c = 0; c < BN; c += 2) {
        const float p0 = ex2_approx(fmaf(sc[c], sl2, -lse2));
        const float p1 = ex2_approx(fmaf(sc[c + 1], sl2, -lse2));
        pk[c / 2] = pack2<C::F16>(p0 * (dp[c] - Drow), p1 * (dp[c + 1] - Drow));
      }
#pragma unroll
      for (int cc = 0; cc < BN / 64; ++cc) tmem_st_x32(lane_base + col_dp + cc * 32, &pk[cc * 32]);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&ds_full[t]);
    }
    if (ok && n_kv > 0) {
      ok = mbar_wait(dq_done, 0, abort_flag, &g_status, p.wait_limit_ns);
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
    }
    // epilogue: dQ * scale -> bf16 -> shared (this tile's Q buffer) -> TMA store
    const uint32_t stage = sQ + t * C::QTILE;
    if (ok) {
#pragma unroll 1
      for (int c = 0; c < C::NCHUNK; ++c) {
        uint32_t ov[64];
        if (n_kv > 0) {
          tmem_ld_x32(lane_base + C::COL_DQ + t * D + c * 64, ov);
          tmem_ld_x32(lane_base + C::COL_DQ + t * D + c * 64 + 32, ov + 32);
          tmem_ld_wait_x32(ov);
          tmem_ld_wait_x32(ov + 32);
        } else {
#pragma unroll
          for (int i = 0; i < 64; ++i) ov[i] = 0u;
        }
        const float sc = p.scale;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float* f = reinterpret_cast<const float*>(ov + 8 * u);
          st_shared_v4(stage + c * C::QCHUNK + sw128_offset(r, u), pack2<C::F16>(f[0] * sc, f[1] * sc),
                       pack2<C::F16>(f[2] * sc, f[3] * sc), pack2<C::F16>(f[4] * sc, f[5] * sc),
                       pack2<C::F16>(f[6] * sc, f[7] * sc));
        }
      }
      fence_proxy_async_smem();
    }
    named_bar_sync(1 + t, BM);
    const int t_row0 = r0 + t * BM;
    if (!VL || t_row0 + BM <= nq) {
      if (r == 0 && *abort_flag == 0 && t_row0 < nq) {
        for (int c = 0; c < C::NCHUNK; ++c)
          tma_store_4d(&tm_dq, stage + c * C::QCHUNK, c * 64, h, sq.q_off + t_row0, sq.tb);
        tma_store_commit();
        tma_store_wait_read();
      }
    } else if (*abort_flag == 0) {  // last tile of a packed sequence
      store_rows_sw128(stage, C::QCHUNK, nq - t_row0, D, p.dq, sq.q_off + t_row0, p.total_q, p.Hq, h, D, 0, r,
                       BM);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == C::MMA_WARP) tmem_dealloc(tmem, C::TMEM_COLS);
}

// =====================================================================
// 2b. dQ, one 128-row query tile per CTA, 128-key tiles (d <= 128)
// =====================================================================
// S = Q K_j^T and dP = dO V_j^T land in TMEM (N = 128, so the shared-memory
// operand traffic matches the tensor core).  Both warpgroups read them (each
// owns 64 of the 128 key columns of every row) and release them at once, so
// S/dP of the next key tile are computed while dS of this one is formed.  dS
// (bf16) goes to its own TMEM columns and feeds dQ += dS K_j as the A operand.
// K is needed first (S) and last (dQ), V only for dP, so K gets the deeper
// ring: each tile's loads are issued two steps ahead of their use.
template <int D_, int KS_, int VS_, int NPOLY_ = 0>
struct Dq2Cfg {
  static constexpr bool F16 = false;  // elements are bf16 (AsF16<> flips it to fp16)
  static constexpr int D = D_, KS = KS_, VS = VS_;
  // of every 8 exponential pairs of an unmasked tile, NPOLY take exp2 on the
  // FMA pipe (exp2_poly_pair).  0 by default: here the FMA work slows the
  // MMA issue more than the MUFU unit limits the warpgroups (timed at 0-4).
  static constexpr int NPOLY = NPOLY_;
  static constexpr int BM = 128, BN = 128;
  static constexpr int NQT = 1;
  static constexpr bool ONE_TILE = true;
  // the next key tile's K stage must be free before this tile's dQ is issued
  static_assert(KS >= 2 && VS >= 2, "needs at least two K and two V stages");
  static constexpr int NCHUNK = D / 64;
  static constexpr int QCHUNK = BM * 128;
  static constexpr int KCHUNK = BN * 128;
  static constexpr int QTILE = NCHUNK * QCHUNK;
  static constexpr int KTILE = NCHUNK * KCHUNK;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_DO = OFF_Q + QTILE;
  static constexpr int OFF_K = OFF_DO + QTILE;                // K stages [KS]
  static constexpr int OFF_V = OFF_K + KS * KTILE;            // V stages [VS]
  static constexpr int OFF_BAR = OFF_V + VS * KTILE;
  // q_full, k_full/k_empty[KS], v_full/v_empty[VS], sp_full, sp_free, ds_full, ds_free, dq_done, drain
  static constexpr int NBAR = 1 + 2 * KS + 2 * VS + 6;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr int NWARPS = 10;
  static constexpr int NTHREADS = 32 * NWARPS;
  static constexpr int TMA_WARP = 8, MMA_WARP = 9;
  // TMEM: S, dP (fp32), dQ (fp32), dS (bf16 pairs: 64 columns)
  static constexpr int COL_S = 0, COL_DP = BN, COL_DQ = 2 * BN, COL_DS = 2 * BN + D;
  static constexpr int TMEM_USED = COL_DS + BN / 2;
  static constexpr int TMEM_COLS = TMEM_USED <= 256 ? 256 : 512;
  static_assert(TMEM_USED <= 512, "TMEM budget");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// dS of 64 score columns of one query row, bf16 pairs into pk[0 .. 32):
// P = 2^(s * scale_log2 - lse2), dS = P (dP - D), on packed fp32 pairs.  nl2 and
// nD hold (-lse2, -lse2) and (-D, -D).  EDGE: masked (-inf) scores or a row
// with no visible key (lse2 = +inf) may be present, so MUFU ex2 only (exact
// zeros); otherwise NPOLY of every 8 pairs use exp2_poly_pair.
template <class C, bool EDGE>
__device__ __forceinline__ void dq_ds64(const uint32_t* sv, const uint32_t* dv, uint64_t sl2x2, uint64_t nl2,
                                        uint64_t nD, uint32_t* pk) {
#pragma unroll
  for (int c = 0; c < 64; c += 2) {
    const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])), sl2x2, nl2);
    float p0, p1;
    if (!EDGE && (c / 2) % 8 < C::NPOLY) {
      exp2_poly_pair(x2, p0, p1);
    } else {
      float x0, x1;
      f2_unpack(x2, x0, x1);
      p0 = ex2_approx(x0);
      p1 = ex2_approx(x1);
    }
    float d0, d1;
    f2_unpack(f2_mul(f2_pack(p0, p1), f2_add(f2_pack(__uint_as_float(dv[c]), __uint_as_float(dv[c + 1])), nD)), d0,
              d1);
    pk[c / 2] = pack2<C::F16>(d0, d1);
  }
}

template <class C, bool VL = false, bool BS = false>
__global__ void __launch_bounds__(C::NTHREADS, 1)
    fa_bwd_dq2_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                      const __grid_constant__ CUtensorMap tm_dq, const BwdParams p) {
  constexpr int D = C::D, BN = C::BN, KS = C::KS, VS = C::VS, BM = C::BM;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + KS;
  uint64_t* v_full = k_empty + KS;
  uint64_t* v_empty = v_full + VS;
  uint64_t* sp_full = v_empty + VS;
  uint64_t* sp_free = sp_full + 1;
  uint64_t* ds_full = sp_free + 1;
  uint64_t* ds_free = ds_full + 1;
  uint64_t* dq_done = ds_free + 1;
  uint64_t* bar_drain = dq_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  const uint32_t sQ = sbase + C::OFF_Q, sdO = sbase + C::OFF_DO, sK = sbase + C::OFF_K,
                 sV = sbase + C::OFF_V;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  const ChunkedOrder order(blockIdx.x, p.B * p.Hq, p.n_qgroups, p.head_chunk);
  const int bh = order.head;
  const int g = p.n_qgroups - 1 - order.rank;  // query tile, latest first
  const int b = bh / p.Hq, h = bh % p.Hq, hk = h / p.group;
  const int r0 = g * BM;
  const SeqView sq(p.mask, VL ? p.cu_q : nullptr, p.cu_k, b);
  const int nq = sq.mask.Nq;
  if (VL && r0 >= nq) return;  // this packed sequence has no query tile g
  const int r_last = min(nq - 1, r0 + BM - 1);
  const int key_lo = sq.mask.lo(r0), key_hi = sq.mask.hi(r_last);
  const int j_begin = key_lo / BN;
  int n_kv = (key_hi >= key_lo) ? (key_hi / BN - j_begin + 1) : 0;
  // block-sparse: the key tiles of that range whose mask block is set for
  // this query tile, listed by the TMA warp before the block-wide sync
  uint32_t* tile_list = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC + 16);
  volatile int* list_count = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);
  if constexpr (BS) {
    if (warp == C::TMA_WARP) {
      const uint8_t* mrow = p.bmask + b * p.bm_sb + h * p.bm_sh + static_cast<long long>(r0 / 128) * p.bm_cols;
      n_kv = warp_compact(n_kv, tile_list, [&](int it) { return __ldg(mrow + (j_begin + it) * BN / 128) != 0; });
      if (lane == 0) *list_count = n_kv;
      __syncwarp();
    }
  }
  auto tile_of = [&](int it) {
    if constexpr (BS)
      return j_begin + static_cast<int>(tile_list[it]);
    else
      return j_begin + it;
  };

  // copies of K or V of key tile `it` into their rings
  auto load_k = [&](int it) {
    const int sk = it % KS, krow = tile_of(it) * BN;
    mbar_expect_tx(&k_full[sk], C::KTILE);
    for (int c = 0; c < C::NCHUNK; ++c)
      tma_load_4d(sK + sk * C::KTILE + c * C::KCHUNK, &tm_k, &k_full[sk], c * 64, hk, sq.k_off + krow, sq.tb);
  };
  auto load_v = [&](int it) {
    const int sv = it % VS, krow = tile_of(it) * BN;
    mbar_expect_tx(&v_full[sv], C::KTILE);
    for (int c = 0; c < C::NCHUNK; ++c)
      tma_load_4d(sV + sv * C::KTILE + c * C::KCHUNK, &tm_v, &v_full[sv], c * 64, hk, sq.k_off + krow, sq.tb);
  };
  // The TMA thread sets up the barriers and issues Q, dO and the first ring
  // stages (nothing to wait for yet) before the block-wide sync.
  const int n_pre_k = min(n_kv, KS), n_pre_v = min(n_kv, VS);
  if (warp == C::TMA_WARP && lane == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < KS; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < VS; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    mbar_init(sp_full, 1);
    mbar_init(sp_free, 256);
    mbar_init(ds_full, 256);
    mbar_init(ds_free, 1);
    mbar_init(dq_done, 1);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    if (n_kv > 0) {
      mbar_expect_tx(q_full, 2 * C::QTILE);
      for (int c = 0; c < C::NCHUNK; ++c) {
        tma_load_4d(sQ + c * C::QCHUNK, &tm_q, q_full, c * 64, h, sq.q_off + r0, sq.tb);
        tma_load_4d(sdO + c * C::QCHUNK, &tm_do, q_full, c * 64, h, sq.q_off + r0, sq.tb);
      }
      for (int it = 0; it < n_pre_k; ++it) load_k(it);
      for (int it = 0; it < n_pre_v; ++it) load_v(it);
    }
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
    if (lane == 0 && n_kv > 0) {
      int nk = n_pre_k, nv = n_pre_v;
      for (int it = 0; it < n_kv; ++it) {
        if (it >= n_pre_k) {
          const int sk = it % KS, uk = it / KS;
          if (!mbar_wait(&k_empty[sk], (uk - 1) & 1, abort_flag, &g_status, p.wait_limit_ns)) break;
          load_k(it);
          ++nk;
        }
        if (it >= n_pre_v) {
          const int sv = it % VS, uv = it / VS;
          if (!mbar_wait(&v_empty[sv], (uv - 1) & 1, abort_flag, &g_status, p.wait_limit_ns)) break;
          load_v(it);
          ++nv;
        }
      }
      mbar_drain(q_full, 0, p.wait_limit_ns);
      for (int s = 0; s < KS; ++s)
        if (nk > s) mbar_drain(&k_full[s], ((nk - 1 - s) / KS) & 1, p.wait_limit_ns);
      for (int s = 0; s < VS; ++s)
        if (nv > s) mbar_drain(&v_full[s], ((nv - 1 - s) / VS) & 1, p.wait_limit_ns);
    }
  } else if (warp == C::MMA_WARP) {
    if (lane == 0 && n_kv > 0) {
      constexpr uint32_t ID_S = idesc_kind_f16<C::F16>(128, BN, false, false);
      constexpr uint32_t ID_DQ = idesc_kind_f16<C::F16>(128, D, false, true);
      auto wait = [&](uint64_t* bar, uint32_t par) {
        const bool ok = mbar_wait(bar, par, abort_flag, &g_status, p.wait_limit_ns);
        tc_fence_after();
        return ok;
      };
      const uint64_t dq_q = sdesc_sw128(sQ, 16, 1024), dq_do = sdesc_sw128(sdO, 16, 1024);
      const uint64_t dq_k = sdesc_sw128(sK, 16, 1024), dq_v = sdesc_sw128(sV, 16, 1024);
      const uint64_t dq_kmn = sdesc_sw128(sK, C::KCHUNK, 1024);
      // S = Q K^T, dP = dO V^T for key tile it
      auto issue_sdp = [&](int it) {
        const uint64_t kb = dq_k + static_cast<uint64_t>(((it % KS) * C::KTILE) >> 4);
        const uint64_t vb = dq_v + static_cast<uint64_t>(((it % VS) * C::KTILE) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t qo = ((kk >> 2) * C::QCHUNK + (kk & 3) * 32) >> 4;
          const uint32_t ko = ((kk >> 2) * C::KCHUNK + (kk & 3) * 32) >> 4;
          mma_ss(tmem + C::COL_S, dq_q + qo, kb + ko, ID_S, kk > 0);
          mma_ss(tmem + C::COL_DP, dq_do + qo, vb + ko, ID_S, kk > 0);
        }
      };
      // dQ (+)= dS K: dS from TMEM, K as MN-major B
      auto issue_dq = [&](int it) {
        const uint64_t kb = dq_kmn + static_cast<uint64_t>(((it % KS) * C::KTILE) >> 4);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          mma_ts(tmem + C::COL_DQ, tmem + C::COL_DS + kk * 8, kb + static_cast<uint64_t>(kk * 128), ID_DQ,
                 (it > 0 || kk > 0) ? 1u : 0u);
      };
      bool ok = wait(q_full, 0) && wait(&k_full[0], 0) && wait(&v_full[0], 0);
      if (ok) {
        issue_sdp(0);
        tc_commit(sp_full);
        tc_commit(&v_empty[0]);
        for (int it = 0; it < n_kv && ok; ++it) {
          if (it + 1 < n_kv) {
            const int nx = it + 1;
            // the next key tile's S/dP as soon as both warpgroups have read this one's
            if (!(ok = wait(sp_free, it & 1))) break;
            if (!(ok = wait(&k_full[nx % KS], (nx / KS) & 1))) break;
            if (!(ok = wait(&v_full[nx % VS], (nx / VS) & 1))) break;
            issue_sdp(nx);
            tc_commit(sp_full);
            tc_commit(&v_empty[nx % VS]);
          }
          if (!(ok = wait(ds_full, it & 1))) break;
          issue_dq(it);
          tc_commit(ds_free);
          tc_commit(&k_empty[it % KS]);
        }
        if (ok) tc_commit(dq_done);
      }
    }
    if (lane == 0) {
      tc_commit(bar_drain);
      mbar_drain(bar_drain, 0, p.wait_limit_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------- dS warpgroups (thread = query row)
    const int wg = warp / 4;          // key columns [64 wg, 64 wg + 64) of every tile
    const int r = threadIdx.x % BM;   // row == TMEM lane
    const int row = r0 + r;
    const int lo = sq.mask.lo(row), hi = sq.mask.hi(row);
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp % 4) * 32) << 16);
    const size_t srow = (static_cast<size_t>(b) * p.Hq + h) * p.Nq_pad + row;  // row < Nq_pad
    const float lse2 = p.lse2[srow];
    const float Drow = p.D[srow];
    const uint64_t sl2x2 = f2_pack(p.scale_log2, p.scale_log2);
    const uint64_t nl2 = f2_pack(-lse2, -lse2), nD = f2_pack(-Drow, -Drow);
    // a row with no visible key (or a padding row) has lse2 = +inf: P = 0
    const bool dead = lse2 == INFINITY;
    bool ok = true;
    for (int it = 0; it < n_kv; ++it) {
      ok = mbar_wait(sp_full, it & 1, abort_flag, &g_status, p.wait_limit_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      uint32_t sv[64], dv[64];
      tmem_ld_x32(lane_base + C::COL_S + wg * 64, sv);
      tmem_ld_x32(lane_base + C::COL_S + wg * 64 + 32, sv + 32);
      tmem_ld_x32(lane_base + C::COL_DP + wg * 64, dv);
      tmem_ld_x32(lane_base + C::COL_DP + wg * 64 + 32, dv + 32);
      tmem_ld_wait_x32(sv);
      tmem_ld_wait_x32(sv + 32);
      tmem_ld_wait_x32(dv);
      tmem_ld_wait_x32(dv + 32);
      tc_fence_before();
      mbar_arrive(sp_free);  // S/dP may now be overwritten by the next key tile
      const int k0 = tile_of(it) * BN + wg * 64;
      const bool masked = k0 < lo || k0 + 63 > hi;
      uint32_t pk[32];
      if (masked || dead) {
        if (masked) {
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            const int key = k0 + c;
            if (key < lo || key > hi) sv[c] = __float_as_uint(-INFINITY);
          }
        }
        dq_ds64<C, true>(sv, dv, sl2x2, nl2, nD, pk);
      } else {
        dq_ds64<C, false>(sv, dv, sl2x2, nl2, nD, pk);
      }
      // the previous key tile's dQ MMA must be done reading dS
      if (it > 0) {
        ok = mbar_wait(ds_free, (it - 1) & 1, abort_flag, &g_status, p.wait_limit_ns);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
      }
      tmem_st_x32(lane_base + C::COL_DS + wg * 32, pk);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(ds_full);
    }
    if (ok && n_kv > 0) {
      ok = mbar_wait(dq_done, 0, abort_flag, &g_status, p.wait_limit_ns);
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
    }
    // epilogue: dQ * scale -> bf16 -> shared (the Q buffer) -> TMA store;
    // warpgroup wg stages the 64-column chunks wg, wg + 2, ...
    if (ok) {
#pragma unroll 1
      for (int c = wg; c < C::NCHUNK; c += 2) {
        uint32_t ov[64];
        if (n_kv > 0) {
          tmem_ld_x32(lane_base + C::COL_DQ + c * 64, ov);
          tmem_ld_x32(lane_base + C::COL_DQ + c * 64 + 32, ov + 32);
          tmem_ld_wait_x32(ov);
          tmem_ld_wait_x32(ov + 32);
        } else {
#pragma unroll
          for (int i = 0; i < 64; ++i) ov[i] = 0u;
        }
        const float sc = p.scale;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float* f = reinterpret_cast<const float*>(ov + 8 * u);
          st_shared_v4(sQ + c * C::QCHUNK + sw128_offset(r, u), pack2<C::F16>(f[0] * sc, f[1] * sc),
                       pack2<C::F16>(f[2] * sc, f[3] * sc), pack2<C::F16>(f[4] * sc, f[5] * sc),
                       pack2<C::F16>(f[6] * sc, f[7] * sc));
        }
      }
      fence_proxy_async_smem();
    }
    named_bar_sync(1, 256);
    if (!VL || r0 + BM <= nq) {
      if (threadIdx.x == 0 && *abort_flag == 0 && r0 < nq) {
        for (int c = 0; c < C::NCHUNK; ++c)
          tma_store_4d(&tm_dq, sQ + c * C::QCHUNK, c * 64, h, sq.q_off + r0, sq.tb);
        tma_store_commit();
        tma_store_wait_read();
      }
    } else if (*abort_flag == 0) {  // last tile of a packed sequence
      store_rows_sw128(sQ, C::QCHUNK, nq - r0, D, p.dq, sq.q_off + r0, p.total_q, p.Hq, h, D, 0, threadIdx.x, 256);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == C::MMA_WARP) tmem_dealloc(tmem, C::TMEM_COLS);
}

// =====================================================================
// 3. dK, dV: key-stationary
// =====================================================================
// D: head dim; DV: the slice of d whose dK/dV this CTA accumulates (D, or
// 128 for D = 256, then blockIdx.y picks the slice); BM: query tile; ST: ring
// depth of the (Q, dO, lse2, D) stages; LA: steps issued ahead (<= 2, <= ST).
template <int D_, int DV_, int BM_, int ST_>
struct DkvCfg {
  static constexpr bool F16 = false;  // elements are bf16 (AsF16<> flips it to fp16)
  static constexpr bool WIDE = false;
  static constexpr int D = D_, DV = DV_, BM = BM_, ST = ST_;
  static constexpr int BN = 128;
  static constexpr int LA = ST >= 2 ? 2 : 1;
  static constexpr int NCHUNK = D / 64;
  static constexpr int KCHUNK = BN * 128;
  static constexpr int QCHUNK = BM * 128;
  static constexpr int KTILE = NCHUNK * KCHUNK;
  static constexpr int QTILE = NCHUNK * QCHUNK;
  static constexpr int STAGE = 2 * QTILE;   // Q, dO (swizzled, 1 KiB aligned)
  static constexpr int SSTAGE = 2 * BM * 4;  // lse2, D of the same step
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + KTILE;
  static constexpr int OFF_ST = OFF_V + KTILE;
  static constexpr int OFF_STAT = OFF_ST + ST * STAGE;
  static constexpr int OFF_BAR = OFF_STAT + ST * SSTAGE;
  static constexpr int NBAR = 1 + 2 * ST + 2 + 2 + 1 + 1;  // kv_full, q_full/q_empty, sp_full[2], ds_full[2], acc_done, drain
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  // two P^T/dS^T warpgroups take alternate steps (one per TMEM slot)
  static constexpr int NWARPS = 10;
  static constexpr int NTHREADS = 32 * NWARPS;
  static constexpr int TMA_WARP = 8, MMA_WARP = 9;
  // TMEM: dK [0, DV), dV [DV, 2DV), slot u: S^T at 2DV + u*2BM, dP^T at +BM
  static constexpr int COL_DK = 0, COL_DV = DV, COL_SLOT = 2 * DV;
  static constexpr int TMEM_USED = 2 * DV + 4 * BM;
  static constexpr int TMEM_COLS = TMEM_USED <= 128 ? 128 : TMEM_USED <= 256 ? 256 : 512;
  static_assert(TMEM_USED <= 512, "TMEM budget");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(STAGE % 1024 == 0, "stages stay 1 KiB aligned");
};

template <class C, bool VL = false, bool BS = false>
__global__ void __launch_bounds__(C::NTHREADS, 1)
    fa_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                       const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                       const BwdParams p) {
  constexpr int D = C::D, DV = C::DV, BM = C::BM, BN = C::BN, ST = C::ST, LA = C::LA;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* kv_full = bars;
  uint64_t* q_full = bars + 1;
  uint64_t* q_empty = q_full + ST;
  uint64_t* sp_full = q_empty + ST;  // [2]
  uint64_t* ds_full = sp_full + 2;   // [2]
  uint64_t* acc_done = ds_full + 2;
  uint64_t* bar_drain = acc_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  const uint32_t sK = sbase + C::OFF_K, sV = sbase + C::OFF_V, sSt = sbase + C::OFF_ST;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  // ---- work unit: (b, hk), key tile j, d slice: the heaviest key tiles (the
  // earliest, for causal) first within L2-sized chunks of head groups
  const ChunkedOrder order(blockIdx.x, p.B * p.Hkv, p.n_kvtiles, p.head_chunk_kv);
  const int bhk = order.head;
  const int j = order.rank;
  const int b = bhk / p.Hkv, hk = bhk % p.Hkv;
  const int dslice = blockIdx.y;  // which DV-wide slice of d
  const int k0 = j * BN;
  const SeqView sq(p.mask, VL ? p.cu_q : nullptr, p.cu_k, b);
  const int nq = sq.mask.Nq, nk = sq.mask.Nk;
  if (VL && k0 >= nk) return;  // this packed sequence has no key tile j
  const int k1 = min(nk - 1, k0 + BN - 1);
  // queries that see some key of this tile: i in [q_lo(k0), q_hi(k1)]
  const int delta = sq.mask.delta();
  int q_lo = (sq.mask.wr < 0) ? 0 : k0 - delta - sq.mask.wr;
  int q_hi = (sq.mask.wl < 0) ? nq - 1 : k1 - delta + sq.mask.wl;
  q_lo = max(q_lo, 0);
  q_hi = min(q_hi, nq - 1);
  const int i_begin = q_lo / BM;
  const int n_qt = (q_hi >= q_lo) ? (q_hi / BM - i_begin + 1) : 0;
  int n_steps = n_qt * p.group;  // (query head in group) x (query tile)
  // block-sparse: the steps whose (query head, query block) mask block is set
  // for this key block, listed by the TMA warp before the block-wide sync
  uint32_t* step_list = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC + 16);
  volatile int* list_count = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);
  if constexpr (BS) {
    if (warp == C::TMA_WARP) {
      const uint8_t* mb = p.bmask + b * p.bm_sb + k0 / 128;
      n_steps = warp_compact(n_steps, step_list, [&](int st) {
        const int hq = hk * p.group + st / n_qt, qb = (i_begin + st % n_qt) * BM / 128;
        return __ldg(mb + hq * p.bm_sh + static_cast<long long>(qb) * p.bm_cols) != 0;
      });
      if (lane == 0) *list_count = n_steps;
      __syncwarp();
    }
  }
  auto step_of = [&](int it) {
    if constexpr (BS)
      return static_cast<int>(step_list[it]);
    else
      return it;
  };
  auto step_head = [&](int it) { return hk * p.group + step_of(it) / n_qt; };
  auto step_q0 = [&](int it) { return (i_begin + step_of(it) % n_qt) * BM; };
  // copies of step `it` (Q, dO and their lse2 / D rows) into stage it % ST
  auto load_step = [&](int it) {
    const int s = it % ST;
    const int hq = step_head(it), q0 = step_q0(it);
    const uint32_t st = sSt + s * C::STAGE;
    mbar_expect_tx(&q_full[s], C::STAGE + C::SSTAGE);
    for (int c = 0; c < C::NCHUNK; ++c) {
      tma_load_4d(st + c * C::QCHUNK, &tm_q, &q_full[s], c * 64, hq, sq.q_off + q0, sq.tb);
      tma_load_4d(st + C::QTILE + c * C::QCHUNK, &tm_do, &q_full[s], c * 64, hq, sq.q_off + q0, sq.tb);
    }
    const size_t srow = (static_cast<size_t>(b) * p.Hq + hq) * p.Nq_pad + q0;
    const uint32_t stat = sbase + C::OFF_STAT + s * C::SSTAGE;
    bulk_load(stat, p.lse2 + srow, BM * 4, &q_full[s]);
    bulk_load(stat + BM * 4, p.D + srow, BM * 4, &q_full[s]);
  };
  // The TMA thread sets up the barriers and issues K, V and the first ST
  // steps (no stage to wait for yet) before the block-wide sync, so the
  // copies overlap the TMEM allocation and the sync.
  const int n_pre = min(n_steps, ST);
  if (warp == C::TMA_WARP && lane == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
    }
    for (int u = 0; u < 2; ++u) {
      mbar_init(&sp_full[u], 1);
      mbar_init(&ds_full[u], BN);
    }
    mbar_init(acc_done, 1);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    if (n_steps > 0) {
      mbar_expect_tx(kv_full, 2 * C::KTILE);
      for (int c = 0; c < C::NCHUNK; ++c) {
        tma_load_4d(sK + c * C::KCHUNK, &tm_k, kv_full, c * 64, hk, sq.k_off + k0, sq.tb);
        tma_load_4d(sV + c * C::KCHUNK, &tm_v, kv_full, c * 64, hk, sq.k_off + k0, sq.tb);
      }
      for (int it = 0; it < n_pre; ++it) load_step(it);
    }
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(smem_addr(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if constexpr (BS) n_steps = *list_count;

  if (warp == C::TMA_WARP) {
    if (lane == 0 && n_steps > 0) {
      int n_issued = n_pre;
      for (int it = n_pre; it < n_steps; ++it) {
        const int s = it % ST, use = it / ST;
        if (!mbar_wait(&q_empty[s], (use - 1) & 1, abort_flag, &g_status, p.wait_limit_ns)) break;
        load_step(it);
        ++n_issued;
      }
      mbar_drain(kv_full, 0, p.wait_limit_ns);
      for (int s = 0; s < ST; ++s)
        if (n_issued > s) mbar_drain(&q_full[s], ((n_issued - 1 - s) / ST) & 1, p.wait_limit_ns);
    }
  } else if (warp == C::MMA_WARP) {
    if (lane == 0 && n_steps > 0) {
      constexpr uint32_t ID_S = idesc_kind_f16<C::F16>(128, BM, false, false);
      constexpr uint32_t ID_ACC = idesc_kind_f16<C::F16>(128, DV, false, true);
      auto wait = [&](uint64_t* bar, uint32_t par) {
        const bool ok = mbar_wait(bar, par, abort_flag, &g_status, p.wait_limit_ns);
        tc_fence_after();
        return ok;
      };
      // Descriptors built once; each MMA adds a compile-time offset.
      const uint64_t dk_k = sdesc_sw128(sK, 16, 1024), dk_v = sdesc_sw128(sV, 16, 1024);
      const uint64_t dk_st = sdesc_sw128(sSt, 16, 1024);                // Q / dO, K-major B
      const uint64_t dk_stmn = sdesc_sw128(sSt + dslice * (DV / 64) * C::QCHUNK, C::QCHUNK, 1024);
      // slot u: S^T = K Q^T, dP^T = V dO^T (M = keys, N = queries)
      auto issue_sdp = [&](int u, int s) {
        const uint32_t d_s = tmem + C::COL_SLOT + u * 2 * BM, d_dp = d_s + BM;
        const uint64_t qb = dk_st + static_cast<uint64_t>((s * C::STAGE) >> 4);
        const uint64_t dob = qb + static_cast<uint64_t>(C::QTILE >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t kofs = ((kk >> 2) * C::KCHUNK + (kk & 3) * 32) >> 4;
          const uint32_t qofs = ((kk >> 2) * C::QCHUNK + (kk & 3) * 32) >> 4;
          mma_ss(d_s, dk_k + kofs, qb + qofs, ID_S, kk > 0);
          mma_ss(d_dp, dk_v + kofs, dob + qofs, ID_S, kk > 0);
        }
      };
      // dV += P^T dO, dK += dS^T Q (A from TMEM, B MN-major over this CTA's d slice)
      auto issue_acc = [&](int u, int s, bool acc) {
        const uint32_t a_p = tmem + C::COL_SLOT + u * 2 * BM, a_ds = a_p + BM;
        const uint64_t qb = dk_stmn + static_cast<uint64_t>((s * C::STAGE) >> 4);
        const uint64_t dob = qb + static_cast<uint64_t>(C::QTILE >> 4);
#pragma unroll
        for (int kk = 0; kk < BM / 16; ++kk) {
          const uint32_t acc_k = (acc || kk > 0) ? 1u : 0u;
          mma_ts(tmem + C::COL_DV, a_p + kk * 8, dob + static_cast<uint64_t>(kk * 128), ID_ACC, acc_k);
          mma_ts(tmem + C::COL_DK, a_ds + kk * 8, qb + static_cast<uint64_t>(kk * 128), ID_ACC, acc_k);
        }
      };
      bool ok = wait(kv_full, 0);
      for (int u = 0; u < LA && u < n_steps && ok; ++u) {
        if (!(ok = wait(&q_full[u % ST], (u / ST) & 1))) break;
        issue_sdp(u & 1, u % ST);
        tc_commit(&sp_full[u & 1]);
      }
      for (int it = 0; it < n_steps && ok; ++it) {
        const int u = it & 1, s = it % ST;
        const int nx = it + LA;
        if (!(ok = wait(&ds_full[u], (it >> 1) & 1))) break;
        // with a deep enough ring the next step's operands share this wait point
        if (nx < n_steps && LA < ST && !(ok = wait(&q_full[nx % ST], (nx / ST) & 1))) break;
        issue_acc(u, s, it > 0);
        tc_commit(&q_empty[s]);
        if (nx < n_steps) {
          if (LA >= ST && !(ok = wait(&q_full[nx % ST], (nx / ST) & 1))) break;
          issue_sdp(nx & 1, nx % ST);
          tc_commit(&sp_full[nx & 1]);
        }
      }
      if (ok) tc_commit(acc_done);
    }
    if (lane == 0) {
      tc_commit(bar_drain);
      mbar_drain(bar_drain, 0, p.wait_limit_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ P^T / dS^T warpgroups (thread = key row)
    const int wg = warp / 4;           // handles the steps of TMEM slot wg
    const int r = threadIdx.x % 128;   // TMEM lane == key within the tile
    const int key = k0 + r;
    // queries that see this key: [kq_lo, kq_hi]
    const int kq_lo = (sq.mask.wr < 0) ? -0x3fffffff : key - delta - sq.mask.wr;
    const int kq_hi = (sq.mask.wl < 0) ? 0x3fffffff : key - delta + sq.mask.wl;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp % 4) * 32) << 16);
    const float sl2 = p.scale_log2;
    bool ok = true;
    for (int it = wg; it < n_steps; it += 2) {
      const int u = it & 1, s = it % ST;
      ok = mbar_wait(&sp_full[u], (it >> 1) & 1, abort_flag, &g_status, p.wait_limit_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      // the stage's lse2 / D landed with the same barrier the MMA already waited on
      ok = mbar_wait(&q_full[s], (it / ST) & 1, abort_flag, &g_status, p.wait_limit_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t col_s = C::COL_SLOT + u * 2 * BM, col_dp = col_s + BM;
      const float* lse2 = reinterpret_cast<const float*>(smem + C::OFF_STAT + s * C::SSTAGE);
      const float* Dv = lse2 + BM;
      const int q0 = step_q0(it);
      const bool need_mask = (q0 < kq_lo) || (q0 + BM - 1 > kq_hi);
      // all of this step's S^T and dP^T columns come in with one wait
      uint32_t sv[BM], dv[BM];
#pragma unroll
      for (int cc = 0; cc < BM / 32; ++cc) {
        tmem_ld_x32(lane_base + col_s + cc * 32, &sv[cc * 32]);
        tmem_ld_x32(lane_base + col_dp + cc * 32, &dv[cc * 32]);
      }
#pragma unroll
      for (int cc = 0; cc < BM / 32; ++cc) {
        tmem_ld_wait_x32(&sv[cc * 32]);
        tmem_ld_wait_x32(&dv[cc * 32]);
      }
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < BM; ++c) {
          const int qi = q0 + c;
          if (qi < kq_lo || qi > kq_hi) sv[c] = __float_as_uint(-INFINITY);
        }
      }
      const float4* lse4 = reinterpret_cast<const float4*>(lse2);
      const float4* d4 = reinterpret_cast<const float4*>(Dv);
      uint32_t pp[BM / 2], dd[BM / 2];
#pragma unroll
      for (int c = 0; c < BM; c += 4) {
        const float4 l4 = lse4[c / 4], D4 = d4[c / 4];
        const float p0 = ex2_approx(fmaf(__uint_as_float(sv[c]), sl2, -l4.x));
        const float p1 = ex2_approx(fmaf(__uint_as_float(sv[c + 1]), sl2, -l4.y));
        const float p2 = ex2_approx(fmaf(__uint_as_float(sv[c + 2]), sl2, -l4.z));
        const float p3 = ex2_approx(fmaf(__uint_as_float(sv[c + 3]), sl2, -l4.w));
        pp[c / 2] = pack2<C::F16>(p0, p1);
        pp[c / 2 + 1] = pack2<C::F16>(p2, p3);
        dd[c / 2] = pack2<C::F16>(p0 * (__uint_as_float(dv[c]) - D4.x), p1 * (__uint_as_float(dv[c + 1]) - D4.y));
        dd[c / 2 + 1] =
            pack2<C::F16>(p2 * (__uint_as_float(dv[c + 2]) - D4.z), p3 * (__uint_as_float(dv[c + 3]) - D4.w));
      }
#pragma unroll
      for (int cc = 0; cc < BM / 32; ++cc) {
        tmem_st_x16(lane_base + col_s + cc * 16, &pp[cc * 16]);
        tmem_st_x16(lane_base + col_dp + cc * 16, &dd[cc * 16]);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&ds_full[u]);
    }
    if (ok && n_steps > 0) {
      ok = mbar_wait(acc_done, 0, abort_flag, &g_status, p.wait_limit_ns);
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
    }
    // epilogue: warpgroup 0 stages dK * scale, warpgroup 1 stages dV, as bf16 in
    // the K and V buffers; one thread then issues the TMA stores
    if (ok) {
      {
        const uint32_t col = (wg == 0) ? C::COL_DK : C::COL_DV;
        const uint32_t stage = (wg == 0) ? sK : sV;
        const float sc = (wg == 0) ? p.scale : 1.f;
#pragma unroll 1
        for (int c = 0; c < DV / 64; ++c) {
          uint32_t ov[64];
          if (n_steps > 0) {
            tmem_ld_x32(lane_base + col + c * 64, ov);
            tmem_ld_x32(lane_base + col + c * 64 + 32, ov + 32);
            tmem_ld_wait_x32(ov);
            tmem_ld_wait_x32(ov + 32);
          } else {
#pragma unroll
            for (int i = 0; i < 64; ++i) ov[i] = 0u;
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const float* f = reinterpret_cast<const float*>(ov + 8 * u);
            st_shared_v4(stage + c * C::KCHUNK + sw128_offset(r, u), pack2<C::F16>(f[0] * sc, f[1] * sc),
                         pack2<C::F16>(f[2] * sc, f[3] * sc), pack2<C::F16>(f[4] * sc, f[5] * sc),
                         pack2<C::F16>(f[6] * sc, f[7] * sc));
          }
        }
      }
      fence_proxy_async_smem();
    }
    named_bar_sync(1, 256);
    if (!VL || k0 + BN <= nk) {
      if (threadIdx.x == 0 && *abort_flag == 0) {
        for (int c = 0; c < DV / 64; ++c) {
          const int x = (dslice * (DV / 64) + c) * 64;
          tma_store_4d(&tm_dk, sK + c * C::KCHUNK, x, hk, sq.k_off + k0, sq.tb);
          tma_store_4d(&tm_dv, sV + c * C::KCHUNK, x, hk, sq.k_off + k0, sq.tb);
        }
        tma_store_commit();
        tma_store_wait_read();
      }
    } else if (*abort_flag == 0) {  // last key tile of a packed sequence
      store_rows_sw128(sK, C::KCHUNK, nk - k0, DV, p.dk, sq.k_off + k0, p.total_k, p.Hkv, hk, D, dslice * DV,
                       threadIdx.x, 256);
      store_rows_sw128(sV, C::KCHUNK, nk - k0, DV, p.dv, sq.k_off + k0, p.total_k, p.Hkv, hk, D, dslice * DV,
                       threadIdx.x, 256);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == C::MMA_WARP) tmem_dealloc(tmem, C::TMEM_COLS);
}

// =====================================================================
// 3b. dK, dV in steps of 128 query rows (d = 64, 128)
// =====================================================================
// The work of fa_bwd_dkdv_kernel in steps of 128 query rows instead of 64.
// S^T and dP^T then are N = 128 MMAs, which run at the tensor core's full
// rate (an M = 128, K = 16 MMA with N = 64 takes about 1.3 times its share of
// the time), and a step issues half as many MMAs.  TMEM holds one step: dK
// [0, d), dV [d, 2d), S^T [2d, 2d + 128), dP^T [2d + 128, 2d + 256).  Both warpgroups
// work on the same step, warpgroup g on query columns [64 g, 64 g + 64); each
// writes its P^T and dS^T (bf16 pairs, 32 columns each) over the S^T and dP^T
// columns it has read.  Per step the tensor core runs dV += P^T dO as soon as
// every P^T is in place, the next step's S^T, dK += dS^T Q once every dS^T is
// in place, and the next step's dP^T (the MMAs of one CTA run in issue order,
// so S^T and dP^T overwrite the columns dV and dK read only after them); dK
// and dP^T run while the warpgroups compute the next step's P^T.  The
// warpgroups' exponentials are on the step's critical path: in an unmasked
// step NPOLY of every 8 pairs are computed on the FMA pipe (exp2_poly_pair)
// beside the MUFU unit.
template <int D_, int ST_, int NPOLY_>
struct DkvWCfg {
  static constexpr bool F16 = false;  // elements are bf16 (AsF16<> flips it to fp16)
  static constexpr bool WIDE = true;
  static constexpr int D = D_, DV = D_, BM = 128, ST = ST_, NPOLY = NPOLY_;
  static constexpr int BN = 128;
  static constexpr int NCHUNK = D / 64;
  static constexpr int KCHUNK = BN * 128;
  static constexpr int QCHUNK = BM * 128;
  static constexpr int KTILE = NCHUNK * KCHUNK;
  static constexpr int QTILE = NCHUNK * QCHUNK;
  static constexpr int STAGE = 2 * QTILE;    // Q, dO (swizzled, 1 KiB aligned)
  static constexpr int SSTAGE = 2 * BM * 4;  // lse2, D of the same step
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + KTILE;
  static constexpr int OFF_ST = OFF_V + KTILE;
  static constexpr int OFF_STAT = OFF_ST + ST * STAGE;
  static constexpr int OFF_BAR = OFF_STAT + ST * SSTAGE;
  static constexpr int NBAR = 1 + 2 * ST + 6;  // kv_full, q_full/q_empty, s_full, dp_full, p_full, ds_full, acc_done, drain
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr int NWARPS = 10;
  static constexpr int NTHREADS = 32 * NWARPS;
  static constexpr int TMA_WARP = 8, MMA_WARP = 9;
  static constexpr int COL_DK = 0, COL_DV = DV, COL_S = 2 * DV, COL_DP = COL_S + BM;
  static constexpr int TMEM_COLS = 512;
  static_assert(D == 64 || D == 128, "one step of S^T and dP^T beside dK and dV fits TMEM up to d = 128");
  static_assert(COL_DP + BM <= TMEM_COLS, "TMEM budget");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(STAGE % 1024 == 0, "stages stay 1 KiB aligned");
};

// P^T of 32 columns [C0, C0 + 32) of one key row: 2^(s * scale_log2 - lse2),
// the fp32 values over s (dS^T needs them), bf16 pairs into pk[C0 / 2 ..].
// EDGE: masked (-inf) scores or padding rows (lse2 = +inf) may be present, so
// MUFU ex2 only (exact zeros); otherwise NPOLY of every 8 pairs use
// exp2_poly_pair.
template <class C, int C0, bool EDGE>
__device__ __forceinline__ void dkdv_p32(uint32_t* sv, const float4* lse4, uint64_t sl2x2, uint32_t* pk) {
#pragma unroll
  for (int c = C0; c < C0 + 32; c += 4) {
    const float4 l4 = lse4[c / 4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int cc = c + 2 * h;
      const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(sv[cc]), __uint_as_float(sv[cc + 1])), sl2x2,
                                 h == 0 ? f2_pack(-l4.x, -l4.y) : f2_pack(-l4.z, -l4.w));
      float p0, p1;
      if (!EDGE && (cc / 2) % 8 < C::NPOLY) {
        exp2_poly_pair(x2, p0, p1);
      } else {
        float x0, x1;
        f2_unpack(x2, x0, x1);
        p0 = ex2_approx(x0);
        p1 = ex2_approx(x1);
      }
      sv[cc] = __float_as_uint(p0);
      sv[cc + 1] = __float_as_uint(p1);
      pk[cc / 2] = pack2<C::F16>(p0, p1);
    }
  }
}

// dS^T = P^T (dP^T - D) of 32 columns [C0, C0 + 32), bf16 pairs into pk[C0 / 2 ..]
template <class C, int C0>
__device__ __forceinline__ void dkdv_ds32(const uint32_t* pv, const uint32_t* dv, const float4* d4, uint32_t* pk) {
#pragma unroll
  for (int c = C0; c < C0 + 32; c += 4) {
    const float4 D4 = d4[c / 4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int cc = c + 2 * h;
      const uint64_t t = f2_add(f2_pack(__uint_as_float(dv[cc]), __uint_as_float(dv[cc + 1])),
                                h == 0 ? f2_pack(-D4.x, -D4.y) : f2_pack(-D4.z, -D4.w));
      float d0, d1;
      f2_unpack(f2_mul(f2_pack(__uint_as_float(pv[cc]), __uint_as_float(pv[cc + 1])), t), d0, d1);
      pk[cc / 2] = pack2<C::F16>(d0, d1);
    }
  }
}

template <class C, bool VL = false, bool BS = false>
__global__ void __launch_bounds__(C::NTHREADS, 1)
    fa_bwd_dkdv_wide_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                            const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                            const BwdParams p) {
  constexpr int D = C::D, DV = C::DV, BM = C::BM, BN = C::BN, ST = C::ST;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* kv_full = bars;
  uint64_t* q_full = bars + 1;
  uint64_t* q_empty = q_full + ST;
  uint64_t* s_full = q_empty + ST;
  uint64_t* dp_full = s_full + 1;
  uint64_t* p_full = dp_full + 1;
  uint64_t* ds_full = p_full + 1;
  uint64_t* acc_done = ds_full + 1;
  uint64_t* bar_drain = acc_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  const uint32_t sK = sbase + C::OFF_K, sV = sbase + C::OFF_V, sSt = sbase + C::OFF_ST;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  // ---- work unit: as in fa_bwd_dkdv_kernel (one d slice: DV = D)
  const ChunkedOrder order(blockIdx.x, p.B * p.Hkv, p.n_kvtiles, p.head_chunk_kv);
  const int bhk = order.head;
  const int j = order.rank;
  const int b = bhk / p.Hkv, hk = bhk % p.Hkv;
  const int k0 = j * BN;
  const SeqView sq(p.mask, VL ? p.cu_q : nullptr, p.cu_k, b);
  const int nq = sq.mask.Nq, nk = sq.mask.Nk;
  if (VL && k0 >= nk) return;  // this packed sequence has no key tile j
  const int k1 = min(nk - 1, k0 + BN - 1);
  const int delta = sq.mask.delta();
  int q_lo = (sq.mask.wr < 0) ? 0 : k0 - delta - sq.mask.wr;
  int q_hi = (sq.mask.wl < 0) ? nq - 1 : k1 - delta + sq.mask.wl;
  q_lo = max(q_lo, 0);
  q_hi = min(q_hi, nq - 1);
  const int i_begin = q_lo / BM;
  const int n_qt = (q_hi >= q_lo) ? (q_hi / BM - i_begin + 1) : 0;
  int n_steps = n_qt * p.group;  // (query head in group) x (query tile)
  uint32_t* step_list = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC + 16);
  volatile int* list_count = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);
  if constexpr (BS) {
    if (warp == C::TMA_WARP) {
      const uint8_t* mb = p.bmask + b * p.bm_sb + k0 / 128;
      n_steps = warp_compact(n_steps, step_list, [&](int st) {
        const int hq = hk * p.group + st / n_qt, qb = (i_begin + st % n_qt) * BM / 128;
        return __ldg(mb + hq * p.bm_sh + static_cast<long long>(qb) * p.bm_cols) != 0;
      });
      if (lane == 0) *list_count = n_steps;
      __syncwarp();
    }
  }
  auto step_of = [&](int it) {
    if constexpr (BS)
      return static_cast<int>(step_list[it]);
    else
      return it;
  };
  auto step_head = [&](int it) { return hk * p.group + step_of(it) / n_qt; };
  auto step_q0 = [&](int it) { return (i_begin + step_of(it) % n_qt) * BM; };
  auto load_step = [&](int it) {
    const int s = it % ST;
    const int hq = step_head(it), q0 = step_q0(it);
    const uint32_t st = sSt + s * C::STAGE;
    mbar_expect_tx(&q_full[s], C::STAGE + C::SSTAGE);
    for (int c = 0; c < C::NCHUNK; ++c) {
      tma_load_4d(st + c * C::QCHUNK, &tm_q, &q_full[s], c * 64, hq, sq.q_off + q0, sq.tb);
      tma_load_4d(st + C::QTILE + c * C::QCHUNK, &tm_do, &q_full[s], c * 64, hq, sq.q_off + q0, sq.tb);
    }
    const size_t srow = (static_cast<size_t>(b) * p.Hq + hq) * p.Nq_pad + q0;
    const uint32_t stat = sbase + C::OFF_STAT + s * C::SSTAGE;
    bulk_load(stat, p.lse2 + srow, BM * 4, &q_full[s]);
    bulk_load(stat + BM * 4, p.D + srow, BM * 4, &q_full[s]);
  };
  const int n_pre = min(n_steps, ST);
  if (warp == C::TMA_WARP && lane == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_full, 2 * 128);
    mbar_init(ds_full, 2 * 128);
    mbar_init(acc_done, 1);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    if (n_steps > 0) {
      mbar_expect_tx(kv_full, 2 * C::KTILE);
      for (int c = 0; c < C::NCHUNK; ++c) {
        tma_load_4d(sK + c * C::KCHUNK, &tm_k, kv_full, c * 64, hk, sq.k_off + k0, sq.tb);
        tma_load_4d(sV + c * C::KCHUNK, &tm_v, kv_full, c * 64, hk, sq.k_off + k0, sq.tb);
      }
      for (int it = 0; it < n_pre; ++it) load_step(it);
    }
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(smem_addr(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if constexpr (BS) n_steps = *list_count;

  if (warp == C::TMA_WARP) {
    if (lane == 0 && n_steps > 0) {
      int n_issued = n_pre;
      for (int it = n_pre; it < n_steps; ++it) {
        const int s = it % ST, use = it / ST;
        if (!mbar_wait(&q_empty[s], (use - 1) & 1, abort_flag, &g_status, p.wait_limit_ns)) break;
        load_step(it);
        ++n_issued;
      }
      mbar_drain(kv_full, 0, p.wait_limit_ns);
      for (int s = 0; s < ST; ++s)
        if (n_issued > s) mbar_drain(&q_full[s], ((n_issued - 1 - s) / ST) & 1, p.wait_limit_ns);
    }
  } else if (warp == C::MMA_WARP) {
    if (lane == 0 && n_steps > 0) {
      constexpr uint32_t ID_S = idesc_kind_f16<C::F16>(128, BM, false, false);
      constexpr uint32_t ID_ACC = idesc_kind_f16<C::F16>(128, DV, false, true);
      auto wait = [&](uint64_t* bar, uint32_t par) {
        const bool ok = mbar_wait(bar, par, abort_flag, &g_status, p.wait_limit_ns);
        tc_fence_after();
        return ok;
      };
      const uint64_t dk_k = sdesc_sw128(sK, 16, 1024), dk_v = sdesc_sw128(sV, 16, 1024);
      const uint64_t dk_st = sdesc_sw128(sSt, 16, 1024);             // Q / dO, K-major B
      const uint64_t dk_stmn = sdesc_sw128(sSt, C::QCHUNK, 1024);    // Q / dO, MN-major B
      // S^T = K Q^T and dP^T = V dO^T (M = keys, N = the step's 128 queries)
      auto issue_s = [&](int s) {
        const uint64_t qb = dk_st + static_cast<uint64_t>((s * C::STAGE) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t kofs = ((kk >> 2) * C::KCHUNK + (kk & 3) * 32) >> 4;
          const uint32_t qofs = ((kk >> 2) * C::QCHUNK + (kk & 3) * 32) >> 4;
          mma_ss(tmem + C::COL_S, dk_k + kofs, qb + qofs, ID_S, kk > 0);
        }
      };
      auto issue_dp = [&](int s) {
        const uint64_t dob = dk_st + static_cast<uint64_t>((s * C::STAGE + C::QTILE) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t kofs = ((kk >> 2) * C::KCHUNK + (kk & 3) * 32) >> 4;
          const uint32_t qofs = ((kk >> 2) * C::QCHUNK + (kk & 3) * 32) >> 4;
          mma_ss(tmem + C::COL_DP, dk_v + kofs, dob + qofs, ID_S, kk > 0);
        }
      };
      // 16-query chunk kk of P^T / dS^T: warpgroup kk / 4's columns, pair kk % 4
      auto a_col = [](int kk) { return 64 * (kk >> 2) + 8 * (kk & 3); };
      auto issue_dv = [&](int s, bool acc) {  // dV += P^T dO
        const uint64_t dob = dk_stmn + static_cast<uint64_t>((s * C::STAGE + C::QTILE) >> 4);
#pragma unroll
        for (int kk = 0; kk < BM / 16; ++kk)
          mma_ts(tmem + C::COL_DV, tmem + C::COL_S + a_col(kk), dob + static_cast<uint64_t>(kk * 128), ID_ACC,
                 (acc || kk > 0) ? 1u : 0u);
      };
      auto issue_dk = [&](int s, bool acc) {  // dK += dS^T Q
        const uint64_t qb = dk_stmn + static_cast<uint64_t>((s * C::STAGE) >> 4);
#pragma unroll
        for (int kk = 0; kk < BM / 16; ++kk)
          mma_ts(tmem + C::COL_DK, tmem + C::COL_DP + a_col(kk), qb + static_cast<uint64_t>(kk * 128), ID_ACC,
                 (acc || kk > 0) ? 1u : 0u);
      };
      // Order per step: dV(it) once P^T(it) is in place, S^T(it + 1), dK(it)
      // once dS^T(it) is, dP^T(it + 1).  S^T(it + 1) overwrites the columns
      // dV(it) reads and dP^T(it + 1) those dK(it) reads, each after them in
      // issue order; dK(it) and dP^T(it + 1) run while the warpgroups compute
      // P^T(it + 1), which needs only S^T(it + 1).
      bool ok = wait(kv_full, 0) && wait(&q_full[0], 0);
      if (ok) {
        issue_s(0);
        tc_commit(s_full);
        issue_dp(0);
        tc_commit(dp_full);
      }
      for (int it = 0; it < n_steps && ok; ++it) {
        const int s = it % ST, nx = it + 1;
        if (!(ok = wait(p_full, it & 1))) break;
        issue_dv(s, it > 0);
        if (nx < n_steps) {
          if (!(ok = wait(&q_full[nx % ST], (nx / ST) & 1))) break;
          issue_s(nx % ST);
          tc_commit(s_full);
        }
        if (!(ok = wait(ds_full, it & 1))) break;
        issue_dk(s, it > 0);
        tc_commit(&q_empty[s]);
        if (nx < n_steps) {
          issue_dp(nx % ST);
          tc_commit(dp_full);
        }
      }
      if (ok) tc_commit(acc_done);
    }
    if (lane == 0) {
      tc_commit(bar_drain);
      mbar_drain(bar_drain, 0, p.wait_limit_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ P^T / dS^T warpgroups (thread = key row)
    const int g = warp / 4;            // query columns [64 g, 64 g + 64) of every step
    const int r = threadIdx.x % 128;   // TMEM lane == key within the tile
    const int key = k0 + r;
    const int kq_lo = (sq.mask.wr < 0) ? -0x3fffffff : key - delta - sq.mask.wr;
    const int kq_hi = (sq.mask.wl < 0) ? 0x3fffffff : key - delta + sq.mask.wl;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp % 4) * 32) << 16);
    const uint64_t sl2x2 = f2_pack(p.scale_log2, p.scale_log2);
    const uint32_t col_s = C::COL_S + 64 * g, col_dp = C::COL_DP + 64 * g;
    bool ok = true;
    for (int it = 0; it < n_steps; ++it) {
      const int s = it % ST;
      ok = mbar_wait(s_full, it & 1, abort_flag, &g_status, p.wait_limit_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      // the stage's lse2 / D landed with the barrier the MMA thread waited on
      ok = mbar_wait(&q_full[s], (it / ST) & 1, abort_flag, &g_status, p.wait_limit_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const float* stat = reinterpret_cast<const float*>(smem + C::OFF_STAT + s * C::SSTAGE);
      const float4* lse4 = reinterpret_cast<const float4*>(stat + 64 * g);
      const float4* d4 = reinterpret_cast<const float4*>(stat + BM + 64 * g);
      const int c0 = step_q0(it) + 64 * g;  // query of column 0
      const bool need_mask = (c0 < kq_lo) || (c0 + 63 > kq_hi);
      // masked scores and padding rows (lse2 = +inf) must take the MUFU exp2
      const bool edge = need_mask || (c0 + 64 > nq);
      // S^T in two 32-column halves (the second in flight during the first's
      // exponentials); dP^T the same way once P^T is handed over
      uint32_t sv[64], dv[64], pk[32];
      auto mask32 = [&](int h) {
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int qi = c0 + 32 * h + c;
          if (qi < kq_lo || qi > kq_hi) sv[32 * h + c] = __float_as_uint(-INFINITY);
        }
      };
      tmem_ld_x32(lane_base + col_s, sv);
      tmem_ld_wait_x32(sv);
      tmem_ld_x32(lane_base + col_s + 32, sv + 32);
      if (edge) {
        if (need_mask) mask32(0);
        dkdv_p32<C, 0, true>(sv, lse4, sl2x2, pk);
      } else {
        dkdv_p32<C, 0, false>(sv, lse4, sl2x2, pk);
      }
      tmem_ld_wait_x32(sv + 32);
      if (edge) {
        if (need_mask) mask32(1);
        dkdv_p32<C, 32, true>(sv, lse4, sl2x2, pk);
      } else {
        dkdv_p32<C, 32, false>(sv, lse4, sl2x2, pk);
      }
      tmem_st_x16(lane_base + col_s, pk);
      tmem_st_x16(lane_base + col_s + 16, pk + 16);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(p_full);
      ok = mbar_wait(dp_full, it & 1, abort_flag, &g_status, p.wait_limit_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      tmem_ld_x32(lane_base + col_dp, dv);
      tmem_ld_wait_x32(dv);
      tmem_ld_x32(lane_base + col_dp + 32, dv + 32);
      dkdv_ds32<C, 0>(sv, dv, d4, pk);
      tmem_ld_wait_x32(dv + 32);
      dkdv_ds32<C, 32>(sv, dv, d4, pk);
      tmem_st_x16(lane_base + col_dp, pk);
      tmem_st_x16(lane_base + col_dp + 16, pk + 16);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(ds_full);
    }
    if (ok && n_steps > 0) {
      ok = mbar_wait(acc_done, 0, abort_flag, &g_status, p.wait_limit_ns);
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
    }
    // epilogue: warpgroup 0 stages dK * scale, warpgroup 1 stages dV, as bf16 in
    // the K and V buffers; one thread then issues the TMA stores
    if (ok) {
      const uint32_t col = (g == 0) ? C::COL_DK : C::COL_DV;
      const uint32_t stage = (g == 0) ? sK : sV;
      const float sc = (g == 0) ? p.scale : 1.f;
#pragma unroll 1
      for (int c = 0; c < DV / 64; ++c) {
        uint32_t ov[64];
        if (n_steps > 0) {
          tmem_ld_x32(lane_base + col + c * 64, ov);
          tmem_ld_x32(lane_base + col + c * 64 + 32, ov + 32);
          tmem_ld_wait_x32(ov);
          tmem_ld_wait_x32(ov + 32);
        } else {
#pragma unroll
          for (int i = 0; i < 64; ++i) ov[i] = 0u;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float* f = reinterpret_cast<const float*>(ov + 8 * u);
          st_shared_v4(stage + c * C::KCHUNK + sw128_offset(r, u), pack2<C::F16>(f[0] * sc, f[1] * sc),
                       pack2<C::F16>(f[2] * sc, f[3] * sc), pack2<C::F16>(f[4] * sc, f[5] * sc),
                       pack2<C::F16>(f[6] * sc, f[7] * sc));
        }
      }
      fence_proxy_async_smem();
    }
    named_bar_sync(1, 256);
    if (!VL || k0 + BN <= nk) {
      if (threadIdx.x == 0 && *abort_flag == 0) {
        for (int c = 0; c < DV / 64; ++c) {
          tma_store_4d(&tm_dk, sK + c * C::KCHUNK, c * 64, hk, sq.k_off + k0, sq.tb);
          tma_store_4d(&tm_dv, sV + c * C::KCHUNK, c * 64, hk, sq.k_off + k0, sq.tb);
        }
        tma_store_commit();
        tma_store_wait_read();
      }
    } else if (*abort_flag == 0) {  // last key tile of a packed sequence
      store_rows_sw128(sK, C::KCHUNK, nk - k0, DV, p.dk, sq.k_off + k0, p.total_k, p.Hkv, hk, D, 0,
                       threadIdx.x, 256);
      store_rows_sw128(sV, C::KCHUNK, nk - k0, DV, p.dv, sq.k_off + k0, p.total_k, p.Hkv, hk, D, 0,
                       threadIdx.x, 256);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == C::MMA_WARP) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace fa
