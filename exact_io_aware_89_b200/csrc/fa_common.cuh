// fa_common.cuh -- shared definitions of the sm_100a attention kernels.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "sm100_ptx.cuh"

namespace fa {

// per-device status word (kDevOk / kDevTimeout), read by fa_get_device_status.
// The library is a single translation unit, so the definition lives here.
__device__ int g_status = 0;

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// The visible key range of query row i: [lo, hi] (inclusive).  The causal
// diagonal is aligned bottom-right (delta = Nk - Nq); a negative window bound
// is unbounded.  Returns lo > hi when nothing is visible.
struct MaskSpec {
  int Nq, Nk;
  int wl, wr;  // wr = 0 when causal
  __host__ __device__ int delta() const { return Nk - Nq; }
  __host__ __device__ int lo(int i) const {
    if (wl < 0) return 0;
    int x = i + delta() - wl;
    return x < 0 ? 0 : x;
  }
  __host__ __device__ int hi(int i) const {
    if (wr < 0) return Nk - 1;
    int x = i + delta() + wr;
    return x > Nk - 1 ? Nk - 1 : x;
  }
};

// Maps a linear CTA index to (head, work index within the head), where the
// work index is ordered heaviest first.  Heads are taken in chunks of
// `chunk` (sized on the host so one chunk's K/V fits comfortably in L2);
// inside a chunk the order is heaviest-first across all its heads, which
// balances causal work like a longest-first schedule, while the CTAs resident
// together only touch one chunk's K/V.
struct ChunkedOrder {
  int head, rank;  // rank 0 = heaviest work unit of the head
  __device__ __forceinline__ ChunkedOrder(int L, int n_heads, int per_head, int chunk) {
    const int full = n_heads / chunk;
    const int span = chunk * per_head;
    int c = L / span, idx = L - c * span, ce = chunk;
    if (c >= full) {  // the last, partial chunk
      c = full;
      idx = L - full * span;
      ce = n_heads - full * chunk;
    }
    rank = idx / ce;
    head = c * chunk + idx % ce;
  }
};

// Byte offset, inside one 128-byte-swizzled [rows][64 x bf16] chunk, of the
// 16-byte unit `u` (0..7) of row `r`: the unit index is XORed with r mod 8.
__device__ __forceinline__ uint32_t sw128_offset(uint32_t r, uint32_t u) {
  return r * 128u + ((u ^ (r & 7u)) << 4);
}

// 2^x for a pair of arguments on the FMA pipe (the MUFU unit alone would
// bound the softmax).  x is clamped to [-126, inf) and split as x = j + f with
// j = round(x), f in [-1/2, 1/2] (Cody and Waite's range reduction; adding
// 1.5 * 2^23 leaves j in the low mantissa bits); 2^f comes from a degree-3
// polynomial and 2^j is added into the exponent field, the bit-level trick of
// Schraudolph's fast exponential (Neural Computation, 1999).  The polynomial is the minimax fit, in relative error,
// of 2^f on [-1/2, 1/2] (Remez exchange; max relative error 7.5e-5, well
// under the 2^-9 rounding of P to bf16).  Arguments below -125 (possible only
// for scores far below the row max) give a value below 2^-125 instead of ~0
// (a subnormal at the clamp); a row sum is at least 1, so that is far below
// fp32 resolution.  Masked (-inf)
// scores must not come here: they take ex2_approx, which returns exact 0.
constexpr float kExp2C0 = 0.99992806f;
constexpr float kExp2C1 = 0.69326097f;
constexpr float kExp2C2 = 0.24261113f;
constexpr float kExp2C3 = 0.05517167f;

__device__ __forceinline__ void exp2_poly_pair(uint64_t x2, float& lo, float& hi) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  float xl, xh;
  f2_unpack(x2, xl, xh);
  const uint64_t x = f2_pack(fmaxf(xl, -126.0f), fmaxf(xh, -126.0f));
  const uint64_t t = f2_add(x, f2_pack(kRound, kRound));    // kRound + j
  const uint64_t j = f2_add(t, f2_pack(-kRound, -kRound));  // j, exact
  const uint64_t f = f2_fma(j, f2_pack(-1.0f, -1.0f), x);   // x - j
  uint64_t p = f2_fma(f, f2_pack(kExp2C3, kExp2C3), f2_pack(kExp2C2, kExp2C2));
  p = f2_fma(p, f, f2_pack(kExp2C1, kExp2C1));
  p = f2_fma(p, f, f2_pack(kExp2C0, kExp2C0));
  float pl, ph, tl, th;
  f2_unpack(p, pl, ph);
  f2_unpack(t, tl, th);
  // the low 9 bits of t's pattern hold j (two's complement); shifted to the
  // exponent field they add j to p's exponent
  lo = __uint_as_float(__float_as_uint(pl) + (__float_as_uint(tl) << 23));
  hi = __uint_as_float(__float_as_uint(ph) + (__float_as_uint(th) << 23));
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

// Block-sparse attention: the calling warp (all 32 lanes) appends, in
// order, the indices i in [0, n) with on(i) true to `list` (ballot
// compaction, 32 indices per round) and returns how many there are.
template <class F>
__device__ __forceinline__ int warp_compact(int n, uint32_t* list, F on) {
  const int lane = threadIdx.x % 32;
  int cnt = 0;
  for (int c0 = 0; c0 < n; c0 += 32) {
    const int i = c0 + lane;
    const bool a = i < n && on(i);
    const unsigned bal = __ballot_sync(0xffffffffu, a);
    if (a) list[cnt + __popc(bal & ((1u << lane) - 1u))] = static_cast<uint32_t>(i);
    cnt += __popc(bal);
  }
  return cnt;
}

// A kernel configuration with fp16 instead of bf16 elements: the same tiles;
// the tensor-core operand type, the conversions to 16 bits and the TMA data
// type follow C::F16.
template <class C>
struct AsF16 : C {
  static constexpr bool F16 = true;
};

// 16-bit float bits to fp32
template <bool F16>
__device__ __forceinline__ float h16_to_f32(uint32_t bits16) {
  if constexpr (F16) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>(bits16)));
  } else {
    return __uint_as_float(bits16 << 16);
  }
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

// One sequence of a call: dense (cu_q null) -- batch b of the tensors, the
// call's mask -- or packed -- rows [cu_q[b], cu_q[b+1]) and [cu_k[b],
// cu_k[b+1]) of one-batch tensors (TMA batch coordinate 0), the mask taken
// with this sequence's own lengths (causal bottom-right per sequence).
struct SeqView {
  int q_off = 0, k_off = 0, tb;
  MaskSpec mask;
  __device__ __forceinline__ SeqView(const MaskSpec& m, const int* cu_q, const int* cu_k, int b)
      : tb(b), mask(m) {
    if (cu_q != nullptr) {
      q_off = __ldg(cu_q + b);
      k_off = __ldg(cu_k + b);
      mask.Nq = __ldg(cu_q + b + 1) - q_off;
      mask.Nk = __ldg(cu_k + b + 1) - k_off;
      tb = 0;
    }
  }
};

// Plain 16-byte stores of rows [0, n_rows) of a tile staged in shared memory
// with the 128-byte swizzle (64-column chunks `chunk_bytes` apart, ncols a
// multiple of 64) to rows row0 + r of a [rows, H, d] bf16 tensor, head h,
// columns [col0, col0 + ncols).  Rows outside [0, total) are skipped.  Used
// for the last tile of a packed sequence, whose following rows belong to the
// next sequence (a TMA store would write them).
__device__ __forceinline__ void store_rows_sw128(uint32_t stage, int chunk_bytes, int n_rows, int ncols,
                                                 uint16_t* dst, int row0, int total, int H, int h,
                                                 int d, int col0, int tid, int nthreads) {
  const int upr = ncols / 8;
  for (int x = tid; x < n_rows * upr; x += nthreads) {
    const int rr = x / upr, u = x % upr;
    const int g = row0 + rr;
    if (g < 0 || g >= total) continue;
    const uint4 v = ld_shared_v4(stage + (u / 8) * chunk_bytes + sw128_offset(rr, u % 8));
    *reinterpret_cast<uint4*>(dst + (static_cast<size_t>(g) * H + h) * d + col0 + u * 8) = v;
  }
}

}  // namespace fa
