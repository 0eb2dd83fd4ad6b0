// fa_common.cuh -- shared definitions of the sm_100a attention kernels.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

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

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

}  // namespace fa
