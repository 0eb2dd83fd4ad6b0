// fa_merge.cuh -- combining partial attention results: the kernels of ring
// (context-parallel) attention, where each GPU holds a slice of the sequence
// and the key/value slices travel around the ring of GPUs.
//
// Forward.  Attention over a union of disjoint key sets follows from the
// results over each set (abeam.tech FlashAttention summary, "computing
// softmax blockwise correctly", applied to whole key sets): with lse_s the
// natural log-sum-exp of set s and O_s its normalised output,
//     lse = ln sum_s exp(lse_s),   O = sum_s exp(lse_s - lse) O_s.
// fa_lse_merge_kernel folds one more set into a running fp32 accumulator.
//
// Backward.  The gradients of attention restricted to a key set, computed
// with the full rows' O and LSE (fa_bwd does exactly that: P from the given
// LSE, D = rowsum(dO * O) from the given O), are that set's share of dQ and
// its keys' dK / dV; fa_grad_accumulate_kernel sums the shares in fp32.
#pragma once
#include "fa_common.cuh"

namespace fa {

// One warp per (b, i, h) row of the part, O [B, Nq, H, D] and LSE [B, H, Nq],
// folded into row row0 + i of the accumulator, O [B, Nq_acc, H, D] and LSE
// [B, H, Nq_acc] (so a part may cover some of the accumulator's rows):
//   first: acc = part; otherwise acc = merge(acc, part) as above.
// Rows where both are empty (lse = -inf) stay O = 0, lse = -inf.  With o_out
// given ([B, Nq_acc, H, D]), the merged row is also written rounded to the
// element type.
template <int D, bool F16>
__global__ void __launch_bounds__(256) fa_lse_merge_kernel(float* __restrict__ o_acc, float* __restrict__ lse_acc,
                                                           const uint16_t* __restrict__ o_part,
                                                           const float* __restrict__ lse_part,
                                                           uint16_t* __restrict__ o_out, int B, int Nq, int H,
                                                           int Nq_acc, int row0, int first) {
  constexpr int E = D / 32;  // elements per lane: 2, 4 or 8
  const long long row = (static_cast<long long>(blockIdx.x) * 256 + threadIdx.x) / 32;
  const int lane = threadIdx.x % 32;
  if (row >= static_cast<long long>(B) * Nq * H) return;
  const int h = static_cast<int>(row % H);
  const long long bi = row / H;
  const int i = static_cast<int>(bi % Nq);
  const int b = static_cast<int>(bi / Nq);
  const long long lp_i = (static_cast<long long>(b) * H + h) * Nq + i;
  const long long li = (static_cast<long long>(b) * H + h) * Nq_acc + row0 + i;
  const float lp = lse_part[lp_i];
  const float la = first ? -INFINITY : lse_acc[li];
  const float m = fmaxf(la, lp);
  float wa = 0.f, wp = 0.f, lnew = -INFINITY;
  if (m != -INFINITY) {
    const float ea = (la == -INFINITY) ? 0.f : expf(la - m);
    const float ep = (lp == -INFINITY) ? 0.f : expf(lp - m);
    const float s = ea + ep;
    lnew = m + logf(s);
    wa = ea / s;
    wp = ep / s;
  }
  const long long poff = row * D + lane * E;
  const long long off = ((static_cast<long long>(b) * Nq_acc + row0 + i) * H + h) * D + lane * E;
  float acc[E], part[E];
#pragma unroll
  for (int e = 0; e < E; e += 2) {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(o_part + poff + e);
    part[e] = h16_to_f32<F16>(w & 0xFFFFu);
    part[e + 1] = h16_to_f32<F16>(w >> 16);
  }
  if (first) {
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
  } else {
#pragma unroll
    for (int e = 0; e < E; e += 2) {
      const float2 a = *reinterpret_cast<const float2*>(o_acc + off + e);
      acc[e] = a.x;
      acc[e + 1] = a.y;
    }
  }
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = wa * acc[e] + wp * part[e];
#pragma unroll
  for (int e = 0; e < E; e += 2) {
    *reinterpret_cast<float2*>(o_acc + off + e) = make_float2(acc[e], acc[e + 1]);
    if (o_out != nullptr) *reinterpret_cast<uint32_t*>(o_out + off + e) = pack2<F16>(acc[e], acc[e + 1]);
  }
  // every lane has read the old lse_acc (above) before lane 0 replaces it
  __syncwarp();
  if (lane == 0) lse_acc[li] = lnew;
}

// Rows of row_elems elements: part [B, rows, row_elems] added to rows
// [row0, row0 + rows) of acc [B, rows_acc, row_elems] (fp32), 8 elements per
// thread (row_elems % 8 == 0, 16-byte aligned buffers), blockIdx.y = b:
//   part given: acc = (first ? 0 : acc) + part;  out given ([B, rows_acc,
//   row_elems]): out = round(acc) on the same rows.
template <bool F16>
__global__ void __launch_bounds__(256) fa_grad_accumulate_kernel(float* __restrict__ acc,
                                                                 const uint16_t* __restrict__ part,
                                                                 uint16_t* __restrict__ out, int rows_acc, int row0,
                                                                 int rows, long long row_elems, int first) {
  const long long n = static_cast<long long>(rows) * row_elems;
  const long long xp = (static_cast<long long>(blockIdx.x) * 256 + threadIdx.x) * 8;
  if (xp >= n) return;
  const long long b = blockIdx.y;
  const long long x = (b * rows_acc + row0) * row_elems + xp;
  float a[8];
  if (first && part != nullptr) {
#pragma unroll
    for (int e = 0; e < 8; ++e) a[e] = 0.f;
  } else {
    const float4 a0 = *reinterpret_cast<const float4*>(acc + x);
    const float4 a1 = *reinterpret_cast<const float4*>(acc + x + 4);
    a[0] = a0.x; a[1] = a0.y; a[2] = a0.z; a[3] = a0.w;
    a[4] = a1.x; a[5] = a1.y; a[6] = a1.z; a[7] = a1.w;
  }
  if (part != nullptr) {
    const uint4 p = *reinterpret_cast<const uint4*>(part + b * n + xp);
    const uint32_t w[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      a[2 * e] += h16_to_f32<F16>(w[e] & 0xFFFFu);
      a[2 * e + 1] += h16_to_f32<F16>(w[e] >> 16);
    }
    *reinterpret_cast<float4*>(acc + x) = make_float4(a[0], a[1], a[2], a[3]);
    *reinterpret_cast<float4*>(acc + x + 4) = make_float4(a[4], a[5], a[6], a[7]);
  }
  if (out != nullptr)
    *reinterpret_cast<uint4*>(out + x) =
        make_uint4(pack2<F16>(a[0], a[1]), pack2<F16>(a[2], a[3]), pack2<F16>(a[4], a[5]), pack2<F16>(a[6], a[7]));
}

}  // namespace fa
