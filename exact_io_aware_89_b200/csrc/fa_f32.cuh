// fa_f32.cuh -- fp32 attention for small problems, on the CUDA cores.
//
// Same operation as the bf16 kernels (softmax(Q K^T * scale) V with the
// online softmax of the Qiita tutorial, section 4.3, and the output rescale of
// the abeam.tech summary), kept in fp32 end to end.  One warp owns one row
// (a query row forward and for dQ, a key row for dK/dV); dot products are
// reduced across the warp with shuffles; each lane holds d/32 columns.  It is
// meant for the tiny fp32 workload (e.g. B=1, H=2, N=128, d=64), not for
// speed.
#pragma once
#include "fa_common.cuh"

namespace fa {

constexpr int kF32MaxPerLane = 8;  // d <= 256, d % 32 == 0

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

struct F32Params {
  int B, Nq, Nk, Hq, Hkv, group, d;
  float scale, scale_log2;
  MaskSpec mask;
  int Nq_pad;
  const float* D;     // [B, Hq, Nq_pad] (backward)
  const float* lse2;  // [B, Hq, Nq_pad] (backward)
};

// forward: warp per (b, i, h) query row
__global__ void __launch_bounds__(128) fa_fwd_f32_kernel(const float* __restrict__ q,
                                                         const float* __restrict__ k,
                                                         const float* __restrict__ v,
                                                         float* __restrict__ o, float* __restrict__ lse,
                                                         const F32Params p) {
  const long long w = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) / 32;
  const int lane = threadIdx.x % 32;
  if (w >= static_cast<long long>(p.B) * p.Nq * p.Hq) return;
  const int h = static_cast<int>(w % p.Hq);
  const int i = static_cast<int>((w / p.Hq) % p.Nq);
  const int b = static_cast<int>(w / (static_cast<long long>(p.Hq) * p.Nq));
  const int hk = h / p.group, npl = p.d / 32;
  const float* qi = q + ((static_cast<size_t>(b) * p.Nq + i) * p.Hq + h) * p.d;
  float qr[kF32MaxPerLane], acc[kF32MaxPerLane];
  for (int c = 0; c < npl; ++c) {
    qr[c] = qi[lane + 32 * c];
    acc[c] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  const int lo = p.mask.lo(i), hi = p.mask.hi(i);
  for (int j = lo; j <= hi; ++j) {
    const size_t kv = ((static_cast<size_t>(b) * p.Nk + j) * p.Hkv + hk) * p.d;
    float part = 0.f;
    for (int c = 0; c < npl; ++c) part = fmaf(qr[c], k[kv + lane + 32 * c], part);
    const float s = warp_sum(part) * p.scale;
    const float m_new = fmaxf(m, s);
    const float alpha = expf(m - m_new);  // 0 on the first key (m = -inf)
    const float pj = expf(s - m_new);
    l = l * alpha + pj;
    for (int c = 0; c < npl; ++c) acc[c] = fmaf(pj, v[kv + lane + 32 * c], acc[c] * alpha);
    m = m_new;
  }
  float* oi = o + ((static_cast<size_t>(b) * p.Nq + i) * p.Hq + h) * p.d;
  const float inv = (l > 0.f) ? 1.f / l : 0.f;
  for (int c = 0; c < npl; ++c) oi[lane + 32 * c] = acc[c] * inv;
  if (lane == 0) lse[(static_cast<size_t>(b) * p.Hq + h) * p.Nq + i] = (l > 0.f) ? m + logf(l) : -INFINITY;
}

// dQ: warp per (b, i, h) query row
__global__ void __launch_bounds__(128) fa_bwd_dq_f32_kernel(const float* __restrict__ q,
                                                            const float* __restrict__ k,
                                                            const float* __restrict__ v,
                                                            const float* __restrict__ dout,
                                                            float* __restrict__ dq, const F32Params p) {
  const long long w = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) / 32;
  const int lane = threadIdx.x % 32;
  if (w >= static_cast<long long>(p.B) * p.Nq * p.Hq) return;
  const int h = static_cast<int>(w % p.Hq);
  const int i = static_cast<int>((w / p.Hq) % p.Nq);
  const int b = static_cast<int>(w / (static_cast<long long>(p.Hq) * p.Nq));
  const int hk = h / p.group, npl = p.d / 32;
  const size_t qo = ((static_cast<size_t>(b) * p.Nq + i) * p.Hq + h) * p.d;
  float qr[kF32MaxPerLane], dor[kF32MaxPerLane], acc[kF32MaxPerLane];
  for (int c = 0; c < npl; ++c) {
    qr[c] = q[qo + lane + 32 * c];
    dor[c] = dout[qo + lane + 32 * c];
    acc[c] = 0.f;
  }
  const size_t srow = (static_cast<size_t>(b) * p.Hq + h) * p.Nq_pad + i;
  const float lse2 = p.lse2[srow], Di = p.D[srow];
  const int lo = p.mask.lo(i), hi = p.mask.hi(i);
  for (int j = lo; j <= hi; ++j) {
    const size_t kv = ((static_cast<size_t>(b) * p.Nk + j) * p.Hkv + hk) * p.d;
    float ps = 0.f, pd = 0.f;
    for (int c = 0; c < npl; ++c) {
      ps = fmaf(qr[c], k[kv + lane + 32 * c], ps);
      pd = fmaf(dor[c], v[kv + lane + 32 * c], pd);
    }
    const float pj = exp2f(warp_sum(ps) * p.scale_log2 - lse2);
    const float ds = pj * (warp_sum(pd) - Di);
    for (int c = 0; c < npl; ++c) acc[c] = fmaf(ds, k[kv + lane + 32 * c], acc[c]);
  }
  for (int c = 0; c < npl; ++c) dq[qo + lane + 32 * c] = acc[c] * p.scale;
}

// dK, dV: warp per (b, j, hk) key row, summed over the query heads of the group
__global__ void __launch_bounds__(128) fa_bwd_dkdv_f32_kernel(
    const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
    const float* __restrict__ dout, float* __restrict__ dk, float* __restrict__ dv,
    const F32Params p) {
  const long long w = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) / 32;
  const int lane = threadIdx.x % 32;
  if (w >= static_cast<long long>(p.B) * p.Nk * p.Hkv) return;
  const int hk = static_cast<int>(w % p.Hkv);
  const int j = static_cast<int>((w / p.Hkv) % p.Nk);
  const int b = static_cast<int>(w / (static_cast<long long>(p.Hkv) * p.Nk));
  const int npl = p.d / 32;
  const size_t ko = ((static_cast<size_t>(b) * p.Nk + j) * p.Hkv + hk) * p.d;
  float kr[kF32MaxPerLane], vr[kF32MaxPerLane], ak[kF32MaxPerLane], av[kF32MaxPerLane];
  for (int c = 0; c < npl; ++c) {
    kr[c] = k[ko + lane + 32 * c];
    vr[c] = v[ko + lane + 32 * c];
    ak[c] = 0.f;
    av[c] = 0.f;
  }
  const int delta = p.mask.delta();
  int i_lo = (p.mask.wr < 0) ? 0 : j - delta - p.mask.wr;
  int i_hi = (p.mask.wl < 0) ? p.Nq - 1 : j - delta + p.mask.wl;
  i_lo = max(i_lo, 0);
  i_hi = min(i_hi, p.Nq - 1);
  for (int hq = hk * p.group; hq < (hk + 1) * p.group; ++hq) {
    for (int i = i_lo; i <= i_hi; ++i) {
      const size_t qo = ((static_cast<size_t>(b) * p.Nq + i) * p.Hq + hq) * p.d;
      float ps = 0.f, pd = 0.f;
      for (int c = 0; c < npl; ++c) {
        ps = fmaf(q[qo + lane + 32 * c], kr[c], ps);
        pd = fmaf(dout[qo + lane + 32 * c], vr[c], pd);
      }
      const size_t srow = (static_cast<size_t>(b) * p.Hq + hq) * p.Nq_pad + i;
      const float pj = exp2f(warp_sum(ps) * p.scale_log2 - p.lse2[srow]);
      const float ds = pj * (warp_sum(pd) - p.D[srow]);
      for (int c = 0; c < npl; ++c) {
        av[c] = fmaf(pj, dout[qo + lane + 32 * c], av[c]);
        ak[c] = fmaf(ds, q[qo + lane + 32 * c], ak[c]);
      }
    }
  }
  for (int c = 0; c < npl; ++c) {
    dk[ko + lane + 32 * c] = ak[c] * p.scale;
    dv[ko + lane + 32 * c] = av[c];
  }
}

}  // namespace fa
