// fa_api.cu -- the C ABI of libfa (declared in include/fa.h): argument
// validation, TMA descriptor encoding and kernel launches on the caller's
// stream.  No device memory is allocated here and nothing runs on the CPU
// besides the checks.
#include <atomic>
#include <type_traits>
#include <cstdio>
#include <mutex>
#include <vector>

#include "fa_bwd.cuh"
#include "fa_decode.cuh"
#include "fa_f32.cuh"
#include "fa_fwd.cuh"
#include "fa_merge.cuh"
#include "fa_host.cuh"

using namespace fa;

namespace {

// ---------------------------------------------------------------- tracing
struct TraceRec {
  int kind;
  cudaEvent_t a, b;
};
std::mutex g_trace_mu;
bool g_trace_on = false;
std::vector<cudaEvent_t> g_event_pool;
std::vector<TraceRec> g_trace;
constexpr int kEventPoolInit = 512;

bool take_event(cudaEvent_t* e) {
  if (!g_event_pool.empty()) {
    *e = g_event_pool.back();
    g_event_pool.pop_back();
    return true;
  }
  return cudaEventCreate(e) == cudaSuccess;
}

// Brackets one launch with events when tracing is on.
struct TraceScope {
  int kind;
  cudaStream_t stream;
  cudaEvent_t a = nullptr, b = nullptr;
  bool active = false;
  TraceScope(int k, cudaStream_t s) : kind(k), stream(s) {
    std::lock_guard<std::mutex> lock(g_trace_mu);
    if (!g_trace_on) return;
    if (!take_event(&a) || !take_event(&b)) return;
    active = cudaEventRecord(a, stream) == cudaSuccess;
  }
  ~TraceScope() {
    if (!active) return;
    std::lock_guard<std::mutex> lock(g_trace_mu);
    if (cudaEventRecord(b, stream) == cudaSuccess) g_trace.push_back({kind, a, b});
  }
};

// Test only: arms fa_test_withhold_next_load's one-shot for the next dense
// forward launch.
std::atomic<int> g_test_withhold{0};

// A device-side wait gives up after this long (the kernels' own waits are
// microseconds; the limit only matters when something is broken).
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

// fwd: {d, Q tiles per CTA, key tile, K/V ring depth}
// {d, Q tiles per CTA, key tile, K/V ring depth, exp2 pairs of 8 on the FMA pipe,
//  P handed over in two halves}
using Fwd64 = FwdCfg<64, 2, 128, 3, 2, true>;
using Fwd128 = FwdCfg<128, 2, 128, 2, 2>;
using Fwd256 = FwdCfg<256, 1, 64, 2>;
// block-sparse forward: one 128-row Q tile per CTA, so a CTA loads only the
// key tiles of its own query block (two Q tiles would load the union of both)
using FwdBs64 = FwdCfg<64, 1, 128, 4>;
using FwdBs128 = FwdCfg<128, 1, 128, 2>;
// dQ: one 128-row query tile per CTA with 128-key tiles {d, K ring, V ring};
// d = 256 keeps 64-key tiles {d, Q tiles per CTA, key tile, K/V ring depth}
using Dq64 = Dq2Cfg<64, 4, 3>;
using Dq128 = Dq2Cfg<128, 3, 2>;
using Dq256 = DqCfg<256, 1, 64, 1>;
// dK/dV, d = 64 and 128: 128-query steps {d, Q/dO ring depth, exp2 pairs of 8
// on the FMA pipe}; d = 256: 64-query steps {d, accumulated d slice, query
// tile, Q/dO ring depth}
using Dkv64 = DkvWCfg<64, 4, 2>;
using Dkv128 = DkvWCfg<128, 2, 2>;
using Dkv256 = DkvCfg<256, 128, 64, 1>;

// split-KV decode: {d, key tile, K/V ring depth, TMEM lanes per copy of the packed rows}
template <int RCP> using Dec64 = DecCfg<64, 128, 6, RCP>;
template <int RCP> using Dec128 = DecCfg<128, 128, 3, RCP>;
template <int RCP> using Dec256 = DecCfg<256, 64, 2, RCP>;
constexpr int kMaxDecodeSplits = 4096;

constexpr int kMaxDevices = 64;

// block-sparse masks are over tiles of 128 query rows x 128 keys
constexpr int kBlockSparseTile = 128;

// a configuration with bf16 elements (F16 false) or fp16 elements
template <bool F16, class C>
using Ty = std::conditional_t<F16, AsF16<C>, C>;

constexpr CUtensorMapDataType tma_type(bool f16) {
  return f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
}

template <typename Kernel>
cudaError_t smem_attr_once(Kernel kernel, int bytes, int* done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (!__atomic_load_n(&done[dev], __ATOMIC_ACQUIRE)) {
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    __atomic_store_n(&done[dev], 1, __ATOMIC_RELEASE);
  }
  return cudaSuccess;
}

int launch_status() { return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA; }

MaskSpec make_mask(int Nq, int Nk, int causal, int win_l, int win_r) {
  MaskSpec m;
  m.Nq = Nq;
  m.Nk = Nk;
  m.wl = win_l < 0 ? -1 : win_l;
  m.wr = causal ? 0 : (win_r < 0 ? -1 : win_r);
  return m;
}

int check_common(const void* q, const void* k, const void* v, int B, int Nq, int Nk, int Hq,
                 int Hkv, float scale) {
  if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return FA_ERR_INVALID_ARG;
  return check_sizes(B, Nq, Nk, Hq, Hkv, scale);
}

int pad_rows(int Nq) { return (Nq + 255) / 256 * 256; }

// Heads per scheduling chunk: at most as many as keep the streamed operands
// of one chunk (bytes_per_head each) within a third of the B200's 126 MB L2,
// then evened out so the last chunk is not a small tail.
int head_chunk(int n_heads, long long bytes_per_head) {
  constexpr long long kBudget = 42ll << 20;
  long long c = bytes_per_head > 0 ? kBudget / bytes_per_head : n_heads;
  if (c < 1) c = 1;
  if (c > n_heads) c = n_heads;
  const long long n_chunks = (n_heads + c - 1) / c;
  return static_cast<int>((n_heads + n_chunks - 1) / n_chunks);
}

// ------------------------------------------------------------------ forward
template <class C>
int launch_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Nq,
               int Nk, int Hq, int Hkv, float scale, const MaskSpec& mask, cudaStream_t stream) {
  static int attr_done[kMaxDevices] = {0};
  CUtensorMap tq, tk, tv, to;
  if (!encode_bnhd(&tq, q, B, Nq, Hq, C::D, C::BM, tma_type(C::F16)) || !encode_bnhd(&tk, k, B, Nk, Hkv, C::D, C::BN, tma_type(C::F16)) ||
      !encode_bnhd(&tv, v, B, Nk, Hkv, C::D, C::BN, tma_type(C::F16)) || !encode_bnhd(&to, o, B, Nq, Hq, C::D, C::BM, tma_type(C::F16)))
    return FA_ERR_CUDA;
  FwdParams p;
  p.B = B; p.Nq = Nq; p.Nk = Nk; p.Hq = Hq; p.Hkv = Hkv; p.group = Hq / Hkv;
  p.scale_log2 = scale * kLog2e;
  p.mask = mask;
  p.n_qgroups = (Nq + C::NQT * C::BM - 1) / (C::NQT * C::BM);
  p.head_chunk = head_chunk(B * Hq, 4ll * Nk * C::D);  // K and V of one head, bf16
  p.lse = lse;
  p.cu_q = nullptr;
  p.cu_k = nullptr;
  p.total_q = 0;
  p.o = static_cast<uint16_t*>(o);
  p.bmask = nullptr;
  p.bm_sb = p.bm_sh = 0;
  p.bm_cols = 0;
  p.wait_limit_ns = kWaitLimitNs;
  p.test_withhold = g_test_withhold.exchange(0);
  auto kern = fa_fwd_kernel<C>;
  if (smem_attr_once(kern, C::SMEM_BYTES, attr_done) != cudaSuccess) return FA_ERR_CUDA;
  const long long grid = static_cast<long long>(p.n_qgroups) * B * Hq;
  {
    TraceScope tr(FA_KERNEL_FWD, stream);
    kern<<<static_cast<unsigned>(grid), C::NTHREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, to, p);
  }
  return launch_status();
}

// Block-sparse forward: the dense launch plus the block mask; each CTA keeps
// its list of key tiles (4 bytes each) in shared memory after the fixed part.

template <class C>
int launch_fwd_bs(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Nq, int Nk,
                  int Hq, int Hkv, float scale, const MaskSpec& mask, const uint8_t* bmask, long long sb,
                  long long sh, cudaStream_t stream) {
  static int attr_done[kMaxDevices] = {0};
  const long long list_bytes = 4ll * ((Nk + C::BN - 1) / C::BN + 1);
  const long long smem = C::SMEM_BYTES + list_bytes;
  if (smem > 232448) return FA_ERR_UNSUPPORTED;  // more key tiles than the list has room for
  CUtensorMap tq, tk, tv, to;
  if (!encode_bnhd(&tq, q, B, Nq, Hq, C::D, C::BM, tma_type(C::F16)) ||
      !encode_bnhd(&tk, k, B, Nk, Hkv, C::D, C::BN, tma_type(C::F16)) ||
      !encode_bnhd(&tv, v, B, Nk, Hkv, C::D, C::BN, tma_type(C::F16)) ||
      !encode_bnhd(&to, o, B, Nq, Hq, C::D, C::BM, tma_type(C::F16)))
    return FA_ERR_CUDA;
  FwdParams p;
  p.B = B; p.Nq = Nq; p.Nk = Nk; p.Hq = Hq; p.Hkv = Hkv; p.group = Hq / Hkv;
  p.scale_log2 = scale * kLog2e;
  p.mask = mask;
  p.n_qgroups = (Nq + C::NQT * C::BM - 1) / (C::NQT * C::BM);
  p.head_chunk = head_chunk(B * Hq, 4ll * Nk * C::D);
  p.lse = lse;
  p.cu_q = nullptr;
  p.cu_k = nullptr;
  p.total_q = 0;
  p.o = static_cast<uint16_t*>(o);
  p.bmask = bmask;
  p.bm_sb = sb;
  p.bm_sh = sh;
  p.bm_cols = (Nk + kBlockSparseTile - 1) / kBlockSparseTile;
  p.wait_limit_ns = kWaitLimitNs;
  p.test_withhold = 0;
  auto kern = fa_fwd_kernel<C, false, true>;
  if (smem_attr_once(kern, 232448, attr_done) != cudaSuccess) return FA_ERR_CUDA;
  const long long grid = static_cast<long long>(p.n_qgroups) * B * Hq;
  {
    TraceScope tr(FA_KERNEL_FWD, stream);
    kern<<<static_cast<unsigned>(grid), C::NTHREADS, static_cast<size_t>(smem), stream>>>(tq, tk, tv, to, p);
  }
  return launch_status();
}

// Packed sequences: the tensors are one batch of total_q / total_k rows;
// sequence b is rows [cu_q[b], cu_q[b+1]) and [cu_k[b], cu_k[b+1]).
template <class C>
int launch_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse, const int* cu_q,
                      const int* cu_k, int B, int max_q, int max_k, int total_q, int total_k, int Hq,
                      int Hkv, float scale, int causal, int win_l, int win_r, cudaStream_t stream) {
  static int attr_done[kMaxDevices] = {0};
  CUtensorMap tq, tk, tv, to;
  if (!encode_bnhd(&tq, q, 1, total_q, Hq, C::D, C::BM, tma_type(C::F16)) || !encode_bnhd(&tk, k, 1, total_k, Hkv, C::D, C::BN, tma_type(C::F16)) ||
      !encode_bnhd(&tv, v, 1, total_k, Hkv, C::D, C::BN, tma_type(C::F16)) || !encode_bnhd(&to, o, 1, total_q, Hq, C::D, C::BM, tma_type(C::F16)))
    return FA_ERR_CUDA;
  FwdParams p;
  p.B = B; p.Nq = max_q; p.Nk = max_k; p.Hq = Hq; p.Hkv = Hkv; p.group = Hq / Hkv;
  p.scale_log2 = scale * kLog2e;
  p.mask = make_mask(max_q, max_k, causal, win_l, win_r);
  p.n_qgroups = (max_q + C::NQT * C::BM - 1) / (C::NQT * C::BM);
  p.head_chunk = head_chunk(B * Hq, 4ll * max_k * C::D);
  p.lse = lse;
  p.cu_q = cu_q;
  p.cu_k = cu_k;
  p.total_q = total_q;
  p.o = static_cast<uint16_t*>(o);
  p.bmask = nullptr;
  p.bm_sb = p.bm_sh = 0;
  p.bm_cols = 0;
  p.wait_limit_ns = kWaitLimitNs;
  p.test_withhold = 0;
  auto kern = fa_fwd_kernel<C, true>;
  if (smem_attr_once(kern, C::SMEM_BYTES, attr_done) != cudaSuccess) return FA_ERR_CUDA;
  const long long grid = static_cast<long long>(p.n_qgroups) * B * Hq;
  if (grid > (1ll << 31) - 1) return FA_ERR_INVALID_ARG;
  {
    TraceScope tr(FA_KERNEL_FWD, stream);
    kern<<<static_cast<unsigned>(grid), C::NTHREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, to, p);
  }
  return launch_status();
}

// ------------------------------------------------------------------ backward
// The backward's dQ and dK/dV kernels (the split backward) depend only on the
// preprocess, not on each other: dQ runs on a side stream (forked from and
// joined back into the caller's stream with events), so the last partial wave
// of one kernel overlaps the other's CTAs.  Each caller stream of a device
// gets its own side stream, so callers on independent streams never wait for
// each other; the fork / launch / join sequence holds that entry's lock so
// concurrent callers on the same stream cannot swap each other's events.
// While the caller's stream is being captured into a CUDA graph, or when the
// table of side streams is full, dQ is launched on the caller's stream itself
// (in order, after the preprocess and before dK/dV): a capture then pulls in
// no stream but the caller's.
struct SideStream {
  cudaStream_t owner = nullptr;  // the caller stream this entry serves
  bool used = false;
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  std::mutex mu;
};
constexpr int kSideStreamsPerDevice = 32;
std::mutex g_side_table_mu;
SideStream g_side[kMaxDevices][kSideStreamsPerDevice];

// The side stream of `caller` on the current device, or nullptr when dQ should
// run on the caller's stream (capture in progress, table full).  FA_ERR_CUDA
// when a CUDA call fails.
int side_stream(cudaStream_t caller, SideStream** out) {
  *out = nullptr;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(caller, &cap) != cudaSuccess) return FA_ERR_CUDA;
  if (cap != cudaStreamCaptureStatusNone) return FA_OK;
  std::lock_guard<std::mutex> lock(g_side_table_mu);
  SideStream* free_slot = nullptr;
  for (SideStream& ss : g_side[dev]) {
    if (ss.used && ss.owner == caller) {
      *out = &ss;
      return FA_OK;
    }
    if (!ss.used && free_slot == nullptr) free_slot = &ss;
  }
  if (free_slot == nullptr) return FA_OK;
  if (cudaStreamCreateWithFlags(&free_slot->stream, cudaStreamNonBlocking) != cudaSuccess ||
      cudaEventCreateWithFlags(&free_slot->fork, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&free_slot->join, cudaEventDisableTiming) != cudaSuccess)
    return FA_ERR_CUDA;
  free_slot->owner = caller;
  free_slot->used = true;
  *out = free_slot;
  return FA_OK;
}

// The split backward runs dQ beside dK/dV while the smaller of the two grids
// is at most this many waves (CTAs per SM).
constexpr long long kOverlapWaves = 4;

int current_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

// Packed sequences of a backward call (all null / 0 when dense).
struct Varlen {
  const int* cu_q = nullptr;
  const int* cu_k = nullptr;
  int total_q = 0, total_k = 0;
};

// Dense (VL false): B batches of Nq / Nk rows.  Packed (VL true, vl set): B
// sequences of at most Nq / Nk rows in one-batch tensors of vl.total_q /
// vl.total_k rows.
// Block mask of a block-sparse backward call (null when dense).
struct BlockMask {
  const uint8_t* mask = nullptr;
  long long sb = 0, sh = 0;
};

template <class CKV, bool VL, bool BS>
constexpr auto dkdv_kernel() {
  if constexpr (CKV::WIDE)
    return fa_bwd_dkdv_wide_kernel<CKV, VL, BS>;
  else
    return fa_bwd_dkdv_kernel<CKV, VL, BS>;
}

template <class CQ, class CKV, bool VL = false, bool BS = false>
int launch_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
               const void* dO, void* dq, void* dk, void* dv, int B, int Nq, int Nk, int Hq, int Hkv,
               float scale, const MaskSpec& mask, float* ws, cudaStream_t stream, const Varlen& vl = Varlen(),
               const BlockMask& bm = BlockMask()) {
  static int attr_dq[kMaxDevices] = {0};
  static int attr_kv[kMaxDevices] = {0};
  // block-sparse: each CTA's list of key tiles (dQ) or steps (dK/dV), 4 bytes
  // an entry, after the fixed shared memory
  const long long dq_smem = CQ::SMEM_BYTES + (BS ? 4ll * ((Nk + CQ::BN - 1) / CQ::BN + 1) : 0);
  const long long kv_smem =
      CKV::SMEM_BYTES + (BS ? 4ll * (Hq / Hkv) * ((Nq + CKV::BM - 1) / CKV::BM + 1) : 0);
  if (dq_smem > 232448 || kv_smem > 232448) return FA_ERR_UNSUPPORTED;
  // dQ beside dK/dV pays off while one of the kernels runs few waves (the
  // other kernel's CTAs fill its partial waves: the training shape, GQA with a
  // window); when both run many waves they only compete for the SMs and for
  // L2 (32 heads at N = 8192: 7% slower side by side), and they run one after
  // the other
  const long long dq_ctas = static_cast<long long>((Nq + CQ::NQT * CQ::BM - 1) / (CQ::NQT * CQ::BM)) * B * Hq;
  const long long kv_ctas = static_cast<long long>((Nk + CKV::BN - 1) / CKV::BN) * B * Hkv * (CQ::D / CKV::DV);
  const bool overlap = (dq_ctas < kv_ctas ? dq_ctas : kv_ctas) <= kOverlapWaves * static_cast<long long>(current_sm_count());
  SideStream* side = nullptr;
  if (overlap && side_stream(stream, &side) != FA_OK) return FA_ERR_CUDA;
  std::unique_lock<std::mutex> side_lock;
  if (side != nullptr) side_lock = std::unique_lock<std::mutex>(side->mu);
  TraceScope whole(FA_KERNEL_BWD_CALL, stream);  // ends after the join below
  constexpr int D = CQ::D;
  const int Nq_pad = pad_rows(Nq);
  const long long rows_pad = static_cast<long long>(B) * Hq * Nq_pad;
  {
    constexpr int G = D / 8;  // lanes per row (16-byte loads)
    constexpr int RPG = 4;    // rows per lane group
    const long long blocks = (rows_pad * G / RPG + 255) / 256;
    TraceScope tr(FA_KERNEL_BWD_PREP, stream);
    fa_bwd_prep_h16_kernel<G, RPG, VL, CQ::F16><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        static_cast<const uint16_t*>(o), static_cast<const uint16_t*>(dO), lse, ws, B, Nq,
        Hq, Nq_pad, vl.cu_q, vl.total_q);
    if (launch_status() != FA_OK) return FA_ERR_CUDA;
  }
  BwdParams p;
  p.B = B; p.Nq = Nq; p.Nk = Nk; p.Hq = Hq; p.Hkv = Hkv; p.group = Hq / Hkv;
  p.scale = scale;
  p.scale_log2 = scale * kLog2e;
  p.mask = mask;
  p.Nq_pad = Nq_pad;
  p.D = ws;
  p.lse2 = ws + rows_pad;
  p.n_qgroups = (Nq + CQ::NQT * CQ::BM - 1) / (CQ::NQT * CQ::BM);
  p.n_kvtiles = (Nk + CKV::BN - 1) / CKV::BN;
  p.head_chunk = head_chunk(B * Hq, 4ll * Nk * D);                  // K and V per query head
  p.head_chunk_kv = head_chunk(B * Hkv, 4ll * Nq * D * (Hq / Hkv));  // Q and dO per key/value head
  p.cu_q = vl.cu_q;
  p.cu_k = vl.cu_k;
  p.total_q = vl.total_q;
  p.total_k = vl.total_k;
  p.dq = static_cast<uint16_t*>(dq);
  p.dk = static_cast<uint16_t*>(dk);
  p.dv = static_cast<uint16_t*>(dv);
  p.bmask = bm.mask;
  p.bm_sb = bm.sb;
  p.bm_sh = bm.sh;
  p.bm_cols = (Nk + kBlockSparseTile - 1) / kBlockSparseTile;
  p.wait_limit_ns = kWaitLimitNs;
  // tensor-map shapes: dense [B, N, H, d]; packed [1, total, H, d]
  const bool packed = VL;
  const int mB = packed ? 1 : B, mNq = packed ? vl.total_q : Nq, mNk = packed ? vl.total_k : Nk;
  {
    CUtensorMap tq, tk, tv, tdo, tdq;
    if (!encode_bnhd(&tq, q, mB, mNq, Hq, D, CQ::BM, tma_type(CQ::F16)) || !encode_bnhd(&tk, k, mB, mNk, Hkv, D, CQ::BN, tma_type(CQ::F16)) ||
        !encode_bnhd(&tv, v, mB, mNk, Hkv, D, CQ::BN, tma_type(CQ::F16)) || !encode_bnhd(&tdo, dO, mB, mNq, Hq, D, CQ::BM, tma_type(CQ::F16)) ||
        !encode_bnhd(&tdq, dq, mB, mNq, Hq, D, CQ::BM, tma_type(CQ::F16)))
      return FA_ERR_CUDA;
    const long long grid = static_cast<long long>(p.n_qgroups) * B * Hq;
    const int attr_bytes = BS ? 232448 : CQ::SMEM_BYTES;
    // fork: the side stream waits for the preprocess
    if (side != nullptr && (cudaEventRecord(side->fork, stream) != cudaSuccess ||
                            cudaStreamWaitEvent(side->stream, side->fork, 0) != cudaSuccess))
      return FA_ERR_CUDA;
    cudaStream_t dq_stream = side != nullptr ? side->stream : stream;
    if constexpr (CQ::ONE_TILE) {
      auto kern = fa_bwd_dq2_kernel<CQ, VL, BS>;
      if (smem_attr_once(kern, attr_bytes, attr_dq) != cudaSuccess) return FA_ERR_CUDA;
      TraceScope tr(FA_KERNEL_BWD_DQ, dq_stream);
      kern<<<static_cast<unsigned>(grid), CQ::NTHREADS, static_cast<size_t>(dq_smem), dq_stream>>>(tq, tk, tv,
                                                                                                 tdo, tdq, p);
    } else {
      auto kern = fa_bwd_dq_kernel<CQ, VL, BS>;
      if (smem_attr_once(kern, attr_bytes, attr_dq) != cudaSuccess) return FA_ERR_CUDA;
      TraceScope tr(FA_KERNEL_BWD_DQ, dq_stream);
      kern<<<static_cast<unsigned>(grid), CQ::NTHREADS, static_cast<size_t>(dq_smem), dq_stream>>>(tq, tk, tv,
                                                                                                 tdo, tdq, p);
    }
    if (launch_status() != FA_OK) return FA_ERR_CUDA;
    if (side != nullptr && cudaEventRecord(side->join, dq_stream) != cudaSuccess) return FA_ERR_CUDA;
  }
  {
    CUtensorMap tq, tk, tv, tdo, tdk, tdv;
    if (!encode_bnhd(&tq, q, mB, mNq, Hq, D, CKV::BM, tma_type(CKV::F16)) || !encode_bnhd(&tk, k, mB, mNk, Hkv, D, CKV::BN, tma_type(CKV::F16)) ||
        !encode_bnhd(&tv, v, mB, mNk, Hkv, D, CKV::BN, tma_type(CKV::F16)) || !encode_bnhd(&tdo, dO, mB, mNq, Hq, D, CKV::BM, tma_type(CKV::F16)) ||
        !encode_bnhd(&tdk, dk, mB, mNk, Hkv, D, CKV::BN, tma_type(CKV::F16)) || !encode_bnhd(&tdv, dv, mB, mNk, Hkv, D, CKV::BN, tma_type(CKV::F16)))
      return FA_ERR_CUDA;
    auto kern = dkdv_kernel<CKV, VL, BS>();
    if (smem_attr_once(kern, BS ? 232448 : CKV::SMEM_BYTES, attr_kv) != cudaSuccess) return FA_ERR_CUDA;
    const dim3 grid(static_cast<unsigned>(static_cast<long long>(p.n_kvtiles) * B * Hkv), D / CKV::DV);
    {
      TraceScope tr(FA_KERNEL_BWD_DKDV, stream);
      kern<<<grid, CKV::NTHREADS, static_cast<size_t>(kv_smem), stream>>>(tq, tk, tv, tdo, tdk, tdv, p);
    }
    if (launch_status() != FA_OK) return FA_ERR_CUDA;
  }
  // join: the caller's stream continues after dQ too
  if (side != nullptr && cudaStreamWaitEvent(stream, side->join, 0) != cudaSuccess) return FA_ERR_CUDA;
  return FA_OK;
}

size_t workspace_bytes(int B, int Nq, int Hq) {
  if (B < 1 || Nq < 1 || Hq < 1) return 0;
  return 2ull * static_cast<size_t>(B) * static_cast<size_t>(Hq) * static_cast<size_t>(pad_rows(Nq)) *
         sizeof(float);
}

// ------------------------------------------------------------ split-KV decode
// Row packing and key split of one fa_fwd_splitkv call.
struct DecodePlan {
  int group, qpt, n_qtiles, rt, rcp, key_tile, n_splits, split_tiles;
  long long units;  // (batch, kv head, query tile) units
};

int decode_key_tile(int d) { return d == 256 ? 64 : 128; }

// Key tiles visible to query tile qt (rows qt * qpt .. +qpt-1).
int decode_tiles(const MaskSpec& m, int Nq, int qpt, int qt, int bn) {
  const int i0 = qt * qpt, i1 = (qt + 1) * qpt - 1 < Nq - 1 ? (qt + 1) * qpt - 1 : Nq - 1;
  const int lo = m.lo(i0), hi = m.hi(i1);
  return hi >= lo ? hi / bn - lo / bn + 1 : 0;
}

// Key splits.  Every split of a unit takes `split_tiles` key tiles (the
// last one the rest), so a unit with fewer visible tiles -- a shorter
// sequence under per-sequence cache lengths -- uses fewer CTAs.
// n_splits <= 0 lets the library choose: with fewer (batch, kv head, query
// tile) units than SMs, the widest unit's tiles are split so that about one
// wave of CTAs (one per SM) streams K and V, keeping at least 4 key tiles per
// split so the copy ring fills.  With per-sequence lengths (ragged) the
// target is 3 waves' worth at full length, so the longest sequences are cut
// finely enough to balance (on 16 sequences of uniformly random length, 3
// waves came within 1% of the best split count, 1 wave was 34% slower).
int plan_decode(int B, int Nq, int Hq, int Hkv, int d, const MaskSpec& m, int n_splits, int sm_count,
                bool ragged, DecodePlan* pl) {
  pl->group = Hq / Hkv;
  if (pl->group > 128) return FA_ERR_UNSUPPORTED;
  pl->qpt = 128 / pl->group < Nq ? 128 / pl->group : Nq;
  pl->n_qtiles = (Nq + pl->qpt - 1) / pl->qpt;
  pl->rt = pl->qpt * pl->group;
  pl->rcp = pl->rt <= 32 ? 32 : pl->rt <= 64 ? 64 : 128;
  pl->key_tile = decode_key_tile(d);
  pl->units = static_cast<long long>(B) * Hkv * pl->n_qtiles;
  if (n_splits > kMaxDecodeSplits) return FA_ERR_INVALID_ARG;
  // the widest query tile's visible key tiles (at full capacity)
  int tiles = 0;
  for (int qt = 0; qt < pl->n_qtiles; ++qt) {
    const int t = decode_tiles(m, Nq, pl->qpt, qt, pl->key_tile);
    if (t > tiles) tiles = t;
  }
  long long n = n_splits;
  if (n_splits <= 0) {
    if (sm_count < 1) return FA_ERR_CUDA;
    const long long target = ragged ? 3ll * sm_count : sm_count;
    n = pl->units >= target ? 1 : (target + pl->units - 1) / pl->units;
    if (!ragged && pl->units < target) n = target / pl->units;
    const long long cap = tiles / 4 > 1 ? tiles / 4 : 1;
    if (n > cap) n = cap;
  }
  pl->split_tiles = tiles > 0 ? static_cast<int>((tiles + n - 1) / n) : 1;
  pl->n_splits = tiles > 0 ? (tiles + pl->split_tiles - 1) / pl->split_tiles : 1;
  if (pl->units * pl->n_splits > (1ll << 31) - 1) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

// Workspace of a split call: the partial O rows (fp32), their LSE, then one
// 8-byte counter per unit (16-byte aligned).
size_t decode_counters_offset(const DecodePlan& pl, int d) {
  const size_t rows = static_cast<size_t>(pl.units) * pl.n_splits * pl.rt;
  return (rows * d * sizeof(float) + rows * sizeof(float) + 15) / 16 * 16;
}

size_t decode_workspace_bytes(const DecodePlan& pl, int d) {
  if (pl.n_splits <= 1) return 0;
  return decode_counters_offset(pl, d) + static_cast<size_t>(pl.units) * sizeof(unsigned long long);
}

// Tag of one split call, so counters left by an earlier call read as zero.
unsigned int next_decode_tag() {
  static std::atomic<unsigned int> counter{0};
  unsigned int t = counter.fetch_add(1, std::memory_order_relaxed) + 1;
  if (t == 0) t = counter.fetch_add(1, std::memory_order_relaxed) + 1;
  return t;
}

template <class C>
int launch_decode_cfg(const void* q, const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& p,
                      long long grid, cudaStream_t stream) {
  static int attr_done[kMaxDevices] = {0};
  auto kern = fa_decode_kernel<C>;
  if (smem_attr_once(kern, C::SMEM_BYTES, attr_done) != cudaSuccess) return FA_ERR_CUDA;
  TraceScope tr(FA_KERNEL_DECODE, stream);
  kern<<<static_cast<unsigned>(grid), C::NTHREADS, C::SMEM_BYTES, stream>>>(
      static_cast<const uint16_t*>(q), tk, tv, p);
  return launch_status();
}

template <int D, template <int> class Cfg, bool F16>
int launch_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Nq,
                  int Nk, int Hq, int Hkv, float scale, const MaskSpec& mask, const DecodePlan& pl,
                  const int* seqlens, int n_new, void* workspace, cudaStream_t stream) {
  CUtensorMap tk, tv;
  const int bn = Cfg<32>::BN;
  if (!encode_bnhd(&tk, k, B, Nk, Hkv, D, bn, tma_type(F16)) || !encode_bnhd(&tv, v, B, Nk, Hkv, D, bn, tma_type(F16)))
    return FA_ERR_CUDA;
  DecodeParams p;
  p.B = B; p.Nq = Nq; p.Nk = Nk; p.Hq = Hq; p.Hkv = Hkv; p.group = pl.group;
  p.qpt = pl.qpt;
  p.n_qtiles = pl.n_qtiles;
  p.n_splits = pl.n_splits;
  p.split_tiles = pl.split_tiles;
  p.scale_log2 = scale * kLog2e;
  p.mask = mask;
  p.seqlens = seqlens;
  p.n_new = n_new;
  p.o = static_cast<uint16_t*>(o);
  p.lse = lse;
  const size_t rows = static_cast<size_t>(pl.units) * pl.n_splits * pl.rt;
  const bool split = pl.n_splits > 1;
  p.part_o = split ? static_cast<float*>(workspace) : nullptr;
  p.part_lse = split ? static_cast<float*>(workspace) + rows * D : nullptr;
  p.counters = split ? reinterpret_cast<unsigned long long*>(static_cast<char*>(workspace) +
                                                             decode_counters_offset(pl, D))
                     : nullptr;
  p.tag = next_decode_tag();
  p.wait_limit_ns = kWaitLimitNs;
  const long long grid = pl.units * pl.n_splits;
  switch (pl.rcp) {
    case 32: return launch_decode_cfg<Ty<F16, Cfg<32>>>(q, tk, tv, p, grid, stream);
    case 64: return launch_decode_cfg<Ty<F16, Cfg<64>>>(q, tk, tv, p, grid, stream);
    default: return launch_decode_cfg<Ty<F16, Cfg<128>>>(q, tk, tv, p, grid, stream);
  }
}

}  // namespace

// ------------------------------------------------- allocation-free backward
// Scratch of fa_bwd_noalloc: the D and lse2 rows the backward preprocess
// writes, held in a fixed array that is part of the library's device image
// (every GPU that loads the library keeps these 16 MiB until the process
// exits).  Host code must not hand the symbol itself to a kernel: on the host
// it only names a stand-in, so the device address is looked up with
// cudaGetSymbolAddress, once per device, with that device current.
constexpr size_t kNoAllocScratchBytes = 16u << 20;
static __device__ __align__(256) unsigned char g_bwd_scratch[kNoAllocScratchBytes];

namespace {
std::mutex g_scratch_mu;
float* g_scratch_ptr[kMaxDevices] = {nullptr};

int scratch_for_current_device(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_bwd_scratch) != cudaSuccess || p == nullptr) return FA_ERR_CUDA;
    g_scratch_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_scratch_ptr[dev];
  return FA_OK;
}
}  // namespace

namespace {

template <bool F16>
int fa_fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Nq, int Nk,
           int Hq, int Hkv, int d, float scale, int causal, int win_l, int win_r,
           fa_stream_t stream) {
  int st = check_common(q, k, v, B, Nq, Nk, Hq, Hkv, scale);
  if (st != FA_OK) return st;
  if (!aligned16(o) || !aligned16(lse)) return FA_ERR_INVALID_ARG;
  const MaskSpec mask = make_mask(Nq, Nk, causal, win_l, win_r);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  switch (d) {
    case 64: return launch_fwd<Ty<F16, Fwd64>>(q, k, v, o, lse, B, Nq, Nk, Hq, Hkv, scale, mask, s);
    case 128: return launch_fwd<Ty<F16, Fwd128>>(q, k, v, o, lse, B, Nq, Nk, Hq, Hkv, scale, mask, s);
    case 256: return launch_fwd<Ty<F16, Fwd256>>(q, k, v, o, lse, B, Nq, Nk, Hq, Hkv, scale, mask, s);
    default: return FA_ERR_UNSUPPORTED;
  }
}

template <bool F16>
int fa_bwd_impl(const void* q, const void* k, const void* v, const void* o, const float* lse,
           const void* dO, void* dq, void* dk, void* dv, int B, int Nq, int Nk, int Hq, int Hkv,
           int d, float scale, int causal, int win_l, int win_r, void* workspace,
           size_t workspace_bytes_, fa_stream_t stream) {
  int st = check_common(q, k, v, B, Nq, Nk, Hq, Hkv, scale);
  if (st != FA_OK) return st;
  if (!aligned16(o) || !aligned16(lse) || !aligned16(dO) || !aligned16(dq) || !aligned16(dk) ||
      !aligned16(dv))
    return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  if (!aligned16(workspace) || workspace_bytes_ < workspace_bytes(B, Nq, Hq)) return FA_ERR_WORKSPACE;
  const MaskSpec mask = make_mask(Nq, Nk, causal, win_l, win_r);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  float* ws = static_cast<float*>(workspace);
  switch (d) {
    case 64:
      return launch_bwd<Ty<F16, Dq64>, Ty<F16, Dkv64>>(q, k, v, o, lse, dO, dq, dk, dv, B, Nq, Nk, Hq, Hkv, scale, mask, ws, s);
    case 128:
      return launch_bwd<Ty<F16, Dq128>, Ty<F16, Dkv128>>(q, k, v, o, lse, dO, dq, dk, dv, B, Nq, Nk, Hq, Hkv, scale, mask, ws, s);
    default:
      return launch_bwd<Ty<F16, Dq256>, Ty<F16, Dkv256>>(q, k, v, o, lse, dO, dq, dk, dv, B, Nq, Nk, Hq, Hkv, scale, mask, ws, s);
  }
}

template <bool F16>
int fa_fwd_splitkv_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Nq,
                   int Nk, int Hq, int Hkv, int d, float scale, int causal, int win_l, int win_r,
                   int n_splits, void* workspace, size_t workspace_bytes_, fa_stream_t stream) {
  int st = check_common(q, k, v, B, Nq, Nk, Hq, Hkv, scale);
  if (st != FA_OK) return st;
  if (!aligned16(o) || !aligned16(lse)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  const MaskSpec mask = make_mask(Nq, Nk, causal, win_l, win_r);
  DecodePlan pl;
  st = plan_decode(B, Nq, Hq, Hkv, d, mask, n_splits, n_splits > 0 ? 0 : current_sm_count(), false, &pl);
  if (st != FA_OK) return st;
  const size_t need = decode_workspace_bytes(pl, d);
  if (need > 0 && (!aligned16(workspace) || workspace_bytes_ < need)) return FA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  switch (d) {
    case 64:
      return launch_decode<64, Dec64, F16>(q, k, v, o, lse, B, Nq, Nk, Hq, Hkv, scale, mask, pl, nullptr, 0, workspace, s);
    case 128:
      return launch_decode<128, Dec128, F16>(q, k, v, o, lse, B, Nq, Nk, Hq, Hkv, scale, mask, pl, nullptr, 0, workspace, s);
    default:
      return launch_decode<256, Dec256, F16>(q, k, v, o, lse, B, Nq, Nk, Hq, Hkv, scale, mask, pl, nullptr, 0, workspace, s);
  }
}

template <bool F16>
int fa_fwd_kvcache_impl(const void* q, void* k_cache, void* v_cache, const void* k_new, const void* v_new,
                   const int* cache_seqlens, void* o, float* lse, int B, int Nq, int Nk, int n_new,
                   int Hq, int Hkv, int d, float scale, int causal, int win_l, int win_r, int n_splits,
                   void* workspace, size_t workspace_bytes_, fa_stream_t stream) {
  int st = check_common(q, k_cache, v_cache, B, Nq, Nk, Hq, Hkv, scale);
  if (st != FA_OK) return st;
  if (!aligned16(o) || !aligned16(lse)) return FA_ERR_INVALID_ARG;
  if (n_new < 0) return FA_ERR_INVALID_ARG;
  if (n_new > 0 && (!aligned16(k_new) || !aligned16(v_new) || cache_seqlens == nullptr))
    return FA_ERR_INVALID_ARG;
  if (cache_seqlens != nullptr && (reinterpret_cast<uintptr_t>(cache_seqlens) & 3u) != 0) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  const MaskSpec mask = make_mask(Nq, Nk, causal, win_l, win_r);
  DecodePlan pl;
  st = plan_decode(B, Nq, Hq, Hkv, d, mask, n_splits, n_splits > 0 ? 0 : current_sm_count(),
                   cache_seqlens != nullptr, &pl);
  if (st != FA_OK) return st;
  const size_t need = decode_workspace_bytes(pl, d);
  if (need > 0 && (!aligned16(workspace) || workspace_bytes_ < need)) return FA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (n_new > 0) {
    const long long units = static_cast<long long>(B) * n_new * Hkv * (d / 8);
    const long long blocks = (units + 255) / 256 < 4096 ? (units + 255) / 256 : 4096;
    TraceScope tr(FA_KERNEL_KVCACHE_APPEND, s);
    fa_kvcache_append_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(
        static_cast<uint16_t*>(k_cache), static_cast<uint16_t*>(v_cache),
        static_cast<const uint16_t*>(k_new), static_cast<const uint16_t*>(v_new), cache_seqlens, B,
        n_new, Nk, Hkv, d);
    if (launch_status() != FA_OK) return FA_ERR_CUDA;
  }
  switch (d) {
    case 64:
      return launch_decode<64, Dec64, F16>(q, k_cache, v_cache, o, lse, B, Nq, Nk, Hq, Hkv, scale, mask, pl,
                                      cache_seqlens, n_new, workspace, s);
    case 128:
      return launch_decode<128, Dec128, F16>(q, k_cache, v_cache, o, lse, B, Nq, Nk, Hq, Hkv, scale, mask, pl,
                                        cache_seqlens, n_new, workspace, s);
    default:
      return launch_decode<256, Dec256, F16>(q, k_cache, v_cache, o, lse, B, Nq, Nk, Hq, Hkv, scale, mask, pl,
                                        cache_seqlens, n_new, workspace, s);
  }
}

template <bool F16>
int fa_fwd_varlen_impl(const void* q, const void* k, const void* v, void* o, float* lse,
                  const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int max_seqlen_q,
                  int max_seqlen_k, int total_q, int total_k, int Hq, int Hkv, int d, float scale,
                  int causal, int win_l, int win_r, fa_stream_t stream) {
  int st = check_common(q, k, v, 1, total_q, total_k, Hq, Hkv, scale);
  if (st != FA_OK) return st;
  if (!aligned16(o) || !aligned16(lse)) return FA_ERR_INVALID_ARG;
  if (cu_seqlens_q == nullptr || cu_seqlens_k == nullptr ||
      (reinterpret_cast<uintptr_t>(cu_seqlens_q) & 3u) != 0 || (reinterpret_cast<uintptr_t>(cu_seqlens_k) & 3u) != 0)
    return FA_ERR_INVALID_ARG;
  if (B < 1 || max_seqlen_q < 1 || max_seqlen_k < 1 || max_seqlen_q > total_q || max_seqlen_k > total_k)
    return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * Hq * ((max_seqlen_q + 127) / 128) > (1ll << 31) - 1) return FA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  switch (d) {
    case 64:
      return launch_fwd_varlen<Ty<F16, Fwd64>>(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, B, max_seqlen_q, max_seqlen_k,
                                      total_q, total_k, Hq, Hkv, scale, causal, win_l, win_r, s);
    case 128:
      return launch_fwd_varlen<Ty<F16, Fwd128>>(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, B, max_seqlen_q, max_seqlen_k,
                                       total_q, total_k, Hq, Hkv, scale, causal, win_l, win_r, s);
    case 256:
      return launch_fwd_varlen<Ty<F16, Fwd256>>(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, B, max_seqlen_q, max_seqlen_k,
                                       total_q, total_k, Hq, Hkv, scale, causal, win_l, win_r, s);
    default:
      return FA_ERR_UNSUPPORTED;
  }
}

template <bool F16>
int fa_bwd_varlen_impl(const void* q, const void* k, const void* v, const void* o, const float* lse,
                  const void* dO, void* dq, void* dk, void* dv, const int* cu_seqlens_q,
                  const int* cu_seqlens_k, int B, int max_seqlen_q, int max_seqlen_k, int total_q,
                  int total_k, int Hq, int Hkv, int d, float scale, int causal, int win_l, int win_r,
                  void* workspace, size_t workspace_bytes_, fa_stream_t stream) {
  int st = check_common(q, k, v, 1, total_q, total_k, Hq, Hkv, scale);
  if (st != FA_OK) return st;
  if (!aligned16(o) || !aligned16(lse) || !aligned16(dO) || !aligned16(dq) || !aligned16(dk) ||
      !aligned16(dv))
    return FA_ERR_INVALID_ARG;
  if (cu_seqlens_q == nullptr || cu_seqlens_k == nullptr ||
      (reinterpret_cast<uintptr_t>(cu_seqlens_q) & 3u) != 0 || (reinterpret_cast<uintptr_t>(cu_seqlens_k) & 3u) != 0)
    return FA_ERR_INVALID_ARG;
  if (B < 1 || max_seqlen_q < 1 || max_seqlen_k < 1 || max_seqlen_q > total_q || max_seqlen_k > total_k)
    return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * Hq * ((max_seqlen_q + 127) / 128) > (1ll << 31) - 1 ||
      static_cast<long long>(B) * Hkv * ((max_seqlen_k + 63) / 64) > (1ll << 31) - 1)
    return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  if (!aligned16(workspace) || workspace_bytes_ < workspace_bytes(B, max_seqlen_q, Hq)) return FA_ERR_WORKSPACE;
  const MaskSpec mask = make_mask(max_seqlen_q, max_seqlen_k, causal, win_l, win_r);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  float* ws = static_cast<float*>(workspace);
  Varlen vl;
  vl.cu_q = cu_seqlens_q;
  vl.cu_k = cu_seqlens_k;
  vl.total_q = total_q;
  vl.total_k = total_k;
  const int Nq = max_seqlen_q, Nk = max_seqlen_k;
  switch (d) {
    case 64:
      return launch_bwd<Ty<F16, Dq64>, Ty<F16, Dkv64>, true>(q, k, v, o, lse, dO, dq, dk, dv, B, Nq, Nk, Hq, Hkv, scale, mask, ws, s, vl);
    case 128:
      return launch_bwd<Ty<F16, Dq128>, Ty<F16, Dkv128>, true>(q, k, v, o, lse, dO, dq, dk, dv, B, Nq, Nk, Hq, Hkv, scale, mask, ws, s, vl);
    default:
      return launch_bwd<Ty<F16, Dq256>, Ty<F16, Dkv256>, true>(q, k, v, o, lse, dO, dq, dk, dv, B, Nq, Nk, Hq, Hkv, scale, mask, ws, s, vl);
  }
}

template <bool F16>
int fa_fwd_blocksparse_impl(const void* q, const void* k, const void* v, void* o, float* lse,
                            const unsigned char* block_mask, long long mask_stride_b,
                            long long mask_stride_h, int B, int Nq, int Nk, int Hq, int Hkv, int d,
                            float scale, int causal, int win_l, int win_r, fa_stream_t stream) {
  int st = check_common(q, k, v, B, Nq, Nk, Hq, Hkv, scale);
  if (st != FA_OK) return st;
  if (!aligned16(o) || !aligned16(lse) || block_mask == nullptr) return FA_ERR_INVALID_ARG;
  if (mask_stride_b < 0 || mask_stride_h < 0) return FA_ERR_INVALID_ARG;
  const MaskSpec mask = make_mask(Nq, Nk, causal, win_l, win_r);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const uint8_t* bm = reinterpret_cast<const uint8_t*>(block_mask);
  switch (d) {
    case 64:
      return launch_fwd_bs<Ty<F16, FwdBs64>>(q, k, v, o, lse, B, Nq, Nk, Hq, Hkv, scale, mask, bm, mask_stride_b,
                                           mask_stride_h, s);
    case 128:
      return launch_fwd_bs<Ty<F16, FwdBs128>>(q, k, v, o, lse, B, Nq, Nk, Hq, Hkv, scale, mask, bm, mask_stride_b,
                                            mask_stride_h, s);
    case 256:
      return launch_fwd_bs<Ty<F16, Fwd256>>(q, k, v, o, lse, B, Nq, Nk, Hq, Hkv, scale, mask, bm, mask_stride_b,
                                            mask_stride_h, s);
    default:
      return FA_ERR_UNSUPPORTED;
  }
}

template <bool F16>
int fa_bwd_blocksparse_impl(const void* q, const void* k, const void* v, const void* o, const float* lse,
                            const void* dO, void* dq, void* dk, void* dv, const unsigned char* block_mask,
                            long long mask_stride_b, long long mask_stride_h, int B, int Nq, int Nk, int Hq,
                            int Hkv, int d, float scale, int causal, int win_l, int win_r, void* workspace,
                            size_t workspace_bytes_, fa_stream_t stream) {
  int st = check_common(q, k, v, B, Nq, Nk, Hq, Hkv, scale);
  if (st != FA_OK) return st;
  if (!aligned16(o) || !aligned16(lse) || !aligned16(dO) || !aligned16(dq) || !aligned16(dk) ||
      !aligned16(dv) || block_mask == nullptr || mask_stride_b < 0 || mask_stride_h < 0)
    return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  if (!aligned16(workspace) || workspace_bytes_ < workspace_bytes(B, Nq, Hq)) return FA_ERR_WORKSPACE;
  const MaskSpec mask = make_mask(Nq, Nk, causal, win_l, win_r);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  float* ws = static_cast<float*>(workspace);
  BlockMask bm;
  bm.mask = reinterpret_cast<const uint8_t*>(block_mask);
  bm.sb = mask_stride_b;
  bm.sh = mask_stride_h;
  const Varlen vl;
  switch (d) {
    case 64:
      return launch_bwd<Ty<F16, Dq64>, Ty<F16, Dkv64>, false, true>(q, k, v, o, lse, dO, dq, dk, dv, B, Nq, Nk, Hq,
                                                                    Hkv, scale, mask, ws, s, vl, bm);
    case 128:
      return launch_bwd<Ty<F16, Dq128>, Ty<F16, Dkv128>, false, true>(q, k, v, o, lse, dO, dq, dk, dv, B, Nq, Nk,
                                                                      Hq, Hkv, scale, mask, ws, s, vl, bm);
    default:
      return launch_bwd<Ty<F16, Dq256>, Ty<F16, Dkv256>, false, true>(q, k, v, o, lse, dO, dq, dk, dv, B, Nq, Nk,
                                                                      Hq, Hkv, scale, mask, ws, s, vl, bm);
  }
}

}  // namespace

extern "C" {

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Nq, int Nk,
           int Hq, int Hkv, int d, float scale, int causal, int win_l, int win_r,
           fa_stream_t stream) {
  return fa_fwd_impl<false>(q, k, v, o, lse, B, Nq, Nk, Hq, Hkv, d, scale, causal, win_l, win_r, stream);
}

int fa_fwd_f16(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Nq, int Nk,
           int Hq, int Hkv, int d, float scale, int causal, int win_l, int win_r,
           fa_stream_t stream) {
  return fa_fwd_impl<true>(q, k, v, o, lse, B, Nq, Nk, Hq, Hkv, d, scale, causal, win_l, win_r, stream);
}

size_t fa_bwd_workspace_size(int B, int Nq, int Hq, int d) {
  if (d < 1) return 0;
  return workspace_bytes(B, Nq, Hq);
}

int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
           const void* dO, void* dq, void* dk, void* dv, int B, int Nq, int Nk, int Hq, int Hkv,
           int d, float scale, int causal, int win_l, int win_r, void* workspace,
           size_t workspace_bytes_, fa_stream_t stream) {
  return fa_bwd_impl<false>(q, k, v, o, lse, dO, dq, dk, dv, B, Nq, Nk, Hq, Hkv, d, scale, causal, win_l, win_r, workspace, workspace_bytes_, stream);
}

int fa_bwd_f16(const void* q, const void* k, const void* v, const void* o, const float* lse,
           const void* dO, void* dq, void* dk, void* dv, int B, int Nq, int Nk, int Hq, int Hkv,
           int d, float scale, int causal, int win_l, int win_r, void* workspace,
           size_t workspace_bytes_, fa_stream_t stream) {
  return fa_bwd_impl<true>(q, k, v, o, lse, dO, dq, dk, dv, B, Nq, Nk, Hq, Hkv, d, scale, causal, win_l, win_r, workspace, workspace_bytes_, stream);
}

int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                   const void* dO, void* dq, void* dk, void* dv, int B, int Nq, int Nk, int Hq,
                   int Hkv, int d, float scale, int causal, int win_l, int win_r,
                   fa_stream_t stream) {
  int st = check_common(q, k, v, B, Nq, Nk, Hq, Hkv, scale);
  if (st != FA_OK) return st;
  if (!aligned16(o) || !aligned16(lse) || !aligned16(dO) || !aligned16(dq) || !aligned16(dk) ||
      !aligned16(dv))
    return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  if (workspace_bytes(B, Nq, Hq) > kNoAllocScratchBytes) return FA_ERR_WORKSPACE;
  float* ws = nullptr;
  st = scratch_for_current_device(&ws);
  if (st != FA_OK) return st;
  // Every D / lse2 entry the kernels read is written by the preprocess kernel
  // of the same call first, so nothing in the shared array needs clearing.
  const MaskSpec mask = make_mask(Nq, Nk, causal, win_l, win_r);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  switch (d) {
    case 64:
      return launch_bwd<Dq64, Dkv64>(q, k, v, o, lse, dO, dq, dk, dv, B, Nq, Nk, Hq, Hkv, scale, mask, ws, s);
    case 128:
      return launch_bwd<Dq128, Dkv128>(q, k, v, o, lse, dO, dq, dk, dv, B, Nq, Nk, Hq, Hkv, scale, mask, ws, s);
    default:
      return launch_bwd<Dq256, Dkv256>(q, k, v, o, lse, dO, dq, dk, dv, B, Nq, Nk, Hq, Hkv, scale, mask, ws, s);
  }
}

static size_t splitkv_workspace(int B, int Nq, int Nk, int Hq, int Hkv, int d, int causal, int win_l,
                                int win_r, int n_splits, bool ragged) {
  if (B < 1 || Nq < 1 || Nk < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return 0;
  if (d != 64 && d != 128 && d != 256) return 0;
  DecodePlan pl;
  const MaskSpec mask = make_mask(Nq, Nk, causal, win_l, win_r);
  if (plan_decode(B, Nq, Hq, Hkv, d, mask, n_splits, n_splits > 0 ? 0 : current_sm_count(), ragged, &pl) !=
      FA_OK)
    return 0;
  return decode_workspace_bytes(pl, d);
}

size_t fa_fwd_splitkv_workspace_size(int B, int Nq, int Nk, int Hq, int Hkv, int d, int causal,
                                      int win_l, int win_r, int n_splits) {
  return splitkv_workspace(B, Nq, Nk, Hq, Hkv, d, causal, win_l, win_r, n_splits, false);
}

size_t fa_fwd_kvcache_workspace_size(int B, int Nq, int Nk, int Hq, int Hkv, int d, int causal,
                                     int win_l, int win_r, int n_splits, int with_seqlens) {
  return splitkv_workspace(B, Nq, Nk, Hq, Hkv, d, causal, win_l, win_r, n_splits, with_seqlens != 0);
}

int fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Nq,
                   int Nk, int Hq, int Hkv, int d, float scale, int causal, int win_l, int win_r,
                   int n_splits, void* workspace, size_t workspace_bytes_, fa_stream_t stream) {
  return fa_fwd_splitkv_impl<false>(q, k, v, o, lse, B, Nq, Nk, Hq, Hkv, d, scale, causal, win_l, win_r, n_splits, workspace, workspace_bytes_, stream);
}

int fa_fwd_splitkv_f16(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Nq,
                   int Nk, int Hq, int Hkv, int d, float scale, int causal, int win_l, int win_r,
                   int n_splits, void* workspace, size_t workspace_bytes_, fa_stream_t stream) {
  return fa_fwd_splitkv_impl<true>(q, k, v, o, lse, B, Nq, Nk, Hq, Hkv, d, scale, causal, win_l, win_r, n_splits, workspace, workspace_bytes_, stream);
}

int fa_fwd_kvcache(const void* q, void* k_cache, void* v_cache, const void* k_new, const void* v_new,
                   const int* cache_seqlens, void* o, float* lse, int B, int Nq, int Nk, int n_new,
                   int Hq, int Hkv, int d, float scale, int causal, int win_l, int win_r, int n_splits,
                   void* workspace, size_t workspace_bytes_, fa_stream_t stream) {
  return fa_fwd_kvcache_impl<false>(q, k_cache, v_cache, k_new, v_new, cache_seqlens, o, lse, B, Nq, Nk, n_new, Hq, Hkv, d, scale, causal, win_l, win_r, n_splits, workspace, workspace_bytes_, stream);
}

int fa_fwd_kvcache_f16(const void* q, void* k_cache, void* v_cache, const void* k_new, const void* v_new,
                   const int* cache_seqlens, void* o, float* lse, int B, int Nq, int Nk, int n_new,
                   int Hq, int Hkv, int d, float scale, int causal, int win_l, int win_r, int n_splits,
                   void* workspace, size_t workspace_bytes_, fa_stream_t stream) {
  return fa_fwd_kvcache_impl<true>(q, k_cache, v_cache, k_new, v_new, cache_seqlens, o, lse, B, Nq, Nk, n_new, Hq, Hkv, d, scale, causal, win_l, win_r, n_splits, workspace, workspace_bytes_, stream);
}

int fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                  const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int max_seqlen_q,
                  int max_seqlen_k, int total_q, int total_k, int Hq, int Hkv, int d, float scale,
                  int causal, int win_l, int win_r, fa_stream_t stream) {
  return fa_fwd_varlen_impl<false>(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, B, max_seqlen_q, max_seqlen_k, total_q, total_k, Hq, Hkv, d, scale, causal, win_l, win_r, stream);
}

int fa_fwd_varlen_f16(const void* q, const void* k, const void* v, void* o, float* lse,
                  const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int max_seqlen_q,
                  int max_seqlen_k, int total_q, int total_k, int Hq, int Hkv, int d, float scale,
                  int causal, int win_l, int win_r, fa_stream_t stream) {
  return fa_fwd_varlen_impl<true>(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, B, max_seqlen_q, max_seqlen_k, total_q, total_k, Hq, Hkv, d, scale, causal, win_l, win_r, stream);
}

int fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const float* lse,
                  const void* dO, void* dq, void* dk, void* dv, const int* cu_seqlens_q,
                  const int* cu_seqlens_k, int B, int max_seqlen_q, int max_seqlen_k, int total_q,
                  int total_k, int Hq, int Hkv, int d, float scale, int causal, int win_l, int win_r,
                  void* workspace, size_t workspace_bytes_, fa_stream_t stream) {
  return fa_bwd_varlen_impl<false>(q, k, v, o, lse, dO, dq, dk, dv, cu_seqlens_q, cu_seqlens_k, B, max_seqlen_q, max_seqlen_k, total_q, total_k, Hq, Hkv, d, scale, causal, win_l, win_r, workspace, workspace_bytes_, stream);
}

int fa_bwd_varlen_f16(const void* q, const void* k, const void* v, const void* o, const float* lse,
                  const void* dO, void* dq, void* dk, void* dv, const int* cu_seqlens_q,
                  const int* cu_seqlens_k, int B, int max_seqlen_q, int max_seqlen_k, int total_q,
                  int total_k, int Hq, int Hkv, int d, float scale, int causal, int win_l, int win_r,
                  void* workspace, size_t workspace_bytes_, fa_stream_t stream) {
  return fa_bwd_varlen_impl<true>(q, k, v, o, lse, dO, dq, dk, dv, cu_seqlens_q, cu_seqlens_k, B, max_seqlen_q, max_seqlen_k, total_q, total_k, Hq, Hkv, d, scale, causal, win_l, win_r, workspace, workspace_bytes_, stream);
}

int fa_fwd_blocksparse(const void* q, const void* k, const void* v, void* o, float* lse,
                       const unsigned char* block_mask, long long mask_stride_b, long long mask_stride_h,
                       int B, int Nq, int Nk, int Hq, int Hkv, int d, float scale, int causal, int win_l,
                       int win_r, fa_stream_t stream) {
  return fa_fwd_blocksparse_impl<false>(q, k, v, o, lse, block_mask, mask_stride_b, mask_stride_h, B, Nq, Nk, Hq,
                                        Hkv, d, scale, causal, win_l, win_r, stream);
}

int fa_fwd_blocksparse_f16(const void* q, const void* k, const void* v, void* o, float* lse,
                           const unsigned char* block_mask, long long mask_stride_b, long long mask_stride_h,
                           int B, int Nq, int Nk, int Hq, int Hkv, int d, float scale, int causal, int win_l,
                           int win_r, fa_stream_t stream) {
  return fa_fwd_blocksparse_impl<true>(q, k, v, o, lse, block_mask, mask_stride_b, mask_stride_h, B, Nq, Nk, Hq,
                                       Hkv, d, scale, causal, win_l, win_r, stream);
}

int fa_bwd_blocksparse(const void* q, const void* k, const void* v, const void* o, const float* lse,
                       const void* dO, void* dq, void* dk, void* dv, const unsigned char* block_mask,
                       long long mask_stride_b, long long mask_stride_h, int B, int Nq, int Nk, int Hq,
                       int Hkv, int d, float scale, int causal, int win_l, int win_r, void* workspace,
                       size_t workspace_bytes_, fa_stream_t stream) {
  return fa_bwd_blocksparse_impl<false>(q, k, v, o, lse, dO, dq, dk, dv, block_mask, mask_stride_b, mask_stride_h,
                                        B, Nq, Nk, Hq, Hkv, d, scale, causal, win_l, win_r, workspace,
                                        workspace_bytes_, stream);
}

int fa_bwd_blocksparse_f16(const void* q, const void* k, const void* v, const void* o, const float* lse,
                           const void* dO, void* dq, void* dk, void* dv, const unsigned char* block_mask,
                           long long mask_stride_b, long long mask_stride_h, int B, int Nq, int Nk, int Hq,
                           int Hkv, int d, float scale, int causal, int win_l, int win_r, void* workspace,
                           size_t workspace_bytes_, fa_stream_t stream) {
  return fa_bwd_blocksparse_impl<true>(q, k, v, o, lse, dO, dq, dk, dv, block_mask, mask_stride_b, mask_stride_h,
                                       B, Nq, Nk, Hq, Hkv, d, scale, causal, win_l, win_r, workspace,
                                       workspace_bytes_, stream);
}

int fa_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse, int B, int Nq,
               int Nk, int Hq, int Hkv, int d, float scale, int causal, int win_l, int win_r,
               fa_stream_t stream) {
  int st = check_common(q, k, v, B, Nq, Nk, Hq, Hkv, scale);
  if (st != FA_OK) return st;
  if (!aligned16(o) || !aligned16(lse)) return FA_ERR_INVALID_ARG;
  if (d < 32 || d > 32 * kF32MaxPerLane || d % 32 != 0) return FA_ERR_UNSUPPORTED;
  F32Params p;
  p.B = B; p.Nq = Nq; p.Nk = Nk; p.Hq = Hq; p.Hkv = Hkv; p.group = Hq / Hkv; p.d = d;
  p.scale = scale;
  p.scale_log2 = scale * kLog2e;
  p.mask = make_mask(Nq, Nk, causal, win_l, win_r);
  p.Nq_pad = pad_rows(Nq);
  p.D = nullptr;
  p.lse2 = nullptr;
  const long long warps = static_cast<long long>(B) * Nq * Hq;
  const long long blocks = (warps + 3) / 4;
  {
    TraceScope tr(FA_KERNEL_F32, reinterpret_cast<cudaStream_t>(stream));
    fa_fwd_f32_kernel<<<static_cast<unsigned>(blocks), 128, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        q, k, v, o, lse, p);
  }
  return launch_status();
}

int fa_bwd_f32(const float* q, const float* k, const float* v, const float* o, const float* lse,
               const float* dO, float* dq, float* dk, float* dv, int B, int Nq, int Nk, int Hq, int Hkv,
               int d, float scale, int causal, int win_l, int win_r, void* workspace,
               size_t workspace_bytes_, fa_stream_t stream) {
  int st = check_common(q, k, v, B, Nq, Nk, Hq, Hkv, scale);
  if (st != FA_OK) return st;
  if (!aligned16(o) || !aligned16(lse) || !aligned16(dO) || !aligned16(dq) || !aligned16(dk) ||
      !aligned16(dv))
    return FA_ERR_INVALID_ARG;
  if (d < 32 || d > 32 * kF32MaxPerLane || d % 32 != 0) return FA_ERR_UNSUPPORTED;
  if (!aligned16(workspace) || workspace_bytes_ < workspace_bytes(B, Nq, Hq)) return FA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  F32Params p;
  p.B = B; p.Nq = Nq; p.Nk = Nk; p.Hq = Hq; p.Hkv = Hkv; p.group = Hq / Hkv; p.d = d;
  p.scale = scale;
  p.scale_log2 = scale * kLog2e;
  p.mask = make_mask(Nq, Nk, causal, win_l, win_r);
  p.Nq_pad = pad_rows(Nq);
  float* ws = static_cast<float*>(workspace);
  const long long rows_pad = static_cast<long long>(B) * Hq * p.Nq_pad;
  p.D = ws;
  p.lse2 = ws + rows_pad;
  {
    TraceScope tr(FA_KERNEL_F32, s);
    fa_bwd_prep_kernel<float><<<static_cast<unsigned>((rows_pad * 32 + 255) / 256), 256, 0, s>>>(
        o, dO, lse, ws, B, Nq, Hq, d, p.Nq_pad);
  }
  if (launch_status() != FA_OK) return FA_ERR_CUDA;
  const long long wq = static_cast<long long>(B) * Nq * Hq;
  {
    TraceScope tr(FA_KERNEL_F32, s);
    fa_bwd_dq_f32_kernel<<<static_cast<unsigned>((wq + 3) / 4), 128, 0, s>>>(q, k, v, dO, dq, p);
  }
  if (launch_status() != FA_OK) return FA_ERR_CUDA;
  const long long wk = static_cast<long long>(B) * Nk * Hkv;
  {
    TraceScope tr(FA_KERNEL_F32, s);
    fa_bwd_dkdv_f32_kernel<<<static_cast<unsigned>((wk + 3) / 4), 128, 0, s>>>(q, k, v, dO, dk, dv, p);
  }
  return launch_status();
}

// ------------------------------------------------ ring attention: combining
}  // extern "C"

namespace {

template <bool F16>
int lse_merge_impl(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part, void* o_out, int B,
                   int Nq, int H, int d, int Nq_acc, int row0, int first, fa_stream_t stream) {
  if (!aligned16(o_acc) || !aligned16(lse_acc) || !aligned16(o_part) || !aligned16(lse_part) ||
      (o_out != nullptr && !aligned16(o_out)))
    return FA_ERR_INVALID_ARG;
  if (B < 1 || Nq < 1 || H < 1 || row0 < 0 || Nq_acc < Nq || row0 > Nq_acc - Nq) return FA_ERR_INVALID_ARG;
  const long long rows = static_cast<long long>(B) * Nq * H;
  if (static_cast<long long>(B) * Nq_acc * H > (1ll << 40)) return FA_ERR_INVALID_ARG;
  const long long blocks = (rows * 32 + 255) / 256;
  if (blocks > (1ll << 31) - 1) return FA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  auto* op = static_cast<const uint16_t*>(o_part);
  auto* oo = static_cast<uint16_t*>(o_out);
  TraceScope tr(FA_KERNEL_MERGE, s);
  const unsigned g = static_cast<unsigned>(blocks);
  switch (d) {
    case 64:
      fa_lse_merge_kernel<64, F16><<<g, 256, 0, s>>>(o_acc, lse_acc, op, lse_part, oo, B, Nq, H, Nq_acc, row0, first);
      break;
    case 128:
      fa_lse_merge_kernel<128, F16><<<g, 256, 0, s>>>(o_acc, lse_acc, op, lse_part, oo, B, Nq, H, Nq_acc, row0, first);
      break;
    case 256:
      fa_lse_merge_kernel<256, F16><<<g, 256, 0, s>>>(o_acc, lse_acc, op, lse_part, oo, B, Nq, H, Nq_acc, row0, first);
      break;
    default:
      return FA_ERR_UNSUPPORTED;
  }
  return launch_status();
}

template <bool F16>
int grad_accumulate_impl(float* acc, const void* part, void* out, int B, int rows_acc, int row0, int rows,
                         long long row_elems, int first, fa_stream_t stream) {
  if (!aligned16(acc) || (part != nullptr && !aligned16(part)) || (out != nullptr && !aligned16(out)))
    return FA_ERR_INVALID_ARG;
  if (part == nullptr && out == nullptr) return FA_ERR_INVALID_ARG;
  if (B < 1 || B > 65535 || rows < 1 || row0 < 0 || rows_acc < rows || row0 > rows_acc - rows)
    return FA_ERR_INVALID_ARG;
  if (row_elems < 8 || row_elems % 8 != 0 || row_elems > (1ll << 40) / rows_acc) return FA_ERR_INVALID_ARG;
  const long long blocks = (static_cast<long long>(rows) * row_elems / 8 + 255) / 256;
  if (blocks > (1ll << 31) - 1) return FA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  TraceScope tr(FA_KERNEL_MERGE, s);
  fa_grad_accumulate_kernel<F16><<<dim3(static_cast<unsigned>(blocks), static_cast<unsigned>(B)), 256, 0, s>>>(
      acc, static_cast<const uint16_t*>(part), static_cast<uint16_t*>(out), rows_acc, row0, rows, row_elems, first);
  return launch_status();
}

}  // namespace

extern "C" {

int fa_lse_merge(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part, void* o_out, int B,
                 int Nq, int H, int d, int Nq_acc, int row0, int first, fa_stream_t stream) {
  return lse_merge_impl<false>(o_acc, lse_acc, o_part, lse_part, o_out, B, Nq, H, d, Nq_acc, row0, first, stream);
}
int fa_lse_merge_f16(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part, void* o_out, int B,
                     int Nq, int H, int d, int Nq_acc, int row0, int first, fa_stream_t stream) {
  return lse_merge_impl<true>(o_acc, lse_acc, o_part, lse_part, o_out, B, Nq, H, d, Nq_acc, row0, first, stream);
}
int fa_grad_accumulate(float* acc, const void* part, void* out, int B, int rows_acc, int row0, int rows,
                       long long row_elems, int first, fa_stream_t stream) {
  return grad_accumulate_impl<false>(acc, part, out, B, rows_acc, row0, rows, row_elems, first, stream);
}
int fa_grad_accumulate_f16(float* acc, const void* part, void* out, int B, int rows_acc, int row0, int rows,
                           long long row_elems, int first, fa_stream_t stream) {
  return grad_accumulate_impl<true>(acc, part, out, B, rows_acc, row0, rows, row_elems, first, stream);
}

int fa_test_withhold_next_load(void) {
  g_test_withhold.store(1);
  return FA_OK;
}

int fa_get_device_status(fa_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return FA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  }
  return v == kDevTimeout ? FA_ERR_TIMEOUT : FA_OK;
}

int fa_trace_enable(int on) {
  std::lock_guard<std::mutex> lock(g_trace_mu);
  if (on && !g_trace_on) {
    while (static_cast<int>(g_event_pool.size()) < kEventPoolInit) {
      cudaEvent_t e;
      if (cudaEventCreate(&e) != cudaSuccess) return FA_ERR_CUDA;
      g_event_pool.push_back(e);
    }
  }
  g_trace_on = on != 0;
  return FA_OK;
}

int fa_trace_read(double* ms, long long* launches) {
  if (!ms || !launches) return FA_ERR_INVALID_ARG;
  for (int i = 0; i < FA_KERNEL_KINDS; ++i) {
    ms[i] = 0.0;
    launches[i] = 0;
  }
  std::lock_guard<std::mutex> lock(g_trace_mu);
  int st = FA_OK;
  for (const TraceRec& r : g_trace) {
    float t = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess)
      st = FA_ERR_CUDA;
    if (r.kind >= 0 && r.kind < FA_KERNEL_KINDS) {
      ms[r.kind] += t;
      launches[r.kind] += 1;
    }
    g_event_pool.push_back(r.a);
    g_event_pool.push_back(r.b);
  }
  g_trace.clear();
  return st;
}

const char* fa_status_string(int status) {
  switch (status) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_CUDA: return "FA_ERR_CUDA";
    case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT";
    default: return "FA_UNKNOWN_STATUS";
  }
}

}  // extern "C"
