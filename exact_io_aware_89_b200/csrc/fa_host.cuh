// fa_host.cuh -- host-side helpers of libfa: argument checks, TMA tensor-map
// encoding (through the driver entry point, so the library needs no -lcuda)
// and per-device kernel attribute setup.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/fa.h"

namespace fa {

inline bool aligned16(const void* ptr) {
  return ptr != nullptr && (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0;
}

inline int check_sizes(int B, int Nq, int Nk, int Hq, int Hkv, float scale) {
  if (B < 1 || Nq < 1 || Nk < 1 || Hq < 1 || Hkv < 1) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return FA_ERR_INVALID_ARG;
  // every index the kernels form stays inside 32-bit ints per tensor row/column
  if (static_cast<long long>(Nq) * Hq > (1ll << 31) - 1) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(Nk) * Hkv > (1ll << 31) - 1) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * Hq * ((Nq + 127) / 128) > (1ll << 31) - 1) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// A [B, N, H, d] bf16 tensor seen by TMA as 4-D {d, H, N, B}; one box is
// `box_rows` consecutive rows of one head and 64 elements (128 bytes) of d,
// stored in shared memory with the 128-byte swizzle.
inline bool encode_bnhd(CUtensorMap* map, const void* ptr, int B, int N, int H, int d,
                        int box_rows, CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                        int elem_bytes = 2, int box_inner = 64) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H),
                        static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(d) * elem_bytes,
                           static_cast<cuuint64_t>(H) * d * elem_bytes,
                           static_cast<cuuint64_t>(N) * H * d * elem_bytes};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(box_inner), 1u, static_cast<cuuint32_t>(box_rows), 1u};
  cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  CUresult r = enc(map, dtype, 4, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace fa
