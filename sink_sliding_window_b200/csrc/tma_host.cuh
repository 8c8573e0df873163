// Host-side construction of TMA tensor maps (cuTensorMapEncodeTiled, reached
// through the runtime's driver entry point so the library does not link
// libcuda directly).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

namespace sa {

// Devices per process the library keeps per-device state for.
constexpr int kMaxDevices = 64;

// Raises a kernel's dynamic shared-memory limit once per device.  The CUDA
// runtime applies cudaFuncSetAttribute to the function on the current
// device only, so a process that launches on several devices needs the call
// on each of them.  Thread-safe: the flags are atomics, and a race between
// two first calls on one device only repeats the (idempotent) call.
struct SmemAttrOnce {
  std::atomic<int> done[kMaxDevices] = {};

  template <typename K>
  bool ensure(K kernel, size_t bytes) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return false;
    if (dev < kMaxDevices && done[dev].load(std::memory_order_acquire)) return true;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes)) !=
        cudaSuccess)
      return false;
    if (dev < kMaxDevices) done[dev].store(1, std::memory_order_release);
    return true;
  }
};

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn get_encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// 3-D bf16 view [outer][mid][64] of a token-major tensor, 128B swizzle.
inline bool make_map_3d(CUtensorMap* map, const void* base, int inner, int mid, int outer, int box_mid, int box_outer) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(mid),
                        static_cast<cuuint64_t>(outer)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(inner) * 2, static_cast<cuuint64_t>(inner) * mid * 2};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(inner), static_cast<cuuint32_t>(box_mid),
                       static_cast<cuuint32_t>(box_outer)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D fp32 view [outer][mid][inner] with a box {32, box_mid, box_outer}
// (128 bytes innermost, 128B swizzle): the dq accumulator seen by the
// backward's TMA reduce-add.
inline bool make_map_3d_f32(CUtensorMap* map, const void* base, int inner, int mid, int outer, int box_mid,
                            int box_outer) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(mid),
                        static_cast<cuuint64_t>(outer)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(inner) * 4, static_cast<cuuint64_t>(inner) * mid * 4};
  cuuint32_t box[3] = {32, static_cast<cuuint32_t>(box_mid), static_cast<cuuint32_t>(box_outer)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D byte view [outer][mid][inner] (e.g. an e4m3 cache) with inner = 64: a
// box lands in shared memory as rows of 64 bytes under the 64-byte swizzle
// (16-byte chunk c of row r at chunk c ^ ((r >> 1) & 3); the destination must
// be 512-byte aligned).
inline bool make_map_3d_u8(CUtensorMap* map, const void* base, int inner, int mid, int outer, int box_mid,
                           int box_outer) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(mid),
                        static_cast<cuuint64_t>(outer)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(inner) * mid};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(inner), static_cast<cuuint32_t>(box_mid),
                       static_cast<cuuint32_t>(box_outer)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace sa
