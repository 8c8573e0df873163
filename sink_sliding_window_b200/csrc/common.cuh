// Shared definitions of the sink-attention kernels.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace sa {

constexpr int kHeadDim = 64;     // D
constexpr int kBlockM = 128;     // MMA rows per query tile: (128 / G) positions x G heads
constexpr int kBlockN = 128;     // keys per key/value tile
constexpr int kTileBytes = 128 * kHeadDim * 2;  // one [128][64] bf16 tile, 128 B per row
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Error code of the last timed-out device wait on this device (0 = none).
__device__ int g_device_error;

// Geometry of one call, shared by the kernels.
struct Geometry {
  int T;            // total tokens
  int Hq, Hkv;      // query / key-value heads
  int G_log2;       // log2(Hq / Hkv)
  int P_log2;       // log2(positions per query tile) = 7 - G_log2
  int num_qblocks;  // ceil(T / positions per query tile)
  int batch;        // documents
  int seqlen;       // common document length when cu_seqlens == nullptr
  const int* cu_seqlens;
  int window;       // <= 0: full causal
};

// First token of the document holding token t.
__device__ __forceinline__ int doc_start(const Geometry& g, int t) {
  if (g.cu_seqlens == nullptr) return (t / g.seqlen) * g.seqlen;
  int lo = 0, hi = g.batch - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(g.cu_seqlens + mid) <= t) lo = mid; else hi = mid - 1;
  }
  return __ldg(g.cu_seqlens + lo);
}

// First key query token t may attend to (absolute token index).
__device__ __forceinline__ int first_key(const Geometry& g, int t) {
  const int a = doc_start(g, t);
  return g.window > 0 ? max(a, t - g.window + 1) : a;
}

// Rounds a dynamic shared-memory pointer up to 1024 bytes (128B-swizzled
// tiles must start on a 1024-byte boundary).
__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

}  // namespace sa
