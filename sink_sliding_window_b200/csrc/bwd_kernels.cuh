// Backward kernels (placeholder until the tcgen05 backward lands).
#pragma once
#include "common.cuh"

namespace sa {

constexpr int kBwdLaunches = 0;

struct BwdWorkspace {
  size_t total;
};

inline BwdWorkspace bwd_workspace_layout(const Geometry&) { return BwdWorkspace{256}; }

inline sink_attn_status bwd_launch(const Geometry&, float, const void*, const void*, const void*, const float*,
                                   const void*, const float*, const void*, void*, void*, void*, float*, uint8_t*,
                                   const BwdWorkspace&, cudaStream_t) {
  return SINK_ATTN_ERR_UNSUPPORTED;
}

}  // namespace sa
