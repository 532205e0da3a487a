// Internal launch interface between the C-ABI layer (fv_api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "fv_common.cuh"

namespace fv {

// Workspace of the attention calls: a 256-byte header (word 0: tile-queue counter,
// word 1: error bits) followed by the LPT tile order and its sort keys.
constexpr size_t kWsHeader = 256;
inline size_t attn_ws_bytes(const Geo& g) {
  const size_t ntiles = static_cast<size_t>(g.B) * g.H * g.nB;
  return kWsHeader + ((ntiles * 8 + 255) / 256) * 256;
}

cudaError_t launch_pool(const Geo& g, const void* q, const void* k, float* qp, float* kp,
                        cudaStream_t st);
cudaError_t launch_route(const Geo& g, const float* qp, const float* kp, float p, int k_floor,
                         float scale, uint32_t* mask, int32_t* counts, cudaStream_t st);
// The same routing in two kernels (logits into `ws`, then selection); ws holds
// route_ws_bytes(g) bytes.
size_t route_ws_bytes(const Geo& g);
cudaError_t launch_route_ws(const Geo& g, const float* qp, const float* kp, float p, int k_floor,
                            float scale, uint32_t* mask, int32_t* counts, void* ws, cudaStream_t st);

// Pool and route in one persistent kernel; ws holds pool_route_ws_bytes(g) bytes (a
// header with the item queue, the error word and per-slice counters, then the logits).
size_t pool_route_ws_bytes(const Geo& g);
cudaError_t launch_pool_route(const Geo& g, const void* q, const void* k, float* qp, float* kp, float p,
                              int k_floor, float scale, uint32_t* mask, int32_t* counts, void* ws, int nsm,
                              cudaStream_t st);

struct AttnMaps {
  CUtensorMap q, qe, k, ke, v, ve;   // full-width and x-edge boxes of Q, K, V
};

// Launches the schedule prep and the persistent attention kernel.  mask == nullptr
// runs every key block (dense).
cudaError_t launch_attn(const Geo& g, const AttnMaps& maps, const uint32_t* mask, float scale,
                        void* out, float* lse, void* ws, unsigned long long* busy, int nsm,
                        cudaStream_t st);

}  // namespace fv
