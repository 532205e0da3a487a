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

// Options of the routing rule beyond Top-p / Top-k / own block (all off by default).
struct RouteOpts {
  int token_mass = 0;   // 1: Top-p over tokens (block masses weighted by real token counts)
  int kf_stride = 0;    // > 0: blocks holding a keyframe ((t - kf_phase) mod kf_stride == 0)
  int kf_phase = 0;     //      are kept in every row
};

cudaError_t launch_pool(const Geo& g, const void* q, const void* k, float* qp, float* kp,
                        cudaStream_t st);
cudaError_t launch_route(const Geo& g, const float* qp, const float* kp, float p, int k_floor,
                         float scale, uint32_t* mask, int32_t* counts, cudaStream_t st);
// The same routing in two kernels (tensor-core logits into `ws`, then selection by mass
// histogram); ws holds route_ws_bytes(g) bytes: a 256-byte header (word 1: error bits),
// then the logits.
size_t route_ws_bytes(const Geo& g);
cudaError_t launch_route_ws(const Geo& g, const float* qp, const float* kp, float p, int k_floor,
                            float scale, uint32_t* mask, int32_t* counts, void* ws, cudaStream_t st,
                            const RouteOpts& o = RouteOpts{});

// Routing logits of every (b, h) slice on the tensor cores (3xTF32 split): logits[b*h]
// [qb][kb] = (Qp[qb] . Kp[kb]) * scale, rows padded to words * 32.  err: the status word a
// bounded wait that gives up raises.
cudaError_t launch_logits_tc(const Geo& g, const float* qp, const float* kp, float scale, float* logits,
                             uint32_t* err, int nsm, cudaStream_t st);

// Runtime mask repair: fills one-block holes of every mask row (in place allowed) and
// rewrites counts.
cudaError_t launch_mask_repair(const Geo& g, const uint32_t* in, uint32_t* out, int32_t* counts,
                               cudaStream_t st);

// Pool, then the workspace route; ws holds pool_route_ws_bytes(g) bytes (the route
// workspace).
size_t pool_route_ws_bytes(const Geo& g);
cudaError_t launch_pool_route(const Geo& g, const void* q, const void* k, float* qp, float* kp, float p,
                              int k_floor, float scale, uint32_t* mask, int32_t* counts, void* ws, int nsm,
                              cudaStream_t st);

struct AttnMaps {
  CUtensorMap q, qe, k, ke, v, ve;   // full-width and x-edge boxes of Q, K, V
};

// Launches the schedule prep and the persistent attention kernel.  mask == nullptr
// runs every key block (dense).  stall_ns > 0 is the test hook of
// fvattn_testing_attn_stall: every CTA gives up a wait of that length and aborts.
cudaError_t launch_attn(const Geo& g, const AttnMaps& maps, const uint32_t* mask, float scale,
                        void* out, float* lse, void* ws, unsigned long long* busy, int nsm,
                        cudaStream_t st, unsigned long long stall_ns = 0);

}  // namespace fv
