// Internal launch interface between the C-ABI layer (fv_api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "fv_common.cuh"

namespace fv {

// Identifier of the calling thread's current driver context (0 when there is none).
unsigned long long current_ctx_id();

// TMA map over an fp32 [slices][rows][d] array: box 32 channels x 128 rows, 128-byte
// swizzle, rows past the end read as zero.  False when the driver refuses it.
bool encode_rows_fp32(CUtensorMap* m, const void* ptr, int slices, int rows, int d);

// Sets `fn`'s dynamic shared-memory limit to at least `bytes`, unless a limit at least that
// large was set already in the current context (the attribute lives with the context's copy
// of the function; setting it on every call costs host time).  `cache` holds, per device
// ordinal, the context id and the limit last set there.  carveout >= 0 also sets the
// preferred shared-memory carveout (percent of the unified L1 / shared array) with it.
struct SmemAttrCache {
  unsigned long long ctx[64];
  int bytes[64];
};
inline cudaError_t set_smem_once(const void* fn, int bytes, SmemAttrCache& cache, int carveout = -1) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool slot = dev >= 0 && dev < 64;
  const unsigned long long id = current_ctx_id();
  if (slot && id != 0 && cache.ctx[dev] == id && cache.bytes[dev] >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && carveout >= 0)
    e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, carveout);
  if (e == cudaSuccess && slot) {
    cache.ctx[dev] = current_ctx_id();
    cache.bytes[dev] = bytes;
  }
  return e;
}

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
// the logits, then the pooled rows split for the tensor cores.
size_t route_ws_bytes(const Geo& g);
cudaError_t launch_route_ws(const Geo& g, const float* qp, const float* kp, float p, int k_floor,
                            float scale, uint32_t* mask, int32_t* counts, void* ws, cudaStream_t st,
                            const RouteOpts& o = RouteOpts{});

// Routing logits of every (b, h) slice on the tensor cores (3xTF32 split): logits[b*h]
// [qb][kb] = (Qp[qb] . Kp[kb]) * scale, rows padded to words * 32.  split: 4 * B*H*nB*d
// floats of scratch (the pooled rows' tf32 high and low parts).  err: the status word a
// bounded wait that gives up raises.
size_t logits_split_bytes(const Geo& g);
cudaError_t launch_logits_tc(const Geo& g, const float* qp, const float* kp, float scale, float* logits,
                             float* split, uint32_t* err, int nsm, cudaStream_t st);

// Slack-aware augmentation of the final wave (fv_augment.cu).  logits: the route
// workspace's logits; scratch: augment_scratch_bytes(g) bytes.
size_t augment_scratch_bytes(const Geo& g);
cudaError_t launch_augment(const Geo& g, const float* logits, float tau, int n_sm, uint32_t* mask, int32_t* counts,
                           void* scratch, cudaStream_t st);

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
