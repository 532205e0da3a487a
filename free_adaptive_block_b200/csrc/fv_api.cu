// C-ABI entry points of libfvattn (declared in include/fvattn.h): argument checks on
// the host, TMA tensor-map encoding, kernel launches.  Nothing here allocates device
// memory or synchronises, except fvattn_device_status.
#include <cudaTypedefs.h>
#include <math.h>

#include <mutex>

#include "fv_launch.h"
#include "fvattn.h"
#include "fvattn_testing.h"

namespace {

using fv::Geo;

thread_local cudaError_t g_last_cuda_error = cudaSuccess;

fvattn_status_t cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return FVATTN_OK;
  g_last_cuda_error = e;
  return FVATTN_ERR_CUDA;
}

constexpr int kMaxBlocks = 2048;   // route keeps a row of nB scores per warp in shared memory

fvattn_status_t make_geo(const fvattn_geom_t* gi, Geo* g) {
  if (gi == nullptr) return FVATTN_ERR_INVALID_ARG;
  if (gi->B < 1 || gi->H < 1 || gi->T < 1 || gi->Hs < 1 || gi->Ws < 1 || gi->d < 1 ||
      gi->bt < 1 || gi->bh < 1 || gi->bw < 1)
    return FVATTN_ERR_INVALID_ARG;
  if (gi->d != 64 && gi->d != 128) return FVATTN_ERR_UNSUPPORTED;
  if (static_cast<long long>(gi->bt) * gi->bh * gi->bw > 128) return FVATTN_ERR_UNSUPPORTED;
  const long long N = static_cast<long long>(gi->T) * gi->Hs * gi->Ws;
  if (N >= (1LL << 31)) return FVATTN_ERR_UNSUPPORTED;
  if (gi->Ws > 65535 || gi->Hs > 65535 || gi->T > 32767) return FVATTN_ERR_UNSUPPORTED;
  Geo r;
  r.B = gi->B; r.H = gi->H; r.T = gi->T; r.Hs = gi->Hs; r.Ws = gi->Ws; r.d = gi->d;
  r.bt = gi->bt; r.bh = gi->bh; r.bw = gi->bw;
  r.nBt = (gi->T + gi->bt - 1) / gi->bt;
  r.nBy = (gi->Hs + gi->bh - 1) / gi->bh;
  r.nBx = (gi->Ws + gi->bw - 1) / gi->bw;
  const long long nB = static_cast<long long>(r.nBt) * r.nBy * r.nBx;
  if (nB > kMaxBlocks) return FVATTN_ERR_UNSUPPORTED;
  if (static_cast<long long>(gi->B) * gi->H * nB >= (1LL << 24)) return FVATTN_ERR_UNSUPPORTED;
  if (static_cast<long long>(gi->B) * gi->H * N * gi->d >= (1LL << 40)) return FVATTN_ERR_UNSUPPORTED;
  r.nB = static_cast<int>(nB);
  r.words = (r.nB + 31) / 32;
  r.r_nBx = 1.0f / static_cast<float>(r.nBx);
  r.r_plane = 1.0f / static_cast<float>(r.nBy * r.nBx);
  r.N = static_cast<int>(N);
  *g = r;
  return FVATTN_OK;
}

fvattn_status_t check_ptr(const void* p) {
  if (p == nullptr) return FVATTN_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(p) & 15u) return FVATTN_ERR_UNSUPPORTED;
  return FVATTN_OK;
}

// mask, counts and lse are read and written one 32-bit word at a time
fvattn_status_t check_ptr4(const void* p) {
  if (p == nullptr) return FVATTN_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(p) & 3u) return FVATTN_ERR_UNSUPPORTED;
  return FVATTN_OK;
}

#define FV_CHECK(expr)                       \
  do {                                       \
    const fvattn_status_t s_ = (expr);       \
    if (s_ != FVATTN_OK) return s_;          \
  } while (0)

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

}  // namespace

// 3D map over an fp32 [slices][rows][d] array (pooled rows split for the tensor cores): box
// 32 channels x 128 rows x 1 slice, 128-byte swizzle, rows past the slice's end read zero.
bool fv::encode_rows_fp32(CUtensorMap* m, const void* ptr, int slices, int rows, int d) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(slices)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 4, static_cast<cuuint64_t>(rows) * d * 4};
  cuuint32_t box[3] = {32u, 128u, 1u};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

namespace {

// 5D map over a bf16 [B*H][T][Hs][Ws][d] tensor; box = 64 channels x box_x columns x
// bh rows x bt frames x 1 slice, 128-byte swizzle, zero fill out of range.
bool encode_map(CUtensorMap* m, const void* ptr, const Geo& g, int box_x) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t es = 2;
  cuuint64_t dims[5] = {static_cast<cuuint64_t>(g.d), static_cast<cuuint64_t>(g.Ws),
                        static_cast<cuuint64_t>(g.Hs), static_cast<cuuint64_t>(g.T),
                        static_cast<cuuint64_t>(g.B) * g.H};
  cuuint64_t strides[4] = {g.d * es, static_cast<cuuint64_t>(g.Ws) * g.d * es,
                           static_cast<cuuint64_t>(g.Hs) * g.Ws * g.d * es,
                           static_cast<cuuint64_t>(g.T) * g.Hs * g.Ws * g.d * es};
  cuuint32_t box[5] = {64u, static_cast<cuuint32_t>(box_x), static_cast<cuuint32_t>(g.bh),
                       static_cast<cuuint32_t>(g.bt), 1u};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(ptr), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int current_num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

fvattn_status_t run_attn(const fvattn_geom_t* gi, const void* q, const void* k, const void* v,
                         const uint32_t* mask, float scale, void* out, float* lse, void* ws,
                         size_t ws_bytes, unsigned long long* busy, fvattn_stream_t stream,
                         unsigned long long stall_ns = 0) {
  Geo g;
  FV_CHECK(make_geo(gi, &g));
  FV_CHECK(check_ptr(q));
  FV_CHECK(check_ptr(k));
  FV_CHECK(check_ptr(v));
  FV_CHECK(check_ptr(out));
  FV_CHECK(check_ptr4(lse));
  if (mask != nullptr) FV_CHECK(check_ptr4(mask));
  if (busy != nullptr && (reinterpret_cast<uintptr_t>(busy) & 7u)) return FVATTN_ERR_UNSUPPORTED;
  if (!(scale > 0.f) || !isfinite(scale)) return FVATTN_ERR_INVALID_ARG;
  if (ws == nullptr || ws_bytes < fv::attn_ws_bytes(g)) return FVATTN_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) & 15u) return FVATTN_ERR_UNSUPPORTED;
  const int nsm = current_num_sms();
  if (nsm <= 0) return cuda_status(cudaGetLastError() == cudaSuccess ? cudaErrorNoDevice : cudaGetLastError());
  // The six tensor maps depend only on the geometry and the Q, K, V addresses: a thread
  // keeps the last set it encoded and reuses it while they stay the same.
  struct MapCache {
    unsigned long long ctx;
    const void *q, *k, *v;
    fvattn_geom_t g;
    fv::AttnMaps maps;
    bool valid;
  };
  thread_local MapCache mc = {};
  const unsigned long long ctx = fv::current_ctx_id();
  const bool hit = mc.valid && ctx != 0 && mc.ctx == ctx && mc.q == q && mc.k == k && mc.v == v &&
                   mc.g.B == gi->B && mc.g.H == gi->H && mc.g.T == gi->T && mc.g.Hs == gi->Hs &&
                   mc.g.Ws == gi->Ws && mc.g.d == gi->d && mc.g.bt == gi->bt && mc.g.bh == gi->bh &&
                   mc.g.bw == gi->bw;
  if (!hit) {
    const int rx_edge = g.Ws - (g.nBx - 1) * g.bw;
    mc.valid = false;
    if (!encode_map(&mc.maps.q, q, g, g.bw) || !encode_map(&mc.maps.qe, q, g, rx_edge) ||
        !encode_map(&mc.maps.k, k, g, g.bw) || !encode_map(&mc.maps.ke, k, g, rx_edge) ||
        !encode_map(&mc.maps.v, v, g, g.bw) || !encode_map(&mc.maps.ve, v, g, rx_edge))
      return FVATTN_ERR_CUDA;
    mc.ctx = ctx;
    mc.q = q;
    mc.k = k;
    mc.v = v;
    mc.g = *gi;
    mc.valid = true;
  }
  return cuda_status(fv::launch_attn(g, mc.maps, mask, scale, out, lse, ws, busy, nsm,
                                     reinterpret_cast<cudaStream_t>(stream), stall_ns));
}

// Scratch for fvattn_block_sparse_attn_noalloc: the tile queue, the error word and the
// LPT order live in this file-scope device array instead of a caller-provided workspace.
// Every device that loads the library holds it until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;   // 1 MiB: up to 131040 tiles
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
struct NoAllocSlot {
  unsigned long long ctx_id;   // driver context the address belongs to (0: none yet)
  void* addr;
};
NoAllocSlot g_noalloc_slot[kMaxDevices] = {};

// Identifier of the calling thread's current driver context (0 when there is none).  A
// device reset or a new context loads the library's module again, and the static array
// may then sit at another address, so the cached address is keyed on this identifier.
}  // namespace

unsigned long long fv::current_ctx_id() {
  static PFN_cuCtxGetCurrent_v4000 get_cur = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  if (get_cur == nullptr || get_id == nullptr) return 0;
  CUcontext ctx = nullptr;
  if (get_cur(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

namespace {

// Device address of g_noalloc_scratch in the current context.  Host code only holds a
// host-side stand-in for the symbol, so the address is asked of the runtime
// (cudaGetSymbolAddress) the first time a device's context is seen, and again whenever
// that device's current context has changed since (for instance after cudaDeviceReset).
fvattn_status_t noalloc_scratch(void** out) {
  int dev = 0;
  fvattn_status_t st = cuda_status(cudaGetDevice(&dev));
  if (st != FVATTN_OK) return st;
  if (dev < 0 || dev >= kMaxDevices) return FVATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoAllocSlot& slot = g_noalloc_slot[dev];
  const unsigned long long id = fv::current_ctx_id();
  if (slot.addr == nullptr || id == 0 || id != slot.ctx_id) {
    void* p = nullptr;
    st = cuda_status(cudaGetSymbolAddress(&p, g_noalloc_scratch));
    if (st != FVATTN_OK) return st;
    slot.addr = p;
    slot.ctx_id = fv::current_ctx_id();   // the runtime call made the primary context current
  }
  *out = slot.addr;
  return FVATTN_OK;
}

}  // namespace

extern "C" {

fvattn_status_t fvattn_num_blocks(const fvattn_geom_t* gi, int* nB, int* words) {
  Geo g;
  FV_CHECK(make_geo(gi, &g));
  if (nB) *nB = g.nB;
  if (words) *words = g.words;
  return FVATTN_OK;
}

fvattn_status_t fvattn_block_pool(const fvattn_geom_t* gi, const void* q, const void* k,
                                  float* q_pool, float* k_pool, fvattn_stream_t stream) {
  Geo g;
  FV_CHECK(make_geo(gi, &g));
  FV_CHECK(check_ptr(q));
  FV_CHECK(check_ptr(k));
  FV_CHECK(check_ptr(q_pool));
  FV_CHECK(check_ptr(k_pool));
  return cuda_status(fv::launch_pool(g, q, k, q_pool, k_pool, reinterpret_cast<cudaStream_t>(stream)));
}

fvattn_status_t fvattn_route(const fvattn_geom_t* gi, const float* q_pool, const float* k_pool,
                             float p, int k_floor, float scale, uint32_t* mask, int32_t* counts,
                             fvattn_stream_t stream) {
  Geo g;
  FV_CHECK(make_geo(gi, &g));
  FV_CHECK(check_ptr(q_pool));
  FV_CHECK(check_ptr(k_pool));
  FV_CHECK(check_ptr4(mask));
  FV_CHECK(check_ptr4(counts));
  if (!(p >= 0.f) || !isfinite(p)) return FVATTN_ERR_INVALID_ARG;
  if (k_floor < 0) return FVATTN_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return FVATTN_ERR_INVALID_ARG;
  return cuda_status(fv::launch_route(g, q_pool, k_pool, p, k_floor, scale, mask, counts,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

size_t fvattn_route_workspace_size(const fvattn_geom_t* gi) {
  Geo g;
  if (make_geo(gi, &g) != FVATTN_OK) return 0;
  return fv::route_ws_bytes(g);
}

fvattn_status_t fvattn_route_ws(const fvattn_geom_t* gi, const float* q_pool, const float* k_pool,
                                float p, int k_floor, float scale, uint32_t* mask, int32_t* counts,
                                void* workspace, size_t ws_bytes, fvattn_stream_t stream) {
  Geo g;
  FV_CHECK(make_geo(gi, &g));
  FV_CHECK(check_ptr(q_pool));
  FV_CHECK(check_ptr(k_pool));
  FV_CHECK(check_ptr4(mask));
  FV_CHECK(check_ptr4(counts));
  if (!(p >= 0.f) || !isfinite(p)) return FVATTN_ERR_INVALID_ARG;
  if (k_floor < 0) return FVATTN_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return FVATTN_ERR_INVALID_ARG;
  if (workspace == nullptr || ws_bytes < fv::route_ws_bytes(g)) return FVATTN_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 15u) return FVATTN_ERR_UNSUPPORTED;
  return cuda_status(fv::launch_route_ws(g, q_pool, k_pool, p, k_floor, scale, mask, counts, workspace,
                                         reinterpret_cast<cudaStream_t>(stream)));
}

fvattn_status_t fvattn_route_ex(const fvattn_geom_t* gi, const float* q_pool, const float* k_pool,
                                const fvattn_route_opts_t* opts, uint32_t* mask, int32_t* counts,
                                void* workspace, size_t ws_bytes, fvattn_stream_t stream) {
  Geo g;
  FV_CHECK(make_geo(gi, &g));
  FV_CHECK(check_ptr(q_pool));
  FV_CHECK(check_ptr(k_pool));
  FV_CHECK(check_ptr4(mask));
  FV_CHECK(check_ptr4(counts));
  if (opts == nullptr) return FVATTN_ERR_INVALID_ARG;
  const float p = opts->p, scale = opts->scale;
  if (!(p >= 0.f) || !isfinite(p)) return FVATTN_ERR_INVALID_ARG;
  if (opts->k_floor < 0) return FVATTN_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return FVATTN_ERR_INVALID_ARG;
  if (opts->token_mass != 0 && opts->token_mass != 1) return FVATTN_ERR_INVALID_ARG;
  if (opts->repair != 0 && opts->repair != 1) return FVATTN_ERR_INVALID_ARG;
  if (opts->kf_stride < 0) return FVATTN_ERR_INVALID_ARG;
  if (workspace == nullptr || ws_bytes < fv::route_ws_bytes(g)) return FVATTN_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 15u) return FVATTN_ERR_UNSUPPORTED;
  fv::RouteOpts o;
  o.token_mass = opts->token_mass;
  o.kf_stride = opts->kf_stride;
  o.kf_phase = opts->kf_stride > 0 ? opts->kf_phase % opts->kf_stride : 0;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  fvattn_status_t s = cuda_status(fv::launch_route_ws(g, q_pool, k_pool, p, opts->k_floor, scale, mask, counts,
                                                      workspace, st, o));
  if (s != FVATTN_OK || !opts->repair) return s;
  return cuda_status(fv::launch_mask_repair(g, mask, mask, counts, st));
}

fvattn_status_t fvattn_slack_augment(const fvattn_geom_t* gi, const void* route_workspace, size_t route_ws_bytes,
                                     float tau, int n_sm, uint32_t* mask, int32_t* counts, void* scratch,
                                     size_t scratch_bytes, fvattn_stream_t stream) {
  Geo g;
  FV_CHECK(make_geo(gi, &g));
  FV_CHECK(check_ptr4(mask));
  FV_CHECK(check_ptr4(counts));
  if (!(tau >= 0.f) || !isfinite(tau)) return FVATTN_ERR_INVALID_ARG;
  if (n_sm < 0) return FVATTN_ERR_INVALID_ARG;
  // tile costs (real query tokens x real key tokens) are held in 26 bits
  if (static_cast<long long>(g.bt) * g.bh * g.bw * g.N >= (1LL << 26)) return FVATTN_ERR_UNSUPPORTED;
  if (route_workspace == nullptr || route_ws_bytes < fv::route_ws_bytes(g)) return FVATTN_ERR_WORKSPACE;
  if (scratch == nullptr || scratch_bytes < fv::augment_scratch_bytes(g)) return FVATTN_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(route_workspace) | reinterpret_cast<uintptr_t>(scratch)) & 15u)
    return FVATTN_ERR_UNSUPPORTED;
  if (n_sm == 0) {
    n_sm = current_num_sms();
    if (n_sm <= 0) return cuda_status(cudaGetLastError() == cudaSuccess ? cudaErrorNoDevice : cudaGetLastError());
  }
  const float* logits = reinterpret_cast<const float*>(static_cast<const unsigned char*>(route_workspace) + 256);
  return cuda_status(fv::launch_augment(g, logits, tau, n_sm, mask, counts, scratch,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

fvattn_status_t fvattn_mask_repair(const fvattn_geom_t* gi, const uint32_t* mask_in, uint32_t* mask_out,
                                   int32_t* counts, fvattn_stream_t stream) {
  Geo g;
  FV_CHECK(make_geo(gi, &g));
  FV_CHECK(check_ptr4(mask_in));
  FV_CHECK(check_ptr4(mask_out));
  FV_CHECK(check_ptr4(counts));
  return cuda_status(fv::launch_mask_repair(g, mask_in, mask_out, counts, reinterpret_cast<cudaStream_t>(stream)));
}

size_t fvattn_pool_route_workspace_size(const fvattn_geom_t* gi) {
  Geo g;
  if (make_geo(gi, &g) != FVATTN_OK) return 0;
  return fv::pool_route_ws_bytes(g);
}

fvattn_status_t fvattn_pool_route(const fvattn_geom_t* gi, const void* q, const void* k, float p,
                                  int k_floor, float scale, float* q_pool, float* k_pool, uint32_t* mask,
                                  int32_t* counts, void* workspace, size_t ws_bytes,
                                  fvattn_stream_t stream) {
  Geo g;
  FV_CHECK(make_geo(gi, &g));
  FV_CHECK(check_ptr(q));
  FV_CHECK(check_ptr(k));
  FV_CHECK(check_ptr(q_pool));
  FV_CHECK(check_ptr(k_pool));
  FV_CHECK(check_ptr4(mask));
  FV_CHECK(check_ptr4(counts));
  if (!(p >= 0.f) || !isfinite(p)) return FVATTN_ERR_INVALID_ARG;
  if (k_floor < 0) return FVATTN_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return FVATTN_ERR_INVALID_ARG;
  if (workspace == nullptr || ws_bytes < fv::pool_route_ws_bytes(g)) return FVATTN_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 15u) return FVATTN_ERR_UNSUPPORTED;
  const int nsm = current_num_sms();
  if (nsm <= 0) return cuda_status(cudaGetLastError() == cudaSuccess ? cudaErrorNoDevice : cudaGetLastError());
  return cuda_status(fv::launch_pool_route(g, q, k, q_pool, k_pool, p, k_floor, scale, mask, counts, workspace,
                                           nsm, reinterpret_cast<cudaStream_t>(stream)));
}

size_t fvattn_attn_workspace_size(const fvattn_geom_t* gi) {
  Geo g;
  if (make_geo(gi, &g) != FVATTN_OK) return 0;
  return fv::attn_ws_bytes(g);
}

int fvattn_num_sms(void) { return current_num_sms(); }

fvattn_status_t fvattn_block_sparse_attn(const fvattn_geom_t* g, const void* q, const void* k,
                                         const void* v, const uint32_t* mask, float scale,
                                         void* out, float* lse, void* workspace, size_t ws_bytes,
                                         unsigned long long* sm_busy_ns, fvattn_stream_t stream) {
  if (mask == nullptr) return FVATTN_ERR_INVALID_ARG;
  return run_attn(g, q, k, v, mask, scale, out, lse, workspace, ws_bytes, sm_busy_ns, stream);
}

fvattn_status_t fvattn_dense_attn(const fvattn_geom_t* g, const void* q, const void* k,
                                  const void* v, float scale, void* out, float* lse,
                                  void* workspace, size_t ws_bytes,
                                  unsigned long long* sm_busy_ns, fvattn_stream_t stream) {
  return run_attn(g, q, k, v, nullptr, scale, out, lse, workspace, ws_bytes, sm_busy_ns, stream);
}

fvattn_status_t fvattn_block_sparse_attn_noalloc(const fvattn_geom_t* gi, const void* q, const void* k,
                                                 const void* v, const uint32_t* mask, float scale,
                                                 void* out, float* lse, unsigned long long* sm_busy_ns,
                                                 fvattn_stream_t stream) {
  Geo g;
  FV_CHECK(make_geo(gi, &g));
  if (mask == nullptr) return FVATTN_ERR_INVALID_ARG;
  if (fv::attn_ws_bytes(g) > kNoAllocScratchBytes) return FVATTN_ERR_WORKSPACE;
  void* scratch = nullptr;
  FV_CHECK(noalloc_scratch(&scratch));
  return run_attn(gi, q, k, v, mask, scale, out, lse, scratch, kNoAllocScratchBytes, sm_busy_ns, stream);
}

fvattn_status_t fvattn_testing_attn_stall(const fvattn_geom_t* g, const void* q, const void* k,
                                          const void* v, const uint32_t* mask, float scale, void* out,
                                          float* lse, void* workspace, size_t ws_bytes,
                                          unsigned long long stall_ns, fvattn_stream_t stream) {
  if (mask == nullptr) return FVATTN_ERR_INVALID_ARG;
  if (stall_ns == 0ull || stall_ns > 100000000ull) return FVATTN_ERR_INVALID_ARG;
  return run_attn(g, q, k, v, mask, scale, out, lse, workspace, ws_bytes, nullptr, stream, stall_ns);
}

fvattn_status_t fvattn_noalloc_device_status(fvattn_stream_t stream) {
  void* scratch = nullptr;
  FV_CHECK(noalloc_scratch(&scratch));
  return fvattn_device_status(scratch, stream);
}

fvattn_status_t fvattn_device_status(const void* workspace, fvattn_stream_t stream) {
  if (workspace == nullptr) return FVATTN_ERR_INVALID_ARG;
  uint32_t hdr[2] = {0, 0};
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  fvattn_status_t s = cuda_status(cudaMemcpyAsync(hdr, workspace, sizeof(hdr), cudaMemcpyDeviceToHost, st));
  if (s != FVATTN_OK) return s;
  s = cuda_status(cudaStreamSynchronize(st));
  if (s != FVATTN_OK) return s;
  if (hdr[1] & fv::kErrTimeout) return FVATTN_ERR_DEVICE_TIMEOUT;
  if (hdr[1] & fv::kErrLayout) return FVATTN_ERR_DEVICE;
  return FVATTN_OK;
}

const char* fvattn_last_cuda_error(void) {
  return g_last_cuda_error == cudaSuccess ? "no error" : cudaGetErrorString(g_last_cuda_error);
}

const char* fvattn_status_string(fvattn_status_t s) {
  switch (s) {
    case FVATTN_OK: return "ok";
    case FVATTN_ERR_INVALID_ARG: return "invalid argument";
    case FVATTN_ERR_UNSUPPORTED: return "unsupported shape, size or alignment";
    case FVATTN_ERR_WORKSPACE: return "workspace missing or too small";
    case FVATTN_ERR_CUDA: return "CUDA call failed";
    case FVATTN_ERR_DEVICE_TIMEOUT: return "a kernel gave up a bounded wait";
    case FVATTN_ERR_DEVICE: return "a kernel found its shared-memory layout misaligned and did no work";
  }
  return "unknown status";
}

}  // extern "C"
