/*
 * fvattn — training-free adaptive block-sparse attention for video diffusion
 * transformers, on NVIDIA B200 (sm_100a).
 *
 * The method: "FVAttn: Adaptive Sparse Attention with Runtime Load Balancing for
 * Video Generation" (explainer of arXiv 2607.16190), section 核心方法 §1
 * 稀疏路由前端 (sparse-routing frontend): spatio-temporal tokens are grouped into
 * 3D blocks (video-aware block organisation); each head routes per query block
 * with Top-p over block similarity mass plus a Top-k safety floor; attention then
 * runs only over the selected key blocks (the kernel that replaces FlashAttention,
 * 核心方法 §2, attn_kernel.run()).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Tensors are row-major and contiguous.  Q, K, V and out are bf16
 *   [B][H][N][d], N = T*Hs*Ws, token n of a (b,h) slice at latent position
 *   (t, y, x) with n = (t*Hs + y)*Ws + x  ("T-major").
 * - 3D block (tb, yb, xb) covers t in [tb*bt, tb*bt+bt), y in [yb*bh, ...),
 *   x in [xb*bw, ...), clipped to the latent: edge blocks are partial.  Blocks are
 *   numbered T-major: j = (tb*nBy + yb)*nBx + xb, nBt = ceil(T/bt), nBy =
 *   ceil(Hs/bh), nBx = ceil(Ws/bw), nB = nBt*nBy*nBx.
 * - Every pointer argument is a DEVICE pointer owned by the caller, 16-byte aligned,
 *   except mask, counts and lse, which need 4-byte alignment only (so that a caller
 *   can pass views of consecutive (b, h) slices of them).  The library allocates no device memory and keeps no state between
 *   calls apart from cached driver entry points.
 * - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *   stream) and never synchronise.  Argument errors are detected on the host
 *   before anything is launched.  Launch failures return FVATTN_ERR_CUDA;
 *   faults during execution surface at the caller's next synchronisation.
 * - No C++ exception crosses this interface.
 * - Every extent of the geometry (B, H, T, Hs, Ws, bt, bh, bw) must be >= 1: an
 *   empty batch, head set or latent is FVATTN_ERR_INVALID_ARG (a caller with nothing
 *   to compute makes no call).
 * - Supported: d in {64, 128}; 1 <= bt*bh*bw <= 128; nB <= 2048; B*H*nB < 2^24;
 *   N < 2^31; B*H*N*d < 2^40; Ws, Hs <= 65535 and T <= 32767 (tensor-map extents).
 *   Other valid geometries return FVATTN_ERR_UNSUPPORTED.
 */
#ifndef FVATTN_H_
#define FVATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define FVATTN_API __attribute__((visibility("default")))
#else
#define FVATTN_API
#endif

struct CUstream_st;                          /* cudaStream_t is struct CUstream_st* */
typedef struct CUstream_st* fvattn_stream_t;

typedef enum {
  FVATTN_OK = 0,
  FVATTN_ERR_INVALID_ARG = 1,     /* null pointer, bad size, p/k/scale out of domain */
  FVATTN_ERR_UNSUPPORTED = 2,     /* valid but unsupported: d, block size, alignment */
  FVATTN_ERR_WORKSPACE = 3,       /* workspace missing or smaller than required */
  FVATTN_ERR_CUDA = 4,            /* a CUDA runtime/driver call failed */
  FVATTN_ERR_DEVICE_TIMEOUT = 5,  /* a kernel gave up a bounded wait (see fvattn_device_status) */
  FVATTN_ERR_DEVICE = 6           /* a kernel detected an internal layout error and did no work */
} fvattn_status_t;

typedef struct {
  int B, H;          /* batch, heads                                  */
  int T, Hs, Ws;     /* latent frames, height, width (tokens)          */
  int d;             /* head dimension: 64 or 128                      */
  int bt, bh, bw;    /* 3D block extent in frames, rows, columns       */
} fvattn_geom_t;

/* Number of 3D blocks nB and of 32-bit mask words per mask row, ceil(nB/32).
 * Returns FVATTN_ERR_INVALID_ARG for a null or malformed geometry. */
FVATTN_API fvattn_status_t fvattn_num_blocks(const fvattn_geom_t* g, int* nB, int* words);

/* 3D block mean-pooling (video-aware block organisation, FVAttn explainer
 * 核心方法 §1).  For every (b, h, block j):
 *   q_pool[b][h][j][:] = mean of q[b][h][n][:] over the real tokens n of block j,
 * and likewise k_pool from k.  Edge blocks average over their real tokens only.
 *   q, k    : bf16 [B][H][N][d]              (read)
 *   q_pool, k_pool : fp32 [B][H][nB][d]       (written)
 * Accumulation in fp32. */
FVATTN_API fvattn_status_t fvattn_block_pool(const fvattn_geom_t* g, const void* q, const void* k,
                                  float* q_pool, float* k_pool, fvattn_stream_t stream);

/* Per-head Top-p block routing with a Top-k floor (FVAttn explainer 核心方法 §1,
 * "Top-p 路由" and "Top-k 安全底").  For every (b, h, query block i):
 *   l_j = (q_pool[i] . k_pool[j]) * scale over all key blocks j,
 *   s   = softmax_j(l)                              (the routing score),
 *   order the key blocks by s descending, ties to the lower index,
 *   m_p = the shortest prefix with cumulative mass >= p (nB when p >= 1 or when
 *         the total mass falls short of p),
 *   m   = max(m_p, min(k_floor, nB)),
 *   kept = the first m blocks of that order, plus block i itself.
 * Outputs:
 *   mask   : uint32 [B][H][nB][words]; bit (j % 32) of word (j / 32) is set when
 *            key block j is kept; bits at j >= nB are zero.
 *   counts : int32  [B][H][nB]; number of kept blocks (popcount of the row).
 * Arguments: 0 <= p (p >= 1 keeps every block), k_floor >= 0, scale > 0 and
 * finite (normally 1/sqrt(d), the same scale the attention uses).
 * Scores and masses are fp32; selection uses the logits' order. */
FVATTN_API fvattn_status_t fvattn_route(const fvattn_geom_t* g, const float* q_pool, const float* k_pool,
                             float p, int k_floor, float scale,
                             uint32_t* mask, int32_t* counts, fvattn_stream_t stream);

/* Bytes of device workspace fvattn_route_ws, fvattn_route_ex and fvattn_pool_route need:
 * a 256-byte header (a status word), one fp32 logit per (query block, key block) pair of
 * every (b, h) with rows padded to words * 32 entries, and the pooled rows split into
 * tf32 high and low parts (256 + B*H*nB*words*32*4 + 4*B*H*nB*d*4 bytes; 13.7 MB at
 * 21x30x52 with 1x8x16 blocks, d = 128 and 12 heads, 229 MB at 121x30x52).  0 for an
 * invalid geometry. */
FVATTN_API size_t fvattn_route_workspace_size(const fvattn_geom_t* g);

/* fvattn_route, computed through a caller-owned workspace: the logits of all block pairs
 * first, written to `workspace`, then the selection, one query block per warp.  Rows of
 * up to 16 mask words (nB <= 512) take fvattn_route's arithmetic in two kernels (a tiled
 * fp32 product, then the bitwise threshold search), so the two calls give the same mask.
 * Longer rows take the tensor cores for the logits (tf32 with each fp32 operand split into
 * a high and a low tf32 part, three products per pair: fp32-grade logits) and select by a
 * mass histogram with the masses summed exactly in fixed point (2^-32 of the row's
 * largest exp); there the two calls may disagree on blocks whose scores nearly tie at the
 * cut.  Same definition, inputs, outputs, argument domains and error behaviour as
 * fvattn_route (FVAttn explainer 核心方法 §1: Top-p with a Top-k floor and the own block
 * over softmax(pooled q . pooled k * scale)).
 *   workspace, ws_bytes : >= fvattn_route_workspace_size(g) bytes of device memory,
 *                         16-byte aligned, owned by the caller; its contents on entry
 *                         do not matter and on return hold the logits (scaled).
 * Returns FVATTN_ERR_WORKSPACE when the workspace is missing or too small.  The logits
 * kernel's waits are bounded; one that gives up is reported by
 * fvattn_device_status(workspace) as FVATTN_ERR_DEVICE_TIMEOUT. */
FVATTN_API fvattn_status_t fvattn_route_ws(const fvattn_geom_t* g, const float* q_pool, const float* k_pool,
                                           float p, int k_floor, float scale, uint32_t* mask,
                                           int32_t* counts, void* workspace, size_t ws_bytes,
                                           fvattn_stream_t stream);

/* Options of fvattn_route_ex: the routing rule of fvattn_route plus the pages' further
 * frontend steps, each off when zero. */
typedef struct {
  float p;          /* Top-p mass, as fvattn_route                                     */
  int k_floor;      /* Top-k floor in blocks, as fvattn_route                          */
  float scale;      /* logit scale, as fvattn_route                                    */
  int token_mass;   /* 1: Top-p over tokens.  The FVAttn explainer (核心方法 §1, Top-p 路由)
                     * keeps the minimal TOKEN set whose mass reaches p, and its 3D blocks
                     * let that decision be taken per block: every real token of key block j
                     * takes the block's pooled logit l_j, so blocks keep the order of l_j
                     * and block j carries the mass n_j exp(l_j) / sum_k n_k exp(l_k), n_j its
                     * real token count.  0: blocks count equally (fvattn_route's rule).  */
  int kf_stride;    /* > 0: keyframe blocks (LVSA Long-Video Showcase README, Results and
                     * Configuration: rotating keyframes).  Latent frame t is a keyframe when
                     * (t - kf_phase) mod kf_stride == 0; every key block holding a keyframe
                     * frame is kept by every query block, added after the prefix rule like
                     * the own block (it counts toward neither p nor the floor).  A caller
                     * rotates the set by changing kf_phase between calls.              */
  int kf_phase;     /* keyframe phase, any integer                                     */
  int repair;       /* 1: then runtime mask repair in place (fvattn_mask_repair)          */
} fvattn_route_opts_t;

/* fvattn_route_ws with the options above: the same logits and selection, with the
 * Top-p masses over tokens when opts->token_mass, keyframe blocks added to every row
 * when opts->kf_stride > 0, and fvattn_mask_repair applied to the result when
 * opts->repair.  Same buffers, workspace (fvattn_route_workspace_size) and error
 * behaviour as fvattn_route_ws; kf_stride < 0 or token_mass / repair outside {0, 1}
 * is FVATTN_ERR_INVALID_ARG.  With every option zero it equals fvattn_route_ws. */
FVATTN_API fvattn_status_t fvattn_route_ex(const fvattn_geom_t* g, const float* q_pool, const float* k_pool,
                                           const fvattn_route_opts_t* opts, uint32_t* mask, int32_t* counts,
                                           void* workspace, size_t ws_bytes, fvattn_stream_t stream);

/* Runtime mask repair (FVAttn explainer, 核心方法 §1, 运行时修补: holes between routing
 * and attention are patched locally, on the materialized mask, without new scores).
 * Reading: in every row, a dropped key block whose two neighbours along the time, height
 * or width axis of the 3D block grid both exist and are both kept is a one-block hole,
 * and is set.  One pass: every decision reads mask_in as given, so holes that only open
 * up after a fill stay.  Bits at j >= nB are cleared.
 *   mask_in  : uint32 [B][H][nB][words]          (read)
 *   mask_out : uint32 [B][H][nB][words]          (written; may equal mask_in)
 *   counts   : int32  [B][H][nB]                 (written: popcount of each repaired row) */
FVATTN_API fvattn_status_t fvattn_mask_repair(const fvattn_geom_t* g, const uint32_t* mask_in, uint32_t* mask_out,
                                              int32_t* counts, fvattn_stream_t stream);

/* Slack-aware sparse augmentation (FVAttn explainer, 核心方法 §3 Slack-Aware Sparse
 * Augmentation: the slack that idle workers leave before the critical path ends is filled
 * with high-value blocks, filtered by a score threshold; 工程落地 item 5).  Reading for one
 * GPU, whose workers are the SMs of the persistent attention kernel: the cost of a
 * (b, h, query block) tile is its real query tokens times the real key tokens of its kept
 * blocks; tiles run longest first (cost descending, ties by tile index), and the last n_sm
 * tiles of that order form the final wave, whose largest tile sets the end, cost c*.
 * Every tile of the wave takes its dropped key blocks of routing score >= tau, in score
 * order (descending, ties by lower index), each while its cost stays <= c*, and stops at
 * the first that does not fit.  Call it after a route that left its logits in
 * route_workspace (fvattn_route_ws, fvattn_route_ex, fvattn_pool_route) and before the
 * attention.
 *   route_workspace, route_ws_bytes : that route call's workspace (read)
 *   tau    : score threshold, >= 0 (routing score = softmax over key blocks of the logits)
 *   n_sm   : workers; 0 = the current device's SM count
 *   mask, counts : updated in place (only the wave's rows change)
 *   scratch, scratch_bytes : >= fvattn_attn_workspace_size(g) bytes of device memory, the
 *            attention call's workspace may serve (its contents are rewritten anyway)
 * Geometries whose tile cost needs 26 bits or more (bt*bh*bw * N >= 2^26) return
 * FVATTN_ERR_UNSUPPORTED. */
FVATTN_API fvattn_status_t fvattn_slack_augment(const fvattn_geom_t* g, const void* route_workspace,
                                                size_t route_ws_bytes, float tau, int n_sm, uint32_t* mask,
                                                int32_t* counts, void* scratch, size_t scratch_bytes,
                                                fvattn_stream_t stream);

/* Bytes of device workspace fvattn_pool_route needs: fvattn_route_workspace_size(g).  0
 * for an invalid geometry. */
FVATTN_API size_t fvattn_pool_route_workspace_size(const fvattn_geom_t* g);

/* fvattn_block_pool followed by fvattn_route_ws in one call (FVAttn explainer 核心方法
 * §1: pooled 3D blocks, then Top-p with a Top-k floor and the own block): the same
 * kernels on the caller's stream, so q_pool, k_pool, mask and counts equal what the two
 * calls write.
 *   q, k              : bf16 [B][H][N][d]           (read)
 *   q_pool, k_pool    : fp32 [B][H][nB][d]          (written)
 *   mask, counts      : as fvattn_route             (written)
 *   workspace, ws_bytes : >= fvattn_pool_route_workspace_size(g) bytes, 16-byte aligned,
 *                       owned by the caller, contents on entry do not matter; not to be
 *                       shared by calls that run concurrently.
 * A wait that gives up is reported by fvattn_device_status(workspace). */
FVATTN_API fvattn_status_t fvattn_pool_route(const fvattn_geom_t* g, const void* q, const void* k, float p,
                                             int k_floor, float scale, float* q_pool, float* k_pool,
                                             uint32_t* mask, int32_t* counts, void* workspace,
                                             size_t ws_bytes, fvattn_stream_t stream);

/* Bytes of device workspace fvattn_block_sparse_attn / fvattn_dense_attn need
 * for geometry g (a tile queue and a status word).  0 for a malformed geometry. */
FVATTN_API size_t fvattn_attn_workspace_size(const fvattn_geom_t* g);

/* Number of entries fvattn_block_sparse_attn writes to sm_busy_ns: the number of
 * streaming multiprocessors of the current device (0 on error). */
FVATTN_API int fvattn_num_sms(void);

/* Block-sparse attention over the kept key blocks (the attention kernel of the
 * FVAttn explainer 核心方法 §2; online softmax over the kept blocks in ascending
 * block order).  For every real query token n of query block i of (b, h):
 *   lse[n] = ln sum_{m in kept(i)} exp((q_n . k_m) * scale),
 *   out[n] = sum_{m in kept(i)} exp((q_n . k_m) * scale - lse[n]) v_m,
 * where m runs over the real tokens of the key blocks whose mask bit is set.
 *   q, k, v : bf16 [B][H][N][d]      (read)
 *   mask    : uint32 [B][H][nB][words], as written by fvattn_route (bit j of a row:
 *             key block j kept).  Bits at j >= nB are ignored.  A row with no bit set
 *             (fvattn_route always sets bit i) gives out = 0 and lse = -inf for its
 *             tokens.  The per-row counts fvattn_route also writes are not an
 *             argument: the kernels derive every row's kept blocks, and their number,
 *             from the mask alone, so no count can disagree with its row.
 *   out     : bf16 [B][H][N][d]      (written, every token)
 *   lse     : fp32 [B][H][N]         (written, every token)
 *   workspace, ws_bytes : >= fvattn_attn_workspace_size(g) bytes, 16-byte aligned,
 *             contents need not be initialised; not to be shared by calls that
 *             run concurrently.
 *   sm_busy_ns : optional (NULL to skip) uint64 [fvattn_num_sms()]; receives, per SM,
 *             the nanoseconds from the start of its CTA to the end of its last tile.
 * Products are bf16 x bf16 with fp32 accumulation; the softmax is fp32 with P
 * rounded to bf16 before the P.V product.  Work is scheduled by a persistent
 * kernel over (b, h, query block) tiles taken from a queue ordered by decreasing
 * cost (longest processing time first). */
FVATTN_API fvattn_status_t fvattn_block_sparse_attn(const fvattn_geom_t* g, const void* q, const void* k,
                                         const void* v, const uint32_t* mask, float scale,
                                         void* out, float* lse,
                                         void* workspace, size_t ws_bytes,
                                         unsigned long long* sm_busy_ns, fvattn_stream_t stream);

/* fvattn_block_sparse_attn for callers that cannot allocate device memory: the same
 * computation and arguments, minus the workspace, which comes from a scratch area the
 * library itself reserves as a static device array of 1 MiB (held on every device
 * that loads the library until the process exits).  It serves code that may not call
 * cudaMalloc or reach a device allocator at the point of the call: runtimes that plan
 * all device memory up front and forbid allocation on the serving path, plugins whose
 * host framework owns every device buffer, callers without a handle to an allocator.
 * The paper has no counterpart; this is an integration convenience of this library.
 * - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 * - Geometries whose tile queue needs more than the scratch area (B*H*nB above
 *   131040 tiles) are rejected with FVATTN_ERR_WORKSPACE.
 * - The first call on a device resolves the scratch area's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call before any
 *   stream capture.  The address is cached per device together with the identifier of
 *   the driver context it was resolved in; when the device's current context changes
 *   (after cudaDeviceReset, or under a context the caller made current), the next call
 *   resolves it again, so that call too belongs outside a stream capture.
 * - Every call shares the one scratch area, which keeps the last call's contents (the
 *   kernels reset what must start at zero).  Calls that overlap on the GPU (different
 *   streams, or different host threads on one device) race on it: serialise them.
 * - A device-side timeout of this entry point is reported by
 *   fvattn_noalloc_device_status (there is no workspace to pass to fvattn_device_status). */
FVATTN_API fvattn_status_t fvattn_block_sparse_attn_noalloc(const fvattn_geom_t* g, const void* q,
                                                            const void* k, const void* v,
                                                            const uint32_t* mask, float scale,
                                                            void* out, float* lse,
                                                            unsigned long long* sm_busy_ns,
                                                            fvattn_stream_t stream);

/* fvattn_device_status for fvattn_block_sparse_attn_noalloc: synchronises `stream` and
 * reports how the last call of that entry point on the current device ran, from the
 * library's static scratch area.  Same return values as fvattn_device_status. */
FVATTN_API fvattn_status_t fvattn_noalloc_device_status(fvattn_stream_t stream);

/* Dense attention: fvattn_block_sparse_attn with every key block kept (the p = 1
 * case), without reading a mask.  Same arguments otherwise. */
FVATTN_API fvattn_status_t fvattn_dense_attn(const fvattn_geom_t* g, const void* q, const void* k,
                                  const void* v, float scale, void* out, float* lse,
                                  void* workspace, size_t ws_bytes,
                                  unsigned long long* sm_busy_ns, fvattn_stream_t stream);

/* Synchronises `stream` and reports whether the last attention or fvattn_pool_route
 * call that used `workspace` ran cleanly: FVATTN_OK, FVATTN_ERR_DEVICE_TIMEOUT (a kernel gave up a
 * bounded wait), FVATTN_ERR_DEVICE (a kernel found its shared memory misaligned and
 * did no work), or FVATTN_ERR_CUDA if the synchronisation failed. */
FVATTN_API fvattn_status_t fvattn_device_status(const void* workspace, fvattn_stream_t stream);

/* Text of the CUDA error behind the calling thread's most recent FVATTN_ERR_CUDA
 * ("no error" if there was none).  Static storage. */
FVATTN_API const char* fvattn_last_cuda_error(void);

/* Static, human-readable name of a status code. */
FVATTN_API const char* fvattn_status_string(fvattn_status_t s);

#ifdef __cplusplus
}
#endif

#endif /* FVATTN_H_ */
