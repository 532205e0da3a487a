// 3D block mean-pooling and per-head Top-p / Top-k block routing.
//
// FVAttn explainer (arXiv 2607.16190), 核心方法 §1 稀疏路由前端: tokens are grouped
// into video-aware 3D blocks and each head decides per block which key blocks a
// query block keeps: the minimal set whose cumulative similarity mass reaches p
// (Top-p), at least k of them (Top-k safety floor).  The routing score is the
// softmax over key blocks of the pooled q . pooled k / sqrt(d); the query's own
// block is always kept.
#include <cuda_bf16.h>
#include <float.h>

#include "fv_common.cuh"
#include "fv_launch.h"
#include "fv_plan.h"

namespace fv {

// ----------------------------------------------------------------------------
// Pooling: one CTA per (block, b*h, tensor), tensor 0 = Q, 1 = K.  A block is rt * ry
// rows of rx tokens, and the tokens of a row are contiguous in memory; warp w takes
// rows w, w + 8, ...  Lane l owns the 16-byte chunk l % (d/8) of tokens l / (d/8),
// l / (d/8) + 32 / (d/8), ... of the row, all of a row's loads are issued before any is
// used, and no address needs a division.  Partial sums are folded with warp shuffles,
// then across warps through shared memory.
// ----------------------------------------------------------------------------
constexpr int kPoolThreads = 256;

// One pooling item: block j of slice bhi of one tensor (src -> dst).  `red` is the
// CTA's [8][D] reduction buffer; the caller separates items with a block barrier.
template <int D>
__device__ __forceinline__ void pool_item(const Geo& g, const uint4* __restrict__ src,
                                          float* __restrict__ dst, int j, int bhi,
                                          float (*red)[D]) {
  constexpr int CH = D / 8;                // 16-byte chunks per token
  constexpr int TPI = 32 / CH;             // tokens a warp covers per load instruction
  constexpr int NW = kPoolThreads / 32;
  constexpr int BATCH = 8;                 // loads in flight per lane

  const BlockInfo bi = block_info(g, j);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int ch = lane % CH, tsub = lane / CH;
  const size_t base = static_cast<size_t>(bhi) * g.N;
  const int t0 = bi.tb * g.bt, y0 = bi.yb * g.bh, x0 = bi.xb * g.bw;

  float a[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) a[e] = 0.f;
  const int nrows = bi.rt * bi.ry;
  for (int row = warp; row < nrows; row += NW) {
    const int tt = row / bi.ry, yy = row - tt * bi.ry;
    const uint4* p = src + (base + (static_cast<size_t>(t0 + tt) * g.Hs + (y0 + yy)) * g.Ws + x0) * CH + ch;
    for (int x = tsub; x < bi.rx; x += BATCH * TPI) {
      uint4 v[BATCH];
#pragma unroll
      for (int u = 0; u < BATCH; ++u) {
        const int xx = x + u * TPI;
        v[u] = xx < bi.rx ? __ldg(p + static_cast<size_t>(xx) * CH) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < BATCH; ++u) {
        const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          a[2 * e] += __uint_as_float(w[e] << 16);
          a[2 * e + 1] += __uint_as_float(w[e] & 0xFFFF0000u);
        }
      }
    }
  }
  // lanes l, l + CH, ... of a warp hold the same chunk
#pragma unroll
  for (int off = CH; off < 32; off <<= 1) {
#pragma unroll
    for (int e = 0; e < 8; ++e) a[e] += __shfl_xor_sync(0xffffffffu, a[e], off);
  }
  if (lane < CH) {
#pragma unroll
    for (int e = 0; e < 8; ++e) red[warp][lane * 8 + e] = a[e];
  }
  __syncthreads();
  const float inv = 1.f / static_cast<float>(bi.nvalid);
  for (int t = threadIdx.x; t < D; t += kPoolThreads) {
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) sum += red[w][t];
    dst[(static_cast<size_t>(bhi) * g.nB + j) * D + t] = sum * inv;
  }
}

template <int D>
__global__ void __launch_bounds__(kPoolThreads, 4) pool_kernel(Geo g, const uint4* __restrict__ q,
                                                               const uint4* __restrict__ k,
                                                               float* __restrict__ qp,
                                                               float* __restrict__ kp) {
  __shared__ float red[kPoolThreads / 32][D];
  pool_item<D>(g, blockIdx.z ? k : q, blockIdx.z ? kp : qp, blockIdx.x, blockIdx.y, red);
}

cudaError_t launch_pool(const Geo& g, const void* q, const void* k, float* qp, float* kp,
                        cudaStream_t st) {
  dim3 grid(g.nB, g.B * g.H, 2);
  if (g.d == 128)
    pool_kernel<128><<<grid, kPoolThreads, 0, st>>>(g, static_cast<const uint4*>(q),
                                                     static_cast<const uint4*>(k), qp, kp);
  else
    pool_kernel<64><<<grid, kPoolThreads, 0, st>>>(g, static_cast<const uint4*>(q),
                                                    static_cast<const uint4*>(k), qp, kp);
  return cudaGetLastError();
}

// ----------------------------------------------------------------------------
// Routing: one CTA per (b*h, 8 query blocks); warp w owns query block w of the CTA.
// Logits: pooled key rows are staged in shared memory 128 blocks x 32 channels at a
// time (coalesced cp.async, two stages in flight) and each lane takes one key block
// against 4 of the CTA's 8 pooled query rows.  Then, per query block, with the row's
// logits and
// scores held in registers: softmax over all key blocks, and a bitwise search for the
// Top-p cut over an order-preserving integer key of the logits, so no sort is needed:
//   u* = the largest key with mass(key >= u*) >= p  -> the key of the m_p-th block;
// equal keys are taken in ascending block index.  The Top-k floor lengthens the
// prefix with a second search on counts.  Reductions are warp shuffles in a fixed
// order, so the result is deterministic.
// ----------------------------------------------------------------------------
constexpr int kRouteRows = 8;
constexpr int kRouteThreads = 256;

__device__ __forceinline__ uint32_t order_key(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}
__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}

// When exactly one valid key of the row has the high 16 bits of u, sets u to that key
// and returns true (uniform over the warp).
template <int MAXW>
__device__ __forceinline__ bool unique_prefix(const uint32_t* key, uint32_t& u) {
  int n = 0;
  uint32_t kmax = 0;
#pragma unroll
  for (int c = 0; c < MAXW; ++c) {
    const bool in = key[c] != 0u && (key[c] >> 16) == (u >> 16);
    n += in ? 1 : 0;
    kmax = in ? max(kmax, key[c]) : kmax;
  }
  if (warp_sum_i(n) != 1) return false;
  u = __reduce_max_sync(0xffffffffu, kmax);
  return true;
}

// Selection for one query block; the row's logits are in sL[i], i = c*32 + lane.
template <int MAXW>
__device__ __forceinline__ void select_row(const float* sL, int nB, int words, int qb, float p,
                                           int k_floor, uint32_t* mrow, int32_t* cnt_out, int lane) {
  uint32_t key[MAXW];
  float sc[MAXW];
  float mx = -INFINITY;
#pragma unroll
  for (int c = 0; c < MAXW; ++c) {
    const int i = c * 32 + lane;
    const bool v = c < words && i < nB;
    const float lg = v ? sL[c * 32 + lane] : -INFINITY;
    key[c] = v ? order_key(lg) : 0u;
    sc[c] = lg;
    mx = fmaxf(mx, lg);
  }
  mx = warp_max(mx);
  float z = 0.f;
#pragma unroll
  for (int c = 0; c < MAXW; ++c) {
    const float e = key[c] ? expf(sc[c] - mx) : 0.f;
    sc[c] = e;
    z += e;
  }
  z = warp_sum(z);
  const float inv_z = 1.f / z;
  float total = 0.f;
#pragma unroll
  for (int c = 0; c < MAXW; ++c) {
    sc[c] *= inv_z;
    total += sc[c];
  }
  total = warp_sum(total);

  const int floor_k = min(max(k_floor, 0), nB);
  int m_p;
  uint32_t u = 0;
  int ties_needed = 0;
  if (p >= 1.f || total < p) {
    m_p = nB;
  } else {
    // The high 16 bits first.  The answer is the key of one logit (the m_p-th in the
    // order), so when a single logit carries the 16-bit prefix found, its key is the
    // answer and the low 16 steps are skipped; otherwise they run as usual.
    auto mass_step = [&](int bit) {
      const uint32_t cand = u | (1u << bit);
      float m0 = 0.f, m1 = 0.f;
#pragma unroll
      for (int c = 0; c < MAXW; c += 2) {
        m0 += key[c] >= cand ? sc[c] : 0.f;
        if (c + 1 < MAXW) m1 += key[c + 1] >= cand ? sc[c + 1] : 0.f;
      }
      if (warp_sum(m0 + m1) >= p) u = cand;
    };
    for (int bit = 31; bit >= 16; --bit) mass_step(bit);
    if (!unique_prefix<MAXW>(key, u)) {
      for (int bit = 15; bit >= 0; --bit) mass_step(bit);
    }
    int gt = 0, eq = 0;
    float gm = 0.f, es = 0.f;
#pragma unroll
    for (int c = 0; c < MAXW; ++c) {
      if (key[c] > u) { ++gt; gm += sc[c]; }
      if (key[c] == u && key[c] != 0u) { ++eq; es = sc[c]; }
    }
    gt = warp_sum_i(gt);
    eq = warp_sum_i(eq);
    gm = warp_sum(gm);
    es = warp_max(es);
    float acc = gm;
    int r = 0;
    while (acc < p && r < eq) {
      acc += es;
      ++r;
    }
    m_p = gt + r;
    ties_needed = r;
  }
  const int M = max(max(m_p, floor_k), 1);
  if (M >= nB) {
    u = 0;
    ties_needed = nB;     // every block (keys of real blocks are nonzero)
  } else if (M > m_p) {
    uint32_t v = 0;
    auto count_step = [&](int bit) {
      const uint32_t cand = v | (1u << bit);
      int n = 0;
#pragma unroll
      for (int c = 0; c < MAXW; ++c) n += key[c] >= cand ? 1 : 0;
      if (warp_sum_i(n) >= M) v = cand;
    };
    for (int bit = 31; bit >= 16; --bit) count_step(bit);
    if (!unique_prefix<MAXW>(key, v)) {
      for (int bit = 15; bit >= 0; --bit) count_step(bit);
    }
    int gt = 0;
#pragma unroll
    for (int c = 0; c < MAXW; ++c) gt += key[c] > v ? 1 : 0;
    u = v;
    ties_needed = M - warp_sum_i(gt);
  }

  int tie_base = 0, cnt = 0;
#pragma unroll
  for (int c = 0; c < MAXW; ++c) {
    if (c < words) {
      const int i = c * 32 + lane;
      const bool valid = key[c] != 0u;
      const bool tie = valid && key[c] == u;
      const uint32_t tb = __ballot_sync(0xffffffffu, tie);
      const int rank = tie_base + __popc(tb & ((1u << lane) - 1u));
      tie_base += __popc(tb);
      const bool kept = valid && (key[c] > u || (tie && rank < ties_needed) || i == qb);
      const uint32_t word = __ballot_sync(0xffffffffu, kept);
      cnt += __popc(word);
      if (lane == 0) mrow[c] = word;
    }
  }
  if (lane == 0) *cnt_out = cnt;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

constexpr int kRouteKT = 128;          // key blocks per staged tile
constexpr int kRouteDC = 32;           // channels per staged tile
constexpr int kRouteKSP = kRouteDC + 4;  // padded tile row (floats)

template <int D, int MAXW>
__global__ void __launch_bounds__(kRouteThreads) route_kernel(Geo g, const float* __restrict__ qp,
                                                              const float* __restrict__ kp, float p,
                                                              int k_floor, float scale,
                                                              uint32_t* __restrict__ mask,
                                                              int32_t* __restrict__ counts) {
  extern __shared__ __align__(16) unsigned char route_smem[];
  constexpr int NDC = D / kRouteDC;    // channel tiles per key row
  const int words = g.words;
  const int nBpad = words * 32;
  float* sQ = reinterpret_cast<float*>(route_smem);              // [8][D]
  float* sL = sQ + kRouteRows * D;                               // [8][nBpad]
  float* sK = sL + kRouteRows * nBpad;                           // [2][128][36]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bhi = blockIdx.y;
  const int nB = g.nB;
  const int row0 = blockIdx.x * kRouteRows;
  const float* kph = kp + static_cast<size_t>(bhi) * nB * D;

  // stage st = (round, channel tile): key blocks [128 round, +128) x channels
  // [32 tile, +32), coalesced 16-byte copies, rows past nB zero-filled
  const int nstage = ((nB + kRouteKT - 1) / kRouteKT) * NDC;
  auto stage = [&](int st) {
    const int round = st / NDC, ct = st - round * NDC;
    float* dst = sK + (st & 1) * kRouteKT * kRouteKSP;
    for (int e = threadIdx.x; e < kRouteKT * kRouteDC / 4; e += kRouteThreads) {
      const int key = e / (kRouteDC / 4), q4 = e - key * (kRouteDC / 4);
      const int j = round * kRouteKT + key;
      cp_async16(smem_u32(dst + key * kRouteKSP + 4 * q4),
                 kph + static_cast<size_t>(j < nB ? j : 0) * D + ct * kRouteDC + 4 * q4, j < nB ? 16u : 0u);
    }
    cp_async_commit();
  };
  stage(0);
  for (int e = threadIdx.x; e < kRouteRows * D / 4; e += kRouteThreads) {
    const int r = e / (D / 4), d4 = e - r * (D / 4);
    const int row = row0 + r;
    reinterpret_cast<float4*>(sQ)[e] =
        row < nB ? reinterpret_cast<const float4*>(qp + (static_cast<size_t>(bhi) * nB + row) * D)[d4]
                 : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  // Logits: warp w takes key blocks 32 (w % 4) + lane of each round against query rows
  // 4 (w / 4) .. + 3.  Per (row, key) the sum over d runs in two partial sums (even and
  // odd components of each float4), in ascending d, added at the end.
  const int kgrp = warp & 3, rgrp = warp >> 2;
  uint64_t acc[4];   // (a0, a1) per query row as an f32x2 pair
  for (int st = 0; st < nstage; ++st) {
    if (st + 1 < nstage) {
      stage(st + 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const int round = st / NDC, ct = st - round * NDC;
    if (ct == 0) {
#pragma unroll
      for (int r = 0; r < 4; ++r) acc[r] = 0ull;
    }
    const float4* kr = reinterpret_cast<const float4*>(sK + (st & 1) * kRouteKT * kRouteKSP + (32 * kgrp + lane) * kRouteKSP);
#pragma unroll
    for (int u = 0; u < kRouteDC / 4; ++u) {
      const float4 k4 = kr[u];
      const uint64_t kxy = f32x2(k4.x, k4.y), kzw = f32x2(k4.z, k4.w);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float4 x = reinterpret_cast<const float4*>(sQ + (4 * rgrp + r) * D)[ct * (kRouteDC / 4) + u];
        acc[r] = ffma2(f32x2(x.x, x.y), kxy, acc[r]);   // a0 += x.x k.x, a1 += x.y k.y
        acc[r] = ffma2(f32x2(x.z, x.w), kzw, acc[r]);   // a0 += x.z k.z, a1 += x.w k.w
      }
    }
    if (ct == NDC - 1) {
      const int key = round * kRouteKT + 32 * kgrp + lane;
      if (key < nB) {
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          float a0, a1;
          unpack_f32x2(acc[r], a0, a1);
          sL[(4 * rgrp + r) * nBpad + key] = (a0 + a1) * scale;
        }
      }
    }
    __syncthreads();   // this buffer is restaged by the next iteration's prefetch
  }
  const int qb = row0 + warp;
  if (qb < nB)
    select_row<MAXW>(sL + warp * nBpad, nB, words, qb, p, k_floor,
                     mask + (static_cast<size_t>(bhi) * nB + qb) * words,
                     counts + static_cast<size_t>(bhi) * nB + qb, lane);
}

size_t route_smem_bytes(const Geo& g) {
  const size_t nBpad = static_cast<size_t>(g.words) * 32;
  return (static_cast<size_t>(kRouteRows) * g.d + static_cast<size_t>(kRouteRows) * nBpad +
          2 * static_cast<size_t>(kRouteKT) * kRouteKSP) * 4;
}

template <int D, int MAXW>
static cudaError_t launch_route_t(const Geo& g, const float* qp, const float* kp, float p, int k_floor,
                                  float scale, uint32_t* mask, int32_t* counts, cudaStream_t st) {
  dim3 grid((g.nB + kRouteRows - 1) / kRouteRows, g.B * g.H);
  const size_t smem = route_smem_bytes(g);
  cudaError_t e = cudaFuncSetAttribute(route_kernel<D, MAXW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  route_kernel<D, MAXW><<<grid, kRouteThreads, smem, st>>>(g, qp, kp, p, k_floor, scale, mask, counts);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_route_d(const Geo& g, const float* qp, const float* kp, float p, int k_floor,
                                  float scale, uint32_t* mask, int32_t* counts, cudaStream_t st) {
  // a lane holds MAXW logits of the row; MAXW close to the word count keeps the 32-step
  // threshold search from running over empty slots
  if (g.words <= 4) return launch_route_t<D, 4>(g, qp, kp, p, k_floor, scale, mask, counts, st);
  if (g.words <= 8) return launch_route_t<D, 8>(g, qp, kp, p, k_floor, scale, mask, counts, st);
  if (g.words <= 12) return launch_route_t<D, 12>(g, qp, kp, p, k_floor, scale, mask, counts, st);
  if (g.words <= 16) return launch_route_t<D, 16>(g, qp, kp, p, k_floor, scale, mask, counts, st);
  if (g.words <= 20) return launch_route_t<D, 20>(g, qp, kp, p, k_floor, scale, mask, counts, st);
  if (g.words <= 24) return launch_route_t<D, 24>(g, qp, kp, p, k_floor, scale, mask, counts, st);
  if (g.words <= 32) return launch_route_t<D, 32>(g, qp, kp, p, k_floor, scale, mask, counts, st);
  if (g.words <= 48) return launch_route_t<D, 48>(g, qp, kp, p, k_floor, scale, mask, counts, st);
  return launch_route_t<D, 64>(g, qp, kp, p, k_floor, scale, mask, counts, st);
}

cudaError_t launch_route(const Geo& g, const float* qp, const float* kp, float p, int k_floor,
                         float scale, uint32_t* mask, int32_t* counts, cudaStream_t st) {
  return g.d == 128 ? launch_route_d<128>(g, qp, kp, p, k_floor, scale, mask, counts, st)
                    : launch_route_d<64>(g, qp, kp, p, k_floor, scale, mask, counts, st);
}

// ----------------------------------------------------------------------------
// Routing in two kernels, for callers that pass a workspace (fvattn_route_ws): the
// logits of every (query block, key block) pair go to the workspace as an fp32 matrix
// per (b, h), rows padded to words * 32; then one warp per query block runs the same
// selection as route_kernel from its row.  The per-logit arithmetic is the fused
// kernel's (two partial sums over the even and odd components of each float4 of d, in
// ascending d, added at the end, times scale), so both paths give the same mask.
// ----------------------------------------------------------------------------

// One 64 x 64 tile of logits: query blocks [64 qt, +64) against key blocks [64 kt, +64)
// of slice bhi.  sQ and sK are [64][D + 4] floats of shared memory each.  kL2 reads the
// pooled rows from L2 only (ld.global.cg): set when they were written earlier in the
// same kernel, by other CTAs.
// kSplit loads each float4 step's (x, y) operands, runs their 16 products, then the
// (z, w) ones: every accumulator sees the same operations in the same order as without
// it, with half the operand registers live (for the fused kernel's register budget).
template <int D, bool kL2, bool kSplit>
__device__ __forceinline__ void logits_tile(const Geo& g, const float* __restrict__ qp,
                                            const float* __restrict__ kp, float scale,
                                            float* __restrict__ logits, int qt, int kt, int bhi,
                                            float* sQ, float* sK) {
  constexpr int RS = D + 4;            // padded row (floats)
  const int nB = g.nB, nBpad = g.words * 32;
  const int q0 = qt * kLogitTile, k0 = kt * kLogitTile;
  const float* qh = qp + static_cast<size_t>(bhi) * nB * D;
  const float* kh = kp + static_cast<size_t>(bhi) * nB * D;
  for (int e = threadIdx.x; e < kLogitTile * D / 4; e += 256) {
    const int r = e / (D / 4), d4 = e - r * (D / 4);
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    const float4* qs = reinterpret_cast<const float4*>(qh + static_cast<size_t>(q0 + r) * D) + d4;
    const float4* ks = reinterpret_cast<const float4*>(kh + static_cast<size_t>(k0 + r) * D) + d4;
    reinterpret_cast<float4*>(sQ + r * RS)[d4] = q0 + r < nB ? (kL2 ? __ldcg(qs) : *qs) : z;
    reinterpret_cast<float4*>(sK + r * RS)[d4] = k0 + r < nB ? (kL2 ? __ldcg(ks) : *ks) : z;
  }
  __syncthreads();
  // thread (ty, tx) takes query rows ty + 16 i and key blocks tx + 16 j, i, j < 4
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  uint64_t acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0ull;
  if constexpr (kSplit) {
#pragma unroll 2
    for (int d4 = 0; d4 < D / 4; ++d4) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {    // h = 0: (x, y) components, h = 1: (z, w)
        uint64_t qv[4], kv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 x = reinterpret_cast<const float2*>(sQ + (ty + 16 * i) * RS)[2 * d4 + h];
          qv[i] = f32x2(x.x, x.y);
          const float2 k2 = reinterpret_cast<const float2*>(sK + (tx + 16 * i) * RS)[2 * d4 + h];
          kv[i] = f32x2(k2.x, k2.y);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = ffma2(qv[i], kv[j], acc[i][j]);
      }
    }
  } else {
#pragma unroll 4
    for (int d4 = 0; d4 < D / 4; ++d4) {
      uint64_t qxy[4], qzw[4], kxy[4], kzw[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 x = reinterpret_cast<const float4*>(sQ + (ty + 16 * i) * RS)[d4];
        qxy[i] = f32x2(x.x, x.y);
        qzw[i] = f32x2(x.z, x.w);
        const float4 k4 = reinterpret_cast<const float4*>(sK + (tx + 16 * i) * RS)[d4];
        kxy[i] = f32x2(k4.x, k4.y);
        kzw[i] = f32x2(k4.z, k4.w);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[i][j] = ffma2(qxy[i], kxy[j], acc[i][j]);   // a0 += x.x k.x, a1 += x.y k.y
          acc[i][j] = ffma2(qzw[i], kzw[j], acc[i][j]);   // a0 += x.z k.z, a1 += x.w k.w
        }
    }
  }
  float* out = logits + static_cast<size_t>(bhi) * nB * nBpad;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int qr = q0 + ty + 16 * i;
    if (qr >= nB) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int kc = k0 + tx + 16 * j;
      if (kc >= nB) continue;
      float a0, a1;
      unpack_f32x2(acc[i][j], a0, a1);
      out[static_cast<size_t>(qr) * nBpad + kc] = (a0 + a1) * scale;
    }
  }
}

template <int D>
__global__ void __launch_bounds__(256) logits_kernel(Geo g, const float* __restrict__ qp,
                                                     const float* __restrict__ kp, float scale,
                                                     float* __restrict__ logits) {
  extern __shared__ __align__(16) unsigned char lg_smem[];
  float* sQ = reinterpret_cast<float*>(lg_smem);   // [64][D + 4]
  float* sK = sQ + kLogitTile * (D + 4);           // [64][D + 4]
  logits_tile<D, false, false>(g, qp, kp, scale, logits, blockIdx.x, blockIdx.y, blockIdx.z, sQ, sK);
}

template <int MAXW>
__global__ void __launch_bounds__(256) select_kernel(Geo g, const float* __restrict__ logits, float p,
                                                     int k_floor, uint32_t* __restrict__ mask,
                                                     int32_t* __restrict__ counts) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nB = g.nB, nBpad = g.words * 32;
  const long long row = static_cast<long long>(blockIdx.x) * 8 + warp;   // (b*h) * nB + qb
  if (row >= static_cast<long long>(g.B) * g.H * nB) return;
  const int qb = static_cast<int>(row % nB);
  select_row<MAXW>(logits + static_cast<size_t>(row) * nBpad, nB, g.words, qb, p, k_floor,
                   mask + static_cast<size_t>(row) * g.words, counts + row, lane);
}

size_t route_ws_bytes(const Geo& g) {
  return static_cast<size_t>(g.B) * g.H * g.nB * (static_cast<size_t>(g.words) * 32) * 4;
}

template <int D, int MAXW>
static cudaError_t launch_route2_t(const Geo& g, const float* qp, const float* kp, float p, int k_floor,
                                   float scale, uint32_t* mask, int32_t* counts, float* logits,
                                   cudaStream_t st) {
  const int tiles = (g.nB + kLogitTile - 1) / kLogitTile;
  const int smem = 2 * kLogitTile * (D + 4) * 4;
  cudaError_t e = cudaFuncSetAttribute(logits_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  logits_kernel<D><<<dim3(tiles, tiles, g.B * g.H), 256, smem, st>>>(g, qp, kp, scale, logits);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const long long rows = static_cast<long long>(g.B) * g.H * g.nB;
  select_kernel<MAXW><<<static_cast<unsigned>((rows + 7) / 8), 256, 0, st>>>(g, logits, p, k_floor, mask, counts);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_route2_d(const Geo& g, const float* qp, const float* kp, float p, int k_floor,
                                   float scale, uint32_t* mask, int32_t* counts, float* logits,
                                   cudaStream_t st) {
  if (g.words <= 4) return launch_route2_t<D, 4>(g, qp, kp, p, k_floor, scale, mask, counts, logits, st);
  if (g.words <= 8) return launch_route2_t<D, 8>(g, qp, kp, p, k_floor, scale, mask, counts, logits, st);
  if (g.words <= 12) return launch_route2_t<D, 12>(g, qp, kp, p, k_floor, scale, mask, counts, logits, st);
  if (g.words <= 16) return launch_route2_t<D, 16>(g, qp, kp, p, k_floor, scale, mask, counts, logits, st);
  if (g.words <= 20) return launch_route2_t<D, 20>(g, qp, kp, p, k_floor, scale, mask, counts, logits, st);
  if (g.words <= 24) return launch_route2_t<D, 24>(g, qp, kp, p, k_floor, scale, mask, counts, logits, st);
  if (g.words <= 32) return launch_route2_t<D, 32>(g, qp, kp, p, k_floor, scale, mask, counts, logits, st);
  if (g.words <= 48) return launch_route2_t<D, 48>(g, qp, kp, p, k_floor, scale, mask, counts, logits, st);
  return launch_route2_t<D, 64>(g, qp, kp, p, k_floor, scale, mask, counts, logits, st);
}

cudaError_t launch_route_ws(const Geo& g, const float* qp, const float* kp, float p, int k_floor,
                            float scale, uint32_t* mask, int32_t* counts, void* ws, cudaStream_t st) {
  float* logits = static_cast<float*>(ws);
  return g.d == 128 ? launch_route2_d<128>(g, qp, kp, p, k_floor, scale, mask, counts, logits, st)
                    : launch_route2_d<64>(g, qp, kp, p, k_floor, scale, mask, counts, logits, st);
}

// ----------------------------------------------------------------------------
// Pool and route in one persistent kernel (fvattn_pool_route).  Pooling streams Q and K
// from HBM and leaves most instruction-issue slots idle; the route is bound by issue and
// reads only the pooled rows and logits, which stay in L2.  So the route of one (b, h)
// slice runs while later slices are still being pooled.  One queue holds three kinds of
// item, one CTA per item at a time:
//   pool      block j of slice s of Q or K                 (2 nB per slice)
//   logits    a 64 x 64 tile of slice s's logits           (tiles^2 per slice)
//   select    8 query blocks of slice s: Top-p / Top-k     (ceil(nB / 8) per slice)
// in steps: step i holds pool(i), then logits(i - 1), then select(i - 2), for the
// slices that exist.  A logits item waits for all pool items of its slice, a select item
// for all logits items of its slice (counters in the workspace header).  Every item
// waited on comes earlier in the queue, where a running CTA took it, so every wait ends;
// waits are bounded all the same, and on a timeout the select items write a mask that
// keeps every block.
// ----------------------------------------------------------------------------
constexpr int kFusedThreads = 256;
constexpr int kFusedMaxWords = 24;     // larger rows run the separate pool and route kernels
constexpr size_t kPrHeader = 256;      // queue counter, error bits; then 2 counters per slice

size_t pool_route_ws_bytes(const Geo& g) {
  const size_t S = static_cast<size_t>(g.B) * g.H;
  const size_t head = ((kPrHeader + 8 * S) + 255) / 256 * 256;
  return head + route_ws_bytes(g);
}

// Thread 0 waits until *cnt >= need: acquire loads, bounded by a clock64 deadline (2 s at
// up to 2 GHz) and by the error word (another item already gave up).  False on either.
__device__ __forceinline__ bool pr_wait(const uint32_t* cnt, uint32_t need, uint32_t* err) {
  long long t0 = clock64();
  for (uint32_t i = 0;; ++i) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(cnt) : "memory");
    if (v >= need) return true;
    if ((i & 15u) == 15u) {
      if (*reinterpret_cast<volatile uint32_t*>(err) & kErrTimeout) return false;
      if (static_cast<uint64_t>(clock64() - t0) > 4000000000ull) {
        atomicOr(err, kErrTimeout);
        return false;
      }
    }
    __nanosleep(128);
  }
}

// Every thread's writes of the item, then one count for the slice.
__device__ __forceinline__ void pr_done(uint32_t* cnt) {
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) atomicAdd(cnt, 1u);
}

template <int D, int MAXW>
__global__ void __launch_bounds__(kFusedThreads, 3) pool_route_kernel(
    Geo g, const uint4* __restrict__ q, const uint4* __restrict__ k, float* qp, float* kp, float p,
    int k_floor, float scale, uint32_t* __restrict__ mask, int32_t* __restrict__ counts,
    uint32_t* hdr, float* logits) {
  extern __shared__ __align__(16) unsigned char pr_smem[];
  float* sQ = reinterpret_cast<float*>(pr_smem);    // [64][D + 4]; select rows reuse it
  float* sK = sQ + kLogitTile * (D + 4);            // [64][D + 4]
  __shared__ float red[kPoolThreads / 32][D];
  __shared__ long long s_item;
  __shared__ int s_ok;
  uint32_t* err = hdr + 1;
  const int nB = g.nB, nBpad = g.words * 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (;;) {
    if (threadIdx.x == 0) s_item = static_cast<long long>(atomicAdd(reinterpret_cast<unsigned long long*>(hdr + 2), 1ull));
    __syncthreads();
    const long long t = s_item;
    __syncthreads();   // s_item is rewritten by the next iteration
    // the plan is recomputed per item (a few integer operations) rather than held in
    // registers across the loop
    const PrPlan pl = pr_plan(g.B * g.H, nB);
    if (t >= pl.total) break;
    uint32_t* cnt_pool = hdr + kPrHeader / 4;
    uint32_t* cnt_logit = cnt_pool + pl.S;
    int kind, slice, idx;
    pr_decode(pl, t, kind, slice, idx);
    if (kind == 0) {
      const int tensor = idx >= nB ? 1 : 0;
      const int j = idx - tensor * nB;
      pool_item<D>(g, tensor ? k : q, tensor ? kp : qp, j, slice, red);
      pr_done(cnt_pool + slice);
    } else if (kind == 1) {
      if (threadIdx.x == 0) s_ok = pr_wait(cnt_pool + slice, static_cast<uint32_t>(pl.nP), err) ? 1 : 0;
      __syncthreads();
      if (s_ok) {
        logits_tile<D, true, true>(g, qp, kp, scale, logits, idx / pl.tiles, idx - (idx / pl.tiles) * pl.tiles,
                             slice, sQ, sK);
        pr_done(cnt_logit + slice);
      }
    } else {
      if (threadIdx.x == 0) s_ok = pr_wait(cnt_logit + slice, static_cast<uint32_t>(pl.nL), err) ? 1 : 0;
      __syncthreads();
      const int qb = idx * 8 + warp;
      const size_t row = static_cast<size_t>(slice) * nB + qb;
      if (qb < nB) {
        uint32_t* mrow = mask + row * g.words;
        if (s_ok) {
          float* sL = sQ + warp * nBpad;
          const float* lrow = logits + row * nBpad;
          for (int c = lane; c < nBpad; c += 32) sL[c] = c < nB ? __ldcg(lrow + c) : 0.f;
          __syncwarp();
          select_row<MAXW>(sL, nB, g.words, qb, p, k_floor, mrow, counts + row, lane);
        } else {
          // the logits never arrived: keep every block, a mask the attention accepts
          const int tail = nB & 31;
          for (int w = lane; w < g.words; w += 32)
            mrow[w] = (w < g.words - 1 || tail == 0) ? 0xffffffffu : (1u << tail) - 1u;
          if (lane == 0) counts[row] = nB;
        }
      }
    }
  }
}

template <int D, int MAXW>
static cudaError_t launch_pool_route_t(const Geo& g, const void* q, const void* k, float* qp, float* kp,
                                       float p, int k_floor, float scale, uint32_t* mask, int32_t* counts,
                                       void* ws, int nsm, cudaStream_t st) {
  const PrPlan pl = pr_plan(g.B * g.H, g.nB);
  const size_t head = pool_route_ws_bytes(g) - route_ws_bytes(g);
  cudaError_t e = cudaMemsetAsync(ws, 0, head, st);
  if (e != cudaSuccess) return e;
  const int smem = 2 * kLogitTile * (D + 4) * 4;
  e = cudaFuncSetAttribute(pool_route_kernel<D, MAXW>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  // resident CTAs per SM, queried once per device (the first call, normally outside any
  // stream capture) and reused
  static int per_sm_of[64] = {};
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int per_sm = dev >= 0 && dev < 64 ? per_sm_of[dev] : 0;
  if (per_sm == 0) {
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, pool_route_kernel<D, MAXW>, kFusedThreads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    if (dev >= 0 && dev < 64) per_sm_of[dev] = per_sm;
  }
  const long long want = static_cast<long long>(nsm) * per_sm;
  const int grid = static_cast<int>(pl.total < want ? pl.total : want);
  uint32_t* hdr = static_cast<uint32_t*>(ws);
  float* logits = reinterpret_cast<float*>(static_cast<unsigned char*>(ws) + head);
  pool_route_kernel<D, MAXW><<<grid, kFusedThreads, smem, st>>>(
      g, static_cast<const uint4*>(q), static_cast<const uint4*>(k), qp, kp, p, k_floor, scale, mask, counts,
      hdr, logits);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_pool_route_d(const Geo& g, const void* q, const void* k, float* qp, float* kp,
                                       float p, int k_floor, float scale, uint32_t* mask, int32_t* counts,
                                       void* ws, int nsm, cudaStream_t st) {
  // MAXW sizes without register spills at three CTAs per SM (20 and, at d = 64, 4 spill);
  // empty slots of a row hold zero keys and add exact zeros, so the mask does not depend
  // on MAXW
  if (g.words <= 8) return launch_pool_route_t<D, 8>(g, q, k, qp, kp, p, k_floor, scale, mask, counts, ws, nsm, st);
  if (g.words <= 12) return launch_pool_route_t<D, 12>(g, q, k, qp, kp, p, k_floor, scale, mask, counts, ws, nsm, st);
  if (g.words <= 16) return launch_pool_route_t<D, 16>(g, q, k, qp, kp, p, k_floor, scale, mask, counts, ws, nsm, st);
  return launch_pool_route_t<D, 24>(g, q, k, qp, kp, p, k_floor, scale, mask, counts, ws, nsm, st);
}

cudaError_t launch_pool_route(const Geo& g, const void* q, const void* k, float* qp, float* kp, float p,
                              int k_floor, float scale, uint32_t* mask, int32_t* counts, void* ws, int nsm,
                              cudaStream_t st) {
  if (g.words > kFusedMaxWords) {
    // rows of more than 768 blocks: the separate kernels (the fused one would need more
    // registers per thread than three CTAs per SM leave)
    const size_t head = pool_route_ws_bytes(g) - route_ws_bytes(g);
    cudaError_t e = cudaMemsetAsync(ws, 0, head, st);   // clean error word for device_status
    if (e != cudaSuccess) return e;
    e = launch_pool(g, q, k, qp, kp, st);
    if (e != cudaSuccess) return e;
    return launch_route_ws(g, qp, kp, p, k_floor, scale, mask, counts,
                           static_cast<unsigned char*>(ws) + head, st);
  }
  return g.d == 128 ? launch_pool_route_d<128>(g, q, k, qp, kp, p, k_floor, scale, mask, counts, ws, nsm, st)
                    : launch_pool_route_d<64>(g, q, k, qp, kp, p, k_floor, scale, mask, counts, ws, nsm, st);
}

}  // namespace fv
