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

namespace fv {

// ----------------------------------------------------------------------------
// Pooling: one CTA per (b*h, block).  Thread t owns the 16-byte chunk t % (d/8) of
// the tokens t / (d/8), t / (d/8) + 256 / (d/8), ...  of the block; partial sums
// are folded with warp shuffles, then across warps through shared memory.
// Loads are 16-byte vectors, and a warp reads whole 256-byte token rows.
// ----------------------------------------------------------------------------
constexpr int kPoolThreads = 256;

template <int D>
__global__ void __launch_bounds__(kPoolThreads) pool_kernel(Geo g, const uint4* __restrict__ q,
                                                            const uint4* __restrict__ k,
                                                            float* __restrict__ qp,
                                                            float* __restrict__ kp) {
  constexpr int CH = D / 8;               // 16-byte chunks per token
  constexpr int G = kPoolThreads / CH;     // tokens processed side by side
  constexpr int MAXR = 128 / G;            // a block holds at most 128 tokens
  __shared__ float red[2][kPoolThreads / 32][D];

  const int j = blockIdx.x;
  const int bhi = blockIdx.y;
  const BlockInfo bi = block_info(g, j);
  const int nreal = bi.nvalid;
  const int plane = bi.ry * bi.rx;
  const int ch = threadIdx.x % CH;
  const int grp = threadIdx.x / CH;
  const size_t base = static_cast<size_t>(bhi) * g.N;
  const int t0 = bi.tb * g.bt, y0 = bi.yb * g.bh, x0 = bi.xb * g.bw;

  uint4 vq[MAXR], vk[MAXR];
#pragma unroll
  for (int i = 0; i < MAXR; ++i) {
    const int r = grp + i * G;
    if (r < nreal) {
      const int tt = r / plane;
      const int r2 = r - tt * plane;
      const int yy = r2 / bi.rx;
      const int xx = r2 - yy * bi.rx;
      const size_t n = base + (static_cast<size_t>(t0 + tt) * g.Hs + (y0 + yy)) * g.Ws + (x0 + xx);
      vq[i] = __ldg(q + n * CH + ch);
      vk[i] = __ldg(k + n * CH + ch);
    } else {
      vq[i] = make_uint4(0, 0, 0, 0);
      vk[i] = make_uint4(0, 0, 0, 0);
    }
  }
  float aq[8], ak[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) aq[e] = ak[e] = 0.f;
#pragma unroll
  for (int i = 0; i < MAXR; ++i) {
    const uint32_t wq[4] = {vq[i].x, vq[i].y, vq[i].z, vq[i].w};
    const uint32_t wk[4] = {vk[i].x, vk[i].y, vk[i].z, vk[i].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      aq[2 * e] += __uint_as_float(wq[e] << 16);
      aq[2 * e + 1] += __uint_as_float(wq[e] & 0xFFFF0000u);
      ak[2 * e] += __uint_as_float(wk[e] << 16);
      ak[2 * e + 1] += __uint_as_float(wk[e] & 0xFFFF0000u);
    }
  }
  // lanes l, l + CH, ... of a warp hold the same chunk
#pragma unroll
  for (int off = CH; off < 32; off <<= 1) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      aq[e] += __shfl_xor_sync(0xffffffffu, aq[e], off);
      ak[e] += __shfl_xor_sync(0xffffffffu, ak[e], off);
    }
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane < CH) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      red[0][warp][lane * 8 + e] = aq[e];
      red[1][warp][lane * 8 + e] = ak[e];
    }
  }
  __syncthreads();
  const float inv = 1.f / static_cast<float>(nreal);
  for (int t = threadIdx.x; t < 2 * D; t += kPoolThreads) {
    const int which = t / D, dd = t - which * D;
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kPoolThreads / 32; ++w) s += red[which][w][dd];
    float* dst = which ? kp : qp;
    dst[(static_cast<size_t>(bhi) * g.nB + j) * D + dd] = s * inv;
  }
}

cudaError_t launch_pool(const Geo& g, const void* q, const void* k, float* qp, float* kp,
                        cudaStream_t st) {
  dim3 grid(g.nB, g.B * g.H);
  if (g.d == 128)
    pool_kernel<128><<<grid, kPoolThreads, 0, st>>>(g, static_cast<const uint4*>(q),
                                                     static_cast<const uint4*>(k), qp, kp);
  else
    pool_kernel<64><<<grid, kPoolThreads, 0, st>>>(g, static_cast<const uint4*>(q),
                                                    static_cast<const uint4*>(k), qp, kp);
  return cudaGetLastError();
}

// ----------------------------------------------------------------------------
// Routing: one CTA per (b*h, 16 query blocks); warp w owns query blocks 2w and 2w+1
// of the CTA.  Logits come from key tiles of 32 blocks staged in shared memory (lane =
// key block, 16-byte loads along d).  Then, per query block, with the row's logits and
// scores held in registers: softmax over all key blocks, and a bitwise search for the
// Top-p cut over an order-preserving integer key of the logits, so no sort is needed:
//   u* = the largest key with mass(key >= u*) >= p  -> the key of the m_p-th block;
// equal keys are taken in ascending block index.  The Top-k floor lengthens the
// prefix with a second search on counts.  Reductions are warp shuffles in a fixed
// order, so the result is deterministic.
// ----------------------------------------------------------------------------
constexpr int kRouteRows = 16;
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
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = u | (1u << bit);
      float m = 0.f;
#pragma unroll
      for (int c = 0; c < MAXW; ++c) m += key[c] >= cand ? sc[c] : 0.f;
      if (warp_sum(m) >= p) u = cand;
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
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = v | (1u << bit);
      int n = 0;
#pragma unroll
      for (int c = 0; c < MAXW; ++c) n += key[c] >= cand ? 1 : 0;
      if (warp_sum_i(n) >= M) v = cand;
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

template <int D, int MAXW>
__global__ void __launch_bounds__(kRouteThreads) route_kernel(Geo g, const float* __restrict__ qp,
                                                              const float* __restrict__ kp, float p,
                                                              int k_floor, float scale,
                                                              uint32_t* __restrict__ mask,
                                                              int32_t* __restrict__ counts) {
  extern __shared__ __align__(16) unsigned char route_smem[];
  constexpr int KS = D + 4;                                      // padded key row (floats)
  const int words = g.words;
  const int nBpad = words * 32;
  float* sQ = reinterpret_cast<float*>(route_smem);              // [16][D]
  float* sK = sQ + kRouteRows * D;                               // [32][D + 4]
  float* sL = sK + 32 * KS;                                      // [16][nBpad]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bhi = blockIdx.y;
  const int nB = g.nB;
  const int row0 = blockIdx.x * kRouteRows;
  const float* kph = kp + static_cast<size_t>(bhi) * nB * D;

  for (int e = threadIdx.x; e < kRouteRows * D / 4; e += kRouteThreads) {
    const int r = e / (D / 4), d4 = e - r * (D / 4);
    const int row = row0 + r;
    reinterpret_cast<float4*>(sQ)[e] =
        row < nB ? reinterpret_cast<const float4*>(qp + (static_cast<size_t>(bhi) * nB + row) * D)[d4]
                 : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  const float4* q0 = reinterpret_cast<const float4*>(sQ + (2 * warp) * D);
  const float4* q1 = reinterpret_cast<const float4*>(sQ + (2 * warp + 1) * D);
  for (int kt = 0; kt < words; ++kt) {
    __syncthreads();
    for (int e = threadIdx.x; e < 32 * D / 4; e += kRouteThreads) {
      const int key = e / (D / 4), d4 = e - key * (D / 4);
      const int j = kt * 32 + key;
      reinterpret_cast<float4*>(sK + key * KS)[d4] =
          j < nB ? reinterpret_cast<const float4*>(kph + static_cast<size_t>(j) * D)[d4]
                 : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncthreads();
    const float4* kr = reinterpret_cast<const float4*>(sK + lane * KS);
    float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
#pragma unroll 8
    for (int d4 = 0; d4 < D / 4; ++d4) {
      const float4 k4 = kr[d4], x = q0[d4], y = q1[d4];
      a0 = fmaf(x.x, k4.x, a0); a1 = fmaf(x.y, k4.y, a1);
      a0 = fmaf(x.z, k4.z, a0); a1 = fmaf(x.w, k4.w, a1);
      b0 = fmaf(y.x, k4.x, b0); b1 = fmaf(y.y, k4.y, b1);
      b0 = fmaf(y.z, k4.z, b0); b1 = fmaf(y.w, k4.w, b1);
    }
    sL[(2 * warp) * nBpad + kt * 32 + lane] = (a0 + a1) * scale;
    sL[(2 * warp + 1) * nBpad + kt * 32 + lane] = (b0 + b1) * scale;
  }
  __syncwarp();
  for (int r = 0; r < 2; ++r) {
    const int lr = 2 * warp + r;
    const int qb = row0 + lr;
    if (qb >= nB) break;
    select_row<MAXW>(sL + lr * nBpad, nB, words, qb, p, k_floor,
                     mask + (static_cast<size_t>(bhi) * nB + qb) * words,
                     counts + static_cast<size_t>(bhi) * nB + qb, lane);
  }
}

size_t route_smem_bytes(const Geo& g) {
  const size_t nBpad = static_cast<size_t>(g.words) * 32;
  return (static_cast<size_t>(kRouteRows) * g.d + 32 * static_cast<size_t>(g.d + 4) +
          static_cast<size_t>(kRouteRows) * nBpad) * 4;
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
  if (g.words <= 16) return launch_route_t<D, 16>(g, qp, kp, p, k_floor, scale, mask, counts, st);
  if (g.words <= 32) return launch_route_t<D, 32>(g, qp, kp, p, k_floor, scale, mask, counts, st);
  return launch_route_t<D, 64>(g, qp, kp, p, k_floor, scale, mask, counts, st);
}

cudaError_t launch_route(const Geo& g, const float* qp, const float* kp, float p, int k_floor,
                         float scale, uint32_t* mask, int32_t* counts, cudaStream_t st) {
  return g.d == 128 ? launch_route_d<128>(g, qp, kp, p, k_floor, scale, mask, counts, st)
                    : launch_route_d<64>(g, qp, kp, p, k_floor, scale, mask, counts, st);
}

}  // namespace fv
