// Slack-aware sparse augmentation on one GPU.
//
// FVAttn explainer (arXiv 2607.16190), 核心方法 §3 Slack-Aware Sparse Augmentation: the
// slack that idle workers leave before the critical path ends is filled with high-value
// blocks, filtered by a score threshold (工程落地 item 5).  On one GPU the workers are the
// SMs of the persistent attention kernel, which runs tiles longest first:
//   cost(tile)  = real query tokens x real key tokens of its kept blocks;
//   final wave  = the last n_sm tiles of the order (cost descending, ties by tile index),
//                 where SMs fall idle; its largest tile sets the end, cost c*;
//   fill        = every tile of the wave takes its dropped blocks of routing score >= tau,
//                 in score order (logit descending, ties by lower index), each while the
//                 tile's cost stays <= c*, stopping at the first that does not fit.
// Three kernels: tile costs (one warp per tile), the wave (one CTA: a two-level radix
// select of the n_sm-th smallest cost, then the tie rule), and the fill (one warp per wave
// tile, scores from the route workspace's logits).
#include "fv_common.cuh"
#include "fv_launch.h"

namespace fv {

constexpr int kAugWarps = 8;
constexpr int kAugThreads = 1024;
constexpr int kAugMaxWords = 64;

__device__ __forceinline__ int aug_real(const Geo& g, int j) { return block_info(g, j).nvalid; }

// cost[t] = q_real(qb) * sum over kept kb of k_real(kb); blocks are classed by whether they
// sit in the last block column, row and frame (their real count follows from the class).
__global__ void __launch_bounds__(32 * kAugWarps) aug_cost_kernel(Geo g, const uint32_t* __restrict__ mask,
                                                                  int* __restrict__ cost, int ntiles) {
  __shared__ uint32_t edge[3][kAugMaxWords];
  __shared__ int cls_real[8];
  for (int w = threadIdx.x; w < g.words; w += blockDim.x) {
    uint32_t ex = 0, ey = 0, et = 0;
    for (int i = 0; i < 32; ++i) {
      const int j = w * 32 + i;
      if (j >= g.nB) break;
      const BlockInfo b = block_info(g, j);
      ex |= (b.xb == g.nBx - 1 ? 1u : 0u) << i;
      ey |= (b.yb == g.nBy - 1 ? 1u : 0u) << i;
      et |= (b.tb == g.nBt - 1 ? 1u : 0u) << i;
    }
    edge[0][w] = ex;
    edge[1][w] = ey;
    edge[2][w] = et;
  }
  if (threadIdx.x < 8) {
    const int k = threadIdx.x;
    const int xb = (k & 1) ? g.nBx - 1 : 0, yb = (k & 2) ? g.nBy - 1 : 0, tb = (k & 4) ? g.nBt - 1 : 0;
    cls_real[k] = aug_real(g, (tb * g.nBy + yb) * g.nBx + xb);
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int tail = g.nB & 31;
  for (int t = blockIdx.x * kAugWarps + (threadIdx.x >> 5); t < ntiles; t += gridDim.x * kAugWarps) {
    const uint32_t* row = mask + static_cast<size_t>(t) * g.words;
    int keys = 0;
    for (int w = lane; w < g.words; w += 32) {
      uint32_t m = row[w];
      if (w == g.words - 1 && tail) m &= (1u << tail) - 1u;
      const uint32_t ex = edge[0][w], ey = edge[1][w], et = edge[2][w];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t sel = ((k & 1) ? ex : ~ex) & ((k & 2) ? ey : ~ey) & ((k & 4) ? et : ~et);
        keys += cls_real[k] * __popc(m & sel);
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) keys += __shfl_xor_sync(0xffffffffu, keys, off);
    if (lane == 0) cost[t] = aug_real(g, t % g.nB) * keys;
  }
}

// The final wave: the n_sm tiles that come last in (cost desc, index asc) order, i.e. the
// n_sm smallest by (cost asc, index desc).  v = the n_sm-th smallest cost (radix select on
// 13 + 13 bits of the cost, costs < 2^26); the wave is every tile of cost < v and the
// largest-index tiles of cost v, as many as complete n_sm.  Writes the wave's tile ids to
// wave[0 .. n) and c* = v (the wave's largest cost) to hdr[3], n to hdr[4].
__global__ void __launch_bounds__(kAugThreads) aug_wave_kernel(const int* __restrict__ cost, int ntiles, int n_sm,
                                                               int* __restrict__ wave, uint32_t* hdr) {
  __shared__ int hist[8192];
  __shared__ int s_sel[2];   // the digit found, the count below it
  __shared__ int s_cnt;
  const int t = threadIdx.x;
  const int n = min(n_sm, ntiles);
  // level 0: high 13 bits; level 1: low 13 bits within the chosen high digit
  int want = n;              // rank (1-based) of the value searched among the remaining
  int prefix = 0;
#pragma unroll 1
  for (int level = 0; level < 2; ++level) {
    for (int i = t; i < 8192; i += kAugThreads) hist[i] = 0;
    __syncthreads();
    for (int i = t; i < ntiles; i += kAugThreads) {
      const int c = cost[i];
      if (level == 0) atomicAdd(&hist[(c >> 13) & 8191], 1);
      else if ((c >> 13) == prefix) atomicAdd(&hist[c & 8191], 1);
    }
    __syncthreads();
    if (t < 32) {
      // the digit where the running count reaches `want`: lane l scans 256 cells
      int run = 0;
      for (int e = 0; e < 256; ++e) run += hist[t * 256 + e];
      int incl = run;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (t >= off) incl += v;
      }
      int excl = incl - run;
      int found = -1, below = 0;
      if (incl >= want && excl < want) {
        for (int e = 0; e < 256; ++e) {
          const int h = hist[t * 256 + e];
          if (excl + h >= want) { found = t * 256 + e; below = excl; break; }
          excl += h;
        }
      }
      // exactly one lane holds the crossing (want <= ntiles, so it exists)
      if (found >= 0) {
        s_sel[0] = found;
        s_sel[1] = below;
      }
    }
    __syncthreads();
    const int digit = s_sel[0], below = s_sel[1];
    __syncthreads();
    want -= below;
    prefix = level == 0 ? digit : (prefix << 13) | digit;
  }
  const int v = prefix;              // the n-th smallest cost
  const int need = want;             // tiles of cost v in the wave (the largest indices)
  // tiles of cost < v, in any order, then the `need` largest-index tiles of cost v
  if (t == 0) s_cnt = 0;
  __syncthreads();
  for (int i = t; i < ntiles; i += kAugThreads)
    if (cost[i] < v) wave[atomicAdd(&s_cnt, 1)] = i;
  __syncthreads();
  const int base = s_cnt;
  __shared__ int s_taken;
  if (t == 0) s_taken = 0;
  __syncthreads();
  // scan index blocks of kAugThreads from the top down; within a block, ranks from the top
  for (int top = ntiles - 1; top >= 0; top -= kAugThreads) {
    const int i = top - t;
    const bool eq = i >= 0 && cost[i] == v;
    // rank among the equal tiles of this block with a higher index (warp ballot + block scan)
    __shared__ int wcnt[kAugThreads / 32];
    const uint32_t bal = __ballot_sync(0xffffffffu, eq);
    if ((t & 31) == 0) wcnt[t >> 5] = __popc(bal);
    __syncthreads();
    int before = 0;
    for (int w = 0; w < (t >> 5); ++w) before += wcnt[w];
    before += __popc(bal & ((1u << (t & 31)) - 1u));
    const int taken = s_taken;
    if (eq && taken + before < need) wave[base + taken + before] = i;
    __syncthreads();
    if (t == 0) {
      int tot = 0;
      for (int w = 0; w < kAugThreads / 32; ++w) tot += wcnt[w];
      s_taken = taken + tot;
    }
    __syncthreads();
    if (s_taken >= need) break;
  }
  if (t == 0) {
    hdr[3] = static_cast<uint32_t>(v);
    hdr[4] = static_cast<uint32_t>(n);
  }
}

// One warp per wave tile: scores from the tile's logit row, then the fill.
template <int MAXW>
__global__ void __launch_bounds__(32 * kAugWarps) aug_fill_kernel(Geo g, const float* __restrict__ logits,
                                                                  const int* __restrict__ wave,
                                                                  const int* __restrict__ cost,
                                                                  const uint32_t* __restrict__ hdr, float tau,
                                                                  uint32_t* __restrict__ mask,
                                                                  int32_t* __restrict__ counts) {
  const int lane = threadIdx.x & 31;
  const int w = blockIdx.x * kAugWarps + (threadIdx.x >> 5);
  const int n = static_cast<int>(hdr[4]);
  if (w >= n) return;
  const int cap = static_cast<int>(hdr[3]);
  const int tile = wave[w];
  const int nB = g.nB, nBpad = g.words * 32;
  const float* lrow = logits + static_cast<size_t>(tile) * nBpad;
  uint32_t* mrow = mask + static_cast<size_t>(tile) * g.words;
  const int qreal = aug_real(g, tile % nB);
  int c = cost[tile];
  float x[MAXW];
  bool cand[MAXW];
  float mx = -INFINITY;
#pragma unroll
  for (int k = 0; k < MAXW; ++k) {
    const int j = k * 32 + lane;
    x[k] = (k < g.words && j < nB) ? lrow[j] : -INFINITY;
    mx = fmaxf(mx, x[k]);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  float z = 0.f;
#pragma unroll
  for (int k = 0; k < MAXW; ++k) z += (x[k] > -INFINITY) ? expf(x[k] - mx) : 0.f;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
  const float inv_z = 1.f / z;
  uint32_t words[MAXW];
#pragma unroll
  for (int k = 0; k < MAXW; ++k) {
    const int j = k * 32 + lane;
    const uint32_t wd = k < g.words ? mrow[k] : 0u;
    words[k] = wd;
    const bool kept = (wd >> lane) & 1u;
    cand[k] = (k < g.words && j < nB) && !kept && expf(x[k] - mx) * inv_z >= tau;
  }
  // take the best remaining candidate (logit desc, index asc) while it fits
#pragma unroll 1
  for (;;) {
    float bx = -INFINITY;
    int bj = 0x7fffffff;
#pragma unroll
    for (int k = 0; k < MAXW; ++k) {
      const int j = k * 32 + lane;
      if (cand[k] && (x[k] > bx || (x[k] == bx && j < bj))) { bx = x[k]; bj = j; }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ox = __shfl_xor_sync(0xffffffffu, bx, off);
      const int oj = __shfl_xor_sync(0xffffffffu, bj, off);
      if (ox > bx || (ox == bx && oj < bj)) { bx = ox; bj = oj; }
    }
    if (bj == 0x7fffffff) break;
    const int add = qreal * aug_real(g, bj);
    if (c + add > cap) break;
    c += add;
#pragma unroll
    for (int k = 0; k < MAXW; ++k) {
      if (k * 32 + lane == bj) cand[k] = false;
      if (k == (bj >> 5)) words[k] |= 1u << (bj & 31);
    }
  }
  int cnt = 0;
#pragma unroll
  for (int k = 0; k < MAXW; ++k) {
    if (k < g.words) {
      cnt += __popc(words[k]);
      if (lane == 0) mrow[k] = words[k];
    }
  }
  if (lane == 0) counts[tile] = cnt;
}

size_t augment_scratch_bytes(const Geo& g) {
  const size_t ntiles = static_cast<size_t>(g.B) * g.H * g.nB;
  return 256 + ((ntiles * 8 + 255) / 256) * 256;
}

template <int MAXW>
static cudaError_t launch_fill(const Geo& g, const float* logits, const int* wave, const int* cost,
                               const uint32_t* hdr, float tau, uint32_t* mask, int32_t* counts, int n_sm,
                               cudaStream_t st) {
  aug_fill_kernel<MAXW><<<(n_sm + kAugWarps - 1) / kAugWarps, 32 * kAugWarps, 0, st>>>(g, logits, wave, cost, hdr,
                                                                                      tau, mask, counts);
  return cudaGetLastError();
}

cudaError_t launch_augment(const Geo& g, const float* logits, float tau, int n_sm, uint32_t* mask, int32_t* counts,
                           void* scratch, cudaStream_t st) {
  const int ntiles = g.B * g.H * g.nB;
  uint32_t* hdr = static_cast<uint32_t*>(scratch);
  int* cost = reinterpret_cast<int*>(static_cast<unsigned char*>(scratch) + 256);
  int* wave = cost + ntiles;
  aug_cost_kernel<<<(ntiles + kAugWarps - 1) / kAugWarps, 32 * kAugWarps, 0, st>>>(g, mask, cost, ntiles);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  aug_wave_kernel<<<1, kAugThreads, 0, st>>>(cost, ntiles, n_sm, wave, hdr);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (g.words <= 8) return launch_fill<8>(g, logits, wave, cost, hdr, tau, mask, counts, n_sm, st);
  if (g.words <= 16) return launch_fill<16>(g, logits, wave, cost, hdr, tau, mask, counts, n_sm, st);
  if (g.words <= 32) return launch_fill<32>(g, logits, wave, cost, hdr, tau, mask, counts, n_sm, st);
  return launch_fill<64>(g, logits, wave, cost, hdr, tau, mask, counts, n_sm, st);
}

}  // namespace fv
