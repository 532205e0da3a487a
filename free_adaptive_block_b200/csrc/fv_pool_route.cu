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

// Whether key block j holds a keyframe: latent frame t is one when (t - phase) mod
// stride == 0 (LVSA README, rotating keyframes); stride 0: no keyframes.
__device__ __forceinline__ bool keyframe_block(const Geo& g, const RouteOpts& o, int j) {
  if (o.kf_stride <= 0) return false;
  const int tb = div_r(j, g.nBy * g.nBx, g.r_plane);
  const int t0 = tb * g.bt, t1 = min(g.T, t0 + g.bt);
  int off = (o.kf_phase - t0) % o.kf_stride;
  if (off < 0) off += o.kf_stride;
  return t0 + off < t1;
}

// Selection for one query block; the row's logits are in sL[i], i = c*32 + lane.
// With o.token_mass the Top-p runs over tokens: the blocks keep the logits' order and a
// block's mass is its real token count times exp(logit - max), normalised over the row.
// Keyframe blocks (o.kf_stride > 0) are kept in every row, after the prefix rule.
template <int MAXW>
__device__ __forceinline__ void select_row(const Geo& g, const RouteOpts& o, const float* sL, int nB,
                                           int words, int qb, float p, int k_floor, uint32_t* mrow,
                                           int32_t* cnt_out, int lane) {
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
    float e = key[c] ? expf(sc[c] - mx) : 0.f;
    if (o.token_mass && key[c]) e *= static_cast<float>(block_info(g, c * 32 + lane).nvalid);
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
    int gt = 0;
    float gm = 0.f;
#pragma unroll
    for (int c = 0; c < MAXW; ++c) {
      if (key[c] > u) { ++gt; gm += sc[c]; }
    }
    gt = warp_sum_i(gt);
    gm = warp_sum(gm);
    // blocks with key u (ties) join in ascending block index, each with its own mass,
    // until the prefix reaches p
    float acc = gm;
    int r = 0;
#pragma unroll
    for (int c = 0; c < MAXW; ++c) {
      uint32_t tb = __ballot_sync(0xffffffffu, key[c] != 0u && key[c] == u);
      while (tb != 0u && acc < p) {
        const int l = __ffs(tb) - 1;
        tb &= tb - 1u;
        acc += __shfl_sync(0xffffffffu, sc[c], l);
        ++r;
      }
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
      const bool kept = valid && (key[c] > u || (tie && rank < ties_needed) || i == qb ||
                                  keyframe_block(g, o, i));
      const uint32_t word = __ballot_sync(0xffffffffu, kept);
      cnt += __popc(word);
      if (lane == 0) mrow[c] = word;
    }
  }
  if (lane == 0) *cnt_out = cnt;
}

// ----------------------------------------------------------------------------
// Selection by mass histogram (the form fvattn_route_ws, fvattn_route_ex and
// fvattn_pool_route use).  Same rule as select_row, with the masses summed exactly: every
// block's mass exp(l - max) (times its real token count for the Top-p over tokens) is
// rounded once to a fixed-point integer of 2^-32 units, and all sums are integer sums, so
// they do not depend on summation order and the prefix test "mass >= p" reads
// sum >= ceil(p * Z) in integers.  Per row (one warp):
//   1. logits into registers (lane l holds blocks c * 32 + l), row maximum;
//   2. a 256-bucket histogram of mass and count in shared memory, bucket
//      b = min(255, floor((max - l) * 16)): buckets are contiguous ranges of the logit
//      order, 1/16 logit wide, the last one holding everything 16 or more below the max
//      (at most e^-16 of the row's mass per block);
//   3. a warp scan over the buckets finds the bucket where the prefix mass reaches p;
//   4. that bucket's blocks (a few at these shapes) are gathered and ranked exactly by
//      (logit desc, index asc); the cut is the first rank at which the prefix reaches p;
//   5. the Top-k floor, when it lengthens the prefix, repeats 3-4 on counts;
//   6. the mask: blocks above the cut's key, tied blocks up to the cut's index, the own
//      block and keyframe blocks.
// A bucket with more than kSelCap blocks (a cut far down a nearly flat tail) runs
// select_row on the row instead.
// ----------------------------------------------------------------------------
constexpr int kSelBuckets = 256;
constexpr float kSelPerLogit = 16.f;
constexpr int kSelCap = 64;

struct SelScratch {                      // one per warp
  unsigned long long hm[kSelBuckets];    // mass per bucket (2^-32 units)
  uint32_t hc[kSelBuckets];              // blocks per bucket
  unsigned long long lw[kSelCap];        // gathered bucket: mass,
  uint32_t lkey[kSelCap];                //   order key,
  uint32_t lidx[kSelCap];                //   block index
};

__device__ __forceinline__ unsigned long long warp_sum_u64(unsigned long long v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

__device__ __forceinline__ int sel_bucket(float mx, float x) {
  return min(kSelBuckets - 1, __float2int_rz((mx - x) * kSelPerLogit));
}

__device__ __forceinline__ unsigned long long sel_fixed(float w) {
  return __float2ull_rn(w * 4294967296.0f);
}

// Finds the bucket where the running sum (mass when `by_mass`, else count) first reaches
// `target`, scanning buckets from the top of the order.  Returns the bucket and, through
// `above`, the sum over the buckets before it (and `cnt_above`, their block count).
__device__ __forceinline__ int sel_find_bucket(const SelScratch& sh, bool by_mass, unsigned long long target,
                                               unsigned long long& above, int& cnt_above, int lane) {
  unsigned long long loc[8];
  int cl[8];
  unsigned long long run = 0;
  int crun = 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int b = lane * 8 + e;
    cl[e] = static_cast<int>(sh.hc[b]);
    loc[e] = by_mass ? sh.hm[b] : static_cast<unsigned long long>(cl[e]);
    run += loc[e];
    crun += cl[e];
  }
  unsigned long long incl = run;
  int cincl = crun;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const unsigned long long v = __shfl_up_sync(0xffffffffu, incl, off);
    const int cv = __shfl_up_sync(0xffffffffu, cincl, off);
    if (lane >= off) { incl += v; cincl += cv; }
  }
  unsigned long long excl = incl - run;
  int cexcl = cincl - crun;
  int found = kSelBuckets;
  unsigned long long f_above = 0;
  int f_cnt = 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    if (found == kSelBuckets && excl + loc[e] >= target) {
      found = lane * 8 + e;
      f_above = excl;
      f_cnt = cexcl;
    }
    excl += loc[e];
    cexcl += cl[e];
  }
  const uint32_t hit = __ballot_sync(0xffffffffu, found < kSelBuckets);
  const int src = hit ? __ffs(hit) - 1 : 31;
  above = __shfl_sync(0xffffffffu, f_above, src);
  cnt_above = __shfl_sync(0xffffffffu, f_cnt, src);
  return hit ? __shfl_sync(0xffffffffu, found, src) : kSelBuckets - 1;
}

template <int MAXW>
__device__ __forceinline__ void select_row_hist(const Geo& g, const RouteOpts& o, const float* lrow, int nB,
                                                int words, int qb, float p, int k_floor, uint32_t* mrow,
                                                int32_t* cnt_out, int lane, SelScratch& sh) {
  uint32_t key[MAXW];
  float x[MAXW];
  float mx = -INFINITY;
#pragma unroll
  for (int c = 0; c < MAXW; ++c) {
    const int i = c * 32 + lane;
    const bool v = c < words && i < nB;
    x[c] = v ? __ldcg(lrow + i) : -INFINITY;
    key[c] = v ? order_key(x[c]) : 0u;
    mx = fmaxf(mx, x[c]);
  }
  mx = warp_max(mx);
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    sh.hm[lane * 8 + e] = 0ull;
    sh.hc[lane * 8 + e] = 0u;
  }
  __syncwarp();
  auto mass_of = [&](int c) -> float {
    float w = expf(x[c] - mx);
    if (o.token_mass) w *= static_cast<float>(block_info(g, c * 32 + lane).nvalid);
    return w;
  };
  unsigned long long z = 0;
#pragma unroll
  for (int c = 0; c < MAXW; ++c) {
    if (key[c] != 0u) {
      const unsigned long long w = sel_fixed(mass_of(c));
      const int b = sel_bucket(mx, x[c]);
      atomicAdd(&sh.hm[b], w);
      atomicAdd(&sh.hc[b], 1u);
      z += w;
    }
  }
  z = warp_sum_u64(z);
  __syncwarp();

  // Gathers bucket b's blocks into the list; false when they do not fit.
  auto gather = [&](int b, int n) -> bool {
    if (n > kSelCap) return false;
    int base = 0;
#pragma unroll
    for (int c = 0; c < MAXW; ++c) {
      const bool in = key[c] != 0u && sel_bucket(mx, x[c]) == b;
      const uint32_t bal = __ballot_sync(0xffffffffu, in);
      if (in) {
        const int pos = base + __popc(bal & ((1u << lane) - 1u));
        sh.lkey[pos] = key[c];
        sh.lidx[pos] = static_cast<uint32_t>(c * 32 + lane);
        sh.lw[pos] = sel_fixed(mass_of(c));
      }
      base += __popc(bal);
    }
    __syncwarp();
    return true;
  };
  // Among the n gathered blocks, the one of smallest rank (key desc, index asc) at which
  // above + (running sum of weights up to it) >= target; weight = mass or 1.
  auto resolve = [&](int n, bool by_mass, unsigned long long above, int& rank_out, uint32_t& key_out,
                     int& idx_out, unsigned long long target) {
    int best = 0x7fffffff;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int j = lane + 32 * h;
      if (j < n) {
        const uint32_t kj = sh.lkey[j], ij = sh.lidx[j];
        int rank = 0;
        unsigned long long pre = 0;
        for (int t = 0; t < n; ++t) {
          const uint32_t kt = sh.lkey[t], it = sh.lidx[t];
          const bool before = kt > kj || (kt == kj && it < ij);
          rank += before ? 1 : 0;
          if (before || t == j) pre += by_mass ? sh.lw[t] : 1ull;
        }
        // a block whose prefix reaches the target codes as its rank; the others code
        // above every such rank, the last in the order lowest (the whole bucket)
        best = min(best, above + pre >= target ? rank * 64 + j : (2 * n - 1 - rank) * 64 + j);
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) best = min(best, __shfl_xor_sync(0xffffffffu, best, off));
    const int j = best & 63;
    rank_out = best >> 6;
    key_out = sh.lkey[j];
    idx_out = static_cast<int>(sh.lidx[j]);
    __syncwarp();
  };

  const int floor_k = min(max(k_floor, 0), nB);
  int m_p = nB;
  uint32_t ucut = 0u;        // blocks with key > ucut, and key == ucut up to index icut, are kept
  int icut = -1;
  bool all = true;
  if (p < 1.f) {
    // at least one unit, so that p = 0 still keeps the first block of the order
    const unsigned long long target =
        max(1ull, static_cast<unsigned long long>(ceil(static_cast<double>(p) * static_cast<double>(z))));
    unsigned long long above;
    int cnt_above;
    const int b = sel_find_bucket(sh, true, target, above, cnt_above, lane);
    if (!gather(b, static_cast<int>(sh.hc[b]))) {
      select_row<MAXW>(g, o, lrow, nB, words, qb, p, k_floor, mrow, cnt_out, lane);
      return;
    }
    int rank;
    resolve(static_cast<int>(sh.hc[b]), true, above, rank, ucut, icut, target);
    m_p = cnt_above + rank + 1;
    all = false;
  }
  const int M = max(max(m_p, floor_k), 1);
  if (M >= nB) {
    all = true;
  } else if (M > m_p) {
    unsigned long long above;
    int cnt_above;
    const int b = sel_find_bucket(sh, false, static_cast<unsigned long long>(M), above, cnt_above, lane);
    if (!gather(b, static_cast<int>(sh.hc[b]))) {
      select_row<MAXW>(g, o, lrow, nB, words, qb, p, k_floor, mrow, cnt_out, lane);
      return;
    }
    int rank;
    resolve(static_cast<int>(sh.hc[b]), false, above, rank, ucut, icut, static_cast<unsigned long long>(M));
    all = false;
  }
  int cnt = 0;
#pragma unroll
  for (int c = 0; c < MAXW; ++c) {
    if (c < words) {
      const int i = c * 32 + lane;
      const bool valid = key[c] != 0u;
      const bool kept = valid && (all || key[c] > ucut || (key[c] == ucut && i <= icut) || i == qb ||
                                  keyframe_block(g, o, i));
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
    select_row<MAXW>(g, RouteOpts{}, sL + warp * nBpad, nB, words, qb, p, k_floor,
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
// Routing in two kernels, for callers that pass a workspace (fvattn_route_ws,
// fvattn_route_ex, fvattn_pool_route): the logits of every (query block, key block) pair go
// to the workspace as an fp32 matrix per (b, h), rows padded to words * 32, computed on
// the tensor cores (fv_route_tc.cu); then one warp per query block selects from its row
// by mass histogram (select_row_hist).
// ----------------------------------------------------------------------------
template <int MAXW>
__global__ void __launch_bounds__(128) select_hist_kernel(Geo g, RouteOpts o, const float* __restrict__ logits,
                                                          float p, int k_floor, uint32_t* __restrict__ mask,
                                                          int32_t* __restrict__ counts) {
  __shared__ SelScratch sh[4];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nB = g.nB, nBpad = g.words * 32;
  const long long row = static_cast<long long>(blockIdx.x) * 4 + warp;   // (b*h) * nB + qb
  if (row >= static_cast<long long>(g.B) * g.H * nB) return;
  const int qb = static_cast<int>(row % nB);
  select_row_hist<MAXW>(g, o, logits + static_cast<size_t>(row) * nBpad, nB, g.words, qb, p, k_floor,
                        mask + static_cast<size_t>(row) * g.words, counts + row, lane, sh[warp]);
}

// Route workspace: a 256-byte header (word 1: error bits of the logits kernel's bounded
// waits), then the logits, [B*H][nB][words * 32] fp32.
constexpr size_t kRouteHdr = 256;

size_t route_logits_bytes(const Geo& g) {
  return static_cast<size_t>(g.B) * g.H * g.nB * (static_cast<size_t>(g.words) * 32) * 4;
}

size_t route_ws_bytes(const Geo& g) { return kRouteHdr + route_logits_bytes(g); }

template <int D, int MAXW>
static cudaError_t launch_route2_t(const Geo& g, const float* qp, const float* kp, float p, int k_floor,
                                   float scale, uint32_t* mask, int32_t* counts, void* ws,
                                   cudaStream_t st, const RouteOpts& o) {
  uint32_t* hdr = static_cast<uint32_t*>(ws);
  float* logits = reinterpret_cast<float*>(static_cast<unsigned char*>(ws) + kRouteHdr);
  cudaError_t e = cudaMemsetAsync(hdr, 0, kRouteHdr, st);
  if (e != cudaSuccess) return e;
  int dev = 0, nsm = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  e = launch_logits_tc(g, qp, kp, scale, logits, hdr + 1, nsm, st);
  if (e != cudaSuccess) return e;
  const long long rows = static_cast<long long>(g.B) * g.H * g.nB;
  select_hist_kernel<MAXW><<<static_cast<unsigned>((rows + 3) / 4), 128, 0, st>>>(g, o, logits, p, k_floor,
                                                                                   mask, counts);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_route2_d(const Geo& g, const float* qp, const float* kp, float p, int k_floor,
                                   float scale, uint32_t* mask, int32_t* counts, void* ws,
                                   cudaStream_t st, const RouteOpts& o) {
  if (g.words <= 4) return launch_route2_t<D, 4>(g, qp, kp, p, k_floor, scale, mask, counts, ws, st, o);
  if (g.words <= 8) return launch_route2_t<D, 8>(g, qp, kp, p, k_floor, scale, mask, counts, ws, st, o);
  if (g.words <= 12) return launch_route2_t<D, 12>(g, qp, kp, p, k_floor, scale, mask, counts, ws, st, o);
  if (g.words <= 16) return launch_route2_t<D, 16>(g, qp, kp, p, k_floor, scale, mask, counts, ws, st, o);
  if (g.words <= 20) return launch_route2_t<D, 20>(g, qp, kp, p, k_floor, scale, mask, counts, ws, st, o);
  if (g.words <= 24) return launch_route2_t<D, 24>(g, qp, kp, p, k_floor, scale, mask, counts, ws, st, o);
  if (g.words <= 32) return launch_route2_t<D, 32>(g, qp, kp, p, k_floor, scale, mask, counts, ws, st, o);
  if (g.words <= 48) return launch_route2_t<D, 48>(g, qp, kp, p, k_floor, scale, mask, counts, ws, st, o);
  return launch_route2_t<D, 64>(g, qp, kp, p, k_floor, scale, mask, counts, ws, st, o);
}

cudaError_t launch_route_ws(const Geo& g, const float* qp, const float* kp, float p, int k_floor,
                            float scale, uint32_t* mask, int32_t* counts, void* ws, cudaStream_t st,
                            const RouteOpts& o) {
  return g.d == 128 ? launch_route2_d<128>(g, qp, kp, p, k_floor, scale, mask, counts, ws, st, o)
                    : launch_route2_d<64>(g, qp, kp, p, k_floor, scale, mask, counts, ws, st, o);
}

// ----------------------------------------------------------------------------
// Runtime mask repair (FVAttn explainer, 核心方法 §1, 运行时修补: the materialized mask
// is patched locally, without new scores).  In each row, a dropped key block whose two
// neighbours along the time, height or width axis of the block grid both exist and are
// both kept is a one-block hole and is restored; every decision reads the mask as given
// (one pass).  One warp per row: the row is staged in shared memory (so the call may
// work in place), and lane l writes words l and l + 32.  Per axis, bit j of a word has
// its neighbours j - step and j + step: two 32-bit windows of the row.  A bit qualifies
// only when its coordinate along the axis is interior (a table per CTA).
// ----------------------------------------------------------------------------
constexpr int kRepairWarps = 8;
constexpr int kRepairMaxWords = 64;    // nB <= 2048

// 32 bits of the row starting at bit `start` (bits outside [0, nB) read as zero).
__device__ __forceinline__ uint32_t row_window(const uint32_t* row, int words, int start) {
  const int w = start >> 5, sh = start & 31;   // arithmetic shift: floor for negative starts
  const uint32_t lo = (w >= 0 && w < words) ? row[w] : 0u;
  const uint32_t hi = (w + 1 >= 0 && w + 1 < words) ? row[w + 1] : 0u;
  return sh == 0 ? lo : ((lo >> sh) | (hi << (32 - sh)));
}

__global__ void __launch_bounds__(32 * kRepairWarps) mask_repair_kernel(Geo g, const uint32_t* in,
                                                                        uint32_t* out, int32_t* counts) {
  __shared__ uint32_t interior[3][kRepairMaxWords];        // per axis: bits with both neighbours
  __shared__ uint32_t rowbuf[kRepairWarps][kRepairMaxWords];
  const int words = g.words, nB = g.nB;
  for (int w = threadIdx.x; w < 3 * words; w += blockDim.x) {
    const int axis = w / words, wi = w - axis * words;
    uint32_t bits = 0u;
    for (int b = 0; b < 32; ++b) {
      const int j = wi * 32 + b;
      if (j >= nB) break;
      const BlockInfo bi = block_info(g, j);
      const int c = axis == 0 ? bi.tb : (axis == 1 ? bi.yb : bi.xb);
      const int ext = axis == 0 ? g.nBt : (axis == 1 ? g.nBy : g.nBx);
      if (c > 0 && c < ext - 1) bits |= 1u << b;
    }
    interior[axis][wi] = bits;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long rows = static_cast<long long>(g.B) * g.H * nB;
  const long long row = static_cast<long long>(blockIdx.x) * kRepairWarps + warp;
  if (row >= rows) return;
  uint32_t* rb = rowbuf[warp];
  const uint32_t* src = in + row * words;
  for (int w = lane; w < words; w += 32) rb[w] = src[w];
  __syncwarp();
  const int steps[3] = {g.nBy * g.nBx, g.nBx, 1};
  int cnt = 0;
  for (int w = lane; w < words; w += 32) {
    uint32_t m = rb[w];
#pragma unroll
    for (int a = 0; a < 3; ++a) {
      const uint32_t left = row_window(rb, words, w * 32 - steps[a]);
      const uint32_t right = row_window(rb, words, w * 32 + steps[a]);
      m |= left & right & interior[a][w];
    }
    if (w == words - 1 && (nB & 31)) m &= (1u << (nB & 31)) - 1u;   // no block at or past nB
    cnt += __popc(m);
    out[row * words + w] = m;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
  if (lane == 0) counts[row] = cnt;
}

cudaError_t launch_mask_repair(const Geo& g, const uint32_t* in, uint32_t* out, int32_t* counts,
                               cudaStream_t st) {
  const long long rows = static_cast<long long>(g.B) * g.H * g.nB;
  mask_repair_kernel<<<static_cast<unsigned>((rows + kRepairWarps - 1) / kRepairWarps), 32 * kRepairWarps, 0,
                       st>>>(g, in, out, counts);
  return cudaGetLastError();
}

// ----------------------------------------------------------------------------
// fvattn_pool_route: pooling, then the workspace route, in one call (three kernels on the
// caller's stream).  Its workspace is the route workspace.
// ----------------------------------------------------------------------------
size_t pool_route_ws_bytes(const Geo& g) { return route_ws_bytes(g); }

cudaError_t launch_pool_route(const Geo& g, const void* q, const void* k, float* qp, float* kp, float p,
                              int k_floor, float scale, uint32_t* mask, int32_t* counts, void* ws, int nsm,
                              cudaStream_t st) {
  (void)nsm;
  cudaError_t e = launch_pool(g, q, k, qp, kp, st);
  if (e != cudaSuccess) return e;
  return launch_route_ws(g, qp, kp, p, k_floor, scale, mask, counts, ws, st);
}

}  // namespace fv
