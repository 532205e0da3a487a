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
// Selection by mass histogram, for rows of more than kHistMinWords mask words (the form
// fvattn_route_ws, fvattn_route_ex and fvattn_pool_route take there).  Same rule as
// select_row, with the masses summed exactly: every block's mass 2^((l - max) log2 e)
// (times its real token count for the Top-p over tokens) is rounded once to a fixed-point
// integer of 2^-32 units, held as two int32 parts, and all sums are integer sums: they do
// not depend on summation order, and the prefix test "mass >= p" reads sum >= ceil(p Z) in
// integers.  Blocks are ordered by (logit desc, index asc), logits compared as floats.
// One warp per row:
//   1. the row into shared memory with 16-byte loads (blocks at or past nB as -inf) and
//      its maximum;
//   2. a 512-bucket histogram of mass (two 32-bit shared atomics per block), bucket
//      round(32 (max - l)) clamped to 511: monotone in l;
//   3. a warp scan over the buckets gives Z and the bucket where the prefix reaches
//      ceil(p Z), and a pass lists that bucket's blocks (up to 256, in index order);
//   4. at most 32 listed blocks are ranked exactly against each other, one per lane, and
//      the cut is the first in the order at which the prefix reaches the target; a longer
//      list is narrowed first by histograms over the 9 key bits below its highest
//      differing bit, level after level;
//   5. the mask: the blocks up to the cut, the own block, keyframe blocks.  The pass also
//      counts m_p, and when the Top-k floor lengthens the prefix the cut is found again
//      on counts and the mask rewritten.
// More than 256 blocks in the cut bucket, or more than 32 blocks of one logit, fall back
// to an exact bitwise search over the row.
// ----------------------------------------------------------------------------
constexpr int kHB = 512;                // buckets (and sub-buckets of the list levels)
constexpr int kSelList = 256;           // listed blocks of the cut bucket
constexpr int kSelWarps = 4;            // rows (warps) per CTA

struct SelSmem {
  int* hh;        // [kHB] per bucket: sum of the mass high parts (or a block count) ...
  int* hl;        // [kHB]   ... and of the low parts (signed); hh, hl contiguous
  float* lx;      // [kSelList] listed blocks: logit ...
  int* li;        //   ... and block index
  float* x;       // [words * 32] the row
};

__host__ __device__ constexpr size_t sel_warp_bytes(int words) {
  return 2 * kHB * 4 + kSelList * 8 + static_cast<size_t>(words) * 128;
}

__device__ __forceinline__ SelSmem sel_smem_at(unsigned char* base) {
  SelSmem s;
  s.hh = reinterpret_cast<int*>(base);
  s.hl = s.hh + kHB;
  s.lx = reinterpret_cast<float*>(s.hl + kHB);
  s.li = reinterpret_cast<int*>(s.lx + kSelList);
  s.x = reinterpret_cast<float*>(s.li + kSelList);
  return s;
}

// Order key of a logit with -0 taken as +0, so that key order is float order.
__device__ __forceinline__ uint32_t sel_key(float x) { return order_key(__fadd_rn(x, 0.f)); }
__device__ __forceinline__ float key_value(uint32_t k) {   // inverse of order_key
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

__device__ __forceinline__ long long warp_sum_ll(long long v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

// Bucket of a logit: the bits of fma(l, -32, cb) with cb = fl(32 max + 1.5 * 2^23), which
// hold round(32 (max - l) + delta) (delta, the rounding of cb, is one constant for the
// row), clamped to [0, 511]; -inf lands in 511.  A higher logit never lands later.
__device__ __forceinline__ int sel_bucket(float x, float cb) {
  return min(max(__float_as_int(__fmaf_rn(x, -32.f, cb)) - 0x4B400000, 0), kHB - 1);
}

// A block's mass in 2^-32 units as hh * 2^20 + hl: a = w * 2^12, hh = round(a),
// hl = round((a - hh) * 2^20), each rounded by the 1.5 * 2^23 shifter (exact: a <= 2^19
// since a block holds at most 2^7 tokens, and |a - hh| <= 1/2).  Over at most 2^11 blocks
// sum(hh) <= 2^30 and |sum(hl)| <= 2^30.  TOKEN: times the block's real token count.
struct MassParts {
  int hh, hl;
};
template <bool TOKEN>
__device__ __forceinline__ MassParts sel_mass(const Geo& g, float x, float nmx, int i) {
  float w = ex2(__fmul_rn(__fadd_rn(x, nmx), 1.4426950408889634f));
  if (TOKEN) w = __fmul_rn(w, static_cast<float>(block_info(g, i).nvalid));
  const float a = __fmul_rn(w, 4096.f);
  const float t1 = __fadd_rn(a, 12582912.f);
  const float lo = __fsub_rn(a, __fsub_rn(t1, 12582912.f));
  const float t2 = __fmaf_rn(lo, 1048576.f, 12582912.f);
  return MassParts{__float_as_int(t1) - 0x4B400000, __float_as_int(t2) - 0x4B400000};
}
__device__ __forceinline__ long long parts64(int hh, int hl) {
  return (static_cast<long long>(hh) << 20) + hl;
}

__device__ __forceinline__ void hist_zero(const SelSmem& sh, int lane) {
  int4* h = reinterpret_cast<int4*>(sh.hh);       // hh and hl: 2 * kHB ints
#pragma unroll
  for (int e = lane; e < 2 * kHB / 4; e += 32) h[e] = make_int4(0, 0, 0, 0);
  __syncwarp();
}

// Warp scan over the buckets, lane l owning buckets 16 l .. 16 l + 15 (by_mass: mass
// parts, else counts in hh).  Returns the total; excl / own: the sums before this lane's
// buckets and of them.
__device__ __forceinline__ long long hist_scan(const SelSmem& sh, bool by_mass, int lane, long long& excl,
                                               long long& own) {
  const int4* h = reinterpret_cast<const int4*>(sh.hh + 16 * lane);
  const int4* l = reinterpret_cast<const int4*>(sh.hl + 16 * lane);
  int sh_ = 0, sl_ = 0;
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    const int4 a = h[v];
    sh_ += (a.x + a.y) + (a.z + a.w);
    if (by_mass) {
      const int4 b = l[v];
      sl_ += (b.x + b.y) + (b.z + b.w);
    }
  }
  own = by_mass ? parts64(sh_, sl_) : static_cast<long long>(sh_);
  long long incl = own;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const long long v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  excl = incl - own;
  return __shfl_sync(0xffffffffu, incl, 31);
}

// The first bucket at which the running sum reaches target (1 <= target <= total), and
// the sum of the buckets before it.
__device__ __forceinline__ int hist_cross(const SelSmem& sh, bool by_mass, int lane, long long excl, long long own,
                                          long long target, long long& above) {
  int found = -1;
  long long f_above = 0;
  if (excl < target && excl + own >= target) {
    long long run = excl;
#pragma unroll 1
    for (int e = 0; e < 16; ++e) {
      const int b = 16 * lane + e;
      const long long v = by_mass ? parts64(sh.hh[b], sh.hl[b]) : static_cast<long long>(sh.hh[b]);
      if (run + v >= target) {
        found = b;
        f_above = run;
        break;
      }
      run += v;
    }
  }
  const uint32_t hit = __ballot_sync(0xffffffffu, found >= 0);
  const int src = hit ? __ffs(hit) - 1 : 31;
  above = __shfl_sync(0xffffffffu, f_above, src);
  return hit ? __shfl_sync(0xffffffffu, found, src) : kHB - 1;
}

// Among n <= 32 candidates (lane j < n holds logit xj, index ij, weight wj), the first in
// the order (logit desc, index asc) at which base + (the sum of weights up to and
// including it) >= target; its lane.  The last candidate in the order always qualifies
// when the candidates hold all the weight up to the target.
__device__ __forceinline__ int resolve32(int n, float xj, int ij, long long wj, long long base, long long target,
                                         int lane) {
  int rank = 0;
  long long pre = 0;
#pragma unroll 1
  for (int t = 0; t < n; ++t) {
    const float xt = __shfl_sync(0xffffffffu, xj, t);
    const int it = __shfl_sync(0xffffffffu, ij, t);
    const long long wt = __shfl_sync(0xffffffffu, wj, t);
    const bool before = xt > xj || (xt == xj && it <= ij);
    rank += (before && t != lane) ? 1 : 0;
    pre += before ? wt : 0ll;
  }
  int code = 0x7fffffff;
  if (lane < n) code = (base + pre >= target ? rank : 2 * n - 1 - rank) * 64 + lane;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) code = min(code, __shfl_xor_sync(0xffffffffu, code, off));
  return code & 63;
}

template <bool TOKEN>
__device__ __forceinline__ long long sel_weight(const Geo& g, bool by_mass, float x, float nmx, int i) {
  if (!by_mass) return 1ll;
  const MassParts m = sel_mass<TOKEN>(g, x, nmx, i);
  return parts64(m.hh, m.hl);
}

// Exact fallback: u = the largest key whose prefix (all blocks of key >= u) reaches the
// target, by a bitwise search over the row; then the blocks of key u in index order.
// Returns false never; sets the cut (logit and index of the block where the sum reaches
// the target).
template <bool TOKEN>
__device__ void sel_search(const Geo& g, const SelSmem& sh, int words, int nB, bool by_mass, float nmx,
                           long long target, int lane, float& xcut, int& icut) {
  uint32_t u = 0;
#pragma unroll 1
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = u | (1u << bit);
    long long m = 0;
#pragma unroll 1
    for (int c = 0; c < words; ++c) {
      const int i = c * 32 + lane;
      const float x = sh.x[i];
      if (i < nB && sel_key(x) >= cand) m += sel_weight<TOKEN>(g, by_mass, x, nmx, i);
    }
    if (warp_sum_ll(m) >= target) u = cand;
  }
  long long acc = 0;
#pragma unroll 1
  for (int c = 0; c < words; ++c) {
    const int i = c * 32 + lane;
    const float x = sh.x[i];
    if (i < nB && sel_key(x) > u) acc += sel_weight<TOKEN>(g, by_mass, x, nmx, i);
  }
  acc = warp_sum_ll(acc);
  int last = -1;
#pragma unroll 1
  for (int c = 0; c < words && acc < target; ++c) {
    const int i = c * 32 + lane;
    const bool tie = i < nB && sel_key(sh.x[i]) == u;
    uint32_t tb = __ballot_sync(0xffffffffu, tie);
    const long long w = tie ? sel_weight<TOKEN>(g, by_mass, sh.x[i], nmx, i) : 0ll;
    while (tb != 0u && acc < target) {
      const int l = __ffs(tb) - 1;
      tb &= tb - 1u;
      acc += __shfl_sync(0xffffffffu, w, l);
      last = c * 32 + l;
    }
  }
  xcut = key_value(u);
  icut = last;
}

// The cut for one target: the block of the order at which the running sum (mass, or block
// count) first reaches target.  The bucket histogram of that kind must be in sh.
template <bool TOKEN>
__device__ void sel_cut(const Geo& g, const SelSmem& sh, int words, int nB, bool by_mass, float nmx, float cb,
                        long long excl, long long own, long long target, int lane, float& xcut, int& icut) {
  long long base;
  const int b0 = hist_cross(sh, by_mass, lane, excl, own, target, base);
  // list the bucket's blocks, in index order (four words per step, loads first)
  int n = 0;
#pragma unroll 1
  for (int c0 = 0; c0 < words; c0 += 4) {
    float x[4];
    bool in[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = (c0 + u) * 32 + lane;
      x[u] = c0 + u < words ? sh.x[i] : -INFINITY;
      in[u] = c0 + u < words && i < nB && sel_bucket(x[u], cb) == b0;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t bal = __ballot_sync(0xffffffffu, in[u]);
      const int pos = n + __popc(bal & ((1u << lane) - 1u));
      if (in[u] && pos < kSelList) {
        sh.lx[pos] = x[u];
        sh.li[pos] = (c0 + u) * 32 + lane;
      }
      n += __popc(bal);
    }
  }
  __syncwarp();
  if (n > kSelList) {
    sel_search<TOKEN>(g, sh, words, nB, by_mass, nmx, target, lane, xcut, icut);
    return;
  }
  // candidates: listed blocks with key in [klo, khi]; base = the order's sum before them
  uint32_t klo = 0u, khi = 0xffffffffu;
#pragma unroll 1
  for (int level = 0;; ++level) {
    int cnt = 0;
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    for (int e = lane; e < n; e += 32) {
      const uint32_t k = sel_key(sh.lx[e]);
      if (k >= klo && k <= khi) {
        ++cnt;
        kmin = min(kmin, k);
        kmax = max(kmax, k);
      }
    }
    cnt = warp_sum_i(cnt);
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    if (cnt <= 32) {
      // the candidates into lanes (list order = index order), then rank them exactly
      float xj = 0.f;
      int ij = 0;
      long long wj = 0;
      int m = 0;
      for (int e0 = 0; e0 < n; e0 += 32) {
        const int e = e0 + lane;
        float x = 0.f;
        bool in = false;
        if (e < n) {
          x = sh.lx[e];
          const uint32_t k = sel_key(x);
          in = k >= klo && k <= khi;
        }
        const uint32_t bal = __ballot_sync(0xffffffffu, in);
        const int idx = e < n ? sh.li[e] : 0;
        // lane m + r takes the r-th candidate of this chunk
        uint32_t rest = bal;
        for (int r = 0; rest != 0u; ++r) {
          const int src = __ffs(rest) - 1;
          rest &= rest - 1u;
          const float xs = __shfl_sync(0xffffffffu, x, src);
          const int is = __shfl_sync(0xffffffffu, idx, src);
          if (lane == m + r) {
            xj = xs;
            ij = is;
          }
        }
        m += __popc(bal);
      }
      if (lane < cnt) wj = sel_weight<TOKEN>(g, by_mass, xj, nmx, ij);
      const int j = resolve32(cnt, xj, ij, wj, base, target, lane);
      xcut = __shfl_sync(0xffffffffu, xj, j);
      icut = __shfl_sync(0xffffffffu, ij, j);
      return;
    }
    if (kmin == kmax || level > 4) {       // more than 32 blocks of one logit
      sel_search<TOKEN>(g, sh, words, nB, by_mass, nmx, target, lane, xcut, icut);
      return;
    }
    // sub-buckets: the 9 key bits below the highest bit where the candidates differ,
    // counted down from kmax (sub-bucket 0 holds the highest keys)
    const int s = max(31 - __clz(kmin ^ kmax) - 8, 0);
    const uint32_t top = kmax >> s;
    hist_zero(sh, lane);
    for (int e = lane; e < n; e += 32) {
      const float x = sh.lx[e];
      const uint32_t k = sel_key(x);
      if (k >= klo && k <= khi) {
        const int sb = static_cast<int>(top - (k >> s));
        if (by_mass) {
          const MassParts mp = sel_mass<TOKEN>(g, x, nmx, sh.li[e]);
          atomicAdd(&sh.hh[sb], mp.hh);
          atomicAdd(&sh.hl[sb], mp.hl);
        } else {
          atomicAdd(&sh.hh[sb], 1);
        }
      }
    }
    __syncwarp();
    long long ex, ow, add;
    hist_scan(sh, by_mass, lane, ex, ow);
    const int sb = hist_cross(sh, by_mass, lane, ex, ow, target - base, add);
    base += add;
    klo = (top - static_cast<uint32_t>(sb)) << s;
    khi = s > 0 ? klo | ((1u << s) - 1u) : klo;
  }
}

template <bool TOKEN>
__device__ void select_row_hist(const Geo& g, const RouteOpts& o, const float* __restrict__ lrow, int nB,
                                int words, int qb, float p, int k_floor, uint32_t* mrow, int32_t* cnt_out,
                                int lane, const SelSmem& sh) {
  // 1. the row, past-the-end blocks as -inf, and its maximum
  float mx = -INFINITY;
  {
    const float4* src = reinterpret_cast<const float4*>(lrow);
    float4* dst = reinterpret_cast<float4*>(sh.x);
    const int n4 = words * 8;
#pragma unroll 4
    for (int q = lane; q < n4; q += 32) {
      float4 v = __ldg(src + q);
      const int i0 = 4 * q;
      if (i0 + 4 > nB) {
        if (i0 + 0 >= nB) v.x = -INFINITY;
        if (i0 + 1 >= nB) v.y = -INFINITY;
        if (i0 + 2 >= nB) v.z = -INFINITY;
        if (i0 + 3 >= nB) v.w = -INFINITY;
      }
      dst[q] = v;
      mx = fmaxf(mx, fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)));
    }
    mx = warp_max(mx);
    __syncwarp();
  }
  const float nmx = -mx;
  const float cb = __fadd_rn(__fmul_rn(mx, 32.f), 12582912.f);
  // 2. mass histogram, four blocks per step: the step's loads and exponentials overlap
  // (a load cannot pass the previous step's atomics)
  hist_zero(sh, lane);
#pragma unroll 1
  for (int c0 = 0; c0 < words; c0 += 4) {
    float x[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) x[u] = c0 + u < words ? sh.x[(c0 + u) * 32 + lane] : -INFINITY;
    MassParts m[4];
    int b[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      m[u] = sel_mass<TOKEN>(g, x[u], nmx, (c0 + u) * 32 + lane);
      b[u] = sel_bucket(x[u], cb);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (c0 + u < words) {
        atomicAdd(&sh.hh[b[u]], m[u].hh);
        atomicAdd(&sh.hl[b[u]], m[u].hl);
      }
    }
  }
  __syncwarp();
  bool all = p >= 1.f;
  float xcut = INFINITY;
  int icut = -1;
  if (!all) {
    long long excl, own;
    const long long z = hist_scan(sh, true, lane, excl, own);
    // at least one unit, so that p = 0 still keeps the first block of the order
    const long long target =
        max(1ll, static_cast<long long>(ceil(static_cast<double>(p) * static_cast<double>(z))));
    sel_cut<TOKEN>(g, sh, words, nB, true, nmx, cb, excl, own, target, lane, xcut, icut);
  }
  // 3. the mask; m_p = the blocks of the prefix rule
  auto write_mask = [&]() -> int {
    int mp = 0, cnt = 0;
#pragma unroll 1
    for (int c0 = 0; c0 < words; c0 += 4) {
      float x[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) x[u] = c0 + u < words ? sh.x[(c0 + u) * 32 + lane] : -INFINITY;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = c0 + u;
        if (c < words) {
          const int i = c * 32 + lane;
          const bool v = i < nB;
          const bool kp = v && (all || x[u] > xcut || (x[u] == xcut && i <= icut));
          mp += __popc(__ballot_sync(0xffffffffu, kp));
          const bool kept = kp || (v && (i == qb || keyframe_block(g, o, i)));
          const uint32_t word = __ballot_sync(0xffffffffu, kept);
          cnt += __popc(word);
          if (lane == 0) mrow[c] = word;
        }
      }
    }
    if (lane == 0) *cnt_out = cnt;
    return mp;
  };
  const int m_p = write_mask();
  if (all) return;
  const int floor_k = min(max(k_floor, 0), nB);
  const int M = max(max(m_p, floor_k), 1);
  if (M <= m_p) return;
  if (M >= nB) {
    all = true;
  } else {
    // the Top-k floor: the cut of the first M blocks, on counts
    hist_zero(sh, lane);
#pragma unroll 4
    for (int c = 0; c < words; ++c) {
      const int i = c * 32 + lane;
      if (i < nB) atomicAdd(&sh.hh[sel_bucket(sh.x[i], cb)], 1);
    }
    __syncwarp();
    long long excl, own;
    hist_scan(sh, false, lane, excl, own);
    sel_cut<TOKEN>(g, sh, words, nB, false, nmx, cb, excl, own, static_cast<long long>(M), lane, xcut, icut);
  }
  write_mask();
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
  static SmemAttrCache attr_ctx = {};
  cudaError_t e = set_smem_once(reinterpret_cast<const void*>(route_kernel<D, MAXW>), static_cast<int>(smem), attr_ctx);
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
template <bool TOKEN>
__global__ void __launch_bounds__(32 * kSelWarps) select_hist_kernel(Geo g, RouteOpts o,
                                                                     const float* __restrict__ logits, float p,
                                                                     int k_floor, uint32_t* __restrict__ mask,
                                                                     int32_t* __restrict__ counts) {
  extern __shared__ __align__(16) unsigned char sel_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nB = g.nB, nBpad = g.words * 32;
  const long long row = static_cast<long long>(blockIdx.x) * kSelWarps + warp;   // (b*h) * nB + qb
  if (row >= static_cast<long long>(g.B) * g.H * nB) return;
  const int qb = static_cast<int>(row % nB);
  const SelSmem sh = sel_smem_at(sel_smem + warp * sel_warp_bytes(g.words));
  select_row_hist<TOKEN>(g, o, logits + static_cast<size_t>(row) * nBpad, nB, g.words, qb, p, k_floor,
                         mask + static_cast<size_t>(row) * g.words, counts + row, lane, sh);
}

// For rows of at most kHistMinWords mask words the route is the fp32 pair: logits_kernel
// (64 x 64 block pairs per CTA, each thread 4 x 4 pairs in f32x2 FMA, in the per-logit
// operation order of route_kernel) and the bitwise selection below.  At those sizes the
// tensor-core path's split and fill cost more than its products save.
constexpr int kHistMinWords = 16;
constexpr int kLogitTile = 64;         // query x key blocks per CTA

template <int D>
__global__ void __launch_bounds__(256) logits_kernel(Geo g, const float* __restrict__ qp,
                                                     const float* __restrict__ kp, float scale,
                                                     float* __restrict__ logits) {
  constexpr int RS = D + 4;            // padded row (floats)
  extern __shared__ __align__(16) unsigned char lg_smem[];
  float* sQ = reinterpret_cast<float*>(lg_smem);   // [64][D + 4]
  float* sK = sQ + kLogitTile * RS;                // [64][D + 4]
  const int nB = g.nB, nBpad = g.words * 32;
  const int bhi = blockIdx.z;
  const int q0 = blockIdx.x * kLogitTile, k0 = blockIdx.y * kLogitTile;
  const float* qh = qp + static_cast<size_t>(bhi) * nB * D;
  const float* kh = kp + static_cast<size_t>(bhi) * nB * D;
  for (int e = threadIdx.x; e < kLogitTile * D / 4; e += 256) {
    const int r = e / (D / 4), d4 = e - r * (D / 4);
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    reinterpret_cast<float4*>(sQ + r * RS)[d4] =
        q0 + r < nB ? reinterpret_cast<const float4*>(qh + static_cast<size_t>(q0 + r) * D)[d4] : z;
    reinterpret_cast<float4*>(sK + r * RS)[d4] =
        k0 + r < nB ? reinterpret_cast<const float4*>(kh + static_cast<size_t>(k0 + r) * D)[d4] : z;
  }
  __syncthreads();
  // thread (ty, tx) takes query rows ty + 16 i and key blocks tx + 16 j, i, j < 4
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  uint64_t acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0ull;
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

// The selection of select_row (bitwise threshold search, one warp per row, the row's
// logits in registers), for rows of at most kHistMinWords mask words: there its fixed cost
// is below the histogram's (a 512-bucket scan and a gathered list per row).
template <int MAXW>
__global__ void __launch_bounds__(256) select_bitwise_kernel(Geo g, RouteOpts o, const float* __restrict__ logits,
                                                             float p, int k_floor, uint32_t* __restrict__ mask,
                                                             int32_t* __restrict__ counts) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nB = g.nB, nBpad = g.words * 32;
  const long long row = static_cast<long long>(blockIdx.x) * 8 + warp;   // (b*h) * nB + qb
  if (row >= static_cast<long long>(g.B) * g.H * nB) return;
  const int qb = static_cast<int>(row % nB);
  select_row<MAXW>(g, o, logits + static_cast<size_t>(row) * nBpad, nB, g.words, qb, p, k_floor,
                   mask + static_cast<size_t>(row) * g.words, counts + row, lane);
}



static cudaError_t launch_select(const Geo& g, const RouteOpts& o, const float* logits, float p, int k_floor,
                                 uint32_t* mask, int32_t* counts, cudaStream_t st) {
  const long long rows = static_cast<long long>(g.B) * g.H * g.nB;
  if (g.words <= kHistMinWords) {
    const unsigned grid = static_cast<unsigned>((rows + 7) / 8);
#define FV_SELECT(W) select_bitwise_kernel<W><<<grid, 256, 0, st>>>(g, o, logits, p, k_floor, mask, counts)
    if (g.words <= 4) FV_SELECT(4);
    else if (g.words <= 8) FV_SELECT(8);
    else if (g.words <= 12) FV_SELECT(12);
    else if (g.words <= 16) FV_SELECT(16);
    else if (g.words <= 20) FV_SELECT(20);
    else if (g.words <= 24) FV_SELECT(24);
    else if (g.words <= 32) FV_SELECT(32);
    else if (g.words <= 48) FV_SELECT(48);
    else FV_SELECT(64);
#undef FV_SELECT
    return cudaGetLastError();
  }
  const int smem = static_cast<int>(kSelWarps * sel_warp_bytes(g.words));
  static SmemAttrCache sel_attr[2] = {};
  const void* fn = o.token_mass ? reinterpret_cast<const void*>(select_hist_kernel<true>)
                                : reinterpret_cast<const void*>(select_hist_kernel<false>);
  // the largest carveout (all of the unified L1 / shared array as shared memory): four
  // CTAs (16 rows) per SM fit at the longest rows (2 048 blocks) only with it
  cudaError_t e = set_smem_once(fn, smem, sel_attr[o.token_mass ? 1 : 0], 100);
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>((rows + kSelWarps - 1) / kSelWarps);
  if (o.token_mass)
    select_hist_kernel<true><<<grid, 32 * kSelWarps, smem, st>>>(g, o, logits, p, k_floor, mask, counts);
  else
    select_hist_kernel<false><<<grid, 32 * kSelWarps, smem, st>>>(g, o, logits, p, k_floor, mask, counts);
  return cudaGetLastError();
}

// Route workspace: a 256-byte header (word 1: error bits of the logits kernel's bounded
// waits), then the logits, [B*H][nB][words * 32] fp32 ...
constexpr size_t kRouteHdr = 256;

size_t route_logits_bytes(const Geo& g) {
  return static_cast<size_t>(g.B) * g.H * g.nB * (static_cast<size_t>(g.words) * 32) * 4;
}

// ... followed by the pooled rows split into tf32 high and low parts (4 planes of
// B*H*nB*d floats) for the tensor-core logits.
size_t route_ws_bytes(const Geo& g) { return kRouteHdr + route_logits_bytes(g) + logits_split_bytes(g); }

static cudaError_t num_sms(int& nsm) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  return cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
}

// Logits of geometry g into `logits` (its rows padded to words * 32), then the selection.
// split: the tensor-core path's scratch (logits_split_bytes(g)); err: its status word.
static cudaError_t route_parts(const Geo& g, const float* qp, const float* kp, float p, int k_floor, float scale,
                               uint32_t* mask, int32_t* counts, float* logits, float* split, uint32_t* err,
                               int nsm, cudaStream_t st, const RouteOpts& o) {
  cudaError_t e;
  if (g.words <= kHistMinWords) {
    const int tiles = (g.nB + kLogitTile - 1) / kLogitTile;
    const int smem = 2 * kLogitTile * (g.d + 4) * 4;
    static SmemAttrCache lg_attr = {};
    const void* fn = g.d == 128 ? reinterpret_cast<const void*>(logits_kernel<128>)
                                : reinterpret_cast<const void*>(logits_kernel<64>);
    e = set_smem_once(fn, smem, lg_attr);
    if (e != cudaSuccess) return e;
    const dim3 grid(tiles, tiles, g.B * g.H);
    if (g.d == 128) logits_kernel<128><<<grid, 256, smem, st>>>(g, qp, kp, scale, logits);
    else logits_kernel<64><<<grid, 256, smem, st>>>(g, qp, kp, scale, logits);
  } else {
    e = launch_logits_tc(g, qp, kp, scale, logits, split, err, nsm, st);
  }
  if (e != cudaSuccess) return e;
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_select(g, o, logits, p, k_floor, mask, counts, st);
}

cudaError_t launch_route_ws(const Geo& g, const float* qp, const float* kp, float p, int k_floor,
                            float scale, uint32_t* mask, int32_t* counts, void* ws, cudaStream_t st,
                            const RouteOpts& o) {
  uint32_t* hdr = static_cast<uint32_t*>(ws);
  float* logits = reinterpret_cast<float*>(static_cast<unsigned char*>(ws) + kRouteHdr);
  float* split = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(logits) + route_logits_bytes(g));
  cudaError_t e = cudaMemsetAsync(hdr, 0, kRouteHdr, st);
  if (e != cudaSuccess) return e;
  int nsm = 0;
  e = num_sms(nsm);
  if (e != cudaSuccess) return e;
  return route_parts(g, qp, kp, p, k_floor, scale, mask, counts, logits, split, hdr + 1, nsm, st, o);
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
