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
// block's mass 2^((l - max) log2 e) (times its real token count for the Top-p over tokens) is
// rounded once to a fixed-point integer of 2^-32 units, and all sums are integer sums, so
// they do not depend on summation order and the prefix test "mass >= p" reads
// sum >= ceil(p * Z) in integers.  Per row (one warp):
//   1. logits into registers (lane l holds blocks c * 32 + l) as order keys, row maximum;
//   2. a 512-bucket histogram of mass and count in shared memory over t = (max - l) * 32:
//      bucket floor(t), the last one holding everything 16 or more below the max (its
//      sums are kept in registers: the blocks of a sparse row pile up there);
//   3. a warp scan over the buckets finds the bucket where the prefix mass reaches p;
//   4. when that bucket holds more than 32 blocks, a second histogram over its fraction
//      of t (512 sub-buckets) narrows it;
//   5. the bucket's blocks are gathered and ranked exactly by (logit desc, index asc); the
//      cut is the first rank at which the prefix reaches p;
//   6. the Top-k floor, when it lengthens the prefix, repeats 2-5 on counts;
//   7. the mask: blocks above the cut's key, tied blocks up to the cut's index, the own
//      block and keyframe blocks.
// A sub-bucket with more than 32 blocks (near-ties by the dozen) runs select_row.
// ----------------------------------------------------------------------------
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

constexpr int kSelBuckets = 512;
constexpr float kSelPerLogit = 32.f;
constexpr int kSelCap = 32;             // gathered blocks: one per lane
constexpr int kSelWarps = 4;            // rows (warps) per CTA

// Shared memory of one warp (one row at a time): the mass histogram, the gathered list and
// the row's order keys, lane l's keys in column l ([c][32], so a lane touches only its own
// words and no synchronisation is needed for them).
struct SelScratch {
  uint32_t* hh;                          // mass per bucket (2^-32 units): high parts (w >> 20) ...
  uint32_t* hl;                          //   ... and low parts (w & 0xfffff), both exact in 32 bits
  uint32_t* hc;                          // blocks per bucket
  unsigned long long* lw;                // gathered bucket: mass,
  uint32_t* lkey;                        //   order key,
  uint32_t* lidx;                        //   block index
  uint32_t* key;                         // the row: key[c * 32 + lane] for block c * 32 + lane
};

__host__ __device__ constexpr size_t sel_warp_bytes(int words) {
  return 3 * kSelBuckets * 4 + kSelCap * 8 + 2 * kSelCap * 4 + static_cast<size_t>(words) * 32 * 4;
}

__device__ __forceinline__ SelScratch sel_scratch(unsigned char* base) {
  SelScratch sh;
  sh.hh = reinterpret_cast<uint32_t*>(base);
  sh.hl = sh.hh + kSelBuckets;
  sh.hc = sh.hl + kSelBuckets;
  sh.lw = reinterpret_cast<unsigned long long*>(sh.hc + kSelBuckets);
  sh.lkey = reinterpret_cast<uint32_t*>(sh.lw + kSelCap);
  sh.lidx = sh.lkey + kSelCap;
  sh.key = sh.lidx + kSelCap;
  return sh;
}

__device__ __forceinline__ float key_value(uint32_t k) {   // inverse of order_key
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

__device__ __forceinline__ unsigned long long warp_sum_u64(unsigned long long v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

__device__ __forceinline__ unsigned long long sel_fixed(float w) {
  return __float2ull_rn(w * 4294967296.0f);
}

// Bucket coordinate of a logit: t = (max - x) * 32; level-0 bucket floor(t) (capped), and
// inside level-0 bucket b0 the level-1 bucket floor((t - b0) * 512) (exact in fp32: t < 512
// carries at most 14 fraction bits, so t - b0 and the scaling round nothing).
__device__ __forceinline__ float sel_t(float mx, float x) { return (mx - x) * kSelPerLogit; }
__device__ __forceinline__ int sel_b0(float t) { return min(kSelBuckets - 1, __float2int_rz(t)); }
__device__ __forceinline__ int sel_b1(float t, int b0) {
  return min(kSelBuckets - 1, __float2int_rz((t - static_cast<float>(b0)) * static_cast<float>(kSelBuckets)));
}

__device__ __forceinline__ unsigned long long sel_bucket_mass(const SelScratch& sh, int b) {
  return (static_cast<unsigned long long>(sh.hh[b]) << 20) + sh.hl[b];
}

// Finds the bucket where the running sum (mass when `by_mass`, else count) first reaches
// `target`, scanning buckets from the top of the order.  Lane l owns buckets 16 l .. 16 l + 15.
// Returns the bucket; `above` / `cnt_above` get the sum and block count before it.
__device__ __forceinline__ int sel_find_bucket(const SelScratch& sh, bool by_mass, unsigned long long target,
                                               unsigned long long& above, int& cnt_above, int lane) {
  constexpr int PER = kSelBuckets / 32;
  unsigned long long run = 0;
  int crun = 0;
#pragma unroll 4
  for (int e = 0; e < PER; ++e) {
    const int b = lane * PER + e;
    const uint32_t n = sh.hc[b];
    run += by_mass ? sel_bucket_mass(sh, b) : static_cast<unsigned long long>(n);
    crun += static_cast<int>(n);
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
  if (incl >= target && excl < target) {      // the crossing lies in this lane's buckets
#pragma unroll 1
    for (int e = 0; e < PER; ++e) {
      const int b = lane * PER + e;
      const uint32_t n = sh.hc[b];
      const unsigned long long v = by_mass ? sel_bucket_mass(sh, b) : static_cast<unsigned long long>(n);
      if (excl + v >= target) {
        found = b;
        f_above = excl;
        f_cnt = cexcl;
        break;
      }
      excl += v;
      cexcl += static_cast<int>(n);
    }
  }
  const uint32_t hit = __ballot_sync(0xffffffffu, found < kSelBuckets);
  const int src = hit ? __ffs(hit) - 1 : 31;
  above = __shfl_sync(0xffffffffu, f_above, src);
  cnt_above = __shfl_sync(0xffffffffu, f_cnt, src);
  return hit ? __shfl_sync(0xffffffffu, found, src) : kSelBuckets - 1;
}

__device__ void select_row_hist(const Geo& g, const RouteOpts& o, const float* lrow, int nB, int words, int qb,
                                float p, int k_floor, uint32_t* mrow, int32_t* cnt_out, int lane,
                                const SelScratch& sh) {
  // the row's words * 32 logits into shared memory in one round trip (16-byte cp.async,
  // all in flight), then each lane turns its column into order keys
  {
    const uint32_t dst = smem_u32(sh.key);
    const int chunks = words * 8;            // 16-byte chunks of the row
    for (int q = lane; q < chunks; q += 32) cp_async16(dst + q * 16, lrow + q * 4, 16u);
    cp_async_commit();
    cp_async_wait<0>();
    __syncwarp();
  }
  uint32_t* key = sh.key + lane;   // this lane's column: key[c * 32]
  float mx = -INFINITY;
#pragma unroll 4
  for (int c = 0; c < words; ++c) {
    const int i = c * 32 + lane;
    const float x = i < nB ? __uint_as_float(key[c * 32]) : -INFINITY;
    key[c * 32] = i < nB ? order_key(x) : 0u;
    mx = fmaxf(mx, x);
  }
  mx = warp_max(mx);
  const float nmx = -mx;
  // a block's mass in 2^-32 units: 2^((x - max) log2 e), times its real token count for
  // the Top-p over tokens; the same rounded operations wherever it is evaluated
  auto mass_of = [&](int c, float x) -> unsigned long long {
    float w = ex2(__fmul_rn(__fadd_rn(x, nmx), 1.4426950408889634f));
    if (o.token_mass) w *= static_cast<float>(block_info(g, c * 32 + lane).nvalid);
    return sel_fixed(w);
  };
  // Histogram of the blocks of level-0 bucket in0 (all blocks when in0 < 0): 32-bit
  // shared-memory atomics per block (a mass w < 2^40 goes in as w >> 20 and w & 0xfffff,
  // so over at most 2^11 blocks the sums stay below 2^31), except for the last bucket
  // (the tail, where the blocks of a sparse row pile up), which each lane sums in
  // registers and one lane stores.  Returns the row's (or bucket's) mass.
  auto histogram = [&](int in0) -> unsigned long long {
#pragma unroll 4
    for (int e = lane; e < kSelBuckets; e += 32) {
      sh.hh[e] = 0u;
      sh.hl[e] = 0u;
      sh.hc[e] = 0u;
    }
    __syncwarp();
    unsigned long long z = 0, tail_w = 0;
    uint32_t tail_c = 0;
#pragma unroll 2
    for (int c = 0; c < words; ++c) {
      const uint32_t k = key[c * 32];
      if (k != 0u) {
        const float x = key_value(k);
        const float t = sel_t(mx, x);
        const int b0 = sel_b0(t);
        const int b = in0 < 0 ? b0 : (b0 == in0 ? sel_b1(t, b0) : -1);
        if (b >= 0) {
          const unsigned long long w = mass_of(c, x);
          z += w;
          if (b == kSelBuckets - 1) {
            tail_w += w;
            ++tail_c;
          } else {
            atomicAdd(&sh.hh[b], static_cast<uint32_t>(w >> 20));
            atomicAdd(&sh.hl[b], static_cast<uint32_t>(w & 0xfffffu));
            atomicAdd(&sh.hc[b], 1u);
          }
        }
      }
    }
    tail_w = warp_sum_u64(tail_w);
    tail_c = static_cast<uint32_t>(warp_sum_i(static_cast<int>(tail_c)));
    __syncwarp();
    if (lane == 0) {
      sh.hh[kSelBuckets - 1] = static_cast<uint32_t>(tail_w >> 20);
      sh.hl[kSelBuckets - 1] = static_cast<uint32_t>(tail_w & 0xfffffu);
      sh.hc[kSelBuckets - 1] = tail_c;
    }
    __syncwarp();
    return warp_sum_u64(z);
  };
  // Gathers the n <= 32 blocks of level-0 bucket b0 (and level-1 bucket b1 >= 0).
  auto gather = [&](int b0, int b1) {
    int base = 0;
#pragma unroll 2
    for (int c = 0; c < words; ++c) {
      const uint32_t k = key[c * 32];
      bool in = false;
      float x = 0.f;
      if (k != 0u) {
        x = key_value(k);
        const float t = sel_t(mx, x);
        const int c0 = sel_b0(t);
        in = c0 == b0 && (b1 < 0 || sel_b1(t, c0) == b1);
      }
      const uint32_t bal = __ballot_sync(0xffffffffu, in);
      if (in) {
        const int pos = base + __popc(bal & ((1u << lane) - 1u));
        sh.lkey[pos] = k;
        sh.lidx[pos] = static_cast<uint32_t>(c * 32 + lane);
        sh.lw[pos] = mass_of(c, x);
      }
      base += __popc(bal);
    }
    __syncwarp();
  };
  // Among the n <= 32 gathered blocks (lane j holds block j), the one of smallest rank
  // (key desc, index asc) at which above + (running sum of weights up to it) >= target;
  // weight = mass or 1.
  auto resolve = [&](int n, bool by_mass, unsigned long long above, unsigned long long target, int& rank_out,
                     uint32_t& key_out, int& idx_out) {
    int best = 0x7fffffff;
    if (lane < n) {
      const uint32_t kj = sh.lkey[lane], ij = sh.lidx[lane];
      int rank = 0;
      unsigned long long pre = 0;
      for (int t = 0; t < n; ++t) {
        const uint32_t kt = sh.lkey[t], it = sh.lidx[t];
        const bool before = kt > kj || (kt == kj && it <= ij);
        rank += (before && t != lane) ? 1 : 0;
        pre += before ? (by_mass ? sh.lw[t] : 1ull) : 0ull;
      }
      // a block whose prefix reaches the target codes as its rank; the others code above
      // every such rank, the last in the order lowest (the whole bucket)
      best = above + pre >= target ? rank * 64 + lane : (2 * n - 1 - rank) * 64 + lane;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) best = min(best, __shfl_xor_sync(0xffffffffu, best, off));
    const int j = best & 63;
    rank_out = best >> 6;
    key_out = sh.lkey[j];
    idx_out = static_cast<int>(sh.lidx[j]);
    __syncwarp();
  };
  // Exact fallback for a bucket of more than 32 near-tied blocks: a bitwise search for the
  // cut's key over the whole row (u = the largest key whose prefix of keys >= u reaches the
  // target), then tied keys in index order.
  auto search = [&](bool by_mass, unsigned long long target, int& m_out, uint32_t& ucut, int& icut) {
    uint32_t u = 0;
#pragma unroll 1
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = u | (1u << bit);
      unsigned long long m = 0;
#pragma unroll 1
      for (int c = 0; c < words; ++c) {
        const uint32_t k = key[c * 32];
        if (k != 0u && k >= cand) m += by_mass ? mass_of(c, key_value(k)) : 1ull;
      }
      if (warp_sum_u64(m) >= target) u = cand;
    }
    unsigned long long acc = 0;
    int gt = 0;
#pragma unroll 1
    for (int c = 0; c < words; ++c) {
      const uint32_t k = key[c * 32];
      if (k != 0u && k > u) {
        acc += by_mass ? mass_of(c, key_value(k)) : 1ull;
        ++gt;
      }
    }
    acc = warp_sum_u64(acc);
    gt = warp_sum_i(gt);
    int r = 0, last = -1;
#pragma unroll 1
    for (int c = 0; c < words && acc < target; ++c) {
      const uint32_t k = key[c * 32];
      uint32_t tb = __ballot_sync(0xffffffffu, k != 0u && k == u);
      while (tb != 0u && acc < target) {
        const int l = __ffs(tb) - 1;
        tb &= tb - 1u;
        const unsigned long long w = by_mass ? mass_of(c, key_value(u)) : 1ull;
        acc += __shfl_sync(0xffffffffu, w, l);
        ++r;
        last = c * 32 + l;
      }
    }
    m_out = gt + r;
    ucut = u;
    icut = last;
  };
  // The cut: the block of the order at which the running sum reaches target (the level-0
  // histogram is in place).
  auto cut = [&](bool by_mass, unsigned long long target, int& m_out, uint32_t& ucut, int& icut) {
    unsigned long long above;
    int cnt_above;
    const int b0 = sel_find_bucket(sh, by_mass, target, above, cnt_above, lane);
    int b1 = -1;
    int n = static_cast<int>(sh.hc[b0]);
    if (n > kSelCap) {
      histogram(b0);
      unsigned long long above1;
      int cnt1;
      b1 = sel_find_bucket(sh, by_mass, target - above, above1, cnt1, lane);
      above += above1;
      cnt_above += cnt1;
      n = static_cast<int>(sh.hc[b1]);
      if (n > kSelCap) {
        search(by_mass, target, m_out, ucut, icut);
        return;
      }
    }
    gather(b0, b1);
    int rank;
    resolve(n, by_mass, above, target, rank, ucut, icut);
    m_out = cnt_above + rank + 1;
  };

  const unsigned long long z = histogram(-1);
  const int floor_k = min(max(k_floor, 0), nB);
  int m_p = nB;
  uint32_t ucut = 0u;        // blocks with key > ucut, and key == ucut up to index icut, are kept
  int icut = -1;
  bool all = true;
  if (p < 1.f) {
    // at least one unit, so that p = 0 still keeps the first block of the order
    const unsigned long long target =
        max(1ull, static_cast<unsigned long long>(ceil(static_cast<double>(p) * static_cast<double>(z))));
    cut(true, target, m_p, ucut, icut);
    all = false;
  }
  const int M = max(max(m_p, floor_k), 1);
  if (M >= nB) {
    all = true;
  } else if (M > m_p) {
    histogram(-1);           // the cut may have left a finer histogram in place
    int m;
    cut(false, static_cast<unsigned long long>(M), m, ucut, icut);
    all = false;
  }
  int cnt = 0;
#pragma unroll 2
  for (int c = 0; c < words; ++c) {
    const int i = c * 32 + lane;
    const uint32_t k = key[c * 32];
    const bool kept = k != 0u && (all || k > ucut || (k == ucut && i <= icut) || i == qb ||
                                  keyframe_block(g, o, i));
    const uint32_t word = __ballot_sync(0xffffffffu, kept);
    cnt += __popc(word);
    if (lane == 0) mrow[c] = word;
  }
  if (lane == 0) *cnt_out = cnt;
}

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
  const SelScratch sh = sel_scratch(sel_smem + warp * sel_warp_bytes(g.words));
  select_row_hist(g, o, logits + static_cast<size_t>(row) * nBpad, nB, g.words, qb, p, k_floor,
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
  static SmemAttrCache sel_attr = {};
  cudaError_t e = set_smem_once(reinterpret_cast<const void*>(select_hist_kernel), smem, sel_attr);
  if (e != cudaSuccess) return e;
  select_hist_kernel<<<static_cast<unsigned>((rows + kSelWarps - 1) / kSelWarps), 32 * kSelWarps, smem, st>>>(
      g, o, logits, p, k_floor, mask, counts);
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

cudaError_t launch_route_ws(const Geo& g, const float* qp, const float* kp, float p, int k_floor,
                            float scale, uint32_t* mask, int32_t* counts, void* ws, cudaStream_t st,
                            const RouteOpts& o) {
  uint32_t* hdr = static_cast<uint32_t*>(ws);
  float* logits = reinterpret_cast<float*>(static_cast<unsigned char*>(ws) + kRouteHdr);
  cudaError_t e = cudaMemsetAsync(hdr, 0, kRouteHdr, st);
  if (e != cudaSuccess) return e;
  int dev = 0, nsm = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
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
    float* split = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(logits) + route_logits_bytes(g));
    e = launch_logits_tc(g, qp, kp, scale, logits, split, hdr + 1, nsm, st);
  }
  if (e != cudaSuccess) return e;
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_select(g, o, logits, p, k_floor, mask, counts, st);
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
