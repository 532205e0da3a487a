// Routing logits on the 5th-generation tensor cores with fp32-grade accuracy.
//
// FVAttn explainer (arXiv 2607.16190), 核心方法 §1: each head routes per query block
// over the similarity of pooled query and key blocks, l[i][j] = (Qp[i] . Kp[j]) * scale.
// Per (b, h) slice that is one nB x nB x d product: 0.35 GFLOP at 21x30x52 with 1x8x16
// blocks and 12 heads, 11.5 GFLOP at 121x30x52, which the fp32 FMA pipes cannot stream
// at HBM speed.  Here it runs as tcgen05 kind::tf32 MMAs.  A tf32 operand keeps 10
// mantissa bits, so each fp32 operand x is split as x = hi + lo with hi = tf32(x) and
// lo = tf32(x - hi), and the product takes three terms,
//   a . b ~= a_hi . b_hi + a_hi . b_lo + a_lo . b_hi,
// the split-precision method of Ootomo and Yokota ("Recovering single precision accuracy
// from Tensor Cores while surpassing the FP32 theoretical peak performance", 2022):
// the dropped terms are below 2^-21 of |a||b| per product.
//
// split_kernel writes the hi and lo parts of every pooled row once, into the route
// workspace.  Then one CTA per work unit = (slice, 128 query blocks, a range of
// 128-key-block tiles):
//   warp 0     loads the query tile's hi and lo parts, then the key tiles' 32 channels at a
//              time through a ring of stages, with TMA in the 128-byte-swizzled K-major
//              layout the MMA descriptors read;
//   warp 1     issues the MMAs (one elected lane) into one of two 128-column fp32
//              accumulators in tensor memory;
//   warps 2-5  read an accumulator (one TMEM lane = one query row per thread), scale it
//              and store the row's 128 logits, while the other accumulator fills.
// Every wait is bounded; a stuck pipeline raises the workspace's error word and the
// kernel drains and returns (fv::mbar_wait).
#include "fv_common.cuh"
#include "fv_launch.h"

namespace fv {

constexpr int kLgThreads = 192;           // 6 warps
constexpr int kLgChunk = 128 * 128;       // bytes: 128 rows x 32 fp32 (one swizzle column)
constexpr int kLgTile = 128;              // query / key blocks per tile

template <int D> __host__ __device__ constexpr int lg_stages() { return D == 128 ? 2 : 4; }
constexpr int kLgXpose = 4 * 32 * 33 * 4;   // bytes: a 32 x 33 fp32 transpose buffer per epilogue warp

struct __align__(8) LgBars {
  uint64_t a_full, a_empty;
  uint64_t st_full[4], st_empty[4];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t fin;
  uint32_t tmem_base;
  int abort;
};

template <int D>
__host__ __device__ constexpr int lg_smem_bytes() {
  return 2 * (D / 32) * kLgChunk + lg_stages<D>() * 2 * kLgChunk + kLgXpose + static_cast<int>(sizeof(LgBars));
}
static_assert(lg_smem_bytes<128>() <= 232448, "logits kernel exceeds 227 KB of shared memory");
static_assert(lg_smem_bytes<64>() <= 232448, "logits kernel exceeds 227 KB of shared memory");

struct LgParams {
  Geo g;
  float* logits;      // [B*H][nB][words*32]
  float scale;
  uint32_t* err;      // error word of the route workspace
  int tiles;          // 128-block tiles per slice side
  int ksplit, kper;   // key-tile ranges per (slice, query tile), key tiles per range
  long long items;    // (slice, query tile, key range) items, in that order
};

struct LgMaps {
  CUtensorMap qh, ql, kh, kl;   // the split pooled rows, [B*H][nB][d] fp32 each
};

// x = hi + lo with hi = tf32(x), lo = tf32(x - hi), both rounded to nearest; stored as the
// fp32 bit patterns the kind::tf32 MMA reads.
template <int D>
__global__ void __launch_bounds__(256) split_kernel(const float4* __restrict__ qp, const float4* __restrict__ kp,
                                                    float4* __restrict__ split, long long n4) {
  const long long i = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x;
  if (i >= n4) return;
#pragma unroll
  for (int src = 0; src < 2; ++src) {
    const float4 x = __ldg((src ? kp : qp) + i);
    const float4 h = make_float4(to_tf32(x.x), to_tf32(x.y), to_tf32(x.z), to_tf32(x.w));
    const float4 l = make_float4(to_tf32(x.x - h.x), to_tf32(x.y - h.y), to_tf32(x.z - h.z), to_tf32(x.w - h.w));
    split[(2 * src) * n4 + i] = h;
    split[(2 * src + 1) * n4 + i] = l;
  }
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* m, uint64_t* bar, int c0, int c1,
                                            int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// Item w -> slice, query tile, key tiles [kt0, kt1).
struct LgItem {
  int bhi, qt, kt0, kt1;
};
__device__ __forceinline__ LgItem lg_item(long long w, const LgParams& p) {
  const long long per_slice = static_cast<long long>(p.tiles) * p.ksplit;
  LgItem r;
  r.bhi = static_cast<int>(w / per_slice);
  const int rem = static_cast<int>(w - r.bhi * per_slice);
  r.qt = rem / p.ksplit;
  const int ks = rem - r.qt * p.ksplit;
  r.kt0 = ks * p.kper;
  r.kt1 = min(p.tiles, r.kt0 + p.kper);
  return r;
}

// Persistent: CTA i takes items i, i + P, i + 2P, ...  The items in flight at any moment
// are consecutive, so the CTAs on one slice sweep the same key tiles at about the same
// time: a key tile comes from DRAM once and from L2 for the slice's other query tiles.  A
// CTA loads its query tile once per item.
template <int D>
__global__ void __launch_bounds__(kLgThreads, 1)
    logits_tc_kernel(const __grid_constant__ CUtensorMap tmQh, const __grid_constant__ CUtensorMap tmQl,
                     const __grid_constant__ CUtensorMap tmKh, const __grid_constant__ CUtensorMap tmKl,
                     const LgParams prm) {
  constexpr int NC = D / 32;                // 32-channel chunks per row
  constexpr int S = lg_stages<D>();
  extern __shared__ __align__(1024) unsigned char lg_dsm[];
  float* xpose = reinterpret_cast<float*>(lg_dsm + 2 * NC * kLgChunk + S * 2 * kLgChunk);
  LgBars& bars = *reinterpret_cast<LgBars*>(lg_dsm + 2 * NC * kLgChunk + S * 2 * kLgChunk + kLgXpose);
  const Geo& g = prm.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort = &bars.abort;
  uint32_t* err = prm.err;

  const uint32_t base = smem_u32(lg_dsm);
  if (base & 1023u) {                       // uniform: nothing issued yet
    if (threadIdx.x == 0) atomicOr(err, kErrLayout);
    return;
  }
  const uint32_t sAhi = base, sAlo = base + NC * kLgChunk;
  auto sBhi = [&](int s) { return base + static_cast<uint32_t>(2 * NC * kLgChunk + s * 2 * kLgChunk); };
  auto sBlo = [&](int s) { return sBhi(s) + static_cast<uint32_t>(kLgChunk); };

  const int nB = g.nB, nBpad = g.words * 32;

  if (threadIdx.x == 0) {
    mbar_init(&bars.a_full, 1);
    mbar_init(&bars.a_empty, 1);
    for (int i = 0; i < S; ++i) { mbar_init(&bars.st_full[i], 1); mbar_init(&bars.st_empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&bars.acc_full[i], 1); mbar_init(&bars.acc_empty[i], 4); }
    mbar_init(&bars.fin, 1);
    bars.abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars.tmem_base, 256);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQh); tma_prefetch_desc(&tmQl);
    tma_prefetch_desc(&tmKh); tma_prefetch_desc(&tmKl);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;
  uint32_t loads = 0, aloads = 0;           // B chunks / query tiles whose copies were issued

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (lane 0)
    if (lane == 0) {
      uint32_t i = 0;
      bool ok = true;
#pragma unroll 1
      for (long long w = blockIdx.x; w < prm.items && ok; w += gridDim.x) {
        const LgItem t = lg_item(w, prm);
        // the previous query tile's MMAs have finished reading it
        if (aloads > 0 && !mbar_wait(&bars.a_empty, (aloads - 1) & 1, abort, err)) break;
        mbar_arrive_expect_tx(&bars.a_full, static_cast<uint32_t>(2 * NC * kLgChunk));
#pragma unroll 1
        for (int c = 0; c < NC; ++c) {
          tma_load_3d(sAhi + c * kLgChunk, &tmQh, &bars.a_full, c * 32, t.qt * kLgTile, t.bhi);
          tma_load_3d(sAlo + c * kLgChunk, &tmQl, &bars.a_full, c * 32, t.qt * kLgTile, t.bhi);
        }
        ++aloads;
#pragma unroll 1
        for (int kt = t.kt0; kt < t.kt1 && ok; ++kt) {
#pragma unroll 1
          for (int c = 0; c < NC; ++c, ++i) {
            const int s = i % S;
            if (!mbar_wait(&bars.st_empty[s], ((i / S) & 1) ^ 1, abort, err)) { ok = false; break; }
            mbar_arrive_expect_tx(&bars.st_full[s], static_cast<uint32_t>(2 * kLgChunk));
            tma_load_3d(sBhi(s), &tmKh, &bars.st_full[s], c * 32, kt * kLgTile, t.bhi);
            tma_load_3d(sBlo(s), &tmKl, &bars.st_full[s], c * 32, kt * kLgTile, t.bhi);
            loads = i + 1;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    const uint32_t idesc = idesc_tf32_f32(128, 128);
    auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, err));
    };
    uint32_t i = 0, na = 0;
    bool ok = true;
    int j = 0;
#pragma unroll 1
    for (long long w = blockIdx.x; w < prm.items && ok; w += gridDim.x) {
      const LgItem t = lg_item(w, prm);
      if (!wwait(&bars.a_full, na & 1)) break;
      ++na;
#pragma unroll 1
    for (int kt = t.kt0; kt < t.kt1 && ok; ++kt, ++j) {
      const int slot = j & 1;
      if (!wwait(&bars.acc_empty[slot], ((j >> 1) & 1) ^ 1)) { ok = false; break; }
      const uint32_t tacc = tmem + static_cast<uint32_t>(slot * 128);
      const bool last_of_a = kt + 1 == t.kt1;
#pragma unroll 1
      for (int c = 0; c < NC; ++c, ++i) {
        const int s = i % S;
        if (!wwait(&bars.st_full[s], (i / S) & 1)) { ok = false; break; }
        tc_fence_after();
        if (elect_one()) {
          const uint64_t dAh = sdesc_sw128(sAhi + c * kLgChunk, 16, 1024);
          const uint64_t dAl = sdesc_sw128(sAlo + c * kLgChunk, 16, 1024);
          const uint64_t dBh = sdesc_sw128(sBhi(s), 16, 1024);
          const uint64_t dBl = sdesc_sw128(sBlo(s), 16, 1024);
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {          // 8 channels (32 bytes) per MMA
            const uint64_t o = static_cast<uint64_t>(2 * k4);
            mma_ss_tf32(tacc, dAl + o, dBh + o, idesc, (c | k4) ? 1u : 0u);
            mma_ss_tf32(tacc, dAh + o, dBl + o, idesc, 1u);
            mma_ss_tf32(tacc, dAh + o, dBh + o, idesc, 1u);
          }
          mma_commit(&bars.st_empty[s]);
          if (c == NC - 1) {
            mma_commit(&bars.acc_full[slot]);
            if (last_of_a) mma_commit(&bars.a_empty);
          }
        }
        __syncwarp();
      }
    }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2-5)
    // Each 32 x 32 block of the accumulator (this warp's 32 rows, 32 key columns) goes
    // through a padded shared buffer: thread r writes its row, then the warp stores row by
    // row, 32 consecutive logits (128 bytes) per instruction.
    const int quarter = warp & 3;
    float* xb = xpose + (warp - 2) * 32 * 33;
    const float sc = prm.scale;
    int j = 0;
    bool ok = true;
#pragma unroll 1
    for (long long w = blockIdx.x; w < prm.items && ok; w += gridDim.x) {
      const LgItem t = lg_item(w, prm);
#pragma unroll 1
    for (int kt = t.kt0; kt < t.kt1; ++kt, ++j) {
      const int slot = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&bars.acc_full[slot], (j >> 1) & 1, abort, err))) { ok = false; break; }
      tc_fence_after();
      const int row0 = t.qt * kLgTile + quarter * 32;
      const int nrows = min(32, nB - row0);
#pragma unroll 1
      for (int g4 = 0; g4 < 4; ++g4) {
        uint32_t v[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(slot * 128 + 32 * g4), v);
        tmem_wait_ld();
        const int col = kt * kLgTile + 32 * g4;
        if (col < nBpad) {                          // uniform over the warp
#pragma unroll
          for (int e = 0; e < 32; ++e) xb[lane * 33 + e] = __uint_as_float(v[e]) * sc;
          __syncwarp();
#pragma unroll 4
          for (int r = 0; r < nrows; ++r)
            prm.logits[(static_cast<size_t>(t.bhi) * nB + row0 + r) * nBpad + col + lane] = xb[r * 33 + lane];
          __syncwarp();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.acc_empty[slot]);
    }
    }
  }

  // ------------------------------------------------------------ teardown
  __syncthreads();
  if (bars.abort) {
    // let every armed copy land and every issued MMA finish before shared and tensor
    // memory are released (bounded, the abort flag ignored)
    int never = 0;
    volatile int* nv = &never;
    if (warp == 0 && lane == 0) {
      if (aloads > 0) mbar_wait(&bars.a_full, (aloads - 1) & 1, nv, nullptr, 100000000ull);
      for (uint32_t i = (loads > static_cast<uint32_t>(S) ? loads - S : 0); i < loads; ++i)
        mbar_wait(&bars.st_full[i % S], (i / S) & 1, nv, nullptr, 100000000ull);
    }
    if (warp == 1 && lane == 0) {
      mma_commit(&bars.fin);
      mbar_wait(&bars.fin, 0, nv, nullptr, 100000000ull);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

size_t logits_split_bytes(const Geo& g) {
  return 4 * static_cast<size_t>(g.B) * g.H * g.nB * g.d * 4;
}

template <int D>
static cudaError_t launch_logits_tc_d(const Geo& g, const float* qp, const float* kp, float scale, float* logits,
                                      float* split, uint32_t* err, int nsm, cudaStream_t st) {
  const int S = g.B * g.H;
  const long long n4 = static_cast<long long>(S) * g.nB * D / 4;
  split_kernel<D><<<static_cast<unsigned>((n4 + 255) / 256), 256, 0, st>>>(
      reinterpret_cast<const float4*>(qp), reinterpret_cast<const float4*>(kp), reinterpret_cast<float4*>(split), n4);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t plane = static_cast<size_t>(S) * g.nB * D;
  // the four maps depend only on the split buffer and the geometry: the last eight sets a
  // thread encoded are reused while they stay the same (a chunked call uses one per chunk)
  struct MapCache {
    unsigned long long ctx;
    const float* split;
    int S, nB;
    LgMaps maps;
    bool valid;
  };
  constexpr int kCached = 8;
  thread_local MapCache cache[kCached] = {};
  thread_local int next = 0;
  const unsigned long long ctx = current_ctx_id();
  MapCache* mcp = nullptr;
  for (int i = 0; i < kCached && mcp == nullptr; ++i) {
    const MapCache& c = cache[i];
    if (c.valid && ctx != 0 && c.ctx == ctx && c.split == split && c.S == S && c.nB == g.nB) mcp = &cache[i];
  }
  if (mcp == nullptr) {
    MapCache& c = cache[next];
    next = (next + 1) % kCached;
    c.valid = false;
    if (!encode_rows_fp32(&c.maps.qh, split, S, g.nB, D) ||
        !encode_rows_fp32(&c.maps.ql, split + plane, S, g.nB, D) ||
        !encode_rows_fp32(&c.maps.kh, split + 2 * plane, S, g.nB, D) ||
        !encode_rows_fp32(&c.maps.kl, split + 3 * plane, S, g.nB, D))
      return cudaErrorInvalidValue;
    c.ctx = ctx;
    c.split = split;
    c.S = S;
    c.nB = g.nB;
    c.valid = true;
    mcp = &c;
  }
  const MapCache& mc = *mcp;
  LgParams prm;
  prm.g = g;
  prm.logits = logits;
  prm.scale = scale;
  prm.err = err;
  prm.tiles = (g.nB + kLgTile - 1) / kLgTile;
  // key ranges: enough items for about three rounds over the SMs, each item at least two
  // key tiles (so that its query tile is used for more than one)
  const long long base = static_cast<long long>(S) * prm.tiles;
  int ksplit = 1;
  while (ksplit < prm.tiles / 2 && base * ksplit < 3LL * nsm) ++ksplit;
  prm.kper = (prm.tiles + ksplit - 1) / ksplit;
  prm.ksplit = (prm.tiles + prm.kper - 1) / prm.kper;
  prm.items = base * prm.ksplit;
  const long long grid = prm.items < nsm ? prm.items : nsm;
  constexpr int smem = lg_smem_bytes<D>();
  static SmemAttrCache attr_ctx = {};
  e = set_smem_once(reinterpret_cast<const void*>(logits_tc_kernel<D>), smem, attr_ctx);
  if (e != cudaSuccess) return e;
  logits_tc_kernel<D><<<static_cast<unsigned>(grid), kLgThreads, smem, st>>>(mc.maps.qh, mc.maps.ql, mc.maps.kh,
                                                                             mc.maps.kl, prm);
  return cudaGetLastError();
}

cudaError_t launch_logits_tc(const Geo& g, const float* qp, const float* kp, float scale, float* logits,
                             float* split, uint32_t* err, int nsm, cudaStream_t st) {
  return g.d == 128 ? launch_logits_tc_d<128>(g, qp, kp, scale, logits, split, err, nsm, st)
                    : launch_logits_tc_d<64>(g, qp, kp, scale, logits, split, err, nsm, st);
}

}  // namespace fv
