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
// One CTA per work unit = (slice, 128 query blocks, a range of 128-key-block tiles):
//   warps 0-3  load Qp / Kp rows from global memory (L2), split them into hi and lo and
//              store both into shared memory in the 128-byte-swizzled K-major layout the
//              MMA descriptors read (the query tile once, key tiles 32 channels at a time
//              through a ring of stages);
//   warp 4     issues the MMAs (one elected lane) into one of two 128-column fp32
//              accumulators in tensor memory;
//   warps 5-8  read an accumulator (one TMEM lane = one query row per thread), scale it
//              and store the row's 128 logits, while the other accumulator fills.
// Every wait is bounded; a stuck pipeline raises the workspace's error word and the
// kernel drains and returns (fv::mbar_wait).
#include "fv_common.cuh"
#include "fv_launch.h"

namespace fv {

constexpr int kLgThreads = 288;           // 9 warps
constexpr int kLgChunk = 128 * 128;       // bytes: 128 rows x 32 fp32 (one swizzle column)
constexpr int kLgTile = 128;              // query / key blocks per tile

template <int D> __host__ __device__ constexpr int lg_stages() { return D == 128 ? 3 : 4; }

struct __align__(8) LgBars {
  uint64_t a_full;
  uint64_t st_full[4], st_empty[4];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t fin;
  uint32_t tmem_base;
  int abort;
};

template <int D>
__host__ __device__ constexpr int lg_smem_bytes() {
  return 2 * (D / 32) * kLgChunk + lg_stages<D>() * 2 * kLgChunk + static_cast<int>(sizeof(LgBars));
}
static_assert(lg_smem_bytes<128>() <= 232448, "logits kernel exceeds 227 KB of shared memory");

struct LgParams {
  Geo g;
  const float* qp;
  const float* kp;
  float* logits;      // [B*H][nB][words*32]
  float scale;
  uint32_t* err;      // error word of the route workspace
  int qtiles, ktiles, kper;   // 128-block tiles per slice (rows, keys); key tiles per unit
  int nsplit;                 // units per (slice, query tile)
};

// 16 bytes (4 channels) of pooled row `row` of a 128-row tile, split and stored at 16-byte
// unit `col16` of the row in the swizzled chunk.
__device__ __forceinline__ void lg_store_split(uint32_t hi_base, uint32_t lo_base, int row, int col16, float4 x) {
  const uint32_t off = static_cast<uint32_t>(row * 128 + ((col16 ^ (row & 7)) << 4));
  const float h0 = to_tf32(x.x), h1 = to_tf32(x.y), h2 = to_tf32(x.z), h3 = to_tf32(x.w);
  const float l0 = to_tf32(x.x - h0), l1 = to_tf32(x.y - h1), l2 = to_tf32(x.z - h2), l3 = to_tf32(x.w - h3);
  asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(hi_base + off), "f"(h0), "f"(h1), "f"(h2), "f"(h3)
               : "memory");
  asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(lo_base + off), "f"(l0), "f"(l1), "f"(l2), "f"(l3)
               : "memory");
}

template <int D>
__global__ void __launch_bounds__(kLgThreads, 1) logits_tc_kernel(const LgParams prm) {
  constexpr int NC = D / 32;                // 32-channel chunks per row
  constexpr int S = lg_stages<D>();
  extern __shared__ __align__(1024) unsigned char lg_dsm[];
  LgBars& bars = *reinterpret_cast<LgBars*>(lg_dsm + 2 * NC * kLgChunk + S * 2 * kLgChunk);
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

  // work unit -> slice, query tile, key tiles [kt0, kt1)
  const int unit = blockIdx.x;
  const int per_slice = prm.qtiles * prm.nsplit;
  const int bhi = unit / per_slice;
  const int rem = unit - bhi * per_slice;
  const int qt = rem / prm.nsplit, sp = rem - qt * prm.nsplit;
  const int kt0 = sp * prm.kper, kt1 = min(prm.ktiles, kt0 + prm.kper);
  const int nt = kt1 - kt0;
  const int nB = g.nB, nBpad = g.words * 32;
  const int q0 = qt * kLgTile;

  if (threadIdx.x == 0) {
    mbar_init(&bars.a_full, 128);
    for (int i = 0; i < S; ++i) { mbar_init(&bars.st_full[i], 128); mbar_init(&bars.st_empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&bars.acc_full[i], 1); mbar_init(&bars.acc_empty[i], 4); }
    mbar_init(&bars.fin, 1);
    bars.abort = 0;
    fence_barrier_init();
  }
  if (warp == 4) {
    tmem_alloc(&bars.tmem_base, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;

  if (warp < 4) {
    // ------------------------------------------------------------ operand staging
    const int t = threadIdx.x;
    const float4* qrows = reinterpret_cast<const float4*>(prm.qp + static_cast<size_t>(bhi) * nB * D);
    const float4* krows = reinterpret_cast<const float4*>(prm.kp + static_cast<size_t>(bhi) * nB * D);
    const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
    for (int c = 0; c < NC; ++c) {
#pragma unroll 2
      for (int u = t; u < 1024; u += 128) {
        const int row = u >> 3, col16 = u & 7;
        const int r = q0 + row;
        const float4 x = r < nB ? __ldcg(qrows + static_cast<size_t>(r) * (D / 4) + c * 8 + col16) : zero;
        lg_store_split(sAhi + c * kLgChunk, sAlo + c * kLgChunk, row, col16, x);
      }
    }
    fence_proxy_async_smem();
    mbar_arrive(&bars.a_full);
    uint32_t i = 0;
    bool ok = true;
#pragma unroll 1
    for (int kt = kt0; kt < kt1 && ok; ++kt) {
#pragma unroll 1
      for (int c = 0; c < NC; ++c, ++i) {
        const int s = i % S;
        if (!mbar_wait(&bars.st_empty[s], ((i / S) & 1) ^ 1, abort, err)) { ok = false; break; }
#pragma unroll 2
        for (int u = t; u < 1024; u += 128) {
          const int row = u >> 3, col16 = u & 7;
          const int r = kt * kLgTile + row;
          const float4 x = r < nB ? __ldcg(krows + static_cast<size_t>(r) * (D / 4) + c * 8 + col16) : zero;
          lg_store_split(sBhi(s), sBlo(s), row, col16, x);
        }
        fence_proxy_async_smem();
        mbar_arrive(&bars.st_full[s]);
      }
    }
  } else if (warp == 4) {
    // ------------------------------------------------------------ MMA issue
    const uint32_t idesc = idesc_tf32_f32(128, 128);
    auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, err));
    };
    bool ok = wwait(&bars.a_full, 0);
    tc_fence_after();
    uint32_t i = 0;
#pragma unroll 1
    for (int j = 0; j < nt && ok; ++j) {
      const int slot = j & 1;
      if (!wwait(&bars.acc_empty[slot], ((j >> 1) & 1) ^ 1)) break;
      const uint32_t tacc = tmem + static_cast<uint32_t>(slot * 128);
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
          if (c == NC - 1) mma_commit(&bars.acc_full[slot]);
        }
        __syncwarp();
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int r = q0 + row;
    float* out = prm.logits + (static_cast<size_t>(bhi) * nB + (r < nB ? r : 0)) * nBpad;
    const float sc = prm.scale;
#pragma unroll 1
    for (int j = 0; j < nt; ++j) {
      const int slot = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&bars.acc_full[slot], (j >> 1) & 1, abort, err))) break;
      tc_fence_after();
      const int k0 = (kt0 + j) * kLgTile;
#pragma unroll 1
      for (int g4 = 0; g4 < 4; ++g4) {
        uint32_t v[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(slot * 128 + 32 * g4), v);
        tmem_wait_ld();
        const int col = k0 + 32 * g4;
        if (r < nB && col < nBpad) {
          float4* dst = reinterpret_cast<float4*>(out + col);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(__uint_as_float(v[4 * e]) * sc, __uint_as_float(v[4 * e + 1]) * sc,
                                 __uint_as_float(v[4 * e + 2]) * sc, __uint_as_float(v[4 * e + 3]) * sc);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.acc_empty[slot]);
    }
  }

  // ------------------------------------------------------------ teardown
  __syncthreads();
  if (bars.abort && warp == 4 && lane == 0) {
    // let every issued MMA finish before tensor and shared memory are released
    int never = 0;
    volatile int* nv = &never;
    mma_commit(&bars.fin);
    mbar_wait(&bars.fin, 0, nv, nullptr, 100000000ull);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

template <int D>
static cudaError_t launch_logits_tc_d(const Geo& g, const float* qp, const float* kp, float scale, float* logits,
                                      uint32_t* err, int nsm, cudaStream_t st) {
  LgParams prm;
  prm.g = g;
  prm.qp = qp;
  prm.kp = kp;
  prm.logits = logits;
  prm.scale = scale;
  prm.err = err;
  prm.qtiles = (g.nB + kLgTile - 1) / kLgTile;
  prm.ktiles = prm.qtiles;
  // split the key tiles of a (slice, query tile) over enough units for two waves
  const long long base = static_cast<long long>(g.B) * g.H * prm.qtiles;
  int nsplit = 1;
  while (nsplit < prm.ktiles && base * nsplit < 2LL * nsm) ++nsplit;
  prm.kper = (prm.ktiles + nsplit - 1) / nsplit;
  prm.nsplit = (prm.ktiles + prm.kper - 1) / prm.kper;
  const long long units = base * prm.nsplit;
  constexpr int smem = lg_smem_bytes<D>();
  cudaError_t e = cudaFuncSetAttribute(logits_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  logits_tc_kernel<D><<<static_cast<unsigned>(units), kLgThreads, smem, st>>>(prm);
  return cudaGetLastError();
}

cudaError_t launch_logits_tc(const Geo& g, const float* qp, const float* kp, float scale, float* logits,
                             uint32_t* err, int nsm, cudaStream_t st) {
  return g.d == 128 ? launch_logits_tc_d<128>(g, qp, kp, scale, logits, err, nsm, st)
                    : launch_logits_tc_d<64>(g, qp, kp, scale, logits, err, nsm, st);
}

}  // namespace fv
