// Block-sparse attention over the kept key blocks, for B200 (sm_100a).
//
// FVAttn explainer (arXiv 2607.16190), 核心方法 §2: after routing, the attention
// kernel (attn_kernel.run(), the part that replaces FlashAttention) runs only over
// the selected KV blocks.  Here it is one persistent kernel per call:
//
//   * a (b, h, query block) "tile" is one query block of up to 128 tokens against
//     its kept key blocks, visited in ascending block order with an online softmax;
//   * tiles come from an atomic queue ordered by decreasing cost (longest processing
//     time first); the order is built by prep_kernel from the mask;
//   * warp 0 loads Q / K / V boxes with TMA (5D tensor maps over
//     [B*H][T][Hs][Ws][d], 128-byte swizzle, out-of-range rows zero-filled; blocks on
//     the W edge use a narrower box so their real rows stay compact), warp 1 issues
//     tcgen05.mma (S = Q K^T into tensor memory, then O += P V with P read from
//     tensor memory), warps 2..5 run the softmax, one TMEM lane (= query row) per
//     thread, and write out / lse;
//   * the running maximum is re-based lazily: O and l are rescaled only when the
//     block maximum exceeds the reference by more than 2^8, which keeps the result
//     exact (O / l and lse use the same reference) and P <= 256.
//
// Every wait is bounded (fv::mbar_wait): a stuck pipeline sets an error bit in the
// workspace, all roles leave their loops, outstanding copies and MMAs are drained,
// tensor memory is released and the kernel returns.
#include <cuda_bf16.h>

#include "fv_common.cuh"
#include "fv_launch.h"

namespace fv {

constexpr int kAttnThreads = 192;
constexpr int kNK = 3;                 // K ring depth
constexpr int kNV = 3;                 // V ring depth
constexpr int kTR = 2;                 // tile-id ring depth
constexpr int kChunkBytes = 128 * 128; // 128 rows x 64 bf16 (one 128-byte swizzle column)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;          // S buffers: columns [0,128) and [128,256)
constexpr uint32_t kColO = 256;        // O accumulator: [256, 256 + d)
constexpr uint32_t kColP = 384;        // P buffers (bf16 pairs): [384,448) and [448,512)
constexpr float kRebase = 8.0f;        // lazy re-basing threshold, log2 units

struct AttnParams {
  Geo g;
  const uint32_t* mask;   // nullptr: every key block
  float scale_log2;       // scale * log2(e)
  __nv_bfloat16* out;
  float* lse;
  uint32_t* hdr;          // [0] queue counter, [1] error bits
  const int* order;
  int ntiles;
  unsigned long long* busy;
};

struct __align__(8) AttnBars {
  uint64_t q_full, q_empty;
  uint64_t k_full[kNK], k_empty[kNK];
  uint64_t v_full[kNV], v_empty[kNV];
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full[2];
  uint64_t pv_done, o_empty;
  uint64_t t_full[kTR], t_empty[kTR];
  uint64_t fin;
  int tile[kTR];
  uint32_t tmem_base;
  int abort;
};

template <int D>
__host__ __device__ constexpr int tile_bytes() { return (D / 64) * kChunkBytes; }
template <int D>
__host__ __device__ constexpr int attn_smem_bytes() { return tile_bytes<D>() * (1 + kNK + kNV) + 1024; }

// Iterates the set bits of a mask row in ascending order (or every block when dense).
struct KvIter {
  const uint32_t* row;
  int nB, words, w, next;
  uint32_t bits;
  __device__ void init(const uint32_t* r, int nB_, int words_) {
    row = r; nB = nB_; words = words_; w = -1; bits = 0; next = -1;
  }
  __device__ int advance() {      // returns the next block id, or -1
    if (row == nullptr) {
      ++next;
      return next < nB ? next : -1;
    }
    while (bits == 0) {
      ++w;
      if (w >= words) return -1;
      bits = __ldg(row + w);
    }
    const int b = __ffs(bits) - 1;
    bits &= bits - 1;
    return w * 32 + b;
  }
};

__device__ __forceinline__ void decode_tile(const Geo& g, int tile, int& bhi, int& qb) {
  bhi = tile / g.nB;
  qb = tile - bhi * g.nB;
}

template <int D>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmQe,
                const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmKe,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmVe,
                const AttnParams prm) {
  constexpr int NCH = D / 64;              // 64-column chunks per row
  constexpr int TILE = tile_bytes<D>();
  extern __shared__ unsigned char attn_dsm[];
  __shared__ AttnBars bars;

  const uint64_t t_start = globaltimer();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Geo& g = prm.g;
  uint32_t* err = prm.hdr + 1;
  volatile int* abort = &bars.abort;

  // 1024-byte aligned operand area: Q | K ring | V ring
  const uint32_t dsm0 = smem_u32(attn_dsm);
  const uint32_t base = (dsm0 + 1023u) & ~1023u;
  unsigned char* gbase = attn_dsm + (base - dsm0);
  const uint32_t sQ = base;
  auto sK = [&](int s) { return base + static_cast<uint32_t>(TILE * (1 + s)); };
  auto sV = [&](int s) { return base + static_cast<uint32_t>(TILE * (1 + kNK + s)); };

  if (threadIdx.x == 0) {
    mbar_init(&bars.q_full, 1);
    mbar_init(&bars.q_empty, 1);
    for (int i = 0; i < kNK; ++i) { mbar_init(&bars.k_full[i], 1); mbar_init(&bars.k_empty[i], 1); }
    for (int i = 0; i < kNV; ++i) { mbar_init(&bars.v_full[i], 1); mbar_init(&bars.v_empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.s_full[i], 1);
      mbar_init(&bars.s_empty[i], 4);
      mbar_init(&bars.p_full[i], 4);
    }
    mbar_init(&bars.pv_done, 1);
    mbar_init(&bars.o_empty, 4);
    for (int i = 0; i < kTR; ++i) { mbar_init(&bars.t_full[i], 1); mbar_init(&bars.t_empty[i], 5); }
    mbar_init(&bars.fin, 1);
    bars.abort = 0;
    fence_barrier_init();
  }
  // Rows past a box are read by the MMAs (multiplied by zero P or masked): start
  // from zeros so they are finite.
  {
    uint4* z = reinterpret_cast<uint4*>(gbase);
    const int n16 = TILE * (1 + kNK + kNV) / 16;
    for (int i = threadIdx.x; i < n16; i += kAttnThreads) z[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(&bars.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ); tma_prefetch_desc(&tmQe);
    tma_prefetch_desc(&tmK); tma_prefetch_desc(&tmKe);
    tma_prefetch_desc(&tmV); tma_prefetch_desc(&tmVe);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;

  uint32_t kc = 0, vc = 0, qc = 0;   // producer-side counters (also used in the drain)

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t tcount = 0;
      bool ok = true;
      while (ok) {
        const int pos = static_cast<int>(atomicAdd(prm.hdr, 1u));
        const int tile = pos < prm.ntiles ? __ldg(prm.order + pos) : -1;
        const int slot = tcount % kTR;
        if (!mbar_wait(&bars.t_empty[slot], ((tcount / kTR) & 1) ^ 1, abort, err)) break;
        bars.tile[slot] = tile;
        mbar_arrive(&bars.t_full[slot]);
        ++tcount;
        if (tile < 0) break;
        int bhi, qb;
        decode_tile(g, tile, bhi, qb);
        const BlockInfo qi = block_info(g, qb);
        if (!mbar_wait(&bars.q_empty, (qc & 1) ^ 1, abort, err)) break;
        mbar_arrive_expect_tx(&bars.q_full, static_cast<uint32_t>(qi.rows * 128 * NCH));
        for (int c = 0; c < NCH; ++c)
          tma_load_5d(sQ + c * kChunkBytes, qi.xedge ? &tmQe : &tmQ, &bars.q_full, c * 64,
                      qi.xb * g.bw, qi.yb * g.bh, qi.tb * g.bt, bhi);
        ++qc;
        KvIter it;
        it.init(prm.mask ? prm.mask + static_cast<size_t>(tile) * g.words : nullptr, g.nB, g.words);
        for (int kb = it.advance(); kb >= 0; kb = it.advance()) {
          const BlockInfo ki = block_info(g, kb);
          const uint32_t bytes = static_cast<uint32_t>(ki.rows * 128 * NCH);
          const int ks = kc % kNK;
          if (!mbar_wait(&bars.k_empty[ks], ((kc / kNK) & 1) ^ 1, abort, err)) { ok = false; break; }
          mbar_arrive_expect_tx(&bars.k_full[ks], bytes);
          for (int c = 0; c < NCH; ++c)
            tma_load_5d(sK(ks) + c * kChunkBytes, ki.xedge ? &tmKe : &tmK, &bars.k_full[ks],
                        c * 64, ki.xb * g.bw, ki.yb * g.bh, ki.tb * g.bt, bhi);
          ++kc;
          const int vs = vc % kNV;
          if (!mbar_wait(&bars.v_empty[vs], ((vc / kNV) & 1) ^ 1, abort, err)) { ok = false; break; }
          mbar_arrive_expect_tx(&bars.v_full[vs], bytes);
          for (int c = 0; c < NCH; ++c)
            tma_load_5d(sV(vs) + c * kChunkBytes, ki.xedge ? &tmVe : &tmV, &bars.v_full[vs],
                        c * 64, ki.xb * g.bw, ki.yb * g.bh, ki.tb * g.bt, bhi);
          ++vc;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t tcount = 0, mkc = 0, mvc = 0, mqc = 0, sc = 0, pc = 0, tiles = 0;
      const uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
      bool ok = true;
      while (ok) {
        const int slot = tcount % kTR;
        if (!mbar_wait(&bars.t_full[slot], (tcount / kTR) & 1, abort, err)) break;
        const int tile = bars.tile[slot];
        mbar_arrive(&bars.t_empty[slot]);
        ++tcount;
        if (tile < 0) break;
        if (!mbar_wait(&bars.q_full, mqc & 1, abort, err)) break;
        ++mqc;
        KvIter it;
        it.init(prm.mask ? prm.mask + static_cast<size_t>(tile) * g.words : nullptr, g.nB, g.words);
        bool have_prev = false, first_pv = true;
        int prev_npad = 0;
        auto issue_pv = [&](int npad) -> bool {
          const int b = pc & 1;
          if (!mbar_wait(&bars.p_full[b], (pc >> 1) & 1, abort, err)) return false;
          const int vs = mvc % kNV;
          if (!mbar_wait(&bars.v_full[vs], (mvc / kNV) & 1, abort, err)) return false;
          if (first_pv && !mbar_wait(&bars.o_empty, (tiles & 1) ^ 1, abort, err)) return false;
          tc_fence_after();
          for (int kk = 0; kk < npad / 16; ++kk) {
            const uint64_t bdesc = sdesc_sw128(sV(vs) + kk * 2048, kChunkBytes, 1024);
            mma_ts(tmem + kColO, tmem + kColP + b * 64 + kk * 8, bdesc, idesc_pv,
                   (first_pv && kk == 0) ? 0u : 1u);
          }
          mma_commit(&bars.v_empty[vs]);
          mma_commit(&bars.pv_done);
          ++mvc;
          ++pc;
          first_pv = false;
          return true;
        };
        for (int kb = it.advance(); kb >= 0; kb = it.advance()) {
          const int npad = block_info(g, kb).npad;
          const int ks = mkc % kNK;
          if (!mbar_wait(&bars.k_full[ks], (mkc / kNK) & 1, abort, err)) { ok = false; break; }
          const int b = sc & 1;
          if (!mbar_wait(&bars.s_empty[b], ((sc >> 1) & 1) ^ 1, abort, err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t idesc_s = idesc_bf16_f32(128, npad, 0, 0);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * kChunkBytes + (kk & 3) * 32;
            mma_ss(tmem + kColS + b * 128, sdesc_sw128(sQ + off, 16, 1024),
                   sdesc_sw128(sK(ks) + off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
          }
          mma_commit(&bars.s_full[b]);
          mma_commit(&bars.k_empty[ks]);
          ++mkc;
          ++sc;
          if (have_prev && !issue_pv(prev_npad)) { ok = false; break; }
          have_prev = true;
          prev_npad = npad;
        }
        if (!ok) break;
        mma_commit(&bars.q_empty);
        if (have_prev && !issue_pv(prev_npad)) break;
        ++tiles;
      }
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    uint32_t tcount = 0, sc = 0, pvc = 0;
    const float sl2 = prm.scale_log2;
    while (true) {
      const int slot = tcount % kTR;
      bool okw = mbar_wait(&bars.t_full[slot], (tcount / kTR) & 1, abort, err);
      if (!__all_sync(0xffffffffu, okw)) break;
      const int tile = bars.tile[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.t_empty[slot]);
      ++tcount;
      if (tile < 0) break;
      int bhi, qb;
      decode_tile(g, tile, bhi, qb);
      const BlockInfo qi = block_info(g, qb);
      const int token = box_row_token(g, qi, row);

      float m_ref = -INFINITY, l = 0.f;
      int j = 0;
      bool ok = true;
      KvIter it;
      it.init(prm.mask ? prm.mask + static_cast<size_t>(tile) * g.words : nullptr, g.nB, g.words);
      for (int kb = it.advance(); kb >= 0; kb = it.advance()) {
        const BlockInfo ki = block_info(g, kb);
        // validity of the 128 key columns of this block (same for every row)
        uint32_t vm[4];
        if (ki.prefix) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int n = ki.nvalid - 32 * q;
            vm[q] = n >= 32 ? 0xffffffffu : (n <= 0 ? 0u : ((1u << n) - 1u));
          }
        } else {
#pragma unroll
          for (int q = 0; q < 4; ++q)
            vm[q] = __ballot_sync(0xffffffffu, box_row_token(g, ki, 32 * q + lane) >= 0);
        }
        const int b = sc & 1;
        okw = mbar_wait(&bars.s_full[b], (sc >> 1) & 1, abort, err);
        if (!__all_sync(0xffffffffu, okw)) { ok = false; break; }
        tc_fence_after();
        float s[128];
        // all 128 columns (columns past the block's rows are masked below); loads
        // under a data-dependent condition would push the row out to local memory
#pragma unroll
        for (int c = 0; c < 4; ++c)
          tmem_ld32(tmem + lane_off + kColS + b * 128 + 32 * c, reinterpret_cast<uint32_t*>(s + 32 * c));
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.s_empty[b]);
        ++sc;

        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          const bool v = (vm[c >> 5] >> (c & 31)) & 1u;
          s[c] = v ? s[c] * sl2 : -INFINITY;
          mx = fmaxf(mx, s[c]);
        }
        float m_use = m_ref, alpha = 1.f;
        bool rebase = false;
        if (j == 0) {
          m_use = mx;
        } else if (mx > m_ref + kRebase) {
          m_use = mx;
          alpha = ex2(m_ref - mx);
          rebase = true;
        }
        uint32_t pk[64];
        float rs = 0.f;
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const float p0 = ex2(s[2 * c] - m_use);
          const float p1 = ex2(s[2 * c + 1] - m_use);
          rs += p0 + p1;
          pk[c] = pack_bf16x2(p0, p1);
        }
        l = l * alpha + rs;
        m_ref = m_use;
        if (j > 0) {
          okw = mbar_wait(&bars.pv_done, pvc & 1, abort, err);
          if (!__all_sync(0xffffffffu, okw)) { ok = false; break; }
          ++pvc;
          tc_fence_after();
          if (__any_sync(0xffffffffu, rebase)) {
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t o[32];
              tmem_ld32(tmem + lane_off + kColO + 32 * c, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              tmem_st32(tmem + lane_off + kColO + 32 * c, o);
            }
          }
        }
#pragma unroll
        for (int c = 0; c < 2; ++c) tmem_st32(tmem + lane_off + kColP + b * 64 + 32 * c, pk + 32 * c);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.p_full[b]);
        ++j;
      }
      if (!ok) break;
      // epilogue: O / l -> out (bf16), lse
      okw = mbar_wait(&bars.pv_done, pvc & 1, abort, err);
      if (!__all_sync(0xffffffffu, okw)) break;
      ++pvc;
      tc_fence_after();
      uint32_t o[D];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) tmem_ld32(tmem + lane_off + kColO + 32 * c, o + 32 * c);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.o_empty);
      if (token >= 0) {
        const float inv = 1.f / l;
        uint4* dst = reinterpret_cast<uint4*>(prm.out + (static_cast<size_t>(bhi) * g.N + token) * D);
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(o[8 * c + 0]) * inv, __uint_as_float(o[8 * c + 1]) * inv);
          w.y = pack_bf16x2(__uint_as_float(o[8 * c + 2]) * inv, __uint_as_float(o[8 * c + 3]) * inv);
          w.z = pack_bf16x2(__uint_as_float(o[8 * c + 4]) * inv, __uint_as_float(o[8 * c + 5]) * inv);
          w.w = pack_bf16x2(__uint_as_float(o[8 * c + 6]) * inv, __uint_as_float(o[8 * c + 7]) * inv);
          dst[c] = w;
        }
        prm.lse[static_cast<size_t>(bhi) * g.N + token] = (m_ref + __log2f(l)) * 0.69314718055994531f;
      }
    }
  }

  // ------------------------------------------------------------ teardown
  __syncthreads();
  if (bars.abort) {
    // Drain: let every armed TMA copy land and every issued MMA finish before the
    // shared and tensor memory they touch is released.  Bounded, abort ignored.
    if (warp == 0 && lane == 0) {
      int never = 0;
      volatile int* nv = &never;
      if (qc > 0) mbar_wait(&bars.q_full, (qc - 1) & 1, nv, nullptr, 100000000ull);
      for (uint32_t i = (kc > kNK ? kc - kNK : 0); i < kc; ++i)
        mbar_wait(&bars.k_full[i % kNK], (i / kNK) & 1, nv, nullptr, 100000000ull);
      for (uint32_t i = (vc > kNV ? vc - kNV : 0); i < vc; ++i)
        mbar_wait(&bars.v_full[i % kNV], (i / kNV) & 1, nv, nullptr, 100000000ull);
    }
    if (warp == 1 && lane == 0) {
      int never = 0;
      volatile int* nv = &never;
      mma_commit(&bars.fin);
      mbar_wait(&bars.fin, 0, nv, nullptr, 100000000ull);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && prm.busy != nullptr)
    atomicAdd(prm.busy + smid(), static_cast<unsigned long long>(globaltimer() - t_start));
}

// ----------------------------------------------------------------------------
// Schedule prep: one CTA.  Resets the queue counter, the error word and the SM busy
// record; scores every tile by its issued work, sum over kept blocks of (rows padded
// to 16 + a per-block overhead), and writes the tile order by decreasing cost
// (2048 cost buckets, counting sort).  Order inside a bucket is arbitrary; it only
// affects timing, never results.
// ----------------------------------------------------------------------------
constexpr int kPrepThreads = 1024;
constexpr int kBuckets = 2048;
constexpr int kBlockOverhead = 64;

__global__ void __launch_bounds__(kPrepThreads) prep_kernel(Geo g, const uint32_t* __restrict__ mask,
                                                            uint32_t* hdr, int* order, int* keys,
                                                            int ntiles, unsigned long long* busy,
                                                            int nsm) {
  __shared__ int hist[kBuckets];
  __shared__ uint32_t edge[64];
  __shared__ int wsum[32];
  const int t = threadIdx.x;
  if (t == 0) { hdr[0] = 0; hdr[1] = 0; }
  if (busy)
    for (int i = t; i < nsm; i += kPrepThreads) busy[i] = 0ull;
  if (mask == nullptr) {
    for (int i = t; i < ntiles; i += kPrepThreads) order[i] = i;
    return;
  }
  const int words = g.words;
  for (int w = t; w < words; w += kPrepThreads) {
    uint32_t bits = 0;
    for (int i = 0; i < 32; ++i) {
      const int j = w * 32 + i;
      if (j < g.nB && (j % g.nBx) == g.nBx - 1) bits |= 1u << i;
    }
    edge[w] = bits;
  }
  for (int i = t; i < kBuckets; i += kPrepThreads) hist[i] = 0;
  __syncthreads();
  const int rx_edge = g.Ws - (g.nBx - 1) * g.bw;
  const long long full = ((g.bt * g.bh * g.bw + 15) & ~15) + kBlockOverhead;
  const long long part = ((g.bt * g.bh * rx_edge + 15) & ~15) + kBlockOverhead;
  const long long maxcost = full * g.nB;
  for (int i = t; i < ntiles; i += kPrepThreads) {
    const uint32_t* row = mask + static_cast<size_t>(i) * words;
    long long cost = 0;
    for (int w = 0; w < words; ++w) {
      const uint32_t m = __ldg(row + w);
      cost += full * __popc(m) - (full - part) * __popc(m & edge[w]);
    }
    int key = static_cast<int>(((maxcost - cost) * (kBuckets - 1)) / maxcost);
    key = min(max(key, 0), kBuckets - 1);
    keys[i] = key;
    atomicAdd(&hist[key], 1);
  }
  __syncthreads();
  // exclusive scan of the histogram: warp 0, 64 buckets per lane
  if (t < 32) {
    int run = 0;
    for (int i = 0; i < kBuckets / 32; ++i) run += hist[t * (kBuckets / 32) + i];
    int incl = run;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (t >= off) incl += v;
    }
    wsum[t] = incl - run;
  }
  __syncthreads();
  if (t < 32) {
    int acc = wsum[t];
    for (int i = 0; i < kBuckets / 32; ++i) {
      const int idx = t * (kBuckets / 32) + i;
      const int c = hist[idx];
      hist[idx] = acc;
      acc += c;
    }
  }
  __syncthreads();
  for (int i = t; i < ntiles; i += kPrepThreads) {
    const int pos = atomicAdd(&hist[keys[i]], 1);
    order[pos] = i;
  }
}

template <int D>
static cudaError_t launch_attn_d(const Geo& g, const AttnMaps& maps, const AttnParams& prm, int grid,
                                 cudaStream_t st) {
  constexpr int smem = attn_smem_bytes<D>();
  cudaError_t e = cudaFuncSetAttribute(attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  attn_kernel<D><<<grid, kAttnThreads, smem, st>>>(maps.q, maps.qe, maps.k, maps.ke, maps.v, maps.ve, prm);
  return cudaGetLastError();
}

cudaError_t launch_attn(const Geo& g, const AttnMaps& maps, const uint32_t* mask, float scale,
                        void* out, float* lse, void* ws, unsigned long long* busy, int nsm,
                        cudaStream_t st) {
  const int ntiles = g.B * g.H * g.nB;
  uint32_t* hdr = static_cast<uint32_t*>(ws);
  int* order = reinterpret_cast<int*>(static_cast<unsigned char*>(ws) + kWsHeader);
  int* keys = order + ntiles;
  prep_kernel<<<1, kPrepThreads, 0, st>>>(g, mask, hdr, order, keys, ntiles, busy, nsm);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  AttnParams prm;
  prm.g = g;
  prm.mask = mask;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.lse = lse;
  prm.hdr = hdr;
  prm.order = order;
  prm.ntiles = ntiles;
  prm.busy = busy;
  const int grid = ntiles < nsm ? ntiles : nsm;
  return g.d == 128 ? launch_attn_d<128>(g, maps, prm, grid, st)
                    : launch_attn_d<64>(g, maps, prm, grid, st);
}

}  // namespace fv
