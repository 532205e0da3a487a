// Block-sparse attention over the kept key blocks, for B200 (sm_100a).
//
// FVAttn explainer (arXiv 2607.16190), 核心方法 §2: after routing, the attention
// kernel (attn_kernel.run(), the part that replaces FlashAttention) runs only over
// the selected KV blocks.  Here it is one persistent kernel per call:
//
//   * a (b, h, query block) "tile" is one query block of up to 128 tokens against
//     its kept key blocks with an online softmax: the wide blocks in ascending order,
//     then the narrow W-edge blocks packed up to 128 / rows_e per 128-row K/V slot;
//   * tiles come from an atomic queue ordered by decreasing cost (longest processing
//     time first); the order is built by prep_kernel from the mask;
//   * warp 0 loads Q / K / V boxes with TMA (5D tensor maps over
//     [B*H][T][Hs][Ws][d], 128-byte swizzle, out-of-range rows zero-filled; blocks on
//     the W edge use a narrower box so their real rows stay compact), warp 1 issues
//     tcgen05.mma (S_j = Q K_j^T into a three-deep ring of S buffers in tensor memory,
//     then O += P_j V_j with P_j read from tensor memory over S_j);
//   * two softmax warpgroups take the kept blocks alternately (even j, odd j), one
//     TMEM lane (= query row) per thread.  They share one O accumulator, so every P_j
//     is taken against one running reference per row: the group that owns block j
//     receives the reference after block j-1 from the other group through shared
//     memory, updates it with its own block maximum and hands it on before computing
//     its exponentials, so the two groups' exponentials overlap each other and the
//     tensor core;
//   * the reference is re-based lazily: O and l are rescaled only when the block
//     maximum exceeds the reference by more than 2^8, which keeps the result exact
//     (O / l and lse use the same reference) and P <= 256.
//
// Every wait is bounded (fv::mbar_wait): a stuck pipeline sets an error bit in the
// workspace, all roles leave their loops, outstanding copies and MMAs are drained,
// tensor memory is released and the kernel returns.
#include <cuda_bf16.h>

#include "fv_common.cuh"
#include "fv_launch.h"

namespace fv {

constexpr int kSoftWarps = 8;          // softmax warps: one per TMEM lane quarter in each group
// Three warpgroups: warps 0-3 (producer, S issuer, P.V issuer, one idle warp) and two softmax
// warpgroups (warps 4-7 and 8-11).  Launched at 168 registers a thread (the register
// file is split per SM partition, and each partition holds one warp of each group);
// setmaxnreg then moves registers from the first group to the softmax groups:
// 128 * 56 + 256 * 224 = 64512 = 384 * 168.
constexpr int kAttnThreads = 384;
constexpr int kRegsCtl = 56;
constexpr int kRegsSoft = 224;
static_assert(128 * kRegsCtl + 256 * kRegsSoft <= kAttnThreads * 168, "register split exceeds the launch budget");
constexpr int kNK = 3;                 // K ring depth
constexpr int kNV = 2;                 // V ring depth (P.V runs a softmax behind S: V has slack)
constexpr int kMaxBlocks = 2048;       // blocks per (b, h) slice, the mask row limit
constexpr int kTR = 2;                 // tile-id ring depth
constexpr int kChunkBytes = 128 * 128; // 128 rows x 64 bf16 (one 128-byte swizzle column)
constexpr uint32_t kTmemCols = 512;
// Tensor memory (512 columns x 128 lanes, lane = query row): three S slots of 128 fp32
// columns and O (d columns).  P_c (bf16 pairs, 64 columns) is written over S_c in its
// own slot: the softmax group holds the whole row of S_c in registers before it stores
// any P, so nothing else waits for a P slot.  S slot c mod 3 takes S_c+3 once P.V c has
// read P_c, three blocks of slack for the tensor core.
constexpr int kNS = 3;                 // S / P ring depth
constexpr int kPV = 6;                 // P.V completion barriers (block c commits [c % 6])
constexpr uint32_t kColS = 0;          // S slot r: columns [128r, 128r+128), P_c over its first 64
constexpr uint32_t kColO = 128 * kNS;  // O: columns [384, 384 + d)
static_assert(kColO + 128 <= 512, "tensor memory layout exceeds 512 columns");
constexpr float kRebase = 8.0f;        // lazy re-basing threshold, log2 units

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

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
  int pack;               // narrow (W-edge) key blocks packed per 128-row K/V slot (1: none)
  int rows_e;             // box rows of a W-edge block (bt * bh * (Ws mod bw))
  int qg;                 // narrow query blocks grouped per 128-row tile (1: none)
  int qps;                // lane quarters per grouped query block (rows_e / 32)
  unsigned long long stall_ns;  // test hook: > 0 makes the S issuer wait this long on a
                                // barrier nothing arrives at, at its first tile (0: off)
};

struct __align__(8) AttnBars {
  uint64_t q_full, q_empty;
  uint64_t k_full[kNK], k_empty[kNK];
  uint64_t v_full[kNV], v_empty[kNV];
  uint64_t s_full[kNS];   // per S slot: S_c written by the MMA
  uint64_t p_full[kNS];   // per S slot: P_c stored over S_c by the softmax group
  uint64_t pv_done[kPV];  // P.V of block c commits [c % 6].  A wait for P.V x on it needs
                          // P.V x-6 complete; every waiter knows P.V c-3 complete for a
                          // block c it has seen S of (S_c is issued only after P.V c-3),
                          // and waits only for P.V of c-3 .. c, so no wait aliases a phase
  uint64_t o_empty;
  uint64_t hb[2][4];      // reference hand-off, [writing group][TMEM lane quarter]
  uint64_t xbar[4];       // end-of-tile row-sum exchange, per TMEM lane quarter: written
  uint64_t xread[4];      //   ... and read by both warps of the quarter pair
  uint64_t t_full[kTR], t_empty[kTR];
  uint64_t fin[2];        // drain after an abort: S issuer, P.V issuer
  uint64_t never;         // no thread arrives here (the stall test hook waits on it)
  int tile[kTR];
  int bcount[kTR];        // kept wide blocks of the tile
  int ncount[kTR];        // kept narrow (packed) blocks of the tile
  uint32_t blist[kTR][kMaxBlocks];  // the tile's kept blocks (pack_blk): wide ones in
                                    // ascending order, then narrow ones in ascending order
  uint32_t edgew[kMaxBlocks / 32];  // per mask word: bits of the blocks that are packed
  uint32_t gmask[kTR][4][kMaxBlocks / 32];  // a query group's member mask rows (tile list slot)
  uint32_t tmem_base;
  int abort;
  float hv[2][128];       // [group][row] reference after the group's latest block, guarded by hb
  float xl[2][128];       // [group][row] row sums at the end of a tile, guarded by xbar / xread
};

template <int D>
__host__ __device__ constexpr int tile_bytes() { return (D / 64) * kChunkBytes; }
// Dynamic shared memory: Q | K ring | V ring (each 1024-byte aligned for the 128-byte
// swizzle) followed by the barrier block.  The dynamic window starts right after the
// 1 KB the hardware reserves per CTA, which is 1024-byte aligned; the kernel checks
// it and reports an error instead of running misaligned.
template <int D>
__host__ __device__ constexpr int attn_smem_bytes() {
  return tile_bytes<D>() * (1 + kNK + kNV) + static_cast<int>(sizeof(AttnBars));
}
static_assert(attn_smem_bytes<128>() <= 232448, "attention kernel exceeds 227 KB of shared memory");

// One kept block of a tile as the consumers need it: block id (bits 0-11), npad / 16
// (12-15), real token count (16-23), real tokens form a prefix of the box (24), some
// keys of the 32-key chunks the softmax reads (those below npad) are not real tokens
// and must be masked (25): a box with gaps, or a real-token count that is not a
// multiple of 32 (the S MMA writes npad columns; the rest of the last chunk is stale).
__device__ __forceinline__ uint32_t pack_blk(const Geo& g, int kb) {
  const BlkEnt e = blk_of(g, kb);
  const bool need_mask = !e.prefix || (e.nvalid & 31) != 0;
  return static_cast<uint32_t>(kb) | (static_cast<uint32_t>(e.npad >> 4) << 12) |
         (static_cast<uint32_t>(e.nvalid) << 16) | (e.prefix ? (1u << 24) : 0u) |
         (need_mask ? (1u << 25) : 0u);
}
__device__ __forceinline__ int blk_id(uint32_t e) { return static_cast<int>(e & 0xFFFu); }
__device__ __forceinline__ int blk_npad(uint32_t e) { return static_cast<int>((e >> 12) & 0xFu) << 4; }
__device__ __forceinline__ int blk_nvalid(uint32_t e) { return static_cast<int>((e >> 16) & 0xFFu); }
__device__ __forceinline__ bool blk_prefix(uint32_t e) { return (e >> 24) & 1u; }
__device__ __forceinline__ bool blk_needmask(uint32_t e) { return (e >> 25) & 1u; }

// The work items of a tile: each kept wide block on its own, then the narrow blocks
// (W-edge blocks whose box has rows_e = 16, 32 or 64 rows) in groups of up to
// pack = 128 / rows_e that share one 128-row K/V slot, one S and one P.V product.
// Sub-block s of a group occupies rows [s * rows_e, (s + 1) * rows_e) of the slot.
struct ItemRange {
  int first, cnt;
};
__device__ __forceinline__ int num_items(int nw, int nn, int pack) { return nw + (nn + pack - 1) / pack; }
__device__ __forceinline__ ItemRange item_range(int i, int nw, int nn, int pack) {
  if (i < nw) return ItemRange{i, 1};
  const int k = i - nw;
  return ItemRange{nw + k * pack, min(pack, nn - k * pack)};
}
__device__ __forceinline__ int item_npad(const uint32_t* bl, int i, int nw, const ItemRange& r, int rows_e) {
  return i < nw ? blk_npad(bl[i]) : r.cnt * rows_e;
}
__device__ __forceinline__ uint32_t range_bits(int lo, int hi, int base) {
  const int a = min(max(lo - base, 0), 32), b = min(max(hi - base, 0), 32);
  const uint32_t hib = b >= 32 ? 0xffffffffu : ((1u << b) - 1u);
  const uint32_t lob = a >= 32 ? 0xffffffffu : ((1u << a) - 1u);
  return hib & ~lob;
}

// Query groups: when qg > 1, the narrow (W-edge) query blocks of a slice are taken qg at
// a time, in ascending order, as one tile.  Query block s of a group fills rows
// [s * rows_e, (s + 1) * rows_e) of the 128-row tile (lane quarters s * qps, ...).  The
// tile's list is the union of the members' kept blocks; each member's own mask row is
// kept next to the list, and a member's warps skip the items it does not keep.  The
// tile is named by its first query block; the others are not tiles of their own.
__host__ __device__ inline bool q_narrow(const Geo& g, int qb) { return (qb % g.nBx) == g.nBx - 1; }
__host__ __device__ inline int q_group_cnt(const Geo& g, int qb, int qg) {
  if (qg <= 1 || !q_narrow(g, qb)) return 1;
  const int r = qb / g.nBx, rows = g.nBt * g.nBy;
  return min(qg, rows - r);
}
__host__ __device__ inline bool q_member_only(const Geo& g, int qb, int qg) {
  return qg > 1 && q_narrow(g, qb) && ((qb / g.nBx) % qg) != 0;
}
__host__ inline int query_group_size(const Geo& g) {
  const int rx_e = g.Ws - (g.nBx - 1) * g.bw, rows_e = g.bt * g.bh * rx_e;
  const bool ok = rx_e < g.bw && (rows_e == 32 || rows_e == 64) && (g.bt == 1 || g.Hs % g.bh == 0);
  return ok ? 128 / rows_e : 1;
}

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
  extern __shared__ __align__(1024) unsigned char attn_dsm[];
  AttnBars& bars = *reinterpret_cast<AttnBars*>(attn_dsm + TILE * (1 + kNK + kNV));

  const uint64_t t_start = globaltimer();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Geo& g = prm.g;
  uint32_t* err = prm.hdr + 1;
  volatile int* abort = &bars.abort;

  // 1024-byte aligned operand area: Q | K ring | V ring
  const uint32_t base = smem_u32(attn_dsm);
  if (base & 1023u) {                      // uniform over the CTA: nothing launched yet
    if (threadIdx.x == 0) atomicOr(err, kErrLayout);
    return;
  }
  unsigned char* gbase = attn_dsm;
  const uint32_t sQ = base;
  auto sK = [&](int s) { return base + static_cast<uint32_t>(TILE * (1 + s)); };
  auto sV = [&](int s) { return base + static_cast<uint32_t>(TILE * (1 + kNK + s)); };

  if (threadIdx.x == 0) {
    mbar_init(&bars.q_full, 1);
    mbar_init(&bars.q_empty, 1);
    for (int i = 0; i < kNK; ++i) { mbar_init(&bars.k_full[i], 1); mbar_init(&bars.k_empty[i], 1); }
    for (int i = 0; i < kNV; ++i) { mbar_init(&bars.v_full[i], 1); mbar_init(&bars.v_empty[i], 1); }
    for (int i = 0; i < kNS; ++i) {
      mbar_init(&bars.s_full[i], 1);
      mbar_init(&bars.p_full[i], kSoftWarps / 2);
    }
    for (int i = 0; i < kPV; ++i) mbar_init(&bars.pv_done[i], 1);
    for (int i = 0; i < 4; ++i) {
      mbar_init(&bars.xbar[i], 2);
      mbar_init(&bars.xread[i], 2);
      mbar_init(&bars.hb[0][i], 1);
      mbar_init(&bars.hb[1][i], 1);
    }
    mbar_init(&bars.o_empty, kSoftWarps);
    for (int i = 0; i < kTR; ++i) { mbar_init(&bars.t_full[i], 1); mbar_init(&bars.t_empty[i], 3 + kSoftWarps); }
    mbar_init(&bars.fin[0], 1);
    mbar_init(&bars.fin[1], 1);
    mbar_init(&bars.never, 1);
    bars.abort = 0;
    fence_barrier_init();
  }
  // Which blocks are packed narrow blocks: the last block column, when packing is on.
  for (int w = threadIdx.x; w < kMaxBlocks / 32; w += kAttnThreads) {
    uint32_t bits = 0;
    if (prm.pack > 1 && w < g.words) {
      for (int i = 0; i < 32; ++i) {
        const int j = w * 32 + i;
        if (j < g.nB && (j % g.nBx) == g.nBx - 1) bits |= 1u << i;
      }
    }
    bars.edgew[w] = bits;
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

  if (warp < 4) {
   asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsCtl));
   // The producer and MMA warps run their loops with all 32 lanes converged, so that
   // tile ids, coordinates and descriptors are warp-uniform; one elected lane issues
   // each TMA copy, MMA and commit.
   auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
     return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, err));
   };
   if (warp == 0) {
    // ------------------------------------------------------------ tile queue, Q and K
    // Takes the next tile, publishes it with its kept-block list (all 32 lanes: each
    // lane expands two mask words, placed by a popcount scan), then loads Q and the K
    // tiles.  V has its own loader (warp 3) so that the K ring never waits on a P.V.
    uint32_t tcount = 0;
    bool ok = true;
    // work tiles in the order (grouped narrow query blocks count once), from the prep
    const int nwork = *reinterpret_cast<volatile const int*>(prm.hdr + 2);
    while (ok) {
      int pos = 0;
      if (lane == 0) pos = static_cast<int>(atomicAdd(prm.hdr, 1u));
      pos = __shfl_sync(0xffffffffu, pos, 0);
      const int tile = pos < nwork ? __ldg(prm.order + pos) : -1;
      const int slot = tcount % kTR;
      if (!wwait(&bars.t_empty[slot], ((tcount / kTR) & 1) ^ 1)) break;
      int nw = 0, nn = 0;
      if (tile >= 0) {
        uint32_t* bl = bars.blist[slot];
        // the tile's members (1, or a query group): the list is the union of their kept
        // blocks; the members' own mask rows go to gmask for the softmax warps
        const int gcnt = q_group_cnt(g, tile - (tile / g.nB) * g.nB, prm.qg);
        const int tail = g.nB & 31;
        // bits of the last word at or past nB: cleared, so that no id past the last block
        // reaches the list (fvattn_route never sets them; a caller's mask might)
        const uint32_t last = tail ? (1u << tail) - 1u : 0xffffffffu;
        uint32_t w0 = 0u, w1 = 0u;
#pragma unroll 1
        for (int s4 = 0; s4 < 4; ++s4) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int w = lane + 32 * h;
            uint32_t m = 0u;
            if (s4 < gcnt && w < g.words) {
              m = (prm.mask != nullptr ? __ldg(prm.mask + static_cast<size_t>(tile + s4 * g.nBx) * g.words + w)
                                       : 0xffffffffu) &
                  (w < g.words - 1 ? 0xffffffffu : last);
            }
            bars.gmask[slot][s4][w] = m;
            if (h == 0) w0 |= m; else w1 |= m;
          }
        }
        const uint32_t n0 = w0 & bars.edgew[lane], n1 = w1 & bars.edgew[lane + 32];
        const uint32_t d0 = w0 & ~n0, d1 = w1 & ~n1;
        int i0 = __popc(d0), i1 = __popc(d1), j0 = __popc(n0), j1 = __popc(n1);
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int a0 = __shfl_up_sync(0xffffffffu, i0, o), a1 = __shfl_up_sync(0xffffffffu, i1, o);
          const int b0 = __shfl_up_sync(0xffffffffu, j0, o), b1 = __shfl_up_sync(0xffffffffu, j1, o);
          if (lane >= o) { i0 += a0; i1 += a1; j0 += b0; j1 += b1; }
        }
        const int tw0 = __shfl_sync(0xffffffffu, i0, 31), tn0 = __shfl_sync(0xffffffffu, j0, 31);
        nw = tw0 + __shfl_sync(0xffffffffu, i1, 31);
        nn = tn0 + __shfl_sync(0xffffffffu, j1, 31);
        int p0 = i0 - __popc(d0), p1 = tw0 + i1 - __popc(d1);
        int q0 = nw + j0 - __popc(n0), q1 = nw + tn0 + j1 - __popc(n1);
        // one placement loop over the four (word, kind) sets keeps a single copy of pack_blk
#pragma unroll 1
        for (int set = 0; set < 4; ++set) {
          uint32_t bits = set == 0 ? d0 : (set == 1 ? d1 : (set == 2 ? n0 : n1));
          const int wbase = ((set & 1) ? lane + 32 : lane) * 32;
          int pos = set == 0 ? p0 : (set == 1 ? p1 : (set == 2 ? q0 : q1));
          for (; bits; bits &= bits - 1) bl[pos++] = pack_blk(g, wbase + __ffs(bits) - 1);
        }
      }
      __syncwarp();
      if (lane == 0) {
        bars.tile[slot] = tile;
        bars.bcount[slot] = nw;
        bars.ncount[slot] = nn;
        mbar_arrive(&bars.t_full[slot]);
      }
      __syncwarp();
      ++tcount;
      if (tile < 0) break;
      int bhi, qb;
      decode_tile(g, tile, bhi, qb);
      const int gq = prm.qg > 1 && q_narrow(g, qb) ? q_group_cnt(g, qb, prm.qg) : 0;   // 0: not a group
      if (!wwait(&bars.q_empty, (qc & 1) ^ 1)) break;
      if (elect_one()) {
        const BlockInfo qi0 = block_info(g, qb);
        mbar_arrive_expect_tx(&bars.q_full, static_cast<uint32_t>(qi0.rows * 128 * NCH * (gq > 0 ? gq : 1)));
#pragma unroll 1
        for (int s4 = 0; s4 < (gq > 0 ? gq : 1); ++s4) {
          const BlockInfo qi = block_info(g, qb + s4 * g.nBx);
          const uint32_t off = static_cast<uint32_t>(s4 * prm.rows_e * 128);
#pragma unroll 1
          for (int c = 0; c < NCH; ++c)
            tma_load_5d(sQ + c * kChunkBytes + off, qi.xedge ? &tmQe : &tmQ, &bars.q_full, c * 64,
                        qi.xb * g.bw, qi.yb * g.bh, qi.tb * g.bt, bhi);
        }
      }
      __syncwarp();
      ++qc;
      const int full_rows = g.bt * g.bh * g.bw;
      const int nitems = num_items(nw, nn, prm.pack);
      for (int n = 0; n < nitems; ++n) {
        const ItemRange ir = item_range(n, nw, nn, prm.pack);
        const int ks = kc % kNK;
        if (!wwait(&bars.k_empty[ks], ((kc / kNK) & 1) ^ 1)) { ok = false; break; }
        if (elect_one()) {
          // every box of an item has the same rows (a wide block, or narrow blocks)
          const uint32_t rows0 = blk_of(g, blk_id(bars.blist[slot][ir.first])).rows;
          mbar_arrive_expect_tx(&bars.k_full[ks], rows0 * 128 * NCH * ir.cnt);
#pragma unroll 1
          for (int sb = 0; sb < ir.cnt; ++sb) {
            const BlkEnt ki = blk_of(g, blk_id(bars.blist[slot][ir.first + sb]));
            const bool xedge = ki.rows != full_rows;
            const uint32_t off = static_cast<uint32_t>(sb * prm.rows_e * 128);
#pragma unroll 1
            for (int c = 0; c < NCH; ++c)
              tma_load_5d(sK(ks) + c * kChunkBytes + off, xedge ? &tmKe : &tmK, &bars.k_full[ks],
                          c * 64, ki.x0, ki.y0, ki.t0, bhi);
          }
        }
        __syncwarp();
        ++kc;
      }
    }
   } else if (warp == 3) {
    // ------------------------------------------------------------ V loader
    uint32_t tcount = 0;
    bool ok = true;
    while (ok) {
      const int slot = tcount % kTR;
      if (!wwait(&bars.t_full[slot], (tcount / kTR) & 1)) break;
      const int tile = bars.tile[slot];
      const int nw = bars.bcount[slot], nn = bars.ncount[slot];
      ++tcount;
      if (tile < 0) break;
      int bhi, qb;
      decode_tile(g, tile, bhi, qb);
      const int full_rows = g.bt * g.bh * g.bw;
      const int nitems = num_items(nw, nn, prm.pack);
      for (int n = 0; n < nitems; ++n) {
        const ItemRange ir = item_range(n, nw, nn, prm.pack);
        const int vs = vc % kNV;
        if (!wwait(&bars.v_empty[vs], ((vc / kNV) & 1) ^ 1)) { ok = false; break; }
        if (elect_one()) {
          // every box of an item has the same rows (a wide block, or narrow blocks)
          const uint32_t rows0 = blk_of(g, blk_id(bars.blist[slot][ir.first])).rows;
          mbar_arrive_expect_tx(&bars.v_full[vs], rows0 * 128 * NCH * ir.cnt);
#pragma unroll 1
          for (int sb = 0; sb < ir.cnt; ++sb) {
            const BlkEnt ki = blk_of(g, blk_id(bars.blist[slot][ir.first + sb]));
            const bool xedge = ki.rows != full_rows;
            const uint32_t off = static_cast<uint32_t>(sb * prm.rows_e * 128);
#pragma unroll 1
            for (int c = 0; c < NCH; ++c)
              tma_load_5d(sV(vs) + c * kChunkBytes + off, xedge ? &tmVe : &tmV, &bars.v_full[vs],
                          c * 64, ki.x0, ki.y0, ki.t0, bhi);
          }
        }
        __syncwarp();
        ++vc;
      }
      if (!ok) break;
      if (lane == 0) mbar_arrive(&bars.t_empty[slot]);   // done with the tile's block list
    }
   } else if (warp == 1) {
    // ------------------------------------------------------------ S issuer
    // Block j of the call's running block count c: S_c = Q K_c^T into S slot c mod kNS,
    // once P.V c-kNS has read P_c-kNS out of it.  The S and the P.V products come
    // from two warps: an MMA issue blocks while the tensor core's queue is full, so one
    // warp's waits and bookkeeping overlap the other warp's issue.
    uint32_t tcount = 0, mqc = 0;
    uint32_t gc = 0;                      // blocks of all tiles so far: ring position
    const uint64_t dQ = sdesc_sw128(sQ, 16, 1024);
    const uint64_t dK0 = sdesc_sw128(sK(0), 16, 1024);
    bool ok = true;
    while (ok) {
      const int slot = tcount % kTR;
      if (!wwait(&bars.t_full[slot], (tcount / kTR) & 1)) break;
      const int tile = bars.tile[slot];
      ++tcount;
      if (tile < 0) break;
      const int nw = bars.bcount[slot], nn = bars.ncount[slot];
      const int nitems = num_items(nw, nn, prm.pack);
      if (!wwait(&bars.q_full, mqc & 1)) break;
      ++mqc;
      if (prm.stall_ns != 0ull && tcount == 1 &&
          !__all_sync(0xffffffffu, mbar_wait(&bars.never, 0, abort, err, prm.stall_ns)))
        break;   // the wait gives up (it always does): the CTA aborts and drains
      int n = 0;
      for (; n < nitems; ++n) {
        const uint32_t c = gc + n;
        const int ss = c % kNS;
        const int ks = c % kNK;
        const ItemRange ir = item_range(n, nw, nn, prm.pack);
        const uint32_t idesc_s = idesc_bf16_f32(128, item_npad(bars.blist[slot], n, nw, ir, prm.rows_e), 0, 0);
        if (!wwait(&bars.k_full[ks], (c / kNK) & 1)) { ok = false; break; }
        if (c >= kNS && !wwait(&bars.pv_done[(c - kNS) % kPV], ((c - kNS) / kPV) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint64_t dK = dK0 + static_cast<uint64_t>((ks * TILE) >> 4);
        const uint32_t tS = tmem + kColS + ss * 128;
        if (elect_one()) {
#pragma unroll
          for (int q = 0; q < D / 16; ++q) {
            const uint64_t off = static_cast<uint64_t>(((q >> 2) * kChunkBytes + (q & 3) * 32) >> 4);
            mma_ss(tS, dQ + off, dK + off, idesc_s, q > 0 ? 1u : 0u);
          }
          mma_commit(&bars.s_full[ss]);
          mma_commit(&bars.k_empty[ks]);
        }
        __syncwarp();
      }
      if (!ok) break;
      gc += n;
      if (elect_one()) mma_commit(&bars.q_empty);      // the tile's last S has read Q
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.t_empty[slot]);   // done with the tile's mask row
    }
   } else if (warp == 2) {
    // ------------------------------------------------------------ P.V issuer
    // O += P_c V_c in block order (one accumulator), P_c from S slot c mod kNS.
    uint32_t tcount = 0, tiles = 0;
    uint32_t gc = 0;
    const uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
    const uint64_t dV0 = sdesc_sw128(sV(0), kChunkBytes, 1024);
    bool ok = true;
    while (ok) {
      const int slot = tcount % kTR;
      if (!wwait(&bars.t_full[slot], (tcount / kTR) & 1)) break;
      const int tile = bars.tile[slot];
      const int nw = bars.bcount[slot], nn = bars.ncount[slot];
      const int nitems = num_items(nw, nn, prm.pack);
      ++tcount;
      if (tile < 0) break;
      int n = 0;
      for (; n < nitems; ++n) {
        const uint32_t c = gc + n;
        const int ps = c % kNS;
        const int vs = c % kNV;
        const int nk = item_npad(bars.blist[slot], n, nw, item_range(n, nw, nn, prm.pack), prm.rows_e) >> 4;
        if (!wwait(&bars.p_full[ps], (c / kNS) & 1)) { ok = false; break; }
        if (!wwait(&bars.v_full[vs], (c / kNV) & 1)) { ok = false; break; }
        if (n == 0 && !wwait(&bars.o_empty, (tiles & 1) ^ 1)) { ok = false; break; }
        tc_fence_after();
        const uint64_t dV = dV0 + static_cast<uint64_t>((vs * TILE) >> 4);
        const uint32_t tP = tmem + kColS + ps * 128;
        if (elect_one()) {
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            if (q < nk)
              mma_ts(tmem + kColO, tP + q * 8, dV + static_cast<uint64_t>((q * 2048) >> 4), idesc_pv,
                     (n == 0 && q == 0) ? 0u : 1u);
          }
          mma_commit(&bars.v_empty[vs]);
          mma_commit(&bars.pv_done[c % kPV]);
        }
        __syncwarp();
      }
      if (!ok) break;
      gc += n;
      if (lane == 0) mbar_arrive(&bars.t_empty[slot]);
      ++tiles;
    }
   }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoft));
    // ------------------------------------------------------------ softmax + epilogue
    // Group grp = (w-4)/4 takes the tile's kept blocks j with j % 2 == grp.  One thread
    // per query row (TMEM lane 32*(w%4) + lane), the 128 key columns of a block in
    // registers.  Per row the running reference m_j (log2 units) is one value for the
    // whole tile: the group of block j takes m_j-1 from the other group (hv / hb, per
    // lane quarter), sets m_j and hands it on before its exponentials.  Each group
    // keeps its own row sum l against the reference of its latest block; at the end of
    // the tile the group that did not run the last block takes the final reference
    // from the other group's last hand-off, both rescale their l to it, exchange l
    // (xl / xbar / xread) and each writes half of the output columns.
    const int grp = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS0 = tmem + lane_off + kColS;
    const uint32_t tO = tmem + lane_off + kColO;
    uint32_t tcount = 0, xn = 0, hr = 0;
    uint32_t gc = 0;                    // blocks of all earlier tiles: S ring position
    const float sl2 = prm.scale_log2;
    const uint64_t sl2x2 = f32x2(sl2, sl2);
    auto sync_wait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, err));
    };
    while (true) {
      const int slot = tcount % kTR;
      if (!sync_wait(&bars.t_full[slot], (tcount / kTR) & 1)) break;
      const int tile = bars.tile[slot];
      ++tcount;
      if (tile < 0) break;
      int bhi, qb;
      decode_tile(g, tile, bhi, qb);
      // in a query group this warp's rows belong to member `sub` (none past the group)
      const bool qgrp = prm.qg > 1 && q_narrow(g, qb);
      const int sub = qgrp ? quarter / prm.qps : 0;
      const int gcnt = qgrp ? q_group_cnt(g, qb, prm.qg) : 1;
      const uint32_t* gm = bars.gmask[slot][qgrp && sub < 4 ? sub : 0];
      int token = -1;
      if (sub < gcnt) {
        const BlockInfo qi = block_info(g, qb + sub * g.nBx);
        token = box_row_token(g, qi, qgrp ? row - sub * prm.rows_e : row);
      }

      float m = -INFINITY, l = 0.f;     // this group's latest reference and its row sum
      const int nw = bars.bcount[slot], nn = bars.ncount[slot];
      const int nkv = num_items(nw, nn, prm.pack);
      const uint32_t* bl = bars.blist[slot];
      bool ok = true;
      for (int j = grp; j < nkv; j += 2) {
        const ItemRange ir = item_range(j, nw, nn, prm.pack);
        const uint32_t e = bl[ir.first];
        const uint32_t c = gc + j;
        const int ss = c % kNS;
        const uint32_t tS = tS0 + ss * 128;
        const uint32_t tP = tS;                     // P_c goes over S_c
        const int npad = item_npad(bl, j, nw, ir, prm.rows_e);
        const int nact = (npad + 31) >> 5;          // 32-column chunks below npad (uniform)
        // member: this warp's query block keeps the item (some sub-block of a packed item)
        auto kept = [&](uint32_t es) -> bool {
          const int kb = blk_id(es);
          return !qgrp || (sub < gcnt && ((gm[kb >> 5] >> (kb & 31)) & 1u));
        };
        bool need_mask = blk_needmask(e);
        bool member = kept(e);
        if (j >= nw) {
          need_mask = (npad & 31) != 0;
          member = false;
#pragma unroll 1
          for (int sb = 0; sb < ir.cnt; ++sb) {
            const uint32_t es = bl[ir.first + sb];
            const bool k = kept(es);
            need_mask |= blk_nvalid(es) < prm.rows_e || !k;
            member |= k;
          }
        }
        if (!sync_wait(&bars.s_full[ss], (c / kNS) & 1)) { ok = false; break; }
        tc_fence_after();
        // The whole row of S in one TMEM round trip (loads are grouped, then one wait).  A
        // warp whose query block does not keep the item takes no part in it: P = 0 for its
        // rows, and its reference carries over unchanged.
        float s[128];
        if (member) {
#pragma unroll
          for (int q = 0; q < 4; ++q) tmem_ld32(tS + 32 * q, reinterpret_cast<uint32_t*>(s + 32 * q));
          tmem_wait_ld();
        }
        tc_fence_before();
        __syncwarp();
        // Keys that are not real tokens (a partial last 16-key group, or the gaps of a box
        // cut at the time and height edges at once) to -inf.  One warp-uniform branch,
        // taken only by such blocks, so the common path carries none of this code.
        if (member && need_mask) {
          uint32_t vm[4];
          if (j >= nw) {
#pragma unroll
            for (int w4 = 0; w4 < 4; ++w4) vm[w4] = 0u;
#pragma unroll 1
            for (int sb = 0; sb < ir.cnt; ++sb) {
              const uint32_t es = bl[ir.first + sb];
              const int lo = sb * prm.rows_e, hi = lo + (kept(es) ? blk_nvalid(es) : 0);
#pragma unroll
              for (int w4 = 0; w4 < 4; ++w4) vm[w4] |= range_bits(lo, hi, 32 * w4);
            }
          } else if (blk_prefix(e)) {
            const int nvalid = blk_nvalid(e);
#pragma unroll
            for (int w4 = 0; w4 < 4; ++w4) {
              const int nn = nvalid - 32 * w4;
              vm[w4] = nn >= 32 ? 0xffffffffu : (nn <= 0 ? 0u : ((1u << nn) - 1u));
            }
          } else {
            const BlockInfo bi = block_info(g, blk_id(e));
#pragma unroll
            for (int w4 = 0; w4 < 4; ++w4)
              vm[w4] = __ballot_sync(0xffffffffu, box_row_token(g, bi, 32 * w4 + lane) >= 0);
          }
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            if (r < nact && vm[r] != 0xffffffffu) {
#pragma unroll
              for (int q = 0; q < 32; ++q)
                s[32 * r + q] = ((vm[r] >> q) & 1u) ? s[32 * r + q] : -INFINITY;
            }
          }
        }
        // Row maximum of each chunk as a shallow tree (depth 4 instead of a 16-long chain).
        float mx = -INFINITY;
        if (member) {
          float mq[4];
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const float* x = s + 32 * r;
            float t[11];
#pragma unroll
            for (int k = 0; k < 10; ++k) t[k] = max3f(x[3 * k], x[3 * k + 1], x[3 * k + 2]);
            t[10] = fmaxf(x[30], x[31]);
            const float u0 = max3f(t[0], t[1], t[2]), u1 = max3f(t[3], t[4], t[5]);
            const float u2 = max3f(t[6], t[7], t[8]), u3 = max3f(t[9], t[10], u0);
            mq[r] = r < nact ? max3f(u1, u2, u3) : -INFINITY;
          }
          mx = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3])) * sl2;
        }
        // reference after block j-1, from the other group
        float mref = mx, mp = mx;
        bool rebase = false;
        if (j > 0) {
          if (!sync_wait(&bars.hb[grp ^ 1][quarter], hr & 1)) { ok = false; break; }
          ++hr;
          mp = bars.hv[grp ^ 1][row];
          rebase = mx > mp + kRebase;
          mref = rebase ? mx : mp;
        }
        bars.hv[grp][row] = mref;
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.hb[grp][quarter]);
        // O holds P_0 V_0 + ... + P_j-1 V_j-1 against the old reference once P.V j-1
        // has finished; re-base it before P_j goes in.
        if (__any_sync(0xffffffffu, rebase)) {
          const float alpha = rebase ? ex2(mp - mx) : 1.f;
          const uint32_t cp = c - 1;
          if (!sync_wait(&bars.pv_done[cp % kPV], (cp / kPV) & 1)) { ok = false; break; }
          tc_fence_after();
#pragma unroll 1
          for (int q = 0; q < D / 32; ++q) {
            uint32_t o[32];
            tmem_ld32(tO + 32 * q, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(tO + 32 * q, o);
          }
        }
        // this group's row sum follows the reference (unchanged unless a group re-based;
        // l is still 0 before the group's first block of the tile)
        const bool lscale = mref != m && m != -INFINITY;
        if (__any_sync(0xffffffffu, lscale)) {
          if (lscale) l *= ex2(m - mref);
        }
        m = mref;
        // P = 2^(s * scale * log2 e - m), packed to bf16 pairs and stored 16 keys at a
        // time (P column k/2 holds keys k, k+1).  Chunks at or past npad are neither
        // computed nor stored: the P.V reads keys < npad only.
        const uint64_t nmx2 = f32x2(-m, -m);
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
        if (!member) {
          const uint32_t zero8[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll 1
          for (int h = 0; h < 2 * nact; ++h) tmem_st8(tP + 8 * h, zero8);
        }
#pragma unroll
        for (int c32 = 0; c32 < 4; ++c32) {
          if (member && c32 < nact) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              uint32_t pk[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const int q = 32 * c32 + 16 * h + 2 * e;
                float x0, x1;
                unpack_f32x2(ffma2(f32x2(s[q], s[q + 1]), sl2x2, nmx2), x0, x1);
                const float p0 = ex2(x0), p1 = ex2(x1);
                acc[e & 3] = fadd2(acc[e & 3], f32x2(p0, p1));
                pk[e] = pack_bf16x2(p0, p1);
              }
              tmem_st8(tP + 16 * c32 + 8 * h, pk);
            }
          }
        }
        float sa, sb, sc2, sd;
        unpack_f32x2(fadd2(acc[0], acc[1]), sa, sb);
        unpack_f32x2(fadd2(acc[2], acc[3]), sc2, sd);
        l += (sa + sb) + (sc2 + sd);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.p_full[c % kNS]);
      }
      if (!ok) break;
      // ---- epilogue
      gc += nkv;
      float mf = m;                      // final reference of the tile
      if (nkv > 0 && ((nkv - 1) & 1) != grp) {
        if (!sync_wait(&bars.hb[grp ^ 1][quarter], hr & 1)) break;
        ++hr;
        mf = bars.hv[grp ^ 1][row];
      }
      if (mf != m) l = (m == -INFINITY) ? 0.f : l * ex2(m - mf);
      if (nkv > 0) {
        const uint32_t cl = gc - 1;      // the tile's last P.V
        if (!sync_wait(&bars.pv_done[cl % kPV], (cl / kPV) & 1)) break;
      }
      if (xn > 0 && !sync_wait(&bars.xread[quarter], (xn - 1) & 1)) break;
      bars.xl[grp][row] = l;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.xbar[quarter]);
      if (!sync_wait(&bars.xbar[quarter], xn & 1)) break;
      const float lt = l + bars.xl[grp ^ 1][row];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.xread[quarter]);
      ++xn;
      // a row whose kept set is empty (possible only with a caller's mask that keeps no
      // block for it) has lt = 0: its out is written as zeros and its lse is -inf
      const bool empty = !(lt > 0.f);
      const float inv = 1.f / lt;
      tc_fence_after();
      uint4* dst = reinterpret_cast<uint4*>(prm.out + (static_cast<size_t>(bhi) * g.N + (token >= 0 ? token : 0)) * D +
                                            (D / 2) * grp);
#pragma unroll
      for (int q = 0; q < D / 64; ++q) {
        uint32_t o[32];
        tmem_ld32(tO + (D / 2) * grp + 32 * q, o);
        tmem_wait_ld();
        if (token >= 0) {
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            uint4 wv;
            wv.x = pack_bf16x2(__uint_as_float(o[8 * q8 + 0]) * inv, __uint_as_float(o[8 * q8 + 1]) * inv);
            wv.y = pack_bf16x2(__uint_as_float(o[8 * q8 + 2]) * inv, __uint_as_float(o[8 * q8 + 3]) * inv);
            wv.z = pack_bf16x2(__uint_as_float(o[8 * q8 + 4]) * inv, __uint_as_float(o[8 * q8 + 5]) * inv);
            wv.w = pack_bf16x2(__uint_as_float(o[8 * q8 + 6]) * inv, __uint_as_float(o[8 * q8 + 7]) * inv);
            if (empty) wv = make_uint4(0u, 0u, 0u, 0u);   // the tensor memory may hold stale values
            dst[4 * q + q8] = wv;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bars.o_empty);
        mbar_arrive(&bars.t_empty[slot]);   // done with the tile's mask row
      }
      if (token >= 0 && grp == 0)
        prm.lse[static_cast<size_t>(bhi) * g.N + token] = (mf + __log2f(lt)) * 0.69314718055994531f;
    }
  }

  // ------------------------------------------------------------ teardown
  __syncthreads();
  if (bars.abort) {
    // Drain: let every armed TMA copy land and every issued MMA finish before the
    // shared and tensor memory they touch is released.  Bounded, abort ignored.
    if ((warp == 0 || warp == 3) && lane == 0) {   // each loader's copies (Q, K / V)
      int never = 0;
      volatile int* nv = &never;
      if (qc > 0) mbar_wait(&bars.q_full, (qc - 1) & 1, nv, nullptr, 100000000ull);
      for (uint32_t i = (kc > kNK ? kc - kNK : 0); i < kc; ++i)
        mbar_wait(&bars.k_full[i % kNK], (i / kNK) & 1, nv, nullptr, 100000000ull);
      for (uint32_t i = (vc > kNV ? vc - kNV : 0); i < vc; ++i)
        mbar_wait(&bars.v_full[i % kNV], (i / kNV) & 1, nv, nullptr, 100000000ull);
    }
    if ((warp == 1 || warp == 2) && lane == 0) {   // each issuer's MMAs
      int never = 0;
      volatile int* nv = &never;
      mma_commit(&bars.fin[warp - 1]);
      mbar_wait(&bars.fin[warp - 1], 0, nv, nullptr, 100000000ull);
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
// Schedule prep, two kernels.
//
// prep_cost_kernel (one warp per tile, many CTAs): a tile's cost is its issued work,
// the sum over its kept blocks of (keys the MMAs read + a per-block overhead).  Blocks
// are classed by whether they sit in the last block column, row and frame (8 classes;
// the caller passes each class's cost, read off the block geometry), so a mask word
// costs eight popcounts.
//
// prep_order_kernel (one CTA): resets the queue counter, the error word and the SM busy
// record, then writes the tile order:
//   * (b, h) slices are ranked by total cost, heaviest first, and a slice's tiles are
//     contiguous in the order, heaviest first (counting sort on cost buckets).
// Grouping by slice keeps the K/V tiles that concurrently running tiles read within a
// slice or two, which fits in L2; ordering slices and tiles by decreasing cost keeps
// the longest-processing-time-first tail (the last tiles are the lightest slice's
// lightest).  Order inside a bucket is arbitrary: it changes timing, never results.
// ----------------------------------------------------------------------------
constexpr int kPrepThreads = 1024;
constexpr int kCostWarps = 8;
constexpr int kHistCells = 8192;       // slices x cost buckets
constexpr int kMaxSlices = 1024;
constexpr int kBlockOverhead = 64;

struct ClassCost {
  int c[8];                            // cost of a block of class (x_edge | y_edge << 1 | t_edge << 2)
};

__global__ void __launch_bounds__(32 * kCostWarps) prep_cost_kernel(Geo g, const uint32_t* __restrict__ mask,
                                                                    int* cost_out, int ntiles, ClassCost cc,
                                                                    int qg) {
  __shared__ uint32_t edge[3][kMaxBlocks / 32];   // per word: last column / row / frame bits
  for (int w = threadIdx.x; w < g.words; w += 32 * kCostWarps) {
    uint32_t ex = 0, ey = 0, et = 0;
    for (int i = 0; i < 32; ++i) {
      const int j = w * 32 + i;
      if (j >= g.nB) break;
      const int xb = j % g.nBx, r = j / g.nBx;
      const int yb = r % g.nBy, tb = r / g.nBy;
      ex |= (xb == g.nBx - 1 ? 1u : 0u) << i;
      ey |= (yb == g.nBy - 1 ? 1u : 0u) << i;
      et |= (tb == g.nBt - 1 ? 1u : 0u) << i;
    }
    edge[0][w] = ex;
    edge[1][w] = ey;
    edge[2][w] = et;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int warp = blockIdx.x * kCostWarps + (threadIdx.x >> 5);
  for (int tile = warp; tile < ntiles; tile += gridDim.x * kCostWarps) {
    // a query group is one tile (its first member), costed by the union of its masks;
    // the other members get cost -1 and are left out of the order
    const int qb = tile - (tile / g.nB) * g.nB;
    if (q_member_only(g, qb, qg)) {
      if (lane == 0) cost_out[tile] = -1;
      continue;
    }
    const int gcnt = q_group_cnt(g, qb, qg);
    const uint32_t* row = mask + static_cast<size_t>(tile) * g.words;
    const int tail = g.nB & 31;
    int cost = 0;
    for (int w = lane; w < g.words; w += 32) {
      uint32_t m = 0u;
      for (int s4 = 0; s4 < gcnt; ++s4) m |= __ldg(row + static_cast<size_t>(s4) * g.nBx * g.words + w);
      if (w == g.words - 1 && tail) m &= (1u << tail) - 1u;   // no block at or past nB
      const uint32_t ex = edge[0][w], ey = edge[1][w], et = edge[2][w];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t sel = ((k & 1) ? ex : ~ex) & ((k & 2) ? ey : ~ey) & ((k & 4) ? et : ~et);
        cost += cc.c[k] * __popc(m & sel);
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) cost += __shfl_xor_sync(0xffffffffu, cost, off);
    if (lane == 0) cost_out[tile] = cost;
  }
}

__global__ void __launch_bounds__(kPrepThreads) prep_order_kernel(Geo g, const uint32_t* __restrict__ mask,
                                                                  uint32_t* hdr, int* order, int* keys,
                                                                  int ntiles, int maxcost,
                                                                  unsigned long long* busy, int nsm, int qg) {
  __shared__ int hist[kHistCells];
  __shared__ unsigned long long total[kMaxSlices];
  __shared__ int rank[kMaxSlices];
  __shared__ int nwork;
  const int t = threadIdx.x;
  if (t == 0) { hdr[0] = 0; hdr[1] = 0; nwork = 0; }
  if (busy)
    for (int i = t; i < nsm; i += kPrepThreads) busy[i] = 0ull;
  __syncthreads();
  if (mask == nullptr) {
    // every tile but the non-first members of query groups, in any order
    for (int i0 = 0; i0 < ntiles; i0 += kPrepThreads) {
      const int i = i0 + t;
      const bool v = i < ntiles && !q_member_only(g, i - (i / g.nB) * g.nB, qg);
      const uint32_t bal = __ballot_sync(0xffffffffu, v);
      int base = 0;
      if ((t & 31) == 0 && bal) base = atomicAdd(&nwork, __popc(bal));
      base = __shfl_sync(0xffffffffu, base, 0);
      if (v) order[base + __popc(bal & ((1u << (t & 31)) - 1u))] = i;
    }
    __syncthreads();
    if (t == 0) hdr[2] = static_cast<uint32_t>(nwork);
    return;
  }
  const int slices = g.B * g.H;
  // slices beyond the shared tables fall back to one group (plain LPT order)
  const bool grouped = slices <= kMaxSlices;
  const int ngroups = grouped ? slices : 1;
  int nbk = kHistCells / ngroups;
  nbk = nbk >= 256 ? 256 : (nbk >= 128 ? 128 : (nbk >= 64 ? 64 : (nbk >= 32 ? 32 : (nbk >= 16 ? 16 : 8))));
  for (int i = t; i < kHistCells; i += kPrepThreads) hist[i] = 0;
  for (int i = t; i < ngroups; i += kPrepThreads) total[i] = 0ull;
  __syncthreads();
  // keys[] holds the tile costs on entry and the cost buckets on exit.  Shared-memory
  // atomics are aggregated per warp (lanes with the same slice or bucket combine first):
  // a warp's tiles are consecutive, so they mostly share a slice and many share a bucket.
  const int lane = t & 31;
  const int iters = (ntiles + kPrepThreads - 1) / kPrepThreads;
  for (int it = 0; it < iters; ++it) {
    const int i = it * kPrepThreads + t;
    const long long cost0 = i < ntiles ? keys[i] : -1;
    const bool valid = cost0 >= 0;                     // -1: a non-first query-group member
    const long long cost = valid ? cost0 : 0;
    if (valid) atomicAdd(&nwork, 1);
    int key = static_cast<int>(((maxcost - cost) * nbk) / (static_cast<long long>(maxcost) + 1));
    key = min(max(key, 0), nbk - 1);
    if (i < ntiles) keys[i] = valid ? key : -1;
    const int grp = valid ? (grouped ? i / g.nB : 0) : -1;
    // one warp reduction and one atomic per distinct slice among the warp's tiles
    uint32_t remaining = __ballot_sync(0xffffffffu, valid);
    while (remaining) {
      const int leader = __ffs(remaining) - 1;
      const int lg = __shfl_sync(0xffffffffu, grp, leader);
      const bool mine = valid && grp == lg;
      unsigned long long v = mine ? static_cast<unsigned long long>(cost) : 0ull;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      if (lane == leader) atomicAdd(&total[lg], v);
      remaining &= ~__ballot_sync(0xffffffffu, mine);
    }
  }
  __syncthreads();
  for (int h = t; h < ngroups; h += kPrepThreads) {
    int r = 0;
    const unsigned long long th = total[h];
    for (int o = 0; o < ngroups; ++o) {
      const unsigned long long to = total[o];
      r += (to > th) || (to == th && o < h);
    }
    rank[h] = r;
  }
  __syncthreads();
  for (int it = 0; it < iters; ++it) {
    const int i = it * kPrepThreads + t;
    const int key = i < ntiles ? keys[i] : -1;
    const int cell = key >= 0 ? rank[grouped ? i / g.nB : 0] * nbk + key : -1;
    const uint32_t peers = __match_any_sync(0xffffffffu, cell);
    if (cell >= 0 && lane == __ffs(peers) - 1) atomicAdd(&hist[cell], __popc(peers));
  }
  __syncthreads();
  // exclusive scan of the histogram in (slice rank, bucket) order over the whole block:
  // thread t owns `per` consecutive cells; warp scans, then a scan of the warp totals
  const int cells = ngroups * nbk;
  const int per = (cells + kPrepThreads - 1) / kPrepThreads;
  __shared__ int wsum[kPrepThreads / 32];
  int run = 0;
  for (int i = 0; i < per; ++i) {
    const int idx = t * per + i;
    if (idx < cells) run += hist[idx];
  }
  int incl = run;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) wsum[t >> 5] = incl;
  __syncthreads();
  if (t < 32) {
    const int w = wsum[t];
    int wi = w;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, wi, off);
      if (t >= off) wi += v;
    }
    wsum[t] = wi - w;   // exclusive prefix of the warp totals
  }
  __syncthreads();
  int acc = wsum[t >> 5] + incl - run;
  for (int i = 0; i < per; ++i) {
    const int idx = t * per + i;
    if (idx < cells) {
      const int c = hist[idx];
      hist[idx] = acc;
      acc += c;
    }
  }
  __syncthreads();
  for (int it = 0; it < iters; ++it) {
    const int i = it * kPrepThreads + t;
    const int key = i < ntiles ? keys[i] : -1;
    const int cell = key >= 0 ? rank[grouped ? i / g.nB : 0] * nbk + key : -1;
    const uint32_t peers = __match_any_sync(0xffffffffu, cell);
    const int leader = __ffs(peers) - 1;
    int base = 0;
    if (cell >= 0 && lane == leader) base = atomicAdd(&hist[cell], __popc(peers));
    base = __shfl_sync(peers, base, leader);
    if (cell >= 0) order[base + __popc(peers & ((1u << lane) - 1u))] = i;
  }
  if (t == 0) hdr[2] = static_cast<uint32_t>(nwork);
}

template <int D>
static cudaError_t launch_attn_d(const Geo& g, const AttnMaps& maps, const AttnParams& prm, int grid,
                                 cudaStream_t st) {
  constexpr int smem = attn_smem_bytes<D>();
  static SmemAttrCache attr_ctx = {};
  cudaError_t e = set_smem_once(reinterpret_cast<const void*>(attn_kernel<D>), smem, attr_ctx);
  if (e != cudaSuccess) return e;
  attn_kernel<D><<<grid, kAttnThreads, smem, st>>>(maps.q, maps.qe, maps.k, maps.ke, maps.v, maps.ve, prm);
  return cudaGetLastError();
}

cudaError_t launch_attn(const Geo& g, const AttnMaps& maps, const uint32_t* mask, float scale,
                        void* out, float* lse, void* ws, unsigned long long* busy, int nsm,
                        cudaStream_t st, unsigned long long stall_ns) {
  const int ntiles = g.B * g.H * g.nB;
  uint32_t* hdr = static_cast<uint32_t*>(ws);
  int* order = reinterpret_cast<int*>(static_cast<unsigned char*>(ws) + kWsHeader);
  int* keys = order + ntiles;
  int maxcost = 0;
  if (mask != nullptr) {
    // cost of each block class, from a block of that class (last column / row / frame)
    ClassCost cc;
    // a packed W-edge block costs its rows plus a 1/pack share of one item's overhead
    const int rx_e = g.Ws - (g.nBx - 1) * g.bw, rows_e = g.bt * g.bh * rx_e;
    const int pack = (rx_e < g.bw && (rows_e == 16 || rows_e == 32 || rows_e == 64) &&
                      (g.bt == 1 || g.Hs % g.bh == 0)) ? 128 / rows_e : 1;
    for (int k = 0; k < 8; ++k) {
      const int xb = (k & 1) ? g.nBx - 1 : 0, yb = (k & 2) ? g.nBy - 1 : 0, tb = (k & 4) ? g.nBt - 1 : 0;
      const BlockInfo bi = block_info(g, (tb * g.nBy + yb) * g.nBx + xb);
      cc.c[k] = (pack > 1 && (k & 1)) ? rows_e + kBlockOverhead / pack : bi.npad + kBlockOverhead;
      maxcost = cc.c[k] > maxcost ? cc.c[k] : maxcost;
    }
    maxcost *= g.nB;
    const int ctas = (ntiles + kCostWarps - 1) / kCostWarps;
    prep_cost_kernel<<<ctas, 32 * kCostWarps, 0, st>>>(g, mask, keys, ntiles, cc, query_group_size(g));
    cudaError_t e0 = cudaGetLastError();
    if (e0 != cudaSuccess) return e0;
  }
  prep_order_kernel<<<1, kPrepThreads, 0, st>>>(g, mask, hdr, order, keys, ntiles, maxcost, busy, nsm,
                                                query_group_size(g));
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
  prm.stall_ns = stall_ns;
  const int rx_edge = g.Ws - (g.nBx - 1) * g.bw;
  prm.rows_e = g.bt * g.bh * rx_edge;
  const bool narrow_ok = rx_edge < g.bw && (prm.rows_e == 16 || prm.rows_e == 32 || prm.rows_e == 64) &&
                         (g.bt == 1 || g.Hs % g.bh == 0);
  prm.pack = narrow_ok ? 128 / prm.rows_e : 1;
  prm.qg = query_group_size(g);
  prm.qps = prm.qg > 1 ? prm.rows_e / 32 : 1;
  const int grid = ntiles < nsm ? ntiles : nsm;
  return g.d == 128 ? launch_attn_d<128>(g, maps, prm, grid, st)
                    : launch_attn_d<64>(g, maps, prm, grid, st);
}

}  // namespace fv
