// Device helpers shared by the fvattn kernels: 3D block geometry, mbarrier / TMA /
// tcgen05 (5th-generation tensor core + tensor memory) wrappers in inline PTX for
// sm_100a, and bounded waits.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fvattn.h"

namespace fv {

// ----------------------------------------------------------------------------
// 3D block geometry (video-aware block organisation)
// ----------------------------------------------------------------------------
struct Geo {
  int B, H, T, Hs, Ws, d;
  int bt, bh, bw;
  int nBt, nBy, nBx, nB, words;
  int N;
  float r_nBx, r_plane;   // 1/nBx and 1/(nBy*nBx), for division by multiplication
};

// a / d for 0 <= a < 2^24, 0 < d < 2^16, given rd ~ 1/d: the float estimate is off by
// at most one, and one correction step makes it exact.
__host__ __device__ inline int div_r(int a, int d, float rd) {
#ifdef __CUDA_ARCH__
  int q = __float2int_rz(__int2float_rn(a) * rd);
#else
  int q = static_cast<int>(static_cast<float>(a) * rd);
#endif
  const int r = a - q * d;
  if (r < 0) --q;
  else if (r >= d) ++q;
  return q;
}

struct BlockInfo {
  int tb, yb, xb;    // block coordinates
  int rt, ry, rx;    // real extents (clipped to the latent)
  int rows;          // rows of the loaded box: bt * bh * rx (x is loaded compactly)
  int npad;          // rows the MMAs read, rounded up to 16 (MMA N / K granularity)
  int nvalid;        // when `prefix`: the real rows are exactly rows [0, nvalid)
  bool prefix;
  bool xedge;        // rx < bw: the block is loaded with the narrow tensor map
};

__host__ __device__ inline BlockInfo block_info(const Geo& g, int j) {
  BlockInfo b;
  const int per_t = g.nBy * g.nBx;
  b.tb = div_r(j, per_t, g.r_plane);
  const int rem = j - b.tb * per_t;
  b.yb = div_r(rem, g.nBx, g.r_nBx);
  b.xb = rem - b.yb * g.nBx;
  b.rt = min(g.bt, g.T - b.tb * g.bt);
  b.ry = min(g.bh, g.Hs - b.yb * g.bh);
  b.rx = min(g.bw, g.Ws - b.xb * g.bw);
  b.rows = g.bt * g.bh * b.rx;
  b.prefix = (g.bt == 1) || (b.ry == g.bh);
  b.nvalid = b.rt * b.ry * b.rx;   // the real token count (a prefix of the box when `prefix`)
  // Rows the MMAs use: when the real tokens are a prefix of the box, the rows past them
  // (zero fill at the latent's H or T edge) are left out of S and P.V altogether.
  b.npad = ((b.prefix ? b.nvalid : b.rows) + 15) & ~15;
  b.xedge = b.rx < g.bw;
  return b;
}

// What the attention roles need of key block j (TMA coordinates, rows, real tokens).
struct BlkEnt {
  int x0, y0, t0, rows, npad, nvalid;
  bool prefix;
};
__host__ __device__ inline BlkEnt blk_of(const Geo& g, int j) {
  const BlockInfo b = block_info(g, j);
  BlkEnt e;
  e.x0 = b.xb * g.bw;
  e.y0 = b.yb * g.bh;
  e.t0 = b.tb * g.bt;
  e.rows = b.rows;
  e.npad = b.npad;
  e.nvalid = b.nvalid;
  e.prefix = b.prefix;
  return e;
}

// Row r of a loaded box (rows ordered (tt, yy, xx), x compact) -> token index, or -1
// when r is not a real token.
__host__ __device__ inline int box_row_token(const Geo& g, const BlockInfo& b, int r) {
  if (r >= b.rows) return -1;
  const int plane = g.bh * b.rx;
  const int tt = r / plane;
  const int r2 = r - tt * plane;
  const int yy = r2 / b.rx;
  const int xx = r2 - yy * b.rx;
  if (tt >= b.rt || yy >= b.ry) return -1;
  return ((b.tb * g.bt + tt) * g.Hs + (b.yb * g.bh + yy)) * g.Ws + (b.xb * g.bw + xx);
}

// ----------------------------------------------------------------------------
// Shared-memory addresses, mbarriers
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smid() {
  uint32_t r;
  asm volatile("mov.u32 %0, %smid;" : "=r"(r));
  return r;
}

// True in exactly one lane of the (converged) warp.
__device__ __forceinline__ bool elect_one() {
  uint32_t pred;
  asm volatile(
      "{\n\t.reg .pred P;\n\telect.sync _|P, 0xffffffff;\n\tselp.u32 %0, 1, 0, P;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

// Status word bits written to the workspace when a kernel gives up a wait.
enum : uint32_t { kErrTimeout = 1u, kErrLayout = 2u };

// A bounded wait on an mbarrier phase.  Returns false (after raising *abort and the
// global error word) when the phase has not completed within about `limit_ns`, or when
// another thread of the CTA has already raised *abort.  The deadline is kept in SM
// cycles (clock64, counted at 2 cycles per ns so that it is never shorter than the
// limit at clocks up to 2 GHz) and starts only after 64 unsuccessful probes: the
// %globaltimer register is slow to read, and a wait that ends within a few probes
// should pay nothing for the deadline.  A failed try_wait suspends the thread until
// the phase completes or a hardware time limit (a few hundred cycles) passes.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          uint32_t* err, uint64_t limit_ns = 2000000000ull) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  long long t0 = 0;
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(a, parity)) return true;
    if ((i & 63u) == 0) {
      if (*abort) return false;
      if (i == 64u) {
        t0 = clock64();
      } else if (static_cast<uint64_t>(clock64() - t0) > 2ull * limit_ns) {
        *abort = 1;
        if (err) atomicOr(err, kErrTimeout);
        return false;
      }
    }
  }
}

// ----------------------------------------------------------------------------
// TMA (tensor memory accelerator) loads, no multicast
// ----------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

__device__ __forceinline__ void tma_load_5d(uint32_t dst, const CUtensorMap* m, uint64_t* bar,
                                            int c0, int c1, int c2, int c3, int c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
      "r"(c4)
      : "memory");
}

// ----------------------------------------------------------------------------
// tcgen05: tensor-memory allocation, MMA, commit, loads/stores
// ----------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle (the layout TMA writes with
// CU_TENSOR_MAP_SWIZZLE_128B).  Offsets in bytes; version 1 (sm_100).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

// Instruction descriptor of tcgen05.mma kind::f16 with bf16 A/B and fp32 D.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, int a_mn_major, int b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(a_mn_major) << 15) |
         (static_cast<uint32_t>(b_mn_major) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// Instruction descriptor of tcgen05.mma kind::tf32 with fp32 D, both operands K-major.
__host__ __device__ constexpr uint32_t idesc_tf32_f32(int M, int N) {
  return (1u << 4) | (2u << 7) | (2u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::tf32
__device__ __forceinline__ void mma_ss_tf32(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
      : "memory");
}

// fp32 -> tf32, round to nearest (ties away from zero), as an fp32 bit pattern whose
// low 13 mantissa bits are zero
__device__ __forceinline__ float to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

// D[tmem] (+)= A[smem] * B[smem]^T
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accum)
      : "memory");
}

// Arrive on `bar` once every tcgen05.mma issued so far by this thread has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

#define FV_R8(i) "=r"(r[i]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), \
                 "=r"(r[i + 4]), "=r"(r[i + 5]), "=r"(r[i + 6]), "=r"(r[i + 7])
#define FV_W8(i) "r"(r[i]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3]), \
                 "r"(r[i + 4]), "r"(r[i + 5]), "r"(r[i + 6]), "r"(r[i + 7])

// Each thread of the warp reads 32 consecutive 32-bit columns of its own TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : FV_R8(0), FV_R8(8), FV_R8(16), FV_R8(24)
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      FV_W8(0), FV_W8(8), FV_W8(16), FV_W8(24)
      : "memory");
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
               FV_W8(0)
               : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Packed pairs of fp32 (Blackwell f32x2 arithmetic: two lanes per instruction).
__device__ __forceinline__ uint64_t f32x2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void unpack_f32x2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

}  // namespace fv
