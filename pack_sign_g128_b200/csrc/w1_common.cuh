// Shared device helpers for the w1 kernels (sm_100a): status word, PDL,
// mbarriers, bulk async copies (TMA), clusters / DSMEM and tcgen05 wrappers.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "w1.h"

namespace w1 {

// One status word per device.  Kernels record the first error they detect
// (bounded-wait timeout, non-finite input, ...) and carry on or exit cleanly;
// the host reads and clears it with w1_sync_status().
__device__ unsigned int g_status = 0;

__device__ __forceinline__ void set_status(unsigned int code) {
  atomicCAS(&g_status, 0u, code);
}

// Upper bound on any spin-wait in these kernels (iterations of a poll that
// includes a nanosleep back-off); about a second or more of wall time.
constexpr uint32_t kSpinLimit = 1u << 22;

// ---------------------------------------------------------------- PDL
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// ---------------------------------------------------------------- smem / misc
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbarrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(smem_u32(bar)),
      "r"(bytes)
      : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: returns false (and records W1_ERR_TIMEOUT) if the phase with
// the given parity does not complete within the spin limit.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  for (uint32_t i = 0; i < kSpinLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (i > 64) __nanosleep(64);
  }
  set_status(W1_ERR_TIMEOUT);
  return false;
}

// Warp-uniform bounded wait: every lane polls, and the warp leaves the loop
// together (all lanes saw the phase complete, or all gave up), so code after
// it that needs a converged warp (mma.sync, tcgen05 .sync.aligned) is safe.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity) {
  for (uint32_t i = 0; i < kSpinLimit; ++i) {
    const bool ok = mbar_try_wait(bar, parity);
    if (__all_sync(0xFFFFFFFFu, ok)) return true;
    if (i > 64) __nanosleep(64);
  }
  set_status(W1_ERR_TIMEOUT);
  return false;
}

// ---------------------------------------------------------------- bulk copies
// 1-D bulk copy global -> shared, completing on an mbarrier (tx bytes).
// Both addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* smem_dst, const void* gsrc, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void bulk_prefetch_l2(const void* gsrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(gsrc), "r"(bytes) : "memory");
}
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// 2-D tiled TMA load (no multicast) completing on an mbarrier.
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const void* tmap, int32_t c0, int32_t c1,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, "
      "{%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
      "l"(tmap), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// ---------------------------------------------------------------- clusters
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t nclusters_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
// Address of the same shared variable in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t map_shared_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
// Split cluster barrier: arrive without ordering (all threads), wait later.
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
}
__device__ __forceinline__ void st_dsmem_f32(uint32_t addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
__device__ __forceinline__ float ld_dsmem_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

// ---------------------------------------------------------------- grid barrier
// Grid-wide barrier over all CTAs of the launch (all co-resident by
// construction of the grid).  bar[0] counts arrivals, bar[1] is the
// generation; the last arrival resets the count, so the state is reusable by
// the next call.  Returns false (and records W1_ERR_TIMEOUT) if the other
// CTAs do not arrive within the spin limit.
__device__ inline bool grid_barrier(unsigned int* bar, unsigned int nblocks) {
  __syncthreads();
  int ok = 1;
  if (threadIdx.x == 0) {
    __threadfence();
    unsigned int gen;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(gen) : "l"(bar + 1) : "memory");
    const unsigned int arrived = atomicAdd(bar, 1u);
    if (arrived == nblocks - 1) {
      atomicExch(bar, 0u);
      __threadfence();
      atomicAdd(bar + 1, 1u);
    } else {
      ok = 0;
      for (uint32_t i = 0; i < kSpinLimit; ++i) {
        unsigned int g;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(g) : "l"(bar + 1) : "memory");
        if (g != gen) {
          ok = 1;
          break;
        }
        __nanosleep(128);
      }
      if (!ok) set_status(W1_ERR_TIMEOUT);
    }
    __threadfence();
  }
  return __syncthreads_and(ok) != 0;
}

// ---------------------------------------------------------------- warp MMA (int8)
// D = A(16x32, s8, row) * B(32x8, s8, col) + C, s32 accumulate.
__device__ __forceinline__ void mma_s8_16832(int (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                             uint32_t b1, const int (&c)[4]) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%11,%12,%13};"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "r"(c[0]), "r"(c[1]),
        "r"(c[2]), "r"(c[3]));
}

}  // namespace w1

namespace w1 {

// ---------------------------------------------------------------- tcgen05 (1-CTA)
__device__ __forceinline__ void tmem_alloc(uint32_t* smem_dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(smem_dst)),
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
// D[tmem] (+)= A[tmem] * B[smem desc]^T, kind::f16 (bf16/f16 in, f32 accumulate).
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::f16.
__device__ __forceinline__ void tc_mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive (once) on an mbarrier when all prior tcgen05 async ops of this thread complete.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

#define W1_R32(a) a[0], a[1], a[2], a[3], a[4], a[5], a[6], a[7], a[8], a[9], a[10], a[11], a[12], \
    a[13], a[14], a[15], a[16], a[17], a[18], a[19], a[20], a[21], a[22], a[23], a[24], a[25],       \
    a[26], a[27], a[28], a[29], a[30], a[31]

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp gets lane
// (quarter base + i), columns taddr.col .. +31.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
      "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]),
      "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]),
      "r"(r[30]), "r"(r[31])
      : "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (SBO), start address in 16-byte units.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(1u) << 16;                 // LBO (unused for this layout)
  d |= static_cast<uint64_t>(1024u >> 4) << 32;         // SBO
  d |= static_cast<uint64_t>(1u) << 46;                 // descriptor version (sm_100)
  d |= static_cast<uint64_t>(2u) << 61;                 // SWIZZLE_128B
  return d;
}

// Instruction descriptor, kind::f16 with f32 accumulate, both operands K-major.
// a_fmt / b_fmt: 0 = f16, 1 = bf16.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, int a_fmt, int b_fmt) {
  return (1u << 4) | (static_cast<uint32_t>(a_fmt) << 7) | (static_cast<uint32_t>(b_fmt) << 10) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

}  // namespace w1

namespace w1 {

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr)
               : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem desc]^T, kind::i8 (s8 x s8 -> s32).
__device__ __forceinline__ void tc_mma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Instruction descriptor, kind::i8: s32 accumulate, signed A and B, both K-major.
__host__ __device__ constexpr uint32_t idesc_i8(int M, int N) {
  return (2u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}
// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (tensor core operand reads).
__device__ __forceinline__ void fence_async_shared() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

}  // namespace w1

// Host: raise a kernel's dynamic shared memory limit to at least `bytes` on
// the current device, calling the driver only when the cached value is lower
// (the attribute is set on every launch path, so this keeps it off the hot
// path).
#include <mutex>
namespace w1 {
inline cudaError_t ensure_dyn_smem(const void* kernel, int bytes) {
  struct Entry {
    const void* k;
    int dev;
    int bytes;
  };
  static Entry tab[256];
  static int n = 0;
  static std::mutex mu;
  int dev = 0;
  cudaGetDevice(&dev);
  {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < n; ++i)
      if (tab[i].k == kernel && tab[i].dev == dev && tab[i].bytes >= bytes) return cudaSuccess;
  }
  const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < n; ++i)
    if (tab[i].k == kernel && tab[i].dev == dev) {
      if (tab[i].bytes < bytes) tab[i].bytes = bytes;
      return cudaSuccess;
    }
  if (n < 256) tab[n++] = Entry{kernel, dev, bytes};
  return cudaSuccess;
}
}  // namespace w1

// Host: process-wide testing and tuning knobs.  They are read from the W1_*
// environment variables once, on first use, and can be changed afterwards
// with w1_set_knob (include/w1.h); no launch path reads the environment.
//   gemv_path     W1_GEMV_PATH      0 = dispatch, else a forced GEMV kernel
//   gemv_split    W1_GEMV_SPLIT     forced K split of the split-capable GEMV kernels (0 = planner)
//   gemv_autotune W1_GEMV_AUTOTUNE  0 = static rule instead of first-call timing
//   moe_path      W1_MOE_PATH       0 = by token count, 1 = tiles, 2 = decode, 3 = decode grouped by expert
//   dbf_path      W1_DBF_PATH       0 = by batch, else a forced small-batch chain form
//   dbf_warps     W1_DBF_WARPS      0 = by group size, 8 or 16 warps per CTA
//   dbf_rank_split W1_DBF_RANK_SPLIT two-launch chain: CTAs per cluster that split r in U . h (0 = planner)
//   sg_bm         W1_SG_BM          sign GEMM token tile: 0 = by tile count, else 128 or 256
//   dbf_core      W1_DBF_CORE       two-launch chain's GEMV core: 0 = register-fed where it fits, 1 = same, 2 = direct
//   moe_tw        W1_MOE_TW         decode MoE gate/up: 8-row n-tiles per warp, 0 = by CTA count, else 2 or 4
//   sg_exp        W1_SG_EXP         sign GEMM expander warps: 0 = by token tile, else 4 or 8
//   sg_a          W1_SG_A           sign GEMM weight operand of 128-token tiles: 0 = default, 1 = smem, 2 = TMEM
//   verbose       W1_VERBOSE        nonzero: plans and choices on stderr
#include <atomic>
#include <cstdlib>
#include <cstring>
namespace w1 {
enum KnobId { kKnobGemvPath, kKnobGemvSplit, kKnobGemvAutotune, kKnobMoePath, kKnobDbfPath, kKnobDbfWarps,
              kKnobDbfRankSplit, kKnobSgBm, kKnobDbfCore, kKnobSgExp, kKnobSgA, kKnobMoeTw, kKnobVerbose, kKnobCount };
// GEMV kernels a knob can force (also the kinds of the dispatcher's choices).
enum GemvPathKnob { kGemvAuto = 0, kGemvDirect8 = 1, kGemvDirect16 = 2, kGemvTc = 3, kGemvRing = 4, kGemvFlat = 5,
                    kGemvFlat16 = 6 };
enum DbfPathKnob { kDbfAuto = 0, kDbfFused = 1, kDbfTwoStep = 2 };

struct KnobSpec {
  const char* name;  // w1_set_knob name
  const char* env;   // environment variable read at first use
  int dflt;
  const char* words[7];  // accepted words for values 1..7 (else an integer)
};
inline const KnobSpec& knob_spec(int id) {
  static const KnobSpec specs[kKnobCount] = {
      {"gemv_path", "W1_GEMV_PATH", 0, {"direct", "direct16", "tc", "ring", "flat", "flat16", nullptr}},
      {"gemv_split", "W1_GEMV_SPLIT", 0, {nullptr}},
      {"gemv_autotune", "W1_GEMV_AUTOTUNE", 1, {nullptr}},
      {"moe_path", "W1_MOE_PATH", 0, {"tiles", "decode", "grouped", nullptr}},
      {"dbf_path", "W1_DBF_PATH", 0, {"fused", "twostep", nullptr}},
      {"dbf_warps", "W1_DBF_WARPS", 0, {nullptr}},
      {"dbf_rank_split", "W1_DBF_RANK_SPLIT", 0, {nullptr}},
      {"sg_bm", "W1_SG_BM", 0, {nullptr}},
      {"dbf_core", "W1_DBF_CORE", 0, {"flat", "direct", nullptr}},
      {"sg_exp", "W1_SG_EXP", 0, {nullptr}},
      {"sg_a", "W1_SG_A", 0, {"smem", "tmem", nullptr}},
      {"moe_tw", "W1_MOE_TW", 0, {nullptr}},
      {"verbose", "W1_VERBOSE", 0, {nullptr}},
  };
  return specs[id];
}
// Parses a knob value: one of the spec's words (-> 1-based index) or an
// integer.  Returns false for anything else.
inline bool parse_knob(int id, const char* v, int* out) {
  const KnobSpec& s = knob_spec(id);
  for (int i = 0; i < 7 && s.words[i]; ++i)
    if (strcmp(v, s.words[i]) == 0) {
      *out = i + 1;
      return true;
    }
  char* end = nullptr;
  const long n = strtol(v, &end, 10);
  if (end == v || *end != '\0' || n < 0 || n > 1 << 20) return false;
  *out = static_cast<int>(n);
  return true;
}
struct KnobTable {
  std::atomic<int> v[kKnobCount];
  int env[kKnobCount];  // the value the environment gave (restored by w1_set_knob(name, NULL))
  KnobTable() {
    for (int i = 0; i < kKnobCount; ++i) {
      int val = knob_spec(i).dflt;
      const char* e = getenv(knob_spec(i).env);
      if (e && *e) {
        int p = 0;
        if (parse_knob(i, e, &p)) val = p;
      }
      env[i] = val;
      v[i].store(val, std::memory_order_relaxed);
    }
  }
};
inline KnobTable& knob_table() {
  static KnobTable t;  // thread-safe initialisation (C++11 statics)
  return t;
}
inline int knob(int id) { return knob_table().v[id].load(std::memory_order_relaxed); }
}  // namespace w1
