// Thin inline-PTX layer for sm_100a: mbarriers, TMA tile loads, tcgen05 MMA
// with TMEM accumulators, TMEM loads/stores, and bounded waits.
//
// Every wait in this library is bounded: after FA_WAIT_LIMIT_NS of wall time
// (read from %globaltimer) it records FA_ERR_DEVICE_TIMEOUT in the device
// status word, raises the CTA's abort flag and returns false. Callers then
// skip the rest of their work, so a stuck barrier ends the kernel instead of
// hanging the GPU.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>

#ifndef FA_WAIT_LIMIT_NS
#define FA_WAIT_LIMIT_NS 2000000000ull  // 2 s
#endif

namespace fa {

// Device status word (FA_OK == 0); read and cleared by fa_check_device_status.
// The library is one translation unit (fa_api.cu), which defines it here.
__device__ int g_status = 0;

// Where a wait gave up: 1 = mbarrier, 2 = dQ ordering counter.
__device__ __forceinline__ void record_timeout(int where) {
  atomicCAS(&g_status, 0, 4 /*FA_ERR_DEVICE_TIMEOUT*/);
  (void)where;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t lane_id() { return threadIdx.x & 31; }

__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "elect.sync _|p, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

// ------------------------------------------------------------------ mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase with the given parity to complete. Returns false
// (and raises *abort) on timeout, or when another role already aborted and
// `honor_abort` is set. Drains (copies or MMAs that must finish before the CTA
// exits) pass honor_abort = false and are bounded by time only.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          bool honor_abort = true, uint64_t limit_ns = FA_WAIT_LIMIT_NS) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t n = 1;; ++n) {
    if (mbar_try_wait(a, parity)) return true;
    if ((n & 255u) == 0) {
      if (honor_abort && *abort) return false;
      if (globaltimer() - t0 > limit_ns) {
        record_timeout(1);
        *abort = 1;
        return false;
      }
    }
  }
}

// Non-blocking test of three phases at once: true when all three have
// completed. The three tests share one round trip to the barrier unit, where
// three waits in a row would pay it three times.
__device__ __forceinline__ bool mbar_ready3(uint64_t* a, uint32_t pa, uint64_t* b, uint32_t pb, uint64_t* c,
                                            uint32_t pc) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p, q, r;\n\t"
      "mbarrier.test_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "mbarrier.test_wait.parity.acquire.cta.shared::cta.b64 q, [%3], %4;\n\t"
      "mbarrier.test_wait.parity.acquire.cta.shared::cta.b64 r, [%5], %6;\n\t"
      "and.pred p, p, q;\n\t"
      "and.pred p, p, r;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(a)), "r"(pa), "r"(smem_u32(b)), "r"(pb), "r"(smem_u32(c)), "r"(pc)
      : "memory");
  return ok != 0;
}

// ------------------------------------------------------ cluster (2 CTAs)

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Every thread of every CTA in the cluster; orders the barrier inits above it
// before any remote arrive.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Address of the same shared-memory offset in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}

// Arrive on an mbarrier in another CTA of the cluster, releasing this thread's
// earlier shared-memory writes at cluster scope.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t remote_bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote_bar) : "memory");
}

__device__ __forceinline__ float4 ld_shared_cluster_v4(uint32_t raddr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(raddr)
               : "memory");
  return v;
}

// Bounded wait with cluster-scope acquire (for phases completed by remote
// arrivals); same limit and error reporting as mbar_wait.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, uint64_t limit_ns = FA_WAIT_LIMIT_NS) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = globaltimer();
  for (uint32_t n = 0;; ++n) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(a), "r"(parity)
        : "memory");
    if (ok) return true;
    if ((n & 255u) == 255u && globaltimer() - t0 > limit_ns) {
      record_timeout(1);
      return false;
    }
  }
}

// Warp-uniform variant for code that follows with warp-collective tcgen05
// instructions: every lane returns the same answer.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity, volatile int* abort) {
  const bool ok = mbar_wait(bar, parity, abort);
  return __all_sync(0xffffffffu, ok);
}

// ----------------------------------------------------------------------- TMA

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 4-D tiled load into this CTA's own shared memory (one destination); completion is
// signalled on `bar` as transaction bytes.
__device__ __forceinline__ void tma_load_4d(const CUtensorMap* map, void* smem_dst, uint64_t* bar, int c0,
                                            int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
      : "memory");
}

// Prefetch one 4-D tile into L2 (no shared-memory destination, no barrier).
__device__ __forceinline__ void tma_prefetch_l2_4d(const CUtensorMap* map, int c0, int c1, int c2, int c3) {
  asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1), "r"(c2), "r"(c3)
               : "memory");
}

// A 128-row tile of a [B, N, H, d] tensor: 64 head-size columns `x`.., head h,
// rows `row`.. of batch coordinate b. The tensor map lists its dimensions as
// (d, H, rows, B), or as (d, rows, H, B) when the head stride exceeds the row
// stride (head-major storage such as [B, H, N, d]); both boxes put the same
// [128 rows][64 columns] tile into shared memory.
// (Coordinates picked by selects, not a branch around two copies of the
// load.)
__device__ __forceinline__ void tma_load_rows(const CUtensorMap* map, bool head_major, void* smem_dst,
                                              uint64_t* bar, int x, int h, int row, int b) {
  tma_load_4d(map, smem_dst, bar, x, head_major ? row : h, head_major ? h : row, b);
}
__device__ __forceinline__ void tma_prefetch_rows(const CUtensorMap* map, bool head_major, int x, int h, int row,
                                                  int b) {
  tma_prefetch_l2_4d(map, x, head_major ? row : h, head_major ? h : row, b);
}

// Bits of FwdArgs::hm / BwdArgs::hm: which tensor maps are head-major.
constexpr uint32_t kHmQ = 1, kHmK = 2, kHmV = 4, kHmDO = 8, kHmO = 16, kHmDK = 32, kHmDV = 64;

// TMA tile store of one box from shared memory (128-byte swizzled like the
// loads), tracked by bulk async-groups of the issuing thread.
__device__ __forceinline__ void tma_store_rows(const CUtensorMap* map, bool head_major, const void* smem_src, int x,
                                               int h, int row, int b) {
  asm volatile(
      "cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(static_cast<uint32_t>(__cvta_generic_to_shared(smem_src))), "r"(x), "r"(head_major ? row : h),
      "r"(head_major ? h : row), "r"(b)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// The shared memory of every committed store has been read.
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Every committed store is complete.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// True on all 128 threads of warpgroup barrier `id` iff v is true on all of them.
__device__ __forceinline__ bool wg_all(bool v, int id) {
  uint32_t r;
  asm volatile(
      "{ .reg .pred p, q; setp.ne.u32 p, %1, 0; bar.red.and.pred q, %2, 128, p; selp.u32 %0, 1, 0, q; }"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(id)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void fence_async_shared() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void st_shared_v4(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(p))),
               "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

// ------------------------------------------------------------------- tcgen05

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor (tcgen05 format): start address, leading and
// stride byte offsets (all >> 4), version bits 46-47 = 1, swizzle mode in
// bits 61-63 (2 = 128-byte swizzle).
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;
  d |= 2ull << 61;
  return d;
}

// Instruction descriptor for kind::f16 with fp32 accumulation.
__host__ __device__ constexpr uint32_t idesc_f16(bool bf16, int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) | ((a_mn_major ? 1u : 0u) << 15) |
         ((b_mn_major ? 1u : 0u) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem]
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` when every tcgen05 operation this thread issued so far
// has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// 32 consecutive 32-bit TMEM columns of this thread's lane -> r[0..31].
// The values are only valid after tmem_ld_wait(); tie_regs32() afterwards keeps
// the compiler from moving their uses above the wait.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
        "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
        "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tie_regs32(uint32_t* r) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                 "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                 "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]),
                 "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]),
                 "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31]));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tie_regs16(uint32_t* r) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                 "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                 "+r"(r[14]), "+r"(r[15]));
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Per-warpgroup register budgets (setmaxnreg): call at the top of a role's
// branch so the role's code is compiled against its own budget.
template <int NREG>
__device__ __forceinline__ void reg_alloc_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(NREG));
}
template <int NREG>
__device__ __forceinline__ void reg_alloc_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(NREG));
}

// Move this warpgroup's budget from the launch count FROM to NREG.
template <int NREG, int FROM>
__device__ __forceinline__ void reg_alloc_set() {
  if constexpr (NREG > FROM) reg_alloc_inc<NREG>();
  else if constexpr (NREG < FROM) reg_alloc_dec<NREG>();
}

// ------------------------------------------------------------ tensor layout

// Rows of batch b in the caller's tensors. Fixed length (cu == nullptr): N
// rows starting at row 0 of batch b. Variable length: cu[b] .. cu[b+1] - 1 of
// the packed tensors (batch index 0), clamped to [0, total] and to at most N
// rows, so a malformed offset array can shorten a sequence but never move an
// access outside the tensors.
struct SeqRows {
  int row0, len, bcoord;  // first row, rows, TMA batch coordinate
};
__device__ __forceinline__ SeqRows seq_rows(const int* cu, int b, int N, int total) {
  SeqRows r;
  if (cu == nullptr) {
    r.row0 = 0;
    r.len = N;
    r.bcoord = b;
  } else {
    int a = __ldg(cu + b), e = __ldg(cu + b + 1);
    a = a < 0 ? 0 : (a > total ? total : a);
    e = e < a ? a : (e > total ? total : e);
    r.row0 = a;
    r.len = e - a < N ? e - a : N;
    r.bcoord = 0;
  }
  return r;
}

// ------------------------------------------------------------------ dropout

// Philox4x32-10 (Salmon, Moraes, Dror and Shaw, "Parallel Random Numbers: As
// Easy as 1, 2, 3", SC 2011): ten rounds of two 32x32->64-bit products with
// the paper's multipliers, the key advanced by its Weyl constants between
// rounds. Four 32-bit words per (counter, key).
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint32_t lo0 = 0xD2511F53u * c.x, hi0 = __umulhi(0xD2511F53u, c.x);
    const uint32_t lo1 = 0xCD9E8D57u * c.z, hi1 = __umulhi(0xCD9E8D57u, c.z);
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return c;
}

// Dropout of attention probabilities: element (query i, key j) of head
// bh = b*H + h (b: the sequence when variable-length, i and j counted from
// the sequence's first row) is dropped when word j % 4 of
// philox(counter (j/4, i, bh, offset), key (seed_lo, seed_hi)) is below
// `thr` = floor(p * 2^32). Kept values are scaled by 1 / (1 - p).
struct Dropout {
  uint32_t thr, seed_lo, seed_hi, offset;
  float rkeep;  // 1 / (1 - p)
};

// Keep bits of keys 4*g .. 4*g+3 for query i (bit w = key 4g + w).
__device__ __forceinline__ uint32_t keep4(const Dropout& dp, uint32_t g, uint32_t i, uint32_t bh) {
  const uint4 w = philox4x32_10(make_uint4(g, i, bh, dp.offset), dp.seed_lo, dp.seed_hi);
  return (w.x >= dp.thr ? 1u : 0u) | (w.y >= dp.thr ? 2u : 0u) | (w.z >= dp.thr ? 4u : 0u) |
         (w.w >= dp.thr ? 8u : 0u);
}

// --------------------------------------------------------------- arithmetic

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Two fp32 -> packed 16-bit pair, RNE; `lo` lands in the low half.
template <bool BF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  uint32_t r;
  if constexpr (BF16) {
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  } else {
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  }
  return r;
}

// Packed 16-bit pair -> two fp32 (low half first).
template <bool BF16>
__device__ __forceinline__ float2 unpack2(uint32_t w) {
  float2 r;
  if constexpr (BF16) {
    r.x = __uint_as_float(w << 16);
    r.y = __uint_as_float(w & 0xFFFF0000u);
  } else {
    __half2 h = *reinterpret_cast<__half2*>(&w);
    r = __half22float2(h);
  }
  return r;
}

// max(a, b, c) in one instruction (three-operand form of max.f32, sm_100).
// Two-lane fp32 arithmetic: sm_100's packed f32x2 forms issue one
// instruction for two IEEE round-to-nearest results, the same values as two
// scalar operations. A 64-bit operand holds lane 0 in its low word.
__device__ __forceinline__ uint64_t bcast2(float x) {
  const uint64_t u = __float_as_uint(x);
  return u | (u << 32);
}
// (y0, y1) = (x0, x1) * a + b
__device__ __forceinline__ void fma2(float& y0, float& y1, float x0, float x1, uint64_t a, uint64_t b) {
  asm("{ .reg .b64 x, y; mov.b64 x, {%2, %3}; fma.rn.f32x2 y, x, %4, %5; mov.b64 {%0, %1}, y; }"
      : "=f"(y0), "=f"(y1)
      : "f"(x0), "f"(x1), "l"(a), "l"(b));
}
// (s0, s1) += (x0, x1)
__device__ __forceinline__ void add2(float& s0, float& s1, float x0, float x1) {
  asm("{ .reg .b64 s, x; mov.b64 s, {%0, %1}; mov.b64 x, {%2, %3}; add.rn.f32x2 s, s, x; mov.b64 {%0, %1}, s; }"
      : "+f"(s0), "+f"(s1)
      : "f"(x0), "f"(x1));
}
// (y0, y1) = (p0, p1) * ((x0, x1) - b)
__device__ __forceinline__ void mul_sub2(float& y0, float& y1, float p0, float p1, float x0, float x1, uint64_t b) {
  asm("{ .reg .b64 p, x, t; mov.b64 p, {%2, %3}; mov.b64 x, {%4, %5}; sub.rn.f32x2 t, x, %6; mul.rn.f32x2 t, p, t;"
      " mov.b64 {%0, %1}, t; }"
      : "=f"(y0), "=f"(y1)
      : "f"(p0), "f"(p1), "f"(x0), "f"(x1), "l"(b));
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// acc + (low 16-bit half of w) and acc + (high half), the half widened
// exactly to fp32 inside the add (mixed-precision add.f32.f16 / .bf16, sm_100).
template <bool BF16>
__device__ __forceinline__ float add_lo16(float acc, uint32_t w) {
  if constexpr (BF16) {
    asm("{ .reg .b16 lo, hi; mov.b32 {lo, hi}, %1; add.rn.f32.bf16 %0, lo, %0; }" : "+f"(acc) : "r"(w));
  } else {
    asm("{ .reg .b16 lo, hi; mov.b32 {lo, hi}, %1; add.rn.f32.f16 %0, lo, %0; }" : "+f"(acc) : "r"(w));
  }
  return acc;
}
template <bool BF16>
__device__ __forceinline__ float add_hi16(float acc, uint32_t w) {
  if constexpr (BF16) {
    asm("{ .reg .b16 lo, hi; mov.b32 {lo, hi}, %1; add.rn.f32.bf16 %0, hi, %0; }" : "+f"(acc) : "r"(w));
  } else {
    asm("{ .reg .b16 lo, hi; mov.b32 {lo, hi}, %1; add.rn.f32.f16 %0, hi, %0; }" : "+f"(acc) : "r"(w));
  }
  return acc;
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

}  // namespace fa
