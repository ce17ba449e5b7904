// Shared device primitives for the sm_100a DSA kernels: shared-memory barriers, TMA
// tensor loads, tcgen05 (5th-generation tensor core) MMA / tensor-memory access, and
// bounded waits that report a timeout instead of hanging.
//
// Written from the public PTX ISA description of these instructions.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <climits>

#include <atomic>
#include <utility>

#include "../../include/dsa.h"

namespace dsa {

// ------------------------------------------------------------------ device status word
// Set by a bounded wait that ran out; read and cleared by dsa_get_device_status().
// (The library is one translation unit, so these are defined here.)
__device__ int g_status = 0;
__device__ int g_status_detail = 0;

constexpr unsigned long long kWaitLimitNs = 4000000000ull;  // 4 s: far above any legal wait

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void record_timeout(int where) {
  atomicExch(&g_status, (int)DSA_ERR_TIMEOUT);
  atomicExch(&g_status_detail, where);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar_addr, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar_addr), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for the phase with the given parity to complete.  Gives up (returns false) when
// *abort_flag is set by another role or after limit_ns, recording a timeout.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          int where, unsigned long long limit_ns = kWaitLimitNs) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(a, parity)) return true;
    if ((it & 63u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        *abort_flag = 1;
        record_timeout(where);
        return false;
      }
    }
  }
}

// ------------------------------------------------------------------ TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2-D tiled TMA load into shared memory; completion is signalled as transaction bytes
// on `bar`.  c0 is the innermost (element) coordinate, c1 the row coordinate.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0,
                                            int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

// 3-D tiled TMA load (c0 innermost), completion counted on `bar`.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                            int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// ------------------------------------------------------------------ tcgen05
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

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 inputs, fp32 accumulate, one CTA.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D (+)= A . B with A read from tensor memory at a_tmem (lane m = row m of A; along K, two
// bf16 per 32-bit column, so K = 16 spans 8 columns) and B from shared memory (descriptor).
__device__ __forceinline__ void umma_bf16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive (once) on `bar` when all previously issued tcgen05.mma of this thread complete.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp gets lane (base + i).
// The load and its wait are one asm statement, so no use of v can be scheduled before
// the data has arrived.
__device__ __forceinline__ void tmem_ld_x32_sync(uint32_t taddr, float* v) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns stored from registers (thread i of the warp to
// lane base + i), and the wait for the stores to complete, in one statement.
__device__ __forceinline__ void tmem_st_x32_sync(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};\n\t"
      "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
        "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
        "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns, load and wait in one statement.
__device__ __forceinline__ void tmem_ld_x16_sync(uint32_t taddr, float* v) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

// 32 lanes x 8 consecutive 32-bit columns, load and wait in one statement.
__device__ __forceinline__ void tmem_ld_x8_sync(uint32_t taddr, float* v) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
      : "r"(taddr)
      : "memory");
}

// 32 lanes x 8 consecutive 32-bit columns stored from registers, and the wait for them.
__device__ __forceinline__ void tmem_st_x8_sync(uint32_t taddr, const float* v) {
  const uint32_t* r = reinterpret_cast<const uint32_t*>(v);
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};\n\t"
      "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
      : "memory");
}

// Shared-memory matrix descriptor for a K-major operand tile stored as rows of
// `swizzle_bytes` (128 or 64) bytes with the matching TMA swizzle; 8-row groups are
// 8*swizzle_bytes apart.  Fields: start address >> 4 (bits 0-13), leading byte offset
// >> 4 (16-29, unused for swizzled K-major, set to 1), stride byte offset >> 4 (32-45),
// descriptor version 1 (46-47), base offset 0 (49-51), layout type (61-63: 2 = 128-byte
// swizzle, 4 = 64-byte swizzle).
__device__ __forceinline__ uint64_t smem_desc_kmajor(uint32_t saddr, int swizzle_bytes) {
  const uint64_t start = (saddr >> 4) & 0x3FFFu;
  const uint64_t lbo = 1;
  const uint64_t sbo = (uint64_t)((8 * swizzle_bytes) >> 4);
  const uint64_t layout = (swizzle_bytes == 128) ? 2 : 4;
  return start | (lbo << 16) | (sbo << 32) | (1ull << 46) | (layout << 61);
}

// Shared-memory matrix descriptor for an MN-major operand in the 128-byte swizzled layout:
// each 128-byte row holds 64 consecutive M (or N) elements of one k, 8 rows (k .. k+7) form
// a 1024-byte swizzle atom.  `mn_block_bytes` is the distance between blocks of 64 M/N
// elements (the leading byte offset), 8-row k groups are 1024 bytes apart (stride offset).
__device__ __forceinline__ uint64_t smem_desc_mn_sw128(uint32_t saddr, uint32_t mn_block_bytes) {
  const uint64_t start = (saddr >> 4) & 0x3FFFu;
  const uint64_t lbo = (mn_block_bytes >> 4) & 0x3FFFu;
  const uint64_t sbo = 1024 >> 4;
  return start | (lbo << 16) | (sbo << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor of tcgen05.mma kind::f16 with bf16 A/B, fp32 D, both K-major.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4)                       // D format: f32
         | (1u << 7)                     // A format: bf16
         | (1u << 10)                    // B format: bf16
         | ((uint32_t)(N >> 3) << 17)    // N / 8
         | ((uint32_t)(M >> 4) << 24);   // M / 16
}
// Instruction-descriptor bits that mark the A operand as MN-major (M contiguous) and the
// B operand as MN-major (N contiguous).
constexpr uint32_t kIdescAMnMajor = 1u << 15;
constexpr uint32_t kIdescBMnMajor = 1u << 16;

// ------------------------------------------------------------------ CTA pairs (cta_group::2)
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// shared::cluster address of the same shared-memory offset in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t map_to_rank(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ void tmem_alloc2(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish2() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc2(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// D[tmem of both CTAs] (+)= A (M = 256 rows, 128 from each CTA) x B^T (N columns, N/2 rows
// from each CTA); issued by the even CTA of the pair with descriptors of its own shared
// memory, the odd CTA's operands sit at the same offsets.
__device__ __forceinline__ void umma2_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// When the pair's previously issued MMAs complete, arrive once on the barrier at this
// shared-memory offset in every CTA of `cta_mask`.
__device__ __forceinline__ void umma2_commit_mc(uint64_t* bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(cta_mask)
      : "memory");
}
// 2-D tiled TMA load into this CTA's shared memory whose completion bytes are counted on
// a barrier of the pair's even CTA (cluster address).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint32_t bar_cluster, int c0,
                                                 int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1)
      : "memory");
}

// ------------------------------------------------------------------ cp.async (16-byte, zero-fill)
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// Arrive on `bar` once every cp.async this thread issued so far has landed (the arrival
// counts toward the barrier's expected count; nothing else arrives for this thread).
__device__ __forceinline__ void cp_async_mbar_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// ------------------------------------------------------------------ programmatic dependent launch
// A kernel launched with the programmatic-serialization attribute may be scheduled before
// the previous kernel of the stream finishes; pdl_wait() blocks (in hardware) until that
// kernel has completed and its memory is visible, and is a no-op otherwise.  Every kernel
// that is launched that way calls pdl_wait() before touching global memory.
// pdl_trigger() lets the next kernel of the stream be scheduled early; kernels call it only
// after their own pdl_wait() returned, so at most one kernel waits ahead of the running
// one (a chain of early triggers would park later kernels' blocks on SMs the running
// kernel needs).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ------------------------------------------------------------------ register reallocation
// Moves registers between the warpgroups of a block (every warp of a warpgroup executes
// the same instruction).  The increases of all warpgroups must fit in what the block was
// launched with (threads x registers per thread) minus what the decreases leave in use.
template <int N>
__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

// ------------------------------------------------------------------ misc
// 2^x by the hardware approximation, subnormal results flushed to zero (ex2.approx.ftz).
__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
  return __uint_as_float(((uint32_t)b) << 16);
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Named barrier over `nthreads` threads that also returns whether `pred` held in any of them.
__device__ __forceinline__ bool named_bar_any(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.cta.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0u;
}

// Query rows [row_begin, row_end) of a varlen batch split, per sequence, into blocks of R
// rows; block 0 is the range's last block (the longest causal rows of the last sequence).
struct RowBlock {
  long long t0;  // first row (global)
  int ntok;      // rows in the block (1..R)
  int i0;        // t0's position in its sequence
  int Lq, Lk, kbase;
};

// `from_last`-th block of the range, or false past its end (n_blocks may be an upper bound).
template <int R>
__device__ __forceinline__ bool chunk_row_block(long long from_last, const int* cu_q, const int* cu_k, int batch,
                                                long long row_begin, long long row_end, long long n_blocks,
                                                RowBlock& rb) {
  if (from_last >= n_blocks) return false;
  long long r = n_blocks - 1 - from_last;
  for (int b = 0; b < batch; ++b) {
    const long long lo = max((long long)cu_q[b], row_begin), hi = min((long long)cu_q[b + 1], row_end);
    if (hi <= lo) continue;
    const long long nb = (hi - lo + R - 1) / R;
    if (r < nb) {
      rb.t0 = lo + r * R;
      rb.ntok = (int)min((long long)R, hi - rb.t0);
      rb.i0 = (int)(rb.t0 - cu_q[b]);
      rb.Lq = cu_q[b + 1] - cu_q[b];
      rb.Lk = cu_k[b + 1] - cu_k[b];
      rb.kbase = cu_k[b];
      return true;
    }
    r -= nb;
  }
  return false;
}

// Persistent-grid slot -> work index in snake order: CTA c takes position c of even rounds
// of gridDim.x slots and gridDim.x - 1 - c of odd ones, which evens out a descending cost.
__device__ __forceinline__ long long snake_slot(long long slot) {
  const long long G = gridDim.x, k = slot / G, pos = slot % G;
  return k * G + ((k & 1) ? G - 1 - pos : pos);
}

// Visible keys of query position i (causal, queries aligned to the end of the keys).
__device__ __forceinline__ int causal_vis(int i, int Lq, int Lk) { return min(max(i + Lk - Lq + 1, 0), Lk); }

// Order-preserving map of fp32 to uint32 (larger float -> larger key); -0.0 maps like +0.0.
__device__ __forceinline__ uint32_t float_order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

}  // namespace dsa

// ------------------------------------------------------------------ host helpers
namespace dsa_host {

// Encodes a 2-D bf16 TMA descriptor over a row-major [rows, cols] matrix with the given
// row pitch (bytes), box [box_rows, box_cols] and shared-memory swizzle (64 or 128 B).
int make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                      uint64_t row_pitch_bytes, uint32_t box_rows, uint32_t box_cols, int swizzle_bytes);

int make_tmap_bf16_3d(CUtensorMap* map, const void* base, const uint64_t dims[3], const uint64_t strides[2],
                      const uint32_t box[3]);

// The union form of the masked tensor-core attention passes (adjacent-query reuse): per
// 16-row block the sorted union of its rows' selected positions, its size, the
// per-(row, union slot) selection words and whether the block takes the form at all.
struct KlUnion {
  const int* ukeys;
  const int* ucount;
  const uint32_t* umask;
  const uint8_t* blk_use;
  int ucap;  // positions per block, a multiple of 128
  const int* blk_list;  // the blocks that take the form, and their number (device)
  const int* n_used;
};

// A one-time-setup flag kept per GPU: cudaFuncSetAttribute applies to the current device
// only, and one process may drive several GPUs.  Reads and writes go to the current
// device's bit (devices past 63 always read false, so their setup simply repeats).
class DeviceFlag {
 public:
  constexpr DeviceFlag() = default;
  operator bool() const {
    const int d = device();
    return d < 64 && ((bits_.load(std::memory_order_acquire) >> d) & 1ull);
  }
  DeviceFlag& operator=(bool v) {
    const int d = device();
    if (d < 64) {
      if (v)
        bits_.fetch_or(1ull << d, std::memory_order_acq_rel);
      else
        bits_.fetch_and(~(1ull << d), std::memory_order_acq_rel);
    }
    return *this;
  }

 private:
  static int device() {
    int d = 0;
    return cudaGetDevice(&d) == cudaSuccess && d >= 0 ? d : 64;
  }
  std::atomic<unsigned long long> bits_{0};
};

int sm_count();
int last_launch_status();    // DSA_ERR_CUDA if the last launch failed, else DSA_OK
int cuda_fail(cudaError_t e);  // records e for dsa_last_cuda_error(); returns DSA_ERR_CUDA

// Launches `kern`, with programmatic stream serialization when `pdl` is set (the kernel
// must then call pdl_wait() before its first global memory access).  The library sets it
// only between the launches of one entry point (the top-k passes, attention and its split
// combine): measured on the decode step, letting a call's first kernel overlap the
// previous call's last one made the step slower.  Returns DSA_OK or DSA_ERR_CUDA.
template <typename... KArgs, typename... Args>
int launch_pdl(bool pdl, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
               Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  if (const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...); e != cudaSuccess)
    return cuda_fail(e);
  return last_launch_status();
}

}  // namespace dsa_host
