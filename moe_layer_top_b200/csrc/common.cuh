// Device-side building blocks for sm_100a: mbarriers with bounded waits,
// TMA tile loads, tcgen05 (5th-generation tensor core) issue / TMEM access,
// and the small numeric helpers the MoE kernels share.
//
// Every spin on an mbarrier is bounded by wall-clock time read from
// %globaltimer.  A wait that runs out records a code in the caller's device
// status word, raises the CTA's abort flag and returns false; the kernel then
// drains what it has in flight, frees its TMEM and returns, so the context
// stays usable and the host sees the failure through moe_read_status().
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "moe_b200.h"

namespace moe {

// --------------------------------------------------------------------------
// status word (int32 in the caller's workspace)
// --------------------------------------------------------------------------
__device__ __forceinline__ void report_status(int* status, int code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// generous: the longest legitimate wait is one tile's main loop (microseconds)
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// --------------------------------------------------------------------------
// mbarrier
// --------------------------------------------------------------------------
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

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait until the phase with the given parity has completed.  Returns false
// (after recording `where` in *status and raising *abort) if it does not
// complete within kWaitTimeoutNs, or if another role raised *abort.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int* status,
                                          int where, uint64_t timeout_ns = kWaitTimeoutNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (globaltimer_ns() - t0 > timeout_ns) {
      *abort = 1;
      report_status(status, where);
      return false;
    }
  }
}

// --------------------------------------------------------------------------
// programmatic dependent launch: every kernel of the pipeline lets the next
// one launch once all of its CTAs are resident, and waits for the previous
// one to complete (and its memory to be visible) before reading its outputs.
// Both are no-ops when the kernel was launched without the attribute.
// Kernels that wait use plain global loads only -- no __ldg and no
// const __restrict__ pointers: those compile to invariant non-coherent loads
// that the compiler may hoist above the wait, reading data the previous
// kernel has not written yet.
// --------------------------------------------------------------------------
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// L2-coherent load (bypasses L1).  Used only for data that a kernel two or
// more launches back wrote, read before griddepcontrol.wait by a kernel whose
// predecessor triggered its launch only after its own wait.
__device__ __forceinline__ int ld_cg_i32(const int32_t* p) {
  int v;
  asm volatile("ld.global.cg.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// --------------------------------------------------------------------------
// TMA (cp.async.bulk.tensor), no multicast
// --------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const void* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* smem_dst, const void* map, uint64_t* bar, int x, int y,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cta.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(policy)
      : "memory");
}

// untiled bulk copy global -> this CTA's shared memory (16-byte aligned
// addresses, size a multiple of 16); completes `bytes` on the mbarrier
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Asynchronous bulk store of `bytes` (a multiple of 16) from shared to global
// memory, both addresses 16-byte aligned, tracked by the issuing thread's bulk
// groups; the shared source must be made visible to the async proxy first
// (fence_proxy_async_smem after the generic stores that wrote it).
__device__ __forceinline__ void bulk_store(void* dst, const void* smem_src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(reinterpret_cast<uint64_t>(dst)),
               "r"(smem_u32(smem_src)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// this thread's earlier bulk stores have finished reading shared memory
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// this thread's earlier bulk stores have completed
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// TMA gather of four rows (tile::gather4): rows y0..y3 of a 2-D tensor map whose
// box is one row high, x the first column, into 4 consecutive box rows at
// smem_dst (the 128-byte swizzle follows the shared-memory address, so four
// rows land exactly as a 4-row slice of a swizzled tile)
__device__ __forceinline__ void tma_gather4(void* smem_dst, const void* map, uint64_t* bar, int x, int y0, int y1,
                                            int y2, int y3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cta.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y0), "r"(y1), "r"(y2), "r"(y3)
      : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t policy_evict_normal() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// --------------------------------------------------------------------------
// tcgen05: TMEM allocation, MMA issue, commit, loads
// --------------------------------------------------------------------------
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

// D[tmem] (+)= A[smem] * B[smem]^T, both K-major; kind::f16 (bf16 inputs)
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// same with E4M3 inputs (kind::f8f6f4)
__device__ __forceinline__ void mma_fp8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// MXFP8 block-scaled MMA (kind::mxf8f6f4, one E8M0 scale per 32 K elements):
// D[tmem] (+)= (A * sfa) x (B * sfb)^T with the scale factors read from TMEM at
// tsfa / tsfb; bits 30-31 of those addresses select the byte (the 32-element
// K block inside a 4-byte TMEM cell) and must equal the ids in the descriptor.
__device__ __forceinline__ void mma_mxf8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate, uint32_t tsfa, uint32_t tsfb) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(tsfa), "r"(tsfb)
      : "memory");
}

// Instruction descriptor of the block-scaled MMA: E4M3 A and B, E8M0 scales
// (bit 23), N >> 3 at bit 17, M >> 4 at bit 24, scale-factor byte ids of B at
// bits 4-5 and of A at bits 29-30.
__host__ __device__ constexpr uint32_t make_idesc_mx(int M, int N, int sf_id) {
  return (static_cast<uint32_t>(sf_id) << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (1u << 23) |
         (static_cast<uint32_t>(M >> 4) << 24) | (static_cast<uint32_t>(sf_id) << 29);
}

// shared-memory descriptor of a non-swizzled K-major operand whose 8-row core
// matrices (8 x 16 bytes) lie 128 bytes apart: a 512-byte SF atom = 32 rows x 16 B
__device__ __forceinline__ uint64_t smem_desc_sf_atom(uint32_t smem_addr) {
  return static_cast<uint64_t>((smem_addr >> 4) & 0x3FFF) | (static_cast<uint64_t>(128 >> 4) << 32) | (1ull << 46);
}

// copy one SF atom (32 lanes x 128 bits) from shared memory into TMEM columns
// [taddr, taddr + 4), replicated to the four lane quarters
__device__ __forceinline__ void tmem_cp_sf_atom(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// arrive on `bar` once every tcgen05.mma issued so far by this thread is done
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 lanes x 16 consecutive 32-bit columns: thread i gets lane (base + i)
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// same, raw 32-bit words
__device__ __forceinline__ void tmem_ld16u(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
  uint32_t r[8];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_ld8u(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
      : "r"(taddr));
}

// 32 lanes x 32 consecutive 32-bit columns (raw bits)
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// two fp32 lanes at once: (a0, a1) <- (d0, d1) * (f, f) + (a0, a1), each correctly rounded
__device__ __forceinline__ void ffma2(uint32_t& a0, uint32_t& a1, uint32_t d0, uint32_t d1, float f) {
  asm("{\n\t.reg .b64 ra, rd, rf;\n\t"
      "mov.b64 ra, {%0, %1};\n\t"
      "mov.b64 rd, {%2, %3};\n\t"
      "mov.b64 rf, {%4, %4};\n\t"
      "fma.rn.f32x2 ra, rd, rf, ra;\n\t"
      "mov.b64 {%0, %1}, ra;\n\t}"
      : "+r"(a0), "+r"(a1)
      : "r"(d0), "r"(d1), "r"(__float_as_uint(f)));
}

// float accumulators: (a0, a1) <- (d0, d1) * (f, f) + (a0, a1), d as raw fp32 words
__device__ __forceinline__ void ffma2f(float& a0, float& a1, uint32_t d0, uint32_t d1, float f) {
  asm("{\n\t.reg .b64 ra, rd, rf;\n\t"
      "mov.b64 ra, {%0, %1};\n\t"
      "mov.b64 rd, {%2, %3};\n\t"
      "mov.b64 rf, {%4, %4};\n\t"
      "fma.rn.f32x2 ra, rd, rf, ra;\n\t"
      "mov.b64 {%0, %1}, ra;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "r"(d0), "r"(d1), "f"(f));
}

// (a0, a1) <- (d0, d1) * (f, f)
__device__ __forceinline__ void fmul2(uint32_t& a0, uint32_t& a1, uint32_t d0, uint32_t d1, float f) {
  asm("{\n\t.reg .b64 ra, rd, rf;\n\t"
      "mov.b64 rd, {%2, %3};\n\t"
      "mov.b64 rf, {%4, %4};\n\t"
      "mul.rn.f32x2 ra, rd, rf;\n\t"
      "mov.b64 {%0, %1}, ra;\n\t}"
      : "=r"(a0), "=r"(a1)
      : "r"(d0), "r"(d1), "r"(__float_as_uint(f)));
}

// Shared-memory matrix descriptor of a K-major tile written by TMA with the
// 128-byte swizzle: rows of 128 bytes, 8-row atoms of 1024 bytes.
//   bits  0-13 start address >> 4, 16-29 leading byte offset >> 4 (unused
//   for swizzled K-major, set to 1), 32-45 stride byte offset >> 4 (1024 B
//   between 8-row groups), 46-47 descriptor version 1, 61-63 layout 2 =
//   128-byte swizzle.  Advancing along K inside the 128-byte row is done by
//   adding the byte offset to the start address.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr & 0x3FFFF) >> 4);
  d |= static_cast<uint64_t>(1) << 16;
  d |= static_cast<uint64_t>(1024 >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

// Instruction descriptor: fp32 accumulator, K-major A and B.
//   bits 4-5 D format (1 = f32), 7-9 A format, 10-12 B format
//   (kind::f16: 1 = bf16; kind::f8f6f4: 0 = e4m3), 15/16 A/B major (0 = K),
//   17-22 N >> 3, 24-28 M >> 4.
__host__ __device__ constexpr uint32_t make_idesc(int m, int n, bool fp8) {
  return (1u << 4) | ((fp8 ? 0u : 1u) << 7) | ((fp8 ? 0u : 1u) << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(m >> 4) << 24);
}

// --------------------------------------------------------------------------
// numerics
// --------------------------------------------------------------------------
__device__ __forceinline__ float bf16_round(float v) { return __bfloat162float(__float2bfloat16_rn(v)); }

// smallest power of two >= s, for positive normal s
__device__ __forceinline__ float pow2_ceil(float s) {
  const uint32_t b = __float_as_uint(s);
  if ((b & 0x007FFFFFu) == 0) return s;
  return __uint_as_float((b & 0x7F800000u) + 0x00800000u);
}

// exact reciprocal of a power of two (exponent field in 1..253)
__device__ __forceinline__ float pow2_recip(float p) {
  const uint32_t e = __float_as_uint(p) >> 23;
  return __uint_as_float((254u - e) << 23);
}

// per-(row,128) activation scale: pow2 ceiling of max(amax, 1e-10) * (1/448) in fp32
__device__ __forceinline__ float act_scale_from_amax(float amax) {
  return pow2_ceil(__fmul_rn(fmaxf(amax, 1e-10f), 1.0f / 448.0f));
}

// E8M0 byte of a power-of-two float (its biased exponent; normal range only)
__device__ __forceinline__ uint8_t e8m0_of_pow2(float s) {
  return static_cast<uint8_t>((__float_as_uint(s) >> 23) & 0xFFu);
}

// Byte offset of the E8M0 scale of element (n, k) of an [N, K] matrix in the
// MXFP8 SF-atom layout: one 512-byte atom per 128 rows x 128 columns, atoms
// K-block-fastest; inside an atom row n sits at (n % 32) * 16 + ((n % 128) / 32) * 4
// and the 32-column group at + (k % 128) / 32.  For a batch of [N, K]
// matrices pass n = batch * N + row (N is a multiple of 128).
__device__ __forceinline__ size_t sf_atom_offset(long long n, int k, int K) {
  return (static_cast<size_t>(n >> 7) * static_cast<size_t>(K >> 7) + static_cast<size_t>(k >> 7)) * 512 +
         static_cast<size_t>(n & 31) * 16 + static_cast<size_t>((n & 127) >> 5) * 4 + static_cast<size_t>((k & 127) >> 5);
}

// two floats -> two E4M3 codes (round to nearest even, saturating); lo in the low byte
__device__ __forceinline__ uint16_t f32x2_to_e4m3x2(float lo, float hi) {
  return static_cast<uint16_t>(__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3));
}

// y = silu(g) rounded to bf16, times u, rounded to bf16 (g, u already bf16 values).
// The fast exponential and division (a few ulp of fp32) are far below the
// bf16 rounding that follows; this runs 64 times per row in the GEMM1
// epilogue, where it is not hidden behind the MMA.  For g < -88, exp(-g) is
// +inf and the quotient is -0.
__device__ __forceinline__ float silu_mul_bf16(float g, float u) {
  const float s = bf16_round(__fdividef(g, 1.0f + __expf(-g)));
  return bf16_round(s * u);
}

// SwiGLU with an optional clamp (limit = +inf: none): gate = min(g, L),
// up = clamp(u, -L, L), then silu_mul_bf16.  g, u are bf16 values.
__device__ __forceinline__ float swiglu_bf16(float g, float u, float limit) {
  return silu_mul_bf16(fminf(g, limit), fminf(fmaxf(u, -limit), limit));
}

// routed weight of flat assignment `flat`, or 1 when it was applied to the input
__device__ __forceinline__ float route_weight(const float* topk_weights, int flat) {
  return topk_weights ? (*(topk_weights + flat)) : 1.0f;
}

}  // namespace moe
