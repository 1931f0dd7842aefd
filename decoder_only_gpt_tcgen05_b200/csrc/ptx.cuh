// Thin inline-PTX layer for sm_100a: mbarriers with bounded waits, TMA tile
// loads, and the tcgen05 tensor-core / tensor-memory instructions.
//
// Every wait on an mbarrier is bounded in wall time (%globaltimer).  When a
// wait runs out the kernel records an error in the device status word, raises
// a CTA-wide abort flag so that its other warps stop waiting too, and returns;
// the host reads the status word after the stream synchronises.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gptk {

// ----------------------------------------------------------------- status

// Device status word: 0 = fine; otherwise (code << 24) | (site << 16) | (block & 0xffff).
struct DevCtl {
  unsigned int* status;        // one word in device memory (owned by the library)
  unsigned long long timeout_ns;
};

enum : unsigned int { DEV_ERR_TIMEOUT = 1u };

__device__ __forceinline__ void dev_report(const DevCtl& c, unsigned int code, unsigned int site) {
  unsigned int v = (code << 24) | ((site & 0xffu) << 16) | (blockIdx.x & 0xffffu);
  atomicCAS(c.status, 0u, v);
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ----------------------------------------------------------------- programmatic dependent launch
//
// A kernel launched with programmatic stream serialization (launch_pdl) may start while the
// kernel before it on the stream is still finishing: its prologue (barrier set-up, TMEM
// allocation, tensor-map prefetch) overlaps the other kernel's last CTAs.  pdl_wait() blocks until
// that kernel has completed and its memory is visible; every thread runs it before its first
// global load or store.  pdl_trigger() lets the next kernel be scheduled as soon as every CTA of
// this one has started (it changes nothing for a kernel launched the usual way).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ----------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait until the phase with the given parity has completed.  Returns false
// (after raising *abort and recording the site) when the wall-time limit runs
// out, or when another warp of the CTA has already aborted.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, const DevCtl& ctl,
                                          volatile int* abort_flag, unsigned int site) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0u) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > ctl.timeout_ns) {
        *abort_flag = 1;
        dev_report(ctl, DEV_ERR_TIMEOUT, site);
        return false;
      }
    }
  }
}

// ----------------------------------------------------------------- TMA

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          smem_u32(dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

// ----------------------------------------------------------------- CTA pairs (cluster of 2)
//
// Two CTAs of a cluster can share one tcgen05.mma (cta_group::2): each supplies half of the A
// rows and half of the B rows from its own shared memory at the same offsets, and each holds
// its half of the accumulator rows in its own tensor memory.

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
__device__ __forceinline__ uint32_t cluster_count_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
// shared::cluster address of the same shared-memory location in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t mapa_shared(uint32_t cta_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(cta_addr), "r"(rank));
  return r;
}
// every thread of both CTAs: cluster-wide execution barrier (memory ordered release/acquire)
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// arrive on an mbarrier given by its shared::cluster address (this CTA's or the peer's)
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// TMA tile load into this CTA's shared memory whose completion is counted on an mbarrier of
// either CTA of the pair (given by its shared::cluster address)
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint32_t bar_cluster, int c0,
                                                 int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(bar_cluster), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                            int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::
          "r"(smem_u32(dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// shared -> global tile store (bulk async-group completion)
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int c0, int c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(map),
               "r"(smem_u32(src)), "r"(c0), "r"(c1)
               : "memory");
}

// global += shared tile (element-wise add performed at L2)
__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap* map, const void* src, int c0, int c1) {
  asm volatile("cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   map),
               "r"(smem_u32(src)), "r"(c0), "r"(c1)
               : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// wait until at most N committed bulk groups still read their shared-memory source
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// wait until every committed bulk group has completed
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// generic-proxy shared-memory writes -> visible to the async proxy (tensor core, TMA)
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ----------------------------------------------------------------- tcgen05

__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)), "r"(ncols)
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
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem] * B[smem]^T  (kind::f16, bf16 inputs, fp32 accumulate), issued by one thread
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Eight MMAs issued back to back from one asm block, every operand in a register beforehand and
// the eight enable-accumulate predicates set up front (bit i of acc_mask for MMA i).  The issue
// of tcgen05.mma is synchronous with the tensor pipe, so any instruction between two MMAs
// lengthens the pipe's cycle; this form leaves none.
__device__ __forceinline__ void umma8_ss(const uint32_t (&d)[8], const uint64_t (&a)[8], const uint64_t (&b)[8],
                                         uint32_t idesc, uint32_t acc_mask) {
  asm volatile(
      "{\n\t.reg .pred p<8>;\n\t.reg .b32 t<8>;\n\t"
      "and.b32 t0, %25, 1;\n\tsetp.ne.b32 p0, t0, 0;\n\t"
      "and.b32 t1, %25, 2;\n\tsetp.ne.b32 p1, t1, 0;\n\t"
      "and.b32 t2, %25, 4;\n\tsetp.ne.b32 p2, t2, 0;\n\t"
      "and.b32 t3, %25, 8;\n\tsetp.ne.b32 p3, t3, 0;\n\t"
      "and.b32 t4, %25, 16;\n\tsetp.ne.b32 p4, t4, 0;\n\t"
      "and.b32 t5, %25, 32;\n\tsetp.ne.b32 p5, t5, 0;\n\t"
      "and.b32 t6, %25, 64;\n\tsetp.ne.b32 p6, t6, 0;\n\t"
      "and.b32 t7, %25, 128;\n\tsetp.ne.b32 p7, t7, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %8, %16, %24, p0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%1], %9, %17, %24, p1;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%2], %10, %18, %24, p2;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%3], %11, %19, %24, p3;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%4], %12, %20, %24, p4;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%5], %13, %21, %24, p5;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%6], %14, %22, %24, p6;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%7], %15, %23, %24, p7;\n\t"
      "}"
      ::"r"(d[0]), "r"(d[1]), "r"(d[2]), "r"(d[3]), "r"(d[4]), "r"(d[5]), "r"(d[6]), "r"(d[7]),
      "l"(a[0]), "l"(a[1]), "l"(a[2]), "l"(a[3]), "l"(a[4]), "l"(a[5]), "l"(a[6]), "l"(a[7]),
      "l"(b[0]), "l"(b[1]), "l"(b[2]), "l"(b[3]), "l"(b[4]), "l"(b[5]), "l"(b[6]), "l"(b[7]), "r"(idesc),
      "r"(acc_mask)
      : "memory");
}
// Four MMAs into one accumulator, back to back (one K = 64 stage of a GEMM); bit i of acc_mask
// enables accumulation for MMA i.  The pair form is the cta_group::2 MMA of a CTA pair.
__device__ __forceinline__ void umma4_ss(uint32_t d, const uint64_t (&a)[4], const uint64_t (&b)[4], uint32_t idesc,
                                         uint32_t acc_mask) {
  asm volatile(
      "{\n\t.reg .pred p<4>;\n\t.reg .b32 t<4>;\n\t"
      "and.b32 t0, %10, 1;\n\tsetp.ne.b32 p0, t0, 0;\n\t"
      "and.b32 t1, %10, 2;\n\tsetp.ne.b32 p1, t1, 0;\n\t"
      "and.b32 t2, %10, 4;\n\tsetp.ne.b32 p2, t2, 0;\n\t"
      "and.b32 t3, %10, 8;\n\tsetp.ne.b32 p3, t3, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %5, %9, p0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %2, %6, %9, p1;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %3, %7, %9, p2;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %4, %8, %9, p3;\n\t"
      "}"
      ::"r"(d), "l"(a[0]), "l"(a[1]), "l"(a[2]), "l"(a[3]), "l"(b[0]), "l"(b[1]), "l"(b[2]), "l"(b[3]), "r"(idesc),
      "r"(acc_mask)
      : "memory");
}
__device__ __forceinline__ void umma4_ss_pair(uint32_t d, const uint64_t (&a)[4], const uint64_t (&b)[4],
                                              uint32_t idesc, uint32_t acc_mask) {
  asm volatile(
      "{\n\t.reg .pred p<4>;\n\t.reg .b32 t<4>;\n\t"
      "and.b32 t0, %10, 1;\n\tsetp.ne.b32 p0, t0, 0;\n\t"
      "and.b32 t1, %10, 2;\n\tsetp.ne.b32 p1, t1, 0;\n\t"
      "and.b32 t2, %10, 4;\n\tsetp.ne.b32 p2, t2, 0;\n\t"
      "and.b32 t3, %10, 8;\n\tsetp.ne.b32 p3, t3, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %5, %9, p0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %2, %6, %9, p1;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %3, %7, %9, p2;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %4, %8, %9, p3;\n\t"
      "}"
      ::"r"(d), "l"(a[0]), "l"(a[1]), "l"(a[2]), "l"(a[3]), "l"(b[0]), "l"(b[1]), "l"(b[2]), "l"(b[3]), "r"(idesc),
      "r"(acc_mask)
      : "memory");
}
// the same with A read from tensor memory: each A is an M x 16 bf16 block stored two per 32-bit
// column (element (m, k) at lane m, column k / 2 from the given address)
__device__ __forceinline__ void umma8_ts(const uint32_t (&d)[8], const uint32_t (&a)[8], const uint64_t (&b)[8],
                                         uint32_t idesc, uint32_t acc_mask) {
  asm volatile(
      "{\n\t.reg .pred p<8>;\n\t.reg .b32 t<8>;\n\t"
      "and.b32 t0, %25, 1;\n\tsetp.ne.b32 p0, t0, 0;\n\t"
      "and.b32 t1, %25, 2;\n\tsetp.ne.b32 p1, t1, 0;\n\t"
      "and.b32 t2, %25, 4;\n\tsetp.ne.b32 p2, t2, 0;\n\t"
      "and.b32 t3, %25, 8;\n\tsetp.ne.b32 p3, t3, 0;\n\t"
      "and.b32 t4, %25, 16;\n\tsetp.ne.b32 p4, t4, 0;\n\t"
      "and.b32 t5, %25, 32;\n\tsetp.ne.b32 p5, t5, 0;\n\t"
      "and.b32 t6, %25, 64;\n\tsetp.ne.b32 p6, t6, 0;\n\t"
      "and.b32 t7, %25, 128;\n\tsetp.ne.b32 p7, t7, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%8], %16, %24, p0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%1], [%9], %17, %24, p1;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%2], [%10], %18, %24, p2;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%3], [%11], %19, %24, p3;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%4], [%12], %20, %24, p4;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%5], [%13], %21, %24, p5;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%6], [%14], %22, %24, p6;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%7], [%15], %23, %24, p7;\n\t"
      "}"
      ::"r"(d[0]), "r"(d[1]), "r"(d[2]), "r"(d[3]), "r"(d[4]), "r"(d[5]), "r"(d[6]), "r"(d[7]),
      "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(a[4]), "r"(a[5]), "r"(a[6]), "r"(a[7]),
      "l"(b[0]), "l"(b[1]), "l"(b[2]), "l"(b[3]), "l"(b[4]), "l"(b[5]), "l"(b[6]), "l"(b[7]), "r"(idesc),
      "r"(acc_mask)
      : "memory");
}

// Four MMAs of kind::f8f6f4 (8-bit A and B, fp32 accumulate, K = 32 each), back to back; the
// pair form is the cta_group::2 MMA of a CTA pair.  The formats are in the instruction descriptor.
__device__ __forceinline__ void umma4_f8(uint32_t d, const uint64_t (&a)[4], const uint64_t (&b)[4], uint32_t idesc,
                                         uint32_t acc_mask) {
  asm volatile(
      "{\n\t.reg .pred p<4>;\n\t.reg .b32 t<4>;\n\t"
      "and.b32 t0, %10, 1;\n\tsetp.ne.b32 p0, t0, 0;\n\t"
      "and.b32 t1, %10, 2;\n\tsetp.ne.b32 p1, t1, 0;\n\t"
      "and.b32 t2, %10, 4;\n\tsetp.ne.b32 p2, t2, 0;\n\t"
      "and.b32 t3, %10, 8;\n\tsetp.ne.b32 p3, t3, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %5, %9, p0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %2, %6, %9, p1;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %3, %7, %9, p2;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %4, %8, %9, p3;\n\t"
      "}"
      ::"r"(d), "l"(a[0]), "l"(a[1]), "l"(a[2]), "l"(a[3]), "l"(b[0]), "l"(b[1]), "l"(b[2]), "l"(b[3]), "r"(idesc),
      "r"(acc_mask)
      : "memory");
}
__device__ __forceinline__ void umma4_f8_pair(uint32_t d, const uint64_t (&a)[4], const uint64_t (&b)[4],
                                              uint32_t idesc, uint32_t acc_mask) {
  asm volatile(
      "{\n\t.reg .pred p<4>;\n\t.reg .b32 t<4>;\n\t"
      "and.b32 t0, %10, 1;\n\tsetp.ne.b32 p0, t0, 0;\n\t"
      "and.b32 t1, %10, 2;\n\tsetp.ne.b32 p1, t1, 0;\n\t"
      "and.b32 t2, %10, 4;\n\tsetp.ne.b32 p2, t2, 0;\n\t"
      "and.b32 t3, %10, 8;\n\tsetp.ne.b32 p3, t3, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %5, %9, p0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %2, %6, %9, p1;\n\t"
      "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %3, %7, %9, p2;\n\t"
      "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %4, %8, %9, p3;\n\t"
      "}"
      ::"r"(d), "l"(a[0]), "l"(a[1]), "l"(a[2]), "l"(a[3]), "l"(b[0]), "l"(b[1]), "l"(b[2]), "l"(b[3]), "r"(idesc),
      "r"(acc_mask)
      : "memory");
}

// Arrive once on the mbarrier at `bar_cluster` (either CTA of the pair) when every pair MMA
// issued so far by this thread has completed.
__device__ __forceinline__ void umma_commit_pair(uint32_t bar_cluster) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar_cluster)
               : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// Arrive once on the mbarrier when every tcgen05 op issued so far by this thread has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B.
// a_mn / b_mn: 1 when the operand is stored MN-major (transposed) in shared memory.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(a_mn) << 15) |
         (static_cast<uint32_t>(b_mn) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// Instruction descriptor, kind::f8f6f4: fp32 accumulator, A and B in the 8-bit formats fa, fb
// (0 = e4m3, 1 = e5m2), both K-major.
__host__ __device__ constexpr uint32_t idesc_f8(int M, int N, int fa, int fb) {
  return (1u << 4) | (static_cast<uint32_t>(fa) << 7) | (static_cast<uint32_t>(fb) << 10) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// fp32 pair -> two 8-bit floats (round to nearest even, saturating at the largest finite value);
// the first value in the low byte
__device__ __forceinline__ uint16_t cvt_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ uint16_t cvt_e5m2x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Shared-memory matrix descriptor for a 128-byte-swizzled operand.
//   K-major : rows of 128 B (64 bf16 along K), 8-row groups SBO apart (LBO unused).
//   MN-major: rows of 128 B (64 bf16 along M/N), one row per K index, 8-row
//             groups SBO apart, further 64-wide M/N chunks LBO apart.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;  // descriptor version for sm_100
  d |= 2ull << 61;  // SWIZZLE_128B
  return d;
}

// A descriptor moved by `byte_off` bytes within the same operand: one 32-bit add on the start-
// address field (bits [4,18) of the shared-memory address; shared memory stays below 256 KB, so
// the field cannot carry into the next one).  Keeps the single MMA-issuing thread lean: it
// shares its SM sub-partition with busy elementwise warps.
__device__ __forceinline__ uint64_t sdesc_add(uint64_t d, uint32_t byte_off) {
  const uint32_t lo = static_cast<uint32_t>(d) + (byte_off >> 4);
  return (static_cast<uint64_t>(static_cast<uint32_t>(d >> 32)) << 32) | lo;
}

// 32 lanes x 32 consecutive 32-bit columns: thread t of the warp gets lane (quadrant*32 + t).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  // the wait names every destination register so that no use of them can be
  // scheduled ahead of it
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]),"+r"(r[1]),"+r"(r[2]),"+r"(r[3]),"+r"(r[4]),"+r"(r[5]),"+r"(r[6]),"+r"(r[7]),"+r"(r[8]),"+r"(r[9]),"+r"(r[10]),"+r"(r[11]),"+r"(r[12]),"+r"(r[13]),"+r"(r[14]),"+r"(r[15]),"+r"(r[16]),"+r"(r[17]),"+r"(r[18]),"+r"(r[19]),"+r"(r[20]),"+r"(r[21]),"+r"(r[22]),"+r"(r[23]),"+r"(r[24]),"+r"(r[25]),"+r"(r[26]),"+r"(r[27]),"+r"(r[28]),"+r"(r[29]),"+r"(r[30]),"+r"(r[31])
               :
               : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// 32 lanes x 32 columns without waiting: several loads can be in flight before one
// tmem_wait_ld(); the registers must then pass through tmem_fence_regs() before use.
__device__ __forceinline__ void tmem_ld32_nowait(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
// 32 lanes x 16 consecutive 32-bit columns, without waiting (see tmem_ld32_nowait)
__device__ __forceinline__ void tmem_ld16_nowait(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// 32 lanes x 8 / 16 consecutive 32-bit columns from registers; tmem_wait_st() before the data
// is handed to an MMA
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* w) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(w[0]),
               "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* w) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]), "r"(w[8]), "r"(w[9]),
      "r"(w[10]), "r"(w[11]), "r"(w[12]), "r"(w[13]), "r"(w[14]), "r"(w[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// orders every later use of r[0..n) after the preceding tmem_wait_ld()
template <int N>
__device__ __forceinline__ void tmem_fence_regs(uint32_t* r) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ----------------------------------------------------------------- math helpers

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Packed fp32 pairs (sm_100 f32x2 instructions: one instruction for two lanes' worth of work).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  uint64_t d;
  asm("{\n\t.reg .b64 pa, pb, pc;\n\tmov.b64 pa, {%1, %2};\n\tmov.b64 pb, {%3, %4};\n\tmov.b64 pc, {%5, %6};\n\t"
      "fma.rn.f32x2 %0, pa, pb, pc;\n\t}"
      : "=l"(d)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(d));
  return r;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  uint64_t d;
  asm("{\n\t.reg .b64 pa, pb;\n\tmov.b64 pa, {%1, %2};\n\tmov.b64 pb, {%3, %4};\n\t"
      "add.rn.f32x2 %0, pa, pb;\n\t}"
      : "=l"(d)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(d));
  return r;
}
// max of three (one instruction on sm_100)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^x for two values at once on the FMA and integer pipes instead of the MUFU unit, so that a
// kernel bound by the MUFU's 16 results per clock can move part of its exponentials elsewhere.
// Range reduction x = n + f with n = rint(x), taken exactly from the low mantissa bits of
// x + 1.5 * 2^23 (f in [-1/2, 1/2]); 2^f from a degree-4 polynomial, the Remez minimax fit of 2^f
// on [-1/2, 1/2] in relative error computed for this library (2.6e-6 exactly, 2.7e-6 with these
// fp32 coefficients and Horner steps); n added to the exponent field.  Within that error for
// -125 <= x <= 127; x is clamped below at -126, so x < -125 (-inf included) gives a value in
// [0, 2^-125] instead of 2^x.
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  constexpr float kShift = 12582912.f;  // 1.5 * 2^23
  x = make_float2(fmaxf(x.x, -126.f), fmaxf(x.y, -126.f));
  const float2 j = fadd2(x, make_float2(kShift, kShift));
  const float2 n = fadd2(j, make_float2(-kShift, -kShift));
  const float2 f = ffma2(n, make_float2(-1.f, -1.f), x);  // x - n, exact
  float2 q = ffma2(make_float2(0.009570102207362652f, 0.009570102207362652f), f,
                   make_float2(0.05591785907745361f, 0.05591785907745361f));
  q = ffma2(q, f, make_float2(0.240247443318367f, 0.240247443318367f));
  q = ffma2(q, f, make_float2(0.6931217908859253f, 0.6931217908859253f));
  q = ffma2(q, f, make_float2(0.9999992847442627f, 0.9999992847442627f));
  return make_float2(__int_as_float(__float_as_int(q.x) + (__float_as_int(j.x) << 23)),
                     __int_as_float(__float_as_int(q.y) + (__float_as_int(j.y) << 23)));
}

// Register budget of a warpgroup (all 128 threads execute it): give back / take registers.
template <int N>
__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

// Hardware square root (sqrt.approx: +0 maps to +0; its error of a few ulp is far below bf16
// rounding).  The IEEE sqrtf leaves its fast path for zero inputs, which ReLU^2 makes common.
__device__ __forceinline__ float sqrt_approx(float x) {
  float y;
  asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float bf16_to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

}  // namespace gptk
