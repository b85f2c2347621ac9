// tcf4_pipe.cuh -- bulk-copy (TMA 1-D) staging of row slabs into a shared-memory ring.
//
// A CTA streams slabs of consecutive rows (stream words, then scale bytes) into NS shared-memory
// buffers with cp.async.bulk, one elected thread issuing each slab, completion tracked by one
// mbarrier per buffer (transaction bytes). Consumers wait on the buffer's barrier with a bounded
// spin; a wait that runs out increments a device counter of its kernel file (read and cleared by
// tcf4_device_timeouts) and the kernel finishes without using the buffer. No copy is ever
// multicast, and every source is this GPU's own memory.
#pragma once
#include <cstdint>

namespace tcf4 {

// A wait gives up after about two seconds (kWaitCycles SM clock cycles), far beyond any real wait
// (microseconds).
constexpr long long kWaitCycles = 4000000000ll;

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

// One try_wait: the thread sleeps until the phase with the given parity completes (it is woken
// then) or at most ~kSuspendNs; true once that phase has completed.
constexpr uint32_t kSuspendNs = 1000000u;
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendNs)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase with the given parity to complete. Returns false on timeout, after
// counting it in *timeouts.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, unsigned int *timeouts) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  do {
    if (mbar_try_wait(bar, parity)) return true;
  } while (clock64() - t0 < kWaitCycles);
  atomicAdd(timeouts, 1u);
  return false;
}

// Global -> shared bulk copy of `bytes` (multiple of 16, both addresses 16-byte aligned),
// completing `bytes` transaction bytes on `bar`.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ uint2 lds_u2(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t lds_u8(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ float4 lds_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
  return v;
}

__host__ __device__ constexpr uint32_t round_up(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

// One slab: `nrows` rows of `st_row` stream bytes and `sc_row` scale bytes each.
struct Slab {
  const unsigned char *st;  // global source of the stream words
  const unsigned char *sc;  // global source of the scale bytes
  uint32_t nrows;
};

// Shared-memory ring of NS slab buffers with their barriers, and the per-thread phase bits.
template <int NS>
struct SlabRing {
  uint64_t *full;       // NS mbarriers
  unsigned char *buf;   // NS buffers of `stride` bytes: stream part at 0, scales at `sc_off`
  uint32_t stride, sc_off, st_row, sc_row;
  int bulk_scales;      // scales may be bulk-copied (16-byte aligned base and row slabs)
  uint32_t phase_bits;  // per buffer: parity of the next phase to wait for
  unsigned int *timeouts;  // device counter of waits that gave up

  __device__ bool st_bulk(uint32_t nrows) const { return (nrows * st_row) % 16u == 0u; }
  __device__ bool sc_bulk(uint32_t nrows) const { return bulk_scales && (nrows * sc_row) % 16u == 0u; }

  // Producer side (one thread): arm buffer b and start the bulk copies of `nparts` slabs with the
  // same row count; part p's rows start at row p * cap of the buffer (stream and scales alike).
  __device__ void issue_parts(int b, const Slab *parts, int nparts, uint32_t cap) const {
    const uint32_t nrows = parts[0].nrows;
    if (!st_bulk(nrows)) return;  // copied cooperatively at consume time
    const uint32_t st_bytes = nrows * st_row;
    const uint32_t sc_bytes = sc_bulk(nrows) ? nrows * sc_row : 0u;
    mbar_arrive_expect_tx(&full[b], (uint32_t)nparts * (st_bytes + sc_bytes));
    unsigned char *d = buf + (size_t)b * stride;
    for (int p = 0; p < nparts; p++) {
      bulk_g2s(d + p * cap * st_row, parts[p].st, st_bytes, &full[b]);
      if (sc_bytes) bulk_g2s(d + sc_off + p * cap * sc_row, parts[p].sc, sc_bytes, &full[b]);
    }
  }

  // Consumer side (all threads, uniform control flow): make buffer b hold the slabs. Returns false
  // if a bounded wait ran out (the caller then skips the slabs). Ends with the data visible to all.
  __device__ bool acquire_parts(int b, const Slab *parts, int nparts, uint32_t cap) {
    bool ok = true;
    const uint32_t nrows = parts[0].nrows;
    const bool sb = st_bulk(nrows), cb = sb && sc_bulk(nrows);
    if (sb) {
      ok = mbar_wait(&full[b], (phase_bits >> b) & 1u, timeouts);
      phase_bits ^= 1u << b;
    }
    if (!sb || !cb) {  // cooperative copies of whatever was not bulk-copied
      unsigned char *d = buf + (size_t)b * stride;
      for (int p = 0; p < nparts; p++) {
        if (!sb)
          for (uint32_t i = threadIdx.x; i < nrows * st_row / 8u; i += blockDim.x)
            reinterpret_cast<uint2 *>(d + p * cap * st_row)[i] = reinterpret_cast<const uint2 *>(parts[p].st)[i];
        for (uint32_t i = threadIdx.x; i < nrows * sc_row; i += blockDim.x)
          d[sc_off + p * cap * sc_row + i] = parts[p].sc[i];
      }
      __syncthreads();
    }
    return ok;
  }

  __device__ void issue(int b, const Slab &s) const { issue_parts(b, &s, 1, 0u); }
  __device__ bool acquire(int b, const Slab &s) { return acquire_parts(b, &s, 1, 0u); }
  __device__ void issue2(int b, const Slab &s0, const Slab &s1, uint32_t cap) const {
    const Slab parts[2] = {s0, s1};
    issue_parts(b, parts, 2, cap);
  }
  __device__ bool acquire2(int b, const Slab &s0, const Slab &s1, uint32_t cap) {
    const Slab parts[2] = {s0, s1};
    return acquire_parts(b, parts, 2, cap);
  }
};

}  // namespace tcf4
