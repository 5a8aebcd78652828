// Device helpers shared by the libpkv kernels (sm_100a): mbarriers, TMA tensor
// loads, bulk copies, bounded waits and bf16 packing.  Inline PTX only; no
// library kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define PKV_DEVINL __device__ __forceinline__

namespace pkv {

// Device status word bits (workspace header); the host maps them to PKV_ERR_*.
enum : uint32_t {
  kStatusBadTable = 1u,
  kStatusTimeout = 2u,
  kStatusPlanMismatch = 4u,
};

// A bounded wait gives up after this many nanoseconds of %globaltimer.  Long
// enough never to trigger on a healthy launch (a tile lands in microseconds),
// short enough that a broken pipeline ends the launch instead of hanging it.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s
// After a timeout, each copy still in flight gets this much longer.
constexpr uint64_t kDrainLimitNs = 50000000ull;    // 50 ms

// 2^x by the hardware approximation (PTX ex2.approx.ftz: relative error
// below 2^-22; -inf gives +0).  The softmax weights it feeds are rounded to
// bf16 (2^-9) before they multiply V.
PKV_DEVINL float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

PKV_DEVINL uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

PKV_DEVINL uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

PKV_DEVINL void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

PKV_DEVINL void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

PKV_DEVINL void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

PKV_DEVINL void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

// Raise the expected transaction count of the current phase without arriving.
PKV_DEVINL void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

PKV_DEVINL void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Programmatic dependent launch: let the next kernel of the stream be
// scheduled, and wait until the kernels this one depends on have completed
// and their writes are visible (no-ops for a launch without the attribute).
PKV_DEVINL void grid_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
PKV_DEVINL void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

PKV_DEVINL bool mbar_try_wait(uint32_t bar, uint32_t parity) {
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

// Wait for phase `parity` of an mbarrier, for at most limit_ns.  Returns
// false (and the caller records kStatusTimeout) if the phase never completed.
PKV_DEVINL bool mbar_wait_bounded(uint32_t bar, uint32_t parity, uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  uint32_t spins = 0;
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((++spins & 63u) == 0 && globaltimer() - t0 > limit_ns) return false;
  }
}

// L2 policy for data read once (the KV stream): evict first, so tables,
// queries and partial states keep their L2 lines.
PKV_DEVINL uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// 4-D tiled TMA load global -> shared, completing on an mbarrier.
PKV_DEVINL void tma_load_4d(uint32_t dst, const void* tmap, int32_t c0, int32_t c1, int32_t c2,
                            int32_t c3, uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3, %4, %5}], [%6], %7;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar),
      "l"(policy)
      : "memory");
}

// 5-D tiled TMA load global -> shared, completing on an mbarrier.
PKV_DEVINL void tma_load_5d(uint32_t dst, const void* tmap, int32_t c0, int32_t c1, int32_t c2,
                            int32_t c3, int32_t c4, uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3, %4, %5, %6}], [%7], %8;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(bar),
      "l"(policy)
      : "memory");
}

// Contiguous bulk copy global -> shared (size and both addresses 16-B aligned).
PKV_DEVINL void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Reduction (no value returned) with release semantics at GPU scope: the
// thread's earlier writes are visible before the addition.
PKV_DEVINL void red_release_gpu_add(unsigned* addr, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(addr), "r"(v) : "memory");
}
// Load with acquire semantics at GPU scope.
PKV_DEVINL unsigned ld_acquire_gpu(const unsigned* addr) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(addr) : "memory");
  return v;
}

// Atomic add with acquire-release semantics at GPU scope.
PKV_DEVINL int atomic_add_acq_rel_gpu(int* addr, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(addr), "r"(v) : "memory");
  return old;
}

PKV_DEVINL float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
PKV_DEVINL float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

PKV_DEVINL void record_status(uint32_t* status, uint32_t bit) {
  if (status) atomicOr(status, bit);
}

template <typename T>
struct Elem;
template <>
struct Elem<__nv_bfloat16> {
  static constexpr int kBytes = 2;
};
template <>
struct Elem<float> {
  static constexpr int kBytes = 4;
};

}  // namespace pkv
