// common.cuh -- device helpers shared by the kernels of libsparse_decode:
// status flags, bounded mbarrier waits, 1-D bulk (TMA) copies, the
// order-preserving score key, and dtype helpers.  sm_100a only.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sd {

// ---- device status word (first 4 bytes of the workspace) -----------------
enum : uint32_t {
  FLAG_NONFINITE = 1u << 0,
  FLAG_CAPACITY = 1u << 1,
  FLAG_TIMEOUT = 1u << 2,
  FLAG_INDEX = 1u << 3,
  FLAG_INTERNAL = 1u << 4,
  // informational, not an error: a top-k select took its exact streaming
  // path (its fast path's preconditions did not hold for some head)
  FLAG_SLOW_SELECT = 1u << 8,
};

__device__ __forceinline__ void raise_flag(uint32_t *status, uint32_t f) {
  if (status) atomicOr(status, f);
}

// Bounded waits give up after this many nanoseconds of %globaltimer.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Counter barriers in global memory: wait (one thread) until *ctr >= target,
// with acquire loads and short sleeps; false, and the TIMEOUT flag, if that
// has not happened within limit_ns of %globaltimer.  Every kernel whose CTAs
// wait for one another waits here.
__device__ __forceinline__ bool wait_counter_geq(const uint32_t *ctr, uint32_t target,
                                                 uint64_t limit_ns, uint32_t *status) {
  const uint64_t t0 = global_ns();
  while (true) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
    if (v >= target) return true;
    if (global_ns() - t0 > limit_ns) {
      raise_flag(status, FLAG_TIMEOUT);
      return false;
    }
    __nanosleep(32);
  }
}

// ---- programmatic dependent launch ----------------------------------------
// Every kernel waits here before touching memory that an earlier kernel on
// the stream may still be writing (a no-op unless launched with programmatic
// stream serialisation), then lets its own dependents start launching.
__device__ __forceinline__ void grid_dep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_dep_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---- mbarrier -------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- thread-block clusters ------------------------------------------------
// Shared-memory address of `p` in the CTA of the cluster with rank `rank`,
// and loads and stores through such an address (distributed shared memory).
__device__ __forceinline__ uint32_t cl_addr(const void *p, int rank) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(p)), "r"(rank));
  return a;
}
__device__ __forceinline__ uint32_t cl_ld_u32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ float4 cl_ld4(uint32_t a) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(a)
               : "memory");
  return v;
}
__device__ __forceinline__ void cl_st2(uint32_t a, float2 v) {
  asm volatile("st.shared::cluster.v2.f32 [%0], {%1,%2};" ::"r"(a), "f"(v.x), "f"(v.y)
               : "memory");
}
// Every thread of every CTA of the cluster: the writes before it (shared
// memory included) are visible to the reads after it, in every CTA.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
               "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar,
                                                      uint32_t bytes) {
  asm volatile(
      "mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(
          smem_u32(bar)),
      "r"(bytes)
      : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
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

// Wait for the phase with the given parity to complete; false (and the
// TIMEOUT flag) if it has not completed within kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity,
                                          uint32_t *status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > kWaitLimitNs) {
      raise_flag(status, FLAG_TIMEOUT);
      return false;
    }
  }
  return true;
}

// ---- shared-memory atomics addressed in the shared window -----------------
// (explicit .shared forms: no generic-address resolution on a hot path)
__device__ __forceinline__ void sh_red_or(uint32_t *p, uint32_t v) {
  asm volatile("red.shared.or.b32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}
__device__ __forceinline__ void sh_red_add(uint32_t *p, uint32_t v) {
  asm volatile("red.shared.add.u32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t sh_atom_add(uint32_t *p, uint32_t v) {
  uint32_t r;
  asm volatile("atom.shared.add.u32 %0, [%1], %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(v)
               : "memory");
  return r;
}

// ---- 1-D bulk copy global -> shared (TMA, no tensor map) ------------------
// Both addresses 16-byte aligned, bytes a multiple of 16.  Completion is
// signalled as transaction bytes on `bar`.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;"
               : "=l"(pol));
  return pol;
}

__device__ __forceinline__ void bulk_g2s(void *smem_dst, const void *gmem_src,
                                         uint32_t bytes, uint64_t *bar,
                                         uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void bulk_g2s(void *smem_dst, const void *gmem_src,
                                         uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1], %2, [%3];" ::"r"(smem_u32(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// ---- order-preserving key of an fp32 score --------------------------------
// Larger score -> larger unsigned key; -0.0 maps like +0.0, so equal scores
// give equal keys.
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---- dtype helpers --------------------------------------------------------
template <typename T>
struct DT;
template <>
struct DT<float> {
  static constexpr int kCode = 0;
  __device__ static float to_f(float x) { return x; }
  __device__ static float from_f(float x) { return x; }
};
template <>
struct DT<__nv_bfloat16> {
  static constexpr int kCode = 1;
  __device__ static float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
  __device__ static __nv_bfloat16 from_f(float x) {
    return __float2bfloat16_rn(x);
  }
};

// Unpack a 16-byte vector of T into fp32.  bf16 widens exactly by a shift.
template <typename T>
__device__ __forceinline__ void unpack16(const uint4 &v, float *f);
template <>
__device__ __forceinline__ void unpack16<float>(const uint4 &v, float *f) {
  f[0] = __uint_as_float(v.x);
  f[1] = __uint_as_float(v.y);
  f[2] = __uint_as_float(v.z);
  f[3] = __uint_as_float(v.w);
}
template <>
__device__ __forceinline__ void unpack16<__nv_bfloat16>(const uint4 &v,
                                                        float *f) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ uint4 lds128(const void *p) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(smem_u32(p)));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1)
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

}  // namespace sd
