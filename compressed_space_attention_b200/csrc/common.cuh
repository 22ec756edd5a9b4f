// Device helpers shared by the libisoq kernels (sm_100a): mbarriers, TMA and
// bulk copies (CTA-local, never multicast), bounded waits, small math.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"

namespace isoq {
namespace dev {

// Error codes a kernel ORs into its translation unit's device error word.
constexpr unsigned kErrWaitTimeout = 1u;

// A bounded wait gives up after this much wall time (globaltimer, ns).
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t *bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
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

// Waits for the phase with the given parity to complete.  Returns false if
// kWaitLimitNs passed first (the caller then reports a timeout and stops).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  for (unsigned it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 63u && globaltimer() - t0 > kWaitLimitNs) return false;
  }
}

// ---------------------------------------------------------------------------
// Async copies (global -> shared through the TMA unit), CTA-local only.
// ---------------------------------------------------------------------------

// Tiled tensor load of one box; coordinates innermost first.
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, uint64_t *bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// Tiled tensor store of one box from shared memory (bulk-group completion).
__device__ __forceinline__ void tma_store_3d(const CUtensorMap *map, const void *src, int c0,
                                             int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// Contiguous bulk copy; dst, src and bytes must be multiples of 16.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes,
                                          uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Makes generic-proxy shared-memory writes visible to the async proxy.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void named_barrier(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---------------------------------------------------------------------------
// Quaternion helpers: (w, x, y, z), Hamilton convention ij = k.
// ---------------------------------------------------------------------------
struct Quat {
  float w, x, y, z;
};

__device__ __forceinline__ Quat qmul(const Quat &p, const Quat &q) {
  Quat r;
  r.w = p.w * q.w - p.x * q.x - p.y * q.y - p.z * q.z;
  r.x = p.w * q.x + p.x * q.w + p.y * q.z - p.z * q.y;
  r.y = p.w * q.y - p.x * q.z + p.y * q.w + p.z * q.x;
  r.z = p.w * q.z + p.x * q.y - p.y * q.x + p.z * q.w;
  return r;
}

__device__ __forceinline__ Quat qconj(const Quat &q) { return Quat{q.w, -q.x, -q.y, -q.z}; }

// Forward block map T(v) = q_L v conj(q_R) (Full) or q_L v (Fast).
__device__ __forceinline__ Quat block_forward(const Quat &ql, const Quat &qr, const Quat &v,
                                              bool full) {
  Quat u = qmul(ql, v);
  return full ? qmul(u, qconj(qr)) : u;
}

// Inverse (transpose) block map conj(q_L) u q_R (Full) or conj(q_L) u (Fast).
__device__ __forceinline__ Quat block_inverse(const Quat &ql, const Quat &qr, const Quat &u,
                                              bool full) {
  Quat v = qmul(qconj(ql), u);
  return full ? qmul(v, qr) : v;
}

__device__ __forceinline__ Quat load_quat(const float *p) {
  float4 v = *reinterpret_cast<const float4 *>(p);
  return Quat{v.x, v.y, v.z, v.w};
}

// Column c of the Sylvester H_4 (entries (-1)^popcount(r & c)).
__device__ __forceinline__ Quat h4_column(int c) {
  return Quat{1.0f, (c & 1) ? -1.0f : 1.0f, (c & 2) ? -1.0f : 1.0f,
              (__popc(c & 3) & 1) ? -1.0f : 1.0f};
}

// ---------------------------------------------------------------------------
// Packed float32 pairs (sm_100 f32x2 arithmetic): one instruction updates two
// lanes of a 64-bit register pair.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}

__device__ __forceinline__ void f2_unpack(uint64_t v, float &a, float &b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}

__device__ __forceinline__ uint64_t f2_swap(uint64_t v) {
  float a, b;
  f2_unpack(v, a, b);
  return f2_pack(b, a);
}

__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

// ---------------------------------------------------------------------------
// Packed-code layout.  b = 2, 4: LSB-first bitstream (code i at bits
// [b*i, b*i + b)).  b = 3: groups of 32 codes in three 32-bit words; code
// 8r + j of a group sits in bits [4j, 4j+3) of word r, and bit r of code
// 24 + j in bit 4j + 3 of word r, so that codes occupy 4-bit fields.
// ---------------------------------------------------------------------------

// ORs code number i (0 <= i < 64, compile-time after unrolling) of a 64-code
// run into the run's packed words w.
template <int BITS>
__device__ __forceinline__ void pack_code(uint32_t *w, int i, uint32_t code) {
  if constexpr (BITS == 3) {
    const int grp = i >> 5, m = i & 31;
    if (m < 24) {
      w[3 * grp + (m >> 3)] += code << (4 * (m & 7));
    } else {
      const int j = m - 24;
#pragma unroll
      for (int r = 0; r < 3; ++r) w[3 * grp + r] |= ((code >> r) & 1u) << (4 * j + 3);
    }
  } else {
    const int bp = BITS * i;
    w[bp >> 5] |= code << (bp & 31);
    if ((bp & 31) + BITS > 32) w[(bp >> 5) + 1] |= code >> (32 - (bp & 31));
  }
}

// Code number i of a run of packed words (the inverse of pack_code).
template <int BITS>
__device__ __forceinline__ uint32_t unpack_code(const uint32_t *w, int i) {
  if constexpr (BITS == 3) {
    const int grp = i >> 5, m = i & 31;
    if (m < 24) return (w[3 * grp + (m >> 3)] >> (4 * (m & 7))) & 7u;
    const int sh = 4 * (m - 24) + 3;
    return ((w[3 * grp] >> sh) & 1u) | (((w[3 * grp + 1] >> sh) & 1u) << 1) |
           (((w[3 * grp + 2] >> sh) & 1u) << 2);
  } else {
    const int bp = BITS * i;
    uint32_t c = w[bp >> 5] >> (bp & 31);
    if ((bp & 31) + BITS > 32) c |= w[(bp >> 5) + 1] << (32 - (bp & 31));
    return c & ((1u << BITS) - 1u);
  }
}

}  // namespace dev
}  // namespace isoq
