// Compressed-space split-K decode attention on sm_100a.
//
// RotaryQuant (arXiv 2608.08081) Figure 1 (bottom), §3.4 Table 2 kernels A-D,
// eq. (5) and Appendix A: the query is rotated once (q~ = R_K q), scores and
// the value sum are computed directly on the packed codes in the rotated
// domain, and the inverse rotation R_V^T is applied once to the merged output.
// K and V are never written out dequantised.
//
// Two launches:
//   split:   grid (n_splits, Hkv, B).  Each CTA owns one token chunk of one
//            (b, kvh) and all G = Hq/Hkv query heads sharing it; it writes one
//            partial state (m, l, acc[d]) per query head into the workspace,
//            acc in the rotated domain (online softmax, natural exponent).
//   combine: grid (Hq, B).  Merges the partials (m* = max m_k,
//            l = sum l_k e^(m_k - m*), o~ = sum acc_k e^(m_k - m*) / l), then
//            applies R_V^T = H_d R_SO4^T / sqrt(d) and stores the output.
//
// This file holds the generic split kernel (CUDA-core FMAs; any dtype, d and
// bits) and the combine kernel; decode_i8.cuh (included below) holds the
// integer tensor-core split kernel used for float16 queries with 3-bit codes,
// and decode_append.cuh the decode-step append.

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <mutex>

#include "common.cuh"
#include "tcgen05.cuh"
#include "decode.h"
#include "internal.h"

namespace isoq {
namespace decode {

using namespace isoq::dev;

__device__ unsigned int g_decode_error = 0;

// Launch with programmatic dependent launch: the kernel may start while the
// previous kernel on the stream is still running (once that kernel's CTAs
// have all started or signalled), and must execute griddepcontrol.wait
// before reading anything the previous kernel writes.  Used only for
// kernels whose predecessor is one of ours (prep -> split -> combine).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Barrier over the threads taking part in a shared-memory rotation: the whole
// CTA (bar_id 0 -> __syncthreads) or a named barrier over `nthreads` threads.
__device__ __forceinline__ void rotation_sync(int bar_id, int nthreads) {
  if (bar_id == 0)
    __syncthreads();
  else
    named_barrier(bar_id, nthreads);
}

// Forward rotation q~ = R q of `nvec` vectors v[nvec][D] held in shared
// memory, all sharing one head's parameters, by threads [0, nthreads): WHT
// butterflies (stride h = 1 ... d/2) for all vectors per barrier, 1/sqrt(d),
// then the per-block quaternion map.
template <int D, bool FULL>
__device__ void rotate_forward_smem(float *v, int nvec, const float *params_head, int tid,
                                    int nthreads, int bar_id) {
#pragma unroll 1
  for (int h = 1; h < D; h <<= 1) {
    for (int idx = tid; idx < nvec * (D / 2); idx += nthreads) {
      const int g = idx / (D / 2), p = idx % (D / 2);
      float *w = v + g * D;
      const int i = (p / h) * 2 * h + (p % h);
      const float a = w[i], b = w[i + h];
      w[i] = a + b;
      w[i + h] = a - b;
    }
    rotation_sync(bar_id, nthreads);
  }
  const float inv = rsqrtf(static_cast<float>(D));
  for (int idx = tid; idx < nvec * (D / 4); idx += nthreads) {
    const int g = idx / (D / 4), bi = idx % (D / 4);
    float *w = v + g * D + 4 * bi;
    const Quat x{w[0] * inv, w[1] * inv, w[2] * inv, w[3] * inv};
    const Quat u = block_forward(load_quat(params_head + 8 * bi), load_quat(params_head + 8 * bi + 4), x, FULL);
    w[0] = u.w;
    w[1] = u.x;
    w[2] = u.y;
    w[3] = u.z;
  }
  rotation_sync(bar_id, nthreads);
}

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__half>(__half v) { return __half2float(v); }

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __half from_f32<__half>(float v) { return __float2half_rn(v); }

// Code of dimension i from a packed row read as 32-bit words (layout in
// common.cuh).
template <int BITS>
__device__ __forceinline__ uint32_t code_at(const uint32_t *row, int i) {
  if constexpr (BITS == 3) {
    const int grp = i >> 5, m = i & 31;
    const uint32_t *gw = row + 3 * grp;
    if (m < 24) return (__ldg(gw + (m >> 3)) >> (4 * (m & 7))) & 7u;
    const int sh = 4 * (m - 24) + 3;
    return ((__ldg(gw) >> sh) & 1u) | (((__ldg(gw + 1) >> sh) & 1u) << 1) |
           (((__ldg(gw + 2) >> sh) & 1u) << 2);
  } else {
    const int bp = BITS * i;
    const uint32_t lo = __ldg(row + (bp >> 5));
    uint32_t c = lo >> (bp & 31);
    if ((bp & 31) + BITS > 32) c |= __ldg(row + (bp >> 5) + 1) << (32 - (bp & 31));
    return c & ((1u << BITS) - 1u);
  }
}

// ---------------------------------------------------------------------------
// Generic split kernel: each warp owns query heads g = warp, warp + 4, ...;
// per 32-token group, lane j scores token j (QK over all d), then the warp
// accumulates V dimension-parallel (lane owns dims lane + 32 k).
// ---------------------------------------------------------------------------
constexpr int kGenericThreads = 128;

template <typename T, int D, int BITS, bool FULL>
__global__ void __launch_bounds__(kGenericThreads) split_generic_kernel(const SplitArgs a) {
  constexpr int PB = D * BITS / 8, WORDS = PB / 4, KD = D / 32;
  __shared__ float cent[16];
  extern __shared__ float qrot[];  // [G][D]

  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.group;
  if (tid < (1 << BITS)) cent[tid] = a.centroid[tid];

  int tlen = a.seq_lens[b];
  tlen = tlen < 0 ? 0 : (tlen > a.tmax ? static_cast<int>(a.tmax) : tlen);
  const long long t0 = static_cast<long long>(split) * a.chunk;
  long long t1 = t0 + a.chunk;
  if (t1 > tlen) t1 = tlen;

  // Rotate the G queries of this KV head with R_K.
  for (int g = 0; g < G; ++g) {
    const T *q = static_cast<const T *>(a.q) + (static_cast<long long>(b) * a.hq + kvh * G + g) * D;
    for (int i = tid; i < D; i += kGenericThreads) qrot[g * D + i] = to_f32<T>(q[i]);
  }
  __syncthreads();
  rotate_forward_smem<D, FULL>(qrot, G, a.params_k + static_cast<size_t>(kvh) * 2 * D, tid,
                               kGenericThreads, 0);

  const long long pair = static_cast<long long>(b) * a.hkv + kvh;
  const uint8_t *kbase = a.packed_k + pair * a.tmax * PB;
  const uint8_t *vbase = a.packed_v + pair * a.tmax * PB;
  const uint16_t *nkbase = a.norms_k + pair * a.tmax;
  const uint16_t *nvbase = a.norms_v + pair * a.tmax;

  for (int g = warp; g < G; g += kGenericThreads / 32) {
    const float *qg = qrot + g * D;
    float m = -INFINITY, l = 0.f;
    float acc[KD];
#pragma unroll
    for (int k = 0; k < KD; ++k) acc[k] = 0.f;

    for (long long tg = t0; tg < t1; tg += 32) {
      const long long tok = tg + lane;
      const bool valid = tok < t1;
      float z = -INFINITY, sv = 0.f;
      if (valid) {
        const uint32_t *row = reinterpret_cast<const uint32_t *>(kbase + tok * PB);
        float dot = 0.f;
#pragma unroll 4
        for (int i = 0; i < D; ++i) dot = fmaf(cent[code_at<BITS>(row, i)], qg[i], dot);
        const float sk = __half2float(__ushort_as_half(nkbase[tok]));
        z = dot * sk * a.scale;
        sv = __half2float(__ushort_as_half(nvbase[tok]));
      }
      float zmax = z;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) zmax = fmaxf(zmax, __shfl_xor_sync(0xffffffffu, zmax, o));
      const float m_new = fmaxf(m, zmax);
      const float alpha = (m == -INFINITY) ? 0.f : expf(m - m_new);
      const float p = valid ? expf(z - m_new) : 0.f;
      l = l * alpha + p;
#pragma unroll
      for (int k = 0; k < KD; ++k) acc[k] *= alpha;
      m = m_new;
      const float w = p * sv;
      const int n = static_cast<int>(t1 - tg < 32 ? t1 - tg : 32);
      for (int j = 0; j < n; ++j) {
        const float wj = __shfl_sync(0xffffffffu, w, j);
        const uint32_t *row = reinterpret_cast<const uint32_t *>(vbase + (tg + j) * PB);
#pragma unroll
        for (int k = 0; k < KD; ++k) acc[k] = fmaf(wj, cent[code_at<BITS>(row, lane + 32 * k)], acc[k]);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);

    const long long slot = (static_cast<long long>(b) * a.hq + kvh * G + g) * a.n_splits + split;
    float *acc_out = a.ws_acc + slot * D;
#pragma unroll
    for (int k = 0; k < KD; ++k) acc_out[lane + 32 * k] = acc[k];
    if (lane == 0) a.ws_ml[slot] = make_float2(m, l);
  }
  (void)WORDS;
}

// ---------------------------------------------------------------------------
// Combine + inverse rotation.
// ---------------------------------------------------------------------------
constexpr int kCombineThreads = 256;
constexpr int kCombineWBlock = 1024;    // split weights held in shared memory per pass

// One CTA per (b, qh).  The split weights w_s = exp(m_s - m*) are computed
// once per split (not once per split and dimension) into shared memory; the
// threads then sum acc_s[i] w_s with kCombineThreads / D threads per
// dimension, each over every (kCombineThreads / D)-th split.  Warp 0 then
// normalises and rotates back in registers, lane j holding dims E j .. + E - 1
// (E = D / 32): x = H_d R_SO4^T u / sqrt(d), the block maps on its own
// 4-dim blocks first, then the Walsh-Hadamard stages h = 1, 2, ..., D/2
// ((a, b) -> (a + b, a - b)), those with h < E inside the lane and the others
// by shuffles.  Three block barriers in all.
template <typename T, int D, bool FULL>
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const CombineArgs a) {
  constexpr int P = D >= kCombineThreads ? 1 : kCombineThreads / D;   // threads per dimension
  constexpr int DPT = D > kCombineThreads ? D / kCombineThreads : 1;  // dimensions per thread
  constexpr int NW = kCombineThreads / 32, E = D / 32;
  __shared__ float part[P][D];
  __shared__ float wsh[kCombineWBlock];
  __shared__ float red_m[NW], red_l[NW];
  const int qh = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int kvh = qh / a.group;
  const long long base = (static_cast<long long>(b) * a.hq + qh) * a.n_splits;
  // The partial states come from the split kernel launched just before.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  float mx = -INFINITY;
  for (int s = tid; s < a.n_splits; s += kCombineThreads) mx = fmaxf(mx, a.ws_ml[base + s].x);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0) red_m[warp] = mx;
  __syncthreads();
  float mstar = red_m[0];
#pragma unroll
  for (int w = 1; w < NW; ++w) mstar = fmaxf(mstar, red_m[w]);

  const int p = tid / (D < kCombineThreads ? D : kCombineThreads);
  const int i0 = tid % (D < kCombineThreads ? D : kCombineThreads);
  float acc[DPT];
#pragma unroll
  for (int k = 0; k < DPT; ++k) acc[k] = 0.f;
  float lsum = 0.f;
  for (int s0 = 0; s0 < a.n_splits; s0 += kCombineWBlock) {
    const int ns = a.n_splits - s0 < kCombineWBlock ? a.n_splits - s0 : kCombineWBlock;
    if (s0 > 0) __syncthreads();   // the previous pass no longer reads wsh
    for (int s = tid; s < ns; s += kCombineThreads) {
      const float2 ml = a.ws_ml[base + s0 + s];
      const float w = ml.y > 0.f ? expf(ml.x - mstar) : 0.f;
      wsh[s] = w;
      lsum += ml.y * w;
    }
    __syncthreads();
    const float *accp = a.ws_acc + (base + s0) * D;
#pragma unroll 4
    for (int s = p; s < ns; s += P) {
      const float w = wsh[s];
#pragma unroll
      for (int k = 0; k < DPT; ++k) acc[k] = fmaf(accp[static_cast<long long>(s) * D + i0 + k * kCombineThreads], w, acc[k]);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
  if (lane == 0) red_l[warp] = lsum;
#pragma unroll
  for (int k = 0; k < DPT; ++k) part[p][i0 + k * kCombineThreads] = acc[k];
  __syncthreads();
  if (warp != 0) return;

  float l = 0.f;
#pragma unroll
  for (int w = 0; w < NW; ++w) l += red_l[w];
  const float inv_l = l > 0.f ? 1.f / l : 0.f;
  float x[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    float t = 0.f;
#pragma unroll
    for (int q = 0; q < P; ++q) t += part[q][E * lane + e];
    x[e] = t * inv_l;
  }
  const float *prm = a.params_v + static_cast<size_t>(kvh) * 2 * D;
#pragma unroll
  for (int u = 0; u < E / 4; ++u) {
    const int bi = (E / 4) * lane + u;
    const Quat r = block_inverse(load_quat(prm + 8 * bi), load_quat(prm + 8 * bi + 4),
                                 Quat{x[4 * u], x[4 * u + 1], x[4 * u + 2], x[4 * u + 3]}, FULL);
    x[4 * u] = r.w;
    x[4 * u + 1] = r.x;
    x[4 * u + 2] = r.y;
    x[4 * u + 3] = r.z;
  }
#pragma unroll
  for (int hs = 1; hs < E; hs <<= 1) {
#pragma unroll
    for (int e = 0; e < E; ++e) {
      if (!(e & hs)) {
        const float u = x[e], v = x[e + hs];
        x[e] = u + v;
        x[e + hs] = u - v;
      }
    }
  }
#pragma unroll
  for (int lm = 1; lm < 32; lm <<= 1) {
    const bool upper = (lane & lm) != 0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const float o = __shfl_xor_sync(0xffffffffu, x[e], lm);
      x[e] = upper ? o - x[e] : x[e] + o;
    }
  }
  const float inv_sqrt_d = rsqrtf(static_cast<float>(D));
  T *out = static_cast<T *>(a.out) + (static_cast<long long>(b) * a.hq + qh) * D + E * lane;
#pragma unroll
  for (int e = 0; e < E; ++e) out[e] = from_f32<T>(x[e] * inv_sqrt_d);
}

#include "decode_i8.cuh"
#include "decode_append.cuh"
#include "prefill.cuh"

// ---------------------------------------------------------------------------
// Host launchers
// ---------------------------------------------------------------------------

template <typename T, int D, int BITS, bool FULL>
int launch_split_generic(const SplitArgs &a, cudaStream_t stream) {
  auto kernel = split_generic_kernel<T, D, BITS, FULL>;
  const size_t smem = static_cast<size_t>(a.group) * D * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return set_error(ISOQ_ERR_CUDA, "decode split: %s", cudaGetErrorString(e));
  }
  dim3 grid(a.n_splits, a.hkv, a.batch);
  kernel<<<grid, kGenericThreads, smem, stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(ISOQ_ERR_CUDA, "decode split launch: %s", cudaGetErrorString(e));
  return ISOQ_OK;
}

template <typename T, int D, bool FULL>
int launch_combine(const CombineArgs &a, cudaStream_t stream) {
  dim3 grid(a.hq, a.batch);
  cudaError_t e = launch_pdl(combine_kernel<T, D, FULL>, grid, dim3(kCombineThreads), 0, stream, a);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(ISOQ_ERR_CUDA, "decode combine launch: %s", cudaGetErrorString(e));
  return ISOQ_OK;
}

int run_split_generic(int dtype, int d, int bits, int variant, const SplitArgs &a, cudaStream_t st) {
#define ISOQ_GV(T, D, B) \
  return variant == ISOQ_FULL ? launch_split_generic<T, D, B, true>(a, st) : launch_split_generic<T, D, B, false>(a, st)
#define ISOQ_GB(T, D)              \
  switch (bits) {                  \
    case 2: ISOQ_GV(T, D, 2);      \
    case 3: ISOQ_GV(T, D, 3);      \
    default: ISOQ_GV(T, D, 4);     \
  }
#define ISOQ_GD(T)                 \
  switch (d) {                     \
    case 128: ISOQ_GB(T, 128);     \
    case 256: ISOQ_GB(T, 256);     \
    default: ISOQ_GB(T, 512);      \
  }
  if (dtype == ISOQ_F16) {
    ISOQ_GD(__half);
  } else {
    ISOQ_GD(float);
  }
#undef ISOQ_GD
#undef ISOQ_GB
#undef ISOQ_GV
}

int run_combine(int dtype, int d, int variant, const CombineArgs &a, cudaStream_t st) {
#define ISOQ_CV(T, D) \
  return variant == ISOQ_FULL ? launch_combine<T, D, true>(a, st) : launch_combine<T, D, false>(a, st)
#define ISOQ_CD(T)              \
  switch (d) {                  \
    case 128: ISOQ_CV(T, 128);  \
    case 256: ISOQ_CV(T, 256);  \
    default: ISOQ_CV(T, 512);   \
  }
  if (dtype == ISOQ_F16) {
    ISOQ_CD(__half);
  } else {
    ISOQ_CD(float);
  }
#undef ISOQ_CD
#undef ISOQ_CV
}

bool aligned(const void *p, unsigned a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int validate_common(int dtype, int B, int Hq, int Hkv, int64_t Tmax, int d, int variant,
                    const void *ws, size_t ws_bytes) {
  if (!supported_d(d)) return set_error(ISOQ_ERR_UNSUPPORTED, "d=%d not supported", d);
  if (!supported_decode_variant(variant)) return set_error(ISOQ_ERR_UNSUPPORTED, "variant=%d", variant);
  if (!supported_dtype(dtype)) return set_error(ISOQ_ERR_UNSUPPORTED, "dtype=%d", dtype);
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Tmax <= 0)
    return set_error(ISOQ_ERR_INVALID_ARG, "B, Hq, Hkv and Tmax must be positive");
  if (Hq % Hkv) return set_error(ISOQ_ERR_INVALID_ARG, "Hq %% Hkv != 0");
  if (Hq / Hkv > kMaxGroup) return set_error(ISOQ_ERR_UNSUPPORTED, "Hq/Hkv > %d", kMaxGroup);
  if (Tmax >= (1ll << 31) || B > 65535 || Hkv > 65535 || Hq > (1 << 24))
    return set_error(ISOQ_ERR_INVALID_ARG, "shape too large");
  if (!ws) return set_error(ISOQ_ERR_INVALID_ARG, "workspace is NULL");
  if (!aligned(ws, 256)) return set_error(ISOQ_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (ws_bytes < isoq_decode_workspace_size(B, Hq, Hkv, Tmax, d))
    return set_error(ISOQ_ERR_INVALID_ARG, "workspace too small: %zu < %zu", ws_bytes,
                     isoq_decode_workspace_size(B, Hq, Hkv, Tmax, d));
  return ISOQ_OK;
}

void workspace_views(void *ws, int B, int Hq, int n_splits, int d, float **acc, float2 **ml,
                     uint32_t **qprep = nullptr) {
  *acc = static_cast<float *>(ws);
  *ml = reinterpret_cast<float2 *>(static_cast<float *>(ws) + static_cast<size_t>(B) * Hq * n_splits * d);
  if (qprep) {
    size_t n = static_cast<size_t>(B) * Hq * n_splits * (d + 2) * 4;
    n = (n + 255) / 256 * 256;
    *qprep = reinterpret_cast<uint32_t *>(static_cast<unsigned char *>(ws) + n);
  }
}

// Self-test of the failure path: thread 0 waits on an mbarrier that nothing
// arrives at, polling it (non-blocking test_wait) the way the pipelines'
// bounded waits poll theirs, until limit_ns of %globaltimer have passed (or,
// should the timer stall, 2^24 polls), then records kErrWaitTimeout in the
// decode error word and returns.  Nothing else is touched.
__global__ void wait_selftest_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    mbar_fence_init();
    const unsigned long long t0 = globaltimer();
    bool done = false;
    for (unsigned it = 0; it < (1u << 24); ++it) {
      uint32_t ok;
      asm volatile("{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                   "selp.u32 %0, 1, 0, p;\n\t}"
                   : "=r"(ok) : "r"(smem_u32(&bar)), "r"(0u) : "memory");
      if (ok) {
        done = true;
        break;
      }
      if ((it & 63u) == 63u && globaltimer() - t0 > limit_ns) break;
    }
    if (!done) atomicOr(&g_decode_error, kErrWaitTimeout);
  }
}

}  // namespace decode
}  // namespace isoq

using namespace isoq;

extern "C" {

int isoq_decode_split(const void *q_dev, int dtype, const uint8_t *packed_k_dev,
                      const uint8_t *packed_v_dev, const uint16_t *norms_k_dev,
                      const uint16_t *norms_v_dev, const int32_t *seq_lens_dev, int B, int Hq,
                      int Hkv, int64_t Tmax, int d, int bits, int variant,
                      const float *params_k_dev, float scale, void *workspace_dev,
                      size_t workspace_bytes, isoq_stream_t stream) {
  clear_error();
  int st = decode::validate_common(dtype, B, Hq, Hkv, Tmax, d, variant, workspace_dev, workspace_bytes);
  if (st) return st;
  if (!supported_bits(bits)) return set_error(ISOQ_ERR_UNSUPPORTED, "bits=%d not supported", bits);
  if (!q_dev || !packed_k_dev || !packed_v_dev || !norms_k_dev || !norms_v_dev || !seq_lens_dev || !params_k_dev)
    return set_error(ISOQ_ERR_INVALID_ARG, "null pointer");
  if (!decode::aligned(q_dev, 16) || !decode::aligned(packed_k_dev, 16) || !decode::aligned(packed_v_dev, 16) ||
      !decode::aligned(params_k_dev, 16) || !decode::aligned(norms_k_dev, 2) || !decode::aligned(norms_v_dev, 2) ||
      !decode::aligned(seq_lens_dev, 4))
    return set_error(ISOQ_ERR_UNSUPPORTED, "misaligned pointer");
  if (!std::isfinite(scale)) return set_error(ISOQ_ERR_INVALID_ARG, "scale is not finite");
  variant = block_map_variant(variant);

  decode::SplitArgs a;
  a.q = q_dev;
  a.packed_k = packed_k_dev;
  a.packed_v = packed_v_dev;
  a.norms_k = norms_k_dev;
  a.norms_v = norms_v_dev;
  a.seq_lens = seq_lens_dev;
  a.params_k = params_k_dev;
  a.batch = B;
  a.hq = Hq;
  a.hkv = Hkv;
  a.group = Hq / Hkv;
  a.tmax = Tmax;
  a.chunk = decode_chunk_tokens(B, Hkv, Tmax, d);
  a.n_splits = decode_num_splits(B, Hkv, Tmax, d);
  a.scale = scale;
  decode::workspace_views(workspace_dev, B, Hq, a.n_splits, d, &a.ws_acc, &a.ws_ml, &a.ws_qprep);
  CodebookF32 cb;
  codebook_f32(d, bits, &cb);
  for (int j = 0; j < 16; ++j) a.centroid[j] = j < cb.levels ? cb.centroid[j] : 0.f;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (decode::i8_path_supported(dtype, d, bits, a)) return decode::run_split_i8(d, variant, a, s);
  return decode::run_split_generic(dtype, d, bits, variant, a, s);
}

int isoq_decode_combine(int dtype, const int32_t *seq_lens_dev, int B, int Hq, int Hkv,
                        int64_t Tmax, int d, int variant, const float *params_v_dev,
                        void *out_dev, const void *workspace_dev, size_t workspace_bytes,
                        isoq_stream_t stream) {
  clear_error();
  int st = decode::validate_common(dtype, B, Hq, Hkv, Tmax, d, variant, workspace_dev, workspace_bytes);
  if (st) return st;
  if (!params_v_dev || !out_dev || !seq_lens_dev) return set_error(ISOQ_ERR_INVALID_ARG, "null pointer");
  if (!decode::aligned(params_v_dev, 16) || !decode::aligned(out_dev, 16))
    return set_error(ISOQ_ERR_UNSUPPORTED, "misaligned pointer");
  variant = block_map_variant(variant);
  decode::CombineArgs a;
  a.params_v = params_v_dev;
  a.out = out_dev;
  a.batch = B;
  a.hq = Hq;
  a.group = Hq / Hkv;
  a.n_splits = decode_num_splits(B, Hkv, Tmax, d);
  float *acc;
  float2 *ml;
  decode::workspace_views(const_cast<void *>(workspace_dev), B, Hq, a.n_splits, d, &acc, &ml);
  a.ws_acc = acc;
  a.ws_ml = ml;
  return decode::run_combine(dtype, d, variant, a, reinterpret_cast<cudaStream_t>(stream));
}

int isoq_decode_attention(const void *q_dev, int dtype, const uint8_t *packed_k_dev,
                          const uint8_t *packed_v_dev, const uint16_t *norms_k_dev,
                          const uint16_t *norms_v_dev, const int32_t *seq_lens_dev, int B,
                          int Hq, int Hkv, int64_t Tmax, int d, int bits, int variant,
                          const float *params_k_dev, const float *params_v_dev, float scale,
                          void *out_dev, void *workspace_dev, size_t workspace_bytes,
                          isoq_stream_t stream) {
  clear_error();
  if (!params_v_dev || !out_dev) return set_error(ISOQ_ERR_INVALID_ARG, "null pointer");
  if (!decode::aligned(params_v_dev, 16) || !decode::aligned(out_dev, 16))
    return set_error(ISOQ_ERR_UNSUPPORTED, "misaligned pointer");
  int st = isoq_decode_split(q_dev, dtype, packed_k_dev, packed_v_dev, norms_k_dev, norms_v_dev,
                             seq_lens_dev, B, Hq, Hkv, Tmax, d, bits, variant, params_k_dev,
                             scale, workspace_dev, workspace_bytes, stream);
  if (st) return st;
  return isoq_decode_combine(dtype, seq_lens_dev, B, Hq, Hkv, Tmax, d, variant, params_v_dev,
                             out_dev, workspace_dev, workspace_bytes, stream);
}

int isoq_selftest_wait_timeout(uint64_t limit_ns, isoq_stream_t stream) {
  clear_error();
  if (limit_ns == 0 || limit_ns > 1000000000ull)
    return set_error(ISOQ_ERR_INVALID_ARG, "limit_ns must be in (0, 1e9]");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  decode::wait_selftest_kernel<<<1, 32, 0, st>>>(static_cast<unsigned long long>(limit_ns));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(ISOQ_ERR_CUDA, "self-test launch: %s", cudaGetErrorString(e));
  return ISOQ_OK;
}

__attribute__((visibility("hidden"))) int isoq_detail_take_decode_error(cudaStream_t stream, unsigned *out) {
  unsigned zero = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(out, decode::g_decode_error, sizeof(unsigned), 0,
                                            cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e == cudaSuccess && *out)
    e = cudaMemcpyToSymbolAsync(decode::g_decode_error, &zero, sizeof(unsigned), 0,
                                cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  return e == cudaSuccess ? ISOQ_OK : set_error(ISOQ_ERR_CUDA, "error word: %s", cudaGetErrorString(e));
}

int isoq_decode_append(const void *k_new_dev, const void *v_new_dev, int dtype,
                       uint8_t *packed_k_dev, uint8_t *packed_v_dev, uint16_t *norms_k_dev,
                       uint16_t *norms_v_dev, int32_t *seq_lens_dev, int B, int Hkv, int64_t Tmax,
                       int d, int bits, int variant, const float *params_k_dev,
                       const float *params_v_dev, isoq_stream_t stream) {
  clear_error();
  if (!supported_d(d)) return set_error(ISOQ_ERR_UNSUPPORTED, "d=%d not supported", d);
  if (!supported_bits(bits)) return set_error(ISOQ_ERR_UNSUPPORTED, "bits=%d not supported", bits);
  if (!supported_decode_variant(variant)) return set_error(ISOQ_ERR_UNSUPPORTED, "variant=%d", variant);
  if (!supported_dtype(dtype)) return set_error(ISOQ_ERR_UNSUPPORTED, "dtype=%d", dtype);
  if (B <= 0 || Hkv <= 0 || Tmax <= 0)
    return set_error(ISOQ_ERR_INVALID_ARG, "B, Hkv and Tmax must be positive");
  if (Tmax >= (1ll << 31) || B > 65535 || Hkv > 65535)
    return set_error(ISOQ_ERR_INVALID_ARG, "shape too large");
  if (!k_new_dev || !v_new_dev || !packed_k_dev || !packed_v_dev || !norms_k_dev || !norms_v_dev ||
      !seq_lens_dev || !params_k_dev || !params_v_dev)
    return set_error(ISOQ_ERR_INVALID_ARG, "null pointer");
  if (!decode::aligned(packed_k_dev, 16) || !decode::aligned(packed_v_dev, 16) ||
      !decode::aligned(params_k_dev, 16) || !decode::aligned(params_v_dev, 16) ||
      !decode::aligned(k_new_dev, 16) || !decode::aligned(v_new_dev, 16) ||
      !decode::aligned(norms_k_dev, 2) || !decode::aligned(norms_v_dev, 2) || !decode::aligned(seq_lens_dev, 4))
    return set_error(ISOQ_ERR_UNSUPPORTED, "misaligned pointer");
  variant = block_map_variant(variant);
  decode::AppendArgs a;
  a.k_new = k_new_dev;
  a.v_new = v_new_dev;
  a.packed_k = packed_k_dev;
  a.packed_v = packed_v_dev;
  a.norms_k = norms_k_dev;
  a.norms_v = norms_v_dev;
  a.seq_lens = seq_lens_dev;
  a.params_k = params_k_dev;
  a.params_v = params_v_dev;
  a.tmax = Tmax;
  a.batch = B;
  a.hkv = Hkv;
  CodebookF32 cb;
  codebook_f32(d, bits, &cb);
  for (int k = 0; k < 15; ++k) a.thr[k] = k < cb.levels - 1 ? cb.threshold[k] : 0.f;
  return decode::run_append(dtype, d, bits, variant, a, seq_lens_dev, reinterpret_cast<cudaStream_t>(stream));
}

int isoq_decode_step(const void *q_dev, const void *k_new_dev, const void *v_new_dev, int dtype,
                     uint8_t *packed_k_dev, uint8_t *packed_v_dev, uint16_t *norms_k_dev,
                     uint16_t *norms_v_dev, int32_t *seq_lens_dev, int B, int Hq, int Hkv,
                     int64_t Tmax, int d, int bits, int variant, const float *params_k_dev,
                     const float *params_v_dev, float scale, void *out_dev, void *workspace_dev,
                     size_t workspace_bytes, isoq_stream_t stream) {
  // Every argument of the attention half is checked before the cache is
  // written, so a rejected call leaves the cache and the lengths as they were.
  clear_error();
  int st = decode::validate_common(dtype, B, Hq, Hkv, Tmax, d, variant, workspace_dev, workspace_bytes);
  if (st) return st;
  if (!q_dev || !out_dev) return set_error(ISOQ_ERR_INVALID_ARG, "null pointer");
  if (!decode::aligned(q_dev, 16) || !decode::aligned(out_dev, 16))
    return set_error(ISOQ_ERR_UNSUPPORTED, "misaligned pointer");
  if (!std::isfinite(scale)) return set_error(ISOQ_ERR_INVALID_ARG, "scale is not finite");
  st = isoq_decode_append(k_new_dev, v_new_dev, dtype, packed_k_dev, packed_v_dev, norms_k_dev,
                          norms_v_dev, seq_lens_dev, B, Hkv, Tmax, d, bits, variant, params_k_dev,
                          params_v_dev, stream);
  if (st) return st;
  return isoq_decode_attention(q_dev, dtype, packed_k_dev, packed_v_dev, norms_k_dev, norms_v_dev,
                               seq_lens_dev, B, Hq, Hkv, Tmax, d, bits, variant, params_k_dev,
                               params_v_dev, scale, out_dev, workspace_dev, workspace_bytes, stream);
}

int isoq_prefill_attention(const void *q_dev, int dtype, const uint8_t *packed_k_dev,
                           const uint8_t *packed_v_dev, const uint16_t *norms_k_dev,
                           const uint16_t *norms_v_dev, const int32_t *seq_lens_dev, int B, int Tq,
                           int Hq, int Hkv, int64_t Tmax, int d, int bits, int variant,
                           const float *params_k_dev, const float *params_v_dev, float scale,
                           void *out_dev, isoq_stream_t stream) {
  clear_error();
  if (d != 128 && d != 256) return set_error(ISOQ_ERR_UNSUPPORTED, "prefill: d=%d (128 or 256)", d);
  if (bits != 3) return set_error(ISOQ_ERR_UNSUPPORTED, "prefill: bits=%d (3)", bits);
  if (!supported_decode_variant(variant)) return set_error(ISOQ_ERR_UNSUPPORTED, "variant=%d", variant);
  if (dtype != ISOQ_F16) return set_error(ISOQ_ERR_UNSUPPORTED, "prefill: dtype=%d (float16 queries)", dtype);
  if (B <= 0 || Tq < 0 || Hq <= 0 || Hkv <= 0 || Tmax <= 0)
    return set_error(ISOQ_ERR_INVALID_ARG, "B, Hq, Hkv and Tmax must be positive, Tq >= 0");
  if (Hq % Hkv) return set_error(ISOQ_ERR_INVALID_ARG, "Hq %% Hkv != 0");
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8)
    return set_error(ISOQ_ERR_UNSUPPORTED, "prefill: Hq/Hkv=%d (1, 2, 4 or 8)", G);
  if (Tmax >= (1ll << 31) || B > 65535 || Hkv > 65535 || Tq > (1 << 24))
    return set_error(ISOQ_ERR_INVALID_ARG, "shape too large");
  if (Tmax % 8) return set_error(ISOQ_ERR_UNSUPPORTED, "prefill: Tmax %% 8 != 0");
  if (!q_dev || !packed_k_dev || !packed_v_dev || !norms_k_dev || !norms_v_dev || !seq_lens_dev ||
      !params_k_dev || !params_v_dev || !out_dev)
    return set_error(ISOQ_ERR_INVALID_ARG, "null pointer");
  if (!decode::aligned(packed_k_dev, 16) || !decode::aligned(packed_v_dev, 16) ||
      !decode::aligned(params_k_dev, 16) || !decode::aligned(params_v_dev, 16) ||
      !decode::aligned(q_dev, 4) || !decode::aligned(out_dev, 4) || !decode::aligned(norms_k_dev, 2) ||
      !decode::aligned(norms_v_dev, 2) || !decode::aligned(seq_lens_dev, 4))
    return set_error(ISOQ_ERR_UNSUPPORTED, "misaligned pointer");
  if (!std::isfinite(scale)) return set_error(ISOQ_ERR_INVALID_ARG, "scale is not finite");
  if (Tq == 0) return ISOQ_OK;
  decode::PrefillArgs a{};
  a.q = q_dev;
  a.packed_k = packed_k_dev;
  a.packed_v = packed_v_dev;
  a.norms_k = norms_k_dev;
  a.norms_v = norms_v_dev;
  a.seq_lens = seq_lens_dev;
  a.params_k = params_k_dev;
  a.params_v = params_v_dev;
  a.out = out_dev;
  a.tmax = Tmax;
  a.batch = B;
  a.tq = Tq;
  a.hq = Hq;
  a.hkv = Hkv;
  a.group = G;
  a.score_unit = static_cast<float>(scale * 1.4426950408889634);
  return decode::run_prefill(d, block_map_variant(variant), a, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode attention without caller-provided scratch.
//
// Some callers cannot allocate device memory: a host program whose device
// memory belongs to another framework's allocator, a plugin that is handed
// only its input and output buffers, or code on a path where cudaMalloc's
// implicit device-wide synchronisation is not acceptable.  For them the
// split-K partial states live in one file-scope device array of fixed size
// (every GPU that loads this library holds it until the process exits), and
// the entry point below allocates nothing.
// ---------------------------------------------------------------------------

namespace isoq {
namespace decode {

constexpr size_t kStaticWorkspaceBytes = size_t(16) << 20;  // 16 MiB per device

static __device__ __align__(256) unsigned char g_static_workspace[kStaticWorkspaceBytes];

// Identifier of the CUDA context current on this thread (0 if none or if the
// driver does not offer the query).  Context ids are unique for the life of
// the process, so a context created after a device reset gets a new one.
unsigned long long current_context_id() {
  using CtxGetCurrentFn = int (*)(void **);
  using CtxGetIdFn = int (*)(void *, unsigned long long *);
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  void *ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != 0 || !ctx || get_id(ctx, &id) != 0) return 0;
  return id;
}

// Device address of g_static_workspace on the current device.  Host code
// sees only a host-side stand-in for the array, so the device address is
// looked up with that device current and cached per device, together with
// the id of the context it belongs to: after a device reset the runtime
// makes a new context, in which the array has a new address, and the first
// call there looks it up again.
int static_workspace_address(void **out) {
  static std::mutex mu;
  static void *addr[256] = {nullptr};
  static unsigned long long ctx_of[256] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return set_error(ISOQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= 256) return set_error(ISOQ_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(mu);
  const unsigned long long ctx = current_context_id();
  if (!addr[dev] || ctx != ctx_of[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_workspace);
    if (e != cudaSuccess || !p)
      return set_error(ISOQ_ERR_CUDA, "cudaGetSymbolAddress(static workspace): %s", cudaGetErrorString(e));
    addr[dev] = p;
    // the lookup may have created the context: take its id now
    ctx_of[dev] = current_context_id();
  }
  *out = addr[dev];
  return ISOQ_OK;
}

}  // namespace decode
}  // namespace isoq

extern "C" size_t isoq_decode_static_workspace_bytes(void) { return isoq::decode::kStaticWorkspaceBytes; }

extern "C" int isoq_decode_attention_static(const void *q_dev, int dtype,
                                            const uint8_t *packed_k_dev,
                                            const uint8_t *packed_v_dev,
                                            const uint16_t *norms_k_dev,
                                            const uint16_t *norms_v_dev,
                                            const int32_t *seq_lens_dev, int B, int Hq, int Hkv,
                                            int64_t Tmax, int d, int bits, int variant,
                                            const float *params_k_dev,
                                            const float *params_v_dev, float scale,
                                            void *out_dev, isoq_stream_t stream) {
  clear_error();
  const size_t need = isoq_decode_workspace_size(B, Hq, Hkv, Tmax, d);
  if (need == 0)  // invalid shapes: let the regular validation report which
    return isoq_decode_attention(q_dev, dtype, packed_k_dev, packed_v_dev, norms_k_dev,
                                 norms_v_dev, seq_lens_dev, B, Hq, Hkv, Tmax, d, bits, variant,
                                 params_k_dev, params_v_dev, scale, out_dev, nullptr, 0, stream);
  if (need > decode::kStaticWorkspaceBytes)
    return set_error(ISOQ_ERR_UNSUPPORTED,
                     "these shapes need %zu bytes of decode workspace; the built-in workspace "
                     "holds %zu (use isoq_decode_attention with a caller-provided workspace)",
                     need, decode::kStaticWorkspaceBytes);
  void *ws = nullptr;
  const int st = decode::static_workspace_address(&ws);
  if (st) return st;
  // The split kernel writes every partial slot the combine reads, so the
  // array needs no clearing between calls.
  return isoq_decode_attention(q_dev, dtype, packed_k_dev, packed_v_dev, norms_k_dev, norms_v_dev,
                               seq_lens_dev, B, Hq, Hkv, Tmax, d, bits, variant, params_k_dev,
                               params_v_dev, scale, out_dev, ws, decode::kStaticWorkspaceBytes,
                               stream);
}
