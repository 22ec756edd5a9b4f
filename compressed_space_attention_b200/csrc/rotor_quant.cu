// RotorQuant comparator on sm_100a: blockwise 3-D Clifford-rotor compression
// and its inverse, the method the IsoQuant page measures its kernels against.
//
// Per vector (the RotorQuant page; IsoQuant arXiv 2603.28430, abstract):
//   s = ||x||; the vector is padded to 3G dimensions, G = ceil(d / 3); each
//   group v of three is rotated by its own unit rotor R = s_R + p12 e12 +
//   p13 e13 + p23 e23 of Cl(3,0) with the sandwich v' = R v rev(R); the 3G
//   rotated coordinates get IsoQuant's Lloyd-Max codes for N(0, 1/d)
//   (compared with s t_k, no division per element) and are packed as one
//   LSB-first bitstream of ceil(3 G b / 32) words; the norm is stored as
//   float16.  Dequantisation applies rev(R) v R to the centroids, drops the
//   padding and scales by the stored norm.
//
// The sandwich is evaluated in its sparse form: R v has only the grade-1
// part t and the grade-3 part t7 for a vector v (12 multiply-adds), and the
// vector part of (t + t7 e123) rev(R) needs four terms per coordinate (12
// more), 24 per group against the 56 of the page's cost figure.
//
// Mapping: one warp per V vectors (V = 2 at d = 128, else 1) so that the
// G V group tasks fill the lanes; rows are staged through shared memory with
// 16-byte loads and stores, the codes through a per-warp byte array from
// which each lane assembles whole 32-bit words.

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "internal.h"

namespace isoq {
namespace rotor {

constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;

__host__ __device__ constexpr int n_groups(int d) { return (d + 2) / 3; }
__host__ __device__ constexpr int n_words(int d, int bits) { return (3 * n_groups(d) * bits + 31) / 32; }

template <int D>
struct Cfg {
  static constexpr int G = n_groups(D);
  static constexpr int V = D == 128 ? 2 : 1;     // vectors per warp pass
  static constexpr int TASKS = G * V;
  static constexpr int ROW = 3 * G;               // padded row (floats)
};

struct Args {
  const void *x;          // quantize: input rows; dequantize: output rows
  void *y;
  const uint8_t *codes_in;
  uint8_t *codes_out;
  const uint16_t *norms_in;
  uint16_t *norms_out;
  const float *rotors;    // [n_heads][G][4]
  long long head_stride, vec_stride;    // elements, of the float rows
  long long code_head_stride;           // vectors, of the codes and norms
  long long n_vec;
  int n_heads;
  float tab[16];          // quantize: thresholds t_k; dequantize: centroids
};

// v' = R v rev(R) (sign = +1) or rev(R) v R (sign = -1: the bivector negated).
__device__ __forceinline__ void sandwich(float4 r, float sign, float &x, float &y, float &z) {
  const float s = r.x, a = sign * r.y, b = sign * r.z, c = sign * r.w;
  const float t1 = fmaf(s, x, fmaf(a, y, b * z));
  const float t2 = fmaf(s, y, fmaf(-a, x, c * z));
  const float t3 = fmaf(s, z, fmaf(-b, x, -c * y));
  const float t7 = fmaf(a, z, fmaf(-b, y, c * x));
  x = fmaf(s, t1, fmaf(a, t2, fmaf(b, t3, c * t7)));
  y = fmaf(s, t2, fmaf(-a, t1, fmaf(c, t3, -b * t7)));
  z = fmaf(s, t3, fmaf(-b, t1, fmaf(-c, t2, a * t7)));
}

// Loads V rows of D elements of T into row[v][0..D) (float), zero padding
// to 3G, with 16-byte loads.
template <typename T, int D>
__device__ __forceinline__ void load_rows(const T *const *src, const bool *valid, float *row, int lane) {
  using C = Cfg<D>;
  constexpr int PER = 16 / sizeof(T);           // elements per 16 bytes
  constexpr int CHUNKS = D / PER;
#pragma unroll
  for (int v = 0; v < C::V; ++v) {
    for (int c = lane; c < CHUNKS; c += 32) {
      float f[PER];
      if (valid[v]) {
        const uint4 u = *reinterpret_cast<const uint4 *>(src[v] + c * PER);
        if constexpr (sizeof(T) == 2) {
          const __half2 *h = reinterpret_cast<const __half2 *>(&u);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 p = __half22float2(h[k]);
            f[2 * k] = p.x;
            f[2 * k + 1] = p.y;
          }
        } else {
          f[0] = __uint_as_float(u.x);
          f[1] = __uint_as_float(u.y);
          f[2] = __uint_as_float(u.z);
          f[3] = __uint_as_float(u.w);
        }
      } else {
#pragma unroll
        for (int k = 0; k < PER; ++k) f[k] = 0.f;
      }
#pragma unroll
      for (int k = 0; k < PER; ++k) row[v * C::ROW + c * PER + k] = f[k];
    }
    for (int i = D + lane; i < C::ROW; i += 32) row[v * C::ROW + i] = 0.f;
  }
}

template <typename T, int D, int BITS>
__global__ void __launch_bounds__(kThreads) rotor_quantize_kernel(const Args a) {
  using C = Cfg<D>;
  constexpr int L = 1 << BITS;
  constexpr int W = n_words(D, BITS);
  __shared__ float rows[kWarps][C::V * C::ROW];
  __shared__ unsigned char codes[kWarps][C::V * C::ROW + 4];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float *row = rows[warp];
  unsigned char *cb = codes[warp];
  const long long per_head = (a.n_vec + C::V - 1) / C::V;
  const long long total = per_head * a.n_heads;
  const long long stride = static_cast<long long>(gridDim.x) * kWarps;

  for (long long item = static_cast<long long>(blockIdx.x) * kWarps + warp; item < total; item += stride) {
    const int head = static_cast<int>(item / per_head);
    const long long v0 = (item % per_head) * C::V;
    const T *src[2];
    bool valid[2];
#pragma unroll
    for (int v = 0; v < 2; ++v) {
      valid[v] = v < C::V && v0 + v < a.n_vec;
      src[v] = static_cast<const T *>(a.x) + head * a.head_stride + (valid[v] ? (v0 + v) : 0) * a.vec_stride;
    }
    load_rows<T, D>(src, valid, row, lane);
    __syncwarp();
    // Norms of the V rows.
    float nrm[2] = {0.f, 0.f};
#pragma unroll
    for (int v = 0; v < C::V; ++v) {
      float ss = 0.f;
      for (int i = lane; i < D; i += 32) ss = fmaf(row[v * C::ROW + i], row[v * C::ROW + i], ss);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      nrm[v] = sqrtf(ss);
    }
    // Rotate and quantise: task -> (vector, group).
    const float4 *rot = reinterpret_cast<const float4 *>(a.rotors) + static_cast<long long>(head) * C::G;
    for (int task = lane; task < C::TASKS; task += 32) {
      const int v = task / C::G, g = task - v * C::G;
      float *e = row + v * C::ROW + 3 * g;
      float x = e[0], y = e[1], z = e[2];
      sandwich(__ldg(rot + g), 1.f, x, y, z);
      const float s = C::V == 1 ? nrm[0] : (v ? nrm[1] : nrm[0]);
      int c0 = 0, c1 = 0, c2 = 0;
#pragma unroll
      for (int k = 0; k < L - 1; ++k) {
        const float t = a.tab[k] * s;
        c0 += x > t;
        c1 += y > t;
        c2 += z > t;
      }
      unsigned char *cc = cb + v * C::ROW + 3 * g;
      cc[0] = static_cast<unsigned char>(c0);
      cc[1] = static_cast<unsigned char>(c1);
      cc[2] = static_cast<unsigned char>(c2);
    }
    __syncwarp();
    // Pack: word w of vector v holds bits [32 w, 32 w + 32) of its stream.
    for (int wt = lane; wt < C::V * W; wt += 32) {
      const int v = wt / W, w = wt - v * W;
      if (!valid[v]) continue;
      const unsigned char *cc = cb + v * C::ROW;
      // codes first..last overlap the word; acc's bit 0 is stream bit BITS * first
      const int first = (32 * w) / BITS, last = (32 * w + 31) / BITS;
      unsigned long long acc = 0;
      for (int i = first; i <= last && i < C::ROW; ++i)
        acc |= static_cast<unsigned long long>(cc[i]) << (BITS * (i - first));
      const uint32_t word = static_cast<uint32_t>(acc >> (32 * w - BITS * first));
      const long long idx = static_cast<long long>(head) * a.code_head_stride + v0 + v;
      reinterpret_cast<uint32_t *>(a.codes_out + idx * (4 * W))[w] = word;
    }
    if (lane < C::V && valid[lane]) {
      const long long idx = static_cast<long long>(head) * a.code_head_stride + v0 + lane;
      a.norms_out[idx] = __half_as_ushort(__float2half_rn(lane ? nrm[1] : nrm[0]));
    }
    __syncwarp();
  }
}

template <typename T, int D, int BITS>
__global__ void __launch_bounds__(kThreads) rotor_dequantize_kernel(const Args a) {
  using C = Cfg<D>;
  constexpr int W = n_words(D, BITS);
  constexpr uint32_t MASK = (1u << BITS) - 1u;
  __shared__ float rows[kWarps][C::V * C::ROW];
  __shared__ uint32_t words[kWarps][C::V * W + 1];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float *row = rows[warp];
  uint32_t *wd = words[warp];
  const long long per_head = (a.n_vec + C::V - 1) / C::V;
  const long long total = per_head * a.n_heads;
  const long long stride = static_cast<long long>(gridDim.x) * kWarps;

  for (long long item = static_cast<long long>(blockIdx.x) * kWarps + warp; item < total; item += stride) {
    const int head = static_cast<int>(item / per_head);
    const long long v0 = (item % per_head) * C::V;
    bool valid[2];
    float s16[2];
#pragma unroll
    for (int v = 0; v < 2; ++v) {
      valid[v] = v < C::V && v0 + v < a.n_vec;
      const long long idx = static_cast<long long>(head) * a.code_head_stride + (valid[v] ? v0 + v : 0);
      s16[v] = valid[v] ? __half2float(__ushort_as_half(a.norms_in[idx])) : 0.f;
    }
    for (int wt = lane; wt < C::V * W; wt += 32) {
      const int v = wt / W, w = wt - v * W;
      const long long idx = static_cast<long long>(head) * a.code_head_stride + (valid[v] ? v0 + v : 0);
      wd[wt] = valid[v] ? reinterpret_cast<const uint32_t *>(a.codes_in + idx * (4 * W))[w] : 0u;
    }
    if (lane == 0) wd[C::V * W] = 0u;
    __syncwarp();
    const float4 *rot = reinterpret_cast<const float4 *>(a.rotors) + static_cast<long long>(head) * C::G;
    for (int task = lane; task < C::TASKS; task += 32) {
      const int v = task / C::G, g = task - v * C::G;
      float e[3];
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        const int bit = BITS * (3 * g + k);
        const uint32_t *p = wd + v * W + (bit >> 5);
        const unsigned long long pair = static_cast<unsigned long long>(p[0]) |
                                        (static_cast<unsigned long long>(p[1]) << 32);
        e[k] = a.tab[static_cast<uint32_t>(pair >> (bit & 31)) & MASK];
      }
      sandwich(__ldg(rot + g), -1.f, e[0], e[1], e[2]);
      const float s = v ? s16[1] : s16[0];
      float *dst = row + v * C::ROW + 3 * g;
      dst[0] = e[0] * s;
      dst[1] = e[1] * s;
      dst[2] = e[2] * s;
    }
    __syncwarp();
    constexpr int PER = 16 / sizeof(T);
    constexpr int CHUNKS = D / PER;
#pragma unroll
    for (int v = 0; v < C::V; ++v) {
      if (!valid[v]) continue;
      T *out = static_cast<T *>(a.y) + head * a.head_stride + (v0 + v) * a.vec_stride;
      for (int c = lane; c < CHUNKS; c += 32) {
        const float *f = row + v * C::ROW + c * PER;
        uint4 u;
        if constexpr (sizeof(T) == 2) {
          __half2 *h = reinterpret_cast<__half2 *>(&u);
#pragma unroll
          for (int k = 0; k < 4; ++k) h[k] = __floats2half2_rn(f[2 * k], f[2 * k + 1]);
        } else {
          u = make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                         __float_as_uint(f[3]));
        }
        reinterpret_cast<uint4 *>(out)[c] = u;
      }
    }
    __syncwarp();
  }
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
  return n;
}

template <typename T, int D, int BITS>
int launch(bool forward, const Args &a, cudaStream_t st) {
  using C = Cfg<D>;
  const long long items = (a.n_vec + C::V - 1) / C::V * a.n_heads;
  long long grid = static_cast<long long>(num_sms()) * 4;
  const long long need = (items + kWarps - 1) / kWarps;
  if (grid > need) grid = need;
  if (forward)
    rotor_quantize_kernel<T, D, BITS><<<static_cast<unsigned>(grid), kThreads, 0, st>>>(a);
  else
    rotor_dequantize_kernel<T, D, BITS><<<static_cast<unsigned>(grid), kThreads, 0, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(ISOQ_ERR_CUDA, "rotor launch: %s", cudaGetErrorString(e));
  return ISOQ_OK;
}

template <typename T, int D>
int launch_b(int bits, bool fwd, const Args &a, cudaStream_t st) {
  if (bits == 2) return launch<T, D, 2>(fwd, a, st);
  if (bits == 3) return launch<T, D, 3>(fwd, a, st);
  return launch<T, D, 4>(fwd, a, st);
}

template <typename T>
int launch_d(int d, int bits, bool fwd, const Args &a, cudaStream_t st) {
  if (d == 128) return launch_b<T, 128>(bits, fwd, a, st);
  if (d == 256) return launch_b<T, 256>(bits, fwd, a, st);
  return launch_b<T, 512>(bits, fwd, a, st);
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace rotor
}  // namespace isoq

using namespace isoq;

extern "C" {

int isoq_rotor_groups(int d) { return supported_d(d) ? rotor::n_groups(d) : ISOQ_ERR_UNSUPPORTED; }

size_t isoq_rotor_packed_bytes(int d, int bits) {
  if (!supported_d(d) || !supported_bits(bits)) return 0;
  return 4u * static_cast<size_t>(rotor::n_words(d, bits));
}

int isoq_rotor_quantize(const void *x_dev, int dtype, int n_heads, int64_t n_vec, int d, int bits,
                        int64_t head_stride, int64_t vec_stride, const float *rotors_dev,
                        uint8_t *codes_dev, uint16_t *norms_dev, int64_t out_head_stride,
                        isoq_stream_t stream) {
  clear_error();
  if (!supported_d(d)) return set_error(ISOQ_ERR_UNSUPPORTED, "d=%d not supported", d);
  if (!supported_bits(bits)) return set_error(ISOQ_ERR_UNSUPPORTED, "bits=%d not supported", bits);
  if (!supported_dtype(dtype)) return set_error(ISOQ_ERR_UNSUPPORTED, "dtype=%d", dtype);
  if (n_heads < 0 || n_vec < 0) return set_error(ISOQ_ERR_INVALID_ARG, "negative size");
  if (n_heads == 0 || n_vec == 0) return ISOQ_OK;
  if (n_vec >= (1ll << 31) || n_heads >= (1 << 24))
    return set_error(ISOQ_ERR_INVALID_ARG, "n_vec or n_heads too large");
  if (!x_dev || !rotors_dev || !codes_dev || !norms_dev) return set_error(ISOQ_ERR_INVALID_ARG, "null pointer");
  if (vec_stride < d || (n_heads > 1 && head_stride < 1) || out_head_stride < n_vec)
    return set_error(ISOQ_ERR_INVALID_ARG, "bad stride");
  const int es = elt_size(dtype);
  if (!rotor::aligned16(x_dev) || (vec_stride * es) % 16 || (n_heads > 1 && (head_stride * es) % 16))
    return set_error(ISOQ_ERR_UNSUPPORTED, "x and its strides must be 16-byte aligned");
  if (!rotor::aligned16(rotors_dev) || (reinterpret_cast<uintptr_t>(codes_dev) & 3) ||
      (reinterpret_cast<uintptr_t>(norms_dev) & 1))
    return set_error(ISOQ_ERR_UNSUPPORTED, "rotors must be 16-byte, codes 4-byte, norms 2-byte aligned");
  rotor::Args a{};
  a.x = x_dev;
  a.codes_out = codes_dev;
  a.norms_out = norms_dev;
  a.rotors = rotors_dev;
  a.head_stride = n_heads > 1 ? head_stride : 0;
  a.vec_stride = vec_stride;
  a.code_head_stride = out_head_stride;
  a.n_vec = n_vec;
  a.n_heads = n_heads;
  CodebookF32 cb;
  codebook_f32(d, bits, &cb);
  for (int k = 0; k < 15; ++k) a.tab[k] = k < cb.levels - 1 ? cb.threshold[k] : 0.f;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return dtype == ISOQ_F16 ? rotor::launch_d<__half>(d, bits, true, a, st)
                           : rotor::launch_d<float>(d, bits, true, a, st);
}

int isoq_rotor_dequantize(const uint8_t *codes_dev, const uint16_t *norms_dev, int n_heads,
                          int64_t n_vec, int d, int bits, int64_t in_head_stride,
                          const float *rotors_dev, void *out_dev, int out_dtype,
                          int64_t head_stride, int64_t vec_stride, isoq_stream_t stream) {
  clear_error();
  if (!supported_d(d)) return set_error(ISOQ_ERR_UNSUPPORTED, "d=%d not supported", d);
  if (!supported_bits(bits)) return set_error(ISOQ_ERR_UNSUPPORTED, "bits=%d not supported", bits);
  if (!supported_dtype(out_dtype)) return set_error(ISOQ_ERR_UNSUPPORTED, "dtype=%d", out_dtype);
  if (n_heads < 0 || n_vec < 0) return set_error(ISOQ_ERR_INVALID_ARG, "negative size");
  if (n_heads == 0 || n_vec == 0) return ISOQ_OK;
  if (n_vec >= (1ll << 31) || n_heads >= (1 << 24))
    return set_error(ISOQ_ERR_INVALID_ARG, "n_vec or n_heads too large");
  if (!codes_dev || !norms_dev || !rotors_dev || !out_dev) return set_error(ISOQ_ERR_INVALID_ARG, "null pointer");
  if (in_head_stride < n_vec || vec_stride < d || (n_heads > 1 && head_stride < 1))
    return set_error(ISOQ_ERR_INVALID_ARG, "bad stride");
  const int es = elt_size(out_dtype);
  if (!rotor::aligned16(out_dev) || (vec_stride * es) % 16 || (n_heads > 1 && (head_stride * es) % 16))
    return set_error(ISOQ_ERR_UNSUPPORTED, "out and its strides must be 16-byte aligned");
  if (!rotor::aligned16(rotors_dev) || (reinterpret_cast<uintptr_t>(codes_dev) & 3) ||
      (reinterpret_cast<uintptr_t>(norms_dev) & 1))
    return set_error(ISOQ_ERR_UNSUPPORTED, "rotors must be 16-byte, codes 4-byte, norms 2-byte aligned");
  rotor::Args a{};
  a.y = out_dev;
  a.codes_in = codes_dev;
  a.norms_in = norms_dev;
  a.rotors = rotors_dev;
  a.head_stride = n_heads > 1 ? head_stride : 0;
  a.vec_stride = vec_stride;
  a.code_head_stride = in_head_stride;
  a.n_vec = n_vec;
  a.n_heads = n_heads;
  CodebookF32 cb;
  codebook_f32(d, bits, &cb);
  for (int k = 0; k < 16; ++k) a.tab[k] = k < cb.levels ? cb.centroid[k] : 0.f;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return out_dtype == ISOQ_F16 ? rotor::launch_d<__half>(d, bits, false, a, st)
                               : rotor::launch_d<float>(d, bits, false, a, st);
}

}  // extern "C"
