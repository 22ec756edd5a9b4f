// IsoQuant compressor and its inverse on sm_100a.
//
// isoq_quantize follows RotaryQuant (arXiv 2608.08081) §3.2 Algorithm 1 and
// eq. (2) with the block maps of IsoQuant (arXiv 2603.28430, abstract):
//   s = ||x||, y = R_SO4(H_d x / (s sqrt d)), code_i = #{k : y_i > t_k},
//   BitPack_b, stored norm float16(s).
// isoq_dequantize is the inverse path (RotaryQuant §3.4 kernel D):
//   x = s16 * H_d(R_SO4^T c[codes]) / sqrt d.
//
// Mapping.  A vector of d elements is held by P = d/64 lanes of one warp,
// 64 consecutive elements per lane, in registers.  The Walsh-Hadamard stages
// with h >= 4 run as butterflies (in-lane for h < 64, by warp shuffle for
// h >= 64).  The stages h = 1, 2 act inside each 4-block and commute with the
// others, so they are folded into one 4x4 matrix per block together with the
// SO(4) map and the 1/sqrt(d) normalisation:
//   quantize:   M_i = R_i H_4 / sqrt(d)   applied after the h >= 4 stages,
//   dequantize: N_i = H_4 R_i^T / sqrt(d) applied before them.
// The quantiser compares the unnormalised R x with s * t_k (no division per
// element) using the symmetry of the codebook: the sign picks the half, and
// the magnitude is counted against the positive thresholds.
//
// Data movement.  quantize stages its input through 128B-swizzled TMA tiles
// (one producer warp, four consumer warps, an mbarrier ring); each lane then
// reads its own 128-byte row segments conflict-free.  Outputs are written with
// 8/16-byte stores that cover whole sectors per warp.

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace isoq {
namespace quant {

using namespace isoq::dev;

constexpr int kE = 64;              // elements per lane
constexpr int kConsumerWarps = 4;
constexpr int kConsumers = 32 * kConsumerWarps;
constexpr int kQuantThreads = kConsumers + 32;  // + one TMA producer warp

__device__ unsigned int g_quant_error = 0;

template <typename T, int D, int BITS>
struct Cfg {
  static constexpr int P = D / kE;              // lanes per vector
  static constexpr int VPW = 32 / P;            // vectors per warp
  static constexpr int NV = kConsumers / P;     // vectors per tile
  static constexpr int ES = sizeof(T);
  static constexpr int BOX_ELEMS = 128 / ES;    // elements in one 128-byte box row
  static constexpr int NBOX = D * ES / 128;     // boxes per tile
  static constexpr int BOX_BYTES = NV * 128;
  static constexpr int STAGE_BYTES = NBOX * BOX_BYTES;
  static constexpr int STAGES = ES == 2 ? 4 : 3;
  static constexpr int L = 1 << BITS;
  static constexpr int NPOS = L / 2 - 1;        // positive thresholds
  static constexpr int PB = D * BITS / 8;       // packed bytes per vector
  static constexpr int TB = kE * BITS / 8;      // packed bytes per lane
  static constexpr int MAT_BYTES = (D / 4) * 16 * 4;
  static constexpr int SMEM = STAGES * STAGE_BYTES + MAT_BYTES + 2 * STAGES * 8 + 16 + 1024;
};

struct QuantArgs {
  const float *params;      // [n_heads][D/4][8]
  uint8_t *codes;
  uint16_t *norms;
  long long out_head_stride;
  long long n_vec;
  int n_heads;
  int tiles_per_head;
  long long total_tiles;
  float tau[7];             // positive thresholds t_{L/2}, ..., t_{L-2}
};

// Builds the per-block 4x4 matrices of one head into shared memory, row-major.
// forward: M_i = R_i H_4 / sqrt(d); inverse: N_i = H_4 R_i^T / sqrt(d).
template <int D, bool FULL, bool FORWARD>
__device__ void build_block_matrices(const float *params_head, float *mat, int tid, int nthreads) {
  const float inv_sqrt_d = rsqrtf(static_cast<float>(D));
  for (int b = tid; b < D / 4; b += nthreads) {
    const Quat ql = load_quat(params_head + 8 * b);
    const Quat qr = load_quat(params_head + 8 * b + 4);
    float m[4][4];
    for (int c = 0; c < 4; ++c) {
      if (FORWARD) {
        // column c = R_i (H_4 e_c)
        const Quat u = block_forward(ql, qr, h4_column(c), FULL);
        m[0][c] = u.w; m[1][c] = u.x; m[2][c] = u.y; m[3][c] = u.z;
      } else {
        // column c = H_4 (R_i^T e_c)
        Quat e{c == 0 ? 1.f : 0.f, c == 1 ? 1.f : 0.f, c == 2 ? 1.f : 0.f, c == 3 ? 1.f : 0.f};
        const Quat u = block_inverse(ql, qr, e, FULL);
        m[0][c] = u.w + u.x + u.y + u.z;
        m[1][c] = u.w - u.x + u.y - u.z;
        m[2][c] = u.w + u.x - u.y - u.z;
        m[3][c] = u.w - u.x - u.y + u.z;
      }
    }
    // Pair order for the packed block product (see apply_block_matrices):
    // (y0, y1) uses (M00,M11) (M01,M10) (M02,M13) (M03,M12) and
    // (y2, y3) uses (M22,M33) (M23,M32) (M20,M31) (M21,M30).
    const int order[16][2] = {{0, 0}, {1, 1}, {0, 1}, {1, 0}, {0, 2}, {1, 3}, {0, 3}, {1, 2},
                              {2, 2}, {3, 3}, {2, 3}, {3, 2}, {2, 0}, {3, 1}, {2, 1}, {3, 0}};
    float *out = mat + 16 * b;
    for (int k = 0; k < 16; ++k) out[k] = m[order[k][0]][order[k][1]] * inv_sqrt_d;
  }
}

// The 64 elements of a lane are held as 32 packed float pairs
// xp[k] = (x[2k], x[2k+1]).

// In-lane Walsh-Hadamard butterflies for the strides 4 <= h < 64 (pair
// strides 2..16): both elements of a pair move together.
__device__ __forceinline__ void wht_inlane_h4_to_32(uint64_t (&xp)[kE / 2]) {
#pragma unroll
  for (int hp = 2; hp < kE / 2; hp <<= 1) {
#pragma unroll
    for (int k = 0; k < kE / 2; ++k) {
      if (!(k & hp)) {
        const uint64_t a = xp[k], b = xp[k + hp];
        xp[k] = f2_add(a, b);
        xp[k + hp] = f2_sub(a, b);
      }
    }
  }
}

// Cross-lane butterflies for h = 64, 128, ..., D/2: the partner part of a
// vector sits VPW lanes away per doubling.
template <int P, int VPW>
__device__ __forceinline__ void wht_crosslane(uint64_t (&xp)[kE / 2], int part) {
#pragma unroll
  for (int k = 1; k < P; k <<= 1) {
    const float sgn = (part & k) ? -1.f : 1.f;
    const uint64_t sgn2 = f2_pack(sgn, sgn);
#pragma unroll
    for (int i = 0; i < kE / 2; ++i) {
      const uint64_t o = __shfl_xor_sync(0xffffffffu, xp[i], k * VPW);
      xp[i] = f2_fma(sgn2, xp[i], o);
    }
  }
}

// Applies the 16 per-block 4x4 matrices of this lane's blocks, in place.
// With z = (z0..z3), Z01 = (z0, z1), Z10 = (z1, z0) and so on:
//   (y0, y1) = (M00,M11) Z01 + (M01,M10) Z10 + (M02,M13) Z23 + (M03,M12) Z32
//   (y2, y3) = (M22,M33) Z23 + (M23,M32) Z32 + (M20,M31) Z01 + (M21,M30) Z10
__device__ __forceinline__ void apply_block_matrices(uint64_t (&xp)[kE / 2], const float *mat_lane) {
#pragma unroll
  for (int lb = 0; lb < kE / 4; ++lb) {
    const float4 *m = reinterpret_cast<const float4 *>(mat_lane + 16 * lb);
    const float4 m0 = m[0], m1 = m[1], m2 = m[2], m3 = m[3];
    const uint64_t z01 = xp[2 * lb], z23 = xp[2 * lb + 1];
    const uint64_t z10 = f2_swap(z01), z32 = f2_swap(z23);
    uint64_t y01 = f2_mul(f2_pack(m0.x, m0.y), z01);
    y01 = f2_fma(f2_pack(m0.z, m0.w), z10, y01);
    y01 = f2_fma(f2_pack(m1.x, m1.y), z23, y01);
    y01 = f2_fma(f2_pack(m1.z, m1.w), z32, y01);
    uint64_t y23 = f2_mul(f2_pack(m2.x, m2.y), z23);
    y23 = f2_fma(f2_pack(m2.z, m2.w), z32, y23);
    y23 = f2_fma(f2_pack(m3.x, m3.y), z01, y23);
    y23 = f2_fma(f2_pack(m3.z, m3.w), z10, y23);
    xp[2 * lb] = y01;
    xp[2 * lb + 1] = y23;
  }
}

template <typename T, int D, int BITS, bool FULL>
__global__ void __launch_bounds__(kQuantThreads)
    quantize_kernel(const __grid_constant__ CUtensorMap xmap, const QuantArgs args) {
  using C = Cfg<T, D, BITS>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char *stages = smem;
  float *mat = reinterpret_cast<float *>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t *full_bar = reinterpret_cast<uint64_t *>(smem + C::STAGES * C::STAGE_BYTES + C::MAT_BYTES);
  uint64_t *empty_bar = full_bar + C::STAGES;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(empty_bar + C::STAGES);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;

  // Contiguous range of tiles for this CTA (few head changes per CTA).
  const long long per_cta = (args.total_tiles + gridDim.x - 1) / gridDim.x;
  const long long tile_begin = static_cast<long long>(blockIdx.x) * per_cta;
  long long tile_end = tile_begin + per_cta;
  if (tile_end > args.total_tiles) tile_end = args.total_tiles;

  if (tid == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], kConsumerWarps);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int issued_any = 0;
      for (long long t = tile_begin; t < tile_end; ++t) {
        const long long it = t - tile_begin;
        const int s = static_cast<int>(it % C::STAGES);
        const uint32_t round = static_cast<uint32_t>(it / C::STAGES);
        if (!mbar_wait_bounded(&empty_bar[s], (round & 1u) ^ 1u) || *abort_flag) {
          atomicOr(&g_quant_error, kErrWaitTimeout);
          *abort_flag = 1;
          break;
        }
        const int head = static_cast<int>(t / args.tiles_per_head);
        const int v0 = static_cast<int>((t % args.tiles_per_head) * C::NV);
        mbar_arrive_expect_tx(&full_bar[s], C::STAGE_BYTES);
        for (int b = 0; b < C::NBOX; ++b)
          tma_load_3d(stages + s * C::STAGE_BYTES + b * C::BOX_BYTES, &xmap, &full_bar[s],
                      b * C::BOX_ELEMS, v0, head);
        issued_any = 1;
      }
      // Drain: wait until every issued load has landed before the CTA may exit.
      if (issued_any) {
        const long long n = tile_end - tile_begin;
        const long long first = n > C::STAGES ? n - C::STAGES : 0;
        for (long long it = first; it < n; ++it) {
          const int s = static_cast<int>(it % C::STAGES);
          if (!mbar_wait_bounded(&full_bar[s], static_cast<uint32_t>(it / C::STAGES) & 1u)) {
            atomicOr(&g_quant_error, kErrWaitTimeout);
            break;
          }
        }
      }
    }
    return;
  }

  // ---------------- consumers ----------------
  constexpr int P = C::P, VPW = C::VPW;
  const int part = lane / VPW;                 // which 64-element slice
  const int vl = lane % VPW;
  const int vt = warp * VPW + vl;              // row of this vector within the tile
  int cur_head = -1;

  for (long long t = tile_begin; t < tile_end; ++t) {
    const long long it = t - tile_begin;
    const int s = static_cast<int>(it % C::STAGES);
    const int head = static_cast<int>(t / args.tiles_per_head);
    const long long v = (t % args.tiles_per_head) * C::NV + vt;

    if (head != cur_head) {
      named_barrier(1, kConsumers);
      build_block_matrices<D, FULL, true>(args.params + static_cast<size_t>(head) * 2 * D, mat,
                                          tid, kConsumers);
      named_barrier(1, kConsumers);
      cur_head = head;
    }

    if (!mbar_wait_bounded(&full_bar[s], static_cast<uint32_t>(it / C::STAGES) & 1u) ||
        *abort_flag) {
      atomicOr(&g_quant_error, kErrWaitTimeout);
      *abort_flag = 1;
      return;
    }

    // Load this lane's 64 elements from the swizzled tile as float pairs.
    uint64_t xp[kE / 2];
    const unsigned char *stage = stages + s * C::STAGE_BYTES;
    if constexpr (C::ES == 2) {
      const unsigned char *box = stage + part * C::BOX_BYTES + vt * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 u = *reinterpret_cast<const uint4 *>(box + ((c ^ (vt & 7)) << 4));
        const __half2 *h = reinterpret_cast<const __half2 *>(&u);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = __half22float2(h[j]);
          xp[4 * c + j] = f2_pack(f.x, f.y);
        }
      }
    } else {
#pragma unroll
      for (int bx = 0; bx < 2; ++bx) {
        const unsigned char *box = stage + (2 * part + bx) * C::BOX_BYTES + vt * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const float4 f = *reinterpret_cast<const float4 *>(box + ((c ^ (vt & 7)) << 4));
          xp[16 * bx + 2 * c] = f2_pack(f.x, f.y);
          xp[16 * bx + 2 * c + 1] = f2_pack(f.z, f.w);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty_bar[s]);  // the stage may be refilled

    // Step 1: norm (float32 accumulation, reduced over the P lanes).
    uint64_t acc2 = f2_pack(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < kE / 2; ++k) acc2 = f2_fma(xp[k], xp[k], acc2);
    float ss_lo, ss_hi;
    f2_unpack(acc2, ss_lo, ss_hi);
    float ss = ss_lo + ss_hi;
#pragma unroll
    for (int k = 1; k < P; k <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, k * VPW);
    const float norm = sqrtf(ss);

    // Step 2: WHT stages h >= 4, then the folded (H_4, SO(4), 1/sqrt d) blocks.
    wht_inlane_h4_to_32(xp);
    wht_crosslane<P, VPW>(xp, part);
    apply_block_matrices(xp, mat + part * (kE / 4) * 16);
    float x[kE];
#pragma unroll
    for (int k = 0; k < kE / 2; ++k) f2_unpack(xp[k], x[2 * k], x[2 * k + 1]);

    // Step 3: Lloyd-Max codes against thresholds scaled by the norm.
    float ts[C::NPOS > 0 ? C::NPOS : 1];
#pragma unroll
    for (int j = 0; j < C::NPOS; ++j) ts[j] = args.tau[j] * norm;
    uint32_t w[C::TB / 4];
#pragma unroll
    for (int k = 0; k < C::TB / 4; ++k) w[k] = 0u;
#pragma unroll
    for (int i = 0; i < kE; ++i) {
      const float y = x[i];
      const float a = fabsf(y);
      int m = 0;
#pragma unroll
      for (int j = 0; j < C::NPOS; ++j) m += (a > ts[j]) ? 1 : 0;
      const uint32_t code = (y > 0.f) ? static_cast<uint32_t>(C::L / 2 + m)
                                      : static_cast<uint32_t>(C::L / 2 - 1 - m);
      // Step 4: bit-pack (layout in common.cuh).
      pack_code<BITS>(w, i, code);
    }

    if (v < args.n_vec) {
      const long long idx = static_cast<long long>(head) * args.out_head_stride + v;
      uint8_t *dst = args.codes + idx * C::PB + part * C::TB;
      if constexpr (C::TB % 16 == 0) {
#pragma unroll
        for (int k = 0; k < C::TB / 16; ++k)
          reinterpret_cast<uint4 *>(dst)[k] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
      } else {
#pragma unroll
        for (int k = 0; k < C::TB / 8; ++k)
          reinterpret_cast<uint2 *>(dst)[k] = make_uint2(w[2 * k], w[2 * k + 1]);
      }
      if (part == 0) args.norms[idx] = __half_as_ushort(__float2half_rn(norm));
    }
  }
}

// ---------------------------------------------------------------------------
// Dequantize
// ---------------------------------------------------------------------------

struct DequantArgs {
  const uint8_t *codes;
  const uint16_t *norms;
  const float *params;
  void *out;
  long long in_head_stride;
  long long head_stride;
  long long vec_stride;
  long long n_vec;
  int n_heads;
  int tiles_per_head;
  long long total_tiles;
  float centroid[16];
};

constexpr int kDequantThreads = 128;

template <typename T, int D, int BITS, bool FULL>
__global__ void __launch_bounds__(kDequantThreads) dequantize_kernel(const DequantArgs args) {
  constexpr int P = D / kE, VPW = 32 / P, NV = kDequantThreads / P;
  constexpr int L = 1 << BITS, PB = D * BITS / 8, TB = kE * BITS / 8;
  __shared__ __align__(16) float mat[(D / 4) * 16];
  __shared__ float cent[16];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int part = lane / VPW, vl = lane % VPW, vt = warp * VPW + vl;
  if (tid < L) cent[tid] = args.centroid[tid];

  const long long per_cta = (args.total_tiles + gridDim.x - 1) / gridDim.x;
  const long long tile_begin = static_cast<long long>(blockIdx.x) * per_cta;
  long long tile_end = tile_begin + per_cta;
  if (tile_end > args.total_tiles) tile_end = args.total_tiles;
  int cur_head = -1;

  for (long long t = tile_begin; t < tile_end; ++t) {
    const int head = static_cast<int>(t / args.tiles_per_head);
    const long long v = (t % args.tiles_per_head) * NV + vt;
    if (head != cur_head) {
      __syncthreads();
      build_block_matrices<D, FULL, false>(args.params + static_cast<size_t>(head) * 2 * D, mat,
                                           tid, kDequantThreads);
      __syncthreads();
      cur_head = head;
    }
    const bool valid = v < args.n_vec;
    const long long idx = static_cast<long long>(head) * args.in_head_stride + (valid ? v : 0);

    uint32_t w[TB / 4];
    const uint8_t *src = args.codes + idx * PB + part * TB;
    if constexpr (TB % 16 == 0) {
#pragma unroll
      for (int k = 0; k < TB / 16; ++k) {
        const uint4 u = reinterpret_cast<const uint4 *>(src)[k];
        w[4 * k] = u.x; w[4 * k + 1] = u.y; w[4 * k + 2] = u.z; w[4 * k + 3] = u.w;
      }
    } else {
#pragma unroll
      for (int k = 0; k < TB / 8; ++k) {
        const uint2 u = reinterpret_cast<const uint2 *>(src)[k];
        w[2 * k] = u.x; w[2 * k + 1] = u.y;
      }
    }
    const float s16 = __half2float(__ushort_as_half(args.norms[idx]));

    uint64_t xp[kE / 2];
#pragma unroll
    for (int k = 0; k < kE / 2; ++k)
      xp[k] = f2_pack(cent[unpack_code<BITS>(w, 2 * k)], cent[unpack_code<BITS>(w, 2 * k + 1)]);
    apply_block_matrices(xp, mat + part * (kE / 4) * 16);
    wht_inlane_h4_to_32(xp);
    wht_crosslane<P, VPW>(xp, part);
    const uint64_t s2 = f2_pack(s16, s16);
#pragma unroll
    for (int k = 0; k < kE / 2; ++k) xp[k] = f2_mul(xp[k], s2);
    float x[kE];
#pragma unroll
    for (int k = 0; k < kE / 2; ++k) f2_unpack(xp[k], x[2 * k], x[2 * k + 1]);

    if (valid) {
      T *dst = static_cast<T *>(args.out) + static_cast<long long>(head) * args.head_stride +
               v * args.vec_stride + part * kE;
      if constexpr (sizeof(T) == 2) {
#pragma unroll
        for (int c = 0; c < kE / 8; ++c) {
          uint4 u;
          __half2 *h = reinterpret_cast<__half2 *>(&u);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            h[j] = __floats2half2_rn(x[8 * c + 2 * j], x[8 * c + 2 * j + 1]);
          reinterpret_cast<uint4 *>(dst)[c] = u;
        }
      } else {
#pragma unroll
        for (int c = 0; c < kE / 4; ++c)
          reinterpret_cast<float4 *>(dst)[c] = make_float4(x[4 * c], x[4 * c + 1], x[4 * c + 2],
                                                           x[4 * c + 3]);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
  return n;
}

template <typename T, int D, int BITS, bool FULL>
int launch_quantize(const void *x, int n_heads, long long n_vec, long long head_stride,
                    long long vec_stride, const float *params, uint8_t *codes, uint16_t *norms,
                    long long out_head_stride, cudaStream_t stream) {
  using C = Cfg<T, D, BITS>;
  auto kernel = quantize_kernel<T, D, BITS, FULL>;
  static int max_ctas_per_sm = -1;
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (max_ctas_per_sm < 0) {
      cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
      if (e != cudaSuccess)
        return set_error(ISOQ_ERR_CUDA, "quantize: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
      int n = 0;
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, kQuantThreads, C::SMEM);
      if (e != cudaSuccess)
        return set_error(ISOQ_ERR_CUDA, "quantize: occupancy: %s", cudaGetErrorString(e));
      max_ctas_per_sm = n < 1 ? 1 : n;
    }
  }

  EncodeTiledFn encode = encode_tiled_fn();
  if (!encode) return set_error(ISOQ_ERR_CUDA, "quantize: cuTensorMapEncodeTiled unavailable");
  CUtensorMap map;
  const cuuint64_t gdim[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(n_vec),
                              static_cast<cuuint64_t>(n_heads)};
  const long long hs = n_heads > 1 ? head_stride : vec_stride * n_vec;
  const cuuint64_t gstride[2] = {static_cast<cuuint64_t>(vec_stride * C::ES),
                                 static_cast<cuuint64_t>(hs * C::ES)};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(C::BOX_ELEMS), static_cast<cuuint32_t>(C::NV), 1u};
  const cuuint32_t estride[3] = {1u, 1u, 1u};
  CUresult r = encode(&map, C::ES == 2 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                      3, const_cast<void *>(x), gdim, gstride, box, estride,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(ISOQ_ERR_UNSUPPORTED, "quantize: tensor map encode failed (%d)", (int)r);

  QuantArgs a;
  a.params = params;
  a.codes = codes;
  a.norms = norms;
  a.out_head_stride = out_head_stride;
  a.n_vec = n_vec;
  a.n_heads = n_heads;
  a.tiles_per_head = static_cast<int>((n_vec + C::NV - 1) / C::NV);
  a.total_tiles = static_cast<long long>(a.tiles_per_head) * n_heads;
  CodebookF32 cb;
  codebook_f32(D, BITS, &cb);
  for (int j = 0; j < 7; ++j) a.tau[j] = j < C::NPOS ? cb.threshold[C::L / 2 + j] : 0.f;

  long long grid = static_cast<long long>(num_sms()) * max_ctas_per_sm;
  if (grid > a.total_tiles) grid = a.total_tiles;
  kernel<<<static_cast<unsigned>(grid), kQuantThreads, C::SMEM, stream>>>(map, a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(ISOQ_ERR_CUDA, "quantize launch: %s", cudaGetErrorString(e));
  return ISOQ_OK;
}

template <typename T, int D, int BITS, bool FULL>
int launch_dequantize(const uint8_t *codes, const uint16_t *norms, int n_heads, long long n_vec,
                      long long in_head_stride, const float *params, void *out,
                      long long head_stride, long long vec_stride, cudaStream_t stream) {
  constexpr int NV = kDequantThreads / (D / kE);
  auto kernel = dequantize_kernel<T, D, BITS, FULL>;
  static int max_ctas_per_sm = -1;
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (max_ctas_per_sm < 0) {
      int n = 0;
      cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, kDequantThreads, 0);
      if (e != cudaSuccess)
        return set_error(ISOQ_ERR_CUDA, "dequantize: occupancy: %s", cudaGetErrorString(e));
      max_ctas_per_sm = n < 1 ? 1 : n;
    }
  }
  DequantArgs a;
  a.codes = codes;
  a.norms = norms;
  a.params = params;
  a.out = out;
  a.in_head_stride = in_head_stride;
  a.head_stride = head_stride;
  a.vec_stride = vec_stride;
  a.n_vec = n_vec;
  a.n_heads = n_heads;
  a.tiles_per_head = static_cast<int>((n_vec + NV - 1) / NV);
  a.total_tiles = static_cast<long long>(a.tiles_per_head) * n_heads;
  CodebookF32 cb;
  codebook_f32(D, BITS, &cb);
  for (int j = 0; j < 16; ++j) a.centroid[j] = j < cb.levels ? cb.centroid[j] : 0.f;
  long long grid = static_cast<long long>(num_sms()) * max_ctas_per_sm;
  if (grid > a.total_tiles) grid = a.total_tiles;
  kernel<<<static_cast<unsigned>(grid), kDequantThreads, 0, stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(ISOQ_ERR_CUDA, "dequantize launch: %s", cudaGetErrorString(e));
  return ISOQ_OK;
}

// Expands the runtime (dtype, d, bits, variant) into a template instantiation.
template <template <typename, int, int, bool> class F, typename... A>
int dispatch(int dtype, int d, int bits, int variant, A... args) {
#define ISOQ_CASE_V(T, D, B)                                              \
  return variant == ISOQ_FULL ? F<T, D, B, true>::run(args...)           \
                              : F<T, D, B, false>::run(args...)
#define ISOQ_CASE_B(T, D)                  \
  switch (bits) {                          \
    case 2: ISOQ_CASE_V(T, D, 2);          \
    case 3: ISOQ_CASE_V(T, D, 3);          \
    default: ISOQ_CASE_V(T, D, 4);         \
  }
#define ISOQ_CASE_D(T)                     \
  switch (d) {                             \
    case 128: ISOQ_CASE_B(T, 128);         \
    case 256: ISOQ_CASE_B(T, 256);         \
    default: ISOQ_CASE_B(T, 512);          \
  }
  if (dtype == ISOQ_F16) {
    ISOQ_CASE_D(__half);
  } else {
    ISOQ_CASE_D(float);
  }
#undef ISOQ_CASE_D
#undef ISOQ_CASE_B
#undef ISOQ_CASE_V
}

template <typename T, int D, int B, bool FULL>
struct QuantizeRunner {
  static int run(const void *x, int n_heads, long long n_vec, long long hs, long long vs,
                 const float *params, uint8_t *codes, uint16_t *norms, long long ohs,
                 cudaStream_t st) {
    return launch_quantize<T, D, B, FULL>(x, n_heads, n_vec, hs, vs, params, codes, norms, ohs, st);
  }
};

template <typename T, int D, int B, bool FULL>
struct DequantizeRunner {
  static int run(const uint8_t *codes, const uint16_t *norms, int n_heads, long long n_vec,
                 long long ihs, const float *params, void *out, long long hs, long long vs,
                 cudaStream_t st) {
    return launch_dequantize<T, D, B, FULL>(codes, norms, n_heads, n_vec, ihs, params, out, hs, vs, st);
  }
};

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace quant
}  // namespace isoq

using namespace isoq;

extern "C" {

int isoq_quantize(const void *x_dev, int dtype, int n_heads, int64_t n_vec, int d, int bits,
                  int variant, int64_t head_stride, int64_t vec_stride, const float *params_dev,
                  uint8_t *codes_dev, uint16_t *norms_dev, int64_t out_head_stride,
                  isoq_stream_t stream) {
  clear_error();
  if (!supported_d(d)) return set_error(ISOQ_ERR_UNSUPPORTED, "d=%d not supported", d);
  if (!supported_bits(bits)) return set_error(ISOQ_ERR_UNSUPPORTED, "bits=%d not supported", bits);
  if (!supported_variant(variant)) return set_error(ISOQ_ERR_UNSUPPORTED, "variant=%d", variant);
  if (!supported_dtype(dtype)) return set_error(ISOQ_ERR_UNSUPPORTED, "dtype=%d", dtype);
  if (n_heads < 0 || n_vec < 0) return set_error(ISOQ_ERR_INVALID_ARG, "negative size");
  if (n_heads == 0 || n_vec == 0) return ISOQ_OK;
  if (n_vec >= (1ll << 31) || n_heads >= (1 << 24))
    return set_error(ISOQ_ERR_INVALID_ARG, "n_vec or n_heads too large");
  if (!x_dev || !params_dev || !codes_dev || !norms_dev)
    return set_error(ISOQ_ERR_INVALID_ARG, "null pointer");
  if (vec_stride < d || (n_heads > 1 && head_stride < 1) || out_head_stride < n_vec)
    return set_error(ISOQ_ERR_INVALID_ARG, "bad stride");
  const int es = elt_size(dtype);
  if (!quant::aligned16(x_dev) || (vec_stride * es) % 16 || (n_heads > 1 && (head_stride * es) % 16))
    return set_error(ISOQ_ERR_UNSUPPORTED, "x and its strides must be 16-byte aligned");
  if (!quant::aligned16(codes_dev) || !quant::aligned16(params_dev) || (reinterpret_cast<uintptr_t>(norms_dev) & 1))
    return set_error(ISOQ_ERR_UNSUPPORTED, "codes/params must be 16-byte aligned, norms 2-byte aligned");
  return quant::dispatch<quant::QuantizeRunner>(dtype, d, bits, variant, x_dev, n_heads,
                                                (long long)n_vec, (long long)head_stride,
                                                (long long)vec_stride, params_dev, codes_dev,
                                                norms_dev, (long long)out_head_stride,
                                                reinterpret_cast<cudaStream_t>(stream));
}

int isoq_dequantize(const uint8_t *codes_dev, const uint16_t *norms_dev, int n_heads,
                    int64_t n_vec, int d, int bits, int variant, int64_t in_head_stride,
                    const float *params_dev, void *out_dev, int out_dtype, int64_t head_stride,
                    int64_t vec_stride, isoq_stream_t stream) {
  clear_error();
  if (!supported_d(d)) return set_error(ISOQ_ERR_UNSUPPORTED, "d=%d not supported", d);
  if (!supported_bits(bits)) return set_error(ISOQ_ERR_UNSUPPORTED, "bits=%d not supported", bits);
  if (!supported_variant(variant)) return set_error(ISOQ_ERR_UNSUPPORTED, "variant=%d", variant);
  if (!supported_dtype(out_dtype)) return set_error(ISOQ_ERR_UNSUPPORTED, "dtype=%d", out_dtype);
  if (n_heads < 0 || n_vec < 0) return set_error(ISOQ_ERR_INVALID_ARG, "negative size");
  if (n_heads == 0 || n_vec == 0) return ISOQ_OK;
  if (n_vec >= (1ll << 31) || n_heads >= (1 << 24))
    return set_error(ISOQ_ERR_INVALID_ARG, "n_vec or n_heads too large");
  if (!codes_dev || !norms_dev || !params_dev || !out_dev)
    return set_error(ISOQ_ERR_INVALID_ARG, "null pointer");
  if (in_head_stride < n_vec || vec_stride < d || (n_heads > 1 && head_stride < 1))
    return set_error(ISOQ_ERR_INVALID_ARG, "bad stride");
  const int es = elt_size(out_dtype);
  if (!quant::aligned16(out_dev) || (vec_stride * es) % 16 || (n_heads > 1 && (head_stride * es) % 16))
    return set_error(ISOQ_ERR_UNSUPPORTED, "out and its strides must be 16-byte aligned");
  if (!quant::aligned16(codes_dev) || !quant::aligned16(params_dev) || (reinterpret_cast<uintptr_t>(norms_dev) & 1))
    return set_error(ISOQ_ERR_UNSUPPORTED, "codes/params must be 16-byte aligned, norms 2-byte aligned");
  return quant::dispatch<quant::DequantizeRunner>(out_dtype, d, bits, variant, codes_dev, norms_dev,
                                                  n_heads, (long long)n_vec, (long long)in_head_stride,
                                                  params_dev, out_dev, (long long)head_stride,
                                                  (long long)vec_stride,
                                                  reinterpret_cast<cudaStream_t>(stream));
}

// Reads and clears this translation unit's device error word.
__attribute__((visibility("hidden"))) int isoq_detail_take_quant_error(cudaStream_t stream, unsigned *out) {
  unsigned zero = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(out, quant::g_quant_error, sizeof(unsigned), 0,
                                            cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e == cudaSuccess && *out)
    e = cudaMemcpyToSymbolAsync(quant::g_quant_error, &zero, sizeof(unsigned), 0,
                                cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  return e == cudaSuccess ? ISOQ_OK : set_error(ISOQ_ERR_CUDA, "error word: %s", cudaGetErrorString(e));
}

}  // extern "C"
