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
// 64 elements per lane, as two groups of 32 (the 32-code groups of the packed
// layout).  Inside a group the elements are held as 16 packed float pairs
// (e, e + 16), so every butterfly or block product that acts on whole pairs
// is one f32x2 instruction for two elements.
//
// The Walsh-Hadamard stages commute, so they run in whatever order suits the
// registers:
//   h = 16       inside a pair (for float16 input, fused with the conversion),
//   h = 4, 8     between pairs of a group,
//   h = 32       between the two groups of a lane,
//   h = 64 .. d/4  by warp shuffle, every pair exchanged,
//   h = d/2      by a half exchange: each lane sends one group and keeps one,
//                so the stage moves half the data of a full exchange.
// The stages h = 1, 2 act inside each 4-block and are folded into one 4x4
// matrix per block together with the SO(4) map and 1/sqrt(d):
//   quantize:   M_i = R_i H_4 / sqrt(d)   applied after the other stages,
//   dequantize: N_i = H_4 R_i^T / sqrt(d) applied before them.
// The block pairs (i, i + 4) of a group share registers, so the matrices are
// stored interleaved (M_i[j][c], M_{i+4}[j][c]).
//
// After the half exchange, the lane whose part has the exchange bit clear
// holds the lower 32 elements of its own 64 and of its partner's, and the
// lane with the bit set holds the upper 32 of both, the latter negated; the
// negation is folded into that group's block matrices.
//
// The quantiser compares the unnormalised R x with s * t_k (no division per
// element) using the symmetry of the codebook: the magnitude is counted
// against the positive thresholds with exact 0/1 steps from saturating FMAs,
// and the sign, taken by the integer pipe, signs the field weight with which
// one FMA adds the code into its packed word.
//
// Data movement.  Each warp of a quantize CTA streams its own rows through a
// ring of 128B-swizzled TMA tiles (no producer warp); each lane reads its own
// 128-byte row segments conflict-free.  Each lane writes whole 32-code groups.
//
// The kernels above serve every shape; for d = 128 with the WHT, float16
// input (quantize) or float16 output with 2- or 3-bit codes (dequantize), the
// launchers take the tensor-core forms instead (quant_tc.cuh, dequant_tc.cuh),
// where the whole rotation is one tcgen05 product per 128-vector tile.

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "tcgen05.cuh"
#include "internal.h"

namespace isoq {
namespace quant {

using namespace isoq::dev;

constexpr int kE = 64;              // elements per lane
constexpr int kPairs = kE / 2;      // packed pairs per lane
constexpr int kGP = 16;             // packed pairs per 32-element group
constexpr int kQuantWarps = 4;
constexpr int kQuantThreads = 32 * kQuantWarps;
constexpr int kDequantThreads = 128;

// Rotation kinds of the kernels (the variants of include/isoq.h map onto
// them in rotation_kind): the WHT composed with the full block map
// q_L v conj(q_R) (Full, and the 2-D special case, whose parameters make the
// same map two plane rotations), the WHT with the left factor only (Fast),
// and the full block map alone (the ablation's v2, and v1 with q_R = q_L).
constexpr int kRotWhtFull = 0;
constexpr int kRotWhtFast = 1;
constexpr int kRotBlock = 2;

__device__ unsigned int g_quant_error = 0;

// Lane geometry shared by both directions.
template <int D>
struct Lanes {
  static constexpr int P = D / kE;      // lanes per vector
  static constexpr int VPW = 32 / P;    // vectors per warp
  static constexpr int KH = P / 2;      // part bit of the half-exchange stage
};

template <typename T, int D, int BITS>
struct Cfg : Lanes<D> {
  using Lanes<D>::P;
  using Lanes<D>::VPW;
  static constexpr int NV = kQuantWarps * VPW;  // vectors per CTA tile
  static constexpr int ES = sizeof(T);
  static constexpr int BOX_ELEMS = 128 / ES;    // elements in one 128-byte chunk of a row
  // A box holds CPB consecutive 128-byte chunks of each of the warp's VPW
  // rows, so that it fills the 1024 bytes a 128B-swizzled box is aligned to
  // (d = 512: 4 rows x 2 chunks; the rows are then viewed as [chunk][elem]
  // by a 4-D tensor map).
  static constexpr int CPB = VPW >= 8 ? 1 : 8 / VPW;
  static constexpr int NBOX = D * ES / 128 / CPB;   // boxes per row
  static constexpr int BOX_BYTES = VPW * CPB * 128; // one warp's rows of one box
  static constexpr int BOX_STRIDE = BOX_BYTES < 1024 ? 1024 : BOX_BYTES;
  static constexpr int STAGE_BYTES = NBOX * BOX_STRIDE;
  static constexpr int STAGES = STAGE_BYTES >= 8192 ? 2 : 3;
  static constexpr int RING_BYTES = STAGES * STAGE_BYTES;
  static constexpr int L = 1 << BITS;
  static constexpr int NPOS = L / 2 - 1;        // positive thresholds
  static constexpr int PB = D * BITS / 8;       // packed bytes per vector
  static constexpr int GB = 32 * BITS / 8;      // packed bytes per 32-code group
  static constexpr int MAT_BYTES = D * 16;      // D/4 blocks of 16 floats
  static constexpr int SMEM = kQuantWarps * RING_BYTES + MAT_BYTES + kQuantWarps * STAGES * 8 + 1024;
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

// ---------------------------------------------------------------------------
// Register-level pieces
// ---------------------------------------------------------------------------

__device__ __forceinline__ void tma_load_4d(void *dst, const CUtensorMap *map, uint64_t *bar,
                                            int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

// Shared address of chunk ch (128 bytes of a row) of the warp's row vl in a
// ring stage, and the row's swizzle phase there: inside a box the 128-byte
// lines run (row, chunk) with the chunk fastest.
template <typename C>
__device__ __forceinline__ uint32_t stage_line(uint32_t stage, int ch, int vl, uint32_t &sw) {
  const int line = vl * C::CPB + ch % C::CPB;
  sw = static_cast<uint32_t>(line & 7);
  return stage + (ch / C::CPB) * C::BOX_STRIDE + line * 128;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

__device__ __forceinline__ void lds2x64(uint32_t addr, uint64_t &a, uint64_t &b) {
  asm volatile("ld.shared.v2.b64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "r"(addr));
}

// Groups of the final layout held by a lane (see the file comment): g[0] and
// g[1] are 32-element group indices within the vector.
template <int D>
__device__ __forceinline__ void lane_groups(int part, int (&g)[2]) {
  constexpr int KH = Lanes<D>::KH;
  if (part & KH) {
    g[0] = 2 * (part - KH) + 1;
    g[1] = 2 * part + 1;
  } else {
    g[0] = 2 * part;
    g[1] = 2 * (part + KH);
  }
}

// True for the groups a lane holds negated after the half exchange.
template <int D>
__host__ __device__ constexpr bool group_negated(int g) {
  return (g & 1) && (((g >> 1) & Lanes<D>::KH) != 0);
}

// Per-block 4x4 matrices of one head, stored for the packed product:
// group g, block pair beta (blocks 8g + beta and 8g + beta + 4), entry
// (j, c) -> float pair at mat[128 g + 32 beta + 2 (4 j + c) + {0, 1}].
//   forward: M_i = R_i H_4 / sqrt(d); inverse: N_i = H_4 R_i^T / sqrt(d);
//   without the WHT (kRotBlock): M_i = R_i, N_i = R_i^T.
template <int D, int RK, bool FORWARD>
__device__ void build_block_matrices(const float *params_head, float *mat, int tid, int nthreads) {
  constexpr bool FULL = RK != kRotWhtFast;
  constexpr bool WHT = RK != kRotBlock;
  const float inv_sqrt_d = WHT ? rsqrtf(static_cast<float>(D)) : 1.f;
  for (int b = tid; b < D / 4; b += nthreads) {
    const Quat ql = load_quat(params_head + 8 * b);
    const Quat qr = load_quat(params_head + 8 * b + 4);
    float m[4][4];
    for (int c = 0; c < 4; ++c) {
      const Quat e{c == 0 ? 1.f : 0.f, c == 1 ? 1.f : 0.f, c == 2 ? 1.f : 0.f, c == 3 ? 1.f : 0.f};
      if (FORWARD) {
        // column c = R_i (H_4 e_c), or R_i e_c without the WHT
        const Quat u = block_forward(ql, qr, WHT ? h4_column(c) : e, FULL);
        m[0][c] = u.w; m[1][c] = u.x; m[2][c] = u.y; m[3][c] = u.z;
      } else if (WHT) {
        // column c = H_4 (R_i^T e_c)
        const Quat u = block_inverse(ql, qr, e, FULL);
        m[0][c] = u.w + u.x + u.y + u.z;
        m[1][c] = u.w - u.x + u.y - u.z;
        m[2][c] = u.w + u.x - u.y - u.z;
        m[3][c] = u.w - u.x - u.y + u.z;
      } else {
        // column c = R_i^T e_c
        const Quat u = block_inverse(ql, qr, e, FULL);
        m[0][c] = u.w; m[1][c] = u.x; m[2][c] = u.y; m[3][c] = u.z;
      }
    }
    const int g = b >> 3, r = b & 7, beta = r & 3, half = r >> 2;
    const float sc = WHT && group_negated<D>(g) ? -inv_sqrt_d : inv_sqrt_d;
    float *out = mat + 128 * g + 32 * beta + half;
    for (int j = 0; j < 4; ++j)
      for (int c = 0; c < 4; ++c) out[2 * (4 * j + c)] = m[j][c] * sc;
  }
}

// Applies the block matrices of one group (16 pairs starting at xp[base]).
template <int NP>
__device__ __forceinline__ void apply_group_matrices(uint64_t (&xp)[NP], int base, uint32_t mat_g) {
#pragma unroll
  for (int beta = 0; beta < 4; ++beta) {
    const uint64_t z0 = xp[base + 4 * beta], z1 = xp[base + 4 * beta + 1];
    const uint64_t z2 = xp[base + 4 * beta + 2], z3 = xp[base + 4 * beta + 3];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint64_t m0, m1, m2, m3;
      lds2x64(mat_g + 128 * beta + 32 * j, m0, m1);
      lds2x64(mat_g + 128 * beta + 32 * j + 16, m2, m3);
      uint64_t y = f2_mul(m0, z0);
      y = f2_fma(m1, z1, y);
      y = f2_fma(m2, z2, y);
      y = f2_fma(m3, z3, y);
      xp[base + 4 * beta + j] = y;
    }
  }
}

// Butterflies between pairs of each group, strides h = 4 and 8 (pair
// distance 4 and 8).
__device__ __forceinline__ void wht_pairs_h4_h8(uint64_t (&xp)[kPairs]) {
#pragma unroll
  for (int hp = 4; hp <= 8; hp <<= 1) {
#pragma unroll
    for (int k = 0; k < kPairs; ++k) {
      if (!(k & hp)) {
        const uint64_t a = xp[k], b = xp[k + hp];
        xp[k] = f2_add(a, b);
        xp[k + hp] = f2_sub(a, b);
      }
    }
  }
}

// Butterfly inside each pair (h = 16): (a, b) -> (a + b, a - b).
__device__ __forceinline__ void wht_in_pair(uint64_t (&xp)[kPairs]) {
#pragma unroll
  for (int k = 0; k < kPairs; ++k) {
    float a, b;
    f2_unpack(xp[k], a, b);
    xp[k] = f2_pack(a + b, a - b);
  }
}

// Full-exchange stages h = 64 .. d/4 (part bits below KH).
template <int D>
__device__ __forceinline__ void wht_cross_full(uint64_t (&xp)[kPairs], int part) {
  constexpr int KH = Lanes<D>::KH, VPW = Lanes<D>::VPW;
#pragma unroll
  for (int k = 1; k < KH; k <<= 1) {
    const float sgn = (part & k) ? -1.f : 1.f;
    const uint64_t sgn2 = f2_pack(sgn, sgn);
#pragma unroll
    for (int i = 0; i < kPairs; ++i) {
      const uint64_t o = __shfl_xor_sync(0xffffffffu, xp[i], k * VPW);
      xp[i] = f2_fma(sgn2, xp[i], o);
    }
  }
}

// The Lloyd-Max search runs on the FMA pipe.  With `big` a power of two that
// scales a coordinate of the vector to about 2^40 (one float ulp of any scaled
// threshold is then >= 1), fma.sat(|y|, big, -t big) is exactly 1.0 when
// |y| > t and 0.0 otherwise (ties go to the lower code).  Codes are then
// small exact integers in float32, and the packing accumulates them as exact
// integers below 2^24 (offset by 2^23, so that the low 16 bits of the float
// are the packed field).
__device__ __forceinline__ float fma_sat(float a, float b, float c) {
  float r;
  asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Power of two about 2^40 / norm (clamped to [2^-126, 2^127]; 2^127 for a
// zero norm).
__device__ __forceinline__ float search_scale(float norm) {
  int e = 294 - static_cast<int>((__float_as_uint(norm) >> 23) & 0xFFu);
  e = e < 1 ? 1 : (e > 254 ? 254 : e);
  return __uint_as_float(static_cast<uint32_t>(e) << 23);
}

// Codes of one group (16 pairs (e, e + 16) from xp[base]) packed into its
// GB/4 words (layout in common.cuh).  tb[j] = -t_j big for the positive
// thresholds t_j scaled by the norm.
//
// With m = #{j : |y| > t_j} (one saturating FMA per threshold), the code is
// L/2 + m for y > 0 and L/2 - 1 - m otherwise, i.e. (L/2 - 1/2) + sg (m + 1/2)
// with sg = +-1.  The packing accumulates code * w for the field weight w of
// each position as one FMA, (sg w) (m + 1/2), onto the constant
// 2^22 + (L/2 - 1/2) sum w; sg w is w with y's sign bit ORed in by one
// integer logic op.  That counts +0 as positive, which only a zero vector
// produces (any other exact zero lies on the threshold 0 itself, where either
// code is nearest): for a zero vector, zmask = 0x80000000 makes every weight
// negative, so all its codes are L/2 - 1 as the rule #{k : y > t_k} gives.  Every partial sum is a multiple of 1/2 in [2^22, 2^23),
// where float32 steps by 1/2, so all of it is exact, and the packed field
// is the float's mantissa shifted right by one bit.
template <int BITS, int NP>
__device__ __forceinline__ void quantize_group(const uint64_t (&xp)[NP], int base,
                                               const float *tb, float big, uint32_t zmask, uint32_t *w) {
  constexpr int L = 1 << BITS, NPOS = L / 2 - 1;
  constexpr int PER_HALF = 16 / BITS == 5 ? 4 : 16 / BITS;   // codes per 16-bit half (3 bits: 4-bit fields)
  constexpr int FIELD = BITS == 3 ? 4 : BITS;
  constexpr int NACC = kGP / PER_HALF;
  constexpr float WSUM = static_cast<float>(((1u << (FIELD * PER_HALF)) - 1u) / ((1u << FIELD) - 1u));
  const float c0 = 4194304.f + (static_cast<float>(L / 2) - 0.5f) * WSUM;
  const uint64_t half2 = f2_pack(0.5f, 0.5f);
  uint32_t lo[NACC], hi[NACC];
#pragma unroll
  for (int q = 0; q < NACC; ++q) {
    uint64_t acc = f2_pack(c0, c0);
#pragma unroll
    for (int j = 0; j < PER_HALF; ++j) {
      const int p = PER_HALF * q + j;
      float y0, y1;
      f2_unpack(xp[base + p], y0, y1);
      const float a0 = fabsf(y0), a1 = fabsf(y1);
      // m + 1/2
      uint64_t m;
      if constexpr (NPOS == 3) {
        // Two levels: s2 = [|y| > t_2], then |y| against t_3 if s2 else t_1
        // (the thresholds increase, so m = 2 s2 + [|y| > that threshold]).
        // The selected threshold t_1 + s2 (t_3 - t_1) is t_1 exactly or t_3
        // to within two roundings (a few 1e-8 of it, far inside the band
        // where the pages' real-valued decision is itself that close).
        const uint64_t s2 = f2_pack(fma_sat(a0, big, tb[1]), fma_sat(a1, big, tb[1]));
        const float d31 = tb[2] - tb[0];
        const uint64_t tsel = f2_fma(s2, f2_pack(d31, d31), f2_pack(tb[0], tb[0]));
        float t0, t1;
        f2_unpack(tsel, t0, t1);
        const uint64_t s13 = f2_pack(fma_sat(a0, big, t0), fma_sat(a1, big, t1));
        m = f2_fma(s2, f2_pack(2.f, 2.f), f2_add(s13, half2));
      } else {
        m = f2_pack(fma_sat(a0, big, tb[0]), fma_sat(a1, big, tb[0]));
#pragma unroll
        for (int k = 1; k < NPOS; ++k) m = f2_add(m, f2_pack(fma_sat(a0, big, tb[k]), fma_sat(a1, big, tb[k])));
        m = f2_add(m, half2);
      }
      // sg w: the field weight with y's sign (negative for a zero vector)
      const uint32_t wb = __float_as_uint(static_cast<float>(1u << (FIELD * j))) | zmask;
      const uint32_t s0 = wb | (__float_as_uint(y0) & 0x80000000u);
      const uint32_t s1 = wb | (__float_as_uint(y1) & 0x80000000u);
      acc = f2_fma(f2_pack(__uint_as_float(s0), __uint_as_float(s1)), m, acc);
    }
    float fl, fh;
    f2_unpack(acc, fl, fh);
    lo[q] = __float_as_uint(fl) >> 1;
    hi[q] = __float_as_uint(fh) >> 1;
  }
  if constexpr (BITS == 2) {
    // words: codes 0..15 (low elements), codes 16..31 (high elements)
    w[0] = __byte_perm(lo[0], lo[1], 0x5410);
    w[1] = __byte_perm(hi[0], hi[1], 0x5410);
  } else {
    // words: codes 0..7, 8..15 (low elements), 16..23, 24..31 (high elements)
    const uint32_t w0 = __byte_perm(lo[0], lo[1], 0x5410), w1 = __byte_perm(lo[2], lo[3], 0x5410);
    const uint32_t w2 = __byte_perm(hi[0], hi[1], 0x5410), w3 = __byte_perm(hi[2], hi[3], 0x5410);
    if constexpr (BITS == 3) {
      // codes 24..31 go to the spare bits: bit r of code 24 + j -> bit 4j + 3 of word r
      w[0] = w0 + (w3 & 0x11111111u) * 8u;
      w[1] = w1 + (w3 & 0x22222222u) * 4u;
      w[2] = w2 + (w3 & 0x44444444u) * 2u;
    } else {
      w[0] = w0;
      w[1] = w1;
      w[2] = w2;
      w[3] = w3;
    }
  }
}

// ---------------------------------------------------------------------------
// Quantize
// ---------------------------------------------------------------------------

template <typename T, int D, int BITS, int RK>
__global__ void __launch_bounds__(kQuantThreads, 4)
    quantize_kernel(const __grid_constant__ CUtensorMap xmap, const QuantArgs args) {
  using C = Cfg<T, D, BITS>;
  constexpr int P = C::P, VPW = C::VPW, KH = C::KH;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  unsigned char *ring = smem + warp * C::RING_BYTES;
  float *mat = reinterpret_cast<float *>(smem + kQuantWarps * C::RING_BYTES);
  uint64_t *full_bar =
      reinterpret_cast<uint64_t *>(smem + kQuantWarps * C::RING_BYTES + C::MAT_BYTES) + warp * C::STAGES;

  // Contiguous range of CTA tiles (few head changes per CTA).  Every warp
  // walks the same tiles, taking rows [warp * VPW, warp * VPW + VPW) of each.
  const long long per_cta = (args.total_tiles + gridDim.x - 1) / gridDim.x;
  const long long tile_begin = static_cast<long long>(blockIdx.x) * per_cta;
  long long tile_end = tile_begin + per_cta;
  if (tile_end > args.total_tiles) tile_end = args.total_tiles;
  const int n_mine = tile_end > tile_begin ? static_cast<int>(tile_end - tile_begin) : 0;

  if (lane == 0) {
    for (int s = 0; s < C::STAGES; ++s) mbar_init(&full_bar[s], 1);
    mbar_fence_init();
  }
  __syncwarp();

  auto issue = [&](int i) {
    const long long t = tile_begin + i;
    const int head = static_cast<int>(t / args.tiles_per_head);
    const int v0 = static_cast<int>((t % args.tiles_per_head) * C::NV) + warp * VPW;
    const int s = i % C::STAGES;
    unsigned char *st = ring + s * C::STAGE_BYTES;
    mbar_arrive_expect_tx(&full_bar[s], C::NBOX * C::BOX_BYTES);
    for (int b = 0; b < C::NBOX; ++b) {
      if constexpr (C::CPB == 1)
        tma_load_3d(st + b * C::BOX_STRIDE, &xmap, &full_bar[s], b * C::BOX_ELEMS, v0, head);
      else
        tma_load_4d(st + b * C::BOX_STRIDE, &xmap, &full_bar[s], 0, b * C::CPB, v0, head);
    }
  };
  int issued = 0;
  if (lane == 0)
    for (; issued < n_mine && issued < C::STAGES; ++issued) issue(issued);

  int cur_head = -1;
  if (n_mine > 0) {
    cur_head = static_cast<int>(tile_begin / args.tiles_per_head);
    build_block_matrices<D, RK, true>(args.params + static_cast<size_t>(cur_head) * 2 * D, mat,
                                        tid, kQuantThreads);
  }
  __syncthreads();

  constexpr bool WHT = RK != kRotBlock;
  const int part = lane / VPW;
  const int vl = lane % VPW;
  const bool hb = (part & KH) != 0;
  // Without the WHT nothing moves between lanes: each lane keeps the two
  // groups it loaded.
  int grp[2] = {2 * part, 2 * part + 1};
  if (WHT) lane_groups<D>(part, grp);
  const uint32_t mat_s = smem_u32(mat);
  const float sg = hb ? -1.f : 1.f;
  const uint64_t sig2 = f2_pack(sg, sg), nsig2 = f2_pack(-sg, -sg);
  bool failed = false;
  int consumed = 0;

  for (int i = 0; i < n_mine; ++i) {
    const long long t = tile_begin + i;
    const int head = static_cast<int>(t / args.tiles_per_head);
    if (head != cur_head) {
      // Every warp walks the same tiles, so all of them meet here.
      named_barrier(1, kQuantThreads);
      build_block_matrices<D, RK, true>(args.params + static_cast<size_t>(head) * 2 * D, mat,
                                          tid, kQuantThreads);
      named_barrier(1, kQuantThreads);
      cur_head = head;
    }
    if (failed) continue;
    const int s = i % C::STAGES;
    const bool ok = mbar_wait_bounded(&full_bar[s], static_cast<uint32_t>(i / C::STAGES) & 1u);
    if (__any_sync(0xffffffffu, !ok)) {
      if (lane == 0) atomicOr(&g_quant_error, kErrWaitTimeout);
      failed = true;
      continue;
    }

    // Load this lane's 64 elements (two groups of 16 pairs (e, e + 16)),
    // doing the h = 16 butterfly on the way.
    uint64_t xp[kPairs];
    const uint32_t stage = smem_u32(ring + s * C::STAGE_BYTES);
    if constexpr (C::ES == 2) {
      uint32_t sw;
      const uint32_t row = stage_line<C>(stage, part, vl, sw);
#pragma unroll
      for (int G = 0; G < 2; ++G) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const uint4 ulo = lds128(row + (((4 * G + c) ^ sw) << 4));
          const uint4 uhi = lds128(row + (((4 * G + 2 + c) ^ sw) << 4));
          const __half2 *hl = reinterpret_cast<const __half2 *>(&ulo);
          const __half2 *hh = reinterpret_cast<const __half2 *>(&uhi);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float2 a = __half22float2(hl[j]);
            const float2 b = __half22float2(hh[j]);
            if (WHT) {
              xp[kGP * G + 8 * c + 2 * j] = f2_pack(a.x + b.x, a.x - b.x);
              xp[kGP * G + 8 * c + 2 * j + 1] = f2_pack(a.y + b.y, a.y - b.y);
            } else {
              xp[kGP * G + 8 * c + 2 * j] = f2_pack(a.x, b.x);
              xp[kGP * G + 8 * c + 2 * j + 1] = f2_pack(a.y, b.y);
            }
          }
        }
      }
    } else {
#pragma unroll
      for (int G = 0; G < 2; ++G) {
        uint32_t sw;
        const uint32_t row = stage_line<C>(stage, 2 * part + G, vl, sw);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 ulo = lds128(row + ((c ^ sw) << 4));
          const uint4 uhi = lds128(row + (((4 + c) ^ sw) << 4));
          const float a0 = __uint_as_float(ulo.x), a1 = __uint_as_float(ulo.y);
          const float a2 = __uint_as_float(ulo.z), a3 = __uint_as_float(ulo.w);
          const float b0 = __uint_as_float(uhi.x), b1 = __uint_as_float(uhi.y);
          const float b2 = __uint_as_float(uhi.z), b3 = __uint_as_float(uhi.w);
          if (WHT) {
            xp[kGP * G + 4 * c] = f2_pack(a0 + b0, a0 - b0);
            xp[kGP * G + 4 * c + 1] = f2_pack(a1 + b1, a1 - b1);
            xp[kGP * G + 4 * c + 2] = f2_pack(a2 + b2, a2 - b2);
            xp[kGP * G + 4 * c + 3] = f2_pack(a3 + b3, a3 - b3);
          } else {
            xp[kGP * G + 4 * c] = f2_pack(a0, b0);
            xp[kGP * G + 4 * c + 1] = f2_pack(a1, b1);
            xp[kGP * G + 4 * c + 2] = f2_pack(a2, b2);
            xp[kGP * G + 4 * c + 3] = f2_pack(a3, b3);
          }
        }
      }
    }
    __syncwarp();
    consumed = i + 1;
    // The warp is done reading stage s: refill it STAGES tiles ahead.
    if (lane == 0 && issued < n_mine) {
      fence_proxy_async_smem();
      issue(issued);
      ++issued;
    }

    // Step 1: norm.  With the WHT the pairs hold (a + b, a - b), whose
    // squares sum to twice a^2 + b^2.
    uint64_t acc2 = f2_pack(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < kPairs; ++k) acc2 = f2_fma(xp[k], xp[k], acc2);
    float ss_lo, ss_hi;
    f2_unpack(acc2, ss_lo, ss_hi);
    float ss = WHT ? 0.5f * (ss_lo + ss_hi) : ss_lo + ss_hi;
#pragma unroll
    for (int k = 1; k < P; k <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, k * VPW);
    const float norm = sqrtf(ss);

    // Step 2: the remaining WHT stages, then the folded block matrices.
    if (WHT) {
      wht_pairs_h4_h8(xp);
      // h = 32, arranged so that group 0 holds what this lane keeps in the
      // half exchange: (G0, G1) <- (G0 + sg G1, G0 - sg G1).
#pragma unroll
      for (int p = 0; p < kGP; ++p) {
        const uint64_t a = xp[p], b = xp[kGP + p];
        xp[p] = f2_fma(sig2, b, a);
        xp[kGP + p] = f2_fma(nsig2, b, a);
      }
      wht_cross_full<D>(xp, part);
#pragma unroll
      for (int p = 0; p < kGP; ++p) {
        const uint64_t r = __shfl_xor_sync(0xffffffffu, xp[kGP + p], KH * VPW);
        const uint64_t k = xp[p];
        xp[p] = f2_add(k, r);
        xp[kGP + p] = f2_sub(k, r);
      }
    }
    apply_group_matrices(xp, 0, mat_s + 512 * grp[0]);
    apply_group_matrices(xp, kGP, mat_s + 512 * grp[1]);

    // Steps 3-4: Lloyd-Max codes and bit-packing, one 32-code group at a time.
    const float big = search_scale(norm);
    float tb[C::NPOS];
#pragma unroll
    for (int j = 0; j < C::NPOS; ++j) tb[j] = -(args.tau[j] * norm) * big;
    const long long v = (t % args.tiles_per_head) * C::NV + warp * VPW + vl;
    if (v < args.n_vec) {
      const long long idx = static_cast<long long>(head) * args.out_head_stride + v;
      uint8_t *dst = args.codes + idx * C::PB;
#pragma unroll
      for (int G = 0; G < 2; ++G) {
        uint32_t w[C::GB / 4];
        quantize_group<BITS>(xp, kGP * G, tb, big, norm > 0.f ? 0u : 0x80000000u, w);
        uint8_t *gd = dst + grp[G] * C::GB;
        if constexpr (C::GB == 16) {
          *reinterpret_cast<uint4 *>(gd) = make_uint4(w[0], w[1], w[2], w[3]);
        } else if constexpr (C::GB == 8) {
          *reinterpret_cast<uint2 *>(gd) = make_uint2(w[0], w[1]);
        } else {
#pragma unroll
          for (int k = 0; k < C::GB / 4; ++k) reinterpret_cast<uint32_t *>(gd)[k] = w[k];
        }
      }
      if (part == 0) args.norms[idx] = __half_as_ushort(__float2half_rn(norm));
    }
  }
  if (failed && lane == 0) {
    // Let every copy still in flight land before the CTA may exit.
    for (int k = consumed; k < issued; ++k)
      if (!mbar_wait_bounded(&full_bar[k % C::STAGES], static_cast<uint32_t>(k / C::STAGES) & 1u)) break;
  }
}

#include "quant_tc.cuh"
#include "dequant_tc.cuh"

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

template <typename T, int D, int BITS, int RK>
__global__ void __launch_bounds__(kDequantThreads) dequantize_kernel(const DequantArgs args) {
  constexpr int P = Lanes<D>::P, VPW = Lanes<D>::VPW, KH = Lanes<D>::KH;
  constexpr int NV = kDequantThreads / P;
  constexpr int PB = D * BITS / 8, GB = 32 * BITS / 8;
  constexpr int L = 1 << BITS;
  __shared__ __align__(16) float mat[D * 4];
  __shared__ float cent[16];

  constexpr bool WHT = RK != kRotBlock;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int part = lane / VPW, vl = lane % VPW;
  const int vt = warp * VPW + vl;
  const bool hb = WHT && (part & KH) != 0;
  int grp[2] = {2 * part, 2 * part + 1};
  if (WHT) lane_groups<D>(part, grp);
  if (tid < L) cent[tid] = args.centroid[tid];
  const uint32_t mat_s = smem_u32(mat);

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
      build_block_matrices<D, RK, false>(args.params + static_cast<size_t>(head) * 2 * D, mat,
                                           tid, kDequantThreads);
      __syncthreads();
      cur_head = head;
    }
    const bool valid = v < args.n_vec;
    const long long idx = static_cast<long long>(head) * args.in_head_stride + (valid ? v : 0);
    const uint8_t *src = args.codes + idx * PB;

    // Centroids of this lane's two groups as pairs (e, e + 16).
    uint64_t xp[kPairs];
#pragma unroll
    for (int G = 0; G < 2; ++G) {
      uint32_t w[GB / 4];
      const uint8_t *gs = src + grp[G] * GB;
      if constexpr (GB == 16) {
        const uint4 u = *reinterpret_cast<const uint4 *>(gs);
        w[0] = u.x; w[1] = u.y; w[2] = u.z; w[3] = u.w;
      } else if constexpr (GB == 8) {
        const uint2 u = *reinterpret_cast<const uint2 *>(gs);
        w[0] = u.x; w[1] = u.y;
      } else {
#pragma unroll
        for (int k = 0; k < GB / 4; ++k) w[k] = reinterpret_cast<const uint32_t *>(gs)[k];
      }
#pragma unroll
      for (int p = 0; p < kGP; ++p)
        xp[kGP * G + p] = f2_pack(cent[unpack_code<BITS>(w, p)], cent[unpack_code<BITS>(w, p + 16)]);
    }
    const float s16 = __half2float(__ushort_as_half(args.norms[idx]));

    apply_group_matrices(xp, 0, mat_s + 512 * grp[0]);
    apply_group_matrices(xp, kGP, mat_s + 512 * grp[1]);
    if (WHT) {
      // Half exchange (h = d/2): keep G0 + G1, send G0 - G1.
#pragma unroll
      for (int p = 0; p < kGP; ++p) {
        const uint64_t a = xp[p], b = xp[kGP + p];
        const uint64_t dsend = f2_sub(a, b);
        xp[p] = f2_add(a, b);
        xp[kGP + p] = __shfl_xor_sync(0xffffffffu, dsend, KH * VPW);
      }
      wht_cross_full<D>(xp, part);
      // h = 32: afterwards G0 holds this lane's lower 32 elements and G1 its
      // upper 32, the latter negated on lanes with the exchange bit set.
#pragma unroll
      for (int p = 0; p < kGP; ++p) {
        const uint64_t a = xp[p], b = xp[kGP + p];
        xp[p] = f2_add(a, b);
        xp[kGP + p] = f2_sub(a, b);
      }
      wht_pairs_h4_h8(xp);
      wht_in_pair(xp);
    }
    const uint64_t sc0 = f2_pack(s16, s16);
    const float s1 = hb ? -s16 : s16;
    const uint64_t sc1 = f2_pack(s1, s1);
#pragma unroll
    for (int p = 0; p < kGP; ++p) {
      xp[p] = f2_mul(xp[p], sc0);
      xp[kGP + p] = f2_mul(xp[kGP + p], sc1);
    }

    if (valid) {
      T *dst = static_cast<T *>(args.out) + static_cast<long long>(head) * args.head_stride +
               v * args.vec_stride + part * kE;
#pragma unroll
      for (int G = 0; G < 2; ++G) {
        float lo[kGP], hi[kGP];
#pragma unroll
        for (int p = 0; p < kGP; ++p) f2_unpack(xp[kGP * G + p], lo[p], hi[p]);
        T *gd = dst + 32 * G;
        if constexpr (sizeof(T) == 2) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const float *e = c < 2 ? lo + 8 * c : hi + 8 * (c - 2);
            uint4 u;
            __half2 *h = reinterpret_cast<__half2 *>(&u);
#pragma unroll
            for (int j = 0; j < 4; ++j) h[j] = __floats2half2_rn(e[2 * j], e[2 * j + 1]);
            reinterpret_cast<uint4 *>(gd)[c] = u;
          }
        } else {
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const float *e = c < 4 ? lo + 4 * c : hi + 4 * (c - 4);
            reinterpret_cast<float4 *>(gd)[c] = make_float4(e[0], e[1], e[2], e[3]);
          }
        }
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

// d = 128 float16 input with the WHT: the tensor-core compressor
// (quant_tc.cuh), one CTA per SM.
template <int BITS, bool FULL>
int launch_quantize_tc(const void *x, int n_heads, long long n_vec, long long head_stride,
                       long long vec_stride, const float *params, uint8_t *codes, uint16_t *norms,
                       long long out_head_stride, cudaStream_t stream) {
  auto kernel = quantize_tc_kernel<BITS, FULL>;
  static bool configured = false;
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!configured) {
      cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kTqSmem);
      if (e != cudaSuccess)
        return set_error(ISOQ_ERR_CUDA, "quantize (tcgen05): cudaFuncSetAttribute: %s", cudaGetErrorString(e));
      configured = true;
    }
  }
  EncodeTiledFn encode = encode_tiled_fn();
  if (!encode) return set_error(ISOQ_ERR_CUDA, "quantize: cuTensorMapEncodeTiled unavailable");
  CUtensorMap map;
  const cuuint64_t gdim[3] = {static_cast<cuuint64_t>(kTqD), static_cast<cuuint64_t>(n_vec),
                              static_cast<cuuint64_t>(n_heads)};
  const long long hs = n_heads > 1 ? head_stride : vec_stride * n_vec;
  const cuuint64_t gstride[2] = {static_cast<cuuint64_t>(vec_stride * 2), static_cast<cuuint64_t>(hs * 2)};
  const cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(kTqRows), 1u};
  const cuuint32_t estride[3] = {1u, 1u, 1u};
  const CUresult r = encode(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void *>(x), gdim, gstride, box,
                            estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(ISOQ_ERR_UNSUPPORTED, "quantize: tensor map encode failed (%d)", (int)r);

  QuantArgs a;
  a.params = params;
  a.codes = codes;
  a.norms = norms;
  a.out_head_stride = out_head_stride;
  a.n_vec = n_vec;
  a.n_heads = n_heads;
  a.tiles_per_head = static_cast<int>((n_vec + kTqRows - 1) / kTqRows);
  a.total_tiles = static_cast<long long>(a.tiles_per_head) * n_heads;
  CodebookF32 cb;
  codebook_f32(kTqD, BITS, &cb);
  constexpr int L = 1 << BITS;
  for (int j = 0; j < 7; ++j) a.tau[j] = j < L / 2 - 1 ? cb.threshold[L / 2 + j] : 0.f;
  long long grid = num_sms();
  if (grid > a.total_tiles) grid = a.total_tiles;
  kernel<<<static_cast<unsigned>(grid), kTqThreads, kTqSmem, stream>>>(map, a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(ISOQ_ERR_CUDA, "quantize (tcgen05) launch: %s", cudaGetErrorString(e));
  return ISOQ_OK;
}

template <typename T, int D, int BITS, int RK>
int launch_quantize(const void *x, int n_heads, long long n_vec, long long head_stride,
                    long long vec_stride, const float *params, uint8_t *codes, uint16_t *norms,
                    long long out_head_stride, cudaStream_t stream) {
  if constexpr (std::is_same<T, __half>::value && D == 128 && RK != kRotBlock)
    return launch_quantize_tc<BITS, RK == kRotWhtFull>(x, n_heads, n_vec, head_stride, vec_stride, params,
                                                       codes, norms, out_head_stride, stream);
  using C = Cfg<T, D, BITS>;
  auto kernel = quantize_kernel<T, D, BITS, RK>;
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
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(C::BOX_ELEMS), static_cast<cuuint32_t>(C::VPW), 1u};
  const cuuint32_t estride[4] = {1u, 1u, 1u, 1u};
  const CUtensorMapDataType dt = C::ES == 2 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  CUresult r;
  if constexpr (C::CPB == 1) {
    r = encode(&map, dt, 3, const_cast<void *>(x), gdim, gstride, box, estride,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  } else {
    // Rows as [D / BOX_ELEMS chunks][BOX_ELEMS], the box CPB chunks x VPW rows.
    const cuuint64_t gdim4[4] = {static_cast<cuuint64_t>(C::BOX_ELEMS), static_cast<cuuint64_t>(D / C::BOX_ELEMS),
                                 static_cast<cuuint64_t>(n_vec), static_cast<cuuint64_t>(n_heads)};
    const cuuint64_t gstride4[3] = {128u, gstride[0], gstride[1]};
    const cuuint32_t box4[4] = {static_cast<cuuint32_t>(C::BOX_ELEMS), static_cast<cuuint32_t>(C::CPB),
                                static_cast<cuuint32_t>(C::VPW), 1u};
    r = encode(&map, dt, 4, const_cast<void *>(x), gdim4, gstride4, box4, estride,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  }
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

template <int BITS, bool FULL>
int launch_dequantize_tc(const uint8_t *codes, const uint16_t *norms, int n_heads, long long n_vec,
                         long long in_head_stride, const float *params, void *out, long long head_stride,
                         long long vec_stride, cudaStream_t stream) {
  auto kernel = dequantize_tc_kernel<BITS, FULL>;
  static bool configured = false;
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!configured) {
      cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kTdSmem);
      if (e != cudaSuccess)
        return set_error(ISOQ_ERR_CUDA, "dequantize (tcgen05): cudaFuncSetAttribute: %s", cudaGetErrorString(e));
      configured = true;
    }
  }
  EncodeTiledFn encode = encode_tiled_fn();
  if (!encode) return set_error(ISOQ_ERR_CUDA, "dequantize: cuTensorMapEncodeTiled unavailable");
  CUtensorMap map;
  const cuuint64_t gdim[3] = {static_cast<cuuint64_t>(kTdD), static_cast<cuuint64_t>(n_vec),
                              static_cast<cuuint64_t>(n_heads)};
  const long long hs = n_heads > 1 ? head_stride : vec_stride * n_vec;
  const cuuint64_t gstride[2] = {static_cast<cuuint64_t>(vec_stride * 2), static_cast<cuuint64_t>(hs * 2)};
  const cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(kTdRows), 1u};
  const cuuint32_t estride[3] = {1u, 1u, 1u};
  const CUresult r = encode(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, out, gdim, gstride, box, estride,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(ISOQ_ERR_UNSUPPORTED, "dequantize: tensor map encode failed (%d)", (int)r);

  DequantTcArgs a;
  a.codes = codes;
  a.norms = norms;
  a.params = params;
  a.in_head_stride = in_head_stride;
  a.n_vec = n_vec;
  a.tiles_per_head = static_cast<int>((n_vec + kTdRows - 1) / kTdRows);
  a.total_tiles = static_cast<long long>(a.tiles_per_head) * n_heads;
  // float16 hi and lo parts of the unit-variance centroids, as byte tables
  double cu[16];
  codebook_unit_f64(BITS, cu);
  uint8_t tb[4][8] = {};
  for (int j = 0; j < (1 << BITS); ++j) {
    const __half hi = __float2half_rn(static_cast<float>(cu[j]));
    const __half lo = __float2half_rn(static_cast<float>(cu[j] - static_cast<double>(__half2float(hi))));
    const uint16_t hb = __half_as_ushort(hi), lb = __half_as_ushort(lo);
    tb[0][j] = static_cast<uint8_t>(hb & 0xFF);
    tb[1][j] = static_cast<uint8_t>(hb >> 8);
    tb[2][j] = static_cast<uint8_t>(lb & 0xFF);
    tb[3][j] = static_cast<uint8_t>(lb >> 8);
  }
  uint32_t *dst[4] = {a.hi_lo, a.hi_hi, a.lo_lo, a.lo_hi};
  for (int k = 0; k < 4; ++k)
    for (int w = 0; w < 2; ++w)
      dst[k][w] = static_cast<uint32_t>(tb[k][4 * w]) | (static_cast<uint32_t>(tb[k][4 * w + 1]) << 8) |
                  (static_cast<uint32_t>(tb[k][4 * w + 2]) << 16) | (static_cast<uint32_t>(tb[k][4 * w + 3]) << 24);
  long long grid = num_sms();
  if (grid > a.total_tiles) grid = a.total_tiles;
  kernel<<<static_cast<unsigned>(grid), kTdThreads, kTdSmem, stream>>>(map, a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(ISOQ_ERR_CUDA, "dequantize (tcgen05) launch: %s", cudaGetErrorString(e));
  return ISOQ_OK;
}

template <typename T, int D, int BITS, int RK>
int launch_dequantize(const uint8_t *codes, const uint16_t *norms, int n_heads, long long n_vec,
                      long long in_head_stride, const float *params, void *out,
                      long long head_stride, long long vec_stride, cudaStream_t stream) {
  if constexpr (std::is_same<T, __half>::value && D == 128 && (BITS == 2 || BITS == 3) && RK != kRotBlock)
    return launch_dequantize_tc<BITS, RK == kRotWhtFull>(codes, norms, n_heads, n_vec, in_head_stride, params,
                                                         out, head_stride, vec_stride, stream);
  constexpr int NV = kDequantThreads / Lanes<D>::P;
  auto kernel = dequantize_kernel<T, D, BITS, RK>;
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
template <template <typename, int, int, int> class F, typename... A>
int dispatch(int dtype, int d, int bits, int variant, A... args) {
  const int rk = variant == ISOQ_FAST ? kRotWhtFast
               : (variant == ISOQ_BLOCK_SO4 || variant == ISOQ_SO3) ? kRotBlock
                                                                      : kRotWhtFull;
#define ISOQ_CASE_V(T, D, B)                                                    \
  return rk == kRotWhtFull ? F<T, D, B, kRotWhtFull>::run(args...)             \
       : rk == kRotWhtFast ? F<T, D, B, kRotWhtFast>::run(args...)             \
                           : F<T, D, B, kRotBlock>::run(args...)
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

template <typename T, int D, int B, int RK>
struct QuantizeRunner {
  static int run(const void *x, int n_heads, long long n_vec, long long hs, long long vs,
                 const float *params, uint8_t *codes, uint16_t *norms, long long ohs,
                 cudaStream_t st) {
    return launch_quantize<T, D, B, RK>(x, n_heads, n_vec, hs, vs, params, codes, norms, ohs, st);
  }
};

template <typename T, int D, int B, int RK>
struct DequantizeRunner {
  static int run(const uint8_t *codes, const uint16_t *norms, int n_heads, long long n_vec,
                 long long ihs, const float *params, void *out, long long hs, long long vs,
                 cudaStream_t st) {
    return launch_dequantize<T, D, B, RK>(codes, norms, n_heads, n_vec, ihs, params, out, hs, vs, st);
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
