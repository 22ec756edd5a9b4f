// Integer tensor-core split kernel of the compressed-space decode: float16
// queries, 3-bit codes, d in {128, 256}, up to 8 query heads per KV head.
// Included by isoq_decode.cu inside namespace isoq::decode.
//
// The work per token is RotaryQuant Table 2 kernels A-C on the packed codes:
// z_j = s^K_j <q~, c[K_j]> scale, online softmax, acc += p_j s^V_j c[V_j], all
// in the rotated domain, with every code turned into an int8 tensor-core
// operand by a register lookup.
//
// Exact integer centroids.  The unit-variance centroids are scaled by a
// host-chosen S (about 6,324) so that every C_k = round(S c_k) is within a few
// hundredths of S c_k; |C_k| <= 16319 is split as C = 128 Ch + Cl with
// Ch in [-128, 127] and Cl in [-64, 63].  Each part is an int8 table of 8
// entries held in two registers, so one prmt turns four codes (a 4-nibble
// selector) into a full int8 MMA register: half a prmt per code per part,
// against one prmt per code for a float16 operand, whose two bytes need a
// lookup each plus an interleave.
//
// QK (kernel A): mma.sync m16n8k32 s8 x s8 -> s32.  A = Ch or Cl of 16 tokens
// x 32 dims; B = the rotated query in 22-bit fixed point,
// Q = 2^14 Qh + 2^7 Qm + Ql (per-head step max|q~| / 2088000), the three
// parts in separate columns (or N tiles).  Each part's two products give
// sum C Q_part exactly in int32; only their conversion to float32 and the
// final 2^14 / 2^7 weighting round.
//
// Softmax (kernel B): float32, log2 domain, on the accumulator fragments.
//
// PV (kernel C): mma.sync m16n8k32 s8 x u8 -> s32 with M = 16 dim quads,
// K = 8 tokens x 4 parities, N = 2 heads x 4 parities:
//   D[u][(h, r)] = sum_(j, r') A[u][(j, r')] B[(j, r')][(h, r)],
//   A[u][(j, r')] = V~[j][4u + r'],   B[(j, r')][(h, r)] = W[j][h] [r' = r],
// so every A register is four consecutive codes of one token, exactly what
// one prmt lookup produces.  W = p s^V is block-scaled per 16-token slab and
// head to 16 bits, W = 256 Wh + Wl (u8 parts); C W = 2^15 Ch Wh +
// 2^7 (Ch Wl + 2 Cl Wh) + Cl Wl, of which the last term (below 2^-15 of one
// token's largest contribution) is dropped.  W is fixed-point against the
// largest p s^V of its 32-token block and head, W_q = rint(p s^V 64000 /
// max_block(p s^V)) with p = 2^(x - m_ref): every block keeps 16 bits
// relative to its own largest weight, so a block of small weights next to
// one dominant token (an attention sink) loses nothing to the dominant
// token's scale.  The int32 sums of each 16-token half are converted once
// and added into float32 accumulators with the block's scale; m_ref moves
// (and l and the accumulators are rescaled) only when a block's maximum
// score passes m_ref + 1, which after the first block is rare.  The pair
// (m_ref, l) it leaves is a valid partial state: l and acc are both relative
// to 2^m_ref.
//
// Fragment orders.  A fixed permutation of the rotated coordinates cancels in
// q~.k~ and is undone when the accumulator is written out:
//   QK: per 16-token tile, lane (g, t) owns tokens g, g+8 and dims
//       [t d/4, (t+1) d/4) (one or two 32-code groups); k-step kk uses quads
//       2kk, 2kk+1 of that range.
//   PV: per 16-token half, lane (g, t) owns tokens t, t+4, t+8, t+12 and the
//       32-code group g (d = 256) or half of group g/2 (d = 128); M-block mb
//       maps row g to the lane's quad 2mb and row g+8 to quad 2mb+1.
//
// Staging: the CTA streams rounds of 128 tokens (warp w takes the round's
// 32-token block w) through a 2-deep ring of CTA-local bulk copies with
// mbarrier completion: four copies per round (packed K and V rows, float16
// norms), issued by the last warp to finish with the stage, so that the
// copies' operands are computed once per round instead of once per block.
//
// Selectors.  A prmt selector is four 3-bit codes in the low nibbles of its
// low 16 bits.  The 32-code group layout (codes in 4-bit fields, codes
// 24..31 spread over the spare bits) needs a mask per word and a shift per
// high half on the integer pipe; the lookups themselves (half a prmt per code
// per part) are the rest of that pipe's work, which bounds the kernel.

constexpr int kI8Warps = 4;
constexpr int kI8Threads = 32 * kI8Warps;
constexpr int kBlk = 32;                 // tokens per ring stage (two 16-token MMA tiles)
constexpr int kI8Stages = 2;             // per-warp ring depth
constexpr int kCentroidIntMax = 16319;   // |C_k| bound that keeps Ch, 2 Cl in int8
constexpr int kQueryIntMax = 2088000;    // |Q| bound that keeps Qh, Qm, Ql in int8
constexpr float kWMax = 64000.f;         // W_q = rint(p s^V kWMax / max_block(p s^V)) < 2^16

template <int D, int GP>
struct I8Cfg {
  static constexpr int PB = D * 3 / 8;                      // packed bytes per token
  static constexpr int BLK_CODES = kBlk * PB;
  static constexpr int BLK_NORMS = kBlk * 2;
  static constexpr int STAGE_BYTES = 2 * BLK_CODES + 2 * BLK_NORMS;   // one warp's block
  static constexpr int RING_BYTES = kI8Stages * STAGE_BYTES;            // per warp
  // A round stage: K codes, V codes, K norms, V norms of the four warps' blocks.
  static constexpr int ROUND_BYTES = kI8Warps * STAGE_BYTES;
  static constexpr int R_V = kI8Warps * BLK_CODES;
  static constexpr int R_NK = 2 * kI8Warps * BLK_CODES;
  static constexpr int R_NV = R_NK + kI8Warps * BLK_NORMS;
  static constexpr int KK = D / 32;                         // QK k-steps (8 codes per lane-row each)
  static constexpr int GRP_QK = D / 128;                    // 32-code groups per QK lane segment
  static constexpr int MB = D / 64;                         // PV M-blocks (64 dims each)
  static constexpr int NQ = GP <= 2 ? 1 : (GP == 4 ? 2 : 3);  // QK N tiles (3 parts x GP columns)
  static constexpr int NV = (GP + 1) / 2;                   // PV N tiles (2 heads each)
  static constexpr int SCRATCH_FLOATS = GP * D;             // the sequential warp merge
  static constexpr int MERGE_FLOATS = kI8Warps * GP * D;    // the sliced warp merge, over the rings
  static constexpr int QPREP_WORDS = 3 * KK * 2 * 32 + 8;   // per (b, kvh), see prep_i8_kernel
  static_assert(MERGE_FLOATS * 4 <= kI8Warps * RING_BYTES, "merge slices fit the rings");
  // GP <= 2: the block's scores go through shared memory to one token per
  // lane (see the softmax), kBlk tokens x 2 heads per warp.
  static constexpr bool COMPACT = GP <= 2;
  // GP = 2: the three query parts' sums of each score go there separately.
  static constexpr int ZX_FLOATS = COMPACT ? kI8Warps * kBlk * 2 * (GP == 2 ? 3 : 1) : 0;
  static constexpr int SMEM = kI8Warps * RING_BYTES + SCRATCH_FLOATS * 4 + ZX_FLOATS * 4 +
                              2 * kI8Warps * 8 * 4 + kI8Warps * kI8Stages * 8 + 128;
  static constexpr int MIN_BLOCKS = (D == 256 && GP == 8) ? 2 : ((D == 256 && GP == 4) || GP == 8 ? 3 : 4);
};

// int8 tables of the centroid parts, four entries per register: kh/kl =
// (Ch, Cl) for the K side, vh/vl = (Ch, 2 Cl) for the V side.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// Shared-memory loads by explicit shared-window address (no generic LD).
__device__ __forceinline__ uint32_t lds32(const unsigned char *p) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)));
  return v;
}

__device__ __forceinline__ uint2 lds64(const unsigned char *p) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(smem_u32(p)));
  return v;
}

__device__ __forceinline__ float lds_half(const unsigned char *p) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(smem_u32(p)));
  return __half2float(__ushort_as_half(v));
}

struct I8Lut {
  uint32_t kh0, kh1, kl0, kl1, vh0, vh1, vl0, vl1;
  uint32_t neg1, one;     // -1 and 1, opaque to the compiler (see group_sel8_im)
};

__device__ __forceinline__ float ex2f(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// c += A B (s8 x s8), and the same with a zero accumulator.
__device__ __forceinline__ void mma_s8s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_s8s8_z(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                           uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{0,0,0,0};"
      : "=r"(c[0]), "=r"(c[1]), "=r"(c[2]), "=r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// c += A B (s8 x u8), and the same with a zero accumulator.
__device__ __forceinline__ void mma_s8u8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_s8u8_z(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                           uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{0,0,0,0};"
      : "=r"(c[0]), "=r"(c[1]), "=r"(c[2]), "=r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// prmt selectors of the eight quads of one 32-code group (three words in the
// layout of common.cuh); quad q = codes 4q..4q+3, in the low 16 bits of s[q].
__device__ __forceinline__ void group_sel8(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t (&s)[8]) {
  const uint32_t m0 = w0 & 0x77777777u, m1 = w1 & 0x77777777u, m2 = w2 & 0x77777777u;
  // The spare bits x_r = w_r - m_r (bit 4j+3 = bit r of code 24+j) gathered
  // into nibbles: the three shifted planes are disjoint, so their sum (integer
  // adds, which the compiler may place on the FMA pipe) is their union.
  const uint32_t x0 = w0 - m0, x1 = w1 - m1, x2 = w2 - m2;
  const uint32_t sum = (x0 >> 2) + (x1 >> 1) + x2;   // code 24+j at bits 4j+1 .. 4j+3
  s[0] = m0;
  s[1] = m0 >> 16;
  s[2] = m1;
  s[3] = m1 >> 16;
  s[4] = m2;
  s[5] = m2 >> 16;
  s[6] = sum >> 1;
  s[7] = sum >> 17;
}

__device__ __forceinline__ uint32_t imad_u32(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;
  asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}

// group_sel8 with the spare-bit planes and their sum formed by multiply-adds
// whose factors (-1, 1) arrive as kernel parameters: the compiler cannot
// turn them into logic ops, so that work moves from the integer (ALU) pipe,
// which bounds the decode, to the separate multiply-add pipe.
__device__ __forceinline__ void group_sel8_im(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t (&s)[8],
                                              uint32_t neg1, uint32_t one) {
  const uint32_t m0 = w0 & 0x77777777u, m1 = w1 & 0x77777777u, m2 = w2 & 0x77777777u;
  const uint32_t x0 = imad_u32(m0, neg1, w0), x1 = imad_u32(m1, neg1, w1), x2 = imad_u32(m2, neg1, w2);
  const uint32_t sum = imad_u32(x0 >> 2, one, imad_u32(x1 >> 1, one, x2));
  s[0] = m0;
  s[1] = m0 >> 16;
  s[2] = m1;
  s[3] = m1 >> 16;
  s[4] = m2;
  s[5] = m2 >> 16;
  s[6] = sum >> 1;
  s[7] = sum >> 17;
}

// Packs the low 16 bits of two words into one (a in bits 0-15, b in 16-31).
__device__ __forceinline__ uint32_t pack_lo16(uint32_t a, uint32_t b) { return prmt(a, b, 0x5410u); }

// Four int8 values into one register, byte i = v[i].
__device__ __forceinline__ uint32_t pack_s8x4(int v0, int v1, int v2, int v3) {
  return (static_cast<uint32_t>(v0) & 0xFFu) | ((static_cast<uint32_t>(v1) & 0xFFu) << 8) |
         ((static_cast<uint32_t>(v2) & 0xFFu) << 16) | ((static_cast<uint32_t>(v3) & 0xFFu) << 24);
}


// Query preparation, one CTA per (b, kvh): rotate the G queries once,
// q~ = R_K q, and write for every lane of the split kernel the B-fragment
// words of the fixed-point query Q = rint(q~ / qinv) = 2^14 Qh + 2^7 Qm + Ql
// (qinv = max|q~_h| / kQueryIntMax per head), then the per-head score factors
// qinv_h * score_unit (0 for padded heads).  Word ((nq KK + kk) 2 + half) 32
// + lane holds tile nq, k-step kk, half `half` of lane (g, t): column g is
// (head, part) with part p of head h in tile 0, column p GP + h (GP <= 2);
// tile 0, column 4p + h for p < 2 and tile 1, column h for p = 2 (GP = 4);
// tile p, column h (GP = 8); the four int8 values are the dims of quad
// 2 (kk mod 4) + half of lane t's 32-code group (D = 128: group t; D = 256:
// group 2t + kk / 4).
//
// One warp per query head h (GP warps), lane j holding dims E j .. E j + E - 1
// (E = d / 32) in registers: the Walsh-Hadamard stages h < E inside the
// lane, the others by shuffles with lane j ^ (h / E), in the same stage
// order and with the same sums as the shared-memory rotation (so q~ is the
// same to the bit), then 1/sqrt(d) and the block map on the lane's own 4-dim
// blocks.  The part words go through shared memory once to their fragment
// positions.
template <int D, bool FULL, int GP>
__global__ void __launch_bounds__(32 * GP) prep_i8_kernel(const SplitArgs a, float score_unit) {
  using C = I8Cfg<D, GP>;
  constexpr int E = D / 32, NQUAD = D / 4;
  __shared__ uint32_t pw[3][GP][NQUAD];   // part p of head h, dims 4 quad .. + 3
  __shared__ float qinv_s[8];
  const int kvh = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x, h = tid >> 5, lane = tid & 31;
  const int G = a.group;
  pdl_launch_dependents();   // the split kernel may start its staging now

  float x[E];
  if (h < G) {
    const __half *qp = static_cast<const __half *>(a.q) + (static_cast<long long>(b) * a.hq + kvh * G + h) * D + E * lane;
#pragma unroll
    for (int e = 0; e < E; e += 2) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(qp + e));
      x[e] = f.x;
      x[e + 1] = f.y;
    }
  } else {
#pragma unroll
    for (int e = 0; e < E; ++e) x[e] = 0.f;
  }
  // Walsh-Hadamard stages (a, b) -> (a + b, a - b), h = 1, 2, ..., d/2.
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
  const float inv = rsqrtf(static_cast<float>(D));
  const float *prm = a.params_k + static_cast<size_t>(kvh) * 2 * D;
  float mx = 0.f;
#pragma unroll
  for (int u = 0; u < E / 4; ++u) {
    const int bi = (E / 4) * lane + u;
    const Quat v{x[4 * u] * inv, x[4 * u + 1] * inv, x[4 * u + 2] * inv, x[4 * u + 3] * inv};
    const Quat r = block_forward(load_quat(prm + 8 * bi), load_quat(prm + 8 * bi + 4), v, FULL);
    x[4 * u] = r.w;
    x[4 * u + 1] = r.x;
    x[4 * u + 2] = r.y;
    x[4 * u + 3] = r.z;
  }
  if (h < G) {
#pragma unroll
    for (int e = 0; e < E; ++e) mx = fmaxf(mx, fabsf(x[e]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  const float qi = mx / static_cast<float>(kQueryIntMax);
  const float qsc = qi > 0.f ? 1.f / qi : 0.f;
  if (lane == 0) qinv_s[h] = qi;
  if (h == 0 && lane >= GP && lane < 8) qinv_s[lane] = 0.f;
#pragma unroll
  for (int u = 0; u < E / 4; ++u) {
    int v[3][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      int q = h < G ? __float2int_rn(x[4 * u + i] * qsc) : 0;
      q = q > kQueryIntMax ? kQueryIntMax : (q < -kQueryIntMax ? -kQueryIntMax : q);
      const int r1 = (q + 64) >> 7, ql = q - 128 * r1;     // arithmetic shifts: floor
      const int r2 = (r1 + 64) >> 7, qm = r1 - 128 * r2;
      v[0][i] = r2;
      v[1][i] = qm;
      v[2][i] = ql;
    }
#pragma unroll
    for (int p = 0; p < 3; ++p) pw[p][h][(E / 4) * lane + u] = pack_s8x4(v[p][0], v[p][1], v[p][2], v[p][3]);
  }
  __syncthreads();

  // Word ((nq KK + kk) 2 + half) 32 + lane of the B fragments (see above).
  uint32_t *out = a.ws_qprep + (static_cast<long long>(b) * a.hkv + kvh) * C::QPREP_WORDS;
  constexpr int NWORDS = C::NQ * C::KK * 2 * 32;
  for (int idx = tid; idx < NWORDS; idx += 32 * GP) {
    const int ln = idx & 31, half = (idx >> 5) & 1, kk = (idx >> 6) % C::KK, nq = (idx >> 6) / C::KK;
    const int g = ln >> 2, t = ln & 3;
    int head, part;
    if constexpr (GP <= 2) {
      part = g / GP;
      head = g % GP;
    } else if constexpr (GP == 4) {
      part = nq == 0 ? (g >> 2) : (g < 4 ? 2 : 3);
      head = g & 3;
    } else {
      part = nq;
      head = g;
    }
    const bool live = part < 3 && head < G;
    const int grp = (D == 256 ? 2 * t : t) + kk / 4;
    out[idx] = live ? pw[part][head][8 * grp + 2 * (kk & 3) + half] : 0u;
  }
  if (tid < 8) out[3 * C::KK * 2 * 32 + tid] = __float_as_uint(tid < G ? qinv_s[tid] * score_unit : 0.f);
}

// GP: query heads per KV head rounded up to 1, 2, 4 or 8 (padded heads carry
// zero queries and zero weights).  SLICES selects the warp merge: every warp
// into its own slice and one barrier (for short chunks, where the merge is a
// visible share of a CTA's time: batch-1 32K-token decode 27.0 -> 22.9 us),
// or one warp after the other into one buffer, a barrier each (for long
// chunks, where the sliced form measured 0.7 % slower: it changes how the
// main loop compiles).
template <int D, bool FULL, int GP, bool SLICES>
__global__ void __launch_bounds__(kI8Threads, I8Cfg<D, GP>::MIN_BLOCKS)
    split_i8_kernel(const SplitArgs a, const I8Lut lut, float out_scale) {
  using C = I8Cfg<D, GP>;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~static_cast<uintptr_t>(127));
  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.group;

  unsigned char *ring = smem;                       // [stage][round]
  float *scratch = reinterpret_cast<float *>(smem + kI8Warps * C::RING_BYTES);
  float *zx = scratch + C::SCRATCH_FLOATS;          // [warps][kBlk * 2] (GP <= 2)
  float *wm = zx + C::ZX_FLOATS;                    // [warps][8]
  float *wl = wm + kI8Warps * 8;                    // [warps][8]
  uint64_t *full_bar = reinterpret_cast<uint64_t *>(wl + kI8Warps * 8);   // [stage]
  uint32_t *done_cnt = reinterpret_cast<uint32_t *>(full_bar + kI8Stages);   // [stage]
  uint32_t *rounds_issued = done_cnt + kI8Stages;

  int tlen = a.seq_lens[b];
  tlen = tlen < 0 ? 0 : (tlen > a.tmax ? static_cast<int>(a.tmax) : tlen);
  const long long t0 = static_cast<long long>(split) * a.chunk;
  long long t1 = t0 + a.chunk;
  if (t1 > tlen) t1 = tlen;
  const int n_tok = t1 > t0 ? static_cast<int>(t1 - t0) : 0;
  const int n_blk = (n_tok + kBlk - 1) / kBlk;
  const int n_mine = n_blk > warp ? (n_blk - warp + kI8Warps - 1) / kI8Warps : 0;

  const long long pair = static_cast<long long>(b) * a.hkv + kvh;
  const uint8_t *kb = a.packed_k + pair * a.tmax * C::PB;
  const uint8_t *vb = a.packed_v + pair * a.tmax * C::PB;
  const uint16_t *nkb = a.norms_k + pair * a.tmax;
  const uint16_t *nvb = a.norms_v + pair * a.tmax;

  // One thread issues the copies of round r (tokens 128 r .. 128 r + 127 of
  // the chunk) into stage r % kI8Stages.
  const int n_rounds = (n_blk + kI8Warps - 1) / kI8Warps;
  auto issue = [&](int r) {
    const long long t = t0 + static_cast<long long>(r) * (kI8Warps * kBlk);
    int n = n_tok - r * (kI8Warps * kBlk);
    if (n > kI8Warps * kBlk) n = kI8Warps * kBlk;
    const int n8 = (n + 7) & ~7;
    const int s = r % kI8Stages;
    unsigned char *st = ring + s * C::ROUND_BYTES;
    mbar_arrive_expect_tx(&full_bar[s], 2u * n * C::PB + 4u * n8);
    bulk_load(st, kb + t * C::PB, n * C::PB, &full_bar[s]);
    bulk_load(st + C::R_V, vb + t * C::PB, n * C::PB, &full_bar[s]);
    bulk_load(st + C::R_NK, nkb + t, 2 * n8, &full_bar[s]);
    bulk_load(st + C::R_NV, nvb + t, 2 * n8, &full_bar[s]);
    *rounds_issued = static_cast<uint32_t>(r + 1);
  };
  if (tid == 0) {
    for (int s = 0; s < kI8Stages; ++s) {
      mbar_init(&full_bar[s], 1);
      done_cnt[s] = 0u;
    }
    *rounds_issued = 0u;
    mbar_fence_init();
    for (int r = 0; r < kI8Stages && r < n_rounds; ++r) issue(r);
  }
  __syncthreads();   // every warp waits on the barriers thread 0 initialised

  const int g = lane >> 2, t = lane & 3;

  // B fragments of the fixed-point query and the per-head score factors,
  // prepared once per (b, kvh) by prep_i8_kernel (launched just before this
  // kernel with programmatic dependent launch: wait for it here, after the
  // staging above has started).
  pdl_launch_dependents();
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const uint32_t *qp = a.ws_qprep + pair * C::QPREP_WORDS;
  uint32_t qb[C::NQ][C::KK][2];
#pragma unroll
  for (int nq = 0; nq < C::NQ; ++nq)
#pragma unroll
    for (int kk = 0; kk < C::KK; ++kk)
#pragma unroll
      for (int half = 0; half < 2; ++half) qb[nq][kk][half] = qp[((nq * C::KK + kk) * 2 + half) * 32 + lane];
  // score factors of the lane's two heads: 2t, 2t + 1, or with the compact
  // softmax (GP <= 2) heads 0, 1 in every lane; 0 for padded heads
  const float qk0 = __uint_as_float(qp[3 * C::KK * 2 * 32 + (C::COMPACT ? 0 : 2 * t)]);
  const float qk1 = __uint_as_float(qp[3 * C::KK * 2 * 32 + (C::COMPACT ? 1 : 2 * t + 1)]);

  // prmt selectors that move byte k of a packed (W_a, W_b) word to byte g&3
  // of a PV B register (zeros elsewhere): lo / hi byte of head parity g>>2.
  const uint32_t r4 = 4u * static_cast<uint32_t>(g & 3);
  const uint32_t hpb = 2u * static_cast<uint32_t>(g >> 2);
  const uint32_t sel_lo = (0x4444u & ~(0xFu << r4)) | (hpb << r4);
  const uint32_t sel_hi = (0x4444u & ~(0xFu << r4)) | ((hpb + 1u) << r4);

  // PV accumulators sum p s^V C (float32, whole chunk, relative to
  // 2^m_ref) in the PV layout: head 2nv + (t >> 1).
  float acc[C::NV][C::MB][4];
#pragma unroll
  for (int nvt = 0; nvt < C::NV; ++nvt)
#pragma unroll
    for (int mb = 0; mb < C::MB; ++mb)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[nvt][mb][e] = 0.f;
  // Softmax state in the QK layout (heads 2t, 2t+1; log2 domain): reference
  // maximum and sum.
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

  bool failed = false;
  for (int i = 0; i < n_mine; ++i) {
    const int s = i % kI8Stages;
    if (!mbar_wait_bounded(&full_bar[s], (i / kI8Stages) & 1)) {
      atomicOr(&g_decode_error, kErrWaitTimeout);
      failed = true;
      break;
    }
    int nvalid = n_tok - (warp + kI8Warps * i) * kBlk;
    nvalid = nvalid > kBlk ? kBlk : nvalid;
    const unsigned char *st = ring + s * C::ROUND_BYTES;
    const unsigned char *kc = st + warp * C::BLK_CODES;
    const unsigned char *vc = st + C::R_V + warp * C::BLK_CODES;
    const unsigned char *nk = st + C::R_NK + warp * C::BLK_NORMS;   // float16 [32]
    const unsigned char *nv = st + C::R_NV + warp * C::BLK_NORMS;

    float *zw = zx + warp * (C::ZX_FLOATS / kI8Warps);   // the warp's score buffer (GP <= 2)
    // ---- QK: exact int32 sums of C * Q_part over the lane's dims, per tile ----
    // sc[T][e]: token 16T + g + 8 (e >> 1), head 2t + (e & 1).
    float sc[2][4];
#pragma unroll
    for (int T = 0; T < 2; ++T) {
      int d1[C::NQ][4], d2[C::NQ][4];
      constexpr int NW = D * 3 / 128;   // words per token segment (6 or 3)
      uint32_t wg[NW], wg8[NW];
      const unsigned char *rg = kc + (16 * T + g) * C::PB + t * (NW * 4);
      const unsigned char *rg8 = rg + 8 * C::PB;
      if constexpr (NW % 2 == 0) {
#pragma unroll
        for (int k = 0; k < NW / 2; ++k) {
          const uint2 x = lds64(rg + 8 * k), y = lds64(rg8 + 8 * k);
          wg[2 * k] = x.x;
          wg[2 * k + 1] = x.y;
          wg8[2 * k] = y.x;
          wg8[2 * k + 1] = y.y;
        }
      } else {
#pragma unroll
        for (int k = 0; k < NW; ++k) {
          wg[k] = lds32(rg + 4 * k);
          wg8[k] = lds32(rg8 + 4 * k);
        }
      }
#pragma unroll
      for (int gq = 0; gq < C::GRP_QK; ++gq) {
        uint32_t sa[8], sb[8];
        group_sel8_im(wg[3 * gq], wg[3 * gq + 1], wg[3 * gq + 2], sa, lut.neg1, lut.one);
        group_sel8_im(wg8[3 * gq], wg8[3 * gq + 1], wg8[3 * gq + 2], sb, lut.neg1, lut.one);
#pragma unroll
        for (int kq = 0; kq < 4; ++kq) {
          const int kk = 4 * gq + kq;
          const uint32_t sa0 = sa[2 * kq], sa1 = sa[2 * kq + 1], sb0 = sb[2 * kq], sb1 = sb[2 * kq + 1];
          {
            const uint32_t a0 = prmt(lut.kh0, lut.kh1, sa0), a1 = prmt(lut.kh0, lut.kh1, sb0);
            const uint32_t a2 = prmt(lut.kh0, lut.kh1, sa1), a3 = prmt(lut.kh0, lut.kh1, sb1);
#pragma unroll
            for (int nq = 0; nq < C::NQ; ++nq) {
              if (kk == 0)
                mma_s8s8_z(d1[nq], a0, a1, a2, a3, qb[nq][kk][0], qb[nq][kk][1]);
              else
                mma_s8s8(d1[nq], a0, a1, a2, a3, qb[nq][kk][0], qb[nq][kk][1]);
            }
          }
          {
            const uint32_t a0 = prmt(lut.kl0, lut.kl1, sa0), a1 = prmt(lut.kl0, lut.kl1, sb0);
            const uint32_t a2 = prmt(lut.kl0, lut.kl1, sa1), a3 = prmt(lut.kl0, lut.kl1, sb1);
#pragma unroll
            for (int nq = 0; nq < C::NQ; ++nq) {
              if (kk == 0)
                mma_s8s8_z(d2[nq], a0, a1, a2, a3, qb[nq][kk][0], qb[nq][kk][1]);
              else
                mma_s8s8(d2[nq], a0, a1, a2, a3, qb[nq][kk][0], qb[nq][kk][1]);
            }
          }
        }
      }
      // sum C Q = 2^14 X_h + 2^7 X_m + X_l with X_p = 128 (sum Ch Q_p) + sum Cl Q_p;
      // c0 = (g, 2t), c1 = (g, 2t+1), c2 = (g+8, 2t), c3 = (g+8, 2t+1).
      float f[C::NQ][4];
#pragma unroll
      for (int nq = 0; nq < C::NQ; ++nq)
#pragma unroll
        for (int e = 0; e < 4; ++e) f[nq][e] = static_cast<float>(128 * d1[nq][e] + d2[nq][e]);
      if constexpr (GP == 1) {
        // columns (hi, mid, lo): hi and mid in lane t = 0, lo in lane t = 1
        const float lo0 = __shfl_xor_sync(0xffffffffu, f[0][0], 1);
        const float lo2 = __shfl_xor_sync(0xffffffffu, f[0][2], 1);
        sc[T][0] = fmaf(f[0][0], 16384.f, fmaf(f[0][1], 128.f, lo0));
        sc[T][2] = fmaf(f[0][2], 16384.f, fmaf(f[0][3], 128.f, lo2));
        sc[T][1] = sc[T][3] = 0.f;
      } else if constexpr (GP == 2) {
        // lane t = 0: hi, t = 1: mid, t = 2: lo of heads 0, 1; each part goes
        // to its own region of the warp's score buffer (slots as below) and
        // the lane that takes the token in the softmax weights them.
        if (t < 3)
          *reinterpret_cast<float4 *>(zw + 64 * t + 8 * g + 4 * T) = make_float4(f[0][0], f[0][1], f[0][2], f[0][3]);
      } else if constexpr (GP == 4) {
        // tile 0: lanes t = 0, 1 hi, t = 2, 3 mid; tile 1: lanes t = 0, 1 lo
#pragma unroll
        for (int e = 0; e < 4; ++e)
          sc[T][e] = fmaf(f[0][e], 16384.f, fmaf(__shfl_xor_sync(0xffffffffu, f[0][e], 2), 128.f, f[1][e]));
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) sc[T][e] = fmaf(f[0][e], 16384.f, fmaf(f[1][e], 128.f, f[2][e]));
      }
    }

    // ---- softmax bookkeeping (log2 domain) ----
    // u[T][hh]: (W head a, W head b) packed as two 16-bit fields; dinv: one
    // unit of 256 E1 + E2 in the PV layout (heads 2nv + (t >> 1)).
    uint32_t u[2][2];
    float dinv[C::NV];
    if constexpr (C::COMPACT) {
      // One token per lane: the scores (GP = 1: combined in the t = 0 lanes;
      // GP = 2: the three parts, stored above) go through shared memory so
      // that lane L holds token L's scores of heads 0, 1, and every softmax
      // step below runs on 2 values per lane instead of 8 (of which 6 belong
      // to padded heads at GP <= 2).  Slot of token 16 T + 8 hh + g, head h:
      // g 8 + T 4 + hh 2 + h (GP = 2: in the region of each part).
      if constexpr (GP == 1) {
        if (t == 0) {
          *reinterpret_cast<float4 *>(zw + 8 * g) = make_float4(sc[0][0], sc[0][1], sc[0][2], sc[0][3]);
          *reinterpret_cast<float4 *>(zw + 8 * g + 4) = make_float4(sc[1][0], sc[1][1], sc[1][2], sc[1][3]);
        }
      }
      __syncwarp();
      const int zs = 8 * (lane & 7) + 4 * (lane >> 4) + 2 * ((lane >> 3) & 1);
      float z0, z1;
      if constexpr (GP == 2) {
        const float2 zh = *reinterpret_cast<const float2 *>(zw + zs);
        const float2 zm = *reinterpret_cast<const float2 *>(zw + 64 + zs);
        const float2 zl = *reinterpret_cast<const float2 *>(zw + 128 + zs);
        z0 = fmaf(zh.x, 16384.f, fmaf(zm.x, 128.f, zl.x));
        z1 = fmaf(zh.y, 16384.f, fmaf(zm.y, 128.f, zl.y));
      } else {
        const float2 z = *reinterpret_cast<const float2 *>(zw + zs);
        z0 = z.x;
        z1 = z.y;
      }
      const float sk = lds_half(nk + 2 * lane);
      float svl = lds_half(nv + 2 * lane);
      float x0 = z0 * sk * qk0, x1 = z1 * sk * qk1;
      if (nvalid < kBlk && lane >= nvalid) {   // the chunk's partial last block
        x0 = x1 = -INFINITY;
        svl = 0.f;
      }
      // Move the reference maximum only when a score passes m_ref + 1.
      if (__any_sync(0xffffffffu, x0 > m0 + 1.f || x1 > m1 + 1.f)) {
        float mx0 = x0, mx1 = x1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
          mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
        }
        const float mn0 = mx0 > m0 + 1.f ? mx0 : m0, mn1 = mx1 > m1 + 1.f ? mx1 : m1;
        const float f0 = ex2f(m0 - mn0), f1 = ex2f(m1 - mn1);   // 0 on the first block
        l0 *= f0;
        l1 *= f1;
        m0 = mn0;
        m1 = mn1;
        const float F = (t >> 1) ? f1 : f0;
#pragma unroll
        for (int mb = 0; mb < C::MB; ++mb)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[0][mb][e] *= F;
      }
      const float p0 = ex2f(x0 - m0), p1 = ex2f(x1 - m1);
      l0 += p0;
      l1 += p1;
      const float pw0 = p0 * svl, pw1 = p1 * svl;
      // Block maxima by one warp reduction each on the bit patterns: as
      // signed integers they order the non-negative floats as floats do and
      // put every negative one below them.
      const float pm0 = __int_as_float(__reduce_max_sync(0xffffffffu, __float_as_int(pw0)));
      const float pm1 = __int_as_float(__reduce_max_sync(0xffffffffu, __float_as_int(pw1)));
      // W_q = rint(p s^V kWMax / pm) <= kWMax from the low 16 bits of
      // p s^V r + 2^23 (r needs no IEEE division: any r <= kWMax (1 + 2^-22)
      // / pm keeps W_q within 16 bits, and dinv below uses pm itself).
      const float r0 = pm0 > 0.f ? kWMax * rcp_approx(pm0) : 0.f, r1 = pm1 > 0.f ? kWMax * rcp_approx(pm1) : 0.f;
      u[0][0] = pack_lo16(__float_as_uint(fmaf(pw0, r0, 8388608.f)), __float_as_uint(fmaf(pw1, r1, 8388608.f)));
      dinv[0] = ((t >> 1) ? pm1 : pm0) * (128.f / kWMax);
    } else {
    // x[T][e]: token 16T + 8(e >> 1) + g, head 2t + (e & 1).  Padded heads
    // (qk = 0) score 0 and never move a maximum; their weights only reach
    // accumulators that are never stored.
    float x[2][4], sv[2][2];
#pragma unroll
    for (int T = 0; T < 2; ++T) {
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int j = 16 * T + 8 * hh + g;
        const float sk = lds_half(nk + 2 * j);
        sv[T][hh] = lds_half(nv + 2 * j);
        x[T][2 * hh] = sc[T][2 * hh] * sk * qk0;
        x[T][2 * hh + 1] = sc[T][2 * hh + 1] * sk * qk1;
      }
    }
    if (nvalid < kBlk) {   // the chunk's partial last block (warp-uniform)
#pragma unroll
      for (int T = 0; T < 2; ++T) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const bool ok = 16 * T + 8 * hh + g < nvalid;
          sv[T][hh] = ok ? sv[T][hh] : 0.f;
          x[T][2 * hh] = ok ? x[T][2 * hh] : -INFINITY;
          x[T][2 * hh + 1] = ok ? x[T][2 * hh + 1] : -INFINITY;
        }
      }
    }
    // Move the reference maximum only when a score passes m_ref + 1.
    // Lane-local maxima decide; the warp-wide ones are only formed when a
    // lane objects.
    float mx0 = fmaxf(fmaxf(x[0][0], x[0][2]), fmaxf(x[1][0], x[1][2]));
    float mx1 = fmaxf(fmaxf(x[0][1], x[0][3]), fmaxf(x[1][1], x[1][3]));
    if (__any_sync(0xffffffffu, mx0 > m0 + 1.f || mx1 > m1 + 1.f)) {
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
      }
      const float mn0 = mx0 > m0 + 1.f ? mx0 : m0, mn1 = mx1 > m1 + 1.f ? mx1 : m1;
      const float f0 = ex2f(m0 - mn0), f1 = ex2f(m1 - mn1);   // 0 on the first block
      l0 *= f0;
      l1 *= f1;
      m0 = mn0;
      m1 = mn1;
#pragma unroll
      for (int nvt = 0; nvt < C::NV; ++nvt) {
        const float fa = __shfl_sync(0xffffffffu, f0, nvt), fb = __shfl_sync(0xffffffffu, f1, nvt);
        const float F = (t >> 1) ? fb : fa;
#pragma unroll
        for (int mb = 0; mb < C::MB; ++mb)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[nvt][mb][e] *= F;
      }
    }
    // p = 2^(x - m_ref) <= 2 and the block's largest p s^V per head.
    float pw[2][4], pm0 = 0.f, pm1 = 0.f;
#pragma unroll
    for (int T = 0; T < 2; ++T) {
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const float p0 = ex2f(x[T][2 * hh] - m0), p1 = ex2f(x[T][2 * hh + 1] - m1);
        l0 += p0;
        l1 += p1;
        pw[T][2 * hh] = p0 * sv[T][hh];
        pw[T][2 * hh + 1] = p1 * sv[T][hh];
        pm0 = fmaxf(pm0, pw[T][2 * hh]);
        pm1 = fmaxf(pm1, pw[T][2 * hh + 1]);
      }
    }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      pm0 = fmaxf(pm0, __shfl_xor_sync(0xffffffffu, pm0, o));
      pm1 = fmaxf(pm1, __shfl_xor_sync(0xffffffffu, pm1, o));
    }
    // W_q = rint(p s^V kWMax / pm) <= kWMax from the low 16 bits of
    // p s^V r + 2^23; one unit of 256 E1 + E2 is then 2^7 pm / kWMax of
    // sum p s^V C (dinv, in the PV layout).  u[T][hh]: (W head 2t, W head
    // 2t+1) of token 16T + 8hh + g.
    // (r needs no IEEE division: any r <= kWMax (1 + 2^-22) / pm keeps W_q
    // within 16 bits, and dinv below uses pm itself.)
    const float r0 = pm0 > 0.f ? kWMax * rcp_approx(pm0) : 0.f, r1 = pm1 > 0.f ? kWMax * rcp_approx(pm1) : 0.f;
#pragma unroll
    for (int T = 0; T < 2; ++T) {
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const float wq0 = fmaf(pw[T][2 * hh], r0, 8388608.f), wq1 = fmaf(pw[T][2 * hh + 1], r1, 8388608.f);
        u[T][hh] = pack_lo16(__float_as_uint(wq0), __float_as_uint(wq1));
      }
    }
#pragma unroll
    for (int nvt = 0; nvt < C::NV; ++nvt) {
      const float da = __shfl_sync(0xffffffffu, pm0, nvt), db = __shfl_sync(0xffffffffu, pm1, nvt);
      dinv[nvt] = ((t >> 1) ? db : da) * (128.f / kWMax);
    }
    }

    // ---- PV, per 16-token half: this lane's tokens t, t+4, t+8, t+12 ----
    // With GP <= 2 the int32 sums of both halves accumulate in one pair of
    // registers per element and are converted once per block (both halves
    // share the block's scale); otherwise once per half.
    int e1c[C::COMPACT ? C::MB : 1][4], e2c[C::COMPACT ? C::MB : 1][4];
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      // B fragments of W for each N tile nv (heads 2nv, 2nv+1): column g =
      // (head 2nv + (g >> 2), parity g & 3); MMA c covers tokens 16 h2 + 8c +
      // {t, t+4}: held by lanes 16 h2 + 8c + t and + 4 (compact layout, in
      // u[0][0]) or by the QK lanes (t or t+4, nv) in u[h2][c].
      uint32_t bh[C::NV][2][2], bl[C::NV][2][2];
#pragma unroll
      for (int nvt = 0; nvt < C::NV; ++nvt) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t xa, xb;
          if constexpr (C::COMPACT) {
            xa = __shfl_sync(0xffffffffu, u[0][0], 16 * h2 + 8 * c + t);
            xb = __shfl_sync(0xffffffffu, u[0][0], 16 * h2 + 8 * c + t + 4);
          } else {
            xa = __shfl_sync(0xffffffffu, u[h2][c], 4 * t + nvt);
            xb = __shfl_sync(0xffffffffu, u[h2][c], 4 * t + 16 + nvt);
          }
          bh[nvt][c][0] = prmt(xa, 0u, sel_hi);
          bh[nvt][c][1] = prmt(xb, 0u, sel_hi);
          bl[nvt][c][0] = prmt(xa, 0u, sel_lo);
          bl[nvt][c][1] = prmt(xb, 0u, sel_lo);
        }
      }
      uint32_t vs[4][8];
      {
        const int goff = (D == 256 ? g : (g >> 1)) * 12;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const unsigned char *row = vc + (16 * h2 + t + 4 * r) * C::PB + goff;
          group_sel8_im(lds32(row), lds32(row + 4), lds32(row + 8), vs[r], lut.neg1, lut.one);
        }
      }
#pragma unroll
      for (int mb = 0; mb < C::MB; ++mb) {
        // Quads of the lane: 2mb, 2mb+1 of its group (d = 256) or of its half
        // group (d = 128: codes 16..31 for odd g).
        uint32_t ah[4][2], al[4][2];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          uint32_t s0, s1;
          if constexpr (D == 256) {
            s0 = vs[r][2 * mb];
            s1 = vs[r][2 * mb + 1];
          } else {
            s0 = (g & 1) ? vs[r][4 + 2 * mb] : vs[r][2 * mb];
            s1 = (g & 1) ? vs[r][5 + 2 * mb] : vs[r][2 * mb + 1];
          }
          ah[r][0] = prmt(lut.vh0, lut.vh1, s0);
          ah[r][1] = prmt(lut.vh0, lut.vh1, s1);
          al[r][0] = prmt(lut.vl0, lut.vl1, s0);
          al[r][1] = prmt(lut.vl0, lut.vl1, s1);
        }
        if constexpr (C::COMPACT) {
          // |256 E1 + E2| < 32 x 2^15 x 255 < 2^31 over the whole block.
          int(&e1)[4] = e1c[mb];
          int(&e2)[4] = e2c[mb];
          if (h2 == 0) {
            mma_s8u8_z(e1, ah[0][0], ah[0][1], ah[1][0], ah[1][1], bh[0][0][0], bh[0][0][1]);
            mma_s8u8_z(e2, ah[0][0], ah[0][1], ah[1][0], ah[1][1], bl[0][0][0], bl[0][0][1]);
          } else {
            mma_s8u8(e1, ah[0][0], ah[0][1], ah[1][0], ah[1][1], bh[0][0][0], bh[0][0][1]);
            mma_s8u8(e2, ah[0][0], ah[0][1], ah[1][0], ah[1][1], bl[0][0][0], bl[0][0][1]);
          }
          mma_s8u8(e1, ah[2][0], ah[2][1], ah[3][0], ah[3][1], bh[0][1][0], bh[0][1][1]);
          mma_s8u8(e2, ah[2][0], ah[2][1], ah[3][0], ah[3][1], bl[0][1][0], bl[0][1][1]);
          mma_s8u8(e2, al[0][0], al[0][1], al[1][0], al[1][1], bh[0][0][0], bh[0][0][1]);
          mma_s8u8(e2, al[2][0], al[2][1], al[3][0], al[3][1], bh[0][1][0], bh[0][1][1]);
          if (h2 == 1) {
#pragma unroll
            for (int e = 0; e < 4; ++e)
              acc[0][mb][e] = fmaf(static_cast<float>(256 * e1[e] + e2[e]), dinv[0], acc[0][mb][e]);
          }
        } else {
#pragma unroll
        for (int nvt = 0; nvt < C::NV; ++nvt) {
          // This half's sums: |256 E1 + E2| < 16 x 2^15 x 255 < 2^31.
          int e1[4], e2[4];
          mma_s8u8_z(e1, ah[0][0], ah[0][1], ah[1][0], ah[1][1], bh[nvt][0][0], bh[nvt][0][1]);
          mma_s8u8(e1, ah[2][0], ah[2][1], ah[3][0], ah[3][1], bh[nvt][1][0], bh[nvt][1][1]);
          mma_s8u8_z(e2, ah[0][0], ah[0][1], ah[1][0], ah[1][1], bl[nvt][0][0], bl[nvt][0][1]);
          mma_s8u8(e2, ah[2][0], ah[2][1], ah[3][0], ah[3][1], bl[nvt][1][0], bl[nvt][1][1]);
          mma_s8u8(e2, al[0][0], al[0][1], al[1][0], al[1][1], bh[nvt][0][0], bh[nvt][0][1]);
          mma_s8u8(e2, al[2][0], al[2][1], al[3][0], al[3][1], bh[nvt][1][0], bh[nvt][1][1]);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            acc[nvt][mb][e] = fmaf(static_cast<float>(256 * e1[e] + e2[e]), dinv[nvt], acc[nvt][mb][e]);
        }
        }
      }
    }
    __syncwarp();
    // The warp is done reading stage s.  When round i + kI8Stages exists,
    // round i is full (all four warps read stage s) and the fourth warp to
    // finish refills it; the counter's acquire-release add orders the other
    // warps' reads before that copy.
    if (lane == 0 && kI8Warps * (i + kI8Stages) < n_blk) {
      uint32_t old;
      asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], 1;"
                   : "=r"(old)
                   : "r"(smem_u32(&done_cnt[s]))
                   : "memory");
      if ((old & (kI8Warps - 1)) == kI8Warps - 1) {
        fence_proxy_async_smem();
        issue(i + kI8Stages);
      }
    }
  }
  // Every copy issued lands before the ring is reused or the CTA exits (in
  // the normal path each was waited for; after a timed-out wait not).
  __syncthreads();
  if (tid == 0) {
    const int ri = static_cast<int>(*rounds_issued);
    for (int r = ri - kI8Stages < 0 ? 0 : ri - kI8Stages; r < ri; ++r)
      if (!mbar_wait_bounded(&full_bar[r % kI8Stages], (r / kI8Stages) & 1)) break;
  }

  // Per-warp totals over the 8 lanes sharing t (over all 32 lanes with
  // the compact softmax, where m0, m1 are the same in every lane).
#pragma unroll
  for (int o = C::COMPACT ? 1 : 4; o < 32; o <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o);
  }
  if constexpr (SLICES) {
    __syncthreads();   // every warp is done with the ring, and its copies have landed
    // Each warp's accumulators go raw into its own slice [warp][head][dim]
    // (rotated domain) over the ring memory; after one barrier the slices are
    // scaled to the common maximum and summed in warp order (a fixed order).
    float *slices = reinterpret_cast<float *>(smem);
    if (C::COMPACT ? lane == 0 : g == 0) {
      const int h0 = C::COMPACT ? 0 : 2 * t;
      wm[warp * 8 + h0] = m0;
      wm[warp * 8 + h0 + 1] = m1;
      wl[warp * 8 + h0] = l0;
      wl[warp * 8 + h0 + 1] = l1;
    }
    {
      const int grp = D == 256 ? g : (g >> 1);
      const int qoff = D == 256 ? 0 : 4 * (g & 1);
  #pragma unroll
      for (int nvt = 0; nvt < C::NV; ++nvt) {
        const int h = 2 * nvt + (t >> 1);
        if (h < G) {
          float *dst = slices + (warp * GP + h) * D;
  #pragma unroll
          for (int mb = 0; mb < C::MB; ++mb)
  #pragma unroll
            for (int e = 0; e < 4; ++e)
              dst[32 * grp + 4 * (2 * mb + (e >> 1) + qoff) + 2 * (t & 1) + (e & 1)] = acc[nvt][mb][e];
        }
      }
    }
    __syncthreads();

    // One partial state per query head: natural-log max, sum, acc (unscaled).
    for (int h = 0; h < G; ++h) {
      float mstar = -INFINITY;
      for (int w2 = 0; w2 < kI8Warps; ++w2) mstar = fmaxf(mstar, wm[w2 * 8 + h]);
      float f[kI8Warps];
  #pragma unroll
      for (int w2 = 0; w2 < kI8Warps; ++w2) {
        const float mw = wm[w2 * 8 + h];
        f[w2] = mw == -INFINITY ? 0.f : exp2f(mw - mstar);
      }
      const long long slot = (static_cast<long long>(b) * a.hq + kvh * G + h) * a.n_splits + split;
      float *acc_out = a.ws_acc + slot * D;
      for (int i = tid; i < D; i += kI8Threads) {
        float sum = 0.f;
  #pragma unroll
        for (int w2 = 0; w2 < kI8Warps; ++w2) sum += slices[(w2 * GP + h) * D + i] * f[w2];
        acc_out[i] = sum * out_scale;
      }
      if (tid == 0) {
        float l = 0.f;
        for (int w2 = 0; w2 < kI8Warps; ++w2) l += wl[w2 * 8 + h] * f[w2];
        a.ws_ml[slot] = make_float2(mstar == -INFINITY ? -INFINITY : mstar * 0.69314718055994531f, l);
      }
    }
  } else {
    __syncthreads();   // all warps are done with the q~ scratch
    if (C::COMPACT ? lane == 0 : g == 0) {
      const int h0 = C::COMPACT ? 0 : 2 * t;
      wm[warp * 8 + h0] = m0;
      wm[warp * 8 + h0 + 1] = m1;
      wl[warp * 8 + h0] = l0;
      wl[warp * 8 + h0 + 1] = l1;
    }
    __syncthreads();
    // Merge the warps' accumulators into scratch[head][dim] (rotated domain),
    // one warp after the other so that the sum order is fixed.
    {
      const int grp = D == 256 ? g : (g >> 1);
      const int qoff = D == 256 ? 0 : 4 * (g & 1);
      float f[C::NV];
  #pragma unroll
      for (int nvt = 0; nvt < C::NV; ++nvt) {
        const int h = 2 * nvt + (t >> 1);
        float mstar = -INFINITY;
        for (int w2 = 0; w2 < kI8Warps; ++w2) mstar = fmaxf(mstar, wm[w2 * 8 + h]);
        const float mine = wm[warp * 8 + h];
        f[nvt] = (mine == -INFINITY) ? 0.f : exp2f(mine - mstar);
      }
      for (int w2 = 0; w2 < kI8Warps; ++w2) {
        if (warp == w2) {
  #pragma unroll
          for (int nvt = 0; nvt < C::NV; ++nvt) {
            const int h = 2 * nvt + (t >> 1);
            if (h < G) {
  #pragma unroll
              for (int mb = 0; mb < C::MB; ++mb) {
  #pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const int dim = 32 * grp + 4 * (2 * mb + (e >> 1) + qoff) + 2 * (t & 1) + (e & 1);
                  float *dst = scratch + h * D + dim;
                  const float v = acc[nvt][mb][e] * f[nvt];
                  *dst = (w2 == 0) ? v : *dst + v;
                }
              }
            }
          }
        }
        __syncthreads();
      }
    }

    // One partial state per query head: natural-log max, sum, acc (unscaled).
    for (int h = 0; h < G; ++h) {
      const long long slot = (static_cast<long long>(b) * a.hq + kvh * G + h) * a.n_splits + split;
      float *acc_out = a.ws_acc + slot * D;
      for (int i = tid; i < D; i += kI8Threads) acc_out[i] = scratch[h * D + i] * out_scale;
      if (tid == 0) {
        float mstar = -INFINITY, l = 0.f;
        for (int w2 = 0; w2 < kI8Warps; ++w2) mstar = fmaxf(mstar, wm[w2 * 8 + h]);
        for (int w2 = 0; w2 < kI8Warps; ++w2) {
          const float mw = wm[w2 * 8 + h];
          if (mw != -INFINITY) l += wl[w2 * 8 + h] * exp2f(mw - mstar);
        }
        a.ws_ml[slot] = make_float2(mstar == -INFINITY ? -INFINITY : mstar * 0.69314718055994531f, l);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

struct I8Tables {
  double scale;   // S: C_k = rint(S c_k) for the unit-variance centroids c_k
  I8Lut lut;
};

inline int floor_div128(int x) { return x >= 0 ? x / 128 : -((-x + 127) / 128); }

// S in [0.75, 1] * 16319 / c_max minimising the largest relative rounding
// error of S c_k over the four positive 3-bit centroids (searched once).
const I8Tables &i8_tables() {
  static I8Tables tb;
  static std::once_flag once;
  std::call_once(once, [] {
    double c[8];
    codebook_unit_f64(3, c);
    const double s_max = kCentroidIntMax / c[7];
    double best = s_max, best_err = 1.0;
    const int steps = 1 << 22;
    for (int i = 0; i <= steps; ++i) {
      const double s = s_max * (0.75 + 0.25 * static_cast<double>(i) / steps);
      double err = 0.0;
      for (int k = 4; k < 8 && err < best_err; ++k) {
        const double v = s * c[k];
        err = std::fmax(err, std::fabs(std::nearbyint(v) - v) / v);
      }
      if (err < best_err) {
        best_err = err;
        best = s;
      }
    }
    tb.scale = best;
    uint32_t kh[2] = {0, 0}, kl[2] = {0, 0}, vl[2] = {0, 0};
    for (int k = 0; k < 8; ++k) {
      const int ck = static_cast<int>(std::lrint(best * c[k]));
      const int ch = floor_div128(ck + 64);
      const int cl = ck - 128 * ch;
      const int sh = 8 * (k % 4);
      kh[k / 4] |= (static_cast<uint32_t>(ch) & 0xFFu) << sh;
      kl[k / 4] |= (static_cast<uint32_t>(cl) & 0xFFu) << sh;
      vl[k / 4] |= (static_cast<uint32_t>(2 * cl) & 0xFFu) << sh;
    }
    tb.lut = I8Lut{kh[0], kh[1], kl[0], kl[1], kh[0], kh[1], vl[0], vl[1], 0xFFFFFFFFu, 1u};
  });
  return tb;
}

template <int D, bool FULL, int GP>
int launch_split_i8(const SplitArgs &a, cudaStream_t stream) {
  using C = I8Cfg<D, GP>;
  // The sliced warp merge for chunks up to 2048 tokens (see split_i8_kernel).
  const bool slices = a.chunk <= 2048;
  auto kernel = slices ? split_i8_kernel<D, FULL, GP, true> : split_i8_kernel<D, FULL, GP, false>;
  static bool configured = false;
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!configured) {
      for (auto k : {split_i8_kernel<D, FULL, GP, true>, split_i8_kernel<D, FULL, GP, false>}) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (e != cudaSuccess) return set_error(ISOQ_ERR_CUDA, "decode i8: %s", cudaGetErrorString(e));
      }
      configured = true;
    }
  }
  const I8Tables &tb = i8_tables();
  const double unit = 1.0 / (tb.scale * std::sqrt(static_cast<double>(D)));
  const float score_unit = static_cast<float>(a.scale * unit * 1.4426950408889634);
  const float out_scale = static_cast<float>(unit);
  dim3 grid(a.n_splits, a.hkv, a.batch);
  static_assert(C::QPREP_WORDS == decode_qprep_words(D), "prepared-query layout");
  prep_i8_kernel<D, FULL, GP><<<dim3(a.hkv, a.batch), 32 * GP, 0, stream>>>(a, score_unit);
  cudaError_t e = launch_pdl(kernel, grid, dim3(kI8Threads), C::SMEM, stream, a, tb.lut, out_scale);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(ISOQ_ERR_CUDA, "decode i8 launch: %s", cudaGetErrorString(e));
  return ISOQ_OK;
}

// Float16 queries, 3-bit codes, d in {128, 256}, G <= 8, and chunks and
// rows whose bulk copies start on 16-byte boundaries (the int32 PV sums cover
// 16 tokens and the QK sums one token, so any chunk length is in range).
bool i8_path_supported(int dtype, int d, int bits, const SplitArgs &a) {
  return dtype == ISOQ_F16 && bits == 3 && (d == 128 || d == 256) && a.group <= 8 &&
         a.tmax % 8 == 0 && a.chunk % kDecodeTokenQuantum == 0 &&
         (reinterpret_cast<uintptr_t>(a.norms_k) & 15u) == 0 &&
         (reinterpret_cast<uintptr_t>(a.norms_v) & 15u) == 0;
}

template <int D, bool FULL>
int run_split_i8_d(const SplitArgs &a, cudaStream_t st) {
  const int G = a.group;
  if (G == 1) return launch_split_i8<D, FULL, 1>(a, st);
  if (G == 2) return launch_split_i8<D, FULL, 2>(a, st);
  if (G <= 4) return launch_split_i8<D, FULL, 4>(a, st);
  return launch_split_i8<D, FULL, 8>(a, st);
}

int run_split_i8(int d, int variant, const SplitArgs &a, cudaStream_t st) {
  if (d == 128)
    return variant == ISOQ_FULL ? run_split_i8_d<128, true>(a, st) : run_split_i8_d<128, false>(a, st);
  return variant == ISOQ_FULL ? run_split_i8_d<256, true>(a, st) : run_split_i8_d<256, false>(a, st);
}
