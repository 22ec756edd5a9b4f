// Tensor-core split kernel of the compressed-space decode: float16 queries,
// 3-bit codes, d in {128, 256}, up to 8 query heads per KV head.
// Included by isoq_decode.cu inside namespace isoq::decode.
//
// Per CTA: one (b, kvh, token chunk) and all G query heads of the KV head.
// The chunk is cut into 16-token slabs; warp w takes slabs w, w+4, w+8, ...
// and streams them through its own 3-deep ring of shared-memory stages with
// CTA-local bulk copies (packed K/V rows and float16 norms; mbarrier
// completion), issuing the copy for slab i+3 as soon as it is done with slab
// i.  There is no producer warp and no cross-warp handshake until the final
// merge, so four CTAs (16 warps) fit on an SM.
//
// QK (RotaryQuant Table 2 kernel A): mma.sync m16n8k16, A = K~ [16 tokens x
// 16 dims] expanded from the codes in registers, B = q~ [16 dims x 8 columns].
// q~ is split into float16 hi + lo parts so that its rounding does not reach
// the scores: for G in {1, 2, 4} the lo parts take the spare columns G..2G-1
// of the same MMA; otherwise a second MMA adds them.
// The online softmax (kernel B) runs on the QK accumulator fragments.
// PV (kernel C): mma.sync with M = 16 dim pairs, K = 8 tokens x 2 parities,
// N = 4 heads x 2 parities:  D[u][(h, r)] = sum_j V~[j][2u + r] P[j][h], i.e.
// B[(j, r')][(h, r)] = P[j][h] [r' = r].  Each A register then holds two
// consecutive dims of one token, exactly what the code lookup produces.
//
// Fragment orders.  A fixed permutation of the rotated coordinates cancels in
// q~.k~ and is undone when the accumulator is written out, and a permutation
// of the tokens inside a slab is applied identically to P and V~; both are
// chosen so that each lane expands whole 32-code groups (three words in the
// layout of common.cuh, codes in 4-bit fields):
//   QK: lane (g, t) owns tokens g and g+8 and dims [t d/4, (t+1) d/4); MMA kk
//       uses its dims t d/4 + 4kk + {0,1} (k = 2t, 2t+1) and {2,3} (2t+8, 2t+9).
//   PV: lane (g, t) owns dims [g d/8, (g+1) d/8) and tokens t, t+4, t+8, t+12;
//       M-block mb maps row g to dims g d/8 + 4mb + {0,1} and row g+8 to
//       + {2,3}; K column 2j + r of a token half is token j (0..3 -> t, 4..7
//       -> t+4 within the lane's pair) with parity r.
// Code -> float16 centroid is a byte lookup with prmt: the low and high bytes
// of the 8 centroids sit in two register pairs, a selector made of four code
// nibbles picks four entries at once, and two more prmt interleave the bytes
// into half2.
// The centroids are scaled by a host-chosen alpha that makes all of them
// nearly exact in float16; alpha is divided out of the scores and the output.

constexpr int kMmaWarps = 4;
constexpr int kMmaThreads = 32 * kMmaWarps;
constexpr int kSlab = 16;          // tokens per slab (the M of one QK tile)
constexpr int kWarpStages = 3;     // per-warp ring depth
constexpr int kChunkQuantum = kSlab * kMmaWarps;

template <int D>
struct MmaCfg {
  static constexpr int PB = D * 3 / 8;                      // packed bytes per token
  static constexpr int SLAB_CODES = kSlab * PB;
  static constexpr int SLAB_NORMS = kSlab * 2;
  static constexpr int STAGE_BYTES = 2 * SLAB_CODES + 2 * SLAB_NORMS;
  static constexpr int RING_BYTES = kWarpStages * STAGE_BYTES;
  static constexpr int KK = D / 16;                         // QK MMAs along d
  static constexpr int QSEG = D / 4;                        // dims per lane in QK
  static constexpr int VSEG = D / 8;                        // dims per lane in PV
  static constexpr int MB = D / 32;                         // PV M-blocks
  static constexpr int SCRATCH_FLOATS = 8 * D;              // q~ staging, then the warp merge
  static constexpr int SMEM = kMmaWarps * RING_BYTES + SCRATCH_FLOATS * 4 +
                              2 * kMmaWarps * 8 * 4 + kMmaWarps * kWarpStages * 8 + 128;
};

struct MmaLut {
  uint32_t lo0, lo1, hi0, hi1;  // low/high bytes of the 8 float16 centroids (scaled)
};

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// prmt selectors of one 32-code group (three words in the layout of
// common.cuh): m_r = codes 8r..8r+7 with the spare bits cleared, and e =
// codes 24..31 gathered from the spare bits.  Quad q (codes 4q..4q+3) is the
// low or high half of one of them.
struct GroupSel {
  uint32_t m0, m1, m2, e;
};

__device__ __forceinline__ GroupSel group_selectors(uint32_t w0, uint32_t w1, uint32_t w2) {
  GroupSel s;
  s.m0 = w0 & 0x77777777u;
  s.m1 = w1 & 0x77777777u;
  s.m2 = w2 & 0x77777777u;
  s.e = ((w0 >> 3) & 0x11111111u) | ((w1 >> 2) & 0x22222222u) | ((w2 >> 1) & 0x44444444u);
  return s;
}

__device__ __forceinline__ uint32_t quad_selector(const GroupSel &s, int q) {
  const uint32_t x = q < 2 ? s.m0 : (q < 4 ? s.m1 : (q < 6 ? s.m2 : s.e));
  return (q & 1) ? (x >> 16) : x;
}

// Two half2 from a 4-nibble selector: (c[s0], c[s1]) and (c[s2], c[s3]).
__device__ __forceinline__ void lut4(const MmaLut &l, uint32_t sel, uint32_t &h01, uint32_t &h23) {
  const uint32_t lo = prmt(l.lo0, l.lo1, sel);
  const uint32_t hi = prmt(l.hi0, l.hi1, sel);
  h01 = prmt(lo, hi, 0x5140u);
  h23 = prmt(lo, hi, 0x7362u);
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

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}

// QIN: q~'s lo parts ride in the spare B columns (G in {1, 2, 4}).
// NT:  number of 4-head N tiles of the PV product (1 for G <= 4, else 2).
template <int D, bool FULL, bool QIN, int NT>
__global__ void __launch_bounds__(kMmaThreads, D == 256 && NT == 2 ? 2 : (D == 256 && !QIN ? 3 : 4))
    split_mma_kernel(const SplitArgs a, const MmaLut lut,
                                                                   float qk_scale_log2, float out_scale) {
  using C = MmaCfg<D>;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~static_cast<uintptr_t>(127));
  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.group;

  unsigned char *ring = smem + warp * C::RING_BYTES;
  float *scratch = reinterpret_cast<float *>(smem + kMmaWarps * C::RING_BYTES);
  float *wm = scratch + C::SCRATCH_FLOATS;          // [warps][8]
  float *wl = wm + kMmaWarps * 8;                   // [warps][8]
  uint64_t *full_bar = reinterpret_cast<uint64_t *>(wl + kMmaWarps * 8) + warp * kWarpStages;

  int tlen = a.seq_lens[b];
  tlen = tlen < 0 ? 0 : (tlen > a.tmax ? static_cast<int>(a.tmax) : tlen);
  const long long t0 = static_cast<long long>(split) * a.chunk;
  long long t1 = t0 + a.chunk;
  if (t1 > tlen) t1 = tlen;
  const int n_tok = t1 > t0 ? static_cast<int>(t1 - t0) : 0;
  const int n_slabs = (n_tok + kSlab - 1) / kSlab;
  const int n_mine = n_slabs > warp ? (n_slabs - warp + kMmaWarps - 1) / kMmaWarps : 0;

  const long long pair = static_cast<long long>(b) * a.hkv + kvh;
  const uint8_t *kb = a.packed_k + pair * a.tmax * C::PB;
  const uint8_t *vb = a.packed_v + pair * a.tmax * C::PB;
  const uint16_t *nkb = a.norms_k + pair * a.tmax;
  const uint16_t *nvb = a.norms_v + pair * a.tmax;

  // Lane 0 of each warp issues the copies of the warp's i-th slab into ring
  // stage i % kWarpStages.
  auto issue = [&](int i) {
    const int j = warp + kMmaWarps * i;                 // slab index within the chunk
    const long long t = t0 + static_cast<long long>(j) * kSlab;
    int n = n_tok - j * kSlab;
    if (n > kSlab) n = kSlab;
    const int n8 = (n + 7) & ~7;
    const int s = i % kWarpStages;
    unsigned char *st = ring + s * C::STAGE_BYTES;
    mbar_arrive_expect_tx(&full_bar[s], 2u * n * C::PB + 4u * n8);
    bulk_load(st, kb + t * C::PB, n * C::PB, &full_bar[s]);
    bulk_load(st + C::SLAB_CODES, vb + t * C::PB, n * C::PB, &full_bar[s]);
    bulk_load(st + 2 * C::SLAB_CODES, nkb + t, 2 * n8, &full_bar[s]);
    bulk_load(st + 2 * C::SLAB_CODES + C::SLAB_NORMS, nvb + t, 2 * n8, &full_bar[s]);
  };
  int issued = 0;
  if (lane == 0) {
    for (int s = 0; s < kWarpStages; ++s) mbar_init(&full_bar[s], 1);
    mbar_fence_init();
    for (; issued < kWarpStages && issued < n_mine; ++issued) issue(issued);
  }

  // Rotate the G queries of this KV head once, q~ = R_K q, while the first
  // slabs stream in.
  for (int i = tid; i < 8 * D; i += kMmaThreads) {
    const int gq = i / D;
    float v = 0.f;
    if (gq < G) {
      const __half *qp = static_cast<const __half *>(a.q) +
                         (static_cast<long long>(b) * a.hq + kvh * G + gq) * D;
      v = __half2float(qp[i % D]);
    }
    scratch[i] = v;
  }
  __syncthreads();
  rotate_forward_smem<D, FULL>(scratch, G, a.params_k + static_cast<size_t>(kvh) * 2 * D, tid,
                               kMmaThreads, 0);

  const int g = lane >> 2, t = lane & 3;

  // B fragments of q~ (hi + lo float16 parts) for QK: column g, dims
  // t*QSEG + 4kk + {0..3}.
  uint32_t qf[C::KK][2];
  uint32_t qflo[QIN ? 1 : C::KK][2];
  {
    const int head = QIN ? (g < G ? g : g - G) : g;
    const bool live = QIN ? (g < 2 * G) : (g < G);
    const bool lo_col = QIN && g >= G;
#pragma unroll
    for (int kk = 0; kk < C::KK; ++kk) {
      float v[4], hi[4], lo[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[j] = live ? scratch[head * D + t * C::QSEG + 4 * kk + j] : 0.f;
        hi[j] = __half2float(__float2half_rn(v[j]));
        lo[j] = v[j] - hi[j];
      }
      if (QIN) {
        const float *src = lo_col ? lo : hi;
        qf[kk][0] = pack_half2(src[0], src[1]);
        qf[kk][1] = pack_half2(src[2], src[3]);
      } else {
        qf[kk][0] = pack_half2(hi[0], hi[1]);
        qf[kk][1] = pack_half2(hi[2], hi[3]);
        qflo[QIN ? 0 : kk][0] = pack_half2(lo[0], lo[1]);
        qflo[QIN ? 0 : kk][1] = pack_half2(lo[2], lo[3]);
      }
    }
  }

  float acc[NT][C::MB][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int mb = 0; mb < C::MB; ++mb) acc[nt][mb][0] = acc[nt][mb][1] = acc[nt][mb][2] = acc[nt][mb][3] = 0.f;
  // Online-softmax state in the QK layout: heads 2t, 2t+1 (log2 domain).
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const bool real0 = 2 * t < G, real1 = 2 * t + 1 < G;

  int consumed = 0;
  bool failed = false;
  for (int i = 0; i < n_mine; ++i) {
    const int s = i % kWarpStages;
    if (!mbar_wait_bounded(&full_bar[s], (i / kWarpStages) & 1)) {
      atomicOr(&g_decode_error, kErrWaitTimeout);
      failed = true;
      break;
    }
    {
      int nvalid = n_tok - (warp + kMmaWarps * i) * kSlab;
      nvalid = nvalid > kSlab ? kSlab : nvalid;
      {
        const unsigned char *st = ring + s * C::STAGE_BYTES;
        const unsigned char *kc = st;
        const unsigned char *vc = st + C::SLAB_CODES;
        const unsigned char *nk = st + 2 * C::SLAB_CODES;                 // float16 [16]
        const unsigned char *nv = st + 2 * C::SLAB_CODES + C::SLAB_NORMS;

        // ---- QK: S[16 tokens x 8 columns] ----
        float sc[4] = {0.f, 0.f, 0.f, 0.f};
        {
          constexpr int NW = C::QSEG * 3 / 32;   // words per token segment (3 or 6)
          uint32_t wg[NW], wg8[NW];
          const unsigned char *rg = kc + g * C::PB + t * (C::QSEG * 3 / 8);
          const unsigned char *rg8 = rg + 8 * C::PB;
          if constexpr (NW % 2 == 0) {   // 8-byte aligned segments: 64-bit loads
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
          for (int gq = 0; gq < C::QSEG / 32; ++gq) {
            const GroupSel sa = group_selectors(wg[3 * gq], wg[3 * gq + 1], wg[3 * gq + 2]);
            const GroupSel sb = group_selectors(wg8[3 * gq], wg8[3 * gq + 1], wg8[3 * gq + 2]);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const int kk = 8 * gq + q;
              uint32_t a0, a1, a2, a3;
              lut4(lut, quad_selector(sa, q), a0, a2);
              lut4(lut, quad_selector(sb, q), a1, a3);
              mma_16816(sc, a0, a1, a2, a3, qf[kk][0], qf[kk][1]);
              if (!QIN) mma_16816(sc, a0, a1, a2, a3, qflo[QIN ? 0 : kk][0], qflo[QIN ? 0 : kk][1]);
            }
          }
        }
        if (QIN) {
          // Add the lo columns G..2G-1 onto the hi columns 0..G-1.
          if (G == 1) {
            sc[0] += sc[1];
            sc[2] += sc[3];
          } else {
            const int o = G >> 1;
#pragma unroll
            for (int e = 0; e < 4; ++e) sc[e] += __shfl_xor_sync(0xffffffffu, sc[e], o);
          }
        }

        // ---- online softmax on the fragments (log2 domain) ----
        const bool vg = g < nvalid, vg8 = g + 8 < nvalid;
        const float skg = vg ? lds_half(nk + 2 * g) * qk_scale_log2 : 0.f;
        const float skg8 = vg8 ? lds_half(nk + 2 * (g + 8)) * qk_scale_log2 : 0.f;
        // Padded heads hold a constant 0 so that they never move the maximum.
        const float x0 = real0 ? (vg ? sc[0] * skg : -INFINITY) : 0.f;
        const float x1 = real1 ? (vg ? sc[1] * skg : -INFINITY) : 0.f;
        const float x2 = real0 ? (vg8 ? sc[2] * skg8 : -INFINITY) : 0.f;
        const float x3 = real1 ? (vg8 ? sc[3] * skg8 : -INFINITY) : 0.f;
        float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
          mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
        }
        // Rescale unconditionally (the factors are 1 when the maximum holds):
        // a few multiplies on the otherwise idle FMA pipe instead of a branch.
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        const float f0 = exp2f(m0 - mn0), f1 = exp2f(m1 - mn1);   // 0 on the first slab
        l0 *= f0;
        l1 *= f1;
        m0 = mn0;
        m1 = mn1;
        // The PV accumulator of lane (g, t) holds head nt*4 + t.
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int h = nt * 4 + t;
          const int src = 4 * g + (h >> 1);
          const float F0 = __shfl_sync(0xffffffffu, f0, src);
          const float F1 = __shfl_sync(0xffffffffu, f1, src);
          const float f = (h & 1) ? F1 : F0;
#pragma unroll
          for (int mb = 0; mb < C::MB; ++mb) {
            acc[nt][mb][0] *= f;
            acc[nt][mb][1] *= f;
            acc[nt][mb][2] *= f;
            acc[nt][mb][3] *= f;
          }
        }
        const float p0 = exp2f(x0 - m0), p1 = exp2f(x1 - m1);
        const float p2 = exp2f(x2 - m0), p3 = exp2f(x3 - m1);
        l0 += p0 + p2;
        l1 += p1 + p3;
        const float svg = vg ? lds_half(nv + 2 * g) : 0.f;
        const float svg8 = vg8 ? lds_half(nv + 2 * (g + 8)) : 0.f;
        const uint32_t u01 = pack_half2(p0 * svg, p1 * svg);      // token g, heads 2t, 2t+1
        const uint32_t u23 = pack_half2(p2 * svg8, p3 * svg8);    // token g+8

        // ---- PV: this lane's 4 tokens, one 32-code group each (d=256) or
        // half a group (d=128: lanes 2m, 2m+1 share group m) ----
        GroupSel vs[4];
        {
          const int goff = (D == 256 ? g : (g >> 1)) * 12;
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const unsigned char *row = vc + (t + 4 * r) * C::PB + goff;
            vs[r] = group_selectors(lds32(row), lds32(row + 4), lds32(row + 8));
            if (D == 128 && (g & 1)) {   // codes 16..31 of the group
              vs[r].m0 = vs[r].m2;
              vs[r].m1 = vs[r].e;
            }
          }
        }
        // B fragments of P for each N tile: column g = (head nt*4 + g/2, parity g&1).
        uint32_t pb[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int h = nt * 4 + (g >> 1);
          const int src1 = 4 * t + (h >> 1), src2 = 16 + 4 * t + (h >> 1);
          const uint32_t x_t = __shfl_sync(0xffffffffu, u01, src1);
          const uint32_t x_t4 = __shfl_sync(0xffffffffu, u01, src2);
          const uint32_t x_t8 = __shfl_sync(0xffffffffu, u23, src1);
          const uint32_t x_t12 = __shfl_sync(0xffffffffu, u23, src2);
          const uint32_t e2 = 2u * (h & 1);
          const uint32_t sel = (g & 1) ? (0x44u | (e2 << 8) | ((e2 + 1u) << 12))
                                       : (e2 | ((e2 + 1u) << 4) | 0x4400u);
          const bool live = h < G;
          pb[nt][0] = live ? prmt(x_t, 0u, sel) : 0u;
          pb[nt][1] = live ? prmt(x_t4, 0u, sel) : 0u;
          pb[nt][2] = live ? prmt(x_t8, 0u, sel) : 0u;
          pb[nt][3] = live ? prmt(x_t12, 0u, sel) : 0u;
        }
#pragma unroll
        for (int mb = 0; mb < C::MB; ++mb) {          // M-block mb = codes 4mb..4mb+3
          uint32_t ta0, ta1, tb0, tb1, tc0, tc1, td0, td1;
          lut4(lut, quad_selector(vs[0], mb), ta0, ta1);   // token t
          lut4(lut, quad_selector(vs[1], mb), tb0, tb1);   // token t+4
          lut4(lut, quad_selector(vs[2], mb), tc0, tc1);   // token t+8
          lut4(lut, quad_selector(vs[3], mb), td0, td1);   // token t+12
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            mma_16816(acc[nt][mb], ta0, ta1, tb0, tb1, pb[nt][0], pb[nt][1]);
            mma_16816(acc[nt][mb], tc0, tc1, td0, td1, pb[nt][2], pb[nt][3]);
          }
        }
      }
    }
    __syncwarp();
    consumed = i + 1;
    // The warp is done reading stage s: refill it with the slab kWarpStages on.
    if (lane == 0 && issued < n_mine) {
      fence_proxy_async_smem();
      issue(issued);
      ++issued;
    }
  }
  if (failed && lane == 0) {
    // Let every copy still in flight land before the CTA may exit.
    for (int k = consumed; k < issued; ++k)
      if (!mbar_wait_bounded(&full_bar[k % kWarpStages], (k / kWarpStages) & 1)) break;
  }

  // Per-warp totals over the 8 lanes sharing t.
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o);
  }
  __syncthreads();   // all warps are done with the q~ scratch
  if (g == 0) {
    wm[warp * 8 + 2 * t] = m0;
    wm[warp * 8 + 2 * t + 1] = m1;
    wl[warp * 8 + 2 * t] = l0;
    wl[warp * 8 + 2 * t + 1] = l1;
  }
  __syncthreads();
  // Merge the warps' accumulators into scratch[head][dim] (rotated domain),
  // one warp after the other so that the sum order is fixed.
  {
    float f[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int h = nt * 4 + t;
      float mstar = -INFINITY;
      for (int w2 = 0; w2 < kMmaWarps; ++w2) mstar = fmaxf(mstar, wm[w2 * 8 + h]);
      const float mine = wm[warp * 8 + h];
      f[nt] = (mine == -INFINITY) ? 0.f : exp2f(mine - mstar);
    }
    for (int w2 = 0; w2 < kMmaWarps; ++w2) {
      if (warp == w2) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int h = nt * 4 + t;
          if (h < G) {
#pragma unroll
            for (int mb = 0; mb < C::MB; ++mb) {
              float *dst = scratch + h * D + g * C::VSEG + 4 * mb;
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float v = acc[nt][mb][e] * f[nt];
                dst[e] = (w2 == 0) ? v : dst[e] + v;
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
    for (int i = tid; i < D; i += kMmaThreads) acc_out[i] = scratch[h * D + i] * out_scale;
    if (tid == 0) {
      float mstar = -INFINITY, l = 0.f;
      for (int w2 = 0; w2 < kMmaWarps; ++w2) mstar = fmaxf(mstar, wm[w2 * 8 + h]);
      for (int w2 = 0; w2 < kMmaWarps; ++w2) {
        const float mw = wm[w2 * 8 + h];
        if (mw != -INFINITY) l += wl[w2 * 8 + h] * exp2f(mw - mstar);
      }
      a.ws_ml[slot] = make_float2(mstar == -INFINITY ? -INFINITY : mstar * 0.69314718055994531f, l);
    }
  }
}

inline uint32_t half_bits(float v) {
  __half h = __float2half_rn(v);
  return static_cast<uint32_t>(*reinterpret_cast<unsigned short *>(&h));
}

// Round-to-nearest-even to an 11-bit significand (float16, normal range).
inline double round_f16(double x) {
  int e;
  const double m = std::frexp(x, &e);
  return std::ldexp(std::nearbyint(std::ldexp(m, 11)), e - 11);
}

// Scale alpha in [1, 2) minimising the largest relative float16 rounding
// error of alpha * c_k over the unit-variance 3-bit centroids (searched once).
double centroid_scale_3bit() {
  static double alpha = 0.0;
  static std::once_flag once;
  std::call_once(once, [] {
    CodebookF32 cb;
    codebook_f32(128, 3, &cb);
    double mags[4];
    for (int k = 0; k < 4; ++k) mags[k] = static_cast<double>(cb.centroid[4 + k]) * std::sqrt(128.0);
    double best = 1.0, best_err = 1.0;
    const int steps = 4000000;
    for (int i = 0; i < steps; ++i) {
      const double al = 1.0 + static_cast<double>(i) / steps;
      double err = 0.0;
      for (int k = 0; k < 4 && err < best_err; ++k) {
        const double v = al * mags[k];
        err = std::fmax(err, std::fabs(round_f16(v) - v) / v);
      }
      if (err < best_err) {
        best_err = err;
        best = al;
      }
    }
    alpha = best;
  });
  return alpha;
}

template <int D, bool FULL, bool QIN, int NT>
int launch_split_mma(const SplitArgs &a, cudaStream_t stream) {
  using C = MmaCfg<D>;
  auto kernel = split_mma_kernel<D, FULL, QIN, NT>;
  static bool configured = false;
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!configured) {
      cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
      if (e != cudaSuccess) return set_error(ISOQ_ERR_CUDA, "decode mma: %s", cudaGetErrorString(e));
      configured = true;
    }
  }
  // float16 centroids of the unit-variance codebook times alpha; the
  // 1/(sqrt(d) alpha) is folded into the score scale and the output scale.
  const double alpha = centroid_scale_3bit();
  const float sqrt_d = std::sqrt(static_cast<float>(D));
  uint32_t lo[2] = {0, 0}, hi[2] = {0, 0};
  for (int k = 0; k < 8; ++k) {
    const uint32_t hb = half_bits(static_cast<float>(a.centroid[k] * sqrt_d * alpha));
    lo[k / 4] |= (hb & 0xFFu) << (8 * (k % 4));
    hi[k / 4] |= (hb >> 8) << (8 * (k % 4));
  }
  MmaLut lut{lo[0], lo[1], hi[0], hi[1]};
  const float inv = static_cast<float>(1.0 / (static_cast<double>(sqrt_d) * alpha));
  const float qk_scale_log2 = a.scale * inv * 1.4426950408889634f;
  dim3 grid(a.n_splits, a.hkv, a.batch);
  kernel<<<grid, kMmaThreads, C::SMEM, stream>>>(a, lut, qk_scale_log2, inv);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(ISOQ_ERR_CUDA, "decode mma launch: %s", cudaGetErrorString(e));
  return ISOQ_OK;
}

bool mma_path_supported(int dtype, int d, int bits, const SplitArgs &a) {
  return dtype == ISOQ_F16 && bits == 3 && (d == 128 || d == 256) && a.group <= 8 &&
         a.tmax % 8 == 0 && a.chunk % kChunkQuantum == 0 &&
         (reinterpret_cast<uintptr_t>(a.norms_k) & 15u) == 0 &&
         (reinterpret_cast<uintptr_t>(a.norms_v) & 15u) == 0;
}

template <int D, bool FULL>
int run_split_mma_d(const SplitArgs &a, cudaStream_t st) {
  const int G = a.group;
  if (G == 1 || G == 2 || G == 4) return launch_split_mma<D, FULL, true, 1>(a, st);
  if (G <= 4) return launch_split_mma<D, FULL, false, 1>(a, st);
  return launch_split_mma<D, FULL, false, 2>(a, st);
}

int run_split_mma(int d, int variant, const SplitArgs &a, cudaStream_t st) {
  if (d == 128)
    return variant == ISOQ_FULL ? run_split_mma_d<128, true>(a, st) : run_split_mma_d<128, false>(a, st);
  return variant == ISOQ_FULL ? run_split_mma_d<256, true>(a, st) : run_split_mma_d<256, false>(a, st);
}
