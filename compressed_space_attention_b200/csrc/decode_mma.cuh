// Tensor-core split kernel of the compressed-space decode: float16 queries,
// 3-bit codes, d in {128, 256}, up to 8 query heads per KV head.
// Included by isoq_decode.cu inside namespace isoq::decode.
//
// Per CTA: one (b, kvh, token chunk).  One producer warp streams the chunk's
// packed K/V rows and float16 norms into shared memory with CTA-local bulk
// copies (64 tokens per stage, an mbarrier ring); four consumer warps each
// take a 16-token slab of every stage.
//
// QK (RotaryQuant Table 2 kernel A) runs as mma.sync m16n8k16 with
// A = dequantised K~ [16 tokens x 16 dims] built in registers and
// B = q~ [16 dims x 8 heads] (heads >= G are zero).  PV (kernel C) runs as
// m16n8k16 with A = V~^T [16 dims x 16 tokens] and B = P [16 tokens x 8 heads].
// The online softmax (kernel B) runs on the QK accumulator fragments.
//
// Fragment orders.  A fixed permutation of the rotated coordinates cancels in
// q~.k~ and is undone when the accumulator is written out, and a permutation
// of the tokens inside a slab is applied identically to P and V~; both are
// chosen so that each lane expands whole 24-bit groups of 8 codes:
//   QK: lane (g, t) owns tokens g and g+8 and dims [t d/4, (t+1) d/4); MMA kk
//       uses its dims t d/4 + 4kk + {0,1} (k = 2t, 2t+1) and {2,3} (2t+8, 2t+9).
//   PV: lane (g, t) owns dims [g d/8, (g+1) d/8) (row g of MMA mm is dim
//       g d/8 + 2mm, row g+8 is the next dim) and tokens t, t+4, t+8, t+12
//       (k = 2t, 2t+1, 2t+8, 2t+9).
// Code -> float16 centroid is a byte lookup with prmt: the low and high bytes
// of the 8 centroids sit in two register pairs, a nibble-spread selector picks
// four entries at once, and two more prmt interleave the bytes into half2.

constexpr int kMmaConsumerWarps = 4;
constexpr int kMmaThreads = 32 * (kMmaConsumerWarps + 1);
constexpr int kMmaStageTokens = 16 * kMmaConsumerWarps;
constexpr int kMmaStages = 4;

template <int D>
struct MmaCfg {
  static constexpr int PB = D * 3 / 8;                      // packed bytes per token
  static constexpr int CODES_BYTES = kMmaStageTokens * PB;
  static constexpr int NORM_BYTES = kMmaStageTokens * 2;
  static constexpr int STAGE_BYTES = 2 * CODES_BYTES + 2 * NORM_BYTES;
  static constexpr int KK = D / 16;                         // MMAs along d (QK) / along dims (PV)
  static constexpr int QSEG = D / 4;                        // dims per lane in QK
  static constexpr int VSEG = D / 8;                        // dims per lane in PV
  static constexpr int SCRATCH_FLOATS = 8 * D;              // q~ staging, then the warp merge
  static constexpr int SMEM = kMmaStages * STAGE_BYTES + SCRATCH_FLOATS * 4 +
                              2 * kMmaConsumerWarps * 8 * 4 + 2 * kMmaStages * 8 + 16 + 128;
};

struct MmaLut {
  uint32_t lo0, lo1, hi0, hi1;  // low/high bytes of the 8 float16 centroids (unit variance)
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

// 8 codes of 3 bits (bits 0..23) -> 8 nibbles (code k at bits 4k..4k+2).
__device__ __forceinline__ uint32_t spread3_to_nibbles(uint32_t w) {
  uint32_t x = (w & 0xFFFu) | ((w << 4) & 0x0FFF0000u);
  x = (x & 0x003F003Fu) | ((x << 2) & 0x3F003F00u);
  x = (x & 0x07070707u) | ((x << 1) & 0x70707070u);
  return x;
}

// 4 codes of 3 bits (bits 0..11) -> 4 bytes (code k at bits 8k..8k+2).
__device__ __forceinline__ uint32_t spread3_to_bytes(uint32_t w) {
  uint32_t x = (w & 0x3Fu) | ((w << 10) & 0x003F0000u);
  x = (x & 0x00070007u) | ((x << 5) & 0x07000700u);
  return x;
}

// Two half2 from a 4-nibble selector: (c[s0], c[s1]) and (c[s2], c[s3]).
__device__ __forceinline__ void lut4(const MmaLut &l, uint32_t sel, uint32_t &h01, uint32_t &h23) {
  const uint32_t lo = prmt(l.lo0, l.lo1, sel);
  const uint32_t hi = prmt(l.hi0, l.hi1, sel);
  h01 = prmt(lo, hi, 0x5140u);
  h23 = prmt(lo, hi, 0x7362u);
}

__device__ __forceinline__ uint32_t lds32(const unsigned char *p) {
  return *reinterpret_cast<const uint32_t *>(p);
}

// Loads the 24-bit code group `grp` from a run of 32-bit words.
template <int NW>
__device__ __forceinline__ uint32_t group24(const uint32_t (&w)[NW], int grp) {
  const int bit = 24 * grp;
  const int wi = bit >> 5, sh = bit & 31;
  if (sh == 0) return w[wi];
  return __funnelshift_r(w[wi], (wi + 1 < NW) ? w[wi + 1] : 0u, sh);
}

template <int D, bool FULL>
__global__ void __launch_bounds__(kMmaThreads) split_mma_kernel(const SplitArgs a, const MmaLut lut,
                                                                float qk_scale_log2) {
  using C = MmaCfg<D>;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~static_cast<uintptr_t>(127));
  unsigned char *stages = smem;
  float *scratch = reinterpret_cast<float *>(smem + kMmaStages * C::STAGE_BYTES);
  float *wm = scratch + C::SCRATCH_FLOATS;          // [warps][8]
  float *wl = wm + kMmaConsumerWarps * 8;           // [warps][8]
  uint64_t *full_bar = reinterpret_cast<uint64_t *>(wl + kMmaConsumerWarps * 8);
  uint64_t *empty_bar = full_bar + kMmaStages;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(empty_bar + kMmaStages);

  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.group;

  int T = a.seq_lens[b];
  T = T < 0 ? 0 : (T > a.tmax ? static_cast<int>(a.tmax) : T);
  const long long t0 = static_cast<long long>(split) * a.chunk;
  long long t1 = t0 + a.chunk;
  if (t1 > T) t1 = T;
  const int n_tok = t1 > t0 ? static_cast<int>(t1 - t0) : 0;
  const int n_stages = (n_tok + kMmaStageTokens - 1) / kMmaStageTokens;

  if (tid == 0) {
    for (int s = 0; s < kMmaStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], kMmaConsumerWarps);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  // Rotate the G queries of this KV head once: q~ = R_K q (all threads).
  for (int i = tid; i < 8 * D; i += kMmaThreads) {
    const int g = i / D;
    float v = 0.f;
    if (g < G) {
      const __half *q = static_cast<const __half *>(a.q) +
                        (static_cast<long long>(b) * a.hq + kvh * G + g) * D;
      v = __half2float(q[i % D]);
    }
    scratch[i] = v;
  }
  __syncthreads();
  for (int g = 0; g < G; ++g)
    rotate_forward_cta<D, FULL>(scratch + g * D, a.params_k + static_cast<size_t>(kvh) * 2 * D);

  const long long pair = static_cast<long long>(b) * a.hkv + kvh;

  if (warp == kMmaConsumerWarps) {
    // ---------------- bulk-copy producer ----------------
    if (lane == 0) {
      const uint8_t *kb = a.packed_k + pair * a.tmax * C::PB;
      const uint8_t *vb = a.packed_v + pair * a.tmax * C::PB;
      const uint16_t *nkb = a.norms_k + pair * a.tmax;
      const uint16_t *nvb = a.norms_v + pair * a.tmax;
      int issued = 0;
      for (int i = 0; i < n_stages; ++i) {
        const int s = i % kMmaStages;
        if (!mbar_wait_bounded(&empty_bar[s], ((i / kMmaStages) & 1) ^ 1) || *abort_flag) {
          atomicOr(&g_decode_error, kErrWaitTimeout);
          *abort_flag = 1;
          break;
        }
        const long long t = t0 + static_cast<long long>(i) * kMmaStageTokens;
        int n = n_tok - i * kMmaStageTokens;
        if (n > kMmaStageTokens) n = kMmaStageTokens;
        const int n8 = (n + 7) & ~7;
        unsigned char *st = stages + s * C::STAGE_BYTES;
        mbar_arrive_expect_tx(&full_bar[s], 2u * n * C::PB + 4u * n8);
        bulk_load(st, kb + t * C::PB, n * C::PB, &full_bar[s]);
        bulk_load(st + C::CODES_BYTES, vb + t * C::PB, n * C::PB, &full_bar[s]);
        bulk_load(st + 2 * C::CODES_BYTES, nkb + t, 2 * n8, &full_bar[s]);
        bulk_load(st + 2 * C::CODES_BYTES + C::NORM_BYTES, nvb + t, 2 * n8, &full_bar[s]);
        issued = i + 1;
      }
      for (int i = issued > kMmaStages ? issued - kMmaStages : 0; i < issued; ++i) {
        if (!mbar_wait_bounded(&full_bar[i % kMmaStages], (i / kMmaStages) & 1)) {
          atomicOr(&g_decode_error, kErrWaitTimeout);
          break;
        }
      }
    }
    // The producer warp joins the final merge barrier below.
  } else {
    // ---------------- consumers ----------------
    const int g = lane >> 2, t = lane & 3;

    // B fragments of q~ for QK: head g, dims t*QSEG + 4kk + {0..3}.
    uint32_t qf[C::KK][2];
#pragma unroll
    for (int kk = 0; kk < C::KK; ++kk) {
      const float *src = scratch + g * D + t * C::QSEG + 4 * kk;
      __half2 h0 = __floats2half2_rn(src[0], src[1]);
      __half2 h1 = __floats2half2_rn(src[2], src[3]);
      if (g >= G) h0 = h1 = __floats2half2_rn(0.f, 0.f);
      qf[kk][0] = *reinterpret_cast<uint32_t *>(&h0);
      qf[kk][1] = *reinterpret_cast<uint32_t *>(&h1);
    }

    float acc[C::KK][4];
#pragma unroll
    for (int mm = 0; mm < C::KK; ++mm) acc[mm][0] = acc[mm][1] = acc[mm][2] = acc[mm][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    const uint32_t psel = (g & 1) ? 0x7632u : 0x5410u;
    const int src1 = 4 * t + (g >> 1), src2 = 16 + 4 * t + (g >> 1);

    for (int i = 0; i < n_stages; ++i) {
      const int s = i % kMmaStages;
      if (!mbar_wait_bounded(&full_bar[s], (i / kMmaStages) & 1) || *abort_flag) {
        atomicOr(&g_decode_error, kErrWaitTimeout);
        *abort_flag = 1;
        break;
      }
      int nvalid = n_tok - i * kMmaStageTokens - 16 * warp;
      nvalid = nvalid > 16 ? 16 : nvalid;
      if (nvalid > 0) {
        const unsigned char *st = stages + s * C::STAGE_BYTES;
        const unsigned char *kc = st + (16 * warp) * C::PB;
        const unsigned char *vc = st + C::CODES_BYTES + (16 * warp) * C::PB;
        const __half *nk = reinterpret_cast<const __half *>(st + 2 * C::CODES_BYTES) + 16 * warp;
        const __half *nv = reinterpret_cast<const __half *>(st + 2 * C::CODES_BYTES + C::NORM_BYTES) + 16 * warp;

        // ---- QK: S[16 tokens x 8 heads] ----
        float sc[4] = {0.f, 0.f, 0.f, 0.f};
        {
          constexpr int NW = C::QSEG * 3 / 32;   // words per token segment (3 or 6)
          uint32_t wg[NW], wg8[NW];
          const unsigned char *rg = kc + g * C::PB + t * (C::QSEG * 3 / 8);
          const unsigned char *rg8 = rg + 8 * C::PB;
#pragma unroll
          for (int k = 0; k < NW; ++k) {
            wg[k] = lds32(rg + 4 * k);
            wg8[k] = lds32(rg8 + 4 * k);
          }
#pragma unroll
          for (int grp = 0; grp < C::QSEG / 8; ++grp) {
            const uint32_t na = spread3_to_nibbles(group24(wg, grp));
            const uint32_t nb = spread3_to_nibbles(group24(wg8, grp));
            uint32_t a0, a1, a2, a3;
            lut4(lut, na, a0, a2);
            lut4(lut, nb, a1, a3);
            mma_16816(sc, a0, a1, a2, a3, qf[2 * grp][0], qf[2 * grp][1]);
            lut4(lut, na >> 16, a0, a2);
            lut4(lut, nb >> 16, a1, a3);
            mma_16816(sc, a0, a1, a2, a3, qf[2 * grp + 1][0], qf[2 * grp + 1][1]);
          }
        }

        // ---- online softmax on the fragments (log2 domain) ----
        const bool vg = g < nvalid, vg8 = g + 8 < nvalid;
        const float skg = vg ? __half2float(nk[g]) * qk_scale_log2 : 0.f;
        const float skg8 = vg8 ? __half2float(nk[g + 8]) * qk_scale_log2 : 0.f;
        const float x0 = vg ? sc[0] * skg : -INFINITY;
        const float x1 = vg ? sc[1] * skg : -INFINITY;
        const float x2 = vg8 ? sc[2] * skg8 : -INFINITY;
        const float x3 = vg8 ? sc[3] * skg8 : -INFINITY;
        float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
          mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
        }
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        if (__any_sync(0xffffffffu, (mn0 > m0) || (mn1 > m1))) {
          const float f0 = (m0 == -INFINITY) ? 0.f : exp2f(m0 - mn0);
          const float f1 = (m1 == -INFINITY) ? 0.f : exp2f(m1 - mn1);
#pragma unroll
          for (int mm = 0; mm < C::KK; ++mm) {
            acc[mm][0] *= f0;
            acc[mm][1] *= f1;
            acc[mm][2] *= f0;
            acc[mm][3] *= f1;
          }
          l0 *= f0;
          l1 *= f1;
          m0 = mn0;
          m1 = mn1;
        }
        const float p0 = exp2f(x0 - m0), p1 = exp2f(x1 - m1);
        const float p2 = exp2f(x2 - m0), p3 = exp2f(x3 - m1);
        l0 += p0 + p2;
        l1 += p1 + p3;
        const float svg = vg ? __half2float(nv[g]) : 0.f;
        const float svg8 = vg8 ? __half2float(nv[g + 8]) : 0.f;
        __half2 h01 = __floats2half2_rn(p0 * svg, p1 * svg);
        __half2 h23 = __floats2half2_rn(p2 * svg8, p3 * svg8);
        const uint32_t u01 = *reinterpret_cast<uint32_t *>(&h01);
        const uint32_t u23 = *reinterpret_cast<uint32_t *>(&h23);
        // P fragment for PV: lane (g, t) needs tokens t, t+4, t+8, t+12 of head g.
        const uint32_t x_t = __shfl_sync(0xffffffffu, u01, src1);
        const uint32_t x_t4 = __shfl_sync(0xffffffffu, u01, src2);
        const uint32_t x_t8 = __shfl_sync(0xffffffffu, u23, src1);
        const uint32_t x_t12 = __shfl_sync(0xffffffffu, u23, src2);
        uint32_t pb0 = prmt(x_t, x_t4, psel);
        uint32_t pb1 = prmt(x_t8, x_t12, psel);
        if (g >= G) pb0 = pb1 = 0u;

        // ---- PV: O^T[dims x 8 heads] += V~^T[dims x 16 tokens] P ----
        {
          constexpr int VB = C::VSEG * 3 / 8;     // bytes per token segment (6 or 12)
          constexpr int NW = (VB + 3) / 4 + 1;    // words loaded per token (room for alignment)
          const int off = g * VB;
          const int off4 = off & ~3, sh = (off & 3) * 8;
          uint32_t w[4][NW];
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const unsigned char *row = vc + (t + 4 * r) * C::PB + off4;
#pragma unroll
            for (int k = 0; k < NW; ++k) w[r][k] = (4 * k < VB + (off & 3)) ? lds32(row + 4 * k) : 0u;
            if (sh) {
#pragma unroll
              for (int k = 0; k + 1 < NW; ++k) w[r][k] = __funnelshift_r(w[r][k], w[r][k + 1], sh);
            }
          }
#pragma unroll
          for (int grp = 0; grp < C::VSEG / 8; ++grp) {
            const uint32_t ga = group24(w[0], grp), gb = group24(w[1], grp);
            const uint32_t gc = group24(w[2], grp), gd = group24(w[3], grp);
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {        // dims 0-3, then 4-7 of the group
              const uint32_t sab = spread3_to_bytes(ga >> (12 * hh)) | (spread3_to_bytes(gb >> (12 * hh)) << 4);
              const uint32_t scd = spread3_to_bytes(gc >> (12 * hh)) | (spread3_to_bytes(gd >> (12 * hh)) << 4);
#pragma unroll
              for (int j = 0; j < 2; ++j) {         // dim pairs (0,1), (2,3)
                uint32_t a0, a1, a2, a3;
                lut4(lut, sab >> (16 * j), a0, a1);
                lut4(lut, scd >> (16 * j), a2, a3);
                mma_16816(acc[4 * grp + 2 * hh + j], a0, a1, a2, a3, pb0, pb1);
              }
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[s]);
    }

    // Per-warp totals over the 8 lanes sharing t.
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, o);
      l1 += __shfl_xor_sync(0xffffffffu, l1, o);
    }
    named_barrier(1, 32 * kMmaConsumerWarps);   // all warps are done with the q~ scratch
    for (int i = tid; i < 8 * D; i += 32 * kMmaConsumerWarps) scratch[i] = 0.f;
    if (g == 0) {
      wm[warp * 8 + 2 * t] = m0;
      wm[warp * 8 + 2 * t + 1] = m1;
      wl[warp * 8 + 2 * t] = l0;
      wl[warp * 8 + 2 * t + 1] = l1;
    }
    named_barrier(1, 32 * kMmaConsumerWarps);
    // Merge the warps' states into scratch[head][dim] (rotated domain).
    float f[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int h = 2 * t + e;
      float mstar = -INFINITY;
      for (int w2 = 0; w2 < kMmaConsumerWarps; ++w2) mstar = fmaxf(mstar, wm[w2 * 8 + h]);
      const float mine = wm[warp * 8 + h];
      f[e] = (mine == -INFINITY) ? 0.f : exp2f(mine - mstar);
    }
    if (2 * t < G) {
#pragma unroll
      for (int mm = 0; mm < C::KK; ++mm) {
        const int dim = g * C::VSEG + 2 * mm;
        atomicAdd(&scratch[(2 * t) * D + dim], acc[mm][0] * f[0]);
        atomicAdd(&scratch[(2 * t) * D + dim + 1], acc[mm][2] * f[0]);
        if (2 * t + 1 < G) {
          atomicAdd(&scratch[(2 * t + 1) * D + dim], acc[mm][1] * f[1]);
          atomicAdd(&scratch[(2 * t + 1) * D + dim + 1], acc[mm][3] * f[1]);
        }
      }
    }
  }
  __syncthreads();

  // Write one partial state per query head: natural-log max, sum, acc / sqrt(d).
  const float inv_sqrt_d = rsqrtf(static_cast<float>(D));
  for (int h = 0; h < G; ++h) {
    const long long slot = (static_cast<long long>(b) * a.hq + kvh * G + h) * a.n_splits + split;
    float *acc_out = a.ws_acc + slot * D;
    for (int i = tid; i < D; i += kMmaThreads) acc_out[i] = scratch[h * D + i] * inv_sqrt_d;
    if (tid == 0) {
      float mstar = -INFINITY, l = 0.f;
      for (int w2 = 0; w2 < kMmaConsumerWarps; ++w2) mstar = fmaxf(mstar, wm[w2 * 8 + h]);
      for (int w2 = 0; w2 < kMmaConsumerWarps; ++w2) {
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

template <int D, bool FULL>
int launch_split_mma(const SplitArgs &a, cudaStream_t stream) {
  using C = MmaCfg<D>;
  auto kernel = split_mma_kernel<D, FULL>;
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
  // float16 centroids of the unit-variance codebook (the 1/sqrt(d) of the
  // N(0, 1/d) codebook is folded into the score scale and the output).
  const float sqrt_d = std::sqrt(static_cast<float>(D));
  uint32_t lo[2] = {0, 0}, hi[2] = {0, 0};
  for (int k = 0; k < 8; ++k) {
    const uint32_t hb = half_bits(a.centroid[k] * sqrt_d);
    lo[k / 4] |= (hb & 0xFFu) << (8 * (k % 4));
    hi[k / 4] |= (hb >> 8) << (8 * (k % 4));
  }
  MmaLut lut{lo[0], lo[1], hi[0], hi[1]};
  const float qk_scale_log2 = a.scale / sqrt_d * 1.4426950408889634f;
  dim3 grid(a.n_splits, a.hkv, a.batch);
  kernel<<<grid, kMmaThreads, C::SMEM, stream>>>(a, lut, qk_scale_log2);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(ISOQ_ERR_CUDA, "decode mma launch: %s", cudaGetErrorString(e));
  return ISOQ_OK;
}

bool mma_path_supported(int dtype, int d, int bits, const SplitArgs &a) {
  return dtype == ISOQ_F16 && bits == 3 && (d == 128 || d == 256) && a.group <= 8 &&
         a.tmax % 8 == 0 && a.chunk % kMmaStageTokens == 0 &&
         (reinterpret_cast<uintptr_t>(a.norms_k) & 15u) == 0 &&
         (reinterpret_cast<uintptr_t>(a.norms_v) & 15u) == 0;
}

int run_split_mma(int d, int variant, const SplitArgs &a, cudaStream_t st) {
  if (d == 128)
    return variant == ISOQ_FULL ? launch_split_mma<128, true>(a, st) : launch_split_mma<128, false>(a, st);
  return variant == ISOQ_FULL ? launch_split_mma<256, true>(a, st) : launch_split_mma<256, false>(a, st);
}
