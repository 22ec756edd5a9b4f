// Causal attention of a chunk of Tq new queries over the packed cache
// (chunked prefill), on dense tensor-core tiles.  Included by isoq_decode.cu
// inside namespace isoq::decode, after the rotation helpers.
//
// Query t of batch row b sits at position p = seq_lens[b] - Tq + t and
// attends to the cached tokens j <= p (RotaryQuant §3.4: kernel A with
// causal masking, which ends each query's token loop early; Figure 1's path
// with more than one query).  Everything stays in the rotated domain as in
// the decode: q~ = R_K q once per query, scores against the centroids,
// softmax, V accumulated as centroids, one inverse rotation per output row.
//
// CTA: (query tile, kvh, b), 4 warps, 64 rows = 64 / GP query positions x
// GP heads (row m: position m / GP, head m % GP; heads >= G are dead rows).
// Per 64-token tile the CTA expands the packed K and V codes into float16
// centroids alpha c_k in shared memory (one prmt lookup per byte, four per
// four codes), then each warp runs, for its 16 rows, FlashAttention-style:
//   S = Q~ K~^T  with mma.sync m16n8k16 f16 -> f32, Q~ split into float16
//                hi and lo parts (two MMAs), so the scores keep 22 bits;
//   x = S s^K_j scale / alpha (log2 units), causal mask on diagonal tiles,
//   online softmax in float32 on the accumulator fragments;
//   O += (p s^V_j) V~  with the probabilities reused as A fragments (float16
//                carries each weight with 11 bits of its own magnitude).
// After the last tile the rows are normalised, written to shared memory,
// rotated back (R_V^T) and stored in the query dtype.
//
// Requires float16 queries (the float16 tiles meet the float16 output
// tolerance, not the float32 one), 3-bit codes, d in {128, 256},
// G = Hq / Hkv in {1, 2, 4, 8}, Tmax % 8 == 0 and 16-byte aligned code rows.

constexpr int kPfWarps = 8;
constexpr int kPfThreads = 32 * kPfWarps;
constexpr int kPfRows = 16 * kPfWarps;   // query-head rows per CTA
constexpr int kPfHalf = kPfRows / 2;     // rows per pass of the prep / epilogue scratch
constexpr int kPfTok = 64;               // tokens per K/V tile
constexpr int kPfStages = 2;             // packed-code staging ring

struct PrefillArgs {
  const void *q;                  // [B][Tq][Hq][d]
  const uint8_t *packed_k, *packed_v;
  const uint16_t *norms_k, *norms_v;
  const int32_t *seq_lens;
  const float *params_k, *params_v;
  void *out;                      // [B][Tq][Hq][d], dtype of q
  long long tmax;
  int batch, tq, hq, hkv, group;
  float score_unit;               // scale * log2(e) / (alpha sqrt(d))
  float out_unit;                 // 1 / (alpha * d)
  uint32_t lut_lo0, lut_lo1, lut_hi0, lut_hi1;   // float16 alpha c_k, low / high bytes
};

template <int D>
struct PfCfg {
  static constexpr int PB = D * 3 / 8;                    // packed bytes per token
  static constexpr int CH = D / 8;                        // 16-byte chunks per f16 row
  static constexpr int ROW_BYTES = 2 * D;
  static constexpr int Q_BYTES = kPfRows * ROW_BYTES;     // one of hi / lo
  static constexpr int KV_BYTES = kPfTok * ROW_BYTES;
  static constexpr int NORM_BYTES = 2 * kPfTok * 4;
  // one staging stage: K codes, V codes, K norms, V norms (float16)
  static constexpr int ST_CODES = kPfTok * PB;
  static constexpr int ST_BYTES = 2 * ST_CODES + 2 * kPfTok * 2;
  static constexpr int SCRATCH_BYTES = kPfHalf * D * 4;   // float rows (prep / epilogue)
  static_assert(SCRATCH_BYTES <= 2 * KV_BYTES, "scratch aliases the K/V tiles");
  static constexpr int OFF_KV = 2 * Q_BYTES;
  static constexpr int OFF_NORM = OFF_KV + 2 * KV_BYTES;
  static constexpr int OFF_STAGE = OFF_NORM + NORM_BYTES;
  static constexpr int OFF_BAR = OFF_STAGE + kPfStages * ST_BYTES;
  static constexpr int SMEM = OFF_BAR + 8 * kPfStages + 128;
  static constexpr int NT_S = kPfTok / 8;     // score n-tiles per warp
  static constexpr int NT_O = D / 8;          // output n-tiles per warp
  static constexpr int MIN_BLOCKS = D == 128 ? 2 : 1;
};

// Byte offset of 16-byte chunk c of row r in a swizzled float16 tile.
template <int D>
__device__ __forceinline__ uint32_t pf_off(int r, int c) {
  return static_cast<uint32_t>(r * (2 * D) + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

__device__ __forceinline__ void mma_f16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&h);
}

// Expands the staged packed codes of a tile's tokens (zeros from token
// `nvalid` on) into float16 centroids in a swizzled [token][D] tile.
template <int D>
__device__ __forceinline__ void pf_expand(const unsigned char *codes, int nvalid, unsigned char *tile,
                                          const PrefillArgs &a, int tid) {
  constexpr int GROUPS = D / 32, PB = D * 3 / 8;
  for (int idx = tid; idx < kPfTok * GROUPS; idx += kPfThreads) {
    const int tok = idx / GROUPS, grp = idx - tok * GROUPS;
    uint32_t w0 = 0, w1 = 0, w2 = 0;
    if (tok < nvalid) {
      const unsigned char *src = codes + tok * PB + 12 * grp;
      w0 = lds32(src);
      w1 = lds32(src + 4);
      w2 = lds32(src + 8);
    }
    uint32_t s[8];
    group_sel8(w0, w1, w2, s);
#pragma unroll
    for (int qd = 0; qd < 8; ++qd) {
      const uint32_t lo = prmt(a.lut_lo0, a.lut_lo1, s[qd]);
      const uint32_t hi = prmt(a.lut_hi0, a.lut_hi1, s[qd]);
      const uint2 v = make_uint2(prmt(lo, hi, 0x5140u), prmt(lo, hi, 0x7362u));
      // dims 32 grp + 4 qd .. + 3: chunk (4 grp + qd / 2), half qd & 1
      const int c = 4 * grp + (qd >> 1);
      *reinterpret_cast<uint2 *>(tile + pf_off<D>(tok, c) + 8 * (qd & 1)) = v;
    }
  }
}

// Multi-row inverse rotation H_d R_SO4^T u (unnormalised) of nvec rows in
// shared memory, by the whole CTA.
template <int D, bool FULL>
__device__ void rotate_inverse_rows(float *v, int nvec, const float *params_head, int tid, int nthreads) {
  for (int idx = tid; idx < nvec * (D / 4); idx += nthreads) {
    const int g = idx / (D / 4), bi = idx % (D / 4);
    float *w = v + g * D + 4 * bi;
    const Quat u{w[0], w[1], w[2], w[3]};
    const Quat x = block_inverse(load_quat(params_head + 8 * bi), load_quat(params_head + 8 * bi + 4), u, FULL);
    w[0] = x.w;
    w[1] = x.x;
    w[2] = x.y;
    w[3] = x.z;
  }
  __syncthreads();
#pragma unroll 1
  for (int h = 1; h < D; h <<= 1) {
    for (int idx = tid; idx < nvec * (D / 2); idx += nthreads) {
      const int g = idx / (D / 2), p = idx % (D / 2);
      float *w = v + g * D;
      const int i = (p / h) * 2 * h + (p % h);
      const float x0 = w[i], x1 = w[i + h];
      w[i] = x0 + x1;
      w[i + h] = x0 - x1;
    }
    __syncthreads();
  }
}

template <typename T, int D, bool FULL, int GP>
__global__ void __launch_bounds__(kPfThreads, PfCfg<D>::MIN_BLOCKS) prefill_kernel(const PrefillArgs a) {
  using C = PfCfg<D>;
  constexpr int BQ = kPfRows / GP;     // query positions per CTA
  extern __shared__ __align__(128) unsigned char smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~static_cast<uintptr_t>(127));
  unsigned char *q_hi = smem;
  unsigned char *q_lo = smem + C::Q_BYTES;
  unsigned char *k_tile = smem + C::OFF_KV;
  unsigned char *v_tile = k_tile + C::KV_BYTES;
  float *nk_s = reinterpret_cast<float *>(smem + C::OFF_NORM);     // [kPfTok] s^K score_unit
  float *nv_s = nk_s + kPfTok;                                      // [kPfTok] s^V
  unsigned char *stage = smem + C::OFF_STAGE;
  uint64_t *full_bar = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
  float *scratch = reinterpret_cast<float *>(smem + C::OFF_KV);     // aliases the K/V tiles

  const int qt = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int G = a.group;

  int len = a.seq_lens[b];
  len = len < 0 ? 0 : (len > a.tmax ? static_cast<int>(a.tmax) : len);
  const int pos_base = a.seq_lens[b] - a.tq;       // position of query 0 (may be negative)
  const int tq0 = qt * BQ;                         // first query of the tile
  const int p_first = pos_base + tq0;
  int p_last = pos_base + tq0 + BQ - 1;
  if (tq0 + BQ > a.tq) p_last = pos_base + a.tq - 1;
  int tend = p_last + 1 < len ? p_last + 1 : len;  // tokens any row of the tile may see
  if (tend < 0) tend = 0;
  const int n_tiles = (tend + kPfTok - 1) / kPfTok;

  const long long pair = static_cast<long long>(b) * a.hkv + kvh;
  const uint8_t *kb = a.packed_k + pair * a.tmax * C::PB;
  const uint8_t *vb = a.packed_v + pair * a.tmax * C::PB;
  const uint16_t *nkb = a.norms_k + pair * a.tmax;
  const uint16_t *nvb = a.norms_v + pair * a.tmax;

  // Thread 0 stages tile i's packed codes and norms with bulk copies (norm
  // rows rounded up to 8 tokens: Tmax % 8 == 0 keeps them inside the cache).
  auto issue = [&](int i) {
    const int t0 = i * kPfTok;
    int n = tend - t0;
    n = n > kPfTok ? kPfTok : n;
    const int n8 = (n + 7) & ~7;
    unsigned char *st = stage + (i % kPfStages) * C::ST_BYTES;
    uint64_t *bar = &full_bar[i % kPfStages];
    mbar_arrive_expect_tx(bar, 2u * n * C::PB + 4u * n8);
    bulk_load(st, kb + static_cast<long long>(t0) * C::PB, n * C::PB, bar);
    bulk_load(st + C::ST_CODES, vb + static_cast<long long>(t0) * C::PB, n * C::PB, bar);
    bulk_load(st + 2 * C::ST_CODES, nkb + t0, 2 * n8, bar);
    bulk_load(st + 2 * C::ST_CODES + 2 * kPfTok, nvb + t0, 2 * n8, bar);
  };
  if (tid == 0) {
    for (int k = 0; k < kPfStages; ++k) mbar_init(&full_bar[k], 1);
    mbar_fence_init();
    if (n_tiles > 0) issue(0);
  }

  // ---- prep, in two passes of 64 rows: rotate, split into float16 hi / lo ----
  for (int half = 0; half < 2; ++half) {
    for (int i = tid; i < kPfHalf * D; i += kPfThreads) {
      const int m = half * kPfHalf + i / D, e = i % D;
      const int tl = m / GP, h = m % GP;
      float v = 0.f;
      if (h < G && tq0 + tl < a.tq) {
        const long long row = (static_cast<long long>(b) * a.tq + tq0 + tl) * a.hq + kvh * G + h;
        v = to_f32<T>(static_cast<const T *>(a.q)[row * D + e]);
      }
      scratch[i] = v;
    }
    __syncthreads();
    rotate_forward_smem<D, FULL>(scratch, kPfHalf, a.params_k + static_cast<size_t>(kvh) * 2 * D, tid,
                                 kPfThreads, 0);
    for (int i = tid; i < kPfHalf * C::CH; i += kPfThreads) {
      const int r = i / C::CH, c = i - r * C::CH, m = half * kPfHalf + r;
      uint32_t hv[4], lv[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float x0 = scratch[r * D + 8 * c + 2 * k], x1 = scratch[r * D + 8 * c + 2 * k + 1];
        const __half h0 = __float2half_rn(x0), h1 = __float2half_rn(x1);
        const __half l0 = __float2half_rn(x0 - __half2float(h0)), l1 = __float2half_rn(x1 - __half2float(h1));
        const __half2 hh = __halves2half2(h0, h1), ll = __halves2half2(l0, l1);
        hv[k] = *reinterpret_cast<const uint32_t *>(&hh);
        lv[k] = *reinterpret_cast<const uint32_t *>(&ll);
      }
      *reinterpret_cast<uint4 *>(q_hi + pf_off<D>(m, c)) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
      *reinterpret_cast<uint4 *>(q_lo + pf_off<D>(m, c)) = make_uint4(lv[0], lv[1], lv[2], lv[3]);
    }
    __syncthreads();
  }

  // Positions of this lane's two rows (g, g + 8 of the warp's 16); the
  // warp's smallest position decides whether a tile needs the causal mask.
  const int m0 = 16 * warp + g, m1 = m0 + 8;
  const int pr0 = p_first + m0 / GP, pr1 = p_first + m1 / GP;
  const int pw_min = p_first + (16 * warp) / GP;

  float o[C::NT_O][4];
#pragma unroll
  for (int n = 0; n < C::NT_O; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float mx0 = -INFINITY, mx1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const uint32_t qh_s = smem_u32(q_hi), ql_s = smem_u32(q_lo), k_s = smem_u32(k_tile), v_s = smem_u32(v_tile);

  int consumed = 0;
  bool failed = false;
  for (int it = 0; it < n_tiles; ++it) {
    const int t0 = it * kPfTok;
    const bool ok = mbar_wait_bounded(&full_bar[it % kPfStages], (it / kPfStages) & 1);
    if (__syncthreads_or(!ok)) {   // also: the previous tile's K/V tiles are no longer read
      if (tid == 0) atomicOr(&g_decode_error, kErrWaitTimeout);
      failed = true;
      break;
    }
    consumed = it + 1;
    // The stage of tile it - 1 was expanded before the barrier: refill it.
    if (tid == 0 && it + 1 < n_tiles) {
      fence_proxy_async_smem();
      issue(it + 1);
    }
    const unsigned char *st = stage + (it % kPfStages) * C::ST_BYTES;
    const int nvalid = tend - t0 < kPfTok ? tend - t0 : kPfTok;
    pf_expand<D>(st, nvalid, k_tile, a, tid);
    pf_expand<D>(st + C::ST_CODES, nvalid, v_tile, a, tid);
    if (tid < kPfTok) {
      const bool in = tid < nvalid;
      const unsigned char *nks = st + 2 * C::ST_CODES, *nvs = nks + 2 * kPfTok;
      nk_s[tid] = in ? lds_half(nks + 2 * tid) * a.score_unit : 0.f;
      nv_s[tid] = in ? lds_half(nvs + 2 * tid) : 0.f;
    }
    __syncthreads();

    // ---- S = Q~ K~^T for this warp's 16 rows x 64 tokens ----
    float s[C::NT_S][4];
#pragma unroll
    for (int n = 0; n < C::NT_S; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll 4
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t ah0, ah1, ah2, ah3, al0, al1, al2, al3;
      const int arow = 16 * warp + (lane & 15), achunk = 2 * kk + (lane >> 4);
      ldsm_x4(qh_s + pf_off<D>(arow, achunk), ah0, ah1, ah2, ah3);
      ldsm_x4(ql_s + pf_off<D>(arow, achunk), al0, al1, al2, al3);
#pragma unroll
      for (int np = 0; np < C::NT_S / 2; ++np) {
        uint32_t b0, b1, b2, b3;
        const int brow = 16 * np + (lane & 7) + ((lane >> 4) << 3), bchunk = 2 * kk + ((lane >> 3) & 1);
        ldsm_x4(k_s + pf_off<D>(brow, bchunk), b0, b1, b2, b3);
        mma_f16(s[2 * np], ah0, ah1, ah2, ah3, b0, b1);
        mma_f16(s[2 * np], al0, al1, al2, al3, b0, b1);
        mma_f16(s[2 * np + 1], ah0, ah1, ah2, ah3, b2, b3);
        mma_f16(s[2 * np + 1], al0, al1, al2, al3, b2, b3);
      }
    }

    // ---- scores (log2 units), causal mask, online softmax ----
#pragma unroll
    for (int n = 0; n < C::NT_S; ++n) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float sc = nk_s[8 * n + 2 * t + e];
        s[n][e] *= sc;
        s[n][2 + e] *= sc;
      }
    }
    if (t0 + kPfTok - 1 > pw_min || t0 + kPfTok > tend) {   // warp-uniform
#pragma unroll
      for (int n = 0; n < C::NT_S; ++n) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int j = t0 + 8 * n + 2 * t + e;
          if (j > pr0 || j >= tend) s[n][e] = -INFINITY;
          if (j > pr1 || j >= tend) s[n][2 + e] = -INFINITY;
        }
      }
    }
    float tmx0 = -INFINITY, tmx1 = -INFINITY;
#pragma unroll
    for (int n = 0; n < C::NT_S; ++n) {
      tmx0 = fmaxf(tmx0, fmaxf(s[n][0], s[n][1]));
      tmx1 = fmaxf(tmx1, fmaxf(s[n][2], s[n][3]));
    }
#pragma unroll
    for (int o2 = 1; o2 < 4; o2 <<= 1) {
      tmx0 = fmaxf(tmx0, __shfl_xor_sync(0xffffffffu, tmx0, o2));
      tmx1 = fmaxf(tmx1, __shfl_xor_sync(0xffffffffu, tmx1, o2));
    }
    const float nm0 = fmaxf(mx0, tmx0), nm1 = fmaxf(mx1, tmx1);
    const float base0 = nm0 == -INFINITY ? 0.f : nm0, base1 = nm1 == -INFINITY ? 0.f : nm1;
    const float f0 = ex2f(mx0 - base0), f1 = ex2f(mx1 - base1);   // 0 while mx = -inf
    mx0 = nm0;
    mx1 = nm1;
    l0 *= f0;
    l1 *= f1;
#pragma unroll
    for (int n = 0; n < C::NT_O; ++n) {
      o[n][0] *= f0;
      o[n][1] *= f0;
      o[n][2] *= f1;
      o[n][3] *= f1;
    }
    // p = 2^(x - m); the A fragments of PV carry p s^V_j.
    uint32_t pa[C::NT_S][2];
#pragma unroll
    for (int n = 0; n < C::NT_S; ++n) {
      const float sv0 = nv_s[8 * n + 2 * t], sv1 = nv_s[8 * n + 2 * t + 1];
      const float p00 = ex2f(s[n][0] - base0), p01 = ex2f(s[n][1] - base0);
      const float p10 = ex2f(s[n][2] - base1), p11 = ex2f(s[n][3] - base1);
      l0 += p00 + p01;
      l1 += p10 + p11;
      pa[n][0] = pack_f16x2(p00 * sv0, p01 * sv1);
      pa[n][1] = pack_f16x2(p10 * sv0, p11 * sv1);
    }

    // ---- O += P V~ ----
#pragma unroll
    for (int kt = 0; kt < kPfTok / 16; ++kt) {
      const uint32_t a0 = pa[2 * kt][0], a1 = pa[2 * kt][1], a2 = pa[2 * kt + 1][0], a3 = pa[2 * kt + 1][1];
#pragma unroll
      for (int np = 0; np < C::NT_O / 2; ++np) {
        uint32_t b0, b1, b2, b3;
        const int vrow = 16 * kt + (lane & 7) + (((lane >> 3) & 1) << 3), vchunk = 2 * np + (lane >> 4);
        ldsm_x4_t(v_s + pf_off<D>(vrow, vchunk), b0, b1, b2, b3);
        mma_f16(o[2 * np], a0, a1, a2, a3, b0, b1);
        mma_f16(o[2 * np + 1], a0, a1, a2, a3, b2, b3);
      }
    }
  }
  if (failed) {
    // Let every copy still in flight land before the CTA may exit.
    if (tid == 0)
      for (int k = consumed; k < n_tiles && k < consumed + kPfStages; ++k)
        if (!mbar_wait_bounded(&full_bar[k % kPfStages], (k / kPfStages) & 1)) break;
    return;
  }

  // ---- epilogue, in two passes of 64 rows: normalise, rotate back, store ----
#pragma unroll
  for (int o2 = 1; o2 < 4; o2 <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o2);
  }
  const float inv0 = l0 > 0.f ? a.out_unit / l0 : 0.f, inv1 = l1 > 0.f ? a.out_unit / l1 : 0.f;
  for (int half = 0; half < 2; ++half) {
    __syncthreads();   // the K/V tiles (or the previous pass) are no longer read
    if ((warp >> 2) == half) {
      const int r0 = m0 - half * kPfHalf, r1 = m1 - half * kPfHalf;
#pragma unroll
      for (int n = 0; n < C::NT_O; ++n) {
        scratch[r0 * D + 8 * n + 2 * t] = o[n][0] * inv0;
        scratch[r0 * D + 8 * n + 2 * t + 1] = o[n][1] * inv0;
        scratch[r1 * D + 8 * n + 2 * t] = o[n][2] * inv1;
        scratch[r1 * D + 8 * n + 2 * t + 1] = o[n][3] * inv1;
      }
    }
    __syncthreads();
    rotate_inverse_rows<D, FULL>(scratch, kPfHalf, a.params_v + static_cast<size_t>(kvh) * 2 * D, tid,
                                 kPfThreads);
    for (int i = tid; i < kPfHalf * D; i += kPfThreads) {
      const int m = half * kPfHalf + i / D, e = i % D;
      const int tl = m / GP, h = m % GP;
      if (h < G && tq0 + tl < a.tq) {
        const long long row = (static_cast<long long>(b) * a.tq + tq0 + tl) * a.hq + kvh * G + h;
        static_cast<T *>(a.out)[row * D + e] = from_f32<T>(scratch[i]);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

inline uint16_t pf_half_bits(double v) {
  const __half h = __double2half(v);
  return *reinterpret_cast<const uint16_t *>(&h);
}

// alpha in [1, 2) minimising the largest relative float16 rounding error of
// alpha c_k over the unit-variance 3-bit centroids (searched once).
struct PfTables {
  double alpha;
  uint32_t lo0, lo1, hi0, hi1;
};

inline const PfTables &pf_tables() {
  static PfTables tb;
  static std::once_flag once;
  std::call_once(once, [] {
    double c[8];
    codebook_unit_f64(3, c);
    double best = 1.0, best_err = 1.0;
    const int steps = 1 << 20;
    for (int i = 0; i < steps; ++i) {
      const double al = 1.0 + static_cast<double>(i) / steps;
      double err = 0.0;
      for (int k = 4; k < 8 && err < best_err; ++k) {
        const double v = al * c[k];
        const double r = static_cast<double>(__half2float(__double2half(v)));
        err = std::fmax(err, std::fabs(r - v) / v);
      }
      if (err < best_err) {
        best_err = err;
        best = al;
      }
    }
    tb.alpha = best;
    tb.lo0 = tb.lo1 = tb.hi0 = tb.hi1 = 0;
    for (int k = 0; k < 8; ++k) {
      const uint16_t hb = pf_half_bits(best * c[k]);
      const int sh = 8 * (k % 4);
      (k < 4 ? tb.lo0 : tb.lo1) |= static_cast<uint32_t>(hb & 0xFFu) << sh;
      (k < 4 ? tb.hi0 : tb.hi1) |= static_cast<uint32_t>(hb >> 8) << sh;
    }
  });
  return tb;
}

template <typename T, int D, bool FULL, int GP>
int launch_prefill(PrefillArgs a, cudaStream_t stream) {
  using C = PfCfg<D>;
  auto kernel = prefill_kernel<T, D, FULL, GP>;
  static bool configured = false;
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!configured) {
      cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
      if (e != cudaSuccess) return set_error(ISOQ_ERR_CUDA, "prefill: %s", cudaGetErrorString(e));
      configured = true;
    }
  }
  constexpr int BQ = kPfRows / GP;
  dim3 grid((a.tq + BQ - 1) / BQ, a.hkv, a.batch);
  kernel<<<grid, kPfThreads, C::SMEM, stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(ISOQ_ERR_CUDA, "prefill launch: %s", cudaGetErrorString(e));
  return ISOQ_OK;
}

template <typename T, int D, bool FULL, int GP>
int launch_prefill_tc(const PrefillArgs &a, cudaStream_t stream);

template <typename T, int D, bool FULL>
int run_prefill_g(const PrefillArgs &a, cudaStream_t st) {
  switch (a.group) {
    case 1: return launch_prefill_tc<T, D, FULL, 1>(a, st);
    case 2: return launch_prefill_tc<T, D, FULL, 2>(a, st);
    case 4: return launch_prefill_tc<T, D, FULL, 4>(a, st);
    default: return launch_prefill_tc<T, D, FULL, 8>(a, st);
  }
}

template <typename T>
int run_prefill_t(int d, int variant, const PrefillArgs &a, cudaStream_t st) {
  if (d == 128)
    return variant == ISOQ_FULL ? run_prefill_g<T, 128, true>(a, st) : run_prefill_g<T, 128, false>(a, st);
  return variant == ISOQ_FULL ? run_prefill_g<T, 256, true>(a, st) : run_prefill_g<T, 256, false>(a, st);
}

int run_prefill(int d, int variant, PrefillArgs a, cudaStream_t st) {
  const PfTables &tb = pf_tables();
  a.lut_lo0 = tb.lo0;
  a.lut_lo1 = tb.lo1;
  a.lut_hi0 = tb.hi0;
  a.lut_hi1 = tb.hi1;
  a.out_unit = static_cast<float>(1.0 / (tb.alpha * d));
  a.score_unit = static_cast<float>(a.score_unit / (tb.alpha * std::sqrt(static_cast<double>(d))));
  return run_prefill_t<__half>(d, variant, a, st);
}
