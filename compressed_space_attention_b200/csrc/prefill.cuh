// Causal attention of a chunk of Tq new queries over the packed cache
// (chunked prefill), on the 5th-generation tensor cores (tcgen05 + TMEM).
// Included by isoq_decode.cu inside namespace isoq::decode, after the
// rotation helpers.
//
// Query t of batch row b sits at position p = seq_lens[b] - Tq + t and
// attends to the cached tokens j <= p (RotaryQuant §3.4: kernel A with
// causal masking, which ends each query tile's token loop early; Figure 1's
// path with more than one query).  Everything stays in the rotated domain as
// in the decode: q~ = R_K q once per query, scores against the centroids,
// softmax, V accumulated as centroids, one inverse rotation per output row.
//
// CTA = 128 query-head rows (128 / GP positions x GP heads; heads >= G are
// dead rows), one TMEM lane each, 4 warps; thread r owns row r for the
// softmax (TMEM lane r lies in its warp's sub-partition).  Per 64-token tile:
//   thread 0 has staged the tile's packed codes and norms with bulk copies
//   (2-deep ring); the CTA expands the K codes into float16 centroids
//   alpha c_k (alpha, searched on the host, makes them nearly exact in
//   float16) in a 128B-swizzled tile; one thread issues
//   S = Q~hi K~^T + Q~lo K~^T with tcgen05.mma kind::f16 (M = 128, N = 64;
//   q~ split into float16 hi and lo parts keeps 22-bit scores) into TMEM;
//   after the commit's mbarrier the V codes are expanded into the same tile
//   buffer while each thread reads its S row (tcgen05.ld), scales it by
//   s^K scale / alpha, masks it on diagonal tiles, updates its running
//   maximum and sum, rescales its O row in TMEM when its warp's maximum
//   moved, and writes p s^V as float16 (11 bits of each weight's own
//   magnitude) into a K-major P tile; one thread issues O += P V~ (N = d, V~
//   read MN-major from the same token-row tile).
// The epilogue reads O from TMEM, normalises, rotates back (R_V^T) in shared
// memory and stores float16.
// Operand tiles use the canonical SW128 layouts: rows of 128 bytes (64
// float16), 16-byte chunks XOR-swizzled by (row % 8), 8-row groups 1024
// bytes apart, 64-element blocks of the row direction `blk_stride` apart.
// Every wait is bounded; on a timeout the CTA records kErrWaitTimeout, waits
// (bounded) for its outstanding copies and products, frees its tensor memory
// and returns.
//
// Requires float16 queries (float16 tiles meet the float16 output tolerance,
// not the float32 one), 3-bit codes, d in {128, 256}, G = Hq / Hkv in
// {1, 2, 4, 8}, Tmax % 8 == 0 and 16-byte aligned code rows.

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

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&h);
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

constexpr int kTcThreads = 128;
constexpr int kTcRows = 128;      // M: query-head rows per CTA
constexpr int kTcTok = 64;        // N of QK, K of PV
constexpr int kTcStages = 2;

template <int D>
struct TcCfg {
  static constexpr int PB = D * 3 / 8;
  static constexpr int Q_BYTES = kTcRows * D * 2;         // one of hi / lo
  static constexpr int KV_BYTES = kTcTok * D * 2;         // one tile buffer (K, then V)
  static constexpr int P_BYTES = kTcRows * kTcTok * 2;
  static constexpr int ST_CODES = kTcTok * PB;
  static constexpr int ST_BYTES = 2 * ST_CODES + 2 * kTcTok * 2;
  static constexpr int NORM_BYTES = 2 * kTcTok * 4;
  static constexpr int OFF_QLO = Q_BYTES;
  static constexpr int OFF_KV = 2 * Q_BYTES;
  static constexpr int OFF_P = OFF_KV + KV_BYTES;
  static constexpr int OFF_NORM = OFF_P + P_BYTES;
  static constexpr int OFF_STAGE = OFF_NORM + NORM_BYTES;
  static constexpr int OFF_BAR = OFF_STAGE + kTcStages * ST_BYTES;
  static constexpr int SMEM = OFF_BAR + 8 * (kTcStages + 2) + 16 + 1024;
  static constexpr int TMEM_COLS = D == 128 ? 256 : 512;     // S (64) + O (D), rounded to a power of 2
  static constexpr int MIN_BLOCKS = D == 128 ? 2 : 1;
  static_assert(32 * D * 4 <= KV_BYTES + P_BYTES, "prep scratch (32 rows) fits the K/V and P buffers");
  static_assert(SMEM <= 232448, "shared memory");
};

__host__ __device__ __forceinline__ uint32_t tc_off(int r, int e, int blk_stride) {
  return static_cast<uint32_t>((e >> 6) * blk_stride + (r >> 3) * 1024 + (r & 7) * 128 +
                               ((((e & 63) >> 3) ^ (r & 7)) << 4) + (e & 7) * 2);
}

__device__ __forceinline__ uint64_t tc_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// kind::f16 instruction descriptor: D float32, A and B float16, A K-major,
// B K-major (b_mn = 0) or MN-major (1), M x N.
__host__ __device__ constexpr uint32_t tc_idesc(int M, int N, int b_mn) {
  return (1u << 4) | (static_cast<uint32_t>(b_mn) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint64_t ad, uint64_t bd, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
      ::"r"(tmem_d), "l"(ad), "l"(bd), "r"(idesc), "r"(acc), "r"(0), "r"(0), "r"(0), "r"(0));
}

__device__ __forceinline__ void tc_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
}

__device__ __forceinline__ void tc_st16(uint32_t taddr, const float (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
      ::"r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15]))
      : "memory");
}

// Staged codes of a tile's tokens (zeros from token nvalid on) -> float16
// centroids in the SW128 token-row layout (64-dim blocks KV_BYTES / (D/64)
// apart); the same layout serves K (K-major B of QK) and V (MN-major B of PV).
template <int D>
__device__ __forceinline__ void tc_expand(const unsigned char *codes, int nvalid, unsigned char *tile,
                                          const PrefillArgs &a, int tid) {
  constexpr int GROUPS = D / 32, PB = D * 3 / 8, BLK = kTcTok * 128;
  for (int idx = tid; idx < kTcTok * GROUPS; idx += kTcThreads) {
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
      *reinterpret_cast<uint2 *>(tile + tc_off(tok, 32 * grp + 4 * qd, BLK)) = v;   // dims 32 grp + 4 qd .. + 3
    }
  }
}

template <typename T, int D, bool FULL, int GP>
__global__ void __launch_bounds__(kTcThreads, TcCfg<D>::MIN_BLOCKS) prefill_tc_kernel(const PrefillArgs a) {
  using C = TcCfg<D>;
  constexpr int BQ = kTcRows / GP;
  constexpr int QBLK = kTcRows * 128, KBLK = kTcTok * 128;
  extern __shared__ unsigned char smem_raw[];
  // Aligned by an offset from the shared array itself (not through an
  // integer cast), so the compiler keeps the shared address space.
  unsigned char *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023u)) & 1023u);
  unsigned char *q_hi = smem, *q_lo = smem + C::OFF_QLO;
  unsigned char *kv = smem + C::OFF_KV, *pt = smem + C::OFF_P;
  float *nk_s = reinterpret_cast<float *>(smem + C::OFF_NORM), *nv_s = nk_s + kTcTok;
  unsigned char *stage = smem + C::OFF_STAGE;
  uint64_t *full_bar = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
  uint64_t *bar_s = full_bar + kTcStages, *bar_o = bar_s + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_o + 1);
  float *scratch = reinterpret_cast<float *>(kv);   // 32 rows x D floats over the K/V and P buffers

  const int qt = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int G = a.group;

  int len = a.seq_lens[b];
  len = len < 0 ? 0 : (len > a.tmax ? static_cast<int>(a.tmax) : len);
  const int pos_base = a.seq_lens[b] - a.tq;
  const int tq0 = qt * BQ;
  const int p_first = pos_base + tq0;
  int p_last = pos_base + tq0 + BQ - 1;
  if (tq0 + BQ > a.tq) p_last = pos_base + a.tq - 1;
  int tend = p_last + 1 < len ? p_last + 1 : len;
  if (tend < 0) tend = 0;
  const int n_tiles = (tend + kTcTok - 1) / kTcTok;

  const long long pair = static_cast<long long>(b) * a.hkv + kvh;
  const uint8_t *kb = a.packed_k + pair * a.tmax * C::PB;
  const uint8_t *vb = a.packed_v + pair * a.tmax * C::PB;
  const uint16_t *nkb = a.norms_k + pair * a.tmax;
  const uint16_t *nvb = a.norms_v + pair * a.tmax;

  auto issue = [&](int i) {
    const int t0 = i * kTcTok;
    int n = tend - t0;
    n = n > kTcTok ? kTcTok : n;
    const int n8 = (n + 7) & ~7;
    unsigned char *st = stage + (i % kTcStages) * C::ST_BYTES;
    uint64_t *bar = &full_bar[i % kTcStages];
    mbar_arrive_expect_tx(bar, 2u * n * C::PB + 4u * n8);
    bulk_load(st, kb + static_cast<long long>(t0) * C::PB, n * C::PB, bar);
    bulk_load(st + C::ST_CODES, vb + static_cast<long long>(t0) * C::PB, n * C::PB, bar);
    bulk_load(st + 2 * C::ST_CODES, nkb + t0, 2 * n8, bar);
    bulk_load(st + 2 * C::ST_CODES + 2 * kTcTok, nvb + t0, 2 * n8, bar);
  };

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(C::TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (tid == 0) {
    for (int k = 0; k < kTcStages; ++k) mbar_init(&full_bar[k], 1);
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    mbar_fence_init();
    if (n_tiles > 0) issue(0);
  }

  // ---- prep, 32 rows per pass: rotate, split into float16 hi / lo (SW128 K-major) ----
  for (int pass = 0; pass < kTcRows / 32; ++pass) {
    for (int i = tid; i < 32 * D; i += kTcThreads) {
      const int m = 32 * pass + i / D, e = i % D;
      const int tl = m / GP, h = m % GP;
      float v = 0.f;
      if (h < G && tq0 + tl < a.tq) {
        const long long row = (static_cast<long long>(b) * a.tq + tq0 + tl) * a.hq + kvh * G + h;
        v = to_f32<T>(static_cast<const T *>(a.q)[row * D + e]);
      }
      scratch[i] = v;
    }
    __syncthreads();
    rotate_forward_smem<D, FULL>(scratch, 32, a.params_k + static_cast<size_t>(kvh) * 2 * D, tid, kTcThreads, 0);
    for (int i = tid; i < 32 * (D / 8); i += kTcThreads) {
      const int r = i / (D / 8), c = i % (D / 8), m = 32 * pass + r;
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
      *reinterpret_cast<uint4 *>(q_hi + tc_off(m, 8 * c, QBLK)) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
      *reinterpret_cast<uint4 *>(q_lo + tc_off(m, 8 * c, QBLK)) = make_uint4(lv[0], lv[1], lv[2], lv[3]);
    }
    __syncthreads();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_s = tmem, t_o = tmem + 64;                 // S columns [0, 64), O columns [64, 64 + D)
  const uint32_t lane_off = static_cast<uint32_t>(32 * warp) << 16;

  const int r = tid;                                          // this thread's row / TMEM lane
  const int pr = p_first + r / GP;
  const int pw_min = p_first + (32 * warp) / GP;
  float mx = -INFINITY, l = 0.f;
  const uint32_t qh_s = smem_u32(q_hi), ql_s = smem_u32(q_lo), kv_s = smem_u32(kv), p_s = smem_u32(pt);

  bool failed = false;
  int consumed = 0, s_done = 0, o_done = 0, o_issued = 0;
  for (int it = 0; it < n_tiles; ++it) {
    const int t0 = it * kTcTok;
    // Staged codes of this tile, and the previous PV product (it reads the
    // tile buffer and P) must be complete.
    bool ok = mbar_wait_bounded(&full_bar[it % kTcStages], (it / kTcStages) & 1);
    if (ok && o_issued > o_done) {
      ok = mbar_wait_bounded(bar_o, o_done & 1);
      if (ok) ++o_done;
    }
    if (__syncthreads_or(!ok)) {
      failed = true;
      break;
    }
    tc_fence_after();
    consumed = it + 1;
    if (tid == 0 && it + 1 < n_tiles) {
      fence_proxy_async_smem();
      issue(it + 1);
    }
    const unsigned char *st = stage + (it % kTcStages) * C::ST_BYTES;
    const int nvalid = tend - t0 < kTcTok ? tend - t0 : kTcTok;
    tc_expand<D>(st, nvalid, kv, a, tid);
    if (tid < kTcTok) {
      const bool in = tid < nvalid;
      const unsigned char *nks = st + 2 * C::ST_CODES, *nvs = nks + 2 * kTcTok;
      nk_s[tid] = in ? lds_half(nks + 2 * tid) * a.score_unit : 0.f;
      nv_s[tid] = in ? lds_half(nvs + 2 * tid) : 0.f;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
      constexpr uint32_t idesc = tc_idesc(kTcRows, kTcTok, 0);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t ko = (ks >> 2) * KBLK + (ks & 3) * 32, qo = (ks >> 2) * QBLK + (ks & 3) * 32;
        const uint64_t bd = tc_desc(kv_s + ko, 16, 1024);
        tc_mma(t_s, tc_desc(qh_s + qo, 16, 1024), bd, idesc, ks > 0 ? 1u : 0u);
        tc_mma(t_s, tc_desc(ql_s + qo, 16, 1024), bd, idesc, 1u);
      }
      tc_commit(bar_s);
    }
    ok = mbar_wait_bounded(bar_s, s_done & 1);
    if (__syncthreads_or(!ok)) {
      failed = true;
      break;
    }
    ++s_done;
    tc_fence_after();

    // V codes into the tile buffer (the QK product no longer reads it).
    tc_expand<D>(st + C::ST_CODES, nvalid, kv, a, tid);

    // ---- softmax on this thread's row ----
    float x[64];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float v[16];
      tc_ld16(t_s + lane_off + 16 * c, v);
#pragma unroll
      for (int j = 0; j < 16; ++j) x[16 * c + j] = v[j] * nk_s[16 * c + j];
    }
    if (t0 + kTcTok - 1 > pw_min || t0 + kTcTok > tend) {   // warp-uniform
#pragma unroll
      for (int j = 0; j < 64; ++j)
        if (t0 + j > pr || t0 + j >= tend) x[j] = -INFINITY;
    }
    float tmx = -INFINITY;
#pragma unroll
    for (int j = 0; j < 64; ++j) tmx = fmaxf(tmx, x[j]);
    const float nm = fmaxf(mx, tmx);
    const float base = nm == -INFINITY ? 0.f : nm;
    const float f = ex2f(mx - base);                            // 0 while mx = -inf
    if (__any_sync(0xffffffffu, nm > mx) && it > 0) {
      // rescale this warp's O rows in tensor memory (the last PV product is complete)
#pragma unroll 1
      for (int c = 0; c < D / 16; ++c) {
        float v[16];
        tc_ld16(t_o + lane_off + 16 * c, v);
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] *= f;
        tc_st16(t_o + lane_off + 16 * c, v);
      }
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
    }
    mx = nm;
    l *= f;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      uint32_t w[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int j = 8 * c + 2 * k;
        const float p0 = ex2f(x[j] - base), p1 = ex2f(x[j + 1] - base);
        l += p0 + p1;
        w[k] = pack_f16x2(p0 * nv_s[j], p1 * nv_s[j + 1]);
      }
      *reinterpret_cast<uint4 *>(pt + tc_off(r, 8 * c, 0)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
      constexpr uint32_t idesc = tc_idesc(kTcRows, D, 1);
#pragma unroll
      for (int ks = 0; ks < kTcTok / 16; ++ks)
        tc_mma(t_o, tc_desc(p_s + ks * 32, 16, 1024), tc_desc(kv_s + ks * 2048, KBLK, 1024), idesc,
               (it > 0 || ks > 0) ? 1u : 0u);
      tc_commit(bar_o);
    }
    ++o_issued;
  }

  if (!failed && o_issued > o_done) {
    const bool ok = mbar_wait_bounded(bar_o, o_done & 1);
    if (__syncthreads_or(!ok))
      failed = true;
    else
      ++o_done;
  }
  if (failed) {
    if (tid == 0) {
      atomicOr(&g_decode_error, kErrWaitTimeout);
      for (int k = consumed; k < n_tiles && k < consumed + kTcStages; ++k)
        if (!mbar_wait_bounded(&full_bar[k % kTcStages], (k / kTcStages) & 1)) break;
      if (o_issued > o_done) mbar_wait_bounded(bar_o, o_done & 1);
    }
  } else {
    // ---- epilogue, 32 rows per pass: O / l from TMEM, rotate back, store ----
    tc_fence_after();
    const float inv = l > 0.f ? a.out_unit / l : 0.f;
    for (int pass = 0; pass < kTcRows / 32; ++pass) {
      __syncthreads();   // scratch (over the K/V and P buffers) is free
      if (warp == pass) {
#pragma unroll 1
        for (int c = 0; c < D / 16; ++c) {
          float v[16];
          if (n_tiles > 0) {
            tc_ld16(t_o + lane_off + 16 * c, v);
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = 0.f;
          }
#pragma unroll
          for (int j = 0; j < 16; ++j) scratch[(r - 32 * pass) * D + 16 * c + j] = v[j] * inv;
        }
      }
      __syncthreads();
      rotate_inverse_rows<D, FULL>(scratch, 32, a.params_v + static_cast<size_t>(kvh) * 2 * D, tid, kTcThreads);
      for (int i = tid; i < 32 * D; i += kTcThreads) {
        const int m = 32 * pass + i / D, e = i % D;
        const int tl = m / GP, h = m % GP;
        if (h < G && tq0 + tl < a.tq) {
          const long long row = (static_cast<long long>(b) * a.tq + tq0 + tl) * a.hq + kvh * G + h;
          static_cast<T *>(a.out)[row * D + e] = from_f32<T>(scratch[i]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::TMEM_COLS));
}

template <typename T, int D, bool FULL, int GP>
int launch_prefill_tc(const PrefillArgs &a, cudaStream_t stream) {
  using C = TcCfg<D>;
  auto kernel = prefill_tc_kernel<T, D, FULL, GP>;
  static bool configured = false;
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!configured) {
      cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
      if (e != cudaSuccess) return set_error(ISOQ_ERR_CUDA, "prefill (tcgen05): %s", cudaGetErrorString(e));
      configured = true;
    }
  }
  constexpr int BQ = kTcRows / GP;
  dim3 grid((a.tq + BQ - 1) / BQ, a.hkv, a.batch);
  kernel<<<grid, kTcThreads, C::SMEM, stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(ISOQ_ERR_CUDA, "prefill (tcgen05) launch: %s", cudaGetErrorString(e));
  return ISOQ_OK;
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
