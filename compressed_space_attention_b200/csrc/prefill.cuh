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
// dead rows), one TMEM lane each, 8 warps: warps w and w + 4 share TMEM
// sub-partition w (lanes 32 w .. + 31) and split each row's S and O columns
// in halves.  Per 64-token tile j, software-pipelined by one product:
//   the packed codes and norms of the next tiles are loaded into registers
//   one phase ahead; the CTA expands K tile j + 1's codes into float16
//   centroids alpha c_k in a 128B-swizzled tile, and their float16
//   residuals alpha c_k - fp16(alpha c_k) into a second tile (alpha is
//   searched on the host; the residuals are below 2^-15 of the centroids,
//   so hi + lo keeps them to about 2^-26), and one thread issues
//   S(j + 1) = Q~hi K~hi^T + Q~lo K~hi^T + Q~hi K~lo^T (tcgen05.mma
//   kind::f16, M = 128, N = 64; q~ split into float16 hi and lo parts) into
//   the other of two TMEM S buffers, so it runs under the softmax of tile j;
//   each thread reads its half row of S(j) (tcgen05.ld), scales it by
//   s^K scale / alpha, masks it on diagonal tiles, exchanges its half-row
//   maximum with the partner warp through the consumed S buffer, writes
//   P = p s^V as float16 hi and lo parts (22 bits of each weight) over that
//   S buffer in TMEM and, when its warp's maximum moved, rescales its half
//   of the O row in TMEM; the CTA expands V tile j into its own tile buffer
//   and one thread issues O += P_hi V~ + P_lo V~ (A = P from tensor memory,
//   N = d, V~ read MN-major from the token-row tile).  The next product into
//   that S buffer (QK of tile j + 2) is issued after the PV product, and the
//   tensor core runs one CTA's products in issue order.
// Both the hi/lo query and the hi/lo centroid residual are needed for the
// float16 output bar on outlier-heavy K/V: float16 centroids alone (relative
// error 1.9e-5) or float16 weights alone (2^-12) move scores or weights
// enough to shift outputs of magnitude 30-80 by several 1e-3.
// d = 128 fits two CTAs per SM (one CTA's thread work runs under the
// other's products); d = 256 one.
// The epilogue reads O from TMEM, normalises, rotates back (R_V^T) in shared
// memory and stores float16.
// Operand tiles use the canonical SW128 layouts: rows of 128 bytes (64
// float16), 16-byte chunks XOR-swizzled by (row % 8), 8-row groups 1024
// bytes apart, 64-element blocks of the row direction `blk_stride` apart.
// Every wait is bounded; on a timeout the CTA records kErrWaitTimeout, waits
// (bounded) for its outstanding products, frees its tensor memory and
// returns.
//
// Requires float16 queries (float16 tiles meet the float16 output tolerance,
// not the float32 one), 3-bit codes, d in {128, 256}, G = Hq / Hkv in
// {1, 2, 4, 8}, Tmax % 8 == 0 and 16-byte aligned code rows.

// The prefill kernel found its dynamic shared memory off a 1024-byte
// boundary (its two-CTAs-per-SM layout keeps no slack to align it) and
// returned without writing its output.
constexpr unsigned kErrSmemAlign = 4u;

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
  uint32_t res_lo0, res_lo1, res_hi0, res_hi1;   // float16 alpha c_k - fp16(alpha c_k), low / high bytes
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

constexpr int kTcThreads = 256;   // 8 warps: two per TMEM sub-partition, one per column half
constexpr int kTcRows = 128;      // M: query-head rows per CTA
constexpr int kTcTok = 64;        // N of QK, K of PV

template <int D>
struct TcCfg {
  static constexpr int PB = D * 3 / 8;
  static constexpr int ITEMS = kTcTok * (D / 32) / kTcThreads;   // 32-code groups per thread per tile
  static constexpr int Q_BYTES = kTcRows * D * 2;         // one of hi / lo
  static constexpr int KV_BYTES = kTcTok * D * 2;         // one K, K-residual or V tile
  static constexpr int NORM_BYTES = 2 * kTcTok * 4;       // s^K score_unit, s^V of one tile
  static constexpr int OFF_QLO = Q_BYTES;
  static constexpr int OFF_K = 2 * Q_BYTES;
  static constexpr int OFF_KLO = OFF_K + KV_BYTES;
  static constexpr int OFF_V = OFF_KLO + KV_BYTES;
  static constexpr int OFF_NORM = OFF_V + KV_BYTES;
  static constexpr int OFF_BAR = OFF_NORM + NORM_BYTES;
  // Two CTAs per SM at d = 128 (the second CTA's softmax and expansion run
  // under the first one's products).  Their layout leaves no room to align
  // the dynamic shared memory by hand: the kernel checks that it starts on a
  // 1024-byte boundary and reports kErrSmemAlign otherwise.
  static constexpr int MIN_BLOCKS = D == 128 ? 2 : 1;
  static constexpr int SLACK = MIN_BLOCKS == 2 ? 0 : 1024;
  static constexpr int SMEM = OFF_BAR + 8 * 3 + 8 + SLACK;
  static constexpr int TMEM_COLS = D == 128 ? 256 : 512;     // S (2 x 64) + O (D), rounded to a power of 2
  static_assert(32 * D * 4 <= 2 * KV_BYTES, "prep scratch (32 rows) fits the K and K-residual tiles");
  static_assert(MIN_BLOCKS * (SMEM + 1024) <= 233472, "shared memory per SM (1 KB reserved per CTA)");
  static_assert(MIN_BLOCKS * TMEM_COLS <= 512, "tensor memory columns");
};

// Packed codes of one tile, this thread's share (ITEMS 32-code groups),
// loaded from global memory one phase before they are expanded.
template <int D>
struct TcCodes {
  uint32_t w[TcCfg<D>::ITEMS][3];
};

template <int D>
__device__ __forceinline__ void tc_fetch(TcCodes<D> &c, const uint8_t *base, int t0, int tend, int tid) {
  constexpr int GROUPS = D / 32, PB = D * 3 / 8;
#pragma unroll
  for (int k = 0; k < TcCfg<D>::ITEMS; ++k) {
    const int idx = tid + k * kTcThreads, tok = idx / GROUPS, grp = idx % GROUPS;
    if (t0 + tok < tend) {
      const uint32_t *src = reinterpret_cast<const uint32_t *>(base + static_cast<long long>(t0 + tok) * PB + 12 * grp);
      c.w[k][0] = __ldg(src);
      c.w[k][1] = __ldg(src + 1);
      c.w[k][2] = __ldg(src + 2);
    } else {
      c.w[k][0] = c.w[k][1] = c.w[k][2] = 0u;
    }
  }
}

// Fetched codes -> float16 centroids alpha c_k in the SW128 token-row tile
// (64-dim blocks kTcTok * 128 bytes apart); the same layout serves K (K-major
// B of QK) and V (MN-major B of PV).  With RES, the float16 residuals
// alpha c_k - fp16(alpha c_k) go to a second tile of the same layout.
template <int D, bool RES>
__device__ __forceinline__ void tc_expand(const TcCodes<D> &c, unsigned char *tile, unsigned char *tile_res,
                                          const PrefillArgs &a, int tid) {
  constexpr int GROUPS = D / 32, BLK = kTcTok * 128;
#pragma unroll
  for (int k = 0; k < TcCfg<D>::ITEMS; ++k) {
    const int idx = tid + k * kTcThreads, tok = idx / GROUPS, grp = idx % GROUPS;
    uint32_t s[8];
    group_sel8(c.w[k][0], c.w[k][1], c.w[k][2], s);
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      uint32_t v[4], r[4];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const uint32_t lo = prmt(a.lut_lo0, a.lut_lo1, s[2 * m + u]);
        const uint32_t hi = prmt(a.lut_hi0, a.lut_hi1, s[2 * m + u]);
        v[2 * u] = prmt(lo, hi, 0x5140u);
        v[2 * u + 1] = prmt(lo, hi, 0x7362u);
        if constexpr (RES) {
          const uint32_t rlo = prmt(a.res_lo0, a.res_lo1, s[2 * m + u]);
          const uint32_t rhi = prmt(a.res_hi0, a.res_hi1, s[2 * m + u]);
          r[2 * u] = prmt(rlo, rhi, 0x5140u);
          r[2 * u + 1] = prmt(rlo, rhi, 0x7362u);
        }
      }
      // dims 32 grp + 8 m .. + 7, as two 8-byte stores (measured faster
      // here than one 16-byte store, despite the latter's fewer bank conflicts)
      *reinterpret_cast<uint2 *>(tile + tc_off(tok, 32 * grp + 8 * m, BLK)) = make_uint2(v[0], v[1]);
      *reinterpret_cast<uint2 *>(tile + tc_off(tok, 32 * grp + 8 * m + 4, BLK)) = make_uint2(v[2], v[3]);
      if constexpr (RES) {
        *reinterpret_cast<uint2 *>(tile_res + tc_off(tok, 32 * grp + 8 * m, BLK)) = make_uint2(r[0], r[1]);
        *reinterpret_cast<uint2 *>(tile_res + tc_off(tok, 32 * grp + 8 * m + 4, BLK)) = make_uint2(r[2], r[3]);
      }
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
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  if (pad > static_cast<uint32_t>(C::SLACK)) {   // uniform over the grid: nothing allocated yet
    if (threadIdx.x == 0) atomicOr(&g_decode_error, kErrSmemAlign);
    return;
  }
  unsigned char *smem = smem_raw + pad;
  unsigned char *q_hi = smem, *q_lo = smem + C::OFF_QLO;
  unsigned char *kt = smem + C::OFF_K, *klt = smem + C::OFF_KLO, *vt = smem + C::OFF_V;
  float *nrm_s = reinterpret_cast<float *>(smem + C::OFF_NORM);   // [2][kTcTok] s^K score_unit, s^V of the tile in the softmax
  uint64_t *bar_s = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);   // [2]: S buffer b's product done
  uint64_t *bar_o = bar_s + 2;                                          // PV product done
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_o + 1);
  // A product wait that gave up in iteration j sets fail_s[j % 2]; it is read
  // after the iteration's last block barrier (see the loop).
  volatile uint8_t *fail_s = reinterpret_cast<volatile uint8_t *>(tmem_slot + 1);
  float *scratch = reinterpret_cast<float *>(kt);   // 32 rows x D floats over the K tiles (prep, epilogue)

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

  // Codes and norms of upcoming tiles, one phase ahead, in registers:
  // kc = the next K tile to expand, vc = the next V tile, nrm = the norm
  // (K for tid < 64, V for tid < 128) of the next tile to enter the softmax.
  TcCodes<D> kc, vc;
  uint16_t nrm = 0;
  auto fetch_norm = [&](int j) {
    const int t0 = j * kTcTok, tok = tid & (kTcTok - 1);
    nrm = (tid < 2 * kTcTok && t0 + tok < tend) ? __ldg(((tid < kTcTok) ? nkb : nvb) + t0 + tok)
                                                : static_cast<uint16_t>(0);
  };
  if (n_tiles > 0) {
    tc_fetch<D>(kc, kb, 0, tend, tid);
    tc_fetch<D>(vc, vb, 0, tend, tid);
    fetch_norm(0);
  }

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(C::TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (tid == 0) {
    mbar_init(&bar_s[0], 1);
    mbar_init(&bar_s[1], 1);
    mbar_init(bar_o, 1);
    fail_s[0] = fail_s[1] = 0;
    mbar_fence_init();
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
  const uint32_t t_o = tmem + 128;                           // S buffers at columns [0, 64), [64, 128); O after
  // Warp w reads TMEM lanes 32 (w % 4) .. + 31 (its sub-partition) and
  // handles column half w / 4 of those rows' S and O.
  const int sub = warp & 3, half = warp >> 2, lane = tid & 31;
  const uint32_t lane_off = static_cast<uint32_t>(32 * sub) << 16;
  const uint32_t qh_s = smem_u32(q_hi), ql_s = smem_u32(q_lo), k_s = smem_u32(kt), kl_s = smem_u32(klt),
                 v_s = smem_u32(vt);

  // Expands K tile j (codes and norms from the registers), then issues its QK
  // product into S buffer j % 2.  The caller has made sure the K tile and
  // that S buffer are free.
  auto store_norm = [&]() {
    if (tid < 2 * kTcTok) nrm_s[tid] = __half2float(__ushort_as_half(nrm)) * (tid < kTcTok ? a.score_unit : 1.f);
  };
  auto stage_qk = [&](int j) {
    tc_expand<D, true>(kc, kt, klt, a, tid);
    if (j + 1 < n_tiles) tc_fetch<D>(kc, kb, (j + 1) * kTcTok, tend, tid);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
      constexpr uint32_t idesc = tc_idesc(kTcRows, kTcTok, 0);
      const uint32_t t_s = tmem + (j & 1) * 64;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t ko = (ks >> 2) * KBLK + (ks & 3) * 32, qo = (ks >> 2) * QBLK + (ks & 3) * 32;
        const uint64_t bd = tc_desc(k_s + ko, 16, 1024), ad = tc_desc(qh_s + qo, 16, 1024);
        tc_mma(t_s, ad, bd, idesc, ks > 0 ? 1u : 0u);
        tc_mma(t_s, tc_desc(ql_s + qo, 16, 1024), bd, idesc, 1u);
        tc_mma(t_s, ad, tc_desc(kl_s + ko, 16, 1024), idesc, 1u);
      }
      tc_commit(&bar_s[j & 1]);
    }
  };

  const int r = 32 * sub + lane;                              // this thread's row / TMEM lane
  const int pr = p_first + r / GP;
  const int pw_min = p_first + (32 * sub) / GP;
  constexpr int HC = kTcTok / 2;                               // score columns per thread
  constexpr int OH = D / 2;                                    // output columns per thread
  float mx = -INFINITY;
  uint64_t l2 = f2_pack(0.f, 0.f);                             // running row sum, two partial lanes
  bool failed = false;
  int qk_issued = 0, qk_done = 0, o_issued = 0, o_done = 0;

  if (n_tiles > 0) {
    store_norm();
    if (n_tiles > 1) fetch_norm(1);
    stage_qk(0);
    ++qk_issued;
  }
  for (int it = 0; it < n_tiles; ++it) {
    const int t0 = it * kTcTok;
    // QK(it) must be complete: its S buffer is read below and the K tile is
    // free.  Every thread waits on the mbarrier itself, so no block barrier
    // follows: a wait that gave up is recorded in fail_s[it % 2], which all
    // threads read after the block barrier that ends the iteration and leave
    // the loop together.  (A flag per iteration parity: the writes of
    // iteration it + 2 come after every thread has passed the barrier that
    // ends iteration it + 1, i.e. after every read of iteration it.)
    if (mbar_wait_bounded(&bar_s[it & 1], (it >> 1) & 1))
      ++qk_done;
    else
      fail_s[it & 1] = 1;
    tc_fence_after();
    // The next tile's QK runs on the tensor cores under this tile's softmax.
    // Its block barrier also publishes this tile's norms, stored after the
    // previous iteration's last barrier; the last tile needs a barrier of
    // its own for that.
    if (it + 1 < n_tiles) {
      stage_qk(it + 1);
      ++qk_issued;
    } else {
      __syncthreads();
    }

    // ---- softmax on this thread's half row of S(it) ----
    // Arithmetic on float pairs (f32x2: one instruction per two columns);
    // the norms are read as 16-byte broadcasts.
    const ulonglong2 *nk4 = reinterpret_cast<const ulonglong2 *>(nrm_s + HC * half);
    const ulonglong2 *nv4 = reinterpret_cast<const ulonglong2 *>(nrm_s + kTcTok + HC * half);
    const int c0 = t0 + HC * half;                             // token of this thread's first column
    float x[HC];
    uint32_t sraw[HC / 16][16];
#pragma unroll
    for (int c = 0; c < HC / 16; ++c) tc_ld16_nowait(tmem + (it & 1) * 64 + HC * half + lane_off + 16 * c, sraw[c]);
    tc_wait_ld();
#pragma unroll
    for (int c = 0; c < HC / 16; ++c) {
      float v[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(sraw[c][j]);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const ulonglong2 n = nk4[4 * c + k];
        f2_unpack(f2_mul(f2_pack(v[4 * k], v[4 * k + 1]), n.x), x[16 * c + 4 * k], x[16 * c + 4 * k + 1]);
        f2_unpack(f2_mul(f2_pack(v[4 * k + 2], v[4 * k + 3]), n.y), x[16 * c + 4 * k + 2], x[16 * c + 4 * k + 3]);
      }
    }
    if (t0 + kTcTok - 1 > pw_min || t0 + kTcTok > tend) {   // uniform over the warp pair
#pragma unroll
      for (int j = 0; j < HC; ++j)
        if (c0 + j > pr || c0 + j >= tend) x[j] = -INFINITY;
    }
    float tmx = -INFINITY;
#pragma unroll
    for (int j = 0; j < HC; ++j) tmx = fmaxf(tmx, x[j]);

    // PV(it - 1) must be complete before O is rescaled and the V tile
    // reused (P(it) goes to the other S buffer, which PV(it - 1) does not read).
    auto wait_pv = [&]() {
      if (o_issued > o_done) {
        if (mbar_wait_bounded(bar_o, o_done & 1))
          ++o_done;
        else
          fail_s[it & 1] = 1;
        tc_fence_after();
      }
    };
    // The row maximum over both column halves, exchanged with the partner
    // warp through the consumed S buffer: each thread leaves its value in a
    // column of its own half of S (already read) that the partner overwrites
    // with its P later, and reads the partner's from a column that it
    // overwrites itself later.  Half 0 reads S columns 0..31 and writes P
    // into 0..15 and 32..47; half 1 reads 32..63 and writes 16..31, 48..63.
    const uint32_t s_col = tmem + (it & 1) * 64 + lane_off;
    tc_st1(s_col + 16 + 16 * half, __float_as_uint(tmx));
    tc_wait_st();
    tc_fence_before();
    named_barrier(1 + sub, 64);
    tc_fence_after();
    tmx = fmaxf(tmx, __uint_as_float(tc_ld1(s_col + 16 + 16 * (half ^ 1))));
    tc_wait_ld();
    const float nm = fmaxf(mx, tmx);
    const float base = nm == -INFINITY ? 0.f : nm;
    const float f = ex2f(mx - base);                            // 0 while mx = -inf
    const bool moved = __any_sync(0xffffffffu, nm > mx);       // the same in both warps of the pair
    mx = nm;
    const uint64_t base2 = f2_pack(base, base);
    l2 = f2_mul(l2, f2_pack(f, f));
    // P = p s^V as float16 hi and lo parts: tokens 2i, 2i + 1 of the tile in
    // column i of the hi block (columns 0..31) and of the lo block (32..63).
    uint32_t phi[HC / 2], plo[HC / 2];
#pragma unroll
    for (int c = 0; c < HC / 8; ++c) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int j = 8 * c + 2 * k;
        float p0, p1;
        f2_unpack(f2_sub(f2_pack(x[j], x[j + 1]), base2), p0, p1);
        const uint64_t p2 = f2_pack(ex2f(p0), ex2f(p1));
        l2 = f2_add(l2, p2);
        const ulonglong2 n = nv4[j >> 2];
        f2_unpack(f2_mul(p2, (k & 1) ? n.y : n.x), p0, p1);
        const __half2 h = __floats2half2_rn(p0, p1);
        const float2 hf = __half22float2(h);
        phi[4 * c + k] = *reinterpret_cast<const uint32_t *>(&h);
        plo[4 * c + k] = pack_f16x2(p0 - hf.x, p1 - hf.y);
      }
    }
    tc_st16u(s_col + 16 * half, phi);
    tc_st16u(s_col + 32 + 16 * half, plo);
    tc_wait_st();
    wait_pv();

    if (moved && it > 0) {
#pragma unroll 1
      for (int c = 0; c < OH / 16; ++c) {
        float v[16];
        tc_ld16(t_o + OH * half + lane_off + 16 * c, v);
        const uint64_t f2 = f2_pack(f, f);
#pragma unroll
        for (int j = 0; j < 16; j += 2) f2_unpack(f2_mul(f2_pack(v[j], v[j + 1]), f2), v[j], v[j + 1]);
        tc_st16(t_o + OH * half + lane_off + 16 * c, v);
      }
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
    }
    tc_expand<D, false>(vc, vt, nullptr, a, tid);
    if (it + 1 < n_tiles) tc_fetch<D>(vc, vb, (it + 1) * kTcTok, tend, tid);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (fail_s[it & 1]) {   // the same value for every thread
      failed = true;
      break;
    }
    // Every thread is past the softmax of tile it: its norms can be replaced.
    if (it + 1 < n_tiles) {
      store_norm();
      if (it + 2 < n_tiles) fetch_norm(it + 2);
    }
    if (tid == 0) {
      constexpr uint32_t idesc = tc_idesc(kTcRows, D, 1);
      const uint32_t pa = tmem + (it & 1) * 64;               // P(it): hi in columns 0..31, lo in 32..63
#pragma unroll
      for (int ks = 0; ks < kTcTok / 16; ++ks) {
        const uint64_t bd = tc_desc(v_s + ks * 2048, KBLK, 1024);
        tc_mma_ts(t_o, pa + 8 * ks, bd, idesc, (it > 0 || ks > 0) ? 1u : 0u);
        tc_mma_ts(t_o, pa + 32 + 8 * ks, bd, idesc, 1u);
      }
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
      for (int j = qk_done; j < qk_issued; ++j)
        if (!mbar_wait_bounded(&bar_s[j & 1], (j >> 1) & 1)) break;
      if (o_issued > o_done) mbar_wait_bounded(bar_o, o_done & 1);
    }
  } else {
    // ---- epilogue, 32 rows per pass: O / l from TMEM, rotate back, store ----
    tc_fence_after();
    __syncthreads();
    float *xchg = reinterpret_cast<float *>(q_hi);   // [2][kTcRows] row sums; the query tiles are free
    float l0, l1;
    f2_unpack(l2, l0, l1);
    const float l = l0 + l1;
    xchg[half * kTcRows + r] = l;
    __syncthreads();
    const float lt = l + xchg[(half ^ 1) * kTcRows + r];
    const float inv = lt > 0.f ? a.out_unit / lt : 0.f;
    for (int pass = 0; pass < kTcRows / 32; ++pass) {
      __syncthreads();   // scratch (over the K and V tiles) is free
      if (sub == pass) {
#pragma unroll 1
        for (int c = 0; c < OH / 16; ++c) {
          float v[16];
          if (n_tiles > 0) {
            tc_ld16(t_o + OH * half + lane_off + 16 * c, v);
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = 0.f;
          }
#pragma unroll
          for (int j = 0; j < 16; ++j) scratch[lane * D + OH * half + 16 * c + j] = v[j] * inv;
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
// alpha c_k over the unit-variance 3-bit centroids (searched once), the
// float16 tables of alpha c_k and of its residual alpha c_k - fp16(alpha c_k)
// (below 2^-15 of the centroid; subnormal float16 values where small).
struct PfTables {
  double alpha;
  uint32_t lo0, lo1, hi0, hi1;
  uint32_t rlo0, rlo1, rhi0, rhi1;
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
    tb.rlo0 = tb.rlo1 = tb.rhi0 = tb.rhi1 = 0;
    for (int k = 0; k < 8; ++k) {
      const double v = best * c[k];
      const uint16_t hb = pf_half_bits(v);
      const double vh = static_cast<double>(__half2float(*reinterpret_cast<const __half *>(&hb)));
      const uint16_t rb = pf_half_bits(v - vh);
      const int sh = 8 * (k % 4);
      (k < 4 ? tb.lo0 : tb.lo1) |= static_cast<uint32_t>(hb & 0xFFu) << sh;
      (k < 4 ? tb.hi0 : tb.hi1) |= static_cast<uint32_t>(hb >> 8) << sh;
      (k < 4 ? tb.rlo0 : tb.rlo1) |= static_cast<uint32_t>(rb & 0xFFu) << sh;
      (k < 4 ? tb.rhi0 : tb.rhi1) |= static_cast<uint32_t>(rb >> 8) << sh;
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
  a.res_lo0 = tb.rlo0;
  a.res_lo1 = tb.rlo1;
  a.res_hi0 = tb.rhi0;
  a.res_hi1 = tb.rhi1;
  a.out_unit = static_cast<float>(1.0 / (tb.alpha * d));
  a.score_unit = static_cast<float>(a.score_unit / (tb.alpha * std::sqrt(static_cast<double>(d))));
  return run_prefill_t<__half>(d, variant, a, st);
}
