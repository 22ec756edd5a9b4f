// Dequantizer for d = 128, 2- and 3-bit codes, float16 output, with the
// whole inverse rotation on the 5th-generation tensor cores (tcgen05 + TMEM).
// Included by isoq_quant.cu inside namespace isoq::quant, after quant_tc.cuh
// (build_rotation_operand's pieces, tc_ld32_nowait).
//
// RotaryQuant §3.2 Algorithm 1, DeQuant, on a tile of 128 vectors of one
// head: x^ = ||x|| H_n^T R_SO4^T c with c the Lloyd-Max centroids of the
// codes for N(0, 1/d) and H_n = H_128 / sqrt(128).  With the unit-variance
// centroids c_u = sqrt(128) c and W = R_SO4 H_128 (the quantizer's matrix),
//   x^_n = (||x|| / 128) sum_k W[k][n] c_u[k],
// one product per tile: D[128 x 128] (float32, TMEM) = C_u (A, float16 hi + lo
// parts in TMEM) . (W^T as a K-major B operand in shared memory, hi + lo),
// three products per K step (C_hi W_hi, C_lo W_hi, C_hi W_lo; the dropped
// C_lo W_lo is below 2^-22 of each term).
//
// The codes become the A operand on the CUDA cores: each pair of threads
// takes one vector (row), each thread 64 dims (two 32-code groups); one prmt
// per four codes and byte table (the low and high bytes of the float16 hi and
// lo parts of the 8 or 4 centroids) and two more that interleave the bytes
// give the float16 pairs, which go to the thread's TMEM lane with
// tcgen05.st.  The selectors are the codes in 4-bit fields: the 3-bit layout
// has them there already (plus the spare-bit codes), the 2-bit bitstream is
// spread into them.  After the product the same threads read their 64 output
// columns back, scale by ||x|| / 128, round to float16 and write them into a
// 128B-swizzled tile in shared memory that one thread stores with TMA.
//
// Warp roles (one CTA per SM, a contiguous range of tiles):
//   warps 0-7 / 8-15: tiles of even / odd local index (warp w: TMEM lane
//     quarter w % 4, rows 32 (w % 4) .. + 31, column half (w / 4) % 2);
//     group g owns TMEM columns 256 g .. 256 g + 255 (A hi 64, A lo 64, D 128);
//   warp 16, lane 0: the MMAs.
// mbarriers per group: afull (the group's 256 threads stored A), tfull (the
// product is in TMEM, by tcgen05.commit), dempty (the group has read D).
// Every wait is bounded; a wait that gives up sets the quantize error word
// and a CTA-wide flag, and the loops stop after the tile (a worker group
// decides that at its barrier, all its warps together).

constexpr int kTdRows = 128;
constexpr int kTdD = 128;
constexpr int kTdWorkWarps = 16;
constexpr int kTdMmaWarp = kTdWorkWarps;
constexpr int kTdThreads = 32 * (kTdWorkWarps + 1);
constexpr int kTdBlk = kTdRows * 128;                 // one 64-column block of a tile (16 KB)
constexpr int kTdWBytes = kTdD * kTdD * 2;            // W^T hi or lo (32 KB)
constexpr int kTdOffWlo = kTdWBytes;
constexpr int kTdOffOut = 2 * kTdWBytes;              // output tiles [group][half] of 16 KB
constexpr int kTdOffRot = kTdOffOut + 4 * kTdBlk;
constexpr int kTdOffBar = kTdOffRot + kTdD / 4 * 16 * 4;
constexpr int kTdBars = 6;
constexpr int kTdSmem = kTdOffBar + 8 * kTdBars + 16 + 1024;
static_assert(kTdSmem <= 232448, "shared memory per CTA");

struct DequantTcArgs {
  const uint8_t *codes;
  const uint16_t *norms;
  const float *params;
  long long in_head_stride;
  long long n_vec;
  int tiles_per_head;
  long long total_tiles;
  // Byte tables of the centroid parts (float16 bits of hi = fp16(c_u) and
  // lo = fp16(c_u - hi)), entry j = code j: low bytes, high bytes.
  uint32_t hi_lo[2], hi_hi[2], lo_lo[2], lo_hi[2];
};

// Builds W^T (entry (n, k) = W[k][n]) as float16 hi and lo parts, 128B-swizzled
// K-major (row n = output dimension, column k = rotated coordinate).
template <bool FULL>
__device__ void build_inverse_operand(const float *params_head, float *rot, unsigned char *whi,
                                      unsigned char *wlo, int tid) {   // tid < kTdThreads
  if (tid < kTdD / 4) {
    // M_i = R_i H_4 (H_4[c][m] = (-1)^popc(c & m)), sums in the order c = 0..3.
    float R[4][4];
    const Quat ql = load_quat(params_head + 8 * tid);
    const Quat qr = load_quat(params_head + 8 * tid + 4);
    for (int c = 0; c < 4; ++c) {
      const Quat e{c == 0 ? 1.f : 0.f, c == 1 ? 1.f : 0.f, c == 2 ? 1.f : 0.f, c == 3 ? 1.f : 0.f};
      const Quat u = block_forward(ql, qr, e, FULL);   // column c of R_i
      R[0][c] = u.w;
      R[1][c] = u.x;
      R[2][c] = u.y;
      R[3][c] = u.z;
    }
    for (int row = 0; row < 4; ++row)
      for (int m = 0; m < 4; ++m) {
        float acc = 0.f;
        for (int c = 0; c < 4; ++c) acc += (__popc(c & m) & 1) ? -R[row][c] : R[row][c];
        rot[16 * tid + 4 * row + m] = acc;
      }
  }
  named_barrier(1, kTdThreads);
  // Consecutive threads take consecutive rows n of one 8-column chunk, so
  // that the rotation entries they read (which depend on k only) are
  // broadcasts and their 16-byte stores fall in distinct banks.
  for (int idx = tid; idx < kTdD * kTdD / 8; idx += kTdThreads) {
    const int n = idx % kTdD, k0 = 8 * (idx / kTdD);
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int j = 0; j < 8; j += 2) {
      float w[2];
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
        // W[k][n] = sum_c R_{k/4}[k mod 4][c] H[4 (k/4) + c][n]
        //         = (-1)^popc((k & ~3) & n) M_{k/4}[k mod 4][n mod 4]
        const int k = k0 + j + jj;
        const float m = rot[16 * (k >> 2) + 4 * (k & 3) + (n & 3)];
        w[jj] = (__popc((k & ~3) & n) & 1) ? -m : m;
      }
      const __half2 h = __floats2half2_rn(w[0], w[1]);
      const float2 hf = __half22float2(h);
      const __half2 l = __floats2half2_rn(w[0] - hf.x, w[1] - hf.y);
      hw[j / 2] = *reinterpret_cast<const uint32_t *>(&h);
      lw[j / 2] = *reinterpret_cast<const uint32_t *>(&l);
    }
    *reinterpret_cast<uint4 *>(whi + tc_off(n, k0, kTdBlk)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    *reinterpret_cast<uint4 *>(wlo + tc_off(n, k0, kTdBlk)) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
  }
}

// prmt selectors of the eight quads of one 32-code 3-bit group (three words:
// codes 0..7, 8..15, 16..23 in 4-bit fields, codes 24..31 in the spare bit of
// each field, bit r of code 24 + j at bit 4 j + 3 of word r); quad q = codes
// 4 q .. 4 q + 3 in the low 16 bits of s[q].
__device__ __forceinline__ void dq_group_sel8(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t (&s)[8]) {
  const uint32_t m0 = w0 & 0x77777777u, m1 = w1 & 0x77777777u, m2 = w2 & 0x77777777u;
  const uint32_t x0 = w0 ^ m0, x1 = w1 ^ m1, x2 = w2 ^ m2;   // the spare bits, at 4 j + 3
  const uint32_t sum = (x0 >> 3) | (x1 >> 2) | (x2 >> 1);    // code 24 + j at bits 4 j .. 4 j + 2
  s[0] = m0;
  s[1] = m0 >> 16;
  s[2] = m1;
  s[3] = m1 >> 16;
  s[4] = m2;
  s[5] = m2 >> 16;
  s[6] = sum;
  s[7] = sum >> 16;
}

// The same for one 32-code 2-bit group (two words of the LSB-first
// bitstream: code j of a word at bits 2 j .. 2 j + 1), spread to 4-bit
// fields.
__device__ __forceinline__ uint32_t dq_spread2(uint32_t x) {   // 8 codes in bits 0..15 -> 8 nibbles
  x = (x | (x << 8)) & 0x00FF00FFu;
  x = (x | (x << 4)) & 0x0F0F0F0Fu;
  x = (x | (x << 2)) & 0x33333333u;
  return x;
}

__device__ __forceinline__ void dq_group_sel8_b2(uint32_t w0, uint32_t w1, uint32_t (&s)[8]) {
  const uint32_t a = dq_spread2(w0 & 0xFFFFu), b = dq_spread2(w0 >> 16);
  const uint32_t c = dq_spread2(w1 & 0xFFFFu), d = dq_spread2(w1 >> 16);
  s[0] = a;
  s[1] = a >> 16;
  s[2] = b;
  s[3] = b >> 16;
  s[4] = c;
  s[5] = c >> 16;
  s[6] = d;
  s[7] = d >> 16;
}

// Named barrier that also ORs a predicate over its threads (every thread
// gets the same answer, so a group of warps can stop together).
__device__ __forceinline__ bool named_barrier_or(int id, int nthreads, bool p) {
  int r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\tsetp.ne.b32 pi, %1, 0;\n\t"
      "barrier.cta.red.or.pred po, %2, %3, pi;\n\tselp.b32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"(static_cast<int>(p)), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ uint32_t dq_prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

template <int BITS, bool FULL>
__global__ void __launch_bounds__(kTdThreads, 1)
    dequantize_tc_kernel(const __grid_constant__ CUtensorMap omap, const DequantTcArgs args) {
  static_assert(BITS == 2 || BITS == 3, "2- or 3-bit codes");
  constexpr int PB = kTdD * BITS / 8;   // 32 or 48 bytes per vector
  constexpr int TB = PB / 2;            // bytes of one thread's two groups
  extern __shared__ unsigned char smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  unsigned char *smem = smem_raw + pad;
  unsigned char *whi = smem, *wlo = smem + kTdOffWlo;
  unsigned char *otile = smem + kTdOffOut;
  float *rot = reinterpret_cast<float *>(smem + kTdOffRot);
  uint64_t *afull = reinterpret_cast<uint64_t *>(smem + kTdOffBar);
  uint64_t *tfull = afull + 2;
  uint64_t *dempty = tfull + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(dempty + 2);
  volatile uint32_t *fail = tmem_slot + 1;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool producer = warp == kTdMmaWarp;
  const long long per_cta = (args.total_tiles + gridDim.x - 1) / gridDim.x;
  const long long tile_begin = static_cast<long long>(blockIdx.x) * per_cta;
  long long tile_end = tile_begin + per_cta;
  if (tile_end > args.total_tiles) tile_end = args.total_tiles;
  const int n_mine = tile_end > tile_begin ? static_cast<int>(tile_end - tile_begin) : 0;

  if (tid == 0) {
    for (int g = 0; g < 2; ++g) {
      mbar_init(&afull[g], 8 * 32);
      mbar_init(&tfull[g], 1);
      mbar_init(&dempty[g], 8 * 32);
    }
    *fail = 0u;
    mbar_fence_init();
  }
  if (producer) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Worker geometry.
  const int grp = warp >> 3, sub = warp & 3, half = (warp >> 2) & 1;
  const int r = 32 * sub + lane;
  const uint32_t t_lane = tmem + (static_cast<uint32_t>(32 * sub) << 16) + 256 * grp;
  unsigned char *out_s = otile + (2 * grp + half) * kTdBlk;
  const bool issuer = (warp & 7) == 0 && lane == 0;   // stores the group's output tiles

  // The codes (TB bytes: groups 2 half, 2 half + 1) and the norm of this
  // thread's vector in local tile i.
  auto load_vec = [&](int i, uint32_t (&c)[6], uint32_t &nrm) {
    const long long t = tile_begin + i;
    const int head = static_cast<int>(t / args.tiles_per_head);
    const long long v = (t % args.tiles_per_head) * kTdRows + r;
    if (i < n_mine && v < args.n_vec) {
      const long long idx = static_cast<long long>(head) * args.in_head_stride + v;
      if constexpr (BITS == 3) {
        const uint2 *src = reinterpret_cast<const uint2 *>(args.codes + idx * PB + TB * half);
#pragma unroll
        for (int k = 0; k < 3; ++k) {
          const uint2 u = src[k];
          c[2 * k] = u.x;
          c[2 * k + 1] = u.y;
        }
      } else {
        const uint4 u = *reinterpret_cast<const uint4 *>(args.codes + idx * PB + TB * half);
        c[0] = u.x;
        c[1] = u.y;
        c[2] = u.z;
        c[3] = u.w;
        c[4] = c[5] = 0u;
      }
      nrm = args.norms[idx];
    } else {
#pragma unroll
      for (int k = 0; k < 6; ++k) c[k] = 0u;
      nrm = 0u;
    }
  };

  int i_seg = 0;
  int mma_done = 0;
  while (i_seg < n_mine) {
    // One run of tiles of one head.
    const int head = static_cast<int>((tile_begin + i_seg) / args.tiles_per_head);
    long long seg_end_ll = static_cast<long long>(head + 1) * args.tiles_per_head - tile_begin;
    const int seg_end = seg_end_ll < n_mine ? static_cast<int>(seg_end_ll) : n_mine;
    build_inverse_operand<FULL>(args.params + static_cast<size_t>(head) * 2 * kTdD, rot, whi, wlo, tid);
    fence_proxy_async_smem();   // W^T is read by the tensor core (async proxy)
    tc_fence_before();
    named_barrier(1, kTdThreads);
    tc_fence_after();

    if (producer) {
      if (lane == 0 && !*fail) {
        constexpr uint32_t idesc = tc_idesc(kTdRows, kTdD, 0);
        const uint32_t wh_s = smem_u32(whi), wl_s = smem_u32(wlo);
        bool ok = true;
        for (int i = i_seg; i < seg_end && ok; ++i) {
          const int g = i & 1, k = i >> 1;
          ok = mbar_wait_bounded(&afull[g], static_cast<uint32_t>(k) & 1u);
          if (ok && k > 0) ok = mbar_wait_bounded(&dempty[g], static_cast<uint32_t>(k - 1) & 1u);
          if (*fail) ok = false;
          if (!ok) break;
          tc_fence_after();
          const uint32_t ta = tmem + 256 * g, td = ta + 128;
#pragma unroll
          for (int ks = 0; ks < kTdD / 16; ++ks) {
            const uint32_t off = (ks >> 2) * kTdBlk + (ks & 3) * 32;
            const uint64_t bh = tc_desc(wh_s + off, 16, 1024), bl = tc_desc(wl_s + off, 16, 1024);
            tc_mma_ts(td, ta + 8 * ks, bh, idesc, ks > 0 ? 1u : 0u);
            tc_mma_ts(td, ta + 64 + 8 * ks, bh, idesc, 1u);
            tc_mma_ts(td, ta + 8 * ks, bl, idesc, 1u);
          }
          tc_commit(&tfull[g]);
          mma_done = i + 1;
        }
        if (!ok) {
          *fail = 1u;
          atomicOr(&g_quant_error, kErrWaitTimeout);
        }
      }
      __syncwarp();
    } else {
      // ---- workers: tiles of parity grp ----
      const int i0 = i_seg + ((i_seg & 1) != grp ? 1 : 0);
      uint32_t cw[6];
      uint32_t nw = 0u;
      load_vec(i0, cw, nw);
      for (int i = i0; i < seg_end; i += 2) {
        const int k = i >> 1;
        const long long t = tile_begin + i;
        const int v0 = static_cast<int>((t % args.tiles_per_head) * kTdRows);
        uint32_t c[6];
#pragma unroll
        for (int k = 0; k < 6; ++k) c[k] = cw[k];
        const uint32_t nrm = nw;
        if (i + 2 < seg_end) load_vec(i + 2, cw, nw);   // the group's next tile, in flight meanwhile

        // A = the centroid parts of this thread's 64 dims: columns 32 half ..
        // + 31 (hi) and 64 + 32 half .. + 31 (lo) of the group's A block.
#pragma unroll
        for (int G = 0; G < 2; ++G) {
          uint32_t s[8];
          if constexpr (BITS == 3)
            dq_group_sel8(c[3 * G], c[3 * G + 1], c[3 * G + 2], s);
          else
            dq_group_sel8_b2(c[2 * G], c[2 * G + 1], s);
          uint32_t hw[16], lw[16];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const uint32_t a = dq_prmt(args.hi_lo[0], args.hi_lo[1], s[q]);
            const uint32_t b = dq_prmt(args.hi_hi[0], args.hi_hi[1], s[q]);
            hw[2 * q] = dq_prmt(a, b, 0x5140u);
            hw[2 * q + 1] = dq_prmt(a, b, 0x7362u);
            const uint32_t e = dq_prmt(args.lo_lo[0], args.lo_lo[1], s[q]);
            const uint32_t f = dq_prmt(args.lo_hi[0], args.lo_hi[1], s[q]);
            lw[2 * q] = dq_prmt(e, f, 0x5140u);
            lw[2 * q + 1] = dq_prmt(e, f, 0x7362u);
          }
          tc_st16u(t_lane + 32 * half + 16 * G, hw);
          tc_st16u(t_lane + 64 + 32 * half + 16 * G, lw);
        }
        tc_wait_st();
        tc_fence_before();
        mbar_arrive(&afull[grp]);

        bool ok = mbar_wait_bounded(&tfull[grp], static_cast<uint32_t>(k) & 1u);
        tc_fence_after();
        const float sc = __half2float(__ushort_as_half(static_cast<unsigned short>(nrm))) * 0.0078125f;
        // Before this group's tile buffer is written again, its last store
        // has finished reading it.
        if (issuer) bulk_wait_read_all();
        named_barrier(2 + grp, 8 * 32);
#pragma unroll
        for (int hc = 0; hc < 2; ++hc) {   // 32 output columns at a time
          uint32_t dv[32];
          tc_ld32_nowait(t_lane + 128 + 64 * half + 32 * hc, dv);
          tc_wait_ld();
          if (hc == 1) {
            tc_fence_before();
            mbar_arrive(&dempty[grp]);   // D is read: the next product may overwrite it
          }
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {   // 16-byte chunks of 8 float16
            uint32_t o[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const __half2 h2 = __floats2half2_rn(__uint_as_float(dv[8 * ch + 2 * j]) * sc,
                                                   __uint_as_float(dv[8 * ch + 2 * j + 1]) * sc);
              o[j] = *reinterpret_cast<const uint32_t *>(&h2);
            }
            *reinterpret_cast<uint4 *>(out_s + tc_off(r, 32 * hc + 8 * ch, 0)) = make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
        fence_proxy_async_smem();
        // The group decides together whether to stop after this tile, so that
        // no warp waits at the group's barrier for one that has left.
        const bool stop = named_barrier_or(2 + grp, 8 * 32, !ok || *fail);
        if (issuer) {
          tma_store_3d(&omap, otile + (2 * grp) * kTdBlk, 0, v0, head);
          tma_store_3d(&omap, otile + (2 * grp + 1) * kTdBlk, 64, v0, head);
          bulk_commit();
        }
        if (stop) {
          if (lane == 0) {
            *fail = 1u;
            atomicOr(&g_quant_error, kErrWaitTimeout);
          }
          break;
        }
      }
    }
    // Every product of the run has been read back: W^T may be rebuilt.
    tc_fence_before();
    named_barrier(1, kTdThreads);
    tc_fence_after();
    if (*fail) break;
    i_seg = seg_end;
  }
  if (issuer) bulk_wait_all();
  if (producer && lane == 0 && mma_done > 0) {
    // The last products finish before the CTA frees the tensor memory.
    const int g = (mma_done - 1) & 1;
    mbar_wait_bounded(&tfull[g], static_cast<uint32_t>((mma_done - 1) >> 1) & 1u);
  }
  tc_fence_before();
  __syncthreads();
  if (producer) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
}
