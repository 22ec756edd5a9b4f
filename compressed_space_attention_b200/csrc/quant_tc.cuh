// Compressor for d = 128 float16 vectors with the whole rotation on the
// 5th-generation tensor cores (tcgen05 + TMEM).  Included by isoq_quant.cu
// inside namespace isoq::quant, after the register-level pieces
// (quantize_group, search_scale).
//
// RotaryQuant §3.2 Algorithm 1 on a tile of 128 vectors x of one head:
//   u = W x  with  W = R_SO4 H_128  (unnormalised; R_SO4 block-diagonal 4 x 4),
//   S = sqrt(128) ||x||  (= ||H_128 x||),
//   code_i = #{k : u_i > t_k S}, stored norm float16(S / sqrt(128)),
// which are the decisions of y = R_SO4 (H x / (||x|| sqrt d)) against t_k.
//
// The rotation is one matrix product per tile: D[128 x 128] (float32, TMEM)
// = X[128 x 128] (float16, TMA-loaded, 128B-swizzled K-major) . W^T, with W
// split into float16 hi and lo parts (W = W_hi + W_lo to about 2^-22 of each
// entry; both are K-major B operands, two products per K step).  W depends on
// the head: the CTA builds it in shared memory at the start of each run of
// tiles of one head (entry W[n][k] = sum_c R_i[n mod 4][c] H[4i + c][k],
// i = n / 4, four products in float32).  The norm, the Lloyd-Max search and
// the packing run on the CUDA cores, two threads per vector: the threads of
// warps w and w + 4 of an epilogue group read the same TMEM lane (row) and
// take columns 0..63 and 64..127 (groups 0, 1 and 2, 3 of the packed
// layout).  They take the norm from x itself, reading the vector's row of
// the X tile in shared memory while the product runs (not from ||u||: the
// float32 rotation parameters make R_SO4 orthogonal only to ~1e-7): each
// sums the squares of its 64 columns and the two swap their partial sums
// through shared memory, with an mbarrier per warp and a bounded wait (both
// add the halves in the same order, so both hold the same norm); the X stage
// is refilled once the product and the 256 epilogue threads of the tile's
// group have all released it.
//
// Warp roles (one CTA per SM, a contiguous range of tiles):
//   warp 17, lane 0: TMA loads of X tiles into a 4-deep ring, running ahead
//     across runs of heads (it takes no part in the run barriers);
//   warp 16, lane 0: the MMAs, each tile into TMEM buffer (tile & 3), so that
//     the products run up to two tiles of each group ahead of the epilogue;
//   warps 0-7 / 8-15: epilogue of the even / odd tiles (warp w reads TMEM
//     sub-partition w % 4, rows 32 (w % 4) .. + 31, column half (w / 4) % 2).
// The epilogue and MMA warps build W between runs of tiles of different heads;
// a barrier of those 17 warps closes each run, after every product of the
// run has been read back (so none still reads W).
// mbarriers: full[s] (TMA landed), empty[s] (the MMA that read stage s is
// done and the epilogue group has read its norms there), tfull[b] (TMEM buffer b holds a finished product), tempty[b] (the
// epilogue group has read buffer b).  Every wait is bounded; a wait that
// gives up sets the quantize error word and a CTA-wide flag, the loops stop,
// the producer lets its copies and products finish (bounded), and the CTA
// frees its tensor memory.

constexpr int kTqRows = 128;                    // vectors per tile (M, one TMEM lane each)
constexpr int kTqD = 128;
constexpr int kTqStages = 4;
constexpr int kTqEpiWarps = 16;
constexpr int kTqMmaWarp = kTqEpiWarps, kTqTmaWarp = kTqEpiWarps + 1;
constexpr int kTqThreads = 32 * (kTqEpiWarps + 2);
constexpr int kTqRunThreads = 32 * (kTqEpiWarps + 1);   // the run barrier: epilogue and MMA warps
constexpr int kTqBlk = kTqRows * 128;           // one 64-column block of a tile (16 KB)
constexpr int kTqXBytes = 2 * kTqBlk;           // one X tile (32 KB)
constexpr int kTqWBytes = kTqD * kTqD * 2;      // W_hi or W_lo (32 KB each)
constexpr int kTqOffWlo = kTqWBytes;
constexpr int kTqOffX = 2 * kTqWBytes;
constexpr int kTqOffRot = kTqOffX + kTqStages * kTqXBytes;    // the head's 4 x 4 blocks R_i H_4, 32 x 16 floats
constexpr int kTqOffBar = kTqOffRot + kTqD / 4 * 16 * 4;
constexpr int kTqBufs = 4;                      // TMEM buffers of 128 columns
constexpr int kTqOffXch = kTqOffBar;            // partial norms [group][half][sub][slot][lane]
constexpr int kTqXchBytes = 2 * 2 * 4 * 2 * 32 * 4;
constexpr int kTqBars = 2 * kTqStages + 2 * kTqBufs + 2 * kTqEpiWarps;   // + two per epilogue warp
constexpr int kTqSmem = kTqOffBar + kTqXchBytes + 8 * kTqBars + 16 + 1024;   // + the flag words, + alignment slack
static_assert(kTqSmem <= 232448, "shared memory per CTA");

__device__ __forceinline__ void tc_ld32_nowait(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

// Builds W_hi, W_lo (128B-swizzled K-major, row n, column k) for one head's
// rotation parameters; all threads of the CTA take part.
template <bool FULL>
__device__ void build_rotation_operand(const float *params_head, float *rot, unsigned char *whi,
                                       unsigned char *wlo, int tid) {   // tid < kTqRunThreads
  if (tid < kTqD / 4) {
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
  named_barrier(1, kTqRunThreads);
  // W[n][k] = sum_c R_{n/4}[n mod 4][c] H[4 (n/4) + c][k]
  //         = (-1)^popc((n & ~3) & k) M_{n/4}[n mod 4][k mod 4]: the rows 4 (n/4) + c
  // and the column k share no bits outside c's, so the sign splits off
  // (the same four products, summed in the same order, with one sign).
  for (int idx = tid; idx < kTqD * kTqD / 8; idx += kTqRunThreads) {
    const int n = idx / (kTqD / 8), k0 = 8 * (idx % (kTqD / 8));
    const float *mm = rot + 16 * (n >> 2) + 4 * (n & 3);
    const int n4 = n & ~3;
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int j = 0; j < 8; j += 2) {
      float w[2];
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
        const int k = k0 + j + jj;
        w[jj] = (__popc(n4 & k) & 1) ? -mm[k & 3] : mm[k & 3];
      }
      const __half2 h = __floats2half2_rn(w[0], w[1]);
      const float2 hf = __half22float2(h);
      const __half2 l = __floats2half2_rn(w[0] - hf.x, w[1] - hf.y);
      hw[j / 2] = *reinterpret_cast<const uint32_t *>(&h);
      lw[j / 2] = *reinterpret_cast<const uint32_t *>(&l);
    }
    *reinterpret_cast<uint4 *>(whi + tc_off(n, k0, kTqBlk)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    *reinterpret_cast<uint4 *>(wlo + tc_off(n, k0, kTqBlk)) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
  }
}

template <int BITS, bool FULL>
__global__ void __launch_bounds__(kTqThreads, 1)
    quantize_tc_kernel(const __grid_constant__ CUtensorMap xmap, const QuantArgs args) {
  constexpr int L = 1 << BITS, NPOS = L / 2 - 1;
  constexpr int PB = kTqD * BITS / 8, GB = 32 * BITS / 8;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  unsigned char *smem = smem_raw + pad;
  unsigned char *whi = smem, *wlo = smem + kTqOffWlo;
  unsigned char *xs = smem + kTqOffX;
  float *rot = reinterpret_cast<float *>(smem + kTqOffRot);
  float *xch = reinterpret_cast<float *>(smem + kTqOffXch);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kTqOffBar + kTqXchBytes);
  uint64_t *empty = full + kTqStages;
  uint64_t *tfull = empty + kTqStages;
  uint64_t *tempty = tfull + kTqBufs;
  uint64_t *pbar = tempty + kTqBufs;   // [epilogue warp][slot]: its partial norms are written
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(pbar + 2 * kTqEpiWarps);
  volatile uint32_t *fail = tmem_slot + 1;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool producer = warp == kTqMmaWarp, loader = warp == kTqTmaWarp;
  const long long per_cta = (args.total_tiles + gridDim.x - 1) / gridDim.x;
  const long long tile_begin = static_cast<long long>(blockIdx.x) * per_cta;
  long long tile_end = tile_begin + per_cta;
  if (tile_end > args.total_tiles) tile_end = args.total_tiles;
  const int n_mine = tile_end > tile_begin ? static_cast<int>(tile_end - tile_begin) : 0;

  if (tid == 0) {
    for (int s = 0; s < kTqStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + 8 * 32);
    }
    for (int b = 0; b < kTqBufs; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 8 * 32);
    }
    for (int w = 0; w < 2 * kTqEpiWarps; ++w) mbar_init(&pbar[w], 32);
    *fail = 0u;
    mbar_fence_init();
  }
  if (producer) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(128 * kTqBufs));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Producer state (lane 0 of the producer warp).
  auto load = [&](int i) {
    const long long t = tile_begin + i;
    const int head = static_cast<int>(t / args.tiles_per_head);
    const int v0 = static_cast<int>((t % args.tiles_per_head) * kTqRows);
    unsigned char *st = xs + (i % kTqStages) * kTqXBytes;
    uint64_t *bar = &full[i % kTqStages];
    mbar_arrive_expect_tx(bar, kTqXBytes);
    tma_load_3d(st, &xmap, bar, 0, v0, head);
    tma_load_3d(st + kTqBlk, &xmap, bar, 64, v0, head);
  };
  int mma_done = 0;

  // Epilogue geometry.
  const int grp = warp >> 3, sub = warp & 3, half = (warp >> 2) & 1;
  const int r = 32 * sub + lane;
  const uint32_t t_lane = tmem + (static_cast<uint32_t>(32 * sub) << 16);

  if (loader) {
    // ---- TMA loads: stage s is refilled once the product and the norms of
    // the tile before have released it ----
    if (lane == 0) {
      int loaded = 0;
      bool ok = true;
      for (; loaded < n_mine; ++loaded) {
        const int s = loaded % kTqStages;
        if (loaded >= kTqStages)
          ok = mbar_wait_bounded(&empty[s], static_cast<uint32_t>(loaded / kTqStages - 1) & 1u);
        if (*fail) ok = false;
        if (!ok) break;
        load(loaded);
      }
      if (!ok) {
        *fail = 1u;
        atomicOr(&g_quant_error, kErrWaitTimeout);
      }
      // every copy issued lands before the CTA may exit
      for (int j = loaded - kTqStages < 0 ? 0 : loaded - kTqStages; j < loaded; ++j)
        if (!mbar_wait_bounded(&full[j % kTqStages], static_cast<uint32_t>(j / kTqStages) & 1u)) break;
    }
    __syncwarp();
  }

  int i_seg = 0;
  while (!loader && i_seg < n_mine) {
    // One run of tiles of one head.
    const int head = static_cast<int>((tile_begin + i_seg) / args.tiles_per_head);
    long long seg_end_ll = static_cast<long long>(head + 1) * args.tiles_per_head - tile_begin;
    const int seg_end = seg_end_ll < n_mine ? static_cast<int>(seg_end_ll) : n_mine;
    build_rotation_operand<FULL>(args.params + static_cast<size_t>(head) * 2 * kTqD, rot, whi, wlo, tid);
    fence_proxy_async_smem();   // W is read by the tensor core (async proxy)
    tc_fence_before();
    named_barrier(1, kTqRunThreads);
    tc_fence_after();

    if (producer) {
      // ---- producer: MMAs of this run (TMA loads run ahead across runs) ----
      if (lane == 0 && !*fail) {
        constexpr uint32_t idesc = tc_idesc(kTqRows, kTqD, 0);
        const uint32_t wh_s = smem_u32(whi), wl_s = smem_u32(wlo);
        bool ok = true;
        for (int i = i_seg; i < seg_end && ok; ++i) {
          const int s = i % kTqStages, b = i % kTqBufs;
          ok = mbar_wait_bounded(&full[s], static_cast<uint32_t>(i / kTqStages) & 1u);
          if (ok && i >= kTqBufs) ok = mbar_wait_bounded(&tempty[b], static_cast<uint32_t>(i / kTqBufs - 1) & 1u);
          if (*fail) ok = false;
          if (!ok) break;
          tc_fence_after();
          const uint32_t x_s = smem_u32(xs + s * kTqXBytes);
#pragma unroll
          for (int ks = 0; ks < kTqD / 16; ++ks) {
            const uint32_t off = (ks >> 2) * kTqBlk + (ks & 3) * 32;
            const uint64_t ad = tc_desc(x_s + off, 16, 1024);
            tc_mma(tmem + 128 * b, ad, tc_desc(wh_s + off, 16, 1024), idesc, ks > 0 ? 1u : 0u);
            tc_mma(tmem + 128 * b, ad, tc_desc(wl_s + off, 16, 1024), idesc, 1u);
          }
          tc_commit(&tfull[b]);
          tc_commit(&empty[s]);
          mma_done = i + 1;
        }
        if (!ok) {
          *fail = 1u;
          atomicOr(&g_quant_error, kErrWaitTimeout);
        }
      }
      __syncwarp();
    } else {
      // ---- epilogue of this run's tiles of parity grp: two threads per vector ----
      for (int i = i_seg + ((i_seg & 1) != grp ? 1 : 0); i < seg_end; i += 2) {
        const long long t = tile_begin + i;
        const int s = i % kTqStages;
        // The norm from the X tile (row r), while the product runs.
        // A wait that gives up leaves ok false; the tile is still carried
        // through (its reads are of this CTA's own memory and its stores go
        // to this tile's rows), and the loop stops after it.
        bool ok = mbar_wait_bounded(&full[s], static_cast<uint32_t>(i / kTqStages) & 1u);
        const uint32_t xrow = smem_u32(xs + s * kTqXBytes);
        uint64_t ss2 = f2_pack(0.f, 0.f);
#pragma unroll
        for (int c = 8 * half; c < 8 * half + 8; ++c) {   // this thread's 64 columns
          const uint4 q = lds128(xrow + tc_off(r, 8 * c, kTqBlk));
          const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&qw[j]));
            const uint64_t p = f2_pack(f.x, f.y);
            ss2 = f2_fma(p, p, ss2);
          }
        }
        mbar_arrive(&empty[s]);   // this thread is done with the stage
        float s_lo, s_hi;
        f2_unpack(ss2, s_lo, s_hi);
        // Swap the partial sums with the partner warp.  Slot (and mbarrier)
        // k & 1 for the group's k-th tile: the partner reads slot k & 1 before
        // it arrives for tile k + 1, and this warp writes that slot again only
        // at tile k + 2, after waiting for that arrival; each mbarrier moves one
        // phase per two tiles, so a wait cannot see a phase two ahead.
        const int k = i >> 1, slot = k & 1;
        float *mine = xch + (((grp * 2 + half) * 4 + sub) * 2 + slot) * 32;
        const float *theirs = xch + (((grp * 2 + (half ^ 1)) * 4 + sub) * 2 + slot) * 32;
        mine[lane] = s_lo + s_hi;
        mbar_arrive(&pbar[2 * warp + slot]);
        ok = mbar_wait_bounded(&pbar[2 * (warp ^ 4) + slot], static_cast<uint32_t>(k >> 1) & 1u) && ok;
        const float other = theirs[lane];
        const float ssq = half == 0 ? mine[lane] + other : other + mine[lane];   // ||x||^2, same order in both
        const uint32_t zmask = ssq > 0.f ? 0u : 0x80000000u;
        const float S = sqrtf(ssq * static_cast<float>(kTqD));
        const float big = search_scale(S);
        float tb[NPOS];
#pragma unroll
        for (int j = 0; j < NPOS; ++j) tb[j] = -(args.tau[j] * S) * big;
        const int b = i % kTqBufs;
        const uint32_t t_row = t_lane + 128 * b;
        ok = mbar_wait_bounded(&tfull[b], static_cast<uint32_t>(i / kTqBufs) & 1u) && ok;
        tc_fence_after();
        const long long v = (t % args.tiles_per_head) * kTqRows + r;
        const bool live = v < args.n_vec;
        const long long idx = static_cast<long long>(head) * args.out_head_stride + v;
        // This thread's two 32-element groups, held as pairs (e, e + 16); the
        // second group's tensor-memory read is in flight while the first is
        // quantised (the first group's words are paired before it is issued,
        // so that 96 registers hold both).
        uint64_t xp[kGP];
        {
          uint32_t va[32];
          tc_ld32_nowait(t_row + 64 * half, va);
          tc_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) xp[e] = f2_pack(__uint_as_float(va[e]), __uint_as_float(va[e + 16]));
        }
        uint32_t vb[32];
        tc_ld32_nowait(t_row + 64 * half + 32, vb);
#pragma unroll
        for (int G = 0; G < 2; ++G) {
          if (G == 1) {
            tc_wait_ld();
            tc_fence_before();
            mbar_arrive(&tempty[b]);   // every read of this buffer is done: free for tile i + 4
#pragma unroll
            for (int e = 0; e < 16; ++e) xp[e] = f2_pack(__uint_as_float(vb[e]), __uint_as_float(vb[e + 16]));
          }
          if (live) {
            uint32_t w[GB / 4];
            quantize_group<BITS>(xp, 0, tb, big, zmask, w);
            uint8_t *gd = args.codes + idx * PB + (2 * half + G) * GB;
            if constexpr (GB == 16) {
              *reinterpret_cast<uint4 *>(gd) = make_uint4(w[0], w[1], w[2], w[3]);
            } else if constexpr (GB == 8) {
              *reinterpret_cast<uint2 *>(gd) = make_uint2(w[0], w[1]);
            } else {
#pragma unroll
              for (int k = 0; k < GB / 4; ++k) reinterpret_cast<uint32_t *>(gd)[k] = w[k];
            }
          }
        }
        if (live && half == 0) args.norms[idx] = __half_as_ushort(__float2half_rn(sqrtf(ssq)));
        if (__any_sync(0xffffffffu, !ok) || *fail) {
          if (lane == 0) {
            *fail = 1u;
            atomicOr(&g_quant_error, kErrWaitTimeout);
          }
          break;
        }
      }
    }
    // Every product of the run has been read back: W may be rebuilt.
    tc_fence_before();
    named_barrier(1, kTqRunThreads);
    tc_fence_after();
    if (*fail) break;
    i_seg = seg_end;
  }
  if (producer && lane == 0 && mma_done > 0) {
    // The last products finish before the CTA frees the tensor memory.
    mbar_wait_bounded(&tfull[(mma_done - 1) % kTqBufs], static_cast<uint32_t>((mma_done - 1) / kTqBufs) & 1u);
  }
  tc_fence_before();
  __syncthreads();
  if (producer) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(128 * kTqBufs));
}
