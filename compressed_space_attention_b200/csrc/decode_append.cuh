// Decode-step append: compress the new token's K and V vectors of every
// (b, kvh) into the packed cache at position seq_lens[b], then advance the
// lengths.  Included by isoq_decode.cu inside namespace isoq::decode.
//
// RotaryQuant §3.2 Algorithm 1 applied to one vector per (b, kvh, K|V): the
// float32 norm, the rotation R = R_SO4 H_d / sqrt(d) of the unnormalised
// vector, codes #{k : y > s t_k} against the norm-scaled Lloyd-Max
// thresholds, and the packed layout of common.cuh.  During decode each new
// entry is compressed once and written into the packed cache, which the fused
// attention then reads (RotaryQuant Figure 1, Appendix D: "invalidated after
// each write"); the bulk compression of the prefill buffer at the
// prefill-to-decode boundary (Appendix C) is isoq_quantize on that buffer.
//
// Grid (Hkv, B, 2): z = 0 appends K, z = 1 appends V.  A row whose length
// is already Tmax cannot take another token: it is left unchanged and the
// device error word records kErrCacheFull.

constexpr unsigned kErrCacheFull = 2u;
constexpr int kAppendThreads = 128;

struct AppendArgs {
  const void *k_new;      // [B][Hkv][d] of the query dtype
  const void *v_new;
  uint8_t *packed_k;      // [B][Hkv][Tmax][d*bits/8]
  uint8_t *packed_v;
  uint16_t *norms_k;      // [B][Hkv][Tmax] float16 bits
  uint16_t *norms_v;
  const int32_t *seq_lens;
  const float *params_k;  // [Hkv][d/4][8]
  const float *params_v;
  long long tmax;
  int batch, hkv;
  float thr[15];          // the L - 1 Lloyd-Max thresholds of N(0, 1/d), ascending
};

template <typename T, int D, int BITS, bool FULL>
__global__ void __launch_bounds__(kAppendThreads) append_kernel(const AppendArgs a) {
  constexpr int L = 1 << BITS;
  constexpr int GW = BITS;           // 32-bit words per 32-code group (32 * BITS / 32)
  __shared__ float v[D];
  __shared__ float red[kAppendThreads / 32];
  __shared__ unsigned char codes[D];
  const int kvh = blockIdx.x, b = blockIdx.y, which = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  int pos = a.seq_lens[b];
  pos = pos < 0 ? 0 : pos;
  if (pos >= a.tmax) {
    if (tid == 0 && kvh == 0 && which == 0) atomicOr(&g_decode_error, kErrCacheFull);
    return;
  }
  const long long row = static_cast<long long>(b) * a.hkv + kvh;
  const T *x = static_cast<const T *>(which ? a.v_new : a.k_new) + row * D;
  float ss = 0.f;
  for (int i = tid; i < D; i += kAppendThreads) {
    const float xi = to_f32<T>(x[i]);
    v[i] = xi;
    ss = fmaf(xi, xi, ss);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane == 0) red[warp] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < kAppendThreads / 32; ++w) tot += red[w];
  const float s = sqrtf(tot);

  // y = R x (unnormalised); the thresholds are scaled by s instead.
  rotate_forward_smem<D, FULL>(v, 1, (which ? a.params_v : a.params_k) + static_cast<size_t>(kvh) * 2 * D,
                               tid, kAppendThreads, 0);
  for (int i = tid; i < D; i += kAppendThreads) {
    const float y = v[i];
    int c = 0;
#pragma unroll
    for (int k = 0; k < L - 1; ++k) c += (y > a.thr[k] * s) ? 1 : 0;
    codes[i] = static_cast<unsigned char>(c);
  }
  __syncthreads();

  constexpr int PB = D * BITS / 8;
  uint8_t *dst = (which ? a.packed_v : a.packed_k) + (row * a.tmax + pos) * PB;
  for (int grp = tid; grp < D / 32; grp += kAppendThreads) {
    uint32_t w[GW];
#pragma unroll
    for (int k = 0; k < GW; ++k) w[k] = 0u;
#pragma unroll
    for (int i = 0; i < 32; ++i) pack_code<BITS>(w, i, codes[32 * grp + i]);
    uint32_t *gd = reinterpret_cast<uint32_t *>(dst + grp * 32 * BITS / 8);
#pragma unroll
    for (int k = 0; k < GW; ++k) gd[k] = w[k];
  }
  if (tid == 0) {
    uint16_t *nrm = which ? a.norms_v : a.norms_k;
    nrm[row * a.tmax + pos] = __half_as_ushort(__float2half_rn(s));
  }
}

// seq_lens[b] <- seq_lens[b] + 1 for every row that took the new token.
__global__ void advance_lengths_kernel(int32_t *seq_lens, int batch, long long tmax) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < batch) {
    int p = seq_lens[b];
    p = p < 0 ? 0 : p;
    if (p < tmax) seq_lens[b] = p + 1;
  }
}

template <typename T, int D, int BITS, bool FULL>
int launch_append(const AppendArgs &a, int32_t *seq_lens, cudaStream_t stream) {
  append_kernel<T, D, BITS, FULL><<<dim3(a.hkv, a.batch, 2), kAppendThreads, 0, stream>>>(a);
  advance_lengths_kernel<<<(a.batch + 127) / 128, 128, 0, stream>>>(seq_lens, a.batch, a.tmax);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(ISOQ_ERR_CUDA, "decode append launch: %s", cudaGetErrorString(e));
  return ISOQ_OK;
}

template <typename T, int D, int BITS>
int run_append_v(int variant, const AppendArgs &a, int32_t *seq_lens, cudaStream_t st) {
  return variant == ISOQ_FULL ? launch_append<T, D, BITS, true>(a, seq_lens, st)
                              : launch_append<T, D, BITS, false>(a, seq_lens, st);
}

template <typename T, int D>
int run_append_b(int bits, int variant, const AppendArgs &a, int32_t *seq_lens, cudaStream_t st) {
  if (bits == 2) return run_append_v<T, D, 2>(variant, a, seq_lens, st);
  if (bits == 3) return run_append_v<T, D, 3>(variant, a, seq_lens, st);
  return run_append_v<T, D, 4>(variant, a, seq_lens, st);
}

template <typename T>
int run_append_d(int d, int bits, int variant, const AppendArgs &a, int32_t *seq_lens, cudaStream_t st) {
  if (d == 128) return run_append_b<T, 128>(bits, variant, a, seq_lens, st);
  if (d == 256) return run_append_b<T, 256>(bits, variant, a, seq_lens, st);
  return run_append_b<T, 512>(bits, variant, a, seq_lens, st);
}

int run_append(int dtype, int d, int bits, int variant, const AppendArgs &a, int32_t *seq_lens,
               cudaStream_t st) {
  return dtype == ISOQ_F16 ? run_append_d<__half>(d, bits, variant, a, seq_lens, st)
                           : run_append_d<float>(d, bits, variant, a, seq_lens, st);
}
