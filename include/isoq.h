/*
 * isoq.h - C ABI of the IsoQuant KV compressor and compressed-space decode
 * attention for NVIDIA B200 (sm_100a).
 *
 * Sources the operations follow (cited by page title and section):
 *   [RQ] "RotaryQuant: Fitting 120B MoE Models on Consumer Hardware via Fused
 *        Compressed-Space Attention", arXiv 2608.08081.
 *   [IQ] "IsoQuant: Hardware-Aligned SO(4) Isoclinic Rotations for LLM KV
 *        Cache Compression", arXiv 2603.28430 (abstract).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every function returns an isoq status (0 = ok, negative = error) and
 *    never throws or aborts.  Arguments are validated on the host before any
 *    device work is queued; a call that fails validation writes nothing.
 *  - Pointers named *_dev are device pointers, *_host host pointers.  The
 *    caller owns every buffer; the library allocates no device memory.  Its
 *    only device state is one 32-bit error word per device (see
 *    isoq_check_device_error) and the fixed workspace array of
 *    isoq_decode_attention_static.  Host state: a mutex-guarded cache of
 *    codebooks and a thread-local error message.
 *  - Device work is queued asynchronously on `stream` (a cudaStream_t; NULL
 *    is the legacy default stream).  Launch failures return ISOQ_ERR_CUDA
 *    with the CUDA error text in isoq_last_error().
 *  - Rotation parameters are float32 arrays [n_heads][d/4][8]: for each
 *    4-dim block the unit quaternions q_L then q_R, each (w, x, y, z).
 *  - Packed codes: d*bits/8 bytes per vector ([RQ] §3.2 Step 4; the pages
 *    fix the size, not the bit order).  bits = 2, 4: an LSB-first
 *    little-endian bitstream (code i at bits [bits*i, bits*i + bits)).
 *    bits = 3: groups of 32 codes in 12 bytes, read as three little-endian
 *    32-bit words w0, w1, w2: bits [4j, 4j+3) of w_r hold code 8r + j of the
 *    group, and bit 4j + 3 of w_r holds bit r of code 24 + j, so that every
 *    code sits in a 4-bit field.  Norms are IEEE float16 bit patterns
 *    (uint16).
 *  - Supported: d in {128, 256, 512}, bits in {2, 3, 4}, variant
 *    ISOQ_FULL or ISOQ_FAST, element dtype ISOQ_F16 or ISOQ_F32.  Anything
 *    else returns ISOQ_ERR_UNSUPPORTED.
 *  - NaN/Inf inputs are not trapped; they propagate.
 */
#ifndef ISOQ_H
#define ISOQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t, declared without the CUDA headers. */
typedef struct CUstream_st *isoq_stream_t;

enum isoq_status {
  ISOQ_OK = 0,
  ISOQ_ERR_INVALID_ARG = -1,  /* null pointer, bad size/stride, too-small workspace */
  ISOQ_ERR_UNSUPPORTED = -2,  /* d, bits, variant, dtype or alignment not supported */
  ISOQ_ERR_CUDA = -3,         /* a CUDA runtime call failed; see isoq_last_error() */
  ISOQ_ERR_TIMEOUT = -4       /* a bounded device-side wait gave up (device error word) */
};

/*
 * Rotation R of a variant, per 4-block (w, x, y, z) = w + x i + y j + z k:
 *   FULL       R = R_SO4 o H_d/sqrt(d), R_SO4: v -> q_L v conj(q_R)
 *              ([IQ] IsoQuant-Full; [RQ] §4.6 Table 8 v3)
 *   FAST       R = R_SO4 o H_d/sqrt(d), R_SO4: v -> q_L v ([IQ] IsoQuant-Fast)
 *   PLANAR     [IQ]'s 2-D special case, read as FULL with q_L and q_R on the
 *              complex line span{1, i}: each block's coordinate pairs (0, 1)
 *              and (2, 3) are rotated independently, by angle(q_L) -
 *              angle(q_R) and angle(q_L) + angle(q_R)
 *   BLOCK_SO4  R = R_SO4 (Full block map) without the WHT ([RQ] Table 8 v2)
 *   SO3        R: v -> q v conj(q) per block, no WHT ([RQ] Table 8 v1; the
 *              parameters hold q in both slots)
 * isoq_quantize and isoq_dequantize take every variant; the decode entry
 * points take FULL, FAST and PLANAR (ISOQ_ERR_UNSUPPORTED otherwise).
 */
enum isoq_variant {
  ISOQ_FULL = 0,
  ISOQ_FAST = 1,
  ISOQ_PLANAR = 2,
  ISOQ_BLOCK_SO4 = 3,
  ISOQ_SO3 = 4
};

enum isoq_dtype {
  ISOQ_F16 = 0,   /* IEEE binary16 */
  ISOQ_F32 = 1    /* IEEE binary32 */
};

/* Human-readable name of a status code (static string). */
const char *isoq_status_string(int status);

/* Detail of the last error raised on the calling thread ("" if none). */
const char *isoq_last_error(void);

/* ABI version, incremented on any incompatible change. */
int isoq_abi_version(void);

/*
 * Floats of rotation parameters per head: 2*d ([RQ] Appendix B: d/4 blocks
 * of (q_L, q_R), 8 floats each, 256 at d = 128).  Returns a negative status
 * for unsupported d.
 */
int isoq_params_size(int d);

/*
 * Bytes of one packed vector: d*bits/8 ([RQ] §3.2 Step 4: 48 bytes at
 * d = 128, bits = 3).  Returns 0 for unsupported (d, bits).
 */
size_t isoq_packed_bytes(int d, int bits);

/*
 * Random rotation parameters ([RQ] §3.2 Algorithm 1 inputs, Appendix B;
 * [IQ] abstract), written to out_host[n_heads][d/4][8] (float32).
 * Generator: SplitMix64 (Steele, Lea & Flood 2014) seeded with `seed`
 * -> uniform doubles ((u >> 11) + 1) * 2^-53 in (0, 1] -> Box-Muller
 * (r cos, then r sin) -> standard normals.  Draw order: heads, blocks, q_L
 * (4 normals), q_R (4 normals); each quaternion is normalised in double and
 * rounded to float32.  ISOQ_FAST keeps Full's q_L (q_R's draws are still
 * consumed) and writes q_R = (1, 0, 0, 0); ISOQ_BLOCK_SO4 writes Full's
 * pair; ISOQ_SO3 writes Full's q_L in both slots; ISOQ_PLANAR normalises
 * the first two of each quaternion's four normals and writes
 * (c, s, 0, 0) for q_L and q_R.  Host only, no device work.
 */
int isoq_make_params(int d, int variant, uint64_t seed, int n_heads, float *out_host);

/*
 * Lloyd-Max codebook for N(0, 1/d) with 2^bits levels ([RQ] §3.2 Step 3):
 * centroids_host[2^bits] ascending and thresholds_host[2^bits - 1]
 * (midpoints of adjacent centroids), in double precision.  Computed by
 * Lloyd's iteration on the unit Gaussian, then scaled by 1/sqrt(d).  Either
 * output pointer may be NULL.  Host only.
 */
int isoq_make_codebook(int d, int bits, double *centroids_host, double *thresholds_host);

/*
 * Compress vectors ([RQ] §3.2 Algorithm 1; [IQ] abstract).
 *   x_dev      [n_heads][n_vec][d] elements of `dtype`, element (h, v, i) at
 *              x_dev + h*head_stride + v*vec_stride + i (strides in
 *              elements).  x_dev and both strides times the element size
 *              must be multiples of 16 bytes (the rows are loaded by TMA).
 *   params_dev [n_heads][d/4][8] float32 rotation parameters.
 *   codes_dev  packed codes of vector (h, v) at byte offset
 *              (h*out_head_stride + v) * d*bits/8; must be 16-byte aligned.
 *   norms_dev  float16 norm of vector (h, v) at index h*out_head_stride + v.
 *   out_head_stride  vectors between heads in the outputs (>= n_vec); lets a
 *              call write into a larger [heads][Tmax] cache.
 * Per vector: s = ||x||_2 (float32 accumulation); the stored norm is
 * float16(s) (round to nearest even); y = R_SO4(H_d x / (s sqrt d)) with
 * H_d the Sylvester Walsh-Hadamard matrix; code_i = #{k : y_i > t_k}.
 * A zero vector gets codes 2^(bits-1) - 1 and norm 0.
 * n_heads == 0 or n_vec == 0 is a no-op.
 */
int isoq_quantize(const void *x_dev, int dtype, int n_heads, int64_t n_vec, int d,
                  int bits, int variant, int64_t head_stride, int64_t vec_stride,
                  const float *params_dev, uint8_t *codes_dev, uint16_t *norms_dev,
                  int64_t out_head_stride, isoq_stream_t stream);

/*
 * Reconstruct vectors ([RQ] §3.4 Table 2 kernel D, Appendix A: R^-1 = R^T):
 *   out(h, v) = float(s16) * H_d(R_SO4^T c[codes]) / sqrt(d), stored as
 *   out_dtype at out_dev + h*head_stride + v*vec_stride (strides in
 *   elements; out_dev and vec_stride*elt must be 16-byte aligned).
 *   codes_dev / norms_dev use the layout of isoq_quantize with
 *   in_head_stride vectors between heads.
 */
int isoq_dequantize(const uint8_t *codes_dev, const uint16_t *norms_dev, int n_heads,
                    int64_t n_vec, int d, int bits, int variant, int64_t in_head_stride,
                    const float *params_dev, void *out_dev, int out_dtype,
                    int64_t head_stride, int64_t vec_stride, isoq_stream_t stream);

/*
 * Number of sequence splits the decode path uses for these shapes.  A
 * deterministic function of (B, Hkv, Tmax, d): every split covers a fixed
 * chunk of tokens, sized so that the grid fills the GPU.  Returns >= 1, or a
 * negative status on invalid shapes.
 */
int isoq_decode_num_splits(int B, int Hkv, int64_t Tmax, int d);

/*
 * Bytes of device workspace isoq_decode_attention needs: the split-K partial
 * states, B * Hq * n_splits * (d + 2) * 4 rounded up to 256, then the
 * prepared queries, B * Hkv * (24 d + 32) rounded up to 256.  Returns 0 on
 * invalid shapes.
 */
size_t isoq_decode_workspace_size(int B, int Hq, int Hkv, int64_t Tmax, int d);

/*
 * Fused decode attention directly on packed K/V ([RQ] Figure 1 bottom, §3.4
 * Table 2 kernels A-D, eq. (5), Appendix A).  For every batch row b and
 * query head qh (kvh = qh / (Hq / Hkv), T = min(max(seq_lens[b], 0), Tmax)):
 *   q~ = R_K q                                   (query rotated once)
 *   z_j = s^K_j * <q~, c[codeK_j]> * scale,  j < T   (packed QK, kernel A)
 *   alpha = softmax(z)                                  (kernel B, online)
 *   o~ = sum_j alpha_j s^V_j c[codeV_j]           (packed PV, kernel C)
 *   o = R_V^T o~                          (inverse rotation once, kernel D)
 * as split-K flash-decode: one kernel computes per-split partial
 * (max, sum, accumulator) states in the rotated domain, a second merges them
 * and applies the inverse rotation.  K and V are never dequantised to memory.
 *   q_dev        [B][Hq][d] of `dtype`, contiguous, 16-byte aligned.
 *   packed_k_dev, packed_v_dev  [B][Hkv][Tmax][d*bits/8], 16-byte aligned.
 *   norms_k_dev, norms_v_dev    [B][Hkv][Tmax] float16 bits.
 *   seq_lens_dev [B] int32; values <= 0 give a zero output row, values above
 *                Tmax are clamped to Tmax.
 *   params_k_dev, params_v_dev  [Hkv][d/4][8] float32 (separate K and V
 *                rotations; both use `variant`).
 *   scale        score scale, usually 1/sqrt(d).
 *   out_dev      [B][Hq][d] of `dtype`, contiguous.
 *   workspace_dev at least isoq_decode_workspace_size(...) bytes,
 *                256-byte aligned; its contents on entry do not matter.
 * Requires Hq % Hkv == 0 and Hq / Hkv <= 16.
 */
int isoq_decode_attention(const void *q_dev, int dtype, const uint8_t *packed_k_dev,
                          const uint8_t *packed_v_dev, const uint16_t *norms_k_dev,
                          const uint16_t *norms_v_dev, const int32_t *seq_lens_dev, int B,
                          int Hq, int Hkv, int64_t Tmax, int d, int bits, int variant,
                          const float *params_k_dev, const float *params_v_dev, float scale,
                          void *out_dev, void *workspace_dev, size_t workspace_bytes,
                          isoq_stream_t stream);

/*
 * The two launches of isoq_decode_attention, exposed separately so that a
 * caller can time or overlap them.  isoq_decode_split writes the partial
 * states into the workspace; isoq_decode_combine reads them and writes
 * out_dev.  Same arguments and rules as isoq_decode_attention.
 */
int isoq_decode_split(const void *q_dev, int dtype, const uint8_t *packed_k_dev,
                      const uint8_t *packed_v_dev, const uint16_t *norms_k_dev,
                      const uint16_t *norms_v_dev, const int32_t *seq_lens_dev, int B, int Hq,
                      int Hkv, int64_t Tmax, int d, int bits, int variant,
                      const float *params_k_dev, float scale, void *workspace_dev,
                      size_t workspace_bytes, isoq_stream_t stream);

int isoq_decode_combine(int dtype, const int32_t *seq_lens_dev, int B, int Hq, int Hkv,
                        int64_t Tmax, int d, int variant, const float *params_v_dev,
                        void *out_dev, const void *workspace_dev, size_t workspace_bytes,
                        isoq_stream_t stream);

/*
 * Decode attention for callers that cannot allocate device memory.  The
 * method's pages have no counterpart to this entry point; it is a
 * convenience of this library.
 *
 * Same computation, arguments and rules as isoq_decode_attention, without
 * the workspace arguments: the split-K partial states go to one device array
 * of isoq_decode_static_workspace_bytes() bytes (16 MiB) that the library
 * defines at file scope, so every GPU that loads the library holds it until
 * the process exits.  Intended for callers that have no device allocator of
 * their own to hand (a host program whose device memory is owned by another
 * framework, a plugin given only its input and output buffers, a path where
 * cudaMalloc's implicit synchronisation is not acceptable).  It calls no
 * cudaMalloc, cudaFree or other allocating routine.
 *   - Shapes whose workspace (isoq_decode_workspace_size) exceeds the array
 *     are rejected with ISOQ_ERR_UNSUPPORTED before any launch.
 *   - The first call on a device looks up the array's device address with
 *     cudaGetSymbolAddress and caches it, with the id of the CUDA context it
 *     belongs to; make that first call before any stream capture on that
 *     device.  A device reset (cudaDeviceReset) ends that context, and the
 *     array's contents with it: the first call in the new context notices
 *     the new context id and looks the address up again, so that call too
 *     belongs before any capture.
 *   - All calls share the one array and it keeps the last call's contents
 *     (nothing in it needs clearing: each call writes every slot it reads).
 *     Calls whose kernels overlap on the GPU, e.g. on two streams without an
 *     ordering between them, race on it.
 */
size_t isoq_decode_static_workspace_bytes(void);
int isoq_decode_attention_static(const void *q_dev, int dtype, const uint8_t *packed_k_dev,
                                 const uint8_t *packed_v_dev, const uint16_t *norms_k_dev,
                                 const uint16_t *norms_v_dev, const int32_t *seq_lens_dev, int B,
                                 int Hq, int Hkv, int64_t Tmax, int d, int bits, int variant,
                                 const float *params_k_dev, const float *params_v_dev,
                                 float scale, void *out_dev, isoq_stream_t stream);

/*
 * Decode-step append ([RQ] §3.2 Algorithm 1 on the new token; Figure 1 and
 * Appendix D: each decode step compresses its new K/V entry once and writes
 * it into the packed cache that the fused attention reads).  For every batch
 * row b and KV head kvh, with p = max(seq_lens[b], 0):
 *   compress k_new[b][kvh] with params_k[kvh] and v_new[b][kvh] with
 *   params_v[kvh] (float32 norm, rotation, Lloyd-Max codes against the
 *   norm-scaled thresholds) into packed_k/v[b][kvh][p] and norms_k/v[b][kvh][p],
 *   then set seq_lens[b] = p + 1.
 *   k_new_dev, v_new_dev  [B][Hkv][d] of `dtype`, 16-byte aligned.
 *   packed_*, norms_*, params_*, seq_lens_dev: the cache and rotations of
 *                isoq_decode_attention (read and written in place).
 * A row with p >= Tmax is left unchanged; the next isoq_check_device_error
 * reports ISOQ_ERR_INVALID_ARG for it.  Argument errors as isoq_quantize.
 * The bulk compression of an FP16 prefill buffer at the prefill-to-decode
 * boundary ([RQ] Appendix C) is isoq_quantize on that buffer.
 */
int isoq_decode_append(const void *k_new_dev, const void *v_new_dev, int dtype,
                       uint8_t *packed_k_dev, uint8_t *packed_v_dev, uint16_t *norms_k_dev,
                       uint16_t *norms_v_dev, int32_t *seq_lens_dev, int B, int Hkv, int64_t Tmax,
                       int d, int bits, int variant, const float *params_k_dev,
                       const float *params_v_dev, isoq_stream_t stream);

/*
 * One decode step: isoq_decode_append of (k_new, v_new), then
 * isoq_decode_attention of q over the cache including the new token, all on
 * `stream` (four to five launches, no host synchronisation).  Arguments as
 * those two functions.  Every argument of both halves is checked before
 * anything is launched: a call that returns an error status has written
 * nothing.
 */
int isoq_decode_step(const void *q_dev, const void *k_new_dev, const void *v_new_dev, int dtype,
                     uint8_t *packed_k_dev, uint8_t *packed_v_dev, uint16_t *norms_k_dev,
                     uint16_t *norms_v_dev, int32_t *seq_lens_dev, int B, int Hq, int Hkv,
                     int64_t Tmax, int d, int bits, int variant, const float *params_k_dev,
                     const float *params_v_dev, float scale, void *out_dev, void *workspace_dev,
                     size_t workspace_bytes, isoq_stream_t stream);

/*
 * Chunked prefill: causal attention of Tq new queries over the packed cache
 * that already holds them ([RQ] §3.4: kernel A "benefits from early
 * termination via causal masking"; Figure 1's compressed-space path with
 * more than one query).  Query t of batch row b sits at position
 * p = seq_lens[b] - Tq + t and attends to the tokens j <= p (j < Tmax);
 * queries with p < 0 get zero rows.  Each output row is what
 * isoq_decode_attention gives for that query over p + 1 tokens.
 *   q_dev      [B][Tq][Hq][d] float16 (dtype ISOQ_F16; 4-byte aligned)
 *   out_dev    [B][Tq][Hq][d] float16, written (4-byte aligned)
 *   the cache, seq_lens, parameters, scale: as isoq_decode_attention
 *              (seq_lens[b] counts the chunk; the chunk's K/V are written
 *              first, e.g. by isoq_quantize into the cache rows).
 * Tensor-core path: d in {128, 256}, bits = 3, Hq/Hkv in {1, 2, 4, 8},
 * variants FULL, FAST and PLANAR; anything else is ISOQ_ERR_UNSUPPORTED.
 * Tq = 0 is a no-op.  No workspace; one launch.  The kernel checks that its
 * dynamic shared memory starts on a 1024-byte boundary (its d = 128 layout
 * keeps no room to align it); otherwise it writes nothing and the next
 * isoq_check_device_error returns ISOQ_ERR_CUDA.
 */
int isoq_prefill_attention(const void *q_dev, int dtype, const uint8_t *packed_k_dev,
                           const uint8_t *packed_v_dev, const uint16_t *norms_k_dev,
                           const uint16_t *norms_v_dev, const int32_t *seq_lens_dev, int B, int Tq,
                           int Hq, int Hkv, int64_t Tmax, int d, int bits, int variant,
                           const float *params_k_dev, const float *params_v_dev, float scale,
                           void *out_dev, isoq_stream_t stream);

/*
 * RotorQuant comparator (the RotorQuant page; [IQ] abstract compares
 * IsoQuant's kernels with it on the stage-1 path).  Each vector is padded
 * to 3G dimensions, G = ceil(d / 3), each group of three is rotated by its
 * own unit rotor R = s + p12 e12 + p13 e13 + p23 e23 of Cl(3,0) with the
 * sandwich R v rev(R), and all 3G rotated coordinates get the Lloyd-Max
 * codes of isoq_make_codebook (N(0, 1/d)), packed as one LSB-first
 * bitstream (code i at bits [b i, b i + b)) padded to whole 32-bit words;
 * the float16 norm is stored as for isoq_quantize.
 *
 * isoq_rotor_groups(d): G, or ISOQ_ERR_UNSUPPORTED.
 * isoq_rotor_packed_bytes(d, bits): 4 ceil(3 G bits / 32) (52 at d = 128,
 *   bits = 3), or 0 for unsupported arguments.
 * isoq_rotor_make_params: out_host[n_heads][G][4] = (s, p12, p13, p23),
 *   four normals per group from the generator of isoq_make_params,
 *   normalised in double, rounded to float32.  Host only.
 * isoq_rotor_quantize / isoq_rotor_dequantize: arguments, layouts, strides
 *   and errors as isoq_quantize / isoq_dequantize, with rotors_dev
 *   [n_heads][G][4] (16-byte aligned) in place of the rotation parameters,
 *   codes of isoq_rotor_packed_bytes per vector (4-byte aligned).
 */
int isoq_rotor_groups(int d);
size_t isoq_rotor_packed_bytes(int d, int bits);
int isoq_rotor_make_params(int d, uint64_t seed, int n_heads, float *out_host);
int isoq_rotor_quantize(const void *x_dev, int dtype, int n_heads, int64_t n_vec, int d, int bits,
                        int64_t head_stride, int64_t vec_stride, const float *rotors_dev,
                        uint8_t *codes_dev, uint16_t *norms_dev, int64_t out_head_stride,
                        isoq_stream_t stream);
int isoq_rotor_dequantize(const uint8_t *codes_dev, const uint16_t *norms_dev, int n_heads,
                          int64_t n_vec, int d, int bits, int64_t in_head_stride,
                          const float *rotors_dev, void *out_dev, int out_dtype,
                          int64_t head_stride, int64_t vec_stride, isoq_stream_t stream);

/*
 * Reads and clears the current device's error word after synchronising
 * `stream`.  Returns ISOQ_OK, ISOQ_ERR_TIMEOUT if a kernel's bounded wait
 * gave up since the last check (the kernel then stopped early and its
 * outputs are incomplete), ISOQ_ERR_INVALID_ARG if a decode append met a
 * row that already held Tmax tokens, or ISOQ_ERR_CUDA (among others when
 * the prefill kernel found its dynamic shared memory off a 1024-byte
 * boundary and returned without output).
 */
int isoq_check_device_error(isoq_stream_t stream);

/*
 * Failure-path self-test: launches one thread that waits on a device
 * mbarrier that nothing arrives at, polling it like the kernels' bounded
 * waits, for limit_ns nanoseconds of the GPU timer (0 < limit_ns <= 1e9;
 * at most 2^24 polls should the timer stall), and then records a timeout in
 * the device error word, exactly as a pipeline wait that gives up does.
 * The next isoq_check_device_error on `stream` returns ISOQ_ERR_TIMEOUT and
 * clears the word; the context stays usable.  Returns ISOQ_OK once launched,
 * ISOQ_ERR_INVALID_ARG for a limit out of range, ISOQ_ERR_CUDA on a launch
 * failure.  Touches no buffer.
 */
int isoq_selftest_wait_timeout(uint64_t limit_ns, isoq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* ISOQ_H */
