// Host-side internals shared by the translation units of libisoq.
#pragma once

#include <cstddef>
#include <cstdint>

#include "isoq.h"

namespace isoq {

// Largest supported codebook (bits = 4).
constexpr int kMaxLevels = 16;

// Thread-local error message setter; returns `status` for chaining.
int set_error(int status, const char *fmt, ...);
void clear_error();

bool supported_d(int d);
bool supported_bits(int bits);
bool supported_variant(int v);
// Variants the decode path takes; block_map_variant gives the one whose
// block map the decode kernels apply (PLANAR's parameters make the Full map
// its two plane rotations).
bool supported_decode_variant(int v);
inline int block_map_variant(int v) { return v == ISOQ_FAST ? ISOQ_FAST : ISOQ_FULL; }
bool supported_dtype(int t);
inline int elt_size(int dtype) { return dtype == ISOQ_F16 ? 2 : 4; }

// Float32 codebook for N(0, 1/d): centroids[L], thresholds[L-1] (L = 2^bits).
struct CodebookF32 {
  float centroid[kMaxLevels];
  float threshold[kMaxLevels - 1];
  int levels;
};
// Memoised; safe to call from several threads.  Returns false on bad args.
bool codebook_f32(int d, int bits, CodebookF32 *out);
// Centroids of the unit-variance (N(0, 1)) codebook in double, L = 2^bits.
bool codebook_unit_f64(int bits, double *centroids);

// Split policy of the decode path.
constexpr int kDecodeTokenQuantum = 64;   // chunk sizes are multiples of this
int64_t decode_chunk_tokens(int B, int Hkv, int64_t Tmax, int d);
int decode_num_splits(int B, int Hkv, int64_t Tmax, int d);
// Per (b, kvh): the prepared query of the int8 decode path, as the B-fragment
// words of up to 3 N tiles x d/32 k-steps x 2 halves x 32 lanes, then 8
// per-head score factors (float32).
constexpr int decode_qprep_words(int d) { return 3 * (d / 32) * 2 * 32 + 8; }
size_t decode_qprep_bytes(int B, int Hkv, int d);

}  // namespace isoq
