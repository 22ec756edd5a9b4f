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

}  // namespace isoq
