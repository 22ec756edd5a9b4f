// Arguments and internal entry points of the decode kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace isoq {
namespace decode {

constexpr int kMaxGroup = 16;  // query heads per KV head

struct SplitArgs {
  const void *q;
  const uint8_t *packed_k;
  const uint8_t *packed_v;
  const uint16_t *norms_k;
  const uint16_t *norms_v;
  const int32_t *seq_lens;
  const float *params_k;
  float *ws_acc;   // [B][Hq][n_splits][d]
  float2 *ws_ml;   // [B][Hq][n_splits] (max, sum)
  uint32_t *ws_qprep;  // [B][Hkv][decode_qprep_words(d)] prepared queries (int8 path)
  long long tmax;
  long long chunk;  // tokens per split
  int batch, hq, hkv, group, n_splits;
  float scale;
  float centroid[16];
};

struct CombineArgs {
  const float *params_v;
  void *out;
  const float *ws_acc;
  const float2 *ws_ml;
  int batch, hq, group, n_splits;
};

bool i8_path_supported(int dtype, int d, int bits, const SplitArgs &a);
int run_split_i8(int d, int variant, const SplitArgs &a, cudaStream_t stream);

}  // namespace decode
}  // namespace isoq
