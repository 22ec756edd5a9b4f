// Device error word collection: each kernel translation unit owns one 32-bit
// word per device that its bounded waits set when they give up.

#include <cuda_runtime.h>

#include "internal.h"

extern "C" __attribute__((visibility("hidden"))) int isoq_detail_take_quant_error(cudaStream_t stream, unsigned *out);
extern "C" __attribute__((visibility("hidden"))) int isoq_detail_take_decode_error(cudaStream_t stream, unsigned *out);

extern "C" int isoq_check_device_error(isoq_stream_t stream) {
  isoq::clear_error();
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned q = 0, d = 0;
  int st = isoq_detail_take_quant_error(s, &q);
  if (st) return st;
  st = isoq_detail_take_decode_error(s, &d);
  if (st) return st;
  // Bit 1: a bounded wait gave up.  Bit 2: a decode append found a full row.
  // Bit 4: the prefill kernel found its shared memory misaligned.
  if ((q | d) & 1u)
    return isoq::set_error(ISOQ_ERR_TIMEOUT, "device wait timed out (quantize=%u, decode=%u)", q, d);
  if (d & 2u)
    return isoq::set_error(ISOQ_ERR_INVALID_ARG, "decode append: a row already held Tmax tokens");
  if (d & 4u)
    return isoq::set_error(ISOQ_ERR_CUDA, "prefill: dynamic shared memory not 1024-byte aligned");
  return ISOQ_OK;
}
