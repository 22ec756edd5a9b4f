// Host-only part of libisoq: status strings, error reporting, the rotation
// parameter generator, the Lloyd-Max codebook and the decode split policy.
// Nothing here touches the GPU.

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "internal.h"

namespace isoq {

namespace {
thread_local char g_last_error[512] = "";
}

int set_error(int status, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return status;
}

void clear_error() { g_last_error[0] = '\0'; }

bool supported_d(int d) { return d == 128 || d == 256 || d == 512; }
bool supported_bits(int bits) { return bits >= 2 && bits <= 4; }
bool supported_variant(int v) { return v >= ISOQ_FULL && v <= ISOQ_SO3; }
bool supported_decode_variant(int v) { return v == ISOQ_FULL || v == ISOQ_FAST || v == ISOQ_PLANAR; }
bool supported_dtype(int t) { return t == ISOQ_F16 || t == ISOQ_F32; }

// ---------------------------------------------------------------------------
// Lloyd-Max quantiser for the unit Gaussian (RotaryQuant §3.2 Step 3).
// Lloyd's iteration: thresholds at midpoints of adjacent centroids, each
// centroid the conditional mean (phi(a) - phi(b)) / (Phi(b) - Phi(a)) of its
// cell.  The fixed point of an even log-concave density is unique and odd
// symmetric; each iterate is symmetrised so rounding cannot break that.
// ---------------------------------------------------------------------------
namespace {

double phi(double x) {
  if (std::isinf(x)) return 0.0;
  return std::exp(-0.5 * x * x) / std::sqrt(2.0 * M_PI);
}

// P(a < X < b), X ~ N(0, 1), in the tail form that keeps precision.
double cell_mass(double a, double b) {
  const double r2 = std::sqrt(2.0);
  if (a >= 0.0) return 0.5 * (std::erfc(a / r2) - std::erfc(b / r2));
  if (b <= 0.0) return 0.5 * (std::erfc(-b / r2) - std::erfc(-a / r2));
  return 1.0 - 0.5 * std::erfc(b / r2) - 0.5 * std::erfc(-a / r2);
}

double normal_quantile(double p) {
  double lo = -40.0, hi = 40.0;
  for (int i = 0; i < 200; ++i) {
    double mid = 0.5 * (lo + hi);
    if (0.5 * std::erfc(-mid / std::sqrt(2.0)) < p)
      lo = mid;
    else
      hi = mid;
  }
  return 0.5 * (lo + hi);
}

void lloyd_max_unit(int bits, double *c, double *t) {
  const int L = 1 << bits;
  double cur[kMaxLevels], nxt[kMaxLevels], edge[kMaxLevels + 1];
  for (int k = 0; k < L; ++k) cur[k] = normal_quantile((k + 0.5) / L);
  for (int k = 0; k < L / 2; ++k) {
    double m = 0.5 * (cur[L - 1 - k] - cur[k]);
    cur[L - 1 - k] = m;
    cur[k] = -m;
  }
  for (int it = 0; it < 100000; ++it) {
    edge[0] = -INFINITY;
    edge[L] = INFINITY;
    for (int k = 0; k + 1 < L; ++k) edge[k + 1] = 0.5 * (cur[k] + cur[k + 1]);
    for (int k = 0; k < L; ++k)
      nxt[k] = (phi(edge[k]) - phi(edge[k + 1])) / cell_mass(edge[k], edge[k + 1]);
    double delta = 0.0;
    for (int k = 0; k < L; ++k) {
      double v = 0.5 * (nxt[k] - nxt[L - 1 - k]);
      delta = std::fmax(delta, std::fabs(v - cur[k]));
      nxt[k] = v;
    }
    std::memcpy(cur, nxt, sizeof(double) * L);
    if (delta <= 2e-15) break;
  }
  for (int k = 0; k < L; ++k) c[k] = cur[k];
  for (int k = 0; k + 1 < L; ++k) t[k] = 0.5 * (cur[k] + cur[k + 1]);
}

struct UnitCodebook {
  bool ready = false;
  double c[kMaxLevels];
  double t[kMaxLevels - 1];
};

std::mutex g_cb_mutex;
UnitCodebook g_unit[5];  // indexed by bits

const UnitCodebook &unit_codebook(int bits) {
  std::lock_guard<std::mutex> lock(g_cb_mutex);
  UnitCodebook &u = g_unit[bits];
  if (!u.ready) {
    lloyd_max_unit(bits, u.c, u.t);
    u.ready = true;
  }
  return u;
}

// SplitMix64 (Steele, Lea & Flood, OOPSLA 2014).
struct SplitMix64 {
  uint64_t s;
  uint64_t next() {
    s += 0x9E3779B97F4A7C15ull;
    uint64_t z = s;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
  }
  double uniform() { return static_cast<double>((next() >> 11) + 1) * 0x1.0p-53; }
};

// Box-Muller: each uniform pair gives r*cos(2 pi u2), then r*sin(2 pi u2).
struct Gaussian {
  SplitMix64 rng;
  double spare = 0.0;
  bool has_spare = false;
  double next() {
    if (has_spare) {
      has_spare = false;
      return spare;
    }
    double u1 = rng.uniform(), u2 = rng.uniform();
    double r = std::sqrt(-2.0 * std::log(u1));
    double th = 2.0 * M_PI * u2;
    spare = r * std::sin(th);
    has_spare = true;
    return r * std::cos(th);
  }
};

}  // namespace

bool codebook_f32(int d, int bits, CodebookF32 *out) {
  if (!supported_d(d) || !supported_bits(bits)) return false;
  const UnitCodebook &u = unit_codebook(bits);
  const double sigma = 1.0 / std::sqrt(static_cast<double>(d));
  out->levels = 1 << bits;
  for (int k = 0; k < out->levels; ++k) out->centroid[k] = static_cast<float>(u.c[k] * sigma);
  for (int k = 0; k + 1 < out->levels; ++k)
    out->threshold[k] = static_cast<float>(u.t[k] * sigma);
  return true;
}

bool codebook_unit_f64(int bits, double *centroids) {
  if (!supported_bits(bits)) return false;
  const UnitCodebook &u = unit_codebook(bits);
  for (int k = 0; k < (1 << bits); ++k) centroids[k] = u.c[k];
  return true;
}

// Each split covers a fixed number of tokens, one of 512, 768, 1024, 1536,
// 2048, 3072 or 4096 (below 512 tokens a split's fixed costs, its set-up and
// its share of the combine, outweigh the parallelism it adds).  The chunk c
// minimises a wave model of the split kernel on a 148-SM B200 with 4 CTAs
// resident per SM:
//   the busiest SM runs m = ceil(n_ctas / 148) CTAs, n_ctas = B Hkv
//   ceil(Tmax / c), in phases of k = min(4, remaining) concurrent CTAs; a
//   phase costs (k + 0.7) (min(c, Tmax) + 160)
// (an SM with k CTAs moves k / (k + 0.7) of its full rate: one CTA's four
// warps hide little latency; each CTA costs about 160 tokens' worth of
// set-up and merge).  Ties go to the larger chunk (fewer partial states to
// combine).  The constants are fitted to the split time over these chunks
// on 17 shapes (batch 1..32, 8 or 4 KV heads, d = 128 and 256, contexts
// 1K..64K): the chunk the model picks is within 7 % of the fastest one on
// every shape, where a fixed target of 8 CTAs per SM lost up to 11 % to a
// nearly empty last wave.
int64_t decode_chunk_tokens(int B, int Hkv, int64_t Tmax, int d) {
  (void)d;
  static constexpr int64_t kChunks[] = {4096, 3072, 2048, 1536, 1024, 768, 512};
  constexpr int64_t kSms = 148, kSlots = 4, kCtaCost = 160;
  const int64_t pairs = static_cast<int64_t>(B) * Hkv;
  int64_t best_chunk = 4096, best_cost = -1;
  for (const int64_t c : kChunks) {
    const int64_t n_ctas = pairs * ((Tmax + c - 1) / c);
    int64_t m = (n_ctas + kSms - 1) / kSms, phases10 = 0;   // sum of 10 (k + 0.7)
    while (m > 0) {
      const int64_t k = m < kSlots ? m : kSlots;
      phases10 += 10 * k + 7;
      m -= k;
    }
    const int64_t cost = phases10 * ((c < Tmax ? c : Tmax) + kCtaCost);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best_chunk = c;
    }
  }
  return best_chunk;
}

size_t decode_qprep_bytes(int B, int Hkv, int d) {
  const size_t n = static_cast<size_t>(B) * Hkv * decode_qprep_words(d) * 4;
  return (n + 255) / 256 * 256;
}

int decode_num_splits(int B, int Hkv, int64_t Tmax, int d) {
  int64_t chunk = decode_chunk_tokens(B, Hkv, Tmax, d);
  int64_t n = (Tmax + chunk - 1) / chunk;
  return n < 1 ? 1 : static_cast<int>(n);
}

}  // namespace isoq

using namespace isoq;

extern "C" {

const char *isoq_status_string(int status) {
  switch (status) {
    case ISOQ_OK: return "ok";
    case ISOQ_ERR_INVALID_ARG: return "invalid argument";
    case ISOQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case ISOQ_ERR_CUDA: return "CUDA error";
    case ISOQ_ERR_TIMEOUT: return "device wait timed out";
    default: return "unknown status";
  }
}

const char *isoq_last_error(void) { return g_last_error; }

int isoq_abi_version(void) { return 1; }

int isoq_params_size(int d) {
  if (!supported_d(d)) return ISOQ_ERR_UNSUPPORTED;
  return 2 * d;
}

size_t isoq_packed_bytes(int d, int bits) {
  if (!supported_d(d) || !supported_bits(bits)) return 0;
  return static_cast<size_t>(d) * bits / 8;
}

int isoq_make_params(int d, int variant, uint64_t seed, int n_heads, float *out_host) {
  clear_error();
  if (!supported_d(d)) return set_error(ISOQ_ERR_UNSUPPORTED, "d=%d not supported", d);
  if (!supported_variant(variant))
    return set_error(ISOQ_ERR_UNSUPPORTED, "variant=%d not supported", variant);
  if (n_heads < 0) return set_error(ISOQ_ERR_INVALID_ARG, "n_heads < 0");
  if (n_heads > 0 && !out_host) return set_error(ISOQ_ERR_INVALID_ARG, "out_host is NULL");
  Gaussian g;
  g.rng.s = seed;
  float *p = out_host;
  for (int h = 0; h < n_heads; ++h) {
    for (int i = 0; i < d / 4; ++i) {
      double q[8];
      for (int k = 0; k < 8; ++k) q[k] = g.next();
      if (variant == ISOQ_PLANAR) q[2] = q[3] = q[6] = q[7] = 0.0;   // the complex line
      for (int half = 0; half < 2; ++half) {
        double *v = q + 4 * half;
        double n = std::sqrt(v[0] * v[0] + v[1] * v[1] + v[2] * v[2] + v[3] * v[3]);
        for (int k = 0; k < 4; ++k) v[k] = v[k] / n;
      }
      for (int k = 0; k < 4; ++k) p[k] = static_cast<float>(q[k]);
      if (variant == ISOQ_FAST) {
        p[4] = 1.0f;
        p[5] = p[6] = p[7] = 0.0f;
      } else {
        const double *r = variant == ISOQ_SO3 ? q : q + 4;
        for (int k = 0; k < 4; ++k) p[4 + k] = static_cast<float>(r[k]);
      }
      p += 8;
    }
  }
  return ISOQ_OK;
}

int isoq_rotor_make_params(int d, uint64_t seed, int n_heads, float *out_host) {
  clear_error();
  if (!supported_d(d)) return set_error(ISOQ_ERR_UNSUPPORTED, "d=%d not supported", d);
  if (n_heads < 0) return set_error(ISOQ_ERR_INVALID_ARG, "n_heads < 0");
  if (n_heads > 0 && !out_host) return set_error(ISOQ_ERR_INVALID_ARG, "out_host is NULL");
  const int G = (d + 2) / 3;
  Gaussian g;
  g.rng.s = seed;
  float *p = out_host;
  for (int h = 0; h < n_heads; ++h) {
    for (int k = 0; k < G; ++k) {
      double v[4];
      for (int j = 0; j < 4; ++j) v[j] = g.next();
      const double n = std::sqrt(v[0] * v[0] + v[1] * v[1] + v[2] * v[2] + v[3] * v[3]);
      for (int j = 0; j < 4; ++j) p[j] = static_cast<float>(v[j] / n);
      p += 4;
    }
  }
  return ISOQ_OK;
}

int isoq_make_codebook(int d, int bits, double *centroids_host, double *thresholds_host) {
  clear_error();
  if (!supported_d(d)) return set_error(ISOQ_ERR_UNSUPPORTED, "d=%d not supported", d);
  if (!supported_bits(bits)) return set_error(ISOQ_ERR_UNSUPPORTED, "bits=%d not supported", bits);
  const UnitCodebook &u = unit_codebook(bits);
  const double sigma = 1.0 / std::sqrt(static_cast<double>(d));
  const int L = 1 << bits;
  if (centroids_host)
    for (int k = 0; k < L; ++k) centroids_host[k] = u.c[k] * sigma;
  if (thresholds_host)
    for (int k = 0; k + 1 < L; ++k) thresholds_host[k] = u.t[k] * sigma;
  return ISOQ_OK;
}

int isoq_decode_num_splits(int B, int Hkv, int64_t Tmax, int d) {
  if (B <= 0 || Hkv <= 0 || Tmax <= 0) return ISOQ_ERR_INVALID_ARG;
  if (!supported_d(d)) return ISOQ_ERR_UNSUPPORTED;
  return decode_num_splits(B, Hkv, Tmax, d);
}

size_t isoq_decode_workspace_size(int B, int Hq, int Hkv, int64_t Tmax, int d) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Tmax <= 0 || !supported_d(d) || Hq % Hkv) return 0;
  size_t n = static_cast<size_t>(B) * Hq * decode_num_splits(B, Hkv, Tmax, d) * (d + 2) * 4;
  n = (n + 255) / 256 * 256;
  return n + decode_qprep_bytes(B, Hkv, d);
}

}  // extern "C"
