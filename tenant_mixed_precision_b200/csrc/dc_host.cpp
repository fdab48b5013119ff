// Host side of the library: error text, descriptor checks, the round-to-nearest quantiser,
// the host packer and the uploads.  No device memory is allocated here.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <thread>
#include <vector>

#include "dc.h"
#include "dc_internal.h"
#include "dc_layout.h"
#include "dc_pack.h"

static thread_local char g_err[512] = "";

dc_status dc_fail(dc_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

dc_status dc_cuda_check(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return DC_OK;
  return dc_fail(DC_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

void dc_clear_error() { g_err[0] = 0; }

extern "C" const char* dc_last_error(void) { return g_err; }

extern "C" const char* dc_version(void) { return "dc-b200 0.1 (sm_100a)"; }

dc_status dc_check_desc(const dc_factor_desc* d, DcLayout* L) {
  if (!d) return dc_fail(DC_ERR_INVALID_ARG, "null descriptor");
  if (d->d_out <= 0 || d->d_in <= 0 || d->d_out % DC_GROUP || d->d_in % DC_GROUP)
    return dc_fail(DC_ERR_SHAPE, "d_out=%d d_in=%d must be positive multiples of 128", d->d_out, d->d_in);
  if (d->n_bands < 0 || d->n_bands > DC_MAX_BANDS)
    return dc_fail(DC_ERR_INVALID_ARG, "n_bands=%d outside 0..%d", d->n_bands, DC_MAX_BANDS);
  int64_t r = 0;
  for (int i = 0; i < d->n_bands; ++i) {
    if (!dc_bits_ok(d->bits[i])) return dc_fail(DC_ERR_BITS, "band %d: bits=%d not in {0,2,3,8}", i, d->bits[i]);
    if (d->rank[i] < 0) return dc_fail(DC_ERR_SHAPE, "band %d: negative rank", i);
    if (d->bits[i]) r += d->rank[i];
  }
  const int64_t cap = d->d_out < d->d_in ? d->d_out : d->d_in;
  if (r > cap) return dc_fail(DC_ERR_SHAPE, "total rank %lld exceeds min(d_out, d_in)=%lld", (long long)r, (long long)cap);
  DcLayout l = dc_layout(*d);
  if (!l.valid) return dc_fail(DC_ERR_INVALID_ARG, "invalid descriptor");
  if (L) *L = l;
  return DC_OK;
}

extern "C" size_t dc_packed_size(const dc_factor_desc* desc) {
  DC_NVTX("dc_packed_size");
  DcLayout L;
  if (dc_check_desc(desc, &L) != DC_OK) return 0;
  return (size_t)L.bytes;
}

// ---------------------------------------------------------------------------------------------
// fp16 <-> fp64 with one correct rounding (round to nearest, ties to even)
// ---------------------------------------------------------------------------------------------
uint16_t dc_f64_to_f16(double x) {
  uint64_t u;
  std::memcpy(&u, &x, 8);
  const uint16_t sign = (uint16_t)((u >> 48) & 0x8000u);
  const double a = std::fabs(x);
  if (std::isnan(x)) return (uint16_t)(sign | 0x7E00u);
  if (std::isinf(a)) return (uint16_t)(sign | 0x7C00u);
  if (a < 0x1p-14) {  // subnormal range: quantum 2^-24 (exact scaling, one rounding)
    const double n = std::nearbyint(a * 0x1p24);
    return (uint16_t)(sign | (uint16_t)n);  // n == 1024 is the smallest normal, bit-compatible
  }
  int E;
  std::frexp(a, &E);  // a = f * 2^E, f in [0.5, 1)
  int e = E - 1;      // a in [2^e, 2^(e+1))
  double n = std::nearbyint(std::ldexp(a, 10 - e));  // in [1024, 2048]
  if (n >= 2048.0) {
    n = 1024.0;
    e += 1;
  }
  if (e > 15) return (uint16_t)(sign | 0x7C00u);
  return (uint16_t)(sign | (uint16_t)((e + 15) << 10) | (uint16_t)(n - 1024.0));
}

double dc_f16_to_f64(uint16_t h) {
  const int s = (h >> 15) & 1, e = (h >> 10) & 31, m = h & 1023;
  double v;
  if (e == 0)
    v = std::ldexp((double)m, -24);
  else if (e == 31)
    v = m ? NAN : INFINITY;
  else
    v = std::ldexp((double)(1024 + m), e - 25);
  return s ? -v : v;
}

// One group of RTN: the rule stated in dc.h.  Returns false on a non-finite value or an fp16
// scale overflow.
bool dc_rtn_group(const float* v, int64_t stride, int n, int bits, uint8_t* codes, int64_t cstride, uint16_t* sz) {
  const double qmax = (double)((1 << bits) - 1);
  double lo = 0.0, hi = 0.0;
  for (int i = 0; i < n; ++i) {
    const double x = v[i * stride];
    if (!std::isfinite(x)) return false;
    lo = x < lo ? x : lo;
    hi = x > hi ? x : hi;
  }
  const uint16_t sh = dc_f64_to_f16((hi - lo) / qmax);
  double sc = dc_f16_to_f64(sh);
  if (!std::isfinite(sc)) return false;
  uint16_t shs = sh;
  if (sc == 0.0) {
    sc = 1.0;
    shs = 0x3C00u;
  }
  double z = std::nearbyint(-lo / sc);
  z = z < 0 ? 0 : (z > qmax ? qmax : z);
  for (int i = 0; i < n; ++i) {
    double c = std::nearbyint((double)v[i * stride] / sc) + z;
    c = c < 0 ? 0 : (c > qmax ? qmax : c);
    codes[i * cstride] = (uint8_t)c;
  }
  sz[0] = shs;
  sz[1] = dc_f64_to_f16(z);
  return true;
}

extern "C" dc_status dc_quantize_rtn(const dc_factor_desc* desc, const float* U, const float* Vt,
                                     uint8_t* codes_u, uint8_t* codes_v, uint16_t* sz_u, uint16_t* sz_v) {
  DC_NVTX("dc_quantize_rtn");
  dc_clear_error();
  DcLayout L;
  dc_status st = dc_check_desc(desc, &L);
  if (st) return st;
  if (L.r > 0 && (!U || !Vt || !codes_u || !codes_v || !sz_u || !sz_v))
    return dc_fail(DC_ERR_INVALID_ARG, "null host buffer");
  const int32_t d_out = L.d_out, d_in = L.d_in, r = L.r;
  std::vector<int> bits_of(r);
  for (int b = 0; b < L.n_bands; ++b)
    for (int i = 0; i < L.band[b].rank; ++i) bits_of[L.band[b].r0 + i] = L.band[b].bits;
  unsigned nth = std::thread::hardware_concurrency();
  if (nth == 0) nth = 1;
  if (nth > 32) nth = 32;
  std::vector<int> bad(nth, -1);
  auto work = [&](unsigned tid) {
    for (int i = (int)tid; i < r; i += (int)nth) {
      const int bits = bits_of[i];
      for (int g = 0; g < L.groups_in; ++g)
        if (!dc_rtn_group(Vt + (int64_t)i * d_in + g * 128, 1, 128, bits, codes_v + (int64_t)i * d_in + g * 128, 1,
                       sz_v + ((int64_t)i * L.groups_in + g) * 2))
          bad[tid] = i;
      for (int g = 0; g < L.groups_out; ++g)
        if (!dc_rtn_group(U + (int64_t)i * d_out + g * 128, 1, 128, bits, codes_u + (int64_t)i * d_out + g * 128, 1,
                       sz_u + ((int64_t)i * L.groups_out + g) * 2))
          bad[tid] = i;
    }
  };
  std::vector<std::thread> th;
  for (unsigned t = 1; t < nth; ++t) th.emplace_back(work, t);
  work(0);
  for (auto& t : th) t.join();
  for (unsigned t = 0; t < nth; ++t)
    if (bad[t] >= 0)
      return dc_fail(DC_ERR_INVALID_ARG, "rank %d: non-finite factor value or fp16 scale overflow", bad[t]);
  return DC_OK;
}

// Host packing of a whole blob (every word through dc_pack_word).
void dc_pack_host(const DcLayout& L, const DcPlain& P, uint8_t* blob) {
  const int64_t nw = L.bytes / 4;
  unsigned nth = std::thread::hardware_concurrency();
  if (nth == 0) nth = 1;
  if (nth > 32) nth = 32;
  auto work = [&](unsigned tid) {
    uint32_t* w = reinterpret_cast<uint32_t*>(blob);
    const int64_t chunk = (nw + nth - 1) / nth;
    const int64_t a = chunk * tid, b = (a + chunk < nw) ? a + chunk : nw;
    for (int64_t i = a; i < b; ++i) w[i] = dc_pack_word(L, i * 4, P);
  };
  std::vector<std::thread> th;
  for (unsigned t = 1; t < nth; ++t) th.emplace_back(work, t);
  work(0);
  for (auto& t : th) t.join();
}

void dc_fill_handle(const dc_factor_desc* desc, const DcLayout& L, void* dev, dc_delta_handle* out) {
  std::memset(out, 0, sizeof(*out));
  out->dev_base = (uint64_t)(uintptr_t)dev;
  out->bytes = (uint64_t)L.bytes;
  out->desc = *desc;
  out->rank_total = L.r;
}

extern "C" dc_status dc_pack_upload(const dc_factor_desc* desc, const uint8_t* codes_u, const uint8_t* codes_v,
                                    const uint16_t* sz_u, const uint16_t* sz_v, const float* S, void* dev_dst,
                                    size_t dev_bytes, void* stream, dc_delta_handle* out) {
  DC_NVTX("dc_pack_upload");
  dc_clear_error();
  DcLayout L;
  dc_status st = dc_check_desc(desc, &L);
  if (st) return st;
  if (!dev_dst || !out) return dc_fail(DC_ERR_INVALID_ARG, "null destination or handle");
  if (L.r > 0 && (!codes_u || !codes_v || !sz_u || !sz_v || !S)) return dc_fail(DC_ERR_INVALID_ARG, "null host buffer");
  if (((uintptr_t)dev_dst) % 256) return dc_fail(DC_ERR_ALIGN, "destination must be 256-byte aligned");
  if (dev_bytes < (size_t)L.bytes)
    return dc_fail(DC_ERR_WORKSPACE, "destination holds %zu bytes, need %lld", dev_bytes, (long long)L.bytes);
  std::vector<uint8_t> blob((size_t)L.bytes, 0);
  // bound on the U scales of the 2/3-bit bands (scales are positive fp16 values)
  double umax = 0.0;
  for (int b = 0; b < L.n_bands; ++b) {
    const DcBand& B = L.band[b];
    if (B.bits == 8) continue;
    for (int64_t i = (int64_t)B.r0 * L.groups_out; i < (int64_t)(B.r0 + B.rank) * L.groups_out; ++i)
      umax = std::max(umax, std::fabs(dc_f16_to_f64(sz_u[2 * i])));
  }
  DcPlain P{codes_u, codes_v, sz_u, sz_v, S, (float)umax};
  dc_pack_host(L, P, blob.data());
  cudaStream_t s = (cudaStream_t)stream;
  st = dc_cuda_check(cudaMemcpyAsync(dev_dst, blob.data(), blob.size(), cudaMemcpyHostToDevice, s), "upload");
  if (st) return st;
  st = dc_cuda_check(cudaStreamSynchronize(s), "upload sync");
  if (st) return st;
  dc_fill_handle(desc, L, dev_dst, out);
  return DC_OK;
}

extern "C" dc_status dc_tenant_table_upload(const dc_delta_handle* handles, int32_t n, void* dev_dst,
                                            size_t dev_bytes, void* stream) {
  DC_NVTX("dc_tenant_table_upload");
  dc_clear_error();
  if (n < 0 || (n > 0 && (!handles || !dev_dst))) return dc_fail(DC_ERR_INVALID_ARG, "bad tenant table arguments");
  if (((uintptr_t)dev_dst) % 16) return dc_fail(DC_ERR_ALIGN, "tenant table must be 16-byte aligned");
  const size_t need = (size_t)n * sizeof(dc_delta_handle);
  if (dev_bytes < need) return dc_fail(DC_ERR_WORKSPACE, "tenant table holds %zu bytes, need %zu", dev_bytes, need);
  for (int i = 0; i < n; ++i) {
    if (handles[i].dev_base == 0) continue;
    DcLayout L;
    dc_status st = dc_check_desc(&handles[i].desc, &L);
    if (st) return dc_fail(st, "tenant %d: %s", i, dc_last_error());
    if (handles[i].dev_base % 256) return dc_fail(DC_ERR_ALIGN, "tenant %d: blob not 256-byte aligned", i);
  }
  if (n == 0) return DC_OK;
  return dc_cuda_check(cudaMemcpyAsync(dev_dst, handles, need, cudaMemcpyHostToDevice, (cudaStream_t)stream),
                       "tenant table upload");
}

// ---------------------------------------------------------------------------------------------
// fp8 (E4M3) backbone weights: per-row scale max|w| / 448, codes rounded to nearest even with
// saturation (OCP 8-bit floating point specification, E4M3: bias 7, 3 mantissa bits, subnormals
// m * 2^-9, largest finite 448, no infinities).
// ---------------------------------------------------------------------------------------------
uint8_t dc_e4m3_rne(float x) {
  const uint8_t sign = std::signbit(x) ? 0x80 : 0x00;
  const double a = std::fabs((double)x);
  if (a != a) return 0x7F;
  if (a >= 448.0) return sign | 0x7E;
  if (a == 0.0) return sign;
  int e2 = 0;
  std::frexp(a, &e2);  // a = f 2^e2, f in [0.5, 1)
  const int E = e2 - 1;
  uint32_t code;
  if (E < -6) {  // subnormals: multiples of 2^-9 (8 * 2^-9 is the smallest normal, code 0x08)
    code = (uint32_t)std::nearbyint(a * 512.0);
  } else {
    double q = std::nearbyint((a / std::ldexp(1.0, E) - 1.0) * 8.0);  // exact scaling, ties to even
    int ee = E + 7;
    if (q == 8.0) {
      q = 0.0;
      ++ee;
    }
    code = ((uint32_t)ee << 3) | (uint32_t)q;
    if (code > 0x7E) code = 0x7E;
  }
  return sign | (uint8_t)code;
}

extern "C" dc_status dc_quantize_fp8_rows(const float* W, int32_t rows, int32_t cols, uint8_t* codes, float* scales) {
  DC_NVTX("dc_quantize_fp8_rows");
  dc_clear_error();
  if (!W || !codes || !scales) return dc_fail(DC_ERR_INVALID_ARG, "null pointer");
  if (rows <= 0 || cols <= 0) return dc_fail(DC_ERR_SHAPE, "rows and cols must be positive");
  for (int32_t r = 0; r < rows; ++r) {
    const float* w = W + (int64_t)r * cols;
    float amax = 0.f;
    for (int32_t c = 0; c < cols; ++c) {
      if (!std::isfinite(w[c])) return dc_fail(DC_ERR_INVALID_ARG, "row %d: non-finite weight", r);
      amax = std::max(amax, std::fabs(w[c]));
    }
    float s = amax / 448.0f;
    if (s == 0.f) s = 1.f;
    scales[r] = s;
    for (int32_t c = 0; c < cols; ++c) codes[(int64_t)r * cols + c] = dc_e4m3_rne(w[c] / s);
  }
  return DC_OK;
}
