// Shared definitions of libsq's kernels: the calibration-record view, the
// per-device Lloyd-Max tables, and small device helpers.
//
// The record layout is the one documented in include/sq.h. The Lloyd-Max
// tables are computed on the host by codebook.cpp (the library's own
// implementation) and uploaded into constant memory once per device.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sq.h"

namespace sq {

constexpr uint32_t kMagic = 0x31435153u;
constexpr uint32_t kVersion = 2u;
constexpr int kHeader = 128;
constexpr int kMaxD = 256;
constexpr uint32_t kFlagKey = 1u, kFlagQjl = 2u, kFlagNormalize = 4u, kFlagRandomRotation = 8u, kFlagCumvar = 16u,
                   kFlagFitted = 32u;
constexpr int kMaxWords = 64;   // B <= 8 bits x 256 coordinates

// Packed-cache layout: the records of 32 consecutive tokens of one (batch,
// head) row are stored word-interleaved. Word w of token t of row r is
//   codes[r * cap * W + ((t / 32) * W + w) * 32 + t % 32]
// (cap a multiple of 32), so a block of 32 tokens is W * 128 contiguous bytes
// whose 128-byte piece w holds word w of the 32 records: one bulk copy of a
// block lands it transposed (word-major, token-minor) in shared memory, and 32
// lanes that write word w of 32 consecutive tokens write one 128-byte line.
constexpr int kBlockTok = 32;
__host__ __device__ inline size_t rec_word0(size_t row, int64_t cap, int W, int64_t t) {
  return row * (size_t)cap * (size_t)W + (size_t)(t >> 5) * (size_t)W * 32u + (size_t)(t & 31);
}

// Device arrays of one packed cache, as the kernels take them.
struct CacheArgs {
  uint32_t* codes;
  float* norm;
  float* rnorm;
  int64_t cap;
  int words;
};

// Offsets of the Lloyd-Max tables of width b inside the packed tables:
// levels of width b start at 2^b - 2 (2 + 4 + ... + 2^(b-1)), thresholds at
// 2^b - 1 - b (1 + 3 + ... + (2^(b-1) - 1)).
__host__ __device__ constexpr int lv_off(int b) { return (1 << b) - 2; }
__host__ __device__ constexpr int th_off(int b) { return (1 << b) - 1 - b; }
constexpr int kLevelsTotal = lv_off(SQ_MAX_BITS + 1);      // 510
constexpr int kThreshTotal = th_off(SQ_MAX_BITS + 1);      // 502

// Host-side record geometry (must match sq.h). The canonical part ends with
// the fitted-codebook section: levels [2][kLevelsTotal] and thresholds
// [2][kThreshTotal] in float64 (regime 0: coordinates below d_eff, 1: the rest).
constexpr size_t kFitBytes = 8u * 2u * ((size_t)kLevelsTotal + (size_t)kThreshTotal);
__host__ __device__ inline size_t fit_off(int d) {
  return (size_t)kHeader + 21u * (size_t)d + 16u * (size_t)d * (size_t)d;
}
__host__ __device__ inline size_t canon_bytes(int d) { return fit_off(d) + kFitBytes; }
__host__ __device__ inline size_t derived_off(int d) { return (canon_bytes(d) + 255u) & ~(size_t)255u; }
// Derived part: float32 copies used by the kernels,
//   sigma_f[d], inv_sigma_f[d], pad to 256 B, V_f[d*d] (same layout as V), S_f[d*d],
// and, for head_dim 128, the tensor-core block of the fast compress kernel
// (from the next 1024-byte boundary; see tc_compress.cuh).
__host__ __device__ inline size_t derived_tc_off(int d) {
  return ((size_t)(256 + 8 * d) + 8 * (size_t)d * d + 1023) & ~(size_t)1023;
}
__host__ __device__ inline size_t derived_tc_bytes(int d) {
  return d == 128 ? 6 * (size_t)d * d + 16 * (size_t)d + 256 + 8 * (size_t)d * d : 0;
}
__host__ __device__ inline size_t derived_bytes(int d) { return derived_tc_off(d) + derived_tc_bytes(d); }
__host__ __device__ inline size_t record_bytes(int d) {
  return (derived_off(d) + derived_bytes(d) + 255u) & ~(size_t)255u;
}

struct RecHeader {
  uint32_t magic, version;
  int32_t d, d_eff, m, total_bits, code_bits, words;
  uint32_t flags;
  int32_t sweeps, stream, max_bits;
  uint64_t seed;
  double trace, kappa, avg_bits;
  uint32_t derived_valid;
  uint32_t reserved[11];
};
static_assert(sizeof(RecHeader) == kHeader, "record header is 128 bytes");

// Typed view of one record.
struct Rec {
  uint8_t* base;
  int d;
  __host__ __device__ Rec(void* p, int d_) : base((uint8_t*)p), d(d_) {}
  __host__ __device__ RecHeader* hdr() const { return (RecHeader*)base; }
  __host__ __device__ double* lam() const { return (double*)(base + kHeader); }
  __host__ __device__ double* sigma() const { return (double*)(base + kHeader + 8 * d); }
  __host__ __device__ double* V() const { return (double*)(base + kHeader + 16 * d); }
  __host__ __device__ double* S() const { return (double*)(base + kHeader + 16 * d + 8 * d * d); }
  __host__ __device__ uint8_t* bits() const { return base + kHeader + 16 * d + 16 * d * d; }
  __host__ __device__ int32_t* offsets() const { return (int32_t*)(base + kHeader + 17 * d + 16 * d * d); }
  __host__ __device__ double* fit_lv() const { return (double*)(base + fit_off(d)); }
  __host__ __device__ double* fit_th() const { return (double*)(base + fit_off(d)) + 2 * kLevelsTotal; }
  __host__ __device__ uint8_t* derived() const { return base + derived_off(d); }
  __host__ __device__ float* sigma_f() const { return (float*)derived(); }
  __host__ __device__ float* inv_sigma_f() const { return (float*)derived() + d; }
  __host__ __device__ float* V_f() const { return (float*)(derived() + ((8 * d + 255) & ~255)); }
  __host__ __device__ float* S_f() const { return V_f() + d * d; }
};

__host__ __device__ inline Rec rec_at(const void* base, int d, int h) {
  return Rec((uint8_t*)base + (size_t)h * record_bytes(d), d);
}

// The per-device Lloyd-Max tables c_lv64, c_th64, c_lv32 and c_D (levels and
// thresholds ascending per width, distortion per width) are defined in api.cu,
// the one translation unit, before the kernel headers.

// Code of z under the b-bit thresholds th[0 .. 2^b - 2]: the number of
// thresholds strictly below z (binary search; a tie takes the lower code).
__device__ __forceinline__ int code_of(double z, const double* th, int b) {
  int lo = 0, n = (1 << b) - 1;   // answer in [0, n]
  int hi = n;
  while (lo < hi) {
    int mid = (lo + hi) >> 1;     // is z > th[mid]?
    if (z > th[mid]) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// Width-b field at bit position o of a little-endian word stream.
__device__ __forceinline__ uint32_t field(const uint32_t* w, int o, int b) {
  int wi = o >> 5, sh = o & 31;
  uint32_t v = w[wi] >> sh;
  if (sh + b > 32) v |= w[wi + 1] << (32 - sh);
  return v & ((1u << b) - 1u);
}

template <typename T> __device__ __forceinline__ float to_float(T v);
template <> __device__ __forceinline__ float to_float<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_float<__half>(__half v) { return __half2float(v); }
template <> __device__ __forceinline__ float to_float<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_float(float v);
template <> __device__ __forceinline__ float from_float<float>(float v) { return v; }
template <> __device__ __forceinline__ __half from_float<__half>(float v) { return __float2half_rn(v); }
template <> __device__ __forceinline__ __nv_bfloat16 from_float<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Header checks shared by the consumers of records: the record must be a
// version-1 record of this head_dim whose derived part has been built.
__device__ __forceinline__ bool record_ok(const RecHeader* h, int d) {
  return h->magic == kMagic && h->version == kVersion && h->d == d && h->derived_valid != 0 &&
         h->words >= 1 && h->words * 32 >= h->total_bits && h->m >= 0 && h->m <= d;
}

constexpr double kQjlScale = 1.2533141373155002512;   // sqrt(pi / 2)

}  // namespace sq
