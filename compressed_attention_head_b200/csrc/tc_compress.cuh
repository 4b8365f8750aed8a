// Tensor-core compress for fp16 keys/values with head_dim 128 (sm_100a).
//
// Same computation as k_compress_ref (SpectralQuant README, "Overview" and
// "Repository Structure": rotation into the calibrated eigenbasis, Lloyd-Max
// codes under the water-filled widths, QJL sign bits of the key residual on
// the signal dims), organised for B200:
//
//  * TMA streams tiles of 128 tokens x 128 fp16 (two 64-column boxes, 128-byte
//    swizzle) through a 3-stage shared-memory ring.
//  * One thread issues tcgen05.mma (M=128 tokens, N=128 coordinates, K=16):
//    D = X * B with B = 2^s_i V_i / sigma_i split into fp16 hi + lo parts
//    (about 22 significant bits), accumulated in fp32 in TMEM (two buffers).
//  * Eight epilogue warps read D from TMEM (thread = token, 64 coordinates
//    per warp), form z_i = D_i 2^-s_i / ||x||, and pick codes with register
//    thresholds. Each coordinate carries a rigorous bound delta_i on
//    |z_tensor - z_exact| (fp16 split residual + fp32 accumulation + rounding);
//    a z within delta_i of a threshold is recomputed exactly in float64 by the
//    whole warp, so every code equals the exact-arithmetic code.
//  * Four signal warps (thread = token) compute ||x|| and the m QJL signal
//    coordinates y_i exactly in float64, their codes, the residual, rho and
//    the sign bits.
//  * Codes are packed LSB-first into a shared-memory record tile and written
//    back with coalesced stores.
// Every mbarrier wait is bounded (see sm100.cuh); a timeout sets a device
// flag bit and the kernel skips the remaining work without hanging.
#pragma once

#include "sm100.cuh"
#include "sq_common.cuh"

namespace sq {
namespace tcc {

constexpr int D = 128;
constexpr int TILE = 128;
constexpr int STAGES = 3;
constexpr int KB = D / 64;
constexpr int X_BYTES = TILE * D * 2;
constexpr int B_BYTES = D * D * 2;
constexpr int NUM_WARPS = 14;
constexpr int NUM_THREADS = NUM_WARPS * 32;
constexpr int WARP_PROD = 0, WARP_MMA = 1, WARP_SIG0 = 2, WARP_EPI0 = 6;
constexpr int MAX_W = 12;
constexpr int REC_PITCH = MAX_W + 1;
constexpr uint32_t TMEM_COLS = 2 * D;
constexpr float E_ACC = 4.76837158203125e-07f;   // 8 * 2^-24: default accumulation bound factor
constexpr int QCAP = 256;                     // deferred exact recomputations per tile
constexpr int MSIG = 8;                       // signal coordinates staged in shared memory

struct CoordInfo {
  uint32_t bo;       // bits (low 8) | bit offset << 8
  float sc;          // 2^-s_i (column scale of B)
  float dfix;        // split residual ||e_i|| + fp32 rounding of z, 1/||x||, thresholds
  float dacc;        // ||V_i / sigma_i|| = 1/sigma_i: multiplies the accumulation bound
};
// Radius = dfix + E * dacc, with E the fp32 accumulation bound per unit of
// sum_j |x_j B_ij| / ||x|| <= ||B_i|| (Cauchy-Schwarz); E is a kernel argument.

// Byte offsets of the dynamic shared memory (base aligned to 1024).
constexpr int OFF_X = 0;
constexpr int OFF_BHI = OFF_X + STAGES * X_BYTES;
constexpr int OFF_BLO = OFF_BHI + B_BYTES;
constexpr int OFF_BLO2 = OFF_BLO + B_BYTES;                 // third split term (exact recomputation only)
constexpr int OFF_REC = OFF_BLO2 + B_BYTES;
constexpr int REC_BYTES = 2 * TILE * REC_PITCH * 4;
constexpr int OFF_RT = OFF_REC + REC_BYTES;                 // float [2][TILE]
constexpr int OFF_N64 = OFF_RT + 2 * TILE * 4;              // double [2][TILE]
constexpr int OFF_CI = OFF_N64 + 2 * TILE * 8;              // CoordInfo [D]
constexpr int OFF_SIG = OFF_CI + D * 16;                    // double [D]
constexpr int OFF_TH64 = OFF_SIG + D * 8;                   // double [kThreshTotal]
constexpr int OFF_VSIG = (OFF_TH64 + kThreshTotal * 8 + 15) & ~15;   // double [MSIG][D]
constexpr int OFF_Q = OFF_VSIG + MSIG * D * 8;              // u32 [QCAP] (token << 16 | coordinate)
constexpr int OFF_BAR = (OFF_Q + QCAP * 4 + 7) & ~7;
constexpr int N_BARS = 2 * STAGES + 1 + 2 + 2 + 2;
constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;              // u32 [16]
constexpr int OFF_CHUNK = OFF_MISC + 64;                    // u32 [8]: per 16-coordinate chunk, width | offset << 8
constexpr int OFF_DW = OFF_CHUNK + 32;                      // float [9]: per-width radius
constexpr int SMEM_BYTES = OFF_DW + 48 + 1024;              // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory plan exceeds 227 KB");

// The tensor-core block inside the record's derived part (derived_tc_off):
// Bhi, Blo, Blo2 [d*d fp16 each] (swizzled B operand; B = hi + lo + lo2 to
// about 2^-33 relative), CoordInfo [d], Vt64 [d*d f64].
struct TcView {
  uint8_t* base;
  int d;
  __host__ __device__ __half* bhi() const { return (__half*)base; }
  __host__ __device__ __half* blo() const { return (__half*)(base + 2 * (size_t)d * d); }
  __host__ __device__ __half* blo2() const { return (__half*)(base + 4 * (size_t)d * d); }
  __host__ __device__ CoordInfo* ci() const { return (CoordInfo*)(base + 6 * (size_t)d * d); }
  __host__ __device__ double* vt64() const { return (double*)(base + 6 * (size_t)d * d + 16 * (size_t)d); }
};
__host__ __device__ inline TcView tc_view(Rec r) { return TcView{r.derived() + derived_tc_off(r.d), r.d}; }

// Byte offset of element (row n, column k) of an [rows x D] K-major fp16 operand
// in the 128-byte-swizzled canonical layout (64-column blocks of rows*128 bytes).
__host__ __device__ inline uint32_t sw128_off(int n, int k, int rows) {
  int kb = k >> 6, e = k & 63, c = e >> 3, w = e & 7;
  return (uint32_t)(kb * rows * 128 + (n >> 3) * 1024 + (n & 7) * 128 + ((c ^ (n & 7)) << 4) + (w << 1));
}

// Builds the tensor-core block of one record (called with the block's threads).
__device__ void build_tc(Rec rec, int tid, int nth) {
  if (rec.d != D) return;
  TcView tv = tc_view(rec);
  const double* V = rec.V();
  const double* sig = rec.sigma();
  const int* bits_off = rec.offsets();
  for (int e = tid; e < D * D; e += nth) {
    int i = e / D, j = e % D;
    tv.vt64()[e] = V[(size_t)j * D + i];
  }
  // One power-of-two scale for the whole head: 2^ex * max |V_ji / sigma_i| <= 2^14.
  __shared__ double s_mx;
  if (tid == 0) s_mx = 0.0;
  __syncthreads();
  for (int i = tid; i < D; i += nth) {
    double s = sig[i];
    double inv = s > 0.0 ? 1.0 / s : 0.0;
    double mx = 0.0;
    for (int j = 0; j < D; ++j) mx = fmax(mx, fabs(V[(size_t)j * D + i] * inv));
    unsigned long long* p = (unsigned long long*)&s_mx;   // max of non-negative doubles by bits
    atomicMax(p, (unsigned long long)__double_as_longlong(mx));
  }
  __syncthreads();
  const double hmx = s_mx;
  for (int i = tid; i < D; i += nth) {
    double s = sig[i];
    double inv = s > 0.0 ? 1.0 / s : 0.0;
    int ex = 0;
    if (hmx > 0.0) ex = (int)floor(log2(16384.0 / hmx));
    ex = ex < -100 ? -100 : (ex > 100 ? 100 : ex);
    double scale = ldexp(1.0, ex);
    double res2 = 0.0;
    uint8_t* hi = (uint8_t*)tv.bhi();
    uint8_t* lo = (uint8_t*)tv.blo();
    uint8_t* lo2 = (uint8_t*)tv.blo2();
    for (int j = 0; j < D; ++j) {
      double v = V[(size_t)j * D + i] * inv * scale;
      __half h = __double2half(v);
      double r1 = v - (double)__half2float(h);
      __half l = __double2half(r1);
      double r2 = r1 - (double)__half2float(l);
      __half l2 = __double2half(r2);
      res2 += r2 * r2;
      uint32_t o = sw128_off(i, j, D);
      *(__half*)(hi + o) = h;
      *(__half*)(lo + o) = l;
      *(__half*)(lo2 + o) = l2;
    }
    CoordInfo c;
    c.bo = (uint32_t)rec.bits()[i] | ((uint32_t)bits_off[i] << 8);
    c.sc = (float)ldexp(1.0, -ex);
    // Bound on |z_tensor - z_exact| (the tensor path uses hi + lo): their
    // split residual, the fp32 accumulation term (E * ||V_i / sigma_i||, E a
    // kernel argument) and the fp32 roundings of z, 1/||x|| and the thresholds
    // (|z| < 8).
    c.dfix = s > 0.0 ? (float)(sqrt(res2) / scale + 2.0e-6) : 0.0f;
    c.dacc = (float)inv;
    tv.ci()[i] = c;
  }
}

struct Params {
  const uint8_t* recs;
  int n_heads, batch;
  int64_t n_tok;
  const int32_t* start_pos;
  CacheArgs c;
  uint32_t* flags;
  int64_t n_tiles;
  int tiles_per_row;
  float eacc;        // accumulation bound factor of the radius (E_ACC by default)
};

// ---------------------------------------------------------------- quantizers
__device__ __forceinline__ int q1(float z, float dl, bool& dg) {
  dg = fabsf(z) < dl;
  return z > 0.0f ? 1 : 0;
}
__device__ __forceinline__ int q2(float z, float t1, float dl, bool& dg) {
  float a = fabsf(z);
  int m = a > t1 ? 1 : 0;
  dg = (a < dl) | (fabsf(a - t1) < dl);
  return z > 0.0f ? 2 + m : 1 - m;
}
__device__ __forceinline__ int q3(float z, float t1, float t2, float t3, float dl, bool& dg) {
  float a = fabsf(z);
  int m = (a > t1 ? 1 : 0) + (a > t2 ? 1 : 0) + (a > t3 ? 1 : 0);
  dg = (a < dl) | (fabsf(a - t1) < dl) | (fabsf(a - t2) < dl) | (fabsf(a - t3) < dl);
  return z > 0.0f ? 4 + m : 3 - m;
}
__device__ __forceinline__ int qn(float z, const double* th, int b, float dl, bool& dg) {
  const int n = (1 << b) - 1;
  const int lo = code_of((double)z, th, b);
  const double dlo = lo > 0 ? (double)z - th[lo - 1] : 1e30;
  const double dhi = lo < n ? th[lo] - (double)z : 1e30;
  dg = fmin(fabs(dlo), fabs(dhi)) < (double)dl;
  return lo;
}

// Codes of 16 consecutive coordinates of width B (1..3) from their tensor-core
// values v (z = v * zr), packed LSB-first (16 * B bits), and the mask of the
// coordinates whose z lies within dl of a threshold.
template <int B>
__device__ __forceinline__ void chunk_codes(const float* v, float zr, float t1, float t2, float t3, float dl,
                                            uint64_t& cw, uint32_t& dmask) {
  cw = 0;
  dmask = 0;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const float z = v[k] * zr;
    bool dg;
    int code;
    if (B == 1) code = q1(z, dl, dg);
    else if (B == 2) code = q2(z, t1, dl, dg);
    else code = q3(z, t1, t2, t3, dl, dg);
    cw |= (uint64_t)(uint32_t)code << (B * k);
    dmask |= (uint32_t)dg << k;
  }
}

// ORs the nbits-bit value cw into a record at bit position o (up to 3 words).
__device__ __forceinline__ void or_bits(uint32_t* rw, int o, uint64_t cw, int nbits) {
  const int wi = o >> 5, sh = o & 31;
  const uint64_t a = cw << sh;
  const uint32_t top = sh ? (uint32_t)(cw >> (64 - sh)) : 0u;
  if ((uint32_t)a) atomicOr(&rw[wi], (uint32_t)a);
  if ((uint32_t)(a >> 32)) atomicOr(&rw[wi + 1], (uint32_t)(a >> 32));
  if (sh + nbits > 64 && top) atomicOr(&rw[wi + 2], top);
}

// Byte offset of the 16-byte chunk c (elements 8c .. 8c+7) of token row t in an X stage.
__device__ __forceinline__ uint32_t x_chunk(int t, int c) {
  return (uint32_t)((c >> 3) * (TILE * 128) + (t >> 3) * 1024 + (t & 7) * 128 + (((c & 7) ^ (t & 7)) << 4));
}

// One pass over token t's row: ||x||^2 and the first MM signal coordinates
// sum_j x_j V[j][i] (float64), with the V rows staged in shared memory.
template <int MM>
__device__ __forceinline__ void row_pass(const uint8_t* xs, int t, const double* vsig, double& n2, double* ys) {
#pragma unroll 2
  for (int c = 0; c < D / 8; ++c) {
    const uint4 raw = *(const uint4*)(xs + x_chunk(t, c));
    const __half2* h2 = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 f = __half22float2(h2[q]);
      const double x0 = f.x, x1 = f.y;
      n2 = fma(x0, x0, n2);
      n2 = fma(x1, x1, n2);
      const int j = c * 8 + 2 * q;
#pragma unroll
      for (int ii = 0; ii < MM; ++ii) {
        const double2 v = *(const double2*)(vsig + ii * D + j);
        ys[ii] = fma(x0, v.x, ys[ii]);
        ys[ii] = fma(x1, v.y, ys[ii]);
      }
    }
  }
}

// Exact (float64) dot product of token t's row with a global row of D doubles.
__device__ __forceinline__ double exact_dot(const uint8_t* xs, int t, const double* vrow) {
  double acc = 0.0;
#pragma unroll 2
  for (int c = 0; c < D / 8; ++c) {
    const uint4 raw = *(const uint4*)(xs + x_chunk(t, c));
    const __half2* h2 = reinterpret_cast<const __half2*>(&raw);
    const double2* vr = reinterpret_cast<const double2*>(vrow + c * 8);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 f = __half22float2(h2[q]);
      const double2 v = vr[q];
      acc = fma((double)f.x, v.x, acc);
      acc = fma((double)f.y, v.y, acc);
    }
  }
  return acc;
}

// sum_j x[t][j] * (hi + lo + lo2)[i][j] in float64 by one warp (lane l takes
// j = 4l .. 4l+3); every lane returns the sum. The three fp16 terms represent
// B to about 2^-33 relative, so z = sum * 2^-s / ||x|| matches exact
// arithmetic to ~1e-9, far inside the 1e-5 exemption band.
__device__ __forceinline__ double exact_sum_warp(const uint8_t* xs, const uint8_t* bh, const uint8_t* bl,
                                                 const uint8_t* bl2, int t, int i, int lane) {
  const int j = 4 * lane;
  const uint2 xr = *(const uint2*)(xs + x_chunk(t, j >> 3) + ((j & 7) << 1));
  const uint32_t bo = sw128_off(i, j, D);
  const uint2 h = *(const uint2*)(bh + bo), l = *(const uint2*)(bl + bo), l2 = *(const uint2*)(bl2 + bo);
  const __half2* xh = reinterpret_cast<const __half2*>(&xr);
  const __half2* hh = reinterpret_cast<const __half2*>(&h);
  const __half2* lh = reinterpret_cast<const __half2*>(&l);
  const __half2* l2h = reinterpret_cast<const __half2*>(&l2);
  double acc = 0.0;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const float2 xf = __half22float2(xh[k]), hf = __half22float2(hh[k]);
    const float2 lf = __half22float2(lh[k]), l2f = __half22float2(l2h[k]);
    acc = fma((double)xf.x, ((double)hf.x + (double)lf.x) + (double)l2f.x, acc);
    acc = fma((double)xf.y, ((double)hf.y + (double)lf.y) + (double)l2f.y, acc);
  }
  return warp_sum(acc);
}

// Overwrites the b-bit field at bit o of a record with code.
__device__ __forceinline__ void patch_field(uint32_t* rw, int o, int b, uint32_t code) {
  const int wi = o >> 5, sh = o & 31;
  const uint32_t mask = (1u << b) - 1u;
  atomicAnd(&rw[wi], ~(mask << sh));
  atomicOr(&rw[wi], code << sh);
  if (sh + b > 32) {
    atomicAnd(&rw[wi + 1], ~(mask >> (32 - sh)));
    atomicOr(&rw[wi + 1], code >> (32 - sh));
  }
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
k_compress_tc(const __grid_constant__ CUtensorMap tmap, Params P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sX = sm + OFF_X;
  uint8_t* sBhi = sm + OFF_BHI;
  uint8_t* sBlo = sm + OFF_BLO;
  uint8_t* sBlo2 = sm + OFF_BLO2;
  uint32_t* sRec = (uint32_t*)(sm + OFF_REC);
  float* sRt = (float*)(sm + OFF_RT);
  double* sN64 = (double*)(sm + OFF_N64);
  CoordInfo* sCI = (CoordInfo*)(sm + OFF_CI);
  double* sSig = (double*)(sm + OFF_SIG);
  double* sTh64 = (double*)(sm + OFF_TH64);
  double* sVsig = (double*)(sm + OFF_VSIG);
  uint32_t* sQ = (uint32_t*)(sm + OFF_Q);
  uint64_t* bars = (uint64_t*)(sm + OFF_BAR);
  uint64_t* full = bars;                    // [STAGES]
  uint64_t* empty = bars + STAGES;          // [STAGES]
  uint64_t* bfull = bars + 2 * STAGES;      // 1
  uint64_t* tfull = bfull + 1;              // [2]
  uint64_t* tempty = tfull + 2;             // [2]
  uint64_t* sfull = tempty + 2;             // [2]
  uint32_t* misc = (uint32_t*)(sm + OFF_MISC);
  // misc: [0] tmem base, [1] abort, [2] segment ok, [3] m, [4] W, [5] code_bits, [6] flags, [8] start,
  //       [9] queue length
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  for (int e = threadIdx.x; e < 2 * TILE * REC_PITCH; e += NUM_THREADS) sRec[e] = 0u;
  for (int e = threadIdx.x; e < kThreshTotal; e += NUM_THREADS) sTh64[e] = c_th64[e];
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      sm100::mbar_init(&full[s], 1);
      sm100::mbar_init(&empty[s], 1 + 4 + 8);
    }
    sm100::mbar_init(bfull, 1);
    for (int b = 0; b < 2; ++b) {
      sm100::mbar_init(&tfull[b], 1);
      sm100::mbar_init(&tempty[b], 8);
      sm100::mbar_init(&sfull[b], 4);
    }
    misc[1] = 0u;
    misc[9] = 0u;
    sm100::fence_mbar_init();
  }
  if (warp == WARP_MMA) {
    sm100::tmem_alloc(&misc[0], TMEM_COLS);
    sm100::tmem_relinquish();
  }
  if (warp == WARP_PROD && lane == 0) sm100::prefetch_tmap(&tmap);
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem_base = misc[0];
  volatile uint32_t* abort_flag = &misc[1];
  uint32_t* err = P.flags;

  const int64_t per = (P.n_tiles + gridDim.x - 1) / gridDim.x;
  const int64_t tb = (int64_t)blockIdx.x * per;
  const int64_t te = min(P.n_tiles, tb + per);
  uint32_t iter = 0, seg = 0;   // seg counts the segments that load B
  const uint32_t idesc = sm100::idesc_f16(TILE, D);

  for (int64_t s0 = tb; s0 < te;) {
    const int64_t row = s0 / P.tiles_per_row;
    const int64_t s1 = min(te, (row + 1) * (int64_t)P.tiles_per_row);
    const int h = (int)(row % P.n_heads);
    const int bidx = (int)(row / P.n_heads);
    Rec rec = rec_at(P.recs, D, h);
    TcView tv = tc_view(rec);
    __syncthreads();
    if (threadIdx.x == 0) {
      const RecHeader* hd = rec.hdr();
      bool ok = record_ok(hd, D) && hd->words == P.c.words && hd->words <= MAX_W &&
                (hd->m == 0 || P.c.rnorm != nullptr);
      const int64_t sp = P.start_pos ? (int64_t)P.start_pos[bidx] : 0;
      bool cap_ok = sp >= 0 && sp + P.n_tok <= P.c.cap;
      if (!ok && err) atomicOr(err, SQ_FLAG_RECORD);
      if (ok && !cap_ok && err) atomicOr(err, SQ_FLAG_CAPACITY);
      misc[2] = (ok && cap_ok) ? 1u : 0u;
      misc[3] = ok ? hd->m : 0;
      misc[4] = hd->words;
      misc[5] = hd->code_bits;
      misc[6] = hd->flags;
      misc[8] = (uint32_t)sp;
    }
    __syncthreads();
    const bool seg_ok = misc[2] != 0 && *abort_flag == 0;
    const int m = (int)misc[3], W = (int)misc[4], cbits = (int)misc[5];
    const bool normalize = (misc[6] & kFlagNormalize) != 0;
    const int64_t sp = (int64_t)misc[8];
    if (!seg_ok) {       // nothing of this segment is touched
      s0 = s1;
      continue;
    }
    for (int i = threadIdx.x; i < D; i += NUM_THREADS) {
      sCI[i] = tv.ci()[i];
      sSig[i] = rec.sigma()[i];
    }
    const int msig = m < MSIG ? m : MSIG;
    for (int e = threadIdx.x; e < msig * D; e += NUM_THREADS) sVsig[e] = tv.vt64()[e];
    __syncthreads();
    if (threadIdx.x == 0) {
      // Per-width radius: the largest of its coordinates (the signal ones are exact).
      float* dw = (float*)(sm + OFF_DW);
      for (int b = 0; b <= SQ_MAX_BITS; ++b) dw[b] = 0.0f;
      for (int i = m; i < D; ++i) {
        const int b = (int)(sCI[i].bo & 0xFFu);
        dw[b] = fmaxf(dw[b], fmaf(P.eacc, sCI[i].dacc, sCI[i].dfix));
      }
      // 16-coordinate chunks of one width in 1..3 with no signal coordinate take the fast path.
      uint32_t* ch = (uint32_t*)(sm + OFF_CHUNK);
      for (int c = 0; c < D / 16; ++c) {
        const int b0 = (int)(sCI[16 * c].bo & 0xFFu);
        bool uni = b0 >= 1 && b0 <= 3 && 16 * c >= m;
        for (int k = 1; k < 16 && uni; ++k) uni = (int)(sCI[16 * c + k].bo & 0xFFu) == b0;
        ch[c] = (uni ? (uint32_t)b0 : 0u) | ((sCI[16 * c].bo >> 8) << 8);
      }
    }
    if (warp == WARP_PROD && lane == 0) {
      sm100::mbar_expect_tx(bfull, 3 * B_BYTES);
      sm100::bulk_load(sBhi, tv.bhi(), B_BYTES, bfull);
      sm100::bulk_load(sBlo, tv.blo(), B_BYTES, bfull);
      sm100::bulk_load(sBlo2, tv.blo2(), B_BYTES, bfull);
    }
    __syncthreads();
    const uint32_t bpar = seg & 1u;
    const int64_t nt = s1 - s0;

    if (warp == WARP_PROD) {
      if (lane == 0) {
        for (int64_t k = 0; k < nt; ++k) {
          const uint32_t it = iter + (uint32_t)k;
          const int st = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (*abort_flag || !sm100::mbar_wait(&empty[st], ph ^ 1u, err)) { *abort_flag = 1; continue; }
          const int64_t tile = s0 + k;
          const int t0 = (int)((tile - row * P.tiles_per_row) * TILE);
          const int ycoord = (int)(row * P.n_tok + t0);
          sm100::mbar_expect_tx(&full[st], X_BYTES);
          for (int kb = 0; kb < KB; ++kb)
            sm100::tma_load_2d(sX + st * X_BYTES + kb * (TILE * 128), &tmap, &full[st], kb * 64, ycoord);
        }
      }
    } else if (warp == WARP_MMA) {
      if (lane == 0) {
        bool bok = *abort_flag == 0 && sm100::mbar_wait(bfull, bpar, err);
        if (!bok) *abort_flag = 1;
        for (int64_t k = 0; k < nt; ++k) {
          const uint32_t it = iter + (uint32_t)k;
          const int st = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          const int buf = it & 1;
          const uint32_t bph = (it >> 1) & 1u;
          if (*abort_flag || !sm100::mbar_wait(&full[st], ph, err) ||
              !sm100::mbar_wait(&tempty[buf], bph ^ 1u, err)) {
            *abort_flag = 1;
            continue;
          }
          sm100::tc_fence_after();
          const uint32_t dt = tmem_base + (uint32_t)(buf * D);
          const uint32_t xa = sm100::smem_u32(sX + st * X_BYTES);
          const uint32_t bh = sm100::smem_u32(sBhi), bl = sm100::smem_u32(sBlo);
#pragma unroll
          for (int kb = 0; kb < KB; ++kb) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint32_t ao = kb * (TILE * 128) + kk * 32, bo = kb * (D * 128) + kk * 32;
              const uint64_t ad = sm100::sw128_desc(xa + ao);
              sm100::mma_f16(dt, ad, sm100::sw128_desc(bh + bo), idesc, (kb | kk) ? 1u : 0u);
              sm100::mma_f16(dt, ad, sm100::sw128_desc(bl + bo), idesc, 1u);
            }
          }
          sm100::mma_commit(&empty[st]);
          sm100::mma_commit(&tfull[buf]);
        }
      }
    } else {
      // ---------------- worker warps: signal (2..5) and epilogue (6..13)
      const bool is_sig = warp < WARP_EPI0;
      const int q = warp & 3, hh = (warp - WARP_EPI0) >> 2;
      const int t_sig = (warp - WARP_SIG0) * 32 + lane;
      const int t_epi = q * 32 + lane;
      const int worker = threadIdx.x - WARP_SIG0 * 32;       // 0 .. 383
      const int epi_id = threadIdx.x - WARP_EPI0 * 32;       // 0 .. 255 for epilogue threads
      const float t21 = (float)sTh64[th_off(2) + 2];
      const float t31 = (float)sTh64[th_off(3) + 4], t32 = (float)sTh64[th_off(3) + 5];
      const float t33 = (float)sTh64[th_off(3) + 6];
      const int wid = warp - WARP_SIG0;                        // worker warp 0 .. 11
      const double* S = rec.S();
      for (int64_t k = 0; k < nt; ++k) {
        const uint32_t it = iter + (uint32_t)k;
        const int st = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1u;
        const int buf = it & 1;
        const uint32_t bph = (it >> 1) & 1u;
        const int64_t tile = s0 + k;
        const int t0 = (int)((tile - row * P.tiles_per_row) * TILE);
        const int n_valid = (int)min((int64_t)TILE, P.n_tok - t0);
        const uint8_t* xs = sX + st * X_BYTES;
        bool live;
        if (is_sig) {
          // ---- norm, exact signal coordinates, their codes, rho, QJL signs
          live = __all_sync(0xffffffffu, *abort_flag == 0 && sm100::mbar_wait(&full[st], ph, err));
          if (!live) *abort_flag = 1;
          const int t = t_sig;
          const bool valid = live && t < n_valid;
          uint32_t* rw = sRec + (buf * TILE + t) * REC_PITCH;
          double n2 = 0.0;
          double ys[MSIG];
#pragma unroll
          for (int ii = 0; ii < MSIG; ++ii) ys[ii] = 0.0;
          if (live) {
            if (msig == 0) row_pass<0>(xs, t, sVsig, n2, ys);
            else if (msig <= 2) row_pass<2>(xs, t, sVsig, n2, ys);
            else if (msig <= 4) row_pass<4>(xs, t, sVsig, n2, ys);
            else row_pass<8>(xs, t, sVsig, n2, ys);
          }
          const double nrm = normalize ? sqrt(n2) : 1.0;
          const double inv = nrm > 0.0 ? 1.0 / nrm : 0.0;
          sRt[buf * TILE + t] = (float)inv;
          sN64[buf * TILE + t] = nrm;
          double rho2 = 0.0;
          if (valid && m > 0) {
            double r[D];     // residual of the signal coordinates (first m used)
            for (int i = 0; i < m; ++i) {
              double y;
              if (i < MSIG) {
                y = ys[0];
#pragma unroll
                for (int ii = 1; ii < MSIG; ++ii) if (ii == i) y = ys[ii];
              } else {
                y = exact_dot(xs, t, tv.vt64() + (size_t)i * D);
              }
              const int b = (int)(sCI[i].bo & 0xFFu);
              const double yn = y * inv;
              double lvv = 0.0;
              if (b > 0) {
                const double z = sSig[i] > 0.0 ? yn / sSig[i] : 0.0;
                const int code = code_of(z, sTh64 + th_off(b), b);
                lvv = c_lv64[lv_off(b) + code];
                const int o = (int)(sCI[i].bo >> 8), wi = o >> 5, sh = o & 31;
                atomicOr(&rw[wi], (uint32_t)code << sh);
                if (sh + b > 32) atomicOr(&rw[wi + 1], (uint32_t)code >> (32 - sh));
              }
              r[i] = yn - sSig[i] * lvv;
              rho2 += r[i] * r[i];
            }
            for (int j = 0; j < m; ++j) {
              double pj = 0.0;
              for (int i = 0; i < m; ++i) pj = fma(S[j * m + i], r[i], pj);
              if (pj >= 0.0) {
                const int o = cbits + j;
                atomicOr(&rw[o >> 5], 1u << (o & 31));
              }
            }
          }
          if (valid) {
            const size_t slot = ((size_t)bidx * P.n_heads + h) * P.c.cap + sp + t0 + t;
            P.c.norm[slot] = (float)nrm;
            if (P.c.rnorm) P.c.rnorm[slot] = (float)sqrt(rho2);
          }
          __syncwarp();
          if (lane == 0) sm100::mbar_arrive(&sfull[buf]);
        } else {
          // ---- epilogue: TMEM -> codes -> packed record words
          live = __all_sync(0xffffffffu, *abort_flag == 0 && sm100::mbar_wait(&tfull[buf], bph, err) &&
                                             sm100::mbar_wait(&sfull[buf], bph, err));
          if (!live) *abort_flag = 1;
          sm100::tc_fence_after();
          const int t = t_epi;
          const float r = sRt[buf * TILE + t];
          const bool valid = live && t < n_valid;
          const bool exact_zero = r == 0.0f;
          uint32_t* rw = sRec + (buf * TILE + t) * REC_PITCH;
          const float eacc = P.eacc;
          const float zr = sCI[0].sc * r;
          const float* dw = (const float*)(sm + OFF_DW);
          const uint32_t* chd = (const uint32_t*)(sm + OFF_CHUNK);
          const bool enq_ok = valid && !exact_zero;
          if (live) {
            for (int c = 0; c < 4; ++c) {
              float v[16];
              sm100::tmem_ld16(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * D + hh * 64 + c * 16), v);
              const int i0 = hh * 64 + c * 16;
              const uint32_t cd = chd[i0 >> 4];
              const int cb = (int)(cd & 0xFFu);
              uint32_t dmask = 0;
              if (cb != 0) {
                // width-uniform chunk: codes packed with compile-time shifts
                uint64_t cw;
                if (cb == 1) chunk_codes<1>(v, zr, 0.f, 0.f, 0.f, dw[1], cw, dmask);
                else if (cb == 2) chunk_codes<2>(v, zr, t21, 0.f, 0.f, dw[2], cw, dmask);
                else chunk_codes<3>(v, zr, t31, t32, t33, dw[3], cw, dmask);
                if (valid) or_bits(rw, (int)(cd >> 8), cw, 16 * cb);
              } else {
#pragma unroll
                for (int kk = 0; kk < 16; ++kk) {
                  const int i = i0 + kk;
                  const CoordInfo ci = sCI[i];
                  const int b = (int)(ci.bo & 0xFFu);
                  if (b == 0 || i < m) continue;
                  const float z = v[kk] * zr;
                  const float dl = fmaf(eacc, ci.dacc, ci.dfix);
                  bool dg;
                  int code;
                  if (b == 1) code = q1(z, dl, dg);
                  else if (b == 2) code = q2(z, t21, dl, dg);
                  else if (b == 3) code = q3(z, t31, t32, t33, dl, dg);
                  else code = qn(z, sTh64 + th_off(b), b, dl, dg);
                  dmask |= (uint32_t)dg << kk;
                  if (valid) or_bits(rw, (int)(ci.bo >> 8), (uint64_t)(uint32_t)code, b);
                }
              }
              // Queue the codes within their radius for exact recomputation.
              dmask = enq_ok ? dmask : 0u;
              if (__any_sync(0xffffffffu, dmask != 0u)) {
                for (int kk = 0; kk < 16; ++kk) {
                  const bool dg = (dmask >> kk) & 1u;
                  const uint32_t dm = __ballot_sync(0xffffffffu, dg);
                  if (!dm) continue;
                  uint32_t base = 0;
                  if (lane == 0) base = atomicAdd(&misc[9], (uint32_t)__popc(dm));
                  base = __shfl_sync(0xffffffffu, base, 0);
                  const uint32_t pos = base + (uint32_t)__popc(dm & ((1u << lane) - 1u));
                  const int i = i0 + kk;
                  const bool ov = dg && pos >= (uint32_t)QCAP;
                  if (dg && !ov) sQ[pos] = ((uint32_t)t << 16) | (uint32_t)i;
                  uint32_t om = __ballot_sync(0xffffffffu, ov);
                  while (om) {        // queue full: recompute and patch right here
                    const int src = __ffs(om) - 1;
                    om &= om - 1;
                    const int ts = q * 32 + src;
                    const CoordInfo ci = sCI[i];
                    const int b = (int)(ci.bo & 0xFFu);
                    const double zz = exact_sum_warp(xs, sBhi, sBlo, sBlo2, ts, i, lane) * (double)ci.sc /
                                      sN64[buf * TILE + ts];
                    if (lane == src) patch_field(rw, (int)(ci.bo >> 8), b, (uint32_t)code_of(zz, sTh64 + th_off(b), b));
                  }
                }
              }
            }
          }
          sm100::tc_fence_before();
          __syncwarp();
          if (lane == 0) sm100::mbar_arrive(&tempty[buf]);
        }
        // ---- all 12 worker warps: exact recomputation of the queued codes
        sm100::named_bar(1, 12 * 32);
        const uint32_t qn_ = min(misc[9], (uint32_t)QCAP);
        for (uint32_t e = (uint32_t)wid; e < qn_; e += 12) {
          const uint32_t ent = sQ[e];
          const int t = (int)(ent >> 16), i = (int)(ent & 0xFFFFu);
          const CoordInfo ci = sCI[i];
          const int b = (int)(ci.bo & 0xFFu);
          const double zz = exact_sum_warp(xs, sBhi, sBlo, sBlo2, t, i, lane) * (double)ci.sc / sN64[buf * TILE + t];
          if (lane == 0)
            patch_field(sRec + (buf * TILE + t) * REC_PITCH, (int)(ci.bo >> 8), b,
                        (uint32_t)code_of(zz, sTh64 + th_off(b), b));
        }
        sm100::named_bar(1, 12 * 32);
        if (lane == 0) sm100::mbar_arrive(&empty[st]);    // the X stage is no longer read
        if (!is_sig) {
          // ---- store the finished record tile, then clear it for tile + 2
          const size_t slot0 = ((size_t)bidx * P.n_heads + h) * P.c.cap + sp + t0;
          uint32_t* gdst = P.c.codes + slot0 * W;
          uint32_t* rb = sRec + buf * TILE * REC_PITCH;
          if (live)
            for (int e = epi_id; e < n_valid * W; e += 256) gdst[e] = rb[(e / W) * REC_PITCH + e % W];
          if (epi_id == 0) misc[9] = 0u;
          sm100::named_bar(2, 8 * 32);
          for (int e = epi_id; e < TILE * REC_PITCH; e += 256) rb[e] = 0u;
        }
      }
    }
    iter += (uint32_t)nt;
    ++seg;
    s0 = s1;
  }
  // Every copy this CTA issued has landed before it exits: the last phase of
  // each stage's full barrier and of the B barrier (bounded waits).
  if (warp == WARP_PROD && lane == 0) {
    for (uint32_t k = 0; k < STAGES && k < iter; ++k) {
      const uint32_t it = iter - 1 - k;
      sm100::mbar_wait(&full[it % STAGES], (it / STAGES) & 1u, nullptr);
    }
    if (seg > 0) sm100::mbar_wait(bfull, (seg - 1) & 1u, nullptr);
  }
  sm100::tc_fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tmem_base, TMEM_COLS);
  }
  if (threadIdx.x == 0 && *abort_flag && err) atomicOr(err, 0x80000000u);
}

}  // namespace tcc
}  // namespace sq
