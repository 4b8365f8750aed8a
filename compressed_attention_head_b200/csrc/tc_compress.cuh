// Tensor-core compress for fp16 keys/values with head_dim 128 (sm_100a).
//
// Same computation as k_compress_ref (SpectralQuant README, "Overview" and
// "Repository Structure": rotation into the calibrated eigenbasis, Lloyd-Max
// codes under the water-filled widths, QJL sign bits of the key residual on
// the signal dims), organised for B200:
//
//  * TMA streams tiles of 128 tokens x 128 fp16 (two 64-column boxes, 128-byte
//    swizzle) into four shared-memory stages.
//  * One thread issues tcgen05.mma (M = 128 tokens, N = 128 coordinates,
//    K = 16): D = X * B with B = 2^s V / sigma split into fp16 hi + lo parts
//    (about 22 significant bits), accumulated in fp32 in one of four TMEM
//    accumulators.
//  * Four epilogue groups of four warps each own one stage and one
//    accumulator (tile k goes to group k mod 4), so no group ever waits for
//    another. A thread owns one token row: it computes ||x|| (float32, or
//    float64 with the exact signal coordinates, rho and the QJL signs for
//    keys) straight from the staged tile, releases the stage, then reads its
//    row of D from TMEM 16 columns at a time, forms z_i = D_i 2^-s / ||x||,
//    picks each code (compare chains for widths 1-3, a cell table for 4-8)
//    and appends it to a register bit stream that goes to global memory one
//    32-bit word at a time.
//  * Every z carries a bound on |z_tensor - z_exact| (fp16 split residual,
//    fp32 accumulation, fp32 roundings). A z within that bound of a threshold
//    is recomputed exactly in float64 by the whole warp from the input row and
//    the float64 eigenvectors, so every code equals the exact-arithmetic code.
// Heads whose QJL dimension m exceeds MSIG are left to the reference kernel.
// Every mbarrier wait is bounded (see sm100.cuh); a timeout sets a device
// flag bit and the kernel skips the remaining work without hanging.
#pragma once

#include "sm100.cuh"
#include "sq_common.cuh"

namespace sq {
namespace tcc {

constexpr int D = 128;
constexpr int TILE = 128;
constexpr int NGRP = 3;                       // epilogue groups = X stages = TMEM accumulators
constexpr int KB = D / 64;
constexpr int X_BYTES = TILE * D * 2;
constexpr int B_BYTES = D * D * 2;
constexpr int NUM_WARPS = 2 + 4 * NGRP;
constexpr int NUM_THREADS = NUM_WARPS * 32;
constexpr int WARP_PROD = 0, WARP_MMA = 1, WARP_EPI0 = 2;
constexpr uint32_t TMEM_COLS = 512;            // NGRP accumulators of D columns (a power of two)
constexpr int MSIG = 8;                       // largest QJL dimension handled here
constexpr int EACC_DEFAULT_UNITS = 32;        // accumulation bound factor, in units of 2^-24

struct CoordInfo {
  uint32_t bo;       // bits (low 8) | bit offset << 8
  float sc;          // 2^-s (column scale of B, one per head)
  float dfix;        // split residual ||e_i|| + fp32 rounding of z, 1/||x||, thresholds
  float dacc;        // ||V_i / sigma_i|| = 1/sigma_i: multiplies the accumulation bound
};
// Per-head summary used by the kernel: chunk classes and per-width radii.
struct TcMeta {
  uint32_t chunk[D / 16];   // width 0..8 if all 16 coordinates share it (no signal one), else kMixed
  float dfix_w[12];         // max dfix over the non-signal coordinates of each width
  float dacc_w[12];         // max dacc over the same
  float dfix_c[D / 16];     // max dfix over the non-signal coordinates of each chunk
  float dacc_c[D / 16];     // max dacc over the same
  uint32_t reserved[16];
};
constexpr uint32_t kMixed = 0xFFu;
static_assert(sizeof(TcMeta) == 256, "meta block is 256 bytes");

// Cell tables of widths 4..8 (built on the host from the library codebook):
// cell g of width b covers |z| in [g h_b, (g+1) h_b) with h_b = 2^-(b-2),
// narrower than every gap between consecutive thresholds, so a cell holds at
// most one threshold. cell[g] = number of positive thresholds below g h_b;
// q[j] = (T_j, T_j+1, T_j+2) with T_0 = 0 and +inf past the last threshold.
__host__ __device__ constexpr int cell_off(int b) {
  return b == 4 ? 0 : b == 5 ? 16 : b == 6 ? 48 : b == 7 ? 112 : 240;
}
__host__ __device__ constexpr int cell_cap(int b) {
  return b == 4 ? 16 : b == 5 ? 32 : b == 6 ? 64 : b == 7 ? 128 : 320;
}
constexpr int kCellBytes = 560;
__host__ __device__ constexpr int q_off(int b) { return (1 << (b - 1)) - 8; }
constexpr int kQEntries = 248;
struct QuantConst {
  float t2;            // positive threshold of width 2
  float t3[3];         // positive thresholds of width 3
  int ncell[12];       // cells in use per width (4..8)
};

// Byte offsets of the dynamic shared memory (base aligned to 1024).
constexpr int OFF_X = 0;
constexpr int OFF_BHI = OFF_X + NGRP * X_BYTES;
constexpr int OFF_BLO = OFF_BHI + B_BYTES;
constexpr int OFF_TH64 = OFF_BLO + B_BYTES;                         // double [kThreshTotal]
constexpr int OFF_LV64 = OFF_TH64 + ((kThreshTotal * 8 + 15) & ~15);   // double [kLevelsTotal]
constexpr int OFF_Q = OFF_LV64 + ((kLevelsTotal * 8 + 15) & ~15);      // float4 [kQEntries]
constexpr int OFF_CELL = OFF_Q + kQEntries * 16;                       // u8 [kCellBytes]
constexpr int OFF_BAR = OFF_CELL + kCellBytes;
constexpr int N_BARS = 4 * NGRP + 3;
constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;                         // u32 [16]
constexpr int OFF_R = OFF_MISC + 64;                                   // float [NGRP][32]: radius per width, per chunk
constexpr int OFF_CD = OFF_R + NGRP * 128;                             // u32 [NGRP][8]: chunk classes
constexpr int OFF_RUN = OFF_CD + NGRP * 32;                            // u16 [NGRP][8][16]: runs of mixed chunks
constexpr int OFF_SC = OFF_RUN + NGRP * 8 * 16 * 2;                    // u8 [NGRP * 4][32][MSIG]: signal codes
constexpr int OFF_VS = (OFF_SC + NGRP * 4 * 32 * MSIG + 15) & ~15;     // double [NGRP][MSIG][D]: signal rows of V^T
constexpr int OFF_MX = OFF_VS + NGRP * MSIG * D * 8;                   // float [NGRP * 4][32][16]: mixed-chunk values
constexpr int SMEM_BYTES = OFF_MX + NGRP * 4 * 32 * 16 * 4 + 1024;     // + alignment slack
// A run of a mixed chunk (u16): width (bits 0-3), signal flag (bit 4), length - 1 (bits 8-11).
static_assert(SMEM_BYTES <= 232448, "shared memory plan exceeds 227 KB");
static_assert(OFF_BAR % 8 == 0, "mbarriers need 8-byte alignment");

// The tensor-core block inside the record's derived part (derived_tc_off):
// Bhi, Blo, Blo2 [d*d fp16 each] (swizzled B operand; B = hi + lo + lo2 to
// about 2^-33 relative), CoordInfo [d], TcMeta, Vt64 [d*d f64].
struct TcView {
  uint8_t* base;
  int d;
  __host__ __device__ __half* bhi() const { return (__half*)base; }
  __host__ __device__ __half* blo() const { return (__half*)(base + 2 * (size_t)d * d); }
  __host__ __device__ __half* blo2() const { return (__half*)(base + 4 * (size_t)d * d); }
  __host__ __device__ CoordInfo* ci() const { return (CoordInfo*)(base + 6 * (size_t)d * d); }
  __host__ __device__ TcMeta* meta() const { return (TcMeta*)(base + 6 * (size_t)d * d + 16 * (size_t)d); }
  __host__ __device__ double* vt64() const {
    return (double*)(base + 6 * (size_t)d * d + 16 * (size_t)d + sizeof(TcMeta));
  }
};
__host__ __device__ inline TcView tc_view(Rec r) { return TcView{r.derived() + derived_tc_off(r.d), r.d}; }

// Byte offset of element (row n, column k) of an [rows x D] K-major fp16 operand
// in the 128-byte-swizzled canonical layout (64-column blocks of rows*128 bytes).
__host__ __device__ inline uint32_t sw128_off(int n, int k, int rows) {
  int kb = k >> 6, e = k & 63, c = e >> 3, w = e & 7;
  return (uint32_t)(kb * rows * 128 + (n >> 3) * 1024 + (n & 7) * 128 + ((c ^ (n & 7)) << 4) + (w << 1));
}

// Builds the tensor-core block of one record (called with all of the block's threads).
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
  __syncthreads();
  if (tid == 0) {
    TcMeta mt;
    const int m = rec.hdr()->m;
    for (int b = 0; b < 12; ++b) mt.dfix_w[b] = mt.dacc_w[b] = 0.0f;
    for (int e = 0; e < 16; ++e) mt.reserved[e] = 0u;
    for (int c = 0; c < D / 16; ++c) mt.dfix_c[c] = mt.dacc_c[c] = 0.0f;
    for (int i = m; i < D; ++i) {
      const int b = (int)(tv.ci()[i].bo & 0xFFu);
      mt.dfix_w[b] = fmaxf(mt.dfix_w[b], tv.ci()[i].dfix);
      mt.dacc_w[b] = fmaxf(mt.dacc_w[b], tv.ci()[i].dacc);
      mt.dfix_c[i / 16] = fmaxf(mt.dfix_c[i / 16], tv.ci()[i].dfix);
      mt.dacc_c[i / 16] = fmaxf(mt.dacc_c[i / 16], tv.ci()[i].dacc);
    }
    for (int c = 0; c < D / 16; ++c) {
      const uint32_t b0 = tv.ci()[16 * c].bo & 0xFFu;
      bool uni = 16 * c >= m;
      for (int k = 1; k < 16 && uni; ++k) uni = (tv.ci()[16 * c + k].bo & 0xFFu) == b0;
      mt.chunk[c] = uni ? b0 : kMixed;
    }
    *tv.meta() = mt;
  }
  __syncthreads();
}

struct Params {
  const uint8_t* recs;
  const __half* x;   // the input rows (exact recomputations reread them)
  int n_heads, batch;
  int64_t n_tok;
  const int32_t* start_pos;
  CacheArgs c;
  uint32_t* flags;
  int64_t n_tiles;
  int tiles_per_row;
  float eacc;        // accumulation bound factor of the radius
};

// ---------------------------------------------------------------- quantizers
// Each returns the code of z under the unit-Gaussian Lloyd-Max thresholds of
// its width and sets dg when z lies within R of a threshold (including 0).
// Ties in that band go to the exact recomputation, so the tie rule of the
// fast path does not matter.
__device__ __forceinline__ uint32_t qz1(float z, float R, bool& dg) {
  dg = fabsf(z) < R;
  return z > 0.0f ? 1u : 0u;
}
__device__ __forceinline__ uint32_t qz2(float z, float t1, float R, bool& dg) {
  const float a = fabsf(z);
  dg = fminf(a, fabsf(a - t1)) < R;
  const uint32_t m = a > t1 ? 1u : 0u;
  return z > 0.0f ? 2u + m : 1u - m;
}
__device__ __forceinline__ uint32_t qz3(float z, float t1, float t2, float t3, float R, bool& dg) {
  const float a = fabsf(z);
  dg = fminf(fminf(a, fabsf(a - t1)), fminf(fabsf(a - t2), fabsf(a - t3))) < R;
  const uint32_t m = (a > t1 ? 1u : 0u) + (a > t2 ? 1u : 0u) + (a > t3 ? 1u : 0u);
  return z > 0.0f ? 4u + m : 3u - m;
}
// Widths 4..8: cell index by the 2^23 rounding trick (floor of |z| / h, or one
// below it on an exact tie, both of which the table handles), then at most
// one comparison.
__device__ __forceinline__ uint32_t qzl(float z, const uint8_t* cell, const float4* q, float invh, int ncell,
                                        uint32_t half, float R, bool& dg) {
  const float a = fabsf(z);
  int g = __float_as_int(fmaf(a, invh, 8388607.5f)) - 0x4B000000;
  g = min(max(g, 0), ncell - 1);
  const int lo = cell[g];
  const float4 e = q[lo];
  const uint32_t up = a > e.y ? 1u : 0u;
  dg = fminf(fminf(a - e.x, fabsf(a - e.y)), e.z - a) < R;
  const uint32_t m = (uint32_t)lo + up;
  return z > 0.0f ? half + m : half - 1u - m;
}

// Per-thread quantization context of one segment (one head).
struct QCtx {
  const uint8_t* smb;      // shared-memory base (cell tables, radii)
  int wr;                  // this group's radius row: radius of width b at float index wr + b (chunks from wr + 16)
  float zr;                // 2^-s / ||x|| of this thread's row
  __device__ __forceinline__ float R(int b) const { return ((const float*)(smb + OFF_R))[wr + b]; }
  __device__ __forceinline__ const uint8_t* cell() const { return smb + OFF_CELL; }
  __device__ __forceinline__ const float4* q() const { return (const float4*)(smb + OFF_Q); }
};

template <int B>
__device__ __forceinline__ uint32_t quant(float z, float R, const QCtx& c, const QuantConst& k, bool& dg) {
  if (B == 1) return qz1(z, R, dg);
  else if (B == 2) return qz2(z, k.t2, R, dg);
  else if (B == 3) return qz3(z, k.t3[0], k.t3[1], k.t3[2], R, dg);
  else
    return qzl(z, c.cell() + cell_off(B), c.q() + q_off(B), (float)(1 << (B >= 2 ? B - 2 : 0)), k.ncell[B], 1u << (B - 1), R,
               dg);
}

// Little-endian bit stream of one record, written to global memory a word at
// a time (word w at dst[32 w]: the interleaved cache layout, so the 32 lanes of
// a warp, 32 consecutive tokens, store one 128-byte line per word). fill and nw
// are the same in every lane of a warp (one head).
struct Stream {
  uint32_t acc;      // the fill (< 32) pending low bits of the next word
  int fill;
  int nw;            // words written so far
  uint32_t* dst;
  bool st;
};
__device__ __forceinline__ void put(Stream& s, uint32_t v, int n) {   // 1 <= n <= 32, v < 2^n
  const uint32_t lo = s.acc | (v << s.fill);
  const uint32_t carry = __funnelshift_l(v, 0u, s.fill);   // bits of v past the word
  const int nf = s.fill + n;
  const bool full = nf >= 32;
  if (full && s.st) s.dst[(size_t)s.nw * 32] = lo;
  s.nw += full ? 1 : 0;
  s.acc = full ? carry : lo;
  s.fill = nf & 31;
}
// Appends the NB bits held in cw[0 .. ceil(NB/32)) (NB a multiple of 16, at
// most 128) in one step: every word that completes is a funnel shift of two
// neighbours, so the appends of a chunk do not form a serial chain.
template <int NB>
__device__ __forceinline__ void put_bits(Stream& s, const uint32_t* cw) {
  constexpr int NI = (NB + 31) / 32;          // input words
  uint32_t w[NI + 1];
  uint32_t prev = s.acc;
#pragma unroll
  for (int j = 0; j <= NI; ++j) {
    const uint32_t cur = j < NI ? cw[j] : 0u;
    w[j] = s.fill ? __funnelshift_l(prev, cur, s.fill) | 0u : cur;
    prev = cur;
  }
  // word 0 also carries the pending bits
  w[0] = s.acc | (cw[0] << s.fill);
  const int tot = s.fill + NB;
  const int nfull = tot >> 5;                 // NB/32 or NB/32 + 1 (NB/32 rounded down)
#pragma unroll
  for (int j = 0; j <= NI; ++j)
    if (j < nfull && s.st) s.dst[(size_t)(s.nw + j) * 32] = w[j];
  constexpr int lo = NB / 32;
  s.acc = (nfull == lo) ? w[lo] : w[lo < NI ? lo + 1 : NI];
  s.nw += nfull;
  s.fill = tot & 31;
}

// Byte offset of the 16-byte chunk c (elements 8c .. 8c+7) of token row t in an X stage.
__device__ __forceinline__ uint32_t x_chunk(int t, int c) {
  return (uint32_t)((c >> 3) * (TILE * 128) + (t >> 3) * 1024 + (t & 7) * 128 + (((c & 7) ^ (t & 7)) << 4));
}

// Flag bits of the coordinates whose z fell within the radius of a threshold:
// 128 bits per lane (fm[q] holds coordinates 32q .. 32q + 31).
__device__ __forceinline__ void flag_chunk(uint32_t (&fm)[4], int c, uint32_t dm) {
  const uint32_t sh = dm << ((c & 1) * 16);
#pragma unroll
  for (int q = 0; q < 4; ++q) fm[q] |= (c >> 1) == q ? sh : 0u;
}

// Exact repair of the flagged codes of a warp's 32 records (word w of the
// lane's record at rec[32 w]), after they have been written: rounds of up to RB (lane, coordinate) entries, each
// recomputed by the whole warp in float64 (lane l takes elements 4l .. 4l+3 of
// the input row and of the eigenvector; the loads of a round are all issued
// before any reduction), z = (V_i . x) / ||x|| / sigma_i, and the owner lane
// overwrites the b_i-bit field of its record.
constexpr int RB = 2;   // repairs per round (their loads are in flight together)
__device__ __forceinline__ void repair_warp(uint4 fmv, const __half* x, int64_t xbase, uint32_t* rec,
                                         const double* vt64, const double* sig, const uint8_t* bits,
                                         const int32_t* offs, bool normalize, const double* th64, int lane) {
  uint32_t fm[4] = {fmv.x, fmv.y, fmv.z, fmv.w};
  for (;;) {
    const uint32_t fl = fm[0] | fm[1] | fm[2] | fm[3];
    uint32_t have = __ballot_sync(0xffffffffu, fl != 0u);
    if (!have) break;
    // my lowest flagged coordinate
    int mine = -1;
#pragma unroll
    for (int q = 3; q >= 0; --q)
      if (fm[q]) mine = q * 32 + __ffs(fm[q]) - 1;
    int src[RB], crd[RB];
    int n = 0;
#pragma unroll
    for (int k = 0; k < RB; ++k) {
      src[k] = -1;
      crd[k] = 0;
      if (have) {
        src[k] = __ffs(have) - 1;
        have &= have - 1u;
        crd[k] = __shfl_sync(0xffffffffu, mine, src[k]);
        ++n;
      }
    }
    uint2 xr[RB];
    double2 va[RB], vb[RB];
#pragma unroll
    for (int k = 0; k < RB; ++k) {
      if (src[k] >= 0) {
        xr[k] = *(const uint2*)(x + (xbase + src[k]) * D + 4 * lane);
        const double* vr = vt64 + (size_t)crd[k] * D + 4 * lane;
        va[k] = *(const double2*)vr;
        vb[k] = *(const double2*)(vr + 2);
      }
    }
#pragma unroll
    for (int k = 0; k < RB; ++k) {
      if (src[k] < 0) continue;
      const __half2* hh = reinterpret_cast<const __half2*>(&xr[k]);
      const float2 a = __half22float2(hh[0]), c = __half22float2(hh[1]);
      double dot = (double)a.x * va[k].x;
      dot = fma((double)a.y, va[k].y, dot);
      dot = fma((double)c.x, vb[k].x, dot);
      dot = fma((double)c.y, vb[k].y, dot);
      double n2 = (double)a.x * a.x;
      n2 = fma((double)a.y, (double)a.y, n2);
      n2 = fma((double)c.x, (double)c.x, n2);
      n2 = fma((double)c.y, (double)c.y, n2);
      dot = warp_sum(dot);
      n2 = warp_sum(n2);
      if (lane == src[k]) {
        const int i = crd[k];
        const double nrm = normalize ? sqrt(n2) : 1.0;
        const double inv = nrm > 0.0 ? 1.0 / nrm : 0.0;
        const double s = sig[i];
        const int b = bits[i];
        const double yn = dot * inv;
        const uint32_t code = (uint32_t)code_of(s > 0.0 ? yn * (1.0 / s) : 0.0, th64 + th_off(b), b);
        // patch the field with two reductions (no read back of the word; the
        // same thread's operations on one address stay in order)
        const int o = offs[i], wi = o >> 5, sh = o & 31;
        const uint32_t mask = (1u << b) - 1u;
        atomicAnd(&rec[(size_t)wi * 32], ~(mask << sh));
        atomicOr(&rec[(size_t)wi * 32], code << sh);
        if (sh + b > 32) {
          atomicAnd(&rec[(size_t)(wi + 1) * 32], ~(mask >> (32 - sh)));
          atomicOr(&rec[(size_t)(wi + 1) * 32], code >> (32 - sh));
        }
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if ((i >> 5) == q) fm[q] &= ~(1u << (i & 31));
      }
    }
  }
}

// Norm phase of a key row with QJL (m <= MM signal coordinates): ||x|| and
// y_i = V_i . x for i < MM in float64 from the staged tile (the rows i >= m
// are computed and ignored), then the signal codes, the residual
// r_i = y_i / ||x|| - sigma_i level_i, rho = ||r|| and the m sign bits of S r.
template <int MM>
__device__ __forceinline__ void key_pass(const uint8_t* xs, int t, int m, const double* vsig, const double* sig,
                                         const uint8_t* bits, const double* S, bool normalize, const double* th64,
                                         const double* lv64, double& nrm, double& rho2, uint8_t* scode,
                                         uint32_t& qbits) {
  // two partial sums per quantity (even and odd j; for MM <= 4) halve the dependent chains
  double n2a = 0.0, n2b = 0.0;
  double ys[MM], yo[MM];
#pragma unroll
  for (int i = 0; i < MM; ++i) ys[i] = yo[i] = 0.0;
#pragma unroll 1
  for (int c = 0; c < D / 8; ++c) {
    const uint4 raw = *(const uint4*)(xs + x_chunk(t, c));
    const __half2* h2 = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __half22float2(h2[e]);
      const double x0 = f.x, x1 = f.y;
      n2a = fma(x0, x0, n2a);
      n2b = fma(x1, x1, n2b);
      const int jj = c * 8 + 2 * e;
#pragma unroll
      for (int i = 0; i < MM; ++i) {
        const double2 vv = *(const double2*)(vsig + i * D + jj);   // same address in every lane
        ys[i] = fma(x0, vv.x, ys[i]);
        if (MM <= 4) yo[i] = fma(x1, vv.y, yo[i]);
        else ys[i] = fma(x1, vv.y, ys[i]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < MM; ++i) ys[i] += yo[i];   // (zero when MM > 4)
  nrm = normalize ? sqrt(n2a + n2b) : 1.0;
  const double inv = nrm > 0.0 ? 1.0 / nrm : 0.0;
  rho2 = 0.0;
#pragma unroll
  for (int i = 0; i < MM; ++i) {
    if (i < m) {
      const int b = bits[i];
      const double yn = ys[i] * inv;
      double lvv = 0.0;
      if (b > 0) {
        const double s = sig[i];
        const double z = s > 0.0 ? yn / s : 0.0;
        const int code = code_of(z, th64 + th_off(b), b);
        lvv = lv64[lv_off(b) + code];
        scode[i] = (uint8_t)code;
      }
      ys[i] = yn - sig[i] * lvv;
      rho2 = fma(ys[i], ys[i], rho2);
    }
  }
  qbits = 0u;
  for (int j = 0; j < m; ++j) {
    double pj = 0.0;
#pragma unroll
    for (int i = 0; i < MM; ++i)
      if (i < m) pj = fma(S[j * m + i], ys[i], pj);
    qbits |= (pj >= 0.0 ? 1u : 0u) << j;
  }
}

// One width-uniform chunk of 16 coordinates: codes into cw (compile-time
// positions), flags of the in-band ones, then the stream.
template <int B>
__device__ __forceinline__ void chunk_uniform(const float* v, float Rc, const QCtx& qc, const QuantConst& kq,
                                              bool fix_ok, int c, uint32_t (&fm)[4], Stream& s) {
  uint32_t cw[4] = {0u, 0u, 0u, 0u};
  uint32_t dm = 0u;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    bool dg;
    const uint32_t code = quant<B>(v[k] * qc.zr, Rc, qc, kq, dg);
    dm |= dg ? (1u << k) : 0u;
    const int p = B * k;
    cw[p >> 5] |= code << (p & 31);
    if ((p & 31) + B > 32) cw[(p >> 5) + 1] |= code >> (32 - (p & 31));
  }
  flag_chunk(fm, c, fix_ok ? dm : 0u);
  put_bits<16 * B>(s, cw);
}

// One run of a mixed chunk: len coordinates of width B starting at chunk
// position k0 (values in the lane's swizzled scratch row), each code appended
// to the stream; returns the in-band flags of the run (bit k for position k).
template <int B>
__device__ __forceinline__ uint32_t run_codes(const float* mx, int lane, int k0, int len, const QCtx& qc,
                                              const QuantConst& kqc, Stream& s) {
  const float R = qc.R(B);
  uint32_t dm = 0u;
#pragma unroll 1
  for (int k = k0; k < k0 + len; ++k) {
    bool dg;
    const uint32_t code = quant<B>(mx[k ^ (lane & 15)] * qc.zr, R, qc, kqc, dg);
    dm |= (dg ? 1u : 0u) << k;
    put(s, code, B);
  }
  return dm;
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
k_compress_tc(const __grid_constant__ CUtensorMap tmap, Params P, const __grid_constant__ QuantConst KQ) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // aligned by pointer arithmetic on the shared array, so that every access
  // below stays a shared-memory access (an integer round trip would make them generic)
  uint8_t* sm = smem_raw + ((1024u - (sm100::smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sX = sm + OFF_X;
  uint8_t* sBhi = sm + OFF_BHI;
  uint8_t* sBlo = sm + OFF_BLO;
  double* sTh64 = (double*)(sm + OFF_TH64);
  double* sLv64 = (double*)(sm + OFF_LV64);
  float4* sQ = (float4*)(sm + OFF_Q);
  uint8_t* sCell = sm + OFF_CELL;
  uint64_t* bars = (uint64_t*)(sm + OFF_BAR);
  uint64_t* full = bars;                    // [NGRP] X stage landed
  uint64_t* empty = bars + NGRP;            // [NGRP] X stage free (MMA done + 4 epilogue warps)
  uint64_t* tfull = bars + 2 * NGRP;        // [NGRP] accumulator ready
  uint64_t* tempty = bars + 3 * NGRP;       // [NGRP] accumulator drained
  uint64_t* bfull = bars + 4 * NGRP;        // B operand landed
  uint64_t* bempty = bfull + 1;             // B operand no longer read
  uint64_t* drain = bfull + 2;              // every MMA this CTA issued has completed (before the free)
  uint32_t* misc = (uint32_t*)(sm + OFF_MISC);   // [0] tmem base, [1] abort
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  for (int e = threadIdx.x; e < kThreshTotal; e += NUM_THREADS) sTh64[e] = c_th64[e];
  for (int e = threadIdx.x; e < kLevelsTotal; e += NUM_THREADS) sLv64[e] = c_lv64[e];
  for (int e = threadIdx.x; e < kQEntries; e += NUM_THREADS) sQ[e] = c_tcq[e];
  for (int e = threadIdx.x; e < kCellBytes; e += NUM_THREADS) sCell[e] = c_tccell[e];
  if (threadIdx.x == 0) {
    for (int s = 0; s < NGRP; ++s) {
      sm100::mbar_init(&full[s], 1);
      sm100::mbar_init(&empty[s], 1 + 4);
      sm100::mbar_init(&tfull[s], 1);
      sm100::mbar_init(&tempty[s], 4);
    }
    sm100::mbar_init(bfull, 1);
    sm100::mbar_init(bempty, 1);
    sm100::mbar_init(drain, 1);
    misc[1] = 0u;
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
  const uint32_t idesc = sm100::idesc_f16(TILE, D);
  // Every role walks the same sequence of segments (rows of tiles of one
  // (batch, head)) and skips the same invalid ones, so k (tiles processed)
  // and nseg (segments processed) agree across roles.
  uint32_t k = 0, nseg = 0;
  uint32_t x_issued = 0, b_issued = 0;   // producer: X tiles and B operands requested (a prefix of each)

  const int grp = (warp - WARP_EPI0) >> 2;             // epilogue group (warps 2..17)
  const int qtr = warp & 3;                            // TMEM lane quarter of this warp
  const int t_row = qtr * 32 + lane;                   // token row within the tile

  for (int64_t s0 = tb; s0 < te;) {
    const int64_t row = s0 / P.tiles_per_row;
    const int64_t s1 = min(te, (row + 1) * (int64_t)P.tiles_per_row);
    const int h = (int)(row % P.n_heads);
    const int bidx = (int)(row / P.n_heads);
    Rec rec = rec_at(P.recs, D, h);
    const RecHeader* hd = rec.hdr();
    const bool rec_ok = record_ok(hd, D) && hd->words == P.c.words && (hd->m == 0 || P.c.rnorm != nullptr);
    // records with fitted codebooks are left to the reference kernel's second pass
    const bool fitted = (hd->flags & kFlagFitted) != 0u;
    const int64_t sp = P.start_pos ? (int64_t)P.start_pos[bidx] : 0;
    const bool cap_ok = sp >= 0 && sp + P.n_tok <= P.c.cap;
    if (threadIdx.x == 0 && err) {
      if (!rec_ok) atomicOr(err, SQ_FLAG_RECORD);
      else if (!cap_ok) atomicOr(err, SQ_FLAG_CAPACITY);
    }
    const int m = rec_ok ? hd->m : 0;
    if (!rec_ok || !cap_ok || m > MSIG || fitted) {   // m > MSIG, fitted: the reference kernel takes this head
      s0 = s1;
      continue;
    }
    TcView tv = tc_view(rec);
    const int64_t nt = s1 - s0;

    if (warp == WARP_PROD) {
      if (lane == 0) {
        bool ok = *abort_flag == 0;
        if (ok && nseg > 0) ok = sm100::mbar_wait(bempty, (nseg - 1) & 1u, err);
        if (!ok) {
          *abort_flag = 1;
        } else {
          sm100::mbar_expect_tx(bfull, 2 * B_BYTES);
          sm100::bulk_load(sBhi, tv.bhi(), B_BYTES, bfull);
          sm100::bulk_load(sBlo, tv.blo(), B_BYTES, bfull);
          ++b_issued;
        }
        for (int64_t j = 0; j < nt; ++j) {
          const uint32_t kk = k + (uint32_t)j;
          const int st = (int)(kk % NGRP);
          const uint32_t ph = (kk / NGRP) & 1u;
          if (*abort_flag || !sm100::mbar_wait(&empty[st], ph ^ 1u, err)) { *abort_flag = 1; continue; }
          const int64_t tile = s0 + j;
          const int t0 = (int)((tile - row * P.tiles_per_row) * TILE);
          const int ycoord = (int)(row * P.n_tok + t0);
          sm100::mbar_expect_tx(&full[st], X_BYTES);
          for (int kb = 0; kb < KB; ++kb)
            sm100::tma_load_2d(sX + st * X_BYTES + kb * (TILE * 128), &tmap, &full[st], kb * 64, ycoord);
          ++x_issued;
        }
      }
    } else if (warp == WARP_MMA) {
      if (lane == 0) {
        if (*abort_flag || !sm100::mbar_wait(bfull, nseg & 1u, err)) *abort_flag = 1;
        for (int64_t j = 0; j < nt; ++j) {
          const uint32_t kk = k + (uint32_t)j;
          const int st = (int)(kk % NGRP);
          const uint32_t ph = (kk / NGRP) & 1u;
          if (*abort_flag || !sm100::mbar_wait(&full[st], ph, err) ||
              !sm100::mbar_wait(&tempty[st], ph ^ 1u, err)) {
            *abort_flag = 1;
            continue;
          }
          sm100::tc_fence_after();
          const uint32_t dt = tmem_base + (uint32_t)(st * D);
          const uint32_t xa = sm100::smem_u32(sX + st * X_BYTES);
          const uint32_t bh = sm100::smem_u32(sBhi), bl = sm100::smem_u32(sBlo);
#pragma unroll
          for (int kb = 0; kb < KB; ++kb) {
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
              const uint32_t ao = kb * (TILE * 128) + k4 * 32, bo = kb * (D * 128) + k4 * 32;
              const uint64_t ad = sm100::sw128_desc(xa + ao);
              sm100::mma_f16(dt, ad, sm100::sw128_desc(bh + bo), idesc, (kb | k4) ? 1u : 0u);
              sm100::mma_f16(dt, ad, sm100::sw128_desc(bl + bo), idesc, 1u);
            }
          }
          sm100::mma_commit(&empty[st]);
          sm100::mma_commit(&tfull[st]);
        }
        sm100::mma_commit(bempty);
      }
    } else {
      // ---------------- epilogue group grp: tiles k with k mod NGRP == grp
      const int W = hd->words;
      const bool normalize = (hd->flags & kFlagNormalize) != 0;
      const TcMeta* mt = tv.meta();
      const double* vt64 = tv.vt64();
      const double* sig = rec.sigma();
      const uint8_t* bits = rec.bits();
      QCtx qc;
      qc.smb = sm;
      qc.wr = grp * 32;
      const float* rch = (const float*)(sm + OFF_R) + grp * 32 + 16;   // radius per chunk
      qc.zr = 0.0f;
      // Per-segment constants of this group: wait until its four warps are done
      // with the previous segment, load, and wait again (named barrier 1 + grp).
      double* vsig = (double*)(sm + OFF_VS) + grp * MSIG * D;
      uint32_t* cdw = (uint32_t*)(sm + OFF_CD) + grp * 8;
      uint16_t* runs = (uint16_t*)(sm + OFF_RUN) + grp * 8 * 16;
      sm100::named_bar(1 + grp, 128);
      {
        const int gt = (warp & 3) * 32 + lane;        // 0..127 within the group
        const int nrow = m < MSIG ? m : MSIG;
        for (int e = gt; e < nrow * D / 2; e += 128)
          ((double2*)vsig)[e] = ((const double2*)vt64)[e];
        if (gt <= 8)
          ((float*)(sm + OFF_R))[grp * 32 + gt] = fmaf(P.eacc, mt->dacc_w[gt], mt->dfix_w[gt]) + 2.0e-6f;
        if (gt >= 16 && gt < 16 + D / 16)
          ((float*)(sm + OFF_R))[grp * 32 + gt] =
              fmaf(P.eacc, mt->dacc_c[gt - 16], mt->dfix_c[gt - 16]) + 2.0e-6f;
        if (gt >= 32 && gt < 40) {
          // chunk class; for a mixed chunk, its runs of one width (signal
          // coordinates in runs of their own)
          const int c = gt - 32;
          uint32_t cd = mt->chunk[c];
          if (cd == kMixed) {
            int nr = 0, k = 0;
            while (k < 16) {
              const int i0 = c * 16 + k;
              const int b0 = bits[i0];
              const bool s0 = i0 < m;
              int len = 1;
              while (k + len < 16 && bits[i0 + len] == b0 && ((i0 + len) < m) == s0) ++len;
              runs[c * 16 + nr] = (uint16_t)(b0 | (s0 ? 16 : 0) | ((len - 1) << 8));
              ++nr;
              k += len;
            }
            cd = kMixed | ((uint32_t)nr << 8);
          }
          cdw[c] = cd;
        }
      }
      sm100::named_bar(1 + grp, 128);
      const float sc = tv.ci()[0].sc;
      const double* S = rec.S();
      for (int64_t j = 0; j < nt; ++j) {
        const uint32_t kk = k + (uint32_t)j;
        if ((int)(kk % NGRP) != grp) continue;
        const int st = grp;
        const uint32_t ph = (kk / NGRP) & 1u;
        const int64_t tile = s0 + j;
        const int t0 = (int)((tile - row * P.tiles_per_row) * TILE);
        const int n_valid = (int)min((int64_t)TILE, P.n_tok - t0);
        const bool valid = t_row < n_valid;
        const uint8_t* xs = sX + st * X_BYTES;
        const size_t slot = ((size_t)bidx * P.n_heads + h) * P.c.cap + sp + t0 + t_row;
        const int64_t xbase = row * P.n_tok + t0 + qtr * 32;   // input row of lane 0 of this warp

        bool live = __all_sync(0xffffffffu, *abort_flag == 0 && sm100::mbar_wait(&full[st], ph, err));
        if (!live) *abort_flag = 1;
        // ---- norm phase (reads the staged tile)
        float inv32 = 0.0f;
        uint8_t* scode = sm + OFF_SC + ((warp - WARP_EPI0) * 32 + lane) * MSIG;   // this lane's signal codes
        uint32_t qbits = 0u;
        if (live) {
          if (m == 0) {
            float acc[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) acc[e] = 0.0f;
#pragma unroll
            for (int c = 0; c < D / 8; ++c) {
              const uint4 raw = *(const uint4*)(xs + x_chunk(t_row, c));
              const __half2* h2 = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 f = __half22float2(h2[e]);
                acc[(c & 1) * 8 + 2 * e] = fmaf(f.x, f.x, acc[(c & 1) * 8 + 2 * e]);
                acc[(c & 1) * 8 + 2 * e + 1] = fmaf(f.y, f.y, acc[(c & 1) * 8 + 2 * e + 1]);
              }
            }
            double n2 = 0.0;
#pragma unroll
            for (int e = 0; e < 16; ++e) n2 += (double)acc[e];
            const double nrm = normalize ? sqrt(n2) : 1.0;
            inv32 = nrm > 0.0 ? (float)(1.0 / nrm) : 0.0f;
            if (valid) P.c.norm[slot] = (float)nrm;
          } else {
            // keys with QJL: ||x||, the m signal coordinates, their codes, the
            // residual, rho and the sign bits, all in float64
            double nrm, rho2;
            if (m <= 2) key_pass<2>(xs, t_row, m, vsig, sig, bits, S, normalize, sTh64, sLv64, nrm, rho2, scode, qbits);
            else if (m == 3) key_pass<3>(xs, t_row, m, vsig, sig, bits, S, normalize, sTh64, sLv64, nrm, rho2, scode, qbits);
            else if (m <= 4) key_pass<4>(xs, t_row, m, vsig, sig, bits, S, normalize, sTh64, sLv64, nrm, rho2, scode, qbits);
            else key_pass<8>(xs, t_row, m, vsig, sig, bits, S, normalize, sTh64, sLv64, nrm, rho2, scode, qbits);
            inv32 = nrm > 0.0 ? (float)(1.0 / nrm) : 0.0f;
            if (valid) {
              P.c.norm[slot] = (float)nrm;
              P.c.rnorm[slot] = (float)sqrt(rho2);
            }
          }
        }
        __syncwarp();
        if (lane == 0) sm100::mbar_arrive(&empty[st]);   // the stage is no longer read by this warp

        // ---- codes from the accumulator
        live = __all_sync(0xffffffffu, live && *abort_flag == 0 && sm100::mbar_wait(&tfull[st], ph, err));
        if (!live) *abort_flag = 1;
        sm100::tc_fence_after();
        if (live) {
          qc.zr = sc * inv32;
          const bool fix_ok = valid && inv32 != 0.0f;
          Stream s{0u, 0, 0, P.c.codes + rec_word0((size_t)bidx * P.n_heads + h, P.c.cap, W, sp + t0 + t_row),
                   valid};
          uint32_t fm[4] = {0u, 0u, 0u, 0u};   // coordinates to repair exactly
          const uint32_t taddr = tmem_base + ((uint32_t)(qtr * 32) << 16) + (uint32_t)(st * D);
#pragma unroll 1
          for (int c = 0; c < D / 16; ++c) {
            const uint32_t cd = cdw[c];
            if (cd == 0u) continue;
            float v[16];
            sm100::tmem_ld16(taddr + (uint32_t)(c * 16), v);
            if ((cd & 0xFFu) == kMixed) {
              // widths vary inside the chunk, or it holds signal coordinates: its
              // runs of one width, each with the quantizer of that width; the
              // values go through this lane's scratch row (16 floats, XOR-swizzled
              // so that the 32 lanes hit distinct banks)
              float* mx = (float*)(sm + OFF_MX) + ((warp - WARP_EPI0) * 32 + lane) * 16;
#pragma unroll
              for (int kq = 0; kq < 16; ++kq) mx[kq ^ (lane & 15)] = v[kq];
              const int nr = (int)((cd >> 8) & 31u);
              int k0 = 0;
              uint32_t dmc = 0u;
#pragma unroll 1
              for (int r = 0; r < nr; ++r) {
                const uint32_t rn = runs[c * 16 + r];
                const int w = (int)(rn & 15u), len = (int)((rn >> 8) & 15u) + 1;
                if (w > 0) {
                  if (rn & 16u) {
                    for (int kq = k0; kq < k0 + len; ++kq) put(s, scode[(c * 16 + kq) & (MSIG - 1)], w);
                  } else {
                    switch (w) {
                      case 1: dmc |= run_codes<1>(mx, lane, k0, len, qc, KQ, s); break;
                      case 2: dmc |= run_codes<2>(mx, lane, k0, len, qc, KQ, s); break;
                      case 3: dmc |= run_codes<3>(mx, lane, k0, len, qc, KQ, s); break;
                      case 4: dmc |= run_codes<4>(mx, lane, k0, len, qc, KQ, s); break;
                      case 5: dmc |= run_codes<5>(mx, lane, k0, len, qc, KQ, s); break;
                      case 6: dmc |= run_codes<6>(mx, lane, k0, len, qc, KQ, s); break;
                      case 7: dmc |= run_codes<7>(mx, lane, k0, len, qc, KQ, s); break;
                      default: dmc |= run_codes<8>(mx, lane, k0, len, qc, KQ, s); break;
                    }
                  }
                }
                k0 += len;
              }
              flag_chunk(fm, c, fix_ok ? dmc : 0u);
            } else {
              switch (cd) {
                case 1: chunk_uniform<1>(v, rch[c], qc, KQ, fix_ok, c, fm, s); break;
                case 2: chunk_uniform<2>(v, rch[c], qc, KQ, fix_ok, c, fm, s); break;
                case 3: chunk_uniform<3>(v, rch[c], qc, KQ, fix_ok, c, fm, s); break;
                case 4: chunk_uniform<4>(v, rch[c], qc, KQ, fix_ok, c, fm, s); break;
                case 5: chunk_uniform<5>(v, rch[c], qc, KQ, fix_ok, c, fm, s); break;
                case 6: chunk_uniform<6>(v, rch[c], qc, KQ, fix_ok, c, fm, s); break;
                case 7: chunk_uniform<7>(v, rch[c], qc, KQ, fix_ok, c, fm, s); break;
                default: chunk_uniform<8>(v, rch[c], qc, KQ, fix_ok, c, fm, s); break;
              }
            }
          }
          if (m > 0) put(s, qbits, m);
          while (s.nw < W) {   // the rest of the record: remaining bits, then zero words
            if (s.st) s.dst[(size_t)s.nw * 32] = s.acc;
            s.acc = 0u;
            ++s.nw;
          }
          sm100::tc_fence_before();
          __syncwarp();
          if (lane == 0) sm100::mbar_arrive(&tempty[st]);   // the accumulator is drained
          // exact repair of the codes whose z fell within the error radius of a
          // threshold (a few per warp tile; the flagged lanes work in parallel)
          if (__any_sync(0xffffffffu, (fm[0] | fm[1] | fm[2] | fm[3]) != 0u))
            repair_warp(make_uint4(fm[0], fm[1], fm[2], fm[3]), P.x, xbase, s.dst, vt64, sig, bits, rec.offsets(),
                        normalize, sTh64, lane);
          __syncwarp();
        } else {
          sm100::tc_fence_before();
          __syncwarp();
          if (lane == 0) sm100::mbar_arrive(&tempty[st]);
        }
      }
    }
    k += (uint32_t)nt;
    ++nseg;
    s0 = s1;
  }
  // Every copy this CTA issued has landed before it exits: the last phase of
  // each stage's full barrier and of the B barrier (bounded waits).
  if (warp == WARP_PROD && lane == 0) {
    for (uint32_t j = 0; j < NGRP && j < x_issued; ++j) {
      const uint32_t it = x_issued - 1 - j;
      sm100::mbar_wait(&full[it % NGRP], (it / NGRP) & 1u, nullptr);
    }
    if (b_issued > 0) sm100::mbar_wait(bfull, (b_issued - 1) & 1u, nullptr);
  }
  // Every MMA this CTA issued has completed before its tensor memory is freed
  // (on the normal path they have: the epilogue waited for each accumulator;
  // after a timeout some may still run). Bounded like every other wait; the
  // memory is freed either way, so that no later CTA on this SM waits on it.
  if (warp == WARP_MMA) {
    if (lane == 0) {
      sm100::mma_commit(drain);
      if (!sm100::mbar_wait(drain, 0u, err)) *abort_flag = 1;
    }
    __syncwarp();
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
