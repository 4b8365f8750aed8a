// Reference-precision codec kernels: compress (rotate, quantize, QJL signs,
// pack) and decompress.
//
// SpectralQuant README, "Overview" (rotation into the calibrated eigenbasis;
// error correction kept only on the signal dimensions) and "Repository
// Structure" (spectral_rotation.py, nonuniform_quantization.py: Lloyd-Max
// codebooks, selective_qjl.py: QJL on the signal dims only).
//
// These kernels compute every coordinate in float64 (one warp per vector), so
// their codes agree with an exact evaluation except within ~1e-13 of a
// threshold. They serve float32 inputs, head_dim 256, and the decompress path.
#pragma once

#include "sq_common.cuh"

namespace sq {

constexpr int kCodecWarps = 4;

// The codebooks that code a record's coordinates, staged into shared memory as
// th[2][kThreshTotal] and lv[2][kLevelsTotal]: the record's per-regime tables
// fitted to its calibration data (flag kFlagFitted; SpectralQuant README,
// "Repository Structure": Lloyd-Max with per-regime codebooks), or the shared
// Gaussian Lloyd-Max tables in both halves.
__device__ inline void stage_codebooks(const Rec& rec, double* th, double* lv, int tid, int nth) {
  const bool fit = (rec.hdr()->flags & kFlagFitted) != 0;
  const double* ft = rec.fit_th();
  const double* fl = rec.fit_lv();
  for (int e = tid; e < 2 * kThreshTotal; e += nth) th[e] = fit ? ft[e] : c_th64[e % kThreshTotal];
  for (int e = tid; e < 2 * kLevelsTotal; e += nth) lv[e] = fit ? fl[e] : c_lv64[e % kLevelsTotal];
}
// Regime of coordinate i: 1 (noise) for i >= d_eff in a record with fitted
// codebooks, else 0 (the signal regime, or the shared tables).
__device__ __forceinline__ int regime_of(const RecHeader* h, int i) {
  return ((h->flags & kFlagFitted) != 0u && i >= h->d_eff) ? 1 : 0;
}

// The per-vector steps after the rotation, shared by the compress kernels
// that take one warp per vector at that stage: the staged tables of the
// vector's head, and the warp's word buffer and QJL residual.
struct VecEnc {
  const RecHeader* hd;
  const double* th[2];   // thresholds of each regime ([kThreshTotal] each)
  const double* lv[2];   // levels of each regime ([kLevelsTotal] each)
  const double* sig;
  const double* isig;
  const int* bits;
  const int* offs;
  uint32_t* wb;          // the record's words (zeroed before the first coordinate)
  double* rs;            // residual of the signal coordinates (keys with QJL)
  int m;
};
// Coordinate i with rotated, normalised value y: its code into the words
// (shared-memory atomics: neighbouring lanes share words) and, below m, the
// residual y - sigma_i * level.
__device__ __forceinline__ void encode_coord(const VecEnc& e, int i, double y) {
  const int bw = e.bits[i];
  int code = 0;
  const int rg = regime_of(e.hd, i);
  if (bw > 0) {
    code = code_of(y * e.isig[i], (rg ? e.th[1] : e.th[0]) + th_off(bw), bw);
    const int o = e.offs[i], wi = o >> 5, sh = o & 31;
    atomicOr(&e.wb[wi], (uint32_t)code << sh);
    if (sh + bw > 32) atomicOr(&e.wb[wi + 1], (uint32_t)code >> (32 - sh));
  }
  if (i < e.m) e.rs[i] = y - e.sig[i] * (bw > 0 ? (rg ? e.lv[1] : e.lv[0])[lv_off(bw) + code] : 0.0);
}
// After every coordinate of the vector (the warp synchronised): rho and the
// QJL signs (bit cbits + j is set when (S r)_j >= 0), then the words, ||x||
// and rho into slot pos of cache row `row`.
__device__ __forceinline__ void finish_vector(const VecEnc& e, const double* S, int cbits, int W, const CacheArgs& c,
                                              size_t row, int64_t pos, double nrm, int lane) {
  const int m = e.m;
  float rho = 0.0f;
  if (m > 0) {
    double r2 = 0.0;
    for (int k = lane; k < m; k += 32) r2 += e.rs[k] * e.rs[k];
    r2 = warp_sum(r2);
    rho = (float)sqrt(r2);
    for (int j = 0; j < m; ++j) {
      double pj = 0.0;
      for (int k = lane; k < m; k += 32) pj = fma(S[j * m + k], e.rs[k], pj);
      pj = warp_sum(pj);
      if (lane == 0 && pj >= 0.0) {
        const int o = cbits + j;
        atomicOr(&e.wb[o >> 5], 1u << (o & 31));
      }
    }
  }
  __syncwarp();
  const size_t slot = row * c.cap + pos;
  const size_t r0 = rec_word0(row, c.cap, W, pos);
  for (int w = lane; w < W; w += 32) c.codes[r0 + (size_t)w * 32] = e.wb[w];
  if (lane == 0) {
    c.norm[slot] = (float)nrm;
    if (c.rnorm) c.rnorm[slot] = rho;
  }
  __syncwarp();
}

// Shared-memory bytes of k_compress_ref / k_decompress_ref for head_dim d.
__host__ __device__ inline size_t codec_ref_smem(int d) {
  size_t v = d <= 128 ? (size_t)8 * d * (d + 1) : 0;             // V (padded rows) in float64
  return v + (size_t)16 * (kThreshTotal + kLevelsTotal)            // tables (two regimes)
         + (size_t)8 * d * 2                                      // sigma, 1/sigma
         + (size_t)4 * d * 2                                      // bits, offsets
         + (size_t)kCodecWarps * (8 * d + 4 * kMaxWords + 8 * d);        // per warp: x row, words, residual
}

// ---------------------------------------------------------------------------
// Compress: grid (token blocks, heads, batch), 4 warps, one warp per vector.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(128) k_compress_ref(const uint8_t* __restrict__ recs, const T* __restrict__ x,
                                                      int n_heads, int d, int64_t n_tok, int tok_per_block,
                                                      const int32_t* __restrict__ start_pos, CacheArgs c,
                                                      uint32_t* __restrict__ flags, int min_m) {
  extern __shared__ __align__(16) unsigned char sm[];
  const int h = blockIdx.y, b = blockIdx.z;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  Rec rec = rec_at(recs, d, h);
  const RecHeader* hd = rec.hdr();
  if (min_m > 0) {   // second pass after another kernel: heads with m >= min_m or fitted codebooks, no flags
    const int64_t sp0 = start_pos ? (int64_t)start_pos[b] : 0;
    const bool take = hd->m >= min_m || (hd->flags & kFlagFitted) != 0u;
    if (!record_ok(hd, d) || hd->words != c.words || !take || (hd->m > 0 && c.rnorm == nullptr) || sp0 < 0 ||
        sp0 + n_tok > c.cap)
      return;
  }
  if (!record_ok(hd, d) || hd->words != c.words || (hd->m > 0 && c.rnorm == nullptr)) {
    if (threadIdx.x == 0 && flags) atomicOr(flags, SQ_FLAG_RECORD);
    return;
  }
  const int64_t sp = start_pos ? (int64_t)start_pos[b] : 0;
  if (sp < 0 || sp + n_tok > c.cap) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && flags) atomicOr(flags, SQ_FLAG_CAPACITY);
    return;
  }
  const bool vsm = d <= 128;
  const int ld = d + 1;
  unsigned char* p = sm;
  double* Vs = (double*)p;            p += vsm ? (size_t)8 * d * ld : 0;
  double* th = (double*)p;            p += 16 * kThreshTotal;
  double* lv = (double*)p;            p += 16 * kLevelsTotal;
  double* sig = (double*)p;           p += 8 * d;
  double* isig = (double*)p;          p += 8 * d;
  int* bits = (int*)p;                p += 4 * d;
  int* offs = (int*)p;                p += 4 * d;
  double* xs = (double*)p + warp * d;                      p += (size_t)8 * d * kCodecWarps;
  uint32_t* wb = (uint32_t*)p + warp * kMaxWords;          p += (size_t)4 * kMaxWords * kCodecWarps;
  double* rs = (double*)p + warp * d;

  const double* Vg = rec.V();
  if (vsm)
    for (int e = threadIdx.x; e < d * d; e += blockDim.x) Vs[(e / d) * ld + e % d] = Vg[e];
  stage_codebooks(rec, th, lv, threadIdx.x, blockDim.x);
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    double s = rec.sigma()[i];
    sig[i] = s;
    isig[i] = s > 0.0 ? 1.0 / s : 0.0;
    bits[i] = rec.bits()[i];
    offs[i] = rec.offsets()[i];
  }
  __syncthreads();
  const int m = hd->m, W = hd->words, cbits = hd->code_bits;
  const bool normalize = (hd->flags & kFlagNormalize) != 0;
  const double* S = rec.S();
  const int64_t t_begin = (int64_t)blockIdx.x * tok_per_block;
  const int64_t t_end = min(n_tok, t_begin + tok_per_block);
  const size_t row = ((size_t)b * n_heads + h);
  const VecEnc enc{hd, {th, th + kThreshTotal}, {lv, lv + kLevelsTotal}, sig, isig, bits, offs, wb, rs, m};
  for (int64_t t = t_begin + warp; t < t_end; t += kCodecWarps) {
    const T* xt = x + (row * n_tok + t) * d;
    double ss = 0.0;
    for (int j = lane; j < d; j += 32) {
      double v = (double)to_float<T>(xt[j]);
      xs[j] = v;
      ss += v * v;
    }
    for (int w = lane; w < W; w += 32) wb[w] = 0u;
    ss = warp_sum(ss);
    __syncwarp();
    const double nrm = normalize ? sqrt(ss) : 1.0;
    const double inv = nrm > 0.0 ? 1.0 / nrm : 0.0;
    for (int i = lane; i < d; i += 32) {
      double y = 0.0;
      if (vsm) {
        for (int j = 0; j < d; ++j) y = fma(Vs[j * ld + i], xs[j], y);
      } else {
        for (int j = 0; j < d; ++j) y = fma(Vg[(size_t)j * d + i], xs[j], y);
      }
      y *= inv;
      encode_coord(enc, i, y);
    }
    __syncwarp();
    finish_vector(enc, S, cbits, W, c, row, sp + t, nrm, lane);
  }
}

// ---------------------------------------------------------------------------
// Append (decode steps, fewer than 16 tokens per row): grid (n_heads, vector
// groups), 256 threads. A block compresses NV (1, 2, 4 or 8, the fewest that
// hold the vectors of a head, at most 8) vectors of one head, the (batch,
// token) pairs g * NV ...; every element of V (float64, read straight from the
// record) is loaded once per block and used for all of them. Same arithmetic
// as k_compress_ref.
// ---------------------------------------------------------------------------

// Vectors per block for an append of nvec vectors per head: 1, 2, 4 or 8.
inline int append_nv(int64_t nvec) { return nvec <= 1 ? 1 : (nvec <= 2 ? 2 : (nvec <= 4 ? 4 : 8)); }

// Shared-memory bytes of append_body<T, NV>.
__host__ __device__ constexpr size_t append_smem(int nv) {
  return (size_t)nv * kMaxD * 8 + (size_t)nv * 256 * 8 + (size_t)kThreshTotal * 16 + (size_t)kLevelsTotal * 16 +
         (size_t)nv * kMaxWords * 4 + (size_t)nv * 8 + (size_t)nv * 4 + 64;
}

// One append block: head h, vectors (batch, token) pairs grp * NV ...; sm is
// append_smem(NV) bytes of shared memory; 256 threads.
template <typename T, int NV>
__device__ void append_body(const uint8_t* __restrict__ recs, const T* __restrict__ x, int batch, int n_heads, int d,
                            int64_t n_tok, const int32_t* __restrict__ start_pos, const CacheArgs& c,
                            uint32_t* __restrict__ flags, int h, int64_t grp, uint8_t* sm) {
  static_assert(NV >= 1 && NV <= 8, "one warp per vector in the norm and QJL steps");
  double (*xs)[kMaxD] = (double (*)[kMaxD])sm;                            // input, then the signal residual
  double (*ys)[256] = (double (*)[256])(sm + (size_t)NV * kMaxD * 8);    // partial sums of V^T x
  double* th = (double*)(sm + (size_t)NV * kMaxD * 8 + (size_t)NV * 256 * 8);
  double* lv = th + 2 * kThreshTotal;
  uint32_t (*wb)[kMaxWords] = (uint32_t (*)[kMaxWords])(lv + 2 * kLevelsTotal);
  double* s_inv = (double*)(wb + NV);
  int* s_ok = (int*)(s_inv + NV);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t total = (int64_t)batch * n_tok;
  const int64_t v0 = grp * NV;
  Rec rec = rec_at(recs, d, h);
  const RecHeader* hd = rec.hdr();
  if (!record_ok(hd, d) || hd->words != c.words || (hd->m > 0 && c.rnorm == nullptr)) {
    if (tid == 0 && grp == 0 && flags) atomicOr(flags, SQ_FLAG_RECORD);
    return;
  }
  const int m = hd->m, W = hd->words, cbits = hd->code_bits;
  const bool normalize = (hd->flags & kFlagNormalize) != 0;
  const double* V = rec.V();
  const double* sig = rec.sigma();
  const uint8_t* bits = rec.bits();
  const int32_t* offs = rec.offsets();
  const double* S = rec.S();
  // y = V^T x below: thread (part, i) sums j in its part of [0, d), reading the
  // column of V in batches of UB loads issued together; the first batch is
  // requested here, before the tables and inputs are staged
  constexpr int UB = NV <= 2 ? 32 : 16;
  const int nparts = 256 / d;
  const int part = tid / d, i_col = tid % d;
  const int jl = d / nparts, j_beg = part * jl, j_end = j_beg + jl;
  double vv[UB];
#pragma unroll
  for (int u = 0; u < UB; ++u) vv[u] = j_beg + u < j_end ? V[(size_t)(j_beg + u) * d + i_col] : 0.0;
  stage_codebooks(rec, th, lv, tid, 256);
  for (int e = tid; e < NV * kMaxWords; e += 256) wb[e / kMaxWords][e % kMaxWords] = 0u;
  // inputs (vectors past the end, or of rows over capacity, are zeros and not stored)
  if (tid < NV) {
    const int64_t vi = v0 + tid;
    bool ok = vi < total;
    if (ok) {
      const int b = (int)(vi / n_tok);
      const int64_t sp = start_pos ? (int64_t)start_pos[b] : 0;
      if (sp < 0 || sp + n_tok > c.cap) {
        ok = false;
        if (flags) atomicOr(flags, SQ_FLAG_CAPACITY);
      }
    }
    s_ok[tid] = ok ? 1 : 0;
  }
  for (int e = tid; e < NV * d; e += 256) {
    const int v = e / d, j = e % d;
    const int64_t vi = v0 + v;
    double xv = 0.0;
    if (vi < total) {
      const int b = (int)(vi / n_tok);
      const int64_t t = vi % n_tok;
      xv = (double)to_float<T>(x[(((size_t)b * n_heads + h) * n_tok + t) * d + j]);
    }
    xs[v][j] = xv;
  }
  __syncthreads();
  // norms: warp v
  if (warp < NV) {
    double ss = 0.0;
    for (int j = lane; j < d; j += 32) ss += xs[warp][j] * xs[warp][j];
    ss = warp_sum(ss);
    if (lane == 0) {
      const double nrm = normalize ? sqrt(ss) : 1.0;
      s_inv[warp] = nrm > 0.0 ? 1.0 / nrm : 0.0;
      const int64_t vi = v0 + warp;
      if (s_ok[warp]) {
        const int b = (int)(vi / n_tok);
        const int64_t t = vi % n_tok;
        const int64_t sp = start_pos ? (int64_t)start_pos[b] : 0;
        c.norm[((size_t)b * n_heads + h) * c.cap + sp + t] = (float)nrm;
      }
    }
  }
  // y = V^T x (first batch of V already in flight)
  {
    double acc[NV];
#pragma unroll
    for (int v = 0; v < NV; ++v) acc[v] = 0.0;
    for (int j0 = j_beg;;) {
#pragma unroll
      for (int u = 0; u < UB; ++u) {
        if (j0 + u < j_end) {
#pragma unroll
          for (int v = 0; v < NV; ++v) acc[v] = fma(vv[u], xs[v][j0 + u], acc[v]);
        }
      }
      j0 += UB;
      if (j0 >= j_end) break;
#pragma unroll
      for (int u = 0; u < UB; ++u) vv[u] = j0 + u < j_end ? V[(size_t)(j0 + u) * d + i_col] : 0.0;
    }
#pragma unroll
    for (int v = 0; v < NV; ++v) ys[v][part * d + i_col] = acc[v];
  }
  __syncthreads();
  // codes, packed into the record words; residual of the signal coordinates
  for (int e = tid; e < NV * d; e += 256) {
    const int v = e / d, i = e % d;
    const int nparts = 256 / d;
    double y = 0.0;
    for (int pt = 0; pt < nparts; ++pt) y += ys[v][pt * d + i];
    y *= s_inv[v];
    const int bw = bits[i];
    const double s = sig[i];
    const int rg = regime_of(hd, i);
    int code = 0;
    if (bw > 0) {
      code = code_of(s > 0.0 ? y * (1.0 / s) : 0.0, th + rg * kThreshTotal + th_off(bw), bw);
      const int o = offs[i], wi = o >> 5, sh = o & 31;
      atomicOr(&wb[v][wi], (uint32_t)code << sh);
      if (sh + bw > 32) atomicOr(&wb[v][wi + 1], (uint32_t)code >> (32 - sh));
    }
    if (i < m) xs[v][i] = y - s * (bw > 0 ? lv[rg * kLevelsTotal + lv_off(bw) + code] : 0.0);
  }
  __syncthreads();
  // rho and the QJL sign bits: warp v
  if (m > 0 && warp < NV) {
    double r2 = 0.0;
    for (int k = lane; k < m; k += 32) r2 += xs[warp][k] * xs[warp][k];
    r2 = warp_sum(r2);
    for (int j = 0; j < m; ++j) {
      double pj = 0.0;
      for (int k = lane; k < m; k += 32) pj = fma(S[j * m + k], xs[warp][k], pj);
      pj = warp_sum(pj);
      if (lane == 0 && pj >= 0.0) {
        const int o = cbits + j;
        atomicOr(&wb[warp][o >> 5], 1u << (o & 31));
      }
    }
    if (lane == 0 && s_ok[warp]) {
      const int64_t vi = v0 + warp;
      const int b = (int)(vi / n_tok);
      const int64_t t = vi % n_tok;
      const int64_t sp = start_pos ? (int64_t)start_pos[b] : 0;
      c.rnorm[((size_t)b * n_heads + h) * c.cap + sp + t] = (float)sqrt(r2);
    }
  }
  __syncthreads();
  for (int e = tid; e < NV * W; e += 256) {
    const int v = e / W, w = e % W;
    if (!s_ok[v]) continue;
    const int64_t vi = v0 + v;
    const int b = (int)(vi / n_tok);
    const int64_t t = vi % n_tok;
    const int64_t sp = start_pos ? (int64_t)start_pos[b] : 0;
    c.codes[rec_word0((size_t)b * n_heads + h, c.cap, W, sp + t) + (size_t)w * 32] = wb[v][w];
  }
}

template <typename T, int NV>
__global__ void __launch_bounds__(256) k_append(const uint8_t* __restrict__ recs, const T* __restrict__ x,
                                                int batch, int n_heads, int d, int64_t n_tok,
                                                const int32_t* __restrict__ start_pos, CacheArgs c,
                                                uint32_t* __restrict__ flags) {
  extern __shared__ __align__(16) uint8_t asmem[];
  append_body<T, NV>(recs, x, batch, n_heads, d, n_tok, start_pos, c, flags, blockIdx.x, blockIdx.y, asmem);
}

// ---------------------------------------------------------------------------
// Decompress: x_hat = norm * V (sigma * level) [+ QJL term]; float32 output.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) k_decompress_ref(const uint8_t* __restrict__ recs, int n_heads, int d,
                                                        CacheArgs c, int64_t t0, int64_t n_tok, int tok_per_block,
                                                        int apply_qjl, float* __restrict__ out,
                                                        uint32_t* __restrict__ flags) {
  extern __shared__ __align__(16) unsigned char sm[];
  const int h = blockIdx.y, b = blockIdx.z;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  Rec rec = rec_at(recs, d, h);
  const RecHeader* hd = rec.hdr();
  if (!record_ok(hd, d) || hd->words != c.words) {
    if (threadIdx.x == 0 && flags) atomicOr(flags, SQ_FLAG_RECORD);
    return;
  }
  if (t0 < 0 || t0 + n_tok > c.cap) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && flags) atomicOr(flags, SQ_FLAG_CAPACITY);
    return;
  }
  const bool vsm = d <= 128;
  const int ld = d + 1;
  unsigned char* p = sm;
  double* Vs = (double*)p;            p += vsm ? (size_t)8 * d * ld : 0;
  double* th = (double*)p;            p += 16 * kThreshTotal;
  double* lv = (double*)p;            p += 16 * kLevelsTotal;
  double* sig = (double*)p;           p += 8 * d;
  p += 8 * d;
  int* bits = (int*)p;                p += 4 * d;
  int* offs = (int*)p;                p += 4 * d;
  double* ws = (double*)p + warp * d; p += (size_t)8 * d * kCodecWarps;
  uint32_t* wb = (uint32_t*)p + warp * kMaxWords;

  const double* Vg = rec.V();
  if (vsm)
    for (int e = threadIdx.x; e < d * d; e += blockDim.x) Vs[(e / d) * ld + e % d] = Vg[e];
  stage_codebooks(rec, th, lv, threadIdx.x, blockDim.x);
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    sig[i] = rec.sigma()[i];
    bits[i] = rec.bits()[i];
    offs[i] = rec.offsets()[i];
  }
  __syncthreads();
  const int m = hd->m, W = hd->words, cbits = hd->code_bits;
  const bool normalize = (hd->flags & kFlagNormalize) != 0;
  const double* S = rec.S();
  const bool qjl = apply_qjl && m > 0 && c.rnorm != nullptr;
  const int64_t t_begin = (int64_t)blockIdx.x * tok_per_block;
  const int64_t t_end = min(n_tok, t_begin + tok_per_block);
  const size_t row = ((size_t)b * n_heads + h);
  for (int64_t t = t_begin + warp; t < t_end; t += kCodecWarps) {
    const size_t slot = row * c.cap + t0 + t;
    const size_t r0 = rec_word0(row, c.cap, W, t0 + t);
    for (int w = lane; w < W; w += 32) wb[w] = c.codes[r0 + (size_t)w * 32];
    __syncwarp();
    for (int i = lane; i < d; i += 32) {
      int bw = bits[i];
      ws[i] = bw > 0 ? sig[i] * lv[regime_of(hd, i) * kLevelsTotal + lv_off(bw) + (int)field(wb, offs[i], bw)] : 0.0;
    }
    __syncwarp();
    if (qjl) {
      const double rho = (double)c.rnorm[slot];
      const double coef = kQjlScale / (double)m * rho;
      for (int k = lane; k < m; k += 32) {
        double acc = 0.0;
        for (int j = 0; j < m; ++j) {
          int o = cbits + j;
          double s = ((wb[o >> 5] >> (o & 31)) & 1u) ? 1.0 : -1.0;
          acc = fma(S[j * m + k], s, acc);
        }
        ws[k] += coef * acc;
      }
      __syncwarp();
    }
    const double nrm = normalize ? (double)c.norm[slot] : 1.0;
    float* ot = out + (row * n_tok + t) * d;
    for (int j = lane; j < d; j += 32) {
      double acc = 0.0;
      if (vsm) {
        for (int i = 0; i < d; ++i) acc = fma(Vs[j * ld + i], ws[i], acc);
      } else {
        for (int i = 0; i < d; ++i) acc = fma(Vg[(size_t)j * d + i], ws[i], acc);
      }
      ot[j] = (float)(nrm * acc);
    }
    __syncwarp();
  }
}

}  // namespace sq
