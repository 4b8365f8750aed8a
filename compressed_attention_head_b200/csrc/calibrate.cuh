// Calibration kernels: second moment, Jacobi eigensolver, finalize, import.
//
// SpectralQuant README, "Overview" (a one-time calibration identifies the few
// signal dimensions of the keys) and "Repository Structure" (calibration.py:
// PCA, d_eff, kappa); tests/conftest.py fixture pre_computed_calibration
// (C = X^T X / N without centring, eigh, descending order, participation-ratio
// d_eff, gap lambda[d_eff-1] / lambda[d_eff]).
#pragma once

#include "sq_common.cuh"
#include "tc_compress.cuh"

namespace sq {

// ---------------------------------------------------------------------------
// C_h = X_h^T X_h / N in float64. Grid (heads, d/32, d/32); a block of 32x8
// threads owns one 32x32 tile of C and streams all tokens through shared
// memory in a fixed order (deterministic result).
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) k_second_moment(const T* __restrict__ x, int d, int64_t n_tok,
                                                       int64_t stride_head, int64_t stride_tok,
                                                       double* __restrict__ cov) {
  const int h = blockIdx.x, i0 = blockIdx.y * 32, j0 = blockIdx.z * 32;
  const int tx = threadIdx.x, ty = threadIdx.y;   // 32 x 8
  __shared__ double xi[32][33], xj[32][33];
  double acc[4] = {0, 0, 0, 0};
  const T* xh = x + (int64_t)h * stride_head;
  for (int64_t t0 = 0; t0 < n_tok; t0 += 32) {
    for (int r = ty; r < 32; r += 8) {
      int64_t t = t0 + r;
      double a = 0.0, b = 0.0;
      if (t < n_tok) {
        a = (double)to_float<T>(xh[t * stride_tok + i0 + tx]);
        b = (double)to_float<T>(xh[t * stride_tok + j0 + tx]);
      }
      xi[r][tx] = a;
      xj[r][tx] = b;
    }
    __syncthreads();
#pragma unroll 4
    for (int r = 0; r < 32; ++r) {
      double b = xj[r][tx];
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[k] = fma(xi[r][ty + 8 * k], b, acc[k]);
    }
    __syncthreads();
  }
  const double inv_n = 1.0 / (double)n_tok;
  double* ch = cov + (size_t)h * d * d;
#pragma unroll
  for (int k = 0; k < 4; ++k) ch[(size_t)(i0 + ty + 8 * k) * d + j0 + tx] = acc[k] * inv_n;
}

// Round-robin ("chess tournament") pairing: in round r of a sweep over d
// indices, pair k joins player 0 with 1 + r (k = 0), and otherwise the players
// 1 + (r + k) mod (d-1) and 1 + (r - k) mod (d-1). Every pair of indices meets
// exactly once per sweep of d - 1 rounds, and the pairs of a round are disjoint.
__device__ __forceinline__ void rr_pair(int r, int k, int d, int& p, int& q) {
  int n = d - 1;
  if (k == 0) {
    p = 0;
    q = 1 + (r % n);
  } else {
    p = 1 + ((r + k) % n);
    q = 1 + ((r - k + n) % n);
  }
  if (p > q) { int t = p; p = q; q = t; }
}

// ---------------------------------------------------------------------------
// Cyclic two-sided Jacobi on one symmetric matrix per block (float64).
// A lives in shared memory when d <= 128 and in the workspace otherwise; the
// accumulated rotations are kept as Vt (row p = current eigenvector p).
// Each round zeroes the d/2 disjoint (p, q) entries: rotation from the
// symmetric 2x2 Schur decomposition (tau = (a_qq - a_pp) / (2 a_pq),
// t = sign(tau) / (|tau| + sqrt(1 + tau^2)), c = 1/sqrt(1 + t^2), s = t c),
// then rows (J^T A), then columns (A J) and Vt.
// Stops when off(A) <= tol * ||A||_F or after max_sweeps sweeps.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_jacobi(double* __restrict__ cov, double* __restrict__ vt_ws,
                                                int d, int max_sweeps, double tol, void* __restrict__ recs,
                                                int* __restrict__ status) {
  extern __shared__ double smem[];
  const int h = blockIdx.x, tid = threadIdx.x, nth = blockDim.x;
  const bool in_smem = d <= 128;
  double* A = in_smem ? smem : cov + (size_t)h * d * d;
  double* Vt = vt_ws + (size_t)h * d * d;
  __shared__ double cs[kMaxD / 2], sn[kMaxD / 2];
  __shared__ int pp[kMaxD / 2], qq[kMaxD / 2];
  __shared__ double red[2][8];
  __shared__ int s_done;
  const double* src = cov + (size_t)h * d * d;
  for (int e = tid; e < d * d; e += nth) {
    if (in_smem) A[e] = src[e];
    Vt[e] = (e / d == e % d) ? 1.0 : 0.0;
  }
  __syncthreads();
  const int half = d / 2;
  int sweep = 0;
  bool converged = false;
  for (;;) {
    // off(A)^2 and ||A||_F^2
    double off = 0.0, tot = 0.0;
    for (int e = tid; e < d * d; e += nth) {
      double a = A[e];
      tot += a * a;
      if (e / d != e % d) off += a * a;
    }
    off = warp_sum(off);
    tot = warp_sum(tot);
    if ((tid & 31) == 0) { red[0][tid >> 5] = off; red[1][tid >> 5] = tot; }
    __syncthreads();
    if (tid == 0) {
      double o = 0.0, t = 0.0;
      for (int w = 0; w < nth / 32; ++w) { o += red[0][w]; t += red[1][w]; }
      s_done = (sqrt(o) <= tol * sqrt(t)) ? 1 : (sweep >= max_sweeps ? 2 : 0);
    }
    __syncthreads();
    if (s_done) { converged = (s_done == 1); break; }
    for (int r = 0; r < d - 1; ++r) {
      for (int k = tid; k < half; k += nth) {
        int p, q;
        rr_pair(r, k, d, p, q);
        double apq = A[p * d + q];
        double c = 1.0, s = 0.0;
        if (apq != 0.0) {
          double tau = (A[q * d + q] - A[p * d + p]) / (2.0 * apq);
          double t = (tau >= 0.0 ? 1.0 : -1.0) / (fabs(tau) + sqrt(1.0 + tau * tau));
          c = 1.0 / sqrt(1.0 + t * t);
          s = t * c;
        }
        cs[k] = c; sn[k] = s; pp[k] = p; qq[k] = q;
      }
      __syncthreads();
      for (int task = tid; task < half * d; task += nth) {     // rows: J^T A
        int k = task / d, j = task % d;
        int p = pp[k], q = qq[k];
        double c = cs[k], s = sn[k];
        double a = A[p * d + j], b = A[q * d + j];
        A[p * d + j] = c * a - s * b;
        A[q * d + j] = s * a + c * b;
      }
      __syncthreads();
      for (int task = tid; task < half * d; task += nth) {     // columns: A J, and Vt
        int k = task % half, i = task / half;
        int p = pp[k], q = qq[k];
        double c = cs[k], s = sn[k];
        double a = A[i * d + p], b = A[i * d + q];
        A[i * d + p] = c * a - s * b;
        A[i * d + q] = s * a + c * b;
        double va = Vt[p * d + i], vb = Vt[q * d + i];
        Vt[p * d + i] = c * va - s * vb;
        Vt[q * d + i] = s * va + c * vb;
      }
      __syncthreads();
    }
    ++sweep;
  }
  // Sort eigenvalues descending (stable on ties), fix signs, write the record.
  Rec rec = rec_at(recs, d, h);
  __shared__ double lam_s[kMaxD];
  __shared__ int order[kMaxD];
  for (int i = tid; i < d; i += nth) lam_s[i] = A[i * d + i];
  __syncthreads();
  for (int i = tid; i < d; i += nth) {
    double li = lam_s[i];
    int rank = 0;
    for (int j = 0; j < d; ++j) {
      double lj = lam_s[j];
      rank += (lj > li) || (lj == li && j < i);
    }
    order[rank] = i;
  }
  __syncthreads();
  double* lam = rec.lam();
  double* V = rec.V();
  for (int c = tid; c < d; c += nth) {
    int src_row = order[c];
    lam[c] = fmax(lam_s[src_row], 0.0);
    const double* v = Vt + (size_t)src_row * d;
    int jmax = 0;
    double amax = -1.0;
    for (int j = 0; j < d; ++j) {
      double a = fabs(v[j]);
      if (a > amax) { amax = a; jmax = j; }
    }
    double sg = v[jmax] < 0.0 ? -1.0 : 1.0;
    for (int j = 0; j < d; ++j) V[(size_t)j * d + c] = sg * v[j];
  }
  if (tid == 0) {
    rec.hdr()->sweeps = sweep;
    if (status) status[h] = converged ? SQ_OK : SQ_ERR_NOT_CONVERGED;
  }
}

// SplitMix64 (S. Vigna): output n of the stream from state s0 is
// mix(s0 + (n + 1) * golden).
__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}
__device__ __forceinline__ uint64_t sm64_at(uint64_t s0, uint64_t n) {
  return mix64(s0 + (n + 1) * 0x9E3779B97F4A7C15ull);
}

struct FinalizeArgs {
  int total_bits, is_key, qjl, normalize, d_eff_override, max_bits;
  uint64_t seed;
  double avg_bits;
  double cumvar;      // 0: participation-ratio d_eff; (0, 1]: cumulative-variance d_eff
  int rotation;       // 1: the basis is the random rotation (record flag only)
  int fitted;         // 1: per-regime codebooks fitted afterwards (k_fit_z, k_fit_lloyd)
};

// Writes one derived part (float copies) of a record whose canonical part is complete.
__device__ void build_derived(Rec rec, int tid, int nth) {
  const int d = rec.d;
  const RecHeader* hd = rec.hdr();
  const int m = hd->m;
  for (int i = tid; i < d; i += nth) {
    double s = rec.sigma()[i];
    rec.sigma_f()[i] = (float)s;
    rec.inv_sigma_f()[i] = s > 0.0 ? (float)(1.0 / s) : 0.0f;
  }
  for (int e = tid; e < d * d; e += nth) rec.V_f()[e] = (float)rec.V()[e];
  for (int e = tid; e < d * d; e += nth) rec.S_f()[e] = e < m * m ? (float)rec.S()[e] : 0.0f;
  if (d == tcc::D) tcc::build_tc(rec, tid, nth);
}

// ---------------------------------------------------------------------------
// Finalize one head per block: d_eff (participation ratio, rounded half to
// even, clamped to [1, d]), kappa, sigma, greedy water-filling, bit offsets,
// QJL matrix, header, derived part.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_finalize(void* __restrict__ recs, int d, FinalizeArgs a,
                                                  int* __restrict__ status) {
  const int h = blockIdx.x, tid = threadIdx.x, nth = blockDim.x;
  Rec rec = rec_at(recs, d, h);
  double* lam = rec.lam();
  __shared__ double red[2][8];
  __shared__ double s_tr, s_s2;
  __shared__ int bits[kMaxD];
  __shared__ double bestv[8];
  __shared__ int besti[8];
  __shared__ int s_m, s_code_bits, s_deff, s_bad;
  double tr = 0.0, s2 = 0.0;
  for (int i = tid; i < d; i += nth) { tr += lam[i]; s2 += lam[i] * lam[i]; }
  tr = warp_sum(tr);
  s2 = warp_sum(s2);
  if ((tid & 31) == 0) { red[0][tid >> 5] = tr; red[1][tid >> 5] = s2; }
  __syncthreads();
  if (tid == 0) {
    double t = 0.0, q = 0.0;
    for (int w = 0; w < nth / 32; ++w) { t += red[0][w]; q += red[1][w]; }
    s_tr = t; s_s2 = q;
    double pr = (q == 0.0) ? (double)d : t * t / q;
    int deff = (int)rint(pr);
    deff = deff < 1 ? 1 : (deff > d ? d : deff);
    if (a.cumvar > 0.0) {
      // smallest k >= 1 whose top-k eigenvalues hold cumvar of the trace
      deff = d;
      if (t > 0.0) {
        double acc = 0.0;
        for (int k = 0; k < d; ++k) {
          acc += lam[k];
          if (acc >= a.cumvar * t) { deff = k + 1; break; }
        }
      }
    }
    s_deff = deff;
    bool use_qjl = a.is_key && a.qjl;
    int m = use_qjl ? (a.d_eff_override > 0 ? a.d_eff_override : deff) : 0;
    int cb = a.total_bits - m;
    s_bad = (m > d) || cb < 0 || cb > a.max_bits * d;
    s_m = s_bad ? 0 : m;
    s_code_bits = s_bad ? 0 : cb;
  }
  __syncthreads();
  const double trace = s_tr;
  double* sigma = rec.sigma();
  for (int i = tid; i < d; i += nth) {
    bits[i] = 0;
    sigma[i] = a.normalize ? (trace > 0.0 ? sqrt(lam[i] / trace) : 0.0) : sqrt(lam[i]);
  }
  __syncthreads();
  // Greedy water-filling: one bit at a time to the largest distortion drop.
  for (int it = 0; it < s_code_bits; ++it) {
    double bv = -1.0;
    int bi = d;
    for (int i = tid; i < d; i += nth) {
      int b = bits[i];
      if (b < a.max_bits) {
        double g = lam[i] * (c_D[b] - c_D[b + 1]);
        if (g > bv || (g == bv && i < bi)) { bv = g; bi = i; }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      double ov = __shfl_xor_sync(0xffffffffu, bv, o);
      int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
    }
    if ((tid & 31) == 0) { bestv[tid >> 5] = bv; besti[tid >> 5] = bi; }
    __syncthreads();
    if (tid == 0) {
      double v = bestv[0];
      int i = besti[0];
      for (int w = 1; w < nth / 32; ++w)
        if (bestv[w] > v || (bestv[w] == v && besti[w] < i)) { v = bestv[w]; i = besti[w]; }
      if (i < d) bits[i] += 1;
    }
    __syncthreads();
  }
  uint8_t* rb = rec.bits();
  for (int i = tid; i < d; i += nth) rb[i] = (uint8_t)bits[i];
  if (tid == 0) {
    int o = 0;
    for (int i = 0; i < d; ++i) { rec.offsets()[i] = o; o += bits[i]; }
  }
  // QJL matrix: Box-Muller pairs from the head's SplitMix64 stream.
  const int m = s_m;
  const uint64_t s0 = mix64(a.seed ^ mix64((uint64_t)h + 1ull));
  double* S = rec.S();
  for (int e = tid; e < d * d; e += nth) if (e >= m * m) S[e] = 0.0;
  // fitted-codebook section: the Gaussian tables in both regimes (the start of
  // the fit, and the tables of widths no coordinate uses) or zeros
  for (int e = tid; e < 2 * kLevelsTotal; e += nth) rec.fit_lv()[e] = a.fitted ? c_lv64[e % kLevelsTotal] : 0.0;
  for (int e = tid; e < 2 * kThreshTotal; e += nth) rec.fit_th()[e] = a.fitted ? c_th64[e % kThreshTotal] : 0.0;
  for (int pidx = tid; 2 * pidx < m * m; pidx += nth) {
    uint64_t r1 = sm64_at(s0, 2ull * pidx), r2 = sm64_at(s0, 2ull * pidx + 1ull);
    double u1 = (double)((r1 >> 11) + 1ull) * 0x1.0p-53;
    double u2 = (double)((r2 >> 11) + 1ull) * 0x1.0p-53;
    double rr = sqrt(-2.0 * log(u1));
    double th = 6.283185307179586477 * u2;
    S[2 * pidx] = rr * cos(th);
    if (2 * pidx + 1 < m * m) S[2 * pidx + 1] = rr * sin(th);
  }
  __syncthreads();
  if (tid == 0) {
    RecHeader* hd = rec.hdr();
    hd->magic = kMagic;
    hd->version = kVersion;
    hd->d = d;
    hd->d_eff = s_deff;
    hd->m = m;
    hd->total_bits = a.total_bits;
    hd->code_bits = s_code_bits;
    hd->words = (a.total_bits + 31) / 32;
    hd->flags = (a.is_key ? kFlagKey : 0u) | (m > 0 ? kFlagQjl : 0u) | (a.normalize ? kFlagNormalize : 0u) |
                (a.rotation ? kFlagRandomRotation : 0u) | (a.cumvar > 0.0 ? kFlagCumvar : 0u) |
                (a.fitted ? kFlagFitted : 0u);
    hd->stream = h;
    hd->max_bits = a.max_bits;
    hd->seed = a.seed;
    hd->trace = trace;
    double kappa = (s_deff >= d || lam[s_deff] == 0.0) ? (double)INFINITY : lam[s_deff - 1] / lam[s_deff];
    hd->kappa = kappa;
    hd->avg_bits = a.avg_bits;
    for (int k = 0; k < 11; ++k) hd->reserved[k] = 0u;
    if (s_bad && status) status[h] = SQ_ERR_ARG;
  }
  __syncthreads();
  build_derived(rec, tid, nth);
  __syncthreads();
  if (tid == 0) rec.hdr()->derived_valid = s_bad ? 0u : 1u;
}

// ---------------------------------------------------------------------------
// Random rotation (the A/B baseline of the README's spectral_rotation.py),
// one head per block, in place of the eigensolver: G = d x d N(0,1) draws
// (row-major, from the stream of seed ^ kRotationSalt and the head's index),
// Q of G = Q R by modified Gram-Schmidt over the columns (R_jj = ||a_j|| > 0),
// the variance q_i^T C q_i of each column, and the columns written to the
// record in descending order of variance (stable), which takes lambda's place.
// The columns are kept contiguous in the workspace (Gt[j * d + i] = G[i][j]).
// ---------------------------------------------------------------------------
constexpr uint64_t kRotationSalt = 0x524F54ull;
__global__ void __launch_bounds__(256) k_random_basis(const double* __restrict__ cov, double* __restrict__ vt_ws,
                                                      int d, uint64_t seed, void* __restrict__ recs,
                                                      int* __restrict__ status) {
  const int h = blockIdx.x, tid = threadIdx.x, nth = blockDim.x, lane = tid & 31, warp = tid >> 5;
  double* Gt = vt_ws + (size_t)h * d * d;
  const double* C = cov + (size_t)h * d * d;
  __shared__ double red[8];
  __shared__ double s_nrm;
  __shared__ double var_s[kMaxD];
  __shared__ int order[kMaxD];
  const uint64_t s0 = mix64((seed ^ kRotationSalt) ^ mix64((uint64_t)h + 1ull));
  for (int pidx = tid; 2 * pidx < d * d; pidx += nth) {
    const uint64_t r1 = sm64_at(s0, 2ull * pidx), r2 = sm64_at(s0, 2ull * pidx + 1ull);
    const double u1 = (double)((r1 >> 11) + 1ull) * 0x1.0p-53;
    const double u2 = (double)((r2 >> 11) + 1ull) * 0x1.0p-53;
    const double rr = sqrt(-2.0 * log(u1));
    const double th = 6.283185307179586477 * u2;
    const int e0 = 2 * pidx, e1 = 2 * pidx + 1;                 // row-major draws G[e / d][e % d]
    Gt[(size_t)(e0 % d) * d + e0 / d] = rr * cos(th);
    if (e1 < d * d) Gt[(size_t)(e1 % d) * d + e1 / d] = rr * sin(th);
  }
  __syncthreads();
  for (int j = 0; j < d; ++j) {
    double* qj = Gt + (size_t)j * d;
    double ss = 0.0;
    for (int i = tid; i < d; i += nth) ss += qj[i] * qj[i];
    ss = warp_sum(ss);
    if (lane == 0) red[warp] = ss;
    __syncthreads();
    if (tid == 0) {
      double t = 0.0;
      for (int w = 0; w < nth / 32; ++w) t += red[w];
      s_nrm = sqrt(t);
    }
    __syncthreads();
    const double inv = s_nrm > 0.0 ? 1.0 / s_nrm : 0.0;
    for (int i = tid; i < d; i += nth) qj[i] *= inv;
    __syncthreads();
    // a_k -= (q_j . a_k) q_j for every later column, one warp per column
    for (int k = j + 1 + warp; k < d; k += nth / 32) {
      double* ak = Gt + (size_t)k * d;
      double dot = 0.0;
      for (int i = lane; i < d; i += 32) dot += qj[i] * ak[i];
      dot = warp_sum(dot);
      for (int i = lane; i < d; i += 32) ak[i] -= dot * qj[i];
    }
    __syncthreads();
  }
  // variance along each column: q^T C q (a warp per column)
  for (int c = warp; c < d; c += nth / 32) {
    const double* qc = Gt + (size_t)c * d;
    double v = 0.0;
    for (int a = 0; a < d; ++a) {
      double t = 0.0;
      for (int b = lane; b < d; b += 32) t += C[(size_t)a * d + b] * qc[b];
      v += qc[a] * warp_sum(t);
    }
    if (lane == 0) var_s[c] = v;
  }
  __syncthreads();
  for (int i = tid; i < d; i += nth) {
    const double li = var_s[i];
    int rank = 0;
    for (int j = 0; j < d; ++j) {
      const double lj = var_s[j];
      rank += (lj > li) || (lj == li && j < i);
    }
    order[rank] = i;
  }
  __syncthreads();
  Rec rec = rec_at(recs, d, h);
  double* lam = rec.lam();
  double* V = rec.V();
  for (int c = tid; c < d; c += nth) lam[c] = fmax(var_s[order[c]], 0.0);
  for (int e = tid; e < d * d; e += nth) {
    const int i = e / d, c = e % d;
    V[e] = Gt[(size_t)order[c] * d + i];
  }
  if (tid == 0) {
    rec.hdr()->sweeps = 0;
    if (status) status[h] = SQ_OK;
  }
}

// ---------------------------------------------------------------------------
// Fitted per-regime codebooks (SpectralQuant README, "Repository Structure":
// nonuniform_quantization.py, Lloyd-Max with per-regime codebooks; the
// conftest fixture gaussian_data_1d: a Lloyd-Max quantizer fitted to samples).
// Regime 0 holds the coordinates i < d_eff, regime 1 the rest; each width a
// regime uses gets a codebook fitted by Lloyd's algorithm to the pooled
// scaled coordinates z of the calibration vectors over the regime's
// coordinates of that width, from the Gaussian Lloyd-Max codebook, for a
// fixed number of iterations: thresholds at the midpoints of neighbouring
// levels, each sample coded as the compressor codes it (the number of
// thresholds strictly below), each level moved to the mean of its samples, a
// level without samples kept.
// ---------------------------------------------------------------------------

constexpr int kFitIters = 30;   // Lloyd iterations of the fit unless the caller sets another count

// z[h][t][i] = (V^T u_t)_i / sigma_i, u = x / ||x|| (normalized records) or x;
// 0 where sigma_i = 0 or ||x|| = 0. Grid (token groups of 8, heads), 256
// threads: warp w takes one token, lane i coordinates i, i + 32, ...
template <typename T>
__global__ void __launch_bounds__(256) k_fit_z(const T* __restrict__ x, int d, int64_t n_tok, int64_t stride_head,
                                               int64_t stride_tok, const void* __restrict__ recs,
                                               double* __restrict__ z) {
  __shared__ double xs[8][kMaxD];
  const int h = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * 8 + warp;
  Rec rec = rec_at(recs, d, h);
  const RecHeader* hd = rec.hdr();
  if (t >= n_tok || !(hd->flags & kFlagFitted) || hd->derived_valid == 0u) return;
  const T* xt = x + (size_t)h * stride_head + (size_t)t * stride_tok;
  double ss = 0.0;
  for (int j = lane; j < d; j += 32) {
    const double v = (double)to_float<T>(xt[j]);
    xs[warp][j] = v;
    ss += v * v;
  }
  ss = warp_sum(ss);
  __syncwarp();
  const bool normalize = (hd->flags & kFlagNormalize) != 0u;
  const double nrm = normalize ? sqrt(ss) : 1.0;
  const double inv = nrm > 0.0 ? 1.0 / nrm : 0.0;
  const double* V = rec.V();
  const double* sig = rec.sigma();
  double* zt = z + ((size_t)h * n_tok + t) * d;
  for (int i = lane; i < d; i += 32) {
    double y = 0.0;
    for (int j = 0; j < d; ++j) y = fma(V[(size_t)j * d + i], xs[warp][j], y);
    y *= inv;
    zt[i] = sig[i] > 0.0 ? y / sig[i] : 0.0;
  }
}

// One codebook per block: grid (heads, 2 regimes, widths 1..SQ_MAX_BITS),
// 256 threads. Widths up to 3 sum in registers (per thread, then per warp);
// wider ones in shared memory.
__global__ void __launch_bounds__(256) k_fit_lloyd(const double* __restrict__ z, int d, int64_t n_tok,
                                                   void* __restrict__ recs, int iters) {
  __shared__ int cols[kMaxD];
  __shared__ int s_nc;
  __shared__ double lvl[256], thr[255], sums[256];
  __shared__ unsigned long long cnts[256];
  const int h = blockIdx.x, r = blockIdx.y, b = blockIdx.z + 1, tid = threadIdx.x, lane = tid & 31;
  Rec rec = rec_at(recs, d, h);
  const RecHeader* hd = rec.hdr();
  if (!(hd->flags & kFlagFitted) || hd->derived_valid == 0u) return;
  const int nl = 1 << b;
  if (tid == 0) {
    int nc = 0;
    for (int i = 0; i < d; ++i)
      if ((int)rec.bits()[i] == b && ((i >= hd->d_eff) ? 1 : 0) == r) cols[nc++] = i;
    s_nc = nc;
  }
  double* lv_out = rec.fit_lv() + r * kLevelsTotal + lv_off(b);
  double* th_out = rec.fit_th() + r * kThreshTotal + th_off(b);
  for (int k = tid; k < nl; k += 256) lvl[k] = lv_out[k];
  __syncthreads();
  const int nc = s_nc;
  if (nc == 0) return;
  // samples (t, c): token t, coordinate cols[c]; thread tid starts at the
  // tid-th and steps by 256 (st_t tokens and st_c columns, with carry)
  const int st_t = 256 / nc, st_c = 256 % nc;
  const double* zh = z + (size_t)h * n_tok * d;
  for (int it = 0; it < iters; ++it) {
    for (int k = tid; k + 1 < nl; k += 256) thr[k] = 0.5 * (lvl[k] + lvl[k + 1]);
    for (int k = tid; k < nl; k += 256) { sums[k] = 0.0; cnts[k] = 0ull; }
    __syncthreads();
    if (b <= 3) {
      double ps[8];
      unsigned pc[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) { ps[k] = 0.0; pc[k] = 0u; }
      for (int64_t t = tid / nc, c = tid % nc; t < n_tok;) {
        const double zv = zh[(size_t)t * d + cols[c]];
        const int code = code_of(zv, thr, b);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if (k == code) { ps[k] += zv; pc[k] += 1u; }
        c += st_c;
        t += st_t;
        if (c >= nc) { c -= nc; ++t; }
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        if (k >= nl) break;
        const double sv = warp_sum(ps[k]);
        unsigned cv = pc[k];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) cv += __shfl_xor_sync(0xffffffffu, cv, o);
        if (lane == 0) {
          atomicAdd(&sums[k], sv);
          atomicAdd(&cnts[k], (unsigned long long)cv);
        }
      }
    } else {
      for (int64_t t = tid / nc, c = tid % nc; t < n_tok;) {
        const double zv = zh[(size_t)t * d + cols[c]];
        const int code = code_of(zv, thr, b);
        atomicAdd(&sums[code], zv);
        atomicAdd(&cnts[code], 1ull);
        c += st_c;
        t += st_t;
        if (c >= nc) { c -= nc; ++t; }
      }
    }
    __syncthreads();
    for (int k = tid; k < nl; k += 256)
      if (cnts[k] > 0ull) lvl[k] = sums[k] / (double)cnts[k];
    __syncthreads();
  }
  for (int k = tid; k < nl; k += 256) lv_out[k] = lvl[k];
  for (int k = tid; k + 1 < nl; k += 256) th_out[k] = 0.5 * (lvl[k] + lvl[k + 1]);
}

// ---------------------------------------------------------------------------
// Import: validate canonical parts written elsewhere and build derived parts.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_import(void* __restrict__ recs, int d, int* __restrict__ status) {
  const int h = blockIdx.x, tid = threadIdx.x, nth = blockDim.x;
  Rec rec = rec_at(recs, d, h);
  RecHeader* hd = rec.hdr();
  __shared__ int s_ok;
  if (tid == 0) {
    bool ok = hd->magic == kMagic && hd->version == kVersion && hd->d == d && hd->m >= 0 && hd->m <= d &&
              hd->total_bits >= 1 && hd->code_bits + hd->m == hd->total_bits &&
              hd->words == (hd->total_bits + 31) / 32 && hd->max_bits >= 1 && hd->max_bits <= SQ_MAX_BITS;
    if (ok) {
      int o = 0;
      for (int i = 0; i < d; ++i) {
        int b = rec.bits()[i];
        if (b > hd->max_bits || rec.offsets()[i] != o) { ok = false; break; }
        o += b;
      }
      ok = ok && (o == hd->code_bits);
    }
    if (ok && (hd->flags & kFlagFitted)) {
      // fitted codebooks: finite, and strictly increasing levels for every
      // width a coordinate of the regime uses
      for (int i = 0; i < d && ok; ++i) {
        const int b = rec.bits()[i];
        if (b == 0) continue;
        const int r = (i >= hd->d_eff) ? 1 : 0;
        const double* l = rec.fit_lv() + r * kLevelsTotal + lv_off(b);
        const double* t = rec.fit_th() + r * kThreshTotal + th_off(b);
        for (int k = 0; k < (1 << b) && ok; ++k) ok = isfinite(l[k]) && (k == 0 || l[k] > l[k - 1]);
        for (int k = 0; k + 1 < (1 << b) && ok; ++k) ok = isfinite(t[k]) && t[k] >= l[k] && t[k] <= l[k + 1];
      }
    }
    s_ok = ok;
    hd->derived_valid = 0u;
  }
  __syncthreads();
  if (s_ok) build_derived(rec, tid, nth);
  __syncthreads();
  if (tid == 0) {
    hd->derived_valid = s_ok ? 1u : 0u;
    if (status) status[h] = s_ok ? SQ_OK : SQ_ERR_RECORD;
  }
}

}  // namespace sq
