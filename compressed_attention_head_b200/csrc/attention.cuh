// Decode attention straight from the packed cache.
//
// SpectralQuant README, "Headline Results" (decode latency per step over the
// compressed cache) and "Key Findings" 3; keys carry the QJL sign correction on
// their signal dims, values do not ("KV spectral asymmetry").
//
// For batch row b, query head h, KV head g = h / G and length L:
//   q' = V_K^T q,  w_i = scale * sigma_i * q'_i,
//   u_j = scale * sqrt(pi/2) / m * (S q'[0:m])_j,
//   s_t = ||k_t|| * (sum_i w_i level_t,i + rho_t * sum_j u_j (2 bit_t,j - 1)),
//   p = softmax(s);  o = V_V (sigma_V * sum_t p_t ||v_t|| level^V_t).
// Three kernels: prepare (q' -> w, u), split-KV partial (online softmax over a
// token range, flash-decoding style), combine (merge the splits, rotate back).
#pragma once

#include "sq_common.cuh"

namespace sq {

constexpr int kAttnTile = 128;     // tokens per tile of the partial kernel
constexpr int kAttnMaxG = 16;      // query heads per KV head

// Shape of one attention call as the kernels see it. Decode: one query per
// (batch row, query head); the kernels' "rows" are batch rows and their
// "columns" the G query heads of a KV head. Prefill (causal): the query tokens
// of a row are cut into blocks of pcols positions, and a kernel row is
// (batch row, block) while its columns are (position in the block, query
// head): group = pcols * qg columns per KV head (at most 16).
struct AttnShape {
  int batch, n_q, n_kv, group, d, splits;   // kernel rows, kernel columns in all, KV heads, columns per KV head
  int64_t max_ctx, chunk;
  int len_offset;     // decode: attended length = seq_lens[b] + len_offset (1 when seq_lens holds the new token's position)
  int causal;         // prefill: seq_lens[b] is the position of row b's first query token
  int pcols;          // prefill: query positions per block (1 for decode)
  int ncb;            // prefill: blocks per batch row (1 for decode)
  int qg;             // query heads per KV head (= group for decode)
  int n_qtok;         // prefill: query tokens per batch row
};

// Cache row of kernel row r (batch row).
__host__ __device__ __forceinline__ int attn_cache_row(const AttnShape& s, int r) { return s.causal ? r / s.ncb : r; }
// Query element (kernel row r, KV head g, column c, coordinate 0) of q:
// decode [batch][n_q][d], prefill [batch][n_kv qg][n_qtok][d].
__host__ __device__ __forceinline__ size_t attn_q_index(const AttnShape& s, int r, int g, int c) {
  if (!s.causal) return ((size_t)r * s.n_q + (size_t)g * s.group + c) * s.d;
  const int b = r / s.ncb, t = (r % s.ncb) * s.pcols + c / s.qg, hh = c % s.qg;
  return (((size_t)b * s.n_kv * s.qg + (size_t)g * s.qg + hh) * s.n_qtok + t) * s.d;
}
// Whether column c of kernel row r is a query at all (the last block of a
// prefill row may be partial).
__host__ __device__ __forceinline__ bool attn_col_live(const AttnShape& s, int r, int c) {
  return !s.causal || ((r % s.ncb) * s.pcols + c / s.qg) < s.n_qtok;
}

// Workspace layout (floats): w[batch][n_q][d], u[batch][n_q][d],
// acc[batch][n_q][splits][d], ml[batch][n_q][splits][2], then one uint32
// arrival counter per (batch, KV head) for the last-block merge.
__host__ __device__ inline size_t attn_ws_floats(int batch, int n_q, int d, int splits) {
  return (size_t)batch * n_q * (2 * (size_t)d + (size_t)splits * (d + 2));
}
__host__ __device__ inline size_t attn_ws_bytes(int batch, int n_q, int n_kv, int d, int splits) {
  return attn_ws_floats(batch, n_q, d, splits) * 4 + (size_t)batch * n_kv * 4;
}
__device__ __forceinline__ uint32_t* attn_counters(float* ws, const AttnShape& s) {
  return (uint32_t*)(ws + attn_ws_floats(s.batch, s.n_q, s.d, s.splits));
}

// Attended length of kernel row r: decode, seq_lens[r] (+ 1 with the new
// token); prefill, the last query position of the row's block + 1.
__device__ __forceinline__ int64_t attn_len(const int32_t* seq_lens, const AttnShape& s, int r) {
  if (!s.causal) return (int64_t)seq_lens[r] + s.len_offset;
  const int b = r / s.ncb, cb = r % s.ncb;
  const int last = min((cb + 1) * s.pcols, s.n_qtok);      // exclusive
  return (int64_t)seq_lens[b] + last;
}
// Causal bound of column c of kernel row r: keys at positions <= this are
// attended (no bound for decode).
__device__ __forceinline__ int64_t attn_col_pos(const int32_t* seq_lens, const AttnShape& s, int r, int c) {
  if (!s.causal) return INT64_MAX;
  const int b = r / s.ncb, cb = r % s.ncb;
  return (int64_t)seq_lens[b] + cb * s.pcols + c / s.qg;
}

// ---------------------------------------------------------------------------
// Prepare: one block rotates the G queries of nb consecutive batch rows
// b0 .. b0 + nb - 1 for one KV head g with the float32 copy of V_K (read once
// for all of them, eight query vectors per pass), w = scale sigma q',
// u = scale sqrt(pi/2) / m S q'[0:m]; it also clears the rows' combine
// counters. smem: floats [nv][d] (queries) + [nv][d] (q'), nv = nb G <= 32.
// ---------------------------------------------------------------------------
constexpr int kPrepVecs = 32;    // query vectors per prepare block
__host__ __device__ inline int prep_rows(int G) { return G >= kPrepVecs ? 1 : kPrepVecs / G; }
__host__ __device__ constexpr size_t prep_smem(int d) { return (size_t)2 * kPrepVecs * d * 4; }

template <typename TQ>
__device__ void prepare_body(const uint8_t* __restrict__ recs_k, const TQ* __restrict__ q, const AttnShape& s,
                             float scale, float* __restrict__ ws, uint32_t* __restrict__ flags, int g, int b0,
                             float* smem, int tid, int nth) {
  const int d = s.d, G = s.group;
  const int nb = min(prep_rows(G), s.batch - b0);
  if (tid < nb) attn_counters(ws, s)[(size_t)(b0 + tid) * s.n_kv + g] = 0u;   // for the last-block merge
  Rec rec = rec_at(recs_k, d, g);
  const RecHeader* hd = rec.hdr();
  if (!record_ok(hd, d)) {
    if (tid == 0 && flags) atomicOr(flags, SQ_FLAG_RECORD);
    return;
  }
  const int nv = nb * G;                 // query vectors: (row r, head hh) -> r * G + hh
  float* qs = smem;                      // [nv][d]
  float* qp = smem + (size_t)kPrepVecs * d;
  for (int e = tid; e < nv * d; e += nth) {
    const int v = e / d, j = e % d;
    const int r = v / G, hh = v % G;
    qs[e] = attn_col_live(s, b0 + r, hh) ? to_float<TQ>(q[attn_q_index(s, b0 + r, g, hh) + j]) : 0.0f;
  }
  __syncthreads();
  const float* V = rec.V_f();
  const float* sig = rec.sigma_f();
  float* w = ws;
  float* u = ws + (size_t)s.batch * s.n_q * d;
  for (int v0 = 0; v0 < nv; v0 += 8) {
    for (int i = tid; i < d; i += nth) {
      float acc[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) acc[k] = 0.0f;
      // the column of V in batches of 32 loads issued together (d is a multiple of 32)
      for (int j0 = 0; j0 < d; j0 += 32) {
        float vv[32];
#pragma unroll
        for (int t = 0; t < 32; ++t) vv[t] = V[(size_t)(j0 + t) * d + i];
#pragma unroll
        for (int t = 0; t < 32; ++t) {
#pragma unroll
          for (int k = 0; k < 8; ++k)
            if (v0 + k < nv) acc[k] = fmaf(vv[t], qs[(size_t)(v0 + k) * d + j0 + t], acc[k]);
        }
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int v = v0 + k;
        if (v < nv) {
          qp[(size_t)v * d + i] = acc[k];
          const int r = v / G, hh = v % G;
          w[((size_t)(b0 + r) * s.n_q + (size_t)g * G + hh) * d + i] = scale * sig[i] * acc[k];
        }
      }
    }
  }
  __syncthreads();
  const int m = hd->m;
  const float* S = rec.S_f();
  const float coef = scale * (float)(kQjlScale / (m > 0 ? m : 1));
  for (int e = tid; e < nv * m; e += nth) {
    const int v = e / m, j = e % m;
    float acc = 0.0f;
    for (int k = 0; k < m; ++k) acc = fmaf(S[j * m + k], qp[(size_t)v * d + k], acc);
    const int r = v / G, hh = v % G;
    u[((size_t)(b0 + r) * s.n_q + (size_t)g * G + hh) * d + j] = coef * acc;
  }
}

// Prepare as a kernel of its own: grid (n_kv, row groups of prep_rows(G)), 256 threads.
template <typename TQ>
__global__ void __launch_bounds__(256) k_attn_prepare(const uint8_t* __restrict__ recs_k, const TQ* __restrict__ q,
                                                      AttnShape s, float scale, float* __restrict__ ws,
                                                      uint32_t* __restrict__ flags) {
  extern __shared__ __align__(16) float pscr[];
  prepare_body<TQ>(recs_k, q, s, scale, ws, flags, blockIdx.x, blockIdx.y * prep_rows(s.group), pscr, threadIdx.x,
                   blockDim.x);
}

// Shared-memory bytes of the partial kernel.
__host__ __device__ inline size_t attn_partial_smem(int d, int G, int wk, int wv) {
  return (size_t)4 * G * d            // w
         + (size_t)4 * G * d          // u (m <= d)
         + (size_t)4 * 4 * kLevelsTotal   // levels of K and V, two regimes each
         + (size_t)4 * 6 * d          // bits / offsets / level bases of K and V
         + (size_t)4 * d              // sigma_V (unused here, reserved)
         + (size_t)4 * kAttnTile * (wk + 1) + (size_t)4 * kAttnTile * (wv + 1)
         + (size_t)4 * 3 * kAttnTile  // k norm, rho, v norm
         + (size_t)4 * G * kAttnTile  // scores / probabilities
         + (size_t)4 * 7 * G + 64;     // running max, sum, rescale; per-warp reductions
}

// ---------------------------------------------------------------------------
// Partial: grid (splits, n_kv, batch), 128 threads. Token tiles of 128: thread
// t scores token t for all G heads; online softmax per head; thread i
// accumulates coordinate i (and i + 128) of sum_t p_t ||v_t|| level^V_t.
// ---------------------------------------------------------------------------
template <int MAXG>
__global__ void __launch_bounds__(128) k_attn_partial(const uint8_t* __restrict__ recs_k,
                                                      const uint8_t* __restrict__ recs_v, CacheArgs kc,
                                                      CacheArgs vc, const int32_t* __restrict__ seq_lens,
                                                      AttnShape s, float* __restrict__ ws,
                                                      float* __restrict__ scores_out,
                                                      uint32_t* __restrict__ flags) {
  extern __shared__ __align__(16) unsigned char sm[];
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int d = s.d, G = s.group;
  Rec rk = rec_at(recs_k, d, g), rv = rec_at(recs_v, d, g);
  const RecHeader* hk = rk.hdr();
  const RecHeader* hv = rv.hdr();
  float* wq = ws;
  float* uq = ws + (size_t)s.batch * s.n_q * d;
  float* acc_out = uq + (size_t)s.batch * s.n_q * d;
  float* ml_out = acc_out + (size_t)s.batch * s.n_q * s.splits * d;
  const bool ok = record_ok(hk, d) && record_ok(hv, d) && hk->words == kc.words && hv->words == vc.words &&
                  (hk->m == 0 || kc.rnorm != nullptr);
  int64_t L = attn_len(seq_lens, s, b);
  if (L < 0 || L > s.max_ctx || L > kc.cap) {
    if (tid == 0 && split == 0 && g == 0 && flags) atomicOr(flags, SQ_FLAG_SEQLEN);
    L = L < 0 ? 0 : (L > s.max_ctx ? s.max_ctx : L);
    L = L > kc.cap ? kc.cap : L;
  }
  if (!ok) {
    if (tid == 0 && flags) atomicOr(flags, SQ_FLAG_RECORD);
    L = 0;
  }
  const int64_t t_lo = (int64_t)split * s.chunk;
  const int64_t t_hi = min(L, t_lo + s.chunk);
  const int m = ok ? hk->m : 0;
  const int wk = kc.words, wv = vc.words, kcb = ok ? hk->code_bits : 0;

  unsigned char* p = sm;
  float* w = (float*)p;        p += (size_t)4 * G * d;
  float* u = (float*)p;        p += (size_t)4 * G * d;
  float* lv = (float*)p;       p += (size_t)4 * 4 * kLevelsTotal;   // K regime 0, 1; V regime 0, 1
  int* kb = (int*)p;           p += (size_t)4 * d;
  int* ko = (int*)p;           p += (size_t)4 * d;
  int* vb = (int*)p;           p += (size_t)4 * d;
  int* vo = (int*)p;           p += (size_t)4 * d;
  int* kl = (int*)p;           p += (size_t)4 * d;   // level-table base of each key coordinate
  int* vl = (int*)p;           p += (size_t)4 * d;
  p += (size_t)4 * d;
  uint32_t* kw = (uint32_t*)p; p += (size_t)4 * kAttnTile * (wk + 1);
  uint32_t* vw = (uint32_t*)p; p += (size_t)4 * kAttnTile * (wv + 1);
  float* kn = (float*)p;       p += (size_t)4 * kAttnTile;
  float* kr = (float*)p;       p += (size_t)4 * kAttnTile;
  float* vn = (float*)p;       p += (size_t)4 * kAttnTile;
  float* sc = (float*)p;       p += (size_t)4 * G * kAttnTile;
  float* mrun = (float*)p;     p += (size_t)4 * G;
  float* lrun = (float*)p;     p += (size_t)4 * G;
  float* alpha = (float*)p;    p += (size_t)4 * G;
  float* red = (float*)p;

  const size_t qbase = ((size_t)b * s.n_q + (size_t)g * G);
  for (int e = tid; e < G * d; e += blockDim.x) w[e] = wq[qbase * d + e];
  for (int e = tid; e < G * m; e += blockDim.x) u[e] = uq[(qbase + e / m) * d + e % m];
  // codebooks: each record's fitted per-regime tables (flag kFlagFitted), else
  // the shared Gaussian Lloyd-Max tables
  for (int e = tid; e < 4 * kLevelsTotal; e += blockDim.x) {
    const Rec& r = e < 2 * kLevelsTotal ? rk : rv;
    const int f = e % (2 * kLevelsTotal);
    lv[e] = (ok && (r.hdr()->flags & kFlagFitted)) ? (float)r.fit_lv()[f] : c_lv32[f % kLevelsTotal];
  }
  if (ok)
    for (int i = tid; i < d; i += blockDim.x) {
      kb[i] = rk.bits()[i]; ko[i] = rk.offsets()[i];
      vb[i] = rv.bits()[i]; vo[i] = rv.offsets()[i];
      const bool kfit = (hk->flags & kFlagFitted) != 0u, vfit = (hv->flags & kFlagFitted) != 0u;
      kl[i] = ((kfit && i >= hk->d_eff) ? kLevelsTotal : 0) + lv_off(kb[i]);
      vl[i] = 2 * kLevelsTotal + ((vfit && i >= hv->d_eff) ? kLevelsTotal : 0) + lv_off(vb[i]);
    }
  for (int hh = tid; hh < G; hh += blockDim.x) { mrun[hh] = -INFINITY; lrun[hh] = 0.0f; }
  float oacc[MAXG][2];
#pragma unroll
  for (int hh = 0; hh < MAXG; ++hh) oacc[hh][0] = oacc[hh][1] = 0.0f;
  __syncthreads();

  const size_t row = (size_t)attn_cache_row(s, b) * s.n_kv + g;
  const uint32_t* kcodes = kc.codes + row * kc.cap * wk;
  const uint32_t* vcodes = vc.codes + row * vc.cap * wv;
  for (int64_t t0 = t_lo; t0 < t_hi; t0 += kAttnTile) {
    const int nt = (int)min((int64_t)kAttnTile, t_hi - t0);
    // word w of token t0 + i (interleaved blocks of 32 tokens; t0 is a multiple of 32)
    for (int e = tid; e < nt * wk; e += blockDim.x) {
      const int w = e / nt, i = e % nt;
      kw[i * (wk + 1) + w] = kcodes[(size_t)((t0 + i) >> 5) * wk * 32 + (size_t)w * 32 + ((t0 + i) & 31)];
    }
    for (int e = tid; e < nt * wv; e += blockDim.x) {
      const int w = e / nt, i = e % nt;
      vw[i * (wv + 1) + w] = vcodes[(size_t)((t0 + i) >> 5) * wv * 32 + (size_t)w * 32 + ((t0 + i) & 31)];
    }
    if (tid < nt) {
      kn[tid] = kc.norm[row * kc.cap + t0 + tid];
      kr[tid] = m > 0 ? kc.rnorm[row * kc.cap + t0 + tid] : 0.0f;
      vn[tid] = vc.norm[row * vc.cap + t0 + tid];
    }
    __syncthreads();
    // Scores: thread tid <-> token t0 + tid.
    {
      float a[MAXG];
#pragma unroll
      for (int hh = 0; hh < MAXG; ++hh) a[hh] = 0.0f;
      if (tid < nt) {
        const uint32_t* rw = kw + tid * (wk + 1);
        for (int i = 0; i < d; ++i) {
          int bw = kb[i];
          if (bw == 0) continue;
          float lvv = lv[kl[i] + (int)field(rw, ko[i], bw)];
#pragma unroll
          for (int hh = 0; hh < MAXG; ++hh)
            if (hh < G) a[hh] = fmaf(w[hh * d + i], lvv, a[hh]);
        }
        if (m > 0) {
          float qa[MAXG];
#pragma unroll
          for (int hh = 0; hh < MAXG; ++hh) qa[hh] = 0.0f;
          for (int j = 0; j < m; ++j) {
            int o = kcb + j;
            float sg = ((rw[o >> 5] >> (o & 31)) & 1u) ? 1.0f : -1.0f;
#pragma unroll
            for (int hh = 0; hh < MAXG; ++hh)
              if (hh < G) qa[hh] = fmaf(u[hh * m + j], sg, qa[hh]);
          }
#pragma unroll
          for (int hh = 0; hh < MAXG; ++hh) a[hh] = fmaf(kr[tid], qa[hh], a[hh]);
        }
      }
      for (int hh = 0; hh < G; ++hh) {
        const bool vis = tid < nt && t0 + tid <= attn_col_pos(seq_lens, s, b, hh);
        float sv = vis ? kn[tid] * a[hh] : -INFINITY;
        sc[hh * kAttnTile + tid] = sv;
        if (scores_out && vis) scores_out[((size_t)b * s.n_q + g * G + hh) * s.max_ctx + t0 + tid] = sv;
      }
    }
    __syncthreads();
    // Online softmax: tile max per head, then probabilities and their sum.
    for (int hh = 0; hh < G; ++hh) {
      float v = warp_max(sc[hh * kAttnTile + tid]);
      if ((tid & 31) == 0) red[hh * 4 + (tid >> 5)] = v;
    }
    __syncthreads();
    for (int hh = tid; hh < G; hh += blockDim.x) {
      float tm = fmaxf(fmaxf(red[hh * 4], red[hh * 4 + 1]), fmaxf(red[hh * 4 + 2], red[hh * 4 + 3]));
      float mn = fmaxf(mrun[hh], tm);
      alpha[hh] = (mrun[hh] == -INFINITY) ? 0.0f : __expf(mrun[hh] - mn);
      mrun[hh] = mn;
    }
    __syncthreads();
    for (int hh = 0; hh < G; ++hh) {
      const float svv = sc[hh * kAttnTile + tid];
      float pv = (tid < nt && svv != -INFINITY) ? __expf(svv - mrun[hh]) : 0.0f;
      float ps = warp_sum(pv);
      sc[hh * kAttnTile + tid] = pv * (tid < nt ? vn[tid] : 0.0f);
      if ((tid & 31) == 0) red[hh * 4 + (tid >> 5)] = ps;
    }
    __syncthreads();
    for (int hh = tid; hh < G; hh += blockDim.x)
      lrun[hh] = lrun[hh] * alpha[hh] + (red[hh * 4] + red[hh * 4 + 1] + red[hh * 4 + 2] + red[hh * 4 + 3]);
    // PV: thread tid <-> coordinates tid and tid + 128.
#pragma unroll
    for (int c2 = 0; c2 < 2; ++c2) {
      int i = tid + c2 * kAttnTile;
      if (i >= d) break;
#pragma unroll
      for (int hh = 0; hh < MAXG; ++hh)
        if (hh < G) oacc[hh][c2] *= alpha[hh];
      int bw = vb[i];
      if (bw == 0) continue;
      int o = vo[i];
      const int lb = vl[i];
      for (int t = 0; t < nt; ++t) {
        float lvv = lv[lb + (int)field(vw + t * (wv + 1), o, bw)];
#pragma unroll
        for (int hh = 0; hh < MAXG; ++hh)
          if (hh < G) oacc[hh][c2] = fmaf(sc[hh * kAttnTile + t], lvv, oacc[hh][c2]);
      }
    }
    __syncthreads();
  }
  // Partial results of this split.
  for (int hh = 0; hh < G; ++hh) {
    size_t base = ((qbase + hh) * s.splits + split);
#pragma unroll
    for (int c2 = 0; c2 < 2; ++c2) {
      int i = tid + c2 * kAttnTile;
      if (i < d) acc_out[base * d + i] = oacc[hh][c2];
    }
    if (tid == 0) {
      ml_out[base * 2] = mrun[hh];
      ml_out[base * 2 + 1] = lrun[hh];
    }
  }
}

// ---------------------------------------------------------------------------
// Combine of one (batch, KV head): merge the splits of its G query heads,
// a_h,i = sigma_V,i * sum_s e^(m_s - M) acc_s,i / sum_s e^(m_s - M) l_s, and
// rotate back, o_h = V_V a_h (combine_one: both in one block, V_V read once
// for the G heads; merge_one + k_rotate_out: the rotation batched over the
// rows of each KV head, V_V read once per 32 column vectors).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void store_out(void* out, int dt, size_t idx, float v) {
  if (dt == SQ_F32) ((float*)out)[idx] = v;
  else if (dt == SQ_F16) ((__half*)out)[idx] = __float2half_rn(v);
  else ((__nv_bfloat16*)out)[idx] = __float2bfloat16_rn(v);
}

// The splits of KV head g in kernel row b merged: for each column hh < G,
// a_h = sigma ⊙ (sum_k w_k acc_k) / l with w_k = exp(m_k - max m), into
// dst[hh * d + i] (zero when the record is invalid). scr: 16 * (splits + 1)
// floats of shared memory; the caller synchronises before reading dst.
__device__ void merge_splits(const Rec& rv, bool ok, const AttnShape& s, const float* ws, int g, int b, float* dst,
                             float* scr, int tid, int nth) {
  const int d = s.d, G = s.group;
  const int lane = tid & 31, warp = tid >> 5, nwarp = nth >> 5;
  float* sw = scr;                      // [16][splits]
  float* s_inv_l = sw + 16 * s.splits;  // [16]
  const float* acc = ws + (size_t)s.batch * s.n_q * d * 2;
  const float* ml = acc + (size_t)s.batch * s.n_q * s.splits * d;
  const size_t qh0 = (size_t)b * s.n_q + (size_t)g * G;
  const float* sig = rv.sigma_f();
  for (int hh = warp; hh < G; hh += nwarp) {
    const float* mlh = ml + (qh0 + hh) * s.splits * 2;
    float M = -INFINITY;
    // partials of other blocks of the same launch may be read here: L2 loads (__ldcg)
    for (int k = lane; k < s.splits; k += 32) M = fmaxf(M, __ldcg(mlh + 2 * k));
    M = warp_max(M);
    float l = 0.0f;
    for (int k = lane; k < s.splits; k += 32) {
      const float mk = __ldcg(mlh + 2 * k);
      const float wk = (mk == -INFINITY) ? 0.0f : __expf(mk - M);
      sw[hh * s.splits + k] = wk;
      l += wk * __ldcg(mlh + 2 * k + 1);
    }
    l = warp_sum(l);
    if (lane == 0) s_inv_l[hh] = l > 0.0f ? 1.0f / l : 0.0f;
  }
  __syncthreads();
  for (int e = tid; e < G * d; e += nth) {
    const int hh = e / d, i = e % d;
    const float* ah = acc + (qh0 + hh) * s.splits * (size_t)d + i;
    const float* swh = sw + hh * s.splits;
    float v = 0.0f;
    int k = 0;
    for (; k + 4 <= s.splits; k += 4) {     // four loads in flight
      const float a0 = __ldcg(ah + (size_t)k * d), a1 = __ldcg(ah + (size_t)(k + 1) * d);
      const float a2 = __ldcg(ah + (size_t)(k + 2) * d), a3 = __ldcg(ah + (size_t)(k + 3) * d);
      v = fmaf(swh[k], a0, v);
      v = fmaf(swh[k + 1], a1, v);
      v = fmaf(swh[k + 2], a2, v);
      v = fmaf(swh[k + 3], a3, v);
    }
    for (; k < s.splits; ++k) v = fmaf(swh[k], __ldcg(ah + (size_t)k * d), v);
    dst[hh * d + i] = ok ? v * s_inv_l[hh] * sig[i] : 0.0f;
  }
}

// The merged column vectors of (b, g) over their query operands w[b][h] in
// the workspace (every block of (b, g) has read them by now): the rotation
// back, o = V_V a, runs for all rows of a KV head at once in k_rotate_out.
__device__ void merge_one(const uint8_t* __restrict__ recs_v, const AttnShape& s, float* ws, int g, int b,
                          float* scr, int tid, int nth) {
  const Rec rv = rec_at(recs_v, s.d, g);
  const bool ok = record_ok(rv.hdr(), s.d);
  merge_splits(rv, ok, s, ws, g, b, ws + ((size_t)b * s.n_q + (size_t)g * s.group) * s.d, scr, tid, nth);
}

// Merge and rotate back in one block per (b, g). scr: [16][d] floats (a),
// [16][splits] (split weights), [16] (1 / l).
__device__ void combine_one(const uint8_t* __restrict__ recs_v, const AttnShape& s, const float* ws, void* out,
                            int out_dt, int g, int b, float* scr, int tid, int nth) {
  const int d = s.d, G = s.group;
  const int lane = tid & 31, warp = tid >> 5, nwarp = nth >> 5;
  const Rec rv = rec_at(recs_v, d, g);
  const bool ok = record_ok(rv.hdr(), d);
  float* a = scr;                       // [16][d]
  merge_splits(rv, ok, s, ws, g, b, a, scr + 16 * d, tid, nth);
  __syncthreads();
  // o_h = V_V a_h: warp w takes rows w, w + nwarp, ... in batches of RB rows
  // whose loads (16-byte pieces, lane-strided) are all in flight together
  const float4* V4 = (const float4*)rv.V_f();
  const int q4 = d / 4;
  constexpr int RB = 8;
  for (int j0 = warp; j0 < d; j0 += nwarp * RB) {
    float4 vv[RB][2];
#pragma unroll
    for (int r = 0; r < RB; ++r) {
      const int j = j0 + nwarp * r;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int col = lane + 32 * c;
        vv[r][c] = (ok && j < d && col < q4) ? __ldg(V4 + (size_t)j * q4 + col) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    for (int hh = 0; hh < G; ++hh) {
      float4 av[2];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int col = lane + 32 * c;
        av[c] = col < q4 ? *(const float4*)&a[hh * d + 4 * col] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int r = 0; r < RB; ++r) {
        const int j = j0 + nwarp * r;
        float o = 0.0f;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          o = fmaf(vv[r][c].x, av[c].x, o);
          o = fmaf(vv[r][c].y, av[c].y, o);
          o = fmaf(vv[r][c].z, av[c].z, o);
          o = fmaf(vv[r][c].w, av[c].w, o);
        }
        o = warp_sum(o);
        if (lane == 0 && j < d && attn_col_live(s, b, hh)) store_out(out, out_dt, attn_q_index(s, b, g, hh) + j, o);
      }
    }
  }
}

// Combine as a kernel of its own (for the partial kernels that do not merge
// their splits themselves): grid (n_kv, batch), 256 threads.
__global__ void __launch_bounds__(256, 2) k_attn_combine(const uint8_t* __restrict__ recs_v, AttnShape s,
                                                      const float* __restrict__ ws, void* out, int out_dt) {
  extern __shared__ __align__(16) float cscr[];
  combine_one(recs_v, s, ws, out, out_dt, blockIdx.x, blockIdx.y, cscr, threadIdx.x, blockDim.x);
}

// The rotation back for the kernels that leave merged column vectors in the
// workspace (merge_one): o = V_V a for every column vector of KV head g, as a
// small product per block, O[32 vectors x D] = A V_V^T, so that V_V is read once
// per 32 vectors instead of once per (row, KV head). grid (n_kv, tiles of 32 of
// the rows x columns vectors, striding when there are more than gridDim.y
// tiles), 256 threads; each thread 4 vectors x D/32 outputs, float32.
template <int D>
__global__ void __launch_bounds__(256) k_rotate_out(const uint8_t* __restrict__ recs_v, AttnShape s,
                                                   const float* __restrict__ ws, void* out, int out_dt) {
  constexpr int RT = 32, KC = 32, OJ = D / 32;
  __shared__ float As[KC][RT + 1];   // chunk of the vectors, coordinate-major
  __shared__ float Vs[KC][D + 1];    // chunk of V_V^T: Vs[i][j] = V_V[j][i0 + i]
  const int g = blockIdx.x, tid = threadIdx.x, tx = tid & 31, ty = tid >> 5;
  const Rec rv = rec_at(recs_v, D, g);
  const bool ok = record_ok(rv.hdr(), D);
  const float* V = rv.V_f();
  const int nvec = s.batch * s.group;
  for (int v0 = blockIdx.y * RT; v0 < nvec; v0 += gridDim.y * RT) {
    float acc[4][OJ];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int u = 0; u < OJ; ++u) acc[a][u] = 0.0f;
    if (ok) {
      for (int i0 = 0; i0 < D; i0 += KC) {
        // vectors: element (v, i0 + ii) of vector v0 + v (rows b, columns hh of head g)
        for (int e = tid; e < RT * KC; e += 256) {
          const int v = e / KC, ii = e % KC, vg = v0 + v;
          float x = 0.0f;
          if (vg < nvec) {
            const int b = vg / s.group, hh = vg % s.group;
            x = ws[((size_t)b * s.n_q + (size_t)g * s.group + hh) * D + i0 + ii];
          }
          As[ii][v] = x;
        }
        for (int e = tid; e < D * KC; e += 256) {
          const int j = e / KC, ii = e % KC;
          Vs[ii][j] = __ldg(V + (size_t)j * D + i0 + ii);
        }
        __syncthreads();
#pragma unroll 8
        for (int ii = 0; ii < KC; ++ii) {
          float av[4];
#pragma unroll
          for (int a = 0; a < 4; ++a) av[a] = As[ii][ty * 4 + a];
#pragma unroll
          for (int u = 0; u < OJ; ++u) {
            const float vv = Vs[ii][tx + 32 * u];
#pragma unroll
            for (int a = 0; a < 4; ++a) acc[a][u] = fmaf(vv, av[a], acc[a][u]);
          }
        }
        __syncthreads();
      }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int vg = v0 + ty * 4 + a;
      if (vg >= nvec) continue;
      const int b = vg / s.group, hh = vg % s.group;
      if (!attn_col_live(s, b, hh)) continue;
      const size_t base = attn_q_index(s, b, g, hh);
#pragma unroll
      for (int u = 0; u < OJ; ++u) store_out(out, out_dt, base + tx + 32 * u, acc[a][u]);
    }
  }
}

// Shared-memory floats combine_one needs.
__host__ __device__ inline size_t combine_scratch_floats(int d, int splits) {
  return (size_t)16 * d + (size_t)16 * splits + 16;
}

}  // namespace sq
