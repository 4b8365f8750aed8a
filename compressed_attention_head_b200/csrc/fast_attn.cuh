// Decode attention partials with tensor-core contractions (sm_100a).
//
// Same computation as k_attn_partial (SpectralQuant README, "Headline Results":
// decode attention over the compressed cache), reorganised so that the two
// contractions run on the tensor pipe and each code is decoded once per block
// for all G query heads of its KV head:
//
//  * A block (4 warps) owns one (batch, KV head, context split) and walks its
//    tokens in tiles of 64. The K and V records of a tile are staged in shared
//    memory transposed (word-major, token-minor), so that every warp decodes
//    the same coordinates for 32 different tokens: bit offsets, widths and
//    lookup-table bases are warp-uniform.
//  * Codes are decoded in pairs of equal width through lane-replicated
//    pair tables (one 32-bit load returns the two fp16 levels) into fp16 tiles
//    K^[64 x d] and V^[64 x d] (16-byte chunks XOR-swizzled by row), plus a
//    64 x 16 tile carrying rho_t * (2 bit_j - 1) for the QJL term (m <= 16).
//  * Scores S^T = W^T K^T with mma.sync m16n8k16 (rows = up to 8 query heads,
//    columns = tokens; W = scale * sigma * q' and the QJL query weights), times
//    ||k_t||; online softmax per warp; then O^T += V^T P^T with the same MMA
//    (rows = coordinates, columns = heads, k = tokens), where P = p * ||v_t||
//    comes straight from the score accumulators.
//  * The four warps' partial (max, sum, acc) are merged at the end and written
//    in the layout k_attn_combine reads.
#pragma once

#include "attention.cuh"
#include "sq_common.cuh"

namespace sq {
namespace fa {

constexpr int TOK = 64;          // tokens per tile
constexpr int NTH = 128;         // threads per block
constexpr int QJL_COLS = 16;     // key columns of the QJL term (m <= 16)
constexpr int MAXW = 32;         // record words handled (B <= 1024 bits)

template <int D>
struct Geo {
  static constexpr int KROW = D * 2;                  // bytes per key / value row
  static constexpr int VROW = D * 2;
  static constexpr int QROW = QJL_COLS * 2;           // bytes per QJL row (unswizzled)
  static constexpr int KSTEPS = D / 16;               // k-steps of the key tile (+1 for QJL)
  static constexpr int MBLK = D / 16;                 // m16 blocks of coordinates in PV
  static constexpr bool SPLITW = D <= 128;            // query weights as fp16 hi + lo
};
constexpr int LOCOLS = 64;       // key coordinates whose wide (>= 4-bit) levels get an fp16 lo part
constexpr int LOROW = LOCOLS * 2;

// Shared-memory plan (bytes): pair LUTs 10.5 KB, single-level table, per-pair
// parameters for K and V, transposed record tiles, fp16 tiles, norms, merge.
struct Smem {
  static constexpr int LUT1 = 0;                   // [4][32] u32
  static constexpr int LUT2 = LUT1 + 4 * 32 * 4;   // [16][32] u32
  static constexpr int LUT3 = LUT2 + 16 * 32 * 4;  // [64][32] u32
  static constexpr int LV16 = LUT3 + 64 * 32 * 4;  // [kLevelsTotal] half
  static constexpr int LVLO = LV16 + kLevelsTotal * 2;   // [kLevelsTotal] half: level - fp16(level)
  static constexpr int PAR = (LVLO + kLevelsTotal * 2 + 15) & ~15;   // uint2 [2][kMaxD/2]
  static constexpr int REC = PAR + 2 * (kMaxD / 2) * 8;              // u32 [2 bufs][2 sides][MAXW][TOK + 1]
  static constexpr int REC_PITCH = TOK + 1;
  static constexpr int REC_SIDE = MAXW * REC_PITCH;                   // words per side
  static constexpr int NRM = REC + 4 * REC_SIDE * 4;                  // float [2 bufs][3][TOK]
  static constexpr int KT = (NRM + 2 * 3 * TOK * 4 + 127) & ~127;
};

// Tiles (key, value, QJL), then norms; the four warps' merge buffer
// [4][8][D + 2] floats reuses the tiles after the last tile.
template <int D>
__host__ __device__ constexpr int tiles_bytes() {
  return TOK * Geo<D>::KROW + TOK * Geo<D>::VROW + TOK * Geo<D>::QROW + TOK * LOROW;
}
template <int D>
__host__ __device__ constexpr int smem_bytes() {
  return Smem::KT + (tiles_bytes<D>() > 4 * 8 * (D + 2) * 4 ? tiles_bytes<D>() : 4 * 8 * (D + 2) * 4) + 128;
}

__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Byte offset of (row, column) in a tile whose rows are `rowbytes` long and
// whose 16-byte chunks are XOR-swizzled by (row & 7).
__device__ __forceinline__ uint32_t swz(int row, int col, int rowbytes) {
  int c = (col >> 3) ^ (row & 7);
  return (uint32_t)(row * rowbytes + (c << 4) + ((col & 7) << 1));
}

__device__ __forceinline__ void mma16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// Per-pair decode parameters (coordinates 2p, 2p+1 of one record):
//   x = word index | shift << 8 | mode << 16 | straddle << 24
//   y = mask of the pair field (mode 0) or of the first code (mode 1) | second width << 16
// mode 0: equal widths <= 3, one pair-table lookup at LUT(b); mode 1: two
// single-level lookups (unequal widths or widths >= 4); mode 2: both uncoded.
__device__ void build_pair_params(const uint8_t* bits, const int32_t* offs, int d, uint2* par, int tid,
                                  int nth) {
  for (int p = tid; p < d / 2; p += nth) {
    int i = 2 * p;
    int b0 = bits[i], b1 = bits[i + 1];
    int o = offs[i];
    uint32_t mode = (b0 == 0 && b1 == 0) ? 2u : ((b0 == b1 && b0 <= 3) ? 0u : 1u);
    int wb = b0 + b1;
    uint32_t straddle = ((o & 31) + wb > 32) ? 1u : 0u;
    par[p].x = (uint32_t)(o >> 5) | ((uint32_t)(o & 31) << 8) | (mode << 16) | (straddle << 24);
    uint32_t m0 = mode == 0 ? ((1u << wb) - 1u) : ((1u << b0) - 1u);
    par[p].y = m0 | ((uint32_t)b0 << 16) | ((uint32_t)b1 << 24);
  }
}

// Decodes coordinates [c0, c0 + n) (n a multiple of 8) of token t into the fp16
// tile row t, reading the transposed records rec[word * REC_PITCH + t].
template <int ROWBYTES, bool LO>
__device__ __forceinline__ void decode_row(const uint32_t* rec, const uint2* par, const uint8_t* sm, int t, int c0,
                                           int n, uint8_t* tile, uint8_t* lotile, int lane) {
  const uint32_t* lut1 = (const uint32_t*)(sm + Smem::LUT1) + lane;
  const uint32_t* lut2 = (const uint32_t*)(sm + Smem::LUT2) + lane;
  const uint32_t* lut3 = (const uint32_t*)(sm + Smem::LUT3) + lane;
  const __half* lv16 = (const __half*)(sm + Smem::LV16);
  const __half* lvlo = (const __half*)(sm + Smem::LVLO);
  for (int c = c0; c < c0 + n; c += 8) {
    uint32_t h[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint2 pp = par[(c >> 1) + k];
      const uint32_t mode = (pp.x >> 16) & 0xFFu;
      uint32_t out = 0u;
      if (mode != 2u) {
        const int wi = (int)(pp.x & 0xFFu), sh = (int)((pp.x >> 8) & 0xFFu);
        uint32_t lo = rec[wi * Smem::REC_PITCH + t];
        uint32_t hi = (pp.x >> 24) ? rec[(wi + 1) * Smem::REC_PITCH + t] : 0u;
        uint32_t f = __funnelshift_r(lo, hi, sh);
        if (mode == 0u) {
          const int b = (int)((pp.y >> 16) & 0xFFu);
          f &= pp.y & 0xFFFFu;
          out = b == 1 ? lut1[f * 32] : (b == 2 ? lut2[f * 32] : lut3[f * 32]);
        } else {
          const int b0 = (int)((pp.y >> 16) & 0xFFu), b1 = (int)(pp.y >> 24);
          const uint32_t c0v = f & (pp.y & 0xFFFFu);
          const uint32_t c1v = (f >> b0) & ((1u << b1) - 1u);
          __half l0 = b0 ? lv16[lv_off(b0) + c0v] : __float2half(0.0f);
          __half l1 = b1 ? lv16[lv_off(b1) + c1v] : __float2half(0.0f);
          __half2 hh = __halves2half2(l0, l1);
          out = *reinterpret_cast<uint32_t*>(&hh);
          if (LO && c + 2 * k < LOCOLS) {
            __half m0 = b0 ? lvlo[lv_off(b0) + c0v] : __float2half(0.0f);
            __half m1 = b1 ? lvlo[lv_off(b1) + c1v] : __float2half(0.0f);
            __half2 mm = __halves2half2(m0, m1);
            *(uint32_t*)(lotile + swz(t, c + 2 * k, LOROW)) = *reinterpret_cast<uint32_t*>(&mm);
          }
        }
      }
      h[k] = out;
    }
    *(uint4*)(tile + swz(t, c, ROWBYTES)) = make_uint4(h[0], h[1], h[2], h[3]);
  }
}

template <int D>
__global__ void __launch_bounds__(NTH) k_attn_partial_tc(const uint8_t* __restrict__ recs_k,
                                                         const uint8_t* __restrict__ recs_v, CacheArgs kc,
                                                         CacheArgs vc, const int32_t* __restrict__ seq_lens,
                                                         AttnShape s, float* __restrict__ ws,
                                                         float* __restrict__ scores_out,
                                                         uint32_t* __restrict__ flags) {
  using G_ = Geo<D>;
  extern __shared__ __align__(128) uint8_t sm[];
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int G = s.group;
  Rec rk = rec_at(recs_k, D, g), rv = rec_at(recs_v, D, g);
  const RecHeader* hk = rk.hdr();
  const RecHeader* hv = rv.hdr();
  float* wq = ws;
  float* uq = ws + (size_t)s.batch * s.n_q * D;
  float* acc_out = uq + (size_t)s.batch * s.n_q * D;
  float* ml_out = acc_out + (size_t)s.batch * s.n_q * s.splits * D;
  const bool ok = record_ok(hk, D) && record_ok(hv, D) && hk->words == kc.words && hv->words == vc.words &&
                  (hk->m == 0 || kc.rnorm != nullptr) && hk->m <= QJL_COLS && kc.words <= MAXW &&
                  vc.words <= MAXW;
  int64_t L = seq_lens[b];
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

  uint2* park = (uint2*)(sm + Smem::PAR);
  uint2* parv = park + kMaxD / 2;
  uint32_t* recbase = (uint32_t*)(sm + Smem::REC);
  float* nrmbase = (float*)(sm + Smem::NRM);
  uint8_t* ktile = sm + Smem::KT;
  uint8_t* vtile = ktile + TOK * G_::KROW;
  uint8_t* qtile = vtile + TOK * G_::VROW;
  uint8_t* lotile = qtile + TOK * G_::QROW;
  float* mrg = (float*)ktile;            // [4 warps][8 heads][D + 2], after the last tile

  // Tables: lane-replicated pair LUTs for widths 1..3 and the fp16 levels.
  for (int e = tid; e < 4 * 32; e += NTH) {
    int f = e >> 5;
    ((uint32_t*)(sm + Smem::LUT1))[e] = pack_h2(c_lv32[lv_off(1) + (f & 1)], c_lv32[lv_off(1) + (f >> 1)]);
  }
  for (int e = tid; e < 16 * 32; e += NTH) {
    int f = e >> 5;
    ((uint32_t*)(sm + Smem::LUT2))[e] = pack_h2(c_lv32[lv_off(2) + (f & 3)], c_lv32[lv_off(2) + (f >> 2)]);
  }
  for (int e = tid; e < 64 * 32; e += NTH) {
    int f = e >> 5;
    ((uint32_t*)(sm + Smem::LUT3))[e] = pack_h2(c_lv32[lv_off(3) + (f & 7)], c_lv32[lv_off(3) + (f >> 3)]);
  }
  for (int e = tid; e < kLevelsTotal; e += NTH) {
    const __half hv = __float2half(c_lv32[e]);
    ((__half*)(sm + Smem::LV16))[e] = hv;
    ((__half*)(sm + Smem::LVLO))[e] = __float2half(c_lv32[e] - __half2float(hv));
  }
  // Wide key codes among the first LOCOLS coordinates get an fp16 lo part.
  bool has_lo = false;
  if (ok)
    for (int i = 0; i < LOCOLS && i < D; ++i) has_lo |= rk.bits()[i] >= 4;
  for (int e = tid; e < TOK * LOCOLS / 2; e += NTH) ((uint32_t*)lotile)[e] = 0u;
  if (ok) {
    build_pair_params(rk.bits(), rk.offsets(), D, park, tid, NTH);
    build_pair_params(rv.bits(), rv.offsets(), D, parv, tid, NTH);
  }
  // The QJL tile stays zero when the keys carry no QJL bits.
  for (int e = tid; e < TOK * QJL_COLS / 2; e += NTH) ((uint32_t*)qtile)[e] = 0u;

  // Query fragments (A operand, rows = heads 0..7, rows 8..15 zero): fp16 of
  // the query weights, scaled by 2^e so that max |w| is near 1.
  const size_t qbase = (size_t)b * s.n_q + (size_t)g * G;
  float wmax = 0.0f;
  for (int e = lane; e < G * D; e += 32) wmax = fmaxf(wmax, fabsf(wq[(qbase + e / D) * D + e % D]));
  for (int e = lane; e < G * m; e += 32) wmax = fmaxf(wmax, fabsf(uq[(qbase + e / m) * D + e % m]));
  wmax = warp_max(wmax);
  const float wsc = wmax > 0.0f ? exp2f(-ceilf(log2f(wmax))) : 1.0f;
  const int qg = lane >> 2, qq = lane & 3;
  uint32_t afrag[G_::KSTEPS + 1][2];
  uint32_t afrag_lo[G_::SPLITW ? G_::KSTEPS : 1][2];
#pragma unroll
  for (int ks = 0; ks <= G_::KSTEPS; ++ks) {
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int col = ks * 16 + half * 8 + 2 * qq;
      float v0 = 0.0f, v1 = 0.0f;
      if (qg < G) {
        const float* wrow = wq + (qbase + qg) * D;
        const float* urow = uq + (qbase + qg) * D;
        v0 = col < D ? wrow[col] : ((col - D) < m ? urow[col - D] : 0.0f);
        v1 = col + 1 < D ? wrow[col + 1] : ((col + 1 - D) < m ? urow[col + 1 - D] : 0.0f);
      }
      const __half2 hv = __floats2half2_rn(v0 * wsc, v1 * wsc);
      afrag[ks][half] = *reinterpret_cast<const uint32_t*>(&hv);
      if (G_::SPLITW && ks < G_::KSTEPS) {
        const float2 back = __half22float2(hv);
        afrag_lo[G_::SPLITW ? ks : 0][half] = pack_h2(v0 * wsc - back.x, v1 * wsc - back.y);
      }
    }
  }
  const float inv_wsc = 1.0f / wsc;

  // Online-softmax state of this warp: head qg in lanes 4qg..4qg+3.
  float m_run = -INFINITY, l_part = 0.0f;
  float oacc[G_::MBLK][4];
#pragma unroll
  for (int mb = 0; mb < G_::MBLK; ++mb) oacc[mb][0] = oacc[mb][1] = oacc[mb][2] = oacc[mb][3] = 0.0f;
  __syncthreads();

  const size_t row = (size_t)b * s.n_kv + g;
  const uint32_t* kcodes = kc.codes + row * kc.cap * wk;
  const uint32_t* vcodes = vc.codes + row * vc.cap * wv;
  // Stage one tile's records (transposed: rec[word][token]) and norms with
  // 4-byte cp.async; tokens past the range read as zeros.
  auto stage = [&](int64_t t0s, int bi) {
    const int nts = (int)min((int64_t)TOK, t_hi - t0s);
    uint32_t* rk_ = recbase + bi * 2 * Smem::REC_SIDE;
    uint32_t* rv_ = rk_ + Smem::REC_SIDE;
    float* nb = nrmbase + bi * 3 * TOK;
    const int tok = tid & (TOK - 1);
    for (int w = tid >> 6; w < wk; w += NTH / TOK) {
      uint32_t* dst = rk_ + w * Smem::REC_PITCH + tok;
      if (tok < nts) cp_async4(dst, kcodes + (t0s + tok) * wk + w); else *dst = 0u;
    }
    for (int w = tid >> 6; w < wv; w += NTH / TOK) {
      uint32_t* dst = rv_ + w * Smem::REC_PITCH + tok;
      if (tok < nts) cp_async4(dst, vcodes + (t0s + tok) * wv + w); else *dst = 0u;
    }
    if (tid < TOK) {
      if (tid < nts) {
        cp_async4(nb + tid, kc.norm + row * kc.cap + t0s + tid);
        cp_async4(nb + 2 * TOK + tid, vc.norm + row * vc.cap + t0s + tid);
        if (m > 0) cp_async4(nb + TOK + tid, kc.rnorm + row * kc.cap + t0s + tid); else nb[TOK + tid] = 0.0f;
      } else {
        nb[tid] = 0.0f; nb[TOK + tid] = 0.0f; nb[2 * TOK + tid] = 0.0f;
      }
    }
    cp_async_commit();
  };
  if (t_lo < t_hi) stage(t_lo, 0);
  int bi = 0;
  for (int64_t t0 = t_lo; t0 < t_hi; t0 += TOK, bi ^= 1) {
    const int nt = (int)min((int64_t)TOK, t_hi - t0);
    if (t0 + TOK < t_hi) {
      stage(t0 + TOK, bi ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const uint32_t* reck = recbase + bi * 2 * Smem::REC_SIDE;
    const uint32_t* recv = reck + Smem::REC_SIDE;
    const float* kn = nrmbase + bi * 3 * TOK;
    const float* kr = kn + TOK;
    const float* vn = kr + TOK;
    // Decode: warp w -> tokens 32 (w & 1) + lane, coordinate half (w >> 1).
    {
      const int t = ((warp & 1) << 5) + lane;
      const int c0 = (warp >> 1) * (D / 2);
      decode_row<G_::KROW, true>(reck, park, sm, t, c0, D / 2, ktile, lotile, lane);
      decode_row<G_::VROW, false>(recv, parv, sm, t, c0, D / 2, vtile, nullptr, lane);
      if ((warp >> 1) == 0 && m > 0) {
        const float rho = kr[t];
        uint32_t hq[8];
#pragma unroll
        for (int j2 = 0; j2 < 8; ++j2) {
          float a0 = 0.0f, a1 = 0.0f;
          const int j = 2 * j2;
          if (j < m) { int o = kcb + j; a0 = ((reck[(o >> 5) * Smem::REC_PITCH + t] >> (o & 31)) & 1u) ? rho : -rho; }
          if (j + 1 < m) { int o = kcb + j + 1; a1 = ((reck[(o >> 5) * Smem::REC_PITCH + t] >> (o & 31)) & 1u) ? rho : -rho; }
          hq[j2] = pack_h2(a0, a1);
        }
        *(uint4*)(qtile + t * G_::QROW) = make_uint4(hq[0], hq[1], hq[2], hq[3]);
        *(uint4*)(qtile + t * G_::QROW + 16) = make_uint4(hq[4], hq[5], hq[6], hq[7]);
      }
    }
    __syncthreads();
    // Scores for this warp's 16 tokens: S^T[head][token].
    const int tb = warp * 16;
    float sc[2][4];
#pragma unroll
    for (int j = 0; j < 2; ++j) sc[j][0] = sc[j][1] = sc[j][2] = sc[j][3] = 0.0f;
    {
      // ldmatrix.x4 over 8 token rows: matrices = k-chunks of 8 (two k-steps).
      const int r = tb + (lane & 7);
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int rr = r + 8 * j;
#pragma unroll
        for (int ks = 0; ks < G_::KSTEPS; ks += 2) {
          const int col = ks * 16 + (lane >> 3) * 8;
          uint32_t b0, b1, b2, b3;
          ldsm_x4(smem_addr(ktile + swz(rr, col, G_::KROW)), b0, b1, b2, b3);
          uint32_t a[4] = {afrag[ks][0], 0u, afrag[ks][1], 0u};
          mma16816(sc[j], a, b0, b1);
          uint32_t a2[4] = {afrag[ks + 1][0], 0u, afrag[ks + 1][1], 0u};
          mma16816(sc[j], a2, b2, b3);
          if (G_::SPLITW) {
            uint32_t al[4] = {afrag_lo[G_::SPLITW ? ks : 0][0], 0u, afrag_lo[G_::SPLITW ? ks : 0][1], 0u};
            mma16816(sc[j], al, b0, b1);
            uint32_t al2[4] = {afrag_lo[G_::SPLITW ? ks + 1 : 0][0], 0u, afrag_lo[G_::SPLITW ? ks + 1 : 0][1], 0u};
            mma16816(sc[j], al2, b2, b3);
          }
          if (has_lo && ks < LOCOLS / 16) {
            uint32_t l0, l1, l2, l3;
            ldsm_x4(smem_addr(lotile + swz(rr, col, LOROW)), l0, l1, l2, l3);
            mma16816(sc[j], a, l0, l1);
            mma16816(sc[j], a2, l2, l3);
          }
        }
        if (m > 0) {       // QJL k-step: matrices (k 0-7, k 8-15) of the QJL tile, twice
          uint32_t b0, b1, b2, b3;
          ldsm_x4(smem_addr(qtile + rr * G_::QROW + ((lane >> 3) & 1) * 16), b0, b1, b2, b3);
          uint32_t a[4] = {afrag[G_::KSTEPS][0], 0u, afrag[G_::KSTEPS][1], 0u};
          mma16816(sc[j], a, b0, b1);
        }
      }
    }
    // sc[j][0..1]: head qg, tokens tb + 8j + 2qq, +1 (sc[j][2..3] are padding rows).
    float sv[4];
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int tl = tb + 8 * j + 2 * qq + e;
        const bool valid = tl < nt && qg < G;
        sv[2 * j + e] = valid ? sc[j][e] * inv_wsc * kn[tl] : -INFINITY;
        if (scores_out && valid) scores_out[((size_t)qbase + qg) * s.max_ctx + t0 + tl] = sv[2 * j + e];
      }
    float tmax = fmaxf(fmaxf(sv[0], sv[1]), fmaxf(sv[2], sv[3]));
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
    const float m_new = fmaxf(m_run, tmax);
    const float alpha = (m_run == -INFINITY) ? 0.0f : __expf(m_run - m_new);
    float p[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) p[e] = (m_new == -INFINITY) ? 0.0f : __expf(sv[e] - m_new);
    l_part = l_part * alpha + (p[0] + p[1] + p[2] + p[3]);
    m_run = m_new;
    // P * ||v_t|| as the B operand (k = tokens, n = heads): b0 tokens 2qq,2qq+1, b1 tokens 8+2qq,+1.
    const uint32_t pb0 = pack_h2(p[0] * vn[tb + 2 * qq], p[1] * vn[tb + 2 * qq + 1]);
    const uint32_t pb1 = pack_h2(p[2] * vn[tb + 8 + 2 * qq], p[3] * vn[tb + 8 + 2 * qq + 1]);
    // Rescale the accumulators: columns are heads 2qq, 2qq+1 -> alpha from lanes 8qq and 8qq+4.
    const float al0 = __shfl_sync(0xffffffffu, alpha, (8 * qq) & 31);
    const float al1 = __shfl_sync(0xffffffffu, alpha, (8 * qq + 4) & 31);
    // PV: A = V^T[16 coords][16 tokens] from the value tile (transposed ldmatrix).
#pragma unroll
    for (int mb = 0; mb < G_::MBLK; ++mb) {
      oacc[mb][0] *= al0; oacc[mb][1] *= al1; oacc[mb][2] *= al0; oacc[mb][3] *= al1;
      // matrices: (tokens 0-7, coords 0-7), (tokens 0-7, coords 8-15), (tokens 8-15, coords 0-7), (8-15, 8-15)
      const int tr = tb + (lane & 7) + ((lane >> 4) << 3);
      const int cc = mb * 16 + ((lane >> 3) & 1) * 8;
      uint32_t a0, a1, a2, a3;
      ldsm_x4_t(smem_addr(vtile + swz(tr, cc, G_::VROW)), a0, a1, a2, a3);
      uint32_t a[4] = {a0, a1, a2, a3};
      mma16816(oacc[mb], a, pb0, pb1);
    }
    __syncthreads();
  }
  // Merge the four warps: per head h (< G): M = max m_w, l = sum l_w e^(m_w - M),
  // acc = sum acc_w e^(m_w - M).
  float l_head = l_part + __shfl_xor_sync(0xffffffffu, l_part, 1);
  l_head += __shfl_xor_sync(0xffffffffu, l_head, 2);
  float* mw = mrg + warp * 8 * (D + 2);       // [8 heads][D + 2]: acc[D], m, l
  if (qq == 0 && qg < 8) {
    mw[qg * (D + 2) + D] = m_run;
    mw[qg * (D + 2) + D + 1] = l_head;
  }
#pragma unroll
  for (int mb = 0; mb < G_::MBLK; ++mb) {
    const int cr = mb * 16 + qg;
    mw[(2 * qq) * (D + 2) + cr] = oacc[mb][0];
    mw[(2 * qq + 1) * (D + 2) + cr] = oacc[mb][1];
    mw[(2 * qq) * (D + 2) + cr + 8] = oacc[mb][2];
    mw[(2 * qq + 1) * (D + 2) + cr + 8] = oacc[mb][3];
  }
  __syncthreads();
  for (int hh = 0; hh < G; ++hh) {
    float Mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) Mx = fmaxf(Mx, mrg[(w * 8 + hh) * (D + 2) + D]);
    float fw[4], lsum = 0.0f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float mwv = mrg[(w * 8 + hh) * (D + 2) + D];
      fw[w] = (mwv == -INFINITY) ? 0.0f : __expf(mwv - Mx);
      lsum += fw[w] * mrg[(w * 8 + hh) * (D + 2) + D + 1];
    }
    const size_t base = ((qbase + hh) * s.splits + split);
    for (int i = tid; i < D; i += NTH) {
      float v = 0.0f;
#pragma unroll
      for (int w = 0; w < 4; ++w) v += fw[w] * mrg[(w * 8 + hh) * (D + 2) + i];
      acc_out[base * D + i] = v;
    }
    if (tid == 0) {
      ml_out[base * 2] = Mx;
      ml_out[base * 2 + 1] = lsum;
    }
  }
}

}  // namespace fa
}  // namespace sq
