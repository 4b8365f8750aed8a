// Decode attention partials on the fifth-generation tensor cores (sm_100a).
//
// Same computation as k_attn_partial (SpectralQuant README, "Headline Results":
// decode attention over the compressed cache; "Overview": the QJL correction on
// the signal dims of the keys only), organised around tcgen05:
//
//  * A block owns one (batch, KV head, context split) and NG groups of four
//    warps; group g takes the split's 128-token tiles g, g + NG, ... . Warp q of
//    a group decodes tokens 32 q .. 32 q + 31 of a tile, lane = token: the
//    records of a tile arrive by one bulk copy (the cache stores 32-token
//    blocks word-interleaved), so lane t reads word w of its own record from
//    bank t, and every 16-coordinate chunk of one width is decoded with
//    compile-time bit positions through small level tables.
//  * Keys: each decoded chunk (8 registers of fp16 pairs of the lane's token)
//    goes straight into tensor memory with tcgen05.st (lane = token = TMEM
//    lane) and is the A operand of S[128 tokens x 16 heads] = K . W, the query
//    weights W in shared memory. The first chunk (the signal coordinates,
//    which carry almost all of q.k) is stored as fp16 hi and lo parts and
//    multiplied by the hi and lo parts of the weights, so its products keep
//    about 22 bits; the QJL signs enter as rho_t * (+-1) against the weights u.
//  * The scores come back per lane (tcgen05.ld). The softmax keeps a reference
//    maximum per head and group; the common tile only votes on whether a score
//    exceeds it by more than ln 4, and only then is it raised and the group's
//    accumulator and sums rescaled (so p <= 4 in the fp16 operand).
//  * Values: each decoded chunk is stored transposed (stmatrix .trans) into a
//    K-major V^T tile (rows = coordinates, tokens along K), p ||v|| likewise
//    into a K-major P tile (rows = heads), and O^T[coordinates x heads] +=
//    V^T . P runs on the tensor core into the group's TMEM accumulator. Tokens
//    sit along K in the order k(t) = 8 (t mod 4) + t / 4 within a warp, which
//    is the order stmatrix .trans produces from lane = token registers; V^T
//    and P share it, so the contraction over tokens is unchanged.
//  * head_dim 256: a tile's keys and values are decoded in halves of 128
//    coordinates; the key operand and the V^T tile hold one half at a time
//    (the score MMAs of the first key half, and the PV of the first value
//    half, finish before the second half overwrites them), which lets three
//    groups fit the 512 TMEM columns and the shared memory.
//  * One elected thread per group issues that group's bulk copies and MMAs;
//    mbarriers (bounded waits) and named barriers order the rest. The groups'
//    partials are merged at the end; the last block of a (row, KV head) to
//    finish merges the splits, and k_rotate_out (a launch of its own, batched
//    over the rows of each KV head) rotates the outputs back.
#pragma once

#include "attention.cuh"
#include "sm100.cuh"
#include "sq_common.cuh"

namespace sq {
namespace td {

constexpr int TILE = 128;          // tokens per tile (4 warps x 32)
constexpr int NW = 16;             // N of every MMA: query heads, padded
constexpr float kMarginLog2 = 2.0f;   // reference max raised when a score exceeds it by > 2 (log2 units)

template <int D>
struct Cfg {
  static constexpr int NCH = D / 16;                          // 16-coordinate chunks
  // head_dim 256 decodes a tile's keys and values in two halves of 128
  // coordinates each (the key operand in tensor memory and the V^T tile hold
  // one half at a time), so that three warp groups fit the SM's 512 TMEM
  // columns and its shared memory
  static constexpr bool SPL = D == 256;
  static constexpr int KCH = SPL ? NCH / 2 : NCH;             // key chunks of the first (or only) part
  static constexpr int NG = D == 256 ? 3 : 4;                 // warp groups decoding tiles
  static constexpr int NTH = NG * 128;
  static constexpr int MH = D > 128 ? 2 : 1;                  // 128-row halves of O^T
  static constexpr int OCOLS = 16 * MH;                       // TMEM columns of O^T
  static constexpr int AK0 = 8 * (KCH + 1);                   // key operand columns of the first part, no QJL
  static constexpr int VTR = SPL ? 128 : D;                   // coordinate rows of the V^T tile
  static constexpr int VT_BYTES = VTR * TILE * 2;             // K-major V^T tile
  static constexpr int P_BYTES = NW * TILE * 2;               // K-major P tile
  static constexpr int NKS_MAX = NCH + 2 + NCH;               // score k-steps with m <= D
  static constexpr int W_BYTES = ((NKS_MAX + 3) / 4) * 2048;  // score B operand
};

// Dynamic shared-memory plan (offsets from a base aligned to 1024 bytes). The
// lane-replicated width-3 table is a static shared array (its address folds
// into the load instructions).
struct Tab {
  static constexpr int W = 0;                          // score B operand (1024-aligned)
};
template <int D>
struct Plan {
  static constexpr int P1 = Tab::W + Cfg<D>::W_BYTES;  // uint2 [16]: width-1 quads
  static constexpr int P2 = P1 + 128;                  // u32 [16]: width-2 pairs
  // 16 zero bytes precede L16 and HL: entry -1 reads as 0 (width-0 coordinates)
  static constexpr int L16 = P2 + 64 + 16;             // half [kLevelsTotal]
  static constexpr int HL = L16 + 1024 + 16;           // u32 [kLevelsTotal]: fp16 hi | fp16 lo << 16
  static constexpr int CH = HL + 2048;                 // u32 [2][16]: chunk descriptors K, V
  static constexpr int CD = CH + 128;                  // u32 [2][D]: coordinate descriptors K, V
  // u64 [NG][10]: key records x2, scores, PV done, drain, spare, first key
  // part consumed, PV of the first V^T half done, value records x2
  static constexpr int BAR = CD + 8 * D;
  static constexpr int MISC = BAR + 8 * 10 * 4;        // u32 [16]: TMEM base, abort, wmax; u64 setup
  static constexpr int GS = MISC + 64;                 // per group: votes [4], maxima [4][16], l [4][16], mref [16], misc
  static constexpr int GS_BYTES = 16 + 256 + 256 + 64 + 64;
  static constexpr int GRP = (GS + Cfg<D>::NG * GS_BYTES + 1023) & ~1023;   // group regions (1024-aligned)
};
static_assert(kLevelsTotal * 2 <= 1024 && kLevelsTotal * 4 <= 2048, "level tables");

// The level tables every block of the kernel starts from, built once per
// device from the Lloyd-Max levels (td_build_tables) and copied into shared
// memory by one bulk copy per block: kImgBytes is the span of the plan from P1
// to CH (width-1 quad and width-2 pair tables, a zero guard, fp16 levels, a
// zero guard, fp16 hi | lo levels); g_p3r is the lane-replicated width-3 table.
constexpr int kImgBytes = 128 + 64 + 16 + 1024 + 16 + 2048;
__device__ __align__(128) uint8_t g_img[kImgBytes];
__device__ __align__(128) uint32_t g_p3r[64 * 32];

// Host side of the tables above, from the levels lv (lv_off layout, float64):
// the same values the kernel's decode steps expect (pairs of fp16 levels of
// the float32 levels; fp16 hi and lo parts of the float64 levels).
inline uint16_t h16_bits(__half h) {
  const __half_raw r = h;
  return r.x;
}
inline uint32_t pair_h2_host(float lo, float hi) {
  return (uint32_t)h16_bits(__float2half_rn(lo)) | ((uint32_t)h16_bits(__float2half_rn(hi)) << 16);
}
inline void build_tables_host(const double* lv, uint8_t* img, uint32_t* p3r) {
  for (int i = 0; i < kImgBytes; ++i) img[i] = 0;
  uint32_t* p1 = (uint32_t*)img;
  uint32_t* p2 = (uint32_t*)(img + 128);
  uint16_t* l16 = (uint16_t*)(img + 128 + 64 + 16);
  uint32_t* hl = (uint32_t*)(img + 128 + 64 + 16 + 1024 + 16);
  auto f = [&](int b, int k) { return (float)lv[lv_off(b) + k]; };
  for (int t = 0; t < 16; ++t) {   // four 1-bit codes: two fp16 level pairs
    p1[2 * t] = pair_h2_host(f(1, t & 1), f(1, (t >> 1) & 1));
    p1[2 * t + 1] = pair_h2_host(f(1, (t >> 2) & 1), f(1, t >> 3));
  }
  for (int t = 0; t < 16; ++t) p2[t] = pair_h2_host(f(2, t & 3), f(2, t >> 2));
  for (int e = 0; e < 64 * 32; ++e) p3r[e] = pair_h2_host(f(3, (e >> 5) & 7), f(3, e >> 8));
  for (int e = 0; e < kLevelsTotal; ++e) {
    const __half hi = __double2half(lv[e]);
    const __half lo = __double2half(lv[e] - (double)__half2float(hi));
    l16[e] = h16_bits(hi);
    hl[e] = (uint32_t)h16_bits(hi) | ((uint32_t)h16_bits(lo) << 16);
  }
}

// Bytes of one group's region: V^T tile, P tile, nrec record buffers.
template <int D>
__host__ __device__ constexpr size_t group_bytes(int wk, int wv, int nrec) {
  return (size_t)Cfg<D>::VT_BYTES + Cfg<D>::P_BYTES +
         (size_t)nrec * (((size_t)(wk + wv) * TILE * 4 + 3 * TILE * 4 + 1023) & ~(size_t)1023);
}
template <int D>
__host__ __device__ constexpr size_t smem_bytes(int wk, int wv, int nrec, int ng) {
  return (size_t)Plan<D>::GRP + (size_t)ng * group_bytes<D>(wk, wv, nrec) + 1024;   // + alignment slack
}

constexpr uint32_t kMixedChunk = 0xFFu;

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// The NP 32-bit pieces of lane's record starting at bit o (records of a
// 32-token block word-interleaved: word w of lane's token at rec[32 w + lane]).
template <int NP>
__device__ __forceinline__ void pieces(const uint32_t* rec, int o, int lane, uint32_t* p) {
  const int wi = o >> 5, sh = o & 31;
  uint32_t w[NP + 1];
#pragma unroll
  for (int j = 0; j <= NP; ++j) w[j] = rec[(wi + j) * 32 + lane];
#pragma unroll
  for (int j = 0; j < NP; ++j) p[j] = __funnelshift_r(w[j], w[j + 1], sh);
}
// Field of n bits at bit position pos of the pieces (compile-time positions).
__device__ __forceinline__ uint32_t fld(const uint32_t* p, int n, int pos) {
  const int a = pos >> 5, s = pos & 31;
  uint32_t v = p[a] >> s;
  if (s + n > 32) v |= p[a + 1] << (32 - s);
  return v & ((1u << n) - 1u);
}
// Field of 6 bits at pos, already multiplied by 128 (the row stride of the
// lane-replicated width-3 table) and OR-ed with the lane's byte offset in it.
__device__ __forceinline__ uint32_t fld6x128(const uint32_t* p, int pos, uint32_t lb) {
  const int a = pos >> 5, s = pos & 31;
  uint32_t v;
  if (s + 6 > 32) v = __funnelshift_r(p[a], p[a + 1], s) << 7;
  else v = s >= 7 ? (p[a] >> (s - 7)) : (p[a] << (7 - s));
  return (v & 0x1F80u) | lb;
}

// Decodes NC consecutive width-B chunks (16 NC coordinates from bit o) of the
// lane's record into fp16 level pairs h[8 NC] (h[k] = coordinates 2k, 2k + 1).
template <int B, int NC>
__device__ __forceinline__ void decode_chunk(const uint32_t* rec, int o, int lane, const uint8_t* sm, int p1off,
                                             const uint8_t* p3r, uint32_t lb3, uint32_t* h) {
  constexpr int NP = (16 * NC * B + 31) / 32;
  uint32_t p[NP];
  pieces<NP>(rec, o, lane, p);
  if (B == 1) {   // four coordinates per lookup
    const uint2* t = (const uint2*)(sm + p1off);
#pragma unroll
    for (int k = 0; k < 4 * NC; ++k) {
      const uint2 e = t[fld(p, 4, 4 * k)];
      h[2 * k] = e.x;
      h[2 * k + 1] = e.y;
    }
  } else if (B == 2) {
    const uint32_t* t = (const uint32_t*)(sm + p1off + 128);
#pragma unroll
    for (int k = 0; k < 8 * NC; ++k) h[k] = t[fld(p, 4, 4 * k)];
  } else if (B == 3) {
#pragma unroll
    for (int k = 0; k < 8 * NC; ++k) h[k] = *(const uint32_t*)(p3r + fld6x128(p, 6 * k, lb3));
  } else {
    const unsigned short* t = (const unsigned short*)(sm + p1off + 128 + 64 + 16) + lv_off(B);
#pragma unroll
    for (int k = 0; k < 8 * NC; ++k) {
      const uint32_t a = t[fld(p, B, B * (2 * k))];
      const uint32_t b = t[fld(p, B, B * (2 * k + 1))];
      h[k] = a | (b << 16);
    }
  }
}

// Coordinate descriptor: bit shift within the word (bits 0-4), code mask
// (bits 8-15), byte offset of the word's row in the interleaved record block
// (bits 16-31: 128 bytes per word); all zero for a width-0 coordinate.
__host__ __device__ constexpr uint32_t coord_desc(int width, int offset) {
  return width == 0 ? 0u
                    : ((uint32_t)(offset & 31) | (((1u << width) - 1u) << 8) |
                       ((uint32_t)((offset >> 5) * 128) << 16));
}
// Level-table index + 1 of the coordinate described by d in the record of the
// lane whose first word is at rl: lv_off(width) + code + 1, and 0 for width 0.
__device__ __forceinline__ uint32_t code_index(const uint32_t* rl, uint32_t d) {
  const uint32_t* w = (const uint32_t*)((const uint8_t*)rl + (d >> 16));
  const uint32_t v = __funnelshift_r(w[0], w[32], d);
  const uint32_t mask = (d >> 8) & 0xFFu;
  return mask + (v & mask);
}
// A chunk of mixed widths, coordinate by coordinate (fp16 levels).
__device__ __forceinline__ void decode_mixed(const uint32_t* rl, const uint32_t* cd, const unsigned short* l16m1,
                                             uint32_t* h) {
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint2 dd = *(const uint2*)(cd + 2 * k);
    const uint32_t x0 = l16m1[code_index(rl, dd.x)];
    const uint32_t x1 = l16m1[code_index(rl, dd.y)];
    h[k] = x0 | (x1 << 16);
  }
}

// Where decoded chunks go: keys into tensor memory (one 8-column store per
// chunk), values into the K-major V^T tile (two transposing matrix stores).
struct KeySink {
  uint32_t taddr;     // TMEM address of this warp's lanes, column 0 of the key operand
  __device__ __forceinline__ void put(int col8, const uint32_t* h) const { sm100::tmem_st8(taddr + col8, h); }
};
// RP: h[k] holds coordinates (2k, 2k + 1); each store takes them re-paired as
// (n, n + 4) of an 8-coordinate group, which keeps the stored rows of every
// 8x8 matrix on eight different swizzle positions (no bank conflicts). Used
// for head_dim <= 128, where it measured 0.5-1.3 % faster; at head_dim 256 the
// extra permutes cost more than the conflicts (+0.8 %).
template <bool RP>
struct ValSink {
  uint32_t base;      // shared address: the V^T tile + this lane's row / chunk offset
  __device__ __forceinline__ void put(int chunk, const uint32_t* h) const {
    if (RP) {
      sm100::stsm_x4_t(base + (uint32_t)chunk * 2048u, __byte_perm(h[0], h[2], 0x5410),
                       __byte_perm(h[0], h[2], 0x7632), __byte_perm(h[1], h[3], 0x5410),
                       __byte_perm(h[1], h[3], 0x7632));
      sm100::stsm_x4_t(base + (uint32_t)chunk * 2048u + 1024u, __byte_perm(h[4], h[6], 0x5410),
                       __byte_perm(h[4], h[6], 0x7632), __byte_perm(h[5], h[7], 0x5410),
                       __byte_perm(h[5], h[7], 0x7632));
    } else {
      sm100::stsm_x4_t(base + (uint32_t)chunk * 2048u, h[0], h[1], h[2], h[3]);
      sm100::stsm_x4_t(base + (uint32_t)chunk * 2048u + 1024u, h[4], h[5], h[6], h[7]);
    }
  }
};

// Decodes chunks c0 .. c1-1 of one side into the sink (keys: column block
// c + 1 - shift, values: chunk c - shift of the V^T tile); two neighbouring
// chunks of one width in one step.
template <int D, bool KEYS, typename Sink>
__device__ __forceinline__ void decode_side(const uint32_t* rec, const uint32_t* chd, const uint32_t* cd, int c0,
                                            int c1, int shift, int lane, const uint8_t* sm, int p1off,
                                            const uint8_t* p3r, uint32_t lb3, const unsigned short* l16m1,
                                            const Sink& sink) {
#pragma unroll 1
  for (int c = c0; c < c1;) {
    const uint32_t cw = chd[c];
    const int o = (int)(cw >> 8);
    const uint32_t w = cw & 0xFFu;
    const bool pair = c + 1 < c1 && w >= 1u && w <= 8u && (chd[c + 1] & 0xFFu) == w;
    uint32_t h[16];
    if (pair) {
      switch (w) {
        case 1: decode_chunk<1, 2>(rec, o, lane, sm, p1off, p3r, lb3, h); break;
        case 2: decode_chunk<2, 2>(rec, o, lane, sm, p1off, p3r, lb3, h); break;
        case 3: decode_chunk<3, 2>(rec, o, lane, sm, p1off, p3r, lb3, h); break;
        case 4: decode_chunk<4, 2>(rec, o, lane, sm, p1off, p3r, lb3, h); break;
        case 5: decode_chunk<5, 2>(rec, o, lane, sm, p1off, p3r, lb3, h); break;
        case 6: decode_chunk<6, 2>(rec, o, lane, sm, p1off, p3r, lb3, h); break;
        case 7: decode_chunk<7, 2>(rec, o, lane, sm, p1off, p3r, lb3, h); break;
        default: decode_chunk<8, 2>(rec, o, lane, sm, p1off, p3r, lb3, h); break;
      }
      sink.put(KEYS ? 8 * (c + 1 - shift) : c - shift, h);
      sink.put(KEYS ? 8 * (c + 2 - shift) : c + 1 - shift, h + 8);
      c += 2;
      continue;
    }
    switch (w) {
      case 0:
#pragma unroll
        for (int k = 0; k < 8; ++k) h[k] = 0u;
        break;
      case 1: decode_chunk<1, 1>(rec, o, lane, sm, p1off, p3r, lb3, h); break;
      case 2: decode_chunk<2, 1>(rec, o, lane, sm, p1off, p3r, lb3, h); break;
      case 3: decode_chunk<3, 1>(rec, o, lane, sm, p1off, p3r, lb3, h); break;
      case 4: decode_chunk<4, 1>(rec, o, lane, sm, p1off, p3r, lb3, h); break;
      case 5: decode_chunk<5, 1>(rec, o, lane, sm, p1off, p3r, lb3, h); break;
      case 6: decode_chunk<6, 1>(rec, o, lane, sm, p1off, p3r, lb3, h); break;
      case 7: decode_chunk<7, 1>(rec, o, lane, sm, p1off, p3r, lb3, h); break;
      case 8: decode_chunk<8, 1>(rec, o, lane, sm, p1off, p3r, lb3, h); break;
      default: decode_mixed(rec + lane, cd + 16 * c, l16m1, h); break;
    }
    sink.put(KEYS ? 8 * (c + 1 - shift) : c - shift, h);
    ++c;
  }
}

// float -> int with the same order (for warp max reductions with redux.sync)
__device__ __forceinline__ int ord_of(float f) {
  const int i = __float_as_int(f);
  return i >= 0 ? i : (i ^ 0x7FFFFFFF);
}
__device__ __forceinline__ float float_of_ord(int i) { return __int_as_float(i >= 0 ? i : (i ^ 0x7FFFFFFF)); }
__device__ __forceinline__ int warp_max_i(int v) {
  int r;
  asm volatile("redux.sync.max.s32 %0, %1, 0xffffffff;" : "=r"(r) : "r"(v));
  return r;
}

// Byte offset of element (row n, column k) of a [rows x K] K-major fp16
// operand in the 128-byte-swizzled canonical layout (64-column atoms of
// rows * 128 bytes, 8-row groups 1024 bytes apart, 16-byte chunks XOR-ed with
// the row within the group).
__host__ __device__ inline uint32_t sw128(int n, int k, int rows) {
  const int kb = k >> 6, e = k & 63, c = e >> 3, w = e & 7;
  return (uint32_t)(kb * rows * 128 + (n >> 3) * 1024 + (n & 7) * 128 + ((c ^ (n & 7)) << 4) + (w << 1));
}

template <int D, int MG>
__global__ void __launch_bounds__(Cfg<D>::NTH, 1)
k_decode_tc(const uint8_t* __restrict__ recs_k, const uint8_t* __restrict__ recs_v, CacheArgs kc, CacheArgs vc,
            const int32_t* __restrict__ seq_lens, AttnShape s, float* __restrict__ ws,
            float* __restrict__ scores_out, uint32_t* __restrict__ flags, int nrec, int ngs) {
  using C = Cfg<D>;
  using PL = Plan<D>;
  constexpr int NCH = C::NCH;
  extern __shared__ __align__(1024) uint8_t smraw[];
  __shared__ __align__(128) uint32_t s_p3r[64 * 32];   // width-3 level pairs, lane-replicated
  // aligned by pointer arithmetic on the shared array, so that every access
  // below stays a shared-memory access
  uint8_t* sm = smraw + ((1024u - (sm100::smem_u32(smraw) & 1023u)) & 1023u);
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31, grp = warp >> 2, q = warp & 3;
  const int G = s.group;
  Rec rk = rec_at(recs_k, D, g), rv = rec_at(recs_v, D, g);
  const RecHeader* hk = rk.hdr();
  const RecHeader* hv = rv.hdr();
  float* wq = ws;
  float* uq = ws + (size_t)s.batch * s.n_q * D;
  float* acc_out = uq + (size_t)s.batch * s.n_q * D;
  float* ml_out = acc_out + (size_t)s.batch * s.n_q * s.splits * D;
  // (records with fitted codebooks are served by the SIMT kernel: refused here)
  const bool ok = record_ok(hk, D) && record_ok(hv, D) && hk->words == kc.words && hv->words == vc.words &&
                  (hk->m == 0 || kc.rnorm != nullptr) && ((hk->flags | hv->flags) & kFlagFitted) == 0u;
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
  const int ntile = t_hi > t_lo ? (int)((t_hi - t_lo + TILE - 1) / TILE) : 0;
  const int m = ok ? hk->m : 0;
  const int nqs = (m + 15) >> 4;
  const int wk = kc.words, wv = vc.words, kcb = ok ? hk->code_bits : 0;
  // TMEM columns per group: key operand (split: the larger part), scores, O^T;
  // as many groups as fit in 512 columns and (ngs) in shared memory
  const int ak_cols = C::SPL ? max(C::AK0, 8 * (C::KCH + nqs)) : C::AK0 + 8 * nqs;
  const int need = ak_cols + NW + C::OCOLS;
  const int gstride = need <= 128 ? 128 : (need <= 256 ? 256 : 512);
  const int ngr = min(min(C::NG, 512 / gstride), ngs);
  const int col_s = gstride - NW - C::OCOLS;     // scores, then O^T, at the end of the group's columns
  const int col_o = gstride - C::OCOLS;

  // ---- records of the block's cache row: the issuer of group gi copies tile
  // kk of the group (tokens t0 .. t0 + 127) into its record buffer bf
  const size_t rowi = (size_t)attn_cache_row(s, b) * s.n_kv + g;
  const uint32_t* kcodes = kc.codes + rowi * (size_t)kc.cap * wk;
  const uint32_t* vcodes = vc.codes + rowi * (size_t)vc.cap * wv;
  const float* knorm = kc.norm + rowi * kc.cap;
  const float* krho = kc.rnorm ? kc.rnorm + rowi * kc.cap : nullptr;
  const float* vnorm = vc.norm + rowi * vc.cap;
  const size_t rec_buf = (((size_t)(wk + wv) * TILE * 4 + 3 * TILE * 4 + 1023) & ~(size_t)1023);
  uint64_t* bars = (uint64_t*)(sm + PL::BAR);
  // parts: 1 = the key words, norms and rho (barrier 10 gi + bf), 2 = the
  // value words and norms (barrier 10 gi + 8 + bf). Without the split both
  // parts are requested together after the vote barrier, on the key barrier
  // (measured: requesting the key part right after the key barrier, or
  // waiting on two barriers, cost 3-4 % at head_dim 128).
  auto issue_records = [&](int gi, int kk, int bf, int parts) {
    const int64_t t0 = t_lo + (int64_t)(gi + kk * ngr) * TILE;
    const int64_t blk0 = t0 >> 5;
    const int nb = (int)min((int64_t)4, (kc.cap - t0) >> 5);    // whole 32-token blocks inside the cache
    uint8_t* rb = sm + PL::GRP + (size_t)gi * group_bytes<D>(wk, wv, nrec) + C::VT_BYTES + C::P_BYTES +
                  (size_t)bf * rec_buf;
    uint8_t* nr = rb + (size_t)(wk + wv) * TILE * 4;
    const uint32_t nbytes = nb * 128;
    const uint32_t kbytes = (uint32_t)(nb * wk * 128), vbytes = (uint32_t)(nb * wv * 128);
    if (parts & 1) {
      uint64_t* bar = bars + 10 * gi + bf;
      sm100::mbar_expect_tx(bar, kbytes + nbytes * (krho ? 2u : 1u) + (C::SPL ? 0u : vbytes + nbytes));
      sm100::bulk_load(rb, kcodes + blk0 * wk * 32, kbytes, bar);
      sm100::bulk_load(nr, knorm + t0, nbytes, bar);
      if (krho) sm100::bulk_load(nr + TILE * 4, krho + t0, nbytes, bar);
    }
    if (parts & 2) {
      uint64_t* bar = bars + 10 * gi + (C::SPL ? 8 : 0) + bf;
      if (C::SPL) sm100::mbar_expect_tx(bar, vbytes + nbytes);
      sm100::bulk_load(rb + (size_t)wk * TILE * 4, vcodes + blk0 * wv * 32, vbytes, bar);
      sm100::bulk_load(nr + 2 * TILE * 4, vnorm + t0, nbytes, bar);
    }
  };

  // ---- block tables (as in the mma.sync kernel, plus the score B operand)
  uint32_t* tCH = (uint32_t*)(sm + PL::CH);
  uint32_t* tCD = (uint32_t*)(sm + PL::CD);
  uint32_t* misc = (uint32_t*)(sm + PL::MISC);    // [0] TMEM base, [1] abort, [2] max |weight| (float bits)
  uint64_t* b_setup = (uint64_t*)(misc + 4);       // level tables copied in
  if (tid == 0) {
    misc[1] = 0u;
    misc[2] = 0u;
    // per group: key records x2, scores, PV, drain, spare, first key part
    // consumed, first PV half, value records x2 (one arrival each: an
    // expect-tx or a commit)
    for (int k = 0; k < 10 * C::NG; ++k) sm100::mbar_init(&bars[k], 1u);
    sm100::mbar_init(b_setup, 1);
    sm100::fence_mbar_init();
    // the level tables, and the first record tiles of every group, start
    // arriving while the block builds its other tables and the query operand
    sm100::mbar_expect_tx(b_setup, (uint32_t)(kImgBytes + 64 * 32 * 4));
    sm100::bulk_load(sm + PL::P1, g_img, (uint32_t)kImgBytes, b_setup);
    sm100::bulk_load(s_p3r, g_p3r, 64u * 32u * 4u, b_setup);
    for (int gi = 0; gi < ngr; ++gi) {
      const int ntk = gi < ntile ? (ntile - gi + ngr - 1) / ngr : 0;
      for (int kk = 0; kk < nrec && kk < ntk; ++kk) issue_records(gi, kk, kk, 3);
    }
  }
  if (tid < 2 * NCH && ok) {
    const Rec r = tid < NCH ? rk : rv;
    const int c = tid % NCH;
    const uint8_t* bt = r.bits();
    const int b0 = bt[16 * c];
    uint32_t diff = 0u;
#pragma unroll
    for (int k = 1; k < 16; ++k) diff |= (uint32_t)(bt[16 * c + k] ^ b0);
    tCH[(tid < NCH ? 0 : 16) + c] = (diff == 0u ? (uint32_t)b0 : kMixedChunk) | ((uint32_t)r.offsets()[16 * c] << 8);
  }
  for (int e = tid; e < 2 * D; e += C::NTH) {
    const Rec r = e < D ? rk : rv;
    const int i = e < D ? e : e - D;
    tCD[e] = ok ? coord_desc(r.bits()[i], r.offsets()[i]) : 0u;
  }
  __syncwarp();
  if (warp == 0) {
    sm100::tmem_alloc(&misc[0], 512);
    sm100::tmem_relinquish();
  }
  // the G heads' weights w (and u on its first m entries) read once into the
  // first group's V^T tile (free until the tiles start), with their max |.|
  // -> one power-of-two scale for the fp16 operand
  const size_t qbase = (size_t)b * s.n_q + (size_t)g * G;
  float* wst = (float*)(sm + PL::GRP);            // [G][D] w, then [G][m] u
  float* ust = wst + G * D;
  static_assert(16 * 2 * D * 4 <= C::VT_BYTES, "weight staging fits the V^T tile");
  __syncthreads();
  {
    float mx = 0.0f;
    for (int e = tid; e < G * D; e += C::NTH) {
      const float x = wq[qbase * D + e];
      wst[e] = x;
      mx = fmaxf(mx, fabsf(x));
    }
    for (int e = tid; e < G * m; e += C::NTH) {
      const float x = uq[(qbase + e / m) * D + e % m];
      ust[e] = x;
      mx = fmaxf(mx, fabsf(x));
    }
    mx = warp_max(mx);
    if (lane == 0) atomicMax(&misc[2], __float_as_uint(mx));
  }
  __syncthreads();
  const float wmax = __uint_as_float(misc[2]);
  const float wsc = wmax > 0.0f ? exp2f(-ceilf(log2f(wmax))) : 1.0f;
  const float inv_wsc = 1.0f / wsc;
  // score B operand: rows n = heads (16), k-steps of 16: [w hi c0][w lo c0][w hi c0][w hi c1..][u blocks]
  {
    uint8_t* Wb = sm + Tab::W;
    const int nks = NCH + 2 + nqs;
    static_assert(NW == 16, "W operand index arithmetic");
    for (int e = tid; e < NW * 16 * nks; e += C::NTH) {
      // e = (st NW + n) 16 + j: k-step st, head n, k j within the step (coalesced over j)
      const int st = e >> 8, n = (e >> 4) & 15, j = e & 15, kk = 16 * st + j;
      float v = 0.0f;
      bool lo = false;
      if (n < G) {
        if (st < 3) {
          v = wst[n * D + j] * wsc;
          lo = st == 1;
        } else if (st < NCH + 2) {
          v = wst[n * D + 16 * (st - 2) + j] * wsc;
        } else {
          const int jj = 16 * (st - NCH - 2) + j;
          v = jj < m ? ust[n * m + jj] * wsc : 0.0f;
        }
      }
      __half h = __float2half_rn(v);
      if (lo) h = __float2half_rn(v - __half2float(h));
      *(__half*)(Wb + sw128(n, kk, NW)) = h;
    }
  }
  sm100::fence_async_smem();
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem_base = misc[0];
  volatile uint32_t* abort_flag = &misc[1];

  // ---- per-group state
  float mref[MG], lpart[MG];
  int cpos[MG];        // causal bound of each column (prefill; no bound for decode)
#pragma unroll
  for (int h = 0; h < MG; ++h) {
    mref[h] = -INFINITY;
    lpart[h] = 0.0f;
    cpos[h] = (h < G && attn_col_live(s, b, h)) ? (int)min(attn_col_pos(seq_lens, s, b, h), (int64_t)INT32_MAX) : -1;
  }
  uint8_t* gr = sm + PL::GRP + (size_t)grp * group_bytes<D>(wk, wv, nrec);
  uint8_t* sVt = gr;
  uint8_t* sP = gr + C::VT_BYTES;
  uint8_t* sRec = sP + C::P_BYTES;
  uint8_t* gs = sm + PL::GS + grp * PL::GS_BYTES;          // votes [4] (u32), maxima [4][16] (int), l [4][16], mref [16]
  uint64_t* b_rec = bars + 10 * grp;                         // [0], [1]: key records of buffer 0 / 1
  uint64_t* b_recv = bars + 10 * grp + 8;                    // [0], [1]: value records of buffer 0 / 1
  uint64_t* b_s = bars + 10 * grp + 2;                       // scores ready
  uint64_t* b_pv = bars + 10 * grp + 3;                      // PV of the group's last tile done
  uint64_t* b_gdrain = bars + 10 * grp + 4;                  // the group's MMAs done (before the free)
  uint64_t* b_ka = bars + 10 * grp + 6;                      // split: the first key part's MMAs done
  uint64_t* b_pv1 = bars + 10 * grp + 7;                     // split: the first V^T half's PV done
  const bool issuer = q == 0 && lane == 0;                   // the group's copies and MMAs
  const bool active = grp < ngr;
  const int ntg = active && grp < ntile ? (ntile - grp + ngr - 1) / ngr : 0;   // tiles of this group
  const uint32_t gcol = (uint32_t)(grp * gstride);
  const uint32_t t_lanes = (uint32_t)(q * 32) << 16;
  const uint32_t idesc = sm100::idesc_f16(TILE, NW);
  const uint32_t lb3 = (uint32_t)lane << 2;
  const uint8_t* p3r = (const uint8_t*)s_p3r;
  const unsigned short* l16m1 = (const unsigned short*)(sm + PL::L16) - 1;
  const uint32_t* hlm1 = (const uint32_t*)(sm + PL::HL) - 1;
  // this lane's stmatrix row address within the V^T and P tiles (see the header)
  const int st_i = lane >> 3, st_c = lane & 7;
  const int st_row = 2 * st_i + (st_c & 1);
  const int st_kc = 4 * q + (st_c >> 1);
  // V^T rows of this lane's matrix row: coordinates (2i, 2i + 1), or (i,
  // i + 4) with the re-paired stores (ValSink)
  constexpr bool RP = D <= 128;
  const int vt_row = RP ? st_i + 4 * (st_c & 1) : st_row;
  const uint32_t vt_lane = sm100::smem_u32(sVt) + (uint32_t)((st_kc >> 3) * (C::VTR * 128) + vt_row * 128 +
                                                            (((st_kc & 7) ^ vt_row) << 4));
  const uint32_t p_lane = sm100::smem_u32(sP) + (uint32_t)((st_kc >> 3) * (NW * 128) + st_row * 128 +
                                                          (((st_kc & 7) ^ st_row) << 4));
  uint32_t* err = flags;
  // descriptor of the score B operand (k-step 0)
  const uint64_t w_desc = sm100::sw128_desc(sm100::smem_u32(sm + Tab::W));

  if (!sm100::mbar_wait(b_setup, 0u, err)) *abort_flag = 1;   // level tables in shared memory
  // tiles whose key / value records were requested (prefixes; the first by thread 0)
  int n_issued = min(ntg, nrec), n_issued_v = min(ntg, nrec);
  const float LOG2E = 1.4426950408889634f;
  // The MMAs of a tile of group gi. Scores, k-steps [s0, s1): A = the keys in
  // tensor memory (k-step st reads c0 hi for st = 0 and 1, c0 lo for 2, chunk
  // st - 2 = column block st - 1 after; the second key part of a split tile
  // sits sub columns lower), B = W (four 32-byte k-steps per 2048-byte atom).
  // PV: O^T += V^T P over the V^T tile (split: the coordinate half h).
  // Descriptors advance in their start-address field (16-byte units, no carry
  // out of it).
  const int nks = NCH + 2 + nqs;
  auto issue_scores = [&](int s0, int s1, int sub, uint64_t* bar) {
    const uint32_t d_s = tmem_base + gcol + (uint32_t)col_s;
    uint32_t a_col = tmem_base + gcol + (uint32_t)((s0 < 2 ? 0 : 8 * (s0 - 1)) - sub);
    uint64_t bd = w_desc + (uint64_t)(((s0 >> 2) * (NW * 128) + (s0 & 3) * 32) >> 4);
    for (int st = s0; st < s1; ++st) {
      sm100::mma_f16_ts(d_s, a_col, bd, idesc, st > 0 ? 1u : 0u);
      a_col += st > 0 ? 8u : 0u;
      bd += (st & 3) == 3 ? (uint64_t)((NW * 128 - 96) >> 4) : 2u;
    }
    sm100::mma_commit(bar);
  };
  const uint64_t vt_desc = sm100::sw128_desc(sm100::smem_u32(sVt));
  const uint64_t p_desc = sm100::sw128_desc(sm100::smem_u32(sP));
  auto issue_pv = [&](int kt, int h, uint64_t* bar) {
#pragma unroll
    for (int ks = 0; ks < TILE / 16; ++ks) {
      const uint64_t bd = p_desc + (uint64_t)(((ks >> 2) * (NW * 128) + (ks & 3) * 32) >> 4);
#pragma unroll
      for (int mh = 0; mh < (C::SPL ? 1 : C::MH); ++mh) {
        const uint64_t ad =
            vt_desc + (uint64_t)(((ks >> 2) * (C::VTR * 128) + mh * (128 * 128) + (ks & 3) * 32) >> 4);
        sm100::mma_f16(tmem_base + gcol + (uint32_t)(col_o + 16 * (mh + h)), ad, bd, idesc,
                       (kt > 0 || ks > 0) ? 1u : 0u);
      }
    }
    sm100::mma_commit(bar);
  };
  // The QJL sign blocks of the lane's token into key-operand columns col ..:
  // bit 2k -> sign of the low half, bit 2k + 1 -> sign of the high half (1 = +rho)
  auto store_qjl = [&](int col, bool valid, const float* nrm, int tok, const uint32_t* recK) {
    if (m == 0) return;
    const float rho = valid ? nrm[TILE + tok] : 0.0f;
    const uint32_t rp = pack_h2(rho, rho);
    for (int j = 0; j < nqs; ++j) {
      uint32_t pc = 0u;
      pieces<1>(recK, kcb + 16 * j, lane, &pc);
      uint32_t qh[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t bits2 = (pc >> (2 * k)) & 3u;
        const uint32_t neg = ((~bits2 & 1u) << 15) | ((~bits2 & 2u) << 30);
        qh[k] = rp ^ neg;
      }
      sm100::tmem_st8(tmem_base + t_lanes + gcol + (uint32_t)(col + 8 * j), qh);
    }
  };
  for (int kk = 0; kk < ntg; ++kk) {
    const int bf = kk % nrec;
    const int64_t t0 = t_lo + (int64_t)(grp + kk * ngr) * TILE;
    const int nt = (int)min((int64_t)TILE, t_hi - t0);          // valid tokens of the tile
    const int tok = 32 * q + lane;                              // this lane's token within the tile
    const bool valid = tok < nt;
    const uint8_t* rb = sRec + (size_t)bf * rec_buf;
    const uint32_t* recK = (const uint32_t*)rb + (size_t)q * wk * 32;
    const uint32_t* recV = (const uint32_t*)(rb + (size_t)wk * TILE * 4) + (size_t)q * wv * 32;
    const float* nrm = (const float*)(rb + (size_t)(wk + wv) * TILE * 4);
    bool live = *abort_flag == 0 && sm100::mbar_wait(&b_rec[bf], (uint32_t)((kk / nrec) & 1), err);
    if (!live) *abort_flag = 1;
    // ---- keys -> tensor memory
    if (live) {
      const KeySink ks{tmem_base + t_lanes + gcol};
      {
        uint32_t hh[8], ll[8];
        const uint32_t* rl = recK + lane;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint2 dd = *(const uint2*)(tCD + 2 * k);
          const uint32_t x0 = hlm1[code_index(rl, dd.x)];
          const uint32_t x1 = hlm1[code_index(rl, dd.y)];
          hh[k] = __byte_perm(x0, x1, 0x5410);
          ll[k] = __byte_perm(x0, x1, 0x7632);
        }
        sm100::tmem_st8(ks.taddr, hh);
        sm100::tmem_st8(ks.taddr + 8, ll);
      }
      decode_side<D, true>(recK, tCH, tCD, 1, C::KCH, 0, lane, sm, PL::P1, p3r, lb3, l16m1, ks);
      if (!C::SPL) store_qjl(8 * (NCH + 1), valid, nrm, tok, recK);
    }
    const float kn = valid ? nrm[tok] : 0.0f;
    sm100::tmem_wait_st();
    sm100::tc_fence_before();
    sm100::named_bar(1 + grp, 128);
    if (issuer && live) {
      sm100::tc_fence_after();
      issue_scores(0, C::SPL ? C::KCH + 2 : nks, 0, C::SPL ? b_ka : b_s);
    }
    // ---- values -> V^T tile (the previous tile's PV must be done with it)
    if (live && kk > 0) live = sm100::mbar_wait(b_pv, (uint32_t)((kk - 1) & 1), err);
    if (C::SPL && live) live = sm100::mbar_wait(&b_recv[bf], (uint32_t)((kk / nrec) & 1), err);
    if (!live) *abort_flag = 1;
    const ValSink<RP> vsnk{vt_lane};
    if (live) decode_side<D, false>(recV, tCH + 16, tCD + D, 0, C::KCH, 0, lane, sm, PL::P1, p3r, lb3, l16m1, vsnk);
    const float vn = valid ? nrm[2 * TILE + tok] : 0.0f;
    sm100::fence_async_smem();
    if constexpr (C::SPL) {
      // ---- keys, second part: chunks KCH .. NCH-1 and the QJL blocks, into
      // the columns of the first part once its MMAs have read them
      if (live) live = sm100::mbar_wait(b_ka, (uint32_t)(kk & 1), err);
      if (!live) *abort_flag = 1;
      sm100::tc_fence_after();
      if (live) {
        const KeySink ks{tmem_base + t_lanes + gcol};
        decode_side<D, true>(recK, tCH, tCD, C::KCH, NCH, C::KCH + 1, lane, sm, PL::P1, p3r, lb3, l16m1, ks);
        store_qjl(8 * C::KCH, valid, nrm, tok, recK);
      }
      sm100::tmem_wait_st();
      sm100::tc_fence_before();
      sm100::named_bar(1 + grp, 128);
      if (issuer && live) {
        sm100::tc_fence_after();
        issue_scores(C::KCH + 2, nks, 8 * (C::KCH + 1), b_s);
        if (kk + nrec < ntg) {   // the key records of this tile are consumed
          issue_records(grp, kk + nrec, bf, 1);
          n_issued = kk + nrec + 1;
        }
      }
    }
    // the records are consumed once all four warps pass the vote barrier
    // below (split: the value records after the second V^T half)
    // ---- scores -> softmax
    float sv[MG];
#pragma unroll
    for (int h = 0; h < MG; ++h) sv[h] = -INFINITY;
    bool over = false;
    if (live) live = sm100::mbar_wait(b_s, (uint32_t)(kk & 1), err);
    if (!live) *abort_flag = 1;
    sm100::tc_fence_after();
    if (live) {
      float raw[16];
      sm100::tmem_ld16(tmem_base + t_lanes + gcol + (uint32_t)col_s, raw);
#pragma unroll
      for (int h = 0; h < MG; ++h) {
        const bool vh = valid && h < G && (int)(t0 + tok) <= cpos[h];
        const float v = kn * inv_wsc * raw[h];
        sv[h] = vh ? v : -INFINITY;
        if (scores_out && vh) scores_out[(qbase + h) * s.max_ctx + t0 + tok] = v;
        over |= vh && v > mref[h] + kMarginLog2 / LOG2E;
      }
    }
    uint32_t* votes = (uint32_t*)gs;
    int* gmax = (int*)(gs + 16);
    const uint32_t wv_any = __any_sync(0xffffffffu, over) ? 1u : 0u;
    if (lane == 0) votes[q] = wv_any;
    sm100::named_bar(1 + grp, 128);
    if (!C::SPL && issuer && live && kk + nrec < ntg) {   // the records of this tile are consumed
      issue_records(grp, kk + nrec, bf, 3);
      n_issued = n_issued_v = kk + nrec + 1;
    }
    const bool raise = (votes[0] | votes[1] | votes[2] | votes[3]) != 0u;
    if (raise) {
      // tile max per head over the group, then the new reference and the rescale
      // (every thread of the group takes this branch: votes are shared)
#pragma unroll
      for (int h = 0; h < MG; ++h) {
        const int mx = warp_max_i(ord_of(sv[h]));
        if (lane == 0) gmax[q * 16 + h] = mx;
      }
      sm100::named_bar(1 + grp, 128);
      float alpha[MG];
      bool any_change = false;
#pragma unroll
      for (int h = 0; h < MG; ++h) {
        float tmax = -INFINITY;
#pragma unroll
        for (int w = 0; w < 4; ++w) tmax = fmaxf(tmax, float_of_ord(gmax[w * 16 + h]));
        const float mnew = fmaxf(mref[h], tmax);
        alpha[h] = (mref[h] == -INFINITY || mnew == mref[h]) ? (mref[h] == -INFINITY ? 0.0f : 1.0f)
                                                            : exp2f((mref[h] - mnew) * LOG2E);
        any_change |= mnew != mref[h] && mref[h] != -INFINITY;
        mref[h] = mnew;
        lpart[h] *= (alpha[h] == 0.0f ? 0.0f : alpha[h]);
      }
      if (any_change && kk > 0 && live) {
        // O^T (lane = coordinate) *= alpha per head column; the PV of the
        // previous tile is done (waited above)
        sm100::tc_fence_after();
#pragma unroll
        for (int mh = 0; mh < C::MH; ++mh) {
          float o[16];
          const uint32_t oa = tmem_base + t_lanes + gcol + (uint32_t)(col_o + 16 * mh);
          sm100::tmem_ld16(oa, o);
#pragma unroll
          for (int h = 0; h < MG; ++h) o[h] *= alpha[h];
          sm100::tmem_st16(oa, o);
        }
        sm100::tmem_wait_st();
      }
    }
    // ---- P = e^(s - mref) ||v|| -> K-major P tile
    {
      uint32_t ph[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        float p0 = 0.0f, p1 = 0.0f;
        if (2 * k < MG && live) {
          p0 = sv[2 * k] == -INFINITY ? 0.0f : exp2f((sv[2 * k] - mref[2 * k]) * LOG2E);
          lpart[2 * k] += p0;
        }
        if (2 * k + 1 < MG && live) {
          p1 = sv[2 * k + 1] == -INFINITY ? 0.0f : exp2f((sv[2 * k + 1] - mref[2 * k + 1]) * LOG2E);
          lpart[2 * k + 1] += p1;
        }
        ph[k] = pack_h2(p0 * vn, p1 * vn);
      }
      sm100::stsm_x4_t(p_lane, ph[0], ph[1], ph[2], ph[3]);
      sm100::stsm_x4_t(p_lane + 1024u, ph[4], ph[5], ph[6], ph[7]);
    }
    sm100::fence_async_smem();
    sm100::tc_fence_before();
    sm100::named_bar(1 + grp, 128);
    if (issuer && live) {
      sm100::tc_fence_after();
      issue_pv(kk, 0, C::SPL ? b_pv1 : b_pv);
    }
    if constexpr (C::SPL) {
      // ---- values, second half: coordinates 128 .. 255 into the V^T tile once
      // the first half's PV has read it
      if (live) live = sm100::mbar_wait(b_pv1, (uint32_t)(kk & 1), err);
      if (!live) *abort_flag = 1;
      if (live) decode_side<D, false>(recV, tCH + 16, tCD + D, C::KCH, NCH, C::KCH, lane, sm, PL::P1, p3r, lb3,
                                      l16m1, vsnk);
      sm100::fence_async_smem();
      sm100::tc_fence_before();
      sm100::named_bar(1 + grp, 128);
      if (issuer && live) {
        sm100::tc_fence_after();
        issue_pv(kk, 1, b_pv);
        if (kk + nrec < ntg) {   // the value records of this tile are consumed
          issue_records(grp, kk + nrec, bf, 2);
          n_issued_v = kk + nrec + 1;
        }
      }
    }
  }
  // ---- the group's sums and accumulator
  bool live_end = ntg > 0 && *abort_flag == 0;
  if (ntg > 0) {
    if (!sm100::mbar_wait(b_pv, (uint32_t)((ntg - 1) & 1), err)) {
      *abort_flag = 1;
      live_end = false;
    }
  }
  float* lsum = (float*)(gs + 16 + 256);          // [4][16]
  float* gref = (float*)(gs + 16 + 256 + 256);    // [16]
#pragma unroll
  for (int h = 0; h < MG; ++h) {
    const float v = warp_sum(lpart[h]);
    if (lane == 0) lsum[q * 16 + h] = v;
  }
  if (issuer) {
#pragma unroll
    for (int h = 0; h < MG; ++h) gref[h] = mref[h];
  }
  sm100::tc_fence_after();
  __syncthreads();
  // the V^T tiles are free now: merge buffer [NG][16][D] floats over the group regions
  float* mrg = (float*)(sm + PL::GRP);
  static_assert(C::NG * 16 * D * 4 <= C::NG * C::VT_BYTES, "merge buffer");
  if (live_end) {
#pragma unroll
    for (int mh = 0; mh < C::MH; ++mh) {
      float o[16];
      sm100::tmem_ld16(tmem_base + t_lanes + gcol + (uint32_t)(col_o + 16 * mh), o);
      const int i = 128 * mh + 32 * q + lane;   // (rows past D, for head_dim 64, are not coordinates)
      if (i < D) {
#pragma unroll
        for (int h = 0; h < MG; ++h) mrg[((size_t)grp * 16 + h) * D + i] = o[h];
      }
    }
  }
  __syncthreads();
  // merge the groups: per head h < G
  for (int h = 0; h < G && h < MG; ++h) {
    float Mx = -INFINITY;
    for (int k = 0; k < ngr; ++k) {
      const int ntk = k < ntile ? (ntile - k + ngr - 1) / ngr : 0;
      if (ntk > 0) Mx = fmaxf(Mx, ((const float*)(sm + PL::GS + k * PL::GS_BYTES + 16 + 512))[h]);
    }
    float fw[C::NG], lt = 0.0f;
#pragma unroll
    for (int k = 0; k < C::NG; ++k) {
      fw[k] = 0.0f;
      const int ntk = (k < ngr && k < ntile) ? (ntile - k + ngr - 1) / ngr : 0;
      if (ntk > 0 && Mx != -INFINITY) {
        const uint8_t* gk = sm + PL::GS + k * PL::GS_BYTES;
        const float mk = ((const float*)(gk + 16 + 512))[h];
        fw[k] = mk == -INFINITY ? 0.0f : exp2f((mk - Mx) * LOG2E);
        const float* lk = (const float*)(gk + 16 + 256);
        lt += fw[k] * (lk[h] + lk[16 + h] + lk[32 + h] + lk[48 + h]);
      }
    }
    const size_t base = (qbase + h) * s.splits + split;
    if (s.splits == 1) {
      // the only block of (b, g): its merged vector a = sigma ⊙ acc / l goes
      // straight over the column's query operand row (what merge_one writes)
      const float inv_l = lt > 0.0f ? 1.0f / lt : 0.0f;
      const bool okv = record_ok(hv, D);
      const float* sigv = rv.sigma_f();
      for (int i = tid; i < D; i += C::NTH) {
        float v = 0.0f;
#pragma unroll
        for (int k = 0; k < C::NG; ++k)
          if (fw[k] != 0.0f) v += fw[k] * mrg[((size_t)k * 16 + h) * D + i];
        wq[(qbase + h) * D + i] = okv ? v * inv_l * sigv[i] : 0.0f;
      }
      continue;
    }
    for (int i = tid; i < D; i += C::NTH) {
      float v = 0.0f;
#pragma unroll
      for (int k = 0; k < C::NG; ++k)
        if (fw[k] != 0.0f) v += fw[k] * mrg[((size_t)k * 16 + h) * D + i];
      acc_out[base * D + i] = v;
    }
    if (tid == 0) {
      ml_out[base * 2] = Mx;
      ml_out[base * 2 + 1] = lt;
    }
  }
  // ---- the last block of (b, g) to finish merges the splits (every block
  // publishes its partials, then counts itself; the counter was cleared by
  // the prepare step of this call)
  __shared__ int s_last;
  if (s.splits > 1) __threadfence();
  __syncthreads();
  if (tid == 0) {
    int last = 1;
    if (s.splits > 1) {
      uint32_t* cnt = attn_counters(ws, s) + (size_t)b * s.n_kv + g;
      last = atomicAdd(cnt, 1u) == (uint32_t)(s.splits - 1);
      if (last) *cnt = 0u;
    }
    s_last = last;
  }
  __syncthreads();
  // every copy and MMA a group's issuer started has completed before the block
  // frees its tensor memory and exits (on the normal path they have; after a
  // timed-out wait some may still run): bounded waits
  if (tid == 0) sm100::mbar_wait(b_setup, 0u, nullptr);
  if (issuer) {
    for (int kk = max(0, n_issued - nrec); kk < n_issued; ++kk)
      sm100::mbar_wait(&b_rec[kk % nrec], (uint32_t)((kk / nrec) & 1), nullptr);
    if (C::SPL)
      for (int kk = max(0, n_issued_v - nrec); kk < n_issued_v; ++kk)
        sm100::mbar_wait(&b_recv[kk % nrec], (uint32_t)((kk / nrec) & 1), nullptr);
  }
  if (issuer) {
    sm100::mma_commit(b_gdrain);
    if (!sm100::mbar_wait(b_gdrain, 0u, err)) *abort_flag = 1;
  }
  sm100::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tmem_base, 512);
  }
  if (tid == 0 && *abort_flag && err) atomicOr(err, SQ_FLAG_TIMEOUT);
  if (s_last && s.splits > 1) {
    __threadfence();
    merge_one(recs_v, s, ws, g, b, (float*)sm, tid, C::NTH);
  }
}

}  // namespace td
}  // namespace sq
