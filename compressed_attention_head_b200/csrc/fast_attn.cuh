// Decode attention partials with tensor-core contractions (sm_100a).
//
// Same computation as k_attn_partial (SpectralQuant README, "Headline Results":
// decode attention over the compressed cache), organised so that every code
// is decoded once, by straight-line code, and both contractions run on the
// tensor pipe:
//
//  * A block (4 warps) owns one (batch, KV head, context split). Its warps
//    take 32-token tiles from a shared counter. A warp stages the K and V
//    records of its tile in shared memory transposed (word-major,
//    token-minor, 4-byte cp.async), so that lane t decodes token t and every
//    bit offset and width is the same in all lanes.
//  * Each 16-coordinate chunk of one width is decoded with compile-time bit
//    positions: widths 1-3 through pair tables (two fp16 levels per load),
//    widths 4-8 through single-level tables; every table a warp reads with
//    data-dependent indices fits one pass of the 32 banks, except the width-3
//    pair table, which is lane-replicated. The first key chunk (the widest,
//    signal codes) is decoded into fp16 hi and lo parts, so that with the
//    query weights also split, its products keep about 22 bits; the rest of the
//    key codes and all value codes use fp16 levels.
//  * Scores with mma.sync m16n8k16: rows = 16 tokens, columns = 8 query heads,
//    k = coordinates (plus a 16-column block of QJL signs +-1 whose weights are
//    u = scale sqrt(pi/2)/m S q'), then ||k_t|| and rho_t per row; online
//    softmax per warp; P = p ||v_t|| is transposed in registers (movmatrix)
//    into the B operand of O^T += V^T P^T (rows = coordinates).
//  * The four warps' (max, sum, acc) are merged at the end and written in the
//    layout k_attn_combine reads.
#pragma once

#include "attention.cuh"
#include "sq_common.cuh"

namespace sq {
namespace fa {

constexpr int TT = 32;           // tokens per warp tile
constexpr int NW = 4;            // warps per block
constexpr int NTH = NW * 32;
constexpr int RP = 33;           // row pitch (words) of the transposed record tiles

template <int D>
struct Geo {
  static constexpr int NCH = D / 16;      // 16-coordinate chunks
  static constexpr int MAXW = D / 8;      // record words per side (4 bits per coordinate)
  static constexpr int RROWS = MAXW + 1;  // staged rows (+1: the upper word of a funnel shift)
  static constexpr int ROW = D * 2;       // bytes of an fp16 tile row
  // Per-warp region: K records, V records, norms, tile, lo tile, QJL tile.
  static constexpr int OFF_RK = 0;
  static constexpr int OFF_RV = OFF_RK + RROWS * RP * 4;
  static constexpr int OFF_NRM = OFF_RV + RROWS * RP * 4;
  static constexpr int OFF_TILE = (OFF_NRM + 3 * TT * 4 + 127) & ~127;
  static constexpr int OFF_LO = OFF_TILE + TT * ROW;
  static constexpr int OFF_QT = OFF_LO + TT * 32;
  static constexpr int WARP_BYTES = (OFF_QT + TT * 32 + 127) & ~127;
};

// Block-wide tables (bytes).
struct Tab {
  static constexpr int P1 = 0;                        // u32 [4]: width-1 level pairs
  static constexpr int P2 = P1 + 16;                  // u32 [16]: width-2 level pairs
  static constexpr int QS = P2 + 64;                  // u32 [4]: QJL sign pairs (+-1)
  static constexpr int P3R = 128;                     // u32 [64][32]: width-3 pairs, lane-replicated
  // 16 zero bytes precede L16 and HL: entry -1 of either table reads as 0 (width-0 coordinates)
  static constexpr int L16 = P3R + 64 * 32 * 4 + 16;  // half [kLevelsTotal]
  static constexpr int HL = L16 + 1024 + 16;          // u32 [kLevelsTotal]: fp16 hi | fp16 lo << 16
  static constexpr int CH = HL + 2048;                // u32 [2][16]: chunk descriptors K, V
  static constexpr int CTR = CH + 128;                // u32: next tile
  static constexpr int CD = CTR + 16;                 // u32 [2][D]: coordinate descriptors K, V
};
static_assert(Tab::L16 % 16 == 0 && Tab::HL % 16 == 0 && Tab::CD % 16 == 0, "table alignment");
static_assert(kLevelsTotal * 2 <= 1024 && kLevelsTotal * 4 <= 2048, "level tables");

template <int D>
__host__ __device__ constexpr int tab_end() {
  return (Tab::CD + 2 * D * 4 + 127) & ~127;
}
template <int D>
__host__ __device__ constexpr int smem_bytes() {
  return tab_end<D>() + NW * Geo<D>::WARP_BYTES + 128;
}
// Resident blocks per SM the kernel is built for (registers capped to match by
// __launch_bounds__; shared memory checked below against the 228 KB of an SM,
// 1 KB of it reserved per block).
__host__ __device__ constexpr int min_blocks(int d) { return d <= 64 ? 4 : (d <= 128 ? 3 : 1); }
static_assert(min_blocks(64) * (smem_bytes<64>() + 1024) <= 233472, "d 64 residency");
static_assert(min_blocks(128) * (smem_bytes<128>() + 1024) <= 233472, "d 128 residency");
static_assert(min_blocks(256) * (smem_bytes<256>() + 1024) <= 233472, "d 256 residency");
// The merge at the end reuses the warp regions: [NW][8 heads][D + 2] floats.
static_assert(NW * 8 * (64 + 2) * 4 <= NW * Geo<64>::WARP_BYTES, "merge buffer (d 64)");
static_assert(NW * 8 * (128 + 2) * 4 <= NW * Geo<128>::WARP_BYTES, "merge buffer (d 128)");
static_assert(NW * 8 * (256 + 2) * 4 <= NW * Geo<256>::WARP_BYTES, "merge buffer (d 256)");

constexpr uint32_t kMixedChunk = 0xFFu;

__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
               : "memory");
}
// 4-byte copy that writes zeros instead when `in` is false (nothing is read then).
__device__ __forceinline__ void cp_async4_z(void* dst, const void* src, bool in) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src), "r"(in ? 4 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Byte offset of (row, column) in a tile whose rows are `rowbytes` long and
// whose 16-byte chunks are XOR-swizzled by (row & 7).
__device__ __forceinline__ uint32_t swz(int row, int col, int rowbytes) {
  int c = (col >> 3) ^ (row & 7);
  return (uint32_t)(row * rowbytes + (c << 4) + ((col & 7) << 1));
}
// Same for the 16-column tiles (32-byte rows, two chunks): chunks swap every
// four rows, so that the eight rows of an ldmatrix load hit distinct banks.
__device__ __forceinline__ uint32_t swz32(int row, int col) {
  int c = (col >> 3) ^ ((row >> 2) & 1);
  return (uint32_t)(row * 32 + (c << 4) + ((col & 7) << 1));
}

__device__ __forceinline__ void mma16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
// Transpose of an 8x8 fp16 matrix held in the mma fragment layout.
__device__ __forceinline__ uint32_t movm_t(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
  return d;
}
__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// The NP 32-bit pieces of the stream of lane's record starting at bit o
// (records transposed: word w of lane's token at rec[w * RP + lane]).
template <int NP>
__device__ __forceinline__ void pieces(const uint32_t* rec, int o, int lane, uint32_t* p) {
  const int wi = o >> 5, sh = o & 31;
  uint32_t w[NP + 1];
#pragma unroll
  for (int j = 0; j <= NP; ++j) w[j] = rec[(wi + j) * RP + lane];
#pragma unroll
  for (int j = 0; j < NP; ++j) p[j] = __funnelshift_r(w[j], w[j + 1], sh);
}
// Field of n bits at bit position pos of the pieces (n and pos are constants
// after unrolling, so the piece index and shifts fold).
__device__ __forceinline__ uint32_t fld(const uint32_t* p, int n, int pos) {
  const int a = pos >> 5, s = pos & 31;
  uint32_t v = p[a] >> s;
  if (s + n > 32) v |= p[a + 1] << (32 - s);
  return v & ((1u << n) - 1u);
}

// Decodes NC consecutive width-B chunks (16 NC coordinates starting at bit o)
// of lane's record into fp16 levels, written as 16-byte pieces of tile row
// lane from column col (two chunks at once give the loads of both to the
// scheduler together).
template <int B, int NC>
__device__ __forceinline__ void decode_chunk(const uint32_t* rec, int o, int lane, const uint8_t* tb,
                                             uint8_t* tile, int rowbytes, int col) {
  constexpr int NP = (16 * NC * B + 31) / 32;
  uint32_t p[NP];
  pieces<NP>(rec, o, lane, p);
  uint32_t h[8 * NC];
  if (B == 1) {
    const uint32_t* t = (const uint32_t*)(tb + Tab::P1);
#pragma unroll
    for (int k = 0; k < 8 * NC; ++k) h[k] = t[fld(p, 2, 2 * k)];
  } else if (B == 2) {
    const uint32_t* t = (const uint32_t*)(tb + Tab::P2);
#pragma unroll
    for (int k = 0; k < 8 * NC; ++k) h[k] = t[fld(p, 4, 4 * k)];
  } else if (B == 3) {
    const uint32_t* t = (const uint32_t*)(tb + Tab::P3R) + lane;
#pragma unroll
    for (int k = 0; k < 8 * NC; ++k) h[k] = t[fld(p, 6, 6 * k) * 32];
  } else {
    const unsigned short* t = (const unsigned short*)(tb + Tab::L16) + lv_off(B);
#pragma unroll
    for (int k = 0; k < 8 * NC; ++k) {
      const uint32_t a = t[fld(p, B, B * (2 * k))];
      const uint32_t b = t[fld(p, B, B * (2 * k + 1))];
      h[k] = a | (b << 16);
    }
  }
#pragma unroll
  for (int q = 0; q < 2 * NC; ++q)
    *(uint4*)(tile + swz(lane, col + 8 * q, rowbytes)) = make_uint4(h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3]);
}

// Coordinate descriptor: bit shift within the word (bits 0-4), code mask
// (bits 8-15), byte offset of the word's row in the transposed record tile
// (bits 16-31); all zero for a width-0 coordinate.
__host__ __device__ constexpr uint32_t coord_desc(int width, int offset) {
  return width == 0 ? 0u
                    : ((uint32_t)(offset & 31) | (((1u << width) - 1u) << 8) |
                       ((uint32_t)((offset >> 5) * RP * 4) << 16));
}
// Level-table index + 1 of the coordinate described by d in the record of the
// lane whose column starts at rl: mask + code, i.e. lv_off(width) + code + 1,
// and 0 for width 0 (entry -1 of the tables is zero).
__device__ __forceinline__ uint32_t code_index(const uint32_t* rl, uint32_t d) {
  const uint32_t* w = (const uint32_t*)((const uint8_t*)rl + (d >> 16));
  const uint32_t v = __funnelshift_r(w[0], w[RP], d);
  const uint32_t mask = (d >> 8) & 0xFFu;
  return mask + (v & mask);
}

// Decodes a chunk of mixed widths coordinate by coordinate (fp16 levels),
// from the chunk's 16 coordinate descriptors cd.
__device__ __forceinline__ void decode_mixed(const uint32_t* rl, const uint32_t* cd, const uint8_t* tb, int lane,
                                             uint8_t* tile, int rowbytes, int col) {
  const unsigned short* t = (const unsigned short*)(tb + Tab::L16) - 1;
  uint32_t h[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint2 dd = *(const uint2*)(cd + 2 * k);
    const uint32_t x0 = t[code_index(rl, dd.x)];
    const uint32_t x1 = t[code_index(rl, dd.y)];
    h[k] = x0 | (x1 << 16);
  }
  *(uint4*)(tile + swz(lane, col, rowbytes)) = make_uint4(h[0], h[1], h[2], h[3]);
  *(uint4*)(tile + swz(lane, col + 8, rowbytes)) = make_uint4(h[4], h[5], h[6], h[7]);
}

// Decodes all chunks of one side (first chunk excluded when skip0); two
// neighbouring chunks of one width go through one call. Not inlined: keys and
// values share one copy of its 17 decoders, which halves the instruction
// working set of the tile loop (measured: 4.6 % faster decode steps at G = 6).
template <int D>
__device__ __noinline__ void decode_side(const uint32_t* rec, const uint32_t* chd, const uint32_t* cd, bool skip0,
                                            int lane, const uint8_t* tb, uint8_t* tile) {
  constexpr int ROW = Geo<D>::ROW;
#pragma unroll 1
  for (int c = skip0 ? 1 : 0; c < Geo<D>::NCH;) {
    const uint32_t cw = chd[c];
    const int o = (int)(cw >> 8);
    const uint32_t w = cw & 0xFFu;
    const bool pair = c + 1 < Geo<D>::NCH && w >= 1u && w <= 8u && (chd[c + 1] & 0xFFu) == w;
    if (pair) {
      switch (w) {
        case 1: decode_chunk<1, 2>(rec, o, lane, tb, tile, ROW, 16 * c); break;
        case 2: decode_chunk<2, 2>(rec, o, lane, tb, tile, ROW, 16 * c); break;
        case 3: decode_chunk<3, 2>(rec, o, lane, tb, tile, ROW, 16 * c); break;
        case 4: decode_chunk<4, 2>(rec, o, lane, tb, tile, ROW, 16 * c); break;
        case 5: decode_chunk<5, 2>(rec, o, lane, tb, tile, ROW, 16 * c); break;
        case 6: decode_chunk<6, 2>(rec, o, lane, tb, tile, ROW, 16 * c); break;
        case 7: decode_chunk<7, 2>(rec, o, lane, tb, tile, ROW, 16 * c); break;
        default: decode_chunk<8, 2>(rec, o, lane, tb, tile, ROW, 16 * c); break;
      }
      c += 2;
      continue;
    }
    switch (w) {
      case 0: {
        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
        *(uint4*)(tile + swz(lane, 16 * c, ROW)) = z;
        *(uint4*)(tile + swz(lane, 16 * c + 8, ROW)) = z;
        break;
      }
      case 1: decode_chunk<1, 1>(rec, o, lane, tb, tile, ROW, 16 * c); break;
      case 2: decode_chunk<2, 1>(rec, o, lane, tb, tile, ROW, 16 * c); break;
      case 3: decode_chunk<3, 1>(rec, o, lane, tb, tile, ROW, 16 * c); break;
      case 4: decode_chunk<4, 1>(rec, o, lane, tb, tile, ROW, 16 * c); break;
      case 5: decode_chunk<5, 1>(rec, o, lane, tb, tile, ROW, 16 * c); break;
      case 6: decode_chunk<6, 1>(rec, o, lane, tb, tile, ROW, 16 * c); break;
      case 7: decode_chunk<7, 1>(rec, o, lane, tb, tile, ROW, 16 * c); break;
      case 8: decode_chunk<8, 1>(rec, o, lane, tb, tile, ROW, 16 * c); break;
      default: decode_mixed(rec + lane, cd + 16 * c, tb, lane, tile, ROW, 16 * c); break;
    }
    ++c;
  }
}

template <int D>
__global__ void __launch_bounds__(NTH, min_blocks(D)) k_attn_partial_tc(const uint8_t* __restrict__ recs_k,
                                                         const uint8_t* __restrict__ recs_v, CacheArgs kc,
                                                         CacheArgs vc, const int32_t* __restrict__ seq_lens,
                                                         AttnShape s, float* __restrict__ ws,
                                                         float* __restrict__ scores_out,
                                                         uint32_t* __restrict__ flags) {
  using GE = Geo<D>;
  constexpr int NCH = GE::NCH;
  constexpr int ROW = GE::ROW;
  extern __shared__ __align__(128) uint8_t smraw[];
  // aligned by pointer arithmetic on the shared array, so that every access
  // below stays a shared-memory access (an integer round trip would make them generic)
  uint8_t* sm = smraw + ((128u - (smem_addr(smraw) & 127u)) & 127u);
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
  // (records with fitted codebooks are served by the SIMT kernel: refused here)
  const bool ok = record_ok(hk, D) && record_ok(hv, D) && hk->words == kc.words && hv->words == vc.words &&
                  (hk->m == 0 || kc.rnorm != nullptr) && kc.words <= GE::MAXW && vc.words <= GE::MAXW &&
                  ((hk->flags | hv->flags) & kFlagFitted) == 0u;
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
  const int ntile = t_hi > t_lo ? (int)((t_hi - t_lo + TT - 1) / TT) : 0;
  const int m = ok ? hk->m : 0;
  const int nqs = (m + 15) >> 4;      // 16-column blocks of QJL signs (one in the common case m <= 16)
  const int wk = kc.words, wv = vc.words, kcb = ok ? hk->code_bits : 0;

  // ---- block tables
  uint32_t* tP1 = (uint32_t*)(sm + Tab::P1);
  uint32_t* tP2 = (uint32_t*)(sm + Tab::P2);
  uint32_t* tQS = (uint32_t*)(sm + Tab::QS);
  uint32_t* tP3 = (uint32_t*)(sm + Tab::P3R);
  __half* tL16 = (__half*)(sm + Tab::L16);
  uint32_t* tHL = (uint32_t*)(sm + Tab::HL);
  uint32_t* tCH = (uint32_t*)(sm + Tab::CH);
  uint32_t* tCD = (uint32_t*)(sm + Tab::CD);
  uint32_t* tCtr = (uint32_t*)(sm + Tab::CTR);
  if (tid < 4) tP1[tid] = pack_h2(c_lv32[lv_off(1) + (tid & 1)], c_lv32[lv_off(1) + (tid >> 1)]);
  if (tid < 16) tP2[tid] = pack_h2(c_lv32[lv_off(2) + (tid & 3)], c_lv32[lv_off(2) + (tid >> 2)]);
  if (tid < 4) tQS[tid] = pack_h2((tid & 1) ? 1.0f : -1.0f, (tid & 2) ? 1.0f : -1.0f);
  for (int e = tid; e < 64 * 32; e += NTH) {
    const int f = e >> 5;
    tP3[e] = pack_h2(c_lv32[lv_off(3) + (f & 7)], c_lv32[lv_off(3) + (f >> 3)]);
  }
  for (int e = tid; e < kLevelsTotal; e += NTH) {
    const double lv = c_lv64[e];
    const __half hi = __double2half(lv);
    const __half lo = __double2half(lv - (double)__half2float(hi));
    tL16[e] = hi;
    tHL[e] = (uint32_t)__half_as_ushort(hi) | ((uint32_t)__half_as_ushort(lo) << 16);
  }
  if (tid < 2 * NCH && ok) {
    // chunk descriptors: width if all 16 coordinates share it, else mixed; bit offset of the chunk
    const Rec r = tid < NCH ? rk : rv;
    const int c = tid % NCH;
    const uint8_t* bt = r.bits();
    const int b0 = bt[16 * c];
    uint32_t diff = 0u;
#pragma unroll
    for (int k = 1; k < 16; ++k) diff |= (uint32_t)(bt[16 * c + k] ^ b0);   // loads issued together
    const bool uni = diff == 0u;
    tCH[(tid < NCH ? 0 : 16) + c] = (uni ? (uint32_t)b0 : kMixedChunk) | ((uint32_t)r.offsets()[16 * c] << 8);
  }
  for (int e = tid; e < 2 * D; e += NTH) {
    const Rec r = e < D ? rk : rv;
    const int i = e < D ? e : e - D;
    tCD[e] = ok ? coord_desc(r.bits()[i], r.offsets()[i]) : 0u;
  }
  if (tid < 4) {
    // zero guards: entry -1 of the level tables
    ((uint32_t*)(sm + Tab::L16))[-1 - tid] = 0u;
    ((uint32_t*)(sm + Tab::HL))[-1 - tid] = 0u;
  }
  if (tid == 0) *tCtr = 0u;

  // ---- query fragments (B operands): rows k = coordinates, columns n = heads.
  // fp16 of w * wsc (hi; and lo for the first chunk) and of the QJL weights u.
  const size_t qbase = (size_t)b * s.n_q + (size_t)g * G;
  // max |w| over the G heads (rows qbase .. qbase + G - 1 are contiguous), four
  // loads in flight per lane; then max |u| over their first m entries
  float wmax = 0.0f;
  {
    const float* wg = wq + qbase * D;
    int e = lane;
    for (; e + 96 < G * D; e += 128) {
      const float a0 = wg[e], a1 = wg[e + 32], a2 = wg[e + 64], a3 = wg[e + 96];
      wmax = fmaxf(wmax, fmaxf(fmaxf(fabsf(a0), fabsf(a1)), fmaxf(fabsf(a2), fabsf(a3))));
    }
    for (; e < G * D; e += 32) wmax = fmaxf(wmax, fabsf(wg[e]));
  }
  for (int e = lane; e < G * m; e += 32) wmax = fmaxf(wmax, fabsf(uq[(qbase + e / m) * D + e % m]));
  wmax = warp_max(wmax);
  const float wsc = wmax > 0.0f ? exp2f(-ceilf(log2f(wmax))) : 1.0f;
  const float inv_wsc = 1.0f / wsc;
  const int hn = lane >> 2, tq = lane & 3;
  uint32_t wB[NCH][2], wL[2], uB[2];
  {
    const float* wrow = wq + (qbase + hn) * D;
    const float* urow = uq + (qbase + hn) * D;
    const bool hv_ok = hn < G;
#pragma unroll
    for (int ks = 0; ks < NCH; ++ks) {
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int col = ks * 16 + hf * 8 + 2 * tq;
        const float v0 = hv_ok ? wrow[col] * wsc : 0.0f;
        const float v1 = hv_ok ? wrow[col + 1] * wsc : 0.0f;
        const __half2 hh = __floats2half2_rn(v0, v1);
        wB[ks][hf] = *reinterpret_cast<const uint32_t*>(&hh);
        if (ks == 0) {
          const float2 back = __half22float2(hh);
          wL[hf] = pack_h2(v0 - back.x, v1 - back.y);
        }
      }
    }
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int j = hf * 8 + 2 * tq;
      const float u0 = (hv_ok && j < m) ? urow[j] * wsc : 0.0f;
      const float u1 = (hv_ok && j + 1 < m) ? urow[j + 1] * wsc : 0.0f;
      uB[hf] = pack_h2(u0, u1);
    }
  }
  __syncthreads();

  // ---- per-warp state
  uint8_t* wr = sm + tab_end<D>() + warp * GE::WARP_BYTES;
  uint32_t* recK = (uint32_t*)(wr + GE::OFF_RK);
  uint32_t* recV = (uint32_t*)(wr + GE::OFF_RV);
  float* nrm = (float*)(wr + GE::OFF_NRM);   // [3][TT]: ||k||, rho, ||v||
  uint8_t* tile = wr + GE::OFF_TILE;
  uint8_t* lot = wr + GE::OFF_LO;
  uint8_t* qt = wr + GE::OFF_QT;
  const size_t rowi = (size_t)b * s.n_kv + g;
  const uint32_t* kcodes = kc.codes + rowi * kc.cap * wk;
  const uint32_t* vcodes = vc.codes + rowi * vc.cap * wv;
  const float* knorm = kc.norm + rowi * kc.cap;
  const float* krho = kc.rnorm ? kc.rnorm + rowi * kc.cap : nullptr;
  const float* vnorm = vc.norm + rowi * vc.cap;

  auto grab = [&]() -> int {
    int t = 0;
    if (lane == 0) t = (int)atomicAdd(tCtr, 1u);
    return __shfl_sync(0xffffffffu, t, 0);
  };
  // Stage one side's records (lane = token); tokens past the range read as zeros.
  auto stage_rec = [&](uint32_t* rec, const uint32_t* src, int wn, int tile_i) {
    const int64_t t0 = t_lo + (int64_t)tile_i * TT;
    const bool in = t0 + lane < t_hi;
    // t0 is a multiple of 32: this tile is one interleaved block, word w at + 32 w
    const uint32_t* sp = src + (in ? (size_t)((t0 + lane) >> 5) * wn * 32 + lane : 0);
    uint32_t* dp = rec + lane;
    int w = 0;
    for (; w + 4 <= wn; w += 4) {
#pragma unroll
      for (int j = 0; j < 4; ++j) cp_async4_z(dp + (w + j) * RP, sp + (w + j) * 32, in);
    }
    for (; w < wn; ++w) cp_async4_z(dp + w * RP, sp + w * 32, in);
  };
  auto stage_nrm = [&](int tile_i) {
    const int64_t t0 = t_lo + (int64_t)tile_i * TT;
    const bool in = t0 + lane < t_hi;
    const int64_t tt = in ? t0 + lane : 0;
    cp_async4_z(nrm + lane, knorm + tt, in);
    cp_async4_z(nrm + 2 * TT + lane, vnorm + tt, in);
    if (m > 0) cp_async4_z(nrm + TT + lane, krho + tt, in); else nrm[TT + lane] = 0.0f;
  };

  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.0f, 0.0f};   // heads 2tq, 2tq + 1
  float oacc[NCH][4];
#pragma unroll
  for (int cb = 0; cb < NCH; ++cb) oacc[cb][0] = oacc[cb][1] = oacc[cb][2] = oacc[cb][3] = 0.0f;

  int cur = grab();
  if (cur < ntile) {
    stage_rec(recK, kcodes, wk, cur);
    stage_nrm(cur);
    stage_rec(recV, vcodes, wv, cur);
    cp_async_commit();
  }
  const uint32_t* chK = tCH;
  const uint32_t* chV = tCH + 16;
  while (cur < ntile) {
    const int nxt = grab();
    const int64_t t0 = t_lo + (int64_t)cur * TT;
    const int nt = (int)min((int64_t)TT, t_hi - t0);
    cp_async_wait_all();
    __syncwarp();

    // ---- decode the keys: first chunk as hi + lo, the rest as fp16, QJL signs
    {
      uint32_t hh[8], ll[8];
      const uint32_t* thl = (const uint32_t*)(sm + Tab::HL) - 1;
      const uint32_t* rl = recK + lane;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint2 dd = *(const uint2*)(tCD + 2 * k);
        const uint32_t x0 = thl[code_index(rl, dd.x)];
        const uint32_t x1 = thl[code_index(rl, dd.y)];
        hh[k] = __byte_perm(x0, x1, 0x5410);
        ll[k] = __byte_perm(x0, x1, 0x7632);
      }
      *(uint4*)(tile + swz(lane, 0, ROW)) = make_uint4(hh[0], hh[1], hh[2], hh[3]);
      *(uint4*)(tile + swz(lane, 8, ROW)) = make_uint4(hh[4], hh[5], hh[6], hh[7]);
      *(uint4*)(lot + swz32(lane, 0)) = make_uint4(ll[0], ll[1], ll[2], ll[3]);
      *(uint4*)(lot + swz32(lane, 8)) = make_uint4(ll[4], ll[5], ll[6], ll[7]);
    }
    decode_side<D>(recK, chK, tCD, true, lane, sm, tile);
    {
      uint32_t qh[8];
      uint32_t pc = 0u;
      if (m > 0) pieces<1>(recK, kcb, lane, &pc);
#pragma unroll
      for (int k = 0; k < 8; ++k) qh[k] = tQS[(pc >> (2 * k)) & 3u];
      *(uint4*)(qt + swz32(lane, 0)) = make_uint4(qh[0], qh[1], qh[2], qh[3]);
      *(uint4*)(qt + swz32(lane, 8)) = make_uint4(qh[4], qh[5], qh[6], qh[7]);
    }
    __syncwarp();
    if (nqs <= 1 && nxt < ntile) {       // the key records of this tile are consumed
      stage_rec(recK, kcodes, wk, nxt);
      cp_async_commit();
    }

    // ---- scores: rows = tokens, columns = heads
    float sv[2][4];
    float acc2[2][4], qa2[2][4];
#pragma unroll
    for (int mb = 0; mb < 2; ++mb) {
      float* acc = acc2[mb];
      float* qa = qa2[mb];
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[e] = qa[e] = 0.0f;
      const int ar = 16 * mb + (lane & 15), ac = (lane >> 4) * 8;
#pragma unroll
      for (int ks = 0; ks < NCH; ++ks) {
        uint32_t a[4];
        ldsm_x4(smem_addr(tile + swz(ar, 16 * ks + ac, ROW)), a);
        mma16816(acc, a, wB[ks][0], wB[ks][1]);
        if (ks == 0) {
          mma16816(acc, a, wL[0], wL[1]);
          uint32_t al[4];
          ldsm_x4(smem_addr(lot + swz32(ar, ac)), al);
          mma16816(acc, al, wB[0][0], wB[0][1]);
        }
      }
      {
        uint32_t aq[4];
        ldsm_x4(smem_addr(qt + swz32(ar, ac)), aq);
        mma16816(qa, aq, uB[0], uB[1]);
      }
    }
    if (nqs > 1) {
      // more than 16 QJL dimensions: the further 16-column blocks of signs, one
      // at a time through the same tile, with their weights u read from the
      // workspace; the key records are restaged only after the last block
      const float* urow = uq + (qbase + hn) * D;
      for (int qs = 1; qs < nqs; ++qs) {
        __syncwarp();
        uint32_t pc = 0u;
        pieces<1>(recK, kcb + 16 * qs, lane, &pc);
        uint32_t qh[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) qh[k] = tQS[(pc >> (2 * k)) & 3u];
        *(uint4*)(qt + swz32(lane, 0)) = make_uint4(qh[0], qh[1], qh[2], qh[3]);
        *(uint4*)(qt + swz32(lane, 8)) = make_uint4(qh[4], qh[5], qh[6], qh[7]);
        __syncwarp();
        uint32_t ub[2];
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int j = 16 * qs + hf * 8 + 2 * tq;
          const float u0 = (hn < G && j < m) ? urow[j] * wsc : 0.0f;
          const float u1 = (hn < G && j + 1 < m) ? urow[j + 1] * wsc : 0.0f;
          ub[hf] = pack_h2(u0, u1);
        }
#pragma unroll
        for (int mb = 0; mb < 2; ++mb) {
          uint32_t aq[4];
          ldsm_x4(smem_addr(qt + swz32(16 * mb + (lane & 15), (lane >> 4) * 8)), aq);
          mma16816(qa2[mb], aq, ub[0], ub[1]);
        }
      }
      __syncwarp();
      if (nxt < ntile) {
        stage_rec(recK, kcodes, wk, nxt);
        cp_async_commit();
      }
    }
#pragma unroll
    for (int mb = 0; mb < 2; ++mb) {
      const float* acc = acc2[mb];
      const float* qa = qa2[mb];
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int tl = 16 * mb + hn + 8 * hr;
        const float kn = nrm[tl], rho = nrm[TT + tl];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int head = 2 * tq + e;
          const bool valid = tl < nt && head < G;
          const float v = kn * inv_wsc * (acc[2 * hr + e] + rho * qa[2 * hr + e]);
          sv[mb][2 * hr + e] = valid ? v : -INFINITY;
          if (scores_out && valid) scores_out[((size_t)qbase + head) * s.max_ctx + t0 + tl] = v;
        }
      }
    }
    // ---- online softmax (per head: this lane holds 4 tokens of heads 2tq, 2tq + 1)
    float alpha[2];
    uint32_t pB[2][2];
    {
      float mx[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float v = fmaxf(fmaxf(sv[0][e], sv[0][2 + e]), fmaxf(sv[1][e], sv[1][2 + e]));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
        mx[e] = v;
      }
      float mnew[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        mnew[e] = fmaxf(m_run[e], mx[e]);
        alpha[e] = (m_run[e] == -INFINITY) ? 0.0f : __expf(m_run[e] - mnew[e]);
        m_run[e] = mnew[e];
      }
      float p[2][4];
#pragma unroll
      for (int mb = 0; mb < 2; ++mb)
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int e = q4 & 1;
          p[mb][q4] = (mnew[e] == -INFINITY || sv[mb][q4] == -INFINITY) ? 0.0f : __expf(sv[mb][q4] - mnew[e]);
        }
#pragma unroll
      for (int e = 0; e < 2; ++e) l_run[e] = l_run[e] * alpha[e] + (p[0][e] + p[0][2 + e] + p[1][e] + p[1][2 + e]);
      // P * ||v_t|| in fp16, transposed into the B operand (k = tokens, n = heads)
#pragma unroll
      for (int mb = 0; mb < 2; ++mb) {
        const float vn0 = nrm[2 * TT + 16 * mb + hn], vn1 = nrm[2 * TT + 16 * mb + hn + 8];
        pB[mb][0] = movm_t(pack_h2(p[mb][0] * vn0, p[mb][1] * vn0));
        pB[mb][1] = movm_t(pack_h2(p[mb][2] * vn1, p[mb][3] * vn1));
      }
    }
    __syncwarp();
    if (nxt < ntile) stage_nrm(nxt);

    // ---- decode the values into the same tile, then O^T += V^T P^T
    decode_side<D>(recV, chV, tCD + D, false, lane, sm, tile);
    __syncwarp();
    if (nxt < ntile) {
      stage_rec(recV, vcodes, wv, nxt);
    }
    cp_async_commit();
#pragma unroll
    for (int cb = 0; cb < NCH; ++cb) {
      oacc[cb][0] *= alpha[0];
      oacc[cb][1] *= alpha[1];
      oacc[cb][2] *= alpha[0];
      oacc[cb][3] *= alpha[1];
    }
#pragma unroll
    for (int mb = 0; mb < 2; ++mb) {
      const int tr = 16 * mb + (lane & 7) + ((lane >> 4) << 3);
      const int cofs = ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int cb = 0; cb < NCH; ++cb) {
        uint32_t a[4];
        ldsm_x4_t(smem_addr(tile + swz(tr, 16 * cb + cofs, ROW)), a);
        mma16816(oacc[cb], a, pB[mb][0], pB[mb][1]);
      }
    }
    __syncwarp();
    cur = nxt;
  }
  cp_async_wait_all();

  // ---- merge the four warps: per head h (< G): M = max m_w, l = sum l_w e^(m_w - M),
  // acc = sum acc_w e^(m_w - M).
  float lh[2];
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    float v = l_run[e];
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    v += __shfl_xor_sync(0xffffffffu, v, 8);
    v += __shfl_xor_sync(0xffffffffu, v, 16);
    lh[e] = v;
  }
  __syncthreads();
  float* mrg = (float*)(sm + tab_end<D>());     // [NW][8][D + 2]: acc[D], m, l
  float* mw = mrg + warp * 8 * (D + 2);
  if (hn == 0) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      mw[(2 * tq + e) * (D + 2) + D] = m_run[e];
      mw[(2 * tq + e) * (D + 2) + D + 1] = lh[e];
    }
  }
#pragma unroll
  for (int cb = 0; cb < NCH; ++cb) {
    const int cr = cb * 16 + hn;
    mw[(2 * tq) * (D + 2) + cr] = oacc[cb][0];
    mw[(2 * tq + 1) * (D + 2) + cr] = oacc[cb][1];
    mw[(2 * tq) * (D + 2) + cr + 8] = oacc[cb][2];
    mw[(2 * tq + 1) * (D + 2) + cr + 8] = oacc[cb][3];
  }
  __syncthreads();
  for (int hh = 0; hh < G; ++hh) {
    float Mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) Mx = fmaxf(Mx, mrg[(w * 8 + hh) * (D + 2) + D]);
    float fw[NW], lsum = 0.0f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float mwv = mrg[(w * 8 + hh) * (D + 2) + D];
      fw[w] = (mwv == -INFINITY) ? 0.0f : __expf(mwv - Mx);
      lsum += fw[w] * mrg[(w * 8 + hh) * (D + 2) + D + 1];
    }
    const size_t base = ((qbase + hh) * s.splits + split);
    for (int i = tid; i < D; i += NTH) {
      float v = 0.0f;
#pragma unroll
      for (int w = 0; w < NW; ++w) v += fw[w] * mrg[(w * 8 + hh) * (D + 2) + i];
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
