// Block-tiled float64 compress for the shapes the tensor-core kernel does not
// take: bf16 and f32 inputs, head_dim 64 and 256, fp16 prompts shorter than
// one 64-token tile.
//
// Same computation as k_compress_ref (SpectralQuant README, "Overview":
// rotation into the calibrated eigenbasis, Lloyd-Max codes under the
// water-filled widths; "Repository Structure": selective_qjl.py, QJL signs of
// the residual on the signal dims only). k_compress_ref reads the d x d
// eigenvector matrix once per vector, 512 KB per vector at head_dim 256, all
// of it from L2. Here one block of 256 threads takes NT = 8192 / D tokens of
// one head:
//
//  * the tokens are staged once, float64 and transposed (coordinate-major,
//    token pairs XOR-swizzled), together with ||x|| of each (the same
//    lane-strided sum and warp reduction as k_compress_ref);
//  * V streams through shared memory in chunks of 8 rows (cp.async,
//    double-buffered), each chunk used by all NT tokens;
//  * each thread accumulates a 4-token x 8-coordinate tile of Y = X V in
//    registers (a warp covers 16 tokens x 64 coordinates, so that every
//    shared-memory load of the inner loop is one wavefront);
//  * Y goes back to shared memory, and one warp per vector forms the codes,
//    the QJL signs and the record words with the per-vector steps of
//    k_compress_ref;
//  * 110 KB of shared memory and at most 128 registers per thread, so that
//    two blocks share an SM and one block's staging and per-vector steps
//    overlap the other's multiply-adds.
//
// Every y_i is the same chain of fused multiply-adds over j = 0 .. d-1 as in
// k_compress_ref, scaled by the same 1/||x||, so the two kernels write the
// same bits.
#pragma once

#include "codec.cuh"

namespace sq {
namespace blk {

constexpr int kThreads = 256;   // 8 warps; two blocks per SM
constexpr int kChunk = 8;       // rows of V per shared-memory stage

template <int D>
struct Geo {
  static constexpr int NT = 8192 / D;        // tokens per block
  static constexpr int XY_BYTES = 8 * D * NT;   // token tile [D][NT], later Y [NT][D] (64 KB)
  static constexpr int VB_BYTES = 8 * kChunk * D;   // one V stage
  static constexpr int WARPS_C = D / 64;     // warps along the coordinates
  static constexpr int WARPS_T = NT / 16;    // warps along the tokens
  static_assert(WARPS_C * WARPS_T == kThreads / 32, "eight warp tiles per block");
  // after the product the two V stages hold each warp's QJL residual and words
  static_assert(8 * D * (kThreads / 32) + 4 * kMaxWords * (kThreads / 32) <= 2 * VB_BYTES, "scratch fits");
  static constexpr int SMEM = XY_BYTES + 2 * VB_BYTES + 8 * kThreshTotal + 8 * kLevelsTotal + 16 * D + 8 * D + 8 * NT;
  static_assert(SMEM <= 113 * 1024, "two blocks per SM");
};

// Column of token tt in row j of the token tile: XOR-swizzled by pairs (a
// token pair stays adjacent), so that the coordinate-major stores of one
// token's row spread over the banks.
template <int D>
__device__ __forceinline__ int xcol(int j, int tt) {
  return tt ^ ((2 * j) & (Geo<D>::NT - 1));
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// grid (token blocks of NT, heads, batch), kThreads threads, Geo<D>::SMEM bytes.
template <typename T, int D>
__global__ void __launch_bounds__(kThreads, 2)
k_compress_blk(const uint8_t* __restrict__ recs, const T* __restrict__ x, int n_heads, int64_t n_tok,
               const int32_t* __restrict__ start_pos, CacheArgs c, uint32_t* __restrict__ flags) {
  using G = Geo<D>;
  extern __shared__ __align__(16) unsigned char sm[];
  const int h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const Rec rec = rec_at(recs, D, h);
  const RecHeader* hd = rec.hdr();
  if (!record_ok(hd, D) || hd->words != c.words || (hd->m > 0 && c.rnorm == nullptr)) {
    if (tid == 0 && flags) atomicOr(flags, SQ_FLAG_RECORD);
    return;
  }
  const int64_t sp = start_pos ? (int64_t)start_pos[b] : 0;
  if (sp < 0 || sp + n_tok > c.cap) {
    if (tid == 0 && blockIdx.x == 0 && flags) atomicOr(flags, SQ_FLAG_CAPACITY);
    return;
  }
  double* XY = (double*)sm;
  double* VB = (double*)(sm + G::XY_BYTES);
  unsigned char* p = sm + G::XY_BYTES + 2 * G::VB_BYTES;
  double* th = (double*)p;       p += 8 * kThreshTotal;   // regime 0 (the only one without fitted tables)
  double* lv = (double*)p;       p += 8 * kLevelsTotal;
  double* sig = (double*)p;      p += 8 * D;
  double* isig = (double*)p;     p += 8 * D;
  int* bits = (int*)p;           p += 4 * D;
  int* offs = (int*)p;           p += 4 * D;
  double* nrm_s = (double*)p;

  const double* Vg = rec.V();
  auto load_chunk = [&](int q) {
    const char* src = (const char*)(Vg + (size_t)q * kChunk * D);
    char* dst = (char*)(VB + (q & 1) * kChunk * D);
    for (int e = tid; e < G::VB_BYTES / 16; e += kThreads) cp_async16(dst + 16 * e, src + 16 * e);
    cp_async_commit();
  };
  load_chunk(0);
  const bool fitted = (hd->flags & kFlagFitted) != 0u;
  {
    const double* ft = rec.fit_th();
    const double* fl = rec.fit_lv();
    for (int e = tid; e < kThreshTotal; e += kThreads) th[e] = fitted ? ft[e] : c_th64[e];
    for (int e = tid; e < kLevelsTotal; e += kThreads) lv[e] = fitted ? fl[e] : c_lv64[e];
  }
  for (int i = tid; i < D; i += kThreads) {
    const double s = rec.sigma()[i];
    sig[i] = s;
    isig[i] = s > 0.0 ? 1.0 / s : 0.0;
    bits[i] = rec.bits()[i];
    offs[i] = rec.offsets()[i];
  }
  const bool normalize = (hd->flags & kFlagNormalize) != 0;
  const int64_t t0 = (int64_t)blockIdx.x * G::NT;
  const size_t row = (size_t)b * n_heads + h;
  // token tile (zero past the end of the prompt) and ||x||: warp per token
  for (int tt = warp; tt < G::NT; tt += kThreads / 32) {
    const int64_t t = t0 + tt;
    double ss = 0.0;
    if (t < n_tok) {
      const T* xt = x + (row * n_tok + t) * D;
      for (int j = lane; j < D; j += 32) {
        double v = (double)to_float<T>(xt[j]);
        XY[j * G::NT + xcol<D>(j, tt)] = v;
        ss += v * v;
      }
    } else {
      for (int j = lane; j < D; j += 32) XY[j * G::NT + xcol<D>(j, tt)] = 0.0;
    }
    ss = warp_sum(ss);
    if (lane == 0) nrm_s[tt] = normalize ? sqrt(ss) : 1.0;
  }

  // Y = X V: this thread's tokens tb, tb + 1, tb + 8, tb + 9 and coordinates
  // cb + 16 s + {0, 1}, s = 0..3
  const int wt = warp / G::WARPS_C, wc = warp % G::WARPS_C;
  const int tb = wt * 16 + 2 * (lane & 3);
  const int cb = wc * 64 + 2 * (lane >> 2);
  double acc[4][8];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[a][e] = 0.0;
  constexpr int NQ = D / kChunk;
#pragma unroll 1
  for (int q = 0; q < NQ; ++q) {
    if (q + 1 < NQ) {
      load_chunk(q + 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const double* vq = VB + (q & 1) * kChunk * D;
#pragma unroll
    for (int kk = 0; kk < kChunk; ++kk) {
      const int j = q * kChunk + kk;
      const double* xr = XY + j * G::NT;
      const double2 x01 = *(const double2*)(xr + xcol<D>(j, tb));
      const double2 x89 = *(const double2*)(xr + xcol<D>(j, tb + 8));
      const double xa[4] = {x01.x, x01.y, x89.x, x89.y};
      double2 v[4];
#pragma unroll
      for (int s = 0; s < 4; ++s) v[s] = *(const double2*)(vq + kk * D + cb + 16 * s);
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          acc[a][2 * s] = fma(v[s].x, xa[a], acc[a][2 * s]);
          acc[a][2 * s + 1] = fma(v[s].y, xa[a], acc[a][2 * s + 1]);
        }
    }
    __syncthreads();   // the stage is free for the chunk after next; the token tile is free after the last
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int t = tb + (a & 1) + 8 * (a >> 1);
#pragma unroll
    for (int s = 0; s < 4; ++s)
      *(double2*)(XY + t * D + cb + 16 * s) = make_double2(acc[a][2 * s], acc[a][2 * s + 1]);
  }
  __syncthreads();

  // codes, QJL signs and words: warp per vector (residual and words in the V stages)
  double* rs = VB + warp * D;
  uint32_t* wb = (uint32_t*)(VB + (kThreads / 32) * D) + warp * kMaxWords;
  const int W = hd->words, cbits = hd->code_bits;
  const double* th1 = fitted ? rec.fit_th() + kThreshTotal : th;
  const double* lv1 = fitted ? rec.fit_lv() + kLevelsTotal : lv;
  const VecEnc enc{hd, {th, th1}, {lv, lv1}, sig, isig, bits, offs, wb, rs, (int)hd->m};
  const double* S = rec.S();
  for (int tt = warp; tt < G::NT; tt += kThreads / 32) {
    const int64_t t = t0 + tt;
    if (t >= n_tok) break;
    for (int w = lane; w < W; w += 32) wb[w] = 0u;
    __syncwarp();
    const double nrm = nrm_s[tt];
    const double inv = nrm > 0.0 ? 1.0 / nrm : 0.0;
    for (int i = lane; i < D; i += 32) {
      double y = XY[tt * D + i];
      y *= inv;
      encode_coord(enc, i, y);
    }
    __syncwarp();
    finish_vector(enc, S, cbits, W, c, row, sp + t, nrm, lane);
  }
}

}  // namespace blk
}  // namespace sq
