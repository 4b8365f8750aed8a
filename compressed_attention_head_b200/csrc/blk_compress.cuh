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
//  * the tokens are staged once, float64 and transposed (coordinate-major),
//    together with ||x|| of each (the same lane-strided sum and warp
//    reduction as k_compress_ref);
//  * V streams through shared memory in chunks of 16 rows (cp.async,
//    double-buffered), each chunk used by all NT tokens;
//  * each thread accumulates a 4-token x 8-coordinate tile of Y = X V in
//    registers (a warp covers 16 tokens x 64 coordinates, so that every
//    shared-memory load of the inner loop is one wavefront);
//  * Y goes back to shared memory, and one warp per vector forms the codes,
//    the QJL signs and the record words with the per-vector steps of
//    k_compress_ref.
//
// Every y_i is the same chain of fused multiply-adds over j = 0 .. d-1 as in
// k_compress_ref, scaled by the same 1/||x||, so the two kernels write the
// same bits.
#pragma once

#include "codec.cuh"

namespace sq {
namespace blk {

constexpr int kThreads = 256;   // 8 warps
constexpr int kChunk = 16;      // rows of V per shared-memory stage

template <int D>
struct Geo {
  static constexpr int NT = 8192 / D;        // tokens per block
  static constexpr int LDX = NT + 2;         // row length (doubles) of the transposed token tile
  static constexpr int LDY = D + 2;          // row length of the Y tile (same storage)
  static constexpr int XY_BYTES = 8 * (D * LDX > NT * LDY ? D * LDX : NT * LDY);
  static constexpr int VB_BYTES = 8 * kChunk * D;   // one V stage
  static constexpr int WARPS_C = D / 64;     // warps along the coordinates
  static constexpr int WARPS_T = NT / 16;    // warps along the tokens
  static_assert(WARPS_C * WARPS_T == kThreads / 32, "eight warp tiles per block");
  static constexpr int SMEM = XY_BYTES + 2 * VB_BYTES + 16 * kThreshTotal + 16 * kLevelsTotal + 16 * D + 8 * D +
                              8 * NT + 4 * kMaxWords * (kThreads / 32) + 8 * D * (kThreads / 32);
};

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
__global__ void __launch_bounds__(kThreads, 1)
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
  double* XY = (double*)sm;                                  // tokens [D][LDX], later Y [NT][LDY]
  double* VB = (double*)(sm + G::XY_BYTES);                  // two stages of kChunk rows of V
  unsigned char* p = sm + G::XY_BYTES + 2 * G::VB_BYTES;
  double* th = (double*)p;       p += 16 * kThreshTotal;
  double* lv = (double*)p;       p += 16 * kLevelsTotal;
  double* sig = (double*)p;      p += 8 * D;
  double* isig = (double*)p;     p += 8 * D;
  int* bits = (int*)p;           p += 4 * D;
  int* offs = (int*)p;           p += 4 * D;
  double* nrm_s = (double*)p;    p += 8 * G::NT;
  uint32_t* wb = (uint32_t*)p + warp * kMaxWords;   p += 4 * kMaxWords * (kThreads / 32);
  double* rs = (double*)p + warp * D;

  const double* Vg = rec.V();
  auto load_chunk = [&](int q) {
    const char* src = (const char*)(Vg + (size_t)q * kChunk * D);
    char* dst = (char*)(VB + (q & 1) * kChunk * D);
    for (int e = tid; e < G::VB_BYTES / 16; e += kThreads) cp_async16(dst + 16 * e, src + 16 * e);
    cp_async_commit();
  };
  load_chunk(0);
  stage_codebooks(rec, th, lv, tid, kThreads);
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
        XY[j * G::LDX + tt] = v;
        ss += v * v;
      }
    } else {
      for (int j = lane; j < D; j += 32) XY[j * G::LDX + tt] = 0.0;
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
#pragma unroll 4
    for (int kk = 0; kk < kChunk; ++kk) {
      const double* xr = XY + (q * kChunk + kk) * G::LDX;
      const double2 x01 = *(const double2*)(xr + tb);
      const double2 x89 = *(const double2*)(xr + tb + 8);
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
      *(double2*)(XY + t * G::LDY + cb + 16 * s) = make_double2(acc[a][2 * s], acc[a][2 * s + 1]);
  }
  __syncthreads();

  // codes, QJL signs and words: warp per vector
  const int W = hd->words, cbits = hd->code_bits;
  const VecEnc enc{hd, th, lv, sig, isig, bits, offs, wb, rs, (int)hd->m};
  const double* S = rec.S();
  for (int tt = warp; tt < G::NT; tt += kThreads / 32) {
    const int64_t t = t0 + tt;
    if (t >= n_tok) break;
    for (int w = lane; w < W; w += 32) wb[w] = 0u;
    __syncwarp();
    const double nrm = nrm_s[tt];
    const double inv = nrm > 0.0 ? 1.0 / nrm : 0.0;
    for (int i = lane; i < D; i += 32) {
      double y = XY[tt * G::LDY + i];
      y *= inv;
      encode_coord(enc, i, y);
    }
    __syncwarp();
    finish_vector(enc, S, cbits, W, c, row, sp + t, nrm, lane);
  }
}

}  // namespace blk
}  // namespace sq
