// libsq host entry points: argument checks, per-device table upload, launches.
// The public contract (arguments, layouts, ownership, errors) is in include/sq.h.
#include <algorithm>
#include <cstdio>
#include <mutex>

#include "sq_common.cuh"

namespace sq {
// Tables that kernels stage into shared memory with one element per thread
// live in global memory (coalesced loads; constant memory would serialise the
// 32 addresses of a warp); c_D is read with warp-uniform indices.
__device__ double c_lv64[kLevelsTotal];
__device__ double c_th64[kThreshTotal];
__device__ float c_lv32[kLevelsTotal];
__constant__ double c_D[SQ_MAX_BITS + 1];
__device__ float4 c_tcq[248];          // tcc cell tables: thresholds (T_j, T_j+1, T_j+2) per width 4..8
__device__ uint8_t c_tccell[560];      // tcc cell tables: positive thresholds below each cell
}  // namespace sq

#include <cudaTypedefs.h>

#include "attention.cuh"
#include "calibrate.cuh"
#include "codec.cuh"
#include "blk_compress.cuh"
#include "fast_attn.cuh"
#include "tc_compress.cuh"
#include "tc_decode.cuh"
#include "decode_step.cuh"

namespace sq {

const double* codebook_levels(int b);
const double* codebook_thresholds(int b);
double codebook_distortion(int b);

namespace {

std::mutex g_mu;
bool g_ready[128];
bool g_force_ref = false;   // route compress to the float64 reference kernel
int g_attn_path = 0;        // attention partials: 0 tcgen05 kernel (auto), 1 SIMT, 2 mma.sync kernel
int g_eacc_units = tcc::EACC_DEFAULT_UNITS;   // accumulation bound of the tensor-core compress radius, in 2^-24
tcc::QuantConst g_kq;       // register thresholds and cell counts of the tensor-core compress
int g_sms[128];

bool supported_d(int d) { return d == 32 || d == 64 || d == 128 || d == 256; }
bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }
bool valid_dtype(int t) { return t == SQ_F32 || t == SQ_F16 || t == SQ_BF16; }

// The name of the last CUDA error a call of this thread ran into (for sq_last_error).
thread_local char g_last_err[160] = "none";
sq_status cuda_ok(cudaError_t e) {
  if (e == cudaSuccess) return SQ_OK;
  snprintf(g_last_err, sizeof(g_last_err), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
  return SQ_ERR_CUDA;
}

// Cell tables of the tensor-core compress for widths 4..8 (see tc_compress.cuh)
// from the float32 positive thresholds T_1 < ... < T_n of each width; false if
// some cell would hold two thresholds (cannot happen for the Gaussian codebook).
bool build_cell_tables(const double* th, float4* q, uint8_t* cell, tcc::QuantConst* kq) {
  kq->t2 = (float)th[th_off(2) + 2];
  for (int j = 0; j < 3; ++j) kq->t3[j] = (float)th[th_off(3) + 4 + j];
  for (int b = 0; b < 12; ++b) kq->ncell[b] = 1;
  for (int e = 0; e < tcc::kCellBytes; ++e) cell[e] = 0;
  const float inf = INFINITY;
  for (int b = 4; b <= 8; ++b) {
    const int n = (1 << (b - 1)) - 1;
    float T[130];
    T[0] = 0.0f;
    for (int j = 1; j <= n; ++j) T[j] = (float)th[th_off(b) + n + j];   // thresholds n+1 .. 2n are positive
    T[n + 1] = inf;
    T[n + 2] = inf;
    for (int j = 0; j <= n; ++j) q[tcc::q_off(b) + j] = make_float4(T[j], T[j + 1], T[j + 2], 0.0f);
    const double h = ldexp(1.0, -(b - 2));
    const int ncell = (int)floor((double)T[n] / h) + 1;
    if (ncell > tcc::cell_cap(b)) return false;
    kq->ncell[b] = ncell;
    for (int g = 0; g < ncell; ++g) {
      int lo = 0, inside = 0;
      for (int j = 1; j <= n; ++j) {
        if ((double)T[j] < g * h) ++lo;
        else if (g + 1 < ncell ? (double)T[j] < (g + 1) * h : true) ++inside;
      }
      if (inside > 1) return false;
      cell[tcc::cell_off(b) + g] = (uint8_t)lo;
    }
    if (th[th_off(b) + n] != 0.0) return false;   // the middle threshold is 0
  }
  return true;
}

// Dynamic shared memory the tcgen05 decode kernel may take: 227 KB per block
// minus its static shared memory (the 8 KB width-3 table, a flag, and the
// padding that aligns the dynamic part to 1 KB), with 1 KB to spare.
constexpr int kTdSmemLimit = 232448 - 9216 - 1024;

// Uploads the Lloyd-Max tables to the current device once.
sq_status ensure_init(int* dev_out = nullptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return SQ_ERR_CUDA;
  if (dev_out) *dev_out = dev;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_ready[dev]) return SQ_OK;
  double lv[kLevelsTotal], th[kThreshTotal], dist[SQ_MAX_BITS + 1];
  float lv32[kLevelsTotal];
  dist[0] = 1.0;
  for (int b = 1; b <= SQ_MAX_BITS; ++b) {
    const double* l = codebook_levels(b);
    const double* t = codebook_thresholds(b);
    for (int k = 0; k < (1 << b); ++k) lv[lv_off(b) + k] = l[k];
    for (int k = 0; k + 1 < (1 << b); ++k) th[th_off(b) + k] = t[k];
    dist[b] = codebook_distortion(b);
  }
  for (int k = 0; k < kLevelsTotal; ++k) lv32[k] = (float)lv[k];
  float4 tq[tcc::kQEntries];
  uint8_t tcell[tcc::kCellBytes];
  if (!build_cell_tables(th, tq, tcell, &g_kq)) return SQ_ERR_CUDA;
  if (cudaMemcpyToSymbol(c_tcq, tq, sizeof(tq)) != cudaSuccess) return SQ_ERR_CUDA;
  if (cudaMemcpyToSymbol(c_tccell, tcell, sizeof(tcell)) != cudaSuccess) return SQ_ERR_CUDA;
  if (cudaMemcpyToSymbol(c_lv64, lv, sizeof(lv)) != cudaSuccess) return SQ_ERR_CUDA;
  if (cudaMemcpyToSymbol(c_th64, th, sizeof(th)) != cudaSuccess) return SQ_ERR_CUDA;
  if (cudaMemcpyToSymbol(c_lv32, lv32, sizeof(lv32)) != cudaSuccess) return SQ_ERR_CUDA;
  if (cudaMemcpyToSymbol(c_D, dist, sizeof(dist)) != cudaSuccess) return SQ_ERR_CUDA;
  {
    static uint8_t img[td::kImgBytes];
    static uint32_t p3r[64 * 32];
    td::build_tables_host(lv, img, p3r);
    if (cudaMemcpyToSymbol(td::g_img, img, sizeof(img)) != cudaSuccess) return SQ_ERR_CUDA;
    if (cudaMemcpyToSymbol(td::g_p3r, p3r, sizeof(p3r)) != cudaSuccess) return SQ_ERR_CUDA;
  }
  // Kernels that take more than 48 KB of dynamic shared memory.
  const int big = 200 * 1024;
  cudaFuncSetAttribute(k_jacobi, cudaFuncAttributeMaxDynamicSharedMemorySize, big);
  cudaFuncSetAttribute(k_compress_ref<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, big);
  cudaFuncSetAttribute(k_compress_ref<__half>, cudaFuncAttributeMaxDynamicSharedMemorySize, big);
  cudaFuncSetAttribute(k_compress_ref<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, big);
  cudaFuncSetAttribute(k_decompress_ref, cudaFuncAttributeMaxDynamicSharedMemorySize, big);
  cudaFuncSetAttribute(k_attn_partial<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, big);
  cudaFuncSetAttribute(k_attn_partial<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, big);
  cudaFuncSetAttribute(k_attn_partial<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, big);
  cudaFuncSetAttribute(k_attn_partial<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, big);
  cudaFuncSetAttribute(k_attn_partial<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, big);
  cudaFuncSetAttribute(tcc::k_compress_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, tcc::SMEM_BYTES);
#define SQ_BLK_ATTR(T)                                                                                        \
  cudaFuncSetAttribute(blk::k_compress_blk<T, 64>, cudaFuncAttributeMaxDynamicSharedMemorySize, blk::Geo<64>::SMEM);  \
  cudaFuncSetAttribute(blk::k_compress_blk<T, 128>, cudaFuncAttributeMaxDynamicSharedMemorySize, blk::Geo<128>::SMEM); \
  cudaFuncSetAttribute(blk::k_compress_blk<T, 256>, cudaFuncAttributeMaxDynamicSharedMemorySize, blk::Geo<256>::SMEM)
  SQ_BLK_ATTR(float); SQ_BLK_ATTR(__half); SQ_BLK_ATTR(__nv_bfloat16);
#undef SQ_BLK_ATTR
  cudaFuncSetAttribute(fa::k_attn_partial_tc<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, fa::smem_bytes<64>());
  cudaFuncSetAttribute(fa::k_attn_partial_tc<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, fa::smem_bytes<128>());
  cudaFuncSetAttribute(fa::k_attn_partial_tc<256>, cudaFuncAttributeMaxDynamicSharedMemorySize, fa::smem_bytes<256>());
  {
    const int dyn = kTdSmemLimit;
#define SQ_TD_ATTR(DD, MG) \
  cudaFuncSetAttribute(td::k_decode_tc<DD, MG>, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn)
    SQ_TD_ATTR(64, 2); SQ_TD_ATTR(64, 4); SQ_TD_ATTR(64, 8); SQ_TD_ATTR(64, 16);
    SQ_TD_ATTR(128, 2); SQ_TD_ATTR(128, 4); SQ_TD_ATTR(128, 8); SQ_TD_ATTR(128, 16);
    SQ_TD_ATTR(256, 2); SQ_TD_ATTR(256, 4); SQ_TD_ATTR(256, 8); SQ_TD_ATTR(256, 16);
#undef SQ_TD_ATTR
    const int ps = (int)prep_smem(kMaxD);
    cudaFuncSetAttribute(k_attn_prepare<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, ps);
    cudaFuncSetAttribute(k_attn_prepare<__half>, cudaFuncAttributeMaxDynamicSharedMemorySize, ps);
    cudaFuncSetAttribute(k_attn_prepare<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, ps);
#define SQ_SP_ATTR(T)                                                                          \
  cudaFuncSetAttribute(k_step_prep<T, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, ps);    \
  cudaFuncSetAttribute(k_step_prep<T, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, ps);    \
  cudaFuncSetAttribute(k_step_prep<T, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize, ps);    \
  cudaFuncSetAttribute(k_step_prep<T, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize, ps)
    SQ_SP_ATTR(float); SQ_SP_ATTR(__half); SQ_SP_ATTR(__nv_bfloat16);
#undef SQ_SP_ATTR
#define SQ_AP_ATTR(T)                                                                                          \
  cudaFuncSetAttribute(k_append<T, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)append_smem(1));     \
  cudaFuncSetAttribute(k_append<T, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)append_smem(2));     \
  cudaFuncSetAttribute(k_append<T, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)append_smem(4));     \
  cudaFuncSetAttribute(k_append<T, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)append_smem(8))
    SQ_AP_ATTR(float); SQ_AP_ATTR(__half); SQ_AP_ATTR(__nv_bfloat16);
#undef SQ_AP_ATTR
  }
  if (cuda_ok(cudaGetLastError()) != SQ_OK) return SQ_ERR_CUDA;
  int sms = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  g_sms[dev] = sms > 0 ? sms : 148;
  g_ready[dev] = true;
  return SQ_OK;
}

// Whole number of bits B = avg_bits * d, or -1.
int budget_bits(double avg_bits, int d) {
  double t = avg_bits * d;
  long r = lround(t);
  if (!(t > 0.0) || fabs(t - (double)r) > 1e-9 || r > (long)SQ_MAX_BITS * 256 + 256) return -1;
  return (int)r;
}

bool cache_ok(const sq_cache* c, int batch, int n_heads) {
  return c && c->codes && c->norm && aligned16(c->codes) && aligned16(c->norm) &&
         (!c->rnorm || aligned16(c->rnorm)) && c->batch == batch && c->n_heads == n_heads &&
         c->cap >= kBlockTok && c->cap % kBlockTok == 0 && c->words >= 1 && c->words <= kMaxWords;
}

CacheArgs cache_args(const sq_cache* c) { return CacheArgs{c->codes, c->norm, c->rnorm, c->cap, c->words}; }

// Splits of the context per (batch, KV head). Each block of the partial
// kernel takes a span of whole 128-token tiles (32 tokens per warp) and pays a
// fixed setup (tables, query fragments, final merge) of about half a warp tile.
// With `slots` blocks resident at once (the device's SMs, 148 on a B200, times
// the blocks per SM the kernel is built for), equal blocks run in ceil(blocks / slots) waves,
// so the cost of a split count S is waves(S) x (1/2 + tiles per warp); the
// cheapest S wins (the smaller on ties, which also keeps the combine short).
// SMs of the current device (its multiprocessor count; 148 on a B200, also the
// answer when no device can be queried, e.g. for a workspace query on a host
// without a GPU).
int device_sms() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) {
    cudaGetLastError();
    return 148;
  }
  if (g_ready[dev]) return g_sms[dev];
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) {
    cudaGetLastError();
    return 148;
  }
  return sms;
}

// tcgen05 decode kernel: the warp groups whose regions fit in shared memory
// (as many as the kernel has, else fewer) and the record buffers per group
// (2, else 1); ng = 0 when not even one group with one buffer fits.
int td_groups(int d) { return d == 64 ? td::Cfg<64>::NG : (d == 128 ? td::Cfg<128>::NG : td::Cfg<256>::NG); }
size_t td_smem(int d, int wk, int wv, int nrec, int ng) {
  return d == 64 ? td::smem_bytes<64>(wk, wv, nrec, ng)
                 : (d == 128 ? td::smem_bytes<128>(wk, wv, nrec, ng) : td::smem_bytes<256>(wk, wv, nrec, ng));
}
void td_config(int d, int wk, int wv, int* nrec_out, int* ng_out) {
  *nrec_out = 0;
  *ng_out = 0;
  for (int ng = td_groups(d); ng >= 1; --ng)
    for (int nrec = 2; nrec >= 1; --nrec)
      if (td_smem(d, wk, wv, nrec, ng) <= (size_t)kTdSmemLimit) {
        *nrec_out = nrec;
        *ng_out = ng;
        return;
      }
}

// Splits of the context for the tcgen05 kernel: one block per SM, whose NG
// warp groups take its 128-token tiles in turn. With equal blocks in
// ceil(blocks / SMs) waves, the cost of S splits is waves(S) x (1 + tiles per
// group), the 1 standing for the block's setup (tables, query operand, merge);
// the cheapest S wins (the smaller on ties).
int attn_splits_td(int batch, int n_kv, int64_t max_ctx, int ngroups) {
  const int64_t units = (int64_t)batch * n_kv;
  const int64_t slots = (int64_t)device_sms();
  const int64_t ctx = max_ctx > 0 ? max_ctx : 1;
  const int64_t ng = ngroups > 0 ? ngroups : 1;
  int best = 1;
  int64_t best_cost = INT64_MAX;
  for (int64_t S = 1; S <= 256; ++S) {
    const int64_t per = (ctx + S - 1) / S;
    const int64_t chunk = ((per + kAttnTile - 1) / kAttnTile) * kAttnTile;
    const int64_t used = (ctx + chunk - 1) / chunk;
    if (used != S) continue;
    const int64_t waves = (units * S + slots - 1) / slots;
    const int64_t tiles = chunk / kAttnTile;
    const int64_t cost = waves * (1 + (tiles + ng - 1) / ng);
    if (cost < best_cost) {
      best_cost = cost;
      best = (int)S;
    }
    if (chunk == kAttnTile) break;
  }
  return best;
}

int attn_splits(int batch, int n_kv, int d, int64_t max_ctx) {
  const int64_t units = (int64_t)batch * n_kv;
  const int64_t slots = (int64_t)device_sms() * fa::min_blocks(d);
  const int64_t ctx = max_ctx > 0 ? max_ctx : 1;
  int best = 1;
  int64_t best_cost = INT64_MAX;
  for (int64_t S = 1; S <= 256; ++S) {
    const int64_t per = (ctx + S - 1) / S;
    const int64_t chunk = ((per + kAttnTile - 1) / kAttnTile) * kAttnTile;
    const int64_t used = (ctx + chunk - 1) / chunk;        // splits that hold tokens
    if (used != S) continue;
    const int64_t waves = (units * S + slots - 1) / slots;
    const int64_t cost = waves * (1 + 2 * (chunk / kAttnTile));
    if (cost < best_cost) {
      best_cost = cost;
      best = (int)S;
    }
    if (chunk == kAttnTile) break;
  }
  return best;
}

// cuTensorMapEncodeTiled, looked up through the runtime so that libsq does not
// link libcuda (it must load on machines without a GPU driver).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (PFN_cuTensorMapEncodeTiled_v12000)p;
  });
  return fn;
}

// Tensor-core compress of one side (fp16, head_dim 128): X viewed as a 2-D
// [batch * n_heads * n_tok, 128] fp16 tensor read in 128 x 64 boxes.
sq_status launch_compress_tc(const void* recs, const void* x, int batch, int n_heads, int64_t n_tok,
                             const int32_t* sp, const sq_cache* c, uint32_t* flags, cudaStream_t st, int dev) {
  auto encode = tensor_map_encoder();
  if (!encode) return SQ_ERR_CUDA;
  const int64_t rows = (int64_t)batch * n_heads * n_tok;
  if (rows >= ((int64_t)1 << 31)) return SQ_ERR_ARG;
  CUtensorMap map;
  cuuint64_t dims[2] = {(cuuint64_t)tcc::D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)tcc::D * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)tcc::TILE};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(x), dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return SQ_ERR_CUDA;
  tcc::Params P;
  P.recs = (const uint8_t*)recs;
  P.x = (const __half*)x;
  P.n_heads = n_heads;
  P.batch = batch;
  P.n_tok = n_tok;
  P.start_pos = sp;
  P.c = cache_args(c);
  P.flags = flags;
  P.tiles_per_row = (int)((n_tok + tcc::TILE - 1) / tcc::TILE);
  P.eacc = (float)ldexp((double)g_eacc_units, -24);
  P.n_tiles = (int64_t)batch * n_heads * P.tiles_per_row;
  int64_t grid = P.n_tiles < g_sms[dev] ? P.n_tiles : g_sms[dev];
  tcc::k_compress_tc<<<(unsigned)grid, tcc::NUM_THREADS, tcc::SMEM_BYTES, st>>>(map, P, g_kq);
  if (cuda_ok(cudaGetLastError()) != SQ_OK) return SQ_ERR_CUDA;
  // Heads with more than tcc::MSIG QJL dimensions: the reference kernel, one
  // block per (batch, head); every other block returns at once.
  dim3 g2(1, n_heads, batch);
  k_compress_ref<__half><<<g2, 128, codec_ref_smem(tcc::D), st>>>((const uint8_t*)recs, (const __half*)x, n_heads,
                                                                tcc::D, n_tok, (int)n_tok, sp, cache_args(c), flags,
                                                                tcc::MSIG + 1);
  return cuda_ok(cudaGetLastError());
}

// Prompts of the shapes the tensor-core kernel does not take: the block-tiled
// float64 kernel (same bits as k_compress_ref).
template <typename T, int D>
sq_status launch_compress_blk(const void* recs, const void* x, int batch, int n_heads, int64_t n_tok,
                              const int32_t* sp, const sq_cache* c, uint32_t* flags, cudaStream_t st) {
  using G = blk::Geo<D>;
  const int64_t gx = (n_tok + G::NT - 1) / G::NT;
  if (gx > 0x7fffffff) return SQ_ERR_ARG;
  dim3 grid((unsigned)gx, n_heads, batch);
  blk::k_compress_blk<T, D><<<grid, blk::kThreads, G::SMEM, st>>>((const uint8_t*)recs, (const T*)x, n_heads, n_tok,
                                                                   sp, cache_args(c), flags);
  return cuda_ok(cudaGetLastError());
}

template <typename T>
sq_status launch_compress(const void* recs, const void* x, int batch, int n_heads, int d, int64_t n_tok,
                          const int32_t* sp, const sq_cache* c, uint32_t* flags, cudaStream_t st) {
  if (n_tok < 16) {      // appends: a block per (head, group of vectors)
    const int64_t nvec = (int64_t)batch * n_tok;
    const int nv = append_nv(nvec);
    const int64_t groups = (nvec + nv - 1) / nv;
    if (groups > 65535) return SQ_ERR_ARG;
    dim3 grid((unsigned)n_heads, (unsigned)groups);
    const uint8_t* r8 = (const uint8_t*)recs;
    const T* xt = (const T*)x;
    const CacheArgs ca = cache_args(c);
    switch (nv) {
      case 1: k_append<T, 1><<<grid, 256, append_smem(1), st>>>(r8, xt, batch, n_heads, d, n_tok, sp, ca, flags); break;
      case 2: k_append<T, 2><<<grid, 256, append_smem(2), st>>>(r8, xt, batch, n_heads, d, n_tok, sp, ca, flags); break;
      case 4: k_append<T, 4><<<grid, 256, append_smem(4), st>>>(r8, xt, batch, n_heads, d, n_tok, sp, ca, flags); break;
      default: k_append<T, 8><<<grid, 256, append_smem(8), st>>>(r8, xt, batch, n_heads, d, n_tok, sp, ca, flags); break;
    }
    return cuda_ok(cudaGetLastError());
  }
  if (!g_force_ref) {
    if (d == 64) return launch_compress_blk<T, 64>(recs, x, batch, n_heads, n_tok, sp, c, flags, st);
    if (d == 128) return launch_compress_blk<T, 128>(recs, x, batch, n_heads, n_tok, sp, c, flags, st);
    if (d == 256) return launch_compress_blk<T, 256>(recs, x, batch, n_heads, n_tok, sp, c, flags, st);
  }
  const int tpb = n_tok >= 1024 ? 256 : 64;
  const int64_t gx = (n_tok + tpb - 1) / tpb;
  if (gx > 0x7fffffff) return SQ_ERR_ARG;
  dim3 grid((unsigned)gx, n_heads, batch);
  k_compress_ref<T><<<grid, 128, codec_ref_smem(d), st>>>((const uint8_t*)recs, (const T*)x, n_heads, d, n_tok,
                                                          tpb, sp, cache_args(c), flags, 0);
  return cuda_ok(cudaGetLastError());
}

}  // namespace
}  // namespace sq

using namespace sq;

extern "C" {

int sq_abi_version(void) { return SQ_ABI_VERSION; }

const char* sq_last_error(void) { return g_last_err; }

const char* sq_status_str(sq_status s) {
  switch (s) {
    case SQ_OK: return "ok";
    case SQ_ERR_ARG: return "invalid argument";
    case SQ_ERR_UNSUPPORTED: return "unsupported head_dim or dtype";
    case SQ_ERR_CUDA: return "CUDA error";
    case SQ_ERR_NOT_CONVERGED: return "eigensolver did not converge within max_sweeps";
    case SQ_ERR_CAPACITY: return "cache capacity exceeded";
    case SQ_ERR_WORKSPACE: return "workspace too small";
    case SQ_ERR_RECORD: return "malformed calibration record";
  }
  return "unknown status";
}

size_t sq_calib_bytes(int d) { return supported_d(d) ? record_bytes(d) : 0; }

int sq_record_words(const sq_calib_params* p) {
  if (!p || !supported_d(p->d)) return 0;
  int bits = budget_bits(p->avg_bits, p->d);
  return bits < 0 ? 0 : (bits + 31) / 32;
}

sq_status sq_init(void) { return ensure_init(); }

sq_status sq_set_option(int option, int value) {
  if (option == SQ_OPT_COMPRESS_PATH && (value == 0 || value == 1)) {
    g_force_ref = value == 1;
    return SQ_OK;
  }
  if (option == SQ_OPT_ATTN_PATH && value >= 0 && value <= 2) {
    g_attn_path = value;
    return SQ_OK;
  }
  if (option == SQ_OPT_TC_ERROR_BOUND && value >= 0 && value <= (1 << 20)) {
    g_eacc_units = value;
    return SQ_OK;
  }
  return SQ_ERR_ARG;
}

size_t sq_calibrate_workspace(const sq_calib_params* p, int64_t n_tokens) {
  if (!p || !supported_d(p->d) || p->n_heads < 1 || n_tokens < 0) return 0;
  size_t b = (size_t)p->n_heads * 16u * (size_t)p->d * (size_t)p->d;
  if (p->codebooks == 1) b += (size_t)p->n_heads * (size_t)n_tokens * (size_t)p->d * 8u;   // z of the fit
  return b;
}

sq_status sq_calibrate(const sq_calib_params* p, const void* x, sq_dtype dtype, int64_t n_tokens,
                       int64_t stride_head, int64_t stride_tok, void* calib_out, void* ws, size_t ws_bytes,
                       int* d_status, sq_stream stream) {
  if (!p) return SQ_ERR_ARG;
  if (!supported_d(p->d)) return SQ_ERR_UNSUPPORTED;
  if (!valid_dtype(dtype)) return SQ_ERR_UNSUPPORTED;
  const int d = p->d;
  const int B = budget_bits(p->avg_bits, d);
  if (p->n_heads < 1 || B < 1 || p->max_bits < 1 || p->max_bits > SQ_MAX_BITS || p->d_eff_override < 0 ||
      p->d_eff_override > d || p->max_sweeps < 1 || !(p->tol > 0.0) || n_tokens < 1 || stride_tok < d ||
      stride_head < 0 || !x || !calib_out || ((uintptr_t)calib_out & 255u) || !ws || !aligned16(ws) ||
      (p->is_key != 0 && p->is_key != 1) || (p->qjl != 0 && p->qjl != 1) ||
      (p->normalize != 0 && p->normalize != 1) || (d_status && !aligned16(d_status)) || (B + 31) / 32 > kMaxWords ||
      (p->rotation != 0 && p->rotation != 1) || !(p->cumvar >= 0.0 && p->cumvar <= 1.0) ||
      (p->codebooks != 0 && p->codebooks != 1) || p->fit_iters < 0 || p->fit_iters > 100000 ||
      (p->codebooks == 1 && (p->n_heads > 65535 || (n_tokens + 7) / 8 > 0x7fffffff)))
    return SQ_ERR_ARG;
  if (ws_bytes < sq_calibrate_workspace(p, n_tokens)) return SQ_ERR_WORKSPACE;
  sq_status s = ensure_init();
  if (s != SQ_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  double* cov = (double*)ws;
  double* vt = cov + (size_t)p->n_heads * d * d;
  dim3 g1(p->n_heads, d / 32, d / 32), b1(32, 8);
  switch (dtype) {
    case SQ_F32: k_second_moment<float><<<g1, b1, 0, st>>>((const float*)x, d, n_tokens, stride_head, stride_tok, cov); break;
    case SQ_F16: k_second_moment<__half><<<g1, b1, 0, st>>>((const __half*)x, d, n_tokens, stride_head, stride_tok, cov); break;
    default: k_second_moment<__nv_bfloat16><<<g1, b1, 0, st>>>((const __nv_bfloat16*)x, d, n_tokens, stride_head, stride_tok, cov); break;
  }
  if (cuda_ok(cudaGetLastError()) != SQ_OK) return SQ_ERR_CUDA;
  if (p->rotation == 1) {
    k_random_basis<<<p->n_heads, 256, 0, st>>>(cov, vt, d, p->seed, calib_out, d_status);
  } else {
    size_t jsm = d <= 128 ? (size_t)8 * d * d : 0;
    k_jacobi<<<p->n_heads, 256, jsm, st>>>(cov, vt, d, p->max_sweeps, p->tol, calib_out, d_status);
  }
  if (cuda_ok(cudaGetLastError()) != SQ_OK) return SQ_ERR_CUDA;
  FinalizeArgs fa{B, p->is_key, p->qjl, p->normalize, p->d_eff_override, p->max_bits, p->seed, p->avg_bits,
                  p->cumvar, p->rotation, p->codebooks};
  k_finalize<<<p->n_heads, 256, 0, st>>>(calib_out, d, fa, d_status);
  if (cuda_ok(cudaGetLastError()) != SQ_OK) return SQ_ERR_CUDA;
  if (p->codebooks == 1) {
    double* z = vt + (size_t)p->n_heads * d * d;
    dim3 gz((unsigned)((n_tokens + 7) / 8), (unsigned)p->n_heads);
    switch (dtype) {
      case SQ_F32: k_fit_z<float><<<gz, 256, 0, st>>>((const float*)x, d, n_tokens, stride_head, stride_tok, calib_out, z); break;
      case SQ_F16: k_fit_z<__half><<<gz, 256, 0, st>>>((const __half*)x, d, n_tokens, stride_head, stride_tok, calib_out, z); break;
      default: k_fit_z<__nv_bfloat16><<<gz, 256, 0, st>>>((const __nv_bfloat16*)x, d, n_tokens, stride_head, stride_tok, calib_out, z); break;
    }
    if (cuda_ok(cudaGetLastError()) != SQ_OK) return SQ_ERR_CUDA;
    const int iters = p->fit_iters > 0 ? p->fit_iters : kFitIters;
    k_fit_lloyd<<<dim3((unsigned)p->n_heads, 2, SQ_MAX_BITS), 256, 0, st>>>(z, d, n_tokens, calib_out, iters);
  }
  return cuda_ok(cudaGetLastError());
}

sq_status sq_calib_import(void* calib, int n_heads, int d, int* d_status, sq_stream stream) {
  if (!supported_d(d)) return SQ_ERR_UNSUPPORTED;
  if (!calib || ((uintptr_t)calib & 255u) || n_heads < 1 || (d_status && !aligned16(d_status))) return SQ_ERR_ARG;
  sq_status s = ensure_init();
  if (s != SQ_OK) return s;
  k_import<<<n_heads, 256, 0, (cudaStream_t)stream>>>(calib, d, d_status);
  return cuda_ok(cudaGetLastError());
}

// One side of sq_compress_kv: the tensor-core path for fp16 head_dim-128
// prompts, the float64 reference kernels otherwise.
static sq_status compress_side(const void* recs, const void* x, sq_dtype dtype, int batch, int n_heads, int d,
                               int64_t n_tok, const int32_t* sp, const sq_cache* c, uint32_t* flags,
                               cudaStream_t st, int dev) {
  if (dtype == SQ_F16 && d == tcc::D && n_tok >= 64 && !g_force_ref)
    return launch_compress_tc(recs, x, batch, n_heads, n_tok, sp, c, flags, st, dev);
  switch (dtype) {
    case SQ_F32: return launch_compress<float>(recs, x, batch, n_heads, d, n_tok, sp, c, flags, st);
    case SQ_F16: return launch_compress<__half>(recs, x, batch, n_heads, d, n_tok, sp, c, flags, st);
    default: return launch_compress<__nv_bfloat16>(recs, x, batch, n_heads, d, n_tok, sp, c, flags, st);
  }
}

sq_status sq_compress_kv(const void* calib_k, const void* calib_v, const void* k, const void* v, sq_dtype dtype,
                         int batch, int n_heads, int d, int64_t n_tok, const int32_t* d_start_pos,
                         const sq_cache* kc, const sq_cache* vc, uint32_t* d_flags, sq_stream stream) {
  if (!supported_d(d) || !valid_dtype(dtype)) return SQ_ERR_UNSUPPORTED;
  if (batch < 1 || n_heads < 1 || n_tok < 0 || batch > 65535 || n_heads > 65535) return SQ_ERR_ARG;
  if (n_tok == 0) return SQ_OK;
  const bool do_k = k != nullptr, do_v = v != nullptr;
  if (!do_k && !do_v) return SQ_ERR_ARG;
  if (do_k && (!calib_k || ((uintptr_t)calib_k & 255u) || !aligned16(k) || !cache_ok(kc, batch, n_heads)))
    return SQ_ERR_ARG;
  if (do_v && (!calib_v || ((uintptr_t)calib_v & 255u) || !aligned16(v) || !cache_ok(vc, batch, n_heads)))
    return SQ_ERR_ARG;
  if (d_start_pos && !aligned16(d_start_pos)) return SQ_ERR_ARG;
  int dev = 0;
  sq_status s = ensure_init(&dev);
  if (s != SQ_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  for (int side = 0; side < 2; ++side) {
    const void* x = side == 0 ? k : v;
    if (!x) continue;
    s = compress_side(side == 0 ? calib_k : calib_v, x, dtype, batch, n_heads, d, n_tok, d_start_pos,
                      side == 0 ? kc : vc, d_flags, st, dev);
    if (s != SQ_OK) return s;
  }
  return SQ_OK;
}

namespace {
size_t dtype_bytes(sq_dtype t) { return t == SQ_F32 ? 4 : 2; }

// Bytes of one staging slab holding `heads` heads of one batch row.
size_t host_slab_bytes(int heads, int d, sq_dtype dtype, int64_t n_tok) {
  const size_t row = (size_t)n_tok * d * dtype_bytes(dtype);
  return ((size_t)heads * row + 255) & ~(size_t)255;
}

// The library's copy stream of each device (created on first use, never destroyed).
cudaStream_t g_copy_stream[128] = {};
sq_status copy_stream(int dev, cudaStream_t* out) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_copy_stream[dev] && cudaStreamCreateWithFlags(&g_copy_stream[dev], cudaStreamNonBlocking) != cudaSuccess) {
    g_copy_stream[dev] = nullptr;
    return SQ_ERR_CUDA;
  }
  *out = g_copy_stream[dev];
  return SQ_OK;
}
}  // namespace

size_t sq_compress_host_staging(int batch, int n_heads, int d, sq_dtype dtype, int64_t n_tok) {
  if (batch < 1 || n_heads < 1 || n_tok < 1 || !supported_d(d) || !valid_dtype(dtype)) return 0;
  const size_t row = (size_t)n_tok * d * dtype_bytes(dtype);
  size_t heads = ((size_t)16 << 20) / row + ((((size_t)16 << 20) % row) ? 1 : 0);
  if (heads < 1) heads = 1;
  if (heads > (size_t)n_heads) heads = (size_t)n_heads;
  return 2 * host_slab_bytes((int)heads, d, dtype, n_tok);
}

sq_status sq_compress_kv_host(const void* calib_k, const void* calib_v, const void* h_k, const void* h_v,
                              sq_dtype dtype, int batch, int n_heads, int d, int64_t n_tok,
                              const int32_t* d_start_pos, const sq_cache* kc, const sq_cache* vc,
                              void* d_staging, size_t staging_bytes, uint32_t* d_flags, sq_stream stream) {
  if (!supported_d(d) || !valid_dtype(dtype)) return SQ_ERR_UNSUPPORTED;
  if (batch < 1 || n_heads < 1 || n_tok < 0 || batch > 65535 || n_heads > 65535) return SQ_ERR_ARG;
  if (n_tok == 0) return SQ_OK;
  const bool do_k = h_k != nullptr, do_v = h_v != nullptr;
  if (!do_k && !do_v) return SQ_ERR_ARG;
  if (do_k && (!calib_k || ((uintptr_t)calib_k & 255u) || !cache_ok(kc, batch, n_heads))) return SQ_ERR_ARG;
  if (do_v && (!calib_v || ((uintptr_t)calib_v & 255u) || !cache_ok(vc, batch, n_heads))) return SQ_ERR_ARG;
  if ((d_start_pos && !aligned16(d_start_pos)) || !d_staging || ((uintptr_t)d_staging & 255u)) return SQ_ERR_ARG;
  // pieces of hc whole heads of one batch row, two slabs
  const size_t row = (size_t)n_tok * d * dtype_bytes(dtype);
  const size_t half = (staging_bytes / 2) & ~(size_t)255;
  size_t hc = half / row;
  if (hc < 1) return SQ_ERR_WORKSPACE;
  if (hc > (size_t)n_heads) hc = (size_t)n_heads;
  const size_t slab = host_slab_bytes((int)hc, d, dtype, n_tok);   // <= half
  int dev = 0;
  sq_status s = ensure_init(&dev);
  if (s != SQ_OK) return s;
  cudaStream_t st = (cudaStream_t)stream, cs = nullptr;
  if ((s = copy_stream(dev, &cs)) != SQ_OK) return s;
  cudaEvent_t ev[5] = {};   // fork, copied[2], free[2]
  for (auto& e : ev)
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
      for (auto& f : ev)
        if (f) cudaEventDestroy(f);
      return SQ_ERR_CUDA;
    }
  cudaEvent_t fork = ev[0], copied[2] = {ev[1], ev[2]}, freed[2] = {ev[3], ev[4]};
  s = (cudaEventRecord(fork, st) == cudaSuccess && cudaStreamWaitEvent(cs, fork, 0) == cudaSuccess) ? SQ_OK
                                                                                                       : SQ_ERR_CUDA;
  int64_t piece = 0;
  for (int side = 0; side < 2 && s == SQ_OK; ++side) {
    const uint8_t* hx = (const uint8_t*)(side == 0 ? h_k : h_v);
    if (!hx) continue;
    const void* recs = side == 0 ? calib_k : calib_v;
    const sq_cache* c = side == 0 ? kc : vc;
    for (int b = 0; b < batch && s == SQ_OK; ++b) {
      for (int h0 = 0; h0 < n_heads && s == SQ_OK; h0 += (int)hc, ++piece) {
        const int hn = (int)((size_t)(n_heads - h0) < hc ? (size_t)(n_heads - h0) : hc);
        const int slot = (int)(piece & 1);
        uint8_t* dx = (uint8_t*)d_staging + (size_t)slot * slab;
        const size_t row0 = (size_t)b * n_heads + h0;
        // the slab is free once the compression of the piece two back has run
        if (piece >= 2 && cudaStreamWaitEvent(cs, freed[slot], 0) != cudaSuccess) { s = SQ_ERR_CUDA; break; }
        if (cudaMemcpyAsync(dx, hx + row0 * row, (size_t)hn * row, cudaMemcpyHostToDevice, cs) != cudaSuccess ||
            cudaEventRecord(copied[slot], cs) != cudaSuccess || cudaStreamWaitEvent(st, copied[slot], 0) != cudaSuccess) {
          s = SQ_ERR_CUDA;
          break;
        }
        sq_cache view = *c;
        view.codes = c->codes + row0 * (size_t)c->cap * c->words;
        view.norm = c->norm + row0 * (size_t)c->cap;
        view.rnorm = c->rnorm ? c->rnorm + row0 * (size_t)c->cap : nullptr;
        view.batch = 1;
        view.n_heads = hn;
        const uint8_t* rh = (const uint8_t*)recs + (size_t)h0 * record_bytes(d);
        s = compress_side(rh, dx, dtype, 1, hn, d, n_tok, d_start_pos ? d_start_pos + b : nullptr, &view, d_flags,
                          st, dev);
        if (s == SQ_OK && cudaEventRecord(freed[slot], st) != cudaSuccess) s = SQ_ERR_CUDA;
      }
    }
  }
  for (auto& e : ev) cudaEventDestroy(e);   // released once their work has completed
  return s;
}

sq_status sq_decompress_kv(const void* calib, const sq_cache* cache, int d, int64_t t0, int64_t n_tok,
                           int apply_qjl, float* out, uint32_t* d_flags, sq_stream stream) {
  if (!supported_d(d)) return SQ_ERR_UNSUPPORTED;
  if (!cache) return SQ_ERR_ARG;
  if (!calib || ((uintptr_t)calib & 255u) || !out || !aligned16(out) || t0 < 0 || n_tok < 0 ||
      !cache_ok(cache, cache->batch, cache->n_heads) || cache->batch < 1 || cache->n_heads < 1 ||
      cache->batch > 65535 || cache->n_heads > 65535)
    return SQ_ERR_ARG;
  if (n_tok == 0) return SQ_OK;
  sq_status s = ensure_init();
  if (s != SQ_OK) return s;
  const int tpb = n_tok >= 1024 ? 256 : 64;
  dim3 grid((unsigned)((n_tok + tpb - 1) / tpb), cache->n_heads, cache->batch);
  k_decompress_ref<<<grid, 128, codec_ref_smem(d), (cudaStream_t)stream>>>(
      (const uint8_t*)calib, cache->n_heads, d, cache_args(cache), t0, n_tok, tpb, apply_qjl, out, d_flags);
  return cuda_ok(cudaGetLastError());
}

size_t sq_attn_workspace(int batch, int n_q_heads, int n_kv_heads, int d, int64_t max_ctx) {
  if (batch < 1 || n_q_heads < 1 || n_kv_heads < 1 || !supported_d(d) || max_ctx < 0) return 0;
  // enough for whichever partial kernel the call picks (that depends on the records)
  int s = attn_splits(batch, n_kv_heads, d, max_ctx);
  for (int ng = 1; ng <= td_groups(d); ++ng) s = std::max(s, attn_splits_td(batch, n_kv_heads, max_ctx, ng));
  return attn_ws_bytes(batch, n_q_heads, n_kv_heads, d, s);
}

}  // extern "C"

namespace {

bool attn_args_ok(const void* calib_k, const void* calib_v, const sq_cache* kc, const sq_cache* vc,
                  const int32_t* d_lens, int batch, int n_q_heads, int n_kv_heads, const void* q, const void* out,
                  const float* scores_out, const void* ws) {
  return !(batch < 1 || batch > 65535 || n_q_heads < 1 || n_kv_heads < 1 || n_kv_heads > 65535 ||
           n_q_heads % n_kv_heads != 0 || n_q_heads / n_kv_heads > kAttnMaxG || n_q_heads > 65535 || !calib_k ||
           !calib_v || ((uintptr_t)calib_k & 255u) || ((uintptr_t)calib_v & 255u) ||
           !cache_ok(kc, batch, n_kv_heads) || !cache_ok(vc, batch, n_kv_heads) || !d_lens || !aligned16(d_lens) ||
           !q || !aligned16(q) || !out || !aligned16(out) || (scores_out && !aligned16(scores_out)) || !ws ||
           !aligned16(ws));
}

// Every launch of one decode-attention call. With k_new / v_new (a decode
// step) the new token of each row is first compressed into the caches at
// d_lens[b] and attended (len_offset 1). The tcgen05 path takes three
// launches (append + prepare in one; partials with the last-block merge; the
// rotation back batched over the rows of each KV head); the others take
// prepare, partials and combine (and the appends before them).
// Query positions per kernel row of a causal prefill with qg query heads per
// KV head: as many as fit 16 MMA columns.
int prefill_cols(int qg) { return qg >= 16 ? 1 : 16 / qg; }

template <typename TQ>
sq_status attn_launch(const void* calib_k, const void* calib_v, const sq_cache* kc, const sq_cache* vc,
                      const int32_t* d_lens, int len_offset, int batch, int n_q_heads, int n_kv_heads, int d,
                      int64_t max_ctx, const void* q, float scale, void* out, sq_dtype out_dtype, float* scores_out,
                      void* ws, uint32_t* d_flags, cudaStream_t st, const void* k_new, const void* v_new, int dev,
                      int n_qtok = 0) {
  // causal prefill when n_qtok > 0: kernel rows (batch row, block of positions), columns (position, head)
  const int qg = n_q_heads / n_kv_heads;
  const bool causal = n_qtok > 0;
  const int pcols = causal ? prefill_cols(qg) : 1;
  const int ncb = causal ? (n_qtok + pcols - 1) / pcols : 1;
  const int group = qg * pcols;
  const int rows = batch * ncb;
  int nrec = 0, ngs = 0;
  td_config(d, kc->words, vc->words, &nrec, &ngs);
  const bool use_td = g_attn_path == 0 && (d == 64 || d == 128 || d == 256) && group <= 16 && nrec > 0;
  AttnShape sh;
  sh.batch = rows;
  sh.n_q = n_kv_heads * group;
  sh.n_kv = n_kv_heads;
  sh.group = group;
  sh.d = d;
  sh.causal = causal ? 1 : 0;
  sh.pcols = pcols;
  sh.ncb = ncb;
  sh.qg = qg;
  sh.n_qtok = n_qtok;
  sh.splits = use_td ? attn_splits_td(rows, n_kv_heads, max_ctx, ngs) : attn_splits(rows, n_kv_heads, d, max_ctx);
  sh.max_ctx = max_ctx;
  sh.len_offset = len_offset;
  int64_t per = (max_ctx + sh.splits - 1) / sh.splits;
  sh.chunk = ((per + kAttnTile - 1) / kAttnTile) * kAttnTile;
  if (sh.chunk < kAttnTile) sh.chunk = kAttnTile;
  const float sc = scale > 0.0f ? scale : 1.0f / sqrtf((float)d);
  float* w = (float*)ws;
  const uint8_t* rk = (const uint8_t*)calib_k;
  const uint8_t* rv = (const uint8_t*)calib_v;
  CacheArgs ka = cache_args(kc), va = cache_args(vc);
  const int prow = prep_rows(group);
  const unsigned n_prep = (unsigned)(n_kv_heads * ((rows + prow - 1) / prow));
  // ---- launch 1: prepare (with the appends of a decode step)
  if (k_new && use_td) {
    const int nv = append_nv(batch);
    const int64_t n_app = (int64_t)n_kv_heads * ((batch + nv - 1) / nv);
    const int64_t blocks = 2 * n_app + n_prep;
    if (blocks > 0x7fffffff) return SQ_ERR_ARG;
    const size_t ps = prep_smem(kMaxD);
    const TQ* kn = (const TQ*)k_new;
    const TQ* vn = (const TQ*)v_new;
    const TQ* qq = (const TQ*)q;
    switch (nv) {
      case 1: k_step_prep<TQ, 1><<<(unsigned)blocks, 256, ps, st>>>(rk, rv, kn, vn, qq, batch, n_kv_heads, d, d_lens, ka, va, sh, sc, w, d_flags, (int)n_app); break;
      case 2: k_step_prep<TQ, 2><<<(unsigned)blocks, 256, ps, st>>>(rk, rv, kn, vn, qq, batch, n_kv_heads, d, d_lens, ka, va, sh, sc, w, d_flags, (int)n_app); break;
      case 4: k_step_prep<TQ, 4><<<(unsigned)blocks, 256, ps, st>>>(rk, rv, kn, vn, qq, batch, n_kv_heads, d, d_lens, ka, va, sh, sc, w, d_flags, (int)n_app); break;
      default: k_step_prep<TQ, 8><<<(unsigned)blocks, 256, ps, st>>>(rk, rv, kn, vn, qq, batch, n_kv_heads, d, d_lens, ka, va, sh, sc, w, d_flags, (int)n_app); break;
    }
  } else {
    if (k_new) {
      sq_status s = launch_compress<TQ>(calib_k, k_new, batch, n_kv_heads, d, 1, d_lens, kc, d_flags, st);
      if (s == SQ_OK) s = launch_compress<TQ>(calib_v, v_new, batch, n_kv_heads, d, 1, d_lens, vc, d_flags, st);
      if (s != SQ_OK) return s;
    }
    dim3 gp(n_kv_heads, (unsigned)((rows + prow - 1) / prow));
    k_attn_prepare<TQ><<<gp, 256, prep_smem(d), st>>>(rk, (const TQ*)q, sh, sc, w, d_flags);
  }
  if (cuda_ok(cudaGetLastError()) != SQ_OK) return SQ_ERR_CUDA;
  // ---- launch 2: partials (the tcgen05 kernel merges the splits itself)
  if (rows > 65535) return SQ_ERR_ARG;
  dim3 gpart(sh.splits, n_kv_heads, rows);
  size_t smem = attn_partial_smem(d, sh.group, kc->words, vc->words);
  const bool fast = !causal && g_attn_path != 1 && sh.group <= 8 && (d == 64 || d == 128 || d == 256) &&
                    kc->words <= d / 8 && vc->words <= d / 8;
  if (use_td) {
    const int MGv = sh.group <= 2 ? 2 : (sh.group <= 4 ? 4 : (sh.group <= 8 ? 8 : 16));
#define SQ_TD_LAUNCH(DD, MG)                                                                                  \
  td::k_decode_tc<DD, MG><<<gpart, td::Cfg<DD>::NTH, td::smem_bytes<DD>(kc->words, vc->words, nrec, ngs), st>>>( \
      rk, rv, ka, va, d_lens, sh, w, scores_out, d_flags, nrec, ngs)
#define SQ_TD_G(DD)                                                                                       \
  if (MGv == 2) SQ_TD_LAUNCH(DD, 2); else if (MGv == 4) SQ_TD_LAUNCH(DD, 4); else if (MGv == 8) SQ_TD_LAUNCH(DD, 8); \
  else SQ_TD_LAUNCH(DD, 16)
    if (d == 64) { SQ_TD_G(64); }
    else if (d == 128) { SQ_TD_G(128); }
    else { SQ_TD_G(256); }
#undef SQ_TD_G
#undef SQ_TD_LAUNCH
    if (cuda_ok(cudaGetLastError()) != SQ_OK) return SQ_ERR_CUDA;
    // ---- launch 3: the rotation back (o = V_V a), batched over the rows of each KV head
    const int64_t nvec = (int64_t)rows * sh.group;
    dim3 gr(n_kv_heads, (unsigned)std::min<int64_t>(65535, (nvec + 31) / 32));
    if (d == 64) k_rotate_out<64><<<gr, 256, 0, st>>>(rv, sh, w, out, (int)out_dtype);
    else if (d == 128) k_rotate_out<128><<<gr, 256, 0, st>>>(rv, sh, w, out, (int)out_dtype);
    else k_rotate_out<256><<<gr, 256, 0, st>>>(rv, sh, w, out, (int)out_dtype);
    return cuda_ok(cudaGetLastError());
  }
  if (fast) {
    if (d == 64)
      fa::k_attn_partial_tc<64><<<gpart, fa::NTH, fa::smem_bytes<64>(), st>>>(rk, rv, ka, va, d_lens, sh, w,
                                                                            scores_out, d_flags);
    else if (d == 128)
      fa::k_attn_partial_tc<128><<<gpart, fa::NTH, fa::smem_bytes<128>(), st>>>(rk, rv, ka, va, d_lens, sh, w,
                                                                              scores_out, d_flags);
    else
      fa::k_attn_partial_tc<256><<<gpart, fa::NTH, fa::smem_bytes<256>(), st>>>(rk, rv, ka, va, d_lens, sh, w,
                                                                              scores_out, d_flags);
  } else if (sh.group <= 1)
    k_attn_partial<1><<<gpart, 128, smem, st>>>(rk, rv, ka, va, d_lens, sh, w, scores_out, d_flags);
  else if (sh.group <= 2)
    k_attn_partial<2><<<gpart, 128, smem, st>>>(rk, rv, ka, va, d_lens, sh, w, scores_out, d_flags);
  else if (sh.group <= 4)
    k_attn_partial<4><<<gpart, 128, smem, st>>>(rk, rv, ka, va, d_lens, sh, w, scores_out, d_flags);
  else if (sh.group <= 8)
    k_attn_partial<8><<<gpart, 128, smem, st>>>(rk, rv, ka, va, d_lens, sh, w, scores_out, d_flags);
  else
    k_attn_partial<16><<<gpart, 128, smem, st>>>(rk, rv, ka, va, d_lens, sh, w, scores_out, d_flags);
  if (cuda_ok(cudaGetLastError()) != SQ_OK) return SQ_ERR_CUDA;
  // ---- launch 3: combine
  dim3 gc(n_kv_heads, rows);
  k_attn_combine<<<gc, 256, combine_scratch_floats(d, sh.splits) * 4, st>>>(rv, sh, w, out, (int)out_dtype);
  (void)dev;
  return cuda_ok(cudaGetLastError());
}

sq_status attn_dispatch(const void* calib_k, const void* calib_v, const sq_cache* kc, const sq_cache* vc,
                        const int32_t* d_lens, int len_offset, int batch, int n_q_heads, int n_kv_heads, int d,
                        int64_t max_ctx, const void* q, sq_dtype dtype, float scale, void* out, sq_dtype out_dtype,
                        float* scores_out, void* ws, uint32_t* d_flags, cudaStream_t st, const void* k_new,
                        const void* v_new, int dev, int n_qtok = 0) {
  switch (dtype) {
    case SQ_F32:
      return attn_launch<float>(calib_k, calib_v, kc, vc, d_lens, len_offset, batch, n_q_heads, n_kv_heads, d,
                                max_ctx, q, scale, out, out_dtype, scores_out, ws, d_flags, st, k_new, v_new, dev,
                                n_qtok);
    case SQ_F16:
      return attn_launch<__half>(calib_k, calib_v, kc, vc, d_lens, len_offset, batch, n_q_heads, n_kv_heads, d,
                                 max_ctx, q, scale, out, out_dtype, scores_out, ws, d_flags, st, k_new, v_new, dev,
                                 n_qtok);
    default:
      return attn_launch<__nv_bfloat16>(calib_k, calib_v, kc, vc, d_lens, len_offset, batch, n_q_heads, n_kv_heads,
                                        d, max_ctx, q, scale, out, out_dtype, scores_out, ws, d_flags, st, k_new,
                                        v_new, dev, n_qtok);
  }
}

}  // namespace

extern "C" {

sq_status sq_attn_decode(const void* calib_k, const void* calib_v, const sq_cache* kc, const sq_cache* vc,
                         const int32_t* d_seq_lens, int batch, int n_q_heads, int n_kv_heads, int d,
                         int64_t max_ctx, const void* q, sq_dtype q_dtype, float scale, void* out,
                         sq_dtype out_dtype, float* scores_out, void* ws, size_t ws_bytes, uint32_t* d_flags,
                         sq_stream stream) {
  if (!supported_d(d) || !valid_dtype(q_dtype) || !valid_dtype(out_dtype)) return SQ_ERR_UNSUPPORTED;
  if (max_ctx < 0 ||
      !attn_args_ok(calib_k, calib_v, kc, vc, d_seq_lens, batch, n_q_heads, n_kv_heads, q, out, scores_out, ws))
    return SQ_ERR_ARG;
  if (ws_bytes < sq_attn_workspace(batch, n_q_heads, n_kv_heads, d, max_ctx)) return SQ_ERR_WORKSPACE;
  int dev = 0;
  sq_status s = ensure_init(&dev);
  if (s != SQ_OK) return s;
  return attn_dispatch(calib_k, calib_v, kc, vc, d_seq_lens, 0, batch, n_q_heads, n_kv_heads, d, max_ctx, q, q_dtype,
                       scale, out, out_dtype, scores_out, ws, d_flags, (cudaStream_t)stream, nullptr, nullptr, dev);
}

sq_status sq_decode_step(const void* calib_k, const void* calib_v, const sq_cache* kc, const sq_cache* vc,
                         const void* k_new, const void* v_new, const void* q, sq_dtype dtype, const int32_t* d_pos,
                         int batch, int n_q_heads, int n_kv_heads, int d, int64_t max_ctx, float scale, void* out,
                         sq_dtype out_dtype, float* scores_out, void* ws, size_t ws_bytes, uint32_t* d_flags,
                         sq_stream stream) {
  if (!supported_d(d) || !valid_dtype(dtype) || !valid_dtype(out_dtype)) return SQ_ERR_UNSUPPORTED;
  if (max_ctx < 1 || !k_new || !v_new || !aligned16(k_new) || !aligned16(v_new) ||
      !attn_args_ok(calib_k, calib_v, kc, vc, d_pos, batch, n_q_heads, n_kv_heads, q, out, scores_out, ws))
    return SQ_ERR_ARG;
  if (ws_bytes < sq_attn_workspace(batch, n_q_heads, n_kv_heads, d, max_ctx)) return SQ_ERR_WORKSPACE;
  int dev = 0;
  sq_status s = ensure_init(&dev);
  if (s != SQ_OK) return s;
  return attn_dispatch(calib_k, calib_v, kc, vc, d_pos, 1, batch, n_q_heads, n_kv_heads, d, max_ctx, q, dtype, scale,
                       out, out_dtype, scores_out, ws, d_flags, (cudaStream_t)stream, k_new, v_new, dev);
}

size_t sq_attn_prefill_workspace(int batch, int n_q_heads, int n_kv_heads, int d, int64_t n_qtok, int64_t max_ctx) {
  if (batch < 1 || n_q_heads < 1 || n_kv_heads < 1 || n_q_heads % n_kv_heads || !supported_d(d) || n_qtok < 1 ||
      max_ctx < 1)
    return 0;
  const int qg = n_q_heads / n_kv_heads;
  const int pcols = prefill_cols(qg);
  const int64_t rows = (int64_t)batch * ((n_qtok + pcols - 1) / pcols);
  if (rows > 65535) return 0;
  int s = attn_splits((int)rows, n_kv_heads, d, max_ctx);
  for (int ng = 1; ng <= td_groups(d); ++ng) s = std::max(s, attn_splits_td((int)rows, n_kv_heads, max_ctx, ng));
  return attn_ws_bytes((int)rows, n_kv_heads * qg * pcols, n_kv_heads, d, s);
}

sq_status sq_attn_prefill(const void* calib_k, const void* calib_v, const sq_cache* kc, const sq_cache* vc,
                          const int32_t* d_start, int batch, int n_q_heads, int n_kv_heads, int d, int64_t n_qtok,
                          int64_t max_ctx, const void* q, sq_dtype q_dtype, float scale, void* out, sq_dtype out_dtype,
                          void* ws, size_t ws_bytes, uint32_t* d_flags, sq_stream stream) {
  if (!supported_d(d) || !valid_dtype(q_dtype) || !valid_dtype(out_dtype)) return SQ_ERR_UNSUPPORTED;
  if (n_qtok < 1 || n_qtok > 0x7fffffff || max_ctx < n_qtok ||
      !attn_args_ok(calib_k, calib_v, kc, vc, d_start, batch, n_q_heads, n_kv_heads, q, out, nullptr, ws))
    return SQ_ERR_ARG;
  const size_t need = sq_attn_prefill_workspace(batch, n_q_heads, n_kv_heads, d, n_qtok, max_ctx);
  if (need == 0) return SQ_ERR_ARG;
  if (ws_bytes < need) return SQ_ERR_WORKSPACE;
  int dev = 0;
  sq_status s = ensure_init(&dev);
  if (s != SQ_OK) return s;
  return attn_dispatch(calib_k, calib_v, kc, vc, d_start, 0, batch, n_q_heads, n_kv_heads, d, max_ctx, q, q_dtype,
                       scale, out, out_dtype, nullptr, ws, d_flags, (cudaStream_t)stream, nullptr, nullptr, dev,
                       (int)n_qtok);
}

// ---------------------------------------------------------------------------
// Decode attention without a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they run decode
// attention: a serving loop whose device memory is reserved once at start-up
// and may not grow, plug-ins that have no handle to the host application's
// allocator, and runtimes that forbid allocation after initialisation. They use
// this entry point: its scratch is a fixed array in the library's own device
// memory (every GPU that loads libsq keeps it until the process exits).
// ---------------------------------------------------------------------------
}  // extern "C"

namespace sq {
// A bounded wait that runs out: one thread waits on an mbarrier that nothing
// arrives on, through the same helper (sm100::mbar_wait) every tensor-core
// kernel waits with, here with a short limit; it gives up, sets the timeout
// flag and returns.
__global__ void k_wait_selftest(uint64_t limit_ns, uint32_t* flags) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1u);
    sm100::fence_mbar_init();
    (void)sm100::mbar_wait(&bar, 0u, flags, limit_ns);
  }
}
}  // namespace sq

extern "C" {

constexpr size_t kStaticScratchBytes = SQ_ATTN_NOALLOC_MAX_BYTES;
static __device__ __align__(256) unsigned char g_attn_scratch[kStaticScratchBytes];
static void* g_attn_scratch_addr[128];     // device address of the array, per device

sq_status sq_attn_decode_noalloc(const void* calib_k, const void* calib_v, const sq_cache* kc, const sq_cache* vc,
                                 const int32_t* d_seq_lens, int batch, int n_q_heads, int n_kv_heads, int d,
                                 int64_t max_ctx, const void* q, sq_dtype q_dtype, float scale, void* out,
                                 sq_dtype out_dtype, float* scores_out, uint32_t* d_flags, sq_stream stream) {
  const size_t need = sq_attn_workspace(batch, n_q_heads, n_kv_heads, d, max_ctx);
  if (need == 0) return supported_d(d) ? SQ_ERR_ARG : SQ_ERR_UNSUPPORTED;
  if (need > kStaticScratchBytes) return SQ_ERR_WORKSPACE;
  int dev = 0;
  sq_status s = ensure_init(&dev);
  if (s != SQ_OK) return s;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_attn_scratch_addr[dev]) {
      // The symbol's name is a host-side stand-in; the kernels need the device
      // address of this device's copy, taken with this device current.
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_attn_scratch) != cudaSuccess || !p) return SQ_ERR_CUDA;
      g_attn_scratch_addr[dev] = p;
    }
  }
  return sq_attn_decode(calib_k, calib_v, kc, vc, d_seq_lens, batch, n_q_heads, n_kv_heads, d, max_ctx, q, q_dtype,
                        scale, out, out_dtype, scores_out, g_attn_scratch_addr[dev], kStaticScratchBytes, d_flags,
                        stream);
}

sq_status sq_wait_selftest(uint32_t limit_us, uint32_t* d_flags, sq_stream stream) {
  if (limit_us < 1 || limit_us > 2000000u || !d_flags || !aligned16(d_flags)) return SQ_ERR_ARG;
  sq_status s = ensure_init();
  if (s != SQ_OK) return s;
  k_wait_selftest<<<1, 32, 0, (cudaStream_t)stream>>>((uint64_t)limit_us * 1000ull, d_flags);
  return cuda_ok(cudaGetLastError());
}

}  // extern "C"
