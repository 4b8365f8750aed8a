/*
 * sq.h -- C ABI of libsq, a CUDA (sm_100a) implementation of the SpectralQuant
 * compressed-KV hot path: per-head calibration, compression of keys and values
 * into packed records, decompression, and decode attention straight from the
 * packed cache.
 *
 * The method is described by the SpectralQuant README (Dynamis-Labs/spectralquant):
 *   - "Overview": keys concentrate their signal in 3-4 % of head_dim; a one-time
 *     calibration finds those dimensions and error correction is dropped on the
 *     remaining noise dimensions;
 *   - "Repository Structure": calibration.py (eigenspectral calibration: PCA,
 *     d_eff, kappa), spectral_rotation.py (rotation into the calibrated basis),
 *     nonuniform_quantization.py (Lloyd-Max codebooks), selective_qjl.py (QJL
 *     correction on the signal dims only);
 *   - title: "Calibrated Eigenbasis Rotation and Water-Filled Bit Allocation";
 *   - "Headline Results": compression ratio by bit accounting, decode latency
 *     per step over the compressed cache;
 * and by the v1 tests/conftest.py fixture pre_computed_calibration (uncentred
 * second moment, eigh, descending order, participation-ratio d_eff, gap).
 *
 * Conventions (all entry points)
 * ------------------------------
 *  - The caller owns all memory. libsq never allocates device memory; calls
 *    that need scratch take a workspace pointer and a size, with a matching
 *    *_workspace() query.
 *  - Device pointers are plain CUDA device addresses; "host" arguments are
 *    plain host memory. Every call that launches work is asynchronous on the
 *    given stream and returns once the work is queued.
 *  - Argument errors are reported synchronously, before any launch:
 *    SQ_ERR_ARG (bad value / null / misaligned pointer), SQ_ERR_UNSUPPORTED
 *    (head_dim not in {32, 64, 128, 256}, or a dtype a call does not take),
 *    SQ_ERR_WORKSPACE (workspace too small). A failed launch returns SQ_ERR_CUDA.
 *  - Conditions only the device can see (a capacity overflow, a record that
 *    does not match the cache, a sequence length past the context bound, a
 *    pipeline wait that timed out) are
 *    OR-ed into the optional device word d_flags (SQ_FLAG_*), and the affected
 *    rows are skipped; the call still returns SQ_OK. No kernel traps.
 *  - Pointers to device arrays must be 16-byte aligned. Strides are in elements.
 *  - The library keeps per-device constant tables (the Lloyd-Max codebooks). The
 *    first launching call on a device uploads them, so make one call (or
 *    sq_init) before capturing a stream into a CUDA graph.
 */
#ifndef SQ_H
#define SQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* sq_stream; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
  SQ_OK = 0,
  SQ_ERR_ARG = 1,
  SQ_ERR_UNSUPPORTED = 2,
  SQ_ERR_CUDA = 3,
  SQ_ERR_NOT_CONVERGED = 4, /* per-head status of sq_calibrate: eigensolver hit max_sweeps */
  SQ_ERR_CAPACITY = 5,
  SQ_ERR_WORKSPACE = 6,
  SQ_ERR_RECORD = 7          /* per-head status: malformed calibration record */
} sq_status;

typedef enum { SQ_F32 = 0, SQ_F16 = 1, SQ_BF16 = 2 } sq_dtype;

/* Bits of the device flag word. */
#define SQ_FLAG_CAPACITY 1u   /* start_pos + n_tok > cap (or start_pos < 0): row skipped */
#define SQ_FLAG_RECORD 2u     /* record magic/version/d/words do not match the call      */
#define SQ_FLAG_SEQLEN 4u     /* seq_len > max_ctx or > cap, or < 0: row clamped          */
/* A pipeline wait of the tensor-core compress (an mbarrier phase that did not
 * complete within 2 s) gave up: the kernel stopped its remaining tiles, drained
 * the copies it had issued, freed its tensor memory and returned; the records
 * of those tiles are not written. */
#define SQ_FLAG_TIMEOUT 0x80000000u

#define SQ_MAX_BITS 8         /* largest code width of one coordinate                     */
#define SQ_ABI_VERSION 3   /* 2: word-interleaved 32-token blocks in sq_cache.codes;
                              3: records of version 2 (fitted-codebook section),
                                 sq_calib_params.codebooks and .fit_iters */

/*
 * Calibration parameters (host struct).
 *  d              head_dim: 32, 64, 128 or 256.
 *  n_heads        heads calibrated by one call (e.g. layers x KV heads).
 *  avg_bits       bits per coordinate; B = avg_bits * d must be a whole number
 *                 (the record's total bits, QJL bits included).
 *  is_key         1 for keys (QJL allowed), 0 for values.
 *  qjl            1: keys store m = d_eff QJL sign bits inside the B bits.
 *  normalize      1: quantize x/||x|| and store ||x|| (default reading);
 *                 0: quantize x itself with sigma_i = sqrt(lambda_i).
 *  d_eff_override 0: m = the participation-ratio d_eff; > 0: m = this value.
 *  max_bits       cap on one coordinate's code width (1..8).
 *  seed           seed of the QJL Gaussian streams; head h of the call uses
 *                 stream h (SplitMix64 state mix(seed ^ mix(h + 1)), 53-bit
 *                 uniforms in (0,1], Box-Muller pairs).
 *  max_sweeps     eigensolver sweep limit (e.g. 30).
 *  tol            eigensolver stop: off-diagonal Frobenius norm <= tol * ||C||_F.
 *  rotation       0: the calibrated eigenbasis (the method); 1: a random
 *                 rotation, the A/B baseline of the README's
 *                 spectral_rotation.py ("spectral rotation vs random rotation
 *                 baseline"): Q of the QR factorisation (diag R > 0) of a d x d
 *                 matrix of N(0,1) draws, row-major, from the stream of seed
 *                 seed ^ 0x524F54 and the head's index (SplitMix64 / Box-Muller
 *                 as for the QJL matrix), its columns ordered by descending
 *                 variance q^T C q, which takes the place of lambda.
 *  cumvar         0: d_eff is the participation ratio; in (0, 1]: d_eff is the
 *                 smallest k >= 1 whose top-k lambda hold at least this fraction
 *                 of the trace (the README's results/deff_sweep/ compares
 *                 "participation ratio vs cumvar").
 *  codebooks      0: every coordinate is coded with the shared unit-Gaussian
 *                 Lloyd-Max codebook of its width; 1: per-regime codebooks
 *                 fitted to the calibration vectors (README "Repository
 *                 Structure": nonuniform_quantization.py, "Lloyd-Max with
 *                 per-regime codebooks"). Regime 0 is the coordinates i < d_eff,
 *                 regime 1 the rest; for each width a regime uses, Lloyd's
 *                 algorithm runs from the Gaussian codebook on the pooled scaled
 *                 coordinates z = (V^T u)_i / sigma_i of the calibration vectors
 *                 over the regime's coordinates of that width: thresholds at the
 *                 midpoints of neighbouring levels, each sample coded as the
 *                 compressor codes it, each level moved to the mean of its
 *                 samples (a level without samples kept). Records with fitted
 *                 codebooks are compressed by the float64 kernels (block-tiled
 *                 or reference; the tensor-core compress leaves them to these)
 *                 and attended by the SIMT kernel (SQ_OPT_ATTN_PATH 1): the
 *                 tensor-core attention kernels refuse them with SQ_FLAG_RECORD.
 *  fit_iters      Lloyd iterations of the fit (0: 30). The sums of a fit are
 *                 accumulated with atomics, in an order that varies between runs.
 */
typedef struct {
  int d;
  int n_heads;
  double avg_bits;
  int is_key;
  int qjl;
  int normalize;
  int d_eff_override;
  int max_bits;
  uint64_t seed;
  int max_sweeps;
  double tol;
  int rotation;
  double cumvar;
  int codebooks;
  int fit_iters;
} sq_calib_params;

/*
 * One packed cache (keys or values of one layer, or of several layers with the
 * layers folded into the head index). Device arrays, caller-owned:
 *  codes  uint32 [batch][n_heads][cap / 32][words][32]
 *                 one packed record per token, the records of 32 consecutive
 *                 tokens word-interleaved: word w of token t of a (batch, head)
 *                 row is element ((t / 32) * words + w) * 32 + t % 32 of the
 *                 row's cap * words words. A block of 32 tokens is then
 *                 words * 128 contiguous bytes, piece w holding word w of all
 *                 32 records, which is how the kernels want it in shared memory
 *                 (one bulk copy per tile) and how 32 lanes store it (one
 *                 128-byte line per word).
 *  norm   float  [batch][n_heads][cap]          ||x|| (1.0 when not normalized)
 *  rnorm  float  [batch][n_heads][cap]          QJL residual norm rho; NULL when
 *                                               the records carry no QJL bits
 *  cap    tokens per (batch, head); a multiple of 32.
 *  words  32-bit words per record, ceil(B / 32); must equal the records'.
 *
 * Record bit layout (the pages fix none; this is the library's reading): stream
 * bit k of a record is bit k % 32 of word k / 32 (little-endian words). The codes
 * of coordinates i = 0..d-1 with b_i > 0 come first, in coordinate order, each
 * least-significant bit first; then the m QJL bits (1 = projection >= 0); then
 * zero padding up to words * 32 bits.
 */
typedef struct {
  uint32_t* codes;
  float* norm;
  float* rnorm;
  int batch;
  int n_heads;
  int64_t cap;
  int words;
} sq_cache;

/*
 * Calibration record of one head: a plain byte block of sq_calib_bytes(d) bytes,
 * 256-byte aligned when records are stored back to back. Little-endian. The
 * canonical part can be written by any program; the library derives the rest.
 *
 *  offset               type  field
 *  0                    u32   magic 0x31435153 ("SQC1")
 *  4                    u32   version 2
 *  8                    i32   d
 *  12                   i32   d_eff (participation ratio (sum l)^2 / sum l^2, rounded half to even)
 *  16                   i32   m (QJL sign dimensions, 0 without QJL)
 *  20                   i32   total_bits B
 *  24                   i32   code_bits = sum of b_i = B - m
 *  28                   i32   words = ceil(B / 32)
 *  32                   u32   flags: 1 key, 2 QJL, 4 normalized, 8 random rotation,
 *                             16 cumulative-variance d_eff, 32 fitted codebooks
 *  36                   i32   eigensolver sweeps used
 *  40                   i32   stream (head index of the QJL Gaussian stream)
 *  44                   i32   max_bits
 *  48                   u64   seed
 *  56                   f64   trace (sum of eigenvalues)
 *  64                   f64   kappa = lambda[d_eff-1] / lambda[d_eff], +inf if d_eff = d
 *  72                   f64   avg_bits
 *  80                   u32   library use: nonzero once the derived part is built
 *  84..127                    zero
 *  128                  f64   lambda[d], descending, >= 0
 *  128 + 8d             f64   sigma[d]: normalized sqrt(lambda_i / trace), else sqrt(lambda_i)
 *  128 + 16d            f64   V[d*d], row-major; V[j*d + i] = component j of eigenvector i,
 *                             whose largest-magnitude component is positive
 *  128 + 16d + 8d^2     f64   S[d*d]: the m x m QJL matrix, row-major, in the first m*m slots
 *  128 + 16d + 16d^2    u8    bits[d]: code width b_i (greedy water-filling)
 *  128 + 17d + 16d^2    i32   offset[d]: bit position of coordinate i's code
 *  128 + 21d + 16d^2    f64   fitted levels [2][510]: regime r (0: i < d_eff, 1: the rest),
 *                             width b at r * 510 + 2^b - 2, 2^b ascending levels;
 *                             zero unless flag 32
 *  8288 + 21d + 16d^2   f64   fitted thresholds [2][502]: width b at r * 502 + 2^b - 1 - b,
 *                             2^b - 1 ascending thresholds (midpoints of the levels)
 *  then, from the next 256-byte boundary: the library's derived part (private).
 */
size_t sq_calib_bytes(int d);

/* ABI version (SQ_ABI_VERSION). */
int sq_abi_version(void);

/* Name and description of the last CUDA error a call of the calling thread
 * returned SQ_ERR_CUDA for ("none" before any). Static per thread; never NULL. */
const char* sq_last_error(void);

/* Static string naming a status. Never NULL. */
const char* sq_status_str(sq_status s);

/* Words of one record for these parameters: ceil(avg_bits * d / 32); 0 if invalid. */
int sq_record_words(const sq_calib_params* p);

/*
 * Gaussian N(0,1) Lloyd-Max quantizer of b bits (1..8), computed by the library
 * on the host (README "Repository Structure": nonuniform_quantization.py,
 * Lloyd-Max codebooks). levels: host array of 2^b doubles, ascending;
 * thresholds: host array of 2^b - 1 doubles (midpoints of adjacent levels);
 * D: host double, E[(Z - Q(Z))^2]. Any output pointer may be NULL.
 * Returns SQ_ERR_ARG for b outside 1..8. Host-only; touches no GPU.
 */
sq_status sq_codebook(int b, double* levels, double* thresholds, double* D);

/*
 * Uploads the per-device constant tables to the current device (done lazily by
 * every launching call otherwise). Call once per device before stream capture.
 */
sq_status sq_init(void);

/*
 * Process-wide options (host-only; no GPU work).
 *  SQ_OPT_COMPRESS_PATH: 0 = automatic (tensor-core kernel for fp16 head_dim-128
 *  prompts of >= 64 tokens; for other prompts of >= 16 tokens at head_dim 64,
 *  128 or 256 a block-tiled float64 kernel; the float64 one-warp-per-vector
 *  reference kernel otherwise), 1 = always the reference kernel. All produce
 *  identical codes (see sq_compress_kv).
 *  SQ_OPT_ATTN_PATH: 0 = automatic (the tcgen05 partials for head_dim 64/128/256
 *  and up to 16 query heads per KV head whose records fit its shared memory;
 *  SIMT partials otherwise), 1 = always the SIMT partials, 2 = the mma.sync
 *  tensor-core partials where they apply (up to 8 query heads, records of up to
 *  4 bits per coordinate), SIMT otherwise. All give the same results within the
 *  attention tolerances.
 *  SQ_OPT_TC_ERROR_BOUND: the fp32-accumulation term of the tensor-core compress
 *  error radius, in units of 2^-24 per unit of ||V_i / sigma_i|| (default 32:
 *  sixteen accumulation steps of one fp32 rounding each, with truncation).
 *  A code whose z lies within the radius of a threshold is recomputed in
 *  float64; a radius below the hardware's accumulation error can change codes,
 *  so values under the default exist only to measure that error.
 * Returns SQ_ERR_ARG for an unknown option or value.
 */
#define SQ_OPT_COMPRESS_PATH 1
#define SQ_OPT_ATTN_PATH 2
#define SQ_OPT_TC_ERROR_BOUND 3
sq_status sq_set_option(int option, int value);

/* Workspace bytes sq_calibrate needs for these parameters and n_tokens. */
size_t sq_calibrate_workspace(const sq_calib_params* p, int64_t n_tokens);

/*
 * Calibrates p->n_heads heads from their calibration vectors (README "Overview":
 * one-time calibration; conftest fixture pre_computed_calibration).
 *  x            device, dtype elements; element j of token t of head h at
 *               x + h * stride_head + t * stride_tok + j.
 *  n_tokens     calibration tokens per head (>= 1).
 *  calib_out    device, n_heads records of sq_calib_bytes(d) bytes back to back.
 *  ws, ws_bytes device workspace of at least sq_calibrate_workspace() bytes.
 *  d_status     device int[n_heads] (may be NULL): SQ_OK, SQ_ERR_NOT_CONVERGED
 *               (the record is still written from the last sweep) or SQ_ERR_ARG
 *               (the budget cannot hold m QJL bits and the codes).
 * Steps: C = X^T X / N (uncentred, float64 accumulation); cyclic Jacobi on C;
 * eigenvalues sorted descending, clamped at 0, eigenvector signs fixed; d_eff,
 * kappa, sigma; greedy water-filling of B - m code bits by the distortion drop
 * lambda_i (D(b_i) - D(b_i + 1)), ties to the lowest index; offsets; the QJL
 * matrix from the seed.
 */
sq_status sq_calibrate(const sq_calib_params* p, const void* x, sq_dtype dtype, int64_t n_tokens,
                       int64_t stride_head, int64_t stride_tok, void* calib_out, void* ws,
                       size_t ws_bytes, int* d_status, sq_stream stream);

/*
 * Imports n_heads records whose canonical part was written elsewhere (saved
 * records, or another implementation): checks each header (magic, version,
 * d, bit counts, offsets; with fitted codebooks, finite tables whose levels
 * increase and whose thresholds lie between them for every width in use) and
 * builds the library's derived part. The record
 * holds what the README's "Overview" calls the one-time calibration (the
 * calibrated eigenbasis, d_eff and kappa of calibration.py, the water-filled
 * widths); importing lets a calibration computed once be reused.
 *  calib     device, n_heads records of sq_calib_bytes(d) bytes.
 *  d_status  device int[n_heads] (may be NULL): SQ_OK or SQ_ERR_RECORD.
 */
sq_status sq_calib_import(void* calib, int n_heads, int d, int* d_status, sq_stream stream);

/*
 * Compresses keys and/or values into packed caches (README "Overview" and
 * "Repository Structure": rotation into the calibrated eigenbasis, Lloyd-Max
 * codes under the water-filled widths, QJL sign bits of the key residual on
 * the top-m signal dimensions).
 *  calib_k, calib_v  device, n_heads records each (either side may be NULL
 *                    together with its input and cache).
 *  k, v        device, dtype [batch][n_heads][n_tok][d], contiguous.
 *  dtype       SQ_F32, SQ_F16 or SQ_BF16 (converted exactly to float).
 *  d_start_pos device int32[batch]: first cache slot written for each row
 *              (NULL = 0). Appending one decode token is n_tok = 1 at the
 *              row's current length.
 *  kc, vc      host structs describing the caches (device arrays inside).
 *  d_flags     device uint32 (may be NULL): SQ_FLAG_CAPACITY, SQ_FLAG_RECORD.
 * Per vector: norm = ||x||; u = x / norm; y = V^T u; z_i = y_i / sigma_i;
 * code_i = number of b_i-bit thresholds strictly below z_i; keys with QJL:
 * r = y[0:m] - sigma[0:m] * level(code[0:m]), rnorm = ||r||, bit j = [(S r)_j >= 0].
 * n_tok = 0 is a no-op.
 */
sq_status sq_compress_kv(const void* calib_k, const void* calib_v, const void* k, const void* v,
                         sq_dtype dtype, int batch, int n_heads, int d, int64_t n_tok,
                         const int32_t* d_start_pos, const sq_cache* kc, const sq_cache* vc,
                         uint32_t* d_flags, sq_stream stream);

/*
 * Device bytes of the staging buffer sq_compress_kv_host uses for this shape:
 * two slabs, each holding the vectors of up to ceil(16 MiB / (n_tok * d *
 * element size)) heads of one batch row (at least one head, at most n_heads),
 * each slab rounded up to 256 bytes. 0 for an unsupported shape.
 */
size_t sq_compress_host_staging(int batch, int n_heads, int d, sq_dtype dtype, int64_t n_tok);

/*
 * sq_compress_kv with the keys and values in HOST memory: the same codes,
 * norms and rho as sq_compress_kv on the same vectors (the same kernels run on
 * the same data), with the host-to-device transfer overlapped with the
 * compression. The vectors go through the caller's device staging buffer in
 * pieces of whole heads of one batch row (keys first, then values); while one
 * piece is compressed on `stream`, the next is copied on the library's copy
 * stream for this device, so that the copy engine and the SMs work together.
 *  h_k, h_v     host, dtype [batch][n_heads][n_tok][d], contiguous; page-locked
 *               (cudaHostAlloc / cudaHostRegister) for the copies to overlap
 *               (pageable memory works but each copy then blocks the host).
 *               Either side may be NULL together with its records and cache.
 *               They must stay valid and unchanged until `stream` has passed
 *               the call's work.
 *  d_staging    device, 256-byte aligned; staging_bytes >= the bytes of two
 *               slabs of one head (else SQ_ERR_WORKSPACE). The piece size is
 *               the most whole heads half of staging_bytes holds (rounded
 *               down to 256 bytes per slab). It is scratch owned by the call
 *               until `stream` has passed its work.
 * Other arguments, layouts, results and flags as sq_compress_kv. The copy
 * stream waits on `stream` before the first copy and `stream` waits on every
 * copy before compressing its piece, so work enqueued on `stream` after the
 * call runs after all of it. Returns SQ_ERR_CUDA if a stream, event or copy
 * cannot be set up (nothing after that point is enqueued).
 */
sq_status sq_compress_kv_host(const void* calib_k, const void* calib_v, const void* h_k, const void* h_v,
                              sq_dtype dtype, int batch, int n_heads, int d, int64_t n_tok,
                              const int32_t* d_start_pos, const sq_cache* kc, const sq_cache* vc,
                              void* d_staging, size_t staging_bytes, uint32_t* d_flags, sq_stream stream);

/*
 * Reconstructs vectors from a packed cache (the inverse of the README's
 * "Repository Structure" steps: spectral_rotation.py rotated into the
 * eigenbasis, nonuniform_quantization.py quantized, selective_qjl.py added the
 * sign correction on the signal dims; here they are undone):
 * x_hat = norm * V (sigma * level(code)),
 * plus, when apply_qjl and the records carry QJL bits,
 * norm * V[:, 0:m] (sqrt(pi/2) / m * rnorm * S^T s), s_j = 2 bit_j - 1.
 *  calib  device, cache->n_heads records of head_dim d.
 *  t0, n_tok  token window [t0, t0 + n_tok) of every (batch, head); must lie
 *         inside [0, cap) (else SQ_FLAG_CAPACITY and nothing is written).
 *  out    device float [batch][n_heads][n_tok][d].
 *  d_flags device uint32 (may be NULL): SQ_FLAG_CAPACITY, SQ_FLAG_RECORD.
 */
sq_status sq_decompress_kv(const void* calib, const sq_cache* cache, int d, int64_t t0, int64_t n_tok,
                           int apply_qjl, float* out, uint32_t* d_flags, sq_stream stream);

/* Workspace bytes sq_attn_decode needs for this shape. */
size_t sq_attn_workspace(int batch, int n_q_heads, int n_kv_heads, int d, int64_t max_ctx);

/*
 * Decode attention over packed caches (README "Headline Results": per-step
 * decode latency over the compressed cache). For batch row b and query head h,
 * KV head g = h / (n_q_heads / n_kv_heads), L = seq_lens[b]:
 *   q' = V_K^T q;
 *   s_t = scale * ||k_t|| * (sum_i q'_i sigma_i level_t,i
 *                            + sqrt(pi/2) / m * rho_t * sum_j (S q'[0:m])_j (2 bit_t,j - 1));
 *   p = softmax_t(s_t), t < L;  o = V_V (sigma_V * sum_t p_t ||v_t|| level^V_t).
 * This is dense softmax attention over the decompressed keys (with their QJL
 * term) and values (without one).
 *  calib_k, calib_v  device, n_kv_heads records each.
 *  kc, vc       packed caches with n_heads = n_kv_heads.
 *  d_seq_lens   device int32[batch]; each <= max_ctx and <= cap.
 *  max_ctx      host bound on the sequence lengths (sizes the split of work).
 *  q            device, q_dtype [batch][n_q_heads][d].
 *  scale        > 0, or <= 0 for 1/sqrt(d).
 *  out          device, out_dtype [batch][n_q_heads][d].
 *  scores_out   device float [batch][n_q_heads][max_ctx] (may be NULL): s_t for
 *               t < L; entries past L are left unwritten.
 *  ws, ws_bytes device workspace of at least sq_attn_workspace() bytes.
 *  d_flags      device uint32 (may be NULL): SQ_FLAG_SEQLEN, SQ_FLAG_RECORD.
 * A row with L = 0 produces zeros.
 */
sq_status sq_attn_decode(const void* calib_k, const void* calib_v, const sq_cache* kc,
                         const sq_cache* vc, const int32_t* d_seq_lens, int batch, int n_q_heads,
                         int n_kv_heads, int d, int64_t max_ctx, const void* q, sq_dtype q_dtype,
                         float scale, void* out, sq_dtype out_dtype, float* scores_out, void* ws,
                         size_t ws_bytes, uint32_t* d_flags, sq_stream stream);

/*
 * One decode step (README "Headline Results": decode latency per step over the
 * compressed cache): for every batch row b, the new token's keys k_new and
 * values v_new of every KV head are compressed into the caches at position
 * d_pos[b] (as sq_compress_kv with n_tok = 1 and start_pos = d_pos), then
 * decode attention runs over d_pos[b] + 1 tokens, the new one included (as
 * sq_attn_decode with seq_lens = d_pos + 1).
 *  k_new, v_new  device, dtype [batch][n_kv_heads][1][d]; q device, dtype
 *                [batch][n_q_heads][d] (one dtype for the three).
 *  d_pos         device int32[batch]; d_pos[b] + 1 <= max_ctx and <= cap.
 *  Other arguments, workspace (sq_attn_workspace of the same shape), results
 *  and flags as sq_compress_kv and sq_attn_decode; max_ctx >= 1.
 * On the tcgen05 path (head_dim 64/128/256, up to 16 query heads per KV head)
 * the step is three launches: the appends share one with the query
 * preparation, the attention partials merge their splits themselves (the last
 * block of each (row, KV head) to finish), and one launch rotates every output
 * back (o = V_V a, batched over the rows of each KV head); otherwise the step
 * runs the appends, prepare, partials and combine as separate launches.
 */
sq_status sq_decode_step(const void* calib_k, const void* calib_v, const sq_cache* kc, const sq_cache* vc,
                         const void* k_new, const void* v_new, const void* q, sq_dtype dtype, const int32_t* d_pos,
                         int batch, int n_q_heads, int n_kv_heads, int d, int64_t max_ctx, float scale, void* out,
                         sq_dtype out_dtype, float* scores_out, void* ws, size_t ws_bytes, uint32_t* d_flags,
                         sq_stream stream);

/* Workspace bytes sq_attn_prefill needs for this shape (0 if unsupported). */
size_t sq_attn_prefill_workspace(int batch, int n_q_heads, int n_kv_heads, int d, int64_t n_qtok, int64_t max_ctx);

/*
 * Causal attention of a chunk of query tokens over the packed cache (prefill or
 * chunked prefill; the README's "Key Findings" 3 measures the method over
 * sequence lengths 512-2048, whose prompts pass through attention before
 * decoding). Query token t of batch row b sits at position d_start[b] + t and
 * attends to the cache positions 0 .. d_start[b] + t, with the same scores,
 * softmax and output as sq_attn_decode gives a single query over that prefix.
 * The cache must already hold those positions (compress the chunk first).
 *  q       device, q_dtype [batch][n_q_heads][n_qtok][d].
 *  out     device, out_dtype [batch][n_q_heads][n_qtok][d].
 *  d_start device int32[batch]; d_start[b] + n_qtok <= max_ctx and <= cap.
 *  ws      device workspace of at least sq_attn_prefill_workspace() bytes.
 * The query positions of a row are taken in blocks of floor(16 / G) (G = query
 * heads per KV head), whose G x block columns share each decoded key and value
 * tile in the 16-column MMAs; the causal mask is applied per column.
 * Returns SQ_ERR_ARG when batch x blocks exceeds 65535.
 */
sq_status sq_attn_prefill(const void* calib_k, const void* calib_v, const sq_cache* kc, const sq_cache* vc,
                          const int32_t* d_start, int batch, int n_q_heads, int n_kv_heads, int d, int64_t n_qtok,
                          int64_t max_ctx, const void* q, sq_dtype q_dtype, float scale, void* out, sq_dtype out_dtype,
                          void* ws, size_t ws_bytes, uint32_t* d_flags, sq_stream stream);

/*
 * sq_attn_decode without a workspace argument, for callers that cannot
 * allocate device memory where they run decode attention: a serving loop whose
 * device memory is reserved once at start-up and may not grow, plug-ins with
 * no access to the host application's allocator, runtimes that forbid
 * allocation after initialisation. The pages have no counterpart: this is a
 * deployment convenience of this library.
 *
 * Arguments and results are those of sq_attn_decode minus ws / ws_bytes. The
 * scratch is one fixed array of SQ_ATTN_NOALLOC_MAX_BYTES in the library's
 * device memory, present on every GPU that loads libsq until the process
 * exits. The call allocates nothing (no cudaMalloc, no allocating library
 * routine). It returns SQ_ERR_WORKSPACE, before any launch, when the shape
 * needs more than the array (sq_attn_workspace() > SQ_ATTN_NOALLOC_MAX_BYTES).
 * The first call on a device looks up the array's device address on that
 * device (cudaGetSymbolAddress) and caches it; make that first call before
 * any stream capture. Every call on a device shares the one array, so calls
 * whose executions overlap on the GPU (on different streams, for instance)
 * race and corrupt each other's results; serialize them. Nothing in
 * the array needs to start at zero: each call writes every scratch entry it
 * later reads.
 */
#define SQ_ATTN_NOALLOC_MAX_BYTES 0x800000u /* 8 MiB */
sq_status sq_attn_decode_noalloc(const void* calib_k, const void* calib_v, const sq_cache* kc,
                                 const sq_cache* vc, const int32_t* d_seq_lens, int batch, int n_q_heads,
                                 int n_kv_heads, int d, int64_t max_ctx, const void* q, sq_dtype q_dtype,
                                 float scale, void* out, sq_dtype out_dtype, float* scores_out,
                                 uint32_t* d_flags, sq_stream stream);

/*
 * Self-test of the bounded waits (no fault, no hang): one GPU thread waits on
 * an mbarrier that nothing arrives on, through the same helper every
 * tensor-core kernel of the library waits with, but with a limit of limit_us
 * microseconds (1 .. 2 000 000; the kernels use 2 s); it then gives up, ORs
 * SQ_FLAG_TIMEOUT into *d_flags and returns, leaving the context usable. For
 * tests of the timeout path.
 *  d_flags  device uint32, 16-byte aligned.
 * Returns SQ_ERR_ARG for a limit out of range or a missing / misaligned word.
 */
sq_status sq_wait_selftest(uint32_t limit_us, uint32_t* d_flags, sq_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* SQ_H */
