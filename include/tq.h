/*
 * tq.h -- C ABI of the B200 (sm_100a) rotated-codebook KV-cache codec.
 *
 * The method (TurboQuant as described on the pages this library follows):
 *   - store the norm nu = ||x|| and quantize the unit vector x / nu
 *     ("FibQuant: Quantizzazione Vettoriale Universale ...", section 2.3);
 *   - rotate it with one shared random orthogonal map, a randomized
 *     Walsh-Hadamard transform Pi = H_d diag(D) / sqrt(d)
 *     ("Ablazione, Inferenza Statistica e Validazione ...", "Configurazione
 *     Sperimentale");
 *   - quantize every rotated coordinate with a Lloyd-Max codebook solved
 *     offline for the Beta coordinate law ("Google presenta TurboQuant ...",
 *     "La mecanica geometrica de TurboQuant", MSE cost C(f_X, b));
 *   - keys use TURBOQUANT_prod: b-1 MSE bits plus a 1-bit QJL sketch
 *     sigma = sign(S r) of the rotated residual r, with rho = ||r||, giving an
 *     unbiased inner-product estimator (same page, "Eliminacion del sesgo
 *     interno del producto");
 *   - attention logits are estimated straight from the packed codes and the
 *     values are accumulated in the rotated domain, with one inverse rotation
 *     per output ("TurboESM ...", section 2.E "Kernel Fuso Triton").
 *
 * Conventions for every call
 *   - Return value: tq_status.  On failure tq_last_error() gives a message
 *     (thread-local, valid until the next call on the same thread).
 *   - Pointers documented "device" must be CUDA device memory of the device
 *     that is current when the call is made; "host" pointers are ordinary
 *     host memory.  The caller owns every buffer it passes in.
 *   - Calls taking a stream are stream-ordered and asynchronous: arguments are
 *     validated synchronously, kernels are enqueued on `stream`
 *     (a cudaStream_t; NULL = legacy default stream), and no call blocks the
 *     host.  Launch failures return TQ_ERR_CUDA; faults inside a kernel
 *     surface at the caller's next synchronisation.
 *   - Supported: d in {64, 128} for the KV-cache calls and d = 1536 for the
 *     vector-search calls; key MSE bits 1..4 (with QJL: 2 <= bits_k <= 5
 *     total); value bits 1..4.
 */
#ifndef TQ_B200_H
#define TQ_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TQ_OK = 0,
  TQ_ERR_INVALID_ARG = 1,   /* NULL where a buffer is required, bad size or shape */
  TQ_ERR_UNSUPPORTED = 2,   /* head dim or bit width this build has no kernel for */
  TQ_ERR_ALIGNMENT = 3,     /* a device buffer misses its required alignment */
  TQ_ERR_CUDA = 4,          /* a CUDA runtime call or kernel launch failed */
  TQ_ERR_WORKSPACE = 5      /* workspace too small (query tq_attention_workspace) */
} tq_status;

typedef enum { TQ_F32 = 0, TQ_BF16 = 1 } tq_dtype;

/* ------------------------------------------------------------------------
 * Offline codebook ("Google presenta TurboQuant ...", "La mecanica
 * geometrica de TurboQuant": minimise C(f_X, b) once per bit width and store).
 *
 * Solves the Lloyd-Max conditions for the density of one coordinate of a
 * uniform point on the unit sphere S^{d-1},
 *     f_d(x) = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)) (1 - x^2)^((d-3)/2),
 * on [-1, 1] (outer cells reach the support ends).  fp64 solve on the host,
 * fp32 results.
 *   centroids  host, 2^bits floats, ascending, odd-symmetric.
 *   thresholds host, 2^bits - 1 floats, midpoints of adjacent centroids; a
 *              coordinate u gets code #{k : u >= thresholds[k]}.
 *   mse_per_coord host, nullable: E[(X - Q(X))^2] at the solution.
 * Errors: TQ_ERR_INVALID_ARG for d < 4, bits outside 1..8 or NULL outputs.
 * ------------------------------------------------------------------------ */
int tq_build_codebook(int d, int bits, float *centroids, float *thresholds,
                      double *mse_per_coord);

/* ------------------------------------------------------------------------
 * Codec: immutable description shared by every call (thread-safe to share).
 *
 * rotation_signs  host, d entries, each +1 or -1: the diagonal D of
 *                 Pi = H_d diag(D) / sqrt(d), H_d Sylvester-ordered.
 * qjl_bf16        host, d*d bf16 bit patterns, row-major S[i][j]: the QJL
 *                 sketch (i.i.d. N(0,1) values stored as bf16).  Required iff
 *                 qjl_k != 0.
 * bits_k          total key bits; with qjl_k the MSE stage uses bits_k - 1.
 * bits_v          value bits (TURBOQUANT_mse).
 * rotation        host, d*d fp32 row-major Pi[i][j], nullable: a dense
 *                 orthogonal rotation used instead of H_d diag(D) / sqrt(d)
 *                 (the theory's shared Haar rotation: "Google presenta
 *                 TurboQuant ...", "La mecanica geometrica de TurboQuant";
 *                 "FibQuant ...", section 2.1; see tq_haar_rotation).  Only for
 *                 d = 64 and 128; rotation_signs may then be NULL.  Quantize,
 *                 decode and dequantize apply it as fp32 matrix-vector
 *                 products; the bidirectional pass and the outlier-channel split
 *                 return TQ_ERR_UNSUPPORTED for such a codec.  Rows of Pi must
 *                 be orthonormal to 1e-5 (TQ_ERR_INVALID_ARG otherwise).
 * tq_codec_create solves both codebooks with tq_build_codebook and copies D,
 * S, the dense rotation and the codebooks to the current device (the only
 * allocations the library makes); tq_codec_destroy frees them.
 * ------------------------------------------------------------------------ */
typedef struct tq_codec tq_codec;

typedef struct {
  int d;
  int bits_k;
  int qjl_k;
  int bits_v;
  const int8_t *rotation_signs;
  const uint16_t *qjl_bf16;
  const float *rotation;
} tq_codec_desc;

/* Host helper: a Haar-distributed rotation from a d x d matrix of i.i.d.
 * N(0,1) entries (host fp32, row-major): the orthogonal factor Q of G = QR
 * with every diagonal entry of R made positive (Householder reflections in
 * fp64), written to rotation (host fp32 d x d, row-major).
 * Errors: TQ_ERR_INVALID_ARG for NULL buffers, d outside 1..4096 or a
 * non-finite entry. */
int tq_haar_rotation(int d, const float *gaussian, float *rotation);

int tq_codec_create(const tq_codec_desc *desc, tq_codec **out);
void tq_codec_destroy(tq_codec *codec);
/* Host copies of the codec's codebooks (fp32) for inspection; any pointer may
 * be NULL.  Sizes: 2^mse_bits_k, 2^mse_bits_k - 1, 2^bits_v, 2^bits_v - 1. */
int tq_codec_codebooks(const tq_codec *codec, float *ck, float *tk, float *cv, float *tv);

/* ------------------------------------------------------------------------
 * Compressed cache: fixed rate, every token at fixed addresses
 * ("FibQuant ...", section 1: decode any token on its own by address
 * arithmetic).  All four planes are device memory owned by the caller.
 *
 *   kcode  uint8  [B][Hkv][rows_cap][planes_k][d/8]  planes_k = mse bits (+1
 *          with QJL).  Plane p < mse bits holds bit p of each coordinate's
 *          code; the last plane holds sigma.  Coordinate i: byte i/8, bit i%8.
 *   kscale fp16   [B][Hkv][rows_cap][2]  (nu, rho) per key; rho = 0 without QJL.
 *   vcode  uint32 [B][Hkv][rows_cap/32][bits_v][d]  32-token column groups:
 *          bit (t % 32) of word [t/32][p][i] is bit p of coordinate i's code
 *          of token t.
 *   vnorm  fp16   [B][Hkv][rows_cap]  nu per value.
 * rows_cap must be a multiple of 32; every plane needs 16-byte alignment.  Bytes per (token, head): d/8*planes_k + 4 for
 * keys, d/8*bits_v + 2 for values.
 * ------------------------------------------------------------------------ */
typedef struct {
  uint8_t *kcode;
  uint16_t *kscale;
  uint32_t *vcode;
  uint16_t *vnorm;
  int B;
  int Hkv;
  int64_t rows_cap;
} tq_cache;

/* Bytes of each plane (kcode, kscale, vcode, vnorm) for a cache shape. */
int tq_cache_bytes(const tq_codec *codec, int B, int Hkv, int64_t rows_cap, size_t bytes[4]);

/* ------------------------------------------------------------------------
 * Quantize-append (prefill or decode append).  One fused kernel per call.
 *
 * k, v     device, [B][Hkv][T][d] with element strides (stride_b, stride_h,
 *          stride_t) and d contiguous; dtype TQ_F32 or TQ_BF16.
 * rope_cos, rope_sin  device fp32 [*][d/2], nullable together: rotate-half
 *          RoPE is applied to keys at positions pos0 + t before encoding
 *          ("TurboESM ...", section 2.A: RoPE first, then Pi).
 * cache    rows [row0, row0 + T) of every (b, h) are written; other tokens of
 *          a partially covered 32-token value group are preserved (calls that
 *          touch the same group must be stream-ordered).
 * status   device uint32, nullable: incremented once per row (key or value)
 *          whose input had a non-finite element or whose fp16 norm overflowed;
 *          such rows are encoded as zero vectors.
 * ------------------------------------------------------------------------ */
int tq_quantize_kv(const tq_codec *codec, const void *k, const void *v, int dtype,
                   int B, int Hkv, int T, int64_t stride_b, int64_t stride_h,
                   int64_t stride_t, const float *rope_cos, const float *rope_sin,
                   int64_t pos0, const tq_cache *cache, int64_t row0, uint32_t *status,
                   void *stream);

/* ------------------------------------------------------------------------
 * Decode attention straight from the compressed cache (split-K).
 *
 * For query head h (KV head h / (Hq/Hkv)) of batch b with length T_b:
 *   q'  = Pi RoPE(q, T_b - 1),  q'' = S q'
 *   l_j = scale * nu_j * (<q', c_k[idx_j]> + sqrt(pi/2)/d * rho_j * <q'', 2 sigma_j - 1>)
 *   out = Pi^T ( sum_j softmax(l)_j * nu^v_j * c_v[idx^v_j] )
 * q        device [B][Hq][d], dtype TQ_F32 or TQ_BF16.
 * seq_lens device int32 [B], nullable (then every batch has max_seq_len);
 *          entries are clamped to 1..max_seq_len; max_seq_len <= rows_cap.
 * rope_cos/rope_sin  as for tq_quantize_kv (nullable together).
 * num_splits  chunks per (b, KV head), at most 512; 0 picks a default of at
 *          most 64 (about two chunks per SM over all (b, KV head), in
 *          128-row multiples), which a workspace sized with num_splits = 0 fits.
 * workspace   device, >= tq_attention_workspace(...) bytes, 16-byte aligned;
 *             scratch owned by the caller, contents need no initialisation.
 * out      device fp32 [B][Hq][d].
 * Every wait inside the kernels is bounded.  If one gives up (a copy or MMA
 * that never completes), the kernel drains its own outstanding copies and
 * MMAs, records it in a status word of the workspace, and every element of
 * out is written as NaN instead of a merge of incomplete partials.
 * ------------------------------------------------------------------------ */
int tq_attention_workspace(const tq_codec *codec, int B, int Hq, int num_splits, size_t *bytes);
int tq_attention_decode(const tq_codec *codec, const void *q, int dtype, int B, int Hq,
                        int Hkv, const tq_cache *cache, const int32_t *seq_lens,
                        int max_seq_len, float scale, const float *rope_cos,
                        const float *rope_sin, int num_splits, void *workspace,
                        size_t ws_bytes, float *out, void *stream);

/* One decode step in one call: append the new token's key and value at row
 * T - 1 of every (b, KV head) (the key RoPE-rotated at position T - 1), then
 * decode the queries over rows 0 .. T - 1.  Equal to tq_quantize_kv (T = 1,
 * row0 = pos0 = T - 1) followed by tq_attention_decode (max_seq_len = T, no
 * seq_lens), with their validation and error codes.
 * k_new, v_new  device [B][Hkv][d], kv_dtype TQ_F32 or TQ_BF16 (contiguous).
 * q             device [B][Hq][d], q_dtype.   out  device fp32 [B][Hq][d]. */
int tq_decode_step(const tq_codec *codec, const void *k_new, const void *v_new, int kv_dtype,
                   const void *q, int q_dtype, int B, int Hq, int Hkv, const tq_cache *cache, int T,
                   float scale, const float *rope_cos, const float *rope_sin, int num_splits,
                   void *workspace, size_t ws_bytes, float *out, void *stream);

/* tq_decode_step fed from and read back to host memory, for a caller whose
 * new token and query live on the host.  The step's input is one host buffer
 * holding k_new [B][Hkv][d], v_new [B][Hkv][d] (both kv_dtype) and q
 * [B][Hq][d] (q_dtype), in that order, each part starting where the previous
 * one ends; in_bytes is its total size.  The call copies it to the device
 * buffer in_dev (in_bytes, 16-byte aligned; owned by the caller), runs
 * tq_decode_step over the three parts, copies out_dev (device fp32
 * [B][Hq][d]) to out_host, and returns once out_host holds the result (the
 * stream is synchronised).  in_host and out_host should be page-locked for
 * the copies to run asynchronously; pageable memory works, more slowly.
 * Errors: those of tq_decode_step, TQ_ERR_INVALID_ARG for NULL buffers or
 * an in_bytes that is not the parts' total, TQ_ERR_CUDA for a failed copy. */
int tq_decode_step_host(const tq_codec *codec, const void *in_host, void *in_dev, size_t in_bytes,
                        int kv_dtype, int q_dtype, int B, int Hq, int Hkv, const tq_cache *cache,
                        int T, float scale, const float *rope_cos, const float *rope_sin,
                        int num_splits, void *workspace, size_t ws_bytes, float *out_dev,
                        float *out_host, void *stream);

/* Same as tq_attention_decode, and also writes the estimated logits
 * l_j (the formula above, scale included) of every query head:
 * logits  device fp32 [B][Hq][max_seq_len]; entries j >= T_b are left
 *         untouched.  Meant for inspection and scoring; costs one extra
 *         store per (head, key). */
int tq_attention_logits(const tq_codec *codec, const void *q, int dtype, int B, int Hq,
                        int Hkv, const tq_cache *cache, const int32_t *seq_lens,
                        int max_seq_len, float scale, const float *rope_cos,
                        const float *rope_sin, int num_splits, void *workspace,
                        size_t ws_bytes, float *out, float *logits, void *stream);

/* ------------------------------------------------------------------------
 * Bidirectional attention over the compressed cache (prefill-style pass):
 * every query i of a sequence attends to all T cached keys, no mask
 * ("TurboESM ...", sections 2.A and 2.E: RoPE then rotation, attention straight
 * from the compressed cache).  Query i is RoPE-rotated at position i.
 * Same estimator as tq_attention_decode, evaluated as dense tiles in the
 * rotated domain on the tensor cores.
 * q      device [B][H][Lq][d] (TQ_F32 or TQ_BF16); query head h reads KV head
 *        h / (H / Hkv).   out  device fp32 [B][H][Lq][d].
 * T      cached tokens per (b, KV head), 1..rows_cap.
 * Supported: d = 64 with the codec's key MSE bits 1..3 (+QJL) and value bits 1..4.
 * workspace: >= tq_attention_bidir_workspace(...) bytes, 16-byte aligned.
 * Every wait inside the kernel is bounded; a CTA whose wait gives up lets its
 * own copies and MMAs land and writes NaN to every element of its 128
 * queries' output rows (the other queries are exact).
 * ------------------------------------------------------------------------ */
int tq_attention_bidir_workspace(const tq_codec *codec, int B, int H, int Lq, size_t *bytes);
int tq_attention_bidir(const tq_codec *codec, const void *q, int dtype, int B, int H, int Hkv,
                       int Lq, const tq_cache *cache, int T, float scale, const float *rope_cos,
                       const float *rope_sin, void *workspace, size_t ws_bytes, float *out,
                       void *stream);

/* ------------------------------------------------------------------------
 * Vector search over TURBOQUANT_prod codes, d = 1536 ("Google presenta
 * TurboQuant ...", "Velocidad y eficiencia de indexacion": the codes are
 * data-oblivious, so indexing is a single encode pass with no training;
 * "Eliminacion del sesgo interno del producto": the prod estimator of <q, x>).
 * The codec must have d = 1536 and QJL keys with key MSE bits 1..3.  For
 * d = 1536 the rotation is Pi = (H_12 kron H_128) diag(D) / sqrt(1536), H_12
 * the Paley type-I matrix of GF(11) (H = I + [[0, 1^T], [-1, Q]],
 * Q[i][j] = chi(j - i)), H_128 Sylvester-ordered.
 *
 * tq_index_build encodes n database rows exactly like keys (no RoPE):
 *   x        device fp32 [n][1536], 16-byte aligned.
 *   kcode    device u8 [n][planes][192] (planes = MSE bits + 1; plane p bit i of
 *            row j = bit p of code i, the last plane = the QJL sign bits),
 *            16-byte aligned.
 *   kscale   device fp16 [n][2] = (nu, rho), 4-byte aligned.
 *   status   device u32, nullable: incremented once per row that had a
 *            non-finite entry (or a norm above the fp16 range); such rows are
 *            stored as zero rows.
 *   workspace >= tq_index_workspace(...) bytes (residual scratch of at most
 *            65536 rows), 16-byte aligned.
 * tq_scan_topk scores nq queries against the n rows with
 *   s_qj = nu_j (<Pi q, c[idx_j]> + sqrt(pi/2)/1536 rho_j <S Pi q, 2 sigma_j - 1>)
 * and returns, per query, the k best rows by (score descending, index
 * ascending):
 *   q        device fp32 [nq][1536], 16-byte aligned (unit norm is not required).
 *   idx      device int32 [nq][k];  score  device fp32 [nq][k].
 *   1 <= k <= min(16, n);  workspace >= tq_scan_workspace(...) bytes, 16-byte aligned.
 * Scores come from one fp16 product per element on the tensor cores (rows
 * [c[idx] | rho (2 sigma - 1)] against the query scaled by a power of two),
 * accumulated in fp32: about 1e-5 |q| absolute error for unit rows, so rows
 * whose scores differ by less than that may swap places.  Every wait inside
 * the scan kernel is bounded; if one gives up, the kernel lets its own copies
 * and MMAs land, records it in a status word of the workspace (cleared by
 * every call), and every result of the call is written as index -1, score
 * NaN.  An index build that gives up sets bit 31 of its status word.
 * ------------------------------------------------------------------------ */
int tq_index_workspace(const tq_codec *codec, int64_t n, size_t *bytes);
int tq_index_build(const tq_codec *codec, const float *x, int64_t n, uint8_t *kcode,
                   uint16_t *kscale, uint32_t *status, void *workspace, size_t ws_bytes,
                   void *stream);
int tq_scan_workspace(const tq_codec *codec, int64_t n, int nq, int k, size_t *bytes);
int tq_scan_topk(const tq_codec *codec, const uint8_t *kcode, const uint16_t *kscale, int64_t n,
                 const float *q, int nq, int k, int32_t *idx, float *score, void *workspace,
                 size_t ws_bytes, void *stream);

/* Same scan by lookup tables instead of tensor-core tiles (the comparison
 * path; same pages and estimator): per query, T[i][m] = (Pi q)_i c[m] and
 * sqrt(pi/2)/1536 (S Pi q)_i in shared memory, one lookup and one signed add
 * per coordinate in fp32, so scores carry only fp32 rounding (no fp16
 * products).  Arguments, workspace (tq_scan_workspace covers both paths) and
 * output order as tq_scan_topk; kcode and kscale need 4-byte alignment. */
int tq_scan_topk_lut(const tq_codec *codec, const uint8_t *kcode, const uint16_t *kscale,
                     int64_t n, const float *q, int nq, int k, int32_t *idx, float *score,
                     void *workspace, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------
 * Decode without a workspace, for callers that cannot allocate device memory.
 *
 * No counterpart on the pages.  Callers that cannot call cudaMalloc (a plugin
 * inside a host application that owns all device allocations, or a serving
 * process whose memory is reserved up front) cannot hand tq_attention_decode
 * a workspace.  This variant runs the same kernels with its scratch taken from
 * a static device array of TQ_NOALLOC_SCRATCH_BYTES (16 MiB) inside the
 * library, held by every GPU that loads the library until the process exits.
 * It calls no cudaMalloc/cudaFree.  Arguments as tq_attention_decode, minus the
 * workspace.
 *   - The first call on each device looks the array's device address up
 *     (cudaGetSymbolAddress, that device current) and caches it.
 *   - Shapes whose scratch, the byte count tq_attention_workspace() returns
 *     for the same codec, B, Hq and num_splits, exceeds the 16 MiB limit
 *     return TQ_ERR_WORKSPACE.
 *   - All calls share the array and each leaves its contents there.  Every
 *     scratch word a call reads it has written itself earlier in the same
 *     call (the status word included), so nothing needs clearing.  Calls
 *     whose kernels overlap on the GPU (other streams, other host threads)
 *     race on it: the caller must serialise them.
 * ------------------------------------------------------------------------ */
#define TQ_NOALLOC_SCRATCH_BYTES (16u << 20)
int tq_attention_decode_noalloc(const tq_codec *codec, const void *q, int dtype, int B, int Hq,
                                int Hkv, const tq_cache *cache, const int32_t *seq_lens,
                                int max_seq_len, float scale, const float *rope_cos,
                                const float *rope_sin, int num_splits, float *out,
                                void *stream);

/* ------------------------------------------------------------------------
 * Dequantize rows [row0, row0 + rows) of every (b, h) ("FibQuant ...",
 * section 2.3 decoder): keys  nu Pi^T (c_k[idx] + sqrt(pi/2)/d rho S^T(2 sigma - 1)),
 * values nu Pi^T c_v[idx].
 * which  0 = keys, 1 = values.   out  device fp32 [B][Hkv][rows][d].
 * ------------------------------------------------------------------------ */
int tq_dequantize(const tq_codec *codec, const tq_cache *cache, int which, int64_t row0,
                  int64_t rows, float *out, void *stream);

/* ------------------------------------------------------------------------
 * Outlier-channel mixed precision ("Google presenta TurboQuant ...",
 * "Desempeno teorico y empirico": for non-integer rates, specific outlier
 * channels get more bits than the rest, e.g. 3 and 2 bits for 2.5 bits per
 * channel, 4 and 3 for 3.5).
 *
 * A head vector of d = 2 * hi->d channels is split, per KV head and separately
 * for keys and values, into two channel sets of d/2 each.  Each set is an
 * independent TurboQuant vector coded by its own codec (own norm, rotation,
 * codebooks and QJL sketch) into its own cache: `hi` (more bits) codes the
 * outlier channels, `lo` the rest.  The rate per channel is the mean of the two
 * codecs' bit widths.  Keys are RoPE-rotated over all d channels before the
 * split ("TurboESM ...", section 2.A).  Decode sums the two codecs' logit
 * estimates; each value half is summed in its own rotated domain and rotated
 * back onto its channels.
 *
 * hi, lo     codecs with the same d (64 or 128); any bit widths and QJL flags.
 * channels   device int16 [Hkv][2][d], 2-byte aligned, owned by the caller:
 *            per KV head, list 0 (keys) and list 1 (values), each a
 *            permutation of 0..d-1 whose first d/2 entries are the channels
 *            coded by `hi` and whose last d/2 are coded by `lo`.  Entries are
 *            taken modulo d; lists that are not permutations give unspecified
 *            (but in-bounds) results.
 * cache_hi, cache_lo  caches of the hi and lo codecs with equal B, Hkv and
 *            rows_cap (tq_cache_bytes with each codec).
 * Bytes per (token, head): the sum of both caches' (keys: d/16 * (planes_hi +
 * planes_lo) + 8; values: d/16 * (bits_v_hi + bits_v_lo) + 4).
 * ------------------------------------------------------------------------ */
typedef struct {
  const tq_codec *hi;
  const tq_codec *lo;
  const int16_t *channels;
} tq_split;

/* Host helper: for each of n rows of score (host fp32 [n][d]), the d/2
 * highest-scoring channels (ties to the lower index) in ascending order, then
 * the other channels ascending -> channels (host int16 [n][d]).  With n = 2 Hkv
 * rows ordered (head, keys|values) the result is the layout above.
 * Errors: TQ_ERR_INVALID_ARG for NULL pointers, n < 1, odd d or a NaN score. */
int tq_split_channels(const float *score, int n, int d, int16_t *channels);

/* Quantize-append into both caches.  Arguments as tq_quantize_kv with d-wide
 * rows of k and v (d = 2 * hi->d); status counts bad half rows (each half is
 * checked on its own). */
int tq_quantize_kv_split(const tq_split *split, const void *k, const void *v, int dtype, int B,
                         int Hkv, int T, int64_t stride_b, int64_t stride_h, int64_t stride_t,
                         const float *rope_cos, const float *rope_sin, int64_t pos0,
                         const tq_cache *cache_hi, const tq_cache *cache_lo, int64_t row0,
                         uint32_t *status, void *stream);

/* Decode over the split caches (CUDA cores, split-K):
 *   l_j = scale * sum over the halves of nu_j (<q'_h, c_h[idx]> +
 *         sqrt(pi/2)/(d/2) rho_j <q''_h, 2 sigma - 1>),
 *   q'_h = Pi_h (RoPE(q, T_b - 1) restricted to half h's key channels),
 * out = each half's sum_j softmax(l)_j nu^v_j Pi_h^T c_v,h[idx] on its value
 * channels.  Arguments as tq_attention_decode (q and out are d wide); the
 * workspace size comes from tq_attention_split_workspace. */
int tq_attention_split_workspace(const tq_split *split, int B, int Hq, int num_splits,
                                 size_t *bytes);
int tq_attention_decode_split(const tq_split *split, const void *q, int dtype, int B, int Hq,
                              int Hkv, const tq_cache *cache_hi, const tq_cache *cache_lo,
                              const int32_t *seq_lens, int max_seq_len, float scale,
                              const float *rope_cos, const float *rope_sin, int num_splits,
                              void *workspace, size_t ws_bytes, float *out, void *stream);

/* Dequantize rows [row0, row0 + rows) of both caches back onto their channels:
 * out device fp32 [B][Hkv][rows][d]. */
int tq_dequantize_split(const tq_split *split, const tq_cache *cache_hi,
                        const tq_cache *cache_lo, int which, int64_t row0, int64_t rows,
                        float *out, void *stream);

/* ------------------------------------------------------------------------
 * FibQuant k = 2: a shared vector code for pairs of rotated coordinates
 * ("FibQuant: Quantizzazione Vettoriale Universale ...", sections 2.1-2.3).
 *
 * Same normalise-rotate interface as the scalar codec (nu = |x|, u = Pi x / nu
 * with the randomized Walsh-Hadamard Pi, RoPE on keys first), but each block
 * (u_2j, u_2j+1) is coded by its nearest codeword of a 2^m-point code of the
 * unit disk, m bits per block: rate m/2 bits per coordinate (0.5 .. 3).  Keys
 * and values both use it (no QJL stage); the logit is
 *   l_j = scale * nu_j * sum_b <q'_(2b, 2b+1), c_k[idx_jb]>,  q' = Pi RoPE(q),
 * and out = Pi^T (sum_j softmax(l)_j nu^v_j concat_b c_v[idx^v_jb]).
 *
 * tq_fq_build_codebook (host, no device work): the code for the law of two
 * coordinates of a uniform point on S^{d-1}, f(x) = (d-2)/(2 pi) (1-|x|^2)^((d-4)/2):
 * codeword n starts at radius sqrt(1 - (1 - (n + delta)/N)^(4/d)) (the
 * Bennett-Gersho density f^(1/2)) and angle n pi (3 - sqrt 5) (golden-angle
 * spiral), then 100 Lloyd steps on a fixed 256 x 256 quadrature of f, from
 * delta = 1/4, 1/2, 3/4, keeping the lowest quadrature MSE.
 *   centroids  host, 2 * 2^bits floats (x0, y0, x1, y1, ...).
 *   mse_per_pair host, nullable: quadrature MSE per block.
 *   Errors: TQ_ERR_INVALID_ARG for d < 4, bits outside 1..8 or NULL output.
 *   Solved once per (d, bits) per process (about a second at 6 bits).
 *
 * Codec: d in {64, 128}, bits_k and bits_v (bits per block) 1..6.  The codec
 * holds no device memory (codebooks travel as kernel parameters), so it can be
 * created without a GPU.
 *
 * Cache planes (struct tq_cache, every plane 16-byte aligned):
 *   kcode  u8 [B][Hkv][rows_cap][bits_k][d/16]: bit p of block j's code at byte
 *          j/8, bit j%8 of plane p.   kscale fp16 [...][rows_cap][2] = (nu, 0).
 *   vcode  u32 [B][Hkv][rows_cap/32][bits_v][d/2]: bit t%32 of word [t/32][p][j]
 *          = bit p of block j's code of token t.   vnorm fp16 [...][rows_cap].
 * The quantize, decode and dequantize calls take the arguments, layouts and
 * error codes of tq_quantize_kv, tq_attention_decode and tq_dequantize.
 * ------------------------------------------------------------------------ */
typedef struct tq_fq_codec tq_fq_codec;

typedef struct {
  int d;
  int bits_k;
  int bits_v;
  const int8_t *rotation_signs;   /* host, d entries of +1 / -1 */
} tq_fq_codec_desc;

int tq_fq_build_codebook(int d, int bits, float *centroids, double *mse_per_pair);
int tq_fq_codec_create(const tq_fq_codec_desc *desc, tq_fq_codec **out);
void tq_fq_codec_destroy(tq_fq_codec *codec);
/* Host copies of the codec's codewords (x, y pairs); either pointer may be NULL. */
int tq_fq_codec_codebooks(const tq_fq_codec *codec, float *ck, float *cv);
int tq_fq_cache_bytes(const tq_fq_codec *codec, int B, int Hkv, int64_t rows_cap,
                      size_t bytes[4]);
int tq_fq_quantize_kv(const tq_fq_codec *codec, const void *k, const void *v, int dtype, int B,
                      int Hkv, int T, int64_t stride_b, int64_t stride_h, int64_t stride_t,
                      const float *rope_cos, const float *rope_sin, int64_t pos0,
                      const tq_cache *cache, int64_t row0, uint32_t *status, void *stream);
int tq_fq_attention_workspace(const tq_fq_codec *codec, int B, int Hq, int num_splits,
                              size_t *bytes);
int tq_fq_attention_decode(const tq_fq_codec *codec, const void *q, int dtype, int B, int Hq,
                           int Hkv, const tq_cache *cache, const int32_t *seq_lens,
                           int max_seq_len, float scale, const float *rope_cos,
                           const float *rope_sin, int num_splits, void *workspace,
                           size_t ws_bytes, float *out, void *stream);
int tq_fq_dequantize(const tq_fq_codec *codec, const tq_cache *cache, int which, int64_t row0,
                     int64_t rows, float *out, void *stream);

/* ------------------------------------------------------------------------
 * Profiling hooks (no counterpart on the pages; used by the benchmark).
 * tq_set_timing_events: when both are non-NULL, every later
 *   tq_attention_decode / tq_attention_logits on this thread records `start`
 *   (a cudaEvent_t) on its stream right before the split-K chunk kernel and
 *   `stop` right after it (event records are captured into CUDA graphs like
 *   any stream work).  Pass NULL, NULL to stop.
 * tq_launch_count: number of kernels this process has launched through the
 *   library so far (all threads).
 * ------------------------------------------------------------------------ */
int tq_set_timing_events(void *start, void *stop);
uint64_t tq_launch_count(void);

/* Message of the last failing call on this thread ("" if none). */
const char *tq_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* TQ_B200_H */
