// C ABI entry points: argument validation, codec lifetime, kernel dispatch.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <string>
#include <vector>

#include "tq_internal.h"

#include <atomic>

namespace {
thread_local std::string g_last_error;
thread_local cudaEvent_t g_ev_start = nullptr, g_ev_stop = nullptr;
std::atomic<uint64_t> g_launches{0};

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool supported_d(int d) { return d == 64 || d == 128 || d == 1536; }

// a_t = 2^-b sum_idx c[idx] prod_{p in S_t} (2 bit_p(idx) - 1) for the odd
// subsets S_t of the b code bits, in increasing bit-mask order.
void walsh_coefficients(const float *c, int bits, float *out, float *absmax, float *sum) {
  int t = 0;
  double amax = 0.0, total = 0.0;
  for (int m = 1; m < (1 << bits) && t < 8; ++m) {
    if (!(__builtin_popcount(m) & 1)) continue;
    double acc = 0.0;
    for (int idx = 0; idx < (1 << bits); ++idx) {
      double sgn = 1.0;
      for (int p = 0; p < bits; ++p)
        if ((m >> p) & 1) sgn *= ((idx >> p) & 1) ? 1.0 : -1.0;
      acc += static_cast<double>(c[idx]) * sgn;
    }
    acc /= static_cast<double>(1 << bits);
    out[t++] = static_cast<float>(acc);
    amax = std::fmax(amax, std::fabs(acc));
    total += acc;
  }
  for (; t < 8; ++t) out[t] = 0.f;
  if (absmax) *absmax = static_cast<float>(amax);
  if (sum) *sum = static_cast<float>(total);
}

// 21-bit fixed-point centroids as three 7-bit digits: V_i = 2^20 + round(c_i F)
// with F = (2^20 - 1) / max |c|, V_i = 2^14 d0 + 2^7 d1 + d2.  tab[k] packs
// digit k of entries 0..15 little-endian, four per word.
void digit_tables(const float *c, int bits, uint32_t tab[3][4], float *scale) {
  const int n = 1 << bits;
  double cmax = 0.0;
  for (int i = 0; i < n; ++i) cmax = std::fmax(cmax, std::fabs(static_cast<double>(c[i])));
  const double F = cmax > 0.0 ? 1048575.0 / cmax : 1.0;
  std::memset(tab, 0, sizeof(uint32_t) * 12);
  for (int i = 0; i < n; ++i) {
    long v = 1048576 + std::lrint(static_cast<double>(c[i]) * F);
    v = v < 0 ? 0 : (v > 2097151 ? 2097151 : v);
    for (int k = 0; k < 3; ++k)
      tab[k][i / 4] |= static_cast<uint32_t>((v >> (14 - 7 * k)) & 127) << (8 * (i % 4));
  }
  *scale = static_cast<float>(F);
}

int check_cache(const tq_codec *c, const tq_cache *cache) {
  if (c && c->d > 128)
    return tq_fail(TQ_ERR_UNSUPPORTED, "KV-cache calls support d = 64 and 128 (d = 1536 is index-only)");
  if (!cache || !cache->kcode || !cache->kscale || !cache->vcode || !cache->vnorm)
    return tq_fail(TQ_ERR_INVALID_ARG, "cache: every plane pointer is required");
  if (cache->B <= 0 || cache->Hkv <= 0 || cache->rows_cap <= 0 || cache->rows_cap % 32)
    return tq_fail(TQ_ERR_INVALID_ARG, "cache: B, Hkv > 0 and rows_cap a positive multiple of 32");
  if (!aligned(cache->kcode, 16) || !aligned(cache->vcode, 16) || !aligned(cache->kscale, 16) ||
      !aligned(cache->vnorm, 16))
    return tq_fail(TQ_ERR_ALIGNMENT, "cache: every plane needs 16-byte alignment");
  (void)c;
  return TQ_OK;
}
}  // namespace

int tq_fail(int code, const std::string &msg) {
  g_last_error = msg;
  return code;
}

void tq_count_launch(int n) { g_launches.fetch_add(static_cast<uint64_t>(n)); }

void tq_timing_events(cudaEvent_t *start, cudaEvent_t *stop) {
  *start = g_ev_start;
  *stop = g_ev_stop;
}

int tq_check_launch(const char *what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return tq_fail(TQ_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
  return TQ_OK;
}

extern "C" {

const char *tq_last_error(void) { return g_last_error.c_str(); }

int tq_set_timing_events(void *start, void *stop) {
  if ((start == nullptr) != (stop == nullptr))
    return tq_fail(TQ_ERR_INVALID_ARG, "timing events: pass both or neither");
  g_ev_start = static_cast<cudaEvent_t>(start);
  g_ev_stop = static_cast<cudaEvent_t>(stop);
  return TQ_OK;
}

uint64_t tq_launch_count(void) { return g_launches.load(); }

int tq_build_codebook(int d, int bits, float *centroids, float *thresholds,
                      double *mse_per_coord) {
  if (!centroids || !thresholds) return tq_fail(TQ_ERR_INVALID_ARG, "codebook: NULL output");
  std::vector<double> c, t;
  double mse = 0.0;
  if (!tqhost::lloyd_max(d, bits, c, t, mse))
    return tq_fail(TQ_ERR_INVALID_ARG, "codebook: need d >= 4 and 1 <= bits <= 8");
  for (size_t i = 0; i < c.size(); ++i) centroids[i] = static_cast<float>(c[i]);
  for (size_t i = 0; i < t.size(); ++i) thresholds[i] = static_cast<float>(t[i]);
  if (mse_per_coord) *mse_per_coord = mse;
  return TQ_OK;
}

int tq_codec_create(const tq_codec_desc *desc, tq_codec **out) {
  if (!desc || !out) return tq_fail(TQ_ERR_INVALID_ARG, "codec: NULL argument");
  *out = nullptr;
  if (!supported_d(desc->d))
    return tq_fail(TQ_ERR_UNSUPPORTED, "codec: d must be 64 or 128 (KV cache) or 1536 (index)");
  const int mse_k = desc->qjl_k ? desc->bits_k - 1 : desc->bits_k;
  if (mse_k < 1 || mse_k > 4 || desc->bits_v < 1 || desc->bits_v > 4)
    return tq_fail(TQ_ERR_UNSUPPORTED,
                   "codec: key MSE bits and value bits must be 1..4 (bits_k >= 2 with QJL)");
  const bool dense = desc->rotation != nullptr;
  if (dense && desc->d > 128)
    return tq_fail(TQ_ERR_UNSUPPORTED, "codec: a dense rotation needs d = 64 or 128");
  if (!dense && !desc->rotation_signs)
    return tq_fail(TQ_ERR_INVALID_ARG, "codec: rotation_signs required without a dense rotation");
  if (desc->qjl_k && !desc->qjl_bf16)
    return tq_fail(TQ_ERR_INVALID_ARG, "codec: qjl_bf16 required when qjl_k != 0");
  if (desc->rotation_signs)
    for (int i = 0; i < desc->d; ++i)
      if (desc->rotation_signs[i] != 1 && desc->rotation_signs[i] != -1)
        return tq_fail(TQ_ERR_INVALID_ARG, "codec: rotation_signs entries must be +1 or -1");
  if (dense) {
    // orthogonality to fp32 accuracy: |Pi Pi^T - I| <= 1e-5 entrywise
    const int d = desc->d;
    for (int i = 0; i < d; ++i)
      for (int j = 0; j < d; ++j) {
        double acc = 0.0;
        for (int k = 0; k < d; ++k)
          acc += static_cast<double>(desc->rotation[static_cast<size_t>(i) * d + k]) *
                 desc->rotation[static_cast<size_t>(j) * d + k];
        if (std::fabs(acc - (i == j ? 1.0 : 0.0)) > 1e-5)
          return tq_fail(TQ_ERR_INVALID_ARG, "codec: the dense rotation is not orthogonal");
      }
  }

  tq_codec *c = new tq_codec();
  std::memset(&c->books, 0, sizeof(c->books));
  c->d = desc->d;
  c->bits_k = desc->bits_k;
  c->qjl_k = desc->qjl_k ? 1 : 0;
  c->bits_v = desc->bits_v;
  c->mse_bits_k = mse_k;
  c->S_dev = nullptr;
  c->rot_dev = nullptr;
  cudaGetDevice(&c->device);

  std::vector<double> cc, tt;
  double mse;
  tqhost::lloyd_max(c->d, mse_k, cc, tt, mse);
  for (size_t i = 0; i < cc.size(); ++i) c->books.ck[i] = static_cast<float>(cc[i]);
  for (size_t i = 0; i < tt.size(); ++i) c->books.tk[i] = static_cast<float>(tt[i]);
  tqhost::lloyd_max(c->d, c->bits_v, cc, tt, mse);
  for (size_t i = 0; i < cc.size(); ++i) c->books.cv[i] = static_cast<float>(cc[i]);
  for (size_t i = 0; i < tt.size(); ++i) c->books.tv[i] = static_cast<float>(tt[i]);
  // unused threshold slots stay above every input (the kernels' code search
  // runs over all TQ_MAX_LEVELS - 1 slots)
  for (int i = (1 << mse_k) - 1; i < TQ_MAX_LEVELS; ++i) c->books.tk[i] = INFINITY;
  for (int i = (1 << c->bits_v) - 1; i < TQ_MAX_LEVELS; ++i) c->books.tv[i] = INFINITY;
  if (desc->rotation_signs)
    for (int i = 0; i < c->d; ++i)
      if (desc->rotation_signs[i] < 0) c->books.dneg[i / 32] |= 1u << (i % 32);
  if (dense) {
    const size_t n = static_cast<size_t>(c->d) * c->d;
    std::vector<float> both(2 * n);
    for (int i = 0; i < c->d; ++i)
      for (int j = 0; j < c->d; ++j) {
        const float v = desc->rotation[static_cast<size_t>(i) * c->d + j];
        both[static_cast<size_t>(i) * c->d + j] = v;       // Pi, row-major
        both[n + static_cast<size_t>(j) * c->d + i] = v;   // Pi^T, row-major
      }
    if (cudaMalloc(&c->rot_dev, both.size() * sizeof(float)) != cudaSuccess) {
      delete c;
      return tq_check_launch("codec: cudaMalloc (rotation)");
    }
    if (cudaMemcpy(c->rot_dev, both.data(), both.size() * sizeof(float), cudaMemcpyHostToDevice) !=
        cudaSuccess) {
      cudaFree(c->rot_dev);
      delete c;
      return tq_check_launch("codec: cudaMemcpy (rotation)");
    }
    c->books.pi = c->rot_dev;
    c->books.pi_t = c->rot_dev + n;
  }
  c->books.mse_bits_k = mse_k;
  c->books.qjl = c->qjl_k;
  walsh_coefficients(c->books.ck, mse_k, c->walsh_k, &c->walsh_k_absmax, nullptr);
  walsh_coefficients(c->books.cv, c->bits_v, c->walsh_v, nullptr, &c->walsh_v_sum);
  digit_tables(c->books.ck, mse_k, c->digit_k, &c->digit_k_scale);
  digit_tables(c->books.cv, c->bits_v, c->digit_v, &c->digit_v_scale);
  c->books.bits_v = c->bits_v;

  c->ST_dev = nullptr;
  c->S_tile = nullptr;
  if (c->qjl_k) {
    const size_t n = static_cast<size_t>(c->d) * c->d;
    // S, S^T, and for d = 1536 (vector search) S again as the sketch GEMM's B
    // operand: K-major core-matrix tiles of 256 output rows x 64 inputs,
    // tile (i / 256, j / 64) at ((i / 256) * (d / 64) + j / 64) * 32 KB
    const bool tiled = c->d == 1536;
    std::vector<uint16_t> both((tiled ? 3 : 2) * n);
    for (int i = 0; i < c->d; ++i)
      for (int j = 0; j < c->d; ++j) {
        const uint16_t v = desc->qjl_bf16[static_cast<size_t>(i) * c->d + j];
        both[static_cast<size_t>(i) * c->d + j] = v;
        both[n + static_cast<size_t>(j) * c->d + i] = v;
        if (tiled) {
          const size_t tile = static_cast<size_t>(i / 256) * (c->d / 64) + j / 64;
          const size_t off = tile * 16384 + ((j % 64) / 8) * 2048 + ((i % 256) / 8) * 64 + (i % 8) * 8 + j % 8;
          both[2 * n + off] = v;
        }
      }
    if (cudaMalloc(&c->S_dev, both.size() * sizeof(uint16_t)) != cudaSuccess) {
      if (c->rot_dev) cudaFree(c->rot_dev);
      delete c;
      return tq_check_launch("codec: cudaMalloc");
    }
    c->ST_dev = c->S_dev + n;
    if (tiled) c->S_tile = c->S_dev + 2 * n;
    if (cudaMemcpy(c->S_dev, both.data(), both.size() * sizeof(uint16_t), cudaMemcpyHostToDevice) !=
        cudaSuccess) {
      cudaFree(c->S_dev);
      if (c->rot_dev) cudaFree(c->rot_dev);
      delete c;
      return tq_check_launch("codec: cudaMemcpy");
    }
  }
  *out = c;
  return TQ_OK;
}

void tq_codec_destroy(tq_codec *codec) {
  if (!codec) return;
  if (codec->S_dev) cudaFree(codec->S_dev);
  if (codec->rot_dev) cudaFree(codec->rot_dev);
  delete codec;
}

int tq_codec_codebooks(const tq_codec *c, float *ck, float *tk, float *cv, float *tv) {
  if (!c) return tq_fail(TQ_ERR_INVALID_ARG, "codebooks: NULL codec");
  const int nk = 1 << c->mse_bits_k, nv = 1 << c->bits_v;
  if (ck) std::memcpy(ck, c->books.ck, sizeof(float) * nk);
  if (tk) std::memcpy(tk, c->books.tk, sizeof(float) * (nk - 1));
  if (cv) std::memcpy(cv, c->books.cv, sizeof(float) * nv);
  if (tv) std::memcpy(tv, c->books.tv, sizeof(float) * (nv - 1));
  return TQ_OK;
}

int tq_cache_bytes(const tq_codec *c, int B, int Hkv, int64_t rows_cap, size_t bytes[4]) {
  if (!c || !bytes || B <= 0 || Hkv <= 0 || rows_cap <= 0 || rows_cap % 32)
    return tq_fail(TQ_ERR_INVALID_ARG, "cache_bytes: bad shape (rows_cap multiple of 32)");
  const size_t rows = static_cast<size_t>(B) * Hkv * rows_cap;
  bytes[0] = rows * (c->mse_bits_k + c->qjl_k) * (c->d / 8);
  bytes[1] = rows * 2 * sizeof(uint16_t);
  bytes[2] = rows / 32 * c->bits_v * c->d * sizeof(uint32_t);
  bytes[3] = rows * sizeof(uint16_t);
  return TQ_OK;
}

int tq_quantize_kv(const tq_codec *c, const void *k, const void *v, int dtype, int B, int Hkv,
                   int T, int64_t stride_b, int64_t stride_h, int64_t stride_t,
                   const float *rope_cos, const float *rope_sin, int64_t pos0,
                   const tq_cache *cache, int64_t row0, uint32_t *status, void *stream) {
  if (!c) return tq_fail(TQ_ERR_INVALID_ARG, "quantize: NULL codec");
  if (int e = check_cache(c, cache)) return e;
  if (dtype != TQ_F32 && dtype != TQ_BF16) return tq_fail(TQ_ERR_INVALID_ARG, "quantize: dtype");
  if (B != cache->B || Hkv != cache->Hkv)
    return tq_fail(TQ_ERR_INVALID_ARG, "quantize: B/Hkv differ from the cache's");
  if (T < 0 || row0 < 0 || row0 + T > cache->rows_cap)
    return tq_fail(TQ_ERR_INVALID_ARG, "quantize: rows [row0, row0+T) outside the cache");
  if (T == 0) return TQ_OK;
  if (!k || !v) return tq_fail(TQ_ERR_INVALID_ARG, "quantize: NULL k or v");
  if ((rope_cos == nullptr) != (rope_sin == nullptr))
    return tq_fail(TQ_ERR_INVALID_ARG, "quantize: rope_cos and rope_sin go together");
  if (rope_cos && pos0 < 0) return tq_fail(TQ_ERR_INVALID_ARG, "quantize: pos0 < 0");
  const size_t es = dtype == TQ_BF16 ? 2 : 4;
  if (!aligned(k, es) || !aligned(v, es))
    return tq_fail(TQ_ERR_ALIGNMENT, "quantize: k/v not aligned to their element size");
  return launch_quantize(c, k, v, dtype, B, Hkv, T, stride_b, stride_h, stride_t, rope_cos,
                         rope_sin, pos0, cache, row0, status, static_cast<cudaStream_t>(stream));
}

int tq_attention_workspace(const tq_codec *c, int B, int Hq, int num_splits, size_t *bytes) {
  if (!c || !bytes || B <= 0 || Hq <= 0 || num_splits < 0)
    return tq_fail(TQ_ERR_INVALID_ARG, "workspace: bad arguments");
  *bytes = decode_workspace_bytes(c, B, Hq, num_splits > 0 ? num_splits : 64);
  return TQ_OK;
}

namespace {
// Split-K chunks per (b, KV head).  Default (num_splits = 0): about one chunk
// per resident CTA (two per SM), 128-row multiples, never more than the 64
// splits a workspace sized with num_splits = 0 holds.
int pick_splits(int num_splits, int max_seq_len, int B, int Hkv) {
  if (num_splits > 0) return num_splits;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int bh = B * Hkv;
  int s = (2 * sms + bh - 1) / bh;
  s = s < 1 ? 1 : (s > 64 ? 64 : s);
  const int chunk = ((max_seq_len + s - 1) / s + 127) / 128 * 128;
  return (max_seq_len + chunk - 1) / chunk;
}

int decode_common(const tq_codec *c, const void *q, int dtype, int B, int Hq, int Hkv,
                  const tq_cache *cache, const int32_t *seq_lens, int max_seq_len, float scale,
                  const float *rope_cos, const float *rope_sin, int num_splits, void *workspace,
                  size_t ws_bytes, float *out, float *logits, void *stream) {
  if (!c) return tq_fail(TQ_ERR_INVALID_ARG, "decode: NULL codec");
  if (int e = check_cache(c, cache)) return e;
  if (!q || !out || !workspace) return tq_fail(TQ_ERR_INVALID_ARG, "decode: NULL q/out/workspace");
  if (dtype != TQ_F32 && dtype != TQ_BF16) return tq_fail(TQ_ERR_INVALID_ARG, "decode: dtype");
  if (B != cache->B || Hkv != cache->Hkv || Hq <= 0 || Hq % Hkv)
    return tq_fail(TQ_ERR_INVALID_ARG, "decode: B/Hkv differ from the cache's or Hq % Hkv != 0");
  if (max_seq_len < 1 || max_seq_len > cache->rows_cap)
    return tq_fail(TQ_ERR_INVALID_ARG, "decode: max_seq_len outside 1..rows_cap");
  if (!std::isfinite(scale)) return tq_fail(TQ_ERR_INVALID_ARG, "decode: scale not finite");
  if ((rope_cos == nullptr) != (rope_sin == nullptr))
    return tq_fail(TQ_ERR_INVALID_ARG, "decode: rope_cos and rope_sin go together");
  const int splits = pick_splits(num_splits, max_seq_len, B, Hkv);
  if (splits > 512) return tq_fail(TQ_ERR_INVALID_ARG, "decode: num_splits must be <= 512");
  if (decode_workspace_bytes(c, B, Hq, splits) > ws_bytes)
    return tq_fail(TQ_ERR_WORKSPACE, "decode: workspace smaller than tq_attention_workspace()");
  if (!aligned(workspace, 16)) return tq_fail(TQ_ERR_ALIGNMENT, "decode: workspace alignment");
  if (!aligned(out, 4) || !aligned(q, dtype == TQ_BF16 ? 2 : 4) || !aligned(logits, 4))
    return tq_fail(TQ_ERR_ALIGNMENT, "decode: q/out/logits alignment");
  return launch_decode(c, q, dtype, B, Hq, Hkv, cache, seq_lens, max_seq_len, scale, rope_cos,
                       rope_sin, splits, workspace, out, logits,
                       static_cast<cudaStream_t>(stream));
}
}  // namespace

int tq_attention_decode(const tq_codec *c, const void *q, int dtype, int B, int Hq, int Hkv,
                        const tq_cache *cache, const int32_t *seq_lens, int max_seq_len,
                        float scale, const float *rope_cos, const float *rope_sin,
                        int num_splits, void *workspace, size_t ws_bytes, float *out,
                        void *stream) {
  return decode_common(c, q, dtype, B, Hq, Hkv, cache, seq_lens, max_seq_len, scale, rope_cos,
                       rope_sin, num_splits, workspace, ws_bytes, out, nullptr, stream);
}

int tq_decode_step(const tq_codec *c, const void *k_new, const void *v_new, int kv_dtype,
                   const void *q, int q_dtype, int B, int Hq, int Hkv, const tq_cache *cache, int T,
                   float scale, const float *rope_cos, const float *rope_sin, int num_splits,
                   void *workspace, size_t ws_bytes, float *out, void *stream) {
  if (!c) return tq_fail(TQ_ERR_INVALID_ARG, "decode step: NULL codec");
  if (T < 1 || (cache && T > cache->rows_cap))
    return tq_fail(TQ_ERR_INVALID_ARG, "decode step: T outside 1..rows_cap");
  const int64_t d = c->d;
  if (int e = tq_quantize_kv(c, k_new, v_new, kv_dtype, B, Hkv, 1, Hkv * d, d, d, rope_cos,
                             rope_sin, T - 1, cache, T - 1, nullptr, stream))
    return e;
  return decode_common(c, q, q_dtype, B, Hq, Hkv, cache, nullptr, T, scale, rope_cos, rope_sin,
                       num_splits, workspace, ws_bytes, out, nullptr, stream);
}

int tq_decode_step_host(const tq_codec *c, const void *in_host, void *in_dev, size_t in_bytes,
                        int kv_dtype, int q_dtype, int B, int Hq, int Hkv, const tq_cache *cache,
                        int T, float scale, const float *rope_cos, const float *rope_sin,
                        int num_splits, void *workspace, size_t ws_bytes, float *out_dev,
                        float *out_host, void *stream) {
  if (!c) return tq_fail(TQ_ERR_INVALID_ARG, "decode step (host): NULL codec");
  if (!in_host || !in_dev || !out_dev || !out_host)
    return tq_fail(TQ_ERR_INVALID_ARG, "decode step (host): NULL buffer");
  const size_t kvs = kv_dtype == TQ_BF16 ? 2 : 4, qs = q_dtype == TQ_BF16 ? 2 : 4;
  if (B <= 0 || Hq <= 0 || Hkv <= 0)
    return tq_fail(TQ_ERR_INVALID_ARG, "decode step (host): bad shape");
  const size_t kv_part = static_cast<size_t>(B) * Hkv * c->d * kvs;
  const size_t q_part = static_cast<size_t>(B) * Hq * c->d * qs;
  if (in_bytes != 2 * kv_part + q_part)
    return tq_fail(TQ_ERR_INVALID_ARG, "decode step (host): in_bytes is not the size of k_new, v_new and q");
  if (reinterpret_cast<uintptr_t>(in_dev) % 16)
    return tq_fail(TQ_ERR_INVALID_ARG, "decode step (host): in_dev not 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  auto cuda_fail = [](cudaError_t e, const char *what) {
    cudaGetLastError();   // the error is reported here, not left for a later call
    return tq_fail(TQ_ERR_CUDA, std::string("decode step (host): ") + what + ": " + cudaGetErrorString(e));
  };
  if (cudaError_t e = cudaMemcpyAsync(in_dev, in_host, in_bytes, cudaMemcpyHostToDevice, st))
    return cuda_fail(e, "input copy");
  const uint8_t *base = static_cast<const uint8_t *>(in_dev);
  if (int e = tq_decode_step(c, base, base + kv_part, kv_dtype, base + 2 * kv_part, q_dtype, B, Hq, Hkv,
                             cache, T, scale, rope_cos, rope_sin, num_splits, workspace, ws_bytes,
                             out_dev, stream))
    return e;
  const size_t out_bytes = static_cast<size_t>(B) * Hq * c->d * sizeof(float);
  if (cudaError_t e = cudaMemcpyAsync(out_host, out_dev, out_bytes, cudaMemcpyDeviceToHost, st))
    return cuda_fail(e, "output copy");
  if (cudaError_t e = cudaStreamSynchronize(st)) return cuda_fail(e, "synchronise");
  return TQ_OK;
}

int tq_attention_logits(const tq_codec *c, const void *q, int dtype, int B, int Hq, int Hkv,
                        const tq_cache *cache, const int32_t *seq_lens, int max_seq_len,
                        float scale, const float *rope_cos, const float *rope_sin,
                        int num_splits, void *workspace, size_t ws_bytes, float *out,
                        float *logits, void *stream) {
  if (!logits) return tq_fail(TQ_ERR_INVALID_ARG, "logits: NULL logits");
  return decode_common(c, q, dtype, B, Hq, Hkv, cache, seq_lens, max_seq_len, scale, rope_cos,
                       rope_sin, num_splits, workspace, ws_bytes, out, logits, stream);
}

int tq_attention_bidir_workspace(const tq_codec *c, int B, int H, int Lq, size_t *bytes) {
  if (!c || !bytes || B <= 0 || H <= 0 || Lq <= 0)
    return tq_fail(TQ_ERR_INVALID_ARG, "bidir workspace: bad arguments");
  *bytes = bidir_workspace_bytes(c, B, H, Lq);
  return TQ_OK;
}

int tq_attention_bidir(const tq_codec *c, const void *q, int dtype, int B, int H, int Hkv,
                       int Lq, const tq_cache *cache, int T, float scale, const float *rope_cos,
                       const float *rope_sin, void *workspace, size_t ws_bytes, float *out,
                       void *stream) {
  if (!c) return tq_fail(TQ_ERR_INVALID_ARG, "bidir: NULL codec");
  if (c->books.pi) return tq_fail(TQ_ERR_UNSUPPORTED, "bidir: built for the Walsh-Hadamard rotation only");
  if (int e = check_cache(c, cache)) return e;
  if (!q || !out || !workspace) return tq_fail(TQ_ERR_INVALID_ARG, "bidir: NULL q/out/workspace");
  if (dtype != TQ_F32 && dtype != TQ_BF16) return tq_fail(TQ_ERR_INVALID_ARG, "bidir: dtype");
  if (B != cache->B || Hkv != cache->Hkv || H <= 0 || H % Hkv || Lq <= 0)
    return tq_fail(TQ_ERR_INVALID_ARG, "bidir: B/Hkv differ from the cache's, H % Hkv, or Lq");
  if (T < 1 || T > cache->rows_cap) return tq_fail(TQ_ERR_INVALID_ARG, "bidir: T outside 1..rows_cap");
  if (!std::isfinite(scale)) return tq_fail(TQ_ERR_INVALID_ARG, "bidir: scale not finite");
  if ((rope_cos == nullptr) != (rope_sin == nullptr))
    return tq_fail(TQ_ERR_INVALID_ARG, "bidir: rope_cos and rope_sin go together");
  if (bidir_workspace_bytes(c, B, H, Lq) > ws_bytes)
    return tq_fail(TQ_ERR_WORKSPACE, "bidir: workspace smaller than tq_attention_bidir_workspace()");
  if (!aligned(workspace, 16) || !aligned(out, 4))
    return tq_fail(TQ_ERR_ALIGNMENT, "bidir: workspace/out alignment");
  return launch_bidir(c, q, dtype, B, H, Hkv, Lq, cache, T, scale, rope_cos, rope_sin, workspace,
                      out, static_cast<cudaStream_t>(stream));
}

int tq_dequantize(const tq_codec *c, const tq_cache *cache, int which, int64_t row0,
                  int64_t rows, float *out, void *stream) {
  if (!c) return tq_fail(TQ_ERR_INVALID_ARG, "dequantize: NULL codec");
  if (int e = check_cache(c, cache)) return e;
  if (which != 0 && which != 1) return tq_fail(TQ_ERR_INVALID_ARG, "dequantize: which is 0 or 1");
  if (row0 < 0 || rows < 0 || row0 + rows > cache->rows_cap)
    return tq_fail(TQ_ERR_INVALID_ARG, "dequantize: rows outside the cache");
  if (rows > 0 && !out) return tq_fail(TQ_ERR_INVALID_ARG, "dequantize: NULL out");
  return launch_dequant(c, cache, which, row0, rows, out, static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------------------
// Outlier-channel split
// ---------------------------------------------------------------------------

namespace {
int check_split(const tq_split *s, const tq_cache *chi, const tq_cache *clo) {
  if (!s || !s->hi || !s->lo || !s->channels)
    return tq_fail(TQ_ERR_INVALID_ARG, "split: NULL codec or channel map");
  if (s->hi->d != s->lo->d || (s->hi->d != 64 && s->hi->d != 128))
    return tq_fail(TQ_ERR_UNSUPPORTED, "split: both codecs need the same d, 64 or 128");
  if (s->hi->books.pi || s->lo->books.pi)
    return tq_fail(TQ_ERR_UNSUPPORTED, "split: built for the Walsh-Hadamard rotation only");
  if (int e = check_cache(s->hi, chi)) return e;
  if (int e = check_cache(s->lo, clo)) return e;
  if (chi->B != clo->B || chi->Hkv != clo->Hkv || chi->rows_cap != clo->rows_cap)
    return tq_fail(TQ_ERR_INVALID_ARG, "split: the two caches differ in B, Hkv or rows_cap");
  if (!aligned(s->channels, 2)) return tq_fail(TQ_ERR_ALIGNMENT, "split: channel map alignment");
  return TQ_OK;
}

// Row maps of the two halves: hi reads entries [0, d/2) of each list, lo
// entries [d/2, d); keys use list 0 and values list 1 of every KV head.
TqRowMap split_map(const tq_split *s, int half) {
  const int d = 2 * s->hi->d;
  TqRowMap m;
  m.k = s->channels + half * (d / 2);
  m.v = s->channels + d + half * (d / 2);
  m.hstride = 2 * d;
  m.dfull = d;
  return m;
}
}  // namespace

int tq_split_channels(const float *score, int n, int d, int16_t *channels) {
  if (!score || !channels || n <= 0 || d < 2 || d % 2 || d > 32767)
    return tq_fail(TQ_ERR_INVALID_ARG, "split_channels: bad arguments");
  std::vector<int> order(d);
  for (int r = 0; r < n; ++r) {
    const float *sr = score + static_cast<size_t>(r) * d;
    for (int i = 0; i < d; ++i) {
      if (std::isnan(sr[i])) return tq_fail(TQ_ERR_INVALID_ARG, "split_channels: NaN score");
      order[i] = i;
    }
    // highest score first, ties to the lower channel
    std::stable_sort(order.begin(), order.end(), [sr](int x, int y) { return sr[x] > sr[y]; });
    std::sort(order.begin(), order.begin() + d / 2);
    std::sort(order.begin() + d / 2, order.end());
    for (int i = 0; i < d; ++i) channels[static_cast<size_t>(r) * d + i] = static_cast<int16_t>(order[i]);
  }
  return TQ_OK;
}

int tq_quantize_kv_split(const tq_split *s, const void *k, const void *v, int dtype, int B,
                         int Hkv, int T, int64_t stride_b, int64_t stride_h, int64_t stride_t,
                         const float *rope_cos, const float *rope_sin, int64_t pos0,
                         const tq_cache *cache_hi, const tq_cache *cache_lo, int64_t row0,
                         uint32_t *status, void *stream) {
  if (int e = check_split(s, cache_hi, cache_lo)) return e;
  if (dtype != TQ_F32 && dtype != TQ_BF16) return tq_fail(TQ_ERR_INVALID_ARG, "quantize split: dtype");
  if (B != cache_hi->B || Hkv != cache_hi->Hkv)
    return tq_fail(TQ_ERR_INVALID_ARG, "quantize split: B/Hkv differ from the caches'");
  if (T < 0 || row0 < 0 || row0 + T > cache_hi->rows_cap)
    return tq_fail(TQ_ERR_INVALID_ARG, "quantize split: rows [row0, row0+T) outside the caches");
  if (T == 0) return TQ_OK;
  if (!k || !v) return tq_fail(TQ_ERR_INVALID_ARG, "quantize split: NULL k or v");
  if ((rope_cos == nullptr) != (rope_sin == nullptr))
    return tq_fail(TQ_ERR_INVALID_ARG, "quantize split: rope_cos and rope_sin go together");
  if (rope_cos && pos0 < 0) return tq_fail(TQ_ERR_INVALID_ARG, "quantize split: pos0 < 0");
  const size_t es = dtype == TQ_BF16 ? 2 : 4;
  if (!aligned(k, es) || !aligned(v, es))
    return tq_fail(TQ_ERR_ALIGNMENT, "quantize split: k/v not aligned to their element size");
  const tq_codec *cd[2] = {s->hi, s->lo};
  const tq_cache *cc[2] = {cache_hi, cache_lo};
  for (int half = 0; half < 2; ++half)
    if (int e = launch_quantize(cd[half], k, v, dtype, B, Hkv, T, stride_b, stride_h, stride_t,
                                rope_cos, rope_sin, pos0, cc[half], row0, status,
                                static_cast<cudaStream_t>(stream), split_map(s, half)))
      return e;
  return TQ_OK;
}

int tq_attention_split_workspace(const tq_split *s, int B, int Hq, int num_splits, size_t *bytes) {
  if (!s || !s->hi || !bytes || B <= 0 || Hq <= 0 || num_splits < 0)
    return tq_fail(TQ_ERR_INVALID_ARG, "split workspace: bad arguments");
  *bytes = split_workspace_bytes(s->hi, B, Hq, num_splits > 0 ? num_splits : 64);
  return TQ_OK;
}

int tq_attention_decode_split(const tq_split *s, const void *q, int dtype, int B, int Hq,
                              int Hkv, const tq_cache *cache_hi, const tq_cache *cache_lo,
                              const int32_t *seq_lens, int max_seq_len, float scale,
                              const float *rope_cos, const float *rope_sin, int num_splits,
                              void *workspace, size_t ws_bytes, float *out, void *stream) {
  if (int e = check_split(s, cache_hi, cache_lo)) return e;
  if (!q || !out || !workspace)
    return tq_fail(TQ_ERR_INVALID_ARG, "split decode: NULL q/out/workspace");
  if (dtype != TQ_F32 && dtype != TQ_BF16) return tq_fail(TQ_ERR_INVALID_ARG, "split decode: dtype");
  if (B != cache_hi->B || Hkv != cache_hi->Hkv || Hq <= 0 || Hq % Hkv)
    return tq_fail(TQ_ERR_INVALID_ARG, "split decode: B/Hkv differ from the caches' or Hq % Hkv != 0");
  if (max_seq_len < 1 || max_seq_len > cache_hi->rows_cap)
    return tq_fail(TQ_ERR_INVALID_ARG, "split decode: max_seq_len outside 1..rows_cap");
  if (!std::isfinite(scale)) return tq_fail(TQ_ERR_INVALID_ARG, "split decode: scale not finite");
  if ((rope_cos == nullptr) != (rope_sin == nullptr))
    return tq_fail(TQ_ERR_INVALID_ARG, "split decode: rope_cos and rope_sin go together");
  const int splits = pick_splits(num_splits, max_seq_len, B, Hkv);
  if (splits > 512) return tq_fail(TQ_ERR_INVALID_ARG, "split decode: num_splits must be <= 512");
  if (split_workspace_bytes(s->hi, B, Hq, splits) > ws_bytes)
    return tq_fail(TQ_ERR_WORKSPACE, "split decode: workspace smaller than tq_attention_split_workspace()");
  if (!aligned(workspace, 16)) return tq_fail(TQ_ERR_ALIGNMENT, "split decode: workspace alignment");
  if (!aligned(out, 4) || !aligned(q, dtype == TQ_BF16 ? 2 : 4))
    return tq_fail(TQ_ERR_ALIGNMENT, "split decode: q/out alignment");
  return launch_decode_split(s->hi, s->lo, s->channels, q, dtype, B, Hq, Hkv, cache_hi, cache_lo,
                             seq_lens, max_seq_len, scale, rope_cos, rope_sin, splits, workspace,
                             out, static_cast<cudaStream_t>(stream));
}

int tq_dequantize_split(const tq_split *s, const tq_cache *cache_hi, const tq_cache *cache_lo,
                        int which, int64_t row0, int64_t rows, float *out, void *stream) {
  if (int e = check_split(s, cache_hi, cache_lo)) return e;
  if (which != 0 && which != 1) return tq_fail(TQ_ERR_INVALID_ARG, "dequantize split: which is 0 or 1");
  if (row0 < 0 || rows < 0 || row0 + rows > cache_hi->rows_cap)
    return tq_fail(TQ_ERR_INVALID_ARG, "dequantize split: rows outside the caches");
  if (rows > 0 && !out) return tq_fail(TQ_ERR_INVALID_ARG, "dequantize split: NULL out");
  const tq_codec *cd[2] = {s->hi, s->lo};
  const tq_cache *cc[2] = {cache_hi, cache_lo};
  for (int half = 0; half < 2; ++half)
    if (int e = launch_dequant(cd[half], cc[half], which, row0, rows, out,
                               static_cast<cudaStream_t>(stream), split_map(s, half)))
      return e;
  return TQ_OK;
}

// ---------------------------------------------------------------------------
// FibQuant k = 2 codec
// ---------------------------------------------------------------------------

int tq_haar_rotation(int d, const float *gaussian, float *rotation) {
  if (!gaussian || !rotation || d < 1 || d > 4096)
    return tq_fail(TQ_ERR_INVALID_ARG, "haar: need 1 <= d <= 4096 and non-NULL buffers");
  for (size_t i = 0; i < static_cast<size_t>(d) * d; ++i)
    if (!std::isfinite(gaussian[i])) return tq_fail(TQ_ERR_INVALID_ARG, "haar: non-finite input");
  std::vector<double> pi;
  tqhost::haar_rotation(d, gaussian, pi);
  for (size_t i = 0; i < pi.size(); ++i) rotation[i] = static_cast<float>(pi[i]);
  return TQ_OK;
}

int tq_fq_build_codebook(int d, int bits, float *centroids, double *mse_per_pair) {
  if (!centroids) return tq_fail(TQ_ERR_INVALID_ARG, "fq codebook: NULL output");
  std::vector<double> c;
  double mse = 0.0;
  if (!tqhost::fq_pair_codebook(d, bits, c, mse))
    return tq_fail(TQ_ERR_INVALID_ARG, "fq codebook: need d >= 4 and 1 <= bits <= 8");
  for (size_t i = 0; i < c.size(); ++i) centroids[i] = static_cast<float>(c[i]);
  if (mse_per_pair) *mse_per_pair = mse;
  return TQ_OK;
}

int tq_fq_codec_create(const tq_fq_codec_desc *desc, tq_fq_codec **out) {
  if (!desc || !out || !desc->rotation_signs)
    return tq_fail(TQ_ERR_INVALID_ARG, "fq codec: NULL descriptor, output or signs");
  *out = nullptr;
  const int d = desc->d;
  if (d != 64 && d != 128) return tq_fail(TQ_ERR_UNSUPPORTED, "fq codec: d must be 64 or 128");
  if (desc->bits_k < 1 || desc->bits_k > FQ_MAX_BITS || desc->bits_v < 1 || desc->bits_v > FQ_MAX_BITS)
    return tq_fail(TQ_ERR_UNSUPPORTED, "fq codec: bits per block must be 1..6");
  tq_fq_codec *c = new tq_fq_codec();
  c->d = d;
  c->bits_k = desc->bits_k;
  c->bits_v = desc->bits_v;
  std::memset(&c->books, 0, sizeof(c->books));
  for (int i = 0; i < d; ++i) {
    const int s = desc->rotation_signs[i];
    if (s != 1 && s != -1) {
      delete c;
      return tq_fail(TQ_ERR_INVALID_ARG, "fq codec: rotation signs must be +1 or -1");
    }
    if (s < 0) c->books.dneg[i / 32] |= 1u << (i % 32);
  }
  std::vector<double> ck, cv;
  tqhost::fq_pair_codebook(d, c->bits_k, ck, c->mse_k);
  tqhost::fq_pair_codebook(d, c->bits_v, cv, c->mse_v);
  for (int n = 0; n < (1 << c->bits_k); ++n)
    c->books.ck[n] = make_float2(static_cast<float>(ck[2 * n]), static_cast<float>(ck[2 * n + 1]));
  for (int n = 0; n < (1 << c->bits_v); ++n)
    c->books.cv[n] = make_float2(static_cast<float>(cv[2 * n]), static_cast<float>(cv[2 * n + 1]));
  c->books.bits_k = c->bits_k;
  c->books.bits_v = c->bits_v;
  *out = c;
  return TQ_OK;
}

void tq_fq_codec_destroy(tq_fq_codec *codec) { delete codec; }

int tq_fq_codec_codebooks(const tq_fq_codec *c, float *ck, float *cv) {
  if (!c) return tq_fail(TQ_ERR_INVALID_ARG, "fq codebooks: NULL codec");
  if (ck) std::memcpy(ck, c->books.ck, sizeof(float) * 2 * (1 << c->bits_k));
  if (cv) std::memcpy(cv, c->books.cv, sizeof(float) * 2 * (1 << c->bits_v));
  return TQ_OK;
}

int tq_fq_cache_bytes(const tq_fq_codec *c, int B, int Hkv, int64_t rows_cap, size_t bytes[4]) {
  if (!c || !bytes || B <= 0 || Hkv <= 0 || rows_cap <= 0 || rows_cap % 32)
    return tq_fail(TQ_ERR_INVALID_ARG, "fq cache_bytes: bad shape (rows_cap multiple of 32)");
  const size_t rows = static_cast<size_t>(B) * Hkv * rows_cap;
  bytes[0] = rows * c->bits_k * (c->d / 16);
  bytes[1] = rows * 2 * sizeof(uint16_t);
  bytes[2] = rows / 32 * c->bits_v * (c->d / 2) * sizeof(uint32_t);
  bytes[3] = rows * sizeof(uint16_t);
  return TQ_OK;
}

int tq_fq_quantize_kv(const tq_fq_codec *c, const void *k, const void *v, int dtype, int B,
                      int Hkv, int T, int64_t stride_b, int64_t stride_h, int64_t stride_t,
                      const float *rope_cos, const float *rope_sin, int64_t pos0,
                      const tq_cache *cache, int64_t row0, uint32_t *status, void *stream) {
  if (!c) return tq_fail(TQ_ERR_INVALID_ARG, "fq quantize: NULL codec");
  if (int e = check_cache(nullptr, cache)) return e;
  if (dtype != TQ_F32 && dtype != TQ_BF16) return tq_fail(TQ_ERR_INVALID_ARG, "fq quantize: dtype");
  if (B != cache->B || Hkv != cache->Hkv)
    return tq_fail(TQ_ERR_INVALID_ARG, "fq quantize: B/Hkv differ from the cache's");
  if (T < 0 || row0 < 0 || row0 + T > cache->rows_cap)
    return tq_fail(TQ_ERR_INVALID_ARG, "fq quantize: rows [row0, row0+T) outside the cache");
  if (T == 0) return TQ_OK;
  if (!k || !v) return tq_fail(TQ_ERR_INVALID_ARG, "fq quantize: NULL k or v");
  if ((rope_cos == nullptr) != (rope_sin == nullptr))
    return tq_fail(TQ_ERR_INVALID_ARG, "fq quantize: rope_cos and rope_sin go together");
  if (rope_cos && pos0 < 0) return tq_fail(TQ_ERR_INVALID_ARG, "fq quantize: pos0 < 0");
  const size_t es = dtype == TQ_BF16 ? 2 : 4;
  if (!aligned(k, es) || !aligned(v, es))
    return tq_fail(TQ_ERR_ALIGNMENT, "fq quantize: k/v not aligned to their element size");
  return launch_fq_quantize(c, k, v, dtype, B, Hkv, T, stride_b, stride_h, stride_t, rope_cos,
                            rope_sin, pos0, cache, row0, status, static_cast<cudaStream_t>(stream));
}

int tq_fq_attention_workspace(const tq_fq_codec *c, int B, int Hq, int num_splits, size_t *bytes) {
  if (!c || !bytes || B <= 0 || Hq <= 0 || num_splits < 0)
    return tq_fail(TQ_ERR_INVALID_ARG, "fq workspace: bad arguments");
  *bytes = fq_workspace_bytes(c, B, Hq, num_splits > 0 ? num_splits : 64);
  return TQ_OK;
}

int tq_fq_attention_decode(const tq_fq_codec *c, const void *q, int dtype, int B, int Hq, int Hkv,
                           const tq_cache *cache, const int32_t *seq_lens, int max_seq_len,
                           float scale, const float *rope_cos, const float *rope_sin,
                           int num_splits, void *workspace, size_t ws_bytes, float *out,
                           void *stream) {
  if (!c) return tq_fail(TQ_ERR_INVALID_ARG, "fq decode: NULL codec");
  if (int e = check_cache(nullptr, cache)) return e;
  if (!q || !out || !workspace) return tq_fail(TQ_ERR_INVALID_ARG, "fq decode: NULL q/out/workspace");
  if (dtype != TQ_F32 && dtype != TQ_BF16) return tq_fail(TQ_ERR_INVALID_ARG, "fq decode: dtype");
  if (B != cache->B || Hkv != cache->Hkv || Hq <= 0 || Hq % Hkv)
    return tq_fail(TQ_ERR_INVALID_ARG, "fq decode: B/Hkv differ from the cache's or Hq % Hkv != 0");
  if (max_seq_len < 1 || max_seq_len > cache->rows_cap)
    return tq_fail(TQ_ERR_INVALID_ARG, "fq decode: max_seq_len outside 1..rows_cap");
  if (!std::isfinite(scale)) return tq_fail(TQ_ERR_INVALID_ARG, "fq decode: scale not finite");
  if ((rope_cos == nullptr) != (rope_sin == nullptr))
    return tq_fail(TQ_ERR_INVALID_ARG, "fq decode: rope_cos and rope_sin go together");
  const int splits = pick_splits(num_splits, max_seq_len, B, Hkv);
  if (splits > 512) return tq_fail(TQ_ERR_INVALID_ARG, "fq decode: num_splits must be <= 512");
  if (fq_workspace_bytes(c, B, Hq, splits) > ws_bytes)
    return tq_fail(TQ_ERR_WORKSPACE, "fq decode: workspace smaller than tq_fq_attention_workspace()");
  if (!aligned(workspace, 16)) return tq_fail(TQ_ERR_ALIGNMENT, "fq decode: workspace alignment");
  if (!aligned(out, 4) || !aligned(q, dtype == TQ_BF16 ? 2 : 4))
    return tq_fail(TQ_ERR_ALIGNMENT, "fq decode: q/out alignment");
  return launch_fq_decode(c, q, dtype, B, Hq, Hkv, cache, seq_lens, max_seq_len, scale, rope_cos,
                          rope_sin, splits, workspace, out, static_cast<cudaStream_t>(stream));
}

int tq_fq_dequantize(const tq_fq_codec *c, const tq_cache *cache, int which, int64_t row0,
                     int64_t rows, float *out, void *stream) {
  if (!c) return tq_fail(TQ_ERR_INVALID_ARG, "fq dequantize: NULL codec");
  if (int e = check_cache(nullptr, cache)) return e;
  if (which != 0 && which != 1) return tq_fail(TQ_ERR_INVALID_ARG, "fq dequantize: which is 0 or 1");
  if (row0 < 0 || rows < 0 || row0 + rows > cache->rows_cap)
    return tq_fail(TQ_ERR_INVALID_ARG, "fq dequantize: rows outside the cache");
  if (rows > 0 && !out) return tq_fail(TQ_ERR_INVALID_ARG, "fq dequantize: NULL out");
  return launch_fq_dequant(c, cache, which, row0, rows, out, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
