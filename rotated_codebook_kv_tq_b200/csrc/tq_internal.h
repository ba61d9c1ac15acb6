// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <string>
#include <vector>

#include "../../include/tq.h"

namespace tqhost {
bool lloyd_max(int d, int bits, std::vector<double> &c, std::vector<double> &t, double &mse);
// FibQuant k = 2 pair codebook (fq_codebook.cpp): c = x0, y0, x1, y1, ...
bool fq_pair_codebook(int d, int bits, std::vector<double> &c, double &mse);
// Dense Haar rotation from a d x d Gaussian matrix (haar.cpp), row-major.
bool haar_rotation(int d, const float *g, std::vector<double> &pi);
}

// Largest head dim the kernels are instantiated for.
constexpr int TQ_MAX_D = 1536;
constexpr int TQ_MAX_LEVELS = 16;

// Codebooks and rotation signs passed by value to every kernel (kernel
// parameter space is broadcast-friendly and needs no device allocation).
struct TqBooks {
  float ck[TQ_MAX_LEVELS];   // key centroids (MSE stage)
  float tk[TQ_MAX_LEVELS];   // key thresholds (count = levels - 1)
  float cv[TQ_MAX_LEVELS];   // value centroids
  float tv[TQ_MAX_LEVELS];   // value thresholds
  uint32_t dneg[TQ_MAX_D / 32];  // bit i set <=> D_i = -1
  // dense rotation (device, fp32, row-major), both null for the randomized
  // Walsh-Hadamard Pi = H diag(D) / sqrt(d): pi[i*d + j] = Pi[i][j] and
  // pi_t[j*d + i] = Pi[i][j]
  const float *pi;
  const float *pi_t;
  int mse_bits_k;
  int qjl;
  int bits_v;
};

// Channel map of an outlier-channel split: coordinate i of KV head h's half
// row is channel k[h * hstride + i] (keys) or v[h * hstride + i] (values) of
// the dfull-wide head vector.  k == nullptr: no map.
struct TqRowMap {
  const int16_t *k = nullptr;
  const int16_t *v = nullptr;
  int64_t hstride = 0;
  int dfull = 0;
};

struct tq_codec {
  int d;
  int bits_k, qjl_k, bits_v, mse_bits_k;
  TqBooks books;
  float *rot_dev;      // dense rotation: Pi then Pi^T (2 d^2 floats), or null
  uint16_t *S_dev;     // bf16 [d][d] row-major S[i][j]
  uint16_t *ST_dev;    // bf16 [d][d] transpose, ST[j][i] = S[i][j] (same allocation)
  uint16_t *S_tile;    // d = 1536 only: S as 256 x 64 K-major core-matrix tiles (same allocation)
  // Walsh expansion of the odd-symmetric codebooks: c[idx] = sum_t a_t (2 x_t - 1)
  // over the odd subsets of the code bits (tensor-core decode path)
  float walsh_k[8], walsh_v[8];
  float walsh_k_absmax, walsh_v_sum;
  // 3- and 4-bit codebooks on that path: centroids c_i ~ (V_i - 2^20) / scale
  // as three 7-bit digits of V_i (weights 2^14, 2^7, 1), entries packed four
  // per word
  uint32_t digit_k[3][4], digit_v[3][4];
  float digit_k_scale, digit_v_scale;
  int device;
};

// FibQuant k = 2 codec: 2^bits codewords of the plane per block of two rotated
// coordinates, passed by value to its kernels.
constexpr int FQ_MAX_BITS = 6;
struct FqBooks {
  float2 ck[1 << FQ_MAX_BITS];   // key codewords
  float2 cv[1 << FQ_MAX_BITS];   // value codewords
  uint32_t dneg[4];              // bit i set <=> D_i = -1 (d <= 128)
  int bits_k, bits_v;
};

struct tq_fq_codec {
  int d;
  int bits_k, bits_v;
  double mse_k, mse_v;   // quadrature MSE per block of the two codebooks
  FqBooks books;
};

// Launch `kern` on `stream` allowing programmatic dependent launch: the kernel
// may be scheduled while the previous kernel of the stream is still running,
// and must call pdl_wait() (tq_sm100.cuh) before touching that kernel's output.
template <typename... Params, typename... Args>
cudaError_t tq_launch_pdl(void (*kern)(Params...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Params>(args)...);
}

// Profiling hooks (api.cu).
void tq_count_launch(int n);
void tq_timing_events(cudaEvent_t *start, cudaEvent_t *stop);

// Error reporting (thread-local message).
int tq_fail(int code, const std::string &msg);
int tq_check_launch(const char *what);

// Kernel launchers (defined in the .cu files).
int launch_quantize(const tq_codec *c, const void *k, const void *v, int dtype, int B, int H,
                    int T, int64_t sb, int64_t sh, int64_t st, const float *rc, const float *rs,
                    int64_t pos0, const tq_cache *cache, int64_t row0, uint32_t *status,
                    cudaStream_t stream, const TqRowMap &map = TqRowMap());
// Prefill quantize with one thread per row (quantize_tile.cu); returns
// TQ_ERR_UNSUPPORTED without launching when the call does not fit its rules.
int launch_quantize_tile(const tq_codec *c, const void *k, const void *v, int dtype, int B, int H,
                         int T, int64_t sb, int64_t sh, int64_t st, const float *rc,
                         const float *rs, int64_t pos0, const tq_cache *cache, int64_t row0,
                         uint32_t *status, cudaStream_t stream);
// Prefill quantize for a codec with a dense rotation, the rotation on the
// tensor cores (quantize_rot.cu); TQ_ERR_UNSUPPORTED without launching when
// the codec has no dense rotation.
int launch_quantize_rot(const tq_codec *c, const void *k, const void *v, int dtype, int B, int H,
                        int T, int64_t sb, int64_t sh, int64_t st, const float *rc,
                        const float *rs, int64_t pos0, const tq_cache *cache, int64_t row0,
                        uint32_t *status, cudaStream_t stream);
size_t decode_workspace_bytes(const tq_codec *c, int B, int Hq, int splits);
int launch_decode(const tq_codec *c, const void *q, int dtype, int B, int Hq, int Hkv,
                  const tq_cache *cache, const int32_t *seq_lens, int max_len, float scale,
                  const float *rc, const float *rs, int splits, void *ws, float *out,
                  float *logits, cudaStream_t stream);
size_t bidir_workspace_bytes(const tq_codec *c, int B, int H, int Lq);
int launch_bidir(const tq_codec *c, const void *q, int dtype, int B, int H, int Hkv, int Lq,
                 const tq_cache *cache, int T, float scale, const float *rc, const float *rs,
                 void *ws, float *out, cudaStream_t stream);
// With a map, out is [B][Hkv][rows][map.dfull] and half-row coordinate i lands
// on channel map.k (keys) or map.v (values) of its head.
int launch_dequant(const tq_codec *c, const tq_cache *cache, int which, int64_t row0,
                   int64_t rows, float *out, cudaStream_t stream,
                   const TqRowMap &map = TqRowMap());
// FibQuant k = 2 kernels (fq.cu).
int launch_fq_quantize(const tq_fq_codec *c, const void *k, const void *v, int dtype, int B, int H,
                       int T, int64_t sb, int64_t sh, int64_t st, const float *rc,
                       const float *rs, int64_t pos0, const tq_cache *cache, int64_t row0,
                       uint32_t *status, cudaStream_t stream);
size_t fq_workspace_bytes(const tq_fq_codec *c, int B, int Hq, int splits);
int launch_fq_decode(const tq_fq_codec *c, const void *q, int dtype, int B, int Hq, int Hkv,
                     const tq_cache *cache, const int32_t *seq_lens, int max_len, float scale,
                     const float *rc, const float *rs, int splits, void *ws, float *out,
                     cudaStream_t stream);
int launch_fq_dequant(const tq_fq_codec *c, const tq_cache *cache, int which, int64_t row0,
                      int64_t rows, float *out, cudaStream_t stream);
// Decode over an outlier-channel split cache (split.cu).
size_t split_workspace_bytes(const tq_codec *hi, int B, int Hq, int splits);
int launch_decode_split(const tq_codec *hi, const tq_codec *lo, const int16_t *channels,
                        const void *q, int dtype, int B, int Hq, int Hkv, const tq_cache *chi,
                        const tq_cache *clo, const int32_t *seq_lens, int max_len, float scale,
                        const float *rc, const float *rs, int splits, void *ws, float *out,
                        cudaStream_t stream);
