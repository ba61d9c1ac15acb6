// Arguments and sizes of the tensor-core decode path (decode_tc.cu).
#pragma once

#include <stdint.h>

#include "tq_internal.h"

// MMA N: 4 limbs per query head, at least 8.
__host__ __device__ constexpr int tc_n(int G) { return 4 * G < 8 ? 8 : 4 * G; }

struct TcArgs {
  const void *q;
  int dtype;
  int B, Hq, Hkv;
  const uint8_t *kcode;
  const uint16_t *kscale;
  const uint32_t *vcode;
  const uint16_t *vnorm;
  int64_t rows_cap;
  const int32_t *seq_lens;
  int max_len;
  float scale;
  float qjl_coef;
  const float *rc;
  const float *rs;
  const uint16_t *S;    // S (bf16, row-major)
  const uint16_t *ST;   // S transposed (bf16)
  int splits;
  int chunk;            // rows per split (multiple of 128)
  int sub;              // rows per shared-memory unit (multiple of 128, <= chunk)
  uint8_t *bk;          // per (b, KV head): B operand bytes then 4 floats per head
  int bk_stride;        // bytes between groups (multiple of 128)
  float *po;            // [B][Hq][splits][128]
  float *pml;           // [B][Hq][splits][2]
  float *logits;        // optional [B][Hq][max_len]
  float wk[8];          // key Walsh coefficients a_S (1- and 2-bit key codebooks)
  float wk_absmax;
  uint32_t ktab[3][4];  // key centroid digits (3- and 4-bit key codebooks)
  float kfc;            // their fixed-point scale
  uint32_t vtab[3][4];  // value centroid digits (3- and 4-bit value codebooks)
  float vcoef[3];       // value: weight of each operand's accumulator
  float vbias;          // value: constant per unit of softmax weight
  uint32_t *err;        // optional device flag set when a bounded wait gives up
  uint32_t wait_limit;  // polls before a wait gives up (TQ_WAIT_LIMIT overrides, for tests)
  TqBooks books;
};

// Whether the tensor-core path has a kernel for this codec / group size.
bool tc_supported(const tq_codec *c, int G);
// Bytes of the per-group B-operand region (one group).
int tc_bk_stride(const tq_codec *c, int G);
int launch_decode_tc(const tq_codec *c, const void *q, int dtype, int B, int Hq, int Hkv,
                     const tq_cache *cache, const int32_t *seq_lens, int max_len, float scale,
                     const float *rc, const float *rs, int splits, float *po, float *pml,
                     uint8_t *bk, float *logits, uint32_t *err, cudaStream_t stream);
