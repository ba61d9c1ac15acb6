// Split-K decode attention straight from the compressed cache.
//
// Sources: "TurboESM ..." section 2.E (one pass over the compressed cache:
// unpack, residual correction, inverse rotation, attention with online
// softmax; no intermediate dequantized buffer) and section 2.A (RoPE before
// the rotation); "Google presenta TurboQuant ..." ("Eliminacion del sesgo":
// the prod estimator of <q, k> is unbiased).
//
// Three kernels per call:
//   qprep   one warp per query head: q' = Pi RoPE(q), q'' = S q' (fp32).
//   chunk   one CTA per (chunk, KV head, batch): logits of the G query heads
//           of the group from the packed key planes, softmax statistics and the
//           value sum in the rotated domain (unnormalised, relative to the
//           chunk max), written to the workspace.
//   combine one warp per query head: log-sum-exp merge of the chunks, then
//           out = Pi^T o / l = D (H o) / (sqrt(d) l).
#include <math_constants.h>

#include <cstdlib>

#include "tq_device.cuh"
#include "tq_sm100.cuh"
#include "tq_tc.h"

namespace {

constexpr int CMB = 4;   // thread groups of combine_kernel (each sums every 4th split)

constexpr int CT = 256;       // threads of the chunk kernel

struct DecodeArgs {
  const void *q;
  int dtype;
  int B, Hq, Hkv, G;
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
  int splits;
  int chunk;          // rows per chunk (multiple of 32)
  const uint16_t *S;
  const uint16_t *ST;  // S transposed
  float *q1;          // [B][Hq][D]
  float *q2;          // [B][Hq][D]
  float *po;          // [B][Hq][splits][D]
  float *pml;         // [B][Hq][splits][2]
  float *out;         // [B][Hq][D]
  float *logits;      // optional [B][Hq][max_len] (phase-1 logits)
  const uint32_t *err;  // optional: nonzero when the chunk kernel gave up a wait
  TqBooks books;
};

__device__ __forceinline__ int seq_len_of(const DecodeArgs &a, int b) {
  return a.seq_lens ? min(max(a.seq_lens[b], 1), a.max_len) : a.max_len;
}

// One block of D threads per query head.  Warp 0 applies RoPE and the
// rotation (4 or 2 coordinates per lane); then thread i forms
// q''_i = sum_j S[i][j] q'_j from the transposed copy of S (coalesced loads).
template <int D>
__global__ void __launch_bounds__(D) qprep_kernel(DecodeArgs a) {
  constexpr int NPL = D / 32;
  __shared__ float qs[D];
  const int tid = threadIdx.x, lane = tid & 31;
  const int head = blockIdx.x;
  const int b = head / a.Hq;
  const int64_t pos = seq_len_of(a, b) - 1;
  if (tid < 32) {
    float x[NPL];
#pragma unroll
    for (int k = 0; k < NPL; ++k)
      x[k] = tq_load_elem(a.q, static_cast<int64_t>(head) * D + lane + 32 * k, a.dtype);
    if (a.rc != nullptr) {
      constexpr int HALF = NPL / 2;
#pragma unroll
      for (int k = 0; k < HALF; ++k) {
        const float c = a.rc[pos * (D / 2) + lane + 32 * k];
        const float s = a.rs[pos * (D / 2) + lane + 32 * k];
        const float u = x[k], v = x[k + HALF];
        x[k] = u * c - v * s;
        x[k + HALF] = v * c + u * s;
      }
    }
    if (a.books.pi != nullptr) {
#pragma unroll
      for (int k = 0; k < NPL; ++k) qs[lane + 32 * k] = x[k];   // RoPE'd q for the product below
    } else {
      tq_apply_signs<NPL>(x, a.books.dneg, lane);
      tq_warp_wht<NPL>(x, lane);
      const float scl = 1.0f / sqrtf(static_cast<float>(D));
#pragma unroll
      for (int k = 0; k < NPL; ++k) {
        x[k] *= scl;
        a.q1[static_cast<int64_t>(head) * D + lane + 32 * k] = x[k];
        qs[lane + 32 * k] = x[k];
      }
    }
  }
  __syncthreads();
  if (a.books.pi != nullptr) {
    // dense rotation q' = Pi q: thread i takes row i of Pi, sums j = 0 .. d-1
    const float4 *row = reinterpret_cast<const float4 *>(a.books.pi + tid * D);
    float acc = 0.f;
#pragma unroll 8
    for (int c = 0; c < D / 4; ++c) {
      const float4 p = row[c];
      acc = fmaf(p.x, qs[4 * c], acc);
      acc = fmaf(p.y, qs[4 * c + 1], acc);
      acc = fmaf(p.z, qs[4 * c + 2], acc);
      acc = fmaf(p.w, qs[4 * c + 3], acc);
    }
    __syncthreads();
    qs[tid] = acc;
    a.q1[static_cast<int64_t>(head) * D + tid] = acc;
    __syncthreads();
  }
  if (!a.books.qjl) return;
  float acc0 = 0.f, acc1 = 0.f;
#pragma unroll 8
  for (int j = 0; j < D; j += 2) {
    acc0 = fmaf(tq_bf16_to_f32(a.ST[j * D + tid]), qs[j], acc0);
    acc1 = fmaf(tq_bf16_to_f32(a.ST[(j + 1) * D + tid]), qs[j + 1], acc1);
  }
  a.q2[static_cast<int64_t>(head) * D + tid] = acc0 + acc1;
}

template <int D, int G>
__global__ void __launch_bounds__(CT) chunk_kernel(DecodeArgs a) {
  constexpr int NPL = D / 32;
  constexpr int SLICES = CT / D;         // thread groups sharing one coordinate
  constexpr int SUB = G >= 8 ? 512 : 1024;  // rows per pass inside a chunk
  __shared__ float q1s[D][G], q2s[D][G];
  __shared__ float cks[TQ_MAX_LEVELS], cvs[TQ_MAX_LEVELS];
  __shared__ float w[SUB][G];            // logits, then weights p * nu_v
  __shared__ float red[CT / 32][G];
  __shared__ float stat[2][G];           // running max, running sum
  __shared__ float oacc[SLICES][G][D];

  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int len = seq_len_of(a, b);
  const int c0 = split * a.chunk;
  const int c1 = min(len, c0 + a.chunk);
  const int64_t bh = static_cast<int64_t>(b) * a.Hkv + kvh;
  const int hq0 = kvh * G;

  for (int e = tid; e < D * G; e += CT) {
    const int i = e / G, h = e % G;
    const int64_t qi = (static_cast<int64_t>(b) * a.Hq + hq0 + h) * D + i;
    q1s[i][h] = a.q1[qi];
    q2s[i][h] = a.books.qjl ? a.q2[qi] : 0.f;
  }
  if (tid < TQ_MAX_LEVELS) {
    cks[tid] = a.books.ck[tid];
    cvs[tid] = a.books.cv[tid];
  }
  if (tid < G) {
    stat[0][tid] = -CUDART_INF_F;
    stat[1][tid] = 0.f;
  }
  __syncthreads();

  const int planes_k = a.books.mse_bits_k + a.books.qjl;
  const int mbk = a.books.mse_bits_k;
  const int coord = tid % D, slice = tid / D;
  float o[G];
#pragma unroll
  for (int h = 0; h < G; ++h) o[h] = 0.f;

  for (int s0 = c0; s0 < c1; s0 += SUB) {
    const int s1 = min(c1, s0 + SUB);
    // ---------------- phase 1: logits from the key planes (thread per row)
    for (int r = s0 + tid; r < s1; r += CT) {
      const uint32_t *krow = reinterpret_cast<const uint32_t *>(
          a.kcode + (bh * a.rows_cap + r) * planes_k * (D / 8));
      uint32_t kw[4][NPL], sw[NPL];
#pragma unroll
      for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int k = 0; k < NPL; ++k) kw[p][k] = p < mbk ? krow[p * NPL + k] : 0u;
#pragma unroll
      for (int k = 0; k < NPL; ++k) sw[k] = planes_k > mbk ? krow[mbk * NPL + k] : 0u;
      const uint32_t sc = reinterpret_cast<const uint32_t *>(a.kscale)[bh * a.rows_cap + r];
      const float nu = tq_half_to_f32(static_cast<uint16_t>(sc & 0xffffu));
      const float rho = tq_half_to_f32(static_cast<uint16_t>(sc >> 16));
      float acc[G], accs[G];
#pragma unroll
      for (int h = 0; h < G; ++h) acc[h] = accs[h] = 0.f;
#pragma unroll
      for (int k = 0; k < NPL; ++k) {
#pragma unroll 8
        for (int bit = 0; bit < 32; ++bit) {
          const int i = 32 * k + bit;
          int idx = 0;
#pragma unroll
          for (int p = 0; p < 4; ++p)
            if (p < mbk) idx |= ((kw[p][k] >> bit) & 1) << p;
          const float cval = cks[idx];
          const bool sg = (sw[k] >> bit) & 1;
#pragma unroll
          for (int h = 0; h < G; ++h) {
            acc[h] = fmaf(q1s[i][h], cval, acc[h]);
            accs[h] += sg ? q2s[i][h] : -q2s[i][h];
          }
        }
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float est = a.books.qjl ? acc[h] + a.qjl_coef * rho * accs[h] : acc[h];
        const float l = a.scale * nu * est;
        w[r - s0][h] = l;
        if (a.logits)
          a.logits[(static_cast<int64_t>(b) * a.Hq + hq0 + h) * a.max_len + r] = l;
      }
    }
    __syncthreads();
    // ---------------- phase 2: softmax statistics, weights p * nu_v
    float lmax[G];
#pragma unroll
    for (int h = 0; h < G; ++h) lmax[h] = -CUDART_INF_F;
    for (int r = tid; r < s1 - s0; r += CT)
#pragma unroll
      for (int h = 0; h < G; ++h) lmax[h] = fmaxf(lmax[h], w[r][h]);
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float m = tq_warp_max(lmax[h]);
      if (lane == 0) red[warp][h] = m;
    }
    __syncthreads();
    float mnew[G], corr[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float m = red[0][h];
      for (int i = 1; i < CT / 32; ++i) m = fmaxf(m, red[i][h]);
      mnew[h] = fmaxf(stat[0][h], m);
      corr[h] = __expf(stat[0][h] - mnew[h]);
    }
    __syncthreads();
    float lsum[G];
#pragma unroll
    for (int h = 0; h < G; ++h) lsum[h] = 0.f;
    for (int r = tid; r < s1 - s0; r += CT) {
      const float nv = tq_half_to_f32(a.vnorm[bh * a.rows_cap + s0 + r]);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float p = __expf(w[r][h] - mnew[h]);
        lsum[h] += p;
        w[r][h] = p * nv;
      }
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float sm = tq_warp_sum(lsum[h]);
      if (lane == 0) red[warp][h] = sm;
    }
    __syncthreads();
    if (tid < G) {
      float sm = 0.f;
      for (int i = 0; i < CT / 32; ++i) sm += red[i][tid];
      stat[1][tid] = stat[1][tid] * corr[tid] + sm;
      stat[0][tid] = mnew[tid];
    }
#pragma unroll
    for (int h = 0; h < G; ++h) o[h] *= corr[h];
    // ---------------- phase 3: rotated-domain value sum (thread per coordinate)
    const int nbv = a.books.bits_v;
    for (int g = s0 / 32 + slice; g * 32 < s1; g += SLICES) {
      const uint32_t *vg = a.vcode + (bh * (a.rows_cap / 32) + g) * nbv * D + coord;
      uint32_t vw[4];
#pragma unroll
      for (int p = 0; p < 4; ++p) vw[p] = p < nbv ? vg[p * D] : 0u;
      const int rlo = max(s0, g * 32), rhi = min(s1, g * 32 + 32);
      for (int r = rlo; r < rhi; ++r) {
        const int bit = r & 31;
        int idx = 0;
#pragma unroll
        for (int p = 0; p < 4; ++p) idx |= ((vw[p] >> bit) & 1) << p;
        const float cval = cvs[idx];
#pragma unroll
        for (int h = 0; h < G; ++h) o[h] = fmaf(w[r - s0][h], cval, o[h]);
      }
    }
    __syncthreads();
  }
  // reduce the coordinate slices and write the chunk partials
#pragma unroll
  for (int h = 0; h < G; ++h) oacc[slice][h][coord] = o[h];
  __syncthreads();
  for (int e = tid; e < G * D; e += CT) {
    const int h = e / D, i = e % D;
    float s = 0.f;
#pragma unroll
    for (int sl = 0; sl < SLICES; ++sl) s += oacc[sl][h][i];
    const int64_t hq = static_cast<int64_t>(b) * a.Hq + hq0 + h;
    a.po[(hq * a.splits + split) * D + i] = s;
  }
  if (tid < G) {
    const int64_t hq = static_cast<int64_t>(b) * a.Hq + hq0 + tid;
    a.pml[(hq * a.splits + split) * 2 + 0] = stat[0][tid];
    a.pml[(hq * a.splits + split) * 2 + 1] = stat[1][tid];
  }
}

// One block of D threads per query head: log-sum-exp weights of the chunks,
// thread i sums coordinate i over the chunks, then warp 0 applies
// Pi^T = D H / sqrt(d) and the 1/l normalisation.
template <int D>
__global__ void __launch_bounds__(CMB * D) combine_kernel(DecodeArgs a) {
  // CMB groups of D threads: group gq sums splits gq, gq + CMB, ... of every
  // coordinate (short independent load chains), then the groups are added
  constexpr int NPL = D / 32;
  constexpr int MAXS = 512;
  constexpr int NT = CMB * D;
  __shared__ float fs[MAXS];
  __shared__ float red[NT / 32][2];
  __shared__ float os[CMB][D];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = tid % D, gq = tid / D;
  const int64_t head = blockIdx.x;
  const int S = a.splits;
  sm100::pdl_wait();   // the chunk kernel has completed (no-op for a plain launch)
  if (a.err && *a.err) {
    // a bounded wait of the chunk kernel gave up: its partials are incomplete
    if (tid < D) a.out[head * D + tid] = CUDART_NAN_F;
    return;
  }
  // this thread's partial outputs (splits gq, gq + CMB, ...) are loaded
  // first, so their latency overlaps the reductions of the chunk statistics
  constexpr int PMAX = 16;
  const float *po = a.po + head * S * D + c;
  float pv[PMAX];
#pragma unroll
  for (int i = 0; i < PMAX; ++i) {
    const int sp = gq + CMB * i;
    pv[i] = sp < S ? po[static_cast<int64_t>(sp) * D] : 0.f;
  }
  float m = -CUDART_INF_F;
  for (int s = tid; s < S; s += NT) m = fmaxf(m, a.pml[(head * S + s) * 2]);
  m = tq_warp_max(m);
  if (lane == 0) red[warp][0] = m;
  __syncthreads();
  float M = red[0][0];
#pragma unroll
  for (int w = 1; w < NT / 32; ++w) M = fmaxf(M, red[w][0]);
  float l = 0.f;
  for (int s = tid; s < S; s += NT) {
    const float ls = a.pml[(head * S + s) * 2 + 1];
    const float f = ls > 0.f ? __expf(a.pml[(head * S + s) * 2] - M) : 0.f;
    fs[s] = f;
    l += f * ls;
  }
  l = tq_warp_sum(l);
  __syncthreads();
  if (lane == 0) red[warp][1] = l;
  __syncthreads();
  float L = 0.f;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) L += red[w][1];
  float o0 = 0.f, o1 = 0.f;
#pragma unroll
  for (int i = 0; i < PMAX; i += 2) {
    const int s0 = gq + CMB * i, s1 = s0 + CMB;
    if (s0 < S) o0 = fmaf(pv[i], fs[s0], o0);
    if (s1 < S) o1 = fmaf(pv[i + 1], fs[s1], o1);
  }
  int s = gq + CMB * PMAX;   // splits beyond the registers (more than CMB * PMAX)
  for (; s + CMB < S; s += 2 * CMB) {
    o0 = fmaf(po[static_cast<int64_t>(s) * D], fs[s], o0);
    o1 = fmaf(po[static_cast<int64_t>(s + CMB) * D], fs[s + CMB], o1);
  }
  if (s < S) o0 = fmaf(po[static_cast<int64_t>(s) * D], fs[s], o0);
  os[gq][c] = o0 + o1;
  __syncthreads();
  if (a.books.pi != nullptr) {
    // dense rotation: out = Pi^T o / l, thread i takes row i of Pi^T
    float v = 0.f;
    if (tid < D) {
#pragma unroll
      for (int g = 0; g < CMB; ++g) v += os[g][tid];
    }
    __syncthreads();
    if (tid < D) os[0][tid] = v;
    __syncthreads();
    if (tid < D) {
      const float4 *row = reinterpret_cast<const float4 *>(a.books.pi_t + tid * D);
      float acc = 0.f;
#pragma unroll 8
      for (int c4 = 0; c4 < D / 4; ++c4) {
        const float4 p = row[c4];
        acc = fmaf(p.x, os[0][4 * c4], acc);
        acc = fmaf(p.y, os[0][4 * c4 + 1], acc);
        acc = fmaf(p.z, os[0][4 * c4 + 2], acc);
        acc = fmaf(p.w, os[0][4 * c4 + 3], acc);
      }
      a.out[head * D + tid] = acc / L;
    }
    return;
  }
  if (warp == 0) {
    float x[NPL];
#pragma unroll
    for (int k = 0; k < NPL; ++k) {
      float v = 0.f;
#pragma unroll
      for (int g = 0; g < CMB; ++g) v += os[g][lane + 32 * k];
      x[k] = v;
    }
    tq_warp_wht<NPL>(x, lane);
    tq_apply_signs<NPL>(x, a.books.dneg, lane);
    const float norm = 1.0f / (sqrtf(static_cast<float>(D)) * L);
#pragma unroll
    for (int k = 0; k < NPL; ++k) a.out[head * D + lane + 32 * k] = x[k] * norm;
  }
}

template <int D>
int run_decode(DecodeArgs &a, cudaStream_t stream) {
  const int heads = a.B * a.Hq;
  qprep_kernel<D><<<heads, D, 0, stream>>>(a);
  if (int e = tq_check_launch("qprep_kernel")) return e;
  dim3 grid(a.splits, a.Hkv, a.B);
  cudaEvent_t ev0, ev1;
  tq_timing_events(&ev0, &ev1);
  // inside stream capture an event record is only a dependency marker unless
  // it is recorded as an external event node
  unsigned ev_flags = cudaEventRecordDefault;
  if (ev0) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaStreamIsCapturing(stream, &cs);
    if (cs == cudaStreamCaptureStatusActive) ev_flags = cudaEventRecordExternal;
    cudaEventRecordWithFlags(ev0, stream, ev_flags);
  }
  switch (a.G) {
    case 1: chunk_kernel<D, 1><<<grid, CT, 0, stream>>>(a); break;
    case 2: chunk_kernel<D, 2><<<grid, CT, 0, stream>>>(a); break;
    case 4: chunk_kernel<D, 4><<<grid, CT, 0, stream>>>(a); break;
    case 8: chunk_kernel<D, 8><<<grid, CT, 0, stream>>>(a); break;
    default: return tq_fail(TQ_ERR_UNSUPPORTED, "decode: GQA group size must be 1, 2, 4 or 8");
  }
  if (int e = tq_check_launch("chunk_kernel")) return e;
  if (ev1) cudaEventRecordWithFlags(ev1, stream, ev_flags);
  combine_kernel<D><<<heads, CMB * D, 0, stream>>>(a);
  tq_count_launch(3);
  return tq_check_launch("combine_kernel");
}

}  // namespace

namespace {
size_t ws_core_bytes(const tq_codec *c, int B, int Hq, int splits) {
  const size_t heads = static_cast<size_t>(B) * Hq;
  const size_t f = sizeof(float) * heads * (2 * c->d + static_cast<size_t>(splits) * (c->d + 2));
  return (f + 127) / 128 * 128;
}
// Upper bound of the tensor-core path's per-group B-operand region, per
// query head (covers every group size it supports).
size_t ws_bk_bytes(const tq_codec *c, int B, int Hq) {
  if (c->d != 128) return 0;
  const size_t ktot = static_cast<size_t>((1 << (c->mse_bits_k - 1)) + c->qjl_k) * 128;
  return static_cast<size_t>(B) * Hq * (8 * ktot + 144);
}
}  // namespace

// Layout: q', q'', chunk partials (ws_core_bytes) | tensor-core B operands
// (ws_bk_bytes) | one status word (128-byte slot).
size_t decode_workspace_bytes(const tq_codec *c, int B, int Hq, int splits) {
  return ws_core_bytes(c, B, Hq, splits) + ws_bk_bytes(c, B, Hq) + 128;
}

int launch_decode(const tq_codec *c, const void *q, int dtype, int B, int Hq, int Hkv,
                  const tq_cache *cache, const int32_t *seq_lens, int max_len, float scale,
                  const float *rc, const float *rs, int splits, void *ws, float *out,
                  float *logits, cudaStream_t stream) {
  DecodeArgs a;
  a.q = q;
  a.dtype = dtype;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.G = Hq / Hkv;
  a.kcode = cache->kcode;
  a.kscale = cache->kscale;
  a.vcode = cache->vcode;
  a.vnorm = cache->vnorm;
  a.rows_cap = cache->rows_cap;
  a.seq_lens = seq_lens;
  a.max_len = max_len;
  a.scale = scale;
  a.qjl_coef = c->qjl_k ? sqrtf(static_cast<float>(M_PI) / 2.0f) / c->d : 0.f;
  a.rc = rc;
  a.rs = rs;
  a.splits = splits;
  const int per = (max_len + splits - 1) / splits;
  a.chunk = (per + 31) / 32 * 32;
  a.S = c->S_dev;
  a.ST = c->ST_dev;
  const size_t heads = static_cast<size_t>(B) * Hq;
  float *f = static_cast<float *>(ws);
  a.q1 = f;
  a.q2 = f + heads * c->d;
  a.po = f + 2 * heads * c->d;
  a.pml = a.po + heads * static_cast<size_t>(splits) * c->d;
  a.out = out;
  a.logits = logits;
  a.err = nullptr;
  a.books = c->books;
  // TQ_DECODE_IMPL=simt selects the CUDA-core kernels (a complete second
  // implementation, used to cross-check the tensor-core path)
  const char *impl = getenv("TQ_DECODE_IMPL");
  const bool want_tc = !(impl && impl[0] == 's');
  if (want_tc && tc_supported(c, a.G)) {
    uint8_t *bk = static_cast<uint8_t *>(ws) + ws_core_bytes(c, B, Hq, splits);
    uint32_t *err = reinterpret_cast<uint32_t *>(bk + ws_bk_bytes(c, B, Hq));
    a.err = err;
    if (int e = launch_decode_tc(c, q, dtype, B, Hq, Hkv, cache, seq_lens, max_len, scale, rc,
                                 rs, splits, a.po, a.pml, bk, logits, err, stream))
      return e;
    if (tq_launch_pdl(combine_kernel<128>, dim3(B * Hq), dim3(CMB * 128), 0, stream, a) != cudaSuccess)
      return tq_check_launch("combine_kernel");
    tq_count_launch(1);
    return TQ_OK;
  }
  switch (c->d) {
    case 64: return run_decode<64>(a, stream);
    case 128: return run_decode<128>(a, stream);
    default: return tq_fail(TQ_ERR_UNSUPPORTED, "decode: head dim not built");
  }
}
