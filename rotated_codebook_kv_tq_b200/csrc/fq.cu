// FibQuant k = 2 cache codec on the GPU: quantize, split-K decode, dequantize.
//
// Source: "FibQuant: Quantizzazione Vettoriale Universale per la Compressione
// della KV-Cache ad Accesso Casuale", section 2.3: store nu = |x|, rotate the
// unit vector (here the codec's randomized Walsh-Hadamard Pi), cut it into
// blocks of k = 2 coordinates and code each block by its nearest codeword of
// the shared code; decode by codeword lookup, inverse rotation and nu.
// "TurboESM ..." sections 2.A and 2.E: RoPE before the rotation, attention in
// one pass over the compressed cache with the values summed in the rotated
// domain and one inverse rotation per output.
//
// Layout (fixed rate, fixed addresses): key row = bits_k planes of d/2 block
// bits (block j at bit j % 32 of word j / 32), kscale (nu, 0) fp16; values in
// 32-token column groups, word [t/32][p][j] bit t % 32 = bit p of block j's
// code of token t, vnorm fp16.
//
// Kernels: fq_quantize (warp per 32-token group, row in registers, shuffle WHT,
// nearest codeword of every block from shared memory, ballots into planes);
// fq_qprep (RoPE + Pi of the query); fq_chunk (thread per key row: one
// codeword lookup and 2G FMAs per block; thread per rotated coordinate for the
// values); fq_combine (log-sum-exp merge, Pi^T); fq_dequant (warp per row).
#include <math_constants.h>

#include "tq_device.cuh"

namespace {

constexpr int FQW = 8;      // warps of fq_quantize_kernel
constexpr int FCT = 256;    // threads of fq_chunk_kernel
constexpr int FCMB = 4;     // thread groups of fq_combine_kernel

__device__ __forceinline__ int fq_nearest(float ux, float uy, const float2 *cb, int n) {
  int best = 0;
  float bd = CUDART_INF_F;
  for (int i = 0; i < n; ++i) {
    const float dx = ux - cb[i].x, dy = uy - cb[i].y;
    const float dd = dx * dx + dy * dy;
    if (dd < bd) {
      bd = dd;
      best = i;
    }
  }
  return best;
}

// nu = |x| (0 for a bad row), x <- Pi x / nu (coordinate lane + 32 k in x[k]).
template <int NPL>
__device__ __forceinline__ float fq_rotate(float (&x)[NPL], const uint32_t *dneg, int lane,
                                           bool &bad) {
  bool finite = true;
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < NPL; ++k) {
    finite &= isfinite(x[k]);
    ss += x[k] * x[k];
  }
  bad = __any_sync(TQ_FULL, !finite);
  float nu = sqrtf(tq_warp_sum(ss));
  if (!bad && isinf(__half2float(__float2half_rn(nu)))) bad = true;
  if (bad) nu = 0.f;
  const float inv = nu > 0.f ? 1.0f / (sqrtf(static_cast<float>(NPL * 32)) * nu) : 0.f;
#pragma unroll
  for (int k = 0; k < NPL; ++k) x[k] = bad ? 0.f : x[k];
  tq_apply_signs<NPL>(x, dneg, lane);
  tq_warp_wht<NPL>(x, lane);
#pragma unroll
  for (int k = 0; k < NPL; ++k) x[k] *= inv;
  return nu;
}

struct FqQuantArgs {
  const void *k, *v;
  int dtype;
  int B, H, T;
  int64_t sb, sh, st;
  const float *rc, *rs;
  int64_t pos0;
  uint8_t *kcode;
  uint16_t *kscale;
  uint32_t *vcode;
  uint16_t *vnorm;
  int64_t rows_cap, row0, g_first, n_groups;
  uint32_t *status;
  FqBooks books;
};

template <int D>
__global__ void __launch_bounds__(FQW * 32) fq_quantize_kernel(FqQuantArgs a) {
  constexpr int NPL = D / 32, NPW = D / 64;   // coordinates per lane, block words per plane
  __shared__ float2 cks[1 << FQ_MAX_BITS], cvs[1 << FQ_MAX_BITS];
  __shared__ float ubuf[FQW][D];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nk = 1 << a.books.bits_k, nv = 1 << a.books.bits_v;
  for (int i = threadIdx.x; i < (1 << FQ_MAX_BITS); i += blockDim.x) {
    cks[i] = a.books.ck[i];
    cvs[i] = a.books.cv[i];
  }
  __syncthreads();
  const int64_t items = static_cast<int64_t>(a.B) * a.H * a.n_groups;
  for (int64_t it = static_cast<int64_t>(blockIdx.x) * FQW + warp; it < items;
       it += static_cast<int64_t>(gridDim.x) * FQW) {
    const int64_t g = a.g_first + it % a.n_groups;
    const int64_t bh = it / a.n_groups;
    const int b = static_cast<int>(bh / a.H), h = static_cast<int>(bh % a.H);
    const int64_t r_begin = max(a.row0, g * 32), r_end = min(a.row0 + a.T, g * 32 + 32);
    uint32_t vw[FQ_MAX_BITS][NPW];
#pragma unroll
    for (int p = 0; p < FQ_MAX_BITS; ++p)
#pragma unroll
      for (int k = 0; k < NPW; ++k) vw[p][k] = 0u;
    for (int64_t r = r_begin; r < r_end; ++r) {
      const int64_t t = r - a.row0;
      const int64_t off = b * a.sb + h * a.sh + t * a.st;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        float x[NPL];
#pragma unroll
        for (int k = 0; k < NPL; ++k) x[k] = tq_load_elem(which ? a.v : a.k, off + lane + 32 * k, a.dtype);
        if (which == 0 && a.rc != nullptr) {
          // rotate-half RoPE, pairs (i, i + d/2) are registers (k, k + NPL/2)
          const int64_t tb = (a.pos0 + t) * (D / 2);
#pragma unroll
          for (int k = 0; k < NPL / 2; ++k) {
            const float c = a.rc[tb + lane + 32 * k], s = a.rs[tb + lane + 32 * k];
            const float u = x[k], w = x[k + NPL / 2];
            x[k] = u * c - w * s;
            x[k + NPL / 2] = w * c + u * s;
          }
        }
        bool bad;
        const float nu = fq_rotate<NPL>(x, a.books.dneg, lane, bad);
#pragma unroll
        for (int k = 0; k < NPL; ++k) ubuf[warp][lane + 32 * k] = x[k];
        __syncwarp();
        int code[NPW];
#pragma unroll
        for (int k = 0; k < NPW; ++k) {
          const int j = lane + 32 * k;
          code[k] = fq_nearest(ubuf[warp][2 * j], ubuf[warp][2 * j + 1], which ? cvs : cks,
                               which ? nv : nk);
        }
        __syncwarp();   // ubuf is rewritten by the next row
        const int64_t crow = bh * a.rows_cap + r;
        if (which == 0) {
          uint32_t myword = 0u;
          for (int p = 0; p < a.books.bits_k; ++p)
#pragma unroll
            for (int k = 0; k < NPW; ++k) {
              const uint32_t w = __ballot_sync(TQ_FULL, (code[k] >> p) & 1);
              if (lane == p * NPW + k) myword = w;
            }
          uint32_t *krow = reinterpret_cast<uint32_t *>(a.kcode + crow * a.books.bits_k * (D / 16));
          if (lane < a.books.bits_k * NPW) krow[lane] = myword;
          if (lane == 0) a.kscale[2 * crow] = tq_f32_to_half(nu), a.kscale[2 * crow + 1] = 0;
        } else {
          const uint32_t bit = 1u << (r & 31);
#pragma unroll
          for (int p = 0; p < FQ_MAX_BITS; ++p)
#pragma unroll
            for (int k = 0; k < NPW; ++k)
              if ((code[k] >> p) & 1) vw[p][k] |= bit;
          if (lane == 0) a.vnorm[crow] = tq_f32_to_half(nu);
        }
        if (lane == 0 && bad && a.status) atomicAdd(a.status, 1u);
      }
    }
    // the group's value words (read-modify-write for partly covered groups)
    const uint32_t nrows = static_cast<uint32_t>(r_end - r_begin);
    const uint32_t mask = nrows == 32 ? TQ_FULL : (((1u << nrows) - 1u) << (r_begin & 31));
    uint32_t *vg = a.vcode + (bh * (a.rows_cap / 32) + g) * a.books.bits_v * (D / 2);
#pragma unroll
    for (int p = 0; p < FQ_MAX_BITS; ++p) {
      if (p >= a.books.bits_v) break;
#pragma unroll
      for (int k = 0; k < NPW; ++k) {
        uint32_t *w = vg + p * (D / 2) + lane + 32 * k;
        if (mask == TQ_FULL) {
          *w = vw[p][k];
        } else {
          atomicAnd(w, ~mask);
          atomicOr(w, vw[p][k] & mask);
        }
      }
    }
  }
}

struct FqDecArgs {
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
  const float *rc, *rs;
  int splits, chunk;
  float *q1;     // [B][Hq][D]
  float *po;     // [B][Hq][splits][D]
  float *pml;    // [B][Hq][splits][2]
  float *out;    // [B][Hq][D]
  FqBooks books;
};

__device__ __forceinline__ int fq_len(const FqDecArgs &a, int b) {
  return a.seq_lens ? min(max(a.seq_lens[b], 1), a.max_len) : a.max_len;
}

// One warp per query head: q' = Pi RoPE(q).
template <int D>
__global__ void __launch_bounds__(32) fq_qprep_kernel(FqDecArgs a) {
  constexpr int NPL = D / 32;
  const int lane = threadIdx.x;
  const int head = blockIdx.x, b = head / a.Hq;
  const int64_t pos = fq_len(a, b) - 1;
  float x[NPL];
#pragma unroll
  for (int k = 0; k < NPL; ++k) x[k] = tq_load_elem(a.q, static_cast<int64_t>(head) * D + lane + 32 * k, a.dtype);
  if (a.rc != nullptr) {
#pragma unroll
    for (int k = 0; k < NPL / 2; ++k) {
      const float c = a.rc[pos * (D / 2) + lane + 32 * k], s = a.rs[pos * (D / 2) + lane + 32 * k];
      const float u = x[k], w = x[k + NPL / 2];
      x[k] = u * c - w * s;
      x[k + NPL / 2] = w * c + u * s;
    }
  }
  tq_apply_signs<NPL>(x, a.books.dneg, lane);
  tq_warp_wht<NPL>(x, lane);
  const float inv = 1.0f / sqrtf(static_cast<float>(D));
#pragma unroll
  for (int k = 0; k < NPL; ++k) a.q1[static_cast<int64_t>(head) * D + lane + 32 * k] = x[k] * inv;
}

// Key row: acc[h] += sum over blocks j of <q'_(2j, 2j+1), c[idx_j]>, with the
// block codes gathered from KB planes of NPW words (only the nb planes the row
// has are read; the generic KB = FQ_MAX_BITS case takes any nb).
template <int KB, int NPW, int G>
__device__ __forceinline__ void fq_key_sums(const uint32_t *krow, int nb, const float2 *cks,
                                            const float (*q1s)[G], float (&acc)[G]) {
#pragma unroll
  for (int k = 0; k < NPW; ++k) {
    uint32_t pw[KB];
#pragma unroll
    for (int p = 0; p < KB; ++p) pw[p] = p < nb ? krow[p * NPW + k] : 0u;
#pragma unroll 4
    for (int t = 0; t < 32; ++t) {
      int idx = 0;
#pragma unroll
      for (int p = 0; p < KB; ++p) idx |= ((pw[p] >> t) & 1) << p;
      const float2 c = cks[idx];
      const int j = 32 * k + t;
#pragma unroll
      for (int h = 0; h < G; ++h) acc[h] = fmaf(q1s[2 * j][h], c.x, fmaf(q1s[2 * j + 1][h], c.y, acc[h]));
    }
  }
}

// Key row from the per-query codeword table: acc[h] += sum over blocks j of
// T[j][idx_j][h], T[j][c][h] = <q'_(2j, 2j+1), c> (16 codewords per block
// at most, G heads per entry).
template <int KB, int NPW, int G>
__device__ __forceinline__ void fq_key_sums_lut(const uint32_t *krow, const float *ktab, float (&acc)[G]) {
#pragma unroll
  for (int k = 0; k < NPW; ++k) {
    uint32_t pw[KB];
#pragma unroll
    for (int p = 0; p < KB; ++p) pw[p] = krow[p * NPW + k];
#pragma unroll 8
    for (int t = 0; t < 32; ++t) {
      int idx = 0;
#pragma unroll
      for (int p = 0; p < KB; ++p) idx |= ((pw[p] >> t) & 1) << p;
      const float *te = ktab + ((32 * k + t) * 16 + idx) * G;
      if constexpr (G == 4) {
        const float4 v = *reinterpret_cast<const float4 *>(te);
        acc[0] += v.x;
        acc[1] += v.y;
        acc[2] += v.z;
        acc[3] += v.w;
      } else {
#pragma unroll
        for (int h = 0; h < G; ++h) acc[h] += te[h];
      }
    }
  }
}

// Values of one 32-token column group for one rotated coordinate (component
// comp of block vg's codes): o[h] += w[r][h] c[idx_r].comp for rows rlo..rhi.
template <int VB, int G>
__device__ __forceinline__ void fq_value_rows(const uint32_t *vg, int nb, int pstride,
                                              const float2 *cvs, int comp, const float (*w)[G],
                                              int s0, int rlo, int rhi, float (&o)[G]) {
  uint32_t vw[VB];
#pragma unroll
  for (int p = 0; p < VB; ++p) vw[p] = p < nb ? vg[p * pstride] : 0u;
  for (int r = rlo; r < rhi; ++r) {
    const int bit = r & 31;
    int idx = 0;
#pragma unroll
    for (int p = 0; p < VB; ++p) idx |= ((vw[p] >> bit) & 1) << p;
    const float2 c = cvs[idx];
    const float val = comp ? c.y : c.x;
#pragma unroll
    for (int h = 0; h < G; ++h) o[h] = fmaf(w[r - s0][h], val, o[h]);
  }
}

template <int D, int G, bool LUT>
__global__ void __launch_bounds__(FCT) fq_chunk_kernel(FqDecArgs a) {
  constexpr int NPW = D / 64;
  constexpr int SLICES = FCT / D;
  constexpr int SUB = G >= 8 ? 512 : 1024;
  // LUT: key codes of at most 4 bits per block read the logit terms
  // <q', c> from a per-query table of (D/2) x 16 x G entries
  __shared__ __align__(16) float ktab[LUT ? (D / 2) * 16 * G : 4];
  __shared__ float q1s[D][G];
  __shared__ float2 cks[1 << FQ_MAX_BITS], cvs[1 << FQ_MAX_BITS];
  __shared__ float w[SUB][G];
  __shared__ float red[FCT / 32][G];
  __shared__ float stat[2][G];
  __shared__ float oacc[SLICES][G][D];

  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int len = fq_len(a, b);
  const int c0 = split * a.chunk;
  const int c1 = min(len, c0 + a.chunk);
  const int64_t bh = static_cast<int64_t>(b) * a.Hkv + kvh;
  const int hq0 = kvh * G;
  for (int e = tid; e < D * G; e += FCT) {
    const int i = e / G, h = e % G;
    q1s[i][h] = a.q1[(static_cast<int64_t>(b) * a.Hq + hq0 + h) * D + i];
  }
  for (int i = tid; i < (1 << FQ_MAX_BITS); i += FCT) {
    cks[i] = a.books.ck[i];
    cvs[i] = a.books.cv[i];
  }
  if (tid < G) {
    stat[0][tid] = -CUDART_INF_F;
    stat[1][tid] = 0.f;
  }
  __syncthreads();
  const int bk = a.books.bits_k, bv = a.books.bits_v;
  if (LUT) {
    for (int e = tid; e < (D / 2) * (1 << bk) * G; e += FCT) {
      const int h = e % G, c = (e / G) % (1 << bk), j = e / (G << bk);
      ktab[(j * 16 + c) * G + h] = fmaf(q1s[2 * j][h], cks[c].x, q1s[2 * j + 1][h] * cks[c].y);
    }
    __syncthreads();
  }
  const int coord = tid % D, slice = tid / D;
  const int blk = coord >> 1, comp = coord & 1;
  float o[G];
#pragma unroll
  for (int h = 0; h < G; ++h) o[h] = 0.f;

  for (int s0 = c0; s0 < c1; s0 += SUB) {
    const int s1 = min(c1, s0 + SUB);
    // ---------------- logits: thread per key row, one codeword per block
    for (int r = s0 + tid; r < s1; r += FCT) {
      const uint32_t *krow =
          reinterpret_cast<const uint32_t *>(a.kcode + (bh * a.rows_cap + r) * bk * (D / 16));
      float acc[G];
#pragma unroll
      for (int h = 0; h < G; ++h) acc[h] = 0.f;
      // the code width selects an instantiation with exactly that many planes
      if constexpr (LUT) {
        switch (bk) {
          case 1: fq_key_sums_lut<1, NPW, G>(krow, ktab, acc); break;
          case 2: fq_key_sums_lut<2, NPW, G>(krow, ktab, acc); break;
          case 3: fq_key_sums_lut<3, NPW, G>(krow, ktab, acc); break;
          default: fq_key_sums_lut<4, NPW, G>(krow, ktab, acc); break;
        }
      } else switch (bk) {
        case 1: fq_key_sums<1, NPW, G>(krow, bk, cks, q1s, acc); break;
        case 2: fq_key_sums<2, NPW, G>(krow, bk, cks, q1s, acc); break;
        case 3: fq_key_sums<3, NPW, G>(krow, bk, cks, q1s, acc); break;
        case 4: fq_key_sums<4, NPW, G>(krow, bk, cks, q1s, acc); break;
        default: fq_key_sums<FQ_MAX_BITS, NPW, G>(krow, bk, cks, q1s, acc); break;   // planes >= bk read as 0
      }
      const float nu = tq_half_to_f32(a.kscale[2 * (bh * a.rows_cap + r)]);
#pragma unroll
      for (int h = 0; h < G; ++h) w[r - s0][h] = a.scale * nu * acc[h];
    }
    __syncthreads();
    // ---------------- softmax statistics, weights p * nu_v
    float lmax[G];
#pragma unroll
    for (int h = 0; h < G; ++h) lmax[h] = -CUDART_INF_F;
    for (int r = tid; r < s1 - s0; r += FCT)
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
      for (int i = 1; i < FCT / 32; ++i) m = fmaxf(m, red[i][h]);
      mnew[h] = fmaxf(stat[0][h], m);
      corr[h] = __expf(stat[0][h] - mnew[h]);
    }
    __syncthreads();
    float lsum[G];
#pragma unroll
    for (int h = 0; h < G; ++h) lsum[h] = 0.f;
    for (int r = tid; r < s1 - s0; r += FCT) {
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
      for (int i = 0; i < FCT / 32; ++i) sm += red[i][tid];
      stat[1][tid] = stat[1][tid] * corr[tid] + sm;
      stat[0][tid] = mnew[tid];
    }
#pragma unroll
    for (int h = 0; h < G; ++h) o[h] *= corr[h];
    // ---------------- values: thread per rotated coordinate
    for (int g = s0 / 32 + slice; g * 32 < s1; g += SLICES) {
      const uint32_t *vg = a.vcode + (bh * (a.rows_cap / 32) + g) * bv * (D / 2) + blk;
      const int rlo = max(s0, g * 32), rhi = min(s1, g * 32 + 32);
      switch (bv) {
        case 1: fq_value_rows<1, G>(vg, bv, D / 2, cvs, comp, w, s0, rlo, rhi, o); break;
        case 2: fq_value_rows<2, G>(vg, bv, D / 2, cvs, comp, w, s0, rlo, rhi, o); break;
        case 3: fq_value_rows<3, G>(vg, bv, D / 2, cvs, comp, w, s0, rlo, rhi, o); break;
        case 4: fq_value_rows<4, G>(vg, bv, D / 2, cvs, comp, w, s0, rlo, rhi, o); break;
        default: fq_value_rows<FQ_MAX_BITS, G>(vg, bv, D / 2, cvs, comp, w, s0, rlo, rhi, o); break;
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int h = 0; h < G; ++h) oacc[slice][h][coord] = o[h];
  __syncthreads();
  for (int e = tid; e < G * D; e += FCT) {
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

// One block per query head: log-sum-exp weights of the chunks, the chunk sum
// of every rotated coordinate, then out = D H o / (sqrt(d) l).
template <int D>
__global__ void __launch_bounds__(FCMB * D) fq_combine_kernel(FqDecArgs a) {
  constexpr int NPL = D / 32, NT = FCMB * D, MAXS = 512;
  __shared__ float fs[MAXS];
  __shared__ float red[NT / 32][2];
  __shared__ float os[FCMB][D];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = tid % D, gq = tid / D;
  const int64_t head = blockIdx.x;
  const int S = a.splits;
  // this thread's partial outputs are loaded first, so their latency
  // overlaps the reductions of the chunk statistics
  constexpr int PMAX = 16;
  float pv[PMAX];
#pragma unroll
  for (int i = 0; i < PMAX; ++i) {
    const int sp = gq + FCMB * i;
    pv[i] = sp < S ? a.po[(head * S + sp) * D + c] : 0.f;
  }
  float m = -CUDART_INF_F;
  for (int s = tid; s < S; s += NT) m = fmaxf(m, a.pml[(head * S + s) * 2]);
  m = tq_warp_max(m);
  if (lane == 0) red[warp][0] = m;
  __syncthreads();
  float M = red[0][0];
#pragma unroll
  for (int i = 1; i < NT / 32; ++i) M = fmaxf(M, red[i][0]);
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
  for (int i = 0; i < NT / 32; ++i) L += red[i][1];
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < PMAX; ++i) {
    const int sp = gq + FCMB * i;
    if (sp < S) acc = fmaf(pv[i], fs[sp], acc);
  }
  for (int s = gq + FCMB * PMAX; s < S; s += FCMB) acc = fmaf(a.po[(head * S + s) * D + c], fs[s], acc);
  os[gq][c] = acc;
  __syncthreads();
  if (warp == 0) {
    float x[NPL];
#pragma unroll
    for (int k = 0; k < NPL; ++k) {
      float v = 0.f;
#pragma unroll
      for (int g = 0; g < FCMB; ++g) v += os[g][lane + 32 * k];
      x[k] = v;
    }
    tq_warp_wht<NPL>(x, lane);
    tq_apply_signs<NPL>(x, a.books.dneg, lane);
    const float norm = 1.0f / (sqrtf(static_cast<float>(D)) * L);
#pragma unroll
    for (int k = 0; k < NPL; ++k) a.out[head * D + lane + 32 * k] = x[k] * norm;
  }
}

struct FqDeqArgs {
  const uint8_t *kcode;
  const uint16_t *kscale;
  const uint32_t *vcode;
  const uint16_t *vnorm;
  int64_t rows_cap;
  int BH;
  int64_t row0, rows;
  int which;
  float *out;
  FqBooks books;
};

// Warp per row: coordinate i = lane + 32 k is component i % 2 of block i / 2.
template <int D>
__global__ void __launch_bounds__(256) fq_dequant_kernel(FqDeqArgs a) {
  constexpr int NPL = D / 32, NPW = D / 64;
  __shared__ float2 cs[1 << FQ_MAX_BITS];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < (1 << FQ_MAX_BITS); i += blockDim.x)
    cs[i] = a.which == 0 ? a.books.ck[i] : a.books.cv[i];
  __syncthreads();
  const int64_t total = static_cast<int64_t>(a.BH) * a.rows;
  for (int64_t it = static_cast<int64_t>(blockIdx.x) * 8 + warp; it < total;
       it += static_cast<int64_t>(gridDim.x) * 8) {
    const int64_t bh = it / a.rows, r = a.row0 + it % a.rows;
    float y[NPL];
    float nu;
    if (a.which == 0) {
      const int bk = a.books.bits_k;
      const uint32_t *krow =
          reinterpret_cast<const uint32_t *>(a.kcode + (bh * a.rows_cap + r) * bk * (D / 16));
#pragma unroll
      for (int k = 0; k < NPL; ++k) {
        const int j = (lane + 32 * k) >> 1;
        int idx = 0;
        for (int p = 0; p < bk; ++p) idx |= ((krow[p * NPW + (j >> 5)] >> (j & 31)) & 1) << p;
        y[k] = (lane & 1) ? cs[idx].y : cs[idx].x;
      }
      nu = tq_half_to_f32(a.kscale[2 * (bh * a.rows_cap + r)]);
    } else {
      const int bv = a.books.bits_v;
      const uint32_t *vg = a.vcode + (bh * (a.rows_cap / 32) + (r >> 5)) * bv * (D / 2);
#pragma unroll
      for (int k = 0; k < NPL; ++k) {
        const int j = (lane + 32 * k) >> 1;
        int idx = 0;
        for (int p = 0; p < bv; ++p) idx |= ((vg[p * (D / 2) + j] >> (r & 31)) & 1) << p;
        y[k] = (lane & 1) ? cs[idx].y : cs[idx].x;
      }
      nu = tq_half_to_f32(a.vnorm[bh * a.rows_cap + r]);
    }
    tq_warp_wht<NPL>(y, lane);
    tq_apply_signs<NPL>(y, a.books.dneg, lane);
    const float f = nu / sqrtf(static_cast<float>(D));
    float *o = a.out + it * D;
#pragma unroll
    for (int k = 0; k < NPL; ++k) o[lane + 32 * k] = y[k] * f;
  }
}

int sm_count() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

template <int D>
int run_fq_decode(FqDecArgs &a, cudaStream_t stream) {
  const int heads = a.B * a.Hq;
  fq_qprep_kernel<D><<<heads, 32, 0, stream>>>(a);
  if (int e = tq_check_launch("fq_qprep_kernel")) return e;
  dim3 grid(a.splits, a.Hkv, a.B);
  cudaEvent_t ev0, ev1;
  tq_timing_events(&ev0, &ev1);
  unsigned ev_flags = cudaEventRecordDefault;
  if (ev0) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaStreamIsCapturing(stream, &cs);
    if (cs == cudaStreamCaptureStatusActive) ev_flags = cudaEventRecordExternal;
    cudaEventRecordWithFlags(ev0, stream, ev_flags);
  }
  // key codes of at most 4 bits per block: logit terms from a per-query table
  const bool lut = a.books.bits_k <= 4;
  switch (a.G) {
    case 1:
      if (lut) fq_chunk_kernel<D, 1, true><<<grid, FCT, 0, stream>>>(a);
      else fq_chunk_kernel<D, 1, false><<<grid, FCT, 0, stream>>>(a);
      break;
    case 2:
      if (lut) fq_chunk_kernel<D, 2, true><<<grid, FCT, 0, stream>>>(a);
      else fq_chunk_kernel<D, 2, false><<<grid, FCT, 0, stream>>>(a);
      break;
    case 4:
      if (lut) fq_chunk_kernel<D, 4, true><<<grid, FCT, 0, stream>>>(a);
      else fq_chunk_kernel<D, 4, false><<<grid, FCT, 0, stream>>>(a);
      break;
    case 8: fq_chunk_kernel<D, 8, false><<<grid, FCT, 0, stream>>>(a); break;
    default: return tq_fail(TQ_ERR_UNSUPPORTED, "fq decode: GQA group size must be 1, 2, 4 or 8");
  }
  if (int e = tq_check_launch("fq_chunk_kernel")) return e;
  if (ev1) cudaEventRecordWithFlags(ev1, stream, ev_flags);
  fq_combine_kernel<D><<<heads, FCMB * D, 0, stream>>>(a);
  tq_count_launch(3);
  return tq_check_launch("fq_combine_kernel");
}

}  // namespace

int launch_fq_quantize(const tq_fq_codec *c, const void *k, const void *v, int dtype, int B, int H,
                       int T, int64_t sb, int64_t sh, int64_t st, const float *rc,
                       const float *rs, int64_t pos0, const tq_cache *cache, int64_t row0,
                       uint32_t *status, cudaStream_t stream) {
  if (T == 0) return TQ_OK;
  FqQuantArgs a;
  a.k = k;
  a.v = v;
  a.dtype = dtype;
  a.B = B;
  a.H = H;
  a.T = T;
  a.sb = sb;
  a.sh = sh;
  a.st = st;
  a.rc = rc;
  a.rs = rs;
  a.pos0 = pos0;
  a.kcode = cache->kcode;
  a.kscale = cache->kscale;
  a.vcode = cache->vcode;
  a.vnorm = cache->vnorm;
  a.rows_cap = cache->rows_cap;
  a.row0 = row0;
  a.g_first = row0 / 32;
  a.n_groups = (row0 + T - 1) / 32 - row0 / 32 + 1;
  a.status = status;
  a.books = c->books;
  const int64_t items = static_cast<int64_t>(B) * H * a.n_groups;
  const int64_t want = (items + FQW - 1) / FQW;
  const int64_t cap = 4LL * sm_count();
  const int grid = static_cast<int>(want < cap ? want : cap);
  switch (c->d) {
    case 64: fq_quantize_kernel<64><<<grid, FQW * 32, 0, stream>>>(a); break;
    case 128: fq_quantize_kernel<128><<<grid, FQW * 32, 0, stream>>>(a); break;
    default: return tq_fail(TQ_ERR_UNSUPPORTED, "fq quantize: head dim not built");
  }
  tq_count_launch(1);
  return tq_check_launch("fq_quantize_kernel");
}

size_t fq_workspace_bytes(const tq_fq_codec *c, int B, int Hq, int splits) {
  const size_t heads = static_cast<size_t>(B) * Hq;
  const size_t f = sizeof(float) * heads * (c->d + static_cast<size_t>(splits) * (c->d + 2));
  return (f + 127) / 128 * 128;
}

int launch_fq_decode(const tq_fq_codec *c, const void *q, int dtype, int B, int Hq, int Hkv,
                     const tq_cache *cache, const int32_t *seq_lens, int max_len, float scale,
                     const float *rc, const float *rs, int splits, void *ws, float *out,
                     cudaStream_t stream) {
  FqDecArgs a;
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
  a.rc = rc;
  a.rs = rs;
  a.splits = splits;
  const int per = (max_len + splits - 1) / splits;
  a.chunk = (per + 31) / 32 * 32;
  const size_t heads = static_cast<size_t>(B) * Hq;
  float *f = static_cast<float *>(ws);
  a.q1 = f;
  a.po = f + heads * c->d;
  a.pml = a.po + heads * static_cast<size_t>(splits) * c->d;
  a.out = out;
  a.books = c->books;
  switch (c->d) {
    case 64: return run_fq_decode<64>(a, stream);
    case 128: return run_fq_decode<128>(a, stream);
    default: return tq_fail(TQ_ERR_UNSUPPORTED, "fq decode: head dim not built");
  }
}

int launch_fq_dequant(const tq_fq_codec *c, const tq_cache *cache, int which, int64_t row0,
                      int64_t rows, float *out, cudaStream_t stream) {
  if (rows == 0) return TQ_OK;
  FqDeqArgs a;
  a.kcode = cache->kcode;
  a.kscale = cache->kscale;
  a.vcode = cache->vcode;
  a.vnorm = cache->vnorm;
  a.rows_cap = cache->rows_cap;
  a.BH = cache->B * cache->Hkv;
  a.row0 = row0;
  a.rows = rows;
  a.which = which;
  a.out = out;
  a.books = c->books;
  const int64_t want = (static_cast<int64_t>(a.BH) * rows + 7) / 8;
  const int64_t cap = 8LL * sm_count();
  const int grid = static_cast<int>(want < cap ? want : cap);
  switch (c->d) {
    case 64: fq_dequant_kernel<64><<<grid, 256, 0, stream>>>(a); break;
    case 128: fq_dequant_kernel<128><<<grid, 256, 0, stream>>>(a); break;
    default: return tq_fail(TQ_ERR_UNSUPPORTED, "fq dequantize: head dim not built");
  }
  tq_count_launch(1);
  return tq_check_launch("fq_dequant_kernel");
}
