// Decode attention over an outlier-channel split cache.
//
// Sources: "Google presenta TurboQuant ..." ("Desempeno teorico y empirico":
// for non-integer rates, outlier channels get more bits than the others, e.g.
// 3 and 2 bits for 2.5 bits per channel); "TurboESM ..." section 2.A (RoPE over
// the head vector before the rotation) and section 2.E (one pass over the
// compressed cache, values summed in the rotated domain, one inverse rotation
// per output).
//
// A head vector of d = 2 DS channels is stored as two independent codecs of
// DS channels each: `hi` codes the outlier channels chan[h][0][0..DS) and `lo`
// the rest chan[h][0][DS..2DS) (keys; chan[h][1] likewise for values).  The
// logit of a key is the sum of both codecs' estimates,
//   l = scale (nu_hi (<q'_hi, c_hi[idx]> + k_hi rho_hi <q''_hi, 2 sigma - 1>)
//            + nu_lo (<q'_lo, c_lo[idx]> + k_lo rho_lo <q''_lo, 2 sigma - 1>)),
// k = sqrt(pi/2)/DS, with q'_half = Pi_half RoPE(q)[channels of the half] and
// q''_half = S_half q'_half; each value half is accumulated in its own rotated
// domain and rotated back by its own Pi_half^T before it lands on its channels.
//
// Three kernels per call (CUDA cores; the same split-K scheme as decode.cu):
//   split_qprep    one block per query head: RoPE over all d channels, the
//                  gather of each half, Pi_half, S_half.
//   split_chunk    one CTA per (chunk, KV head, batch): logits from both key
//                  halves, softmax statistics, both value halves' sums.
//   split_combine  one block per query head: log-sum-exp merge, Pi_half^T,
//                  1/l, scatter of each half to its channels.
#include <math_constants.h>

#include "tq_device.cuh"

namespace {

constexpr int SCT = 256;   // threads of split_chunk_kernel
constexpr int SCMB = 4;    // thread groups of split_combine_kernel

struct SplitArgs {
  const void *q;
  int dtype;
  int B, Hq, Hkv, G;
  const uint8_t *kcode[2];
  const uint16_t *kscale[2];
  const uint32_t *vcode[2];
  const uint16_t *vnorm[2];
  int64_t rows_cap;
  const int32_t *seq_lens;
  int max_len;
  float scale;
  float qjl_coef[2];
  const float *rc;
  const float *rs;
  int splits;
  int chunk;              // rows per chunk (multiple of 32)
  const uint16_t *ST[2];  // S_half transposed (bf16, [DS][DS])
  const int16_t *chan;    // [Hkv][2][d]: key map, value map
  float *q1;              // [B][Hq][d]: q'_hi | q'_lo
  float *q2;              // [B][Hq][d]: q''_hi | q''_lo
  float *po;              // [B][Hq][splits][d]
  float *pml;             // [B][Hq][splits][2]
  float *out;             // [B][Hq][d]
  TqBooks books[2];
};

__device__ __forceinline__ int split_len(const SplitArgs &a, int b) {
  return a.seq_lens ? min(max(a.seq_lens[b], 1), a.max_len) : a.max_len;
}

template <int DS>
__global__ void __launch_bounds__(2 * DS) split_qprep_kernel(SplitArgs a) {
  constexpr int D = 2 * DS, NPS = DS / 32;
  __shared__ float qf[D];       // RoPE'd query, channel order
  __shared__ float qs[2][DS];   // q'_hi, q'_lo
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int head = blockIdx.x;
  const int b = head / a.Hq, kvh = (head % a.Hq) / a.G;
  const int64_t pos = split_len(a, b) - 1;
  {
    // thread c: channel c, rotate-half pair (c, c + DS) of the whole vector
    const int c = tid;
    const int64_t base = static_cast<int64_t>(head) * D;
    float v = tq_load_elem(a.q, base + c, a.dtype);
    if (a.rc != nullptr) {
      const bool first = c < DS;
      const int f = first ? c : c - DS;
      const float w = tq_load_elem(a.q, base + (first ? c + DS : c - DS), a.dtype);
      const float cs = a.rc[pos * DS + f], sn = a.rs[pos * DS + f];
      v = first ? v * cs - w * sn : v * cs + w * sn;
    }
    qf[c] = v;
  }
  __syncthreads();
  if (warp < 2) {
    // warp w gathers half w's channels and rotates them with Pi_w
    const int16_t *ch = a.chan + static_cast<int64_t>(kvh) * 2 * D + warp * DS;
    float x[NPS];
#pragma unroll
    for (int k = 0; k < NPS; ++k) x[k] = qf[ch[lane + 32 * k] & (D - 1)];
    tq_apply_signs<NPS>(x, a.books[warp].dneg, lane);
    tq_warp_wht<NPS>(x, lane);
    const float inv = 1.0f / sqrtf(static_cast<float>(DS));
#pragma unroll
    for (int k = 0; k < NPS; ++k) {
      x[k] *= inv;
      a.q1[static_cast<int64_t>(head) * D + warp * DS + lane + 32 * k] = x[k];
      qs[warp][lane + 32 * k] = x[k];
    }
  }
  __syncthreads();
  // thread (w, i): q''_w[i] = sum_j S_w[i][j] q'_w[j] (coalesced over S_w^T)
  const int w = tid / DS, i = tid % DS;
  float acc = 0.f;
  if (a.books[w].qjl) {
    const uint16_t *st = a.ST[w];
#pragma unroll 8
    for (int j = 0; j < DS; ++j) acc = fmaf(tq_bf16_to_f32(st[j * DS + i]), qs[w][j], acc);
  }
  a.q2[static_cast<int64_t>(head) * D + tid] = acc;
}

// LIN (key codebooks of at most 2 bits): a symmetric codebook of 1 or 2 bits
// is linear in its bit planes, c[idx] = sum_p alpha_p (2 bit_p - 1), and so is
// the sign term; then sum_i q_i (2 b_i - 1) = 2 sum_{b_i = 1} q_i - sum_i q_i,
// and the first sum is read from nibble tables T[n][v] = sum over the set bits
// t of v of q_{4n + t}: one lookup per 4 coordinates, plane and head instead
// of per-coordinate index assembly and multiply-adds.
template <int DS, int G, bool LIN>
__global__ void __launch_bounds__(SCT) split_chunk_kernel(SplitArgs a) {
  constexpr int D = 2 * DS, NPS = DS / 32;
  constexpr int SLICES = SCT / D;         // thread groups sharing one coordinate
  constexpr int SUB = G >= 8 ? 256 : 512;  // rows per pass inside a chunk
  constexpr int NN = LIN ? DS / 4 : 1;     // nibbles of a half
  __shared__ float q1s[D][G], q2s[D][G];
  __shared__ float cks[2][TQ_MAX_LEVELS], cvs[2][TQ_MAX_LEVELS];
  __shared__ float lut[LIN ? 2 * G * 2 : 1][NN][16];   // [(half, head, q'|q'')][nibble][value]
  __shared__ float qsum[2][2][G];                      // [half][q'|q''][head]
  __shared__ float w[2][SUB][G];          // logits, then p * nu_v of each half
  __shared__ float red[SCT / 32][G];
  __shared__ float stat[2][G];            // running max, running sum
  __shared__ float oacc[SLICES][G][D];

  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int len = split_len(a, b);
  const int c0 = split * a.chunk;
  const int c1 = min(len, c0 + a.chunk);
  const int64_t bh = static_cast<int64_t>(b) * a.Hkv + kvh;
  const int hq0 = kvh * G;

  for (int e = tid; e < D * G; e += SCT) {
    const int i = e / G, h = e % G;
    const int64_t qi = (static_cast<int64_t>(b) * a.Hq + hq0 + h) * D + i;
    q1s[i][h] = a.q1[qi];
    q2s[i][h] = a.q2[qi];
  }
  if (tid < 2 * TQ_MAX_LEVELS) {
    const int hf = tid / TQ_MAX_LEVELS, m = tid % TQ_MAX_LEVELS;
    cks[hf][m] = a.books[hf].ck[m];
    cvs[hf][m] = a.books[hf].cv[m];
  }
  if (tid < G) {
    stat[0][tid] = -CUDART_INF_F;
    stat[1][tid] = 0.f;
  }
  __syncthreads();
  if (LIN) {
    for (int e = tid; e < 2 * G * 2 * NN * 16; e += SCT) {
      const int v = e & 15, n = (e >> 4) % NN, tab = (e >> 4) / NN;
      const int vec = tab & 1, h = (tab >> 1) % G, hf = (tab >> 1) / G;
      float acc = 0.f;
#pragma unroll
      for (int t = 0; t < 4; ++t)
        if ((v >> t) & 1) acc += vec ? q2s[hf * DS + 4 * n + t][h] : q1s[hf * DS + 4 * n + t][h];
      lut[tab][n][v] = acc;
    }
    if (tid < 4 * G) {
      const int h = tid % G, vec = (tid / G) & 1, hf = tid / (2 * G);
      float acc = 0.f;
      for (int i = 0; i < DS; ++i) acc += vec ? q2s[hf * DS + i][h] : q1s[hf * DS + i][h];
      qsum[hf][vec][h] = acc;
    }
    __syncthreads();
  }

  const int coord = tid % D, slice = tid / D;
  const int vhalf = coord / DS, vcol = coord % DS;
  const int nbv = a.books[vhalf].bits_v;
  float o[G];
#pragma unroll
  for (int h = 0; h < G; ++h) o[h] = 0.f;

  for (int s0 = c0; s0 < c1; s0 += SUB) {
    const int s1 = min(c1, s0 + SUB);
    // ---------------- phase 1: logits from both key halves (thread per row)
    for (int r = s0 + tid; r < s1; r += SCT) {
      float tot[G];
#pragma unroll
      for (int h = 0; h < G; ++h) tot[h] = 0.f;
      if (LIN) {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int mbk = a.books[hf].mse_bits_k;
          const int qjl = a.books[hf].qjl;
          const uint32_t *krow = reinterpret_cast<const uint32_t *>(
              a.kcode[hf] + (bh * a.rows_cap + r) * (mbk + qjl) * (DS / 8));
          const uint32_t sc = reinterpret_cast<const uint32_t *>(a.kscale[hf])[bh * a.rows_cap + r];
          const float nu = tq_half_to_f32(static_cast<uint16_t>(sc & 0xffffu));
          const float rho = tq_half_to_f32(static_cast<uint16_t>(sc >> 16));
          // plane p < mbk: alpha_p; the sign plane: coef rho
          const float c0 = cks[hf][0], c1 = cks[hf][1], c2 = cks[hf][2];
          float est[G];
#pragma unroll
          for (int h = 0; h < G; ++h) est[h] = 0.f;
#pragma unroll
          for (int p = 0; p < 3; ++p) {
            if (p >= mbk + qjl) break;
            const bool sgn = p == mbk;
            const float coefp = sgn ? a.qjl_coef[hf] * rho
                                    : (mbk == 1 ? 0.5f * (c1 - c0) : (p == 0 ? 0.5f * (c1 - c0) : 0.5f * (c2 - c0)));
            const int tab0 = sgn ? 1 : 0;
            float acc[G];
#pragma unroll
            for (int h = 0; h < G; ++h) acc[h] = 0.f;
#pragma unroll
            for (int k = 0; k < NPS; ++k) {
              const uint32_t wd = krow[p * NPS + k];
#pragma unroll
              for (int n8 = 0; n8 < 8; ++n8) {
                const int v = (wd >> (4 * n8)) & 15, n = 8 * k + n8;
#pragma unroll
                for (int h = 0; h < G; ++h) acc[h] += lut[(hf * G + h) * 2 + tab0][n][v];
              }
            }
#pragma unroll
            for (int h = 0; h < G; ++h) est[h] = fmaf(coefp, 2.f * acc[h] - qsum[hf][tab0][h], est[h]);
          }
#pragma unroll
          for (int h = 0; h < G; ++h) tot[h] = fmaf(nu, est[h], tot[h]);
        }
#pragma unroll
        for (int h = 0; h < G; ++h) w[0][r - s0][h] = a.scale * tot[h];
        continue;
      }
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int mbk = a.books[hf].mse_bits_k;
        const int qjl = a.books[hf].qjl;
        const uint32_t *krow = reinterpret_cast<const uint32_t *>(
            a.kcode[hf] + (bh * a.rows_cap + r) * (mbk + qjl) * (DS / 8));
        uint32_t kw[4][NPS], sw[NPS];
#pragma unroll
        for (int p = 0; p < 4; ++p)
#pragma unroll
          for (int k = 0; k < NPS; ++k) kw[p][k] = p < mbk ? krow[p * NPS + k] : 0u;
#pragma unroll
        for (int k = 0; k < NPS; ++k) sw[k] = qjl ? krow[mbk * NPS + k] : 0u;
        const uint32_t sc = reinterpret_cast<const uint32_t *>(a.kscale[hf])[bh * a.rows_cap + r];
        const float nu = tq_half_to_f32(static_cast<uint16_t>(sc & 0xffffu));
        const float rho = tq_half_to_f32(static_cast<uint16_t>(sc >> 16));
        float acc[G], accs[G];
#pragma unroll
        for (int h = 0; h < G; ++h) acc[h] = accs[h] = 0.f;
#pragma unroll
        for (int k = 0; k < NPS; ++k) {
#pragma unroll 8
          for (int bit = 0; bit < 32; ++bit) {
            const int i = hf * DS + 32 * k + bit;
            int idx = 0;
#pragma unroll
            for (int p = 0; p < 4; ++p) idx |= ((kw[p][k] >> bit) & 1) << p;
            const float cval = cks[hf][idx];
            const bool sg = (sw[k] >> bit) & 1;
#pragma unroll
            for (int h = 0; h < G; ++h) {
              acc[h] = fmaf(q1s[i][h], cval, acc[h]);
              accs[h] += sg ? q2s[i][h] : -q2s[i][h];
            }
          }
        }
#pragma unroll
        for (int h = 0; h < G; ++h)
          tot[h] = fmaf(nu, qjl ? acc[h] + a.qjl_coef[hf] * rho * accs[h] : acc[h], tot[h]);
      }
#pragma unroll
      for (int h = 0; h < G; ++h) w[0][r - s0][h] = a.scale * tot[h];
    }
    __syncthreads();
    // ---------------- phase 2: softmax statistics, weights p * nu_v per half
    float lmax[G];
#pragma unroll
    for (int h = 0; h < G; ++h) lmax[h] = -CUDART_INF_F;
    for (int r = tid; r < s1 - s0; r += SCT)
#pragma unroll
      for (int h = 0; h < G; ++h) lmax[h] = fmaxf(lmax[h], w[0][r][h]);
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
      for (int i = 1; i < SCT / 32; ++i) m = fmaxf(m, red[i][h]);
      mnew[h] = fmaxf(stat[0][h], m);
      corr[h] = __expf(stat[0][h] - mnew[h]);
    }
    __syncthreads();
    float lsum[G];
#pragma unroll
    for (int h = 0; h < G; ++h) lsum[h] = 0.f;
    for (int r = tid; r < s1 - s0; r += SCT) {
      const float nv0 = tq_half_to_f32(a.vnorm[0][bh * a.rows_cap + s0 + r]);
      const float nv1 = tq_half_to_f32(a.vnorm[1][bh * a.rows_cap + s0 + r]);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float p = __expf(w[0][r][h] - mnew[h]);
        lsum[h] += p;
        w[0][r][h] = p * nv0;
        w[1][r][h] = p * nv1;
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
      for (int i = 0; i < SCT / 32; ++i) sm += red[i][tid];
      stat[1][tid] = stat[1][tid] * corr[tid] + sm;
      stat[0][tid] = mnew[tid];
    }
#pragma unroll
    for (int h = 0; h < G; ++h) o[h] *= corr[h];
    // ---------------- phase 3: value sums in each half's rotated domain
    for (int g = s0 / 32 + slice; g * 32 < s1; g += SLICES) {
      const uint32_t *vg = a.vcode[vhalf] + (bh * (a.rows_cap / 32) + g) * nbv * DS + vcol;
      uint32_t vw[4];
#pragma unroll
      for (int p = 0; p < 4; ++p) vw[p] = p < nbv ? vg[p * DS] : 0u;
      const int rlo = max(s0, g * 32), rhi = min(s1, g * 32 + 32);
      for (int r = rlo; r < rhi; ++r) {
        const int bit = r & 31;
        int idx = 0;
#pragma unroll
        for (int p = 0; p < 4; ++p) idx |= ((vw[p] >> bit) & 1) << p;
        const float cval = cvs[vhalf][idx];
#pragma unroll
        for (int h = 0; h < G; ++h) o[h] = fmaf(w[vhalf][r - s0][h], cval, o[h]);
      }
    }
    __syncthreads();
  }
  // reduce the coordinate slices and write the chunk partials
#pragma unroll
  for (int h = 0; h < G; ++h) oacc[slice][h][coord] = o[h];
  __syncthreads();
  for (int e = tid; e < G * D; e += SCT) {
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
// of every rotated-domain coordinate, then warp w applies Pi_w^T = D_w H / sqrt(DS)
// and 1/l to half w and writes it to the head's value channels of that half.
template <int DS>
__global__ void __launch_bounds__(SCMB * 2 * DS) split_combine_kernel(SplitArgs a) {
  constexpr int D = 2 * DS, NPS = DS / 32;
  constexpr int MAXS = 512;
  constexpr int NT = SCMB * D;
  __shared__ float fs[MAXS];
  __shared__ float red[NT / 32][2];
  __shared__ float os[SCMB][D];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = tid % D, gq = tid / D;
  const int64_t head = blockIdx.x;
  const int kvh = static_cast<int>(head % a.Hq) / a.G;
  const int S = a.splits;
  // this thread's partial outputs are loaded first, so their latency
  // overlaps the reductions of the chunk statistics
  constexpr int PMAX = 16;
  const float *po = a.po + head * S * D + c;
  float pv[PMAX];
#pragma unroll
  for (int i = 0; i < PMAX; ++i) {
    const int sp = gq + SCMB * i;
    pv[i] = sp < S ? po[static_cast<int64_t>(sp) * D] : 0.f;
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
  float o0 = 0.f, o1 = 0.f;
#pragma unroll
  for (int i = 0; i < PMAX; i += 2) {
    const int s0 = gq + SCMB * i, s1 = s0 + SCMB;
    if (s0 < S) o0 = fmaf(pv[i], fs[s0], o0);
    if (s1 < S) o1 = fmaf(pv[i + 1], fs[s1], o1);
  }
  int s = gq + SCMB * PMAX;   // splits beyond the registers
  for (; s + SCMB < S; s += 2 * SCMB) {
    o0 = fmaf(po[static_cast<int64_t>(s) * D], fs[s], o0);
    o1 = fmaf(po[static_cast<int64_t>(s + SCMB) * D], fs[s + SCMB], o1);
  }
  if (s < S) o0 = fmaf(po[static_cast<int64_t>(s) * D], fs[s], o0);
  os[gq][c] = o0 + o1;
  __syncthreads();
  if (warp < 2) {
    float x[NPS];
#pragma unroll
    for (int k = 0; k < NPS; ++k) {
      float v = 0.f;
#pragma unroll
      for (int g = 0; g < SCMB; ++g) v += os[g][warp * DS + lane + 32 * k];
      x[k] = v;
    }
    tq_warp_wht<NPS>(x, lane);
    tq_apply_signs<NPS>(x, a.books[warp].dneg, lane);
    const float norm = 1.0f / (sqrtf(static_cast<float>(DS)) * L);
    const int16_t *ch = a.chan + static_cast<int64_t>(kvh) * 2 * D + D + warp * DS;
#pragma unroll
    for (int k = 0; k < NPS; ++k) a.out[head * D + (ch[lane + 32 * k] & (D - 1))] = x[k] * norm;
  }
}

template <int DS, int G>
void launch_chunk(SplitArgs &a, dim3 grid, cudaStream_t stream) {
  // the table path for key codebooks of at most 2 bits (d/2 = 64, G <= 4:
  // its tables fit the static shared memory)
  const bool lin = DS == 64 && G <= 4 && a.books[0].mse_bits_k <= 2 && a.books[1].mse_bits_k <= 2;
  if (lin)
    split_chunk_kernel<DS, G, DS == 64 && G <= 4><<<grid, SCT, 0, stream>>>(a);
  else
    split_chunk_kernel<DS, G, false><<<grid, SCT, 0, stream>>>(a);
}

template <int DS>
int run_split(SplitArgs &a, cudaStream_t stream) {
  const int heads = a.B * a.Hq;
  split_qprep_kernel<DS><<<heads, 2 * DS, 0, stream>>>(a);
  if (int e = tq_check_launch("split_qprep_kernel")) return e;
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
  switch (a.G) {
    case 1: launch_chunk<DS, 1>(a, grid, stream); break;
    case 2: launch_chunk<DS, 2>(a, grid, stream); break;
    case 4: launch_chunk<DS, 4>(a, grid, stream); break;
    case 8: launch_chunk<DS, 8>(a, grid, stream); break;
    default: return tq_fail(TQ_ERR_UNSUPPORTED, "split decode: GQA group size must be 1, 2, 4 or 8");
  }
  if (int e = tq_check_launch("split_chunk_kernel")) return e;
  if (ev1) cudaEventRecordWithFlags(ev1, stream, ev_flags);
  split_combine_kernel<DS><<<heads, SCMB * 2 * DS, 0, stream>>>(a);
  tq_count_launch(3);
  return tq_check_launch("split_combine_kernel");
}

}  // namespace

// q', q'', chunk partials and statistics, all fp32 (d = 2 * hi->d).
size_t split_workspace_bytes(const tq_codec *hi, int B, int Hq, int splits) {
  const size_t heads = static_cast<size_t>(B) * Hq, d = 2 * static_cast<size_t>(hi->d);
  const size_t f = sizeof(float) * heads * (2 * d + static_cast<size_t>(splits) * (d + 2));
  return (f + 127) / 128 * 128;
}

int launch_decode_split(const tq_codec *hi, const tq_codec *lo, const int16_t *channels,
                        const void *q, int dtype, int B, int Hq, int Hkv, const tq_cache *chi,
                        const tq_cache *clo, const int32_t *seq_lens, int max_len, float scale,
                        const float *rc, const float *rs, int splits, void *ws, float *out,
                        cudaStream_t stream) {
  SplitArgs a;
  a.q = q;
  a.dtype = dtype;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.G = Hq / Hkv;
  const tq_cache *cc[2] = {chi, clo};
  const tq_codec *cd[2] = {hi, lo};
  for (int i = 0; i < 2; ++i) {
    a.kcode[i] = cc[i]->kcode;
    a.kscale[i] = cc[i]->kscale;
    a.vcode[i] = cc[i]->vcode;
    a.vnorm[i] = cc[i]->vnorm;
    a.qjl_coef[i] = cd[i]->qjl_k ? sqrtf(static_cast<float>(M_PI) / 2.0f) / cd[i]->d : 0.f;
    a.ST[i] = cd[i]->ST_dev;
    a.books[i] = cd[i]->books;
  }
  a.rows_cap = chi->rows_cap;
  a.seq_lens = seq_lens;
  a.max_len = max_len;
  a.scale = scale;
  a.rc = rc;
  a.rs = rs;
  a.splits = splits;
  const int per = (max_len + splits - 1) / splits;
  a.chunk = (per + 31) / 32 * 32;
  a.chan = channels;
  const size_t heads = static_cast<size_t>(B) * Hq, d = 2 * static_cast<size_t>(hi->d);
  float *f = static_cast<float *>(ws);
  a.q1 = f;
  a.q2 = f + heads * d;
  a.po = f + 2 * heads * d;
  a.pml = a.po + heads * static_cast<size_t>(splits) * d;
  a.out = out;
  switch (hi->d) {
    case 64: return run_split<64>(a, stream);
    case 128: return run_split<128>(a, stream);
    default: return tq_fail(TQ_ERR_UNSUPPORTED, "split decode: each half must have 64 or 128 channels");
  }
}
