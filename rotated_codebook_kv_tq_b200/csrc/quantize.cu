// Fused quantize-append kernel: RoPE -> norm -> randomized WHT -> scalar codes
// -> bit planes, plus the QJL residual sketch for keys.
//
// Sources: "TurboESM ..." section 2.A (RoPE, then the rotation); "FibQuant ..."
// section 2.3 (store nu, rotate x/nu, quantize); "Ablazione ..."
// ("Configurazione Sperimentale": randomized Walsh-Hadamard rotation, Beta
// Lloyd-Max codebook, optional 1-bit QJL residual sketch on the key path);
// "Google presenta TurboQuant ..." ("Eliminacion del sesgo": b-1 MSE bits then a
// 1-bit QJL transform of the residual).
//
// Work split: one warp per (batch, head, 32-token group).  Coordinate
// i = lane + 32 k lives in register k of `lane`, so rotate-half RoPE pairs
// (i, i + d/2) are register-local, the transform runs on shuffles, and
// __ballot_sync over the warp produces each 32-coordinate key-plane word
// directly.  Value codes are accumulated per coordinate across the group's
// 32 tokens and stored as column-group words.
#include "tq_device.cuh"

namespace {

constexpr int QWARPS = 8;

struct QuantArgs {
  const void *k;
  const void *v;
  int dtype;
  int B, H, T;
  int64_t sb, sh, st;
  const float *rc;
  const float *rs;
  int64_t pos0;
  uint8_t *kcode;
  uint16_t *kscale;
  uint32_t *vcode;
  uint16_t *vnorm;
  int64_t rows_cap;
  int64_t row0;
  uint32_t *status;
  const uint16_t *S;
  int64_t g_first;   // first 32-token group touched
  int64_t n_groups;  // groups touched per (b, h)
  TqBooks books;
};

// Load one row (coordinates lane + 32 k), optional RoPE at position pos.
template <int NPL>
__device__ __forceinline__ void load_row(float (&x)[NPL], const void *base, int64_t off,
                                         int dtype, int lane, const float *rc, const float *rs,
                                         int64_t pos) {
#pragma unroll
  for (int k = 0; k < NPL; ++k) x[k] = tq_load_elem(base, off + lane + 32 * k, dtype);
  if (rc != nullptr) {
    constexpr int HALF = NPL / 2;  // register offset of coordinate i + d/2
    const int64_t tb = pos * (NPL * 16);
#pragma unroll
    for (int k = 0; k < HALF; ++k) {
      const float c = rc[tb + lane + 32 * k];
      const float s = rs[tb + lane + 32 * k];
      const float a = x[k], b = x[k + HALF];
      x[k] = a * c - b * s;
      x[k + HALF] = b * c + a * s;
    }
  }
}

// Normalise and rotate: returns nu (0 for bad rows), u = H D x / (sqrt(d) nu).
template <int NPL>
__device__ __forceinline__ float normalize_rotate(float (&x)[NPL], const uint32_t *dneg,
                                                  int lane, bool &bad) {
  bool finite = true;
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < NPL; ++k) {
    finite &= isfinite(x[k]);
    ss += x[k] * x[k];
  }
  bad = __any_sync(TQ_FULL, !finite);
  ss = tq_warp_sum(ss);
  float nu = sqrtf(ss);
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

template <int D>
__global__ void __launch_bounds__(QWARPS * 32) quantize_kernel(QuantArgs a) {
  constexpr int NPL = D / 32;
  extern __shared__ float smem[];
  float *ST = smem;                      // S^T fp32 [D][D]: ST[j*D + i] = S[i][j]
  __shared__ float cks[TQ_MAX_LEVELS], tks[TQ_MAX_LEVELS], tvs[TQ_MAX_LEVELS];
  __shared__ float rbuf[QWARPS][D];

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nlk = 1 << a.books.mse_bits_k, nlv = 1 << a.books.bits_v;
  if (threadIdx.x < TQ_MAX_LEVELS) {
    cks[threadIdx.x] = a.books.ck[threadIdx.x];
    tks[threadIdx.x] = a.books.tk[threadIdx.x];
    tvs[threadIdx.x] = a.books.tv[threadIdx.x];
  }
  if (a.books.qjl) {
    for (int e = threadIdx.x; e < D * D; e += blockDim.x) {
      const int i = e / D, j = e % D;
      ST[j * D + i] = tq_bf16_to_f32(a.S[e]);
    }
  }
  __syncthreads();

  const int planes_k = a.books.mse_bits_k + a.books.qjl;
  const int64_t items = static_cast<int64_t>(a.B) * a.H * a.n_groups;
  for (int64_t it = static_cast<int64_t>(blockIdx.x) * QWARPS + warp; it < items;
       it += static_cast<int64_t>(gridDim.x) * QWARPS) {
    const int64_t g = a.g_first + it % a.n_groups;
    const int64_t bh = it / a.n_groups;
    const int b = static_cast<int>(bh / a.H), h = static_cast<int>(bh % a.H);
    const int64_t r_begin = max(a.row0, g * 32), r_end = min(a.row0 + a.T, g * 32 + 32);
    const int64_t cache_bh = static_cast<int64_t>(b) * a.H + h;

    uint32_t vw[4][NPL];
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
      for (int k = 0; k < NPL; ++k) vw[p][k] = 0u;

    for (int64_t r = r_begin; r < r_end; ++r) {
      const int64_t t = r - a.row0;
      const int64_t in_off = b * a.sb + h * a.sh + t * a.st;
      // ------------------------------------------------------------ keys
      float x[NPL];
      load_row<NPL>(x, a.k, in_off, a.dtype, lane, a.rc, a.rs, a.pos0 + t);
      bool bad;
      const float nu = normalize_rotate<NPL>(x, a.books.dneg, lane, bad);
      int idx[NPL];
#pragma unroll
      for (int k = 0; k < NPL; ++k) idx[k] = tq_code(x[k], tks, nlk - 1);
      // plane words: lane p*NPL + k stores word k of plane p
      uint32_t myword = 0u;
      for (int p = 0; p < a.books.mse_bits_k; ++p) {
#pragma unroll
        for (int k = 0; k < NPL; ++k) {
          const uint32_t w = __ballot_sync(TQ_FULL, (idx[k] >> p) & 1);
          if (lane == p * NPL + k) myword = w;
        }
      }
      float rho = 0.f;
      if (a.books.qjl) {
        float r2 = 0.f;
#pragma unroll
        for (int k = 0; k < NPL; ++k) {
          const float rr = x[k] - cks[idx[k]];
          rbuf[warp][lane + 32 * k] = rr;
          r2 += rr * rr;
        }
        rho = sqrtf(tq_warp_sum(r2));
        __syncwarp();
        float z[NPL];
#pragma unroll
        for (int k = 0; k < NPL; ++k) z[k] = 0.f;
        for (int j = 0; j < D; ++j) {
          const float rj = rbuf[warp][j];
#pragma unroll
          for (int k = 0; k < NPL; ++k) z[k] = fmaf(ST[j * D + lane + 32 * k], rj, z[k]);
        }
        __syncwarp();
        const int p = a.books.mse_bits_k;
#pragma unroll
        for (int k = 0; k < NPL; ++k) {
          const uint32_t w = __ballot_sync(TQ_FULL, z[k] >= 0.f);
          if (lane == p * NPL + k) myword = w;
        }
      }
      uint32_t *krow = reinterpret_cast<uint32_t *>(
          a.kcode + (cache_bh * a.rows_cap + r) * planes_k * (D / 8));
      if (lane < planes_k * NPL) krow[lane] = myword;
      if (lane == 0) {
        const uint32_t pair = static_cast<uint32_t>(tq_f32_to_half(nu)) |
                              (static_cast<uint32_t>(tq_f32_to_half(rho)) << 16);
        reinterpret_cast<uint32_t *>(a.kscale)[cache_bh * a.rows_cap + r] = pair;
        if (bad && a.status) atomicAdd(a.status, 1u);
      }
      // ------------------------------------------------------------ values
      load_row<NPL>(x, a.v, in_off, a.dtype, lane, nullptr, nullptr, 0);
      const float nv = normalize_rotate<NPL>(x, a.books.dneg, lane, bad);
      const uint32_t bit = 1u << (r & 31);
#pragma unroll
      for (int k = 0; k < NPL; ++k) {
        const int iv = tq_code(x[k], tvs, nlv - 1);
#pragma unroll
        for (int p = 0; p < 4; ++p)
          if ((iv >> p) & 1) vw[p][k] |= bit;
      }
      if (lane == 0) {
        a.vnorm[cache_bh * a.rows_cap + r] = tq_f32_to_half(nv);
        if (bad && a.status) atomicAdd(a.status, 1u);
      }
    }
    // store the group's value words (read-modify-write for partial groups)
    const uint32_t nrows = static_cast<uint32_t>(r_end - r_begin);
    const uint32_t mask = nrows == 32 ? TQ_FULL : (((1u << nrows) - 1u) << (r_begin & 31));
    uint32_t *vg = a.vcode + (cache_bh * (a.rows_cap / 32) + g) * a.books.bits_v * D;
    for (int p = 0; p < a.books.bits_v; ++p) {
#pragma unroll
      for (int k = 0; k < NPL; ++k) {
        uint32_t *w = vg + p * D + lane + 32 * k;
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

template <int D>
int run_quantize(const QuantArgs &a, cudaStream_t stream) {
  const size_t shm = a.books.qjl ? sizeof(float) * D * D : 0;
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(quantize_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             sizeof(float) * D * D) != cudaSuccess)
      return tq_check_launch("cudaFuncSetAttribute(quantize)");
    attr_set = true;
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t items = static_cast<int64_t>(a.B) * a.H * a.n_groups;
  const int64_t want = (items + QWARPS - 1) / QWARPS;
  const int grid = static_cast<int>(want < 4LL * sms ? want : 4LL * sms);
  quantize_kernel<D><<<grid, QWARPS * 32, shm, stream>>>(a);
  tq_count_launch(1);
  return tq_check_launch("quantize_kernel");
}

}  // namespace

int launch_quantize(const tq_codec *c, const void *k, const void *v, int dtype, int B, int H,
                    int T, int64_t sb, int64_t sh, int64_t st, const float *rc, const float *rs,
                    int64_t pos0, const tq_cache *cache, int64_t row0, uint32_t *status,
                    cudaStream_t stream) {
  QuantArgs a;
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
  a.status = status;
  a.S = c->S_dev;
  a.g_first = row0 / 32;
  a.n_groups = (row0 + T - 1) / 32 - row0 / 32 + 1;
  a.books = c->books;
  if (T == 0) return TQ_OK;
  switch (c->d) {
    case 64: return run_quantize<64>(a, stream);
    case 128: return run_quantize<128>(a, stream);
    default: return tq_fail(TQ_ERR_UNSUPPORTED, "quantize: head dim not built");
  }
}
