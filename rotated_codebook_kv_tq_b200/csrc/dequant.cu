// Dequantize rows of the compressed cache ("FibQuant ...", section 2.3, decoder:
// look the code up, rotate back, scale by the norm; keys add the QJL term of
// "Google presenta TurboQuant ...", "Eliminacion del sesgo").
//   keys   x~ = nu Pi^T (c_k[idx] + sqrt(pi/2)/d rho S^T (2 sigma - 1))
//   values v~ = nu Pi^T c_v[idx]
// One warp per row; coordinate i = lane + 32 k in register k.
#include "tq_device.cuh"

namespace {

constexpr int DW = 8;

struct DequantArgs {
  const uint8_t *kcode;
  const uint16_t *kscale;
  const uint32_t *vcode;
  const uint16_t *vnorm;
  int64_t rows_cap;
  int BH;
  int64_t row0, rows;
  int which;
  float qjl_coef;
  const uint16_t *S;
  float *out;
  int Hkv;
  TqRowMap map;
  TqBooks books;
};

template <int D>
__global__ void __launch_bounds__(DW * 32) dequant_kernel(DequantArgs a) {
  constexpr int NPL = D / 32;
  __shared__ float cs[TQ_MAX_LEVELS];
  __shared__ float dsc[DW][D];   // dense-rotation scratch, one row per warp
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x < TQ_MAX_LEVELS)
    cs[threadIdx.x] = a.which == 0 ? a.books.ck[threadIdx.x] : a.books.cv[threadIdx.x];
  __syncthreads();
  const int64_t total = static_cast<int64_t>(a.BH) * a.rows;
  for (int64_t it = static_cast<int64_t>(blockIdx.x) * DW + warp; it < total;
       it += static_cast<int64_t>(gridDim.x) * DW) {
    const int64_t bh = it / a.rows, r = a.row0 + it % a.rows;
    float y[NPL];
    float nu;
    if (a.which == 0) {
      const int mbk = a.books.mse_bits_k, planes = mbk + a.books.qjl;
      const uint32_t *krow = reinterpret_cast<const uint32_t *>(
          a.kcode + (bh * a.rows_cap + r) * planes * (D / 8));
      const uint32_t sc = reinterpret_cast<const uint32_t *>(a.kscale)[bh * a.rows_cap + r];
      nu = tq_half_to_f32(static_cast<uint16_t>(sc & 0xffffu));
      const float rho = tq_half_to_f32(static_cast<uint16_t>(sc >> 16));
#pragma unroll
      for (int k = 0; k < NPL; ++k) {
        int idx = 0;
        for (int p = 0; p < mbk; ++p) idx |= ((krow[p * NPL + k] >> lane) & 1) << p;
        y[k] = cs[idx];
      }
      if (a.books.qjl) {
        // (S^T s)_j = sum_i S[i][j] s_i with s_i = 2 sigma_i - 1
        uint32_t sw[NPL];
#pragma unroll
        for (int k = 0; k < NPL; ++k) sw[k] = krow[mbk * NPL + k];
        float acc[NPL];
#pragma unroll
        for (int k = 0; k < NPL; ++k) acc[k] = 0.f;
        for (int i = 0; i < D; ++i) {
          const bool pos = (sw[i >> 5] >> (i & 31)) & 1;
#pragma unroll
          for (int k = 0; k < NPL; ++k) {
            const float s = tq_bf16_to_f32(a.S[i * D + lane + 32 * k]);
            acc[k] += pos ? s : -s;
          }
        }
        const float f = a.qjl_coef * rho;
#pragma unroll
        for (int k = 0; k < NPL; ++k) y[k] = fmaf(f, acc[k], y[k]);
      }
    } else {
      const int nb = a.books.bits_v;
      const uint32_t *vg = a.vcode + (bh * (a.rows_cap / 32) + (r >> 5)) * nb * D;
#pragma unroll
      for (int k = 0; k < NPL; ++k) {
        int idx = 0;
        for (int p = 0; p < nb; ++p) idx |= ((vg[p * D + lane + 32 * k] >> (r & 31)) & 1) << p;
        y[k] = cs[idx];
      }
      nu = tq_half_to_f32(a.vnorm[bh * a.rows_cap + r]);
    }
    // Pi^T y = D (H y) / sqrt(d), or the dense Pi^T
    float f = nu;
    if (a.books.pi != nullptr) {
      tq_warp_dense<NPL>(y, a.books.pi, dsc[warp], lane);
    } else {
      tq_warp_wht<NPL>(y, lane);
      tq_apply_signs<NPL>(y, a.books.dneg, lane);
      f /= sqrtf(static_cast<float>(D));
    }
    if (a.map.k != nullptr) {
      // outlier-channel split: coordinate i goes to channel map[h][i]
      const int16_t *m = (a.which == 0 ? a.map.k : a.map.v) + (bh % a.Hkv) * a.map.hstride;
      float *o = a.out + it * a.map.dfull;
#pragma unroll
      for (int k = 0; k < NPL; ++k) o[m[lane + 32 * k] & (a.map.dfull - 1)] = y[k] * f;
      continue;
    }
    float *o = a.out + it * D;
#pragma unroll
    for (int k = 0; k < NPL; ++k) o[lane + 32 * k] = y[k] * f;
  }
}

template <int D>
int run_dequant(const DequantArgs &a, cudaStream_t stream) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t total = static_cast<int64_t>(a.BH) * a.rows;
  const int64_t want = (total + DW - 1) / DW;
  const int grid = static_cast<int>(want < 8LL * sms ? want : 8LL * sms);
  dequant_kernel<D><<<grid, DW * 32, 0, stream>>>(a);
  tq_count_launch(1);
  return tq_check_launch("dequant_kernel");
}

}  // namespace

int launch_dequant(const tq_codec *c, const tq_cache *cache, int which, int64_t row0,
                   int64_t rows, float *out, cudaStream_t stream, const TqRowMap &map) {
  DequantArgs a;
  a.kcode = cache->kcode;
  a.kscale = cache->kscale;
  a.vcode = cache->vcode;
  a.vnorm = cache->vnorm;
  a.rows_cap = cache->rows_cap;
  a.BH = cache->B * cache->Hkv;
  a.row0 = row0;
  a.rows = rows;
  a.which = which;
  a.qjl_coef = c->qjl_k ? sqrtf(static_cast<float>(M_PI) / 2.0f) / c->d : 0.f;
  a.S = c->S_dev;
  a.out = out;
  a.Hkv = cache->Hkv;
  a.map = map;
  a.books = c->books;
  if (rows == 0) return TQ_OK;
  switch (c->d) {
    case 64: return run_dequant<64>(a, stream);
    case 128: return run_dequant<128>(a, stream);
    default: return tq_fail(TQ_ERR_UNSUPPORTED, "dequantize: head dim not built");
  }
}
