// Decode attention for callers that cannot allocate device memory.
//
// tq_attention_decode needs a caller-provided scratch workspace (the rotated
// and sketched queries plus one partial result per split-K chunk).  Some
// callers cannot provide one because they cannot call cudaMalloc: a plugin
// loaded into a host application that owns every device allocation through
// its own allocator, or a serving process that reserved nearly all HBM for its
// KV pool up front and must not grow its device footprint afterwards.  This
// entry point takes its scratch from a fixed array in the library's own device
// image instead, so it allocates nothing.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds TQ_NOALLOC_SCRATCH_BYTES of it until the process exits.  In host
// code its name is only a host-side stand-in, so its device address is looked
// up once per device with cudaGetSymbolAddress (with that device current) and
// cached.  Every call shares the array and leaves the previous call's contents
// in it; each call writes every scratch word it reads (the partials of each
// chunk, and the status word, which the query prologue clears), so no
// clearing is needed.  Calls whose kernels overlap on the GPU (different
// streams, or several host threads) race on the array and must be serialised
// by the caller.
#include <mutex>

#include "tq_internal.h"

namespace {

__device__ __align__(256) unsigned char g_tq_static_scratch[TQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void *g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

int scratch_for_current_device(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return tq_check_launch("no-alloc decode: cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices)
    return tq_fail(TQ_ERR_UNSUPPORTED, "no-alloc decode: device index beyond 63");
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_tq_static_scratch);
    if (e != cudaSuccess)
      return tq_fail(TQ_ERR_CUDA, std::string("no-alloc decode: cudaGetSymbolAddress: ") +
                                      cudaGetErrorString(e));
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return TQ_OK;
}

}  // namespace

extern "C" int tq_attention_decode_noalloc(const tq_codec *c, const void *q, int dtype, int B,
                                           int Hq, int Hkv, const tq_cache *cache,
                                           const int32_t *seq_lens, int max_seq_len,
                                           float scale, const float *rope_cos,
                                           const float *rope_sin, int num_splits, float *out,
                                           void *stream) {
  if (!c) return tq_fail(TQ_ERR_INVALID_ARG, "no-alloc decode: NULL codec");
  if (B <= 0 || Hq <= 0 || num_splits < 0)
    return tq_fail(TQ_ERR_INVALID_ARG, "no-alloc decode: bad B/Hq/num_splits");
  const int splits = num_splits > 0 ? num_splits : 64;
  const size_t need = decode_workspace_bytes(c, B, Hq, splits);
  if (need > static_cast<size_t>(TQ_NOALLOC_SCRATCH_BYTES))
    return tq_fail(TQ_ERR_WORKSPACE,
                   "no-alloc decode: the scratch this shape needs (tq_attention_workspace for the same "
                   "codec, B, Hq and num_splits) exceeds the 16 MiB static array");
  void *ws = nullptr;
  if (int e = scratch_for_current_device(&ws)) return e;
  return tq_attention_decode(c, q, dtype, B, Hq, Hkv, cache, seq_lens, max_seq_len, scale,
                             rope_cos, rope_sin, splits, ws, need, out, stream);
}
