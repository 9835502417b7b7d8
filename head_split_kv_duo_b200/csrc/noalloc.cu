// noalloc.cu -- decode attention whose split-KV scratch lives in a static device array.
//
// Some callers cannot allocate device memory at the moment they decode: code running
// while a CUDA graph is being captured (cudaMalloc is not allowed there), or a runtime
// whose device memory is owned by a pool sized once at start-up (every further
// cudaMalloc fails or fragments it).  duo_decode_attention_static_scratch serves them:
// it allocates nothing and asks the caller for no scratch.  The partial results and
// merge tickets of the split-KV decode go to g_decode_scratch, a fixed array of
// kStaticScratchBytes that every GPU which loads this library holds until the process
// exits.  The caller still passes the cache, the queries and the outputs.
#include <mutex>

#include "duo_internal.h"
#include "nvtx_range.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(4) << 20;  // 4 MiB
constexpr int kMaxDevices = 64;

// Device-side scratch shared by every call on a device.  In host code this name is
// only a stand-in for the symbol: its device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

struct DeviceScratch {
  bool ready = false;
  unsigned char *ptr = nullptr;  // device address of g_decode_scratch on that device
};
DeviceScratch g_dev[kMaxDevices];
std::mutex g_dev_mutex;

// Once per device, with that device current: look up the array's device address.
duo_status scratch_for_current_device(unsigned char **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DUO_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return DUO_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  if (!g_dev[dev].ready) {
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess || ptr == nullptr) return DUO_ERR_CUDA;
    g_dev[dev].ptr = static_cast<unsigned char *>(ptr);
    g_dev[dev].ready = true;
  }
  *out = g_dev[dev].ptr;
  return DUO_OK;
}

}  // namespace

extern "C" duo_status duo_decode_attention_static_scratch(duo_cache *c, int layer, const void *q, void *out,
                                                          float *lse, void *stream) {
  DUO_NVTX_RANGE("duo_decode_attention_static_scratch");
  using namespace duo;
  if (!c || layer < 0 || layer >= c->layers || !q || !out) return DUO_ERR_INVALID;
  if ((reinterpret_cast<uintptr_t>(q) & 15u) || (reinterpret_cast<uintptr_t>(out) & 15u) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return DUO_ERR_INVALID;
  const Layer &ly = c->L[layer];
  if (ly.len < 1 || !c->initialised) return DUO_ERR_INVALID;  // a token must have been appended

  DecodeParams p{};
  p.q = static_cast<const char *>(q);
  p.out = static_cast<char *>(out);
  p.lse = lse;
  p.rk = ly.rk;
  p.rv = ly.rv;
  p.rk_sz = ly.rk_sz;
  p.rv_sz = ly.rv_sz;
  p.sk = ly.sk;
  p.sv = ly.sv;
  p.status = c->status;
  p.B = c->B;
  p.Hq = c->Hq;
  p.Hkv = c->Hkv;
  p.G = c->G;
  p.D = c->D;
  p.Hr = ly.Hr;
  p.Hs = ly.Hs;
  p.S = c->S;
  p.W = c->W;
  p.len = ly.len;
  p.max_len = c->cap;
  p.qg = c->G;
  p.nqg = 1;
  p.scale_log2 = c->scale * 1.4426950408889634f;
  p.hm = ly.hm;
  // quantised retrieval caches (INT4, FP8) are not served here
  if (c->fmt != DUO_KV_SAME || !decode_tc_supported(p, c->dtype, false)) return DUO_ERR_UNSUPPORTED;

  // Scratch layout: tickets [B][Hkv] (256-byte padded), then partials
  // [B][Hkv][ctas][G][d+4] floats.  Fewer CTAs are used when the partials of one
  // CTA per SM would not fit; a cache with more heads than fit at one CTA is refused.
  const size_t items = static_cast<size_t>(c->B) * c->Hkv;
  const size_t ticket_bytes = (items * 4 + 255) / 256 * 256;
  const size_t per_cta = items * c->G * (static_cast<size_t>(c->D) + 4) * 4;
  if (ticket_bytes >= kStaticScratchBytes || per_cta > kStaticScratchBytes - ticket_bytes) return DUO_ERR_CAPACITY;
  size_t ctas = (kStaticScratchBytes - ticket_bytes) / per_cta;
  if (ctas > static_cast<size_t>(c->num_sms)) ctas = static_cast<size_t>(c->num_sms);
  if (ctas > static_cast<size_t>(kMaxSplits)) ctas = kMaxSplits;

  unsigned char *scratch = nullptr;
  duo_status s = scratch_for_current_device(&scratch);
  if (s != DUO_OK) return s;
  p.counters = reinterpret_cast<uint32_t *>(scratch);
  p.partials = reinterpret_cast<float *>(scratch + ticket_bytes);
  p.max_splits = static_cast<int>(ctas);

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // tickets must start at zero; the previous call's contents are still in the array
  if (cudaMemsetAsync(p.counters, 0, items * 4, st) != cudaSuccess) return DUO_ERR_CUDA;
  if (launch_decode_tc(p, static_cast<int>(ctas), false, st) != cudaSuccess) return DUO_ERR_CUDA;
  return DUO_OK;
}
