// duo_host.cu -- the C ABI of include/duo.h: argument checks, cache layout inside
// the caller's buffer, host-side length bookkeeping, and kernel launches.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <new>

#include "duo_internal.h"
#include "nvtx_range.h"

using namespace duo;

namespace {

constexpr size_t kMaxBytes = size_t(1) << 50;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct Cfg {
  int layers, Hkv, D, S, W;
  int64_t max_len;
  int B, Hq, G;
  duo_dtype dtype;
  duo_kv_fmt fmt;
  float scale;
  int esize;
};

struct LayerOff {
  int Hr, Hs;
  size_t rk, rv, rk_sz, rv_sz, sk, sv;
};

struct Layout {
  size_t total = 0;
  size_t status = 0, counters = 0, partials = 0, hist_k = 0, hist_v = 0;
  int max_splits = 1, hs_max = 0;
  int64_t cap = 0;
  std::vector<LayerOff> layer;
};

duo_status make_cfg(int layers, int kv_heads, int head_dim, const uint8_t *mask, int S, int W, int64_t max_len,
                    const duo_opts *opts, Cfg *c) {
  if (layers < 1 || layers > 65536) return DUO_ERR_INVALID;
  if (kv_heads < 1 || kv_heads > kMaxKvHeads) return DUO_ERR_INVALID;
  if (head_dim != 64 && head_dim != 128) return DUO_ERR_INVALID;
  if (!mask) return DUO_ERR_INVALID;
  if (S < 0 || W < 1 || S > (1 << 24) || W > (1 << 24)) return DUO_ERR_INVALID;
  if (max_len < 1 || max_len > (int64_t(1) << 36)) return DUO_ERR_INVALID;
  duo_opts o = {1, 0, DUO_BF16, DUO_KV_SAME, 0.f};
  if (opts) o = *opts;
  if (o.batch < 1 || o.batch > 65536) return DUO_ERR_INVALID;
  if (o.q_heads == 0) o.q_heads = kv_heads;
  if (o.q_heads < kv_heads || o.q_heads % kv_heads != 0 || o.q_heads > 4096) return DUO_ERR_INVALID;
  if (o.dtype != DUO_BF16 && o.dtype != DUO_FP32) return DUO_ERR_INVALID;
  if (o.retr_fmt != DUO_KV_SAME && o.retr_fmt != DUO_KV_INT4_G128 && o.retr_fmt != DUO_KV_FP8_E4M3)
    return DUO_ERR_INVALID;
  if (!(o.softmax_scale >= 0.f) || !std::isfinite(o.softmax_scale)) return DUO_ERR_INVALID;
  if (o.retr_fmt != DUO_KV_SAME && (o.dtype != DUO_BF16 || head_dim != 128)) return DUO_ERR_UNSUPPORTED;
  for (int i = 0; i < layers * kv_heads; ++i)
    if (mask[i] > 1) return DUO_ERR_INVALID;
  c->layers = layers;
  c->Hkv = kv_heads;
  c->D = head_dim;
  c->S = S;
  c->W = W;
  c->max_len = max_len;
  c->B = o.batch;
  c->Hq = o.q_heads;
  c->G = o.q_heads / kv_heads;
  c->dtype = o.dtype;
  c->fmt = o.retr_fmt;
  c->scale = o.softmax_scale > 0.f ? o.softmax_scale : 1.f / std::sqrt(static_cast<float>(head_dim));
  c->esize = o.dtype == DUO_BF16 ? 2 : 4;
  return DUO_OK;
}

// Carves the caller's buffer; false on size overflow.
bool make_layout(const Cfg &c, const uint8_t *mask, Layout *L) {
  const double est = static_cast<double>(c.layers) * c.B * c.Hkv * (static_cast<double>(c.max_len) + c.S + c.W) *
                     c.D * c.esize * 2.0;
  if (est > static_cast<double>(kMaxBytes)) return false;
  L->cap = static_cast<int64_t>(align_up(static_cast<size_t>(c.max_len), 256));
  // partial slots per head: enough for every 128-token unit of a retrieval head (or of
  // the sink+ring slots), capped at kMaxSplits
  const int64_t units = std::max<int64_t>((c.max_len + 127) / 128, (static_cast<int64_t>(c.S) + c.W + 127) / 128);
  L->max_splits = static_cast<int>(std::min<int64_t>(kMaxSplits, std::max<int64_t>(1, units)));
  const size_t row = static_cast<size_t>(c.D) * c.esize;
  // retrieval row bytes: d elements, d/2 INT4 code bytes, or d FP8 code bytes
  const size_t rrow = c.fmt == DUO_KV_INT4_G128 ? static_cast<size_t>(c.D / 2)
                      : c.fmt == DUO_KV_FP8_E4M3 ? static_cast<size_t>(c.D)
                                                 : row;
  const size_t nslots = static_cast<size_t>(c.S) + c.W;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, kAlign);
    return at;
  };
  L->status = take(256);
  L->counters = take(static_cast<size_t>(c.B) * c.Hq * 4);
  L->partials = take(static_cast<size_t>(c.B) * c.Hkv * L->max_splits * c.G * (c.D + 4) * 4);
  L->hs_max = 0;
  L->layer.resize(c.layers);
  for (int l = 0; l < c.layers; ++l) {
    int hr = 0;
    for (int h = 0; h < c.Hkv; ++h) hr += mask[l * c.Hkv + h];
    L->layer[l].Hr = hr;
    L->layer[l].Hs = c.Hkv - hr;
    L->hs_max = std::max(L->hs_max, c.Hkv - hr);
  }
  const size_t hist = static_cast<size_t>(c.B) * L->hs_max * nslots * row;
  L->hist_k = take(hist);
  L->hist_v = take(hist);
  for (int l = 0; l < c.layers; ++l) {
    LayerOff &lo = L->layer[l];
    const size_t rbytes = static_cast<size_t>(c.B) * lo.Hr * L->cap * rrow;
    lo.rk = take(rbytes);
    lo.rv = take(rbytes);
    if (c.fmt != DUO_KV_SAME) {  // INT4 fp16 scale + zero, or FP8 fp32 scale: 4 bytes per row
      const size_t zbytes = static_cast<size_t>(c.B) * lo.Hr * L->cap * 4 + 16;
      lo.rk_sz = take(zbytes);
      lo.rv_sz = take(zbytes);
    } else {
      lo.rk_sz = lo.rv_sz = 0;
    }
    const size_t sbytes = static_cast<size_t>(c.B) * lo.Hs * nslots * row;
    lo.sk = take(sbytes);
    lo.sv = take(sbytes);
  }
  L->total = off;
  return off <= kMaxBytes;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool layer_ok(const duo_cache *c, int layer) { return c && layer >= 0 && layer < c->layers; }

// Test controls (duo_debug_launch_controls): process-wide.
std::atomic<int> g_dry_run{0};
std::atomic<int64_t> g_fail_countdown{-1};
std::atomic<int> g_device_stall{0};

duo_status ensure_init(duo_cache *c, cudaStream_t st) {
  if (c->initialised) return DUO_OK;
  if (duo::dry_run()) {  // no device: the count of a full B200 for the work split
    c->num_sms = 148;
    c->initialised = true;
    return DUO_OK;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DUO_ERR_CUDA;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return DUO_ERR_CUDA;
  if (cudaMemsetAsync(c->buf, 0, c->bytes, st) != cudaSuccess) return DUO_ERR_CUDA;
  c->num_sms = sms;
  c->initialised = true;
  return DUO_OK;
}

AppendParams append_params(const duo_cache *c, const Layer &ly, const void *k, const void *v, int n) {
  AppendParams p{};
  p.k = static_cast<const char *>(k);
  p.v = static_cast<const char *>(v);
  p.rk = ly.rk;
  p.rv = ly.rv;
  p.rk_sz = ly.rk_sz;
  p.rv_sz = ly.rv_sz;
  p.sk = ly.sk;
  p.sv = ly.sv;
  p.B = c->B;
  p.n = n;
  p.Hkv = c->Hkv;
  p.D = c->D;
  p.Hr = ly.Hr;
  p.Hs = ly.Hs;
  p.S = c->S;
  p.W = c->W;
  p.len = ly.len;
  p.max_len = c->cap;
  p.ring_from = std::max<int64_t>(c->S, ly.len + n - c->W);
  p.int4 = c->fmt == DUO_KV_INT4_G128 ? 1 : 0;
  p.fp8 = c->fmt == DUO_KV_FP8_E4M3 ? 1 : 0;
  p.hm = ly.hm;
  return p;
}

}  // namespace

extern "C" {

const char *duo_status_str(duo_status s) {
  switch (s) {
    case DUO_OK: return "ok";
    case DUO_ERR_INVALID: return "invalid argument";
    case DUO_ERR_CAPACITY: return "cache capacity exceeded";
    case DUO_ERR_CUDA: return "CUDA error";
    case DUO_ERR_TIMEOUT: return "device wait timed out";
    case DUO_ERR_UNSUPPORTED: return "unsupported configuration";
  }
  return "unknown status";
}

size_t duo_cache_bytes(int layers, int kv_heads, int head_dim, const uint8_t *mask, int S, int W, int64_t max_len,
                       const duo_opts *opts) {
  Cfg c;
  if (make_cfg(layers, kv_heads, head_dim, mask, S, W, max_len, opts, &c) != DUO_OK) return 0;
  Layout L;
  if (!make_layout(c, mask, &L)) return 0;
  return L.total;
}

duo_status duo_cache_create(int layers, int kv_heads, int head_dim, const uint8_t *mask, int S, int W,
                            int64_t max_len, const duo_opts *opts, void *dev_buf, size_t dev_bytes, duo_cache **out) {
  DUO_NVTX_RANGE("duo_cache_create");
  if (!out) return DUO_ERR_INVALID;
  *out = nullptr;
  Cfg c;
  duo_status st = make_cfg(layers, kv_heads, head_dim, mask, S, W, max_len, opts, &c);
  if (st != DUO_OK) return st;
  Layout L;
  if (!make_layout(c, mask, &L)) return DUO_ERR_INVALID;
  if (!dev_buf || (reinterpret_cast<uintptr_t>(dev_buf) & 255u) || dev_bytes < L.total) return DUO_ERR_INVALID;
  duo_cache *h = new (std::nothrow) duo_cache();
  if (!h) return DUO_ERR_INVALID;
  h->layers = c.layers;
  h->Hkv = c.Hkv;
  h->Hq = c.Hq;
  h->G = c.G;
  h->D = c.D;
  h->B = c.B;
  h->S = c.S;
  h->W = c.W;
  h->max_len = c.max_len;
  h->cap = L.cap;
  h->dtype = c.dtype;
  h->fmt = c.fmt;
  h->scale = c.scale;
  h->esize = c.esize;
  h->buf = static_cast<char *>(dev_buf);
  h->bytes = L.total;
  h->status = reinterpret_cast<uint32_t *>(h->buf + L.status);
  h->counters = reinterpret_cast<uint32_t *>(h->buf + L.counters);
  h->partials = reinterpret_cast<float *>(h->buf + L.partials);
  h->max_splits = L.max_splits;
  h->hist_k = h->buf + L.hist_k;
  h->hist_v = h->buf + L.hist_v;
  h->hs_max = L.hs_max;
  h->L.resize(c.layers);
  for (int l = 0; l < c.layers; ++l) {
    Layer &ly = h->L[l];
    const LayerOff &lo = L.layer[l];
    ly.Hr = lo.Hr;
    ly.Hs = lo.Hs;
    int ri = 0, si = 0;
    for (int g = 0; g < c.Hkv; ++g) {
      const bool r = mask[l * c.Hkv + g] != 0;
      ly.hm.is_retr[g] = r ? 1 : 0;
      ly.hm.kind_idx[g] = static_cast<uint8_t>(r ? ri : si);
      if (r) ly.hm.retr_head[ri++] = static_cast<uint8_t>(g);
      else ly.hm.strm_head[si++] = static_cast<uint8_t>(g);
    }
    ly.rk = h->buf + lo.rk;
    ly.rv = h->buf + lo.rv;
    ly.rk_sz = c.fmt != DUO_KV_SAME ? h->buf + lo.rk_sz : nullptr;
    ly.rv_sz = c.fmt != DUO_KV_SAME ? h->buf + lo.rv_sz : nullptr;
    ly.sk = h->buf + lo.sk;
    ly.sv = h->buf + lo.sv;
    ly.len = 0;
  }
  *out = h;
  return DUO_OK;
}

void duo_cache_destroy(duo_cache *cache) { delete cache; }

duo_status duo_append_kv(duo_cache *c, int layer, const void *k, const void *v, int n, void *stream) {
  DUO_NVTX_RANGE("duo_append_kv");
  if (!layer_ok(c, layer) || !k || !v || n < 1 || !aligned16(k) || !aligned16(v)) return DUO_ERR_INVALID;
  Layer &ly = c->L[layer];
  if (ly.len + n > c->max_len) return DUO_ERR_CAPACITY;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  duo_status s = ensure_init(c, st);
  if (s != DUO_OK) return s;
  const AppendParams ap = append_params(c, ly, k, v, n);
  if (launch_via_hook([&] { return launch_append(ap, c->dtype, st); }) != cudaSuccess) return DUO_ERR_CUDA;
  ly.len += n;
  return DUO_OK;
}

duo_status duo_prefill_chunk(duo_cache *c, int layer, const void *q, const void *k, const void *v, int n, void *out,
                             float *lse, void *stream) {
  DUO_NVTX_RANGE("duo_prefill_chunk");
  if (!layer_ok(c, layer) || !q || !k || !v || !out || n < 1) return DUO_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return DUO_ERR_INVALID;
  if (c->fmt != DUO_KV_SAME) return DUO_ERR_UNSUPPORTED;  // quantised caches: decode only
  Layer &ly = c->L[layer];
  if (ly.len + n > c->max_len) return DUO_ERR_CAPACITY;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  duo_status s = ensure_init(c, st);
  if (s != DUO_OK) return s;

  // 1. stage the streaming history the chunk may see, in position order
  const int64_t len = ly.len;
  HistParams hp{};
  hp.sk = ly.sk;
  hp.sv = ly.sv;
  hp.hk = c->hist_k;
  hp.hv = c->hist_v;
  hp.B = c->B;
  hp.Hs = ly.Hs;
  hp.HsMax = c->hs_max;
  hp.D = c->D;
  hp.S = c->S;
  hp.W = c->W;
  hp.hs = static_cast<int>(std::min<int64_t>(c->S, len));
  hp.wstart = std::max<int64_t>(c->S, len - c->W + 1);
  hp.hw = static_cast<int>(std::max<int64_t>(0, len - hp.wstart));

  // 2. attention: cached positions from the cache, the chunk from k and v
  PrefillParams p{};
  p.q = static_cast<const char *>(q);
  p.k = static_cast<const char *>(k);
  p.v = static_cast<const char *>(v);
  p.out = static_cast<char *>(out);
  p.lse = lse;
  p.rk = ly.rk;
  p.rv = ly.rv;
  p.hk = c->hist_k;
  p.hv = c->hist_v;
  p.status = c->status;
  p.B = c->B;
  p.n = n;
  p.Hq = c->Hq;
  p.Hkv = c->Hkv;
  p.G = c->G;
  p.D = c->D;
  p.Hr = ly.Hr;
  p.Hs = ly.Hs;
  p.HsMax = c->hs_max;
  p.S = c->S;
  p.W = c->W;
  p.len = len;
  p.max_len = c->cap;
  p.hs = hp.hs;
  p.hw = hp.hw;
  p.wstart = hp.wstart;
  p.scale_log2 = c->scale * 1.4426950408889634f;
  p.hm = ly.hm;
  p.mix_alpha = nullptr;

  // 3. append the chunk (the only launch that changes the cache, so it goes last: a call
  // that fails leaves the cache as it was)
  const AppendParams ap = append_params(c, ly, k, v, n);

  // every fallible set-up step comes before the first launch
  const bool tc = prefill_tc_supported(p, c->dtype) && !dry_run();
  PrefillTcLaunch tl;
  if (tc && prepare_prefill_tc(p, &tl) != cudaSuccess) return DUO_ERR_CUDA;
  if (ly.Hs > 0 && hp.hs + hp.hw > 0)
    if (launch_via_hook([&] { return launch_hist(hp, c->dtype, st); }) != cudaSuccess) return DUO_ERR_CUDA;
  if (launch_via_hook([&] { return tc ? launch_prefill_tc(tl, st) : launch_prefill_simt(p, c->dtype, st); }) !=
      cudaSuccess)
    return DUO_ERR_CUDA;
  if (launch_via_hook([&] { return launch_append(ap, c->dtype, st); }) != cudaSuccess) return DUO_ERR_CUDA;
  ly.len += n;
  return DUO_OK;
}

}  // extern "C"

namespace {

// Decode parameters of `layer` at its current length (the query is position len - 1).
DecodeParams decode_params(const duo_cache *c, const Layer &ly, const void *q, void *out, float *lse) {
  const bool int4 = c->fmt == DUO_KV_INT4_G128;
  DecodeParams p{};
  p.debug_stall = g_device_stall.load(std::memory_order_relaxed);
  p.q = static_cast<const char *>(q);
  p.out = static_cast<char *>(out);
  p.lse = lse;
  p.rk = ly.rk;
  p.rv = ly.rv;
  p.rk_sz = ly.rk_sz;
  p.rv_sz = ly.rv_sz;
  p.sk = ly.sk;
  p.sv = ly.sv;
  p.partials = c->partials;
  p.counters = c->counters;
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
  p.qg = (c->G % 4 == 0) ? 4 : (c->G % 2 == 0) ? 2 : 1;
  p.nqg = c->G / p.qg;
  p.max_splits = c->max_splits;
  p.scale_log2 = c->scale * 1.4426950408889634f;
  p.hm = ly.hm;
  // split-KV sizing of the CUDA-core kernel: about four CTAs per SM in total, splits a
  // whole number of stages
  const int64_t tps = std::max(decode_tokens_per_stage(c->dtype, c->D, int4), kMinSplitTokens);
  const int64_t heads = static_cast<int64_t>(c->B) * ly.Hr * p.nqg;
  int64_t nsplit = 1;
  if (heads > 0) {
    const int64_t target = static_cast<int64_t>(c->num_sms) * 4;
    nsplit = std::min<int64_t>(c->max_splits, std::max<int64_t>(1, (target + heads - 1) / heads));
  }
  int64_t split_len = (ly.len + nsplit - 1) / nsplit;
  split_len = (split_len + tps - 1) / tps * tps;
  nsplit = (ly.len + split_len - 1) / split_len;
  p.nsplit = static_cast<int>(nsplit);
  p.split_len = split_len;
  p.n_retr_ctas = static_cast<int>(heads * nsplit);
  return p;
}

// SMs for a quantised layer's bf16 streaming heads, decoded beside its retrieval heads:
// a share in proportion to their bytes (1.5 times, a lone CTA hides less latency), at
// least one, at most an eighth of the SMs, and no more than their tiles.
static int streaming_ctas(const DecodeParams &p, int num_sms, bool int4) {
  const int64_t slots = static_cast<int64_t>(p.S) + p.W, reach = static_cast<int64_t>(p.S) + p.len;
  const int64_t used = reach < slots ? reach : slots;
  const int64_t units_s = static_cast<int64_t>(p.B) * p.Hs * ((used + 127) / 128);
  const int64_t units_r = static_cast<int64_t>(p.B) * p.Hr * ((p.len + 127) / 128);
  const double bs = static_cast<double>(units_s) * 128 * p.D * 2 * 2;                 // bf16 K and V
  const double br = static_cast<double>(units_r) * 128 * (int4 ? 2 * (p.D / 2 + 4) : 2 * (p.D + 4));
  int k = static_cast<int>(1.5 * num_sms * bs / (bs + br) + 0.999);
  const int hi = num_sms / 8 > 1 ? num_sms / 8 : 1;
  k = k < 1 ? 1 : (k > hi ? hi : k);
  return static_cast<int>(units_s < k ? (units_s > 0 ? units_s : 1) : k);
}

// A quantised layer: its bf16 streaming heads on the bf16 kernel (a few CTAs, leading)
// and its retrieval heads on the INT4 or FP8 kernel beside it on the other SMs; the two
// write disjoint heads, partial rows and tickets.  Each launch goes through the test
// controls when `hooked`.
static cudaError_t launch_quantised_layer(const duo_cache *c, const DecodeParams &p, bool int4, bool hooked,
                                          cudaStream_t st) {
  auto run = [&](auto &&f) { return hooked ? launch_via_hook(f) : f(); };
  int rest = c->num_sms;
  DecodeParams pr = p;
  if (p.Hs > 0) {
    DecodeParams ps = p;
    ps.Hr = 0;
    ps.pdl_mode = 1;
    const int k = streaming_ctas(p, c->num_sms, int4);
    const cudaError_t e = run([&] { return launch_decode_tc(ps, k, true, st); });
    if (e != cudaSuccess) return e;
    rest -= k;
    pr.pdl_mode = 2;
  }
  return run([&] {
    return int4 ? launch_decode_int4_tc(pr, rest, true, st) : launch_decode_fp8_tc(pr, rest, true, st);
  });
}

cudaError_t launch_decode_any(const duo_cache *c, const DecodeParams &p, cudaStream_t st) {
  const bool int4 = c->fmt == DUO_KV_INT4_G128;
  if (c->fmt == DUO_KV_FP8_E4M3) {
    if (!decode_fp8_tc_supported(p, c->dtype)) return cudaErrorNotSupported;
    return launch_quantised_layer(c, p, false, false, st);
  }
  // the tcgen05 decodes overlap their start-up with the previous kernel on the stream
  // (decode_int4_tc_supported implies decode_tc_supported for the streaming view)
  if (int4 && decode_int4_tc_supported(p, c->dtype)) return launch_quantised_layer(c, p, true, false, st);
  if (decode_tc_supported(p, c->dtype, int4)) return launch_decode_tc(p, c->num_sms, true, st);
  return launch_decode(p, c->dtype, int4, st);
}

// The decode launches of `p`, each through the test controls.
cudaError_t decode_any(const duo_cache *c, const DecodeParams &p, cudaStream_t st) {
  const bool int4 = c->fmt == DUO_KV_INT4_G128 && decode_int4_tc_supported(p, c->dtype);
  const bool fp8 = c->fmt == DUO_KV_FP8_E4M3 && decode_fp8_tc_supported(p, c->dtype);
  if (dry_run() || (!int4 && !fp8) || p.Hs == 0) return launch_via_hook([&] { return launch_decode_any(c, p, st); });
  // quantised layer with streaming heads: two launches (each counted by the test controls)
  return launch_quantised_layer(c, p, int4, true, st);
}

bool decode_args_ok(const void *q, const void *out, const float *lse) {
  return q && out && aligned16(q) && aligned16(out) && !(reinterpret_cast<uintptr_t>(lse) & 3u);
}

}  // namespace

extern "C" {

duo_status duo_decode_attention(duo_cache *c, int layer, const void *q, void *out, float *lse, void *stream) {
  DUO_NVTX_RANGE("duo_decode_attention");
  if (!layer_ok(c, layer) || !decode_args_ok(q, out, lse)) return DUO_ERR_INVALID;
  Layer &ly = c->L[layer];
  if (ly.len < 1) return DUO_ERR_INVALID;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  duo_status s = ensure_init(c, st);
  if (s != DUO_OK) return s;
  if (decode_any(c, decode_params(c, ly, q, out, lse), st) != cudaSuccess) return DUO_ERR_CUDA;
  return DUO_OK;
}

duo_status duo_append_decode(duo_cache *c, int layer, const void *q, const void *k, const void *v, void *out,
                             float *lse, void *stream) {
  DUO_NVTX_RANGE("duo_append_decode");
  if (!layer_ok(c, layer) || !decode_args_ok(q, out, lse) || !k || !v || !aligned16(k) || !aligned16(v))
    return DUO_ERR_INVALID;
  Layer &ly = c->L[layer];
  if (ly.len + 1 > c->max_len) return DUO_ERR_CAPACITY;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  duo_status s = ensure_init(c, st);
  if (s != DUO_OK) return s;
  const bool int4 = c->fmt != DUO_KV_SAME;  // quantised caches take the two-launch path
  Layer next = ly;
  next.len = ly.len + 1;
  DecodeParams p = decode_params(c, next, q, out, lse);
  // One launch where it measured faster (batch 1: 53.1 against 55.4 us per Llama-3 128K
  // layer step); at batch 4 the append kernel ahead of a dependent decode measured
  // faster (169.5 against 177.6 us), so larger batches keep the two launches.
  if (!int4 && c->B == 1 && !dry_run() && decode_tc_supported(p, c->dtype, int4)) {
    // one launch: the decode kernel writes the token's rows before it reads their tiles
    p.nk = static_cast<const char *>(k);
    p.nv = static_cast<const char *>(v);
    p.npos = ly.len;
    if (launch_via_hook([&] { return launch_decode_tc(p, c->num_sms, true, st); }) != cudaSuccess) return DUO_ERR_CUDA;
    ly.len += 1;
    return DUO_OK;
  }
  const AppendParams ap = append_params(c, ly, k, v, 1);
  if (launch_via_hook([&] { return launch_append(ap, c->dtype, st); }) != cudaSuccess) return DUO_ERR_CUDA;
  // the token is in the cache now: len follows what the cache holds, even if the
  // attention launch below fails
  ly.len += 1;
  if (decode_any(c, p, st) != cudaSuccess) return DUO_ERR_CUDA;
  return DUO_OK;
}

duo_status duo_cache_len(const duo_cache *c, int layer, int64_t *len) {
  if (!layer_ok(c, layer) || !len) return DUO_ERR_INVALID;
  *len = c->L[layer].len;
  return DUO_OK;
}

duo_status duo_kv_bytes(const duo_cache *c, int64_t Lq, uint64_t *retained, uint64_t *full) {
  if (!c || Lq < 0) return DUO_ERR_INVALID;
  const uint64_t row = static_cast<uint64_t>(c->D) * c->esize;
  const uint64_t rrow = c->fmt == DUO_KV_INT4_G128   ? static_cast<uint64_t>(c->D / 2 + 4)
                        : c->fmt == DUO_KV_FP8_E4M3 ? static_cast<uint64_t>(c->D + 4)
                                                    : row;
  const uint64_t keep = static_cast<uint64_t>(std::min<int64_t>(Lq, static_cast<int64_t>(c->S) + c->W));
  uint64_t r = 0;
  for (const Layer &ly : c->L) r += static_cast<uint64_t>(ly.Hr) * Lq * rrow + static_cast<uint64_t>(ly.Hs) * keep * row;
  if (retained) *retained = 2ull * c->B * r;
  if (full) *full = 2ull * c->B * c->layers * c->Hkv * static_cast<uint64_t>(Lq) * row;
  return DUO_OK;
}

duo_status duo_debug_slot_position(const duo_cache *c, int layer, int kv_head, int slot, int64_t *pos) {
  if (!layer_ok(c, layer) || kv_head < 0 || kv_head >= c->Hkv || !pos || slot < 0) return DUO_ERR_INVALID;
  const Layer &ly = c->L[layer];
  const int64_t len = ly.len;
  if (ly.hm.is_retr[kv_head]) {
    if (slot >= c->max_len) return DUO_ERR_INVALID;
    *pos = slot < len ? slot : -1;
    return DUO_OK;
  }
  if (slot >= c->S + c->W) return DUO_ERR_INVALID;
  if (slot < c->S) {
    *pos = slot < len ? slot : -1;
    return DUO_OK;
  }
  // latest position p < len with p >= S and p mod W == slot - S
  const int64_t off = slot - c->S;
  if (len < 1) {
    *pos = -1;
    return DUO_OK;
  }
  const int64_t last = len - 1;
  const int64_t back = ((last - off) % c->W + c->W) % c->W;
  const int64_t p = last - back;
  *pos = p >= c->S ? p : -1;
  return DUO_OK;
}

duo_status duo_debug_region(const duo_cache *c, int layer, duo_region which, void **ptr, uint64_t *bytes,
                            int64_t *cap) {
  if (!layer_ok(c, layer)) return DUO_ERR_INVALID;
  const Layer &ly = c->L[layer];
  const bool quant = c->fmt != DUO_KV_SAME;
  const uint64_t row = static_cast<uint64_t>(c->D) * c->esize;
  const uint64_t rrow = c->fmt == DUO_KV_INT4_G128   ? static_cast<uint64_t>(c->D / 2)
                        : c->fmt == DUO_KV_FP8_E4M3 ? static_cast<uint64_t>(c->D)
                                                    : row;
  const uint64_t rrows = static_cast<uint64_t>(c->B) * ly.Hr * c->cap;
  const uint64_t srows = static_cast<uint64_t>(c->B) * ly.Hs * (static_cast<uint64_t>(c->S) + c->W);
  char *p = nullptr;
  uint64_t n = 0;
  switch (which) {
    case DUO_REGION_RETR_K: p = ly.rk; n = rrows * rrow; break;
    case DUO_REGION_RETR_V: p = ly.rv; n = rrows * rrow; break;
    case DUO_REGION_RETR_KSZ: if (!quant) return DUO_ERR_INVALID; p = ly.rk_sz; n = rrows * 4; break;
    case DUO_REGION_RETR_VSZ: if (!quant) return DUO_ERR_INVALID; p = ly.rv_sz; n = rrows * 4; break;
    case DUO_REGION_STRM_K: p = ly.sk; n = srows * row; break;
    case DUO_REGION_STRM_V: p = ly.sv; n = srows * row; break;
    default: return DUO_ERR_INVALID;
  }
  if (ptr) *ptr = p;
  if (bytes) *bytes = n;
  if (cap) *cap = c->cap;
  return DUO_OK;
}

duo_status duo_get_device_status(duo_cache *c, void *stream) {
  DUO_NVTX_RANGE("duo_get_device_status");
  if (!c) return DUO_ERR_INVALID;
  if (!c->initialised || dry_run()) return DUO_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return DUO_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpy(&word, c->status, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return DUO_ERR_CUDA;
  if (word == 0) return DUO_OK;
  if (cudaMemset(c->status, 0, 4) != cudaSuccess) return DUO_ERR_CUDA;
  return (word & kDevTimeout) ? DUO_ERR_TIMEOUT : DUO_ERR_CUDA;
}

duo_status duo_debug_launch_controls(int dry_run, int64_t fail_after) {
  if ((dry_run != 0 && dry_run != 1) || fail_after < -1) return DUO_ERR_INVALID;
  g_dry_run.store(dry_run);
  g_fail_countdown.store(fail_after);
  return DUO_OK;
}

duo_status duo_debug_device_stall(int on) {
  if (on != 0 && on != 1) return DUO_ERR_INVALID;
  g_device_stall.store(on);
  return DUO_OK;
}

}  // extern "C"

namespace duo {

bool dry_run() { return g_dry_run.load(std::memory_order_relaxed) != 0; }

bool launch_intercepted(cudaError_t *e) {
  int64_t left = g_fail_countdown.load(std::memory_order_relaxed);
  while (left >= 0) {
    if (g_fail_countdown.compare_exchange_weak(left, left - 1)) {
      if (left == 0) {  // this launch is the one that fails; nothing is launched
        *e = cudaErrorLaunchFailure;
        return true;
      }
      break;
    }
  }
  if (dry_run()) {
    *e = cudaSuccess;
    return true;
  }
  return false;
}

}  // namespace duo
