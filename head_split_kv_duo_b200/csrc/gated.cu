// gated.cu -- gated mixed attention of the identification phase ("Gate
// Parameterization"): per KV head g, alpha[g] * full_attn + (1 - alpha[g]) *
// streaming_attn over whole sequences, with the masks of "The Full and Streaming
// Attention Masks".
//
// The two terms run through the library's own chunked pre-fill path, each on a
// one-layer cache carved from the caller's workspace: once with every KV head a
// retrieval head (causal mask, written to `out`) and once with every head a streaming
// head (Lambda mask, tile-skipping, written to the workspace).  A fused single pass
// would only save recomputing the logits of the Lambda-visible tiles, about (S+W)/L of
// the causal work, while needing a second output accumulator in tensor memory; the
// streaming pass is that small.  One elementwise kernel then mixes the two in place.
#include <algorithm>
#include <vector>

#include "device_common.cuh"

namespace duo {

namespace {

constexpr size_t kWsAlign = 1024;

size_t round_up(size_t x) { return (x + kWsAlign - 1) / kWsAlign * kWsAlign; }

// out = a * out + (1 - a) * strm, a = alpha[(element's query head) / G]; 16-byte vectors.
template <typename T>
__global__ void __launch_bounds__(256) gated_mix_kernel(char *out, const char *strm, const float *alpha,
                                                        int64_t nvec, int d, int Hq, int G) {
  constexpr int kPer = Elem<T>::per16;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nvec;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t e0 = i * kPer;  // first element of the vector; a vector never crosses a head row
    const int h = static_cast<int>((e0 / d) % Hq);
    const float a = alpha[h / G];
    const uint4 uo = reinterpret_cast<const uint4 *>(out)[i];
    const uint4 us = reinterpret_cast<const uint4 *>(strm)[i];
    float fo[kPer], fs[kPer];
    Elem<T>::unpack(uo, fo);
    Elem<T>::unpack(us, fs);
#pragma unroll
    for (int e = 0; e < kPer; ++e) Elem<T>::store(out, e0 + e, fmaf(a, fo[e] - fs[e], fs[e]));
  }
}

struct GatedLayout {
  size_t full, strm, o_strm, total;
};

bool gated_layout(int B, int L, int Hq, int Hkv, int d, duo_dtype dt, int S, int W, GatedLayout *g) {
  if (B < 1 || L < 1 || Hkv < 1 || Hq < Hkv || Hq % Hkv || (d != 64 && d != 128) || S < 0 || W < 1) return false;
  if (dt != DUO_BF16 && dt != DUO_FP32) return false;
  duo_opts o{};
  o.batch = B;
  o.q_heads = Hq;
  o.dtype = dt;
  o.retr_fmt = DUO_KV_SAME;
  o.softmax_scale = 0.f;
  std::vector<uint8_t> all(static_cast<size_t>(Hkv), 1), none(static_cast<size_t>(Hkv), 0);
  g->full = duo_cache_bytes(1, Hkv, d, all.data(), S, W, L, &o);
  g->strm = duo_cache_bytes(1, Hkv, d, none.data(), S, W, L, &o);
  if (g->full == 0 || g->strm == 0) return false;
  const size_t esize = dt == DUO_BF16 ? 2 : 4;
  g->o_strm = static_cast<size_t>(B) * L * Hq * d * esize;
  g->total = round_up(g->full) + round_up(g->strm) + round_up(g->o_strm);
  return true;
}

}  // namespace

}  // namespace duo

extern "C" size_t duo_gated_workspace_bytes(int batch, int seq_len, int q_heads, int kv_heads, int head_dim,
                                            duo_dtype dtype, int S, int W) {
  duo::GatedLayout g;
  return duo::gated_layout(batch, seq_len, q_heads, kv_heads, head_dim, dtype, S, W, &g) ? g.total : 0;
}

extern "C" duo_status duo_gated_attention(const void *q, const void *k, const void *v, int batch, int seq_len,
                                          int q_heads, int kv_heads, int head_dim, duo_dtype dtype,
                                          const float *alpha, int S, int W, float softmax_scale, void *out,
                                          void *workspace, size_t workspace_bytes, void *stream) {
  using namespace duo;
  GatedLayout g;
  if (!gated_layout(batch, seq_len, q_heads, kv_heads, head_dim, dtype, S, W, &g)) return DUO_ERR_INVALID;
  if (!q || !k || !v || !alpha || !out || !workspace || !(softmax_scale >= 0.f)) return DUO_ERR_INVALID;
  const uintptr_t mis = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                        reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(out);
  if ((mis & 15u) || (reinterpret_cast<uintptr_t>(alpha) & 3u) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return DUO_ERR_INVALID;
  if (workspace_bytes < g.total) return DUO_ERR_CAPACITY;

  duo_opts o{};
  o.batch = batch;
  o.q_heads = q_heads;
  o.dtype = dtype;
  o.retr_fmt = DUO_KV_SAME;
  o.softmax_scale = softmax_scale;
  std::vector<uint8_t> all(static_cast<size_t>(kv_heads), 1), none(static_cast<size_t>(kv_heads), 0);
  char *ws = static_cast<char *>(workspace);
  char *o_strm = ws + round_up(g.full) + round_up(g.strm);
  duo_cache *cf = nullptr, *cs = nullptr;
  duo_status s = duo_cache_create(1, kv_heads, head_dim, all.data(), S, W, seq_len, &o, ws, g.full, &cf);
  if (s == DUO_OK)
    s = duo_cache_create(1, kv_heads, head_dim, none.data(), S, W, seq_len, &o, ws + round_up(g.full), g.strm, &cs);
  // causal term into `out`, Lambda term into the workspace: one chunk of the whole sequence each
  if (s == DUO_OK) s = duo_prefill_chunk(cf, 0, q, k, v, seq_len, out, nullptr, stream);
  if (s == DUO_OK) s = duo_prefill_chunk(cs, 0, q, k, v, seq_len, o_strm, nullptr, stream);
  duo_cache_destroy(cf);
  duo_cache_destroy(cs);
  if (s != DUO_OK) return s;

  const int esize = dtype == DUO_BF16 ? 2 : 4;
  const int64_t nvec = static_cast<int64_t>(batch) * seq_len * q_heads * head_dim * esize / 16;
  const int64_t blocks = std::min<int64_t>((nvec + 255) / 256, 148 * 16);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int G = q_heads / kv_heads;
  if (dtype == DUO_BF16)
    gated_mix_kernel<__nv_bfloat16><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        static_cast<char *>(out), o_strm, alpha, nvec, head_dim, q_heads, G);
  else
    gated_mix_kernel<float><<<static_cast<unsigned>(blocks), 256, 0, st>>>(static_cast<char *>(out), o_strm, alpha,
                                                                         nvec, head_dim, q_heads, G);
  return cudaGetLastError() == cudaSuccess ? DUO_OK : DUO_ERR_CUDA;
}
