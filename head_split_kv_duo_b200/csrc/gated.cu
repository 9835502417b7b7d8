// gated.cu -- gated mixed attention of the identification phase ("Gate
// Parameterization"): per KV head g, alpha[g] * full_attn + (1 - alpha[g]) *
// streaming_attn over whole sequences, with the masks of "The Full and Streaming
// Attention Masks".
//
// Both terms run through the library's pre-fill kernels straight over the caller's q,
// k and v, as one chunk at position 0 (no cache, nothing appended, no copy of K or V):
// the first launch treats every KV head as a retrieval head (causal mask) and writes
// the full-attention term to `out`; the second treats every head as a streaming head
// (Lambda mask, tile-skipping) and, in its epilogue, blends each row with the row the
// first launch wrote: out = alpha[g] * out + (1 - alpha[g]) * streaming.  Fusing the two
// into one pass would save only the logits of the Lambda-visible tiles, about (S+W)/L of
// the causal work, and would need a second output accumulator in tensor memory.
#include <cmath>

#include "duo_internal.h"
#include "nvtx_range.h"

namespace duo {

namespace {

bool gated_args_ok(int B, int L, int Hq, int Hkv, int d, duo_dtype dt, int S, int W) {
  if (B < 1 || B > 65536 || L < 1 || Hkv < 1 || Hkv > kMaxKvHeads || Hq < Hkv || Hq % Hkv || Hq > 4096) return false;
  if ((d != 64 && d != 128) || S < 0 || W < 1 || S > (1 << 24) || W > (1 << 24)) return false;
  return dt == DUO_BF16 || dt == DUO_FP32;
}

// One pass over whole sequences: every KV head retrieval (causal) or streaming (Lambda).
PrefillParams pass_params(const void *q, const void *k, const void *v, int B, int L, int Hq, int Hkv, int d, int S,
                          int W, float scale, void *out, bool causal, const float *mix_alpha) {
  PrefillParams p{};
  p.q = static_cast<const char *>(q);
  p.k = static_cast<const char *>(k);
  p.v = static_cast<const char *>(v);
  p.out = static_cast<char *>(out);
  p.B = B;
  p.n = L;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.D = d;
  p.Hr = causal ? Hkv : 0;
  p.Hs = causal ? 0 : Hkv;
  p.HsMax = p.Hs;
  p.S = S;
  p.W = W;
  p.len = 0;      // no cached positions and no streaming history: every key is in the chunk
  p.max_len = 256;
  p.hs = p.hw = 0;
  p.wstart = S;
  p.scale_log2 = scale * 1.4426950408889634f;
  for (int g = 0; g < Hkv; ++g) {
    p.hm.is_retr[g] = causal ? 1 : 0;
    p.hm.kind_idx[g] = static_cast<uint8_t>(g);
    p.hm.retr_head[g] = static_cast<uint8_t>(g);
    p.hm.strm_head[g] = static_cast<uint8_t>(g);
  }
  p.mix_alpha = mix_alpha;
  return p;
}

}  // namespace

}  // namespace duo

extern "C" duo_status duo_gated_attention(const void *q, const void *k, const void *v, int batch, int seq_len,
                                          int q_heads, int kv_heads, int head_dim, duo_dtype dtype,
                                          const float *alpha, int S, int W, float softmax_scale, void *out,
                                          void *stream) {
  DUO_NVTX_RANGE("duo_gated_attention");
  using namespace duo;
  if (!gated_args_ok(batch, seq_len, q_heads, kv_heads, head_dim, dtype, S, W)) return DUO_ERR_INVALID;
  if (!q || !k || !v || !alpha || !out || !(softmax_scale >= 0.f) || !std::isfinite(softmax_scale))
    return DUO_ERR_INVALID;
  const uintptr_t mis = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                        reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(out);
  if ((mis & 15u) || (reinterpret_cast<uintptr_t>(alpha) & 3u)) return DUO_ERR_INVALID;
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.f / std::sqrt(static_cast<float>(head_dim));
  const PrefillParams full = pass_params(q, k, v, batch, seq_len, q_heads, kv_heads, head_dim, S, W, scale, out,
                                         true, nullptr);
  const PrefillParams strm = pass_params(q, k, v, batch, seq_len, q_heads, kv_heads, head_dim, S, W, scale, out,
                                         false, alpha);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // every fallible set-up step before the first launch
  const bool tc = prefill_tc_supported(full, dtype) && prefill_tc_supported(strm, dtype) && !dry_run();
  PrefillTcLaunch lf, ls;
  if (tc && (prepare_prefill_tc(full, &lf) != cudaSuccess || prepare_prefill_tc(strm, &ls) != cudaSuccess))
    return DUO_ERR_CUDA;
  cudaError_t e = launch_via_hook([&] { return tc ? launch_prefill_tc(lf, st) : launch_prefill_simt(full, dtype, st); });
  if (e == cudaSuccess)
    e = launch_via_hook([&] { return tc ? launch_prefill_tc(ls, st) : launch_prefill_simt(strm, dtype, st); });
  return e == cudaSuccess ? DUO_OK : DUO_ERR_CUDA;
}
