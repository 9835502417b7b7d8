// k_prefill_simt.cu -- chunked pre-fill attention on the CUDA cores
// ("Chunked Pre-filling"; masks of "The Full and Streaming Attention Masks").
//
// Used for fp32 caches and for head_dim 64; bf16 / head_dim 128 pre-fill runs on the
// tensor cores (k_prefill_tc.cu).  One warp owns one query row (b, r, h) at position
// i = len + r; lanes split head_dim.  Keys come from two places:
//   * retrieval heads: the full cache for positions 0..len-1, then the chunk's own rows
//     0..r from the chunk input (the caller appends the chunk after the attention);
//   * streaming heads: the staged history (sinks 0..hs-1 and positions wstart..len-1)
//     and then the chunk's own rows, each filtered by the Lambda mask
//     (j < S or i - j < W) -- tiles of keys outside the mask are never touched.
#include "device_common.cuh"

namespace duo {

namespace {

template <typename T, int D>
struct WarpRow {
  static constexpr int E = D / 32;  // elements per lane
  float q[E], o[E];
  float m = -INFINITY, l = 0.f;

  __device__ __forceinline__ void key(const char *krow, const char *vrow, int lane) {
    float dot = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) dot = fmaf(q[e], Elem<T>::load(krow, lane * E + e), dot);
    const float s = warp_sum(dot);  // log2-domain logit (q is pre-scaled)
    const float mn = fmaxf(m, s);
    const float alpha = ex2(m - mn);  // 0 on the first key
    const float pj = ex2(s - mn);
    l = fmaf(l, alpha, pj);
#pragma unroll
    for (int e = 0; e < E; ++e) o[e] = fmaf(o[e], alpha, pj * Elem<T>::load(vrow, lane * E + e));
    m = mn;
  }
};

template <typename T, int D>
__global__ void __launch_bounds__(256) prefill_simt_kernel(const PrefillParams p) {
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t rows = static_cast<int64_t>(p.B) * p.n * p.Hq;
  if (warp >= rows) return;
  const int h = static_cast<int>(warp % p.Hq);
  const int64_t br = warp / p.Hq;
  const int r = static_cast<int>(br % p.n);
  const int b = static_cast<int>(br / p.n);
  const int g = h / p.G;
  const int64_t i = p.len + r;
  constexpr int RB = D * static_cast<int>(sizeof(T));
  WarpRow<T, D> st;
  const char *qrow = p.q + ((static_cast<int64_t>(b) * p.n + r) * p.Hq + h) * RB;
#pragma unroll
  for (int e = 0; e < WarpRow<T, D>::E; ++e) {
    st.q[e] = Elem<T>::load(qrow, lane * WarpRow<T, D>::E + e) * p.scale_log2;
    st.o[e] = 0.f;
  }
  const int idx = p.hm.kind_idx[g];
  if (p.hm.is_retr[g]) {
    const int64_t base = (static_cast<int64_t>(b) * p.Hr + idx) * p.max_len;
    for (int64_t j = 0; j < p.len; ++j) st.key(p.rk + (base + j) * RB, p.rv + (base + j) * RB, lane);
    for (int t = 0; t <= r; ++t) {  // positions len..i, causal
      const int64_t off = ((static_cast<int64_t>(b) * p.n + t) * p.Hkv + g) * RB;
      st.key(p.k + off, p.v + off, lane);
    }
  } else {
    const int64_t hbase = (static_cast<int64_t>(b) * p.HsMax + idx) * (p.S + p.W);
    // history rows: sinks (always visible) then the window rows still within W of i
    for (int t = 0; t < p.hs + p.hw; ++t) {
      const int64_t pos = t < p.hs ? t : p.wstart + (t - p.hs);
      if (pos < p.S || i - pos < p.W) st.key(p.hk + (hbase + t) * RB, p.hv + (hbase + t) * RB, lane);
    }
    // the chunk's own rows 0..r (positions len..i), Lambda mask
    for (int t = 0; t <= r; ++t) {
      const int64_t pos = p.len + t;
      if (pos < p.S || i - pos < p.W) {
        const int64_t off = ((static_cast<int64_t>(b) * p.n + t) * p.Hkv + g) * RB;
        st.key(p.k + off, p.v + off, lane);
      }
    }
  }
  const float inv = 1.f / st.l;
  char *orow = p.out + ((static_cast<int64_t>(b) * p.n + r) * p.Hq + h) * RB;
  // gated mixing: blend with the row already in out (each lane reads what it rewrites)
  const float mixa = p.mix_alpha ? p.mix_alpha[g] : 0.f;
#pragma unroll
  for (int e = 0; e < WarpRow<T, D>::E; ++e) {
    const int col = lane * WarpRow<T, D>::E + e;
    float x = st.o[e] * inv;
    if (p.mix_alpha) x = fmaf(mixa, Elem<T>::load(orow, col) - x, x);
    Elem<T>::store(orow, col, x);
  }
  if (lane == 0 && p.lse) p.lse[(static_cast<int64_t>(b) * p.n + r) * p.Hq + h] = (st.m + lg2(st.l)) * kLn2;
}

}  // namespace

cudaError_t launch_prefill_simt(const PrefillParams &p, duo_dtype dt, cudaStream_t st) {
  const int64_t warps = static_cast<int64_t>(p.B) * p.n * p.Hq;
  const unsigned blocks = static_cast<unsigned>((warps + 7) / 8);
  if (dt == DUO_BF16) {
    if (p.D == 128) prefill_simt_kernel<__nv_bfloat16, 128><<<blocks, 256, 0, st>>>(p);
    else if (p.D == 64) prefill_simt_kernel<__nv_bfloat16, 64><<<blocks, 256, 0, st>>>(p);
    else return cudaErrorNotSupported;
  } else {
    if (p.D == 128) prefill_simt_kernel<float, 128><<<blocks, 256, 0, st>>>(p);
    else if (p.D == 64) prefill_simt_kernel<float, 64><<<blocks, 256, 0, st>>>(p);
    else return cudaErrorNotSupported;
  }
  return cudaGetLastError();
}

}  // namespace duo
