// k_append.cu -- cache update ("Decoding Procedure" step 4; "Chunked Pre-filling"
// pruning) and the staging copy of streaming-head history used by pre-fill.
//
// Slot rule (streaming heads): position p lives in slot p when p < S, else in ring
// slot S + (p mod W); writing a ring slot evicts the position W earlier.  Of an
// n-token append only the sinks and positions >= ring_from = max(S, len+n-W) are
// written: the others would be evicted inside the same call.
#include "device_common.cuh"

namespace duo {

namespace {

// One warp copies one row of `bytes` (a multiple of 16) with 16-byte vectors.
__device__ __forceinline__ void copy_row(char *dst, const char *src, int bytes, int lane) {
  const uint4 *s = reinterpret_cast<const uint4 *>(src);
  uint4 *d = reinterpret_cast<uint4 *>(dst);
  for (int c = lane; c < bytes / 16; c += 32) d[c] = __ldg(s + c);
}

// INT4 asymmetric quantisation of one bf16 row of 128 elements by one warp
// (format of duo.h: fp32 min/max, fp16 scale and zero, IEEE fp32 steps, rint).
__device__ __forceinline__ void quantize_row_int4(const char *src, uint8_t *codes, __half *sz, int lane) {
  const uint2 u = __ldg(reinterpret_cast<const uint2 *>(src) + lane);  // elements 4*lane .. 4*lane+3
  float x[4] = {bf16lo(u.x), bf16hi(u.x), bf16lo(u.y), bf16hi(u.y)};
  float mn = fminf(fminf(x[0], x[1]), fminf(x[2], x[3]));
  float mx = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  const float step = __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
  const __half scale_h = __float2half_rn(step);
  const __half zero_h = __float2half_rn(mn);
  const float scale = __half2float(scale_h);
  const float zero = __half2float(zero_h);
  uint32_t c[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    float r = 0.f;
    if (scale != 0.f) {
      r = rintf(__fdiv_rn(__fsub_rn(x[e], zero), scale));
      r = fminf(fmaxf(r, 0.f), 15.f);
    }
    c[e] = static_cast<uint32_t>(r);
  }
  const uint16_t packed = static_cast<uint16_t>(c[0] | (c[1] << 4) | (c[2] << 8) | (c[3] << 12));
  reinterpret_cast<uint16_t *>(codes)[lane] = packed;
  if (lane == 0) {
    sz[0] = scale_h;
    sz[1] = zero_h;
  }
}

// FP8 (OCP E4M3) quantisation of one bf16 row of 128 elements by one warp (format of
// duo.h: fp32 max |x|, scale = max / 448 and x / scale in IEEE fp32, nearest E4M3 value
// with ties to even, held at +-448).
__device__ __forceinline__ void quantize_row_fp8(const char *src, uint8_t *codes, float *scale_out, int lane) {
  const uint2 u = __ldg(reinterpret_cast<const uint2 *>(src) + lane);  // elements 4*lane .. 4*lane+3
  const float x[4] = {bf16lo(u.x), bf16hi(u.x), bf16lo(u.y), bf16hi(u.y)};
  float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
  amax = warp_max(amax);
  const float scale = __fdiv_rn(amax, 448.0f);
  float y[4] = {0.f, 0.f, 0.f, 0.f};
  if (scale != 0.f) {
#pragma unroll
    for (int e = 0; e < 4; ++e) y[e] = __fdiv_rn(x[e], scale);
  }
  uint16_t lo, hi;  // the first source lands in the upper byte
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(y[1]), "f"(y[0]));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(y[3]), "f"(y[2]));
  reinterpret_cast<uint32_t *>(codes)[lane] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
  if (lane == 0) *scale_out = scale;
}

template <typename T>
__global__ void __launch_bounds__(256) append_kernel(const AppendParams p) {
  // a decode launched right after may start its set-up now; it waits for this grid to
  // finish before its first global read
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t total = static_cast<int64_t>(p.B) * p.n * p.Hkv;
  if (warp >= total) return;
  const int g = static_cast<int>(warp % p.Hkv);
  const int64_t bt = warp / p.Hkv;
  const int t = static_cast<int>(bt % p.n);
  const int b = static_cast<int>(bt / p.n);
  const int64_t pos = p.len + t;
  const int RB = p.D * static_cast<int>(sizeof(T));
  const int64_t src_off = ((static_cast<int64_t>(b) * p.n + t) * p.Hkv + g) * RB;
  const int idx = p.hm.kind_idx[g];
  if (p.hm.is_retr[g]) {
    const int64_t row = (static_cast<int64_t>(b) * p.Hr + idx) * p.max_len + pos;
    if (p.fp8) {
      const int CB = p.D;  // code bytes per row
      quantize_row_fp8(p.k + src_off, reinterpret_cast<uint8_t *>(p.rk) + row * CB,
                       reinterpret_cast<float *>(p.rk_sz) + row, lane);
      quantize_row_fp8(p.v + src_off, reinterpret_cast<uint8_t *>(p.rv) + row * CB,
                       reinterpret_cast<float *>(p.rv_sz) + row, lane);
    } else if (!p.int4) {
      copy_row(p.rk + row * RB, p.k + src_off, RB, lane);
      copy_row(p.rv + row * RB, p.v + src_off, RB, lane);
    } else {
      const int CB = p.D / 2;  // code bytes per row
      quantize_row_int4(p.k + src_off, reinterpret_cast<uint8_t *>(p.rk) + row * CB,
                        reinterpret_cast<__half *>(p.rk_sz) + row * 2, lane);
      quantize_row_int4(p.v + src_off, reinterpret_cast<uint8_t *>(p.rv) + row * CB,
                        reinterpret_cast<__half *>(p.rv_sz) + row * 2, lane);
    }
  } else {
    if (pos >= p.S && pos < p.ring_from) return;  // evicted within this call: never stored
    const int64_t slot = pos < p.S ? pos : p.S + pos % p.W;
    const int64_t row = (static_cast<int64_t>(b) * p.Hs + idx) * (p.S + p.W) + slot;
    copy_row(p.sk + row * RB, p.k + src_off, RB, lane);
    copy_row(p.sv + row * RB, p.v + src_off, RB, lane);
  }
}

// Copies the streaming history a pre-fill chunk may see into position order:
// rows [0, hs) are the sinks 0..hs-1, rows [hs, hs+hw) are positions wstart.. .
template <typename T>
__global__ void __launch_bounds__(256) hist_kernel(const HistParams p) {
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int rows = p.hs + p.hw;
  const int64_t total = static_cast<int64_t>(p.B) * p.Hs * rows;
  if (warp >= total) return;
  const int r = static_cast<int>(warp % rows);
  const int64_t bs = warp / rows;
  const int si = static_cast<int>(bs % p.Hs);
  const int b = static_cast<int>(bs / p.Hs);
  const int64_t pos = r < p.hs ? r : p.wstart + (r - p.hs);
  const int64_t slot = pos < p.S ? pos : p.S + pos % p.W;
  const int RB = p.D * static_cast<int>(sizeof(T));
  const int64_t src = ((static_cast<int64_t>(b) * p.Hs + si) * (p.S + p.W) + slot) * RB;
  const int64_t dst = ((static_cast<int64_t>(b) * p.HsMax + si) * (p.S + p.W) + r) * RB;
  copy_row(p.hk + dst, p.sk + src, RB, lane);
  copy_row(p.hv + dst, p.sv + src, RB, lane);
}

}  // namespace

cudaError_t launch_append(const AppendParams &p, duo_dtype dt, cudaStream_t st) {
  const int64_t warps = static_cast<int64_t>(p.B) * p.n * p.Hkv;
  const int64_t blocks = (warps + 7) / 8;
  if (dt == DUO_BF16)
    append_kernel<__nv_bfloat16><<<static_cast<unsigned>(blocks), 256, 0, st>>>(p);
  else
    append_kernel<float><<<static_cast<unsigned>(blocks), 256, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_hist(const HistParams &p, duo_dtype dt, cudaStream_t st) {
  const int64_t warps = static_cast<int64_t>(p.B) * p.Hs * (p.hs + p.hw);
  if (warps == 0) return cudaSuccess;
  const int64_t blocks = (warps + 7) / 8;
  if (dt == DUO_BF16)
    hist_kernel<__nv_bfloat16><<<static_cast<unsigned>(blocks), 256, 0, st>>>(p);
  else
    hist_kernel<float><<<static_cast<unsigned>(blocks), 256, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace duo
