// decode_merge.cuh -- the split-KV merge ("Decoding Procedure", step 5: the outputs of
// the parts of one head's cache are combined) shared by the tcgen05 decode kernels.
//
// A partial row is [o_0 .. o_{d-1}, m, l, pad, pad] in fp32: the unnormalised output
// sum_t exp2(s_t - m) v_t, the reference max m (log2 domain) and the sum l of the same
// weights.  The rows of one (batch, KV head) item sit at
//   part + (segment * G + q) * (d + 4).
#pragma once

#include "device_common.cuh"

namespace duo {

constexpr int kPartRow = 128 + 4;  // partial row length for head_dim 128

// Merges the nseg partial rows of every query head q < G of one item and writes the
// bf16 outputs out[b][h0 + q][.] and lse[b][h0 + q] (natural log).  Run by the 128
// threads of named barrier `bar_id`; t is the caller's index among them and `cmb` is
// 128 * 6 floats of shared memory.
//
// Thread work: column c (one float4 of one query head's output row) and segment lane
// sl; with fewer than 128 columns the threads split the segments into nsl interleaved
// lanes, combined through `cmb` at the end.  Loads are issued in batches of 8
// segments, so the merge costs about ceil(nseg / (8 nsl)) round trips to L2.
__device__ __forceinline__ void merge_partials(const float *part, int nseg, int G, int b, int h0, int Hq, char *out,
                                               float *lse, float *cmb, int t, int bar_id) {
  constexpr int kD = 128;
  constexpr int kBatch = 8;
  const int cols = G * (kD / 4);
  const int nsl = cols >= 128 ? 1 : 128 / cols;
  for (int c0 = 0; c0 < cols; c0 += 128) {
    const int col = cols >= 128 ? c0 + t : t % cols;
    const int sl = cols >= 128 ? 0 : t / cols;
    const bool active = col < cols && sl < nsl;
    const int q = col >> 5, c4 = col & 31;
    float M = -INFINITY, den = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (active) {
      for (int s0 = sl; s0 < nseg; s0 += kBatch * nsl) {
        float mm[kBatch], ll[kBatch];
        float4 vv[kBatch];
#pragma unroll
        for (int i = 0; i < kBatch; ++i) {
          const int sg = s0 + i * nsl;
          if (sg < nseg) {
            const float *row = part + (static_cast<int64_t>(sg) * G + q) * kPartRow;
            mm[i] = __ldcg(row + kD);
            ll[i] = __ldcg(row + kD + 1);
            vv[i] = __ldcg(reinterpret_cast<const float4 *>(row) + c4);
          } else {
            mm[i] = -INFINITY;
            ll[i] = 0.f;
            vv[i] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
        float Mb = M;
#pragma unroll
        for (int i = 0; i < kBatch; ++i) Mb = fmaxf(Mb, mm[i]);
        if (Mb == -INFINITY) continue;  // nothing visible so far
        const float r = (M == -INFINITY) ? 0.f : ex2(M - Mb);
        den *= r;
        acc.x *= r;
        acc.y *= r;
        acc.z *= r;
        acc.w *= r;
#pragma unroll
        for (int i = 0; i < kBatch; ++i) {
          const float w = (mm[i] == -INFINITY) ? 0.f : ex2(mm[i] - Mb);
          den = fmaf(w, ll[i], den);
          acc.x = fmaf(w, vv[i].x, acc.x);
          acc.y = fmaf(w, vv[i].y, acc.y);
          acc.z = fmaf(w, vv[i].z, acc.z);
          acc.w = fmaf(w, vv[i].w, acc.w);
        }
        M = Mb;
      }
    }
    if (nsl > 1) {
      if (active) {
        float *e = cmb + t * 6;
        e[0] = M;
        e[1] = den;
        e[2] = acc.x;
        e[3] = acc.y;
        e[4] = acc.z;
        e[5] = acc.w;
      }
      asm volatile("bar.sync %0, 128;" ::"r"(bar_id) : "memory");
      if (active && sl == 0) {
        for (int k = 1; k < nsl; ++k) {
          const float *e = cmb + (t + k * cols) * 6;
          const float Mn = fmaxf(M, e[0]);
          if (Mn == -INFINITY) continue;
          const float ra = (M == -INFINITY) ? 0.f : ex2(M - Mn);
          const float rb = (e[0] == -INFINITY) ? 0.f : ex2(e[0] - Mn);
          den = den * ra + e[1] * rb;
          acc.x = acc.x * ra + e[2] * rb;
          acc.y = acc.y * ra + e[3] * rb;
          acc.z = acc.z * ra + e[4] * rb;
          acc.w = acc.w * ra + e[5] * rb;
          M = Mn;
        }
      }
    }
    if (active && sl == 0) {
      const float inv = 1.f / den;
      const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
      const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
      uint2 pk;
      pk.x = *reinterpret_cast<const uint32_t *>(&lo);
      pk.y = *reinterpret_cast<const uint32_t *>(&hi);
      const int h = h0 + q;
      *reinterpret_cast<uint2 *>(out + ((static_cast<int64_t>(b) * Hq + h) * kD + 4 * c4) * 2) = pk;
      if (c4 == 0 && lse) lse[b * Hq + h] = (M + lg2(den)) * kLn2;
    }
  }
  asm volatile("bar.sync %0, 128;" ::"r"(bar_id) : "memory");  // cmb is reused by the caller
}

// merge_partials for rows already copied into (writable) shared memory: the per-head
// maxima are found first and each row's m is replaced by its weight exp2(m - max), so
// the weighted sums that follow are independent (no rescaling chain).
__device__ __forceinline__ void merge_partials_smem(float *rows, int nseg, int G, int b, int h0, int Hq, char *out,
                                                    float *lse, float *cmb, int t, int bar_id) {
  constexpr int kD = 128;
  if (t < G) {
    float M0 = -INFINITY, M1 = -INFINITY;
    int s = 0;
    for (; s + 1 < nseg; s += 2) {
      M0 = fmaxf(M0, rows[(s * G + t) * kPartRow + kD]);
      M1 = fmaxf(M1, rows[((s + 1) * G + t) * kPartRow + kD]);
    }
    if (s < nseg) M0 = fmaxf(M0, rows[(s * G + t) * kPartRow + kD]);
    cmb[t] = fmaxf(M0, M1);
  }
  asm volatile("bar.sync %0, 128;" ::"r"(bar_id) : "memory");
  for (int i = t; i < nseg * G; i += 128) {
    float *r = rows + i * kPartRow;
    r[kD] = (r[kD] == -INFINITY) ? 0.f : ex2(r[kD] - cmb[i % G]);
  }
  asm volatile("bar.sync %0, 128;" ::"r"(bar_id) : "memory");
  const int cols = G * (kD / 4);
  const int nsl = cols >= 128 ? 1 : 128 / cols;
  float *lanes = cmb + 16;  // [128][5] per segment lane: den, acc
  for (int c0 = 0; c0 < cols; c0 += 128) {
    const int col = cols >= 128 ? c0 + t : t % cols;
    const int sl = cols >= 128 ? 0 : t / cols;
    const bool active = col < cols && sl < nsl;
    const int q = col >> 5, c4 = col & 31;
    float den = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (active) {
#pragma unroll 4
      for (int sg = sl; sg < nseg; sg += nsl) {
        const float *r = rows + (sg * G + q) * kPartRow;
        const float w = r[kD];
        const float4 v = reinterpret_cast<const float4 *>(r)[c4];
        den = fmaf(w, r[kD + 1], den);
        acc.x = fmaf(w, v.x, acc.x);
        acc.y = fmaf(w, v.y, acc.y);
        acc.z = fmaf(w, v.z, acc.z);
        acc.w = fmaf(w, v.w, acc.w);
      }
    }
    if (nsl > 1) {
      if (active) {
        float *e = lanes + t * 5;
        e[0] = den;
        e[1] = acc.x;
        e[2] = acc.y;
        e[3] = acc.z;
        e[4] = acc.w;
      }
      asm volatile("bar.sync %0, 128;" ::"r"(bar_id) : "memory");
      if (active && sl == 0) {
        for (int k = 1; k < nsl; ++k) {
          const float *e = lanes + (t + k * cols) * 5;
          den += e[0];
          acc.x += e[1];
          acc.y += e[2];
          acc.z += e[3];
          acc.w += e[4];
        }
      }
    }
    if (active && sl == 0) {
      const float inv = 1.f / den;
      const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
      const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
      uint2 pk;
      pk.x = *reinterpret_cast<const uint32_t *>(&lo);
      pk.y = *reinterpret_cast<const uint32_t *>(&hi);
      const int h = h0 + q;
      *reinterpret_cast<uint2 *>(out + ((static_cast<int64_t>(b) * Hq + h) * kD + 4 * c4) * 2) = pk;
      if (c4 == 0 && lse) lse[b * Hq + h] = (cmb[q] + lg2(den)) * kLn2;
    }
  }
  asm volatile("bar.sync %0, 128;" ::"r"(bar_id) : "memory");  // cmb is reused by the caller
}

}  // namespace duo
