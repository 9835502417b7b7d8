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
// 128 * 6 floats of shared memory.  `part` is global memory, or with kSmem a copy of
// the item's rows in shared memory: the arithmetic, and so every bit of the result, is
// the same either way, whichever CTA merges.
//
// Thread work: column c (one float4 of one query head's output row) and segment lane
// sl; with fewer than 128 columns the threads split the segments into nsl interleaved
// lanes, combined through `cmb` at the end.  Loads are issued in batches of 8
// segments, so the merge costs about ceil(nseg / (8 nsl)) round trips to L2.
template <bool kSmem = false>
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
            if (kSmem) {
              mm[i] = row[kD];
              ll[i] = row[kD + 1];
              vv[i] = reinterpret_cast<const float4 *>(row)[c4];
            } else {
              mm[i] = __ldcg(row + kD);
              ll[i] = __ldcg(row + kD + 1);
              vv[i] = __ldcg(reinterpret_cast<const float4 *>(row) + c4);
            }
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

}  // namespace duo
