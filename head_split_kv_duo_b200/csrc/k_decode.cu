// k_decode.cu -- single-token decode attention over the hybrid cache
// ("Decoding Procedure", steps 2, 3 and 5).
//
// One launch covers every head of a layer:
//   * retrieval heads: split-KV flash-decode.  CTA (b, retrieval head, query group,
//     split) streams rows [split*split_len, ...) of the full cache, keeps a running
//     (max, sum, output) per query head, and writes a partial; the last CTA of a head
//     (atomic ticket, no waiting) merges the partials with their log-sum-exp weights.
//   * streaming heads: one CTA per (b, head, query group) over the S+W sink and ring
//     slots; every valid slot is visible to the newest query.
// The query heads of one GQA group share each K/V row a CTA reads.
//
// K/V rows are staged into shared memory by the TMA engine (cp.async.bulk, one
// contiguous block of rows per stage, mbarrier completion, 3 stages).  Four warps
// split a stage; inside a warp 8 lanes cover one 128-byte segment of a row, so four
// rows are read per instruction without bank conflicts.  Dot products are reduced
// over the 8 lanes by recursive halving (several tokens per shuffle round).
#include <type_traits>

#include "device_common.cuh"

namespace duo {

namespace {

constexpr int kThreads = 128;
constexpr int kWarps = 4;
constexpr int kStages = 3;
constexpr unsigned kFull = 0xffffffffu;

template <typename T, int D>
struct RowCfg {
  static constexpr int RB = D * static_cast<int>(sizeof(T));  // row bytes
  static constexpr int TPS = 16384 / RB;                       // rows per stage (16 KiB of K)
  static constexpr int TPW = TPS / kWarps;                     // rows per warp per stage
  static constexpr int SUB = (TPW / 4) >= 4 ? 4 : (TPW / 4);   // 4-row steps per softmax batch
  static constexpr int NSUB = TPW / (4 * SUB);
  static constexpr int PER16 = 16 / static_cast<int>(sizeof(T));
  static constexpr int CPL = RB / 128;                         // 16-byte chunks per lane per row
  static constexpr int EPL = CPL * PER16;                      // elements per lane = D / 8
  static constexpr int STAGE = 2 * TPS * RB;                   // K rows then V rows
};

struct I4Cfg {  // INT4 retrieval rows, d = 128
  static constexpr int CB = 64;                         // code bytes per row
  static constexpr int TPS = 256;                       // rows per stage
  static constexpr int TPW = TPS / kWarps;              // 64
  static constexpr int SUB = 4;
  static constexpr int NSUB = TPW / (4 * SUB);          // 4
  static constexpr int OFF_VC = TPS * CB;               // V codes
  static constexpr int OFF_KS = 2 * TPS * CB;           // K scale/zero
  static constexpr int OFF_VS = 2 * TPS * CB + TPS * 4; // V scale/zero
  static constexpr int STAGE = 2 * TPS * CB + 2 * TPS * 4;
};

// Step index held by lane j of an 8-lane group after group_reduce<N>, and the
// lowest lane holding a given step.
template <int N> __device__ __forceinline__ int lane_step(int j) {
  if constexpr (N == 4) return ((j >> 2) & 1) * 2 + ((j >> 1) & 1);
  else if constexpr (N == 2) return (j >> 2) & 1;
  else return 0;
}
template <int N> __device__ __forceinline__ int step_lane(int st) {
  if constexpr (N == 4) return ((st >> 1) << 2) | ((st & 1) << 1);
  else if constexpr (N == 2) return st << 2;
  else return 0;
}

// Sums v[0..N) over the 8 lanes of each group; lane j ends with the full sum for
// step lane_step<N>(j).  Recursive halving: N-1 + (3 - log2 N) shuffles.
template <int N>
__device__ __forceinline__ float group_reduce(float (&v)[N], int j) {
  if constexpr (N == 4) {
    const bool up4 = (j & 4) != 0;
    float a0 = (up4 ? v[2] : v[0]) + __shfl_xor_sync(kFull, up4 ? v[0] : v[2], 4);
    float a1 = (up4 ? v[3] : v[1]) + __shfl_xor_sync(kFull, up4 ? v[1] : v[3], 4);
    const bool up2 = (j & 2) != 0;
    float b0 = (up2 ? a1 : a0) + __shfl_xor_sync(kFull, up2 ? a0 : a1, 2);
    return b0 + __shfl_xor_sync(kFull, b0, 1);
  } else if constexpr (N == 2) {
    const bool up4 = (j & 4) != 0;
    float a0 = (up4 ? v[1] : v[0]) + __shfl_xor_sync(kFull, up4 ? v[0] : v[1], 4);
    a0 += __shfl_xor_sync(kFull, a0, 2);
    return a0 + __shfl_xor_sync(kFull, a0, 1);
  } else {
    float a0 = v[0] + __shfl_xor_sync(kFull, v[0], 4);
    a0 += __shfl_xor_sync(kFull, a0, 2);
    return a0 + __shfl_xor_sync(kFull, a0, 1);
  }
}

// Online-softmax update of one batch: s[q] is this lane's (log2-domain) logit,
// -inf when its token is invalid.  Returns p[q] and rescales the running state.
template <int QG, int EPL, int SUB>
__device__ __forceinline__ void softmax_batch(float (&s)[QG], float (&p)[QG], float (&m)[QG], float (&l)[QG],
                                              float (&o)[QG][EPL], float (&z)[QG]) {
  constexpr float kDup = static_cast<float>(SUB) / 8.0f;  // each token appears on 8/SUB lanes
#pragma unroll
  for (int q = 0; q < QG; ++q) {
    const float mt = warp_max(s[q]);
    if (mt > m[q]) {  // warp-uniform
      const float alpha = ex2(m[q] - mt);  // 0 while m is still -inf
      l[q] *= alpha;
      z[q] *= alpha;
#pragma unroll
      for (int e = 0; e < EPL; ++e) o[q][e] *= alpha;
      m[q] = mt;
    }
    p[q] = (s[q] == -INFINITY) ? 0.f : ex2(s[q] - m[q]);
    l[q] += p[q] * kDup;
  }
}

struct CtaSmem {
  char *stages;
  uint32_t bar0;  // kStages consecutive 8-byte mbarriers
  float *red;     // [kWarps][QG][D+2]
  float *wts;     // [QG][kMaxSplits]
  int *flag;
};

// ---- streaming/retrieval rows in the working dtype ----
template <typename T, int D, int QG, typename Valid>
__device__ __forceinline__ void run_rows(const char *kbase, const char *vbase, int64_t ntok, Valid valid,
                                         const float (&qf)[QG][D / 8], float (&m)[QG], float (&l)[QG],
                                         float (&o)[QG][D / 8], float (&z)[QG], const CtaSmem &sm,
                                         uint32_t *status) {
  using C = RowCfg<T, D>;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, g = lane >> 3, j = lane & 7;
  const int ntiles = static_cast<int>((ntok + C::TPS - 1) / C::TPS);
  auto issue = [&](int t) {
    const int s = t % kStages;
    const int64_t r0 = static_cast<int64_t>(t) * C::TPS;
    const int64_t nr = (ntok - r0) < C::TPS ? (ntok - r0) : C::TPS;
    const uint32_t bytes = static_cast<uint32_t>(nr * C::RB);
    const uint32_t bar = sm.bar0 + 8 * s;
    const uint32_t dst = smem_u32(sm.stages + s * C::STAGE);
    mbar_expect_tx(bar, 2 * bytes);
    bulk_g2s(dst, kbase + r0 * C::RB, bytes, bar);
    bulk_g2s(dst + C::TPS * C::RB, vbase + r0 * C::RB, bytes, bar);
  };
  if (tid == 0)
    for (int t = 0; t < kStages && t < ntiles; ++t) issue(t);

#pragma unroll 1
  for (int t = 0; t < ntiles; ++t) {
    const int s = t % kStages;
    mbar_wait(sm.bar0 + 8 * s, (t / kStages) & 1, status);
    const char *ks = sm.stages + s * C::STAGE;
    const char *vs = ks + C::TPS * C::RB;
    const int64_t tbase = static_cast<int64_t>(t) * C::TPS;
#pragma unroll
    for (int sb = 0; sb < C::NSUB; ++sb) {
      const int rbase = w * C::TPW + sb * C::SUB * 4;  // first row of this batch in the stage
      float part[C::SUB][QG];
#pragma unroll
      for (int st = 0; st < C::SUB; ++st) {
        const char *krow = ks + (rbase + st * 4 + g) * C::RB;
#pragma unroll
        for (int q = 0; q < QG; ++q) part[st][q] = 0.f;
#pragma unroll
        for (int c = 0; c < C::CPL; ++c) {
          const uint4 u = *reinterpret_cast<const uint4 *>(krow + (j + 8 * c) * 16);
          float f[C::PER16];
          Elem<T>::unpack(u, f);
#pragma unroll
          for (int e = 0; e < C::PER16; ++e)
#pragma unroll
            for (int q = 0; q < QG; ++q) part[st][q] = fmaf(qf[q][c * C::PER16 + e], f[e], part[st][q]);
        }
      }
      float sc[QG], p[QG];
      const int my_row = rbase + lane_step<C::SUB>(j) * 4 + g;
      const bool my_ok = (tbase + my_row < ntok) && valid(tbase + my_row);
#pragma unroll
      for (int q = 0; q < QG; ++q) {
        float v[C::SUB];
#pragma unroll
        for (int st = 0; st < C::SUB; ++st) v[st] = part[st][q];
        const float r = group_reduce<C::SUB>(v, j);
        sc[q] = my_ok ? r : -INFINITY;
      }
      softmax_batch<QG, D / 8, C::SUB>(sc, p, m, l, o, z);
#pragma unroll
      for (int st = 0; st < C::SUB; ++st) {
        const int row = rbase + st * 4 + g;
        float pt[QG];
#pragma unroll
        for (int q = 0; q < QG; ++q) pt[q] = __shfl_sync(kFull, p[q], (g << 3) | step_lane<C::SUB>(st));
        const bool ok = (tbase + row < ntok) && valid(tbase + row);
        if (ok) {
          const char *vrow = vs + row * C::RB;
#pragma unroll
          for (int c = 0; c < C::CPL; ++c) {
            const uint4 u = *reinterpret_cast<const uint4 *>(vrow + (j + 8 * c) * 16);
            float f[C::PER16];
            Elem<T>::unpack(u, f);
#pragma unroll
            for (int e = 0; e < C::PER16; ++e)
#pragma unroll
              for (int q = 0; q < QG; ++q) o[q][c * C::PER16 + e] = fmaf(pt[q], f[e], o[q][c * C::PER16 + e]);
          }
        }
      }
    }
    __syncthreads();  // every warp is done with stage s
    if (tid == 0 && t + kStages < ntiles) issue(t + kStages);
  }
}

// ---- INT4 retrieval rows (bf16 queries, d = 128) ----
// logit = scale_k * sum_t q_t c_t + zero_k * sum_t q_t ; output = sum_j p_j (scale_v c_j + zero_v)
template <int QG>
__device__ __forceinline__ void run_rows_int4(const uint8_t *kc, const uint8_t *vc, const __half *ksz,
                                              const __half *vsz, int64_t ntok, const float (&qf)[QG][16],
                                              const float (&qsum)[QG], float (&m)[QG], float (&l)[QG],
                                              float (&o)[QG][16], float (&z)[QG], const CtaSmem &sm,
                                              uint32_t *status) {
  using C = I4Cfg;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, g = lane >> 3, j = lane & 7;
  const int ntiles = static_cast<int>((ntok + C::TPS - 1) / C::TPS);
  auto issue = [&](int t) {
    const int s = t % kStages;
    const int64_t r0 = static_cast<int64_t>(t) * C::TPS;
    const int64_t nr = (ntok - r0) < C::TPS ? (ntok - r0) : C::TPS;
    const uint32_t cbytes = static_cast<uint32_t>(nr * C::CB);
    const uint32_t zbytes = static_cast<uint32_t>(((nr * 4) + 15) & ~15ll);  // rows are padded to 16 B
    const uint32_t bar = sm.bar0 + 8 * s;
    const uint32_t dst = smem_u32(sm.stages + s * C::STAGE);
    mbar_expect_tx(bar, 2 * cbytes + 2 * zbytes);
    bulk_g2s(dst, kc + r0 * C::CB, cbytes, bar);
    bulk_g2s(dst + C::OFF_VC, vc + r0 * C::CB, cbytes, bar);
    bulk_g2s(dst + C::OFF_KS, ksz + r0 * 2, zbytes, bar);
    bulk_g2s(dst + C::OFF_VS, vsz + r0 * 2, zbytes, bar);
  };
  if (tid == 0)
    for (int t = 0; t < kStages && t < ntiles; ++t) issue(t);

  auto decode16 = [](uint2 u, float (&f)[16]) {
    // element 2t in the low nibble of byte t; float(2^23 + c) - 2^23 = c exactly
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t wv = h ? u.y : u.x;
      const uint32_t lo = wv & 0x0F0F0F0Fu, hi = (wv >> 4) & 0x0F0F0F0Fu;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        f[h * 8 + 2 * k] = __uint_as_float(__byte_perm(lo, 0x4B000000u, 0x7540u + k)) - 8388608.0f;
        f[h * 8 + 2 * k + 1] = __uint_as_float(__byte_perm(hi, 0x4B000000u, 0x7540u + k)) - 8388608.0f;
      }
    }
  };

#pragma unroll 1
  for (int t = 0; t < ntiles; ++t) {
    const int s = t % kStages;
    mbar_wait(sm.bar0 + 8 * s, (t / kStages) & 1, status);
    const char *st_base = sm.stages + s * C::STAGE;
    const int64_t tbase = static_cast<int64_t>(t) * C::TPS;
#pragma unroll 1
    for (int sb = 0; sb < C::NSUB; ++sb) {
      const int rbase = w * C::TPW + sb * C::SUB * 4;
      float part[C::SUB][QG];
#pragma unroll
      for (int st = 0; st < C::SUB; ++st) {
        const int row = rbase + st * 4 + g;
        const uint2 u = *reinterpret_cast<const uint2 *>(st_base + row * C::CB + j * 8);
        float f[16];
        decode16(u, f);
#pragma unroll
        for (int q = 0; q < QG; ++q) {
          float a = 0.f;
#pragma unroll
          for (int e = 0; e < 16; ++e) a = fmaf(qf[q][e], f[e], a);
          part[st][q] = a;
        }
      }
      const int my_row = rbase + lane_step<C::SUB>(j) * 4 + g;
      const bool my_ok = tbase + my_row < ntok;
      const float2 szk = __half22float2(*reinterpret_cast<const __half2 *>(st_base + C::OFF_KS + my_row * 4));
      float sc[QG], p[QG];
#pragma unroll
      for (int q = 0; q < QG; ++q) {
        float v[C::SUB];
#pragma unroll
        for (int st = 0; st < C::SUB; ++st) v[st] = part[st][q];
        const float dot = group_reduce<C::SUB>(v, j);
        sc[q] = my_ok ? fmaf(szk.x, dot, szk.y * qsum[q]) : -INFINITY;
      }
      softmax_batch<QG, 16, C::SUB>(sc, p, m, l, o, z);
#pragma unroll
      for (int st = 0; st < C::SUB; ++st) {
        const int row = rbase + st * 4 + g;
        float pt[QG];
#pragma unroll
        for (int q = 0; q < QG; ++q) pt[q] = __shfl_sync(kFull, p[q], (g << 3) | step_lane<C::SUB>(st));
        if (tbase + row < ntok) {
          const float2 szv = __half22float2(*reinterpret_cast<const __half2 *>(st_base + C::OFF_VS + row * 4));
          const uint2 u = *reinterpret_cast<const uint2 *>(st_base + C::OFF_VC + row * C::CB + j * 8);
          float f[16];
          decode16(u, f);
#pragma unroll
          for (int q = 0; q < QG; ++q) {
            const float ps = pt[q] * szv.x;
            z[q] = fmaf(pt[q], szv.y, z[q]);
#pragma unroll
            for (int e = 0; e < 16; ++e) o[q][e] = fmaf(ps, f[e], o[q][e]);
          }
        }
      }
    }
    __syncthreads();
    if (tid == 0 && t + kStages < ntiles) issue(t + kStages);
  }
}

// Combines the four warps' states and writes either the final output (and lse) or
// a split partial; the last split of a head then merges all partials.
// dim_of(c) maps this lane's element slot to a head dimension.
template <typename T, int D, int QG, int EPL, typename DimOf>
__device__ __forceinline__ void finish(const DecodeParams &p, float (&m)[QG], float (&l)[QG], float (&o)[QG][EPL],
                                       float (&z)[QG], DimOf dim_of, const CtaSmem &sm, int b, int h0,
                                       bool split_mode, int split, int64_t part_head) {
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, g = lane >> 3;
#pragma unroll
  for (int q = 0; q < QG; ++q) {
    l[q] = warp_sum(l[q]);
    z[q] += __shfl_xor_sync(kFull, z[q], 8);
    z[q] += __shfl_xor_sync(kFull, z[q], 16);
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      o[q][e] += __shfl_xor_sync(kFull, o[q][e], 8);
      o[q][e] += __shfl_xor_sync(kFull, o[q][e], 16);
    }
  }
  float *red = sm.red;  // [kWarps][QG][D+2] : m, l, o[D]
  if (g == 0) {
#pragma unroll
    for (int q = 0; q < QG; ++q) {
      float *r = red + (w * QG + q) * (D + 2);
      if (lane == 0) {
        r[0] = m[q];
        r[1] = l[q];
      }
#pragma unroll
      for (int e = 0; e < EPL; ++e) r[2 + dim_of(e)] = o[q][e] + z[q];
    }
  }
  __syncthreads();
  float *part = p.partials + part_head * p.max_splits * QG * (D + 2);
  for (int idx = tid; idx < QG * D; idx += kThreads) {
    const int q = idx / D, d = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int ww = 0; ww < kWarps; ++ww) M = fmaxf(M, red[(ww * QG + q) * (D + 2)]);
    float num = 0.f, den = 0.f;
#pragma unroll
    for (int ww = 0; ww < kWarps; ++ww) {
      const float *r = red + (ww * QG + q) * (D + 2);
      const float wt = (r[0] == -INFINITY) ? 0.f : ex2(r[0] - M);
      num = fmaf(wt, r[2 + d], num);
      den = fmaf(wt, r[1], den);
    }
    if (!split_mode) {
      Elem<T>::store(p.out, (static_cast<int64_t>(b) * p.Hq + h0 + q) * D + d, num / den);
      if (d == 0 && p.lse) p.lse[b * p.Hq + h0 + q] = (M + lg2(den)) * kLn2;
    } else {
      float *dst = part + (static_cast<int64_t>(split) * QG + q) * (D + 2);
      dst[2 + d] = num;
      if (d == 0) {
        dst[0] = M;
        dst[1] = den;
      }
    }
  }
  if (!split_mode) return;

  // ---- ticket: the last split of this head merges ----
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const uint32_t prev = atomicAdd(p.counters + part_head, 1u);
    *sm.flag = (prev == static_cast<uint32_t>(p.nsplit - 1)) ? 1 : 0;
  }
  __syncthreads();
  if (!*sm.flag) return;
  __threadfence();
  // per query head: global max, denominator, and normalised split weights
  if (w < QG) {
    const int q = w;
    float M = -INFINITY;
    for (int sp = lane; sp < p.nsplit; sp += 32) M = fmaxf(M, __ldcg(part + (static_cast<int64_t>(sp) * QG + q) * (D + 2)));
    M = warp_max(M);
    float den = 0.f;
    for (int sp = lane; sp < p.nsplit; sp += 32) {
      const float *r = part + (static_cast<int64_t>(sp) * QG + q) * (D + 2);
      const float ms = __ldcg(r);
      const float e = (ms == -INFINITY) ? 0.f : ex2(ms - M);
      sm.wts[q * kMaxSplits + sp] = e;
      den = fmaf(e, __ldcg(r + 1), den);
    }
    den = warp_sum(den);
    const float inv = 1.f / den;
    for (int sp = lane; sp < p.nsplit; sp += 32) sm.wts[q * kMaxSplits + sp] *= inv;
    if (lane == 0 && p.lse) p.lse[b * p.Hq + h0 + q] = (M + lg2(den)) * kLn2;
  }
  __syncthreads();
  for (int idx = tid; idx < QG * D; idx += kThreads) {
    const int q = idx / D, d = idx % D;
    float acc = 0.f;
    for (int sp = 0; sp < p.nsplit; ++sp)
      acc = fmaf(sm.wts[q * kMaxSplits + sp], __ldcg(part + (static_cast<int64_t>(sp) * QG + q) * (D + 2) + 2 + d), acc);
    Elem<T>::store(p.out, (static_cast<int64_t>(b) * p.Hq + h0 + q) * D + d, acc);
  }
  if (tid == 0) p.counters[part_head] = 0u;  // ready for the next call
}

template <typename T, int D, int QG>
__device__ __forceinline__ void load_q(const DecodeParams &p, int b, int h0, float (&qf)[QG][D / 8]) {
  using C = RowCfg<T, D>;
  const int j = threadIdx.x & 7;
#pragma unroll
  for (int q = 0; q < QG; ++q) {
    const char *qrow = p.q + ((static_cast<int64_t>(b) * p.Hq + h0 + q) * D) * static_cast<int>(sizeof(T));
#pragma unroll
    for (int c = 0; c < C::CPL; ++c) {
      const uint4 u = __ldg(reinterpret_cast<const uint4 *>(qrow + (j + 8 * c) * 16));
      float f[C::PER16];
      Elem<T>::unpack(u, f);
#pragma unroll
      for (int e = 0; e < C::PER16; ++e) qf[q][c * C::PER16 + e] = f[e] * p.scale_log2;
    }
  }
}

template <typename T, int D, int QG, bool INT4>
__global__ void __launch_bounds__(kThreads, 2) decode_kernel(const DecodeParams p) {
  using C = RowCfg<T, D>;
  extern __shared__ __align__(1024) char smem[];
  constexpr int STAGE = (INT4 && I4Cfg::STAGE > C::STAGE) ? I4Cfg::STAGE : C::STAGE;
  // stages; after the main loop the stage area is reused for the cross-warp and
  // cross-split reductions (every bulk copy has completed by then)
  CtaSmem sm;
  sm.stages = smem;
  sm.red = reinterpret_cast<float *>(smem);
  sm.wts = sm.red + kWarps * QG * (D + 2);
  sm.bar0 = smem_u32(smem + kStages * STAGE);
  sm.flag = reinterpret_cast<int *>(smem + kStages * STAGE + 8 * kStages);
  static_assert((kWarps * QG * (D + 2) + QG * kMaxSplits) * 4 <= kStages * STAGE, "reduction scratch");
  const int tid = threadIdx.x, j = tid & 7;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(sm.bar0 + 8 * s, 1);
    fence_mbar_init();
  }
  __syncthreads();

  float m[QG], l[QG], z[QG];
  float o[QG][D / 8];
#pragma unroll
  for (int q = 0; q < QG; ++q) {
    m[q] = -INFINITY;
    l[q] = 0.f;
    z[q] = 0.f;
#pragma unroll
    for (int e = 0; e < D / 8; ++e) o[q][e] = 0.f;
  }

  const int bid = blockIdx.x;
  if (bid < p.n_retr_ctas) {
    const int split = bid % p.nsplit;
    int rest = bid / p.nsplit;
    const int qgi = rest % p.nqg;
    rest /= p.nqg;
    const int ri = rest % p.Hr;
    const int b = rest / p.Hr;
    const int g = p.hm.retr_head[ri];
    const int h0 = g * p.G + qgi * QG;
    const int64_t t0 = static_cast<int64_t>(split) * p.split_len;
    const int64_t t1 = (t0 + p.split_len < p.len) ? t0 + p.split_len : p.len;
    const int64_t head_row = (static_cast<int64_t>(b) * p.Hr + ri) * p.max_len;
    const int64_t part_head = (static_cast<int64_t>(b) * p.Hr + ri) * p.nqg + qgi;
    const bool split_mode = p.nsplit > 1;
    if constexpr (INT4) {
      // lane j holds dims 16j .. 16j+15
      float qf[QG][16], qsum[QG];
#pragma unroll
      for (int q = 0; q < QG; ++q) {
        const uint4 *qrow = reinterpret_cast<const uint4 *>(p.q + ((static_cast<int64_t>(b) * p.Hq + h0 + q) * D) * 2);
        const uint4 u0 = __ldg(qrow + 2 * j), u1 = __ldg(qrow + 2 * j + 1);
        float f[8];
        Elem<__nv_bfloat16>::unpack(u0, f);
        for (int e = 0; e < 8; ++e) qf[q][e] = f[e] * p.scale_log2;
        Elem<__nv_bfloat16>::unpack(u1, f);
        for (int e = 0; e < 8; ++e) qf[q][8 + e] = f[e] * p.scale_log2;
        float s = 0.f;
        for (int e = 0; e < 16; ++e) s += qf[q][e];
        s += __shfl_xor_sync(kFull, s, 1);
        s += __shfl_xor_sync(kFull, s, 2);
        s += __shfl_xor_sync(kFull, s, 4);
        qsum[q] = s;
      }
      float o16[QG][16];
#pragma unroll
      for (int q = 0; q < QG; ++q)
#pragma unroll
        for (int e = 0; e < 16; ++e) o16[q][e] = 0.f;
      run_rows_int4<QG>(reinterpret_cast<const uint8_t *>(p.rk) + (head_row + t0) * I4Cfg::CB,
                        reinterpret_cast<const uint8_t *>(p.rv) + (head_row + t0) * I4Cfg::CB,
                        reinterpret_cast<const __half *>(p.rk_sz) + (head_row + t0) * 2,
                        reinterpret_cast<const __half *>(p.rv_sz) + (head_row + t0) * 2, t1 - t0, qf, qsum, m, l,
                        o16, z, sm, p.status);
      finish<T, D, QG, 16>(p, m, l, o16, z, [j](int e) { return 16 * j + e; }, sm, b, h0, split_mode, split,
                           part_head);
    } else {
      float qf[QG][D / 8];
      load_q<T, D, QG>(p, b, h0, qf);
      const int RB = C::RB;
      run_rows<T, D, QG>(p.rk + (head_row + t0) * RB, p.rv + (head_row + t0) * RB, t1 - t0,
                         [](int64_t) { return true; }, qf, m, l, o, z, sm, p.status);
      finish<T, D, QG, D / 8>(p, m, l, o, z, [j](int e) { return (j + 8 * (e / C::PER16)) * C::PER16 + e % C::PER16; },
                              sm, b, h0, split_mode, split, part_head);
    }
  } else {
    // streaming head: slots 0..S+W-1 (sinks, then the ring)
    int rest = bid - p.n_retr_ctas;
    const int qgi = rest % p.nqg;
    rest /= p.nqg;
    const int si = rest % p.Hs;
    const int b = rest / p.Hs;
    const int g = p.hm.strm_head[si];
    const int h0 = g * p.G + qgi * QG;
    const int S = p.S, W = p.W;
    const int64_t len = p.len;
    const int64_t nslots = S + W;
    // ring positions held: [max(S, len-W), len); count c <= W
    const int64_t rstart = (len - W > S) ? len - W : S;
    const int64_t rcount = len > rstart ? len - rstart : 0;
    const int64_t rphase = S % W;  // residue of position S
    auto valid = [=](int64_t slot) {
      if (slot < S) return slot < len;
      if (rcount >= W) return true;
      const int64_t off = slot - S;  // residue held by this ring slot
      return ((off - rphase) % W + W) % W < rcount;
    };
    const int64_t row0 = (static_cast<int64_t>(b) * p.Hs + si) * nslots;
    using TS = T;
    float qf[QG][D / 8];
    load_q<TS, D, QG>(p, b, h0, qf);
    const int RB = D * static_cast<int>(sizeof(TS));
    run_rows<TS, D, QG>(p.sk + row0 * RB, p.sv + row0 * RB, nslots, valid, qf, m, l, o, z, sm, p.status);
    finish<TS, D, QG, D / 8>(p, m, l, o, z,
                             [j](int e) { return (j + 8 * (e / RowCfg<TS, D>::PER16)) * RowCfg<TS, D>::PER16 + e % RowCfg<TS, D>::PER16; },
                             sm, b, h0, false, 0, 0);
  }
}

template <typename T, int D, int QG, bool INT4>
cudaError_t launch_t(const DecodeParams &p, cudaStream_t st) {
  using C = RowCfg<T, D>;
  constexpr int STAGE = (INT4 && I4Cfg::STAGE > C::STAGE) ? I4Cfg::STAGE : C::STAGE;
  constexpr int smem = kStages * STAGE + 8 * kStages + 16;
  static std::atomic<uint64_t> attr{0};
  const cudaError_t e = opt_in_smem(decode_kernel<T, D, QG, INT4>, smem, attr);
  if (e != cudaSuccess) return e;
  const int grid = p.n_retr_ctas + p.B * p.Hs * p.nqg;
  decode_kernel<T, D, QG, INT4><<<grid, kThreads, smem, st>>>(p);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_qg(const DecodeParams &p, bool int4, cudaStream_t st) {
  if constexpr (std::is_same<T, __nv_bfloat16>::value && D == 128) {
    if (int4) {
      switch (p.qg) {
        case 1: return launch_t<T, D, 1, true>(p, st);
        case 2: return launch_t<T, D, 2, true>(p, st);
        case 4: return launch_t<T, D, 4, true>(p, st);
      }
      return cudaErrorInvalidValue;
    }
  }
  if (int4) return cudaErrorNotSupported;
  switch (p.qg) {
    case 1: return launch_t<T, D, 1, false>(p, st);
    case 2: return launch_t<T, D, 2, false>(p, st);
    case 4: return launch_t<T, D, 4, false>(p, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

int decode_tokens_per_stage(duo_dtype dt, int D, bool int4) {
  if (int4) return I4Cfg::TPS;
  return 16384 / (D * (dt == DUO_BF16 ? 2 : 4));
}

cudaError_t launch_decode(const DecodeParams &p, duo_dtype dt, bool int4, cudaStream_t st) {
  if (dt == DUO_BF16) {
    if (p.D == 128) return launch_qg<__nv_bfloat16, 128>(p, int4, st);
    if (p.D == 64) return launch_qg<__nv_bfloat16, 64>(p, int4, st);
  } else {
    if (p.D == 128) return launch_qg<float, 128>(p, int4, st);
    if (p.D == 64) return launch_qg<float, 64>(p, int4, st);
  }
  return cudaErrorNotSupported;
}

}  // namespace duo
