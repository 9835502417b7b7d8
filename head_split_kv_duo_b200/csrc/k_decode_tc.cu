// k_decode_tc.cu -- single-token decode attention on the tcgen05 tensor cores
// (bf16, head_dim 128, up to 16 query heads per KV head).
//
// Operation ("Decoding Procedure", steps 2, 3 and 5): the newest query (position
// len-1) of every query head attends to all cached tokens of its retrieval KV head,
// or to the valid sink and ring slots of its streaming KV head.
//
// Tokens sit on the M side of the MMA, so a GQA group of G query heads costs one
// N = 16 column block instead of G passes over the cache:
//   S^T (128 tokens x 16)  = K_tile (128 x d)   . Qpad^T (d x 16)      A K-major, B K-major
//   O^T (d 128 x 16)       = V_tile^T (d x 128) . P^T (128 tokens x 16) A MN-major, B K-major
// Each K/V tile (128 rows, 64 KiB) and the group's queries (16 rows, 4 KiB) arrive by
// TMA (128-byte swizzle) into a 3-stage ring.  Thread t of the softmax warpgroup owns
// token t of S^T (TMEM lane t) and dimension t of O^T.
//
// Work balance: every (batch, KV head) is an item of 128-token units (retrieval:
// ceil(len/128), streaming: ceil((S+W)/128)); the units of all items are laid end to
// end and cut into one equal range per CTA (one CTA per SM).  A CTA flushes a partial
// (max, sum, unnormalised output) whenever an item ends inside its range; the last CTA
// of an item to flush (a ticket per item) merges the item's partials.  Items held by a
// single CTA are written directly.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "device_common.cuh"

namespace duo {

namespace {

constexpr int kThreads = 192;  // warp 0 TMA, warp 1 MMA + TMEM, warps 2-5 softmax
constexpr int kTile = 128;
constexpr int kD = 128;
constexpr int kN = 16;         // padded query heads per item
constexpr int kStages = 3;
// Each contraction (over d for S^T, over tokens for O^T) is split into kAcc partial
// accumulators in separate TMEM columns, so the tensor core runs kAcc independent
// chains of 8 / kAcc MMAs instead of one chain of 8; the softmax warps add them up.
constexpr int kAcc = 4;
constexpr int kTmO = 2 * kAcc * 16;         // TMEM column of the O^T double buffer
constexpr int kTmemCols = 4 * kAcc * 16;    // S^T x 2 and O^T x 2, kAcc blocks of 16 each
// shared memory map per stage: K [128][128] (2 swizzle atoms of 16 KiB), V likewise, Q [16][128]
constexpr int kStK = 0, kStV = 32768, kStQ = 65536, kStage = 65536 + 4096;
constexpr int kSmP = kStages * kStage;     // 2 x P^T [16][128] bf16 (2 atoms of 2 KiB each)
constexpr int kSmRed = kSmP + 8192;        // cross-warp reductions [4][16] + merge exchange [128][6]
constexpr int kSmBar = kSmRed + (4 * 16 + 128 * 6) * 4;
constexpr int kSmMisc = kSmBar + 256;
constexpr int kSmemAlloc = kSmMisc + 64 + 1024;
// Double-buffered resources (S, P, O) each have one barrier per buffer, so that no
// barrier can complete two phases ahead of the thread waiting on it (parity waits).
constexpr int kBarFull = 0, kBarEmpty = 3, kBarSFull = 6, kBarSFree = 8, kBarPFull = 10, kBarOFull = 12,
              kBarDrain = 14, kNumBars = 15;

struct TcDecodeArgs {
  DecodeParams p;
  int units_r, units_s;    // units per retrieval / streaming item
  int n_items_r;           // B * Hr
  int64_t total_units;
  int num_ctas;
  CUtensorMap tm_q, tm_kr, tm_vr, tm_ks, tm_vs;
};

__device__ __forceinline__ void tma_2d(uint32_t dst, const CUtensorMap *m, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tma_3d(uint32_t dst, const CUtensorMap *m, int x, int y, int z, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(acc)
      : "memory");
}
// 16 consecutive fp32 columns of this thread's TMEM lane
__device__ __forceinline__ void tc_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
// N (1, 2, 4, 8 or 16) consecutive fp32 columns of this thread's TMEM lane
template <int N>
__device__ __forceinline__ void tc_ld(uint32_t taddr, float (&v)[N]) {
  if constexpr (N == 16) {
    tc_ld16(taddr, v);
  } else {
    uint32_t r[8];
    if constexpr (N == 1)
      asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r[0]) : "r"(taddr));
    else if constexpr (N == 2)
      asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0, %1}, [%2];" : "=r"(r[0]), "=r"(r[1]) : "r"(taddr));
    else if constexpr (N == 4)
      asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                   : "r"(taddr));
    else
      asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                   : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                   : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < N; ++i) v[i] = __uint_as_float(r[i]);
  }
}
// Sum of kAcc partial accumulators, 16 columns apart
template <int N>
__device__ __forceinline__ void tc_ld_sum(uint32_t taddr, float (&v)[N]) {
  tc_ld<N>(taddr, v);
#pragma unroll
  for (int a = 1; a < kAcc; ++a) {
    float w[N];
    tc_ld<N>(taddr + a * 16, w);
#pragma unroll
    for (int q = 0; q < N; ++q) v[q] += w[q];
  }
}
// OR of `v` over the threads of named barrier `id` (all `n` threads receive it)
__device__ __forceinline__ int bar_or(int id, int n, int v) {
  int r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.or.pred po, %2, %3, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"(v), "r"(id), "r"(n)
      : "memory");
  return r;
}
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// kind::f16, fp32 accumulator, bf16 operands, M 128, N 16
constexpr uint32_t idesc_m128n16(bool a_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) | ((16u >> 3) << 17) | ((128u >> 4) << 24);
}
__device__ __forceinline__ void named_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, uint32_t *status, volatile int *abort_flag) {
#pragma unroll 1
  for (int i = 0; i < 64; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
#pragma unroll 1
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer() - t0 > kWaitLimitNs) {
      flag_status(status, kDevTimeout);
      *abort_flag = 1;
      return false;
    }
  }
}

// unit u -> (item, tile within item)
struct Unit {
  int item, tile;
  bool retr;
};
__device__ __forceinline__ Unit unit_of(const TcDecodeArgs &a, int64_t u) {
  const int64_t ur = static_cast<int64_t>(a.n_items_r) * a.units_r;
  if (u < ur) return {static_cast<int>(u / a.units_r), static_cast<int>(u % a.units_r), true};
  const int64_t us = u - ur;
  return {a.n_items_r + static_cast<int>(us / a.units_s), static_cast<int>(us % a.units_s), false};
}
// first unit of CTA c: floor(c * U / C); the CTA holding unit u: ceil((u+1) C / U) - 1
__device__ __forceinline__ int64_t cta_begin(const TcDecodeArgs &a, int c) {
  return static_cast<int64_t>(c) * a.total_units / a.num_ctas;
}
__device__ __forceinline__ int cta_of(const TcDecodeArgs &a, int64_t u) {
  return static_cast<int>(((u + 1) * a.num_ctas + a.total_units - 1) / a.total_units) - 1;
}

template <int NQ>
__global__ void __launch_bounds__(kThreads, 1) decode_tc_kernel(const __grid_constant__ TcDecodeArgs a) {
  const DecodeParams &p = a.p;
  extern __shared__ char smem_raw[];
  char *smem = reinterpret_cast<char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) { return sbase + kSmBar + 8u * i; };
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kSmMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kSmMisc + 4);
  volatile int *last_flag = reinterpret_cast<volatile int *>(smem + kSmMisc + 8);
  float *red = reinterpret_cast<float *>(smem + kSmRed);  // [4 warps][16]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t u0 = cta_begin(a, blockIdx.x), u1 = cta_begin(a, blockIdx.x + 1);
  const int nu = static_cast<int>(u1 - u0);
  const int G = p.G;

  if (tid == 0) {
    for (int i = 0; i < kNumBars; ++i)
      mbar_init(bar(i), (i == kBarSFree || i == kBarSFree + 1 || i == kBarPFull || i == kBarPFull + 1) ? 128 : 1);
    fence_mbar_init();
    *abort_flag = 0;
  }
  // P^T rows >= G stay zero for the whole kernel
  for (int i = tid; i < 8192 / 16; i += kThreads) reinterpret_cast<uint4 *>(smem + kSmP)[i] = make_uint4(0, 0, 0, 0);
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ================= TMA producer =================
    if (lane == 0) {
      // Launched as a programmatic dependent, this grid's set-up overlaps the previous
      // kernel on the stream; nothing is read from global memory before that kernel has
      // finished (every other read and every write of this grid follows these loads).
      asm volatile("griddepcontrol.wait;" ::: "memory");
      for (int j = 0; j < nu; ++j) {
        const int s = j % kStages;
        if (j >= kStages && !wait_bar(bar(kBarEmpty + s), ((j / kStages) - 1) & 1, p.status, abort_flag)) break;
        const Unit un = unit_of(a, u0 + j);
        const uint32_t dst = sbase + s * kStage;
        const uint32_t fb = bar(kBarFull + s);
        mbar_expect_tx(fb, 65536 + 4096);
        int b, g, z;
        const CUtensorMap *mk, *mv;
        if (un.retr) {
          b = un.item / p.Hr;
          const int ri = un.item % p.Hr;
          g = p.hm.retr_head[ri];
          z = b * p.Hr + ri;
          mk = &a.tm_kr;
          mv = &a.tm_vr;
        } else {
          const int it = un.item - a.n_items_r;
          b = it / p.Hs;
          const int si = it % p.Hs;
          g = p.hm.strm_head[si];
          z = b * p.Hs + si;
          mk = &a.tm_ks;
          mv = &a.tm_vs;
        }
        const int y = un.tile * kTile;
        tma_3d(dst + kStK, mk, 0, y, z, fb);
        tma_3d(dst + kStK + 16384, mk, 64, y, z, fb);
        tma_3d(dst + kStV, mv, 0, y, z, fb);
        tma_3d(dst + kStV + 16384, mv, 64, y, z, fb);
        const int qrow = b * p.Hq + g * G;  // rows beyond this group's G heads are never used
        tma_2d(dst + kStQ, &a.tm_q, 0, qrow, fb);
        tma_2d(dst + kStQ + 2048, &a.tm_q, 64, qrow, fb);
      }
    }
  } else if (warp == 1) {
    // ================= MMA issuer =================
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_m128n16(false);
      constexpr uint32_t kIdO = idesc_m128n16(true);
      bool ok = true;
      auto issue_o = [&](int jj) {
        const int s = jj % kStages;
        const uint32_t vb = sbase + s * kStage + kStV;
        const uint32_t pb = sbase + kSmP + (jj & 1) * 4096;
        for (int i = 0; i < 8; ++i) {  // K = 128 tokens in steps of 16, kAcc independent chains
          const int kk = (i % kAcc) * (8 / kAcc) + i / kAcc;
          const uint64_t ad = sdesc(vb + kk * 2048, 16384, 1024);                    // V^T, MN-major
          const uint64_t bd = sdesc(pb + (kk >> 2) * 2048 + (kk & 3) * 32, 16, 1024);  // P^T, K-major
          tc_mma(tmem + kTmO + (jj & 1) * kAcc * 16 + (i % kAcc) * 16, ad, bd, kIdO, i >= kAcc ? 1u : 0u);
        }
        tc_commit(bar(kBarOFull + (jj & 1)));
        tc_commit(bar(kBarEmpty + s));
      };
      for (int j = 0; j < nu && ok; ++j) {
        const int s = j % kStages;
        if (!wait_bar(bar(kBarFull + s), (j / kStages) & 1, p.status, abort_flag)) { ok = false; break; }
        if (j >= 2 && !wait_bar(bar(kBarSFree + (j & 1)), ((j - 2) >> 1) & 1, p.status, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t st = sbase + s * kStage;
        for (int i = 0; i < 8; ++i) {  // K = d 128 in steps of 16, kAcc independent chains
          const int kk = (i % kAcc) * (8 / kAcc) + i / kAcc;
          const uint64_t ad = sdesc(st + kStK + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);  // K tile, K-major
          const uint64_t bd = sdesc(st + kStQ + (kk >> 2) * 2048 + (kk & 3) * 32, 16, 1024);   // Qpad, K-major
          tc_mma(tmem + (j & 1) * kAcc * 16 + (i % kAcc) * 16, ad, bd, kIdS, i >= kAcc ? 1u : 0u);
        }
        tc_commit(bar(kBarSFull + (j & 1)));
        if (j >= 1) {
          if (!wait_bar(bar(kBarPFull + ((j - 1) & 1)), ((j - 1) >> 1) & 1, p.status, abort_flag)) { ok = false; break; }
          tc_fence_after();
          issue_o(j - 1);
        }
      }
      if (ok && nu > 0 && wait_bar(bar(kBarPFull + ((nu - 1) & 1)), ((nu - 1) >> 1) & 1, p.status, abort_flag)) {
        tc_fence_after();
        issue_o(nu - 1);
      }
      tc_commit(bar(kBarDrain));
      mbar_wait(bar(kBarDrain), 0, p.status);
    }
  } else {
    // ================= softmax warpgroup =================
    // Thread t owns token t of each S^T tile and dimension t of each O^T tile.  The
    // running max m[q] is a reference: a tile's probabilities are exp2(s*c - m[q]);
    // m is raised (and everything before rescaled) only when some logit of the tile
    // exceeds it by more than kSlack, decided by one barrier-reduction vote.
    constexpr float kSlack = 8.0f;
    const int t = ((warp & 3) << 5) | lane;
    const int wq = warp & 3;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq << 5) << 16);
    const float c = p.scale_log2;
    float m[NQ], l[NQ], o[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      m[q] = -INFINITY;
      l[q] = 0.f;
      o[q] = 0.f;
    }
    bool ok = true;
    int cur_item = -1;

    // Merges the nseg partial rows of one item (run by the item's last CTA).  A row is one
    // float4 column c of query head c / 32's output; with fewer than 128 columns the
    // threads split the segments into nsl interleaved lanes, combined through shared
    // memory at the end.  Loads are issued in batches of 8 segments, so the merge costs
    // about ceil(nseg / (8 nsl)) round trips to L2.
    auto merge = [&](const float *part, int nseg, int b, int h0) {
      constexpr int kRow = kD + 4;
      constexpr int kBatch = 8;
      const int cols = G * (kD / 4);
      const int nsl = cols >= 128 ? 1 : 128 / cols;
      float *cmb = red + 4 * kN;  // [128][6]: M, den, acc
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
                const float *row = part + (static_cast<int64_t>(sg) * G + q) * kRow;
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
          named_sync(1, 128);
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
          *reinterpret_cast<uint2 *>(p.out + ((static_cast<int64_t>(b) * p.Hq + h) * kD + 4 * c4) * 2) = pk;
          if (c4 == 0 && p.lse) p.lse[b * p.Hq + h] = (M + lg2(den)) * kLn2;
        }
      }
      named_sync(1, 128);  // cmb and red are reused by the next flush
    };

    // Writes this CTA's result for `item` (partial or final) and merges when last.
    auto flush = [&](int item) {
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        const float v = warp_sum(l[q]);
        if (lane == 0) red[wq * kN + q] = v;
      }
      named_sync(1, 128);
      float lt[NQ];
#pragma unroll
      for (int q = 0; q < NQ; ++q) lt[q] = red[q] + red[kN + q] + red[2 * kN + q] + red[3 * kN + q];
      named_sync(1, 128);
      const bool retr = item < a.n_items_r;
      const int units = retr ? a.units_r : a.units_s;
      const int64_t ia = retr ? static_cast<int64_t>(item) * a.units_r
                              : static_cast<int64_t>(a.n_items_r) * a.units_r +
                                    static_cast<int64_t>(item - a.n_items_r) * a.units_s;
      const int cfirst = cta_of(a, ia), clast = cta_of(a, ia + units - 1);
      const int nseg = clast - cfirst + 1;
      int b, g;
      if (retr) {
        b = item / p.Hr;
        g = p.hm.retr_head[item % p.Hr];
      } else {
        const int it = item - a.n_items_r;
        b = it / p.Hs;
        g = p.hm.strm_head[it % p.Hs];
      }
      const int h0 = g * G;
      if (nseg == 1) {
#pragma unroll
        for (int q = 0; q < NQ; ++q)
          if (q < G) {
            Elem<__nv_bfloat16>::store(p.out, (static_cast<int64_t>(b) * p.Hq + h0 + q) * kD + t, o[q] / lt[q]);
            if (t == 0 && p.lse) p.lse[b * p.Hq + h0 + q] = (m[q] + lg2(lt[q])) * kLn2;
          }
        return;
      }
      const int seg = blockIdx.x - cfirst;
      const int64_t pitem = static_cast<int64_t>(b) * p.Hkv + g;
      // partial row of (segment, query head): o[0..d), m at d, l at d+1 (16-byte aligned rows)
      constexpr int kRow = kD + 4;
      float *part = p.partials + (pitem * p.max_splits) * G * kRow;
#pragma unroll
      for (int q = 0; q < NQ; ++q)
        if (q < G) {
          float *dst = part + (static_cast<int64_t>(seg) * G + q) * kRow;
          dst[t] = o[q];
          if (t == 0) {
            dst[kD] = m[q];
            dst[kD + 1] = lt[q];
          }
        }
      __threadfence();
      named_sync(1, 128);
      if (t == 0) {
        const uint32_t prev = atomicAdd(p.counters + pitem, 1u);
        *last_flag = (prev == static_cast<uint32_t>(nseg - 1)) ? 1 : 0;
      }
      named_sync(1, 128);
      if (!*last_flag) return;
      __threadfence();
      merge(part, nseg, b, h0);
      if (t == 0) p.counters[pitem] = 0u;  // ready for the next call
    };

    // o = (o + O^T(jj)) * alpha for this thread's dimension t
    auto fold = [&](int jj, const float (&alpha)[NQ]) {
      if (ok) ok = wait_bar(bar(kBarOFull + (jj & 1)), (jj >> 1) & 1, p.status, abort_flag);
      tc_fence_after();
      float v[NQ];
      tc_ld_sum<NQ>(lane_base + kTmO + (jj & 1) * kAcc * 16, v);
#pragma unroll
      for (int q = 0; q < NQ; ++q) o[q] = (o[q] + v[q]) * alpha[q];
    };
    float one[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q) one[q] = 1.f;

    bool pending = false;  // O^T of the previous unit still to be folded
    for (int j = 0; j < nu; ++j) {
      const Unit un = unit_of(a, u0 + j);
      if (ok) ok = wait_bar(bar(kBarSFull + (j & 1)), (j >> 1) & 1, p.status, abort_flag);
      tc_fence_after();
      float sv[NQ];
      tc_ld_sum<NQ>(lane_base + (j & 1) * kAcc * 16, sv);
      tc_fence_before();
      mbar_arrive(bar(kBarSFree + (j & 1)));  // S buffer j % 2 is free again
      // this token's validity
      bool valid;
      const int64_t tok = static_cast<int64_t>(un.tile) * kTile + t;
      if (un.retr) {
        valid = tok < p.len;
      } else {
        const int S = p.S, W = p.W;
        const int64_t len = p.len;
        const int64_t rstart = (len - W > S) ? len - W : S;
        const int64_t rcount = len > rstart ? len - rstart : 0;
        if (tok >= S + W) valid = false;
        else if (tok < S) valid = tok < len;
        else if (rcount >= W) valid = true;
        else valid = (((tok - S) - (S % W)) % W + W) % W < rcount;
      }
      if (un.item != cur_item) {
        if (cur_item >= 0) {
          if (pending) fold(j - 1, one);
          flush(cur_item);
        }
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          m[q] = -INFINITY;
          l[q] = 0.f;
          o[q] = 0.f;
        }
        pending = false;
        cur_item = un.item;
      }
      // does any logit of this tile exceed the reference max by more than kSlack?
      int need = 0;
#pragma unroll
      for (int q = 0; q < NQ; ++q)
        if (q < G && valid && sv[q] * c > m[q] + kSlack) need = 1;
      need = bar_or(1, 128, need);
      float alpha[NQ];
#pragma unroll
      for (int q = 0; q < NQ; ++q) alpha[q] = 1.f;
      if (need) {  // uniform over the warpgroup
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          const float x = warp_max((valid && q < G) ? sv[q] : -INFINITY);
          if (lane == 0) red[wq * kN + q] = x;
        }
        named_sync(1, 128);
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          const float mt = fmaxf(fmaxf(red[q], red[kN + q]), fmaxf(red[2 * kN + q], red[3 * kN + q])) * c;
          const float mn = fmaxf(m[q], mt);
          alpha[q] = (mn == -INFINITY) ? 1.f : ex2(m[q] - mn);
          m[q] = mn;
        }
        named_sync(1, 128);  // red is reused later
      }
      uint16_t pb[NQ];
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        const float pv = (valid && q < G && m[q] != -INFINITY) ? ex2(fmaf(sv[q], c, -m[q])) : 0.f;
        l[q] = fmaf(l[q], alpha[q], pv);
        const __nv_bfloat16 hb = __float2bfloat16_rn(pv);
        pb[q] = *reinterpret_cast<const uint16_t *>(&hb);
      }
      // P^T[q][t] into buffer j % 2 (its previous reader, unit j-2, was folded at j-1)
      {
        const int atom = t >> 6, col = t & 63;
        char *pbase = smem + kSmP + (j & 1) * 4096 + atom * 2048;
#pragma unroll
        for (int q = 0; q < NQ; ++q)
          if (q < G) {
            const int chunk = (col >> 3) ^ (q & 7);
            *reinterpret_cast<uint16_t *>(pbase + q * 128 + chunk * 16 + (col & 7) * 2) = pb[q];
          }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tc_fence_before();
      mbar_arrive(bar(kBarPFull + (j & 1)));
      // fold the previous unit of the same item, bringing it to this unit's scale
      if (pending) {
        fold(j - 1, alpha);
      } else {
#pragma unroll
        for (int q = 0; q < NQ; ++q) o[q] *= alpha[q];
      }
      pending = true;
    }
    if (nu > 0) {
      if (pending) fold(nu - 1, one);
      flush(cur_item);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

bool map_bf16(CUtensorMap *m, const void *base, int rank, const uint64_t *dims, const uint64_t *strides,
              const uint32_t *box) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gd[3], gs[2];
  cuuint32_t bx[3], es[3] = {1, 1, 1};
  for (int r = 0; r < rank; ++r) {
    gd[r] = dims[r];
    bx[r] = box[r];
  }
  for (int r = 0; r < rank - 1; ++r) gs[r] = strides[r];
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(base), gd, gs, bx, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NQ>
cudaError_t launch_nq(const TcDecodeArgs &a, bool overlap_previous, cudaStream_t st) {
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(decode_tc_kernel<NQ>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.num_ctas);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemAlloc;
  cfg.stream = st;
  cudaLaunchAttribute attrs[1];
  attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[0].val.programmaticStreamSerializationAllowed = overlap_previous ? 1 : 0;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, decode_tc_kernel<NQ>, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

bool decode_tc_supported(const DecodeParams &p, duo_dtype dt, bool int4) {
  return dt == DUO_BF16 && !int4 && p.D == kD && p.G >= 1 && p.G <= kN && encode_fn() != nullptr;
}

cudaError_t launch_decode_tc(const DecodeParams &p, int num_sms, bool overlap_previous, cudaStream_t st) {
  TcDecodeArgs a{};
  a.p = p;
  a.units_r = static_cast<int>((p.len + kTile - 1) / kTile);
  const int64_t slots = static_cast<int64_t>(p.S) + p.W;
  const int64_t used = p.len < slots ? p.len : slots;  // streaming slots that can hold a token
  a.units_s = static_cast<int>((used + kTile - 1) / kTile);
  a.n_items_r = p.B * p.Hr;
  a.total_units = static_cast<int64_t>(a.n_items_r) * a.units_r + static_cast<int64_t>(p.B) * p.Hs * a.units_s;
  // at most one CTA per SM, and never more segments per item than partial slots
  int64_t ctas = num_sms;
  if (ctas > a.total_units) ctas = a.total_units;
  if (ctas > kMaxSplits) ctas = kMaxSplits;
  a.num_ctas = static_cast<int>(ctas);
  const uint64_t row = kD * 2;
  bool ok = true;
  {  // queries [B*Hq][d]
    const uint64_t d[2] = {kD, static_cast<uint64_t>(p.B) * p.Hq};
    const uint64_t s[1] = {row};
    const uint32_t bx[2] = {64, kN};
    ok &= map_bf16(&a.tm_q, p.q, 2, d, s, bx);
  }
  {  // retrieval [B*Hr][cap][d]
    const uint64_t d[3] = {kD, static_cast<uint64_t>(p.max_len), static_cast<uint64_t>(p.B) * (p.Hr > 0 ? p.Hr : 1)};
    const uint64_t s[2] = {row, row * p.max_len};
    const uint32_t bx[3] = {64, kTile, 1};
    ok &= map_bf16(&a.tm_kr, p.rk, 3, d, s, bx);
    ok &= map_bf16(&a.tm_vr, p.rv, 3, d, s, bx);
  }
  {  // streaming [B*Hs][S+W][d]
    const uint64_t d[3] = {kD, static_cast<uint64_t>(slots), static_cast<uint64_t>(p.B) * (p.Hs > 0 ? p.Hs : 1)};
    const uint64_t s[2] = {row, row * slots};
    const uint32_t bx[3] = {64, kTile, 1};
    ok &= map_bf16(&a.tm_ks, p.sk, 3, d, s, bx);
    ok &= map_bf16(&a.tm_vs, p.sv, 3, d, s, bx);
  }
  if (!ok) return cudaErrorInvalidValue;
  if (p.G <= 1) return launch_nq<1>(a, overlap_previous, st);
  if (p.G <= 2) return launch_nq<2>(a, overlap_previous, st);
  if (p.G <= 4) return launch_nq<4>(a, overlap_previous, st);
  if (p.G <= 8) return launch_nq<8>(a, overlap_previous, st);
  return launch_nq<16>(a, overlap_previous, st);
}

}  // namespace duo
