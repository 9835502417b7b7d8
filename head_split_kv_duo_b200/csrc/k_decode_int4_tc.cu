// k_decode_int4_tc.cu -- single-token decode attention when the retrieval heads keep
// K and V as 4-bit codes ("Combination with Quantization", Figure 12: DuoAttention
// with a 4-bit KV cache), on the tcgen05 tensor cores.  bf16 queries, head_dim 128,
// up to 16 query heads per KV head; the streaming heads stay bf16.
//
// Operation ("Decoding Procedure", steps 2, 3 and 5) as in k_decode_tc.cu.  A stored
// element is c s + z (code c in 0..15, per-token fp16 scale s and zero z).  K codes
// become c' = c + 128, exact in bf16 (bit pattern 0x4300 | c); V codes c" = c + 1024,
// exact in fp16 (0x6400 | c).  For token t
//   q . k_t       = s_t (q . c'_t) + (z_t - 128 s_t) sum(q)
//   sum_t p_t v_t = sum_t (p_t s_t) c"_t + sum_t (p_t z_t - 1024 (p_t s_t))
// so both contractions run on the tensor cores (Q . K' in bf16, V" . P' in fp16), and
// the scale and zero enter as a row scale of S^T and one scalar correction per query
// head of O.  The correction uses the fp16-rounded p_t s_t that the MMA consumes, so
// the offset cancels exactly; fp16 keeps that product to 11 bits.  INT4 items keep the
// running max exact (p <= 1), so p_t s_t <= s_t stays in fp16 range.
//
// One 32-bit word of codes holds elements e0..e7 (e0 in the low nibble); the pair
// ((w >> 4i) & 0x000F000F) | 0x43004300 (or 0x64006400) is (c'_i, c'_{4+i}).  An
// expanded row is thus
// stored in the order perm(x) = (x & ~7) | ((x & 7) >> 1) | ((x & 1) << 2): position x
// holds element perm(x).  K rows and the queries are both expanded in that order, which
// leaves q . k unchanged; V rows too, so lane x of O^T holds output element perm(x).
//
// Roles of a CTA (one per SM, 448 threads):
//   warp 0     TMA producer.  INT4 tile: the codes of 128 K rows and 128 V rows (64 B
//              each, 64-byte swizzle), their scale/zero rows (2 x 512 B) and, at the
//              first tile of an item, the group's queries.  bf16 (streaming) tile: four
//              pieces of 32 K and V rows (128-byte swizzle).  Raw ring of kRaw stages.
//   warp 1     MMA issuer and TMEM owner.  S^T = K'_tile . Qpad^T with K' read from
//              tensor memory; O^T = V'^T . P'^T with V' from shared memory.
//   warps 2-5  softmax: thread t owns token t of S^T and position t of O^T.
//   warps 6-13 expansion: a thread expands one half (64 elements) of token t's K row into
//              TMEM lane t and of its V row into the swizzled V tile; warps 6-9 also
//              stage the scale and zero, warp 12 the queries.  Expanded ring of kCvt
//              stages.
//
// Work balance: every (batch, KV head) is an item of 128-token tiles; the tiles of all
// items are laid end to end (retrieval first) and cut into one range per CTA, an INT4
// tile counting 1 and a bf16 tile kWs (about 4x the bytes).  Split partials are merged
// by the last CTA of each item, as in the bf16 kernel.
#include "decode_merge.cuh"
#include "tcgen05.cuh"

namespace duo {

namespace {

constexpr int kThreads = 448;
constexpr int kTile = 128;
constexpr int kD = 128;
constexpr int kN = 16;  // padded query heads per item
constexpr int kAcc = 4;  // independent accumulator chains per contraction (as in the bf16 kernel)
constexpr int kRaw = 4;  // raw stages
constexpr int kCvt = 3;  // expanded stages
constexpr int kWs = 4;   // cost of a bf16 tile in INT4 tiles

// raw stage: INT4 tile -- K codes [128][64 B], V codes, K scale/zero [128][4 B], V
// scale/zero, queries [16][128] bf16 (2 atoms); bf16 piece -- K rows 32 x 256 B as two
// 64-column halves [32][128 B] at 0 / 4096, V halves at 8192 / 12288, queries as above
constexpr int kRawKc = 0, kRawVc = 8192, kRawKsz = 16384, kRawVsz = 16896, kRawQ = 17408, kRawStage = 21504;
// expanded stage: V" [128][128] fp16 (bf16 for streaming tiles; 2 atoms of 16 KiB),
// per-token {s_k, z_k - 128 s_k, s_v, z_v}
constexpr int kCvtV = 0, kCvtMisc = 32768, kCvtStage = 32768 + 2048;
constexpr int kSmRaw = 0;
constexpr int kSmCvt = kSmRaw + kRaw * kRawStage;
constexpr int kSmQ = kSmCvt + kCvt * kCvtStage;  // 2 x expanded queries [16][128] bf16 (one per item parity)
constexpr int kSmP = kSmQ + 2 * 4096;         // 2 x P'^T [16][128] bf16
constexpr int kSmQsum = kSmP + 8192;          // [2][16] fp32 sums of the queries
constexpr int kSmRed = kSmQsum + 128;         // [4][16] l sums, [4][16] correction sums, [128][6] merge
constexpr int kSmBar = kSmRed + (2 * 4 * 16 + 128 * 6) * 4;
constexpr int kSmMisc = kSmBar + 256;
constexpr int kSmemAlloc = kSmMisc + 64 + 1024;
static_assert(kSmCvt % 1024 == 0 && kSmQ % 1024 == 0 && kSmP % 1024 == 0, "swizzle atoms need 1 KiB alignment");
static_assert(kRawStage % 1024 == 0 && kCvtStage % 1024 == 0 && kRawQ % 1024 == 0, "stage alignment");

// tensor memory columns: S^T x 2, O^T x 2 (64 columns each), K' x kCvt (64 each)
constexpr int kTmS = 0, kTmO = 128, kTmK = 256, kTmemCols = 512;
static_assert(kTmK + kCvt * 64 <= kTmemCols, "tensor memory");

constexpr int kBarRawFull = 0, kBarRawEmpty = kRaw, kBarCvtFull = 2 * kRaw, kBarCvtEmpty = 2 * kRaw + kCvt,
              kBarSFull = 2 * kRaw + 2 * kCvt, kBarSFree = kBarSFull + 2, kBarPFull = kBarSFull + 4,
              kBarOFull = kBarSFull + 6, kBarDrain = kBarSFull + 8, kNumBars = kBarSFull + 9;
static_assert(kNumBars * 8 <= 256, "barrier area");

struct Int4DecodeArgs {
  DecodeParams p;
  int units_r, units_s;  // tiles per retrieval / streaming item
  int n_items_r;         // B * Hr
  int64_t ur;            // retrieval tiles in total
  int64_t total_units;   // ur + streaming tiles
  int64_t total_cost;    // ur + kWs * streaming tiles
  int num_ctas;
  CUtensorMap tm_q, tm_kc, tm_vc, tm_ks, tm_vs;
};

struct Unit {
  int item, tile;
  bool retr;
};
__device__ __forceinline__ Unit unit_of(const Int4DecodeArgs &a, int64_t u) {
  if (u < a.ur) return {static_cast<int>(u / a.units_r), static_cast<int>(u % a.units_r), true};
  const int64_t us = u - a.ur;
  return {a.n_items_r + static_cast<int>(us / a.units_s), static_cast<int>(us % a.units_s), false};
}
// Walks a CTA's units in order without a division per step.
struct UnitIter {
  Unit un;
  int units;  // tiles of the current item
  __device__ __forceinline__ UnitIter(const Int4DecodeArgs &a, int64_t u) : un(unit_of(a, u)) {
    units = un.retr ? a.units_r : a.units_s;
  }
  __device__ __forceinline__ void next(const Int4DecodeArgs &a) {
    if (++un.tile == units) {
      ++un.item;
      un.tile = 0;
      un.retr = un.item < a.n_items_r;
      units = un.retr ? a.units_r : a.units_s;
    }
  }
};
__device__ __forceinline__ int64_t start_cost(const Int4DecodeArgs &a, int64_t u) {
  return u < a.ur ? u : a.ur + (u - a.ur) * kWs;
}
// CTA c takes the units whose start cost lies in [floor(c T / C), floor((c+1) T / C))
__device__ __forceinline__ int64_t cta_begin(const Int4DecodeArgs &a, int c) {
  const int64_t x = static_cast<int64_t>(c) * a.total_cost / a.num_ctas;
  return x <= a.ur ? x : a.ur + (x - a.ur + kWs - 1) / kWs;
}
__device__ __forceinline__ int cta_of(const Int4DecodeArgs &a, int64_t u) {
  return static_cast<int>(((start_cost(a, u) + 1) * a.num_ctas + a.total_cost - 1) / a.total_cost) - 1;
}
// A CTA whose cost range falls strictly inside a bf16 tile u holds no unit.  It still
// lies between the CTAs of u's item when tile u+1 belongs to the same item; it then
// counts as one (empty) segment of that item.  Returns that item, or -1.
__device__ __forceinline__ int empty_cta_item(const Int4DecodeArgs &a, int c) {
  const int64_t x = static_cast<int64_t>(c) * a.total_cost / a.num_ctas;
  if (x <= a.ur) return -1;  // every cost below ur starts a tile
  const int64_t u = a.ur + (x - a.ur) / kWs;
  if (u + 1 >= a.total_units) return -1;
  const int item = unit_of(a, u).item;
  return unit_of(a, u + 1).item == item ? item : -1;
}
// (batch, KV head, row of the per-kind arrays) of an item
__device__ __forceinline__ void item_coords(const Int4DecodeArgs &a, int item, int &b, int &g, int &z) {
  const DecodeParams &p = a.p;
  if (item < a.n_items_r) {
    b = item / p.Hr;
    const int ri = item % p.Hr;
    g = p.hm.retr_head[ri];
    z = b * p.Hr + ri;
  } else {
    const int it = item - a.n_items_r;
    b = it / p.Hs;
    const int si = it % p.Hs;
    g = p.hm.strm_head[si];
    z = b * p.Hs + si;
  }
}

__device__ __forceinline__ int perm(int x) { return (x & ~7) | ((x & 7) >> 1) | ((x & 1) << 2); }

// codes e0..e7 of one word -> pairs (c_0, c_4), (c_1, c_5), (c_2, c_6), (c_3, c_7), each code
// OR-ed into the mantissa of kBase: 0x43004300 gives bf16 128 + c, 0x64006400 fp16 1024 + c
template <uint32_t kBase>
__device__ __forceinline__ uint4 expand8(uint32_t w) {
  constexpr uint32_t kM = 0x000F000Fu;
  return make_uint4((w & kM) | kBase, ((w >> 4) & kM) | kBase, ((w >> 8) & kM) | kBase, ((w >> 12) & kM) | kBase);
}
constexpr uint32_t kBf16Base = 0x43004300u;  // K codes: bf16 128 + c
constexpr uint32_t kFp16Base = 0x64006400u;  // V codes: fp16 1024 + c

// One warp copies the 16 query rows of an item from a raw stage to an expanded-query
// buffer (both [16][128] bf16 in two 128-byte-swizzled atoms), reordering each 8-element
// chunk by perm when `permute`, and writes the fp32 sum of every row.
__device__ __forceinline__ void stage_queries(const char *src, char *dst, float *qsum, int lane, bool permute) {
  const int r = lane >> 1, atom = lane & 1;
  float s = 0.f;
#pragma unroll
  for (int ch = 0; ch < 8; ++ch) {
    const int off = atom * 2048 + r * 128 + ((ch ^ (r & 7)) << 4);
    const uint4 w = *reinterpret_cast<const uint4 *>(src + off);
    s += (bf16lo(w.x) + bf16hi(w.x)) + (bf16lo(w.y) + bf16hi(w.y)) + (bf16lo(w.z) + bf16hi(w.z)) +
         (bf16lo(w.w) + bf16hi(w.w));
    uint4 o = w;
    if (permute) {
      o.x = __byte_perm(w.x, w.z, 0x5410);
      o.y = __byte_perm(w.x, w.z, 0x7632);
      o.z = __byte_perm(w.y, w.w, 0x5410);
      o.w = __byte_perm(w.y, w.w, 0x7632);
    }
    *reinterpret_cast<uint4 *>(dst + off) = o;
  }
  s += __shfl_xor_sync(0xffffffffu, s, 1);
  if (atom == 0) qsum[r] = s;
}

template <int NQ>
__global__ void __launch_bounds__(kThreads, 1) decode_int4_kernel(const __grid_constant__ Int4DecodeArgs a) {
  const DecodeParams &p = a.p;
  extern __shared__ char smem_raw[];
  char *smem = reinterpret_cast<char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) { return sbase + kSmBar + 8u * i; };
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kSmMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kSmMisc + 4);
  volatile int *last_flag = reinterpret_cast<volatile int *>(smem + kSmMisc + 8);
  float *red = reinterpret_cast<float *>(smem + kSmRed);
  const float *qsum_all = reinterpret_cast<const float *>(smem + kSmQsum);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // A decode launched next on the stream may start its set-up on the SMs this grid
  // frees; it touches global memory only after its own griddepcontrol.wait, which
  // returns once this whole grid has completed.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int64_t u0 = cta_begin(a, blockIdx.x), u1 = cta_begin(a, blockIdx.x + 1);
  const int nu = static_cast<int>(u1 - u0);
  const int G = p.G;

  if (tid == 0) {
    for (int i = 0; i < kRaw; ++i) {
      mbar_init(bar(kBarRawFull + i), 1);
      mbar_init(bar(kBarRawEmpty + i), 256);
    }
    for (int i = 0; i < kCvt; ++i) {
      mbar_init(bar(kBarCvtFull + i), 256);
      mbar_init(bar(kBarCvtEmpty + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(kBarSFull + i), 1);
      mbar_init(bar(kBarSFree + i), 128);
      mbar_init(bar(kBarPFull + i), 128);
      mbar_init(bar(kBarOFull + i), 1);
    }
    mbar_init(bar(kBarDrain), 1);
    fence_mbar_init();
    *abort_flag = 0;
  }
  // P'^T rows >= G stay zero for the whole kernel
  for (int i = tid; i < 8192 / 16; i += kThreads) reinterpret_cast<uint4 *>(smem + kSmP)[i] = make_uint4(0, 0, 0, 0);
  if (warp == 1) tc::tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  tc::fence_async_smem();
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ================= TMA producer =================
    if (lane == 0) {
      // Launched as a programmatic dependent, this grid's set-up overlaps the previous
      // kernel on the stream; nothing is read from global memory before that kernel has
      // finished (every other read and every write of this grid follows these loads).
      asm volatile("griddepcontrol.wait;" ::: "memory");
      int r = 0, prev_item = -1;
      bool ok = true;
      UnitIter it(a, u0);
      for (int j = 0; j < nu && ok; ++j, it.next(a)) {
        const Unit un = it.un;
        const bool first = un.item != prev_item;
        prev_item = un.item;
        int b, g, z;
        item_coords(a, un.item, b, g, z);
        const int qrow = b * p.Hq + g * G;  // rows beyond this group's G heads are never used
        const int pieces = un.retr ? 1 : 4;
        for (int c = 0; c < pieces; ++c, ++r) {
          const int s = r % kRaw;
          if (r >= kRaw && !tc::wait_bar(bar(kBarRawEmpty + s), ((r / kRaw) - 1) & 1, p.status, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t dst = sbase + kSmRaw + s * kRawStage;
          const uint32_t fb = bar(kBarRawFull + s);
          const bool with_q = first && c == 0;
          if (un.retr) {
            mbar_expect_tx(fb, 2 * 8192 + 2 * 512 + (with_q ? 4096 : 0));
            const int y = un.tile * kTile;
            tc::tma_3d(dst + kRawKc, &a.tm_kc, 0, y, z, fb);
            tc::tma_3d(dst + kRawVc, &a.tm_vc, 0, y, z, fb);
            const int64_t row = static_cast<int64_t>(z) * p.max_len + y;
            bulk_g2s(dst + kRawKsz, p.rk_sz + row * 4, 512, fb);
            bulk_g2s(dst + kRawVsz, p.rv_sz + row * 4, 512, fb);
          } else {
            mbar_expect_tx(fb, 4 * 4096 + (with_q ? 4096 : 0));
            const int y = un.tile * kTile + 32 * c;  // rows past S+W read as zeros
            tc::tma_3d(dst, &a.tm_ks, 0, y, z, fb);
            tc::tma_3d(dst + 4096, &a.tm_ks, 64, y, z, fb);
            tc::tma_3d(dst + 8192, &a.tm_vs, 0, y, z, fb);
            tc::tma_3d(dst + 12288, &a.tm_vs, 64, y, z, fb);
          }
          if (with_q) {
            tc::tma_2d(dst + kRawQ, &a.tm_q, 0, qrow, fb);
            tc::tma_2d(dst + kRawQ + 2048, &a.tm_q, 64, qrow, fb);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ================= MMA issuer =================
    // Event-driven: S(js) as soon as its expanded stage is ready and its S buffer free,
    // O(jo) as soon as the softmax has written P'(jo), whichever comes first.
    if (lane == 0) {
      constexpr uint32_t kIdS = tc::idesc_bf16(128, 16, false, false);
      constexpr uint32_t kIdO = tc::idesc_bf16(128, 16, true, false);
      constexpr uint32_t kIdO16 = tc::idesc_f16(128, 16, true, false, false);  // INT4 tiles: fp16 V" and P'
      // descriptors of every operand base; a K step adds its byte offset >> 4
      const uint64_t dq0 = tc::sdesc(sbase + kSmQ, 16, 1024);                         // Qpad, K-major
      const uint64_t dv0 = tc::sdesc(sbase + kSmCvt + kCvtV, 16384, 1024);           // V"^T, MN-major
      const uint64_t dp0 = tc::sdesc(sbase + kSmP, 16, 1024);                         // P'^T, K-major
      int js = 0, jo = 0, nitem = -1, prev_item = -1;
      UnitIter its(a, u0), ito(a, u0);
      uint32_t idle = 0;
      unsigned long long t_idle = 0;
      while (jo < nu) {
        bool did = false;
        if (js < nu) {
          const int cs = js % kCvt;
          if (mbar_test_wait(bar(kBarCvtFull + cs), (js / kCvt) & 1) &&
              (js < 2 || mbar_test_wait(bar(kBarSFree + (js & 1)), ((js - 2) >> 1) & 1))) {
            const int item = its.un.item;
            its.next(a);
            if (item != prev_item) {
              prev_item = item;
              ++nitem;
            }
            tc::fence_after();
            const uint64_t dq = dq0 + (nitem & 1) * (4096 >> 4);
            const uint32_t d = tmem + kTmS + (js & 1) * kAcc * 16;
            const uint32_t ka = tmem + kTmK + cs * 64;
#pragma unroll
            for (int i = 0; i < 8; ++i) {  // K = d 128 in steps of 16 (8 TMEM columns each)
              const int kk = (i % kAcc) * (8 / kAcc) + i / kAcc;
              tc::mma_ts(d + (i % kAcc) * 16, ka + kk * 8, dq + (kk >> 2) * 128 + (kk & 3) * 2, kIdS, i >= kAcc ? 1u : 0u);
            }
            tc::commit(bar(kBarSFull + (js & 1)));
            ++js;
            did = true;
          }
        }
        if (jo < js && mbar_test_wait(bar(kBarPFull + (jo & 1)), (jo >> 1) & 1)) {
          tc::fence_after();
          const int cs = jo % kCvt;
          const uint32_t id = ito.un.retr ? kIdO16 : kIdO;
          ito.next(a);
          const uint64_t dv = dv0 + cs * (kCvtStage >> 4);
          const uint64_t dp = dp0 + (jo & 1) * (4096 >> 4);
          const uint32_t d = tmem + kTmO + (jo & 1) * kAcc * 16;
#pragma unroll
          for (int i = 0; i < 8; ++i) {  // K = 128 tokens in steps of 16
            const int kk = (i % kAcc) * (8 / kAcc) + i / kAcc;
            tc::mma_ss(d + (i % kAcc) * 16, dv + kk * 128, dp + (kk >> 2) * 128 + (kk & 3) * 2, id, i >= kAcc ? 1u : 0u);
          }
          tc::commit(bar(kBarOFull + (jo & 1)));
          tc::commit(bar(kBarCvtEmpty + cs));  // V", K' and the stage's scales are no longer read
          ++jo;
          did = true;
        }
        if (did) {
          idle = 0;
        } else {
          // sleep on the event expected next rather than spin beside the other warps
          if (jo < js)
            mbar_try_wait_ns(bar(kBarPFull + (jo & 1)), (jo >> 1) & 1, 100);
          else
            mbar_try_wait_ns(bar(kBarCvtFull + js % kCvt), (js / kCvt) & 1, 100);
          if (++idle == 1) t_idle = globaltimer();
        }
        if (idle > 0 && (idle & 63) == 0) {
          if (*abort_flag) break;
          if (globaltimer() - t_idle > kWaitLimitNs) {
            flag_status(p.status, kDevTimeout);
            *abort_flag = 1;
            break;
          }
        }
      }
      tc::commit(bar(kBarDrain));
      mbar_wait(bar(kBarDrain), 0, p.status);
    }
  } else if (warp < 6) {
    // ================= softmax warpgroup =================
    // As in the bf16 kernel (lazy rescaling against a reference max, exact for INT4
    // items), plus the scale and zero of every token: s = s_k (q . c') + (z_k - 128 s_k)
    // sum(q); the MMA gets p' = fp16(p s_v) and zc accumulates p z_v - 1024 p' (bf16
    // tiles: p' = bf16(p), zc = 0).
    constexpr float kSlack = 8.0f;
    const int wq = warp & 3;
    const int t = (wq << 5) | lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq << 5) << 16);
    const float c = p.scale_log2;
    float m[NQ], l[NQ], zc[NQ], o[NQ], qs[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      m[q] = -INFINITY;
      l[q] = 0.f;
      zc[q] = 0.f;
      o[q] = 0.f;
      qs[q] = 0.f;
    }
    bool ok = true, cur_int4 = false;
    int cur_item = -1, nitem = -1;

    // Writes this CTA's result for `item` (partial or final) and merges when last.
    auto flush = [&](int item) {
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        const float vl = warp_sum(l[q]);
        const float vz = warp_sum(zc[q]);
        if (lane == 0) {
          red[wq * kN + q] = vl;
          red[64 + wq * kN + q] = vz;
        }
      }
      tc::named_sync(1, 128);
      float lt[NQ], zt[NQ];
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        lt[q] = red[q] + red[kN + q] + red[2 * kN + q] + red[3 * kN + q];
        zt[q] = red[64 + q] + red[64 + kN + q] + red[64 + 2 * kN + q] + red[64 + 3 * kN + q];
      }
      tc::named_sync(1, 128);
      const bool retr = item < a.n_items_r;
      const int units = retr ? a.units_r : a.units_s;
      const int64_t ia = retr ? static_cast<int64_t>(item) * a.units_r
                              : a.ur + static_cast<int64_t>(item - a.n_items_r) * a.units_s;
      const int cfirst = cta_of(a, ia), clast = cta_of(a, ia + units - 1);
      const int nseg = clast - cfirst + 1;
      int b, g, z;
      item_coords(a, item, b, g, z);
      const int h0 = g * G;
      const int e = cur_int4 ? perm(t) : t;  // output element held by this thread's O^T lane
      if (nseg == 1) {
#pragma unroll
        for (int q = 0; q < NQ; ++q)
          if (q < G) {
            Elem<__nv_bfloat16>::store(p.out, (static_cast<int64_t>(b) * p.Hq + h0 + q) * kD + e,
                                       (o[q] + zt[q]) / lt[q]);
            if (t == 0 && p.lse) p.lse[b * p.Hq + h0 + q] = (m[q] + lg2(lt[q])) * kLn2;
          }
        return;
      }
      const int seg = blockIdx.x - cfirst;
      const int64_t pitem = static_cast<int64_t>(b) * p.Hkv + g;
      float *part = p.partials + (pitem * p.max_splits) * G * kPartRow;
#pragma unroll
      for (int q = 0; q < NQ; ++q)
        if (q < G) {
          float *dst = part + (static_cast<int64_t>(seg) * G + q) * kPartRow;
          dst[e] = o[q] + zt[q];
          if (t == 0) {
            dst[kD] = m[q];
            dst[kD + 1] = lt[q];
          }
        }
      __threadfence();
      tc::named_sync(1, 128);
      if (t == 0) {
        const uint32_t prev = atomicAdd(p.counters + pitem, 1u);
        *last_flag = (prev == static_cast<uint32_t>(nseg - 1)) ? 1 : 0;
      }
      tc::named_sync(1, 128);
      if (!*last_flag) return;
      __threadfence();
      merge_partials(part, nseg, G, b, h0, p.Hq, p.out, p.lse, red + 128, t, 1);
      if (t == 0) p.counters[pitem] = 0u;  // ready for the next call
    };

    // o = (o + O^T(jj)) * alpha for this thread's position t
    auto fold = [&](int jj, const float (&alpha)[NQ]) {
      if (ok) ok = tc::wait_bar(bar(kBarOFull + (jj & 1)), (jj >> 1) & 1, p.status, abort_flag);
      tc::fence_after();
      float v[NQ];
      tc::ld_sum<NQ, kAcc>(lane_base + kTmO + (jj & 1) * kAcc * 16, 16, v);
#pragma unroll
      for (int q = 0; q < NQ; ++q) o[q] = (o[q] + v[q]) * alpha[q];
    };
    float one[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q) one[q] = 1.f;

    bool pending = false;  // O^T of the previous unit still to be folded
    UnitIter it(a, u0);
    for (int j = 0; j < nu; ++j, it.next(a)) {
      const Unit un = it.un;
      const int cb = j & 1;
      if (ok) ok = tc::wait_bar(bar(kBarSFull + cb), (j >> 1) & 1, p.status, abort_flag);
      tc::fence_after();
      float sv[NQ];
      tc::ld_sum<NQ, kAcc>(lane_base + kTmS + cb * kAcc * 16, 16, sv);
      tc::fence_before();
      mbar_arrive(bar(kBarSFree + cb));  // S buffer j % 2 is free again
      // the expanded stage of this tile (complete already: its MMA has run) holds the
      // scales; waiting here orders the expansion warps' writes before these reads
      const int cs = j % kCvt;
      if (ok) ok = tc::wait_bar(bar(kBarCvtFull + cs), (j / kCvt) & 1, p.status, abort_flag);
      const float4 mi = *reinterpret_cast<const float4 *>(smem + kSmCvt + cs * kCvtStage + kCvtMisc + t * 16);
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
        ++nitem;
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          m[q] = -INFINITY;
          l[q] = 0.f;
          zc[q] = 0.f;
          o[q] = 0.f;
          qs[q] = qsum_all[(nitem & 1) * kN + q];
        }
        pending = false;
        cur_item = un.item;
        cur_int4 = un.retr;
      }
#pragma unroll
      for (int q = 0; q < NQ; ++q) sv[q] = fmaf(mi.x, sv[q], mi.y * qs[q]);
      const float slack = cur_int4 ? 0.f : kSlack;
      // does any logit of this tile exceed the reference max by more than kSlack?
      int need = 0;
#pragma unroll
      for (int q = 0; q < NQ; ++q)
        if (q < G && valid && sv[q] * c > m[q] + slack) need = 1;
      need = tc::bar_or(1, 128, need);
      float alpha[NQ];
#pragma unroll
      for (int q = 0; q < NQ; ++q) alpha[q] = 1.f;
      if (need) {  // uniform over the warpgroup
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          const float x = warp_max((valid && q < G) ? sv[q] : -INFINITY);
          if (lane == 0) red[wq * kN + q] = x;
        }
        tc::named_sync(1, 128);
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          const float mt = fmaxf(fmaxf(red[q], red[kN + q]), fmaxf(red[2 * kN + q], red[3 * kN + q])) * c;
          const float mn = fmaxf(m[q], mt);
          alpha[q] = (mn == -INFINITY) ? 1.f : ex2(m[q] - mn);
          m[q] = mn;
        }
        tc::named_sync(1, 128);  // red is reused later
      }
      uint16_t pb[NQ];
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        const float pv = (valid && q < G && m[q] != -INFINITY) ? ex2(fmaf(sv[q], c, -m[q])) : 0.f;
        l[q] = fmaf(l[q], alpha[q], pv);
        if (cur_int4) {
          const __half hp = __float2half_rn(pv * mi.z);
          zc[q] = fmaf(zc[q], alpha[q], fmaf(pv, mi.w, -1024.f * __half2float(hp)));
          pb[q] = __half_as_ushort(hp);
        } else {
          const __nv_bfloat16 hb = __float2bfloat16_rn(pv);
          pb[q] = *reinterpret_cast<const uint16_t *>(&hb);
        }
      }
      // P'^T[q][t] into buffer j % 2 (its previous reader, unit j-2, was folded at j-1)
      {
        const int atom = t >> 6, col = t & 63;
        char *pbase = smem + kSmP + cb * 4096 + atom * 2048;
#pragma unroll
        for (int q = 0; q < NQ; ++q)
          if (q < G) {
            const int chunk = (col >> 3) ^ (q & 7);
            *reinterpret_cast<uint16_t *>(pbase + q * 128 + chunk * 16 + (col & 7) * 2) = pb[q];
          }
      }
      tc::fence_async_smem();
      tc::fence_before();
      mbar_arrive(bar(kBarPFull + cb));
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
    } else {
      const int item = empty_cta_item(a, blockIdx.x);
      if (item >= 0) flush(item);  // m = -inf, l = 0, o = 0: a segment that sees nothing
    }
  } else {
    // ================= expansion warps =================
    const int wq = warp & 3;
    const int h = (warp - 6) >> 2;    // half of the row: elements 64 h .. 64 h + 63
    const int ct = (wq << 5) | lane;  // token row of the tile = TMEM lane
    const uint32_t tm_lane = tmem + (static_cast<uint32_t>(wq << 5) << 16);
    const int rot = (ct >> 1) & 3;    // 64-byte swizzle of code row ct: chunk i sits at i ^ rot
    int r = 0, prev_item = -1, nitem = -1;
    UnitIter it(a, u0);
    for (int j = 0; j < nu; ++j, it.next(a)) {
      const Unit un = it.un;
      const bool first = un.item != prev_item;
      if (first) {
        prev_item = un.item;
        ++nitem;
      }
      const int cb = j % kCvt;
      if (j >= kCvt && !tc::wait_bar(bar(kBarCvtEmpty + cb), ((j / kCvt) - 1) & 1, p.status, abort_flag)) break;
      char *cv = smem + kSmCvt + cb * kCvtStage;
      char *qdst = smem + kSmQ + (nitem & 1) * 4096;
      float *qsum = reinterpret_cast<float *>(smem + kSmQsum) + (nitem & 1) * kN;
      const uint32_t tk = tm_lane + kTmK + cb * 64 + h * 32;
      if (un.retr) {
        const int s = r % kRaw;
        if (!tc::wait_bar(bar(kBarRawFull + s), (r / kRaw) & 1, p.status, abort_flag)) break;
        const char *rs = smem + kSmRaw + s * kRawStage;
        uint4 kw[2], vw[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int off = ct * 64 + (((2 * h + i) ^ rot) << 4);
          kw[i] = *reinterpret_cast<const uint4 *>(rs + kRawKc + off);
          vw[i] = *reinterpret_cast<const uint4 *>(rs + kRawVc + off);
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {  // K: 32 codes -> TMEM columns 32 h + 16 i ..
          const uint4 e0 = expand8<kBf16Base>(kw[i].x), e1 = expand8<kBf16Base>(kw[i].y),
                      e2 = expand8<kBf16Base>(kw[i].z), e3 = expand8<kBf16Base>(kw[i].w);
          const uint32_t v[16] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w,
                                  e2.x, e2.y, e2.z, e2.w, e3.x, e3.y, e3.z, e3.w};
          tc::st16(tk + i * 16, v);
        }
        char *vrow = cv + kCvtV + h * 16384 + ct * 128;
#pragma unroll
        for (int i = 0; i < 2; ++i) {  // V: 32 codes -> chunks 4 i .. 4 i + 3 of atom h
          const uint32_t ws[4] = {vw[i].x, vw[i].y, vw[i].z, vw[i].w};
#pragma unroll
          for (int mm = 0; mm < 4; ++mm)
            *reinterpret_cast<uint4 *>(vrow + (((4 * i + mm) ^ (ct & 7)) << 4)) = expand8<kFp16Base>(ws[mm]);
        }
        if (h == 0) {
          const uint32_t ksz = *reinterpret_cast<const uint32_t *>(rs + kRawKsz + ct * 4);
          const uint32_t vsz = *reinterpret_cast<const uint32_t *>(rs + kRawVsz + ct * 4);
          const float ks = __half2float(__ushort_as_half(static_cast<unsigned short>(ksz & 0xffffu)));
          const float kz = __half2float(__ushort_as_half(static_cast<unsigned short>(ksz >> 16)));
          const float vs = __half2float(__ushort_as_half(static_cast<unsigned short>(vsz & 0xffffu)));
          const float vz = __half2float(__ushort_as_half(static_cast<unsigned short>(vsz >> 16)));
          *reinterpret_cast<float4 *>(cv + kCvtMisc + ct * 16) = make_float4(ks, fmaf(-128.f, ks, kz), vs, vz);
        } else if (first && wq == 0) {
          stage_queries(rs + kRawQ, qdst, qsum, lane, true);
        }
        mbar_arrive(bar(kBarRawEmpty + s));  // all 256 threads read this stage
        ++r;
      } else {
        // the two warps of quarter wq expand piece wq (tokens 32 wq .. 32 wq + 31)
        const int s = (r + wq) % kRaw;
        if (!tc::wait_bar(bar(kBarRawFull + s), ((r + wq) / kRaw) & 1, p.status, abort_flag)) break;
        const char *rs = smem + kSmRaw + s * kRawStage;
#pragma unroll
        for (int i = 0; i < 2; ++i) {  // K half h -> TMEM columns 32 h + 16 i ..
          uint32_t v[16];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int ch = 4 * i + k;
            const uint4 w = *reinterpret_cast<const uint4 *>(rs + h * 4096 + lane * 128 + ((ch ^ (lane & 7)) << 4));
            v[4 * k] = w.x;
            v[4 * k + 1] = w.y;
            v[4 * k + 2] = w.z;
            v[4 * k + 3] = w.w;
          }
          tc::st16(tk + i * 16, v);
        }
        // V half h: the piece's swizzle matches the tile's (row ct = 32 wq + lane)
#pragma unroll
        for (int ch = 0; ch < 8; ++ch)
          *reinterpret_cast<uint4 *>(cv + kCvtV + h * 16384 + ct * 128 + ch * 16) =
              *reinterpret_cast<const uint4 *>(rs + 8192 + h * 4096 + lane * 128 + ch * 16);
        if (h == 0)
          *reinterpret_cast<float4 *>(cv + kCvtMisc + ct * 16) = make_float4(1.f, 0.f, 1.f, 0.f);
        else if (first && wq == 0)
          stage_queries(rs + kRawQ, qdst, qsum, lane, false);
        mbar_arrive_n(bar(kBarRawEmpty + s), 4);  // the piece's only readers: 64 threads x 4
        r += 4;
      }
      tc::fence_async_smem();
      tc::st_wait();
      tc::fence_before();
      mbar_arrive(bar(kBarCvtFull + cb));
    }
  }

  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  if (warp == 1) tc::tmem_free(tmem, kTmemCols);
}

template <int NQ>
cudaError_t launch_nq(const Int4DecodeArgs &a, bool overlap_previous, cudaStream_t st) {
  static bool attr = false;
  if (!attr) {
    const cudaError_t e =
        cudaFuncSetAttribute(decode_int4_kernel<NQ>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc);
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
  const cudaError_t e = cudaLaunchKernelEx(&cfg, decode_int4_kernel<NQ>, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

bool decode_int4_tc_supported(const DecodeParams &p, duo_dtype dt) {
  return dt == DUO_BF16 && p.D == kD && p.G >= 1 && p.G <= kN && tc::encode_fn() != nullptr;
}

cudaError_t launch_decode_int4_tc(const DecodeParams &p, int num_sms, bool overlap_previous, cudaStream_t st) {
  Int4DecodeArgs a{};
  a.p = p;
  a.units_r = static_cast<int>((p.len + kTile - 1) / kTile);
  const int64_t slots = static_cast<int64_t>(p.S) + p.W;
  // highest ring slot in use + 1: position p >= S sits in slot S + p mod W, so before the
  // ring wraps (len <= W) the slots reach S + len - 1, beyond len itself
  const int64_t reach = static_cast<int64_t>(p.S) + p.len;
  const int64_t used = reach < slots ? reach : slots;
  a.units_s = static_cast<int>((used + kTile - 1) / kTile);
  a.n_items_r = p.B * p.Hr;
  a.ur = static_cast<int64_t>(a.n_items_r) * a.units_r;
  const int64_t us = static_cast<int64_t>(p.B) * p.Hs * a.units_s;
  a.total_units = a.ur + us;
  a.total_cost = a.ur + kWs * us;
  // at most one CTA per SM, and never more segments per item than partial slots
  int64_t ctas = num_sms;
  if (ctas > a.ur + us) ctas = a.ur + us;
  if (ctas > kMaxSplits) ctas = kMaxSplits;
  a.num_ctas = static_cast<int>(ctas);
  bool ok = true;
  {  // queries [B*Hq][d]
    const uint64_t d[2] = {kD, static_cast<uint64_t>(p.B) * p.Hq};
    const uint64_t s[1] = {kD * 2};
    const uint32_t bx[2] = {64, kN};
    ok &= tc::make_map(&a.tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.q, 2, d, s, bx, CU_TENSOR_MAP_SWIZZLE_128B);
  }
  {  // retrieval codes [B*Hr][cap][64 B]
    const uint64_t rows = static_cast<uint64_t>(p.B) * (p.Hr > 0 ? p.Hr : 1);
    const uint64_t d[3] = {kD / 2, static_cast<uint64_t>(p.max_len), rows};
    const uint64_t s[2] = {kD / 2, static_cast<uint64_t>(kD / 2) * p.max_len};
    const uint32_t bx[3] = {kD / 2, kTile, 1};
    ok &= tc::make_map(&a.tm_kc, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.rk, 3, d, s, bx, CU_TENSOR_MAP_SWIZZLE_64B);
    ok &= tc::make_map(&a.tm_vc, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.rv, 3, d, s, bx, CU_TENSOR_MAP_SWIZZLE_64B);
  }
  {  // streaming [B*Hs][S+W][d] bf16, pieces of 32 rows
    const uint64_t d[3] = {kD, static_cast<uint64_t>(slots), static_cast<uint64_t>(p.B) * (p.Hs > 0 ? p.Hs : 1)};
    const uint64_t s[2] = {kD * 2, static_cast<uint64_t>(kD * 2) * slots};
    const uint32_t bx[3] = {64, 32, 1};
    ok &= tc::make_map(&a.tm_ks, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.sk, 3, d, s, bx, CU_TENSOR_MAP_SWIZZLE_128B);
    ok &= tc::make_map(&a.tm_vs, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.sv, 3, d, s, bx, CU_TENSOR_MAP_SWIZZLE_128B);
  }
  if (!ok) return cudaErrorInvalidValue;
  if (p.G <= 1) return launch_nq<1>(a, overlap_previous, st);
  if (p.G <= 2) return launch_nq<2>(a, overlap_previous, st);
  if (p.G <= 4) return launch_nq<4>(a, overlap_previous, st);
  if (p.G <= 8) return launch_nq<8>(a, overlap_previous, st);
  return launch_nq<16>(a, overlap_previous, st);
}

}  // namespace duo
