// k_decode_fp8_tc.cu -- single-token decode attention over retrieval heads that keep K
// and V as 8-bit floating point (OCP E4M3, one fp32 scale per token row), on the
// tcgen05 tensor cores with 8-bit operands.  bf16 queries, head_dim 128, up to 16 query
// heads per KV head; the layer's streaming heads (bf16) run on the bf16 decode kernel.
//
// Operation ("Decoding Procedure", steps 2, 3 and 5) as in k_decode_tc.cu; the stored
// value of element e of token t is c_te s_t (code c, scale s_t), the format pairing the
// method with an 8-bit KV cache ("Integration with Existing Optimizations").
//
// The tensor cores read the stored codes as they are (kind::f8f6f4, E4M3 x E4M3, fp32
// accumulators); the fp32 operands enter as three E4M3 limbs each, limb l scaled by
// 16^l, so that x = v0 + v1 / 16 + v2 / 256 to 12 bits of x:
//   S^T (128 tokens x 3 NQ) = Kc . Ql^T     Ql: limbs of 2^e_q q (largest |q| of head q
//                                          in [2^7, 2^8)), one row per (limb, head)
//   O^T (d x 3 NQ)         = Vc^T . P'^T   P'_t = p_t s^V_t 2^6 / smax (smax the tile's
//                                          largest V scale; p <= 4 keeps P' <= 2^8)
// Per token the scales then give
//   q . k_t = s^K_t 2^-e_q (S0 + S1 / 16 + S2 / 256),
//   sum_t p_t v_t = smax 2^-6 (O0 + O1 / 16 + O2 / 256) summed over tiles.
//
// Roles of a CTA (one per SM, 384 threads):
//   warp 0     TMA producer: per 128-token tile the K and V code rows (128 B each,
//              128-byte swizzle) and their scale rows, at an item's first tile the
//              group's bf16 queries; a ring of kStages stages, released after O^T.
//   warp 1     TMEM owner and S^T issuer (4 MMAs per tile); at an item's first tile the
//              whole warp turns the queries into limbs first.  Warp 2 issues O^T.
//   warps 4-11 softmax, two warpgroups taking alternate tiles (each with its own
//              running max and sums, combined when an item ends): thread t owns token t
//              of S^T and dimension t of O^T.
//
// Work balance and the split merge are those of the other decode kernels: the
// 128-token tiles of all (batch, retrieval head) items are laid end to end and cut
// into one equal range per CTA; the last CTA of an item merges its partials.
#include "decode_merge.cuh"
#include "tcgen05.cuh"

namespace duo {

namespace {

constexpr int kThreads = 384;
constexpr int kTile = 128;
constexpr int kD = 128;
constexpr int kStages = 5;
constexpr int kPrefetch = 4;  // tiles asked of L2 before the previous grid has finished
constexpr float kSlack = 2.f;  // the running max trails the true one by at most this (log2)
// stage: K and V codes [128][128 B] (128-byte swizzle, as the TMA writes them), the K and
// V scale rows [128] fp32, at an item's first tile the queries [16][128] bf16 (two
// 128-byte-swizzled atoms)
constexpr int kStKc = 0, kStVc = 16384, kStKs = 32768, kStVs = 33280, kStQ = 33792, kStage = 37888;
constexpr int kQlBytes = 6144;                // query limbs [48][128 B] E4M3, 128-byte swizzle
constexpr int kPBuf = 6144;                   // P'^T limbs of a tile: up to 3 blocks of 16 rows
constexpr int kSmQl = kStages * kStage;       // 2 x query limbs (item parity)
constexpr int kSmP = kSmQl + 2 * kQlBytes;    // 4 x P'^T (MN-major, no swizzle); flush exchange
constexpr int kSmQinfo = kSmP + 4 * kPBuf;    // [2][16] 2^-e_q per query head
constexpr int kSmVmax = kSmQinfo + 128;       // [2 groups][2][4 warps] largest V scale
constexpr int kSmRed = kSmVmax + 128;         // per softmax group [4][16]; [128][6] merge
constexpr int kSmBar = kSmRed + (2 * 64 + 128 * 6) * 4;
constexpr int kSmMisc = kSmBar + 256;
constexpr int kSmemAlloc = kSmMisc + 64 + 1024;
static_assert(kStage % 1024 == 0 && kStQ % 1024 == 0 && kSmQl % 1024 == 0 && kSmP % 1024 == 0 &&
                  kQlBytes % 1024 == 0, "alignment");
static_assert(kSmemAlloc <= 232448, "shared memory");

// P' and O^T have four buffers each, and so four barriers: with two groups a group
// publishes P'(j + 2) before the issuer need have taken P'(j)
constexpr int kBarFull = 0, kBarEmpty = kStages, kBarSFull = 2 * kStages, kBarSFree = kBarSFull + 2,
              kBarPFull = kBarSFull + 4, kBarOFull = kBarSFull + 8, kBarQFree = kBarSFull + 12,
              kBarQInfo = kBarSFull + 14, kBarDrain = kBarSFull + 16,  // a drain barrier per issuer
              kBarMerge = kBarSFull + 18, kNumBars = kBarSFull + 19;
static_assert(kNumBars * 8 <= 256, "barrier area");

// tensor memory columns: S^T x 2 and O^T x 4, three limb columns per query head each
template <int NQ>
struct Cols {
  static constexpr int kS = (3 * NQ + 15) / 16 * 16;
  static constexpr int kO = kS;
  static constexpr int kUsed = 2 * kS + 4 * kO;
  static constexpr int kAlloc = kUsed <= 128 ? 128 : kUsed <= 256 ? 256 : 512;
};

struct Fp8DecodeArgs {
  DecodeParams p;
  int units_r;          // tiles per item
  int n_items;          // B * Hr
  int64_t total_units;  // n_items * units_r
  int num_ctas;
  CUtensorMap tm_q, tm_kc, tm_vc;
};

// shared-memory matrix descriptor without swizzle (layout 0), descriptor version 1
__device__ __forceinline__ uint64_t sdesc_plain(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}
// kind::f8f6f4 instruction descriptor: fp32 accumulator, A and B E4M3 (format 0)
constexpr uint32_t idesc_e4m3(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         ((static_cast<uint32_t>(N) >> 3) << 17) | ((static_cast<uint32_t>(M) >> 4) << 24);
}
__device__ __forceinline__ void mma_e4m3(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(acc)
      : "memory");
}

// two fp32 -> two E4M3 codes (lo in the low byte), round to nearest even, saturating
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  unsigned short r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}
// the values of two E4M3 codes (low byte first) as fp32; exact
__device__ __forceinline__ void e4m3x2_values(uint32_t two, float &lo, float &hi) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(static_cast<unsigned short>(two)));
  const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&h2));
  lo = f.x;
  hi = f.y;
}
// Three E4M3 limbs of a and b (|a|, |b| <= 2^8): a = v0 + v1 / 16 + v2 / 256 up to 2^-12 |a|
// (or 2^-18 absolute where the limbs leave the normal range); w[l] holds limb l of a in
// the low byte and of b in the next.  x - v is exact, and 16 (x - v) <= |x|.
__device__ __forceinline__ void limbs3(float a, float b, uint32_t (&w)[3]) {
#pragma unroll
  for (int l = 0; l < 3; ++l) {
    w[l] = e4m3x2(a, b);
    if (l < 2) {
      float va, vb;
      e4m3x2_values(w[l], va, vb);
      a = (a - va) * 16.f;
      b = (b - vb) * 16.f;
    }
  }
}
// byte (row n, column k) of a [rows][128 B] K-major operand with 128-byte swizzle
__device__ __forceinline__ int sw128(int n, int k) { return (n >> 3) * 1024 + (n & 7) * 128 + (((k >> 4) ^ (n & 7)) << 4) + (k & 15); }

// N (a multiple of 16) fp32 columns of this thread's TMEM lane, loads issued only;
// ld_wait names every destination register, so that no use precedes the wait
template <int N>
__device__ __forceinline__ void ld_issue(uint32_t taddr, uint32_t (&r)[N]) {
#pragma unroll
  for (int c = 0; c < N; c += 16) {
    uint32_t *q = r + c;
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(q[0]), "=r"(q[1]), "=r"(q[2]), "=r"(q[3]), "=r"(q[4]), "=r"(q[5]), "=r"(q[6]), "=r"(q[7]), "=r"(q[8]),
          "=r"(q[9]), "=r"(q[10]), "=r"(q[11]), "=r"(q[12]), "=r"(q[13]), "=r"(q[14]), "=r"(q[15])
        : "r"(taddr + c));
  }
}
template <int N>
__device__ __forceinline__ void ld_wait(uint32_t (&r)[N]) {
#pragma unroll
  for (int c = 0; c < N; c += 16) {  // the first wait covers every load; the others name registers
    uint32_t *q = r + c;
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(q[0]), "+r"(q[1]), "+r"(q[2]), "+r"(q[3]), "+r"(q[4]), "+r"(q[5]), "+r"(q[6]), "+r"(q[7]),
                   "+r"(q[8]), "+r"(q[9]), "+r"(q[10]), "+r"(q[11]), "+r"(q[12]), "+r"(q[13]), "+r"(q[14]), "+r"(q[15])
                 :
                 : "memory");
  }
}

struct Unit {
  int item, tile;
};
// Walks a CTA's units in order without a division per step.
struct UnitIter {
  Unit un;
  int units;
  __device__ __forceinline__ UnitIter(const Fp8DecodeArgs &a, int64_t u)
      : un{static_cast<int>(u / a.units_r), static_cast<int>(u % a.units_r)}, units(a.units_r) {}
  __device__ __forceinline__ void next() {
    if (++un.tile == units) {
      ++un.item;
      un.tile = 0;
    }
  }
};
__device__ __forceinline__ int64_t cta_begin(const Fp8DecodeArgs &a, int c) {
  return static_cast<int64_t>(c) * a.total_units / a.num_ctas;
}
__device__ __forceinline__ int cta_of(const Fp8DecodeArgs &a, int64_t u) {
  return static_cast<int>(((u + 1) * a.num_ctas + a.total_units - 1) / a.total_units) - 1;
}

// One warp turns the G query rows of an item (bf16 [16][128], two 128-byte-swizzled
// atoms) into the B operand of S^T: row l NQ + q holds E4M3 limb l of 2^e_q q, column k
// its element k.  Rows of heads q >= G are never written (they stay zero).  Writes 2^-e_q.
template <int NQ>
__device__ __forceinline__ void prep_queries(const char *qr, char *ql, float *qinfo, int G, int lane) {
  for (int q = 0; q < G; ++q) {
    float x[4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {  // columns c, c + 1 with c = 2 lane + 64 h
      const int c = 2 * lane;
      const int off = h * 2048 + q * 128 + (((c >> 3) ^ (q & 7)) << 4) + (c & 7) * 2;
      const uint32_t w = *reinterpret_cast<const uint32_t *>(qr + off);
      x[2 * h] = bf16lo(w);
      x[2 * h + 1] = bf16hi(w);
    }
    const float amax = warp_max(fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3]))));
    // 2^e with the largest |q| in [2^7, 2^8) (bf16 values: amax is normal or zero)
    int e = 0;
    if (amax > 0.f) {
      e = 7 - (((__float_as_int(amax) >> 23) & 0xFF) - 127);
      e = e < -100 ? -100 : (e > 100 ? 100 : e);
    }
    const float sc = __int_as_float((127 + e) << 23);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t w[3];
      limbs3(x[2 * h] * sc, x[2 * h + 1] * sc, w);
      const int c = 2 * lane + 64 * h;
#pragma unroll
      for (int l = 0; l < 3; ++l) *reinterpret_cast<uint16_t *>(ql + sw128(l * NQ + q, c)) = static_cast<uint16_t>(w[l]);
    }
    if (lane == 0) qinfo[q] = __int_as_float((127 - e) << 23);
  }
}

template <int NQ>
__global__ void __launch_bounds__(kThreads, 1) decode_fp8_kernel(const __grid_constant__ Fp8DecodeArgs a) {
  using C = Cols<NQ>;
  const DecodeParams &p = a.p;
  extern __shared__ char smem_raw[];
  char *smem = reinterpret_cast<char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) { return sbase + kSmBar + 8u * i; };
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kSmMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kSmMisc + 4);
  volatile int *last_flag = reinterpret_cast<volatile int *>(smem + kSmMisc + 8);
  float *red = reinterpret_cast<float *>(smem + kSmRed);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // A kernel launched next on the stream may start its set-up on the SMs this grid
  // frees; it touches global memory only after its own griddepcontrol.wait, which
  // returns once this whole grid has completed.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int64_t u0 = cta_begin(a, blockIdx.x), u1 = cta_begin(a, blockIdx.x + 1);
  const int nu = static_cast<int>(u1 - u0);
  const int G = p.G;

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(bar(kBarFull + i), 1);
      mbar_init(bar(kBarEmpty + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(kBarSFull + i), 1);
      mbar_init(bar(kBarSFree + i), 4);  // one arrival per warp of a softmax group
      mbar_init(bar(kBarQFree + i), 3);  // the item's last S^T product (commit) + each softmax group
      mbar_init(bar(kBarQInfo + i), 1);  // the query limbs and 2^-e_q of an item are written
      mbar_init(bar(kBarDrain + i), 1);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(bar(kBarPFull + i), 4);  // one arrival per warp of a softmax group
      mbar_init(bar(kBarOFull + i), 1);
    }
    mbar_init(bar(kBarMerge), 1);  // partial rows copied in for the final merge
    fence_mbar_init();
    *abort_flag = 0;
  }
  // query limb rows of heads >= G and the P'^T rows past 3 NQ stay zero
  for (int i = tid; i < (2 * kQlBytes + 4 * kPBuf) / 16; i += kThreads)
    reinterpret_cast<uint4 *>(smem + kSmQl)[i] = make_uint4(0u, 0u, 0u, 0u);
  if (warp == 1) tc::tmem_alloc(smem_u32(tmem_slot), C::kAlloc);
  tc::fence_async_smem();
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ================= TMA producer =================
    if (lane == 0) {
      for (const CUtensorMap *m : {&a.tm_q, &a.tm_kc, &a.tm_vc}) tc::prefetch_map(m);
      {  // L2 prefetch of the first tiles; nothing is consumed before the wait below
        UnitIter it(a, u0);
        for (int j = 0; j < nu && j < kPrefetch; ++j, it.next()) {
          const int64_t row = static_cast<int64_t>(it.un.item) * p.max_len + static_cast<int64_t>(it.un.tile) * kTile;
          prefetch_l2(p.rk + row * kD, kTile * kD);
          prefetch_l2(p.rv + row * kD, kTile * kD);
          prefetch_l2(p.rk_sz + row * 4, kTile * 4);
          prefetch_l2(p.rv_sz + row * 4, kTile * 4);
        }
      }
      // launched as a programmatic dependent: no global read before the previous kernel
      // ends (beside a leading grid, that grid's release already implies it); every
      // other read and every write of this grid follows these loads
      if (p.pdl_mode != 2) asm volatile("griddepcontrol.wait;" ::: "memory");
      int prev_item = -1, issued = 0;
      UnitIter it(a, u0);
      for (int j = 0; j < nu; ++j, it.next()) {
        const int s = j % kStages;
        if (j >= kStages && !tc::wait_bar(bar(kBarEmpty + s), ((j / kStages) - 1) & 1, p.status, abort_flag)) break;
        const Unit un = it.un;
        const bool first = un.item != prev_item;
        prev_item = un.item;
        const uint32_t dst = sbase + s * kStage;
        const uint32_t fb = bar(kBarFull + s);
        mbar_expect_tx(fb, 2 * 16384 + 2 * 512 + (first ? 4096 : 0));
        const int y = un.tile * kTile;
        const int z = un.item;  // = b * Hr + retrieval index
        tc::tma_3d(dst + kStKc, &a.tm_kc, 0, y, z, fb);
        tc::tma_3d(dst + kStVc, &a.tm_vc, 0, y, z, fb);
        const int64_t row = static_cast<int64_t>(z) * p.max_len + y;
        bulk_g2s(dst + kStKs, p.rk_sz + row * 4, 512, fb);
        bulk_g2s(dst + kStVs, p.rv_sz + row * 4, 512, fb);
        if (first) {
          const int b = un.item / p.Hr;
          const int g = p.hm.retr_head[un.item % p.Hr];
          const int qrow = b * p.Hq + g * G;  // rows beyond this group's G heads are never used
          tc::tma_2d(dst + kStQ, &a.tm_q, 0, qrow, fb);
          tc::tma_2d(dst + kStQ + 2048, &a.tm_q, 64, qrow, fb);
        }
        ++issued;
      }
      // after an abort, loads may still be landing: none may outlive the CTA
      tc::drain_loads(bar(kBarFull), kStages, issued, p.status);
    }
  } else if (warp == 1) {
    // ================= S^T issuer (lane 0) and query limbs (whole warp) =================
    // S^T(j) once the stage has landed and the softmax has read S^T(j - 2) (its
    // buffer); at an item's first tile the warp first writes the item's query limbs
    // into the buffer of its parity, once the item two before has released it.
    // tcgen05.commit tracks the committing thread's own MMAs.
    constexpr uint32_t kIdS = idesc_e4m3(128, C::kS, false, false);  // Kc . Ql^T, both K-major
    const uint64_t ak0 = tc::sdesc(sbase + kStKc, 16, 1024);
    const uint64_t bq0 = tc::sdesc(sbase + kSmQl, 16, 1024);
    bool ok = true;
    int nitem = -1, prev_item = -1;
    UnitIter its(a, u0);
    int ss = 0, sph = 0;  // stage of S^T(js) and the phase of its full barrier
    for (int js = 0; js < nu; ++js) {
      const int item = its.un.item;
      its.next();
      const bool first = item != prev_item;
      if (first) {
        prev_item = item;
        ++nitem;
      }
      ok = __all_sync(0xffffffffu, tc::wait_bar(bar(kBarFull + ss), sph, p.status, abort_flag));
      if (ok && first) {
        if (nitem >= 2)
          ok = __all_sync(0xffffffffu,
                          tc::wait_bar(bar(kBarQFree + (nitem & 1)), ((nitem - 2) >> 1) & 1, p.status, abort_flag));
        if (ok) {
          prep_queries<NQ>(smem + ss * kStage + kStQ, smem + kSmQl + (nitem & 1) * kQlBytes,
                           reinterpret_cast<float *>(smem + kSmQinfo) + (nitem & 1) * 16, G, lane);
          tc::fence_async_smem();  // the limbs are an MMA operand
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(kBarQInfo + (nitem & 1)));
        }
      }
      if (ok && js >= 2)
        ok = __all_sync(0xffffffffu,
                        tc::wait_bar(bar(kBarSFree + (js & 1)), ((js - 2) >> 1) & 1, p.status, abort_flag));
      if (!ok) break;
      if (lane == 0) {
        tc::fence_after();
        const uint64_t ak = ak0 + ss * (kStage >> 4);
        const uint64_t bq = bq0 + (nitem & 1) * (kQlBytes >> 4);
        const uint32_t d = tmem + (js & 1) * C::kS;
#pragma unroll
        for (int k = 0; k < 4; ++k)  // K = 128 dimensions in steps of 32 (32 bytes)
          mma_e4m3(d, ak + 2 * k, bq + 2 * k, kIdS, k > 0 ? 1u : 0u);
        tc::commit(bar(kBarSFull + (js & 1)));
        // the item's query limbs are free once its last S^T product has run
        if (js + 1 == nu || its.un.item != item) tc::commit(bar(kBarQFree + (nitem & 1)));
      }
      __syncwarp();
      if (++ss == kStages) {
        ss = 0;
        sph ^= 1;
      }
    }
    if (lane == 0) {  // every MMA this thread issued has completed before TMEM is freed
      tc::commit(bar(kBarDrain));
      mbar_wait(bar(kBarDrain), 0, p.status);
    }
  } else if (warp == 2) {
    // ================= O^T issuer =================
    // O^T(j) once P'(j) is written; then the stage is released (S^T(j) has completed:
    // the softmax saw it land before writing P'(j)).
    if (lane == 0) {
      constexpr uint32_t kIdO = idesc_e4m3(128, C::kO, true, true);  // Vc^T . P'^T, both MN-major
      // Vc^T MN-major: a code row (128 dimensions) is one 128-byte swizzle row, 8 tokens
      // per 1 KiB atom; P'^T MN-major without swizzle: a token's 16 limb bytes per row, 8
      // tokens per 128-byte core matrix (the leading byte offset steps along the tokens),
      // blocks of 16 limb rows 2 KiB apart
      const uint64_t av0 = tc::sdesc(sbase + kStVc, 16384, 1024);
      const uint64_t bp0 = sdesc_plain(sbase + kSmP, 128, 2048);
      bool ok = true;
      int os = 0;  // stage of O^T(jo)
      for (int jo = 0; jo < nu && ok; ++jo) {
        if (!(ok = tc::wait_bar(bar(kBarPFull + (jo & 3)), (jo >> 2) & 1, p.status, abort_flag))) break;
        tc::fence_after();
        const uint64_t av = av0 + os * (kStage >> 4);
        const uint64_t bp = bp0 + (jo & 3) * (kPBuf >> 4);
        const uint32_t d = tmem + 2 * C::kS + (jo & 3) * C::kO;
#pragma unroll
        for (int k = 0; k < 4; ++k)  // 32 tokens per step
          mma_e4m3(d, av + k * (4096 >> 4), bp + k * (512 >> 4), kIdO, k > 0 ? 1u : 0u);
        tc::commit(bar(kBarOFull + (jo & 3)));
        tc::commit(bar(kBarEmpty + os));  // the stage is no longer read
        if (++os == kStages) os = 0;
      }
      tc::commit(bar(kBarDrain + 1));
      mbar_wait(bar(kBarDrain + 1), 0, p.status);
    }
  } else if (warp >= 4) {
    // ================= softmax warpgroups (warps 4-11) =================
    // Group g takes the tiles j with j % 2 == g.  The running max m is raised to the
    // tile's max only when a logit exceeds m + kSlack (log2 units), so p <= 2^kSlack; the
    // MMA gets P' = p s_v 2^6 / smax as three E4M3 limbs.  When an item ends the two
    // groups' states are combined (group 0 writes the result).
    const int grp = (warp - 4) >> 2;
    const int gbar = 1 + grp;  // the group's named barrier; barrier 3 joins both groups
    const int wq = warp & 3;
    const int t = (wq << 5) | lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq << 5) << 16);
    float *gred = red + grp * 64;                                           // [4 warps][16]
    float *vmx = reinterpret_cast<float *>(smem + kSmVmax) + grp * 8;      // [2][4 warps]
    const float c = p.scale_log2;
    float m[NQ], l[NQ], o[NQ], sg[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      m[q] = -INFINITY;
      l[q] = 0.f;
      o[q] = 0.f;
      sg[q] = 0.f;
    }
    bool ok = true, qread = true;  // qread: this group has read (or released) the item's 2^-e_q
    int cur_item = -1, nitem = -1;
    int jp = -1;            // this group's last tile, its O^T still to be folded
    float sigp_prev = 0.f;  // smax 2^-6 of tile jp

    // Both groups arrive here when an item ends, every tile of it folded.  Group 1 hands
    // its state over; group 0 combines the two, writes this CTA's result for `item`
    // (partial or final) and merges when last.
    auto flush = [&](int item, bool final_flush) {
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        const float vl = warp_sum(l[q]);
        if (lane == 0) gred[wq * 16 + q] = vl;
      }
      float *xo = reinterpret_cast<float *>(smem + kSmP);  // [16][128] o of group 1, then its m[16]
      tc::named_sync(3, 256);  // no P' buffer is in use: every product of the item has been folded
      if (grp == 1) {
#pragma unroll
        for (int q = 0; q < NQ; ++q) xo[q * 128 + t] = o[q];
        if (t == 0) {
#pragma unroll
          for (int q = 0; q < NQ; ++q) xo[16 * 128 + q] = m[q];
        }
      }
      tc::named_sync(3, 256);
      if (grp == 1) {
        tc::named_sync(3, 256);  // group 0 has read the hand-over
        return;
      }
      float lt[NQ];
      const float *r1 = red + 64;
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        const float l0 = gred[q] + gred[16 + q] + gred[32 + q] + gred[48 + q];
        const float l1 = r1[q] + r1[16 + q] + r1[32 + q] + r1[48 + q];
        const float m1 = xo[16 * 128 + q];
        const float mn = fmaxf(m[q], m1);
        const float a0 = m[q] == -INFINITY ? 0.f : ex2(m[q] - mn);
        const float a1 = m1 == -INFINITY ? 0.f : ex2(m1 - mn);
        lt[q] = fmaf(l0, a0, l1 * a1);
        o[q] = fmaf(o[q], a0, xo[q * 128 + t] * a1);
        m[q] = mn;
      }
      tc::named_sync(3, 256);  // release group 1: the hand-over is read
      const int64_t ia = static_cast<int64_t>(item) * a.units_r;
      const int cfirst = cta_of(a, ia), clast = cta_of(a, ia + a.units_r - 1);
      const int nseg = clast - cfirst + 1;
      const int b = item / p.Hr;
      const int g = p.hm.retr_head[item % p.Hr];
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
      float *part = p.partials + (pitem * p.max_splits) * G * kPartRow;
#pragma unroll
      for (int q = 0; q < NQ; ++q)
        if (q < G) {
          float *dst = part + (static_cast<int64_t>(seg) * G + q) * kPartRow;
          dst[t] = o[q];
          if (t == 0) {
            dst[kD] = m[q];
            dst[kD + 1] = lt[q];
          }
        }
      __threadfence();
      tc::named_sync(gbar, 128);
      // at the CTA's last item the code stages are idle (every load consumed, every
      // product run): the merging CTA copies the item's partial rows in with one bulk
      // copy and merges from shared memory (1: merge from global memory, 2: from here)
      const uint32_t bytes = static_cast<uint32_t>(nseg) * G * kPartRow * 4;
      if (t == 0) {
        const uint32_t prev = atomicAdd(p.counters + pitem, 1u);
        const bool here = final_flush && bytes <= static_cast<uint32_t>(kSmQl) && *abort_flag == 0;
        *last_flag = (prev == static_cast<uint32_t>(nseg - 1)) ? (here ? 2 : 1) : 0;
      }
      tc::named_sync(gbar, 128);
      const int how = *last_flag;
      if (!how) return;
      __threadfence();
      if (how == 2) {
        if (t == 0) {
          asm volatile("fence.proxy.async.global;" ::: "memory");  // the rows were written by other CTAs
          mbar_expect_tx(bar(kBarMerge), bytes);
          bulk_g2s(sbase, part, bytes, bar(kBarMerge));
        }
        // waited for even after an abort (bounded): the copy must not outlive the CTA
        if (!mbar_wait(bar(kBarMerge), 0, p.status)) ok = false;
        merge_partials<true>(reinterpret_cast<const float *>(smem), nseg, G, b, h0, p.Hq, p.out, p.lse, red + 128, t,
                             gbar);
      } else {
        merge_partials(part, nseg, G, b, h0, p.Hq, p.out, p.lse, red + 128, t, gbar);
      }
      if (t == 0) p.counters[pitem] = 0u;  // ready for the next call
    };

    // o = (o + sigp O^T(jj)) * alpha for this thread's dimension, in two halves: the
    // load of O^T(jj) is issued at the start of the group's next tile (its product has
    // long run) and the limbs are added once that tile's alpha is known
    uint32_t orow[C::kO];
    auto fold_issue = [&](int jj) {
      if (ok) ok = tc::wait_bar(bar(kBarOFull + (jj & 3)), (jj >> 2) & 1, p.status, abort_flag);
      tc::fence_after();
      ld_issue<C::kO>(lane_base + 2 * C::kS + (jj & 3) * C::kO, orow);
    };
    auto fold_finish = [&](float sigp, const float (&alpha)[NQ]) {
      ld_wait<C::kO>(orow);
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        const float r = fmaf(fmaf(__uint_as_float(orow[2 * NQ + q]), 0.0625f, __uint_as_float(orow[NQ + q])), 0.0625f,
                             __uint_as_float(orow[q]));
        o[q] = fmaf(sigp, r, o[q]) * alpha[q];
      }
    };
    auto fold = [&](int jj, float sigp, const float (&alpha)[NQ]) {
      fold_issue(jj);
      fold_finish(sigp, alpha);
    };
    float one[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q) one[q] = 1.f;
    // the item's query information is released by a group that never reads it
    auto release_unread = [&]() {
      if (!qread && t == 0) mbar_arrive(bar(kBarQFree + (nitem & 1)));
      qread = true;
    };

    UnitIter it(a, u0);
    for (int j = 0; j < nu; ++j, it.next()) {
      const Unit un = it.un;
      if (un.item != cur_item) {
        if (cur_item >= 0) {
          if (jp >= 0) fold(jp, sigp_prev, one);
          jp = -1;
          release_unread();
          flush(cur_item, false);
        }
        ++nitem;
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          m[q] = -INFINITY;
          l[q] = 0.f;
          o[q] = 0.f;
        }
        qread = false;
        cur_item = un.item;
      }
      if ((j & 1) != grp) continue;  // the other group's tile
      const int s = j % kStages;
      if (ok) ok = tc::wait_bar(bar(kBarSFull + grp), (j >> 1) & 1, p.status, abort_flag);
      tc::fence_after();
      uint32_t sr[C::kS];
      ld_issue<C::kS>(lane_base + grp * C::kS, sr);
      ld_wait<C::kS>(sr);
      tc::fence_before();
      mbar_arrive_warp(bar(kBarSFree + grp));  // S buffer j % 2 is free again
      if (jp >= 0) fold_issue(jp);             // finished below, once alpha is known
      // the stage's scale rows have landed (waiting orders the copy before these reads)
      if (ok) ok = tc::wait_bar(bar(kBarFull + s), (j / kStages) & 1, p.status, abort_flag);
      const char *st = smem + s * kStage;
      const bool valid = static_cast<int64_t>(un.tile) * kTile + t < p.len;
      const float sk = valid ? reinterpret_cast<const float *>(st + kStKs)[t] : 0.f;
      const float svv = valid ? reinterpret_cast<const float *>(st + kStVs)[t] : 0.f;
      if (!qread) {  // this group's first tile of the item: its 2^-e_q
        if (ok) ok = tc::wait_bar(bar(kBarQInfo + (nitem & 1)), (nitem >> 1) & 1, p.status, abort_flag);
        const float *qi = reinterpret_cast<const float *>(smem + kSmQinfo) + (nitem & 1) * 16;
#pragma unroll
        for (int q = 0; q < NQ; ++q) sg[q] = qi[q];
        tc::named_sync(gbar, 128);
        if (t == 0) mbar_arrive(bar(kBarQFree + (nitem & 1)));
        qread = true;
      }
      // the tile's largest V scale: non-negative fp32 values order as their bit patterns
      const uint32_t wmax = __reduce_max_sync(0xffffffffu, __float_as_uint(svv));
      float *vslot = vmx + ((j >> 1) & 1) * 4;
      if (lane == 0) vslot[wq] = __uint_as_float(wmax);
      const float fk = sk * c;
      float sv[NQ];
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        const float r = fmaf(fmaf(__uint_as_float(sr[2 * NQ + q]), 0.0625f, __uint_as_float(sr[NQ + q])), 0.0625f,
                             __uint_as_float(sr[q]));
        sv[q] = r * sg[q] * fk;  // log2-domain logit
      }
      // does any logit of this tile exceed the group's running max by more than kSlack?
      int need = 0;
#pragma unroll
      for (int q = 0; q < NQ; ++q)
        if (q < G && valid && sv[q] > m[q] + kSlack) need = 1;
      need = tc::bar_or(gbar, 128, need);  // also orders the V-scale maxima written above
      const float smax = fmaxf(fmaxf(vslot[0], vslot[1]), fmaxf(vslot[2], vslot[3]));
      float alpha[NQ];
#pragma unroll
      for (int q = 0; q < NQ; ++q) alpha[q] = 1.f;
      if (need) {  // uniform over the warpgroup
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          const float x = warp_max((valid && q < G) ? sv[q] : -INFINITY);
          if (lane == 0) gred[wq * 16 + q] = x;
        }
        tc::named_sync(gbar, 128);
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          const float mt = fmaxf(fmaxf(gred[q], gred[16 + q]), fmaxf(gred[32 + q], gred[48 + q]));
          const float mn = fmaxf(m[q], mt);
          alpha[q] = (mn == -INFINITY) ? 1.f : ex2(m[q] - mn);
          m[q] = mn;
        }
        tc::named_sync(gbar, 128);  // gred is reused later
      }
      // P'^T limbs into buffer j % 4 (its previous reader, tile j-4 of this group, was
      // folded at tile j-2): x = p s_v 2^6 / smax <= 2^8 (1 + 2^-20)
      const float pf = smax > 0.f ? svv * __fdividef(64.f, smax) : 0.f;
      constexpr int kPB = 3 * NQ;  // limb bytes of this token: byte l NQ + q is limb l of head q
      uint32_t pw[(kPB + 3) / 4];
#pragma unroll
      for (int w = 0; w < (kPB + 3) / 4; ++w) pw[w] = 0u;
      float pv[NQ];
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        pv[q] = (valid && q < G && m[q] != -INFINITY) ? ex2(sv[q] - m[q]) : 0.f;
        l[q] = fmaf(l[q], alpha[q], pv[q]);
      }
      if constexpr (NQ >= 2) {
#pragma unroll
        for (int q = 0; q < NQ; q += 2) {  // heads q, q + 1: bytes l NQ + q, l NQ + q + 1 (q even)
          uint32_t w[3];
          limbs3(pv[q] * pf, pv[q + 1] * pf, w);
#pragma unroll
          for (int li = 0; li < 3; ++li) {
            const int n = li * NQ + q;
            pw[n >> 2] |= w[li] << (8 * (n & 3));
          }
        }
      } else {
        uint32_t w[3];
        limbs3(pv[0] * pf, 0.f, w);
        pw[0] = (w[0] & 0xFFu) | ((w[1] & 0xFFu) << 8) | ((w[2] & 0xFFu) << 16);
      }
      // P'^T is MN-major without swizzle: token t's limb bytes are contiguous, 16 per
      // 2 KiB block (byte (n, t) at (n / 16) * 2048 + 16 t + n % 16): one store per block
      char *pt = smem + kSmP + (j & 3) * kPBuf + 16 * t;
      if constexpr (kPB <= 4) {
        *reinterpret_cast<uint32_t *>(pt) = pw[0];
      } else if constexpr (kPB <= 8) {
        *reinterpret_cast<uint2 *>(pt) = make_uint2(pw[0], pw[1]);
      } else {
#pragma unroll
        for (int b = 0; b < (kPB + 15) / 16; ++b) {
          const uint32_t w0 = 4 * b < (kPB + 3) / 4 ? pw[4 * b] : 0u;
          const uint32_t w1 = 4 * b + 1 < (kPB + 3) / 4 ? pw[4 * b + 1] : 0u;
          const uint32_t w2 = 4 * b + 2 < (kPB + 3) / 4 ? pw[4 * b + 2] : 0u;
          const uint32_t w3 = 4 * b + 3 < (kPB + 3) / 4 ? pw[4 * b + 3] : 0u;
          *reinterpret_cast<uint4 *>(pt + 2048 * b) = make_uint4(w0, w1, w2, w3);
        }
      }
      tc::fence_async_smem();
      tc::fence_before();
      mbar_arrive_warp(bar(kBarPFull + (j & 3)));
      // fold this group's previous tile of the item, bringing it to this tile's scale
      if (jp >= 0) {
        fold_finish(sigp_prev, alpha);
      } else {
#pragma unroll
        for (int q = 0; q < NQ; ++q) o[q] *= alpha[q];
      }
      jp = j;
      sigp_prev = smax * (1.f / 64.f);
    }
    if (nu > 0) {
      if (jp >= 0) fold(jp, sigp_prev, one);
      release_unread();
      flush(cur_item, true);
    }
  }

  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  if (p.pdl_mode == 2 && tid == 0) asm volatile("griddepcontrol.wait;" ::: "memory");  // the leader has ended
  if (warp == 1) tc::tmem_free(tmem, C::kAlloc);
}

template <int NQ>
cudaError_t launch_nq(const Fp8DecodeArgs &a, bool overlap_previous, cudaStream_t st) {
  static std::atomic<uint64_t> attr{0};
  {
    const cudaError_t e = opt_in_smem(decode_fp8_kernel<NQ>, kSmemAlloc, attr);
    if (e != cudaSuccess) return e;
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
  const cudaError_t e = cudaLaunchKernelEx(&cfg, decode_fp8_kernel<NQ>, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

bool decode_fp8_tc_supported(const DecodeParams &p, duo_dtype dt) {
  return dt == DUO_BF16 && p.D == kD && p.G >= 1 && p.G <= 16 && tc::encode_fn() != nullptr;
}

cudaError_t launch_decode_fp8_tc(const DecodeParams &p, int num_sms, bool overlap_previous, cudaStream_t st) {
  if (p.Hr < 1 || p.len < 1) return cudaSuccess;  // no retrieval head: nothing to do here
  Fp8DecodeArgs a{};
  a.p = p;
  a.units_r = static_cast<int>((p.len + kTile - 1) / kTile);
  a.n_items = p.B * p.Hr;
  a.total_units = static_cast<int64_t>(a.n_items) * a.units_r;
  // at most one CTA per SM, and never more segments per item than partial slots
  int64_t ctas = num_sms;
  if (ctas > a.total_units) ctas = a.total_units;
  if (ctas > kMaxSplits) ctas = kMaxSplits;
  a.num_ctas = static_cast<int>(ctas);
  bool ok = true;
  {  // queries [B*Hq][d] bf16
    const uint64_t d[2] = {kD, static_cast<uint64_t>(p.B) * p.Hq};
    const uint64_t s[1] = {kD * 2};
    const uint32_t bx[2] = {64, 16};
    ok &= tc::make_map(&a.tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.q, 2, d, s, bx, CU_TENSOR_MAP_SWIZZLE_128B);
  }
  {  // retrieval codes [B*Hr][cap][128 B]
    const uint64_t d[3] = {kD, static_cast<uint64_t>(p.max_len), static_cast<uint64_t>(a.n_items)};
    const uint64_t s[2] = {kD, static_cast<uint64_t>(kD) * p.max_len};
    const uint32_t bx[3] = {kD, kTile, 1};
    ok &= tc::make_map(&a.tm_kc, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.rk, 3, d, s, bx, CU_TENSOR_MAP_SWIZZLE_128B);
    ok &= tc::make_map(&a.tm_vc, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.rv, 3, d, s, bx, CU_TENSOR_MAP_SWIZZLE_128B);
  }
  if (!ok) return cudaErrorInvalidValue;
  if (p.G <= 1) return launch_nq<1>(a, overlap_previous, st);
  if (p.G <= 2) return launch_nq<2>(a, overlap_previous, st);
  if (p.G <= 4) return launch_nq<4>(a, overlap_previous, st);
  if (p.G <= 8) return launch_nq<8>(a, overlap_previous, st);
  return launch_nq<16>(a, overlap_previous, st);
}

}  // namespace duo
