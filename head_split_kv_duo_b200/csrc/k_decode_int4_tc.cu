// k_decode_int4_tc.cu -- single-token decode attention over the retrieval heads when
// they keep K and V as 4-bit codes ("Combination with Quantization", Figure 12:
// DuoAttention with a 4-bit KV cache), on the tcgen05 integer tensor cores.  bf16
// queries, head_dim 128, up to 16 query heads per KV head.  The streaming heads (bf16)
// of such a layer run on the bf16 decode kernel.
//
// Operation ("Decoding Procedure", steps 2, 3 and 5) as in k_decode_tc.cu.  A stored
// element is c s + z (code c in 0..15, per-token fp16 scale s and zero z).  A token's
// 64 code bytes are read by the tensor core as they are stored: byte j is
// U_j = c_{2j} + 16 c_{2j+1} (kind::i8, unsigned); the only conversion is the low
// nibble L_j = c_{2j}, one AND per four bytes.  Then
//   sum_d q_d c_d = sum_j (q_{2j+1} / 16) U_j + (q_{2j} - q_{2j+1} / 16) L_j
// so S^T = [U | L] . Qx^T over K = 128 bytes, with Qx the two coefficient rows above,
// and for the output (dimension pair j of one query head)
//   sum_t p'_t L_tj = O_{2j},  sum_t p'_t U_tj = O_{2j} + 16 O_{2j+1}
// so O^T = [U_V | L_V]^T . P'^T (M = 128: 64 byte rows, 64 low-nibble rows).  The fp32
// operands Qx and P' = p s_v enter as signed 8-bit limbs with a scale: Qx per query
// head as three limbs (21 bits below the row's largest coefficient), P' per tile as two
// (15 bits below the tile's largest s_v, which bounds p s_v since INT4 items keep the
// running max exact, p <= 1).  The int32 accumulators are exact; the limbs are split
// and recombined in fp32 by exact magic-number adds (no conversion instructions).  Per
// token the scale and zero then give
//   q . k_t = s_t (q . c_t) + z_t sum(q),   sum_t p_t v_t = sum_t p'_t c_t + sum_t p_t z_t.
//
// Roles of a CTA (one per SM, 480 threads):
//   warp 0     TMA producer: per 128-token tile the K and V code rows (64 B each,
//              64-byte swizzle) and their scale/zero rows, at an item's first tile the
//              group's bf16 queries; a ring of kStages stages.
//   warp 1     TMEM owner and S^T issuer (4 MMAs per tile; the K low nibbles are read
//              from tensor memory); warp 14 issues O^T (4 MMAs per tile).
//   warps 2-9  softmax, two warpgroups taking alternate tiles (each with its own running
//              max and sums, combined when an item ends), so that the dependent chain
//              of one tile overlaps the next: thread t owns token t of S^T and row t of
//              O^T.
//   warps 10-13 prep: a thread writes the low nibbles of token t's K row into TMEM lane
//              t and those of its V row beside the V codes, and the token's {s_k, z_k,
//              s_v, z_v}; warp 10 also turns an item's queries into limbs.
//
// Work balance: every (batch, retrieval head) is an item of 128-token tiles; the tiles
// of all items are laid end to end and cut into one equal range per CTA.  Split partials
// are merged by the last CTA of each item, as in the bf16 kernel.
#include "decode_merge.cuh"
#include "tcgen05.cuh"

namespace duo {

namespace {

constexpr int kThreads = 480;
constexpr int kTile = 128;
constexpr int kD = 128;
constexpr int kStages = 6;
constexpr int kPrefetch = 4;  // tiles asked of L2 before the previous grid has finished
// stage: K and V codes [128][64 B] (64-byte swizzle, as the TMA writes them), the V low
// nibbles in the same layout, the scale/zero rows [128][4 B], per token {s_k, z_k, s_v,
// z_v}, per prep warp the largest s_v, at an item's first tile the queries [16][128]
// bf16 (two 128-byte-swizzled atoms)
constexpr int kStKc = 0, kStVc = 8192, kStLv = 16384, kStKsz = 24576, kStVsz = 25088, kStMisc = 25600,
              kStTmax = 27648, kStQ = 28672, kStage = 32768;
constexpr int kQlBytes = 6144;                 // query limbs [48][128 B] s8, 128-byte swizzle
constexpr int kSmQl = kStages * kStage;        // 2 x query limbs (item parity)
constexpr int kSmP = kSmQl + 2 * kQlBytes;     // 4 x P'^T limbs (MN-major, 4 KiB each); flush exchanges
constexpr int kSmQinfo = kSmP + 4 * 4096;      // [2][32]: sigma[16], sum(q)[16] per query head
constexpr int kSmRed = kSmQinfo + 256;         // per softmax group [4][16] l, [4][16] zc; [128][6] merge
constexpr int kSmBar = kSmRed + (2 * 128 + 128 * 6) * 4;
constexpr int kSmMisc = kSmBar + 512;
constexpr int kSmemAlloc = kSmMisc + 64 + 1024;
static_assert(kStage % 1024 == 0 && kStQ % 1024 == 0 && kSmQl % 1024 == 0 && kSmP % 1024 == 0 &&
                  kQlBytes % 1024 == 0, "alignment");
static_assert(kSmemAlloc <= 232448, "shared memory");

// P' and O^T have four buffers each, and so four barriers: with two groups a group
// publishes P'(j + 2) before the issuer need have taken P'(j), so a barrier per
// buffer pair would complete a second phase ahead of its waiter
constexpr int kBarFull = 0, kBarEmpty = kStages, kBarCvt = 2 * kStages, kBarSFull = 3 * kStages,
              kBarSFree = kBarSFull + 2, kBarPFull = kBarSFull + 4, kBarOFull = kBarSFull + 8,
              kBarQFree = kBarSFull + 12, kBarDrain = kBarSFull + 14,
              kNumBars = kBarSFull + 16;  // a drain barrier per issuer
static_assert(kNumBars * 8 <= 512, "barrier area");

// tensor memory columns: S^T (three limbs per query head) x 2, O^T (two limbs) x 4, and
// per stage the K low nibbles (16 columns: 4 bytes each)
template <int NQ>
struct Cols {
  static constexpr int kS = (3 * NQ + 15) / 16 * 16;
  static constexpr int kO = (2 * NQ + 15) / 16 * 16;
  static constexpr int kLk = 2 * kS + 4 * kO;
  static constexpr int kUsed = kLk + kStages * 16;
  static constexpr int kAlloc = kUsed <= 128 ? 128 : kUsed <= 256 ? 256 : 512;
};

struct Int4DecodeArgs {
  DecodeParams p;
  int units_r;          // tiles per item
  int n_items;          // B * Hr
  int64_t total_units;  // n_items * units_r
  int num_ctas;
  CUtensorMap tm_q, tm_kc, tm_vc;
};

// shared-memory matrix descriptor with an explicit layout (2: 128-byte swizzle, 4: 64-byte)
__device__ __forceinline__ uint64_t sdesc_l(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (static_cast<uint64_t>(layout) << 61);
}
// kind::i8 instruction descriptor: int32 accumulator, A unsigned, B signed or unsigned
constexpr uint32_t idesc_i8(int M, int N, bool b_signed, bool a_mn_major, bool b_mn_major = false) {
  return (2u << 4) | ((b_signed ? 1u : 0u) << 10) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         ((static_cast<uint32_t>(N) >> 3) << 17) | ((static_cast<uint32_t>(M) >> 4) << 24);
}
__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(acc)
      : "memory");
}
// same with A read from tensor memory (lane = row, one column = 4 consecutive K bytes)
__device__ __forceinline__ void mma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(acc)
      : "memory");
}
// Exact int <-> float for |x| < 2^22 on the ALU and FMA pipes: 1.5 * 2^23 has unit
// mantissa steps, so x + 1.5 * 2^23 holds x in its low mantissa bits.
constexpr float kMagic = 12582912.0f;
constexpr int kMagicBits = 0x4B400000;
__device__ __forceinline__ float to_float(int x) { return __int_as_float(x + kMagicBits) - kMagic; }  // exact
// x rounded to the nearest integer: its low byte (two's complement) and its value
__device__ __forceinline__ uint32_t round_byte(float x, float &rounded) {
  const float t = x + kMagic;
  rounded = t - kMagic;
  return static_cast<uint32_t>(__float_as_int(t)) & 0xFFu;
}
// N (a multiple of 16) int32 columns of this thread's TMEM lane
template <int N>
__device__ __forceinline__ void ld_i32(uint32_t taddr, int (&v)[N]) {
#pragma unroll
  for (int c = 0; c < N; c += 16) {
    float f[16];
    tc::ld<16>(taddr + c, f);
#pragma unroll
    for (int i = 0; i < 16; ++i) v[c + i] = __float_as_int(f[i]);
  }
}
// N (a multiple of 16) int32 columns of this thread's TMEM lane, loads issued only:
// ld_i32_wait names every destination register, so that no use precedes the wait
template <int N>
__device__ __forceinline__ void ld_i32_issue(uint32_t taddr, uint32_t (&r)[N]) {
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
__device__ __forceinline__ void ld_i32_wait(uint32_t (&r)[N]) {
  static_assert(N == 16 || N == 32, "16 or 32 columns");
  if constexpr (N == 16) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
                 :
                 : "memory");
  } else {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]),
                   "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]),
                   "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
                   "+r"(r[30]), "+r"(r[31])
                 :
                 : "memory");
  }
}
// byte (row n, column k) of a [rows][128 B] K-major operand with 128-byte swizzle
__device__ __forceinline__ int sw128(int n, int k) { return (n >> 3) * 1024 + (n & 7) * 128 + (((k >> 4) ^ (n & 7)) << 4) + (k & 15); }

struct Unit {
  int item, tile;
};
// Walks a CTA's units in order without a division per step.
struct UnitIter {
  Unit un;
  int units;
  __device__ __forceinline__ UnitIter(const Int4DecodeArgs &a, int64_t u)
      : un{static_cast<int>(u / a.units_r), static_cast<int>(u % a.units_r)}, units(a.units_r) {}
  __device__ __forceinline__ void next() {
    if (++un.tile == units) {
      ++un.item;
      un.tile = 0;
    }
  }
};
__device__ __forceinline__ int64_t cta_begin(const Int4DecodeArgs &a, int c) {
  return static_cast<int64_t>(c) * a.total_units / a.num_ctas;
}
__device__ __forceinline__ int cta_of(const Int4DecodeArgs &a, int64_t u) {
  return static_cast<int>(((u + 1) * a.num_ctas + a.total_units - 1) / a.total_units) - 1;
}

// One warp turns the G query rows of an item (bf16 [16][128], two 128-byte-swizzled
// atoms) into the B operand of S^T: row 3q + l holds limb l of query head q's
// coefficients, columns 0..63 those of U (q_{2j+1} / 16), 64..127 those of L
// (q_{2j} - q_{2j+1} / 16).  Also writes sigma (coefficient = sigma * (l0 + l1 / 2^7 +
// l2 / 2^14)) and sum(q) of every head.
__device__ __forceinline__ void prep_queries(const char *qr, char *ql, float *qinfo, int G, int lane) {
  for (int q = 0; q < G; ++q) {
    float cu[2], cl[2], qs = 0.f;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int j = lane + 32 * h, c = 2 * j;  // columns c, c + 1 of atom h
      const int off = h * 2048 + q * 128 + ((((c & 63) >> 3) ^ (q & 7)) << 4) + (c & 7) * 2;
      const uint32_t w = *reinterpret_cast<const uint32_t *>(qr + off);
      const float e = bf16lo(w), o = bf16hi(w);
      cu[h] = o * 0.0625f;
      cl[h] = e - cu[h];
      qs += e + o;
    }
    const float amax = warp_max(fmaxf(fmaxf(fabsf(cu[0]), fabsf(cu[1])), fmaxf(fabsf(cl[0]), fabsf(cl[1]))));
    qs = warp_sum(qs);
    const float inv = amax > 0.f ? 127.f / amax : 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float x = (i < 2 ? cu[i] : cl[i - 2]) * inv;
      const int k = (i < 2 ? 0 : 64) + lane + 32 * (i & 1);
      const float l0 = rintf(x);
      const float r1 = (x - l0) * 128.f;
      const float l1 = rintf(r1);
      const float l2 = rintf((r1 - l1) * 128.f);
      ql[sw128(3 * q, k)] = static_cast<char>(static_cast<int>(l0));
      ql[sw128(3 * q + 1, k)] = static_cast<char>(static_cast<int>(l1));
      ql[sw128(3 * q + 2, k)] = static_cast<char>(static_cast<int>(l2));
    }
    if (lane == 0) {
      qinfo[q] = amax * (1.f / 127.f);
      qinfo[16 + q] = qs;
    }
  }
}

template <int NQ>
__global__ void __launch_bounds__(kThreads, 1) decode_int4_kernel(const __grid_constant__ Int4DecodeArgs a) {
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
      mbar_init(bar(kBarCvt + i), 4);   // one arrival per prep warp
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(kBarSFull + i), 1);
      mbar_init(bar(kBarSFree + i), 4);  // one arrival per warp of a softmax group
      mbar_init(bar(kBarQFree + i), 3);  // the item's last S^T product (commit) + each softmax group
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(bar(kBarPFull + i), 4);  // one arrival per warp of a softmax group
      mbar_init(bar(kBarOFull + i), 1);
    }
    mbar_init(bar(kBarDrain), 1);
    mbar_init(bar(kBarDrain + 1), 1);
    fence_mbar_init();
    *abort_flag = 0;
  }
  if (warp == 1) tc::tmem_alloc(smem_u32(tmem_slot), C::kAlloc);
  tc::fence_async_smem();
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ================= TMA producer =================
    if (lane == 0) {
      for (const CUtensorMap *m : {&a.tm_q, &a.tm_kc, &a.tm_vc})
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
      {  // L2 prefetch of the first tiles; no data is consumed before the wait below
        UnitIter it(a, u0);
        for (int j = 0; j < nu && j < kPrefetch; ++j, it.next()) {
          const int64_t row = static_cast<int64_t>(it.un.item) * p.max_len + static_cast<int64_t>(it.un.tile) * kTile;
          prefetch_l2(p.rk + row * (kD / 2), kTile * kD / 2);
          prefetch_l2(p.rv + row * (kD / 2), kTile * kD / 2);
          prefetch_l2(p.rk_sz + row * 4, kTile * 4);
          prefetch_l2(p.rv_sz + row * 4, kTile * 4);
        }
      }
      // Launched as a programmatic dependent, this grid's set-up overlaps the previous
      // kernel on the stream; nothing is read from global memory before that kernel has
      // finished (every other read and every write of this grid follows these loads).
      if (p.pdl_mode != 2) asm volatile("griddepcontrol.wait;" ::: "memory");  // (beside a leader: implied)
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
        mbar_expect_tx(fb, 2 * 8192 + 2 * 512 + (first ? 4096 : 0));
        const int y = un.tile * kTile;
        const int z = un.item;  // = b * Hr + retrieval index
        tc::tma_3d(dst + kStKc, &a.tm_kc, 0, y, z, fb);
        tc::tma_3d(dst + kStVc, &a.tm_vc, 0, y, z, fb);
        const int64_t row = static_cast<int64_t>(z) * p.max_len + y;
        bulk_g2s(dst + kStKsz, p.rk_sz + row * 4, 512, fb);
        bulk_g2s(dst + kStVsz, p.rv_sz + row * 4, 512, fb);
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
  } else if (warp == 1 || warp == 14) {
    // ================= MMA issuers: S^T on warp 1, O^T on warp 14 =================
    // Warp 1 issues S^T(j) once the prep of tile j is done and the softmax has read
    // S^T(j - 2) (its buffer); warp 14 issues O^T(j) once P'(j) is written.  A barrier
    // wait and an MMA issue each cost a thread hundreds of cycles on a loaded SM, and a
    // thread issuing dependent instructions sets the pace of the pipeline: two issuers,
    // each with little per-tile work (descriptors as a base plus a constant, stage and
    // phase as running counters), keep S^T ahead of the softmax.  tcgen05.commit tracks
    // the committing thread's own MMAs; the stage is released after O^T(j), and S^T(j)
    // has completed by then (the softmax saw it land before writing P'(j)).
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_i8(128, C::kS, true, false);   // [U | L] . Qx^T
      constexpr uint32_t kIdO = idesc_i8(128, C::kO, true, true, true);  // [U_V | L_V]^T . P'^T (both MN-major)
      constexpr uint32_t kStDesc = kStage >> 4;                       // one stage in descriptor units
      bool ok = true;
      if (warp == 1) {
        const uint64_t ak0 = sdesc_l(sbase + kStKc, 16, 512, 4);
        const uint64_t bq0 = sdesc_l(sbase + kSmQl, 16, 1024, 2);
        int nitem = -1, prev_item = -1;
        UnitIter its(a, u0);
        int ss = 0, sph = 0;  // stage of S^T(js) and the phase of its prep barrier
        auto issue_s = [&](int js) {  // S^T(js), its prep done and its S buffer read
          const int item = its.un.item;
          its.next();
          if (item != prev_item) {
            prev_item = item;
            ++nitem;
          }
          tc::fence_after();
          const uint64_t ak = ak0 + ss * kStDesc;
          const uint64_t bq = bq0 + (nitem & 1) * (kQlBytes >> 4);
          const uint32_t al = tmem + C::kLk + ss * 16;
          const uint32_t d = tmem + (js & 1) * C::kS;
          mma_i8(d, ak, bq, kIdS, 0u);             // bytes 0..31 of the code rows
          mma_i8(d, ak + 2, bq + 2, kIdS, 1u);     // bytes 32..63
          mma_i8_ts(d, al, bq + 4, kIdS, 1u);      // low nibbles 0..31 (TMEM)
          mma_i8_ts(d, al + 8, bq + 6, kIdS, 1u);  // low nibbles 32..63
          tc::commit(bar(kBarSFull + (js & 1)));
          // the item's query limbs are free once its last S^T product has run
          if (js + 1 == nu || its.un.item != item) tc::commit(bar(kBarQFree + (nitem & 1)));
          if (++ss == kStages) {
            ss = 0;
            sph ^= 1;
          }
        };
        for (int js = 0; js < nu && ok; ++js) {
          ok = tc::wait_bar(bar(kBarCvt + ss), sph, p.status, abort_flag) &&
               (js < 2 || tc::wait_bar(bar(kBarSFree + (js & 1)), ((js - 2) >> 1) & 1, p.status, abort_flag));
          if (ok) issue_s(js);
        }
      } else {
        const uint64_t av0 = sdesc_l(sbase + kStVc, kStLv - kStVc, 512, 4);  // MN-major, 2 chunks
        // P'^T MN-major without swizzle: 16 limb bytes of a token per row, 8 tokens per
        // 128-byte core matrix (the leading byte offset steps along the tokens), blocks of
        // 16 limb rows 2 KiB apart
        const uint64_t bp0 = sdesc_l(sbase + kSmP, 128, 2048, 0);
        int os = 0;  // stage of O^T(jo)
        for (int jo = 0; jo < nu && ok; ++jo) {
          if (!(ok = tc::wait_bar(bar(kBarPFull + (jo & 3)), (jo >> 2) & 1, p.status, abort_flag))) break;
          tc::fence_after();
          const uint64_t av = av0 + os * kStDesc;
          const uint64_t bp = bp0 + (jo & 3) * (4096 >> 4);
          const uint32_t d = tmem + 2 * C::kS + (jo & 3) * C::kO;
#pragma unroll
          for (int k = 0; k < 4; ++k)  // 32 tokens per step
            mma_i8(d, av + k * (2048 >> 4), bp + k * (512 >> 4), kIdO, k > 0 ? 1u : 0u);
          tc::commit(bar(kBarOFull + (jo & 3)));
          tc::commit(bar(kBarEmpty + os));  // the stage and its K low nibbles are no longer read
          if (++os == kStages) os = 0;
        }
      }
      // drain: every MMA this thread issued has completed before TMEM is freed
      const uint32_t drain = bar(kBarDrain + (warp == 1 ? 0 : 1));
      tc::commit(drain);
      mbar_wait(drain, 0, p.status);
    }
  } else if (warp < 10) {
    // ================= softmax warpgroups =================
    // Group g takes the tiles j with j % 2 == g.  Exact running max (p <= 1, which bounds
    // the P' limbs); s = s_k (q . c) + z_k sum(q); the MMA gets P' = p s_v as two signed
    // limbs below the tile's largest s_v; zc accumulates p z_v.  When an item ends the two
    // groups' states are combined (group 0 writes the result).
    const int grp = (warp - 2) >> 2;
    const int gbar = 1 + grp;  // the group's named barrier; barrier 3 joins both groups
    const int wq = warp & 3;
    const int t = (wq << 5) | lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq << 5) << 16);
    float *gred = red + grp * 128;  // [4 warps][16] l (or maxima), [4][16] zc
    const float c = p.scale_log2;
    float m[NQ], l[NQ], zc[NQ], o[NQ], sg[NQ], qs[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      m[q] = -INFINITY;
      l[q] = 0.f;
      zc[q] = 0.f;
      o[q] = 0.f;
      sg[q] = 0.f;
      qs[q] = 0.f;
    }
    bool ok = true, qread = true;  // qread: this group has read (or released) the item's sigma, sum(q)
    int cur_item = -1, nitem = -1;
    int jp = -1;            // this group's last tile, its O^T still to be folded
    float sigp_prev = 0.f;  // P' limb scale of tile jp

    // Both groups arrive here when an item ends, every tile of it folded.  Group 1 hands
    // its state over; group 0 combines the two, writes this CTA's result for `item`
    // (partial or final) and merges when last.  Thread t < 64 of group 0 ends with
    // dimensions 2t, 2t + 1 of every head: its lane summed the code bytes of pair t,
    // lane 64 + t the low nibbles.
    auto flush = [&](int item) {
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        const float vl = warp_sum(l[q]);
        const float vz = warp_sum(zc[q]);
        if (lane == 0) {
          gred[wq * 16 + q] = vl;
          gred[64 + wq * 16 + q] = vz;
        }
      }
      float *xo = reinterpret_cast<float *>(smem + kSmP);  // [16][128] o of group 1, then its m[16]
      float *xch = xo + 16 * 128 + 16;                     // [16][64] low-nibble sums
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
        tc::named_sync(3, 256);  // group 0 has read the hand-over and the exchange area
        return;
      }
      float lt[NQ], zt[NQ];
      const float *r1 = red + 128;
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        const float l0 = gred[q] + gred[16 + q] + gred[32 + q] + gred[48 + q];
        const float z0 = gred[64 + q] + gred[80 + q] + gred[96 + q] + gred[112 + q];
        const float l1 = r1[q] + r1[16 + q] + r1[32 + q] + r1[48 + q];
        const float z1 = r1[64 + q] + r1[80 + q] + r1[96 + q] + r1[112 + q];
        const float m1 = xo[16 * 128 + q];
        const float mn = fmaxf(m[q], m1);
        const float a0 = m[q] == -INFINITY ? 0.f : ex2(m[q] - mn);
        const float a1 = m1 == -INFINITY ? 0.f : ex2(m1 - mn);
        lt[q] = fmaf(l0, a0, l1 * a1);
        zt[q] = fmaf(z0, a0, z1 * a1);
        o[q] = fmaf(o[q], a0, xo[q * 128 + t] * a1);
        m[q] = mn;
      }
      if (t >= 64) {
#pragma unroll
        for (int q = 0; q < NQ; ++q)
          if (q < G) xch[q * 64 + (t - 64)] = o[q];
      }
      tc::named_sync(gbar, 128);
      float ev[NQ], od[NQ];
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        const float lo = t < 64 && q < G ? xch[q * 64 + t] : 0.f;
        ev[q] = lo + zt[q];
        od[q] = (o[q] - lo) * 0.0625f + zt[q];
      }
      tc::named_sync(3, 256);  // release group 1: the shared-memory areas are read
      const int units = a.units_r;
      const int64_t ia = static_cast<int64_t>(item) * units;
      const int cfirst = cta_of(a, ia), clast = cta_of(a, ia + units - 1);
      const int nseg = clast - cfirst + 1;
      const int b = item / p.Hr;
      const int g = p.hm.retr_head[item % p.Hr];
      const int h0 = g * G;
      if (nseg == 1) {
        if (t < 64) {
#pragma unroll
          for (int q = 0; q < NQ; ++q)
            if (q < G) {
              const float inv = 1.f / lt[q];
              const __nv_bfloat162 pr = __floats2bfloat162_rn(ev[q] * inv, od[q] * inv);
              *reinterpret_cast<__nv_bfloat162 *>(p.out + ((static_cast<int64_t>(b) * p.Hq + h0 + q) * kD + 2 * t) * 2) = pr;
              if (t == 0 && p.lse) p.lse[b * p.Hq + h0 + q] = (m[q] + lg2(lt[q])) * kLn2;
            }
        }
        return;
      }
      const int seg = blockIdx.x - cfirst;
      const int64_t pitem = static_cast<int64_t>(b) * p.Hkv + g;
      float *part = p.partials + (pitem * p.max_splits) * G * kPartRow;
      if (t < 64) {
#pragma unroll
        for (int q = 0; q < NQ; ++q)
          if (q < G) {
            float *dst = part + (static_cast<int64_t>(seg) * G + q) * kPartRow;
            *reinterpret_cast<float2 *>(dst + 2 * t) = make_float2(ev[q], od[q]);
            if (t == 0) {
              dst[kD] = m[q];
              dst[kD + 1] = lt[q];
            }
          }
      }
      __threadfence();
      tc::named_sync(gbar, 128);
      if (t == 0) {
        const uint32_t prev = atomicAdd(p.counters + pitem, 1u);
        *last_flag = (prev == static_cast<uint32_t>(nseg - 1)) ? 1 : 0;
      }
      tc::named_sync(gbar, 128);
      if (!*last_flag) return;
      __threadfence();
      merge_partials(part, nseg, G, b, h0, p.Hq, p.out, p.lse, red + 256, t, gbar);
      if (t == 0) p.counters[pitem] = 0u;  // ready for the next call
    };

    // o = (o + O^T(jj)) * alpha for this thread's row of O^T, in two halves: the load of
    // O^T(jj) is issued at the start of the group's next tile (its product has long run)
    // and the rows are added once that tile's alpha is known, so that the load's
    // latency overlaps the tile's arithmetic
    uint32_t orow[C::kO];
    auto fold_issue = [&](int jj) {
      if (ok) ok = tc::wait_bar(bar(kBarOFull + (jj & 3)), (jj >> 2) & 1, p.status, abort_flag);
      tc::fence_after();
      ld_i32_issue<C::kO>(lane_base + 2 * C::kS + (jj & 3) * C::kO, orow);
    };
    auto fold_finish = [&](float sigp, const float (&alpha)[NQ]) {
      ld_i32_wait<C::kO>(orow);
#pragma unroll
      for (int q = 0; q < NQ; ++q)  // |R| < 2^22
        o[q] = fmaf(sigp, fmaf(to_float(static_cast<int>(orow[2 * q + 1])), 1.f / 254.f,
                               to_float(static_cast<int>(orow[2 * q]))), o[q]) * alpha[q];
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
          flush(cur_item);
        }
        ++nitem;
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          m[q] = -INFINITY;
          l[q] = 0.f;
          zc[q] = 0.f;
          o[q] = 0.f;
        }
        qread = false;
        cur_item = un.item;
      }
      if ((j & 1) != grp) continue;  // the other group's tile
      const int cb = grp, s = j % kStages;
      if (ok) ok = tc::wait_bar(bar(kBarSFull + cb), (j >> 1) & 1, p.status, abort_flag);
      tc::fence_after();
      int sr[C::kS];
      ld_i32<C::kS>(lane_base + cb * C::kS, sr);
      tc::fence_before();
      mbar_arrive_warp(bar(kBarSFree + cb));  // S buffer j % 2 is free again
      if (jp >= 0) fold_issue(jp);  // finished below, once alpha is known
      // the stage's prep is complete (its S^T product has run); waiting here orders the
      // prep warps' writes before these reads
      if (ok) ok = tc::wait_bar(bar(kBarCvt + s), (j / kStages) & 1, p.status, abort_flag);
      const char *st = smem + s * kStage;
      const float4 mi = *reinterpret_cast<const float4 *>(st + kStMisc + t * 16);  // s_k, z_k, s_v, z_v
      const float4 tm4 = *reinterpret_cast<const float4 *>(st + kStTmax);
      const float tmax = fmaxf(fmaxf(tm4.x, tm4.y), fmaxf(tm4.z, tm4.w));
      const bool valid = static_cast<int64_t>(un.tile) * kTile + t < p.len;
      if (!qread) {  // this group's first tile of the item: its sigma and sum(q)
        const float *qi = reinterpret_cast<const float *>(smem + kSmQinfo) + (nitem & 1) * 32;
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          sg[q] = qi[q];
          qs[q] = qi[16 + q];
        }
        tc::named_sync(gbar, 128);
        if (t == 0) mbar_arrive(bar(kBarQFree + (nitem & 1)));
        qread = true;
      }
      float sv[NQ];
      if constexpr (NQ >= 2) {
        // two heads per packed fp32 instruction; the same roundings as one head at a time
        const uint64_t nmag = pack2(-kMagic, -kMagic), r128 = pack2(1.f / 128.f, 1.f / 128.f);
        const uint64_t kx = pack2(mi.x, mi.x), ky = pack2(mi.y, mi.y);
        auto limbs = [&](int i, int q) {  // exact int -> float of limb i of heads q, q + 1
          return fadd2(pack2(__int_as_float(sr[3 * q + i] + kMagicBits), __int_as_float(sr[3 * q + 3 + i] + kMagicBits)),
                       nmag);
        };
#pragma unroll
        for (int q = 0; q < NQ; q += 2) {  // S0 + S1 / 2^7 + S2 / 2^14, |S| < 2^22
          const uint64_t x = ffma2(ffma2(limbs(2, q), r128, limbs(1, q)), r128, limbs(0, q));
          const uint64_t v = ffma2(kx, fmul2(pack2(sg[q], sg[q + 1]), x), fmul2(ky, pack2(qs[q], qs[q + 1])));
          unpack2(v, sv[q], sv[q + 1]);
        }
      } else {
        const float x = fmaf(fmaf(to_float(sr[2]), 1.f / 128.f, to_float(sr[1])), 1.f / 128.f, to_float(sr[0]));
        sv[0] = fmaf(mi.x, sg[0] * x, mi.y * qs[0]);
      }
      // does any logit of this tile exceed the group's running max?
      int need = 0;
#pragma unroll
      for (int q = 0; q < NQ; ++q)
        if (q < G && valid && sv[q] * c > m[q]) need = 1;
      need = tc::bar_or(gbar, 128, need);
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
          const float mt = fmaxf(fmaxf(gred[q], gred[16 + q]), fmaxf(gred[32 + q], gred[48 + q])) * c;
          const float mn = fmaxf(m[q], mt);
          alpha[q] = (mn == -INFINITY) ? 1.f : ex2(m[q] - mn);
          m[q] = mn;
        }
        tc::named_sync(gbar, 128);  // gred is reused later
      }
      // P'^T limbs into buffer j % 4 (its previous reader, tile j-4 of this group, was
      // folded at tile j-2): p s_v = sigp (l0 + l1 / 254) with l0 = rint(x) in [0, 127],
      // x = p s_v / sigp, l1 = rint(254 (x - l0)) in [-127, 127]; sigp = tmax / 126.99
      // (approximate division: the limbs only need x <= 126.99 (1 + 2^-21) < 127.5)
      const float invp = tmax > 0.f ? __fdividef(126.99f, tmax) : 0.f;
      const float zi = mi.z * invp;
      // limb bytes of this token, row n = 2q + limb of P'^T, four to a word (heads q >= G
      // have p = 0 and give zero bytes)
      constexpr int kPB = 2 * NQ;
      uint32_t pw[(kPB + 3) / 4];
#pragma unroll
      for (int w = 0; w < (kPB + 3) / 4; ++w) pw[w] = 0u;
      float pv[NQ];
#pragma unroll
      for (int q = 0; q < NQ; ++q) pv[q] = (valid && q < G && m[q] != -INFINITY) ? ex2(fmaf(sv[q], c, -m[q])) : 0.f;
      // l, zc and the limb bytes, two heads per packed instruction where NQ >= 2 (the same
      // roundings: (x - r0) * 254 is exact before its one rounding, as x * 254 - 254 r0 is)
      auto limb_bytes = [&](int q, float x) {
        float r0, r1;
        const uint32_t b0 = round_byte(x, r0);
        const uint32_t b1 = round_byte((x - r0) * 254.f, r1);
        pw[(2 * q) >> 2] |= b0 << (8 * ((2 * q) & 3));
        pw[(2 * q + 1) >> 2] |= b1 << (8 * ((2 * q + 1) & 3));
      };
      if constexpr (NQ >= 2) {
        const uint64_t mag = pack2(kMagic, kMagic), nmag = pack2(-kMagic, -kMagic), f254 = pack2(254.f, 254.f),
                       n254 = pack2(-254.f, -254.f), w2 = pack2(mi.w, mi.w), zi2 = pack2(zi, zi);
#pragma unroll
        for (int q = 0; q < NQ; q += 2) {
          const uint64_t p2 = pack2(pv[q], pv[q + 1]), a2 = pack2(alpha[q], alpha[q + 1]);
          unpack2(ffma2(pack2(l[q], l[q + 1]), a2, p2), l[q], l[q + 1]);
          unpack2(ffma2(pack2(zc[q], zc[q + 1]), a2, fmul2(p2, w2)), zc[q], zc[q + 1]);
          const uint64_t x2 = fmul2(p2, zi2);
          const uint64_t t2 = fadd2(x2, mag);                       // x + 1.5 * 2^23: rint(x) in the low bits
          const uint64_t u2 = fadd2(ffma2(x2, f254, fmul2(fadd2(t2, nmag), n254)), mag);
          float t0, t1, u0, u1;
          unpack2(t2, t0, t1);
          unpack2(u2, u0, u1);
          pw[(2 * q) >> 2] |= (static_cast<uint32_t>(__float_as_int(t0)) & 0xFFu) << (8 * ((2 * q) & 3));
          pw[(2 * q + 1) >> 2] |= (static_cast<uint32_t>(__float_as_int(u0)) & 0xFFu) << (8 * ((2 * q + 1) & 3));
          pw[(2 * q + 2) >> 2] |= (static_cast<uint32_t>(__float_as_int(t1)) & 0xFFu) << (8 * ((2 * q + 2) & 3));
          pw[(2 * q + 3) >> 2] |= (static_cast<uint32_t>(__float_as_int(u1)) & 0xFFu) << (8 * ((2 * q + 3) & 3));
        }
      } else {
        l[0] = fmaf(l[0], alpha[0], pv[0]);
        zc[0] = fmaf(zc[0], alpha[0], pv[0] * mi.w);
        limb_bytes(0, pv[0] * zi);
      }
      // P'^T is MN-major without swizzle: token t's limb bytes are contiguous, 16 per
      // 2 KiB block (byte (n, t) at (n / 16) * 2048 + 16 t + n % 16): one store
      char *pt = smem + kSmP + (j & 3) * 4096 + 16 * t;
      if constexpr (kPB == 2) {
        *reinterpret_cast<uint16_t *>(pt) = static_cast<uint16_t>(pw[0]);
      } else if constexpr (kPB == 4) {
        *reinterpret_cast<uint32_t *>(pt) = pw[0];
      } else if constexpr (kPB == 8) {
        *reinterpret_cast<uint2 *>(pt) = make_uint2(pw[0], pw[1]);
      } else {
#pragma unroll
        for (int b = 0; b < kPB / 16; ++b)
          *reinterpret_cast<uint4 *>(pt + 2048 * b) = make_uint4(pw[4 * b], pw[4 * b + 1], pw[4 * b + 2], pw[4 * b + 3]);
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
      sigp_prev = tmax * (1.f / 126.99f);
    }
    if (nu > 0) {
      if (jp >= 0) fold(jp, sigp_prev, one);
      release_unread();
      flush(cur_item);
    }
  } else {
    // ================= prep warps (10-13) =================
    const int wq = warp & 3;
    const int ct = (wq << 5) | lane;  // token row of the tile
    const int rot = (ct >> 1) & 3;    // 64-byte swizzle of row ct: chunk i sits at i ^ rot
    const uint32_t tm_lane = tmem + (static_cast<uint32_t>(wq << 5) << 16);
    int prev_item = -1, nitem = -1;
    UnitIter it(a, u0);
    for (int j = 0; j < nu; ++j, it.next()) {
      const Unit un = it.un;
      const bool first = un.item != prev_item;
      if (first) {
        prev_item = un.item;
        ++nitem;
      }
      const int s = j % kStages;
      // the warp leaves together (its arrive below is warp-collective)
      if (!__all_sync(0xffffffffu, tc::wait_bar(bar(kBarFull + s), (j / kStages) & 1, p.status, abort_flag))) break;
      tc::fence_after();  // the TMEM columns written below were last read by an MMA
      char *st = smem + s * kStage;
      uint32_t lk[16];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int off = ct * 64 + ((i ^ rot) << 4);
        const uint4 kw = *reinterpret_cast<const uint4 *>(st + kStKc + off);
        const uint4 vw = *reinterpret_cast<const uint4 *>(st + kStVc + off);
        lk[4 * i] = kw.x & 0x0F0F0F0Fu;
        lk[4 * i + 1] = kw.y & 0x0F0F0F0Fu;
        lk[4 * i + 2] = kw.z & 0x0F0F0F0Fu;
        lk[4 * i + 3] = kw.w & 0x0F0F0F0Fu;
        *reinterpret_cast<uint4 *>(st + kStLv + off) =
            make_uint4(vw.x & 0x0F0F0F0Fu, vw.y & 0x0F0F0F0Fu, vw.z & 0x0F0F0F0Fu, vw.w & 0x0F0F0F0Fu);
      }
      tc::st16(tm_lane + C::kLk + s * 16, lk);  // K low nibbles: TMEM lane ct, bytes in order
      // rows past len (the tail of the last tile) get zero scales: they then add nothing,
      // and do not enter the tile's largest s_v
      const bool tvalid = static_cast<int64_t>(un.tile) * kTile + ct < p.len;
      const uint32_t ksz = tvalid ? *reinterpret_cast<const uint32_t *>(st + kStKsz + ct * 4) : 0u;
      const uint32_t vsz = tvalid ? *reinterpret_cast<const uint32_t *>(st + kStVsz + ct * 4) : 0u;
      const float2 kf = __half22float2(*reinterpret_cast<const __half2 *>(&ksz));
      const float2 vf = __half22float2(*reinterpret_cast<const __half2 *>(&vsz));
      *reinterpret_cast<float4 *>(st + kStMisc + ct * 16) = make_float4(kf.x, kf.y, vf.x, vf.y);
      // the warp's largest s_v in one step: fp16 bits of non-negative values order as the values
      const uint32_t vmax = __reduce_max_sync(0xffffffffu, vsz & 0xffffu);
      if (lane == 0)
        reinterpret_cast<float *>(st + kStTmax)[wq] = __half2float(__ushort_as_half(static_cast<unsigned short>(vmax)));
      if (first && warp == 10) {
        // the item's query limbs replace those of the item two before, once its last
        // S^T product has run and the softmax has read its sigma and sum(q)
        if (nitem >= 2 &&
            !__all_sync(0xffffffffu, tc::wait_bar(bar(kBarQFree + (nitem & 1)), ((nitem - 2) >> 1) & 1, p.status, abort_flag)))
          break;
        prep_queries(st + kStQ, smem + kSmQl + (nitem & 1) * kQlBytes,
                     reinterpret_cast<float *>(smem + kSmQinfo) + (nitem & 1) * 32, G, lane);
      }
      tc::st_wait();
      tc::fence_async_smem();  // the low nibbles and query limbs are MMA operands
      tc::fence_before();
      mbar_arrive_warp(bar(kBarCvt + s));
    }
  }

  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  if (p.pdl_mode == 2 && tid == 0) asm volatile("griddepcontrol.wait;" ::: "memory");  // the leader has ended
  if (warp == 1) tc::tmem_free(tmem, C::kAlloc);
}

template <int NQ>
cudaError_t launch_nq(const Int4DecodeArgs &a, bool overlap_previous, cudaStream_t st) {
  static std::atomic<uint64_t> attr{0};
  {
    const cudaError_t e = opt_in_smem(decode_int4_kernel<NQ>, kSmemAlloc, attr);
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
  const cudaError_t e = cudaLaunchKernelEx(&cfg, decode_int4_kernel<NQ>, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

bool decode_int4_tc_supported(const DecodeParams &p, duo_dtype dt) {
  return dt == DUO_BF16 && p.D == kD && p.G >= 1 && p.G <= 16 && tc::encode_fn() != nullptr;
}

cudaError_t launch_decode_int4_tc(const DecodeParams &p, int num_sms, bool overlap_previous, cudaStream_t st) {
  if (p.Hr < 1 || p.len < 1) return cudaSuccess;  // no retrieval head: nothing to do here
  Int4DecodeArgs a{};
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
  {  // queries [B*Hq][d]
    const uint64_t d[2] = {kD, static_cast<uint64_t>(p.B) * p.Hq};
    const uint64_t s[1] = {kD * 2};
    const uint32_t bx[2] = {64, 16};
    ok &= tc::make_map(&a.tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.q, 2, d, s, bx, CU_TENSOR_MAP_SWIZZLE_128B);
  }
  {  // retrieval codes [B*Hr][cap][64 B]
    const uint64_t d[3] = {kD / 2, static_cast<uint64_t>(p.max_len), static_cast<uint64_t>(a.n_items)};
    const uint64_t s[2] = {kD / 2, static_cast<uint64_t>(kD / 2) * p.max_len};
    const uint32_t bx[3] = {kD / 2, kTile, 1};
    ok &= tc::make_map(&a.tm_kc, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.rk, 3, d, s, bx, CU_TENSOR_MAP_SWIZZLE_64B);
    ok &= tc::make_map(&a.tm_vc, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.rv, 3, d, s, bx, CU_TENSOR_MAP_SWIZZLE_64B);
  }
  if (!ok) return cudaErrorInvalidValue;
  if (p.G <= 1) return launch_nq<1>(a, overlap_previous, st);
  if (p.G <= 2) return launch_nq<2>(a, overlap_previous, st);
  if (p.G <= 4) return launch_nq<4>(a, overlap_previous, st);
  if (p.G <= 8) return launch_nq<8>(a, overlap_previous, st);
  return launch_nq<16>(a, overlap_previous, st);
}

}  // namespace duo
