// k_decode_fp8_tc.cu -- single-token decode attention over retrieval heads that keep K
// and V as 8-bit floating point (OCP E4M3, one fp32 scale per token row), on the
// tcgen05 tensor cores.  bf16 queries, head_dim 128, up to 16 query heads per KV head;
// the layer's streaming heads (bf16) run on the bf16 decode kernel.
//
// Operation ("Decoding Procedure", steps 2, 3 and 5) as in k_decode_tc.cu; the stored
// value of element e of token t is c_te s_t (code c, scale s_t), the format pairing the
// method with an 8-bit KV cache ("Integration with Existing Optimizations").
//
// Every E4M3 value is exactly a (normal or zero) fp16 value, so the codes are widened
// with one conversion per pair and multiplied on the fp16 tensor cores:
//   S^T (128 tokens x 16) = K16 (128 x d, in TMEM) . Q16^T       logit_t = S_t s^K_t 2^-e
//   O^T (d x 16)          = V16^T (smem)          . P'^T          P'_t = p_t s^V_t / smax
// Q16 is the group's bf16 queries times 2^e (e puts the tile's largest |q| just below
// 2^14, so no query overflows or loses bits in fp16), and smax is the tile's largest
// V scale (P' stays in [0, 2^8] whatever the scales); both factors are undone in fp32.
//
// Roles of a CTA (one per SM, 480 threads):
//   warp 0     TMA producer: per 128-token tile the K and V code rows (128 B each,
//              128-byte swizzle), their scale rows, the group's bf16 queries.
//   warp 1     TMEM owner and S^T issuer; warp 10 issues O^T.
//   warps 2-5  softmax: thread t owns token t of S^T and dimension t of O^T.
//   warps 6-9, 11-14  convert: thread t of either group widens half of token t's K
//              row into TMEM lane t (the A operand of S^T) and half of its V row into
//              the swizzled shared-memory V tile, converts its share of the queries in
//              place, and (first group) writes the token's scales for the softmax.
// A widened tile lives from its conversion until its O^T product, so there are three
// widened buffers; the K half is released after S^T, the V half after O^T, and the
// codes' stage once both are widened and S^T has read the queries.
//
// Work balance and the split merge are those of the other decode kernels: the
// 128-token tiles of all (batch, retrieval head) items are laid end to end and cut
// into one equal range per CTA; the last CTA of an item merges its partials.
#include "decode_merge.cuh"
#include "tcgen05.cuh"

namespace duo {

namespace {

constexpr int kThreads = 480;
constexpr int kTile = 128;
constexpr int kD = 128;
constexpr int kN = 16;  // padded query heads per item
constexpr int kStages = 3;   // code stages (TMA ring): three hide the HBM latency of a tile
constexpr int kBufs = 3;     // widened K16 / V16 / scale buffers
constexpr int kPrefetch = 4;
constexpr int kAcc = 4;  // independent accumulator chains per contraction
// stage: K codes [128][128 B] and V codes [128][128 B] (128-byte swizzle), the bf16
// queries [16][128] (two 128-byte-swizzled halves, widened to fp16 in place), the K and
// V scale rows [128] fp32
constexpr int kStKc = 0, kStVc = 16384, kStQ = 32768, kStKs = 36864, kStVs = 37376, kStage = 38912;
constexpr int kSmV = kStages * kStage;     // kBufs x V16 [2 halves][128 tokens][64 dims] fp16
constexpr int kSmP = kSmV + kBufs * 32768; // 2 x P'^T [16][128] fp16 (2 atoms of 2 KiB)
constexpr int kSmScl = kSmP + 8192;        // kBufs x {s_k' [128], s_v' [128], smax, pad}
constexpr int kSclBytes = 2 * 128 * 4 + 64;
constexpr int kSmCred = kSmScl + kBufs * kSclBytes;  // convert reductions: kBufs x [8 warps][2]
constexpr int kSmRed = kSmCred + 256;      // softmax reductions [4][16] + merge exchange [128][6]
constexpr int kSmBar = kSmRed + (4 * 16 + 128 * 6) * 4;
constexpr int kSmMisc = kSmBar + 256;
constexpr int kSmemAlloc = kSmMisc + 64 + 1024;
static_assert(kStage % 1024 == 0 && kSmV % 1024 == 0 && kSmP % 1024 == 0, "alignment");
static_assert(kSmemAlloc <= 232448, "shared memory");

// TMEM columns: S^T x 2 and O^T x 2 (kAcc blocks of 16 each), K16 x kBufs (64 columns each)
constexpr int kTmS = 0, kTmO = 2 * kAcc * 16, kTmK = 4 * kAcc * 16, kTmemCols = 512;
static_assert(kTmK + kBufs * 64 <= kTmemCols, "tensor memory");

// Per widened buffer b (tile j uses b = j % kBufs, phase j / kBufs):
//   CvtK   K16, Q16 and the scales of the tile are written    (8 convert warps)
//   CvtV   V16 of the tile is written                         (8 convert warps)
//   KFree  S^T of the tile has run (K16 free)                 (MMA commit)
//   VFree  O^T of the tile has run (V16 free)                 (MMA commit)
//   SclFree the softmax has read the tile's scales            (4 softmax warps)
// The convert warps rewrite buffer b for tile j + kBufs only after KFree, SclFree and
// VFree of tile j, so no waiter on CvtK or CvtV can find its barrier two phases ahead.
// A code stage s (tile j, phase j / kStages) is free (Empty) once the 8 convert warps
// have read its codes and S^T has read its queries.
constexpr int kBarFull = 0, kBarEmpty = kStages, kBarCvtK = 2 * kStages, kBarCvtV = kBarCvtK + kBufs,
              kBarKFree = kBarCvtV + kBufs, kBarVFree = kBarKFree + kBufs, kBarSclFree = kBarVFree + kBufs,
              kBarSFull = kBarSclFree + kBufs, kBarSFree = kBarSFull + 2, kBarPFull = kBarSFree + 2,
              kBarOFull = kBarPFull + 2, kBarDrain = kBarOFull + 2, kBarMerge = kBarDrain + 2,  // a drain per issuer
              kNumBars = kBarMerge + 1;
static_assert(kNumBars * 8 <= 256, "barrier area");

struct Fp8DecodeArgs {
  DecodeParams p;
  int units_r;          // tiles per item
  int n_items;          // B * Hr
  int64_t total_units;  // n_items * units_r
  int num_ctas;
  CUtensorMap tm_q, tm_kc, tm_vc;
};

struct Unit {
  int item, tile;
};
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

// two E4M3 codes (low byte first) -> two fp16 (low half first); exact
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
  uint32_t r;
  const unsigned short h = static_cast<unsigned short>(two);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(h));
  return r;
}
// four codes (one 32-bit word) -> two fp16x2 words
__device__ __forceinline__ void widen4(uint32_t w, uint32_t &lo, uint32_t &hi) {
  lo = e4m3x2_to_f16x2(w & 0xFFFFu);
  hi = e4m3x2_to_f16x2(w >> 16);
}
__device__ __forceinline__ uint32_t f16x2_bits(float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t *>(&h);
}

template <int NQ>
__global__ void __launch_bounds__(kThreads, 1) decode_fp8_kernel(const __grid_constant__ Fp8DecodeArgs a) {
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
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int64_t u0 = cta_begin(a, blockIdx.x), u1 = cta_begin(a, blockIdx.x + 1);
  const int nu = static_cast<int>(u1 - u0);
  const int G = p.G;

  if (tid == 0) {
    for (int i = 0; i < kNumBars; ++i) {
      const bool many = (i >= kBarCvtK && i < kBarKFree) || (i >= kBarSclFree && i < kBarSclFree + kBufs) ||
                        i == kBarSFree || i == kBarSFree + 1 || i == kBarPFull || i == kBarPFull + 1;
      const bool empty = i >= kBarEmpty && i < kBarEmpty + kStages;
      // the convert (8) and softmax (4) warps arrive once per warp; a code stage is also
      // released by the S^T issuer's commit
      const bool cvt = i >= kBarCvtK && i < kBarKFree;
      mbar_init(bar(i), empty ? 9 : (cvt ? 8 : (many ? 4 : 1)));
    }
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
      // ends (beside a leading grid, that grid's release already implies it)
      if (p.pdl_mode != 2) asm volatile("griddepcontrol.wait;" ::: "memory");
      int issued = 0;
      UnitIter it(a, u0);
      for (int j = 0; j < nu; ++j, it.next()) {
        const int s = j % kStages;
        if (j >= kStages && !tc::wait_bar(bar(kBarEmpty + s), ((j / kStages) - 1) & 1, p.status, abort_flag)) break;
        const Unit un = it.un;
        const uint32_t dst = sbase + s * kStage;
        const uint32_t fb = bar(kBarFull + s);
        mbar_expect_tx(fb, 2 * 16384 + 4096 + 2 * 512);
        const int y = un.tile * kTile;
        const int z = un.item;  // = b * Hr + retrieval index
        tc::tma_3d(dst + kStKc, &a.tm_kc, 0, y, z, fb);
        tc::tma_3d(dst + kStVc, &a.tm_vc, 0, y, z, fb);
        const int64_t row = static_cast<int64_t>(z) * p.max_len + y;
        bulk_g2s(dst + kStKs, p.rk_sz + row * 4, 512, fb);
        bulk_g2s(dst + kStVs, p.rv_sz + row * 4, 512, fb);
        const int b = un.item / p.Hr;
        const int g = p.hm.retr_head[un.item % p.Hr];
        const int qrow = b * p.Hq + g * G;  // rows beyond this group's G heads are zeroed
        tc::tma_2d(dst + kStQ, &a.tm_q, 0, qrow, fb);
        tc::tma_2d(dst + kStQ + 2048, &a.tm_q, 64, qrow, fb);
        ++issued;
      }
      tc::drain_loads(bar(kBarFull), kStages, issued, p.status);
    }
  } else if (warp == 1 || warp == 10) {
    // ================= MMA issuers: S^T on warp 1, O^T on warp 10 =================
    // A barrier wait and an MMA issue each cost a thread hundreds of cycles on a loaded
    // SM, and a thread issuing dependent instructions sets the pace of the pipeline, so
    // the two products have an issuer each.  tcgen05.commit tracks the committing
    // thread's own MMAs.
    if (lane == 0) {
      constexpr uint32_t kIdS = tc::idesc_f16(128, kN, false, false, false);  // fp16, A from TMEM
      constexpr uint32_t kIdO = tc::idesc_f16(128, kN, true, false, false);   // V16^T MN-major
      bool ok = true;
      if (warp == 1) {
        // S^T(j) once K16(j) is widened and the softmax has read S^T(j - 2) (its buffer)
        const uint64_t dq0 = tc::sdesc(sbase + kStQ, 16, 1024);  // Q16, K-major
        for (int j = 0; j < nu && ok; ++j) {
          const int s = j % kStages, pb = j & 1, kb = j % kBufs;
          if (!tc::wait_bar(bar(kBarCvtK + kb), (j / kBufs) & 1, p.status, abort_flag)) { ok = false; break; }
          if (j >= 2 && !tc::wait_bar(bar(kBarSFree + pb), ((j - 2) >> 1) & 1, p.status, abort_flag)) { ok = false; break; }
          tc::fence_after();
          const uint64_t dq = dq0 + s * (kStage >> 4);
          const uint32_t d = tmem + kTmS + pb * kAcc * 16;
          const uint32_t ka = tmem + kTmK + kb * 64;
#pragma unroll
          for (int i = 0; i < 8; ++i) {  // K = d 128 in steps of 16 (8 TMEM columns each)
            const int kk = (i % kAcc) * (8 / kAcc) + i / kAcc;
            tc::mma_ts(d + (i % kAcc) * 16, ka + kk * 8, dq + (kk >> 2) * 128 + (kk & 3) * 2, kIdS, i >= kAcc ? 1u : 0u);
          }
          tc::commit(bar(kBarSFull + pb));
          tc::commit(bar(kBarKFree + kb));  // K16 of this buffer is free again
          tc::commit(bar(kBarEmpty + s));   // the stage's queries are read (its codes: the convert warps)
        }
      } else {
        // O^T(j) once the softmax has written P'(j) and V16(j) is widened
        const uint64_t dv0 = tc::sdesc(sbase + kSmV, 16384, 1024);  // V16^T, MN-major
        const uint64_t dp0 = tc::sdesc(sbase + kSmP, 16, 1024);    // P'^T, K-major
        for (int j = 0; j < nu && ok; ++j) {
          const int pb = j & 1, vb = j % kBufs;
          if (!tc::wait_bar(bar(kBarPFull + pb), (j >> 1) & 1, p.status, abort_flag) ||
              !tc::wait_bar(bar(kBarCvtV + vb), (j / kBufs) & 1, p.status, abort_flag)) {
            ok = false;
            break;
          }
          tc::fence_after();
          const uint64_t dv = dv0 + vb * (32768 >> 4);
          const uint64_t dp = dp0 + pb * (4096 >> 4);
          const uint32_t d = tmem + kTmO + pb * kAcc * 16;
#pragma unroll
          for (int i = 0; i < 8; ++i) {  // K = 128 tokens in steps of 16
            const int kk = (i % kAcc) * (8 / kAcc) + i / kAcc;
            tc::mma_ss(d + (i % kAcc) * 16, dv + kk * 128, dp + (kk >> 2) * 128 + (kk & 3) * 2, kIdO, i >= kAcc ? 1u : 0u);
          }
          tc::commit(bar(kBarOFull + pb));
          tc::commit(bar(kBarVFree + vb));  // V16 of this buffer is free again
        }
      }
      // drain: every MMA this thread issued has completed before TMEM is freed
      const uint32_t drain = bar(kBarDrain + (warp == 1 ? 0 : 1));
      tc::commit(drain);
      mbar_wait(drain, 0, p.status);
    }
  } else if (warp >= 6) {
    // ================= convert warps (6-9: dims 0-63, 11-14: dims 64-127) =================
    const int wq = warp & 3;
    const int t = (wq << 5) | lane;
    const int hf = warp >= 11 ? 1 : 0;                     // which half of the row
    const int cw = hf * 4 + ((warp - (hf ? 11 : 6)) & 3);  // convert warp 0..7
    const uint32_t tm_lane = tmem + (static_cast<uint32_t>(wq << 5) << 16);
    float *cred = reinterpret_cast<float *>(smem + kSmCred);  // [buffer][8 warps][2]
    // After an abort the loop still runs to its end (on whatever the buffers hold): the
    // eight warps meet at a named barrier every tile, so none may leave early.
    bool ok = true;
    UnitIter it(a, u0);
    for (int j = 0; j < nu; ++j, it.next()) {
      const int s = j % kStages, b = j % kBufs;
      const uint32_t ph = static_cast<uint32_t>((j - kBufs) / kBufs) & 1u;  // phase of tile j - kBufs
      if (ok) ok = tc::wait_bar(bar(kBarFull + s), (j / kStages) & 1, p.status, abort_flag);
      if (ok && j >= kBufs) ok = tc::wait_bar(bar(kBarKFree + b), ph, p.status, abort_flag);
      if (ok && j >= kBufs) ok = tc::wait_bar(bar(kBarSclFree + b), ph, p.status, abort_flag);
      tc::fence_after();  // K16 of this buffer was last read by an MMA
      char *st = smem + s * kStage;
      const bool valid = static_cast<int64_t>(it.un.tile) * kTile + t < p.len;
      const float sk = valid ? reinterpret_cast<const float *>(st + kStKs)[t] : 0.f;
      const float sv = valid ? reinterpret_cast<const float *>(st + kStVs)[t] : 0.f;
      // this thread's 8 query elements: half qh, row qr, 16-byte chunk qc + hf
      const int qh = t >> 6, qr = (t & 63) >> 2, qc = (t & 3) * 2;
      char *qrow = st + kStQ + qh * 2048 + qr * 128;
      uint4 *pq = reinterpret_cast<uint4 *>(qrow + (((qc + hf) ^ (qr & 7)) << 4));
      const uint4 qw = qr < G ? *pq : make_uint4(0, 0, 0, 0);
      float qmax = 0.f;
      {
        const uint32_t w4[4] = {qw.x, qw.y, qw.z, qw.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) qmax = fmaxf(qmax, fmaxf(fabsf(bf16lo(w4[e])), fabsf(bf16hi(w4[e]))));
      }
      // tile-wide largest |q| and largest V scale, over the 256 convert threads
      const float wqm = warp_max(qmax), wsm = warp_max(sv);
      if (lane == 0) {
        cred[(b * 8 + cw) * 2] = wqm;
        cred[(b * 8 + cw) * 2 + 1] = wsm;
      }
      tc::named_sync(2, 256);
      float qm = 0.f, smax = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        qm = fmaxf(qm, cred[(b * 8 + w) * 2]);
        smax = fmaxf(smax, cred[(b * 8 + w) * 2 + 1]);
      }
      // 2^e with the largest |q| in [2^13, 2^14): every query element fits fp16 exactly
      // unless it is 2^24 times smaller than the largest (then it only rounds)
      int e = 0;
      if (qm > 0.f) {
        const int ex = ((__float_as_int(qm) >> 23) & 0xFF) - 127;  // floor(log2 qm) for normal qm
        e = 13 - ex;
        e = e < -100 ? -100 : (e > 100 ? 100 : e);
      }
      const float qs = __int_as_float((127 + e) << 23);  // 2^e, exact
      {
        const uint32_t w4[4] = {qw.x, qw.y, qw.z, qw.w};
        uint4 o;
        o.x = f16x2_bits(bf16lo(w4[0]) * qs, bf16hi(w4[0]) * qs);
        o.y = f16x2_bits(bf16lo(w4[1]) * qs, bf16hi(w4[1]) * qs);
        o.z = f16x2_bits(bf16lo(w4[2]) * qs, bf16hi(w4[2]) * qs);
        o.w = f16x2_bits(bf16lo(w4[3]) * qs, bf16hi(w4[3]) * qs);
        *pq = o;
      }
      // K row t -> TMEM lane t, 64 columns of fp16 pairs (dims 2c, 2c+1 in column c);
      // 8 chunks of 16 codes: chunk c holds dims 16c .. 16c+15 = columns 8c .. 8c+7.
      // This thread widens chunks 4 hf .. 4 hf + 3.
      const int rot = t & 7;
#pragma unroll
      for (int q4 = 2 * hf; q4 < 2 * hf + 2; ++q4) {  // 2 chunks -> 16 columns per store
        uint32_t cols[16];
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int c = q4 * 2 + cc;
          const uint4 w = *reinterpret_cast<const uint4 *>(st + kStKc + t * 128 + ((c ^ rot) << 4));
          widen4(w.x, cols[cc * 8 + 0], cols[cc * 8 + 1]);
          widen4(w.y, cols[cc * 8 + 2], cols[cc * 8 + 3]);
          widen4(w.z, cols[cc * 8 + 4], cols[cc * 8 + 5]);
          widen4(w.w, cols[cc * 8 + 6], cols[cc * 8 + 7]);
        }
        tc::st16(tm_lane + kTmK + b * 64 + q4 * 16, cols);
      }
      // the token's factors for the softmax: logit = S * s_k * 2^-e * scale * log2(e),
      // P' = p * s_v / smax
      if (hf == 0) {
        float *scl = reinterpret_cast<float *>(smem + kSmScl + b * kSclBytes);
        scl[t] = sk * __int_as_float((127 - e) << 23) * p.scale_log2;
        scl[128 + t] = smax > 0.f ? sv / smax : 0.f;
        if (t == 0) scl[256] = smax;
      }
      tc::st_wait();
      tc::fence_async_smem();  // Q16 is read by the MMA (async proxy)
      tc::fence_before();
      mbar_arrive_warp(bar(kBarCvtK + b));
      // V row t -> V16 [half][token t][64 dims], 128-byte swizzle (the layout a TMA of a
      // bf16 tile would write): dims 8m .. 8m+7 of a half form 16-byte chunk m
      if (ok && j >= kBufs) ok = tc::wait_bar(bar(kBarVFree + b), ph, p.status, abort_flag);
      char *vbuf = smem + kSmV + b * 32768;
#pragma unroll
      for (int c = 4 * hf; c < 4 * hf + 4; ++c) {
        const uint4 w = *reinterpret_cast<const uint4 *>(st + kStVc + t * 128 + ((c ^ rot) << 4));
        uint4 o0, o1;
        widen4(w.x, o0.x, o0.y);
        widen4(w.y, o0.z, o0.w);
        widen4(w.z, o1.x, o1.y);
        widen4(w.w, o1.z, o1.w);
        const int d0 = 16 * c, half = d0 >> 6, m0 = (d0 & 63) >> 3;
        char *rowp = vbuf + half * 16384 + (t >> 3) * 1024 + (t & 7) * 128;
        *reinterpret_cast<uint4 *>(rowp + ((m0 ^ rot) << 4)) = o0;
        *reinterpret_cast<uint4 *>(rowp + (((m0 + 1) ^ rot) << 4)) = o1;
      }
      tc::fence_async_smem();  // V16 is read by the MMA (async proxy)
      mbar_arrive_warp(bar(kBarCvtV + b));
      mbar_arrive_warp(bar(kBarEmpty + s));  // the warp has read the stage's codes
    }
  } else {
    // ================= softmax warpgroup (warps 2-5) =================
    constexpr float kSlack = 8.0f;
    const int t = ((warp & 3) << 5) | lane;
    const int wq = warp & 3;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq << 5) << 16);
    float m[NQ], l[NQ], o[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      m[q] = -INFINITY;
      l[q] = 0.f;
      o[q] = 0.f;
    }
    bool ok = true;
    int cur_item = -1;

    // Writes this CTA's result for `item` (partial or final) and merges when last.
    auto flush = [&](int item, bool final_flush) {
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        const float v = warp_sum(l[q]);
        if (lane == 0) red[wq * kN + q] = v;
      }
      tc::named_sync(1, 128);
      float lt[NQ];
#pragma unroll
      for (int q = 0; q < NQ; ++q) lt[q] = red[q] + red[kN + q] + red[2 * kN + q] + red[3 * kN + q];
      tc::named_sync(1, 128);
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
      tc::named_sync(1, 128);
      if (t == 0) {
        const uint32_t prev = atomicAdd(p.counters + pitem, 1u);
        *last_flag = (prev == static_cast<uint32_t>(nseg - 1)) ? 1 : 0;
      }
      tc::named_sync(1, 128);
      if (!*last_flag) return;
      __threadfence();
      const uint32_t bytes = static_cast<uint32_t>(nseg) * G * kPartRow * 4;
      if (final_flush && bytes <= kSmP) {  // the idle code stages and V16 buffers
        if (t == 0) {
          asm volatile("fence.proxy.async.global;" ::: "memory");
          mbar_expect_tx(bar(kBarMerge), bytes);
          bulk_g2s(sbase, part, bytes, bar(kBarMerge));
        }
        // waited for even after an abort (bounded): the copy must not outlive the CTA
        if (!mbar_wait(bar(kBarMerge), 0, p.status)) ok = false;
        merge_partials<true>(reinterpret_cast<const float *>(smem), nseg, G, b, h0, p.Hq, p.out, p.lse, red + 4 * kN, t, 1);
      } else {
        merge_partials(part, nseg, G, b, h0, p.Hq, p.out, p.lse, red + 4 * kN, t, 1);
      }
      if (t == 0) p.counters[pitem] = 0u;
    };

    // o = (o + smax_jj O^T(jj)) * alpha for this thread's dimension t
    auto fold = [&](int jj, float smax_jj, const float (&alpha)[NQ]) {
      if (ok) ok = tc::wait_bar(bar(kBarOFull + (jj & 1)), (jj >> 1) & 1, p.status, abort_flag);
      tc::fence_after();
      float v[NQ];
      tc::ld_sum<NQ, kAcc>(lane_base + kTmO + (jj & 1) * kAcc * 16, 16, v);
#pragma unroll
      for (int q = 0; q < NQ; ++q) o[q] = fmaf(v[q], smax_jj, o[q]) * alpha[q];
    };
    float one[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q) one[q] = 1.f;

    bool pending = false;
    float smax_prev = 0.f;
    UnitIter it(a, u0);
    for (int j = 0; j < nu; ++j, it.next()) {
      const Unit un = it.un;
      const int b = j & 1;
      if (ok) ok = tc::wait_bar(bar(kBarSFull + b), (j >> 1) & 1, p.status, abort_flag);
      tc::fence_after();
      float sv[NQ];
      tc::ld_sum<NQ, kAcc>(lane_base + kTmS + b * kAcc * 16, 16, sv);
      tc::fence_before();
      mbar_arrive_warp(bar(kBarSFree + b));
      // the convert warps' factors of this tile (ordered before these reads by its barrier)
      const int kb = j % kBufs;
      if (ok) ok = tc::wait_bar(bar(kBarCvtK + kb), (j / kBufs) & 1, p.status, abort_flag);
      const float *scl = reinterpret_cast<const float *>(smem + kSmScl + kb * kSclBytes);
      const float fk = scl[t], fv = scl[128 + t], smax = scl[256];
      mbar_arrive_warp(bar(kBarSclFree + kb));
      const bool valid = static_cast<int64_t>(un.tile) * kTile + t < p.len;
      if (un.item != cur_item) {
        if (cur_item >= 0) {
          if (pending) fold(j - 1, smax_prev, one);
          flush(cur_item, false);
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
      float x[NQ];
#pragma unroll
      for (int q = 0; q < NQ; ++q) x[q] = sv[q] * fk;  // log2-domain logit
      int need = 0;
#pragma unroll
      for (int q = 0; q < NQ; ++q)
        if (q < G && valid && x[q] > m[q] + kSlack) need = 1;
      need = tc::bar_or(1, 128, need);
      float alpha[NQ];
#pragma unroll
      for (int q = 0; q < NQ; ++q) alpha[q] = 1.f;
      if (need) {
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          const float xm = warp_max((valid && q < G) ? x[q] : -INFINITY);
          if (lane == 0) red[wq * kN + q] = xm;
        }
        tc::named_sync(1, 128);
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          const float mt = fmaxf(fmaxf(red[q], red[kN + q]), fmaxf(red[2 * kN + q], red[3 * kN + q]));
          const float mn = fmaxf(m[q], mt);
          alpha[q] = (mn == -INFINITY) ? 1.f : ex2(m[q] - mn);
          m[q] = mn;
        }
        tc::named_sync(1, 128);
      }
      uint16_t pb[NQ];
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        const float pv = (valid && q < G && m[q] != -INFINITY) ? ex2(x[q] - m[q]) : 0.f;
        l[q] = fmaf(l[q], alpha[q], pv);
        const __half hb = __float2half_rn(pv * fv);
        pb[q] = *reinterpret_cast<const uint16_t *>(&hb);
      }
      {  // P'^T[q][t] into buffer j % 2 (its previous reader, tile j-2, was folded at j-1)
        const int atom = t >> 6, col = t & 63;
        char *pbase = smem + kSmP + b * 4096 + atom * 2048;
#pragma unroll
        for (int q = 0; q < NQ; ++q)
          if (q < G) {
            const int chunk = (col >> 3) ^ (q & 7);
            *reinterpret_cast<uint16_t *>(pbase + q * 128 + chunk * 16 + (col & 7) * 2) = pb[q];
          }
      }
      tc::fence_async_smem();
      tc::fence_before();
      mbar_arrive_warp(bar(kBarPFull + b));
      if (pending) {
        fold(j - 1, smax_prev, alpha);
      } else {
#pragma unroll
        for (int q = 0; q < NQ; ++q) o[q] *= alpha[q];
      }
      pending = true;
      smax_prev = smax;
    }
    if (nu > 0) {
      if (pending) fold(nu - 1, smax_prev, one);
      flush(cur_item, true);
    }
  }

  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  if (p.pdl_mode == 2 && tid == 0) asm volatile("griddepcontrol.wait;" ::: "memory");  // the leader has ended
  if (warp == 1) tc::tmem_free(tmem, kTmemCols);
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
  return dt == DUO_BF16 && p.D == kD && p.G >= 1 && p.G <= kN && tc::encode_fn() != nullptr;
}

cudaError_t launch_decode_fp8_tc(const DecodeParams &p, int num_sms, bool overlap_previous, cudaStream_t st) {
  if (p.Hr < 1 || p.len < 1) return cudaSuccess;  // no retrieval head: nothing to do here
  Fp8DecodeArgs a{};
  a.p = p;
  a.units_r = static_cast<int>((p.len + kTile - 1) / kTile);
  a.n_items = p.B * p.Hr;
  a.total_units = static_cast<int64_t>(a.n_items) * a.units_r;
  int64_t ctas = num_sms;
  if (ctas > a.total_units) ctas = a.total_units;
  if (ctas > kMaxSplits) ctas = kMaxSplits;
  a.num_ctas = static_cast<int>(ctas);
  bool ok = true;
  {  // queries [B*Hq][d] bf16
    const uint64_t d[2] = {kD, static_cast<uint64_t>(p.B) * p.Hq};
    const uint64_t s[1] = {kD * 2};
    const uint32_t bx[2] = {64, kN};
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
