// k_prefill_tc.cu -- chunked pre-fill attention on the 5th-generation tensor cores
// (tcgen05 + TMEM), bf16 in, fp32 accumulate, head_dim 128.
//
// Operation ("Chunked Pre-filling", masks of "The Full and Streaming Attention
// Masks"): the n chunk queries at positions len .. len+n-1 attend to
//   * retrieval heads: every key 0 .. i (causal): positions before len from the full
//     cache, the chunk's own positions from the chunk input (so the attention does not
//     depend on the chunk having been appended: the caller appends after it);
//   * streaming heads: the staged history (sinks, then positions wstart..len-1) and
//     the chunk's own keys, with the Lambda mask j < S or i - j < W.  Key tiles that
//     hold no visible key for any row of the CTA's query tiles are never loaded (tile
//     skip).
//
// One CTA = two 128-row query tiles (each a GQA group of heads x 128/G positions, the
// second following the first) that share every K/V tile it loads; 12 warps:
//   warp 0      TMA producer: both Q tiles once, then K tiles of 128 keys (2-stage ring)
//   warp 1      TMEM allocator; lane 0 issues every tcgen05.mma
//   warp 2      TMA producer: V tiles (2-stage ring)
//   warps 4..7  softmax of query tile 0, warps 8..11 of query tile 1: one thread per
//               query row (TMEM lane), all 128 logits of a key tile in registers
// TMEM (512 columns): S_t at 128 t, O_t at 256 + 128 t for query tile t; the softmax
// writes P_t (bf16 pairs) over the first 64 columns of S_t.
//   S_t(j) = Q_t K_j^T   (M 128, N 128, K 128: 8 MMAs of K 16), into S_t
//   O_t += P_t(j) V_j    (M 128, N 128, K 128 keys), A = P_t(j) from TMEM, B = V_j (smem)
// The MMA thread issues PV_0(j), S_0(j+1), PV_1(j), S_1(j+1), ...: the tensor core
// works on one query tile while the other tile's softmax runs (ping-pong).  tcgen05.mma
// operations of one thread complete in issue order, so S_t(j+1) overwrites P_t(j) only
// after PV_t(j) has read it, and when S_t(j) has landed PV_t(j-1) has too: O_t may then
// be rescaled in place.  The running max m is a reference: P = exp2(s*c - m) may exceed
// 1 by up to 2^kSlack, and m (with O and l) is rescaled only when a row's tile maximum
// passes m + kSlack.
//
// Every mbarrier wait is bounded; a wait that runs out latches kDevTimeout in the
// status word and sets an abort flag so that every role drains and exits (the
// producers first wait, bounded, for the loads they issued).
#include "tcgen05.cuh"

namespace duo {

namespace {

constexpr int kBM = 128;  // query rows per tile
constexpr int kBN = 128;  // keys per tile
constexpr int kQT = 2;    // query tiles per CTA
constexpr int kSoftWarp0 = 4;                       // first softmax warp (tile t: warps 4 + 4t .. 7 + 4t)
constexpr int kTcThreads = 32 * (kSoftWarp0 + 4 * kQT);
constexpr int kD = 128;
constexpr int kKStages = 2;  // K ring: a stage is free once S_1(j) is computed
constexpr int kVStages = 2;  // V ring: a stage is free once P_1(j) V_j is computed
constexpr int kMaxStrmTiles = 48;

// shared memory map (bytes from the 1 KiB-aligned base); every tile is two 128B-swizzled
// [128][64] bf16 halves of 16 KiB
constexpr int kSmQ = 0;                             // query tile t at kSmQ + t * 32 KiB
constexpr int kSmK = kQT * 32768;                   // K stage s at kSmK + s * 32 KiB
constexpr int kSmV = kSmK + kKStages * 32768;       // V stage s at kSmV + s * 32 KiB
constexpr int kSmBar = kSmV + kVStages * 32768;
constexpr int kSmMisc = kSmBar + 256;
constexpr int kSmTotal = kSmMisc + 1024 + kMaxStrmTiles * 16;
constexpr int kSmemAlloc = kSmTotal + 1024;  // slack for aligning the base to 1 KiB

// TMEM columns of query tile t: S_t (P_t over its first 64) and O_t
constexpr int kTmS = 0, kTmO = 256;

// barrier indices (8 bytes each)
constexpr int kBarQ = 0, kBarKFull = 1, kBarKEmpty = kBarKFull + kKStages, kBarVFull = kBarKEmpty + kKStages,
              kBarVEmpty = kBarVFull + kVStages, kBarSFull = kBarVEmpty + kVStages, kBarPFull = kBarSFull + kQT,
              kBarOFull = kBarPFull + kQT, kBarDrain = kBarOFull + kQT, kNumBars = kBarDrain + 1;
static_assert(kNumBars * 8 <= 256, "barrier area");
static_assert(kSmemAlloc <= 227 * 1024, "shared memory");

struct TileDesc {
  int src;      // 0 retrieval cache, 1 streaming history, 2 chunk input
  int y;        // first row in the source
};

using TcArgs = PrefillTcLaunch;  // the kernel's parameter block (host-prepared tensor maps)

// ---------------------------------------------------------------- tile lists

struct Plan {
  bool retr;
  int nh;          // retrieval: tiles of cached positions 0 .. len-1 (then chunk tiles)
  int64_t q0;      // absolute position of query row 0 of this tile
  int kvrow;       // retrieval: z index of the head in the cache map / streaming: in the hist map
};

// Streaming heads: which history / chunk tiles hold a visible key for some row of
// the query tile.  Writes the list into `tl` and returns its length.
__device__ int streaming_tiles(const PrefillParams &p, int r0, int npos, TileDesc *tl) {
  int nt = 0;
  const int64_t qlo = p.len + r0;                                      // smallest query position
  const int rows_hi = (r0 + npos < p.n) ? r0 + npos : p.n;              // chunk rows this block needs
  const int hrows = p.hs + p.hw;
  const int nh = (hrows + kBN - 1) / kBN;
  for (int t = 0; t < nh && nt < kMaxStrmTiles; ++t) {
    const int a = t * kBN, b = ((t + 1) * kBN < hrows ? (t + 1) * kBN : hrows) - 1;
    const bool sinks = a < p.hs;
    const int64_t maxpos = b < p.hs ? b : p.wstart + (b - p.hs);
    // the smallest query position reaches furthest back: pos > qlo - W
    const bool recent = maxpos > qlo - p.W;
    if (sinks || recent) tl[nt++] = {1, a};
  }
  const int nc = (rows_hi + kBN - 1) / kBN;
  int c0 = r0 - p.W + 1;
  c0 = c0 < 0 ? 0 : c0 / kBN;
  // chunk tiles holding sinks (positions < S) that lie before the window tiles
  const int sink_rows = p.len < p.S ? static_cast<int>(p.S - p.len) : 0;
  const int ns = (sink_rows + kBN - 1) / kBN;
  for (int t = 0; t < ns && t < c0 && t < nc && nt < kMaxStrmTiles; ++t) tl[nt++] = {2, t * kBN};
  for (int t = c0; t < nc && nt < kMaxStrmTiles; ++t) tl[nt++] = {2, t * kBN};
  return nt;
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// exp2(v*c - mc) of the N logits v[B .. B+N) on MUFU, their sum into rowsum and bf16
// pairs into pk.  The scaling and the sums run on packed fp32 pairs.  (With two query
// tiles in ping-pong, moving part of the exponentials to an FMA-pipe polynomial only
// added instructions.)
template <int N, int B = 0, int M>
__device__ __forceinline__ void probabilities(const float (&v)[M], float c, float mc, float &rowsum,
                                              uint32_t (&pk)[N / 2]) {
  static_assert(B + N <= M, "logit range");
  const uint64_t cc = pack2(c, c), mm = pack2(-mc, -mc);
  uint64_t acc[2] = {pack2(0.f, 0.f), pack2(0.f, 0.f)};
#pragma unroll
  for (int e = 0; e < N; e += 2) {
    const uint64_t x = ffma2(pack2(v[B + e], v[B + e + 1]), cc, mm);
    float x0, x1;
    unpack2(x, x0, x1);
    const float p0 = ex2(x0), p1 = ex2(x1);
    acc[(e >> 1) & 1] = fadd2(acc[(e >> 1) & 1], pack2(p0, p1));
    const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
    pk[e >> 1] = *reinterpret_cast<const uint32_t *>(&pb);
  }
  float a0, a1, b0, b1;
  unpack2(acc[0], a0, a1);
  unpack2(acc[1], b0, b1);
  rowsum = (a0 + a1) + (b0 + b1);
}

// A key offset relative to a tile start, clamped to [-1, 127].
__device__ __forceinline__ int clamp_col(int64_t x) { return static_cast<int>(x < -1 ? -1 : (x > kBN - 1 ? kBN - 1 : x)); }

// Tile j of the query tile's key sequence: retrieval heads visit the cached positions
// 0 .. len-1 (nh tiles, the last one possibly partial), then the chunk from its start;
// streaming heads follow their tile list.
__device__ __forceinline__ TileDesc tile_of(const Plan &pl, const TileDesc *tl, int j) {
  if (pl.retr) return j < pl.nh ? TileDesc{0, j * kBN} : TileDesc{2, (j - pl.nh) * kBN};
  return tl[j];
}

// TMA of one 128-key tile (K when is_k, else V) from its source into two swizzled halves
__device__ __forceinline__ void load_tile(const TcArgs &a, const TileDesc &t, const Plan &pl, int g, int b,
                                          uint32_t dst, uint32_t fb, bool is_k) {
  if (t.src == 0) {
    const CUtensorMap *m = is_k ? &a.tm_kc : &a.tm_vc;
    tc::tma_3d(dst, m, 0, t.y, pl.kvrow, fb);
    tc::tma_3d(dst + 16384, m, 64, t.y, pl.kvrow, fb);
  } else if (t.src == 1) {
    const CUtensorMap *m = is_k ? &a.tm_kh : &a.tm_vh;
    tc::tma_3d(dst, m, 0, t.y, pl.kvrow, fb);
    tc::tma_3d(dst + 16384, m, 64, t.y, pl.kvrow, fb);
  } else {
    const CUtensorMap *m = is_k ? &a.tm_kn : &a.tm_vn;
    tc::tma_4d(dst, m, 0, g, t.y, b, fb);
    tc::tma_4d(dst + 16384, m, 64, g, t.y, b, fb);
  }
}

// ---------------------------------------------------------------- the kernel

// 128 consecutive fp32 columns of this thread's lane: four loads, one wait that names
// every destination register (so that no use is scheduled before it)
#define DUO_R4(x) "+r"(r[(x)]), "+r"(r[(x) + 1]), "+r"(r[(x) + 2]), "+r"(r[(x) + 3])
#define DUO_R16(x) DUO_R4(x), DUO_R4((x) + 4), DUO_R4((x) + 8), DUO_R4((x) + 12)
#define DUO_O4(x) "=r"(r[(x)]), "=r"(r[(x) + 1]), "=r"(r[(x) + 2]), "=r"(r[(x) + 3])
#define DUO_O16(x) DUO_O4(x), DUO_O4((x) + 4), DUO_O4((x) + 8), DUO_O4((x) + 12)
__device__ __forceinline__ void ld128(uint32_t taddr, float (&v)[128]) {
  uint32_t r[128];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t *q = r + 32 * c;
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(q[0]), "=r"(q[1]), "=r"(q[2]), "=r"(q[3]), "=r"(q[4]), "=r"(q[5]), "=r"(q[6]), "=r"(q[7]), "=r"(q[8]),
          "=r"(q[9]), "=r"(q[10]), "=r"(q[11]), "=r"(q[12]), "=r"(q[13]), "=r"(q[14]), "=r"(q[15]), "=r"(q[16]),
          "=r"(q[17]), "=r"(q[18]), "=r"(q[19]), "=r"(q[20]), "=r"(q[21]), "=r"(q[22]), "=r"(q[23]), "=r"(q[24]),
          "=r"(q[25]), "=r"(q[26]), "=r"(q[27]), "=r"(q[28]), "=r"(q[29]), "=r"(q[30]), "=r"(q[31])
        : "r"(taddr + 32 * c));
  }
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : DUO_R16(0), DUO_R16(16), DUO_R16(32), DUO_R16(48), DUO_R16(64), DUO_R16(80), DUO_R16(96), DUO_R16(112)
               :
               : "memory");
#pragma unroll
  for (int i = 0; i < 128; ++i) v[i] = __uint_as_float(r[i]);
}
#undef DUO_R4
#undef DUO_R16
#undef DUO_O4
#undef DUO_O16

// P of logits v[B .. B+32) as 16 bf16 pairs into TMEM columns B/2 .. B/2+15 of s_cols
// (no wait), their sum into rs
template <int B>
__device__ __forceinline__ void p_chunk(const float (&v)[128], float c, float mc, float &rs, uint32_t s_cols) {
  uint32_t pk[16];
  probabilities<32, B>(v, c, mc, rs, pk);
  tc::st16(s_cols + B / 2, pk);
}

__global__ void __launch_bounds__(kTcThreads, 1) prefill_tc_kernel(const __grid_constant__ TcArgs a) {
  const PrefillParams &p = a.p;
  extern __shared__ char smem_raw[];
  char *smem = reinterpret_cast<char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + kSmBar;
  auto bar = [&](int i) { return bar0 + 8u * i; };
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kSmMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kSmMisc + 4);
  int *ntiles_sm = reinterpret_cast<int *>(smem + kSmMisc + 8);
  TileDesc *tl = reinterpret_cast<TileDesc *>(smem + kSmMisc + 1024);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- which query tiles ----
  // GQA packing: the 128 rows of a query tile are npos = 128 / G consecutive positions x
  // the G query heads of one KV head (row r = position r / G, head r % G), so every K/V
  // tile a CTA loads serves the whole group, for both of its query tiles.
  const int G = p.G;
  const int npos = kBM / G;
  const int ntq = (p.n + npos - 1) / npos;         // query tiles of one (sequence, KV head)
  const int ncta = (ntq + kQT - 1) / kQT;
  const int bg = blockIdx.x % (p.B * p.Hkv);
  const int qc = ncta - 1 - blockIdx.x / (p.B * p.Hkv);  // heaviest (latest) blocks first
  const int b = bg / p.Hkv, g = bg % p.Hkv;
  const int r0 = qc * kQT * npos;                   // first chunk row (position offset) of the CTA
  const int nq = (ntq - qc * kQT) < kQT ? (ntq - qc * kQT) : kQT;  // query tiles present (1 or 2)
  Plan pl;
  pl.retr = p.hm.is_retr[g] != 0;
  pl.nh = pl.retr ? static_cast<int>((p.len + kBN - 1) / kBN) : 0;
  pl.q0 = p.len + r0;
  pl.kvrow = b * (pl.retr ? p.Hr : p.HsMax) + p.hm.kind_idx[g];

  if (tid == 0) {
    // P_t is published by one arrival per softmax warp
    for (int i = 0; i < kNumBars; ++i) mbar_init(bar(i), (i >= kBarPFull && i < kBarPFull + kQT) ? kBM / 32 : 1);
    if (smem_u32(smem) & 1023u) flag_status(p.status, kDevTimeout);  // layout assumption (never expected)
    fence_mbar_init();
    *abort_flag = 0;
    int nt;
    const int rows = (r0 + nq * npos < p.n) ? r0 + nq * npos : p.n;  // chunk rows 0 .. rows-1 are needed
    if (pl.retr) {
      nt = pl.nh + (rows + kBN - 1) / kBN;
    } else {
      nt = streaming_tiles(p, r0, rows - r0, tl);
    }
    *ntiles_sm = nt;
  }
  if (warp == 1) tc::tmem_alloc(smem_u32(tmem_slot), 512);
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *tmem_slot;
  const int nt = *ntiles_sm;

  if (warp == 0) {
    // ================= TMA producer: the Q tiles, then the K ring =================
    if (lane == 0) {
      tc::prefetch_map(&a.tm_q);
      mbar_expect_tx(bar(kBarQ), 32768 * nq);
      for (int t = 0; t < nq; ++t) {  // box: 64 dims x G heads x npos positions
        tc::tma_4d(sbase + kSmQ + t * 32768, &a.tm_q, 0, g * G, r0 + t * npos, b, bar(kBarQ));
        tc::tma_4d(sbase + kSmQ + t * 32768 + 16384, &a.tm_q, 64, g * G, r0 + t * npos, b, bar(kBarQ));
      }
      int issued = 0;
      for (int j = 0; j < nt; ++j) {
        const int s = j % kKStages;
        if (j >= kKStages && !tc::wait_bar(bar(kBarKEmpty + s), ((j / kKStages) - 1) & 1, p.status, abort_flag)) break;
        const TileDesc t = tile_of(pl, tl, j);
        const uint32_t dst = sbase + kSmK + s * 32768, fb = bar(kBarKFull + s);
        mbar_expect_tx(fb, 32768);
        load_tile(a, t, pl, g, b, dst, fb, true);
        ++issued;
      }
      // nothing may still be landing in shared memory when the CTA ends
      mbar_wait(bar(kBarQ), 0, p.status);
      tc::drain_loads(bar(kBarKFull), kKStages, issued, p.status);
    }
  } else if (warp == 2) {
    // ================= TMA producer: the V ring =================
    if (lane == 0) {
      int issued = 0;
      for (int j = 0; j < nt; ++j) {
        const int s = j % kVStages;
        if (j >= kVStages && !tc::wait_bar(bar(kBarVEmpty + s), ((j / kVStages) - 1) & 1, p.status, abort_flag)) break;
        const TileDesc t = tile_of(pl, tl, j);
        const uint32_t dst = sbase + kSmV + s * 32768, fb = bar(kBarVFull + s);
        mbar_expect_tx(fb, 32768);
        load_tile(a, t, pl, g, b, dst, fb, false);
        ++issued;
      }
      tc::drain_loads(bar(kBarVFull), kVStages, issued, p.status);
    }
  } else if (warp == 1) {
    // ================= MMA issuer =================
    if (lane == 0) {
      constexpr uint32_t kIdS = tc::idesc_bf16(kBM, kBN, false, false);
      constexpr uint32_t kIdPV = tc::idesc_bf16(kBM, kD, false, true);
      // Shared-memory descriptors are built once: the start address sits in the low 14
      // bits as addr >> 4 and every operand lies below 256 KiB, so an operand at byte
      // offset o from a base is the base's descriptor + (o >> 4).  A single thread issues
      // every MMA; keeping its per-MMA work to an add keeps the tensor pipe fed.
      const uint64_t qd0 = tc::sdesc(sbase + kSmQ, 16, 1024), kd0 = tc::sdesc(sbase + kSmK, 16, 1024);
      const uint64_t vd0 = tc::sdesc(sbase + kSmV, 16384, 1024);
      // S_t(j) = Q_t K_j^T : K = d 128 in 8 steps of 16 (16 dims = 32 bytes within a
      // 128-byte swizzled row, the second 64 dims in the other half); Q and K K-major
      auto issue_s = [&](int t, int j) {
        const uint64_t qd = qd0 + t * (32768 >> 4), kd = kd0 + (j % kKStages) * (32768 >> 4);
        const uint32_t d = tmem + kTmS + t * 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t o = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
          tc::mma_ss(d, qd + o, kd + o, kIdS, kk > 0 ? 1u : 0u);
        }
        tc::commit(bar(kBarSFull + t));
      };
      // O_t += P_t(j) V_j : K = 128 keys in 8 steps of 16 (16 keys = 2 KiB of V); P from
      // TMEM (bf16 pairs, K-major), V from shared memory (d contiguous, MN-major)
      auto issue_pv = [&](int t, int j) {
        const uint64_t vd = vd0 + (j % kVStages) * (32768 >> 4);
        const uint32_t d = tmem + kTmO + t * 128, pa = tmem + kTmS + t * 128;
        const uint32_t acc0 = j > 0 ? 1u : 0u;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) tc::mma_ts(d, pa + kk * 8, vd + kk * (2048 >> 4), kIdPV, kk > 0 ? 1u : acc0);
      };
      bool ok = nt > 0 && tc::wait_bar(bar(kBarQ), 0, p.status, abort_flag) &&
                tc::wait_bar(bar(kBarKFull), 0, p.status, abort_flag);
      if (ok) {
        tc::fence_after();
        for (int t = 0; t < nq; ++t) issue_s(t, 0);
        tc::commit(bar(kBarKEmpty));
      }
      for (int j = 0; j < nt && ok; ++j) {
        for (int t = 0; t < nq && ok; ++t) {
          if (!tc::wait_bar(bar(kBarPFull + t), j & 1, p.status, abort_flag)) { ok = false; break; }
          if (t == 0 &&
              !tc::wait_bar(bar(kBarVFull + (j % kVStages)), (j / kVStages) & 1, p.status, abort_flag)) {
            ok = false;
            break;
          }
          tc::fence_after();
          issue_pv(t, j);
          if (t == nq - 1) tc::commit(bar(kBarVEmpty + (j % kVStages)));
          if (j + 1 < nt) {
            if (t == 0) {
              if (!tc::wait_bar(bar(kBarKFull + ((j + 1) % kKStages)), ((j + 1) / kKStages) & 1, p.status,
                                abort_flag)) {
                ok = false;
                break;
              }
              tc::fence_after();
            }
            issue_s(t, j + 1);
            if (t == nq - 1) tc::commit(bar(kBarKEmpty + ((j + 1) % kKStages)));
          } else {
            tc::commit(bar(kBarOFull + t));
          }
        }
      }
      // drain: every MMA this thread issued has completed before TMEM is freed
      tc::commit(bar(kBarDrain));
      mbar_wait(bar(kBarDrain), 0, p.status);
    }
  } else if (warp >= kSoftWarp0 && (warp - kSoftWarp0) / 4 < nq) {
    // ================= softmax of query tile qt: one thread per query row =================
    constexpr float kSlack = 8.0f;
    const int qt = (warp - kSoftWarp0) >> 2;
    const int wq = warp & 3;
    const int row = (wq << 5) | lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq << 5) << 16);
    const uint32_t s_cols = lane_base + kTmS + qt * 128, o_cols = lane_base + kTmO + qt * 128;
    const int rpos = qt * npos + row / G;      // position offset of this row within the CTA
    const int h = g * G + row % G;             // its query head
    const int64_t i = pl.q0 + rpos;            // absolute query position
    const float c = p.scale_log2;
    float m = -INFINITY, l = 0.f;
    bool ok = true;

    for (int j = 0; j < nt; ++j) {
      const TileDesc t = tile_of(pl, tl, j);
      // Mask of this row over the tile's 128 keys, as three column bounds: key col is
      // visible iff col <= hi && (col < sink_c || col > win_c).
      int hi, sink_c = kBN, win_c = -1;
      if (t.src == 0) {  // retrieval cache: positions y + col < len, all before the query
        hi = clamp_col(p.len - 1 - t.y);
      } else {
        int64_t base, sink_rel, win_rel;
        int valid;
        if (t.src == 2) {  // chunk rows: positions len + y + col
          base = p.len + t.y;
          valid = p.n - t.y;
          hi = clamp_col(i - base);
          sink_rel = p.S - base;
          win_rel = i - p.W - base;
        } else {  // history rows: col < hs - y are sinks, later rows are wstart + (row - hs)
          valid = p.hs + p.hw - t.y;
          hi = kBN - 1;
          sink_rel = p.hs - t.y;
          win_rel = i - p.W - p.wstart + p.hs - t.y;
        }
        hi = min(hi, valid - 1);
        if (!pl.retr) {  // retrieval heads see every key up to the query (causal only)
          sink_c = static_cast<int>(sink_rel < 0 ? 0 : (sink_rel > kBN ? kBN : sink_rel));
          win_c = clamp_col(win_rel);
        }
      }
      const bool full_vis = hi >= kBN - 1 && (sink_c >= kBN || win_c < 0);

      if (ok) ok = tc::wait_bar(bar(kBarSFull + qt), j & 1, p.status, abort_flag);
      tc::fence_after();
      float v[128];
      ld128(s_cols, v);
      if (!full_vis) {
#pragma unroll
        for (int e = 0; e < 128; ++e) {
          const bool vis = e <= hi && (e < sink_c || e > win_c);
          v[e] = vis ? v[e] : -INFINITY;
        }
      }
      float mx8[8];  // eight independent chains of three-input maxima
#pragma unroll
      for (int u = 0; u < 8; ++u) mx8[u] = fmaxf(v[2 * u], v[2 * u + 1]);
#pragma unroll
      for (int e = 16; e < 128; e += 2) mx8[(e >> 1) & 7] = fmax3(mx8[(e >> 1) & 7], v[e], v[e + 1]);
      const float mx = fmaxf(fmaxf(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5])), fmaxf(mx8[6], mx8[7]));
      const float tmax = mx * c;  // -inf when nothing in the tile is visible
      const bool need = tmax > m + kSlack;
      float alpha = 1.f;
      if (need) {
        alpha = ex2(m - tmax);  // 0 while m is -inf
        m = tmax;
      }
      if (j >= 1 && __any_sync(0xffffffffu, need)) {
        // rescale this row of O_t: S_t(j) has landed, so P_t(j-1) V_{j-1} has too
#pragma unroll 1
        for (int q = 0; q < 8; ++q) {  // 16 columns at a time: the logits stay in registers
          float w[16];
          tc::ld<16>(o_cols + 16 * q, w);
          uint32_t u[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) u[e] = __float_as_uint(w[e] * alpha);
          tc::st16(o_cols + 16 * q, u);
        }
        tc::st_wait();
      }
      // probabilities (masked logits are -inf and give 0), row sum, bf16 pairs of P_t(j)
      // over the first 64 columns of S_t
      const float mc = (m == -INFINITY) ? 0.f : m;
      float rs[4];
      p_chunk<0>(v, c, mc, rs[0], s_cols);
      p_chunk<32>(v, c, mc, rs[1], s_cols);
      p_chunk<64>(v, c, mc, rs[2], s_cols);
      p_chunk<96>(v, c, mc, rs[3], s_cols);
      const float rsum = (rs[0] + rs[1]) + (rs[2] + rs[3]);
      tc::st_wait();
      tc::fence_before();
      mbar_arrive_warp(bar(kBarPFull + qt));
      l = l * alpha + rsum;
    }
    // the last product, then the epilogue: normalise and store the row (bf16) and its
    // lse; in gated mixing, blend with the row already in out
    if (nt > 0 && ok) ok = tc::wait_bar(bar(kBarOFull + qt), 0, p.status, abort_flag);
    tc::fence_after();
    const bool store = r0 + rpos < p.n;
    char *orow = p.out + ((static_cast<int64_t>(b) * p.n + r0 + rpos) * p.Hq + h) * (kD * 2);
    const float inv = 1.f / l;
    const float mixa = p.mix_alpha ? p.mix_alpha[g] : 0.f;
#pragma unroll 1
    for (int q = 0; q < 4; ++q) {
      float w[32];
      tc::ld<32>(o_cols + 32 * q, w);
      if (store) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float x[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) x[e] = w[8 * u + e] * inv;
          char *dst = orow + q * 64 + u * 16;
          if (p.mix_alpha) {
            const uint4 old = *reinterpret_cast<const uint4 *>(dst);
            float f[8];
            Elem<__nv_bfloat16>::unpack(old, f);
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = fmaf(mixa, f[e] - x[e], x[e]);
          }
          uint32_t wd[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 pb = __floats2bfloat162_rn(x[2 * e], x[2 * e + 1]);
            wd[e] = *reinterpret_cast<const uint32_t *>(&pb);
          }
          *reinterpret_cast<uint4 *>(dst) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
        }
      }
    }
    if (store && p.lse) p.lse[(static_cast<int64_t>(b) * p.n + r0 + rpos) * p.Hq + h] = (m + lg2(l)) * kLn2;
  }

  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  if (warp == 1) tc::tmem_free(tmem, 512);
}

}  // namespace

bool prefill_tc_supported(const PrefillParams &p, duo_dtype dt) {
  if (dt != DUO_BF16 || p.D != kD) return false;
  if (p.G < 1 || p.G > kBM || (p.G & (p.G - 1)) != 0) return false;  // the group must tile 128 rows
  if (tc::encode_fn() == nullptr) return false;
  // streaming tile list must fit: history tiles + window tiles + a sink tile
  const int hist_tiles = (p.hs + p.hw + kBN - 1) / kBN;
  const int win_tiles = (p.W + 3 * kBN - 2) / kBN + 1;  // window of two query tiles
  const int sink_tiles = (p.S + kBN - 1) / kBN;
  return hist_tiles + win_tiles + sink_tiles <= kMaxStrmTiles;
}

cudaError_t prepare_prefill_tc(const PrefillParams &p, PrefillTcLaunch *l) {
  TcArgs &a = *l;
  a.p = p;
  const uint64_t row = kD * 2;
  const CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B;
  // maps of sources this launch never reads (no cached positions, no streaming history)
  // still need a valid description: they point at the chunk input
  const void *rk = p.len > 0 && p.Hr > 0 ? p.rk : p.k, *rv = p.len > 0 && p.Hr > 0 ? p.rv : p.v;
  const void *hk = p.hs + p.hw > 0 ? p.hk : p.k, *hv = p.hs + p.hw > 0 ? p.hv : p.v;
  bool ok = true;
  {  // q [B][n][Hq][d]; box = 64 dims x G heads x 128/G positions (one GQA group)
    const uint64_t d[4] = {kD, static_cast<uint64_t>(p.Hq), static_cast<uint64_t>(p.n), static_cast<uint64_t>(p.B)};
    const uint64_t s[3] = {row, row * p.Hq, row * p.Hq * p.n};
    const uint32_t bx[4] = {64, static_cast<uint32_t>(p.G), static_cast<uint32_t>(kBM / p.G), 1};
    ok &= tc::make_map(&a.tm_q, bf, p.q, 4, d, s, bx, sw);
  }
  {  // chunk k, v [B][n][Hkv][d]
    const uint64_t d[4] = {kD, static_cast<uint64_t>(p.Hkv), static_cast<uint64_t>(p.n), static_cast<uint64_t>(p.B)};
    const uint64_t s[3] = {row, row * p.Hkv, row * p.Hkv * p.n};
    const uint32_t bx[4] = {64, 1, kBN, 1};
    ok &= tc::make_map(&a.tm_kn, bf, p.k, 4, d, s, bx, sw);
    ok &= tc::make_map(&a.tm_vn, bf, p.v, 4, d, s, bx, sw);
  }
  {  // retrieval cache [B*Hr][cap][d]
    const uint64_t d[3] = {kD, static_cast<uint64_t>(p.max_len), static_cast<uint64_t>(p.B) * (p.Hr > 0 ? p.Hr : 1)};
    const uint64_t s[2] = {row, row * p.max_len};
    const uint32_t bx[3] = {64, kBN, 1};
    ok &= tc::make_map(&a.tm_kc, bf, rk, 3, d, s, bx, sw);
    ok &= tc::make_map(&a.tm_vc, bf, rv, 3, d, s, bx, sw);
  }
  {  // streaming history [B*HsMax][S+W][d]
    const uint64_t d[3] = {kD, static_cast<uint64_t>(p.S + p.W), static_cast<uint64_t>(p.B) * (p.HsMax > 0 ? p.HsMax : 1)};
    const uint64_t s[2] = {row, row * (p.S + p.W)};
    const uint32_t bx[3] = {64, kBN, 1};
    ok &= tc::make_map(&a.tm_kh, bf, hk, 3, d, s, bx, sw);
    ok &= tc::make_map(&a.tm_vh, bf, hv, 3, d, s, bx, sw);
  }
  if (!ok) return cudaErrorInvalidValue;
  static std::atomic<uint64_t> attr{0};
  return opt_in_smem(prefill_tc_kernel, kSmemAlloc, attr);
}

cudaError_t launch_prefill_tc(const PrefillTcLaunch &l, cudaStream_t st) {
  const PrefillParams &p = l.p;
  const int npos = kBM / p.G;
  const int ntq = (p.n + npos - 1) / npos;
  const int grid = (ntq + kQT - 1) / kQT * p.B * p.Hkv;
  prefill_tc_kernel<<<grid, kTcThreads, kSmemAlloc, st>>>(l);
  return cudaGetLastError();
}

}  // namespace duo
