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
//     hold no visible key for any row of a query tile are never loaded (tile skip).
//
// One CTA = one 128-row query tile (a GQA group of heads x 128/G positions); 19 warps:
//   warp 0      TMA producer: Q once, then K tiles of 128 keys into a 3-stage ring
//   warp 18     TMA producer: V tiles into a 2-stage ring
//   warp 1      TMEM allocator; lane 0 issues every tcgen05.mma
//   warps 2..17 softmax: four threads per query row (TMEM lane), 32 columns each, so
//               that 16 warps hide the latency of the tensor-memory loads
// TMEM (512 columns): S double buffer at 0 and 128, O accumulator at 256, P (bf16
// pairs) double buffer at 384 and 448.
//   S_j = Q K_j^T      (M 128, N 128, K 128: 8 MMAs of K 16), into S[j % 2]
//   O += P_j V_j       (M 128, N 128, K 128 keys), A = P_j from TMEM, B = V_j (smem)
// The softmax warps read S_j once from TMEM, release it, and write P_j (bf16) back
// into TMEM; O stays in TMEM and is rescaled there only when a row's maximum grows
// past its reference by 2^8.  K stages are released as soon as S_j is computed and V
// stages once P_j V_j is, so the tensor core computes S_{j+1} and P_j V_j while the
// softmax warps work.
//
// Every mbarrier wait is bounded; a wait that runs out latches kDevTimeout in the
// status word and sets an abort flag so that every role drains and exits (the
// producers first wait, bounded, for the loads they issued).
#include "tcgen05.cuh"

namespace duo {

namespace {

constexpr int kBM = 128;  // query rows per tile
constexpr int kBN = 128;  // keys per tile
constexpr int kSplit = 4;                      // softmax threads per query row
constexpr int kCols = kBN / kSplit;            // S, P and O columns per softmax thread
constexpr int kVWarp = 2 + 4 * kSplit;         // the V producer follows the softmax warps
constexpr int kTcThreads = 32 * (kVWarp + 1);  // warp 0 K/Q TMA, warp 1 MMA + TMEM, softmax, V TMA
constexpr int kD = 128;
constexpr int kKStages = 3;  // K ring: a stage is free once S_j is computed
constexpr int kVStages = 2;  // V ring: a stage is free once P_j V_j is computed
constexpr int kMaxStrmTiles = 48;

// shared memory map (bytes from the 1 KiB-aligned base); every tile is two 128B-swizzled
// [128][64] bf16 halves of 16 KiB
constexpr int kSmQ = 0;
constexpr int kSmK = 32768;                         // K stage s at kSmK + s * 32 KiB
constexpr int kSmV = kSmK + kKStages * 32768;       // V stage s at kSmV + s * 32 KiB
constexpr int kSmBar = kSmV + kVStages * 32768;
constexpr int kSmMisc = kSmBar + 256;
constexpr int kSmXchg = kSmMisc + 1024 + kMaxStrmTiles * 16;  // row max / sum exchange, 3 kSplit x 128 floats
constexpr int kSmTotal = kSmXchg + 3 * kSplit * 128 * 4;
constexpr int kSmemAlloc = kSmTotal + 1024;  // slack for aligning the base to 1 KiB

// TMEM columns: S double buffer, O accumulator, P double buffer (bf16 pairs, A operand)
constexpr int kTmS = 0, kTmO = 256, kTmP = 384;

// barrier indices (8 bytes each).  Double-buffered resources (S, P) have one barrier
// per buffer, so that no barrier can complete two phases ahead of a thread waiting on
// it (parity waits).
constexpr int kBarQ = 0, kBarKFull = 1, kBarKEmpty = kBarKFull + kKStages, kBarVFull = kBarKEmpty + kKStages,
              kBarVEmpty = kBarVFull + kVStages, kBarSFull = kBarVEmpty + kVStages, kBarSFree = kBarSFull + 2,
              kBarPFull = kBarSFree + 2, kBarOFull = kBarPFull + 2, kBarDrain = kBarOFull + 1, kNumBars = kBarDrain + 1;
static_assert(kNumBars * 8 <= 256, "barrier area");

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

// ---- packed fp32 pairs (sm_100 f32x2 arithmetic: two lanes per instruction) ----
__device__ __forceinline__ uint64_t pack2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void unpack2(uint64_t v, float &a, float &b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^x of a pair on the FMA pipe: x = n + f with n the nearest integer (|f| <= 1/2),
// 2^f by a cubic fitted for this kernel by weighted least squares on [-1/2, 1/2]
// (maximum relative error 1.0e-4, below bf16's 2^-9), and n added to the exponent
// field.  Arguments below -126 give 2^-126 (the callers' tiles hold no -inf).
__device__ __forceinline__ void exp2_poly2(uint64_t x2, float &r0, float &r1) {
  float x0, x1;
  unpack2(x2, x0, x1);
  x2 = pack2(fmaxf(x0, -126.0f), fmaxf(x1, -126.0f));
  const uint64_t t = fadd2(x2, pack2(12582912.0f, 12582912.0f));  // 1.5 * 2^23: rounds to an integer
  const uint64_t n = fadd2(t, pack2(-12582912.0f, -12582912.0f));
  const uint64_t f = ffma2(n, pack2(-1.0f, -1.0f), x2);  // x - n, exact
  uint64_t q = ffma2(pack2(0.05500858f, 0.05500858f), f, pack2(0.24221036f, 0.24221036f));
  q = ffma2(q, f, pack2(0.6932829f, 0.6932829f));
  q = ffma2(q, f, pack2(1.0f, 1.0f));
  float q0, q1, t0, t1;
  unpack2(q, q0, q1);
  unpack2(t, t0, t1);
  r0 = __int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23));
  r1 = __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23));
}

// exp2(v*c - mc) of N logits, their sum into rowsum and bf16 pairs into pk; logits
// [P0, P0+PN) use the FMA-pipe polynomial (which needs finite arguments), the rest MUFU.
// The scaling and the sums run on packed fp32 pairs.
template <int N, int P0, int PN>
__device__ __forceinline__ void probabilities(const float (&v)[N], float c, float mc, float &rowsum,
                                              uint32_t (&pk)[N / 2]) {
  const uint64_t cc = pack2(c, c), mm = pack2(-mc, -mc);
  uint64_t acc[2] = {pack2(0.f, 0.f), pack2(0.f, 0.f)};
#pragma unroll
  for (int e = 0; e < N; e += 2) {
    const uint64_t x = ffma2(pack2(v[e], v[e + 1]), cc, mm);
    float p0, p1;
    if (e >= P0 && e < P0 + PN) {
      exp2_poly2(x, p0, p1);
    } else {
      float x0, x1;
      unpack2(x, x0, x1);
      p0 = ex2(x0);
      p1 = ex2(x1);
    }
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

  // ---- which query tile ----
  // GQA packing: the 128 rows of the tile are npos = 128 / G consecutive positions x the
  // G query heads of one KV head (row r = position r / G, head r % G), so every K/V tile
  // a CTA loads serves the whole group.
  const int G = p.G;
  const int npos = kBM / G;
  const int ntq = (p.n + npos - 1) / npos;
  const int bg = blockIdx.x % (p.B * p.Hkv);
  const int qt = ntq - 1 - blockIdx.x / (p.B * p.Hkv);  // heaviest (latest) blocks first
  const int b = bg / p.Hkv, g = bg % p.Hkv;
  const int r0 = qt * npos;  // first chunk row (position offset) of the block
  Plan pl;
  pl.retr = p.hm.is_retr[g] != 0;
  pl.nh = pl.retr ? static_cast<int>((p.len + kBN - 1) / kBN) : 0;
  pl.q0 = p.len + r0;
  pl.kvrow = b * (pl.retr ? p.Hr : p.HsMax) + p.hm.kind_idx[g];

  if (tid == 0) {
    for (int i = 0; i < kNumBars; ++i)
      mbar_init(bar(i), (i == kBarSFree || i == kBarSFree + 1 || i == kBarPFull || i == kBarPFull + 1) ? 128 * kSplit : 1);
    if (smem_u32(smem) & 1023u) flag_status(p.status, kDevTimeout);  // layout assumption (never expected)
    fence_mbar_init();
    *abort_flag = 0;
    int nt;
    if (pl.retr) {
      const int rows = (r0 + npos < p.n) ? r0 + npos : p.n;  // chunk rows 0 .. rows-1 are needed
      nt = pl.nh + (rows + kBN - 1) / kBN;
    } else {
      nt = streaming_tiles(p, r0, npos, tl);
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
    // ================= TMA producer: Q, then the K ring =================
    if (lane == 0) {
      tc::prefetch_map(&a.tm_q);
      mbar_expect_tx(bar(kBarQ), 32768);
      tc::tma_4d(sbase + kSmQ, &a.tm_q, 0, g * G, r0, b, bar(kBarQ));  // box: 64 dims x G heads x npos positions
      tc::tma_4d(sbase + kSmQ + 16384, &a.tm_q, 64, g * G, r0, b, bar(kBarQ));
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
  } else if (warp == kVWarp) {
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
      bool ok = tc::wait_bar(bar(kBarQ), 0, p.status, abort_flag);
      auto issue_pv = [&](int jj) {
        // O += P_jj V_jj : K = 128 keys in 8 steps of 16; P from TMEM (bf16 pairs, K-major),
        // V from shared memory (d contiguous, MN-major)
        const int sv = jj % kVStages;
        const uint32_t vbase = sbase + kSmV + sv * 32768;
        const uint32_t pcol = tmem + kTmP + (jj & 1) * 64;
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t bd = tc::sdesc(vbase + kk * 2048, 16384, 1024);
          tc::mma_ts(tmem + kTmO, pcol + kk * 8, bd, kIdPV, (jj > 0 || kk > 0) ? 1u : 0u);
        }
        tc::commit(bar(kBarOFull));
        tc::commit(bar(kBarVEmpty + sv));
      };
      for (int j = 0; j < nt && ok; ++j) {
        const int sk = j % kKStages;
        if (!tc::wait_bar(bar(kBarKFull + sk), (j / kKStages) & 1, p.status, abort_flag)) { ok = false; break; }
        if (j >= 2 && !tc::wait_bar(bar(kBarSFree + (j & 1)), ((j - 2) >> 1) & 1, p.status, abort_flag)) { ok = false; break; }
        tc::fence_after();
        // S_j = Q K_j^T : K = d 128 in 8 steps of 16; Q and K are K-major
        const uint32_t kbase = sbase + kSmK + sk * 32768;
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          tc::mma_ss(tmem + kTmS + (j & 1) * 128, tc::sdesc(sbase + kSmQ + off, 16, 1024),
                     tc::sdesc(kbase + off, 16, 1024), kIdS, kk > 0 ? 1u : 0u);
        }
        tc::commit(bar(kBarSFull + (j & 1)));
        tc::commit(bar(kBarKEmpty + sk));
        if (j >= 1) {
          if (!tc::wait_bar(bar(kBarPFull + ((j - 1) & 1)), ((j - 1) >> 1) & 1, p.status, abort_flag)) { ok = false; break; }
          if (!tc::wait_bar(bar(kBarVFull + ((j - 1) % kVStages)), ((j - 1) / kVStages) & 1, p.status, abort_flag)) { ok = false; break; }
          tc::fence_after();
          issue_pv(j - 1);
        }
      }
      if (ok && nt > 0 && tc::wait_bar(bar(kBarPFull + ((nt - 1) & 1)), ((nt - 1) >> 1) & 1, p.status, abort_flag) &&
          tc::wait_bar(bar(kBarVFull + ((nt - 1) % kVStages)), ((nt - 1) / kVStages) & 1, p.status, abort_flag)) {
        tc::fence_after();
        issue_pv(nt - 1);
      }
      // drain: every MMA this thread issued has completed before TMEM is freed
      tc::commit(bar(kBarDrain));
      mbar_wait(bar(kBarDrain), 0, p.status);
    }
  } else {
    // ================= softmax: 4 kSplit warps, kSplit threads per query row =================
    // Warp w reads TMEM lanes 32*(w%4).. (rows) and columns [kCols*part, kCols*part+kCols)
    // of S, O and P.  The running max m is a reference: P = exp2(s*c - m) may exceed 1 by
    // up to 2^kSlack, and m (with O in TMEM and l) is rescaled only when a row's tile
    // maximum passes m + kSlack.  S is read from TMEM once per tile.
    constexpr float kSlack = 8.0f;
    constexpr int kSoft = 128 * kSplit;  // softmax threads (named barrier 1)
    const int wq = warp & 3;
    const int part = (warp - 2) >> 2;
    const int row = (wq << 5) | lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq << 5) << 16);
    const int rpos = row / G;                  // position offset of this row within the block
    const int h = g * G + row % G;             // its query head
    const int64_t i = pl.q0 + rpos;            // absolute query position
    const float c = p.scale_log2;
    float m = -INFINITY, l = 0.f;
    float *xch = reinterpret_cast<float *>(smem + kSmXchg);  // [tile parity][part][row] partial maxima
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

      if (ok) ok = tc::wait_bar(bar(kBarSFull + (j & 1)), (j >> 1) & 1, p.status, abort_flag);
      tc::fence_after();
      // this thread's kCols logits of S_j, then the S buffer is released
      float v[kCols];
      tc::ld<kCols>(lane_base + kTmS + (j & 1) * 128 + part * kCols, v);
      tc::fence_before();
      mbar_arrive(bar(kBarSFree + (j & 1)));
      if (!full_vis) {
#pragma unroll
        for (int e = 0; e < kCols; ++e) {
          const int col = part * kCols + e;
          const bool vis = col <= hi && (col < sink_c || col > win_c);
          v[e] = vis ? v[e] : -INFINITY;
        }
      }
      float mx4[4];  // four independent chains of three-input maxima
#pragma unroll
      for (int u = 0; u < 4; ++u) mx4[u] = fmaxf(v[2 * u], v[2 * u + 1]);
#pragma unroll
      for (int e = 8; e < kCols; e += 2) mx4[(e >> 1) & 3] = fmax3(mx4[(e >> 1) & 3], v[e], v[e + 1]);
      float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
      xch[((j & 1) * kSplit + part) * kBM + row] = mx;
      tc::named_sync(1, kSoft);
#pragma unroll
      for (int o = 1; o < kSplit; ++o) mx = fmaxf(mx, xch[((j & 1) * kSplit + ((part + o) % kSplit)) * kBM + row]);
      const float tmax = mx * c;  // -inf when nothing in the tile is visible
      const bool need = tmax > m + kSlack;
      float alpha = 1.f;
      if (need) {
        alpha = ex2(m - tmax);  // 0 while m is -inf
        m = tmax;
      }
      l *= alpha;
      bool waited = false;
      if (j >= 1 && __any_sync(0xffffffffu, need)) {
        // rescale this thread's kCols columns of O once P_{j-1} V_{j-1} has landed
        if (ok) ok = tc::wait_bar(bar(kBarOFull), (j - 1) & 1, p.status, abort_flag);
        tc::fence_after();
        float w[kCols];
        const uint32_t oa = lane_base + kTmO + part * kCols;
        tc::ld<kCols>(oa, w);
#pragma unroll
        for (int e = 0; e < kCols; ++e) w[e] *= alpha;
        tc::st32(oa, w);
        waited = true;
      }
      // probabilities (masked logits are -inf and give 0), row sum, bf16 pairs of P_j
      float rsum;
      const float mc = (m == -INFINITY) ? 0.f : m;
      uint32_t pk[kCols / 2];
      // 3/8 of the exponentials of interior tiles on the FMA pipe, the rest on MUFU
      if (!full_vis) probabilities<kCols, 0, 0>(v, c, mc, rsum, pk);
      else probabilities<kCols, 0, kCols * 3 / 8>(v, c, mc, rsum, pk);
      // P_j into TMEM buffer j % 2 (its previous reader P_{j-2} V_{j-2} was waited for at j-1)
      tc::st16(lane_base + kTmP + (j & 1) * 64 + part * (kCols / 2), pk);
      tc::st_wait();
      // one wait per P V product, in order (here unless the rescale already waited)
      if (j >= 1 && !waited) {
        if (ok) ok = tc::wait_bar(bar(kBarOFull), (j - 1) & 1, p.status, abort_flag);
      }
      l += rsum;
      tc::fence_before();
      mbar_arrive(bar(kBarPFull + (j & 1)));
    }
    // the last product, then the row's normaliser from all parts
    if (nt > 0 && ok) ok = tc::wait_bar(bar(kBarOFull), (nt - 1) & 1, p.status, abort_flag);
    tc::fence_after();
    float *xl = xch + 2 * kSplit * kBM;  // [part][row]
    xl[part * kBM + row] = l;
    tc::named_sync(1, kSoft);
    float lrow = 0.f;
#pragma unroll
    for (int o = 0; o < kSplit; ++o) lrow += xl[o * kBM + row];
    // epilogue: normalise and store this thread's kCols dims of the row (bf16) and its lse;
    // in gated mixing, blend with the row already in out
    const bool store = r0 + rpos < p.n;
    char *orow = p.out + ((static_cast<int64_t>(b) * p.n + r0 + rpos) * p.Hq + h) * (kD * 2) + part * (kCols * 2);
    const float inv = 1.f / lrow;
    const float mixa = p.mix_alpha ? p.mix_alpha[g] : 0.f;
    {
      float w[kCols];
      tc::ld<kCols>(lane_base + kTmO + part * kCols, w);
      if (store) {
#pragma unroll
        for (int q = 0; q < kCols / 8; ++q) {
          float x[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) x[e] = w[8 * q + e] * inv;
          if (p.mix_alpha) {
            const uint4 old = *reinterpret_cast<const uint4 *>(orow + q * 16);
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
          *reinterpret_cast<uint4 *>(orow + q * 16) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
        }
      }
    }
    if (store && part == 0 && p.lse) p.lse[(static_cast<int64_t>(b) * p.n + r0 + rpos) * p.Hq + h] = (m + lg2(lrow)) * kLn2;
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
  const int win_tiles = (p.W + 2 * kBN - 2) / kBN + 1;
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
  const int grid = ntq * p.B * p.Hkv;
  prefill_tc_kernel<<<grid, kTcThreads, kSmemAlloc, st>>>(l);
  return cudaGetLastError();
}

}  // namespace duo
