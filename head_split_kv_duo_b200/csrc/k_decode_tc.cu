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
#include "decode_merge.cuh"
#include "tcgen05.cuh"

namespace duo {

namespace {

constexpr int kThreads = 224;  // warp 0 TMA, warp 1 MMA + TMEM, warps 2-5 softmax, warp 6 append
constexpr int kTile = 128;
constexpr int kD = 128;
constexpr int kN = 16;         // padded query heads per item
constexpr int kStages = 3;
// Tiles of its range a CTA asks L2 to fetch before the previous grid on the stream has
// finished: that grid's tail (its last CTAs and their merges) leaves HBM mostly idle.
constexpr int kPrefetch = 4;
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
              kBarDrain = 14, kBarAppend = 15, kBarMerge = 16,
              kBarStall = 17,  // test control: nothing ever arrives here
              kNumBars = 18;

// ---- work plans: how the flattened 128-token units of a launch map onto items ----
//
// An item is one (sequence, KV head) of the launch; its units are its 128-token tiles.
// The units of all items are laid end to end and cut into one equal range per CTA.
struct Item {
  int64_t ua;   // its first unit
  int units;    // its tiles
  int ordinal;  // its position among the launch's items (in unit order)
  int retr;     // 1: retrieval head (keys 0 .. len-1); 0: streaming head (sinks + ring)
  int g;        // KV head: query heads g*G .. g*G+G-1
  int kidx;     // index among the heads of its kind
  int bq;       // row block of q / out / lse: rows bq * Hq + h
  int zrow;     // contiguous cache: z of its K/V in the tensor maps; pool: sequence slot
  int layer;    // pool: layer
  int64_t len;  // tokens held (the query is position len - 1)
};

// Contiguous cache: items are the batch's retrieval heads (b, ri), then its streaming
// heads (b, si); every retrieval item has units_r tiles, every streaming item units_s.
struct ContigPlan {
  static constexpr bool kPool = false;
  int units_r, units_s;  // units per retrieval / streaming item
  int n_items_r;         // B * Hr
  int64_t total_units;
  int num_ctas;
  CUtensorMap tm_q, tm_kr, tm_vr, tm_ks, tm_vs;
};

// Pool: (layer, sequence) pairs i = (layer - layer0) * nseq + s, each with its layer's
// retrieval heads (pages through the block table) then its streaming heads.
struct PoolPlan {
  static constexpr bool kPool = true;
  int64_t total_units;
  int num_ctas;
  int n_super;                       // nlayers * nseq
  PoolDecodeCall c;
  int uprefix[kPoolMaxSuper + 1];    // units before pair i
  CUtensorMap tm_q;                  // q [nlayers * nseq * Hq][d]
};

template <class Plan>
struct TcArgs {
  DecodeParams p;
  Plan pl;
};

// unit u -> its item, and the tile of u within it
__device__ __forceinline__ Item item_at(const TcArgs<ContigPlan> &a, int64_t u, int &tile) {
  const DecodeParams &p = a.p;
  const ContigPlan &pl = a.pl;
  const int64_t ur = static_cast<int64_t>(pl.n_items_r) * pl.units_r;
  Item it;
  it.len = p.len;
  it.layer = 0;
  if (u < ur) {
    const int idx = static_cast<int>(u / pl.units_r);
    tile = static_cast<int>(u % pl.units_r);
    it.retr = 1;
    it.kidx = idx % p.Hr;
    it.bq = idx / p.Hr;
    it.g = p.hm.retr_head[it.kidx];
    it.zrow = idx;  // b * Hr + ri
    it.ua = static_cast<int64_t>(idx) * pl.units_r;
    it.units = pl.units_r;
    it.ordinal = idx;
  } else {
    const int idx = static_cast<int>((u - ur) / pl.units_s);
    tile = static_cast<int>((u - ur) % pl.units_s);
    it.retr = 0;
    it.kidx = idx % p.Hs;
    it.bq = idx / p.Hs;
    it.g = p.hm.strm_head[it.kidx];
    it.zrow = idx;  // b * Hs + si
    it.ua = ur + static_cast<int64_t>(idx) * pl.units_s;
    it.units = pl.units_s;
    it.ordinal = pl.n_items_r + idx;
  }
  return it;
}

__device__ __forceinline__ Item item_at(const TcArgs<PoolPlan> &a, int64_t u, int &tile) {
  const DecodeParams &p = a.p;
  const PoolPlan &pl = a.pl;
  int lo = 0, hi = pl.n_super - 1;  // the last pair i with uprefix[i] <= u
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pl.uprefix[mid] <= u) lo = mid;
    else hi = mid - 1;
  }
  const int i = lo, s = i % pl.c.nseq;
  Item it;
  it.layer = pl.c.layer0 + i / pl.c.nseq;
  const PoolLayerDesc &L = pl.c.layers[it.layer];
  const int Hr = L.Hr;
  it.len = pl.c.len[s];
  const int ur = static_cast<int>((it.len + kTile - 1) / kTile);
  const int64_t used = p.S + it.len < static_cast<int64_t>(p.S) + p.W ? p.S + it.len : static_cast<int64_t>(p.S) + p.W;
  const int us = static_cast<int>((used + kTile - 1) / kTile);
  const int64_t v = u - pl.uprefix[i];
  if (v < static_cast<int64_t>(Hr) * ur) {
    it.retr = 1;
    it.kidx = static_cast<int>(v / ur);
    tile = static_cast<int>(v % ur);
    it.g = L.hm.retr_head[it.kidx];
    it.ua = pl.uprefix[i] + static_cast<int64_t>(it.kidx) * ur;
    it.units = ur;
    it.ordinal = i * p.Hkv + it.kidx;
  } else {
    const int64_t v2 = v - static_cast<int64_t>(Hr) * ur;
    it.retr = 0;
    it.kidx = static_cast<int>(v2 / us);
    tile = static_cast<int>(v2 % us);
    it.g = L.hm.strm_head[it.kidx];
    it.ua = pl.uprefix[i] + static_cast<int64_t>(Hr) * ur + static_cast<int64_t>(it.kidx) * us;
    it.units = us;
    it.ordinal = i * p.Hkv + Hr + it.kidx;
  }
  it.bq = i;
  it.zrow = pl.c.slot[s];
  return it;
}

// Walks a CTA's units in order.
template <class Plan>
struct UnitIter {
  Item it;
  int tile;
  __device__ __forceinline__ UnitIter(const TcArgs<Plan> &a, int64_t u) { it = item_at(a, u, tile); }
  __device__ __forceinline__ void next(const TcArgs<Plan> &a) {
    if (++tile == it.units) it = item_at(a, it.ua + it.units, tile);
  }
};

// first unit of CTA c: floor(c * U / C); the CTA holding unit u: ceil((u+1) C / U) - 1
template <class Plan>
__device__ __forceinline__ int64_t cta_begin(const TcArgs<Plan> &a, int c) {
  return static_cast<int64_t>(c) * a.pl.total_units / a.pl.num_ctas;
}
template <class Plan>
__device__ __forceinline__ int cta_of(const TcArgs<Plan> &a, int64_t u) {
  return static_cast<int>(((u + 1) * a.pl.num_ctas + a.pl.total_units - 1) / a.pl.total_units) - 1;
}

// Split-merge scratch of an item: its segment-0 partial rows and its ticket.  Contiguous
// cache: max_splits slots per (batch, KV head).  Pool: the segments of the item in unit
// order o occupy slots cfirst + o .. clast + o, which no other item of the launch uses.
__device__ __forceinline__ float *part_base(const TcArgs<ContigPlan> &a, const Item &it, int /*cfirst*/) {
  const int64_t pitem = static_cast<int64_t>(it.bq) * a.p.Hkv + it.g;
  return a.p.partials + pitem * a.p.max_splits * a.p.G * kPartRow;
}
__device__ __forceinline__ float *part_base(const TcArgs<PoolPlan> &a, const Item &it, int cfirst) {
  return a.p.partials + static_cast<int64_t>(cfirst + it.ordinal) * a.p.G * kPartRow;
}
__device__ __forceinline__ uint32_t *ticket_of(const TcArgs<ContigPlan> &a, const Item &it) {
  return a.p.counters + static_cast<int64_t>(it.bq) * a.p.Hkv + it.g;
}
__device__ __forceinline__ uint32_t *ticket_of(const TcArgs<PoolPlan> &a, const Item &it) {
  return a.p.counters + it.ordinal;
}

// TMA of the K and V rows of (item, tile) and of the item's queries into one stage.
__device__ __forceinline__ void load_stage(const TcArgs<ContigPlan> &a, const Item &it, int tile, uint32_t dst,
                                           uint32_t fb) {
  const CUtensorMap *mk = it.retr ? &a.pl.tm_kr : &a.pl.tm_ks, *mv = it.retr ? &a.pl.tm_vr : &a.pl.tm_vs;
  const int y = tile * kTile, z = it.zrow;
  tc::tma_3d(dst + kStK, mk, 0, y, z, fb);
  tc::tma_3d(dst + kStK + 16384, mk, 64, y, z, fb);
  tc::tma_3d(dst + kStV, mv, 0, y, z, fb);
  tc::tma_3d(dst + kStV + 16384, mv, 64, y, z, fb);
  const int qrow = it.bq * a.p.Hq + it.g * a.p.G;  // rows beyond this group's G heads are never used
  tc::tma_2d(dst + kStQ, &a.pl.tm_q, 0, qrow, fb);
  tc::tma_2d(dst + kStQ + 2048, &a.pl.tm_q, 64, qrow, fb);
}
__device__ __forceinline__ void load_stage(const TcArgs<PoolPlan> &a, const Item &it, int tile, uint32_t dst,
                                           uint32_t fb) {
  const PoolLayerDesc &L = a.pl.c.layers[it.layer];
  const CUtensorMap *mk, *mv;
  int y, z;
  if (it.retr) {  // page `tile` of the sequence: z = page * Hr + ri, all 128 rows
    // the block table was written by the append launch before this one (L2, not L1)
    const int page = __ldcg(a.pl.c.table + static_cast<int64_t>(it.zrow) * a.pl.c.pages_per_seq + tile);
    mk = &L.tm_kr;
    mv = &L.tm_vr;
    y = 0;
    z = page * L.Hr + it.kidx;
  } else {
    mk = &L.tm_ks;
    mv = &L.tm_vs;
    y = tile * kTile;
    z = it.zrow * L.Hs + it.kidx;
  }
  tc::tma_3d(dst + kStK, mk, 0, y, z, fb);
  tc::tma_3d(dst + kStK + 16384, mk, 64, y, z, fb);
  tc::tma_3d(dst + kStV, mv, 0, y, z, fb);
  tc::tma_3d(dst + kStV + 16384, mv, 64, y, z, fb);
  const int qrow = it.bq * a.p.Hq + it.g * a.p.G;
  tc::tma_2d(dst + kStQ, &a.pl.tm_q, 0, qrow, fb);
  tc::tma_2d(dst + kStQ + 2048, &a.pl.tm_q, 64, qrow, fb);
}

template <int NQ, class Plan>
__global__ void __launch_bounds__(kThreads, 1) decode_tc_kernel(const __grid_constant__ TcArgs<Plan> a) {
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
  // A decode launched next on the stream may start its set-up on the SMs this grid
  // frees; it touches global memory only after its own griddepcontrol.wait, which
  // returns once this whole grid has completed.  A leading grid (pdl_mode 1) releases
  // its dependent only after its own wait (below).
  if (p.pdl_mode != 1) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
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
    tc::tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  }
  tc::fence_async_smem();
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ================= TMA producer =================
    if (lane == 0) {
      if constexpr (!Plan::kPool) {
        for (const CUtensorMap *m : {&a.pl.tm_q, &a.pl.tm_kr, &a.pl.tm_vr, &a.pl.tm_ks, &a.pl.tm_vs})
          tc::prefetch_map(m);
        // L2 prefetch of the first tiles; no data is consumed before the wait below
        UnitIter<Plan> it(a, u0);
        for (int j = 0; j < nu && j < kPrefetch; ++j, it.next(a)) {
          const int64_t y = static_cast<int64_t>(it.tile) * kTile;
          const int64_t rows = it.it.retr ? p.max_len : static_cast<int64_t>(p.S) + p.W;
          const int64_t base = (static_cast<int64_t>(it.it.zrow) * rows + y) * kD * 2;
          const uint32_t bytes = static_cast<uint32_t>((rows - y < kTile ? rows - y : kTile) * kD * 2);
          prefetch_l2((it.it.retr ? p.rk : p.sk) + base, bytes);
          prefetch_l2((it.it.retr ? p.rv : p.sv) + base, bytes);
        }
      } else {
        tc::prefetch_map(&a.pl.tm_q);
      }
      // Launched as a programmatic dependent, this grid's set-up overlaps the previous
      // kernel on the stream; nothing is read from global memory before that kernel has
      // finished (every other read and every write of this grid follows this wait or the
      // append warp's).
      asm volatile("griddepcontrol.wait;" ::: "memory");
      if (p.pdl_mode == 1) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    }
    if (lane == 0) {
      // contiguous cache, fused append: the tile of each item that holds the appended row
      // waits for the append warp (retrieval: row npos; streaming: the row's slot)
      const int64_t tile_r = p.npos / kTile, tile_s = (p.npos < p.S ? p.npos : p.S + p.npos % p.W) / kTile;
      bool appended = Plan::kPool || p.nk == nullptr;
      int issued = 0, layer_seen = -1;
      UnitIter<Plan> it(a, u0);
      for (int j = 0; j < nu; ++j, it.next(a)) {
        const int s = j % kStages;
        if (j >= kStages && !tc::wait_bar(bar(kBarEmpty + s), ((j / kStages) - 1) & 1, p.status, abort_flag)) break;
        if (!appended && it.tile == (it.it.retr ? tile_r : tile_s)) {
          if (!tc::wait_bar(bar(kBarAppend), 0, p.status, abort_flag)) break;
          asm volatile("fence.proxy.async.global;" ::: "memory");
          appended = true;
        }
        if constexpr (Plan::kPool) {
          if (it.it.layer != layer_seen) {
            // the layer's tensor maps live in device memory (written by the host before
            // the launch): order them for the TMA's view of them
            layer_seen = it.it.layer;
            const PoolLayerDesc *L = a.pl.c.layers + layer_seen;
            for (const CUtensorMap *m : {&L->tm_kr, &L->tm_vr, &L->tm_ks, &L->tm_vs})
              asm volatile("fence.proxy.tensormap::generic.acquire.gpu [%0], 128;" ::"l"(m) : "memory");
          }
        }
        const uint32_t dst = sbase + s * kStage;
        const uint32_t fb = bar(kBarFull + s);
        mbar_expect_tx(fb, 65536 + 4096);
        load_stage(a, it.it, it.tile, dst, fb);
        ++issued;
      }
      // after an abort, loads may still be landing: none may outlive the CTA
      tc::drain_loads(bar(kBarFull), kStages, issued, p.status);
    }
  } else if (warp == 1) {
    // ================= MMA issuer =================
    if (lane == 0) {
      constexpr uint32_t kIdS = tc::idesc_bf16(128, 16, false, false);
      constexpr uint32_t kIdO = tc::idesc_bf16(128, 16, true, false);
      bool ok = true;
      // descriptors of every operand base; a K step adds its byte offset >> 4
      const uint64_t dk0 = tc::sdesc(sbase + kStK, 16, 1024);      // K tile, K-major
      const uint64_t dq0 = tc::sdesc(sbase + kStQ, 16, 1024);      // Qpad, K-major
      const uint64_t dv0 = tc::sdesc(sbase + kStV, 16384, 1024);   // V^T, MN-major
      const uint64_t dp0 = tc::sdesc(sbase + kSmP, 16, 1024);      // P^T, K-major
      auto issue_o = [&](int jj) {
        const int s = jj % kStages;
        const uint64_t dv = dv0 + s * (kStage >> 4);
        const uint64_t dp = dp0 + (jj & 1) * (4096 >> 4);
        const uint32_t d = tmem + kTmO + (jj & 1) * kAcc * 16;
#pragma unroll
        for (int i = 0; i < 8; ++i) {  // K = 128 tokens in steps of 16, kAcc independent chains
          const int kk = (i % kAcc) * (8 / kAcc) + i / kAcc;
          tc::mma_ss(d + (i % kAcc) * 16, dv + kk * 128, dp + (kk >> 2) * 128 + (kk & 3) * 2, kIdO, i >= kAcc ? 1u : 0u);
        }
        tc::commit(bar(kBarOFull + (jj & 1)));
        tc::commit(bar(kBarEmpty + s));
      };
      for (int j = 0; j < nu && ok; ++j) {
        const int s = j % kStages;
        if (!tc::wait_bar(bar(kBarFull + s), (j / kStages) & 1, p.status, abort_flag)) { ok = false; break; }
        if (j >= 2 && !tc::wait_bar(bar(kBarSFree + (j & 1)), ((j - 2) >> 1) & 1, p.status, abort_flag)) { ok = false; break; }
        tc::fence_after();
        const uint64_t dk = dk0 + s * (kStage >> 4), dq = dq0 + s * (kStage >> 4);
        const uint32_t d = tmem + (j & 1) * kAcc * 16;
#pragma unroll
        for (int i = 0; i < 8; ++i) {  // K = d 128 in steps of 16, kAcc independent chains
          const int kk = (i % kAcc) * (8 / kAcc) + i / kAcc;
          tc::mma_ss(d + (i % kAcc) * 16, dk + (kk >> 2) * 1024 + (kk & 3) * 2, dq + (kk >> 2) * 128 + (kk & 3) * 2,
                     kIdS, i >= kAcc ? 1u : 0u);
        }
        tc::commit(bar(kBarSFull + (j & 1)));
        if (j >= 1) {
          if (!tc::wait_bar(bar(kBarPFull + ((j - 1) & 1)), ((j - 1) >> 1) & 1, p.status, abort_flag)) { ok = false; break; }
          tc::fence_after();
          issue_o(j - 1);
        }
      }
      if (ok && nu > 0 && tc::wait_bar(bar(kBarPFull + ((nu - 1) & 1)), ((nu - 1) >> 1) & 1, p.status, abort_flag)) {
        tc::fence_after();
        issue_o(nu - 1);
      }
      tc::commit(bar(kBarDrain));
      mbar_wait(bar(kBarDrain), 0, p.status);
    }
  } else if (warp == 6) {
    // ================= append (contiguous cache only) =================
    if constexpr (!Plan::kPool) {
      if (p.nk) {
        // Fused append ("Decoding Procedure", step 4): the token at position npos goes to
        // row npos of every retrieval head and to slot npos < S ? npos : S + npos mod W of
        // every streaming head.  The only CTA that reads the tile holding that row writes
        // it (lanes 0-15 the K row, 16-31 the V row); the producer loads that tile only
        // after this warp's barrier, so its other loads are not held up by these writes.
        asm volatile("griddepcontrol.wait;" ::: "memory");
        const int64_t slot = p.npos < p.S ? p.npos : p.S + p.npos % p.W;
        int tile0 = 0;
        Item it = item_at(a, u0, tile0);
        while (nu > 0 && it.ua < u1) {
          // the unit of this item whose tile holds the new row, if this CTA owns it
          const int64_t row = it.retr ? p.npos : slot;
          const int64_t u = it.ua + row / kTile;
          if (u >= u0 && u < u1) {
            char *dst;
            if (it.retr)
              dst = const_cast<char *>(lane < 16 ? p.rk : p.rv) + (static_cast<int64_t>(it.zrow) * p.max_len + row) * kD * 2;
            else
              dst = const_cast<char *>(lane < 16 ? p.sk : p.sv) +
                    (static_cast<int64_t>(it.zrow) * (p.S + p.W) + row) * kD * 2;
            const char *src = (lane < 16 ? p.nk : p.nv) + (static_cast<int64_t>(it.bq) * p.Hkv + it.g) * kD * 2;
            reinterpret_cast<uint4 *>(dst)[lane & 15] = reinterpret_cast<const uint4 *>(src)[lane & 15];
          }
          if (it.ua + it.units >= a.pl.total_units) break;
          it = item_at(a, it.ua + it.units, tile0);
        }
        // the rows are read back through the TMA (async proxy)
        asm volatile("fence.proxy.async.global;" ::: "memory");
        __syncwarp();
      }
    }
    if (lane == 0) mbar_arrive(bar(kBarAppend));
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
    int cur = -1;  // ordinal of the item being accumulated
    Item cur_item;

    // Writes this CTA's result for `item` (partial or final) and merges when last.  At
    // the CTA's final flush the stage buffers are idle: the merge then brings the item's
    // partial rows in with one bulk copy instead of a chain of round trips to L2.
    auto flush = [&](const Item &item, bool final_flush) {
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
      const int cfirst = cta_of(a, item.ua), clast = cta_of(a, item.ua + item.units - 1);
      const int nseg = clast - cfirst + 1;
      const int b = item.bq, h0 = item.g * G;
      if (nseg == 1) {
#pragma unroll
        for (int q = 0; q < NQ; ++q)
          if (q < G) {
            Elem<__nv_bfloat16>::store(p.out, (static_cast<int64_t>(b) * p.Hq + h0 + q) * kD + t, o[q] / lt[q]);
            if (t == 0 && p.lse) p.lse[static_cast<int64_t>(b) * p.Hq + h0 + q] = (m[q] + lg2(lt[q])) * kLn2;
          }
        return;
      }
      const int seg = blockIdx.x - cfirst;
      // partial row of (segment, query head): o[0..d), m at d, l at d+1 (16-byte aligned rows)
      constexpr int kRow = kPartRow;
      float *part = part_base(a, item, cfirst);
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
      tc::named_sync(1, 128);
      uint32_t *ticket = ticket_of(a, item);
      if (t == 0) {
        const uint32_t prev = atomicAdd(ticket, 1u);
        *last_flag = (prev == static_cast<uint32_t>(nseg - 1)) ? 1 : 0;
      }
      tc::named_sync(1, 128);
      if (!*last_flag) return;
      __threadfence();
      const uint32_t bytes = static_cast<uint32_t>(nseg) * G * kRow * 4;
      if (final_flush && bytes <= kStages * kStage) {
        if (t == 0) {
          asm volatile("fence.proxy.async.global;" ::: "memory");  // the rows are read by the async proxy
          mbar_expect_tx(bar(kBarMerge), bytes);
          bulk_g2s(sbase, part, bytes, bar(kBarMerge));
        }
        // waited for even after an abort (bounded): the copy must not outlive the CTA
        if (!mbar_wait(bar(kBarMerge), 0, p.status)) ok = false;
        merge_partials<true>(reinterpret_cast<const float *>(smem), nseg, G, b, h0, p.Hq, p.out, p.lse, red + 4 * kN, t, 1);
      } else {
        merge_partials(part, nseg, G, b, h0, p.Hq, p.out, p.lse, red + 4 * kN, t, 1);
      }
      if (t == 0) *ticket = 0u;  // ready for the next call
    };

    // o = (o + O^T(jj)) * alpha for this thread's dimension t
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
    UnitIter<Plan> iter(a, u0);
    for (int j = 0; j < nu; ++j, iter.next(a)) {
      const Item &un = iter.it;
      // test control: a wait that runs out (the bounded-wait and abort paths on a GPU)
      if (j == 0 && p.debug_stall && ok) ok = tc::wait_bar(bar(kBarStall), 0, p.status, abort_flag);
      if (ok) ok = tc::wait_bar(bar(kBarSFull + (j & 1)), (j >> 1) & 1, p.status, abort_flag);
      tc::fence_after();
      float sv[NQ];
      tc::ld_sum<NQ, kAcc>(lane_base + (j & 1) * kAcc * 16, 16, sv);
      tc::fence_before();
      mbar_arrive(bar(kBarSFree + (j & 1)));  // S buffer j % 2 is free again
      // this token's validity
      bool valid;
      const int64_t tok = static_cast<int64_t>(iter.tile) * kTile + t;
      if (un.retr) {
        valid = tok < un.len;
      } else {
        const int S = p.S, W = p.W;
        const int64_t len = un.len;
        const int64_t rstart = (len - W > S) ? len - W : S;
        const int64_t rcount = len > rstart ? len - rstart : 0;
        if (tok >= S + W) valid = false;
        else if (tok < S) valid = tok < len;
        else if (rcount >= W) valid = true;
        else valid = (((tok - S) - (S % W)) % W + W) % W < rcount;
      }
      if (un.ordinal != cur) {
        if (cur >= 0) {
          if (pending) fold(j - 1, one);
          flush(cur_item, false);
        }
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          m[q] = -INFINITY;
          l[q] = 0.f;
          o[q] = 0.f;
        }
        pending = false;
        cur = un.ordinal;
        cur_item = un;
      }
      // does any logit of this tile exceed the reference max by more than kSlack?
      int need = 0;
#pragma unroll
      for (int q = 0; q < NQ; ++q)
        if (q < G && valid && sv[q] * c > m[q] + kSlack) need = 1;
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
      tc::fence_async_smem();
      tc::fence_before();
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
      flush(cur_item, true);
    }
  }

  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  if (warp == 1) tc::tmem_free(tmem, kTmemCols);
}

template <int NQ, class Plan>
cudaError_t launch_nq(const TcArgs<Plan> &a, bool overlap_previous, cudaStream_t st) {
  static std::atomic<uint64_t> attr{0};
  {
    const cudaError_t e = opt_in_smem(decode_tc_kernel<NQ, Plan>, kSmemAlloc, attr);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.pl.num_ctas);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemAlloc;
  cfg.stream = st;
  cudaLaunchAttribute attrs[1];
  attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[0].val.programmaticStreamSerializationAllowed = overlap_previous ? 1 : 0;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, decode_tc_kernel<NQ, Plan>, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <class Plan>
cudaError_t launch_group(const TcArgs<Plan> &a, int G, bool overlap_previous, cudaStream_t st) {
  if (G <= 1) return launch_nq<1>(a, overlap_previous, st);
  if (G <= 2) return launch_nq<2>(a, overlap_previous, st);
  if (G <= 4) return launch_nq<4>(a, overlap_previous, st);
  if (G <= 8) return launch_nq<8>(a, overlap_previous, st);
  return launch_nq<16>(a, overlap_previous, st);
}

bool make_q_map(CUtensorMap *m, const void *q, int64_t rows) {
  const uint64_t d[2] = {kD, static_cast<uint64_t>(rows)};
  const uint64_t s[1] = {kD * 2};
  const uint32_t bx[2] = {64, kN};
  return tc::make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q, 2, d, s, bx, CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

bool decode_tc_supported(const DecodeParams &p, duo_dtype dt, bool int4) {
  return dt == DUO_BF16 && !int4 && p.D == kD && p.G >= 1 && p.G <= kN && tc::encode_fn() != nullptr;
}

cudaError_t launch_decode_tc(const DecodeParams &p, int num_sms, bool overlap_previous, cudaStream_t st) {
  TcArgs<ContigPlan> a{};
  a.p = p;
  ContigPlan &pl = a.pl;
  pl.units_r = static_cast<int>((p.len + kTile - 1) / kTile);
  const int64_t slots = static_cast<int64_t>(p.S) + p.W;
  // highest ring slot in use + 1: position p >= S sits in slot S + p mod W, so before the
  // ring wraps (len <= W) the slots reach S + len - 1, beyond len itself
  const int64_t reach = static_cast<int64_t>(p.S) + p.len;
  const int64_t used = reach < slots ? reach : slots;
  pl.units_s = static_cast<int>((used + kTile - 1) / kTile);
  pl.n_items_r = p.B * p.Hr;
  pl.total_units = static_cast<int64_t>(pl.n_items_r) * pl.units_r + static_cast<int64_t>(p.B) * p.Hs * pl.units_s;
  // at most one CTA per SM, and never more segments per item than partial slots
  int64_t ctas = num_sms;
  if (ctas > pl.total_units) ctas = pl.total_units;
  if (ctas > kMaxSplits) ctas = kMaxSplits;
  pl.num_ctas = static_cast<int>(ctas);
  const uint64_t row = kD * 2;
  bool ok = make_q_map(&pl.tm_q, p.q, static_cast<int64_t>(p.B) * p.Hq);
  {  // retrieval [B*Hr][cap][d]
    const uint64_t d[3] = {kD, static_cast<uint64_t>(p.max_len), static_cast<uint64_t>(p.B) * (p.Hr > 0 ? p.Hr : 1)};
    const uint64_t s[2] = {row, row * p.max_len};
    const uint32_t bx[3] = {64, kTile, 1};
    ok &= tc::make_map(&pl.tm_kr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.rk, 3, d, s, bx, CU_TENSOR_MAP_SWIZZLE_128B);
    ok &= tc::make_map(&pl.tm_vr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.rv, 3, d, s, bx, CU_TENSOR_MAP_SWIZZLE_128B);
  }
  {  // streaming [B*Hs][S+W][d]
    const uint64_t d[3] = {kD, static_cast<uint64_t>(slots), static_cast<uint64_t>(p.B) * (p.Hs > 0 ? p.Hs : 1)};
    const uint64_t s[2] = {row, row * slots};
    const uint32_t bx[3] = {64, kTile, 1};
    ok &= tc::make_map(&pl.tm_ks, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.sk, 3, d, s, bx, CU_TENSOR_MAP_SWIZZLE_128B);
    ok &= tc::make_map(&pl.tm_vs, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.sv, 3, d, s, bx, CU_TENSOR_MAP_SWIZZLE_128B);
  }
  if (!ok) return cudaErrorInvalidValue;
  return launch_group(a, p.G, overlap_previous, st);
}

cudaError_t launch_decode_pool_tc(const DecodeParams &p, const PoolDecodeCall &c, const int *layer_hr,
                                  const int *layer_hs, int num_sms, cudaStream_t st) {
  if (c.nseq < 1 || c.nseq > kPoolMaxSeqs || c.nlayers < 1 || c.nlayers * c.nseq > kPoolMaxSuper)
    return cudaErrorInvalidValue;
  static_assert(sizeof(TcArgs<PoolPlan>) <= 32000, "kernel parameters");
  TcArgs<PoolPlan> a{};
  a.p = p;
  PoolPlan &pl = a.pl;
  pl.c = c;
  pl.n_super = c.nlayers * c.nseq;
  int64_t u = 0;
  for (int i = 0; i < pl.n_super; ++i) {
    pl.uprefix[i] = static_cast<int>(u);
    const int l = c.layer0 + i / c.nseq, s = i % c.nseq;
    const int64_t len = c.len[s];
    const int64_t ur = (len + kTile - 1) / kTile;
    const int64_t used = std::min<int64_t>(static_cast<int64_t>(p.S) + len, static_cast<int64_t>(p.S) + p.W);
    const int64_t us = (used + kTile - 1) / kTile;
    u += layer_hr[l] * ur + layer_hs[l] * us;
  }
  if (u >= (int64_t(1) << 31)) return cudaErrorInvalidValue;
  pl.uprefix[pl.n_super] = static_cast<int>(u);
  pl.total_units = u;
  int64_t ctas = num_sms;
  if (ctas > pl.total_units) ctas = pl.total_units;
  pl.num_ctas = static_cast<int>(ctas);
  if (!make_q_map(&pl.tm_q, p.q, static_cast<int64_t>(pl.n_super) * p.Hq)) return cudaErrorInvalidValue;
  return launch_group(a, p.G, true, st);
}

}  // namespace duo
