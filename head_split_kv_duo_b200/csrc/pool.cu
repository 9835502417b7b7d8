// pool.cu -- a paged pool of sequences: ragged batching of the hybrid-head KV cache.
//
// The pages name batched serving, and how the dual cache fits paged memory management,
// as open questions ("Critical Assessment": every efficiency measurement is at batch
// size 1).  Here sequences of different lengths share one caller-owned buffer:
//   * retrieval heads keep their K/V in pages of 128 tokens; page p of layer l is
//     [H_r(l)][128][d] and holds the same 128 positions of one sequence for all of the
//     layer's retrieval heads.  A sequence's logical page i is physical page
//     table[slot][i] on every layer (one block table per pool);
//   * streaming heads keep their sinks + ring per sequence slot, [slot][H_s][S+W][d]
//     ("Decoding Procedure": a constant-length cache per streaming head);
//   * the host keeps each sequence's length per layer and the free pages.
// duo_pool_decode_step appends one token to each listed sequence on each listed layer
// (one launch) and attends for all of them (one launch of the tcgen05 decode kernel
// over every (layer, sequence, KV head) item).
#include <algorithm>
#include <cmath>
#include <cstring>
#include <new>
#include <vector>

#include "decode_merge.cuh"
#include "tcgen05.cuh"
#include "nvtx_range.h"

struct duo_pool {
  int layers = 0, Hkv = 0, Hq = 0, G = 0, D = 0, S = 0, W = 0, max_seqs = 0, pages_per_seq = 0;
  int64_t num_pages = 0, max_len = 0;
  float scale = 0.f;
  char *buf = nullptr;
  size_t bytes = 0;
  bool initialised = false;
  int num_sms = 0;
  uint32_t *status = nullptr;
  uint32_t *counters = nullptr;  // one ticket per item of a call
  float *partials = nullptr;     // (max CTAs + items) segments of G partial rows
  int max_items = 0;
  duo::PoolLayerDesc *d_layers = nullptr;
  int *d_table = nullptr;
  std::vector<duo::PoolLayerDesc> h_layers;
  std::vector<int> hr, hs;
  std::vector<int> free_pages;                 // stack of free physical pages
  std::vector<uint8_t> open;                   // per slot
  std::vector<std::vector<int>> pages;         // per slot: physical page of each logical page
  std::vector<std::vector<int64_t>> len;       // per slot, per layer
};

namespace duo {

namespace {

constexpr int kMaxCtas = 1024;  // partial-row segments reserved for CTAs of one call

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct PoolLayout {
  size_t status, counters, partials, layers, table, total;
  std::vector<size_t> rk, rv, sk, sv;
  int max_items, pages_per_seq;
};

bool pool_layout(int layers, int Hkv, int Hq, const uint8_t *mask, int S, int W, int max_seqs, int64_t max_len,
                 int64_t num_pages, PoolLayout *L) {
  const int G = Hq / Hkv;
  const size_t page_row = 128 * 2;  // d = 128 bf16
  L->pages_per_seq = static_cast<int>((max_len + kPoolTile - 1) / kPoolTile);
  L->max_items = static_cast<int>(std::min<int64_t>(kPoolMaxSuper, static_cast<int64_t>(layers) * max_seqs)) * Hkv;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, 1024);
    return at;
  };
  L->status = take(256);
  L->counters = take(static_cast<size_t>(L->max_items) * 4);
  L->partials = take((static_cast<size_t>(kMaxCtas) + L->max_items) * G * kPartRow * 4);
  L->layers = take(static_cast<size_t>(layers) * sizeof(PoolLayerDesc));
  L->table = take(static_cast<size_t>(max_seqs) * L->pages_per_seq * 4);
  const double est = static_cast<double>(num_pages) * layers * Hkv * kPoolTile * page_row * 2 +
                     static_cast<double>(max_seqs) * layers * Hkv * (S + W) * page_row * 2;
  if (est > static_cast<double>(size_t(1) << 50)) return false;
  L->rk.resize(layers);
  L->rv.resize(layers);
  L->sk.resize(layers);
  L->sv.resize(layers);
  for (int l = 0; l < layers; ++l) {
    int hr = 0;
    for (int g = 0; g < Hkv; ++g) hr += mask[l * Hkv + g];
    const size_t rbytes = static_cast<size_t>(num_pages) * hr * kPoolTile * page_row;
    const size_t sbytes = static_cast<size_t>(max_seqs) * (Hkv - hr) * (S + W) * page_row;
    L->rk[l] = take(rbytes);
    L->rv[l] = take(rbytes);
    L->sk[l] = take(sbytes);
    L->sv[l] = take(sbytes);
  }
  L->total = off;
  return true;
}

duo_status pool_args(int layers, int kv_heads, int head_dim, const uint8_t *mask, int S, int W, int max_seqs,
                     int64_t max_len, int64_t num_pages, const duo_opts *opts, int *Hq, float *scale) {
  if (layers < 1 || layers > 65536 || kv_heads < 1 || kv_heads > kMaxKvHeads || !mask) return DUO_ERR_INVALID;
  if (S < 0 || W < 1 || S > (1 << 24) || W > (1 << 24)) return DUO_ERR_INVALID;
  if (max_seqs < 1 || max_seqs > (1 << 20) || max_len < 1 || max_len > (int64_t(1) << 31) - kPoolTile)
    return DUO_ERR_INVALID;
  if (num_pages < 1 || num_pages > (int64_t(1) << 30)) return DUO_ERR_INVALID;
  duo_opts o = {1, 0, DUO_BF16, DUO_KV_SAME, 0.f};
  if (opts) o = *opts;
  if (o.q_heads == 0) o.q_heads = kv_heads;
  if (o.q_heads < kv_heads || o.q_heads % kv_heads != 0 || o.q_heads > 4096) return DUO_ERR_INVALID;
  if (!(o.softmax_scale >= 0.f) || !std::isfinite(o.softmax_scale)) return DUO_ERR_INVALID;
  if (o.dtype != DUO_BF16 && o.dtype != DUO_FP32) return DUO_ERR_INVALID;
  if (o.retr_fmt != DUO_KV_SAME && o.retr_fmt != DUO_KV_INT4_G128 && o.retr_fmt != DUO_KV_FP8_E4M3)
    return DUO_ERR_INVALID;
  // the pool runs on the tcgen05 bf16 decode kernel: bf16, head_dim 128, groups up to 16
  if (o.dtype != DUO_BF16 || head_dim != 128 || o.retr_fmt != DUO_KV_SAME || o.q_heads / kv_heads > 16)
    return DUO_ERR_UNSUPPORTED;
  for (int i = 0; i < layers * kv_heads; ++i)
    if (mask[i] > 1) return DUO_ERR_INVALID;
  *Hq = o.q_heads;
  *scale = o.softmax_scale > 0.f ? o.softmax_scale : 1.f / std::sqrt(128.f);
  return DUO_OK;
}

// ---- kernels ----

__device__ __forceinline__ void copy_row256(char *dst, const char *src, int lane) {
  if (lane < 16) reinterpret_cast<uint4 *>(dst)[lane] = __ldg(reinterpret_cast<const uint4 *>(src) + lane);
}
__device__ __forceinline__ void zero_rows(char *dst, int rows, int lane) {  // rows of 256 bytes
  for (int c = lane; c < rows * 16; c += 32) reinterpret_cast<uint4 *>(dst)[c] = make_uint4(0, 0, 0, 0);
}

// One warp per (layer, sequence, KV head): the step's token into its page row or ring
// slot.  A page's row 0 opens the page on that layer: its other rows are cleared (a
// recycled page holds an old sequence's rows).
__global__ void __launch_bounds__(256) pool_append_kernel(const __grid_constant__ PoolAppendCall c) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int64_t w = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t total = static_cast<int64_t>(c.nlayers) * c.nseq * c.Hkv;
  if (w >= total) return;
  const int g = static_cast<int>(w % c.Hkv);
  const int s = static_cast<int>((w / c.Hkv) % c.nseq);
  const int li = static_cast<int>(w / (static_cast<int64_t>(c.Hkv) * c.nseq));
  const PoolLayerDesc &L = c.layers[c.layer0 + li];
  const int64_t src = ((static_cast<int64_t>(li) * c.nseq + s) * c.Hkv + g) * 256;
  const int pos = c.pos[s], slot = c.slot[s], idx = L.hm.kind_idx[g];
  if (L.hm.is_retr[g]) {
    const int row = pos % kPoolTile;
    const int64_t head0 = (static_cast<int64_t>(c.page[s]) * L.Hr + idx) * kPoolTile;
    copy_row256(L.rk + (head0 + row) * 256, c.k + src, lane);
    copy_row256(L.rv + (head0 + row) * 256, c.v + src, lane);
    if (row == 0) {
      zero_rows(L.rk + (head0 + 1) * 256, kPoolTile - 1, lane);
      zero_rows(L.rv + (head0 + 1) * 256, kPoolTile - 1, lane);
    }
  } else {
    const int64_t srow = pos < c.S ? pos : c.S + pos % c.W;
    const int64_t dst = ((static_cast<int64_t>(slot) * L.Hs + idx) * (c.S + c.W) + srow) * 256;
    copy_row256(L.sk + dst, c.k + src, lane);
    copy_row256(L.sv + dst, c.v + src, lane);
  }
  if (li == 0 && g == 0 && lane == 0 && c.new_page[s])
    c.table[static_cast<int64_t>(slot) * c.pages_per_seq + pos / kPoolTile] = c.page[s];
}

// n tokens of one sequence on one layer: warps over (token, KV head), then warps that
// clear the rest of the chunk's last page when the chunk opened it, and one thread that
// writes the block-table entries.
__global__ void __launch_bounds__(256) pool_chunk_append_kernel(const __grid_constant__ PoolChunkAppend c) {
  const int64_t w = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const PoolLayerDesc &L = *c.layer;
  const int64_t rows = static_cast<int64_t>(c.n) * c.Hkv;
  if (w < rows) {
    const int g = static_cast<int>(w % c.Hkv);
    const int t = static_cast<int>(w / c.Hkv);
    const int64_t pos = c.pos0 + t;
    const int64_t src = (static_cast<int64_t>(t) * c.Hkv + g) * 256;
    const int idx = L.hm.kind_idx[g];
    if (L.hm.is_retr[g]) {
      const int page = c.pages[pos / kPoolTile - c.first_page];
      const int64_t dst = ((static_cast<int64_t>(page) * L.Hr + idx) * kPoolTile + pos % kPoolTile) * 256;
      copy_row256(L.rk + dst, c.k + src, lane);
      copy_row256(L.rv + dst, c.v + src, lane);
    } else if (pos < c.S || pos >= c.ring_from) {  // the others are evicted within the call
      const int64_t srow = pos < c.S ? pos : c.S + pos % c.W;
      const int64_t dst = ((static_cast<int64_t>(c.slot) * L.Hs + idx) * (c.S + c.W) + srow) * 256;
      copy_row256(L.sk + dst, c.k + src, lane);
      copy_row256(L.sv + dst, c.v + src, lane);
    }
    return;
  }
  const int64_t wz = w - rows;
  const int64_t end = c.pos0 + c.n, last_start = (end - 1) / kPoolTile * kPoolTile;
  if (wz < L.Hr && last_start >= c.pos0 && end % kPoolTile != 0) {  // the chunk opened its last page
    const int page = c.pages[last_start / kPoolTile - c.first_page];
    const int64_t head0 = (static_cast<int64_t>(page) * L.Hr + wz) * kPoolTile;
    const int nrow = static_cast<int>(last_start + kPoolTile - end);
    zero_rows(L.rk + (head0 + end % kPoolTile) * 256, nrow, lane);
    zero_rows(L.rv + (head0 + end % kPoolTile) * 256, nrow, lane);
  }
  if (wz == 0 && lane == 0)
    for (int i = 0; i < c.npages; ++i) c.table[static_cast<int64_t>(c.slot) * c.pages_per_seq + c.first_page + i] = c.pages[i];
}

// Clears the sink and ring rows of one slot on every layer (a recycled slot holds an
// old sequence's rows): one block per (layer, K or V).
__global__ void __launch_bounds__(256) pool_clear_slot_kernel(const PoolLayerDesc *layers, int slot, int S, int W) {
  const PoolLayerDesc &L = layers[blockIdx.x >> 1];
  char *base = (blockIdx.x & 1) ? L.sv : L.sk;
  const int64_t n16 = static_cast<int64_t>(L.Hs) * (S + W) * 16;
  uint4 *dst = reinterpret_cast<uint4 *>(base + static_cast<int64_t>(slot) * L.Hs * (S + W) * 256);
  for (int64_t i = threadIdx.x; i < n16; i += blockDim.x) dst[i] = make_uint4(0, 0, 0, 0);
}

}  // namespace

cudaError_t launch_pool_append(const PoolAppendCall &c, cudaStream_t st) {
  const int64_t warps = static_cast<int64_t>(c.nlayers) * c.nseq * c.Hkv;
  pool_append_kernel<<<static_cast<unsigned>((warps + 7) / 8), 256, 0, st>>>(c);
  return cudaGetLastError();
}

cudaError_t launch_pool_chunk_append(const PoolChunkAppend &c, int Hr, int /*Hs*/, cudaStream_t st) {
  const int64_t warps = static_cast<int64_t>(c.n) * c.Hkv + std::max(Hr, 1);
  pool_chunk_append_kernel<<<static_cast<unsigned>((warps + 7) / 8), 256, 0, st>>>(c);
  return cudaGetLastError();
}

}  // namespace duo

using namespace duo;

namespace {

// First use: clear the buffer, describe every layer (tensor maps encoded on the host)
// and copy the descriptions to the device.
duo_status pool_init(duo_pool *P, cudaStream_t st) {
  if (P->initialised) return DUO_OK;
  if (dry_run()) {
    P->num_sms = 148;
    P->initialised = true;
    return DUO_OK;
  }
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DUO_ERR_CUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return DUO_ERR_CUDA;
  if (!tc::encode_fn()) return DUO_ERR_UNSUPPORTED;
  const uint64_t row = 256;
  for (int l = 0; l < P->layers; ++l) {
    PoolLayerDesc &L = P->h_layers[l];
    bool ok = true;
    {  // pages [num_pages * Hr][128][d]
      const uint64_t d[3] = {128, kPoolTile, static_cast<uint64_t>(P->num_pages) * std::max(L.Hr, 1)};
      const uint64_t s[2] = {row, row * kPoolTile};
      const uint32_t bx[3] = {64, kPoolTile, 1};
      ok &= tc::make_map(&L.tm_kr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L.Hr ? L.rk : P->buf, 3, d, s, bx,
                         CU_TENSOR_MAP_SWIZZLE_128B);
      ok &= tc::make_map(&L.tm_vr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L.Hr ? L.rv : P->buf, 3, d, s, bx,
                         CU_TENSOR_MAP_SWIZZLE_128B);
    }
    {  // streaming [max_seqs * Hs][S+W][d]
      const uint64_t slots = static_cast<uint64_t>(P->S) + P->W;
      const uint64_t d[3] = {128, slots, static_cast<uint64_t>(P->max_seqs) * std::max(L.Hs, 1)};
      const uint64_t s[2] = {row, row * slots};
      const uint32_t bx[3] = {64, kPoolTile, 1};
      ok &= tc::make_map(&L.tm_ks, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L.Hs ? L.sk : P->buf, 3, d, s, bx,
                         CU_TENSOR_MAP_SWIZZLE_128B);
      ok &= tc::make_map(&L.tm_vs, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L.Hs ? L.sv : P->buf, 3, d, s, bx,
                         CU_TENSOR_MAP_SWIZZLE_128B);
    }
    if (!ok) return DUO_ERR_CUDA;
  }
  if (cudaMemsetAsync(P->buf, 0, P->bytes, st) != cudaSuccess) return DUO_ERR_CUDA;
  if (cudaMemcpyAsync(P->d_layers, P->h_layers.data(), sizeof(PoolLayerDesc) * P->layers, cudaMemcpyHostToDevice,
                      st) != cudaSuccess)
    return DUO_ERR_CUDA;
  // the copy reads pageable host memory: finish it before the host vector can change
  if (cudaStreamSynchronize(st) != cudaSuccess) return DUO_ERR_CUDA;
  P->num_sms = sms;
  P->initialised = true;
  return DUO_OK;
}

bool seq_ok(const duo_pool *P, int seq) { return P && seq >= 0 && seq < P->max_seqs && P->open[seq]; }

}  // namespace

extern "C" {

size_t duo_pool_bytes(int layers, int kv_heads, int head_dim, const uint8_t *mask, int S, int W, int max_seqs,
                      int64_t max_len, int64_t num_pages, const duo_opts *opts) {
  int Hq = 0;
  float scale = 0.f;
  if (pool_args(layers, kv_heads, head_dim, mask, S, W, max_seqs, max_len, num_pages, opts, &Hq, &scale) != DUO_OK)
    return 0;
  PoolLayout L;
  if (!pool_layout(layers, kv_heads, Hq, mask, S, W, max_seqs, max_len, num_pages, &L)) return 0;
  return L.total;
}

duo_status duo_pool_create(int layers, int kv_heads, int head_dim, const uint8_t *mask, int S, int W, int max_seqs,
                           int64_t max_len, int64_t num_pages, const duo_opts *opts, void *dev_buf, size_t dev_bytes,
                           duo_pool **out) {
  DUO_NVTX_RANGE("duo_pool_create");
  if (!out) return DUO_ERR_INVALID;
  *out = nullptr;
  int Hq = 0;
  float scale = 0.f;
  duo_status st = pool_args(layers, kv_heads, head_dim, mask, S, W, max_seqs, max_len, num_pages, opts, &Hq, &scale);
  if (st != DUO_OK) return st;
  PoolLayout L;
  if (!pool_layout(layers, kv_heads, Hq, mask, S, W, max_seqs, max_len, num_pages, &L)) return DUO_ERR_INVALID;
  if (!dev_buf || (reinterpret_cast<uintptr_t>(dev_buf) & 255u) || dev_bytes < L.total) return DUO_ERR_INVALID;
  duo_pool *P = new (std::nothrow) duo_pool();
  if (!P) return DUO_ERR_INVALID;
  P->layers = layers;
  P->Hkv = kv_heads;
  P->Hq = Hq;
  P->G = Hq / kv_heads;
  P->D = head_dim;
  P->S = S;
  P->W = W;
  P->max_seqs = max_seqs;
  P->pages_per_seq = L.pages_per_seq;
  P->num_pages = num_pages;
  P->max_len = max_len;
  P->scale = scale;
  P->buf = static_cast<char *>(dev_buf);
  P->bytes = L.total;
  P->status = reinterpret_cast<uint32_t *>(P->buf + L.status);
  P->counters = reinterpret_cast<uint32_t *>(P->buf + L.counters);
  P->partials = reinterpret_cast<float *>(P->buf + L.partials);
  P->max_items = L.max_items;
  P->d_layers = reinterpret_cast<PoolLayerDesc *>(P->buf + L.layers);
  P->d_table = reinterpret_cast<int *>(P->buf + L.table);
  P->h_layers.assign(layers, PoolLayerDesc{});
  P->hr.assign(layers, 0);
  P->hs.assign(layers, 0);
  for (int l = 0; l < layers; ++l) {
    PoolLayerDesc &D = P->h_layers[l];
    int ri = 0, si = 0;
    for (int g = 0; g < kv_heads; ++g) {
      const bool r = mask[l * kv_heads + g] != 0;
      D.hm.is_retr[g] = r ? 1 : 0;
      D.hm.kind_idx[g] = static_cast<uint8_t>(r ? ri : si);
      if (r) D.hm.retr_head[ri++] = static_cast<uint8_t>(g);
      else D.hm.strm_head[si++] = static_cast<uint8_t>(g);
    }
    D.Hr = ri;
    D.Hs = si;
    P->hr[l] = ri;
    P->hs[l] = si;
    D.rk = P->buf + L.rk[l];
    D.rv = P->buf + L.rv[l];
    D.sk = P->buf + L.sk[l];
    D.sv = P->buf + L.sv[l];
  }
  P->free_pages.reserve(static_cast<size_t>(num_pages));
  for (int64_t pg = num_pages - 1; pg >= 0; --pg) P->free_pages.push_back(static_cast<int>(pg));
  P->open.assign(max_seqs, 0);
  P->pages.assign(max_seqs, {});
  P->len.assign(max_seqs, std::vector<int64_t>(layers, 0));
  *out = P;
  return DUO_OK;
}

void duo_pool_destroy(duo_pool *pool) { delete pool; }

duo_status duo_pool_open(duo_pool *P, void *stream, int *seq) {
  DUO_NVTX_RANGE("duo_pool_open");
  if (!P || !seq) return DUO_ERR_INVALID;
  int s = -1;
  for (int i = 0; i < P->max_seqs; ++i)
    if (!P->open[i]) {
      s = i;
      break;
    }
  if (s < 0) return DUO_ERR_CAPACITY;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  duo_status r = pool_init(P, st);
  if (r != DUO_OK) return r;
  bool any_strm = false;
  for (int l = 0; l < P->layers; ++l) any_strm |= P->hs[l] > 0;
  if (any_strm && launch_via_hook([&] {
        pool_clear_slot_kernel<<<static_cast<unsigned>(2 * P->layers), 256, 0, st>>>(P->d_layers, s, P->S, P->W);
        return cudaGetLastError();
      }) != cudaSuccess)
    return DUO_ERR_CUDA;
  P->open[s] = 1;
  P->pages[s].clear();
  std::fill(P->len[s].begin(), P->len[s].end(), 0);
  *seq = s;
  return DUO_OK;
}

duo_status duo_pool_close(duo_pool *P, int seq) {
  if (!seq_ok(P, seq)) return DUO_ERR_INVALID;
  for (int pg : P->pages[seq]) P->free_pages.push_back(pg);
  P->pages[seq].clear();
  P->open[seq] = 0;
  return DUO_OK;
}

duo_status duo_pool_len(const duo_pool *P, int seq, int layer, int64_t *len) {
  if (!seq_ok(P, seq) || layer < 0 || layer >= P->layers || !len) return DUO_ERR_INVALID;
  *len = P->len[seq][layer];
  return DUO_OK;
}

duo_status duo_pool_free_pages(const duo_pool *P, int64_t *pages) {
  if (!P || !pages) return DUO_ERR_INVALID;
  *pages = static_cast<int64_t>(P->free_pages.size());
  return DUO_OK;
}

duo_status duo_pool_page(const duo_pool *P, int seq, int logical_page, int *physical_page) {
  if (!seq_ok(P, seq) || !physical_page || logical_page < 0 ||
      logical_page >= static_cast<int>(P->pages[seq].size()))
    return DUO_ERR_INVALID;
  *physical_page = P->pages[seq][logical_page];
  return DUO_OK;
}

duo_status duo_pool_region(const duo_pool *P, int layer, duo_region which, void **ptr, uint64_t *bytes) {
  if (!P || layer < 0 || layer >= P->layers) return DUO_ERR_INVALID;
  const PoolLayerDesc &L = P->h_layers[layer];
  const uint64_t rbytes = static_cast<uint64_t>(P->num_pages) * L.Hr * kPoolTile * 256;
  const uint64_t sbytes = static_cast<uint64_t>(P->max_seqs) * L.Hs * (P->S + P->W) * 256;
  char *p = nullptr;
  uint64_t n = 0;
  switch (which) {
    case DUO_REGION_RETR_K: p = L.rk; n = rbytes; break;
    case DUO_REGION_RETR_V: p = L.rv; n = rbytes; break;
    case DUO_REGION_STRM_K: p = L.sk; n = sbytes; break;
    case DUO_REGION_STRM_V: p = L.sv; n = sbytes; break;
    default: return DUO_ERR_INVALID;
  }
  if (ptr) *ptr = p;
  if (bytes) *bytes = n;
  return DUO_OK;
}

duo_status duo_pool_append_kv(duo_pool *P, int layer, int seq, const void *k, const void *v, int n, void *stream) {
  DUO_NVTX_RANGE("duo_pool_append_kv");
  if (!seq_ok(P, seq) || layer < 0 || layer >= P->layers || !k || !v || n < 1) return DUO_ERR_INVALID;
  if ((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v)) & 15u) return DUO_ERR_INVALID;
  const int64_t len = P->len[seq][layer];
  if (len + n > P->max_len) return DUO_ERR_CAPACITY;
  const int64_t need = (len + n + kPoolTile - 1) / kPoolTile;  // pages the sequence must hold
  const int64_t have = static_cast<int64_t>(P->pages[seq].size());
  if (need - have > static_cast<int64_t>(P->free_pages.size())) return DUO_ERR_CAPACITY;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  duo_status r = pool_init(P, st);
  if (r != DUO_OK) return r;
  // pages opened by this call come off the free stack; they go back if a launch fails
  std::vector<int> &pg = P->pages[seq];
  for (int64_t i = have; i < need; ++i) {
    pg.push_back(P->free_pages.back());
    P->free_pages.pop_back();
  }
  auto undo = [&] {
    while (static_cast<int64_t>(pg.size()) > have) {
      P->free_pages.push_back(pg.back());
      pg.pop_back();
    }
  };
  const char *kc = static_cast<const char *>(k), *vc = static_cast<const char *>(v);
  const int64_t row_bytes = static_cast<int64_t>(P->Hkv) * 256;
  constexpr int kChunk = 32512;  // tokens per launch: their pages fit the parameter block
  for (int t0 = 0; t0 < n; t0 += kChunk) {
    PoolChunkAppend c{};
    c.layer = P->d_layers + layer;
    c.table = P->d_table;
    c.pages_per_seq = P->pages_per_seq;
    c.slot = seq;
    c.Hkv = P->Hkv;
    c.D = 128;
    c.S = P->S;
    c.W = P->W;
    c.n = std::min(kChunk, n - t0);
    c.pos0 = len + t0;
    c.ring_from = std::max<int64_t>(P->S, len + n - P->W);
    c.k = kc + t0 * row_bytes;
    c.v = vc + t0 * row_bytes;
    c.first_page = static_cast<int>(c.pos0 / kPoolTile);
    const int last_page = static_cast<int>((c.pos0 + c.n - 1) / kPoolTile);
    c.npages = last_page - c.first_page + 1;
    for (int i = 0; i < c.npages; ++i) c.pages[i] = pg[c.first_page + i];
    if (launch_via_hook([&] { return launch_pool_chunk_append(c, P->hr[layer], P->hs[layer], st); }) != cudaSuccess) {
      if (t0 == 0) {
        undo();
        return DUO_ERR_CUDA;
      }
      // earlier pieces are in the cache: the length follows them (the contract: len
      // describes what the cache holds)
      P->len[seq][layer] = len + t0;
      while (static_cast<int64_t>(pg.size()) > (len + t0 + kPoolTile - 1) / kPoolTile) {
        P->free_pages.push_back(pg.back());
        pg.pop_back();
      }
      return DUO_ERR_CUDA;
    }
  }
  P->len[seq][layer] = len + n;
  return DUO_OK;
}

duo_status duo_pool_decode_step(duo_pool *P, int layer0, int nlayers, int nseq, const int *seqs, const void *q,
                                const void *k, const void *v, void *out, float *lse, void *stream) {
  DUO_NVTX_RANGE("duo_pool_decode_step");
  if (!P || nlayers < 1 || layer0 < 0 || layer0 + nlayers > P->layers || nseq < 1 || nseq > kPoolMaxSeqs ||
      nlayers * nseq > kPoolMaxSuper || !seqs || !q || !k || !v || !out)
    return DUO_ERR_INVALID;
  if (((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v) |
        reinterpret_cast<uintptr_t>(out)) & 15u) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return DUO_ERR_INVALID;
  if (nlayers * nseq * P->Hkv > P->max_items) return DUO_ERR_CAPACITY;
  std::vector<uint8_t> seen(P->max_seqs, 0);
  int new_pages = 0;
  for (int i = 0; i < nseq; ++i) {
    const int s = seqs[i];
    if (!seq_ok(P, s) || seen[s]) return DUO_ERR_INVALID;
    seen[s] = 1;
    const int64_t len = P->len[s][layer0];
    for (int l = layer0; l < layer0 + nlayers; ++l)
      if (P->len[s][l] != len) return DUO_ERR_INVALID;  // one position per sequence in a step
    if (len + 1 > P->max_len) return DUO_ERR_CAPACITY;
    if (len / kPoolTile >= static_cast<int64_t>(P->pages[s].size())) ++new_pages;
  }
  if (new_pages > static_cast<int>(P->free_pages.size())) return DUO_ERR_CAPACITY;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  duo_status r = pool_init(P, st);
  if (r != DUO_OK) return r;

  PoolAppendCall ac{};
  ac.layers = P->d_layers;
  ac.table = P->d_table;
  ac.pages_per_seq = P->pages_per_seq;
  ac.layer0 = layer0;
  ac.nlayers = nlayers;
  ac.nseq = nseq;
  ac.Hkv = P->Hkv;
  ac.D = 128;
  ac.S = P->S;
  ac.W = P->W;
  ac.k = static_cast<const char *>(k);
  ac.v = static_cast<const char *>(v);
  PoolDecodeCall dc{};
  dc.layers = P->d_layers;
  dc.table = P->d_table;
  dc.pages_per_seq = P->pages_per_seq;
  dc.layer0 = layer0;
  dc.nlayers = nlayers;
  dc.nseq = nseq;
  std::vector<int> opened;
  for (int i = 0; i < nseq; ++i) {
    const int s = seqs[i];
    const int64_t len = P->len[s][layer0];
    const int lp = static_cast<int>(len / kPoolTile);
    int fresh = 0;
    if (lp >= static_cast<int>(P->pages[s].size())) {
      P->pages[s].push_back(P->free_pages.back());
      P->free_pages.pop_back();
      opened.push_back(s);
      fresh = 1;
    }
    ac.slot[i] = s;
    ac.pos[i] = static_cast<int>(len);
    ac.page[i] = P->pages[s][lp];
    ac.new_page[i] = fresh;
    dc.slot[i] = s;
    dc.len[i] = static_cast<int>(len + 1);
  }
  DecodeParams p{};
  p.q = static_cast<const char *>(q);
  p.out = static_cast<char *>(out);
  p.lse = lse;
  p.partials = P->partials;
  p.counters = P->counters;
  p.status = P->status;
  p.B = nlayers * nseq;
  p.Hq = P->Hq;
  p.Hkv = P->Hkv;
  p.G = P->G;
  p.D = 128;
  p.S = P->S;
  p.W = P->W;
  p.scale_log2 = P->scale * 1.4426950408889634f;
  if (launch_via_hook([&] { return launch_pool_append(ac, st); }) != cudaSuccess) {
    for (auto it = opened.rbegin(); it != opened.rend(); ++it) {  // nothing was written
      P->free_pages.push_back(P->pages[*it].back());
      P->pages[*it].pop_back();
    }
    return DUO_ERR_CUDA;
  }
  // the token is in the cache: lengths follow what the cache holds even if the
  // attention launch fails
  for (int i = 0; i < nseq; ++i)
    for (int l = layer0; l < layer0 + nlayers; ++l) P->len[seqs[i]][l] += 1;
  if (launch_via_hook([&] { return launch_decode_pool_tc(p, dc, P->hr.data(), P->hs.data(), P->num_sms, st); }) !=
      cudaSuccess)
    return DUO_ERR_CUDA;
  return DUO_OK;
}

duo_status duo_pool_device_status(duo_pool *P, void *stream) {
  DUO_NVTX_RANGE("duo_pool_device_status");
  if (!P) return DUO_ERR_INVALID;
  if (!P->initialised || dry_run()) return DUO_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return DUO_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpy(&word, P->status, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return DUO_ERR_CUDA;
  if (word == 0) return DUO_OK;
  if (cudaMemset(P->status, 0, 4) != cudaSuccess) return DUO_ERR_CUDA;
  return (word & kDevTimeout) ? DUO_ERR_TIMEOUT : DUO_ERR_CUDA;
}

}  // extern "C"
