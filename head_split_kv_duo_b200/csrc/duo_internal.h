// duo_internal.h -- host/device shared structures of the hybrid-head KV cache.
// Not part of the public ABI (include/duo.h is).
#pragma once

#include <atomic>
#include <cstddef>
#include <cstdint>
#include <vector>

#include <cuda.h>
#include <cuda_runtime.h>

#include "duo.h"

namespace duo {

constexpr int kMaxKvHeads = 128;
constexpr int kAlign = 1024;          // every carved region starts on a 1 KiB boundary
constexpr int kMinSplitTokens = 256;  // shortest split of a retrieval head in decode
constexpr int kMaxSplits = 512;       // most splits of one retrieval head in decode

// Device status word bits (latched, cleared by duo_get_device_status).
constexpr uint32_t kDevTimeout = 1u;

// Head partition of one layer, passed to kernels by value.
struct HeadMap {
  uint8_t is_retr[kMaxKvHeads];   // kv head -> 1 retrieval / 0 streaming
  uint8_t kind_idx[kMaxKvHeads];  // kv head -> index among heads of its kind
  uint8_t retr_head[kMaxKvHeads]; // retrieval index -> kv head
  uint8_t strm_head[kMaxKvHeads]; // streaming index -> kv head
};

struct Layer {
  int Hr = 0, Hs = 0;
  HeadMap hm{};
  // retrieval K/V: [B][Hr][max_len][row] (row = d elements, or d/2 INT4 bytes)
  char *rk = nullptr, *rv = nullptr;
  // INT4 scale/zero: [B][Hr][max_len][2] fp16
  char *rk_sz = nullptr, *rv_sz = nullptr;
  // streaming K/V: [B][Hs][S+W][d]
  char *sk = nullptr, *sv = nullptr;
  int64_t len = 0;
};

}  // namespace duo

struct duo_cache {
  int layers = 0, Hkv = 0, Hq = 0, G = 0, D = 0, B = 0, S = 0, W = 0;
  int64_t max_len = 0;  // capacity in tokens
  int64_t cap = 0;      // row stride of retrieval arrays: max_len rounded up to 256
  duo_dtype dtype = DUO_BF16;
  duo_kv_fmt fmt = DUO_KV_SAME;
  float scale = 0.f;
  int esize = 2;
  char *buf = nullptr;
  size_t bytes = 0;
  bool initialised = false;
  int num_sms = 0;
  // scratch
  uint32_t *status = nullptr;    // device status word
  uint32_t *counters = nullptr;  // [B][Hq] split-merge tickets
  float *partials = nullptr;     // [B][Hkv][max_splits][G][d+4]
  int max_splits = 1;
  char *hist_k = nullptr, *hist_v = nullptr;  // [B][HsMax][S+W][d] pre-fill staging
  int hs_max = 0;
  std::vector<duo::Layer> L;
};

namespace duo {

// ---- kernel parameter blocks ----

struct AppendParams {
  const char *k, *v;  // [B][n][Hkv][d]
  char *rk, *rv, *rk_sz, *rv_sz, *sk, *sv;
  int B, n, Hkv, D, Hr, Hs, S, W;
  int64_t len, max_len;  // max_len: row stride of retrieval arrays (capacity rounded up to 256)
  int64_t ring_from;  // first non-sink position that reaches the ring
  int int4;           // retrieval rows stored INT4
  int fp8;            // retrieval rows stored FP8 (E4M3 + fp32 scale)
  HeadMap hm;
};

struct HistParams {
  const char *sk, *sv;  // streaming cache of the layer
  char *hk, *hv;        // staging [B][HsMax][S+W][d]
  int B, Hs, HsMax, D, S, W;
  int hs, hw;           // sink rows, window rows staged
  int64_t wstart;       // position of the first window row
};

struct DecodeParams {
  const char *q;
  char *out;
  float *lse;
  const char *rk, *rv, *rk_sz, *rv_sz, *sk, *sv;
  float *partials;
  uint32_t *counters, *status;
  int B, Hq, Hkv, G, D, Hr, Hs, S, W;
  int64_t len, max_len;  // max_len: row stride of retrieval arrays
  int nsplit;
  int64_t split_len;
  int qg, nqg;        // query heads per CTA, CTAs per KV head
  int max_splits;
  int n_retr_ctas;
  float scale_log2;   // softmax scale * log2(e)
  HeadMap hm;
  // fused append: the new token's rows [B][Hkv][d] (nullptr: already in the cache), at
  // position npos = len - 1; the CTA that reads a row's tile writes it first
  const char *nk, *nv;
  int64_t npos;
  // Programmatic dependent launch of a quantised layer's two decodes (the bf16 streaming
  // heads and the quantised retrieval heads, disjoint heads, partial rows and tickets):
  //   0  alone: dependents are released at once; global memory is touched only after the
  //      previous grid on the stream has completed
  //   1  leading (the streaming heads, on a few CTAs): dependents are released only once
  //      the previous grid has completed, so that the next grid may start at once
  //   2  beside the leader (the retrieval heads, on the other SMs): no wait at the start
  //      (the leader's release implies the grid before it has completed); the grid waits
  //      for the leader before it ends, so that whatever follows it sees both complete
  int pdl_mode;
  // test control (duo_debug_device_stall): the bf16 decode's softmax first waits for a
  // barrier that nothing arrives at, so that its bounded wait runs out
  int debug_stall;
};

struct PrefillParams {
  const char *q, *k, *v;  // q [B][n][Hq][d]; k, v [B][n][Hkv][d] (the chunk)
  char *out;
  float *lse;
  const char *rk, *rv;    // retrieval cache: positions 0 .. len-1 (the chunk itself is read from k, v)
  const char *hk, *hv;    // streaming history staging
  uint32_t *status;
  int B, n, Hq, Hkv, G, D, Hr, Hs, HsMax, S, W;
  int64_t len, max_len;  // max_len: row stride of retrieval arrays
  int hs, hw;
  int64_t wstart;
  float scale_log2;
  HeadMap hm;
  // gated mixing (identification-phase forward): when set, every output row becomes
  // mix_alpha[g] * (the row already in out) + (1 - mix_alpha[g]) * (this attention)
  const float *mix_alpha;
};

// Raises the dynamic shared-memory limit of `kernel` to `bytes` on the current device.
// The attribute belongs to the device, so `done` keeps one bit per device (devices 0-63)
// that already has it; a device past 63 sets it at every call (harmless, only slower).
template <typename Kernel>
cudaError_t opt_in_smem(Kernel kernel, int bytes, std::atomic<uint64_t> &done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

// ---- launchers (return cudaSuccess or the launch error) ----
cudaError_t launch_append(const AppendParams &p, duo_dtype dt, cudaStream_t st);
cudaError_t launch_hist(const HistParams &p, duo_dtype dt, cudaStream_t st);
cudaError_t launch_decode(const DecodeParams &p, duo_dtype dt, bool int4, cudaStream_t st);
cudaError_t launch_prefill_simt(const PrefillParams &p, duo_dtype dt, cudaStream_t st);
// tcgen05 pre-fill (bf16, d = 128).  prepare_prefill_tc does every host step that can
// fail (tensor maps, the shared-memory limit), so that a call can finish its set-up
// before its first launch; launch_prefill_tc then only launches.
struct PrefillTcLaunch {
  PrefillParams p;
  CUtensorMap tm_q, tm_kc, tm_vc, tm_kh, tm_vh, tm_kn, tm_vn;
};
bool prefill_tc_supported(const PrefillParams &p, duo_dtype dt);
cudaError_t prepare_prefill_tc(const PrefillParams &p, PrefillTcLaunch *l);
cudaError_t launch_prefill_tc(const PrefillTcLaunch &l, cudaStream_t st);

// Test controls of the host bookkeeping (duo_debug_launch_controls): true when the launch
// about to be made must be skipped, with *e the result to report for it.
bool launch_intercepted(cudaError_t *e);
bool dry_run();
// Runs one launch (a callable returning its cudaError_t) unless the test controls
// intercept it.
template <typename F>
cudaError_t launch_via_hook(F &&launch) {
  cudaError_t e;
  if (launch_intercepted(&e)) return e;
  return launch();
}

// tcgen05 decode (bf16, d = 128, up to 16 query heads per KV head), one CTA per SM.
// overlap_previous: launch as a programmatic dependent of the previous kernel on the
// stream; the kernel waits for it (griddepcontrol.wait) before its first global read.
bool decode_tc_supported(const DecodeParams &p, duo_dtype dt, bool int4);
cudaError_t launch_decode_tc(const DecodeParams &p, int num_sms, bool overlap_previous, cudaStream_t st);
// tcgen05 decode over an INT4 retrieval cache (bf16, head_dim 128, G <= 16)
bool decode_int4_tc_supported(const DecodeParams &p, duo_dtype dt);
cudaError_t launch_decode_int4_tc(const DecodeParams &p, int num_sms, bool overlap_previous, cudaStream_t st);

// tcgen05 decode over an FP8 (E4M3) retrieval cache (bf16, head_dim 128, G <= 16)
bool decode_fp8_tc_supported(const DecodeParams &p, duo_dtype dt);
cudaError_t launch_decode_fp8_tc(const DecodeParams &p, int num_sms, bool overlap_previous, cudaStream_t st);

// ---- paged pool of sequences (ragged batching) ----
constexpr int kPoolTile = 128;       // tokens per retrieval page (= one decode tile)
constexpr int kPoolMaxSeqs = 128;    // sequences in one pool decode call
constexpr int kPoolMaxSuper = 1024;  // (layer, sequence) pairs in one pool decode call

// One layer of a pool as the kernels see it, kept in device memory (written once):
// the tensor maps of its retrieval pages [pages][Hr][128][d] and of its streaming
// arrays [max_seqs][Hs][S+W][d], its head partition and its array bases.
struct alignas(64) PoolLayerDesc {
  CUtensorMap tm_kr, tm_vr, tm_ks, tm_vs;
  HeadMap hm;
  int Hr, Hs;
  char *rk, *rv, *sk, *sv;
};

// A pool decode call: layers layer0 .. layer0+nlayers-1 of the listed sequences.
struct PoolDecodeCall {
  const PoolLayerDesc *layers;  // device, every layer of the pool
  const int *table;             // device block table [max_seqs][pages_per_seq]
  int pages_per_seq;
  int layer0, nlayers, nseq;
  int slot[kPoolMaxSeqs];       // sequence slots
  int len[kPoolMaxSeqs];        // tokens per sequence, the step's token included
};

// tcgen05 decode over a pool (bf16, d 128, G <= 16): every (layer, sequence, KV head)
// of the call in one launch; p supplies q / out / lse ([nlayers][nseq][Hq][...]), the
// scratch (partials for num_sms + items segments, one ticket per item), status, the
// shape (Hq, Hkv, G, D, S, W) and the logit scale.
cudaError_t launch_decode_pool_tc(const DecodeParams &p, const PoolDecodeCall &c, const int *layer_hr,
                                  const int *layer_hs, int num_sms, cudaStream_t st);

// Append of one token per listed sequence on every layer of a pool call (rows of the
// retrieval pages and the sink / ring slots), also writing the block-table entries of
// pages the step opens.  k, v [nlayers][nseq][Hkv][d].
struct PoolAppendCall {
  const PoolLayerDesc *layers;
  int *table;
  int pages_per_seq;
  int layer0, nlayers, nseq, Hkv, D, S, W;
  const char *k, *v;
  int slot[kPoolMaxSeqs];
  int pos[kPoolMaxSeqs];        // position of the token (tokens before it)
  int page[kPoolMaxSeqs];       // physical page holding it
  int new_page[kPoolMaxSeqs];   // 1: the step opens that page (write the table entry)
};
cudaError_t launch_pool_append(const PoolAppendCall &c, cudaStream_t st);
// Append of n tokens of one sequence on one layer; pages[i] is the physical page of
// logical page first_page + i (entries written to the table too).
struct PoolChunkAppend {
  const PoolLayerDesc *layer;
  int *table;
  int pages_per_seq, slot, Hkv, D, S, W, n, first_page, npages;
  int64_t pos0, ring_from;
  const char *k, *v;            // [n][Hkv][d]
  int pages[256];
};
cudaError_t launch_pool_chunk_append(const PoolChunkAppend &c, int Hr, int Hs, cudaStream_t st);

// decode tiling shared by host (split sizing) and device
int decode_tokens_per_stage(duo_dtype dt, int D, bool int4);

}  // namespace duo
