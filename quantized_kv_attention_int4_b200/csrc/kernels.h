// Internal launcher declarations shared by the CUDA translation units.
#pragma once

#include <atomic>
#include <mutex>

#include "common.cuh"

namespace fl {

struct EncodeBaseArgs {
  CacheView c;
  int layer, row0, n_rows;
  const uint16_t* k;
  const uint16_t* v;
  int64_t head_stride;
};

struct EncodeResArgs {
  CacheView c;
  int layer, r, row0, n_span, slot0, n_rows, compact;
  const int32_t* rows;
  const uint16_t* k;
  const uint16_t* v;
  int64_t head_stride;
};

// Layers one persistent sparse launch can flush (beyond: one launch per layer).
constexpr int kFlushLayersMax = 256;

struct ReaderArgs {
  CacheView c;
  int layer, r, n_q, n_tail, k_sel, n_splits, keep;
  const uint16_t* q;
  const uint16_t* k_new;
  const uint16_t* v_new;
  const float* o_prev;
  float* o;
  float* part;
  int32_t* counter;
  // fused tail flush (flush != 0): after attending, write store r of the 64 tail rows
  // [n_q, n_q + 64); a residual store takes the rows set in flush_act into the 64-slot
  // group that starts at residual slot flush_slot0
  int flush, flush_slot0;
  unsigned long long flush_act;
  // a launch over layers [layer, layer + n_layers) (the persistent sparse reader): q, k_new,
  // v_new, o_prev and o of layer layer + i start io_layer_stride elements * i further
  int n_layers;
  int64_t io_layer_stride;
  // the fused flush of a launch over several layers: flush_slot0 of layer layer + i
  int32_t flush_slot0s[kFlushLayersMax];
};

struct SelectArgs {
  CacheView c;
  int layer0, r, n_q, n_tail, k_sel;
};

struct TokenArgs {
  const uint16_t* h_prev;   // BF16 [n_tokens][row_stride]: state entering the ranked loop
  const uint16_t* h_cur;    // BF16 [n_tokens][row_stride]: state leaving it
  int64_t row_stride;
  int32_t d_model, n_tokens;
  const int32_t* rows;      // candidates, ascending
  int64_t n_rows;
  int32_t k;
  int32_t* rows_out;        // [k]
  double* keys;             // [n_rows]
  int32_t* status;          // optional device int32[3]
};

struct PrefillArgs {
  const uint16_t* q;        // BF16 [heads][n_act][128]: the active tokens' queries
  const int32_t* pos;       // [n_act] their token positions, ascending
  int32_t n_act, n_tokens, heads;
  const uint16_t* k;        // BF16 [heads][n_tokens][128]
  const uint16_t* v;
  int64_t q_head_stride, kv_head_stride, o_head_stride;
  float* o;                 // fp32 [heads][n_act][128]
  int32_t* status;          // optional device int32[3]
};

cudaError_t launch_encode_base(const EncodeBaseArgs& a, cudaStream_t s);
cudaError_t launch_encode_residual(const EncodeResArgs& a, cudaStream_t s);
// chain = false: an ordinary stream-ordered launch (no programmatic overlap with the
// preceding kernel)
cudaError_t launch_dense(ReaderArgs a, cudaStream_t s, bool chain = true);
cudaError_t launch_dense_direct(ReaderArgs a, cudaStream_t s);
// a.n_splits is set by the launcher (sparse_launch_splits); it must fit the partials buffer
cudaError_t launch_sparse(ReaderArgs a, cudaStream_t s, bool chain = true);
cudaError_t launch_sparse_direct(ReaderArgs a, cudaStream_t s, bool chain = true);
cudaError_t launch_select(const SelectArgs& a, int n_layers, cudaStream_t s);
cudaError_t launch_token_select(const TokenArgs& a, cudaStream_t s);
cudaError_t launch_prefill_attn(const PrefillArgs& a, cudaStream_t s);

int dense_splits(int heads, int n_q);

// Number of devices the per-device caches below cover.
constexpr int kMaxDevices = 64;

// SM count of the current device, looked up once per device (safe when several host
// threads make their first call at the same time); 0 when it cannot be read.
int device_sms();

// Runs fn(dev) once per device (device = the current one), under a lock, so host threads
// that make their first call at the same time neither race nor repeat it; a failed set-up
// is retried by the next call.
template <class F>
cudaError_t once_per_device(std::atomic<bool>* done, std::mutex& mu, F&& fn) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  std::lock_guard<std::mutex> lock(mu);
  if (done[dev].load(std::memory_order_relaxed)) return cudaSuccess;
  const cudaError_t e = fn(dev);
  if (e == cudaSuccess) done[dev].store(true, std::memory_order_release);
  return e;
}

// Plan entries (selected columns) one sparse-reader CTA holds in shared memory.
int sparse_cta_columns(int loops);
// Split-K partitions per (layer, head) that launch_sparse uses for a loop-r reader over
// k_sel columns of a cache with codec `codec` on a device with `sms` SMs, with or without
// the fused tail flush: never fewer than the plan copy of one CTA (or work item) needs.
int sparse_launch_splits(int heads, int loops, int codec, int r, int k_sel, int sms, bool flush);
// Split-K partials per head that a workspace for these dims holds for the one-layer
// launches: enough for every dense launch and every sparse launch with k_sel <= max_select.
int workspace_splits(int loops, int max_select);
// The direct sparse reader's split count and per-CTA plan capacity (sparse.cu).
int direct_splits(int heads, int k_sel, int loops, int sms);
int direct_cta_columns(int loops);
// The persistent sparse reader (sparse_persist.cu): the method's 4-bit residual stores,
// loops r <= kPersistMaxLoop, with or without the fused flush; one launch for a range of
// layers (work items of at most persist_item_columns(loops) selected columns of one
// (layer, head)), then one launch of its combine.
constexpr int kPersistMaxLoop = 8;
int persist_item_columns(int loops);
int persist_splits(int k_sel, int loops);
cudaError_t launch_sparse_persist(ReaderArgs a, cudaStream_t s, bool chain);

}  // namespace fl
