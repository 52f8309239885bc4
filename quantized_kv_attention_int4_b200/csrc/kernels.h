// Internal launcher declarations shared by the CUDA translation units.
#pragma once

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
cudaError_t launch_sparse(ReaderArgs a, cudaStream_t s);
cudaError_t launch_sparse_direct(ReaderArgs a, cudaStream_t s);
cudaError_t launch_select(const SelectArgs& a, int n_layers, cudaStream_t s);
cudaError_t launch_token_select(const TokenArgs& a, cudaStream_t s);
cudaError_t launch_prefill_attn(const PrefillArgs& a, cudaStream_t s);

int dense_splits(int heads, int n_q);
int sparse_splits(int heads, int k_sel, int loops);

}  // namespace fl
