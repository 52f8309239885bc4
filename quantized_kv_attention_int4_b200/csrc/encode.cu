// Base (loop 1) and residual (loop r >= 2) encoders.
//
// FlashLoop project page, "The Method", Step 03: loop-1 K/V are quantised as the
// base; each later loop stores only its residual against the reconstructed state of
// the preceding loop.  flozi guide "FlashLoop: store changes between repeated
// passes", section 3: group-wise asymmetric 4-bit, group 64, keys per channel,
// values per token, residuals for active tokens only.  Section 4 of the same guide
// (the "Per-loop KIVI4" row, and the 2-bit row of Figure 5) gives the two codec
// variants of the loop r >= 2 stores: the full state X^(r) in 4 bits, or the residual
// in 2 bits.
//
// Every arithmetic step of the quantiser is one IEEE fp32 operation with explicit
// round-to-nearest intrinsics so that codes, scales and zero points are exact
// functions of the inputs (the contract in include/flashloop.h).
#include "kernels.h"
#include "quant.cuh"

namespace fl {
namespace {

// 64 rows x 128 BF16 (row i at src + i*128) into xs as fp32.
__device__ __forceinline__ void load_rows(const uint16_t* src, float (*xs)[129], int tid) {
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    int i = tid + 256 * it;
    int row = i >> 4, c8 = (i & 15) * 8;
    bf16x8(ldg_u4(src + (size_t)row * kD + c8), &xs[row][c8]);
  }
}

__global__ void __launch_bounds__(256) encode_base_kernel(EncodeBaseArgs a) {
  const int blk = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
  const CacheView& c = a.c;
  const int cap = c.cap, ncb = cap / kG;
  const int tok0 = a.row0 + blk * kG, gb = tok0 / kG;
  __shared__ EncodeSmem sm;

  uint8_t* rec = arr<uint8_t>(c, A_BREC, a.layer) + ((size_t)h * ncb + gb) * kRec;
  const size_t in_off = (size_t)h * a.head_stride + (size_t)blk * kG * kD;
  for (int part = 0; part < 2; ++part) {
    const bool is_v = part == 1;
    load_rows((is_v ? a.v : a.k) + in_off, sm.xs, tid);
    __syncthreads();
    if (is_v) value_params(sm, rec, 0, kG, kG, tid, 256);
    else key_params(sm, rec, 0, kD, kG, tid, 256);
    __syncthreads();
    group_codes(sm, rec, is_v, 0, kG, 0, kD / 8, kG, tid, 256);
    __syncthreads();
  }

  if (h == 0) {
    uint8_t* depth = arr<uint8_t>(c, A_DEPTH, a.layer);
    if (tid < kG) depth[tok0 + tid] = 1;
    unsigned long long* mask = arr<unsigned long long>(c, A_MASK, a.layer);
    int32_t* first = arr<int32_t>(c, A_FIRST, a.layer);
    for (int r = 2 + tid; r <= c.R; r += 256) {
      mask[(size_t)r * ncb + gb] = 0ull;
      first[(size_t)r * ncb + gb] = -1;
    }
  }
}

template <int kCodec>
__global__ void __launch_bounds__(256) encode_residual_kernel(EncodeResArgs a) {
  using CT = CodecT<kCodec>;
  constexpr int kRB = CT::kResBits;
  const int g = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
  const CacheView& c = a.c;
  const int cap = c.cap, ncb = cap / kG, T = c.total_slots, r = a.r;
  const int i0 = g * kG;
  const int nr = min(kG, a.n_rows - i0);
  __shared__ EncodeSmem sm;
  int* tok = sm.row;
  float(*xs)[129] = sm.xs;

  const unsigned long long* mask = arr<unsigned long long>(c, A_MASK, a.layer);
  const int32_t* first = arr<int32_t>(c, A_FIRST, a.layer);
  uint8_t* depth = arr<uint8_t>(c, A_DEPTH, a.layer);

  if (tid < kG) {
    int j = -1;
    if (tid < nr) {
      const int i = i0 + tid;
      j = a.rows[i];
      int err = 0;
      if (j < a.row0 || j >= a.row0 + a.n_span) err = FL_DEV_ROWS_RANGE;
      else if (i > 0 && a.rows[i - 1] >= j) err = FL_DEV_ROWS_ORDER;
      else if (r >= 3 && !((mask[(size_t)(r - 1) * ncb + (j >> 6)] >> (j & 63)) & 1ull)) err = FL_DEV_NOT_NESTED;
      else if (r == 2 && depth[j] < 1) err = FL_DEV_NOT_NESTED;
      if (err) {
        if (h == 0) record_error(c.status, err, j);
        j = -1;
      }
    }
    tok[tid] = j;
  }
  __syncthreads();

  const int gslot0 = c.slot_base[r] + a.slot0 + i0;  // a multiple of 64
  const uint8_t* brec = arr<uint8_t>(c, A_BREC, a.layer) + (size_t)h * ncb * kRec;
  uint8_t* rrec = arr<uint8_t>(c, A_RREC, a.layer) + (size_t)h * (T / kG) * Rec<kRB>::kBytes;
  uint8_t* orec = rrec + (size_t)(gslot0 >> 6) * Rec<kRB>::kBytes;  // this CTA's output group record

  for (int part = 0; part < 2; ++part) {
    const bool is_v = part == 1;
    const uint16_t* src = is_v ? a.v : a.k;

    // residual E = X^(r) - X_hat^(r-1) (the full-state codec: X^(r) itself), 8 channels per item
    for (int item = tid; item < kG * 16; item += 256) {
      const int tt = item >> 4, c8 = (item & 15) * 8;
      const int j = tok[tt];
      if (tt >= nr || j < 0) {
#pragma unroll
        for (int e = 0; e < 8; ++e) xs[tt][c8 + e] = 0.f;
        continue;
      }
      const size_t row = a.compact ? (size_t)(i0 + tt) : (size_t)(j - a.row0);
      float x[8];
      bf16x8(ldg_u4(src + (size_t)h * a.head_stride + row * kD + c8), x);
      if constexpr (CT::kFullState) {
#pragma unroll
        for (int e = 0; e < 8; ++e) xs[tt][c8 + e] = x[e];
      } else {
        float xh[8];
        recon8<false, kRB>(c, brec, rrec, mask, first, j, r, is_v, c8, xh);
#pragma unroll
        for (int e = 0; e < 8; ++e) xs[tt][c8 + e] = __fsub_rn(x[e], xh[e]);
      }
    }
    __syncthreads();

    if (is_v) value_params<kRB>(sm, orec, 0, kG, nr, tid, 256);
    else key_params<kRB>(sm, orec, 0, kD, nr, tid, 256);
    __syncthreads();
    if constexpr (kRB == 4) group_codes(sm, orec, is_v, 0, kG, 0, kD / 8, nr, tid, 256);
    else group_codes2(sm, orec, is_v, nr, tid, 256);
    __syncthreads();
  }

  if (h == 0 && tid < nr) {
    const int j = tok[tid];
    if (j >= 0) {
      unsigned long long* mk = arr<unsigned long long>(c, A_MASK, a.layer);
      int32_t* fs = arr<int32_t>(c, A_FIRST, a.layer);
      const int i = i0 + tid;
      atomicOr(&mk[(size_t)r * ncb + (j >> 6)], 1ull << (j & 63));
      if (i == 0 || (a.rows[i - 1] >> 6) != (j >> 6)) fs[(size_t)r * ncb + (j >> 6)] = a.slot0 + i;
      depth[j] = (uint8_t)r;
    }
  }
}

}  // namespace

cudaError_t launch_encode_base(const EncodeBaseArgs& a, cudaStream_t s) {
  dim3 grid(a.n_rows / kG, a.c.H);
  encode_base_kernel<<<grid, 256, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_encode_residual(const EncodeResArgs& a, cudaStream_t s) {
  if (a.n_rows == 0) return cudaSuccess;
  dim3 grid((a.n_rows + kG - 1) / kG, a.c.H);
  if (a.c.codec == FL_CODEC_FULL_INT4)
    encode_residual_kernel<FL_CODEC_FULL_INT4><<<grid, 256, 0, s>>>(a);
  else if (a.c.codec == FL_CODEC_RESIDUAL_INT2)
    encode_residual_kernel<FL_CODEC_RESIDUAL_INT2><<<grid, 256, 0, s>>>(a);
  else
    encode_residual_kernel<FL_CODEC_RESIDUAL_INT4><<<grid, 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace fl
