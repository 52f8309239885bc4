// Shared device helpers of the FlashLoop B200 decode-path library.
//
// Cache layout, quantiser and status conventions are declared in include/flashloop.h.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "flashloop.h"

namespace fl {

constexpr int kD = 128;     // head dim
constexpr int kG = 64;      // group size / block of tokens
constexpr int kTail = 64;   // BF16 tail rows
constexpr int kOffStride = FL_MAX_LOOPS + 1;  // offset[L][H][33]
constexpr int kMaxSplits = 256;
constexpr int kPartStride = 132;  // M, L, pad, pad, o[128]
constexpr unsigned kFull = 0xffffffffu;

// Array ids, in fl_layout order.
enum Arr {
  A_KCODE = 0, A_VCODE, A_KSZ, A_VSZ, A_RKCODE, A_RVCODE, A_RKSZ, A_RVSZ,
  A_MASK, A_FIRST, A_DEPTH, A_TAILK, A_TAILV, A_SCORE, A_TAG, A_OFFSET,
  A_SEL, A_MASS, A_UNSEL, A_COUNT
};

// Device view of one cache buffer: base pointer, array offsets and per-layer strides.
struct CacheView {
  uint8_t* base;
  uint64_t off[A_COUNT];
  uint64_t lstride[A_COUNT];
  int32_t slot_base[FL_MAX_LOOPS + 1];
  int32_t* status;
  int32_t H, R, cap, total_slots, max_select;
};

template <class T>
__device__ __forceinline__ T* arr(const CacheView& c, int a, int layer) {
  return reinterpret_cast<T*>(c.base + c.off[a] + c.lstride[a] * (uint64_t)layer);
}

__device__ __forceinline__ void record_error(int32_t* status, int code, int detail) {
  if (atomicCAS(&status[0], 0, code) == 0) atomicExch(&status[1], detail);
  atomicAdd(&status[2], 1);
}

// ---- loads ------------------------------------------------------------------
__device__ __forceinline__ uint4 ldg_u4(const void* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}
__device__ __forceinline__ uint32_t ldg_u32(const void* p) {
  return __ldg(reinterpret_cast<const unsigned int*>(p));
}

// ---- small math ---------------------------------------------------------------
// Hardware base-2 exponential (MUFU.EX2); exp2(-inf) = +0.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
  return v;
}

// (scale, zero) fp16 pair packed in a 32-bit word (scale in the low half).
__device__ __forceinline__ float2 unpack_sz(uint32_t w) {
  __half2 h = *reinterpret_cast<__half2*>(&w);
  return __half22float2(h);  // .x = scale, .y = zero
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// 1 + n/128 for the nibble n that sits at bits [16, 20) of w: an exact fp32 value,
// built with one logic op; the caller pre-scales its weights by 128 and removes the
// constant part separately.
__device__ __forceinline__ float nib16(uint32_t w) {
  return __uint_as_float((w & 0x000F0000u) | 0x3F800000u);
}

// Nibble k of a 32-bit code word is channel 8*word + k (byte b = channels 2b, 2b+1).
// sum_k q[k] * (1 + n_k/128) for the 8 nibbles of w.
__device__ __forceinline__ float dot8(uint32_t w, const float* q, float s) {
  s = fmaf(q[0], nib16(w << 16), s);
  s = fmaf(q[1], nib16(w << 12), s);
  s = fmaf(q[2], nib16(w << 8), s);
  s = fmaf(q[3], nib16(w << 4), s);
  s = fmaf(q[4], nib16(w), s);
  s = fmaf(q[5], nib16(w >> 4), s);
  s = fmaf(q[6], nib16(w >> 8), s);
  s = fmaf(q[7], nib16(w >> 12), s);
  return s;
}

// 32 channels (one 16-byte code quarter) against 32 pre-scaled weights.
__device__ __forceinline__ float dot32(uint4 w, const float* q) {
  float a = dot8(w.x, q, 0.f);
  float b = dot8(w.y, q + 8, 0.f);
  a = dot8(w.z, q + 16, a);
  b = dot8(w.w, q + 24, b);
  return a + b;
}

// acc[k] += P * (1 + n_k/128) over the 32 nibbles of a code quarter.
__device__ __forceinline__ void axpy8(uint32_t w, float P, float* acc) {
  acc[0] = fmaf(P, nib16(w << 16), acc[0]);
  acc[1] = fmaf(P, nib16(w << 12), acc[1]);
  acc[2] = fmaf(P, nib16(w << 8), acc[2]);
  acc[3] = fmaf(P, nib16(w << 4), acc[3]);
  acc[4] = fmaf(P, nib16(w), acc[4]);
  acc[5] = fmaf(P, nib16(w >> 4), acc[5]);
  acc[6] = fmaf(P, nib16(w >> 8), acc[6]);
  acc[7] = fmaf(P, nib16(w >> 12), acc[7]);
}
__device__ __forceinline__ void axpy32(uint4 w, float P, float* acc) {
  axpy8(w.x, P, acc);
  axpy8(w.y, P, acc + 8);
  axpy8(w.z, P, acc + 16);
  axpy8(w.w, P, acc + 24);
}

// 32 BF16 values (64 bytes at p) dotted with 32 fp32 weights.
__device__ __forceinline__ float dot_bf16_32(const uint16_t* p, const float* q) {
  const uint4* v = reinterpret_cast<const uint4*>(p);
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 w = __ldg(v + i);
    s = fmaf(q[8 * i + 0], bf16_lo(w.x), s);
    s = fmaf(q[8 * i + 1], bf16_hi(w.x), s);
    s = fmaf(q[8 * i + 2], bf16_lo(w.y), s);
    s = fmaf(q[8 * i + 3], bf16_hi(w.y), s);
    s = fmaf(q[8 * i + 4], bf16_lo(w.z), s);
    s = fmaf(q[8 * i + 5], bf16_hi(w.z), s);
    s = fmaf(q[8 * i + 6], bf16_lo(w.w), s);
    s = fmaf(q[8 * i + 7], bf16_hi(w.w), s);
  }
  return s;
}

__device__ __forceinline__ void axpy_bf16_32(const uint16_t* p, float P, float* acc) {
  const uint4* v = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 w = __ldg(v + i);
    acc[8 * i + 0] = fmaf(P, bf16_lo(w.x), acc[8 * i + 0]);
    acc[8 * i + 1] = fmaf(P, bf16_hi(w.x), acc[8 * i + 1]);
    acc[8 * i + 2] = fmaf(P, bf16_lo(w.y), acc[8 * i + 2]);
    acc[8 * i + 3] = fmaf(P, bf16_hi(w.y), acc[8 * i + 3]);
    acc[8 * i + 4] = fmaf(P, bf16_lo(w.z), acc[8 * i + 4]);
    acc[8 * i + 5] = fmaf(P, bf16_hi(w.z), acc[8 * i + 5]);
    acc[8 * i + 6] = fmaf(P, bf16_lo(w.w), acc[8 * i + 6]);
    acc[8 * i + 7] = fmaf(P, bf16_hi(w.w), acc[8 * i + 7]);
  }
}

// Per-lane share of a key group's pre-scaled query weights: lane l handles channels
// 4l..4l+3 of the group's (scale, zero) record; writes qs'_c = 128 * q_c * s_c to
// `qs_out` and returns the warp total of sum_c (q_c * z_c - qs'_c), the group's
// additive constant (so that sum_c qs'_c * (1 + n_c/128) + const = q . k_hat).
__device__ __forceinline__ float group_weights(const uint32_t* rec, const float* q_s, float* qs_out,
                                               int lane) {
  uint4 r = ldg_u4(rec + 4 * lane);
  float4 qv = *reinterpret_cast<const float4*>(q_s + 4 * lane);
  float2 a = unpack_sz(r.x), b = unpack_sz(r.y), c = unpack_sz(r.z), d = unpack_sz(r.w);
  float4 w;
  w.x = 128.f * (qv.x * a.x);
  w.y = 128.f * (qv.y * b.x);
  w.z = 128.f * (qv.z * c.x);
  w.w = 128.f * (qv.w * d.x);
  float cpart = fmaf(qv.x, a.y, -w.x) + fmaf(qv.y, b.y, -w.y) + fmaf(qv.z, c.y, -w.z) +
                fmaf(qv.w, d.y, -w.w);
  *reinterpret_cast<float4*>(qs_out + 4 * lane) = w;
  return warp_sum(cpart);
}

__device__ __forceinline__ void load32(const float* src, float* dst) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float4 v = *reinterpret_cast<const float4*>(src + 4 * i);
    dst[4 * i + 0] = v.x;
    dst[4 * i + 1] = v.y;
    dst[4 * i + 2] = v.z;
    dst[4 * i + 3] = v.w;
  }
}

// log2(e) / sqrt(128): scores are kept in the base-2 domain.
constexpr float kQScale = 1.4426950408889634f * 0.08838834764831845f;

}  // namespace fl
