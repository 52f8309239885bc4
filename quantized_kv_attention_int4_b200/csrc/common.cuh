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
constexpr int kPartStride = 260;  // M, L, m, pad, o[128], u[128]
constexpr unsigned kFull = 0xffffffffu;

// Array ids, in fl_layout order.
enum Arr {
  A_BREC = 0, A_RREC, A_MASK, A_FIRST, A_DEPTH, A_TAILK, A_TAILV, A_SCORE, A_TAG, A_OFFSET,
  A_SEL, A_MASS, A_UNSEL, A_PLAN, A_COUNT
};

// Group record: 64 rows of (64 B key codes, 64 B value codes), then 64 x 2 value
// (scale, zero) words, then 128 key (scale, zero) words.
constexpr int kRec = FL_GROUP_RECORD;
constexpr int kRecVsz = 8192;
constexpr int kRecKsz = 8704;

// Byte geometry of a group record with kBits-bit codes: 4 (the base, and the residual
// stores of the 4-bit codecs) or 2 (2-bit residual stores: 64-byte rows of 32 B key
// codes and 32 B value codes, the value and key (scale, zero) words after them).
template <int kBits>
struct Rec {
  static constexpr int kBytes = kBits == 4 ? FL_GROUP_RECORD : FL_GROUP_RECORD_INT2;
  static constexpr int kRow = kBits == 4 ? 128 : 64;  // bytes of one row
  static constexpr int kHalf = kRow / 2;              // offset of the value codes in a row
  static constexpr int kVsz = kG * kRow;
  static constexpr int kKsz = kVsz + kG * 8;
  static constexpr float kLevels = kBits == 4 ? 15.0f : 3.0f;
  static constexpr int kMaxCode = kBits == 4 ? 15 : 3;
};
static_assert(Rec<4>::kVsz == kRecVsz && Rec<4>::kKsz == kRecKsz, "4-bit record geometry");
static_assert(Rec<2>::kKsz + 512 == FL_GROUP_RECORD_INT2, "2-bit record geometry");

// What the loop r >= 2 stores of a codec hold (FL_CODEC_*): full states or residuals,
// and their code width.
template <int kCodec>
struct CodecT {
  static constexpr bool kFullState = kCodec == FL_CODEC_FULL_INT4;
  static constexpr int kResBits = kCodec == FL_CODEC_RESIDUAL_INT2 ? 2 : 4;
};

// A 2-bit record word holds channels 16w .. 16w + 15: channel 16w + k (k < 8) in bits
// 4k .. 4k + 1 and 16w + 8 + k in bits 4k + 2 .. 4k + 3.  Masking gives the 4-bit
// layout's 8-channel words (channel k in nibble k) with codes 0 .. 3.
constexpr uint32_t kInt2Mask = 0x33333333u;
__device__ __forceinline__ uint32_t int2_word(uint32_t w, int upper) { return (w >> (2 * upper)) & kInt2Mask; }
// 32 consecutive channels of 2-bit codes (8 bytes) as the 16-byte 4-bit layout.
__device__ __forceinline__ uint4 int2_to_nib(uint2 x) {
  return make_uint4(x.x & kInt2Mask, (x.x >> 2) & kInt2Mask, x.y & kInt2Mask, (x.y >> 2) & kInt2Mask);
}

// Device view of one cache buffer: base pointer, array offsets and per-layer strides.
struct CacheView {
  uint8_t* base;
  uint64_t off[A_COUNT];
  uint64_t lstride[A_COUNT];
  int32_t slot_base[FL_MAX_LOOPS + 1];
  int32_t* status;
  int32_t H, R, cap, total_slots, max_select, plan_stride;
  int32_t codec;  // FL_CODEC_*
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
// Warp maximum in one redux.sync: floats map to signed integers in the same order
// (non-negative ones keep their bits, negative ones flip their magnitude bits), so the
// integer maximum is the image of the float maximum (inputs are never NaN).
__device__ __forceinline__ float warp_max(float v) {
  const int b = __float_as_int(v);
  const int m = __reduce_max_sync(kFull, b >= 0 ? b : b ^ 0x7fffffff);
  return __int_as_float(m >= 0 ? m : m ^ 0x7fffffff);
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

// group_weights for a record already in shared memory, rewritten in place as fp32
// weights qs'_c; returns the record's additive constant.
__device__ __forceinline__ float group_weights_smem(uint32_t* rec, const float* q_s, int lane) {
  const uint4 r = *reinterpret_cast<const uint4*>(rec + 4 * lane);
  const float4 qv = *reinterpret_cast<const float4*>(q_s + 4 * lane);
  const float2 a = unpack_sz(r.x), b = unpack_sz(r.y), c = unpack_sz(r.z), d = unpack_sz(r.w);
  float4 w;
  w.x = 128.f * (qv.x * a.x);
  w.y = 128.f * (qv.y * b.x);
  w.z = 128.f * (qv.z * c.x);
  w.w = 128.f * (qv.w * d.x);
  const float cpart = fmaf(qv.x, a.y, -w.x) + fmaf(qv.y, b.y, -w.y) + fmaf(qv.z, c.y, -w.z) +
                      fmaf(qv.w, d.y, -w.w);
  *reinterpret_cast<float4*>(rec + 4 * lane) = w;
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

// ---- asynchronous bulk copies (TMA engine) into shared memory, mbarrier completion ----
__device__ __forceinline__ unsigned smem_addr(const void* p) { return (unsigned)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("{ .reg .b64 st; mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1; }" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}
// global -> shared bulk copy; dst, src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// try_wait that lets the hardware suspend the thread for up to `ns` nanoseconds while
// the phase is incomplete (no issue slots are spent meanwhile).
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, unsigned parity, unsigned ns) {
  unsigned ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3; selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}
// Bounded wait for phase `parity` of `bar` (2 s of device time); false if the bound ran out.
constexpr uint64_t kWaitNs = 2000000000ull;
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, unsigned parity) {
  if (mbar_try_wait_sleep(bar, parity, 1000000u)) return true;
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait_sleep(bar, parity, 1000000u))
    if (global_ns() - t0 > kWaitNs) return false;
  return true;
}

// fp32 accumulate of an fp16 product: acc += a * b with a, b binary16 (exact product).
__device__ __forceinline__ void hfma_f32(float& acc, unsigned short a, unsigned short b) {
  asm("{ .reg .f16 x, y; mov.b16 x, %1; mov.b16 y, %2; fma.rn.f32.f16 %0, x, y, %0; }"
      : "+f"(acc)
      : "h"(a), "h"(b));
}

// acc[k] += code_k * (weight) over the 8 nibbles of one code word, with the nibbles
// turned into binary16 values 1024 + n (even channels, weight we) and 1024 + 16 n (odd
// channels, weight wo = we / 16); the constant 1024 * weight per channel is removed by
// the caller's correction terms.  Channel order follows the code word: nibble k at
// bits 4k..4k+3 is channel k.
__device__ __forceinline__ void axpy8_h(uint32_t w, unsigned short we, unsigned short wo, float* acc) {
  const uint32_t a = (w & 0x000F000Fu) | 0x64006400u;          // ch 0, 4
  const uint32_t b = (w & 0x00F000F0u) | 0x64006400u;          // ch 1, 5 (x16)
  const uint32_t w8 = w >> 8;
  const uint32_t c = (w8 & 0x000F000Fu) | 0x64006400u;         // ch 2, 6
  const uint32_t d = (w8 & 0x00F000F0u) | 0x64006400u;         // ch 3, 7 (x16)
  hfma_f32(acc[0], (unsigned short)a, we);
  hfma_f32(acc[4], (unsigned short)(a >> 16), we);
  hfma_f32(acc[1], (unsigned short)b, wo);
  hfma_f32(acc[5], (unsigned short)(b >> 16), wo);
  hfma_f32(acc[2], (unsigned short)c, we);
  hfma_f32(acc[6], (unsigned short)(c >> 16), we);
  hfma_f32(acc[3], (unsigned short)d, wo);
  hfma_f32(acc[7], (unsigned short)(d >> 16), wo);
}

// 2^e as an fp32 value, for -126 <= e <= 127 (built from the exponent field).
__device__ __forceinline__ float pow2i(int e) { return __int_as_float((e + 127) << 23); }
// The exponent e of x > 0 written as f * 2^e with f in [0.5, 1); subnormal x gives -126.
__device__ __forceinline__ int exp_frexp(float x) { return (int)((__float_as_uint(x) >> 23) & 0xffu) - 126; }

// ---- exact integer key dots (dp4a) against fixed-point query weights ----
// A key group's weights qs_c = q_c * s_c become Q_c = rint(qs_c * 2^E) with
// |Q_c| < 2^23 (24-bit fixed point, E per record from the largest |qs_c|), split into
// bytes b0, b1 (unsigned) and b2 (signed): Q = b2 * 2^16 + b1 * 2^8 + b0.  For code
// word w (channels 8w..8w+7, nibble k = channel 8w + k) the limbs are 6 words:
// b0, b1, b2 of the even channels (8w, 8w+2, 8w+4, 8w+6), then b0, b1, b2 of the odd
// channels -- matching the low / high nibbles of the code word's four bytes.
constexpr int kLimbWords = 6;
constexpr int kLimbE = 16 * kLimbWords;   // record word holding E
constexpr int kLimbC = kLimbE + 1;        // record word holding C = sum_c q_c z_c (fp32 bits)

// One warp turns a key (scale, zero) record (128 words: channel c at word c, scale in
// the low half) into limbs in place: words 0..95 limbs, word 96 E, word 97 C.
__device__ __forceinline__ void record_to_limbs(uint32_t* rec, const float* q_s, int lane) {
  const uint4 raw = *reinterpret_cast<const uint4*>(rec + 4 * lane);
  const float4 qv = *reinterpret_cast<const float4*>(q_s + 4 * lane);
  const float2 s0 = unpack_sz(raw.x), s1 = unpack_sz(raw.y), s2 = unpack_sz(raw.z), s3 = unpack_sz(raw.w);
  const float qs0 = qv.x * s0.x, qs1 = qv.y * s1.x, qs2 = qv.z * s2.x, qs3 = qv.w * s3.x;
  float cz = fmaf(qv.x, s0.y, fmaf(qv.y, s1.y, fmaf(qv.z, s2.y, qv.w * s3.y)));
  float mx = fmaxf(fmaxf(fabsf(qs0), fabsf(qs1)), fmaxf(fabsf(qs2), fabsf(qs3)));
  mx = warp_max(mx);
  cz = warp_sum(cz);
  int E = 0;
  if (mx > 0.f) E = min(23 - exp_frexp(mx), 126);
  const float sc = pow2i(E);
  auto fix = [&](float v) {
    const int x = __float2int_rn(v * sc);
    return x > 8388607 ? 8388607 : (x < -8388607 ? -8388607 : x);
  };
  const int Q0 = fix(qs0), Q1 = fix(qs1), Q2 = fix(qs2), Q3 = fix(qs3);
  __syncwarp();
  // lane l holds channels 4l..4l+3 of code word w = l/2: even channels 4l, 4l+2 and odd
  // channels 4l+1, 4l+3 fill bytes 2*(l&1), 2*(l&1)+1 of the word's limb words.
  const int w = lane >> 1, hb = (lane & 1) * 2;
  uint16_t* lh = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(rec + kLimbWords * w) + hb);
  // byte sh / 8 of a, then the same byte of b (one byte permute)
  auto pair = [](int a, int b, int sh) { return (uint16_t)__byte_perm(a, b, (unsigned)((sh >> 3) | ((4 + (sh >> 3)) << 4))); };
  lh[0] = pair(Q0, Q2, 0);
  lh[2] = pair(Q0, Q2, 8);
  lh[4] = pair(Q0, Q2, 16);
  lh[6] = pair(Q1, Q3, 0);
  lh[8] = pair(Q1, Q3, 8);
  lh[10] = pair(Q1, Q3, 16);
  if (lane == 0) {
    rec[kLimbE] = (uint32_t)E;
    rec[kLimbC] = __float_as_uint(cz);
  }
}

// record_to_limbs for two records at once (ra, rb), so that their reductions and shared
// memory round trips overlap; the same words as two calls.
__device__ __forceinline__ void record_to_limbs2(uint32_t* ra, uint32_t* rb, const float* q_s, int lane) {
  uint32_t* rec[2] = {ra, rb};
  const float4 qv = *reinterpret_cast<const float4*>(q_s + 4 * lane);
  float qs[2][4], cz[2], mx[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const uint4 raw = *reinterpret_cast<const uint4*>(rec[i] + 4 * lane);
    const float2 s0 = unpack_sz(raw.x), s1 = unpack_sz(raw.y), s2 = unpack_sz(raw.z), s3 = unpack_sz(raw.w);
    qs[i][0] = qv.x * s0.x;
    qs[i][1] = qv.y * s1.x;
    qs[i][2] = qv.z * s2.x;
    qs[i][3] = qv.w * s3.x;
    cz[i] = fmaf(qv.x, s0.y, fmaf(qv.y, s1.y, fmaf(qv.z, s2.y, qv.w * s3.y)));
    mx[i] = fmaxf(fmaxf(fabsf(qs[i][0]), fabsf(qs[i][1])), fmaxf(fabsf(qs[i][2]), fabsf(qs[i][3])));
  }
  mx[0] = warp_max(mx[0]);
  mx[1] = warp_max(mx[1]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    cz[0] += __shfl_xor_sync(kFull, cz[0], o);
    cz[1] += __shfl_xor_sync(kFull, cz[1], o);
  }
  int Q[2][4], E[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    E[i] = mx[i] > 0.f ? min(23 - exp_frexp(mx[i]), 126) : 0;
    const float sc = pow2i(E[i]);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int x = __float2int_rn(qs[i][k] * sc);
      Q[i][k] = x > 8388607 ? 8388607 : (x < -8388607 ? -8388607 : x);
    }
  }
  __syncwarp();
  const int w = lane >> 1, hb = (lane & 1) * 2;
  // byte sh / 8 of a, then the same byte of b (one byte permute)
  auto pair = [](int a, int b, int sh) { return (uint16_t)__byte_perm(a, b, (unsigned)((sh >> 3) | ((4 + (sh >> 3)) << 4))); };
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    uint16_t* lh = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(rec[i] + kLimbWords * w) + hb);
    lh[0] = pair(Q[i][0], Q[i][2], 0);
    lh[2] = pair(Q[i][0], Q[i][2], 8);
    lh[4] = pair(Q[i][0], Q[i][2], 16);
    lh[6] = pair(Q[i][1], Q[i][3], 0);
    lh[8] = pair(Q[i][1], Q[i][3], 8);
    lh[10] = pair(Q[i][1], Q[i][3], 16);
    if (lane == 0) {
      rec[i][kLimbE] = (uint32_t)E[i];
      rec[i][kLimbC] = __float_as_uint(cz[i]);
    }
  }
}

// Dot of one 32-channel quarter of a code row (4 code words) with the record's 24 limb
// words of that quarter (words 24*qq.., held in registers), in units of 2^-E.  Odd
// channels are taken in place (their nibble x16) and scaled back here.
__device__ __forceinline__ float limb_dot(uint4 code, const uint32_t* L) {
  int e0 = 0, e1 = 0, e2 = 0, o0 = 0, o1 = 0, o2 = 0;
  const uint32_t cw[4] = {code.x, code.y, code.z, code.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t ne = cw[i] & 0x0F0F0F0Fu, no = cw[i] & 0xF0F0F0F0u;
    asm("dp4a.u32.u32 %0, %1, %2, %0;" : "+r"(e0) : "r"(ne), "r"(L[6 * i + 0]));
    asm("dp4a.u32.u32 %0, %1, %2, %0;" : "+r"(e1) : "r"(ne), "r"(L[6 * i + 1]));
    asm("dp4a.u32.s32 %0, %1, %2, %0;" : "+r"(e2) : "r"(ne), "r"(L[6 * i + 2]));
    asm("dp4a.u32.u32 %0, %1, %2, %0;" : "+r"(o0) : "r"(no), "r"(L[6 * i + 3]));
    asm("dp4a.u32.u32 %0, %1, %2, %0;" : "+r"(o1) : "r"(no), "r"(L[6 * i + 4]));
    asm("dp4a.u32.s32 %0, %1, %2, %0;" : "+r"(o2) : "r"(no), "r"(L[6 * i + 5]));
  }
  const int le = e1 * 256 + e0, lo = o1 * 256 + o0;
  return fmaf((float)e2, 65536.f, (float)le) + 0.0625f * fmaf((float)o2, 65536.f, (float)lo);
}

// The 24 limb words of quarter qq of a converted record, into registers.
__device__ __forceinline__ void load_limbs(const uint32_t* rec, int qq, uint32_t* L) {
  const uint4* p = reinterpret_cast<const uint4*>(rec) + 6 * qq;
#pragma unroll
  for (int j = 0; j < 6; ++j) {
    const uint4 x = p[j];
    L[4 * j + 0] = x.x;
    L[4 * j + 1] = x.y;
    L[4 * j + 2] = x.z;
    L[4 * j + 3] = x.w;
  }
}

// ---- exact integer value sums (dp4a) against fixed-point row weights ----
__device__ __forceinline__ void dp4a_u(int& acc, uint32_t a, uint32_t b) {
  asm("dp4a.u32.u32 %0, %1, %2, %0;" : "+r"(acc) : "r"(a), "r"(b));
}

// Four rows' code words x0..x3 (same word, channels 8w..8w+7) against the four rows'
// weight limbs (byte 0, 1, 2 words): a0/a1/a2[c] accumulate channel 8w + c (odd
// channels x16).
__device__ __forceinline__ void v_group(uint32_t x0, uint32_t x1, uint32_t x2, uint32_t x3, uint4 wq,
                                        int* a0, int* a1, int* a2) {
  const uint32_t a_lo = __byte_perm(x0, x1, 0x5140), a_hi = __byte_perm(x0, x1, 0x7362);
  const uint32_t b_lo = __byte_perm(x2, x3, 0x5140), b_hi = __byte_perm(x2, x3, 0x7362);
  uint32_t T[4];
  T[0] = __byte_perm(a_lo, b_lo, 0x5410);  // byte 0 of rows 0..3
  T[1] = __byte_perm(a_lo, b_lo, 0x7632);  // byte 1
  T[2] = __byte_perm(a_hi, b_hi, 0x5410);  // byte 2
  T[3] = __byte_perm(a_hi, b_hi, 0x7632);  // byte 3
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    const uint32_t ev = T[b] & 0x0F0F0F0Fu, od = T[b] & 0xF0F0F0F0u;
    dp4a_u(a0[2 * b], ev, wq.x);
    dp4a_u(a1[2 * b], ev, wq.y);
    dp4a_u(a2[2 * b], ev, wq.z);
    dp4a_u(a0[2 * b + 1], od, wq.x);
    dp4a_u(a1[2 * b + 1], od, wq.y);
    dp4a_u(a2[2 * b + 1], od, wq.z);
  }
}

__device__ __forceinline__ uint32_t fix24(float w, float sc) {
  const uint32_t q = __float2uint_rn(w * sc);
  return q > 16777215u ? 16777215u : q;
}

// Row weights w >= 0 of one 4-row group (lanes 4m..4m+3 hold rows 4m..4m+3) as 24-bit
// fixed point at scale sc, gathered to lane 4m as three limb words (bytes 0, 1, 2 of the
// four rows' values; the fourth word is 0).
__device__ __forceinline__ uint4 pack_group24(float wgt, float sc) {
  const uint32_t Q = fix24(wgt, sc);
  const uint32_t Qb = __shfl_down_sync(kFull, Q, 1), Qc = __shfl_down_sync(kFull, Q, 2),
                 Qd = __shfl_down_sync(kFull, Q, 3);
  const uint32_t A = __byte_perm(Q, Qb, 0x5140), B = __byte_perm(Qc, Qd, 0x5140);
  const uint32_t C = __byte_perm(Q, Qb, 0x7362), D = __byte_perm(Qc, Qd, 0x7362);
  return make_uint4(__byte_perm(A, B, 0x5410), __byte_perm(A, B, 0x7632), __byte_perm(C, D, 0x5410), 0u);
}

// The exponent E of a 24-bit fixed-point scale for weights whose largest is mx (0 if none).
__device__ __forceinline__ int fix24_exp(float mx) { return mx > 0.f ? min(24 - exp_frexp(mx), 126) : 0; }

// ---- programmatic dependent launch ----
// A reader lets the next kernel of its stream start as soon as all of its own CTAs are
// running (the next reader stages and computes meanwhile), and waits for the previous
// kernel to finish before it touches the state readers share: the split partials and
// tickets of the workspace, and the previous loop's outputs.  Both are no-ops for a
// kernel launched without the programmatic-serialization attribute.
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Launch `kernel` on `s`; with `chain`, programmatic stream serialization is allowed
// (the kernel may start while its predecessor finishes), otherwise it is an ordinary
// stream-ordered launch.
template <class... KArgs, class... Args>
inline cudaError_t launch_pdl_if(bool chain, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                 cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = chain ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <class... KArgs, class... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args) {
  return launch_pdl_if(true, kernel, grid, block, smem, s, args...);
}

// log2(e) / sqrt(128): scores are kept in the base-2 domain.
constexpr float kQScale = 1.4426950408889634f * 0.08838834764831845f;

}  // namespace fl
