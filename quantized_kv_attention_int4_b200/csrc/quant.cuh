// Group quantiser shared by the encode kernels and the readers' fused tail flush.
//
// flozi guide "FlashLoop: store changes between repeated passes", section 3:
// group-wise asymmetric 4-bit codes, group 64, keys grouped per channel, values per
// token; section 4 and the 2-bit row of its Figure 5: 2-bit residual codes.  Every
// arithmetic step is one IEEE fp32 operation with an explicit round-to-nearest
// intrinsic, so codes, scales and zero points are exact functions of the inputs (the
// contract in include/flashloop.h): s = fp16_rn((max - min) / L), z = fp16_rn(min),
// code = clamp(rint_even((x - z) / s), 0, L), x_hat = fma(code, s, z), with L = 15
// for 4-bit codes and 3 for 2-bit codes.
#pragma once

#include "common.cuh"

namespace fl {

__device__ __forceinline__ uint32_t pack_sz(__half s, __half z) {
  return (uint32_t)__half_as_ushort(s) | ((uint32_t)__half_as_ushort(z) << 16);
}

// One group's scale and zero from its exact min and max.
template <int kBits = 4>
__device__ __forceinline__ void group_sz(float mn, float mx, __half& hs, __half& hz) {
  hs = __float2half_rn(__fdiv_rn(__fsub_rn(mx, mn), Rec<kBits>::kLevels));
  hz = __float2half_rn(mn);
}

template <int kBits = 4>
__device__ __forceinline__ uint32_t quant(float x, float s, float z) {
  if (s == 0.0f) return 0u;
  int q = __float2int_rn(__fdiv_rn(__fsub_rn(x, z), s));  // round half to even
  q = q < 0 ? 0 : (q > Rec<kBits>::kMaxCode ? Rec<kBits>::kMaxCode : q);
  return (uint32_t)q;
}

__device__ __forceinline__ float deq(uint32_t code, float2 sz) {
  return __fmaf_rn((float)code, sz.x, sz.y);
}

// Eight BF16 values of one uint4 as fp32.
__device__ __forceinline__ void bf16x8(uint4 w, float* x) {
  x[0] = bf16_lo(w.x);
  x[1] = bf16_hi(w.x);
  x[2] = bf16_lo(w.y);
  x[3] = bf16_hi(w.y);
  x[4] = bf16_lo(w.z);
  x[5] = bf16_hi(w.z);
  x[6] = bf16_lo(w.w);
  x[7] = bf16_hi(w.w);
}

// Loads of stored records: through L2 (ld.global.cg) with kL2, for records that an
// earlier kernel of a dependent launch chain wrote; plain loads otherwise.
template <bool kL2, class T>
__device__ __forceinline__ T ld_rec(const T* p) {
  if constexpr (kL2) return __ldcg(p);
  else return *p;
}

// Dequantised channels c8 .. c8 + 7 (c8 a multiple of 8) of row `row` of group record g
// (kBits-bit codes): keys use the record's per-channel (scale, zero) words, values the
// row's half.
template <bool kL2, int kBits = 4>
__device__ __forceinline__ void deq8(const uint8_t* g, int row, bool is_v, int c8, float* out) {
  using RB = Rec<kBits>;
  uint32_t cw;
  if constexpr (kBits == 4) {
    cw = ld_rec<kL2>(reinterpret_cast<const unsigned int*>(g + (size_t)row * RB::kRow + (is_v ? RB::kHalf : 0) + c8 / 2));
  } else {
    cw = int2_word(ld_rec<kL2>(reinterpret_cast<const unsigned int*>(g + (size_t)row * RB::kRow + (is_v ? RB::kHalf : 0) +
                                                                     (c8 >> 4) * 4)),
                   (c8 >> 3) & 1);
  }
  if (is_v) {
    const float2 sz = unpack_sz(ld_rec<kL2>(reinterpret_cast<const unsigned int*>(g + RB::kVsz) + row * 2 + (c8 >> 6)));
#pragma unroll
    for (int e = 0; e < 8; ++e) out[e] = deq((cw >> (4 * e)) & 15u, sz);
  } else {
    const uint4* ks = reinterpret_cast<const uint4*>(g + RB::kKsz + (size_t)c8 * 4);
    const uint4 lo = ld_rec<kL2>(ks), hi = ld_rec<kL2>(ks + 1);
    const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) out[e] = deq((cw >> (4 * e)) & 15u, unpack_sz(w[e]));
  }
}

// X_hat^(r-1) of channels c8 .. c8 + 7 of token j (keys, or values when is_v): the base
// record's dequantised row plus the residual stores 2 .. r - 1 that hold j, added in
// loop order (FlashLoop project page, "The Method", Step 03).  brec / rrec are the
// head's base and residual record arrays; the residual records have kResBits-bit codes.
template <bool kL2, int kResBits = 4>
__device__ __forceinline__ void recon8(const CacheView& c, const uint8_t* brec, const uint8_t* rrec,
                                       const unsigned long long* mask, const int32_t* first, int j, int r,
                                       bool is_v, int c8, float* xh) {
  const int ncb = c.cap / kG, b = j >> 6, jt = j & 63;
  deq8<kL2>(brec + (size_t)b * kRec, jt, is_v, c8, xh);
  for (int rp = 2; rp < r; ++rp) {
    const unsigned long long mk = ld_rec<kL2>(mask + (size_t)rp * ncb + b);
    const int gs = c.slot_base[rp] + ld_rec<kL2>(first + (size_t)rp * ncb + b) + __popcll(mk & ((1ull << jt) - 1ull));
    float d[8];
    deq8<kL2, kResBits>(rrec + (size_t)(gs >> 6) * Rec<kResBits>::kBytes, gs & 63, is_v, c8, d);
#pragma unroll
    for (int e = 0; e < 8; ++e) xh[e] = __fadd_rn(xh[e], d[e]);
  }
}

// Shared memory of one group encode: the 64 x 128 fp32 inputs (padded rows), the group
// parameters, a slot -> row map and per-store metadata.
struct EncodeSmem {
  float xs[kG][129];
  float sk[kD], zk[kD];
  float sv[kG][2], zv[kG][2];
  int row[kG];
  int g0[FL_MAX_LOOPS + 1];                 // first global slot of the block in store r
  unsigned long long mk[FL_MAX_LOOPS + 1];  // the block's mask in store r
};

// Key groups of channels [ch0, ch0 + nch): scale/zero over xs rows 0 .. nr - 1, written
// to the record's per-channel words and to shared memory.  Block-strided over tid / nt.
template <int kBits = 4>
__device__ __forceinline__ void key_params(EncodeSmem& sm, uint8_t* rec, int ch0, int nch, int nr, int tid, int nt) {
  uint32_t* ks = reinterpret_cast<uint32_t*>(rec + Rec<kBits>::kKsz);
  for (int i = tid; i < nch; i += nt) {
    const int ch = ch0 + i;
    float mn = sm.xs[0][ch], mx = mn;
    for (int rr = 1; rr < nr; ++rr) {
      mn = fminf(mn, sm.xs[rr][ch]);
      mx = fmaxf(mx, sm.xs[rr][ch]);
    }
    __half hs, hz;
    group_sz<kBits>(mn, mx, hs, hz);
    sm.sk[ch] = __half2float(hs);
    sm.zk[ch] = __half2float(hz);
    ks[ch] = pack_sz(hs, hz);
  }
}

// Value groups of rows [t0, t0 + nt_rows), one per (row, 64-channel half); rows >= nr
// (absent slots) get zero words.
template <int kBits = 4>
__device__ __forceinline__ void value_params(EncodeSmem& sm, uint8_t* rec, int t0, int n_rows, int nr, int tid,
                                             int nt) {
  uint32_t* vs = reinterpret_cast<uint32_t*>(rec + Rec<kBits>::kVsz);
  for (int i = tid; i < 2 * n_rows; i += nt) {
    const int tt = t0 + (i >> 1), hf = i & 1;
    float sval = 0.f, zval = 0.f;
    uint32_t packed = 0u;
    if (tt < nr) {
      float mn = sm.xs[tt][64 * hf], mx = mn;
      for (int ch = 1; ch < 64; ++ch) {
        mn = fminf(mn, sm.xs[tt][64 * hf + ch]);
        mx = fmaxf(mx, sm.xs[tt][64 * hf + ch]);
      }
      __half hs, hz;
      group_sz<kBits>(mn, mx, hs, hz);
      sval = __half2float(hs);
      zval = __half2float(hz);
      packed = pack_sz(hs, hz);
    }
    sm.sv[tt][hf] = sval;
    sm.zv[tt][hf] = zval;
    vs[tt * 2 + hf] = packed;
  }
}

// Code words of rows [t0, t0 + n_rows) x 8-channel words [w0, w0 + nw) of one part: word
// w of row t holds channels 8w .. 8w + 7, one nibble each (low nibble first); rows >= nr
// get zero words.
__device__ __forceinline__ void group_codes(const EncodeSmem& sm, uint8_t* rec, bool is_v, int t0, int n_rows,
                                            int w0, int nw, int nr, int tid, int nt) {
  uint32_t* words = reinterpret_cast<uint32_t*>(rec + (is_v ? 64 : 0));
  for (int i = tid; i < n_rows * nw; i += nt) {
    const int t = t0 + i / nw, w = w0 + i % nw;
    uint32_t word = 0u;
    if (t < nr) {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int ch = 8 * w + k;
        const float s = is_v ? sm.sv[t][ch >> 6] : sm.sk[ch];
        const float z = is_v ? sm.zv[t][ch >> 6] : sm.zk[ch];
        word |= quant(sm.xs[t][ch], s, z) << (4 * k);
      }
    }
    words[(size_t)t * 32 + w] = word;
  }
}

// 2-bit code words of every row of one part (the layout in include/flashloop.h: word w
// of a row's part holds channels 16w .. 16w + 15); rows >= nr get zero words.
__device__ __forceinline__ void group_codes2(const EncodeSmem& sm, uint8_t* rec, bool is_v, int nr, int tid, int nt) {
  uint32_t* words = reinterpret_cast<uint32_t*>(rec + (is_v ? Rec<2>::kHalf : 0));
  for (int i = tid; i < kG * 8; i += nt) {
    const int t = i >> 3, w = i & 7;
    uint32_t word = 0u;
    if (t < nr) {
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const int ch = 16 * w + k;
        const float s = is_v ? sm.sv[t][ch >> 6] : sm.sk[ch];
        const float z = is_v ? sm.zv[t][ch >> 6] : sm.zk[ch];
        word |= quant<2>(sm.xs[t][ch], s, z) << (k < 8 ? 4 * k : 4 * (k - 8) + 2);
      }
    }
    words[(size_t)t * (Rec<2>::kRow / 4) + w] = word;
  }
}

}  // namespace fl
