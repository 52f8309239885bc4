// Base (loop 1) and residual (loop r >= 2) INT4 encoders.
//
// FlashLoop project page, "The Method", Step 03: loop-1 K/V are quantised as the
// base; each later loop stores only its residual against the reconstructed state of
// the preceding loop.  flozi guide "FlashLoop: store changes between repeated
// passes", section 3: group-wise asymmetric 4-bit, group 64, keys per channel,
// values per token, residuals for active tokens only.
//
// Every arithmetic step of the quantiser is one IEEE fp32 operation with explicit
// round-to-nearest intrinsics so that codes, scales and zero points are exact
// functions of the inputs (the contract in include/flashloop.h).
#include "kernels.h"

namespace fl {
namespace {

__device__ __forceinline__ uint32_t pack_sz(__half s, __half z) {
  return (uint32_t)__half_as_ushort(s) | ((uint32_t)__half_as_ushort(z) << 16);
}

// One group's scale and zero from its exact min and max.
__device__ __forceinline__ void group_sz(float mn, float mx, __half& hs, __half& hz) {
  hs = __float2half_rn(__fdiv_rn(__fsub_rn(mx, mn), 15.0f));
  hz = __float2half_rn(mn);
}

__device__ __forceinline__ uint32_t quant(float x, float s, float z) {
  if (s == 0.0f) return 0u;
  int q = __float2int_rn(__fdiv_rn(__fsub_rn(x, z), s));  // round half to even
  q = q < 0 ? 0 : (q > 15 ? 15 : q);
  return (uint32_t)q;
}

__device__ __forceinline__ float deq(uint32_t code, float2 sz) {
  return __fmaf_rn((float)code, sz.x, sz.y);
}

// 64 rows x 128 BF16 (row i at src + i*128) into xs as fp32.
__device__ __forceinline__ void load_rows(const uint16_t* src, float (*xs)[129], int tid) {
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    int i = tid + 256 * it;
    int row = i >> 4, c8 = (i & 15) * 8;
    uint4 w = ldg_u4(src + (size_t)row * kD + c8);
    xs[row][c8 + 0] = bf16_lo(w.x);
    xs[row][c8 + 1] = bf16_hi(w.x);
    xs[row][c8 + 2] = bf16_lo(w.y);
    xs[row][c8 + 3] = bf16_hi(w.y);
    xs[row][c8 + 4] = bf16_lo(w.z);
    xs[row][c8 + 5] = bf16_hi(w.z);
    xs[row][c8 + 6] = bf16_lo(w.w);
    xs[row][c8 + 7] = bf16_hi(w.w);
  }
}

// Thread (row t = tid/4, channel quarter qq = tid%4) packs 32 codes of row t.
template <class SZ>
__device__ __forceinline__ uint4 pack_quarter(const float (*xs)[129], int t, int qq, SZ sz_of) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t word = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      int ch = 32 * qq + 8 * i + k;
      float2 sz = sz_of(t, ch);
      word |= quant(xs[t][ch], sz.x, sz.y) << (4 * k);
    }
    w[i] = word;
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

__global__ void __launch_bounds__(256) encode_base_kernel(EncodeBaseArgs a) {
  const int blk = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
  const CacheView& c = a.c;
  const int cap = c.cap, ncb = cap / kG;
  const int tok0 = a.row0 + blk * kG, gb = tok0 / kG;
  __shared__ float xs[kG][129];
  __shared__ float sk[kD], zk[kD];
  __shared__ float sv[kG][2], zv[kG][2];

  uint8_t* rec = arr<uint8_t>(c, A_BREC, a.layer) + ((size_t)h * ncb + gb) * kRec;
  uint32_t* ksz = reinterpret_cast<uint32_t*>(rec + kRecKsz);
  uint32_t* vsz = reinterpret_cast<uint32_t*>(rec + kRecVsz);
  const size_t in_off = (size_t)h * a.head_stride + (size_t)blk * kG * kD;
  const int t = tid >> 2, qq = tid & 3;

  // keys: one group per (block, channel)
  load_rows(a.k + in_off, xs, tid);
  __syncthreads();
  if (tid < kD) {
    float mn = xs[0][tid], mx = mn;
    for (int r = 1; r < kG; ++r) {
      mn = fminf(mn, xs[r][tid]);
      mx = fmaxf(mx, xs[r][tid]);
    }
    __half hs, hz;
    group_sz(mn, mx, hs, hz);
    sk[tid] = __half2float(hs);
    zk[tid] = __half2float(hz);
    ksz[tid] = pack_sz(hs, hz);
  }
  __syncthreads();
  reinterpret_cast<uint4*>(rec + (size_t)t * 128)[qq] =
      pack_quarter(xs, t, qq, [&](int, int ch) { return make_float2(sk[ch], zk[ch]); });
  __syncthreads();

  // values: one group per (token, 64-channel half)
  load_rows(a.v + in_off, xs, tid);
  __syncthreads();
  if (tid < 2 * kG) {
    const int tt = tid >> 1, hf = tid & 1;
    float mn = xs[tt][64 * hf], mx = mn;
    for (int ch = 1; ch < 64; ++ch) {
      mn = fminf(mn, xs[tt][64 * hf + ch]);
      mx = fmaxf(mx, xs[tt][64 * hf + ch]);
    }
    __half hs, hz;
    group_sz(mn, mx, hs, hz);
    sv[tt][hf] = __half2float(hs);
    zv[tt][hf] = __half2float(hz);
    vsz[tt * 2 + hf] = pack_sz(hs, hz);
  }
  __syncthreads();
  reinterpret_cast<uint4*>(rec + (size_t)t * 128 + 64)[qq] =
      pack_quarter(xs, t, qq, [&](int tt, int ch) { return make_float2(sv[tt][ch >> 6], zv[tt][ch >> 6]); });

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

__global__ void __launch_bounds__(256) encode_residual_kernel(EncodeResArgs a) {
  const int g = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
  const CacheView& c = a.c;
  const int cap = c.cap, ncb = cap / kG, T = c.total_slots, r = a.r;
  const int i0 = g * kG;
  const int nr = min(kG, a.n_rows - i0);
  __shared__ int tok[kG];
  __shared__ float xs[kG][129];
  __shared__ float sk[kD], zk[kD];
  __shared__ float sv[kG][2], zv[kG][2];

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
  const int t = tid >> 2, qq = tid & 3;
  const uint8_t* brec = arr<uint8_t>(c, A_BREC, a.layer) + (size_t)h * ncb * kRec;
  uint8_t* rrec = arr<uint8_t>(c, A_RREC, a.layer) + (size_t)h * (T / kG) * kRec;
  uint8_t* orec = rrec + (size_t)(gslot0 >> 6) * kRec;  // this CTA's output group record

  for (int part = 0; part < 2; ++part) {
    const bool is_v = part == 1;
    const uint16_t* src = is_v ? a.v : a.k;
    const int code_off = is_v ? 64 : 0;

    // residual E = X^(r) - X_hat^(r-1) for 8 channels per item
    for (int item = tid; item < kG * 16; item += 256) {
      const int tt = item >> 4, c8 = (item & 15) * 8;
      const int j = tok[tt];
      if (tt >= nr || j < 0) {
#pragma unroll
        for (int e = 0; e < 8; ++e) xs[tt][c8 + e] = 0.f;
        continue;
      }
      const size_t row = a.compact ? (size_t)(i0 + tt) : (size_t)(j - a.row0);
      const uint4 xw = ldg_u4(src + (size_t)h * a.head_stride + row * kD + c8);
      float x[8] = {bf16_lo(xw.x), bf16_hi(xw.x), bf16_lo(xw.y), bf16_hi(xw.y),
                    bf16_lo(xw.z), bf16_hi(xw.z), bf16_lo(xw.w), bf16_hi(xw.w)};
      const int b = j >> 6, jt = j & 63;
      float xh[8];
      {
        const uint8_t* g = brec + (size_t)b * kRec;
        const uint32_t cw = *reinterpret_cast<const uint32_t*>(g + (size_t)jt * 128 + code_off + c8 / 2);
        const uint32_t* ks = reinterpret_cast<const uint32_t*>(g + kRecKsz);
        const uint32_t* vs = reinterpret_cast<const uint32_t*>(g + kRecVsz);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const uint32_t szw = is_v ? vs[jt * 2 + (c8 >> 6)] : ks[c8 + e];
          xh[e] = deq((cw >> (4 * e)) & 15u, unpack_sz(szw));
        }
      }
      for (int rp = 2; rp < r; ++rp) {
        const unsigned long long mk = mask[(size_t)rp * ncb + b];
        const int gs = c.slot_base[rp] + first[(size_t)rp * ncb + b] +
                       __popcll(mk & ((1ull << jt) - 1ull));
        const uint8_t* g = rrec + (size_t)(gs >> 6) * kRec;
        const int rw = gs & 63;
        const uint32_t cw = *reinterpret_cast<const uint32_t*>(g + (size_t)rw * 128 + code_off + c8 / 2);
        const uint32_t* ks = reinterpret_cast<const uint32_t*>(g + kRecKsz);
        const uint32_t* vs = reinterpret_cast<const uint32_t*>(g + kRecVsz);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const uint32_t szw = is_v ? vs[rw * 2 + (c8 >> 6)] : ks[c8 + e];
          xh[e] = __fadd_rn(xh[e], deq((cw >> (4 * e)) & 15u, unpack_sz(szw)));
        }
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) xs[tt][c8 + e] = __fsub_rn(x[e], xh[e]);
    }
    __syncthreads();

    uint32_t* oks = reinterpret_cast<uint32_t*>(orec + kRecKsz);
    uint32_t* ovs = reinterpret_cast<uint32_t*>(orec + kRecVsz);
    if (!is_v) {
      if (tid < kD) {  // one group per (64 consecutive slots, channel), rows present only
        float mn = xs[0][tid], mx = mn;
        for (int rr = 1; rr < nr; ++rr) {
          mn = fminf(mn, xs[rr][tid]);
          mx = fmaxf(mx, xs[rr][tid]);
        }
        __half hs, hz;
        group_sz(mn, mx, hs, hz);
        sk[tid] = __half2float(hs);
        zk[tid] = __half2float(hz);
        oks[tid] = pack_sz(hs, hz);
      }
    } else if (tid < 2 * kG) {  // one group per (slot, half)
      const int tt = tid >> 1, hf = tid & 1;
      float sval = 0.f, zval = 0.f;
      uint32_t packed = 0u;
      if (tt < nr) {
        float mn = xs[tt][64 * hf], mx = mn;
        for (int ch = 1; ch < 64; ++ch) {
          mn = fminf(mn, xs[tt][64 * hf + ch]);
          mx = fmaxf(mx, xs[tt][64 * hf + ch]);
        }
        __half hs, hz;
        group_sz(mn, mx, hs, hz);
        sval = __half2float(hs);
        zval = __half2float(hz);
        packed = pack_sz(hs, hz);
      }
      sv[tt][hf] = sval;
      zv[tt][hf] = zval;
      ovs[tt * 2 + hf] = packed;
    }
    __syncthreads();
    uint4 w = make_uint4(0u, 0u, 0u, 0u);
    if (t < nr) {
      if (!is_v)
        w = pack_quarter(xs, t, qq, [&](int, int ch) { return make_float2(sk[ch], zk[ch]); });
      else
        w = pack_quarter(xs, t, qq, [&](int tt, int ch) { return make_float2(sv[tt][ch >> 6], zv[tt][ch >> 6]); });
    }
    reinterpret_cast<uint4*>(orec + (size_t)t * 128 + code_off)[qq] = w;
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
  encode_residual_kernel<<<grid, 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace fl
