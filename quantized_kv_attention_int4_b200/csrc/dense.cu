// Dense decode reader, direct-load form: single-query attention of one loop over every
// column.  The staged reader (dense_staged.cu) covers loops whose residual rows come from
// at most two stores; this form serves every other loop.
//
// FlashLoop project page, "The Method": dense loops attend over all columns; a
// column's key/value in loop r is the loop-1 base plus its residuals of loops 2..r
// (Step 03), or the loop's BF16 tail row (flashloop 0.1.0 PyPI description,
// "Configuration and supported scope": 64-token BF16 tail).
//
// Work split: grid (splits, heads); a CTA of 8 warps owns a contiguous range of
// 64-token blocks ("units", plus one unit for the tail).  A warp processes one unit
// at a time entirely on its own:
//   1. the block's key (scale, zero) record becomes 128 pre-scaled query weights
//      (qs'_c = 128 q_c s_c, one constant per group) in the warp's shared slice;
//   2. 8 coalesced 512-byte loads bring the 64 key rows; lane (row tr, quarter qq)
//      dots its 32 nibbles with 32 weights, a quad shuffle finishes each logit;
//   3. each residual loop's rows of the block (consecutive slots) add their logit
//      contribution through a slot->token map, one group's weights at a time;
//   4. online softmax (base-2, running max per warp);
//   5. the value rows (base, then residuals) are accumulated with per-token weights
//      128 p s and a per-half correction sum(p z - 128 p s).
// Warps merge in shared memory, CTAs write (M, L, o) partials, and the last CTA of
// each head (an atomic ticket, no waiting) combines them by log-sum-exp.
//
// Codec variants (flozi guide, section 4: the "Per-loop KIVI4" row and the 2-bit row
// of Figure 5): with 2-bit residual stores each row quarter is loaded as 8 bytes and
// widened to the 4-bit layout (codes 0..3), the arithmetic is unchanged; with
// full-state stores a token's loop-r key/value is its store min(r, depth) alone, so
// each store contributes only the rows of tokens whose last store it is, and their
// logits are assigned rather than added (the base is skipped when every token of the
// block has a later store).
#include "flush.cuh"
#include "kernels.h"

namespace fl {
namespace {

constexpr int kWarps = 8;

// kFlush: the step also writes this loop's store of a full tail (fused flush);
// kCodec: FL_CODEC_* of the loop r >= 2 stores
template <bool kFlush, int kCodec>
__global__ void __launch_bounds__(kWarps * 32, 2) dense_direct_kernel(ReaderArgs a) {
  using CT = CodecT<kCodec>;
  using RB = Rec<CT::kResBits>;
  const int h = blockIdx.y, split = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, qq = lane & 3, tr = lane >> 2;
  const CacheView& c = a.c;
  const int H = c.H, cap = c.cap, ncb = cap / kG, T = c.total_slots, r = a.r;

  const uint8_t* brec = arr<uint8_t>(c, A_BREC, a.layer) + (size_t)h * ncb * kRec;
  const uint8_t* rrec = arr<uint8_t>(c, A_RREC, a.layer) + (size_t)h * (T / kG) * RB::kBytes;
  // residual slot gs: row (gs & 63) of group record (gs >> 6)
  auto rrow = [&](int gs) { return rrec + (size_t)(gs >> 6) * RB::kBytes + (size_t)(gs & 63) * RB::kRow; };
  // quarter qq of a residual row's key / value codes in the 4-bit layout
  auto res_key = [&](const uint8_t* row) -> uint4 {
    if constexpr (CT::kResBits == 4) return __ldg(reinterpret_cast<const uint4*>(row) + qq);
    else return int2_to_nib(__ldg(reinterpret_cast<const uint2*>(row) + qq));
  };
  auto res_val = [&](const uint8_t* row) -> uint4 {
    if constexpr (CT::kResBits == 4) return __ldg(reinterpret_cast<const uint4*>(row + RB::kHalf) + qq);
    else return int2_to_nib(__ldg(reinterpret_cast<const uint2*>(row + RB::kHalf) + qq));
  };
  const unsigned long long* mask = arr<unsigned long long>(c, A_MASK, a.layer);
  const int32_t* first = arr<int32_t>(c, A_FIRST, a.layer);
  uint16_t* tail_k = arr<uint16_t>(c, A_TAILK, a.layer) + ((size_t)(r - 1) * H + h) * kTail * kD;
  uint16_t* tail_v = arr<uint16_t>(c, A_TAILV, a.layer) + ((size_t)(r - 1) * H + h) * kTail * kD;
  float* score = arr<float>(c, A_SCORE, a.layer) + (size_t)h * cap;
  uint8_t* tag = arr<uint8_t>(c, A_TAG, a.layer) + (size_t)h * cap;

  __shared__ __align__(16) float q_s[kD];
  __shared__ __align__(16) float qs_w[kWarps][kD];
  __shared__ float lg_w[kWarps][kG];
  __shared__ uint8_t tok_w[kWarps][kG];
  __shared__ float m_w[kWarps], l_w[kWarps];
  __shared__ __align__(16) float o_w[kWarps][kD];
  __shared__ int last_cta;

  if (tid < kD) q_s[tid] = __uint_as_float((uint32_t)a.q[(size_t)h * kD + tid] << 16) * kQScale;
  __syncthreads();

  const int nb = a.n_q / kG;
  const int n_units = nb + 1;
  const int u0 = (int)((long long)split * n_units / a.n_splits);
  const int u1 = (int)((long long)(split + 1) * n_units / a.n_splits);
  const bool has_new = a.k_new != nullptr;

  float acc[32];
#pragma unroll
  for (int k = 0; k < 32; ++k) acc[k] = 0.f;
  float corr = 0.f, M = -INFINITY, Ls = 0.f;
  float* qsw = qs_w[warp];
  float* lgw = lg_w[warp];
  uint8_t* tokw = tok_w[warp];

  for (int u = u0 + warp; u < u1; u += kWarps) {
    float qsr[32];
    if (u < nb) {
      const int b = u;
      // full-state stores: tokens whose key/value is the base (no store of loops 2..r)
      const unsigned long long need_b = (CT::kFullState && r >= 2) ? ~mask[(size_t)2 * ncb + b] : ~0ull;
      // ---- keys: base ----
      if (need_b) {
        __syncwarp();
        const uint8_t* rec = brec + (size_t)b * kRec;
        float cb = group_weights(reinterpret_cast<const uint32_t*>(rec + kRecKsz), q_s, qsw, lane);
        __syncwarp();
        load32(qsw + 32 * qq, qsr);
        const uint4* kc = reinterpret_cast<const uint4*>(rec);
        uint4 w[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = __ldg(kc + (8 * i + tr) * 8 + qq);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float p = dot32(w[i], qsr);
          p += __shfl_xor_sync(kFull, p, 1);
          p += __shfl_xor_sync(kFull, p, 2);
          if (qq == 0) lgw[8 * i + tr] = p + cb;
        }
      }
      // ---- keys: stores of loops 2..r ----
      for (int rp = 2; rp <= r; ++rp) {
        const unsigned long long mk = mask[(size_t)rp * ncb + b];
        // full-state: only the tokens whose last store in loop r is this one
        const unsigned long long need =
            CT::kFullState && rp < r ? mk & ~mask[(size_t)(rp + 1) * ncb + b] : mk;
        if (need == 0ull) continue;
        const int na = __popcll(mk);
        const int gs0 = c.slot_base[rp] + first[(size_t)rp * ncb + b];
        __syncwarp();
        for (int tt = lane; tt < kG; tt += 32)
          if ((mk >> tt) & 1ull) tokw[__popcll(mk & ((1ull << tt) - 1ull))] = (uint8_t)tt;
        __syncwarp();
        int row = 0;
        while (row < na) {  // the block's rows of one group record at a time (at most two)
          const int grp = (gs0 + row) >> 6;
          const int row_end = min(na, ((grp + 1) << 6) - gs0);
          // rows of the piece in flight four passes (32 rows) at a time; the first four are
          // issued before the weights are built
          constexpr int kB = 4;
          uint4 x[kB];
          auto issue = [&](int r0) {
#pragma unroll
            for (int i = 0; i < kB; ++i) {
              const int rw = r0 + 8 * i + tr;
              const bool act = rw < row_end && (!CT::kFullState || ((need >> tokw[rw]) & 1ull));
              x[i] = act ? res_key(rrow(gs0 + rw)) : make_uint4(0u, 0u, 0u, 0u);
            }
          };
          issue(row);
          const float cg = group_weights(
              reinterpret_cast<const uint32_t*>(rrec + (size_t)grp * RB::kBytes + RB::kKsz), q_s, qsw, lane);
          __syncwarp();
          load32(qsw + 32 * qq, qsr);
          for (int r0 = row; r0 < row_end; r0 += 8 * kB) {
            if (r0 != row) issue(r0);
#pragma unroll
            for (int i = 0; i < kB; ++i) {
              if (r0 + 8 * i >= row_end) break;
              const int rw = r0 + 8 * i + tr;
              const bool act = rw < row_end && (!CT::kFullState || ((need >> tokw[rw]) & 1ull));
              float p = dot32(x[i], qsr);
              p += __shfl_xor_sync(kFull, p, 1);
              p += __shfl_xor_sync(kFull, p, 2);
              if (act && qq == 0) {
                if constexpr (CT::kFullState) lgw[tokw[rw]] = p + cg;
                else lgw[tokw[rw]] += p + cg;
              }
            }
          }
          row = row_end;
          __syncwarp();  // the piece's weights are used up before the next piece's are built
        }
      }
      __syncwarp();
      // ---- online softmax over the block ----
      const float l0 = lgw[lane], l1 = lgw[lane + 32];
      if (a.keep) {
        score[(size_t)b * kG + lane] = l0;
        score[(size_t)b * kG + lane + 32] = l1;
        tag[(size_t)b * kG + lane] = (uint8_t)r;
        tag[(size_t)b * kG + lane + 32] = (uint8_t)r;
      }
      const float mb = warp_max(fmaxf(l0, l1));
      if (mb > M) {
        const float al = ex2(M - mb);
#pragma unroll
        for (int k = 0; k < 32; ++k) acc[k] *= al;
        corr *= al;
        Ls *= al;
        M = mb;
      }
      const float p0 = ex2(l0 - M), p1 = ex2(l1 - M);
      Ls += p0 + p1;
      __syncwarp();
      lgw[lane] = p0;
      lgw[lane + 32] = p1;
      __syncwarp();
      // ---- values: base ----
      if (need_b) {
        const uint8_t* rec = brec + (size_t)b * kRec;
        const uint4* vc = reinterpret_cast<const uint4*>(rec);
        const uint32_t* vs = reinterpret_cast<const uint32_t*>(rec + kRecVsz);
        uint4 vw[8];
        uint32_t sw[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          vw[i] = __ldg(vc + (8 * i + tr) * 8 + 4 + qq);
          sw[i] = __ldg(vs + 2 * (8 * i + tr) + (qq >> 1));
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float p = ((need_b >> (8 * i + tr)) & 1ull) ? lgw[8 * i + tr] : 0.f;
          const float2 sz = unpack_sz(sw[i]);
          const float P = 128.f * (p * sz.x);
          corr += fmaf(p, sz.y, -P);
          axpy32(vw[i], P, acc);
        }
      }
      // ---- values: stores of loops 2..r ----
      for (int rp = 2; rp <= r; ++rp) {
        const unsigned long long mk = mask[(size_t)rp * ncb + b];
        const unsigned long long need =
            CT::kFullState && rp < r ? mk & ~mask[(size_t)(rp + 1) * ncb + b] : mk;
        if (need == 0ull) continue;
        const int na = __popcll(mk);
        const int gs0 = c.slot_base[rp] + first[(size_t)rp * ncb + b];
        __syncwarp();
        for (int tt = lane; tt < kG; tt += 32)
          if ((mk >> tt) & 1ull) tokw[__popcll(mk & ((1ull << tt) - 1ull))] = (uint8_t)tt;
        __syncwarp();
        // all of the store's rows of the block (at most 64, 8 a pass) in flight together
        uint4 x[8];
        uint32_t sw[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int rw = 8 * i + tr;
          const bool act = rw < na && (!CT::kFullState || ((need >> tokw[rw]) & 1ull));
          const int gs = gs0 + rw;
          x[i] = act ? res_val(rrow(gs)) : make_uint4(0u, 0u, 0u, 0u);
          sw[i] = act ? __ldg(reinterpret_cast<const uint32_t*>(rrec + (size_t)(gs >> 6) * RB::kBytes + RB::kVsz) +
                              (gs & 63) * 2 + (qq >> 1))
                      : 0u;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int rw = 8 * i + tr;
          if (8 * i >= na) break;
          if (rw < na && (!CT::kFullState || ((need >> tokw[rw]) & 1ull))) {
            const float2 sz = unpack_sz(sw[i]);
            const float p = lgw[tokw[rw]];
            const float P = 128.f * (p * sz.x);
            corr += fmaf(p, sz.y, -P);
            axpy32(x[i], P, acc);
          }
        }
      }
    } else {
      // ---- BF16 tail unit: rows [0, n_tail) of this loop; row n_tail-1 may be new ----
      const int nt = a.n_tail;
      if (has_new) {
        __syncwarp();
        const uint2* kn = reinterpret_cast<const uint2*>(a.k_new + (size_t)h * kD);
        const uint2* vn = reinterpret_cast<const uint2*>(a.v_new + (size_t)h * kD);
        reinterpret_cast<uint2*>(tail_k + (size_t)(nt - 1) * kD)[lane] = kn[lane];
        reinterpret_cast<uint2*>(tail_v + (size_t)(nt - 1) * kD)[lane] = vn[lane];
      }
      load32(q_s + 32 * qq, qsr);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int t = 8 * i + tr;
        const bool act = t < nt;
        float p = 0.f;
        if (act) {
          const uint16_t* row = (has_new && t == nt - 1) ? a.k_new + (size_t)h * kD : tail_k + (size_t)t * kD;
          p = dot_bf16_32(row + 32 * qq, qsr);
        }
        p += __shfl_xor_sync(kFull, p, 1);
        p += __shfl_xor_sync(kFull, p, 2);
        if (qq == 0) lgw[t] = act ? p : -INFINITY;
      }
      __syncwarp();
      const float l0 = lgw[lane], l1 = lgw[lane + 32];
      if (a.keep) {
        if (lane < nt) {
          score[(size_t)a.n_q + lane] = l0;
          tag[(size_t)a.n_q + lane] = (uint8_t)r;
        }
        if (lane + 32 < nt) {
          score[(size_t)a.n_q + lane + 32] = l1;
          tag[(size_t)a.n_q + lane + 32] = (uint8_t)r;
        }
      }
      const float mb = warp_max(fmaxf(l0, l1));
      if (mb > M) {
        const float al = ex2(M - mb);
#pragma unroll
        for (int k = 0; k < 32; ++k) acc[k] *= al;
        corr *= al;
        Ls *= al;
        M = mb;
      }
      const float p0 = ex2(l0 - M), p1 = ex2(l1 - M);
      Ls += p0 + p1;
      __syncwarp();
      lgw[lane] = p0;
      lgw[lane + 32] = p1;
      __syncwarp();
      for (int i = 0; i < 8; ++i) {
        const int t = 8 * i + tr;
        if (t < nt) {
          const uint16_t* row = (has_new && t == nt - 1) ? a.v_new + (size_t)h * kD : tail_v + (size_t)t * kD;
          axpy_bf16_32(row + 32 * qq, lgw[t], acc);
        }
      }
    }
  }

  // ---- warp reduction: lanes sharing a channel quarter ----
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    acc[k] += __shfl_xor_sync(kFull, acc[k], 4);
    acc[k] += __shfl_xor_sync(kFull, acc[k], 8);
    acc[k] += __shfl_xor_sync(kFull, acc[k], 16);
  }
  corr += __shfl_xor_sync(kFull, corr, 4);
  corr += __shfl_xor_sync(kFull, corr, 8);
  corr += __shfl_xor_sync(kFull, corr, 16);
  Ls = warp_sum(Ls);
  if (tr == 0) {
#pragma unroll
    for (int k = 0; k < 32; ++k) o_w[warp][32 * qq + k] = acc[k] + corr;
  }
  if (lane == 0) {
    m_w[warp] = M;
    l_w[warp] = Ls;
  }
  __syncthreads();

  // ---- CTA partial (M, L, o) ----
  float* part = a.part + ((size_t)h * a.n_splits + split) * kPartStride;
  if (tid < kD) {
    float Mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) Mx = fmaxf(Mx, m_w[w]);
    float Lt = 0.f, ot = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      if (m_w[w] != -INFINITY) {
        const float e = ex2(m_w[w] - Mx);
        Lt = fmaf(l_w[w], e, Lt);
        ot = fmaf(o_w[w][tid], e, ot);
      }
    }
    part[4 + tid] = ot;
    if (tid == 0) {
      part[0] = Mx;
      part[1] = Lt;
    }
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) last_cta = (atomicAdd(&a.counter[h], 1) == a.n_splits - 1);
  __syncthreads();
  if (last_cta) __threadfence();

  // ---- last CTA of this head: log-sum-exp combine of every split ----
  if (last_cta && tid < kD) {
    const float* hp = a.part + (size_t)h * a.n_splits * kPartStride;
    float Mx = -INFINITY;
    for (int s = 0; s < a.n_splits; ++s) Mx = fmaxf(Mx, __ldcg(hp + (size_t)s * kPartStride));
    float Lt = 0.f, ot = 0.f;
    for (int s = 0; s < a.n_splits; ++s) {
      const float ms = __ldcg(hp + (size_t)s * kPartStride);
      if (ms == -INFINITY) continue;
      const float e = ex2(ms - Mx);
      Lt = fmaf(__ldcg(hp + (size_t)s * kPartStride + 1), e, Lt);
      ot = fmaf(__ldcg(hp + (size_t)s * kPartStride + 4 + tid), e, ot);
    }
    a.o[(size_t)h * kD + tid] = ot / Lt;
    if (tid == 0) {
      arr<float>(c, A_OFFSET, a.layer)[(size_t)h * kOffStride + r] = Mx + log2f(Lt);
      a.counter[h] = 0;
    }
  }
  if constexpr (kFlush) {  // dynamic shared memory holds the encoder's staging (launched with it)
    extern __shared__ __align__(16) uint8_t flush_smem[];
    flush_tail(a, blockIdx.y * gridDim.x + blockIdx.x, gridDim.x * gridDim.y,
               *reinterpret_cast<EncodeSmem*>(flush_smem), tid, kWarps * 32);
  }
}

}  // namespace

int dense_splits(int heads, int n_q) {
  const int n_units = n_q / kG + 1;
  int by_work = (n_units + 2 * kWarps - 1) / (2 * kWarps);  // >= ~2 units per warp
  int by_sms = (148 * 2) / heads;                            // one wave at 2 CTAs per SM
  int s = by_work < by_sms ? by_work : by_sms;
  if (s < 1) s = 1;
  if (s > n_units) s = n_units;
  if (s > kMaxSplits) s = kMaxSplits;
  return s;
}

cudaError_t launch_dense_direct(ReaderArgs a, cudaStream_t s) {
  a.n_splits = dense_splits(a.c.H, a.n_q);
  dim3 grid(a.n_splits, a.c.H);
  if (a.c.codec == FL_CODEC_FULL_INT4)
    dense_direct_kernel<false, FL_CODEC_FULL_INT4><<<grid, kWarps * 32, 0, s>>>(a);
  else if (a.c.codec == FL_CODEC_RESIDUAL_INT2)
    dense_direct_kernel<false, FL_CODEC_RESIDUAL_INT2><<<grid, kWarps * 32, 0, s>>>(a);
  else if (a.flush)
    dense_direct_kernel<true, FL_CODEC_RESIDUAL_INT4><<<grid, kWarps * 32, sizeof(EncodeSmem), s>>>(a);
  else
    dense_direct_kernel<false, FL_CODEC_RESIDUAL_INT4><<<grid, kWarps * 32, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace fl
