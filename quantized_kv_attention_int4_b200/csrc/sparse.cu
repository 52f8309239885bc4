// Sparse decode reader: loop-aware sparse attention over the selected columns S.
//
// FlashLoop project page, "The Method", Step 02: a sparse loop recomputes attention
// only for the columns chosen from the preceding loop and keeps their global
// probability mass m; flozi guide "FlashLoop: store changes between repeated passes",
// section 3: the loop's output is a rank-K correction of the previous one.  With u the
// unselected columns' cached contribution:
//     o_r = u + m * softmax_S(q_r K_S^T / sqrt(d)) V_S.
//
// Work split: grid (splits, heads), 4 warps per CTA, each warp a contiguous run of S
// (ascending column ids).  A warp takes up to 8 columns of one 64-token block per
// iteration: the block's key (scale, zero) record becomes pre-scaled query weights
// once for all of them (shared memory), each column's residual rows of loops
// 2..min(r, depth) are gathered by slot (first_slot + popcount of the block mask),
// and the residual store's key groups touched by the block (at most two) are
// prepared the same way.  Tail columns read BF16 rows.  Online softmax per warp,
// shared-memory merge per CTA, (M, L, o) partials, and the last CTA of each head
// combines them and applies u and m.  The same pass splices the selector state:
// score/tag of every j in S become loop r's and offset[r] = M + log2 L - log2 m.
#include "kernels.h"

namespace fl {
namespace {

constexpr int kWarps = 4;

__global__ void __launch_bounds__(kWarps * 32) sparse_kernel(ReaderArgs a) {
  const int h = blockIdx.y, split = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, qq = lane & 3, tr = lane >> 2;
  const CacheView& c = a.c;
  const int H = c.H, cap = c.cap, ncb = cap / kG, T = c.total_slots, r = a.r;
  const int n_q = a.n_q, N = a.n_q + a.n_tail, K = a.k_sel;

  const uint8_t* kcode = arr<uint8_t>(c, A_KCODE, a.layer) + (size_t)h * cap * 64;
  const uint8_t* vcode = arr<uint8_t>(c, A_VCODE, a.layer) + (size_t)h * cap * 64;
  const uint32_t* ksz = arr<uint32_t>(c, A_KSZ, a.layer) + (size_t)h * ncb * kD;
  const uint32_t* vsz = arr<uint32_t>(c, A_VSZ, a.layer) + (size_t)h * cap * 2;
  const uint8_t* rkcode = arr<uint8_t>(c, A_RKCODE, a.layer) + (size_t)h * T * 64;
  const uint8_t* rvcode = arr<uint8_t>(c, A_RVCODE, a.layer) + (size_t)h * T * 64;
  const uint32_t* rksz = arr<uint32_t>(c, A_RKSZ, a.layer) + (size_t)h * (T / kG) * kD;
  const uint32_t* rvsz = arr<uint32_t>(c, A_RVSZ, a.layer) + (size_t)h * T * 2;
  const unsigned long long* mask = arr<unsigned long long>(c, A_MASK, a.layer);
  const int32_t* first = arr<int32_t>(c, A_FIRST, a.layer);
  const uint8_t* depth = arr<uint8_t>(c, A_DEPTH, a.layer);
  uint16_t* tail_k = arr<uint16_t>(c, A_TAILK, a.layer) + ((size_t)(r - 1) * H + h) * kTail * kD;
  uint16_t* tail_v = arr<uint16_t>(c, A_TAILV, a.layer) + ((size_t)(r - 1) * H + h) * kTail * kD;
  float* score = arr<float>(c, A_SCORE, a.layer) + (size_t)h * cap;
  uint8_t* tag = arr<uint8_t>(c, A_TAG, a.layer) + (size_t)h * cap;
  const int32_t* sel = arr<int32_t>(c, A_SEL, a.layer) + (size_t)h * c.max_select;

  __shared__ __align__(16) float q_s[kD];
  __shared__ __align__(16) float qa_w[kWarps][kD];
  __shared__ __align__(16) float qb_w[kWarps][kD];
  __shared__ float m_w[kWarps], l_w[kWarps];
  __shared__ __align__(16) float o_w[kWarps][kD];
  __shared__ int last_cta;

  const bool has_new = a.k_new != nullptr;
  if (tid < kD) q_s[tid] = __uint_as_float((uint32_t)a.q[(size_t)h * kD + tid] << 16) * kQScale;
  if (split == 0 && has_new && warp == 0) {
    const uint2* kn = reinterpret_cast<const uint2*>(a.k_new + (size_t)h * kD);
    const uint2* vn = reinterpret_cast<const uint2*>(a.v_new + (size_t)h * kD);
    reinterpret_cast<uint2*>(tail_k + (size_t)(a.n_tail - 1) * kD)[lane] = kn[lane];
    reinterpret_cast<uint2*>(tail_v + (size_t)(a.n_tail - 1) * kD)[lane] = vn[lane];
  }
  __syncthreads();

  const int k0 = (int)((long long)split * K / a.n_splits);
  const int k1 = (int)((long long)(split + 1) * K / a.n_splits);
  const int wk0 = k0 + (int)((long long)warp * (k1 - k0) / kWarps);
  const int wk1 = k0 + (int)((long long)(warp + 1) * (k1 - k0) / kWarps);

  float acc[32];
#pragma unroll
  for (int k = 0; k < 32; ++k) acc[k] = 0.f;
  float corr = 0.f, M = -INFINITY, Ls = 0.f;
  float* qa = qa_w[warp];
  float* qb = qb_w[warp];

  // Running-max update; returns the column's weight exp2(logit - M).
  auto softmax_step = [&](bool act, float logit) -> float {
    const float lg = act ? logit : -INFINITY;
    const float mb = warp_max(lg);
    if (mb > M) {
      const float al = ex2(M - mb);
#pragma unroll
      for (int k = 0; k < 32; ++k) acc[k] *= al;
      corr *= al;
      Ls *= al;
      M = mb;
    }
    const float p = act ? ex2(lg - M) : 0.f;
    if (qq == 0) Ls += p;
    return p;
  };

  int kk = wk0;
  while (kk < wk1) {
    const int idx = kk + tr;
    const bool inr = idx < wk1;
    const int j = inr ? sel[idx] : -1;
    const bool valid = inr && j >= 0 && j < N;
    if (inr && !valid && qq == 0) record_error(c.status, FL_DEV_SEL_RANGE, j);
    const int j0 = __shfl_sync(kFull, j, 0);
    float qsr[32];

    if (j0 >= 0 && j0 < n_q) {
      // ---------------- quantised columns of block b ----------------
      const int b = j0 >> 6;
      const bool same = valid && j < n_q && (j >> 6) == b;
      const unsigned bal = __ballot_sync(kFull, same && qq == 0);
      unsigned run = 0;
#pragma unroll
      for (int t = 0; t < 8; ++t) run |= ((bal >> (4 * t)) & 1u) << t;
      const int take = __ffs(~run) - 1;  // leading columns of this block (>= 1)
      const bool act = tr < take;

      __syncwarp();
      const float cb = group_weights(ksz + (size_t)b * kD, q_s, qa, lane);
      __syncwarp();
      load32(qa + 32 * qq, qsr);
      float part = 0.f, bias = cb;
      if (act) part = dot32(__ldg(reinterpret_cast<const uint4*>(kcode + (size_t)j * 64) + qq), qsr);
      const int dep = act ? (int)depth[j] : 0;
      const int jt = j & 63;
      for (int rp = 2; rp <= r; ++rp) {
        const bool need = act && rp <= dep;
        if (!__any_sync(kFull, need)) break;
        const unsigned long long mk = mask[(size_t)rp * ncb + b];
        const int gsf = c.slot_base[rp] + first[(size_t)rp * ncb + b];
        const int ga = gsf >> 6, gb = (gsf + __popcll(mk) - 1) >> 6;
        __syncwarp();
        const float ca = group_weights(rksz + (size_t)ga * kD, q_s, qa, lane);
        float cbb = 0.f;
        if (gb != ga) cbb = group_weights(rksz + (size_t)gb * kD, q_s, qb, lane);
        __syncwarp();
        if (need) {
          const int gs = gsf + __popcll(mk & ((1ull << jt) - 1ull));
          const bool in_a = (gs >> 6) == ga;
          load32((in_a ? qa : qb) + 32 * qq, qsr);
          part += dot32(__ldg(reinterpret_cast<const uint4*>(rkcode + (size_t)gs * 64) + qq), qsr);
          bias += in_a ? ca : cbb;
        }
      }
      part += __shfl_xor_sync(kFull, part, 1);
      part += __shfl_xor_sync(kFull, part, 2);
      const float logit = part + bias;
      const float p = softmax_step(act, logit);
      if (act && qq == 0) {
        score[j] = logit;
        tag[j] = (uint8_t)r;
      }
      if (act) {
        {
          const uint4 x = __ldg(reinterpret_cast<const uint4*>(vcode + (size_t)j * 64) + qq);
          const float2 sz = unpack_sz(__ldg(vsz + (size_t)j * 2 + (qq >> 1)));
          const float P = 128.f * (p * sz.x);
          corr += fmaf(p, sz.y, -P);
          axpy32(x, P, acc);
        }
        const int top = dep < r ? dep : r;
        for (int rp = 2; rp <= top; ++rp) {
          const unsigned long long mk = mask[(size_t)rp * ncb + b];
          const int gs = c.slot_base[rp] + first[(size_t)rp * ncb + b] + __popcll(mk & ((1ull << jt) - 1ull));
          const uint4 x = __ldg(reinterpret_cast<const uint4*>(rvcode + (size_t)gs * 64) + qq);
          const float2 sz = unpack_sz(__ldg(rvsz + (size_t)gs * 2 + (qq >> 1)));
          const float P = 128.f * (p * sz.x);
          corr += fmaf(p, sz.y, -P);
          axpy32(x, P, acc);
        }
      }
      kk += take;
    } else if (j0 >= n_q && j0 < N) {
      // ---------------- BF16 tail columns ----------------
      const unsigned bal = __ballot_sync(kFull, valid && j >= n_q && qq == 0);
      unsigned run = 0;
#pragma unroll
      for (int t = 0; t < 8; ++t) run |= ((bal >> (4 * t)) & 1u) << t;
      const int take = __ffs(~run) - 1;  // leading tail columns (>= 1)
      const bool act = tr < take;
      load32(q_s + 32 * qq, qsr);
      float part = 0.f;
      const bool is_new = has_new && j == N - 1;
      if (act) {
        const uint16_t* row = is_new ? a.k_new + (size_t)h * kD : tail_k + (size_t)(j - n_q) * kD;
        part = dot_bf16_32(row + 32 * qq, qsr);
      }
      part += __shfl_xor_sync(kFull, part, 1);
      part += __shfl_xor_sync(kFull, part, 2);
      const float p = softmax_step(act, part);
      if (act) {
        if (qq == 0) {
          score[j] = part;
          tag[j] = (uint8_t)r;
        }
        const uint16_t* row = is_new ? a.v_new + (size_t)h * kD : tail_v + (size_t)(j - n_q) * kD;
        axpy_bf16_32(row + 32 * qq, p, acc);
      }
      kk += take;
    } else {
      kk += 1;  // an invalid entry (recorded above): skip it
    }
  }

  // ---- warp and CTA reduction (as in the dense reader) ----
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
  if (!last_cta) return;
  __threadfence();

  if (tid < kD) {
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
    const float m = arr<float>(c, A_MASS, a.layer)[h];
    const float u = arr<float>(c, A_UNSEL, a.layer)[(size_t)h * kD + tid];
    a.o[(size_t)h * kD + tid] = fmaf(m, ot / Lt, u);
    if (tid == 0) {
      arr<float>(c, A_OFFSET, a.layer)[(size_t)h * kOffStride + r] = Mx + log2f(Lt) - log2f(m);
      a.counter[h] = 0;
    }
  }
}

}  // namespace

int sparse_splits(int heads, int k_sel) {
  int by_work = (k_sel + 16 * kWarps - 1) / (16 * kWarps);  // >= ~16 columns per warp
  int by_sms = (148 * 4) / heads;                            // one wave at 4 CTAs per SM
  int s = by_work < by_sms ? by_work : by_sms;
  if (s < 1) s = 1;
  if (s > kMaxSplits) s = kMaxSplits;
  return s;
}

cudaError_t launch_sparse(ReaderArgs a, cudaStream_t s) {
  a.n_splits = sparse_splits(a.c.H, a.k_sel);
  dim3 grid(a.n_splits, a.c.H);
  sparse_kernel<<<grid, kWarps * 32, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace fl
