// Column selector for sparse loops: top-K of the preceding loop's distribution, the
// selected mass m, and the gather plan the sparse reader follows.
//
// FlashLoop project page, "The Method", Step 02: the preceding loop identifies the
// columns to recompute, and their global probability mass under the preceding loop's
// full distribution is cached so the sparse softmax is not renormalised to 1.
// flozi guide "FlashLoop: store changes between repeated passes", section 3: each
// sparse loop ranks key columns by the previous loop's attention statistics.
//
// One CTA (1024 threads) per (layer, head), launched for a range of layers at once.
//   keys:     log2 p~_j = score_j - offset[tag_j], mapped to an order-preserving u32
//             and kept in shared memory (N <= FL_MAX_SELECT_COLS);
//   select:   radix select of the K-th largest key over the bits where the keys
//             differ (the prefix every key shares is skipped), digits of up to 13
//             bits, each pass a shared-memory histogram over the keys that still match
//             the prefix and a block-wide scan from the top bin;
//   compact:  keys above the threshold plus the lowest-index ties, written in index
//             order (per-warp ballots and a block prefix), so S is ascending;
//   m, plan:  m = sum_S p~_j; for every j in S its tag, p~_j, the number of stores it
//             has in loop r (min(r, depth_j); 0 for a BF16 tail column) and its slot in
//             each residual store (block first slot + popcount of the block mask), so the
//             sparse reader can issue all of a column's loads at once.
#include "kernels.h"

namespace fl {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarpsSel = kThreads / 32;
constexpr int kDynMax = 194 * 1024;  // dynamic shared memory: keys [, selected columns]

// Selected columns are kept in shared memory after the keys when both fit.
__host__ __device__ inline bool sel_fits(int N, int K) {
  return ((size_t)((N + 3) & ~3) + (size_t)K) * sizeof(uint32_t) <= (size_t)kDynMax;
}

__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t o) {
  return __uint_as_float((o & 0x80000000u) ? (o & 0x7fffffffu) : ~o);
}

// Inclusive block scan of one value per thread (1024 threads).
__device__ __forceinline__ uint32_t block_scan(uint32_t v, uint32_t* wtot, int lane, int warp) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t n = __shfl_up_sync(kFull, v, o);
    if (lane >= o) v += n;
  }
  __syncthreads();
  if (lane == 31) wtot[warp] = v;
  __syncthreads();
  if (warp == 0) {
    uint32_t t = wtot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t n = __shfl_up_sync(kFull, t, o);
      if (lane >= o) t += n;
    }
    wtot[lane] = t;
  }
  __syncthreads();
  return v + (warp > 0 ? wtot[warp - 1] : 0u);
}

__global__ void __launch_bounds__(kThreads, 1) select_kernel(SelectArgs a) {
  extern __shared__ uint32_t keys[];  // [N] keys, then [K] selected columns when they fit
  const bool sel_smem = sel_fits(a.n_q + a.n_tail, a.k_sel);
  int32_t* sel_s = reinterpret_cast<int32_t*>(keys + ((a.n_q + a.n_tail + 3) & ~3));
  __shared__ __align__(16) uint32_t hist[8192];
  __shared__ float offs[kOffStride];
  __shared__ uint32_t wtot[32];
  __shared__ uint32_t sh_digit, sh_krem;
  __shared__ float red[32];

  const int h = blockIdx.x, layer = a.layer0 + blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const CacheView& c = a.c;
  const int cap = c.cap, ncb = cap / kG, R = c.R;
  const int n_q = a.n_q, N = a.n_q + a.n_tail, K = a.k_sel;

  const float* score = arr<float>(c, A_SCORE, layer) + (size_t)h * cap;
  const uint8_t* tag = arr<uint8_t>(c, A_TAG, layer) + (size_t)h * cap;
  int32_t* sel = arr<int32_t>(c, A_SEL, layer) + (size_t)h * c.max_select;

  if (tid < kOffStride) offs[tid] = arr<float>(c, A_OFFSET, layer)[(size_t)h * kOffStride + tid];
  __syncthreads();
  // keys, four columns per thread per step (score rows are 16-byte and tag rows 4-byte
  // aligned: cap is a multiple of 64); loads of several steps are in flight together
  auto key_of = [&](float sc, int t, int j) {
    if (t < 1 || t > R) {
      record_error(c.status, FL_DEV_TAG_RANGE, j);
      t = t < 1 ? 1 : R;
    }
    return order_key(sc - offs[t]);
  };
  const int N4 = N & ~3;
  uint32_t kand = 0xffffffffu, kor = 0u;  // bits common to every key
#pragma unroll 4
  for (int j = 4 * tid; j < N4; j += 4 * kThreads) {
    const float4 sc = *reinterpret_cast<const float4*>(score + j);
    const uint32_t tg = *reinterpret_cast<const uint32_t*>(tag + j);
    const uint32_t k0 = key_of(sc.x, (int)(tg & 0xff), j), k1 = key_of(sc.y, (int)((tg >> 8) & 0xff), j + 1);
    const uint32_t k2 = key_of(sc.z, (int)((tg >> 16) & 0xff), j + 2), k3 = key_of(sc.w, (int)(tg >> 24), j + 3);
    keys[j] = k0;
    keys[j + 1] = k1;
    keys[j + 2] = k2;
    keys[j + 3] = k3;
    kand &= k0 & k1 & k2 & k3;
    kor |= k0 | k1 | k2 | k3;
  }
  for (int j = N4 + tid; j < N; j += kThreads) {
    const uint32_t k = key_of(score[j], tag[j], j);
    keys[j] = k;
    kand &= k;
    kor |= k;
  }
  kand = __reduce_and_sync(kFull, kand);
  kor = __reduce_or_sync(kFull, kor);
  if (lane == 0) {
    hist[warp] = kand;
    hist[32 + warp] = kor;
  }
  __syncthreads();
  if (warp == 0) {
    kand = __reduce_and_sync(kFull, hist[lane]);
    kor = __reduce_or_sync(kFull, hist[32 + lane]);
    if (lane == 0) {
      hist[64] = kand;
      hist[65] = kor;
    }
  }
  __syncthreads();
  kand = hist[64];
  kor = hist[65];
  __syncthreads();

  // ---- radix select of the K-th largest key, over the bits where keys differ ----
  const uint32_t diff = kand ^ kor;
  int nbits = diff ? 32 - __clz(diff) : 0;  // digits cover bits [0, nbits)
  uint32_t pmask = nbits >= 32 ? 0u : ~((1u << nbits) - 1u);
  uint32_t prefix = kand & pmask, krem = (uint32_t)K;
  while (nbits > 0) {
    // up to 13-bit digits; two balanced passes whenever the keys differ in <= 26 bits
    const int wbits = nbits > 26 ? 13 : (nbits > 13 ? (nbits + 1) / 2 : nbits);
    const int shift = nbits - wbits;
    nbits = shift;
    const int nbins = 1 << wbits;
    const uint32_t dmask = (uint32_t)nbins - 1u;
    for (int i = tid; i < nbins; i += kThreads) hist[i] = 0u;
    __syncthreads();
    for (int j = tid; j < N; j += kThreads) {
      const uint32_t u = keys[j];
      if ((u & pmask) == prefix) atomicAdd(&hist[(u >> shift) & dmask], 1u);
    }
    __syncthreads();
    // thread t owns bins [nbins - per*(t+1), nbins - per*t), i.e. descending order
    const int per = nbins / kThreads > 0 ? nbins / kThreads : 1;
    const int owners = nbins / per;
    uint32_t local = 0u;
    if (tid < owners)
      for (int i = 0; i < per; ++i) local += hist[nbins - per * tid - 1 - i];
    const uint32_t incl = block_scan(local, wtot, lane, warp);
    const uint32_t excl = incl - local;
    if (tid < owners && excl < krem && krem <= incl) {
      uint32_t cum = excl;
      for (int i = 0; i < per; ++i) {
        const int bin = nbins - per * tid - 1 - i;
        if (cum + hist[bin] >= krem) {
          sh_digit = (uint32_t)bin;
          sh_krem = krem - cum;
          break;
        }
        cum += hist[bin];
      }
    }
    __syncthreads();
    prefix |= sh_digit << shift;
    pmask |= dmask << shift;
    krem = sh_krem;
    __syncthreads();
  }
  const uint32_t thr = prefix;  // the K-th largest key; take krem of the keys equal to it

  // ---- compaction in index order ----
  const int chunk = ((((N + kWarpsSel - 1) / kWarpsSel) + 31) / 32) * 32;
  const int wbeg = warp * chunk;
  const unsigned lt = (1u << lane) - 1u;
  // one pass counts this warp's keys above the threshold and equal to it; the number it
  // selects follows from the equal keys of the warps before it (lowest indices first)
  uint32_t gtc = 0u, eqc = 0u;
  for (int i = 0; i < chunk; i += 32) {
    const int j = wbeg + i + lane;
    const uint32_t u = j < N ? keys[j] : 0u;
    gtc += __popc(__ballot_sync(kFull, j < N && u > thr));
    eqc += __popc(__ballot_sync(kFull, j < N && u == thr));
  }
  if (lane == 0) {
    wtot[warp] = eqc;
    hist[warp] = gtc;  // the histogram is no longer needed
  }
  __syncthreads();
  uint32_t eq_base = 0u, pos = 0u;
  for (int w = 0; w < warp; ++w) {
    const uint32_t eb = eq_base;
    eq_base += wtot[w];
    const uint32_t take = krem > eb ? min(krem - eb, wtot[w]) : 0u;
    pos += hist[w] + take;
  }
  __syncthreads();
  uint32_t eqrun = eq_base;
  float mpart = 0.f;
  for (int i = 0; i < chunk; i += 32) {
    const int j = wbeg + i + lane;
    const uint32_t u = j < N ? keys[j] : 0u;
    const unsigned be = __ballot_sync(kFull, j < N && u == thr);
    const bool s = (j < N && u > thr) || (j < N && u == thr && eqrun + __popc(be & lt) < krem);
    eqrun += __popc(be);
    const unsigned bs = __ballot_sync(kFull, s);
    if (s) {
      const int k = pos + __popc(bs & lt);
      sel[k] = j;
      if (sel_smem) sel_s[k] = j;
      mpart += ex2(key_value(u));
    }
    pos += __popc(bs);
  }
  mpart = warp_sum(mpart);
  if (lane == 0) red[warp] = mpart;
  __syncthreads();

  // ---- gather plan of S: column, tag, stores, p~, residual slots ----
  const unsigned long long* mask = arr<unsigned long long>(c, A_MASK, layer);
  const int32_t* first = arr<int32_t>(c, A_FIRST, layer);
  const uint8_t* depth = arr<uint8_t>(c, A_DEPTH, layer);
  const int ps = c.plan_stride;
  int32_t* plan = arr<int32_t>(c, A_PLAN, layer) + (size_t)h * c.max_select * ps;
  const int r = a.r;
  __syncthreads();
#pragma unroll 2
  for (int k = tid; k < K; k += kThreads) {
    const int j = sel_smem ? sel_s[k] : sel[k];
    int lam = tag[j];
    lam = lam < 1 ? 1 : (lam > R ? R : lam);
    int stores = 0;
    if (j < n_q) {
      const int dep = depth[j];
      stores = dep < r ? dep : r;
    }
    // the entry's words, stored 16 bytes at a time (ps is a multiple of 4; unused words 0)
    const int b = j >> 6, jt = j & 63;
    uint4* e = reinterpret_cast<uint4*>(plan + (size_t)k * ps);
    const int w2 = __float_as_int(ex2(key_value(keys[j])));
    auto word = [&](int i) -> int {
      if (i == 0) return j;
      if (i == 1) return lam | (stores << 8);
      if (i == 2) return w2;
      const int rp = i - 1;
      if (rp > stores) return 0;
      const unsigned long long mk = mask[(size_t)rp * ncb + b];
      return c.slot_base[rp] + first[(size_t)rp * ncb + b] + __popcll(mk & ((1ull << jt) - 1ull));
    };
    for (int q4 = 0; q4 < ps; q4 += 4)
      e[q4 >> 2] = make_uint4((uint32_t)word(q4), (uint32_t)word(q4 + 1), (uint32_t)word(q4 + 2), (uint32_t)word(q4 + 3));
  }
  if (tid == 0) {
    float m = 0.f;
    for (int w = 0; w < kWarpsSel; ++w) m += red[w];
    arr<float>(c, A_MASS, layer)[h] = m;
  }
}

}  // namespace

cudaError_t launch_select(const SelectArgs& a, int n_layers, cudaStream_t s) {
  const int N = a.n_q + a.n_tail;
  const size_t smem = ((size_t)((N + 3) & ~3) + (sel_fits(N, a.k_sel) ? (size_t)a.k_sel : 0)) * sizeof(uint32_t);
  cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDynMax);
  if (e != cudaSuccess) return e;
  dim3 grid(a.c.H, n_layers);
  select_kernel<<<grid, kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace fl
