// Column selector for sparse loops: top-K of the preceding loop's distribution, the
// selected mass m, and the gather plan the sparse reader follows.
//
// FlashLoop project page, "The Method", Step 02: the preceding loop identifies the
// columns to recompute, and their global probability mass under the preceding loop's
// full distribution is cached so the sparse softmax is not renormalised to 1.
// flozi guide "FlashLoop: store changes between repeated passes", section 3: each
// sparse loop ranks key columns by the previous loop's attention statistics.
//
// Two forms of the same computation, launched for a range of layers at once:
//   select_cta_kernel      one CTA (1024 threads) per (layer, head), every key of the head
//                          in its shared memory (N <= 49152);
//   select_cluster_kernel  one thread-block cluster of cs CTAs (512 threads; cs = 2, 4 or 8
//                          from N) per (layer, head), CTA rank c owning the columns
//                          [c span, (c + 1) span), for N up to FL_MAX_SELECT_COLS.
// Each:
//   keys:     log2 p~_j = score_j - offset[tag_j], mapped to an order-preserving u32,
//             kept in shared memory;
//   select:   radix select of the K-th largest key over the bits where the head's keys
//             differ (the prefix every key shares is skipped), each pass a shared-memory
//             histogram of the keys that still match the prefix (in the cluster form summed
//             bin by bin over the cluster's CTAs through distributed shared memory, so every
//             CTA reaches the same digit) and a block-wide scan from the top bin;
//   compact:  keys above the threshold plus the lowest-index ties, written in index order
//             (per-warp ballots, a block prefix, and in the cluster form the counts of the
//             lower-ranked CTAs), so S is ascending;
//   m, plan:  m = sum_S p~_j; for every j in S its tag, p~_j, the number of stores it has
//             in loop r (min(r, depth_j); 0 for a BF16 tail column) and its slot in each
//             residual store (block first slot + popcount of the block mask), so the sparse
//             reader can issue all of a column's loads at once.
#include "kernels.h"

namespace fl {
namespace {

constexpr int kThreads = 512;
constexpr int kWarpsSel = kThreads / 32;
constexpr int kDigit = 12;                 // bits per radix digit at most
constexpr int kBins = 1 << kDigit;
constexpr int kKeysCta = 18432;            // keys per CTA when the cluster has <= 4 CTAs (two CTAs per SM)
constexpr int kKeysCtaMax = 48128;         // ... and with 8 (one CTA per SM then)
constexpr int kClusterMax = 8;
constexpr int kPlanPer = 4;               // gather-plan entries a thread forms together

__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t o) {
  return __uint_as_float((o & 0x80000000u) ? (o & 0x7fffffffu) : ~o);
}

// ---- thread-block cluster helpers ----
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// every thread of every CTA of the cluster arrives; shared-memory writes before it are
// visible to the cluster's CTAs after it
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned; barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// a 32-bit word of CTA `rank`'s shared memory at the address of `p` in this CTA's
__device__ __forceinline__ uint32_t ld_peer(const void* p, uint32_t rank) {
  uint32_t a = smem_addr(p), ra, v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(ra) : "memory");
  return v;
}

struct SelShared {
  uint32_t hist[2][kBins];   // one per radix pass, alternating: a CTA clears the next one while
                             // the cluster may still read the current one
  uint32_t wtot[32];
  uint32_t wgt[32];
  uint32_t xchg[8];      // this CTA's contributions the cluster reads: and, or, gt, eq, mass bits
  uint32_t digit, krem;
  float offs[kOffStride];
  float red[kWarpsSel];
};

// Inclusive block scan of one value per thread (kNT threads).
template <int kNT>
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
    uint32_t t = lane < kNT / 32 ? wtot[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t n = __shfl_up_sync(kFull, t, o);
      if (lane >= o) t += n;
    }
    if (lane < kNT / 32) wtot[lane] = t;
  }
  __syncthreads();
  return v + (warp > 0 ? wtot[warp - 1] : 0u);
}

// ---- one CTA per (layer, head) ----
constexpr int kThreads1 = 1024;
constexpr int kWarps1 = kThreads1 / 32;
constexpr int kDynMax1 = 194 * 1024;  // dynamic shared memory: keys [, selected columns]
constexpr int kCols1 = 49152;         // the keys of one head that fit it

// Selected columns are kept in shared memory after the keys when both fit.
__host__ __device__ inline bool sel_fits1(int N, int K) {
  return ((size_t)((N + 3) & ~3) + (size_t)K) * sizeof(uint32_t) <= (size_t)kDynMax1;
}
// The head's scores and tags are staged in shared memory by two bulk copies (the scores in
// the key array, turned into keys in place; the tags after it), with the selected columns
// after those, when all three fit.
__host__ __device__ inline size_t stage_bytes1(int N, int K) {
  return (size_t)((N + 3) & ~3) * sizeof(uint32_t) + (size_t)((N + 15) & ~15) + (size_t)K * sizeof(int32_t);
}
__host__ __device__ inline bool stage_fits1(int N, int K) { return stage_bytes1(N, K) <= (size_t)kDynMax1; }

__global__ void __launch_bounds__(kThreads1, 1) select_cta_kernel(SelectArgs a) {
  // [N] keys, then (staged) the N tags, then [K] selected columns when they fit
  extern __shared__ __align__(16) uint32_t keys[];
  const bool staged = stage_fits1(a.n_q + a.n_tail, a.k_sel);
  const bool sel_smem = staged || sel_fits1(a.n_q + a.n_tail, a.k_sel);
  uint8_t* tag_s = reinterpret_cast<uint8_t*>(keys + ((a.n_q + a.n_tail + 3) & ~3));
  int32_t* sel_s = staged ? reinterpret_cast<int32_t*>(tag_s + ((a.n_q + a.n_tail + 15) & ~15))
                          : reinterpret_cast<int32_t*>(keys + ((a.n_q + a.n_tail + 3) & ~3));
  __shared__ uint64_t stage_bar;
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
  if (staged && tid == 0) {
    mbar_init(&stage_bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (staged) {
    // the head's scores and tags in two bulk copies (rows start 256-byte aligned: cap is a
    // multiple of 64; the copies round up to 16 bytes, within the row's capacity)
    if (tid == 0) {
      const unsigned sb = (unsigned)(((N + 3) & ~3) * sizeof(float)), tb = (unsigned)((N + 15) & ~15);
      mbar_expect_tx(&stage_bar, sb + tb);
      bulk_g2s(keys, score, sb, &stage_bar);
      bulk_g2s(tag_s, tag, tb, &stage_bar);
    }
    const bool ok = mbar_wait(&stage_bar, 0);
    if (__syncthreads_or(!ok)) {
      if (tid == 0) record_error(c.status, FL_DEV_TIMEOUT, blockIdx.y * gridDim.x + blockIdx.x);
      return;
    }
  }
  // keys, four columns per thread per step (score rows are 16-byte and tag rows 4-byte
  // aligned: cap is a multiple of 64); from the staged copies, or from global memory with
  // the loads of several steps in flight together
  auto key_of = [&](float sc, int t, int j) {
    if (t < 1 || t > R) {
      record_error(c.status, FL_DEV_TAG_RANGE, j);
      t = t < 1 ? 1 : R;
    }
    return order_key(sc - offs[t]);
  };
  const int N4 = N & ~3;
  uint32_t kand = 0xffffffffu, kor = 0u;  // bits common to every key
  auto keys4 = [&](int j, float4 sc, uint32_t tg) {  // columns j .. j + 3 into keys[j .. j + 3]
    const uint32_t k0 = key_of(sc.x, (int)(tg & 0xff), j), k1 = key_of(sc.y, (int)((tg >> 8) & 0xff), j + 1);
    const uint32_t k2 = key_of(sc.z, (int)((tg >> 16) & 0xff), j + 2), k3 = key_of(sc.w, (int)(tg >> 24), j + 3);
    *reinterpret_cast<uint4*>(keys + j) = make_uint4(k0, k1, k2, k3);
    kand &= k0 & k1 & k2 & k3;
    kor |= k0 | k1 | k2 | k3;
  };
  if (staged) {
    for (int j = 4 * tid; j < N4; j += 4 * kThreads1)  // each thread turns its own scores into keys
      keys4(j, *reinterpret_cast<const float4*>(keys + j), *reinterpret_cast<const uint32_t*>(tag_s + j));
    for (int j = N4 + tid; j < N; j += kThreads1) {
      const uint32_t k = key_of(__uint_as_float(keys[j]), tag_s[j], j);
      keys[j] = k;
      kand &= k;
      kor |= k;
    }
  } else {
#pragma unroll 4
    for (int j = 4 * tid; j < N4; j += 4 * kThreads1)
      keys4(j, *reinterpret_cast<const float4*>(score + j), *reinterpret_cast<const uint32_t*>(tag + j));
    for (int j = N4 + tid; j < N; j += kThreads1) {
      const uint32_t k = key_of(score[j], tag[j], j);
      keys[j] = k;
      kand &= k;
      kor |= k;
    }
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
    for (int i = tid; i < nbins; i += kThreads1) hist[i] = 0u;
    __syncthreads();
    for (int j = tid; j < N; j += kThreads1) {
      const uint32_t u = keys[j];
      if ((u & pmask) == prefix) atomicAdd(&hist[(u >> shift) & dmask], 1u);
    }
    __syncthreads();
    // thread t owns bins [nbins - per*(t+1), nbins - per*t), i.e. descending order
    const int per = nbins / kThreads1 > 0 ? nbins / kThreads1 : 1;
    const int owners = nbins / per;
    uint32_t local = 0u;
    if (tid < owners)
      for (int i = 0; i < per; ++i) local += hist[nbins - per * tid - 1 - i];
    const uint32_t incl = block_scan<kThreads1>(local, wtot, lane, warp);
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
  const int chunk = ((((N + kWarps1 - 1) / kWarps1) + 31) / 32) * 32;
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
  // one gather-plan entry: column j with tag tg, depth dp and key u, written 16 bytes at a
  // time (ps is a multiple of 4; unused words 0)
  auto plan_entry = [&](int32_t* ent, int j, int tg, int dp, uint32_t u) {
    const int lam = tg < 1 ? 1 : (tg > R ? R : tg);
    const int stores = dp < r ? dp : r;  // dp = 0 for a tail column
    const int b = j >> 6, jt = j & 63;
    const int w2 = __float_as_int(ex2(key_value(u)));
    auto word = [&](int i) -> int {
      if (i == 0) return j;
      if (i == 1) return lam | (stores << 8);
      if (i == 2) return w2;
      const int rp = i - 1;
      if (rp > stores) return 0;
      const unsigned long long mk = __ldg(mask + (size_t)rp * ncb + b);
      return c.slot_base[rp] + __ldg(first + (size_t)rp * ncb + b) + __popcll(mk & ((1ull << jt) - 1ull));
    };
    uint4* e = reinterpret_cast<uint4*>(ent);
    for (int q4 = 0; q4 < ps; q4 += 4)
      e[q4 >> 2] = make_uint4((uint32_t)word(q4), (uint32_t)word(q4 + 1), (uint32_t)word(q4 + 2), (uint32_t)word(q4 + 3));
  };
  __syncthreads();
  // the layer's tags, depths, masks and first slots are read-only here (non-coherent loads
  // the compiler may issue ahead of the entries' stores); kPlanPer entries per thread at a
  // time, their columns' tags and depths loaded together before any entry is formed
  for (int k0 = 0; k0 < K; k0 += kPlanPer * kThreads1) {
    int jj[kPlanPer], tg[kPlanPer], dp[kPlanPer];
#pragma unroll
    for (int u = 0; u < kPlanPer; ++u) {
      const int k = k0 + u * kThreads1 + tid;
      jj[u] = k < K ? (sel_smem ? sel_s[k] : sel[k]) : -1;
    }
#pragma unroll
    for (int u = 0; u < kPlanPer; ++u) {
      const int j = jj[u];
      tg[u] = j >= 0 ? __ldg(tag + j) : 1;
      dp[u] = j >= 0 && j < n_q ? __ldg(depth + j) : 0;
    }
#pragma unroll
    for (int u = 0; u < kPlanPer; ++u)
      if (jj[u] >= 0) plan_entry(plan + (size_t)(k0 + u * kThreads1 + tid) * ps, jj[u], tg[u], dp[u], keys[jj[u]]);
  }
  if (tid == 0) {
    float m = 0.f;
    for (int w = 0; w < kWarps1; ++w) m += red[w];
    arr<float>(c, A_MASS, layer)[h] = m;
  }
}


// ---- one cluster per (layer, head) ----
__global__ void __launch_bounds__(kThreads, 2) select_cluster_kernel(SelectArgs a, int cs, int span) {
  extern __shared__ __align__(16) uint32_t keys[];  // [span]
  __shared__ SelShared sh;

  const uint32_t crank = cluster_rank();
  const int h = blockIdx.x / cs, layer = a.layer0 + blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const CacheView& c = a.c;
  const int cap = c.cap, ncb = cap / kG, R = c.R;
  const int n_q = a.n_q, N = a.n_q + a.n_tail, K = a.k_sel;
  const int j0 = (int)crank * span;
  const int nk = max(0, min(span, N - j0));  // this CTA's columns

  const float* score = arr<float>(c, A_SCORE, layer) + (size_t)h * cap;
  const uint8_t* tag = arr<uint8_t>(c, A_TAG, layer) + (size_t)h * cap;
  int32_t* sel = arr<int32_t>(c, A_SEL, layer) + (size_t)h * c.max_select;

  if (tid < kOffStride) sh.offs[tid] = arr<float>(c, A_OFFSET, layer)[(size_t)h * kOffStride + tid];
  __syncthreads();

  // ---- keys, four columns per thread per step (span and cap are multiples of 4 and 64:
  //      16-byte score and 4-byte tag loads), all of a thread's loads in flight together ----
  auto key_of = [&](float sc, int t, int j) {
    if (t < 1 || t > R) {
      record_error(c.status, FL_DEV_TAG_RANGE, j);
      t = t < 1 ? 1 : R;
    }
    return order_key(sc - sh.offs[t]);
  };
  const int nk4 = nk & ~3;
  uint32_t kand = 0xffffffffu, kor = 0u;
#pragma unroll 8
  for (int i = 4 * tid; i < nk4; i += 4 * kThreads) {
    const float4 sc = *reinterpret_cast<const float4*>(score + j0 + i);
    const uint32_t tg = *reinterpret_cast<const uint32_t*>(tag + j0 + i);
    const uint32_t k0 = key_of(sc.x, (int)(tg & 0xff), j0 + i), k1 = key_of(sc.y, (int)((tg >> 8) & 0xff), j0 + i + 1);
    const uint32_t k2 = key_of(sc.z, (int)((tg >> 16) & 0xff), j0 + i + 2), k3 = key_of(sc.w, (int)(tg >> 24), j0 + i + 3);
    *reinterpret_cast<uint4*>(keys + i) = make_uint4(k0, k1, k2, k3);
    kand &= k0 & k1 & k2 & k3;
    kor |= k0 | k1 | k2 | k3;
  }
  for (int i = nk4 + tid; i < nk; i += kThreads) {
    const uint32_t k = key_of(score[j0 + i], tag[j0 + i], j0 + i);
    keys[i] = k;
    kand &= k;
    kor |= k;
  }
  kand = __reduce_and_sync(kFull, kand);
  kor = __reduce_or_sync(kFull, kor);
  if (lane == 0) {
    sh.wtot[warp] = kand;
    sh.wgt[warp] = kor;
  }
  __syncthreads();
  if (tid == 0) {
    uint32_t A = 0xffffffffu, O = 0u;
    for (int w = 0; w < kWarpsSel; ++w) {
      A &= sh.wtot[w];
      O |= sh.wgt[w];
    }
    sh.xchg[0] = A;
    sh.xchg[1] = O;
  }
  cluster_sync();
  kand = 0xffffffffu;
  kor = 0u;
  for (int r = 0; r < cs; ++r) {
    kand &= ld_peer(&sh.xchg[0], r);
    kor |= ld_peer(&sh.xchg[1], r);
  }

  // ---- radix select of the K-th largest key of the head, over the bits where keys differ ----
  const uint32_t diff = kand ^ kor;
  int nbits = diff ? 32 - __clz(diff) : 0;  // digits cover bits [0, nbits)
  uint32_t pmask = nbits >= 32 ? 0u : ~((1u << nbits) - 1u);
  uint32_t prefix = kand & pmask, krem = (uint32_t)K;
  for (int pass = 0; nbits > 0; ++pass) {
    uint32_t* hist = sh.hist[pass & 1];
    const int npass = (nbits + kDigit - 1) / kDigit;
    const int wbits = (nbits + npass - 1) / npass;  // balanced digits
    const int shift = nbits - wbits;
    nbits = shift;
    const int nbins = 1 << wbits;
    const uint32_t dmask = (uint32_t)nbins - 1u;
    for (int i = tid; i < nbins; i += kThreads) hist[i] = 0u;
    cluster_sync();  // every CTA has cleared this pass's histogram (and is done reading the
                     // one this buffer held two passes ago)
    for (int i = tid; i < nk; i += kThreads) {
      const uint32_t u = keys[i];
      if ((u & pmask) == prefix) atomicAdd(&hist[(u >> shift) & dmask], 1u);
    }
    cluster_sync();  // every CTA's histogram is complete
    // thread t owns bins [nbins - per (t + 1), nbins - per t) of the cluster's histogram,
    // i.e. descending order
    const int per = nbins / kThreads > 0 ? nbins / kThreads : 1;
    const int owners = nbins / per;
    constexpr int kPer = kBins / kThreads;  // bins per thread at most
    uint32_t local = 0u;
    uint32_t binc[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      binc[i] = 0u;
      if (tid < owners && i < per) {
        const int bin = nbins - per * tid - 1 - i;
        for (int r = 0; r < cs; ++r) binc[i] += ld_peer(&hist[bin], r);
        local += binc[i];
      }
    }
    const uint32_t incl = block_scan<kThreads>(local, sh.wtot, lane, warp);
    const uint32_t excl = incl - local;
    if (tid < owners && excl < krem && krem <= incl) {
      uint32_t cum = excl;
      bool found = false;
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        if (!found && i < per && cum + binc[i] >= krem) {
          sh.digit = (uint32_t)(nbins - per * tid - 1 - i);
          sh.krem = krem - cum;
          found = true;
        }
        cum += binc[i];
      }
    }
    __syncthreads();
    prefix |= sh.digit << shift;
    pmask |= dmask << shift;
    krem = sh.krem;
    __syncthreads();
  }
  const uint32_t thr = prefix;  // the K-th largest key; take krem of the keys equal to it (index order)

  // ---- compaction in index order: warp w owns keys [w chunk, (w + 1) chunk) ----
  const int chunk = ((((nk + kWarpsSel - 1) / kWarpsSel) + 31) / 32) * 32;
  const int wbeg = warp * chunk;
  const unsigned lt = (1u << lane) - 1u;
  uint32_t gtc = 0u, eqc = 0u;
  for (int i = 0; i < chunk; i += 32) {
    const int j = wbeg + i + lane;
    const uint32_t u = j < nk ? keys[j] : 0u;
    gtc += __popc(__ballot_sync(kFull, j < nk && u > thr));
    eqc += __popc(__ballot_sync(kFull, j < nk && u == thr));
  }
  if (lane == 0) {
    sh.wtot[warp] = eqc;
    sh.wgt[warp] = gtc;
  }
  __syncthreads();
  if (tid == 0) {
    uint32_t g = 0u, e = 0u;
    for (int w = 0; w < kWarpsSel; ++w) {
      g += sh.wgt[w];
      e += sh.wtot[w];
    }
    sh.xchg[2] = g;
    sh.xchg[3] = e;
  }
  cluster_sync();
  // ties go to the lowest indices: the lower-ranked CTAs' equal keys come first
  uint32_t eq_before = 0u, sel_before = 0u;
  for (uint32_t r = 0; r < crank; ++r) {
    const uint32_t g = ld_peer(&sh.xchg[2], r), e = ld_peer(&sh.xchg[3], r);
    const uint32_t take = krem > eq_before ? min(krem - eq_before, e) : 0u;
    sel_before += g + take;
    eq_before += e;
  }
  uint32_t eq_base = eq_before, pos = sel_before;
  for (int w = 0; w < warp; ++w) {
    const uint32_t eb = eq_base;
    eq_base += sh.wtot[w];
    const uint32_t take = krem > eb ? min(krem - eb, sh.wtot[w]) : 0u;
    pos += sh.wgt[w] + take;
  }
  uint32_t eqrun = eq_base;
  float mpart = 0.f;
  for (int i = 0; i < chunk; i += 32) {
    const int j = wbeg + i + lane;
    const uint32_t u = j < nk ? keys[j] : 0u;
    const unsigned be = __ballot_sync(kFull, j < nk && u == thr);
    const bool s = (j < nk && u > thr) || (j < nk && u == thr && eqrun + __popc(be & lt) < krem);
    eqrun += __popc(be);
    const unsigned bs = __ballot_sync(kFull, s);
    if (s) {
      sel[pos + __popc(bs & lt)] = j0 + j;
      mpart += ex2(key_value(u));
    }
    pos += __popc(bs);
  }
  mpart = warp_sum(mpart);
  if (lane == 0) sh.red[warp] = mpart;
  __syncthreads();  // this CTA's part of S is written (global, visible to the block)
  if (tid == 0) {
    float m = 0.f;
    for (int w = 0; w < kWarpsSel; ++w) m += sh.red[w];
    sh.xchg[4] = __float_as_uint(m);
  }
  cluster_sync();  // every CTA's mass part is in place
  // this CTA's part of S: [sel0, sel1) -- its keys above the threshold plus its share of
  // the ties
  const uint32_t sel0 = sel_before;
  const uint32_t sel1 = sel0 + sh.xchg[2] + (krem > eq_before ? min(krem - eq_before, sh.xchg[3]) : 0u);
  if (crank == 0 && tid == 0) {
    float m = 0.f;
    for (int r = 0; r < cs; ++r) m += __uint_as_float(ld_peer(&sh.xchg[4], r));
    arr<float>(c, A_MASS, layer)[h] = m;
  }

  // ---- gather plan of this CTA's part of S: column, tag, stores, p~, residual slots ----
  const unsigned long long* mask = arr<unsigned long long>(c, A_MASK, layer);
  const int32_t* first = arr<int32_t>(c, A_FIRST, layer);
  const uint8_t* depth = arr<uint8_t>(c, A_DEPTH, layer);
  const int ps = c.plan_stride;
  int32_t* plan = arr<int32_t>(c, A_PLAN, layer) + (size_t)h * c.max_select * ps;
  const int r = a.r;
  // one gather-plan entry: column j with tag tg, depth dp and key u, written 16 bytes at a
  // time (ps is a multiple of 4; unused words 0)
  auto plan_entry = [&](int32_t* ent, int j, int tg, int dp, uint32_t u) {
    const int lam = tg < 1 ? 1 : (tg > R ? R : tg);
    const int stores = dp < r ? dp : r;  // dp = 0 for a tail column
    const int b = j >> 6, jt = j & 63;
    const int w2 = __float_as_int(ex2(key_value(u)));
    auto word = [&](int i) -> int {
      if (i == 0) return j;
      if (i == 1) return lam | (stores << 8);
      if (i == 2) return w2;
      const int rp = i - 1;
      if (rp > stores) return 0;
      const unsigned long long mk = __ldg(mask + (size_t)rp * ncb + b);
      return c.slot_base[rp] + __ldg(first + (size_t)rp * ncb + b) + __popcll(mk & ((1ull << jt) - 1ull));
    };
    uint4* e = reinterpret_cast<uint4*>(ent);
    for (int q4 = 0; q4 < ps; q4 += 4)
      e[q4 >> 2] = make_uint4((uint32_t)word(q4), (uint32_t)word(q4 + 1), (uint32_t)word(q4 + 2), (uint32_t)word(q4 + 3));
  };
  for (int k0 = (int)sel0; k0 < (int)sel1; k0 += kPlanPer * kThreads) {
    int jj[kPlanPer], tg[kPlanPer], dp[kPlanPer];
#pragma unroll
    for (int u = 0; u < kPlanPer; ++u) {
      const int k = k0 + u * kThreads + tid;
      jj[u] = k < (int)sel1 ? sel[k] : -1;
    }
#pragma unroll
    for (int u = 0; u < kPlanPer; ++u) {
      const int j = jj[u];
      tg[u] = j >= 0 ? __ldg(tag + j) : 1;
      dp[u] = j >= 0 && j < n_q ? __ldg(depth + j) : 0;
    }
#pragma unroll
    for (int u = 0; u < kPlanPer; ++u)
      if (jj[u] >= 0)
        plan_entry(plan + (size_t)(k0 + u * kThreads + tid) * ps, jj[u], tg[u], dp[u], keys[jj[u] - j0]);
  }
  cluster_sync();  // no CTA leaves while another may still read its shared memory
}

// CTAs per cluster (at least `want`, at least 2) and columns per CTA for N columns; cs = 0
// when N is too large.
void select_shape(int N, int want, int* cs, int* span) {
  *cs = 0;
  *span = 0;
  for (int c = want > 2 ? want : 2; c <= kClusterMax; c *= 2) {
    const int sp = ((N + c - 1) / c + 63) / 64 * 64;
    if (sp <= (c < kClusterMax ? kKeysCta : kKeysCtaMax)) {
      *cs = c;
      *span = sp;
      return;
    }
  }
}

}  // namespace

static_assert(kClusterMax * kKeysCtaMax == FL_MAX_SELECT_COLS, "the header states the selector's column limit");

cudaError_t launch_select(const SelectArgs& a, int n_layers, cudaStream_t s) {
  const int N = a.n_q + a.n_tail;
  // one CTA per (layer, head) whenever the head's keys fit one CTA (measured faster than
  // clusters even when the heads leave SMs idle: 23.5 against 26.8 us per selection for
  // 16 heads of 8192 columns); beyond that, clusters of at least as many CTAs per head as
  // it takes to occupy every SM
  const int sms = device_sms() > 0 ? device_sms() : 148;
  const long long heads_all = (long long)a.c.H * n_layers;
  int want = 1;
  while (want < kClusterMax && heads_all * want < sms) want *= 2;
  if (N <= kCols1) {
    const size_t smem = stage_fits1(N, a.k_sel)
                            ? stage_bytes1(N, a.k_sel)
                            : ((size_t)((N + 3) & ~3) + (sel_fits1(N, a.k_sel) ? (size_t)a.k_sel : 0)) * sizeof(uint32_t);
    cudaError_t e = cudaFuncSetAttribute(select_cta_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDynMax1);
    if (e != cudaSuccess) return e;
    select_cta_kernel<<<dim3(a.c.H, n_layers), kThreads1, smem, s>>>(a);
    return cudaGetLastError();
  }
  int cs = 0, span = 0;
  select_shape(N, want, &cs, &span);
  if (cs == 0) return cudaErrorInvalidValue;
  const size_t smem = (size_t)span * sizeof(uint32_t);
  cudaError_t e = cudaFuncSetAttribute(select_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kKeysCtaMax * (int)sizeof(uint32_t));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.c.H * cs, n_layers);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, select_cluster_kernel, a, cs, span);
}

}  // namespace fl
