// Token-sparse update selector: A_r from A_{r-1} by normalized hidden-state change.
//
// FlashLoop project page, "The Method", Step 01: only the tokens that stay active are
// updated in a loop; flozi guide "FlashLoop: store changes between repeated passes",
// section 3: after the dense early loops each loop ranks the previously updated tokens
// by normalized hidden-state change and keeps a top-k subset; later selections are
// restricted to earlier active sets, so the sets nest.
//
// Two launches:
//   token_change_kernel  one warp per candidate token: key = ||h_cur - h_prev||^2 /
//                        ||h_prev||^2 with fp64 sums of the exactly widened BF16 values
//                        (HBM-bound: 2 x d_model x 2 bytes per token);
//   token_select_kernel  one CTA: radix select of the k-th largest key, 12-bit digits
//                        from the top, stopping once the wanted key's bin is taken whole;
//                        then the chosen tokens in index order (the candidates are
//                        ascending, so the output is too).
#include "kernels.h"

namespace fl {
namespace {

constexpr int kChangeWarps = 8;
constexpr int kSelThreads = 1024;
constexpr int kDigitBits = 12;

// Order-preserving 64-bit image of a key: valid keys (>= 0, +inf included) map above
// every invalid one (NaN: a candidate outside [0, n_tokens) or non-finite inputs).
__device__ __forceinline__ unsigned long long key_bits(double v) {
  return v >= 0.0 ? (unsigned long long)__double_as_longlong(v) + 1ull : 0ull;
}

__global__ void __launch_bounds__(kChangeWarps * 32, 4) token_change_kernel(TokenArgs a) {
  const int lane = threadIdx.x & 31;
  const int n_vec = a.d_model / 8;
  for (long long i = (long long)blockIdx.x * kChangeWarps + (threadIdx.x >> 5); i < a.n_rows;
       i += (long long)gridDim.x * kChangeWarps) {
    const int j = __ldg(a.rows + i);
    if (j < 0 || j >= a.n_tokens || (i > 0 && __ldg(a.rows + i - 1) >= j)) {
      if (lane == 0 && a.status)
        record_error(a.status, (j < 0 || j >= a.n_tokens) ? FL_DEV_ROWS_RANGE : FL_DEV_ROWS_ORDER, j);
      if (j < 0 || j >= a.n_tokens) {
        if (lane == 0) a.keys[i] = __longlong_as_double(0x7ff8000000000000ll);  // NaN: ranks last
        continue;
      }
    }
    const uint4* p = reinterpret_cast<const uint4*>(a.h_prev + (size_t)j * a.row_stride);
    const uint4* c = reinterpret_cast<const uint4*>(a.h_cur + (size_t)j * a.row_stride);
    double num = 0.0, den = 0.0;
#pragma unroll 8
    for (int v = lane; v < n_vec; v += 32) {
      const uint4 pw = __ldcs(p + v), cw = __ldcs(c + v);
      const uint32_t pp[4] = {pw.x, pw.y, pw.z, pw.w}, cc[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const double p0 = (double)bf16_lo(pp[e]), p1 = (double)bf16_hi(pp[e]);
        const double d0 = (double)bf16_lo(cc[e]) - p0, d1 = (double)bf16_hi(cc[e]) - p1;
        num = fma(d0, d0, num);
        num = fma(d1, d1, num);
        den = fma(p0, p0, den);
        den = fma(p1, p1, den);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      num += __shfl_xor_sync(kFull, num, o);
      den += __shfl_xor_sync(kFull, den, o);
    }
    if (lane == 0) a.keys[i] = (den == 0.0 && num == 0.0) ? 0.0 : __ddiv_rn(num, den);
  }
}

// Exclusive block prefix sum of one value per thread (kSelThreads threads); `red` holds
// 32 words; `total` receives the block's sum.
__device__ __forceinline__ int block_excl_scan(int v, int* red, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) red[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = red[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(kFull, w, o);
      if (lane >= o) w += y;
    }
    red[lane] = w;
  }
  __syncthreads();
  total = red[31];
  const int before = (warp > 0 ? red[warp - 1] : 0) + x - v;
  __syncthreads();
  return before;
}

// The keys are read in chunks of kPer x kSelThreads: warp w takes the kPer x 32
// consecutive keys [c0 + 256 w, c0 + 256 w + 256) of each chunk, lane l key
// c0 + 256 w + 32 q + l in round q (coalesced), all loads of a chunk issued before any
// is used.  Index order within a chunk is warp, then round, then lane.
constexpr int kPer = 8;
constexpr int kChunk = kPer * kSelThreads;

__device__ __forceinline__ void load_chunk(const double* keys, int n, int c0, unsigned long long* u, unsigned& valid) {
  const int i0 = c0 + kPer * 32 * (int)(threadIdx.x >> 5) + (int)(threadIdx.x & 31);
  double v[kPer];
  valid = 0u;
#pragma unroll
  for (int q = 0; q < kPer; ++q) {
    const bool in = i0 + 32 * q < n;
    v[q] = in ? __ldg(keys + i0 + 32 * q) : -1.0;
    valid |= in ? 1u << q : 0u;
  }
#pragma unroll
  for (int q = 0; q < kPer; ++q) u[q] = key_bits(v[q]);
}

__global__ void __launch_bounds__(kSelThreads) token_select_kernel(TokenArgs a) {
  __shared__ unsigned hist[1 << kDigitBits];
  __shared__ int red[32];
  __shared__ int s_digit, s_above, s_count;
  const int tid = threadIdx.x;
  const int n = (int)a.n_rows, k = a.k;
  unsigned long long u[kPer];
  unsigned valid;

  // Radix passes over the key bits, most significant digit first.  After each pass the
  // wanted (k-th largest) key's digit is known; once every key that shares the known
  // high bits with it is taken (its bin holds exactly the remaining count), the lower
  // bits no longer matter.
  int shift = 64;
  unsigned long long known = 0ull, prefix = 0ull;
  int krem = k;  // rank (from the top, 1-based) of the wanted key among those matching prefix
  while (shift > 0) {
    const int wb = shift < kDigitBits ? shift : kDigitBits;
    shift -= wb;
    const int nb = 1 << wb;
    const unsigned dmask = (unsigned)nb - 1u;
    for (int b = tid; b < nb; b += kSelThreads) hist[b] = 0u;
    __syncthreads();
    for (int c0 = 0; c0 < n; c0 += kChunk) {
      load_chunk(a.keys, n, c0, u, valid);
#pragma unroll
      for (int q = 0; q < kPer; ++q)
        if (((valid >> q) & 1u) && (u[q] & known) == prefix) atomicAdd(&hist[(unsigned)(u[q] >> shift) & dmask], 1u);
    }
    __syncthreads();
    // thread t owns the 4 bins [hi - 4, hi), hi = nb - 4t, counted down from the top bin
    const int hi = nb - 4 * tid;
    int cb[4], c4 = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int b = hi - 1 - q;
      cb[q] = b >= 0 ? (int)hist[b] : 0;
      c4 += cb[q];
    }
    int total;
    const int before = block_excl_scan(c4, red, total);
    if (before < krem && before + c4 >= krem) {
      int acc = before;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (acc + cb[q] >= krem) {
          s_digit = hi - 1 - q;
          s_above = acc;
          s_count = cb[q];
          break;
        }
        acc += cb[q];
      }
    }
    __syncthreads();
    prefix |= (unsigned long long)s_digit << shift;
    known |= (unsigned long long)dmask << shift;
    krem -= s_above;
    const bool all_taken = s_count == krem;
    __syncthreads();
    if (all_taken) break;
  }

  // the chosen candidates in index order: every key whose known bits exceed prefix, then
  // the first krem of those equal to it
  const int lane = tid & 31;
  const unsigned below = (1u << lane) - 1u;
  int gt_base = 0, eq_base = 0;
  for (int c0 = 0; c0 < n; c0 += kChunk) {
    load_chunk(a.keys, n, c0, u, valid);
    unsigned gtm[kPer], eqm[kPer];
    int g = 0, e = 0;
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const unsigned long long m = u[q] & known;
      const bool in = (valid >> q) & 1u;
      gtm[q] = __ballot_sync(kFull, in && m > prefix);
      eqm[q] = __ballot_sync(kFull, in && m == prefix);
      g += __popc(gtm[q]);
      e += __popc(eqm[q]);
    }
    // counts of the warps before this one (g, e <= 256 each: packed in one word)
    int tot;
    const int packed = block_excl_scan(lane == 0 ? (g << 16) | e : 0, red, tot);
    const int wb = __shfl_sync(kFull, packed, 0);
    int gt_run = gt_base + (wb >> 16), eq_run = eq_base + (wb & 0xffff);
    const int i0 = c0 + kPer * 32 * (tid >> 5) + lane;
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int gr = gt_run + __popc(gtm[q] & below), er = eq_run + __popc(eqm[q] & below);
      if ((gtm[q] >> lane) & 1u) a.rows_out[gr + (er < krem ? er : krem)] = __ldg(a.rows + i0 + 32 * q);
      else if (((eqm[q] >> lane) & 1u) && er < krem) a.rows_out[gr + er] = __ldg(a.rows + i0 + 32 * q);
      gt_run += __popc(gtm[q]);
      eq_run += __popc(eqm[q]);
    }
    gt_base += tot >> 16;
    eq_base += tot & 0xffff;
  }
}

}  // namespace

cudaError_t launch_token_select(const TokenArgs& a, cudaStream_t s) {
  if (a.n_rows == 0) return cudaSuccess;
  // a resident grid (4 CTAs of 8 warps per SM) striding over the candidates
  long long blocks = (a.n_rows + kChangeWarps - 1) / kChangeWarps;
  if (blocks > 148LL * 4) blocks = 148LL * 4;
  token_change_kernel<<<(unsigned)blocks, kChangeWarps * 32, 0, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || a.k == 0) return e;
  token_select_kernel<<<1, kSelThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace fl
