// Sparse prefill attention on the 5th-generation tensor cores (tcgen05, TMEM).
//
// FlashLoop project page, "The Method": in a token-sparse loop only the active tokens
// are recomputed (Step 01), and the selected tokens are gathered into compact buffers
// so that the work stays a regular GEMM (the paragraph after Step 03).  Here: the
// queries of the active tokens (compact, in token order) attend causally over every
// token's key and value of the loop:
//     o_i = softmax_{j <= pos_i}(q_i k_j^T / sqrt(128)) v_j.
//
// One CTA of 8 softmax warps and one MMA warp per (128 active queries, head).  The query
// tile stays in shared memory; key tiles of 128 tokens and value tiles stream through two
// buffers each, copied by a load warp with tensor maps (TMA: 64 x 128 boxes in the
// 128-byte swizzle the MMA descriptors name, zeros past the end) as soon as the tensor
// cores release a buffer.  The MMA warp issues S = Q K^T (8 tcgen05.mma of M = N = 128,
// K = 16; BF16 operands from 128-byte-swizzled shared memory; fp32 accumulators in TMEM)
// one tile ahead into alternating TMEM buffers, and O += P V once P is written (V read
// MN-major).  P reaches the tensor cores as two BF16 tiles, P = P_hi + P_lo with
// P_hi = bf16(p) and P_lo = bf16(p - P_hi), so the value product carries p to about 16
// significant bits rather than BF16's 8 (16 MMAs per value tile instead of 8).  Softmax warp w reads TMEM lanes
// 32 (w % 4) ..: its thread t owns query row 32 (w % 4) + t and the 64 columns of half
// w / 4 -- it masks, runs the online softmax in the base-2 domain, writes its half of
// P_hi and P_lo to shared memory in the operand layout and rescales its half of the output row
// in TMEM.  The warps hand over through mbarriers only (copies count transaction bytes,
// softmax threads arrive when a score buffer is consumed and when P is in place,
// tcgen05.commit signals finished MMAs), so no CTA-wide barrier sits in the loop; every
// wait is bounded.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "kernels.h"

namespace fl {
namespace {

constexpr int kPT = 128;                      // queries per tile = keys per tile = head dim
constexpr int kTileB = kPT * kPT * 2;         // one 128 x 128 BF16 tile
constexpr int kSoftmaxThreads = 256;          // 8 softmax warps: TMEM lane group w % 4, column half w / 4
constexpr int kMmaWarp = kSoftmaxThreads / 32;  // issues the MMAs
constexpr int kLoadWarp = kMmaWarp + 1;         // issues the tensor-map copies
constexpr int kPrefillThreads = kSoftmaxThreads + 64;
constexpr int kTmemCols = 512;                // S buffers: columns 0..127, 128..255; O: 256..383
constexpr uint32_t kIdescS = (1u << 4) | (1u << 7) | (1u << 10) | ((kPT >> 3) << 17) | ((kPT >> 4) << 24);
constexpr uint32_t kIdescPV = kIdescS | (1u << 16);  // B (V) read MN-major

struct PrefillCtl {
  uint64_t bar_s[2], bar_o;      // tensor cores -> softmax warps (tcgen05.commit)
  uint64_t bar_a[2], bar_e[2];   // softmax warps -> MMA warp, one arrival per softmax thread
  uint64_t qfull, kfull[2], vfull[2];  // copies landed (transaction bytes)
  uint64_t kempty[2], vempty[2];       // tensor cores done with a K / V buffer (tcgen05.commit)
  uint32_t tmem;
  int32_t pmax;
  int32_t failed;                // a bounded wait ran out somewhere
  int32_t pad;
  float rmax[2][kPT];            // per column half: this tile's row maxima
};
// the control block, then 1024-byte-aligned tiles: Q, K[3], V[2], P
constexpr int kPrefillSmem = (int)sizeof(PrefillCtl) + 1023 + 7 * kTileB;

// Operand tiles (128 x 128 BF16): two 64-column blocks of 128 rows x 128 bytes, 16 KB
// apart; within each 1024-byte group of 8 rows the 16-byte chunk index is XOR-ed with
// (row mod 8) -- the 128-byte swizzle that the tensor-map copies write and the
// descriptors below name.

// Shared-memory matrix descriptors (tcgen05): start address >> 4 in bits 0..13, leading
// byte offset >> 4 in bits 16..29, stride byte offset >> 4 in bits 32..45, version 1 in
// bits 46..47, layout 2 (128-byte swizzle) in bits 61..63.
// K-major: rows 128 bytes apart, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_k(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}
// MN-major: 64-element blocks along N 16 KB apart, 8-row groups along K 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_mn(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | (1024ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}

// D (TMEM) = A B^T (+ D when acc != 0); no output lane is disabled
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  const uint32_t z0 = 0u, z1 = 0u, z2 = 0u, z3 = 0u;
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
      ::"r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(z0), "r"(z1), "r"(z2), "r"(z3)
      : "memory");
}
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive fp32 columns of this thread's TMEM lane
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
               : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float* v) {
  uint32_t r[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(v[i]);
  asm volatile("tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
               ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
               : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// A 128-row x 64-column BF16 box of a [heads][rows][128] tensor (tensor map `map`: 128-byte
// swizzle, zeros past the rows) into shared memory at dst (1024-byte aligned); completion
// is counted in transaction bytes on `bar`.
__device__ __forceinline__ void tma_box(uint32_t dst, const CUtensorMap* map, int col, int row, int head, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(col), "r"(row), "r"(head), "r"(smem_addr(bar))
      : "memory");
}
// a whole 128 x 128 tile: its two 64-column blocks, 16 KB apart
__device__ __forceinline__ void tma_tile(uint32_t dst, const CUtensorMap* map, int row, int head, uint64_t* bar) {
  mbar_expect_tx(bar, kTileB);
  tma_box(dst, map, 0, row, head, bar);
  tma_box(dst + 16384u, map, 64, row, head, bar);
}

// barrier of the two warps (w, w + 4) that share TMEM lanes 32 w ..
__device__ __forceinline__ void pair_bar(int grp) { asm volatile("bar.sync %0, 64;" ::"r"(grp + 1) : "memory"); }
// barrier of the eight softmax warps
__device__ __forceinline__ void softmax_bar() { asm volatile("bar.sync 5, %0;" ::"n"(kSoftmaxThreads) : "memory"); }
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{ .reg .b64 st; mbarrier.arrive.shared::cta.b64 st, [%0]; }" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&b);
}

__global__ void __launch_bounds__(kPrefillThreads, 1)
    prefill_attn_kernel(const __grid_constant__ PrefillArgs a, const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  PrefillCtl& ctl = *reinterpret_cast<PrefillCtl*>(smem_raw);
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + (uint32_t)sizeof(PrefillCtl) + 1023u) & ~1023u;  // 1024-byte aligned tiles
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sQ = base;
  auto sK = [&](int t) { return base + (uint32_t)(1 + (t & 1)) * kTileB; };  // K(t): buffer t % 2
  auto sV = [&](int t) { return base + (uint32_t)(3 + (t & 1)) * kTileB; };  // V(t): buffer t % 2
  const uint32_t sP = base + 5u * kTileB;     // P_hi, then P_lo one tile further

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool softmax_warp = warp < kMmaWarp;
  const int grp = warp & 3, hf = (warp >> 2) & 1;
  const int row = 32 * grp + lane;  // a softmax thread's query row = its TMEM lane
  const int h = blockIdx.y, i0 = blockIdx.x * kPT;

  // the row's position (-1: a padding row or a bad position)
  int qp = -1;
  if (softmax_warp && i0 + row < a.n_act) {
    qp = __ldg(a.pos + i0 + row);
    const bool bad_order = i0 + row > 0 && __ldg(a.pos + i0 + row - 1) >= qp;
    const bool bad_range = qp < 0 || qp >= a.n_tokens;
    if ((bad_order || bad_range) && hf == 0 && a.status)
      record_error(a.status, bad_range ? FL_DEV_ROWS_RANGE : FL_DEV_ROWS_ORDER, qp);
    if (bad_range) qp = -1;
  }
  if (tid == 0) {
    mbar_init(&ctl.bar_s[0], 1);
    mbar_init(&ctl.bar_s[1], 1);
    mbar_init(&ctl.bar_o, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl.bar_a[i], kSoftmaxThreads);
      mbar_init(&ctl.bar_e[i], kSoftmaxThreads);
      mbar_init(&ctl.vfull[i], 1);
      mbar_init(&ctl.vempty[i], 1);
      mbar_init(&ctl.kfull[i], 1);
      mbar_init(&ctl.kempty[i], 1);
    }
    mbar_init(&ctl.qfull, 1);
    fence_mbar_init();
    ctl.pmax = -1;
    ctl.failed = 0;
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&ctl.tmem)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  __syncthreads();
  {
    int m = qp;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(kFull, m, o));
    if (lane == 0) atomicMax(&ctl.pmax, m);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem;
  const uint32_t tO = tmem + 2 * kPT;
  auto tS = [&](int b) { return tmem + (uint32_t)(b * kPT); };
  const int pmax = ctl.pmax;
  const int n_kt = pmax < 0 ? 0 : pmax / kPT + 1;  // key tiles up to the tile's last position

  // A wait that ran out marks the CTA failed; later waits are then skipped (every barrier
  // and arrival still happens, so nothing can block), and the results are not used.
  bool failed = false;
  auto wait = [&](uint64_t* bar, unsigned parity) {
    if (failed) return;
    if (!mbar_wait(bar, parity)) {
      failed = true;
      ctl.failed = 1;
    }
  };

  if (warp == kMmaWarp) {
    // ---- MMA warp: lane 0 issues; S(t+1) once its key tile has landed and S buffer
    //      (t+1) % 2 is consumed, PV(t) once P(t) is written and V(t) has landed ----
    for (int t = 0; t < n_kt; ++t) {
      const int b = t & 1;
      wait(&ctl.bar_a[b], (unsigned)((t >> 1) & 1));
      if (t == 0) wait(&ctl.qfull, 0u);
      for (int u = t == 0 ? 0 : t + 1; u <= t + 1 && u < n_kt; ++u) {
        wait(&ctl.kfull[u & 1], (unsigned)((u >> 1) & 1));
        tc_fence_after();
        if (lane == 0 && !failed) {
#pragma unroll
          for (int s = 0; s < kPT / 16; ++s) {
            const uint32_t off = (uint32_t)((s >> 2) * 16384 + (s & 3) * 32);
            mma_bf16(tS(u & 1), desc_k(sQ + off), desc_k(sK(u) + off), kIdescS, s > 0 ? 1u : 0u);
          }
          mma_commit(&ctl.bar_s[u & 1]);
          mma_commit(&ctl.kempty[u & 1]);
        }
        __syncwarp();
      }
      wait(&ctl.bar_e[b], (unsigned)((t >> 1) & 1));
      wait(&ctl.vfull[b], (unsigned)((t >> 1) & 1));
      tc_fence_after();
      if (lane == 0 && !failed) {
#pragma unroll
        for (int s = 0; s < kPT / 16; ++s) {
          const uint32_t off = (uint32_t)((s >> 2) * 16384 + (s & 3) * 32);
          const uint64_t vd = desc_mn(sV(t) + (uint32_t)s * 2048u);
          mma_bf16(tO, desc_k(sP + off), vd, kIdescPV, (t > 0 || s > 0) ? 1u : 0u);       // P_hi V
          mma_bf16(tO, desc_k(sP + (uint32_t)kTileB + off), vd, kIdescPV, 1u);             // P_lo V
        }
        mma_commit(&ctl.bar_o);
        mma_commit(&ctl.vempty[b]);
      }
      __syncwarp();
    }
  } else if (warp == kLoadWarp) {
    // ---- load warp: lane 0 copies Q once, then K(t) into buffer t % 2 and V(t) into
    //      buffer t % 2 as soon as the tensor cores are done with the tile they held ----
    if (lane == 0 && n_kt > 0) {
      tma_tile(sQ, &tm_q, i0, h, &ctl.qfull);
      for (int t = 0; t < n_kt; ++t) {
        if (t >= 2) wait(&ctl.kempty[t & 1], (unsigned)(((t - 2) >> 1) & 1));
        if (!failed) tma_tile(sK(t), &tm_k, t * kPT, h, &ctl.kfull[t & 1]);
        if (t >= 2) wait(&ctl.vempty[t & 1], (unsigned)(((t - 2) >> 1) & 1));
        if (!failed) tma_tile(sV(t), &tm_v, t * kPT, h, &ctl.vfull[t & 1]);
      }
    }
    __syncwarp();
  } else if (n_kt > 0) {
    // ---- softmax warps ----
    const uint32_t lane_off = (uint32_t)(32 * grp) << 16;  // this warp's TMEM lanes
    const float kScale = 1.4426950408889634f * 0.08838834764831845f;  // log2(e) / sqrt(128)
    uint8_t* p_row = gbase + 5 * kTileB + hf * 16384 + row * 128;   // this thread's half-row of P_hi
    uint8_t* p_row_lo = p_row + kTileB;                             // ... and of P_lo
    float m_run = -INFINITY, l_half = 0.f;
    for (int t = 0; t < n_kt; ++t) {
      const int b = t & 1, j0 = t * kPT;
      // (A) S(t-1) is consumed: S buffer (t+1) % 2 may be overwritten
      tc_fence_before();
      mbar_arrive(&ctl.bar_a[b]);
      // (B) S(t) is complete
      wait(&ctl.bar_s[b], (unsigned)((t >> 1) & 1));
      tc_fence_after();
      // (C) softmax of this row's own 64 columns (in registers); the row maximum is
      //     exchanged with the partner half.  Lazy rescaling: the running maximum is kept
      //     unless this tile exceeds it by more than 8 (weights then stay below 2^8, and O
      //     and l share the scale, so o = O / l is unchanged).
      float sv[64];
      tmem_ld32(tS(b) + lane_off + 64 * hf, sv);
      tmem_ld32(tS(b) + lane_off + 64 * hf + 32, sv + 32);
      const int c_own = j0 + 64 * hf;
      const bool full = c_own + 63 <= qp;  // every own column visible (no mask needed)
      float mx8[8];  // eight independent partial maxima (short dependency chains)
#pragma unroll
      for (int k = 0; k < 8; ++k) mx8[k] = -INFINITY;
      if (full) {
#pragma unroll
        for (int i = 0; i < 64; ++i) mx8[i & 7] = fmaxf(mx8[i & 7], sv[i]);
      } else {
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if (c_own + i <= qp) mx8[i & 7] = fmaxf(mx8[i & 7], sv[i]);
      }
      float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                       fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      ctl.rmax[hf][row] = mx;
      pair_bar(grp);
      mx = fmaxf(mx, ctl.rmax[1 - hf][row]);
      pair_bar(grp);  // both halves have read the maxima before either writes the next tile's
      const float m_tile = mx * kScale;
      float alpha = 1.f;
      if (m_tile > m_run + 8.f) {  // also the first visible tile (m_run = -inf): alpha = 0
        alpha = ex2(m_run - m_tile);
        m_run = m_tile;
      }
      // weights (fp32 row sum in four partial sums; P split into BF16 P_hi + P_lo for the
      // tensor cores: p - P_hi is exact in fp32, then rounded to BF16)
      float ls4[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t pw[32], pl[32];
      auto split2 = [&](int e, float p0, float p1) {
        pw[e] = pack_bf16(p0, p1);
        pl[e] = pack_bf16(p0 - __uint_as_float(pw[e] << 16), p1 - __uint_as_float(pw[e] & 0xffff0000u));
      };
      if (full) {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float p0 = ex2(fmaf(sv[2 * e], kScale, -m_run)), p1 = ex2(fmaf(sv[2 * e + 1], kScale, -m_run));
          split2(e, p0, p1);
          ls4[e & 3] += p0 + p1;
        }
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int i = 2 * e;
          const float p0 = (c_own + i <= qp) ? ex2(fmaf(sv[i], kScale, -m_run)) : 0.f;
          const float p1 = (c_own + i + 1 <= qp) ? ex2(fmaf(sv[i + 1], kScale, -m_run)) : 0.f;
          split2(e, p0, p1);
          ls4[e & 3] += p0 + p1;
        }
      }
      l_half = fmaf(l_half, alpha, (ls4[0] + ls4[1]) + (ls4[2] + ls4[3]));

      // (D) PV(t-1) is complete: P may be overwritten and the output accumulator rescaled
      if (t > 0) {
        wait(&ctl.bar_o, (unsigned)((t - 1) & 1));
        tc_fence_after();
        if (__any_sync(kFull, alpha != 1.f)) {
          float ov[32];
#pragma unroll 1
          for (int c = 0; c < 2; ++c) {
            tmem_ld32(tO + lane_off + 64 * hf + 32 * c, ov);
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] *= alpha;
            tmem_st32(tO + lane_off + 64 * hf + 32 * c, ov);
          }
        }
      }
#pragma unroll
      for (int q8 = 0; q8 < 8; ++q8) {  // 16-byte chunk 8 hf + q8 of the row, swizzled
        *reinterpret_cast<uint4*>(p_row + ((q8 ^ (row & 7)) << 4)) =
            make_uint4(pw[4 * q8], pw[4 * q8 + 1], pw[4 * q8 + 2], pw[4 * q8 + 3]);
        *reinterpret_cast<uint4*>(p_row_lo + ((q8 ^ (row & 7)) << 4)) =
            make_uint4(pl[4 * q8], pl[4 * q8 + 1], pl[4 * q8 + 2], pl[4 * q8 + 3]);
      }
      // (E) P(t) and the rescaled O are in place: the MMA warp may issue O += P(t) V(t)
      fence_proxy_async();
      tc_fence_before();
      mbar_arrive(&ctl.bar_e[b]);
    }
    // the last PV, then o = O / l for this thread's half-row; the halves' row sums meet in
    // the idle P_lo buffer
    wait(&ctl.bar_o, (unsigned)((n_kt - 1) & 1));
    tc_fence_after();
    float* lx = reinterpret_cast<float*>(gbase + 6 * kTileB);
    softmax_bar();  // every softmax warp is done reading P
    lx[hf * kPT + row] = l_half;
    softmax_bar();
    const float l = lx[row] + lx[kPT + row];
    const float inv = l > 0.f ? 1.f / l : 0.f;
    float* orow = a.o + (size_t)h * a.o_head_stride + (size_t)(i0 + row) * kD + 64 * hf;
    float ov[32];
#pragma unroll 1
    for (int c = 0; c < 2; ++c) {
      tmem_ld32(tO + lane_off + 64 * hf + 32 * c, ov);
      if (qp >= 0 && !ctl.failed) {
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4*>(orow + 32 * c + i) =
              make_float4(ov[i] * inv, ov[i + 1] * inv, ov[i + 2] * inv, ov[i + 3] * inv);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (ctl.failed) {
    // a wait ran out: record it, and give any MMA still in flight time to finish before
    // TMEM is released
    if (tid == 0) {
      if (a.status) record_error(a.status, FL_DEV_TIMEOUT, i0);
      const uint64_t t0 = global_ns();
      while (global_ns() - t0 < 2000000ull) __nanosleep(1000);
    }
    __syncthreads();
  }
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

}  // namespace

namespace {

// cuTensorMapEncodeTiled, fetched once from the driver through the runtime
// cuTensorMapEncodeTiled, fetched once from the driver through the runtime (a function-
// local static: initialised once even when several host threads arrive together)
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    return nullptr;
  }();
  return fn;
}

std::atomic<bool> g_attr_done[kMaxDevices];
std::mutex g_attr_mu;

// [heads][rows][128] BF16 (row stride 256 bytes, head stride head_stride elements) as a 3-D
// tensor map read in 64 x 128 boxes with the 128-byte swizzle; rows past `rows` read as 0
bool make_map(CUtensorMap* m, const uint16_t* base, int rows, int heads, int64_t head_stride) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
  if (!fn) return false;
  if (heads == 1 || head_stride < (int64_t)rows * kD) head_stride = (int64_t)rows * kD;  // unused with one head
  const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)rows, (cuuint64_t)heads};
  const cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)head_stride * 2};
  const cuuint32_t box[3] = {64, (cuuint32_t)kPT, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_prefill_attn(const PrefillArgs& a, cudaStream_t s) {
  if (a.n_act == 0) return cudaSuccess;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, a.q, a.n_act, a.heads, a.q_head_stride) || !make_map(&mk, a.k, a.n_tokens, a.heads, a.kv_head_stride) ||
      !make_map(&mv, a.v, a.n_tokens, a.heads, a.kv_head_stride))
    return cudaErrorInvalidValue;
  const cudaError_t e = once_per_device(g_attr_done, g_attr_mu, [](int) {
    return cudaFuncSetAttribute(prefill_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kPrefillSmem);
  });
  if (e != cudaSuccess) return e;
  dim3 grid((a.n_act + kPT - 1) / kPT, a.heads);
  prefill_attn_kernel<<<grid, kPrefillThreads, kPrefillSmem, s>>>(a, mq, mk, mv);
  return cudaGetLastError();
}

}  // namespace fl
