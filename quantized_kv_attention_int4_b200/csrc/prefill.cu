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
// tile stays in shared memory; key tiles of 128 tokens stream through three buffers
// (fetched two tiles ahead) and value tiles through two (one tile ahead), by cp.async
// issued by the softmax warps, zero-filled past the end.  The MMA warp issues S = Q K^T
// (8 tcgen05.mma of M = N = 128, K = 16; BF16 operands from 128-byte-swizzled shared
// memory; fp32 accumulators in TMEM) one tile ahead into alternating TMEM buffers, and
// O += P V once P is written (V read MN-major).  Softmax warp w reads TMEM lanes
// 32 (w % 4) ..: its thread t owns query row 32 (w % 4) + t and the 64 columns of half
// w / 4 -- it masks, runs the online softmax in the base-2 domain, writes its half of P
// (BF16) to shared memory in the operand layout and rescales its half of the output row
// in TMEM.  The two sides hand over through mbarriers only (softmax threads arrive when
// their copies and P are in place; tcgen05.commit signals finished MMAs), so no CTA-wide
// barrier sits in the loop; every wait is bounded.
#include "kernels.h"

namespace fl {
namespace {

constexpr int kPT = 128;                      // queries per tile = keys per tile = head dim
constexpr int kTileB = kPT * kPT * 2;         // one 128 x 128 BF16 tile
constexpr int kSoftmaxThreads = 256;          // 8 softmax warps: TMEM lane group w % 4, column half w / 4
constexpr int kPrefillThreads = kSoftmaxThreads + 32;  // + one warp that issues the MMAs
constexpr int kTmemCols = 512;                // S buffers: columns 0..127, 128..255; O: 256..383
constexpr uint32_t kIdescS = (1u << 4) | (1u << 7) | (1u << 10) | ((kPT >> 3) << 17) | ((kPT >> 4) << 24);
constexpr uint32_t kIdescPV = kIdescS | (1u << 16);  // B (V) read MN-major

struct PrefillCtl {
  uint64_t bar_s[2], bar_o;      // tensor cores -> softmax warps (tcgen05.commit)
  uint64_t bar_a[2], bar_e[2];   // softmax warps -> MMA warp, one arrival per softmax thread
  uint32_t tmem;
  int32_t pmax;
  int32_t failed;                // a bounded wait ran out somewhere
  int32_t pad;
  float rmax[2][kPT];            // per column half: this tile's row maxima
};
// the control block, then 1024-byte-aligned tiles: Q, K[3], V[2], P
constexpr int kPrefillSmem = (int)sizeof(PrefillCtl) + 1023 + 7 * kTileB;

// Byte offset of 16-byte chunk c (0..15) of row r in a 128 x 128 BF16 tile: two 64-column
// blocks of 128 rows x 128 bytes (16 KB apart); within each 1024-byte group of 8 rows the
// chunk index is XOR-ed with (row mod 8) -- the 128-byte swizzle the descriptors name.
__device__ __forceinline__ uint32_t sw128(int r, int c) {
  return (uint32_t)((c >> 3) * 16384 + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

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

__device__ __forceinline__ void cp16_zfill(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0) : "memory");
}

// rows [row0, row0 + 128) of a BF16 [n][128] matrix into a swizzled tile (zero past n):
// thread t copies chunk t % 16 of rows t / 16 + 16 i (rows 16 apart keep their swizzle
// phase, so the shared-memory offset steps by 16 x 128 bytes)
__device__ __forceinline__ void load_tile(uint32_t tile, const uint16_t* src, int row0, int n, int tid) {
  constexpr int kRowsPer = kSoftmaxThreads / 16;
  const int r0 = tid >> 4, c = tid & 15;
  const uint32_t d0 = tile + sw128(r0, c);
  const uint16_t* s0 = src + (size_t)(row0 + r0) * kD + c * 8;
#pragma unroll
  for (int it = 0; it < kPT / kRowsPer; ++it) {
    const bool ok = row0 + r0 + kRowsPer * it < n;
    cp16_zfill(d0 + (uint32_t)(it * kRowsPer * 128), ok ? s0 + (size_t)it * kRowsPer * kD : src, ok);
  }
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

__global__ void __launch_bounds__(kPrefillThreads, 1) prefill_attn_kernel(PrefillArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  PrefillCtl& ctl = *reinterpret_cast<PrefillCtl*>(smem_raw);
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + (uint32_t)sizeof(PrefillCtl) + 1023u) & ~1023u;  // 1024-byte aligned tiles
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sQ = base;
  auto sK = [&](int t) { return base + (uint32_t)(1 + t % 3) * kTileB; };  // K(t): buffer t % 3
  auto sV = [&](int t) { return base + (uint32_t)(4 + (t & 1)) * kTileB; };  // V(t): buffer t % 2
  const uint32_t sP = base + 6u * kTileB;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool mma_warp = warp == kSoftmaxThreads / 32;
  const int grp = warp & 3, hf = (warp >> 2) & 1;
  const int row = 32 * grp + lane;  // a softmax thread's query row = its TMEM lane
  const int h = blockIdx.y, i0 = blockIdx.x * kPT;
  const uint16_t* qh = a.q + (size_t)h * a.q_head_stride;
  const uint16_t* kh = a.k + (size_t)h * a.kv_head_stride;
  const uint16_t* vh = a.v + (size_t)h * a.kv_head_stride;

  // the row's position (-1: a padding row or a bad position)
  int qp = -1;
  if (!mma_warp && i0 + row < a.n_act) {
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
    }
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

  if (mma_warp) {
    // ---- MMA warp: lane 0 issues; S(t+1) as soon as its key tile is in place, PV(t) once
    //      the softmax warps have written P(t) ----
    for (int t = 0; t < n_kt; ++t) {
      const int b = t & 1;
      wait(&ctl.bar_a[b], (unsigned)((t >> 1) & 1));
      tc_fence_after();
      if (lane == 0 && !failed) {
        for (int u = t == 0 ? 0 : t + 1; u <= t + 1 && u < n_kt; ++u) {
#pragma unroll
          for (int s = 0; s < kPT / 16; ++s) {
            const uint32_t off = (uint32_t)((s >> 2) * 16384 + (s & 3) * 32);
            mma_bf16(tS(u & 1), desc_k(sQ + off), desc_k(sK(u) + off), kIdescS, s > 0 ? 1u : 0u);
          }
          mma_commit(&ctl.bar_s[u & 1]);
        }
      }
      __syncwarp();
      wait(&ctl.bar_e[b], (unsigned)((t >> 1) & 1));
      tc_fence_after();
      if (lane == 0 && !failed) {
#pragma unroll
        for (int s = 0; s < kPT / 16; ++s) {
          const uint32_t off = (uint32_t)((s >> 2) * 16384 + (s & 3) * 32);
          mma_bf16(tO, desc_k(sP + off), desc_mn(sV(t) + (uint32_t)s * 2048u), kIdescPV,
                   (t > 0 || s > 0) ? 1u : 0u);
        }
        mma_commit(&ctl.bar_o);
      }
      __syncwarp();
    }
  } else if (n_kt > 0) {
    // ---- softmax warps ----
    const uint32_t lane_off = (uint32_t)(32 * grp) << 16;  // this warp's TMEM lanes
    const float kScale = 1.4426950408889634f * 0.08838834764831845f;  // log2(e) / sqrt(128)
    uint8_t* p_row = gbase + 6 * kTileB + hf * 16384 + row * 128;   // this thread's half-row of P
    // cp.async groups (committed in the same order by every softmax thread, empty ones
    // included): {Q, K(0), V(0)}, {K(1)}; then per tile t: {K(t+2)} in (A), {V(t+1)} in (D)
    load_tile(sQ, qh, i0, a.n_act, tid);
    load_tile(sK(0), kh, 0, a.n_tokens, tid);
    load_tile(sV(0), vh, 0, a.n_tokens, tid);
    asm volatile("cp.async.commit_group;" ::: "memory");
    if (n_kt > 1) load_tile(sK(1), kh, kPT, a.n_tokens, tid);
    asm volatile("cp.async.commit_group;" ::: "memory");
    float m_run = -INFINITY, l_half = 0.f;
    for (int t = 0; t < n_kt; ++t) {
      const int b = t & 1, j0 = t * kPT;
      // (A) this thread's part of K(t+1) (at t = 0 also Q, K(0)) has landed and S(t-1)
      //     is consumed: tell the MMA warp; fetch K(t+2) into the buffer S(t-1) used
      if (t == 0) asm volatile("cp.async.wait_group 0;" ::: "memory");
      else asm volatile("cp.async.wait_group 1;" ::: "memory");
      fence_proxy_async();
      tc_fence_before();
      mbar_arrive(&ctl.bar_a[b]);
      if (t + 2 < n_kt) load_tile(sK(t + 2), kh, j0 + 2 * kPT, a.n_tokens, tid);
      asm volatile("cp.async.commit_group;" ::: "memory");
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
      const float m_tile = mx * kScale;
      float alpha = 1.f;
      if (m_tile > m_run + 8.f) {  // also the first visible tile (m_run = -inf): alpha = 0
        alpha = ex2(m_run - m_tile);
        m_run = m_tile;
      }
      // weights (fp32 row sum in four partial sums; P rounded to BF16 for the tensor cores)
      float ls4[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t pw[32];
      if (full) {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float p0 = ex2(fmaf(sv[2 * e], kScale, -m_run)), p1 = ex2(fmaf(sv[2 * e + 1], kScale, -m_run));
          pw[e] = pack_bf16(p0, p1);
          ls4[e & 3] += p0 + p1;
        }
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int i = 2 * e;
          const float p0 = (c_own + i <= qp) ? ex2(fmaf(sv[i], kScale, -m_run)) : 0.f;
          const float p1 = (c_own + i + 1 <= qp) ? ex2(fmaf(sv[i + 1], kScale, -m_run)) : 0.f;
          pw[e] = pack_bf16(p0, p1);
          ls4[e & 3] += p0 + p1;
        }
      }
      l_half = fmaf(l_half, alpha, (ls4[0] + ls4[1]) + (ls4[2] + ls4[3]));

      // (D) PV(t-1) is complete: P may be overwritten, the output accumulator rescaled and
      //     V buffer (t+1) % 2 refilled
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
      for (int q8 = 0; q8 < 8; ++q8)  // 16-byte chunk 8 hf + q8 of the row (see sw128)
        *reinterpret_cast<uint4*>(p_row + ((q8 ^ (row & 7)) << 4)) =
            make_uint4(pw[4 * q8], pw[4 * q8 + 1], pw[4 * q8 + 2], pw[4 * q8 + 3]);
      if (t + 1 < n_kt) load_tile(sV(t + 1), vh, j0 + kPT, a.n_tokens, tid);
      asm volatile("cp.async.commit_group;" ::: "memory");
      // (E) V(t) has landed (the two newest groups may still be in flight), P(t) and the
      //     rescaled O are in place: the MMA warp may issue O += P(t) V(t)
      asm volatile("cp.async.wait_group 2;" ::: "memory");
      fence_proxy_async();
      tc_fence_before();
      mbar_arrive(&ctl.bar_e[b]);
    }
    // the last PV, then o = O / l for this thread's half-row; the halves' row sums meet in
    // the idle P buffer
    wait(&ctl.bar_o, (unsigned)((n_kt - 1) & 1));
    tc_fence_after();
    asm volatile("cp.async.wait_group 0;" ::: "memory");
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

cudaError_t launch_prefill_attn(const PrefillArgs& a, cudaStream_t s) {
  if (a.n_act == 0) return cudaSuccess;
  static bool attr_set[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    const cudaError_t e =
        cudaFuncSetAttribute(prefill_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kPrefillSmem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  dim3 grid((a.n_act + kPT - 1) / kPT, a.heads);
  prefill_attn_kernel<<<grid, kPrefillThreads, kPrefillSmem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace fl
