// Sparse prefill attention on the 5th-generation tensor cores (tcgen05, TMEM).
//
// FlashLoop project page, "The Method": in a token-sparse loop only the active tokens
// are recomputed (Step 01), and the selected tokens are gathered into compact buffers
// so that the work stays a regular GEMM (the paragraph after Step 03).  Here: the
// queries of the active tokens (compact, in token order) attend causally over every
// token's key and value of the loop:
//     o_i = softmax_{j <= pos_i}(q_i k_j^T / sqrt(128)) v_j.
//
// One CTA of 4 warps per (128 active queries, head).  The query tile stays in shared
// memory; key/value tiles of 128 tokens stream through it (cp.async, zero-filled past
// the end).  Per key tile one thread issues S = Q K^T as 8 tcgen05.mma (M = N = 128,
// K = 16, BF16 operands from 128-byte-swizzled shared memory, fp32 accumulator in
// TMEM); warp w reads TMEM lanes 32w..32w+31, so thread t owns query row t: it masks,
// runs the online softmax in the base-2 domain, writes P (BF16) back to shared memory
// in the operand layout and rescales its row of the output accumulator in TMEM; then
// O += P V as 8 more tcgen05.mma (V read MN-major).  Completion of each group of MMAs
// is signalled by tcgen05.commit on an mbarrier; every wait is bounded.
#include "kernels.h"

namespace fl {
namespace {

constexpr int kPT = 128;                      // queries per tile = keys per tile = head dim
constexpr int kTileB = kPT * kPT * 2;         // one 128 x 128 BF16 tile
constexpr int kPrefillThreads = 128;
constexpr int kTmemCols = 256;                // S: columns 0..127, O: 128..255
constexpr uint32_t kIdescS = (1u << 4) | (1u << 7) | (1u << 10) | ((kPT >> 3) << 17) | ((kPT >> 4) << 24);
constexpr uint32_t kIdescPV = kIdescS | (1u << 16);  // B (V) read MN-major

struct PrefillCtl {
  uint64_t bar_s, bar_o;
  uint32_t tmem;
  int32_t pad;
  int32_t qpos[kPT];
};
constexpr int kPrefillSmem = 4 * kTileB + (int)sizeof(PrefillCtl) + 1024;  // + alignment slack

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

// rows [row0, row0 + 128) of a BF16 [n][128] matrix into a swizzled tile (zero past n)
__device__ __forceinline__ void load_tile(uint32_t tile, const uint16_t* src, int row0, int n, int tid) {
#pragma unroll 4
  for (int it = 0; it < 16; ++it) {
    const int r = it * 8 + (tid >> 4), c = tid & 15;
    const bool ok = row0 + r < n;
    cp16_zfill(tile + sw128(r, c), src + (size_t)(ok ? row0 + r : 0) * kD + c * 8, ok);
  }
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&b);
}

__global__ void __launch_bounds__(kPrefillThreads, 1) prefill_attn_kernel(PrefillArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;               // 1024-byte aligned tiles
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sQ = base, sK = base + kTileB, sV = base + 2 * kTileB, sP = base + 3 * kTileB;
  uint8_t* gP = gbase + 3 * kTileB;
  PrefillCtl& ctl = *reinterpret_cast<PrefillCtl*>(gbase + 4 * kTileB);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int h = blockIdx.y, i0 = blockIdx.x * kPT;
  const uint16_t* qh = a.q + (size_t)h * a.q_head_stride;
  const uint16_t* kh = a.k + (size_t)h * a.kv_head_stride;
  const uint16_t* vh = a.v + (size_t)h * a.kv_head_stride;

  // this thread's query row and its position (-1: padding row or a bad position)
  int qp = -1;
  if (i0 + tid < a.n_act) {
    qp = __ldg(a.pos + i0 + tid);
    const bool bad_order = i0 + tid > 0 && __ldg(a.pos + i0 + tid - 1) >= qp;
    if (qp < 0 || qp >= a.n_tokens || bad_order) {
      if (a.status) record_error(a.status, bad_order ? FL_DEV_ROWS_ORDER : FL_DEV_ROWS_RANGE, qp);
      if (qp < 0 || qp >= a.n_tokens) qp = -1;
    }
  }
  ctl.qpos[tid] = qp;
  if (tid == 0) {
    mbar_init(&ctl.bar_s, 1);
    mbar_init(&ctl.bar_o, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&ctl.tmem)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  load_tile(sQ, qh, i0, a.n_act, tid);
  asm volatile("cp.async.commit_group;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem;
  const uint32_t tS = tmem, tO = tmem + kPT;
  const uint32_t lane_off = (uint32_t)(32 * warp) << 16;     // this warp's TMEM lanes

  int pmax = -1;  // the tile's last real position decides how many key tiles it needs
  for (int r = 0; r < kPT; ++r) pmax = max(pmax, ctl.qpos[r]);
  const int n_kt = pmax < 0 ? 0 : pmax / kPT + 1;
  const float kScale = 1.4426950408889634f * 0.08838834764831845f;  // log2(e) / sqrt(128)

  float m_run = -INFINITY, l_run = 0.f;
  unsigned ph_s = 0, ph_o = 0;
  bool ok = true;
  uint64_t* pend = nullptr;  // the barrier whose commit is still outstanding after a failed wait
  unsigned pend_ph = 0;
  for (int t = 0; t < n_kt; ++t) {
    const int j0 = t * kPT;
    load_tile(sK, kh, j0, a.n_tokens, tid);
    load_tile(sV, vh, j0, a.n_tokens, tid);
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    fence_proxy_async();  // this thread's shared-memory writes, before the tensor cores read them
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
#pragma unroll
      for (int s = 0; s < kPT / 16; ++s) {
        const uint32_t off = (uint32_t)((s >> 2) * 16384 + (s & 3) * 32);
        mma_bf16(tS, desc_k(sQ + off), desc_k(sK + off), kIdescS, s > 0 ? 1u : 0u);
      }
      mma_commit(&ctl.bar_s);
    }
    ok = __syncthreads_and(mbar_wait(&ctl.bar_s, ph_s));
    if (!ok) {
      pend = &ctl.bar_s;
      pend_ph = ph_s;
      break;
    }
    ph_s ^= 1u;
    tc_fence_after();

    // row max of this tile's visible keys (scores in the base-2 domain)
    float mx = -INFINITY;
    float sv[32];
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      tmem_ld32(tS + lane_off + 32 * c, sv);
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (j0 + 32 * c + i <= qp) mx = fmaxf(mx, sv[i] * kScale);
    }
    const float m_new = fmaxf(m_run, mx);
    const float alpha = m_new == -INFINITY ? 1.f : ex2(m_run - m_new);
    // P = 2^(s - m_new) on visible keys, rounded to BF16; the row sum uses the rounded values
    float lsum = 0.f;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      tmem_ld32(tS + lane_off + 32 * c, sv);
      uint32_t w[16];
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        const float p0 = (j0 + 32 * c + i <= qp) ? ex2(sv[i] * kScale - m_new) : 0.f;
        const float p1 = (j0 + 32 * c + i + 1 <= qp) ? ex2(sv[i + 1] * kScale - m_new) : 0.f;
        w[i >> 1] = pack_bf16(p0, p1);
        const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&w[i >> 1]);
        lsum += __low2float(b) + __high2float(b);
      }
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4)
        *reinterpret_cast<uint4*>(gP + sw128(tid, 4 * c + q4)) =
            make_uint4(w[4 * q4], w[4 * q4 + 1], w[4 * q4 + 2], w[4 * q4 + 3]);
    }
    l_run = l_run * alpha + lsum;
    m_run = m_new;
    if (t > 0 && __any_sync(kFull, alpha != 1.f)) {  // rescale the warp's rows of the output accumulator
      float ov[32];
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        tmem_ld32(tO + lane_off + 32 * c, ov);
#pragma unroll
        for (int i = 0; i < 32; ++i) ov[i] *= alpha;
        tmem_st32(tO + lane_off + 32 * c, ov);
      }
    }
    fence_proxy_async();  // P, written by this thread, before the tensor cores read it
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
#pragma unroll
      for (int s = 0; s < kPT / 16; ++s) {
        const uint32_t off = (uint32_t)((s >> 2) * 16384 + (s & 3) * 32);
        mma_bf16(tO, desc_k(sP + off), desc_mn(sV + (uint32_t)s * 2048u), kIdescPV, (t > 0 || s > 0) ? 1u : 0u);
      }
      mma_commit(&ctl.bar_o);
    }
    ok = __syncthreads_and(mbar_wait(&ctl.bar_o, ph_o));
    if (!ok) {
      pend = &ctl.bar_o;
      pend_ph = ph_o;
      break;
    }
    ph_o ^= 1u;
    tc_fence_after();
  }

  if (!ok) {
    if (tid == 0 && a.status) record_error(a.status, FL_DEV_TIMEOUT, i0);
    // a last bounded wait for the outstanding MMAs before TMEM is released
    mbar_wait(pend, pend_ph);
  } else if (n_kt > 0) {
    // o = O / l for this thread's row (every lane reads TMEM; padding rows store nothing)
    const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
    float* orow = a.o + (size_t)h * a.o_head_stride + (size_t)(i0 + tid) * kD;
    float ov[32];
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      tmem_ld32(tO + lane_off + 32 * c, ov);
      if (qp >= 0) {
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4*>(orow + 32 * c + i) =
              make_float4(ov[i] * inv, ov[i + 1] * inv, ov[i + 2] * inv, ov[i + 3] * inv);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
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
