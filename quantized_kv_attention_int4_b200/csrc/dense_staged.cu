// Dense decode reader, staged form: single-query attention of one loop r <= 3 over
// every column, with the block's bytes staged in shared memory by bulk copies.
//
// FlashLoop project page, "The Method": dense loops attend over all columns; a
// column's key/value in loop r is the loop-1 base plus its residuals of loops 2..r
// (Step 03), or the loop's BF16 tail row (flashloop 0.1.0 PyPI description,
// "Configuration and supported scope": 64-token BF16 tail).
//
// Grid: one persistent CTA per SM of kPairs teams of two warps.  The units of all heads
// (each head's 64-token blocks, then its tail unit) are numbered head-major and cut into
// one contiguous range per CTA (at most two heads per range); team p takes units p,
// p + kPairs, ... of its CTA's range and owns a ring of shared memory.  Its first warp
// stages into the ring, ahead of use, for each block, one span:
//   [0, 9216)   the block's base group record (one bulk copy);
//   per residual store s of loops 2..r, if the block has rows there: the rows' code
//               lines (128 B each, from one or two group records), then per group record
//               its key (scale, zero) record (512 B) and the value (scale, zero) words of
//               the rows (rounded out to an even slot so the copy is 16-byte aligned).
// The copies of one span complete on one mbarrier (kSlots per team, round robin).  The
// two warps of a team share each block (named barrier per team): warp h takes key rows
// 32h..32h+31 and alternate passes of residual rows, and the values of channel half h.
//
// Per block, all on the staged bytes:
//   keys    every key (scale, zero) record becomes 24-bit fixed-point query weights
//           Q_c = rint(q_c s_c 2^E) split into byte limbs; a code row is dotted with
//           them by dp4a (exact integer sums), then scaled by 2^-E, plus sum_c q_c z_c;
//           each residual row's part is added to the logit of its token in store order;
//   softmax p'_t = 2^(l_t - m_b) with m_b the block maximum (both warps, identically);
//           the running (M, L) and output are rescaled once per block;
//   values  row weights W = p' s_h of the warp's half h become 24-bit fixed point
//           numbers (E_h from the block's largest weight); the code words of four rows are
//           transposed by byte permutes into per-channel nibble quadruples and dotted
//           by dp4a with the four rows' weight limbs; plus Z_h = sum_t p'_t z_t,h.
// The tail unit reads its BF16 rows from global memory in fp32.
// Teams' partials merge per CTA; the last CTA of each head (atomic ticket) combines the
// CTA partials by log-sum-exp and writes o and offset[r] = M + log2 L.
//
// Codec variants (flozi guide, section 4: the "Per-loop KIVI4" row and the 2-bit row of
// Figure 5): 2-bit residual rows are staged as 64-byte lines and read through the 4-bit
// layout (codes 0..3); with full-state stores a token's key and value are those of its
// last store min(r, depth) alone: the block's base is not staged when every token has a
// loop-2 row, a residual row's logit replaces (not adds to) its token's, and base or
// residual rows of tokens that have a later store get zero value weight.
#include "flush.cuh"
#include "kernels.h"

namespace fl {
namespace {

constexpr int kPairs = 7;                        // teams of two warps per CTA
constexpr int kThreads = kPairs * 64;
constexpr int kSlots = 4;                        // staged blocks in flight per team
constexpr int kStores = 2;                       // residual stores staged (loops 2, 3)
constexpr int kMaxGroups = 16 + kStores * 16;    // 4-row weight groups of one block
constexpr int kSmemTotal = 232448;               // opt-in shared memory per CTA
constexpr int kHdr = 64 + 2 * kD * 4;            // flags + the CTA's two queries

struct alignas(16) TeamCtl {
  uint64_t bar[kSlots];
  int32_t slot_off[kSlots];
  int32_t slot_gs0[kSlots][kStores];
  unsigned long long slot_mk[kSlots][kStores];
  float lg[kG];                  // base logits of the block (tail unit: its logits)
  float rl[kStores][kG];         // residual logit part of each residual row
  float pw[kG];                  // tail unit: p'
  uint8_t tok[kStores][kG];      // token of each residual row
  uint4 wl[kMaxGroups][2];       // weight limbs (bytes 0, 1, 2 of four rows) per group, half
  float part0[2 + kD];           // (M, L, o) of the team's first head
  int32_t has[2];
  int32_t ok[2];                 // each warp's staged-block wait succeeded
};

constexpr int kRing = ((kSmemTotal - kHdr - kPairs * (int)sizeof(TeamCtl)) / kPairs) & ~15;
// largest span: base record + 2 stores x (64 code rows + 2 key records + 66 value words)
constexpr int kMaxSpan = kRec + kStores * (kG * 128 + 2 * 512 + (kG + 2) * 8);
static_assert(kRing >= kMaxSpan, "ring must hold the largest span");

// Geometry of one block's rows in one residual store, as staged in the span.
struct StoreGeom {
  int na, n1;          // rows, rows in the first group record
  int off_codes;       // code rows 0..na-1, kRow B each (rows past na read padding)
  int off_k0, off_k1;  // key (scale, zero) records, turned into limbs in place
  int off_v0, off_v1;  // value (scale, zero) words: row i of piece p at off_vp + (vskip_p + i) * 8
  int vskip0;
};

template <int kRow>
__device__ __forceinline__ int store_geom(unsigned long long mk, int gs0, int pos, StoreGeom& g) {
  g.na = __popcll(mk);
  g.n1 = 0;
  g.off_codes = g.off_k0 = g.off_k1 = g.off_v0 = g.off_v1 = pos;
  g.vskip0 = 0;
  if (g.na == 0) return pos;
  const int s0 = gs0 & 63;
  g.n1 = min(g.na, kG - s0);
  g.off_codes = pos;
  pos += g.na * kRow;
  g.off_k0 = pos;
  pos += 512;
  g.off_v0 = pos;
  g.vskip0 = s0 & 1;
  pos += (((s0 + g.n1 + 1) & ~1) - (s0 & ~1)) * 8;
  g.off_k1 = g.off_k0;
  g.off_v1 = g.off_v0;
  if (g.n1 < g.na) {
    const int n2 = g.na - g.n1;
    g.off_k1 = pos;
    pos += 512;
    g.off_v1 = pos;
    pos += ((n2 + 1) & ~1) * 8;
  }
  return pos;
}

// Bulk copies of one span (lane 0 only); `bytes` is the span size; the base record is
// staged when `base` (the residual stores' records have RB's geometry).
template <class RB>
__device__ __forceinline__ void issue_span(uint8_t* sp, const uint8_t* brec_b, const uint8_t* rrec,
                                           const StoreGeom* g, const int* gs0, int bytes, bool base, uint64_t* bar) {
  fence_proxy_async();
  mbar_expect_tx(bar, (unsigned)bytes);
  if (base) bulk_g2s(sp, brec_b, kRec, bar);
#pragma unroll
  for (int s = 0; s < kStores; ++s) {
    const StoreGeom& G = g[s];
    if (G.na == 0) continue;
    const int s0 = gs0[s] & 63;
    const uint8_t* R0 = rrec + (size_t)(gs0[s] >> 6) * RB::kBytes;
    bulk_g2s(sp + G.off_codes, R0 + s0 * RB::kRow, G.n1 * RB::kRow, bar);
    bulk_g2s(sp + G.off_k0, R0 + RB::kKsz, 512, bar);
    const int a0 = s0 & ~1, a1 = (s0 + G.n1 + 1) & ~1;
    bulk_g2s(sp + G.off_v0, R0 + RB::kVsz + a0 * 8, (a1 - a0) * 8, bar);
    if (G.n1 < G.na) {
      const int n2 = G.na - G.n1;
      const uint8_t* R1 = R0 + RB::kBytes;
      bulk_g2s(sp + G.off_codes + G.n1 * RB::kRow, R1, n2 * RB::kRow, bar);
      bulk_g2s(sp + G.off_k1, R1 + RB::kKsz, 512, bar);
      bulk_g2s(sp + G.off_v1, R1 + RB::kVsz, ((n2 + 1) & ~1) * 8, bar);
    }
  }
}

// CTA holding unit x when U units are cut into n contiguous ranges floor(cU/n).
__device__ __forceinline__ int cta_of(long long x, long long U, int n) {
  return (int)(((x + 1) * n + U - 1) / U) - 1;
}


__device__ __forceinline__ void pair_sync(int pair) {
  asm volatile("bar.sync %0, 64;" ::"r"(pair + 1) : "memory");
}

// kFlush: the step also writes this loop's store of a full tail (fused flush);
// kCodec: FL_CODEC_* of the loop r >= 2 stores
template <bool kFlush, int kCodec>
__global__ void __launch_bounds__(kThreads, 1) dense_staged_kernel(ReaderArgs a, int n_cta) {
  using CT = CodecT<kCodec>;
  using RB = Rec<CT::kResBits>;
  constexpr bool kFullS = CT::kFullState;
  constexpr bool kPk = CT::kResBits == 2;
  extern __shared__ __align__(128) uint8_t smem[];
  int* last = reinterpret_cast<int*>(smem);
  float* q_all = reinterpret_cast<float*>(smem + 64);
  TeamCtl* ctl = reinterpret_cast<TeamCtl*>(smem + kHdr);
  uint8_t* rings = smem + kHdr + kPairs * sizeof(TeamCtl);

  const CacheView& c = a.c;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int pair = warp >> 1, hw = warp & 1;          // team and this warp's value half
  const int qq = lane & 3, tr = lane >> 2;             // key mapping: row tr of 8, quarter qq
  const int w8 = lane & 7, g4 = lane >> 3;             // value mapping: word of the half, row group mod 4
  const int wv = 8 * hw + w8;                          // code word (channels 8 wv .. 8 wv + 7)
  const int H = c.H, cap = c.cap, ncb = cap / kG, T = c.total_slots, r = a.r;
  const int nb = a.n_q / kG, nbp = nb + 1;
  const long long U = (long long)H * nbp;
  const int cta = blockIdx.x;
  const int U0 = (int)((long long)cta * U / n_cta), U1 = (int)((long long)(cta + 1) * U / n_cta);
  const int h0 = U0 / nbp, h1 = (U1 - 1) / nbp;
  const int nst = r - 1;
  grid_dep_launch();

  for (int i = tid; i < 2 * kD; i += kThreads) {
    const int hh = h0 + i / kD;
    q_all[i] = hh <= h1 ? __uint_as_float((uint32_t)a.q[(size_t)hh * kD + (i % kD)] << 16) * kQScale : 0.f;
  }
  TeamCtl& w = ctl[pair];
  uint8_t* ring = rings + (size_t)pair * kRing;
  if (tid == 64 * pair) {
    for (int i = 0; i < kSlots; ++i) mbar_init(&w.bar[i], 1);
    fence_mbar_init();
    w.has[0] = w.has[1] = 0;
  }
  __syncthreads();

  const unsigned long long* mask = arr<unsigned long long>(c, A_MASK, a.layer);
  const int32_t* first = arr<int32_t>(c, A_FIRST, a.layer);
  const uint8_t* brec_l = arr<uint8_t>(c, A_BREC, a.layer);
  const uint8_t* rrec_l = arr<uint8_t>(c, A_RREC, a.layer);
  const int n_my = U1 - U0 > pair ? (U1 - U0 - pair + kPairs - 1) / kPairs : 0;
  const bool has_new = a.k_new != nullptr;

  // metadata window (producer warp): lane (k_off = lane >> 1, s = lane & 1) holds store 2+s
  // of unit iss_k + k_off
  const int ms = lane & 1;
  auto load_meta = [&](int k, unsigned long long& mk, int& g0) {
    mk = 0ull;
    g0 = 0;
    if (k < n_my && ms < nst) {
      const int u = U0 + pair + k * kPairs, b = u % nbp;
      if (b < nb) {
        const int rp = 2 + ms;
        mk = __ldg(mask + (size_t)rp * ncb + b);
        g0 = c.slot_base[rp] + __ldg(first + (size_t)rp * ncb + b);
      }
    }
  };
  unsigned long long m_mk = 0ull;
  int m_gs = 0;
  if (hw == 0) load_meta(lane >> 1, m_mk, m_gs);

  int iss_k = 0, iss_seq = 0, con_seq = 0, wpos = 0;
  bool failed = false;

  float acc[8];
  float M = -INFINITY, Ls = 0.f;
  int cur_hs = -1;

  // write this warp's half of the team's (M, L, o) for head slot hs
  auto flush = [&](int hs) {
    float* dst = hs == 0 ? w.part0 : reinterpret_cast<float*>(ring);
    float o8[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      o8[k] = acc[k] + __shfl_xor_sync(kFull, acc[k], 8);
      o8[k] += __shfl_xor_sync(kFull, o8[k], 16);
    }
    const float Lw = warp_sum(Ls);
    if (g4 == 0) {
#pragma unroll
      for (int k = 0; k < 8; ++k) dst[2 + 8 * wv + k] = o8[k];
    }
    if (hw == 0 && lane == 0) {
      dst[0] = M;
      dst[1] = Lw;
      w.has[hs] = 1;
    }
  };
  // merge one block's (max, per-lane sum, per-channel values) into the running state
  auto merge = [&](float mb, float bs, const float* val) {
    const float Mn = fmaxf(M, mb);
    const float ao = ex2(M - Mn), ab = ex2(mb - Mn);
    Ls = fmaf(Ls, ao, bs * ab);
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] = fmaf(acc[k], ao, ab * val[k]);
    M = Mn;
  };

  for (int k = 0; k < n_my; ++k) {
    pair_sync(pair);  // both warps are done with the previous unit: its span may be reused
    // ---- producer warp: issue spans while a slot and ring space are free ----
    if (hw == 0) {
      while (iss_k < n_my) {
        const int u = U0 + pair + iss_k * kPairs, b = u % nbp;
        if (b < nb) {
          if (iss_seq - con_seq >= kSlots) break;
          unsigned long long mk2[kStores];
          int gs[kStores];
          mk2[0] = __shfl_sync(kFull, m_mk, 0);
          mk2[1] = __shfl_sync(kFull, m_mk, 1);
          gs[0] = __shfl_sync(kFull, m_gs, 0);
          gs[1] = __shfl_sync(kFull, m_gs, 1);
          StoreGeom g[kStores];
          // full-state stores: no base when every token of the block has a loop-2 row
          const bool base = !kFullS || nst == 0 || mk2[0] != ~0ull;
          int pos = store_geom<RB::kRow>(mk2[0], gs[0], base ? kRec : 0, g[0]);
          pos = store_geom<RB::kRow>(mk2[1], gs[1], pos, g[1]);
          int start = -1;
          if (iss_seq == con_seq) {
            start = 0;
          } else {
            const int rp = w.slot_off[con_seq % kSlots];
            if (wpos > rp) {
              if (wpos + pos <= kRing) start = wpos;
              else if (pos <= rp) start = 0;
            } else if (wpos + pos <= rp) {
              start = wpos;
            }
          }
          if (start < 0) break;
          wpos = start + pos;
          const int slot = iss_seq % kSlots;
          __syncwarp();
          if (lane == 0) {
            w.slot_off[slot] = start;
            w.slot_mk[slot][0] = mk2[0];
            w.slot_mk[slot][1] = mk2[1];
            w.slot_gs0[slot][0] = gs[0];
            w.slot_gs0[slot][1] = gs[1];
            const int h = u / nbp;
            issue_span<RB>(ring + start, brec_l + ((size_t)h * ncb + b) * kRec,
                           rrec_l + (size_t)h * (T / kG) * RB::kBytes, g, gs, pos, base, &w.bar[slot]);
          }
          ++iss_seq;
        }
        ++iss_k;
        // slide the metadata window by one unit
        const unsigned lo_m = __shfl_down_sync(kFull, (unsigned)m_mk, 2);
        const unsigned hi_m = __shfl_down_sync(kFull, (unsigned)(m_mk >> 32), 2);
        m_gs = __shfl_down_sync(kFull, m_gs, 2);
        m_mk = ((unsigned long long)hi_m << 32) | lo_m;
        if (lane >= 30) load_meta(iss_k + 15, m_mk, m_gs);
      }
      __syncwarp();
    }

    const int u = U0 + pair + k * kPairs, h = u / nbp, b = u % nbp, hs = h - h0;
    if (hs != cur_hs) {
      if (cur_hs >= 0) flush(cur_hs);
      cur_hs = hs;
      M = -INFINITY;
      Ls = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    }
    const float* qh = q_all + hs * kD;
    float* score = arr<float>(c, A_SCORE, a.layer) + (size_t)h * cap;
    uint8_t* tag = arr<uint8_t>(c, A_TAG, a.layer) + (size_t)h * cap;

    if (b < nb) {
      // ================= staged block =================
      const int slot = con_seq % kSlots;
      const bool okw = __any_sync(kFull, mbar_wait(&w.bar[slot], (unsigned)(con_seq / kSlots) & 1u));
      if (lane == 0) w.ok[hw] = okw ? 1 : 0;
      uint8_t* sp = ring + w.slot_off[slot];
      StoreGeom g[kStores];
      const unsigned long long mkA = w.slot_mk[slot][0], mkB = w.slot_mk[slot][1];
      const bool base = !kFullS || nst == 0 || mkA != ~0ull;  // as the producer decided
      {
        const int pos = store_geom<RB::kRow>(mkA, w.slot_gs0[slot][0], base ? kRec : 0, g[0]);
        store_geom<RB::kRow>(mkB, w.slot_gs0[slot][1], pos, g[1]);
      }
      // full-state: the tokens whose last store in loop r is the base / staged store s
      const unsigned long long need_b = kFullS && nst >= 1 ? ~mkA : ~0ull;
      const unsigned long long need0 = kFullS && nst >= 2 ? mkA & ~mkB : mkA;
      const unsigned long long need1 = mkB;
      // ---- key limbs (warp 1: the base record and the token maps; warp 0, which also
      //      staged the spans: the residual records) ----
      if (hw == 1) {
        if (base) record_to_limbs(reinterpret_cast<uint32_t*>(sp + kRecKsz), qh, lane);
#pragma unroll
        for (int s = 0; s < kStores; ++s) {
          if (g[s].na == 0) continue;
          const unsigned long long mk = s == 0 ? mkA : mkB;
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int tt = lane + 32 * e;
            if ((mk >> tt) & 1ull) w.tok[s][__popcll(mk & ((1ull << tt) - 1ull))] = (uint8_t)tt;
          }
        }
      } else {
#pragma unroll
        for (int s = 0; s < kStores; ++s) {
          if (g[s].na == 0) continue;
          record_to_limbs(reinterpret_cast<uint32_t*>(sp + g[s].off_k0), qh, lane);
          if (g[s].n1 < g[s].na) record_to_limbs(reinterpret_cast<uint32_t*>(sp + g[s].off_k1), qh, lane);
        }
      }
      pair_sync(pair);
      if (!(w.ok[0] && w.ok[1])) {
        if (hw == 0 && lane == 0) record_error(c.status, FL_DEV_TIMEOUT, b);
        failed = true;
        break;
      }

      // ---- base logits: rows 32 hw .. 32 hw + 31 ----
      if (base) {
        const uint32_t* lim = reinterpret_cast<const uint32_t*>(sp + kRecKsz);
        uint32_t lw[24];
        load_limbs(lim, qq, lw);
        const float sc = pow2i(-(int)lim[kLimbE]);
        const float C = __uint_as_float(lim[kLimbC]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int t = 32 * hw + 8 * i + tr;
          const uint4 code = *reinterpret_cast<const uint4*>(sp + t * 128 + 16 * qq);
          float v = limb_dot(code, lw) * sc;
          v += __shfl_xor_sync(kFull, v, 1);
          v += __shfl_xor_sync(kFull, v, 2);
          if (qq == 0) w.lg[t] = v + C;
        }
      }
      // ---- residual logit parts, one per residual row (passes of 8 rows, alternating warps) ----
#pragma unroll
      for (int s = 0; s < kStores; ++s) {
        const StoreGeom& G = g[s];
        if (G.na == 0) continue;
        for (int i0 = 8 * hw; i0 < G.na; i0 += 16) {
          const int i = i0 + tr;
          const bool act = i < G.na;
          const int ii = act ? i : G.na - 1;
          const uint32_t* lim = reinterpret_cast<const uint32_t*>(sp + (ii < G.n1 ? G.off_k0 : G.off_k1));
          uint32_t lw[24];
          load_limbs(lim, qq, lw);
          uint4 code;
          if constexpr (kPk) code = int2_to_nib(*reinterpret_cast<const uint2*>(sp + G.off_codes + ii * 64 + 8 * qq));
          else code = *reinterpret_cast<const uint4*>(sp + G.off_codes + ii * 128 + 16 * qq);
          float v = limb_dot(code, lw) * pow2i(-(int)lim[kLimbE]);
          v += __shfl_xor_sync(kFull, v, 1);
          v += __shfl_xor_sync(kFull, v, 2);
          if (act && qq == 0) w.rl[s][i] = v + __uint_as_float(lim[kLimbC]);
        }
      }
      pair_sync(pair);

      // ---- block softmax (both warps, identically) ----
      float l0 = base ? w.lg[lane] : 0.f, l1 = base ? w.lg[lane + 32] : 0.f;
#pragma unroll
      for (int s = 0; s < kStores; ++s) {
        if (g[s].na == 0) continue;
        const unsigned long long mk = s == 0 ? mkA : mkB;
        if constexpr (kFullS) {  // the logit of the token's last store
          const unsigned long long nd = s == 0 ? need0 : need1;
          if ((nd >> lane) & 1ull) l0 = w.rl[s][__popcll(mk & ((1ull << lane) - 1ull))];
          if ((nd >> (lane + 32)) & 1ull) l1 = w.rl[s][__popcll(mk & ((1ull << (lane + 32)) - 1ull))];
        } else {
          if ((mk >> lane) & 1ull) l0 += w.rl[s][__popcll(mk & ((1ull << lane) - 1ull))];
          if ((mk >> (lane + 32)) & 1ull) l1 += w.rl[s][__popcll(mk & ((1ull << (lane + 32)) - 1ull))];
        }
      }
      if (a.keep && hw == 0) {
        score[(size_t)b * kG + lane] = l0;
        score[(size_t)b * kG + lane + 32] = l1;
        tag[(size_t)b * kG + lane] = (uint8_t)r;
        tag[(size_t)b * kG + lane + 32] = (uint8_t)r;
      }
      const float mb = warp_max(fmaxf(l0, l1));
      const float p0 = ex2(l0 - mb), p1 = ex2(l1 - mb);

      // ---- value weights of this warp's half: W = p' s as 24-bit fixed point ----
      const int pad0 = (g[0].na + 3) & ~3, pad1 = (g[1].na + 3) & ~3;
      const int nvr = kG + pad0 + pad1;
      float Wt[6];
      float zs = 0.f, mx = 0.f;
#pragma unroll
      for (int i = 0; i < 6; ++i) {
        Wt[i] = 0.f;
        if (32 * i >= nvr) break;
        const int v = lane + 32 * i;
        int tok = v, off = kRecVsz + v * 8;  // base rows: token v, (scale, zero) in the base record
        bool act = v < kG;
        if constexpr (kFullS) act = act && base && ((need_b >> v) & 1ull);
        if (v >= kG && v < nvr) {
          int vv = v - kG;
          const int s = vv >= pad0 ? 1 : 0;
          if (s) vv -= pad0;
          const int na = s ? g[1].na : g[0].na, n1 = s ? g[1].n1 : g[0].n1;
          if (vv < na) {
            act = true;
            tok = w.tok[s][vv];
            off = vv < n1 ? (s ? g[1].off_v0 : g[0].off_v0) + ((s ? g[1].vskip0 : g[0].vskip0) + vv) * 8
                          : (s ? g[1].off_v1 : g[0].off_v1) + (vv - n1) * 8;
            if constexpr (kFullS) act = (((s ? need1 : need0) >> tok) & 1ull) != 0;  // its last store
          }
        }
        // p' of the row's token sits in lane tok & 31 (p0 for tokens < 32, else p1)
        const float pa = __shfl_sync(kFull, p0, tok & 31), pb = __shfl_sync(kFull, p1, tok & 31);
        if (act) {
          const float p = tok < 32 ? pa : pb;
          const float2 e = unpack_sz(*reinterpret_cast<const uint32_t*>(sp + off + 4 * hw));
          Wt[i] = p * e.x;
          zs = fmaf(p, e.y, zs);
          mx = fmaxf(mx, Wt[i]);
        }
      }
      mx = warp_max(mx);
      zs = warp_sum(zs);
      const int E = mx > 0.f ? min(24 - exp_frexp(mx), 126) : 0;
      const float scw = pow2i(E);
#pragma unroll
      for (int i = 0; i < 6; ++i) {
        if (32 * i >= nvr) break;
        const int v = lane + 32 * i;
        const uint32_t Q = fix24(Wt[i], scw);
        // lane 4m gathers rows 4m..4m+3 and writes their three limb words
        const uint32_t Qb = __shfl_down_sync(kFull, Q, 1), Qc = __shfl_down_sync(kFull, Q, 2),
                       Qd = __shfl_down_sync(kFull, Q, 3);
        if ((lane & 3) == 0 && v < nvr) {
          const uint32_t A = __byte_perm(Q, Qb, 0x5140), B = __byte_perm(Qc, Qd, 0x5140);
          const uint32_t C = __byte_perm(Q, Qb, 0x7362), D = __byte_perm(Qc, Qd, 0x7362);
          w.wl[v >> 2][hw] = make_uint4(__byte_perm(A, B, 0x5410), __byte_perm(A, B, 0x7632),
                                        __byte_perm(C, D, 0x5410), 0u);
        }
      }
      __syncwarp();

      // ---- values of this warp's half: dp4a over transposed nibbles ----
      int a0[8], a1[8], a2[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) a0[i] = a1[i] = a2[i] = 0;
      if (base) {
        const uint8_t* vb = sp + 64 + 4 * wv;
#pragma unroll
        for (int kg = g4; kg < 16; kg += 4) {
          const uint8_t* rp = vb + kg * 512;
          v_group(*reinterpret_cast<const uint32_t*>(rp), *reinterpret_cast<const uint32_t*>(rp + 128),
                  *reinterpret_cast<const uint32_t*>(rp + 256), *reinterpret_cast<const uint32_t*>(rp + 384),
                  w.wl[kg][hw], a0, a1, a2);
        }
      }
#pragma unroll
      for (int s = 0; s < kStores; ++s) {
        const int ng = (s ? pad1 : pad0) >> 2;
        const int kb = 16 + (s ? (pad0 >> 2) : 0);
        if constexpr (kPk) {  // 64-byte rows: value word wv / 2, its half wv % 2
          const uint8_t* vb = sp + (s ? g[1].off_codes : g[0].off_codes) + 32 + 4 * (wv >> 1);
          const int up = wv & 1;
          for (int kg = g4; kg < ng; kg += 4) {
            const uint8_t* rp = vb + kg * 256;
            v_group(int2_word(*reinterpret_cast<const uint32_t*>(rp), up),
                    int2_word(*reinterpret_cast<const uint32_t*>(rp + 64), up),
                    int2_word(*reinterpret_cast<const uint32_t*>(rp + 128), up),
                    int2_word(*reinterpret_cast<const uint32_t*>(rp + 192), up), w.wl[kb + kg][hw], a0, a1, a2);
          }
        } else {
          const uint8_t* vb = sp + (s ? g[1].off_codes : g[0].off_codes) + 64 + 4 * wv;
          for (int kg = g4; kg < ng; kg += 4) {
            const uint8_t* rp = vb + kg * 512;
            v_group(*reinterpret_cast<const uint32_t*>(rp), *reinterpret_cast<const uint32_t*>(rp + 128),
                    *reinterpret_cast<const uint32_t*>(rp + 256), *reinterpret_cast<const uint32_t*>(rp + 384),
                    w.wl[kb + kg][hw], a0, a1, a2);
          }
        }
      }
      const float isc = pow2i(-E);
      const float zh = g4 == 0 ? zs : 0.f;
      float val[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        val[i] = fmaf(fmaf((float)a2[i], 65536.f, fmaf((float)a1[i], 256.f, (float)a0[i])),
                      (i & 1) ? isc * 0.0625f : isc, zh);
      merge(mb, p0 + p1, val);
      fence_proxy_async();  // this span's generic reads and writes precede its reuse by bulk copies
      ++con_seq;
    } else {
      // ================= BF16 tail unit (global loads) =================
      const int nt = a.n_tail;
      uint16_t* tail_k = arr<uint16_t>(c, A_TAILK, a.layer) + ((size_t)(r - 1) * H + h) * kTail * kD;
      uint16_t* tail_v = arr<uint16_t>(c, A_TAILV, a.layer) + ((size_t)(r - 1) * H + h) * kTail * kD;
      const uint16_t* kn = has_new ? a.k_new + (size_t)h * kD : nullptr;
      const uint16_t* vn = has_new ? a.v_new + (size_t)h * kD : nullptr;
      if (has_new && hw == 0) {
        reinterpret_cast<uint2*>(tail_k + (size_t)(nt - 1) * kD)[lane] = reinterpret_cast<const uint2*>(kn)[lane];
        reinterpret_cast<uint2*>(tail_v + (size_t)(nt - 1) * kD)[lane] = reinterpret_cast<const uint2*>(vn)[lane];
      }
      float qsr[32];
      load32(qh + 32 * qq, qsr);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int t = 32 * hw + 8 * i + tr;
        const bool act = t < nt;
        float p = 0.f;
        if (act) {
          const uint16_t* row = (has_new && t == nt - 1) ? kn : tail_k + (size_t)t * kD;
          p = dot_bf16_32(row + 32 * qq, qsr);
        }
        p += __shfl_xor_sync(kFull, p, 1);
        p += __shfl_xor_sync(kFull, p, 2);
        if (qq == 0) w.lg[t] = act ? p : -INFINITY;
      }
      pair_sync(pair);
      const float l0 = w.lg[lane], l1 = w.lg[lane + 32];
      if (a.keep && hw == 0) {
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
      const float p0 = mb == -INFINITY ? 0.f : ex2(l0 - mb), p1 = mb == -INFINITY ? 0.f : ex2(l1 - mb);
      if (hw == 0) {
        w.pw[lane] = p0;
        w.pw[lane + 32] = p1;
      }
      pair_sync(pair);
      if (mb != -INFINITY) {
        float val[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) val[i] = 0.f;
        for (int t = g4; t < nt; t += 4) {
          const uint16_t* row = (has_new && t == nt - 1) ? vn : tail_v + (size_t)t * kD;
          const uint4 x = __ldg(reinterpret_cast<const uint4*>(row) + wv);
          const float pt = w.pw[t];
          val[0] = fmaf(pt, bf16_lo(x.x), val[0]);
          val[1] = fmaf(pt, bf16_hi(x.x), val[1]);
          val[2] = fmaf(pt, bf16_lo(x.y), val[2]);
          val[3] = fmaf(pt, bf16_hi(x.y), val[3]);
          val[4] = fmaf(pt, bf16_lo(x.z), val[4]);
          val[5] = fmaf(pt, bf16_hi(x.z), val[5]);
          val[6] = fmaf(pt, bf16_lo(x.w), val[6]);
          val[7] = fmaf(pt, bf16_hi(x.w), val[7]);
        }
        merge(mb, p0 + p1, val);
      }
    }
  }

  if (failed) {
    // staged copies still in flight land before the ring is reused below
    for (int s = con_seq; s < iss_seq; ++s) mbar_wait(&w.bar[s % kSlots], (unsigned)(s / kSlots) & 1u);
    __syncwarp();
  }
  pair_sync(pair);  // both warps of the team are done with the ring
  if (cur_hs >= 0) flush(cur_hs);
  __syncthreads();
  grid_dep_wait();  // the previous reader's partials and tickets are final from here

  // ---- CTA partials per head, then the last CTA of each head combines ----
  for (int hs = 0; hs <= h1 - h0; ++hs) {
    const int h = h0 + hs;
    const int c_lo = cta_of((long long)h * nbp, U, n_cta);
    float* part = a.part + ((size_t)h * kMaxSplits + (cta - c_lo)) * kPartStride;
    if (tid < kD) {
      float Mx = -INFINITY;
      for (int v = 0; v < kPairs; ++v)
        if (ctl[v].has[hs]) {
          const float* src = hs == 0 ? ctl[v].part0 : reinterpret_cast<const float*>(rings + (size_t)v * kRing);
          Mx = fmaxf(Mx, src[0]);
        }
      float Lt = 0.f, ot = 0.f;
      for (int v = 0; v < kPairs; ++v)
        if (ctl[v].has[hs]) {
          const float* src = hs == 0 ? ctl[v].part0 : reinterpret_cast<const float*>(rings + (size_t)v * kRing);
          if (src[0] == -INFINITY) continue;
          const float e = ex2(src[0] - Mx);
          Lt = fmaf(src[1], e, Lt);
          ot = fmaf(src[2 + tid], e, ot);
        }
      part[4 + tid] = ot;
      if (tid == 0) {
        part[0] = Mx;
        part[1] = Lt;
      }
    }
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    for (int hs = 0; hs < 2; ++hs) {
      last[hs] = 0;
      if (hs > h1 - h0) continue;
      const int h = h0 + hs;
      const int n_parts = cta_of((long long)(h + 1) * nbp - 1, U, n_cta) - cta_of((long long)h * nbp, U, n_cta) + 1;
      last[hs] = atomicAdd(&a.counter[h], 1) == n_parts - 1;
    }
  }
  __syncthreads();
  for (int hs = 0; hs <= h1 - h0; ++hs) {
    if (!last[hs]) continue;
    __threadfence();
    const int h = h0 + hs;
    const int c_lo = cta_of((long long)h * nbp, U, n_cta);
    const int n_parts = cta_of((long long)(h + 1) * nbp - 1, U, n_cta) - c_lo + 1;
    // the CTA partials, staged in shared memory with coalesced loads (one round trip)
    const float* hp = a.part + (size_t)h * kMaxSplits * kPartStride;
    const int nwords = n_parts * kPartStride;
    const bool staged = (size_t)nwords * sizeof(float) <= (size_t)kPairs * kRing;
    float* stp = reinterpret_cast<float*>(rings);
    __syncthreads();  // the previous head's combine is done reading the staged partials
    if (staged) {
      for (int i = tid; i < nwords; i += kThreads) stp[i] = __ldcg(hp + i);
      __syncthreads();
    }
    auto ld = [&](int i) { return staged ? stp[i] : __ldcg(hp + i); };
    if (tid < kD) {
      float Mx = -INFINITY;
      for (int s = 0; s < n_parts; ++s) Mx = fmaxf(Mx, ld(s * kPartStride));
      float Lt = 0.f, ot = 0.f;
      for (int s = 0; s < n_parts; ++s) {
        const float m_s = ld(s * kPartStride);
        if (m_s == -INFINITY) continue;
        const float e = ex2(m_s - Mx);
        Lt = fmaf(ld(s * kPartStride + 1), e, Lt);
        ot = fmaf(ld(s * kPartStride + 4 + tid), e, ot);
      }
      a.o[(size_t)h * kD + tid] = ot / Lt;
      if (tid == 0) {
        arr<float>(c, A_OFFSET, a.layer)[(size_t)h * kOffStride + r] = Mx + log2f(Lt);
        a.counter[h] = 0;
      }
    }
  }
  if constexpr (kFlush) {
    __syncthreads();  // the combines above are done with the staged partials
    flush_tail(a, cta, n_cta, *reinterpret_cast<EncodeSmem*>(rings), tid, kThreads);
  }
}

std::atomic<bool> g_attr_done[kMaxDevices];
std::mutex g_attr_mu;

}  // namespace

cudaError_t launch_dense(ReaderArgs a, cudaStream_t s, bool chain) {
  const int sms = device_sms();
  const long long U = (long long)a.c.H * (a.n_q / kG + 1);
  long long n = sms < U ? sms : U;
  if (n < a.c.H) n = a.c.H;  // every CTA range then touches at most two heads
  if (a.r > 3 || sms == 0 || n > kMaxSplits) return launch_dense_direct(a, s);
  const cudaError_t e = once_per_device(g_attr_done, g_attr_mu, [](int) {
    for (auto k : {dense_staged_kernel<false, FL_CODEC_RESIDUAL_INT4>, dense_staged_kernel<true, FL_CODEC_RESIDUAL_INT4>,
                   dense_staged_kernel<false, FL_CODEC_FULL_INT4>, dense_staged_kernel<false, FL_CODEC_RESIDUAL_INT2>}) {
      const cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemTotal);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  });
  if (e != cudaSuccess) return e;
  a.n_splits = (int)n;
  auto kern = a.c.codec == FL_CODEC_FULL_INT4       ? dense_staged_kernel<false, FL_CODEC_FULL_INT4>
              : a.c.codec == FL_CODEC_RESIDUAL_INT2 ? dense_staged_kernel<false, FL_CODEC_RESIDUAL_INT2>
              : a.flush                             ? dense_staged_kernel<true, FL_CODEC_RESIDUAL_INT4>
                                                    : dense_staged_kernel<false, FL_CODEC_RESIDUAL_INT4>;
  return launch_pdl_if(chain, kern, dim3((int)n), dim3(kThreads), (size_t)kSmemTotal, s, a, (int)n);
}

}  // namespace fl
