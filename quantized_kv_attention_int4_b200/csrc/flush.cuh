// Fused decode-time KV update: the readers' tail flush.
//
// FlashLoop project page, "The Method", the paragraph after Step 03: the cross-loop KV
// update and its quantisation are fused into the attention kernel rather than run as
// separate cache-update and quantise launches.  Here, in the decode step whose
// BF16 tail holds a full group of 64 rows, the reader of loop r attends over the tail
// as usual and then writes store r of that group: the base record for r = 1 (FlashLoop
// project page, "The Method", Step 03: loop-1 K/V are the base), the residual record of
// the rows active in loop r otherwise (residuals for active tokens only).  The bytes
// are the ones the separate base / residual encoders write for the same rows: the same
// quantiser routines, in the same order.
#pragma once

#include "kernels.h"
#include "quant.cuh"

namespace fl {

// Store a.r of the 64 tail rows [a.n_q, a.n_q + 64) of layer a.layer.  Work unit
// u = 8 h + 4 part + quarter of head h: keys (part 0) take channels [32 quarter,
// 32 quarter + 32) of all 64 slots, values (part 1) slots [16 quarter, 16 quarter + 16)
// with all 128 channels, so that each unit holds whole quantisation groups.  CTA `cta`
// of `n_cta` takes units cta, cta + n_cta, ...; CTA 0 also writes the group's mask /
// first-slot / depth entries.  Must run after the kernel's dependent-launch wait: store
// r is a residual against the records that the readers of loops 1 .. r - 1 wrote
// earlier in the step.  The new token (tail row 63) comes from k_new / v_new when the
// step supplies it, since the tail copy of that row is written by another CTA of this
// same launch.
// The same for layer `layer` with its group's first slot `slot0` and its new token's
// key / value rows k_new / v_new (a launch over several layers).
static __device__ __forceinline__ void flush_tail_layer(const ReaderArgs& a, int layer, int slot0,
                                                        const uint16_t* k_new, const uint16_t* v_new, int cta,
                                                        int n_cta, EncodeSmem& sm, int tid, int nt) {
  const CacheView& c = a.c;
  const int r = a.r, H = c.H, ncb = c.cap / kG, T = c.total_slots, gb = a.n_q / kG;
  const unsigned long long act = r == 1 ? ~0ull : a.flush_act;
  const int nr = __popcll(act);
  uint8_t* depth = arr<uint8_t>(c, A_DEPTH, layer);
  unsigned long long* mask = arr<unsigned long long>(c, A_MASK, layer);
  int32_t* first = arr<int32_t>(c, A_FIRST, layer);

  // store r is a residual against stores 1 .. r - 1 of the same rows: those flushes must
  // have run (loops in order); otherwise record the error and write nothing
  bool bad = false;
  if (r == 2) {
    for (int t = tid; t < kG; t += nt)
      if (((act >> t) & 1ull) && __ldcg(depth + a.n_q + t) < 1) bad = true;
  } else if (r >= 3) {
    bad = (act & ~__ldcg(mask + (size_t)(r - 1) * ncb + gb)) != 0ull;
  }
  if (__syncthreads_or(bad)) {
    if (cta == 0 && tid == 0) record_error(c.status, FL_DEV_NOT_NESTED, a.n_q);
    return;
  }

  if (cta == 0) {
    if (r == 1) {
      for (int t = tid; t < kG; t += nt) depth[a.n_q + t] = 1;
      for (int rp = 2 + tid; rp <= c.R; rp += nt) {
        mask[(size_t)rp * ncb + gb] = 0ull;
        first[(size_t)rp * ncb + gb] = -1;
      }
    } else {
      for (int t = tid; t < kG; t += nt)
        if ((act >> t) & 1ull) depth[a.n_q + t] = (uint8_t)r;
      if (tid == 0) {
        mask[(size_t)r * ncb + gb] = act;
        first[(size_t)r * ncb + gb] = nr ? slot0 : -1;
      }
    }
  }
  if (nr == 0 || cta >= 8 * H) return;

  // slot -> tail row, and where the block's rows sit in stores 2 .. r - 1
  for (int t = tid; t < kG; t += nt)
    if ((act >> t) & 1ull) sm.row[__popcll(act & ((1ull << t) - 1ull))] = t;
  for (int rp = 2 + tid; rp < r; rp += nt) {
    sm.mk[rp] = __ldcg(mask + (size_t)rp * ncb + gb);
    sm.g0[rp] = c.slot_base[rp] + __ldcg(first + (size_t)rp * ncb + gb);
  }

  const uint8_t* brec_l = arr<uint8_t>(c, A_BREC, layer);
  const uint8_t* rrec_l = arr<uint8_t>(c, A_RREC, layer);
  for (int u = cta; u < 8 * H; u += n_cta) {
    const int h = u >> 3, qt = u & 3;
    const bool is_v = ((u >> 2) & 1) != 0;
    const uint8_t* bgrp = brec_l + ((size_t)h * ncb + gb) * kRec;
    const uint8_t* rrec = rrec_l + (size_t)h * (T / kG) * kRec;
    uint8_t* rec = const_cast<uint8_t*>(r == 1 ? bgrp : rrec + (size_t)((c.slot_base[r] + slot0) >> 6) * kRec);
    const uint16_t* src =
        arr<uint16_t>(c, is_v ? A_TAILV : A_TAILK, layer) + ((size_t)(r - 1) * H + h) * kTail * kD;
    const uint16_t* xnew = is_v ? v_new : k_new;
    if (xnew) xnew += (size_t)h * kD;

    __syncthreads();  // the row map is in place; the previous unit is done with shared memory
    // slot i < nr holds tail row row[i]: X (base) or E = X^(r) - X_hat^(r-1) (residual)
    for (int item = tid; item < 256; item += nt) {
      const int i = is_v ? 16 * qt + (item >> 4) : item >> 2;
      const int c8 = is_v ? 8 * (item & 15) : 32 * qt + 8 * (item & 3);
      float* xs = &sm.xs[i][c8];
      if (i >= nr) {
#pragma unroll
        for (int e = 0; e < 8; ++e) xs[e] = 0.f;
        continue;
      }
      const int t = sm.row[i];
      const uint16_t* rowp = (xnew && t == kTail - 1) ? xnew : src + (size_t)t * kD;
      float x[8];
      bf16x8(__ldcg(reinterpret_cast<const uint4*>(rowp + c8)), x);
      if (r == 1) {
#pragma unroll
        for (int e = 0; e < 8; ++e) xs[e] = x[e];
      } else {
        float xh[8];
        deq8<true>(bgrp, t, is_v, c8, xh);
        for (int rp = 2; rp < r; ++rp) {
          const int gs = sm.g0[rp] + __popcll(sm.mk[rp] & ((1ull << t) - 1ull));
          float d[8];
          deq8<true>(rrec + (size_t)(gs >> 6) * kRec, gs & 63, is_v, c8, d);
#pragma unroll
          for (int e = 0; e < 8; ++e) xh[e] = __fadd_rn(xh[e], d[e]);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) xs[e] = __fsub_rn(x[e], xh[e]);
      }
    }
    __syncthreads();
    if (is_v) value_params(sm, rec, 16 * qt, 16, nr, tid, nt);
    else key_params(sm, rec, 32 * qt, 32, nr, tid, nt);
    __syncthreads();
    if (is_v) group_codes(sm, rec, true, 16 * qt, 16, 0, kD / 8, nr, tid, nt);
    else group_codes(sm, rec, false, 0, kG, 4 * qt, 4, nr, tid, nt);
  }
}

// Store a.r of the 64 tail rows of layer a.layer (the one-layer launches).
static __device__ __forceinline__ void flush_tail(const ReaderArgs& a, int cta, int n_cta, EncodeSmem& sm, int tid,
                                                  int nt) {
  flush_tail_layer(a, a.layer, a.flush_slot0, a.k_new, a.v_new, cta, n_cta, sm, tid, nt);
}

}  // namespace fl
