// Sparse decode reader, staged form: loop-aware sparse attention over the selected
// columns S for loops r <= 8 of the codec variants (per-loop KIVI4 full state, INT2
// residuals); the method's 4-bit residual stores take the persistent reader
// (sparse_persist.cu).
//
// FlashLoop project page, "The Method", Step 02: a sparse loop recomputes attention
// only for the columns chosen from the preceding loop and keeps their global
// probability mass m; flozi guide "FlashLoop: store changes between repeated passes",
// section 3: the loop's output is a rank-K correction of the previous one:
//     o_r = u + m * softmax_S(q_r K_S^T / sqrt(d)) V_S,
//     u   = o_{r-1} - sum_{j in S} p~_j v_j      (v_j at the loop that last computed j),
// with m = sum_{j in S} p~_j.  u and m are formed from the rows this pass gathers
// anyway (a column's value at loop tag_j is a prefix of its rows at loop r).
//
// Work split: grid (splits, heads), three CTAs of 5 warps per SM.  The CTA copies its
// part of the gather plan (column, tag, stores, p~, residual slots; written by the
// selector) into shared memory; each warp walks its own run of columns span by span.
// A span is up to 32 consecutive columns, cut so that it holds at most kMaxRows rows
// and kMaxRecs key records.  Its rows are laid out store-major (the base rows of its
// columns, then their loop-2 rows, ...), so each store's rows meet their group records
// in order and a record shared by neighbouring rows is staged once.  Every row (128 B:
// key and value codes), its 8-byte value (scale, zero) pair and each distinct key
// record (512 B) is copied by the warp's lanes in cp.async pieces, one commit
// group per span, and a warp keeps up to kSlots spans in flight in its ring of shared
// memory (cp.async.wait_group parks the warp in hardware until its span has landed).
// Per span:
//   records -> 24-bit fixed-point query weights q_c s_c 2^E in byte limbs (in place);
//   keys    -> one logit part per row (8 rows per pass, a lane per row quarter, exact
//              dp4a dots), then each column sums its parts in store order;
//   softmax -> online, base-2, over the warp's columns; score and tag are spliced;
//   values  -> per-row weights 128 p s_h and 128 p~ s_h (the latter for rows within
//              the column's tag-loop prefix) accumulate two fp32 sums.
// BF16 tail columns are handled last from global memory.  Warps merge in shared memory,
// CTAs write (M, L, m, sum p v, sum p~ v) partials, and the last CTA of each head
// combines them (atomic ticket, no waiting).
//
// Codec variants (flozi guide, section 4: the "Per-loop KIVI4" row and the 2-bit row
// of Figure 5).  2-bit residual rows are 64 bytes (32 B key codes, 32 B value codes):
// they are staged in the first half of their 128-byte row slot and read through the
// 4-bit layout (codes 0..3).  With full-state stores a column's loop-r key and value
// are its store st = min(r, depth) alone and its tag-loop value the store min(tag, st):
// a span holds each column's row of store st and, when the tag-loop store differs, that
// store's row for its value half only (no key record, no key dot).
#include "flush.cuh"
#include "kernels.h"

namespace fl {
namespace {

constexpr int kW = 5;              // warps per CTA
constexpr int kNT = kW * 32;
constexpr int kCtaPerSm = 3;
constexpr int kStoresMax = 8;      // loops served
constexpr int kMaxRows = 52;       // rows per span
constexpr int kMaxRecs = 10;       // key records per span
constexpr int kSlotsS = 4;         // spans in flight per warp
constexpr int kPlanWords = 1024;   // plan words of one CTA
constexpr int kSmemCta = 76800;    // three CTAs per SM

struct SpanHdr {
  uint32_t bal[kStoresMax];        // columns with a row in store s+1
  int32_t rowbase[kStoresMax];     // first row of store s+1
  uint8_t row_col[kMaxRows], row_rec[kMaxRows], row_pin[kMaxRows], row_store[kMaxRows];
  int32_t first, ncol, nrows, nrecs, smax;
};
constexpr int kHdrS = (int)((sizeof(SpanHdr) + 15) / 16 * 16);

struct alignas(16) WarpCtlS {
  int32_t slot_off[kSlotsS];
  float2 wrow[kMaxRows][2];        // span being consumed: per row and half (wS, wU)
  float lr[kMaxRows];              // span being consumed: per-row logit parts
  const uint8_t* rec_src[kMaxRecs];  // span being issued: source of each key record
  const uint8_t* row_src[kMaxRows];  // span being issued: source of each row
};

struct alignas(16) CtaHdr {
  float q[kD];
  float mw[kW], lw[kW], msw[kW];
  int32_t last_cta;
  int32_t pad[3];
};

constexpr int kRingS =
    ((kSmemCta - (int)sizeof(CtaHdr) - kPlanWords * 4 - kW * (int)sizeof(WarpCtlS)) / kW) & ~15;
constexpr int kMaxSpanS = kHdrS + kMaxRows * 136 + 8 + kMaxRecs * 512;
static_assert(kRingS >= kMaxSpanS, "ring must hold the largest span");
static_assert(kRingS >= 2 * kW * kD * 4, "warp 0's ring holds the merge area");

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async8(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
// Wait until at most n of this thread's commit groups are pending (n = 0..3).
__device__ __forceinline__ void cp_async_wait(int n) {
  if (n <= 0) asm volatile("cp.async.wait_group 0;" ::: "memory");
  else if (n == 1) asm volatile("cp.async.wait_group 1;" ::: "memory");
  else if (n == 2) asm volatile("cp.async.wait_group 2;" ::: "memory");
  else asm volatile("cp.async.wait_group 3;" ::: "memory");
}

__device__ __forceinline__ unsigned lanes_below(int c) { return c >= 32 ? 0xffffffffu : ((1u << c) - 1u); }

__device__ __forceinline__ int scan_incl(int v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(kFull, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

constexpr uint8_t kValueOnly = 0xff;  // row_rec of a row staged for its value half only

// kFlush: the step also writes this loop's store of a full tail (fused flush);
// kCodec: FL_CODEC_* of the loop r >= 2 stores
template <bool kFlush, int kCodec>
__global__ void __launch_bounds__(kNT, kCtaPerSm) sparse_staged_kernel(ReaderArgs a) {
  using CT = CodecT<kCodec>;
  using RB = Rec<CT::kResBits>;
  constexpr bool kFullS = CT::kFullState;
  constexpr bool kPk = CT::kResBits == 2;
  extern __shared__ __align__(128) uint8_t smem[];
  CtaHdr& ch = *reinterpret_cast<CtaHdr*>(smem);
  int32_t* plan_s = reinterpret_cast<int32_t*>(smem + sizeof(CtaHdr));
  WarpCtlS* ctls = reinterpret_cast<WarpCtlS*>(smem + sizeof(CtaHdr) + kPlanWords * 4);
  uint8_t* rings = smem + sizeof(CtaHdr) + kPlanWords * 4 + kW * sizeof(WarpCtlS);

  const int h = blockIdx.y, split = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int qq = lane & 3, tr = lane >> 2;
  const CacheView& c = a.c;
  const int H = c.H, cap = c.cap, ncb = cap / kG, T = c.total_slots, r = a.r;
  const int n_q = a.n_q, N = a.n_q + a.n_tail, K = a.k_sel, ps = c.plan_stride;
  const unsigned lt = lanes_below(lane);

  const uint8_t* brec = arr<uint8_t>(c, A_BREC, a.layer) + (size_t)h * ncb * kRec;
  const uint8_t* rrec = arr<uint8_t>(c, A_RREC, a.layer) + (size_t)h * (T / kG) * RB::kBytes;
  uint16_t* tail_k = arr<uint16_t>(c, A_TAILK, a.layer) + ((size_t)(r - 1) * H + h) * kTail * kD;
  uint16_t* tail_v = arr<uint16_t>(c, A_TAILV, a.layer) + ((size_t)(r - 1) * H + h) * kTail * kD;
  const uint16_t* tail_v_all = arr<uint16_t>(c, A_TAILV, a.layer);
  float* score = arr<float>(c, A_SCORE, a.layer) + (size_t)h * cap;
  uint8_t* tag = arr<uint8_t>(c, A_TAG, a.layer) + (size_t)h * cap;
  const int32_t* plan_g = arr<int32_t>(c, A_PLAN, a.layer) + (size_t)h * c.max_select * ps;
  const bool has_new = a.k_new != nullptr;

  grid_dep_launch();
  const int k0 = (int)((long long)split * K / a.n_splits);
  const int k1 = (int)((long long)(split + 1) * K / a.n_splits);
  const int ncols = k1 - k0;

  // ---- prologue: q, the new tail row, the plan, the warps' barriers ----
  if (tid < kD) ch.q[tid] = __uint_as_float((uint32_t)a.q[(size_t)h * kD + tid] << 16) * kQScale;
  if (split == 0 && has_new && warp == 0) {
    const uint2* kn = reinterpret_cast<const uint2*>(a.k_new + (size_t)h * kD);
    const uint2* vn = reinterpret_cast<const uint2*>(a.v_new + (size_t)h * kD);
    reinterpret_cast<uint2*>(tail_k + (size_t)(a.n_tail - 1) * kD)[lane] = kn[lane];
    reinterpret_cast<uint2*>(tail_v + (size_t)(a.n_tail - 1) * kD)[lane] = vn[lane];
  }
  for (int w = tid; w < ncols * ps; w += kNT) plan_s[w] = plan_g[(size_t)k0 * ps + w];
  WarpCtlS& wc = ctls[warp];
  uint8_t* ring = rings + (size_t)warp * kRingS;
  __syncthreads();

  // this warp's columns (indices into plan_s); validate them, find where the tail starts
  const int wk0 = (int)((long long)warp * ncols / kW);
  const int wk1 = (int)((long long)(warp + 1) * ncols / kW);
  int wtail = wk1;
  for (int c0 = wk0; c0 < wk1; c0 += 32) {
    const int cc = c0 + lane;
    bool tailc = false;
    if (cc < wk1) {
      int32_t* e = plan_s + (size_t)cc * ps;
      const int j = e[0], st = (e[1] >> 8) & 0xff, lam = e[1] & 0xff;
      bool ok = j >= 0 && j < N && lam >= 1 && lam <= c.R;
      if (ok && j < n_q) {
        ok = st >= 1 && st <= r;
        for (int s = 2; ok && s <= st; ++s) ok = e[1 + s] >= 0 && e[1 + s] < T;
      } else if (ok) {
        ok = st == 0;
        tailc = true;
      }
      if (!ok) {  // skipped: no rows, no score, no weight
        record_error(c.status, FL_DEV_SEL_RANGE, j);
        e[0] = -1;
        e[1] = 0;
        e[2] = 0;
      }
    }
    const unsigned tb = __ballot_sync(kFull, tailc);
    if (tb && wtail == wk1) wtail = c0 + __ffs(tb) - 1;
  }
  __syncwarp();

  float M = -INFINITY, Ls = 0.f, msum = 0.f;
  float accS[8], accU[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) accS[k] = accU[k] = 0.f;
  // per-lane parts of the per-half constants of the S and U sums (summed over the warp
  // once, at the end); Ls and msum are per-lane parts too
  float kS0 = 0.f, kS1 = 0.f, kU0 = 0.f, kU1 = 0.f;
  const int w16 = lane & 15, par16 = lane >> 4, half = w16 >> 3;

  // record of column lane's row in store s (base block or residual group record)
  auto rec_of = [&](const int32_t* e, int s) { return s == 1 ? (e[0] >> 6) : (e[1 + s] >> 6); };

  int iss_pos = wk0, iss_seq = 0, con_seq = 0, wpos = 0;
  int f_ncol = 0, f_nrows = 0, f_nrecs = 0, f_smax = 0;  // a formed span waiting for ring space
  bool formed = false;
  while (true) {
    // ---- form and issue spans while a slot and ring space are free ----
    while (iss_pos < wtail && iss_seq - con_seq < kSlotsS) {
      const int cpos = iss_pos + lane;
      const bool in = cpos < wtail;
      const int32_t* e = plan_s + (size_t)(in ? cpos : iss_pos) * ps;
      const int st = in ? (e[1] >> 8) & 0xff : 0;
      // full-state: the store of the column's tag-loop value (== st: no extra row)
      const int sv = kFullS ? min(e[1] & 0xff, st) : 0;
      if (!formed) {
        const int smax = __reduce_max_sync(kFull, st);
        int nrec_c = 0;
        for (int s = 1; s <= smax; ++s) {
          const bool act = kFullS ? st == s : st >= s;  // rows with a key part
          const int g = act ? rec_of(e, s) : -1;
          const unsigned pb = __ballot_sync(kFull, act) & lt;
          const int gp = __shfl_sync(kFull, g, pb ? 31 - __clz(pb) : lane);
          if (act && (pb == 0u || gp != g)) ++nrec_c;
        }
        const int nrow_c = kFullS ? (st > 0) + (sv != st) : st;
        const int rows_i = scan_incl(nrow_c, lane), recs_i = scan_incl(nrec_c, lane);
        const unsigned over = __ballot_sync(kFull, in && (rows_i > kMaxRows || recs_i > kMaxRecs));
        f_ncol = min(32, wtail - iss_pos);
        if (over) f_ncol = __ffs(over) - 1;  // >= 1: one column has at most 8 rows and 8 records
        static_assert(kMaxRows >= kStoresMax && kMaxRecs >= kStoresMax, "a column fits one span");
        f_nrows = __shfl_sync(kFull, rows_i, f_ncol - 1);
        f_nrecs = __shfl_sync(kFull, recs_i, f_ncol - 1);
        f_smax = smax;
        formed = true;
      }
      const int ncol = f_ncol, nrows = f_nrows, nrecs = f_nrecs, smax = f_smax;
      const int szb = (nrows * 8 + 15) & ~15;
      const int need = kHdrS + nrows * 128 + szb + nrecs * 512;
      int start = -1;
      if (iss_seq == con_seq) {
        start = 0;
      } else {
        const int rp = wc.slot_off[con_seq % kSlotsS];
        if (wpos > rp) {
          if (wpos + need <= kRingS) start = wpos;
          else if (need <= rp) start = 0;
        } else if (wpos + need <= rp) {
          start = wpos;
        }
      }
      if (start < 0) break;
      formed = false;
      wpos = start + need;
      const int slot = iss_seq % kSlotsS;
      uint8_t* sp = ring + start;
      SpanHdr& hd = *reinterpret_cast<SpanHdr*>(sp);
      uint8_t* rows = sp + kHdrS;
      uint8_t* szs = rows + nrows * 128;
      uint8_t* recs = szs + szb;
      const bool mine = lane < ncol;
      if (lane == 0) {
        wc.slot_off[slot] = start;
        hd.first = iss_pos;
        hd.ncol = ncol;
        hd.nrows = nrows;
        hd.nrecs = nrecs;
        hd.smax = smax;
      }
      int rowbase = 0, recbase = 0, nbase = 0;  // nbase: rows of the base (store 1), first in the span
      for (int s = 1; s <= smax; ++s) {
        const bool kact = mine && (kFullS ? st == s : st >= s);  // key and value parts
        const bool act = kact || (kFullS && mine && s == sv);     // ... or the value part alone
        const int g = act ? rec_of(e, s) : -1;
        const unsigned b = __ballot_sync(kFull, act);
        unsigned pb = b & lt;
        if constexpr (kFullS) pb = __ballot_sync(kFull, kact) & lt;
        const int gp = __shfl_sync(kFull, g, pb ? 31 - __clz(pb) : lane);
        const bool isnew = kact && (pb == 0u || gp != g);
        const unsigned nb = __ballot_sync(kFull, isnew);
        if (lane == 0 && s <= kStoresMax) {
          hd.bal[s - 1] = b;
          hd.rowbase[s - 1] = rowbase;
        }
        if (act) {
          const int ri = rowbase + (kFullS ? __popc(b & lt) : __popc(pb));
          const int ki = recbase + __popc(nb & (lt | (1u << lane))) - 1;
          const int pin = s == 1 ? (e[0] & 63) : (e[1 + s] & 63);
          hd.row_col[ri] = (uint8_t)lane;
          hd.row_rec[ri] = kact ? (uint8_t)ki : kValueOnly;
          hd.row_pin[ri] = (uint8_t)pin;
          hd.row_store[ri] = (uint8_t)s;
          // the row's source (copied below by eight lanes at a time) and its value (scale,
          // zero) pair, issued by the column's lane
          if constexpr (kPk) {
            const uint8_t* base = s == 1 ? brec + (size_t)g * kRec : rrec + (size_t)g * RB::kBytes;
            wc.row_src[ri] = base + pin * (s == 1 ? 128 : RB::kRow);
            cp_async8(szs + ri * 8, base + (s == 1 ? kRecVsz : RB::kVsz) + pin * 8);
            if (isnew) wc.rec_src[ki] = base + (s == 1 ? kRecKsz : RB::kKsz);
          } else {
            const uint8_t* base = (s == 1 ? brec : rrec) + (size_t)g * kRec;
            wc.row_src[ri] = base + pin * 128;
            cp_async8(szs + ri * 8, base + kRecVsz + pin * 8);
            if (isnew) wc.rec_src[ki] = base + kRecKsz;
          }
        }
        rowbase += __popc(b);
        recbase += __popc(nb);
        if (s == 1) nbase = rowbase;
      }
      __syncwarp();
      // rows: eight lanes per 128-byte row, four rows per copy instruction (contiguous
      // pieces, so each instruction touches four lines rather than 32)
      for (int ri = lane >> 3; ri < nrows; ri += 4) {
        // 2-bit rows are 64 bytes; a value-only row needs its value half (bytes 64..127)
        if constexpr (kPk) {
          if ((lane & 7) >= 4 && ri >= nbase) continue;
        }
        if constexpr (kFullS) {
          if ((lane & 7) < 4 && hd.row_rec[ri] == kValueOnly) continue;
        }
        cp_async16(rows + ri * 128 + (lane & 7) * 16, wc.row_src[ri] + (lane & 7) * 16);
      }
      // key records: 32 pieces each, spread over the lanes
      for (int k = 0; k < nrecs; ++k) cp_async16(recs + k * 512 + lane * 16, wc.rec_src[k] + lane * 16);
      asm volatile("cp.async.commit_group;" ::: "memory");
      iss_pos += ncol;
      ++iss_seq;
    }
    if (con_seq == iss_seq) break;

    // ---- consume the oldest span ----
    cp_async_wait(iss_seq - con_seq - 1);
    __syncwarp();
    const int slot = con_seq % kSlotsS;
    uint8_t* sp = ring + wc.slot_off[slot];
    SpanHdr& hd = *reinterpret_cast<SpanHdr*>(sp);
    const int ncol = hd.ncol, nrows = hd.nrows, nrecs = hd.nrecs, smax = hd.smax;
    const uint8_t* rows = sp + kHdrS;
    const uint8_t* szs = rows + nrows * 128;
    uint8_t* recs = sp + kHdrS + nrows * 128 + ((nrows * 8 + 15) & ~15);
    const int nbase = smax >= 2 ? hd.rowbase[1] : nrows;  // rows of the base come first

    // records -> 24-bit fixed-point query weights in byte limbs, in place
    for (int k = 0; k < nrecs; ++k) record_to_limbs(reinterpret_cast<uint32_t*>(recs + k * 512), ch.q, lane);
    __syncwarp();
    // one logit part per row: exact dp4a dot of the row quarter with its record's limbs
#pragma unroll 2
    for (int p0 = 0; p0 < nrows; p0 += 8) {
      const int row = p0 + tr;
      bool act = row < nrows;
      int rid = act ? hd.row_rec[row] : 0;
      if constexpr (kFullS) {
        act = act && rid != kValueOnly;
        rid = act ? rid : 0;
      }
      const uint32_t* lim = reinterpret_cast<const uint32_t*>(recs + rid * 512);
      float d = 0.f;
      if (act) {
        uint32_t lw[24];
        load_limbs(lim, qq, lw);
        if constexpr (kPk) {
          const uint4 code = row >= nbase
                                 ? int2_to_nib(*reinterpret_cast<const uint2*>(rows + row * 128 + 8 * qq))
                                 : *reinterpret_cast<const uint4*>(rows + row * 128 + 16 * qq);
          d = limb_dot(code, lw) * pow2i(-(int)lim[kLimbE]);
        } else {
          d = limb_dot(*reinterpret_cast<const uint4*>(rows + row * 128 + 16 * qq), lw) * pow2i(-(int)lim[kLimbE]);
        }
      }
      d += __shfl_xor_sync(kFull, d, 1);
      d += __shfl_xor_sync(kFull, d, 2);
      if (act && qq == 0) wc.lr[row] = d + __uint_as_float(lim[kLimbC]);
    }
    __syncwarp();
    // columns: sum the parts in store order, online softmax, splice score and tag
    const int32_t* ec = plan_s + (size_t)(hd.first + (lane < ncol ? lane : 0)) * ps;
    const int j_c = ec[0], ls_c = ec[1];
    const int st_c = lane < ncol ? (ls_c >> 8) & 0xff : 0;
    const int lam_c = ls_c & 0xff;
    const float pt_c = lane < ncol ? __int_as_float(ec[2]) : 0.f;
    float l = 0.f;
    if constexpr (kFullS) {
      if (st_c > 0) l = wc.lr[hd.rowbase[st_c - 1] + __popc(hd.bal[st_c - 1] & lt)];
    } else {
      for (int s = 1; s <= smax; ++s)
        if (st_c >= s) l += wc.lr[hd.rowbase[s - 1] + __popc(hd.bal[s - 1] & lt)];
    }
    const bool in = st_c > 0;
    l = in ? l : -INFINITY;
    const float mb = warp_max(l);
    const float Mn = fmaxf(M, mb);
    const float al = Mn == -INFINITY ? 1.f : ex2(M - Mn);
    const float p = in ? ex2(l - Mn) : 0.f;
    Ls = Ls * al + p;
    msum += in ? pt_c : 0.f;
    M = Mn;
#pragma unroll
    for (int k = 0; k < 8; ++k) accS[k] *= al;
    kS0 *= al;
    kS1 *= al;
    if (in) {
      score[j_c] = l;
      tag[j_c] = (uint8_t)r;
    }
    // per-row value weights, lanes = rows
    {
      for (int row0 = 0; row0 < nrows; row0 += 32) {
        const int row = row0 + lane;
        const bool act = row < nrows;
        const int cc = act ? hd.row_col[row] : 0;
        float pc = __shfl_sync(kFull, p, cc);
        const float ptc = __shfl_sync(kFull, pt_c, cc);
        const int lamc = __shfl_sync(kFull, lam_c, cc);
        int stc = 0;
        if constexpr (kFullS) stc = __shfl_sync(kFull, st_c, cc);
        if (act) {
          const uint32_t* pr = reinterpret_cast<const uint32_t*>(szs + row * 8);
          const float2 z0 = unpack_sz(pr[0]), z1 = unpack_sz(pr[1]);
          float pu;
          if constexpr (kFullS) {
            const int rs = hd.row_store[row];
            pc = rs == stc ? pc : 0.f;               // the loop-r value: store st
            pu = rs == min(lamc, stc) ? ptc : 0.f;   // the tag-loop value: store min(tag, st)
          } else {
            pu = hd.row_store[row] <= lamc ? ptc : 0.f;  // the tag loop's rows: a prefix of the stores
          }
          const float wS0 = 128.f * (pc * z0.x), wS1 = 128.f * (pc * z1.x);
          const float wU0 = 128.f * (pu * z0.x), wU1 = 128.f * (pu * z1.x);
          wc.wrow[row][0] = make_float2(wS0, wU0);
          wc.wrow[row][1] = make_float2(wS1, wU1);
          kS0 += fmaf(pc, z0.y, -wS0);
          kS1 += fmaf(pc, z1.y, -wS1);
          kU0 += fmaf(pu, z0.y, -wU0);
          kU1 += fmaf(pu, z1.y, -wU1);
        }
      }
    }
    __syncwarp();
#pragma unroll 4
    for (int row = par16; row < nrows; row += 2) {
      uint32_t x;
      if constexpr (kPk) {
        x = row >= nbase
                ? int2_word(*reinterpret_cast<const uint32_t*>(rows + row * 128 + 32 + 4 * (w16 >> 1)), w16 & 1)
                : *reinterpret_cast<const uint32_t*>(rows + row * 128 + 64 + 4 * w16);
      } else {
        x = *reinterpret_cast<const uint32_t*>(rows + row * 128 + 64 + 4 * w16);
      }
      const float2 wgt = wc.wrow[row][half];
      const float x0 = nib16(x << 16), x1 = nib16(x << 12), x2 = nib16(x << 8), x3 = nib16(x << 4);
      const float x4 = nib16(x), x5 = nib16(x >> 4), x6 = nib16(x >> 8), x7 = nib16(x >> 12);
      accS[0] = fmaf(wgt.x, x0, accS[0]);
      accS[1] = fmaf(wgt.x, x1, accS[1]);
      accS[2] = fmaf(wgt.x, x2, accS[2]);
      accS[3] = fmaf(wgt.x, x3, accS[3]);
      accS[4] = fmaf(wgt.x, x4, accS[4]);
      accS[5] = fmaf(wgt.x, x5, accS[5]);
      accS[6] = fmaf(wgt.x, x6, accS[6]);
      accS[7] = fmaf(wgt.x, x7, accS[7]);
      accU[0] = fmaf(wgt.y, x0, accU[0]);
      accU[1] = fmaf(wgt.y, x1, accU[1]);
      accU[2] = fmaf(wgt.y, x2, accU[2]);
      accU[3] = fmaf(wgt.y, x3, accU[3]);
      accU[4] = fmaf(wgt.y, x4, accU[4]);
      accU[5] = fmaf(wgt.y, x5, accU[5]);
      accU[6] = fmaf(wgt.y, x6, accU[6]);
      accU[7] = fmaf(wgt.y, x7, accU[7]);
    }
    __syncwarp();
    ++con_seq;
  }

  // ---- BF16 tail columns of this warp, from global memory (at most 64 per head) ----
  for (int c0 = wtail; c0 < wk1; c0 += 8) {
    const int ci = c0 + (lane >> 2);
    const bool in = ci < wk1 && plan_s[(size_t)ci * ps] >= n_q;
    const int32_t* e = plan_s + (size_t)(in ? ci : wk0) * ps;
    const int j = e[0];
    float d = 0.f;
    if (in) {
      const uint16_t* row = (has_new && j == N - 1) ? a.k_new + (size_t)h * kD : tail_k + (size_t)(j - n_q) * kD;
      float qsr[32];
      load32(ch.q + 32 * qq, qsr);
      d = dot_bf16_32(row + 32 * qq, qsr);
    }
    d += __shfl_xor_sync(kFull, d, 1);
    d += __shfl_xor_sync(kFull, d, 2);
    const float l = in ? d : -INFINITY;
    const float mb = warp_max(l);
    const float Mn = fmaxf(M, mb);
    const float al = Mn == -INFINITY ? 1.f : ex2(M - Mn);
    const float p = in ? ex2(l - Mn) : 0.f;
    const float pt = in ? __int_as_float(e[2]) : 0.f;
    Ls = Ls * al + (qq == 0 ? p : 0.f);
    msum += qq == 0 ? pt : 0.f;
    M = Mn;
#pragma unroll
    for (int k = 0; k < 8; ++k) accS[k] *= al;
    kS0 *= al;
    kS1 *= al;
    if (in && qq == 0) {
      score[j] = l;
      tag[j] = (uint8_t)r;
    }
    for (int k = par16; k < 8; k += 2) {
      const int src = 4 * k;
      const float pk = __shfl_sync(kFull, p, src);
      const float tk = __shfl_sync(kFull, pt, src);
      const int jk = __shfl_sync(kFull, j, src);
      const bool ink = __shfl_sync(kFull, in ? 1 : 0, src) != 0;
      const int lk = __shfl_sync(kFull, e[1] & 0xff, src);
      if (!ink) continue;
      const uint16_t* vr = (has_new && jk == N - 1) ? a.v_new + (size_t)h * kD : tail_v + (size_t)(jk - n_q) * kD;
      const uint16_t* ur = tail_v_all + (((size_t)(lk - 1) * H + h) * kTail + (jk - n_q)) * kD;
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(vr) + w16);
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(ur) + w16);
      const float vv[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                           bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
      const float uv[8] = {bf16_lo(u.x), bf16_hi(u.x), bf16_lo(u.y), bf16_hi(u.y),
                           bf16_lo(u.z), bf16_hi(u.z), bf16_lo(u.w), bf16_hi(u.w)};
#pragma unroll
      for (int q8 = 0; q8 < 8; ++q8) {
        accS[q8] = fmaf(pk, vv[q8], accS[q8]);
        accU[q8] = fmaf(tk, uv[q8], accU[q8]);
      }
    }
  }

  // ---- merge the warps: lane (w16, parity) holds channels 8*w16..8*w16+7 ----
  Ls = warp_sum(Ls);
  msum = warp_sum(msum);
  kS0 = warp_sum(kS0);
  kS1 = warp_sum(kS1);
  kU0 = warp_sum(kU0);
  kU1 = warp_sum(kU1);
  // one lane of each (word, parity) pair carries the constants
  const float corrS = par16 == 0 ? (half ? kS1 : kS0) : 0.f;
  const float corrU = par16 == 0 ? (half ? kU1 : kU0) : 0.f;
  float outS[8], outU[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    outS[k] = accS[k] + corrS;
    outU[k] = accU[k] + corrU;
    outS[k] += __shfl_xor_sync(kFull, outS[k], 16);
    outU[k] += __shfl_xor_sync(kFull, outU[k], 16);
  }
  __syncthreads();  // every warp is done with its ring; warp 0's ring becomes the merge area
  float* redS = reinterpret_cast<float*>(rings);  // [kW][128]
  float* redU = redS + kW * kD;
  if (par16 == 0) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      redS[warp * kD + 8 * w16 + k] = outS[k];
      redU[warp * kD + 8 * w16 + k] = outU[k];
    }
  }
  if (lane == 0) {
    ch.mw[warp] = M;
    ch.lw[warp] = Ls;
    ch.msw[warp] = msum;
  }
  __syncthreads();
  grid_dep_wait();
  float* part = a.part + ((size_t)h * a.n_splits + split) * kPartStride;
  if (tid < kD) {
    float Mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < kW; ++w) Mx = fmaxf(Mx, ch.mw[w]);
    float Lt = 0.f, St = 0.f, Ut = 0.f, mt = 0.f;
#pragma unroll
    for (int w = 0; w < kW; ++w) {
      Ut += redU[w * kD + tid];
      mt += ch.msw[w];
      if (ch.mw[w] == -INFINITY) continue;
      const float e = ex2(ch.mw[w] - Mx);
      Lt = fmaf(ch.lw[w], e, Lt);
      St = fmaf(redS[w * kD + tid], e, St);
    }
    part[4 + tid] = St;
    part[4 + kD + tid] = Ut;
    if (tid == 0) {
      part[0] = Mx;
      part[1] = Lt;
      part[2] = mt;
    }
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) ch.last_cta = (atomicAdd(&a.counter[h], 1) == a.n_splits - 1);
  __syncthreads();
  if (ch.last_cta) {
    __threadfence();

    // ---- last CTA of the head: combine every split (partials first staged in shared
    //      memory with coalesced loads, so the combine waits for one round trip) ----
    const float* hp = a.part + (size_t)h * a.n_splits * kPartStride;
    const int nwords = a.n_splits * kPartStride;
    const bool staged = (size_t)nwords * sizeof(float) <= (size_t)kW * kRingS;
    float* stp = reinterpret_cast<float*>(rings);
    if (staged) {
      for (int i = tid; i < nwords; i += kNT) stp[i] = __ldcg(hp + i);
      __syncthreads();
    }
    auto ld = [&](int i) { return staged ? stp[i] : __ldcg(hp + i); };
    if (tid < kD) {
      float Mx = -INFINITY;
      for (int s = 0; s < a.n_splits; ++s) Mx = fmaxf(Mx, ld(s * kPartStride));
      float Lt = 0.f, St = 0.f, Ut = 0.f, mt = 0.f;
      for (int s = 0; s < a.n_splits; ++s) {
        const int pp = s * kPartStride;
        Ut += ld(pp + 4 + kD + tid);
        mt += ld(pp + 2);
        const float ms = ld(pp);
        if (ms == -INFINITY) continue;
        const float e = ex2(ms - Mx);
        Lt = fmaf(ld(pp + 1), e, Lt);
        St = fmaf(ld(pp + 4 + tid), e, St);
      }
      const float op = a.o_prev[(size_t)h * kD + tid];
      const float u = op - Ut;
      a.o[(size_t)h * kD + tid] = Lt > 0.f ? fmaf(mt, St / Lt, u) : u;
      arr<float>(c, A_UNSEL, a.layer)[(size_t)h * kD + tid] = u;
      if (tid == 0) {
        arr<float>(c, A_MASS, a.layer)[h] = mt;
        arr<float>(c, A_OFFSET, a.layer)[(size_t)h * kOffStride + r] = Mx + log2f(Lt) - log2f(mt);
        a.counter[h] = 0;
      }
    }
  }
  if constexpr (kFlush) {
    __syncthreads();  // the combine is done with shared memory
    flush_tail(a, blockIdx.y * gridDim.x + blockIdx.x, gridDim.x * gridDim.y, *reinterpret_cast<EncodeSmem*>(smem),
               tid, kNT);
  }
}

// Splits of the staged reader: one wave at kCtaPerSm CTAs per SM and >= ~32 columns per
// CTA, but never fewer than the plan needs (a CTA holds at most kPlanWords / plan_stride
// columns in shared memory).
int staged_splits(int heads, int k_sel, int ps, int sms) {
  const int per = kPlanWords / ps;                                 // plan entries a CTA can hold
  const int need = (k_sel + per - 1) / per;
  const int by_sms = (sms * kCtaPerSm) / heads;                  // one wave
  const int by_work = (k_sel + 31) / 32;                          // at least ~32 columns per CTA
  int s = by_sms < by_work ? by_sms : by_work;
  if (s < need) s = need;
  if (s < 1) s = 1;
  return s;
}

std::atomic<bool> g_attr_done[kMaxDevices];
std::mutex g_attr_mu;

}  // namespace

int sparse_cta_columns(int loops) {
  const int ps = (loops + 2 + 3) / 4 * 4;
  int cols = kPlanWords / ps;
  if (direct_cta_columns(loops) < cols) cols = direct_cta_columns(loops);
  return cols;
}

int sparse_launch_splits(int heads, int loops, int codec, int r, int k_sel, int sms, bool flush) {
  (void)flush;
  if (codec == FL_CODEC_RESIDUAL_INT4 && r <= kPersistMaxLoop) return persist_splits(k_sel, loops);
  if (r <= kStoresMax && sms > 0) {
    const int n = staged_splits(heads, k_sel, (loops + 2 + 3) / 4 * 4, sms);
    if (n <= kMaxSplits) return n;
  }
  return direct_splits(heads, k_sel, loops, sms > 0 ? sms : 148);
}

int workspace_splits(int loops, int max_select) {
  const int cols = sparse_cta_columns(loops);
  const int need = (max_select + cols - 1) / cols;
  return need > kMaxSplits ? need : kMaxSplits;
}

cudaError_t launch_sparse(ReaderArgs a, cudaStream_t s, bool chain) {
  if (a.c.codec == FL_CODEC_RESIDUAL_INT4 && a.r <= kPersistMaxLoop) {
    if (a.n_layers < 1) a.n_layers = 1;
    if (a.flush && a.n_layers == 1) a.flush_slot0s[0] = a.flush_slot0;
    return launch_sparse_persist(a, s, chain);
  }
  a.n_layers = 1;  // one layer per launch below
  const int sms = device_sms();
  const int n = sparse_launch_splits(a.c.H, a.c.R, a.c.codec, a.r, a.k_sel, sms, a.flush != 0);
  if (a.r > kStoresMax || sms == 0 || n > kMaxSplits) return launch_sparse_direct(a, s, chain);
  const cudaError_t e = once_per_device(g_attr_done, g_attr_mu, [](int) {
    for (auto k : {sparse_staged_kernel<false, FL_CODEC_FULL_INT4>, sparse_staged_kernel<false, FL_CODEC_RESIDUAL_INT2>}) {
      cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemCta);
      if (e != cudaSuccess) return e;
      e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  });
  if (e != cudaSuccess) return e;
  a.n_splits = n;
  dim3 grid(n, a.c.H);
  // the variants only (the method's 4-bit residuals went to the persistent reader above;
  // the variants never take the fused flush)
  auto kern = a.c.codec == FL_CODEC_FULL_INT4 ? sparse_staged_kernel<false, FL_CODEC_FULL_INT4>
                                              : sparse_staged_kernel<false, FL_CODEC_RESIDUAL_INT2>;
  return launch_pdl_if(chain, kern, grid, dim3(kNT), (size_t)kSmemCta, s, a);
}

}  // namespace fl
