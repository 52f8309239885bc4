// Sparse decode reader: loop-aware sparse attention over the selected columns S.
//
// FlashLoop project page, "The Method", Step 02: a sparse loop recomputes attention
// only for the columns chosen from the preceding loop and keeps their global
// probability mass m; flozi guide "FlashLoop: store changes between repeated passes",
// section 3: the loop's output is a rank-K correction of the previous one:
//     o_r = u + m * softmax_S(q_r K_S^T / sqrt(d)) V_S,
//     u   = o_{r-1} - sum_{j in S} p~_j v_j      (v_j at the loop that last computed j),
// with m = sum_{j in S} p~_j.  u and m are formed here from the rows this pass gathers
// anyway (a column's value at loop tag_j is a prefix of its rows at loop r), so the
// unselected columns are never touched.
//
// Work split: grid (splits, heads), 4 independent warps per CTA, each owning a
// contiguous run of S.  The CTA loads its gather plan (column, tag, p~, store count,
// residual slots; written by the selector) into shared memory once.  A warp walks its
// columns in chunks of 32 (one column per lane).  A chunk's rows are streamed through
// shared memory store by store (the base rows of its columns, then their loop-2
// residual rows, ...), double-buffered with 16-byte cp.async copies (one commit group
// per stage):
//   key stages:   the rows' 64-byte key halves plus the distinct key (scale, zero)
//                 records they need (at most 8; a store continues in the next stage
//                 when it needs more); records become pre-scaled fp32 query weights;
//                 each row adds its logit part to its column;
//   -> after the chunk's last key stage: online softmax (base-2) over its columns;
//   value stages: the rows' 64-byte value halves and (scale, zero) pairs; per-row
//                 weights p s and p~ s (the latter only for rows within the column's
//                 tag-loop prefix) accumulate into fp32.
// BF16 tail columns are handled last from global memory.  Warps merge in shared memory,
// CTAs write (M, L, m, sum p v, sum p~ v) partials, and the last CTA of each head
// combines them (atomic ticket, no waiting).
//
// Codec variants (flozi guide, section 4: the "Per-loop KIVI4" row and the 2-bit row
// of Figure 5): 2-bit residual rows are staged as 32-byte halves and read through the
// 4-bit layout (codes 0..3); with full-state stores a column's loop-r key/value is its
// store st = min(r, depth) alone and its value at its tag loop the store
// min(tag, st), so a key stage of store s holds the columns with st == s and a value
// stage the columns for which s is one of those two stores.
#include "flush.cuh"
#include "kernels.h"

namespace fl {
namespace {

constexpr int NWARP = 4;
constexpr int NT = NWARP * 32;
constexpr int CHUNK = 32;     // columns per chunk = most rows of one stage
constexpr int SRECS = 8;      // key records per key stage
constexpr int PLANW = 1024;   // plan words of one CTA held in shared memory

struct __align__(128) Stage {
  uint8_t code[CHUNK][64];        // key or value halves of the staged rows
  uint32_t rec[SRECS][kD];        // key stages: records -> fp32 weights;
                                  // value stages: [0] value sz pairs, [1..2] per-row weights
  float rec_c[SRECS];             // key records: additive constant sum_c (q_c z_c - qs'_c)
  const uint8_t* row_src[CHUNK];  // the row's 64-byte key or value half
  const uint8_t* sz_src[CHUNK];   // value stages: the 16-byte value sz pair holding the row
  const uint8_t* rec_src[SRECS];  // key stages: the records' key sz (512 bytes)
  uint8_t row_col[CHUNK], row_rec[CHUNK], row_par[CHUNK];
  int kind, tab, store, nrow, nrec, last, use_u;
};

struct ChunkTab {
  int start, ncol, smax;  // smax = most stores of any column
  int j[CHUNK], st[CHUNK], lam[CHUNK], ploc[CHUNK];
  float pt[CHUNK], l[CHUNK], p[CHUNK], pu[CHUNK];
};

struct WarpMem {
  Stage s[2];
  ChunkTab t[2];
};

struct __align__(128) Smem {
  WarpMem w[NWARP];
  int32_t plan[PLANW];
  float q[kD];
  float mw[NWARP], lw[NWARP], msw[NWARP];
  int last_cta;
};

struct Ctx {
  const uint8_t* brec;
  const uint8_t* rrec;
  int ps, r;
};

// Position of the walk: chunk table, phase (0 = keys, 1 = values), store, first column.
struct Cursor {
  int tab, phase, store, col;
};

// lanes = columns: fill chunk table `t` for columns [start, min(start + 32, end)).
__device__ void setup_chunk(ChunkTab& t, const Smem& sm, int start, int end, int ps, int lane) {
  const int c = start + lane;
  const bool have = c < end;
  int j = -1, st = 0, lam = 0;
  float pt = 0.f;
  if (have) {
    const int32_t* e = sm.plan + (size_t)c * ps;
    j = e[0];
    st = (e[1] >> 8) & 0xff;
    lam = e[1] & 0xff;
    pt = __int_as_float(e[2]);
  }
  t.j[lane] = j;
  t.st[lane] = st;
  t.lam[lane] = lam;
  t.pt[lane] = pt;
  t.l[lane] = 0.f;
  t.ploc[lane] = c;
  const int mx = __reduce_max_sync(kFull, st);
  if (lane == 0) {
    t.start = start;
    t.ncol = min(CHUNK, max(0, end - start));
    t.smax = mx;
  }
  __syncwarp();
}

__device__ __forceinline__ unsigned below(int c) { return c >= 32 ? 0xffffffffu : ((1u << c) - 1u); }

// Does a column with `st` stores and tag `lam` read a row of store s in a key (kind 0)
// or value (kind 1) stage?
template <int kCodec>
__device__ __forceinline__ bool uses_row(int kind, int s, int st, int lam) {
  if constexpr (CodecT<kCodec>::kFullState) return s == st || (kind == 1 && s == min(lam, st));
  else return st >= s;
}

// lanes = columns: lay out the stage of store `s` that starts at chunk column `c0`;
// returns the first column after it (32 when the store is done).
template <int kCodec>
__device__ int form_stage(Stage& sg, const ChunkTab& t, const Smem& sm, const Ctx& cx, int kind, int tab, int s,
                          int c0, int lane) {
  using RB = Rec<CodecT<kCodec>::kResBits>;
  const bool act = lane < t.ncol && uses_row<kCodec>(kind, s, t.st[lane], t.lam[lane]) && lane >= c0;
  const unsigned bal = __ballot_sync(kFull, act);
  int grp = 0, pos = 0;
  if (act) {
    if (s == 1) {
      grp = t.j[lane] >> 6;
      pos = t.j[lane] & 63;
    } else {
      const int slot = sm.plan[(size_t)t.ploc[lane] * cx.ps + 1 + s];
      grp = slot >> 6;
      pos = slot & 63;
    }
  }
  const uint8_t* recb = s == 1 ? cx.brec + (size_t)grp * kRec : cx.rrec + (size_t)grp * RB::kBytes;
  const int row_bytes = s == 1 ? 128 : RB::kRow;
  const unsigned lt = below(lane);
  const int row = __popc(bal & lt);
  int c_to = 32, nrec = 0;
  if (kind == 0) {
    // keys of one store group monotonically along the columns: a row needs a new
    // record unless the previous row of the stage uses the same one
    const unsigned prevs = bal & lt;
    const int prev = prevs ? 31 - __clz(prevs) : 0;
    const int gp = __shfl_sync(kFull, grp, prev);
    const bool isnew = act && (prevs == 0u || gp != grp);
    const unsigned nb = __ballot_sync(kFull, isnew);
    const int upto = __popc(nb & (lt | (1u << lane)));
    const unsigned over = __ballot_sync(kFull, act && upto > SRECS);
    if (over) c_to = __ffs(over) - 1;
    nrec = __popc(nb & below(c_to));
    if (act && lane < c_to) {
      sg.row_src[row] = recb + (size_t)pos * row_bytes;
      sg.row_rec[row] = (uint8_t)(upto - 1);
      if (isnew) sg.rec_src[upto - 1] = recb + (s == 1 ? kRecKsz : RB::kKsz);
    }
  } else if (act) {
    sg.row_src[row] = recb + (size_t)pos * row_bytes + row_bytes / 2;
    sg.sz_src[row] = recb + (s == 1 ? kRecVsz : RB::kVsz) + (size_t)(pos & ~1) * 8;
    sg.row_par[row] = (uint8_t)(pos & 1);
  }
  if (act && lane < c_to) sg.row_col[row] = (uint8_t)lane;
  const int nrow = __popc(bal & below(c_to));
  const bool uses_u = CodecT<kCodec>::kFullState ? s == min(t.lam[lane], t.st[lane]) : s <= t.lam[lane];
  const unsigned uball = __ballot_sync(kFull, act && uses_u);
  if (lane == 0) {
    sg.kind = kind;
    sg.tab = tab;
    sg.store = s;
    sg.nrow = nrow;
    sg.nrec = nrec;
    sg.last = kind == 0 && s == t.smax && (bal & ~below(c_to)) == 0u;
    sg.use_u = uball != 0u;
  }
  __syncwarp();
  return c_to;
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}

// Every lane issues its share of the stage's 16-byte asynchronous copies (one commit
// group per stage): 4 chunks per staged row (2 for a 2-bit row), 32 chunks per key
// record, and one value (scale, zero) pair per row.
template <int kCodec>
__device__ void issue_stage(Stage& sg, int lane) {
  const int nrow = sg.nrow, nrec = sg.nrec, kind = sg.kind;
  if (CodecT<kCodec>::kResBits == 2 && sg.store >= 2) {
    for (int t = lane; t < 2 * nrow; t += 32)
      cp_async16(&sg.code[t >> 1][16 * (t & 1)], sg.row_src[t >> 1] + 16 * (t & 1));
  } else {
    for (int t = lane; t < 4 * nrow; t += 32)
      cp_async16(&sg.code[t >> 2][16 * (t & 3)], sg.row_src[t >> 2] + 16 * (t & 3));
  }
  if (kind == 0) {
    for (int k = 0; k < nrec; ++k) cp_async16(&sg.rec[k][4 * lane], sg.rec_src[k] + 16 * lane);
  } else if (lane < nrow) {
    cp_async16(&sg.rec[0][4 * lane], sg.sz_src[lane]);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}

// kFlush: the step also writes this loop's store of a full tail (fused flush);
// kCodec: FL_CODEC_* of the loop r >= 2 stores
template <bool kFlush, int kCodec>
__global__ void __launch_bounds__(NT, 3) sparse_kernel(ReaderArgs a) {
  using CT = CodecT<kCodec>;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  const int h = blockIdx.y, split = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const CacheView& c = a.c;
  const int H = c.H, cap = c.cap, ncb = cap / kG, T = c.total_slots, r = a.r;
  const int n_q = a.n_q, N = a.n_q + a.n_tail, K = a.k_sel, ps = c.plan_stride;

  Ctx cx;
  cx.brec = arr<uint8_t>(c, A_BREC, a.layer) + (size_t)h * ncb * kRec;
  cx.rrec = arr<uint8_t>(c, A_RREC, a.layer) + (size_t)h * (T / kG) * Rec<CT::kResBits>::kBytes;
  cx.ps = ps;
  cx.r = r;
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

  // ---- prologue: q, the new tail row, the plan ----
  if (tid < kD) sm.q[tid] = __uint_as_float((uint32_t)a.q[(size_t)h * kD + tid] << 16) * kQScale;
  if (split == 0 && has_new && warp == 0) {
    const uint2* kn = reinterpret_cast<const uint2*>(a.k_new + (size_t)h * kD);
    const uint2* vn = reinterpret_cast<const uint2*>(a.v_new + (size_t)h * kD);
    reinterpret_cast<uint2*>(tail_k + (size_t)(a.n_tail - 1) * kD)[lane] = kn[lane];
    reinterpret_cast<uint2*>(tail_v + (size_t)(a.n_tail - 1) * kD)[lane] = vn[lane];
  }
  for (int w = tid; w < ncols * ps; w += NT) sm.plan[w] = plan_g[(size_t)k0 * ps + w];
  WarpMem& wm = sm.w[warp];
  __syncthreads();

  // this warp's columns; validate them, find where the BF16 tail columns start
  const int wk0 = (int)((long long)warp * ncols / NWARP);
  const int wk1 = (int)((long long)(warp + 1) * ncols / NWARP);
  int wtail = wk1;
  for (int c0 = wk0; c0 < wk1; c0 += 32) {
    const int cc = c0 + lane;
    bool tailc = false;
    if (cc < wk1) {
      int32_t* e = sm.plan + (size_t)cc * ps;
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
  float corrS = 0.f, corrU = 0.f;  // per-half constants (this lane's half)
  const int w16 = lane & 15, par16 = lane >> 4, half = w16 >> 3;

  // ---- quantised columns: chunk by chunk, store by store ----
  // settle: move `p` to the next stage position; false when the warp has nothing left.
  // A chunk with no rows never stages anything, so its table is reused at once;
  // otherwise the next chunk takes the other table, which no staged data refers to
  // any more (at most one stage is prefetched).
  auto settle = [&](Cursor& p) -> bool {
    while (true) {
      const ChunkTab& t = wm.t[p.tab];
      if (p.store <= t.smax && p.col < 32) {
        const bool act = lane < t.ncol && uses_row<kCodec>(p.phase, p.store, t.st[lane], t.lam[lane]) && lane >= p.col;
        const unsigned bal = __ballot_sync(kFull, act);
        if (bal) {
          p.col = __ffs(bal) - 1;
          return true;
        }
      }
      if (p.store < t.smax) {
        ++p.store;
        p.col = 0;
        continue;
      }
      if (p.phase == 0 && t.smax > 0) {
        p.phase = 1;
        p.store = 1;
        p.col = 0;
        continue;
      }
      const int nxt = t.start + t.ncol;
      if (nxt >= wtail) return false;
      const int nt = t.smax == 0 ? p.tab : (p.tab ^ 1);
      setup_chunk(wm.t[nt], sm, nxt, wtail, ps, lane);
      p = Cursor{nt, 0, 1, 0};
    }
  };

  int cur = 0;
  bool pending = false;
  Cursor pos{0, 0, 1, 0};
  if (wtail > wk0) {
    setup_chunk(wm.t[0], sm, wk0, wtail, ps, lane);
    if (settle(pos)) {
      pos.col = form_stage<kCodec>(wm.s[0], wm.t[pos.tab], sm, cx, pos.phase, pos.tab, pos.store, pos.col, lane);
      issue_stage<kCodec>(wm.s[0], lane);
      pending = true;
    }
  }
  while (pending) {
    Stage& sg = wm.s[cur];
    Stage& nx = wm.s[cur ^ 1];
    bool more = settle(pos);
    if (more) {
      pos.col = form_stage<kCodec>(nx, wm.t[pos.tab], sm, cx, pos.phase, pos.tab, pos.store, pos.col, lane);
      issue_stage<kCodec>(nx, lane);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncwarp();
    ChunkTab& t = wm.t[sg.tab];
    if (sg.kind == 0) {
      // records -> pre-scaled fp32 query weights, in place (one warp per record)
      for (int rr = 0; rr < sg.nrec; ++rr) {
        const float cst = group_weights_smem(sg.rec[rr], sm.q, lane);
        if (lane == 0) sg.rec_c[rr] = cst;
      }
      __syncwarp();
      // each row's logit part goes to its column (one row per column per stage)
#pragma unroll
      for (int k = 0; k < CHUNK / 8; ++k) {
        const int row = 8 * k + (lane >> 2), qq = lane & 3;
        if (8 * k >= sg.nrow) break;
        float d = 0.f;
        if (row < sg.nrow) {
          const int rid = sg.row_rec[row];
          float qsr[32];
          load32(reinterpret_cast<const float*>(sg.rec[rid]) + 32 * qq, qsr);
          const uint4 x = (CT::kResBits == 2 && sg.store >= 2)
                              ? int2_to_nib(*reinterpret_cast<const uint2*>(&sg.code[row][8 * qq]))
                              : *reinterpret_cast<const uint4*>(&sg.code[row][16 * qq]);
          d = dot32(x, qsr);
          if (qq == 0) d += sg.rec_c[rid];
        }
        d += __shfl_xor_sync(kFull, d, 1);
        d += __shfl_xor_sync(kFull, d, 2);
        if (row < sg.nrow && qq == 0) t.l[sg.row_col[row]] += d;
      }
      __syncwarp();
      // after the chunk's last key stage: online softmax over its columns, splice score/tag
      if (sg.last) {
        const bool in = lane < t.ncol && t.st[lane] > 0;
        const float l = in ? t.l[lane] : -INFINITY;
        const float mb = warp_max(l);
        const float Mn = fmaxf(M, mb);
        const float al = Mn == -INFINITY ? 1.f : ex2(M - Mn);
        const float p = in ? ex2(l - Mn) : 0.f;
        Ls = Ls * al + warp_sum(p);
        msum += warp_sum(in ? t.pt[lane] : 0.f);
        M = Mn;
        t.p[lane] = p;
        t.pu[lane] = in ? t.pt[lane] : 0.f;
        if (in) {
          score[t.j[lane]] = l;
          tag[t.j[lane]] = (uint8_t)r;
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) accS[k] *= al;
        corrS *= al;
        __syncwarp();
      }
    } else {
      // per-row weights, lanes = rows: for each half h, wS = 128 p s_h, wU = 128 p~ s_h
      // (p~ only when the store lies within the column's tag-loop prefix), and the
      // matching constants p z_h - wS, p~ z_h - wU, folded in once per stage
      float4* wrow = reinterpret_cast<float4*>(&sg.rec[1][0]);  // [CHUNK][2] = {wS, wU, -, -}
      {
        float cS0 = 0.f, cS1 = 0.f, cU0 = 0.f, cU1 = 0.f;
        if (lane < sg.nrow) {
          const uint32_t* pr = &sg.rec[0][4 * lane + 2 * sg.row_par[lane]];
          const float2 z0 = unpack_sz(pr[0]), z1 = unpack_sz(pr[1]);
          const int ci = sg.row_col[lane];
          float p = t.p[ci], pu;
          if constexpr (CT::kFullState) {
            p = sg.store == t.st[ci] ? p : 0.f;
            pu = sg.store == min(t.lam[ci], t.st[ci]) ? t.pu[ci] : 0.f;
          } else {
            pu = sg.store <= t.lam[ci] ? t.pu[ci] : 0.f;
          }
          const float wS0 = 128.f * (p * z0.x), wS1 = 128.f * (p * z1.x);
          const float wU0 = 128.f * (pu * z0.x), wU1 = 128.f * (pu * z1.x);
          wrow[2 * lane] = make_float4(wS0, wU0, 0.f, 0.f);
          wrow[2 * lane + 1] = make_float4(wS1, wU1, 0.f, 0.f);
          cS0 = fmaf(p, z0.y, -wS0);
          cS1 = fmaf(p, z1.y, -wS1);
          cU0 = fmaf(pu, z0.y, -wU0);
          cU1 = fmaf(pu, z1.y, -wU1);
        }
        cS0 = warp_sum(cS0);
        cS1 = warp_sum(cS1);
        cU0 = warp_sum(cU0);
        cU1 = warp_sum(cU1);
        if (par16 == 0) {  // one lane of each (word, parity) pair carries the constants
          corrS += half ? cS1 : cS0;
          corrU += half ? cU1 : cU0;
        }
      }
      __syncwarp();
      const bool packed = CT::kResBits == 2 && sg.store >= 2;  // 2-bit codes in the first 32 bytes
      if (sg.use_u) {
        for (int row = par16; row < sg.nrow; row += 2) {
          const uint32_t x = packed ? int2_word(*reinterpret_cast<const uint32_t*>(&sg.code[row][4 * (w16 >> 1)]), w16 & 1)
                                    : *reinterpret_cast<const uint32_t*>(&sg.code[row][4 * w16]);
          const float2 wgt = *reinterpret_cast<const float2*>(&wrow[2 * row + half]);
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
      } else {
        for (int row = par16; row < sg.nrow; row += 2) {
          const uint32_t x = packed ? int2_word(*reinterpret_cast<const uint32_t*>(&sg.code[row][4 * (w16 >> 1)]), w16 & 1)
                                    : *reinterpret_cast<const uint32_t*>(&sg.code[row][4 * w16]);
          const float ws = wrow[2 * row + half].x;
          accS[0] = fmaf(ws, nib16(x << 16), accS[0]);
          accS[1] = fmaf(ws, nib16(x << 12), accS[1]);
          accS[2] = fmaf(ws, nib16(x << 8), accS[2]);
          accS[3] = fmaf(ws, nib16(x << 4), accS[3]);
          accS[4] = fmaf(ws, nib16(x), accS[4]);
          accS[5] = fmaf(ws, nib16(x >> 4), accS[5]);
          accS[6] = fmaf(ws, nib16(x >> 8), accS[6]);
          accS[7] = fmaf(ws, nib16(x >> 12), accS[7]);
        }
      }
    }
    __syncwarp();
    cur ^= 1;
    pending = more;
  }

  // ---- BF16 tail columns of this warp, from global memory (at most 64 per head) ----
  for (int c0 = wtail; c0 < wk1; c0 += 8) {
    const int ci = c0 + (lane >> 2), qq = lane & 3;
    const bool in = ci < wk1 && sm.plan[(size_t)ci * ps] >= n_q;
    const int32_t* e = sm.plan + (size_t)(in ? ci : wk0) * ps;
    const int j = e[0];
    float d = 0.f;
    if (in) {
      const uint16_t* row = (has_new && j == N - 1) ? a.k_new + (size_t)h * kD : tail_k + (size_t)(j - n_q) * kD;
      float qsr[32];
      load32(sm.q + 32 * qq, qsr);
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
    Ls = Ls * al + warp_sum(qq == 0 ? p : 0.f);
    msum += warp_sum(qq == 0 ? pt : 0.f);
    M = Mn;
#pragma unroll
    for (int k = 0; k < 8; ++k) accS[k] *= al;
    corrS *= al;
    if (in && qq == 0) {
      score[j] = l;
      tag[j] = (uint8_t)r;
    }
    // values: lane (word w16, parity) walks the (up to 8) columns of this round
    for (int k = par16; k < 8; k += 2) {
      const int src = 4 * k;  // a lane of column k
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
  float outS[8], outU[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    outS[k] = accS[k] + corrS;
    outU[k] = accU[k] + corrU;
    outS[k] += __shfl_xor_sync(kFull, outS[k], 16);
    outU[k] += __shfl_xor_sync(kFull, outU[k], 16);
  }
  __syncthreads();  // every warp is done with its staging area; reuse it for the merge
  float* redS = reinterpret_cast<float*>(&sm.w[0].s[0].code[0][0]);  // [NWARP][128]
  float* redU = redS + NWARP * kD;
  if (par16 == 0) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      redS[warp * kD + 8 * w16 + k] = outS[k];
      redU[warp * kD + 8 * w16 + k] = outU[k];
    }
  }
  if (lane == 0) {
    sm.mw[warp] = M;
    sm.lw[warp] = Ls;
    sm.msw[warp] = msum;
  }
  __syncthreads();
  grid_dep_wait();  // the previous reader's partials, tickets and outputs are final from here
  float* part = a.part + ((size_t)h * a.n_splits + split) * kPartStride;
  if (tid < kD) {
    float Mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < NWARP; ++w) Mx = fmaxf(Mx, sm.mw[w]);
    float Lt = 0.f, St = 0.f, Ut = 0.f, mt = 0.f;
#pragma unroll
    for (int w = 0; w < NWARP; ++w) {
      Ut += redU[w * kD + tid];
      mt += sm.msw[w];
      if (sm.mw[w] == -INFINITY) continue;
      const float e = ex2(sm.mw[w] - Mx);
      Lt = fmaf(sm.lw[w], e, Lt);
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
  if (tid == 0) sm.last_cta = (atomicAdd(&a.counter[h], 1) == a.n_splits - 1);
  __syncthreads();
  if (sm.last_cta) {
    __threadfence();

    // ---- last CTA of the head: combine every split ----
    if (tid < kD) {
      const float* hp = a.part + (size_t)h * a.n_splits * kPartStride;
      float Mx = -INFINITY;
      for (int s = 0; s < a.n_splits; ++s) Mx = fmaxf(Mx, __ldcg(hp + (size_t)s * kPartStride));
      float Lt = 0.f, St = 0.f, Ut = 0.f, mt = 0.f;
      for (int s = 0; s < a.n_splits; ++s) {
        const float* pp = hp + (size_t)s * kPartStride;
        Ut += __ldcg(pp + 4 + kD + tid);
        mt += __ldcg(pp + 2);
        const float ms = __ldcg(pp);
        if (ms == -INFINITY) continue;
        const float e = ex2(ms - Mx);
        Lt = fmaf(__ldcg(pp + 1), e, Lt);
        St = fmaf(__ldcg(pp + 4 + tid), e, St);
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
    flush_tail(a, blockIdx.y * gridDim.x + blockIdx.x, gridDim.x * gridDim.y, *reinterpret_cast<EncodeSmem*>(smem_raw),
               tid, NT);
  }
}

}  // namespace

// Splits of the direct reader: about one wave at 3 CTAs per SM and >= ~16 columns per
// CTA, but never fewer than the plan needs (a CTA holds at most PLANW / plan_stride
// columns), so no CTA's share of the plan overruns its shared-memory copy.
int direct_splits(int heads, int k_sel, int loops, int sms) {
  const int ps = (loops + 2 + 3) / 4 * 4;
  const int cmax = PLANW / ps;                    // plan entries a CTA can hold
  const int need = (k_sel + cmax - 1) / cmax;
  const int by_sms = (sms * 3) / heads;           // one wave at 3 CTAs per SM
  const int by_work = (k_sel + 15) / 16;          // at least ~16 columns per CTA
  int s = by_sms < by_work ? by_sms : by_work;
  if (s > kMaxSplits) s = kMaxSplits;
  if (s < need) s = need;
  if (s < 1) s = 1;
  return s;
}

int direct_cta_columns(int loops) { return PLANW / ((loops + 2 + 3) / 4 * 4); }

cudaError_t launch_sparse_direct(ReaderArgs a, cudaStream_t s, bool chain) {
  a.n_splits = direct_splits(a.c.H, a.k_sel, a.c.R, device_sms() > 0 ? device_sms() : 148);
  const bool flush = a.flush && a.c.codec == FL_CODEC_RESIDUAL_INT4;
  const size_t smem = flush && sizeof(EncodeSmem) > sizeof(Smem) ? sizeof(EncodeSmem) : sizeof(Smem);
  auto kern = a.c.codec == FL_CODEC_FULL_INT4       ? sparse_kernel<false, FL_CODEC_FULL_INT4>
              : a.c.codec == FL_CODEC_RESIDUAL_INT2 ? sparse_kernel<false, FL_CODEC_RESIDUAL_INT2>
              : flush                               ? sparse_kernel<true, FL_CODEC_RESIDUAL_INT4>
                                                    : sparse_kernel<false, FL_CODEC_RESIDUAL_INT4>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.n_splits, a.c.H);
  return launch_pdl_if(chain, kern, grid, dim3(NT), smem, s, a);
}

}  // namespace fl
