// Sparse decode reader, persistent form: the method's 4-bit residual stores, loops r <= 8,
// every layer of a loop in one launch.
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
// Work: items of at most 2048 plan words of selected columns of one (layer, head) --
// (layer, head, split), layer-major -- taken by a resident grid (two CTAs per SM) in
// strides of the grid, so that one item's start-up (its plan, its first tables and
// copies) overlaps the previous item's work.  A CTA is one producer warp, two copy warps
// and eight consumer warps, handing batches on through mbarriers:
//   producer  copies an item's query and plan (two item slots), validates the entries,
//             and cuts the item into batches of at most 64 columns, 160 rows and 32 key
//             records, writing each batch's table (a ring of three): the rows laid out
//             store-major -- the base rows of its columns, then their loop-2 rows, ... --
//             so each store's rows meet their group records in order and a record shared
//             by neighbouring rows is staged once.  It runs up to two batches ahead.
//   copiers   (columns 0..31 and 32..63 of a batch) complete the table -- each row's
//             source, column, record and store, each column's rows -- and issue the 16-byte
//             cp.async pieces of their rows (key codes | value codes), the rows' 8-byte
//             value (scale, zero) pairs and the key records, into the buffer (two) that
//             the consumers left; the buffer's mbarrier completes once they land.
//   consumers (all eight warps on every phase, named barriers between) consume batch b:
//             records -> 24-bit fixed-point query weights in byte limbs (in place);
//             keys    -> one exact dp4a logit part per row (a lane per row quarter);
//             columns -> warp w sums the parts of columns 8 w .. 8 w + 7 in store order,
//                        splices score and tag; the running maximum (base 2) over the item
//                        is the same in every consumer thread;
//             weights -> per row and half: 128 p s and 128 p~ s (the latter for rows
//                        within the column's tag-loop prefix); a column's base row adds
//                        its p to the softmax sum;
//             values  -> packed fp32 pair FMAs (fma.rn.f32x2) of the nibbles against
//                        both weights, each warp accumulating its own rows.
//             After an item's last batch: its BF16 tail columns from global memory, the
//             warps' merge (in the item's plan slot, which no one reads any more) and the
//             item's partial (M, L, m, sum p v, sum p~ v) in the workspace.
// A second, small kernel launched after the reader combines each (layer, head)'s partials
// into o, u, m and the loop's offset.  With the fused tail flush (a step whose tail holds
// 64 rows), each CTA of the reader then takes its share of every layer's flush units once
// its items are done.
#include "flush.cuh"
#include "kernels.h"

namespace fl {
namespace {

constexpr int kCW = 8;                 // consumer warps
constexpr int kCT = kCW * 32;          // consumer threads
constexpr int kPWarp = kCW;            // the producer warp
constexpr int kCWarp = kCW + 1;        // the first of the two copy warps
constexpr int kNT = kCT + 96;
constexpr int kCtaPerSm = 2;
constexpr int kStoresMax = 8;          // loops served
constexpr int kBCols = 64;             // columns of a batch at most
constexpr int kRowsMax = 160;          // rows of a batch at most
constexpr int kRecsMax = 32;           // key records of a batch at most
constexpr int kRowB = 144;             // a staged row: key codes 64 | value codes 64 | value sz 8 | pad 8
constexpr int kItemWords = 2048;       // plan words of one work item
constexpr int kTailMax = 64;           // BF16 tail columns of a head at most
constexpr int kTabs = 3;               // batch tables in the ring
static_assert(kRowsMax >= kStoresMax && kRecsMax >= kStoresMax, "one column always fits a batch");
static_assert(kRowsMax <= kCT, "one consumer thread per row for the weights");

// One batch: written by the producer, read by the consumers.
struct BatchTab {
  int32_t item, c0, ncol, nrows, nrecs, smax, done, last;  // item: the CTA's item sequence number
  int32_t rowbase[kStoresMax + 1];     // rows of store s start at rowbase[s - 1]
  int32_t recbase[kStoresMax + 1];     // key records of store s start at recbase[s - 1]
  uintptr_t src0, src1;                // the head's base and residual group records
  uint32_t bal[kStoresMax][2];         // columns (two rounds of 32) with a row in store s + 1
  uint32_t nbal[kStoresMax][2];        // ... whose row opens a new record
  uint8_t row_col[kRowsMax], row_rec[kRowsMax], row_store[kRowsMax], row_pin[kRowsMax];
  uint8_t colrow[kBCols][kStoresMax];  // row of (column, store s + 1)
  const uint8_t* row_src[kRowsMax];
  const uint8_t* rec_src[kRecsMax];
};
constexpr int kBufB = kRowsMax * kRowB + kRecsMax * 512;  // staged rows, then records

// A work item in flight (two slots, like the plan copies).
struct ItemInfo {
  float q[kD];                         // the head's query, pre-scaled to the base-2 domain
  int32_t layer, h, split, ncols, ktail, pad[3];
};

struct alignas(16) CtaB {
  ItemInfo item[2];
  float4 wrow[kRowsMax][2];            // per row: (wS0, wS0, wU0, wU0), the same for half 1
  float lr[kRowsMax];                  // per row: logit part
  float lcol[kBCols];                  // per column of the batch: logit (-inf: no quantised column)
  float wmax[kCW];                     // per warp: maximum logit of its columns of the batch
  float pcol[kTailMax];                // tail columns: weight p relative to the running max
  float lt[kTailMax];                  // tail columns: logits
  float redk[kCW][4];                  // per warp: the value-sum constants
  float redl[kCW][2];                  // per warp: its parts of L and m
  uint64_t tfull[kTabs], tempty[kTabs], dfull[2], bempty[2], pempty[2], pfull[2];
  float alpha;                         // rescale of the running sums for the batch being consumed
  int32_t failed;
  float mw;
};
constexpr int kCtaB = (int)((sizeof(CtaB) + 127) / 128 * 128);
constexpr int kTabB = (int)((sizeof(BatchTab) + 15) / 16 * 16);
constexpr int kSmemP = kCtaB + 2 * kItemWords * 4 + kTabs * kTabB + 2 * kBufB;
static_assert(kSmemP <= 113 * 1024, "two CTAs per SM");

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async8(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
// The mbarrier's phase completes (one pending arrival fewer) once every cp.async this
// thread issued before has landed.
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive1(uint64_t* bar) {
  asm volatile("{ .reg .b64 st; mbarrier.arrive.shared::cta.b64 st, [%0]; }" ::"r"(smem_addr(bar)) : "memory");
}
// barrier of the consumer warps
__device__ __forceinline__ void bar_c() { asm volatile("bar.sync 1, %0;" ::"n"(kCT) : "memory"); }
// the same barrier, returning whether any consumer thread passed v = true
__device__ __forceinline__ bool bar_c_or(bool v) {
  unsigned res;
  asm volatile(
      "{ .reg .pred p, q; setp.ne.u32 p, %1, 0; bar.red.or.pred q, 1, %2, p; selp.u32 %0, 1, 0, q; }"
      : "=r"(res)
      : "r"((unsigned)v), "n"(kCT)
      : "memory");
  return res != 0;
}

// A plan entry's first 4 nv words (j, tag | stores << 8, p~, the residual slots) into
// registers by 16-byte loads: with a lane per entry, two or three vector loads instead of a
// bank-conflicting load per field.
constexpr int kEntryMax = 12;  // words of loops r <= kStoresMax: r + 2 <= 10, rounded up to 4
static_assert(kEntryMax >= kStoresMax + 2, "an entry of loop kStoresMax fits");
__device__ __forceinline__ void load_entry(const int32_t* e, int* ev, int nv) {
#pragma unroll
  for (int k = 0; k < kEntryMax / 4; ++k)
    if (k < nv) {
      const int4 v = reinterpret_cast<const int4*>(e)[k];
      ev[4 * k] = v.x;
      ev[4 * k + 1] = v.y;
      ev[4 * k + 2] = v.z;
      ev[4 * k + 3] = v.w;
    }
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

// acc += a * b on two fp32 lanes at once (two independent round-to-nearest fmas, one
// packed instruction)
__device__ __forceinline__ void ffma2(float2& acc, float2 a, float2 b) { acc = __ffma2_rn(a, b, acc); }

// The eight nibbles of a code word (channel 8w + k in nibble k) as exact fp32 values
// 1 + n/128, in channel pairs: each nibble is shifted to bits 16..19 (mantissa bits below
// the exponent field, which starts at bit 23) and one logic op adds the exponent of 1.
__device__ __forceinline__ void nib_pairs(uint32_t x, float2* f) {
  auto v = [](uint32_t y) { return __uint_as_float((y & 0x000F0000u) | 0x3F800000u); };
  f[0] = make_float2(v(x << 16), v(x << 12));
  f[1] = make_float2(v(x << 8), v(x << 4));
  f[2] = make_float2(v(x), v(x >> 4));
  f[3] = make_float2(v(x >> 8), v(x >> 12));
}

// kFlush: the step also writes this loop's store of a full tail (fused flush)
template <bool kFlush>
__global__ void __launch_bounds__(kNT, kCtaPerSm) sparse_persist_kernel(ReaderArgs a, int n_items) {
  extern __shared__ __align__(128) uint8_t smem[];
  CtaB& cb = *reinterpret_cast<CtaB*>(smem);
  int32_t* plans = reinterpret_cast<int32_t*>(smem + kCtaB);   // [2][kItemWords]
  uint8_t* tabs = reinterpret_cast<uint8_t*>(plans + 2 * kItemWords);
  uint8_t* bufs = tabs + kTabs * kTabB;
  auto tab = [&](int b) -> BatchTab& { return *reinterpret_cast<BatchTab*>(tabs + (size_t)(b % kTabs) * kTabB); };
  auto rows_of = [&](int b) { return bufs + (size_t)(b & 1) * kBufB; };
  auto recs_of = [&](int b) { return bufs + (size_t)(b & 1) * kBufB + kRowsMax * kRowB; };

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const CacheView& c = a.c;
  const int H = c.H, cap = c.cap, ncb = cap / kG, T = c.total_slots, r = a.r;
  const int n_q = a.n_q, N = a.n_q + a.n_tail, K = a.k_sel, ps = c.plan_stride, ns = a.n_splits;
  const unsigned lt = lanes_below(lane);
  const bool has_new = a.k_new != nullptr;
  const int nv = (r + 2 + 3) / 4;  // 16-byte pieces of a plan entry that hold its r + 2 words

  grid_dep_launch();
  if (tid == 0) {
    for (int i = 0; i < kTabs; ++i) {
      mbar_init(&cb.tfull[i], 32);     // every producer lane, after its table writes
      mbar_init(&cb.tempty[i], kCW);   // one lane of each consumer warp, after its reads
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&cb.dfull[i], 128);    // every copy-warp lane: its table writes, and its copies once landed
      mbar_init(&cb.bempty[i], kCW);   // one lane of each consumer warp, done with the buffer
      mbar_init(&cb.pempty[i], kCW);   // one lane of each consumer warp, done with an item
      mbar_init(&cb.pfull[i], 1);      // an item's plan copy (bulk, transaction bytes)
    }
    fence_mbar_init();
    cb.failed = 0;
  }
  __syncthreads();

  if (warp == kPWarp) {
    // =========================== producer ===========================
    int b = 0;  // batch sequence number
    int seq = 0;
    for (int item = blockIdx.x; item < n_items && !*reinterpret_cast<volatile int32_t*>(&cb.failed);
         item += gridDim.x, ++seq) {
      const int pb = seq & 1;
      if (seq >= 2 && !mbar_wait(&cb.pempty[pb], (unsigned)(((seq - 2) >> 1) & 1))) {
        cb.failed = 1;
        break;
      }
      // ---- the item: (layer, head, split), its query and plan ----
      const int lh = item / ns, split = item - lh * ns;
      const int layer = a.layer + lh / H, h = lh % H;
      const int k0 = (int)((long long)split * K / ns), k1 = (int)((long long)(split + 1) * K / ns);
      const int ncols = k1 - k0;
      ItemInfo& it = cb.item[pb];
      int32_t* plan_s = plans + pb * kItemWords;
      const int64_t io = (int64_t)(layer - a.layer) * a.io_layer_stride;
      if (lane == 0) {
        it.layer = layer;
        it.h = h;
        it.split = split;
      }
      {
        const uint2 qw = reinterpret_cast<const uint2*>(a.q + io + (size_t)h * kD)[lane];
        it.q[4 * lane + 0] = __uint_as_float(qw.x << 16) * kQScale;
        it.q[4 * lane + 1] = __uint_as_float(qw.x & 0xffff0000u) * kQScale;
        it.q[4 * lane + 2] = __uint_as_float(qw.y << 16) * kQScale;
        it.q[4 * lane + 3] = __uint_as_float(qw.y & 0xffff0000u) * kQScale;
      }
      if (split == 0 && has_new) {
        uint16_t* tail_k = arr<uint16_t>(c, A_TAILK, layer) + ((size_t)(r - 1) * H + h) * kTail * kD;
        uint16_t* tail_v = arr<uint16_t>(c, A_TAILV, layer) + ((size_t)(r - 1) * H + h) * kTail * kD;
        reinterpret_cast<uint2*>(tail_k + (size_t)(a.n_tail - 1) * kD)[lane] =
            reinterpret_cast<const uint2*>(a.k_new + io + (size_t)h * kD)[lane];
        reinterpret_cast<uint2*>(tail_v + (size_t)(a.n_tail - 1) * kD)[lane] =
            reinterpret_cast<const uint2*>(a.v_new + io + (size_t)h * kD)[lane];
      }
      const int32_t* plan_g = arr<int32_t>(c, A_PLAN, layer) + (size_t)h * c.max_select * ps;
      // the item's plan entries in one bulk copy (entries are 16-byte multiples)
      if (lane == 0) {
        fence_proxy_async();  // generic writes of this slot's previous item come first
        const unsigned bytes = (unsigned)ncols * (unsigned)ps * 4u;
        mbar_expect_tx(&cb.pfull[pb], bytes);
        bulk_g2s(plan_s, plan_g + (size_t)k0 * ps, bytes, &cb.pfull[pb]);
      }
      if (!mbar_wait(&cb.pfull[pb], (unsigned)((seq >> 1) & 1))) {
        cb.failed = 1;
        break;
      }
      const uint8_t* brec = arr<uint8_t>(c, A_BREC, layer) + (size_t)h * ncb * kRec;
      const uint8_t* rrec = arr<uint8_t>(c, A_RREC, layer) + (size_t)h * (T / kG) * kRec;
      auto rec_of = [&](const int* ev, int s) { return s == 1 ? (ev[0] >> 6) : (ev[1 + s] >> 6); };
      // an entry is skipped (no rows, no score, no weight; the error recorded) when its column,
      // tag, store count or slots are out of range; 1: a quantised column, 2: a tail column
      // (ev: the entry's words, loaded whole)
      auto validate = [&](int32_t* e, int* ev) -> int {
        const int j = ev[0], st = (ev[1] >> 8) & 0xff, lam = ev[1] & 0xff;
        bool ok = j >= 0 && j < N && lam >= 1 && lam <= c.R;
        int kind = 0;
        if (ok && j < n_q) {
          ok = st >= 1 && st <= r;
#pragma unroll
          for (int s2 = 2; s2 <= kStoresMax; ++s2)
            if (s2 <= st) ok = ok && ev[1 + s2] >= 0 && ev[1 + s2] < T;
          kind = 1;
        } else if (ok) {
          ok = st == 0;
          kind = 2;
        }
        if (!ok) {
          record_error(c.status, FL_DEV_SEL_RANGE, j);
          e[0] = -1;
          e[1] = 0;
          e[2] = 0;
          ev[0] = -1;
          ev[1] = 0;
          return 0;
        }
        return kind;
      };

      // ---- the item's batches (at least one: an item of tail columns only has an empty one);
      //      the columns are validated as formation reaches them, and the quantised part ends
      //      at the first tail column (S is ascending) ----
      int cpos = 0;
      int kt = ncols;  // first tail column
      do {
        if (b >= kTabs && !mbar_wait(&cb.tempty[b % kTabs], (unsigned)(((b - kTabs) / kTabs) & 1))) {
          cb.failed = 1;
          break;
        }
        BatchTab& tb = tab(b);
        // formation: how many columns fit the budgets (one or two rounds of 32); the
        // ballots of each store (rows, and rows opening a new record) are kept
        int ncol = 0, nrows = 0, nrecs = 0, smax = 0;
        int lastg[kStoresMax];
#pragma unroll
        for (int s = 0; s < kStoresMax; ++s) lastg[s] = -1;
        int rounds = 0;
        for (int rd = 0; rd < 2 && cpos + 32 * rd < kt; ++rd) {
          const int cc = cpos + 32 * rd + lane;
          const bool inr = cc < kt && 32 * rd + lane < kBCols;
          int32_t* e = plan_s + (size_t)(inr ? cc : cpos) * ps;
          int ev[kEntryMax];
          load_entry(e, ev, nv);
          const int kind = inr ? validate(e, ev) : 0;
          const unsigned tb2 = __ballot_sync(kFull, kind == 2);
          if (tb2) kt = cpos + 32 * rd + __ffs(tb2) - 1;  // the quantised part ends here
          const bool in = inr && cc < kt;
          const int st = in && kind == 1 ? (ev[1] >> 8) & 0xff : 0;
          const int smr = __reduce_max_sync(kFull, st);
          int nrec_c = 0;
#pragma unroll
          for (int s = 1; s <= kStoresMax; ++s) {
            unsigned ab = 0u, nb = 0u;
            if (s <= smr) {
              const bool act = st >= s;
              const int g = act ? rec_of(ev, s) : -1;
              ab = __ballot_sync(kFull, act);
              const unsigned pb2 = ab & lt;
              const int gs = __shfl_sync(kFull, g, pb2 ? 31 - __clz(pb2) : 0);
              const int gp = pb2 ? gs : lastg[s - 1];
              const bool isnew = act && gp != g;
              nrec_c += isnew ? 1 : 0;
              nb = __ballot_sync(kFull, isnew);
              if (ab) lastg[s - 1] = __shfl_sync(kFull, g, 31 - __clz(ab));
            }
            if (lane == 0) {
              tb.bal[s - 1][rd] = ab;
              tb.nbal[s - 1][rd] = nb;
            }
          }
          const int rows_i = scan_incl(st, lane) + nrows, recs_i = scan_incl(nrec_c, lane) + nrecs;
          const unsigned inb = __ballot_sync(kFull, in);
          const unsigned over = __ballot_sync(kFull, in && (rows_i > kRowsMax || recs_i > kRecsMax));
          const int take = over ? __ffs(over) - 1 : __popc(inb);
          if (take > 0) {
            nrows = __shfl_sync(kFull, rows_i, take - 1);
            nrecs = __shfl_sync(kFull, recs_i, take - 1);
            smax = max(smax, __reduce_max_sync(kFull, lane < take ? st : 0));
          }
          ncol += take;
          rounds = rd + 1;
          if (take < 32) {
            __syncwarp();
            if (lane < kStoresMax) {  // the cut round keeps the columns below the cut
              tb.bal[lane][rd] &= lanes_below(take);
              tb.nbal[lane][rd] &= lanes_below(take);
            }
          }
          if (over || take < 32) break;
        }
        __syncwarp();
        if (lane < kStoresMax) {
          for (int rd = rounds; rd < 2; ++rd) {
            tb.bal[lane][rd] = 0u;
            tb.nbal[lane][rd] = 0u;
          }
        }
        const bool last = cpos + ncol >= kt;
        if (last) {
          // the tail columns [kt, ncols): validated here (those of the cut round again:
          // validation is idempotent), attended by the consumers at the item's end
          for (int cc = kt + lane; cc < ncols; cc += 32) {
            int ev[kEntryMax];
            load_entry(plan_s + (size_t)cc * ps, ev, nv);
            validate(plan_s + (size_t)cc * ps, ev);
          }
        }
        __syncwarp();
        if (lane == 0) {
          int rb = 0, kb = 0;
          for (int s = 1; s <= smax; ++s) {
            tb.rowbase[s - 1] = rb;
            tb.recbase[s - 1] = kb;
            rb += __popc(tb.bal[s - 1][0]) + __popc(tb.bal[s - 1][1]);
            kb += __popc(tb.nbal[s - 1][0]) + __popc(tb.nbal[s - 1][1]);
          }
          tb.rowbase[smax] = rb;
          tb.recbase[smax] = kb;
          tb.item = seq;
          tb.c0 = cpos;
          tb.ncol = ncol;
          tb.nrows = nrows;
          tb.nrecs = nrecs;
          tb.smax = smax;
          tb.done = 0;
          tb.last = last;
          tb.src0 = reinterpret_cast<uintptr_t>(brec);
          tb.src1 = reinterpret_cast<uintptr_t>(rrec);
          if (last) {
            it.ncols = ncols;
            it.ktail = kt;
          }
        }
        __syncwarp();
        mbar_arrive1(&cb.tfull[b % kTabs]);  // the table is complete (release)
        cpos += ncol;
        ++b;
      } while (cpos < kt);
    }
    // the end marker
    if (!(b >= kTabs && !mbar_wait(&cb.tempty[b % kTabs], (unsigned)(((b - kTabs) / kTabs) & 1)))) {
      if (lane == 0) tab(b).done = 1;
      __syncwarp();
      mbar_arrive1(&cb.tfull[b % kTabs]);
    } else {
      cb.failed = 1;
    }
  }

  // =========================== copies ===========================
  // Copy warp cw takes the columns 32 cw .. 32 cw + 31 of each batch (a lane each): their rows'
  // table entries, then 16-byte cp.async pieces of those rows (eight per row: key codes | value
  // codes), their 8-byte value (scale, zero) pairs and the key records their rows open.  In
  // each store, a warp's rows and records form one run.
  if (warp == kCWarp || warp == kCWarp + 1) {
    const int cw = warp - kCWarp;
    for (int b = 0;; ++b) {
      // batch b's table is formed, and (b >= 2) the consumers are done with batch b - 2, whose
      // buffer batch b takes
      bool ok = mbar_wait(&cb.tfull[b % kTabs], (unsigned)((b / kTabs) & 1));
      if (ok && b >= 2) ok = mbar_wait(&cb.bempty[b & 1], (unsigned)(((b - 2) >> 1) & 1));
      ok = __all_sync(kFull, ok);
      if (!ok) cb.failed = 1;
      BatchTab& tb = tab(b);
      const bool stop = !ok || tb.done;
      if (!stop) {
        uint8_t* rows = rows_of(b);
        uint8_t* recs = recs_of(b);
        const int ncol = tb.ncol, c0 = tb.c0;
        const int col = 32 * cw + lane;
        const int32_t* plan_s = plans + (tb.item & 1) * kItemWords;
        const uint8_t* brec = reinterpret_cast<const uint8_t*>(tb.src0);
        const uint8_t* rrec = reinterpret_cast<const uint8_t*>(tb.src1);
        int ev[kEntryMax];
        load_entry(plan_s + (size_t)(c0 + (col < ncol ? col : 0)) * ps, ev, nv);
        const int st = col < ncol && ev[0] >= 0 ? (ev[1] >> 8) & 0xff : 0;
#pragma unroll
        for (int s = 0; s < kStoresMax; ++s) {  // store s + 1
          if (s >= st) break;
          const unsigned ab = tb.bal[s][cw], nb = tb.nbal[s][cw];
          const int ri = tb.rowbase[s] + (cw ? __popc(tb.bal[s][0]) : 0) + __popc(ab & lt);
          const int ki = tb.recbase[s] + (cw ? __popc(tb.nbal[s][0]) : 0) + __popc(nb & (lt | (1u << lane))) - 1;
          const int slot = s == 0 ? ev[0] : ev[2 + s];
          const uint8_t* base = (s == 0 ? brec : rrec) + (size_t)(slot >> 6) * kRec;
          tb.row_col[ri] = (uint8_t)col;
          tb.row_rec[ri] = (uint8_t)ki;
          tb.row_store[ri] = (uint8_t)(s + 1);
          tb.row_pin[ri] = (uint8_t)(slot & 63);
          tb.row_src[ri] = base + (slot & 63) * 128;
          tb.colrow[col][s] = (uint8_t)ri;
          if ((nb >> lane) & 1u) tb.rec_src[ki] = base + kRecKsz;
        }
        __syncwarp();
        for (int s = 0; s < tb.smax; ++s) {
          const int n = __popc(tb.bal[s][cw]), nk = __popc(tb.nbal[s][cw]);
          const int r0 = tb.rowbase[s] + (cw ? __popc(tb.bal[s][0]) : 0);
          const int k0 = tb.recbase[s] + (cw ? __popc(tb.nbal[s][0]) : 0);
          for (int t = lane; t < 8 * n; t += 32) {  // row pieces
            const int ri = r0 + (t >> 3);
            cp_async16(rows + ri * kRowB + (t & 7) * 16, tb.row_src[ri] + (t & 7) * 16);
          }
          for (int t = lane; t < n; t += 32) {      // the rows' value (scale, zero) pairs
            const int ri = r0 + t, pin = tb.row_pin[ri];
            cp_async8(rows + ri * kRowB + 128, tb.row_src[ri] - pin * 128 + kRecVsz + pin * 8);
          }
          for (int k = 0; k < nk; ++k)              // key records: a 16-byte piece per lane
            cp_async16(recs + (k0 + k) * 512 + lane * 16, tb.rec_src[k0 + k] + lane * 16);
        }
      }
      __syncwarp();
      mbar_arrive1(&cb.dfull[b & 1]);      // the table (release)
      cp_async_arrive(&cb.dfull[b & 1]);   // the copies, once landed
      if (stop) break;
    }
  }

  // =========================== consumers ===========================
  if (warp < kCW) {
    const int qq = lane & 3, tr = lane >> 2;
    const int wd = lane & 15, par = lane >> 4, hv = wd >> 3;
    // per item: warp 0 keeps the running maximum M (uniform) and per-lane parts of L and m;
    // every thread its value sums and its parts of the constants sum of (p z - W) per half
    float M = -INFINITY, Ls = 0.f, msum = 0.f;
    float2 accS[4], accU[4];
    float kS[2], kU[2];
    auto reset = [&]() {
      M = -INFINITY;
      Ls = msum = 0.f;
#pragma unroll
      for (int k = 0; k < 4; ++k) accS[k] = accU[k] = make_float2(0.f, 0.f);
      kS[0] = kS[1] = kU[0] = kU[1] = 0.f;
    };
    reset();
    bool waited = false;  // the dependent-launch wait, before the first partial
    for (int b = 0;; ++b) {
      const bool ok = mbar_wait(&cb.dfull[b & 1], (unsigned)((b >> 1) & 1));
      if (!ok) cb.failed = 1;
      // every consumer agrees: the end marker, or a wait ran out here or elsewhere
      if (bar_c_or(!ok || tab(b).done || *reinterpret_cast<volatile int32_t*>(&cb.failed))) break;
      const BatchTab& hd = tab(b);
      // every field read after this warp releases the table comes from these copies
      const int seq = hd.item, c0 = hd.c0, ncol = hd.ncol, nrows = hd.nrows, nrecs = hd.nrecs;
      const bool last = hd.last != 0;
      const ItemInfo& it = cb.item[seq & 1];
      const int32_t* plan_s = plans + (seq & 1) * kItemWords;
      const int layer = it.layer, h = it.h;
      float* score = arr<float>(c, A_SCORE, layer) + (size_t)h * cap;
      uint8_t* tag = arr<uint8_t>(c, A_TAG, layer) + (size_t)h * cap;
      const uint8_t* rows = rows_of(b);
      uint8_t* recs = recs_of(b);

      if (ncol > 0) {
        // (1) records -> 24-bit fixed-point query weights in byte limbs, in place
        for (int k = warp; k < nrecs; k += 2 * kCW) {  // two records per step where there are two
          uint32_t* ra = reinterpret_cast<uint32_t*>(recs + k * 512);
          if (k + kCW < nrecs) record_to_limbs2(ra, reinterpret_cast<uint32_t*>(recs + (k + kCW) * 512), it.q, lane);
          else record_to_limbs(ra, it.q, lane);
        }
        bar_c();
        // (2) one logit part per row: exact dp4a dot of the row quarter with its record's limbs
        for (int p0 = 8 * warp; p0 < nrows; p0 += 8 * kCW) {
          const int row = p0 + tr;
          const bool act = row < nrows;
          const uint32_t* lim = reinterpret_cast<const uint32_t*>(recs + (act ? hd.row_rec[row] : 0) * 512);
          float d = 0.f;
          if (act) {
            uint32_t lw[24];
            load_limbs(lim, qq, lw);
            d = limb_dot(*reinterpret_cast<const uint4*>(rows + row * kRowB + 16 * qq), lw) * pow2i(-(int)lim[kLimbE]);
          }
          d += __shfl_xor_sync(kFull, d, 1);
          d += __shfl_xor_sync(kFull, d, 2);
          if (act && qq == 0) cb.lr[row] = d + __uint_as_float(lim[kLimbC]);
        }
        bar_c();
        // (3) columns: warp w takes columns 8 w .. 8 w + 7, a lane each: the parts summed in
        //     store order, score and tag spliced, the warp's maximum logit
        {
          const int col = 8 * warp + lane;  // < kBCols for lane < 8
          const bool in = lane < 8 && col < ncol;
          const int32_t* e = plan_s + (size_t)(c0 + (in ? col : 0)) * ps;
          const int st = in && e[0] >= 0 ? (e[1] >> 8) & 0xff : 0;
          float part[kStoresMax];
#pragma unroll
          for (int s = 0; s < kStoresMax; ++s) part[s] = s < st ? cb.lr[hd.colrow[col][s]] : 0.f;
          float l = 0.f;
#pragma unroll
          for (int s = 0; s < kStoresMax; ++s)
            if (s < st) l += part[s];
          l = st > 0 ? l : -INFINITY;
          if (lane < 8) cb.lcol[col] = l;
          if (st > 0) {
            msum += __int_as_float(e[2]);
            score[e[0]] = l;
            tag[e[0]] = (uint8_t)r;
          }
          const float wm = warp_max(l);
          if (lane == 0) cb.wmax[warp] = wm;
        }
        bar_c();
        // (4) the running maximum (the same M in every consumer thread), then per-row value
        //     weights, one consumer thread per row; a column's base row adds its p to L
        float Mn = M;
#pragma unroll
        for (int w = 0; w < kCW; ++w) Mn = fmaxf(Mn, cb.wmax[w]);
        const float al = Mn == -INFINITY ? 1.f : ex2(M - Mn);
        M = Mn;
        Ls *= al;
        kS[0] *= al;
        kS[1] *= al;
        if (tid < nrows) {
          const int col = hd.row_col[tid], s = hd.row_store[tid];
          const int32_t* e = plan_s + (size_t)(c0 + col) * ps;
          const float p = ex2(cb.lcol[col] - Mn);
          if (s == 1) Ls += p;
          const float pu = s <= (e[1] & 0xff) ? __int_as_float(e[2]) : 0.f;  // the tag loop's rows: a prefix
          const uint2 szw = *reinterpret_cast<const uint2*>(rows + tid * kRowB + 128);
          const float2 z0 = unpack_sz(szw.x), z1 = unpack_sz(szw.y);
          const float wS0 = 128.f * (p * z0.x), wS1 = 128.f * (p * z1.x);
          const float wU0 = 128.f * (pu * z0.x), wU1 = 128.f * (pu * z1.x);
          cb.wrow[tid][0] = make_float4(wS0, wS0, wU0, wU0);
          cb.wrow[tid][1] = make_float4(wS1, wS1, wU1, wU1);
          kS[0] += fmaf(p, z0.y, -wS0);
          kS[1] += fmaf(p, z1.y, -wS1);
          kU[0] += fmaf(pu, z0.y, -wU0);
          kU[1] += fmaf(pu, z1.y, -wU1);
        }
        bar_c();
        // (5) values: lane (word wd, parity par) takes channels 8 wd .. 8 wd + 7 of rows
        //     r0 + 4 par + i (the two parities 16 banks apart)
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          accS[k].x *= al;
          accS[k].y *= al;
        }
        for (int r0 = 8 * warp; r0 < nrows; r0 += 8 * kCW) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int row = r0 + 4 * par + i;
            if (row < nrows) {
              const uint32_t x = *reinterpret_cast<const uint32_t*>(rows + row * kRowB + 64 + 4 * wd);
              const float4 w = cb.wrow[row][hv];
              float2 f[4];
              nib_pairs(x, f);
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                ffma2(accS[k], make_float2(w.x, w.y), f[k]);
                ffma2(accU[k], make_float2(w.z, w.w), f[k]);
              }
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) {  // this warp is done with the table and the buffer
        mbar_arrive1(&cb.tempty[b % kTabs]);
        mbar_arrive1(&cb.bempty[b & 1]);
      }

      if (last) {
        // ---- the item's BF16 tail columns [ktail, ncols) (at most 64 per head), from global
        //      memory: logits (four lanes per column), softmax (warp 0), values ----
        const int ktail = it.ktail, ntail = min(it.ncols - ktail, kTailMax);
        const int64_t io = (int64_t)(layer - a.layer) * a.io_layer_stride;
        const uint16_t* tail_k = arr<uint16_t>(c, A_TAILK, layer) + ((size_t)(r - 1) * H + h) * kTail * kD;
        const uint16_t* tail_v = arr<uint16_t>(c, A_TAILV, layer) + ((size_t)(r - 1) * H + h) * kTail * kD;
        const uint16_t* tail_v_all = arr<uint16_t>(c, A_TAILV, layer);
        if (ntail > 0) {
          for (int t0 = 8 * warp; t0 < ntail; t0 += 8 * kCW) {
            const int t = t0 + tr;
            const int32_t* e = plan_s + (size_t)(ktail + (t < ntail ? t : 0)) * ps;
            const int j = e[0];
            const bool in = t < ntail && j >= n_q && j < N;
            float d = 0.f;
            if (in) {
              const uint16_t* rowp =
                  (has_new && j == N - 1) ? a.k_new + io + (size_t)h * kD : tail_k + (size_t)(j - n_q) * kD;
              float qsr[32];
              load32(it.q + 32 * qq, qsr);
              d = dot_bf16_32(rowp + 32 * qq, qsr);
            }
            d += __shfl_xor_sync(kFull, d, 1);
            d += __shfl_xor_sync(kFull, d, 2);
            if (t < ntail && qq == 0) cb.lt[t] = in ? d : -INFINITY;
          }
          bar_c();
          if (warp == 0) {
            float l2[2];
#pragma unroll
            for (int rd = 0; rd < 2; ++rd) l2[rd] = 32 * rd + lane < ntail ? cb.lt[32 * rd + lane] : -INFINITY;
            const float Mn = fmaxf(M, warp_max(fmaxf(l2[0], l2[1])));
            const float al = Mn == -INFINITY ? 1.f : ex2(M - Mn);
            M = Mn;
            Ls *= al;
#pragma unroll
            for (int rd = 0; rd < 2; ++rd) {
              const int t = 32 * rd + lane;
              const bool in = l2[rd] != -INFINITY;
              const float p = in ? ex2(l2[rd] - Mn) : 0.f;
              cb.pcol[t] = p;
              if (in) {
                const int32_t* e = plan_s + (size_t)(ktail + t) * ps;
                Ls += p;
                msum += __int_as_float(e[2]);
                score[e[0]] = l2[rd];
                tag[e[0]] = (uint8_t)r;
              }
            }
            if (lane == 0) cb.alpha = al;
          }
          bar_c();
          const float al = cb.alpha;
          if (warp != 0) Ls *= al;  // warp 0 rescaled its parts of L before adding the tail's
          kS[0] *= al;
          kS[1] *= al;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            accS[k].x *= al;
            accS[k].y *= al;
          }
          // lane (wd, par): channels 8 wd .. 8 wd + 7 of tail columns t = 2 (warp + 8 m) + par
          for (int t = 2 * warp + par; t < ntail; t += 2 * kCW) {
            if (cb.lt[t] == -INFINITY) continue;
            const float p = cb.pcol[t];
            const int32_t* e = plan_s + (size_t)(ktail + t) * ps;
            const int j = e[0], lam = e[1] & 0xff;
            const float pt = __int_as_float(e[2]);
            const uint16_t* vr =
                (has_new && j == N - 1) ? a.v_new + io + (size_t)h * kD : tail_v + (size_t)(j - n_q) * kD;
            const uint16_t* ur = tail_v_all + (((size_t)(lam - 1) * H + h) * kTail + (j - n_q)) * kD;
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(vr) + wd);
            const uint4 u = __ldg(reinterpret_cast<const uint4*>(ur) + wd);
            const uint32_t vw[4] = {v.x, v.y, v.z, v.w}, uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              ffma2(accS[k], make_float2(p, p), make_float2(bf16_lo(vw[k]), bf16_hi(vw[k])));
              ffma2(accU[k], make_float2(pt, pt), make_float2(bf16_lo(uw[k]), bf16_hi(uw[k])));
            }
          }
          bar_c();  // every warp is done with the item's plan entries (the merge area)
        }

        // ---- merge the warps (lane (wd, par) holds channels 8 wd .. 8 wd + 7) and write
        //      the item's partial (M, L, m, sum p v, sum p~ v); the item's plan slot, read by
        //      no one any more, holds the warps' sums ----
        float kk[4] = {kS[0], kS[1], kU[0], kU[1]};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          kk[i] = warp_sum(kk[i]);
          if (lane == 0) cb.redk[warp][i] = kk[i];
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          accS[k].x += __shfl_xor_sync(kFull, accS[k].x, 16);
          accS[k].y += __shfl_xor_sync(kFull, accS[k].y, 16);
          accU[k].x += __shfl_xor_sync(kFull, accU[k].x, 16);
          accU[k].y += __shfl_xor_sync(kFull, accU[k].y, 16);
        }
        Ls = warp_sum(Ls);
        msum = warp_sum(msum);
        if (lane == 0) {
          cb.redl[warp][0] = Ls;
          cb.redl[warp][1] = msum;
          if (warp == 0) cb.mw = M;
        }
        if (!waited) {
          grid_dep_wait();  // the workspace's partials are free from here (the previous combine read them)
          waited = true;
        }
        float* red = reinterpret_cast<float*>(plans + (seq & 1) * kItemWords);  // [S, U][kCW][kD]
        static_assert(kItemWords >= 2 * kCW * kD, "the plan slot holds the warps' sums");
        if (par == 0) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            red[warp * kD + 8 * wd + 2 * k] = accS[k].x;
            red[warp * kD + 8 * wd + 2 * k + 1] = accS[k].y;
            red[(kCW + warp) * kD + 8 * wd + 2 * k] = accU[k].x;
            red[(kCW + warp) * kD + 8 * wd + 2 * k + 1] = accU[k].y;
          }
        }
        bar_c();
        {
          // thread (half, ch): half 0 sums S, half 1 sums U, of channel ch
          const int half = tid >> 7, ch = tid & (kD - 1);
          const int lh = (layer - a.layer) * H + h;
          float* part = a.part + ((size_t)lh * ns + it.split) * kPartStride;
          float Xt = 0.f, kXt = 0.f;
#pragma unroll
          for (int w = 0; w < kCW; ++w) {
            Xt += red[(half * kCW + w) * kD + ch];
            kXt += cb.redk[w][2 * half + (ch >> 6)];
          }
          part[4 + half * kD + ch] = Xt + kXt;
          if (tid == 0) {
            float Lt = 0.f, mt = 0.f;
#pragma unroll
            for (int w = 0; w < kCW; ++w) {
              Lt += cb.redl[w][0];
              mt += cb.redl[w][1];
            }
            part[0] = cb.mw;
            part[1] = Lt;
            part[2] = mt;
          }
        }
        static_assert(kCT == 2 * kD, "a consumer thread per (half, channel)");
        __syncwarp();
        if (lane == 0) mbar_arrive1(&cb.pempty[seq & 1]);  // this warp is done with the item's slots
        reset();
      }
    }
    if (cb.failed && tid == 0) record_error(c.status, FL_DEV_TIMEOUT, blockIdx.x);
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();
  if constexpr (kFlush) {
    // the readers of loops 1 .. r - 1 wrote the stores this flush builds on: they are final
    // after the dependent-launch wait; the batch buffers hold the staging
    grid_dep_wait();
    static_assert(2 * kBufB >= (int)sizeof(EncodeSmem), "the batch buffers hold the fused flush's staging");
    for (int i = 0; i < a.n_layers; ++i) {
      // layer i's 8 H units are the grid-wide units [8 H i, 8 H (i + 1)): CTA c takes the
      // units congruent to c modulo the grid, so the work spreads over every CTA
      const int G = (int)gridDim.x;
      const int rot = (int)(((long long)blockIdx.x - 8LL * H * i) % G + G) % G;
      const int64_t io = (int64_t)i * a.io_layer_stride;
      flush_tail_layer(a, a.layer + i, a.flush_slot0s[i], a.k_new ? a.k_new + io : nullptr,
                       a.v_new ? a.v_new + io : nullptr, rot, G, *reinterpret_cast<EncodeSmem*>(bufs), tid, kNT);
    }
  }
}

// The combine of each (layer, head) of a launch of the reader above: its items' partials
// merged by log-sum-exp (M, L over the splits), u = o_prev - sum p~ v, o = u + m S / L, and the
// loop's offset M + log2 L - log2 m, by which the next selection turns a kept score back into
// a global probability.  A CTA per (layer, head), a thread per channel; launched after the
// reader (dependent launch: it waits for the reader's partials).
__global__ void __launch_bounds__(kD) sparse_combine_kernel(ReaderArgs a) {
  grid_dep_launch();
  grid_dep_wait();
  const CacheView& c = a.c;
  const int H = c.H, r = a.r, ns = a.n_splits, tid = threadIdx.x;
  const int lh = blockIdx.x, layer = a.layer + lh / H, h = lh % H;
  const int64_t io = (int64_t)(layer - a.layer) * a.io_layer_stride;
  const float* hp = a.part + (size_t)lh * ns * kPartStride;
  float Mx = -INFINITY;
  for (int s = 0; s < ns; ++s) Mx = fmaxf(Mx, hp[(size_t)s * kPartStride]);
  float Lt = 0.f, St = 0.f, Ut = 0.f, mt = 0.f;
  for (int s = 0; s < ns; ++s) {
    const float* pp = hp + (size_t)s * kPartStride;
    Ut += pp[4 + kD + tid];
    mt += pp[2];
    const float ms = pp[0];
    if (ms == -INFINITY) continue;
    const float e = ex2(ms - Mx);
    Lt = fmaf(pp[1], e, Lt);
    St = fmaf(pp[4 + tid], e, St);
  }
  const float u = a.o_prev[io + (size_t)h * kD + tid] - Ut;
  a.o[io + (size_t)h * kD + tid] = Lt > 0.f ? fmaf(mt, St / Lt, u) : u;
  arr<float>(c, A_UNSEL, layer)[(size_t)h * kD + tid] = u;
  if (tid == 0) {
    arr<float>(c, A_MASS, layer)[h] = mt;
    arr<float>(c, A_OFFSET, layer)[(size_t)h * kOffStride + r] = Mx + log2f(Lt) - log2f(mt);
  }
}

std::atomic<bool> g_attr_done[kMaxDevices];
std::mutex g_attr_mu;

}  // namespace

int persist_item_columns(int loops) { return kItemWords / ((loops + 2 + 3) / 4 * 4); }

int persist_splits(int k_sel, int loops) {
  const int per = persist_item_columns(loops);
  return (k_sel + per - 1) / per;
}

cudaError_t launch_sparse_persist(ReaderArgs a, cudaStream_t s, bool chain) {
  const cudaError_t e = once_per_device(g_attr_done, g_attr_mu, [](int) {
    for (auto k : {sparse_persist_kernel<false>, sparse_persist_kernel<true>}) {
      cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemP);
      if (e != cudaSuccess) return e;
      e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  });
  if (e != cudaSuccess) return e;
  if (a.flush && a.n_layers > kFlushLayersMax) return cudaErrorInvalidValue;
  const int sms = device_sms() > 0 ? device_sms() : 148;
  a.n_splits = persist_splits(a.k_sel, a.c.R);
  const int n_items = a.n_layers * a.c.H * a.n_splits;
  int grid = n_items < kCtaPerSm * sms ? n_items : kCtaPerSm * sms;
  // the flush units of a layer (8 per head) are spread over the grid
  if (a.flush && grid < 8 * a.c.H) grid = 8 * a.c.H < kCtaPerSm * sms ? 8 * a.c.H : kCtaPerSm * sms;
  auto kern = a.flush ? sparse_persist_kernel<true> : sparse_persist_kernel<false>;
  const cudaError_t e1 = launch_pdl_if(chain, kern, dim3(grid), dim3(kNT), (size_t)kSmemP, s, a, n_items);
  if (e1 != cudaSuccess) return e1;
  return launch_pdl_if(true, sparse_combine_kernel, dim3(a.n_layers * a.c.H), dim3(kD), (size_t)0, s, a);
}

}  // namespace fl
