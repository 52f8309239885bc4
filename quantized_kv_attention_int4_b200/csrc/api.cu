// Host side of the C ABI declared in include/flashloop.h: layout arithmetic, argument
// validation and kernel launches.  Nothing here allocates device memory.
#include <atomic>
#include <cstring>

#include "kernels.h"

using namespace fl;

namespace {

constexpr uint64_t kAlign = 256;

inline uint64_t align_up(uint64_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

fl_status check_dims(const fl_dims* d) {
  if (!d) return FL_ERR_INVALID;
  if (d->head_dim != FL_HEAD_DIM || d->group != FL_GROUP) return FL_ERR_UNSUPPORTED;
  if (d->layers < 1 || d->heads < 1 || d->loops < 1 || d->loops > FL_MAX_LOOPS) return FL_ERR_INVALID;
  if (d->capacity < FL_GROUP || d->capacity % FL_GROUP != 0) return FL_ERR_INVALID;
  if (d->max_select < 1) return FL_ERR_INVALID;
  if (d->codec != FL_CODEC_RESIDUAL_INT4 && d->codec != FL_CODEC_FULL_INT4 && d->codec != FL_CODEC_RESIDUAL_INT2)
    return FL_ERR_UNSUPPORTED;
  for (int r = 2; r <= d->loops; ++r)
    if (d->res_capacity[r] < 0 || d->res_capacity[r] % FL_GROUP != 0) return FL_ERR_INVALID;
  return FL_OK;
}

inline int plan_stride(const fl_dims* d) { return (d->loops + 2 + 3) / 4 * 4; }

// Per-layer byte sizes of every array, in fl_layout order.
void layer_sizes(const fl_dims* d, uint64_t* sz, int32_t* slot_base, int32_t* total_slots) {
  const uint64_t H = d->heads, C = d->capacity, R = d->loops;
  uint64_t T = 0;
  for (int r = 0; r <= FL_MAX_LOOPS; ++r) slot_base[r] = 0;
  for (int r = 2; r <= d->loops; ++r) {
    slot_base[r] = (int32_t)T;
    T += (uint64_t)d->res_capacity[r];
  }
  *total_slots = (int32_t)T;
  sz[A_BREC] = H * (C / 64) * (uint64_t)FL_GROUP_RECORD;
  const uint64_t rrec_bytes = d->codec == FL_CODEC_RESIDUAL_INT2 ? FL_GROUP_RECORD_INT2 : FL_GROUP_RECORD;
  sz[A_RREC] = H * (T / 64) * rrec_bytes;
  sz[A_MASK] = (R + 1) * (C / 64) * 8;
  sz[A_FIRST] = (R + 1) * (C / 64) * 4;
  sz[A_DEPTH] = C;
  sz[A_TAILK] = R * H * 64 * 128 * 2;
  sz[A_TAILV] = R * H * 64 * 128 * 2;
  sz[A_SCORE] = H * C * 4;
  sz[A_TAG] = H * C;
  sz[A_OFFSET] = H * (FL_MAX_LOOPS + 1) * 4;
  sz[A_SEL] = H * (uint64_t)d->max_select * 4;
  sz[A_MASS] = H * 4;
  sz[A_UNSEL] = H * 128 * 4;
  sz[A_PLAN] = H * (uint64_t)d->max_select * plan_stride(d) * 4;
}

fl_status make_layout(const fl_dims* d, fl_layout* L) {
  fl_status st = check_dims(d);
  if (st != FL_OK) return st;
  std::memset(L, 0, sizeof(*L));
  uint64_t sz[A_COUNT];
  layer_sizes(d, sz, L->slot_base, &L->total_slots);
  uint64_t* offs[A_COUNT] = {&L->brec,  &L->rrec,   &L->mask,  &L->first, &L->depth,
                             &L->tail_k, &L->tail_v, &L->score, &L->tag,   &L->offset,
                             &L->sel,   &L->mass,   &L->unsel, &L->plan};
  uint64_t cur = 0;
  for (int i = 0; i < A_COUNT; ++i) {
    const uint64_t stride = align_up(sz[i]);
    *offs[i] = cur;
    L->layer_stride[i] = stride;
    cur += stride * (uint64_t)d->layers;
  }
  L->status = cur;
  cur += align_up(16 * sizeof(int32_t));
  L->total_bytes = cur;
  L->plan_stride = plan_stride(d);
  return FL_OK;
}

CacheView make_view(const fl_dims* d, const fl_layout& L, void* cache) {
  CacheView v;
  std::memset(&v, 0, sizeof(v));
  v.base = static_cast<uint8_t*>(cache);
  const uint64_t offs[A_COUNT] = {L.brec,  L.rrec, L.mask, L.first, L.depth, L.tail_k, L.tail_v,
                                  L.score, L.tag,  L.offset, L.sel, L.mass, L.unsel, L.plan};
  for (int i = 0; i < A_COUNT; ++i) {
    v.off[i] = offs[i];
    v.lstride[i] = L.layer_stride[i];
  }
  for (int r = 0; r <= FL_MAX_LOOPS; ++r) v.slot_base[r] = L.slot_base[r];
  v.status = reinterpret_cast<int32_t*>(v.base + L.status);
  v.H = d->heads;
  v.R = d->loops;
  v.cap = d->capacity;
  v.total_slots = L.total_slots;
  v.max_select = d->max_select;
  v.plan_stride = L.plan_stride;
  v.codec = d->codec;
  return v;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

fl_status cuda_status(cudaError_t e) { return e == cudaSuccess ? FL_OK : FL_ERR_CUDA; }

// Split-K partials the workspace holds: those of the one-layer launches (per head), or those
// of a persistent sparse launch over every layer (per layer and head), whichever is more.
uint64_t ws_partials(const fl_dims* d) {
  const uint64_t one = (uint64_t)d->heads * workspace_splits(d->loops, d->max_select);
  const uint64_t all = (uint64_t)d->layers * d->heads * persist_splits(d->max_select, d->loops);
  return one > all ? one : all;
}
uint64_t ws_part_bytes(const fl_dims* d) { return ws_partials(d) * kPartStride * sizeof(float); }
// completion tickets: one per (layer, head)
uint64_t ws_ticket_bytes(const fl_dims* d) { return (uint64_t)d->layers * d->heads * sizeof(int32_t); }

// The split counts a sparse launch of `loop` over k_sel columns uses, with and without the
// fused flush, fit the workspace's partials (they always do for k_sel <= max_select; checked
// before any launch all the same).
fl_status check_sparse_splits(const fl_dims* d, int loop, int k_sel) {
  const int sms = device_sms();
  const uint64_t one = (uint64_t)d->heads * sparse_launch_splits(d->heads, d->loops, d->codec, loop, k_sel, sms, true);
  const uint64_t all =
      (uint64_t)d->layers * d->heads * sparse_launch_splits(d->heads, d->loops, d->codec, loop, k_sel, sms, false);
  return one <= ws_partials(d) && all <= ws_partials(d) ? FL_OK : FL_ERR_UNSUPPORTED;
}

fl_status check_reader(const fl_dims* d, void* cache, int layer, int loop, int n_q, int n_tail,
                       const uint16_t* q, const uint16_t* k_new, const uint16_t* v_new, float* o,
                       void* ws, size_t ws_bytes) {
  fl_status st = check_dims(d);
  if (st != FL_OK) return st;
  if (!cache || !q || !o) return FL_ERR_INVALID;
  if (layer < 0 || layer >= d->layers || loop < 1 || loop > d->loops) return FL_ERR_INVALID;
  if (n_q < 0 || n_q % FL_GROUP != 0 || n_tail < 1 || n_tail > FL_TAIL) return FL_ERR_INVALID;
  if ((int64_t)n_q + n_tail > d->capacity) return FL_ERR_INVALID;
  if ((k_new == nullptr) != (v_new == nullptr)) return FL_ERR_INVALID;
  if (!aligned16(q) || !aligned16(o) || (k_new && (!aligned16(k_new) || !aligned16(v_new))))
    return FL_ERR_INVALID;
  if (!ws || ws_bytes < fl_workspace_bytes(d)) return FL_ERR_WORKSPACE;
  return FL_OK;
}

// The fused tail flush of layer l's loop-r reader (none when flush is NULL).
void set_flush(ReaderArgs& a, const fl_flush* flush, int l, int r) {
  a.flush = flush ? 1 : 0;
  a.flush_act = flush && r >= 2 ? flush->active[r] : 0ull;
  a.flush_slot0 = flush && r >= 2 ? flush->slot0[(size_t)l * (FL_MAX_LOOPS + 1) + r] : 0;
}

}  // namespace

namespace fl {
namespace {
std::atomic<int> g_sms[kMaxDevices];
}  // namespace

int device_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  int n = g_sms[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    g_sms[dev].store(n, std::memory_order_relaxed);  // the same value from every thread
  }
  return n;
}
}  // namespace fl

extern "C" {

const char* fl_version(void) { return "flashloop-b200 0.1.0 (sm_100a)"; }

const char* fl_status_string(fl_status st) {
  switch (st) {
    case FL_OK: return "FL_OK";
    case FL_ERR_INVALID: return "FL_ERR_INVALID: invalid argument";
    case FL_ERR_UNSUPPORTED: return "FL_ERR_UNSUPPORTED: unsupported shape";
    case FL_ERR_CUDA: return "FL_ERR_CUDA: CUDA runtime or launch error";
    case FL_ERR_WORKSPACE: return "FL_ERR_WORKSPACE: workspace missing or too small";
    case FL_ERR_DEVICE: return "FL_ERR_DEVICE: a kernel recorded a data error";
  }
  return "unknown fl_status";
}

fl_status fl_cache_layout(const fl_dims* dims, fl_layout* out) {
  if (!out) return FL_ERR_INVALID;
  return make_layout(dims, out);
}

fl_status fl_cache_init(const fl_dims* dims, void* cache, void* stream) {
  fl_layout L;
  fl_status st = make_layout(dims, &L);
  if (st != FL_OK) return st;
  if (!cache) return FL_ERR_INVALID;
  return cuda_status(cudaMemsetAsync(cache, 0, L.total_bytes, (cudaStream_t)stream));
}

size_t fl_workspace_bytes(const fl_dims* dims) {
  if (check_dims(dims) != FL_OK) return 0;
  return ws_part_bytes(dims) + align_up(ws_ticket_bytes(dims));
}

fl_status fl_workspace_init(const fl_dims* dims, void* ws, size_t ws_bytes, void* stream) {
  fl_status st = check_dims(dims);
  if (st != FL_OK) return st;
  if (!ws || ws_bytes < fl_workspace_bytes(dims)) return FL_ERR_WORKSPACE;
  return cuda_status(cudaMemsetAsync(static_cast<uint8_t*>(ws) + ws_part_bytes(dims), 0, ws_ticket_bytes(dims),
                                     (cudaStream_t)stream));
}

fl_status fl_write_tail(const fl_dims* dims, void* cache, int32_t layer, int32_t loop, int32_t row0,
                        int32_t n_rows, const uint16_t* k, const uint16_t* v, int64_t head_stride,
                        void* stream) {
  fl_layout L;
  fl_status st = make_layout(dims, &L);
  if (st != FL_OK) return st;
  if (!cache || !k || !v) return FL_ERR_INVALID;
  if (layer < 0 || layer >= dims->layers || loop < 1 || loop > dims->loops) return FL_ERR_INVALID;
  if (row0 < 0 || n_rows < 0 || row0 + n_rows > FL_TAIL || head_stride < (int64_t)n_rows * FL_HEAD_DIM)
    return FL_ERR_INVALID;
  if (n_rows == 0) return FL_OK;
  uint8_t* base = static_cast<uint8_t*>(cache);
  const size_t row_bytes = FL_HEAD_DIM * 2;
  const size_t dpitch = (size_t)FL_TAIL * row_bytes;
  const size_t per_loop = (size_t)dims->heads * dpitch;
  for (int which = 0; which < 2; ++which) {
    uint8_t* dst = base + (which ? L.tail_v : L.tail_k) + L.layer_stride[which ? A_TAILV : A_TAILK] * layer +
                   per_loop * (loop - 1) + (size_t)row0 * row_bytes;
    const uint16_t* src = which ? v : k;
    cudaError_t e = cudaMemcpy2DAsync(dst, dpitch, src, (size_t)head_stride * 2, (size_t)n_rows * row_bytes,
                                      dims->heads, cudaMemcpyDeviceToDevice, (cudaStream_t)stream);
    if (e != cudaSuccess) return FL_ERR_CUDA;
  }
  return FL_OK;
}

fl_status fl_encode_base(const fl_dims* dims, void* cache, int32_t layer, int32_t row0, int32_t n_rows,
                         const uint16_t* k, const uint16_t* v, int64_t head_stride, void* stream) {
  fl_layout L;
  fl_status st = make_layout(dims, &L);
  if (st != FL_OK) return st;
  if (!cache || !k || !v) return FL_ERR_INVALID;
  if (layer < 0 || layer >= dims->layers) return FL_ERR_INVALID;
  if (row0 < 0 || row0 % FL_GROUP || n_rows < 0 || n_rows % FL_GROUP) return FL_ERR_INVALID;
  if ((int64_t)row0 + n_rows > dims->capacity) return FL_ERR_INVALID;
  if (!aligned16(k) || !aligned16(v) || head_stride % 8 || head_stride < (int64_t)n_rows * FL_HEAD_DIM)
    return FL_ERR_INVALID;
  if (n_rows == 0) return FL_OK;
  EncodeBaseArgs a;
  a.c = make_view(dims, L, cache);
  a.layer = layer;
  a.row0 = row0;
  a.n_rows = n_rows;
  a.k = k;
  a.v = v;
  a.head_stride = head_stride;
  return cuda_status(launch_encode_base(a, (cudaStream_t)stream));
}

fl_status fl_encode_residual(const fl_dims* dims, void* cache, int32_t layer, int32_t loop, int32_t row0,
                             int32_t n_span, int32_t slot0, const int32_t* rows, int32_t n_rows,
                             const uint16_t* k, const uint16_t* v, int64_t head_stride, int32_t compact,
                             void* stream) {
  fl_layout L;
  fl_status st = make_layout(dims, &L);
  if (st != FL_OK) return st;
  if (!cache) return FL_ERR_INVALID;
  if (layer < 0 || layer >= dims->layers || loop < 2 || loop > dims->loops) return FL_ERR_INVALID;
  if (row0 < 0 || row0 % FL_GROUP || n_span < 0 || n_span % FL_GROUP) return FL_ERR_INVALID;
  if ((int64_t)row0 + n_span > dims->capacity) return FL_ERR_INVALID;
  if (n_rows < 0 || n_rows > n_span) return FL_ERR_INVALID;
  if (slot0 < 0 || slot0 % FL_GROUP || (int64_t)slot0 + n_rows > dims->res_capacity[loop]) return FL_ERR_INVALID;
  if (n_rows > 0) {
    if (!rows || !k || !v || !aligned16(k) || !aligned16(v) || head_stride % 8) return FL_ERR_INVALID;
    const int64_t rows_in = compact ? n_rows : n_span;
    if (head_stride < rows_in * FL_HEAD_DIM) return FL_ERR_INVALID;
  }
  const int ncb = dims->capacity / FL_GROUP;
  uint8_t* base = static_cast<uint8_t*>(cache);
  const int b0 = row0 / FL_GROUP, nbk = n_span / FL_GROUP;
  cudaStream_t s = (cudaStream_t)stream;
  if (nbk > 0) {
    uint8_t* m = base + L.mask + L.layer_stride[A_MASK] * layer + ((size_t)loop * ncb + b0) * 8;
    uint8_t* f = base + L.first + L.layer_stride[A_FIRST] * layer + ((size_t)loop * ncb + b0) * 4;
    if (cudaMemsetAsync(m, 0, (size_t)nbk * 8, s) != cudaSuccess) return FL_ERR_CUDA;
    if (cudaMemsetAsync(f, 0xff, (size_t)nbk * 4, s) != cudaSuccess) return FL_ERR_CUDA;
  }
  EncodeResArgs a;
  a.c = make_view(dims, L, cache);
  a.layer = layer;
  a.r = loop;
  a.row0 = row0;
  a.n_span = n_span;
  a.slot0 = slot0;
  a.n_rows = n_rows;
  a.compact = compact ? 1 : 0;
  a.rows = rows;
  a.k = k;
  a.v = v;
  a.head_stride = head_stride;
  return cuda_status(launch_encode_residual(a, s));
}

fl_status fl_decode_attn_dense(const fl_dims* dims, void* cache, int32_t layer, int32_t loop, int32_t n_q,
                               int32_t n_tail, const uint16_t* q, const uint16_t* k_new,
                               const uint16_t* v_new, float* o, int32_t keep_scores, void* ws,
                               size_t ws_bytes, void* stream) {
  fl_status st = check_reader(dims, cache, layer, loop, n_q, n_tail, q, k_new, v_new, o, ws, ws_bytes);
  if (st != FL_OK) return st;
  fl_layout L;
  make_layout(dims, &L);
  ReaderArgs a{};
  a.c = make_view(dims, L, cache);
  a.layer = layer;
  a.r = loop;
  a.n_q = n_q;
  a.n_tail = n_tail;
  a.k_sel = 0;
  a.n_splits = 1;
  a.keep = keep_scores ? 1 : 0;
  a.q = q;
  a.k_new = k_new;
  a.v_new = v_new;
  a.o_prev = nullptr;
  a.o = o;
  a.part = static_cast<float*>(ws);
  a.counter = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + ws_part_bytes(dims));
  // a standalone call is an ordinary stream-ordered launch: nothing of it may overlap the
  // caller's preceding kernel (which may be a reader of the same layer)
  return cuda_status(launch_dense(a, (cudaStream_t)stream, false));
}

fl_status fl_select_topk(const fl_dims* dims, void* cache, int32_t layer0, int32_t n_layers, int32_t loop,
                         int32_t n_q, int32_t n_tail, int32_t k_sel, void* stream) {
  fl_layout L;
  fl_status st = make_layout(dims, &L);
  if (st != FL_OK) return st;
  if (!cache) return FL_ERR_INVALID;
  if (layer0 < 0 || n_layers < 1 || (int64_t)layer0 + n_layers > dims->layers) return FL_ERR_INVALID;
  if (loop < 2 || loop > dims->loops) return FL_ERR_INVALID;
  if (n_q < 0 || n_q % FL_GROUP != 0 || n_tail < 1 || n_tail > FL_TAIL) return FL_ERR_INVALID;
  const int64_t N = (int64_t)n_q + n_tail;
  if (N > dims->capacity) return FL_ERR_INVALID;
  if (N > FL_MAX_SELECT_COLS) return FL_ERR_UNSUPPORTED;
  if (k_sel < 1 || k_sel > N || k_sel > dims->max_select) return FL_ERR_INVALID;
  SelectArgs a;
  a.c = make_view(dims, L, cache);
  a.layer0 = layer0;
  a.r = loop;
  a.n_q = n_q;
  a.n_tail = n_tail;
  a.k_sel = k_sel;
  return cuda_status(launch_select(a, n_layers, (cudaStream_t)stream));
}

fl_status fl_decode_attn_sparse(const fl_dims* dims, void* cache, int32_t layer, int32_t loop, int32_t n_q,
                                int32_t n_tail, int32_t k_sel, const uint16_t* q, const uint16_t* k_new,
                                const uint16_t* v_new, const float* o_prev, float* o, void* ws, size_t ws_bytes,
                                void* stream) {
  fl_status st = check_reader(dims, cache, layer, loop, n_q, n_tail, q, k_new, v_new, o, ws, ws_bytes);
  if (st != FL_OK) return st;
  if (!o_prev || loop < 2) return FL_ERR_INVALID;
  const int64_t N = (int64_t)n_q + n_tail;
  if (k_sel < 1 || k_sel > N || k_sel > dims->max_select) return FL_ERR_INVALID;
  st = check_sparse_splits(dims, loop, k_sel);
  if (st != FL_OK) return st;
  fl_layout L;
  make_layout(dims, &L);
  ReaderArgs a{};
  a.c = make_view(dims, L, cache);
  a.layer = layer;
  a.r = loop;
  a.n_q = n_q;
  a.n_tail = n_tail;
  a.k_sel = k_sel;
  a.n_splits = 1;
  a.keep = 1;
  a.q = q;
  a.k_new = k_new;
  a.v_new = v_new;
  a.o_prev = o_prev;
  a.o = o;
  a.part = static_cast<float*>(ws);
  a.counter = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + ws_part_bytes(dims));
  // unchained, like the standalone dense reader
  return cuda_status(launch_sparse(a, (cudaStream_t)stream, false));
}

// ---- sparse reader with library-owned scratch (for callers that cannot allocate) ----
// The scratch is one file-scope device array; its address is looked up once per device
// (cudaGetSymbolAddress, with that device current) and cached here.  Nothing is
// allocated: the array is part of the library's loaded module.
}  // extern "C"
namespace {
__device__ __align__(256) uint8_t g_noalloc_scratch[FL_NOALLOC_SCRATCH_BYTES];
std::atomic<void*> g_noalloc_ptr[kMaxDevices];
}  // namespace
extern "C" {

fl_status fl_decode_attn_sparse_noalloc(const fl_dims* dims, void* cache, int32_t layer, int32_t loop,
                                        int32_t n_q, int32_t n_tail, int32_t k_sel, const uint16_t* q,
                                        const uint16_t* k_new, const uint16_t* v_new, const float* o_prev,
                                        float* o, void* stream) {
  fl_status st = check_dims(dims);
  if (st != FL_OK) return st;
  if (!cache || !q || !o || !o_prev) return FL_ERR_INVALID;
  if (layer < 0 || layer >= dims->layers || loop < 2 || loop > dims->loops) return FL_ERR_INVALID;
  if (n_q < 0 || n_q % FL_GROUP != 0 || n_tail < 1 || n_tail > FL_TAIL) return FL_ERR_INVALID;
  const int64_t N = (int64_t)n_q + n_tail;
  if (N > dims->capacity) return FL_ERR_INVALID;
  if ((k_new == nullptr) != (v_new == nullptr)) return FL_ERR_INVALID;
  if (!aligned16(q) || !aligned16(o) || (k_new && (!aligned16(k_new) || !aligned16(v_new))))
    return FL_ERR_INVALID;
  if (k_sel < 1 || k_sel > N || k_sel > dims->max_select) return FL_ERR_INVALID;
  // scratch: per-head tickets (must start at zero), then the split partials of exactly the
  // split count the launch below uses; a size that no device could fit is refused before
  // any CUDA call (at least ceil(k_sel / columns per CTA) splits per head)
  const uint64_t ticket_bytes = ((uint64_t)dims->heads * sizeof(int32_t) + 255) / 256 * 256;
  const auto scratch_bytes = [&](int splits) {
    return ticket_bytes + (uint64_t)dims->heads * splits * kPartStride * sizeof(float);
  };
  const int cols = sparse_cta_columns(dims->loops);
  if (scratch_bytes((k_sel + cols - 1) / cols) > FL_NOALLOC_SCRATCH_BYTES) return FL_ERR_UNSUPPORTED;
  const int sms = device_sms();
  if (sms <= 0) return FL_ERR_CUDA;
  if (scratch_bytes(sparse_launch_splits(dims->heads, dims->loops, dims->codec, loop, k_sel, sms, false)) >
      FL_NOALLOC_SCRATCH_BYTES)
    return FL_ERR_UNSUPPORTED;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FL_ERR_CUDA;
  void* p = g_noalloc_ptr[dev].load(std::memory_order_acquire);
  if (!p) {
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return FL_ERR_CUDA;
    g_noalloc_ptr[dev].store(p, std::memory_order_release);  // the same address from every thread
  }
  uint8_t* scratch = static_cast<uint8_t*>(p);
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(scratch, 0, (size_t)dims->heads * sizeof(int32_t), s) != cudaSuccess) return FL_ERR_CUDA;
  fl_layout L;
  make_layout(dims, &L);
  ReaderArgs a{};
  a.c = make_view(dims, L, cache);
  a.layer = layer;
  a.r = loop;
  a.n_q = n_q;
  a.n_tail = n_tail;
  a.k_sel = k_sel;
  a.n_splits = 1;
  a.keep = 1;
  a.q = q;
  a.k_new = k_new;
  a.v_new = v_new;
  a.o_prev = o_prev;
  a.o = o;
  a.counter = reinterpret_cast<int32_t*>(scratch);
  a.part = reinterpret_cast<float*>(scratch + ticket_bytes);
  return cuda_status(launch_sparse(a, s, false));
}

fl_status fl_sparse_splits(const fl_dims* dims, int32_t loop, int32_t k_sel, int32_t sm_count, int32_t* splits,
                           int32_t* capacity) {
  fl_status st = check_dims(dims);
  if (st != FL_OK) return st;
  if (!splits || loop < 2 || loop > dims->loops || k_sel < 1 || k_sel > dims->max_select || sm_count < 1)
    return FL_ERR_INVALID;
  *splits = sparse_launch_splits(dims->heads, dims->loops, dims->codec, loop, k_sel, sm_count, false);
  if (capacity) *capacity = (int32_t)(ws_partials(dims) / ((uint64_t)dims->layers * dims->heads));
  return FL_OK;
}

fl_status fl_decode_step(const fl_dims* dims, void* cache, int32_t n_q, int32_t n_tail, int32_t dense_loops,
                         int32_t k_sel, int32_t loop_first, int32_t loop_last, const uint16_t* q,
                         const uint16_t* k_new, const uint16_t* v_new, float* o, void* ws, size_t ws_bytes,
                         void* const* events, void* stream) {
  return fl_decode_step_flush(dims, cache, n_q, n_tail, dense_loops, k_sel, loop_first, loop_last, q, k_new, v_new,
                              o, ws, ws_bytes, events, nullptr, stream);
}

namespace {
// The executor behind fl_decode_step_flush and fl_decode_step_io: with `inputs_ready`, the
// stream waits on that event before its first reader (the selection before it reads no
// query), so a host -> device copy of the inputs can overlap the loop's selection.
fl_status decode_step(const fl_dims* dims, void* cache, int32_t n_q, int32_t n_tail, int32_t dense_loops,
                      int32_t k_sel, int32_t loop_first, int32_t loop_last, const uint16_t* q, const uint16_t* k_new,
                      const uint16_t* v_new, float* o, void* ws, size_t ws_bytes, void* const* events,
                      const fl_flush* flush, void* stream, cudaEvent_t inputs_ready, bool validate_only = false) {
  fl_status st = check_reader(dims, cache, 0, 1, n_q, n_tail, q, k_new, v_new, o, ws, ws_bytes);
  if (st != FL_OK) return st;
  const int R = dims->loops, L = dims->layers, H = dims->heads;
  if (dense_loops < 0 || dense_loops > R || loop_first < 1 || loop_last > R || loop_first > loop_last)
    return FL_ERR_INVALID;
  if (flush) {
    if (dims->codec != FL_CODEC_RESIDUAL_INT4) return FL_ERR_UNSUPPORTED;  // the fused flush writes 4-bit residuals
    if (n_tail != FL_TAIL || (int64_t)n_q + FL_TAIL > dims->capacity || !flush->slot0) return FL_ERR_INVALID;
    uint64_t prev = ~0ull;
    for (int r = 2; r <= R; ++r) {
      const uint64_t act = flush->active[r];
      if (act & ~prev) return FL_ERR_INVALID;  // the active sets nest
      prev = act;
      if (!act) continue;
      const int nr = __builtin_popcountll(act);
      for (int l = 0; l < L; ++l) {
        const int32_t s0 = flush->slot0[(size_t)l * (FL_MAX_LOOPS + 1) + r];
        if (s0 < 0 || s0 % FL_GROUP || (int64_t)s0 + nr > dims->res_capacity[r]) return FL_ERR_INVALID;
      }
    }
  }
  const int64_t N = (int64_t)n_q + n_tail;
  const bool any_sparse = loop_last > dense_loops;
  if (any_sparse) {
    if (N > FL_MAX_SELECT_COLS) return FL_ERR_UNSUPPORTED;
    if (k_sel < 1 || k_sel > N || k_sel > dims->max_select) return FL_ERR_INVALID;
    if (loop_first == 1 && dense_loops == 0) return FL_ERR_INVALID;  // a sparse loop needs a predecessor
    for (int r = loop_first > dense_loops + 1 ? loop_first : dense_loops + 1; r <= loop_last; ++r) {
      st = check_sparse_splits(dims, r, k_sel);
      if (st != FL_OK) return st;
    }
  }
  if (validate_only) return FL_OK;
  fl_layout lay;
  make_layout(dims, &lay);
  cudaStream_t s = (cudaStream_t)stream;
  const size_t row = (size_t)H * FL_HEAD_DIM;              // one (loop, layer) slice
  const size_t ostride_r = (size_t)L * row;                // elements between loops
  auto rec = [&](int i) -> bool {
    return !events || cudaEventRecord((cudaEvent_t)events[i], s) == cudaSuccess;
  };
  auto wait_inputs = [&]() -> bool {
    const bool ok = !inputs_ready || cudaStreamWaitEvent(s, inputs_ready, 0) == cudaSuccess;
    inputs_ready = nullptr;
    return ok;
  };
  ReaderArgs a{};
  a.c = make_view(dims, lay, cache);
  a.o_prev = nullptr;
  a.n_q = n_q;
  a.n_tail = n_tail;
  a.k_sel = k_sel;
  a.n_splits = 1;
  a.part = static_cast<float*>(ws);
  a.counter = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + ws_part_bytes(dims));
  // the step's first reader is an ordinary launch: nothing of it runs before the
  // previous step (including its tail flush) has completed
  bool first_launch = true;
  if (!rec(0)) return FL_ERR_CUDA;
  for (int r = loop_first; r <= loop_last; ++r) {
    a.r = r;
    if (r <= dense_loops) {
      if (!rec(2 * r - 1)) return FL_ERR_CUDA;
      a.keep = r == dense_loops ? 1 : 0;
      if (!wait_inputs()) return FL_ERR_CUDA;
      for (int l = 0; l < L; ++l) {
        const size_t qo = (size_t)r * ostride_r + (size_t)l * row;
        a.layer = l;
        a.q = q + qo;
        a.k_new = k_new ? k_new + qo : nullptr;
        a.v_new = v_new ? v_new + qo : nullptr;
        a.o = o + qo;
        set_flush(a, flush, l, r);
        if (launch_dense(a, s, !first_launch) != cudaSuccess) return FL_ERR_CUDA;
        first_launch = false;
      }
    } else {
      SelectArgs sa;
      sa.c = a.c;
      sa.layer0 = 0;
      sa.r = r;
      sa.n_q = n_q;
      sa.n_tail = n_tail;
      sa.k_sel = k_sel;
      if (launch_select(sa, L, s) != cudaSuccess) return FL_ERR_CUDA;
      if (!rec(2 * r - 1)) return FL_ERR_CUDA;
      if (!wait_inputs()) return FL_ERR_CUDA;
      a.keep = 1;
      if (dims->codec == FL_CODEC_RESIDUAL_INT4 && r <= kPersistMaxLoop) {
        // every layer of the loop through the persistent reader: one launch (per
        // kFlushLayersMax layers with the fused flush)
        const int span = flush ? kFlushLayersMax : L;
        for (int l0 = 0; l0 < L; l0 += span) {
          const size_t qo = (size_t)r * ostride_r + (size_t)l0 * row;
          a.layer = l0;
          a.n_layers = L - l0 < span ? L - l0 : span;
          a.io_layer_stride = (int64_t)row;
          a.q = q + qo;
          a.k_new = k_new ? k_new + qo : nullptr;
          a.v_new = v_new ? v_new + qo : nullptr;
          a.o = o + qo;
          a.o_prev = o + qo - ostride_r;
          set_flush(a, flush, l0, r);
          if (flush)
            for (int i = 0; i < a.n_layers; ++i)
              a.flush_slot0s[i] = flush->slot0[(size_t)(l0 + i) * (FL_MAX_LOOPS + 1) + r];
          if (launch_sparse(a, s) != cudaSuccess) return FL_ERR_CUDA;
        }
        a.layer = 0;
        a.n_layers = 1;
        a.io_layer_stride = 0;
      } else {
        for (int l = 0; l < L; ++l) {
          const size_t qo = (size_t)r * ostride_r + (size_t)l * row;
          a.layer = l;
          a.q = q + qo;
          a.k_new = k_new ? k_new + qo : nullptr;
          a.v_new = v_new ? v_new + qo : nullptr;
          a.o = o + qo;
          a.o_prev = o + qo - ostride_r;
          set_flush(a, flush, l, r);
          if (launch_sparse(a, s) != cudaSuccess) return FL_ERR_CUDA;
        }
      }
    }
    if (!rec(2 * r)) return FL_ERR_CUDA;
  }
  return FL_OK;
}

// per device, the stream fl_decode_step_io copies its inputs on (created on first use)
std::atomic<bool> g_side_done[kMaxDevices];
std::mutex g_side_mu;
cudaStream_t g_side[kMaxDevices];
}  // namespace

fl_status fl_decode_step_flush(const fl_dims* dims, void* cache, int32_t n_q, int32_t n_tail, int32_t dense_loops,
                               int32_t k_sel, int32_t loop_first, int32_t loop_last, const uint16_t* q,
                               const uint16_t* k_new, const uint16_t* v_new, float* o, void* ws, size_t ws_bytes,
                               void* const* events, const fl_flush* flush, void* stream) {
  return decode_step(dims, cache, n_q, n_tail, dense_loops, k_sel, loop_first, loop_last, q, k_new, v_new, o, ws,
                     ws_bytes, events, flush, stream, nullptr);
}

fl_status fl_decode_step_io(const fl_dims* dims, void* cache, int32_t n_q, int32_t n_tail, int32_t dense_loops,
                            int32_t k_sel, int32_t loop_first, int32_t loop_last, uint16_t* qkv, const uint16_t* host_qkv,
                            float* o, float* host_o, void* ws, size_t ws_bytes, void* const* events,
                            const fl_flush* flush, void* stream) {
  fl_status st = check_dims(dims);
  if (st != FL_OK) return st;
  if (!qkv || !host_qkv || !o || !host_o) return FL_ERR_INVALID;
  const int R = dims->loops;
  if (loop_first < 1 || loop_last > R || loop_first > loop_last) return FL_ERR_INVALID;
  const size_t slice = (size_t)dims->layers * dims->heads * FL_HEAD_DIM;  // one (loop) slice of L x H x 128
  const size_t nl = (size_t)(loop_last - loop_first + 1);
  uint16_t* q = qkv;
  uint16_t* kn = qkv + (size_t)(R + 1) * slice;
  uint16_t* vn = qkv + (size_t)2 * (R + 1) * slice;
  cudaStream_t s = (cudaStream_t)stream;
  // validate the whole step before anything is enqueued
  st = decode_step(dims, cache, n_q, n_tail, dense_loops, k_sel, loop_first, loop_last, q, kn, vn, o, ws, ws_bytes,
                   events, flush, stream, nullptr, true);
  if (st != FL_OK) return st;
  // q, k_new, v_new of loops loop_first..loop_last (three equally spaced device rows) are
  // copied on a side stream once the stream's earlier work is done, beside the first
  // loop's selection; the first reader waits for them
  if (once_per_device(g_side_done, g_side_mu, [](int dev) {
        return cudaStreamCreateWithFlags(&g_side[dev], cudaStreamNonBlocking);
      }) != cudaSuccess)
    return FL_ERR_CUDA;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FL_ERR_CUDA;
  const cudaStream_t side = g_side[dev];
  cudaEvent_t ev_start = nullptr, ev_copied = nullptr;
  auto release = [&]() {
    if (ev_start) cudaEventDestroy(ev_start);
    if (ev_copied) cudaEventDestroy(ev_copied);
  };
  if (cudaEventCreateWithFlags(&ev_start, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&ev_copied, cudaEventDisableTiming) != cudaSuccess || cudaEventRecord(ev_start, s) != cudaSuccess ||
      cudaStreamWaitEvent(side, ev_start, 0) != cudaSuccess ||
      cudaMemcpy2DAsync(q + (size_t)loop_first * slice, (size_t)(R + 1) * slice * 2, host_qkv, nl * slice * 2,
                        nl * slice * 2, 3, cudaMemcpyHostToDevice, side) != cudaSuccess ||
      cudaEventRecord(ev_copied, side) != cudaSuccess) {
    release();
    return FL_ERR_CUDA;
  }
  st = decode_step(dims, cache, n_q, n_tail, dense_loops, k_sel, loop_first, loop_last, q, kn, vn, o, ws, ws_bytes,
                   events, flush, stream, ev_copied);
  release();  // destroyed once their work is done
  if (st != FL_OK) return st;
  if (cudaMemcpyAsync(host_o, o + (size_t)loop_first * slice, nl * slice * sizeof(float), cudaMemcpyDeviceToHost,
                      s) != cudaSuccess)
    return FL_ERR_CUDA;
  return FL_OK;
}

fl_status fl_select_active(const uint16_t* h_prev, const uint16_t* h_cur, int32_t n_tokens, int32_t d_model,
                           int64_t row_stride, const int32_t* rows, int32_t n_rows, int32_t k, int32_t* rows_out,
                           double* keys, int32_t* status, void* stream) {
  if (n_tokens < 1 || d_model < 8 || d_model % 8 || row_stride < d_model || row_stride % 8) return FL_ERR_INVALID;
  if (n_rows < 0 || n_rows > n_tokens || k < 0 || k > n_rows) return FL_ERR_INVALID;
  if (n_rows > 0 && (!h_prev || !h_cur || !rows || !keys || !aligned16(h_prev) || !aligned16(h_cur)))
    return FL_ERR_INVALID;
  if (k > 0 && !rows_out) return FL_ERR_INVALID;
  if (reinterpret_cast<uintptr_t>(keys) % 8 || reinterpret_cast<uintptr_t>(status) % 4) return FL_ERR_INVALID;
  TokenArgs a;
  a.h_prev = h_prev;
  a.h_cur = h_cur;
  a.row_stride = row_stride;
  a.d_model = d_model;
  a.n_tokens = n_tokens;
  a.rows = rows;
  a.n_rows = n_rows;
  a.k = k;
  a.rows_out = rows_out;
  a.keys = keys;
  a.status = status;
  return cuda_status(launch_token_select(a, (cudaStream_t)stream));
}

fl_status fl_prefill_attn_sparse(const uint16_t* q, const int32_t* pos, int32_t n_act, const uint16_t* k,
                                 const uint16_t* v, int32_t n_tokens, int32_t heads, int64_t q_head_stride,
                                 int64_t kv_head_stride, float* o, int64_t o_head_stride, int32_t* status,
                                 void* stream) {
  if (n_act < 0 || n_tokens < 1 || heads < 1 || n_act > n_tokens) return FL_ERR_INVALID;
  if (n_act == 0) return FL_OK;
  if (!q || !pos || !k || !v || !o) return FL_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return FL_ERR_INVALID;
  if (reinterpret_cast<uintptr_t>(pos) % 4 || reinterpret_cast<uintptr_t>(status) % 4) return FL_ERR_INVALID;
  if (q_head_stride % 8 || kv_head_stride % 8 || o_head_stride % 4) return FL_ERR_INVALID;
  if (heads > 1 && (q_head_stride < (int64_t)n_act * FL_HEAD_DIM || kv_head_stride < (int64_t)n_tokens * FL_HEAD_DIM ||
                    o_head_stride < (int64_t)n_act * FL_HEAD_DIM))
    return FL_ERR_INVALID;
  if ((int64_t)heads > 65535) return FL_ERR_UNSUPPORTED;
  PrefillArgs a;
  a.q = q;
  a.pos = pos;
  a.n_act = n_act;
  a.n_tokens = n_tokens;
  a.heads = heads;
  a.k = k;
  a.v = v;
  a.q_head_stride = q_head_stride;
  a.kv_head_stride = kv_head_stride;
  a.o_head_stride = o_head_stride;
  a.o = o;
  a.status = status;
  return cuda_status(launch_prefill_attn(a, (cudaStream_t)stream));
}

fl_status fl_read_status(const fl_dims* dims, void* cache, int32_t* out, int32_t clear, void* stream) {
  fl_layout L;
  fl_status st = make_layout(dims, &L);
  if (st != FL_OK) return st;
  if (!cache || !out) return FL_ERR_INVALID;
  cudaStream_t s = (cudaStream_t)stream;
  int32_t* dev = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(cache) + L.status);
  if (cudaMemcpyAsync(out, dev, 3 * sizeof(int32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess) return FL_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return FL_ERR_CUDA;
  if (clear) {
    if (cudaMemsetAsync(dev, 0, 16 * sizeof(int32_t), s) != cudaSuccess) return FL_ERR_CUDA;
  }
  return out[0] != 0 ? FL_ERR_DEVICE : FL_OK;
}

}  // extern "C"
