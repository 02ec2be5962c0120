// C ABI of libcalibatt.so (declared in include/calibatt.h): argument
// validation, the mask dictionary with its longest-processing-time schedules,
// TMA tensor-map encoding and kernel dispatch.  All host logic is here; the
// kernels live in attn_tc.cu, attn_simt.cu and energy.cu.
#include "calibatt.h"
#include "internal.h"

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <functional>
#include <memory>
#include <mutex>
#include <numeric>
#include <queue>
#include <string>
#include <utility>
#include <vector>

using calibatt::AnchorGeom;
using calibatt::LayerSchedule;
using calibatt::SimtParams;
using calibatt::TcParams;

namespace {

thread_local std::string g_last_error;
std::atomic<unsigned long long> g_timeout_ns{4000000000ull};

__device__ int32_t g_status_word;

calibatt_status fail(calibatt_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

calibatt_status cuda_fail(cudaError_t e, const char* what) {
  cudaGetLastError();  // clear the sticky-free error state
  return fail(e == cudaErrorMemoryAllocation ? CALIBATT_ERR_OOM : CALIBATT_ERR_CUDA, "%s: %s", what,
              cudaGetErrorString(e));
}

int32_t* status_word_ptr() {
  static std::mutex mu;
  static int32_t* ptrs[128] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    ptrs[dev] = static_cast<int32_t*>(p);
  }
  return ptrs[dev];
}

int device_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  return n;
}

int ceil_div(int64_t a, int64_t b) { return static_cast<int>((a + b - 1) / b); }

// ------------------------------------------------------------- schedule

void lpt(int32_t n, const int64_t* cost, int32_t bins, int32_t* bin_ptr, int32_t* order,
         int64_t* makespan) {
  std::vector<int32_t> idx(n);
  std::iota(idx.begin(), idx.end(), 0);
  std::stable_sort(idx.begin(), idx.end(), [&](int32_t a, int32_t b) { return cost[a] > cost[b]; });
  using Slot = std::pair<int64_t, int32_t>;  // (load, bin): least load, then lowest bin
  std::priority_queue<Slot, std::vector<Slot>, std::greater<Slot>> heap;
  for (int32_t b = 0; b < bins; ++b) heap.push({0, b});
  std::vector<std::vector<int32_t>> per_bin(bins);
  for (int32_t i : idx) {
    Slot s = heap.top();
    heap.pop();
    per_bin[s.second].push_back(i);
    heap.push({s.first + cost[i], s.second});
  }
  int64_t mk = 0;
  while (!heap.empty()) {
    mk = std::max(mk, heap.top().first);
    heap.pop();
  }
  int32_t pos = 0;
  for (int32_t b = 0; b < bins; ++b) {
    bin_ptr[b] = pos;
    for (int32_t i : per_bin[b]) order[pos++] = i;
  }
  bin_ptr[bins] = pos;
  if (makespan) *makespan = mk;
}

// LPT over consecutive groups of items: inside a group, items in descending
// cost go to the least-loaded bin; bin loads carry over from group to group,
// and every bin lists its items group by group.  With one group per few heads
// the persistent CTAs move through the heads roughly together, so the keys and
// values of the heads in flight stay resident in L2.
void lpt_grouped(int32_t n, const int64_t* cost, const int32_t* group, int32_t bins, int32_t* bin_ptr,
                 int32_t* order) {
  std::vector<int32_t> idx(n);
  std::iota(idx.begin(), idx.end(), 0);
  std::stable_sort(idx.begin(), idx.end(), [&](int32_t a, int32_t b) {
    return group[a] != group[b] ? group[a] < group[b] : cost[a] > cost[b];
  });
  using Slot = std::pair<int64_t, int32_t>;
  std::priority_queue<Slot, std::vector<Slot>, std::greater<Slot>> heap;
  for (int32_t b = 0; b < bins; ++b) heap.push({0, b});
  std::vector<std::vector<int32_t>> per_bin(bins);
  for (int32_t i : idx) {
    Slot s = heap.top();
    heap.pop();
    per_bin[s.second].push_back(i);
    heap.push({s.first + cost[i], s.second});
  }
  int32_t pos = 0;
  for (int32_t b = 0; b < bins; ++b) {
    bin_ptr[b] = pos;
    for (int32_t i : per_bin[b]) order[pos++] = i;
  }
  bin_ptr[bins] = pos;
}

// Heads whose keys and values (at head_dim 128) fit together in about 40 MB
// of L2, a third of it and within one die's half.  On the 720p call (38.7 MB
// per head) one, two and three heads per group measured 35.4, 36.8 and
// 38.4 ms in one run: the fewer heads in flight, the fewer K/V re-reads.
#ifndef CALIBATT_L2_GROUP_MB
#define CALIBATT_L2_GROUP_MB 40
#endif
int32_t heads_per_group(int32_t nq) {
  const int64_t per_head = static_cast<int64_t>(nq) * 128 * 128 * 2 * 2;
  return static_cast<int32_t>(std::max<int64_t>(1, (static_cast<int64_t>(CALIBATT_L2_GROUP_MB) << 20) / per_head));
}

// Items in the order the CTAs take them under dynamic assignment: group by
// group, cost descending inside a group (ties by position) -- the order in
// which the LPT lists are dealt out.
std::vector<int32_t> consumption_order(const std::vector<int64_t>& cost, const std::vector<int32_t>& group) {
  std::vector<int32_t> idx(cost.size());
  std::iota(idx.begin(), idx.end(), 0);
  std::stable_sort(idx.begin(), idx.end(), [&](int32_t a, int32_t b) {
    return group[a] != group[b] ? group[a] < group[b] : cost[a] > cost[b];
  });
  return idx;
}

// Dictionary calls assign work dynamically (a ticket counter per call) unless
// built with CALIBATT_DYNAMIC=0 (static per-CTA lists, as the direct-CSR call).
#ifndef CALIBATT_DYNAMIC
#define CALIBATT_DYNAMIC 1
#endif
constexpr int kTicketSlots = 64;

// Schedule group of the work item (k-th sparse head of the layer, query block
// r).  Heads go in L2 groups of heads_per_group; with waves on, each head
// group is further cut into waves of `grid` consecutive query blocks (in head,
// then query-block order), so that every CTA takes about one item per wave and
// the grid sweeps each head in query-block order: the keys and values in use
// at a time are the band around the current wave (plus the first frame's and
// the scattered blocks) rather than the whole head's.
#ifndef CALIBATT_WAVES
#define CALIBATT_WAVES 1
#endif
int32_t schedule_group(int32_t k, int32_t r, int32_t nq, int32_t hpg, int32_t grid) {
  if (!CALIBATT_WAVES) return k / hpg;
  const int64_t per_group = static_cast<int64_t>(hpg) * nq;
  const int64_t waves = (per_group + grid - 1) / grid;
  const int64_t pos = static_cast<int64_t>(k % hpg) * nq + r;
  return static_cast<int32_t>((k / hpg) * waves + pos / grid);
}

// ------------------------------------------------------------ tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    cudaGetLastError();
  });
  return fn;
}

// 4-D bf16 map {D, x1, x2, x3} with (x1, x2, x3) the N, H, batch dimensions in
// increasing stride order; box {64, 128 rows of N, 1, 1}, 128-byte swizzle.
// The N extent is seq_len, so rows past the valid tokens read as zeros.
calibatt_status encode_qkv_map(CUtensorMap* map, const void* base, const calibatt_shape& s, int* pos_n,
                               int* pos_h, int* pos_b) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(CALIBATT_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  struct Dim {
    int64_t stride;
    uint64_t size;
    int which;  // 0 = N, 1 = H, 2 = batch
  } d[3] = {{s.stride_n, static_cast<uint64_t>(s.seq_len), 0},
            {s.stride_h, static_cast<uint64_t>(s.heads), 1},
            {s.stride_b, static_cast<uint64_t>(s.batch), 2}};
  std::stable_sort(d, d + 3, [](const Dim& a, const Dim& b) { return a.stride < b.stride; });
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(s.head_dim), d[0].size, d[1].size, d[2].size};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(d[0].stride * 2), static_cast<cuuint64_t>(d[1].stride * 2),
                           static_cast<cuuint64_t>(d[2].stride * 2)};
  cuuint32_t box[4] = {64, d[0].which == 0 ? 128u : 1u, d[1].which == 0 ? 128u : 1u, d[2].which == 0 ? 128u : 1u};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  for (int i = 0; i < 3; ++i) {
    if (d[i].which == 0) *pos_n = i + 1;
    if (d[i].which == 1) *pos_h = i + 1;
    if (d[i].which == 2) *pos_b = i + 1;
  }
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(CALIBATT_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
  return CALIBATT_OK;
}

// ------------------------------------------------------------ validation

calibatt_status check_shape(const calibatt_shape* s) {
  if (!s) return fail(CALIBATT_ERR_INVALID_ARG, "shape is NULL");
  if (s->reserved != 0) return fail(CALIBATT_ERR_INVALID_ARG, "shape.reserved must be 0");
  if (s->batch < 1 || s->seq_len < 1 || s->heads < 1)
    return fail(CALIBATT_ERR_INVALID_ARG, "batch, seq_len and heads must be >= 1 (got %d, %d, %d)", s->batch,
                s->seq_len, s->heads);
  if (s->heads > 65535) return fail(CALIBATT_ERR_UNSUPPORTED, "heads must be <= 65535");
  if (s->head_dim != 64 && s->head_dim != 128)
    return fail(CALIBATT_ERR_UNSUPPORTED, "head_dim %d not supported (64 or 128)", s->head_dim);
  if (s->dtype != CALIBATT_DTYPE_BF16 && s->dtype != CALIBATT_DTYPE_FP32)
    return fail(CALIBATT_ERR_UNSUPPORTED, "dtype %d not supported", s->dtype);
  if (s->stride_b < 1 || s->stride_n < 1 || s->stride_h < 1)
    return fail(CALIBATT_ERR_INVALID_ARG, "strides must be positive");
  const int64_t align = s->dtype == CALIBATT_DTYPE_BF16 ? 8 : 4;
  if (s->stride_b % align || s->stride_n % align || s->stride_h % align)
    return fail(CALIBATT_ERR_INVALID_ARG, "strides must be multiples of %lld elements (16 bytes)", (long long)align);
  if (s->stride_n < s->head_dim && s->stride_h < s->head_dim)
    return fail(CALIBATT_ERR_INVALID_ARG, "rows of head_dim elements overlap (stride_n and stride_h < head_dim)");
  return CALIBATT_OK;
}

calibatt_status check_ptrs(const void* q, const void* k, const void* v, const void* o) {
  if (!q || !k || !v || !o) return fail(CALIBATT_ERR_INVALID_ARG, "q, k, v and o must be non-NULL");
  for (const void* p : {q, k, v, o})
    if (reinterpret_cast<uintptr_t>(p) % 16)
      return fail(CALIBATT_ERR_INVALID_ARG, "q, k, v and o must be 16-byte aligned");
  return CALIBATT_OK;
}

calibatt_status check_block(int32_t block) {
  if (block != 64 && block != 128) return fail(CALIBATT_ERR_UNSUPPORTED, "block %d not supported (64 or 128)", block);
  return CALIBATT_OK;
}

calibatt_status validate_csr(int32_t nq, int32_t nk, const int32_t* row_ptr, const int32_t* col_idx,
                             bool require_diag, const char* what) {
  if (nq < 0 || nk < 1) return fail(CALIBATT_ERR_INVALID_ARG, "%s: nq must be >= 0 and nk >= 1", what);
  if (!row_ptr) return fail(CALIBATT_ERR_INVALID_ARG, "%s: row_ptr is NULL", what);
  if (row_ptr[0] != 0) return fail(CALIBATT_ERR_INVALID_ARG, "%s: row_ptr[0] = %d, expected 0", what, row_ptr[0]);
  for (int32_t r = 0; r < nq; ++r)
    if (row_ptr[r + 1] < row_ptr[r])
      return fail(CALIBATT_ERR_INVALID_ARG, "%s: row_ptr decreases at row %d", what, r);
  if (row_ptr[nq] > 0 && !col_idx) return fail(CALIBATT_ERR_INVALID_ARG, "%s: col_idx is NULL", what);
  if (require_diag && nq != nk)
    return fail(CALIBATT_ERR_INVALID_ARG, "%s: diagonal requested but nq %d != nk %d", what, nq, nk);
  for (int32_t r = 0; r < nq; ++r) {
    bool diag = false;
    for (int32_t i = row_ptr[r]; i < row_ptr[r + 1]; ++i) {
      const int32_t c = col_idx[i];
      if (c < 0 || c >= nk)
        return fail(CALIBATT_ERR_INVALID_ARG, "%s: row %d column %d outside [0, %d)", what, r, c, nk);
      if (i > row_ptr[r] && c <= col_idx[i - 1])
        return fail(CALIBATT_ERR_INVALID_ARG, "%s: row %d columns not strictly ascending", what, r);
      diag |= (c == r);
    }
    if (require_diag && !diag) return fail(CALIBATT_ERR_INVALID_ARG, "%s: row %d lacks its diagonal block", what, r);
  }
  return CALIBATT_OK;
}

// Rows of a frame served by each anchor: nearest anchor, distance ties to the lower one.
void anchor_groups(int32_t rows, const int32_t* anchors, int32_t n, AnchorGeom& g) {
  for (int a = 0; a < n; ++a) {
    g.anchor_row[a] = static_cast<int16_t>(anchors[a]);
    g.group_lo[a] = static_cast<int16_t>(rows);
    g.group_hi[a] = -1;
  }
  for (int32_t rho = 0; rho < rows; ++rho) {
    int best = 0;
    for (int a = 1; a < n; ++a)
      if (std::abs(rho - anchors[a]) < std::abs(rho - anchors[best])) best = a;
    g.group_lo[best] = static_cast<int16_t>(std::min<int>(g.group_lo[best], rho));
    g.group_hi[best] = static_cast<int16_t>(std::max<int>(g.group_hi[best], rho));
  }
}

float scale_log2_of(float softmax_scale, int head_dim) {
  const double sc = softmax_scale > 0.f ? static_cast<double>(softmax_scale) : 1.0 / std::sqrt(static_cast<double>(head_dim));
  return static_cast<float>(sc * 1.4426950408889634);
}

}  // namespace

namespace calibatt {
void set_last_error(const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
}
}  // namespace calibatt

// ================================================================ dictionary

struct calibatt_dict {
  int32_t T = 0, L = 0, H = 0, nq = 0, nk = 0, block = 0, G = 0;
  int32_t device = 0;
  int64_t nnz_cap = 0, nnz_used = 0;
  int32_t* d_row_ptr = nullptr;
  int64_t* d_col_base = nullptr;
  uint16_t* d_col = nullptr;
  uint32_t* d_items = nullptr;
  int32_t* d_cta_ptr = nullptr;
  int64_t device_bytes = 0;
  std::vector<uint8_t> layer_set;   // [T*L]
  std::vector<uint8_t> rep;         // [T*L*H]
  std::vector<int32_t> n_sparse;    // [T*L]
  std::vector<int32_t> n_rep;       // [T*L]
  std::vector<int64_t> retained;    // [T*L]
  // Anchor geometry of the dual path (calibatt_dict_set_anchor_geometry) and
  // the joint sparse + anchor schedules built with it, one per layer.
  // Bitmap format (calibatt_dict_create_bitmap): one bit per (query block,
  // key block) per record instead of index lists.
  bool bitmap = false;
  int32_t words = 0;
  uint32_t* d_bitmap = nullptr;
  bool has_geom = false;
  int32_t g_frames = 0, g_rows = 0, g_cols = 0, g_tiles = 0;
  std::vector<int32_t> g_anchors;
  int64_t f_stride = 0;              // item slots per layer
  uint32_t* d_fitems = nullptr;
  int32_t* d_fcta_ptr = nullptr;
  // Interval format (calibatt_dict_create_intervals): per row, contiguous
  // key-block runs (start | length << 16) instead of one index per block;
  // nnz_cap / nnz_used then count runs and blocks_used the retained blocks.
  bool intervals = false;
  int32_t* d_run_ptr = nullptr;
  uint32_t* d_runs = nullptr;
  int64_t blocks_used = 0;
  // Dynamic assignment: per layer, the items in consumption order (sparse
  // schedule and joint schedule), their counts, and a pool of ticket counters
  // taken round-robin by the calls, so that calls in flight together on
  // different streams use different counters.
  uint32_t* d_order = nullptr;   // [layers][H * nq]
  uint32_t* d_forder = nullptr;  // [layers][f_stride]
  std::vector<int32_t> n_order, n_forder;
  uint32_t* d_tickets = nullptr;  // [kTicketSlots]
  mutable std::atomic<uint32_t> next_ticket{0};

  int64_t layer(int t, int l) const { return static_cast<int64_t>(t) * L + l; }

  LayerSchedule fused_schedule(int t, int l) const {
    LayerSchedule s = schedule(t, l);
    const int64_t ly = layer(t, l);
    s.items = d_fitems + ly * f_stride;
    s.cta_ptr = d_fcta_ptr + ly * (G + 1);
    return s;
  }

  // Dynamic assignment for one call on `stream`: a ticket counter from the
  // pool (round-robin), zeroed on the stream ahead of the launch, and the
  // layer's consumption order.  Returns false if the counter cannot be set.
  bool take_ticket(LayerSchedule& s, int t, int l, bool fused, cudaStream_t stream) const {
    if (!CALIBATT_DYNAMIC) return true;
    const int64_t ly = layer(t, l);
    const uint32_t slot = next_ticket.fetch_add(1u) % kTicketSlots;
    if (cudaMemsetAsync(d_tickets + slot, 0, sizeof(uint32_t), stream) != cudaSuccess) return false;
    s.ticket = d_tickets + slot;
    s.order = fused ? d_forder + ly * f_stride : d_order + ly * H * nq;
    s.n_order = fused ? n_forder[ly] : n_order[ly];
    return true;
  }

  LayerSchedule schedule(int t, int l) const {
    const int64_t ly = layer(t, l);
    LayerSchedule s{};
    s.row_ptr = d_row_ptr + ly * H * (nq + 1);
    s.col_base = d_col_base + ly * H;
    s.col = d_col;
    s.items = d_items + ly * H * nq;
    s.cta_ptr = d_cta_ptr + ly * (G + 1);
    s.nq = nq;
    s.bitmap = bitmap ? d_bitmap + ly * H * nq * static_cast<int64_t>(words) : nullptr;
    s.words = words;
    if (intervals) {
      s.col = nullptr;
      s.run_ptr = d_run_ptr + ly * H * (nq + 1);
      s.runs = d_runs;
    }
    s.csr_gate = 0;  // lists validated on the host when the layer was set
    return s;
  }

  void release() {
    cudaFree(d_order);
    cudaFree(d_forder);
    cudaFree(d_tickets);
    d_order = d_forder = d_tickets = nullptr;
    cudaFree(d_row_ptr);
    cudaFree(d_col_base);
    cudaFree(d_col);
    cudaFree(d_items);
    cudaFree(d_cta_ptr);
    cudaFree(d_fitems);
    cudaFree(d_fcta_ptr);
    cudaFree(d_bitmap);
    cudaFree(d_run_ptr);
    cudaFree(d_runs);
    d_run_ptr = nullptr;
    d_runs = nullptr;
    d_bitmap = nullptr;
    d_fitems = nullptr;
    d_fcta_ptr = nullptr;
    d_row_ptr = nullptr;
    d_col_base = nullptr;
    d_col = nullptr;
    d_items = nullptr;
    d_cta_ptr = nullptr;
  }
};

namespace {

calibatt_status check_dict_layer(const calibatt_dict* d, int32_t t, int32_t l) {
  if (!d) return fail(CALIBATT_ERR_INVALID_ARG, "dictionary is NULL");
  if (t < 0 || t >= d->T || l < 0 || l >= d->L)
    return fail(CALIBATT_ERR_INVALID_ARG, "record (t=%d, l=%d) outside the dictionary (%d x %d)", t, l, d->T, d->L);
  if (!d->layer_set[d->layer(t, l)]) return fail(CALIBATT_ERR_INVALID_ARG, "layer (t=%d, l=%d) was never set", t, l);
  return CALIBATT_OK;
}

// Block-sparse attention over one set of skip lists, shared by the dictionary
// and direct-CSR calls: the tensor-core kernel runs the schedule's items on
// `grid` persistent CTAs, the CUDA-core kernel walks `heads`.
calibatt_status run_sparse(const void* q, const void* k, const void* v, void* o, const calibatt_shape& s,
                           int32_t block, const LayerSchedule& sch, int32_t grid, const std::vector<int16_t>& heads,
                           float softmax_scale, float* lse, cudaStream_t stream) {
  const float sl2 = scale_log2_of(softmax_scale, s.head_dim);
  if (s.dtype == CALIBATT_DTYPE_BF16 && block == 128) {
    TcParams p;
    std::memset(&p, 0, sizeof(p));
    calibatt_status st;
    if ((st = encode_qkv_map(&p.tm_q, q, s, &p.pos_n, &p.pos_h, &p.pos_b)) != CALIBATT_OK) return st;
    if ((st = encode_qkv_map(&p.tm_k, k, s, &p.pos_n, &p.pos_h, &p.pos_b)) != CALIBATT_OK) return st;
    if ((st = encode_qkv_map(&p.tm_v, v, s, &p.pos_n, &p.pos_h, &p.pos_b)) != CALIBATT_OK) return st;
    p.q = static_cast<const uint16_t*>(q);
    p.o = static_cast<uint16_t*>(o);
    p.lse = lse;
    p.sb = s.stride_b;
    p.sn = s.stride_n;
    p.sh = s.stride_h;
    p.batch = s.batch;
    p.seq_len = s.seq_len;
    p.heads = s.heads;
    p.nb = ceil_div(s.seq_len, 128);
    p.scale_log2 = sl2;
    p.sched = sch;
    p.status = status_word_ptr();
    p.timeout_ns = g_timeout_ns.load();
    cudaError_t e = calibatt::launch_tc_attn(p, s.head_dim, calibatt::kModeSparse, grid, stream);
    if (e != cudaSuccess) return cuda_fail(e, "block-sparse tensor-core launch");
    return CALIBATT_OK;
  }
  // CUDA-core path, heads in chunks of kMaxHeadsPerCall.
  if (sch.bitmap || sch.runs)
    return fail(CALIBATT_ERR_UNSUPPORTED,
                "bitmap and interval dictionaries run on the tensor-core path only (bf16, block 128)");
  for (size_t h0 = 0; h0 < heads.size(); h0 += calibatt::kMaxHeadsPerCall) {
    SimtParams p;
    std::memset(&p, 0, sizeof(p));
    p.q = q;
    p.k = k;
    p.v = v;
    p.o = o;
    p.lse = lse;
    p.sb = s.stride_b;
    p.sn = s.stride_n;
    p.sh = s.stride_h;
    p.batch = s.batch;
    p.seq_len = s.seq_len;
    p.heads = s.heads;
    p.nb = ceil_div(s.seq_len, block);
    p.scale_log2 = sl2;
    p.status = status_word_ptr();
    p.sched = sch;
    const size_t nh = std::min<size_t>(calibatt::kMaxHeadsPerCall, heads.size() - h0);
    p.n_heads = static_cast<int32_t>(nh);
    for (size_t i = 0; i < nh; ++i) p.head_ids[i] = heads[h0 + i];
    const int64_t n_items = static_cast<int64_t>(s.batch) * nh * sch.nq;
    cudaError_t e = calibatt::launch_simt_attn(p, s.head_dim, block, s.dtype, false, static_cast<int>(n_items), stream);
    if (e != cudaSuccess) return cuda_fail(e, "block-sparse CUDA-core launch");
  }
  return CALIBATT_OK;
}

calibatt_status launch_sparse(const void* q, const void* k, const void* v, void* o, const calibatt_shape& s,
                              int32_t block, const calibatt_dict* d, int32_t t, int32_t l, float softmax_scale,
                              float* lse, cudaStream_t stream) {
  const int64_t ly = d->layer(t, l);
  if (d->n_sparse[ly] == 0) return CALIBATT_OK;
  std::vector<int16_t> heads;
  for (int h = 0; h < d->H; ++h)
    if (!d->rep[ly * d->H + h]) heads.push_back(static_cast<int16_t>(h));
  LayerSchedule sch = d->schedule(t, l);
  if (s.dtype == CALIBATT_DTYPE_BF16 && block == 128 && !d->take_ticket(sch, t, l, false, stream)) {
    cudaGetLastError();
    return fail(CALIBATT_ERR_CUDA, "work-ticket reset failed");
  }
  return run_sparse(q, k, v, o, s, block, sch, d->G, heads, softmax_scale, lse, stream);
}

// Split plan of the anchor-only launch: `tiles` equal anchor tiles on `grid`
// persistent CTAs leave a last partial wave of r = tiles mod grid tiles (all
// of them when tiles < grid).  Cut into s key ranges each, that wave takes
// ceil(r s / grid) / s of a tile's time instead of a whole tile's.  s runs
// over 1..4, each part keeping at least two key blocks; the smallest s with
// the shortest wave wins.  The split tiles are the last r of the sequence.
void anchor_split_plan(int64_t tiles, int64_t grid, int32_t nb, int64_t& first, int32_t& parts) {
  parts = 1;
  first = tiles;
  if (grid <= 0 || tiles <= 0) return;
  const int64_t r = tiles % grid;
  if (r == 0) return;
  int64_t best_num = 1, best_den = 1;  // the wave as it is: one tile's time
  for (int32_t sp = 2; sp <= 4 && nb >= 2 * sp; ++sp) {
    const int64_t num = (r * sp + grid - 1) / grid;
    if (num * best_den < best_num * sp) {
      best_num = num;
      best_den = sp;
      parts = sp;
    }
  }
  if (parts > 1) first = tiles - r;
}

// Byte layout of the anchor split workspace: partial outputs, (m, l) pairs and
// counters, each region 256-byte aligned.
struct SplitLayout {
  size_t o_bytes, ml_bytes, cnt_bytes, total;
};
SplitLayout split_layout(int64_t slots, int32_t parts, int32_t head_dim) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  SplitLayout L;
  L.o_bytes = up(static_cast<size_t>(slots) * parts * 8 * (head_dim / 2) * 32 * sizeof(float));
  L.ml_bytes = up(static_cast<size_t>(slots) * parts * 8 * 32 * 2 * sizeof(float));
  L.cnt_bytes = up(static_cast<size_t>(slots) * 8 * sizeof(uint32_t));
  L.total = slots > 0 && parts > 1 ? L.o_bytes + L.ml_bytes + L.cnt_bytes : 0;
  return L;
}

// Tiles of one anchor-only call (batch x heads x tiles per head).
int64_t anchor_call_tiles(const calibatt_shape& s, int32_t frames, int32_t cols, int32_t n_anchors, int32_t n_heads) {
  const int64_t per_head = (static_cast<int64_t>(frames) * n_anchors * cols + 127) / 128;
  return static_cast<int64_t>(s.batch) * n_heads * per_head;
}

calibatt_status launch_anchor(const void* q, const void* k, const void* v, void* o, const calibatt_shape& s,
                              int32_t block, int32_t frames, int32_t rows, int32_t cols, const int32_t* anchors,
                              int32_t n_anchors, const int32_t* head_ids, int32_t n_heads, float softmax_scale,
                              void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (frames < 1 || rows < 1 || cols < 1)
    return fail(CALIBATT_ERR_INVALID_ARG, "frames, rows and cols must be >= 1");
  if (static_cast<int64_t>(frames) * rows * cols != s.seq_len)
    return fail(CALIBATT_ERR_INVALID_ARG, "frames*rows*cols = %lld != seq_len %d",
                (long long)frames * rows * cols, s.seq_len);
  if (!anchors || n_anchors < 1 || n_anchors > calibatt::kMaxAnchors)
    return fail(CALIBATT_ERR_INVALID_ARG, "n_anchors must be in [1, %d] with a non-NULL list", calibatt::kMaxAnchors);
  for (int a = 0; a < n_anchors; ++a) {
    if (anchors[a] < 0 || anchors[a] >= rows)
      return fail(CALIBATT_ERR_INVALID_ARG, "anchor row %d outside [0, %d)", anchors[a], rows);
    if (a > 0 && anchors[a] <= anchors[a - 1])
      return fail(CALIBATT_ERR_INVALID_ARG, "anchor rows must be strictly ascending");
  }
  if (n_heads == 0) return CALIBATT_OK;
  if (!head_ids || n_heads < 0 || n_heads > calibatt::kMaxHeadsPerCall)
    return fail(CALIBATT_ERR_INVALID_ARG, "n_heads must be in [0, %d] with a non-NULL list", calibatt::kMaxHeadsPerCall);
  std::vector<uint8_t> seen(s.heads, 0);
  for (int i = 0; i < n_heads; ++i) {
    if (head_ids[i] < 0 || head_ids[i] >= s.heads)
      return fail(CALIBATT_ERR_INVALID_ARG, "head id %d outside [0, %d)", head_ids[i], s.heads);
    if (seen[head_ids[i]]++) return fail(CALIBATT_ERR_INVALID_ARG, "head id %d listed twice", head_ids[i]);
  }
  AnchorGeom g;
  std::memset(&g, 0, sizeof(g));
  g.frames = frames;
  g.rows = rows;
  g.cols = cols;
  g.n_anchors = n_anchors;
  g.anchor_tokens = frames * n_anchors * cols;
  g.n_heads = n_heads;
  anchor_groups(rows, anchors, n_anchors, g);
  for (int i = 0; i < n_heads; ++i) g.head_ids[i] = static_cast<int16_t>(head_ids[i]);
  const float sl2 = scale_log2_of(softmax_scale, s.head_dim);
  if (s.dtype == CALIBATT_DTYPE_BF16) {
    TcParams p;
    std::memset(&p, 0, sizeof(p));
    calibatt_status st;
    if ((st = encode_qkv_map(&p.tm_q, q, s, &p.pos_n, &p.pos_h, &p.pos_b)) != CALIBATT_OK) return st;
    if ((st = encode_qkv_map(&p.tm_k, k, s, &p.pos_n, &p.pos_h, &p.pos_b)) != CALIBATT_OK) return st;
    if ((st = encode_qkv_map(&p.tm_v, v, s, &p.pos_n, &p.pos_h, &p.pos_b)) != CALIBATT_OK) return st;
    p.q = static_cast<const uint16_t*>(q);
    p.o = static_cast<uint16_t*>(o);
    p.sb = s.stride_b;
    p.sn = s.stride_n;
    p.sh = s.stride_h;
    p.batch = s.batch;
    p.seq_len = s.seq_len;
    p.heads = s.heads;
    p.nb = ceil_div(s.seq_len, 128);
    p.scale_log2 = sl2;
    g.tiles_per_head = ceil_div(g.anchor_tokens, 128);
    p.anc = g;
    p.status = status_word_ptr();
    p.timeout_ns = g_timeout_ns.load();
    const int sms = device_sm_count();
    if (sms < 1) return fail(CALIBATT_ERR_CUDA, "cannot query the SM count");
    const int64_t tiles = anchor_call_tiles(s, frames, cols, n_anchors, n_heads);
    if (tiles > (int64_t{1} << 28)) return fail(CALIBATT_ERR_UNSUPPORTED, "more than 2^28 anchor tiles in one call");
    int64_t first = tiles;
    int32_t parts = 1;
    if (workspace != nullptr) anchor_split_plan(tiles, sms, p.nb, first, parts);
    const SplitLayout sl = split_layout(tiles - first, parts, s.head_dim);
    p.split.first = static_cast<int32_t>(first);
    p.split.parts = parts;
    p.split.n_tiles = static_cast<int32_t>(tiles);
    if (parts > 1) {
      if (reinterpret_cast<uintptr_t>(workspace) % 256)
        return fail(CALIBATT_ERR_INVALID_ARG, "the anchor workspace must be 256-byte aligned");
      if (workspace_bytes < sl.total)
        return fail(CALIBATT_ERR_INVALID_ARG, "anchor workspace of %zu bytes, this call needs %zu", workspace_bytes,
                    sl.total);
      uint8_t* w = static_cast<uint8_t*>(workspace);
      p.split.o = reinterpret_cast<float*>(w);
      p.split.ml = reinterpret_cast<float2*>(w + sl.o_bytes);
      p.split.cnt = reinterpret_cast<uint32_t*>(w + sl.o_bytes + sl.ml_bytes);
      if (cudaMemsetAsync(p.split.cnt, 0, sl.cnt_bytes, stream) != cudaSuccess) {
        cudaGetLastError();
        return fail(CALIBATT_ERR_CUDA, "anchor split counter reset failed");
      }
    }
    const int64_t items = first + (tiles - first) * parts;
    const int grid = static_cast<int>(std::min<int64_t>(sms, items));
    cudaError_t e = calibatt::launch_tc_attn(p, s.head_dim, calibatt::kModeAnchor, grid, stream);
    if (e != cudaSuccess) return cuda_fail(e, "anchor tensor-core launch");
    return CALIBATT_OK;
  }
  SimtParams p;
  std::memset(&p, 0, sizeof(p));
  p.q = q;
  p.k = k;
  p.v = v;
  p.o = o;
  p.sb = s.stride_b;
  p.sn = s.stride_n;
  p.sh = s.stride_h;
  p.batch = s.batch;
  p.seq_len = s.seq_len;
  p.heads = s.heads;
  p.nb = ceil_div(s.seq_len, block);
  p.scale_log2 = sl2;
  p.status = status_word_ptr();
  g.tiles_per_head = ceil_div(g.anchor_tokens, block);
  p.anc = g;
  const int64_t n_items = static_cast<int64_t>(s.batch) * n_heads * g.tiles_per_head;
  cudaError_t e = calibatt::launch_simt_attn(p, s.head_dim, block, s.dtype, true, static_cast<int>(n_items), stream);
  if (e != cudaSuccess) return cuda_fail(e, "anchor CUDA-core launch");
  return CALIBATT_OK;
}

// One persistent launch over the joint sparse + anchor schedule of a layer
// (the dictionary's anchor geometry matches the call's).
calibatt_status launch_fused(const void* q, const void* k, const void* v, void* o, const calibatt_shape& s,
                             const calibatt_dict* d, int32_t t, int32_t l, float softmax_scale, float* lse,
                             cudaStream_t stream) {
  AnchorGeom g;
  std::memset(&g, 0, sizeof(g));
  g.frames = d->g_frames;
  g.rows = d->g_rows;
  g.cols = d->g_cols;
  g.n_anchors = static_cast<int32_t>(d->g_anchors.size());
  g.anchor_tokens = g.frames * g.n_anchors * g.cols;
  g.tiles_per_head = d->g_tiles;
  anchor_groups(g.rows, d->g_anchors.data(), g.n_anchors, g);
  TcParams p;
  std::memset(&p, 0, sizeof(p));
  calibatt_status st;
  if ((st = encode_qkv_map(&p.tm_q, q, s, &p.pos_n, &p.pos_h, &p.pos_b)) != CALIBATT_OK) return st;
  if ((st = encode_qkv_map(&p.tm_k, k, s, &p.pos_n, &p.pos_h, &p.pos_b)) != CALIBATT_OK) return st;
  if ((st = encode_qkv_map(&p.tm_v, v, s, &p.pos_n, &p.pos_h, &p.pos_b)) != CALIBATT_OK) return st;
  p.q = static_cast<const uint16_t*>(q);
  p.o = static_cast<uint16_t*>(o);
  p.lse = lse;
  p.sb = s.stride_b;
  p.sn = s.stride_n;
  p.sh = s.stride_h;
  p.batch = s.batch;
  p.seq_len = s.seq_len;
  p.heads = s.heads;
  p.nb = ceil_div(s.seq_len, 128);
  p.scale_log2 = scale_log2_of(softmax_scale, s.head_dim);
  p.sched = d->fused_schedule(t, l);
  if (!d->take_ticket(p.sched, t, l, true, stream)) {
    cudaGetLastError();
    return fail(CALIBATT_ERR_CUDA, "work-ticket reset failed");
  }
  p.anc = g;
  p.status = status_word_ptr();
  p.timeout_ns = g_timeout_ns.load();
  cudaError_t e = calibatt::launch_tc_attn(p, s.head_dim, calibatt::kModeFused, d->G, stream);
  if (e != cudaSuccess) return cuda_fail(e, "dual-path tensor-core launch");
  return CALIBATT_OK;
}

}  // namespace

namespace {

// Runs an entry point's body so that no C++ exception crosses the C ABI: a
// failed host allocation (std::bad_alloc from a container or new) becomes
// CALIBATT_ERR_OOM, anything else CALIBATT_ERR_INVALID_ARG with its message.
template <typename Body>
calibatt_status guarded(Body&& body) {
  try {
    return body();
  } catch (const std::bad_alloc&) {
    return fail(CALIBATT_ERR_OOM, "host memory allocation failed");
  } catch (const std::exception& e) {
    return fail(CALIBATT_ERR_INVALID_ARG, "internal error: %s", e.what());
  } catch (...) {
    return fail(CALIBATT_ERR_INVALID_ARG, "internal error");
  }
}

}  // namespace

// ===================================================================== ABI

extern "C" {

const char* calibatt_status_string(calibatt_status status) {
  switch (status) {
    case CALIBATT_OK: return "ok";
    case CALIBATT_ERR_INVALID_ARG: return "invalid argument";
    case CALIBATT_ERR_UNSUPPORTED: return "unsupported configuration";
    case CALIBATT_ERR_CUDA: return "CUDA error";
    case CALIBATT_ERR_TIMEOUT: return "device wait timed out";
    case CALIBATT_ERR_OOM: return "out of device memory";
    default: return "unknown status";
  }
}

const char* calibatt_last_error(void) { return g_last_error.c_str(); }

int32_t calibatt_abi_version(void) { return 1; }

calibatt_status calibatt_csr_validate(int32_t nq, int32_t nk, const int32_t* row_ptr, const int32_t* col_idx,
                                      int32_t require_diagonal) {
  return guarded([&]() -> calibatt_status {
    return validate_csr(nq, nk, row_ptr, col_idx, require_diagonal != 0, "csr");
  });
}

calibatt_status calibatt_csr_to_intervals(int32_t nq, const int32_t* row_ptr, const int32_t* col_idx,
                                          int32_t* interval_ptr, int32_t* interval_start, int32_t* interval_len,
                                          int64_t capacity, int64_t* n_intervals) {
  return guarded([&]() -> calibatt_status {
    if (nq < 0 || !row_ptr || !interval_ptr || !n_intervals) return fail(CALIBATT_ERR_INVALID_ARG, "NULL argument");
    if (row_ptr[nq] > 0 && !col_idx) return fail(CALIBATT_ERR_INVALID_ARG, "col_idx is NULL");
    int64_t total = 0;
    for (int32_t r = 0; r < nq; ++r) {
      interval_ptr[r] = static_cast<int32_t>(std::min<int64_t>(total, INT32_MAX));
      for (int32_t i = row_ptr[r]; i < row_ptr[r + 1]; ++i) {
        const bool starts = (i == row_ptr[r]) || (col_idx[i] != col_idx[i - 1] + 1);
        if (starts) {
          if (total < capacity && interval_start && interval_len) {
            interval_start[total] = col_idx[i];
            interval_len[total] = 1;
          }
          ++total;
        } else if (total - 1 < capacity && interval_len) {
          interval_len[total - 1] += 1;
        }
      }
    }
    interval_ptr[nq] = static_cast<int32_t>(std::min<int64_t>(total, INT32_MAX));
    *n_intervals = total;
    if (total > capacity) return fail(CALIBATT_ERR_INVALID_ARG, "capacity %lld < %lld intervals", (long long)capacity, (long long)total);
    return CALIBATT_OK;
  });
}

calibatt_status calibatt_lpt_schedule(int32_t n_items, const int64_t* cost, int32_t n_bins, int32_t* bin_ptr,
                                      int32_t* item_order, int64_t* makespan) {
  return guarded([&]() -> calibatt_status {
    if (n_items < 0 || n_bins < 1) return fail(CALIBATT_ERR_INVALID_ARG, "n_items must be >= 0 and n_bins >= 1");
    if (!bin_ptr || (n_items > 0 && (!cost || !item_order))) return fail(CALIBATT_ERR_INVALID_ARG, "NULL argument");
    for (int32_t i = 0; i < n_items; ++i)
      if (cost[i] < 0) return fail(CALIBATT_ERR_INVALID_ARG, "negative cost at item %d", i);
    lpt(n_items, cost, n_bins, bin_ptr, item_order, makespan);
    return CALIBATT_OK;
  });
}

calibatt_status calibatt_csr_schedule(int32_t heads, int32_t nq, const int32_t* row_ptr, const int32_t* head_ids,
                                      int32_t n_heads, int32_t grid, uint32_t* items, int32_t* cta_ptr) {
  return guarded([&]() -> calibatt_status {
    if (heads < 1 || heads > 65535 || nq < 1 || nq > 65535)
      return fail(CALIBATT_ERR_INVALID_ARG, "heads and nq must be in [1, 65535]");
    if (grid < 1) return fail(CALIBATT_ERR_INVALID_ARG, "grid must be >= 1");
    if (n_heads < 0 || n_heads > calibatt::kMaxHeadsPerCall)
      return fail(CALIBATT_ERR_INVALID_ARG, "n_heads must be in [0, %d]", calibatt::kMaxHeadsPerCall);
    if (!row_ptr || !cta_ptr || (n_heads > 0 && (!head_ids || !items)))
      return fail(CALIBATT_ERR_INVALID_ARG, "NULL argument");
    std::vector<uint8_t> seen(heads, 0);
    for (int i = 0; i < n_heads; ++i) {
      const int32_t h = head_ids[i];
      if (h < 0 || h >= heads) return fail(CALIBATT_ERR_INVALID_ARG, "head id %d outside [0, %d)", h, heads);
      if (seen[h]++) return fail(CALIBATT_ERR_INVALID_ARG, "head id %d listed twice", h);
      const int32_t* rp = row_ptr + static_cast<int64_t>(h) * (nq + 1);
      if (rp[0] != 0) return fail(CALIBATT_ERR_INVALID_ARG, "head %d: row_ptr[0] != 0", h);
      for (int r = 0; r < nq; ++r)
        if (rp[r + 1] < rp[r] || rp[r + 1] - rp[r] > nq)
          return fail(CALIBATT_ERR_INVALID_ARG, "head %d: row %d has %d blocks", h, r, rp[r + 1] - rp[r]);
    }
    // The dictionary's cost model and L2 head groups (calibatt_dict_set_layer).
    std::vector<uint32_t> all;
    std::vector<int64_t> cost;
    std::vector<int32_t> group;
    const int32_t hpg = heads_per_group(nq);
    for (int i = 0; i < n_heads; ++i) {
      const int32_t* rp = row_ptr + static_cast<int64_t>(head_ids[i]) * (nq + 1);
      for (int r = 0; r < nq; ++r) {
        all.push_back((static_cast<uint32_t>(head_ids[i]) << 16) | static_cast<uint32_t>(r));
        cost.push_back(static_cast<int64_t>(rp[r + 1] - rp[r]) + 2);
        group.push_back(schedule_group(i, r, nq, hpg, grid));
      }
    }
    std::vector<int32_t> order(all.size());
    lpt_grouped(static_cast<int32_t>(all.size()), cost.data(), group.data(), grid, cta_ptr, order.data());
    for (size_t i = 0; i < all.size(); ++i) items[i] = all[order[i]];
    return CALIBATT_OK;
  });
}

calibatt_status calibatt_dict_create(int32_t T, int32_t L, int32_t H, int32_t nq, int32_t nk, int32_t block,
                                     int64_t nnz_capacity, int32_t num_ctas, calibatt_dict** out) {
  return guarded([&]() -> calibatt_status {
    if (!out) return fail(CALIBATT_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    if (T < 1 || L < 1 || H < 1 || nq < 1 || nk < 1 || nnz_capacity < 0)
      return fail(CALIBATT_ERR_INVALID_ARG, "T, L, H, nq, nk must be >= 1 and nnz_capacity >= 0");
    if (nq != nk) return fail(CALIBATT_ERR_INVALID_ARG, "self-attention dictionary needs nq == nk");
    if (nq > 65535 || H > 65535) return fail(CALIBATT_ERR_UNSUPPORTED, "nq and H must be <= 65535");
    calibatt_status st = check_block(block);
    if (st != CALIBATT_OK) return st;
    int G = num_ctas;
    if (G <= 0) G = device_sm_count();
    if (G <= 0) return fail(CALIBATT_ERR_CUDA, "cannot query the SM count");
    // owned here until returned, so an exception frees it (host vectors are
    // sized before any device allocation)
    std::unique_ptr<calibatt_dict> holder(new calibatt_dict());
    calibatt_dict* d = holder.get();
    d->T = T;
    d->L = L;
    d->H = H;
    d->nq = nq;
    d->nk = nk;
    d->block = block;
    d->G = G;
    cudaGetDevice(&d->device);
    d->nnz_cap = nnz_capacity;
    const int64_t layers = static_cast<int64_t>(T) * L;
    d->layer_set.assign(layers, 0);
    d->rep.assign(layers * H, 0);
    d->n_sparse.assign(layers, 0);
    d->n_rep.assign(layers, 0);
    d->retained.assign(layers, 0);
    const size_t b_rp = sizeof(int32_t) * layers * H * (nq + 1);
    const size_t b_cb = sizeof(int64_t) * layers * H;
    const size_t b_col = sizeof(uint16_t) * std::max<int64_t>(1, nnz_capacity);
    const size_t b_it = sizeof(uint32_t) * layers * H * nq;
    const size_t b_cta = sizeof(int32_t) * layers * (G + 1);
    cudaError_t e = cudaMalloc(&d->d_row_ptr, b_rp);
    if (e == cudaSuccess) e = cudaMalloc(&d->d_col_base, b_cb);
    if (e == cudaSuccess) e = cudaMalloc(&d->d_col, b_col);
    if (e == cudaSuccess) e = cudaMalloc(&d->d_items, b_it);
    if (e == cudaSuccess) e = cudaMalloc(&d->d_cta_ptr, b_cta);
    if (e == cudaSuccess) e = cudaMalloc(&d->d_order, b_it);
    if (e == cudaSuccess) e = cudaMalloc(&d->d_tickets, sizeof(uint32_t) * kTicketSlots);
    if (e != cudaSuccess) {
      d->release();
      return cuda_fail(e, "dictionary allocation");
    }
    d->n_order.assign(layers, 0);
    d->n_forder.assign(layers, 0);
    d->device_bytes = static_cast<int64_t>(b_rp + b_cb + b_col + 2 * b_it + b_cta + sizeof(uint32_t) * kTicketSlots);
    *out = holder.release();
    return CALIBATT_OK;
  });
}

calibatt_status calibatt_dict_create_bitmap(int32_t T, int32_t L, int32_t H, int32_t nq, int32_t nk,
                                            int32_t block, int32_t num_ctas, calibatt_dict** out) {
  return guarded([&]() -> calibatt_status {
    if (!out) return fail(CALIBATT_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    if (T < 1 || L < 1 || H < 1 || nq < 1 || nk < 1)
      return fail(CALIBATT_ERR_INVALID_ARG, "T, L, H, nq, nk must be >= 1");
    if (nq != nk) return fail(CALIBATT_ERR_INVALID_ARG, "self-attention dictionary needs nq == nk");
    if (nq > calibatt::kMaxBitmapBlocks)
      return fail(CALIBATT_ERR_UNSUPPORTED, "bitmap dictionaries hold at most %d blocks per row", calibatt::kMaxBitmapBlocks);
    if (H > 65535) return fail(CALIBATT_ERR_UNSUPPORTED, "H must be <= 65535");
    calibatt_status st = check_block(block);
    if (st != CALIBATT_OK) return st;
    int G = num_ctas;
    if (G <= 0) G = device_sm_count();
    if (G <= 0) return fail(CALIBATT_ERR_CUDA, "cannot query the SM count");
    std::unique_ptr<calibatt_dict> holder(new calibatt_dict());
    calibatt_dict* d = holder.get();
    d->T = T;
    d->L = L;
    d->H = H;
    d->nq = nq;
    d->nk = nk;
    d->block = block;
    d->G = G;
    d->bitmap = true;
    d->words = (nk + 31) / 32;
    cudaGetDevice(&d->device);
    const int64_t layers = static_cast<int64_t>(T) * L;
    d->layer_set.assign(layers, 0);
    d->rep.assign(layers * H, 0);
    d->n_sparse.assign(layers, 0);
    d->n_rep.assign(layers, 0);
    d->retained.assign(layers, 0);
    const size_t b_bm = sizeof(uint32_t) * layers * H * nq * d->words;
    const size_t b_it = sizeof(uint32_t) * layers * H * nq;
    const size_t b_cta = sizeof(int32_t) * layers * (G + 1);
    cudaError_t e = cudaMalloc(&d->d_bitmap, b_bm);
    if (e == cudaSuccess) e = cudaMalloc(&d->d_items, b_it);
    if (e == cudaSuccess) e = cudaMalloc(&d->d_cta_ptr, b_cta);
    if (e == cudaSuccess) e = cudaMalloc(&d->d_order, b_it);
    if (e == cudaSuccess) e = cudaMalloc(&d->d_tickets, sizeof(uint32_t) * kTicketSlots);
    if (e != cudaSuccess) {
      d->release();
      return cuda_fail(e, "bitmap dictionary allocation");
    }
    d->n_order.assign(layers, 0);
    d->n_forder.assign(layers, 0);
    d->device_bytes = static_cast<int64_t>(b_bm + 2 * b_it + b_cta + sizeof(uint32_t) * kTicketSlots);
    *out = holder.release();
    return CALIBATT_OK;
  });
}

calibatt_status calibatt_dict_create_intervals(int32_t T, int32_t L, int32_t H, int32_t nq, int32_t nk,
                                               int32_t block, int64_t run_capacity, int32_t num_ctas,
                                               calibatt_dict** out) {
  return guarded([&]() -> calibatt_status {
    if (!out) return fail(CALIBATT_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    if (T < 1 || L < 1 || H < 1 || nq < 1 || nk < 1 || run_capacity < 0)
      return fail(CALIBATT_ERR_INVALID_ARG, "T, L, H, nq, nk must be >= 1 and run_capacity >= 0");
    if (nq != nk) return fail(CALIBATT_ERR_INVALID_ARG, "self-attention dictionary needs nq == nk");
    if (nq > calibatt::kMaxBitmapBlocks)
      return fail(CALIBATT_ERR_UNSUPPORTED, "interval dictionaries hold at most %d blocks per row",
                  calibatt::kMaxBitmapBlocks);
    if (H > 65535) return fail(CALIBATT_ERR_UNSUPPORTED, "H must be <= 65535");
    calibatt_status st = check_block(block);
    if (st != CALIBATT_OK) return st;
    int G = num_ctas;
    if (G <= 0) G = device_sm_count();
    if (G <= 0) return fail(CALIBATT_ERR_CUDA, "cannot query the SM count");
    std::unique_ptr<calibatt_dict> holder(new calibatt_dict());
    calibatt_dict* d = holder.get();
    d->T = T;
    d->L = L;
    d->H = H;
    d->nq = nq;
    d->nk = nk;
    d->block = block;
    d->G = G;
    d->intervals = true;
    cudaGetDevice(&d->device);
    d->nnz_cap = run_capacity;
    const int64_t layers = static_cast<int64_t>(T) * L;
    d->layer_set.assign(layers, 0);
    d->rep.assign(layers * H, 0);
    d->n_sparse.assign(layers, 0);
    d->n_rep.assign(layers, 0);
    d->retained.assign(layers, 0);
    const size_t b_rp = sizeof(int32_t) * layers * H * (nq + 1);
    const size_t b_cb = sizeof(int64_t) * layers * H;
    const size_t b_runs = sizeof(uint32_t) * std::max<int64_t>(1, run_capacity);
    const size_t b_it = sizeof(uint32_t) * layers * H * nq;
    const size_t b_cta = sizeof(int32_t) * layers * (G + 1);
    cudaError_t e = cudaMalloc(&d->d_row_ptr, b_rp);
    if (e == cudaSuccess) e = cudaMalloc(&d->d_run_ptr, b_rp);
    if (e == cudaSuccess) e = cudaMalloc(&d->d_col_base, b_cb);
    if (e == cudaSuccess) e = cudaMalloc(&d->d_runs, b_runs);
    if (e == cudaSuccess) e = cudaMalloc(&d->d_items, b_it);
    if (e == cudaSuccess) e = cudaMalloc(&d->d_cta_ptr, b_cta);
    if (e == cudaSuccess) e = cudaMalloc(&d->d_order, b_it);
    if (e == cudaSuccess) e = cudaMalloc(&d->d_tickets, sizeof(uint32_t) * kTicketSlots);
    if (e != cudaSuccess) {
      d->release();
      return cuda_fail(e, "interval dictionary allocation");
    }
    d->n_order.assign(layers, 0);
    d->n_forder.assign(layers, 0);
    d->device_bytes = static_cast<int64_t>(2 * b_rp + b_cb + b_runs + 2 * b_it + b_cta + sizeof(uint32_t) * kTicketSlots);
    *out = holder.release();
    return CALIBATT_OK;
  });
}

calibatt_status calibatt_dict_set_layer(calibatt_dict* d, int32_t t, int32_t l, const int32_t* row_ptr,
                                        const int32_t* col_idx, const uint8_t* repetitive) {
  return guarded([&]() -> calibatt_status {
    if (!d) return fail(CALIBATT_ERR_INVALID_ARG, "dictionary is NULL");
    if (t < 0 || t >= d->T || l < 0 || l >= d->L)
      return fail(CALIBATT_ERR_INVALID_ARG, "record (t=%d, l=%d) outside the dictionary", t, l);
    const int64_t ly = d->layer(t, l);
    if (d->layer_set[ly]) return fail(CALIBATT_ERR_INVALID_ARG, "layer (t=%d, l=%d) is already set", t, l);
    if (!row_ptr) return fail(CALIBATT_ERR_INVALID_ARG, "row_ptr is NULL");
    const int H = d->H, nq = d->nq;
    std::vector<int64_t> head_off(H + 1, 0);
    char what[64];
    for (int h = 0; h < H; ++h) {
      const int32_t* rp = row_ptr + static_cast<int64_t>(h) * (nq + 1);
      snprintf(what, sizeof(what), "layer (%d, %d) head %d", t, l, h);
      calibatt_status st = validate_csr(nq, d->nk, rp, col_idx ? col_idx + head_off[h] : nullptr, false, what);
      if (st != CALIBATT_OK) return st;
      if (repetitive && repetitive[h] && rp[nq] != 0)
        return fail(CALIBATT_ERR_INVALID_ARG, "%s is repetitive but has a non-empty skip list", what);
      head_off[h + 1] = head_off[h] + rp[nq];
    }
    const int64_t nnz = head_off[H];
    // Interval format: each row's contiguous runs, and per head its run
    // pointers (counted from the head's first run) and its first run's offset.
    std::vector<uint32_t> runs;
    std::vector<int32_t> run_ptr;
    std::vector<int64_t> run_head_off(H + 1, 0);
    if (d->intervals) {
      run_ptr.assign(static_cast<size_t>(H) * (nq + 1), 0);
      for (int h = 0; h < H; ++h) {
        const int32_t* rp = row_ptr + static_cast<int64_t>(h) * (nq + 1);
        const int32_t* ci = col_idx ? col_idx + head_off[h] : nullptr;
        int32_t* hp = run_ptr.data() + static_cast<size_t>(h) * (nq + 1);
        const size_t head_start = runs.size();
        for (int r = 0; r < nq; ++r) {
          hp[r] |= static_cast<int32_t>(runs.size() - head_start);  // keeps row r - 1's end flag
          for (int32_t x = rp[r]; x < rp[r + 1]; ++x) {
            if (x > rp[r] && ci[x] == ci[x - 1] + 1)
              runs.back() += 1u << 16;                         // extends the current run
            else
              runs.push_back(static_cast<uint32_t>(ci[x]) | (1u << 16));
          }
          // bit 31 of the row's end entry: the row keeps the last key block
          if (rp[r + 1] > rp[r] && ci[rp[r + 1] - 1] == nq - 1) hp[r + 1] = INT32_MIN;
        }
        hp[nq] |= static_cast<int32_t>(runs.size() - head_start);
        run_head_off[h + 1] = static_cast<int64_t>(runs.size());
      }
    }
    const int64_t units = d->intervals ? static_cast<int64_t>(runs.size()) : nnz;
    if (!d->bitmap && d->nnz_used + units > d->nnz_cap)
      return fail(CALIBATT_ERR_INVALID_ARG, "dictionary capacity exceeded (%lld + %lld > %lld %s)",
                  (long long)d->nnz_used, (long long)units, (long long)d->nnz_cap,
                  d->intervals ? "intervals" : "blocks");
    std::vector<uint16_t> col16(d->bitmap || d->intervals ? 0 : nnz);
    for (size_t i = 0; i < col16.size(); ++i) col16[i] = static_cast<uint16_t>(col_idx[i]);
    std::vector<uint32_t> bits;
    if (d->bitmap) {
      bits.assign(static_cast<size_t>(H) * nq * d->words, 0u);
      for (int h = 0; h < H; ++h) {
        const int32_t* rp = row_ptr + static_cast<int64_t>(h) * (nq + 1);
        for (int r = 0; r < nq; ++r)
          for (int32_t x = rp[r]; x < rp[r + 1]; ++x) {
            const int32_t c = col_idx[head_off[h] + x];
            bits[(static_cast<size_t>(h) * nq + r) * d->words + (c >> 5)] |= 1u << (c & 31);
          }
      }
    }
    std::vector<int64_t> col_base(H);
    for (int h = 0; h < H; ++h) col_base[h] = d->nnz_used + (d->intervals ? run_head_off[h] : head_off[h]);
    // Work items of the sparse heads and their LPT schedule over the grid.
    std::vector<uint32_t> items;
    std::vector<int64_t> cost;
    std::vector<int32_t> group;
    int32_t n_sparse = 0, n_rep = 0;
    int64_t retained = 0;
    const int32_t hpg = heads_per_group(nq);
    for (int h = 0; h < H; ++h) {
      if (repetitive && repetitive[h]) {
        ++n_rep;
        continue;
      }
      const int32_t k = n_sparse++;
      const int32_t* rp = row_ptr + static_cast<int64_t>(h) * (nq + 1);
      for (int r = 0; r < nq; ++r) {
        items.push_back((static_cast<uint32_t>(h) << 16) | static_cast<uint32_t>(r));
        cost.push_back(static_cast<int64_t>(rp[r + 1] - rp[r]) + 2);  // +2: Q load and epilogue
        group.push_back(schedule_group(k, r, nq, hpg, d->G));
        retained += rp[r + 1] - rp[r];
      }
    }
    std::vector<int32_t> cta_ptr(d->G + 1), order(items.size());
    lpt_grouped(static_cast<int32_t>(items.size()), cost.data(), group.data(), d->G, cta_ptr.data(), order.data());
    std::vector<uint32_t> sched(items.size());
    for (size_t i = 0; i < items.size(); ++i) sched[i] = items[order[i]];
    // the same items in consumption order, for dynamic assignment
    std::vector<uint32_t> dyn(items.size());
    {
      const std::vector<int32_t> co = consumption_order(cost, group);
      for (size_t i = 0; i < items.size(); ++i) dyn[i] = items[co[i]];
    }
    // Joint schedule of the dual path.  All anchor tiles of the repetitive
    // heads come first, as one group in head order (a tile visits all nq key
    // blocks; its epilogue writes about rows / n_anchors output rows per query,
    // counted as that many extra blocks): the equal-cost tiles go round-robin
    // over the CTAs, so the grid works on two or three heads at a time.  The
    // sparse items follow in the L2 groups of the sparse-only schedule, with the
    // running balance starting from the anchor loads.  (Interleaving both kinds
    // in head-order groups let CTAs drift several groups apart behind the large
    // anchor tiles, and the keys and values of the heads in flight no longer
    // fitted in L2.)
    std::vector<uint32_t> fsched, fdyn;
    std::vector<int32_t> fcta_ptr;
    if (d->has_geom) {
      std::vector<uint32_t> fitems;
      std::vector<int64_t> fcost;
      std::vector<int32_t> fgroup;
      const int64_t bcast = std::max<int64_t>(1, d->g_rows / static_cast<int64_t>(d->g_anchors.size()));
      int32_t sparse_rank = 0;
      for (int h = 0; h < H; ++h) {
        if (repetitive && repetitive[h]) {
          for (int tile = 0; tile < d->g_tiles; ++tile) {
            fitems.push_back(calibatt::kItemAnchorBit | (static_cast<uint32_t>(h) << 16) | static_cast<uint32_t>(tile));
            fcost.push_back(static_cast<int64_t>(nq) + 2 + bcast);
            fgroup.push_back(0);
          }
        } else {
          const int32_t k = sparse_rank++;
          const int32_t* rp = row_ptr + static_cast<int64_t>(h) * (nq + 1);
          for (int r = 0; r < nq; ++r) {
            fitems.push_back((static_cast<uint32_t>(h) << 16) | static_cast<uint32_t>(r));
            fcost.push_back(static_cast<int64_t>(rp[r + 1] - rp[r]) + 2);
            fgroup.push_back(1 + schedule_group(k, r, nq, hpg, d->G));
          }
        }
      }
      fcta_ptr.assign(d->G + 1, 0);
      std::vector<int32_t> forder(fitems.size());
      lpt_grouped(static_cast<int32_t>(fitems.size()), fcost.data(), fgroup.data(), d->G, fcta_ptr.data(),
                  forder.data());
      fsched.resize(fitems.size());
      for (size_t i = 0; i < fitems.size(); ++i) fsched[i] = fitems[forder[i]];
      const std::vector<int32_t> co = consumption_order(fcost, fgroup);
      fdyn.resize(fitems.size());
      for (size_t i = 0; i < fitems.size(); ++i) fdyn[i] = fitems[co[i]];
    }
    int prev = 0;
    cudaGetDevice(&prev);
    if (prev != d->device) cudaSetDevice(d->device);
    cudaError_t e = cudaSuccess;
    if (d->bitmap) {
      e = cudaMemcpy(d->d_bitmap + ly * H * nq * static_cast<int64_t>(d->words), bits.data(),
                     sizeof(uint32_t) * bits.size(), cudaMemcpyHostToDevice);
    } else if (d->intervals) {
      if (!runs.empty())
        e = cudaMemcpy(d->d_runs + d->nnz_used, runs.data(), runs.size() * sizeof(uint32_t), cudaMemcpyHostToDevice);
      if (e == cudaSuccess)
        e = cudaMemcpy(d->d_run_ptr + ly * H * (nq + 1), run_ptr.data(), sizeof(int32_t) * H * (nq + 1),
                       cudaMemcpyHostToDevice);
      if (e == cudaSuccess)
        e = cudaMemcpy(d->d_row_ptr + ly * H * (nq + 1), row_ptr, sizeof(int32_t) * H * (nq + 1),
                       cudaMemcpyHostToDevice);
      if (e == cudaSuccess)
        e = cudaMemcpy(d->d_col_base + ly * H, col_base.data(), sizeof(int64_t) * H, cudaMemcpyHostToDevice);
    } else {
      if (nnz > 0)
        e = cudaMemcpy(d->d_col + d->nnz_used, col16.data(), nnz * sizeof(uint16_t), cudaMemcpyHostToDevice);
      if (e == cudaSuccess)
        e = cudaMemcpy(d->d_row_ptr + ly * H * (nq + 1), row_ptr, sizeof(int32_t) * H * (nq + 1),
                       cudaMemcpyHostToDevice);
      if (e == cudaSuccess)
        e = cudaMemcpy(d->d_col_base + ly * H, col_base.data(), sizeof(int64_t) * H, cudaMemcpyHostToDevice);
    }
    if (e == cudaSuccess && !sched.empty())
      e = cudaMemcpy(d->d_items + ly * H * nq, sched.data(), sizeof(uint32_t) * sched.size(), cudaMemcpyHostToDevice);
    if (e == cudaSuccess && !dyn.empty())
      e = cudaMemcpy(d->d_order + ly * H * nq, dyn.data(), sizeof(uint32_t) * dyn.size(), cudaMemcpyHostToDevice);
    if (e == cudaSuccess && d->has_geom && !fdyn.empty())
      e = cudaMemcpy(d->d_forder + ly * d->f_stride, fdyn.data(), sizeof(uint32_t) * fdyn.size(),
                     cudaMemcpyHostToDevice);
    if (e == cudaSuccess)
      e = cudaMemcpy(d->d_cta_ptr + ly * (d->G + 1), cta_ptr.data(), sizeof(int32_t) * (d->G + 1), cudaMemcpyHostToDevice);
    if (e == cudaSuccess && d->has_geom && !fsched.empty())
      e = cudaMemcpy(d->d_fitems + ly * d->f_stride, fsched.data(), sizeof(uint32_t) * fsched.size(),
                     cudaMemcpyHostToDevice);
    if (e == cudaSuccess && d->has_geom)
      e = cudaMemcpy(d->d_fcta_ptr + ly * (d->G + 1), fcta_ptr.data(), sizeof(int32_t) * (d->G + 1),
                     cudaMemcpyHostToDevice);
    if (prev != d->device) cudaSetDevice(prev);
    if (e != cudaSuccess) return cuda_fail(e, "dictionary upload");
    d->nnz_used += d->bitmap ? nnz : units;
    d->blocks_used += nnz;
    for (int h = 0; h < H; ++h) d->rep[ly * H + h] = (repetitive && repetitive[h]) ? 1 : 0;
    d->n_sparse[ly] = n_sparse;
    d->n_rep[ly] = n_rep;
    d->n_order[ly] = static_cast<int32_t>(dyn.size());
    d->n_forder[ly] = static_cast<int32_t>(fdyn.size());
    d->retained[ly] = retained;
    d->layer_set[ly] = 1;
    return CALIBATT_OK;
  });
}

calibatt_status calibatt_dict_set_anchor_geometry(calibatt_dict* d, int32_t frames, int32_t rows, int32_t cols,
                                                  const int32_t* anchor_rows, int32_t n_anchors) {
  return guarded([&]() -> calibatt_status {
    if (!d) return fail(CALIBATT_ERR_INVALID_ARG, "dictionary is NULL");
    if (d->has_geom) return fail(CALIBATT_ERR_INVALID_ARG, "the anchor geometry is already set");
    for (uint8_t set : d->layer_set)
      if (set) return fail(CALIBATT_ERR_INVALID_ARG, "the anchor geometry must be set before the first layer");
    if (frames < 1 || rows < 1 || cols < 1) return fail(CALIBATT_ERR_INVALID_ARG, "frames, rows and cols must be >= 1");
    const int64_t tokens = static_cast<int64_t>(frames) * rows * cols;
    if (ceil_div(tokens, d->block) != d->nq)
      return fail(CALIBATT_ERR_INVALID_ARG, "frames*rows*cols = %lld tokens do not make the dictionary's %d blocks",
                  (long long)tokens, d->nq);
    if (!anchor_rows || n_anchors < 1 || n_anchors > calibatt::kMaxAnchors)
      return fail(CALIBATT_ERR_INVALID_ARG, "n_anchors must be in [1, %d] with a non-NULL list", calibatt::kMaxAnchors);
    for (int a = 0; a < n_anchors; ++a) {
      if (anchor_rows[a] < 0 || anchor_rows[a] >= rows)
        return fail(CALIBATT_ERR_INVALID_ARG, "anchor row %d outside [0, %d)", anchor_rows[a], rows);
      if (a > 0 && anchor_rows[a] <= anchor_rows[a - 1])
        return fail(CALIBATT_ERR_INVALID_ARG, "anchor rows must be strictly ascending");
    }
    if (d->H > 32767) return fail(CALIBATT_ERR_UNSUPPORTED, "joint schedules need H <= 32767");
    const int64_t tiles = ceil_div(static_cast<int64_t>(frames) * n_anchors * cols, 128);
    if (tiles > 65535) return fail(CALIBATT_ERR_UNSUPPORTED, "more than 65535 anchor tiles per head");
    const int64_t layers = static_cast<int64_t>(d->T) * d->L;
    const int64_t stride = static_cast<int64_t>(d->H) * std::max<int64_t>(d->nq, tiles);
    int prev = 0;
    cudaGetDevice(&prev);
    if (prev != d->device) cudaSetDevice(d->device);
    cudaError_t e = cudaMalloc(&d->d_fitems, sizeof(uint32_t) * layers * stride);
    if (e == cudaSuccess) e = cudaMalloc(&d->d_forder, sizeof(uint32_t) * layers * stride);
    if (e == cudaSuccess) e = cudaMalloc(&d->d_fcta_ptr, sizeof(int32_t) * layers * (d->G + 1));
    if (prev != d->device) cudaSetDevice(prev);
    if (e != cudaSuccess) {
      cudaFree(d->d_fitems);
      cudaFree(d->d_fcta_ptr);
      d->d_fitems = nullptr;
      d->d_fcta_ptr = nullptr;
      return cuda_fail(e, "joint schedule allocation");
    }
    d->device_bytes += static_cast<int64_t>(2 * sizeof(uint32_t) * layers * stride + sizeof(int32_t) * layers * (d->G + 1));
    d->f_stride = stride;
    d->g_frames = frames;
    d->g_rows = rows;
    d->g_cols = cols;
    d->g_tiles = static_cast<int32_t>(tiles);
    d->g_anchors.assign(anchor_rows, anchor_rows + n_anchors);
    d->has_geom = true;
    return CALIBATT_OK;
  });
}

calibatt_status calibatt_dict_info(const calibatt_dict* d, int64_t* device_bytes, int64_t* nnz_total,
                                   int32_t* num_ctas) {
  return guarded([&]() -> calibatt_status {
    if (!d) return fail(CALIBATT_ERR_INVALID_ARG, "dictionary is NULL");
    if (device_bytes) *device_bytes = d->device_bytes;
    if (nnz_total) *nnz_total = d->blocks_used;
    if (num_ctas) *num_ctas = d->G;
    return CALIBATT_OK;
  });
}

calibatt_status calibatt_dict_layer_info(const calibatt_dict* d, int32_t t, int32_t l, int32_t* n_sparse_heads,
                                         int32_t* n_repetitive_heads, int64_t* retained_tiles) {
  return guarded([&]() -> calibatt_status {
    calibatt_status st = check_dict_layer(d, t, l);
    if (st != CALIBATT_OK) return st;
    const int64_t ly = d->layer(t, l);
    if (n_sparse_heads) *n_sparse_heads = d->n_sparse[ly];
    if (n_repetitive_heads) *n_repetitive_heads = d->n_rep[ly];
    if (retained_tiles) *retained_tiles = d->retained[ly];
    return CALIBATT_OK;
  });
}

calibatt_status calibatt_dict_destroy(calibatt_dict* d) {
  return guarded([&]() -> calibatt_status {
    if (!d) return CALIBATT_OK;
    int prev = 0;
    cudaGetDevice(&prev);
    if (prev != d->device) cudaSetDevice(d->device);
    cudaDeviceSynchronize();
    d->release();
    if (prev != d->device) cudaSetDevice(prev);
    delete d;
    cudaGetLastError();
    return CALIBATT_OK;
  });
}

// ------------------------------------------------------------ dictionary file

namespace {

constexpr char kDictMagic[8] = {'C', 'A', 'L', 'I', 'B', 'D', 'C', 'T'};
constexpr char kDictEnd[8] = {'C', 'A', 'L', 'I', 'B', 'E', 'N', 'D'};
constexpr uint32_t kDictFileVersion = 1;

struct DictFileHeader {
  char magic[8];
  uint32_t version;
  uint32_t format;  // 0 index lists, 1 bitmap, 2 intervals
  int32_t T, L, H, nq, nk, block;
  int32_t has_geom, frames, rows, cols, n_anchors;
  int32_t anchors[calibatt::kMaxAnchors];
  int32_t reserved;
  int64_t records;
  int64_t nnz_total;
};
static_assert(sizeof(DictFileHeader) == 144, "dictionary file header layout");

struct DictFileRecord {
  int32_t t, l;
  int64_t nnz;
};

// 64-bit FNV-1a over the file's 8-byte little-endian words.
struct WordHash {
  uint64_t h = 0xcbf29ce484222325ull;
  void add(const unsigned char* p, size_t n) {  // n is a multiple of 8
    for (size_t i = 0; i < n; i += 8) {
      uint64_t w;
      std::memcpy(&w, p + i, 8);
      h = (h ^ w) * 0x100000001b3ull;
    }
  }
};

size_t padded8(size_t n) { return (n + 7) & ~static_cast<size_t>(7); }

struct DictWriter {
  FILE* f = nullptr;
  WordHash hash;
  bool ok = true;
  std::vector<unsigned char> buf;
  // Writes n bytes followed by zeros up to the next multiple of 8.
  void put(const void* p, size_t n) {
    if (!ok) return;
    buf.assign(padded8(n), 0);
    if (n) std::memcpy(buf.data(), p, n);
    hash.add(buf.data(), buf.size());
    ok = std::fwrite(buf.data(), 1, buf.size(), f) == buf.size();
  }
};

struct DictReader {
  FILE* f = nullptr;
  WordHash hash;
  std::vector<unsigned char> buf;
  // Reads n bytes and their zero padding; false on a short read or a non-zero pad.
  bool get(void* p, size_t n) {
    buf.resize(padded8(n));
    if (std::fread(buf.data(), 1, buf.size(), f) != buf.size()) return false;
    for (size_t i = n; i < buf.size(); ++i)
      if (buf[i] != 0) return false;
    hash.add(buf.data(), buf.size());
    if (n) std::memcpy(p, buf.data(), n);
    return true;
  }
};

}  // namespace

calibatt_status calibatt_dict_save(const calibatt_dict* d, const char* path) {
  return guarded([&]() -> calibatt_status {
    if (!d || !path) return fail(CALIBATT_ERR_INVALID_ARG, "dictionary and path must be non-NULL");
    const int H = d->H, nq = d->nq;
    const int64_t layers = static_cast<int64_t>(d->T) * d->L;
    DictFileHeader hd;
    std::memset(&hd, 0, sizeof(hd));
    std::memcpy(hd.magic, kDictMagic, 8);
    hd.version = kDictFileVersion;
    hd.format = d->bitmap ? 1u : (d->intervals ? 2u : 0u);
    hd.T = d->T;
    hd.L = d->L;
    hd.H = H;
    hd.nq = nq;
    hd.nk = d->nk;
    hd.block = d->block;
    if (d->has_geom) {
      hd.has_geom = 1;
      hd.frames = d->g_frames;
      hd.rows = d->g_rows;
      hd.cols = d->g_cols;
      hd.n_anchors = static_cast<int32_t>(d->g_anchors.size());
      for (size_t a = 0; a < d->g_anchors.size(); ++a) hd.anchors[a] = d->g_anchors[a];
    }
    for (uint8_t set : d->layer_set) hd.records += set;
    hd.nnz_total = d->nnz_used;
    const std::string tmp = std::string(path) + ".tmp";
    DictWriter w;
    w.f = std::fopen(tmp.c_str(), "wb");
    if (!w.f) return fail(CALIBATT_ERR_INVALID_ARG, "cannot open %s for writing", tmp.c_str());
    int prev = 0;
    cudaGetDevice(&prev);
    if (prev != d->device) cudaSetDevice(d->device);
    cudaError_t e = cudaSuccess;
    w.put(&hd, sizeof(hd));
    std::vector<int32_t> rp;
    std::vector<int64_t> cb;
    std::vector<uint16_t> col;
    std::vector<uint32_t> bits;
    std::vector<int32_t> run_ptr;
    for (int64_t ly = 0; ly < layers && w.ok && e == cudaSuccess; ++ly) {
      if (!d->layer_set[ly]) continue;
      DictFileRecord rec{static_cast<int32_t>(ly / d->L), static_cast<int32_t>(ly % d->L), 0};
      if (d->intervals) {
        // the record's unit count is its number of runs
        rp.resize(static_cast<size_t>(H) * (nq + 1));
        run_ptr.resize(rp.size());
        cb.resize(H);
        e = cudaMemcpy(rp.data(), d->d_row_ptr + ly * H * (nq + 1), sizeof(int32_t) * rp.size(),
                       cudaMemcpyDeviceToHost);
        if (e == cudaSuccess)
          e = cudaMemcpy(run_ptr.data(), d->d_run_ptr + ly * H * (nq + 1), sizeof(int32_t) * run_ptr.size(),
                         cudaMemcpyDeviceToHost);
        if (e == cudaSuccess)
          e = cudaMemcpy(cb.data(), d->d_col_base + ly * H, sizeof(int64_t) * H, cudaMemcpyDeviceToHost);
        for (int32_t& x : run_ptr) x &= 0x7FFFFFFF;  // the file stores plain offsets (end flags are rebuilt)
        for (int h = 0; h < H; ++h) rec.nnz += run_ptr[static_cast<size_t>(h) * (nq + 1) + nq];
        bits.resize(rec.nnz);
        if (e == cudaSuccess && rec.nnz > 0)
          e = cudaMemcpy(bits.data(), d->d_runs + cb[0], sizeof(uint32_t) * rec.nnz, cudaMemcpyDeviceToHost);
      } else if (d->bitmap) {
        bits.resize(static_cast<size_t>(H) * nq * d->words);
        e = cudaMemcpy(bits.data(), d->d_bitmap + ly * H * nq * static_cast<int64_t>(d->words),
                       sizeof(uint32_t) * bits.size(), cudaMemcpyDeviceToHost);
        for (uint32_t x : bits) rec.nnz += __builtin_popcount(x);
      } else {
        rp.resize(static_cast<size_t>(H) * (nq + 1));
        cb.resize(H);
        e = cudaMemcpy(rp.data(), d->d_row_ptr + ly * H * (nq + 1), sizeof(int32_t) * rp.size(),
                       cudaMemcpyDeviceToHost);
        if (e == cudaSuccess)
          e = cudaMemcpy(cb.data(), d->d_col_base + ly * H, sizeof(int64_t) * H, cudaMemcpyDeviceToHost);
        for (int h = 0; h < H; ++h) rec.nnz += rp[static_cast<size_t>(h) * (nq + 1) + nq];
        col.resize(rec.nnz);
        // a layer's lists are stored contiguously, head after head, from head 0's offset
        if (e == cudaSuccess && rec.nnz > 0)
          e = cudaMemcpy(col.data(), d->d_col + cb[0], sizeof(uint16_t) * rec.nnz, cudaMemcpyDeviceToHost);
      }
      if (e != cudaSuccess) break;
      w.put(&rec, sizeof(rec));
      w.put(d->rep.data() + ly * H, H);
      if (d->intervals) {
        w.put(rp.data(), sizeof(int32_t) * rp.size());
        w.put(run_ptr.data(), sizeof(int32_t) * run_ptr.size());
        w.put(bits.data(), sizeof(uint32_t) * bits.size());
      } else if (d->bitmap) {
        w.put(bits.data(), sizeof(uint32_t) * bits.size());
      } else {
        w.put(rp.data(), sizeof(int32_t) * rp.size());
        w.put(col.data(), sizeof(uint16_t) * col.size());
      }
    }
    if (prev != d->device) cudaSetDevice(prev);
    if (w.ok && e == cudaSuccess) {
      unsigned char trailer[16];
      std::memcpy(trailer, kDictEnd, 8);
      const uint64_t hv = w.hash.h;
      std::memcpy(trailer + 8, &hv, 8);
      w.ok = std::fwrite(trailer, 1, 16, w.f) == 16;
    }
    const bool closed = std::fclose(w.f) == 0;
    if (e != cudaSuccess || !w.ok || !closed) {
      std::remove(tmp.c_str());
      if (e != cudaSuccess) return cuda_fail(e, "dictionary copy to host");
      return fail(CALIBATT_ERR_INVALID_ARG, "writing %s failed", tmp.c_str());
    }
    if (std::rename(tmp.c_str(), path) != 0) {
      std::remove(tmp.c_str());
      return fail(CALIBATT_ERR_INVALID_ARG, "cannot rename %s to %s", tmp.c_str(), path);
    }
    return CALIBATT_OK;
  });
}

namespace {

calibatt_status load_records(DictReader& r, const DictFileHeader& hd, calibatt_dict* d, const char* path) {
  const int H = hd.H, nq = hd.nq;
  const int32_t words = (hd.nk + 31) / 32;
  const int64_t per_record_max = static_cast<int64_t>(H) * nq * hd.nk;
  int64_t prev_ly = -1, nnz_seen = 0;
  std::vector<uint8_t> rep(H);
  std::vector<int32_t> rp(static_cast<size_t>(H) * (nq + 1)), col32;
  std::vector<uint16_t> col;
  std::vector<uint32_t> bits;
  for (int64_t i = 0; i < hd.records; ++i) {
    DictFileRecord rec;
    if (!r.get(&rec, sizeof(rec))) return fail(CALIBATT_ERR_INVALID_ARG, "%s: record %lld is cut short", path, (long long)i);
    if (rec.t < 0 || rec.t >= hd.T || rec.l < 0 || rec.l >= hd.L)
      return fail(CALIBATT_ERR_INVALID_ARG, "%s: record (%d, %d) outside %d x %d", path, rec.t, rec.l, hd.T, hd.L);
    const int64_t ly = static_cast<int64_t>(rec.t) * hd.L + rec.l;
    if (ly <= prev_ly) return fail(CALIBATT_ERR_INVALID_ARG, "%s: records out of order", path);
    prev_ly = ly;
    if (rec.nnz < 0 || rec.nnz > per_record_max || nnz_seen + rec.nnz > hd.nnz_total)
      return fail(CALIBATT_ERR_INVALID_ARG, "%s: record (%d, %d) has %lld blocks", path, rec.t, rec.l, (long long)rec.nnz);
    nnz_seen += rec.nnz;
    if (!r.get(rep.data(), H)) return fail(CALIBATT_ERR_INVALID_ARG, "%s: record (%d, %d) is cut short", path, rec.t, rec.l);
    if (hd.format == 2) {
      // rec.nnz runs: row pointers (blocks), run pointers, packed runs
      std::vector<int32_t> run_ptr(rp.size());
      bits.resize(rec.nnz);
      if (!r.get(rp.data(), sizeof(int32_t) * rp.size()) ||
          !r.get(run_ptr.data(), sizeof(int32_t) * run_ptr.size()) ||
          !r.get(bits.data(), sizeof(uint32_t) * bits.size()))
        return fail(CALIBATT_ERR_INVALID_ARG, "%s: record (%d, %d) is cut short", path, rec.t, rec.l);
      // expand into per-head CSR; each row's runs must add up to its block count
      col32.clear();
      int64_t run_at = 0;
      for (int h = 0; h < H; ++h) {
        const int32_t* hp = rp.data() + static_cast<size_t>(h) * (nq + 1);
        const int32_t* rr = run_ptr.data() + static_cast<size_t>(h) * (nq + 1);
        if (rr[0] != 0) return fail(CALIBATT_ERR_INVALID_ARG, "%s: record (%d, %d) head %d run_ptr[0] != 0", path, rec.t, rec.l, h);
        const size_t head_start = col32.size();
        for (int q = 0; q < nq; ++q) {
          if (rr[q + 1] < rr[q] || run_at + (rr[q + 1] - rr[q]) > rec.nnz || hp[q] != static_cast<int32_t>(col32.size() - head_start))
            return fail(CALIBATT_ERR_INVALID_ARG, "%s: record (%d, %d) head %d runs do not match its rows", path, rec.t, rec.l, h);
          for (int32_t x = rr[q]; x < rr[q + 1]; ++x) {
            const uint32_t run = bits[run_at++];
            const int64_t start = run & 0xFFFFu, len = run >> 16;
            if (len < 1 || start + len > hd.nk || static_cast<int64_t>(col32.size() - head_start) + len > static_cast<int64_t>(nq) * (q + 1))
              return fail(CALIBATT_ERR_INVALID_ARG, "%s: record (%d, %d) has an invalid run", path, rec.t, rec.l);
            for (int64_t c = start; c < start + len; ++c) col32.push_back(static_cast<int32_t>(c));
          }
        }
        if (hp[nq] != static_cast<int32_t>(col32.size() - head_start))
          return fail(CALIBATT_ERR_INVALID_ARG, "%s: record (%d, %d) head %d runs do not match its rows", path, rec.t, rec.l, h);
      }
      if (run_at != rec.nnz)
        return fail(CALIBATT_ERR_INVALID_ARG, "%s: record (%d, %d) run count mismatch", path, rec.t, rec.l);
    } else if (hd.format == 1) {
      bits.resize(static_cast<size_t>(H) * nq * words);
      if (!r.get(bits.data(), sizeof(uint32_t) * bits.size()))
        return fail(CALIBATT_ERR_INVALID_ARG, "%s: record (%d, %d) is cut short", path, rec.t, rec.l);
      // decode into per-head CSR: row pointers counted from each head's first block
      col32.clear();
      for (int h = 0; h < H; ++h) {
        int32_t* hp = rp.data() + static_cast<size_t>(h) * (nq + 1);
        const size_t head_start = col32.size();
        for (int q = 0; q < nq; ++q) {
          hp[q] = static_cast<int32_t>(col32.size() - head_start);
          const uint32_t* row = bits.data() + (static_cast<size_t>(h) * nq + q) * words;
          for (int32_t wd = 0; wd < words; ++wd) {
            for (uint32_t x = row[wd]; x; x &= x - 1) {
              const int c = wd * 32 + __builtin_ctz(x);
              if (c >= hd.nk) return fail(CALIBATT_ERR_INVALID_ARG, "%s: bit beyond the last key block", path);
              col32.push_back(c);
            }
          }
        }
        hp[nq] = static_cast<int32_t>(col32.size() - head_start);
      }
    } else {
      if (!r.get(rp.data(), sizeof(int32_t) * rp.size()))
        return fail(CALIBATT_ERR_INVALID_ARG, "%s: record (%d, %d) is cut short", path, rec.t, rec.l);
      col.resize(rec.nnz);
      if (!r.get(col.data(), sizeof(uint16_t) * col.size()))
        return fail(CALIBATT_ERR_INVALID_ARG, "%s: record (%d, %d) is cut short", path, rec.t, rec.l);
      col32.assign(col.begin(), col.end());
    }
    // every head's row pointers start at 0 and never decrease, and together
    // they cover exactly the record's blocks, so each head's list lies inside col32
    int64_t total = 0;
    for (int h = 0; h < H; ++h) {
      const int32_t* hp = rp.data() + static_cast<size_t>(h) * (nq + 1);
      if (hp[0] != 0) return fail(CALIBATT_ERR_INVALID_ARG, "%s: record (%d, %d) head %d row_ptr[0] != 0", path, rec.t, rec.l, h);
      for (int q = 0; q < nq; ++q)
        if (hp[q + 1] < hp[q])
          return fail(CALIBATT_ERR_INVALID_ARG, "%s: record (%d, %d) head %d row_ptr decreases", path, rec.t, rec.l, h);
      total += hp[nq];
    }
    if (hd.format != 2 && (total != rec.nnz || static_cast<int64_t>(col32.size()) != rec.nnz))
      return fail(CALIBATT_ERR_INVALID_ARG, "%s: record (%d, %d) block count mismatch", path, rec.t, rec.l);
    if (hd.format == 2 && total != static_cast<int64_t>(col32.size()))
      return fail(CALIBATT_ERR_INVALID_ARG, "%s: record (%d, %d) block count mismatch", path, rec.t, rec.l);
    calibatt_status st = calibatt_dict_set_layer(d, rec.t, rec.l, rp.data(), col32.empty() ? nullptr : col32.data(), rep.data());
    if (st != CALIBATT_OK) return st;
  }
  if (nnz_seen != hd.nnz_total) return fail(CALIBATT_ERR_INVALID_ARG, "%s: total block count mismatch", path);
  return CALIBATT_OK;
}

}  // namespace

calibatt_status calibatt_dict_load(const char* path, int32_t num_ctas, calibatt_dict** out) {
  return guarded([&]() -> calibatt_status {
    if (!out || !path) return fail(CALIBATT_ERR_INVALID_ARG, "path and out must be non-NULL");
    *out = nullptr;
    DictReader r;
    r.f = std::fopen(path, "rb");
    if (!r.f) return fail(CALIBATT_ERR_INVALID_ARG, "cannot open %s", path);
    struct Closer {
      FILE* f;
      ~Closer() { std::fclose(f); }
    } closer{r.f};
    DictFileHeader hd;
    if (!r.get(&hd, sizeof(hd)) || std::memcmp(hd.magic, kDictMagic, 8) != 0)
      return fail(CALIBATT_ERR_INVALID_ARG, "%s is not a dictionary file", path);
    if (hd.version != kDictFileVersion || hd.format > 2 || hd.reserved != 0)
      return fail(CALIBATT_ERR_INVALID_ARG, "%s: unsupported version %u / format %u", path, hd.version, hd.format);
    if (hd.T < 1 || hd.L < 1 || hd.H < 1 || hd.nq < 1 || hd.nk != hd.nq || hd.H > 65535 || hd.nq > 65535 ||
        (hd.block != 64 && hd.block != 128) || hd.records < 0 || hd.records > static_cast<int64_t>(hd.T) * hd.L ||
        hd.nnz_total < 0 || (hd.format >= 1 && hd.nq > calibatt::kMaxBitmapBlocks) || hd.n_anchors < 0 ||
        hd.n_anchors > calibatt::kMaxAnchors || (hd.has_geom != 0 && hd.has_geom != 1))
      return fail(CALIBATT_ERR_INVALID_ARG, "%s: header fields out of range", path);
    calibatt_dict* d = nullptr;
    calibatt_status st =
        hd.format == 1 ? calibatt_dict_create_bitmap(hd.T, hd.L, hd.H, hd.nq, hd.nk, hd.block, num_ctas, &d)
        : hd.format == 2
            ? calibatt_dict_create_intervals(hd.T, hd.L, hd.H, hd.nq, hd.nk, hd.block, hd.nnz_total, num_ctas, &d)
            : calibatt_dict_create(hd.T, hd.L, hd.H, hd.nq, hd.nk, hd.block, hd.nnz_total, num_ctas, &d);
    if (st != CALIBATT_OK) return st;
    if (hd.has_geom) st = calibatt_dict_set_anchor_geometry(d, hd.frames, hd.rows, hd.cols, hd.anchors, hd.n_anchors);
    if (st == CALIBATT_OK) {
      try {
        st = load_records(r, hd, d, path);
      } catch (...) {
        calibatt_dict_destroy(d);  // then the guard reports the exception
        throw;
      }
    }
    if (st == CALIBATT_OK) {
      const uint64_t want = r.hash.h;
      unsigned char trailer[16];
      uint64_t got = 0;
      if (std::fread(trailer, 1, 16, r.f) != 16 || std::memcmp(trailer, kDictEnd, 8) != 0) {
        st = fail(CALIBATT_ERR_INVALID_ARG, "%s: trailer missing", path);
      } else {
        std::memcpy(&got, trailer + 8, 8);
        if (got != want) st = fail(CALIBATT_ERR_INVALID_ARG, "%s: checksum mismatch", path);
        else if (std::fgetc(r.f) != EOF) st = fail(CALIBATT_ERR_INVALID_ARG, "%s: trailing bytes", path);
      }
    }
    if (st != CALIBATT_OK) {
      const std::string msg = g_last_error;
      calibatt_dict_destroy(d);
      g_last_error = msg;
      return st;
    }
    *out = d;
    return CALIBATT_OK;
  });
}

calibatt_status calibatt_block_sparse_attn(const void* q, const void* k, const void* v, void* o,
                                           const calibatt_shape* shape, int32_t block, const calibatt_dict* dict,
                                           int32_t t, int32_t l, float softmax_scale, float* lse, void* stream) {
  return guarded([&]() -> calibatt_status {
    calibatt_status st;
    if ((st = check_shape(shape)) != CALIBATT_OK) return st;
    if ((st = check_ptrs(q, k, v, o)) != CALIBATT_OK) return st;
    if ((st = check_block(block)) != CALIBATT_OK) return st;
    if ((st = check_dict_layer(dict, t, l)) != CALIBATT_OK) return st;
    if (dict->H != shape->heads) return fail(CALIBATT_ERR_INVALID_ARG, "dictionary has %d heads, shape %d", dict->H, shape->heads);
    if (dict->block != block) return fail(CALIBATT_ERR_INVALID_ARG, "dictionary block %d != %d", dict->block, block);
    if (dict->nq != ceil_div(shape->seq_len, block))
      return fail(CALIBATT_ERR_INVALID_ARG, "dictionary has %d blocks, seq_len %d needs %d", dict->nq, shape->seq_len,
                  ceil_div(shape->seq_len, block));
    if (reinterpret_cast<uintptr_t>(lse) % 4) return fail(CALIBATT_ERR_INVALID_ARG, "lse must be 4-byte aligned");
    return launch_sparse(q, k, v, o, *shape, block, dict, t, l, softmax_scale, lse, static_cast<cudaStream_t>(stream));
  });
}

calibatt_status calibatt_block_sparse_attn_host(const void* q_host, const void* k_host, const void* v_host,
                                                void* o_host, void* q, void* k, void* v, void* o,
                                                const calibatt_shape* shape, int32_t block, const calibatt_dict* dict,
                                                int32_t t, int32_t l, float softmax_scale, float* lse,
                                                void* stream) {
  return guarded([&]() -> calibatt_status {
    calibatt_status st;
    if ((st = check_shape(shape)) != CALIBATT_OK) return st;
    if (!q_host || !k_host || !v_host || !o_host)
      return fail(CALIBATT_ERR_INVALID_ARG, "host buffers must be non-NULL");
    if ((st = check_ptrs(q, k, v, o)) != CALIBATT_OK) return st;
    // bytes from each tensor's base to one past its last element
    const int64_t elt = shape->dtype == CALIBATT_DTYPE_BF16 ? 2 : 4;
    const int64_t extent = ((static_cast<int64_t>(shape->batch) - 1) * shape->stride_b +
                            (static_cast<int64_t>(shape->seq_len) - 1) * shape->stride_n +
                            (static_cast<int64_t>(shape->heads) - 1) * shape->stride_h + shape->head_dim) * elt;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const void* src[3] = {q_host, k_host, v_host};
    void* dst[3] = {q, k, v};
    for (int i = 0; i < 3; ++i) {
      cudaError_t e = cudaMemcpyAsync(dst[i], src[i], static_cast<size_t>(extent), cudaMemcpyHostToDevice, cs);
      if (e != cudaSuccess) return cuda_fail(e, "host-to-device copy");
    }
    st = calibatt_block_sparse_attn(q, k, v, o, shape, block, dict, t, l, softmax_scale, lse, stream);
    if (st != CALIBATT_OK) return st;
    cudaError_t e = cudaMemcpyAsync(o_host, o, static_cast<size_t>(extent), cudaMemcpyDeviceToHost, cs);
    if (e != cudaSuccess) return cuda_fail(e, "device-to-host copy");
    return CALIBATT_OK;
  });
}

calibatt_status calibatt_block_sparse_attn_csr(const void* q, const void* k, const void* v, void* o,
                                               const calibatt_shape* shape, int32_t block, const int32_t* row_ptr,
                                               const uint16_t* col_idx, const int64_t* col_base,
                                               const int32_t* head_ids, int32_t n_heads, const uint32_t* items,
                                               const int32_t* cta_ptr, int32_t grid, float softmax_scale, float* lse,
                                               void* stream) {
  return guarded([&]() -> calibatt_status {
    calibatt_status st;
    if ((st = check_shape(shape)) != CALIBATT_OK) return st;
    if ((st = check_ptrs(q, k, v, o)) != CALIBATT_OK) return st;
    if ((st = check_block(block)) != CALIBATT_OK) return st;
    if (n_heads < 0 || n_heads > calibatt::kMaxHeadsPerCall)
      return fail(CALIBATT_ERR_INVALID_ARG, "n_heads must be in [0, %d]", calibatt::kMaxHeadsPerCall);
    if (n_heads == 0) return CALIBATT_OK;
    if (!head_ids || !row_ptr || !col_idx || !col_base)
      return fail(CALIBATT_ERR_INVALID_ARG, "head_ids, row_ptr, col_idx and col_base must be non-NULL");
    const int32_t nq = ceil_div(shape->seq_len, block);
    if (nq > 65535) return fail(CALIBATT_ERR_UNSUPPORTED, "more than 65535 blocks");
    std::vector<uint8_t> seen(shape->heads, 0);
    std::vector<int16_t> heads;
    for (int i = 0; i < n_heads; ++i) {
      if (head_ids[i] < 0 || head_ids[i] >= shape->heads)
        return fail(CALIBATT_ERR_INVALID_ARG, "head id %d outside [0, %d)", head_ids[i], shape->heads);
      if (seen[head_ids[i]]++) return fail(CALIBATT_ERR_INVALID_ARG, "head id %d listed twice", head_ids[i]);
      heads.push_back(static_cast<int16_t>(head_ids[i]));
    }
    const bool tc = shape->dtype == CALIBATT_DTYPE_BF16 && block == 128;
    if (tc && (!items || !cta_ptr || grid < 1))
      return fail(CALIBATT_ERR_INVALID_ARG, "the tensor-core path needs a device schedule (items, cta_ptr, grid >= 1)");
    if (reinterpret_cast<uintptr_t>(lse) % 4) return fail(CALIBATT_ERR_INVALID_ARG, "lse must be 4-byte aligned");
    // the lists were never read on the host: check them on the device first
    calibatt::CsrCheckParams chk;
    std::memset(&chk, 0, sizeof(chk));
    chk.row_ptr = row_ptr;
    chk.col = col_idx;
    chk.col_base = col_base;
    chk.nq = nq;
    chk.n_heads = n_heads;
    for (int i = 0; i < n_heads; ++i) chk.head_ids[i] = heads[i];
    chk.status = status_word_ptr();
    if (!chk.status) return fail(CALIBATT_ERR_CUDA, "status word unavailable");
    if (tc) {
      chk.items = items;
      chk.cta_ptr = cta_ptr;
      chk.grid = grid;
    }
    cudaError_t e = calibatt::launch_csr_check(chk, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "skip-list check launch");
    LayerSchedule sch;
    std::memset(&sch, 0, sizeof(sch));
    sch.row_ptr = row_ptr;
    sch.col_base = col_base;
    sch.col = col_idx;
    sch.items = items;
    sch.cta_ptr = cta_ptr;
    sch.nq = nq;
    sch.csr_gate = 1;
    return run_sparse(q, k, v, o, *shape, block, sch, tc ? grid : 1, heads, softmax_scale, lse,
                      static_cast<cudaStream_t>(stream));
  });
}

calibatt_status calibatt_anchor_attn(const void* q, const void* k, const void* v, void* o,
                                     const calibatt_shape* shape, int32_t block, int32_t frames, int32_t rows,
                                     int32_t cols, const int32_t* anchor_rows, int32_t n_anchors,
                                     const int32_t* head_ids, int32_t n_heads, float softmax_scale,
                                     void* workspace, size_t workspace_bytes, void* stream) {
  return guarded([&]() -> calibatt_status {
    calibatt_status st;
    if ((st = check_shape(shape)) != CALIBATT_OK) return st;
    if ((st = check_ptrs(q, k, v, o)) != CALIBATT_OK) return st;
    if ((st = check_block(block)) != CALIBATT_OK) return st;
    return launch_anchor(q, k, v, o, *shape, block, frames, rows, cols, anchor_rows, n_anchors, head_ids, n_heads,
                         softmax_scale, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
  });
}

calibatt_status calibatt_anchor_attn_workspace_size(const calibatt_shape* shape, int32_t frames, int32_t rows,
                                                    int32_t cols, int32_t n_anchors, int32_t n_heads, size_t* bytes) {
  return guarded([&]() -> calibatt_status {
    calibatt_status st;
    if ((st = check_shape(shape)) != CALIBATT_OK) return st;
    if (!bytes) return fail(CALIBATT_ERR_INVALID_ARG, "bytes is NULL");
    if (frames < 1 || rows < 1 || cols < 1 || n_anchors < 1 || n_anchors > calibatt::kMaxAnchors || n_heads < 0 ||
        n_heads > calibatt::kMaxHeadsPerCall)
      return fail(CALIBATT_ERR_INVALID_ARG, "frames, rows, cols, n_anchors or n_heads out of range");
    *bytes = 0;
    if (shape->dtype != CALIBATT_DTYPE_BF16 || n_heads == 0) return CALIBATT_OK;
    const int sms = device_sm_count();
    if (sms < 1) return fail(CALIBATT_ERR_CUDA, "cannot query the SM count");
    int64_t first = 0;
    int32_t parts = 1;
    const int64_t tiles = anchor_call_tiles(*shape, frames, cols, n_anchors, n_heads);
    anchor_split_plan(tiles, sms, ceil_div(shape->seq_len, 128), first, parts);
    *bytes = split_layout(tiles - first, parts, shape->head_dim).total;
    return CALIBATT_OK;
  });
}

calibatt_status calibatt_anchor_split_plan(int64_t tiles, int32_t grid, int32_t key_blocks, int64_t* first,
                                           int32_t* parts) {
  return guarded([&]() -> calibatt_status {
    if (!first || !parts) return fail(CALIBATT_ERR_INVALID_ARG, "first and parts must be non-NULL");
    if (tiles < 0 || grid < 1 || key_blocks < 1)
      return fail(CALIBATT_ERR_INVALID_ARG, "tiles >= 0, grid >= 1 and key_blocks >= 1 are required");
    anchor_split_plan(tiles, grid, key_blocks, *first, *parts);
    return CALIBATT_OK;
  });
}

calibatt_status calibatt_dual_path_attn(const void* q, const void* k, const void* v, void* o,
                                        const calibatt_shape* shape, int32_t block, const calibatt_dict* dict,
                                        int32_t t, int32_t l, int32_t frames, int32_t rows, int32_t cols,
                                        const int32_t* anchor_rows, int32_t n_anchors, float softmax_scale,
                                        float* lse, void* stream) {
  return guarded([&]() -> calibatt_status {
    // One launch when the dictionary carries this call's anchor geometry and
    // the tensor-core path applies; otherwise the sparse and anchor launches.
    if (dict && shape && dict->has_geom && shape->dtype == CALIBATT_DTYPE_BF16 && block == 128 &&
        frames == dict->g_frames && rows == dict->g_rows && cols == dict->g_cols && anchor_rows &&
        n_anchors == static_cast<int32_t>(dict->g_anchors.size()) &&
        std::equal(dict->g_anchors.begin(), dict->g_anchors.end(), anchor_rows)) {
      calibatt_status st;
      if ((st = check_shape(shape)) != CALIBATT_OK) return st;
      if ((st = check_ptrs(q, k, v, o)) != CALIBATT_OK) return st;
      if ((st = check_dict_layer(dict, t, l)) != CALIBATT_OK) return st;
      if (dict->H != shape->heads)
        return fail(CALIBATT_ERR_INVALID_ARG, "dictionary has %d heads, shape %d", dict->H, shape->heads);
      if (dict->block != block) return fail(CALIBATT_ERR_INVALID_ARG, "dictionary block %d != %d", dict->block, block);
      if (dict->nq != ceil_div(shape->seq_len, block))
        return fail(CALIBATT_ERR_INVALID_ARG, "dictionary has %d blocks, seq_len %d needs %d", dict->nq,
                    shape->seq_len, ceil_div(shape->seq_len, block));
      if (static_cast<int64_t>(frames) * rows * cols != shape->seq_len)
        return fail(CALIBATT_ERR_INVALID_ARG, "frames*rows*cols = %lld != seq_len %d", (long long)frames * rows * cols,
                    shape->seq_len);
      if (reinterpret_cast<uintptr_t>(lse) % 4) return fail(CALIBATT_ERR_INVALID_ARG, "lse must be 4-byte aligned");
      const int64_t ly = dict->layer(t, l);
      if (dict->n_sparse[ly] + dict->n_rep[ly] == 0) return CALIBATT_OK;
      return launch_fused(q, k, v, o, *shape, dict, t, l, softmax_scale, lse, static_cast<cudaStream_t>(stream));
    }
    calibatt_status st = calibatt_block_sparse_attn(q, k, v, o, shape, block, dict, t, l, softmax_scale, lse, stream);
    if (st != CALIBATT_OK) return st;
    const int64_t ly = dict->layer(t, l);
    std::vector<int32_t> heads;
    for (int h = 0; h < dict->H; ++h)
      if (dict->rep[ly * dict->H + h]) heads.push_back(h);
    if (heads.empty()) return CALIBATT_OK;
    for (size_t h0 = 0; h0 < heads.size(); h0 += calibatt::kMaxHeadsPerCall) {
      const int32_t nh = static_cast<int32_t>(std::min<size_t>(calibatt::kMaxHeadsPerCall, heads.size() - h0));
      st = launch_anchor(q, k, v, o, *shape, block, frames, rows, cols, anchor_rows, n_anchors, heads.data() + h0, nh,
                         softmax_scale, nullptr, 0, static_cast<cudaStream_t>(stream));
      if (st != CALIBATT_OK) return st;
    }
    return CALIBATT_OK;
  });
}

calibatt_status calibatt_block_energy_workspace_size(const calibatt_shape* shape, size_t* bytes) {
  return guarded([&]() -> calibatt_status {
    calibatt_status st = check_shape(shape);
    if (st != CALIBATT_OK) return st;
    if (!bytes) return fail(CALIBATT_ERR_INVALID_ARG, "bytes is NULL");
    *bytes = sizeof(float) * static_cast<size_t>(shape->batch) * shape->heads * shape->seq_len;
    return CALIBATT_OK;
  });
}

calibatt_status calibatt_block_energy(const void* q, const void* k, const calibatt_shape* shape, int32_t block,
                                      float softmax_scale, float* energy, void* workspace, size_t workspace_bytes,
                                      void* stream) {
  return guarded([&]() -> calibatt_status {
    calibatt_status st;
    if ((st = check_shape(shape)) != CALIBATT_OK) return st;
    if ((st = check_block(block)) != CALIBATT_OK) return st;
    if (!q || !k || !energy || !workspace) return fail(CALIBATT_ERR_INVALID_ARG, "q, k, energy and workspace must be non-NULL");
    size_t need = 0;
    calibatt_block_energy_workspace_size(shape, &need);
    if (workspace_bytes < need)
      return fail(CALIBATT_ERR_INVALID_ARG, "workspace of %zu bytes < %zu needed", workspace_bytes, need);
    const int nb = ceil_div(shape->seq_len, block);
    if (nb > 65535) return fail(CALIBATT_ERR_UNSUPPORTED, "more than 65535 blocks");
    if (shape->dtype == CALIBATT_DTYPE_BF16 && block == 128) {
      // Tensor-core path: the LSE pass, then the energy pass, as persistent
      // launches of the attention pipeline without V.
      TcParams t;
      std::memset(&t, 0, sizeof(t));
      if ((st = encode_qkv_map(&t.tm_q, q, *shape, &t.pos_n, &t.pos_h, &t.pos_b)) != CALIBATT_OK) return st;
      if ((st = encode_qkv_map(&t.tm_k, k, *shape, &t.pos_n, &t.pos_h, &t.pos_b)) != CALIBATT_OK) return st;
      t.tm_v = t.tm_k;  // no V in these modes
      t.q = static_cast<const uint16_t*>(q);
      t.lse = static_cast<float*>(workspace);
      t.energy = energy;
      t.sb = shape->stride_b;
      t.sn = shape->stride_n;
      t.sh = shape->stride_h;
      t.batch = shape->batch;
      t.seq_len = shape->seq_len;
      t.heads = shape->heads;
      t.nb = nb;
      t.scale_log2 = scale_log2_of(softmax_scale, shape->head_dim);
      t.status = status_word_ptr();
      t.timeout_ns = g_timeout_ns.load();
      const int sms = device_sm_count();
      if (sms < 1) return fail(CALIBATT_ERR_CUDA, "cannot query the SM count");
      const int grid = static_cast<int>(std::min<int64_t>(sms, static_cast<int64_t>(shape->heads) * nb));
      cudaStream_t cs = static_cast<cudaStream_t>(stream);
      cudaError_t e = calibatt::launch_tc_attn(t, shape->head_dim, calibatt::kModeLse, grid, cs);
      if (e == cudaSuccess) e = calibatt::launch_tc_attn(t, shape->head_dim, calibatt::kModeEnergy, grid, cs);
      if (e != cudaSuccess) return cuda_fail(e, "tensor-core block energy launch");
      return CALIBATT_OK;
    }
    calibatt::EnergyParams p;
    std::memset(&p, 0, sizeof(p));
    p.q = q;
    p.k = k;
    p.energy = energy;
    p.lse = static_cast<float*>(workspace);
    p.sb = shape->stride_b;
    p.sn = shape->stride_n;
    p.sh = shape->stride_h;
    p.batch = shape->batch;
    p.seq_len = shape->seq_len;
    p.heads = shape->heads;
    p.nb = nb;
    p.scale_log2 = scale_log2_of(softmax_scale, shape->head_dim);
    cudaError_t e = calibatt::launch_block_energy(p, shape->head_dim, block, shape->dtype, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "block energy launch");
    return CALIBATT_OK;
  });
}

calibatt_status calibatt_spatial_similarity_workspace_size(const calibatt_shape* shape, size_t* bytes) {
  return guarded([&]() -> calibatt_status {
    calibatt_status st;
    if ((st = check_shape(shape)) != CALIBATT_OK) return st;
    if (!bytes) return fail(CALIBATT_ERR_INVALID_ARG, "bytes is NULL");
    // per query: its log-sum-exp, and on the tensor-core path (bf16) its three sums
    const size_t per_query = shape->dtype == CALIBATT_DTYPE_BF16 ? 4 : 1;
    *bytes = sizeof(float) * per_query * static_cast<size_t>(shape->batch) * shape->heads * shape->seq_len;
    return CALIBATT_OK;
  });
}

calibatt_status calibatt_spatial_similarity(const void* q, const void* k, const calibatt_shape* shape, int32_t frames,
                                            int32_t rows, int32_t cols, const int32_t* anchor_rows, int32_t n_anchors,
                                            float softmax_scale, float* similarity, void* workspace,
                                            size_t workspace_bytes, void* stream) {
  return guarded([&]() -> calibatt_status {
    calibatt_status st;
    if ((st = check_shape(shape)) != CALIBATT_OK) return st;
    if (!q || !k || !similarity || !workspace)
      return fail(CALIBATT_ERR_INVALID_ARG, "q, k, similarity and workspace must be non-NULL");
    if (frames < 1 || rows < 1 || cols < 1) return fail(CALIBATT_ERR_INVALID_ARG, "frames, rows and cols must be >= 1");
    if (static_cast<int64_t>(frames) * rows * cols != shape->seq_len)
      return fail(CALIBATT_ERR_INVALID_ARG, "frames*rows*cols = %lld != seq_len %d", (long long)frames * rows * cols,
                  shape->seq_len);
    if (rows > calibatt::kMaxRepetitionRows)
      return fail(CALIBATT_ERR_UNSUPPORTED, "more than %d spatial rows per frame", calibatt::kMaxRepetitionRows);
    if (!anchor_rows || n_anchors < 1 || n_anchors > calibatt::kMaxAnchors)
      return fail(CALIBATT_ERR_INVALID_ARG, "n_anchors must be in [1, %d] with a non-NULL list", calibatt::kMaxAnchors);
    for (int a = 0; a < n_anchors; ++a) {
      if (anchor_rows[a] < 0 || anchor_rows[a] >= rows)
        return fail(CALIBATT_ERR_INVALID_ARG, "anchor row %d outside [0, %d)", anchor_rows[a], rows);
      if (a > 0 && anchor_rows[a] <= anchor_rows[a - 1])
        return fail(CALIBATT_ERR_INVALID_ARG, "anchor rows must be strictly ascending");
    }
    size_t need = 0;
    calibatt_spatial_similarity_workspace_size(shape, &need);
    if (workspace_bytes < need)
      return fail(CALIBATT_ERR_INVALID_ARG,
                  "workspace of %zu bytes < %zu needed (calibatt_spatial_similarity_workspace_size)",
                  workspace_bytes, need);
    const float sl2 = scale_log2_of(softmax_scale, shape->head_dim);
    if (shape->dtype == CALIBATT_DTYPE_BF16) {
      if (reinterpret_cast<uintptr_t>(q) % 16 || reinterpret_cast<uintptr_t>(k) % 16)
        return fail(CALIBATT_ERR_INVALID_ARG, "q and k must be 16-byte aligned");
      // Tensor-core path: the LSE pass, the pass of per-query sums (two score
      // tiles per key block: the queries and their anchor-row partners), and
      // the rows' fixed-order reduction.
      TcParams t;
      std::memset(&t, 0, sizeof(t));
      if ((st = encode_qkv_map(&t.tm_q, q, *shape, &t.pos_n, &t.pos_h, &t.pos_b)) != CALIBATT_OK) return st;
      if ((st = encode_qkv_map(&t.tm_k, k, *shape, &t.pos_n, &t.pos_h, &t.pos_b)) != CALIBATT_OK) return st;
      t.tm_v = t.tm_k;  // no V in these modes
      const int64_t plane = static_cast<int64_t>(shape->batch) * shape->heads * shape->seq_len;
      t.q = static_cast<const uint16_t*>(q);
      t.lse = static_cast<float*>(workspace);
      t.energy = static_cast<float*>(workspace) + plane;  // three planes of per-query sums
      t.sb = shape->stride_b;
      t.sn = shape->stride_n;
      t.sh = shape->stride_h;
      t.batch = shape->batch;
      t.seq_len = shape->seq_len;
      t.heads = shape->heads;
      t.nb = ceil_div(shape->seq_len, 128);
      t.scale_log2 = sl2;
      t.anc.frames = frames;
      t.anc.rows = rows;
      t.anc.cols = cols;
      t.anc.n_anchors = n_anchors;
      anchor_groups(rows, anchor_rows, n_anchors, t.anc);
      t.status = status_word_ptr();
      t.timeout_ns = g_timeout_ns.load();
      const int sms = device_sm_count();
      if (sms < 1) return fail(CALIBATT_ERR_CUDA, "cannot query the SM count");
      const int grid = static_cast<int>(std::min<int64_t>(sms, static_cast<int64_t>(shape->heads) * t.nb));
      cudaStream_t cs = static_cast<cudaStream_t>(stream);
      cudaError_t e = calibatt::launch_tc_attn(t, shape->head_dim, calibatt::kModeLse, grid, cs);
      if (e == cudaSuccess) e = calibatt::launch_tc_attn(t, shape->head_dim, calibatt::kModeSimilarity, grid, cs);
      if (e == cudaSuccess)
        e = calibatt::launch_similarity_from_sums(t.energy, plane, shape->batch * shape->heads, shape->seq_len,
                                                  frames, rows, cols, similarity, cs);
      if (e != cudaSuccess) return cuda_fail(e, "tensor-core spatial similarity launch");
      return CALIBATT_OK;
    }
    calibatt::EnergyParams e;
    std::memset(&e, 0, sizeof(e));
    e.q = q;
    e.k = k;
    e.lse = static_cast<float*>(workspace);
    e.sb = shape->stride_b;
    e.sn = shape->stride_n;
    e.sh = shape->stride_h;
    e.batch = shape->batch;
    e.seq_len = shape->seq_len;
    e.heads = shape->heads;
    e.scale_log2 = sl2;
    cudaError_t ce = calibatt::launch_row_lse(e, shape->head_dim, shape->dtype, static_cast<cudaStream_t>(stream));
    if (ce != cudaSuccess) return cuda_fail(ce, "row log-sum-exp launch");
    calibatt::RepetitionParams p;
    std::memset(&p, 0, sizeof(p));
    p.q = q;
    p.k = k;
    p.lse = static_cast<const float*>(workspace);
    p.sim = similarity;
    p.sb = shape->stride_b;
    p.sn = shape->stride_n;
    p.sh = shape->stride_h;
    p.batch = shape->batch;
    p.seq_len = shape->seq_len;
    p.heads = shape->heads;
    p.frames = frames;
    p.rows = rows;
    p.cols = cols;
    p.scale_log2 = sl2;
    // nearest anchor of each row, ties to the lower anchor (as the anchor path)
    for (int32_t rho = 0; rho < rows; ++rho) {
      int best = 0;
      for (int a = 1; a < n_anchors; ++a)
        if (std::abs(rho - anchor_rows[a]) < std::abs(rho - anchor_rows[best])) best = a;
      p.nearest[rho] = static_cast<int16_t>(anchor_rows[best]);
    }
    ce = calibatt::launch_spatial_similarity(p, shape->head_dim, shape->dtype, static_cast<cudaStream_t>(stream));
    if (ce != cudaSuccess) return cuda_fail(ce, "spatial similarity launch");
    return CALIBATT_OK;
  });
}

calibatt_status calibatt_repetition_flags(const float* similarity, int32_t n_prompts, int32_t n_heads,
                                          int32_t per_head, float threshold, float* mean, uint8_t* flags,
                                          void* stream) {
  return guarded([&]() -> calibatt_status {
    if (n_prompts < 1 || n_heads < 0 || per_head < 1)
      return fail(CALIBATT_ERR_INVALID_ARG, "n_prompts and per_head must be >= 1, n_heads >= 0");
    if (n_heads > 0 && (!similarity || !flags))
      return fail(CALIBATT_ERR_INVALID_ARG, "similarity and flags must be non-NULL");
    if (!(threshold == threshold)) return fail(CALIBATT_ERR_INVALID_ARG, "threshold is NaN");
    cudaError_t e = calibatt::launch_repetition_flags(similarity, n_prompts, n_heads, per_head, threshold, mean, flags,
                                                      static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "repetition flags launch");
    return CALIBATT_OK;
  });
}

calibatt_status calibatt_select_blocks(const float* energy, int64_t n_rows, int32_t nk, float tau, uint8_t* mask,
                                       int32_t* count_accum, void* stream) {
  return guarded([&]() -> calibatt_status {
    if (n_rows < 0 || nk < 1) return fail(CALIBATT_ERR_INVALID_ARG, "n_rows must be >= 0 and nk >= 1");
    if (nk > 4096) return fail(CALIBATT_ERR_UNSUPPORTED, "nk %d > 4096", nk);
    if (n_rows > 2147483647LL) return fail(CALIBATT_ERR_UNSUPPORTED, "too many rows");
    if (n_rows > 0 && (!energy || !mask)) return fail(CALIBATT_ERR_INVALID_ARG, "energy and mask must be non-NULL");
    if (!(tau == tau)) return fail(CALIBATT_ERR_INVALID_ARG, "tau is NaN");
    cudaError_t e = calibatt::launch_select_blocks(energy, n_rows, nk, tau, mask, count_accum, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "select launch");
    return CALIBATT_OK;
  });
}

calibatt_status calibatt_aggregate_masks(const int32_t* counts, int64_t n, int32_t n_prompts, float rho,
                                         uint8_t* mask, void* stream) {
  return guarded([&]() -> calibatt_status {
    if (n < 0 || n_prompts < 1) return fail(CALIBATT_ERR_INVALID_ARG, "n must be >= 0 and n_prompts >= 1");
    if (n > 0 && (!counts || !mask)) return fail(CALIBATT_ERR_INVALID_ARG, "counts and mask must be non-NULL");
    if (!(rho == rho)) return fail(CALIBATT_ERR_INVALID_ARG, "rho is NaN");
    cudaError_t e = calibatt::launch_aggregate(counts, n, n_prompts, rho, mask, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "aggregate launch");
    return CALIBATT_OK;
  });
}

calibatt_status calibatt_debug_exp2_fma(const float* x, float* y, int64_t n, void* stream) {
  return guarded([&]() -> calibatt_status {
    if (n < 0) return fail(CALIBATT_ERR_INVALID_ARG, "n must be >= 0");
    if (n > 0 && (!x || !y)) return fail(CALIBATT_ERR_INVALID_ARG, "x and y must be non-NULL");
    cudaError_t e = calibatt::launch_exp2_fma(x, y, n, false, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "exp2 launch");
    return CALIBATT_OK;
  });
}

calibatt_status calibatt_debug_exp2_fma_quintic(const float* x, float* y, int64_t n, void* stream) {
  return guarded([&]() -> calibatt_status {
    if (n < 0) return fail(CALIBATT_ERR_INVALID_ARG, "n must be >= 0");
    if (n > 0 && (!x || !y)) return fail(CALIBATT_ERR_INVALID_ARG, "x and y must be non-NULL");
    cudaError_t e = calibatt::launch_exp2_fma(x, y, n, true, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "exp2 launch");
    return CALIBATT_OK;
  });
}

calibatt_status calibatt_debug_bounded_wait(void* stream) {
  return guarded([&]() -> calibatt_status {
    int32_t* p = status_word_ptr();
    if (!p) return fail(CALIBATT_ERR_CUDA, "status word unavailable");
    cudaError_t e = calibatt::launch_bounded_wait(p, g_timeout_ns.load(), static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "bounded wait launch");
    return CALIBATT_OK;
  });
}

calibatt_status calibatt_device_status(void* stream, int32_t* code, int32_t clear) {
  return guarded([&]() -> calibatt_status {
    if (!code) return fail(CALIBATT_ERR_INVALID_ARG, "code is NULL");
    int32_t* p = status_word_ptr();
    if (!p) return fail(CALIBATT_ERR_CUDA, "status word unavailable");
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
    e = cudaMemcpy(code, p, sizeof(int32_t), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "status read");
    if (clear) {
      e = cudaMemset(p, 0, sizeof(int32_t));
      if (e != cudaSuccess) return cuda_fail(e, "status clear");
    }
    if (*code != 0) {
      if ((*code & 0xFF) == CALIBATT_ERR_INVALID_ARG && ((*code >> 8) & 0xFF) == calibatt::kCodeScheduleViolation)
        return fail(CALIBATT_ERR_INVALID_ARG,
                    "a direct-CSR call's device schedule names an unlisted head or a query block >= nq, or its "
                    "CTA offsets are not 0 .. n_heads*nq non-decreasing (code 0x%x)", *code);
      if ((*code & 0xFF) == CALIBATT_ERR_INVALID_ARG)
        return fail(CALIBATT_ERR_INVALID_ARG,
                    "a kernel met a key-block index outside the key range, or a direct-CSR call's row pointers "
                    "or list order were invalid (code 0x%x)", *code);
      return fail(CALIBATT_ERR_TIMEOUT, "device wait gave up (code 0x%x)", *code);
    }
    return CALIBATT_OK;
  });
}

calibatt_status calibatt_set_wait_timeout_ms(int32_t ms) {
  return guarded([&]() -> calibatt_status {
    if (ms < 1) return fail(CALIBATT_ERR_INVALID_ARG, "timeout must be >= 1 ms");
    g_timeout_ns.store(static_cast<unsigned long long>(ms) * 1000000ull);
    return CALIBATT_OK;
  });
}

calibatt_status calibatt_device_sm_count(int32_t* out) {
  return guarded([&]() -> calibatt_status {
    if (!out) return fail(CALIBATT_ERR_INVALID_ARG, "out is NULL");
    const int n = device_sm_count();
    if (n < 1) {
      cudaGetLastError();
      return fail(CALIBATT_ERR_CUDA, "no CUDA device");
    }
    *out = n;
    return CALIBATT_OK;
  });
}

}  // extern "C"
