// Tensor-core attention for CalibAtt on sm_100a (B200): the block-sparse path
// and the anchor-row path with broadcast, one persistent kernel template.
//
// What it computes ("Accelerating Text-to-Video Generation with Calibrated
// Sparse Attention", paper note, Key Designs 3 and 4): for each scheduled
// 128-query tile, softmax attention over a list of 128-key blocks -- the
// calibrated skip list of the (head, query block) on the sparse path, or every
// key block for a tile of gathered anchor-row queries on the anchor path --
// normalised and written once per query on the sparse path and to every row
// an anchor serves on the anchor path.
//
// Two softmax streams per query tile.  Key blocks at even list positions go
// to stream 0 and odd positions to stream 1; each stream keeps its own running
// maximum m, row sum l and output accumulator O in tensor memory, and the
// epilogue merges them exactly:
//   m = max(m0, m1),  a_s = 2^(m_s - m),  O = (a0 O0 + a1 O1) / (a0 l0 + a1 l1).
// The MMA warp issues S(j) = Q K_j^T, then O_s += P(j-1) V_{j-1} for the other
// stream, then S(j+1), ... so the tensor core computes one stream's products
// while the other stream's softmax warps exponentiate.  K and V tiles are still
// loaded once each, in list order.
//
// CTA layout (352 threads, one CTA per SM, persistent):
//   warps 0-3  softmax of stream 0, warps 4-7 softmax of stream 1: thread t of
//              a group owns query row t (TMEM lane t) and a whole 128-key score
//              row; in the epilogue the two groups split the output columns
//   warp  8    producer of Q (TMA, or a plain-load gather of anchor rows)
//              and of the K tiles gathered by block index
//   warp  9    TMEM allocator and MMA issuer (one lane issues tcgen05.mma)
//   warp 10    producer of the V tiles
// Tensor memory (512 columns): stream s has S_s at 128*s (f32 scores; its bf16
// probabilities P_s overwrite the first 64 columns once the scores are in
// registers) and O_s at 256 + 128*s.  S_s(j+2) is issued after O_s += P_s(j) V_j
// on the same thread, and tcgen05 MMAs from one thread run in issue order, so
// the P values are read before the next scores overwrite them.
// The softmax keeps a reference maximum per stream and only rescales O_s and
// l_s when a row maximum exceeds it by more than 2^8 (exp2 domain), so P <= 256.
#include "internal.h"
#include "ptx.cuh"

#include <math.h>

namespace calibatt {
namespace {

using namespace ptx;

// Pipeline trace (compiled only with -DCALIBATT_TRACE): lane 0 of selected
// warps of CTA 0 records the SM clock per (event, key-block iteration) into a
// device array, read back by calibatt_trace_read.  Off in the shipped library.
#ifdef CALIBATT_TRACE
constexpr unsigned kTraceIters = 4096;
constexpr unsigned kTraceEvents = 64;
__device__ unsigned long long g_trace[kTraceEvents * kTraceIters];
__device__ __forceinline__ void trace_event(int ev, uint32_t idx) {
  if (blockIdx.x == 0 && idx < kTraceIters) g_trace[ev * kTraceIters + idx] = clock64();
}
#define CALIBATT_TRACE_EVENT(cond, ev, idx) \
  do {                                     \
    if (cond) trace_event(ev, idx);        \
  } while (0)
#else
#define CALIBATT_TRACE_EVENT(cond, ev, idx) \
  do {                                     \
  } while (0)
#endif

constexpr int kThreads = 352;       // 8 softmax warps, Q/K producer, MMA, V producer
constexpr int kProducerWarp = 8;    // Q and K tiles
constexpr int kMmaWarp = 9;
constexpr int kVProducerWarp = 10;  // V tiles
constexpr int kGroupThreads = 128;  // softmax threads per stream
constexpr int kSoftmaxThreads = 256;
constexpr int kKStages = 3;
constexpr int kVStages = 2;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;    // S_s (and P_s) at kColS + 128 * s
constexpr uint32_t kColO = 256;  // O_s at kColO + 128 * s
constexpr float kRescaleLog2 = 8.0f;
// One pair in kPolyEvery of exponentials runs on the FMA pipe (exp2_fma)
// instead of the MUFU unit (0 = all on MUFU).
#ifndef CALIBATT_POLY_EVERY
#define CALIBATT_POLY_EVERY 0
#endif
constexpr int kPolyEvery = CALIBATT_POLY_EVERY;
// Exponential phases of consecutive key blocks (which alternate between the
// two streams) take turns on the MUFU unit instead of overlapping (1 = on;
// measured slower than free overlap on B200, so off by default).
#ifndef CALIBATT_EXP_TURNS
#define CALIBATT_EXP_TURNS 0
#endif
constexpr bool kExpTurns = CALIBATT_EXP_TURNS != 0;
constexpr int kChunkBytes = 128 * 128;  // 128 rows x 64 bf16 (one 128-byte swizzle span)

// Shared-memory layout (offsets from a 1024-byte aligned base).
template <int HD>
struct Layout {
  static constexpr int kTile = 128 * HD * 2;
  static constexpr int kQ = 0;
  static constexpr int kK = kTile;
  static constexpr int kV = kK + kKStages * kTile;
  static constexpr int kBar = kV + kVStages * kTile;
  // barrier indices
  static constexpr int bQFull = 0, bQEmpty = 1;
  static constexpr int bKFull = 2, bKEmpty = bKFull + kKStages;
  static constexpr int bVFull = bKEmpty + kKStages, bVEmpty = bVFull + kVStages;
  static constexpr int bSFull = bVEmpty + kVStages;  // [2] scores of stream s ready
  static constexpr int bPFull = bSFull + 2;          // [2] probabilities of stream s ready
  static constexpr int bPVDone = bPFull + 2;         // [2] O_s += P_s V finished
  static constexpr int bOFree = bPVDone + 2;         // epilogue has read O_0 and O_1
  static constexpr int bTurn = bOFree + 1;           // [2] stream s may start its exponentials
  static constexpr int bDrain = bTurn + 2;
  static constexpr int kNumBars = bDrain + 1;
  static constexpr int kMisc = kBar + kNumBars * 8;  // u32 tmem base, i32 abort flag
  static constexpr int kXchg = kMisc + 16;  // float [2 item parity][2 streams][2 (m, l)][128 rows]
  static constexpr int kUsed = kXchg + 2 * 2 * 2 * 128 * 4;
  // +1024 for aligning the base; at least 120 KB so only one CTA fits per SM
  // (each CTA holds all 512 tensor-memory columns).
  static constexpr int kBytes = (kUsed + 1024) > 120 * 1024 ? (kUsed + 1024) : 120 * 1024;
};

struct Item {
  int b, h, tile;            // batch, head, query block (sparse) or anchor tile
  int n;                     // key blocks to visit
  const uint16_t* cols;      // retained key blocks (sparse), nullptr = 0..n-1
  bool ragged_last;          // last visited key block is the partial one
};

// Walks this CTA's work items in the same order in every role.
template <bool ANCHOR>
struct Cursor {
  int b, idx, begin, end, step;
  __device__ void init(const TcParams& p) {
    b = 0;
    if (ANCHOR) {
      begin = blockIdx.x;
      end = p.anc.n_heads * p.anc.tiles_per_head;
      step = gridDim.x;
    } else {
      begin = p.sched.cta_ptr[blockIdx.x];
      end = p.sched.cta_ptr[blockIdx.x + 1];
      step = 1;
    }
    idx = begin;
  }
  __device__ bool next(const TcParams& p, Item& it) {
    while (b < p.batch) {
      if (idx < end) {
        it.b = b;
        if (ANCHOR) {
          it.h = p.anc.head_ids[idx / p.anc.tiles_per_head];
          it.tile = idx % p.anc.tiles_per_head;
          it.n = p.nb;
          it.cols = nullptr;
          it.ragged_last = (p.seq_len % 128) != 0;
        } else {
          const uint32_t w = p.sched.items[idx];
          it.h = static_cast<int>(w >> 16);
          it.tile = static_cast<int>(w & 0xFFFFu);
          const int32_t* rp = p.sched.row_ptr + static_cast<int64_t>(it.h) * (p.sched.nq + 1);
          const int s0 = rp[it.tile];
          it.n = rp[it.tile + 1] - s0;
          it.cols = p.sched.col + p.sched.col_base[it.h] + s0;
          it.ragged_last = it.n > 0 && (p.seq_len % 128) != 0 && it.cols[it.n - 1] == p.nb - 1;
        }
        idx += step;
        return true;
      }
      ++b;
      idx = begin;
    }
    return false;
  }
};

__device__ __forceinline__ void map_coords(const TcParams& p, int n0, int h, int b, int& c1,
                                           int& c2, int& c3) {
  c1 = p.pos_n == 1 ? n0 : (p.pos_h == 1 ? h : b);
  c2 = p.pos_n == 2 ? n0 : (p.pos_h == 2 ? h : b);
  c3 = p.pos_n == 3 ? n0 : (p.pos_h == 3 ? h : b);
}

template <int HD>
__device__ __forceinline__ void tma_tile(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                         const TcParams& p, int n0, int h, int b) {
  int c1, c2, c3;
  map_coords(p, n0, h, b, c1, c2, c3);
#pragma unroll
  for (int ch = 0; ch < HD / 64; ++ch) tma_load_4d(dst + ch * kChunkBytes, map, bar, ch * 64, c1, c2, c3);
}

// Bounded wait on a barrier whose waiters have already given up elsewhere:
// used only to let this role's own asynchronous copies/MMAs land before exit.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const unsigned long long t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > 200000000ull) break;  // 0.2 s
  }
}

// --------------------------------------------------------------- producers
// Q/K producer (V == false) and V producer (V == true) walk the same items and
// key blocks; each lets its own in-flight bulk copies land before exiting.
template <int HD, bool ANCHOR, bool V>
__device__ void producer_role(const TcParams& p, uint32_t base, const Waiter& W, int lane) {
  using L = Layout<HD>;
  auto bar = [&](int i) { return base + L::kBar + 8u * i; };
  constexpr int kStages = V ? kVStages : kKStages;
  constexpr int kFull = V ? L::bVFull : L::bKFull;
  constexpr int kEmpty = V ? L::bVEmpty : L::bKEmpty;
  constexpr int kRing = V ? L::kV : L::kK;
  const CUtensorMap* map = V ? &p.tm_v : &p.tm_k;
  Cursor<ANCHOR> cur;
  cur.init(p);
  Item it;
  uint32_t kv = 0, item = 0, issued = 0, q_issued = 0;
  bool ok = true;
  while (ok && cur.next(p, it)) {
    if (!V) {
      if (item > 0 && !W.wait(bar(L::bQEmpty), (item - 1) & 1, 1)) break;
      if (ANCHOR) {
        // Gather this tile's 128 anchor-row queries into the 128-byte swizzled
        // K-major layout the MMA expects (16-byte unit u of row r lands at
        // chunk u/8, row r, position (u%8) ^ (r%8)).
        constexpr int kUnits = HD / 8;
        const int per_frame = p.anc.n_anchors * p.anc.cols;
        const uint16_t* qb = p.q + static_cast<int64_t>(it.b) * p.sb + static_cast<int64_t>(it.h) * p.sh;
        for (int idx = lane; idx < 128 * kUnits; idx += 32) {
          const int r = idx / kUnits, u = idx % kUnits;
          const int pq = it.tile * 128 + r;
          uint4 val = make_uint4(0u, 0u, 0u, 0u);
          if (pq < p.anc.anchor_tokens) {
            const int f = pq / per_frame, rem = pq % per_frame;
            const int a = rem / p.anc.cols, w = rem % p.anc.cols;
            const int64_t token = (static_cast<int64_t>(f) * p.anc.rows + p.anc.anchor_row[a]) * p.anc.cols + w;
            val = __ldg(reinterpret_cast<const uint4*>(qb + token * p.sn + u * 8));
          }
          const uint32_t dst = base + L::kQ + (u >> 3) * kChunkBytes + r * 128 + (((u & 7) ^ (r & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(val.x), "r"(val.y),
                       "r"(val.z), "r"(val.w)
                       : "memory");
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::bQFull));
      } else {
        if (lane == 0) {
          mbar_arrive_expect_tx(bar(L::bQFull), L::kTile);
          tma_tile<HD>(base + L::kQ, &p.tm_q, bar(L::bQFull), p, it.tile * 128, it.h, it.b);
        }
        ++q_issued;
      }
    }
    uint32_t my_col = 0;
    for (int j = 0; j < it.n; ++j) {
      if ((j & 31) == 0) {
        const int jj = j + lane;
        my_col = ANCHOR ? static_cast<uint32_t>(jj) : (jj < it.n ? it.cols[jj] : 0u);
      }
      const int c = static_cast<int>(__shfl_sync(0xFFFFFFFFu, my_col, j & 31));
      const uint32_t slot = kv % kStages, use = kv / kStages;
      if (use > 0 && !W.wait(bar(kEmpty + slot), (use - 1) & 1, V ? 3 : 2)) { ok = false; break; }
      if (lane == 0) {
        mbar_arrive_expect_tx(bar(kFull + slot), L::kTile);
        tma_tile<HD>(base + kRing + slot * L::kTile, map, bar(kFull + slot), p, c * 128, it.h, it.b);
      }
      CALIBATT_TRACE_EVENT(lane == 0, V ? 2 : 1, kv);
      ++issued;
      ++kv;
    }
    ++item;
  }
  // Let every bulk copy this warp issued land before the CTA can exit.
  for (uint32_t s = 0; s < static_cast<uint32_t>(kStages); ++s)
    if (issued > s) drain_wait(bar(kFull + s), ((issued - 1 - s) / kStages) & 1);
  if (q_issued > 0) drain_wait(bar(L::bQFull), (q_issued - 1) & 1);
}


// -------------------------------------------------------------------- MMA
template <int HD, bool ANCHOR>
__device__ void mma_role(const TcParams& p, uint32_t base, uint32_t tmem, const Waiter& W, int lane) {
  using L = Layout<HD>;
  auto bar = [&](int i) { return base + L::kBar + 8u * i; };
  constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, 0);
  constexpr uint32_t kIdescO = idesc_bf16_f32(128, HD, 1);
  Cursor<ANCHOR> cur;
  cur.init(p);
  Item it;
  uint32_t kv = 0, item = 0;  // global key-block iteration, item counter
  uint32_t ta = 0, tb = 0;    // key blocks issued to stream 0 / stream 1 (global)
  bool ok = true;

  // O_s += P_s(g) V_g for the item-local block index jl (stream jl & 1) whose
  // global iteration is g and whose per-stream ordinal is ts.
  auto issue_pv = [&](int jl, uint32_t g, uint32_t ts) -> bool {
    const int s = jl & 1;
    const uint32_t vs = g % kVStages;
    if (!W.wait(bar(L::bVFull + vs), (g / kVStages) & 1, 7)) return false;
    if (!W.wait(bar(L::bPFull + s), ts & 1, 8)) return false;
    if (jl == 0 && item > 0 && !W.wait(bar(L::bOFree), (item - 1) & 1, 9)) return false;
    tc_fence_after();
    CALIBATT_TRACE_EVENT(lane == 0, 4, g);
    if (lane == 0) {
      const uint32_t v_base = base + L::kV + vs * L::kTile;
      const bool first = jl < 2;  // first block of this stream in the item
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        // A = P_s in tensor memory (16 keys = 8 columns per step); B = V
        // (MN-major): 16 keys per step = 2048 bytes; next 64 columns of D at +16 KB.
        mma_ts(tmem + kColO + s * 128, tmem + kColS + s * 128 + k * 8,
               sw128_desc(v_base + k * 2048, kChunkBytes, 1024), kIdescO, (first && k == 0) ? 0u : 1u);
      }
      mma_commit(bar(L::bVEmpty + vs));
      mma_commit(bar(L::bPVDone + s));
    }
    __syncwarp();
    return true;
  };

  while (ok && cur.next(p, it)) {
    if (!W.wait(bar(L::bQFull), item & 1, 4)) break;
    tc_fence_after();
    const uint32_t kv0 = kv, ta0 = ta, tb0 = tb;
    // Per-stream ordinal of item-local block jl.
    auto ordinal = [&](int jl) -> uint32_t { return ((jl & 1) ? tb0 : ta0) + (jl >> 1); };
    for (int j = 0; j < it.n; ++j) {
      const int s = j & 1;
      const uint32_t ks = kv % kKStages;
      if (!W.wait(bar(L::bKFull + ks), (kv / kKStages) & 1, 5)) { ok = false; break; }
      tc_fence_after();
      CALIBATT_TRACE_EVENT(lane == 0, 3, kv);
      if (lane == 0) {
        const uint32_t k_base = base + L::kK + ks * L::kTile;
#pragma unroll
        for (int k = 0; k < HD / 16; ++k) {
          // K-major operands: 16 columns = 32 bytes per step inside a 64-column chunk.
          const uint32_t off = (k >> 2) * kChunkBytes + (k & 3) * 32;
          mma_ss(tmem + kColS + s * 128, sw128_desc(base + L::kQ + off, 16, 1024),
                 sw128_desc(k_base + off, 16, 1024), kIdescS, k > 0 ? 1u : 0u);
        }
        mma_commit(bar(L::bKEmpty + ks));
        mma_commit(bar(L::bSFull + s));
        if (j == it.n - 1) mma_commit(bar(L::bQEmpty));
      }
      __syncwarp();
      if (s) ++tb; else ++ta;
      // The previous block belongs to the other stream; its P.V goes next, so
      // each stream's P(j) is consumed before that stream's S(j + 2) is issued.
      if (j >= 1) {
        const int jp = j - 1;
        if (!issue_pv(jp, kv0 + jp, ordinal(jp))) { ok = false; break; }
      }
      ++kv;
    }
    if (!ok) break;
    if (it.n >= 1) {
      const int jp = it.n - 1;
      if (!issue_pv(jp, kv0 + jp, ordinal(jp))) break;
    } else if (lane == 0) {
      mbar_arrive(bar(L::bQEmpty));
    }
    __syncwarp();
    ++item;
  }
  // Every MMA this warp issued must finish before tensor memory is freed.
  if (lane == 0) mma_commit(bar(L::bDrain));
  __syncwarp();
  drain_wait(bar(L::bDrain), 0);
}

// --------------------------------------------------------- softmax/epilogue
// Group s (warps 4s .. 4s+3) runs the softmax of stream s; thread t of the
// group owns query row t.  In the epilogue the two groups exchange (m_s, l_s)
// through shared memory at a pair barrier (warps w and w+4, bar.red.or, which
// also carries "a wait failed" so both warps leave together), then group s
// writes output columns [s*D/2, (s+1)*D/2) of the merged result.
template <int HD, bool ANCHOR>
__device__ void softmax_role(const TcParams& p, uint32_t base, uint8_t* gbase, uint32_t tmem,
                             const Waiter& W, int warp, int lane) {
  using L = Layout<HD>;
  auto bar = [&](int i) { return base + L::kBar + 8u * i; };
  const int quarter = warp & 3, s = warp >> 2;
  const int row = quarter * 32 + lane;  // query row within the tile == TMEM lane
  const int pair_bar = 1 + quarter;     // named barrier shared with the partner warp
  float* xchg = reinterpret_cast<float*>(gbase + L::kXchg);
  const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
  const uint32_t tS = tmem + lane_off + kColS + s * 128;   // this stream's scores / probabilities
  const uint32_t tO0 = tmem + lane_off + kColO;            // O_0 (O_1 at +128)
  const int ragged_cols = p.seq_len % 128;
  const float sl2 = p.scale_log2;
  // Waits until the P.V numbered ts of stream st has completed.
  auto wait_pv = [&](int st, uint32_t ts, int where) -> bool {
    if (!W.wait(bar(L::bPVDone + st), ts & 1, where)) return false;
    tc_fence_after();
    return true;
  };
  Cursor<ANCHOR> cur;
  cur.init(p);
  Item it;
  uint32_t kv = 0, item = 0;
  uint32_t t_me = 0, t_other = 0;  // key blocks of this / the other stream so far (global)
  uint32_t turns = 0;                // turns this stream has waited for
  bool ok = true;
  while (cur.next(p, it)) {
    const int n_s = (it.n + 1 - s) / 2;  // blocks of this stream in the item
    float m_ref = -INFINITY, l = 0.f;
    for (int k = 0; k < n_s; ++k) {
      const int j = 2 * k + s;  // item-local block index
      ok = ok && W.wait(bar(L::bSFull + s), t_me & 1, 10);
      if (ok) tc_fence_after();
      CALIBATT_TRACE_EVENT(lane == 0, 32 + warp, kv + j);
      uint32_t sr[128];
      tmem_ld_x128(tS, sr);
      CALIBATT_TRACE_EVENT(lane == 0, 40 + warp, kv + j);
      float sc[128];
#pragma unroll
      for (int c = 0; c < 128; ++c) sc[c] = __uint_as_float(sr[c]);
      if (j == it.n - 1 && it.ragged_last) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= ragged_cols) sc[c] = -INFINITY;
      }
      // Row maximum: 8 independent three-input max chains.
      float mx8[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) mx8[a] = fmaxf(sc[a], sc[a + 8]);
#pragma unroll
      for (int c = 16; c < 128; c += 16) {
#pragma unroll
        for (int a = 0; a < 8; ++a) mx8[a] = fmax3(mx8[a], sc[c + a], sc[c + a + 8]);
      }
      const float mx_s =
          fmaxf(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(fmax3(mx8[3], mx8[4], mx8[5]), mx8[6], mx8[7])) * sl2;
      // The decision is taken per warp (tcgen05.ld/st are .sync.aligned and
      // need all 32 lanes); rows of a rescaling warp whose maximum did not grow
      // get alpha = 1.  O_s itself is rescaled after the probabilities are
      // written (the scores are no longer live then); it only has to happen
      // before this block's P.V, which waits for p_full.
      const bool rescale = __any_sync(0xFFFFFFFFu, mx_s > m_ref + kRescaleLog2);
      float alpha = 1.f;
      if (rescale) {
        const float m_new = fmaxf(m_ref, mx_s);
        alpha = (m_new == -INFINITY) ? 1.f : fast_exp2(m_ref - m_new);
        l *= alpha;
        m_ref = m_new;
      }
      const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
      // Wait for this block's turn on the MUFU unit: the previous key block
      // (of the other stream, or the last block of the previous item) has
      // finished its exponentials.
      const uint32_t g = kv + j;
      if (kExpTurns && g > 0) {
        ok = ok && W.wait(bar(L::bTurn + s), turns & 1, 14);
        ++turns;
      }
      // Probabilities in four chunks of 32 keys; each chunk's 16 packed
      // columns go to tensor memory (over the already-read scores) at once.
      float la = 0.f, lb = 0.f, lc = 0.f, ld = 0.f;
#pragma unroll
      for (int hh = 0; hh < 4; ++hh) {
        uint32_t pk[16];
#pragma unroll
        for (int cc = 0; cc < 16; ++cc) {
          const int c = hh * 16 + cc;
          float x0, x1;
          fma2(x0, x1, sc[2 * c], sc[2 * c + 1], sl2, sl2, -m_use, -m_use);
          const bool poly = kPolyEvery > 0 && (c % kPolyEvery) == kPolyEvery - 1;
          const float p0 = poly ? exp2_fma(x0) : fast_exp2(x0);
          const float p1 = poly ? exp2_fma(x1) : fast_exp2(x1);
          if (cc & 1) add2(lc, ld, lc, ld, p0, p1); else add2(la, lb, la, lb, p0, p1);
          pk[cc] = pack_bf16x2(p0, p1);
        }
        if (ok) tmem_st_x16(tS + hh * 16, pk);
      }
      l += (la + lb) + (lc + ld);
      // Hand the MUFU unit to the next key block in issue order: the other
      // stream within the item, or stream 0 of the next item.
      if (kExpTurns && ok) mbar_arrive(bar(L::bTurn + ((j + 1 < it.n) ? 1 - s : 0)));
      CALIBATT_TRACE_EVENT(lane == 0, 48 + warp, kv + j);
      if (rescale && k > 0) {
        // O_s is stable once this stream's previous P.V has completed.
        ok = ok && wait_pv(s, t_me - 1, 11);
        if (ok) {
          const uint32_t tOs = tO0 + s * 128;
#pragma unroll 1
          for (int ch = 0; ch < HD / 32; ++ch) {
            uint32_t o[32];
            tmem_ld_x32(tOs + ch * 32, o);
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st_x32(tOs + ch * 32, o);
          }
        }
      }
      if (ok) {
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(L::bPFull + s));
      }
      CALIBATT_TRACE_EVENT(lane == 0, 20 + warp, kv + j);
      ++t_me;
    }
    // The other stream's block count, to track its P.V completions too.
    t_other += (it.n + s) / 2;
    const uint32_t ta = s == 0 ? t_me : t_other, tb = s == 0 ? t_other : t_me;
    kv += it.n;

    // ------------------------------------------------------------ epilogue
    // (A failed wait is acted on at the pair barrier below, which both warps
    // of the pair reach; leaving earlier could strand the partner there.)
    const int n0 = (it.n + 1) / 2, n1 = it.n / 2;
    if (n0 > 0) ok = ok && wait_pv(0, ta - 1, 12);
    if (n1 > 0) ok = ok && wait_pv(1, tb - 1, 12);
    CALIBATT_TRACE_EVENT(lane == 0 && warp == 0, 10, kv);
    // Exchange buffer alternates by item so the partner's read of the
    // previous item's values can never meet this item's writes.
    float* xb = xchg + (item & 1) * 512;
    xb[(s * 2 + 0) * 128 + row] = m_ref;
    xb[(s * 2 + 1) * 128 + row] = l;
    if (bar_red_or(pair_bar, 64, !ok)) { ok = false; break; }
    const float m_o = xb[((1 - s) * 2 + 0) * 128 + row];
    const float l_o = xb[((1 - s) * 2 + 1) * 128 + row];
    const float m0 = s == 0 ? m_ref : m_o, m1 = s == 0 ? m_o : m_ref;
    const float l0 = s == 0 ? l : l_o, l1 = s == 0 ? l_o : l;
    const float m = fmaxf(m0, m1);
    const float a0 = (m0 == -INFINITY) ? 0.f : fast_exp2(m0 - m);
    const float a1 = (m1 == -INFINITY) ? 0.f : fast_exp2(m1 - m);
    const float l_row = l0 * a0 + l1 * a1;
    const float inv_l = l_row > 0.f ? 1.f / l_row : 0.f;
    const float w0 = a0 * inv_l, w1 = a1 * inv_l;
    const int64_t bh_off = static_cast<int64_t>(it.b) * p.sb + static_cast<int64_t>(it.h) * p.sh;
    // Destination rows of this thread's output.
    int64_t dst_token = -1;
    int n_dst = 0, anchor_f = 0, anchor_w = 0, lo = 0;
    if (ANCHOR) {
      const int pq = it.tile * 128 + row;
      if (pq < p.anc.anchor_tokens) {
        const int per_frame = p.anc.n_anchors * p.anc.cols;
        anchor_f = pq / per_frame;
        const int rem = pq % per_frame;
        const int a = rem / p.anc.cols;
        anchor_w = rem % p.anc.cols;
        lo = p.anc.group_lo[a];
        n_dst = p.anc.group_hi[a] - lo + 1;
      }
    } else {
      const int token = it.tile * 128 + row;
      if (token < p.seq_len) {
        dst_token = token;
        n_dst = 1;
      }
    }
#pragma unroll 1
    for (int ch = 0; ch < HD / 64; ++ch) {
      const int col = s * (HD / 2) + ch * 32;  // this group's output columns
      uint32_t o0[32], o1[32];
      if (n0 > 0) {
        tmem_ld_x32(tO0 + col, o0);
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) o0[c] = 0u;
      }
      if (n1 > 0) {
        tmem_ld_x32(tO0 + 128 + col, o1);
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) o1[c] = 0u;
      }
      uint4 pkd[4];
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        float v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
          v[e] = __uint_as_float(o0[8 * g + e]) * w0 + __uint_as_float(o1[8 * g + e]) * w1;
        pkd[g].x = pack_bf16x2(v[0], v[1]);
        pkd[g].y = pack_bf16x2(v[2], v[3]);
        pkd[g].z = pack_bf16x2(v[4], v[5]);
        pkd[g].w = pack_bf16x2(v[6], v[7]);
      }
#pragma unroll 1
      for (int d = 0; d < n_dst; ++d) {
        const int64_t token = ANCHOR
            ? (static_cast<int64_t>(anchor_f) * p.anc.rows + lo + d) * p.anc.cols + anchor_w
            : dst_token;
        uint4* dst = reinterpret_cast<uint4*>(p.o + bh_off + token * p.sn + col);
#pragma unroll
        for (int g = 0; g < 4; ++g) dst[g] = pkd[g];
      }
    }
    if (!ANCHOR && s == 0 && p.lse != nullptr && dst_token >= 0) {
      p.lse[(static_cast<int64_t>(it.b) * p.heads + it.h) * p.seq_len + dst_token] =
          it.n > 0 ? (m + __log2f(l_row)) * 0.69314718055994531f : -INFINITY;
    }
    tc_fence_before();
    mbar_arrive(bar(L::bOFree));
    CALIBATT_TRACE_EVENT(lane == 0 && warp == 0, 11, kv);
    ++item;
  }
}

template <int HD, bool ANCHOR>
__global__ void __launch_bounds__(kThreads, 1) tc_attn_kernel(const __grid_constant__ TcParams p) {
  using L = Layout<HD>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::kMisc + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    auto bar = [&](int i) { return base + L::kBar + 8u * i; };
    mbar_init(bar(L::bQFull), 1);
    mbar_init(bar(L::bQEmpty), 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(bar(L::bKFull + s), 1);
      mbar_init(bar(L::bKEmpty + s), 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(bar(L::bVFull + s), 1);
      mbar_init(bar(L::bVEmpty + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(L::bSFull + s), 1);
      mbar_init(bar(L::bPFull + s), kGroupThreads);
      mbar_init(bar(L::bPVDone + s), 1);
    }
    mbar_init(bar(L::bOFree), kSoftmaxThreads);
    mbar_init(bar(L::bTurn + 0), kGroupThreads);
    mbar_init(bar(L::bTurn + 1), kGroupThreads);
    mbar_init(bar(L::bDrain), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kProducerWarp && lane == 0 && !ANCHOR) {
    prefetch_tensormap(&p.tm_q);
    prefetch_tensormap(&p.tm_k);
  }
  if (warp == kVProducerWarp && lane == 0) prefetch_tensormap(&p.tm_v);
  if (warp == kMmaWarp) {
    tmem_alloc(smem_addr(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Waiter W{abort_flag, p.status, p.timeout_ns};

  if (warp == kProducerWarp) {
    producer_role<HD, ANCHOR, false>(p, base, W, lane);
  } else if (warp == kVProducerWarp) {
    producer_role<HD, ANCHOR, true>(p, base, W, lane);
  } else if (warp == kMmaWarp) {
    mma_role<HD, ANCHOR>(p, base, tmem, W, lane);
  } else {
    softmax_role<HD, ANCHOR>(p, base, gbase, tmem, W, warp, lane);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int HD, bool ANCHOR>
cudaError_t launch_one(const TcParams& p, int grid, cudaStream_t s) {
  auto kern = tc_attn_kernel<HD, ANCHOR>;
  const int bytes = Layout<HD>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, bytes, s>>>(p);
  return cudaGetLastError();
}

__global__ void exp2_fma_kernel(const float* __restrict__ x, float* __restrict__ y, int64_t n) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    y[i] = exp2_fma(x[i]);
}

}  // namespace

#ifdef CALIBATT_TRACE
extern "C" int calibatt_trace_read(unsigned long long* host, int max_records) {
  const int n = static_cast<int>(kTraceEvents * kTraceIters);
  cudaMemcpyFromSymbol(host, g_trace, sizeof(unsigned long long) * (n < max_records ? n : max_records));
  return n;
}
extern "C" void calibatt_trace_reset() {
  cudaMemset(nullptr, 0, 0);
  static unsigned long long zeros[kTraceEvents * kTraceIters];
  cudaMemcpyToSymbol(g_trace, zeros, sizeof(zeros));
}
#endif

cudaError_t launch_exp2_fma(const float* x, float* y, int64_t n, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const int64_t blocks = (n + 255) / 256;
  exp2_fma_kernel<<<static_cast<unsigned>(blocks < 1024 ? blocks : 1024), 256, 0, s>>>(x, y, n);
  return cudaGetLastError();
}

size_t tc_smem_bytes(int head_dim) {
  return head_dim == 64 ? Layout<64>::kBytes : Layout<128>::kBytes;
}

cudaError_t launch_tc_attn(const TcParams& p, int head_dim, bool anchor, int grid, cudaStream_t s) {
  if (head_dim == 128) return anchor ? launch_one<128, true>(p, grid, s) : launch_one<128, false>(p, grid, s);
  if (head_dim == 64) return anchor ? launch_one<64, true>(p, grid, s) : launch_one<64, false>(p, grid, s);
  return cudaErrorInvalidValue;
}

}  // namespace calibatt
