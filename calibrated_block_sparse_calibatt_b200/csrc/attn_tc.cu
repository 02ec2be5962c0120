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
// to stream 0 and odd positions to stream 1, and both streams accumulate into
// ONE output accumulator O in tensor memory.  That works because the
// reference maximum is a single in-order sequence m(0) <= m(1) <= ...: the
// softmax of block j takes m(j-1) from the other stream (published as soon as
// that block's row maximum is known, long before its exponentials end), keeps
// it unless a row maximum exceeds it by more than 2^8 (exp2 domain), and
// publishes m(j).  P(j) = 2^(s*log2e*scale - m(j)) <= 256.  When m grows at
// block j, O is rescaled by 2^(m(j-1) - m(j)) after P(j-1).V has landed and
// before P(j).V is issued (it waits for P(j)), so O always carries the
// reference of the last block accumulated.  Each stream keeps its own row sum
// relative to the reference of its latest block; the epilogue combines the
// two sums against the final reference.
//
// Freeing the second accumulator leaves room for separate score and
// probability buffers per stream: a stream's next S is issued as soon as its
// softmax warps have loaded the current scores into registers, so it finds
// the scores of its next block ready when its current block ends, and the
// tensor core's P.V + S work is off the softmax chain.
//
// CTA layout (384 threads, one CTA per SM, persistent):
//   warps 0-3  softmax of stream 0, warps 4-7 softmax of stream 1: thread t of
//              a group owns query row t (TMEM lane t) and a whole 128-key score
//              row; in the epilogue the two groups split the output columns
//   warp  8    producer of Q (TMA, or a plain-load gather of anchor rows)
//              and of the K tiles gathered by block index
//   warp  9    TMEM allocator; one lane issues the S = Q K^T MMAs
//   warp 10    producer of the V tiles
//   warp 11    one lane issues the O += P V MMAs
// Tensor memory (512 columns): stream s has its f32 scores S_s at 128*s and
// its bf16 probabilities P_s at 256 + 64*s; O is at 384.
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
// Start and end (globaltimer, ns) of every CTA.
__device__ unsigned long long g_cta_span[2 * 1024];
// Per CTA: nanoseconds spent in the epilogue stores of anchor tiles, and the
// number of such tiles (warp 0, lane 0 times its warp's stores).
__device__ unsigned long long g_epi_ns[1024];
__device__ unsigned long long g_epi_items[1024];
// Start (globaltimer, ns) and work-item word of the first kItemTrace items
// of every CTA, recorded by the Q/K producer.
constexpr int kItemTrace = 256;
__device__ unsigned long long g_item_t[1024 * kItemTrace];
__device__ unsigned int g_item_w[1024 * kItemTrace];
#ifndef CALIBATT_TRACE_OFFSET
#define CALIBATT_TRACE_OFFSET 0
#endif
#ifndef CALIBATT_TRACE_CTA
#define CALIBATT_TRACE_CTA 0
#endif
__device__ __forceinline__ void trace_event(int ev, uint32_t idx) {
  idx -= CALIBATT_TRACE_OFFSET;
  if (blockIdx.x == CALIBATT_TRACE_CTA && idx < kTraceIters) g_trace[ev * kTraceIters + idx] = clock64();
}
#define CALIBATT_TRACE_EVENT(cond, ev, idx) \
  do {                                     \
    if (cond) trace_event(ev, idx);        \
  } while (0)
// Stores from the MMA-issuing thread delay its next tcgen05.mma, so its
// events are recorded only on request.
#ifdef CALIBATT_TRACE_MMA
constexpr bool kTraceMma = true;
#else
constexpr bool kTraceMma = false;
#endif
#else
#define CALIBATT_TRACE_EVENT(cond, ev, idx) \
  do {                                     \
  } while (0)
#endif

// Three full warpgroups so registers can be moved between them (setmaxnreg
// acts per warpgroup): two softmax groups and one for the producers, the MMA
// issuer and a spare warp.  At launch every thread has kLaunchRegs; the
// softmax groups then raise theirs to kSoftmaxRegs and the third group drops
// to kOtherRegs, keeping 128 * (2 * kSoftmaxRegs + kOtherRegs) within the
// 384 * kLaunchRegs the CTA was launched with.
constexpr int kThreads = 384;       // 8 softmax warps, Q/K producer, MMA, V producer, spare
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 232;
constexpr int kOtherRegs = 40;
static_assert(128 * (2 * kSoftmaxRegs + kOtherRegs) <= kThreads * kLaunchRegs, "register split");
constexpr int kEndBarrier = 5;      // named barrier id (1-4: softmax warp pairs)
constexpr int kProducerWarp = 8;    // Q and K tiles
constexpr int kMmaWarp = 9;         // TMEM allocator, issues S = Q K^T
constexpr int kPvWarp = 11;         // issues O += P V
constexpr int kVProducerWarp = 10;  // V tiles
constexpr int kGroupThreads = 128;  // softmax threads per stream
constexpr int kSoftmaxThreads = 256;
#ifndef CALIBATT_K_STAGES
#define CALIBATT_K_STAGES 3
#endif
#ifndef CALIBATT_V_STAGES
#define CALIBATT_V_STAGES 2
#endif
constexpr int kKStages = CALIBATT_K_STAGES;
constexpr int kVStages = CALIBATT_V_STAGES;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;    // stream s's f32 scores at kColS + 128 * s
constexpr uint32_t kColP = 256;  // stream s's bf16 probabilities at kColP + 64 * s
constexpr uint32_t kColO = 384;  // the output accumulator O
constexpr float kRescaleLog2 = 8.0f;
// One pair in kPolyEvery of exponentials runs on the FMA pipe (exp2_fma2)
// instead of the MUFU unit (0 = all on MUFU; measured fastest on B200).
#ifndef CALIBATT_POLY_EVERY
#define CALIBATT_POLY_EVERY 0
#endif
constexpr int kPolyEvery = CALIBATT_POLY_EVERY;
// The offline energy passes (LSE and energy modes) have half the tensor work
// of attention per key block but the same 16,384 exponentials, so the MUFU
// unit is their busiest pipe while the FMA pipe idles: one pair in
// kEnergyPolyEvery runs on the FMA pipe with the quintic (as accurate as
// ex2.approx).  Measured on the 720p energy call under the power cap: 1/4 of
// the pairs is 2% faster than none, 1/3 and 1/2 are 6% and 12% slower (the
// polynomial spends more energy per result than the MUFU).
#ifndef CALIBATT_ENERGY_POLY_EVERY
#define CALIBATT_ENERGY_POLY_EVERY 4
#endif
constexpr int kEnergyPolyEvery = CALIBATT_ENERGY_POLY_EVERY;

constexpr int kChunkBytes = 128 * 128;  // 128 rows x 64 bf16 (one 128-byte swizzle span)
// Dynamic assignment: the Q/K producer takes each ticket and hands it to the
// other eleven warps through a ring of kItemRing slots in shared memory.
constexpr int kItemRing = 4;
constexpr int kItemReaders = 11;  // softmax warps 0-7, S issuer, V producer, P.V issuer

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
  static constexpr int bSFree = bSFull + 2;          // [2] stream s has read its scores
  static constexpr int bPFull = bSFree + 2;          // [2] probabilities of stream s ready
  static constexpr int bPFree = bPFull + 2;          // [2] P.V of stream s's block finished
  static constexpr int bOFull = bPFree + 2;          // every P.V of the item finished
  static constexpr int bOFree = bOFull + 1;          // epilogue has read O
  static constexpr int bDrain = bOFree + 1;
  static constexpr int bItemFull = bDrain + 1;              // [kItemRing] ticket published
  static constexpr int bItemEmpty = bItemFull + kItemRing;  // [kItemRing] every other role has read it
  static constexpr int kNumBars = bItemEmpty + kItemRing;
  static constexpr int kMisc = kBar + kNumBars * 8;  // u32 tmem base, i32 abort flag, u32 tickets [kItemRing]
  static constexpr int kRing = kMisc + 8;
  static constexpr int kXchg = kMisc + 8 + 4 * kItemRing;  // float [2 item parity][2 streams][2 (m, l)][128 rows]
  // {m bits, stream ordinal + 1} [2 streams][128 rows], 8-byte slots
  static constexpr int kMSlot = kXchg + 2 * 2 * 2 * 128 * 4;
  // uint16 lists of kept key blocks decoded from bitmap rows, one per producer
  static constexpr int kListBytes = kMaxBitmapBlocks * 2;
  static constexpr int kList = kMSlot + 2 * 128 * 8;
  // per softmax warp: 8 output rows' halves (HD bytes each) staged for the
  // anchor broadcast
  static constexpr int kStageRowBytes = HD;
  static constexpr int kStageBytes = 8 * kStageRowBytes;
  static constexpr int kStage = (kList + 2 * kListBytes + 127) & ~127;
  static constexpr int kUsed = kStage + 8 * kStageBytes;
  // +1024 for aligning the base; at least 120 KB so only one CTA fits per SM
  // (each CTA holds all 512 tensor-memory columns).
  static constexpr int kBytes = (kUsed + 1024) > 120 * 1024 ? (kUsed + 1024) : 120 * 1024;
};

// Modes without V and P.V: the offline calibration passes.
__host__ __device__ constexpr bool calibration_mode(int mode) {
  return mode == kModeLse || mode == kModeEnergy || mode == kModeSimilarity;
}

// Token whose query partners token `i` in the spatial-similarity mode: the
// same frame and column in the nearest anchor row (Key Designs 3); the anchor
// geometry's groups hold each anchor's rows.
__device__ __forceinline__ int64_t partner_token(const AnchorGeom& g, int64_t i) {
  const int64_t per_frame = static_cast<int64_t>(g.rows) * g.cols;
  const int64_t f = i / per_frame;
  const int rem = static_cast<int>(i - f * per_frame);
  const int rho = rem / g.cols, w = rem - rho * g.cols;
  int a = 0;
  for (int x = 1; x < g.n_anchors; ++x)
    if (rho >= g.group_lo[x]) a = x;
  return (f * g.rows + g.anchor_row[a]) * g.cols + w;
}

struct Item {
  int b, h, tile;            // batch, head, query block (sparse) or anchor tile
  int n;                     // key blocks to visit
  const uint16_t* cols;      // retained key blocks (index lists), nullptr = bitmap row or 0..n-1
  bool ragged_last;          // last visited key block is the partial one
  bool anchor;               // anchor-row tile (gathered queries, broadcast epilogue)
  int part;                  // key-range part of a split anchor tile: slot * 4 + part; -1 = whole
};

// Key-block indices 0, 1, ..., 65535, built at compile time: a key-range part
// of a split anchor tile visits blocks k0 .. k1 - 1 as the list starting at
// entry k0, so the producers walk it like any retained-block list.
struct KeyIdentity {
  uint16_t v[65536];
  constexpr KeyIdentity() : v() {
    for (int i = 0; i < 65536; ++i) v[i] = static_cast<uint16_t>(i);
  }
};
__device__ const KeyIdentity g_key_identity;


// Row (head h, query block r) of a bitmap dictionary layer.
__device__ __forceinline__ const uint32_t* bitmap_row(const TcParams& p, int h, int r) {
  return p.sched.bitmap + (static_cast<int64_t>(h) * p.sched.nq + r) * p.sched.words;
}

// Walks this CTA's work items in the same order in every role.
template <int HD, int MODE>
struct Cursor {
  int b, idx, begin, end, step;
  uint32_t ring = 0;  // dynamic assignment: shared-memory base of the ring
  uint32_t seq = 0;   // tickets taken from the ring so far
  bool fetcher = false;
  __device__ bool dynamic(const TcParams& p) const {
    return (MODE == kModeSparse || MODE == kModeFused) && p.sched.ticket != nullptr;
  }
  // base: the CTA's 1024-aligned shared-memory base; is_fetcher: this warp
  // takes the tickets (the Q/K producer) and the others read them.
  __device__ void init(const TcParams& p, uint32_t base, bool is_fetcher) {
    ring = base;
    fetcher = is_fetcher;
    b = 0;
    if (MODE == kModeAnchor) {
      // one item sequence over batch x heads x tiles, the split parts last
      begin = blockIdx.x;
      end = p.split.first + (p.split.n_tiles - p.split.first) * p.split.parts;
      step = gridDim.x;
    } else if (calibration_mode(MODE)) {
      begin = blockIdx.x;
      end = p.heads * p.nb;
      step = gridDim.x;
    } else {
      begin = dynamic(p) ? 0 : p.sched.cta_ptr[blockIdx.x];
      end = dynamic(p) ? 0 : p.sched.cta_ptr[blockIdx.x + 1];
      step = 1;
    }
    idx = begin;
  }
  // Dynamic assignment: the next ticket, through the ring.  The fetcher waits
  // until all readers are done with the slot's previous ticket, takes a ticket
  // (atomicAdd) and publishes it; a reader waits for the slot, reads it and
  // frees it.  Returns false past the last ticket or when a wait gives up.
  __device__ bool take_ticket(const TcParams& p, const Waiter& W, uint32_t& t) {
    using L = Layout<HD>;
    const int lane = threadIdx.x & 31;
    const uint32_t slot = seq % kItemRing, use = seq / kItemRing;
    const uint32_t full = ring + L::kBar + 8u * (L::bItemFull + slot);
    const uint32_t empty = ring + L::kBar + 8u * (L::bItemEmpty + slot);
    const uint32_t cell = ring + L::kRing + 4u * slot;
    t = 0;
    if (fetcher) {
      if (use > 0 && !W.wait(empty, (use - 1) & 1, 16)) return false;
      if (lane == 0) {
        t = atomicAdd(p.sched.ticket, 1u);
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(cell), "r"(t) : "memory");
        mbar_arrive(full);
      }
      t = __shfl_sync(0xFFFFFFFFu, t, 0);
    } else {
      if (!W.wait(full, use & 1, 17)) return false;
      asm volatile("ld.shared.u32 %0, [%1];" : "=r"(t) : "r"(cell) : "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(empty);
    }
    ++seq;
    return t < static_cast<uint32_t>(p.batch) * static_cast<uint32_t>(p.sched.n_order);
  }
  __device__ bool next(const TcParams& p, Item& it, const Waiter& W) {
    if (MODE == kModeAnchor) {
      if (idx >= end) return false;
      int t = idx, part = -1, slot = 0;
      if (idx >= p.split.first) {
        slot = (idx - p.split.first) / p.split.parts;
        part = (idx - p.split.first) % p.split.parts;
        t = p.split.first + slot;
      }
      const int per_b = p.anc.n_heads * p.anc.tiles_per_head;
      it.b = t / per_b;
      const int r = t % per_b;
      it.h = p.anc.head_ids[r / p.anc.tiles_per_head];
      it.tile = r % p.anc.tiles_per_head;
      it.anchor = true;
      if (part < 0) {
        it.n = p.nb;
        it.cols = nullptr;
        it.ragged_last = (p.seq_len % 128) != 0;
        it.part = -1;
      } else {
        const int k0 = p.nb * part / p.split.parts, k1 = p.nb * (part + 1) / p.split.parts;
        it.n = k1 - k0;
        it.cols = g_key_identity.v + k0;
        it.ragged_last = k1 == p.nb && (p.seq_len % 128) != 0;
        it.part = slot * 4 + part;
      }
      idx += step;
      return true;
    }
    it.part = -1;
    while (b < p.batch) {
      uint32_t t_dyn = 0;
      const bool dyn = dynamic(p);
      if (dyn) {
        if (!take_ticket(p, W, t_dyn)) return false;
        b = static_cast<int>(t_dyn / static_cast<uint32_t>(p.sched.n_order));
        idx = static_cast<int>(t_dyn % static_cast<uint32_t>(p.sched.n_order));
      }
      if (dyn || idx < end) {
        it.b = b;
        uint32_t w = 0;
        if (calibration_mode(MODE)) {
          // every key block of query block (idx mod nb) of head (idx / nb)
          it.anchor = false;
          it.h = idx / p.nb;
          it.tile = idx % p.nb;
          it.n = p.nb;
          it.cols = nullptr;
          it.ragged_last = (p.seq_len % 128) != 0;
          idx += step;
          return true;
        }
        w = dyn ? p.sched.order[idx] : p.sched.items[idx];
        if (MODE == kModeFused && (w & kItemAnchorBit)) {
          it.anchor = true;
          it.h = static_cast<int>((w >> 16) & 0x7FFFu);
          it.tile = static_cast<int>(w & 0xFFFFu);
          it.n = p.nb;
          it.cols = nullptr;
          it.ragged_last = (p.seq_len % 128) != 0;
        } else {
          it.anchor = false;
          it.h = static_cast<int>(MODE == kModeFused ? (w >> 16) & 0x7FFFu : w >> 16);
          it.tile = static_cast<int>(w & 0xFFFFu);
          if (p.sched.bitmap != nullptr) {
            const uint32_t* bm = bitmap_row(p, it.h, it.tile);
            // every role calls next() with its whole warp: lane x counts word x
            const int lane = threadIdx.x & 31;
            int cnt = 0;
            for (int w0 = 0; w0 < p.sched.words; w0 += 32) {
              const int x = w0 + lane;
              cnt += __reduce_add_sync(0xFFFFFFFFu, x < p.sched.words ? __popc(bm[x]) : 0);
            }
            it.n = cnt;
            it.cols = nullptr;
            const int last = p.nb - 1;
            it.ragged_last = cnt > 0 && (p.seq_len % 128) != 0 && ((bm[last >> 5] >> (last & 31)) & 1u);
          } else {
            const int32_t* rp = p.sched.row_ptr + static_cast<int64_t>(it.h) * (p.sched.nq + 1);
            const int s0 = rp[it.tile];
            it.n = rp[it.tile + 1] - s0;
            if (p.sched.runs == nullptr) {
              it.cols = p.sched.col + p.sched.col_base[it.h] + s0;
              it.ragged_last = it.n > 0 && (p.seq_len % 128) != 0 && it.cols[it.n - 1] == p.nb - 1;
            } else {
              // interval row: the producers decode its runs, and only the
              // softmax warps need the last block (a flag in run_ptr)
              it.cols = nullptr;
              it.ragged_last = false;
            }
          }
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
template <int HD, int MODE, bool V>
__device__ void producer_role(const TcParams& p, uint32_t base, uint8_t* gbase, const Waiter& W, int lane) {
  using L = Layout<HD>;
  auto bar = [&](int i) { return base + L::kBar + 8u * i; };
  constexpr int kStages = V ? kVStages : kKStages;
  constexpr int kFull = V ? L::bVFull : L::bKFull;
  constexpr int kEmpty = V ? L::bVEmpty : L::bKEmpty;
  constexpr int kRing = V ? L::kV : L::kK;
  const CUtensorMap* map = V ? &p.tm_v : &p.tm_k;
  if (V && calibration_mode(MODE)) return;  // no P.V in the calibration modes
  Cursor<HD, MODE> cur;
  cur.init(p, base, !V);  // the Q/K producer takes the tickets
  Item it;
  uint32_t kv = 0, item = 0, issued = 0, q_items = 0;
  bool ok = true;
  while (ok && cur.next(p, it, W)) {
    // The row's list first (bitmap and interval rows are expanded into this
    // producer's shared-memory list), so that the Q/K producer does it while
    // the previous item's last score MMAs still hold the Q buffer.
    const uint16_t* cols = it.cols;
    if (p.sched.bitmap != nullptr && !it.anchor) {
      // Bitmap row -> this producer's list of kept key blocks, ascending:
      // lane x takes word x of each 32-word stretch, a prefix sum of the
      // words' bit counts places its indices.
      uint16_t* list = reinterpret_cast<uint16_t*>(gbase + L::kList + (V ? 1 : 0) * L::kListBytes);
      int offset = 0;
      for (int w0 = 0; w0 < p.sched.words; w0 += 32) {
        const int x = w0 + lane;
        uint32_t word = x < p.sched.words ? bitmap_row(p, it.h, it.tile)[x] : 0u;
        const int c = __popc(word);
        int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
          if (lane >= o) incl += t;
        }
        int pos = offset + incl - c;
        while (word) {
          list[pos++] = static_cast<uint16_t>(x * 32 + __ffs(word) - 1);
          word &= word - 1u;
        }
        offset += __shfl_sync(0xFFFFFFFFu, incl, 31);
      }
      __syncwarp();
      cols = list;
    } else if (p.sched.runs != nullptr && !it.anchor) {
      // Interval row -> this producer's list of kept key blocks: runs are
      // read 32 at a time, one per lane, then the warp writes each run's
      // blocks lane-parallel in order.
      uint16_t* list = reinterpret_cast<uint16_t*>(gbase + L::kList + (V ? 1 : 0) * L::kListBytes);
      const int64_t ro = static_cast<int64_t>(it.h) * (p.sched.nq + 1) + it.tile;
      const int r0 = p.sched.run_ptr[ro] & 0x7FFFFFFF, n_runs = (p.sched.run_ptr[ro + 1] & 0x7FFFFFFF) - r0;
      const uint32_t* runs = p.sched.runs + p.sched.col_base[it.h] + r0;
      int pos = 0;
      for (int x0 = 0; x0 < n_runs; x0 += 32) {
        const uint32_t mine = x0 + lane < n_runs ? runs[x0 + lane] : 0u;
        const int cnt = min(32, n_runs - x0);
        for (int x = 0; x < cnt; ++x) {
          const uint32_t run = __shfl_sync(0xFFFFFFFFu, mine, x);
          const int start = static_cast<int>(run & 0xFFFFu), len = static_cast<int>(run >> 16);
          for (int i = lane; i < len; i += 32) list[pos + i] = static_cast<uint16_t>(start + i);
          pos += len;
        }
      }
      __syncwarp();
      cols = list;
    }
    if (!V) {
      if (item > 0 && !W.wait(bar(L::bQEmpty), (item - 1) & 1, 1)) break;
      CALIBATT_TRACE_EVENT(kTraceMma && lane == 0, 9, item + CALIBATT_TRACE_OFFSET);
#ifdef CALIBATT_TRACE
      if (lane == 0 && blockIdx.x < 1024 && item < static_cast<uint32_t>(kItemTrace)) {
        g_item_t[blockIdx.x * kItemTrace + item] = globaltimer();
        g_item_w[blockIdx.x * kItemTrace + item] =
            (it.anchor ? 0x80000000u : 0u) | (static_cast<uint32_t>(it.h) << 16) | static_cast<uint32_t>(it.tile);
      }
#endif
      if (it.anchor) {
        // Gather this tile's 128 anchor-row queries into the 128-byte swizzled
        // K-major layout the MMA expects (16-byte unit u of row r lands at
        // chunk u/8, row r, position (u%8) ^ (r%8)).
        // Every copy is an asynchronous 16-byte global -> shared copy, all of
        // them in flight at once (no registers hold the data; the producer
        // warpgroup has 40 per thread); queries past the anchor tokens are
        // zero-filled.
        constexpr int kUnits = HD / 8;
        const int per_frame = p.anc.n_anchors * p.anc.cols;
        const uint16_t* qb = p.q + static_cast<int64_t>(it.b) * p.sb + static_cast<int64_t>(it.h) * p.sh;
        for (int idx = lane; idx < 128 * kUnits; idx += 32) {
          const int r = idx / kUnits, u = idx % kUnits;
          const int pq = it.tile * 128 + r;
          const uint16_t* src = qb;
          uint32_t bytes = 0;
          if (pq < p.anc.anchor_tokens) {
            const int f = pq / per_frame, rem = pq % per_frame;
            const int a = rem / p.anc.cols, w = rem % p.anc.cols;
            const int64_t token = (static_cast<int64_t>(f) * p.anc.rows + p.anc.anchor_row[a]) * p.anc.cols + w;
            src = qb + token * p.sn + u * 8;
            bytes = 16;
          }
          cp_async_16(base + L::kQ + (u >> 3) * kChunkBytes + r * 128 + (((u & 7) ^ (r & 7)) << 4), src, bytes);
        }
        cp_async_wait_all();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::bQFull));
      } else {
        if (MODE == kModeSimilarity) {
          // The partner queries (nearest anchor row, same frame and column) of
          // the tile's 128 queries, gathered into the swizzled layout in the
          // V ring's space (no V in this mode), before the tile's own Q is
          // requested: q_full then completes only after both are in place.
          constexpr int kUnits = HD / 8;
          const uint16_t* qb = p.q + static_cast<int64_t>(it.b) * p.sb + static_cast<int64_t>(it.h) * p.sh;
          for (int idx = lane; idx < 128 * kUnits; idx += 32) {
            const int r = idx / kUnits, u = idx % kUnits;
            const int64_t tok = static_cast<int64_t>(it.tile) * 128 + r;
            const bool in = tok < p.seq_len;
            cp_async_16(base + L::kV + (u >> 3) * kChunkBytes + r * 128 + (((u & 7) ^ (r & 7)) << 4),
                        in ? qb + partner_token(p.anc, tok) * p.sn + u * 8 : qb, in ? 16u : 0u);
          }
          cp_async_wait_all();
          fence_proxy_async_smem();
          __syncwarp();
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(bar(L::bQFull), L::kTile);
          tma_tile<HD>(base + L::kQ, &p.tm_q, bar(L::bQFull), p, it.tile * 128, it.h, it.b);
        }
      }
      ++q_items;  // every item completes one phase of q_full, whichever way its Q came
    }
    uint32_t my_col = 0;
    for (int j = 0; j < it.n; ++j) {
      if ((j & 31) == 0) {
        const int jj = j + lane;
        my_col = cols == nullptr ? static_cast<uint32_t>(jj) : (jj < it.n ? cols[jj] : 0u);
      }
      const int c = static_cast<int>(__shfl_sync(0xFFFFFFFFu, my_col, j & 31));
      const uint32_t slot = kv % kStages, use = kv / kStages;
      if (use > 0 && !W.wait(bar(kEmpty + slot), (use - 1) & 1, V ? 3 : 2)) { ok = false; break; }
      if (lane == 0) {
        mbar_arrive_expect_tx(bar(kFull + slot), L::kTile);
        tma_tile<HD>(base + kRing + slot * L::kTile, map, bar(kFull + slot), p, c * 128, it.h, it.b);
      }
      CALIBATT_TRACE_EVENT(kTraceMma && lane == 0, V ? 2 : 1, kv);
      ++issued;
      ++kv;
    }
    ++item;
  }
  // Let every bulk copy this warp issued land before the CTA can exit.
  for (uint32_t s = 0; s < static_cast<uint32_t>(kStages); ++s)
    if (issued > s) drain_wait(bar(kFull + s), ((issued - 1 - s) / kStages) & 1);
  // Only the last item's Q copy can still be in flight (each earlier one was
  // consumed before the next Q load): wait for that phase of q_full.
  if (q_items > 0) drain_wait(bar(L::bQFull), (q_items - 1) & 1);
}


// -------------------------------------------------------------------- MMA
// Two issuing threads share the tensor core: warp 9 issues every S(j) and
// warp 11 every O += P(j) V_j.  A wait on an mbarrier by the issuing thread
// leaves the tensor core idle once its queue drains, so with one issuer every
// wait is a bubble; with two, one thread's MMAs run while the other waits.
// Block j belongs to stream j mod 2 of its item; t is its ordinal within
// that stream over the whole launch, and the barriers of stream s count
// those ordinals.
template <int HD, int MODE>
__device__ void mma_s_role(const TcParams& p, uint32_t base, uint32_t tmem, const Waiter& W, int lane) {
  using L = Layout<HD>;
  auto bar = [&](int i) { return base + L::kBar + 8u * i; };
  constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, 0);
  Cursor<HD, MODE> cur;
  cur.init(p, base, false);
  Item it;
  uint32_t g = 0, item = 0;      // global key-block iteration, item counter
  uint32_t t0 = 0, t1 = 0;       // blocks issued per stream
  bool ok = true;
  while (ok && cur.next(p, it, W)) {
    if (!W.wait(bar(L::bQFull), item & 1, 4)) break;
    tc_fence_after();
    CALIBATT_TRACE_EVENT(kTraceMma && lane == 0, 8, item + CALIBATT_TRACE_OFFSET);
    for (int j = 0; j < it.n; ++j, ++g) {
      const int s = j & 1;
      const uint32_t t = s ? t1++ : t0++;
      const uint32_t ks = g % kKStages;
      // The stream's previous scores must be in its softmax warps' registers.
      CALIBATT_TRACE_EVENT(kTraceMma && lane == 0, 6, g);
      if (t > 0 && !W.wait(bar(L::bSFree + s), (t - 1) & 1, 6)) { ok = false; break; }
      CALIBATT_TRACE_EVENT(kTraceMma && lane == 0, 7, g);
      if (!W.wait(bar(L::bKFull + ks), (g / kKStages) & 1, 5)) { ok = false; break; }
      tc_fence_after();
      CALIBATT_TRACE_EVENT(kTraceMma && lane == 0, 3, g);
      if (lane == 0) {
        const uint32_t k_base = base + L::kK + ks * L::kTile;
        // similarity mode: stream s has its two score tiles at 256 s and 256 s + 128
        const uint32_t d = tmem + kColS + s * (MODE == kModeSimilarity ? 256 : 128);
#pragma unroll
        for (int k = 0; k < HD / 16; ++k) {
          // K-major operands: 16 columns = 32 bytes per step inside a 64-column chunk.
          const uint32_t off = (k >> 2) * kChunkBytes + (k & 3) * 32;
          mma_ss(d, sw128_desc(base + L::kQ + off, 16, 1024), sw128_desc(k_base + off, 16, 1024), kIdescS,
                 k > 0 ? 1u : 0u);
        }
        if (MODE == kModeSimilarity) {
#pragma unroll
          for (int k = 0; k < HD / 16; ++k) {
            const uint32_t off = (k >> 2) * kChunkBytes + (k & 3) * 32;
            mma_ss(d + 128, sw128_desc(base + L::kV + off, 16, 1024), sw128_desc(k_base + off, 16, 1024), kIdescS,
                   k > 0 ? 1u : 0u);
          }
        }
        mma_commit(bar(L::bKEmpty + ks));
        mma_commit(bar(L::bSFull + s));
        if (j == it.n - 1) mma_commit(bar(L::bQEmpty));
      }
      __syncwarp();
    }
    if (!ok) break;
    if (it.n == 0 && lane == 0) mbar_arrive(bar(L::bQEmpty));
    __syncwarp();
    ++item;
  }
  // Every MMA this thread issued must finish before tensor memory is freed.
  if (lane == 0) mma_commit(bar(L::bDrain));
  __syncwarp();
  drain_wait(bar(L::bDrain), 0);
}

template <int HD, int MODE>
__device__ void mma_pv_role(const TcParams& p, uint32_t base, uint32_t tmem, const Waiter& W, int lane) {
  using L = Layout<HD>;
  auto bar = [&](int i) { return base + L::kBar + 8u * i; };
  constexpr uint32_t kIdescO = idesc_bf16_f32(128, HD, 1);
  if (calibration_mode(MODE)) {
    // No P.V: only this thread's share of the drain barrier.
    if (lane == 0) mma_commit(bar(L::bDrain));
    __syncwarp();
    return;
  }
  Cursor<HD, MODE> cur;
  cur.init(p, base, false);
  Item it;
  uint32_t g = 0, item = 0;
  uint32_t t0 = 0, t1 = 0;
  bool ok = true;
  while (ok && cur.next(p, it, W)) {
    // The epilogue of the previous item has read O (waited for every item,
    // empty ones included, so each phase of o_free is consumed in order).
    if (item > 0 && !W.wait(bar(L::bOFree), (item - 1) & 1, 9)) break;
    for (int j = 0; j < it.n; ++j, ++g) {
      const int s = j & 1;
      const uint32_t t = s ? t1++ : t0++;
      const uint32_t vs = g % kVStages;
      if (!W.wait(bar(L::bVFull + vs), (g / kVStages) & 1, 7)) { ok = false; break; }
      if (!W.wait(bar(L::bPFull + s), t & 1, 8)) { ok = false; break; }
      tc_fence_after();
      if (lane == 0) {
        const uint32_t v_base = base + L::kV + vs * L::kTile;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          // A = P in tensor memory (16 keys = 8 columns per step); B = V
          // (MN-major): 16 keys per step = 2048 bytes; next 64 columns of D at +16 KB.
          mma_ts(tmem + kColO, tmem + kColP + s * 64 + k * 8,
                 sw128_desc(v_base + k * 2048, kChunkBytes, 1024), kIdescO, (j == 0 && k == 0) ? 0u : 1u);
        }
        mma_commit(bar(L::bVEmpty + vs));
        mma_commit(bar(L::bPFree + s));
        if (j == it.n - 1) mma_commit(bar(L::bOFull));
      }
      __syncwarp();
    }
    if (!ok) break;
    if (it.n == 0 && lane == 0) mbar_arrive(bar(L::bOFull));
    __syncwarp();
    ++item;
  }
  if (lane == 0) mma_commit(bar(L::bDrain));
  __syncwarp();
  drain_wait(bar(L::bDrain), 0);
}

// --------------------------------------------------------- softmax/epilogue
// Group s (warps 4s .. 4s+3) runs the softmax of stream s; thread t of the
// group owns query row t.  In the epilogue the two groups exchange (m_s, l_s)
// through shared memory at a pair barrier (warps w and w+4, bar.red.or, which
// also carries "a wait failed" so both warps leave together), then group s
// writes output columns [s*D/2, (s+1)*D/2) of O / l.
template <int HD, int MODE>
__device__ void softmax_role(const TcParams& p, uint32_t base, uint8_t* gbase, uint32_t tmem,
                             const Waiter& W, int warp, int lane) {
  using L = Layout<HD>;
  auto bar = [&](int i) { return base + L::kBar + 8u * i; };
  const int quarter = warp & 3, s = warp >> 2;
  const int row = quarter * 32 + lane;  // query row within the tile == TMEM lane
  const int pair_bar = 1 + quarter;     // named barrier shared with the partner warp
  float* xchg = reinterpret_cast<float*>(gbase + L::kXchg);
  // Row `row`'s reference maximum is handed between the two threads that own
  // the row (one per stream) through an 8-byte slot {m, ordinal + 1} written
  // in one store; the reader spins (bounded) until the ordinal it needs shows.
  const uint32_t my_slot = smem_addr(gbase + L::kMSlot) + (s * 128 + row) * 8;
  const uint32_t other_slot = smem_addr(gbase + L::kMSlot) + ((1 - s) * 128 + row) * 8;
  const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
  const uint32_t tS = tmem + lane_off + kColS + s * 128;  // this stream's scores
  const uint32_t tP = tmem + lane_off + kColP + s * 64;   // and probabilities
  const uint32_t tO = tmem + lane_off + kColO;
  const int ragged_cols = p.seq_len % 128;
  const float sl2 = p.scale_log2;
  Cursor<HD, MODE> cur;
  cur.init(p, base, false);
  Item it;
  uint32_t kv = 0, item = 0;
  uint32_t t_me = 0, t_other = 0;  // key blocks of this / the other stream so far (global)
  bool ok = true;
  while (cur.next(p, it, W)) {
    // Interval rows: bit 31 of the row's end entry in run_ptr says that the
    // row keeps the last key block.  Loaded here, used only at the last block.
    const int32_t run_end =
        (p.sched.runs != nullptr && !it.anchor) ? p.sched.run_ptr[static_cast<int64_t>(it.h) * (p.sched.nq + 1) + it.tile + 1] : 0;
    const int n_s = (it.n + 1 - s) / 2;  // blocks of this stream in the item
    const uint32_t t_other0 = t_other;
    float m_own = -INFINITY, l = 0.f;    // this stream's row sum, relative to m_own
    for (int k = 0; k < n_s; ++k) {
      const int j = 2 * k + s;  // item-local block index
      [[maybe_unused]] const uint32_t g = kv + j;
      ok = ok && W.wait(bar(L::bSFull + s), t_me & 1, 10);
      if (ok) tc_fence_after();
      CALIBATT_TRACE_EVENT(lane == 0 && quarter == 0, 32 + warp, g);
      uint32_t sr[128];
      tmem_ld_x128(tS, sr);
      // The scores are in registers: the next S of this stream may overwrite them.
      tc_fence_before();
      if (ok) mbar_arrive(bar(L::bSFree + s));
      CALIBATT_TRACE_EVENT(lane == 0 && quarter == 0, 40 + warp, g);
      float sc[128];
#pragma unroll
      for (int c = 0; c < 128; ++c) sc[c] = __uint_as_float(sr[c]);
      if (j == it.n - 1 && (it.ragged_last || (run_end < 0 && ragged_cols != 0))) {
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
      // m(j - 1), published by the partner warp of the other stream (same
      // rows; block j - 1 is that stream's block number t_other0 + (j - 1) / 2
      // in global order).  The partner cannot publish again before it has
      // read m(j), so the barrier is never two phases ahead of this wait.
      CALIBATT_TRACE_EVENT(lane == 0 && quarter == 0, 12 + s, g);
      float m_prev = -INFINITY;
      if (j > 0) {
        const uint32_t prev_ord = t_other0 + static_cast<uint32_t>(j - 1) / 2;
        ok = ok && W.spin_slot(other_slot, prev_ord + 1u, 13, m_prev);
      }
      CALIBATT_TRACE_EVENT(lane == 0 && quarter == 0, 14 + s, g);
      const bool rescale = __any_sync(0xFFFFFFFFu, mx_s > m_prev + kRescaleLog2);
      const float m_j = rescale ? fmaxf(m_prev, mx_s) : m_prev;
      st_shared_v2(my_slot, __float_as_uint(m_j), t_me + 1u);
      if (m_j != m_own) {
        l = (m_own == -INFINITY) ? 0.f : l * fast_exp2(m_own - m_j);
        m_own = m_j;
      }
      const float m_use = (m_j == -INFINITY) ? 0.f : m_j;
      CALIBATT_TRACE_EVENT(lane == 0 && quarter == 0, 16 + s, g);
      if (t_me > 0) {
        // P of this stream's previous block must have been consumed by its P.V.
        ok = ok && W.wait(bar(L::bPFree + s), (t_me - 1) & 1, 14);
        if (ok) tc_fence_after();
      }
      CALIBATT_TRACE_EVENT(lane == 0 && quarter == 0, 56 + warp, g);
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
          float p0, p1;
          if (kPolyEvery > 0 && (c % kPolyEvery) == kPolyEvery - 1) {
            exp2_fma2(p0, p1, x0, x1);
          } else {
            p0 = fast_exp2(x0);
            p1 = fast_exp2(x1);
          }
          if (cc & 1) add2(lc, ld, lc, ld, p0, p1); else add2(la, lb, la, lb, p0, p1);
          pk[cc] = pack_bf16x2(p0, p1);
        }
        if (ok) tmem_st_x16(tP + hh * 16, pk);
      }
      l += (la + lb) + (lc + ld);
      CALIBATT_TRACE_EVENT(lane == 0 && quarter == 0, 48 + warp, g);
      if (rescale && j > 0) {
        // O carries m(j - 1) once P(j - 1).V has completed; P(j).V waits for
        // p_full below, so nothing else touches these rows of O meanwhile.
        // (The other stream's previous P.V, block j - 3, completed before
        // this stream's P.V of block j - 2, seen above; its next, block
        // j + 1, needs P(j): so the parity names P(j - 1).V.)
        const uint32_t prev_ord = t_other0 + static_cast<uint32_t>(j - 1) / 2;
        ok = ok && W.wait(bar(L::bPFree + (1 - s)), prev_ord & 1, 11);
        if (ok) {
          tc_fence_after();
          // O's factor; O is still zero while m_prev = -inf (every earlier P was 0).
          const float alpha = (m_prev == -INFINITY) ? 0.f : fast_exp2(m_prev - m_j);
#pragma unroll 1
          for (int ch = 0; ch < HD / 32; ++ch) {
            uint32_t o[32];
            tmem_ld_x32(tO + ch * 32, o);
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st_x32(tO + ch * 32, o);
          }
        }
      }
      if (ok) {
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(L::bPFull + s));
      }
      CALIBATT_TRACE_EVENT(lane == 0 && quarter == 0, 20 + warp, g);
      ++t_me;
    }
    // The other stream's block count, to name its P.V completions.
    t_other += (it.n + s) / 2;

    // ------------------------------------------------------------ epilogue
    // (A failed wait is acted on at the pair barrier below, which both warps
    // of the pair reach; leaving earlier could strand the partner there.)
    ok = ok && W.wait(bar(L::bOFull), item & 1, 12);
    if (ok) tc_fence_after();
    kv += it.n;
    CALIBATT_TRACE_EVENT(lane == 0 && warp == 0, 10, item + CALIBATT_TRACE_OFFSET);
    // Exchange buffer alternates by item so the partner's read of the
    // previous item's values can never meet this item's writes.
    float* xb = xchg + (item & 1) * 512;
    xb[(s * 2 + 0) * 128 + row] = m_own;
    xb[(s * 2 + 1) * 128 + row] = l;
    if (bar_red_or(pair_bar, 64, !ok)) { ok = false; break; }
    const float m_o = xb[((1 - s) * 2 + 0) * 128 + row];
    const float l_o = xb[((1 - s) * 2 + 1) * 128 + row];
    // References only grow along the list, so the larger one is m of the last block.
    const float m = fmaxf(m_own, m_o);
    const float l_row = (m_own == -INFINITY ? 0.f : l * fast_exp2(m_own - m)) +
                        (m_o == -INFINITY ? 0.f : l_o * fast_exp2(m_o - m));
    float inv_l = l_row > 0.f ? 1.f / l_row : 0.f;
    const int64_t bh_off = static_cast<int64_t>(it.b) * p.sb + static_cast<int64_t>(it.h) * p.sh;
    // Destination rows of this thread's output.
    int64_t dst_token = -1;
    int n_dst = 0, anchor_f = 0, anchor_w = 0, lo = 0;
    if (it.anchor) {
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
    // A key-range part of a split anchor tile (anchor-only launch): this
    // warp's 32 rows x HD/2 columns of O and the rows' (m, l) go to the
    // workspace, float32, coalesced (column-major over the warp's rows);
    // after a fence the warp counts itself in.  The warp that completes the
    // (tile, rows, half) merges every part in part order -- so the result does
    // not depend on which part ends last -- and writes the output below; the
    // others write nothing.  No warp ever waits for another CTA.
    [[maybe_unused]] bool merge = false;
    [[maybe_unused]] float w_part[4] = {0.f, 0.f, 0.f, 0.f};
    [[maybe_unused]] int64_t rec0 = 0;
    if (MODE == kModeAnchor && it.part >= 0) {
      const int parts = p.split.parts, slot = it.part >> 2, part = it.part & 3;
      const int qs = quarter * 2 + s;  // this warp's rows (quarter) and column half (stream)
      rec0 = static_cast<int64_t>(slot) * parts * 8 + qs;  // record of part i: rec0 + 8 * i
      const int64_t rec = rec0 + 8 * part;
      float* po = p.split.o + rec * (HD / 2) * 32 + lane;
#pragma unroll 1
      for (int ch = 0; ch < HD / 64; ++ch) {
        uint32_t o[32];
        tmem_ld_x32(tO + s * (HD / 2) + ch * 32, o);
#pragma unroll
        for (int c = 0; c < 32; ++c) po[(ch * 32 + c) * 32] = __uint_as_float(o[c]);
      }
      p.split.ml[rec * 32 + lane] = make_float2(m, l_row);
      __threadfence();
      __syncwarp();
      uint32_t arrived = 0;
      if (lane == 0) arrived = atomicAdd(p.split.cnt + static_cast<int64_t>(slot) * 8 + qs, 1u);
      arrived = __shfl_sync(0xFFFFFFFFu, arrived, 0);
      merge = arrived == static_cast<uint32_t>(parts - 1);
      if (!merge) {
        n_dst = 0;
      } else {
        __threadfence();
        float mi[4], li[4];
        float mm = -INFINITY;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          mi[i] = -INFINITY;
          li[i] = 0.f;
          if (i < parts) {
            const float2 v = i == part ? make_float2(m, l_row) : __ldcg(p.split.ml + (rec0 + 8 * i) * 32 + lane);
            mi[i] = v.x;
            li[i] = v.y;
            mm = fmaxf(mm, v.x);
          }
        }
        float lsum = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          w_part[i] = (i < parts && mi[i] != -INFINITY) ? fast_exp2(mi[i] - mm) : 0.f;
          lsum = fmaf(w_part[i], li[i], lsum);
        }
        inv_l = lsum > 0.f ? 1.f / lsum : 0.f;
      }
    }
#ifdef CALIBATT_TRACE
    const unsigned long long t_epi = globaltimer();
#endif
    if ((MODE == kModeFused || MODE == kModeAnchor) && it.anchor) {
      // Anchor broadcast through shared memory: the warp stages 8 of its rows
      // at a time (each row's HD/2 output columns, HD bytes), then every
      // destination row is written by HD/16 lanes storing its contiguous
      // bytes, so one warp-wide store covers 32*16/HD rows instead of 32
      // rows 16 bytes each (half the L2 write sectors; the stores issue at
      // HBM rate).
      uint4 pk[HD / 64][4];
#pragma unroll
      for (int ch = 0; ch < HD / 64; ++ch) {
        uint32_t o[32];
        if (it.n > 0) {
          tmem_ld_x32(tO + s * (HD / 2) + ch * 32, o);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = 0u;
        }
        if (MODE == kModeAnchor && merge) {
          // sum over the parts in part order (this part's values from tensor
          // memory are the ones it wrote)
          const int parts = p.split.parts, part = it.part & 3;
          float acc[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) acc[c] = 0.f;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            if (i < parts) {
              const float* src = p.split.o + (rec0 + 8 * i) * (HD / 2) * 32 + (ch * 32) * 32 + lane;
#pragma unroll
              for (int c = 0; c < 32; ++c) {
                const float x = i == part ? __uint_as_float(o[c]) : __ldcg(src + c * 32);
                acc[c] = fmaf(w_part[i], x, acc[c]);
              }
            }
          }
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(acc[c]);
        }
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          float v[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) v[e] = __uint_as_float(o[8 * g + e]) * inv_l;
          pk[ch][g].x = pack_bf16x2(v[0], v[1]);
          pk[ch][g].y = pack_bf16x2(v[2], v[3]);
          pk[ch][g].z = pack_bf16x2(v[4], v[5]);
          pk[ch][g].w = pack_bf16x2(v[6], v[7]);
        }
      }
      constexpr int kUnits = HD / 16;            // 16-byte units of a staged row
      constexpr int kRowsPerStore = 32 / kUnits;  // rows one warp-wide store covers
      uint8_t* stg = gbase + L::kStage + warp * L::kStageBytes;
      const int u = lane % kUnits;
      // this thread's first destination (in 16-byte units from O) and the step
      // between the rows its anchor serves (same column, next spatial row)
      const int64_t first = (bh_off + ((static_cast<int64_t>(anchor_f) * p.anc.rows + lo) * p.anc.cols + anchor_w) * p.sn +
                             s * (HD / 2)) / 8;
      const int64_t step = static_cast<int64_t>(p.anc.cols) * p.sn / 8;
      uint4* const o16 = reinterpret_cast<uint4*>(p.o);
#pragma unroll 1
      for (int pass = 0; pass < 4; ++pass) {
        if ((lane >> 3) == pass) {
          // unit g of staged row r sits at position g ^ r (no bank conflicts
          // between the 8 rows written at once)
          const int r = lane & 7;
          uint4* sp = reinterpret_cast<uint4*>(stg + r * L::kStageRowBytes);
#pragma unroll
          for (int ch = 0; ch < HD / 64; ++ch)
#pragma unroll
            for (int g = 0; g < 4; ++g) sp[((ch * 4 + g) ^ r) & (kUnits - 1)] = pk[ch][g];
        }
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 8 / kRowsPerStore; ++i) {
          const int r = lane / kUnits + kRowsPerStore * i;  // staged row 0..7
          const int src = pass * 8 + r;                     // lane that owns it
          const int nd = __shfl_sync(0xFFFFFFFFu, n_dst, src);
          uint4* dst = o16 + __shfl_sync(0xFFFFFFFFu, first, src) + u;
          const uint4 val = reinterpret_cast<const uint4*>(stg + r * L::kStageRowBytes)[(u ^ r) & (kUnits - 1)];
#pragma unroll 1
          for (int d = 0; d < nd; ++d, dst += step) *dst = val;
        }
        __syncwarp();
      }
    } else {
    // block-sparse item: this thread's row, its HD/2 output columns
#pragma unroll 1
    for (int ch = 0; ch < HD / 64; ++ch) {
      const int col = s * (HD / 2) + ch * 32;  // this group's output columns
      uint32_t o[32];
      if (it.n > 0) {
        tmem_ld_x32(tO + col, o);
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) o[c] = 0u;
      }
      uint4 pkd[4];
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        float v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = __uint_as_float(o[8 * g + e]) * inv_l;
        pkd[g].x = pack_bf16x2(v[0], v[1]);
        pkd[g].y = pack_bf16x2(v[2], v[3]);
        pkd[g].z = pack_bf16x2(v[4], v[5]);
        pkd[g].w = pack_bf16x2(v[6], v[7]);
      }
      if (n_dst > 0) {
        uint4* dst = reinterpret_cast<uint4*>(p.o + bh_off + static_cast<int64_t>(dst_token) * p.sn + col);
#pragma unroll
        for (int g = 0; g < 4; ++g) dst[g] = pkd[g];
      }
    }
    }
#ifdef CALIBATT_TRACE
    if (it.anchor && warp == 0 && lane == 0 && blockIdx.x < 1024) {
      g_epi_ns[blockIdx.x] += globaltimer() - t_epi;
      g_epi_items[blockIdx.x] += 1;
    }
#endif
    if (!it.anchor && s == 0 && p.lse != nullptr && dst_token >= 0) {
      p.lse[(static_cast<int64_t>(it.b) * p.heads + it.h) * p.seq_len + dst_token] =
          it.n > 0 ? (m + __log2f(l_row)) * 0.69314718055994531f : -INFINITY;
    }
    tc_fence_before();
    mbar_arrive(bar(L::bOFree));
    CALIBATT_TRACE_EVENT(lane == 0 && warp == 0, 11, item + CALIBATT_TRACE_OFFSET);
    ++item;
  }
}

// ------------------------------------------------- calibration (energy) roles
// Key Designs 1, Eq. (5) on the tensor-core pipeline.  LSE mode: each stream
// keeps an exact running maximum and sum of its rows over its key blocks, and
// the epilogue merges the two streams into lse2 = log2 sum_j 2^(s_ij log2e
// scale).  Energy mode: per key block c, each thread sums 2^(s log2e scale -
// lse2) over the block's keys for its query row; the block's rows are summed
// in a fixed order (warp shuffle tree, then the four warps of the stream in
// order) and E[r, c] = sum / |I_r| is written by one thread.
constexpr int kEnergyBarrier = 6;  // named barriers 6 and 7: the two streams' warps

template <int HD, int MODE>
__device__ void softmax_energy_role(const TcParams& p, uint32_t base, uint8_t* gbase, uint32_t tmem,
                                    const Waiter& W, int warp, int lane) {
  using L = Layout<HD>;
  auto bar = [&](int i) { return base + L::kBar + 8u * i; };
  const int quarter = warp & 3, s = warp >> 2;
  const int row = quarter * 32 + lane;
  const int pair_bar = 1 + quarter;
  float* xchg = reinterpret_cast<float*>(gbase + L::kXchg);
  // per-warp partial sums [2 block parity][2 streams][4 warps] (energy mode)
  float* part = reinterpret_cast<float*>(gbase + L::kMSlot);
  const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
  const uint32_t tS = tmem + lane_off + kColS + s * 128;
  const int ragged_cols = p.seq_len % 128;
  const float sl2 = p.scale_log2;
  Cursor<HD, MODE> cur;
  cur.init(p, base, false);
  Item it;
  uint32_t item = 0, t_me = 0;
  bool ok = true;
  while (cur.next(p, it, W)) {
    const int n_s = (it.n + 1 - s) / 2;
    const int token = it.tile * 128 + row;
    const bool valid = token < p.seq_len;
    const int64_t bh = static_cast<int64_t>(it.b) * p.heads + it.h;
    float lse2 = 0.f;
    if (MODE == kModeEnergy && valid) lse2 = p.lse[bh * p.seq_len + token];
    float m = -INFINITY, l = 0.f;
    for (int k = 0; k < n_s; ++k) {
      const int j = 2 * k + s;
      ok = ok && W.wait(bar(L::bSFull + s), t_me & 1, 10);
      if (ok) tc_fence_after();
      uint32_t sr[128];
      tmem_ld_x128(tS, sr);
      tc_fence_before();
      if (ok) mbar_arrive(bar(L::bSFree + s));
      float sc[128];
#pragma unroll
      for (int c = 0; c < 128; ++c) sc[c] = __uint_as_float(sr[c]);
      if (j == it.n - 1 && it.ragged_last) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= ragged_cols) sc[c] = -INFINITY;
      }
      float la = 0.f, lb = 0.f, lc = 0.f, ld = 0.f;
      float off;
      if (MODE == kModeLse) {
        float mx8[8];
#pragma unroll
        for (int a = 0; a < 8; ++a) mx8[a] = fmaxf(sc[a], sc[a + 8]);
#pragma unroll
        for (int c = 16; c < 128; c += 16) {
#pragma unroll
          for (int a = 0; a < 8; ++a) mx8[a] = fmax3(mx8[a], sc[c + a], sc[c + a + 8]);
        }
        const float mx = fmaxf(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(fmax3(mx8[3], mx8[4], mx8[5]), mx8[6], mx8[7])) * sl2;
        const float m_new = fmaxf(m, mx);
        if (m_new != m) {
          l = (m == -INFINITY) ? 0.f : l * fast_exp2(m - m_new);
          m = m_new;
        }
        off = (m == -INFINITY) ? 0.f : m;
      } else {
        off = lse2;
      }
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        float x0, x1;
        fma2(x0, x1, sc[2 * c], sc[2 * c + 1], sl2, sl2, -off, -off);
        float p0, p1;
        if (kEnergyPolyEvery > 0 && (c % kEnergyPolyEvery) == kEnergyPolyEvery - 1) {
          exp2_fma2_quintic(p0, p1, x0, x1);
        } else {
          p0 = fast_exp2(x0);
          p1 = fast_exp2(x1);
        }
        if (c & 1) add2(lc, ld, lc, ld, p0, p1); else add2(la, lb, la, lb, p0, p1);
      }
      const float rs = (la + lb) + (lc + ld);
      if (MODE == kModeLse) {
        l += rs;
      } else {
        // sum over the block's valid query rows, in a fixed order
        float v = valid ? rs : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
        float* pb = part + ((k & 1) * 2 + s) * 4;
        if (lane == 0) pb[quarter] = v;
        cta_bar_sync(kEnergyBarrier + s, 128);
        if (quarter == 0 && lane == 0) {
          const int valid_rows = min(128, p.seq_len - it.tile * 128);
          const float e = (((pb[0] + pb[1]) + pb[2]) + pb[3]) / static_cast<float>(valid_rows);
          p.energy[(bh * p.nb + it.tile) * p.nb + j] = e;
        }
      }
      ++t_me;
    }
    if (MODE == kModeLse) {
      // merge the two streams' (m, l) of every row; group 0 writes lse2
      float* xb = xchg + (item & 1) * 512;
      xb[(s * 2 + 0) * 128 + row] = m;
      xb[(s * 2 + 1) * 128 + row] = l;
      if (bar_red_or(pair_bar, 64, !ok)) { ok = false; break; }
      if (s == 0 && valid) {
        const float m1 = xb[(2 + 0) * 128 + row], l1 = xb[(2 + 1) * 128 + row];
        const float mm = fmaxf(m, m1);
        const float ll = (m == -INFINITY ? 0.f : l * fast_exp2(m - mm)) + (m1 == -INFINITY ? 0.f : l1 * fast_exp2(m1 - mm));
        p.lse[bh * p.seq_len + token] = mm + __log2f(ll);
      }
    }
    ++item;
  }
}

// Spatial-repetition sums (Key Designs 3) on the tensor-core pipeline.  Per
// key block, thread t of stream s reads row t of its two score tiles: its
// query i = tile * 128 + t and the partner query i' (same frame and column,
// nearest anchor row).  With P_ij = 2^(s_ij log2e scale - lse2_i) from the
// LSE pass, it accumulates sum_j P_ij P_i'j, sum_j P_ij^2 and sum_j P_i'j^2
// (four partial sums each, combined in a fixed order); the two streams'
// sums are added in the epilogue and written per query, three planes of
// [batch * heads * seq_len] floats.  The rows' cosine similarities come from
// those per-query sums in a separate fixed-order reduction.
template <int HD>
__device__ void softmax_similarity_role(const TcParams& p, uint32_t base, uint8_t* gbase, uint32_t tmem,
                                        const Waiter& W, int warp, int lane) {
  using L = Layout<HD>;
  constexpr int MODE = kModeSimilarity;
  auto bar = [&](int i) { return base + L::kBar + 8u * i; };
  const int quarter = warp & 3, s = warp >> 2;
  const int row = quarter * 32 + lane;
  const int pair_bar = 1 + quarter;
  float* xchg = reinterpret_cast<float*>(gbase + L::kXchg);  // [2 item parity][3 sums][128 rows]
  const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
  const uint32_t tA = tmem + lane_off + kColS + s * 256;  // own queries
  const uint32_t tB = tA + 128;                           // partner queries
  const int ragged_cols = p.seq_len % 128;
  const float sl2 = p.scale_log2;
  const int64_t plane = static_cast<int64_t>(p.batch) * p.heads * p.seq_len;
  Cursor<HD, MODE> cur;
  cur.init(p, base, false);
  Item it;
  uint32_t item = 0, t_me = 0;
  bool ok = true;
  while (cur.next(p, it, W)) {
    const int n_s = (it.n + 1 - s) / 2;
    const int64_t token = static_cast<int64_t>(it.tile) * 128 + row;
    const bool valid = token < p.seq_len;
    const int64_t bh = static_cast<int64_t>(it.b) * p.heads + it.h;
    float la = 0.f, lb = 0.f;  // log2-sum-exp of the own and the partner query
    if (valid) {
      la = p.lse[bh * p.seq_len + token];
      lb = p.lse[bh * p.seq_len + partner_token(p.anc, token)];
    }
    float ab[4] = {0.f, 0.f, 0.f, 0.f}, aa[4] = {0.f, 0.f, 0.f, 0.f}, bb[4] = {0.f, 0.f, 0.f, 0.f};
    for (int k = 0; k < n_s; ++k) {
      const int j = 2 * k + s;
      ok = ok && W.wait(bar(L::bSFull + s), t_me & 1, 10);
      if (ok) tc_fence_after();
      const bool ragged = j == it.n - 1 && it.ragged_last;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t ra[64], rb[64];
        tmem_ld_x64(tA + hh * 64, ra);
        tmem_ld_x64(tB + hh * 64, rb);
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          float x0, x1, y0, y1;
          fma2(x0, x1, __uint_as_float(ra[2 * c]), __uint_as_float(ra[2 * c + 1]), sl2, sl2, -la, -la);
          fma2(y0, y1, __uint_as_float(rb[2 * c]), __uint_as_float(rb[2 * c + 1]), sl2, sl2, -lb, -lb);
          float p0, p1, q0, q1;
          if (kEnergyPolyEvery > 0 && (c % kEnergyPolyEvery) == kEnergyPolyEvery - 1) {
            exp2_fma2_quintic(p0, p1, x0, x1);
          } else {
            p0 = fast_exp2(x0);
            p1 = fast_exp2(x1);
          }
          q0 = fast_exp2(y0);
          q1 = fast_exp2(y1);
          if (ragged) {
            const int col = hh * 64 + 2 * c;
            if (col >= ragged_cols) p0 = q0 = 0.f;
            if (col + 1 >= ragged_cols) p1 = q1 = 0.f;
          }
          const int acc = c & 3;
          ab[acc] = fmaf(p0, q0, fmaf(p1, q1, ab[acc]));
          aa[acc] = fmaf(p0, p0, fmaf(p1, p1, aa[acc]));
          bb[acc] = fmaf(q0, q0, fmaf(q1, q1, bb[acc]));
        }
      }
      // both score tiles are in registers: the stream's next S may overwrite them
      tc_fence_before();
      if (ok) mbar_arrive(bar(L::bSFree + s));
      ++t_me;
    }
    // the two streams' sums of every row meet in shared memory; group 0 writes them
    const float sums[3] = {(ab[0] + ab[1]) + (ab[2] + ab[3]), (aa[0] + aa[1]) + (aa[2] + aa[3]),
                           (bb[0] + bb[1]) + (bb[2] + bb[3])};
    float* xb = xchg + (item & 1) * 384;
    if (s == 1) {
#pragma unroll
      for (int q = 0; q < 3; ++q) xb[q * 128 + row] = sums[q];
    }
    if (bar_red_or(pair_bar, 64, !ok)) { ok = false; break; }
    if (s == 0 && valid) {
#pragma unroll
      for (int q = 0; q < 3; ++q) p.energy[q * plane + bh * p.seq_len + token] = sums[q] + xb[q * 128 + row];
    }
    ++item;
  }
}

template <int HD, int MODE>
__global__ void __launch_bounds__(kThreads, 1) tc_attn_kernel(const __grid_constant__ TcParams p) {
  using L = Layout<HD>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::kMisc + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (MODE == kModeSparse && p.sched.csr_gate) {
    // Caller-held lists: skip the whole CTA if the check that ran before
    // this launch recorded a violation (one read, shared by the CTA, before
    // any barrier or tensor memory is set up).
    __shared__ int skip;
    if (threadIdx.x == 0) skip = csr_violation_recorded(p.status);
    __syncthreads();
    if (skip) return;
  }
#ifdef CALIBATT_TRACE
  if (threadIdx.x == 0 && blockIdx.x < 1024) g_cta_span[2 * blockIdx.x] = globaltimer();
#endif
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
    for (int st = 0; st < 2; ++st) {
      mbar_init(bar(L::bSFull + st), 1);
      mbar_init(bar(L::bSFree + st), kGroupThreads);
      mbar_init(bar(L::bPFull + st), kGroupThreads);
      mbar_init(bar(L::bPFree + st), 1);
    }
    mbar_init(bar(L::bOFull), 1);
    mbar_init(bar(L::bOFree), kSoftmaxThreads);
    mbar_init(bar(L::bDrain), 2);  // one commit from each MMA-issuing thread
    for (int r = 0; r < kItemRing; ++r) {
      mbar_init(bar(L::bItemFull + r), 1);
      mbar_init(bar(L::bItemEmpty + r), kItemReaders);
    }
    for (int i = 0; i < 256; ++i) st_shared_v2(base + L::kMSlot + i * 8, 0u, 0u);  // tag 0: no m yet
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kProducerWarp && lane == 0 && MODE != kModeAnchor) {
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

  // After the register split the two kinds of warpgroup never share code
  // again: each ends with its own copy of the final CTA barrier.
  if (warp >= 8) {
    reg_dealloc<kOtherRegs>();
    if (warp == kProducerWarp) {
      producer_role<HD, MODE, false>(p, base, gbase, W, lane);
    } else if (warp == kVProducerWarp) {
      producer_role<HD, MODE, true>(p, base, gbase, W, lane);
    } else if (warp == kMmaWarp) {
      mma_s_role<HD, MODE>(p, base, tmem, W, lane);
    } else if (warp == kPvWarp) {
      mma_pv_role<HD, MODE>(p, base, tmem, W, lane);
    }
    tc_fence_before();
    cta_bar_sync(kEndBarrier, kThreads);
    if (warp == kMmaWarp) {
      tc_fence_after();
      tmem_dealloc(tmem, kTmemCols);
    }
#ifdef CALIBATT_TRACE
    if (warp == kMmaWarp && lane == 0 && blockIdx.x < 1024) g_cta_span[2 * blockIdx.x + 1] = globaltimer();
#endif
  } else {
    reg_alloc<kSoftmaxRegs>();
    if (MODE == kModeSimilarity)
      softmax_similarity_role<HD>(p, base, gbase, tmem, W, warp, lane);
    else if (MODE == kModeLse || MODE == kModeEnergy)
      softmax_energy_role<HD, MODE>(p, base, gbase, tmem, W, warp, lane);
    else
      softmax_role<HD, MODE>(p, base, gbase, tmem, W, warp, lane);
    tc_fence_before();
    cta_bar_sync(kEndBarrier, kThreads);
  }
}

template <int HD, int MODE>
cudaError_t launch_one(const TcParams& p, int grid, cudaStream_t s) {
  auto kern = tc_attn_kernel<HD, MODE>;
  const int bytes = Layout<HD>::kBytes;
  // The register split above assumes the CTA is launched with kLaunchRegs per
  // thread; with fewer, setmaxnreg.inc could never be satisfied.
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, bytes, s>>>(p);
  return cudaGetLastError();
}

// Even elements go through the packed pair routine the softmax uses (with their
// odd neighbour), a trailing odd element through the scalar one.
template <bool QUINTIC>
__global__ void exp2_fma_kernel(const float* __restrict__ x, float* __restrict__ y, int64_t n) {
  for (int64_t i = 2 * (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x); i < n;
       i += 2 * static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float x1 = i + 1 < n ? x[i + 1] : 0.f;
    float y0, y1;
    if (QUINTIC) {
      exp2_fma2_quintic(y0, y1, x[i], x1);
    } else if (i + 1 < n) {
      exp2_fma2(y0, y1, x[i], x1);
    } else {
      y0 = exp2_fma(x[i]);
    }
    y[i] = y0;
    if (i + 1 < n) y[i + 1] = y1;
  }
}

}  // namespace

#ifdef CALIBATT_TRACE
extern "C" int calibatt_trace_read(unsigned long long* host, int max_records) {
  const int n = static_cast<int>(kTraceEvents * kTraceIters);
  cudaMemcpyFromSymbol(host, g_trace, sizeof(unsigned long long) * (n < max_records ? n : max_records));
  return n;
}
extern "C" int calibatt_cta_span_read(unsigned long long* host, int max_records) {
  const int n = 2 * 1024;
  cudaMemcpyFromSymbol(host, g_cta_span, sizeof(unsigned long long) * (n < max_records ? n : max_records));
  return n;
}
extern "C" int calibatt_epilogue_probe_read(unsigned long long* ns, unsigned long long* items, int max_ctas) {
  const int n = max_ctas < 1024 ? max_ctas : 1024;
  cudaMemcpyFromSymbol(ns, g_epi_ns, sizeof(unsigned long long) * n);
  cudaMemcpyFromSymbol(items, g_epi_items, sizeof(unsigned long long) * n);
  return n;
}
extern "C" int calibatt_item_trace_read(unsigned long long* t, unsigned int* w, int max_records) {
  const int n = 1024 * kItemTrace < max_records ? 1024 * kItemTrace : max_records;
  cudaMemcpyFromSymbol(t, g_item_t, sizeof(unsigned long long) * n);
  cudaMemcpyFromSymbol(w, g_item_w, sizeof(unsigned int) * n);
  return n;
}
extern "C" void calibatt_trace_reset() {
  static unsigned long long zeros_cta[1024];
  cudaMemcpyToSymbol(g_epi_ns, zeros_cta, sizeof(zeros_cta));
  cudaMemcpyToSymbol(g_epi_items, zeros_cta, sizeof(zeros_cta));
  cudaMemset(nullptr, 0, 0);
  static unsigned long long zeros[kTraceEvents * kTraceIters];
  cudaMemcpyToSymbol(g_trace, zeros, sizeof(zeros));
  static unsigned long long zeros_items[1024 * kItemTrace];
  cudaMemcpyToSymbol(g_item_t, zeros_items, sizeof(zeros_items));
}
#endif

cudaError_t launch_exp2_fma(const float* x, float* y, int64_t n, bool quintic, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const int64_t blocks = (n + 255) / 256;
  const unsigned grid = static_cast<unsigned>(blocks < 1024 ? blocks : 1024);
  if (quintic)
    exp2_fma_kernel<true><<<grid, 256, 0, s>>>(x, y, n);
  else
    exp2_fma_kernel<false><<<grid, 256, 0, s>>>(x, y, n);
  return cudaGetLastError();
}

size_t tc_smem_bytes(int head_dim) {
  return head_dim == 64 ? Layout<64>::kBytes : Layout<128>::kBytes;
}

cudaError_t launch_tc_attn(const TcParams& p, int head_dim, int mode, int grid, cudaStream_t s) {
  if (head_dim == 128) {
    if (mode == kModeSparse) return launch_one<128, kModeSparse>(p, grid, s);
    if (mode == kModeAnchor) return launch_one<128, kModeAnchor>(p, grid, s);
    if (mode == kModeFused) return launch_one<128, kModeFused>(p, grid, s);
    if (mode == kModeLse) return launch_one<128, kModeLse>(p, grid, s);
    if (mode == kModeEnergy) return launch_one<128, kModeEnergy>(p, grid, s);
    if (mode == kModeSimilarity) return launch_one<128, kModeSimilarity>(p, grid, s);
  }
  if (head_dim == 64) {
    if (mode == kModeSparse) return launch_one<64, kModeSparse>(p, grid, s);
    if (mode == kModeAnchor) return launch_one<64, kModeAnchor>(p, grid, s);
    if (mode == kModeFused) return launch_one<64, kModeFused>(p, grid, s);
    if (mode == kModeLse) return launch_one<64, kModeLse>(p, grid, s);
    if (mode == kModeEnergy) return launch_one<64, kModeEnergy>(p, grid, s);
    if (mode == kModeSimilarity) return launch_one<64, kModeSimilarity>(p, grid, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace calibatt
