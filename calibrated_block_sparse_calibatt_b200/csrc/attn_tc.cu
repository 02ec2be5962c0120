// Tensor-core attention for CalibAtt on sm_100a (B200): the block-sparse path
// and the anchor-row path with broadcast, one persistent kernel template.
//
// What it computes ("Accelerating Text-to-Video Generation with Calibrated
// Sparse Attention", paper note, Key Designs 3 and 4): for each scheduled
// 128-query tile, online-softmax attention over a list of 128-key blocks --
// the calibrated skip list of the (head, query block) on the sparse path, or
// every key block for a tile of gathered anchor-row queries on the anchor
// path -- normalised and written to the output, once per query on the sparse
// path and to every row an anchor serves on the anchor path.
//
// CTA layout (320 threads, one CTA per SM, persistent):
//   warps 0-7  softmax + epilogue; warp w owns query rows 32*(w%4)..+31 (its
//              TMEM lane quarter) and score columns 64*(w/4)..+63
//   warp  8    producer: TMA loads of Q and of K/V tiles gathered by block
//              index (or a plain-load gather of anchor Q rows)
//   warp  9    TMEM allocator and MMA issuer (one lane issues tcgen05.mma)
// Tensor memory (512 columns): S = Q K^T at 0..127 (f32), two P buffers
// (bf16 pairs) at 128..191 and 192..255, O accumulator at 256..256+D.  With P
// double-buffered the softmax writes P_{j+1} while O += P_j V_j still runs.
// Pipelines (mbarriers): Q 1 stage, K 3 stages, V 2 stages; S/P/O handshakes
// between the MMA warp and the softmax warps.  Per key block j the MMA warp
// issues S_j = Q K_j^T as soon as the softmax warps have read S_{j-1} out of
// tensor memory, then O += P_{j-1} V_{j-1}, so the tensor core works on the
// next block's scores while the softmax warps exponentiate the current one.
// The softmax keeps a reference maximum m and only rescales O and l when a
// row maximum exceeds m by more than 2^8 (exp2 domain), so P stays <= 256.
#include "internal.h"
#include "ptx.cuh"

#include <math.h>

namespace calibatt {
namespace {

using namespace ptx;

constexpr int kThreads = 320;  // 8 softmax warps, producer, MMA
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kSoftmaxThreads = 256;
constexpr int kKStages = 3;
constexpr int kVStages = 2;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;
constexpr uint32_t kColP = 128;  // P buffer b at kColP + 64 * b
constexpr uint32_t kColO = 256;
constexpr float kRescaleLog2 = 8.0f;
// One pair in kPolyEvery of exponentials runs on the FMA pipe (exp2_fma)
// instead of the MUFU unit, which would otherwise bound the softmax at D=128.
constexpr int kPolyEvery = 4;
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
  static constexpr int bSFull = bVEmpty + kVStages, bSFree = bSFull + 1;
  static constexpr int bPFull = bSFree + 1;      // [2], one per P buffer
  static constexpr int bPVDone = bPFull + 2;     // [2], P.V reading P buffer b finished
  static constexpr int bOFree = bPVDone + 2, bDrain = bOFree + 1;
  static constexpr int kNumBars = bDrain + 1;
  static constexpr int kMisc = kBar + kNumBars * 8;  // u32 tmem base, i32 abort flag
  static constexpr int kXchg = kMisc + 16;  // float [2][2][128] row maxima + [2][128] row sums
  static constexpr int kUsed = kXchg + (512 + 256) * 4;
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

// --------------------------------------------------------------- producer
template <int HD, bool ANCHOR>
__device__ void producer_role(const TcParams& p, uint32_t base, const Waiter& W, int lane) {
  using L = Layout<HD>;
  auto bar = [&](int i) { return base + L::kBar + 8u * i; };
  Cursor<ANCHOR> cur;
  cur.init(p);
  Item it;
  uint32_t kv = 0, item = 0;
  uint32_t k_issued = 0, v_issued = 0, q_issued = 0;
  bool ok = true;
  while (ok && cur.next(p, it)) {
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
    uint32_t my_col = 0;
    for (int j = 0; j < it.n; ++j) {
      if ((j & 31) == 0) {
        const int jj = j + lane;
        my_col = ANCHOR ? static_cast<uint32_t>(jj) : (jj < it.n ? it.cols[jj] : 0u);
      }
      const int c = static_cast<int>(__shfl_sync(0xFFFFFFFFu, my_col, j & 31));
      const uint32_t ks = kv % kKStages, ku = kv / kKStages;
      if (ku > 0 && !W.wait(bar(L::bKEmpty + ks), (ku - 1) & 1, 2)) { ok = false; break; }
      if (lane == 0) {
        mbar_arrive_expect_tx(bar(L::bKFull + ks), L::kTile);
        tma_tile<HD>(base + L::kK + ks * L::kTile, &p.tm_k, bar(L::bKFull + ks), p, c * 128, it.h, it.b);
      }
      ++k_issued;
      const uint32_t vs = kv % kVStages, vu = kv / kVStages;
      if (vu > 0 && !W.wait(bar(L::bVEmpty + vs), (vu - 1) & 1, 3)) { ok = false; break; }
      if (lane == 0) {
        mbar_arrive_expect_tx(bar(L::bVFull + vs), L::kTile);
        tma_tile<HD>(base + L::kV + vs * L::kTile, &p.tm_v, bar(L::bVFull + vs), p, c * 128, it.h, it.b);
      }
      ++v_issued;
      ++kv;
    }
    ++item;
  }
  // Let every bulk copy this warp issued land before the CTA can exit.
  for (uint32_t s = 0; s < kKStages; ++s)
    if (k_issued > s) drain_wait(bar(L::bKFull + s), ((k_issued - 1 - s) / kKStages) & 1);
  for (uint32_t s = 0; s < kVStages; ++s)
    if (v_issued > s) drain_wait(bar(L::bVFull + s), ((v_issued - 1 - s) / kVStages) & 1);
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
  uint32_t kv = 0, item = 0;
  bool ok = true;

  // O += P_t V_t for key-block iteration t (global counter); `first` zeroes O.
  // P_t lives in tensor-memory buffer t & 1.
  auto issue_pv = [&](uint32_t t, bool first) -> bool {
    const uint32_t vs = t % kVStages, pb = t & 1;
    if (!W.wait(bar(L::bVFull + vs), (t / kVStages) & 1, 7)) return false;
    if (!W.wait(bar(L::bPFull + pb), (t >> 1) & 1, 8)) return false;
    if (first && item > 0 && !W.wait(bar(L::bOFree), (item - 1) & 1, 9)) return false;
    tc_fence_after();
    if (lane == 0) {
      const uint32_t v_base = base + L::kV + vs * L::kTile;
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        // B = V (MN-major): 16 keys per step = 2048 bytes; next 64 columns of D at +16 KB.
        mma_ts(tmem + kColO, tmem + kColP + pb * 64 + s * 8, sw128_desc(v_base + s * 2048, kChunkBytes, 1024),
               kIdescO, (first && s == 0) ? 0u : 1u);
      }
      mma_commit(bar(L::bVEmpty + vs));
      mma_commit(bar(L::bPVDone + pb));
    }
    __syncwarp();
    return true;
  };

  while (ok && cur.next(p, it)) {
    if (!W.wait(bar(L::bQFull), item & 1, 4)) break;
    tc_fence_after();
    for (int j = 0; j < it.n; ++j) {
      const uint32_t ks = kv % kKStages;
      if (!W.wait(bar(L::bKFull + ks), (kv / kKStages) & 1, 5)) { ok = false; break; }
      if (kv > 0 && !W.wait(bar(L::bSFree), (kv - 1) & 1, 6)) { ok = false; break; }
      tc_fence_after();
      if (lane == 0) {
        const uint32_t k_base = base + L::kK + ks * L::kTile;
#pragma unroll
        for (int s = 0; s < HD / 16; ++s) {
          // K-major operands: 16 columns = 32 bytes per step inside a 64-column chunk.
          const uint32_t off = (s >> 2) * kChunkBytes + (s & 3) * 32;
          mma_ss(tmem + kColS, sw128_desc(base + L::kQ + off, 16, 1024), sw128_desc(k_base + off, 16, 1024),
                 kIdescS, s > 0 ? 1u : 0u);
        }
        mma_commit(bar(L::bKEmpty + ks));
        mma_commit(bar(L::bSFull));
        if (j == it.n - 1) mma_commit(bar(L::bQEmpty));
      }
      __syncwarp();
      if (j > 0 && !issue_pv(kv - 1, j == 1)) { ok = false; break; }
      ++kv;
    }
    if (!ok) break;
    if (it.n > 0) {
      if (!issue_pv(kv - 1, it.n == 1)) break;
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
// Eight warps: warp w handles query rows 32*(w%4) .. +31 (its TMEM lane
// quarter) and score columns 64*(w/4) .. +63.  The two warps sharing rows (w
// and w+4) exchange their partial row maxima once per key block, and their
// partial row sums at the end, through shared memory at a pair barrier
// (bar.red.or, 64 threads).  The barrier also carries "a wait failed" so that
// both warps of a pair always leave the loop together.
template <int HD, bool ANCHOR>
__device__ void softmax_role(const TcParams& p, uint32_t base, uint8_t* gbase, uint32_t tmem,
                             const Waiter& W, int warp, int lane) {
  using L = Layout<HD>;
  auto bar = [&](int i) { return base + L::kBar + 8u * i; };
  const int quarter = warp & 3, half = warp >> 2;
  const int row = quarter * 32 + lane;  // query row within the tile == TMEM lane
  const int pair_bar = 1 + quarter;     // named barrier shared with the partner warp
  float* xchg = reinterpret_cast<float*>(gbase + L::kXchg);  // [2 buffers][2 halves][128 rows]
  const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
  const uint32_t tS = tmem + lane_off + kColS + half * 64;
  const uint32_t tP = tmem + lane_off + kColP + half * 32;
  const uint32_t tO = tmem + lane_off + kColO + half * (HD / 2);
  const int ragged_cols = p.seq_len % 128;
  const int col0 = half * 64;
  const float sl2 = p.scale_log2;
  // Waits until O += P_t V_t (key-block iteration t) has completed.
  auto wait_pv = [&](uint32_t t, int where) -> bool {
    if (!W.wait(bar(L::bPVDone + (t & 1)), (t >> 1) & 1, where)) return false;
    tc_fence_after();
    return true;
  };
  Cursor<ANCHOR> cur;
  cur.init(p);
  Item it;
  uint32_t kv = 0;
  bool ok = true;
  while (cur.next(p, it)) {
    float m_ref = -INFINITY, l = 0.f;
    for (int j = 0; j < it.n; ++j) {
      ok = ok && W.wait(bar(L::bSFull), kv & 1, 10);
      if (ok) tc_fence_after();
      uint32_t sr[64];
      tmem_ld_x64(tS, sr);
      tc_fence_before();
      if (ok) mbar_arrive(bar(L::bSFree));
      float s[64];
#pragma unroll
      for (int c = 0; c < 64; ++c) s[c] = __uint_as_float(sr[c]);
      if (j == it.n - 1 && it.ragged_last) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (col0 + c >= ragged_cols) s[c] = -INFINITY;
      }
      float mx8[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) mx8[a] = s[a];
#pragma unroll
      for (int c = 8; c < 64; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], s[c]);
      const float mx_half = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                  fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      float* xb = xchg + (kv & 1) * 256;
      xb[half * 128 + row] = mx_half;
      if (bar_red_or(pair_bar, 64, !ok)) { ok = false; break; }
      const float mx_s = fmaxf(mx_half, xb[(1 - half) * 128 + row]) * sl2;
      // The decision is taken per warp (tcgen05.ld/st are .sync.aligned and
      // need all 32 lanes); both warps of a pair see the same row maxima and
      // so decide alike.  Rows of a rescaling warp whose maximum did not grow
      // get alpha = 1.
      if (__any_sync(0xFFFFFFFFu, mx_s > m_ref + kRescaleLog2)) {
        const float m_new = fmaxf(m_ref, mx_s);
        const float alpha = (m_new == -INFINITY) ? 1.f : fast_exp2(m_ref - m_new);
        l *= alpha;
        if (j > 0) {
          // O is stable once the previous block's P.V has completed.
          ok = ok && wait_pv(kv - 1, 11);
          if (ok) {
#pragma unroll 1
            for (int ch = 0; ch < HD / 64; ++ch) {
              uint32_t o[32];
              tmem_ld_x32(tO + ch * 32, o);
#pragma unroll
              for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
              tmem_st_x32(tO + ch * 32, o);
            }
            tmem_wait_st();
          }
        }
        m_ref = m_new;
      }
      const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
      uint32_t pk[32];
      float ls[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const float x0 = fmaf(s[2 * c], sl2, -m_use);
        const float x1 = fmaf(s[2 * c + 1], sl2, -m_use);
        const bool poly = (c % kPolyEvery) == kPolyEvery - 1;
        const float p0 = poly ? exp2_fma(x0) : fast_exp2(x0);
        const float p1 = poly ? exp2_fma(x1) : fast_exp2(x1);
        ls[c & 7] += p0 + p1;
        pk[c] = pack_bf16x2(p0, p1);
      }
      l += ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
      // P buffer kv & 1 was last read by the P.V of iteration kv - 2.
      const uint32_t pb = kv & 1;
      if (kv >= 2) ok = ok && wait_pv(kv - 2, 13);
      if (ok) {
        tmem_st_x32(tP + pb * 64, pk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(L::bPFull + pb));
      }
      ++kv;
    }

    // ------------------------------------------------------------ epilogue
    // (A failed wait is acted on at the pair barrier below, which both warps
    // of the pair reach; leaving earlier could strand the partner there.)
    if (it.n > 0) ok = ok && wait_pv(kv - 1, 12);
    float* xl = xchg + 512;  // partial row sums
    xl[half * 128 + row] = l;
    if (bar_red_or(pair_bar, 64, !ok)) { ok = false; break; }
    const float l_row = l + xl[(1 - half) * 128 + row];
    const float inv_l = l_row > 0.f ? 1.f / l_row : 0.f;
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
      uint32_t o[32];
      if (it.n > 0) {
        tmem_ld_x32(tO + ch * 32, o);
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) o[c] = 0u;
      }
      uint4 pkd[4];
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        pkd[g].x = pack_bf16x2(__uint_as_float(o[8 * g + 0]) * inv_l, __uint_as_float(o[8 * g + 1]) * inv_l);
        pkd[g].y = pack_bf16x2(__uint_as_float(o[8 * g + 2]) * inv_l, __uint_as_float(o[8 * g + 3]) * inv_l);
        pkd[g].z = pack_bf16x2(__uint_as_float(o[8 * g + 4]) * inv_l, __uint_as_float(o[8 * g + 5]) * inv_l);
        pkd[g].w = pack_bf16x2(__uint_as_float(o[8 * g + 6]) * inv_l, __uint_as_float(o[8 * g + 7]) * inv_l);
      }
      const int dcol = half * (HD / 2) + ch * 32;
#pragma unroll 1
      for (int d = 0; d < n_dst; ++d) {
        const int64_t token = ANCHOR
            ? (static_cast<int64_t>(anchor_f) * p.anc.rows + lo + d) * p.anc.cols + anchor_w
            : dst_token;
        uint4* dst = reinterpret_cast<uint4*>(p.o + bh_off + token * p.sn + dcol);
#pragma unroll
        for (int g = 0; g < 4; ++g) dst[g] = pkd[g];
      }
    }
    if (!ANCHOR && half == 0 && p.lse != nullptr && dst_token >= 0) {
      p.lse[(static_cast<int64_t>(it.b) * p.heads + it.h) * p.seq_len + dst_token] =
          it.n > 0 ? (m_ref + __log2f(l_row)) * 0.69314718055994531f : -INFINITY;
    }
    tc_fence_before();
    mbar_arrive(bar(L::bOFree));
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
    mbar_init(bar(L::bSFull), 1);
    mbar_init(bar(L::bSFree), kSoftmaxThreads);
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(L::bPFull + b), kSoftmaxThreads);
      mbar_init(bar(L::bPVDone + b), 1);
    }
    mbar_init(bar(L::bOFree), kSoftmaxThreads);
    mbar_init(bar(L::bDrain), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kProducerWarp && lane == 0 && !ANCHOR) {
    prefetch_tensormap(&p.tm_q);
    prefetch_tensormap(&p.tm_k);
    prefetch_tensormap(&p.tm_v);
  }
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
    producer_role<HD, ANCHOR>(p, base, W, lane);
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
