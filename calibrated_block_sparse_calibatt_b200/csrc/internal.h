// Internal declarations shared by the library's translation units: kernel
// parameter blocks and the launch functions the C ABI layer calls.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace calibatt {

constexpr int kMaxAnchors = 16;
constexpr int kMaxHeadsPerCall = 128;

// Skip lists and persistent schedule of one dictionary layer (t, l).
// Work item = (head << 16) | query_block.
struct LayerSchedule {
  const int32_t* row_ptr;   // [H][nq + 1], per head, starting at 0
  const int64_t* col_base;  // [H], offset of each head's list in `col`
  const uint16_t* col;      // retained key-block indices
  const uint32_t* items;    // work items grouped by CTA
  const int32_t* cta_ptr;   // [grid + 1], CTA c runs items[cta_ptr[c] .. cta_ptr[c+1])
  int32_t nq;
  // Bitmap dictionaries instead: bit c of row r of head h says key block c is
  // kept, words 32-bit words per row, [H][nq][words]; row_ptr/col unused.
  const uint32_t* bitmap;
  int32_t words;
  // Interval dictionaries instead of index lists: each row is a list of
  // contiguous key-block runs, packed start | (length << 16), ascending and
  // disjoint.  Head h's runs of query block r are
  // runs[col_base[h] + run_ptr[h][r] .. col_base[h] + run_ptr[h][r+1]);
  // row_ptr still counts blocks (the row's block count is the difference).
  // Bit 31 of run_ptr[h][r + 1] is set when row r keeps the last key block
  // (nq - 1); offsets are the low 31 bits.
  const int32_t* run_ptr;  // [H][nq + 1]
  const uint32_t* runs;
  // Dynamic assignment (dictionary calls): instead of the per-CTA lists in
  // items/cta_ptr, the CTAs take tickets 0, 1, ... from *ticket (zeroed before
  // the launch); ticket t is item order[t % n_order] of batch t / n_order.
  // order lists the layer's items in consumption order (L2 group, wave, cost
  // descending).  nullptr = static lists.
  uint32_t* ticket;
  const uint32_t* order;
  int32_t n_order;
  // Nonzero when the lists and schedule come from the caller's device memory
  // (direct-CSR call): the kernels then do nothing if the status word holds a
  // skip-list or schedule violation (codes 23, 24) recorded by the check that
  // runs before them on the same stream.
  int32_t csr_gate;
};
// Status-word codes (bits 8-15) of the direct-CSR checks.
constexpr int kCodeListViolation = 23;
constexpr int kCodeScheduleViolation = 24;

// True when the status word holds a violation of caller-held lists or
// schedule; read once per CTA by one thread (the caller shares the answer).
__device__ __forceinline__ bool csr_violation_recorded(const int32_t* status) {
  const int code = (*reinterpret_cast<const volatile int32_t*>(status) >> 8) & 0xFF;
  return code == kCodeListViolation || code == kCodeScheduleViolation;
}
// Longest skip list a bitmap or interval dictionary may hold per row (the
// producers decode each row into a shared-memory list of this many 16-bit
// indices).
constexpr int kMaxBitmapBlocks = 2048;

// Frame geometry of the anchor path.  Token = (f * rows + row) * cols + col.
// Packed anchor query p (0 <= p < anchor_tokens) is
//   f = p / (n_anchors * cols), a = (p / cols) % n_anchors, col = p % cols,
// served rows of anchor a are [group_lo[a], group_hi[a]].
struct AnchorGeom {
  int32_t frames, rows, cols, n_anchors;
  int32_t anchor_tokens;   // frames * n_anchors * cols
  int32_t tiles_per_head;  // ceil(anchor_tokens / 128)
  int32_t n_heads;
  int16_t anchor_row[kMaxAnchors];
  int16_t group_lo[kMaxAnchors];
  int16_t group_hi[kMaxAnchors];
  int16_t head_ids[kMaxHeadsPerCall];
};

// Anchor-only launch: the last tiles of the item sequence split into key
// ranges, so that the persistent grid ends together.  Items [0, first) are
// whole tiles; item first + e is part e % parts of tile first + e / parts
// (keys [nb * part / parts, nb * (part + 1) / parts)).  Each softmax warp of a
// part writes its rows x column half of O (float32, relative to its maximum)
// and (maximum, row sum) to the workspace, then counts itself in; the warp
// that completes a (tile, rows, half) merges the parts in part order and
// writes the output.  parts == 1: no split (first == n_tiles).
struct AnchorSplit {
  int32_t first;    // whole tiles before the split ones
  int32_t parts;    // key ranges per split tile, 1..4
  int32_t n_tiles;  // tiles over batch x heads x tiles per head
  float* o;         // [slot][part][8 warps][HD / 2 columns][32 rows]
  float2* ml;       // [slot][part][8 warps][32 rows] (maximum, row sum), exp2 domain
  uint32_t* cnt;    // [slot][8 warps] parts counted in, zeroed before the launch
};

// Tensor-core (tcgen05) attention kernel parameters, passed as __grid_constant__.
struct TcParams {
  CUtensorMap tm_q;  // bf16 Q/K/V, dims {D, x1, x2, x3}, box {64, 1|128, ...}
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  const uint16_t* q;  // raw Q (anchor-row gather)
  uint16_t* o;
  float* lse;  // nullable [batch, heads, seq_len]; energy modes: log2 LSE workspace
  float* energy;  // energy mode: [batch, heads, nb, nb]
  int64_t sb, sn, sh;  // element strides shared by Q, K, V, O
  int32_t batch, seq_len, heads, nb;
  int32_t pos_n, pos_h, pos_b;  // which tensor-map dimension (1..3) holds N, H, batch
  float scale_log2;             // softmax_scale * log2(e)
  LayerSchedule sched;
  AnchorGeom anc;
  AnchorSplit split;  // anchor-only mode
  int32_t* status;
  unsigned long long timeout_ns;
};

// CUDA-core attention kernel parameters (FP32 or BF16, any supported block).
struct SimtParams {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  float* lse;
  int64_t sb, sn, sh;
  int32_t batch, seq_len, heads, nb;
  float scale_log2;
  LayerSchedule sched;           // sparse mode: items unused, heads from head list
  int32_t n_heads;               // sparse mode: number of heads in head_ids
  int16_t head_ids[kMaxHeadsPerCall];
  AnchorGeom anc;
  int32_t* status;               // device status word (a block index out of range is recorded)
};

struct EnergyParams {
  const void* q;
  const void* k;
  float* energy;  // [batch, heads, nb, nb]
  float* lse;     // workspace [batch, heads, seq_len]
  int64_t sb, sn, sh;
  int32_t batch, seq_len, heads, nb;
  float scale_log2;
};

// Tensor-core kernel modes: block-sparse items only, anchor tiles only, or
// both kinds in one persistent launch under a joint schedule (dual path).
constexpr int kModeSparse = 0;
constexpr int kModeAnchor = 1;
constexpr int kModeFused = 2;
// Offline calibration on the same pipeline (no V, no P.V): every (head,
// query block) visits all key blocks; the LSE mode writes each query's log2
// log-sum-exp, the energy mode the block energies from it.
constexpr int kModeLse = 3;
constexpr int kModeEnergy = 4;
// Spatial-repetition score on the same pipeline (no V, no P.V): every (head,
// query tile) visits all key blocks with two score tiles per block, its own
// 128 queries and their partner queries in the nearest anchor row (same
// frame and column, gathered); each query's sums of p p', p^2 and p'^2 over
// all keys are written to `energy` as three planes [3][batch * heads * seq_len].
constexpr int kModeSimilarity = 5;
// Work-item word of the dictionary schedules: bit 31 marks an anchor tile
// (fused schedules only), bits 16-30 the head, bits 0-15 the query block or
// anchor tile.
constexpr uint32_t kItemAnchorBit = 0x80000000u;

cudaError_t launch_tc_attn(const TcParams& p, int head_dim, int mode, int grid, cudaStream_t s);
cudaError_t launch_simt_attn(const SimtParams& p, int head_dim, int block, int dtype, bool anchor,
                             int n_items, cudaStream_t s);
cudaError_t launch_block_energy(const EnergyParams& p, int head_dim, int block, int dtype,
                                cudaStream_t s);
cudaError_t launch_row_lse(const EnergyParams& p, int head_dim, int dtype, cudaStream_t s);

// Spatial-repetition score, pass 2 (repetition.cu).
struct RepetitionParams {
  const void* q;
  const void* k;
  const float* lse;   // pass-1 log2 LSE [batch, heads, seq_len]
  float* sim;         // [batch, heads, frames, rows]
  int64_t sb, sn, sh;
  int32_t batch, seq_len, heads;
  int32_t frames, rows, cols;
  float scale_log2;
  int16_t nearest[256];  // nearest anchor row of each spatial row
};
constexpr int kMaxRepetitionRows = 256;
cudaError_t launch_spatial_similarity(const RepetitionParams& p, int head_dim, int dtype, cudaStream_t s);
cudaError_t launch_similarity_from_sums(const float* sums, int64_t plane, int32_t bh_count, int32_t seq_len,
                                        int32_t frames, int32_t rows, int32_t cols, float* sim, cudaStream_t s);
cudaError_t launch_repetition_flags(const float* sim, int32_t n_prompts, int32_t n_heads, int32_t per_head,
                                    float threshold, float* mean, uint8_t* flags, cudaStream_t s);

cudaError_t launch_select_blocks(const float* energy, int64_t n_rows, int32_t nk, float tau,
                                 uint8_t* mask, int32_t* count_accum, cudaStream_t s);
cudaError_t launch_aggregate(const int32_t* counts, int64_t n, int32_t n_prompts, float rho,
                             uint8_t* mask, cudaStream_t s);

// Device-side check of caller-held skip lists (csr_check.cu).
struct CsrCheckParams {
  const int32_t* row_ptr;   // [heads][nq + 1]
  const uint16_t* col;
  const int64_t* col_base;  // [heads]
  int32_t nq;
  int32_t n_heads;
  int16_t head_ids[kMaxHeadsPerCall];
  int32_t* status;
  // persistent schedule of the tensor-core kernel (nullable): items
  // [n_heads * nq], cta_ptr [grid + 1]
  const uint32_t* items;
  const int32_t* cta_ptr;
  int32_t grid;
};
cudaError_t launch_csr_check(const CsrCheckParams& p, cudaStream_t s);

cudaError_t launch_exp2_fma(const float* x, float* y, int64_t n, bool quintic, cudaStream_t s);
cudaError_t launch_bounded_wait(int32_t* status, unsigned long long timeout_ns, cudaStream_t s);

// Records a failure message for calibatt_last_error() on the calling thread.
void set_last_error(const char* fmt, ...);

// Dynamic shared memory the tensor-core kernel needs for a head dimension.
size_t tc_smem_bytes(int head_dim);

}  // namespace calibatt
