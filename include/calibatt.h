/*
 * calibatt.h - C ABI of the CalibAtt B200 library (libcalibatt.so).
 *
 * CalibAtt ("Accelerating Text-to-Video Generation with Calibrated Sparse
 * Attention", paper note on papernotes.org, section "Method") runs video
 * self-attention through one of two precompiled paths per (timestep, layer,
 * head):
 *   - block-sparse attention over a calibrated list of retained key blocks
 *     per query block (Key Designs 1, 2 and 4);
 *   - anchor-row attention with output broadcast for heads flagged spatially
 *     repetitive (Key Designs 3 and 4).
 * It also exposes the offline calibration steps: block energy (Eq. (5)),
 * top-mass selection and cross-prompt aggregation (Eq. (8)-(9)).
 *
 * Conventions for every entry point:
 *   - Every call returns a calibatt_status.  No C++ exception crosses the ABI.
 *     On failure calibatt_last_error() returns a message for the calling thread.
 *   - Device pointers are owned by the caller.  The library never allocates
 *     device memory on the attention or calibration calls; the mask dictionary
 *     is the one library-owned object and is allocated at creation.
 *   - GPU work is enqueued asynchronously on the caller's stream (a
 *     cudaStream_t passed as void*; NULL is the legacy default stream).
 *     Nothing is synchronised except where a function says so.
 *   - Attention calls on a dictionary (bf16, block 128) hand out their work
 *     dynamically: each call zeroes one of the dictionary's 64 work counters
 *     on its stream (taken round-robin, call by call) and the persistent CTAs
 *     take work items from it.  Up to 64 calls on one dictionary may be in
 *     flight on the GPU at once; a call captured in a CUDA graph keeps its
 *     counter, so a replay must not overlap the 64th call after it on
 *     another stream.
 *   - Activations are [batch, N_alloc, heads, head_dim] with the last dimension
 *     contiguous; strides are in elements.  Tokens are ordered frame-major,
 *     then spatial row, then column: token = f*R*C + row*C + col.  Only the
 *     first seq_len tokens are read; padded rows of the output are not written.
 *   - A block is B consecutive tokens; nb = ceil(seq_len / B) blocks, the last
 *     one possibly partial.  Keys at index >= seq_len are excluded.
 *   - softmax_scale <= 0 selects 1/sqrt(head_dim).
 *   - Arguments are validated on the host before anything is enqueued:
 *     CALIBATT_ERR_INVALID_ARG for null pointers, inconsistent sizes, strides or
 *     misaligned bases; CALIBATT_ERR_UNSUPPORTED for head_dim, block or dtype
 *     outside the supported set; CALIBATT_ERR_CUDA when a CUDA call or a launch
 *     fails (the CUDA error is cleared and named in calibatt_last_error()).
 */
#ifndef CALIBATT_H_
#define CALIBATT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t calibatt_status;

#define CALIBATT_OK 0
#define CALIBATT_ERR_INVALID_ARG 1
#define CALIBATT_ERR_UNSUPPORTED 2
#define CALIBATT_ERR_CUDA 3
#define CALIBATT_ERR_TIMEOUT 4
#define CALIBATT_ERR_OOM 5

#define CALIBATT_DTYPE_BF16 0
#define CALIBATT_DTYPE_FP32 1

/* Shape of Q, K, V and O (all four share it).  head_dim in {64, 128};
 * dtype CALIBATT_DTYPE_BF16 or CALIBATT_DTYPE_FP32.  Strides in elements;
 * the head_dim dimension has stride 1.  For BF16 every stride must be a
 * multiple of 8 elements and every base 16-byte aligned. */
typedef struct calibatt_shape {
  int32_t batch;
  int32_t seq_len;   /* N: valid tokens */
  int32_t heads;     /* H */
  int32_t head_dim;  /* D */
  int64_t stride_b;
  int64_t stride_n;
  int64_t stride_h;
  int32_t dtype;
  int32_t reserved;  /* must be 0 */
} calibatt_shape;

/* Opaque mask dictionary: per (timestep t, layer l, head h) either a skip
 * list of retained key blocks for every query block, or the repetitive flag
 * that routes the head to the anchor path (Key Designs 4: "the current
 * timestep, layer, and head select the appropriate record"). */
typedef struct calibatt_dict calibatt_dict;

/* ---------------------------------------------------------------- status */

/* Static text for a status code.
 * Diagnostics; no counterpart in the paper note. */
const char* calibatt_status_string(calibatt_status status);

/* Message describing the last failure on the calling thread ("" if none).
 * Diagnostics; no counterpart in the paper note. */
const char* calibatt_last_error(void);

/* ABI version of this header (incremented on incompatible change).
 * No counterpart in the paper note. */
int32_t calibatt_abi_version(void);

/* ------------------------------------------------- host-only utilities */

/* Checks one skip list in CSR form (Key Designs 4: each binary mask becomes
 * a read-only list of key blocks to compute for each query block).
 *   row_ptr: host int32[nq + 1], row_ptr[0] == 0, non-decreasing;
 *   col_idx: host int32[row_ptr[nq]], each row strictly ascending, in [0, nk);
 *   require_diagonal != 0 additionally demands block r in row r (nq == nk).
 * Returns CALIBATT_OK or CALIBATT_ERR_INVALID_ARG naming the first offence. */
calibatt_status calibatt_csr_validate(int32_t nq, int32_t nk, const int32_t* row_ptr,
                                      const int32_t* col_idx, int32_t require_diagonal);

/* Re-encodes a validated CSR skip list as contiguous key-block intervals, the
 * encoding the paper note describes (Key Designs 4).  Outputs (host):
 *   interval_ptr int32[nq + 1]; interval_start, interval_len int32[capacity].
 * *n_intervals receives the total.  CALIBATT_ERR_INVALID_ARG if capacity is
 * too small (*n_intervals still receives the needed count). */
calibatt_status calibatt_csr_to_intervals(int32_t nq, const int32_t* row_ptr,
                                          const int32_t* col_idx, int32_t* interval_ptr,
                                          int32_t* interval_start, int32_t* interval_len,
                                          int64_t capacity, int64_t* n_intervals);

/* Longest-processing-time list scheduling of n_items work items with the
 * given costs onto n_bins bins: items in descending cost (ties by index) each
 * go to the currently least-loaded bin (ties by lower bin).  Outputs (host):
 *   bin_ptr int32[n_bins + 1]; item_order int32[n_items] lists the items of
 *   bin b at item_order[bin_ptr[b] .. bin_ptr[b+1]) in assignment order;
 *   *makespan (nullable) receives the largest bin load.
 * The paper note does not describe a schedule; this balances the persistent
 * attention kernel's query-block work by retained key-block count. */
calibatt_status calibatt_lpt_schedule(int32_t n_items, const int64_t* cost, int32_t n_bins,
                                      int32_t* bin_ptr, int32_t* item_order,
                                      int64_t* makespan);

/* --------------------------------------------------------- dictionary */

/* Creates an empty dictionary for T timesteps x L layers x H heads with
 * nq == nk == number of blocks of size `block` (64 or 128).  Device memory
 * for up to nnz_capacity retained blocks in total (2 bytes each) plus
 * per-record offsets and schedules is allocated now, on the current device.
 * num_ctas <= 0 selects the device's SM count (the persistent grid size the
 * schedules are built for).  CALIBATT_ERR_OOM if the allocation fails.
 * Key Designs 4: the calibrated masks become read-only skip lists, loaded onto the GPU before generation. */
calibatt_status calibatt_dict_create(int32_t T, int32_t L, int32_t H, int32_t nq, int32_t nk,
                                     int32_t block, int64_t nnz_capacity, int32_t num_ctas,
                                     calibatt_dict** out);

/* Like calibatt_dict_create, but each record stores one bit per (query
 * block, key block) instead of a 2-byte index per kept block: fixed
 * T*L*H*nq*ceil(nk/32)*4 bytes whatever the density (the 720p schedule of
 * 50 x 40 x 40 records: 3.6 GB instead of about 17 GB of index lists at
 * 20-60% density).  The tensor-core kernels decode each row into a list of
 * kept blocks in shared memory; results equal those of the list format.
 * Bitmap dictionaries serve the tensor-core path only (bf16, block 128;
 * otherwise the attention calls return CALIBATT_ERR_UNSUPPORTED) and hold
 * nq <= 2048.  All other dictionary functions apply unchanged.
 * Limitations & Future Work of the paper note: the 21.5 GB of mask memory
 * at Wan 720p, reducible to 3.6 GB, and compacting the skip lists. */
calibatt_status calibatt_dict_create_bitmap(int32_t T, int32_t L, int32_t H, int32_t nq,
                                            int32_t nk, int32_t block, int32_t num_ctas,
                                            calibatt_dict** out);

/* Like calibatt_dict_create, but each row's skip list is stored as its
 * contiguous key-block intervals, the encoding the paper note describes (Key
 * Designs 4: a read-only skip list of contiguous key-block intervals per
 * query block): one 32-bit word per interval (start | length << 16), plus a
 * second int32 [H][nq + 1] interval pointer per record.  run_capacity is the
 * total number of intervals the dictionary can hold (count them with
 * calibatt_csr_to_intervals).  The banded masks of calibration take a few
 * intervals per row, so the records take a small fraction of the bytes of
 * index lists.  The tensor-core producers expand each row's intervals into a
 * list of kept blocks in shared memory; results equal those of the list
 * format, bit for bit.  Interval dictionaries serve the tensor-core path only
 * (bf16, block 128; otherwise the attention calls return
 * CALIBATT_ERR_UNSUPPORTED) and hold nq <= 2048.  calibatt_dict_set_layer
 * takes the same CSR input and encodes it; calibatt_dict_info reports
 * retained blocks as for the other formats.
 * Key Designs 4 (interval-encoded skip lists); Limitations & Future Work of
 * the paper note (compacting the skip lists). */
calibatt_status calibatt_dict_create_intervals(int32_t T, int32_t L, int32_t H, int32_t nq,
                                               int32_t nk, int32_t block, int64_t run_capacity,
                                               int32_t num_ctas, calibatt_dict** out);

/* Fills the records of layer l at timestep t for all H heads (each layer
 * may be set once).  Host inputs:
 *   row_ptr int32[H][nq + 1]: each head's CSR row pointer, starting at 0;
 *   col_idx int32[...]: the heads' column lists concatenated in head order;
 *   repetitive uint8[H] (nullable = none): non-zero routes the head to the
 *     anchor path (Key Designs 3); its CSR must then be empty (row_ptr all 0).
 * Every CSR is validated as calibatt_csr_validate (no diagonal requirement),
 * converted to 16-bit indices, copied to the device (synchronously), and a
 * longest-processing-time schedule of the layer's (head, query block) work
 * is built for the dictionary's num_ctas: heads are taken in groups whose
 * keys and values fit in about 40 MB of L2, and the schedule keeps one
 * running LPT balance across the groups while listing each CTA's items group
 * by group, so the persistent CTAs work on the same few heads at a time. */
calibatt_status calibatt_dict_set_layer(calibatt_dict* dict, int32_t t, int32_t l,
                                        const int32_t* row_ptr, const int32_t* col_idx,
                                        const uint8_t* repetitive);

/* Records the anchor geometry of the dual path (Key Designs 3: anchor rows
 * of each frame, every other row served by its nearest anchor row, ties to
 * the lower one) so that every layer set afterwards also gets a joint
 * schedule of its block-sparse work items and the anchor-row tiles of its
 * repetitive heads.  calibatt_dual_path_attn then runs a layer in ONE
 * persistent launch when its call passes the same frames, rows, cols and
 * anchor rows, a bf16 shape and block 128 (otherwise two launches, as
 * without a geometry).  Host inputs: anchor_rows int32[n_anchors], strictly
 * ascending in [0, rows), 1 <= n_anchors <= 16; frames*rows*cols tokens must
 * make the dictionary's nq blocks.  Must be called at most once, before the
 * first calibatt_dict_set_layer; allocates the joint schedules on the device
 * (CALIBATT_ERR_CUDA if that fails).  CALIBATT_ERR_UNSUPPORTED for H > 32767
 * or more than 65535 anchor tiles per head. */
calibatt_status calibatt_dict_set_anchor_geometry(calibatt_dict* dict, int32_t frames, int32_t rows,
                                                  int32_t cols, const int32_t* anchor_rows,
                                                  int32_t n_anchors);

/* Totals: device bytes held, retained blocks stored, persistent grid size.
 * Bookkeeping; no counterpart in the paper note. */
calibatt_status calibatt_dict_info(const calibatt_dict* dict, int64_t* device_bytes,
                                   int64_t* nnz_total, int32_t* num_ctas);

/* Per-layer counts: heads on each path and retained (query, key) block tiles
 * of its sparse heads.  CALIBATT_ERR_INVALID_ARG if the layer is not set.
 * Bookkeeping; no counterpart in the paper note. */
calibatt_status calibatt_dict_layer_info(const calibatt_dict* dict, int32_t t, int32_t l,
                                         int32_t* n_sparse_heads, int32_t* n_repetitive_heads,
                                         int64_t* retained_tiles);

/* Frees the dictionary's device and host memory (synchronises the device).
 * Bookkeeping; no counterpart in the paper note. */
calibatt_status calibatt_dict_destroy(calibatt_dict* dict);

/* Checkpoint of the calibration output (the dictionary is the method's only
 * persistent artefact, computed offline and loaded before generation, Key
 * Designs 4).  Writes to `path` (replaced atomically: written to a temporary
 * name, then renamed) a little-endian file:
 *   header: "CALIBDCT", version 1, format (0 index lists, 1 bitmap, 2
 *     intervals), T, L, H, nq, nk, block, the anchor geometry if set,
 *     records stored, total stored units (retained blocks; intervals for
 *     format 2) (144 bytes);
 *   one entry per set record (t, l) in (t, l) order: t, l, stored units,
 *     the H repetitive flags, then the H CSR row pointers and the 16-bit
 *     block indices (index lists), the H*nq*ceil(nk/32) bitmap words, or the
 *     H CSR row pointers, the H interval pointers and the packed intervals,
 *     each part zero-padded to 8 bytes;
 *   trailer: "CALIBEND" and a 64-bit FNV-1a hash of every 8-byte word before
 *     it.
 * Schedules are not stored.  Copies the records from the device
 * (synchronously).  CALIBATT_ERR_INVALID_ARG if the file cannot be written
 * (the message names the cause). */
calibatt_status calibatt_dict_save(const calibatt_dict* dict, const char* path);

/* Reads a file written by calibatt_dict_save into a new dictionary of the
 * same format on the current device, rebuilding every record's schedules
 * for num_ctas persistent CTAs (<= 0: the device's SM count).  The header,
 * every record (through calibatt_dict_set_layer's validation), the record
 * order and counts, the padding and the trailing hash are checked;
 * CALIBATT_ERR_INVALID_ARG on any mismatch, a short file or trailing bytes,
 * and then no dictionary is returned.  Allocation failures as
 * calibatt_dict_create. */
calibatt_status calibatt_dict_load(const char* path, int32_t num_ctas, calibatt_dict** out);

/* ------------------------------------------------------- hot path */

/* Block-sparse attention for every non-repetitive head of record (t, l)
 * (Key Designs 4: non-repetitive heads skip unselected blocks and compute the
 * retained connections from the current input).  For query i of head h:
 *   O_i = softmax over keys j < N with M_h[floor(i/B), floor(j/B)] = 1 of
 *         (scale * q_i . k_j), weighting v_j;
 * a query block whose list is empty produces zeros.  q, k, v, o: device
 * arrays of `shape` (the output shares the input strides and dtype); only
 * heads routed to this path are written.  lse (nullable): device float32
 * [batch, heads, seq_len], receives ln(sum_j exp(scale * q_i . k_j)) over the
 * retained keys, -inf for empty lists.  shape->heads must equal the
 * dictionary's H and block its block size.
 * BF16 with block 128 runs the tensor-core kernel; other combinations run the
 * CUDA-core kernel (FP32 keeps float32 products). */
calibatt_status calibatt_block_sparse_attn(const void* q, const void* k, const void* v, void* o,
                                           const calibatt_shape* shape, int32_t block,
                                           const calibatt_dict* dict, int32_t t, int32_t l,
                                           float softmax_scale, float* lse, void* stream);

/* End-to-end form of calibatt_block_sparse_attn for inputs in host memory:
 * enqueues on `stream` the copies of q_host, k_host, v_host into the
 * caller-owned device buffers q, k, v, the attention (into device o), and the
 * copy of o into o_host; it does not synchronise.  Host and device tensors
 * share `shape` (dtype, strides); each copy moves the bytes from the tensor's
 * base to one past its last element.  Host buffers should be page-locked for
 * the copies to be asynchronous (they are then ordered on `stream` only);
 * callers may alternate streams and device buffer sets so that the copies of
 * one call overlap the attention of another.  Other arguments and errors as
 * calibatt_block_sparse_attn; a copy failure returns CALIBATT_ERR_CUDA.
 * Key Designs 4 (the operation of calibatt_block_sparse_attn). */
calibatt_status calibatt_block_sparse_attn_host(const void* q_host, const void* k_host,
                                                const void* v_host, void* o_host, void* q,
                                                void* k, void* v, void* o,
                                                const calibatt_shape* shape, int32_t block,
                                                const calibatt_dict* dict, int32_t t, int32_t l,
                                                float softmax_scale, float* lse, void* stream);

/* Work schedule of a direct-CSR call (calibatt_block_sparse_attn_csr), on the
 * host: one item (head << 16) | query_block per query block of every listed
 * head, placed on `grid` bins by longest-processing-time first (cost: the
 * block's retained key blocks + 2), heads taken in list order in groups whose
 * keys and values fit in L2 together, as the dictionary does per record.
 *   row_ptr: host int32[heads][nq + 1], each head's offsets starting at 0;
 *   head_ids: host int32[n_heads], distinct, in [0, heads), n_heads <= 128;
 *   items: host uint32[n_heads * nq]; cta_ptr: host int32[grid + 1], the
 *     items of CTA c are items[cta_ptr[c] .. cta_ptr[c+1]).
 * nq <= 65535, heads <= 65535.  CALIBATT_ERR_INVALID_ARG on a bad argument
 * or a decreasing row_ptr; column indices are not read.
 * No counterpart in the paper note: host scheduling for the persistent kernel. */
calibatt_status calibatt_csr_schedule(int32_t heads, int32_t nq, const int32_t* row_ptr,
                                      const int32_t* head_ids, int32_t n_heads, int32_t grid,
                                      uint32_t* items, int32_t* cta_ptr);

/* Block-sparse attention from skip lists the caller holds in device memory,
 * without a dictionary (same operation and outputs as
 * calibatt_block_sparse_attn, for the listed heads only; an all-ones list
 * gives dense attention):
 *   row_ptr: device int32[shape->heads][nq + 1], nq = ceil(seq_len / block),
 *     each head's offsets starting at 0;
 *   col_idx: device uint16, head h's list at col_idx + col_base[h], each row
 *     strictly ascending in [0, nq) (the rules calibatt_csr_validate checks);
 *   col_base: device int64[shape->heads];
 *     the caller guarantees that every listed head's lists lie inside the
 *     col_idx allocation (col_base[h] + row_ptr[h][nq] entries), which the
 *     library cannot see;
 *   head_ids: host int32[n_heads], distinct, in [0, heads), n_heads <= 128;
 *   items, cta_ptr, grid: the device copy of a calibatt_csr_schedule result
 *     for the same row_ptr and head_ids (used by the tensor-core kernel, BF16
 *     with block 128, which runs `grid` persistent CTAs; the CUDA-core
 *     kernel walks head_ids and ignores them, and they may then be NULL).
 * Device checks: the call does not read device arrays on the host.  Small
 * kernels check them on `stream` before the attention: row pointers start at
 * 0, do not decrease and hold at most nq blocks per row, block indices are
 * strictly ascending in [0, nq) (status code 23); every schedule item names a
 * listed head and a query block < nq, and cta_ptr runs from 0 to
 * n_heads * nq without decreasing (code 24).  The first violation is
 * recorded in the device status word (calibatt_device_status, low byte
 * CALIBATT_ERR_INVALID_ARG), and the attention kernels then return before
 * reading any list or writing any output -- in that call and in every later
 * direct-CSR call until the status word is read and cleared.
 * All device arrays are caller-owned and must stay valid until the call's
 * work on `stream` completes.  n_heads == 0 is a no-op.
 * Key Designs 4 (the operation of calibatt_block_sparse_attn). */
calibatt_status calibatt_block_sparse_attn_csr(const void* q, const void* k, const void* v, void* o,
                                               const calibatt_shape* shape, int32_t block,
                                               const int32_t* row_ptr, const uint16_t* col_idx,
                                               const int64_t* col_base, const int32_t* head_ids,
                                               int32_t n_heads, const uint32_t* items,
                                               const int32_t* cta_ptr, int32_t grid,
                                               float softmax_scale, float* lse, void* stream);

/* Anchor-row attention with broadcast for the given heads (Key Designs 3):
 * only queries of the anchor rows of every frame attend, densely over all N
 * keys and values; every token (f, row, col) takes the output of the anchor
 * row nearest to `row` in the same frame and column (distance ties go to the
 * lower anchor).  frames * rows * cols must equal shape->seq_len.
 *   anchor_rows: host int32[n_anchors], strictly ascending in [0, rows),
 *     1 <= n_anchors <= 16;
 *   head_ids: host int32[n_heads], distinct heads in [0, heads), n_heads <= 128.
 *   workspace: NULL, or caller-owned device scratch of at least
 *     calibatt_anchor_attn_workspace_size() bytes, 256-byte aligned.  With it
 *     (bf16) the last, partial wave of anchor tiles on the persistent grid is
 *     cut into key ranges that run on different SMs and are merged exactly
 *     (per-range maximum and row sum, float32 partial outputs, summed in
 *     range order by whichever SM finishes a tile's last range), so the grid
 *     ends together; the result is deterministic, and differs from the
 *     unsplit tiles' only by float32 rounding.  Without it every tile runs
 *     whole.  The call zeroes the workspace's counters on `stream`; calls in
 *     flight together need workspaces of their own.  A workspace smaller
 *     than this call's need is CALIBATT_ERR_INVALID_ARG.
 * Every token of the listed heads is written. */
calibatt_status calibatt_anchor_attn(const void* q, const void* k, const void* v, void* o,
                                     const calibatt_shape* shape, int32_t block,
                                     int32_t frames, int32_t rows, int32_t cols,
                                     const int32_t* anchor_rows, int32_t n_anchors,
                                     const int32_t* head_ids, int32_t n_heads,
                                     float softmax_scale, void* workspace,
                                     size_t workspace_bytes, void* stream);

/* Device scratch bytes calibatt_anchor_attn uses to split its last wave of
 * tiles, for `shape` and n_heads listed heads on the current device (its SM
 * count sizes the persistent grid); 0 when the call would not split (no
 * partial wave, fewer than four key blocks, or float32 inputs).  The
 * workspace holds, per split tile and key range, 128 x head_dim float32
 * partial outputs and 256 (maximum, row sum) pairs (one per row and output
 * column half), and 8 counters per split tile.  No counterpart in the pages: a scheduling device of this
 * implementation (Key Designs 3 defines the operation). */
calibatt_status calibatt_anchor_attn_workspace_size(const calibatt_shape* shape, int32_t frames,
                                                    int32_t rows, int32_t cols, int32_t n_anchors,
                                                    int32_t n_heads, size_t* bytes);

/* The split plan calibatt_anchor_attn follows (host only, no device):
 * `tiles` equal anchor tiles on `grid` persistent CTAs leave r = tiles mod
 * grid tiles in a last partial wave; each is cut into `parts` key ranges,
 * parts in 1..4 minimising ceil(r * parts / grid) / parts (the smallest on
 * ties, each range at least two of the key_blocks blocks).  The split tiles
 * are the last r of the call's sequence (batch, then listed head, then
 * tile): *first = tiles - r, or *first = tiles and *parts = 1 when nothing is
 * split.  No counterpart in the pages. */
calibatt_status calibatt_anchor_split_plan(int64_t tiles, int32_t grid, int32_t key_blocks,
                                           int64_t* first, int32_t* parts);

/* Both paths of record (t, l): the dictionary's repetitive heads through the
 * anchor path and the rest through the block-sparse path, enqueued on one
 * stream (Key Designs 4: the repetition flag selects one path per head; the
 * paths are alternatives, never stacked).  Arguments as above; lse
 * (nullable) is written for the sparse heads only.  With a matching
 * calibatt_dict_set_anchor_geometry (bf16, block 128) both kinds of work run
 * in one persistent launch under the layer's joint schedule; otherwise as
 * calibatt_block_sparse_attn followed by calibatt_anchor_attn. */
calibatt_status calibatt_dual_path_attn(const void* q, const void* k, const void* v, void* o,
                                        const calibatt_shape* shape, int32_t block,
                                        const calibatt_dict* dict, int32_t t, int32_t l,
                                        int32_t frames, int32_t rows, int32_t cols,
                                        const int32_t* anchor_rows, int32_t n_anchors,
                                        float softmax_scale, float* lse, void* stream);

/* ------------------------------------------------ offline calibration */

/* Device scratch bytes calibatt_block_energy needs for `shape`.
 * Key Designs 1, Eq. (5): the workspace of calibatt_block_energy. */
calibatt_status calibatt_block_energy_workspace_size(const calibatt_shape* shape,
                                                     size_t* bytes);

/* Block energies (Key Designs 1, Eq. (5)) of the dense, unmasked attention:
 *   E[b, h, r, c] = (1/|I_r|) * sum_{i in I_r} sum_{j in J_c} P_ij
 * with |I_r| the valid queries of block r (B for full blocks), so every row
 * of E sums to one.  energy: device float32 [batch, heads, nb, nb].
 * workspace: caller-owned device scratch of at least
 * calibatt_block_energy_workspace_size() bytes (row log-sum-exp values).
 * bf16 inputs with block 128 run on the tensor cores (the attention
 * pipeline without V: a log-sum-exp pass, then the energy pass); other cases
 * on CUDA cores in float32.  Both sum in fixed orders, so repeated calls give
 * bitwise identical energies. */
calibatt_status calibatt_block_energy(const void* q, const void* k,
                                      const calibatt_shape* shape, int32_t block,
                                      float softmax_scale, float* energy, void* workspace,
                                      size_t workspace_bytes, void* stream);

/* The same block energies as calibatt_block_energy, for callers that may not
 * allocate device memory (the paper has no counterpart; this is a deployment
 * variant).  Some processes cannot call cudaMalloc when they calibrate: a
 * server that reserved all device memory at start-up for weights and caches,
 * a host runtime that owns the allocator and forbids plug-ins to go around
 * it, or an integration whose host code may not call the CUDA memory API.
 * This entry point allocates nothing: its row log-sum-exp scratch is a fixed
 * array inside the library, 2^20 float32 rows (4 MiB, held on every GPU that
 * loads the library until the process exits), so batch * heads * seq_len
 * must not exceed 2^20 (CALIBATT_ERR_INVALID_ARG otherwise, with a message;
 * use calibatt_block_energy and a caller workspace for larger problems).
 * All calls share that array and it keeps the previous call's contents
 * (nothing in it needs clearing: every row is written before it is read);
 * calls whose work overlaps on the GPU race on it, so order them on one
 * stream.  The first call on each device looks up the array's device address
 * with that device current; make that first call before capturing any
 * stream.  Other arguments and errors as calibatt_block_energy. */
calibatt_status calibatt_block_energy_noalloc(const void* q, const void* k,
                                              const calibatt_shape* shape, int32_t block,
                                              float softmax_scale, float* energy, void* stream);

/* Top-mass selection (Key Designs 1, after Eq. (5)) for n_rows rows of nk
 * energies (device float32 [n_rows, nk], nk <= 4096): order each row by
 * energy descending, ties to the lower key block; keep the shortest prefix
 * whose cumulative mass, summed in float64 in that order, is >= tau (as
 * float64); keep every block if none is.  mask: device uint8 [n_rows, nk]
 * (1 = kept).  count_accum (nullable): device int32 [n_rows, nk], incremented
 * by the mask (for cross-prompt aggregation). */
calibatt_status calibatt_select_blocks(const float* energy, int64_t n_rows, int32_t nk,
                                       float tau, uint8_t* mask, int32_t* count_accum,
                                       void* stream);

/* Cross-prompt aggregation (Key Designs 2, Eq. (8)-(9)): mask[i] =
 * (counts[i] / n_prompts >= rho), evaluated in float64 with rho widened from
 * float.  counts: device int32[n]; mask: device uint8[n]. */
calibatt_status calibatt_aggregate_masks(const int32_t* counts, int64_t n, int32_t n_prompts,
                                         float rho, uint8_t* mask, void* stream);

/* Spatial-repetition score (Key Designs 3) of every spatial row of every
 * head: with tokens ordered (frame, row, column), frames * rows * cols ==
 * seq_len, and a*(rho) the anchor row nearest to row rho (ties to the lower
 * anchor), the cosine similarity of the flattened post-softmax attention of
 * the row's cols queries over all keys and that of a*(rho)'s cols queries
 * (same frame, same columns):
 *   sim[b, h, f, rho] = sum_w <P[(f,rho,w)], P[(f,a,w)]>
 *                       / sqrt(sum_w |P[(f,rho,w)]|^2 * sum_w |P[(f,a,w)]|^2)
 * with P the dense, unmasked softmax of scale * q.k.  Anchor rows score one.
 * similarity: device float32 [batch, heads, frames, rows].  workspace:
 * caller-owned device scratch of at least
 * calibatt_spatial_similarity_workspace_size bytes.  anchor_rows: host int32,
 * strictly ascending in [0, rows), 1..16 of them; rows <= 256.  BF16 inputs
 * run on the tensor cores (q and k 16-byte aligned): a pass of each query's
 * log-sum-exp, then a pass that pairs every 128-query tile with the gathered
 * tile of its partner queries in the nearest anchor row and accumulates, key
 * block by key block, each query's sums of P P', P^2 and P'^2 (float32), then
 * a fixed-order sum over each row's cols queries.  FP32 inputs run on CUDA
 * cores in float32.  Both use fixed summation orders (bitwise repeatable). */
/* Device scratch bytes calibatt_spatial_similarity needs for `shape`: one
 * float per query (its log-sum-exp), four on the tensor-core path (BF16: the
 * log-sum-exp and three per-query sums).
 * Key Designs 3: the workspace of calibatt_spatial_similarity. */
calibatt_status calibatt_spatial_similarity_workspace_size(const calibatt_shape* shape,
                                                           size_t* bytes);

calibatt_status calibatt_spatial_similarity(const void* q, const void* k,
                                            const calibatt_shape* shape, int32_t frames,
                                            int32_t rows, int32_t cols,
                                            const int32_t* anchor_rows, int32_t n_anchors,
                                            float softmax_scale, float* similarity,
                                            void* workspace, size_t workspace_bytes,
                                            void* stream);

/* Repetition flags (Key Designs 3): for each of n_heads heads, the mean of
 * its per_head similarities over n_prompts calibration prompts (similarity:
 * device float32 [n_prompts][n_heads][per_head], e.g. per_head = frames *
 * rows of calibatt_spatial_similarity and n_heads = batch * heads), summed in
 * float64 in a fixed order; flags[h] = 1 when the mean is strictly greater
 * than threshold (the page's default is 0.87).  mean (nullable): device
 * float32 [n_heads]; flags: device uint8 [n_heads]. */
calibatt_status calibatt_repetition_flags(const float* similarity, int32_t n_prompts,
                                          int32_t n_heads, int32_t per_head, float threshold,
                                          float* mean, uint8_t* flags, void* stream);

/* ------------------------------------------------------- diagnostics */

/* Synchronises `stream`, then reports the device status word and optionally
 * clears it.  The kernels set it (first event wins) when a bounded wait runs
 * out (CALIBATT_ERR_TIMEOUT in the low byte, the waiting role and barrier
 * above it) or when a skip list the host never read breaks the list rules
 * (CALIBATT_ERR_INVALID_ARG in the low byte; 23 and 24: the device-side
 * checks of lists and schedule that calibatt_block_sparse_attn_csr runs
 * before its attention kernel, which then skips its work; 22: the CUDA-core
 * kernel met a block index >= nq and skipped that block).  Returns
 * the low byte's status when the word is non-zero.
 * Diagnostics; no counterpart in the paper note. */
calibatt_status calibatt_device_status(void* stream, int32_t* code, int32_t clear);

/* Failure-path check of the bounded waits: launches one warp that waits on
 * an mbarrier nothing arrives on, through the same bounded wait the kernels
 * use, with the current calibatt_set_wait_timeout_ms limit.  When the limit
 * passes it sets the status word (CALIBATT_ERR_TIMEOUT, wait point 15 in the
 * byte above it) and returns; no fault, no hang, the context stays usable.
 * Read the result with calibatt_device_status.
 * Diagnostics; no counterpart in the paper note. */
calibatt_status calibatt_debug_bounded_wait(void* stream);

/* Evaluates, on the device, the FMA-pipe base-2 exponential that the
 * tensor-core softmax uses for part of its probabilities (no counterpart in
 * the paper; exposed so its error bound can be tested): y[i] = 2^x[i] with
 * relative error below 1e-4 for -125 <= x <= 126, about 2^-125 for smaller x.
 * x, y: device float32[n]. */
calibatt_status calibatt_debug_exp2_fma(const float* x, float* y, int64_t n, void* stream);

/* The same for the quintic FMA-pipe exponential that the offline energy
 * passes use for a quarter of their exponentials: relative error below 3e-7
 * (the fit's 7.5e-8 plus float32 evaluation) for -125 <= x <= 126, about
 * 2^-125 for smaller x.  x, y: device float32[n].
 * No counterpart in the paper note (exposed so its error bound can be tested). */
calibatt_status calibatt_debug_exp2_fma_quintic(const float* x, float* y, int64_t n, void* stream);

/* Time limit of every in-kernel barrier wait, in milliseconds (default 4000;
 * applies to launches made after the call).
 * Diagnostics; no counterpart in the paper note. */
calibatt_status calibatt_set_wait_timeout_ms(int32_t ms);

/* Number of SMs of the current device (the default persistent grid size).
 * No counterpart in the paper note. */
calibatt_status calibatt_device_sm_count(int32_t* out);

#ifdef __cplusplus
}
#endif

#endif /* CALIBATT_H_ */
