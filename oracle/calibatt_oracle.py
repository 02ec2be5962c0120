"""CPU oracle for the CalibAtt inference hot path.  TEST INFRASTRUCTURE ONLY.

This module is the slow, plain, float64 statement of what the GPU library
computes.  Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
``cpu_baseline`` / ``--impl reference`` legs may import it.  The product
package ``calibrated_block_sparse_calibatt_b200`` never imports it, and it
imports nothing from the product: the two share no code.

Source of every definition: the paper note "Accelerating Text-to-Video
Generation with Calibrated Sparse Attention" (papernotes.org, ECCV2026 entry),
section "Method" -> "Key Designs" 1-4 and "A Worked Example".  Citations below
name the section and equation of that page.

Notation follows the page: P is post-softmax attention, I_r and J_c are the
query and key token sets of block r and c, B the block side, E_{r,c} the block
energy, M_p the per-prompt binary mask, M-bar the keep frequency, rho the
agreement threshold, tau the energy threshold, k the anchor count.

Readings taken where the page is silent:
  * softmax scale defaults to 1/sqrt(D);
  * tokens are ordered frame-major, then spatial row, then column;
  * keys at index >= N (padding) are excluded and padded queries are not
    produced;
  * E_{r,c} divides by |I_r| (the number of valid queries of block r), which is
    B for full blocks and makes each q-block's energies sum to one, the
    property the page states after Eq. (5);
  * the prefix "reaches" tau means cumulative mass >= tau, summed in float64 in
    sorted order; equal energies are ordered by lower key-block index first;
  * a q-block with no retained key block produces O = 0 and LSE = -inf;
  * the nearest anchor of a spatial row breaks distance ties toward the lower
    anchor row.

Pins (tests/test_oracle_pins.py, run with ``-m "not gpu"``):
  attention_rows / block_sparse_attention:
      all-ones mask == torch scaled_dot_product_attention (float64);
      diagonal-only mask == explicit per-block loops on a tiny case;
      constant keys == mean of the retained value rows (closed form);
      one query over two keys == the two-term softmax closed form;
      empty row == zeros and LSE = -inf.
  attention_probabilities: rows sum to one.
  block_sparse_attention_bnhd, anchor_attention_bnhd, block_energy_bnhd:
      every (batch, head) slice equals the one-head function on explicitly
      sliced inputs whose heads and batches differ in scale; the anchor and
      energy wrappers also equal torch's batched SDPA / softmax over
      [batch, heads, N, D] (gathered or block-summed outside the oracle).
  anchor_attention / nearest_anchor_rows:
      nearest-anchor tables of the tiny and 720p layouts
      (tests/golden/nearest_anchor_tables.json);
      anchor rows == SDPA rows, other rows copy their anchor;
      query reduction HW -> kW, sparsity 1 - k/H
      (tests/golden/anchor_query_reduction.json).
  block_energy: rows sum to one; constant keys give |J_c|/N; double-loop brute
      force on a tiny ragged case.
  select_blocks: exhaustive subset search on tiny cases (minimal size,
      canonical set).
  aggregate_masks: the worked example of the page, 64 prompts at rho = 0.5
      keep a block selected 32 times and drop one selected 31 times
      (tests/golden/aggregation_worked_example.json).
  spatial_similarity / repetition_flags: anchor rows score exactly one;
      frames whose rows repeat the anchor queries score one; rows attending
      to disjoint keys score zero; a two-key closed form; a double-loop brute
      force over (column, key) on a tiny case; Cauchy-Schwarz bounds; the
      flag is the strict "exceeds" of the mean over prompts, frames and rows.

Readings for the spatial-repetition branch (Key Designs 3):
  * the attention "associated with a spatial row" is the post-softmax rows of
    that row's W queries over all N keys, concatenated in column order into
    one W*N vector; the nearest anchor row's vector is built the same way
    from its W queries (the same columns);
  * the mean runs over every spatial row of every frame, anchor rows
    included (they score one), and over the calibration prompts;
  * a head is repetitive when the mean is strictly greater than the
    threshold (0.87 by default).
"""

from __future__ import annotations

import math

import numpy as np

__all__ = [
    "default_scale",
    "attention_rows",
    "attention_probabilities",
    "block_sparse_attention",
    "block_sparse_attention_bnhd",
    "nearest_anchor_rows",
    "anchor_source_tokens",
    "anchor_attention",
    "anchor_attention_bnhd",
    "block_energy",
    "block_energy_bnhd",
    "select_blocks",
    "aggregate_masks",
    "attention_probability_rows",
    "spatial_similarity",
    "repetition_flags",
    "num_blocks",
]


def default_scale(head_dim: int) -> float:
    """Softmax scale 1/sqrt(D); the page does not state one."""
    return 1.0 / math.sqrt(head_dim)


def num_blocks(seq_len: int, block: int) -> int:
    """Number of B-token blocks covering N tokens (last block may be partial)."""
    return (seq_len + block - 1) // block


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def attention_rows(q_rows, k, v, seq_len, scale, allowed=None):
    """Softmax attention of the given query rows over keys 0..N-1.

    q_rows: [n, D]; k, v: [>=N, D]; allowed: optional bool [n, N] saying which
    (query, key) interactions are computed (the rest get score -inf).
    Returns (O [n, D], LSE [n]) with LSE the natural log of the softmax
    denominator of the scaled scores.  A row with no allowed key returns O = 0
    and LSE = -inf.
    """
    q_rows = _f64(q_rows)
    kk = _f64(k)[:seq_len]
    vv = _f64(v)[:seq_len]
    s = scale * (q_rows @ kk.T)
    if allowed is not None:
        s = np.where(allowed, s, -np.inf)
    m = s.max(axis=1)
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    p = np.exp(s - m_safe[:, None])
    p[empty] = 0.0
    l = p.sum(axis=1)
    o = (p @ vv) / np.where(empty, 1.0, l)[:, None]
    o[empty] = 0.0
    lse = np.where(empty, -np.inf, m_safe + np.log(np.where(empty, 1.0, l)))
    return o, lse


def attention_probabilities(q, k, seq_len, scale):
    """Dense post-softmax attention P [N, N] over the N valid tokens (Key Designs 1)."""
    qq = _f64(q)[:seq_len]
    kk = _f64(k)[:seq_len]
    s = scale * (qq @ kk.T)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    return p / p.sum(axis=1, keepdims=True)


def block_sparse_attention(q, k, v, block_mask, block, seq_len=None, scale=None,
                           rows=None, chunk=256):
    """Block-sparse attention of one head (Key Designs 4: retained connections use
    the current input's queries, keys and values; unselected blocks are skipped).

    Written as dense float64 attention in which every (query i, key j) pair whose
    block pair (floor(i/B), floor(j/B)) is not retained scores -inf.

    q, k, v: [>=N, D]; block_mask: bool [nq, nk] with nq = nk = ceil(N/B).
    rows: query indices to evaluate (default all N).  Returns (O, LSE).
    """
    q = _f64(q)
    n = q.shape[0] if seq_len is None else int(seq_len)
    d = q.shape[1]
    scale = default_scale(d) if scale is None else float(scale)
    mask = np.asarray(block_mask, dtype=bool)
    nb = num_blocks(n, block)
    if mask.shape != (nb, nb):
        raise ValueError(f"block mask shape {mask.shape} != ({nb}, {nb})")
    rows = np.arange(n) if rows is None else np.asarray(rows, dtype=np.int64)
    key_block = np.arange(n) // block
    out = np.zeros((len(rows), d))
    lse = np.zeros(len(rows))
    for s0 in range(0, len(rows), chunk):
        rr = rows[s0:s0 + chunk]
        allowed = mask[rr // block][:, key_block]
        o, l = attention_rows(q[rr], k, v, n, scale, allowed)
        out[s0:s0 + chunk] = o
        lse[s0:s0 + chunk] = l
    return out, lse


def block_sparse_attention_bnhd(q, k, v, masks, block, seq_len=None, scale=None,
                                heads=None, rows=None):
    """block_sparse_attention over tensors laid out [batch, N, H, D].

    masks: sequence indexed by head of bool [nq, nk].  heads: heads to evaluate
    (default all).  Returns O [batch, len(rows), len(heads), D] and LSE
    [batch, len(heads), len(rows)].
    """
    q = _f64(q)
    b_, n_alloc, h_, d = q.shape
    n = n_alloc if seq_len is None else int(seq_len)
    heads = list(range(h_)) if heads is None else list(heads)
    rows = np.arange(n) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.zeros((b_, len(rows), len(heads), d))
    lse = np.zeros((b_, len(heads), len(rows)))
    for b in range(b_):
        for hi, h in enumerate(heads):
            o, l = block_sparse_attention(q[b, :, h], _f64(k[b, :, h]), _f64(v[b, :, h]),
                                          masks[h], block, n, scale, rows)
            out[b, :, hi] = o
            lse[b, hi] = l
    return out, lse


def nearest_anchor_rows(rows_per_frame: int, anchors) -> np.ndarray:
    """For each spatial row rho in 0..R-1, the anchor row nearest to it
    (Key Designs 3: each anchor's output goes to its nearest spatial rows within
    the frame).  Distance ties go to the lower anchor row."""
    anchors = sorted(int(a) for a in anchors)
    if not anchors:
        raise ValueError("at least one anchor row is required")
    out = np.empty(rows_per_frame, dtype=np.int64)
    for rho in range(rows_per_frame):
        best = anchors[0]
        for a in anchors[1:]:
            if abs(rho - a) < abs(rho - best):
                best = a
        out[rho] = best
    return out


def anchor_source_tokens(frames, rows_per_frame, cols, anchors, tokens=None):
    """Token whose query produces the output of each token under the anchor path.

    Token i = f*R*C + rho*C + w is served by the anchor query
    f*R*C + a*(rho)*C + w: same frame, same column, nearest anchor row."""
    n = frames * rows_per_frame * cols
    tokens = np.arange(n) if tokens is None else np.asarray(tokens, dtype=np.int64)
    near = nearest_anchor_rows(rows_per_frame, anchors)
    f = tokens // (rows_per_frame * cols)
    rho = (tokens % (rows_per_frame * cols)) // cols
    w = tokens % cols
    return f * rows_per_frame * cols + near[rho] * cols + w


def anchor_attention(q, k, v, frames, rows_per_frame, cols, anchors, scale=None,
                     rows=None):
    """Anchor-row attention with output broadcast, one head (Key Designs 3 and 4).

    Only anchor-row queries attend, against all N keys and values with no block
    mask; every other token takes the output of its nearest anchor row in the
    same frame and column.  Returns (O [len(rows), D], LSE of the serving anchor).
    """
    q = _f64(q)
    n = frames * rows_per_frame * cols
    d = q.shape[1]
    scale = default_scale(d) if scale is None else float(scale)
    rows = np.arange(n) if rows is None else np.asarray(rows, dtype=np.int64)
    src = anchor_source_tokens(frames, rows_per_frame, cols, anchors, rows)
    return attention_rows(q[src], k, v, n, scale, None)


def anchor_attention_bnhd(q, k, v, frames, rows_per_frame, cols, anchors, scale=None,
                          heads=None, rows=None):
    """anchor_attention over [batch, N, H, D] tensors; output [batch, rows, heads, D]."""
    q = _f64(q)
    b_, _, h_, d = q.shape
    n = frames * rows_per_frame * cols
    heads = list(range(h_)) if heads is None else list(heads)
    rows = np.arange(n) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.zeros((b_, len(rows), len(heads), d))
    for b in range(b_):
        for hi, h in enumerate(heads):
            o, _ = anchor_attention(q[b, :, h], _f64(k[b, :, h]), _f64(v[b, :, h]),
                                    frames, rows_per_frame, cols, anchors, scale, rows)
            out[b, :, hi] = o
    return out


def block_energy(q, k, block, seq_len=None, scale=None):
    """Block energies of one head (Key Designs 1, Eq. (5)).

    E_{r,c} = (1/|I_r|) * sum_{i in I_r} sum_{j in J_c} P_ij with P the dense,
    unmasked post-softmax attention over the N valid tokens, and |I_r| the number
    of valid queries of block r (B for a full block).  Returns float64 [nq, nk].
    """
    q = _f64(q)
    n = q.shape[0] if seq_len is None else int(seq_len)
    d = q.shape[1]
    scale = default_scale(d) if scale is None else float(scale)
    p = attention_probabilities(q, k, n, scale)
    nb = num_blocks(n, block)
    e = np.zeros((nb, nb))
    for r in range(nb):
        i_r = slice(r * block, min(n, (r + 1) * block))
        size_r = i_r.stop - i_r.start
        for c in range(nb):
            j_c = slice(c * block, min(n, (c + 1) * block))
            e[r, c] = p[i_r, j_c].sum() / size_r
    return e


def block_energy_bnhd(q, k, block, seq_len=None, scale=None):
    """block_energy for every (batch, head) of [batch, N, H, D] tensors -> [batch, H, nq, nk]."""
    q = _f64(q)
    b_, n_alloc, h_, _ = q.shape
    n = n_alloc if seq_len is None else int(seq_len)
    nb = num_blocks(n, block)
    out = np.zeros((b_, h_, nb, nb))
    for b in range(b_):
        for h in range(h_):
            out[b, h] = block_energy(q[b, :, h], _f64(k[b, :, h]), block, n, scale)
    return out


def select_blocks(energy, tau):
    """Top-mass block selection per q-block (Key Designs 1, after Eq. (5)).

    For each row r of E: order the key blocks by energy descending (equal
    energies: lower index first), keep the shortest prefix whose cumulative mass,
    accumulated in float64 in that order, is >= tau, and map the kept blocks back
    to their original positions.  If no prefix reaches tau every block is kept.
    energy: [..., nq, nk]; returns bool of the same shape.
    """
    e = _f64(energy)
    tau = float(tau)
    flat = e.reshape(-1, e.shape[-1])
    nk = flat.shape[1]
    out = np.zeros(flat.shape, dtype=bool)
    idx = np.arange(nk)
    for r in range(flat.shape[0]):
        order = np.lexsort((idx, -flat[r]))
        cum = np.add.accumulate(flat[r, order])
        reached = np.nonzero(cum >= tau)[0]
        kstar = int(reached[0]) + 1 if len(reached) else nk
        out[r, order[:kstar]] = True
    return out.reshape(e.shape)


def aggregate_masks(masks_or_counts, n_prompts, rho):
    """Cross-prompt aggregation (Key Designs 2, Eq. (8) and Eq. (9)).

    M-bar = (1/|D|) * sum_p M_p (the keep frequency), M = 1[M-bar >= rho],
    evaluated in float64.  Accepts either the stacked masks [|D|, ...] (bool) or
    the per-block selection counts (integers) with n_prompts = |D|.
    """
    a = np.asarray(masks_or_counts)
    if a.dtype == bool:
        if a.shape[0] != n_prompts:
            raise ValueError("stacked masks must have |D| on axis 0")
        counts = a.sum(axis=0, dtype=np.int64)
    else:
        counts = a.astype(np.int64)
    mbar = counts.astype(np.float64) / float(n_prompts)
    return mbar >= float(rho)


# ------------------------------------------------------ spatial repetition

def attention_probability_rows(q_rows, k, seq_len, scale):
    """Post-softmax attention rows P[i, :] of the given queries over keys 0..N-1."""
    qq = _f64(q_rows)
    kk = _f64(k)[:seq_len]
    s = scale * (qq @ kk.T)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    return p / p.sum(axis=1, keepdims=True)


def spatial_similarity(q, k, frames, rows_per_frame, cols, anchors, scale=None, only=None):
    """Spatial-repetition score of one head (Key Designs 3): for every frame f
    and spatial row rho, the cosine similarity between the flattened attention
    of the row's W = cols queries and that of the nearest anchor row's W
    queries (same frame, same columns):

        v(f, rho) = [P[(f, rho, 0), :], ..., P[(f, rho, W-1), :]]   (length W*N)
        sim(f, rho) = <v(f, rho), v(f, a*(rho))> / (|v(f, rho)| |v(f, a*(rho))|)

    q, k: [>= N, D] with N = frames * rows * cols.  only: optional list of
    (f, rho) to evaluate (the others are NaN).  Returns float64 [frames, rows]."""
    n = frames * rows_per_frame * cols
    q = _f64(q)
    scale = default_scale(q.shape[1]) if scale is None else float(scale)
    near = nearest_anchor_rows(rows_per_frame, anchors)
    pairs = [(f, r) for f in range(frames) for r in range(rows_per_frame)] if only is None else list(only)
    out = np.full((frames, rows_per_frame), np.nan)
    for f, rho in pairs:
        base = f * rows_per_frame * cols
        a = int(near[rho])
        pr = attention_probability_rows(q[base + rho * cols: base + (rho + 1) * cols], k, n, scale)
        pa = attention_probability_rows(q[base + a * cols: base + (a + 1) * cols], k, n, scale)
        out[f, rho] = float(np.sum(pr * pa) / math.sqrt(float(np.sum(pr * pr)) * float(np.sum(pa * pa))))
    return out


def repetition_flags(similarities, threshold=0.87):
    """Per-head repetition decision (Key Designs 3): the mean of the spatial
    similarities over calibration prompts, frames and rows, and whether it
    exceeds the threshold.  similarities: [prompts, heads, frames, rows].
    Returns (mean float64 [heads], flag bool [heads])."""
    s = _f64(similarities)
    mean = s.reshape(s.shape[0], s.shape[1], -1).mean(axis=(0, 2))
    return mean, mean > float(threshold)
