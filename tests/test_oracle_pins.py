"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test fixes one function of oracle/calibatt_oracle.py to a library routine,
a closed form, a brute-force enumeration or a value stated by the paper note
"Accelerating Text-to-Video Generation with Calibrated Sparse Attention".
"""

import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import calibatt_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rand(seed, *shape, std=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * std


# ---------------------------------------------------------------- attention

@pytest.mark.parametrize("n,block,d", [(37, 8, 16), (64, 16, 8), (100, 32, 64)])
def test_all_ones_mask_equals_sdpa(n, block, d):
    q, k, v = (_rand(s, n, d) for s in (1, 2, 3))
    nb = O.num_blocks(n, block)
    o, lse = O.block_sparse_attention(q, k, v, np.ones((nb, nb), bool), block)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None])[0]
    np.testing.assert_allclose(o, ref.numpy(), rtol=0, atol=1e-12)
    ref_lse = torch.logsumexp(torch.from_numpy(q) @ torch.from_numpy(k).T / math.sqrt(d), dim=1)
    np.testing.assert_allclose(lse, ref_lse.numpy(), rtol=0, atol=1e-12)


def test_diagonal_only_mask_matches_bruteforce_loops():
    n, block, d = 21, 8, 4          # ragged: last block has 5 tokens
    q, k, v = (_rand(s, n, d) for s in (4, 5, 6))
    nb = O.num_blocks(n, block)
    o, _ = O.block_sparse_attention(q, k, v, np.eye(nb, dtype=bool), block, scale=0.7)
    for i in range(n):
        r = i // block
        keys = [j for j in range(n) if j // block == r]
        scores = []
        for j in keys:
            acc = 0.0
            for t in range(d):
                acc += q[i, t] * k[j, t]
            scores.append(0.7 * acc)
        mx = max(scores)
        w = [math.exp(s - mx) for s in scores]
        tot = sum(w)
        for t in range(d):
            expect = sum(w[a] * v[keys[a], t] for a in range(len(keys))) / tot
            assert abs(o[i, t] - expect) < 1e-12


def test_constant_keys_give_mean_of_retained_values():
    n, block, d = 50, 16, 8
    q = _rand(7, n, d, std=3.0)
    k = np.tile(_rand(8, 1, d), (n, 1))
    v = _rand(9, n, d)
    nb = O.num_blocks(n, block)
    mask = np.random.default_rng(10).random((nb, nb)) < 0.5
    mask[np.arange(nb), np.arange(nb)] = True
    o, _ = O.block_sparse_attention(q, k, v, mask, block)
    for i in range(n):
        keep = [j for j in range(n) if mask[i // block, j // block]]
        np.testing.assert_allclose(o[i], v[keep].mean(axis=0), rtol=0, atol=1e-12)


def test_one_query_two_keys_closed_form():
    d = 4
    q = np.array([[1.0, -2.0, 0.5, 3.0]])
    k = np.array([[0.5, 1.0, -1.0, 2.0], [-1.0, 0.0, 2.0, 1.0]])
    v = np.array([[1.0, 2.0, 3.0, 4.0], [-4.0, 0.0, 8.0, 1.0]])
    s1 = (0.5 - 2.0 - 0.5 + 6.0) / 2.0     # q.k1 / sqrt(4)
    s2 = (-1.0 + 0.0 + 1.0 + 3.0) / 2.0
    w1 = 1.0 / (1.0 + math.exp(s2 - s1))
    expect = w1 * v[0] + (1 - w1) * v[1]
    o, lse = O.attention_rows(q, k, v, 2, 1.0 / math.sqrt(d))
    np.testing.assert_allclose(o[0], expect, rtol=0, atol=1e-14)
    assert abs(lse[0] - math.log(math.exp(s1) + math.exp(s2))) < 1e-14


def test_empty_row_gives_zero_output_and_minus_inf_lse():
    n, block, d = 32, 8, 4
    q, k, v = (_rand(s, n, d) for s in (11, 12, 13))
    mask = np.eye(4, dtype=bool)
    mask[2, 2] = False
    o, lse = O.block_sparse_attention(q, k, v, mask, block)
    assert np.all(o[16:24] == 0.0)
    assert np.all(np.isneginf(lse[16:24]))
    assert np.all(np.isfinite(lse[:16]))


def test_padding_rows_beyond_seq_len_are_never_read():
    n, block, d = 40, 16, 8
    q, k, v = (_rand(s, 48, d) for s in (14, 15, 16))
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    for t in (q2, k2, v2):
        t[n:] = np.nan
    nb = O.num_blocks(n, block)
    m = np.ones((nb, nb), bool)
    o1, _ = O.block_sparse_attention(q, k, v, m, block, seq_len=n)
    o2, _ = O.block_sparse_attention(q2, k2, v2, m, block, seq_len=n)
    np.testing.assert_array_equal(o1, o2)


def test_probability_rows_sum_to_one():
    n, d = 77, 16
    q, k = _rand(17, n, d, std=2.0), _rand(18, n, d, std=2.0)
    p = O.attention_probabilities(q, k, n, 0.25)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    assert np.all(p >= 0)


def test_bnhd_wrapper_indexes_heads_and_batches():
    b, n, h, d, block = 2, 24, 3, 8, 8
    q, k, v = (_rand(s, b, n, h, d) for s in (19, 20, 21))
    rng = np.random.default_rng(22)
    masks = [rng.random((3, 3)) < 0.6 for _ in range(h)]
    for m in masks:
        m[np.arange(3), np.arange(3)] = True
    out, _ = O.block_sparse_attention_bnhd(q, k, v, masks, block)
    for bi in range(b):
        for hi in range(h):
            ref, _ = O.block_sparse_attention(q[bi, :, hi], k[bi, :, hi], v[bi, :, hi],
                                              masks[hi], block)
            np.testing.assert_array_equal(out[bi, :, hi], ref)


def _distinct_heads(seed, b, n, h, d):
    """[b, n, h, d] draws whose heads and batches differ in scale as well as in
    values, so that an exchanged (batch, head) slice changes every result."""
    x = _rand(seed, b, n, h, d)
    for bi in range(b):
        for hi in range(h):
            x[bi, :, hi] *= 0.5 + 0.6 * hi + 0.25 * bi
    return x


def test_anchor_bnhd_wrapper_indexes_heads_and_batches():
    """anchor_attention_bnhd on batch 2, 3 heads, a head subset in reverse
    order and a row subset, against (1) the one-head function on explicitly
    sliced inputs and (2) torch's batched SDPA over [batch, heads, N, D]
    followed by a gather of each token's nearest-anchor row written out by
    loops (Key Designs 3: same frame, same column, nearest anchor row)."""
    b, frames, rows, cols, h, d = 2, 2, 6, 3, 3, 8
    n = frames * rows * cols
    anchors = [1, 4]
    q, k, v = (_distinct_heads(s, b, n, h, d) for s in (40, 41, 42))
    heads = [2, 0]
    sel = np.array([0, 5, 7, 17, 18, 26, 35])
    out = O.anchor_attention_bnhd(q, k, v, frames, rows, cols, anchors, heads=heads, rows=sel)
    assert out.shape == (b, len(sel), len(heads), d)
    for bi in range(b):
        for hi, hh in enumerate(heads):
            ref, _ = O.anchor_attention(q[bi, :, hh], k[bi, :, hh], v[bi, :, hh],
                                        frames, rows, cols, anchors, rows=sel)
            np.testing.assert_array_equal(out[bi, :, hi], ref)
    t = lambda x: torch.from_numpy(x).permute(0, 2, 1, 3)      # [b, h, n, d]
    dense = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v)).numpy()
    near = {0: 1, 1: 1, 2: 1, 3: 4, 4: 4, 5: 4}                  # row 2: |2-1| < |2-4|
    for bi in range(b):
        for hi, hh in enumerate(heads):
            for si, tok in enumerate(sel):
                f, rho, w = tok // (rows * cols), (tok // cols) % rows, tok % cols
                src = (f * rows + near[rho]) * cols + w
                np.testing.assert_allclose(out[bi, si, hi], dense[bi, hh, src], rtol=0, atol=1e-12)


def test_energy_bnhd_wrapper_indexes_heads_and_batches():
    """block_energy_bnhd on batch 2, 3 heads and a ragged length, against (1)
    the one-head function on explicitly sliced inputs and (2) Eq. (5) computed
    by torch over [batch, heads, N, N] at once: a batched softmax, block sums
    by reshaping the zero-padded probabilities, divided by each query block's
    valid row count."""
    b, n, h, d, block = 2, 29, 3, 4, 8                           # 4 blocks, the last holds 5 tokens
    q, k = (_distinct_heads(s, b, n + 3, h, d) for s in (43, 44))
    q[:, n:] = np.nan                                             # padding rows are never read
    k[:, n:] = np.nan
    e = O.block_energy_bnhd(q, k, block, seq_len=n)
    assert e.shape == (b, h, 4, 4)
    for bi in range(b):
        for hh in range(h):
            np.testing.assert_array_equal(
                e[bi, hh], O.block_energy(q[bi, :, hh], k[bi, :, hh], block, seq_len=n))
    qt = torch.from_numpy(q[:, :n]).permute(0, 2, 1, 3)
    kt = torch.from_numpy(k[:, :n]).permute(0, 2, 1, 3)
    p = torch.softmax(qt @ kt.transpose(-1, -2) / math.sqrt(d), dim=-1)   # [b, h, n, n]
    pad = torch.zeros(b, h, 32, 32, dtype=torch.float64)
    pad[:, :, :n, :n] = p
    sums = pad.reshape(b, h, 4, block, 4, block).sum(dim=(3, 5))
    valid = torch.tensor([8.0, 8.0, 8.0, 5.0], dtype=torch.float64)
    np.testing.assert_allclose(e, (sums / valid[:, None]).numpy(), rtol=0, atol=1e-14)


# ---------------------------------------------------------------- anchors

def test_nearest_anchor_tables():
    for t in _golden("nearest_anchor_tables.json")["tables"]:
        got = O.nearest_anchor_rows(t["rows"], t["anchors"])
        assert got.tolist() == t["nearest"]


def test_anchor_query_reduction():
    for c in _golden("anchor_query_reduction.json")["cases"]:
        anchors = list(range(c["k"]))  # any k distinct rows
        src = O.anchor_source_tokens(1, c["H"], c["W"], anchors)
        assert len(np.unique(src)) == c["queries_after"]
        assert c["H"] * c["W"] == c["queries_before"]
        assert abs(1 - len(np.unique(src)) / c["queries_before"] - c["sparsity"]) < 1e-12


def test_anchor_attention_rows():
    frames, rows, cols, d = 2, 8, 5, 16
    n = frames * rows * cols
    q, k, v = (_rand(s, n, d) for s in (23, 24, 25))
    anchors = [0, 4]
    o, _ = O.anchor_attention(q, k, v, frames, rows, cols, anchors)
    dense = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None])[0].numpy()
    near = [0, 0, 0, 4, 4, 4, 4, 4]
    for f in range(frames):
        for rho in range(rows):
            for w in range(cols):
                i = (f * rows + rho) * cols + w
                a = (f * rows + near[rho]) * cols + w
                np.testing.assert_allclose(o[i], dense[a], rtol=0, atol=1e-12)
                if rho in anchors:
                    np.testing.assert_allclose(o[i], dense[i], rtol=0, atol=1e-12)


# ---------------------------------------------------------------- energy

def test_block_energy_rows_sum_to_one_ragged():
    n, block, d = 45, 16, 8          # last block has 13 valid tokens
    q, k = _rand(26, n, d, std=2.0), _rand(27, n, d, std=2.0)
    e = O.block_energy(q, k, block)
    assert e.shape == (3, 3)
    np.testing.assert_allclose(e.sum(axis=1), 1.0, rtol=0, atol=1e-12)


def test_block_energy_constant_keys_closed_form():
    n, block, d = 45, 16, 8
    q = _rand(28, n, d)
    k = np.tile(_rand(29, 1, d), (n, 1))
    e = O.block_energy(q, k, block)
    sizes = np.array([16, 16, 13], float)
    np.testing.assert_allclose(e, np.tile(sizes / n, (3, 1)), rtol=0, atol=1e-14)


def test_block_energy_double_loop_bruteforce():
    n, block, d = 11, 4, 3
    q, k = _rand(30, n, d, std=1.5), _rand(31, n, d, std=1.5)
    e = O.block_energy(q, k, block, scale=0.9)
    for r in range(3):
        rows = [i for i in range(n) if i // block == r]
        for c in range(3):
            tot = 0.0
            for i in rows:
                scores = [0.9 * sum(q[i, t] * k[j, t] for t in range(d)) for j in range(n)]
                mx = max(scores)
                z = sum(math.exp(s - mx) for s in scores)
                tot += sum(math.exp(scores[j] - mx) / z for j in range(n) if j // block == c)
            assert abs(e[r, c] - tot / len(rows)) < 1e-13


# ---------------------------------------------------------------- selection

def _bruteforce_min_size(row, tau):
    """Smallest number of blocks of which SOME subset carries mass >= tau (exhaustive)."""
    nk = len(row)
    for size in range(1, nk + 1):
        for subset in itertools.combinations(range(nk), size):
            if math.fsum(row[list(subset)]) >= tau:
                return size
    return nk


@pytest.mark.parametrize("seed", range(12))
def test_select_blocks_minimal_and_canonical(seed):
    rng = np.random.default_rng(100 + seed)
    nk = 6
    e = rng.dirichlet(np.full(nk, 0.4), size=5)
    if seed % 3 == 0:                       # exact ties at the boundary
        e[:, 1] = e[:, 2]
        e /= e.sum(axis=1, keepdims=True)
    for tau in (0.5, 0.9, 0.99):
        sel = O.select_blocks(e, tau)
        for r in range(e.shape[0]):
            size = _bruteforce_min_size(e[r], tau)
            chosen = tuple(np.flatnonzero(sel[r]))
            assert len(chosen) == size
            # the chosen set is the canonical (energy desc, index asc) prefix of that size
            canonical = sorted(range(nk), key=lambda c: (-e[r, c], c))[:size]
            assert chosen == tuple(sorted(canonical))
            if math.fsum(e[r]) >= tau:
                assert math.fsum(e[r, list(chosen)]) >= tau


def test_select_blocks_keeps_all_when_mass_never_reaches_tau():
    e = np.array([[0.25, 0.25, 0.25, 0.25 - 1e-9]])
    assert O.select_blocks(e, 1.0).all()


def test_select_blocks_single_dominant_block():
    e = np.array([[0.01, 0.97, 0.01, 0.01]])
    assert O.select_blocks(e, 0.95).tolist() == [[False, True, False, False]]
    assert O.select_blocks(e, 0.99).sum() == 3


# ---------------------------------------------------------------- aggregation

def test_aggregation_worked_example():
    g = _golden("aggregation_worked_example.json")
    counts = np.array(g["kept_counts"] + g["dropped_counts"])
    keep = O.aggregate_masks(counts, g["n_prompts"], g["rho"])
    assert keep.tolist() == [True] * len(g["kept_counts"]) + [False] * len(g["dropped_counts"])


def test_aggregation_from_stacked_masks_and_union():
    rng = np.random.default_rng(33)
    masks = rng.random((4, 3, 5)) < 0.3
    union = O.aggregate_masks(masks, 4, 0.25)
    np.testing.assert_array_equal(union, masks.any(axis=0))
    inter = O.aggregate_masks(masks, 4, 1.0)
    np.testing.assert_array_equal(inter, masks.all(axis=0))


# ------------------------------------------------------- spatial repetition

def test_spatial_similarity_anchor_rows_score_one():
    rng = np.random.default_rng(31)
    frames, rows, cols, d = 2, 6, 5, 8
    n = frames * rows * cols
    q, k = rng.standard_normal((n, d)), rng.standard_normal((n, d))
    sim = O.spatial_similarity(q, k, frames, rows, cols, (1, 4))
    assert np.abs(sim[:, [1, 4]] - 1.0).max() < 1e-12
    assert (sim >= 0).all() and (sim <= 1 + 1e-12).all()          # probabilities: Cauchy-Schwarz, non-negative


def test_spatial_similarity_repeated_rows_score_one():
    """A frame whose every spatial row repeats the anchor row's queries column
    by column attends identically row by row: similarity one everywhere."""
    rng = np.random.default_rng(32)
    frames, rows, cols, d = 2, 5, 4, 6
    n = frames * rows * cols
    q, k = rng.standard_normal((n, d)), rng.standard_normal((n, d))
    qf = q.reshape(frames, rows, cols, d)
    qf[0] = qf[0, 2][None]                                        # frame 0: all rows = row 2
    sim = O.spatial_similarity(qf.reshape(n, d), k, frames, rows, cols, (2,))
    assert np.abs(sim[0] - 1.0).max() < 1e-12
    assert sim[1].min() < 0.999                                   # frame 1 keeps its own rows


def test_spatial_similarity_disjoint_attention_scores_zero():
    """Non-anchor rows attend (almost) only to keys of one kind and the anchor
    row only to keys of another: the flattened distributions are orthogonal."""
    frames, rows, cols = 1, 3, 4
    n = frames * rows * cols
    k = np.zeros((n, 2))
    k[: n // 2, 0] = 1.0                                          # keys of kind A
    k[n // 2:, 1] = 1.0                                           # keys of kind B
    q = np.zeros((n, 2))
    for rho in range(rows):
        q[rho * cols:(rho + 1) * cols, 0 if rho != 1 else 1] = 60.0
    sim = O.spatial_similarity(q, k, frames, rows, cols, (1,), scale=1.0)
    assert abs(sim[0, 1] - 1.0) < 1e-12
    assert sim[0, 0] < 1e-20 and sim[0, 2] < 1e-20


def test_spatial_similarity_two_token_closed_form():
    """Two tokens (one frame, two rows of one column, anchor row 0): each
    attention row is a two-point distribution [sigma(x), 1 - sigma(x)] with x
    the scaled score difference, so the cosine has a closed form."""
    q = np.array([[0.7], [-1.3]])
    k = np.array([[1.1], [-0.4]])
    scale = 0.9
    sig = lambda x: 1.0 / (1.0 + math.exp(-x))
    a, b = sig(scale * 0.7 * 1.5), sig(scale * -1.3 * 1.5)
    cos = (a * b + (1 - a) * (1 - b)) / math.sqrt((a * a + (1 - a) ** 2) * (b * b + (1 - b) ** 2))
    sim = O.spatial_similarity(q, k, 1, 2, 1, (0,), scale=scale)
    assert abs(sim[0, 1] - cos) < 1e-14 and abs(sim[0, 0] - 1.0) < 1e-14


def test_spatial_similarity_double_loop():
    """Brute force: explicit loops over columns and keys with math.exp."""
    rng = np.random.default_rng(33)
    frames, rows, cols, d = 2, 3, 2, 3
    n = frames * rows * cols
    q, k = rng.standard_normal((n, d)), rng.standard_normal((n, d))
    scale = 0.6
    near = {0: 0, 1: 0, 2: 2}                                     # anchors {0, 2}; row 1 ties -> lower
    got = O.spatial_similarity(q, k, frames, rows, cols, (0, 2), scale=scale)

    def prob_row(i):
        e = [math.exp(scale * sum(q[i, t] * k[j, t] for t in range(d))) for j in range(n)]
        z = sum(e)
        return [x / z for x in e]

    for f in range(frames):
        for rho in range(rows):
            num = na = nb = 0.0
            for w in range(cols):
                pr = prob_row(f * rows * cols + rho * cols + w)
                pa = prob_row(f * rows * cols + near[rho] * cols + w)
                for j in range(n):
                    num += pr[j] * pa[j]
                    na += pr[j] * pr[j]
                    nb += pa[j] * pa[j]
            assert abs(got[f, rho] - num / math.sqrt(na * nb)) < 1e-13


def test_repetition_flags_mean_and_strict_threshold():
    sims = np.full((3, 2, 2, 4), 0.87)
    sims[:, 1] += 0.01                                            # head 1 above the threshold
    mean, flag = O.repetition_flags(sims, 0.87)
    assert abs(mean[0] - 0.87) < 1e-15 and not flag[0]            # equal is not "exceeds"
    assert flag[1]
    sims[2, 0, 1, 3] = 0.87 + 24 * 0.001                          # one of 24 entries raises the mean by 0.001
    mean, flag = O.repetition_flags(sims, 0.87)
    assert abs(mean[0] - 0.871) < 1e-12 and flag[0]
