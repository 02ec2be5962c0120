"""Checks of the seeded input generators (structure of the synthetic masks and layouts)."""

import numpy as np

import workloads as W


def test_synthetic_mask_structure_720p():
    wl = W.WORKLOADS["720p"]
    nb = wl.num_blocks
    assert nb == 591 and wl.seq_len == 75600
    for target in (0.32, 0.35, 0.38):
        m = W.synthetic_block_mask(7, nb, wl.block, wl.tokens_per_frame, target)
        assert m.shape == (nb, nb)
        assert m[np.arange(nb), np.arange(nb)].all()
        first_frame_cols = np.flatnonzero(np.arange(nb) * wl.block < wl.tokens_per_frame)
        assert m[:, first_frame_cols].all()
        assert abs(m.sum() - round(target * nb * nb)) <= 0
    # the structured band alone: w=2 -> ~26.6%, w=3 -> ~34.6%
    assert abs(W.band_mask(nb, 128, 3600, 2).mean() - 0.266) < 0.005
    assert abs(W.band_mask(nb, 128, 3600, 3).mean() - 0.346) < 0.005


def test_masks_are_seeded_and_deterministic():
    a = W.synthetic_block_mask(3, 300, 128, 3600, 0.35)
    b = W.synthetic_block_mask(3, 300, 128, 3600, 0.35)
    c = W.synthetic_block_mask(4, 300, 128, 3600, 0.35)
    assert (a == b).all() and (a != c).any()


def test_tiny_mask_density_and_diagonal():
    m = W.tiny_block_mask(1, 4, 0.5)
    assert m.sum() == 8 and m[np.arange(4), np.arange(4)].all()


def test_anchor_placement_and_repetitive_heads():
    assert W.equally_spaced_anchors(45, 5) == (4, 13, 22, 31, 40)
    rep = W.repetitive_heads(5, 40, 12)
    assert len(rep) == 12 and len(set(rep)) == 12 and all(0 <= h < 40 for h in rep)


def test_mask_to_csr_roundtrip():
    rng = np.random.default_rng(0)
    m = rng.random((9, 7)) < 0.4
    rp, ci = W.mask_to_csr(m)
    back = np.zeros_like(m)
    for r in range(9):
        cols = ci[rp[r]:rp[r + 1]]
        assert (np.diff(cols) > 0).all()
        back[r, cols] = True
    assert (back == m).all()


def test_sweep_density_ramp():
    assert abs(W.sweep_density(0, 50, 1) - 0.60) <= 0.03 + 1e-12
    assert abs(W.sweep_density(49, 50, 1) - 0.20) <= 0.03 + 1e-12


def test_sweep_recipe_small():
    """The schedule-sweep mask recipe on a small geometry: exact retained-block
    counts from the recipe alone, diagonal and first-frame key blocks kept, an
    empty mask for anchor-path heads, the density ramp, determinism, and the
    per-head CSR layout."""
    import dataclasses

    wl = dataclasses.replace(W.WORKLOADS["720p_sweep"], frames=4, rows=8, cols=16, block=64, heads=12)
    nb = wl.num_blocks
    for t, l in [(0, 0), (30, 3), (49, 7)]:
        masks, rep = W.sweep_layer_masks(wl, t, l)
        assert rep == W.sweep_repetitive_heads(t, l, wl.heads) and len(rep) == W.SWEEP_REPETITIVE
        m = masks.numpy()
        first = np.arange(nb) * wl.block < wl.tokens_per_frame
        for h in range(wl.heads):
            assert m[h].sum() == W.sweep_record_blocks(wl, t, l, h)
            if h in rep:
                assert not m[h].any()
            else:
                assert m[h][np.arange(nb), np.arange(nb)].all()
                assert m[h][:, first].all()
        again, _ = W.sweep_layer_masks(wl, t, l)
        assert np.array_equal(again.numpy(), m)
        rp, ci = W.layer_csr(masks)
        assert rp.shape == (wl.heads, nb + 1) and rp.dtype == np.int32 and (rp[:, 0] == 0).all()
        off = 0
        for h in range(wl.heads):
            r, c = W.mask_to_csr(m[h])
            assert np.array_equal(rp[h], r)
            assert np.array_equal(ci[off:off + c.size], c)
            off += c.size
        assert off == ci.size
    d0 = [W.sweep_record_density(0, 0, h) for h in range(20)]
    d49 = [W.sweep_record_density(49, 0, h) for h in range(20)]
    assert all(0.57 <= d <= 0.63 for d in d0) and all(0.17 <= d <= 0.23 for d in d49)


def test_traffic_record_is_tied_to_the_kernel_sources(tmp_path):
    """bench.py reports the captured DRAM traffic only while every device
    source of the kernel hashes as it did at the capture."""
    import json
    import os
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench

    rec = json.load(open(os.path.join(root, "profiles", "tc_attn_sparse_720p_traffic.json")))
    assert all(os.path.exists(os.path.join(root, f)) for f in rec["kernel_sources_sha256"])
    per_tile = rec["dram_bytes_per_retained_tile"]
    assert per_tile == (rec["dram_read_bytes"] + rec["dram_write_bytes"]) / rec["retained_tiles"]
    tampered = dict(rec, kernel_sources_sha256=dict(rec["kernel_sources_sha256"]))
    first = next(iter(tampered["kernel_sources_sha256"]))
    tampered["kernel_sources_sha256"][first] = "0" * 64
    path = tmp_path / "traffic.json"
    path.write_text(json.dumps(tampered))
    assert bench.measured_traffic(1000, str(path)) is None
    assert bench.measured_traffic(1000, str(tmp_path / "missing.json")) is None


def test_cpu_baseline_leg_reports_parity_of_the_given_output():
    """bench.py's CPU-baseline leg times the oracle on sampled query blocks and,
    given the library's output of the same call, reports its error on those
    rows: zero-ish for the oracle's own output, large for a wrong one."""
    import os
    import sys

    import torch

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    from oracle import calibatt_oracle as O

    wl = W.WORKLOADS["tiny"]
    q, k, v = W.make_qkv(wl.seed, 1, wl.seq_len, wl.heads, wl.head_dim, "fp32", wl.input_std, "cpu")
    nb = wl.num_blocks
    masks = {0: np.ones((nb, nb), bool), 1: np.eye(nb, dtype=bool)}
    ref, _ = O.block_sparse_attention_bnhd(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                           [masks[0], masks[1]], wl.block)
    base, par = bench.cpu_baseline(wl, masks, q, k, v, torch.from_numpy(ref).float(), budget_s=0.3)
    assert base["kind"] == "oracle" and base["cores"] >= 1 and base["value"] > 0
    assert par["within_tolerance"] and par["max_abs"] < 1e-6
    _, bad = bench.cpu_baseline(wl, masks, q, k, v, torch.from_numpy(ref).float() + 0.1, budget_s=0.3)
    assert not bad["within_tolerance"] and abs(bad["max_abs"] - 0.1) < 1e-3
    assert isinstance(bench.cpu_baseline(wl, masks, q, k, v, budget_s=0.1), dict)   # no output: baseline only


def test_sweep_sample_spreads_over_the_schedule():
    """The bench's sampled sweep: the same number of calls at every timestep
    (the density ramp is sampled evenly), distinct calls, layers in range."""
    import bench

    picks = bench.sweep_sample_picks(100)
    assert len(picks) == 100 == len(set(picks))
    per_t = {}
    for t, l in picks:
        assert 0 <= t < W.SWEEP_STEPS and 0 <= l < W.SWEEP_LAYERS
        per_t[t] = per_t.get(t, 0) + 1
    assert sorted(per_t) == list(range(W.SWEEP_STEPS)) and set(per_t.values()) == {2}


def test_mufu_peak_arithmetic():
    import bench

    assert bench.mufu_exp2_peak(148, 1965.0) == 16 * 148 * 1965e6
