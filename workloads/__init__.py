"""Seeded synthetic inputs for the CalibAtt attention workloads.

This module only produces inputs: Q/K/V tensors, synthetic block masks with the
structure of calibrated video-attention masks, anchor-row placements and head
flags.  It contains none of the attention arithmetic, so both the CPU oracle's
tests and the GPU library's tests and benchmark draw from it.

Workload shapes follow Wan 2.1 14B self-attention (40 heads, head_dim 128),
with latent video of 21 frames at 30x52 (480p) or 45x80 (720p) tokens per
frame, and 128x128 blocks ("Accelerating Text-to-Video Generation with
Calibrated Sparse Attention", Key Designs 1 uses 128x128 FlashAttention blocks;
Key Designs 3 uses five equally spaced anchor rows per frame).
"""

from __future__ import annotations

import dataclasses
import hashlib

import numpy as np

__all__ = [
    "Workload",
    "WORKLOADS",
    "make_qkv",
    "band_mask",
    "synthetic_block_mask",
    "tiny_block_mask",
    "equally_spaced_anchors",
    "repetitive_heads",
    "sweep_density",
    "seed_for",
    "mask_to_csr",
    "SWEEP_STEPS",
    "SWEEP_LAYERS",
    "sweep_record_density",
    "sweep_repetitive_heads",
    "sweep_layer_masks",
    "layer_csr",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    """One attention-call shape and the recipe for its synthetic inputs."""

    name: str
    batch: int
    heads: int
    head_dim: int
    frames: int
    rows: int          # spatial rows per frame (R)
    cols: int          # tokens per spatial row (C)
    block: int
    dtype: str         # "bf16" or "fp32"
    input_std: float   # elementwise standard deviation of Q, K, V
    density: tuple     # (low, high) per-head target block density of sparse heads
    n_repetitive: int  # heads taking the anchor path
    anchors: tuple     # anchor rows per frame
    seed: int

    @property
    def seq_len(self) -> int:
        return self.frames * self.rows * self.cols

    @property
    def tokens_per_frame(self) -> int:
        return self.rows * self.cols

    @property
    def num_blocks(self) -> int:
        return (self.seq_len + self.block - 1) // self.block


def equally_spaced_anchors(rows: int, k: int) -> tuple:
    """k anchor rows at the centres of k equal bands of the frame's R rows:
    floor((2m+1) * R / (2k)) for m = 0..k-1 (rows 4, 13, 22, 31, 40 for R=45, k=5)."""
    return tuple(((2 * m + 1) * rows) // (2 * k) for m in range(k))


# Input std N(0,1) * 128**-0.25: q.k then has unit variance before the 1/sqrt(D) scale.
_WAN_STD = 128.0 ** -0.25

WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 64, 2, 8, 16, 64, "fp32", 1.0, (0.5, 0.5), 1, (0, 4), 0),
    "480p": Workload("480p", 1, 40, 128, 21, 30, 52, 128, "bf16", _WAN_STD, (0.32, 0.38), 0,
                     equally_spaced_anchors(30, 5), 1000),
    "720p": Workload("720p", 1, 40, 128, 21, 45, 80, 128, "bf16", _WAN_STD, (0.32, 0.38), 0,
                     equally_spaced_anchors(45, 5), 2000),
    "720p_dual": Workload("720p_dual", 1, 40, 128, 21, 45, 80, 128, "bf16", _WAN_STD,
                          (0.32, 0.38), 12, equally_spaced_anchors(45, 5), 3000),
    "720p_sweep": Workload("720p_sweep", 1, 40, 128, 21, 45, 80, 128, "bf16", _WAN_STD,
                           (0.20, 0.60), 10, equally_spaced_anchors(45, 5), 4000),
}

# Mask seeds per head: 100+h (480p), 200+h (720p), 300+h (dual-path 720p).
MASK_SEED_BASE = {"480p": 100, "720p": 200, "720p_dual": 300}


def seed_for(*parts) -> int:
    """Deterministic 63-bit seed from a tuple of labels (used for the sweep's per-(t, l, h) draws)."""
    h = hashlib.sha256(repr(parts).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def make_qkv(seed, batch, seq_len, heads, head_dim, dtype="bf16", std=1.0, device="cpu",
             seq_alloc=None):
    """Seeded Q, K, V of layout [batch, N_alloc, H, D] with N(0, std^2) entries.

    Drawn with torch's generator on `device` in float32, then cast (bf16 values
    are the rounded draws).  Rows >= seq_len (allocation padding) are filled with
    NaN so that any read of them shows up in the results.
    """
    import torch

    n_alloc = seq_len if seq_alloc is None else int(seq_alloc)
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    tdtype = {"bf16": torch.bfloat16, "fp32": torch.float32}[dtype]
    out = []
    for _ in range(3):
        t = torch.randn((batch, n_alloc, heads, head_dim), generator=g, device=device,
                        dtype=torch.float32)
        t.mul_(std)
        if n_alloc > seq_len:
            t[:, seq_len:] = float("nan")
        out.append(t.to(tdtype))
    return tuple(out)


def band_mask(num_blocks, block, tokens_per_frame, w):
    """Structured part of a synthetic calibrated mask: temporal diagonal band of
    half-width w frames, every key block holding a first-frame token, and the
    diagonal block.  frame(block) is the frame of the block's first token."""
    idx = np.arange(num_blocks)
    frame = (idx * block) // tokens_per_frame
    m = np.abs(frame[:, None] - frame[None, :]) <= w
    m |= (idx * block < tokens_per_frame)[None, :]
    m |= np.eye(num_blocks, dtype=bool)
    return m


def synthetic_block_mask(seed, num_blocks, block, tokens_per_frame, target):
    """Synthetic calibrated mask at a target block density.

    The band half-width w is the largest whose structured density stays <= the
    target (w = 0 if none does); uniformly random extra blocks are then added
    until round(target * nb^2) blocks are kept.  Diagonal blocks are always kept.
    """
    rng = np.random.default_rng(int(seed))
    total = num_blocks * num_blocks
    want = int(round(target * total))
    w = 0
    while True:
        nxt = band_mask(num_blocks, block, tokens_per_frame, w + 1)
        if nxt.sum() > want or w + 1 > num_blocks:
            break
        w += 1
    m = band_mask(num_blocks, block, tokens_per_frame, w)
    extra = want - int(m.sum())
    if extra > 0:
        free = np.flatnonzero(~m.ravel())
        pick = rng.choice(free, size=min(extra, len(free)), replace=False)
        m.ravel()[pick] = True
    return m


def tiny_block_mask(seed, num_blocks, density):
    """Diagonal plus uniformly random off-diagonal blocks up to round(density * nb^2)."""
    rng = np.random.default_rng(int(seed))
    m = np.eye(num_blocks, dtype=bool)
    want = int(round(density * num_blocks * num_blocks))
    free = np.flatnonzero(~m.ravel())
    extra = max(0, want - num_blocks)
    pick = rng.choice(free, size=min(extra, len(free)), replace=False)
    m.ravel()[pick] = True
    return m


def repetitive_heads(seed, heads, n_repetitive):
    """A seeded choice of n_repetitive of the heads (the first entries of a permutation)."""
    rng = np.random.default_rng(int(seed))
    return tuple(sorted(int(h) for h in rng.permutation(heads)[:n_repetitive]))


def sweep_density(t, steps, seed):
    """Density of the schedule sweep: linear 0.60 -> 0.20 over the steps, plus a
    seeded per-head jitter in [-0.03, 0.03]."""
    rng = np.random.default_rng(int(seed))
    base = 0.60 - 0.40 * t / max(1, steps - 1)
    return float(min(1.0, max(0.0, base + rng.uniform(-0.03, 0.03))))


def head_densities(seed, heads, low, high):
    """Per-head target densities drawn uniformly in [low, high]."""
    rng = np.random.default_rng(int(seed))
    return rng.uniform(low, high, size=heads)


def mask_to_csr(mask):
    """Per-q-block lists of retained key-block indices, ascending: (row_ptr, col_idx) int32."""
    m = np.asarray(mask, dtype=bool)
    counts = m.sum(axis=1)
    row_ptr = np.zeros(m.shape[0] + 1, dtype=np.int32)
    np.cumsum(counts, out=row_ptr[1:])
    col_idx = np.nonzero(m)[1].astype(np.int32)
    return row_ptr, col_idx


def workload_masks(wl: Workload, heads=None, seed_base=None):
    """Per-head synthetic masks of a workload (None for heads on the anchor path)."""
    heads = range(wl.heads) if heads is None else heads
    base = MASK_SEED_BASE.get(wl.name, wl.seed) if seed_base is None else seed_base
    dens = head_densities(base + 10_000, wl.heads, *wl.density)
    rep = set(repetitive_heads(base + 20_000, wl.heads, wl.n_repetitive))
    out = {}
    for h in heads:
        if h in rep:
            out[h] = None
        else:
            out[h] = synthetic_block_mask(base + h, wl.num_blocks, wl.block,
                                          wl.tokens_per_frame, float(dens[h]))
    return out, tuple(sorted(rep))


def dense_flops_per_tile(block, head_dim):
    """Multiply-add work of one retained (q-block, k-block) tile: QK^T and PV, 2 flops per MAC."""
    return 4 * block * block * head_dim


def ceil_div(a, b):
    return -(-a // b)


def count_bytes(*arrays):
    return int(sum(a.numel() * a.element_size() for a in arrays))



# ------------------------------------------------------------- schedule sweep
# One 720p-shaped call per (timestep t, layer l) of a 50-step, 40-layer
# schedule; per-(t, l, h) seeded masks whose density ramps from 60 % at the
# first timestep to 20 % at the last, and 10 of the 40 heads of every call on
# the anchor path.

SWEEP_STEPS = 50
SWEEP_LAYERS = 40
SWEEP_REPETITIVE = 10


def sweep_record_density(t, l, h, steps=SWEEP_STEPS):
    """Target block density of record (t, l, h) of the sweep."""
    return sweep_density(t, steps, seed_for("sweep-density", t, l, h) % (1 << 32))


def sweep_repetitive_heads(t, l, heads=40, n=SWEEP_REPETITIVE):
    """Heads of call (t, l) on the anchor path."""
    return repetitive_heads(seed_for("sweep-repetitive", t, l) % (1 << 32), heads, n)


def _band_counts(num_blocks, block, tokens_per_frame):
    """Blocks kept by band_mask for every half-width w = 0 .. last frame."""
    frames = ((num_blocks - 1) * block) // tokens_per_frame + 1
    return [int(band_mask(num_blocks, block, tokens_per_frame, w).sum()) for w in range(frames + 1)]


_BAND_COUNTS = {}


def sweep_record_blocks(wl, t, l, h, steps=SWEEP_STEPS):
    """Retained blocks of record (t, l, h) (0 for heads on the anchor path), from
    the recipe alone: the band of the largest half-width within the target,
    topped up with random blocks to round(density * nb^2)."""
    if h in sweep_repetitive_heads(t, l, wl.heads):
        return 0
    key = (wl.num_blocks, wl.block, wl.tokens_per_frame)
    if key not in _BAND_COUNTS:
        _BAND_COUNTS[key] = _band_counts(*key)
    counts = _BAND_COUNTS[key]
    want = int(round(sweep_record_density(t, l, h, steps) * wl.num_blocks ** 2))
    w = max([0] + [i for i, c in enumerate(counts) if c <= want])
    return max(want, counts[w])


def sweep_layer_masks(wl, t, l, device="cpu", steps=SWEEP_STEPS):
    """Block masks of call (t, l) of the sweep: a bool tensor [H, nb, nb] on
    `device` (all False for the heads on the anchor path) and the tuple of
    anchor-path heads.

    The structure follows synthetic_block_mask (band of the largest half-width
    within the target, every first-frame key block, the diagonal), and the
    random top-up is the round(density * nb^2) - |band| free blocks with the
    smallest uniform keys drawn by torch's generator on `device` with seed
    seed_for("sweep-fill", t, l, h): a uniform random subset, drawn fast enough
    on the GPU for the 2,000 calls of the sweep.  The masks depend on the
    device whose generator drew them."""
    import torch

    nb = wl.num_blocks
    rep = sweep_repetitive_heads(t, l, wl.heads)
    key = (nb, wl.block, wl.tokens_per_frame)
    if key not in _BAND_COUNTS:
        _BAND_COUNTS[key] = _band_counts(*key)
    counts = _BAND_COUNTS[key]
    idx = torch.arange(nb, device=device)
    frame = (idx * wl.block) // wl.tokens_per_frame
    first = (idx * wl.block < wl.tokens_per_frame)[None, :]
    eye = torch.eye(nb, dtype=torch.bool, device=device)
    masks = torch.zeros((wl.heads, nb, nb), dtype=torch.bool, device=device)
    for h in range(wl.heads):
        if h in rep:
            continue
        want = int(round(sweep_record_density(t, l, h, steps) * nb * nb))
        w = max([0] + [i for i, c in enumerate(counts) if c <= want])
        band = ((frame[:, None] - frame[None, :]).abs() <= w) | first | eye
        extra = want - counts[w]
        if extra > 0:
            g = torch.Generator(device=device)
            g.manual_seed(seed_for("sweep-fill", t, l, h))
            keys = torch.rand(nb * nb, generator=g, device=device)
            keys[band.view(-1)] = 2.0
            pick = torch.argsort(keys)[:extra]
            flat = band.view(-1).clone()
            flat[pick] = True
            band = flat.view(nb, nb)
        masks[h] = band
    return masks, rep


def layer_csr(masks):
    """Per-head CSR of a [H, nb, nb] bool tensor, on the host: row_ptr int32
    [H, nb + 1] (each head's starting at 0) and the heads' column lists
    concatenated in head order (int32)."""
    import torch

    counts = masks.sum(dim=2, dtype=torch.int32)
    row_ptr = torch.zeros((masks.shape[0], masks.shape[1] + 1), dtype=torch.int32, device=masks.device)
    row_ptr[:, 1:] = torch.cumsum(counts, dim=1, dtype=torch.int32)
    col_idx = torch.nonzero(masks)[:, 2].to(torch.int32)
    return row_ptr.cpu().numpy(), col_idx.cpu().numpy()
