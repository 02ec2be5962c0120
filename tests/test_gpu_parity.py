"""GPU parity of libcalibatt.so against the float64 CPU oracle.

Every call goes through the C ABI (ctypes binding).  Tolerances: float32
inputs max-abs <= 1e-4; bf16 inputs max-abs <= 2e-2 and mean-abs <= 2e-3;
selected block sets bit-exact.
"""

import math

import numpy as np
import pytest
import torch

import workloads as W
from oracle import calibatt_oracle as O

pytestmark = pytest.mark.gpu

BF16_MAX, BF16_MEAN, FP32_MAX = 2e-2, 2e-3, 1e-4


@pytest.fixture(scope="module")
def C(calibatt_lib):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    calibatt_lib.set_wait_timeout_ms(4000)
    return calibatt_lib


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def _check_status(C):
    torch.cuda.synchronize()
    assert C.device_status() == 0


def _assert_close(got, ref, dtype):
    err = np.abs(got - ref)
    assert np.isfinite(got).all(), "non-finite output"
    if dtype == "fp32":
        assert err.max() <= FP32_MAX, f"max-abs {err.max():.3e}"
    else:
        assert err.max() <= BF16_MAX, f"max-abs {err.max():.3e}"
        assert err.mean() <= BF16_MEAN, f"mean-abs {err.mean():.3e}"
    return float(err.max()), float(err.mean())


def _run_sparse(C, q, k, v, masks, block, lse=False, num_ctas=0):
    b, n, h, d = q.shape
    nb = O.num_blocks(n, block)
    rp, ci, rep = C.masks_to_layer_csr(masks, h, nb)
    out = torch.full_like(q, float("nan"))
    lse_t = torch.full((b, h, n), float("nan"), device=q.device) if lse else None
    with C.MaskDictionary(1, 1, h, nb, nb, block, max(1, ci.size), num_ctas) as dct:
        dct.set_layer(0, 0, rp, ci, rep)
        C.calibatt_block_sparse_attn(q, k, v, out, dct, 0, 0, block, lse=lse_t)
        _check_status(C)
    return out, lse_t


def _random_masks(seed, h, nb, density, empty_row_head=None):
    rng = np.random.default_rng(seed)
    masks = []
    for hh in range(h):
        m = rng.random((nb, nb)) < density
        m[np.arange(nb), np.arange(nb)] = True
        if hh == empty_row_head:
            m[1, :] = False
        masks.append(m)
    return masks


# ------------------------------------------------------------------ tiny config

def _tiny_inputs(dtype):
    wl = W.WORKLOADS["tiny"]
    q, k, v = W.make_qkv(wl.seed, wl.batch, wl.seq_len, wl.heads, wl.head_dim, dtype, wl.input_std, "cuda")
    mask0 = W.tiny_block_mask(1, wl.num_blocks, 0.5)
    return wl, q, k, v, mask0


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_tiny_dual_path(C, dtype):
    wl, q, k, v, mask0 = _tiny_inputs(dtype)
    nb = wl.num_blocks
    rp, ci, rep = C.masks_to_layer_csr([mask0, None], wl.heads, nb)
    out = torch.full_like(q, float("nan"))
    with C.MaskDictionary(1, 1, wl.heads, nb, nb, wl.block, ci.size) as dct:
        dct.set_layer(0, 0, rp, ci, rep)
        C.calibatt_dual_path_attn(q, k, v, out, dct, 0, 0, wl.frames, wl.rows, wl.cols, wl.anchors, wl.block)
        _check_status(C)
    qn, kn, vn = _np(q)[0], _np(k)[0], _np(v)[0]
    ref0, _ = O.block_sparse_attention(qn[:, 0], kn[:, 0], vn[:, 0], mask0, wl.block)
    ref1, _ = O.anchor_attention(qn[:, 1], kn[:, 1], vn[:, 1], wl.frames, wl.rows, wl.cols, wl.anchors)
    got = _np(out)[0]
    _assert_close(got[:, 0], ref0, dtype)
    _assert_close(got[:, 1], ref1, dtype)


# ------------------------------------------------------------ tensor-core sparse

@pytest.mark.parametrize("d", [128, 64])
def test_tc_sparse_ragged_multi_batch(C, d):
    b, n, h, block = 2, 1000, 3, 128            # 8 blocks, last holds 104 tokens
    # allocations of 1024 rows whose padding rows are NaN; the library sees views of the n valid rows
    qa, ka, va = W.make_qkv(11, b, n, h, d, "bf16", 1.0, "cuda", seq_alloc=1024)
    q, k, v = qa[:, :n], ka[:, :n], va[:, :n]
    nb = O.num_blocks(n, block)
    masks = _random_masks(5, h, nb, 0.5, empty_row_head=2)
    out_alloc = torch.full_like(qa, float("nan"))
    lse = torch.full((b, h, n), float("nan"), device="cuda")
    rp, ci, rep = C.masks_to_layer_csr(masks, h, nb)
    with C.MaskDictionary(1, 1, h, nb, nb, block, ci.size) as dct:
        dct.set_layer(0, 0, rp, ci, rep)
        C.calibatt_block_sparse_attn(q, k, v, out_alloc[:, :n], dct, 0, 0, block, lse=lse)
        _check_status(C)
    out = out_alloc[:, :n]
    ref, ref_lse = O.block_sparse_attention_bnhd(_np(q), _np(k), _np(v), masks, block, seq_len=n)
    _assert_close(_np(out), ref, "bf16")
    assert torch.isnan(out_alloc[:, n:]).all(), "padding rows of the output were written"
    got_lse = lse.cpu().numpy().astype(np.float64)
    finite = np.isfinite(ref_lse)
    assert (np.isneginf(got_lse) == ~finite).all()
    assert np.abs(got_lse[finite] - ref_lse[finite]).max() < 2e-2
    # head 2 row-block 1 is empty -> zeros
    assert (out[:, 128:256, 2].float() == 0).all()


def test_tc_all_ones_mask_is_dense_attention(C):
    b, n, h, d, block = 1, 777, 2, 128, 128
    q, k, v = W.make_qkv(12, b, n, h, d, "bf16", 1.0, "cuda")
    nb = O.num_blocks(n, block)
    out, _ = _run_sparse(C, q, k, v, [np.ones((nb, nb), bool)] * h, block)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.double().permute(0, 2, 1, 3).cpu(), k.double().permute(0, 2, 1, 3).cpu(),
        v.double().permute(0, 2, 1, 3).cpu()).permute(0, 2, 1, 3).numpy()
    _assert_close(_np(out), ref, "bf16")


def test_tc_sparse_deterministic_and_schedule_independent(C):
    b, n, h, d, block = 1, 2048, 4, 128, 128
    q, k, v = W.make_qkv(13, b, n, h, d, "bf16", 128 ** -0.25, "cuda")
    masks = _random_masks(6, h, 16, 0.35)
    o1, _ = _run_sparse(C, q, k, v, masks, block)
    o2, _ = _run_sparse(C, q, k, v, masks, block)
    o3, _ = _run_sparse(C, q, k, v, masks, block, num_ctas=7)   # different persistent grid
    assert torch.equal(o1, o2)
    assert torch.equal(o1, o3)


def test_tc_sparse_peaked_scores_rescale(C):
    # large logits make the running maximum jump across blocks (rescale path)
    b, n, h, d, block = 1, 1536, 2, 128, 128
    q, k, v = W.make_qkv(14, b, n, h, d, "bf16", 1.0, "cuda")
    q = (q.float() * 3.0).to(torch.bfloat16)
    masks = _random_masks(7, h, 12, 0.6)
    out, _ = _run_sparse(C, q, k, v, masks, block)
    ref, _ = O.block_sparse_attention_bnhd(_np(q), _np(k), _np(v), masks, block)
    _assert_close(_np(out), ref, "bf16")


# ------------------------------------------------------------ tensor-core anchor

def test_tc_anchor_broadcast(C):
    frames, rows, cols, h, d = 3, 10, 24, 3, 128
    n = frames * rows * cols
    anchors = (1, 4, 8)
    q, k, v = W.make_qkv(15, 1, n, h, d, "bf16", 1.0, "cuda")
    out = torch.full_like(q, float("nan"))
    C.calibatt_anchor_attn(q, k, v, out, frames, rows, cols, anchors, [0, 2])
    _check_status(C)
    ref = O.anchor_attention_bnhd(_np(q), _np(k), _np(v), frames, rows, cols, anchors, heads=[0, 2])
    got = _np(out)
    _assert_close(got[:, :, [0, 2]], ref, "bf16")
    assert torch.isnan(out[:, :, 1]).all(), "a head not listed was written"
    # every broadcast row is a bitwise copy of its anchor row
    near = O.nearest_anchor_rows(rows, anchors)
    o = out.view(1, frames, rows, cols, h, d)
    for rho in range(rows):
        assert torch.equal(o[:, :, rho, :, [0, 2]], o[:, :, near[rho], :, [0, 2]])


@pytest.mark.parametrize("batch,heads,d,frames,rows,cols,anchors", [
    (1, 22, 128, 4, 9, 100, (2, 6)),    # N = 3600: 29 key blocks (last of 16 tokens), 7 tiles per head
    (1, 33, 128, 4, 9, 100, (2, 6)),    # 231 tiles: the last 83 in 3 ranges
    (2, 11, 64, 4, 9, 100, (2, 6)),     # two batches, head_dim 64
    (1, 50, 128, 5, 10, 10, (2, 7)),    # N = 500: 4 key blocks (last of 116 tokens), 1 tile per head, all
])                                      # 50 tiles split in 2 ranges of 2 blocks
def test_tc_anchor_split_last_wave(C, batch, heads, d, frames, rows, cols, anchors):
    """With a workspace the anchor call cuts its last partial wave of tiles
    into key ranges and merges them exactly: every listed head matches the
    oracle; whole tiles are bitwise those of the call without a workspace and
    split tiles agree with them to rounding; a repeated call is bitwise equal
    (the merge sums the ranges in range order, whichever ends last); broadcast
    rows are bitwise copies of their anchors; the workspace's counters are
    reset by the call (it starts as NaN bytes)."""
    n = frames * rows * cols
    nb, tph = O.num_blocks(n, 128), -(-frames * len(anchors) * cols // 128)
    q, k, v = W.make_qkv(71 + heads, batch, n, heads, d, "bf16", 1.0, "cuda")
    head_ids = list(np.random.default_rng(heads).permutation(heads))
    tiles = batch * heads * tph
    first, parts = C.anchor_split_plan(tiles, C.device_sm_count(), nb)
    assert parts > 1 and first < tiles, "this case must split its last wave"
    nbytes = C.calibatt_anchor_attn_workspace_size(q, frames, rows, cols, len(anchors), heads)
    assert nbytes > 0
    ws = torch.full((nbytes // 4,), float("nan"), device="cuda")
    with pytest.raises(C.CalibattError):          # too small
        C.calibatt_anchor_attn(q, k, v, torch.empty_like(q), frames, rows, cols, anchors, head_ids,
                               workspace=ws[:-64])
    with pytest.raises(C.CalibattError):          # not 256-byte aligned
        C.calibatt_anchor_attn(q, k, v, torch.empty_like(q), frames, rows, cols, anchors, head_ids,
                               workspace=ws[1:])
    split = torch.full_like(q, float("nan"))
    whole = torch.full_like(q, float("nan"))
    C.calibatt_anchor_attn(q, k, v, split, frames, rows, cols, anchors, head_ids, workspace=ws)
    C.calibatt_anchor_attn(q, k, v, whole, frames, rows, cols, anchors, head_ids)
    again = torch.full_like(q, float("nan"))
    C.calibatt_anchor_attn(q, k, v, again, frames, rows, cols, anchors, head_ids, workspace=ws)
    _check_status(C)
    assert not torch.isnan(split).any()
    assert torch.equal(split, again)
    ref = O.anchor_attention_bnhd(_np(q), _np(k), _np(v), frames, rows, cols, anchors)
    _assert_close(_np(split), ref, "bf16")
    # the tokens of the split tiles: item t = (batch, listed head, tile) for t >= first
    near = O.nearest_anchor_rows(rows, anchors)
    a_of_row = np.array([list(anchors).index(near[r]) for r in range(rows)])
    f, rho, w = np.meshgrid(np.arange(frames), np.arange(rows), np.arange(cols), indexing="ij")
    tile_of_token = torch.as_tensor(((f * len(anchors) + a_of_row[rho]) * cols + w).reshape(-1) // 128)
    in_split = torch.zeros((batch, n, heads), dtype=torch.bool)
    for t in range(first, tiles):
        b, r = divmod(t, heads * tph)
        in_split[b, :, head_ids[r // tph]] |= tile_of_token == r % tph
    in_split = in_split.cuda()
    assert in_split.any()
    assert torch.equal(split[~in_split], whole[~in_split])
    diff = (split[in_split].float() - whole[in_split].float()).abs().max().item()
    assert diff <= 1e-2, diff
    o = split.view(batch, frames, rows, cols, heads, d)
    for r in range(rows):
        assert torch.equal(o[:, :, r], o[:, :, near[r]])


@pytest.mark.parametrize("rows,anchors", [(16, tuple(range(16))), (9, (5,))])
def test_tc_anchor_degenerate_geometries(C, rows, anchors):
    """The anchor path's degenerate cases, with and without the split
    workspace: every spatial row an anchor (16 anchors, the most a call
    takes) makes every query attend densely and serve only itself, so the
    output is dense attention (the oracle's block-sparse attention with
    all-ones masks); a single anchor row serves every row of its frame, so
    all rows of a frame and column are bitwise equal."""
    frames, cols, h, d = 2, 64, 3, 128
    n = frames * rows * cols
    q, k, v = W.make_qkv(91 + rows, 1, n, h, d, "bf16", 1.0, "cuda")
    nbytes = C.calibatt_anchor_attn_workspace_size(q, frames, rows, cols, len(anchors), h)
    ws = torch.empty(max(1, nbytes // 4), device="cuda")
    outs = []
    for w in (None, ws if nbytes else None):
        out = torch.full_like(q, float("nan"))
        C.calibatt_anchor_attn(q, k, v, out, frames, rows, cols, anchors, list(range(h)), workspace=w)
        outs.append(out)
    _check_status(C)
    ref = O.anchor_attention_bnhd(_np(q), _np(k), _np(v), frames, rows, cols, anchors)
    for out in outs:
        _assert_close(_np(out), ref, "bf16")
    o = outs[0].view(1, frames, rows, cols, h, d)
    if len(anchors) == rows:
        nb = O.num_blocks(n, 128)
        dense, _ = O.block_sparse_attention_bnhd(_np(q), _np(k), _np(v), [np.ones((nb, nb), bool)] * h, 128)
        np.testing.assert_allclose(ref, dense, rtol=0, atol=1e-12)
        _assert_close(_np(outs[0]), dense, "bf16")
    else:
        for r in range(rows):
            assert torch.equal(o[:, :, r], o[:, :, anchors[0]])


def test_simt_anchor_fp32(C):
    frames, rows, cols, h, d = 2, 9, 16, 2, 64
    n = frames * rows * cols
    anchors = (2, 6)
    q, k, v = W.make_qkv(16, 1, n, h, d, "fp32", 1.0, "cuda")
    out = torch.full_like(q, float("nan"))
    C.calibatt_anchor_attn(q, k, v, out, frames, rows, cols, anchors, [1], block=64)
    _check_status(C)
    ref = O.anchor_attention_bnhd(_np(q), _np(k), _np(v), frames, rows, cols, anchors, heads=[1])
    _assert_close(_np(out)[:, :, [1]], ref, "fp32")


def test_simt_sparse_bf16_block64_and_fp32_block128(C):
    for dtype, block, d in (("bf16", 64, 128), ("fp32", 128, 128)):
        b, n, h = 1, 700, 2
        q, k, v = W.make_qkv(17, b, n, h, d, dtype, 1.0, "cuda")
        nb = O.num_blocks(n, block)
        masks = _random_masks(8, h, nb, 0.5, empty_row_head=1)
        out, lse = _run_sparse(C, q, k, v, masks, block, lse=True)
        ref, _ = O.block_sparse_attention_bnhd(_np(q), _np(k), _np(v), masks, block)
        _assert_close(_np(out), ref, dtype)


# ------------------------------------------------------ direct CSR (no dictionary)

def _device_csr(C, masks, h, nb):
    """Device row_ptr / 16-bit col_idx / col_base of per-head masks, and the host row_ptr."""
    rp, ci, _ = C.masks_to_layer_csr(masks, h, nb)
    base = np.zeros(h, np.int64)
    base[1:] = np.cumsum(rp[:, -1].astype(np.int64))[:-1]
    col = ci.astype(np.uint16).view(np.int16) if ci.size else np.zeros(1, np.int16)
    return (torch.from_numpy(rp).cuda(), torch.from_numpy(col).cuda(), torch.from_numpy(base).cuda(), rp)


@pytest.mark.parametrize("d,density", [(128, 0.4), (64, 0.4), (128, 1.0)])   # 1.0: all-ones lists, dense
def test_csr_call_matches_dictionary_and_oracle(C, d, density):
    b, n, h, block, grid = 2, 1000, 4, 128, 11
    q, k, v = W.make_qkv(31, b, n, h, d, "bf16", 1.0, "cuda")
    nb = O.num_blocks(n, block)
    masks = _random_masks(9, h, nb, density, empty_row_head=3 if density < 1 else None)
    rp_d, col_d, base_d, rp = _device_csr(C, masks, h, nb)
    heads = [3, 0, 2]
    items, cta_ptr = C.csr_schedule(rp, heads, grid)
    items_d = torch.from_numpy(items.view(np.int32)).cuda()
    cta_d = torch.from_numpy(cta_ptr).cuda()
    out = torch.full_like(q, float("nan"))
    lse = torch.full((b, h, n), float("nan"), device="cuda")
    C.calibatt_block_sparse_attn_csr(q, k, v, out, rp_d, col_d, base_d, heads, items_d, cta_d, grid, block,
                                     lse=lse)
    _check_status(C)
    assert torch.isnan(out[:, :, 1]).all() and torch.isnan(lse[:, 1]).all(), "a head not listed was written"
    # the dictionary call on the same lists (head 1 routed to the other path) gives the same bits
    ref_out, ref_lse = _run_sparse(C, q, k, v, [m if i in heads else None for i, m in enumerate(masks)], block,
                                   lse=True)
    assert torch.equal(out[:, :, heads], ref_out[:, :, heads])
    assert torch.equal(lse[:, heads], ref_lse[:, heads])
    ref, _ = O.block_sparse_attention_bnhd(_np(q)[:, :, heads], _np(k)[:, :, heads], _np(v)[:, :, heads],
                                           [masks[i] for i in heads], block)
    _assert_close(_np(out)[:, :, heads], ref, "bf16")


@pytest.mark.parametrize("dtype,block,d", [("bf16", 128, 128), ("fp32", 64, 64)])
def test_csr_call_flags_block_index_out_of_range(C, dtype, block, d):
    """Device lists are not read on the host: an index >= nq in one row is
    caught on the device (the list check ahead of the attention, code 23; no
    kernel reads outside the tensors), recorded in the status word (low byte
    CALIBATT_ERR_INVALID_ARG) and cleared by the read; the next valid call is
    unaffected."""
    b, n, h = 1, 1000, 2
    q, k, v = W.make_qkv(33, b, n, h, d, dtype, 1.0, "cuda")
    nb = O.num_blocks(n, block)
    masks = _random_masks(11, h, nb, 0.5)
    rp_d, col_d, base_d, rp = _device_csr(C, masks, h, nb)
    bad = col_d.clone()
    bad[int(rp[0, 3])] = nb + 5                # first block of head 0, row 3
    bad[int(rp[0, nb] - 1)] = 0x7FFF           # last block of head 0's last row
    items, cta_ptr = C.csr_schedule(rp, [0, 1], 5)
    sched = (torch.from_numpy(items.view(np.int32)).cuda(), torch.from_numpy(cta_ptr).cuda(), 5)
    out = torch.zeros_like(q)
    C.calibatt_block_sparse_attn_csr(q, k, v, out, rp_d, bad, base_d, [0, 1], *sched, block=block)
    code = C.device_status()
    assert code & 0xFF == C.ERR_INVALID_ARG and code >> 8 == 23, hex(code)
    assert "key-block index" in C.last_error()
    assert C.device_status() == 0                                   # the read cleared it
    C.calibatt_block_sparse_attn_csr(q, k, v, out, rp_d, col_d, base_d, [0, 1], *sched, block=block)
    _check_status(C)
    ref, _ = O.block_sparse_attention_bnhd(_np(q), _np(k), _np(v), masks, block)
    _assert_close(_np(out), ref, dtype)
    # indices in range but out of order (head 1, the first row with two blocks) are flagged too
    r = next(r for r in range(nb) if rp[1, r + 1] - rp[1, r] >= 2)
    i = int(rp[0, nb] + rp[1, r])
    swapped = col_d.clone()
    swapped[i], swapped[i + 1] = col_d[i + 1], col_d[i]
    C.calibatt_block_sparse_attn_csr(q, k, v, out, rp_d, swapped, base_d, [0, 1], *sched, block=block)
    code = C.device_status()
    assert code & 0xFF == C.ERR_INVALID_ARG and code >> 8 == 23, hex(code)


def _padded_col(col_d, nb):
    """The device list with nb + 64 zero entries after its end, so that even a
    row pointer run past the lists stays inside the allocation."""
    return torch.cat([col_d, torch.zeros(nb + 64, dtype=col_d.dtype, device=col_d.device)])


@pytest.mark.parametrize("dtype,block,d", [("bf16", 128, 128), ("fp32", 64, 64)])
def test_csr_call_with_invalid_row_pointers_writes_nothing(C, dtype, block, d):
    """A row longer than nq (row pointers of head 0 shifted from row 4 on, so
    they still increase) is flagged by the device check (code 23), and the
    attention of that call then returns before reading any list: no output
    is written.  The flag holds for later direct-CSR calls until the status
    word is read and cleared; then the same call with valid lists runs."""
    b, n, h = 1, 1000, 2
    q, k, v = W.make_qkv(34, b, n, h, d, dtype, 1.0, "cuda")
    nb = O.num_blocks(n, block)
    masks = _random_masks(12, h, nb, 0.5)
    rp_d, col_d, base_d, rp = _device_csr(C, masks, h, nb)
    col_d = _padded_col(col_d, nb)
    delta = nb + 1 - int(rp[0, 4] - rp[0, 3])            # row 3 now holds nb + 1 blocks
    bad_rp = rp_d.clone()
    bad_rp[0, 4:] += delta
    sched = None
    if block == 128 and dtype == "bf16":
        items, cta_ptr = C.csr_schedule(rp, [0, 1], 7)
        sched = (torch.from_numpy(items.view(np.int32)).cuda(), torch.from_numpy(cta_ptr).cuda(), 7)
    out = torch.full_like(q, float("nan"))
    kw = dict(block=block)
    C.calibatt_block_sparse_attn_csr(q, k, v, out, bad_rp, col_d, base_d, [0, 1], *(sched or ()), **kw)
    C.calibatt_block_sparse_attn_csr(q, k, v, out, rp_d, col_d, base_d, [0, 1], *(sched or ()), **kw)
    torch.cuda.synchronize()
    assert torch.isnan(out).all(), "the attention ran on lists the check had flagged"
    code = C.device_status()
    assert code & 0xFF == C.ERR_INVALID_ARG and code >> 8 == 23, hex(code)
    C.calibatt_block_sparse_attn_csr(q, k, v, out, rp_d, col_d, base_d, [0, 1], *(sched or ()), **kw)
    _check_status(C)
    ref, _ = O.block_sparse_attention_bnhd(_np(q), _np(k), _np(v), masks, block)
    _assert_close(_np(out), ref, dtype)


def test_csr_call_with_invalid_schedule_writes_nothing(C):
    """The tensor-core kernel's device schedule is checked before it runs
    (code 24): an item naming a head that is not listed, a last CTA offset
    that is not n_heads * nq, and decreasing CTA offsets are each flagged,
    and the call writes no output."""
    b, n, h, block, grid = 1, 1000, 2, 128, 6
    q, k, v = W.make_qkv(35, b, n, h, 128, "bf16", 1.0, "cuda")
    nb = O.num_blocks(n, block)
    masks = _random_masks(13, h, nb, 0.5)
    rp_d, col_d, base_d, rp = _device_csr(C, masks, h, nb)
    items, cta_ptr = C.csr_schedule(rp, [0], grid)                     # head 0 only
    unlisted = items.copy()
    unlisted[3] = (1 << 16) | (int(items[3]) & 0xFFFF)                # head 1 is not listed
    short_end = cta_ptr.copy()
    short_end[grid] -= 1
    decreasing = cta_ptr.copy()
    c = int(np.argmax(np.diff(cta_ptr) > 0))                          # a CTA with work
    decreasing[c + 1] = decreasing[c] - 1 if decreasing[c] > 0 else 0
    decreasing[c] = max(decreasing[c], 1)
    for it, cp in ((unlisted, cta_ptr), (items, short_end), (items, decreasing)):
        out = torch.full_like(q, float("nan"))
        C.calibatt_block_sparse_attn_csr(q, k, v, out, rp_d, col_d, base_d, [0],
                                         torch.from_numpy(it.view(np.int32)).cuda(),
                                         torch.from_numpy(cp).cuda(), grid, block=block)
        torch.cuda.synchronize()
        assert torch.isnan(out).all(), "the attention ran on a schedule the check had flagged"
        code = C.device_status()
        assert code & 0xFF == C.ERR_INVALID_ARG and code >> 8 == 24, hex(code)
        assert "schedule" in C.last_error()
    out = torch.full_like(q, float("nan"))
    C.calibatt_block_sparse_attn_csr(q, k, v, out, rp_d, col_d, base_d, [0],
                                     torch.from_numpy(items.view(np.int32)).cuda(),
                                     torch.from_numpy(cta_ptr).cuda(), grid, block=block)
    _check_status(C)
    ref, _ = O.block_sparse_attention_bnhd(_np(q)[:, :, :1], _np(k)[:, :, :1], _np(v)[:, :, :1], masks[:1], block)
    _assert_close(_np(out)[:, :, :1], ref, "bf16")
    assert torch.isnan(out[:, :, 1]).all()


def test_csr_call_cuda_core_paths(C):
    for dtype, block, d in (("fp32", 64, 64), ("bf16", 64, 128), ("fp32", 128, 128)):
        b, n, h = 1, 700, 3
        q, k, v = W.make_qkv(32, b, n, h, d, dtype, 1.0, "cuda")
        nb = O.num_blocks(n, block)
        masks = _random_masks(10, h, nb, 0.5, empty_row_head=2)
        rp_d, col_d, base_d, _ = _device_csr(C, masks, h, nb)
        out = torch.full_like(q, float("nan"))
        C.calibatt_block_sparse_attn_csr(q, k, v, out, rp_d, col_d, base_d, [2, 0], block=block)   # no schedule
        _check_status(C)
        assert torch.isnan(out[:, :, 1]).all()
        ref, _ = O.block_sparse_attention_bnhd(_np(q)[:, :, [0, 2]], _np(k)[:, :, [0, 2]], _np(v)[:, :, [0, 2]],
                                               [masks[0], masks[2]], block)
        _assert_close(_np(out)[:, :, [0, 2]], ref, dtype)


# ------------------------------------------------------ full-size sampled parity

def _sampled_blocks(rng, nb, k):
    mid = rng.choice(np.arange(1, nb - 1), size=k - 2, replace=False)
    return sorted({0, nb - 1, *mid.tolist()})


def _f32(t):
    return t.detach().float().cpu().numpy()


def _block_rows(blocks, seq_len):
    return np.concatenate([np.arange(r * 128, min(seq_len, (r + 1) * 128)) for r in blocks])


@pytest.mark.parametrize("name", ["480p", "720p"])
def test_full_size_sparse_sampled(C, name):
    """Every head at full size, 8 sampled q-blocks each including the first and
    the ragged last one, against the oracle (evaluated in spawned workers); at
    720p the interval dictionary's output equals the index lists' bitwise."""
    import _oracle_jobs as J

    wl = W.WORKLOADS[name]
    q, k, v = W.make_qkv(wl.seed, wl.batch, wl.seq_len, wl.heads, wl.head_dim, "bf16", wl.input_std, "cuda")
    masks, _ = W.workload_masks(wl)
    masks = [masks[h] for h in range(wl.heads)]
    out, _ = _run_sparse(C, q, k, v, masks, wl.block)
    if name == "720p":
        # the interval dictionary (the pages' encoding) gives the same output bit for bit
        rp, ci, rep = C.masks_to_layer_csr(masks, wl.heads, wl.num_blocks)
        alt = torch.full_like(q, float("nan"))
        with _dictionary(C, "intervals", 1, 1, wl.heads, wl.num_blocks, wl.block, rp, ci) as dct:
            dct.set_layer(0, 0, rp, ci, rep)
            C.calibatt_block_sparse_attn(q, k, v, alt, dct, 0, 0, wl.block)
            _check_status(C)
            # the masks' random top-up blocks are mostly runs of one: about 41
            # intervals per row here, 3.6x fewer bytes than the 16-bit lists
            assert dct.info()["device_bytes"] < 0.35 * (ci.size * 2)
        assert torch.equal(alt, out)
        del alt
    rng = np.random.default_rng(1)
    jobs, got = [], []
    for h in range(wl.heads):
        rows = _block_rows(_sampled_blocks(rng, wl.num_blocks, 8), wl.seq_len)
        jobs.append((_f32(q[0, rows, h]), _f32(k[0, :wl.seq_len, h]), _f32(v[0, :wl.seq_len, h]), masks[h],
                     wl.block, rows))
        got.append(_np(out[0, torch.as_tensor(rows, device=q.device), h]))
    refs = J.sparse_rows_many(jobs)
    err = np.concatenate([np.abs(g - r).ravel() for g, r in zip(got, refs)])
    assert err.max() <= BF16_MAX and err.mean() <= BF16_MEAN, (err.max(), err.mean())


def test_full_size_dual_path_sampled(C):
    """The dual-path 720p layer as ONE fused launch (the dictionary carries the
    anchor geometry; a bitmap dictionary): every anchor head on sampled rows
    of two frames, every sparse head on 8 sampled q-blocks, broadcast rows
    bitwise equal; and bitwise the output of the two-launch path over an
    index-list dictionary."""
    import _oracle_jobs as J

    wl = W.WORKLOADS["720p_dual"]
    q, k, v = W.make_qkv(wl.seed, wl.batch, wl.seq_len, wl.heads, wl.head_dim, "bf16", wl.input_std, "cuda")
    masks, rep_heads = W.workload_masks(wl)
    assert len(rep_heads) == 12
    rp, ci, rep = C.masks_to_layer_csr([masks[h] for h in range(wl.heads)], wl.heads, wl.num_blocks)
    out = torch.full_like(q, float("nan"))
    with C.MaskDictionary(1, 1, wl.heads, wl.num_blocks, wl.num_blocks, wl.block, ci.size, bitmap=True) as dct:
        dct.set_anchor_geometry(wl.frames, wl.rows, wl.cols, wl.anchors)
        dct.set_layer(0, 0, rp, ci, rep)
        C.calibatt_dual_path_attn(q, k, v, out, dct, 0, 0, wl.frames, wl.rows, wl.cols, wl.anchors, wl.block)
        _check_status(C)
    assert not torch.isnan(out).any()
    two = torch.full_like(q, float("nan"))
    with C.MaskDictionary(1, 1, wl.heads, wl.num_blocks, wl.num_blocks, wl.block, ci.size) as dct:
        dct.set_layer(0, 0, rp, ci, rep)
        C.calibatt_dual_path_attn(q, k, v, two, dct, 0, 0, wl.frames, wl.rows, wl.cols, wl.anchors, wl.block)
        _check_status(C)
    assert torch.equal(out, two)
    del two
    rng = np.random.default_rng(2)
    # anchor heads: rows of two frames, including the last frame's last row
    f_rows = np.concatenate([np.arange(f * wl.tokens_per_frame, (f + 1) * wl.tokens_per_frame)
                             for f in (int(rng.integers(0, wl.frames - 1)), wl.frames - 1)])
    sample = np.union1d(f_rows[rng.choice(len(f_rows), 400, replace=False)], [wl.seq_len - 1])
    a_jobs = [(_f32(q[0, :wl.seq_len, h]), _f32(k[0, :wl.seq_len, h]), _f32(v[0, :wl.seq_len, h]),
               wl.frames, wl.rows, wl.cols, wl.anchors, sample) for h in rep_heads]
    # sparse heads: 8 sampled q-blocks each
    sparse_heads = [h for h in range(wl.heads) if h not in rep_heads]
    s_rows = {h: _block_rows(_sampled_blocks(rng, wl.num_blocks, 8), wl.seq_len) for h in sparse_heads}
    s_jobs = [(_f32(q[0, s_rows[h], h]), _f32(k[0, :wl.seq_len, h]), _f32(v[0, :wl.seq_len, h]), masks[h],
               wl.block, s_rows[h]) for h in sparse_heads]
    a_refs = J.anchor_rows_many(a_jobs)
    for h, ref in zip(rep_heads, a_refs):
        _assert_close(_np(out[0, torch.as_tensor(sample, device=q.device), h]), ref, "bf16")
    s_refs = J.sparse_rows_many(s_jobs)
    for h, ref in zip(sparse_heads, s_refs):
        _assert_close(_np(out[0, torch.as_tensor(s_rows[h], device=q.device), h]), ref, "bf16")
    # broadcast rows are bitwise copies of their anchor rows, for every repetitive head
    near = O.nearest_anchor_rows(wl.rows, wl.anchors)
    o = out.view(1, wl.frames, wl.rows, wl.cols, wl.heads, wl.head_dim)[..., list(rep_heads), :]
    for rho in range(wl.rows):
        assert torch.equal(o[:, :, rho], o[:, :, near[rho]])


def test_full_size_anchor_split_sampled(C):
    """The anchor path alone at the dual-path 720p layer's size (12
    repetitive heads, 792 tiles on the grid) with its split workspace: the
    split tiles' rows match the oracle on a sample, every other row is
    bitwise the call's output without a workspace, repeated calls are
    bitwise equal, and broadcast rows are bitwise copies of their anchors."""
    import _oracle_jobs as J

    wl = W.WORKLOADS["720p_dual"]
    q, k, v = W.make_qkv(wl.seed, wl.batch, wl.seq_len, wl.heads, wl.head_dim, "bf16", wl.input_std, "cuda")
    _, rep_heads = W.workload_masks(wl)
    heads = list(rep_heads)
    tph = -(-wl.frames * len(wl.anchors) * wl.cols // 128)
    first, parts = C.anchor_split_plan(len(heads) * tph, C.device_sm_count(), wl.num_blocks)
    assert parts > 1
    ws = torch.empty(C.calibatt_anchor_attn_workspace_size(q, wl.frames, wl.rows, wl.cols, len(wl.anchors),
                                                           len(heads)) // 4, device="cuda")
    split = torch.full_like(q, float("nan"))
    again = torch.full_like(q, float("nan"))
    whole = torch.full_like(q, float("nan"))
    C.calibatt_anchor_attn(q, k, v, split, wl.frames, wl.rows, wl.cols, wl.anchors, heads, workspace=ws)
    C.calibatt_anchor_attn(q, k, v, again, wl.frames, wl.rows, wl.cols, wl.anchors, heads, workspace=ws)
    C.calibatt_anchor_attn(q, k, v, whole, wl.frames, wl.rows, wl.cols, wl.anchors, heads)
    _check_status(C)
    assert torch.equal(split[:, :, heads], again[:, :, heads])   # the other heads stay NaN
    assert torch.isnan(split[:, :, [h for h in range(wl.heads) if h not in heads]]).all()
    del again
    # tokens of the split tiles: item t >= first is tile t % tph of listed head t // tph
    near = O.nearest_anchor_rows(wl.rows, wl.anchors)
    a_of_row = np.array([list(wl.anchors).index(near[r]) for r in range(wl.rows)])
    f, rho, w = np.meshgrid(np.arange(wl.frames), np.arange(wl.rows), np.arange(wl.cols), indexing="ij")
    tile_of_token = ((f * len(wl.anchors) + a_of_row[rho]) * wl.cols + w).reshape(-1) // 128
    split_tokens = {}
    for t in range(first, len(heads) * tph):
        split_tokens.setdefault(heads[t // tph], set()).add(t % tph)
    for h in heads:
        sel = np.isin(tile_of_token, sorted(split_tokens.get(h, ())))
        idx = torch.as_tensor(np.nonzero(~sel)[0], device=q.device)
        assert torch.equal(split[0, idx, h], whole[0, idx, h])
    del whole
    rng = np.random.default_rng(5)
    jobs, checks = [], []
    for h, tiles in sorted(split_tokens.items()):
        toks = np.nonzero(np.isin(tile_of_token, sorted(tiles)))[0]
        sample = np.sort(rng.choice(toks, min(300, len(toks)), replace=False))
        jobs.append((_f32(q[0, :wl.seq_len, h]), _f32(k[0, :wl.seq_len, h]), _f32(v[0, :wl.seq_len, h]),
                     wl.frames, wl.rows, wl.cols, wl.anchors, sample))
        checks.append((h, sample))
    for (h, sample), ref in zip(checks, J.anchor_rows_many(jobs)):
        _assert_close(_np(split[0, torch.as_tensor(sample, device=q.device), h]), ref, "bf16")
    o = split.view(1, wl.frames, wl.rows, wl.cols, wl.heads, wl.head_dim)[..., heads, :]
    for r in range(wl.rows):
        assert torch.equal(o[:, :, r], o[:, :, near[r]])


# --------------------------------------------------------- offline calibration

def _energy(C, q, k, block):
    b, n, h, _ = q.shape
    nb = O.num_blocks(n, block)
    e = torch.full((b, h, nb, nb), float("nan"), device=q.device)
    ws = torch.empty(C.calibatt_block_energy_workspace_size(q) // 4, device=q.device)
    C.calibatt_block_energy(q, k, e, ws, block)
    _check_status(C)
    return e


@pytest.mark.parametrize("dtype,n,block,d,std", [("fp32", 256, 64, 64, 1.0), ("bf16", 300, 64, 128, 1.0),
                                                  ("fp32", 500, 64, 128, 0.3)])
def test_block_energy(C, dtype, n, block, d, std):
    """CUDA-core energy path (float32, or bf16 with 64-token blocks)."""
    q, k, _ = W.make_qkv(20, 1, n, 2, d, dtype, std, "cuda")
    e = _energy(C, q, k, block)
    ref = O.block_energy_bnhd(_np(q), _np(k), block)
    got = e.cpu().numpy().astype(np.float64)
    assert np.abs(got - ref).max() < 2e-6
    np.testing.assert_allclose(got.sum(-1), 1.0, atol=1e-5)
    e2 = _energy(C, q, k, block)
    assert torch.equal(e, e2), "energies are not bitwise repeatable"


@pytest.mark.parametrize("b,n,h,d,std", [(1, 300, 2, 128, 1.0), (2, 2000, 3, 128, 0.5), (1, 1100, 2, 64, 2.0)])
def test_block_energy_tensor_core(C, b, n, h, d, std):
    """bf16 with 128-token blocks runs on the tensor cores (LSE pass + energy
    pass): energies within 1e-5 of the oracle (scores accumulate in float32
    on the tensor core, exponentials are the MUFU's), rows sum to one,
    bitwise repeatable; ragged last blocks on both axes."""
    q, k, _ = W.make_qkv(22, b, n, h, d, "bf16", std, "cuda")
    e = _energy(C, q, k, 128)
    ref = O.block_energy_bnhd(_np(q), _np(k), 128)
    got = e.cpu().numpy().astype(np.float64)
    assert np.abs(got - ref).max() < 1e-5, np.abs(got - ref).max()
    np.testing.assert_allclose(got.sum(-1), 1.0, atol=1e-4)
    assert torch.equal(e, _energy(C, q, k, 128)), "energies are not bitwise repeatable"


def test_select_blocks_bit_exact_on_identical_energies(C):
    rng = np.random.default_rng(21)
    n_rows, nk = 300, 37
    e = rng.dirichlet(np.full(nk, 0.3), size=n_rows).astype(np.float32)
    e[::3, 5] = e[::3, 6]                          # exact ties
    e[::7] = np.round(e[::7] * 64) / 64            # many ties
    et = torch.from_numpy(e).cuda()
    for tau in (0.5, 0.9, 0.99, 1.0):
        mask = torch.zeros((n_rows, nk), dtype=torch.uint8, device="cuda")
        cnt = torch.zeros((n_rows, nk), dtype=torch.int32, device="cuda")
        C.calibatt_select_blocks(et, tau, mask, cnt)
        _check_status(C)
        ref = O.select_blocks(e.astype(np.float64), float(np.float32(tau)))
        assert (mask.cpu().numpy().astype(bool) == ref).all()
        assert (cnt.cpu().numpy() == ref.astype(np.int32)).all()


def test_aggregate_worked_example(C):
    counts = torch.tensor([32, 33, 63, 64, 0, 1, 30, 31], dtype=torch.int32, device="cuda")
    mask = torch.zeros(8, dtype=torch.uint8, device="cuda")
    C.calibatt_aggregate_masks(counts, 64, 0.5, mask)
    _check_status(C)
    assert mask.cpu().tolist() == [1, 1, 1, 1, 0, 0, 0, 0]


def _margin_ok(e_ref, tau, margin=1e-5):
    """Rows whose selection is decided with a float64 margin above `margin`."""
    ok = []
    for row in e_ref.reshape(-1, e_ref.shape[-1]):
        srt = np.sort(row)[::-1]
        cum = np.add.accumulate(srt)
        gaps = np.abs(np.diff(srt)) if len(srt) > 1 else np.array([1.0])
        ok.append(min(np.abs(cum - tau).min(), gaps.min() if gaps.size else 1.0) > margin)
    return np.array(ok)


def _check_selection(got, e_ref, tau, margin=1e-5):
    """Every row of the GPU selection `got` (bool [rows, nk]) is checked
    against the float64 energies `e_ref` (Key Designs 1: the shortest
    energy-descending prefix whose cumulative mass reaches tau).

    Rows decided with a margin above `margin` (no energy gap and no partial
    mass within `margin` of tau) must equal the oracle's set bit for bit.  In
    the other rows several sets are correct; the GPU set must be one of them:
    its size is the oracle's k* (or, where the mass at the GPU's size is within
    `margin` of tau, one of the sizes the rounding allows); its float64 mass
    reaches tau - margin; it is a prefix of the energy order up to ties within
    `margin` (no excluded block outweighs a kept one by more than that); and
    dropping its lightest block leaves a mass below tau + margin.
    Returns (rows checked bit for bit, rows checked for validity, rows whose
    size differs from k* within the rounding margin)."""
    ref = O.select_blocks(e_ref, tau)
    ok = _margin_ok(e_ref, tau, margin)
    assert (got[ok] == ref[ok]).all(), "a decided row differs from the oracle"
    boundary = 0
    for r in np.flatnonzero(~ok):
        e, sel = e_ref[r], got[r]
        kstar = int(ref[r].sum())
        size = int(sel.sum())
        mass = math.fsum(e[sel])
        assert size >= 1, f"row {r}: empty selection"
        if size != kstar:
            cum = np.add.accumulate(np.sort(e)[::-1])
            assert abs(cum[size - 1] - tau) <= margin or abs(cum[kstar - 1] - tau) <= margin, \
                f"row {r}: size {size} != k* {kstar} away from the tau boundary"
            boundary += 1
        assert mass >= tau - margin or size == len(e), f"row {r}: mass {mass} < tau {tau}"
        kept_min = e[sel].min()
        excl = e[~sel]
        assert excl.size == 0 or excl.max() <= kept_min + margin, f"row {r}: not an energy-descending prefix"
        assert mass - kept_min < tau + margin, f"row {r}: a smaller prefix already reaches tau"
    return int(ok.sum()), int((~ok).sum()), boundary


@pytest.mark.parametrize("std,tau", [(1.0, 0.99), (4.0, 0.5), (4.0, 0.9)])
def test_energy_select_union_tiny(C, std, tau):
    """Tiny configuration: 4 seeded Q/K draws, selection at tau, masks unioned
    (rho = 1/4), on the CUDA-core energies (float32, 64-token blocks).  Every
    row is checked (_check_selection); the union equals the OR of the draws'
    GPU selections everywhere and the oracle's union on rows every draw
    decided with a margin."""
    wl = W.WORKLOADS["tiny"]
    _select_and_union(C, [W.make_qkv(s, wl.batch, wl.seq_len, wl.heads, wl.head_dim, "fp32", std, "cuda")[:2]
                          for s in (10, 11, 12, 13)], wl.block, tau)


@pytest.mark.parametrize("tau", [0.5, 0.9])
def test_energy_select_union_tensor_core(C, tau):
    """The same energy -> selection -> union chain on the tensor-core energies
    (bf16, 128-token blocks): 2 heads, N = 2000 (15 full blocks and one of 80
    tokens), peaked logits (std 4), 3 seeded draws, their union (rho = 0.25)."""
    draws = [W.make_qkv(s, 1, 2000, 2, 128, "bf16", 4.0, "cuda")[:2] for s in (40, 41, 42)]
    _select_and_union(C, draws, 128, tau)


def _select_and_union(C, draws, block, tau):
    q0 = draws[0][0]
    b, n, h, _ = q0.shape
    nb = O.num_blocks(n, block)
    rows = b * h * nb
    cnt = torch.zeros((rows, nb), dtype=torch.int32, device="cuda")
    tau64 = float(np.float32(tau))
    gpu_masks, ref_masks, decided = [], [], []
    exact = checked = boundary = 0
    for q, k in draws:
        e = _energy(C, q, k, block)
        mask = torch.zeros((rows, nb), dtype=torch.uint8, device="cuda")
        C.calibatt_select_blocks(e.view(-1, nb), tau, mask, cnt)
        _check_status(C)
        e_ref = O.block_energy_bnhd(_np(q), _np(k), block).reshape(-1, nb)
        got = mask.cpu().numpy().astype(bool)
        x, c, bd = _check_selection(got, e_ref, tau64)
        exact, checked, boundary = exact + x, checked + c, boundary + bd
        gpu_masks.append(got)
        ref_masks.append(O.select_blocks(e_ref, tau64))
        decided.append(_margin_ok(e_ref, tau64))
    assert (cnt.cpu().numpy() == np.sum(gpu_masks, axis=0)).all(), "selection counts"
    union = torch.zeros_like(cnt, dtype=torch.uint8)
    # rho = 0.25 is exact in float32 and keeps every block chosen at least
    # once for 3 or 4 draws (a union); 1/3 would round up above 1/3
    C.calibatt_aggregate_masks(cnt, len(draws), 0.25, union)
    _check_status(C)
    union = union.cpu().numpy().astype(bool)
    assert (union == np.logical_or.reduce(gpu_masks)).all(), "union of the GPU selections"
    all_ok = np.logical_and.reduce(decided)
    ref_union = O.aggregate_masks(np.stack(ref_masks), len(draws), 0.25)
    assert (union[all_ok] == ref_union[all_ok]).all(), \
        f"{exact} rows bit-exact, {checked} margin rows checked for validity ({boundary} at the tau boundary)"
    print(f"selection: {exact} rows bit-exact, {checked} margin rows valid, {boundary} at the tau boundary")


def test_fma_exp2_error_bound(C):
    rng = np.random.default_rng(22)
    x = np.concatenate([rng.uniform(-125, 126, 200000), np.arange(-125, 127, 0.25),
                        [0.0, -0.5, 0.5, 8.0, -1e-7, 1e-7]]).astype(np.float32)
    xt = torch.from_numpy(x).cuda()
    y = torch.empty_like(xt)
    C.calibatt_debug_exp2_fma(xt, y)
    _check_status(C)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y.cpu().numpy().astype(np.float64) / ref - 1.0)
    assert rel.max() < 1e-4, rel.max()
    low = torch.tensor([-126.0, -200.0, float("-inf")], device="cuda")
    yl = torch.empty_like(low)
    C.calibatt_debug_exp2_fma(low, yl)
    _check_status(C)
    assert (yl >= 0).all() and (yl < 1e-37).all()


def test_fma_exp2_quintic_error_bound(C):
    """The quintic FMA-pipe 2^x of the offline energy passes: relative error
    below 3e-7 against float64 over the whole input range (the fit's 7.5e-8
    plus float32 evaluation), odd lengths included, tiny values for x < -125."""
    rng = np.random.default_rng(23)
    x = np.concatenate([rng.uniform(-125, 126, 200000), rng.uniform(-1, 1, 50001), np.arange(-125, 127, 0.125),
                        [0.0, -0.5, 0.5, 8.0, -1e-7, 1e-7, -0.4999999, 0.4999999]]).astype(np.float32)
    assert x.size % 2 == 1
    xt = torch.from_numpy(x).cuda()
    y = torch.empty_like(xt)
    C.calibatt_debug_exp2_fma_quintic(xt, y)
    _check_status(C)
    rel = np.abs(y.cpu().numpy().astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 3e-7, rel.max()
    low = torch.tensor([-126.0, -200.0, float("-inf")], device="cuda")
    yl = torch.empty_like(low)
    C.calibatt_debug_exp2_fma_quintic(low, yl)
    _check_status(C)
    assert (yl >= 0).all() and (yl < 1e-37).all()


@pytest.mark.parametrize("fmt", ["lists", "bitmap"])
def test_sweep_records_sampled(C, fmt):
    """Records of the schedule sweep in one dictionary spanning all 50 x 40
    (timestep, layer) slots, with the anchor geometry (one fused launch per
    call): the dual-path call of (t, l) must use that record's masks and
    anchor heads (checked against the oracle on sampled rows), and
    retained-tile counts must match the recipe."""
    wl = W.WORKLOADS["720p_sweep"]
    nb = wl.num_blocks
    records = [(0, 0), (25, 17), (49, 39)]
    nnz = sum(W.sweep_record_blocks(wl, t, l, h) for t, l in records for h in range(wl.heads))
    rng = np.random.default_rng(5)
    with C.MaskDictionary(W.SWEEP_STEPS, W.SWEEP_LAYERS, wl.heads, nb, nb, wl.block, nnz,
                          bitmap=fmt == "bitmap") as dct:
        dct.set_anchor_geometry(wl.frames, wl.rows, wl.cols, wl.anchors)
        host = {}
        for t, l in records:
            masks, rep = W.sweep_layer_masks(wl, t, l, "cuda")
            rp, ci = W.layer_csr(masks)
            rep_arr = np.zeros(wl.heads, np.uint8)
            rep_arr[list(rep)] = 1
            dct.set_layer(t, l, rp, ci, rep_arr)
            host[(t, l)] = (masks.cpu().numpy(), rep)
            li = dct.layer_info(t, l)
            assert li["repetitive_heads"] == W.SWEEP_REPETITIVE
            assert li["retained_tiles"] == sum(W.sweep_record_blocks(wl, t, l, h) for h in range(wl.heads))
        for t, l in records:
            masks, rep = host[(t, l)]
            q, k, v = W.make_qkv(W.seed_for("sweep-qkv", t, l) % (1 << 62), 1, wl.seq_len, wl.heads,
                                 wl.head_dim, "bf16", wl.input_std, "cuda")
            out = torch.full_like(q, float("nan"))
            C.calibatt_dual_path_attn(q, k, v, out, dct, t, l, wl.frames, wl.rows, wl.cols, wl.anchors, wl.block)
            _check_status(C)
            assert not torch.isnan(out).any()
            sparse_heads = [h for h in range(wl.heads) if h not in rep]
            for h in rng.choice(sparse_heads, 2, replace=False):
                blocks = _sampled_blocks(rng, nb, 3)
                rows = np.concatenate([np.arange(r * 128, min(wl.seq_len, (r + 1) * 128)) for r in blocks])
                qh, kh, vh = _np(q[0, :, h]), _np(k[0, :, h]), _np(v[0, :, h])
                ref, _ = O.block_sparse_attention(qh, kh, vh, masks[h], wl.block, rows=rows)
                _assert_close(_np(out[0, torch.as_tensor(rows, device=q.device), h]), ref, "bf16")
            h = int(rng.choice(rep))
            sample = np.sort(rng.choice(wl.seq_len, 300, replace=False))
            qh, kh, vh = _np(q[0, :, h]), _np(k[0, :, h]), _np(v[0, :, h])
            ref, _ = O.anchor_attention(qh, kh, vh, wl.frames, wl.rows, wl.cols, wl.anchors, rows=sample)
            _assert_close(_np(out[0, torch.as_tensor(sample, device=q.device), h]), ref, "bf16")
            near = O.nearest_anchor_rows(wl.rows, wl.anchors)
            o = out.view(1, wl.frames, wl.rows, wl.cols, wl.heads, wl.head_dim)[..., list(rep), :]
            for rho in range(wl.rows):
                assert torch.equal(o[:, :, rho], o[:, :, near[rho]])
            del q, k, v, out


# ------------------------------------------------------- fused dual path (one launch)

@pytest.mark.parametrize("d,frames,rows,cols,anchors,batch", [
    (128, 2, 8, 64, (0, 4), 1),          # N = 1024: 8 full blocks, 2 anchor tiles per head
    (128, 3, 9, 40, (1, 4, 7), 2),       # N = 1080: ragged last block (56 tokens), ragged anchor tile; 2 batches
    (64, 3, 9, 40, (2, 6), 1),           # head_dim 64, ties broken to the lower anchor
])
def test_fused_dual_path(C, d, frames, rows, cols, anchors, batch):
    """A dictionary carrying the anchor geometry runs the dual path in one
    launch over a joint schedule: every row matches the oracle (block-sparse
    heads with their LSE, anchor heads with the broadcast), and the result is
    bitwise the one of the two-launch path (each work item is computed the
    same way whatever CTA runs it)."""
    n, h, block = frames * rows * cols, 5, 128
    nb = O.num_blocks(n, block)
    q, k, v = W.make_qkv(21, batch, n, h, d, "bf16", 1.0, "cuda")
    rep_heads = (1, 3)
    masks = _random_masks(9, h, nb, 0.45)
    masks = [None if i in rep_heads else masks[i] for i in range(h)]
    rp, ci, rep = C.masks_to_layer_csr(masks, h, nb)
    fused = torch.full_like(q, float("nan"))
    two = torch.full_like(q, float("nan"))
    lse_f = torch.full((batch, h, n), float("nan"), device="cuda")
    lse_t = torch.full((batch, h, n), float("nan"), device="cuda")
    with C.MaskDictionary(2, 1, h, nb, nb, block, 2 * max(1, ci.size)) as dg, \
            C.MaskDictionary(1, 1, h, nb, nb, block, max(1, ci.size)) as dp:
        dg.set_anchor_geometry(frames, rows, cols, anchors)
        dg.set_layer(1, 0, rp, ci, rep)
        dp.set_layer(0, 0, rp, ci, rep)
        C.calibatt_dual_path_attn(q, k, v, fused, dg, 1, 0, frames, rows, cols, anchors, block, lse=lse_f)
        C.calibatt_dual_path_attn(q, k, v, two, dp, 0, 0, frames, rows, cols, anchors, block, lse=lse_t)
        _check_status(C)
    assert torch.equal(fused, two)
    sparse = [i for i in range(h) if i not in rep_heads]
    assert torch.equal(lse_f[:, sparse], lse_t[:, sparse])
    for bb in range(batch):
        qn, kn, vn = _np(q)[bb], _np(k)[bb], _np(v)[bb]
        got = _np(fused)[bb]
        for i in range(h):
            if i in rep_heads:
                ref, _ = O.anchor_attention(qn[:, i], kn[:, i], vn[:, i], frames, rows, cols, anchors)
            else:
                ref, ref_lse = O.block_sparse_attention(qn[:, i], kn[:, i], vn[:, i], masks[i], block)
                np.testing.assert_allclose(lse_f[bb, i].cpu().numpy(), ref_lse, atol=2e-2)
            _assert_close(got[:, i], ref, "bf16")


def test_fused_geometry_rules(C):
    """The geometry is checked and must come before the first layer; a call
    whose geometry differs from the dictionary's takes the two-launch path."""
    n, h, nb = 1024, 2, 8
    rp, ci, rep = C.masks_to_layer_csr([np.eye(nb, dtype=bool), None], h, nb)
    with C.MaskDictionary(1, 1, h, nb, nb, 128, ci.size) as dg:
        with pytest.raises(C.CalibattError):
            dg.set_anchor_geometry(2, 8, 32, (0, 4))       # 512 tokens: not the dictionary's 8 blocks
        with pytest.raises(C.CalibattError):
            dg.set_anchor_geometry(2, 8, 64, (4, 0))       # not ascending
        dg.set_anchor_geometry(2, 8, 64, (0, 4))
        with pytest.raises(C.CalibattError):
            dg.set_anchor_geometry(2, 8, 64, (0, 4))       # only once
        dg.set_layer(0, 0, rp, ci, rep)
        q, k, v = W.make_qkv(3, 1, n, h, 128, "bf16", 1.0, "cuda")
        a, b = torch.empty_like(q), torch.empty_like(q)
        C.calibatt_dual_path_attn(q, k, v, a, dg, 0, 0, 2, 8, 64, (0, 4))      # one launch
        C.calibatt_dual_path_attn(q, k, v, b, dg, 0, 0, 2, 8, 64, (1, 4))      # other anchors: two launches
        _check_status(C)
        assert torch.equal(a[:, :, 0], b[:, :, 0])                           # the sparse head agrees
        qn, kn, vn = _np(q)[0], _np(k)[0], _np(v)[0]
        ref, _ = O.anchor_attention(qn[:, 1], kn[:, 1], vn[:, 1], 2, 8, 64, (1, 4))
        _assert_close(_np(b)[0][:, 1], ref, "bf16")
    with C.MaskDictionary(1, 1, h, nb, nb, 128, ci.size) as dl:
        dl.set_layer(0, 0, rp, ci, rep)
        with pytest.raises(C.CalibattError):
            dl.set_anchor_geometry(2, 8, 64, (0, 4))       # after a layer


# ------------------------------------------------------- spatial repetition

def _similarity(C, q, k, frames, rows, cols, anchors):
    b, n, h, _ = q.shape
    ws = torch.empty(C.calibatt_spatial_similarity_workspace_size(q) // 4, dtype=torch.float32, device=q.device)
    sim = torch.full((b, h, frames, rows), float("nan"), dtype=torch.float32, device=q.device)
    C.calibatt_spatial_similarity(q, k, sim, ws, frames, rows, cols, anchors)
    _check_status(C)
    return sim


@pytest.mark.parametrize("dtype,d,frames,rows,cols,anchors,batch,heads", [
    ("fp32", 64, 2, 8, 16, (0, 4), 1, 2),              # the tiny layout
    ("bf16", 128, 3, 9, 40, (1, 4, 7), 2, 3),          # 40 columns, two batches, three anchors
    ("bf16", 64, 2, 6, 100, (2,), 1, 2),               # 100 columns: two column passes
])
def test_spatial_similarity_matches_oracle(C, dtype, d, frames, rows, cols, anchors, batch, heads):
    n = frames * rows * cols
    q, k, _ = W.make_qkv(41, batch, n, heads, d, dtype, 1.0, "cuda")
    sim = _similarity(C, q, k, frames, rows, cols, anchors)
    again = _similarity(C, q, k, frames, rows, cols, anchors)
    assert torch.equal(sim, again)                                    # fixed summation orders
    got = sim.cpu().numpy().astype(np.float64)
    for bb in range(batch):
        for hh in range(heads):
            ref = O.spatial_similarity(_np(q[bb, :, hh]), _np(k[bb, :, hh]), frames, rows, cols, anchors)
            assert np.abs(got[bb, hh] - ref).max() <= 1e-4, np.abs(got[bb, hh] - ref).max()
    assert np.abs(got[:, :, :, list(anchors)] - 1.0).max() <= 1e-5


def test_spatial_similarity_720p_sampled_and_flags(C):
    """Two heads of the 720p layout (75,600 tokens), sampled (frame, row)
    scores against the oracle; then the flags of three prompts' scores
    against repetition_flags on the same scores (threshold between the heads'
    means, so both outcomes occur)."""
    wl = W.WORKLOADS["720p"]
    heads = 2
    sims = []
    for prompt in range(3):
        q, k, _ = W.make_qkv(500 + prompt, 1, wl.seq_len, heads, wl.head_dim, "bf16", wl.input_std * 2.0, "cuda")
        if prompt == 0:
            # make head 1 strongly repetitive: every row of a frame repeats its nearest anchor row's queries
            near = O.nearest_anchor_rows(wl.rows, wl.anchors)
            qv = q.view(1, wl.frames, wl.rows, wl.cols, heads, wl.head_dim)
            qv[:, :, :, :, 1] = qv[:, :, torch.as_tensor(near, device=q.device), :, 1]
        sim = _similarity(C, q, k, wl.frames, wl.rows, wl.cols, wl.anchors)
        if prompt == 0:
            rng = np.random.default_rng(3)
            pairs = [(0, 0), (int(rng.integers(wl.frames)), int(rng.integers(wl.rows))), (wl.frames - 1, wl.rows - 1)]
            for hh in range(heads):
                ref = O.spatial_similarity(_np(q[0, :, hh]), _np(k[0, :, hh]), wl.frames, wl.rows, wl.cols,
                                           wl.anchors, only=pairs)
                for f, rho in pairs:
                    got = float(sim[0, hh, f, rho])
                    assert abs(got - ref[f, rho]) <= 1e-4, (hh, f, rho, got, ref[f, rho])
            assert float(sim[0, 1].min()) > 0.999999
        sims.append(sim[0])
        del q, k
    stack = torch.stack(sims)                                          # [prompts, heads, frames, rows]
    ref_mean, _ = O.repetition_flags(stack.cpu().numpy(), 0.0)
    thr = float(ref_mean.mean())
    mean, flags = C.calibatt_repetition_flags(stack, thr)
    _check_status(C)
    ref_mean, ref_flags = O.repetition_flags(stack.cpu().numpy(), thr)
    assert np.abs(mean.cpu().numpy() - ref_mean).max() <= 1e-6
    assert np.array_equal(flags.cpu().numpy().astype(bool), ref_flags)
    assert ref_flags.any() and not ref_flags.all()


# ------------------------------------------- bitmap and interval dictionaries

FORMATS = ("lists", "bitmap", "intervals")


def _dictionary(C, fmt, T, L, h, nb, block, rp, ci, extra_capacity=1):
    """An empty dictionary of format `fmt` with room for `extra_capacity`
    layers like (rp, ci): blocks for index lists, intervals for the interval
    format, nothing for bitmaps."""
    if fmt == "intervals":
        return C.MaskDictionary(T, L, h, nb, nb, block, max(1, extra_capacity * C.count_intervals(rp, ci)),
                                intervals=True)
    return C.MaskDictionary(T, L, h, nb, nb, block, max(1, extra_capacity * ci.size), bitmap=fmt == "bitmap")


@pytest.mark.parametrize("d,n,h", [(128, 1000, 3), (64, 4100, 2)])  # ragged; 33 blocks -> 2 words per row
def test_compact_dictionaries_match_lists(C, d, n, h):
    """Bitmap and interval dictionaries give bitwise the results of the
    index-list one: sparse call with LSE (an empty row, a row keeping every
    block, single-block runs and the ragged last key block included) and the
    fused dual path."""
    q, k, v = W.make_qkv(61, 1, n, h, d, "bf16", 1.0, "cuda")
    nb = O.num_blocks(n, 128)
    masks = _random_masks(62, h, nb, 0.4, empty_row_head=1)
    masks[0][:, nb - 1] = True                                  # ragged last key block kept by every row
    masks[0][2, :] = True                                       # one run over the whole row
    masks[h - 1][3, :] = np.arange(nb) % 2 == 0                 # runs of one block each
    rp, ci, rep = C.masks_to_layer_csr(masks, h, nb)
    outs, lses = [], []
    for fmt in FORMATS:
        out = torch.full_like(q, float("nan"))
        lse = torch.full((1, h, n), float("nan"), device="cuda")
        with _dictionary(C, fmt, 1, 1, h, nb, 128, rp, ci) as dct:
            dct.set_layer(0, 0, rp, ci, rep)
            C.calibatt_block_sparse_attn(q, k, v, out, dct, 0, 0, 128, lse=lse)
            _check_status(C)
            assert dct.layer_info(0, 0)["retained_tiles"] == sum(int(m.sum()) for m in masks)
            assert dct.info()["nnz"] == ci.size
        outs.append(out)
        lses.append(lse)
    for i in (1, 2):
        assert torch.equal(outs[0], outs[i]), FORMATS[i]
        assert torch.equal(lses[0], lses[i]), FORMATS[i]
    ref, _ = O.block_sparse_attention_bnhd(_np(q), _np(k), _np(v), masks, 128, seq_len=n)
    _assert_close(_np(outs[2]), ref, "bf16")
    # fused dual path over each format
    frames, rows, cols = (2, 5, n // 10) if n % 10 == 0 else (1, 41, 100)
    assert frames * rows * cols == n
    dmasks = [None if i == h - 1 else masks[i] for i in range(h)]
    rp2, ci2, rep2 = C.masks_to_layer_csr(dmasks, h, nb)
    res = []
    for fmt in FORMATS:
        out = torch.full_like(q, float("nan"))
        with _dictionary(C, fmt, 1, 1, h, nb, 128, rp2, ci2) as dct:
            dct.set_anchor_geometry(frames, rows, cols, (1, 3) if rows == 5 else (10, 30))
            dct.set_layer(0, 0, rp2, ci2, rep2)
            C.calibatt_dual_path_attn(q, k, v, out, dct, 0, 0, frames, rows, cols, (1, 3) if rows == 5 else (10, 30))
            _check_status(C)
        res.append(out)
    assert torch.equal(res[0], res[1]) and torch.equal(res[0], res[2])


def _compact_reference(q, k, v, n, r, cols, block=128):
    """Oracle output and LSE of query block r whose skip list is `cols`: plain
    attention of its rows over exactly the keys of the listed blocks (the
    retained key set; gathering it is index selection only)."""
    rows = np.arange(r * block, min(n, (r + 1) * block))
    keys = np.concatenate([np.arange(c * block, min(n, (c + 1) * block)) for c in cols])
    kt = torch.as_tensor(keys, device=k.device)
    qr = _f32(q[0, torch.as_tensor(rows, device=q.device), 0])
    ref, lse = O.attention_rows(qr, _f32(k[0, kt, 0]), _f32(v[0, kt, 0]), len(keys), O.default_scale(q.shape[-1]))
    return rows, ref, lse


def _check_rows(C, out, lse, q, k, v, n, lists, sample):
    for r in sample:
        rows, ref, ref_lse = _compact_reference(q, k, v, n, r, lists[r])
        rt = torch.as_tensor(rows, device=out.device)
        _assert_close(_np(out[0, rt, 0]), ref, "bf16")
        assert np.abs(lse[0, 0, rt].cpu().numpy() - ref_lse).max() < 2e-2


def test_longest_sequence_of_index_lists(C):
    """The largest problem the index-list dictionary takes: 65,535 blocks of 128
    (16-bit block indices), N = 8,388,429 tokens with a ragged last block of 77
    tokens and NaN rows behind it, one head; sampled query blocks against the
    oracle over exactly their retained keys."""
    nb, block = 65535, 128
    n = (nb - 1) * block + 77
    qa, ka, va = W.make_qkv(41, 1, n, 1, 128, "bf16", 1.0, "cuda", seq_alloc=nb * block)
    q, k, v = qa[:, :n], ka[:, :n], va[:, :n]
    rng = np.random.default_rng(7)
    extra = rng.integers(0, nb, (nb, 5))
    lists = []
    for r in range(nb):
        c = [r, 0, *extra[r].tolist()] + ([nb - 1] if r % 1000 == 0 else [])
        lists.append(np.unique(np.asarray(c, np.int32)))
    row_ptr = np.zeros((1, nb + 1), np.int32)
    row_ptr[0, 1:] = np.cumsum([len(c) for c in lists])
    col = np.concatenate(lists)
    out = torch.full_like(qa, float("nan"))
    lse = torch.full((1, 1, n), float("nan"), device="cuda")
    with C.MaskDictionary(1, 1, 1, nb, nb, block, col.size) as dct:
        dct.set_layer(0, 0, row_ptr, col, None)
        C.calibatt_block_sparse_attn(q, k, v, out[:, :n], dct, 0, 0, block, lse=lse)
        _check_status(C)
    assert torch.isnan(out[:, n:]).all(), "padding rows of the output were written"
    _check_rows(C, out, lse, q, k, v, n, lists, [0, 1, 31000, nb - 2, nb - 1])
    del qa, ka, va, q, k, v, out
    torch.cuda.empty_cache()


def test_longest_bitmap_row(C):
    """The largest bitmap and interval dictionary row: 2,048 key blocks, N =
    262,066 (ragged last block of 50 tokens), one query block keeping every key
    block and others keeping few; bitwise equal to the index-list dictionary
    and against the oracle."""
    nb, block = 2048, 128
    n = (nb - 1) * block + 50
    q, k, v = W.make_qkv(42, 1, n, 1, 128, "bf16", 1.0, "cuda")
    rng = np.random.default_rng(8)
    masks = rng.random((nb, nb)) < 0.01
    masks[np.arange(nb), np.arange(nb)] = True
    masks[777, :] = True                      # the longest row: all 2,048 key blocks
    masks[5, :] = False                       # an empty row
    rp, ci, rep = C.masks_to_layer_csr([masks], 1, nb)
    outs, lses = [], []
    for fmt in FORMATS:
        out = torch.full_like(q, float("nan"))
        lse = torch.full((1, 1, n), float("nan"), device="cuda")
        with _dictionary(C, fmt, 1, 1, 1, nb, block, rp, ci) as dct:
            dct.set_layer(0, 0, rp, ci, rep)
            C.calibatt_block_sparse_attn(q, k, v, out, dct, 0, 0, block, lse=lse)
            _check_status(C)
        outs.append(out)
        lses.append(lse)
    for i in (1, 2):
        assert torch.equal(outs[0], outs[i]) and torch.equal(lses[0], lses[i]), FORMATS[i]
    lists = [np.nonzero(masks[r])[0] for r in range(nb)]
    _check_rows(C, outs[1], lses[1], q, k, v, n, lists, [0, 777, 1500, nb - 1])
    assert (outs[1][0, 5 * 128:6 * 128].float() == 0).all() and torch.isneginf(lses[1][0, 0, 5 * 128:6 * 128]).all()


def test_bitmap_dictionary_size_and_rules(C):
    """Device bytes of the two formats at the 720p layer, and the bitmap
    format's limits."""
    wl = W.WORKLOADS["720p"]
    nb = wl.num_blocks
    masks, _ = W.workload_masks(wl, heads=range(4))
    rp, ci, rep = C.masks_to_layer_csr([masks[i] for i in range(4)], 4, nb)
    with C.MaskDictionary(2, 2, 4, nb, nb, 128, 4 * ci.size) as dl, \
            C.MaskDictionary(2, 2, 4, nb, nb, 128, bitmap=True) as db:
        bl, bb = dl.info()["device_bytes"], db.info()["device_bytes"]
        # bitmap words, the work items and their consumption order, CTA offsets, the ticket counters
        assert bb == (4 * 4 * nb * ((nb + 31) // 32) * 4 + 2 * 4 * 4 * nb * 4 + 4 * (db.info()["num_ctas"] + 1) * 4
                      + 64 * 4)
        db.set_layer(1, 1, rp, ci, rep)
        assert db.info()["nnz"] == ci.size
        assert bb < bl
        # CUDA-core path (fp32) cannot read a bitmap dictionary
        q = torch.zeros((1, wl.seq_len, 4, 128), dtype=torch.float32, device="cuda")
        with pytest.raises(C.CalibattError):
            C.calibatt_block_sparse_attn(q, q, q, q, db, 1, 1, 128)
    with pytest.raises(C.CalibattError):
        C.MaskDictionary(1, 1, 1, 4096, 4096, 128, bitmap=True)    # more than 2048 blocks per row


def test_interval_dictionary_size_and_rules(C):
    """Device bytes of the interval format at the 720p layer against index
    lists, its capacity counted in intervals, and its limits."""
    wl = W.WORKLOADS["720p"]
    nb = wl.num_blocks
    masks, _ = W.workload_masks(wl, heads=range(4))
    rp, ci, rep = C.masks_to_layer_csr([masks[i] for i in range(4)], 4, nb)
    runs = C.count_intervals(rp, ci)
    assert runs < ci.size / 3        # band + first frame in a few runs; random top-up blocks mostly alone
    with C.MaskDictionary(2, 2, 4, nb, nb, 128, 4 * ci.size) as dl, \
            C.MaskDictionary(2, 2, 4, nb, nb, 128, 4 * runs, intervals=True) as di:
        assert di.info()["device_bytes"] < dl.info()["device_bytes"] / 2
        di.set_layer(1, 1, rp, ci, rep)
        assert di.info()["nnz"] == ci.size
        q = torch.zeros((1, wl.seq_len, 4, 128), dtype=torch.float32, device="cuda")
        with pytest.raises(C.CalibattError):                         # the CUDA-core path reads lists only
            C.calibatt_block_sparse_attn(q, q, q, q, di, 1, 1, 128)
    with C.MaskDictionary(1, 1, 4, nb, nb, 128, runs - 1, intervals=True) as small:
        with pytest.raises(C.CalibattError) as e:                    # capacity is counted in intervals
            small.set_layer(0, 0, rp, ci, rep)
        assert "intervals" in str(e.value)
    with pytest.raises(C.CalibattError):
        C.MaskDictionary(1, 1, 1, 4096, 4096, 128, 10, intervals=True)   # more than 2048 blocks per row


@pytest.mark.parametrize("fmt", FORMATS)
def test_dictionary_save_load_round_trip(C, tmp_path, fmt):
    """calibatt_dict_save / calibatt_dict_load: a dictionary with the anchor
    geometry, three of its four records set (repetitive heads included), written
    and read back with another persistent grid; every record's counts match and
    its single-path and dual-path outputs are bitwise those of the original;
    damaged files are refused."""
    frames, rows, cols, anchors = 3, 10, 100, (2, 7)
    n, h, d, block = frames * rows * cols, 4, 128, 128
    nb = O.num_blocks(n, block)
    q, k, v = W.make_qkv(51, 1, n, h, d, "bf16", 1.0, "cuda")
    path = tmp_path / "masks.dict"
    records = {(0, 0): (0, 3), (0, 1): (), (1, 1): (1,)}           # (t, l) -> repetitive heads
    with C.MaskDictionary(2, 2, h, nb, nb, block, 4 * h * nb * nb, bitmap=fmt == "bitmap",
                          intervals=fmt == "intervals") as dct:
        dct.set_anchor_geometry(frames, rows, cols, anchors)
        for i, ((t, l), rep) in enumerate(records.items()):
            masks = _random_masks(60 + i, h, nb, 0.4)
            masks = [None if hh in rep else masks[hh] for hh in range(h)]
            rp, ci, rf = C.masks_to_layer_csr(masks, h, nb)
            dct.set_layer(t, l, rp, ci, rf)
        dct.save(path)
        ref = {}
        for (t, l) in records:
            o1, o2 = torch.zeros_like(q), torch.zeros_like(q)
            C.calibatt_block_sparse_attn(q, k, v, o1, dct, t, l, block)
            C.calibatt_dual_path_attn(q, k, v, o2, dct, t, l, frames, rows, cols, anchors, block)
            ref[t, l] = (o1, o2, dct.layer_info(t, l))
        info = dct.info()
        _check_status(C)
    loaded = C.MaskDictionary.load(path, num_ctas=11)
    try:
        assert loaded.info()["nnz"] == info["nnz"] and loaded.info()["num_ctas"] == 11
        for (t, l), (o1, o2, li) in ref.items():
            g1, g2 = torch.zeros_like(q), torch.zeros_like(q)
            C.calibatt_block_sparse_attn(q, k, v, g1, loaded, t, l, block)
            C.calibatt_dual_path_attn(q, k, v, g2, loaded, t, l, frames, rows, cols, anchors, block)
            _check_status(C)
            assert loaded.layer_info(t, l) == li
            assert torch.equal(g1, o1) and torch.equal(g2, o2)
        with pytest.raises(C.CalibattError):
            loaded.layer_info(1, 0)                                 # the record never set stays unset
    finally:
        loaded.close()
    raw = path.read_bytes()
    damaged = tmp_path / "damaged.dict"
    for blob in (raw[:-1], raw + b"\0", raw[:len(raw) // 2],
                 raw[:len(raw) // 2] + bytes([raw[len(raw) // 2] ^ 0x10]) + raw[len(raw) // 2 + 1:]):
        damaged.write_bytes(blob)
        with pytest.raises(C.CalibattError) as e:
            C.MaskDictionary.load(damaged)
        assert e.value.status == C.ERR_INVALID_ARG
    with pytest.raises(C.CalibattError):
        with C.MaskDictionary(1, 1, 1, 4, 4, 128, 16) as small:
            small.save(tmp_path / "no_such_dir" / "x.dict")


def test_host_buffer_entry_point(C):
    """calibatt_block_sparse_attn_host: host inputs copied in, attention, output
    copied out, in stream order; equal to the device-buffer call."""
    n, h, d = 1000, 2, 128
    q, k, v = W.make_qkv(71, 1, n, h, d, "bf16", 1.0, "cuda")
    nb = O.num_blocks(n, 128)
    masks = _random_masks(72, h, nb, 0.5)
    rp, ci, rep = C.masks_to_layer_csr(masks, h, nb)
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    ho = torch.full_like(q, float("nan"), device="cpu").pin_memory()
    dq, dk, dv, do = (torch.empty_like(q) for _ in range(4))
    ref_out = torch.empty_like(q)
    s = torch.cuda.Stream()
    with C.MaskDictionary(1, 1, h, nb, nb, 128, ci.size) as dct:
        dct.set_layer(0, 0, rp, ci, rep)
        C.calibatt_block_sparse_attn_host(hq, hk, hv, ho, dq, dk, dv, do, dct, 0, 0, 128, stream=s)
        s.synchronize()
        C.calibatt_block_sparse_attn(q, k, v, ref_out, dct, 0, 0, 128)
        _check_status(C)
    assert torch.equal(ho, ref_out.cpu())
    assert torch.equal(dq, q)


@pytest.mark.parametrize("batch", [1, 2])
def test_head_major_storage_matches_token_major(C, batch):
    """The calls take any strides: the same logical [batch, N, heads, D]
    tensors stored head-major ([batch, heads, N, D] in memory) give bitwise
    the outputs of token-major storage -- block-sparse and fused dual-path
    dictionary calls, the anchor call with its split workspace, and the block
    energy."""
    frames, rows, cols, anchors = 3, 10, 100, (2, 7)
    n, h, d, block = frames * rows * cols, 4, 128, 128
    nb = O.num_blocks(n, block)
    q, k, v = W.make_qkv(95 + batch, batch, n, h, d, "bf16", 1.0, "cuda")

    def head_major(t):
        return t.permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)

    qh, kh, vh = head_major(q), head_major(k), head_major(v)
    assert qh.stride(2) == n * d and qh.stride(1) == d and torch.equal(qh, q)
    masks = _random_masks(96, h, nb, 0.45)
    masks[1] = None
    rp, ci, rep = C.masks_to_layer_csr(masks, h, nb)
    nbytes = C.calibatt_anchor_attn_workspace_size(q, frames, rows, cols, len(anchors), h)
    ws = torch.empty(max(1, nbytes // 4), device="cuda")
    outs = {}
    with C.MaskDictionary(1, 1, h, nb, nb, block, ci.size) as dct:
        dct.set_anchor_geometry(frames, rows, cols, anchors)
        dct.set_layer(0, 0, rp, ci, rep)
        for name, (a, b_, c_) in (("token", (q, k, v)), ("head", (qh, kh, vh))):
            o_s, o_d, o_a = (torch.full_like(a, float("nan")) for _ in range(3))
            C.calibatt_block_sparse_attn(a, b_, c_, o_s, dct, 0, 0, block)
            C.calibatt_dual_path_attn(a, b_, c_, o_d, dct, 0, 0, frames, rows, cols, anchors, block)
            C.calibatt_anchor_attn(a, b_, c_, o_a, frames, rows, cols, anchors, list(range(h)),
                                   workspace=ws if nbytes else None)
            e = torch.full((batch, h, nb, nb), float("nan"), device="cuda")
            e_ws = torch.empty(C.calibatt_block_energy_workspace_size(a) // 4, device="cuda")
            C.calibatt_block_energy(a, b_, e, e_ws, block)
            _check_status(C)
            assert o_a.stride() == a.stride()
            outs[name] = (o_s, o_d, o_a, e)
    sparse = [i for i in range(h) if i != 1]
    ts, td, ta, te = outs["token"]
    hs, hd, ha, he = outs["head"]
    assert torch.equal(ts[:, :, sparse], hs[:, :, sparse])     # head 1 (repetitive) is not written there
    assert torch.equal(td, hd) and torch.equal(ta, ha) and torch.equal(te, he)
    ref, _ = O.block_sparse_attention_bnhd(_np(q), _np(k), _np(v), masks, block, heads=sparse)
    _assert_close(_np(hs)[:, :, sparse], ref, "bf16")


def test_calls_replay_in_a_cuda_graph(C):
    """The block-sparse, the fused dual-path and the anchor call with its
    split workspace enqueue only kernels and memsets on the caller's stream
    (no host sync, no allocation after the first call), so they capture into
    a CUDA graph; replays compute on whatever the input buffers hold, bitwise
    equal to direct calls."""
    frames, rows, cols, anchors = 3, 10, 100, (2, 7)
    n, h, d, block = frames * rows * cols, 3, 128, 128
    nb = O.num_blocks(n, block)
    q, k, v = W.make_qkv(61, 1, n, h, d, "bf16", 1.0, "cuda")
    q2, k2, v2 = W.make_qkv(62, 1, n, h, d, "bf16", 1.0, "cuda")
    masks = _random_masks(63, h, nb, 0.4)
    rp, ci, rep = C.masks_to_layer_csr([masks[0], None, masks[2]], h, nb)
    with C.MaskDictionary(1, 1, h, nb, nb, block, ci.size) as dct:
        dct.set_anchor_geometry(frames, rows, cols, anchors)
        dct.set_layer(0, 0, rp, ci, rep)
        o_sparse, o_dual, o_anchor = torch.zeros_like(q), torch.zeros_like(q), torch.zeros_like(q)
        a_ws = torch.empty(C.calibatt_anchor_attn_workspace_size(q, frames, rows, cols, len(anchors), 1) // 4,
                           device="cuda")
        assert a_ws.numel() > 0                         # 5 tiles on the SMs: split in key ranges

        def step():
            C.calibatt_block_sparse_attn(q, k, v, o_sparse, dct, 0, 0, block)
            C.calibatt_dual_path_attn(q, k, v, o_dual, dct, 0, 0, frames, rows, cols, anchors, block)
            C.calibatt_anchor_attn(q, k, v, o_anchor, frames, rows, cols, anchors, [1], workspace=a_ws)

        step()                                          # warm-up outside the capture
        torch.cuda.synchronize()
        outs = (o_sparse, o_dual, o_anchor)
        direct = tuple(o.clone() for o in outs)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        for o in outs:
            o.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert all(torch.equal(o, r) for o, r in zip(outs, direct))
        for dst, src in ((q, q2), (k, k2), (v, v2)):     # new inputs in the captured buffers
            dst.copy_(src)
        graph.replay()
        torch.cuda.synchronize()
        got = tuple(o.clone() for o in outs)
        step()
        _check_status(C)
        assert all(torch.equal(g, o) for g, o in zip(got, outs))
        assert not torch.equal(got[1], direct[1]) and not torch.equal(got[2], direct[2])
        del graph


def test_bounded_wait_runs_out_and_context_survives(C):
    """A wait that nothing satisfies ends after the configured limit with the
    timeout status (wait point 15), no fault and no hang; the status clears
    and the next attention call runs normally."""
    import time
    C.set_wait_timeout_ms(50)
    try:
        t0 = time.time()
        C.debug_bounded_wait()
        code = C.device_status()                       # synchronises, reads and clears
        assert code & 0xFF == 4 and (code >> 8) == 15, hex(code)
        assert time.time() - t0 < 5.0
        assert C.device_status() == 0
    finally:
        C.set_wait_timeout_ms(4000)
    n, h, d = 512, 2, 128
    q, k, v = W.make_qkv(81, 1, n, h, d, "bf16", 1.0, "cuda")
    masks = _random_masks(82, h, O.num_blocks(n, 128), 0.5)
    out, _ = _run_sparse(C, q, k, v, masks, 128)
    ref, _ = O.block_sparse_attention_bnhd(_np(q), _np(k), _np(v), masks, 128)
    _assert_close(_np(out), ref, "bf16")


def test_anchor_calls_in_flight_with_their_own_workspaces(C):
    """Anchor calls with split workspaces issued on three streams at once,
    each stream with its own workspace, 8 rounds: every output is bitwise the
    one of a call made alone (no counter or partial output is shared)."""
    frames, rows, cols, anchors, h, d = 4, 9, 100, (2, 6), 22, 128
    n = frames * rows * cols
    q, k, v = W.make_qkv(83, 1, n, h, d, "bf16", 1.0, "cuda")
    heads = list(range(h))
    nbytes = C.calibatt_anchor_attn_workspace_size(q, frames, rows, cols, len(anchors), h)
    assert nbytes > 0
    ref = torch.zeros_like(q)
    ws0 = torch.empty(nbytes // 4, device="cuda")
    C.calibatt_anchor_attn(q, k, v, ref, frames, rows, cols, anchors, heads, workspace=ws0)
    _check_status(C)
    streams = [torch.cuda.Stream() for _ in range(3)]
    wss = [torch.empty(nbytes // 4, device="cuda") for _ in streams]
    outs = [torch.zeros_like(q) for _ in streams]
    torch.cuda.synchronize()
    for _ in range(8):
        for st, ws, o in zip(streams, wss, outs):
            C.calibatt_anchor_attn(q, k, v, o, frames, rows, cols, anchors, heads, workspace=ws, stream=st)
    torch.cuda.synchronize()
    _check_status(C)
    for o in outs:
        assert torch.equal(o, ref)


def test_dictionary_calls_in_flight_on_several_streams(C):
    """Dictionary calls hand out work through per-call counters (64 per
    dictionary, taken round-robin): calls on one dictionary issued on three
    streams at once, 72 of them in all (the pool wraps), each give bitwise the
    output of a call made alone; block-sparse and fused dual-path calls."""
    frames, rows, cols, anchors = 2, 10, 64, (2, 7)
    n, h, d, block = frames * rows * cols, 4, 128, 128
    nb = O.num_blocks(n, block)
    masks = _random_masks(81, h, nb, 0.5)
    masks[1] = None                                              # one head on the anchor path
    rp, ci, rep = C.masks_to_layer_csr(masks, h, nb)
    q, k, v = W.make_qkv(82, 1, n, h, d, "bf16", 1.0, "cuda")
    with C.MaskDictionary(1, 1, h, nb, nb, block, ci.size) as dct:
        dct.set_anchor_geometry(frames, rows, cols, anchors)
        dct.set_layer(0, 0, rp, ci, rep)
        ref_s, ref_d = torch.zeros_like(q), torch.zeros_like(q)
        C.calibatt_block_sparse_attn(q, k, v, ref_s, dct, 0, 0, block)
        C.calibatt_dual_path_attn(q, k, v, ref_d, dct, 0, 0, frames, rows, cols, anchors, block)
        _check_status(C)
        streams = [torch.cuda.Stream() for _ in range(3)]
        outs = [[torch.zeros_like(q), torch.zeros_like(q)] for _ in streams]
        for rnd in range(12):                                   # 12 rounds x 3 streams x 2 calls = 72
            for st, (os_, od) in zip(streams, outs):
                C.calibatt_block_sparse_attn(q, k, v, os_, dct, 0, 0, block, stream=st)
                C.calibatt_dual_path_attn(q, k, v, od, dct, 0, 0, frames, rows, cols, anchors, block, stream=st)
        torch.cuda.synchronize()
        _check_status(C)
    for os_, od in outs:
        assert torch.equal(os_, ref_s) and torch.equal(od, ref_d)
