"""The fused construction + selection call (losa_dense_mass_select) against
the separate calls and the oracle.

The fused call runs the selection's per-row cut inside the construction
kernel (one warpgroup per row, a bucketed cut) instead of in the selection
kernels (one warp per row for n <= 512, one CTA per row above). Per case:

  * o, lse and mass are bit for bit those of losa_dense_mass on the same
    inputs (the construction kernel's arithmetic is unchanged);
  * every array of the pattern (row_ptr, col_idx, retained_fx, total_fx,
    tile lists) is bit for bit that of losa_select on the same mass map,
    which for n <= 512 compares two different cut algorithms, and the tile
    order is the same up to ties;
  * the selection on sampled rows equals the oracle's selection run on the
    GPU's masses (LoSA abstract: the smallest key-block set per head and
    query block reaching tau; ubos.tech LoSA post, Phase 2), so the fused
    path is pinned to the pages without going through losa_select;
  * the sparse step on the fused pattern gives what it gives on the
    separate pattern.
"""
import dataclasses
import zlib

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def losa():
    assert torch.cuda.is_available()
    import block_sparse_attention_losa_b200 as m
    return m


def compare(losa, q, k, v, L, b, tau, out_dtype=torch.float32, sample_rows=32, seed=0):
    o1, lse1, m1 = losa.dense_mass(q, k, v, L, b, out_dtype=out_dtype)
    p1 = losa.select(m1, b, tau)
    o2, lse2, m2, p2 = losa.dense_mass_select(q, k, v, L, b, tau=tau, out_dtype=out_dtype)
    torch.cuda.synchronize()
    losa.check_status()
    assert torch.equal(o1, o2) and torch.equal(lse1, lse2) and torch.equal(m1, m2)
    e1, e2 = p1.export("cpu"), p2.export("cpu")
    for key in e1:
        if key != "tile_order":
            assert torch.equal(e1[key], e2[key]), key
    # The tile order is unique up to ties (tiles of one head with equal entry
    # counts are placed by atomics): both are permutations with the same
    # (head, entry count) sequence.
    n_qt = p1.n_tiles // (p1.B * p1.H)
    cnt = (e1["tile_ptr"][1:] - e1["tile_ptr"][:-1]).numpy()
    key_seq = lambda order: [(int(t) // n_qt, int(cnt[t])) for t in order]
    for e in (e1, e2):
        assert sorted(e["tile_order"].tolist()) == list(range(p1.n_tiles))
    assert key_seq(e1["tile_order"]) == key_seq(e2["tile_order"])
    # sampled rows against the oracle's selection on the GPU's masses
    n = m2.shape[-1]
    flat = m2.reshape(-1, n).cpu().numpy()
    rp = e2["row_ptr"].numpy()
    rng = np.random.default_rng(seed)
    rows = rng.choice(flat.shape[0], min(sample_rows, flat.shape[0]), replace=False)
    for r in sorted(set(rows.tolist()) | {flat.shape[0] - 1}):
        kept, C, S = O.select_row(O.to_fixed(flat[r]).tolist(), tau)
        assert e2["col_idx"][rp[r]:rp[r + 1]].tolist() == kept, r
        assert int(e2["retained_fx"][r]) == C and int(e2["total_fx"][r]) == S
    # the sparse step on either pattern
    s1 = losa.sparse_attn(q, k, v, L, p1, out_dtype=out_dtype)
    s2 = losa.sparse_attn(q, k, v, L, p2, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert torch.equal(s1[0], s2[0]) and torch.equal(s1[1], s2[1])
    p1.close()
    p2.close()
    return n


SHAPES = [
    # name, heads, d, grid, block, text, batch
    ("d128_b64_partial_tile", 3, 128, (3, 10, 13), 64, 0, 1),
    ("d64_b128_text", 2, 64, (2, 12, 20), 128, 30, 1),
    ("d128_b32_partial_tile", 2, 128, (3, 7, 9), 32, 0, 1),
    ("d64_b64_text", 2, 64, (4, 9, 11), 64, 20, 1),
    ("d128_b64_batch2", 2, 128, (2, 8, 16), 64, 0, 2),
    ("d128_b128_10_blocks", 2, 128, (4, 16, 20), 128, 0, 1),
    ("d64_b32_exact", 1, 64, (2, 8, 8), 32, 0, 1),
]


@pytest.mark.parametrize("name,heads,d,grid,block,text,batch", SHAPES, ids=[s[0] for s in SHAPES])
@pytest.mark.parametrize("tau", [0.5, 0.99, 1.0])
def test_fused_matches_separate_calls(losa, name, heads, d, grid, block, text, batch, tau):
    wl = W.custom(name, heads, d, grid, block, text_tokens=text, batch=batch, amplitude=1.2,
                  seed=zlib.crc32(name.encode()) % 1000)
    q, k, v = (t.cuda() for t in W.generate(wl, dtype=torch.bfloat16))
    compare(losa, q, k, v, wl.seq_len, block, tau)


@pytest.mark.parametrize("d,block", [(128, 64), (64, 32)])
def test_fused_on_fp32_inputs(losa, d, block):
    """The kind::tf32 construction kernels carry the same epilogue."""
    wl = W.custom("fused_tf32", 2, d, (3, 10, 13), block, amplitude=1.2, seed=31,
                  in_dtype="fp32")
    q, k, v = (t.cuda() for t in W.generate(wl, dtype=torch.float32))
    compare(losa, q, k, v, wl.seq_len, block, 0.95)


@pytest.mark.parametrize("d,block,grid", [(64, 32, (5, 60, 64)), (128, 32, (2, 50, 180))])
def test_fused_on_rows_of_more_than_512_blocks(losa, d, block, grid):
    """n = 600 and 563: above 512 both paths run the bucketed cut, the
    separate one with a 256-thread CTA per row, the fused one with a
    warpgroup."""
    wl = W.custom("fused_long", 1, d, grid, block, amplitude=1.0, seed=37)
    q, k, v = (t.cuda() for t in W.generate(wl, dtype=torch.bfloat16))
    n = compare(losa, q, k, v, wl.seq_len, block, 0.99, out_dtype=torch.bfloat16)
    assert n == wl.n_blocks


def test_fused_on_tied_masses(losa):
    """Q = K = 0: every key of a row weighs the same, so the masses of the
    full blocks tie exactly and the cut orders them by key-block index."""
    wl = W.custom("fused_ties", 2, 64, (3, 10, 13), 64, amplitude=1.0, seed=41)
    q, k, v = (t.cuda() for t in W.generate(wl, dtype=torch.bfloat16))
    q.zero_()
    k.zero_()
    compare(losa, q, k, v, wl.seq_len, 64, 0.7)


@pytest.mark.parametrize("name", ["wan2.1-1.3b", "hunyuanvideo"])
def test_fused_at_full_size(losa, name):
    """The Wan2.1-1.3B-shaped layer (n = 512: the separate path's warp cut
    against the fused bucketed cut) and 4 heads of the HunyuanVideo-shaped
    layer (n = 929), in the benchmark's launch configuration (bf16 out)."""
    wl = W.WORKLOADS[name]
    if name == "hunyuanvideo":
        wl = dataclasses.replace(wl, heads=4)
    q, k, v = W.generate(wl, device="cuda")
    compare(losa, q, k, v, wl.seq_len, wl.block, 0.99, out_dtype=torch.bfloat16,
            sample_rows=64)


def test_fused_call_reports_a_timeout_and_leaves_no_pattern(losa):
    """With a one-cycle wait limit the construction kernel gives up a wait:
    both warpgroups skip the cut, the call returns LOSA_ERR_TIMEOUT (read at
    its one synchronisation, which clears the status word) and no pattern,
    and the next call gives the normal result."""
    wl = W.custom("fused_abort", 4, 128, (2, 16, 64), 64, amplitude=1.2, seed=17)
    q, k, v = (t.cuda() for t in W.generate(wl, dtype=torch.bfloat16))
    L, b = wl.seq_len, wl.block
    losa.check_status()
    try:
        losa.set_wait_limit(1)
        with pytest.raises(losa.LosaError) as e:
            losa.dense_mass_select(q, k, v, L, b, tau=0.95)
        assert e.value.status == -4
    finally:
        losa.set_wait_limit(0)
    losa.check_status()
    compare(losa, q, k, v, L, b, 0.95)
