"""Stored patterns: losa_pattern_export and losa_pattern_import through the
C ABI (the frozen mask kept for reuse, ubos.tech LoSA post, Phase 2).

  * A selected pattern exported to host memory and imported again is the
    same pattern: the CSR and fixed-point sums bit for bit, the tile lists
    bit for bit, the tile order a valid order of the same keys, and the
    sparse kernel's O and lse on fresh inputs bit-identical.
  * A pattern that no GPU selection produced (the oracle's own selection on
    its fp64 masses, a hand-written band) runs the sparse step to the same
    tolerances as the parity tests, against the oracle's sparse attention
    with that pattern.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from test_gpu_parity import assert_lse_close, assert_o_close, check_tiles

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def losa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import block_sparse_attention_losa_b200 as m
    return m


CASES = [  # heads, d, grid, block, text tokens
    (2, 128, (3, 10, 13), 64, 0),
    (2, 64, (2, 8, 16), 32, 7),
    (1, 128, (4, 12, 12), 128, 0),
]


@pytest.mark.parametrize("heads,d,grid,block,text", CASES)
def test_export_import_round_trip(losa, heads, d, grid, block, text):
    wl = W.custom("io", heads, d, grid, block, text_tokens=text, amplitude=1.2, seed=31)
    q, k, v = W.generate(wl, dtype=torch.float32)
    qd, kd, vd = (t.to("cuda", torch.bfloat16) for t in (q, k, v))
    _, _, mass = losa.dense_mass(qd, kd, vd, wl.seq_len, block)
    pat = losa.select(mass, block, 0.9)
    ex = pat.export("cpu")
    imp = losa.import_pattern(ex["row_ptr"], ex["col_idx"], wl.batch, heads, wl.n_blocks, block,
                              retained_fx=ex["retained_fx"], total_fx=ex["total_fx"])
    ex2 = imp.export("cpu")
    assert (imp.nnz, imp.n_tiles, imp.tile_entries) == (pat.nnz, pat.n_tiles, pat.tile_entries)
    for key in ("row_ptr", "col_idx", "retained_fx", "total_fx", "tile_ptr", "tile_entry"):
        assert torch.equal(ex[key], ex2[key]), key
    check_tiles(ex2, imp, wl.n_blocks)

    q2, k2, v2 = W.drift(wl, (q, k, v), step=1, dtype=torch.float32)
    q2d, k2d, v2d = (t.to("cuda", torch.bfloat16) for t in (q2, k2, v2))
    o1, lse1 = losa.sparse_attn(q2d, k2d, v2d, wl.seq_len, pat)
    o2, lse2 = losa.sparse_attn(q2d, k2d, v2d, wl.seq_len, imp)
    torch.cuda.synchronize()
    losa.check_status()
    assert torch.equal(o1, o2)
    assert torch.equal(lse1, lse2)
    pat.close()
    imp.close()


def _sparse_against_oracle(losa, wl, row_ptr, col_idx, seed_step=1):
    q, k, v = W.generate(wl, dtype=torch.float32)
    q2, k2, v2 = W.drift(wl, (q, k, v), step=seed_step, dtype=torch.float32)
    imp = losa.import_pattern(row_ptr, col_idx, wl.batch, wl.heads, wl.n_blocks, wl.block)
    ex = imp.export("cpu")
    np.testing.assert_array_equal(ex["row_ptr"].numpy(), np.asarray(row_ptr))
    np.testing.assert_array_equal(ex["col_idx"].numpy(), np.asarray(col_idx))
    assert np.all(ex["retained_fx"].numpy() == -1) and np.all(ex["total_fx"].numpy() == -1)
    check_tiles(ex, imp, wl.n_blocks)
    o, lse = losa.sparse_attn(*(t.to("cuda", torch.bfloat16) for t in (q2, k2, v2)),
                              wl.seq_len, imp)
    torch.cuda.synchronize()
    losa.check_status()
    scale = 1 / math.sqrt(wl.head_dim)
    o_ref, lse_ref = O.sparse_attention(q2.double().numpy(), k2.double().numpy(),
                                        v2.double().numpy(), wl.seq_len, wl.block, scale,
                                        np.asarray(row_ptr), np.asarray(col_idx))
    assert_o_close(o, o_ref, wl.seq_len, what="sparse O (imported pattern)")
    assert_lse_close(lse, lse_ref, wl.seq_len)
    imp.close()


def test_import_of_the_oracles_own_selection(losa):
    wl = W.custom("io_oracle", 2, 128, (3, 10, 13), 64, amplitude=1.2, seed=33)
    q, k, _ = (t.double().numpy() for t in W.generate(wl, dtype=torch.float32))
    mass = O.block_mass(q, k, wl.seq_len, wl.block, 1 / math.sqrt(wl.head_dim))
    sel = O.select(mass, 0.95)
    _sparse_against_oracle(losa, wl, sel["row_ptr"], sel["col_idx"])


@pytest.mark.parametrize("block,d", [(32, 64), (64, 128), (128, 128)])
def test_import_of_a_banded_pattern(losa, block, d):
    # Query block I keeps key blocks I-1, I, I+1 and block 0 (a sink), a
    # pattern no mass map produced; ragged sequence (text tokens).
    wl = W.custom("io_band", 2, d, (2, 8, 12), block, text_tokens=5, amplitude=1.0, seed=35)
    n = wl.n_blocks
    row_ptr, cols = [0], []
    for _ in range(wl.batch * wl.heads):
        for I in range(n):
            keep = sorted({0, max(I - 1, 0), I, min(I + 1, n - 1)})
            cols.extend(keep)
            row_ptr.append(len(cols))
    _sparse_against_oracle(losa, wl, np.array(row_ptr), np.array(cols))
