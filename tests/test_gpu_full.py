"""The full-size workloads, in the launch configuration the benchmark times
(bf16 inputs and outputs), checked against the oracle.

Per workload, at every threshold the workload names (the Wan2.1-14B-shaped
layer is a sweep over tau in {0.95, 0.99, 0.999, 1.0}; LoSA abstract:
retained-mass threshold; legiblepapers.com FAQ Q4):

  * whole map: every mass row sums to 1 and is non-negative; every selected
    row keeps >= tau of its own fixed-point total, exactly; at tau = 1 the
    kept set is every positive-mass block;
  * selection bit-exact against the oracle run on the GPU's masses, on 16
    sampled rows per head plus the sampled query blocks below;
  * on PER_HEAD sampled query blocks of every head (the last, ragged block
    always included): dense O element by element within
    1e-2 + 2^-8 |O_ref| (bf16 output: the bound plus half an ulp), lse within
    1e-4, the block's masses within 1e-5, the kept set holding >= tau - 1e-5
    of the oracle's own fp64 masses, and the sparse step's O and lse on fresh
    (drifted) Q/K/V against the oracle over the retained keys;
  * mean |dO| <= 1e-3 over all sampled elements, for the dense output and
    for the sparse output at every tau.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from test_gpu_parity import LSE_ATOL, MASS_ATOL, O_MAX, O_MEAN

pytestmark = pytest.mark.gpu

PER_HEAD = 8          # sampled query blocks per head (O, lse, mass, sparse O)
SELECT_PER_HEAD = 16  # sampled rows per head for the selection-only check
RETAIN_SLACK = 1e-5   # oracle-mass retained >= tau - this


@pytest.fixture(scope="module")
def losa():
    assert torch.cuda.is_available()
    import block_sparse_attention_losa_b200 as m
    return m


class ErrAcc:
    """Elementwise bf16-output bound, plus the running mean of |delta|."""

    def __init__(self, what):
        self.what, self.total, self.count = what, 0.0, 0

    def add(self, got, ref):
        d = np.abs(got - ref)
        bound = O_MAX + 2.0 ** -8 * np.abs(ref)
        assert np.all(d <= bound), f"{self.what}: max excess {np.max(d - bound)}"
        self.total += float(d.sum())
        self.count += d.size

    def check_mean(self):
        mean = self.total / max(1, self.count)
        assert mean <= O_MEAN, f"{self.what}: mean |d| {mean}"
        return mean


def _rows(t, bb, h, rows):
    return t[bb, h, rows].to("cpu", torch.float64).numpy()


@pytest.mark.parametrize("name", ["wan2.1-1.3b", "cogvideox", "hunyuanvideo", "wan2.1-14b"])
def test_full_size_workload(losa, name):
    wl = W.WORKLOADS[name]
    L, Lp, b, d, n = wl.seq_len, wl.seq_pad, wl.block, wl.head_dim, wl.n_blocks
    scale = 1 / math.sqrt(d)
    q, k, v = W.generate(wl, device="cuda")
    o, lse, mass = losa.dense_mass(q, k, v, L, b, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    losa.check_status()
    # Every row of the mass map sums to 1 (fp32 sum of n entries).
    rs = mass.double().sum(-1)
    assert torch.max(torch.abs(rs - 1)).item() < 1e-4
    assert torch.all(mass >= 0).item()
    mass_cpu = mass.cpu().numpy()
    q2, k2, v2 = W.drift(wl, (q, k, v), step=1, device="cuda")

    samples = W.sample_query_blocks(wl, PER_HEAD, seed=99)
    sel_samples = W.sample_query_blocks(wl, SELECT_PER_HEAD, seed=7)
    row_of = lambda bb, h, I: (bb * wl.heads + h) * n + I

    # ---- per tau: selection (whole-map properties, sampled rows bit-exact)
    # and the sparse step; the sampled rows' results are kept on the host.
    kept_at, o2_at, lse2_at = {}, {}, {}
    for tau in wl.taus:
        pat = losa.select(mass, b, tau)
        ex = pat.export("cpu")
        t_fx = O.tau_fixed(tau)
        ret, tot = ex["retained_fx"].tolist(), ex["total_fx"].tolist()
        assert all((1 << 48) * c >= t_fx * s for c, s in zip(ret, tot))
        rp = ex["row_ptr"].numpy()
        assert np.all(np.diff(rp) >= 1)
        if tau == 1.0:
            x = O.to_fixed(mass_cpu).reshape(-1, n)
            pos = (x > 0).sum(axis=1)
            assert np.array_equal(np.diff(rp), np.maximum(pos, 1))
        for (bb, h, I) in sel_samples + samples:
            r = row_of(bb, h, I)
            kept, C, S = O.select_row(O.to_fixed(mass_cpu[bb, h, I]).tolist(), tau)
            assert ex["col_idx"][rp[r]:rp[r + 1]].tolist() == kept, (tau, bb, h, I)
            assert ret[r] == C and tot[r] == S
        o2, lse2 = losa.sparse_attn(q2, k2, v2, L, pat, out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        losa.check_status()
        for (bb, h, I) in samples:
            r = row_of(bb, h, I)
            rows = np.arange(I * b, min((I + 1) * b, L))
            kept_at[tau, bb, h, I] = ex["col_idx"][rp[r]:rp[r + 1]].tolist()
            o2_at[tau, bb, h, I] = _rows(o2, bb, h, rows)
            lse2_at[tau, bb, h, I] = _rows(lse2, bb, h, rows)
        if Lp > L:
            assert torch.all(o2[:, :, L:] == 0).item()
        del o2, lse2, ex
        pat.close()

    # ---- the oracle on the sampled query blocks, head by head
    dense_err = ErrAcc(f"{name} dense O")
    sparse_err = {tau: ErrAcc(f"{name} sparse O, tau={tau}") for tau in wl.taus}
    heads = sorted({(bb, h) for (bb, h, _) in samples})
    for (bb, h) in heads:
        qh, kh, vh = (t[bb, h].to("cpu", torch.float64).numpy() for t in (q, k, v))
        q2h, k2h, v2h = (t[bb, h].to("cpu", torch.float64).numpy() for t in (q2, k2, v2))
        for I in [I for (b2, h2, I) in samples if (b2, h2) == (bb, h)]:
            rows = np.arange(I * b, min((I + 1) * b, L))
            o_ref, lse_ref = O.attention_rows(qh[rows], kh[:L], vh[:L], scale)
            dense_err.add(_rows(o, bb, h, rows), o_ref)
            assert np.max(np.abs(_rows(lse, bb, h, rows) - lse_ref)) <= LSE_ATOL
            m_ref = O.block_mass_row(qh[None, None], kh[None, None], L, b, scale, 0, 0, I)
            assert np.max(np.abs(mass_cpu[bb, h, I] - m_ref)) <= MASS_ATOL
            for tau in wl.taus:
                cols = kept_at[tau, bb, h, I]
                assert m_ref[cols].sum() >= tau - RETAIN_SLACK, (tau, bb, h, I)
                keys = O.retained_keys(cols, b, L)
                o2_ref, lse2_ref = O.attention_rows(q2h[rows], k2h[keys], v2h[keys], scale)
                sparse_err[tau].add(o2_at[tau, bb, h, I], o2_ref)
                assert np.max(np.abs(lse2_at[tau, bb, h, I] - lse2_ref)) <= LSE_ATOL
    dense_err.check_mean()
    for tau in wl.taus:
        sparse_err[tau].check_mean()
    # padded rows
    if Lp > L:
        assert torch.all(o[:, :, L:] == 0).item()
        assert torch.all(torch.isneginf(lse[:, :, L:])).item()


@pytest.mark.parametrize("name", ["cogvideox", "wan2.1-1.3b"])
def test_full_size_fp32_inputs_take_the_tf32_path(losa, name):
    """The kind::tf32 kernels at full size: the layer's inputs drawn in fp32
    and left unrounded, the library rounding them to tf32 on entry; the
    oracle is handed the same tf32 values. Sampled query blocks of every
    head: O within 1e-2 + 2^-8 |O|, lse within 1e-4, masses within 1e-5,
    selection bit-exact on the GPU's masses, and the sparse step's O."""
    import dataclasses
    wl = dataclasses.replace(W.WORKLOADS[name], in_dtype="fp32")
    L, b, d, n = wl.seq_len, wl.block, wl.head_dim, wl.n_blocks
    scale = 1 / math.sqrt(d)
    tau = 0.99
    q, k, v = W.generate(wl, device="cuda", dtype=torch.float32)
    o, lse, mass = losa.dense_mass(q, k, v, L, b, out_dtype=torch.bfloat16)
    pat = losa.select(mass, b, tau)
    q2, k2, v2 = W.drift(wl, (q, k, v), step=1, device="cuda", dtype=torch.float32)
    o2, lse2 = losa.sparse_attn(q2, k2, v2, L, pat, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    losa.check_status()
    ex = pat.export("cpu")
    rp, mass_cpu = ex["row_ptr"].numpy(), mass.cpu().numpy()
    err_d, err_s = ErrAcc(f"{name} fp32 dense O"), ErrAcc(f"{name} fp32 sparse O")
    samples = W.sample_query_blocks(wl, 4, seed=5)
    for (bb, h) in sorted({(x, y) for (x, y, _) in samples}):
        qh, kh, vh = (W.round_tf32(t[bb, h].cpu()).double().numpy() for t in (q, k, v))
        q2h, k2h, v2h = (W.round_tf32(t[bb, h].cpu()).double().numpy() for t in (q2, k2, v2))
        for I in [I for (x, y, I) in samples if (x, y) == (bb, h)]:
            rows = np.arange(I * b, min((I + 1) * b, L))
            o_ref, lse_ref = O.attention_rows(qh[rows], kh[:L], vh[:L], scale)
            err_d.add(_rows(o, bb, h, rows), o_ref)
            assert np.max(np.abs(_rows(lse, bb, h, rows) - lse_ref)) <= LSE_ATOL
            m_ref = O.block_mass_row(qh[None, None], kh[None, None], L, b, scale, 0, 0, I)
            assert np.max(np.abs(mass_cpu[bb, h, I] - m_ref)) <= MASS_ATOL
            r = (bb * wl.heads + h) * n + I
            kept, C, S = O.select_row(O.to_fixed(mass_cpu[bb, h, I]).tolist(), tau)
            assert ex["col_idx"][rp[r]:rp[r + 1]].tolist() == kept
            keys = O.retained_keys(kept, b, L)
            o2_ref, lse2_ref = O.attention_rows(q2h[rows], k2h[keys], v2h[keys], scale)
            err_s.add(_rows(o2, bb, h, rows), o2_ref)
            assert np.max(np.abs(_rows(lse2, bb, h, rows) - lse2_ref)) <= LSE_ATOL
    err_d.check_mean()
    err_s.check_mean()
