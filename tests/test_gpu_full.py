"""The full-size workloads, in the launch configuration the benchmark times,
checked against the oracle on a seeded sample of query blocks (every head,
the last ragged block always included) and by properties that hold at any
size on every row."""
import math

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from test_gpu_parity import LSE_ATOL, MASS_ATOL, O_MAX

pytestmark = pytest.mark.gpu

PER_HEAD = 2  # sampled query blocks per head
SELECT_PER_HEAD = 16  # sampled rows per head for the selection-only check


@pytest.fixture(scope="module")
def losa():
    assert torch.cuda.is_available()
    import block_sparse_attention_losa_b200 as m
    return m


def _rows_np(t, b, h, rows):
    return t[b, h, rows].to("cpu", torch.float64).numpy()


@pytest.mark.parametrize("name", ["wan2.1-1.3b", "cogvideox", "hunyuanvideo", "wan2.1-14b"])
def test_full_size_workload(losa, name):
    wl = W.WORKLOADS[name]
    L, Lp, b, d = wl.seq_len, wl.seq_pad, wl.block, wl.head_dim
    scale = 1 / math.sqrt(d)
    tau = 0.99
    q, k, v = W.generate(wl, device="cuda")
    o, lse, mass = losa.dense_mass(q, k, v, L, b, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    losa.check_status()
    # Every row of the mass map sums to 1 (fp32 sum of n entries).
    rs = mass.double().sum(-1)
    assert torch.max(torch.abs(rs - 1)).item() < 1e-4
    assert torch.all(mass >= 0).item()

    pat = losa.select(mass, b, tau)
    ex = {kk: vv for kk, vv in pat.export("cpu").items()}
    # Every row keeps >= tau of its own fixed-point total, exactly.
    t_fx = O.tau_fixed(tau)
    ret, tot = ex["retained_fx"].tolist(), ex["total_fx"].tolist()
    assert all((1 << 48) * c >= t_fx * s for c, s in zip(ret, tot))
    rp = ex["row_ptr"].numpy()
    assert np.all(np.diff(rp) >= 1)

    q2, k2, v2 = W.drift(wl, (q, k, v), step=1, device="cuda")
    o2, lse2 = losa.sparse_attn(q2, k2, v2, L, pat, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    losa.check_status()

    mass_cpu = mass.cpu().numpy()
    # Selection alone on a wider sample (it is cheap): bit-exact rows.
    for (bb, h, I) in W.sample_query_blocks(wl, SELECT_PER_HEAD, seed=7):
        r = (bb * wl.heads + h) * wl.n_blocks + I
        kept, C, S = O.select_row(O.to_fixed(mass_cpu[bb, h, I]).tolist(), tau)
        assert ex["col_idx"][rp[r]:rp[r + 1]].tolist() == kept
        assert ret[r] == C and tot[r] == S
    for (bb, h, I) in W.sample_query_blocks(wl, PER_HEAD, seed=99):
        r = (bb * wl.heads + h) * wl.n_blocks + I
        # selection: bit-exact against the oracle on the GPU masses
        kept, C, S = O.select_row(O.to_fixed(mass_cpu[bb, h, I]).tolist(), tau)
        cols = ex["col_idx"][rp[r]:rp[r + 1]].tolist()
        assert cols == kept and ret[r] == C and tot[r] == S
        qh, kh, vh = (t[bb, h].to("cpu", torch.float64).numpy() for t in (q, k, v))
        rows = np.arange(I * b, min((I + 1) * b, L))
        # dense O / lse / mass of the sampled block
        o_ref, lse_ref = O.attention_rows(qh[rows], kh[:L], vh[:L], scale)
        og = o[bb, h, rows].to("cpu", torch.float64).numpy()
        assert np.max(np.abs(og - o_ref)) <= O_MAX + 2.0 ** -8 * np.max(np.abs(o_ref))
        lg = lse[bb, h, rows].to("cpu", torch.float64).numpy()
        assert np.max(np.abs(lg - lse_ref)) <= LSE_ATOL
        m_ref = O.block_mass_row(qh[None, None], kh[None, None], L, b,
                                 scale, 0, 0, I)
        assert np.max(np.abs(mass_cpu[bb, h, I] - m_ref)) <= MASS_ATOL
        # sparse O of the sampled block over the kept blocks
        q2h, k2h, v2h = (t[bb, h].to("cpu", torch.float64).numpy() for t in (q2, k2, v2))
        keys = O.retained_keys(cols, b, L)
        o2_ref, lse2_ref = O.attention_rows(q2h[rows], k2h[keys], v2h[keys], scale)
        o2g = o2[bb, h, rows].to("cpu", torch.float64).numpy()
        assert np.max(np.abs(o2g - o2_ref)) <= O_MAX + 2.0 ** -8 * np.max(np.abs(o2_ref))
        l2g = lse2[bb, h, rows].to("cpu", torch.float64).numpy()
        assert np.max(np.abs(l2g - lse2_ref)) <= LSE_ATOL
    # padded rows
    if Lp > L:
        assert torch.all(o[:, :, L:] == 0).item() and torch.all(o2[:, :, L:] == 0).item()
        assert torch.all(torch.isneginf(lse[:, :, L:])).item()
