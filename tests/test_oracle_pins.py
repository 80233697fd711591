"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each pin is a closed form, an invariant the pages fix, brute force over all
subsets, a hand-worked case (tests/golden/selection_cases.txt), or an
independent library routine (torch's scaled_dot_product_attention in fp64,
torch.logsumexp, exact rational arithmetic with fractions.Fraction).

The last group plants plausible mistakes in copies of oracle functions and
checks that some pin catches each one.
"""
import itertools
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "selection_cases.txt")
RNG = np.random.default_rng(20260812)


def _rand_qkv(B=1, H=2, Lp=96, d=16, L=83, scale_q=1.0, seed=0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, Lp, d)) * scale_q
    k = rng.standard_normal((B, H, Lp, d))
    v = rng.standard_normal((B, H, Lp, d))
    for x in (q, k, v):
        x[:, :, L:] = 0.0
    return q, k, v


def _sdpa(q, k, v, mask, scale):
    """torch SDPA in fp64; mask [.., n, m] True = attend."""
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    return torch.nn.functional.scaled_dot_product_attention(
        t(q), t(k), t(v), attn_mask=t(mask), scale=scale).numpy()


# ------------------------------------------------------------------ pin helpers
# Each takes the implementation under test so the mutation tests can reuse it.

def pin_dense_vs_sdpa(dense_fn):
    q, k, v = _rand_qkv(L=83)
    L, scale = 83, 1 / math.sqrt(16)
    o, lse = dense_fn(q, k, v, L, scale)
    mask = np.zeros((96, 96), dtype=bool)
    mask[:, :L] = True
    ref = _sdpa(q, k, v, mask, scale)
    np.testing.assert_allclose(o[:, :, :L], ref[:, :, :L], atol=1e-12, rtol=0)
    assert np.all(o[:, :, L:] == 0)
    s = torch.from_numpy(q[:, :, :L]) @ torch.from_numpy(k[:, :, :L]).transpose(-1, -2)
    ref_lse = torch.logsumexp(s * scale, dim=-1).numpy()
    np.testing.assert_allclose(lse[:, :, :L], ref_lse, atol=1e-12, rtol=0)
    assert np.all(np.isneginf(lse[:, :, L:]))


def pin_mass_vs_indicator_attention(mass_fn):
    """m[I, J] = mean over valid i in I of the attention output computed with
    V = indicator of key block J (column J of a one-hot block matrix)."""
    Lp, L, bsz = 96, 83, 16
    q, k, _ = _rand_qkv(L=L, Lp=Lp, scale_q=2.0)
    scale = 1 / math.sqrt(16)
    n = Lp // bsz
    ind = np.zeros((1, 2, Lp, n))
    for j in range(Lp):
        ind[:, :, j, j // bsz] = 1.0
    mask = np.zeros((Lp, Lp), dtype=bool)
    mask[:, :L] = True
    w = _sdpa(q, k, ind, mask, scale)  # [1, 2, Lp, n]
    mass = mass_fn(q, k, L, bsz, scale)
    for I in range(n):
        rows = [i for i in range(I * bsz, (I + 1) * bsz) if i < L]
        np.testing.assert_allclose(mass[:, :, I], w[:, :, rows].mean(axis=2), atol=1e-13, rtol=0)


def load_golden():
    cases = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        tau, xs, kept, why = [f.strip() for f in line.split("|")]
        cases.append((float(tau), [int(t) for t in xs.split()], [int(t) for t in kept.split()], why))
    return cases


def pin_selection_golden(select_row_fn):
    for tau, xs, kept, why in load_golden():
        got = select_row_fn(xs, tau)[0]
        assert list(got) == kept, f"{why}: tau={tau} x={xs} got {got} want {kept}"


def brute_force_min_set(x, tau):
    """Smallest cardinality of any subset reaching tau of the total, by
    enumerating every subset (exact rational arithmetic)."""
    S = sum(x)
    t = O.tau_fixed(tau)
    for r in range(1, len(x) + 1):
        for sub in itertools.combinations(range(len(x)), r):
            if (1 << 48) * sum(x[j] for j in sub) >= t * S:
                return r
    raise AssertionError("unreachable: the full set always reaches")


def pin_selection_brute_force(select_row_fn, rows=300, n=8):
    for it in range(rows):
        if it % 3 == 0:   # few distinct values: many ties
            x = RNG.integers(0, 4, size=n) * (1 << 45)
        else:
            x = np.rint(RNG.dirichlet(np.ones(n) * 0.5) * (1 << 48)).astype(np.int64)
        x = [int(v) for v in x]
        tau = float(RNG.choice([0.5, 0.8, 0.9, 0.95, 0.99, 0.999, 1.0]))
        kept, C, S = select_row_fn(x, tau)
        t = O.tau_fixed(tau)
        assert S == sum(x)
        assert C == sum(x[j] for j in kept)
        # (2) the retained mass reaches tau of the total
        assert (1 << 48) * C >= t * S
        # (5) no smaller set reaches it
        assert len(kept) == brute_force_min_set(x, tau)
        # the set is the top-k under (mass desc, index asc)
        order = sorted(range(n), key=lambda j: (-x[j], j))
        assert sorted(kept) == sorted(order[:len(kept)])
        # (3) minimality of the cut: dropping the smallest retained block fails
        if len(kept) > 1:
            smallest = min(x[j] for j in kept)
            assert (1 << 48) * (C - smallest) < t * S
        assert list(kept) == sorted(kept)


# ------------------------------------------------------------------ dense attention

def test_dense_matches_torch_sdpa_fp64():
    pin_dense_vs_sdpa(O.dense_attention)


def test_dense_zero_keys_closed_form():
    q, k, v = _rand_qkv(L=50, Lp=64)
    k[:] = 0.0
    o, lse = O.dense_attention(q, k, v, 50, 0.25)
    np.testing.assert_allclose(o[:, :, :50], np.broadcast_to(v[:, :, :50].mean(axis=2, keepdims=True), o[:, :, :50].shape), atol=1e-14)
    np.testing.assert_allclose(lse[:, :, :50], math.log(50), atol=1e-14)


def test_dense_single_key():
    q, k, v = _rand_qkv(L=1, Lp=8)
    o, lse = O.dense_attention(q, k, v, 1, 0.3)
    np.testing.assert_allclose(o[:, :, 0], v[:, :, 0], atol=1e-15)
    np.testing.assert_allclose(lse[:, :, 0], 0.3 * np.sum(q[:, :, 0] * k[:, :, 0], axis=-1), atol=1e-14)


# ------------------------------------------------------------------ block mass

def test_mass_matches_indicator_attention():
    pin_mass_vs_indicator_attention(O.block_mass)


def test_mass_rows_sum_to_one_and_nonnegative():
    wl = W.WORKLOADS["tiny"]
    q, k, v = W.generate(wl, dtype=torch.float64)
    m = O.block_mass(q.numpy(), k.numpy(), wl.seq_len, wl.block, 1 / math.sqrt(wl.head_dim))
    assert m.shape == (1, 2, 8, 8)
    assert np.all(m >= 0)
    np.testing.assert_allclose(m.sum(axis=-1), 1.0, atol=1e-12)


def test_mass_zero_keys_closed_form():
    q, k, _ = _rand_qkv(L=83, Lp=96)
    k[:] = 0.0
    m = O.block_mass(q, k, 83, 16, 0.25)
    want = np.array([min(16, max(0, 83 - 16 * J)) / 83 for J in range(6)])
    np.testing.assert_allclose(m, np.broadcast_to(want, m.shape), atol=1e-14)


def test_mass_one_hot_attention_is_identity():
    Lp, d = 32, 32
    k = np.zeros((1, 1, Lp, d))
    k[0, 0] = np.eye(d) * 12.0
    q = k.copy()
    m = O.block_mass(q, k, Lp, 8, 1.0)   # s_ii = 144, s_ij = 0: off-diagonal e^-144
    np.testing.assert_allclose(m[0, 0], np.eye(4), atol=1e-50)


# ------------------------------------------------------------------ selection

def test_to_fixed_is_exact_rounding():
    vals = np.concatenate([RNG.random(2000).astype(np.float32),
                           np.float32([0.0, 1.0, 0.5, 1 / 3, 2.0 ** -49, 3 * 2.0 ** -49,
                                       2.0 ** -48, 5 * 2.0 ** -50, 2.0 ** -60])])
    got = O.to_fixed(vals)
    for m, x in zip(vals.tolist(), got.tolist()):
        assert x == round(Fraction(m) * (1 << 48)), m  # Fraction rounds half to even


def test_to_fixed_rejects_nonfinite():
    with pytest.raises(ValueError):
        O.to_fixed(np.array([0.5, np.nan]))


def test_tau_fixed():
    assert O.tau_fixed(1.0) == 1 << 48
    assert O.tau_fixed(0.5) == 1 << 47
    assert O.tau_fixed(0.99) == round(Fraction(0.99) * (1 << 48))


def test_selection_golden_cases():
    pin_selection_golden(O.select_row)


def test_selection_brute_force_and_invariants():
    pin_selection_brute_force(O.select_row)


def test_selection_tau_one_keeps_positive_blocks():
    for _ in range(50):
        x = [int(v) for v in RNG.integers(0, 3, size=12)]
        if sum(x) == 0:
            continue
        kept, C, S = O.select_row(x, 1.0)
        assert kept == [j for j in range(12) if x[j] > 0] and C == S


def test_select_csr_layout():
    m = RNG.random((1, 2, 4, 5)).astype(np.float32)
    m /= m.sum(axis=-1, keepdims=True)
    s = O.select(m, 0.9)
    assert s["row_ptr"][0] == 0 and len(s["row_ptr"]) == 9
    for r in range(8):
        cols = s["col_idx"][s["row_ptr"][r]:s["row_ptr"][r + 1]]
        b, h, I = 0, r // 4, r % 4
        kept = O.select_row(O.to_fixed(m[b, h, I]).tolist(), 0.9)[0]
        assert cols.tolist() == kept


# ------------------------------------------------------------------ sparse attention

def _pattern_mask(row_ptr, col_idx, H, Lp, L, bsz):
    n = Lp // bsz
    mask = np.zeros((1, H, Lp, Lp), dtype=bool)
    for h in range(H):
        for I in range(n):
            r = h * n + I
            for J in col_idx[row_ptr[r]:row_ptr[r + 1]]:
                mask[0, h, I * bsz:(I + 1) * bsz, J * bsz:(J + 1) * bsz] = True
    mask[..., L:] = False
    mask[:, :, L:, :L] = True   # padded query rows: anything finite, not compared
    return mask


def test_sparse_matches_masked_sdpa():
    Lp, L, bsz, H = 96, 83, 16, 2
    q, k, v = _rand_qkv(L=L, Lp=Lp, scale_q=2.0)
    m = O.block_mass(q, k, L, bsz, 0.25)
    s = O.select(m, 0.9)
    assert len(s["col_idx"]) < H * 6 * 6  # the pattern is really sparse
    o, lse = O.sparse_attention(q, k, v, L, bsz, 0.25, s["row_ptr"], s["col_idx"])
    ref = _sdpa(q, k, v, _pattern_mask(s["row_ptr"], s["col_idx"], H, Lp, L, bsz), 0.25)
    np.testing.assert_allclose(o[:, :, :L], ref[:, :, :L], atol=1e-12)
    assert np.all(o[:, :, L:] == 0) and np.all(np.isneginf(lse[:, :, L:]))


def test_sparse_tau_one_equals_dense():
    wl = W.WORKLOADS["tiny"]
    q, k, v = (t.numpy() for t in W.generate(wl, dtype=torch.float64))
    L, scale = wl.seq_len, 1 / math.sqrt(wl.head_dim)
    m = O.block_mass(q, k, L, wl.block, scale)
    s = O.select(m, 1.0)
    assert np.all(s["x"] > 0)          # every block keeps mass: tau=1 keeps all
    o_s, lse_s = O.sparse_attention(q, k, v, L, wl.block, scale, s["row_ptr"], s["col_idx"])
    o_d, lse_d = O.dense_attention(q, k, v, L, scale)
    np.testing.assert_allclose(o_s, o_d, atol=1e-12)
    np.testing.assert_allclose(lse_s[:, :, :L], lse_d[:, :, :L], atol=1e-12)


def test_sparse_constant_values_closed_form():
    q, k, v = _rand_qkv(L=70, Lp=80)
    v[:, :, :70] = np.array([1.5, -2.0] * 8)
    m = O.block_mass(q, k, 70, 16, 0.25)
    s = O.select(m, 0.8)
    o, _ = O.sparse_attention(q, k, v, 70, 16, 0.25, s["row_ptr"], s["col_idx"])
    np.testing.assert_allclose(o[:, :, :70], np.broadcast_to(v[:, :, :1], o[:, :, :70].shape), atol=1e-13)


def test_sparse_zero_keys_is_mean_of_retained_values():
    q, k, v = _rand_qkv(L=70, Lp=80)
    k[:] = 0.0
    row_ptr = np.array([0, 1, 3, 4, 6, 7] * 1 + [8, 9, 10, 11, 12], dtype=np.int64)
    col_idx = np.array([0, 1, 4, 2, 0, 4, 3, 1, 2, 0, 4, 3], dtype=np.int64)
    o, _ = O.sparse_attention(q, k, v, 70, 16, 0.25, row_ptr, col_idx)
    for h in range(2):
        for I in range(5):
            r = h * 5 + I
            keys = [j for J in col_idx[row_ptr[r]:row_ptr[r + 1]] for j in range(16 * J, 16 * J + 16) if j < 70]
            want = v[0, h, keys].mean(axis=0)
            for i in range(16 * I, min(16 * I + 16, 70)):
                np.testing.assert_allclose(o[0, h, i], want, atol=1e-14)


# ------------------------------------------------------------------ workload calibration

def test_tiny_workload_prunes_in_band():
    """The small workload keeps 50-70 % of the blocks at tau = 0.99 (30-50 %
    pruned, the band the workload description states)."""
    wl = W.WORKLOADS["tiny"]
    q, k, _ = W.generate(wl, dtype=torch.float64)
    m = O.block_mass(q.numpy(), k.numpy(), wl.seq_len, wl.block, 1 / math.sqrt(wl.head_dim))
    s = O.select(m.astype(np.float32), 0.99)
    kept = len(s["col_idx"]) / (wl.heads * wl.n_blocks ** 2)
    assert 0.5 <= kept <= 0.7, kept


def test_generator_is_seeded_and_bf16_exact():
    """bf16 workloads hand out bf16-exact values (any requested dtype); the
    fp32 small workload hands out fp32 values that are not all bf16-exact."""
    wl = W.custom("b16", 2, 64, (2, 8, 8), 32, amplitude=1.1, seed=4)
    for dtype in (torch.float32, torch.float64):
        for x in W.generate(wl, dtype=dtype):
            assert x.dtype == dtype
            assert torch.equal(x, x.to(torch.bfloat16).to(dtype))
    tiny = W.WORKLOADS["tiny"]
    a = W.generate(tiny)
    b = W.generate(tiny)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
        assert x.dtype == torch.float32
        assert not torch.equal(x, x.to(torch.bfloat16).to(torch.float32))
        assert torch.all(x[:, :, tiny.seq_len:] == 0)
    c = W.drift(tiny, a, step=1)
    assert not torch.equal(c[0], a[0])
    assert float((c[0] - a[0]).abs().max()) < 0.5


def _tf32_exact(x):
    """Round-to-nearest-even to 11 significant bits, in exact rationals."""
    X = Fraction(float(x))
    if X == 0:
        return 0.0
    e = math.floor(math.log2(abs(X)))
    while Fraction(2) ** e > abs(X):
        e -= 1
    while Fraction(2) ** (e + 1) <= abs(X):
        e += 1
    ulp = Fraction(2) ** (max(e, -126) - 10)
    return float(round(X / ulp) * ulp)  # round() on a Fraction: ties to even


def test_round_tf32_matches_exact_rational_rounding():
    """workloads.round_tf32 (the tf32 values the oracle is handed for fp32
    inputs) against round-half-even in exact rationals: random values over
    many binades, and every tie and near-tie pattern of the dropped bits."""
    g = torch.Generator().manual_seed(11)
    x = torch.randn(4000, generator=g) * torch.pow(2.0, torch.randint(-30, 30, (4000,),
                                                                      generator=g).float())
    base = torch.tensor([1.0, 1.5, -3.25, 1e-3, 7e5], dtype=torch.float32)
    bits = base.view(torch.int32)
    pats = []
    for low in (0x0000, 0x0FFF, 0x1000, 0x1001, 0x1FFF, 0x0001, 0x17FF, 0x0800):
        for odd in (0, 1):
            pats.append(((bits & ~0x3FFF) | (odd << 13) | low).view(torch.float32))
    x = torch.cat([x.float()] + pats)
    r = W.round_tf32(x)
    want = torch.tensor([_tf32_exact(v) for v in x.tolist()], dtype=torch.float64)
    assert torch.equal(r.double(), want)
    assert torch.all((r.view(torch.int32) & 0x1FFF) == 0)
    # ties: half an ulp rounds to the even neighbour
    one = torch.tensor([1 + 2 ** -11, 1 + 3 * 2 ** -11, -(1 + 2 ** -11)], dtype=torch.float32)
    assert W.round_tf32(one).tolist() == [1.0, 1 + 2 ** -9, -1.0]
    assert torch.equal(W.round_tf32(torch.tensor([float("inf"), 0.0])),
                       torch.tensor([float("inf"), 0.0]))


# ------------------------------------------------------------------ planted mistakes

def _mutant_dense_no_scale(q, k, v, L, scale):
    return O.dense_attention(q, k, v, L, 1.0)


def _mutant_dense_no_key_mask(q, k, v, L, scale):
    Lp = q.shape[2]
    return O.dense_attention(q, k, v, Lp, scale)


def _mutant_mass_unnormalised(q, k, L, block, scale):
    m = O.block_mass(q, k, L, block, scale)
    return m * block


def _mutant_mass_transposed(q, k, L, block, scale):
    return np.swapaxes(O.block_mass(q, k, L, block, scale), -1, -2)


def _mutant_select_strict(x, tau):
    x = [int(v) for v in x]
    t, S = O.tau_fixed(tau), sum(x)
    order = sorted(range(len(x)), key=lambda J: (-x[J], J))
    C, kept = 0, []
    for J in order:
        C += x[J]
        kept.append(J)
        if (1 << 48) * C > t * S:     # mistake: strict comparison
            break
    return sorted(kept), C, S


def _mutant_select_ties_high_index(x, tau):
    x = [int(v) for v in x]
    t, S = O.tau_fixed(tau), sum(x)
    order = sorted(range(len(x)), key=lambda J: (-x[J], -J))  # mistake
    C, kept = 0, []
    for J in order:
        C += x[J]
        kept.append(J)
        if (1 << 48) * C >= t * S:
            break
    return sorted(kept), C, S


def _mutant_select_ascending(x, tau):
    x = [int(v) for v in x]
    t, S = O.tau_fixed(tau), sum(x)
    order = sorted(range(len(x)), key=lambda J: (x[J], J))  # mistake: smallest first
    C, kept = 0, []
    for J in order:
        C += x[J]
        kept.append(J)
        if (1 << 48) * C >= t * S:
            break
    return sorted(kept), C, S


@pytest.mark.parametrize("pin,mutant", [
    (pin_dense_vs_sdpa, _mutant_dense_no_scale),
    (pin_dense_vs_sdpa, _mutant_dense_no_key_mask),
    (pin_mass_vs_indicator_attention, _mutant_mass_unnormalised),
    (pin_mass_vs_indicator_attention, _mutant_mass_transposed),
    (pin_selection_golden, _mutant_select_strict),
    (pin_selection_golden, _mutant_select_ties_high_index),
    (pin_selection_brute_force, _mutant_select_ascending),
])
def test_pins_catch_planted_mistakes(pin, mutant):
    with pytest.raises(AssertionError):
        pin(mutant)
