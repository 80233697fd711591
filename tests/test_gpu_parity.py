"""GPU path (through the C ABI) against the CPU oracle, element by element.

Inputs: the oracle is handed the values the library computes on: bf16
inputs as they are, and fp32 inputs rounded to tf32 (round to nearest even,
workloads.round_tf32), since the library rounds fp32 inputs to tf32 on entry
and runs kind::tf32 MMAs on them.

Tolerances, per output:
  * block mass: |delta| <= 1e-5 absolute (fp32 accumulation of exact
    bf16 x bf16 or tf32 x tf32 products; the row sums to 1, so fp32 rounding
    of the sum and of exp2 stays near 1e-7 per term).
  * selection: bit-exact (row_ptr, col_idx, retained_fx, total_fx) against
    the oracle's selection run on the GPU's own fp32 masses; with the
    oracle's fp64 masses, the kept set still holds >= tau - 1e-5 of the mass.
  * O (fp32 output): max |delta| <= 1e-2 and mean |delta| <= 1e-3 against
    fp64 on the same rounded inputs. P is rounded to bf16 (tf32 on the fp32
    path) before the P.V product (relative 2^-9, resp. 2^-11, per weight),
    which bounds the error near 2^-9 * max|v| ~ 0.008 in the worst case and
    ~1e-4 on average.
  * O (bf16 output): additionally the output's own rounding, half an ulp:
    |delta| <= 1e-2 + 2^-8 |O|.
  * lse: |delta| <= 1e-4 (fp32 scores of exact products; the sum of exp
    uses the unrounded fp32 values).
"""
import math
import zlib

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W

pytestmark = pytest.mark.gpu

MASS_ATOL = 1e-5
O_MAX, O_MEAN = 1e-2, 1e-3
LSE_ATOL = 1e-4


@pytest.fixture(scope="module")
def losa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import block_sparse_attention_losa_b200 as m
    return m


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def assert_o_close(o_gpu, o_ref, L, bf16_out=False, what="O"):
    o = f64(o_gpu)
    d = np.abs(o[:, :, :L] - o_ref[:, :, :L])
    if bf16_out:
        bound = O_MAX + 2.0 ** -8 * np.abs(o_ref[:, :, :L])
        assert np.all(d <= bound), f"{what}: max excess {np.max(d - bound)}"
    else:
        assert d.max() <= O_MAX, f"{what}: max |d| {d.max()}"
    assert d.mean() <= O_MEAN, f"{what}: mean |d| {d.mean()}"
    assert np.all(o[:, :, L:] == 0), f"{what}: padded rows not zero"


def assert_lse_close(lse_gpu, lse_ref, L):
    l = f64(lse_gpu)
    assert np.max(np.abs(l[:, :, :L] - lse_ref[:, :, :L])) <= LSE_ATOL
    assert np.all(np.isneginf(l[:, :, L:]))


def check_tiles(ex, pat, n):
    """The sparse kernel's work list is the per-tile union of the rows'
    kept sets, with correct masks, ordered head by head and, within a head,
    by entry count (largest first)."""
    row_ptr = ex["row_ptr"].numpy()
    col_idx = ex["col_idx"].numpy()
    tile_ptr = ex["tile_ptr"].numpy()
    tile_entry = ex["tile_entry"].numpy()
    order = ex["tile_order"].numpy()
    qpt = 128 // pat.block
    n_qt = (n * pat.block + 127) // 128
    assert sorted(order.tolist()) == list(range(pat.n_tiles))
    counts = np.diff(tile_ptr)
    heads = order // n_qt
    assert np.all(np.diff(heads) >= 0)
    same = np.diff(heads) == 0
    assert np.all(np.diff(counts[order])[same] <= 0)
    for t in range(pat.n_tiles):
        bh, qt = divmod(t, n_qt)
        want = {}
        for q in range(qpt):
            I = qt * qpt + q
            if I >= n:
                break
            r = bh * n + I
            for J in col_idx[row_ptr[r]:row_ptr[r + 1]]:
                want[int(J)] = want.get(int(J), 0) | (1 << q)
        got = tile_entry[tile_ptr[t]:tile_ptr[t + 1]]
        assert [int(e) & 0xFFFF for e in got] == sorted(want)
        assert [int(e) >> 16 for e in got] == [want[J] for J in sorted(want)]


def check_selection(pat, mass_gpu, tau, check_tile_lists=True):
    mass_np = mass_gpu.cpu().numpy()
    ref = O.select(mass_np, tau)
    ex = {k: v.cpu() for k, v in pat.export("cpu").items()}
    assert pat.nnz == len(ref["col_idx"])
    np.testing.assert_array_equal(ex["row_ptr"].numpy(), ref["row_ptr"])
    np.testing.assert_array_equal(ex["col_idx"].numpy(), ref["col_idx"])
    assert ex["retained_fx"].tolist() == ref["retained_fx"]
    assert ex["total_fx"].tolist() == ref["total_fx"]
    if check_tile_lists:
        check_tiles(ex, pat, mass_np.shape[-1])
    return ref, ex


class Guarded:
    """An output buffer followed by a canary tail of 4,096 elements holding
    a fixed value: a kernel that writes past the buffer's end changes it."""

    def __init__(self, shape, dtype):
        n = math.prod(shape)
        self.buf = torch.full((n + 4096,), 12345.5, dtype=dtype, device="cuda")
        self.out = self.buf[:n].view(shape)
        self.tail0 = self.buf[n:].clone()

    def check(self, what):
        assert torch.equal(self.buf[self.out.numel():], self.tail0), f"{what} wrote past its end"


def computed_on(t, in_fp32):
    """The values the library computes on for inputs t (fp32 on the host)."""
    return W.round_tf32(t) if in_fp32 else t.to(torch.bfloat16).to(torch.float32)


def run_small(losa, wl, tau=0.99, out_dtype=torch.float32, in_fp32=None):
    q, k, v = W.generate(wl, dtype=torch.float32)
    if in_fp32 is None:
        in_fp32 = wl.in_dtype == "fp32"
    dt = torch.float32 if in_fp32 else torch.bfloat16
    qd, kd, vd = (t.to("cuda", dt) for t in (q, k, v))
    L, b, scale = wl.seq_len, wl.block, 1 / math.sqrt(wl.head_dim)
    B, H, Lp, d = qd.shape
    g_o, g_lse, g_mass = (Guarded((B, H, Lp, d), out_dtype), Guarded((B, H, Lp), torch.float32),
                          Guarded((B, H, wl.n_blocks, wl.n_blocks), torch.float32))
    o, lse, mass = losa.dense_mass(qd, kd, vd, L, b, out_dtype=out_dtype, o=g_o.out,
                                   lse=g_lse.out, mass=g_mass.out)
    torch.cuda.synchronize()
    losa.check_status()
    for g, what in ((g_o, "dense O"), (g_lse, "dense lse"), (g_mass, "mass")):
        g.check(what)
    q64, k64, v64 = (computed_on(t, in_fp32).double().numpy() for t in (q, k, v))
    o_ref, lse_ref = O.dense_attention(q64, k64, v64, L, scale)
    mass_ref = O.block_mass(q64, k64, L, b, scale)
    assert_o_close(o, o_ref, L, bf16_out=out_dtype == torch.bfloat16, what="dense O")
    assert_lse_close(lse, lse_ref, L)
    m = f64(mass)
    assert np.max(np.abs(m - mass_ref)) <= MASS_ATOL, np.max(np.abs(m - mass_ref))

    pat = losa.select(mass, b, tau)
    ref, ex = check_selection(pat, mass, tau)
    # Against the oracle's own fp64 masses the kept set still reaches tau.
    for r in range(pat.rows):
        bb, rest = divmod(r, wl.heads * wl.n_blocks)
        h, I = divmod(rest, wl.n_blocks)
        cols = ex["col_idx"][ex["row_ptr"][r]:ex["row_ptr"][r + 1]].numpy()
        assert mass_ref[bb, h, I, cols].sum() >= tau - 1e-5

    q2, k2, v2 = W.drift(wl, (q, k, v), step=1, dtype=torch.float32)
    q2d, k2d, v2d = (t.to("cuda", dt) for t in (q2, k2, v2))
    g_o2, g_lse2 = Guarded((B, H, Lp, d), out_dtype), Guarded((B, H, Lp), torch.float32)
    o2, lse2 = losa.sparse_attn(q2d, k2d, v2d, L, pat, out_dtype=out_dtype, o=g_o2.out,
                                lse=g_lse2.out)
    torch.cuda.synchronize()
    losa.check_status()
    g_o2.check("sparse O")
    g_lse2.check("sparse lse")
    o2_ref, lse2_ref = O.sparse_attention(*(computed_on(t, in_fp32).double().numpy()
                                            for t in (q2, k2, v2)), L, b, scale,
                                          ref["row_ptr"], ref["col_idx"])
    assert_o_close(o2, o2_ref, L, bf16_out=out_dtype == torch.bfloat16, what="sparse O")
    assert_lse_close(lse2, lse2_ref, L)
    return pat


def test_tiny_workload(losa):
    pat = run_small(losa, W.WORKLOADS["tiny"])
    assert 0.3 <= 1 - pat.density() <= 0.5


SMALL = [
    # name, heads, d, grid, block, text, batch — ragged tails and partial tiles
    ("d128_b64_partial_tile", 3, 128, (3, 10, 13), 64, 0, 1),
    ("d64_b128_text", 2, 64, (2, 12, 20), 128, 30, 1),
    ("d128_b32_partial_tile", 2, 128, (3, 7, 9), 32, 0, 1),
    ("d64_b64_text", 2, 64, (4, 9, 11), 64, 20, 1),
    ("d128_b64_batch2", 2, 128, (2, 8, 16), 64, 0, 2),
    ("d128_b128_10_blocks", 2, 128, (4, 16, 20), 128, 0, 1),
    ("d64_b32_exact", 1, 64, (2, 8, 8), 32, 0, 1),
]


@pytest.mark.parametrize("name,heads,d,grid,block,text,batch", SMALL, ids=[s[0] for s in SMALL])
def test_small_shapes(losa, name, heads, d, grid, block, text, batch):
    wl = W.custom(name, heads, d, grid, block, text_tokens=text, batch=batch, amplitude=1.2,
                  seed=zlib.crc32(name.encode()) % 1000)
    run_small(losa, wl)


@pytest.mark.parametrize("tau", [0.5, 0.95, 0.999])
def test_tau_values(losa, tau):
    wl = W.custom("tau", 2, 128, (3, 10, 13), 64, amplitude=1.2, seed=5)
    run_small(losa, wl, tau=tau)


def test_bf16_io(losa):
    wl = W.custom("bf16io", 2, 128, (3, 10, 13), 64, amplitude=1.2, seed=9)
    run_small(losa, wl, out_dtype=torch.bfloat16, in_fp32=False)


TF32 = [
    # name, heads, d, grid, block, text: the kind::tf32 kernels (d 128 runs
    # 64-key stages, so a 128-token block spans two of them)
    ("tf32_d64_b64", 2, 64, (3, 10, 13), 64, 0),
    ("tf32_d64_b128_text", 2, 64, (2, 12, 20), 128, 30),
    ("tf32_d64_b32", 2, 64, (3, 7, 9), 32, 0),
    ("tf32_d128_b64", 2, 128, (3, 10, 13), 64, 0),
    ("tf32_d128_b128_text", 2, 128, (2, 12, 20), 128, 30),
    ("tf32_d128_b32", 2, 128, (3, 7, 9), 32, 5),
]


@pytest.mark.parametrize("name,heads,d,grid,block,text", TF32, ids=[s[0] for s in TF32])
def test_fp32_inputs_take_the_tf32_path(losa, name, heads, d, grid, block, text):
    wl = W.custom(name, heads, d, grid, block, text_tokens=text, amplitude=1.2,
                  seed=zlib.crc32(name.encode()) % 1000, in_dtype="fp32")
    run_small(losa, wl, in_fp32=True)
    run_small(losa, wl, in_fp32=True, out_dtype=torch.bfloat16, tau=0.95)


def test_tf32_path_is_more_accurate_than_bf16_on_fp32_inputs(losa):
    """On unrounded fp32 inputs, against fp64 on those same inputs: the fp32
    (tf32) path's errors in the masses and in O are several times smaller
    than those of the same inputs handed over as bf16."""
    wl = W.custom("acc", 2, 128, (3, 10, 13), 64, amplitude=1.2, seed=13, in_dtype="fp32")
    q, k, v = W.generate(wl, dtype=torch.float32)
    L, b, scale = wl.seq_len, wl.block, 1 / math.sqrt(wl.head_dim)
    q64, k64, v64 = (t.double().numpy() for t in (q, k, v))
    o_ref, _ = O.dense_attention(q64, k64, v64, L, scale)
    m_ref = O.block_mass(q64, k64, L, b, scale)
    err = {}
    for dt in (torch.float32, torch.bfloat16):
        o, _, mass = losa.dense_mass(*(t.to("cuda", dt) for t in (q, k, v)), L, b)
        torch.cuda.synchronize()
        err[dt] = (np.abs(f64(mass) - m_ref).max(), np.abs(f64(o)[:, :, :L] - o_ref[:, :, :L]).max())
    assert err[torch.float32][0] * 4 < err[torch.bfloat16][0], err
    assert err[torch.float32][1] * 4 < err[torch.bfloat16][1], err


def test_tau_one_keeps_every_positive_block_and_equals_dense(losa):
    wl = W.custom("tau1", 2, 64, (2, 8, 16), 32, amplitude=0.8, seed=3)
    q, k, v = (t.cuda() for t in W.generate(wl, dtype=torch.bfloat16))
    L, b = wl.seq_len, wl.block
    o, lse, mass = losa.dense_mass(q, k, v, L, b)
    pat = losa.select(mass, b, 1.0)
    x = O.to_fixed(mass.cpu().numpy())
    assert pat.nnz == int((x > 0).sum())
    o2, lse2 = losa.sparse_attn(q, k, v, L, pat)
    torch.cuda.synchronize()
    # These inputs give every block a positive mass (the smallest is ~1e-6,
    # far above 2^-49), so tau = 1 keeps every block and the sparse kernel
    # must compute the dense result.
    assert pat.nnz == pat.rows * pat.n_blocks
    q64, k64, v64 = (t.double().cpu().numpy() for t in (q, k, v))
    o_ref, lse_ref = O.dense_attention(q64, k64, v64, L, 1 / math.sqrt(wl.head_dim))
    assert_o_close(o2, o_ref, L, what="tau=1 sparse O")
    assert_lse_close(lse2, lse_ref, L)


def test_one_hot_mass_rows_keep_one_block(losa):
    """A mass map with one block per row at mass 1 keeps exactly that block."""
    n = 40
    mass = torch.zeros(1, 3, n, n)
    rng = np.random.default_rng(0)
    hot = rng.integers(0, n, size=(3, n))
    for h in range(3):
        for I in range(n):
            mass[0, h, I, hot[h, I]] = 1.0
    pat = losa.select(mass.cuda(), 64, 0.99)
    ex = pat.export("cpu")
    assert pat.nnz == 3 * n
    assert ex["col_idx"].numpy().tolist() == hot.reshape(-1).tolist()


def test_equal_masses_break_ties_by_lower_index(losa):
    n = 16
    mass = torch.full((1, 1, n, n), 1.0 / n)
    pat = losa.select(mass.cuda(), 32, 0.5)
    ex = pat.export("cpu")
    assert ex["col_idx"].numpy().tolist() == list(range(8)) * n


def test_random_mass_maps_select_bit_exact(losa):
    """Selection alone on random and adversarial mass maps (many ties,
    zeros, tiny values), against the oracle."""
    rng = np.random.default_rng(7)
    for trial in range(6):
        n = int(rng.choice([8, 33, 129, 500, 2047]))
        H = 2 if n <= 500 else 1
        if trial % 3 == 0:
            m = rng.integers(0, 5, size=(1, H, n, n)).astype(np.float32)
        elif trial % 3 == 1:
            m = (rng.random((1, H, n, n)) ** 8).astype(np.float32)
        else:
            m = rng.dirichlet(np.ones(n) * 0.1, size=(1, H, n)).astype(np.float32)
        m /= np.maximum(m.sum(axis=-1, keepdims=True), 1e-30)
        m = m.astype(np.float32)
        for tau in (0.3, 0.99, 1.0):
            t = torch.from_numpy(m).cuda()
            pat = losa.select(t, 64, tau)
            check_selection(pat, t, tau, check_tile_lists=(n <= 129))


def test_bad_mass_is_reported(losa):
    mass = torch.full((1, 1, 8, 8), 0.125)
    mass[0, 0, 3, 5] = float("nan")
    with pytest.raises(losa.LosaError) as e:
        losa.select(mass.cuda(), 32, 0.99)
    assert e.value.status == -5
    mass[0, 0, 3, 5] = -0.1
    with pytest.raises(losa.LosaError):
        losa.select(mass.cuda(), 32, 0.99)
    # the status word was cleared: a good map goes through
    mass[0, 0, 3, 5] = 0.125
    losa.select(mass.cuda(), 32, 0.99)


def test_shape_mismatch_is_rejected(losa):
    wl = W.custom("mm", 1, 64, (2, 8, 8), 32, amplitude=1.0, seed=1)
    q, k, v = (t.cuda() for t in W.generate(wl, dtype=torch.bfloat16))
    _, _, mass = losa.dense_mass(q, k, v, wl.seq_len, wl.block)
    pat = losa.select(mass, wl.block, 0.99)
    q2 = torch.zeros(1, 1, 256 + 32, 64, device="cuda", dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        losa.sparse_attn(q2, q2, q2, wl.seq_len, pat)


def test_fma_pipe_exp2_error_bound(losa):
    """The FMA-pipe exp2 inside the softmax against float64 exp2: relative
    error below 4e-7 on [-125, 127] (fit: 3.1e-7), tiny below -125."""
    g = torch.Generator().manual_seed(3)
    x = torch.cat([torch.rand(1 << 20, generator=g) * 133.0 - 125.0,
                   torch.linspace(-125.0, 8.0, 100001),
                   torch.tensor([0.0, -0.5, 0.5, 1.0, -1.0, 7.999, -124.5, 127.0])])
    y = losa.exp2_eval(x.cuda()).cpu().double()
    ref = torch.exp2(x.double())
    rel = ((y - ref) / ref).abs()
    assert rel.max().item() < 4e-7, rel.max().item()
    low = losa.exp2_eval(torch.tensor([-126.0, -300.0, float("-inf")]).cuda()).cpu()
    assert torch.all(low >= 0).item() and torch.all(low < 3e-38).item()


def test_bounded_wait_reports_timeout_and_context_survives(losa):
    """A wait nothing completes gives up after its limit (here ~1 ms of SM
    cycles), the status word reports it once, and the device keeps working."""
    lib = losa.lib()
    losa.check_status()                      # start clean
    assert lib.losa_selftest_wait(2_000_000, None) == 0
    with pytest.raises(losa.LosaError) as e:
        losa.check_status(torch.cuda.default_stream())
    assert e.value.status == -4              # LOSA_ERR_TIMEOUT
    losa.check_status()                      # cleared
    assert lib.losa_selftest_wait(0, None) == -1
    # the context is still usable: a normal call after the timeout
    wl = W.custom("after_timeout", 1, 64, (2, 8, 8), 32, amplitude=1.0, seed=2)
    q, k, v = (t.cuda() for t in W.generate(wl, dtype=torch.bfloat16))
    o, lse, mass = losa.dense_mass(q, k, v, wl.seq_len, wl.block)
    torch.cuda.synchronize()
    losa.check_status()
    assert torch.allclose(mass.sum(-1), torch.ones_like(mass.sum(-1)), atol=1e-4)


def test_attention_kernels_abort_on_a_short_wait_limit(losa):
    """The attention kernels' own failure path: with a wait limit of one SM
    cycle, the first wait of the construction and of the sparse kernel that
    is not satisfied at once gives up; the call reports LOSA_ERR_TIMEOUT
    through the status word, every warp leaves, the copies and MMAs in
    flight land, tensor memory is freed, and the next normal calls give
    bit for bit what they gave before."""
    lib = losa.lib()
    wl = W.custom("abort", 4, 128, (2, 16, 64), 64, amplitude=1.2, seed=17)
    q, k, v = (t.cuda() for t in W.generate(wl, dtype=torch.bfloat16))
    L, b = wl.seq_len, wl.block
    losa.check_status()
    o_ref, lse_ref, mass_ref = losa.dense_mass(q, k, v, L, b)
    pat = losa.select(mass_ref, b, 0.95)
    o2_ref, lse2_ref = losa.sparse_attn(q, k, v, L, pat)
    torch.cuda.synchronize()
    losa.check_status()
    assert lib.losa_set_wait_limit(-1) == -1
    try:
        losa.set_wait_limit(1)
        losa.dense_mass(q, k, v, L, b)
        with pytest.raises(losa.LosaError) as e:
            losa.check_status()
        assert e.value.status == -4          # LOSA_ERR_TIMEOUT
        losa.sparse_attn(q, k, v, L, pat)
        with pytest.raises(losa.LosaError) as e:
            losa.check_status()
        assert e.value.status == -4
    finally:
        losa.set_wait_limit(0)               # back to the default
    o, lse, mass = losa.dense_mass(q, k, v, L, b)
    o2, lse2 = losa.sparse_attn(q, k, v, L, pat)
    torch.cuda.synchronize()
    losa.check_status()
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref) and torch.equal(mass, mass_ref)
    assert torch.equal(o2, o2_ref) and torch.equal(lse2, lse2_ref)
