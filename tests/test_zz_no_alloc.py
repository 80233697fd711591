"""losa_select_noalloc, the selection for callers that cannot allocate device
memory (engines that reserve all memory at start-up, code inside another
framework's allocator, loops that cannot take cudaMalloc's synchronisation).

It is called through the C ABI with caller-owned buffers and must give
exactly what losa_select gives (selection is integer work, so the two are
compared bit for bit), on two calls in a row: the second call reuses the
library's fixed scratch array after the first one left its contents there.
This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def losa():
    assert torch.cuda.is_available()
    import block_sparse_attention_losa_b200 as m
    return m


def _noalloc(losa, mass, tau, capacity=None):
    B, H, n, _ = mass.shape
    R = B * H * n
    cap = R * n if capacity is None else capacity
    dev = mass.device
    row_ptr = torch.full((R + 1,), -7, dtype=torch.int32, device=dev)
    col_idx = torch.full((max(cap, 1),), -7, dtype=torch.int32, device=dev)
    ret = torch.full((R,), -7, dtype=torch.int64, device=dev)
    tot = torch.full((R,), -7, dtype=torch.int64, device=dev)
    st = losa.lib().losa_select_noalloc(
        mass.data_ptr(), B, H, n, ctypes.c_double(tau), row_ptr.data_ptr(), col_idx.data_ptr(),
        ctypes.c_int64(cap), ret.data_ptr(), tot.data_ptr(),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, row_ptr, col_idx, ret, tot


def _masses(losa, seed, amplitude):
    wl = W.custom("noalloc", 3, 128, (3, 10, 13), 64, amplitude=amplitude, seed=seed)
    q, k, v = (t.cuda() for t in W.generate(wl, dtype=torch.bfloat16))
    _, _, mass = losa.dense_mass(q, k, v, wl.seq_len, wl.block)
    return mass, wl.block


def test_noalloc_select_matches_select_on_two_calls(losa):
    for seed, amplitude, tau in ((21, 1.2, 0.99), (22, 0.9, 0.95)):
        mass, block = _masses(losa, seed, amplitude)
        pat = losa.select(mass, block, tau)
        ref = pat.export("cpu")
        st, row_ptr, col_idx, ret, tot = _noalloc(losa, mass, tau)
        assert st == 0, losa.lib().losa_strerror(st)
        torch.cuda.synchronize()
        losa.check_status()
        nnz = int(row_ptr[-1].item())
        assert nnz == pat.nnz
        assert torch.equal(row_ptr.cpu(), ref["row_ptr"])
        assert torch.equal(col_idx[:nnz].cpu(), ref["col_idx"])
        assert torch.equal(ret.cpu(), ref["retained_fx"])
        assert torch.equal(tot.cpu(), ref["total_fx"])
        pat.close()


def _random_mass(H, n, seed):
    """Mass rows of n key blocks with ties (every 5th block shares one
    value), exact zeros and a heavy tail, each row summing to ~1 in fp32."""
    g = torch.Generator().manual_seed(seed)
    m = torch.rand(1, H, n, n, generator=g, dtype=torch.float64) ** 8
    m[..., ::5] = m[..., 1:2]
    m[..., 3::11] = 0.0
    m = m / m.sum(-1, keepdim=True)
    return m.to(torch.float32).cuda().contiguous()


def _same_as_select(losa, mass, tau):
    pat = losa.select(mass, 64, tau)
    ref = pat.export("cpu")
    st, row_ptr, col_idx, ret, tot = _noalloc(losa, mass, tau)
    assert st == 0, losa.lib().losa_strerror(st)
    torch.cuda.synchronize()
    losa.check_status()
    nnz = int(row_ptr[-1].item())
    assert nnz == pat.nnz
    assert torch.equal(row_ptr.cpu(), ref["row_ptr"])
    assert torch.equal(col_idx[:nnz].cpu(), ref["col_idx"])
    assert torch.equal(ret.cpu(), ref["retained_fx"])
    assert torch.equal(tot.cpu(), ref["total_fx"])
    pat.close()
    return nnz


def test_noalloc_long_rows_take_the_bucketed_cut(losa):
    """Rows of more than 512 key blocks go through the bucketed cut kernel;
    two calls in a row, each bit-exact against losa_select."""
    _same_as_select(losa, _random_mass(2, 1500, seed=3), 0.99)
    _same_as_select(losa, _random_mass(1, 2047, seed=4), 0.95)


def test_noalloc_truncates_at_col_capacity(losa):
    """With col_capacity below the number of kept blocks, the row offsets
    are still complete, the first col_capacity entries are the full list's,
    and nothing past col_capacity is written."""
    mass = _random_mass(3, 600, seed=5)
    full = _same_as_select(losa, mass, 0.99)
    cap = full // 2
    B, H, n, _ = mass.shape
    R = B * H * n
    row_ptr = torch.full((R + 1,), -7, dtype=torch.int32, device="cuda")
    col_idx = torch.full((cap + 4096,), -7, dtype=torch.int32, device="cuda")
    ret = torch.empty(R, dtype=torch.int64, device="cuda")
    tot = torch.empty(R, dtype=torch.int64, device="cuda")
    st = losa.lib().losa_select_noalloc(
        mass.data_ptr(), B, H, n, ctypes.c_double(0.99), row_ptr.data_ptr(),
        col_idx.data_ptr(), ctypes.c_int64(cap), ret.data_ptr(), tot.data_ptr(),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    torch.cuda.synchronize()
    losa.check_status()
    pat = losa.select(mass, 64, 0.99)
    ref = pat.export("cpu")
    assert int(row_ptr[-1].item()) == full
    assert torch.equal(row_ptr.cpu(), ref["row_ptr"])
    assert torch.equal(col_idx[:cap].cpu(), ref["col_idx"][:cap])
    assert torch.all(col_idx[cap:] == -7).item()
    pat.close()


def test_noalloc_call_allocates_no_device_memory(losa):
    """After a first call (which loads the kernels and looks up the scratch
    array), a call leaves the device's free memory exactly as it was."""
    mass = _random_mass(2, 300, seed=6)
    B, H, n, _ = mass.shape
    R = B * H * n
    bufs = [torch.empty(R + 1, dtype=torch.int32, device="cuda"),
            torch.empty(R * n, dtype=torch.int32, device="cuda"),
            torch.empty(R, dtype=torch.int64, device="cuda"),
            torch.empty(R, dtype=torch.int64, device="cuda")]

    def call():
        st = losa.lib().losa_select_noalloc(
            mass.data_ptr(), B, H, n, ctypes.c_double(0.99), bufs[0].data_ptr(),
            bufs[1].data_ptr(), ctypes.c_int64(R * n), bufs[2].data_ptr(), bufs[3].data_ptr(),
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == 0
        torch.cuda.synchronize()

    call()
    free0, _ = torch.cuda.mem_get_info()
    reserved0 = torch.cuda.memory_reserved()
    call()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    assert torch.cuda.memory_reserved() == reserved0
    losa.check_status()


def test_noalloc_rejects_rows_beyond_its_scratch(losa):
    mass = torch.zeros(1, 1, 8, 8, device="cuda")
    out = torch.zeros(16, dtype=torch.int64, device="cuda")
    lib = losa.lib()
    # 40 heads x 2047 blocks = 81,880 rows > LOSA_NOALLOC_MAX_ROWS: refused
    # before any device work, so the small buffers are never touched.
    st = lib.losa_select_noalloc(mass.data_ptr(), 1, 40, 2047, ctypes.c_double(0.99),
                                 out.data_ptr(), out.data_ptr(), ctypes.c_int64(16),
                                 out.data_ptr(), out.data_ptr(), None)
    assert st == -1
    assert losa.NOALLOC_MAX_ROWS == 65536
