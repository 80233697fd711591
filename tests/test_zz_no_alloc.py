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
