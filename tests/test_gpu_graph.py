"""The sparse step inside a CUDA graph.

A frozen pattern is reused at every later step, so a caller can capture the
sparse call once and replay it on fresh Q/K/V copied into the captured input
buffers. losa_sparse_attn (bf16 inputs) does no host synchronisation and no
allocation, so it is capturable; a replay must give exactly what an eager
call gives on the same inputs (same kernel, same launch, same order of
accumulation).
"""
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def losa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import block_sparse_attention_losa_b200 as m
    return m


@pytest.mark.parametrize("heads,d,grid,block", [(2, 128, (3, 10, 13), 64), (2, 64, (2, 8, 16), 32)])
def test_captured_sparse_step_replays_bit_exact(losa, heads, d, grid, block):
    wl = W.custom("graph", heads, d, grid, block, text_tokens=3, amplitude=1.2, seed=41)
    q, k, v = (t.to("cuda", torch.bfloat16) for t in W.generate(wl, dtype=torch.float32))
    _, _, mass = losa.dense_mass(q, k, v, wl.seq_len, block)
    pat = losa.select(mass, block, 0.95)

    qs, ks, vs = (torch.empty_like(t) for t in (q, k, v))
    o_s = torch.empty(q.shape, device="cuda", dtype=torch.bfloat16)
    lse_s = torch.empty(q.shape[:3], device="cuda", dtype=torch.float32)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm-up outside the capture
        losa.sparse_attn(qs, ks, vs, wl.seq_len, pat, out_dtype=torch.bfloat16, o=o_s, lse=lse_s)
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        losa.sparse_attn(qs, ks, vs, wl.seq_len, pat, out_dtype=torch.bfloat16, o=o_s, lse=lse_s)

    for step in (1, 2, 3):
        q2, k2, v2 = (t.to("cuda", torch.bfloat16)
                      for t in W.drift(wl, (q.float().cpu(), k.float().cpu(), v.float().cpu()),
                                       step=step, dtype=torch.float32))
        qs.copy_(q2)
        ks.copy_(k2)
        vs.copy_(v2)
        g.replay()
        o_e, lse_e = losa.sparse_attn(q2, k2, v2, wl.seq_len, pat, out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        losa.check_status()
        assert torch.equal(o_s, o_e)
        assert torch.equal(lse_s, lse_e)
    del g
    pat.close()
