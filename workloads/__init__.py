"""Seeded synthetic Q/K/V workloads for LoSA's attention hot path.

This module only draws inputs. It holds none of the method's arithmetic
(no attention, no masses, no selection), so both the CUDA path and the CPU
oracle can be fed from it without sharing any of the computation.

The pages evaluate on real video diffusion transformers (Wan2.1-1.3B,
Wan2.1-14B, HunyuanVideo-13B, CogVideoX; legiblepapers.com LoSA page, FAQ Q8)
and score quality with VBench (LoSA abstract, arXiv 2608.12032). Neither the
weights nor VBench exist here, so these seeded tensors stand in for one
attention layer of each model, with the token-grid shapes, head counts and
head dims of those models.

Recipe (all workloads):
  * tokens are a 3D grid (t, h, w) flattened row-major; text tokens, where a
    model has them, come first; the sequence is padded with zero rows at the
    end to a multiple of the block size.
  * E(p) is a random-Fourier-feature map of the grid position p = (t, h, w):
    E(p)_k = A * sqrt(2) * cos(omega_k . p + phi_k), omega_k ~ N(0, 0.3^2 I_3),
    phi_k ~ U[0, 2 pi), one (omega, phi) draw per head, k < head_dim.
  * Q = beta*E(p) + N(0, sigma^2), K = beta*E(p) + N(0, sigma^2), V = N(0, 1)
    with beta = 2, sigma = 0.5; text tokens have E = 0 and N(0, 1) features.
  * 2 % of the key tokens (a seeded choice, per head) get 3*sqrt(d)*u added,
    u one seeded unit direction per head shared by those keys (the sink).
  * The amplitude A is not given by the workload description. It sets how
    far the local peak of the scores stands above the near-uniform
    background, and the pruned fraction swings from ~0 % to ~97 % over a
    narrow range of A whose position depends on the grid size and head dim
    (A = 0.5 prunes 34 % of one Wan2.1-1.3B-shaped head but 2 % of the
    256-token grid; A = 1.0 prunes 34 % of the small grid but 97.5 % of the
    1.3B-shaped head). So A is fixed once per workload, on head 0 at
    tau = 0.99, to prune about 40 % of blocks (the pages' figure, inside the
    30-50 % band the workloads state), and is never retuned.
  * Later denoising steps drift every tensor: X_s = X_{s-1} + 0.05 * N(0, 1).
  * Values are drawn in fp32. For a workload whose caller hands bf16 to the
    library they are rounded once to bf16 (round to nearest even), and the
    bf16 values are what both sides consume. For an fp32 workload (the small
    one) they stay fp32: the library rounds them to tf32 on entry, and the
    oracle is handed round_tf32 of the same values.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

BETA = 2.0
SIGMA = 0.5
OMEGA_STD = 0.3
SINK_FRACTION = 0.02
SINK_GAIN = 3.0
DRIFT = 0.05


@dataclass(frozen=True)
class Workload:
    name: str
    heads: int
    head_dim: int
    grid: tuple  # (T, H, W) video token grid
    block: int
    text_tokens: int = 0
    batch: int = 1
    taus: tuple = (0.99,)
    in_dtype: str = "bf16"  # dtype the caller hands to the library
    sparse_steps: int = 0
    seed: int = 1000
    amplitude: float = 1.0  # A of E(p); fixed once per workload, see above
    notes: str = ""

    @property
    def video_tokens(self) -> int:
        t, h, w = self.grid
        return t * h * w

    @property
    def seq_len(self) -> int:
        return self.text_tokens + self.video_tokens

    @property
    def seq_pad(self) -> int:
        b = self.block
        return (self.seq_len + b - 1) // b * b

    @property
    def n_blocks(self) -> int:
        return self.seq_pad // self.block


WORKLOADS = {
    "tiny": Workload("tiny", heads=2, head_dim=64, grid=(4, 8, 8), block=32,
                     in_dtype="fp32", seed=1000, amplitude=1.1,
                     notes="2 heads, d=64, 4x8x8 grid, block 32, fp32 in"),
    "wan2.1-1.3b": Workload("wan2.1-1.3b", heads=12, head_dim=128, grid=(21, 30, 52),
                            block=64, sparse_steps=10, seed=1001, amplitude=0.505,
                            notes="Wan2.1-1.3B-shaped layer, 32,760 tokens"),
    "cogvideox": Workload("cogvideox", heads=48, head_dim=64, grid=(13, 30, 45),
                          block=64, text_tokens=226, seed=1002, amplitude=0.605,
                          notes="CogVideoX-shaped layer, 226 text + 17,550 video tokens"),
    "hunyuanvideo": Workload("hunyuanvideo", heads=24, head_dim=128, grid=(33, 45, 80),
                             block=128, sparse_steps=40, seed=1003, amplitude=0.545,
                             notes="HunyuanVideo-shaped layer, 118,800 tokens"),
    "wan2.1-14b": Workload("wan2.1-14b", heads=40, head_dim=128, grid=(21, 45, 80),
                           block=64, taus=(0.95, 0.99, 0.999, 1.0), seed=1004,
                           amplitude=0.535,
                           notes="Wan2.1-14B-shaped tau sweep, 75,600 tokens"),
}


def custom(name, heads, head_dim, grid, block, text_tokens=0, seed=7, in_dtype="bf16",
           amplitude=1.0, batch=1):
    """A workload of any shape with the same recipe (edge-case tests)."""
    return Workload(name, heads=heads, head_dim=head_dim, grid=tuple(grid), block=block,
                    text_tokens=text_tokens, seed=seed, in_dtype=in_dtype,
                    amplitude=amplitude, batch=batch)


def _positions(wl: Workload, device) -> torch.Tensor:
    t, h, w = wl.grid
    tt, hh, ww = torch.meshgrid(torch.arange(t, device=device, dtype=torch.float32),
                                torch.arange(h, device=device, dtype=torch.float32),
                                torch.arange(w, device=device, dtype=torch.float32),
                                indexing="ij")
    return torch.stack([tt.reshape(-1), hh.reshape(-1), ww.reshape(-1)], dim=1)  # [Lv, 3]


def generate(wl: Workload, device="cpu", seed=None, amplitude=None, dtype=None):
    """Draw the construction-step Q, K, V of one layer.

    Returns (q, k, v), each [B, H, L_pad, d] contiguous, in `dtype` (default:
    float32 when wl.in_dtype == 'fp32', else bfloat16). Values are
    bf16-rounded for bf16 workloads whatever `dtype` is, and left unrounded
    for fp32 workloads unless `dtype` is bfloat16. Rows >= L are zero.
    """
    seed = wl.seed if seed is None else seed
    amplitude = wl.amplitude if amplitude is None else amplitude
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    B, H, d = wl.batch, wl.heads, wl.head_dim
    Lt, Lv, L, Lp = wl.text_tokens, wl.video_tokens, wl.seq_len, wl.seq_pad
    f32 = torch.float32
    pos = _positions(wl, device)
    q = torch.zeros(B, H, Lp, d, device=device, dtype=f32)
    k = torch.zeros(B, H, Lp, d, device=device, dtype=f32)
    v = torch.zeros(B, H, Lp, d, device=device, dtype=f32)
    n_sink = max(1, int(round(SINK_FRACTION * L)))
    for b in range(B):
        for h in range(H):
            omega = torch.randn(d, 3, generator=g, device=device, dtype=f32) * OMEGA_STD
            phi = torch.rand(d, generator=g, device=device, dtype=f32) * (2 * math.pi)
            E = amplitude * math.sqrt(2.0) * torch.cos(pos @ omega.T + phi)  # [Lv, d]
            qv = BETA * E + SIGMA * torch.randn(Lv, d, generator=g, device=device, dtype=f32)
            kv = BETA * E + SIGMA * torch.randn(Lv, d, generator=g, device=device, dtype=f32)
            q[b, h, Lt:L] = qv
            k[b, h, Lt:L] = kv
            if Lt:
                q[b, h, :Lt] = torch.randn(Lt, d, generator=g, device=device, dtype=f32)
                k[b, h, :Lt] = torch.randn(Lt, d, generator=g, device=device, dtype=f32)
            v[b, h, :L] = torch.randn(L, d, generator=g, device=device, dtype=f32)
            u = torch.randn(d, generator=g, device=device, dtype=f32)
            u = u / u.norm()
            sink = torch.randperm(L, generator=g, device=device)[:n_sink]
            k[b, h, sink] += SINK_GAIN * math.sqrt(d) * u
    return _finish(wl, (q, k, v), dtype)


def drift(wl: Workload, qkv, step: int, device="cpu", dtype=None):
    """One later denoising step: X_s = X_{s-1} + 0.05*N(0,1) on valid rows.

    The step's noise stream is seeded by (workload seed * 100 + step).
    """
    g = torch.Generator(device=device)
    g.manual_seed(wl.seed * 100 + step)
    L = wl.seq_len
    out = []
    for x in qkv:
        y = x.to(device=device, dtype=torch.float32).clone()
        y[:, :, :L] += DRIFT * torch.randn(y[:, :, :L].shape, generator=g, device=device,
                                           dtype=torch.float32)
        out.append(y)
    return _finish(wl, out, dtype)


def _finish(wl, tensors, dtype):
    if dtype is None:
        dtype = torch.float32 if wl.in_dtype == "fp32" else torch.bfloat16
    if wl.in_dtype == "fp32" and dtype != torch.bfloat16:
        return tuple(t.to(dtype).contiguous() for t in tensors)
    rounded = [t.to(torch.bfloat16) for t in tensors]
    return tuple(t.to(dtype).contiguous() for t in rounded)


def round_tf32(x: torch.Tensor) -> torch.Tensor:
    """The value a tf32 operand holds for each fp32 element: the nearest
    number with 11 significant bits (10 stored), ties to even, returned as
    float32. This is input preparation for the oracle (the values the
    library's tf32 path computes on), done through frexp and an integer
    rounding of the significand rather than on the bit pattern: with
    x = m * 2^e and 1/2 <= |m| < 1, the result is round(m * 2^11) * 2^(e - 11)
    (torch.round rounds half to even); below the normal range the spacing
    stays that of the smallest normal exponent. NaN and Inf pass through."""
    x64 = x.to(torch.float64)
    m, e = torch.frexp(x64)
    e = torch.clamp(e, min=-125)
    m = x64 * torch.pow(2.0, (-e).to(torch.float64))
    r = torch.round(m * 2048.0) * torch.pow(2.0, (e - 11).to(torch.float64))
    r = torch.where(torch.isfinite(x64), r, x64)
    return r.to(torch.float32)


def sample_query_blocks(wl: Workload, per_head: int, seed: int = 12345):
    """Seeded sample of (b, h, I) query blocks, always including the last
    (ragged) block of each head. Returns a list of tuples."""
    g = torch.Generator()
    g.manual_seed(seed)
    nq = wl.n_blocks
    out = []
    for b in range(wl.batch):
        for h in range(wl.heads):
            picks = torch.randperm(nq, generator=g)[:max(0, per_head - 1)].tolist()
            picks = sorted(set(picks) | {nq - 1})
            out.extend((b, h, I) for I in picks)
    return out
