"""Plain, slow fp64 CPU oracle for LoSA's attention hot path.

TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's CPU
baseline leg may import this module. The library's compute path never calls
it, and it shares no code with the CUDA kernels.

What it computes, and where the pages state it (page, section):

  1. Dense construction attention and its row log-sum-exp
     (ubos.tech LoSA post, "How It Works in Practice", Phase 1 - Dense
     Calibration; LoSA abstract, arXiv 2608.12032: "one early dense step").
  2. The exact attention mass of every (head, query block, key block) pair,
     the "mass map" (ubos.tech post, "What the Researchers Propose", stage 1,
     and Phase 1; LoSA abstract: "measures exact block attention masses";
     legiblepapers.com LoSA page, "Summary & Methodology Analysis").
  3. For each head and query block, the smallest key-block set whose
     cumulative mass reaches tau: sort by descending mass, accumulate until
     the threshold is met (ubos.tech post, Phase 2 - Block Mask Generation;
     LoSA abstract; legiblepapers.com, "Summary & Methodology Analysis" and
     FAQ Q4; default tau = 0.99). Masses are turned into 64-bit fixed point
     round(m * 2^48) first, so the sort, the prefix sum and the cut are exact
     integer work.
  4. Block-sparse attention on fresh Q/K/V over the frozen retained key
     blocks (ubos.tech post, Phase 3 - Repeated Sparse Inference;
     legiblepapers.com: later steps attend only to the frozen retained keys
     while Q, K, V are recomputed).

Readings where the pages are silent (each is listed in the design notes):
  * softmax scale 1/sqrt(d) is passed in; attention is bidirectional;
    key rows j >= L (padding) are excluded, query rows i >= L produce O = 0
    and lse = -inf.
  * block mass = the softmax weight summed over the block's valid query rows
    and the key block's columns, divided by the number of valid query rows in
    the block, so each query block's masses sum to 1.
  * "reaches" means cumulative >= threshold, and the threshold is relative
    to the row's own fixed-point total S: keep the first k (k >= 1) in sorted
    order with 2^48 * C_k >= tau_fx * S, tau_fx = round(tau * 2^48).
  * equal masses order by ascending key-block index; a retained row is stored
    in ascending key-block order.
  * sparse steps renormalise the softmax over the retained keys only.

Pins: every function here is checked, in the CPU tests, against closed
forms, invariants, brute force and an independent library routine
(torch scaled_dot_product_attention, scipy logsumexp); see
tests/test_oracle_pins.py.
"""
from __future__ import annotations

import numpy as np

FX_ONE = 1 << 48  # fixed-point scale of a mass: x = round(m * 2^48)


# ---------------------------------------------------------------- attention

def attention_rows(q_rows, k_valid, v_valid, scale):
    """Softmax attention of some query rows over a set of keys (fp64).

    q_rows [n, d], k_valid [m, d], v_valid [m, d], m >= 1.
    Returns (o [n, d], lse [n]) with lse_i = log sum_j exp(scale * q_i . k_j).
    """
    q_rows = np.asarray(q_rows, dtype=np.float64)
    k_valid = np.asarray(k_valid, dtype=np.float64)
    v_valid = np.asarray(v_valid, dtype=np.float64)
    s = (q_rows @ k_valid.T) * scale
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    o = (e / l) @ v_valid
    lse = (m + np.log(l))[:, 0]
    return o, lse


def dense_attention(q, k, v, L, scale):
    """Full attention of the construction step.

    q, k, v: [B, H, L_pad, d]. Keys j >= L are padding and take no weight.
    Returns o [B, H, L_pad, d] (rows >= L are 0) and lse [B, H, L_pad]
    (rows >= L are -inf), both fp64.
    """
    q = np.asarray(q, dtype=np.float64)
    B, H, Lp, d = q.shape
    o = np.zeros((B, H, Lp, d))
    lse = np.full((B, H, Lp), -np.inf)
    for b in range(B):
        for h in range(H):
            ob, lb = attention_rows(q[b, h, :L], k[b, h, :L], v[b, h, :L], scale)
            o[b, h, :L] = ob
            lse[b, h, :L] = lb
    return o, lse


def attention_probs(q, k, L, scale, b, h, rows):
    """softmax(scale * q k^T) for the given valid query rows of one head,
    over all L_pad key columns (columns >= L are 0)."""
    q = np.asarray(q[b, h], dtype=np.float64)
    k = np.asarray(k[b, h], dtype=np.float64)
    Lp = k.shape[0]
    s = (q[rows] @ k[:L].T) * scale
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    p = np.zeros((len(rows), Lp))
    p[:, :L] = e / e.sum(axis=1, keepdims=True)
    return p


# ---------------------------------------------------------------- block mass

def block_mass_row(q, k, L, block, scale, b, h, I):
    """Masses m[b, h, I, :] of one query block: for each key block J, the
    softmax weight summed over the block's valid query rows and J's columns,
    divided by the number of valid query rows of I. Returns [nK] fp64."""
    Lp = np.asarray(k).shape[2]
    nK = Lp // block
    rows = np.arange(I * block, min((I + 1) * block, L))
    p = attention_probs(q, k, L, scale, b, h, rows)  # [|I|, Lp]
    per_key = p.sum(axis=0)                          # summed over the query rows
    return per_key.reshape(nK, block).sum(axis=1) / len(rows)


def block_mass(q, k, L, block, scale):
    """The full mass map [B, H, nQ, nK] (fp64)."""
    B, H, Lp, _ = np.asarray(q).shape
    n = Lp // block
    mass = np.zeros((B, H, n, n))
    for b in range(B):
        for h in range(H):
            for I in range(n):
                mass[b, h, I] = block_mass_row(q, k, L, block, scale, b, h, I)
    return mass


# ---------------------------------------------------------------- selection

def to_fixed(mass):
    """Fixed-point masses: round(m * 2^48), ties to even, as int64.

    m * 2^48 only moves the exponent, so it is exact in fp64 for fp32 and
    fp64 masses alike; np.rint rounds half to even."""
    m = np.asarray(mass, dtype=np.float64)
    if not np.all(np.isfinite(m)):
        raise ValueError("mass map holds NaN or Inf")
    return np.rint(m * float(FX_ONE)).astype(np.int64)


def tau_fixed(tau):
    """tau_fx = round(tau * 2^48), ties to even."""
    return int(np.rint(float(tau) * float(FX_ONE)))


def select_row(x, tau):
    """Smallest key-block set of one query block whose cumulative fixed-point
    mass reaches tau of the row total.

    x: sequence of non-negative ints (fixed-point masses, one per key block).
    Order the blocks by mass, largest first (equal masses: smaller index
    first), accumulate, and stop at the first k >= 1 with
    2^48 * C_k >= tau_fx * S, S = sum(x). Returns (sorted retained indices,
    C_k, S) as Python ints.
    """
    x = [int(v) for v in x]
    t = tau_fixed(tau)
    S = sum(x)
    order = sorted(range(len(x)), key=lambda J: (-x[J], J))
    C = 0
    kept = []
    for J in order:
        C += x[J]
        kept.append(J)
        if FX_ONE * C >= t * S:
            break
    return sorted(kept), C, S


def select(mass, tau):
    """Selection over a whole mass map [B, H, nQ, nK].

    Returns a dict with the CSR pattern (row_ptr int64 [R+1], col_idx int64
    [nnz], rows ordered (b, h, I) row-major), retained_fx and total_fx
    (Python ints, one per row), and x, the fixed-point masses."""
    x = to_fixed(mass)
    B, H, nQ, nK = x.shape
    rows = x.reshape(B * H * nQ, nK)
    row_ptr = [0]
    cols, ret, tot = [], [], []
    for r in range(rows.shape[0]):
        kept, C, S = select_row(rows[r].tolist(), tau)
        cols.extend(kept)
        row_ptr.append(len(cols))
        ret.append(C)
        tot.append(S)
    return dict(row_ptr=np.array(row_ptr, dtype=np.int64),
                col_idx=np.array(cols, dtype=np.int64),
                retained_fx=ret, total_fx=tot, x=x)


# ---------------------------------------------------------------- sparse step

def retained_keys(blocks, block, L):
    """Token indices of the retained key blocks, padding (>= L) dropped."""
    idx = [np.arange(J * block, (J + 1) * block) for J in blocks]
    idx = np.concatenate(idx) if idx else np.zeros(0, dtype=np.int64)
    return idx[idx < L]


def sparse_attention_block(q, k, v, L, block, scale, b, h, I, blocks):
    """Attention of query block I of head (b, h) over the retained key
    blocks only, renormalised over those keys. Returns (o [|I|, d], lse)."""
    rows = np.arange(I * block, min((I + 1) * block, L))
    keys = retained_keys(blocks, block, L)
    return attention_rows(np.asarray(q[b, h], dtype=np.float64)[rows],
                          np.asarray(k[b, h], dtype=np.float64)[keys],
                          np.asarray(v[b, h], dtype=np.float64)[keys], scale)


def sparse_attention(q, k, v, L, block, scale, row_ptr, col_idx):
    """Block-sparse attention for a whole layer with a frozen CSR pattern
    (rows (b, h, I) row-major). Returns o, lse like dense_attention."""
    q = np.asarray(q, dtype=np.float64)
    B, H, Lp, d = q.shape
    n = Lp // block
    o = np.zeros((B, H, Lp, d))
    lse = np.full((B, H, Lp), -np.inf)
    for b in range(B):
        for h in range(H):
            for I in range(n):
                r = (b * H + h) * n + I
                blocks = [int(J) for J in col_idx[row_ptr[r]:row_ptr[r + 1]]]
                rows = np.arange(I * block, min((I + 1) * block, L))
                if len(rows) == 0:
                    continue
                ob, lb = sparse_attention_block(q, k, v, L, block, scale, b, h, I, blocks)
                o[b, h, rows] = ob
                lse[b, h, rows] = lb
    return o, lse
