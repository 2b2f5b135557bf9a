"""fp64 CPU oracle for exact attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import this package.  The library under
``exact_io_aware_55_b200/`` never imports it, and it imports nothing from
there: the two share no code.

What it computes is the plain definition of attention that the pages say the
tiled kernel reproduces exactly (explainers.rudrite.com "flash-attention-anatomy",
Q&A "What is online softmax and how does tiling keep it exact?"; chipfoundryservices
glossary "flash attention", comparison table row "Result: exact"):

    S   = scale * Q K^T                       (per batch b, head h)
    S_ij = -inf for j > i           when causal (top-left aligned, Nq == Nk)
    m_i = max_j S_ij,  l_i = sum_j exp(S_ij - m_i)
    P   = exp(S - m) / l                      (two-pass row softmax, materialised)
    O   = P V,         LSE_i = m_i + ln l_i

and its gradient for a loss L with dL/dO = dO (explainers.rudrite.com, Q&A
"How does FlashAttention save memory in the backward pass?" -- the backward needs
P; here P is simply materialised):

    D_i = sum_c dO_ic O_ic
    dV  = P^T dO,   dP = dO V^T,   dS = P o (dP - D)
    dQ  = scale * dS K,            dK = scale * dS^T Q

The factor ``scale`` on dQ and dK is the chain rule through S = scale*QK^T.
Everything is float64.  Rows are processed in blocks only to bound memory
(a full 32768 x 32768 fp64 score matrix is 8.6 GB); each row's softmax is
always taken over the complete row, never online.

Pins (see tests/test_oracle_pins.py): brute-force triple loops, an independent
online-softmax recurrence, closed forms (constant scores -> mean of V, N = 1),
convex hull / affine / permutation invariants, central finite differences of
L = sum(dO o O), and the gradient sum identities.  No function here is
"parity unpinned": the rectangular (decode) functions are pinned in
tests/test_oracle_decode.py.
"""
from __future__ import annotations

import numpy as np

# Largest number of fp64 score entries materialised at once (256 MB).
_MAX_BLOCK_ELEMS = 32 * 1024 * 1024


def _row_block(n_rows: int, n_cols: int) -> int:
    return max(1, min(n_rows, _MAX_BLOCK_ELEMS // max(1, n_cols)))


def _scores(qh, kh, scale, causal, r0, r1):
    """S rows r0:r1 of one head, with the causal mask applied as -inf."""
    s = scale * (qh[r0:r1] @ kh.T)
    if causal:
        rows = np.arange(r0, r1)[:, None]
        cols = np.arange(kh.shape[0])[None, :]
        s = np.where(cols > rows, -np.inf, s)
    return s


def _softmax_rows(s):
    """Two-pass row softmax: returns (P, m, l)."""
    m = np.max(s, axis=1)
    e = np.exp(s - m[:, None])
    l = np.sum(e, axis=1)
    return e / l[:, None], m, l


def head_forward(qh, kh, vh, scale, causal, rows=None):
    """Forward of one head.  ``rows`` (optional index array) restricts the
    output rows; each is still a full-row softmax over all keys.
    Returns (O[rows], LSE[rows])."""
    n = qh.shape[0]
    if rows is None:
        o = np.empty((n, vh.shape[1]), dtype=np.float64)
        lse = np.empty(n, dtype=np.float64)
        rb = _row_block(n, kh.shape[0])
        for r0 in range(0, n, rb):
            r1 = min(n, r0 + rb)
            p, m, l = _softmax_rows(_scores(qh, kh, scale, causal, r0, r1))
            o[r0:r1] = p @ vh
            lse[r0:r1] = m + np.log(l)
        return o, lse
    rows = np.asarray(rows)
    s = scale * (qh[rows] @ kh.T)
    if causal:
        s = np.where(np.arange(kh.shape[0])[None, :] > rows[:, None], -np.inf, s)
    p, m, l = _softmax_rows(s)
    return p @ vh, m + np.log(l)


def attention_forward(q, k, v, scale, causal):
    """O [B,H,N,d] and LSE [B,H,N] (natural log) in float64."""
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    B, H, N, d = q.shape
    o = np.empty_like(q)
    lse = np.empty((B, H, N), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            o[b, h], lse[b, h] = head_forward(q[b, h], k[b, h], v[b, h], scale, causal)
    return o, lse


def attention_probs(q, k, scale, causal):
    """The materialised P of one head (small cases only)."""
    s = _scores(np.asarray(q, np.float64), np.asarray(k, np.float64), scale, causal, 0, q.shape[0])
    return _softmax_rows(s)[0]


def head_backward(qh, kh, vh, doh, scale, causal):
    """Gradients of one head: (dQ, dK, dV, O, LSE), all float64."""
    n = qh.shape[0]
    o, lse = head_forward(qh, kh, vh, scale, causal)
    dq = np.empty_like(qh)
    dk = np.zeros_like(kh)
    dv = np.zeros_like(vh)
    rb = _row_block(n, kh.shape[0])
    for r0 in range(0, n, rb):
        r1 = min(n, r0 + rb)
        p, _, _ = _softmax_rows(_scores(qh, kh, scale, causal, r0, r1))
        dob = doh[r0:r1]
        dvec = np.sum(dob * o[r0:r1], axis=1)          # D_i = rowsum(dO o O)
        dv += p.T @ dob                                 # dV = P^T dO
        dp = dob @ vh.T                                 # dP = dO V^T
        ds = p * (dp - dvec[:, None])                   # dS = P o (dP - D)
        dq[r0:r1] = scale * (ds @ kh)                   # dQ = scale dS K
        dk += scale * (ds.T @ qh[r0:r1])                # dK = scale dS^T Q
    return dq, dk, dv, o, lse


def attention_backward(q, k, v, do, scale, causal):
    """(dQ, dK, dV) [B,H,N,d] float64 for dL/dO = do."""
    q, k, v, do = (np.asarray(x, dtype=np.float64) for x in (q, k, v, do))
    B, H, N, d = q.shape
    dq, dk, dv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    for b in range(B):
        for h in range(H):
            dq[b, h], dk[b, h], dv[b, h], _, _ = head_backward(
                q[b, h], k[b, h], v[b, h], do[b, h], scale, causal)
    return dq, dk, dv


def head_backward_sampled(qh, kh, vh, doh, scale, causal, rows, cols):
    """Gradients of one head at sampled positions, for sizes where the full
    backward is too slow: dQ at query ``rows``, dK and dV at key ``cols``.

    dQ_i needs only row i of P and dP.  dK_j and dV_j need column j of P and
    dS for every query row, hence m, l and D for every row: a full forward of
    the head is run first (row-blocked, full-row softmax)."""
    rows = np.asarray(rows)
    cols = np.asarray(cols)
    n = qh.shape[0]
    # dQ rows
    s = scale * (qh[rows] @ kh.T)
    if causal:
        s = np.where(np.arange(kh.shape[0])[None, :] > rows[:, None], -np.inf, s)
    p, _, _ = _softmax_rows(s)
    o_r = p @ vh
    dvec_r = np.sum(doh[rows] * o_r, axis=1)
    ds = p * (doh[rows] @ vh.T - dvec_r[:, None])
    dq_rows = scale * (ds @ kh)
    # statistics of every row
    m_all = np.empty(n)
    l_all = np.empty(n)
    d_all = np.empty(n)
    rb = _row_block(n, kh.shape[0])
    for r0 in range(0, n, rb):
        r1 = min(n, r0 + rb)
        pb, mb, lb = _softmax_rows(_scores(qh, kh, scale, causal, r0, r1))
        m_all[r0:r1] = mb
        l_all[r0:r1] = lb
        d_all[r0:r1] = np.sum(doh[r0:r1] * (pb @ vh), axis=1)
    # columns of P, dP, dS
    sc = scale * (qh @ kh[cols].T)                       # [n, |cols|]
    if causal:
        sc = np.where(cols[None, :] > np.arange(n)[:, None], -np.inf, sc)
    pc = np.exp(sc - m_all[:, None]) / l_all[:, None]
    dpc = doh @ vh[cols].T
    dsc = pc * (dpc - d_all[:, None])
    dv_cols = pc.T @ doh
    dk_cols = scale * (dsc.T @ qh)
    return dq_rows, dk_cols, dv_cols



def head_forward_rect(qh, kh, vh, scale, causal):
    """Forward of one head with Nq query rows against Nk keys: decoding new
    queries against a KV cache (chipfoundryservices glossary "flash attention",
    closing section, which names inference with a KV cache as the setting the
    method is used in).  Causal masking is aligned to the end of the key sequence:
    query i (0-based among the Nq) sees keys j <= Nk - Nq + i, so the Nq queries
    are the last Nq positions of a causal sequence of length Nk.  Plain
    definition, full rows, two-pass softmax.  Returns (O [Nq, d], LSE [Nq])."""
    nq, nk = qh.shape[0], kh.shape[0]
    s = scale * (qh @ kh.T)
    if causal:
        lim = nk - nq + np.arange(nq)[:, None]
        s = np.where(np.arange(nk)[None, :] > lim, -np.inf, s)
    p, m, l = _softmax_rows(s)
    return p @ vh, m + np.log(l)


def attention_forward_rect(q, k, v, scale, causal):
    """O [B,H,Nq,d] and LSE [B,H,Nq] for queries q [B,H,Nq,d] against k, v [B,H,Nk,d]."""
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    B, H, Nq, d = q.shape
    o = np.empty((B, H, Nq, v.shape[3]))
    lse = np.empty((B, H, Nq))
    for b in range(B):
        for h in range(H):
            o[b, h], lse[b, h] = head_forward_rect(q[b, h], k[b, h], v[b, h], scale, causal)
    return o, lse
