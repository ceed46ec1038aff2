"""Plain fp64 CPU oracle for exact softmax attention (forward) and its logsumexp.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may call it.  It shares no code,
header, table or helper with the CUDA path.

What it computes (the plain definition, written out):

    s_ij   = scale * sum_k q_ik k_jk                  for j in allowed(i)
    LSE_i  = log sum_{j in allowed(i)} exp(s_ij)
    P_ij   = exp(s_ij - LSE_i)
    O_i    = sum_j P_ij v_j
    allowed(i) = {0..N-1}  (non-causal)   or   {0..i}  (causal)

Sources (web pages about Tri Dao, "FlashAttention-2: Faster Attention with
Better Parallelism and Work Partitioning", arXiv 2307.08691):

* arXiv abstract page, "Abstract": the method computes attention "with no
  approximation"; the standard layer's runtime and memory are quadratic in the
  sequence length because it forms the full score matrix.
* iplexlaw blog "FlashAttention-2: making long-context attention run
  efficiently on GPUs", section "Why long inputs put pressure on memory": a
  conventional implementation materialises the score and probability
  matrices -- which is exactly what this oracle does, on purpose.
* same blog, section "Tiling preserves the attention calculation": the tiled
  method reaches the globally normalised softmax result (only floating-point
  rounding differs), so this untiled definition is the result it must match.
* same blog, section "Three changes improve GPU utilisation": causal masking
  (keys after the query are excluded).

Readings where the pages are silent (each is also listed in the design notes):

* scale is the caller's; the benchmark uses 1/sqrt(d).
* causal alignment: query and key sequences have the same length N, so the
  mask is "key index j > query index i is excluded"; every row keeps >= 1 key.
* LSE is the natural log of sum exp(scaled scores), i.e. after scale.
* an empty row (no allowed key; unreachable with N_q == N_k) gives O = 0 and
  LSE = -inf.

The backward (``attention_bwd_ref``) is the chain rule through the same
three steps, written out at the end of this module.

The oracle is NOT tiled over keys and uses no online softmax: per (b, h) it
materialises S for a block of query rows (at most ``row_block`` rows at a time
so N = 16k fits in RAM; row blocking does not change any value, each row is
computed from all of its keys at once), subtracts the row max, exponentiates,
normalises, and multiplies by V.
"""
from __future__ import annotations

import numpy as np

__all__ = ["attention_ref", "attention_ref_rows", "attention_probs", "attention_ref_rect", "attention_bwd_ref",
           "attention_bwd_ref_rows"]


def _as_f64(x) -> np.ndarray:
    a = np.asarray(x, dtype=np.float64)
    if a.ndim != 4:
        raise ValueError(f"expected a [B,H,N,d] array, got shape {a.shape}")
    return a


def _allowed_mask(rows: np.ndarray, n_keys: int, causal: bool, offset: int = 0) -> np.ndarray:
    """Boolean [len(rows), n_keys]: True where key j is allowed for query row i.

    Causal masking excludes keys after the query (iplexlaw blog, "Three changes
    improve GPU utilisation" names causal-mask handling).  Query row i sits at
    sequence position offset + i; with equal query and key lengths offset = 0
    and the rule is j > i excluded.  With fewer queries than keys (decoding the
    last Nq positions of an Nk-long sequence) offset = Nk - Nq.
    """
    j = np.arange(n_keys)[None, :]
    if causal:
        return j <= rows[:, None] + offset
    return np.ones((rows.shape[0], n_keys), dtype=bool)


def _rows_one_head(q_rows: np.ndarray, k: np.ndarray, v: np.ndarray,
                   rows: np.ndarray, causal: bool, scale: float, offset: int = 0):
    """Exact attention for selected query rows of one (batch, head).

    q_rows: [R, d] (the query vectors of ``rows``), k, v: [N, d].
    Returns (O [R, d], LSE [R]) in float64.
    """
    n_keys = k.shape[0]
    # Scores: the full R x N block, materialised (the "standard attention"
    # the abstract contrasts with the tiled method).
    s = scale * (q_rows @ k.T)
    allowed = _allowed_mask(rows, n_keys, causal, offset)
    s = np.where(allowed, s, -np.inf)
    m = np.max(s, axis=1, keepdims=True)                 # row max over allowed keys
    empty = ~np.isfinite(m)                              # row with no allowed key
    m_safe = np.where(empty, 0.0, m)
    e = np.exp(s - m_safe)                               # exp(-inf) = 0 on masked keys
    l = np.sum(e, axis=1, keepdims=True)                 # row sum
    with np.errstate(divide="ignore", invalid="ignore"):
        p = np.where(empty, 0.0, e / np.where(empty, 1.0, l))
        lse = np.where(empty[:, 0], -np.inf, m_safe[:, 0] + np.log(np.where(empty[:, 0], 1.0, l[:, 0])))
    o = p @ v
    return o, lse


def attention_ref(q, k, v, causal: bool = False, scale: float | None = None,
                  row_block: int = 2048):
    """Exact attention forward for [B, H, N, d] inputs.

    Returns ``(O, LSE)``: O float64 [B, H, N, d], LSE float64 [B, H, N]
    (natural log).  Inputs of any real dtype are upcast to float64 first, so
    bf16 values are taken exactly.
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    B, H, N, d = q.shape
    if k.shape != (B, H, N, d) or v.shape != (B, H, N, d):
        raise ValueError("q, k, v must share the shape [B, H, N, d]")
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    o = np.empty((B, H, N, d), dtype=np.float64)
    lse = np.empty((B, H, N), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            for r0 in range(0, N, row_block):
                rows = np.arange(r0, min(N, r0 + row_block))
                ob, lb = _rows_one_head(q[b, h, rows], k[b, h], v[b, h], rows,
                                        causal, float(scale))
                o[b, h, rows] = ob
                lse[b, h, rows] = lb
    return o, lse


def attention_ref_rows(q, k, v, b: int, h: int, rows, causal: bool = False,
                       scale: float | None = None):
    """Exact attention for a sample of query rows of one head.

    Same definition as :func:`attention_ref`, evaluated only for ``rows`` of
    head (b, h); used to check full-size launches on sampled outputs.
    q, k, v may be any array-likes indexable as [B, H, N, d] (e.g. float64
    numpy views of bf16 tensors).  Returns (O [R, d], LSE [R]) float64.
    """
    rows = np.asarray(rows, dtype=np.int64)
    qb = np.asarray(q[b, h], dtype=np.float64)
    kb = np.asarray(k[b, h], dtype=np.float64)
    vb = np.asarray(v[b, h], dtype=np.float64)
    d = qb.shape[-1]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    return _rows_one_head(qb[rows], kb, vb, rows, causal, float(scale))


def attention_probs(q, k, causal: bool = False, scale: float | None = None):
    """The materialised probability matrix P [B, H, N, N] (small inputs only).

    P_ij = exp(s_ij - LSE_i) on allowed keys, 0 elsewhere.  Exposed so tests
    can check the row-stochastic property directly.
    """
    q, k = _as_f64(q), _as_f64(k)
    B, H, N, d = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    p = np.zeros((B, H, N, N), dtype=np.float64)
    rows = np.arange(N)
    allowed = _allowed_mask(rows, N, causal)
    for b in range(B):
        for h in range(H):
            s = np.where(allowed, float(scale) * (q[b, h] @ k[b, h].T), -np.inf)
            m = np.max(s, axis=1, keepdims=True)
            e = np.exp(s - m)
            p[b, h] = e / np.sum(e, axis=1, keepdims=True)
    return p


def attention_ref_rect(q, k, v, causal: bool = False, scale: float | None = None,
                       row_block: int = 2048):
    """Exact attention with Nq query rows and Nk >= Nq keys.

    q: [B, H, Nq, d]; k, v: [B, H, Nk, d].  Query row i is sequence position
    Nk - Nq + i (the last Nq positions, as when decoding or prefilling a
    chunk after a cached prefix); causal masking excludes keys after that
    position.  With Nq == Nk this is exactly :func:`attention_ref`.
    Returns (O [B, H, Nq, d], LSE [B, H, Nq]) in float64.
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    if k.shape != (B, H, Nk, d) or v.shape != (B, H, Nk, d) or Nq > Nk:
        raise ValueError("need q [B,H,Nq,d], k and v [B,H,Nk,d] with Nq <= Nk")
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    offset = Nk - Nq
    o = np.empty((B, H, Nq, d), dtype=np.float64)
    lse = np.empty((B, H, Nq), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            for r0 in range(0, Nq, row_block):
                rows = np.arange(r0, min(Nq, r0 + row_block))
                ob, lb = _rows_one_head(q[b, h, rows], k[b, h], v[b, h], rows, causal, float(scale), offset)
                o[b, h, rows] = ob
                lse[b, h, rows] = lb
    return o, lse


# ---------------------------------------------------------------------- backward
#
# Gradients of the same definition for an upstream gradient dO (the pages say
# only that gradient comparisons use tolerances -- iplexlaw blog, "Tiling
# preserves the attention calculation" -- so the definition is the chain rule
# through the three steps above, written out):
#
#     dV     = P^T dO
#     dP     = dO V^T
#     dS_ij  = P_ij (dP_ij - sum_k P_ik dP_ik)       (softmax Jacobian, per row)
#     dQ     = scale * dS K
#     dK     = scale * dS^T Q
#
# Masked entries have P_ij = 0, hence dS_ij = 0.  The row sum
# sum_k P_ik dP_ik is taken from P and dP as written (not from O).

def _probs_one_head(q, k, causal, scale, offset=0):
    """The materialised P [Nq, Nk] of one head (rows with no key: zeros)."""
    rows = np.arange(q.shape[0])
    s = np.where(_allowed_mask(rows, k.shape[0], causal, offset), scale * (q @ k.T), -np.inf)
    m = np.max(s, axis=1, keepdims=True)
    empty = ~np.isfinite(m)
    e = np.exp(s - np.where(empty, 0.0, m))
    l = np.sum(e, axis=1, keepdims=True)
    return np.where(empty, 0.0, e / np.where(empty, 1.0, l))


def _bwd_one_head(q, k, v, do, causal, scale):
    p = _probs_one_head(q, k, causal, scale)
    dv = p.T @ do
    dp = do @ v.T
    ds = p * (dp - np.sum(p * dp, axis=1, keepdims=True))
    return scale * (ds @ k), scale * (ds.T @ q), dv


def attention_bwd_ref(q, k, v, do, causal: bool = False, scale: float | None = None):
    """Exact gradients (dQ, dK, dV) of attention for [B, H, N, d] inputs and dO.

    Float64 throughout; the full N x N probability matrix of each head is
    materialised (test sizes only).
    """
    q, k, v, do = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(do)
    B, H, N, d = q.shape
    if k.shape != q.shape or v.shape != q.shape or do.shape != q.shape:
        raise ValueError("q, k, v, do must share the shape [B, H, N, d]")
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
    for b in range(B):
        for h in range(H):
            dq[b, h], dk[b, h], dv[b, h] = _bwd_one_head(q[b, h], k[b, h], v[b, h], do[b, h], causal, float(scale))
    return dq, dk, dv


def attention_bwd_ref_rows(q, k, v, do, b: int, h: int, rows, causal: bool = False, scale: float | None = None,
                           row_block: int = 1024):
    """dQ, dK and dV rows ``rows`` of head (b, h), for long sequences.

    dQ row i needs row i of P and dP; dK and dV row j need column j of P and
    dS, i.e. every query row, which is processed ``row_block`` rows at a time
    (blocking over query rows changes no value: each row is computed from all
    of its keys at once, and column sums are plain sums over rows).
    Returns (dQ [R, d], dK [R, d], dV [R, d]) float64.
    """
    rows = np.asarray(rows, dtype=np.int64)
    qb, kb, vb, dob = (np.asarray(t[b, h], dtype=np.float64) for t in (q, k, v, do))
    N, d = qb.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    scale = float(scale)
    dk = np.zeros((rows.size, d))
    dv = np.zeros((rows.size, d))
    dq = np.zeros((rows.size, d))
    for r0 in range(0, N, row_block):
        qr = np.arange(r0, min(N, r0 + row_block))
        s = np.where(_allowed_mask(qr, N, causal), scale * (qb[qr] @ kb.T), -np.inf)
        m = np.max(s, axis=1, keepdims=True)
        e = np.exp(s - m)
        p = e / np.sum(e, axis=1, keepdims=True)
        dp = dob[qr] @ vb.T
        ds = p * (dp - np.sum(p * dp, axis=1, keepdims=True))
        dv += p[:, rows].T @ dob[qr]
        dk += scale * (ds[:, rows].T @ qb[qr])
        sel = (rows >= r0) & (rows < r0 + qr.size)
        dq[sel] = scale * (ds[rows[sel] - r0] @ kb)
    return dq, dk, dv
