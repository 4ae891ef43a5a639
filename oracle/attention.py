"""Plain, slow fp64 CPU oracle for exact softmax attention and its gradients.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import this module:
only the test-suite, the smoke check in ``__graft_entry__`` and the ``cpu_baseline``
/ ``--impl reference`` legs of ``bench.py`` call it. It shares no code with the
CUDA path (no kernels, headers, helpers or constants) and imports nothing from it.

What it computes is the plain definition of attention, written out with the full
N x N score matrix materialised per (batch, head), in float64:

    S   = scale * Q K^T                         (then -inf where masked)
    P   = softmax_rows(S)                       (max-subtracted)
    lse = m + ln sum_j exp(S_ij - m)            (natural log, scale and mask included)
    O   = P V

The pages on which the method is described state that the tiled algorithm reaches
this same result "with no approximation" ("FlashAttention-2: Faster Attention with
Better Parallelism and Work Partitioning" review, Abstract; "... Proposed method",
first bullet: output unchanged) and that it computes accurate attention ("Researchers
at Stanford University Propose FlashAttention: Fast and Memory-Efficient Exact
Attention with IO-Awareness", method paragraph). The oracle is therefore the
definition itself; it deliberately does what the method avoids (store S and P).

Masks:
  * causal: key j is visible to query i iff j <= i + (N_k - N_q): the last query
    sees every key (bottom-right alignment, the usual reading for decoding and for
    a query block appended to a longer key sequence); for N_q = N_k this is j <= i.
    The review's "Proposed method" bullet on causal masking gives no formula; the
    alignment for N_q != N_k is this library's reading.
  * block-sparse: a [ceil(N/T), ceil(N/T)] 0/1 tile mask with T = ``mask_block``
    keeps S_ij iff mask[i // T][j // T] != 0 (the block-sparse paragraph of the
    Stanford summary page; the granularity T = 128 is this library's choice).
    Causal and block-sparse may be combined (logical AND).
  * a row with no visible key has P = 0, O = 0 and lse = -inf (the pages are
    silent; this is the only value consistent with lse = ln sum exp over an empty
    set).

Backward: the gradients of L = sum(O * dO) with respect to Q, K, V, from the
materialised P (the Stanford summary page, method paragraph: the normalisation
factor saved by the forward lets the backward recompute attention):

    dV = P^T dO,  dP = dO V^T,  D_i = sum_j P_ij dP_ij  (= sum_c dO_ic O_ic),
    dS = P * (dP - D),  dQ = scale dS K,  dK = scale dS^T Q.

Parity status: every function below is pinned by tests/test_oracle.py against
closed forms, invariants, brute-force finite differences and a library routine;
none is "parity unpinned".
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "attn_scores_ref",
    "attn_probs_ref",
    "attn_fwd_ref",
    "attn_fwd_rows_ref",
    "attn_bwd_ref",
    "attn_dq_rows_ref",
    "attn_dkdv_cols_ref",
    "attn_fwd_block_ref",
    "attn_bwd_block_ref",
]


def _f64(x) -> np.ndarray:
    """Exact upcast of any real array (bf16/fp32 via torch or numpy) to float64."""
    if hasattr(x, "detach"):  # a torch tensor; keep torch out of the arithmetic
        x = x.detach().to("cpu")
        if str(x.dtype) in ("torch.bfloat16", "torch.float16"):
            x = x.float()
        x = x.numpy()
    return np.asarray(x, dtype=np.float64)


def _visible(n_q_rows: np.ndarray, n_k: int, causal: bool, block_mask, mask_block: int,
             causal_offset: int = 0, key_cols=None) -> np.ndarray:
    """Boolean [len(rows), n_k] visibility for the given absolute query rows (or
    [len(rows), len(key_cols)] for the given absolute key columns); with the causal mask
    key j is visible to row i iff j <= i + causal_offset."""
    rows = np.asarray(n_q_rows, dtype=np.int64)
    cols = np.arange(n_k, dtype=np.int64) if key_cols is None else np.asarray(key_cols, dtype=np.int64)
    vis = np.ones((rows.shape[0], cols.shape[0]), dtype=bool)
    if causal:
        vis &= cols[None, :] <= rows[:, None] + causal_offset
    if block_mask is not None:
        bm = np.asarray(block_mask) != 0
        vis &= bm[rows[:, None] // mask_block, cols[None, :] // mask_block]
    return vis


def attn_scores_ref(q, k, scale: float, causal: bool = False, block_mask=None,
                    mask_block: int = 128, rows=None, n_q=None) -> np.ndarray:
    """Masked, scaled scores S for one head: q [R, d], k [N_k, d] -> [R, N_k] fp64.

    ``rows`` gives the absolute index of each query row (default 0..R-1) and ``n_q``
    the problem's number of query rows N_q (default: R when ``rows`` is not given,
    else N_k, i.e. sampled rows of a square problem); masked entries are -inf.
    """
    q = _f64(q)
    k = _f64(k)
    n_k = k.shape[0]
    if rows is None:
        rows = np.arange(q.shape[0])
        if n_q is None:
            n_q = q.shape[0]
    if n_q is None:
        n_q = n_k
    s = float(scale) * (q @ k.T)
    vis = _visible(rows, n_k, causal, block_mask, mask_block, n_k - n_q)
    return np.where(vis, s, -np.inf)


def _softmax_rows(s: np.ndarray):
    """Row softmax of a masked score matrix; returns (P, lse). Empty rows -> (0, -inf)."""
    m = np.max(s, axis=1, keepdims=True)
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    e = np.exp(s - m_safe)  # exp(-inf) = 0 for masked entries
    z = np.sum(e, axis=1, keepdims=True)
    with np.errstate(divide="ignore", invalid="ignore"):
        p = np.where(empty, 0.0, e / np.where(empty, 1.0, z))
        lse = np.where(empty, -np.inf, m_safe + np.log(np.where(empty, 1.0, z)))
    return p, lse[:, 0]


def attn_probs_ref(q, k, scale: float, causal: bool = False, block_mask=None,
                   mask_block: int = 128) -> np.ndarray:
    """Attention probabilities P for one head ([N, d] inputs) -> [N, N] fp64."""
    p, _ = _softmax_rows(attn_scores_ref(q, k, scale, causal, block_mask, mask_block))
    return p


def attn_fwd_ref(q, k, v, causal: bool = False, scale: float | None = None,
                 block_mask=None, mask_block: int = 128):
    """Forward for q [B, H, N_q, d], k and v [B, H, N_k, d] -> (O [B,H,N_q,d],
    lse [B,H,N_q]) in fp64.

    One (b, h) at a time: S materialised, masked, softmaxed, multiplied by V.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    o = np.zeros((B, H, N, v.shape[-1]))
    lse = np.zeros((B, H, N))
    for b in range(B):
        for h in range(H):
            s = attn_scores_ref(q[b, h], k[b, h], scale, causal, block_mask, mask_block)
            p, l = _softmax_rows(s)
            o[b, h] = p @ v[b, h]
            lse[b, h] = l
    return o, lse


def attn_fwd_rows_ref(q_rows, rows, k, v, causal: bool, scale: float,
                      block_mask=None, mask_block: int = 128, n_q=None):
    """Forward for a sample of query rows of ONE head.

    q_rows [R, d] are the queries at absolute positions ``rows`` (length R); k, v are
    the head's full [N, d] keys and values. Returns (O [R, d], lse [R]). Used for
    sampled checks at sizes where the full N x N matrix is too large to hold.
    """
    s = attn_scores_ref(q_rows, k, scale, causal, block_mask, mask_block, rows=rows, n_q=n_q)
    p, lse = _softmax_rows(s)
    return p @ _f64(v), lse


def attn_bwd_ref(q, k, v, do, causal: bool = False, scale: float | None = None,
                 block_mask=None, mask_block: int = 128):
    """Gradients of L = sum(O * dO) for q, dO [B, H, N_q, d] and k, v [B, H, N_k, d],
    in fp64.

    Returns a dict with dq ([B,H,N_q,d]), dk, dv ([B,H,N_k,d]), D ([B,H,N_q],
    sum_j P dP), and the forward's o and lse. D is computed both as
    sum_j P_ij dP_ij and as sum_c dO_ic O_ic; the two must agree (asserted).
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, H, N, d = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = {"dq": np.zeros_like(q), "dk": np.zeros_like(k), "dv": np.zeros_like(v)}
    out["o"] = np.zeros((B, H, N, v.shape[-1]))
    out["lse"] = np.zeros((B, H, N))
    out["D"] = np.zeros((B, H, N))
    for b in range(B):
        for h in range(H):
            s = attn_scores_ref(q[b, h], k[b, h], scale, causal, block_mask, mask_block)
            p, lse = _softmax_rows(s)
            o = p @ v[b, h]
            dv = p.T @ do[b, h]
            dp = do[b, h] @ v[b, h].T
            D = np.sum(p * dp, axis=1)
            D_alt = np.sum(do[b, h] * o, axis=1)
            assert np.allclose(D, D_alt, rtol=1e-9, atol=1e-9 * (1.0 + np.max(np.abs(D_alt), initial=0.0)))
            ds = p * (dp - D[:, None])
            out["dq"][b, h] = scale * (ds @ k[b, h])
            out["dk"][b, h] = scale * (ds.T @ q[b, h])
            out["dv"][b, h] = dv
            out["o"][b, h] = o
            out["lse"][b, h] = lse
            out["D"][b, h] = D
    return out



def attn_dq_rows_ref(q_rows, rows, k, v, do_rows, causal: bool, scale: float,
                     block_mask=None, mask_block: int = 128, n_q=None) -> np.ndarray:
    """dQ for a sample of query rows of ONE head (same definition as attn_bwd_ref).

    Row i needs only its own scores: P_i = softmax(S_i), dP_i = dO_i V^T,
    D_i = sum_j P_ij dP_ij, dS_i = P_i * (dP_i - D_i), dQ_i = scale dS_i K.
    q_rows, do_rows [R, d] at absolute positions ``rows``; k, v the head's [N, d].
    """
    k, v, do_rows = _f64(k), _f64(v), _f64(do_rows)
    s = attn_scores_ref(q_rows, k, scale, causal, block_mask, mask_block, rows=rows, n_q=n_q)
    p, _ = _softmax_rows(s)
    dp = do_rows @ v.T
    D = np.sum(p * dp, axis=1)
    ds = p * (dp - D[:, None])
    return scale * (ds @ k)


def attn_dkdv_cols_ref(q, k, v, do, cols, causal: bool, scale: float, block_mask=None,
                       mask_block: int = 128, row_block: int = 1024):
    """dK and dV for a sample of key rows (columns of S) of ONE head, same definition as
    attn_bwd_ref, for sizes where the N x N matrices are too large to hold at once.

    Column j of the gradients needs every query row's lse_i and D_i = sum_c dO_ic O_ic
    over ALL keys, so those row statistics are computed first, row by row (``row_block``
    rows at a time only to bound memory; each row is the plain softmax of its own
    scores). Then, for the chosen keys j: P_ij = exp(S_ij - lse_i) (0 where masked or
    where row i sees nothing), dP_ij = dO_i . v_j, dS_ij = P_ij (dP_ij - D_i),
    dK_j = scale sum_i dS_ij q_i and dV_j = sum_i P_ij dO_i.
    q, do [N_q, d]; k, v [N_k, d]; cols: absolute key indices. Returns (dK [C, d], dV [C, d]).
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    n_q, n_k = q.shape[0], k.shape[0]
    cols = np.asarray(cols, dtype=np.int64)
    lse = np.empty(n_q)
    D = np.empty(n_q)
    for r0 in range(0, n_q, row_block):
        rows = np.arange(r0, min(n_q, r0 + row_block))
        p, lse[rows] = _softmax_rows(attn_scores_ref(q[rows], k, scale, causal, block_mask, mask_block,
                                                     rows=rows, n_q=n_q))
        D[rows] = np.sum(do[rows] * (p @ v), axis=1)
    vis = _visible(np.arange(n_q), n_k, causal, block_mask, mask_block, n_k - n_q, key_cols=cols)
    s_c = np.where(vis, float(scale) * (q @ k[cols].T), -np.inf)
    fin = np.isfinite(lse)[:, None]
    p_c = np.where(vis & fin, np.exp(s_c - np.where(fin, lse[:, None], 0.0)), 0.0)
    dp_c = do @ v[cols].T
    ds_c = p_c * (dp_c - D[:, None])
    return scale * (ds_c.T @ q), p_c.T @ do


# ---------------------------------------------------------------- key blocks
# Attention over a key sequence split into blocks (one block per GPU of a ring). With
# the causal mask the rule is the global one: key j is visible to query i iff j <= i,
# for absolute positions i = q_off + row and j = k_off + column.

def _block_scores(q, k, scale: float, causal: bool, q_off: int, k_off: int) -> np.ndarray:
    s = float(scale) * (_f64(q) @ _f64(k).T)
    if causal:
        rows = q_off + np.arange(s.shape[0])[:, None]
        cols = k_off + np.arange(s.shape[1])[None, :]
        s = np.where(cols <= rows, s, -np.inf)
    return s


def attn_fwd_block_ref(q, k, v, scale: float, causal: bool = False, q_off: int = 0, k_off: int = 0):
    """One head's partial result over one key block: (O_b, lse_b), the softmax taken over
    the block's visible keys only (O_b = 0, lse_b = -inf for a row that sees none of
    them). q [R, d] at positions q_off.., k and v [C, d] at positions k_off..."""
    p, lse = _softmax_rows(_block_scores(q, k, scale, causal, q_off, k_off))
    return p @ _f64(v), lse


def attn_bwd_block_ref(q, k, v, do, lse, D, scale: float, causal: bool = False, q_off: int = 0, k_off: int = 0):
    """One head's share of the gradients from one key block, given each query row's
    log-sum-exp and D_i = sum_c dO_ic O_ic over the WHOLE key sequence: with
    P = exp(S - lse) on the block, dV_b = P^T dO, dP = dO V_b^T, dS = P (dP - D),
    dQ += scale dS K_b, dK_b = scale dS^T Q. Summed over the blocks these are the
    full gradients (the sum over j of the definition splits along the key blocks).
    Returns (dq_part, dk_b, dv_b)."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    s = _block_scores(q, k, scale, causal, q_off, k_off)
    lse = _f64(lse)[:, None]
    with np.errstate(invalid="ignore"):
        p = np.where(np.isfinite(s) & np.isfinite(lse), np.exp(s - np.where(np.isfinite(lse), lse, 0.0)), 0.0)
    dp = do @ v.T
    ds = p * (dp - _f64(D)[:, None])
    return scale * (ds @ k), scale * (ds.T @ q), p.T @ do

