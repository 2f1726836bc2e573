"""fp64 CPU oracle for the fused chunked KL-distillation loss.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It shares no code
with the CUDA library (``chunked_kl_loss_ckl_b200``) and imports nothing from
it; both sides read the same seeded arrays from ``ckl_synth``.

What it computes, and where that comes from
-------------------------------------------
The pages describe the method ("Efficient Knowledge Distillation for LLMs:
Offline Top-K Logits and a Fused Chunked KL Loss", Multiverse Computing) in
four summaries:

* "Дистилляция LLM на одной GPU: offline-кэш и chunked KL loss"
  (aivibenews.ru), section «Два приёма»: the teacher is run once and its 100
  most likely tokens per position are cached; the loss is computed chunk by
  chunk of the context, hidden states are projected to logits only for the
  chunk, folded into a running loss, and the chunk is dropped; the backward
  recomputes each chunk.
* "Destylacja wiedzy AI taniej o 50% ..." (aifeed.pl), section "Dwie kluczowe
  zmiany systemowe": dense KL builds the grid with one row per vocabulary
  entry and one column per sequence position; dense, forward-chunked and
  fused-chunked compute the same loss.
* "Tối ưu hóa chi phí chưng cất tri thức ..." (aihot.vn), section "Hai thay
  đổi hệ thống": the three ways compute one loss and are mathematically
  equivalent; the paper gives a closed-form gradient (not reproduced on the
  pages).

The pages never print the loss formula.  The reading used here (the plainest
one those statements support) is the forward KL of the renormalised teacher
top-K distribution against the full-vocabulary student softmax, averaged
over the positions that count:

    z_tv   = sum_j H_tj W_vj                               (the dense grid)
    lse_t  = log sum_v exp(z_tv)                           (every row)
    p_tk   = exp(logp_tk - log sum_k' exp(logp_tk'))       (top-K renormalised)
    KL_t   = sum_k p_tk (log p_tk - (z_{t,idx_tk} - lse_t))   (p = 0 terms: 0)
    loss   = sum_t m_t KL_t / N,  N = sum_t m_t            (loss = 0 if N = 0)
    dL/dz_tv = G_tv = (g m_t / N) (q_tv - sum_k p_tk [idx_tk = v]),
               q_tv = exp(z_tv - lse_t)
    dH = G W,   dW = G^T H

Repeated ids within a row are taken literally: every cached entry is its own
term of the sum over k, and the gradient adds the entries' p at that id.

Inputs are the bf16-rounded H and W (widened exactly to fp64), int32 ids,
fp32 teacher log-probs and an optional uint8 mask (non-zero = counts).  All
arithmetic is fp64; matrix products use numpy's matmul as a library step.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "widen_bf16",
    "check_inputs",
    "renormalise_topk",
    "logits",
    "logsumexp_rows",
    "kl_rows",
    "grad_logits",
    "dense_values",
    "dense",
    "chunked",
    "rows_subset",
    "dw_rows_from_subset",
    "topk_cache",
]


def widen_bf16(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> fp64 values, exactly."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def check_inputs(idx: np.ndarray, logp: np.ndarray, V: int) -> None:
    """Reject ids outside [0, V) and teacher rows with no finite log-prob.

    A row whose log-probs are all -inf has no distribution to renormalise;
    NaN or +inf log-probs are not log-probabilities.
    """
    idx = np.asarray(idx)
    if idx.size and (idx.min() < 0 or idx.max() >= V):
        raise ValueError("teacher id outside [0, V)")
    lp = np.asarray(logp, dtype=np.float64)
    if np.isnan(lp).any() or np.isposinf(lp).any():
        raise ValueError("teacher log-prob is NaN or +inf")
    if lp.size and (~np.isfinite(lp)).all(axis=-1).any():
        raise ValueError("teacher row with every log-prob = -inf")


def renormalise_topk(logp: np.ndarray):
    """p_tk = softmax over the K cached log-probs of row t.

    The cache keeps only the teacher's top-K tokens per position (page
    «Два приёма», aivibenews.ru); the mass outside them is dropped and the
    K entries are renormalised to sum to one.  Returns (p, log p), with
    log p = -inf where the cached log-prob is -inf.
    """
    lp = np.asarray(logp, dtype=np.float64)
    mx = lp.max(axis=-1, keepdims=True)
    ell = mx + np.log(np.exp(lp - mx).sum(axis=-1, keepdims=True))
    logp_n = lp - ell
    return np.exp(logp_n), logp_n


def logits(H: np.ndarray, W: np.ndarray) -> np.ndarray:
    """z_tv = sum_j H_tj W_vj: the student's logit grid for these rows.

    "One row per vocabulary entry and one column per sequence position"
    (aifeed.pl, "Dwie kluczowe zmiany systemowe"); stored here as [T, V].
    """
    return H @ W.T


def logsumexp_rows(Z: np.ndarray) -> np.ndarray:
    """lse_t = log sum_v exp(z_tv), shifted by the row max for range."""
    M = Z.max(axis=1, keepdims=True)
    return (M + np.log(np.exp(Z - M).sum(axis=1, keepdims=True)))[:, 0]


def kl_rows(Z: np.ndarray, lse: np.ndarray, idx: np.ndarray, p: np.ndarray,
            logp_n: np.ndarray) -> np.ndarray:
    """KL_t = sum_k p_tk (log p_tk - log q_{t, idx_tk}), 0 log 0 = 0.

    log q_tv = z_tv - lse_t is the student's full-vocabulary log-softmax.
    """
    zg = np.take_along_axis(Z, np.asarray(idx, dtype=np.int64), axis=1)
    logq = zg - lse[:, None]
    safe_logp = np.where(p > 0, logp_n, 0.0)
    terms = np.where(p > 0, p * (safe_logp - logq), 0.0)
    return terms.sum(axis=1)


def grad_logits(Z: np.ndarray, lse: np.ndarray, idx: np.ndarray, p: np.ndarray,
                scale_rows: np.ndarray) -> np.ndarray:
    """G_tv = scale_t (q_tv - sum_k p_tk [idx_tk = v]).

    The closed form of dL/dz: the sum over k of -p_tk log q_{t, idx_tk} has
    derivative q_tv sum_k p_tk - sum_k p_tk [idx_tk = v], and sum_k p_tk = 1
    after renormalisation; p log p does not depend on z.  ``scale_rows`` is
    g m_t / N.
    """
    G = np.exp(Z - lse[:, None])
    rows = np.repeat(np.arange(Z.shape[0]), idx.shape[1])
    np.add.at(G, (rows, np.asarray(idx, dtype=np.int64).ravel()), -p.ravel())
    return G * scale_rows[:, None]


def _mask_vec(mask, T):
    if mask is None:
        return np.ones(T, dtype=np.float64)
    return (np.asarray(mask) != 0).astype(np.float64)


def dense_values(H: np.ndarray, W: np.ndarray, idx, logp, mask=None, g: float = 1.0,
                 want_grad: bool = True) -> dict:
    """The textbook dense loss on fp64 H [T, d] and W [V, d].

    Builds the whole [T, V] grid, then reduces.  Returns loss, lse[T], kl[T]
    (every row, masked or not) and, when asked, dH[T, d] and dW[V, d] for
    upstream gradient ``g``.
    """
    T, V = H.shape[0], W.shape[0]
    check_inputs(idx, logp, V)
    m = _mask_vec(mask, T)
    N = m.sum()
    p, logp_n = renormalise_topk(logp)
    Z = logits(H, W)
    lse = logsumexp_rows(Z)
    kl = kl_rows(Z, lse, idx, p, logp_n)
    loss = float((m * kl).sum() / N) if N > 0 else 0.0
    out = dict(loss=loss, lse=lse, kl=kl, N=int(N))
    if want_grad:
        scale = (g * m / N) if N > 0 else np.zeros(T)
        G = grad_logits(Z, lse, idx, p, scale)
        out["dH"] = G @ W
        out["dW"] = G.T @ H
    return out


def dense(H_bits, W_bits, idx, logp, mask=None, g: float = 1.0, want_grad: bool = True) -> dict:
    """``dense_values`` on the bf16 inputs, widened exactly to fp64."""
    return dense_values(widen_bf16(H_bits), widen_bf16(W_bits), idx, logp, mask, g, want_grad)


def chunked(H_bits, W_bits, idx, logp, mask=None, g: float = 1.0, chunk: int = 64,
            want_grad: bool = True) -> dict:
    """The same loss one block of ``chunk`` rows at a time (never holds [T, V]).

    Each block projects its rows to logits, adds its share to the running
    loss and to dW, writes its rows of lse and dH, and is dropped
    (aivibenews.ru «Два приёма»; agentlenshq.com section
    "2つのシステム変更").  N is counted over the whole mask first, because
    the mean divides every row by it.
    """
    H = widen_bf16(H_bits)
    W = widen_bf16(W_bits)
    T, d, V = H.shape[0], H.shape[1], W.shape[0]
    check_inputs(idx, logp, V)
    m = _mask_vec(mask, T)
    N = m.sum()
    p, logp_n = renormalise_topk(logp)
    lse = np.empty(T)
    kl = np.empty(T)
    running = 0.0
    dH = np.empty((T, d)) if want_grad else None
    dW = np.zeros((V, d)) if want_grad else None
    for c0 in range(0, T, chunk):
        c1 = min(T, c0 + chunk)
        Zc = logits(H[c0:c1], W)
        lse[c0:c1] = logsumexp_rows(Zc)
        kl[c0:c1] = kl_rows(Zc, lse[c0:c1], idx[c0:c1], p[c0:c1], logp_n[c0:c1])
        running += float((m[c0:c1] * kl[c0:c1]).sum())
        if want_grad:
            scale = (g * m[c0:c1] / N) if N > 0 else np.zeros(c1 - c0)
            Gc = grad_logits(Zc, lse[c0:c1], idx[c0:c1], p[c0:c1], scale)
            dH[c0:c1] = Gc @ W
            dW += Gc.T @ H[c0:c1]
    out = dict(loss=running / N if N > 0 else 0.0, lse=lse, kl=kl, N=int(N))
    if want_grad:
        out["dH"] = dH
        out["dW"] = dW
    return out


def rows_subset(H_bits, W_bits, idx, logp, rows, N: int, g: float = 1.0,
                mask=None, block_v: int = 32768) -> dict:
    """lse, KL and dH for a few rows of a workload too large for ``dense``.

    Each selected row is computed exactly as in ``dense``; N (the count of
    positions that count over the WHOLE workload) is passed in, since the
    mean divides by it.  W is widened to fp64 one block of vocabulary rows
    at a time to bound memory; every z_tv is still one dot product.
    """
    rows = np.asarray(rows, dtype=np.int64)
    V = W_bits.shape[0]
    check_inputs(idx[rows], logp[rows], V)
    Hs = widen_bf16(H_bits[rows])
    Z = np.empty((rows.size, V))
    for v0 in range(0, V, block_v):
        v1 = min(V, v0 + block_v)
        Z[:, v0:v1] = logits(Hs, widen_bf16(W_bits[v0:v1]))
    p, logp_n = renormalise_topk(logp[rows])
    lse = logsumexp_rows(Z)
    kl = kl_rows(Z, lse, idx[rows], p, logp_n)
    m = _mask_vec(None if mask is None else np.asarray(mask)[rows], rows.size)
    scale = (g * m / N) if N > 0 else np.zeros(rows.size)
    G = grad_logits(Z, lse, idx[rows], p, scale)
    dH = np.zeros((rows.size, H_bits.shape[1]))
    for v0 in range(0, V, block_v):
        v1 = min(V, v0 + block_v)
        dH += G[:, v0:v1] @ widen_bf16(W_bits[v0:v1])
    return dict(lse=lse, kl=kl, dH=dH, G=G, rows=rows)


def dw_rows_from_subset(H_bits, G: np.ndarray, rows, vrows) -> np.ndarray:
    """dW_v = sum_t G_tv H_t for the vocabulary rows ``vrows``.

    Valid when every position outside ``rows`` is masked (G is zero there),
    which is how the full-size dW checks are set up.  ``G`` is the
    ``rows_subset`` gradient of those rows.
    """
    rows = np.asarray(rows, dtype=np.int64)
    vrows = np.asarray(vrows, dtype=np.int64)
    Hs = widen_bf16(H_bits[rows])
    return G[:, vrows].T @ Hs


def topk_cache(logits_bits: np.ndarray, K: int):
    """The teacher's offline cache: per row, the K most likely tokens.

    "Дистилляция LLM на одной GPU: offline-кэш и chunked KL loss", section
    «Два приёма»: the teacher runs once and the 100 most likely tokens per
    position are kept.  Given the teacher's logits (bf16 bits, [T, V]),
    returns ids [T, K] ordered by descending logit (equal logits: smaller id
    first) and their log-probabilities under the full-vocabulary softmax,
    z_v - log sum_u exp z_u, in fp64.
    """
    z = widen_bf16(logits_bits)
    T, V = z.shape
    if K < 1 or K > V:
        raise ValueError("need 1 <= K <= V")
    ids = np.empty((T, K), dtype=np.int64)
    cols = np.arange(V)
    for t in range(T):
        order = np.lexsort((cols, -z[t]))   # primary: -z, then id
        ids[t] = order[:K]
    lse = logsumexp_rows(z)
    logp = np.take_along_axis(z, ids, axis=1) - lse[:, None]
    return ids.astype(np.int32), logp
