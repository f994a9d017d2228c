"""Float64 CPU oracle for Parallax attention.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It shares no code
with the CUDA path (the seeded input generator is the only module both sides
use), and it is deliberately plain and slow.

What it computes ("Parallax: Parameterized Local Linear Attention for Language
Modeling", arXiv 2605.29157):

* The layer output is softmax attention minus a covariance correction,
  ``o_i = o^SA_i - Sigma_KV^(i) rho_i`` (gist.science summary, "Mecanismo
  central", the one printed formula), where ``rho_i`` is the per-query probe
  (agihunt.info summary: rho = W_R x, with its own RMSNorm and RoPE; the
  kernels receive it as the tensor R).
* ``Sigma_KV^(i)`` is the softmax-weighted covariance of the visible values
  and keys, ``sum_j p_ij (v_j - vbar_i)(k_j - kbar_i)^T``, with
  ``p_ij = softmax_j(q_i . k_j / sqrt(d))`` (rainbus.top summary, "Softmax
  Attention" and the six-step forward in "方法步骤详情": softmax weights, key
  differences, probe inner products, corrected weights, two outputs, combine).
* The boundary amplification factor eta is zero (gist.science, "Eliminación
  de la Amplificación de Frontera"), so nothing multiplies the correction.

The function below writes that definition out in two passes per query row:
first the softmax weights and the weighted means kbar and vbar, then the
centred second moment applied to rho.  It never uses the streamed
(O1, O2, tbar) rearrangement that the kernels use; the tests pin the two
against each other.

Readings of the pages adopted here (the pages print no layout or mask rule):
scores are scaled by 1/sqrt(d) and the probe term is not scaled; the causal
mask lets query i see keys j <= i; a decode query at KV length n sees keys
0..n-1; Q, K, V, R are [B, H, N, d] and all heads have their own K and V.
Sliding window (the pages list kernels combining Parallax with sliding-window
sparsity as future work, rainbus.top "未来方向"; they fix no rule): with a
window of W keys, query i sees keys max(0, i - W + 1)..i, and a decode query
at KV length n sees keys max(0, n - W)..n-1.
Block sparsity (the same list; no rule either): a boolean mask over (tile of
128 queries, block of 64 keys) pairs; query i sees key j when j <= i and the
pair (i // 128, j // 64) is active.
"""
from __future__ import annotations

import math

import numpy as np


def parallax_row(q: np.ndarray, rho: np.ndarray, K: np.ndarray, V: np.ndarray) -> np.ndarray:
    """Parallax output for one query over its visible keys.

    q, rho: [d]; K, V: [n, d] (only the keys the query may see, n >= 1).
    Returns float64 [d] = vbar - sum_j p_j (v_j - vbar) ((k_j - kbar) . rho).
    """
    q = np.asarray(q, dtype=np.float64)
    rho = np.asarray(rho, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    d = q.shape[0]
    # Softmax weights over the visible keys.
    s = (K @ q) / math.sqrt(d)
    w = np.exp(s - s.max())
    p = w / w.sum()
    # First pass: weighted means.
    kbar = p @ K
    vbar = p @ V
    # Second pass: centred covariance applied to the probe.
    kc = K - kbar
    vc = V - vbar
    probe = kc @ rho                     # (k_j - kbar) . rho   for every j
    correction = vc.T @ (p * probe)      # Sigma_KV rho
    return vbar - correction


def visible_keys(i: int, N: int, causal: bool, window=None):
    """[lo, hi) of the keys query i sees: j <= i when causal, and j > i - window
    when a window is given (a window implies the causal mask)."""
    if window is not None:
        return max(0, i - int(window) + 1), i + 1
    return 0, (i + 1 if causal else N)


BLOCK_Q, BLOCK_K = 128, 64  # query tile and key block of the block-sparse mask


def sparse_visible_keys(i: int, block_mask) -> np.ndarray:
    """Indices of the keys query i sees under a block mask [tiles, key blocks] (causal)."""
    t = i // BLOCK_Q
    keys = [j for j in range(i + 1) if block_mask[t, j // BLOCK_K]]
    return np.asarray(keys, dtype=np.int64)


def prefill_block_sparse_ref(Q, K, V, R, block_mask, rows=None) -> np.ndarray:
    """Oracle for a block-sparse causal prefill (mask shared by all heads).

    block_mask: bool [ceil(N/128), ceil(N/64)].  Every query must see at least
    one key (the tile's own diagonal block active).  ``rows`` as prefill_ref.
    """
    B, H, N, d = Q.shape
    rows_iter = ([(b, h, i) for b in range(B) for h in range(H) for i in range(N)] if rows is None
                 else list(rows))
    res = []
    for (b, h, i) in rows_iter:
        ks = sparse_visible_keys(i, block_mask)
        res.append(parallax_row(Q[b, h, i], R[b, h, i], K[b, h, ks], V[b, h, ks]))
    if rows is None:
        return np.stack(res).reshape(B, H, N, d)
    return np.stack(res) if res else np.zeros((0, d))


def prefill_ref(Q, K, V, R, causal: bool = True, rows=None, window=None) -> np.ndarray:
    """Oracle for a prefill.

    Q, K, V, R: float64 arrays [B, H, N, d].  ``rows`` is None (every output
    row) or an iterable of (b, h, i) triples; the result is then [len(rows), d]
    in the same order.  ``window`` (None or W >= 1) restricts query i to its
    last W keys (causal).
    """
    B, H, N, d = Q.shape
    if rows is None:
        rows_iter = [(b, h, i) for b in range(B) for h in range(H) for i in range(N)]
    else:
        rows_iter = list(rows)
    res = []
    for (b, h, i) in rows_iter:
        lo, hi = visible_keys(i, N, causal, window)
        res.append(parallax_row(Q[b, h, i], R[b, h, i], K[b, h, lo:hi], V[b, h, lo:hi]))
    if rows is None:
        return np.stack(res).reshape(B, H, N, d)
    return np.stack(res) if res else np.zeros((0, d))


def dilated_visible_keys(i: int, dilation: int, window=None) -> np.ndarray:
    """Indices of the keys query i sees under a dilated window: i, i - r,
    i - 2r, ... (r = dilation), the last ``window`` of them (all when None)."""
    keys = np.arange(i, -1, -int(dilation), dtype=np.int64)[::-1]
    if window is not None:
        keys = keys[-int(window):]
    return keys


def prefill_dilated_ref(Q, K, V, R, dilation: int, window=None, rows=None) -> np.ndarray:
    """Oracle for a dilated causal prefill (the pages list dilated sparsity
    with sliding-window and block-sparse patterns as future work, rainbus.top
    "未来方向", and fix no rule).  Reading: the dilated sliding window, query i
    sees its own key and every r-th key before it, i - k r for k = 0 ..
    window - 1 (all k when window is None).  Q, R [B, H, N, d]; K, V
    [B, Hkv, N, d] (query head h reads KV head h // (H // Hkv)).  ``rows`` as
    prefill_ref."""
    B, H, N, d = Q.shape
    G = H // K.shape[1]
    rows_iter = ([(b, h, i) for b in range(B) for h in range(H) for i in range(N)] if rows is None
                 else list(rows))
    res = []
    for (b, h, i) in rows_iter:
        ks = dilated_visible_keys(i, dilation, window)
        res.append(parallax_row(Q[b, h, i], R[b, h, i], K[b, h // G, ks], V[b, h // G, ks]))
    if rows is None:
        return np.stack(res).reshape(B, H, N, d)
    return np.stack(res) if res else np.zeros((0, d))


def prefill_gqa_ref(Q, K, V, R, causal: bool = True) -> np.ndarray:
    """Oracle for a prefill with grouped KV heads: Q, R [B, H, N, d]; K, V
    [B, Hkv, N, d]; query head h reads KV head h // (H // Hkv)."""
    B, H, N, d = Q.shape
    G = H // K.shape[1]
    out = np.empty((B, H, N, d), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            kv = h // G
            for i in range(N):
                lo, hi = visible_keys(i, N, causal)
                out[b, h, i] = parallax_row(Q[b, h, i], R[b, h, i], K[b, kv, lo:hi], V[b, kv, lo:hi])
    return out


def decode_ref(q, r, Kc, Vc, seqlens, units=None, window=None) -> np.ndarray:
    """Oracle for one decode step.

    q, r: [B, H, d]; Kc, Vc: [B, H, L, d]; seqlens: [B] ints in 1..L.  The
    query of sequence b sits at position seqlens[b]-1 and sees keys
    0..seqlens[b]-1 (with a window W: the last W of them).  ``units`` is None
    (all (b, h)) or a list of (b, h).
    """
    B, H, d = q.shape
    if units is None:
        units = [(b, h) for b in range(B) for h in range(H)]
        full = True
    else:
        full = False
    res = []
    for (b, h) in units:
        n = int(seqlens[b])
        lo = 0 if window is None else max(0, n - int(window))
        res.append(parallax_row(q[b, h], r[b, h], Kc[b, h, lo:n], Vc[b, h, lo:n]))
    out = np.stack(res)
    return out.reshape(B, H, d) if full else out


def decode_gqa_ref(q, r, Kc, Vc, seqlens, units=None) -> np.ndarray:
    """Oracle for one decode step with grouped KV heads.

    q, r: [B, H, d]; Kc, Vc: [B, Hkv, L, d] with H a multiple of Hkv; query
    head h reads KV head h // (H // Hkv) (consecutive query heads share a KV
    head).  The pages name grouping only as the place where packing the q and
    rho rows of many heads into one tensor-core tile pays; each head's output
    is the plain per-query definition over its group's keys.  ``units`` is
    None (all (b, h)) or a list of (b, h) query heads.
    """
    B, H, d = q.shape
    Hkv = Kc.shape[1]
    assert H % Hkv == 0
    G = H // Hkv
    if units is None:
        units = [(b, h) for b in range(B) for h in range(H)]
        full = True
    else:
        full = False
    res = []
    for (b, h) in units:
        n = int(seqlens[b])
        kv = h // G
        res.append(parallax_row(q[b, h], r[b, h], Kc[b, kv, :n], Vc[b, kv, :n]))
    out = np.stack(res)
    return out.reshape(B, H, d) if full else out


def softmax_weights_row(q, K) -> np.ndarray:
    """p_j for one query (exposed for the invariant tests on s_ij)."""
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    s = (K @ q) / math.sqrt(q.shape[0])
    w = np.exp(s - s.max())
    return w / w.sum()
