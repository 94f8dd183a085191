"""fp64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import this module.  The
CUDA library never calls it and it never calls the CUDA library: the two share
no code.

What it computes is the plain definition, written out with the full N x N score
matrix materialised (the very matrix the fused kernels never write to HBM):

    Attention(Q, K, V) = softmax(Q K^T * scale) V,   scale = 1/sqrt(d_k)

-- "FlashAttention — フラッシュアテンション" (systems-analysis.info wiki),
section 標準的なアテンションの問題点, the displayed formula.  The pages state the
fused method reaches this same result up to floating-point rounding
("FlashAttentionとは？…" (issoh.co.jp), section 最大値と正規化項を持ち回るオンライン
softmaxの再スケール; wiki, section オンラインSoftmax計算), so the definition is
the oracle.

Readings of points the pages leave open:

* causal = lower triangular, key j visible to query i iff j <= i (the pages say
  only "lower-triangular mask", mypcrig.com post, section "FA2 の改善").
* masked scores are -inf; a fully masked row cannot occur for N_q == N_k.
* the saved "normalisation statistics" (issoh.co.jp, section 逆伝播でL×L行列を
  保存せず再計算する設計) are the natural-log row logsumexp
  LSE_i = ln sum_j exp(scale * q_i . k_j) over visible j.
* the backward is the chain rule of L = sum(O * dO) through the materialised P
  (the pages give only the recompute idea):
      dV = P^T dO,  dP = dO V^T,  D_i = sum_j P_ij dP_ij,
      dS = P * (dP - D),  dQ = scale dS K,  dK = scale dS^T Q.

Every function takes array-likes (numpy or torch CPU tensors of any float
dtype) and converts them to float64 first.
"""
from __future__ import annotations

import numpy as np

ROW_BLOCK = 4096   # rows of S materialised at once for very long heads


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().cpu()
        if str(x.dtype).startswith("torch.float8") or str(x.dtype) == "torch.bfloat16":
            x = x.double()
        x = x.numpy()
    return np.asarray(x, dtype=np.float64)


def _scores(q2: np.ndarray, k2: np.ndarray, scale: float, causal: bool, row0: int) -> np.ndarray:
    """S = scale * Q K^T for rows row0..row0+len(q2)-1, causal entries j > i set to -inf."""
    s = (q2 @ k2.T) * scale
    if causal:
        rows = np.arange(row0, row0 + q2.shape[0])[:, None]
        cols = np.arange(k2.shape[0])[None, :]
        s = np.where(cols > rows, -np.inf, s)
    return s


def softmax_probs(q, k, scale: float, causal: bool) -> np.ndarray:
    """P = softmax(scale Q K^T) [B,H,N,N] by the two-pass definition (small shapes only)."""
    q, k = _f64(q), _f64(k)
    B, H, N, _ = q.shape
    P = np.empty((B, H, N, k.shape[2]))
    for b in range(B):
        for h in range(H):
            s = _scores(q[b, h], k[b, h], scale, causal, 0)
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            P[b, h] = e / e.sum(axis=1, keepdims=True)
    return P


def _head_fwd(q2, k2, v2, scale, causal, rows=None):
    """Forward of one head: returns (O rows, LSE rows) for the requested rows (default all)."""
    N = q2.shape[0]
    if rows is None:
        rows = np.arange(N)
    rows = np.asarray(rows)
    o = np.empty((len(rows), v2.shape[1]))
    lse = np.empty(len(rows))
    for i0 in range(0, len(rows), ROW_BLOCK):
        r = rows[i0:i0 + ROW_BLOCK]
        s = (q2[r] @ k2.T) * scale
        if causal:
            s = np.where(np.arange(k2.shape[0])[None, :] > r[:, None], -np.inf, s)
        m = s.max(axis=1, keepdims=True)           # pass 1: row max
        e = np.exp(s - m)                           # pass 2: exponentials and sum
        l = e.sum(axis=1, keepdims=True)
        o[i0:i0 + len(r)] = (e / l) @ v2
        lse[i0:i0 + len(r)] = (m + np.log(l))[:, 0]
    return o, lse


def attention_fwd(q, k, v, scale: float, causal: bool):
    """O [B,H,N,d] and LSE [B,H,N] in fp64 by the two-pass softmax definition."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, _ = q.shape
    o = np.empty((B, H, N, v.shape[3]))
    lse = np.empty((B, H, N))
    for b in range(B):
        for h in range(H):
            o[b, h], lse[b, h] = _head_fwd(q[b, h], k[b, h], v[b, h], scale, causal)
    return o, lse


def attention_fwd_rows(q, k, v, scale: float, causal: bool, picks):
    """O and LSE for selected (b, h, row) triples only; each row still sees its full key set.

    ``picks`` is an int array of shape [P, 3].  Used for full-size workloads
    where computing every row in fp64 would take too long on the host.
    """
    picks = np.asarray(picks)
    d_v = v.shape[3]
    o = np.empty((len(picks), d_v))
    lse = np.empty(len(picks))
    for (b, h) in sorted(set(map(tuple, picks[:, :2].tolist()))):
        sel = np.nonzero((picks[:, 0] == b) & (picks[:, 1] == h))[0]
        rows = picks[sel, 2]
        q2 = _f64(q[b, h][rows])
        k2 = _f64(k[b, h])
        v2 = _f64(v[b, h])
        s = (q2 @ k2.T) * scale
        if causal:
            s = np.where(np.arange(k2.shape[0])[None, :] > rows[:, None], -np.inf, s)
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        l = e.sum(axis=1, keepdims=True)
        o[sel] = (e / l) @ v2
        lse[sel] = (m + np.log(l))[:, 0]
    return o, lse


def _head_bwd(q2, k2, v2, do2, scale, causal):
    """Backward of one head from the materialised P (no use of a saved LSE)."""
    N = q2.shape[0]
    dq = np.empty_like(q2)
    dk = np.zeros_like(k2)
    dv = np.zeros_like(v2)
    for i0 in range(0, N, ROW_BLOCK):
        r = np.arange(i0, min(N, i0 + ROW_BLOCK))
        s = (q2[r] @ k2.T) * scale
        if causal:
            s = np.where(np.arange(k2.shape[0])[None, :] > r[:, None], -np.inf, s)
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        p = e / e.sum(axis=1, keepdims=True)        # P rows for this block
        dov = do2[r]
        dv += p.T @ dov                             # dV = P^T dO
        dp = dov @ v2.T                             # dP = dO V^T
        D = (p * dp).sum(axis=1, keepdims=True)     # D_i = sum_j P_ij dP_ij
        ds = p * (dp - D)                           # dS = P * (dP - D)
        dq[r] = scale * (ds @ k2)                   # dQ = scale dS K
        dk += scale * (ds.T @ q2[r])                # dK = scale dS^T Q
    return dq, dk, dv


def attention_bwd(q, k, v, do, scale: float, causal: bool, heads=None):
    """dQ, dK, dV in fp64 for L = sum(O * dO) (chain rule through the materialised P).

    ``heads`` optionally restricts the work to a list of (b, h) pairs; the
    returned arrays then have shape [len(heads), N, d].
    """
    if heads is None:
        q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
        B, H = q.shape[:2]
        dq, dk, dv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
        for b in range(B):
            for h in range(H):
                dq[b, h], dk[b, h], dv[b, h] = _head_bwd(q[b, h], k[b, h], v[b, h], do[b, h],
                                                         scale, causal)
        return dq, dk, dv
    out = [_head_bwd(_f64(q[b, h]), _f64(k[b, h]), _f64(v[b, h]), _f64(do[b, h]), scale, causal)
           for b, h in heads]
    return tuple(np.stack([o[i] for o in out]) for i in range(3))


def attention_fwd_heads(q, k, v, scale: float, causal: bool, heads):
    """Forward for a list of (b, h) pairs; returns O [P,N,d], LSE [P,N]."""
    outs = [_head_fwd(_f64(q[b, h]), _f64(k[b, h]), _f64(v[b, h]), scale, causal) for b, h in heads]
    return np.stack([o for o, _ in outs]), np.stack([l for _, l in outs])


def attention_fwd_online(q, k, v, scale: float, causal: bool, block_sizes):
    """Blocked single-pass (online) softmax in fp64: a second, independent forward.

    Keys are visited in consecutive blocks of the given sizes (cycled).  For
    every row the running max m and running sum l are carried; when a block
    raises m, the accumulated output and l are rescaled by exp(m_old - m_new)
    before the block is added (issoh.co.jp, section 最大値と正規化項を持ち回る
    オンラインsoftmaxの再スケール; wiki, section オンラインSoftmax計算).
    Returns O and LSE like ``attention_fwd``.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, _ = q.shape
    Nk = k.shape[2]
    o = np.empty((B, H, N, v.shape[3]))
    lse = np.empty((B, H, N))
    for b in range(B):
        for h in range(H):
            m = np.full((N, 1), -np.inf)
            l = np.zeros((N, 1))
            acc = np.zeros((N, v.shape[3]))
            j0, bi = 0, 0
            rows = np.arange(N)[:, None]
            while j0 < Nk:
                bs = int(block_sizes[bi % len(block_sizes)])
                bi += 1
                j1 = min(Nk, j0 + bs)
                s = (q[b, h] @ k[b, h, j0:j1].T) * scale
                if causal:
                    s = np.where(np.arange(j0, j1)[None, :] > rows, -np.inf, s)
                m_new = np.maximum(m, s.max(axis=1, keepdims=True))
                m_safe = np.where(np.isfinite(m_new), m_new, 0.0)
                alpha = np.exp(m - m_safe)          # exp(-inf) = 0 on the first visible block
                p = np.exp(s - m_safe)
                l = l * alpha + p.sum(axis=1, keepdims=True)
                acc = acc * alpha + p @ v[b, h, j0:j1]
                m = m_new
                j0 = j1
            o[b, h] = acc / l
            lse[b, h] = (m + np.log(l))[:, 0]
    return o, lse


def attention_bwd_rows_dq(q, k, v, do, scale: float, causal: bool, picks):
    """dQ rows for selected (b, h, i): row i of dQ needs only row i of P and dP.

    D_i = sum_j P_ij dP_ij is formed from the row's own P and dP, so each
    picked row costs O(N d) and still sees its full key set.
    """
    picks = np.asarray(picks)
    out = np.empty((len(picks), q.shape[3]))
    for n, (b, h, i) in enumerate(picks.tolist()):
        q2 = _f64(q[b, h, i:i + 1])
        k2 = _f64(k[b, h])
        v2 = _f64(v[b, h])
        do2 = _f64(do[b, h, i:i + 1])
        s = (q2 @ k2.T) * scale
        if causal:
            s = np.where(np.arange(k2.shape[0])[None, :] > i, -np.inf, s)
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        p = e / e.sum(axis=1, keepdims=True)
        dp = do2 @ v2.T
        D = (p * dp).sum(axis=1, keepdims=True)
        out[n] = (scale * ((p * (dp - D)) @ k2))[0]
    return out


def attention_decode(q, k, v, scale: float, causal: bool):
    """Few queries against a long key/value sequence with grouped heads, by definition.

    q [B, Hq, Nq, d]; k, v [B, Hkv, Nk, d] with Hq = g * Hkv; query head h reads
    key/value head h // g (the GQA / MQA sharing of "FlashAttention —
    フラッシュアテンション" (systems-analysis.info), section FlashAttention-2（2023年）).
    Causal reading: the Nq queries are the last Nq positions of the Nk-long sequence
    (decoding with a KV cache, "FlashAttentionとは？…" (issoh.co.jp), section
    短い系列の効果とデコード向け最適化の違い), so query i sees keys j <= Nk - Nq + i; for
    Nq == Nk this is the lower-triangular mask of attention_fwd.
    Returns (O [B, Hq, Nq, d], LSE [B, Hq, Nq]) in fp64: the full Nq x Nk score
    matrix, two-pass softmax, O = P V, LSE = m + ln(sum exp(S - m)).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    g = Hq // Hkv
    O = np.empty((B, Hq, Nq, v.shape[3]))
    L = np.empty((B, Hq, Nq))
    last = np.arange(Nq)[:, None] + (Nk - Nq)          # last visible key of each query
    cols = np.arange(Nk)[None, :]
    for b in range(B):
        for h in range(Hq):
            s = (q[b, h] @ k[b, h // g].T) * scale
            if causal:
                s = np.where(cols > last, -np.inf, s)
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            l = e.sum(axis=1, keepdims=True)
            O[b, h] = (e / l) @ v[b, h // g]
            L[b, h] = (m + np.log(l))[:, 0]
    return O, L


def attention_bwd_gqa(q, k, v, do, scale: float, causal: bool):
    """dQ, dK, dV in fp64 with grouped heads: q, do [B, Hq, N, d]; k, v [B, Hkv, N, d].

    Query head h attends through key/value head h // g (g = Hq / Hkv; "FlashAttention —
    フラッシュアテンション" (systems-analysis.info), section FlashAttention-2（2023年）).
    A shared K/V head is used by g attention computations, so by the chain rule its
    gradient is the sum of the g per-use gradients; each use is the one-head backward
    above (materialised P, no saved LSE).
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, Hq = q.shape[:2]
    Hkv = k.shape[1]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    g = Hq // Hkv
    dq = np.empty_like(q)
    dk, dv = np.zeros_like(k), np.zeros_like(v)
    for b in range(B):
        for h in range(Hq):
            hk = h // g
            dq[b, h], dkh, dvh = _head_bwd(q[b, h], k[b, hk], v[b, hk], do[b, h], scale, causal)
            dk[b, hk] += dkh
            dv[b, hk] += dvh
    return dq, dk, dv
