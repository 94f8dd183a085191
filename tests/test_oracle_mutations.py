"""Planted mistakes in copies of the oracle must each fail at least one pin.

The mistakes are planted here, on the CPU, in the oracle's arithmetic (never in
the CUDA path).  If a plausible slip (dropped scale, shifted mask, transposed
operand, wrong sign, dropped term) passed every check, the checks would not be
pinning the oracle.
"""
import numpy as np
import pytest

import oracle
import oracle_checks as oc


def _fwd_generic(q, k, v, scale, causal, *, mask_strict=False, use_scale=True, lse_no_max=False,
                 transpose=False, axis=-1, v_shift=False):
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    s = (k @ np.swapaxes(q, -1, -2)) if transpose else (q @ np.swapaxes(k, -1, -2))
    if use_scale:
        s = s * scale
    N, Nk = s.shape[-2], s.shape[-1]
    if causal:
        j, i = np.meshgrid(np.arange(Nk), np.arange(N))
        bad = (j >= i) & (j != 0) if mask_strict else (j > i)
        s = np.where(bad, -np.inf, s)
    m = s.max(axis=axis, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=axis, keepdims=True)
    p = e / l
    vv = np.roll(v, 1, axis=-2) if v_shift else v
    o = p @ vv
    lse = (np.log(l) if lse_no_max else m + np.log(l))
    lse = lse[..., 0] if axis == -1 else np.broadcast_to(lse, s.shape)[..., 0]
    return o, lse


MUTANTS_FWD = {
    "dropped_scale": dict(use_scale=False),
    "mask_excludes_diagonal": dict(mask_strict=True),
    "lse_without_max": dict(lse_no_max=True),
    "transposed_scores": dict(transpose=True),
    "softmax_wrong_axis": dict(axis=-2),
    "v_rows_shifted": dict(v_shift=True),
}


def test_unmutated_generic_passes():
    f = lambda q, k, v, s, c: _fwd_generic(q, k, v, s, c)
    for chk in oc.FWD_CHECKS:
        assert chk(f), chk.__name__


@pytest.mark.parametrize("name", sorted(MUTANTS_FWD))
def test_forward_mutant_is_caught(name):
    kw = MUTANTS_FWD[name]
    f = lambda q, k, v, s, c: _fwd_generic(q, k, v, s, c, **kw)
    failures = []
    for chk in oc.FWD_CHECKS:
        try:
            ok = chk(f)
        except Exception:
            ok = False
        if not ok:
            failures.append(chk.__name__)
    assert failures, f"mutant {name} passed every forward check"


def _bwd_generic(q, k, v, do, scale, causal, *, dk_unscaled=False, ds_sign=1.0, drop_D=False,
                 dv_transposed=False):
    q, k, v, do = (np.asarray(x, dtype=np.float64) for x in (q, k, v, do))
    s = (q @ np.swapaxes(k, -1, -2)) * scale
    N = s.shape[-1]
    if causal:
        s = np.where(np.triu(np.ones((N, N), bool), 1), -np.inf, s)
    e = np.exp(s - s.max(-1, keepdims=True))
    p = e / e.sum(-1, keepdims=True)
    pt = np.swapaxes(p, -1, -2)
    dv = (p @ do) if dv_transposed else (pt @ do)
    dp = do @ np.swapaxes(v, -1, -2)
    D = 0.0 if drop_D else (p * dp).sum(-1, keepdims=True)
    ds = ds_sign * p * (dp - D)
    dq = scale * ds @ k
    dk = (1.0 if dk_unscaled else scale) * np.swapaxes(ds, -1, -2) @ q
    return dq, dk, dv


MUTANTS_BWD = {
    "dk_missing_scale": dict(dk_unscaled=True),
    "ds_sign_flipped": dict(ds_sign=-1.0),
    "D_term_dropped": dict(drop_D=True),
    "dv_uses_P_not_PT": dict(dv_transposed=True),
}


def test_unmutated_generic_bwd_passes():
    f = lambda *a: _bwd_generic(*a)
    for chk in oc.BWD_CHECKS:
        assert chk(f), chk.__name__


@pytest.mark.parametrize("name", sorted(MUTANTS_BWD))
def test_backward_mutant_is_caught(name):
    kw = MUTANTS_BWD[name]
    f = lambda *a: _bwd_generic(*a, **kw)
    failures = []
    for chk in oc.BWD_CHECKS:
        try:
            ok = chk(f)
        except Exception:
            ok = False
        if not ok:
            failures.append(chk.__name__)
    assert failures, f"mutant {name} passed every backward check"


# ----------------------------------------------------------------------------- decoding
def _dec_generic(q, k, v, scale, causal, *, head_mod=False, offset=0, top_left=False,
                 use_scale=True, lse_no_max=False):
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    B, Hq, Nq, _ = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    g = Hq // Hkv
    O = np.empty((B, Hq, Nq, v.shape[3]))
    L = np.empty((B, Hq, Nq))
    for b in range(B):
        for h in range(Hq):
            kh = h % Hkv if head_mod else h // g
            s = q[b, h] @ k[b, kh].T
            if use_scale:
                s = s * scale
            if causal:
                i = np.arange(Nq)[:, None]
                j = np.arange(Nk)[None, :]
                last = i if top_left else i + (Nk - Nq) + offset
                s = np.where(j > last, -np.inf, s)
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            l = e.sum(axis=1, keepdims=True)
            O[b, h] = (e / l) @ v[b, kh]
            L[b, h] = (np.log(l) if lse_no_max else m + np.log(l))[:, 0]
    return O, L


MUTANTS_DEC = {
    "kv_head_modulo": dict(head_mod=True),
    "mask_from_start": dict(top_left=True),
    "mask_one_key_short": dict(offset=-1),
    "mask_one_key_long": dict(offset=1),
    "dropped_scale": dict(use_scale=False),
    "lse_without_max": dict(lse_no_max=True),
}


def test_unmutated_decode_passes():
    for chk in oc.DEC_CHECKS:
        assert chk(_dec_generic), chk.__name__


# a mutant that masks every key of a row produces NaN rows on purpose
@pytest.mark.filterwarnings("ignore:invalid value encountered:RuntimeWarning")
@pytest.mark.parametrize("name", sorted(MUTANTS_DEC))
def test_decode_mutant_is_caught(name):
    kw = MUTANTS_DEC[name]
    f = lambda q, k, v, s, c: _dec_generic(q, k, v, s, c, **kw)
    failures = []
    for chk in oc.DEC_CHECKS:
        try:
            ok = chk(f)
        except Exception:
            ok = False
        if not ok:
            failures.append(chk.__name__)
    assert failures, f"mutant {name} passed every decoding check"


# ----------------------------------------------------------------------------- grouped-head backward
def _gqa_bwd_generic(q, k, v, do, scale, causal, *, last_only=False, head_mod=False):
    q, k, v, do = (np.asarray(x, dtype=np.float64) for x in (q, k, v, do))
    B, Hq = q.shape[:2]
    Hkv = k.shape[1]
    g = Hq // Hkv
    dq = np.empty_like(q)
    dk, dv = np.zeros_like(k), np.zeros_like(v)
    for b in range(B):
        for h in range(Hq):
            hk = h % Hkv if head_mod else h // g
            a, bk, bv = oracle.attention_bwd(q[b:b + 1, h:h + 1], k[b:b + 1, hk:hk + 1],
                                             v[b:b + 1, hk:hk + 1], do[b:b + 1, h:h + 1], scale, causal)
            dq[b, h] = a[0, 0]
            if last_only:
                dk[b, hk], dv[b, hk] = bk[0, 0], bv[0, 0]
            else:
                dk[b, hk] += bk[0, 0]
                dv[b, hk] += bv[0, 0]
    return dq, dk, dv


MUTANTS_GQA_BWD = {"shared_grad_not_summed": dict(last_only=True), "kv_head_modulo": dict(head_mod=True)}


def test_unmutated_gqa_backward_passes():
    for chk in oc.GQA_BWD_CHECKS:
        assert chk(_gqa_bwd_generic), chk.__name__


@pytest.mark.parametrize("name", sorted(MUTANTS_GQA_BWD))
def test_gqa_backward_mutant_is_caught(name):
    kw = MUTANTS_GQA_BWD[name]
    f = lambda q, k, v, do, s, c: _gqa_bwd_generic(q, k, v, do, s, c, **kw)
    assert not all(chk(f) for chk in oc.GQA_BWD_CHECKS), f"mutant {name} passed every check"


def _probs_generic(q, k, scale, causal, *, transpose=False, axis=-1, use_scale=True):
    q, k = (np.asarray(x, dtype=np.float64) for x in (q, k))
    s = (k @ np.swapaxes(q, -1, -2)) if transpose else (q @ np.swapaxes(k, -1, -2))
    if use_scale:
        s = s * scale
    if causal:
        N = s.shape[-1]
        s = np.where(np.triu(np.ones((N, N), bool), 1), -np.inf, s)
    e = np.exp(s - s.max(axis=axis, keepdims=True))
    return e / e.sum(axis=axis, keepdims=True)


def test_unmutated_probs_pass():
    for chk in oc.PROBS_CHECKS:
        assert chk(lambda q, k, s, c: _probs_generic(q, k, s, c)), chk.__name__


@pytest.mark.parametrize("kw", [dict(transpose=True), dict(axis=-2), dict(use_scale=False)],
                         ids=["transposed_scores", "wrong_axis", "dropped_scale"])
def test_probs_mutant_is_caught(kw):
    f = lambda q, k, s, c: _probs_generic(q, k, s, c, **kw)
    failures = []
    for chk in oc.PROBS_CHECKS:
        try:
            ok = chk(f)
        except Exception:
            ok = False
        if not ok:
            failures.append(chk.__name__)
    assert failures, f"softmax_probs mutant {kw} passed every check"
