"""Checks that pin the fp64 oracle to facts other than itself.

Each ``pin_*`` takes an ``oracle.Oracle`` handle and raises ``AssertionError``
on a mismatch.  They are collected by ``test_oracle.py`` (the real oracle must
pass all of them) and by ``test_oracle_mutants.py`` (every planted mistake must
fail at least one of them).

What pins what:
  * ``pin_zero_query``   -- closed form: with q = 0 every visible score is 0, so
    O is the plain mean of the visible V rows and LSE = ln |J_i|.
  * ``pin_single_key``   -- a row that sees exactly one key (causal row 0):
    O equals that V row and LSE equals that one scaled score.
  * ``pin_dominant_key`` -- one key with a score margin >= 40 over every other:
    O equals its V row to within (|J|-1) e^-40 max|V|.
  * ``pin_merge``        -- the mergeable-statistics identity ("FlashAttention-2
    and -3: From Algebra to GPU Scheduling", "Keep the unchanged mathematical
    target in view" and "Another use of mergeable statistics"): two disjoint
    key ranges combined through their LSEs give the full-range result.
  * ``pin_library``      -- PyTorch's scaled_dot_product_attention (fp64, CPU,
    explicit mask, enable_gqa) for O and scipy's logsumexp for LSE.
  * ``pin_bruteforce``   -- an independent pure-Python evaluation with
    math.exp / math.fsum on tiny inputs.
  * ``pin_invariants``   -- O is affine in V, the non-causal result is
    invariant to permuting the keys, and GQA equals explicitly repeated heads.
  * ``pin_window_diagonal`` -- a local window of width (0, 0) leaves each row
    exactly its diagonal key j = i + Nk - Nq: O equals that V row exactly and
    LSE equals the one scaled score (rows whose diagonal lies outside the keys
    get O = 0, LSE = -inf).
  * ``pin_window_limits`` -- windows wider than both sequences reduce to the
    pinned full cases: (wide, wide) is non-causal and (wide, 0) is causal,
    bit for bit.
  * ``pin_window_bruteforce`` -- the pure-Python evaluation with window
    visibility, over left/right widths, causal and Nq != Nk.
  * ``pin_window_merge`` -- a windowed result is the merge of its two key
    halves (the mergeable-statistics identity again, under a window).
"""

from __future__ import annotations

import math

import numpy as np
import scipy.special
import torch

from exact_tiled_attention_29_b200.inputs import bf16_bits

TOL = 1e-12

# (B, Hq, Hkv, Nq, Nk, d, causal): covers GQA, Nq < Nk, Nq > Nk (rows with
# no visible key), a single row, non-causal.
SHAPES = [
    (1, 2, 2, 13, 13, 8, True),
    (2, 4, 2, 9, 17, 16, True),
    (1, 4, 1, 17, 9, 8, True),
    (1, 2, 2, 11, 11, 8, False),
    (2, 4, 2, 7, 19, 4, False),
    (1, 1, 1, 1, 5, 4, True),
]


def _randn_bf16(shape, g, scale=1.0):
    return (torch.randn(shape, generator=g, dtype=torch.float32) * scale).to(torch.bfloat16)


def _make(shape, seed, zero_q=False):
    B, Hq, Hkv, Nq, Nk, d, causal = shape
    g = torch.Generator().manual_seed(seed)
    q = _randn_bf16((B, Nq, Hq, d), g)
    k = _randn_bf16((B, Nk, Hkv, d), g)
    v = _randn_bf16((B, Nk, Hkv, d), g)
    if zero_q:
        q = torch.zeros_like(q)
    return q, k, v


def _visible(i, Nq, Nk, causal, window=(-1, -1)):
    """Key indices visible to row i: the causal rule (bottom-right aligned) and
    a local window [g - left, g + right] around g = i + Nk - Nq, a negative
    width leaving that side open."""
    g = i + Nk - Nq
    out = []
    for j in range(Nk):
        if causal and j > g:
            continue
        if window[0] >= 0 and j < g - window[0]:
            continue
        if window[1] >= 0 and j > g + window[1]:
            continue
        out.append(j)
    return out


def _f64(t):
    return t.to(torch.float64).numpy()


def _close(a, b, tol=TOL, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    same_inf = (np.isinf(a) & np.isinf(b) & (np.sign(a) == np.sign(b)))
    finite = ~same_inf
    assert not np.isnan(a[finite]).any() and not np.isnan(b[finite]).any(), f"{what}: NaN"
    err = np.abs(a[finite] - b[finite])
    m = float(err.max()) if err.size else 0.0
    assert m <= tol, f"{what}: max abs diff {m:g} > {tol:g}"


def _run(orc, q, k, v, causal, scale, **kw):
    return orc.attention(bf16_bits(q), bf16_bits(k), bf16_bits(v), causal, scale, **kw)


def pin_zero_query(orc):
    for n, shape in enumerate(SHAPES):
        B, Hq, Hkv, Nq, Nk, d, causal = shape
        q, k, v = _make(shape, 100 + n, zero_q=True)
        o, lse = _run(orc, q, k, v, causal, 0.37)
        vv = _f64(v)
        r = Hq // Hkv
        for b in range(B):
            for hq in range(Hq):
                for i in range(Nq):
                    vis = _visible(i, Nq, Nk, causal)
                    if not vis:
                        _close(o[b, i, hq], np.zeros(d), what="empty row O")
                        assert lse[b, hq, i] == -math.inf, "empty row LSE"
                        continue
                    _close(o[b, i, hq], vv[b, vis, hq // r].mean(axis=0), what="q=0 mean")
                    _close(lse[b, hq, i], math.log(len(vis)), what="q=0 lse")


def pin_single_key(orc):
    # causal, Nq == Nk: row 0 sees key 0 only; Nq > Nk: row Nq-Nk sees key 0 only.
    for shape in [(2, 4, 2, 16, 16, 8, True), (1, 2, 1, 12, 5, 16, True)]:
        B, Hq, Hkv, Nq, Nk, d, causal = shape
        q, k, v = _make(shape, 7)
        scale = 0.5
        o, lse = _run(orc, q, k, v, True, scale)
        qq, kk, vv = _f64(q), _f64(k), _f64(v)
        i = Nq - Nk if Nq > Nk else 0
        r = Hq // Hkv
        for b in range(B):
            for hq in range(Hq):
                _close(o[b, i, hq], vv[b, 0, hq // r], what="single-key O")
                s = scale * float(np.dot(qq[b, i, hq], kk[b, 0, hq // r]))
                _close(lse[b, hq, i], s, what="single-key LSE")


def pin_dominant_key(orc):
    B, Hq, Hkv, Nq, Nk, d = 1, 2, 1, 8, 24, 8
    g = torch.Generator().manual_seed(11)
    q = torch.zeros((B, Nq, Hq, d))
    q[..., 0] = 1.0                                       # q_i = e_0
    k = torch.randn((B, Nk, Hkv, d), generator=g) * 0.25  # |score| of ordinary keys < ~1.5
    k[..., 0].clamp_(-1.5, 1.5)
    jstar = 5
    k[:, jstar, :, :] = 0.0
    k[:, jstar, :, 0] = 64.0                              # score margin >= 62
    v = torch.randn((B, Nk, Hkv, d), generator=g)
    q, k, v = (t.to(torch.bfloat16) for t in (q, k, v))
    o, lse = _run(orc, q, k, v, False, 1.0)
    vv = _f64(v)
    bound = (Nk - 1) * math.exp(-40.0) * float(np.abs(vv).max()) * 2
    for hq in range(Hq):
        for i in range(Nq):
            _close(o[0, i, hq], vv[0, jstar, 0], tol=bound, what="dominant key O")
            assert abs(lse[0, hq, i] - 64.0) < 1e-3, "dominant key LSE"


def pin_merge(orc):
    for n, shape in enumerate(SHAPES):
        B, Hq, Hkv, Nq, Nk, d, causal = shape
        q, k, v = _make(shape, 300 + n)
        scale = 1.0 / math.sqrt(d)
        o, lse = _run(orc, q, k, v, causal, scale)
        for split in sorted({0, 1, Nk // 2, Nk - 1, Nk}):
            oa, la = _run(orc, q, k, v, causal, scale, k_range=(0, split))
            ob, lb = _run(orc, q, k, v, causal, scale, k_range=(split, Nk))
            lm = np.logaddexp(la, lb)                         # [B,Hq,R]
            with np.errstate(invalid="ignore"):
                wa = np.where(np.isinf(la), 0.0, np.exp(la - lm))
                wb = np.where(np.isinf(lb), 0.0, np.exp(lb - lm))
            wa = np.nan_to_num(wa).transpose(0, 2, 1)[..., None]   # [B,R,Hq,1]
            wb = np.nan_to_num(wb).transpose(0, 2, 1)[..., None]
            om = wa * oa + wb * ob
            _close(om, o, what=f"merge O split={split}")
            _close(lm, lse, what=f"merge LSE split={split}")


def pin_library(orc):
    for n, shape in enumerate(SHAPES):
        B, Hq, Hkv, Nq, Nk, d, causal = shape
        q, k, v = _make(shape, 500 + n)
        scale = 1.0 / math.sqrt(d)
        o, lse = _run(orc, q, k, v, causal, scale)
        mask = torch.ones((Nq, Nk), dtype=torch.bool)
        if causal:
            mask = torch.tensor([[j <= i + Nk - Nq for j in range(Nk)] for i in range(Nq)])
        live = mask.any(dim=1).numpy()
        qt = q.to(torch.float64).permute(0, 2, 1, 3)      # [B,H,N,d]
        kt = k.to(torch.float64).permute(0, 2, 1, 3)
        vt = v.to(torch.float64).permute(0, 2, 1, 3)
        ref = torch.nn.functional.scaled_dot_product_attention(
            qt, kt, vt, attn_mask=mask, scale=scale, enable_gqa=(Hq != Hkv))
        ref = ref.permute(0, 2, 1, 3).numpy()              # [B,Nq,Hq,d]
        _close(o[:, live], ref[:, live], what="SDPA O")
        # the sampled-row path (used at full size) against the same library result
        rows = [i for i in (Nq - 1, 0, Nq // 2) if live[i]]
        if rows:
            o_r, _ = _run(orc, q, k, v, causal, scale, rows=rows)
            _close(o_r, ref[:, rows], what="SDPA O, row subset")
        # LSE: scipy logsumexp of the masked score rows.
        kr = np.repeat(_f64(k), Hq // Hkv, axis=2)           # [B,Nk,Hq,d]
        s = scale * np.einsum("bihc,bjhc->bhij", _f64(q), kr)
        s = np.where(mask.numpy()[None, None], s, -np.inf)
        ref_lse = scipy.special.logsumexp(s, axis=-1)
        _close(lse, ref_lse, what="scipy LSE")


def pin_bruteforce(orc):
    for shape in [(1, 2, 1, 5, 7, 3, True), (1, 1, 1, 4, 6, 4, False), (2, 2, 2, 6, 3, 2, True)]:
        B, Hq, Hkv, Nq, Nk, d, causal = shape
        q, k, v = _make(shape, 900)
        scale = 0.8
        o, lse = _run(orc, q, k, v, causal, scale)
        qq, kk, vv = q.float().tolist(), k.float().tolist(), v.float().tolist()
        r = Hq // Hkv
        for b in range(B):
            for hq in range(Hq):
                for i in range(Nq):
                    vis = _visible(i, Nq, Nk, causal)
                    if not vis:
                        continue
                    sc = [scale * math.fsum(qq[b][i][hq][c] * kk[b][j][hq // r][c] for c in range(d))
                          for j in vis]
                    big = max(sc)
                    w = [math.exp(x - big) for x in sc]
                    tot = math.fsum(w)
                    ref = [math.fsum(w[t] * vv[b][j][hq // r][c] for t, j in enumerate(vis)) / tot
                           for c in range(d)]
                    _close(o[b, i, hq], ref, what="brute-force O")
                    _close(lse[b, hq, i], big + math.log(tot), what="brute-force LSE")


def pin_invariants(orc):
    # Affine in V: O(3V + 5) = 3 O(V) + 5 (V on small integers, exact in bf16).
    shape = (1, 4, 2, 10, 14, 8, True)
    B, Hq, Hkv, Nq, Nk, d, causal = shape
    q, k, _ = _make(shape, 41)
    g = torch.Generator().manual_seed(42)
    vi = torch.randint(-8, 9, (B, Nk, Hkv, d), generator=g).to(torch.bfloat16)
    v2 = (3 * vi.float() + 5).to(torch.bfloat16)
    o1, l1 = _run(orc, q, k, vi, causal, 0.3)
    o2, l2 = _run(orc, q, k, v2, causal, 0.3)
    _close(o2, 3 * o1 + 5, tol=1e-10, what="affine V")
    _close(l2, l1, what="affine V lse")

    # Key permutation invariance (non-causal).
    shape = (2, 2, 2, 6, 12, 8, False)
    q, k, v = _make(shape, 43)
    perm = torch.randperm(12, generator=torch.Generator().manual_seed(44))
    o1, l1 = _run(orc, q, k, v, False, 0.5)
    o2, l2 = _run(orc, q, k[:, perm], v[:, perm], False, 0.5)
    _close(o2, o1, tol=1e-13, what="key permutation O")
    _close(l2, l1, tol=1e-13, what="key permutation LSE")

    # GQA equals the same problem with each KV head repeated for its query group.
    shape = (2, 6, 2, 9, 9, 8, True)
    q, k, v = _make(shape, 45)
    o1, l1 = _run(orc, q, k, v, True, 0.4)
    kr = k.repeat_interleave(3, dim=2)
    vr = v.repeat_interleave(3, dim=2)
    o2, l2 = _run(orc, q, kr, vr, True, 0.4)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2), "GQA != repeated heads"


def pin_window_diagonal(orc):
    for shape in [(1, 2, 1, 9, 9, 8, False), (2, 2, 2, 5, 11, 4, True), (1, 2, 2, 12, 7, 8, False)]:
        B, Hq, Hkv, Nq, Nk, d, causal = shape
        q, k, v = _make(shape, 1000)
        scale = 0.6
        o, lse = _run(orc, q, k, v, causal, scale, window=(0, 0))
        qd, kd, vd = _f64(q), _f64(k), _f64(v)
        r = Hq // Hkv
        for b in range(B):
            for hq in range(Hq):
                for i in range(Nq):
                    g = i + Nk - Nq
                    if not 0 <= g < Nk:
                        assert np.all(o[b, i, hq] == 0) and lse[b, hq, i] == -np.inf
                        continue
                    assert np.array_equal(o[b, i, hq], vd[b, g, hq // r]), "window (0,0): O != V[g]"
                    _close(lse[b, hq, i], scale * float(qd[b, i, hq] @ kd[b, g, hq // r]),
                           what="window (0,0) LSE")


def pin_window_limits(orc):
    for shape in SHAPES:
        B, Hq, Hkv, Nq, Nk, d, causal = shape
        q, k, v = _make(shape, 1100)
        wide = Nq + Nk
        o_full, l_full = _run(orc, q, k, v, False, 0.5)
        o_w, l_w = _run(orc, q, k, v, False, 0.5, window=(wide, wide))
        assert np.array_equal(o_full, o_w) and np.array_equal(l_full, l_w), "wide window != full"
        o_c, l_c = _run(orc, q, k, v, True, 0.5)
        o_w, l_w = _run(orc, q, k, v, False, 0.5, window=(wide, 0))
        assert np.array_equal(o_c, o_w) and np.array_equal(l_c, l_w), "(wide, 0) window != causal"


def pin_window_bruteforce(orc):
    cases = [((1, 2, 1, 9, 9, 4, True), (2, -1)), ((1, 2, 2, 7, 10, 3, False), (1, 2)),
             ((2, 2, 1, 10, 6, 4, True), (3, -1)), ((1, 1, 1, 8, 8, 2, False), (-1, 1)),
             ((1, 2, 2, 6, 9, 4, True), (0, -1))]
    for shape, window in cases:
        B, Hq, Hkv, Nq, Nk, d, causal = shape
        q, k, v = _make(shape, 1200)
        scale = 0.7
        o, lse = _run(orc, q, k, v, causal, scale, window=window)
        qq, kk, vv = q.float().tolist(), k.float().tolist(), v.float().tolist()
        r = Hq // Hkv
        for b in range(B):
            for hq in range(Hq):
                for i in range(Nq):
                    vis = _visible(i, Nq, Nk, causal, window)
                    if not vis:
                        assert np.all(o[b, i, hq] == 0) and lse[b, hq, i] == -np.inf
                        continue
                    sc = [scale * math.fsum(qq[b][i][hq][c] * kk[b][j][hq // r][c] for c in range(d))
                          for j in vis]
                    big = max(sc)
                    w = [math.exp(x - big) for x in sc]
                    tot = math.fsum(w)
                    ref = [math.fsum(w[t] * vv[b][j][hq // r][c] for t, j in enumerate(vis)) / tot
                           for c in range(d)]
                    _close(o[b, i, hq], ref, what=f"window {window} brute-force O")
                    _close(lse[b, hq, i], big + math.log(tot), what=f"window {window} brute-force LSE")


def pin_window_merge(orc):
    shape = (2, 4, 2, 12, 16, 8, True)
    B, Hq, Hkv, Nq, Nk, d, causal = shape
    q, k, v = _make(shape, 1300)
    for window in [(3, -1), (5, 2), (-1, 0)]:
        o, lse = _run(orc, q, k, v, causal, 0.45, window=window)
        oa, la = _run(orc, q, k, v, causal, 0.45, k_range=(0, 8), window=window)
        ob, lb = _run(orc, q, k, v, causal, 0.45, k_range=(8, Nk), window=window)
        m = np.maximum(la, lb)
        safe = np.where(np.isfinite(m), m, 0.0)
        tot = np.exp(la - safe) + np.exp(lb - safe)
        l_ref = np.where(np.isfinite(m), safe + np.log(np.where(tot > 0, tot, 1.0)), -np.inf)
        _close(lse, l_ref, what=f"window {window} merged LSE")
        wa = np.where(np.isfinite(la), np.exp(la - np.where(np.isfinite(l_ref), l_ref, 0.0)), 0.0)
        wb = np.where(np.isfinite(lb), np.exp(lb - np.where(np.isfinite(l_ref), l_ref, 0.0)), 0.0)
        o_ref = (np.transpose(wa, (0, 2, 1))[..., None] * oa + np.transpose(wb, (0, 2, 1))[..., None] * ob)
        _close(o, o_ref, tol=1e-11, what=f"window {window} merged O")


ALL_PINS = [pin_zero_query, pin_single_key, pin_dominant_key, pin_merge, pin_library,
            pin_bruteforce, pin_invariants, pin_window_diagonal, pin_window_limits,
            pin_window_bruteforce, pin_window_merge]


# ---------------------------------------------------------------------------
# Backward pass (gradients), pinned to calculus and to a library:
#   * ``pin_bwd_finite_difference`` -- central differences of the scalar
#     L = sum(G * O) of a plain fp64 forward (numpy, masked softmax) agree with
#     the oracle's dQ, dK, dV at sampled elements.
#   * ``pin_bwd_autograd`` -- torch autograd through scaled_dot_product_attention
#     in fp64 (explicit mask, enable_gqa).
#   * ``pin_bwd_single_key`` -- window (0, 0): every row sees one key, P = 1,
#     so dS = 0 (dQ = dK = 0 exactly) and dV_j is the plain sum of the dO rows
#     whose diagonal key is j.
#   * ``pin_bwd_gqa`` -- GQA equals the repeated-head problem with dK, dV summed
#     over each group.
# ---------------------------------------------------------------------------

def _run_bwd(orc, q, k, v, g, causal, scale, **kw):
    return orc.backward(bf16_bits(q), bf16_bits(k), bf16_bits(v), bf16_bits(g), causal, scale, **kw)


def _forward_np(q, k, v, causal, scale, window=(-1, -1)):
    """Plain masked-softmax attention in fp64 numpy ([B,N,H,d] layouts)."""
    B, Nq, Hq, d = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    r = Hq // Hkv
    o = np.zeros_like(q)
    for b in range(B):
        for h in range(Hq):
            s = scale * q[b, :, h] @ k[b, :, h // r].T
            for i in range(Nq):
                vis = _visible(i, Nq, Nk, causal, window)
                mask = np.full(Nk, -np.inf)
                mask[vis] = 0.0
                row = s[i] + mask
                if not vis:
                    continue
                w = np.exp(row - row.max())
                o[b, i, h] = (w / w.sum()) @ v[b, :, h // r]
    return o


def pin_bwd_finite_difference(orc):
    for shape, window in [((1, 2, 1, 7, 9, 4, True), (-1, -1)), ((1, 2, 2, 6, 6, 3, False), (2, 1))]:
        B, Hq, Hkv, Nq, Nk, d, causal = shape
        q, k, v = _make(shape, 2000)
        g = _randn_bf16((B, Nq, Hq, d), torch.Generator().manual_seed(2001))
        scale = 0.55
        dq, dk, dv = _run_bwd(orc, q, k, v, g, causal, scale, window=window)
        qd, kd, vd, gd = _f64(q), _f64(k), _f64(v), _f64(g)
        loss = lambda qq, kk, vv: float((gd * _forward_np(qq, kk, vv, causal, scale, window)).sum())
        eps = 1e-5
        rng = np.random.default_rng(2002)
        for name, base, grad in (("dQ", qd, dq), ("dK", kd, dk), ("dV", vd, dv)):
            for _ in range(12):
                idx = tuple(int(rng.integers(n)) for n in base.shape)
                args_p = [qd.copy(), kd.copy(), vd.copy()]
                args_m = [qd.copy(), kd.copy(), vd.copy()]
                which = "QKV".index(name[1])
                args_p[which][idx] += eps
                args_m[which][idx] -= eps
                fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
                assert abs(fd - grad[idx]) <= 1e-7 * max(1.0, abs(fd)), \
                    f"{name}{idx}: finite difference {fd} vs oracle {grad[idx]}"


def pin_bwd_autograd(orc):
    for shape in [(2, 4, 2, 9, 17, 8, True), (1, 2, 2, 11, 11, 8, False), (1, 4, 1, 17, 9, 8, True)]:
        B, Hq, Hkv, Nq, Nk, d, causal = shape
        q, k, v = _make(shape, 2100)
        g = _randn_bf16((B, Nq, Hq, d), torch.Generator().manual_seed(2101))
        scale = 0.4
        dq, dk, dv = _run_bwd(orc, q, k, v, g, causal, scale)
        qt = q.double().permute(0, 2, 1, 3).requires_grad_(True)
        kt = k.double().permute(0, 2, 1, 3).requires_grad_(True)
        vt = v.double().permute(0, 2, 1, 3).requires_grad_(True)
        mask = torch.ones(Nq, Nk, dtype=torch.bool)
        if causal:
            mask = torch.tensor([[j <= i + Nk - Nq for j in range(Nk)] for i in range(Nq)])
        out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale,
                                                               enable_gqa=True)
        # rows with no visible key: the oracle's convention (O = 0) has zero gradient
        keep = mask.any(dim=1)
        out = torch.where(keep[None, None, :, None], out, torch.zeros_like(out))
        out.backward(g.double().permute(0, 2, 1, 3))
        _close(dq, qt.grad.permute(0, 2, 1, 3).numpy(), tol=1e-11, what="autograd dQ")
        _close(dk, kt.grad.permute(0, 2, 1, 3).numpy(), tol=1e-11, what="autograd dK")
        _close(dv, vt.grad.permute(0, 2, 1, 3).numpy(), tol=1e-11, what="autograd dV")


def pin_bwd_single_key(orc):
    shape = (2, 4, 2, 9, 12, 8, False)
    B, Hq, Hkv, Nq, Nk, d, causal = shape
    q, k, v = _make(shape, 2200)
    g = _randn_bf16((B, Nq, Hq, d), torch.Generator().manual_seed(2201))
    dq, dk, dv = _run_bwd(orc, q, k, v, g, False, 0.9, window=(0, 0))
    assert np.all(dq == 0) and np.all(dk == 0), "one visible key: dS must vanish"
    gd = _f64(g)
    ref = np.zeros_like(dv)
    r = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            for i in range(Nq):
                ref[b, i + Nk - Nq, h // r] += gd[b, i, h]
    _close(dv, ref, what="one visible key: dV = sum of dO rows")


def pin_bwd_gqa(orc):
    shape = (2, 6, 2, 9, 11, 8, True)
    B, Hq, Hkv, Nq, Nk, d, causal = shape
    q, k, v = _make(shape, 2300)
    g = _randn_bf16((B, Nq, Hq, d), torch.Generator().manual_seed(2301))
    dq1, dk1, dv1 = _run_bwd(orc, q, k, v, g, True, 0.5)
    r = Hq // Hkv
    dq2, dk2, dv2 = _run_bwd(orc, q, k.repeat_interleave(r, dim=2), v.repeat_interleave(r, dim=2), g, True, 0.5)
    _close(dq1, dq2, tol=1e-13, what="GQA dQ")
    _close(dk1, dk2.reshape(B, Nk, Hkv, r, d).sum(axis=3), tol=1e-13, what="GQA dK")
    _close(dv1, dv2.reshape(B, Nk, Hkv, r, d).sum(axis=3), tol=1e-13, what="GQA dV")


BWD_PINS = [pin_bwd_finite_difference, pin_bwd_autograd, pin_bwd_single_key, pin_bwd_gqa]
