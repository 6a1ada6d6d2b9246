"""Pins for the float64 oracle: checks against things other than the oracle.

Each pin takes an oracle object and returns None when it holds or a string
describing the violation.  The same functions run against the real oracle
(every one must hold) and against deliberately broken builds of it (each
broken build must violate at least one), which shows that a plausible
mistake -- a dropped mask, a dropped scale, a wrong head->group map, a wrong
pooling divisor, a reversed tie-break, a lost window token, a residual not
passed on, a codeword tie to the wrong index -- cannot hide.

Sources the pins come from (none of them is the oracle's own code):
  * closed form: with K = 0 every visible logit is 0, so each window row is
    uniform over the keys it may see;
  * a library attention routine: torch's scaled_dot_product_attention in
    float64 with V = identity returns the attention probabilities (with the
    rows' normalisers given, scipy's logsumexp supplies them);
  * arbitrary-precision brute force (mpmath) on tiny inputs;
  * the total mass invariant sum_j A[g, j] = w * G;
  * scipy's zero-padded uniform filter for the pooling;
  * the defining order property of a top-k with the lower-position tie-break;
  * closed forms of entropy / top-1% mass / variance for uniform and one-hot
    distributions, and scipy.stats.entropy / numpy.var.
"""
from __future__ import annotations

import math

import numpy as np

from workloads import f32_to_bf16_bits


def _bf16(x):
    return f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def _rand_qk(rng, N, H, Hkv, d, w, qscale=1.0, kscale=1.0):
    q = _bf16(rng.standard_normal((w, H, d)) * qscale)
    k = _bf16(rng.standard_normal((N, Hkv, d)) * kscale)
    return q, k


def _widen(b):
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------- #
# scores
# --------------------------------------------------------------------------- #
def closed_form_zero_keys(N, H, Hkv, w):
    """A for K = 0: row i is uniform over its p_i + 1 visible keys."""
    G = H // Hkv
    p = N - w + np.arange(w)          # last visible key of each window row
    A = np.zeros(N)
    for i in range(w):
        A[: p[i] + 1] += 1.0 / (p[i] + 1)
    return np.tile(G * A, (Hkv, 1))


def pin_zero_keys(orc):
    rng = np.random.default_rng(7)
    for (N, H, Hkv, d, w) in [(40, 4, 2, 64, 6), (33, 6, 3, 128, 33), (17, 2, 1, 64, 1)]:
        q = _bf16(rng.standard_normal((w, H, d)))
        k = np.zeros((N, Hkv, d), dtype=np.uint16)
        A = orc.window_scores(q, k, H, Hkv, w, 1 / math.sqrt(d))
        ref = closed_form_zero_keys(N, H, Hkv, w)
        err = np.max(np.abs(A - ref) / ref)
        if err > 1e-13:
            return f"K=0 closed form violated (N={N}, w={w}): rel err {err:.3e}"
    return None


def sdpa_probabilities(q_bits, k_bits, H, Hkv, w, scale):
    """Attention probabilities from torch's SDPA (float64, V = identity)."""
    import torch
    q = torch.from_numpy(_widen(q_bits))            # [w][H][d]
    k = torch.from_numpy(_widen(k_bits))            # [N][Hkv][d]
    N = k.shape[0]
    G = H // Hkv
    qh = q.permute(1, 0, 2)                         # [H][w][d]
    kh = k.permute(1, 0, 2).repeat_interleave(G, dim=0)   # [H][N][d], query head h -> KV head h // G
    eye = torch.eye(N, dtype=torch.float64).expand(H, N, N)
    pos = N - w + torch.arange(w)
    mask = torch.arange(N)[None, :] <= pos[:, None]       # [w][N]
    P = torch.nn.functional.scaled_dot_product_attention(qh, kh, eye, attn_mask=mask, scale=scale)
    return P.numpy()                                # [H][w][N]


def pin_sdpa(orc):
    rng = np.random.default_rng(11)
    for (N, H, Hkv, d, w) in [(48, 6, 2, 64, 5), (70, 8, 2, 128, 12), (24, 3, 3, 64, 24)]:
        q, k = _rand_qk(rng, N, H, Hkv, d, w, qscale=1.5)
        scale = 1 / math.sqrt(d)
        A = orc.window_scores(q, k, H, Hkv, w, scale)
        P = sdpa_probabilities(q, k, H, Hkv, w, scale)
        G = H // Hkv
        ref = P.reshape(Hkv, G, w, N).sum(axis=(1, 2))
        err = np.max(np.abs(A - ref) / np.maximum(ref, 1e-300))
        if err > 1e-10:
            return f"SDPA(V=I) mismatch (N={N}, H={H}, Hkv={Hkv}, w={w}): rel err {err:.3e}"
    return None


def logsumexp_rows(q_bits, k_bits, H, Hkv, w, scale):
    """lse [w][H]: scipy's logsumexp of each window row's visible logits,
    the normaliser a causal prefill attention returns for that query."""
    from scipy.special import logsumexp
    q, k = _widen(q_bits), _widen(k_bits)
    N = k.shape[0]
    G = H // Hkv
    out = np.empty((w, H))
    for h in range(H):
        s = scale * (q[:, h, :] @ k[:, h // G, :].T)   # [w][N]
        for i in range(w):
            out[i, h] = logsumexp(s[i, : N - w + i + 1])
    return out


def pin_lse_sdpa(orc):
    """Given the true row log-sum-exp, the scores are the SDPA probabilities
    summed over the group's heads and the window rows."""
    rng = np.random.default_rng(19)
    for (N, H, Hkv, d, w) in [(48, 6, 2, 64, 5), (70, 8, 2, 128, 12)]:
        q, k = _rand_qk(rng, N, H, Hkv, d, w, qscale=1.5)
        scale = 1 / math.sqrt(d)
        lse = logsumexp_rows(q, k, H, Hkv, w, scale)
        lse_view = np.ascontiguousarray(lse.T).T          # [w][H] view of [H][w] storage
        A = orc.window_scores_lse(q, k, lse_view, H, Hkv, w, scale)
        P = sdpa_probabilities(q, k, H, Hkv, w, scale)
        ref = P.reshape(Hkv, H // Hkv, w, N).sum(axis=(1, 2))
        err = np.max(np.abs(A - ref) / np.maximum(ref, 1e-300))
        if err > 1e-10:
            return f"given-lse scores != SDPA(V=I) (N={N}, H={H}, Hkv={Hkv}, w={w}): rel err {err:.3e}"
    return None


def pin_lse_zero_keys(orc):
    """K = 0 with lse[i, h] = ln(#visible keys of row i): the uniform closed form."""
    for (N, H, Hkv, d, w) in [(40, 4, 2, 64, 6), (19, 3, 1, 64, 19)]:
        q = _bf16(np.random.default_rng(N).standard_normal((w, H, d)))
        k = np.zeros((N, Hkv, d), dtype=np.uint16)
        lse = np.log(N - w + np.arange(w) + 1.0)[:, None].repeat(H, axis=1)
        A = orc.window_scores_lse(q, k, lse, H, Hkv, w, 1 / math.sqrt(d))
        ref = closed_form_zero_keys(N, H, Hkv, w)
        err = np.max(np.abs(A - ref) / ref)
        if err > 1e-13:
            return f"given-lse K=0 closed form violated (N={N}, w={w}): rel err {err:.3e}"
    return None


def pin_lse_shift(orc):
    """exp(s - lse - delta) = exp(-delta) exp(s - lse): shifting one row's
    normaliser scales exactly that row's contribution."""
    rng = np.random.default_rng(23)
    N, H, Hkv, d, w = 50, 4, 2, 64, 5
    q, k = _rand_qk(rng, N, H, Hkv, d, w)
    scale = 1 / math.sqrt(d)
    lse = 3.0 * rng.standard_normal((w, H))
    A0 = orc.window_scores_lse(q, k, lse, H, Hkv, w, scale)
    i, h, delta = 2, 3, 1.75
    lse1 = lse.copy()
    lse1[i, h] += delta
    A1 = orc.window_scores_lse(q, k, lse1, H, Hkv, w, scale)
    one = np.full((w, H), np.inf)       # lse = +inf removes a row
    one[i, h] = lse[i, h]
    Arow = orc.window_scores_lse(q, k, one, H, Hkv, w, scale)
    ref = A0 + (math.exp(-delta) - 1.0) * Arow
    err = np.max(np.abs(A1 - ref) / A0)
    if err > 1e-13:
        return f"row normaliser shift not exact: rel err {err:.3e}"
    g = h // (H // Hkv)
    if not (np.all(Arow[1 - g] == 0) and np.all(Arow[g, N - w + i + 1:] == 0) and np.all(Arow[g, : N - w + i + 1] > 0)):
        return "a single row's contribution reaches keys it may not see or another KV head"
    return None


def mpmath_scores(q_bits, k_bits, H, Hkv, w, scale, dps=40):
    import mpmath
    mpmath.mp.dps = dps
    q = _widen(q_bits)
    k = _widen(k_bits)
    N, _, d = k.shape
    G = H // Hkv
    A = [[mpmath.mpf(0) for _ in range(N)] for _ in range(Hkv)]
    sc = mpmath.mpf(scale)
    for h in range(H):
        g = h // G
        for i in range(w):
            last = N - w + i
            s = [sc * mpmath.fsum(mpmath.mpf(float(q[i, h, c])) * mpmath.mpf(float(k[j, g, c]))
                                  for c in range(d)) for j in range(last + 1)]
            e = [mpmath.exp(x) for x in s]
            z = mpmath.fsum(e)
            for j in range(last + 1):
                A[g][j] += e[j] / z
    return np.array([[float(x) for x in row] for row in A])


def pin_mpmath(orc):
    rng = np.random.default_rng(13)
    N, H, Hkv, d, w = 12, 4, 2, 8, 3
    q, k = _rand_qk(rng, N, H, Hkv, d, w, qscale=3.0, kscale=2.0)
    scale = 1 / math.sqrt(d)
    A = orc.window_scores(q, k, H, Hkv, w, scale)
    ref = mpmath_scores(q, k, H, Hkv, w, scale)
    err = np.max(np.abs(A - ref) / ref)
    if err > 1e-12:
        return f"mpmath brute force mismatch: rel err {err:.3e}"
    return None


def pin_mass(orc):
    rng = np.random.default_rng(17)
    N, H, Hkv, d, w = 300, 8, 2, 64, 8
    q, k = _rand_qk(rng, N, H, Hkv, d, w, qscale=2.0)
    A = orc.window_scores(q, k, H, Hkv, w, 1 / math.sqrt(d))
    tot = A.sum(axis=1)
    err = np.max(np.abs(tot - w * (H // Hkv)))
    if err > 1e-9:
        return f"total mass != w*G (err {err:.3e})"
    return None


def pin_dominant_key(orc):
    """A key far more aligned with every window query than any other takes
    (almost) all the mass of every row that can see it."""
    rng = np.random.default_rng(19)
    N, H, Hkv, d, w = 64, 4, 2, 64, 4
    q = _bf16(np.abs(rng.standard_normal((w, H, d))))
    k = _bf16(rng.standard_normal((N, Hkv, d)) * 0.05)
    k[10, :, :] = _bf16(np.full((Hkv, d), 8.0))
    A = orc.window_scores(q, k, H, Hkv, w, 1 / math.sqrt(d))
    G = H // Hkv
    if np.any(A[:, 10] < w * G * (1 - 1e-9)):
        return f"dominant key mass {A[:, 10]} below w*G={w * G}"
    return None


# --------------------------------------------------------------------------- #
# pooling
# --------------------------------------------------------------------------- #
def pin_pool(orc):
    from scipy.ndimage import uniform_filter1d
    rng = np.random.default_rng(23)
    for L in (1, 2, 5, 9, 100):
        for p in (1, 3, 7):
            x = rng.random(L)
            y = orc.avg_pool(x, p)
            ref = uniform_filter1d(x, size=p, mode="constant", cval=0.0)
            if np.max(np.abs(y - ref)) > 1e-14:
                return f"pool mismatch vs scipy uniform_filter1d (L={L}, p={p})"
    # closed form on a constant vector: c * (h + 1 + t) / p at distance t < h from an end
    c, p, L = 3.0, 7, 20
    y = orc.avg_pool(np.full(L, c), p)
    h = p // 2
    for t in range(h):
        want = c * (h + 1 + t) / p
        if abs(y[t] - want) > 1e-14 or abs(y[L - 1 - t] - want) > 1e-14:
            return f"pool edge closed form violated at t={t}"
    if np.max(np.abs(y[h:L - h] - c)) > 1e-14:
        return "pool interior of a constant vector is not the constant"
    return None


# --------------------------------------------------------------------------- #
# selection
# --------------------------------------------------------------------------- #
def check_selection(S, N, w, k, idx):
    """Defining property of the selection; returns a message or None."""
    idx = np.asarray(idx)
    if k >= N:
        return None if np.array_equal(idx, np.arange(N)) else "k >= N must keep every position"
    if len(idx) != k:
        return f"|set| = {len(idx)} != k = {k}"
    if np.any(np.diff(idx) <= 0):
        return "indices not strictly increasing"
    L = N - w
    if not np.all(np.isin(np.arange(L, N), idx)):
        return "window not kept"
    chosen = idx[idx < L]
    if len(chosen) != k - w:
        return "wrong number of prefix positions"
    mask = np.zeros(L, bool)
    mask[chosen] = True
    if mask.all() or not mask.any():
        return None
    lo = S[mask].min()
    hi = S[~mask].max()
    if lo < hi:
        return "an unselected prefix position outranks a selected one"
    if lo == hi:
        # equal scores at the boundary: selected ones must have the lower positions
        sel_eq = np.flatnonzero(mask & (S == lo))
        uns_eq = np.flatnonzero(~mask & (S == lo))
        if sel_eq.max() > uns_eq.min():
            return "tie at the boundary not broken toward the lower position"
    return None


def pin_select(orc):
    rng = np.random.default_rng(29)
    for trial in range(200):
        N = int(rng.integers(2, 60))
        w = int(rng.integers(1, N + 1))
        k = int(rng.integers(w, N + 3))
        S = rng.integers(0, 4, size=N - w).astype(np.float64)   # many ties
        idx = orc.select_topk(S, N, w, k)
        msg = check_selection(S, N, w, k, idx)
        if msg:
            return f"{msg} (N={N}, w={w}, k={k})"
    # all scores equal: the lowest k-w prefix positions plus the window
    N, w, k = 50, 5, 12
    idx = orc.select_topk(np.ones(N - w), N, w, k)
    want = np.concatenate([np.arange(k - w), np.arange(N - w, N)])
    if not np.array_equal(idx, want):
        return "all-equal scores must select 0..k-w-1 plus the window"
    return None


# --------------------------------------------------------------------------- #
# gather
# --------------------------------------------------------------------------- #
def pin_gather(orc):
    rng = np.random.default_rng(31)
    src = rng.integers(0, 1 << 16, size=(50, 3, 16), dtype=np.uint16)
    idx = np.array([3, 0, 49, 7, -1, 12], dtype=np.int32)
    for g in range(3):
        out, bad = orc.gather_rows(src[:, g, :], idx)
        ref = src[np.where(idx < 0, 0, idx), g, :].copy()
        ref[idx < 0] = 0
        if bad != 0 or not np.array_equal(out, ref):
            return "gather differs from numpy indexing"
    out, bad = orc.gather_rows(src[:, 0, :], np.array([1, 50, -7, 2], dtype=np.int32))
    if bad != 2 or np.any(out[1:3] != 0):
        return "out-of-range indices must be counted and zero-filled"
    return None


# --------------------------------------------------------------------------- #
# statistics
# --------------------------------------------------------------------------- #
def pin_stats(orc):
    from scipy.stats import entropy
    N = 1000
    m = (N + 99) // 100
    uni = orc.layer_stats(np.full(N, 5.0), 5.0 * N)
    if abs(uni[0] - math.log(N)) > 1e-12 or abs(uni[1] - m / N) > 1e-12 or abs(uni[2]) > 1e-18:
        return f"uniform closed form violated: {uni}"
    one = np.zeros(N)
    one[37] = 2.5
    oh = orc.layer_stats(one, 2.5)
    if abs(oh[0]) > 1e-15 or abs(oh[1] - 1.0) > 1e-15 or abs(oh[2] - (1 / N) * (1 - 1 / N)) > 1e-15:
        return f"one-hot closed form violated: {oh}"
    rng = np.random.default_rng(37)
    a = rng.random(777) ** 3
    st = orc.layer_stats(a, a.sum())
    ah = a / a.sum()
    top = np.sort(ah)[::-1][: (777 + 99) // 100].sum()
    if (abs(st[0] - entropy(ah)) > 1e-12 or abs(st[1] - top) > 1e-12
            or abs(st[2] - np.var(ah)) > 1e-15):
        return "stats differ from scipy.stats.entropy / numpy.var / sorted sum"
    return None


# --------------------------------------------------------------------------- #
# dynamic pivot detection
# --------------------------------------------------------------------------- #
def _stats(E, S, heads=2):
    """[L][heads][3] float32 with every head's entropy E[l] and top-1% mass S[l]."""
    st = np.zeros((len(E), heads, 3), dtype=np.float32)
    st[:, :, 0] = np.asarray(E, dtype=np.float32)[:, None]
    st[:, :, 1] = np.asarray(S, dtype=np.float32)[:, None]
    return st


def pin_pivot_hand_cases(orc):
    """Each clause of the rule on sequences worked out by hand."""
    flat_s = [0.1] * 6
    rise_s = [0.1, 0.1, 0.1, 0.2, 0.3, 0.4]
    cases = [
        # (E per layer, S per layer, tau, l_min, l_max, expected, what)
        ([5, 5, 5, 3, 3, 3], rise_s, 0.25, 1, 6, 4, "a 40 % drop with rising sparsity at layer 4"),
        ([5, 5, 5, 3, 3, 3], flat_s, 0.25, 1, 6, 6, "no sparsity rise: no pivot, l_max"),
        ([5, 5, 5, 3, 3, 3], rise_s, 0.5, 1, 6, 6, "drop below tau: l_max"),
        ([4, 4, 4, 3, 2, 2], rise_s, 0.25, 1, 6, 4, "drop of exactly tau * E_prev counts"),
        ([4, 4, 4, 3.0000002, 2, 2], rise_s, 0.25, 1, 6, 5, "just under tau * E_prev does not"),
        ([5, 3, 3, 3, 3, 3], [0.1, 0.2, 0.3, 0.4, 0.5, 0.6], 0.25, 3, 6, 6, "a drop before l_min is ignored"),
        ([5, 5, 5, 5, 5, 3], rise_s, 0.25, 1, 4, 4, "a drop after l_max is ignored"),
    ]
    for E, S, tau, lo, hi, want, what in cases:
        got = orc.pivot_layer(_stats(E, S), tau, lo, hi)
        if got != want:
            return f"pivot rule: {what}: got {got}, expected {want}"
    # the per-layer statistic is the mean over the KV heads
    st = _stats([4, 4, 4, 4], [0.1, 0.1, 0.2, 0.3])
    st[2, 0, 0] = 1.0   # one head collapses at layer 3: mean 4 -> 2.5, a 37.5 % drop
    if orc.pivot_layer(st, 0.3, 1, 4) != 3:
        return "pivot rule: a head-mean drop above tau did not fire"
    if orc.pivot_layer(st, 0.4, 1, 4) != 4:
        return "pivot rule: a head-mean drop below tau fired"
    st[2, 1, 0] = 7.0   # the other head rises: the mean stays 4, no drop
    if orc.pivot_layer(st, 0.3, 1, 4) != 4:
        return "pivot rule: one head's collapse fired without a head-mean drop"
    return None


def _phase_change_scores(rng, N, heads, layer, pivot):
    """Per-head aggregates of mass 1: flat noise before the pivot layer,
    a few dominant keys from it on (attention settling on hubs)."""
    A = rng.random((heads, N)) + 0.5
    if layer >= pivot:
        hubs = rng.choice(N, size=8, replace=False)
        A[:, hubs] += 40.0 * N / 8
    return A / A.sum(axis=1, keepdims=True)


def pin_pivot_synthetic_phase_change(orc):
    """Statistics of aggregates whose attention concentrates from layer 7 on
    (computed by the stats routine, itself pinned to closed forms) put the
    pivot at layer 7; without the change it falls back to l_max."""
    rng = np.random.default_rng(29)
    N, heads, L = 4096, 4, 12
    for pivot, want in ((7, 7), (L + 1, 10)):
        st = np.zeros((L, heads, 3), dtype=np.float32)
        for l in range(1, L + 1):
            A = _phase_change_scores(rng, N, heads, l, pivot)
            for g in range(heads):
                st[l - 1, g] = orc.layer_stats(A[g], 1.0)
        got = orc.pivot_layer(st, 0.1, 2, 10)
        if got != want:
            return f"synthetic phase change at layer {pivot}: pivot {got}, expected {want}"
    return None


# --------------------------------------------------------------------------- #
# decode attention over the compacted cache
# --------------------------------------------------------------------------- #
def pin_decode_sdpa(orc):
    """Against torch SDPA in float64 (one query per head, every entry visible)."""
    import torch
    rng = np.random.default_rng(37)
    for (H, Hkv, kk, d) in [(8, 2, 50, 64), (6, 3, 7, 128), (4, 4, 1, 64)]:
        q = _bf16(rng.standard_normal((H, d)) * 1.5)
        kc = _bf16(rng.standard_normal((Hkv, kk, d)))
        vc = _bf16(rng.standard_normal((Hkv, kk, d)))
        scale = 1 / math.sqrt(d)
        out = orc.decode_attention(q, kc, vc, H, Hkv, scale)
        G = H // Hkv
        qt = torch.from_numpy(_widen(q))[:, None, :]                                  # [H][1][d]
        kt = torch.from_numpy(_widen(kc)).repeat_interleave(G, dim=0)                 # [H][kk][d]
        vt = torch.from_numpy(_widen(vc)).repeat_interleave(G, dim=0)
        ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=scale)[:, 0, :].numpy()
        err = np.max(np.abs(out - ref)) / max(np.max(np.abs(ref)), 1e-300)
        if err > 1e-12:
            return f"decode attention != SDPA (H={H}, Hkv={Hkv}, kk={kk}): err {err:.3e}"
    return None


def pin_decode_closed_forms(orc):
    """K = 0: each head's output is the mean of its KV head's V rows; one
    retained entry: exactly that V row."""
    rng = np.random.default_rng(41)
    H, Hkv, kk, d = 6, 2, 9, 64
    q = _bf16(rng.standard_normal((H, d)))
    vc = _bf16(rng.standard_normal((Hkv, kk, d)))
    out = orc.decode_attention(q, np.zeros((Hkv, kk, d), dtype=np.uint16), vc, H, Hkv, 0.125)
    ref = np.repeat(_widen(vc).mean(axis=1), H // Hkv, axis=0)
    if np.max(np.abs(out - ref)) > 1e-14:
        return "decode attention with K = 0 is not the mean of V"
    kc1 = _bf16(rng.standard_normal((Hkv, 1, d)))
    out1 = orc.decode_attention(q, kc1, vc[:, :1, :], H, Hkv, 0.125)
    if not np.array_equal(out1, np.repeat(_widen(vc[:, 0, :]), H // Hkv, axis=0)):
        return "decode attention with one retained entry is not that entry's V row"
    return None


# --------------------------------------------------------------------------- #
# residual vector quantisation of retained K/V rows
# --------------------------------------------------------------------------- #
def _nearest(r, Cs):
    """scipy's squared-Euclidean distances: (argmin, best, second best) per row."""
    from scipy.spatial.distance import cdist
    D = cdist(r, Cs.astype(np.float64), metric="sqeuclidean")
    order = np.argsort(D, axis=1, kind="stable")
    rows = np.arange(len(r))
    return order[:, 0], D[rows, order[:, 0]], D[rows, order[:, 1]]


def pin_rvq_nearest_and_residual(orc):
    """Stage 1 is scipy's nearest codeword; stage 2 is scipy's nearest
    codeword of the residual the test forms itself; the gaps are scipy's."""
    rng = np.random.default_rng(43)
    n, d, M = 300, 32, 64
    x = _bf16(rng.standard_normal((n, d)))
    C = rng.standard_normal((2, M, d)).astype(np.float32)
    codes, gap = orc.rvq_encode(x, C)
    r = _widen(x)
    for st in range(2):
        arg, best, second = _nearest(r, C[st])
        if not np.array_equal(codes[:, st], arg):
            return f"stage {st + 1} codes differ from scipy's nearest codeword"
        if np.max(np.abs(gap[:, st] - (second - best))) > 1e-9:
            return f"stage {st + 1} gaps differ from scipy's"
        r = r - C[st][arg].astype(np.float64)
    return None


def pin_rvq_planted_codes(orc):
    """Codebooks at scales 1, 1/8, 1/64 with entries +-scale: a row built as
    the sum of one codeword per stage (exact in bf16) gives those codes back
    and reconstructs exactly."""
    rng = np.random.default_rng(47)
    n, d, M, S = 200, 16, 32, 3
    C = np.stack([rng.choice([-1.0, 1.0], size=(M, d)) * 8.0 ** -s for s in range(S)]).astype(np.float32)
    planted = rng.integers(0, M, size=(n, S))
    xf = sum(C[s][planted[:, s]].astype(np.float64) for s in range(S))
    x = _bf16(xf)
    if not np.array_equal(_widen(x), xf):
        return "planted rows are not exact in bf16 (test construction)"
    codes, gap = orc.rvq_encode(x, C)
    if not np.array_equal(codes, planted):
        return "planted codes not recovered"
    rec = sum(C[s][codes[:, s]].astype(np.float64) for s in range(S))
    if not np.array_equal(rec, xf) or np.any(gap <= 0):
        return "planted rows do not reconstruct exactly"
    return None


def pin_rvq_tie_to_lowest_index(orc):
    """Equal codewords: the lower index wins; the gap is zero."""
    rng = np.random.default_rng(53)
    d, M = 16, 10
    C = rng.standard_normal((1, M, d)).astype(np.float32)
    C[0, 7] = C[0, 3]
    x = _bf16(C[0, 3].astype(np.float64)[None, :])
    C[0, 3] = _widen(x)[0]
    C[0, 7] = C[0, 3]
    codes, gap = orc.rvq_encode(x, C)
    if codes[0, 0] != 3 or gap[0, 0] != 0.0:
        return f"tie between codewords 3 and 7 gave code {codes[0, 0]}, gap {gap[0, 0]}"
    return None


# --------------------------------------------------------------------------- #
# causal prefill attention with the rows' log-sum-exp
# --------------------------------------------------------------------------- #
def pin_prefill_sdpa(orc):
    """Against torch SDPA in float64 (causal, GQA by repeating the KV heads)
    for the outputs, and scipy's logsumexp of the masked logits the test
    forms itself for the log-sum-exp."""
    import torch
    from scipy.special import logsumexp
    rng = np.random.default_rng(53)
    for (N, H, Hkv, d) in [(37, 4, 2, 64), (9, 6, 3, 128), (1, 2, 1, 64)]:
        q = _bf16(rng.standard_normal((N, H, d)) * 1.5)
        k = _bf16(rng.standard_normal((N, Hkv, d)))
        v = _bf16(rng.standard_normal((N, Hkv, d)))
        scale = 1 / math.sqrt(d)
        out, lse = orc.prefill_attention(q, k, v, H, Hkv, scale)
        G = H // Hkv
        qt = torch.from_numpy(_widen(q)).permute(1, 0, 2)                              # [H][N][d]
        kt = torch.from_numpy(_widen(k)).permute(1, 0, 2).repeat_interleave(G, dim=0)  # [H][N][d]
        vt = torch.from_numpy(_widen(v)).permute(1, 0, 2).repeat_interleave(G, dim=0)
        ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=scale)
        ref = ref.permute(1, 0, 2).numpy()
        err = np.max(np.abs(out - ref)) / max(np.max(np.abs(ref)), 1e-300)
        if err > 1e-12:
            return f"prefill attention != causal SDPA (N={N}, H={H}, Hkv={Hkv}): err {err:.3e}"
        s = np.einsum("nhd,mhd->hnm", _widen(q), np.repeat(_widen(k), G, axis=1)) * scale    # [H][N][N]
        s = np.where(np.tril(np.ones((N, N), dtype=bool))[None], s, -np.inf)
        ref_lse = logsumexp(s, axis=2).T                                                       # [N][H]
        if np.max(np.abs(lse - ref_lse)) > 1e-12 * max(1.0, np.max(np.abs(ref_lse))):
            return f"prefill log-sum-exp != scipy logsumexp (N={N}, H={H})"
    return None


def pin_prefill_closed_forms(orc):
    """K = 0: query i is uniform over keys 0..i, so its output is the mean of
    V rows 0..i and its log-sum-exp is ln(i + 1); query 0 returns V row 0."""
    rng = np.random.default_rng(59)
    N, H, Hkv, d = 20, 4, 2, 64
    q = _bf16(rng.standard_normal((N, H, d)))
    v = _bf16(rng.standard_normal((N, Hkv, d)))
    out, lse = orc.prefill_attention(q, np.zeros((N, Hkv, d), dtype=np.uint16), v, H, Hkv, 0.125)
    vm = np.cumsum(_widen(v), axis=0) / np.arange(1, N + 1)[:, None, None]     # running means [N][Hkv][d]
    ref = np.repeat(vm, H // Hkv, axis=1)
    if np.max(np.abs(out - ref)) > 1e-13:
        return "prefill attention with K = 0 is not the running mean of V"
    if np.max(np.abs(lse - np.log(np.arange(1, N + 1))[:, None])) > 1e-13:
        return "prefill log-sum-exp with K = 0 is not ln(i + 1)"
    out1, _ = orc.prefill_attention(q, _bf16(rng.standard_normal((N, Hkv, d))), v, H, Hkv, 0.125)
    if not np.array_equal(out1[0], np.repeat(_widen(v[0]), H // Hkv, axis=0)):
        return "the first query's output is not V row 0"
    return None


def pin_prefill_lse_feeds_window_scores(orc):
    """The window rows' log-sum-exp from the prefill attention, handed to the
    given-normaliser scores, reproduces the two-pass window scores (the
    scoring normaliser is the attention's)."""
    rng = np.random.default_rng(61)
    N, H, Hkv, d, w = 60, 4, 2, 64, 5
    qa = _bf16(rng.standard_normal((N, H, d)))
    k = _bf16(rng.standard_normal((N, Hkv, d)))
    _, lse = orc.prefill_attention(qa, k, np.zeros_like(k), H, Hkv, 0.125)
    qw = qa[N - w:]
    A2 = orc.window_scores(qw, k, H, Hkv, w, 0.125)
    A1 = orc.window_scores_lse(qw, k, np.ascontiguousarray(lse[N - w:]), H, Hkv, w, 0.125)
    if np.max(np.abs(A1 - A2)) > 1e-12 * max(1.0, np.max(np.abs(A2))):
        return "window scores from the prefill log-sum-exp differ from the two-pass scores"
    return None


ALL_PINS = [pin_zero_keys, pin_sdpa, pin_mpmath, pin_mass, pin_dominant_key, pin_lse_sdpa, pin_lse_zero_keys,
            pin_lse_shift, pin_pool, pin_select, pin_gather, pin_stats, pin_pivot_hand_cases,
            pin_pivot_synthetic_phase_change, pin_decode_sdpa, pin_decode_closed_forms,
            pin_rvq_nearest_and_residual, pin_rvq_planted_codes, pin_rvq_tie_to_lowest_index,
            pin_prefill_sdpa, pin_prefill_closed_forms, pin_prefill_lse_feeds_window_scores]
