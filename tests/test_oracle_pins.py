"""Pins for the fp64 oracle: closed forms, invariants and brute force.

Each check compares the oracle with something other than itself: a value the
mathematics fixes (closed forms, invariants) or an independent brute-force
formulation (full matrices in numpy, complex-number rotation, sorting).  The
sizes are tiny so the whole file runs in seconds on the CPU.
"""
import math

import numpy as np
import pytest

from conftest import bits_to_f64, f64_to_bits

BLOCK = 64


def rng(seed):
    return np.random.default_rng(seed)


def rand_bits(shape, seed, scale=1.0, shift=0.0):
    return f64_to_bits(rng(seed).standard_normal(shape) * scale + shift)


# --------------------------------------------------------------------------- a1
def test_pool_constant_blocks(oracle):
    B, H, S, d = 1, 2, 256, 8
    vals = np.arange(B * H * (S // BLOCK), dtype=np.float64).reshape(B, H, S // BLOCK) * 0.25
    x = np.repeat(vals[..., None], BLOCK, axis=-1).reshape(B, H, S)[..., None].repeat(d, -1)
    out = oracle.pool_avg(f64_to_bits(x))
    np.testing.assert_array_equal(out, np.repeat(vals[..., None], d, -1))


def test_pool_brute_force(oracle):
    bits = rand_bits((2, 3, 192, 16), 1)
    x = bits_to_f64(bits)
    want = x.reshape(2, 3, 3, BLOCK, 16).sum(axis=3) / BLOCK
    np.testing.assert_allclose(oracle.pool_avg(bits), want, rtol=0, atol=1e-14)


# ------------------------------------------------------------------------- RoPE
def test_rope_identity_at_block_zero(oracle):
    x = rng(2).standard_normal(16)
    np.testing.assert_array_equal(oracle.block_rope(x, 0, 5e5), x)


def test_rope_closed_form_basis_vectors(oracle):
    dg, theta = 8, 100.0
    for t in range(dg // 2):
        for p in (1, 3, 17):
            e = np.zeros(dg)
            e[t] = 1.0
            y = oracle.block_rope(e, p, theta)
            ang = p * theta ** (-2.0 * t / dg)
            want = np.zeros(dg)
            want[t] = math.cos(ang)
            want[t + dg // 2] = math.sin(ang)
            np.testing.assert_allclose(y, want, atol=1e-15)


def test_rope_matches_complex_rotation(oracle):
    dg, theta = 32, 5e5
    x = rng(3).standard_normal(dg)
    for p in (0, 1, 5, 511, 2047):
        z = x[: dg // 2] + 1j * x[dg // 2:]
        freqs = theta ** (-2.0 * np.arange(dg // 2) / dg)
        z = z * np.exp(1j * p * freqs)
        want = np.concatenate([z.real, z.imag])
        np.testing.assert_allclose(oracle.block_rope(x, p, theta), want, atol=1e-12)


def test_rope_norm_and_relative_position(oracle):
    dg, theta = 64, 5e5
    a, b = rng(4).standard_normal((2, dg))
    for p in (1, 100, 1000):
        assert abs(np.linalg.norm(oracle.block_rope(a, p, theta)) - np.linalg.norm(a)) < 1e-12
    dot = lambda i, j: oracle.block_rope(a, i, theta) @ oracle.block_rope(b, j, theta)
    for i, j, s in ((5, 2, 7), (40, 40, 3), (9, 0, 100)):
        assert abs(dot(i, j) - dot(i + s, j + s)) < 1e-10


# ------------------------------------------------------------------------ a2/a3
def test_project_identity_weight(oracle):
    B, H, nb, d = 1, 2, 3, 8
    xp = rng(5).standard_normal((B, H, nb, d))
    w = f64_to_bits(np.eye(d))
    out = oracle.project_rope(xp, w, 5e5)          # shared weight (stride 0)
    for i in range(nb):
        for h in range(H):
            np.testing.assert_allclose(out[0, h, i], oracle.block_rope(xp[0, h, i], i, 5e5), atol=1e-14)
    np.testing.assert_array_equal(out[:, :, 0], xp[:, :, 0])


def test_project_per_head_weights_brute_force(oracle):
    B, H, nb, d, dg = 2, 3, 4, 16, 8
    xp = rng(6).standard_normal((B, H, nb, d))
    wbits = rand_bits((H, d, dg), 7, scale=0.2)
    w = bits_to_f64(wbits)
    out = oracle.project_rope(xp, wbits, 1e4)
    for b in range(B):
        for h in range(H):
            for i in range(nb):
                y = xp[b, h, i] @ w[h]
                z = (y[: dg // 2] + 1j * y[dg // 2:]) * np.exp(1j * i * 1e4 ** (-2.0 * np.arange(dg // 2) / dg))
                np.testing.assert_allclose(out[b, h, i], np.concatenate([z.real, z.imag]), atol=1e-12)


def test_block_softmax_rows_and_zero_query(oracle):
    B, Hq, Hkv, nb, dg = 1, 4, 2, 9, 8
    kt = rng(8).standard_normal((B, Hkv, nb, dg))
    s = oracle.block_softmax(np.zeros((B, Hq, nb, dg)), kt)
    for i in range(nb):
        np.testing.assert_allclose(s[..., i, : i + 1], 1.0 / (i + 1), atol=1e-15)
        assert np.all(s[..., i, i + 1:] == 0)
    qt = rng(9).standard_normal((B, Hq, nb, dg)) * 3
    s = oracle.block_softmax(qt, kt)
    np.testing.assert_allclose(s.sum(-1), 1.0, atol=1e-13)
    assert np.all(np.triu(s[0, 0], 1) == 0)


def test_block_softmax_brute_force_gqa(oracle):
    B, Hq, Hkv, nb, dg = 2, 6, 2, 7, 16
    qt = rng(10).standard_normal((B, Hq, nb, dg))
    kt = rng(11).standard_normal((B, Hkv, nb, dg))
    got = oracle.block_softmax(qt, kt)
    kfull = np.repeat(kt, Hq // Hkv, axis=1)
    logits = np.einsum("bhid,bhjd->bhij", qt, kfull) / math.sqrt(dg)
    logits = np.where(np.tril(np.ones((nb, nb), bool)), logits, -np.inf)
    e = np.exp(logits - logits.max(-1, keepdims=True))
    np.testing.assert_allclose(got, e / e.sum(-1, keepdims=True), rtol=1e-12, atol=1e-15)


def _np_gate(q, k, wq, wk, theta):
    """Independent numpy formulation of the gate (reshape-mean, matmul, complex rotation)."""
    B, Hq, S, d = q.shape
    Hkv, nb = k.shape[1], S // BLOCK
    dg = wq.shape[-1]
    qp = q.reshape(B, Hq, nb, BLOCK, d).mean(3)
    kp = k.reshape(B, Hkv, nb, BLOCK, d).mean(3)
    qt = np.einsum("bhid,hde->bhie", qp, wq)
    kt = np.einsum("bhid,hde->bhie", kp, wk)
    rot = np.exp(1j * np.arange(nb)[:, None] * theta ** (-2.0 * np.arange(dg // 2) / dg)[None, :])

    def apply(x):
        z = (x[..., : dg // 2] + 1j * x[..., dg // 2:]) * rot
        return np.concatenate([z.real, z.imag], -1)

    qt, kt = apply(qt), apply(kt)
    kt = np.repeat(kt, Hq // Hkv, axis=1)
    lg = np.einsum("bhie,bhje->bhij", qt, kt) / math.sqrt(dg)
    lg = np.where(np.tril(np.ones((nb, nb), bool)), lg, -np.inf)
    e = np.exp(lg - lg.max(-1, keepdims=True))
    return e / e.sum(-1, keepdims=True)


@pytest.mark.parametrize("dg", [4, 12, 16])
def test_gate_scores_brute_force(oracle, dg):
    """Also at d_gate 4 and 12 (rotation halves of 2 and 6 features)."""
    B, Hq, Hkv, S, d = 1, 4, 2, 512, 32
    qb, kb = rand_bits((B, Hq, S, d), 12, scale=4.0), rand_bits((B, Hkv, S, d), 13, scale=4.0, shift=0.5)
    wqb, wkb = rand_bits((Hq, d, dg), 14, scale=0.5), rand_bits((Hkv, d, dg), 15, scale=0.5)
    got = oracle.gate_scores(qb, kb, wqb, wkb, theta=1e2)
    want = _np_gate(bits_to_f64(qb), bits_to_f64(kb), bits_to_f64(wqb), bits_to_f64(wkb), 1e2)
    np.testing.assert_allclose(got, want, rtol=1e-11, atol=1e-15)


def test_gate_scores_zero_key_weight_is_uniform(oracle):
    B, Hq, Hkv, S, d, dg = 1, 2, 1, 384, 16, 8
    qb, kb = rand_bits((B, Hq, S, d), 16), rand_bits((B, Hkv, S, d), 17)
    wqb = rand_bits((Hq, d, dg), 18)
    wkb = f64_to_bits(np.zeros((Hkv, d, dg)))
    s = oracle.gate_scores(qb, kb, wqb, wkb)
    nb = S // BLOCK
    for i in range(nb):
        np.testing.assert_allclose(s[..., i, : i + 1], 1.0 / (i + 1), atol=1e-15)


# --------------------------------------------------------------------------- a4
def test_threshold_strict_forced_and_monotone(oracle):
    nb = 12
    s = np.abs(rng(19).standard_normal((1, 2, nb, nb))).astype(np.float32)
    s = np.tril(s)
    tau = float(s[0, 0, 7, 3])                          # an exact score value
    m = oracle.block_mask(s, "threshold", tau, force_first=False, force_diag=False)
    assert m[0, 0, 7, 3] == 0                           # strict >
    np.testing.assert_array_equal(m, (s > np.float32(tau)) & np.tril(np.ones((nb, nb), bool)))
    mf = oracle.block_mask(s, "threshold", 1e9)
    want = np.zeros((nb, nb), np.uint8)
    want[:, 0] = 1
    want[np.arange(nb), np.arange(nb)] = 1
    np.testing.assert_array_equal(mf[0, 1], want)
    prev = None
    for t in (0.0, 0.2, 0.5, 1.0, 2.0):
        cur = oracle.block_mask(s, "threshold", t)
        if prev is not None:
            assert np.all(cur <= prev)
        prev = cur
    assert np.all(np.triu(prev[0, 0], 1) == 0)


def _np_topk_mask(s, k_row, ff, fd):
    B, H, nb, _ = s.shape
    out = np.zeros_like(s, dtype=np.uint8)
    for b in range(B):
        for h in range(H):
            for i in range(nb):
                forced = set()
                if ff:
                    forced.add(0)
                if fd:
                    forced.add(i)
                k = min(max(int(k_row[i]), len(forced)), i + 1)
                rest = sorted((j for j in range(i + 1) if j not in forced),
                              key=lambda j: (-float(s[b, h, i, j]), j))
                for j in list(forced) + rest[: k - len(forced)]:
                    out[b, h, i, j] = 1
    return out


@pytest.mark.parametrize("ff,fd", [(True, True), (False, False), (True, False), (False, True)])
def test_topk_exact_count_and_brute_force(oracle, ff, fd):
    nb = 16
    s = np.tril(np.abs(rng(20).standard_normal((2, 3, nb, nb)))).astype(np.float32)
    s[0, 0, 10, :6] = 0.5                                # ties: lower j must win
    k_row = np.array([oracle.topk_count(0.3, i, 0) for i in range(nb)], np.int32)
    m = oracle.block_mask(s, "topk", k_row=k_row, force_first=ff, force_diag=fd)
    np.testing.assert_array_equal(m, _np_topk_mask(s, k_row, ff, fd))
    for i in range(nb):
        nf = len(({0} if ff else set()) | ({i} if fd else set()))
        assert np.all(m[..., i, :].sum(-1) == min(max(k_row[i], nf), i + 1))


def test_topk_count_closed_form(oracle):
    assert oracle.topk_count(0.1, 0, 1) == 1
    assert oracle.topk_count(0.1, 9, 2) == 2        # ceil(1.0) = 1 -> clamped to 2 forced
    assert oracle.topk_count(0.1, 99, 2) == 10
    assert oracle.topk_count(0.1, 100, 2) == 11     # ceil(10.1)
    assert oracle.topk_count(1.0, 511, 2) == 512
    assert oracle.topk_count(0.5, 7, 0) == 4
    assert oracle.topk_count(2.0, 3, 0) == 4        # clamped to i + 1


# --------------------------------------------------------------------------- a5
def test_compact_lists(oracle):
    nb = 10
    m = (rng(21).random((2, 3, nb, nb)) < 0.4).astype(np.uint8) * np.tril(np.ones((nb, nb), np.uint8))
    lists, counts = oracle.compact(m)
    np.testing.assert_array_equal(counts, m.sum(-1))
    for b in range(2):
        for h in range(3):
            for i in range(nb):
                off = i * (i + 1) // 2
                np.testing.assert_array_equal(lists[b, h, off: off + counts[b, h, i]], np.nonzero(m[b, h, i])[0])


# --------------------------------------------------------------------------- a6
def _np_masked_attention(q, k, v, mask, scale):
    """Full-matrix formulation: token-level mask from the block mask, then softmax."""
    B, Hq, S, d = q.shape
    g = Hq // k.shape[1]
    kf, vf = np.repeat(k, g, 1), np.repeat(v, g, 1)
    tok = np.repeat(np.repeat(mask.astype(bool), BLOCK, -1), BLOCK, -2)
    tok &= np.tril(np.ones((S, S), bool))
    s = np.einsum("bhrd,bhcd->bhrc", q, kf) * scale
    s = np.where(tok, s, -np.inf)
    mx = s.max(-1, keepdims=True)
    has = np.isfinite(mx)
    p = np.where(has, np.exp(s - np.where(has, mx, 0)), 0.0)
    l = p.sum(-1, keepdims=True)
    o = np.where(has, np.einsum("bhrc,bhcd->bhrd", p, vf) / np.where(has, l, 1), 0.0)
    lse = np.where(has[..., 0], (mx + np.log(np.where(has, l, 1)))[..., 0], -np.inf)
    return o, lse


def _as_units(o, B, H, nb, d):
    return o.reshape(B * H * nb, BLOCK, d)


def test_attention_random_mask_brute_force(oracle):
    B, Hq, Hkv, S, d = 1, 4, 2, 384, 32
    nb = S // BLOCK
    qb, kb, vb = (rand_bits((B, h, S, d), 22 + i) for i, h in enumerate((Hq, Hkv, Hkv)))
    m = (rng(25).random((B, Hq, nb, nb)) < 0.5).astype(np.uint8) * np.tril(np.ones((nb, nb), np.uint8))
    m[0, 1, 3, :] = 0                      # a row with no active block at all
    o, lse = oracle.masked_attention(qb, kb, vb, m)
    wo, wl = _np_masked_attention(bits_to_f64(qb), bits_to_f64(kb), bits_to_f64(vb), m, 1 / math.sqrt(d))
    np.testing.assert_allclose(o, _as_units(wo, B, Hq, nb, d), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(lse, wl.reshape(-1, BLOCK), rtol=1e-12)
    assert np.all(o.reshape(B, Hq, nb, BLOCK, d)[0, 1, 3] == 0)


def test_attention_density_one_is_dense_causal(oracle):
    B, Hq, Hkv, S, d = 1, 2, 1, 256, 16
    nb = S // BLOCK
    qb, kb, vb = (rand_bits((B, h, S, d), 30 + i, scale=2.0) for i, h in enumerate((Hq, Hkv, Hkv)))
    full = np.ones((B, Hq, nb, nb), np.uint8)
    o, lse = oracle.masked_attention(qb, kb, vb, full, scale=0.3)
    q, k, v = bits_to_f64(qb), bits_to_f64(kb), bits_to_f64(vb)
    s = np.einsum("hrd,cd->hrc", q[0], k[0, 0]) * 0.3 + np.triu(np.full((S, S), -np.inf), 1)
    p = np.exp(s - s.max(-1, keepdims=True))
    want = (p / p.sum(-1, keepdims=True)) @ v[0, 0]
    np.testing.assert_allclose(o.reshape(Hq, S, d), want, rtol=1e-10, atol=1e-12)


def test_attention_all_diagonal_is_block_local(oracle):
    B, Hq, Hkv, S, d = 1, 2, 2, 256, 16
    nb = S // BLOCK
    qb, kb, vb = (rand_bits((B, h, S, d), 40 + i) for i, h in enumerate((Hq, Hkv, Hkv)))
    diag = np.broadcast_to(np.eye(nb, dtype=np.uint8), (B, Hq, nb, nb)).copy()
    o, _ = oracle.masked_attention(qb, kb, vb, diag)
    q, k, v = bits_to_f64(qb), bits_to_f64(kb), bits_to_f64(vb)
    for h in range(Hq):
        for i in range(nb):
            sl = slice(i * BLOCK, (i + 1) * BLOCK)
            s = q[0, h, sl] @ k[0, h, sl].T / 4.0 + np.triu(np.full((BLOCK, BLOCK), -np.inf), 1)
            p = np.exp(s - s.max(-1, keepdims=True))
            want = (p / p.sum(-1, keepdims=True)) @ v[0, h, sl]
            np.testing.assert_allclose(o[h * nb + i], want, rtol=1e-10, atol=1e-12)


def test_attention_zero_query_prefix_mean_and_constant_v(oracle):
    B, Hq, Hkv, S, d = 1, 1, 1, 192, 8
    nb = S // BLOCK
    kb, vb = rand_bits((B, Hkv, S, d), 50), rand_bits((B, Hkv, S, d), 51)
    qz = f64_to_bits(np.zeros((B, Hq, S, d)))
    full = np.ones((B, Hq, nb, nb), np.uint8)
    o, lse = oracle.masked_attention(qz, kb, vb, full)
    v = bits_to_f64(vb)[0, 0]
    want = np.cumsum(v, 0) / np.arange(1, S + 1)[:, None]
    np.testing.assert_allclose(o.reshape(S, d), want, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse.reshape(S), np.log(np.arange(1, S + 1)), rtol=1e-14)
    vc = f64_to_bits(np.full((B, Hkv, S, d), 1.5))
    m = (rng(52).random((B, Hq, nb, nb)) < 0.5).astype(np.uint8) | np.eye(nb, dtype=np.uint8)
    o, _ = oracle.masked_attention(rand_bits((B, Hq, S, d), 53), kb, vc, np.tril(m))
    np.testing.assert_allclose(o, 1.5, rtol=1e-14)


# --------------------------------------------------------------------------- a7
def test_pooled_map_brute_force_and_bounds(oracle):
    B, Hq, Hkv, S, d = 1, 2, 1, 320, 16
    nb = S // BLOCK
    qb, kb, vb = (rand_bits((B, h, S, d), 60 + i, scale=2.0) for i, h in enumerate((Hq, Hkv, Hkv)))
    o, A = oracle.pooled_map(qb, kb, vb)
    q, k, v = bits_to_f64(qb), bits_to_f64(kb), bits_to_f64(vb)
    A = A.reshape(Hq, nb, nb)
    for h in range(Hq):
        s = q[0, h] @ k[0, 0].T / 4.0 + np.triu(np.full((S, S), -np.inf), 1)
        p = np.exp(s - s.max(-1, keepdims=True))
        p /= p.sum(-1, keepdims=True)
        np.testing.assert_allclose(o.reshape(Hq, S, d)[h], p @ v[0, 0], rtol=1e-10, atol=1e-12)
        pooled = p.reshape(nb, BLOCK, nb, BLOCK).max(axis=(1, 3))
        np.testing.assert_allclose(A[h], pooled, rtol=1e-12, atol=0)
    assert np.all(A[:, 0, 0] == 1.0)
    assert np.all((A >= 0) & (A <= 1))
    assert np.all(np.triu(A, 1) == 0)
    for i in range(nb):
        assert np.all(A[:, i].max(-1) >= 1.0 / (BLOCK * i + 1) - 1e-15)
        assert np.all(A[:, i].sum(-1) >= 1.0 / BLOCK) and np.all(A[:, i].sum(-1) <= BLOCK)


def test_pooled_map_zero_query_closed_form(oracle):
    B, Hq, Hkv, S, d = 1, 1, 1, 256, 8
    nb = S // BLOCK
    qz = f64_to_bits(np.zeros((B, Hq, S, d)))
    _, A = oracle.pooled_map(qz, rand_bits((B, Hkv, S, d), 70), rand_bits((B, Hkv, S, d), 71))
    for i in range(nb):
        np.testing.assert_allclose(A[i, : i + 1], 1.0 / (BLOCK * i + 1), rtol=1e-14)
        assert np.all(A[i, i + 1:] == 0)


def test_pooled_map_units_subset_matches_full(oracle):
    B, Hq, Hkv, S, d = 2, 2, 1, 256, 8
    nb = S // BLOCK
    qb, kb, vb = (rand_bits((B, h, S, d), 80 + i) for i, h in enumerate((Hq, Hkv, Hkv)))
    of, Af = oracle.pooled_map(qb, kb, vb)
    units = np.array([[1, 1, 3], [0, 0, 0], [1, 0, 2]], np.int32)
    o, A = oracle.pooled_map(qb, kb, vb, units=units)
    for n, (b, h, i) in enumerate(units):
        idx = (b * Hq + h) * nb + i
        np.testing.assert_array_equal(o[n], of[idx])
        np.testing.assert_array_equal(A[n], Af[idx])


# ------------------------------------------------------------ distillation loss
def test_distill_loss_pins(oracle):
    B, Hq, nb = 2, 3, 9
    r = rng(90)
    G = np.tril(r.random((B, Hq, nb, nb))).astype(np.float32)
    G /= G.sum(-1, keepdims=True)
    G = G.astype(np.float32)
    # A proportional to G row by row -> target equals G (up to f32 rounding) -> loss ~ 0
    scale = r.random((B, Hq, nb, 1)).astype(np.float32) + 0.5
    ahat, rows, heads = oracle.distill_loss(G, (G * scale).astype(np.float32))
    np.testing.assert_allclose(ahat, G, rtol=1e-6, atol=1e-7)
    assert np.all(heads < 1e-12)
    # rows of the target sum to 1; zero rows stay zero; loss is then sum G^2
    A = np.tril(r.random((B, Hq, nb, nb))).astype(np.float32)
    A[0, 1, 4, :] = 0
    ahat, rows, heads = oracle.distill_loss(G, A)
    s = ahat.sum(-1)
    s[0, 1, 4] = 1.0
    np.testing.assert_allclose(s, 1.0, rtol=1e-12)
    assert np.all(ahat[0, 1, 4] == 0)
    np.testing.assert_allclose(rows[0, 1, 4], (G[0, 1, 4].astype(np.float64) ** 2).sum(), rtol=1e-12)
    # brute force
    Ad, Gd = A.astype(np.float64), G.astype(np.float64)
    tot = Ad.sum(-1, keepdims=True)
    want_hat = np.where(tot > 0, Ad / np.where(tot > 0, tot, 1), 0.0)
    np.testing.assert_allclose(ahat, want_hat, rtol=1e-12, atol=0)
    lower = np.tril(np.ones((nb, nb), bool))
    want_rows = (((Gd - want_hat) ** 2) * lower).sum(-1)
    np.testing.assert_allclose(rows, want_rows, rtol=1e-12)
    np.testing.assert_allclose(heads, want_rows.sum(-1) / (nb * (nb + 1) / 2), rtol=1e-12)


# ------------------------------------------------------------ max+min K pooling
def test_pool_maxmin_pins(oracle):
    bits = rand_bits((2, 3, 192, 16), 91)
    x = bits_to_f64(bits).reshape(2, 3, 3, BLOCK, 16)
    out = oracle.pool_maxmin(bits)
    np.testing.assert_array_equal(out[..., :16], x.max(axis=3))
    np.testing.assert_array_equal(out[..., 16:], x.min(axis=3))
    # constant blocks: max == min == the constant
    const = f64_to_bits(np.full((1, 1, 128, 4), 0.75))
    o = oracle.pool_maxmin(const)
    assert np.all(o == 0.75)


def test_gate_scores_maxmin_brute_force(oracle):
    B, Hq, Hkv, S, d, dg = 1, 4, 2, 512, 16, 8
    qb, kb = rand_bits((B, Hq, S, d), 92, scale=3.0), rand_bits((B, Hkv, S, d), 93, scale=3.0)
    wqb, wkb = rand_bits((Hq, d, dg), 94, scale=0.5), rand_bits((Hkv, 2 * d, dg), 95, scale=0.5)
    got = oracle.gate_scores(qb, kb, wqb, wkb, theta=1e2, k_maxmin=True)
    q, k = bits_to_f64(qb), bits_to_f64(kb)
    nb = S // BLOCK
    qp = q.reshape(B, Hq, nb, BLOCK, d).mean(3)
    kr = k.reshape(B, Hkv, nb, BLOCK, d)
    kp = np.concatenate([kr.max(3), kr.min(3)], -1)
    qt = np.einsum("bhid,hde->bhie", qp, bits_to_f64(wqb))
    kt = np.einsum("bhid,hde->bhie", kp, bits_to_f64(wkb))
    rot = np.exp(1j * np.arange(nb)[:, None] * 1e2 ** (-2.0 * np.arange(dg // 2) / dg)[None, :])

    def apply(xx):
        z = (xx[..., : dg // 2] + 1j * xx[..., dg // 2:]) * rot
        return np.concatenate([z.real, z.imag], -1)

    qt, kt = apply(qt), np.repeat(apply(kt), Hq // Hkv, axis=1)
    lg = np.einsum("bhie,bhje->bhij", qt, kt) / math.sqrt(dg)
    lg = np.where(np.tril(np.ones((nb, nb), bool)), lg, -np.inf)
    e = np.exp(lg - lg.max(-1, keepdims=True))
    np.testing.assert_allclose(got, e / e.sum(-1, keepdims=True), rtol=1e-11, atol=1e-15)
    # the avg path is unchanged by the new entry point
    np.testing.assert_array_equal(oracle.gate_scores(qb, kb, wqb, rand_bits((Hkv, d, dg), 96)),
                                  oracle.gate_scores(qb, kb, wqb, rand_bits((Hkv, d, dg), 96), k_maxmin=False))


# ----------------------------------------------------- S not a multiple of 64
def _blocks(S):
    """(start, stop) of every 64-token block of a sequence of S tokens."""
    return [(s, min(s + BLOCK, S)) for s in range(0, S, BLOCK)]


def test_ragged_pool_brute_force(oracle):
    """The last block of a ragged sequence pools only its real tokens."""
    S = 3 * BLOCK + 17
    bits = rand_bits((2, 3, S, 8), 101)
    x = bits_to_f64(bits)
    want_avg = np.stack([x[:, :, a:b].mean(2) for a, b in _blocks(S)], 2)
    want_max = np.stack([x[:, :, a:b].max(2) for a, b in _blocks(S)], 2)
    want_min = np.stack([x[:, :, a:b].min(2) for a, b in _blocks(S)], 2)
    np.testing.assert_allclose(oracle.pool_avg(bits), want_avg, rtol=0, atol=1e-14)
    mm = oracle.pool_maxmin(bits)
    np.testing.assert_array_equal(mm[..., :8], want_max)
    np.testing.assert_array_equal(mm[..., 8:], want_min)
    # a constant tail block pools to that constant whatever its length
    for tail in (1, 5, 63):
        c = f64_to_bits(np.full((1, 1, BLOCK + tail, 4), -1.5))
        assert np.all(oracle.pool_avg(c) == -1.5)


def test_ragged_gate_brute_force(oracle):
    B, Hq, Hkv, S, d, dg = 1, 4, 2, 5 * BLOCK + 9, 16, 8
    qb, kb = rand_bits((B, Hq, S, d), 102, scale=4.0), rand_bits((B, Hkv, S, d), 103, scale=4.0, shift=0.5)
    wqb, wkb = rand_bits((Hq, d, dg), 104, scale=0.5), rand_bits((Hkv, d, dg), 105, scale=0.5)
    got = oracle.gate_scores(qb, kb, wqb, wkb, theta=1e3)
    q, k = bits_to_f64(qb), bits_to_f64(kb)
    nb = len(_blocks(S))
    qp = np.stack([q[:, :, a:b].mean(2) for a, b in _blocks(S)], 2)
    kp = np.stack([k[:, :, a:b].mean(2) for a, b in _blocks(S)], 2)
    qt = np.einsum("bhid,hde->bhie", qp, bits_to_f64(wqb))
    kt = np.einsum("bhid,hde->bhie", kp, bits_to_f64(wkb))
    rot = np.exp(1j * np.arange(nb)[:, None] * 1e3 ** (-2.0 * np.arange(dg // 2) / dg)[None, :])

    def apply(xx):
        z = (xx[..., : dg // 2] + 1j * xx[..., dg // 2:]) * rot
        return np.concatenate([z.real, z.imag], -1)

    qt, kt = apply(qt), np.repeat(apply(kt), Hq // Hkv, axis=1)
    lg = np.einsum("bhie,bhje->bhij", qt, kt) / math.sqrt(dg)
    lg = np.where(np.tril(np.ones((nb, nb), bool)), lg, -np.inf)
    e = np.exp(lg - lg.max(-1, keepdims=True))
    assert got.shape == (B, Hq, nb, nb)
    np.testing.assert_allclose(got, e / e.sum(-1, keepdims=True), rtol=1e-11, atol=1e-15)


def test_ragged_attention_brute_force_and_prefix(oracle):
    """Rows past S do not exist (zero, LSE -inf); the rest equals a token-level
    brute force, and equals the same rows of a longer sequence (causality: a
    token never sees later ones), whatever the extra tokens hold."""
    B, Hq, Hkv, d = 1, 4, 2, 16
    S = 4 * BLOCK + 21
    nb = len(_blocks(S))
    qb, kb, vb = (rand_bits((B, h, S, d), 106 + i, scale=1.5) for i, h in enumerate((Hq, Hkv, Hkv)))
    m = (rng(109).random((B, Hq, nb, nb)) < 0.6).astype(np.uint8) * np.tril(np.ones((nb, nb), np.uint8))
    m[..., np.arange(nb), np.arange(nb)] = 1
    o, lse = oracle.masked_attention(qb, kb, vb, m, scale=0.2)
    q, k, v = bits_to_f64(qb), bits_to_f64(kb), bits_to_f64(vb)
    blk = np.arange(S) // BLOCK
    o = o.reshape(B, Hq, nb * BLOCK, d)
    lse = lse.reshape(B, Hq, nb * BLOCK)
    for h in range(Hq):
        tok = m[0, h][blk[:, None], blk[None, :]].astype(bool) & np.tril(np.ones((S, S), bool))
        s = np.where(tok, q[0, h] @ k[0, h // 2].T * 0.2, -np.inf)
        mx = s.max(-1, keepdims=True)
        p = np.exp(s - mx)
        np.testing.assert_allclose(o[0, h, :S], (p @ v[0, h // 2]) / p.sum(-1, keepdims=True), rtol=1e-10,
                                   atol=1e-12)
        np.testing.assert_allclose(lse[0, h, :S], (mx + np.log(p.sum(-1, keepdims=True)))[:, 0], rtol=1e-12)
    assert np.all(o[:, :, S:] == 0) and np.all(np.isneginf(lse[:, :, S:]))
    # the same rows of a block-aligned sequence with arbitrary extra tokens
    pad = nb * BLOCK - S
    ext = [np.concatenate([t, rand_bits((B, t.shape[1], pad, d), 110 + i, scale=9.0)], 2)
           for i, t in enumerate((qb, kb, vb))]
    o2, lse2 = oracle.masked_attention(*ext, m, scale=0.2)
    np.testing.assert_array_equal(o2.reshape(B, Hq, nb * BLOCK, d)[:, :, :S], o[:, :, :S])
    np.testing.assert_array_equal(lse2.reshape(B, Hq, nb * BLOCK)[:, :, :S], lse[:, :, :S])


def test_ragged_pooled_map_brute_force(oracle):
    B, Hq, Hkv, d = 1, 2, 1, 16
    S = 4 * BLOCK + 30
    nb = len(_blocks(S))
    qb, kb, vb = (rand_bits((B, h, S, d), 112 + i, scale=2.0) for i, h in enumerate((Hq, Hkv, Hkv)))
    o, A = oracle.pooled_map(qb, kb, vb)
    q, k, v = bits_to_f64(qb), bits_to_f64(kb), bits_to_f64(vb)
    A = A.reshape(Hq, nb, nb)
    o = o.reshape(Hq, nb * BLOCK, d)
    for h in range(Hq):
        s = q[0, h] @ k[0, 0].T / 4.0 + np.triu(np.full((S, S), -np.inf), 1)
        p = np.exp(s - s.max(-1, keepdims=True))
        p /= p.sum(-1, keepdims=True)
        np.testing.assert_allclose(o[h, :S], p @ v[0, 0], rtol=1e-10, atol=1e-12)
        assert np.all(o[h, S:] == 0)
        want = np.array([[p[a:b, c:e].max() if j <= i else 0.0 for j, (c, e) in enumerate(_blocks(S))]
                         for i, (a, b) in enumerate(_blocks(S))])
        np.testing.assert_allclose(A[h], want, rtol=1e-12, atol=0)


# --------------------------------------------------------------------- decode
def _rot(x, pos, theta, dg):
    """Rotate-half RoPE at integer positions `pos` (broadcast over leading axes) via complex numbers."""
    ang = np.asarray(pos)[..., None] * theta ** (-2.0 * np.arange(dg // 2) / dg)
    z = (x[..., : dg // 2] + 1j * x[..., dg // 2:]) * np.exp(1j * ang)
    return np.concatenate([z.real, z.imag], -1)


@pytest.mark.parametrize("L,maxmin", [(5 * BLOCK + 20, False), (3 * BLOCK, True), (41, False)])
def test_decode_gate_brute_force(oracle, L, maxmin):
    """Decode gate: the token's own q (no pooling) projected and rotated at its
    block (the last), against the pooled, projected, rotated K of every block."""
    B, Hq, Hkv, d, dg, theta = 2, 4, 2, 16, 8, 1e3
    qb = rand_bits((B, Hq, d), 120, scale=3.0)
    kb = rand_bits((B, Hkv, L, d), 121, scale=3.0, shift=0.3)
    dk = 2 * d if maxmin else d
    wqb, wkb = rand_bits((Hq, d, dg), 122, scale=0.5), rand_bits((Hkv, dk, dg), 123, scale=0.5)
    got = oracle.decode_gate_scores(qb, kb, wqb, wkb, theta=theta, k_maxmin=maxmin)
    q, k = bits_to_f64(qb), bits_to_f64(kb)
    blocks = _blocks(L)
    nb = len(blocks)
    if maxmin:
        kp = np.stack([np.concatenate([k[:, :, a:b].max(2), k[:, :, a:b].min(2)], -1) for a, b in blocks], 2)
    else:
        kp = np.stack([k[:, :, a:b].mean(2) for a, b in blocks], 2)
    kt = _rot(np.einsum("bhjd,hde->bhje", kp, bits_to_f64(wkb)), np.arange(nb), theta, dg)
    qt = _rot(np.einsum("bhd,hde->bhe", q, bits_to_f64(wqb)), nb - 1, theta, dg)
    lg = np.einsum("bhe,bhje->bhj", qt, np.repeat(kt, Hq // Hkv, axis=1)) / math.sqrt(dg)
    e = np.exp(lg - lg.max(-1, keepdims=True))
    assert got.shape == (B, Hq, nb)
    np.testing.assert_allclose(got, e / e.sum(-1, keepdims=True), rtol=1e-11, atol=1e-15)
    np.testing.assert_allclose(got.sum(-1), 1.0, rtol=1e-13)


def test_decode_mask_brute_force(oracle):
    B, Hq, nb = 2, 3, 37
    s = rng(124).random((B, Hq, nb)).astype(np.float32)
    s[0, 0, 5] = s[0, 0, 9] = s[0, 0, 20]            # ties go to the lower block
    for k in (1, 2, 5, 11, nb, nb + 4):
        got = oracle.decode_mask(s, "topk", k=k)
        for b in range(B):
            for h in range(Hq):
                want = np.zeros(nb, np.uint8)
                want[0] = want[nb - 1] = 1
                rest = [j for j in sorted(range(1, nb - 1), key=lambda j: (-s[b, h, j], j))]
                for j in rest[: max(0, min(k, nb) - 2)]:
                    want[j] = 1
                np.testing.assert_array_equal(got[b, h], want)
    thr = np.float32(0.5)
    got = oracle.decode_mask(s, "threshold", threshold=thr)
    want = (s > thr).astype(np.uint8)
    want[..., 0] = want[..., nb - 1] = 1
    np.testing.assert_array_equal(got, want)


@pytest.mark.parametrize("L", [7 * BLOCK + 13, 4 * BLOCK, 30])
def test_decode_attention_brute_force(oracle, L):
    B, Hq, Hkv, d = 1, 4, 2, 16
    nb = len(_blocks(L))
    qb = rand_bits((B, Hq, d), 125, scale=2.0)
    kb, vb = rand_bits((B, Hkv, L, d), 126), rand_bits((B, Hkv, L, d), 127)
    m = (rng(128).random((B, Hq, nb)) < 0.5).astype(np.uint8)
    m[..., nb - 1] = 1
    o, lse = oracle.decode_attention(qb, kb, vb, m, scale=0.3)
    q, k, v = bits_to_f64(qb), bits_to_f64(kb), bits_to_f64(vb)
    for h in range(Hq):
        act = m[0, h][np.arange(L) // BLOCK].astype(bool)
        s = np.where(act, k[0, h // 2] @ q[0, h] * 0.3, -np.inf)
        p = np.exp(s - s.max())
        np.testing.assert_allclose(o[0, h], p @ v[0, h // 2] / p.sum(), rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(lse[0, h], s.max() + np.log(p.sum()), rtol=1e-12)
    # every block active: plain softmax over all L keys (the token sees the whole cache)
    o1, _ = oracle.decode_attention(qb, kb, vb, np.ones((B, Hq, nb), np.uint8), scale=0.3)
    s = np.einsum("hcd,hd->hc", np.repeat(k[0], 2, axis=0), q[0]) * 0.3
    p = np.exp(s - s.max(-1, keepdims=True))
    np.testing.assert_allclose(o1[0], np.einsum("hc,hcd->hd", p, np.repeat(v[0], 2, axis=0)) / p.sum(-1, keepdims=True),
                               rtol=1e-10, atol=1e-12)


# ------------------------------------------------- pooling: shapes and torch
def _golden_rows(name):
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", name)
    rows = []
    for line in open(path):
        line = line.split("#", 1)[0].strip()
        if line:
            lhs, rhs = line.split("->")
            rows.append((lhs.split(), tuple(int(v) for v in rhs.split())))
    return rows


def test_pool_shapes_golden(oracle):
    """Worked shape example of the pooling (rebuttal, Weakness 3 and 4)."""
    rows = _golden_rows("pooling_shapes.txt")
    assert len(rows) >= 5
    for (b, h, s, d, kind), want in rows:
        bits = rand_bits((int(b), int(h), int(s), int(d)), 7)
        out = oracle.pool_avg(bits) if kind == "avg" else oracle.pool_maxmin(bits)
        assert out.shape == want, (b, h, s, d, kind)


def test_pool_matches_torch_ceil_mode(oracle):
    """Rebuttal, Weakness 4: ragged sequences pool like torch's pooling with
    ceil_mode=True (the window past the end covers only the real tokens)."""
    torch = pytest.importorskip("torch")
    F = torch.nn.functional
    for S in (BLOCK, 2 * BLOCK + 1, 3 * BLOCK + 40, 5 * BLOCK - 1):
        bits = rand_bits((2, 3, S, 8), 200 + S)
        x = torch.from_numpy(bits_to_f64(bits))                      # [B, H, S, d]
        xs = x.permute(0, 1, 3, 2).reshape(-1, 1, S)                 # pool along S
        avg = F.avg_pool1d(xs, BLOCK, BLOCK, ceil_mode=True)
        mx = F.max_pool1d(xs, BLOCK, BLOCK, ceil_mode=True)
        mn = -F.max_pool1d(-xs, BLOCK, BLOCK, ceil_mode=True)
        nb = -(-S // BLOCK)
        to4 = lambda t: t.reshape(2, 3, 8, nb).permute(0, 1, 3, 2).numpy()
        np.testing.assert_allclose(oracle.pool_avg(bits), to4(avg), rtol=0, atol=1e-14)
        mm = oracle.pool_maxmin(bits)
        np.testing.assert_array_equal(mm[..., :8], to4(mx))
        np.testing.assert_array_equal(mm[..., 8:], to4(mn))
