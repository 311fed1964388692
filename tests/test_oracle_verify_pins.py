"""Pins of the oracle's block verification against things other than itself.

Page: "MiMo-V2.5-Pro-FP4-DFlash" (alphaneural mirror), section 3
"Block-Diffusion Speculative Decoding (DFlash)": a block of at most 8 drafted
tokens is verified by the backbone in one step, and rejection-sampling
verification keeps the output lossless. The tests pin the reading (greedy
prefix match; per-position acceptance u q(d) < p(d); residual max(0, p - q) at
the first rejection; the bonus token from p_K; inverse-CDF draws in token
order) with hand-worked blocks, closed forms, the losslessness the page
states (checked by brute force over a fine grid of uniforms) and a
temperature invariant. None of them runs on a GPU.
"""
import numpy as np

import oracle


def _logits(p_rows):
    """float32 logits whose softmax at temperature 1 is the given rows."""
    return np.log(np.asarray(p_rows, np.float64)).astype(np.float32)


def test_verify_greedy_worked_block():
    # V = 6, K = 3. Position 0's logits tie at tokens 2 and 4: the argmax is
    # the lower index, 2. Argmaxes by position: 2, 5, 1 and (bonus) 4.
    V = 6
    z = np.full((1, 4, V), -1.0, np.float32)
    z[0, 0, 2] = z[0, 0, 4] = 3.0
    z[0, 1, 5] = 1.0
    z[0, 2, 1] = 2.0
    z[0, 3, 4] = 0.5
    u = np.zeros((1, 4), np.float32)
    acc, tok, _, _ = oracle.verify_block(z, None, np.array([[2, 5, 0]], np.int32), u, 0.0)
    assert acc[0] == 2 and tok[0].tolist() == [2, 5, 1, -1]  # third draft mismatches: correction is 1
    acc, tok, _, _ = oracle.verify_block(z, None, np.array([[2, 5, 1]], np.int32), u, 0.0)
    assert acc[0] == 3 and tok[0].tolist() == [2, 5, 1, 4]  # all match: bonus is position 3's argmax
    acc, tok, _, _ = oracle.verify_block(z, None, np.array([[4, 5, 1]], np.int32), u, 0.0)
    assert acc[0] == 0 and tok[0].tolist() == [2, -1, -1, -1]  # the tie's other token is not the argmax


def test_verify_out_of_range_draft_is_rejected():
    V = 4
    z = np.zeros((1, 3, V), np.float32)
    z[0, :, 3] = 1.0
    w = z[:, :2].copy()
    u = np.zeros((1, 3), np.float32)
    for bad in (-1, V):
        acc, tok, _, _ = oracle.verify_block(z, None, np.array([[3, bad]], np.int32), u, 0.0)
        assert acc[0] == 1 and tok[0].tolist() == [3, 3, -1]
        acc, tok, _, _ = oracle.verify_block(z, w, np.array([[3, bad]], np.int32), u, 1.0)
        assert acc[0] == 1 and tok[0, 0] == 3


def test_verify_equal_distributions_accept_every_draft():
    # q = p: the ratio p(d)/q(d) is 1 and every u < 1 accepts; the bonus token
    # is drawn from p_K = (0.1, 0.2, 0.3, 0.4) by inverse CDF: running sums
    # 0.1, 0.3, 0.6, 1.0, so u = 0.25 -> 1, 0.65 -> 3, 0.05 -> 0, 0.3 -> 2.
    rng = np.random.default_rng(3)
    K, V = 8, 4
    z = rng.standard_normal((1, K + 1, V)).astype(np.float32)
    z[0, K] = _logits([0.1, 0.2, 0.3, 0.4])
    d = rng.integers(0, V, (1, K)).astype(np.int32)
    for uk, want in ((0.25, 1), (0.65, 3), (0.05, 0), (0.30000001, 2)):
        u = np.concatenate([rng.random((1, K)) * 0.999, [[uk]]], axis=1).astype(np.float32)
        acc, tok, _, _ = oracle.verify_block(z, z[:, :K].copy(), d, u, 1.0)
        assert acc[0] == K
        assert tok[0, :K].tolist() == d[0].tolist() and tok[0, K] == want


def test_verify_rejection_closed_form():
    # p = (0.5, 0.3, 0.2), q = (0.2, 0.6, 0.2). Draft 1 has p/q = 1/2: accepted
    # iff u_0 < 1/2. On rejection the residual max(0, p - q) = (0.3, 0, 0)
    # leaves token 0 whatever u_1 is. After an acceptance the bonus token is
    # drawn from p_1 = (0.1, 0.1, 0.8): running sums 0.1, 0.2, 1.0, so u_1 =
    # 0.5 -> 2, 0.15 -> 1. Draft 0 has p/q = 5/2: always accepted.
    z = np.stack([_logits([0.5, 0.3, 0.2]), _logits([0.1, 0.1, 0.8])])[None]
    w = _logits([[0.2, 0.6, 0.2]])[None]
    for u0, u1, want_acc, want_tok in ((0.4, 0.5, 1, [1, 2]), (0.4, 0.15, 1, [1, 1]), (0.7, 0.0, 0, [0, -1]),
                                       (0.7, 0.99, 0, [0, -1]), (0.49, 0.95, 1, [1, 2])):
        u = np.array([[u0, u1]], np.float32)
        acc, tok, _, _ = oracle.verify_block(z, w, np.array([[1]], np.int32), u, 1.0)
        assert acc[0] == want_acc and tok[0].tolist() == want_tok, (u0, u1)
    acc, _, _, _ = oracle.verify_block(z, w, np.array([[0]], np.int32), np.array([[0.999, 0.5]], np.float32), 1.0)
    assert acc[0] == 1


def test_verify_is_lossless_by_brute_force():
    # The first output token of a block must be distributed as p_0 when the
    # draft token is drawn from q_0: P(v) = sum_d q(d) [A_d 1{v = d} +
    # (1 - A_d) S(v)], A_d the acceptance probability of draft d over u_0 and
    # S the distribution of the residual draw over u_1, both measured here on
    # a grid of N midpoints (exact up to 1/N each).
    rng = np.random.default_rng(11)
    V, N = 5, 4000
    grid = ((np.arange(N) + 0.5) / N).astype(np.float32)
    for _ in range(3):
        p = rng.dirichlet(np.ones(V))
        q = rng.dirichlet(np.ones(V))
        z = np.stack([np.log(p), np.log(rng.dirichlet(np.ones(V)))]).astype(np.float32)[None]
        w = np.log(q).astype(np.float32)[None, None]
        p32 = np.exp(z[0, 0].astype(np.float64) - z[0, 0].max())
        p32 /= p32.sum()
        q32 = np.exp(w[0, 0].astype(np.float64) - w[0, 0].max())
        q32 /= q32.sum()
        B = N
        A = np.empty(V)
        for d in range(V):
            u = np.stack([grid, np.full(N, 0.5, np.float32)], axis=1)
            acc, _, _, _ = oracle.verify_block(np.repeat(z, B, 0), np.repeat(w, B, 0), np.full((B, 1), d, np.int32), u,
                                            1.0)
            A[d] = acc.mean()
            assert abs(A[d] - min(1.0, p32[d] / q32[d])) <= 1.0 / N + 1e-12
        d_rej = int(np.argmin(p32 / q32))  # a draft the grid can reject
        u = np.stack([np.full(N, 0.99999, np.float32), grid], axis=1)
        acc, tok, _, _ = oracle.verify_block(np.repeat(z, B, 0), np.repeat(w, B, 0), np.full((B, 1), d_rej, np.int32), u,
                                          1.0)
        assert (acc == 0).all()
        S = np.bincount(tok[:, 0], minlength=V) / N
        P = q32 * A + (q32 * (1.0 - A)).sum() * S
        np.testing.assert_allclose(P, p32, atol=3.0 / N)


def test_verify_temperature_divides_the_logits():
    # softmax(z / tau): logits scaled by 2 at tau = 2 verify as the originals
    # at tau = 1 (the decisions' margins keep float rounding out of the way).
    rng = np.random.default_rng(5)
    B, K, V = 64, 8, 50
    z = rng.standard_normal((B, K + 1, V)).astype(np.float32)
    w = (z[:, :K] + 0.7 * rng.standard_normal((B, K, V))).astype(np.float32)
    d = rng.integers(0, V, (B, K)).astype(np.int32)
    u = rng.random((B, K + 1)).astype(np.float32)
    a1, t1, m1, n1 = oracle.verify_block(z, w, d, u, 1.0)
    a2, t2, m2, n2 = oracle.verify_block(2 * z, 2 * w, d, u, 2.0)
    ok = (np.minimum(m1, n1) > 1e-9) & (np.minimum(m2, n2) > 1e-9)
    assert ok.sum() >= B - 2
    assert (a1[ok] == a2[ok]).all() and (t1[ok] == t2[ok]).all()
    a3, _, _, _ = oracle.verify_block(z, w, d, u, 0.5)
    assert (a3 != a1).any()  # the temperature does change the test


def test_verify_draw_interval_matches_the_draw():
    # The interval a token covers in the normalised running sum is where the
    # draw's uniform must lie: p = (0.1, 0.2, 0.3, 0.4) gives [0.3, 0.6) for
    # token 2; with q = (0.4, 0.1, 0.1, 0.4) the residual (0, 0.1, 0.2, 0)
    # gives [1/3, 1) for token 2; and the draws of the block agree with them.
    z = _logits([0.1, 0.2, 0.3, 0.4])
    w = _logits([0.4, 0.1, 0.1, 0.4])
    lo, hi = oracle.draw_interval(z, None, 1.0, 2)
    assert abs(lo - 0.3) < 1e-7 and abs(hi - 0.6) < 1e-7
    lo, hi = oracle.draw_interval(z, w, 1.0, 2)
    assert abs(lo - 1 / 3) < 1e-7 and abs(hi - 1.0) < 1e-7
    rng = np.random.default_rng(9)
    B, K, V = 40, 2, 30
    zz = rng.standard_normal((B, K + 1, V)).astype(np.float32)
    ww = rng.standard_normal((B, K, V)).astype(np.float32)
    d = rng.integers(0, V, (B, K)).astype(np.int32)
    u = rng.random((B, K + 1)).astype(np.float32)
    acc, tok, _, _ = oracle.verify_block(zz, ww, d, u, 1.0)
    for b in range(B):
        n = acc[b]
        lo, hi = oracle.draw_interval(zz[b, n], ww[b, n] if n < K else None, 1.0, tok[b, n])
        assert lo <= u[b, K] < hi
