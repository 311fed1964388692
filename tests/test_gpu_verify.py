"""Parity of the CUDA block verification (mxmoe_verify_block) with the
float64 oracle on the same seeded inputs.

Greedy verification compares float logits exactly on both sides, so accepted
counts and tokens must be identical. Sampling takes its decisions in fp32 on
the GPU and in float64 in the oracle: where the oracle reports every decision
of a block at a relative distance above 1e-4 from its threshold the results
must be identical; closer draws must still land in the token's own interval
of the running sum (within 1e-5), and blocks whose acceptance tests sit on a
threshold are left out (at most a few per cent of them).

Page: "MiMo-V2.5-Pro-FP4-DFlash" (alphaneural mirror), section 3: blocks of at
most 8 drafted tokens, verified in one step of the backbone.
"""
import numpy as np
import pytest
import torch

import datagen
import oracle

pytestmark = pytest.mark.gpu
DEV = "cuda"
MARGIN = 1e-4


def run_gpu(mx, z, w, d, u, tau):
    B, K1, V = z.shape
    K = K1 - 1
    zt = torch.from_numpy(z).to(DEV)
    wt = torch.from_numpy(w).to(DEV) if tau > 0 else None
    dt = torch.from_numpy(d).to(DEV)
    ut = torch.from_numpy(u).to(DEV)
    acc = torch.full((B,), -7, dtype=torch.int32, device=DEV)
    tok = torch.full((B, K + 1), -7, dtype=torch.int32, device=DEV)
    ws = torch.empty(max(mx.mxmoe_verify_workspace_size(B, K, V), 1), dtype=torch.uint8, device=DEV)
    mx.mxmoe_verify_block(zt, wt, dt, ut, tau, acc, tok, ws)
    torch.cuda.synchronize()
    return acc.cpu().numpy(), tok.cpu().numpy()


def check(mx, z, w, d, u, tau, max_skipped=0.1):
    B, K1, V = z.shape
    K = K1 - 1
    a_ref, t_ref, m_acc, m_draw = oracle.verify_block(z, w if tau > 0 else None, d, u, tau)
    a, t = run_gpu(mx, z, w, d, u, tau)
    if tau == 0:
        np.testing.assert_array_equal(a, a_ref)
        np.testing.assert_array_equal(t, t_ref)
        return a_ref
    skipped = 0
    for b in range(B):
        if m_acc[b] <= MARGIN:
            skipped += 1
            continue
        assert a[b] == a_ref[b], (b, a[b], a_ref[b])
        n = a[b]
        assert t[b, :n].tolist() == t_ref[b, :n].tolist() and (t[b, n + 1:] == -1).all()
        if m_draw[b] > MARGIN:
            assert t[b, n] == t_ref[b, n], (b, t[b, n], t_ref[b, n])
        else:  # a draw next to a boundary: the GPU's token must still hold u_K in its interval
            lo, hi = oracle.draw_interval(z[b, n], w[b, n] if n < K else None, tau, int(t[b, n]))
            assert lo - 1e-5 <= u[b, K] <= hi + 1e-5, (b, lo, hi, u[b, K])
    assert skipped <= max(1, max_skipped * B), skipped
    return a_ref


@pytest.mark.parametrize("B,K,V,tau", [(5, 3, 50, 0.0), (5, 3, 50, 1.0), (37, 8, 1000, 1.0), (37, 8, 1000, 0.0),
                                       (9, 8, 20011, 1.0), (9, 8, 20011, 0.0), (3, 1, 8192, 0.7), (4, 2, 8193, 1.3),
                                       (16, 8, 33000, 0.5), (3, 32, 500, 1.0), (3, 32, 500, 0.0)])
def test_verify_matches_oracle(mx, B, K, V, tau):
    z, w, d, u = datagen.make_verify_inputs(B, K, V, seed=B * 131 + V)
    check(mx, z, w, d, u, tau)


def test_verify_draw_beyond_one_round_of_chunks(mx):
    # V just above 2^21 = 256 chunks of 8192: the draw's chunk scan carries its
    # running sum across rounds of 256 chunks, and the first chunk of the second
    # round is searched
    V = (1 << 21) + 8193
    z, w, d, u = datagen.make_verify_inputs(1, 2, V, seed=21)
    check(mx, z, w, d, u, 1.0)
    # a flat row (every weight equal) with u_K near 1 puts the draw in the last chunks
    z2 = np.zeros_like(z)
    w2 = np.zeros_like(w)
    u2 = u.copy()
    u2[:, -1] = np.float32(0.9999)
    check(mx, z2, w2, d, u2, 1.0)


@pytest.mark.parametrize("B,tau", [(32, 1.0), (32, 0.0), (1, 1.0), (1, 0.0)])
def test_verify_full_size(mx, B, tau):
    # V = 152064, K = 8: one block (8 tokens) and 32 blocks (256 tokens)
    z, w, d, u = datagen.make_verify_inputs(B, 8, datagen.VERIFY_VOCAB, seed=7 + B)
    a = check(mx, z, w, d, u, tau)
    assert 0 <= a.min() and a.max() <= 8


def test_verify_edge_cases(mx):
    rng = np.random.default_rng(3)
    B, K, V = 6, 4, 3000
    z = rng.standard_normal((B, K + 1, V)).astype(np.float32)
    w = (z[:, :K] + 0.3 * rng.standard_normal((B, K, V))).astype(np.float32)
    d = np.argmax(w, axis=2).astype(np.int32)
    d[0, 1] = -1          # out of range: rejected at position 1
    d[1, 0] = V           # out of range: rejected at position 0
    z[2] = 0.0            # all-equal logits: greedy argmax is token 0
    w[2] = 0.0            # and p = q: every draft accepted when sampling
    d[2] = 0
    z[3, :, 100:] = -np.inf  # a masked vocabulary: only the first 100 tokens can be drawn
    w[3, :, 100:] = -np.inf
    d[3] = np.argmax(w[3], axis=1)
    u = rng.random((B, K + 1)).astype(np.float32)
    for tau in (0.0, 1.0):
        check(mx, z, w, d, u, tau, max_skipped=0.5)
        a, t = run_gpu(mx, z, w, d, u, tau)
        assert a[0] <= 1 and a[1] == 0
        assert a[2] == K  # flat rows: token 0 is every argmax (lowest index), and p = q accepts every draft
        if tau == 0.0:
            assert t[2, K] == 0
        n = a[3]
        assert 0 <= t[3, n] < 100


def test_verify_is_deterministic(mx):
    z, w, d, u = datagen.make_verify_inputs(8, 8, 50000, seed=99)
    r1 = run_gpu(mx, z, w, d, u, 1.0)
    r2 = run_gpu(mx, z, w, d, u, 1.0)
    np.testing.assert_array_equal(r1[0], r2[0])
    np.testing.assert_array_equal(r1[1], r2[1])
