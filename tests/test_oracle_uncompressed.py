"""Pins of the oracle's uncompressed processor path.

Without neural compression every target split is processed together with its
k weighted retrieved splits: the (k+1)S-token context [X_t ; w_1 X_c1 ; ... ;
w_k X_ck] goes through every layer as one block, and the first S rows are the
target's output (Avey-B paperlayer summary §4.3, the ablation behind the
4.37x throughput figure; papernotes 关键设计 4 for the context itself).
"""
import numpy as np
import pytest

import oracle as orc
import synthetic as sy
from tests import bruteforce as bf


def _sel_idx_w(rng, B, n, k, holes=True):
    sel = np.array([(b, t) for b in range(B) for t in range(n)], dtype=np.int32)
    idx = np.empty((sel.shape[0], k), dtype=np.int32)
    w = rng.uniform(0.1, 1.0, size=(sel.shape[0], k))
    for r, (b, t) in enumerate(sel.tolist()):
        others = [c for c in range(n) if c != t]
        pick = rng.choice(others, size=min(k, len(others)), replace=False).tolist()
        if holes and r % 3 == 0 and k > 1:
            pick[-1] = -1
        idx[r] = pick + [-1] * (k - len(pick))
    return sel, idx, w


@pytest.mark.parametrize("N,S,k", [(22, 4, 2), (37, 8, 3), (16, 4, 3)])
def test_context_matches_bruteforce(N, S, k):
    rng = np.random.default_rng(N * 10 + k)
    B, d = 2, 5
    X = rng.standard_normal((B, N, d))
    n = -(-N // S)
    sel, idx, w = _sel_idx_w(rng, B, n, k)
    ctx = orc.context(X, S, k, sel, idx, w)
    assert ctx.shape == (sel.shape[0], (k + 1) * S, d)
    Xl = X.tolist()
    for r, (b, t) in enumerate(sel.tolist()):
        ref = bf.context(Xl, S, k, b, t, idx[r].tolist(), w[r].tolist())
        np.testing.assert_array_equal(ctx[r], np.array(ref))


def test_context_times_P_plus_residual_is_the_compressor():
    # eq. 8: X_hat = P X_cat, plus the residual X_t; the compressor is pinned on
    # its own (hand example, identity / zero P, brute force)
    rng = np.random.default_rng(5)
    B, N, S, k, d = 2, 30, 5, 3, 7
    X = rng.standard_normal((B, N, d))
    n = -(-N // S)
    sel, idx, w = _sel_idx_w(rng, B, n, k)
    P = rng.standard_normal((S, (k + 1) * S))
    ctx = orc.context(X, S, k, sel, idx, w)
    comp = orc.compress(X, S, k, sel, idx, w, P)
    ref = np.einsum("ij,rjq->riq", P, ctx) + ctx[:, :S, :]
    np.testing.assert_allclose(comp, ref, rtol=1e-12, atol=1e-12)


def test_default_block_keeps_every_draw():
    w = sy.custom(B=1, N=64, S=8, d=12, m=16, m_h=8, k=3, pattern=(sy.STATIC, sy.DYNAMIC, sy.STATIC),
                  dtype="f32")
    a, b = sy.gen_weights(w), sy.gen_weights(w, block=w.S)
    c = sy.gen_weights(w, block=(w.k + 1) * w.S)
    np.testing.assert_array_equal(a.P, c.P)
    for la, lb, lc in zip(a.layers, b.layers, c.layers):
        np.testing.assert_array_equal(la.U, lb.U)
        np.testing.assert_array_equal(la.U, lc.U)
        np.testing.assert_array_equal(la.O, lc.O)
        if la.V is not None:
            np.testing.assert_array_equal(la.V, lb.V)
            assert lc.V.shape == ((w.k + 1) * w.S, (w.k + 1) * w.S)


@pytest.mark.parametrize("pattern,prenorm", [((sy.STATIC, sy.DYNAMIC), False),
                                             ((sy.DYNAMIC, sy.STATIC), True)])
def test_uncompressed_forward_matches_bruteforce(pattern, prenorm):
    w = sy.custom(B=2, N=22, S=4, d=6, m=8, m_h=3, k=2, pattern=pattern, dtype="f32", centers=3,
                  sigma=0.4, prenorm=prenorm)
    E = sy.gen_embeddings(w)
    W = sy.gen_weights(w, block=(w.k + 1) * w.S)
    res = orc.forward_uncompressed(E.X, W, w)
    Xl = E.X.astype(np.float64).tolist()
    sc = bf.maxsim_matrix(Xl, w.S)
    for r, (b, t) in enumerate(res["sel"].tolist()):
        idx, wt = bf.topk(sc[b][t], t, w.k)
        assert res["idx"][r].tolist() == idx
        x = bf.context(Xl, w.S, w.k, b, t, idx, wt)
        for lw in W.layers:
            x = bf.layer(x, lw.U.tolist(), lw.bU.tolist(),
                         None if lw.V is None else lw.V.tolist(), lw.O.tolist(), w.m_h, lw.kind,
                         w.eps, w.prenorm)
        np.testing.assert_allclose(res["layers"][-1][r], np.array(x), rtol=1e-10, atol=1e-10)
        np.testing.assert_allclose(res["out"][r], np.array(x[:w.S]), rtol=1e-10, atol=1e-10)


def test_block_diagonal_static_stack_reduces_to_the_split_processor():
    # With only static layers whose (k+1)S x (k+1)S map does not couple the
    # target block to the retrieved blocks (V' = blockdiag(V, R)), the target
    # rows see nothing but X_t: the output equals the per-split processor run on
    # the uncompressed target split with V.
    w = sy.custom(B=1, N=48, S=4, d=6, m=8, m_h=4, k=3, pattern=(sy.STATIC, sy.STATIC), dtype="f32",
                  centers=3, sigma=0.4)
    E = sy.gen_embeddings(w)
    L = (w.k + 1) * w.S
    Wb = sy.gen_weights(w, block=L)
    rng = np.random.default_rng(9)
    small = []
    for lw in Wb.layers:
        V = lw.V[:w.S, :w.S].copy()
        Vb = np.zeros((L, L), dtype=lw.V.dtype)
        Vb[:w.S, :w.S] = V
        Vb[w.S:, w.S:] = rng.standard_normal((L - w.S, L - w.S))
        Vb[w.S:, :w.S] = rng.standard_normal((L - w.S, w.S))  # the retrieved rows may read X_t
        lw.V = Vb
        small.append(sy.LayerWeights(lw.kind, lw.U, lw.bU, V, lw.O))
    res = orc.forward_uncompressed(E.X, Wb, w)
    n = w.n
    X = E.X.astype(np.float64)
    xs = np.zeros((n, w.S, w.d))
    for t in range(n):
        rows = X[0, t * w.S:min((t + 1) * w.S, w.N)]
        xs[t, :rows.shape[0]] = rows
    for lw in small:
        xs = orc.layer(xs, lw, w.S, w.m_h, w.eps, w.prenorm)
    np.testing.assert_allclose(res["out"], xs[res["sel"][:, 1]], rtol=1e-12, atol=1e-12)
