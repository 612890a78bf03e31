"""GPU vs fp64 oracle parity, through the C ABI (via the thin binding).

Small shapes are compared in full; they span several tiles, ragged token
tails (N not a multiple of S), contraction tails (d not a multiple of 64),
partial output tiles, k > n-1 and sequences shorter than one split.  The five named workloads run at full size
in the same launch configuration as the benchmark; the oracle checks a seeded
sample of target splits (a split's scores, selection, compression and layer
outputs depend only on its own row of scores and its retrieved splits, so the
sample is exact, not approximate).
"""
import dataclasses

import numpy as np
import pytest
import torch

import attention_free_long_b200 as av
import oracle as orc
import synthetic as sy
from tests.parity import TOL, check_topk, degenerate_rows, oracle_selection, rel_err

pytestmark = pytest.mark.gpu


def _tdtype(wl):
    return torch.bfloat16 if wl.dtype == "bf16" else torch.float32


def _rows_of(wl, sel):
    """Row indices of the padded [B*n*S] token axis for the selected splits."""
    return np.concatenate([np.arange(b * wl.n * wl.S + t * wl.S, b * wl.n * wl.S + (t + 1) * wl.S)
                           for b, t in sel.tolist()])


def run_gpu(wl, E, W, sel, dev, causal=False):
    dt = _tdtype(wl)
    x = torch.from_numpy(E.X).to(dev, dtype=dt)
    P = torch.from_numpy(W.P).to(dev, dtype=dt)
    layers = av.device_layers(W, dt, dev)
    idx, w, scores = av.avey_rank(x, wl.S, wl.k, return_scores=True, causal=causal)
    outs = run_downstream(wl, x, P, layers, idx, w, sel, dev)
    torch.cuda.synchronize()
    assert av.device_status() == 0
    sb, st = torch.from_numpy(sel[:, 0]).long(), torch.from_numpy(sel[:, 1]).long()
    res = dict(idx=idx.cpu()[sb, st].numpy(), w=w.cpu()[sb, st].numpy(),
               scores=scores.cpu()[sb, st].numpy(), outs=outs,
               idx_full=idx.cpu().numpy(), idx_dev=idx, w_dev=w, x=x, P=P, layers=layers)
    return res


def run_downstream(wl, x, P, layers, idx, w, sel, dev):
    """avey_compress, then every avey_layer_forward, on the selection idx / w;
    returns the sampled rows after each call (compression first)."""
    out, pair = av.avey_compress(x, wl.S, wl.k, idx, w, P)
    rows = torch.from_numpy(_rows_of(wl, sel)).to(dev)
    cur, cp = out.view(-1, wl.d), pair
    outs = [cur.index_select(0, rows).cpu().numpy()]
    for lay in layers:
        cur, cp = av.avey_layer_forward(lay, wl.S, wl.m_h, wl.eps, wl.prenorm, cur, cp)
        outs.append(cur.index_select(0, rows).cpu().numpy())
    torch.cuda.synchronize()
    assert av.device_status() == 0
    return outs


def compare(wl, E, W, sel, dev, causal=False):
    """Scores and selection against the oracle, then compression and every
    layer twice: end to end on the GPU's own selection (rows whose list
    matches the oracle's), and on the oracle's selection (every row)."""
    g = run_gpu(wl, E, W, sel, dev, causal)
    o = orc.forward(E.X, W, wl, sel=sel, causal=causal)
    tol = TOL[wl.dtype]
    assert rel_err(g["scores"], o["scores"]) <= tol, "scores"
    exact = check_topk(g["idx"], g["w"], o["idx"], o["scores"], sel[:, 1], tol)
    # a best score <= 0 makes the weights divide by the 1e-30 floor: such a
    # split's compressed output is meaningless, so it is not compared further
    degen = degenerate_rows(o["idx"], o["scores"])
    if not causal:
        assert not degen.any(), "a bidirectional row with a best score <= 0"
    valid = ~degen
    ref = [o["compressed"].reshape(-1, wl.d)] + [a.reshape(-1, wl.d) for a in o["layers"]]
    # (1) the product's own selection, on the rows whose list is the oracle's
    keep = np.repeat(exact & valid, wl.S)
    errs = [rel_err(gg[keep], oo[keep]) for gg, oo in zip(g["outs"], ref)]
    for i, e in enumerate(errs):
        assert e <= tol, f"own selection, stage {i} (0 = compression, then layers): err {e:.3g}"
    # (2) the GPU's compression and layers on the oracle's selection, every row
    idx2, w2 = oracle_selection(g["idx_dev"], g["w_dev"], sel, o["idx"], o["w"])
    outs2 = run_downstream(wl, g["x"], g["P"], g["layers"], idx2, w2, sel, dev)
    keep2 = np.repeat(valid, wl.S)
    errs2 = [rel_err(gg[keep2], oo[keep2]) for gg, oo in zip(outs2, ref)]
    for i, e in enumerate(errs2):
        assert e <= tol, f"oracle selection, stage {i} (0 = compression, then layers): err {e:.3g}"
    n_rows = sel.shape[0]
    assert int(valid.sum()) + int(degen.sum()) == n_rows
    print(f"{wl.name}: {n_rows} target splits; {int((~exact).sum())} near-tie lists; "
          f"{int(degen.sum())} degenerate; {int(valid.sum())} compared downstream on the oracle's "
          f"selection, {int((exact & valid).sum())} also on the GPU's own")
    return g, o, errs + errs2


SMALL = [
    sy.custom("f32_s8", B=2, N=100, S=8, d=32, m=48, m_h=24, k=4, pattern=(sy.STATIC, sy.DYNAMIC),
              dtype="f32", centers=6, sigma=0.4),
    sy.custom("f32_s16_pre", B=1, N=250, S=16, d=64, m=128, k=3, pattern=(sy.DYNAMIC, sy.STATIC),
              dtype="f32", centers=8, sigma=0.3, prenorm=True),
    sy.custom("bf16_s16", B=3, N=777, S=16, d=64, m=128, k=3, pattern=(sy.STATIC, sy.DYNAMIC),
              centers=24, sigma=0.3),
    sy.custom("bf16_s32", B=2, N=2053, S=32, d=96, m=192, m_h=64, k=7,
              pattern=(sy.DYNAMIC, sy.STATIC), centers=32, sigma=0.5),
    sy.custom("bf16_s64_ragged", B=2, N=1000, S=64, d=136, m=272, m_h=136, k=5,
              pattern=(sy.STATIC, sy.DYNAMIC), centers=8, sigma=0.5),
    sy.custom("bf16_s128_pre", B=1, N=3000, S=128, d=128, m=256, k=15,
              pattern=(sy.STATIC, sy.DYNAMIC, sy.STATIC), centers=12, sigma=0.5, prenorm=True),
    sy.custom("bf16_k_gt_n", B=2, N=200, S=64, d=64, m=128, k=7, pattern=(sy.DYNAMIC,),
              centers=2, sigma=0.5),
    # compression with P streamed per block (k + 1 > 8 at S = 64) and S = 128 with few blocks
    sy.custom("bf16_s64_k9", B=2, N=1500, S=64, d=192, m=256, k=9, pattern=(sy.STATIC, sy.DYNAMIC),
              centers=10, sigma=0.5),
    sy.custom("bf16_s128_k3", B=1, N=2000, S=128, d=256, m=256, k=3, pattern=(sy.DYNAMIC,),
              centers=6, sigma=0.5),
    # an odd number of blocks per tile at S = 64, where compression takes the
    # blocks two per ring stage: the last group holds one block (P resident
    # for k + 1 = 5, streamed per block for k + 1 = 11)
    sy.custom("bf16_s64_k4", B=2, N=1300, S=64, d=128, m=256, k=4, pattern=(sy.STATIC, sy.DYNAMIC),
              centers=8, sigma=0.5),
    sy.custom("bf16_s64_k10", B=1, N=1500, S=64, d=192, m=256, k=10, pattern=(sy.DYNAMIC,),
              centers=6, sigma=0.5),
    # the largest k the ranker takes: 33 blocks per target (the target and 32
    # candidates) for compression
    sy.custom("bf16_s64_k32", B=1, N=2560, S=64, d=64, m=128, k=32, pattern=(sy.DYNAMIC,),
              centers=4, sigma=0.5),
    sy.custom("bf16_s128_k32", B=1, N=4608, S=128, d=128, m=256, k=32, pattern=(sy.STATIC,),
              centers=4, sigma=0.5),
    # 16 < k + 1 <= 32 (the 32-block lists) at S = 64 and 128, and large k on
    # the smaller splits' kernel
    sy.custom("bf16_s64_k20", B=1, N=1920, S=64, d=128, m=256, k=20, pattern=(sy.STATIC,),
              centers=4, sigma=0.5),
    sy.custom("bf16_s128_k24", B=1, N=3840, S=128, d=128, m=256, k=24, pattern=(sy.DYNAMIC,),
              centers=4, sigma=0.5),
    sy.custom("bf16_s32_k32", B=1, N=1280, S=32, d=96, m=192, m_h=64, k=32, pattern=(sy.DYNAMIC,),
              centers=4, sigma=0.5),
    sy.custom("bf16_s16_k20", B=2, N=480, S=16, d=64, m=128, k=20, pattern=(sy.STATIC,),
              centers=4, sigma=0.4),
    # the narrowest widths the layer takes: an 8-feature head, an 8-feature
    # tail (the contextualized part), and d = 8
    sy.custom("bf16_head8", B=1, N=700, S=64, d=64, m=144, m_h=8, k=3,
              pattern=(sy.STATIC, sy.DYNAMIC), centers=4, sigma=0.5),
    sy.custom("bf16_tail8", B=1, N=700, S=32, d=64, m=72, m_h=64, k=3,
              pattern=(sy.DYNAMIC, sy.STATIC), centers=4, sigma=0.5),
    sy.custom("bf16_d8", B=1, N=300, S=16, d=8, m=16, m_h=8, k=2, pattern=(sy.DYNAMIC,),
              centers=3, sigma=0.4),
    # sequences shorter than one split (n = 1): no candidate anywhere, eq. 8
    # keeps the target's own block alone
    sy.custom("bf16_one_split", B=2, N=40, S=64, d=64, m=128, k=3, pattern=(sy.STATIC, sy.DYNAMIC),
              centers=2, sigma=0.5),
    sy.custom("bf16_s16_one_split", B=3, N=16, S=16, d=64, m=128, k=2,
              pattern=(sy.DYNAMIC, sy.STATIC), centers=2),
    sy.custom("f32_one_split", B=1, N=5, S=8, d=32, m=48, m_h=24, k=2, pattern=(sy.DYNAMIC,),
              dtype="f32"),
]


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
def test_small_shapes_full(wl, cuda_dev):
    E, W = sy.gen_embeddings(wl), sy.gen_weights(wl)
    compare(wl, E, W, orc.all_targets(wl.B, wl.n), cuda_dev)


def _small(name):
    return next(w for w in SMALL if w.name == name)


def test_rank_scores_optional_and_padding(cuda_dev):
    wl = _small("bf16_k_gt_n")  # k > n - 1: the lists end in padding
    assert wl.k > wl.n - 1
    E = sy.gen_embeddings(wl)
    x = torch.from_numpy(E.X).to(cuda_dev, dtype=torch.bfloat16)
    i1, w1 = av.avey_rank(x, wl.S, wl.k)
    i2, w2, _ = av.avey_rank(x, wl.S, wl.k, return_scores=True)
    assert torch.equal(i1, i2) and torch.equal(w1, w2)
    assert (i1[:, :, wl.n - 1:] == -1).all() and (w1[:, :, wl.n - 1:] == 0).all()


@pytest.mark.parametrize("name", ["tiny_f32", "base_bf16"])
def test_named_workloads_full(name, cuda_dev):
    wl = sy.WORKLOADS[name]
    E, W = sy.gen_embeddings(wl), sy.gen_weights(wl)
    compare(wl, E, W, orc.all_targets(wl.B, wl.n), cuda_dev)


@pytest.mark.parametrize("name,per_seq", [("mid_bf16", 24), ("long_bf16", 48), ("large_bf16", 32)])
def test_named_workloads_sampled(name, per_seq, cuda_dev):
    wl = sy.WORKLOADS[name]
    E, W = sy.gen_embeddings(wl), sy.gen_weights(wl)
    must = [(b, t) for b in range(wl.B) for t, _ in E.dup_pairs[b]]
    sel = sy.sample_targets(wl, per_seq, must=must)
    g, o, _ = compare(wl, E, W, sel, cuda_dev)
    # planted exact duplicates: the copy is the top-1 choice, bit-exact index
    pos = {(int(b), int(t)): r for r, (b, t) in enumerate(sel.tolist())}
    for b in range(wl.B):
        for t, s in E.dup_pairs[b]:
            assert g["idx"][pos[(b, t)], 0] == s
            assert abs(g["scores"][pos[(b, t)], s] - wl.S) <= 1e-2 * wl.S


@pytest.mark.parametrize("dtype", ["bf16x2", "f32"])
@pytest.mark.parametrize("S", [16, 32, 64, 128])
def test_dynamic_mix_entry_point(dtype, S, cuda_dev):
    if dtype == "f32" and S > 64:
        pytest.skip("fp32 path covers S <= 64")
    rng = np.random.default_rng(S)
    blocks, mt, ld = 5, 200, 208
    z = np.maximum(rng.standard_normal((blocks * S, ld)), 0).astype(np.float32) ** 2
    z[3] = 0.0  # a zero row: its weights are all zero
    ref = np.concatenate([orc.dynamic_mix(z[b * S:(b + 1) * S, :mt], 1e-8) for b in range(blocks)])
    if dtype == "f32":
        zt = torch.from_numpy(z).to(cuda_dev)
        tol = TOL["f32"]
        got = av.avey_dynamic_mix(zt, S, 1e-8, mt=mt).cpu().numpy()[:, :mt]
        inplace = av.avey_dynamic_mix(zt, S, 1e-8, mt=mt, out=zt).cpu().numpy()[:, :mt]
    else:
        hi = sy.round_bf16(z)
        lo = sy.round_bf16(z - hi)
        pair = torch.from_numpy(np.stack([hi, lo])).to(cuda_dev, torch.bfloat16).contiguous()
        # the oracle sees exactly the value the pair represents
        zrep = hi.astype(np.float64) + lo.astype(np.float64)
        ref = np.concatenate([orc.dynamic_mix(zrep[b * S:(b + 1) * S, :mt], 1e-8)
                              for b in range(blocks)])
        tol = TOL["bf16"]
        o = av.avey_dynamic_mix(pair, S, 1e-8, mt=mt)
        got = (o[0].float() + o[1].float()).cpu().numpy()[:, :mt]
        o2 = av.avey_dynamic_mix(pair, S, 1e-8, mt=mt, out=pair)
        inplace = (o2[0].float() + o2[1].float()).cpu().numpy()[:, :mt]
    torch.cuda.synchronize()
    assert av.device_status() == 0
    assert rel_err(got, ref) <= tol
    np.testing.assert_array_equal(got, inplace)


def test_kernels_launched_through_the_library(cuda_dev):
    before = av.kernel_launches()
    wl = _small("bf16_s16")
    E, W = sy.gen_embeddings(wl), sy.gen_weights(wl)
    run_gpu(wl, E, W, orc.all_targets(1, 2), cuda_dev)
    # rank: normalize + maxsim + topk; compress; per layer: enrich + mix + fuse
    assert av.kernel_launches() - before == 3 + 1 + 3 * len(W.layers)


# ---- the variants of the pages' ablations: unidirectional ranker (candidates
# c < t) and the original Avey's coupled causal contextualizer

NEXT = [
    sy.custom("uni_coupled_s64", B=2, N=1500, S=64, d=128, m=256, k=5,
              pattern=(sy.COUPLED, sy.DYNAMIC, sy.STATIC), centers=12, sigma=0.5),
    sy.custom("uni_coupled_s32", B=1, N=2000, S=32, d=96, m=192, m_h=64, k=7,
              pattern=(sy.STATIC, sy.COUPLED), centers=32, sigma=0.5),
    sy.custom("uni_coupled_f32", B=1, N=300, S=16, d=64, m=128, k=3, pattern=(sy.COUPLED,),
              dtype="f32", centers=10, sigma=0.3),
]


@pytest.mark.parametrize("wl", NEXT, ids=lambda w: w.name)
def test_unidirectional_ranker_and_coupled_layers(wl, cuda_dev):
    E, W = sy.gen_embeddings(wl), sy.gen_weights(wl)
    g, o, _ = compare(wl, E, W, orc.all_targets(wl.B, wl.n), cuda_dev, causal=True)
    idx = g["idx_full"]
    for t in range(wl.n):
        real = idx[:, t][idx[:, t] >= 0]
        assert np.all(real < t)
        assert (idx[:, t] >= 0).sum(axis=-1).max() == min(wl.k, t)
