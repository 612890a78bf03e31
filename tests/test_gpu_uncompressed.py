"""GPU vs fp64 oracle parity of the processor without neural compression.

Each split's (k+1)S-token context goes through every layer as one block
(Avey-B paperlayer summary §4.3), so the contextualizer mixes blocks of
(k+1)S tokens: 64 and 128 run on the split-size kernels, 256 and 512 on the
long-block kernels (tcgen05, Z_t read as an MN-major operand, c into its own
buffer that the fuser reads beside Z_h).  Shapes cover ragged token tails,
feature tails (m_t not a multiple of 64) and both layer kinds.  As in the compressed parity tests, the
oracle never takes the GPU's selection as input: rows whose top-k lists differ
by a near tie are left out of the layer comparison.
"""
import numpy as np
import pytest
import torch

import attention_free_long_b200 as av
import oracle as orc
import synthetic as sy
from tests.parity import TOL, check_topk, degenerate_rows, oracle_selection, rel_err

pytestmark = pytest.mark.gpu

UNCOMP = [
    sy.custom("u_f32_s16_k3", B=1, N=250, S=16, d=64, m=128, k=3, pattern=(sy.DYNAMIC, sy.STATIC),
              dtype="f32", centers=8, sigma=0.3),
    sy.custom("u_bf16_s32_k3", B=2, N=700, S=32, d=96, m=192, m_h=64, k=3,
              pattern=(sy.STATIC, sy.DYNAMIC), centers=12, sigma=0.5),
    sy.custom("u_bf16_s64_k3_ragged", B=2, N=1000, S=64, d=136, m=264, m_h=128, k=3,
              pattern=(sy.STATIC, sy.DYNAMIC), centers=8, sigma=0.5),
    sy.custom("u_bf16_s64_k7_pre", B=1, N=2048, S=64, d=128, m=256, k=7,
              pattern=(sy.DYNAMIC, sy.STATIC, sy.DYNAMIC), centers=12, sigma=0.5, prenorm=True),
    sy.custom("u_bf16_s128_k3", B=1, N=1500, S=128, d=64, m=128, k=3,
              pattern=(sy.STATIC, sy.DYNAMIC), centers=6, sigma=0.5),
]


def _tdtype(wl):
    return torch.bfloat16 if wl.dtype == "bf16" else torch.float32


@pytest.mark.parametrize("wl", UNCOMP, ids=lambda w: w.name)
def test_uncompressed_forward(wl, cuda_dev):
    E = sy.gen_embeddings(wl)
    W = sy.gen_weights(wl, block=(wl.k + 1) * wl.S)
    dt = _tdtype(wl)
    x = torch.from_numpy(E.X).to(cuda_dev, dtype=dt)
    layers = av.device_layers(W, dt, cuda_dev)
    ws = av.make_workspace(wl.B, wl.N, wl.d, wl.S, wl.k, wl.m, dt, wl.prenorm, cuda_dev,
                           uncompressed=True)
    before = av.kernel_launches()
    out = av.encoder_forward_uncompressed(x, layers, wl.S, wl.k, wl.m_h, wl.eps, wl.prenorm, ws=ws)
    torch.cuda.synchronize()
    assert av.device_status() == 0
    assert av.kernel_launches() > before
    g_out = out.cpu().numpy().reshape(-1, wl.S, wl.d)
    g_idx = ws.idx.cpu().numpy().reshape(-1, wl.k)
    g_w = ws.w.cpu().numpy().reshape(-1, wl.k)

    o = orc.forward_uncompressed(E.X, W, wl)
    assert np.array_equal(o["sel"], orc.all_targets(wl.B, wl.n))
    tol = TOL[wl.dtype]
    # every list matches the oracle's except at its near ties (check_topk)
    exact = check_topk(g_idx, g_w, o["idx"], o["scores"], o["sel"][:, 1], tol)
    valid = ~degenerate_rows(o["idx"], o["scores"])
    assert valid.all(), "a bidirectional row with a best score <= 0"
    # (1) the product's own selection, on the rows whose list is the oracle's
    err = rel_err(g_out[exact], o["out"][exact])
    assert err <= tol, f"uncompressed output err {err:.3g} > {tol} (own selection)"
    # (2) the GPU's context and layers on the oracle's selection, every row
    idx_o = torch.from_numpy(o["idx"].astype(np.int32).reshape(wl.B, wl.n, wl.k)).to(cuda_dev)
    w_o = torch.from_numpy(o["w"].astype(np.float32).reshape(wl.B, wl.n, wl.k)).to(cuda_dev)
    out2 = av.processor_forward_uncompressed(x, layers, wl.S, wl.k, wl.m_h, wl.eps, wl.prenorm,
                                             idx_o, w_o, ws=ws)
    torch.cuda.synchronize()
    assert av.device_status() == 0
    err2 = rel_err(out2.cpu().numpy().reshape(-1, wl.S, wl.d), o["out"])
    assert err2 <= tol, f"uncompressed output err {err2:.3g} > {tol} (oracle selection)"
    print(f"{wl.name}: {exact.size} target splits; {int((~exact).sum())} near-tie lists; "
          f"all compared on the oracle's selection, {int(exact.sum())} also on the GPU's own")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_context_entry_is_exact(dtype, cuda_dev):
    # fed the oracle's own selection (with the weights rounded to fp32, the
    # width the ABI takes): every value is w * x, one correctly rounded fp32
    # product, so the fp32 output is bit-exact; the split pair represents it
    wl = sy.custom("ctx", B=2, N=333, S=16, d=40, m=48, m_h=24, k=5, pattern=(sy.STATIC,), dtype=dtype,
                   centers=5, sigma=0.4)
    E = sy.gen_embeddings(wl)
    sel, _, oidx, ow = orc.rank(E.X, wl.S, wl.k)
    w32 = ow.astype(np.float32)
    oidx = oidx.copy()
    oidx[::7, -1] = -1  # missing candidates give zero blocks
    ref = orc.context(E.X, wl.S, wl.k, sel, oidx, w32.astype(np.float64)).astype(np.float32)
    dt = _tdtype(wl)
    x = torch.from_numpy(E.X).to(cuda_dev, dtype=dt)
    idx = torch.from_numpy(oidx.reshape(wl.B, wl.n, wl.k)).to(cuda_dev)
    w = torch.from_numpy(w32.reshape(wl.B, wl.n, wl.k)).to(cuda_dev)
    out, pair = av.avey_context(x, wl.S, wl.k, idx, w)
    torch.cuda.synchronize()
    assert av.device_status() == 0
    g = out.cpu().numpy().reshape(-1, (wl.k + 1) * wl.S, wl.d)
    np.testing.assert_array_equal(g, ref)
    if dtype == "bf16":
        p = pair.float().cpu().numpy().astype(np.float64)
        rec = (p[0] + p[1]).reshape(g.shape)
        assert np.all(np.abs(rec - g) <= 2.0 ** -16 * np.abs(g) + 1e-38)
    else:
        assert pair is None


def test_context_rejects_out_of_range_index(cuda_dev):
    wl = sy.custom("ctx_oob", B=1, N=64, S=16, d=16, m=32, k=2, pattern=(sy.STATIC,), dtype="f32")
    E = sy.gen_embeddings(wl)
    x = torch.from_numpy(E.X).to(cuda_dev)
    idx = torch.zeros((1, wl.n, wl.k), dtype=torch.int32, device=cuda_dev)
    idx[0, 1, 1] = wl.n  # one past the last split
    w = torch.ones((1, wl.n, wl.k), dtype=torch.float32, device=cuda_dev)
    out, _ = av.avey_context(x, wl.S, wl.k, idx, w)
    torch.cuda.synchronize()
    assert av.device_status() == 5  # AVEY_ERR_DEVICE_BOUNDS
    assert av.device_status() == 0
    blk = out[0, 1, 2 * wl.S:3 * wl.S]
    assert torch.count_nonzero(blk).item() == 0


@pytest.mark.parametrize("S", [256, 512])
@pytest.mark.parametrize("kind", [sy.STATIC, sy.DYNAMIC])
def test_long_block_mix_closed_forms(kind, S, cuda_dev):
    # Closed forms independent of the oracle, on blocks of 256 / 512 tokens:
    # with U = 0 every token's Z is relu(b)^2 (identical rows), so the dynamic
    # weights are uniform, 1/(S + eps) (eq. 6), and c = S/(S + eps) relu(b_t)^2;
    # a static V = I gives c = Z_t.  An O that copies c into the residual
    # (x_out = x + c on the first m_t features) exposes c.
    blocks, d, m, m_h = 3, 64, 128, 64
    eps = 1e-3
    wl = sy.custom("lm", B=1, N=blocks * S, S=S, d=d, m=m, m_h=m_h, k=1, pattern=(kind,))
    W = sy.gen_weights(wl)
    lay = av.device_layers(W, torch.bfloat16, cuda_dev)[0]
    lay.Ut.zero_()
    b = torch.linspace(0.5, 1.5, m, device=cuda_dev)
    lay.bU.copy_(b)
    lay.Ot.zero_()
    mt = m - m_h
    for q in range(min(d, mt)):
        lay.Ot[q, m_h + q] = 1.0
    if kind == sy.STATIC:
        lay.V = torch.eye(S, dtype=torch.bfloat16, device=cuda_dev)
    x = torch.randn(blocks * S, d, device=cuda_dev)
    y, _ = av.avey_layer_forward(lay, S, m_h, eps, False, x)
    torch.cuda.synchronize()
    assert av.device_status() == 0
    z_t = (torch.relu(b[m_h:]) ** 2).double()
    c = z_t * (S / (S + eps)) if kind == sy.DYNAMIC else z_t
    expect = x.double() + c[:d].unsqueeze(0)
    torch.testing.assert_close(y.double(), expect, rtol=2e-4, atol=2e-4)


def test_long_blocks_need_head_width_multiple_of_64(cuda_dev):
    # the fuser reads [Z_h || c] from two buffers split at a K chunk of 64
    S, blocks, d, m, m_h = 256, 1, 64, 136, 72
    wl = sy.custom("lm_bad", B=1, N=blocks * S, S=S, d=d, m=m, m_h=m_h, k=1, pattern=(sy.STATIC,))
    lay = av.device_layers(sy.gen_weights(wl), torch.bfloat16, cuda_dev)[0]
    x = torch.randn(blocks * S, d, device=cuda_dev)
    before = av.kernel_launches()
    with pytest.raises(av.AveyError):
        av.avey_layer_forward(lay, S, m_h, 1e-8, False, x)
    assert av.kernel_launches() == before


def test_uncompressed_long_workload_sampled(cuda_dev):
    # the bench's workload at full size (1536 blocks of 512 tokens), in the
    # launch configuration the bench times; the oracle computes seeded target
    # splits one by one (each needs only its own score row and context)
    wl = sy.WORKLOADS["long_bf16"]
    E = sy.gen_embeddings(wl)
    W = sy.gen_weights(wl, block=(wl.k + 1) * wl.S)
    x = torch.from_numpy(E.X).to(cuda_dev, torch.bfloat16)
    layers = av.device_layers(W, torch.bfloat16, cuda_dev)
    out = av.encoder_forward_uncompressed(x, layers, wl.S, wl.k, wl.m_h, wl.eps, wl.prenorm)
    torch.cuda.synchronize()
    assert av.device_status() == 0
    sel = sy.sample_targets(wl, per_seq=16, seed=7)
    sb, st = torch.from_numpy(sel[:, 0]).long(), torch.from_numpy(sel[:, 1]).long()
    g_out = out.cpu()[sb, st].numpy()
    g_idx, g_w = av.avey_rank(x, wl.S, wl.k)
    o = orc.forward_uncompressed(E.X, W, wl, sel=sel)
    exact = check_topk(g_idx.cpu()[sb, st].numpy(), g_w.cpu()[sb, st].numpy(), o["idx"], o["scores"],
                       sel[:, 1], TOL["bf16"])
    assert not degenerate_rows(o["idx"], o["scores"]).any()
    # end to end on the GPU's own selection, rows whose list is the oracle's
    err = rel_err(g_out[exact], o["out"][exact])
    assert err <= TOL["bf16"], f"uncompressed output, own selection: err {err:.3g}"
    # every sampled row: the same processor on the oracle's selection
    del out
    idx2, w2 = oracle_selection(g_idx, g_w, sel, o["idx"], o["w"])
    out2 = av.processor_forward_uncompressed(x, layers, wl.S, wl.k, wl.m_h, wl.eps, wl.prenorm,
                                             idx2, w2)
    torch.cuda.synchronize()
    assert av.device_status() == 0
    err2 = rel_err(out2.cpu()[sb, st].numpy(), o["out"])
    assert err2 <= TOL["bf16"], f"uncompressed output, oracle selection: err {err2:.3g}"
    print(f"uncompressed long_bf16: {sel.shape[0]} sampled splits, "
          f"{int((~exact).sum())} near-tie lists, all compared")
    del out2, layers
    torch.cuda.empty_cache()
