"""The single-kernel entry points avey_static_mix and avey_topk against the
oracle, through the C ABI.  Each runs the kernel that the layer and the ranker
launch internally (static_mix_tc / static_mix_f32, topk_warp)."""
import numpy as np
import pytest
import torch

import attention_free_long_b200 as av
import oracle as orc
import synthetic as sy
from tests.parity import TOL, rel_err

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("S", [16, 32, 64, 128])
def test_static_mix_entry_point(dtype, S, cuda_dev):
    if dtype == "f32" and S > 64:
        pytest.skip("fp32 path covers S <= 64")
    rng = np.random.default_rng(100 + S)
    blocks, mt, ld = 5, 200, 208
    z = np.maximum(rng.standard_normal((blocks * S, ld)), 0).astype(np.float32) ** 2
    V = (rng.standard_normal((S, S)) / np.sqrt(S)).astype(np.float32)
    if dtype == "f32":
        Vd = torch.from_numpy(V).to(cuda_dev)
        zt = torch.from_numpy(z).to(cuda_dev)
        ref = np.concatenate([orc.static_mix(V, z[b * S:(b + 1) * S, :mt]) for b in range(blocks)])
        got = av.avey_static_mix(Vd, zt, S, mt=mt).cpu().numpy()[:, :mt]
        inplace = av.avey_static_mix(Vd, zt, S, mt=mt, out=zt).cpu().numpy()[:, :mt]
        tol = TOL["f32"]
    else:
        Vb = sy.round_bf16(V)
        hi = sy.round_bf16(z)
        lo = sy.round_bf16(z - hi)
        pair = torch.from_numpy(np.stack([hi, lo])).to(cuda_dev, torch.bfloat16).contiguous()
        Vd = torch.from_numpy(Vb).to(cuda_dev, torch.bfloat16)
        zrep = hi.astype(np.float64) + lo.astype(np.float64)
        ref = np.concatenate([orc.static_mix(Vb, zrep[b * S:(b + 1) * S, :mt]) for b in range(blocks)])
        o = av.avey_static_mix(Vd, pair, S, mt=mt)
        got = (o[0].double() + o[1].double()).cpu().numpy()[:, :mt]
        o2 = av.avey_static_mix(Vd, pair, S, mt=mt, out=pair)
        inplace = (o2[0].double() + o2[1].double()).cpu().numpy()[:, :mt]
        tol = TOL["bf16"]
    torch.cuda.synchronize()
    assert av.device_status() == 0
    assert rel_err(got, ref) <= tol
    np.testing.assert_array_equal(got, inplace)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n,k", [(37, 5), (300, 7), (1, 3), (4, 7), (301, 12), (64, 20), (2053, 32)])
def test_topk_entry_point(n, k, causal, cuda_dev):
    # The kernel and the oracle rank the same fp32 scores (the oracle widened
    # to fp64): the ordered index lists agree bit for bit, ties included
    # (planted), and w = s_r / s_1 is one fp32 division.
    rng = np.random.default_rng(n * 10 + k)
    B = 3
    sc = rng.uniform(0.0, 10.0, size=(B, n, n)).astype(np.float32)
    if n > 10:
        sc[0, 5, 7] = sc[0, 5, 9]  # exact tie: the lower index wins
        sc[1, 2, :] = 3.0          # a row of equal scores
    g_idx, g_w = av.avey_topk(torch.from_numpy(sc).to(cuda_dev), k, causal=causal)
    torch.cuda.synchronize()
    assert av.device_status() == 0
    g_idx, g_w = g_idx.cpu().numpy(), g_w.cpu().numpy()
    rows = sc.reshape(B * n, n).astype(np.float64)
    targets = np.tile(np.arange(n, dtype=np.int32), B)
    o_idx, o_w = orc.topk(rows, targets, k, causal)
    np.testing.assert_array_equal(g_idx.reshape(B * n, k), o_idx)
    np.testing.assert_allclose(g_w.reshape(B * n, k), o_w, rtol=2e-7, atol=0)


def test_smoke_entry_passes(cuda_dev):
    # the build's one-call smoke check: rank, compression and two layers on
    # cuda:0 against the oracle
    import __graft_entry__ as ge
    ge.smoke()


def test_kernel_trace_times_every_launch_of_a_forward(cuda_dev):
    wl = sy.custom("trace", B=1, N=2048, S=64, d=128, m=256, k=5,
                   pattern=(sy.STATIC, sy.DYNAMIC), centers=8, sigma=0.5)
    E, W = sy.gen_embeddings(wl), sy.gen_weights(wl)
    x = torch.from_numpy(E.X).to(cuda_dev, torch.bfloat16)
    P = torch.from_numpy(W.P).to(cuda_dev, torch.bfloat16)
    layers = av.device_layers(W, torch.bfloat16, cuda_dev)
    ws = av.make_workspace(wl.B, wl.N, wl.d, wl.S, wl.k, wl.m, torch.bfloat16, wl.prenorm, cuda_dev)
    av.encoder_forward(x, P, layers, wl.S, wl.k, wl.m_h, wl.eps, wl.prenorm, ws)
    before = av.kernel_launches()
    with av.KernelTrace(64) as tr:
        av.encoder_forward(x, P, layers, wl.S, wl.k, wl.m_h, wl.eps, wl.prenorm, ws)
    torch.cuda.synchronize()
    assert av.device_status() == 0
    ks = tr.kernels()
    assert len(ks) == av.kernel_launches() - before == 3 + 1 + 3 * len(layers)
    names = [n for n, _ in ks]
    assert names[:4] == ["inv_norms", "maxsim_pair", "topk_warp", "compress_tc"]
    assert names[4:] == ["enrich_tc", "static_mix_tc", "fuse_tc",
                         "enrich_tc", "dynamic_mix_tc", "fuse_tc"]
    assert all(ms > 0 for _, ms in ks)
    # a second trace reuses the library's events
    with av.KernelTrace(8) as tr2:
        av.avey_rank(x, wl.S, wl.k)
    torch.cuda.synchronize()
    assert [n for n, _ in tr2.kernels()] == ["inv_norms", "maxsim_pair", "topk_warp"]
