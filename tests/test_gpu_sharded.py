"""One long sequence split across GPUs, emulated in one process on one GPU.

Each rank's share runs through the C ABI exactly as it would on its own GPU;
the all-reduce of the score partials is emulated by summing them (the ranks'
kernels never wait on one another).  The unsharded forward is the reference:
every score entry comes from the same tile and every output row from the same
per-split arithmetic, so the sharded result must be identical bit for bit.
The unsharded path itself is checked against the oracle in test_gpu_parity.
"""
import numpy as np
import pytest
import torch

import attention_free_long_b200 as av
import synthetic as sy

pytestmark = pytest.mark.gpu

WL = [
    sy.custom("sh_s64", B=2, N=3000, S=64, d=128, m=256, k=5, pattern=(sy.STATIC, sy.DYNAMIC),
              centers=16, sigma=0.5),
    sy.custom("sh_s32_pre", B=1, N=5000, S=32, d=96, m=192, m_h=64, k=7,
              pattern=(sy.DYNAMIC, sy.STATIC, sy.DYNAMIC), centers=24, sigma=0.5, prenorm=True),
    sy.custom("sh_s128", B=1, N=2500, S=128, d=64, m=128, k=3, pattern=(sy.STATIC,), centers=6,
              sigma=0.5),
]


@pytest.mark.parametrize("world", [2, 3, 8])
@pytest.mark.parametrize("wl", WL, ids=lambda w: w.name)
def test_sharded_forward_equals_unsharded(wl, world, cuda_dev):
    E, W = sy.gen_embeddings(wl), sy.gen_weights(wl)
    x = torch.from_numpy(E.X).to(cuda_dev, torch.bfloat16)
    P = torch.from_numpy(W.P).to(cuda_dev, torch.bfloat16)
    layers = av.device_layers(W, torch.bfloat16, cuda_dev)
    ref = av.encoder_forward(x, P, layers, wl.S, wl.k, wl.m_h, wl.eps, wl.prenorm).clone()
    _, _, ref_scores = av.avey_rank(x, wl.S, wl.k, return_scores=True)
    n = wl.n
    # phase 1 on every rank, then the emulated all-reduce
    partials = []
    for r in range(world):
        sc = torch.zeros((wl.B, n, n), dtype=torch.float32, device=cuda_dev)
        av.avey_maxsim_part(x, wl.S, r, world, sc)
        partials.append(sc)
    total = torch.stack(partials).sum(0)
    torch.cuda.synchronize()
    assert torch.equal(total, ref_scores)
    # every entry is owned by exactly one part
    owned = torch.stack([(p != 0) for p in partials]).sum(0)
    assert int(owned.max()) <= 1

    def allreduce(buf):
        buf.copy_(total)

    outs = []
    for r in range(world):
        out = av.encoder_forward_sharded(x, P, layers, wl.S, wl.k, wl.m_h, wl.eps, wl.prenorm, r,
                                         world, allreduce)
        outs.append(out.clone())
    torch.cuda.synchronize()
    assert av.device_status() == 0
    got = torch.cat(outs, dim=1)
    assert torch.equal(got, ref)


def test_sharded_rejects_bad_part(cuda_dev):
    x = torch.zeros((1, 256, 64), dtype=torch.bfloat16, device=cuda_dev)
    sc = torch.zeros((1, 4, 4), dtype=torch.float32, device=cuda_dev)
    before = av.kernel_launches()
    with pytest.raises(av.AveyError):
        av.avey_maxsim_part(x, 64, 2, 2, sc)
    with pytest.raises(av.AveyError):
        av.avey_maxsim_part(x, 16, 0, 1, sc)  # the sharded MaxSim needs S >= 32
    assert av.kernel_launches() == before
