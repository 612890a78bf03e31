"""Failure detection on the GPU without a fault: a bounded wait that runs out
(a barrier nothing arrives on) is reported through the device status word,
the context stays usable, and host-side errors enqueue nothing."""
import ctypes

import pytest
import torch

import attention_free_long_b200 as av
import synthetic as sy

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives(cuda_dev):
    L = av.lib()
    L.avey_selftest_wait_timeout.argtypes = [ctypes.c_uint32, ctypes.c_void_p]
    L.avey_selftest_wait_timeout.restype = ctypes.c_int
    assert av.device_status() == 0
    assert L.avey_selftest_wait_timeout(20000, None) == 0  # 20 ms limit
    assert av.device_status() == 4  # AVEY_ERR_DEVICE_TIMEOUT
    assert av.device_status() == 0  # read-and-clear
    # the context is still usable: a normal ranker call succeeds afterwards
    wl = sy.custom(B=1, N=512, S=64, d=64, k=3, centers=4)
    x = torch.from_numpy(sy.gen_embeddings(wl).X).to(cuda_dev, torch.bfloat16)
    idx, w = av.avey_rank(x, wl.S, wl.k)
    torch.cuda.synchronize()
    assert av.device_status() == 0
    assert (w[..., 0] == 1.0).all()


def test_out_of_range_candidates_are_reported_not_followed(cuda_dev):
    wl = sy.custom(B=1, N=256, S=64, d=64, k=2, centers=2)
    x = torch.from_numpy(sy.gen_embeddings(wl).X).to(cuda_dev, torch.bfloat16)
    P = torch.zeros((wl.S, (wl.k + 1) * wl.S), dtype=torch.bfloat16, device=cuda_dev)
    idx = torch.full((1, wl.n, wl.k), 99, dtype=torch.int32, device=cuda_dev)  # n = 4
    w = torch.ones((1, wl.n, wl.k), dtype=torch.float32, device=cuda_dev)
    out, _ = av.avey_compress(x, wl.S, wl.k, idx, w, P)
    torch.cuda.synchronize()
    assert av.device_status() == 5  # AVEY_ERR_DEVICE_BOUNDS
    # P = 0: the output is the residual X_t alone
    torch.testing.assert_close(out.view(-1, wl.d), x.view(-1, wl.d).float(), rtol=0, atol=0)


def test_host_rejection_enqueues_nothing(cuda_dev):
    before = av.kernel_launches()
    x = torch.zeros((1, 100, 60), dtype=torch.bfloat16, device=cuda_dev)  # d % 8 != 0
    with pytest.raises(av.AveyError) as e:
        av.avey_rank(x, 16, 3)
    assert e.value.code == 1
    assert av.kernel_launches() == before
