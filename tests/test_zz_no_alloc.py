"""avey_rank_static, the ranker entry point for callers that cannot allocate
device memory (its scratch is a fixed array inside the library), against
avey_rank with a caller workspace.  Called through the C ABI directly, twice in
a row, on three shapes (the second call must leave device memory untouched); this file is collected last so that a run stopping at the
first failure has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import attention_free_long_b200 as av
import synthetic as sy

pytestmark = pytest.mark.gpu


def _static_fn():
    L = av.lib()
    f = L.avey_rank_static
    f.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                  ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    f.restype = ctypes.c_int
    L.avey_rank_static_max_scratch_bytes.restype = ctypes.c_size_t
    return f


@pytest.mark.parametrize("wl", [
    sy.custom("static_s64", B=2, N=3000, S=64, d=256, k=7, centers=24, sigma=0.5),
    sy.custom("static_s16_bf16", B=2, N=1500, S=16, d=128, k=5, centers=24, sigma=0.4),
    sy.custom("static_s16_f32", B=1, N=500, S=16, d=64, k=3, dtype="f32", centers=16, sigma=0.3),
], ids=lambda w: w.name)
def test_static_scratch_matches_workspace_entry_point(wl, cuda_dev):
    f = _static_fn()
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    x = torch.from_numpy(sy.gen_embeddings(wl).X).to(cuda_dev, dt)
    ref_idx, ref_w = av.avey_rank(x, wl.S, wl.k)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    code = av.AVEY_BF16 if wl.dtype == "bf16" else av.AVEY_F32
    for call in range(2):  # the second call reuses the array left by the first
        idx = torch.full_like(ref_idx, -7)
        w = torch.full_like(ref_w, -7.0)
        torch.cuda.synchronize()
        before = (torch.cuda.memory_allocated(cuda_dev), torch.cuda.mem_get_info(cuda_dev)[0])
        rc = f(ctypes.c_void_p(x.data_ptr()), code, wl.B, wl.N, wl.d, wl.S, wl.k,
               ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(w.data_ptr()), stream)
        assert rc == 0, av.lib().avey_last_error_detail().decode()
        torch.cuda.synchronize()
        after = (torch.cuda.memory_allocated(cuda_dev), torch.cuda.mem_get_info(cuda_dev)[0])
        if call == 1:
            # nothing allocated: neither through torch nor on the device
            # (the first call may still load the library's device code)
            assert after == before, (before, after)
        assert av.device_status() == 0
        assert torch.equal(idx, ref_idx)
        np.testing.assert_allclose(w.cpu().numpy(), ref_w.cpu().numpy(), rtol=1e-6, atol=0)


def test_static_scratch_rejects_oversized_shapes(cuda_dev):
    f = _static_fn()
    limit = av.lib().avey_rank_static_max_scratch_bytes()
    # n = 4096 splits: the score matrix alone is 64 MiB, beyond the array
    B, N, d, S = 1, 4096 * 16, 64, 16
    assert av.rank_workspace_bytes(av.AVEY_BF16, B, N, d, S) > limit
    x = torch.zeros((B, N, d), dtype=torch.bfloat16, device=cuda_dev)
    idx = torch.empty((B, 4096, 3), dtype=torch.int32, device=cuda_dev)
    w = torch.empty((B, 4096, 3), dtype=torch.float32, device=cuda_dev)
    rc = f(ctypes.c_void_p(x.data_ptr()), av.AVEY_BF16, B, N, d, S, 3,
           ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(w.data_ptr()), None)
    assert rc == 2  # AVEY_ERR_UNSUPPORTED, nothing enqueued
    assert "scratch" in av.lib().avey_last_error_detail().decode()
