"""Device-side failure detection without a GPU fault: a kernel's bounded wait on an
mbarrier that nothing arrives on must expire, record S2_ERR_DEVICE_TIMEOUT in the
workspace status word, and leave the CUDA context usable for the next call."""
import numpy as np
import pytest
import torch

from tests import gpu_helpers as H
from workloads import Workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def s2():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from longlora_shifted_sparse_b200 import s2attn
    return s2attn


def test_expired_wait_is_reported_and_context_survives(s2):
    w = Workload("after", 1, 1024, 4, 2, 128, 256, 2.0, "bf16", 0.5, True, seed=21)
    ws = s2.workspace(w.B, w.N, w.Hq, w.Hkv, w.d, s2.S2_BF16, torch.device("cuda"))
    stream = torch.cuda.current_stream().cuda_stream
    assert s2.s2attn_selftest_wait_timeout(ws.data_ptr(), ws.numel(), stream) == s2.S2_OK
    assert s2.device_status(ws) == s2.S2_ERR_DEVICE_TIMEOUT
    assert s2.device_status(ws) == s2.S2_OK  # reading clears it
    # the context is still usable: a normal call succeeds and reports a clean status
    q, k, v, _ = H.inputs(w, with_dout=False)
    tq, tk, tv = (H.to_device(x, "bf16") for x in (q, k, v))
    o, lse = s2.forward(tq, tk, tv, w.G, w.pi_scale, ws=ws)
    assert s2.device_status(ws) == s2.S2_OK
    assert bool(torch.isfinite(o).all()) and bool(torch.isfinite(lse).all())


def test_fma_pipe_exp2_matches_exp2(s2):
    """The polynomial exp2 that takes part of the softmax's exponentials off the MUFU unit
    agrees with exp2 to a relative 1e-4 over the range the softmax feeds it."""
    x = np.concatenate([np.linspace(-125.0, 8.0, 200001), np.arange(-125, 9, dtype=np.float64),
                        np.arange(-125, 9) + 0.5]).astype(np.float32)
    tx = torch.from_numpy(x).cuda()
    ty = torch.empty_like(tx)
    assert s2.s2attn_selftest_exp2(tx.data_ptr(), ty.data_ptr(), tx.numel(),
                                   torch.cuda.current_stream().cuda_stream) == s2.S2_OK
    torch.cuda.synchronize()
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(ty.cpu().numpy().astype(np.float64) - ref) / ref
    assert rel.max() < 1e-4, rel.max()
