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


def _bits(t):
    return t.detach().contiguous().view(torch.uint8).cpu()


@pytest.mark.parametrize("site", ["fwd", "dkdv"])
def test_injected_missing_arrival_in_a_tensor_core_kernel(s2, site):
    """A tcgen05 kernel's own abort path: the issuer of the first CTA withholds one barrier
    arrival, so real waits inside the forward (or the dK/dV pass) expire after 50 ms. The
    call reports S2_ERR_DEVICE_TIMEOUT; every CTA drained its loads and MMAs and freed its
    TMEM, so the next normal calls on the same context reproduce, bit for bit, the results
    recorded before the injection."""
    w = Workload("inject", 1, 1024, 4, 2, 128, 256, 2.0, "bf16", 0.5, True, seed=22)
    assert s2.s2attn_kernel_path(w.B, w.N, w.Hq, w.Hkv, w.d, w.G, 1, s2.S2_BF16) == 1
    q, k, v, do = H.inputs(w)
    tq, tk, tv, tdo = (H.to_device(x, "bf16") for x in (q, k, v, do))
    ws = s2.workspace(w.B, w.N, w.Hq, w.Hkv, w.d, s2.S2_BF16, torch.device("cuda"))
    o, lse = s2.forward(tq, tk, tv, w.G, w.pi_scale, ws=ws)
    grads = s2.backward(tq, tk, tv, o, lse, tdo, w.G, w.pi_scale, ws=ws)
    assert s2.device_status(ws) == s2.S2_OK
    before = [_bits(t) for t in (o, lse) + tuple(grads)]

    stream = torch.cuda.current_stream().cuda_stream
    o2, lse2 = torch.empty_like(o), torch.empty_like(lse)
    g2 = [torch.empty_like(t) for t in grads]
    shape = (w.B, w.N, w.Hq, w.Hkv, w.d, w.G, 1, w.pi_scale, 10000.0, s2.S2_BF16)
    if site == "fwd":
        rc = s2.s2attn_selftest_inject(s2.S2_INJECT_FWD, tq.data_ptr(), tk.data_ptr(),
                                       tv.data_ptr(), o2.data_ptr(), lse2.data_ptr(),
                                       None, None, None, None, *shape, ws.data_ptr(),
                                       ws.numel(), stream)
    else:
        rc = s2.s2attn_selftest_inject(s2.S2_INJECT_DKDV, tq.data_ptr(), tk.data_ptr(),
                                       tv.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                       tdo.data_ptr(), *(t.data_ptr() for t in g2), *shape,
                                       ws.data_ptr(), ws.numel(), stream)
    assert rc == s2.S2_OK, s2.s2attn_status_string(rc)
    assert s2.device_status(ws) == s2.S2_ERR_DEVICE_TIMEOUT
    assert s2.device_status(ws) == s2.S2_OK  # reading clears it

    o3, lse3 = s2.forward(tq, tk, tv, w.G, w.pi_scale, ws=ws, check_status=True)
    grads3 = s2.backward(tq, tk, tv, o3, lse3, tdo, w.G, w.pi_scale, ws=ws, check_status=True)
    after = [_bits(t) for t in (o3, lse3) + tuple(grads3)]
    for name, a, b in zip(("o", "lse", "dq", "dk", "dv"), before, after):
        assert torch.equal(a, b), name


def test_injection_needs_the_tensor_core_path(s2):
    stream = torch.cuda.current_stream().cuda_stream
    buf = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    p = buf.data_ptr()
    # fp32 runs on the CUDA-core kernels, which have no injection site
    rc = s2.s2attn_selftest_inject(s2.S2_INJECT_FWD, p, p, p, p, p, None, None, None, None,
                                   1, 256, 4, 4, 64, 64, 1, 2.0, 10000.0, s2.S2_FP32, p,
                                   buf.numel(), stream)
    assert rc == s2.S2_ERR_ARG
    rc = s2.s2attn_selftest_inject(7, p, p, p, p, p, p, p, p, p, 1, 1024, 4, 2, 128, 256, 1,
                                   2.0, 10000.0, s2.S2_BF16, p, buf.numel(), stream)
    assert rc == s2.S2_ERR_ARG
    assert bool((buf == 0).all())


def test_autograd_backward_reports_a_forward_timeout(s2):
    """The autograd wrapper reads the forward's status word before the backward would reset
    it: a timeout recorded there raises S2Error instead of yielding silent gradients."""
    w = Workload("autograd", 1, 1024, 4, 2, 128, 256, 2.0, "bf16", 0.5, True, seed=23)
    q, k, v, do = H.inputs(w)
    tq, tk, tv, tdo = (H.to_device(x, "bf16").requires_grad_(x is not do)
                       for x in (q, k, v, do))
    o = s2.s2_attention(tq, tk, tv, w.G, w.pi_scale)
    ws = o.grad_fn.saved_tensors[5]
    stream = torch.cuda.current_stream().cuda_stream
    # records a timeout in the forward's workspace exactly as an expired wait would
    assert s2.s2attn_selftest_wait_timeout(ws.data_ptr(), ws.numel(), stream) == s2.S2_OK
    with pytest.raises(s2.S2Error) as err:
        o.backward(tdo)
    assert err.value.status == s2.S2_ERR_DEVICE_TIMEOUT
    # a clean forward + backward through the same wrapper passes its checks
    o = s2.s2_attention(tq, tk, tv, w.G, w.pi_scale)
    o.backward(tdo)
    assert bool(torch.isfinite(tq.grad).all())


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_backward_after_forward_detects_another_forwards_workspace(s2, dtype):
    """s2attn_bwd_after_fwd reuses the rotation the forward left in the workspace. A call
    whose arguments or q/k buffers differ from that forward's is caught on the device and
    reported as S2_ERR_STALE_WORKSPACE; the matching call still works afterwards."""
    w = Workload("stale", 1, 1024, 4, 2, 128, 256, 2.0, dtype, 0.5, True, seed=24)
    q, k, v, do = H.inputs(w)
    tq, tk, tv, tdo = (H.to_device(x, dtype) for x in (q, k, v, do))
    code = s2.S2_BF16 if dtype == "bf16" else s2.S2_FP32
    ws = s2.workspace(w.B, w.N, w.Hq, w.Hkv, w.d, code, torch.device("cuda"))
    o, lse = s2.forward(tq, tk, tv, w.G, w.pi_scale, ws=ws)
    good = s2.backward(tq, tk, tv, o, lse, tdo, w.G, w.pi_scale, ws=ws, after_forward=True)
    assert s2.device_status(ws) == s2.S2_OK
    before = [_bits(t) for t in good]
    scratch = tuple(torch.empty_like(t) for t in good)
    # another PI scale than the forward's
    s2.backward(tq, tk, tv, o, lse, tdo, w.G, 4.0, ws=ws, after_forward=True, grads=scratch)
    assert s2.device_status(ws) == s2.S2_ERR_STALE_WORKSPACE
    # another q buffer (same contents): the rotation in the workspace is not its rotation
    s2.backward(tq.clone(), tk, tv, o, lse, tdo, w.G, w.pi_scale, ws=ws, after_forward=True,
                grads=scratch)
    assert s2.device_status(ws) == s2.S2_ERR_STALE_WORKSPACE
    # the forward's own arguments still match, and give the same gradients bit for bit
    again = s2.backward(tq, tk, tv, o, lse, tdo, w.G, w.pi_scale, ws=ws, after_forward=True)
    assert s2.device_status(ws) == s2.S2_OK
    for a, b in zip(before, (_bits(t) for t in again)):
        assert torch.equal(a, b)
