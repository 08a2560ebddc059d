"""s2attn_fwd_noalloc: the forward for callers that cannot allocate device memory per call
(a plugin whose host application owns every device allocation, a latency-critical loop that
cannot afford cudaMalloc's implicit synchronisation, a C caller with no allocator). Its
scratch is a fixed array inside the library instead of a caller-provided workspace.

The test calls it through the C ABI twice in a row and checks each result against the
workspace-based s2attn_fwd on the same inputs and against the fp64 oracle, within the parity
tolerances of the other GPU tests, and reads the call's device status through
s2attn_noalloc_device_status (the no-allocation caller cannot address the status word in
the library's scratch). It lives in a file of its own, collected last, and needs no state
from other tests.
"""
import pytest
import torch

import oracle
import synth
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu

CASES = [
    # B, N, Hq, Hkv, d, G, pi_scale, dtype, causal
    (1, 1024, 4, 2, 128, 256, 2.0, "bf16", True),
    (1, 256, 4, 4, 64, 64, 2.0, "f32", True),
    (2, 512, 4, 4, 128, 128, 1.0, "bf16", False),
]


@pytest.fixture(scope="module")
def s2():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from longlora_shifted_sparse_b200 import s2attn
    return s2attn


@pytest.mark.parametrize("case", CASES, ids=["bf16_gqa", "f32_tiny", "bf16_noncausal_b2"])
def test_noalloc_forward_matches_workspace_forward(s2, case):
    B, N, Hq, Hkv, d, G, s, dt, causal = case
    scale = 0.5 if dt == "bf16" else 1.0
    q, k, v, _ = synth.s2attn_inputs(31, B, N, Hq, Hkv, d, scale, dt, with_dout=False)
    tq, tk, tv = (H.to_device(x, dt) for x in (q, k, v))
    code = s2.S2_BF16 if dt == "bf16" else s2.S2_FP32
    assert s2.s2attn_workspace_bytes(B, N, Hq, Hkv, d, code) <= s2.NOALLOC_SCRATCH_BYTES
    o_ref, lse_ref = s2.forward(tq, tk, tv, G, s, causal=causal)
    torch.cuda.synchronize()
    o_or, lse_or = oracle.fwd(q, k, v, G, s, causal=causal)
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        o = torch.full_like(o_ref, float("nan"))
        lse = torch.full_like(lse_ref, float("nan"))
        rc = s2.s2attn_fwd_noalloc(tq.data_ptr(), tk.data_ptr(), tv.data_ptr(), o.data_ptr(),
                                   lse.data_ptr(), B, N, Hq, Hkv, d, G, int(causal), s, 10000.0,
                                   code, stream)
        assert rc == s2.S2_OK, s2.s2attn_status_string(rc)
        assert s2.s2attn_noalloc_device_status(stream) == s2.S2_OK
        torch.cuda.synchronize()
        o_h, lse_h = H.to_host_f64(o), H.to_host_f64(lse)
        H.assert_close_o(o_h, H.to_host_f64(o_ref), dt)
        H.assert_close_lse(lse_h, H.to_host_f64(lse_ref), dt)
        H.assert_close_o(o_h, o_or, dt, "o vs oracle")
        H.assert_close_lse(lse_h, lse_or, dt, "lse vs oracle")


def test_noalloc_rejects_shapes_beyond_its_scratch(s2):
    B, N, Hq, Hkv, d, G = 1, 65536, 32, 32, 128, 16384
    assert s2.s2attn_workspace_bytes(B, N, Hq, Hkv, d, s2.S2_BF16) > s2.NOALLOC_SCRATCH_BYTES
    small = torch.zeros(1024, dtype=torch.bfloat16, device="cuda")
    p = small.data_ptr()
    rc = s2.s2attn_fwd_noalloc(p, p, p, p, p, B, N, Hq, Hkv, d, G, 1, 16.0, 10000.0, s2.S2_BF16,
                               torch.cuda.current_stream().cuda_stream)
    assert rc == s2.S2_ERR_WORKSPACE
    assert bool((small == 0).all())


def test_noalloc_status_query_reads_and_clears(s2):
    """The status query needs no workspace and allocates nothing; after a clean call it
    reports S2_OK, and reading it twice gives S2_OK both times (reading clears the word)."""
    stream = torch.cuda.current_stream().cuda_stream
    assert s2.s2attn_noalloc_device_status(stream) == s2.S2_OK
    assert s2.noalloc_device_status() == s2.S2_OK
