"""ar_tune_step_noalloc against ar_tune_step.

ar_tune_step_noalloc serves callers that cannot allocate device memory (a
process whose GPU memory another allocator owns, or a loop that cannot take
cudaMalloc's implicit synchronisation): it runs the same tuning step with its
scratch in a fixed device array inside the library.  Here it must give
exactly (bit for bit) what the workspace entry point gives, on two calls in a
row (the second call starts from the state the first one left, and reuses the
array the first one wrote).

This file is collected last so that a run stopping at the first failure has
already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ar():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import post_weight_quantization_autoround_b200 as m

    m.lib()
    return m


def _dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def test_noalloc_matches_workspace_entry_point_on_two_calls(ar):
    N, K, M, g, steps = 256, 512, 320, 128, 3
    d = synth.make_linear(N, K, M, seed=21)
    V0, a0, b0 = synth.make_state(N, K, g, seed=4, spread=True)
    cfg = ar.ar_qconfig_default(group_size=g)
    W, X = _dev_bf16(d["W"]), _dev_bf16(d["X"])
    Y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    ar.ar_linear_forward(X, W, Y)
    ref = [torch.from_numpy(x.copy()).cuda() for x in (V0, a0, b0)]
    new = [torch.from_numpy(x.copy()).cuda() for x in (V0, a0, b0)]
    ws = torch.empty(ar.ar_tune_step_workspace(W, *ref, M, cfg, steps), dtype=torch.uint8, device="cuda")
    assert ws.numel() <= ar.AR_NOALLOC_SCRATCH_BYTES
    for call in range(2):
        l_ref = torch.empty(steps, device="cuda")
        l_new = torch.empty(steps, device="cuda")
        dv_ref = torch.empty((N, K), device="cuda")
        dv_new = torch.empty((N, K), device="cuda")
        ar.ar_tune_step(W, *ref, X, Y, cfg, steps, l_ref, ws, dV=dv_ref)
        ar.ar_tune_step_noalloc(W, *new, X, Y, cfg, steps, l_new, dV=dv_new)
        assert ar.ar_get_device_status() == 0, ar.ar_last_error()
        # the same kernels on the same inputs in the same order: bit-identical
        # results, so a fault in the scratch layout cannot hide inside a tolerance
        assert np.array_equal(l_new.cpu().numpy(), l_ref.cpu().numpy()), call
        assert np.array_equal(dv_new.cpu().numpy(), dv_ref.cpu().numpy()), call
        for x, y in zip(new, ref):
            assert np.array_equal(x.cpu().numpy(), y.cpu().numpy()), call


def test_noalloc_rejects_problems_above_its_scratch(ar):
    """A 4096x4096 layer with 16384 tokens needs ~170 MB of scratch: refused before any launch."""
    cfg = ar.ar_qconfig_default()
    fake = 0x10000  # never dereferenced: the size check comes first
    layer = ar.Layer(fake, fake, fake, fake, 4096, 4096)
    loss = torch.empty(1, device="cuda")
    st = ar.lib().ar_tune_step_noalloc(0, ctypes.byref(layer), 1, fake, 16384, fake, ctypes.byref(cfg), 1,
                                       loss.data_ptr(), None, None)
    assert st == ar.AR_ERR_WORKSPACE
    assert "limit" in ar.ar_last_error()
