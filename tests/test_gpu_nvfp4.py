"""NVFP4 QDQ on the GPU against the oracle: codes, E4M3 block scales, the per-tensor scale and Ŵ,
all bit-exact (both sides take every step in fp32 in the same order, and the roundings to E4M3 and
E2M1 are round-to-nearest-even with saturation on both)."""
import numpy as np
import pytest
import torch

import synth
from oracle import autoround_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ar():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    import post_weight_quantization_autoround_b200 as m
    return m


def _run(ar, Wb, V, a):
    N, K = Wb.shape
    dev = "cuda"
    W = torch.from_numpy(Wb.view(np.int16)).to(dev).view(torch.bfloat16)
    Vd = None if V is None else torch.from_numpy(V).to(dev)
    ad = None if a is None else torch.from_numpy(a).to(dev)
    amax = torch.empty(1, dtype=torch.float32, device=dev)
    What = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
    codes = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((N, K // 16), dtype=torch.uint8, device=dev)
    gs = torch.empty(1, dtype=torch.float32, device=dev)
    ar.ar_absmax_bf16(W, amax)
    ar.ar_qdq_nvfp4(W, Vd, ad, amax, What, codes, scales, gs)
    torch.cuda.synchronize()
    return (amax.item(), What.view(torch.int16).cpu().numpy().view(np.uint16), codes.cpu().numpy(),
            scales.cpu().numpy(), gs.item())


def _inputs(N, K, seed, with_v=True, with_a=True):
    d = synth.make_linear(N, K, 1, seed=seed)
    Wb = d["W"]
    rng = np.random.default_rng(seed + 1)
    V = rng.uniform(-0.5, 0.5, (N, K)).astype(np.float32) if with_v else None
    a = rng.uniform(0.5, 1.0, (N, K // 16)).astype(np.float32) if with_a else None
    return Wb, V, a


@pytest.mark.parametrize("N,K,with_v,with_a", [(37, 64, True, True), (128, 1024, True, True), (1000, 272, True, False),
                                               (64, 4096, False, False), (3, 16, True, True)])
def test_qdq_nvfp4_bit_exact(ar, N, K, with_v, with_a):
    Wb, V, a = _inputs(N, K, seed=N + K, with_v=with_v, with_a=with_a)
    amax, What, codes, scales, gs = _run(ar, Wb, V, a)
    ref = O.nvfp4_qdq(synth.bf16_bits_to_f32(Wb), V, a)
    assert amax == float(np.max(np.abs(synth.bf16_bits_to_f32(Wb))))
    assert np.float32(gs) == ref["S"]
    assert np.array_equal(scales, ref["scale_codes"])
    assert np.array_equal(codes, O.pack_fp4(ref["codes"]))
    assert np.array_equal(What, ref["What_bf16"].view(np.uint32) >> 16)
    assert "qdq_nvfp4_kernel" in ar.ar_last_kernels()


def test_qdq_nvfp4_zero_matrix_and_underflowing_blocks(ar):
    N, K = 8, 64
    W = np.zeros((N, K), np.float32)
    z = (W.view(np.uint32) >> 16).astype(np.uint16)
    amax, What, codes, scales, gs = _run(ar, z, None, None)
    assert amax == 0.0 and gs == 0.0 and not What.any() and not codes.any() and not scales.any()
    # one large block and blocks 2^-20 smaller: their scale rounds to 0 in E4M3, so they quantize to 0
    W = np.full((N, K), 2.0 ** -20, np.float32)
    W[0, :16] = 100.0
    b = (W.view(np.uint32) >> 16).astype(np.uint16)
    amax, What, codes, scales, gs = _run(ar, b, None, None)
    ref = O.nvfp4_qdq(W)
    assert np.array_equal(scales, ref["scale_codes"]) and not ref["scale_codes"][1:].any()
    assert np.array_equal(What, ref["What_bf16"].view(np.uint32) >> 16)


def test_absmax_flags_non_finite_input(ar):
    W = np.zeros((4, 64), np.float32)
    W[2, 5] = np.inf
    b = (W.view(np.uint32) >> 16).astype(np.uint16)
    x = torch.from_numpy(b.view(np.int16)).cuda().view(torch.bfloat16)
    amax = torch.empty(1, dtype=torch.float32, device="cuda")
    ar.ar_absmax_bf16(x, amax)
    assert ar.ar_get_device_status() == ar.AR_ERR_NONFINITE
    assert ar.ar_get_device_status() == 0


def test_qdq_nvfp4_full_size_sampled_rows(ar):
    """8192 x 28672: the tensor maximum over the whole matrix, 64 sampled rows against the oracle."""
    wl = synth.WORKLOADS["down_8192_28672"]
    N, K = wl.n_out, wl.n_in
    d = synth.make_linear(N, K, 1, seed=wl.seed, x_outlier_channels=0)
    rng = np.random.default_rng(7)
    V = rng.uniform(-0.5, 0.5, (N, K)).astype(np.float32)
    a = rng.uniform(0.5, 1.0, (N, K // 16)).astype(np.float32)
    amax, What, codes, scales, gs = _run(ar, d["W"], V, a)
    Wf = synth.bf16_bits_to_f32(d["W"])
    assert amax == float(np.max(np.abs(Wf)))
    rows = np.sort(rng.choice(N, 64, replace=False))
    ref = O.nvfp4_qdq(Wf[rows], V[rows], a[rows], amax=amax)
    assert np.float32(gs) == ref["S"]
    assert np.array_equal(scales[rows], ref["scale_codes"])
    assert np.array_equal(codes[rows], O.pack_fp4(ref["codes"]))
    assert np.array_equal(What[rows], ref["What_bf16"].view(np.uint32) >> 16)
