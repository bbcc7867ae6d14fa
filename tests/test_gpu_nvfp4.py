"""NVFP4 QDQ on the GPU against the oracle: codes, E4M3 block scales, the per-tensor scale and Ŵ,
all bit-exact (both sides take every step in fp32 in the same order, and the roundings to E4M3 and
E2M1 are round-to-nearest-even with saturation on both).  The NVFP4 weights' matmul against the
oracle's fp64 matmul on the same codes, scales and S: every E2M1 value times its E4M3 block scale is
exact in bf16 and every product in the tensor cores is exact, so only the fp32 accumulation and the
bf16 rounding of the output (2^-9 relative) remain; bar 3e-3 relative L2."""
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


# ----------------------------------------------------------------------------
# tuning steps on NVFP4
# ----------------------------------------------------------------------------

GRAD_RTOL = 1e-3


def _dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def _rel_l2(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


def _nv_state(N, K, seed, spread):
    rng = np.random.default_rng(seed)
    if not spread:
        return np.zeros((N, K), np.float32), np.ones((N, K // 16), np.float32)
    return rng.uniform(-0.4, 0.4, (N, K)).astype(np.float32), rng.uniform(0.6, 1.0, (N, K // 16)).astype(np.float32)


@pytest.mark.parametrize("N,K,M,spread", [(256, 256, 64, False), (136, 768, 200, True), (512, 512, 1024, True)])
def test_tune_step_nvfp4_matches_oracle(ar, N, K, M, spread):
    d = synth.make_linear(N, K, M, seed=N + M)
    Wf, Xf = synth.bf16_bits_to_f32(d["W"]), synth.bf16_bits_to_f32(d["X"])
    V0, a0 = _nv_state(N, K, seed=5, spread=spread)
    Y = O.reference_forward(Xf, Wf)
    W, X = _dev_bf16(d["W"]), _dev_bf16(d["X"])
    V, a = torch.from_numpy(V0.copy()).cuda(), torch.from_numpy(a0.copy()).cuda()
    amax = torch.empty(1, dtype=torch.float32, device="cuda")
    ar.ar_absmax_bf16(W, amax)
    cfg = ar.ar_qconfig_default()
    ws = torch.empty(ar.ar_tune_step_nvfp4_workspace(M, N, K, 1), dtype=torch.uint8, device="cuda")
    loss = torch.empty(1, dtype=torch.float32, device="cuda")
    dV = torch.empty((N, K), dtype=torch.float32, device="cuda")
    da = torch.empty((N, K // 16), dtype=torch.float32, device="cuda")
    ar.ar_tune_step_nvfp4(W, V, a, amax, X, torch.from_numpy(Y).cuda(), cfg, 1, loss, ws, dV, da)
    kern = ar.ar_last_kernels()
    assert "qdq_nvfp4_kernel" in kern and "fold_nvfp4_kernel" in kern
    L, (V1, a1), gr, _ = O.nvfp4_tune_step_linear(Wf, Xf, Y, V0, a0, O.QConfig())
    assert loss.item() == pytest.approx(L, rel=1e-4)
    assert _rel_l2(dV.cpu().numpy(), gr["dV"]) <= GRAD_RTOL
    assert _rel_l2(da.cpu().numpy(), gr["dalpha"]) <= GRAD_RTOL
    assert np.mean(V.cpu().numpy() == V1) >= 0.999
    assert np.mean(a.cpu().numpy() == a1) >= 0.99


def test_tune_step_nvfp4_steps_in_one_call_equal_single_calls_and_lower_the_loss(ar):
    N, K, M = 256, 512, 256
    d = synth.make_linear(N, K, M, seed=17)
    Wf, Xf = synth.bf16_bits_to_f32(d["W"]), synth.bf16_bits_to_f32(d["X"])
    Y = torch.from_numpy(O.reference_forward(Xf, Wf)).cuda()
    W, X = _dev_bf16(d["W"]), _dev_bf16(d["X"])
    amax = torch.empty(1, dtype=torch.float32, device="cuda")
    ar.ar_absmax_bf16(W, amax)
    cfg = ar.ar_qconfig_default()
    V0, a0 = _nv_state(N, K, 0, False)
    Va, aa = torch.from_numpy(V0.copy()).cuda(), torch.from_numpy(a0.copy()).cuda()
    Vb, ab = torch.from_numpy(V0.copy()).cuda(), torch.from_numpy(a0.copy()).cuda()
    ws = torch.empty(ar.ar_tune_step_nvfp4_workspace(M, N, K, 20), dtype=torch.uint8, device="cuda")
    la = torch.empty(20, dtype=torch.float32, device="cuda")
    ar.ar_tune_step_nvfp4(W, Va, aa, amax, X, Y, cfg, 20, la, ws)
    lb = []
    one = torch.empty(1, dtype=torch.float32, device="cuda")
    for _ in range(20):
        ar.ar_tune_step_nvfp4(W, Vb, ab, amax, X, Y, cfg, 1, one, ws)
        lb.append(one.item())
    assert np.array_equal(la.cpu().numpy(), np.array(lb, np.float32))
    assert torch.equal(Va, Vb) and torch.equal(aa, ab)
    assert lb[-1] < lb[0]


NVFP4_GEMM_RTOL = 3e-3


def _rel_l2(x, y):
    x = np.asarray(x, np.float64)
    y = np.asarray(y, np.float64)
    return float(np.linalg.norm(x - y) / max(np.linalg.norm(y), 1e-300))


def _nvfp4_weights(ar, Wb, V, a):
    """The GPU QDQ's exports (device tensors) of bf16 bits Wb."""
    N, K = Wb.shape
    dev = "cuda"
    W = torch.from_numpy(Wb.view(np.int16)).to(dev).view(torch.bfloat16)
    amax = torch.empty(1, dtype=torch.float32, device=dev)
    codes = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((N, K // 16), dtype=torch.uint8, device=dev)
    gs = torch.empty(1, dtype=torch.float32, device=dev)
    ar.ar_absmax_bf16(W, amax)
    ar.ar_qdq_nvfp4(W, None if V is None else torch.from_numpy(V).to(dev),
                    None if a is None else torch.from_numpy(a).to(dev), amax, None, codes, scales, gs)
    return codes, scales, gs


def _gemm(ar, A_bits, codes, scales, gs):
    T = A_bits.shape[0]
    N = codes.shape[0]
    A = torch.from_numpy(A_bits.view(np.int16)).cuda().view(torch.bfloat16)
    out = torch.empty((T, N), dtype=torch.bfloat16, device="cuda")
    ar.ar_nvfp4_gemm(A, codes, scales, gs, out)
    torch.cuda.synchronize()
    return out.float().cpu().numpy()


@pytest.mark.parametrize("N,K,T", [(136, 256, 1), (200, 768, 5), (1000, 1024, 16), (320, 2048, 40),
                                   (256, 384, 64), (130, 640, 129), (40, 4096, 3)])
def test_nvfp4_gemm_matches_oracle(ar, N, K, T):
    """Ragged N (not a multiple of 128 rows), K with 1-8 accumulation groups, every token-tile width
    (16, 32, 64, 128 tokens, two 128-token tiles at T = 129) and the CTA pair splitting K (small N)."""
    Wb, V, a = _inputs(N, K, seed=3 * N + K)
    codes, scales, gs = _nvfp4_weights(ar, Wb, V, a)
    A_bits = synth.make_activations(T, K, seed=T + 7)
    got = _gemm(ar, A_bits, codes, scales, gs)
    assert "nvfp4_tc_kernel" in ar.ar_last_kernels()
    ref = O.nvfp4_matmul(synth.bf16_bits_to_f32(A_bits), codes.cpu().numpy(), scales.cpu().numpy(), gs.item())
    assert _rel_l2(got, ref) <= NVFP4_GEMM_RTOL
    for t in range(T):
        assert _rel_l2(got[t], ref[t]) <= NVFP4_GEMM_RTOL
    # the same against the oracle's own QDQ of the weights (the GPU QDQ is bit-exact, so its codes are these)
    st = O.nvfp4_qdq(synth.bf16_bits_to_f32(Wb), V, a)
    ref2 = O.nvfp4_matmul(synth.bf16_bits_to_f32(A_bits), O.pack_fp4(st["codes"]), st["scale_codes"], st["S"])
    assert _rel_l2(got, ref2) <= NVFP4_GEMM_RTOL


def test_nvfp4_gemm_zero_weights(ar):
    """An all-zero matrix: S = 0, every code and scale 0, the product exactly 0."""
    N, K, T = 64, 256, 4
    Wb = np.zeros((N, K), np.uint16)
    codes, scales, gs = _nvfp4_weights(ar, Wb, None, None)
    got = _gemm(ar, synth.make_activations(T, K, seed=1), codes, scales, gs)
    assert np.all(got == 0.0)


@pytest.mark.parametrize("T", [1, 16, 256])
def test_nvfp4_gemm_full_size_sampled_rows(ar, T):
    """The 8192 x 28672 layer, checked on 64 sampled output rows (the rows of a linear layer are
    independent): the oracle recomputes them from the GPU's codes, scales and S of those rows."""
    N, K = 8192, 28672
    d = synth.make_linear(N, K, 1, seed=5, x_outlier_channels=0)
    codes, scales, gs = _nvfp4_weights(ar, d["W"], None, None)
    A_bits = synth.make_activations(T, K, seed=11)
    got = _gemm(ar, A_bits, codes, scales, gs)
    rows = np.sort(np.random.default_rng(2).choice(N, 64, replace=False))
    ref = O.nvfp4_matmul(synth.bf16_bits_to_f32(A_bits), codes.cpu().numpy()[rows], scales.cpu().numpy()[rows],
                         gs.item())
    assert _rel_l2(got[:, rows], ref) <= NVFP4_GEMM_RTOL
