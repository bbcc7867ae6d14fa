"""GPU path vs the CPU oracle, on the same seeded inputs (needs a B200 and the built library).

Bars (the task's acceptance criteria):
  * integer codes, packed INT4 words, scale / zero: bit-exact given the same
    V, alpha, beta (both sides decide in fp32 with the same IEEE operations);
  * per-step gradients dV, dalpha, dbeta: relative L2 error <= 1e-3;
  * gradient signs: >= 99.9 % agreement where |g| > 1e-6 and where
    |g| > 1e-3 * RMS(oracle gradient);
  * after a full run: codes agree on >= 99.5 % of elements, final MSE within 1 %;
  * W4A16 output: relative L2 error <= 2e-2 against the oracle's fp64 dequant-matmul.
The oracle computes its own reference output Y and never sees a GPU result.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import autoround_oracle as O

pytestmark = pytest.mark.gpu

GRAD_RTOL = 1e-3
SIGN_AGREE = 0.999
CODE_AGREE = 0.995
MSE_RTOL = 0.01
W4A16_RTOL = 2e-2
# tcgen05 W4A16 path: (q - z) and every product are exact, groups are summed in
# fp32, so the bf16 rounding of the output (relative 2^-9 per element) bounds
# the relative L2 error, plus a little fp32 summation error.
W4A16_TC_RTOL = 3e-3


@pytest.fixture(scope="module")
def ar():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import post_weight_quantization_autoround_b200 as m

    m.lib()
    return m


def bf16_dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def f32_dev(a) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def bits16(t: torch.Tensor) -> np.ndarray:
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def rel_l2(x, y):
    x = np.asarray(x, np.float64)
    y = np.asarray(y, np.float64)
    return float(np.linalg.norm(x - y) / max(np.linalg.norm(y), 1e-300))


def sign_agreement(g, ref, thresh):
    mask = np.abs(ref) > thresh
    if not mask.any():
        return 1.0, 0
    return float(np.mean(np.sign(g[mask]) == np.sign(ref[mask]))), int(mask.sum())


def cfg_pair(ar, bits=4, g=128, sym=False, lr=0.005):
    return ar.ar_qconfig_default(bits=bits, group_size=g, symmetric=int(sym), lr=lr), \
        O.QConfig(bits=bits, group_size=g, symmetric=sym, lr=lr)


# ----------------------------------------------------------------------------
# QDQ and INT4 packing: bit-exact
# ----------------------------------------------------------------------------

QDQ_CASES = [
    # N, K, g, bits, symmetric, spread state
    (200, 512, 128, 4, False, True),
    (200, 512, 128, 4, False, False),
    (64, 1024, 32, 3, False, True),
    (64, 1024, 32, 2, False, True),
    (48, 2048, 256, 8, False, True),
    (40, 512, 128, 4, True, True),
    (24, 64, 8, 4, False, True),
    (16, 3072, 1024, 4, False, True),
    (1, 128, 128, 4, False, True),
]


@pytest.mark.parametrize("N,K,g,bits,sym,spread", QDQ_CASES)
def test_qdq_bit_exact(ar, N, K, g, bits, sym, spread):
    d = synth.make_linear(N, K, 1, seed=N + K + bits, x_outlier_channels=0)
    V, a, b = synth.make_state(N, K, g, seed=bits, spread=spread)
    W = synth.bf16_bits_to_f32(d["W"])
    cfg, _ = cfg_pair(ar, bits, g, sym)
    Wd = bf16_dev(d["W"])
    What = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
    codes = torch.empty((N, K), dtype=torch.uint8, device="cuda")
    sc = torch.empty((N, K // g), dtype=torch.float32, device="cuda")
    zp = torch.empty((N, K // g), dtype=torch.float32, device="cuda")
    ar.ar_qdq(Wd, f32_dev(V), f32_dev(a), f32_dev(b), cfg, What, codes, sc, zp)
    assert ar.ar_get_device_status() == 0
    st = O.qdq(W, V, a, b, bits, g, sym)
    assert np.array_equal(sc.cpu().numpy().view(np.uint32), st["s"].view(np.uint32))
    assert np.array_equal(zp.cpu().numpy(), st["zp"])
    assert np.array_equal(codes.cpu().numpy(), st["q"].astype(np.uint8))
    assert np.array_equal(bits16(What), O.bf16_rne(st["What"]).view(np.uint32).__rshift__(16).astype(np.uint16))


@pytest.mark.parametrize("N,K,g,sym", [(200, 512, 128, False), (64, 1024, 32, True), (16, 2048, 1024, False),
                                       (8, 64, 8, False)])
def test_pack_int4_bit_exact(ar, N, K, g, sym):
    d = synth.make_linear(N, K, 1, seed=7 + K, x_outlier_channels=0)
    V, a, b = synth.make_state(N, K, g, seed=3, spread=True)
    cfg, _ = cfg_pair(ar, 4, g, sym)
    packed = torch.empty((N, K // 8), dtype=torch.int32, device="cuda")
    s16 = torch.empty((N, K // g), dtype=torch.float16, device="cuda")
    z16 = torch.empty((N, K // g), dtype=torch.float16, device="cuda")
    ar.ar_pack_int4(bf16_dev(d["W"]), f32_dev(V), f32_dev(a), f32_dev(b), cfg, packed, s16, z16)
    st = O.qdq(synth.bf16_bits_to_f32(d["W"]), V, a, b, 4, g, sym)
    words, s_ref, z_ref = O.pack_int4(st["q"], st["s"], st["zp"])
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), words)
    assert np.array_equal(s16.cpu().view(torch.int16).numpy().view(np.uint16), s_ref)
    assert np.array_equal(z16.cpu().view(torch.int16).numpy().view(np.uint16), z_ref)


def test_f32_to_bf16_matches_oracle_rounding(ar):
    x = np.random.default_rng(0).standard_normal(100003).astype(np.float32) * 3
    out = torch.empty(x.size, dtype=torch.bfloat16, device="cuda")
    ar.ar_f32_to_bf16(f32_dev(x), out)
    assert np.array_equal(bits16(out), (O.bf16_rne(x).view(np.uint32) >> 16).astype(np.uint16))


# ----------------------------------------------------------------------------
# tensor-core GEMM building block and the reference forward
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("a_mn,b_mn", [(False, False), (False, True), (True, False), (True, True)])
@pytest.mark.parametrize("M,N,K", [(200, 320, 192), (128, 256, 64), (512, 512, 1024), (8, 8, 8), (120, 136, 72),
                                   (1000, 776, 136)])
def test_gemm_all_operand_layouts(ar, a_mn, b_mn, M, N, K):
    """256 x 256 tiles on tcgen05 CTA pairs; ragged M, N, K leave the odd CTA's rows or B half
    partly or wholly outside the matrices."""
    rng = np.random.default_rng(M + N + K)
    A = synth.to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    B = synth.to_bf16_bits(rng.standard_normal((N, K)).astype(np.float32))
    Af, Bf = synth.bf16_bits_to_f32(A), synth.bf16_bits_to_f32(B)
    ref = O.reference_forward(Af, Bf).astype(np.float64)
    Ad = bf16_dev(np.ascontiguousarray(A.T) if a_mn else A)
    Bd = bf16_dev(np.ascontiguousarray(B.T) if b_mn else B)
    D = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    ar.ar_gemm_bf16(Ad, a_mn, Bd, b_mn, D, M, N, K)
    assert ",pair>" in ar.ar_last_kernels()
    got = D.cpu().numpy()
    assert np.isfinite(got).all()
    tol = 1e-5 * np.sqrt(K) * 4
    assert np.max(np.abs(got - ref)) <= tol, np.max(np.abs(got - ref))


@pytest.mark.parametrize("a_mn,b_mn", [(False, False), (True, True)])
def test_gemm_last_wave_half_width_units(ar, a_mn, b_mn):
    """2048 x 2560 output = 8 x 10 pair tiles of 256 x 256: on a 148-SM B200 (74 clusters) one wave of
    74 whole tiles, then the last 6 tiles as 12 units of 256 x 128; every output element is checked."""
    M, N, K = 2048, 2560, 128
    rng = np.random.default_rng(21)
    A = synth.to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    B = synth.to_bf16_bits(rng.standard_normal((N, K)).astype(np.float32))
    ref = O.reference_forward(synth.bf16_bits_to_f32(A), synth.bf16_bits_to_f32(B)).astype(np.float64)
    Ad = bf16_dev(np.ascontiguousarray(A.T) if a_mn else A)
    Bd = bf16_dev(np.ascontiguousarray(B.T) if b_mn else B)
    D = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    ar.ar_gemm_bf16(Ad, a_mn, Bd, b_mn, D, M, N, K)
    assert ar.ar_get_device_status() == 0
    got = D.cpu().numpy()
    assert np.isfinite(got).all()
    assert np.max(np.abs(got - ref)) <= 1e-5 * np.sqrt(K) * 4


@pytest.mark.parametrize("a_mn,b_mn", [(False, False), (True, True)])
def test_gemm_grouped_raster_covers_every_tile(ar, a_mn, b_mn):
    """B of 4608 x 8192 bf16 (75 MB) does not stay resident in L2, so the tiles run in groups of
    16 tile rows (20 rows: a full and a partial group); every output tile is computed once, checked on
    sampled rows from every tile row and the last one."""
    M, N, K = 5000, 4608, 8192
    rng = np.random.default_rng(8)
    A = synth.to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    B = synth.to_bf16_bits(rng.standard_normal((N, K)).astype(np.float32))
    Ad = bf16_dev(np.ascontiguousarray(A.T) if a_mn else A)
    Bd = bf16_dev(np.ascontiguousarray(B.T) if b_mn else B)
    D = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    ar.ar_gemm_bf16(Ad, a_mn, Bd, b_mn, D, M, N, K)
    assert ar.ar_get_device_status() == 0
    got = D.cpu().numpy()
    assert np.isfinite(got).all()
    rows = np.unique(np.concatenate([np.arange(0, M, 256) + 7, [M - 1]]))
    ref = O.reference_forward(synth.bf16_bits_to_f32(A[rows]), synth.bf16_bits_to_f32(B)).astype(np.float64)
    # a tile run with another tile's coordinates would be off by O(1) relative; fp32 sums over 8192 terms
    # of O(1) products are off by ~1e-7 relative
    assert rel_l2(got[rows], ref) <= 1e-5


def test_reference_forward(ar):
    d = synth.make_linear(320, 512, 200, seed=2)
    Xd, Wd = bf16_dev(d["X"]), bf16_dev(d["W"])
    Y = torch.empty((200, 320), dtype=torch.float32, device="cuda")
    ar.ar_linear_forward(Xd, Wd, Y)
    ref = O.reference_forward(synth.bf16_bits_to_f32(d["X"]), synth.bf16_bits_to_f32(d["W"]))
    assert rel_l2(Y.cpu().numpy(), ref) < 1e-6


# ----------------------------------------------------------------------------
# one tuning step: loss, gradients, update
# ----------------------------------------------------------------------------

class GpuLinear:
    """Device copies of one linear problem plus the workspace of ar_tune_step."""

    def __init__(self, ar, Wbits, Xbits, V, a, b, cfg, n_steps=1):
        self.ar = ar
        self.W = bf16_dev(Wbits)
        self.X = bf16_dev(Xbits)
        self.V, self.a, self.b = f32_dev(V), f32_dev(a), f32_dev(b)
        N, K = Wbits.shape
        M = Xbits.shape[0]
        self.Y = torch.empty((M, N), dtype=torch.float32, device="cuda")
        ar.ar_linear_forward(self.X, self.W, self.Y)
        self.cfg = cfg
        self.alloc_ws(n_steps)

    def alloc_ws(self, n_steps):
        n = self.ar.ar_tune_step_workspace(self.W, self.V, self.a, self.b, self.X.shape[0], self.cfg, n_steps)
        self.ws = torch.empty(n, dtype=torch.uint8, device="cuda")

    def step(self, n_steps=1, grads=False):
        N, K = self.W.shape
        G = K // self.cfg.group_size
        loss = torch.empty(max(n_steps, 1), dtype=torch.float32, device="cuda")
        dV = torch.full((N, K), float("nan"), device="cuda") if grads else None
        da = torch.full((N, G), float("nan"), device="cuda") if grads else None
        db = torch.full((N, G), float("nan"), device="cuda") if grads else None
        need = self.ar.ar_tune_step_workspace(self.W, self.V, self.a, self.b, self.X.shape[0], self.cfg, n_steps)
        if self.ws.numel() < need:
            self.alloc_ws(n_steps)
        self.ar.ar_tune_step(self.W, self.V, self.a, self.b, self.X, self.Y, self.cfg, n_steps, loss, self.ws,
                             dV=dV, dalpha=da, dbeta=db)
        assert self.ar.ar_get_device_status() == 0
        out = {"loss": loss.cpu().numpy()}
        if grads:
            out.update(dV=dV.cpu().numpy(), dalpha=da.cpu().numpy(), dbeta=db.cpu().numpy())
        return out

    def codes(self):
        N, K = self.W.shape
        c = torch.empty((N, K), dtype=torch.uint8, device="cuda")
        self.ar.ar_qdq(self.W, self.V, self.a, self.b, self.cfg, None, c, None, None)
        return c.cpu().numpy()

    def state(self):
        return self.V.cpu().numpy(), self.a.cpu().numpy(), self.b.cpu().numpy()


STEP_CASES = [
    # N, K, M, bits, g, sym, spread
    (256, 512, 320, 4, 128, False, True),
    (256, 512, 320, 4, 128, False, False),
    (136, 768, 200, 3, 32, False, True),
    (128, 512, 256, 2, 64, False, True),
    (64, 1024, 128, 8, 256, False, True),
    (192, 512, 160, 4, 128, True, True),
    # 8192 tokens: the fold in the GEMM epilogue (group sizes 32 and 128, symmetric)
    (136, 768, 8192, 3, 32, False, True),
    (192, 512, 8192, 4, 128, True, True),
]


@pytest.mark.parametrize("N,K,M,bits,g,sym,spread", STEP_CASES)
def test_single_step_matches_oracle(ar, N, K, M, bits, g, sym, spread):
    d = synth.make_linear(N, K, M, seed=N * 7 + bits, x_outlier_channels=4)
    V, a, b = synth.make_state(N, K, g, seed=11, spread=spread)
    cfg, ocfg = cfg_pair(ar, bits, g, sym)
    gl = GpuLinear(ar, d["W"], d["X"], V, a, b, cfg)
    out = gl.step(1, grads=True)
    kern = ar.ar_last_kernels()
    # the fold runs in the weight-gradient GEMM's epilogue from 8192 tokens (and for g = 256),
    # below that in the standalone fold kernel after a plain weight-gradient GEMM
    fused = M >= 8192 or g == 256
    assert "resid,pair>" in kern and (("fold,pair>" in kern) if fused else ("fold_int_kernel" in kern)), kern
    Wf, Xf = synth.bf16_bits_to_f32(d["W"]), synth.bf16_bits_to_f32(d["X"])
    L, (V1, a1, b1), gr, _ = O.tune_step_linear(Wf, Xf, O.reference_forward(Xf, Wf), V, a, b, ocfg)
    assert out["loss"][0] == pytest.approx(L, rel=1e-4)
    for k in ("dV", "dalpha", "dbeta"):
        assert rel_l2(out[k], gr[k]) <= GRAD_RTOL, (k, rel_l2(out[k], gr[k]))
        rms = np.sqrt(np.mean(gr[k].astype(np.float64) ** 2))
        for thr in (1e-6, 1e-3 * rms):
            agree, n = sign_agreement(out[k], gr[k], thr)
            assert agree >= SIGN_AGREE, (k, thr, agree, n)
    Vg, ag, bg = gl.state()
    # the update is exactly one fp32 step of +-lr (or none) from the GPU's own gradient sign
    for p0, p1, dg, lo, hi in [(V, Vg, out["dV"], -0.5, 0.5), (a, ag, out["dalpha"], 0.5, 1.0),
                               (b, bg, out["dbeta"], 0.5, 1.0)]:
        step = (np.float32(0.005) * np.sign(dg).astype(np.float32)).astype(np.float32)
        assert np.array_equal(p1, np.clip((p0 - step).astype(np.float32), np.float32(lo), np.float32(hi)))
    assert np.mean(Vg == V1) >= SIGN_AGREE and np.mean(ag == a1) >= 0.99 and np.mean(bg == b1) >= 0.99


def test_eval_only_call_updates_nothing(ar):
    d = synth.make_linear(64, 256, 96, seed=5)
    V, a, b = synth.make_state(64, 256, 128, seed=5, spread=True)
    cfg, ocfg = cfg_pair(ar)
    gl = GpuLinear(ar, d["W"], d["X"], V, a, b, cfg, n_steps=0)
    out = gl.step(0)
    Vg, ag, bg = gl.state()
    assert np.array_equal(Vg, V) and np.array_equal(ag, a) and np.array_equal(bg, b)
    Wf, Xf = synth.bf16_bits_to_f32(d["W"]), synth.bf16_bits_to_f32(d["X"])
    ref = O.eval_loss_linear(Wf, Xf, O.reference_forward(Xf, Wf), V, a, b, ocfg)
    assert out["loss"][0] == pytest.approx(ref, rel=1e-4)


# ----------------------------------------------------------------------------
# trajectories
# ----------------------------------------------------------------------------

def test_small_workload_full_trajectory(ar):
    """256x256 fp32 layer, 32 fp32 tokens, 4-bit g128, 10 steps: the whole run against the oracle."""
    wl = synth.WORKLOADS["linear_256"]
    d = synth.make_linear(wl.n_out, wl.n_in, wl.m_tokens, seed=wl.seed, dtype="f32", x_outlier_channels=0)
    # fp32 inputs are rounded to bf16 on the device by the library's own conversion
    Wb = torch.empty((wl.n_out, wl.n_in), dtype=torch.bfloat16, device="cuda")
    Xb = torch.empty((wl.m_tokens, wl.n_in), dtype=torch.bfloat16, device="cuda")
    ar.ar_f32_to_bf16(f32_dev(d["W"]), Wb)
    ar.ar_f32_to_bf16(f32_dev(d["X"]), Xb)
    V, a, b = synth.make_state(wl.n_out, wl.n_in, wl.group_size)
    cfg, ocfg = cfg_pair(ar, wl.bits, wl.group_size, lr=wl.lr)
    gl = GpuLinear(ar, bits16(Wb).reshape(wl.n_out, wl.n_in), bits16(Xb).reshape(wl.m_tokens, wl.n_in), V, a, b,
                   cfg, n_steps=wl.steps)
    out = gl.step(wl.steps)
    final_gpu = gl.step(0)["loss"][0]
    Wf, Xf = O.bf16_rne(d["W"]), O.bf16_rne(d["X"])
    losses, (Vo, ao, bo), final = O.tune_linear(Wf, Xf, V, a, b, ocfg, wl.steps)
    assert np.allclose(out["loss"], losses, rtol=1e-3)
    st = O.qdq(Wf, Vo, ao, bo, wl.bits, wl.group_size)
    assert np.mean(gl.codes() == st["q"]) >= CODE_AGREE
    assert final_gpu == pytest.approx(final, rel=MSE_RTOL)


def test_row_shards_reproduce_the_unsharded_step(ar):
    """ar_tune_step_shard on two row ranges of one layer gives the unsharded call's rows bit for bit."""
    N, K, M, g, steps, cut = 320, 512, 200, 128, 3, 136  # 136/320: the ratio is not a power of two
    d = synth.make_linear(N, K, M, seed=31)
    V, a, b = synth.make_state(N, K, g, seed=6, spread=True)
    cfg, ocfg = cfg_pair(ar, 4, g)
    full = GpuLinear(ar, d["W"], d["X"], V, a, b, cfg, n_steps=steps)
    l_full = full.step(steps)["loss"]
    shard_losses, shard_states = [], []
    for lo, hi in ((0, cut), (cut, N)):
        sh = GpuLinear(ar, d["W"][lo:hi], d["X"], V[lo:hi], a[lo:hi], b[lo:hi], cfg, n_steps=steps)
        loss = torch.empty(steps, dtype=torch.float32, device="cuda")
        ar.ar_tune_step_shard(sh.W, sh.V, sh.a, sh.b, sh.X, sh.Y, N, cfg, steps, loss, sh.ws)
        assert ar.ar_get_device_status() == 0
        shard_losses.append(loss.cpu().numpy())
        shard_states.append(sh.state())
    for i, ref in enumerate(full.state()):
        assert np.array_equal(np.concatenate([shard_states[0][i], shard_states[1][i]]), ref), i
    assert np.allclose(shard_losses[0] + shard_losses[1], l_full, rtol=1e-5)
    # and the oracle on the second shard with the layer's normaliser
    Wf, Xf = synth.bf16_bits_to_f32(d["W"][cut:]), synth.bf16_bits_to_f32(d["X"])
    L, _, _, _ = O.tune_step_linear(Wf, Xf, O.reference_forward(Xf, Wf), V[cut:], a[cut:], b[cut:], ocfg,
                                    count=M * N)
    assert shard_losses[1][0] == pytest.approx(L, rel=1e-4)


def test_steps_are_deterministic_and_resumable(ar):
    d = synth.make_linear(256, 512, 384, seed=9)
    V, a, b = synth.make_state(256, 512, 128, seed=1, spread=True)
    cfg, _ = cfg_pair(ar)
    g1 = GpuLinear(ar, d["W"], d["X"], V, a, b, cfg, n_steps=6)
    l1 = g1.step(6)["loss"]
    g2 = GpuLinear(ar, d["W"], d["X"], V, a, b, cfg, n_steps=3)
    l2 = np.concatenate([g2.step(3)["loss"], g2.step(3)["loss"]])
    assert np.array_equal(l1, l2)
    for x, y in zip(g1.state(), g2.state()):
        assert np.array_equal(x, y)


# ----------------------------------------------------------------------------
# W4A16
# ----------------------------------------------------------------------------

def _packed(ar, Wbits, V, a, b, g):
    N, K = Wbits.shape
    cfg, _ = cfg_pair(ar, 4, g)
    packed = torch.empty((N, K // 8), dtype=torch.int32, device="cuda")
    s16 = torch.empty((N, K // g), dtype=torch.float16, device="cuda")
    z16 = torch.empty((N, K // g), dtype=torch.float16, device="cuda")
    ar.ar_pack_int4(bf16_dev(Wbits), f32_dev(V), f32_dev(a), f32_dev(b), cfg, packed, s16, z16)
    return packed, s16, z16


@pytest.mark.parametrize("T", [1, 3, 4, 16])
@pytest.mark.parametrize("N,K,g", [(320, 1024, 128), (64, 4096, 32), (40, 2048, 1024)])
def test_w4a16_matches_oracle(ar, T, N, K, g):
    d = synth.make_linear(N, K, 1, seed=T + N)
    V, a, b = synth.make_state(N, K, g, seed=2, spread=True)
    packed, s16, z16 = _packed(ar, d["W"], V, a, b, g)
    A = synth.make_activations(T, K, seed=T)
    out = torch.empty((T, N), dtype=torch.bfloat16, device="cuda")
    ar.ar_w4a16_gemm(bf16_dev(A), packed, s16, z16, g, out)
    st = O.qdq(synth.bf16_bits_to_f32(d["W"]), V, a, b, 4, g)
    words, s_ref, z_ref = O.pack_int4(st["q"], st["s"], st["zp"])
    ref = O.w4a16_matmul(synth.bf16_bits_to_f32(A), words, s_ref, z_ref, g)
    got = out.float().cpu().numpy()
    assert rel_l2(got, ref) <= W4A16_RTOL


@pytest.mark.parametrize("T", [1, 5, 8, 9, 16])
@pytest.mark.parametrize("N,K,g,tag", [
    (1000, 1280, 32, "g=32,nt8>"),              # N not a multiple of 8; last 512-k stage half empty
    (10000, 512, 64, "g=64,nt8>"),              # 72 rows per CTA: two row passes (64 + 8); last CTA one pass
    (10000, 1024, 128, "g>=128,nt8>"),          # the same passes with one group per 128-k chunk
    (4096, 2048, 128, "g>=128,ksplit2,nt7>"),   # 56-row CTA pairs splitting K
    (296, 4096, 256, "g>=128,ksplit2,nt1>"),    # 8-row CTA pairs
])
def test_w4a16_decode_row_ranges_match_oracle(ar, T, N, K, g, tag):
    """T <= 16 on the decode kernel that gives each SM a contiguous range of weight rows."""
    d = synth.make_linear(N, K, 1, seed=T + N)
    V, a, b = synth.make_state(N, K, g, seed=2, spread=True)
    packed, s16, z16 = _packed(ar, d["W"], V, a, b, g)
    A = synth.make_activations(T, K, seed=T)
    out = torch.empty((T, N), dtype=torch.bfloat16, device="cuda")
    ar.ar_w4a16_gemm(bf16_dev(A), packed, s16, z16, g, out)
    kern = ar.ar_last_kernels()
    assert "w4a16_dec_kernel<T<=%d,%s" % (8 if T <= 8 else 16, tag) in kern, kern
    st = O.qdq(synth.bf16_bits_to_f32(d["W"]), V, a, b, 4, g)
    words, s_ref, z_ref = O.pack_int4(st["q"], st["s"], st["zp"])
    ref = O.w4a16_matmul(synth.bf16_bits_to_f32(A), words, s_ref, z_ref, g)
    got = out.float().cpu().numpy()
    assert rel_l2(got, ref) <= W4A16_RTOL
    # each token on its own, and the first and last rows (the ends of the row ranges)
    for t in range(T):
        assert rel_l2(got[t], ref[t]) <= W4A16_RTOL
    assert rel_l2(got[:, :8], ref[:, :8]) <= W4A16_RTOL and rel_l2(got[:, -8:], ref[:, -8:]) <= W4A16_RTOL
    # on the device's own codes, scales and zeros only the bf16 rounding of the output remains
    own = O.w4a16_matmul(synth.bf16_bits_to_f32(A), packed.cpu().numpy().view(np.uint32),
                         s16.cpu().numpy().view(np.uint16), z16.cpu().numpy().view(np.uint16), g)
    assert rel_l2(got, own) <= W4A16_TC_RTOL


def test_w4a16_decode_falls_back_when_scale_rows_are_not_16_byte_multiples(ar):
    """K/g = 2 groups per row: the scale/zero rows cannot be TMA boxes, the older decode kernel runs."""
    N, K, g, T = 40, 2048, 1024, 3
    d = synth.make_linear(N, K, 1, seed=9)
    V, a, b = synth.make_state(N, K, g, seed=2, spread=True)
    packed, s16, z16 = _packed(ar, d["W"], V, a, b, g)
    A = synth.make_activations(T, K, seed=4)
    out = torch.empty((T, N), dtype=torch.bfloat16, device="cuda")
    ar.ar_w4a16_gemm(bf16_dev(A), packed, s16, z16, g, out)
    assert "w4a16_tma_kernel" in ar.ar_last_kernels()
    st = O.qdq(synth.bf16_bits_to_f32(d["W"]), V, a, b, 4, g)
    words, s_ref, z_ref = O.pack_int4(st["q"], st["s"], st["zp"])
    ref = O.w4a16_matmul(synth.bf16_bits_to_f32(A), words, s_ref, z_ref, g)
    assert rel_l2(out.float().cpu().numpy(), ref) <= W4A16_RTOL


@pytest.mark.parametrize("T", [17, 40, 64, 100, 256])
@pytest.mark.parametrize("N,K,g", [(320, 1024, 128), (64, 4096, 32), (40, 2048, 1024)])
def test_w4a16_tensor_core_path_matches_oracle(ar, T, N, K, g):
    """T > 16 runs the tcgen05 dequant GEMM (one group per TMEM accumulator)."""
    d = synth.make_linear(N, K, 1, seed=T + N)
    V, a, b = synth.make_state(N, K, g, seed=2, spread=True)
    packed, s16, z16 = _packed(ar, d["W"], V, a, b, g)
    A = synth.make_activations(T, K, seed=T)
    out = torch.empty((T, N), dtype=torch.bfloat16, device="cuda")
    ar.ar_w4a16_gemm(bf16_dev(A), packed, s16, z16, g, out)
    assert "w4a16_tc_kernel" in ar.ar_last_kernels()
    st = O.qdq(synth.bf16_bits_to_f32(d["W"]), V, a, b, 4, g)
    words, s_ref, z_ref = O.pack_int4(st["q"], st["s"], st["zp"])
    ref = O.w4a16_matmul(synth.bf16_bits_to_f32(A), words, s_ref, z_ref, g)
    assert rel_l2(out.float().cpu().numpy(), ref) <= W4A16_TC_RTOL


def test_w4a16_tensor_core_path_many_tiles(ar):
    """Enough (row, token) tiles that K is not split; ragged token tail (1000 = 7 x 128 + 104)."""
    N, K, g, T = 1280, 512, 64, 1000
    d = synth.make_linear(N, K, 1, seed=11)
    V, a, b = synth.make_state(N, K, g, seed=3, spread=True)
    packed, s16, z16 = _packed(ar, d["W"], V, a, b, g)
    A = synth.make_activations(T, K, seed=12)
    out = torch.empty((T, N), dtype=torch.bfloat16, device="cuda")
    ar.ar_w4a16_gemm(bf16_dev(A), packed, s16, z16, g, out)
    assert "w4a16_tc_kernel<TN=128>" in ar.ar_last_kernels()
    st = O.qdq(synth.bf16_bits_to_f32(d["W"]), V, a, b, 4, g)
    words, s_ref, z_ref = O.pack_int4(st["q"], st["s"], st["zp"])
    ref = O.w4a16_matmul(synth.bf16_bits_to_f32(A), words, s_ref, z_ref, g)
    got = out.float().cpu().numpy()
    assert rel_l2(got, ref) <= W4A16_TC_RTOL
    # every token row on its own (a wrong tile origin would show in one row only)
    for t in (0, 127, 128, 895, 896, 999):
        assert rel_l2(got[t], ref[t]) <= W4A16_TC_RTOL


@pytest.mark.parametrize("T", [1, 16, 64, 256])
def test_w4a16_full_size_sampled_rows(ar, T):
    """8192 x 28672 down projection, sampled output rows against the oracle."""
    wl = synth.WORKLOADS["down_8192_28672"]
    N, K, g = wl.n_out, wl.n_in, wl.group_size
    d = synth.make_linear(N, K, 1, seed=wl.seed, x_outlier_channels=0)
    V, a, b = synth.make_state(N, K, g)
    packed, s16, z16 = _packed(ar, d["W"], V, a, b, g)
    A = synth.make_activations(T, K, seed=1)
    out = torch.empty((T, N), dtype=torch.bfloat16, device="cuda")
    ar.ar_w4a16_gemm(bf16_dev(A), packed, s16, z16, g, out)
    rows = np.sort(np.random.default_rng(5).choice(N, 64, replace=False))
    st = O.qdq(synth.bf16_bits_to_f32(d["W"][rows]), V[rows], a[rows], b[rows], 4, g)
    words, s_ref, z_ref = O.pack_int4(st["q"], st["s"], st["zp"])
    assert np.array_equal(packed.cpu().numpy().view(np.uint32)[rows], words)
    ref = O.w4a16_matmul(synth.bf16_bits_to_f32(A), words, s_ref, z_ref, g)
    assert rel_l2(out.float().cpu().numpy()[:, rows], ref) <= W4A16_RTOL


# ----------------------------------------------------------------------------
# device status: no silent acceptance of non-finite data
# ----------------------------------------------------------------------------

def test_nonfinite_weight_raises_status(ar):
    d = synth.make_linear(16, 256, 1, seed=1)
    Wb = d["W"].copy()
    Wb[3, 17] = 0x7FC0  # bf16 NaN
    V, a, b = synth.make_state(16, 256, 128)
    cfg, _ = cfg_pair(ar)
    What = torch.empty((16, 256), dtype=torch.bfloat16, device="cuda")
    ar.ar_qdq(bf16_dev(Wb), f32_dev(V), f32_dev(a), f32_dev(b), cfg, What)
    assert ar.ar_get_device_status() == ar.AR_ERR_NONFINITE
    assert ar.ar_get_device_status() == 0  # sticky until read, then cleared


@pytest.mark.parametrize("g", [128, 256])
def test_split_reduction_pairs_match_oracle(ar, g):
    """32768 tokens over a 512x512 layer: the weight-gradient GEMM splits the token
    reduction across CTA pairs (rank 1 ships its partial accumulator to rank 0).
    Every output row is checked against the oracle."""
    N, K, M = 512, 512, 32768
    d = synth.make_linear(N, K, M, seed=31 + g)
    V, a, b = synth.make_state(N, K, g, seed=4, spread=True)
    cfg, ocfg = cfg_pair(ar, 4, g)
    gl = GpuLinear(ar, d["W"], d["X"], V, a, b, cfg)
    out = gl.step(1, grads=True)
    assert "split2" in ar.ar_last_kernels()
    Wf, Xf = synth.bf16_bits_to_f32(d["W"]), synth.bf16_bits_to_f32(d["X"])
    L, (V1, a1, b1), gr, _ = O.tune_step_linear(Wf, Xf, O.reference_forward(Xf, Wf), V, a, b, ocfg)
    assert out["loss"][0] == pytest.approx(L, rel=1e-4)
    for k in ("dV", "dalpha", "dbeta"):
        assert rel_l2(out[k], gr[k]) <= GRAD_RTOL, (k, rel_l2(out[k], gr[k]))
    Vg, ag, bg = gl.state()
    assert np.mean(Vg == V1) >= SIGN_AGREE and np.mean(ag == a1) >= 0.99 and np.mean(bg == b1) >= 0.99


def test_bounded_wait_gives_up_and_reports_timeout(ar):
    """A device wait on a barrier nothing completes ends after its limit with AR_ERR_TIMEOUT;
    the context stays usable (a normal call follows)."""
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    ar.ar_debug_wait_timeout(20_000_000, flag)  # 20 ms
    assert ar.ar_get_device_status() == ar.AR_ERR_TIMEOUT
    assert int(flag.item()) == 1
    assert ar.ar_get_device_status() == 0
    x = np.arange(8, dtype=np.float32)
    out = torch.empty(8, dtype=torch.bfloat16, device="cuda")
    ar.ar_f32_to_bf16(f32_dev(x), out)
    assert out.float().cpu().numpy().tolist() == x.tolist()
