"""SwiGLU MLP block tuned jointly on the GPU vs the CPU oracle (needs a B200).

Block: down(silu(gate(x)) * up(x)); the three weights are quantized and tuned
together against the block output.  Same bars as the single-layer tests:
gradients within 1e-3 relative L2, signs >= 99.9 %, codes >= 99.5 % and the
final MSE within 1 % after several steps.  The full-shape case keeps the
Llama-7B block's weight shapes (4096 <-> 11008) with 256 tokens so that the
oracle finishes in seconds.
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


@pytest.fixture(scope="module")
def ar():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import post_weight_quantization_autoround_b200 as m

    m.lib()
    return m


def bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def f32_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def rel_l2(x, y):
    return float(np.linalg.norm(np.asarray(x, np.float64) - y) / max(np.linalg.norm(np.asarray(y, np.float64)), 1e-300))


class GpuMlp:
    def __init__(self, ar, d, states, cfg, n_steps):
        self.ar, self.cfg = ar, cfg
        self.W = [bf16_dev(d[k]) for k in ("Wg", "Wu", "Wd")]
        self.X = bf16_dev(d["X"])
        self.st = [tuple(f32_dev(x) for x in s) for s in states]
        M, Hd = d["X"].shape
        self.Y = torch.empty((M, Hd), dtype=torch.float32, device="cuda")
        fws = torch.empty(ar.ar_block_forward_workspace(ar.AR_BLOCK_SWIGLU_MLP, self.W, M), dtype=torch.uint8,
                          device="cuda")
        ar.ar_block_forward(ar.AR_BLOCK_SWIGLU_MLP, self.W, self.X, self.Y, fws)
        self.ws = torch.empty(ar.ar_tune_block_workspace(ar.AR_BLOCK_SWIGLU_MLP, self.layers(), M, cfg, n_steps),
                              dtype=torch.uint8, device="cuda")

    def layers(self):
        return [(W, *s) for W, s in zip(self.W, self.st)]

    def step(self, n_steps, grads=False):
        loss = torch.empty(max(n_steps, 1), device="cuda")
        gr = None
        if grads:
            gr = []
            for W in self.W:
                N, K = W.shape
                G = K // self.cfg.group_size
                gr.append((torch.empty((N, K), device="cuda"), torch.empty((N, G), device="cuda"),
                           torch.empty((N, G), device="cuda")))
        self.ar.ar_tune_block(self.ar.AR_BLOCK_SWIGLU_MLP, self.layers(), self.X, self.Y, self.cfg, n_steps, loss,
                              self.ws, grads=gr)
        assert self.ar.ar_get_device_status() == 0, self.ar.ar_last_error()
        out = {"loss": loss.cpu().numpy()}
        if grads:
            out["grads"] = [tuple(t.cpu().numpy() for t in g) for g in gr]
        return out

    def state(self):
        return [tuple(t.cpu().numpy() for t in s) for s in self.st]

    def codes(self, i):
        W = self.W[i]
        c = torch.empty(W.shape, dtype=torch.uint8, device="cuda")
        self.ar.ar_qdq(W, *self.st[i], self.cfg, None, c, None, None)
        return c.cpu().numpy()


def _problem(Hd, F, M, g, seed, spread=True):
    d = synth.make_mlp(Hd, F, M, seed=seed, x_outlier_channels=4)
    states = []
    for k, (n, kk) in zip(("Wg", "Wu", "Wd"), ((F, Hd), (F, Hd), (Hd, F))):
        states.append(synth.make_state(n, kk, g, seed=seed + len(states), spread=spread))
    return d, states


def _oracle_inputs(d):
    Ws = [synth.bf16_bits_to_f32(d[k]) for k in ("Wg", "Wu", "Wd")]
    X = synth.bf16_bits_to_f32(d["X"])
    return Ws, X, O.mlp_reference(X, *Ws)


@pytest.mark.parametrize("Hd,F,M,g,bits", [(256, 384, 200, 128, 4), (512, 1376, 160, 32, 3), (256, 512, 128, 64, 2)])
def test_mlp_single_step_matches_oracle(ar, Hd, F, M, g, bits):
    d, states = _problem(Hd, F, M, g, seed=Hd + F)
    cfg = ar.ar_qconfig_default(bits=bits, group_size=g)
    ocfg = O.QConfig(bits=bits, group_size=g)
    gm = GpuMlp(ar, d, states, cfg, 1)
    out = gm.step(1, grads=True)
    Ws, X, Y = _oracle_inputs(d)
    L, new_states, grads, _, _ = O.tune_step_mlp(Ws, X, Y, states, ocfg)
    assert out["loss"][0] == pytest.approx(L, rel=1e-3)
    for li in range(3):
        for k, ref in zip((0, 1, 2), (grads[li]["dV"], grads[li]["dalpha"], grads[li]["dbeta"])):
            got = out["grads"][li][k]
            assert rel_l2(got, ref) <= GRAD_RTOL, (li, k, rel_l2(got, ref))
            mask = np.abs(ref) > 1e-3 * np.sqrt(np.mean(ref.astype(np.float64) ** 2))
            assert np.mean(np.sign(got[mask]) == np.sign(ref[mask])) >= SIGN_AGREE, (li, k)
    for (Vg, ag, bg), (Vo, ao, bo) in zip(gm.state(), new_states):
        assert np.mean(Vg == Vo) >= SIGN_AGREE


def test_mlp_full_shapes_token_sample(ar):
    """Llama-7B block shapes (4096 <-> 11008, g128, W4), 256 tokens: one joint step."""
    wl = synth.WORKLOADS["mlp_4096_11008"]
    d, states = _problem(wl.n_in, wl.inter, 256, wl.group_size, seed=0, spread=False)
    cfg = ar.ar_qconfig_default()
    gm = GpuMlp(ar, d, states, cfg, 1)
    out = gm.step(1, grads=True)
    Ws, X, Y = _oracle_inputs(d)
    L, _, grads, _, _ = O.tune_step_mlp(Ws, X, Y, states, O.QConfig())
    assert out["loss"][0] == pytest.approx(L, rel=1e-3)
    for li in range(3):
        for k, name in enumerate(("dV", "dalpha", "dbeta")):
            assert rel_l2(out["grads"][li][k], grads[li][name]) <= GRAD_RTOL, (li, name)


def test_mlp_trajectory(ar):
    Hd, F, M, g, steps = 256, 640, 192, 128, 6
    d, states = _problem(Hd, F, M, g, seed=5, spread=False)
    cfg = ar.ar_qconfig_default(group_size=g)
    ocfg = O.QConfig(group_size=g)
    gm = GpuMlp(ar, d, states, cfg, steps)
    out = gm.step(steps)
    final_gpu = gm.step(0)["loss"][0]
    Ws, X, Y = _oracle_inputs(d)
    st = states
    losses = []
    for _ in range(steps):
        L, st, _, _, _ = O.tune_step_mlp(Ws, X, Y, st, ocfg)
        losses.append(L)
    assert np.allclose(out["loss"], losses, rtol=1e-3)
    for i in range(3):
        q = O.qdq(Ws[i], *st[i], 4, g)["q"]
        assert np.mean(gm.codes(i) == q) >= CODE_AGREE
    assert final_gpu == pytest.approx(O.eval_loss_mlp(Ws, X, Y, st, ocfg), rel=MSE_RTOL)
