"""2-, 3- and 8-bit packed export and the WbA16 matmul (the INT4 layout and the
tcgen05 dequant GEMM generalised; the pages define no packing for these
widths) against the oracle.  Packing follows the oracle's per-row bit stream
(``pack_bitstream``), which at 2, 4 and 8 bits is the per-word layout."""
import numpy as np
import pytest
import torch

import synth
from oracle import autoround_oracle as O

pytestmark = pytest.mark.gpu

# every product (q - z) a is exact and each group's sum is scaled once in fp32, so the
# bf16 rounding of the output (relative 2^-9 per element) bounds the relative L2 error
TC_RTOL = 3e-3


@pytest.fixture(scope="module")
def ar():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import post_weight_quantization_autoround_b200 as m
    m.lib()
    return m


def bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def f32_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def rel_l2(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def pack_gpu(ar, Wbits, V, a, b, bits, g, sym=False):
    N, K = Wbits.shape
    cfg = ar.ar_qconfig_default(bits=bits, group_size=g, symmetric=int(sym))
    packed = torch.empty((N, K * bits // 32), dtype=torch.int32, device="cuda")
    s16 = torch.empty((N, K // g), dtype=torch.float16, device="cuda")
    z16 = torch.empty((N, K // g), dtype=torch.float16, device="cuda")
    ar.ar_pack_codes(bf16_dev(Wbits), f32_dev(V), f32_dev(a), f32_dev(b), cfg, packed, s16, z16)
    return packed, s16, z16


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("g,sym", [(32, False), (128, False), (128, True), (256, False)])
def test_pack_codes_bit_exact(ar, bits, g, sym):
    N, K = 136, 1024
    d = synth.make_linear(N, K, 1, seed=bits + g)
    V, a, b = synth.make_state(N, K, g, seed=4, spread=True)
    packed, s16, z16 = pack_gpu(ar, d["W"], V, a, b, bits, g, sym)
    assert "pack_codes_kernel<b=%d" % bits in ar.ar_last_kernels()
    st = O.qdq(synth.bf16_bits_to_f32(d["W"]), V, a, b, bits, g, sym)
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), O.pack_bitstream(st["q"], bits))
    assert np.array_equal(s16.cpu().numpy(), np.asarray(st["s"], np.float32).astype(np.float16))
    assert np.array_equal(z16.cpu().numpy(), np.asarray(st["zp"], np.float32).astype(np.float16))


@pytest.mark.parametrize("bits", [2, 3, 8])
@pytest.mark.parametrize("T", [1, 5, 16, 40, 256])
@pytest.mark.parametrize("N,K,g", [(320, 1024, 128), (64, 4096, 32), (200, 2048, 256), (1000, 768, 64)])
def test_wxa16_matches_oracle(ar, bits, T, N, K, g):
    d = synth.make_linear(N, K, 1, seed=T + N + bits)
    V, a, b = synth.make_state(N, K, g, seed=2, spread=True)
    packed, s16, z16 = pack_gpu(ar, d["W"], V, a, b, bits, g)
    A = synth.make_activations(T, K, seed=T)
    out = torch.full((T, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    ar.ar_wxa16_gemm(bf16_dev(A), packed, s16, z16, g, bits, out)
    assert ar.ar_get_device_status() == 0
    if bits == 3 or (bits == 2 and T <= 16):
        assert "wbx_dec_kernel<b=%d" % bits in ar.ar_last_kernels()
    else:
        assert "wxa16_tc_kernel<b=%d" % bits in ar.ar_last_kernels()
    st = O.qdq(synth.bf16_bits_to_f32(d["W"]), V, a, b, bits, g)
    words = O.pack_bitstream(st["q"], bits)
    ref = O.wxa16_matmul(synth.bf16_bits_to_f32(A), words, s16.cpu().numpy().view(np.uint16),
                         z16.cpu().numpy().view(np.uint16), g, bits)
    assert rel_l2(out.float().cpu().numpy(), ref) <= TC_RTOL


def test_wxa16_four_bits_is_w4a16(ar):
    N, K, g, T = 256, 1024, 128, 40
    d = synth.make_linear(N, K, 1, seed=5)
    V, a, b = synth.make_state(N, K, g, seed=5, spread=True)
    packed, s16, z16 = pack_gpu(ar, d["W"], V, a, b, 4, g)
    A = bf16_dev(synth.make_activations(T, K, seed=6))
    o1 = torch.empty((T, N), dtype=torch.bfloat16, device="cuda")
    o2 = torch.empty_like(o1)
    ar.ar_wxa16_gemm(A, packed, s16, z16, g, 4, o1)
    ar.ar_w4a16_gemm(A, packed, s16, z16, g, o2)
    assert torch.equal(o1, o2)
