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
    if bits in (2, 3) and T <= 8 and g >= 64 and (K // g) % 8 == 0:
        assert "w%da16_dec_kernel<T<=8" % bits in ar.ar_last_kernels()
    elif bits == 8 and T <= 8 and (K // g) % 8 == 0:
        assert "w8a16_dec_kernel<T<=8" in ar.ar_last_kernels()
    elif bits in (2, 3) and T <= 8:
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


def test_wxa16_three_bit_tensor_core_many_tiles(ar):
    """3-bit codes on the tcgen05 dequant GEMM: K = 4096 is 32 stages of 128 k, four
    three-box code slots of eight stages each; eight row tiles with a ragged last one
    (1000 rows) and a ragged token tail (300 = 2 x 128 + 44)."""
    N, K, g, T = 1000, 4096, 64, 300
    d = synth.make_linear(N, K, 1, seed=31)
    V, a, b = synth.make_state(N, K, g, seed=3, spread=True)
    packed, s16, z16 = pack_gpu(ar, d["W"], V, a, b, 3, g)
    A = synth.make_activations(T, K, seed=32)
    out = torch.full((T, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    ar.ar_wxa16_gemm(bf16_dev(A), packed, s16, z16, g, 3, out)
    assert ar.ar_get_device_status() == 0
    assert "wxa16_tc_kernel<b=3,TN=128" in ar.ar_last_kernels()
    st = O.qdq(synth.bf16_bits_to_f32(d["W"]), V, a, b, 3, g)
    words = O.pack_bitstream(st["q"], 3)
    ref = O.wxa16_matmul(synth.bf16_bits_to_f32(A), words, s16.cpu().numpy().view(np.uint16),
                         z16.cpu().numpy().view(np.uint16), g, 3)
    got = out.float().cpu().numpy()
    for t in range(T):  # every token row, the ragged tail included
        assert rel_l2(got[t], ref[t]) <= TC_RTOL


@pytest.mark.parametrize("T", [17, 256])
def test_wxa16_three_bit_full_size_sampled_rows(ar, T):
    """8192 x 28672 down projection at 3 bits (g 128) on the tensor-core path, sampled
    output rows against the oracle."""
    wl = synth.WORKLOADS["down_8192_28672"]
    N, K, g = wl.n_out, wl.n_in, wl.group_size
    d = synth.make_linear(N, K, 1, seed=wl.seed, x_outlier_channels=0)
    V, a, b = synth.make_state(N, K, g)
    packed, s16, z16 = pack_gpu(ar, d["W"], V, a, b, 3, g)
    A = synth.make_activations(T, K, seed=1)
    out = torch.empty((T, N), dtype=torch.bfloat16, device="cuda")
    ar.ar_wxa16_gemm(bf16_dev(A), packed, s16, z16, g, 3, out)
    assert ar.ar_get_device_status() == 0
    assert "wxa16_tc_kernel<b=3" in ar.ar_last_kernels()
    rows = np.sort(np.random.default_rng(7).choice(N, 64, replace=False))
    st = O.qdq(synth.bf16_bits_to_f32(d["W"][rows]), V[rows], a[rows], b[rows], 3, g)
    words = O.pack_bitstream(st["q"], 3)
    assert np.array_equal(packed.cpu().numpy().view(np.uint32)[rows], words)
    ref = O.wxa16_matmul(synth.bf16_bits_to_f32(A), words, s16.cpu().numpy().view(np.uint16)[rows],
                         z16.cpu().numpy().view(np.uint16)[rows], g, 3)
    assert rel_l2(out.float().cpu().numpy()[:, rows], ref) <= TC_RTOL


@pytest.mark.parametrize("T", [1, 5, 8])
@pytest.mark.parametrize("N,K,g,tag", [
    (10000, 512, 64, "g=64,nt8>"),              # 72 rows per CTA: two row passes (64 + 8); last CTA one pass
    (10000, 1024, 128, "g>=128,nt8>"),          # the same passes with one group per 128-k chunk
    (4096, 2048, 128, "g>=128,ksplit2,nt7>"),   # 56-row CTA pairs splitting K
    (296, 4096, 256, "g>=128,ksplit2,nt1>"),    # 8-row CTA pairs
    (1001, 1024, 128, "g>=128,nt1>"),           # the last CTA holds one row
    (10000, 4096, 128, "g>=128,nt8>"),          # two row passes; 2048-k stages at T = 1
    (2000, 8192, 64, "g=64,nt8>"),              # 16-row CTAs, eight 1024-k stages with 16-group windows
    (296, 8192, 128, "g>=128,ksplit2,nt1>"),    # 8-row CTA pairs, each CTA two 2048-k stages at T = 1
])
def test_w2a16_decode_row_ranges_match_oracle(ar, T, N, K, g, tag):
    """2-bit codes up to 8 tokens on the W4A16 decode kernel's 2-bit form (16 codes a word,
    codes taken at three mantissa positions, activations scaled to match)."""
    d = synth.make_linear(N, K, 1, seed=T + N + 2)
    V, a, b = synth.make_state(N, K, g, seed=2, spread=True)
    packed, s16, z16 = pack_gpu(ar, d["W"], V, a, b, 2, g)
    A = synth.make_activations(T, K, seed=T)
    out = torch.full((T, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    ar.ar_wxa16_gemm(bf16_dev(A), packed, s16, z16, g, 2, out)
    assert ar.ar_get_device_status() == 0
    kern = ar.ar_last_kernels()
    assert "w2a16_dec_kernel<T<=8,%s" % tag in kern, kern
    st = O.qdq(synth.bf16_bits_to_f32(d["W"]), V, a, b, 2, g)
    words = O.pack_bitstream(st["q"], 2)
    ref = O.wxa16_matmul(synth.bf16_bits_to_f32(A), words, s16.cpu().numpy().view(np.uint16),
                         z16.cpu().numpy().view(np.uint16), g, 2)
    got = out.float().cpu().numpy()
    assert rel_l2(got, ref) <= TC_RTOL
    # each token on its own, and the first and last rows (the ends of the row ranges)
    for t in range(T):
        assert rel_l2(got[t], ref[t]) <= TC_RTOL
    assert rel_l2(got[:, :8], ref[:, :8]) <= TC_RTOL and rel_l2(got[:, -8:], ref[:, -8:]) <= TC_RTOL


def test_w2a16_decode_extreme_codes(ar):
    """All-zero and all-three code rows (every code at each of the three mantissa positions at
    its extreme) against the oracle: rows alternate between q = 0 and q = 3 words."""
    N, K, g, T = 64, 1024, 128, 3
    words = np.zeros((N, K // 16), np.uint32)
    words[1::2] = 0xFFFFFFFF
    s16 = np.full((N, K // g), 0.0123, np.float16)
    z16 = np.tile(np.array([0.0, 1.0, 2.0, 3.0], np.float16), (N, K // g // 4))
    A = synth.make_activations(T, K, seed=5)
    out = torch.full((T, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    ar.ar_wxa16_gemm(bf16_dev(A), torch.from_numpy(words.view(np.int32)).cuda(), torch.from_numpy(s16).cuda(),
                     torch.from_numpy(z16).cuda(), g, 2, out)
    assert ar.ar_get_device_status() == 0
    assert "w2a16_dec_kernel<T<=8" in ar.ar_last_kernels()
    ref = O.wxa16_matmul(synth.bf16_bits_to_f32(A), words, s16.view(np.uint16), z16.view(np.uint16), g, 2)
    assert rel_l2(out.float().cpu().numpy(), ref) <= TC_RTOL


@pytest.mark.parametrize("T", [1, 8])
def test_w2a16_decode_full_size_sampled_rows(ar, T):
    """8192 x 28672 down projection at 2 bits (g 128) on the decode kernel, sampled output rows
    against the oracle."""
    wl = synth.WORKLOADS["down_8192_28672"]
    N, K, g = wl.n_out, wl.n_in, wl.group_size
    d = synth.make_linear(N, K, 1, seed=wl.seed, x_outlier_channels=0)
    V, a, b = synth.make_state(N, K, g)
    packed, s16, z16 = pack_gpu(ar, d["W"], V, a, b, 2, g)
    A = synth.make_activations(T, K, seed=1)
    out = torch.empty((T, N), dtype=torch.bfloat16, device="cuda")
    ar.ar_wxa16_gemm(bf16_dev(A), packed, s16, z16, g, 2, out)
    assert ar.ar_get_device_status() == 0
    assert "w2a16_dec_kernel<T<=8" in ar.ar_last_kernels()
    rows = np.sort(np.random.default_rng(7).choice(N, 64, replace=False))
    st = O.qdq(synth.bf16_bits_to_f32(d["W"][rows]), V[rows], a[rows], b[rows], 2, g)
    words = O.pack_bitstream(st["q"], 2)
    assert np.array_equal(packed.cpu().numpy().view(np.uint32)[rows], words)
    ref = O.wxa16_matmul(synth.bf16_bits_to_f32(A), words, s16.cpu().numpy().view(np.uint16)[rows],
                         z16.cpu().numpy().view(np.uint16)[rows], g, 2)
    assert rel_l2(out.float().cpu().numpy()[:, rows], ref) <= TC_RTOL


@pytest.mark.parametrize("T", [1, 5, 8])
@pytest.mark.parametrize("N,K,g,tag", [
    (10000, 512, 64, "g=64,nt8>"),              # 72 rows per CTA: two row passes (64 + 8); last CTA one pass
    (10000, 1024, 128, "g>=128,nt8>"),          # the same passes with one group per 128-k quarter
    (4096, 2048, 128, "g>=128,ksplit2,nt7>"),   # 56-row CTA pairs splitting K
    (296, 4096, 256, "g>=128,ksplit2,nt1>"),    # 8-row CTA pairs
    (1000, 1280, 32, "g=32,nt8>"),              # the last 512-k stage half empty; 16-group windows
    (1001, 1024, 128, "g>=128,nt1>"),           # the last CTA holds one row
])
def test_w8a16_decode_row_ranges_match_oracle(ar, T, N, K, g, tag):
    """8-bit codes up to 8 tokens on the W4A16 decode kernel's 8-bit form (each code split into its
    two nibbles, the high one taken at mantissa bits 3-6 against doubled activations)."""
    d = synth.make_linear(N, K, 1, seed=T + N + 8)
    V, a, b = synth.make_state(N, K, g, seed=2, spread=True)
    packed, s16, z16 = pack_gpu(ar, d["W"], V, a, b, 8, g)
    A = synth.make_activations(T, K, seed=T)
    out = torch.full((T, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    ar.ar_wxa16_gemm(bf16_dev(A), packed, s16, z16, g, 8, out)
    assert ar.ar_get_device_status() == 0
    kern = ar.ar_last_kernels()
    assert "w8a16_dec_kernel<T<=8,%s" % tag in kern, kern
    st = O.qdq(synth.bf16_bits_to_f32(d["W"]), V, a, b, 8, g)
    words = O.pack_bitstream(st["q"], 8)
    ref = O.wxa16_matmul(synth.bf16_bits_to_f32(A), words, s16.cpu().numpy().view(np.uint16),
                         z16.cpu().numpy().view(np.uint16), g, 8)
    got = out.float().cpu().numpy()
    assert rel_l2(got, ref) <= TC_RTOL
    for t in range(T):
        assert rel_l2(got[t], ref[t]) <= TC_RTOL
    assert rel_l2(got[:, :8], ref[:, :8]) <= TC_RTOL and rel_l2(got[:, -8:], ref[:, -8:]) <= TC_RTOL


def test_w8a16_decode_extreme_codes(ar):
    """Codes 0, 255, 0x0F and 0xF0 (each nibble at its extremes) against the oracle."""
    N, K, g, T = 64, 1024, 128, 3
    words = np.zeros((N, K // 4), np.uint32)
    words[1::4] = 0xFFFFFFFF
    words[2::4] = 0x0F0F0F0F
    words[3::4] = 0xF0F0F0F0
    s16 = np.full((N, K // g), 0.0123, np.float16)
    z16 = np.tile(np.array([0.0, 17.0, 128.0, 255.0], np.float16), (N, K // g // 4))
    A = synth.make_activations(T, K, seed=6)
    out = torch.full((T, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    ar.ar_wxa16_gemm(bf16_dev(A), torch.from_numpy(words.view(np.int32)).cuda(), torch.from_numpy(s16).cuda(),
                     torch.from_numpy(z16).cuda(), g, 8, out)
    assert ar.ar_get_device_status() == 0
    assert "w8a16_dec_kernel<T<=8" in ar.ar_last_kernels()
    ref = O.wxa16_matmul(synth.bf16_bits_to_f32(A), words, s16.view(np.uint16), z16.view(np.uint16), g, 8)
    assert rel_l2(out.float().cpu().numpy(), ref) <= TC_RTOL


@pytest.mark.parametrize("T", [1, 8])
def test_w8a16_decode_full_size_sampled_rows(ar, T):
    """8192 x 28672 down projection at 8 bits (g 128) on the decode kernel, sampled output rows
    against the oracle."""
    wl = synth.WORKLOADS["down_8192_28672"]
    N, K, g = wl.n_out, wl.n_in, wl.group_size
    d = synth.make_linear(N, K, 1, seed=wl.seed, x_outlier_channels=0)
    V, a, b = synth.make_state(N, K, g)
    packed, s16, z16 = pack_gpu(ar, d["W"], V, a, b, 8, g)
    A = synth.make_activations(T, K, seed=1)
    out = torch.empty((T, N), dtype=torch.bfloat16, device="cuda")
    ar.ar_wxa16_gemm(bf16_dev(A), packed, s16, z16, g, 8, out)
    assert ar.ar_get_device_status() == 0
    assert "w8a16_dec_kernel<T<=8" in ar.ar_last_kernels()
    rows = np.sort(np.random.default_rng(7).choice(N, 64, replace=False))
    st = O.qdq(synth.bf16_bits_to_f32(d["W"][rows]), V[rows], a[rows], b[rows], 8, g)
    words = O.pack_bitstream(st["q"], 8)
    assert np.array_equal(packed.cpu().numpy().view(np.uint32)[rows], words)
    ref = O.wxa16_matmul(synth.bf16_bits_to_f32(A), words, s16.cpu().numpy().view(np.uint16)[rows],
                         z16.cpu().numpy().view(np.uint16)[rows], g, 8)
    assert rel_l2(out.float().cpu().numpy()[:, rows], ref) <= TC_RTOL


@pytest.mark.parametrize("T", [1, 5, 8])
@pytest.mark.parametrize("N,K,g,tag", [
    (10000, 512, 64, "g=64,nt8>"),              # 72 rows per CTA: two row passes; one half-empty 1024-k stage
    (10000, 1024, 128, "g>=128,nt8>"),          # the same passes with one group per 128 k
    (4096, 2048, 128, "g>=128,ksplit2,nt7>"),   # 56-row CTA pairs splitting K
    (296, 4096, 256, "g>=128,ksplit2,nt1>"),    # 8-row CTA pairs
    (1001, 1024, 128, "g>=128,nt1>"),           # the last CTA holds one row
])
def test_w3a16_decode_row_ranges_match_oracle(ar, T, N, K, g, tag):
    """3-bit codes up to 8 tokens on the W4A16 decode kernel's 3-bit form (a lane's 16 codes read as
    the two aligned words that hold them, codes taken at mantissa bits 0-2 and 3-5)."""
    d = synth.make_linear(N, K, 1, seed=T + N + 3)
    V, a, b = synth.make_state(N, K, g, seed=2, spread=True)
    packed, s16, z16 = pack_gpu(ar, d["W"], V, a, b, 3, g)
    A = synth.make_activations(T, K, seed=T)
    out = torch.full((T, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    ar.ar_wxa16_gemm(bf16_dev(A), packed, s16, z16, g, 3, out)
    assert ar.ar_get_device_status() == 0
    kern = ar.ar_last_kernels()
    assert "w3a16_dec_kernel<T<=8,%s" % tag in kern, kern
    st = O.qdq(synth.bf16_bits_to_f32(d["W"]), V, a, b, 3, g)
    words = O.pack_bitstream(st["q"], 3)
    ref = O.wxa16_matmul(synth.bf16_bits_to_f32(A), words, s16.cpu().numpy().view(np.uint16),
                         z16.cpu().numpy().view(np.uint16), g, 3)
    got = out.float().cpu().numpy()
    assert rel_l2(got, ref) <= TC_RTOL
    for t in range(T):
        assert rel_l2(got[t], ref[t]) <= TC_RTOL
    assert rel_l2(got[:, :8], ref[:, :8]) <= TC_RTOL and rel_l2(got[:, -8:], ref[:, -8:]) <= TC_RTOL


def test_w3a16_decode_extreme_codes(ar):
    """All-zero and all-seven code rows (every code, straddling ones included, at its extremes)."""
    N, K, g, T = 64, 1024, 128, 3
    words = np.zeros((N, K * 3 // 32), np.uint32)
    words[1::2] = 0xFFFFFFFF
    s16 = np.full((N, K // g), 0.0123, np.float16)
    z16 = np.tile(np.array([0.0, 3.0, 4.0, 7.0], np.float16), (N, K // g // 4))
    A = synth.make_activations(T, K, seed=7)
    out = torch.full((T, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    ar.ar_wxa16_gemm(bf16_dev(A), torch.from_numpy(words.view(np.int32)).cuda(), torch.from_numpy(s16).cuda(),
                     torch.from_numpy(z16).cuda(), g, 3, out)
    assert ar.ar_get_device_status() == 0
    assert "w3a16_dec_kernel<T<=8" in ar.ar_last_kernels()
    ref = O.wxa16_matmul(synth.bf16_bits_to_f32(A), words, s16.view(np.uint16), z16.view(np.uint16), g, 3)
    assert rel_l2(out.float().cpu().numpy(), ref) <= TC_RTOL


@pytest.mark.parametrize("T", [1, 8])
def test_w3a16_decode_full_size_sampled_rows(ar, T):
    """8192 x 28672 down projection at 3 bits (g 128) on the decode kernel, sampled output rows
    against the oracle."""
    wl = synth.WORKLOADS["down_8192_28672"]
    N, K, g = wl.n_out, wl.n_in, wl.group_size
    d = synth.make_linear(N, K, 1, seed=wl.seed, x_outlier_channels=0)
    V, a, b = synth.make_state(N, K, g)
    packed, s16, z16 = pack_gpu(ar, d["W"], V, a, b, 3, g)
    A = synth.make_activations(T, K, seed=1)
    out = torch.empty((T, N), dtype=torch.bfloat16, device="cuda")
    ar.ar_wxa16_gemm(bf16_dev(A), packed, s16, z16, g, 3, out)
    assert ar.ar_get_device_status() == 0
    assert "w3a16_dec_kernel<T<=8" in ar.ar_last_kernels()
    rows = np.sort(np.random.default_rng(7).choice(N, 64, replace=False))
    st = O.qdq(synth.bf16_bits_to_f32(d["W"][rows]), V[rows], a[rows], b[rows], 3, g)
    words = O.pack_bitstream(st["q"], 3)
    assert np.array_equal(packed.cpu().numpy().view(np.uint32)[rows], words)
    ref = O.wxa16_matmul(synth.bf16_bits_to_f32(A), words, s16.cpu().numpy().view(np.uint16)[rows],
                         z16.cpu().numpy().view(np.uint16)[rows], g, 3)
    assert rel_l2(out.float().cpu().numpy()[:, rows], ref) <= TC_RTOL
