"""Host-only checks of the C ABI: the library loads, exports every declared
entry point, and rejects invalid arguments before any device work.

No call here reaches a kernel: every argument set below fails host-side
validation, so these run without a GPU (pointers are fake, never touched).
"""
import ctypes
import os
import re

import pytest

import post_weight_quantization_autoround_b200 as ar

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "autoround.h")

pytestmark = pytest.mark.skipif(not os.path.exists(ar.library_path), reason="libautoround.so not built")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^AR_API\s+[\w\s\*]+?\b(ar_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_four_hot_path_entry_points():
    syms = declared_symbols()
    for name in ["ar_qdq", "ar_tune_step", "ar_pack_int4", "ar_w4a16_gemm"]:
        assert name in syms


def test_library_exports_every_declared_symbol():
    L = ctypes.CDLL(ar.library_path)
    missing = [s for s in declared_symbols() if not hasattr(L, s)]
    assert not missing, missing
    # the binding wraps every exported entry point under the same name
    for s in declared_symbols():
        assert hasattr(ar, s), s


def test_defaults_follow_the_pages():
    cfg = ar.ar_qconfig_default()
    assert (cfg.bits, cfg.group_size, cfg.symmetric, cfg.iters) == (4, 128, 0, 200)
    assert cfg.lr == pytest.approx(0.005)
    assert (cfg.v_min, cfg.v_max, cfg.clip_min, cfg.clip_max) == (-0.5, 0.5, 0.5, 1.0)
    assert "sm_100a" in ar.ar_version()


FAKE = 0x10000  # 16-byte aligned, never dereferenced


def qdq_raw(cfg, N=8, K=128, W=FAKE, V=FAKE, a=FAKE, b=FAKE, out=FAKE):
    return ar.lib().ar_qdq(W, V, a, b, N, K, ctypes.byref(cfg), out, None, None, None, None)


@pytest.mark.parametrize("bits", [1, 9, 0])
def test_qdq_rejects_unsupported_bits(bits):
    assert qdq_raw(ar.ar_qconfig_default(bits=bits)) == ar.AR_ERR_UNSUPPORTED
    assert "bits" in ar.ar_last_error()


def test_qdq_rejects_bad_shapes_and_pointers():
    cfg = ar.ar_qconfig_default()
    assert qdq_raw(cfg, K=100) == ar.AR_ERR_INVALID_ARG  # K % g != 0
    assert qdq_raw(cfg, N=0) == ar.AR_ERR_INVALID_ARG
    assert qdq_raw(cfg, W=FAKE + 2) == ar.AR_ERR_INVALID_ARG  # misaligned
    assert qdq_raw(cfg, V=None) == ar.AR_ERR_INVALID_ARG
    assert qdq_raw(cfg, out=None) == ar.AR_ERR_INVALID_ARG  # nothing requested
    assert qdq_raw(ar.ar_qconfig_default(group_size=96), K=192) == ar.AR_ERR_UNSUPPORTED
    assert qdq_raw(ar.ar_qconfig_default(symmetric=2)) == ar.AR_ERR_INVALID_ARG
    assert qdq_raw(ar.ar_qconfig_default(lr=float("nan"))) == ar.AR_ERR_INVALID_ARG
    assert qdq_raw(ar.ar_qconfig_default(v_min=1.0, v_max=0.0)) == ar.AR_ERR_INVALID_ARG


def _tune_raw(cfg, N=256, K=256, M=32, ws_bytes=1 << 40, X=FAKE, Y=FAKE, loss=FAKE, n_steps=1, ws=0x100000):
    layer = ar.Layer(FAKE, FAKE, FAKE, FAKE, N, K)
    return ar.lib().ar_tune_step(0, ctypes.byref(layer), 1, X, M, Y, ctypes.byref(cfg), n_steps, loss, None, ws,
                                 ws_bytes, None)


def test_tune_step_validation():
    cfg = ar.ar_qconfig_default()
    assert _tune_raw(ar.ar_qconfig_default(group_size=16)) == ar.AR_ERR_UNSUPPORTED
    assert _tune_raw(ar.ar_qconfig_default(group_size=512), K=1024) == ar.AR_ERR_UNSUPPORTED
    assert _tune_raw(cfg, N=100) == ar.AR_ERR_INVALID_ARG  # N % 8
    assert _tune_raw(cfg, K=200) == ar.AR_ERR_INVALID_ARG  # K % g
    assert _tune_raw(cfg, Y=None) == ar.AR_ERR_INVALID_ARG
    assert _tune_raw(cfg, n_steps=-1) == ar.AR_ERR_INVALID_ARG
    assert _tune_raw(cfg, ws_bytes=16) == ar.AR_ERR_WORKSPACE
    assert _tune_raw(cfg, ws=0x100010) == ar.AR_ERR_INVALID_ARG  # workspace alignment
    layer = ar.Layer(FAKE, FAKE, FAKE, FAKE, 256, 256)
    bad_kind = ar.lib().ar_tune_step(7, ctypes.byref(layer), 1, FAKE, 32, FAKE, ctypes.byref(cfg), 1, FAKE, None,
                                     0x100000, 1 << 40, None)
    assert bad_kind == ar.AR_ERR_UNSUPPORTED


def test_workspace_size_grows_with_steps_and_tokens():
    cfg = ar.ar_qconfig_default()
    layer = ar.Layer(FAKE, FAKE, FAKE, FAKE, 4096, 4096)
    f = ar.lib().ar_tune_step_workspace
    w1 = f(0, ctypes.byref(layer), 1, 16384, ctypes.byref(cfg), 1)
    w200 = f(0, ctypes.byref(layer), 1, 16384, ctypes.byref(cfg), 200)
    w_small = f(0, ctypes.byref(layer), 1, 2048, ctypes.byref(cfg), 1)
    # W_hat (N K bf16) + G (M N bf16) + four per-group arrays + loss partials
    assert w1 >= 4096 * 4096 * 2 + 16384 * 4096 * 2 + 4 * 4096 * 32 * 4
    assert w200 > w1 > w_small > 0
    assert f(5, ctypes.byref(layer), 1, 16384, ctypes.byref(cfg), 1) == 0


def test_pack_and_w4a16_validation():
    cfg3 = ar.ar_qconfig_default(bits=3)
    assert ar.lib().ar_pack_int4(FAKE, FAKE, FAKE, FAKE, 8, 128, ctypes.byref(cfg3), FAKE, FAKE, FAKE, None) == \
        ar.AR_ERR_UNSUPPORTED
    w4 = ar.lib().ar_w4a16_gemm
    assert w4(FAKE, 1 << 31, FAKE, FAKE, FAKE, 64, 256, 128, FAKE, None) == ar.AR_ERR_UNSUPPORTED
    assert w4(FAKE, 1, FAKE, FAKE, FAKE, 64, 4096, 2048, FAKE, None) == ar.AR_ERR_UNSUPPORTED
    assert w4(FAKE, 1, FAKE, FAKE, FAKE, 64, 256, 16, FAKE, None) == ar.AR_ERR_UNSUPPORTED
    assert w4(FAKE, 1, FAKE, FAKE, FAKE, 64, 200, 128, FAKE, None) == ar.AR_ERR_INVALID_ARG
    assert w4(FAKE, 1, FAKE, FAKE, FAKE, 64, 96, 32, FAKE, None) == ar.AR_ERR_INVALID_ARG  # K % 128
    assert w4(FAKE, 0, FAKE, FAKE, FAKE, 64, 256, 128, FAKE, None) == ar.AR_ERR_INVALID_ARG
    assert ar.lib().ar_linear_forward(FAKE, 32, FAKE, 100, 256, FAKE, None) == ar.AR_ERR_INVALID_ARG
    assert ar.lib().ar_gemm_bf16(FAKE, 1, FAKE, 0, FAKE, 12, 64, 64, None) == ar.AR_ERR_INVALID_ARG


def test_debug_wait_validation():
    assert ar.lib().ar_debug_wait_timeout(0, FAKE, None) == ar.AR_ERR_INVALID_ARG
    assert ar.lib().ar_debug_wait_timeout(2_000_000_000, FAKE, None) == ar.AR_ERR_INVALID_ARG
    assert ar.lib().ar_debug_wait_timeout(1000, None, None) == ar.AR_ERR_INVALID_ARG


def test_binding_refuses_host_tensors():
    import torch

    with pytest.raises(ar.ARError):
        ar.ar_f32_to_bf16(torch.zeros(8), torch.zeros(8, dtype=torch.bfloat16))


def test_gather_samples_validation():
    g = ar.lib().ar_gather_samples
    idx = (ctypes.c_int32 * 3)(0, 2, 1)
    assert g(FAKE, 4, 64, idx, 0, 0x20000, None) == ar.AR_ERR_INVALID_ARG           # no samples
    assert g(FAKE, 4, 64, idx, 65, 0x20000, None) == ar.AR_ERR_INVALID_ARG          # more than 64
    assert g(FAKE, 4, 60, idx, 3, 0x20000, None) == ar.AR_ERR_INVALID_ARG           # not a multiple of 16 bytes
    assert g(FAKE, 2, 64, idx, 3, 0x20000, None) == ar.AR_ERR_INVALID_ARG           # index 2 out of range
    assert g(FAKE, 4, 64, idx, 3, FAKE + 64, None) == ar.AR_ERR_INVALID_ARG         # dst overlaps src
    assert g(FAKE + 8, 4, 64, idx, 3, 0x20000, None) == ar.AR_ERR_INVALID_ARG       # misaligned
    assert g(FAKE, 4, 64, None, 3, 0x20000, None) == ar.AR_ERR_INVALID_ARG          # no index array


def test_pack_codes_and_wxa16_validation():
    c5 = ar.ar_qconfig_default(bits=5)
    assert ar.lib().ar_pack_codes(FAKE, FAKE, FAKE, FAKE, 8, 128, ctypes.byref(c5), FAKE, FAKE, FAKE, None) == \
        ar.AR_ERR_UNSUPPORTED
    c3 = ar.ar_qconfig_default(bits=3, group_size=16)
    assert ar.lib().ar_pack_codes(FAKE, FAKE, FAKE, FAKE, 8, 48, ctypes.byref(c3), FAKE, FAKE, FAKE, None) == \
        ar.AR_ERR_INVALID_ARG  # 3-bit rows fill whole words: K % 32
    c2 = ar.ar_qconfig_default(bits=2, group_size=8)
    assert ar.lib().ar_pack_codes(FAKE, FAKE, FAKE, FAKE, 8, 8, ctypes.byref(c2), FAKE, FAKE, FAKE, None) == \
        ar.AR_ERR_INVALID_ARG  # K % 16 for 2-bit words
    w = ar.lib().ar_wxa16_gemm
    assert w(FAKE, 1, FAKE, FAKE, FAKE, 64, 256, 128, 5, FAKE, None) == ar.AR_ERR_UNSUPPORTED
    assert w(FAKE, 1, FAKE, FAKE, FAKE, 64, 256, 16, 2, FAKE, None) == ar.AR_ERR_UNSUPPORTED
    assert w(FAKE, 1, FAKE, FAKE, FAKE, 64, 192, 64, 8, FAKE, None) == ar.AR_ERR_INVALID_ARG  # K % 128
    assert w(FAKE, 0, FAKE, FAKE, FAKE, 64, 256, 128, 2, FAKE, None) == ar.AR_ERR_INVALID_ARG



def test_absmax_and_qdq_nvfp4_validation():
    am = ar.lib().ar_absmax_bf16
    assert am(FAKE, 12, FAKE, None) == ar.AR_ERR_INVALID_ARG          # n % 8
    assert am(FAKE, 0, FAKE, None) == ar.AR_ERR_INVALID_ARG
    assert am(FAKE + 8, 16, FAKE, None) == ar.AR_ERR_INVALID_ARG      # x misaligned
    assert am(FAKE, 16, None, None) == ar.AR_ERR_INVALID_ARG
    q = ar.lib().ar_qdq_nvfp4
    assert q(FAKE, None, None, 4, 40, FAKE, FAKE, None, None, None, None) == ar.AR_ERR_INVALID_ARG   # K % 16
    assert q(FAKE, None, None, 0, 64, FAKE, FAKE, None, None, None, None) == ar.AR_ERR_INVALID_ARG
    assert q(FAKE, None, None, 4, 64, FAKE, None, None, None, None, None) == ar.AR_ERR_INVALID_ARG  # no output
    assert q(FAKE, None, None, 4, 64, None, FAKE, None, None, None, None) == ar.AR_ERR_INVALID_ARG  # no amax
    assert q(FAKE, FAKE + 4, None, 4, 64, FAKE, FAKE, None, None, None, None) == ar.AR_ERR_INVALID_ARG  # V misaligned
    assert q(FAKE, None, FAKE + 2, 4, 64, FAKE, FAKE, None, None, None, None) == ar.AR_ERR_INVALID_ARG  # alpha
    assert q(FAKE, None, None, 4, 64, FAKE, None, FAKE + 8, None, None, None) == ar.AR_ERR_INVALID_ARG  # codes


def test_nvfp4_gemm_validation():
    g = ar.lib().ar_nvfp4_gemm
    assert g(FAKE, 1, FAKE, FAKE, FAKE, 64, 192, FAKE, None) == ar.AR_ERR_INVALID_ARG       # K % 128
    assert g(FAKE, 0, FAKE, FAKE, FAKE, 64, 256, FAKE, None) == ar.AR_ERR_INVALID_ARG       # T
    assert g(FAKE, 1, FAKE, FAKE, FAKE, 0, 256, FAKE, None) == ar.AR_ERR_INVALID_ARG        # N
    assert g(FAKE, 1, FAKE, FAKE + 8, FAKE, 64, 256, FAKE, None) == ar.AR_ERR_INVALID_ARG   # scales misaligned
    assert g(FAKE, 1, FAKE, FAKE, None, 64, 256, FAKE, None) == ar.AR_ERR_INVALID_ARG       # no global scale
    assert g(FAKE, 1, None, FAKE, FAKE, 64, 256, FAKE, None) == ar.AR_ERR_INVALID_ARG       # no codes


def test_tune_step_nvfp4_validation():
    cfg = ar.ar_qconfig_default()
    f = ar.lib().ar_tune_step_nvfp4
    ws = ar.lib().ar_tune_step_nvfp4_workspace

    def call(N=64, K=64, M=32, n_steps=1, ws_bytes=1 << 40, V=FAKE, amax=FAKE, wsp=0x100000):
        return f(FAKE, V, FAKE, N, K, amax, FAKE, M, FAKE, ctypes.byref(cfg), n_steps, FAKE, None, None, wsp,
                 ws_bytes, None)

    assert call(K=40) == ar.AR_ERR_INVALID_ARG          # K % 16
    assert call(N=12) == ar.AR_ERR_INVALID_ARG          # N % 8
    assert call(M=30) == ar.AR_ERR_INVALID_ARG          # M % 8
    assert call(n_steps=-1) == ar.AR_ERR_INVALID_ARG
    assert call(V=None) == ar.AR_ERR_INVALID_ARG
    assert call(amax=None) == ar.AR_ERR_INVALID_ARG
    assert call(ws_bytes=16) == ar.AR_ERR_WORKSPACE
    assert call(wsp=0x100010) == ar.AR_ERR_INVALID_ARG  # workspace alignment
    # W_hat + G + dW_hat + loss partials
    assert ws(16384, 4096, 4096, 1) >= 4096 * 4096 * (2 + 4) + 16384 * 4096 * 2
    assert ws(16384, 4096, 4096, 200) > ws(16384, 4096, 4096, 1) > 0
    assert ws(16384, 4096, 40, 1) == 0


def test_header_is_plain_c_and_a_c_program_links_against_the_library(tmp_path):
    """The boundary is a C ABI: a C99 program (no C++ compiler involved) includes the header, links
    against the library and calls two host-only entry points."""
    import shutil
    import subprocess

    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    src = tmp_path / "use_ar.c"
    src.write_text(
        '#include "autoround.h"\n'
        "int main(void) {\n"
        "  ar_qconfig c;\n"
        "  ar_qconfig_default(&c);\n"
        "  if (c.bits != 4 || c.group_size != 128) return 1;\n"
        "  if (ar_tune_step_nvfp4_workspace(4096, 4096, 4096, 1) == 0) return 2;\n"
        "  if (ar_tune_step_nvfp4_workspace(4096, 4096, 40, 1) != 0) return 3;\n"
        "  return 0;\n"
        "}\n")
    libdir = os.path.dirname(ar.library_path)
    exe = tmp_path / "use_ar"
    subprocess.run([gcc, "-std=c99", "-pedantic-errors", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-L", libdir, "-lautoround", f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    assert subprocess.run([str(exe)]).returncode == 0


def test_tune_step_shard_rejects_a_total_below_the_shard():
    cfg = ar.ar_qconfig_default()
    layer = ar.Layer(FAKE, FAKE, FAKE, FAKE, 256, 256)
    st = ar.lib().ar_tune_step_shard(ctypes.byref(layer), FAKE, 32, FAKE, 128, ctypes.byref(cfg), 1, FAKE, None,
                                     0x100000, 1 << 40, None)
    assert st == ar.AR_ERR_INVALID_ARG
    assert "n_total" in ar.ar_last_error()
