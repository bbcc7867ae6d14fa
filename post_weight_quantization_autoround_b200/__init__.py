"""Python binding of libautoround.so: AutoRound tuning step, INT4 export, W4A16 matmul on B200.

Argument marshalling only.  Every function below has the name of the C entry
point it calls (``include/autoround.h``); tensors are ``torch`` CUDA tensors
(bf16 tensors as ``torch.bfloat16``, fp16 bit patterns as ``torch.float16``),
streams default to the current torch stream.  There is no CPU path: importing
works without a GPU, but every call needs the built library and a CUDA device
and raises :class:`ARError` otherwise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

__all__ = [
    "ARError", "QConfig", "Layer", "Grads", "lib", "library_path",
    "ar_qconfig_default", "ar_f32_to_bf16", "ar_qdq", "ar_linear_forward", "ar_tune_step_workspace",
    "ar_tune_step", "ar_pack_int4", "ar_w4a16_gemm", "ar_gemm_bf16", "ar_get_device_status",
    "ar_last_error", "ar_last_kernels", "ar_version", "ar_profile_start", "ar_profile_stop", "AR_BLOCK_LINEAR",
    "ar_tune_step_noalloc", "AR_NOALLOC_SCRATCH_BYTES", "AR_BLOCK_SWIGLU_MLP", "ar_block_forward",
    "ar_block_forward_workspace", "ar_tune_block", "ar_tune_block_workspace", "ar_debug_wait_timeout",
    "ar_absmax_bf16", "ar_qdq_nvfp4", "ar_nvfp4_gemm", "ar_tune_step_nvfp4_workspace", "ar_tune_step_nvfp4",
    "ar_tune_step_shard", "DecoderCfg", "DECODER_LAYERS", "ar_decoder_forward_workspace", "ar_decoder_forward",
    "ar_tune_step_decoder_workspace", "ar_tune_step_decoder", "ar_rmsnorm", "ar_attention_forward",
    "ar_attention_backward_workspace", "ar_attention_backward",
]

library_path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libautoround.so")

AR_OK, AR_ERR_INVALID_ARG, AR_ERR_UNSUPPORTED, AR_ERR_CUDA, AR_ERR_NONFINITE, AR_ERR_TIMEOUT, AR_ERR_WORKSPACE = range(7)
_STATUS_NAMES = ["AR_OK", "AR_ERR_INVALID_ARG", "AR_ERR_UNSUPPORTED", "AR_ERR_CUDA", "AR_ERR_NONFINITE",
                 "AR_ERR_TIMEOUT", "AR_ERR_WORKSPACE"]
AR_BLOCK_LINEAR = 0
AR_BLOCK_SWIGLU_MLP = 1


class ARError(RuntimeError):
    """A non-zero ``ar_status`` from the library, with its ``ar_last_error()`` text."""

    def __init__(self, status: int, message: str):
        name = _STATUS_NAMES[status] if 0 <= status < len(_STATUS_NAMES) else str(status)
        super().__init__(f"{name}: {message}")
        self.status = status


class QConfig(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int), ("group_size", ctypes.c_int), ("symmetric", ctypes.c_int),
                ("lr", ctypes.c_float), ("iters", ctypes.c_int), ("v_min", ctypes.c_float),
                ("v_max", ctypes.c_float), ("clip_min", ctypes.c_float), ("clip_max", ctypes.c_float)]


class Layer(ctypes.Structure):
    _fields_ = [("W", ctypes.c_void_p), ("V", ctypes.c_void_p), ("alpha", ctypes.c_void_p),
                ("beta", ctypes.c_void_p), ("N", ctypes.c_int64), ("K", ctypes.c_int64)]


class Grads(ctypes.Structure):
    _fields_ = [("dV", ctypes.c_void_p), ("dalpha", ctypes.c_void_p), ("dbeta", ctypes.c_void_p)]


class DecoderCfg(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int64), ("intermediate", ctypes.c_int64), ("n_heads", ctypes.c_int),
                ("seq_len", ctypes.c_int64), ("gamma1", ctypes.c_void_p), ("gamma2", ctypes.c_void_p)]


DECODER_LAYERS = ("q", "k", "v", "o", "gate", "up", "down")

_lib = None
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_INT = ctypes.c_int

_SIGNATURES = {
    "ar_qconfig_default": (None, [ctypes.POINTER(QConfig)]),
    "ar_f32_to_bf16": (_INT, [_P, _P, _I64, _P]),
    "ar_qdq": (_INT, [_P, _P, _P, _P, _I64, _I64, ctypes.POINTER(QConfig), _P, _P, _P, _P, _P]),
    "ar_linear_forward": (_INT, [_P, _I64, _P, _I64, _I64, _P, _P]),
    "ar_tune_step_workspace": (ctypes.c_size_t, [_INT, ctypes.POINTER(Layer), _INT, _I64, ctypes.POINTER(QConfig), _INT]),
    "ar_tune_step": (_INT, [_INT, ctypes.POINTER(Layer), _INT, _P, _I64, _P, ctypes.POINTER(QConfig), _INT, _P,
                            ctypes.POINTER(Grads), _P, ctypes.c_size_t, _P]),
    "ar_tune_step_shard": (_INT, [ctypes.POINTER(Layer), _P, _I64, _P, _I64, ctypes.POINTER(QConfig), _INT, _P,
                                  ctypes.POINTER(Grads), _P, ctypes.c_size_t, _P]),
    "ar_decoder_forward_workspace": (ctypes.c_size_t, [ctypes.POINTER(DecoderCfg), _I64]),
    "ar_decoder_forward": (_INT, [ctypes.POINTER(DecoderCfg), ctypes.POINTER(Layer), _P, _I64, _P, _P, ctypes.c_size_t,
                                  _P]),
    "ar_tune_step_decoder_workspace": (ctypes.c_size_t, [ctypes.POINTER(DecoderCfg), ctypes.POINTER(Layer), _I64,
                                                         ctypes.POINTER(QConfig), _INT]),
    "ar_tune_step_decoder": (_INT, [ctypes.POINTER(DecoderCfg), ctypes.POINTER(Layer), _P, _I64, _P,
                                    ctypes.POINTER(QConfig), _INT, _P, ctypes.POINTER(Grads), _P, ctypes.c_size_t,
                                    _P]),
    "ar_rmsnorm": (_INT, [_P, _INT, _P, _I64, _I64, _P, _P, _P]),
    "ar_attention_forward": (_INT, [_P, _I64, _I64, _I64, _INT, _P, _P, _P]),
    "ar_attention_backward_workspace": (ctypes.c_size_t, [_I64, _I64, _I64, _INT]),
    "ar_attention_backward": (_INT, [_P, _P, _P, _P, _I64, _I64, _I64, _INT, _P, _P, ctypes.c_size_t, _P]),
    "ar_pack_int4": (_INT, [_P, _P, _P, _P, _I64, _I64, ctypes.POINTER(QConfig), _P, _P, _P, _P]),
    "ar_w4a16_gemm": (_INT, [_P, _I64, _P, _P, _P, _I64, _I64, _INT, _P, _P]),
    "ar_gemm_bf16": (_INT, [_P, _INT, _P, _INT, _P, _I64, _I64, _I64, _P]),
    "ar_get_device_status": (_INT, [_P]),
    "ar_last_error": (ctypes.c_char_p, []),
    "ar_last_kernels": (ctypes.c_char_p, []),
    "ar_version": (ctypes.c_char_p, []),
    "ar_block_forward_workspace": (ctypes.c_size_t, [_INT, ctypes.POINTER(Layer), _INT, _I64]),
    "ar_block_forward": (_INT, [_INT, ctypes.POINTER(Layer), _INT, _P, _I64, _P, _P, ctypes.c_size_t, _P]),
    "ar_tune_step_noalloc": (_INT, [_INT, ctypes.POINTER(Layer), _INT, _P, _I64, _P, ctypes.POINTER(QConfig), _INT,
                                    _P, ctypes.POINTER(Grads), _P]),
    "ar_debug_wait_timeout": (_INT, [ctypes.c_uint64, _P, _P]),
    "ar_profile_start": (_INT, []),
    "ar_profile_stop": (_INT, [ctypes.c_char_p, ctypes.c_size_t]),
    "ar_gather_samples": (_INT, [_P, _I64, _I64, ctypes.POINTER(ctypes.c_int32), _INT, _P, _P]),
    "ar_pack_codes": (_INT, [_P, _P, _P, _P, _I64, _I64, ctypes.POINTER(QConfig), _P, _P, _P, _P]),
    "ar_wxa16_gemm": (_INT, [_P, _I64, _P, _P, _P, _I64, _I64, _INT, _INT, _P, _P]),
    "ar_absmax_bf16": (_INT, [_P, _I64, _P, _P]),
    "ar_qdq_nvfp4": (_INT, [_P, _P, _P, _I64, _I64, _P, _P, _P, _P, _P, _P]),
    "ar_nvfp4_gemm": (_INT, [_P, _I64, _P, _P, _P, _I64, _I64, _P, _P]),
    "ar_tune_step_nvfp4_workspace": (ctypes.c_size_t, [_I64, _I64, _I64, _INT]),
    "ar_tune_step_nvfp4": (_INT, [_P, _P, _P, _I64, _I64, _P, _P, _I64, _P, ctypes.POINTER(QConfig), _INT, _P, _P, _P,
                                  _P, ctypes.c_size_t, _P]),
}


def lib() -> ctypes.CDLL:
    """Load libautoround.so (built in-tree by ``build.py``); raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(library_path):
            raise ARError(AR_ERR_UNSUPPORTED, f"{library_path} is not built; run "
                          "`python -m post_weight_quantization_autoround_b200.build`")
        L = ctypes.CDLL(library_path)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ARError(AR_ERR_INVALID_ARG, "tensor must be on a CUDA device")
    if not t.is_contiguous():
        raise ARError(AR_ERR_INVALID_ARG, "tensor must be contiguous")
    return t.data_ptr()


def _check(status: int):
    if status != AR_OK:
        raise ARError(status, lib().ar_last_error().decode())


def ar_last_error() -> str:
    return lib().ar_last_error().decode()


def ar_last_kernels() -> str:
    return lib().ar_last_kernels().decode()


def ar_version() -> str:
    return lib().ar_version().decode()


def ar_qconfig_default(**overrides) -> QConfig:
    cfg = QConfig()
    lib().ar_qconfig_default(ctypes.byref(cfg))
    for k, v in overrides.items():
        setattr(cfg, k, v)
    return cfg


def ar_f32_to_bf16(src: torch.Tensor, dst: torch.Tensor, stream=None) -> None:
    _check(lib().ar_f32_to_bf16(_ptr(src), _ptr(dst), src.numel(), _stream(stream)))


def ar_qdq(W, V, alpha, beta, cfg: QConfig, W_hat=None, codes=None, scale=None, zero=None, stream=None) -> None:
    N, K = W.shape
    _check(lib().ar_qdq(_ptr(W), _ptr(V), _ptr(alpha), _ptr(beta), N, K, ctypes.byref(cfg), _ptr(W_hat),
                        _ptr(codes), _ptr(scale), _ptr(zero), _stream(stream)))


def ar_linear_forward(X, W, Y, stream=None) -> None:
    M, K = X.shape
    N = W.shape[0]
    _check(lib().ar_linear_forward(_ptr(X), M, _ptr(W), N, K, _ptr(Y), _stream(stream)))


def _layer(W, V, alpha, beta) -> Layer:
    N, K = W.shape
    return Layer(_ptr(W), _ptr(V), _ptr(alpha), _ptr(beta), N, K)


def ar_tune_step_workspace(W, V, alpha, beta, M: int, cfg: QConfig, n_steps: int,
                           block_kind: int = AR_BLOCK_LINEAR) -> int:
    layer = _layer(W, V, alpha, beta)
    n = lib().ar_tune_step_workspace(block_kind, ctypes.byref(layer), 1, M, ctypes.byref(cfg), n_steps)
    if n == 0:
        raise ARError(AR_ERR_INVALID_ARG, ar_last_error())
    return int(n)


def ar_tune_step(W, V, alpha, beta, X, Y, cfg: QConfig, n_steps: int, loss, workspace,
                 dV=None, dalpha=None, dbeta=None, stream=None, block_kind: int = AR_BLOCK_LINEAR) -> None:
    """Run ``n_steps`` tuning steps; V, alpha, beta are updated in place, losses go to ``loss``."""
    layer = _layer(W, V, alpha, beta)
    grads = Grads(_ptr(dV), _ptr(dalpha), _ptr(dbeta))
    gp = ctypes.byref(grads) if (dV is not None or dalpha is not None or dbeta is not None) else None
    _check(lib().ar_tune_step(block_kind, ctypes.byref(layer), 1, _ptr(X), X.shape[0], _ptr(Y), ctypes.byref(cfg),
                              n_steps, _ptr(loss), gp, _ptr(workspace), workspace.numel() * workspace.element_size(),
                              _stream(stream)))


def ar_tune_step_shard(W, V, alpha, beta, X, Y, n_total: int, cfg: QConfig, n_steps: int, loss, workspace,
                       dV=None, dalpha=None, dbeta=None, stream=None) -> None:
    """``ar_tune_step`` on a shard of a layer's output rows (W, V, alpha, beta hold this shard's rows, Y its
    columns); ``n_total`` is the whole layer's row count, which sets the loss normaliser."""
    layer = _layer(W, V, alpha, beta)
    grads = Grads(_ptr(dV), _ptr(dalpha), _ptr(dbeta))
    gp = ctypes.byref(grads) if (dV is not None or dalpha is not None or dbeta is not None) else None
    _check(lib().ar_tune_step_shard(ctypes.byref(layer), _ptr(X), X.shape[0], _ptr(Y), n_total, ctypes.byref(cfg),
                                    n_steps, _ptr(loss), gp, _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream(stream)))


def _layers(ws):
    """ctypes array of Layer from a list of (W, V, alpha, beta) tuples (V/alpha/beta may be None)."""
    arr = (Layer * len(ws))()
    for i, (W, V, a, b) in enumerate(ws):
        N, K = W.shape
        arr[i] = Layer(_ptr(W), _ptr(V), _ptr(a), _ptr(b), N, K)
    return arr


def ar_block_forward_workspace(block_kind: int, weights, M: int) -> int:
    arr = _layers([(W, None, None, None) for W in weights])
    n = lib().ar_block_forward_workspace(block_kind, arr, len(weights), M)
    if n == 0:
        raise ARError(AR_ERR_INVALID_ARG, ar_last_error())
    return int(n)


def ar_block_forward(block_kind: int, weights, X, Y, workspace, stream=None) -> None:
    """Reference output of a block with its original weights (list of W tensors)."""
    arr = _layers([(W, None, None, None) for W in weights])
    _check(lib().ar_block_forward(block_kind, arr, len(weights), _ptr(X), X.shape[0], _ptr(Y), _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _stream(stream)))


def ar_tune_block_workspace(block_kind: int, layers, M: int, cfg: QConfig, n_steps: int) -> int:
    """``ar_tune_step_workspace`` for a block given as a list of (W, V, alpha, beta)."""
    arr = _layers(layers)
    n = lib().ar_tune_step_workspace(block_kind, arr, len(layers), M, ctypes.byref(cfg), n_steps)
    if n == 0:
        raise ARError(AR_ERR_INVALID_ARG, ar_last_error())
    return int(n)


def ar_tune_block(block_kind: int, layers, X, Y, cfg: QConfig, n_steps: int, loss, workspace, grads=None,
                  stream=None) -> None:
    """``ar_tune_step`` for a block given as a list of (W, V, alpha, beta); grads: list of (dV, dalpha, dbeta)."""
    arr = _layers(layers)
    gp = None
    if grads is not None:
        g = (Grads * len(layers))()
        for i, (dv, da, db) in enumerate(grads):
            g[i] = Grads(_ptr(dv), _ptr(da), _ptr(db))
        gp = g
    _check(lib().ar_tune_step(block_kind, arr, len(layers), _ptr(X), X.shape[0], _ptr(Y), ctypes.byref(cfg), n_steps,
                              _ptr(loss), gp, _ptr(workspace), workspace.numel() * workspace.element_size(),
                              _stream(stream)))


AR_NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024


def ar_tune_step_noalloc(W, V, alpha, beta, X, Y, cfg: QConfig, n_steps: int, loss,
                         dV=None, dalpha=None, dbeta=None, stream=None, block_kind: int = AR_BLOCK_LINEAR) -> None:
    """``ar_tune_step`` without a workspace, for callers that cannot allocate device memory.

    The scratch is a fixed device array of ``AR_NOALLOC_SCRATCH_BYTES`` inside
    the library, shared by all calls on a device (serialise overlapping calls);
    larger problems raise ``ARError`` (AR_ERR_WORKSPACE).
    """
    layer = _layer(W, V, alpha, beta)
    grads = Grads(_ptr(dV), _ptr(dalpha), _ptr(dbeta))
    gp = ctypes.byref(grads) if (dV is not None or dalpha is not None or dbeta is not None) else None
    _check(lib().ar_tune_step_noalloc(block_kind, ctypes.byref(layer), 1, _ptr(X), X.shape[0], _ptr(Y),
                                      ctypes.byref(cfg), n_steps, _ptr(loss), gp, _stream(stream)))


def ar_pack_int4(W, V, alpha, beta, cfg: QConfig, packed, scale16, zero16, stream=None) -> None:
    N, K = W.shape
    _check(lib().ar_pack_int4(_ptr(W), _ptr(V), _ptr(alpha), _ptr(beta), N, K, ctypes.byref(cfg), _ptr(packed),
                              _ptr(scale16), _ptr(zero16), _stream(stream)))


def ar_w4a16_gemm(A, packed, scale16, zero16, group_size: int, out, stream=None) -> None:
    T, K = A.shape
    N = packed.shape[0]
    _check(lib().ar_w4a16_gemm(_ptr(A), T, _ptr(packed), _ptr(scale16), _ptr(zero16), N, K, group_size, _ptr(out),
                               _stream(stream)))


def ar_pack_codes(W, V, alpha, beta, cfg: QConfig, packed, scale16, zero16, stream=None) -> None:
    """cfg.bits in {2, 4, 8}: packed uint32 [N][K*bits/32] (as int32 tensor), fp16 scale/zero [N][K/g]."""
    N, K = W.shape
    _check(lib().ar_pack_codes(_ptr(W), _ptr(V), _ptr(alpha), _ptr(beta), N, K, ctypes.byref(cfg), _ptr(packed),
                               _ptr(scale16), _ptr(zero16), _stream(stream)))


def ar_wxa16_gemm(A, packed, scale16, zero16, group_size: int, bits: int, out, stream=None) -> None:
    T, K = A.shape
    N = packed.shape[0]
    _check(lib().ar_wxa16_gemm(_ptr(A), T, _ptr(packed), _ptr(scale16), _ptr(zero16), N, K, group_size, bits,
                               _ptr(out), _stream(stream)))


def ar_gather_samples(src, idx, dst, stream=None) -> None:
    """dst[i] = src[idx[i]] for whole samples (first dimension); idx: host sequence of ints."""
    n_src = src.shape[0]
    sample_bytes = src[0].numel() * src.element_size() if n_src else 0
    arr = (ctypes.c_int32 * len(idx))(*[int(i) for i in idx])
    if dst.shape[0] != len(idx) or dst[0].numel() * dst.element_size() != sample_bytes:
        raise ARError(AR_ERR_INVALID_ARG, "dst must hold len(idx) samples of src's size")
    _check(lib().ar_gather_samples(_ptr(src), n_src, sample_bytes, arr, len(idx), _ptr(dst), _stream(stream)))


def ar_absmax_bf16(x, amax, stream=None) -> None:
    """amax (fp32 device scalar) = max |x| over a bf16 device tensor."""
    _check(lib().ar_absmax_bf16(_ptr(x), x.numel(), _ptr(amax), _stream(stream)))


def ar_qdq_nvfp4(W, V, alpha, amax, W_hat=None, codes=None, scales=None, global_scale=None, stream=None) -> None:
    """NVFP4 fake quantization of W [N][K] (bf16): V [N][K] fp32 or None, alpha [N][K/16] fp32 or None,
    amax fp32 device scalar (``ar_absmax_bf16`` of W); outputs W_hat bf16 [N][K], codes uint8 [N][K/2],
    scales uint8 [N][K/16] (E4M3 codes), global_scale fp32 scalar."""
    N, K = W.shape
    _check(lib().ar_qdq_nvfp4(_ptr(W), _ptr(V), _ptr(alpha), N, K, _ptr(amax), _ptr(W_hat), _ptr(codes),
                              _ptr(scales), _ptr(global_scale), _stream(stream)))


def ar_nvfp4_gemm(A, codes, scales, global_scale, out, stream=None) -> None:
    """out [T][N] bf16 = A [T][K] bf16 times the NVFP4 weights: codes uint8 [N][K/2], scales uint8
    [N][K/16] (E4M3 codes), global_scale fp32 device scalar (as ``ar_qdq_nvfp4`` writes them)."""
    T, K = A.shape
    N = codes.shape[0]
    _check(lib().ar_nvfp4_gemm(_ptr(A), T, _ptr(codes), _ptr(scales), _ptr(global_scale), N, K, _ptr(out),
                               _stream(stream)))


def ar_tune_step_nvfp4_workspace(M: int, N: int, K: int, n_steps: int) -> int:
    n = lib().ar_tune_step_nvfp4_workspace(M, N, K, n_steps)
    if n == 0:
        raise ARError(AR_ERR_INVALID_ARG, ar_last_error())
    return n


def ar_tune_step_nvfp4(W, V, alpha, amax, X, Y, cfg: QConfig, n_steps: int, loss_per_step, workspace,
                       dV=None, dalpha=None, stream=None) -> None:
    """``n_steps`` SignSGD steps of one linear layer on NVFP4 (V [N][K], alpha [N][K/16] updated in place);
    loss_per_step: fp32 device [max(n_steps, 1)]; workspace: uint8 device tensor of
    ``ar_tune_step_nvfp4_workspace`` bytes."""
    N, K = W.shape
    M = X.shape[0]
    _check(lib().ar_tune_step_nvfp4(_ptr(W), _ptr(V), _ptr(alpha), N, K, _ptr(amax), _ptr(X), M, _ptr(Y),
                                    ctypes.byref(cfg), n_steps, _ptr(loss_per_step), _ptr(dV), _ptr(dalpha),
                                    _ptr(workspace), workspace.numel(), _stream(stream)))


def ar_gemm_bf16(A, a_mn_major: bool, B, b_mn_major: bool, D, M: int, N: int, K: int, stream=None) -> None:
    _check(lib().ar_gemm_bf16(_ptr(A), int(a_mn_major), _ptr(B), int(b_mn_major), _ptr(D), M, N, K,
                              _stream(stream)))


def ar_profile_start() -> None:
    _check(lib().ar_profile_start())


def ar_profile_stop() -> dict:
    """Stop device-time profiling; returns {kernel name: (launches, total ms)}."""
    buf = ctypes.create_string_buffer(1 << 16)
    _check(lib().ar_profile_stop(buf, len(buf)))
    out = {}
    for line in buf.value.decode().splitlines():
        name, n, ms = line.rsplit(" ", 2)
        out[name] = (int(n), float(ms))
    return out


def ar_debug_wait_timeout(limit_ns: int, gave_up, stream=None) -> None:
    """Run the bounded-wait diagnostic: a wait on a barrier nothing completes gives up after limit_ns."""
    _check(lib().ar_debug_wait_timeout(int(limit_ns), _ptr(gave_up), _stream(stream)))


def ar_get_device_status(stream=None) -> int:
    """Synchronise and return (and clear) the sticky device status code."""
    return int(lib().ar_get_device_status(_stream(stream)))


class LinearTuner:
    """Device buffers for tuning one linear layer from host memory (the end-to-end path).

    ``run_host`` copies W, X and the state (V, alpha, beta) from pinned host
    tensors to the device, computes the reference output, runs ``n_steps``
    tuning steps and copies the tuned state and the per-step losses back into
    the host tensors.  Device memory is allocated once here, so repeated runs
    allocate nothing.
    """

    def __init__(self, N: int, K: int, M: int, cfg: QConfig, n_steps: int, device=None):
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        g = cfg.group_size
        self.cfg, self.n_steps = cfg, n_steps
        self.W = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
        self.X = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
        self.V = torch.empty((N, K), dtype=torch.float32, device=dev)
        self.alpha = torch.empty((N, K // g), dtype=torch.float32, device=dev)
        self.beta = torch.empty((N, K // g), dtype=torch.float32, device=dev)
        self.Y = torch.empty((M, N), dtype=torch.float32, device=dev)
        self.loss = torch.empty(max(n_steps, 1), dtype=torch.float32, device=dev)
        nbytes = ar_tune_step_workspace(self.W, self.V, self.alpha, self.beta, M, cfg, n_steps)
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)

    def h2d_bytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in (self.W, self.X, self.V, self.alpha, self.beta))

    def d2h_bytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in (self.V, self.alpha, self.beta, self.loss))

    def run_host(self, W, X, V, alpha, beta, loss, stream=None) -> None:
        for dst, src in ((self.W, W), (self.X, X), (self.V, V), (self.alpha, alpha), (self.beta, beta)):
            dst.copy_(src, non_blocking=True)
        ar_linear_forward(self.X, self.W, self.Y, stream=stream)
        ar_tune_step(self.W, self.V, self.alpha, self.beta, self.X, self.Y, self.cfg, self.n_steps, self.loss,
                     self.workspace, stream=stream)
        for dst, src in ((V, self.V), (alpha, self.alpha), (beta, self.beta), (loss, self.loss)):
            dst.copy_(src, non_blocking=True)


# ---- decoder block ----------------------------------------------------------

def _decoder_cfg(H: int, F: int, n_heads: int, seq_len: int, gamma1, gamma2) -> DecoderCfg:
    return DecoderCfg(H, F, n_heads, seq_len, _ptr(gamma1), _ptr(gamma2))


def ar_decoder_forward_workspace(H: int, F: int, n_heads: int, seq_len: int, M: int) -> int:
    d = DecoderCfg(H, F, n_heads, seq_len, None, None)
    n = lib().ar_decoder_forward_workspace(ctypes.byref(d), M)
    if n == 0:
        raise ARError(AR_ERR_INVALID_ARG, ar_last_error())
    return int(n)


def ar_decoder_forward(weights, gamma1, gamma2, n_heads: int, seq_len: int, X, Y, workspace, stream=None) -> None:
    """Block output with the original weights; ``weights``: seven W tensors in DECODER_LAYERS order."""
    H, F = weights[0].shape[0], weights[4].shape[0]
    d = _decoder_cfg(H, F, n_heads, seq_len, gamma1, gamma2)
    arr = _layers([(W, None, None, None) for W in weights])
    _check(lib().ar_decoder_forward(ctypes.byref(d), arr, _ptr(X), X.shape[0], _ptr(Y), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream(stream)))


def ar_tune_step_decoder_workspace(layers, gamma1, gamma2, n_heads: int, seq_len: int, M: int, cfg: QConfig,
                                   n_steps: int) -> int:
    H, F = layers[0][0].shape[0], layers[4][0].shape[0]
    d = _decoder_cfg(H, F, n_heads, seq_len, gamma1, gamma2)
    n = lib().ar_tune_step_decoder_workspace(ctypes.byref(d), _layers(layers), M, ctypes.byref(cfg), n_steps)
    if n == 0:
        raise ARError(AR_ERR_INVALID_ARG, ar_last_error())
    return int(n)


def ar_tune_step_decoder(layers, gamma1, gamma2, n_heads: int, seq_len: int, X, Y, cfg: QConfig, n_steps: int, loss,
                         workspace, grads=None, stream=None) -> None:
    """Joint steps on the decoder block; ``layers``: seven (W, V, alpha, beta) in DECODER_LAYERS order."""
    H, F = layers[0][0].shape[0], layers[4][0].shape[0]
    d = _decoder_cfg(H, F, n_heads, seq_len, gamma1, gamma2)
    gp = None
    if grads is not None:
        g = (Grads * len(layers))()
        for i, (dv, da, db) in enumerate(grads):
            g[i] = Grads(_ptr(dv), _ptr(da), _ptr(db))
        gp = g
    _check(lib().ar_tune_step_decoder(ctypes.byref(d), _layers(layers), _ptr(X), X.shape[0], _ptr(Y),
                                      ctypes.byref(cfg), n_steps, _ptr(loss), gp, _ptr(workspace),
                                      workspace.numel() * workspace.element_size(), _stream(stream)))


def ar_rmsnorm(x, gamma, r, inv=None, stream=None) -> None:
    M, H = x.shape
    _check(lib().ar_rmsnorm(_ptr(x), int(x.dtype == torch.float32), _ptr(gamma), M, H, _ptr(r), _ptr(inv),
                            _stream(stream)))


def ar_attention_forward(qkv, S: int, L: int, n_heads: int, out, lse, stream=None) -> None:
    H = qkv.shape[1] // 3
    _check(lib().ar_attention_forward(_ptr(qkv), S, L, H, n_heads, _ptr(out), _ptr(lse), _stream(stream)))


def ar_attention_backward_workspace(S: int, L: int, H: int, n_heads: int) -> int:
    n = lib().ar_attention_backward_workspace(S, L, H, n_heads)
    if n == 0:
        raise ARError(AR_ERR_INVALID_ARG, ar_last_error())
    return int(n)


def ar_attention_backward(qkv, out, dout, lse, S: int, L: int, n_heads: int, dqkv, workspace, stream=None) -> None:
    H = qkv.shape[1] // 3
    _check(lib().ar_attention_backward(_ptr(qkv), _ptr(out), _ptr(dout), _ptr(lse), S, L, H, n_heads, _ptr(dqkv),
                                       _ptr(workspace), workspace.numel() * workspace.element_size(),
                                       _stream(stream)))
