"""Block-by-block tuning of a stack of SwiGLU MLP blocks on the GPU.

[AR] §3 "Algorithm Flow" (the blocks are tuned one after another):

* step 2: the block's reference output, its forward with the original bf16
  weights on the block's input (all calibration samples), ``ar_block_forward``;
* steps 3-6: ``iters`` joint SignSGD steps, each on the minibatch of
  calibration samples its row of the schedule names (``ar_gather_samples``
  assembles the tokens and their reference outputs, ``ar_tune_step`` runs the
  step);
* step 7: the block's parameters are frozen; ``ar_qdq`` gives its quantized
  weights, and the quantized block's output (``ar_block_forward`` on them,
  rounded to bf16 by ``ar_f32_to_bf16``) is the next block's input.

``PRESETS`` are the four modes of [AR] §8's preset table (batch size,
iterations, sequence length, calibration samples; lr 5e-3 in all).  The
minibatch draws are data (``synth.make_schedule`` or the caller's own), so a
run is reproducible and checkable against the oracle.

Every step of the method runs in the library's kernels; this module only
allocates buffers and orders the calls.  ([AR] = "Low-Bit Quantization in
Practice with vLLM: Core Mechanisms and Architectural Optimizations of
AutoRound".)
"""
from __future__ import annotations

from typing import Dict, List, Sequence

import numpy as np
import torch

from . import (AR_BLOCK_SWIGLU_MLP, QConfig, ar_block_forward, ar_block_forward_workspace, ar_f32_to_bf16,
               ar_gather_samples, ar_pack_int4, ar_qdq, ar_tune_block, ar_tune_block_workspace)

PRESETS: Dict[str, Dict[str, int]] = {
    "default": {"batch": 8, "iters": 200, "seqlen": 2048, "samples": 128},
    "best": {"batch": 8, "iters": 1000, "seqlen": 2048, "samples": 128},
    "light": {"batch": 8, "iters": 50, "seqlen": 512, "samples": 128},
    "fast": {"batch": 4, "iters": 200, "seqlen": 2048, "samples": 128},
}
LR = 0.005


def tune_mlp_block(Ws: Sequence[torch.Tensor], X: torch.Tensor, cfg: QConfig, schedule: np.ndarray,
                   export_int4: bool = False, stream=None) -> dict:
    """One block of ``tune_mlp_blocks``: Ws = (Wg [F][H], Wu [F][H], Wd [H][F]) bf16 device tensors, X the
    block's input (bf16 [samples][tokens][H]).  Returns the dict described there."""
    schedule = np.asarray(schedule, dtype=np.int32)
    if schedule.ndim != 2 or schedule.shape[0] < 1:
        raise ValueError("schedule must be [steps][batch]")
    S, L, H = X.shape
    dev = X.device
    batch = schedule.shape[1]
    Ws = list(Ws)
    g = cfg.group_size
    # step 2: reference output of the block on its input
    fws = torch.empty(ar_block_forward_workspace(AR_BLOCK_SWIGLU_MLP, Ws, S * L), dtype=torch.uint8, device=dev)
    Y = torch.empty((S, L, H), dtype=torch.float32, device=dev)
    ar_block_forward(AR_BLOCK_SWIGLU_MLP, Ws, X.view(S * L, H), Y.view(S * L, H), fws, stream=stream)
    states = [(torch.zeros(W.shape, dtype=torch.float32, device=dev),
               torch.ones((W.shape[0], W.shape[1] // g), dtype=torch.float32, device=dev),
               torch.ones((W.shape[0], W.shape[1] // g), dtype=torch.float32, device=dev)) for W in Ws]
    layers = [(W, V, a, b) for W, (V, a, b) in zip(Ws, states)]
    # steps 3-6 on the drawn minibatches
    Mb = batch * L
    Xb = torch.empty((batch, L, H), dtype=torch.bfloat16, device=dev)
    Yb = torch.empty((batch, L, H), dtype=torch.float32, device=dev)
    ws = torch.empty(ar_tune_block_workspace(AR_BLOCK_SWIGLU_MLP, layers, Mb, cfg, 1), dtype=torch.uint8, device=dev)
    losses = torch.empty(schedule.shape[0], dtype=torch.float32, device=dev)
    for t, idx in enumerate(schedule):
        ar_gather_samples(X, idx, Xb, stream=stream)
        ar_gather_samples(Y, idx, Yb, stream=stream)
        ar_tune_block(AR_BLOCK_SWIGLU_MLP, layers, Xb.view(Mb, H), Yb.view(Mb, H), cfg, 1, losses[t:t + 1], ws,
                      stream=stream)
    del ws, Xb, Yb
    # step 7: frozen parameters; the quantized block's output is the next input
    What = [torch.empty_like(W) for W in Ws]
    for W, (V, a, b), Wh in zip(Ws, states, What):
        ar_qdq(W, V, a, b, cfg, W_hat=Wh, stream=stream)
    ar_block_forward(AR_BLOCK_SWIGLU_MLP, What, X.view(S * L, H), Y.view(S * L, H), fws, stream=stream)
    Xn = torch.empty((S, L, H), dtype=torch.bfloat16, device=dev)
    ar_f32_to_bf16(Y.view(-1), Xn.view(-1), stream=stream)
    res = {"states": states, "losses": losses, "x_out": Xn}
    if export_int4:
        packs = []
        for W, (V, a, b) in zip(Ws, states):
            N, K = W.shape
            packed = torch.empty((N, K // 8), dtype=torch.int32, device=dev)
            s16 = torch.empty((N, K // g), dtype=torch.float16, device=dev)
            z16 = torch.empty((N, K // g), dtype=torch.float16, device=dev)
            ar_pack_int4(W, V, a, b, cfg, packed, s16, z16, stream=stream)
            packs.append((packed, s16, z16))
        res["int4"] = packs
    return res


def tune_mlp_blocks(blocks: Sequence[Sequence[torch.Tensor]], X0: torch.Tensor, cfg: QConfig,
                    schedule: np.ndarray, export_int4: bool = False, stream=None) -> List[dict]:
    """Tunes ``blocks`` (list of (Wg [F][H], Wu [F][H], Wd [H][F]) bf16 device
    tensors) in order on the calibration tokens ``X0`` (bf16 device tensor
    [samples][tokens][H]); ``schedule``: int [steps][batch] sample indices per
    step (host array).

    Returns one dict per block: ``states`` (three (V, alpha, beta) device
    tensors), ``losses`` (host float32 [steps], the MSE of each step's
    minibatch before its update), ``x_out`` (bf16 [samples][tokens][H], the
    next block's input) and, with ``export_int4`` (4-bit configs), ``int4``:
    three (packed, scale16, zero16) as ``ar_pack_int4`` writes them.
    """
    X = X0
    results = []
    for Ws in blocks:
        res = tune_mlp_block(Ws, X, cfg, schedule, export_int4, stream)
        results.append(res)
        X = res["x_out"]
    for r in results:
        r["losses"] = r["losses"].cpu().numpy()
    return results


def tune_mlp_blocks_streamed(host_blocks: Sequence[Sequence[torch.Tensor]], X0: torch.Tensor, cfg: QConfig,
                             schedule: np.ndarray) -> List[dict]:
    """``tune_mlp_blocks`` for models whose weights live in host memory: each
    block's weights (pinned host bf16 tensors) are copied to the device on a
    side stream while the previous block is tuned, and only what a block
    exports (INT4 words, fp16 scale/zero, the losses) comes back to host
    memory, so the device holds at most two blocks' weights at a time.  The
    calibration tokens ``X0`` stay on the device.  Returns per block
    ``losses`` and ``int4`` (host tensors) and, for the last block, ``x_out``.
    """
    dev = X0.device
    main = torch.cuda.current_stream(dev)
    copy = torch.cuda.Stream(dev)

    def upload(Ws):
        with torch.cuda.stream(copy):
            d = [W.to(dev, non_blocking=True) for W in Ws]
            ev = torch.cuda.Event()
            ev.record(copy)
        return d, ev

    results = []
    X = X0
    nxt = upload(host_blocks[0]) if host_blocks else None
    for b in range(len(host_blocks)):
        Wd, ev = nxt
        main.wait_event(ev)
        for W in Wd:
            W.record_stream(main)
        if b + 1 < len(host_blocks):
            nxt = upload(host_blocks[b + 1])  # overlaps this block's tuning
        res = tune_mlp_block(Wd, X, cfg, schedule, export_int4=True)
        out = {"losses": res["losses"].cpu(), "int4": [tuple(t.cpu() for t in p) for p in res["int4"]]}
        X = res["x_out"]
        del res, Wd
        results.append(out)
    if results:
        results[-1]["x_out"] = X
    for r in results:
        r["losses"] = r["losses"].numpy()
    return results


def save_int4_checkpoint(path: str, results: Sequence[dict], cfg: QConfig) -> None:
    """Writes the INT4 export of every layer of every block to one ``.npz``
    file: arrays ``b{block}.{gate|up|down}.{packed|scale|zero}`` (uint32
    [N][K/8] with element k at bits 4(k mod 8) of word k/8; fp16 [N][K/g]) and
    a ``meta`` JSON string (bits, group_size, symmetric, layout)."""
    import json

    arrays = {}
    for b, r in enumerate(results):
        for name, (packed, s16, z16) in zip(("gate", "up", "down"), r["int4"]):
            arrays[f"b{b}.{name}.packed"] = packed.cpu().numpy().view(np.uint32)
            arrays[f"b{b}.{name}.scale"] = s16.cpu().numpy()
            arrays[f"b{b}.{name}.zero"] = z16.cpu().numpy()
    meta = {"bits": 4, "group_size": int(cfg.group_size), "symmetric": int(cfg.symmetric), "blocks": len(results),
            "layout": "uint32 [N][K/8], element k at bits 4*(k mod 8) of word k/8; fp16 scale/zero [N][K/g]; "
                      "dequant (q - zero) * scale"}
    np.savez(path, meta=np.array(json.dumps(meta)), **arrays)


def load_int4_checkpoint(path: str):
    """Reads ``save_int4_checkpoint``'s file: (meta dict, {name: array})."""
    import json

    with np.load(path) as f:
        meta = json.loads(str(f["meta"]))
        arrays = {k: f[k] for k in f.files if k != "meta"}
    return meta, arrays


_CFG_FIELDS = ("bits", "group_size", "symmetric", "lr", "iters", "v_min", "v_max", "clip_min", "clip_max")


def save_tuning_state(path: str, layers: Sequence[Sequence[torch.Tensor]], step: int, cfg: QConfig,
                      names: Sequence[str] | None = None) -> None:
    """Writes a resumable tuning state to one ``.npz`` file: each layer's
    rounding offsets V (fp32 [N][K]) and clip factors alpha, beta (fp32
    [N][K/g]) as ``{name}.V`` / ``.alpha`` / ``.beta``, the number of steps
    already taken and the quantizer/optimiser settings (``meta``, JSON).
    ``layers`` holds (V, alpha, beta) device tensors.  SignSGD keeps no other
    state (no moments), so these arrays and the step count are everything a
    later call of ``ar_tune_step`` needs to continue exactly where this one
    stopped."""
    import json

    names = list(names) if names is not None else [f"layer{i}" for i in range(len(layers))]
    if len(names) != len(layers):
        raise ValueError("one name per layer")
    arrays = {}
    for name, (V, a, b) in zip(names, layers):
        arrays[f"{name}.V"] = V.detach().cpu().numpy()
        arrays[f"{name}.alpha"] = a.detach().cpu().numpy()
        arrays[f"{name}.beta"] = b.detach().cpu().numpy()
    meta = {"step": int(step), "layers": names, "cfg": {k: getattr(cfg, k) for k in _CFG_FIELDS},
            "content": "AutoRound tuning state: V fp32 [N][K]; alpha, beta fp32 [N][K/group_size]"}
    np.savez(path, meta=np.array(json.dumps(meta)), **arrays)


def load_tuning_state(path: str, device="cuda"):
    """Reads ``save_tuning_state``'s file: (step, QConfig, [(V, alpha, beta)] device tensors, names)."""
    import json

    from . import ar_qconfig_default

    with np.load(path) as f:
        meta = json.loads(str(f["meta"]))
        names = meta["layers"]
        layers = [tuple(torch.from_numpy(np.array(f[f"{n}.{k}"])).to(device) for k in ("V", "alpha", "beta"))
                  for n in names]
    cfg = ar_qconfig_default(**meta["cfg"])
    return int(meta["step"]), cfg, layers, names
