"""CPU oracle for the AutoRound tuning step, INT4 packing and the W4A16 matmul.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It shares no code with
the CUDA library and imports nothing from it; the two meet only through the
seeded inputs of ``synth``.

It is plain and slow on purpose: each function takes the method's steps in the
order and notation of the pages, with numpy doing element-wise IEEE operations
and fp64 matrix products.  Sources (page title, then section):

* [AR] "Low-Bit Quantization in Practice with vLLM: Core Mechanisms and
  Architectural Optimizations of AutoRound" (English write-up of the talk).
  §2 "Minimal Example" (the [0.1, 0.2, 0.15, 8.0] vector), §3 "Optimization
  Variables" table (v, min, max; shapes, ranges, initial values), §3
  "Algorithm Flow" (steps 2-5), §3 "SignSGD" update rule, §3 "Minimal
  State-Evolution Example" (3.3 rounds up once v passes 0.2), §4 "Minimal
  State Evolution" table (w = 0.37, scale 0.05, zero 8).
* [QC] "量化：从 Scale 到 W4A8 的完整坐标", §1.2 (symmetric mapping
  q = clip(round(x/s)), x̂ = s·q; asymmetric adds a zero-point).
* [IA] "Intel AutoRound 高级量化" (hotdry blog), section on the sign-gradient
  mechanism: rounding is treated as the identity in the backward pass (STE).
* [QC] §2 table (E2M1 and E4M3 layouts) and §5 table row "NVFP4 recipe";
  [NQ] "量化" (note.yj-dis.top), section "低比特浮点：FP8 与 NVFP4": the
  NVFP4 QDQ function and the NVFP4 weights' matmul (``nvfp4_matmul``) at the
  end of this module.

Readings where the pages are silent or disagree:

* The group range always contains 0: mx = max(0, max W), mn = min(0, min W).
  [AR] §2 needs this: "no clipping" on [0.1, 0.2, 0.15, 8.0] gives scale 8/15.
* Rounding is half away from zero ([AR] §2: 0.1/0.04 = 2.5 must become 3 to
  give 0.12).
* Clip bounds are multiplicative: hi = alpha·mx, lo = beta·mn with
  alpha, beta in [0.5, 1], init 1 ([AR] §3 table gives min/max per group
  initialised to the group's range; the parameterisation is the task's).
* q = clamp(round(W/s + V) + zp, 0, 2^b - 1), zp = round(-lo/s),
  s = (hi - lo)/(2^b - 1), guarded below at 1e-8.
* STE: both roundings have derivative 1; clamp passes the gradient where
  0 <= round(W/s+V)+zp <= 2^b-1 (inclusive).
* Loss = mean squared error over all M·N outputs; dL/dŶ = 2R/(M·N).
* Update p <- clamp(p - lr·sign(dp)) with sign(0) = 0 (descent; the page's
  formula prints the step without its minus sign).
* Precision points shared with the GPU path: X, W are bf16; the QDQ runs in
  fp32 (it decides integer codes, so both sides decide in the kernel's
  precision); Ŵ is rounded to bf16; products accumulate in fp64 here (fp32 on
  the GPU) and are rounded to fp32; G is rounded to bf16.
* Symmetric mode: s = max(hi, -lo)/(2^(b-1) - 1), zp = 2^(b-1) fixed, codes in
  [0, 2^b - 1]; ds flows to whichever of hi, -lo is larger (ties to hi).
* INT4 layout: row-major [N][K/8] uint32, element k at bits 4·(k mod 8);
  scale and zero as fp16 (round to nearest even).  The pages give no layout.
"""
from __future__ import annotations

import numpy as np

f32 = np.float32
f64 = np.float64

S_GUARD = 1e-8  # lower bound on the scale; never reached by the workloads


# ----------------------------------------------------------------------------
# rounding helpers (IEEE definitions written out)
# ----------------------------------------------------------------------------

def bf16_rne(x) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returns float32.

    bfloat16 keeps the top 16 bits of the float32 encoding.  Round to nearest
    even adds 0x7FFF plus the lowest kept bit before truncating.  NaN stays NaN.
    """
    x = np.asarray(x, dtype=f32)
    b = x.view(np.uint32).astype(np.uint64)
    keep_lsb = (b >> 16) & 1
    r = ((b + 0x7FFF + keep_lsb) >> 16).astype(np.uint32) << np.uint32(16)
    out = r.view(f32).reshape(x.shape)
    return np.where(np.isnan(x), x, out).astype(f32)


def round_half_away(x: np.ndarray) -> np.ndarray:
    """Round to the nearest integer, halves away from zero, in the array's own dtype.

    r = trunc(x); x - r is exact, so the half test decides exactly.
    """
    x = np.asarray(x)
    r = np.trunc(x)
    frac = x - r
    step = np.where(np.abs(frac) >= x.dtype.type(0.5), np.sign(x), x.dtype.type(0))
    return (r + step).astype(x.dtype)


def round_identity(x: np.ndarray) -> np.ndarray:
    """'Rounding' that does nothing: the smooth surrogate used to check STE gradients by finite differences."""
    return np.asarray(x)


def sign0(x: np.ndarray) -> np.ndarray:
    """sign with sign(0) = 0 and sign(NaN) = 0."""
    s = np.sign(x)
    return np.where(np.isnan(s), 0, s).astype(x.dtype)


# ----------------------------------------------------------------------------
# the quantizer ([AR] §2, §3 table, §4 table; [QC] §1.2)
# ----------------------------------------------------------------------------

def group_range(W: np.ndarray, g: int):
    """Per-group range including zero: mx = max(0, max_k W), mn = min(0, min_k W).

    ``W`` is [N][K]; groups are ``g`` consecutive entries along K.
    """
    N, K = W.shape
    assert K % g == 0
    Wg = W.reshape(N, K // g, g)
    mx = np.maximum(Wg.max(axis=-1), 0).astype(W.dtype)
    mn = np.minimum(Wg.min(axis=-1), 0).astype(W.dtype)
    return mx, mn


def qparams(mx, mn, alpha, beta, bits: int, symmetric: bool = False, dtype=f32, rnd=round_half_away):
    """Scale and zero-point of each group from the learnable clip factors.

    Asymmetric: hi = alpha·mx, lo = beta·mn, s = (hi - lo)/(2^b - 1),
    zp = round(-lo/s).  Symmetric: s = max(hi, -lo)/(2^(b-1) - 1), zp = 2^(b-1).
    Returns (hi, lo, s, zp, guarded).
    """
    T = dtype
    mx, mn, alpha, beta = (np.asarray(a, dtype=T) for a in (mx, mn, alpha, beta))
    hi = (alpha * mx).astype(T)
    lo = (beta * mn).astype(T)
    if not symmetric:
        Q = T(2 ** bits - 1)
        s = ((hi - lo) / Q).astype(T)
    else:
        Qs = T(2 ** (bits - 1) - 1)
        s = (np.maximum(hi, -lo) / Qs).astype(T)
    guarded = s < T(S_GUARD)
    s = np.where(guarded, T(S_GUARD), s).astype(T)
    if not symmetric:
        zp = rnd((-lo / s).astype(T)).astype(T)
    else:
        zp = np.full_like(s, T(2 ** (bits - 1)))
    return hi, lo, s, zp, guarded


def quantize(W, V, s, zp, bits: int, dtype=f32, rnd=round_half_away):
    """Codes and dequantized weights for given per-element offsets and per-group (s, zp).

    q = clamp(round(W/s + V) + zp, 0, 2^b - 1);  Ŵ = s·(q - zp).
    ``W, V`` are [N][K]; ``s, zp`` are [N][G].  Returns dict with the
    intermediate ``wq = W/s``, the unclamped integer ``t``, the in-range mask
    ``m``, the codes ``q`` and ``What`` (not yet rounded to bf16).
    """
    T = dtype
    N, K = W.shape
    G = s.shape[1]
    g = K // G
    Wg = np.asarray(W, T).reshape(N, G, g)
    Vg = np.asarray(V, T).reshape(N, G, g)
    s3 = np.asarray(s, T)[:, :, None]
    z3 = np.asarray(zp, T)[:, :, None]
    Q = T(2 ** bits - 1)
    wq = (Wg / s3).astype(T)
    u = (wq + Vg).astype(T)
    r = rnd(u).astype(T)
    t = (r + z3).astype(T)
    m = (t >= 0) & (t <= Q)
    q = np.clip(t, T(0), Q).astype(T)
    what = (s3 * (q - z3)).astype(T)
    return {
        "wq": wq.reshape(N, K),
        "t": t.reshape(N, K),
        "m": m.reshape(N, K),
        "q": q.reshape(N, K),
        "What": what.reshape(N, K),
    }


def qdq(W, V, alpha, beta, bits: int, group_size: int, symmetric: bool = False, dtype=f32, rnd=round_half_away):
    """The fake-quant (QDQ) forward of one weight matrix ([AR] §4 'QDQ / Fake Quantization').

    Returns every per-group and per-element quantity the backward needs, plus
    ``What_bf16`` (Ŵ rounded to bf16, the operand of the tuning GEMMs; only in
    the fp32 instantiation).
    """
    T = dtype
    W = np.asarray(W, T)
    mx, mn = group_range(W, group_size)
    hi, lo, s, zp, guarded = qparams(mx, mn, alpha, beta, bits, symmetric, T, rnd)
    qd = quantize(W, V, s, zp, bits, T, rnd)
    out = dict(qd)
    out.update(mx=mx, mn=mn, hi=hi, lo=lo, s=s, zp=zp, guarded=guarded)
    if T is f32:
        out["What_bf16"] = bf16_rne(qd["What"])
    return out


# ----------------------------------------------------------------------------
# forward, loss and gradients ([AR] §3 'Algorithm Flow' steps 2-4)
# ----------------------------------------------------------------------------

def reference_forward(Xb, Wb) -> np.ndarray:
    """Y = X·Wᵀ with the original (bf16) weights, fp64 accumulation, rounded to fp32."""
    return (np.asarray(Xb, f64) @ np.asarray(Wb, f64).T).astype(f32)


def forward_loss(Xb, What_b, Y, count: int, *, round_g_bf16: bool = True, dtype=f32):
    """QDQ forward and MSE: Ŷ = X·Ŵᵀ, R = Ŷ - Y, L = ΣR²/count, G = dL/dŶ = 2R/count.

    ``count`` is M·N of the whole layer (a row subset passes the full count).
    In the fp32 instantiation Ŷ and R are fp32 and G is rounded to bf16, the
    rounding points the GPU path shares; the fp64 instantiation keeps fp64.
    """
    if dtype is f32:
        Yhat = (np.asarray(Xb, f64) @ np.asarray(What_b, f64).T).astype(f32)
        R = (Yhat - np.asarray(Y, f32)).astype(f32)
        gscale = f32(2.0 / float(count))
        G = (R * gscale).astype(f32)
        if round_g_bf16:
            G = bf16_rne(G)
        L = float(np.sum(R.astype(f64) ** 2) / count)
        return {"Yhat": Yhat, "R": R, "G": G, "loss": L}
    Yhat = np.asarray(Xb, f64) @ np.asarray(What_b, f64).T
    R = Yhat - np.asarray(Y, f64)
    G = 2.0 * R / float(count)
    L = float(np.sum(R ** 2) / count)
    return {"Yhat": Yhat, "R": R, "G": G, "loss": L}


def weight_grad(G, Xb, dtype=f32) -> np.ndarray:
    """dL/dŴ = Gᵀ·X (reduction over the M tokens), fp64 accumulation."""
    d = np.asarray(G, f64).T @ np.asarray(Xb, f64)
    return d.astype(f32) if dtype is f32 else d


def ste_fold(gW, W, st, bits: int, symmetric: bool = False):
    """Straight-through backward of the QDQ, per element into dV and per group into dalpha, dbeta.

    Reverse mode over the forward of ``qdq`` with d round(x)/dx := 1 ([IA],
    [AR] §3 'SignSGD') and d clamp/dt := m (1 inside [0, 2^b-1]):

        dV     = g·s·m
        c      = g·((q - zp) - m·W/s - (1-m)·lo/s)        (= g·dŴ/ds)
        dhi    = Σ_group c / Q
        dlo    = -Σ_group c / Q + Σ_group g·(1-m)
        dalpha = mx·dhi,   dbeta = mn·dlo

    (symmetric: c = g·((q - zp) - m·W/s); ds goes to the larger of hi, -lo).
    When the scale guard is active s does not depend on hi, lo and c := 0.
    Evaluated in fp64 from the forward's values; returned as fp64.
    """
    N, K = gW.shape
    G = st["s"].shape[1]
    g = K // G
    gw = np.asarray(gW, f64).reshape(N, G, g)
    Wd = np.asarray(W, f64).reshape(N, G, g)
    s = np.asarray(st["s"], f64)[:, :, None]
    zp = np.asarray(st["zp"], f64)[:, :, None]
    lo = np.asarray(st["lo"], f64)[:, :, None]
    q = np.asarray(st["q"], f64).reshape(N, G, g)
    m = np.asarray(st["m"], f64).reshape(N, G, g)
    dV = gw * s * m
    if not symmetric:
        Q = float(2 ** bits - 1)
        c = gw * ((q - zp) - m * Wd / s - (1.0 - m) * lo / s)
        c = np.where(st["guarded"][:, :, None], 0.0, c)
        csum = c.sum(axis=-1)
        dhi = csum / Q
        dlo = -csum / Q + (gw * (1.0 - m)).sum(axis=-1)
    else:
        Qs = float(2 ** (bits - 1) - 1)
        c = gw * ((q - zp) - m * Wd / s)
        c = np.where(st["guarded"][:, :, None], 0.0, c)
        dsum = c.sum(axis=-1) / Qs
        hi = np.asarray(st["hi"], f64)
        lo2 = np.asarray(st["lo"], f64)
        take_hi = hi >= -lo2
        dhi = np.where(take_hi, dsum, 0.0)
        dlo = np.where(take_hi, 0.0, -dsum)
    dalpha = np.asarray(st["mx"], f64) * dhi
    dbeta = np.asarray(st["mn"], f64) * dlo
    return dV.reshape(N, K), dalpha, dbeta


def signsgd(p, d, lr: float, lo: float, hi: float) -> np.ndarray:
    """SignSGD step and clamp ([AR] §3 'SignSGD'): p <- clamp(p - lr·sign(d), lo, hi), in fp32.

    Each step moves by exactly ±lr (one fp32 subtraction), or not at all when
    the gradient is zero.
    """
    p = np.asarray(p, f32)
    step = (f32(lr) * sign0(np.asarray(d, f64)).astype(f32)).astype(f32)
    return np.clip((p - step).astype(f32), f32(lo), f32(hi)).astype(f32)


# ----------------------------------------------------------------------------
# one tuning step of a single linear layer ([AR] §3 'Algorithm Flow' 3-5)
# ----------------------------------------------------------------------------

class QConfig:
    """Quantizer and optimiser settings: bits, group size, symmetric flag, learning rate and bounds."""

    def __init__(self, bits=4, group_size=128, symmetric=False, lr=0.005,
                 v_min=-0.5, v_max=0.5, clip_min=0.5, clip_max=1.0):
        self.bits, self.group_size, self.symmetric, self.lr = bits, group_size, bool(symmetric), lr
        self.v_min, self.v_max, self.clip_min, self.clip_max = v_min, v_max, clip_min, clip_max


def tune_step_linear(Wb, Xb, Y, V, alpha, beta, cfg: QConfig, count: int | None = None):
    """One SignSGD step on one linear layer.

    Wb [N][K] and Xb [M][K] are bf16 values held in float32; Y [M][N] is the
    reference output; V, alpha, beta are the current state (not modified).
    ``count`` is the loss normaliser M·N_total (defaults to this layer's M·N);
    pass the full layer's count when ``Wb`` holds only a subset of rows, which
    then gives exactly those rows of the full result.

    Returns (loss, (V', alpha', beta'), grads dict, qdq dict).
    """
    M = Xb.shape[0]
    N = Wb.shape[0]
    count = M * N if count is None else count
    st = qdq(Wb, V, alpha, beta, cfg.bits, cfg.group_size, cfg.symmetric)
    fw = forward_loss(Xb, st["What_bf16"], Y, count)
    gW = weight_grad(fw["G"], Xb)
    dV, da, db = ste_fold(gW, Wb, st, cfg.bits, cfg.symmetric)
    V1 = signsgd(V, dV, cfg.lr, cfg.v_min, cfg.v_max)
    a1 = signsgd(alpha, da, cfg.lr, cfg.clip_min, cfg.clip_max)
    b1 = signsgd(beta, db, cfg.lr, cfg.clip_min, cfg.clip_max)
    grads = {"gW": gW, "dV": dV.astype(f32), "dalpha": da.astype(f32), "dbeta": db.astype(f32), "G": fw["G"]}
    return fw["loss"], (V1, a1, b1), grads, st


def eval_loss_linear(Wb, Xb, Y, V, alpha, beta, cfg: QConfig, count: int | None = None) -> float:
    """Reconstruction MSE of the current state (QDQ forward only)."""
    M, N = Xb.shape[0], Wb.shape[0]
    count = M * N if count is None else count
    st = qdq(Wb, V, alpha, beta, cfg.bits, cfg.group_size, cfg.symmetric)
    return forward_loss(Xb, st["What_bf16"], Y, count)["loss"]


def tune_linear(Wb, Xb, V, alpha, beta, cfg: QConfig, steps: int, Y=None, count: int | None = None):
    """Run ``steps`` SignSGD steps; returns (losses per step, final state, final MSE)."""
    if Y is None:
        Y = reference_forward(Xb, Wb)
    losses = []
    for _ in range(steps):
        L, (V, alpha, beta), _, _ = tune_step_linear(Wb, Xb, Y, V, alpha, beta, cfg, count)
        losses.append(L)
    final = eval_loss_linear(Wb, Xb, Y, V, alpha, beta, cfg, count)
    return np.array(losses), (V, alpha, beta), final


# ----------------------------------------------------------------------------
# smooth surrogate for finite-difference checks of the STE chain rule
# ----------------------------------------------------------------------------

def smooth_loss_linear(W, X, Y, V, alpha, beta, bits, group_size, symmetric=False):
    """fp64 loss with every rounding replaced by the identity (no bf16, no round).

    With the roundings gone the STE gradients are the exact gradients of this
    function (away from the clamp kinks), which finite differences can check.
    """
    st = qdq(W, V, alpha, beta, bits, group_size, symmetric, dtype=f64, rnd=round_identity)
    fw = forward_loss(X, st["What"], Y, X.shape[0] * W.shape[0], dtype=f64)
    return fw["loss"], st, fw


def smooth_grads_linear(W, X, Y, V, alpha, beta, bits, group_size, symmetric=False):
    """Analytic (STE-fold) gradients of ``smooth_loss_linear``."""
    L, st, fw = smooth_loss_linear(W, X, Y, V, alpha, beta, bits, group_size, symmetric)
    gW = weight_grad(fw["G"], X, dtype=f64)
    return L, ste_fold(gW, W, st, bits, symmetric)


# ----------------------------------------------------------------------------
# INT4 export and the W4A16 matmul ([AR] §4 'Real INT4 Kernel')
# ----------------------------------------------------------------------------

def pack_int4(q: np.ndarray, s: np.ndarray, zp: np.ndarray):
    """Pack 4-bit codes and per-group metadata.

    words[n][j] = Σ_{i<8} q[n][8j+i] · 16^i  (uint32);  scale = fp16(s), zero = fp16(zp),
    both round to nearest even (zp is an integer ≤ 15, exact).  Returns the
    words and the fp16 bit patterns of scale and zero.
    """
    N, K = q.shape
    assert K % 8 == 0
    qi = np.asarray(q).astype(np.uint32).reshape(N, K // 8, 8)
    assert qi.max(initial=0) <= 15
    shifts = (4 * np.arange(8, dtype=np.uint32))[None, None, :]
    words = np.bitwise_or.reduce(qi << shifts, axis=-1).astype(np.uint32)
    scale16 = np.asarray(s, f32).astype(np.float16).view(np.uint16)
    zero16 = np.asarray(zp, f32).astype(np.float16).view(np.uint16)
    return words, scale16, zero16


def unpack_int4(words: np.ndarray, K: int) -> np.ndarray:
    """Inverse of the code layout of ``pack_int4``."""
    N = words.shape[0]
    shifts = (4 * np.arange(8, dtype=np.uint32))[None, None, :]
    q = (words[:, :, None] >> shifts) & np.uint32(0xF)
    return q.reshape(N, K).astype(np.uint8)


def w4a16_matmul(A, words, scale16, zero16, group_size: int) -> np.ndarray:
    """out[t][n] = Σ_k A[t][k]·(q[n][k] - zero[n][k/g])·scale[n][k/g], fp64 (returned as fp64).

    ``A`` holds bf16 values as float32; scale and zero are fp16 bit patterns.
    """
    N = words.shape[0]
    K = words.shape[1] * 8
    q = unpack_int4(words, K).astype(f64)
    s = scale16.view(np.float16).astype(f64)
    z = zero16.view(np.float16).astype(f64)
    deq = (q.reshape(N, K // group_size, group_size) - z[:, :, None]) * s[:, :, None]
    return np.asarray(A, f64) @ deq.reshape(N, K).T


def pack_bitstream(q: np.ndarray, bits: int) -> np.ndarray:
    """b-bit codes as a little-endian bit stream per row: element k occupies bits
    [b k, b k + b) of its row, stream bit i in uint32 word i / 32 at position
    i mod 32; K b must be a multiple of 32.  For b in {2, 4, 8} this is the
    per-word layout of ``pack_codes``; for b = 3 it puts 32 codes in 3 words,
    codes 10 and 21 of each 32 straddling two words (the pages define no
    packing at any width but 4)."""
    N, K = q.shape
    assert (K * bits) % 32 == 0
    qi = np.asarray(q).astype(np.uint32)
    assert qi.max(initial=0) < (1 << bits)
    stream = ((qi[:, :, None] >> np.arange(bits, dtype=np.uint32)) & 1).astype(np.uint8).reshape(N, K * bits)
    return np.ascontiguousarray(np.packbits(stream, axis=-1, bitorder="little")).view("<u4").astype(np.uint32)


def unpack_bitstream(words: np.ndarray, K: int, bits: int) -> np.ndarray:
    """Inverse of ``pack_bitstream``."""
    N = words.shape[0]
    stream = np.unpackbits(np.ascontiguousarray(words.astype("<u4")).view(np.uint8), axis=-1, bitorder="little")
    b = stream[:, : K * bits].reshape(N, K, bits).astype(np.uint16)
    return np.sum(b << np.arange(bits, dtype=np.uint16), axis=-1).astype(np.uint16)


def pack_codes(q: np.ndarray, bits: int) -> np.ndarray:
    """b-bit codes packed little end first along K: 32/b codes per uint32,
    element k at bits b*(k mod 32/b) of word k/(32/b) (the INT4 layout of
    ``pack_int4`` for other widths; b in {2, 4, 8})."""
    assert bits in (2, 4, 8)
    per = 32 // bits
    N, K = q.shape
    assert K % per == 0
    qi = np.asarray(q).astype(np.uint32).reshape(N, K // per, per)
    assert qi.max(initial=0) < (1 << bits)
    shifts = (bits * np.arange(per, dtype=np.uint32))[None, None, :]
    return np.bitwise_or.reduce(qi << shifts, axis=-1).astype(np.uint32)


def unpack_codes(words: np.ndarray, K: int, bits: int) -> np.ndarray:
    """Inverse of ``pack_codes``."""
    per = 32 // bits
    N = words.shape[0]
    shifts = (bits * np.arange(per, dtype=np.uint32))[None, None, :]
    q = (words[:, :, None] >> shifts) & np.uint32((1 << bits) - 1)
    return q.reshape(N, K).astype(np.uint16)


def wxa16_matmul(A, words, scale16, zero16, group_size: int, bits: int) -> np.ndarray:
    """out[t][n] = Σ_k A[t][k]·(q[n][k] - zero[n][k/g])·scale[n][k/g] for b-bit codes, fp64.

    ``words`` is the per-row bit stream of ``pack_bitstream`` (at 2, 4 and 8 bits
    the per-word layout of ``pack_codes``; 3 bits: 32 codes in 3 words)."""
    N = words.shape[0]
    K = words.shape[1] * 32 // bits
    q = unpack_bitstream(words, K, bits).astype(f64)
    s = scale16.view(np.float16).astype(f64)
    z = zero16.view(np.float16).astype(f64)
    deq = (q.reshape(N, K // group_size, group_size) - z[:, :, None]) * s[:, :, None]
    return np.asarray(A, f64) @ deq.reshape(N, K).T


# ----------------------------------------------------------------------------
# SwiGLU MLP block tuned jointly ([AR] §3 "Why Block-Wise Optimization": the
# error of downstream sub-layers back-propagates to upstream weights)
# ----------------------------------------------------------------------------
#
# Block: Y = (silu(X Wgᵀ) ⊙ (X Wuᵀ)) Wdᵀ with silu(x) = x / (1 + e^{-x}).
# Rounding points shared with the GPU path (fp32 instantiation): the gate and
# up products a, b are rounded to bf16, h = bf16(silu(a) b), the down product
# accumulates in fp32; in the backward G, dA = bf16(dH · b · silu'(a)) and
# dB = bf16(dH · silu(a)) are the bf16 operands of the next products.

def silu(x):
    x = np.asarray(x, f64)
    return x / (1.0 + np.exp(-x))


def silu_grad(x):
    """d/dx [x·σ(x)] = σ(x)·(1 + x·(1 − σ(x)))."""
    x = np.asarray(x, f64)
    s = 1.0 / (1.0 + np.exp(-x))
    return s * (1.0 + x * (1.0 - s))


def mlp_forward(Xb, Wg, Wu, Wd, dtype=f32):
    """SwiGLU block forward with the given (bf16-valued) weights.

    Returns a, b (the gate/up products), h and the block output y.
    """
    X = np.asarray(Xb, f64)
    if dtype is f32:
        a = bf16_rne((X @ np.asarray(Wg, f64).T).astype(f32))
        b = bf16_rne((X @ np.asarray(Wu, f64).T).astype(f32))
        h = bf16_rne((silu(a) * np.asarray(b, f64)).astype(f32))
        y = (np.asarray(h, f64) @ np.asarray(Wd, f64).T).astype(f32)
        return {"a": a, "b": b, "h": h, "y": y}
    a = X @ np.asarray(Wg, f64).T
    b = X @ np.asarray(Wu, f64).T
    h = silu(a) * b
    return {"a": a, "b": b, "h": h, "y": h @ np.asarray(Wd, f64).T}


def mlp_backward(Xb, fw, G, Wd_hat, dtype=f32):
    """Gradients of the block loss w.r.t. the three fake-quantized weights.

    dŴd = Gᵀ h;  dH = G Ŵd;  dA = dH · b · silu'(a);  dB = dH · silu(a);
    dŴg = dAᵀ X;  dŴu = dBᵀ X.
    """
    X = np.asarray(Xb, f64)
    G64 = np.asarray(G, f64)
    a = np.asarray(fw["a"], f64)
    b = np.asarray(fw["b"], f64)
    gWd = G64.T @ np.asarray(fw["h"], f64)
    dH = G64 @ np.asarray(Wd_hat, f64)
    if dtype is f32:
        dH = dH.astype(f32).astype(f64)
        dA = bf16_rne((dH * b * silu_grad(a)).astype(f32))
        dB = bf16_rne((dH * silu(a)).astype(f32))
        gWg = np.asarray(dA, f64).T @ X
        gWu = np.asarray(dB, f64).T @ X
        return gWg.astype(f32), gWu.astype(f32), gWd.astype(f32), {"dA": dA, "dB": dB, "dH": dH.astype(f32)}
    dA = dH * b * silu_grad(a)
    dB = dH * silu(a)
    return dA.T @ X, dB.T @ X, gWd, {"dA": dA, "dB": dB, "dH": dH}


def mlp_reference(Xb, Wg, Wu, Wd):
    """Block output with the original bf16 weights ([AR] §3 'Algorithm Flow' step 2)."""
    return mlp_forward(Xb, Wg, Wu, Wd)["y"]


def tune_step_mlp(Ws, Xb, Y, states, cfg: QConfig):
    """One joint SignSGD step on the three weights of the SwiGLU block.

    ``Ws`` = (Wg, Wu, Wd) bf16 values in float32; ``states`` = three
    (V, alpha, beta) tuples.  Returns (loss, new states, grads, qdq dicts).
    """
    sts = [qdq(W, *st, cfg.bits, cfg.group_size, cfg.symmetric) for W, st in zip(Ws, states)]
    fw = mlp_forward(Xb, sts[0]["What_bf16"], sts[1]["What_bf16"], sts[2]["What_bf16"])
    M, H = fw["y"].shape
    count = M * H
    R = (fw["y"] - np.asarray(Y, f32)).astype(f32)
    loss = float(np.sum(R.astype(f64) ** 2) / count)
    G = bf16_rne((R * f32(2.0 / float(count))).astype(f32))
    gWg, gWu, gWd, extra = mlp_backward(Xb, fw, G, sts[2]["What_bf16"])
    new_states, grads = [], []
    for W, st, (V, a, b), gW in zip(Ws, sts, states, (gWg, gWu, gWd)):
        dV, da, db = ste_fold(gW, W, st, cfg.bits, cfg.symmetric)
        new_states.append((signsgd(V, dV, cfg.lr, cfg.v_min, cfg.v_max),
                           signsgd(a, da, cfg.lr, cfg.clip_min, cfg.clip_max),
                           signsgd(b, db, cfg.lr, cfg.clip_min, cfg.clip_max)))
        grads.append({"gW": gW, "dV": dV.astype(f32), "dalpha": da.astype(f32), "dbeta": db.astype(f32)})
    extra.update(G=G, fw=fw)
    return loss, new_states, grads, sts, extra


def eval_loss_mlp(Ws, Xb, Y, states, cfg: QConfig) -> float:
    sts = [qdq(W, *st, cfg.bits, cfg.group_size, cfg.symmetric) for W, st in zip(Ws, states)]
    y = mlp_forward(Xb, sts[0]["What_bf16"], sts[1]["What_bf16"], sts[2]["What_bf16"])["y"]
    R = (y - np.asarray(Y, f32)).astype(f64)
    return float(np.sum(R ** 2) / R.size)


def smooth_grads_mlp(Ws, X, Y, states, bits, group_size, symmetric=False):
    """fp64 block loss with all roundings replaced by the identity, and its STE-fold gradients."""
    sts = [qdq(W, *st, bits, group_size, symmetric, dtype=f64, rnd=round_identity) for W, st in zip(Ws, states)]
    fw = mlp_forward(X, sts[0]["What"], sts[1]["What"], sts[2]["What"], dtype=f64)
    R = fw["y"] - np.asarray(Y, f64)
    L = float(np.sum(R ** 2) / R.size)
    G = 2.0 * R / R.size
    gWg, gWu, gWd, _ = mlp_backward(X, fw, G, sts[2]["What"], dtype=f64)
    grads = [ste_fold(gW, W, st, bits, symmetric) for W, st, gW in zip(Ws, sts, (gWg, gWu, gWd))]
    return L, grads


def smooth_loss_mlp(Ws, X, Y, states, bits, group_size, symmetric=False):
    sts = [qdq(W, *st, bits, group_size, symmetric, dtype=f64, rnd=round_identity) for W, st in zip(Ws, states)]
    fw = mlp_forward(X, sts[0]["What"], sts[1]["What"], sts[2]["What"], dtype=f64)
    R = fw["y"] - np.asarray(Y, f64)
    return float(np.sum(R ** 2) / R.size)


# ----------------------------------------------------------------------------
# Block-by-block tuning of a stack of SwiGLU blocks ([AR] §3 "Algorithm Flow")
# ----------------------------------------------------------------------------

def tune_blocks_mlp(blocks, X0, cfg: QConfig, schedule):
    """The blocks in order ([AR] §3 "Algorithm Flow"):

    * step 2: the block's reference output, its forward with the original
      weights on the block's input (all calibration samples);
    * steps 3-6: one joint SignSGD step (``tune_step_mlp``) per row of
      ``schedule`` on the samples the row names, their tokens in that order
      (the minibatch of [AR] §8's preset table);
    * step 7: the block's parameters are frozen and the output of the
      quantized block, rounded to bf16, is the next block's input.

    ``blocks``: list of (Wg, Wu, Wd) bf16 values in float32; ``X0``:
    [samples][tokens][H] bf16 values in float32; ``schedule``: int
    [steps][batch] (the random draws, passed in).  Returns one dict per block:
    ``states`` (three (V, alpha, beta)), ``losses`` [steps] and ``x_out``
    ([samples][tokens][H], the next block's input).
    """
    X = np.asarray(X0, f32)
    S, L, H = X.shape
    out = []
    for Ws in blocks:
        Xf = X.reshape(S * L, H)
        Y = mlp_reference(Xf, *Ws).reshape(S, L, H)
        states = [(np.zeros(W.shape, f32), np.ones((W.shape[0], W.shape[1] // cfg.group_size), f32),
                   np.ones((W.shape[0], W.shape[1] // cfg.group_size), f32)) for W in Ws]
        losses = []
        for idx in np.asarray(schedule):
            Xb = X[idx].reshape(-1, H)
            Yb = Y[idx].reshape(-1, H)
            loss, states, _, _, _ = tune_step_mlp(Ws, Xb, Yb, states, cfg)
            losses.append(loss)
        sts = [qdq(W, *st, cfg.bits, cfg.group_size, cfg.symmetric) for W, st in zip(Ws, states)]
        y = mlp_forward(Xf, sts[0]["What_bf16"], sts[1]["What_bf16"], sts[2]["What_bf16"])["y"]
        X = bf16_rne(y).reshape(S, L, H)
        out.append({"states": states, "losses": np.asarray(losses, f64), "x_out": X})
    return out



# ----------------------------------------------------------------------------
# NVFP4 fake quantization: a QDQ function for a new data type ([AR] §4 "Why the
# Tuning Stage Must Take the QDQ Path", point 3: a new type needs only a
# tensor-level QDQ function)
# ----------------------------------------------------------------------------
#
# Format: [QC] §2 table ("FP4 E2M1: 1 sign + 2 exponent + 1 mantissa", "FP8
# E4M3: 1 sign + 4 exponent + 3 mantissa"); [NQ] "量化" (note.yj-dis.top),
# section "低比特浮点：FP8 与 NVFP4", table row NVFP4: E2M1 values, one FP8
# scale per micro-block of 16 values, plus a per-tensor scale; [QC] §5 table
# row "NVFP4 recipe" (E2M1, 16-element block scale and global scale).
#
# Readings (the pages give the layout of the values, not the recipe):
# * exponent bias 2^(e-1) - 1 (1 for E2M1, 7 for E4M3), subnormals at exponent
#   field 0; E4M3 has no infinities (its all-ones code is NaN), so its largest
#   finite value is 448; E2M1's is 6;
# * both conversions round to nearest, ties to the even code, and saturate at
#   the largest finite value;
# * global scale S = amax(|W|) / (6 * 448), so the largest block scale, as a
#   multiple of S, fits E4M3;
# * AutoRound's variables act as in the integer quantizer: the learnable clip
#   factor alpha multiplies each block's range (E2M1 is symmetric, so there is
#   no separate lower bound), V is added to W / s before rounding; block scale
#   s = E4M3(alpha * amax_block / 6 / S) * S;
# * every step in fp32 (the codes are decided in the kernel's precision), in
#   the order written in ``nvfp4_qdq``; a block whose scale rounds to 0 gives 0.

NVFP4_BLOCK = 16
E2M1_MAX = 6.0
E4M3_MAX = 448.0


def _minifloat_values(e_bits: int, m_bits: int, nan_codes=()):
    """Value of every code of a sign/exponent/mantissa format with bias 2^(e-1) - 1 and subnormals."""
    bias = 2 ** (e_bits - 1) - 1
    vals = []
    for code in range(2 ** (1 + e_bits + m_bits)):
        sgn = -1.0 if code >> (e_bits + m_bits) else 1.0
        e = (code >> m_bits) & (2 ** e_bits - 1)
        m = code & (2 ** m_bits - 1)
        if code in nan_codes:
            vals.append(np.nan)
        elif e == 0:
            vals.append(sgn * (m / 2 ** m_bits) * 2.0 ** (1 - bias))
        else:
            vals.append(sgn * (1 + m / 2 ** m_bits) * 2.0 ** (e - bias))
    return np.array(vals, f64)


def e2m1_values() -> np.ndarray:
    """The 16 E2M1 codes' values (code = sign << 3 | exponent << 1 | mantissa)."""
    return _minifloat_values(2, 1)


def e4m3_values() -> np.ndarray:
    """The 256 E4M3 codes' values; 0x7F and 0xFF are NaN."""
    return _minifloat_values(4, 3, nan_codes=(0x7F, 0xFF))


def _round_to_codes(x, values, vmax):
    """Nearest finite code to each x (ties to the even code, i.e. mantissa bit 0), saturating at +-vmax.
    Returns the codes (as int) of the non-negative magnitudes with the sign bit of x."""
    x = np.asarray(x, f64)
    n = values.size // 2
    mags = values[:n]                      # codes 0 .. n-1: the non-negative values, increasing
    fin = np.isfinite(mags)
    a = np.minimum(np.abs(x), vmax)
    d = np.abs(a[..., None] - np.where(fin, mags, np.inf)[None, :])
    best = d.min(axis=-1, keepdims=True)
    cand = d == best
    # among equally near codes take the even one (codes are consecutive, so at most two tie)
    even = cand & ((np.arange(n) % 2) == 0)[None, :]
    pick = np.where(even.any(axis=-1), even.argmax(axis=-1), cand.argmax(axis=-1))
    return np.where(np.signbit(x), pick + n, pick).astype(np.int64)


def e2m1_round(x):
    """(code, value) of round-to-nearest-even E2M1 with saturation at +-6."""
    vals = e2m1_values()
    code = _round_to_codes(x, vals, E2M1_MAX)
    return code, vals[code]


def e4m3_round(x):
    """(code, value) of round-to-nearest-even E4M3 with saturation at +-448 (no NaN produced)."""
    vals = e4m3_values()
    code = _round_to_codes(x, vals, E4M3_MAX)
    return code, vals[code]


def nvfp4_qdq(W, V=None, alpha=None, amax=None):
    """NVFP4 fake quantization of W [N][K] (K a multiple of 16) in fp32.

    amax_t = max |W|; S = amax_t / 2688; per block b of 16 along K:
    s_b = E4M3((alpha_b * amax_b) / 6 / S) * S; codes q = E2M1(W / s_b + V),
    Ŵ = q * s_b (0 where s_b = 0).  V [N][K] defaults to 0, alpha [N][K/16]
    to 1.  ``amax`` is max |W| of the whole tensor when W holds only some of its
    rows (default: W's own).  Returns codes (uint8 0..15), scale codes (uint8,
    E4M3), S, the effective block scales, Ŵ (fp32) and Ŵ rounded to bf16.
    """
    W = np.asarray(W, f32)
    N, K = W.shape
    assert K % NVFP4_BLOCK == 0
    nb = K // NVFP4_BLOCK
    V = np.zeros_like(W) if V is None else np.asarray(V, f32)
    alpha = np.ones((N, nb), f32) if alpha is None else np.asarray(alpha, f32)
    amax_t = f32(amax) if amax is not None else (f32(np.max(np.abs(W))) if W.size else f32(0))
    S = f32(amax_t / f32(E2M1_MAX * E4M3_MAX))
    Wb = W.reshape(N, nb, NVFP4_BLOCK)
    amax_b = np.max(np.abs(Wb), axis=-1).astype(f32)
    sb_raw = ((alpha * amax_b).astype(f32) / f32(E2M1_MAX)).astype(f32)
    if S > 0:
        ratio = (sb_raw / S).astype(f32)
    else:
        ratio = np.zeros_like(sb_raw)
    scode, s8 = e4m3_round(ratio)
    s_eff = (s8.astype(f32) * S).astype(f32)
    se = np.repeat(s_eff, NVFP4_BLOCK, axis=1).reshape(N, K)
    live = se > 0
    x = np.where(live, (W / np.where(live, se, f32(1))).astype(f32) + V, f32(0)).astype(f32)
    qcode, qval = e2m1_round(x)
    qcode = np.where(live, qcode, 0)
    What = np.where(live, (qval.astype(f32) * se).astype(f32), f32(0)).astype(f32)
    return {"codes": qcode.astype(np.uint8), "scale_codes": scode.astype(np.uint8), "S": S, "s": s_eff,
            "x": x, "q": np.where(live, qval, 0.0).astype(f32), "amax_b": amax_b,
            "What": What, "What_bf16": bf16_rne(What)}


def pack_fp4(codes: np.ndarray) -> np.ndarray:
    """Two E2M1 codes per byte along K, element k in the low nibble when k is even: uint8 [N][K/2]."""
    c = np.asarray(codes).astype(np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def unpack_fp4(packed: np.ndarray) -> np.ndarray:
    """Inverse of ``pack_fp4``: uint8 [N][K/2] -> codes uint8 [N][K]."""
    b = np.asarray(packed).astype(np.uint8)
    out = np.empty((b.shape[0], 2 * b.shape[1]), np.uint8)
    out[:, 0::2] = b & 0x0F
    out[:, 1::2] = b >> 4
    return out


def nvfp4_matmul(A, packed_codes, scale_codes, S) -> np.ndarray:
    """The NVFP4 weights' matmul with bf16-valued activations, in fp64:
    out[t][n] = S * sum_k A[t][k] * E4M3(scale_codes[n][k/16]) * E2M1(code[n][k])
    ([QC] §2 table and §5 row "NVFP4 recipe"; [NQ] "量化", section "低比特浮点：FP8 与
    NVFP4": E2M1 values, one E4M3 scale per 16-value block, a per-tensor scale).
    A [T][K] (values), packed_codes uint8 [N][K/2] (``pack_fp4``), scale_codes uint8
    [N][K/16], S the per-tensor scale.  Returns fp64 [T][N]."""
    codes = unpack_fp4(packed_codes)
    N, K = codes.shape
    q = e2m1_values()[codes.astype(np.int64)]
    sb = np.repeat(e4m3_values()[np.asarray(scale_codes).astype(np.int64)], NVFP4_BLOCK, axis=1).reshape(N, K)
    W = f64(S) * sb * q
    return np.asarray(A, f64) @ W.T


# ----------------------------------------------------------------------------
# one tuning step on NVFP4: the integer step with the NVFP4 QDQ function in
# its place ([AR] §4 "Why the Tuning Stage Must Take the QDQ Path", point 3;
# [AR] §3 "Algorithm Flow" steps 3-5 and "SignSGD")
# ----------------------------------------------------------------------------
#
# Straight-through backward as in the integer quantizer: both roundings (E4M3
# of the block scale, E2M1 of the codes) count as the identity, the saturation
# at +-6 passes the gradient where |W/s + V| <= 6 (inclusive), and the products
# use the forward's values:
#     dV_i     = g_i s_b m_i
#     dalpha_b = (amax_b / 6) sum_i g_i (q_i - m_i W_i / s_b)
# (s_b = alpha_b amax_b / 6 up to the E4M3 rounding, so ds_b/dalpha_b =
# amax_b / 6); a block whose scale is 0 gets no gradient.

def nvfp4_qdq_smooth(W, V, alpha):
    """``nvfp4_qdq`` in fp64 with both roundings replaced by the identity (the saturation kept):
    s_b = alpha_b amax_b / 6, x = W / s_b + V, q = clip(x, -6, 6), Ŵ = q s_b.  Its exact gradient is
    what ``nvfp4_ste_fold`` computes, so finite differences can check the fold."""
    W = np.asarray(W, f64)
    N, K = W.shape
    nb = K // NVFP4_BLOCK
    amax_b = np.abs(W.reshape(N, nb, NVFP4_BLOCK)).max(-1)
    s = np.asarray(alpha, f64) * amax_b / E2M1_MAX
    se = np.repeat(s, NVFP4_BLOCK, axis=1)
    live = se > 0
    x = np.where(live, W / np.where(live, se, 1.0) + np.asarray(V, f64), 0.0)
    q = np.clip(x, -E2M1_MAX, E2M1_MAX)
    return {"s": s, "x": x, "q": q, "amax_b": amax_b, "What": q * se}


def nvfp4_ste_fold(gW, W, st):
    """(dV [N][K], dalpha [N][K/16]) in fp64 from dL/dŴ and the forward's values."""
    N, K = gW.shape
    nb = K // NVFP4_BLOCK
    g = np.asarray(gW, f64).reshape(N, nb, NVFP4_BLOCK)
    Wd = np.asarray(W, f64).reshape(N, nb, NVFP4_BLOCK)
    s = np.asarray(st["s"], f64)[:, :, None]
    x = np.asarray(st["x"], f64).reshape(N, nb, NVFP4_BLOCK)
    q = np.asarray(st["q"], f64).reshape(N, nb, NVFP4_BLOCK)
    live = np.broadcast_to(s > 0, g.shape)
    m = live & (np.abs(x) <= E2M1_MAX)
    sd = np.where(live, s, 1.0)
    dV = np.where(m, g * s, 0.0)
    c = np.where(live, g * (q - np.where(m, Wd / sd, 0.0)), 0.0)
    dalpha = (np.asarray(st["amax_b"], f64) / E2M1_MAX) * c.sum(-1)
    return dV.reshape(N, K), dalpha


def nvfp4_tune_step_linear(Wb, Xb, Y, V, alpha, cfg: QConfig, amax=None, count: int | None = None):
    """One SignSGD step of one linear layer on NVFP4 (the state is V [N][K] and alpha [N][K/16];
    ``cfg`` gives lr and the bounds).  Returns (loss, (V', alpha'), grads, qdq dict)."""
    M, N = Xb.shape[0], Wb.shape[0]
    count = M * N if count is None else count
    st = nvfp4_qdq(Wb, V, alpha, amax)
    fw = forward_loss(Xb, st["What_bf16"], Y, count)
    gW = weight_grad(fw["G"], Xb)
    dV, da = nvfp4_ste_fold(gW, Wb, st)
    V1 = signsgd(V, dV, cfg.lr, cfg.v_min, cfg.v_max)
    a1 = signsgd(alpha, da, cfg.lr, cfg.clip_min, cfg.clip_max)
    return fw["loss"], (V1, a1), {"gW": gW, "dV": dV.astype(f32), "dalpha": da.astype(f32), "G": fw["G"]}, st


# ----------------------------------------------------------------------------
# A decoder block tuned jointly ([AR] §3 "Why Block-Wise Optimization": the
# block's output error reaches every weight of the block; [AR] §3 "Algorithm
# Flow": the block, not the layer, is the unit of tuning)
# ----------------------------------------------------------------------------
#
# Readings (the pages name the decoder block as the unit, not its layers):
# * a pre-norm block of the Llama family: r1 = rmsnorm(X) γ1; Q, K, V = r1 Wqᵀ,
#   r1 Wkᵀ, r1 Wvᵀ (nh heads of d = H / nh each, no shared K/V heads); the
#   rotary embedding on Q and K (the halves of each head rotate as complex
#   pairs (x_i, x_{i+d/2}) by the angle t 10000^(-2i/d), t the token's position
#   in its sample); causal softmax attention per head with scale 1/sqrt(d),
#   within each sample; A = O Woᵀ; X2 = X + A; r2 = rmsnorm(X2) γ2;
#   Y = X2 + (silu(r2 Wgᵀ) ⊙ (r2 Wuᵀ)) Wdᵀ;
# * rmsnorm(x) = x / sqrt(mean(x²) + 1e-6) over the hidden dimension; γ1, γ2 are
#   neither quantized nor tuned;
# * the seven linear weights (q, k, v, o, gate, up, down) are fake-quantized with
#   their own V, alpha, beta and tuned jointly from the MSE of Y.
# This section is in fp64 after the QDQ (whose codes are decided in fp32 as
# everywhere in this module).  With ``rounding=True`` it applies the rounding
# points a GPU path shares with it, in the same order (no page fixes them; the
# rule is that every operand of a matrix product is bf16 and everything else is
# fp32):
# * bf16: r1, r2 (normalised inputs of the projections), Qr, Kr (after the
#   rotation), V, the attention probabilities P, the attention output O, a, b,
#   h of the MLP, G, dA, dB, dX2, dO, dS (the softmax gradient times 1/sqrt(d)),
#   dQ, dK (after the inverse rotation), dV;
# * fp32: the products' results (Q, K before the rotation, the scores z, Ŷ
#   parts, dH, dr2, dP, dQr, dKr), the residual stream X2 and Ŷ, R, the row
#   statistic D = rowsum(dO ⊙ O); the scale 1/sqrt(d) and the rotation's
#   cos/sin are fp32 constants;
# * the probabilities come from a two-pass softmax, P = exp(z - lse) with
#   lse = log sum_j exp(z_j) over the row's keys, so that their rounding to bf16
#   does not depend on the order in which keys are visited; O = P V is then
#   the normalised output (no division after the product).

RMS_EPS = 1e-6
ROPE_BASE = 10000.0
DECODER_LAYERS = ("q", "k", "v", "o", "gate", "up", "down")


def _rounders(rounding: bool):
    """(to_bf16, to_fp32) as fp64 arrays when rounding, else the identity."""
    if not rounding:
        ident = lambda x: np.asarray(x, f64)
        return ident, ident
    return (lambda x: bf16_rne(np.asarray(x, f64).astype(f32)).astype(f64),
            lambda x: np.asarray(x, f64).astype(f32).astype(f64))


def rmsnorm(x, gamma):
    """(x / sqrt(mean_j x_j² + eps) * gamma, the per-row 1/sqrt(...)) along the last axis."""
    x = np.asarray(x, f64)
    inv = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + RMS_EPS)
    return x * inv * np.asarray(gamma, f64), inv


def rmsnorm_backward(x, gamma, inv, dy):
    """dx of y = x r gamma, r = (mean(x²) + eps)^(-1/2): r gamma dy - x r³ mean(dy gamma x)."""
    x = np.asarray(x, f64)
    gdy = np.asarray(dy, f64) * np.asarray(gamma, f64)
    return inv * gdy - x * inv ** 3 * np.mean(gdy * x, axis=-1, keepdims=True)


def rope_angles(L: int, d: int, rounding: bool = False):
    """cos, sin [L][d/2] of the angles t * base^(-2i/d) (fp32 constants when rounding)."""
    i = np.arange(d // 2, dtype=f64)
    ang = np.arange(L, dtype=f64)[:, None] * ROPE_BASE ** (-2.0 * i / d)[None, :]
    c, s = np.cos(ang), np.sin(ang)
    if rounding:
        c, s = c.astype(f32).astype(f64), s.astype(f32).astype(f64)
    return c, s


def rope(x, nh: int, sign: float = 1.0, rounding: bool = False):
    """Rotate each head of x [S][L][H]: (x_i, x_{i+d/2}) -> (x_i cos - x_{i+d/2} sin, x_{i+d/2} cos + x_i sin);
    ``sign`` = -1 rotates back (the transpose, used by the backward)."""
    x = np.asarray(x, f64)
    S, L, H = x.shape
    d = H // nh
    c, s = rope_angles(L, d, rounding)
    s = sign * s
    xh = x.reshape(S, L, nh, d)
    x1, x2 = xh[..., : d // 2], xh[..., d // 2:]
    c, s = c[None, :, None, :], s[None, :, None, :]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1).reshape(S, L, H)


def attention_scale(d: int, rounding: bool = False):
    return float(f32(1.0 / np.sqrt(d))) if rounding else 1.0 / np.sqrt(d)


def attention_forward(Q, K, V, nh: int, rounding: bool = False):
    """Causal softmax attention per sample and head: z = Q Kᵀ / sqrt(d) (keys up to the query's
    position), lse = log sum exp(z) over those keys, P = exp(z - lse), O = P V.
    Returns O [S][L][H], P [S][nh][L][L] and lse [S][nh][L]."""
    rb, rf = _rounders(rounding)
    S, L, H = Q.shape
    d = H // nh
    q = Q.reshape(S, L, nh, d).transpose(0, 2, 1, 3)
    k = K.reshape(S, L, nh, d).transpose(0, 2, 1, 3)
    v = V.reshape(S, L, nh, d).transpose(0, 2, 1, 3)
    z = rf(rf(q @ k.transpose(0, 1, 3, 2)) * attention_scale(d, rounding))
    causal = np.tril(np.ones((L, L), bool))[None, None]
    z = np.where(causal, z, -np.inf)
    m = z.max(axis=-1, keepdims=True)
    lse = m + np.log(np.sum(np.exp(z - m), axis=-1, keepdims=True))
    p = rb(np.exp(z - lse))
    o = rb(p @ v)
    return o.transpose(0, 2, 1, 3).reshape(S, L, H), p, lse[..., 0]


def attention_backward(Q, K, V, P, dO, nh: int, rounding: bool = False, O=None):
    """dQ, dK, dV of attention_forward: dP = dO Vᵀ, dV = Pᵀ dO, D = rowsum(dO ⊙ O) (= rowsum(dP ⊙ P)),
    dS = P (dP - D) / sqrt(d), dQ = dS K, dK = dSᵀ Q."""
    rb, rf = _rounders(rounding)
    S, L, H = Q.shape
    d = H // nh
    split = lambda t: np.asarray(t, f64).reshape(S, L, nh, d).transpose(0, 2, 1, 3)
    merge = lambda t: t.transpose(0, 2, 1, 3).reshape(S, L, H)
    q, k, v, do = split(Q), split(K), split(V), split(dO)
    dp = rf(do @ v.transpose(0, 1, 3, 2))
    dv = rb(P.transpose(0, 1, 3, 2) @ do)
    if O is None:
        D = np.sum(dp * P, axis=-1, keepdims=True)
    else:
        D = rf(np.sum(do * split(O), axis=-1, keepdims=True))
    ds = rb(P * (dp - D) * attention_scale(d, rounding))
    dq = rf(ds @ k)
    dk = rf(ds.transpose(0, 1, 3, 2) @ q)
    return merge(dq), merge(dk), merge(dv)


def decoder_forward(X, Wh, gammas, nh: int, rounding: bool = False):
    """The block on X [S][L][H] with the seven weights Wh (dict by DECODER_LAYERS; q/k/v/o [H][H],
    gate/up [F][H], down [H][F]) and gammas (γ1, γ2).  fp64 (with ``rounding``, the shared rounding
    points); returns every intermediate."""
    rb, rf = _rounders(rounding)
    X = np.asarray(X, f64)
    S, L, H = X.shape
    W = {n: np.asarray(Wh[n], f64) for n in DECODER_LAYERS}
    r1, inv1 = rmsnorm(X, gammas[0])
    r1 = rb(r1)
    Qp, Kp, Vv = rf(r1 @ W["q"].T), rf(r1 @ W["k"].T), rb(r1 @ W["v"].T)
    Qr, Kr = rb(rope(Qp, nh, 1.0, rounding)), rb(rope(Kp, nh, 1.0, rounding))
    O, P, lse = attention_forward(Qr, Kr, Vv, nh, rounding)
    X2 = rf(X + rf(O @ W["o"].T))
    r2, inv2 = rmsnorm(X2, gammas[1])
    r2 = rb(r2)
    a, b = rb(r2 @ W["gate"].T), rb(r2 @ W["up"].T)
    h = rb(silu(a) * b)
    Y = rf(X2 + rf(h @ W["down"].T))
    return {"X": X, "r1": r1, "inv1": inv1, "Qr": Qr, "Kr": Kr, "V": Vv, "P": P, "lse": lse, "O": O, "X2": X2,
            "r2": r2, "inv2": inv2, "a": a, "b": b, "h": h, "Y": Y}


def decoder_backward(fw, dY, Wh, gammas, nh: int, rounding: bool = False):
    """dL/dŴ for the seven weights from dY = dL/dY [S][L][H] (fp64; with ``rounding``, the shared
    rounding points, dY being the bf16 G)."""
    rb, rf = _rounders(rounding)
    W = {n: np.asarray(Wh[n], f64) for n in DECODER_LAYERS}
    S, L, H = fw["X"].shape
    flat = lambda t: t.reshape(S * L, -1)
    dY = np.asarray(dY, f64)
    g = {}
    # MLP and its norm: Y = X2 + h Wdᵀ
    g["down"] = flat(dY).T @ flat(fw["h"])
    dh = rf(dY @ W["down"])
    da = rb(dh * fw["b"] * silu_grad(fw["a"]))
    db = rb(dh * silu(fw["a"]))
    g["gate"] = flat(da).T @ flat(fw["r2"])
    g["up"] = flat(db).T @ flat(fw["r2"])
    dr2 = rf(da @ W["gate"] + db @ W["up"])
    dX2 = rb(dY + rmsnorm_backward(fw["X2"], gammas[1], fw["inv2"], dr2))
    # attention: X2 = X + O Woᵀ
    g["o"] = flat(dX2).T @ flat(fw["O"])
    dO = rb(dX2 @ W["o"])
    dQr, dKr, dV = attention_backward(fw["Qr"], fw["Kr"], fw["V"], fw["P"], dO, nh, rounding,
                                      O=fw["O"] if rounding else None)
    dQ, dK = rb(rope(dQr, nh, -1.0, rounding)), rb(rope(dKr, nh, -1.0, rounding))
    g["q"] = flat(dQ).T @ flat(fw["r1"])
    g["k"] = flat(dK).T @ flat(fw["r1"])
    g["v"] = flat(dV).T @ flat(fw["r1"])
    if rounding:
        g = {n: rf(v) for n, v in g.items()}
    return g


def decoder_smooth_loss(Ws, X, Y, states, gammas, nh, bits, group_size):
    """fp64 block loss with every rounding replaced by the identity (the smooth surrogate whose exact
    gradient the STE fold gives), its QDQ states and its forward."""
    sts = {n: qdq(Ws[n], *states[n], bits, group_size, dtype=f64, rnd=round_identity) for n in DECODER_LAYERS}
    fw = decoder_forward(X, {n: sts[n]["What"] for n in DECODER_LAYERS}, gammas, nh)
    R = fw["Y"] - np.asarray(Y, f64)
    return float(np.sum(R ** 2) / R.size), sts, fw, 2.0 * R / R.size


def decoder_smooth_grads(Ws, X, Y, states, gammas, nh, bits, group_size):
    """Loss and the STE-fold gradients (dV, dalpha, dbeta per layer) of ``decoder_smooth_loss``."""
    L, sts, fw, dY = decoder_smooth_loss(Ws, X, Y, states, gammas, nh, bits, group_size)
    gW = decoder_backward(fw, dY, {n: sts[n]["What"] for n in DECODER_LAYERS}, gammas, nh)
    return L, {n: ste_fold(gW[n], Ws[n], sts[n], bits) for n in DECODER_LAYERS}


def tune_step_decoder(Ws, X, Y, states, gammas, nh: int, cfg: QConfig, rounding: bool = False):
    """One joint SignSGD step on the seven weights of the block (QDQ in fp32 deciding the codes, the
    block in fp64, or with ``rounding`` at the GPU path's rounding points: then the loss's gradient
    G = bf16(2R/count) as for a single layer).  Returns (loss, new states, grads per layer)."""
    sts = {n: qdq(Ws[n], *states[n], cfg.bits, cfg.group_size, cfg.symmetric) for n in DECODER_LAYERS}
    Wh = {n: np.asarray(sts[n]["What_bf16"], f64) for n in DECODER_LAYERS}
    fw = decoder_forward(X, Wh, gammas, nh, rounding)
    if rounding:
        R = (fw["Y"] - np.asarray(Y, f32)).astype(f32)
        loss = float(np.sum(R.astype(f64) ** 2) / R.size)
        dY = bf16_rne((R * f32(2.0 / float(R.size))).astype(f32)).astype(f64)
    else:
        R = fw["Y"] - np.asarray(Y, f64)
        loss = float(np.sum(R ** 2) / R.size)
        dY = 2.0 * R / R.size
    gW = decoder_backward(fw, dY, Wh, gammas, nh, rounding)
    new, grads = {}, {}
    for n in DECODER_LAYERS:
        dV, da, db = ste_fold(gW[n], Ws[n], sts[n], cfg.bits, cfg.symmetric)
        V, a, b = states[n]
        new[n] = (signsgd(V, dV, cfg.lr, cfg.v_min, cfg.v_max), signsgd(a, da, cfg.lr, cfg.clip_min, cfg.clip_max),
                  signsgd(b, db, cfg.lr, cfg.clip_min, cfg.clip_max))
        grads[n] = (dV, da, db)
    return loss, new, grads
