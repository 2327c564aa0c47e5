"""Plain float64 restatement of the joint-attention hot path.

TEST INFRASTRUCTURE ONLY (see the package docstring).  Layout conventions
shared with the CUDA path are only the array shapes: activations are
``[B, N, H, d]`` token-major with ``N = N_txt + N_img + N_ref`` tokens in the
order text, noisy target image, reference image.
"""

from __future__ import annotations

import numpy as np

# Largest finite E4M3FN magnitude (OCP 8-bit floating point format, E4M3 with
# bias 7, no infinities, S.1111.111 reserved for NaN): 1.75 * 2**8.
E4M3_MAX = 448.0


# ---------------------------------------------------------------------------
# bf16 rounding (used to model the bf16 tensors the pipeline stores)
# ---------------------------------------------------------------------------

def bf16_round(x) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 value, ties to even.

    bfloat16 has 8 significant bits (1 implicit + 7 stored) and the float32
    exponent range.  Written from the definition: scale the value so that
    its significand is an integer on the bf16 grid, round half to even
    (``np.rint``), scale back.  Values below the smallest normal 2**-126
    use the fixed subnormal quantum 2**-133.  Overflow is not expected on
    any workload and maps to +-inf.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    finite = np.isfinite(x) & (x != 0)
    m, e = np.frexp(x[finite])  # x = m * 2**e, 0.5 <= |m| < 1
    normal = (e - 1) >= -126
    q = np.where(normal, np.rint(m * 256.0) * np.ldexp(1.0, e - 8),
                 np.rint(x[finite] * 2.0 ** 133) * 2.0 ** -133)
    q = np.where(np.abs(q) > 3.3895313892515355e38, np.copysign(np.inf, q), q)
    out[finite] = q
    out[~np.isfinite(x)] = x[~np.isfinite(x)]
    return out


def bf16_ulp_distance(a, b) -> np.ndarray:
    """Distance in bf16 code points between two arrays of bf16-exact values.

    Both inputs must already be exactly representable in bf16.  The distance
    is taken on the sign-magnitude ordinal of the float32 bit pattern, so
    +0 and -0 are 0 apart and adjacent bf16 values are 1 apart.
    """
    def ordinal(v):
        bits = np.asarray(v, dtype=np.float32).view(np.uint32).astype(np.int64) >> 16
        mag = bits & 0x7FFF
        return np.where(bits & 0x8000, -mag, mag)
    return np.abs(ordinal(a) - ordinal(b))


# ---------------------------------------------------------------------------
# Prologue: per-head RMSNorm, then 2-D RoPE on (row, col) token positions
# ---------------------------------------------------------------------------

def rmsnorm(x, w=None, eps: float = 1e-6) -> np.ndarray:
    """RMSNorm over the last axis: ``x / sqrt(mean(x**2) + eps) * w``.

    The tutorial's "GEMM kernel optimization" section names query/key
    normalisation in the QKV epilogue without defining it; the reading here
    is the usual per-head RMSNorm over head_dim with a learned weight of
    length head_dim (1.0 on every workload) and eps = 1e-6.
    """
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    y = x / np.sqrt(ms + eps)
    if w is not None:
        y = y * np.asarray(w, dtype=np.float64)
    return y


def token_positions(n_txt: int, img_h: int, img_w: int,
                    ref_h: int = 0, ref_w: int = 0, ref_row_offset: int = 0, ref_grids=None):
    """(row, col) RoPE positions of the joint sequence [text | image | ref].

    Text tokens sit at (0, 0).  Image token t' (0-based within the image
    stream) sits at (t' // img_w, t' % img_w), i.e. the latent grid is
    flattened row-major.  Reference token t'' sits at
    (ref_row_offset + t'' // ref_w, t'' % ref_w): the reference grid is a
    second grid shifted down by ``ref_row_offset`` rows.

    Several reference images (the tutorial's editing command repeats
    ``--image`` for multiple references; the pages give no position rule
    for them): ``ref_grids`` lists one ``(h, w, row_offset, col_offset)``
    per reference, in sequence order, and replaces ref_h / ref_w /
    ref_row_offset.  Token u of reference g sits at
    (row_offset_g + u // w_g, col_offset_g + u % w_g).  One grid
    ``(ref_h, ref_w, ref_row_offset, 0)`` is the single-reference rule.
    """
    if ref_grids is None:
        ref_grids = [(ref_h, ref_w, ref_row_offset, 0)] if ref_h * ref_w > 0 else []
    n_img = img_h * img_w
    n_ref = sum(h * w for h, w, _, _ in ref_grids)
    rows = np.zeros(n_txt + n_img + n_ref, dtype=np.int64)
    cols = np.zeros_like(rows)
    for t in range(n_img):
        rows[n_txt + t] = t // img_w
        cols[n_txt + t] = t % img_w
    start = n_txt + n_img
    for h, w, row0, col0 in ref_grids:
        for u in range(h * w):
            rows[start + u] = row0 + u // w
            cols[start + u] = col0 + u % w
        start += h * w
    return rows, cols


def rope_2d(x, pos_row, pos_col, theta: float = 10000.0) -> np.ndarray:
    """Two-axis rotary embedding of vectors ``x[..., N, H, d]``.

    Reading of the workload text "split 64/64 over (row, col)": channels
    0..d/2-1 are an ordinary RoPE of width d/2 driven by the row position,
    channels d/2..d-1 the same driven by the column position.  Inside a
    half, channel pair (2i, 2i+1) rotates by angle pos * theta**(-2i/(d/2)):

        (a, b) -> (a cos(phi) - b sin(phi), a sin(phi) + b cos(phi)).

    ``pos_row`` / ``pos_col`` have length N (one position per token).
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    half = d // 2
    out = x.copy()
    for axis, pos in ((0, pos_row), (1, pos_col)):
        pos = np.asarray(pos, dtype=np.float64)
        for i in range(half // 2):
            omega = theta ** (-2.0 * i / half)
            phi = pos * omega                      # [N]
            c = np.cos(phi)[:, None]               # broadcast over heads
            s = np.sin(phi)[:, None]
            ia = axis * half + 2 * i
            a = x[..., ia]
            b = x[..., ia + 1]
            out[..., ia] = a * c - b * s
            out[..., ia + 1] = a * s + b * c
    return out


def prologue(q, k, *, n_txt: int, img_h: int, img_w: int,
             ref_h: int = 0, ref_w: int = 0, ref_row_offset: int = 0, ref_grids=None,
             theta: float = 10000.0, eps: float = 1e-6,
             q_norm_w=None, k_norm_w=None):
    """Q' = RoPE(RMSNorm(Q)), K' = RoPE(RMSNorm(K)), in float64.

    Order norm-then-RoPE as the QKV epilogue in the tutorial's "GEMM kernel
    optimization" section lists them.  V passes through untouched.  Inputs
    ``[B, N, H, d]``; returns unrounded float64 arrays of the same shape.
    """
    rows, cols = token_positions(n_txt, img_h, img_w, ref_h, ref_w, ref_row_offset, ref_grids)
    qn = rmsnorm(q, q_norm_w, eps)
    kn = rmsnorm(k, k_norm_w, eps)
    return rope_2d(qn, rows, cols, theta), rope_2d(kn, rows, cols, theta)


def rope_table(n_txt: int, img_h: int, img_w: int, ref_h: int = 0, ref_w: int = 0,
               ref_row_offset: int = 0, ref_grids=None, theta: float = 10000.0) -> np.ndarray:
    """(cos, sin) of every token's 64 rotation angles, ``[N, 64, 2]`` float64.

    Entry (t, j): angle pos * theta**(-2 (j mod 32) / 64) with pos the row
    position of token t for j < 32 and its column position for j >= 32 --
    the angle ``rope_2d`` applies to channel pair (2j, 2j+1) of a 128-wide
    head.
    """
    rows, cols = token_positions(n_txt, img_h, img_w, ref_h, ref_w, ref_row_offset, ref_grids)
    n = len(rows)
    out = np.empty((n, 64, 2), dtype=np.float64)
    for j in range(64):
        pos = (rows if j < 32 else cols).astype(np.float64)
        phi = pos * theta ** (-2.0 * (j % 32) / 64.0)
        out[:, j, 0] = np.cos(phi)
        out[:, j, 1] = np.sin(phi)
    return out


def qkv_fused(x, w_txt, w_img, *, n_txt: int, img_h: int, img_w: int, H: int,
              ref_h: int = 0, ref_w: int = 0, ref_row_offset: int = 0, ref_grids=None,
              theta: float = 10000.0, eps: float = 1e-6,
              q_norm_w=(None, None), k_norm_w=(None, None)):
    """QKV projection with the prologue in its epilogue, in float64.

    The tutorial's "GEMM kernel optimization" section fuses query/key
    normalisation and RoPE into the QKV projection; its "FLUX 3 inference"
    section has the text and image streams processed separately until the
    joint attention.  Reading: each stream s has its own projection
    ``W_s`` (``[3 H d, C]``, rows = Q heads, K heads, V heads) and its own
    Q/K norm weights; reference-image tokens use the image stream's.
    ``x`` is ``[B, N, C]``.  Returns unrounded float64 ``Q', K', V``
    ``[B, N, H, d]``: Q' = RoPE(RMSNorm(x W_s,q^T) * q_norm_w[s]), K' likewise,
    V = x W_s,v^T.
    """
    x = np.asarray(x, dtype=np.float64)
    B, N, C = x.shape
    d = 128
    y = np.empty((B, N, 3 * H * d), dtype=np.float64)
    y[:, :n_txt] = x[:, :n_txt] @ np.asarray(w_txt, dtype=np.float64).T if n_txt > 0 else 0.0
    if N > n_txt:
        y[:, n_txt:] = x[:, n_txt:] @ np.asarray(w_img, dtype=np.float64).T
    q = y[..., :H * d].reshape(B, N, H, d)
    k = y[..., H * d:2 * H * d].reshape(B, N, H, d)
    v = y[..., 2 * H * d:].reshape(B, N, H, d)
    qn = np.empty_like(q)
    kn = np.empty_like(k)
    for s, sl in ((0, slice(0, n_txt)), (1, slice(n_txt, N))):
        qn[:, sl] = rmsnorm(q[:, sl], q_norm_w[s], eps)
        kn[:, sl] = rmsnorm(k[:, sl], k_norm_w[s], eps)
    rows, cols = token_positions(n_txt, img_h, img_w, ref_h, ref_w, ref_row_offset, ref_grids)
    return rope_2d(qn, rows, cols, theta), rope_2d(kn, rows, cols, theta), v


# ---------------------------------------------------------------------------
# E4M3 block quantisation (FP8 path)
# ---------------------------------------------------------------------------

def e4m3_decode(codes) -> np.ndarray:
    """Value of each E4M3FN byte, from the format definition.

    Bit 7 sign, bits 6..3 exponent (bias 7), bits 2..0 mantissa.  Exponent
    field 0 is subnormal: (m/8) * 2**-6.  Otherwise (1 + m/8) * 2**(E-7).
    The all-ones exponent with mantissa 7 is NaN; there is no infinity.
    """
    c = np.asarray(codes, dtype=np.int64) & 0xFF
    s = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 7).astype(np.float64)
    val = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = np.where((e == 15) & (m == 7), np.nan, val)
    return s * val


_POS_CODES = np.arange(0x7F, dtype=np.int64)          # 0x00..0x7E: all finite >= 0
_POS_VALUES = e4m3_decode(_POS_CODES)                  # strictly increasing


def e4m3_encode(v) -> np.ndarray:
    """Round values to E4M3FN codes: nearest, ties to even, saturate to finite.

    Written from the definition of round-to-nearest-even on the finite
    value set: clamp |v| to 448 ("satfinite"), pick the nearest of the 127
    non-negative finite values, and on an exact tie take the code whose
    last mantissa bit is 0.  The sign bit is carried separately and kept
    when the magnitude rounds to zero (a negative value gives -0, code
    0x80, as IEEE rounding does); NaN maps to 0x7F.
    """
    v = np.asarray(v, dtype=np.float64)
    a = np.minimum(np.abs(v), E4M3_MAX)
    hi = np.clip(np.searchsorted(_POS_VALUES, a, side="left"), 0, len(_POS_VALUES) - 1)
    lo = np.clip(hi - 1, 0, None)
    d_hi = _POS_VALUES[hi] - a
    d_lo = a - _POS_VALUES[lo]
    pick_lo = (d_lo < d_hi) | ((d_lo == d_hi) & ((_POS_CODES[lo] & 1) == 0))
    code = np.where(pick_lo, _POS_CODES[lo], _POS_CODES[hi])
    code = np.where(np.signbit(v), code | 0x80, code)
    code = np.where(np.isnan(v), 0x7F, code)
    return code.astype(np.uint8)


def block_quantize_e4m3(x, block: int = 64):
    """Per-(b, h, 64-token block) absmax E4M3 quantisation of ``x[B, N, H, d]``.

    Reading of the FP8 workload: one scale per (batch, head, block of 64
    consecutive joint-sequence tokens counted from token 0) covering all d
    channels; the last block may be partial and blocks may straddle the
    text/image boundary.  All arithmetic is float32, emulated exactly:

        amax  = max |x| over the block            (x exact in float32)
        inv   = fl32(448 / amax)                  (correctly rounded)
        code  = E4M3_RNE_satfinite(fl32(x * inv))
        scale = fl32(amax / 448)

    An all-zero block stores scale 1.0 and all-zero codes.  Returns
    ``codes uint8 [B, N, H, d]`` and ``scales float32 [B, H, ceil(N/64)]``;
    the value a code stands for is ``e4m3_decode(code) * scale``.
    """
    x32 = np.asarray(x, dtype=np.float32)
    if not np.array_equal(x32.astype(np.float64), np.asarray(x, dtype=np.float64)):
        raise ValueError("block_quantize_e4m3 expects values exact in float32")
    B, N, H, d = x32.shape
    nblk = -(-N // block)
    codes = np.zeros((B, N, H, d), dtype=np.uint8)
    scales = np.ones((B, H, nblk), dtype=np.float32)
    f448 = np.float32(E4M3_MAX)
    for b in range(B):
        for h in range(H):
            for j in range(nblk):
                t0, t1 = j * block, min(N, (j + 1) * block)
                tile = x32[b, t0:t1, h, :]
                amax = np.float32(np.max(np.abs(tile)))
                if amax == 0:
                    continue
                inv = np.float32(f448 / amax)
                codes[b, t0:t1, h, :] = e4m3_encode(tile * inv)   # float32 multiply
                scales[b, h, j] = np.float32(amax / f448)
    return codes, scales


def dequantize_e4m3(codes, scales, block: int = 64) -> np.ndarray:
    """float64 values ``e4m3_decode(code) * scale`` in ``[B, N, H, d]``."""
    B, N, H, d = codes.shape
    vals = e4m3_decode(codes)
    tok_blk = np.arange(N) // block
    s = np.asarray(scales, dtype=np.float64)[:, :, tok_blk]      # [B, H, N]
    return vals * np.transpose(s, (0, 2, 1))[..., None]


# ---------------------------------------------------------------------------
# Joint attention
# ---------------------------------------------------------------------------

def joint_attention(q, k, v, scale: float, rows=None):
    """O = softmax(scale * Q K^T) V over the whole joint sequence, per (b, h).

    The tutorial's "FLUX 3 inference with TensorRT LLM VisualGen" section
    has the three token streams meet in one joint attention; no mask is
    stated, so every query attends to every key of all streams.  ``scale``
    is the caller's float, widened to float64.  ``rows`` optionally selects
    query indices per call (same for every (b, h)); the result then has
    ``len(rows)`` rows.  Returns ``O [B, R, H, d]`` float64 and the
    log-sum-exp ``L [B, H, R]`` = ln sum_j exp(scale * q.k_j).
    """
    B, N, H, d = q.shape
    idx = np.arange(N) if rows is None else np.asarray(rows)
    R = len(idx)
    out = np.empty((B, R, H, v.shape[-1]), dtype=np.float64)
    lse = np.empty((B, H, R), dtype=np.float64)
    sc = float(scale)
    f64 = lambda a: np.asarray(a, dtype=np.float64)   # widen one (b, h) slice at a time
    for b in range(B):
        for h in range(H):
            s = sc * (f64(q[b, idx, h, :]) @ f64(k[b, :, h, :]).T)   # [R, N]
            m = np.max(s, axis=1, keepdims=True)
            p = np.exp(s - m)
            l = np.sum(p, axis=1, keepdims=True)
            out[b, :, h, :] = (p / l) @ f64(v[b, :, h, :])
            lse[b, h, :] = (m + np.log(l))[:, 0]
    return out, lse


__all__ = [
    "E4M3_MAX", "bf16_round", "bf16_ulp_distance", "rmsnorm", "token_positions",
    "rope_2d", "prologue", "e4m3_decode", "e4m3_encode", "block_quantize_e4m3",
    "dequantize_e4m3", "joint_attention",
]


# ---------------------------------------------------------------------------
# FP8 attention with a repair budget (VC-Attention style)
# ---------------------------------------------------------------------------

def repair_count(n: int, rho: float) -> int:
    """Tokens repaired per (b, h): ceil(rho * N), at most N (0 for rho 0)."""
    return min(n, int(np.ceil(rho * n - 1e-9))) if rho > 0 else 0


def repair_select(k_exact, v_exact, k_deq, v_deq, rho: float):
    """Key/value tokens with the highest quantisation error, per (b, h).

    The tutorial's "Quantized and sparse attention" section runs
    VC-Attention FP8 with a repair budget rho = 0.005: a share rho of the
    tokens, those that quantisation hurt most, gets a residual correction.
    The pages do not define the error.  Reading: the error of token t
    of (b, h) is the squared distance between its exact key and value rows
    (the bf16 K' and V the prologue quantises) and their dequantised E4M3
    values, summed over the d channels of both:

        e_t = sum_c (K'_tc - Kd_tc)^2 + sum_c (V_tc - Vd_tc)^2,

    and the ``repair_count(N, rho)`` tokens with the largest e_t (ties to the
    lower token index) are selected.  Returns ``idx int64 [B, H, m]`` (the
    selected tokens in increasing token order) and the errors ``[B, H, N]``
    (float64).
    """
    ke, ve = np.asarray(k_exact, np.float64), np.asarray(v_exact, np.float64)
    kd, vd = np.asarray(k_deq, np.float64), np.asarray(v_deq, np.float64)
    B, N, H, d = ke.shape
    err = np.transpose(np.sum((ke - kd) ** 2, axis=-1) + np.sum((ve - vd) ** 2, axis=-1), (0, 2, 1))
    m = repair_count(N, rho)
    idx = np.empty((B, H, m), dtype=np.int64)
    for b in range(B):
        for h in range(H):
            # Stable sort on -err: equal errors keep increasing token order.
            idx[b, h] = np.sort(np.argsort(-err[b, h], kind="stable")[:m])
    return idx, err


def repaired_attention(q_deq, k_deq, v_deq, k_exact, v_exact, idx, scale: float):
    """FP8 attention whose selected keys are repaired: for each (b, h), the
    tokens in ``idx[b, h]`` attend with their exact K' and V rows, all other
    keys with the dequantised ones; queries stay dequantised.  Returns
    ``O [B, N, H, d]`` and ``L [B, H, N]`` (float64), as joint_attention."""
    k = np.array(k_deq, dtype=np.float64)
    v = np.array(v_deq, dtype=np.float64)
    B, N, H, d = k.shape
    for b in range(B):
        for h in range(H):
            t = np.asarray(idx[b, h])
            k[b, t, h, :] = np.asarray(k_exact, np.float64)[b, t, h, :]
            v[b, t, h, :] = np.asarray(v_exact, np.float64)[b, t, h, :]
    return joint_attention(q_deq, k, v, scale)


# ---------------------------------------------------------------------------
# Block-sparse attention (Sol-Attention style)
# ---------------------------------------------------------------------------
#
# The tutorial's "Quantized and sparse attention" section runs Sol-Attention
# through a generic block-sparse attention kernel, with the sparsity set by
# a parameter tau (tau = 1.0 in its tests; a higher tau lowers quality for
# little extra speed) and the first denoising steps kept dense.  It does not
# define tau or the block rule.  Reading used here (parity unpinned against
# the pages for the meaning of tau; the rule below is pinned as stated):
#
#   blocks     query blocks of SPARSE_QBLOCK consecutive joint-sequence
#              tokens, key blocks of SPARSE_KBLOCK, counted from token 0 of
#              each (b, h); the last block of each kind may be partial;
#   pooled     qbar_i, kbar_j = mean of the block's Q' (resp. K') rows;
#   score      p_ij = softmax_j(scale * qbar_i . kbar_j) over the n_kb key
#              blocks of the (b, h);
#   keep       key block j for query block i iff p_ij >= tau / n_kb (at least
#              tau times the uniform share), and always the block with the
#              largest p_ij (lowest index among equals), so no row is empty;
#   attention  each query attends, with an ordinary softmax, to the keys of
#              its query block's kept key blocks only.
# tau = 0 keeps every block (dense attention); a larger tau keeps a subset.

SPARSE_QBLOCK = 256
SPARSE_KBLOCK = 128


def sparse_pool(x, block: int) -> np.ndarray:
    """Mean of ``x[B, N, H, d]`` over consecutive blocks of ``block`` tokens
    (the last one partial), per (b, h): ``[B, H, ceil(N / block), d]``."""
    x = np.asarray(x, dtype=np.float64)
    B, N, H, d = x.shape
    nb = -(-N // block)
    out = np.empty((B, H, nb, d), dtype=np.float64)
    for i in range(nb):
        out[:, :, i, :] = np.mean(x[:, i * block:min(N, (i + 1) * block)], axis=1)
    return out


def sparse_probs(q, k, scale: float, qblock: int = SPARSE_QBLOCK, kblock: int = SPARSE_KBLOCK) -> np.ndarray:
    """Pooled block attention ``p [B, H, n_qb, n_kb]`` (float64): row i is
    softmax_j(scale * qbar_i . kbar_j)."""
    qb, kb = sparse_pool(q, qblock), sparse_pool(k, kblock)
    s = float(scale) * np.einsum("bhic,bhjc->bhij", qb, kb)
    s -= np.max(s, axis=-1, keepdims=True)
    e = np.exp(s)
    return e / np.sum(e, axis=-1, keepdims=True)


def sparse_keep(probs, tau: float) -> np.ndarray:
    """Kept key blocks ``bool [..., n_qb, n_kb]`` from pooled probabilities.

    The decision is taken in float32, the precision the GPU path computes
    ``probs`` in: keep iff ``float32(p) >= float32(tau) / float32(n_kb)``
    (one correctly rounded division), plus the first block of largest p.
    """
    p = np.asarray(probs, dtype=np.float32)
    nkb = p.shape[-1]
    thr = np.float32(tau) / np.float32(nkb)
    keep = p >= thr
    top = np.argmax(p, axis=-1)   # first index of the maximum
    np.put_along_axis(keep, top[..., None], True, axis=-1)
    return keep


def block_sparse_attention(q, k, v, keep, scale: float, rows=None,
                           qblock: int = SPARSE_QBLOCK, kblock: int = SPARSE_KBLOCK):
    """Attention of each query over the keys of its query block's kept key
    blocks: ``keep[b, h, i, j]`` for query block i = t // qblock and key
    block j.  A query whose block keeps nothing gets O = 0 and L = -inf.
    ``rows`` selects query indices as in joint_attention.  Returns
    ``O [B, R, H, d]`` and ``L [B, H, R]`` (float64)."""
    B, N, H, d = q.shape
    idx = np.arange(N) if rows is None else np.asarray(rows)
    R = len(idx)
    keep = np.asarray(keep, dtype=bool)
    out = np.zeros((B, R, H, v.shape[-1]), dtype=np.float64)
    lse = np.full((B, H, R), -np.inf, dtype=np.float64)
    sc = float(scale)
    f64 = lambda a: np.asarray(a, dtype=np.float64)
    key_block = np.arange(N) // kblock
    for b in range(B):
        for h in range(H):
            # Rows sharing a query block share the key set.
            for i in np.unique(idx // qblock):
                sel = np.nonzero(idx // qblock == i)[0]
                cols = np.nonzero(keep[b, h, i][key_block])[0]
                if cols.size == 0:
                    continue
                s = sc * (f64(q[b, idx[sel], h, :]) @ f64(k[b, cols, h, :]).T)   # [rows, keys]
                m = np.max(s, axis=1, keepdims=True)
                p = np.exp(s - m)
                l = np.sum(p, axis=1, keepdims=True)
                out[b, sel, h, :] = (p / l) @ f64(v[b, cols, h, :])
                lse[b, h, sel] = (m + np.log(l))[:, 0]
    return out, lse
