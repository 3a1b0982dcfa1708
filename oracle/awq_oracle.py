"""Plain CPU oracle for the AWQ group-wise W4A16 path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this module:
only the tests, the smoke check (``__graft_entry__.smoke``) and the benchmark's
CPU-baseline / reference arm use it.  It shares no code with the CUDA library.

What it follows
---------------
* "AI-Research-SKILLs AWQ advanced usage guide" (lshu.cn), section 算法原理:
  the objective L(s) = || Q(W*s)(s^-1*X) - W*X ||, with s a per-input-channel
  scale derived from activation statistics, protecting salient channels by
  scaling instead of mixed precision.
* Same page, section 量化超参数调优 (group size 32/128/256 table; zero-point on =
  asymmetric with an offset, off = symmetric quantization).
* "Optimization Awq" (skillsdirectory.com), quantization-config block:
  ``{"zero_point", "q_group_size", "w_bit": 4, "version"}``.
* The quantiser's remaining arithmetic, which the pages leave open: scale = (max-min)/15,
  zero = clamp(round(-min/scale), 0, 15), q = clamp(round_half_even(w/scale) +
  zero, 0, 15) in fp32, dequant (q - zero)*scale, fp64 matmul, s = mean|X|^alpha
  over an alpha grid, int4 codes packed 8 per uint32.

Readings taken where the pages are silent (each is listed with its reason in
the design notes):
  R1  alpha grid = i/n_grid, i = 0..n_grid-1 (20 points in [0, 1)).
  R2  s = fp16_rn(pow(m, alpha)) evaluated in fp64 and rounded once to fp16,
      clamped below at 2^-14 (smallest fp16 normal); no normalisation of s.
  R3  ws = fp32(W) * fp32(s) is exact (11-bit x 11-bit significands), not rounded to fp16.
  R4  scale32 is floored at 1e-5 (constant groups); the fp16-rounded scale is
      the one stored and the one every later step divides/multiplies by.
  R5  zero = clamp(rint(-min/scale16), 0, 15) with rint = round-half-even.
  R6  zero_point off: scale = max|ws|/7, q = clamp(rint(ws/scale16), -8, 7) + 8,
      implicit zero 8, no zeros buffer.
  R7  packing: qweight [N][K/8] uint32, the 8 codes k = 8w .. 8w+7 of word w
      interleaved over its two 16-bit halves: code 8w+j in nibble CODE_NIBBLE[j] =
      (0, 4, 1, 5, 2, 6, 3, 7)[j] (bits 4*nibble ..), so that codes k, k+1 sit at the
      same place of the low and high half; zeros [N][ceil(ng/8)] uint32 in plain
      little-endian nibble order (group 8v+j in nibble j), unused nibbles 0; scales
      [N][ng] fp16.
  R8  loss = mean over (m, n) of (sum_k X[m,k] * (deq/s - W)[n,k])^2 in fp64;
      argmin with ties to the smallest alpha; the same G / zero_point as the
      final quantisation.

Pins: every function here is checked in tests/test_oracle_pins.py against
closed forms, invariants, exact rational arithmetic or brute force that do not
call the function under test.
"""
from __future__ import annotations

import numpy as np

W_BIT = 4
QMAX = 15
SCALE_FLOOR = np.float32(1e-5)
S_MIN = 2.0 ** -14
GROUP_SIZES = (32, 64, 128, 256)


# ----------------------------------------------------------------------------
# fp16 rounding
# ----------------------------------------------------------------------------

def fp16_rn(x) -> np.ndarray:
    """Round float32 or float64 values to fp16, nearest-even, in one step.

    numpy casts a float64 straight to float16 (no detour through float32), so a
    double just above an fp16 midpoint rounds up.  Pinned against exact
    rational rounding in the tests.
    """
    return np.asarray(x).astype(np.float16)


# ----------------------------------------------------------------------------
# Activation statistic and the alpha grid (scale search, steps 1-2)
# ----------------------------------------------------------------------------

def act_absmean(X16: np.ndarray) -> np.ndarray:
    """m_k = (sum_t |X[t, k]|) / M in fp64.

    Every fp16 is a multiple of 2^-24 and, for M <= 8192 tokens, the sums stay
    below 2^29, so every partial sum is exact in fp64 and the result does not
    depend on the order of summation; the single division is IEEE fp64
    round-to-nearest.
    """
    X = np.abs(np.asarray(X16, dtype=np.float16).astype(np.float64))
    return X.sum(axis=0) / np.float64(X.shape[0])


def alpha_grid(n_grid: int) -> np.ndarray:
    """alpha_i = i / n_grid for i = 0 .. n_grid-1 (reading R1)."""
    return np.arange(n_grid, dtype=np.float64) / np.float64(n_grid)


def scales_for_alpha(m: np.ndarray, alpha: float) -> np.ndarray:
    """s_k = fp16_rn(max(pow(m_k, alpha), 2^-14)) (reading R2).

    pow(0, 0) = 1, so alpha = 0 gives s = 1 everywhere (plain round-to-nearest).
    """
    p = np.power(np.asarray(m, dtype=np.float64), np.float64(alpha))
    p = np.maximum(p, S_MIN)
    return fp16_rn(p)


# ----------------------------------------------------------------------------
# Group quantisation (steps a6-a7)
# ----------------------------------------------------------------------------

def scaled_weights(W16: np.ndarray, s16) -> np.ndarray:
    """ws = fp32(W) * fp32(s) per input channel (exact, reading R3); s None means 1."""
    W16 = np.asarray(W16, dtype=np.float16)
    w32 = W16.astype(np.float32)
    if s16 is not None:
        s32 = np.asarray(s16, dtype=np.float16).astype(np.float32)
        ws = w32 * s32[None, :]                         # exact (R3)
    else:
        ws = w32
    return ws


def quantize_scaled_groups(g: np.ndarray, zero_point: bool):
    """The group quantiser on scaled weights grouped as [N][ng][G] float32: returns
    (q [N][ng][G] float32 codes 0..15, scale16 [N][ng] float16, zero [N][ng] float32).
    All arithmetic is IEEE float32 (numpy float32 ops, no fused multiply-add), rint is
    round-half-even."""
    N, ng, _ = g.shape
    if zero_point:
        mx = g.max(axis=2)
        mn = g.min(axis=2)
        scale32 = (mx - mn) / np.float32(QMAX)
        scale32 = np.maximum(scale32, SCALE_FLOOR)      # R4
        scale16 = fp16_rn(scale32)
        sc = scale16.astype(np.float32)
        zero = np.clip(np.rint(-mn / sc), 0, QMAX)      # R5
        q = np.clip(np.rint(g / sc[:, :, None]) + zero[:, :, None], 0, QMAX)
    else:
        amax = np.abs(g).max(axis=2)
        scale32 = amax / np.float32(7)
        scale32 = np.maximum(scale32, SCALE_FLOOR)
        scale16 = fp16_rn(scale32)
        sc = scale16.astype(np.float32)
        q = np.clip(np.rint(g / sc[:, :, None]), -8, 7) + 8   # R6
        zero = np.full((N, ng), 8, dtype=np.float32)
    return q, scale16, zero


def quantize_groups(W16: np.ndarray, s16, G: int, zero_point: bool):
    """Group-wise 4-bit quantisation of ws = W * diag(s).

    Returns (codes [N][K] uint8 in 0..15, scale16 [N][ng] float16,
    zeros [N][ng] uint8).  With zero_point off the zeros are the implicit 8.
    """
    W16 = np.asarray(W16, dtype=np.float16)
    N, K = W16.shape
    if K % G:
        raise ValueError("K must be a multiple of the group size")
    ng = K // G
    g = scaled_weights(W16, s16).reshape(N, ng, G)
    q, scale16, zero = quantize_scaled_groups(g, zero_point)
    codes = q.reshape(N, K).astype(np.uint8)
    return codes, scale16, zero.astype(np.uint8)


# ----------------------------------------------------------------------------
# Packing (reading R7)
# ----------------------------------------------------------------------------

def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """Plain packing (the zero points, R7): [R][C] values 0..15 -> [R][ceil(C/8)] uint32,
    value j of a word in bits 4j..4j+3."""
    codes = np.asarray(codes, dtype=np.uint32)
    R, C = codes.shape
    W = (C + 7) // 8
    padded = np.zeros((R, W * 8), dtype=np.uint32)
    padded[:, :C] = codes
    p = padded.reshape(R, W, 8)
    out = np.zeros((R, W), dtype=np.uint32)
    for j in range(8):
        out |= p[:, :, j] << np.uint32(4 * j)
    return out


def unpack_nibbles(words: np.ndarray, C: int) -> np.ndarray:
    """Inverse of pack_nibbles: [R][W] uint32 -> [R][C] uint8."""
    words = np.asarray(words, dtype=np.uint32)
    R, W = words.shape
    out = np.zeros((R, W, 8), dtype=np.uint8)
    for j in range(8):
        out[:, :, j] = (words >> np.uint32(4 * j)) & np.uint32(0xF)
    return out.reshape(R, W * 8)[:, :C]


# Nibble of code j (0..7) within a qweight word: codes k, k+1 share a position in the
# two 16-bit halves, so one mask of a word yields the adjacent pair (k, k+1).
CODE_NIBBLE = (0, 4, 1, 5, 2, 6, 3, 7)


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """qweight packing (R7): [R][C] codes 0..15 -> [R][ceil(C/8)] uint32, code j of a word
    in nibble CODE_NIBBLE[j]."""
    codes = np.asarray(codes, dtype=np.uint32)
    R, C = codes.shape
    W = (C + 7) // 8
    padded = np.zeros((R, W * 8), dtype=np.uint32)
    padded[:, :C] = codes
    p = padded.reshape(R, W, 8)
    out = np.zeros((R, W), dtype=np.uint32)
    for j in range(8):
        out |= p[:, :, j] << np.uint32(4 * CODE_NIBBLE[j])
    return out


def unpack_codes(words: np.ndarray, C: int) -> np.ndarray:
    """Inverse of pack_codes: [R][W] uint32 -> [R][C] uint8."""
    words = np.asarray(words, dtype=np.uint32)
    R, W = words.shape
    out = np.zeros((R, W, 8), dtype=np.uint8)
    for j in range(8):
        out[:, :, j] = (words >> np.uint32(4 * CODE_NIBBLE[j])) & np.uint32(0xF)
    return out.reshape(R, W * 8)[:, :C]


def quantize_pack(W16: np.ndarray, s16, G: int, zero_point: bool):
    """The awq_quantize_pack operation: (qweight, scales, qzeros or None)."""
    codes, scale16, zeros = quantize_groups(W16, s16, G, zero_point)
    qweight = pack_codes(codes)
    qzeros = pack_nibbles(zeros) if zero_point else None
    return qweight, scale16, qzeros


def dequantize(qweight, scales, qzeros, K: int, G: int, zero_point: bool) -> np.ndarray:
    """deq[n][k] = (q - zero) * scale16 in fp64 (exact)."""
    N = qweight.shape[0]
    ng = K // G
    q = unpack_codes(qweight, K).astype(np.float64).reshape(N, ng, G)
    if zero_point:
        z = unpack_nibbles(qzeros, ng).astype(np.float64)
    else:
        z = np.full((N, ng), 8.0)
    sc = np.asarray(scales, dtype=np.float16).astype(np.float64)
    return ((q - z[:, :, None]) * sc[:, :, None]).reshape(N, K)


# ----------------------------------------------------------------------------
# The fused linear (steps a8-a9): y = X . deq(W)^T
# ----------------------------------------------------------------------------

def linear(X16, qweight, scales, qzeros, K: int, G: int, zero_point: bool) -> np.ndarray:
    """y_ref[m][n] = sum_k X[m][k] * deq[n][k], fp64 (library matmul as one step)."""
    deq = dequantize(qweight, scales, qzeros, K, G, zero_point)
    X = np.asarray(X16, dtype=np.float16).astype(np.float64)
    return X @ deq.T


def linear_rows(X16, qweight, scales, qzeros, K: int, G: int, zero_point: bool, rows) -> np.ndarray:
    """y_ref restricted to output channels ``rows`` (sampled checks at full size)."""
    rows = np.asarray(rows)
    sub_q = np.asarray(qweight)[rows]
    sub_s = np.asarray(scales)[rows]
    sub_z = np.asarray(qzeros)[rows] if zero_point else None
    return linear(X16, sub_q, sub_s, sub_z, K, G, zero_point)


def fold_inverse_scale(X16, s16) -> np.ndarray:
    """X' = fp16_rn(fp32(X) / fp32(s)): the activation side s^-1 * X of the
    objective, rounded to fp16 once (IEEE fp32 division)."""
    X = np.asarray(X16, dtype=np.float16).astype(np.float32)
    s = np.asarray(s16, dtype=np.float16).astype(np.float32)
    return fp16_rn(X / s[None, :])


# ----------------------------------------------------------------------------
# Scale search (steps a1-a5)
# ----------------------------------------------------------------------------

def search_loss(X16, W16, s16, G: int, zero_point: bool) -> float:
    """mean_{m,n} (X . (Q(W s)/s - W)^T)^2 in fp64 (reading R8)."""
    codes, scale16, zeros = quantize_groups(W16, s16, G, zero_point)
    N, K = codes.shape
    ng = K // G
    q = codes.astype(np.float64).reshape(N, ng, G)
    z = zeros.astype(np.float64)[:, :, None]
    sc = scale16.astype(np.float64)[:, :, None]
    deq = ((q - z) * sc).reshape(N, K)
    s = np.asarray(s16, dtype=np.float16).astype(np.float64)
    dW = deq / s[None, :] - np.asarray(W16, dtype=np.float16).astype(np.float64)
    X = np.asarray(X16, dtype=np.float16).astype(np.float64)
    E = X @ dW.T
    return float(np.mean(E * E))


def scale_search(X16, W16, G: int, zero_point: bool, n_grid: int = 20):
    """Grid search over alpha: returns (best_index, alpha*, s* fp16 [K], losses fp64 [n_grid])."""
    m = act_absmean(X16)
    alphas = alpha_grid(n_grid)
    losses = np.empty(n_grid, dtype=np.float64)
    for i, a in enumerate(alphas):
        losses[i] = search_loss(X16, W16, scales_for_alpha(m, a), G, zero_point)
    best = int(np.argmin(losses))           # first minimum: ties go to the smaller alpha
    return best, float(alphas[best]), scales_for_alpha(m, alphas[best]), losses


# ----------------------------------------------------------------------------
# duo_scaling: the scale from an activation and a weight statistic (reading D1)
# ----------------------------------------------------------------------------

S_MAX = 65504.0


def weight_absmean(W16) -> np.ndarray:
    """w_k = (sum_n |W[n, k]|) / N in fp64: the weights' counterpart of act_absmean (the
    sums are exact while N * max|W| < 2^29)."""
    Wa = np.abs(np.asarray(W16, dtype=np.float16).astype(np.float64))
    return Wa.sum(axis=0) / np.float64(Wa.shape[0])


def duo_scales_for_alpha(m: np.ndarray, w: np.ndarray, alpha: float) -> np.ndarray:
    """s_k = fp16_rn(min(max(a_k / b_k, 2^-14), 65504)) with a_k = max(pow(m_k, alpha), 2^-14)
    and b_k = max(pow(w_k, 1 - alpha), 2^-14), all in fp64, rounded once to fp16.

    The activation statistic raised to alpha, divided by the weight statistic raised to
    1 - alpha (the weights' share of the scaling).  With w = 1 it is scales_for_alpha."""
    a = np.maximum(np.power(np.asarray(m, dtype=np.float64), np.float64(alpha)), S_MIN)
    b = np.maximum(np.power(np.asarray(w, dtype=np.float64), np.float64(1.0) - np.float64(alpha)), S_MIN)
    return fp16_rn(np.minimum(np.maximum(a / b, S_MIN), S_MAX))


def scale_search_duo(X16, W16, G: int, zero_point: bool, n_grid: int = 20):
    """The grid search with duo scaling: (best_index, alpha*, s* fp16 [K], losses [n_grid]),
    the loss and the tie rule as in scale_search."""
    m = act_absmean(X16)
    w = weight_absmean(W16)
    alphas = alpha_grid(n_grid)
    losses = np.empty(n_grid, dtype=np.float64)
    for i, a in enumerate(alphas):
        losses[i] = search_loss(X16, W16, duo_scales_for_alpha(m, w, a), G, zero_point)
    top = int(np.argmin(losses))            # first minimum: ties go to the smaller alpha
    return top, float(alphas[top]), duo_scales_for_alpha(m, w, alphas[top]), losses


# ----------------------------------------------------------------------------
# apply_clip: per-group weight clipping chosen by the group's output error (reading C1)
# ----------------------------------------------------------------------------

def clip_ratios(n_grid: int, n_clip: int) -> np.ndarray:
    """r_j = 1 - j / n_grid for j = 0 .. n_clip - 1, evaluated in fp64, rounded to fp32."""
    j = np.arange(n_clip, dtype=np.float64)
    return (np.float64(1.0) - j / np.float64(n_grid)).astype(np.float32)


def clip_groups(g: np.ndarray, ratio) -> np.ndarray:
    """Clamp each group of scaled weights [N][ng][G] to [-c, c] with c = fl32(ratio *
    max|group|); `ratio` is a float32 scalar or an [N][ng] array."""
    amax = np.abs(g).max(axis=2)
    c = (np.asarray(ratio, dtype=np.float32) * amax).astype(np.float32)
    return np.clip(g, -c[:, :, None], c[:, :, None])


def clip_errors(X16, W16, s16, G: int, zero_point: bool, n_grid: int = 20, n_clip: int = 10) -> np.ndarray:
    """err[n, g, j] = sum_t (sum_{k in g} X[t, k] (Q(clip_j(W s)) / s - W)[n, k])^2 in fp64:
    the objective's share of one group of one output channel, for clip ratio r_j."""
    W16 = np.asarray(W16, dtype=np.float16)
    N, K = W16.shape
    ng = K // G
    X = np.asarray(X16, dtype=np.float16).astype(np.float64)
    Wd = W16.astype(np.float64)
    s = np.asarray(s16, dtype=np.float16).astype(np.float64)
    g = scaled_weights(W16, s16).reshape(N, ng, G)
    err = np.empty((N, ng, n_clip), dtype=np.float64)
    for j, r in enumerate(clip_ratios(n_grid, n_clip)):
        q, scale16, zero = quantize_scaled_groups(clip_groups(g, r), zero_point)
        deq = ((q.astype(np.float64) - zero.astype(np.float64)[:, :, None])
               * scale16.astype(np.float64)[:, :, None]).reshape(N, K)
        dW = deq / s[None, :] - Wd
        for gi in range(ng):
            E = X[:, gi * G:(gi + 1) * G] @ dW[:, gi * G:(gi + 1) * G].T      # [M][N]
            err[:, gi, j] = (E * E).sum(axis=0)
    return err


def quantize_pack_clipped(W16, s16, G: int, zero_point: bool, clip_index, n_grid: int = 20):
    """awq_quantize_pack of W * diag(s) with group (n, g) first clipped at ratio
    r_{clip_index[n, g]}: (qweight, scales, qzeros or None)."""
    W16 = np.asarray(W16, dtype=np.float16)
    N, K = W16.shape
    ng = K // G
    idx = np.asarray(clip_index)
    ratios = clip_ratios(n_grid, int(idx.max()) + 1)[idx]
    g = clip_groups(scaled_weights(W16, s16).reshape(N, ng, G), ratios)
    q, scale16, zero = quantize_scaled_groups(g, zero_point)
    qweight = pack_codes(q.reshape(N, K).astype(np.uint8))
    qzeros = pack_nibbles(zero.astype(np.uint8)) if zero_point else None
    return qweight, scale16, qzeros


def clip_search(X16, W16, s16, G: int, zero_point: bool, n_grid: int = 20, n_clip: int = 10):
    """apply_clip: per (n, g) the clip index with the smallest error (ties to the smaller
    index, i.e. less clipping), and the packed weights clipped accordingly:
    (clip_index [N][ng] int, err [N][ng][n_clip], (qweight, scales, qzeros))."""
    err = clip_errors(X16, W16, s16, G, zero_point, n_grid, n_clip)
    idx = np.argmin(err, axis=2)            # first minimum
    return idx, err, quantize_pack_clipped(W16, s16, G, zero_point, idx, n_grid)
