"""CPU oracle for the W4A8 MoE expert FFN -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its CPU-baseline
and reference legs) may import this module.  The product path (the CUDA library
and its Python binding) never calls it and shares no code with it.

It is a plain, slow, step-by-step restatement of what the pages define, in
numpy.  Floating point that only feeds a tolerance comparison is carried in
fp64; floating point that *decides an integer* (a 4-bit code, a zero point, an
INT8 activation code) is done in IEEE fp32 exactly as written, because the
CUDA kernels take the same decisions in fp32 and the codes must agree bit for
bit.  Integer work (codes, nibble packing, permutation, the per-group INT8 x
INT4 dot products) is exact.

Sources (cited per function):
  [P2] «Kimi 2.7 Moe 从 4 bit 存储到 INT8 拆解» (pptc.cn/news/121597)
  [P1] Kimi 2.7T MoE W4A8 article (hotelren.com/news/5173946)
  [P3] LLM quantisation primer (hotelren.com/news/5982361)
  [P4] «MoE部署别把激活参数当成存储需求» (feinterview.poetries.top)

Readings taken where the pages are silent or garbled (each one is listed with
its reason in the design notes):
  R1  the integer zero-point form of [P2] §2.2 is used, not the min-offset form of [P1] §2.1;
  R2  the quantisation range is the group's min and max (not a percentile);
  R3  the range is widened to contain 0 (mn = min(v, 0), mx = max(v, 0)); an fp16
      scale that rounds to 0 is replaced by 1;
  R4  every "round" is round-half-to-even;
  R5  codes are computed with the fp16-rounded scale, so the stored scale and zero
      point reproduce them;
  R6  divisions are correctly rounded fp32 divisions (no reciprocal, no FMA);
  R7  activation codes are limited to [-127, 127];
  R9  weights are [N][K] (output channel major), groups of 128 run along K;
  R10 the up projection's rows are [gate (F rows) | up (F rows)];
  R11 softmax routing: top-k experts by logit (ties -> lower id), gate weight = the
      softmax probability over all E experts, not renormalised;
  R12 tokens inside an expert's segment keep their slot order (t * k + j ascending);
  R14 h, the SwiGLU of the up projection's result, is rounded once to bf16 and enters
      the requantisation as that bf16 value ([P1] §4.3 step 4: the GEMM result is
      handed on in FP16/BF16; step 3: the next op quantises it per token);
  R18 symmetric INT4 variant: q clamped to [-7, 7], stored as code q + 8 with zero point 8;
  R19 percentile-clipped variant: per group the 0.1th and 99.9th percentiles by linear
      interpolation at q * (n - 1), in fp32 with fractions fp32(0.127) and fp32(0.873);
  R20 INT8 KV cache: static symmetric per-head scale max|x|/127 over the calibration
      values (0 for an all-zero head, which then quantises to 0); dequantisation rounds
      the fp32 product q * scale once to bf16;
  R21 W4A16 comparison layer: activations unquantised bf16, h rounded to bf16 between
      the projections.

Parity status: every function below is pinned by tests/test_oracle_pins.py
against values the pages print, closed forms, brute force or an independent
formulation; none is "parity unpinned".
"""

from __future__ import annotations

import numpy as np

GROUP = 128  # [P2] §2.1: one scale and one zero point per 128 weights along K
INT4_MAX = 15  # [P2] §2.2: 2^4 - 1
INT8_QMAX = 127  # [P3] §2.1: 2^(b-1) - 1 for b = 8 (symmetric)
INT4_SYM_QMAX = 7  # [P3] §2.1: 2^(b-1) - 1 for b = 4 (symmetric weights)
INT4_SYM_ZP = 8  # the symmetric codes are stored as q + 8


# --------------------------------------------------------------------------- #
# shapes
# --------------------------------------------------------------------------- #
def padded_k(K: int, group: int = GROUP) -> int:
    """K rounded up to a whole number of groups ([P2] §2.1: pad the matrix to a
    multiple of the group size at conversion time)."""
    return ((K + group - 1) // group) * group


def pad_k(a: np.ndarray, group: int = GROUP) -> np.ndarray:
    """Zero-pad the last axis to padded_k ([P2] §2.1)."""
    K = a.shape[-1]
    Kp = padded_k(K, group)
    if Kp == K:
        return a
    pad = [(0, 0)] * (a.ndim - 1) + [(0, Kp - K)]
    return np.pad(a, pad)


# --------------------------------------------------------------------------- #
# a1: weight quantisation and packing  ([P2] §2.1, §2.2)
# --------------------------------------------------------------------------- #
# R19: the 0.1th / 99.9th percentiles of a 128-value group, by linear interpolation
# between order statistics at position q * (n - 1): 0.127 and 126.873
PCT_LO_FRAC = np.float32(0.127)
PCT_HI_FRAC = np.float32(0.873)


def group_range_percentile(v: np.ndarray):
    """Clipped range of each row of v [N][128] (fp32): the 0.1th and 99.9th
    percentiles ([P2] §2.2: a percentile filters outliers better than min/max; R19:
    linear interpolation at position q * (n - 1), evaluated in fp32 as
    a + f * (b - a) with separate roundings)."""
    srt = np.sort(np.asarray(v, dtype=np.float32), axis=1)
    assert srt.shape[1] == GROUP
    lo = srt[:, 0] + PCT_LO_FRAC * (srt[:, 1] - srt[:, 0])
    hi = srt[:, 126] + PCT_HI_FRAC * (srt[:, 127] - srt[:, 126])
    return lo.astype(np.float32), hi.astype(np.float32)


def quantize_weights(w: np.ndarray, clip999: bool = False, group: int = GROUP):
    """Group-wise asymmetric INT4 of one weight matrix w [N][K] (float32, bf16 values).

    [P2] §2.2, per group of 128 along K:
        scale      = (max - min) / (2^4 - 1)
        zero_point = round(-min / scale)
        index      = clamp(round(weight / scale) + zero_point, 0, 15)
    with readings R2-R6 (min/max widened to contain 0; fp16 scale used for the
    codes; round half to even; fp32 correctly rounded division).  With clip999 the
    range is the group's 0.1th..99.9th percentile instead of its min..max ([P2] §2.2,
    R19); values outside it land on codes 0 or 15 through the clamp.  `group` is the
    number of weights per group along K ([P1] §5 names 128 or 256; [P2] §2.1 trades
    accuracy against the scale storage; 128 unless stated).

    Returns codes uint8 [N][Kp] (values 0..15), scale float16 [N][G], zp float16 [N][G].
    """
    assert not clip999 or group == GROUP, "the percentile positions are those of 128-value groups"
    w = pad_k(np.asarray(w, dtype=np.float32), group)
    N, Kp = w.shape
    G = Kp // group
    codes = np.zeros((N, Kp), dtype=np.uint8)
    scale = np.zeros((N, G), dtype=np.float16)
    zp = np.zeros((N, G), dtype=np.float16)
    f15 = np.float32(INT4_MAX)
    for g in range(G):
        v = w[:, g * group:(g + 1) * group]  # [N][group]
        if clip999:
            lo, hi = group_range_percentile(v)
        else:
            lo, hi = v.min(axis=1), v.max(axis=1)
        mn = np.minimum(lo, np.float32(0))  # R3
        mx = np.maximum(hi, np.float32(0))  # R3
        s32 = (mx - mn) / f15  # fp32 division
        s16 = s32.astype(np.float16)  # round to nearest even fp16 (R5)
        s16[s16 == 0] = np.float16(1.0)  # R3: degenerate (all-zero) group
        sf = s16.astype(np.float32)
        # R4, R6; the zero point is an integer index offset, so -0.0 is stored as 0
        z = np.clip(np.rint(-mn / sf), 0, INT4_MAX) + np.float32(0)
        q = np.rint(v / sf[:, None]) + z[:, None]
        codes[:, g * group:(g + 1) * group] = np.clip(q, 0, INT4_MAX).astype(np.uint8)
        scale[:, g] = s16
        zp[:, g] = z.astype(np.float16)
    return codes, scale, zp


def quantize_weights_symmetric(w: np.ndarray, group: int = GROUP):
    """Group-wise symmetric INT4 of one weight matrix w [N][K] (the packer's
    symmetric variant).

    [P3] §2.1, symmetric form with b = 4, per group of 128 along K:
        scale = max|weight| / (2^(4-1) - 1)
        q     = clamp(round(weight / scale), -7, 7)
    stored in the same format as the asymmetric scheme: code = q + 8 with a zero
    point of 8, so (code - zp) * scale reproduces q * scale.  Readings R4-R6 as
    above; R18: the clamp is the formula's own range [-(2^3 - 1), 2^3 - 1]; an fp16
    scale that rounds to 0 is replaced by 1.

    Returns codes uint8 [N][Kp] (values 1..15), scale float16 [N][G], zp float16 [N][G] (all 8).
    """
    w = pad_k(np.asarray(w, dtype=np.float32), group)
    N, Kp = w.shape
    G = Kp // group
    codes = np.zeros((N, Kp), dtype=np.uint8)
    scale = np.zeros((N, G), dtype=np.float16)
    zp = np.full((N, G), INT4_SYM_ZP, dtype=np.float16)
    qmax = np.float32(INT4_SYM_QMAX)
    for g in range(G):
        v = w[:, g * group:(g + 1) * group]  # [N][group]
        amax = np.abs(v).max(axis=1)
        s16 = (amax / qmax).astype(np.float16)  # fp32 division, then fp16 RNE (R5, R6)
        s16[s16 == 0] = np.float16(1.0)
        sf = s16.astype(np.float32)
        q = np.clip(np.rint(v / sf[:, None]), -qmax, qmax)  # R4, R6
        codes[:, g * group:(g + 1) * group] = (q + INT4_SYM_ZP).astype(np.uint8)
        scale[:, g] = s16
    return codes, scale, zp


def dequantize_weights(codes: np.ndarray, scale: np.ndarray, zp: np.ndarray) -> np.ndarray:
    """weight ~= (index - zero_point) * scale  ([P2] §2.1), in fp64, shape [N][Kp]
    (the group size is Kp / G)."""
    group = codes.shape[1] // scale.shape[1]
    sc = np.repeat(scale.astype(np.float64), group, axis=1)
    z = np.repeat(zp.astype(np.float64), group, axis=1)
    return (codes.astype(np.float64) - z) * sc


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """Two 4-bit codes per byte, the first in the low 4 bits and the second in the
    high 4 bits ([P2] §2.2).  codes [..., Kp] -> bytes [..., Kp/2]."""
    c = np.asarray(codes, dtype=np.uint8)
    first = c[..., 0::2]
    second = c[..., 1::2]
    return (first | (second << 4)).astype(np.uint8)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    """Inverse of pack_nibbles."""
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 0x0F
    out[..., 1::2] = p >> 4
    return out


# --------------------------------------------------------------------------- #
# a2 / a6: per-token symmetric INT8 ([P3] §2.1, [P1] §4.3 step 3)
# --------------------------------------------------------------------------- #
def quantize_act(x: np.ndarray, group: int = GROUP):
    """Dynamic per-token symmetric INT8 of x [T][K] (fp32 values).

    [P3] §2.1 symmetric form: scale = max|x| / (2^(b-1) - 1), q = round(x / scale),
    computed per token at run time ([P1] §4.3).  fp32 arithmetic, round half to even,
    codes clamped to [-127, 127] (R7).  A row of zeros gets scale 0 and codes 0.

    Returns q int8 [T][Kp] (zero padded to a whole number of weight groups) and
    s float32 [T].
    """
    x = np.asarray(x, dtype=np.float32)
    T = x.shape[0]
    amax = np.abs(x).max(axis=1) if x.shape[1] else np.zeros(T, np.float32)
    s = (amax / np.float32(INT8_QMAX)).astype(np.float32)
    q = np.zeros(x.shape, dtype=np.int8)
    nz = s > 0
    if nz.any():
        r = np.rint(x[nz] / s[nz][:, None])
        q[nz] = np.clip(r, -INT8_QMAX, INT8_QMAX).astype(np.int8)
    return pad_k(q, group), s


# --------------------------------------------------------------------------- #
# a3: routing ([P1] §5.2: the router stays in 16-bit float, never quantised)
# --------------------------------------------------------------------------- #
def route_topk(logits: np.ndarray, k: int):
    """Top-k softmax gating (R11).

    Expert choice: the k largest logits per token, ties broken towards the lower
    expert id (a stable sort) -- the same set as the k largest softmax probabilities.
    Gate weight: softmax over all E experts (fp64), not renormalised over the k.
    Returns ids int32 [T][k], w float64 [T][k].
    """
    lg = np.asarray(logits, dtype=np.float64)
    T, E = lg.shape
    ids = np.zeros((T, k), dtype=np.int32)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-lg[t, e], e))
        ids[t] = order[:k]
    p = np.exp(lg - lg.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    w = np.take_along_axis(p, ids.astype(np.int64), axis=1)
    return ids, w


# --------------------------------------------------------------------------- #
# a4: permutation (grouping tokens by expert)
# --------------------------------------------------------------------------- #
def permute(ids: np.ndarray, E: int):
    """Stable grouping of the T*k routed slots by expert (R12).

    Slot i = t*k + j carries expert ids[t, j].  counts[e] = number of slots routed
    to e; offs = exclusive prefix sum of counts (length E+1); perm[offs[e] + p] = the
    p-th slot (in ascending slot order) routed to e; inv[i] = position of slot i in
    the grouped order.
    """
    flat = np.asarray(ids, dtype=np.int64).reshape(-1)
    counts = np.zeros(E, dtype=np.int64)
    for e in flat:
        counts[e] += 1
    offs = np.zeros(E + 1, dtype=np.int64)
    for e in range(E):
        offs[e + 1] = offs[e] + counts[e]
    fill = offs[:-1].copy()
    perm = np.zeros(flat.size, dtype=np.int64)
    inv = np.zeros(flat.size, dtype=np.int64)
    for i, e in enumerate(flat):
        perm[fill[e]] = i
        inv[i] = fill[e]
        fill[e] += 1
    return counts, offs, perm, inv


def expected_distinct_experts(E: int, B: int) -> float:
    """Mean number of distinct experts hit by B tokens that each pick one of E
    experts independently and uniformly: E * (1 - (1 - 1/E)^B)  ([P4], toy model)."""
    return E * (1.0 - (1.0 - 1.0 / E) ** B)


# --------------------------------------------------------------------------- #
# a5 / a7: W4A8 linear with per-group INT32 partials ([P2] §3.2, [P1] §4.3)
# --------------------------------------------------------------------------- #
def group_partials(qa: np.ndarray, codes: np.ndarray, zp: np.ndarray) -> np.ndarray:
    """acc[m, n, g] = sum over k in group g of qa[m, k] * (codes[n, k] - zp[n, g]).

    INT8 activations times INT4 weights dequantised to integers, accumulated in
    32 bits per group ([P2] §3.2: INT8 x INT8 accumulates into INT32).  Computed
    per group with an fp64 matrix product, which is exact here because every
    partial is an integer of magnitude <= 128 * 127 * 15 < 2^53.
    Returns int64 [M][N][G].
    """
    qa = np.asarray(qa)
    M, Kp = qa.shape
    N = codes.shape[0]
    G = zp.shape[1]
    group = Kp // G  # 128 unless the weights were quantised with another group size
    assert group * G == Kp and codes.shape[1] == Kp
    acc = np.zeros((M, N, G), dtype=np.int64)
    for g in range(G):
        sl = slice(g * group, (g + 1) * group)
        a = qa[:, sl].astype(np.float64)  # [M][group]
        wq = codes[:, sl].astype(np.float64) - zp[:, g].astype(np.float64)[:, None]  # [N][group]
        acc[:, :, g] = np.rint(a @ wq.T).astype(np.int64)
    return acc


def w4a8_linear(qa, sa, codes, scale, zp, acc=None) -> np.ndarray:
    """y[m, n] = sa[m] * sum_g scale[n, g] * acc[m, n, g]   (fp64).

    [P1] §4.3 steps 2-4: INT8 matrix product, then the INT32 result is scaled back
    to floating point -- the weight scale of each group times the token's scale.
    """
    if acc is None:
        acc = group_partials(qa, codes, zp)
    y = np.zeros(acc.shape[:2], dtype=np.float64)
    for g in range(acc.shape[2]):
        y += scale[:, g].astype(np.float64)[None, :] * acc[:, :, g].astype(np.float64)
    return np.asarray(sa, dtype=np.float64)[:, None] * y


# --------------------------------------------------------------------------- #
# a6: SwiGLU between the projections
# --------------------------------------------------------------------------- #
def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def swiglu(y_up: np.ndarray, F: int) -> np.ndarray:
    """h = silu(gate) * up with gate = columns [0, F) and up = columns [F, 2F) (R10)."""
    return silu(y_up[:, :F]) * y_up[:, F:2 * F]


# --------------------------------------------------------------------------- #
# a8: weighted combine
# --------------------------------------------------------------------------- #
def combine(y2: np.ndarray, w: np.ndarray, inv: np.ndarray, T: int, k: int) -> np.ndarray:
    """out[t] = sum over j < k of w[t, j] * y2[inv[t*k + j]]  (fp64, j ascending)."""
    out = np.zeros((T, y2.shape[1]), dtype=np.float64)
    for j in range(k):
        out += np.asarray(w, dtype=np.float64)[:, j:j + 1] * y2[inv[np.arange(T) * k + j]]
    return out


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to the nearest bf16 (ties to even), returned as fp64.

    [P1] §4.3 step 4: the result is converted back to 16-bit float (BF16) for the
    layers that follow.  bf16 keeps 8 significant bits; the fp64 mantissa is cut to
    its top 7 stored bits with round-half-to-even on the integer bit pattern, a
    single correctly rounded step for every normal value (the layer's outputs are
    far from the bf16 subnormal and overflow ranges).
    """
    b = np.ascontiguousarray(x, dtype=np.float64).view(np.uint64)
    drop = np.uint64(52 - 7)
    half = np.uint64(1) << (drop - np.uint64(1))
    lsb = (b >> drop) & np.uint64(1)
    r = (b + (half - np.uint64(1)) + lsb) & ~((np.uint64(1) << drop) - np.uint64(1))
    return r.view(np.float64)


# --------------------------------------------------------------------------- #
# the whole layer
# --------------------------------------------------------------------------- #
class QuantExpert:
    """Quantised weights of one expert: up [2F][Hp] (gate|up rows) and down [H][Fp]
    (asymmetric INT4, or the symmetric variant), `group` weights per scale along K."""

    def __init__(self, w_up: np.ndarray, w_down: np.ndarray, symmetric: bool = False, clip999: bool = False,
                 group: int = GROUP):
        self.group = group
        if symmetric:
            def quant(w):
                return quantize_weights_symmetric(w, group)
        else:
            def quant(w):
                return quantize_weights(w, clip999, group)
        self.up = quant(w_up)
        self.down = quant(w_down)


def expert_forward(xq, xs, qe: QuantExpert, F: int, stages: dict | None = None):
    """One expert on its tokens: up GEMM -> SwiGLU (rounded to bf16, R14) ->
    requantise -> down GEMM.

    xq int8 [M][Hp], xs float32 [M]; returns y2 float64 [M][H].
    """
    cu, su, zu = qe.up
    y_up = w4a8_linear(xq, xs, cu, su, zu)  # [M][2F]
    h = round_to_bf16(swiglu(y_up, F)).astype(np.float32)  # R14: h is handed on in bf16
    qh, sh = quantize_act(h, qe.group)  # [P1] §4.3 step 3: the next op's input is quantised per token
    cd, sd, zd = qe.down
    y2 = w4a8_linear(qh, sh, cd, sd, zd)
    if stages is not None:
        stages.setdefault("h", []).append(h)
        stages.setdefault("qh", []).append(qh)
        stages.setdefault("sh", []).append(sh)
    return y2


def moe_forward(x, ids, w, experts: dict, E: int, F: int, stages: dict | None = None):
    """Full W4A8 MoE expert FFN, [T][H]: the fp64 sum of a8 rounded to bf16
    ([P1] §4.3 step 4), returned as fp64 values.

    x [T][H] float32 (bf16 values); ids [T][k]; w [T][k]; experts[e] = QuantExpert
    (only experts that receive tokens are needed).
    """
    x = np.asarray(x, dtype=np.float32)
    T, H = x.shape
    k = ids.shape[1]
    group = next(iter(experts.values())).group if experts else GROUP
    xq, xs = quantize_act(x, group)
    counts, offs, perm, inv = permute(ids, E)
    y2 = np.zeros((T * k, H), dtype=np.float64)
    for e in range(E):
        if counts[e] == 0:
            continue
        slots = perm[offs[e]:offs[e + 1]]
        tok = slots // k
        y2[offs[e]:offs[e + 1]] = expert_forward(xq[tok], xs[tok], experts[e], F, stages)[:, :H]
    if stages is not None:
        stages.update(counts=counts, offs=offs, perm=perm, inv=inv, xq=xq, xs=xs, y2=y2)
    return round_to_bf16(combine(y2, w, inv, T, k))


def token_forward(t: int, x, ids, w, experts: dict, F: int) -> np.ndarray:
    """The layer's output (bf16-rounded) for one token only (used to sample large layers)."""
    group = experts[int(ids[t, 0])].group
    xq, xs = quantize_act(np.asarray(x, dtype=np.float32)[t:t + 1], group)
    out = 0.0
    for j in range(ids.shape[1]):
        y2 = expert_forward(xq, xs, experts[int(ids[t, j])], F)[0]
        out = out + float(w[t, j]) * y2
    return round_to_bf16(out)


# --------------------------------------------------------------------------- #
# INT8 KV cache with static per-head scales (the next W4A8 deployment step)
# --------------------------------------------------------------------------- #
def kv_calibrate(x: np.ndarray) -> np.ndarray:
    """Static per-head scales of a KV cache from calibration data x [T][H][D] (fp32,
    bf16 values).

    [P1] §5 (deployment): the attention KV cache is quantised to INT8 statically,
    with per-head scales fixed from a little calibration data; [P3] §2.1 symmetric
    form: scale = max|x| / 127 over the head's calibration values (fp32 division).
    A head whose calibration values are all zero gets scale 0 (R20).
    """
    x = np.asarray(x, dtype=np.float32)
    amax = np.abs(x).max(axis=(0, 2)) if x.shape[0] else np.zeros(x.shape[1], np.float32)
    return (amax.astype(np.float32) / np.float32(INT8_QMAX)).astype(np.float32)


def kv_quantize(x: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """q[t, h, d] = clamp(round(x / scale[h]), -127, 127), fp32 division, round half to
    even (R4, R6, R7); values beyond the calibrated range saturate; scale 0 -> q = 0."""
    x = np.asarray(x, dtype=np.float32)
    s = np.asarray(scale, dtype=np.float32)[None, :, None]
    safe = np.where(s > 0, s, np.float32(1))
    q = np.clip(np.rint(x / safe), -INT8_QMAX, INT8_QMAX)
    return np.where(s > 0, q, 0).astype(np.int8)


def kv_dequantize(q: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """x'[t, h, d] = bf16(q * scale[h]): the fp32 product rounded once to bf16 (RNE),
    returned as float32 values (R20)."""
    y = np.asarray(q, dtype=np.float32) * np.asarray(scale, dtype=np.float32)[None, :, None]
    return round_to_bf16(y.astype(np.float64)).astype(np.float32)


# --------------------------------------------------------------------------- #
# W4A16: the same INT4 weights with 16-bit activations (the comparison point)
# --------------------------------------------------------------------------- #
def w4a16_linear(x, codes, scale, zp) -> np.ndarray:
    """y[m, n] = sum_k x[m, k] * (code[n, k] - zp[n, g(k)]) * scale[n, g(k)]  (fp64).

    [P2] §1 and §3.3: W4A16 keeps the 4-bit weights but multiplies with 16-bit
    activations (no activation quantisation); x [M][K] holds bf16 values.
    """
    x = pad_k(np.asarray(x, dtype=np.float32)).astype(np.float64)
    return x @ dequantize_weights(codes, scale, zp).T


def w4a16_expert_forward(x, qe: QuantExpert, F: int) -> np.ndarray:
    """One expert with 16-bit activations: up GEMM -> SwiGLU -> h rounded to bf16
    (R21: the activations between the projections stay 16-bit) -> down GEMM."""
    h = round_to_bf16(swiglu(w4a16_linear(x, *qe.up), F))
    return w4a16_linear(h, *qe.down)


def moe_forward_w4a16(x, ids, w, experts: dict, E: int, F: int):
    """The MoE expert FFN with W4A16 experts (same routing, permutation and combine
    as moe_forward), output rounded to bf16."""
    x = np.asarray(x, dtype=np.float32)
    T, H = x.shape
    k = ids.shape[1]
    counts, offs, perm, inv = permute(ids, E)
    y2 = np.zeros((T * k, H), dtype=np.float64)
    for e in range(E):
        if counts[e] == 0:
            continue
        tok = perm[offs[e]:offs[e + 1]] // k
        y2[offs[e]:offs[e + 1]] = w4a16_expert_forward(x[tok], experts[e], F)[:, :H]
    return round_to_bf16(combine(y2, w, inv, T, k))
