"""Test-side helpers: tolerance checks and decoders of the library's tiled layouts.

The decoders restate the layouts documented in include/w4a8.h so that tests can
compare device buffers with the oracle's canonical arrays; they take no part in
the product path.
"""

from __future__ import annotations

import numpy as np

BLOCK = 8704
HEADER = 256


def rms(a) -> float:
    a = np.asarray(a, dtype=np.float64)
    return float(np.sqrt(np.mean(a * a))) if a.size else 0.0


def assert_close(gpu, ref, max_rel=1e-2, mae_rel=1e-3, what="output"):
    """Tolerance of the float results against the oracle.

    max relative error <= max_rel, where the relative error of an element is
    |gpu - ref| / max(|ref|, rms(ref)) (elements far below the output's rms are
    judged against the rms), and mean absolute error <= mae_rel * rms(ref).
    """
    g = np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    if r.size == 0:
        return
    s = rms(r)
    err = np.abs(g - r)
    assert np.all(np.isfinite(g)), f"{what}: non-finite values"
    denom = np.maximum(np.abs(r), s if s > 0 else 1.0)
    worst = float((err / denom).max())
    mae = float(err.mean())
    assert worst <= max_rel, f"{what}: max relative error {worst:.3e} > {max_rel}"
    assert mae <= mae_rel * max(s, 1e-30), f"{what}: mean abs error {mae:.3e} > {mae_rel} * rms {s:.3e}"
    return worst, mae


def packed_tiles(N: int, layout: int) -> int:
    return -(-(N // 2) // 64) if layout == 1 else -(-N // 128)


def decode_packed(buf: np.ndarray, E: int, N: int, K: int, layout: int, group: int = 128):
    """Tiled packed buffer -> (codes uint8 [E][N][Kp], scale f16 [E][N][Gq], zp f16 [E][N][Gq]).

    One block per 128-wide plane: codes, then per row the fp16 scale and zero point of
    the plane's group (group 64: of its two groups, the second pair 512 bytes after
    the first; group 256: both planes of a group carry the pair, checked equal)."""
    m = max(128, group)
    Kp = -(-K // m) * m
    G = Kp // 128
    Gq = Kp // group
    blk_bytes = BLOCK + 512 if group == 64 else BLOCK
    NT = packed_tiles(N, layout)
    blocks = np.asarray(buf, dtype=np.uint8)[HEADER:HEADER + E * NT * G * blk_bytes].reshape(E, NT, G, blk_bytes)
    codes = np.zeros((E, N, Kp), np.uint8)
    scale = np.zeros((E, N, Gq), np.float16)
    zp = np.zeros((E, N, Gq), np.float16)
    r = np.arange(128)
    if layout == 1:
        F = N // 2
    for t in range(NT):
        if layout == 1:
            f = t * 64 + (r >> 1)
            src = np.where(r & 1, F + f, f)
            valid = f < F
        else:
            src = t * 128 + r
            valid = src < N
        for g in range(G):
            blk = blocks[:, t, g]  # [E][BLOCK]
            rows = np.zeros((E, 128, 128), np.uint8)
            for c in range(4):
                pos = r * 64 + ((c ^ (r >> 1)) & 3) * 16
                chunk = blk[:, pos[:, None] + np.arange(16)[None, :]]  # [E][128][16]
                words = chunk.reshape(E, 128, 4, 4).astype(np.uint32)
                words = words[..., 0] | (words[..., 1] << 8) | (words[..., 2] << 16) | (words[..., 3] << 24)
                for q in range(4):
                    i = 4 * c + q
                    x = words[:, :, q]
                    for b in range(4):
                        rows[:, :, 8 * i + b] = (x >> (8 * b)) & 0xF
                        rows[:, :, 8 * i + 4 + b] = (x >> (8 * b + 4)) & 0xF
            codes[:, src[valid], g * 128:(g + 1) * 128] = rows[:, valid]
            for sub in range(2 if group == 64 else 1):
                o = 8192 + 512 * sub
                sc = blk[:, o:o + 256].copy().view(np.float16).reshape(E, 128)
                z = blk[:, o + 256:o + 512].copy().view(np.float16).reshape(E, 128)
                q = g * 128 // group + sub
                if group == 256 and g % 2 == 1:  # the group's second plane repeats its pair
                    assert np.array_equal(sc[:, valid].view(np.uint16), scale[:, src[valid], q].view(np.uint16))
                    assert np.array_equal(z[:, valid].view(np.uint16), zp[:, src[valid], q].view(np.uint16))
                    continue
                scale[:, src[valid], q] = sc[:, valid]
                zp[:, src[valid], q] = z[:, valid]
    return codes, scale, zp


def untile_act(buf: np.ndarray, R: int, Kp: int, RB: int | None = None) -> np.ndarray:
    """Tiled INT8 rows [R/RB][Kp/128][RB][128] (16-byte chunk c of row i of a block at
    chunk position c ^ (i & 7)) -> [R][Kp].  RB defaults to R (plain planes)."""
    RB = R if RB is None else RB
    G = Kp // 128
    p = np.asarray(buf).reshape(R // RB, G, RB, 8, 16)
    out = np.zeros((R, Kp), dtype=p.dtype)
    i = np.arange(RB)
    for c in range(8):
        phys = c ^ (i & 7)
        for g in range(G):
            out.reshape(R // RB, RB, Kp)[:, :, g * 128 + c * 16:g * 128 + (c + 1) * 16] = p[:, g, i, phys]
    return out


def untile_act16(buf: np.ndarray, R: int, Kp: int, RB: int = 16) -> np.ndarray:
    """Tiled bf16 rows [R/RB][Kp/128][2][RB][128 bytes] (the two 64-column halves of a
    K group one after the other, 16-byte chunk c of row i at chunk position c ^ (i & 7))
    -> uint16 bf16 bits [R][Kp]."""
    G = Kp // 128
    p = np.asarray(buf, dtype=np.uint8)[:R * G * 256].reshape(R // RB, G, 2, RB, 8, 16)
    out = np.zeros((R // RB, RB, Kp * 2), dtype=np.uint8)
    i = np.arange(RB)
    for g in range(G):
        for hh in range(2):
            for c in range(8):
                b0 = g * 256 + hh * 128 + c * 16
                out[:, :, b0:b0 + 16] = p[:, g, hh, i, c ^ (i & 7)]
    return out.reshape(R, Kp * 2).view(np.uint16)


def w4a16_error_bound(x, codes, scale, zp) -> np.ndarray:
    """Largest error of the fp32 W4A16 GEMM against the exact result, per output.

    Every product x * (code - zp) is exact in fp32 (8-bit by 5-bit significands), a
    group's 128 products are summed in fp32 (at most 127 additions), the partial is
    scaled (one rounding) and the G scaled partials are added (G roundings); with at
    most 2^-23 relative error per operation (a truncating adder included) the error
    is below (127 + G + 1) * 2^-23 * sum_k |x_k| * |w_k|."""
    x = np.abs(np.asarray(x, dtype=np.float64))
    G = scale.shape[1]
    group = codes.shape[1] // G
    Kp = codes.shape[1]
    if x.shape[1] < Kp:
        x = np.pad(x, ((0, 0), (0, Kp - x.shape[1])))
    wabs = np.abs(codes.astype(np.float64) - np.repeat(zp.astype(np.float64), group, axis=1)) * \
        np.repeat(scale.astype(np.float64), group, axis=1)
    return (group - 1 + G + 1) * 2.0 ** -23 * (x @ wabs.T)


def bf16_ulp(v) -> np.ndarray:
    """The spacing of bf16 values at |v| (8 significant bits): 2^(e - 7) for |v| in
    [2^e, 2^(e+1)); the smallest normal spacing for 0 and subnormals."""
    a = np.abs(np.asarray(v, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def assert_bf16_adjacent(got, ref, what="value", max_frac=0.02):
    """got: the kernel's bf16 values; ref: the oracle's bf16-rounded values of the same
    quantity.  Both round a value computed on identical inputs (the kernel in fp32,
    the oracle in fp64, about 1e-6 apart), so they are equal or, where that value
    lies next to a bf16 rounding boundary, one bf16 step apart; at most max_frac of
    the elements may differ."""
    g = np.asarray(got, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    if r.size == 0:
        return
    assert np.all(np.isfinite(g)), f"{what}: non-finite values"
    d = np.abs(g - r)
    step = np.maximum(bf16_ulp(r), bf16_ulp(g))
    assert np.all(d <= step * (1 + 1e-9)), f"{what}: {int((d > step).sum())} values more than one bf16 step off"
    frac = float((d > 0).mean())
    assert frac <= max_frac, f"{what}: {frac:.3%} of the values differ (> {max_frac:.1%})"
