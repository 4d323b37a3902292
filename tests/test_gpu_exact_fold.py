"""Bit-exact INT32 partials through the kernel instances the layer actually runs.

The dense entry point can write the per-group INT32 partials, but when it does it
runs a separate instance of the wide-tile kernel; the MoE layer and a call without
a partials buffer run the production instance, whose epilogue keeps the partials in
registers and only emits y = sa * sum_g scale[n, g] * P[m, n, g].

These tests make that output itself a bit-exact image of the partials.  Every
weight group spans exactly [-8, 7] * 2^-6, so by the formulas of «Kimi 2.7 Moe 从 4
bit 存储到 INT8 拆解» (pptc.cn), section 2.2, its fp16 scale is exactly 2^-6 and its
zero point exactly 8.  Then every term scale * P is an
integer multiple of 2^-6 below 2^24 * 2^-6 (at most 64 groups of |P| <= 243840), so
the fp32 fold is exact in any order, and y = RN_fp32(sa * S) with the exact sum S.
The oracle's fp64 result of the same product is exact too, so fp32(oracle) must
equal the kernel's y bit for bit; any wrong, dropped or duplicated partial shows.
"""

import numpy as np
import pytest
import torch

from helpers import untile_act
from oracle import w4a8_oracle as O
from w4a8_quantized_moe_token_b200 import binding as B
from w4a8_quantized_moe_token_b200 import synth

pytestmark = pytest.mark.gpu

STEP = 2.0 ** -6  # the weight scale every group gets


def exact_scale_weights(seed, N, K):
    """[N][K] weights on the grid {-8..7} * 2^-6, every 128-group (the valid part of
    a ragged last group included) holding both -8 and 7 at seeded positions."""
    rng = np.random.default_rng([seed, N, K])
    lv = rng.integers(-8, 8, size=(N, K))
    rows = np.arange(N)
    for k0 in range(0, K, 128):
        n = min(K, k0 + 128) - k0
        pick = np.argsort(rng.random((N, n)), axis=1)[:, :2]  # two distinct positions per row
        lv[rows, k0 + pick[:, 0]] = -8
        lv[rows, k0 + pick[:, 1]] = 7
    return (lv * STEP).astype(np.float32)


def check_exact_scale(codes, scale, zp):
    assert np.all(scale.astype(np.float32) == np.float32(STEP)), "every group must get scale 2^-6"
    assert np.all(zp.astype(np.float32) == 8.0), "every group must get zero point 8"


def to_dev_bf16(a):
    a = np.ascontiguousarray(a, dtype=np.float32)
    assert np.array_equal(synth.bf16_round(a), a)
    return torch.from_numpy(synth.bf16_bits(a).view(np.int16)).view(torch.bfloat16).cuda()


@pytest.mark.parametrize("M,N,K", [(300, 256, 640), (129, 384, 200), (17, 128, 1024), (16, 256, 512), (5, 128, 8192),
                                   (40, 130, 256),  # N % 4 != 0: rows not 16-byte aligned, direct stores
                                   (5, 20480, 1024), (16, 38400, 2048)])  # more tiles than CTAs
def test_dense_gemm_without_partials_is_bit_exact(M, N, K):
    """M > 16: the wide-tile production instance (no partials buffer); M <= 16: the
    decode-tile kernel.  K = 8192 is the largest K (64 groups) for which the exact
    fold argument holds.  With 160 or 300 column tiles every CTA of the decode kernel
    takes several tiles, so its pipeline rings wrap across tile boundaries."""
    x = synth.activations(M * 7 + K, M, K)
    qa, sa = O.quantize_act(x)
    w = exact_scale_weights(M + N + K, N, K)
    codes, scale, zp = O.quantize_weights(w)
    check_exact_scale(codes, scale, zp)
    packed = B.empty_aligned(B.w4a8_packed_bytes(1, N, K, 0))
    B.w4a8_pack_weights(to_dev_bf16(w), 0, packed)
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    ws = B.empty_aligned(B.w4a8_gemm_workspace_bytes(M, N, K))
    B.w4a8_gemm(torch.from_numpy(qa).cuda(), torch.from_numpy(sa).cuda(), packed, N, K, y, ws)
    torch.cuda.synchronize()
    assert B.w4a8_last_device_error(ws) == 0
    ref = O.w4a8_linear(qa, sa, codes, scale, zp).astype(np.float32)
    got = y.cpu().numpy()
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32)), \
        f"{int((got != ref).sum())} of {got.size} outputs differ"


@pytest.mark.parametrize("T,E,k,H,F,routing", [
    (600, 4, 2, 512, 384, "uniform"),  # wide tiles, ragged last row tile of each expert
    (4096, 8, 1, 2048, 1024, "uniform"),  # the toy layer's shape
    (48, 8, 2, 256, 640, "zipf"),  # decode tiles (<= 16 tokens per expert on average)
])
def test_moe_down_projection_is_bit_exact(T, E, k, H, F, routing):
    """The down projection (the production GEMM instance in its plain-output mode)
    inside w4a8_moe_forward: on the requantised h that the layer itself produced,
    y2 must equal the oracle's fp32-rounded result bit for bit."""
    x = synth.activations(T + 11, T, H)
    ids, wts = synth.synthetic_routing(T + 5, T, E, k, routing, 1.1)
    up = B.empty_aligned(B.w4a8_packed_bytes(E, 2 * F, H, B.W4A8_LAYOUT_GATEUP))
    dn = B.empty_aligned(B.w4a8_packed_bytes(E, H, F, B.W4A8_LAYOUT_PLAIN))
    wu = np.stack([synth.expert_weight(T, e, "up", 2 * F, H) for e in range(E)])
    wd = np.stack([exact_scale_weights(1000 + e, H, F) for e in range(E)])
    B.w4a8_pack_weights(to_dev_bf16(wu), B.W4A8_LAYOUT_GATEUP, up)
    B.w4a8_pack_weights(to_dev_bf16(wd), B.W4A8_LAYOUT_PLAIN, dn)
    ws = B.empty_aligned(B.w4a8_moe_workspace_bytes(T, E, k, H, F))
    out = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    B.w4a8_moe_forward(up, dn, E, H, F, to_dev_bf16(x), torch.from_numpy(ids).cuda(),
                       torch.from_numpy(wts).cuda(), out, ws)
    torch.cuda.synchronize()
    assert B.w4a8_last_device_error(ws) == 0

    def dump(what, dt):
        return B.w4a8_debug_dump(ws, T, E, k, H, F, what).cpu().numpy().view(dt)

    R = B.w4a8_moe_rows_capacity(T, E, k)
    RB = B.w4a8_moe_act_block_rows(T, E, k)
    Fp = O.padded_k(F)
    rows = dump("inv", np.int32)
    act2 = untile_act(dump("act2", np.int8), R, Fp, RB)[rows]
    s2 = dump("s2", np.float32)[rows]
    y2 = dump("y2", np.float32).reshape(R, H)[rows]
    flat = ids.reshape(-1)
    ref = np.zeros((T * k, H), np.float32)
    for e in range(E):
        sel = np.nonzero(flat == e)[0]
        if sel.size:
            codes, scale, zp = O.quantize_weights(wd[e])
            check_exact_scale(codes, scale, zp)
            ref[sel] = O.w4a8_linear(act2[sel], s2[sel], codes, scale, zp).astype(np.float32)
    assert np.array_equal(y2.view(np.uint32), ref.view(np.uint32)), \
        f"{int((y2 != ref).sum())} of {y2.size} values of y2 differ"
