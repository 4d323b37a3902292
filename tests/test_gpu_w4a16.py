"""GPU parity of the W4A16 comparison path against the CPU oracle.

W4A16 multiplies the same packed INT4 weights with bf16 activations that are not
quantised («Kimi 2.7 Moe 从 4 bit 存储到 INT8 拆解», pptc.cn, sections 1 and 3.3).  The
kernel forms (code - zp) as bf16 exactly and sums one fp32 partial per K group on the
tensor core, so its GEMM result differs from the oracle's fp64 one only by fp32
rounding, bounded in helpers.w4a16_error_bound; the tests hold it to that bound on
identical inputs, stage by stage, and hold the final bf16 output to the layer's
tolerance (max relative error 1e-2, mean absolute error <= 1e-3 * rms).
"""

import numpy as np
import pytest
import torch

from helpers import assert_bf16_adjacent, assert_close, untile_act16, w4a16_error_bound
from oracle import w4a8_oracle as O
from test_gpu_moe import Layer, bf16_to_f32, dev_bf16
from w4a8_quantized_moe_token_b200 import binding as B
from w4a8_quantized_moe_token_b200 import synth

pytestmark = pytest.mark.gpu


def assert_within_bound(got, ref, bound, what):
    err = np.abs(np.asarray(got, dtype=np.float64) - ref)
    bad = err > bound
    assert not bad.any(), f"{what}: {int(bad.sum())} of {err.size} outside the fp32 bound " \
                          f"(worst {float((err - bound).max()):.3e} over)"


@pytest.mark.parametrize("M,N,K", [(1, 128, 128), (16, 256, 512), (17, 384, 200), (40, 130, 1024),
                                   (5, 256, 7168), (100, 128, 384)])
def test_w4a16_gemm_within_fp32_bound(M, N, K):
    x = synth.activations(M + N + K, M, K)
    w = synth.dense_gemm_inputs(M, M, K, N)[1]
    codes, scale, zp = O.quantize_weights(w)
    packed = B.empty_aligned(B.w4a8_packed_bytes(1, N, K, 0))
    B.w4a8_pack_weights(dev_bf16(w), 0, packed)
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    ws = B.empty_aligned(B.w4a16_gemm_workspace_bytes(M, N, K))
    B.w4a16_gemm(dev_bf16(x), packed, N, K, y, ws)
    torch.cuda.synchronize()
    assert B.w4a8_last_device_error(ws) == 0
    xb = synth.bf16_round(x)
    ref = O.w4a16_linear(xb, codes, scale, zp)
    assert_within_bound(y.cpu().numpy(), ref, w4a16_error_bound(xb, codes, scale, zp), "y")


def run_w4a16(L: Layer):
    T, E, k, H, F = L.T, L.E, L.k, L.H, L.F
    ws = B.empty_aligned(B.w4a16_moe_workspace_bytes(T, E, k, H, F))
    out = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    B.w4a16_moe_forward(L.packed_up, L.packed_down, E, H, F, dev_bf16(L.x), torch.from_numpy(L.ids).cuda(),
                        torch.from_numpy(L.w.astype(np.float32)).cuda(), out, ws)
    torch.cuda.synchronize()
    assert B.w4a8_last_device_error(ws) == 0
    return bf16_to_f32(out), ws


LAYERS = [
    # T, E, k, H, F, routing
    (1, 4, 2, 256, 128, "uniform"),
    (37, 5, 3, 200, 100, "uniform"),   # K and F off the 128 grid, F % 8 != 0
    (48, 16, 4, 1024, 640, "zipf"),    # hot experts span several 16-token tiles
    (64, 64, 6, 512, 352, "softmax"),  # decode-shaped routing from router logits
]


@pytest.mark.parametrize("T,E,k,H,F,routing", LAYERS)
def test_w4a16_moe_stages_and_output(T, E, k, H, F, routing):
    L = Layer(T, E, k, H, F, routing, seed=3 * T + E)
    out, ws = run_w4a16(L)
    Hp, Fp = O.padded_k(H), O.padded_k(F)
    R = B.w4a8_moe_rows_capacity(T, E, k)

    def dump(what, dt):
        return B.w4a8_debug_dump(ws, T, E, k, H, F, B.DUMP[what] | B.W4A8_DUMP_W4A16).cpu().numpy().view(dt)

    counts, offs, perm, inv = O.permute(L.ids, E)
    assert np.array_equal(dump("perm", np.int32), perm)
    rows = dump("inv", np.int32)
    tok = np.arange(T * k) // k
    # the token rows: the bf16 bits of x, pad columns zero
    x16 = untile_act16(dump("act1", np.uint8), R, Hp)[rows]
    xbits = synth.bf16_bits(L.x)
    assert np.array_equal(x16[:, :H], xbits[tok])
    assert not x16[:, H:].any()
    # up GEMM + SwiGLU -> bf16 h, on identical inputs
    experts = L.experts()
    xb = synth.bf16_round(L.x)
    h16 = untile_act16(dump("act2", np.uint8), R, Fp)[rows]
    assert not h16[:, F:].any(), "pad columns of h must be zero"
    h = synth.bf16_from_bits(h16[:, :F])
    h_ref = np.zeros((T * k, F))
    for e, qe in experts.items():
        sl = perm[offs[e]:offs[e + 1]]
        if sl.size:
            h_ref[sl] = O.round_to_bf16(O.swiglu(O.w4a16_linear(xb[sl // k], *qe.up), F))
    # one bf16 rounding of h on either side: equal or one bf16 step apart
    assert_bf16_adjacent(h, h_ref, what="h")
    # down GEMM on the dumped h
    y2 = dump("y2", np.float32).reshape(R, H)[rows]
    for e, qe in experts.items():
        sl = perm[offs[e]:offs[e + 1]]
        if sl.size:
            ref = O.w4a16_linear(h[sl], *qe.down)
            assert_within_bound(y2[sl], ref, w4a16_error_bound(h[sl], *qe.down), f"y2 of expert {e}")
    # the whole layer
    ref = O.moe_forward_w4a16(L.x, L.ids, L.w, experts, E, F)
    assert_close(out, ref, what="out")


def test_w4a16_decode_config_output_on_sampled_tokens():
    """The decode layer's shape (64 experts, top-6 from router logits, 64 tokens,
    hidden 4096, expert ffn 1408, 0.1% outlier channels x20), output on a token sample."""
    T, E, k, H, F = 64, 64, 6, 4096, 1408
    L = Layer(T, E, k, H, F, "softmax", seed=11, outlier=0.001)
    out, _ = run_w4a16(L)
    experts = L.experts()
    for t in (0, 17, 63):
        ref = O.moe_forward_w4a16(L.x[t:t + 1], L.ids[t:t + 1], L.w[t:t + 1], experts, E, F)
        assert_close(out[t:t + 1], ref, what=f"token {t}")
