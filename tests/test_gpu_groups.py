"""Group sizes 64 and 256 on the GPU: packer, both GEMM kernels and the layer.

«Kimi 2.7 Moe 从 4 bit 存储到 INT8 拆解» (pptc.cn), section 4.3, tried groups of 64,
128 and 256 weights; the Kimi 2.7T MoE W4A8 article (hotelren.com 5173946), section 5,
names 128 or 256.  With another group size the codes, scales and zero points must
still be bit-exact against the oracle's quantize_weights(..., group), the per-group
INT32 partials bit-exact against group_partials (one partial per group: two per
128-wide plane for group 64, one per two planes for group 256), the fp32 fold exact
on inputs that make it exact, and the layer within the output tolerance.
"""

import numpy as np
import pytest
import torch

from helpers import assert_bf16_adjacent, assert_close, decode_packed, untile_act
from oracle import w4a8_oracle as O
from test_gpu_exact_fold import STEP
from test_gpu_moe import Layer, bf16_to_f32, dev_bf16
from w4a8_quantized_moe_token_b200 import binding as B
from w4a8_quantized_moe_token_b200 import synth

pytestmark = pytest.mark.gpu

GROUPS = [64, 256]
QUANT = {"asym": (0, lambda w, g: O.quantize_weights(w, group=g)),
         "sym": (B.W4A8_PACK_SYMMETRIC, lambda w, g: O.quantize_weights_symmetric(w, g))}


def pack_group(w, layout, group, flag=0):
    E, N, K = w.shape
    Kp = B.padded_k(K, group)
    packed = B.empty_aligned(B.w4a8_packed_bytes(E, N, K, layout | flag | B.GROUP_FLAG[group]))
    codes = torch.empty((E, N, Kp // 2), dtype=torch.uint8, device="cuda")
    scale = torch.empty((E, N, Kp // group), dtype=torch.float16, device="cuda")
    zp = torch.empty((E, N, Kp // group), dtype=torch.float16, device="cuda")
    B.w4a8_pack_weights(dev_bf16(w), layout | flag | B.GROUP_FLAG[group], packed, codes, scale, zp)
    return packed, codes, scale, zp


@pytest.mark.parametrize("group", GROUPS)
@pytest.mark.parametrize("scheme", sorted(QUANT))
@pytest.mark.parametrize("E,N,K,layout", [(1, 256, 512, 0), (2, 130, 200, 0), (2, 256, 1000, 1), (1, 128, 384, 0)])
def test_pack_bit_exact(E, N, K, layout, scheme, group):
    rng = np.random.default_rng(E * 1000 + N + K + group)
    w = synth.bf16_round((rng.standard_normal((E, N, K)) * 0.02).astype(np.float32))
    w[0, 0, :] = 0.0  # degenerate groups
    w[0, 1, :64] += 0.3  # a skewed 64-group
    w[-1, -1, 0] = 0.4  # an outlier
    w = synth.bf16_round(w)
    flag, quant = QUANT[scheme]
    packed, codes, scale, zp = pack_group(w, layout, group, flag)
    dc, ds, dz = decode_packed(packed.cpu().numpy(), E, N, K, layout, group)
    for e in range(E):
        c, sc, z = quant(w[e], group)
        assert np.array_equal(codes[e].cpu().numpy(), O.pack_nibbles(c)), f"canonical bytes, matrix {e}"
        assert np.array_equal(scale[e].cpu().numpy().view(np.uint16), sc.view(np.uint16))
        assert np.array_equal(zp[e].cpu().numpy().view(np.uint16), z.view(np.uint16))
        assert np.array_equal(dc[e], c), f"tiled codes, matrix {e}"
        assert np.array_equal(ds[e].view(np.uint16), sc.view(np.uint16))
        assert np.array_equal(dz[e].view(np.uint16), z.view(np.uint16))
    hdr = packed[:48].cpu().numpy().view(np.uint32)
    assert hdr[0] == 0x38413457 and hdr[1] == 2 and hdr[11] == group


@pytest.mark.parametrize("group", GROUPS)
@pytest.mark.parametrize("M,N,K", [(300, 256, 640), (129, 130, 200), (16, 256, 1024), (5, 128, 384), (40, 384, 512)])
def test_dense_partials_bit_exact(M, N, K, group):
    """M > 16: the wide-tile kernel; M <= 16: the decode-tile kernel."""
    x, w = synth.dense_gemm_inputs(M * 3 + K + group, M, K, N)
    qa, sa = O.quantize_act(x)  # [M][K rounded to 128]: the row padding to Kp is implicit
    codes, scale, zp = O.quantize_weights(w, group=group)
    packed = pack_group(w[None], 0, group)[0]
    Gq = codes.shape[1] // group
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    part = torch.zeros((M, N, Gq), dtype=torch.int32, device="cuda")
    ws = B.empty_aligned(B.w4a8_gemm_workspace_bytes_g(M, N, K, group))
    qa_d, sa_d = torch.from_numpy(qa).cuda(), torch.from_numpy(sa).cuda()
    B.w4a8_gemm_g(qa_d, sa_d, packed, N, K, group, y, ws, part)
    torch.cuda.synchronize()
    assert B.w4a8_last_device_error(ws) == 0
    qg = O.pad_k(qa, group)
    acc = O.group_partials(qg, codes, zp)
    assert np.array_equal(part.cpu().numpy().astype(np.int64), acc)
    assert_close(y.cpu().numpy(), O.w4a8_linear(qg, sa, codes, scale, zp, acc), max_rel=1e-4, mae_rel=1e-5)
    # the production instance (no partials buffer) on the same inputs
    y2 = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    B.w4a8_gemm_g(qa_d, sa_d, packed, N, K, group, y2, ws)
    torch.cuda.synchronize()
    assert_close(y2.cpu().numpy(), O.w4a8_linear(qg, sa, codes, scale, zp, acc), max_rel=1e-4, mae_rel=1e-5)


def exact_scale_weights(seed, N, K, group):
    """Weights on the grid {-8..7} * 2^-6 with both -8 and 7 in every group: every
    group's scale is exactly 2^-6 and its zero point 8 (see test_gpu_exact_fold)."""
    rng = np.random.default_rng([seed, N, K, group])
    lv = rng.integers(-8, 8, size=(N, K))
    rows = np.arange(N)
    for k0 in range(0, K, group):
        n = min(K, k0 + group) - k0
        pick = np.argsort(rng.random((N, n)), axis=1)[:, :2]
        lv[rows, k0 + pick[:, 0]] = -8
        lv[rows, k0 + pick[:, 1]] = 7
    return (lv * STEP).astype(np.float32)


@pytest.mark.parametrize("group", GROUPS)
@pytest.mark.parametrize("M,N,K", [(300, 256, 640), (16, 256, 512), (129, 128, 8192), (7, 130, 1000)])
def test_dense_without_partials_is_bit_exact(M, N, K, group):
    """The production instances: every term scale * P is a multiple of 2^-6 below
    2^24 * 2^-6 (K <= 8192), so the fp32 fold is exact in any order and y must equal
    the oracle's fp32-rounded result bit for bit."""
    x = synth.activations(M * 5 + K + group, M, K)
    qa, sa = O.quantize_act(x)
    w = exact_scale_weights(M + N + K, N, K, group)
    codes, scale, zp = O.quantize_weights(w, group=group)
    assert np.all(scale.astype(np.float32) == np.float32(STEP)) and np.all(zp.astype(np.float32) == 8.0)
    packed = pack_group(w[None], 0, group)[0]
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    ws = B.empty_aligned(B.w4a8_gemm_workspace_bytes_g(M, N, K, group))
    B.w4a8_gemm_g(torch.from_numpy(qa).cuda(), torch.from_numpy(sa).cuda(), packed, N, K, group, y, ws)
    torch.cuda.synchronize()
    assert B.w4a8_last_device_error(ws) == 0
    ref = O.w4a8_linear(O.pad_k(qa, group), sa, codes, scale, zp).astype(np.float32)
    got = y.cpu().numpy()
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32)), f"{int((got != ref).sum())} of {got.size} differ"


class GroupLayer(Layer):
    """A Layer whose experts are packed (and quantised by the oracle) with `group`."""

    def __init__(self, T, E, k, H, F, routing, seed, group):
        self.group = group
        super().__init__(T, E, k, H, F, routing, seed=seed)
        up = B.empty_aligned(B.w4a8_packed_bytes(E, 2 * F, H, B.W4A8_LAYOUT_GATEUP | B.GROUP_FLAG[group]))
        dn = B.empty_aligned(B.w4a8_packed_bytes(E, H, F, B.W4A8_LAYOUT_PLAIN | B.GROUP_FLAG[group]))
        B.w4a8_pack_weights(dev_bf16(np.stack([self.w_up(e) for e in range(E)])),
                            B.W4A8_LAYOUT_GATEUP | B.GROUP_FLAG[group], up)
        B.w4a8_pack_weights(dev_bf16(np.stack([self.w_down(e) for e in range(E)])),
                            B.W4A8_LAYOUT_PLAIN | B.GROUP_FLAG[group], dn)
        self.packed_up, self.packed_down = up, dn
        torch.cuda.synchronize()

    def experts(self):
        for e in np.unique(self.ids):
            if e not in self._experts:
                self._experts[int(e)] = O.QuantExpert(self.w_up(int(e)), self.w_down(int(e)), group=self.group)
        return self._experts

    def run_g(self):
        T, E, k, H, F = self.T, self.E, self.k, self.H, self.F
        self.ws = B.empty_aligned(B.w4a8_moe_workspace_bytes_g(T, E, k, H, F, self.group))
        out = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
        B.w4a8_moe_forward_g(self.packed_up, self.packed_down, E, H, F, self.group, dev_bf16(self.x),
                             torch.from_numpy(self.ids).cuda(), torch.from_numpy(self.w.astype(np.float32)).cuda(),
                             out, self.ws)
        torch.cuda.synchronize()
        assert B.w4a8_last_device_error(self.ws) == 0
        return bf16_to_f32(out)

    def dump(self, what, dtype):
        return B.w4a8_debug_dump(self.ws, self.T, self.E, self.k, self.H, self.F,
                                 B.DUMP[what] | B.DUMP_GROUP[self.group]).cpu().numpy().view(dtype)


@pytest.mark.parametrize("group", GROUPS)
@pytest.mark.parametrize("T,E,k,H,F,routing", [
    (600, 4, 2, 512, 384, "uniform"),  # wide tiles, ragged last row tile of each expert
    (37, 5, 3, 200, 100, "uniform"),   # K and F off the 128 / 256 grid
    (48, 8, 2, 256, 640, "zipf"),      # decode tiles
])
def test_moe_layer_stages_and_output(T, E, k, H, F, routing, group):
    L = GroupLayer(T, E, k, H, F, routing, seed=T + E + group, group=group)
    out = L.run_g()
    Hp, Fp = B.padded_k(H, group), B.padded_k(F, group)
    R = B.w4a8_moe_rows_capacity(T, E, k)
    RB = B.w4a8_moe_act_block_rows(T, E, k)
    counts, offs, perm, inv = O.permute(L.ids, E)
    rows = L.dump("inv", np.int32)
    tok = np.arange(T * k) // k
    xq, xs = O.quantize_act(L.x, group)
    act1 = untile_act(L.dump("act1", np.int8), R, Hp, RB)
    assert np.array_equal(act1[rows], xq[tok]), "INT8 token rows, padded to whole groups"
    experts = L.experts()
    h = synth.bf16_from_bits(L.dump("h", np.uint16).reshape(R, Fp))[rows]
    h_ref = np.zeros((T * k, F))
    for e, qe in experts.items():
        sl = perm[offs[e]:offs[e + 1]]
        if sl.size:
            h_ref[sl] = O.round_to_bf16(O.swiglu(O.w4a8_linear(xq[sl // k], xs[sl // k], *qe.up), F))
    assert_bf16_adjacent(h[:, :F], h_ref, what="h")
    act2 = untile_act(L.dump("act2", np.int8), R, Fp, RB)[rows]
    qh, sh = O.quantize_act(h[:, :F].astype(np.float32), group)
    assert np.array_equal(act2, qh)
    y2 = L.dump("y2", np.float32).reshape(R, H)[rows]
    y2_ref = np.zeros((T * k, H))
    for e, qe in experts.items():
        sl = perm[offs[e]:offs[e + 1]]
        if sl.size:
            y2_ref[sl] = O.w4a8_linear(qh[sl], sh[sl], *qe.down)
    assert_close(y2, y2_ref, max_rel=1e-4, mae_rel=1e-5, what="y2")
    ref = O.moe_forward(L.x, L.ids, L.w, experts, E, F)
    assert_close(out, ref, what="out")
