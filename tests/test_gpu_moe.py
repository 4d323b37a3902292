"""GPU parity of the whole W4A8 MoE layer against the CPU oracle.

Stage by stage on identical inputs: permutation (bit-exact), INT8 activations
(bit-exact), h after the up GEMM + SwiGLU (tolerance), requantised h
(bit-exact on the dumped h), down GEMM output (tolerance), and the final bf16
output (max relative error 1e-2, mean absolute error <= 1e-3 * rms)."""

import numpy as np
import pytest
import torch

from helpers import assert_bf16_adjacent, assert_close, untile_act
from oracle import w4a8_oracle as O
from w4a8_quantized_moe_token_b200 import binding as B
from w4a8_quantized_moe_token_b200 import synth

pytestmark = pytest.mark.gpu


def dev_bf16(a):
    a = np.ascontiguousarray(a, dtype=np.float32)
    return torch.from_numpy(synth.bf16_bits(a).view(np.int16)).view(torch.bfloat16).cuda()


def bf16_to_f32(t):
    return synth.bf16_from_bits(t.view(torch.int16).cpu().numpy().view(np.uint16))


class Layer:
    """One synthetic MoE layer, packed on the GPU, with lazily quantised oracle experts."""

    def __init__(self, T, E, k, H, F, routing="uniform", seed=0, zipf_s=1.1, outlier=0.0, scheme="asym"):
        self.T, self.E, self.k, self.H, self.F, self.seed = T, E, k, H, F, seed
        self.scheme = scheme
        flag = {"asym": 0, "sym": B.W4A8_PACK_SYMMETRIC, "clip999": B.W4A8_PACK_CLIP999}[scheme]
        self.x = synth.activations(seed, T, H, outlier, 20.0)
        if routing == "softmax":
            self.logits = synth.router_logits(seed, T, E)
            self.ids, self.w = O.route_topk(self.logits, k)
        else:
            self.logits = None
            self.ids, w = synth.synthetic_routing(seed, T, E, k, routing, zipf_s)
            self.w = w.astype(np.float64)
        self._w_up = {}
        self._w_down = {}
        self._experts = {}
        self.packed_up = B.empty_aligned(B.w4a8_packed_bytes(E, 2 * F, H, B.W4A8_LAYOUT_GATEUP))
        self.packed_down = B.empty_aligned(B.w4a8_packed_bytes(E, H, F, B.W4A8_LAYOUT_PLAIN))
        # pack expert by expert into slices of one buffer (experts are independent in the layout)
        up_stride = (B.w4a8_packed_bytes(E, 2 * F, H, 1) - 256) // E
        dn_stride = (B.w4a8_packed_bytes(E, H, F, 0) - 256) // E
        tmp_up = B.empty_aligned(B.w4a8_packed_bytes(1, 2 * F, H, 1))
        tmp_dn = B.empty_aligned(B.w4a8_packed_bytes(1, H, F, 0))
        for e in range(E):
            B.w4a8_pack_weights(dev_bf16(self.w_up(e)), B.W4A8_LAYOUT_GATEUP | flag, tmp_up)
            B.w4a8_pack_weights(dev_bf16(self.w_down(e)), B.W4A8_LAYOUT_PLAIN | flag, tmp_dn)
            self.packed_up[256 + e * up_stride:256 + (e + 1) * up_stride].copy_(tmp_up[256:])
            self.packed_down[256 + e * dn_stride:256 + (e + 1) * dn_stride].copy_(tmp_dn[256:])
        torch.cuda.synchronize()

    def w_up(self, e):
        if e not in self._w_up:
            self._w_up[e] = synth.expert_weight(self.seed, e, "up", 2 * self.F, self.H)
        return self._w_up[e]

    def w_down(self, e):
        if e not in self._w_down:
            self._w_down[e] = synth.expert_weight(self.seed, e, "down", self.H, self.F)
        return self._w_down[e]

    def experts(self):
        for e in np.unique(self.ids):
            if e not in self._experts:
                self._experts[int(e)] = O.QuantExpert(self.w_up(int(e)), self.w_down(int(e)),
                                                      symmetric=self.scheme == "sym",
                                                      clip999=self.scheme == "clip999")
        return self._experts

    def run(self, use_router=False):
        T, E, k, H, F = self.T, self.E, self.k, self.H, self.F
        self.ws = B.empty_aligned(B.w4a8_moe_workspace_bytes(T, E, k, H, F))
        x = dev_bf16(self.x)
        if use_router:
            ids = torch.empty((T, k), dtype=torch.int32, device="cuda")
            w = torch.empty((T, k), dtype=torch.float32, device="cuda")
            B.w4a8_route_topk(dev_bf16(self.logits), k, ids, w)
        else:
            ids = torch.from_numpy(self.ids).cuda()
            w = torch.from_numpy(self.w.astype(np.float32)).cuda()
        out = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
        B.w4a8_moe_forward(self.packed_up, self.packed_down, E, H, F, x, ids, w, out, self.ws)
        torch.cuda.synchronize()
        assert B.w4a8_last_device_error(self.ws) == 0
        self.dev_ids, self.dev_w = ids.cpu().numpy(), w.cpu().numpy()
        return bf16_to_f32(out)

    def dump(self, what, dtype):
        return B.w4a8_debug_dump(self.ws, self.T, self.E, self.k, self.H, self.F, what).cpu().numpy().view(dtype)


def check_stages(L: Layer, out):
    T, E, k, H, F = L.T, L.E, L.k, L.H, L.F
    Hp, Fp = O.padded_k(H), O.padded_k(F)
    R = B.w4a8_moe_rows_capacity(T, E, k)
    # a4: permutation, bit-exact
    counts, offs, perm, inv = O.permute(L.ids, E)
    assert np.array_equal(L.dump("counts", np.int32), counts)
    assert np.array_equal(L.dump("offs", np.int32), offs)
    assert np.array_equal(L.dump("perm", np.int32), perm)
    poffs = L.dump("poffs", np.int32)
    assert poffs[0] == 0 and np.all(np.diff(poffs) == (counts + 15) // 16 * 16)
    inv_d = L.dump("inv", np.int32)
    flat = L.ids.reshape(-1)
    assert np.array_equal(inv_d - poffs[flat] + offs[flat], inv)
    # a2: INT8 activations of the grouped rows, bit-exact
    xq, xs = O.quantize_act(L.x)
    RB = B.w4a8_moe_act_block_rows(T, E, k)
    assert RB in (16, R)
    act1 = untile_act(L.dump("act1", np.int8), R, Hp, RB)
    s1 = L.dump("s1", np.float32)
    rows = inv_d  # padded row of each slot
    tok = np.arange(T * k) // k
    assert np.array_equal(act1[rows], xq[tok])
    assert np.array_equal(s1[rows], xs[tok])
    # a5 + a6: h (bf16) on identical INT8 inputs
    experts = L.experts()
    h = synth.bf16_from_bits(L.dump("h", np.uint16).reshape(R, Fp))
    h_ref = np.zeros((T * k, F))
    for e, qe in experts.items():
        sl = perm[offs[e]:offs[e + 1]]
        if sl.size:
            t_e = sl // k
            h_ref[sl] = O.round_to_bf16(O.swiglu(O.w4a8_linear(xq[t_e], xs[t_e], *qe.up), F))
    assert_bf16_adjacent(h[rows, :F], h_ref, what="h")
    # a6: requantisation of the dumped h, bit-exact
    act2 = untile_act(L.dump("act2", np.int8), R, Fp, RB)
    s2 = L.dump("s2", np.float32)
    qh, sh = O.quantize_act(h[rows, :F].astype(np.float32))
    assert np.array_equal(act2[rows], qh)
    assert np.array_equal(s2[rows], sh)
    # a7: down GEMM on identical INT8 inputs
    y2 = L.dump("y2", np.float32).reshape(R, H)
    y2_ref = np.zeros((T * k, H))
    for e, qe in experts.items():
        sl = perm[offs[e]:offs[e + 1]]
        if sl.size:
            y2_ref[sl] = O.w4a8_linear(qh[sl], sh[sl], *qe.down)
    assert_close(y2[rows], y2_ref, max_rel=1e-4, mae_rel=1e-5, what="y2")
    # a8: combine of the dumped y2
    comb = O.round_to_bf16(O.combine(y2[rows].astype(np.float64), L.w, np.arange(T * k), T, k))
    assert_close(out, comb, max_rel=1e-2, mae_rel=1e-3, what="combine")


SMALL = [
    # T, E, k, H, F, routing
    (1, 4, 2, 256, 128, "uniform"),
    (37, 5, 3, 200, 100, "uniform"),   # K and F off the 128 / 64 grid
    (3, 16, 1, 256, 128, "uniform"),   # most experts empty
    (300, 4, 2, 512, 256, "uniform"),  # several row tiles per expert
    (64, 12, 4, 384, 192, "zipf"),
    (64, 32, 4, 256, 256, "zipf"),     # decode kernel, hot experts span several 16-token tiles
    (4500, 16, 4, 256, 128, "uniform"),  # > 16384 slots: multi-CTA permutation
]


@pytest.mark.parametrize("T,E,k,H,F,routing", SMALL)
def test_moe_small_stages_and_output(T, E, k, H, F, routing):
    L = Layer(T, E, k, H, F, routing, seed=T + E)
    out = L.run()
    check_stages(L, out)
    ref = O.moe_forward(L.x, L.ids, L.w, L.experts(), E, F)
    assert_close(out, ref, what="out")


@pytest.mark.parametrize("scheme", ["sym", "clip999"])
@pytest.mark.parametrize("T,E,k,H,F,routing", [(300, 4, 2, 512, 256, "uniform"), (64, 32, 4, 256, 256, "zipf")])
def test_moe_other_weight_schemes_stages_and_output(T, E, k, H, F, routing, scheme):
    """The symmetric and percentile-clipped packer variants through the whole layer
    (wide and decode tiles)."""
    L = Layer(T, E, k, H, F, routing, seed=T + E + 1, scheme=scheme)
    out = L.run()
    check_stages(L, out)
    ref = O.moe_forward(L.x, L.ids, L.w, L.experts(), E, F)
    assert_close(out, ref, what="out")


def test_moe_empty_batch():
    L = Layer(1, 4, 2, 256, 128)
    ws = B.empty_aligned(B.w4a8_moe_workspace_bytes(0, 4, 2, 256, 128))
    out = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    B.w4a8_moe_forward(L.packed_up, L.packed_down, 4, 256, 128, out, torch.empty((0, 2), dtype=torch.int32,
                       device="cuda"), torch.empty((0, 2), dtype=torch.float32, device="cuda"), out, ws)
    torch.cuda.synchronize()


def test_moe_bad_expert_id_flags_device_error():
    L = Layer(8, 4, 2, 256, 128)
    L.ids = L.ids.copy()
    L.ids[3, 1] = 7  # out of range: the slot is dropped and the error word is set
    T, E, k, H, F = L.T, L.E, L.k, L.H, L.F
    ws = B.empty_aligned(B.w4a8_moe_workspace_bytes(T, E, k, H, F))
    out = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    B.w4a8_moe_forward(L.packed_up, L.packed_down, E, H, F, dev_bf16(L.x), torch.from_numpy(L.ids).cuda(),
                       torch.from_numpy(L.w.astype(np.float32)).cuda(), out, ws)
    torch.cuda.synchronize()
    assert B.w4a8_last_device_error(ws) & 2


def test_toy_moe_config():
    """8 experts, top-1 uniform, 4096 tokens, hidden 2048, expert ffn 1024."""
    w = synth.WORKLOADS["toy_moe"]
    L = Layer(w.T, w.E, w.topk, w.H, w.F, w.routing, seed=0)
    out = L.run()
    check_stages(L, out)
    ref = O.moe_forward(L.x, L.ids, L.w, L.experts(), w.E, w.F)
    assert_close(out, ref, what="out")


def test_decode_config_with_router():
    """64 experts, top-6 softmax routing from N(0,1) logits, 64 tokens, hidden 4096,
    expert ffn 1408, 0.1% outlier channels x20."""
    w = synth.WORKLOADS["decode"]
    L = Layer(w.T, w.E, w.topk, w.H, w.F, "softmax", seed=0, outlier=w.outlier_frac)
    out = L.run(use_router=True)
    assert np.array_equal(L.dev_ids, L.ids)
    np.testing.assert_allclose(L.dev_w, L.w, rtol=2e-6)
    check_stages(L, out)
    ref = O.moe_forward(L.x, L.ids, L.w, L.experts(), w.E, w.F)
    assert_close(out, ref, what="out")


def test_host_buffer_entry_point_matches_device_entry_point():
    L = Layer(37, 5, 3, 256, 128, seed=3)
    out_dev = L.run()
    T, E, k, H, F = L.T, L.E, L.k, L.H, L.F
    ws = B.empty_aligned(B.w4a8_moe_host_workspace_bytes(T, E, k, H, F))
    xh = torch.from_numpy(synth.bf16_bits(L.x).view(np.int16)).view(torch.bfloat16).pin_memory()
    idh = torch.from_numpy(L.ids).pin_memory()
    wh = torch.from_numpy(L.w.astype(np.float32)).pin_memory()
    outh = torch.empty((T, H), dtype=torch.bfloat16).pin_memory()
    B.w4a8_moe_forward_host(L.packed_up, L.packed_down, E, H, F, xh, idh, wh, outh, ws)
    torch.cuda.synchronize()
    assert np.array_equal(bf16_to_f32(outh), out_dev)


def test_logits_host_entry_point_matches_router_and_device_entry_point():
    L = Layer(37, 8, 3, 256, 128, "softmax", seed=5)
    out_dev = L.run(use_router=True)
    T, E, k, H, F = L.T, L.E, L.k, L.H, L.F
    ws = B.empty_aligned(B.w4a8_moe_host_workspace_bytes(T, E, k, H, F))
    xh = torch.from_numpy(synth.bf16_bits(L.x).view(np.int16)).view(torch.bfloat16).pin_memory()
    lgh = torch.from_numpy(synth.bf16_bits(L.logits).view(np.int16)).view(torch.bfloat16).pin_memory()
    outh = torch.empty((T, H), dtype=torch.bfloat16).pin_memory()
    B.w4a8_moe_forward_logits_host(L.packed_up, L.packed_down, E, H, F, xh, lgh, k, outh, ws)
    torch.cuda.synchronize()
    assert B.w4a8_last_device_error(ws) == 0
    assert np.array_equal(bf16_to_f32(outh), out_dev)


def test_binding_rejects_undersized_buffers():
    """The kernels trust the sizes they are given, so the binding checks every buffer
    against the shapes before the call."""
    M, N, K = 32, 256, 512
    qa = torch.zeros((M, K), dtype=torch.int8, device="cuda")
    sa = torch.ones(M, dtype=torch.float32, device="cuda")
    packed = B.empty_aligned(B.w4a8_packed_bytes(1, N, K, 0))
    ws = B.empty_aligned(B.w4a8_gemm_workspace_bytes(M, N, K))
    with pytest.raises(B.W4A8Error):
        B.w4a8_gemm(qa, sa, packed, N, K, torch.empty(M * N - 1, dtype=torch.float32, device="cuda"), ws)
    with pytest.raises(B.W4A8Error):
        B.w4a8_gemm(qa[:, :256], sa, packed, N, K, torch.empty((M, N), dtype=torch.float32, device="cuda"), ws)
    with pytest.raises(B.W4A8Error):
        B.w4a8_gemm(qa, sa[:M - 1], packed, N, K, torch.empty((M, N), dtype=torch.float32, device="cuda"), ws)
    with pytest.raises(B.W4A8Error):
        B.w4a8_gemm_noalloc(qa, sa, packed, N, K, torch.empty((M, N), dtype=torch.float32, device="cuda"),
                            torch.empty((M, N, 3), dtype=torch.int32, device="cuda"))
    L = Layer(8, 4, 2, 256, 128)
    with pytest.raises(B.W4A8Error):  # out has the wrong shape
        B.w4a8_moe_forward(L.packed_up, L.packed_down, 4, 256, 128, dev_bf16(L.x), torch.from_numpy(L.ids).cuda(),
                           torch.from_numpy(L.w.astype(np.float32)).cuda(),
                           torch.empty((8, 128), dtype=torch.bfloat16, device="cuda"),
                           B.empty_aligned(B.w4a8_moe_workspace_bytes(8, 4, 2, 256, 128)))
