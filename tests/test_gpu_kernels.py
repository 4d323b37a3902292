"""GPU parity of the single kernels against the CPU oracle: activation INT8,
weight INT4 packing, routing and the dense W4A8 GEMM (per-group INT32 partials
bit-exact)."""

import numpy as np
import pytest
import torch

from helpers import assert_close, decode_packed
from oracle import w4a8_oracle as O
from w4a8_quantized_moe_token_b200 import binding as B
from w4a8_quantized_moe_token_b200 import synth

pytestmark = pytest.mark.gpu


def dev_bf16(a):
    a = np.ascontiguousarray(a, dtype=np.float32)
    assert np.array_equal(synth.bf16_round(a), a), "inputs must be bf16-exact"
    return torch.from_numpy(synth.bf16_bits(a).view(np.int16)).view(torch.bfloat16).cuda()


def pack_on_gpu(w_f32, layout, canonical=True):
    """w_f32: [E][N][K] bf16-exact float32 -> (packed tensor, codes, scale, zp) on the GPU."""
    E, N, K = w_f32.shape
    G = -(-K // 128)
    packed = B.empty_aligned(B.w4a8_packed_bytes(E, N, K, layout))
    codes = scale = zp = None
    if canonical:
        codes = torch.empty((E, N, G * 64), dtype=torch.uint8, device="cuda")
        scale = torch.empty((E, N, G), dtype=torch.float16, device="cuda")
        zp = torch.empty((E, N, G), dtype=torch.float16, device="cuda")
    B.w4a8_pack_weights(dev_bf16(w_f32), layout, packed, codes, scale, zp)
    return packed, codes, scale, zp


# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("T,K,outl", [(16, 512, 0), (37, 200, 0), (5, 7168, 0), (1, 128, 0), (64, 4096, 0.001),
                                      (300, 1000, 0)])
def test_quant_act_bit_exact(T, K, outl):
    x = synth.activations(T + K, T, K, outl, 20.0)
    if T > 3:
        x[2] = 0.0  # an all-zero row
        x[3, ::7] = 0.5  # ties at x/s = k + 0.5 are possible
        # a row with max 1.0 (s = 1/127): +-0.5 and +-1.5 * 2^-k land within a few ulp of
        # half-integers, the quantiser's slow (exact division) path
        x[T - 1] = 0.0
        x[T - 1, 0] = 1.0
        x[T - 1, 1:9] = [0.5, -0.5, 0.75, -0.25, 0.125, 1.0, -1.0, 0.0625]
    q = torch.empty((T, O.padded_k(K)), dtype=torch.int8, device="cuda")
    s = torch.empty(T, dtype=torch.float32, device="cuda")
    B.w4a8_quant_act(dev_bf16(x), q, s)
    qo, so = O.quantize_act(x)
    assert np.array_equal(s.cpu().numpy(), so)
    assert np.array_equal(q.cpu().numpy(), qo)


def test_quant_act_worked_example():
    x = np.zeros((2, 128), np.float32)
    x[0, :3] = [0.2, -0.5, 0.5]
    x[1, :3] = [0.2, -1.0, 1.0]
    x = synth.bf16_round(x)
    q = torch.empty((2, 128), dtype=torch.int8, device="cuda")
    s = torch.empty(2, dtype=torch.float32, device="cuda")
    B.w4a8_quant_act(dev_bf16(x), q, s)
    qo, so = O.quantize_act(x)
    assert np.array_equal(q.cpu().numpy(), qo)
    assert int(q[0, 0]) == int(qo[0, 0])


SCHEMES = {"asym": (0, O.quantize_weights),
           "sym": (B.W4A8_PACK_SYMMETRIC, O.quantize_weights_symmetric),
           "clip999": (B.W4A8_PACK_CLIP999, lambda w: O.quantize_weights(w, clip999=True))}


@pytest.mark.parametrize("scheme", sorted(SCHEMES))
@pytest.mark.parametrize("E,N,K,layout", [(2, 256, 512, 0), (3, 200, 200, 0), (2, 384, 256, 1), (1, 130, 1000, 1),
                                          (4, 128, 128, 0)])
def test_pack_bit_exact(E, N, K, layout, scheme):
    rng = np.random.default_rng(E * 1000 + N + K)
    w = synth.bf16_round((rng.standard_normal((E, N, K)) * 0.02).astype(np.float32))
    w[0, 0, :] = 0.0  # degenerate group
    w[0, 1, :128] += 0.3  # skewed group
    w[-1, -1, 0] = 0.4  # an outlier
    w[-1, -2, 1:3] = -0.25  # two equal low outliers
    w = synth.bf16_round(w)
    flag, quant = SCHEMES[scheme]
    packed, codes, scale, zp = pack_on_gpu(w, layout | flag)
    codes_h, scale_h, zp_h = codes.cpu().numpy(), scale.cpu().numpy(), zp.cpu().numpy()
    dc, ds, dz = decode_packed(packed.cpu().numpy(), E, N, K, layout)
    for e in range(E):
        c, sc, z = quant(w[e])
        assert np.array_equal(codes_h[e], O.pack_nibbles(c)), f"canonical bytes, expert {e}"
        assert np.array_equal(scale_h[e].view(np.uint16), sc.view(np.uint16))
        assert np.array_equal(zp_h[e].view(np.uint16), z.view(np.uint16))
        assert np.array_equal(dc[e], c), f"tiled codes, expert {e}"
        assert np.array_equal(ds[e].view(np.uint16), sc.view(np.uint16))
        assert np.array_equal(dz[e].view(np.uint16), z.view(np.uint16))
    hdr = packed[:48].cpu().numpy().view(np.uint32)
    assert hdr[0] == 0x38413457 and hdr[3] == E and hdr[4] == N and hdr[5] == K


def test_route_topk():
    T, E, k = 64, 64, 6
    lg = synth.router_logits(0, T, E)
    lg[0, :10] = 1.5  # ties resolved towards the lower id
    ids = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    B.w4a8_route_topk(dev_bf16(lg), k, ids, w)
    io, wo = O.route_topk(lg, k)
    assert np.array_equal(ids.cpu().numpy(), io)
    np.testing.assert_allclose(w.cpu().numpy(), wo, rtol=2e-6, atol=0)


# --------------------------------------------------------------------------- #
def run_dense_gemm(M, N, K, seed=0, scheme="asym"):
    x, w = synth.dense_gemm_inputs(seed, M, K, N)
    qa, sa = O.quantize_act(x)
    flag, quant = SCHEMES[scheme]
    codes, scale, zp = quant(w)
    packed, _, _, _ = pack_on_gpu(w[None], flag, canonical=False)
    G = O.padded_k(K) // 128
    qa_d = torch.from_numpy(qa).cuda()
    sa_d = torch.from_numpy(sa).cuda()
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    part = torch.zeros((M, N, G), dtype=torch.int32, device="cuda")
    ws = B.empty_aligned(B.w4a8_gemm_workspace_bytes(M, N, K))
    B.w4a8_gemm(qa_d, sa_d, packed, N, K, y, ws, part)
    torch.cuda.synchronize()
    assert B.w4a8_last_device_error(ws) == 0
    acc = O.group_partials(qa, codes, zp)
    return y.cpu().numpy(), part.cpu().numpy(), acc, O.w4a8_linear(qa, sa, codes, scale, zp, acc)


def test_dense_gemm_16x512x256_partials_bit_exact():
    y, part, acc, yo = run_dense_gemm(16, 256, 512)
    assert np.array_equal(part.astype(np.int64), acc)
    assert_close(y, yo, max_rel=1e-4, mae_rel=1e-5, what="y")


@pytest.mark.parametrize("scheme", ["sym", "clip999"])
@pytest.mark.parametrize("M,N,K", [(16, 256, 512), (300, 100, 640)])
def test_dense_gemm_other_schemes_partials_bit_exact(M, N, K, scheme):
    """Symmetric (zero point 8) and percentile-clipped weights through both GEMM kernels
    (M <= 16: decode tiles)."""
    y, part, acc, yo = run_dense_gemm(M, N, K, seed=7 + M, scheme=scheme)
    assert np.array_equal(part.astype(np.int64), acc)
    assert_close(y, yo, max_rel=1e-4, mae_rel=1e-5, what="y")


@pytest.mark.parametrize("M,N,K", [(1, 128, 128), (5, 128, 256), (130, 384, 200), (256, 256, 1024),
                                   (300, 100, 640), (129, 256, 384)])
def test_dense_gemm_shapes(M, N, K):
    y, part, acc, yo = run_dense_gemm(M, N, K, seed=M + N + K)
    assert np.array_equal(part.astype(np.int64), acc)
    assert_close(y, yo, max_rel=1e-4, mae_rel=1e-5, what="y")
