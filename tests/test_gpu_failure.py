"""Failure detection on the GPU without a fault: a bounded wait that runs out.

Every wait inside the GEMM kernels has a limit; when it runs out the kernel sets
bit 0 of the device error word, drains the copies and tensor-core work it issued,
frees its tensor memory and returns, so the context stays usable.  The test hook
w4a8_debug_inject shortens the limit to about a millisecond and has the first CTA
skip the copies of its first pipeline step, so that the waits for that stage run
out.  Each test checks that the error is reported and that the next normal call
on the same workspace gives the right result.
"""

import numpy as np
import pytest
import torch

from helpers import assert_close
from oracle import w4a8_oracle as O
from w4a8_quantized_moe_token_b200 import binding as B
from w4a8_quantized_moe_token_b200 import synth

pytestmark = pytest.mark.gpu

SHORT_WAIT = 2_000_000  # clock cycles, about 1 ms


def to_dev_bf16(a):
    a = np.ascontiguousarray(a, dtype=np.float32)
    return torch.from_numpy(synth.bf16_bits(a).view(np.int16)).view(torch.bfloat16).cuda()


@pytest.fixture(autouse=True)
def _restore_normal_waits():
    yield
    B.w4a8_debug_inject(0, 0)


@pytest.mark.parametrize("M", [300, 16])  # wide tiles, decode tiles
def test_gemm_wait_timeout_is_reported_and_recovers(M):
    N, K = 256, 640
    x, w = synth.dense_gemm_inputs(M, M, K, N)
    qa, sa = O.quantize_act(x)
    codes, scale, zp = O.quantize_weights(w)
    packed = B.empty_aligned(B.w4a8_packed_bytes(1, N, K, 0))
    B.w4a8_pack_weights(to_dev_bf16(w), 0, packed)
    qa_d, sa_d = torch.from_numpy(qa).cuda(), torch.from_numpy(sa).cuda()
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    ws = B.empty_aligned(B.w4a8_gemm_workspace_bytes(M, N, K))

    B.w4a8_debug_inject(B.W4A8_DEBUG_SKIP_FIRST_COPY, SHORT_WAIT)
    B.w4a8_gemm(qa_d, sa_d, packed, N, K, y, ws)
    torch.cuda.synchronize()
    assert B.w4a8_last_device_error(ws) & 1, "the wait that ran out must set bit 0"
    B.w4a8_debug_inject(0, 0)

    part = torch.zeros((M, N, O.padded_k(K) // 128), dtype=torch.int32, device="cuda")
    B.w4a8_gemm(qa_d, sa_d, packed, N, K, y, ws, part)
    torch.cuda.synchronize()
    assert B.w4a8_last_device_error(ws) == 0
    acc = O.group_partials(qa, codes, zp)
    assert np.array_equal(part.cpu().numpy().astype(np.int64), acc)
    assert_close(y.cpu().numpy(), O.w4a8_linear(qa, sa, codes, scale, zp, acc), max_rel=1e-4, mae_rel=1e-5)


@pytest.mark.parametrize("T,E,k", [(600, 4, 2), (48, 8, 2)])  # wide tiles, decode tiles
def test_moe_wait_timeout_is_reported_and_recovers(T, E, k):
    H, F = 256, 256
    x = synth.activations(T, T, H)
    ids, wts = synth.synthetic_routing(T, T, E, k, "uniform")
    up = B.empty_aligned(B.w4a8_packed_bytes(E, 2 * F, H, B.W4A8_LAYOUT_GATEUP))
    dn = B.empty_aligned(B.w4a8_packed_bytes(E, H, F, B.W4A8_LAYOUT_PLAIN))
    wu = np.stack([synth.expert_weight(T, e, "up", 2 * F, H) for e in range(E)])
    wd = np.stack([synth.expert_weight(T, e, "down", H, F) for e in range(E)])
    B.w4a8_pack_weights(to_dev_bf16(wu), B.W4A8_LAYOUT_GATEUP, up)
    B.w4a8_pack_weights(to_dev_bf16(wd), B.W4A8_LAYOUT_PLAIN, dn)
    ws = B.empty_aligned(B.w4a8_moe_workspace_bytes(T, E, k, H, F))
    out = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    args = (up, dn, E, H, F, to_dev_bf16(x), torch.from_numpy(ids).cuda(), torch.from_numpy(wts).cuda(), out, ws)

    B.w4a8_debug_inject(B.W4A8_DEBUG_SKIP_FIRST_COPY, SHORT_WAIT)
    B.w4a8_moe_forward(*args)
    torch.cuda.synchronize()
    assert B.w4a8_last_device_error(ws) & 1
    B.w4a8_debug_inject(0, 0)

    B.w4a8_moe_forward(*args)
    torch.cuda.synchronize()
    assert B.w4a8_last_device_error(ws) == 0
    experts = {e: O.QuantExpert(wu[e], wd[e]) for e in range(E)}
    ref = O.moe_forward(x, ids, wts.astype(np.float64), experts, E, F)
    got = synth.bf16_from_bits(out.view(torch.int16).cpu().numpy().view(np.uint16))
    assert_close(got, ref, what="out")

