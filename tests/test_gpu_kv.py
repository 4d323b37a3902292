"""GPU parity of the INT8 KV cache (static per-head scales) against the oracle:
calibrated scales, INT8 codes and dequantised bf16 values bit-exact."""

import numpy as np
import pytest
import torch

from oracle import w4a8_oracle as O
from w4a8_quantized_moe_token_b200 import binding as B
from w4a8_quantized_moe_token_b200 import synth

pytestmark = pytest.mark.gpu


def dev_bf16(a):
    a = np.ascontiguousarray(a, dtype=np.float32)
    return torch.from_numpy(synth.bf16_bits(a).view(np.int16)).view(torch.bfloat16).cuda()


def to_f32(t):
    return synth.bf16_from_bits(t.view(torch.int16).cpu().numpy().view(np.uint16))


@pytest.mark.parametrize("Tc,T,H,D", [(64, 1, 1, 16), (100, 37, 8, 128), (256, 513, 4, 64), (8, 2048, 16, 128),
                                      (3, 5, 1024, 16)])
def test_kv_int8_bit_exact(Tc, T, H, D):
    rng = np.random.default_rng(Tc + T + H + D)
    calib = synth.bf16_round((rng.standard_normal((Tc, H, D)) * rng.uniform(0.1, 3.0, size=(1, H, 1))).astype(np.float32))
    calib[:, 0] = 0.0 if H > 1 else calib[:, 0]  # an all-zero head (when there is more than one)
    x = synth.bf16_round((rng.standard_normal((T, H, D)) * 1.5).astype(np.float32))
    x[0, -1, 0] = 1e4  # saturates
    if H > 1:
        # head 1 calibrated to max 1.0 (scale 1/127): +-0.5 lands next to 63.5, the
        # quantiser's slow (exact division) path
        calib[:, 1] = np.clip(calib[:, 1], -0.9, 0.9)
        calib[0, 1, 0] = 1.0
        x[-1, 1, :4] = [0.5, -0.5, 1.0, 0.25]
    scale = torch.empty(H, dtype=torch.float32, device="cuda")
    B.w4a8_kv_calibrate(dev_bf16(calib), scale)
    q = torch.empty((T, H, D), dtype=torch.int8, device="cuda")
    B.w4a8_kv_quant(dev_bf16(x), scale, q)
    y = torch.empty((T, H, D), dtype=torch.bfloat16, device="cuda")
    B.w4a8_kv_dequant(q, scale, y)
    torch.cuda.synchronize()
    s_ref = O.kv_calibrate(calib)
    assert np.array_equal(scale.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    q_ref = O.kv_quantize(x, s_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    y_ref = O.kv_dequantize(q_ref, s_ref)
    assert np.array_equal(to_f32(y).view(np.uint32), y_ref.astype(np.float32).view(np.uint32))


def test_kv_int8_empty_calibration_gives_zero_scales():
    scale = torch.full((4,), 7.0, dtype=torch.float32, device="cuda")
    B.w4a8_kv_calibrate(torch.empty((0, 4, 32), dtype=torch.bfloat16, device="cuda"), scale)
    torch.cuda.synchronize()
    assert np.all(scale.cpu().numpy() == 0)
