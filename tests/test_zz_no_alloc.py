"""The dense W4A8 GEMM entry point that allocates nothing (w4a8_gemm_noalloc).

It serves callers that cannot give the library a workspace (a plugin whose host
owns all device memory, code where an allocation is not allowed).  It must give
the same result as w4a8_gemm with a caller workspace, call after call, although
every call reuses the same fixed scratch array inside the library.  This file is
collected last so that a failure here does not stop the other tests from running.
"""

import numpy as np
import pytest
import torch

from helpers import assert_close
from oracle import w4a8_oracle as O
from w4a8_quantized_moe_token_b200 import binding as B
from w4a8_quantized_moe_token_b200 import synth

pytestmark = pytest.mark.gpu


def _inputs(M, K, N, seed):
    x, w = synth.dense_gemm_inputs(seed, M, K, N)
    qa, sa = O.quantize_act(x)
    packed = B.empty_aligned(B.w4a8_packed_bytes(1, N, K, 0))
    wd = torch.from_numpy(synth.bf16_bits(w).view(np.int16)).view(torch.bfloat16).cuda()
    B.w4a8_pack_weights(wd, 0, packed)
    return torch.from_numpy(qa).cuda(), torch.from_numpy(sa).cuda(), packed


def test_noalloc_gemm_matches_workspace_gemm_on_consecutive_calls():
    # two calls in a row; the second is smaller, so stale rows of the first call
    # would show up in its result if the shared scratch were not rewritten
    for M, N, K, seed in [(300, 256, 640, 1), (16, 256, 512, 2)]:
        qa, sa, packed = _inputs(M, K, N, seed)
        G = O.padded_k(K) // 128
        y_ref = torch.empty((M, N), dtype=torch.float32, device="cuda")
        p_ref = torch.empty((M, N, G), dtype=torch.int32, device="cuda")
        ws = B.empty_aligned(B.w4a8_gemm_workspace_bytes(M, N, K))
        B.w4a8_gemm(qa, sa, packed, N, K, y_ref, ws, p_ref)
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        p = torch.zeros((M, N, G), dtype=torch.int32, device="cuda")
        B.w4a8_gemm_noalloc(qa, sa, packed, N, K, y, p)
        torch.cuda.synchronize()
        assert B.w4a8_gemm_noalloc_last_error() == 0
        assert torch.equal(p, p_ref)
        assert_close(y.cpu().numpy(), y_ref.cpu().numpy(), max_rel=1e-4, mae_rel=1e-5, what="y")
        # and against the oracle on its own: exact INT32 partials, y within the GEMM tolerance
        x, w = synth.dense_gemm_inputs(seed, M, K, N)
        qo, so = O.quantize_act(x)
        codes, scale, zp = O.quantize_weights(w)
        acc = O.group_partials(qo, codes, zp)
        assert np.array_equal(p.cpu().numpy().astype(np.int64), acc)
        assert_close(y.cpu().numpy(), O.w4a8_linear(qo, so, codes, scale, zp, acc), max_rel=1e-4, mae_rel=1e-5,
                     what="y vs oracle")


def test_noalloc_gemm_rejects_sizes_beyond_its_scratch():
    qa, sa, packed = _inputs(16, 512, 256, 3)
    y = torch.empty((16, 256), dtype=torch.float32, device="cuda")
    # 4096 x 7168 INT8 values need 28 MiB of scratch, more than the fixed 8 MiB:
    # rejected with W4A8_ENOSPACE before anything is launched
    st = B.lib().w4a8_gemm_noalloc(B._ptr(qa), B._ptr(sa), 4096, B._ptr(packed), 256, 7168, B._ptr(y), None,
                                   B._stream())
    assert st == -3
