"""GPU parity at the full sizes of the two 384-expert layers, on sampled tokens.

Both layers (large decode: 256 tokens, top-8 Zipf(1.1) routing; prefill: 16384
tokens, top-8 uniform routing; hidden 7168, expert ffn 2048) run through the same
entry point and launch configuration the benchmark times.  The oracle cannot run
them whole, so:

- the permutation is compared in full (bit-exact);
- for a handful of sampled tokens, every stage of every slot of the token is
  checked against the oracle on identical inputs: the INT8 activation row
  (bit-exact), h after the up GEMM and SwiGLU (tolerance), the requantised h
  (bit-exact on the dumped h), the down GEMM row (tolerance), the combine of the
  dumped rows and the final bf16 output (max relative error 1e-2, mean absolute
  error <= 1e-3 * rms).

The sampled tokens include the first and last token and tokens whose slots land in
the last, partial row tile of an expert (and, for the Zipf layer, in the hottest
expert, which spans many 16-token tiles).
"""

import numpy as np
import pytest
import torch

from helpers import assert_bf16_adjacent, assert_close
from oracle import w4a8_oracle as O
from w4a8_quantized_moe_token_b200 import binding as B
from w4a8_quantized_moe_token_b200 import synth

pytestmark = pytest.mark.gpu

SEED = 0


def dev_bf16(a):
    a = np.ascontiguousarray(a, dtype=np.float32)
    return torch.from_numpy(synth.bf16_bits(a).view(np.int16)).view(torch.bfloat16).cuda()


@pytest.fixture(scope="module")
def packed_384():
    """Every expert of the 384-expert layers (shared E, H, F and seed), packed on the GPU."""
    w = synth.WORKLOADS["prefill"]
    w2 = synth.WORKLOADS["large_decode"]
    assert (w.E, w.H, w.F) == (w2.E, w2.H, w2.F)
    E, H, F = w.E, w.H, w.F
    up = B.empty_aligned(B.w4a8_packed_bytes(E, 2 * F, H, B.W4A8_LAYOUT_GATEUP))
    dn = B.empty_aligned(B.w4a8_packed_bytes(E, H, F, B.W4A8_LAYOUT_PLAIN))
    su = (up.numel() - 256) // E
    sd = (dn.numel() - 256) // E
    tu = B.empty_aligned(B.w4a8_packed_bytes(1, 2 * F, H, B.W4A8_LAYOUT_GATEUP))
    td = B.empty_aligned(B.w4a8_packed_bytes(1, H, F, B.W4A8_LAYOUT_PLAIN))
    for which, buf, tmp, stride, rows, cols, layout in (
            ("up", up, tu, su, 2 * F, H, B.W4A8_LAYOUT_GATEUP),
            ("down", dn, td, sd, H, F, B.W4A8_LAYOUT_PLAIN)):
        for e, wt in synth.expert_weights_parallel(SEED, E, which, rows, cols):
            B.w4a8_pack_weights(dev_bf16(wt), layout, tmp)
            buf[256 + e * stride:256 + (e + 1) * stride].copy_(tmp[256:])
    torch.cuda.synchronize()
    return up, dn


def act_row_index(rows, Kp, RB):
    """Byte offsets of rows of the tiled INT8 buffer ([R/RB][Kp/128][RB][128], 16-byte
    chunk c of in-block row i stored at chunk c ^ (i & 7)), as an index array [len(rows)][Kp]."""
    rows = np.asarray(rows, dtype=np.int64)[:, None]
    k = np.arange(Kp, dtype=np.int64)[None, :]
    G = Kp // 128
    i = rows % RB
    return ((rows // RB) * G + (k >> 7)) * RB * 128 + i * 128 + ((((k & 127) >> 4) ^ (i & 7)) << 4) + (k & 15)


def sample_tokens(ids, offs_counts_poffs, tile_rows, extra):
    """First and last token, tokens in the last row tile of two experts, plus `extra`."""
    counts, _, _ = offs_counts_poffs
    T, k = ids.shape
    chosen = [0, T - 1]
    flat = ids.reshape(-1)
    for e in np.argsort(-counts, kind="stable")[:2]:
        slots = np.nonzero(flat == e)[0]
        c = slots.size
        if c > tile_rows:
            # a slot of the expert's last (partial) tile: the order within an expert is by slot
            chosen.append(int(slots[(c - 1) // tile_rows * tile_rows]) // k)
    chosen += list(extra)
    return sorted(set(chosen))


def run_and_check(wl_name, packed, extra_tokens):
    W = synth.WORKLOADS[wl_name]
    T, E, k, H, F = W.T, W.E, W.topk, W.H, W.F
    Hp, Fp = O.padded_k(H), O.padded_k(F)
    inp = synth.moe_inputs(W, SEED)
    x, ids, wts = inp["x"], inp["ids"], inp["wts"].astype(np.float64)
    up, dn = packed
    ws = B.empty_aligned(B.w4a8_moe_workspace_bytes(T, E, k, H, F))
    out = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    B.w4a8_moe_forward(up, dn, E, H, F, dev_bf16(x), torch.from_numpy(ids).cuda(),
                       torch.from_numpy(wts.astype(np.float32)).cuda(), out, ws)
    torch.cuda.synchronize()
    assert B.w4a8_last_device_error(ws) == 0

    def dump(what):
        return B.w4a8_debug_dump(ws, T, E, k, H, F, what)

    # a4 in full, bit-exact
    counts, offs, perm, inv = O.permute(ids, E)
    assert np.array_equal(dump("counts").cpu().numpy().view(np.int32), counts)
    assert np.array_equal(dump("offs").cpu().numpy().view(np.int32), offs)
    assert np.array_equal(dump("perm").cpu().numpy().view(np.int32), perm)
    poffs = dump("poffs").cpu().numpy().view(np.int32)
    assert poffs[0] == 0 and np.all(np.diff(poffs) == (counts + 15) // 16 * 16)
    inv_d = dump("inv").cpu().numpy().view(np.int32)
    flat = ids.reshape(-1)
    assert np.array_equal(inv_d - poffs[flat] + offs[flat], inv)

    R = B.w4a8_moe_rows_capacity(T, E, k)
    RB = B.w4a8_moe_act_block_rows(T, E, k)
    tile_rows = 16 if RB == 16 else 128
    tokens = sample_tokens(ids, (counts, offs, poffs), tile_rows, extra_tokens)
    slots = np.array([t * k + j for t in tokens for j in range(k)])
    rows = inv_d[slots]
    experts = {}
    for e in np.unique(ids[tokens]):
        experts[int(e)] = O.QuantExpert(synth.expert_weight(SEED, int(e), "up", 2 * F, H),
                                        synth.expert_weight(SEED, int(e), "down", H, F))

    # a2: INT8 rows of the sampled slots, bit-exact
    xq, xs = O.quantize_act(x[tokens])
    tpos = {t: i for i, t in enumerate(tokens)}
    src = np.array([tpos[s // k] for s in slots])
    idx = torch.from_numpy(act_row_index(rows, Hp, RB)).cuda()
    act1 = dump("act1").view(torch.int8)[idx].cpu().numpy()
    s1 = dump("s1").view(torch.float32)[torch.from_numpy(rows).long().cuda()].cpu().numpy()
    assert np.array_equal(act1, xq[src])
    assert np.array_equal(s1, xs[src])

    # a5 + a6: h of the sampled rows on identical INT8 inputs
    rows_t = torch.from_numpy(rows).long().cuda()
    h = synth.bf16_from_bits(dump("h").view(torch.int16).view(R, Fp)[rows_t].cpu().numpy().view(np.uint16))
    h_ref = np.zeros((slots.size, F))
    for i, s in enumerate(slots):
        qe = experts[int(flat[s])]
        h_ref[i] = O.round_to_bf16(O.swiglu(O.w4a8_linear(xq[src[i]:src[i] + 1], xs[src[i]:src[i] + 1], *qe.up), F))[0]
    assert_bf16_adjacent(h[:, :F], h_ref, what="h")

    # a6: requantisation of the dumped h, bit-exact
    qh, sh = O.quantize_act(h[:, :F].astype(np.float32))
    idx2 = torch.from_numpy(act_row_index(rows, Fp, RB)).cuda()
    act2 = dump("act2").view(torch.int8)[idx2].cpu().numpy()
    s2 = dump("s2").view(torch.float32)[rows_t].cpu().numpy()
    assert np.array_equal(act2, qh)
    assert np.array_equal(s2, sh)

    # a7: down GEMM rows on identical INT8 inputs
    y2 = dump("y2").view(torch.float32).view(R, H)[rows_t].cpu().numpy()
    y2_ref = np.zeros((slots.size, H))
    for i, s in enumerate(slots):
        qe = experts[int(flat[s])]
        y2_ref[i] = O.w4a8_linear(qh[i:i + 1], sh[i:i + 1], *qe.down)[0]
    assert_close(y2, y2_ref, max_rel=1e-4, mae_rel=1e-5, what="y2")

    # a8 of the dumped rows, and the whole layer against the oracle, per sampled token
    out_s = out[torch.tensor(tokens).cuda()].view(torch.int16).cpu().numpy().view(np.uint16)
    out_s = synth.bf16_from_bits(out_s)
    comb = O.round_to_bf16(O.combine(y2.astype(np.float64), wts[tokens], np.arange(slots.size), len(tokens), k))
    assert_close(out_s, comb, max_rel=1e-2, mae_rel=1e-3, what="combine")
    ref = np.stack([O.token_forward(t, x, ids, wts, experts, F) for t in tokens])
    assert_close(out_s, ref, what="out")
    return tokens


def test_large_decode_layer_sampled(packed_384):
    """384 experts, top-8 Zipf(1.1) routing, 256 tokens, hidden 7168, expert ffn 2048."""
    tokens = run_and_check("large_decode", packed_384, extra_tokens=[])
    assert len(tokens) >= 3


def test_prefill_layer_sampled(packed_384):
    """384 experts, top-8 uniform routing, 16384 tokens, hidden 7168, expert ffn 2048."""
    tokens = run_and_check("prefill", packed_384, extra_tokens=[])
    assert len(tokens) >= 3
