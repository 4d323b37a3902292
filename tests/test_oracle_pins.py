"""Pins for the CPU oracle: values the pages print, closed forms, brute force and
independent formulations.  CPU only; these run before anything is compared with
the CUDA path, so that the oracle itself is known to be right."""

import itertools
import math

import numpy as np
import pytest

from oracle import w4a8_oracle as O
from w4a8_quantized_moe_token_b200 import synth


# --------------------------------------------------------------------------- #
# activation INT8 (symmetric, per token)
# --------------------------------------------------------------------------- #
def test_worked_example_tight_range(golden):
    g = golden("p3_worked_example.txt")
    v = np.float32(g["value"])
    row = np.array([[v, -0.5, 0.5, 0.1, 0.0]], dtype=np.float32)
    q, s = O.quantize_act(row)
    assert abs(float(s[0]) - float(g["scale_tight_approx"])) < 5e-6
    assert int(q[0, 0]) == int(g["code_tight"])
    deq = int(q[0, 0]) * float(s[0])
    assert abs(deq - float(g["dequant_tight_approx"])) < 5e-4
    assert abs(deq - float(v)) / float(v) < float(g["rel_error_tight_max"])
    # extremes map to the end codes, zero maps to zero
    assert q[0, 1] == -127 and q[0, 2] == 127 and q[0, 4] == 0


def test_worked_example_loose_range(golden):
    g = golden("p3_worked_example.txt")
    v = np.float32(g["value"])
    row = np.array([[v, -1.0, 1.0]], dtype=np.float32)
    q, s = O.quantize_act(row)
    opts = [int(c) for c in g["code_loose_options"].split(",")]
    assert int(q[0, 0]) in opts
    rel = abs(int(q[0, 0]) * float(s[0]) - float(v)) / float(v)
    # "approaches 2%": clearly worse than the tight range, at most a little over 2%
    assert 0.01 < rel < 0.025


def test_act_quant_roundtrip_bound_and_padding():
    rng = np.random.default_rng(1)
    x = synth.bf16_round(rng.standard_normal((37, 200)).astype(np.float32) * 3)
    x[5] = 0.0
    q, s = O.quantize_act(x)
    assert q.shape == (37, 256) and q.dtype == np.int8
    assert np.all(q[:, 200:] == 0)
    assert s[5] == 0 and np.all(q[5] == 0)
    err = np.abs(x - q[:, :200].astype(np.float64) * s[:, None])
    # half a step, plus the fp32 rounding of x/s (at most 127 * 2^-24 of a step)
    assert np.all(err <= s[:, None] * (0.5 + 1e-5))
    assert np.all(np.abs(q) <= 127)
    # the largest magnitude of every non-zero row lands on +-127
    nz = s > 0
    assert np.all(np.abs(q[nz]).max(axis=1) == 127)


def test_act_quant_ties_round_to_even():
    # 127 * 0.5 / 127 -> x/s = 0.5 exactly -> rint -> 0; 1.5 -> 2; 2.5 -> 2
    s_target = np.float32(1.0)
    row = np.array([[127.0, 0.5, 1.5, 2.5, -0.5, -1.5]], dtype=np.float32)
    q, s = O.quantize_act(row)
    assert s[0] == s_target
    assert list(q[0, :6]) == [127, 0, 2, 2, 0, -2]


# --------------------------------------------------------------------------- #
# weight INT4, asymmetric, group 128
# --------------------------------------------------------------------------- #
def _group_with(values):
    g = np.zeros(128, dtype=np.float32)
    g[: len(values)] = values
    return g[None, :]


def test_asym_int4_closed_form():
    # range [-0.5, 0.5]: scale = 1/15 (fp16 0.0666504), zero point = round(7.5018) = 8
    w = _group_with([-0.5, 0.5, 0.2, 0.0, -0.2])
    codes, scale, zp = O.quantize_weights(w)
    assert scale.dtype == np.float16 and zp.dtype == np.float16
    assert float(scale[0, 0]) == float(np.float16(np.float32(1.0) / np.float32(15.0)))
    assert float(zp[0, 0]) == 8.0
    assert list(codes[0, :5]) == [0, 15, 11, 8, 5]
    deq = O.dequantize_weights(codes, scale, zp)
    assert abs(deq[0, 2] - 0.2) < 1e-3  # 3 steps of 0.0666504
    assert deq[0, 3] == 0.0  # zero is exact (it maps to the zero point)
    # zero padding to the group is exact too
    assert np.all(codes[0, 5:] == 8) and np.all(deq[0, 5:] == 0.0)


def test_asym_int4_positive_only_group_includes_zero():
    # a group that does not straddle 0: range widened to [0, max] -> zp = 0
    w = _group_with([0.1, 0.3, 0.15])
    w[0, 3:] = 0.05
    codes, scale, zp = O.quantize_weights(w)
    assert float(zp[0, 0]) == 0.0
    assert codes[0, 1] == 15
    w2 = -w
    codes2, scale2, zp2 = O.quantize_weights(w2)
    assert float(zp2[0, 0]) == 15.0 and codes2[0, 1] == 0


def test_asym_int4_degenerate_group():
    codes, scale, zp = O.quantize_weights(np.zeros((2, 128), np.float32))
    assert np.all(scale == np.float16(1.0)) and np.all(zp == 0) and np.all(codes == 0)


def test_asym_int4_roundtrip_bound():
    rng = np.random.default_rng(7)
    w = synth.bf16_round((rng.standard_normal((64, 384)) * 0.02).astype(np.float32))
    w[3, :128] += 0.5  # a skewed group
    codes, scale, zp = O.quantize_weights(w)
    deq = O.dequantize_weights(codes, scale, zp)
    sc = np.repeat(scale.astype(np.float64), 128, axis=1)
    z = np.repeat(zp.astype(np.float64), 128, axis=1)
    raw = np.rint(w.astype(np.float32) / sc.astype(np.float32)) + z
    inside = (raw >= 0) & (raw <= 15)
    err = np.abs(w - deq)
    assert np.all(err[inside] <= sc[inside] / 2 * (1 + 1e-3))
    # clamped values sit at the ends of the range: at most one step off
    assert np.all(err <= sc * (1 + 1e-3))
    assert codes.max() <= 15


def test_sym_int4_closed_form():
    # [P3] section 2.1 symmetric form with b = 4: scale = max|w| / 7.  Group max 0.7 ->
    # scale fp16(0.1) = 0.0999755859375; 0.35 / 0.09998 = 3.5009 -> 4 (code 12);
    # -0.35 -> -4 (code 4); 0.2 -> 2.0005 -> 2 (code 10); 0.7 -> 7.0017 -> 7 (code 15);
    # -0.7 -> -7 (code 1); 0 -> 0 (code 8 = the zero point, exact)
    w = _group_with([0.7, -0.35, 0.35, 0.2, 0.0, -0.7])
    codes, scale, zp = O.quantize_weights_symmetric(w)
    assert float(scale[0, 0]) == float(np.float16(np.float32(0.7) / np.float32(7.0)))
    assert float(scale[0, 0]) == 0.0999755859375
    assert float(zp[0, 0]) == 8.0
    assert list(codes[0, :6]) == [15, 4, 12, 10, 8, 1]
    deq = O.dequantize_weights(codes, scale, zp)
    assert deq[0, 4] == 0.0 and np.all(deq[0, 6:] == 0.0)  # zero and the padding are exact
    assert abs(deq[0, 3] - 0.2) <= float(scale[0, 0]) / 2


def test_sym_int4_roundtrip_bound_and_symmetry():
    rng = np.random.default_rng(11)
    w = synth.bf16_round((rng.standard_normal((32, 256)) * 0.02).astype(np.float32))
    codes, scale, zp = O.quantize_weights_symmetric(w)
    assert codes.min() >= 1 and codes.max() <= 15 and np.all(zp == 8)
    deq = O.dequantize_weights(codes, scale, zp)
    sc = np.repeat(scale.astype(np.float64), 128, axis=1)
    assert np.all(np.abs(w - deq) <= sc / 2 * (1 + 1e-3))
    # the scheme is odd-symmetric: -w gives the mirrored codes and the same scales
    c2, s2, _ = O.quantize_weights_symmetric(-w)
    assert np.array_equal(s2, scale) and np.array_equal(c2.astype(int) - 8, -(codes.astype(int) - 8))
    # the largest magnitude of every group lands on +-7
    q = codes.astype(int) - 8
    for g in range(2):
        blk = w[:, g * 128:(g + 1) * 128]
        i = np.abs(blk).argmax(axis=1)
        assert np.all(np.abs(q[np.arange(32), g * 128 + i]) == 7)


def test_sym_int4_degenerate_group():
    codes, scale, zp = O.quantize_weights_symmetric(np.zeros((2, 128), np.float32))
    assert np.all(scale == np.float16(1.0)) and np.all(zp == 8) and np.all(codes == 8)


def test_percentile_range_closed_form_and_numpy():
    # one outlier in a group: sorted tail ... 0.1, 1.0 -> 99.9th percentile
    # = 0.1 + 0.873 * (1.0 - 0.1) = 0.8857 (position 0.999 * 127 = 126.873)
    rng = np.random.default_rng(5)
    v = synth.bf16_round((rng.uniform(-0.1, 0.1, size=(1, 128))).astype(np.float32))
    v[0, :2] = [-0.1, -0.1]
    v[0, 2] = 0.1
    v[0, 3] = 1.0
    v = np.clip(v, -0.1, 1.0)
    lo, hi = O.group_range_percentile(v)
    assert abs(float(hi[0]) - (0.1 + 0.873 * 0.9)) < 1e-6
    assert float(lo[0]) == np.float32(-0.1)  # the two lowest are equal
    # against numpy's percentile (linear interpolation) on random groups
    w = (rng.standard_normal((64, 128)) * 0.02).astype(np.float32)
    lo, hi = O.group_range_percentile(w)
    np.testing.assert_allclose(lo, np.percentile(w.astype(np.float64), 0.1, axis=1), rtol=1e-6, atol=1e-9)
    np.testing.assert_allclose(hi, np.percentile(w.astype(np.float64), 99.9, axis=1), rtol=1e-6, atol=1e-9)


def test_clip999_codes_and_outlier():
    rng = np.random.default_rng(9)
    w = synth.bf16_round((rng.standard_normal((8, 256)) * 0.02).astype(np.float32))
    w[2, 5] = 0.5  # an outlier far beyond the group's second largest value
    w = synth.bf16_round(w)
    c0, s0, z0 = O.quantize_weights(w)
    c1, s1, z1 = O.quantize_weights(w, clip999=True)
    # the clipped range is inside the min..max range: scales never grow
    assert np.all(s1.astype(np.float32) <= s0.astype(np.float32))
    # the outlier's group gets a much tighter scale and the outlier sits on code 15
    assert float(s1[2, 0]) < float(s0[2, 0])
    assert c1[2, 5] == 15
    # reconstruct the codes from the stored scale and zero point (R5)
    sf = np.repeat(s1.astype(np.float32), 128, axis=1)
    z = np.repeat(z1.astype(np.float32), 128, axis=1)
    assert np.array_equal(np.clip(np.rint(w / sf) + z, 0, 15).astype(np.uint8), c1)


def test_quantize_uses_fp16_scale_for_codes():
    # reconstructing the codes from the stored fp16 scale + zp reproduces them (R5)
    rng = np.random.default_rng(3)
    w = synth.bf16_round((rng.standard_normal((16, 256)) * 0.02).astype(np.float32))
    codes, scale, zp = O.quantize_weights(w)
    sf = np.repeat(scale.astype(np.float32), 128, axis=1)
    z = np.repeat(zp.astype(np.float32), 128, axis=1)
    again = np.clip(np.rint(w / sf) + z, 0, 15)
    assert np.array_equal(again.astype(np.uint8), codes)


# --------------------------------------------------------------------------- #
# nibble packing and group alignment
# --------------------------------------------------------------------------- #
def test_pack_low_nibble_first():
    assert O.pack_nibbles(np.array([1, 2], np.uint8)).tolist() == [0x21]
    row = np.arange(16, dtype=np.uint8)
    assert O.pack_nibbles(row).tolist() == [0x10, 0x32, 0x54, 0x76, 0x98, 0xBA, 0xDC, 0xFE]
    rng = np.random.default_rng(0)
    c = rng.integers(0, 16, size=(5, 256), dtype=np.uint8)
    assert np.array_equal(O.unpack_nibbles(O.pack_nibbles(c)), c)


def test_group_alignment_k200():
    assert O.padded_k(200) == 256 and O.padded_k(128) == 128 and O.padded_k(1) == 128
    rng = np.random.default_rng(5)
    w = synth.bf16_round((rng.standard_normal((4, 200)) * 0.02).astype(np.float32))
    codes, scale, zp = O.quantize_weights(w)
    assert codes.shape == (4, 256) and scale.shape == (4, 2)
    packed = O.pack_nibbles(codes)
    assert packed.shape == (4, 128)
    # group 1 starts on a whole byte: byte 64 holds codes 128 and 129
    assert np.array_equal(packed[:, 64] & 0xF, codes[:, 128])
    assert np.array_equal(packed[:, 64] >> 4, codes[:, 129])
    # the padding codes equal the zero point, so they add exactly 0 to group 1
    assert np.all(codes[:, 200:] == zp[:, 1:2].astype(np.uint8))
    qa = rng.integers(-127, 128, size=(3, 200)).astype(np.int8)
    acc = O.group_partials(O.pad_k(qa), codes, zp)
    manual = (qa[:, None, 128:200].astype(np.int64)
              * (codes[None, :, 128:200].astype(np.int64) - zp[None, :, 1:2].astype(np.int64))).sum(-1)
    assert np.array_equal(acc[:, :, 1], manual)


def test_scale_overhead_accounting(golden):
    g = golden("p2_scale_overhead.txt")
    gs = int(g["group_size"])
    per_group = 2 + 2  # one fp16 scale + one fp16 zero point
    assert per_group == int(g["param_bytes_per_group"])
    extra = per_group / gs
    assert extra == float(g["extra_bytes_per_weight"])
    ratio = 2.0 / (0.5 + extra)
    assert abs(ratio - float(g["compression_vs_fp16_approx"])) < 0.05
    # the oracle's stored format has exactly that size
    rng = np.random.default_rng(0)
    codes, scale, zp = O.quantize_weights(rng.standard_normal((8, 1024)).astype(np.float32) * 0.02)
    nbytes = O.pack_nibbles(codes).nbytes + scale.nbytes + zp.nbytes
    assert nbytes / codes.size == 0.5 + extra


# --------------------------------------------------------------------------- #
# INT32 per-group partials and the scale fold
# --------------------------------------------------------------------------- #
def test_group_partials_brute_force():
    rng = np.random.default_rng(11)
    for M, N, K in [(1, 1, 128), (3, 4, 256), (4, 2, 130)]:
        Kp = O.padded_k(K)
        qa = O.pad_k(rng.integers(-127, 128, size=(M, K)).astype(np.int8))
        codes = rng.integers(0, 16, size=(N, Kp)).astype(np.uint8)
        zp = rng.integers(0, 16, size=(N, Kp // 128)).astype(np.float16)
        acc = O.group_partials(qa, codes, zp)
        for m in range(M):
            for n in range(N):
                for g in range(Kp // 128):
                    s = 0
                    for kk in range(g * 128, (g + 1) * 128):
                        s += int(qa[m, kk]) * (int(codes[n, kk]) - int(zp[n, g]))
                    assert acc[m, n, g] == s


def test_group_partials_extremes_fit_int32():
    qa = np.full((1, 128), 127, np.int8)
    codes = np.full((1, 128), 15, np.uint8)
    acc = O.group_partials(qa, codes, np.zeros((1, 1), np.float16))
    assert acc[0, 0, 0] == 128 * 127 * 15 == 243840
    acc = O.group_partials(-qa, np.zeros((1, 128), np.uint8), np.full((1, 1), 15, np.float16))
    assert acc[0, 0, 0] == 243840
    assert 243840 < 2 ** 31 and 243840 > 2 ** 15  # INT16 would overflow, INT32 does not


def test_linear_textbook_special_case():
    # scale 1, zero point 0: the W4A8 linear is a plain integer matmul times sa
    rng = np.random.default_rng(2)
    qa = rng.integers(-127, 128, size=(5, 256)).astype(np.int8)
    codes = rng.integers(0, 16, size=(6, 256)).astype(np.uint8)
    sa = rng.random(5).astype(np.float32)
    ones = np.ones((6, 2), np.float16)
    y = O.w4a8_linear(qa, sa, codes, ones, np.zeros((6, 2), np.float16))
    ref = sa.astype(np.float64)[:, None] * (qa.astype(np.int64) @ codes.astype(np.int64).T)
    assert np.array_equal(y, ref)


def test_linear_equals_dequantized_matmul():
    # an independent formulation: dequantise both operands, multiply in fp64
    rng = np.random.default_rng(4)
    x = synth.bf16_round(rng.standard_normal((7, 300)).astype(np.float32))
    w = synth.bf16_round((rng.standard_normal((9, 300)) * 0.02).astype(np.float32))
    qa, sa = O.quantize_act(x)
    codes, scale, zp = O.quantize_weights(w)
    y = O.w4a8_linear(qa, sa, codes, scale, zp)
    a_deq = qa.astype(np.float64) * sa.astype(np.float64)[:, None]
    ref = a_deq @ O.dequantize_weights(codes, scale, zp).T
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-15)
    # and it approximates the unquantised product (4-bit weights: ~10% rms error)
    exact = x.astype(np.float64) @ w.astype(np.float64).T
    rms = lambda a: float(np.sqrt(np.mean(a * a)))
    assert rms(y - exact) < 0.2 * rms(exact)


@pytest.mark.parametrize("group", [64, 256])
def test_other_group_sizes(group):
    # [P1] section 5 names group sizes 128 or 256; [P2] section 2.1 trades accuracy
    # against scale storage.  Brute-force partials, the dequantised formulation, the
    # half-step bound, padding to the group and the storage accounting per group size.
    rng = np.random.default_rng(group)
    K = 300
    Kp = O.padded_k(K, group)
    assert Kp == -(-K // group) * group
    x = synth.bf16_round(rng.standard_normal((3, K)).astype(np.float32))
    w = synth.bf16_round((rng.standard_normal((5, K)) * 0.02).astype(np.float32))
    qa, sa = O.quantize_act(x, group)
    codes, scale, zp = O.quantize_weights(w, group=group)
    assert codes.shape == (5, Kp) and scale.shape == (5, Kp // group) and qa.shape == (3, Kp)
    deq = O.dequantize_weights(codes, scale, zp)
    sc = np.repeat(scale.astype(np.float64), group, axis=1)
    assert np.all(np.abs(O.pad_k(w, group) - deq) <= sc / 2 * (1 + 1e-3))
    assert np.all(deq[:, K:] == 0.0)  # padding is exact
    acc = O.group_partials(qa, codes, zp)
    for m, n, g in [(0, 0, 0), (2, 4, Kp // group - 1), (1, 2, 0)]:
        ref = sum(int(qa[m, kk]) * (int(codes[n, kk]) - int(zp[n, g])) for kk in range(g * group, (g + 1) * group))
        assert acc[m, n, g] == ref
    y = O.w4a8_linear(qa, sa, codes, scale, zp)
    ref = (qa.astype(np.float64) * sa.astype(np.float64)[:, None]) @ deq.T
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-15)
    # 4 bytes of fp16 scale + zero point per group: 4 / group bytes per weight
    assert scale.nbytes + zp.nbytes == 4 * codes.size // group
    cs, ss, zs = O.quantize_weights_symmetric(w, group)
    assert ss.shape == scale.shape and np.all(zs == 8) and cs.max() <= 15


# --------------------------------------------------------------------------- #
# routing and permutation
# --------------------------------------------------------------------------- #
def test_route_topk_brute_force_and_ties():
    rng = np.random.default_rng(9)
    lg = synth.bf16_round(rng.standard_normal((20, 6)).astype(np.float32))
    lg[0] = [1.0, 2.0, 2.0, 0.5, 2.0, -1.0]  # three-way tie
    ids, w = O.route_topk(lg, 3)
    assert ids[0].tolist() == [1, 2, 4]
    for t in range(lg.shape[0]):
        # brute force: e is chosen iff fewer than k experts rank strictly before it
        chosen = [e for e in range(6)
                  if sum(1 for f in range(6) if lg[t, f] > lg[t, e] or (lg[t, f] == lg[t, e] and f < e)) < 3]
        assert sorted(ids[t].tolist()) == chosen
        p = np.exp(lg[t].astype(np.float64) - lg[t].max())
        p /= p.sum()
        np.testing.assert_allclose(w[t], p[ids[t]], rtol=1e-14)
        assert np.all(np.diff(lg[t, ids[t]]) <= 0)


def test_permute_bijection_and_stability():
    rng = np.random.default_rng(12)
    T, k, E = 50, 3, 7
    ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    counts, offs, perm, inv = O.permute(ids, E)
    assert counts.sum() == T * k and offs[-1] == T * k
    assert np.array_equal(np.sort(perm), np.arange(T * k))
    assert np.array_equal(perm[inv], np.arange(T * k))
    flat = ids.reshape(-1)
    for e in range(E):
        seg = perm[offs[e]:offs[e + 1]]
        assert np.all(flat[seg] == e)
        assert np.all(np.diff(seg) > 0)  # slot order kept


def test_expected_distinct_experts_pages_values(golden):
    g = golden("p4_expected_experts.txt")
    E = int(g["experts"])
    for B in (1, 2, 4):
        assert f"{O.expected_distinct_experts(E, B):.6f}" == g[f"batch_{B}"]


def test_permutation_histogram_matches_distinct_expert_identity(golden):
    # exhaustive: over all E^B top-1 routings of B tokens, the mean number of
    # experts with a non-zero count in the oracle's permutation equals 8(1-(7/8)^B)
    g = golden("p4_expected_experts.txt")
    E = int(g["experts"])
    for B in (1, 2, 4):
        total = 0
        for route in itertools.product(range(E), repeat=B):
            counts, _, _, _ = O.permute(np.array(route, np.int32)[:, None], E)
            total += int(np.count_nonzero(counts))
        mean = total / E ** B
        assert abs(mean - O.expected_distinct_experts(E, B)) < 1e-12
        assert f"{mean:.6f}" == g[f"batch_{B}"]


# --------------------------------------------------------------------------- #
# SwiGLU, combine, and the whole layer against an independent formulation
# --------------------------------------------------------------------------- #
def test_swiglu_values():
    assert O.silu(np.array([0.0]))[0] == 0.0
    assert abs(O.silu(np.array([30.0]))[0] - 30.0) < 1e-9
    assert abs(O.silu(np.array([-30.0]))[0]) < 1e-9
    y = np.zeros((1, 4))
    y[0, 0], y[0, 2] = 1.0, 2.0  # F = 2: gate col 0, up col 2
    h = O.swiglu(y, 2)
    assert abs(h[0, 0] - 2.0 / (1.0 + math.exp(-1.0))) < 1e-15 and h[0, 1] == 0.0


def test_combine_by_hand():
    y2 = np.array([[1.0, 2.0], [10.0, 20.0], [100.0, 200.0]])
    inv = np.array([2, 0, 1])  # token0 slot0 -> row2, slot1 -> row0; token1? T=1,k=3 here
    w = np.array([[0.5, 0.25, 0.125]])
    out = O.combine(y2, w, inv, 1, 3)
    assert out.tolist() == [[0.5 * 100 + 0.25 * 1 + 0.125 * 10, 0.5 * 200 + 0.25 * 2 + 0.125 * 20]]


def _tiny_layer(seed=0, T=9, E=4, k=2, H=256, F=128):
    x = synth.activations(seed, T, H)
    ids, w = synth.synthetic_routing(seed, T, E, k, "uniform")
    experts = {}
    for e in range(E):
        experts[e] = O.QuantExpert(synth.expert_weight(seed, e, "up", 2 * F, H),
                                   synth.expert_weight(seed, e, "down", H, F))
    return x, ids, w, experts


@pytest.mark.parametrize("group", [128, 64, 256])
def test_moe_forward_equals_per_token_dequantized_formulation(group):
    T, E, k, H, F = 9, 4, 2, 256, 128
    x, ids, w, experts = _tiny_layer(T=T, E=E, k=k, H=H, F=F)
    if group != 128:  # the same weights quantised with another group size
        experts = {e: O.QuantExpert(synth.expert_weight(0, e, "up", 2 * F, H), synth.expert_weight(0, e, "down", H, F),
                                    group=group) for e in experts}
        assert experts[0].up[1].shape == (2 * F, H // group)
    out = O.moe_forward(x, ids, w, experts, E, F)
    xq, xs = O.quantize_act(x, group)
    for t in range(T):
        acc = np.zeros(H)
        a = xq[t].astype(np.float64) * float(xs[t])
        for j in range(k):
            qe = experts[int(ids[t, j])]
            wu = O.dequantize_weights(*qe.up)
            wd = O.dequantize_weights(*qe.down)
            yu = wu @ a
            # h is handed on in bf16 ([P1] §4.3 step 4)
            hh = O.round_to_bf16(yu[:F] / (1 + np.exp(-yu[:F])) * yu[F:]).astype(np.float32)
            qh, sh = O.quantize_act(hh[None, :], group)
            acc += float(w[t, j]) * (wd @ (qh[0].astype(np.float64) * float(sh[0])))
        # the layer's output is rounded to bf16: within half a bf16 ulp of the fp64 value
        assert np.all(np.abs(out[t] - acc) <= np.abs(acc) * 2.0 ** -8 + 1e-30)
        np.testing.assert_allclose(O.token_forward(t, x, ids, w, experts, F), out[t], rtol=1e-12, atol=1e-15)


def test_planted_mistakes_are_caught():
    """A dropped zero point, a swapped nibble order or a transposed scale must fail the pins."""
    rng = np.random.default_rng(0)
    w = synth.bf16_round((rng.standard_normal((4, 256)) * 0.02).astype(np.float32))
    codes, scale, zp = O.quantize_weights(w)
    deq = O.dequantize_weights(codes, scale, zp)
    # dropped zp: error no longer within one step
    wrong = codes.astype(np.float64) * np.repeat(scale.astype(np.float64), 128, axis=1)
    assert np.abs(wrong - w).max() > np.abs(deq - w).max() * 10
    # swapped nibbles
    swapped = ((codes[:, 0::2] << 4) | codes[:, 1::2]).astype(np.uint8)
    assert not np.array_equal(swapped, O.pack_nibbles(codes))
    # transposed scale use
    qa, sa = O.quantize_act(synth.bf16_round(rng.standard_normal((4, 256)).astype(np.float32)))
    acc = O.group_partials(qa, codes, zp)
    good = O.w4a8_linear(qa, sa, codes, scale, zp, acc)
    bad = sa[:, None] * np.einsum("mng,mg->mn", acc.astype(np.float64), scale.astype(np.float64))
    assert np.abs(good - bad).max() > 1e-6


def test_round_to_bf16_against_library_rounding():
    # independent: torch's float32 -> bfloat16 conversion is round-half-to-even; on
    # fp64 values that are exactly float32 the two single roundings must agree
    import torch
    rng = np.random.default_rng(8)
    v = (rng.standard_normal(20000) * 10.0 ** rng.integers(-6, 6, 20000)).astype(np.float32).astype(np.float64)
    ties = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 0.0, 3.0])  # exact midpoints
    v = np.concatenate([v, ties])
    ref = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(O.round_to_bf16(v), ref)
    assert O.round_to_bf16(np.array([1.0 + 2.0 ** -8]))[0] == 1.0  # tie to even
    assert O.round_to_bf16(np.array([1.0 + 3 * 2.0 ** -8]))[0] == 1.0 + 2.0 ** -6


# --------------------------------------------------------------------------- #
# INT8 KV cache (static per-head scales)
# --------------------------------------------------------------------------- #
def test_kv_int8_worked_example_per_head():
    # the primer's worked example per head: calibrated range 0.5 -> s = 0.5/127,
    # 0.2 -> 51 -> 51 * s = 0.20079 (bf16: 0.2001953125... rounding of 0.2007874)
    x = np.zeros((2, 2, 4), np.float32)
    x[0, 0] = [0.5, -0.5, 0.2, 0.0]
    x[1, 1] = [1.0, 0.2, -0.2, 0.1]
    s = O.kv_calibrate(x)
    assert s[0] == np.float32(0.5) / np.float32(127) and s[1] == np.float32(1.0) / np.float32(127)
    q = O.kv_quantize(x, s)
    assert list(q[0, 0]) == [127, -127, 51, 0]
    assert list(q[1, 1]) == [127, 25, -25, 13]  # 25.4 -> 25 (page: "25 or 26"), 12.7 -> 13
    dq = O.kv_dequantize(q, s)
    assert dq[0, 0, 2] == np.float32(synth.bf16_round(np.array([51 * (0.5 / 127)], np.float32))[0])
    assert abs(dq[0, 0, 2] - 0.2) < 2e-3


def test_kv_int8_roundtrip_saturation_and_zero_head():
    rng = np.random.default_rng(21)
    calib = synth.bf16_round(rng.standard_normal((64, 4, 32)).astype(np.float32))
    calib[:, 3] = 0.0  # an all-zero head
    s = O.kv_calibrate(calib)
    assert s[3] == 0
    x = synth.bf16_round(rng.standard_normal((16, 4, 32)).astype(np.float32) * 0.5)
    x[0, 0, 0] = 100.0  # beyond the calibrated range: saturates
    q = O.kv_quantize(x, s)
    assert q[0, 0, 0] == 127 and np.all(q[:, 3] == 0)
    dq = O.kv_dequantize(q, s)
    inside = np.abs(x) <= (127 * s)[None, :, None]
    sc = np.broadcast_to(s[None, :, None], x.shape)
    # half a step of quantisation plus the bf16 rounding of the result
    err = np.abs(dq - x)
    assert np.all(err[inside] <= sc[inside] / 2 + np.abs(x[inside]) * 2.0 ** -8 + 1e-12)
    # the brute-force definition, element by element, on a few values
    for (t, h, d) in [(1, 0, 3), (5, 2, 31), (15, 1, 0)]:
        ref = max(-127, min(127, int(np.rint(np.float32(x[t, h, d]) / s[h]))))
        assert q[t, h, d] == ref


# --------------------------------------------------------------------------- #
# W4A16 comparison layer
# --------------------------------------------------------------------------- #
def test_w4a16_linear_brute_force():
    rng = np.random.default_rng(31)
    x = synth.bf16_round(rng.standard_normal((3, 200)).astype(np.float32))
    w = synth.bf16_round((rng.standard_normal((4, 200)) * 0.02).astype(np.float32))
    codes, scale, zp = O.quantize_weights(w)
    y = O.w4a16_linear(x, codes, scale, zp)
    for m in range(3):
        for n in range(4):
            ref = 0.0
            for kk in range(200):
                g = kk // 128
                ref += float(x[m, kk]) * (int(codes[n, kk]) - float(zp[n, g])) * float(scale[n, g])
            assert abs(y[m, n] - ref) <= 1e-12 * max(1.0, abs(ref))


def test_w4a16_reduces_to_w4a8_on_int8_exact_activations():
    # rows that are exactly s * q with q in [-127, 127] (the row maximum at 127) and s a
    # power of two are quantised by the activation quantiser without loss, so the
    # W4A16 layer (fp64 matmul on dequantised weights) and the W4A8 layer (exact INT32
    # group partials, then the fold) must agree
    rng = np.random.default_rng(32)
    q = rng.integers(-127, 128, size=(5, 256))
    q[:, 0] = 127
    s = np.float32(2.0 ** -6)
    x = (q.astype(np.float32) * s).astype(np.float32)
    w = synth.bf16_round((rng.standard_normal((8, 256)) * 0.02).astype(np.float32))
    codes, scale, zp = O.quantize_weights(w)
    qa, sa = O.quantize_act(x)
    assert np.array_equal(qa[:, :256], q) and np.all(sa == s)  # lossless
    np.testing.assert_allclose(O.w4a16_linear(x, codes, scale, zp), O.w4a8_linear(qa, sa, codes, scale, zp),
                               rtol=1e-12, atol=1e-15)


def test_w4a16_layer_single_expert_top1():
    rng = np.random.default_rng(33)
    T, H, F = 6, 256, 128
    x = synth.bf16_round(rng.standard_normal((T, H)).astype(np.float32))
    qe = O.QuantExpert(synth.bf16_round((rng.standard_normal((2 * F, H)) * 0.02).astype(np.float32)),
                       synth.bf16_round((rng.standard_normal((H, F)) * 0.02).astype(np.float32)))
    ids = np.zeros((T, 1), np.int32)
    out = O.moe_forward_w4a16(x, ids, np.ones((T, 1)), {0: qe}, 1, F)
    direct = O.round_to_bf16(O.w4a16_expert_forward(x, qe, F))
    assert np.array_equal(out, direct)
