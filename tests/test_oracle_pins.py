"""Pins of the CPU oracle to facts outside itself (no GPU).

Each check ties the oracle to something the pages or mathematics fix:
counts stated on the pages, brute force over all 32 patterns, closed forms,
an independent rounding routine (Python's ``struct``), hand-derived golden
blocks, and exact rational arithmetic.  A plausible slip in the oracle (a
wrong sign, lane, nibble or bit order, a dropped term in the scale fit) makes
at least one of them fail; ``test_planted_mistakes_are_caught`` shows that for
a few such slips.
"""

import itertools
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------------------
# Format facts stated on the pages
# ---------------------------------------------------------------------------


def test_codebook_has_32_distinct_one_zero_patterns():
    # 4 zero positions x 8 sign combinations = 32 patterns, values in {-1, 0, +1}
    # with exactly one zero (lemmy post, "Four weights, five bits").
    cb = oracle.codebook()
    assert cb.shape == (32, 4)
    assert len({tuple(r) for r in cb}) == 32
    for row in cb:
        assert (row == 0).sum() == 1
        assert set(np.abs(row[row != 0]).tolist()) == {1}
    # every (zero lane, signs of the other three) combination appears once
    seen = set()
    for row in cb:
        z = int(np.flatnonzero(row == 0)[0])
        seen.add((z, tuple(int(v) for v in row if v != 0)))
    assert seen == {(z, s) for z in range(4) for s in itertools.product((-1, 1), repeat=3)}


def test_select_bit_is_a_table_of_16():
    # 4-bit code plus a 1-bit table-select into 32 entries ("How STQ1_0 works"):
    # each table value of t holds 16 distinct patterns; reading: table 1 = -table 0.
    cb = oracle.codebook()
    assert len({tuple(r) for r in cb[:16]}) == 16
    assert np.array_equal(cb[16:], -cb[:16])


def test_storage_rate():
    # 42 bytes per 256 weights = 1.3125 bits/weight; 5 bits per group = 1.25 bits/weight.
    assert oracle.BLOCK_BYTES * 8 / oracle.BLOCK_WEIGHTS == 1.3125
    assert 5 * oracle.GROUPS_PER_BLOCK == (oracle.BLOCK_BYTES - 2) * 8
    assert 5 / 4 == 1.25
    assert oracle.packed_size(512, 2048) == 512 * 8 * 42
    w = np.ones((3, 512), np.float32)
    assert oracle.encode_plain(w).size == 3 * 2 * 42


def test_roundtrip_all_codes_and_scales():
    # Every code, at 8 random scales plus the extremes, survives encode(decode(.)).
    scales = list(workloads.code_sweep_scales())
    specials = [2.0 ** -24, 65504.0, 1.0]
    for d in scales + specials:
        d_bits = oracle.fp16_bits(np.array([d]))[0]
        dv = float(oracle.fp16_value(d_bits))
        codes = np.tile(np.arange(32, dtype=np.uint8), 2)[None, :]
        packed = oracle.pack_blocks(np.array([d_bits]), codes)
        w = oracle.decode(packed, 1, 256)
        # decoded values are exactly +/-d or 0 with one zero per group
        g = w.reshape(64, 4)
        assert np.all((g == 0).sum(axis=1) == 1)
        assert set(np.unique(np.abs(g[g != 0]))) == {dv}
        again = oracle.encode_plain(w.astype(np.float32))
        assert np.array_equal(again, packed), d
    # d = 0: every weight decodes to zero
    packed0 = oracle.pack_blocks(np.array([0], np.uint16), np.arange(64, dtype=np.uint8) % 32)
    assert np.all(oracle.decode(packed0, 1, 256) == 0)


def test_layout_byte_offsets():
    # layout reading: d at bytes 0-1, nibble of group g at qs[g>>1] (even g low),
    # select bit of g at qh[g>>3] bit g&7.
    for g in range(64):
        for code in (1, 16, 31):
            codes = np.zeros((1, 64), np.uint8)
            codes[0, g] = code
            b = oracle.pack_blocks(np.array([0x1234], np.uint16), codes)
            assert b[0] == 0x34 and b[1] == 0x12
            nib = code & 0xF
            exp_qs = np.zeros(32, np.uint8)
            exp_qs[g >> 1] = nib << (4 * (g & 1))
            exp_qh = np.zeros(8, np.uint8)
            exp_qh[g >> 3] = ((code >> 4) & 1) << (g & 7)
            assert np.array_equal(b[2:34], exp_qs)
            assert np.array_equal(b[34:42], exp_qh)


# ---------------------------------------------------------------------------
# Golden worked examples (hand-derived; see tests/golden/README.md)
# ---------------------------------------------------------------------------


def _read_golden(name):
    kv = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if "=" in line:
                k, v = (s.strip() for s in line.split("=", 1))
                kv[k] = v
    return kv


def _floats(s):
    return [float(v) for v in s.split()]


@pytest.mark.parametrize("name", ["plain_uniform_a.txt", "plain_uniform_b.txt"])
def test_golden_plain_uniform(name):
    kv = _read_golden(name)
    w = np.tile(np.array(_floats(kv["group"]), np.float32), 64)[None, :]
    packed = oracle.encode_plain(w)
    assert packed.tobytes().hex() == kv["bytes"]
    dec = oracle.decode(packed, 1, 256).reshape(64, 4)
    assert np.array_equal(dec, np.tile(_floats(kv["decoded_group"]), (64, 1)))


def test_golden_plain_bit_order():
    kv = _read_golden("plain_bit_order.txt")
    groups = np.tile(np.array(_floats(kv["other"]), np.float32), (64, 1))
    for g in (0, 1, 3):
        groups[g] = _floats(kv[f"group{g}"])
    packed = oracle.encode_plain(groups.reshape(1, 256))
    assert packed.tobytes().hex() == kv["bytes"]


def test_golden_sherry_moves_zero():
    kv = _read_golden("sherry_moves_zero.txt")
    w = np.tile(np.array(_floats(kv["group"]), np.float32), 64)[None, :]
    h = np.tile(np.array(_floats(kv["h_group"]), np.float32), 64)
    assert oracle.encode_sherry(w, h, rounds=3).tobytes().hex() == kv["bytes"]
    assert oracle.encode_plain(w).tobytes().hex() == kv["plain_bytes"]


# ---------------------------------------------------------------------------
# Brute force over the 32 patterns
# ---------------------------------------------------------------------------


def _best_pattern_errors(wg, hg, d):
    """For each group, the weighted squared error of all 32 patterns at scale d."""
    cb = oracle.codebook().astype(np.float64)            # [32, 4]
    r = wg[:, None, :] - d * cb[None, :, :]             # [G, 32, 4]
    return np.sum(hg[:, None, :] * r * r, axis=2)       # [G, 32]


def test_plain_encoder_is_the_best_pattern_at_amax_scale():
    # With d fixed at amax, the chosen pattern minimises the unweighted squared error
    # over all 32 patterns (ternary rounding with one forced zero).
    rng = np.random.default_rng(123)
    w = (rng.standard_normal((6, 512)) * 0.02).astype(np.float32)
    packed = oracle.encode_plain(w)
    d_bits, codes = oracle.unpack_blocks(packed)
    d = oracle.fp16_value(d_bits)
    blocks = w.reshape(-1, 64, 4).astype(np.float64)
    for b in range(blocks.shape[0]):
        err = _best_pattern_errors(blocks[b], np.ones((64, 4)), d[b])
        chosen = err[np.arange(64), codes[b]]
        assert np.all(chosen <= err.min(axis=1) * (1 + 1e-12) + 1e-30)


def test_sherry_zero_choice_matches_brute_force():
    # In each round, with d fixed at that round's fit, each group's new zero lane
    # gives the least weighted error among all 32 patterns.
    rng = np.random.default_rng(7)
    w = (rng.standard_normal((4, 512)) * 0.03).astype(np.float32)
    h = rng.uniform(0.05, 20.0, size=512).astype(np.float32)
    _, tr = oracle.encode_sherry(w, h, rounds=3, trace=True)
    blocks = w.reshape(-1, 64, 4).astype(np.float64)
    hb = tr["h_blocks"].reshape(-1, 64, 4)
    cb = oracle.codebook()
    for d, z in tr["rounds"][1:]:
        for b in range(blocks.shape[0]):
            err = _best_pattern_errors(blocks[b], hb[b], d[b])
            best = err.min(axis=1)
            # the pattern with zero lane z and signs of w
            codes = oracle.codes_from_choice(z[b][None, :], blocks[b][None])[0]
            chosen = err[np.arange(64), codes]
            assert np.all(chosen <= best * (1 + 1e-12) + 1e-30)
            assert np.all(cb[codes][np.arange(64), z[b]] == 0)


def test_wls_scale_is_the_least_squares_minimiser():
    # Final d is the stationary point of sum h (w - d s)^2 for the final codes:
    # the derivative vanishes, and a dense scan finds nothing lower.
    rng = np.random.default_rng(11)
    w = (rng.standard_normal((3, 256)) * rng.uniform(0.005, 0.05, (3, 1))).astype(np.float32)
    h = rng.uniform(0.1, 5.0, size=256).astype(np.float32)
    _, tr = oracle.encode_sherry(w, h, rounds=3, trace=True)
    z = tr["rounds"][-1][1]
    d = tr["d_final"]
    blocks = w.reshape(-1, 64, 4).astype(np.float64)
    hb = tr["h_blocks"]
    for b in range(3):
        lanes = np.arange(4)[None, :] != z[b][:, None]
        s = np.where(lanes, np.sign(blocks[b]), 0.0).reshape(-1)
        ww = blocks[b].reshape(-1)
        grad = np.sum(hb[b] * (ww - d[b] * s) * s)
        assert abs(grad) <= 1e-12 * np.sum(hb[b] * np.abs(ww))
        f = lambda dd: np.sum(hb[b] * (ww - dd * s) ** 2)  # noqa: E731
        scan = np.linspace(0.5 * d[b], 1.5 * d[b], 2001)
        assert f(d[b]) <= min(f(v) for v in scan) + 1e-15


def test_sherry_objective_never_increases():
    # Both half-steps are exact minimisers, so the weighted error is monotone.
    w, h, _ = workloads.decode_gemv_inputs(n=8, k=1024)
    _, tr = oracle.encode_sherry(w, h, rounds=3, trace=True)
    blocks = w.reshape(-1, 64, 4)
    hb = tr["h_blocks"]
    hist = tr["rounds"]
    prev = None
    for r in range(1, len(hist)):
        d, z = hist[r]
        z_prev = hist[r - 1][1]
        e_fit = oracle.weighted_error(blocks, hb, d, z_prev)     # after the d-fit
        e_zero = oracle.weighted_error(blocks, hb, d, z)         # after the zero choice
        if prev is not None:
            assert np.all(e_fit <= prev * (1 + 1e-12))
        assert np.all(e_zero <= e_fit * (1 + 1e-12))
        prev = e_zero


def test_uniform_importance_reduces_to_plain_zero_lane_and_mean_scale():
    # h = 1: zeroing cost d(2|w| - d) grows with |w|, so the zero lane is E0's,
    # and d is the mean |w| over the non-zero lanes.
    rng = np.random.default_rng(5)
    w = (rng.standard_normal((5, 768)) * 0.02).astype(np.float32)
    _, tr = oracle.encode_sherry(w, None, rounds=3, trace=True)
    z0 = np.argmin(np.abs(w.reshape(-1, 64, 4)), axis=2)
    assert np.array_equal(tr["rounds"][-1][1], z0)
    aw = np.abs(w.reshape(-1, 64, 4)).astype(np.float64)
    nz = np.arange(4)[None, None, :] != z0[:, :, None]
    mean = np.array([Fraction(0)] * aw.shape[0])
    for b in range(aw.shape[0]):
        vals = aw[b][nz[b]]
        mean[b] = sum(Fraction(float(v)) for v in vals) / len(vals)
    assert np.allclose(tr["d_final"], mean.astype(float), rtol=1e-14, atol=0)


def test_error_reduction_is_of_the_pages_order():
    # Context, not a hard pin: the pages report ~90% lower weighted error than
    # the amax encoder after three rounds on real expert rows; synthetic rows
    # should land in the same region.
    w, h, _ = workloads.decode_gemv_inputs(n=64, k=2048)
    blocks = w.reshape(-1, 64, 4)
    hb = np.broadcast_to(h.astype(np.float64).reshape(1, -1), w.shape).reshape(-1, 256)
    def err(packed):
        wh = oracle.decode(packed, *w.shape)
        return float(np.sum(hb.reshape(w.shape) * (w.astype(np.float64) - wh) ** 2))
    e0 = err(oracle.encode_plain(w))
    e1 = err(oracle.encode_sherry(w, h, rounds=3))
    assert 0.75 < 1 - e1 / e0 < 0.99
    assert blocks.shape[0] > 0


# ---------------------------------------------------------------------------
# Rounding
# ---------------------------------------------------------------------------


def test_fp16_rounding_matches_struct_half():
    # Python's struct 'e' format rounds a double to binary16 with ties to even,
    # independently of NumPy.
    allh = np.arange(0, 0x7C00, dtype=np.uint16)              # every finite positive half
    vals = allh.view(np.float16).astype(np.float64)
    assert np.array_equal(oracle.fp16_bits(vals), allh)
    rng = np.random.default_rng(3)
    xs = np.concatenate([
        rng.uniform(0, 65504, 2000), np.exp(rng.uniform(np.log(1e-8), np.log(6e4), 20000)),
        # exact halfway points between neighbouring halves: ties go to even
        (vals[:-1] + vals[1:]) / 2,
    ])
    got = oracle.fp16_bits(xs)
    exp = np.array([oracle.half_from_struct(float(x)) for x in xs], dtype=np.uint16)
    assert np.array_equal(got, exp)
    assert np.array_equal(oracle.fp16_bits(-xs[:100]), exp[:100] | 0x8000)


def test_fp16_saturates_and_rejects_non_finite():
    assert oracle.fp16_bits(np.array([65519.0, 65520.0, 1e30]))[1:].tolist() == [0x7BFF, 0x7BFF]
    assert oracle.fp16_bits(np.array([65519.0]))[0] == 0x7BFF
    for bad in (np.nan, np.inf):
        with pytest.raises(oracle.OracleValueError):
            oracle.fp16_bits(np.array([bad]))
    with pytest.raises(oracle.OracleValueError):
        oracle.encode_plain(np.full((1, 256), np.nan, np.float32))


def test_bf16_dequant_matches_torch_cast():
    torch = pytest.importorskip("torch")
    w = workloads.gaussian_matrix(16, 512, 0.02, seed=99)
    packed = oracle.encode_plain(w)
    got = oracle.dequant_bf16(packed, 16, 512)
    ref = torch.from_numpy(oracle.decode(packed, 16, 512).astype(np.float32)).to(torch.bfloat16)
    ref_bits = ref.view(torch.int16).numpy().view(np.uint16)
    ref_bits = np.where(ref_bits == 0x8000, 0, ref_bits)   # zero lanes are stored as +0.0
    assert np.array_equal(got, ref_bits)
    assert not np.any(got == 0x8000)


# ---------------------------------------------------------------------------
# Contractions
# ---------------------------------------------------------------------------


def test_gemv_closed_form_all_code_zero():
    # Code 0 is (0, +, +, +): y = d * sum over groups of x[4g+1] + x[4g+2] + x[4g+3].
    d_bits = oracle.fp16_bits(np.array([0.375]))
    packed = oracle.pack_blocks(d_bits, np.zeros((1, 64), np.uint8))
    x = workloads.activations_bf16(1, 256, seed=42)
    xf = oracle.bf16_to_f64(x).reshape(64, 4)
    y = oracle.gemv(packed, x, 1, 256)
    assert y[0, 0] == 0.375 * float(np.sum(xf[:, 1:]))


def test_gemv_one_hot_returns_columns():
    w = workloads.gaussian_matrix(7, 512, 0.02, seed=8)
    packed = oracle.encode_plain(w)
    dense = oracle.decode(packed, 7, 512)
    for col in (0, 3, 255, 256, 511):
        x = np.zeros((1, 512), np.float32)
        x[0, col] = 1.0
        y = oracle.gemv(packed, workloads.bf16_bits_from_f32(x), 7, 512)
        assert np.array_equal(y[0], dense[:, col])


def test_gemv_matches_exact_rational_sum():
    w = workloads.gaussian_matrix(3, 256, 0.05, seed=21)
    packed = oracle.encode_plain(w)
    x = workloads.activations_bf16(2, 256, seed=22)
    y = oracle.gemv(packed, x, 3, 256)
    d_bits, codes = oracle.unpack_blocks(packed)
    cb = oracle.codebook()
    xf = oracle.bf16_to_f64(x)
    for t in range(2):
        for j in range(3):
            d = Fraction(float(oracle.fp16_value(d_bits[j])))
            s = Fraction(0)
            for g in range(64):
                pat = cb[codes[j, g]]
                for lane in range(4):
                    s += int(pat[lane]) * Fraction(float(xf[t, 4 * g + lane]))
            exact = d * s
            assert abs(Fraction(float(y[t, j])) - exact) <= abs(exact) * Fraction(1, 2 ** 45) + Fraction(1, 2 ** 80)


def test_moe_equals_per_slot_gemv_and_weighting():
    n, k, E = 32, 512, 5
    experts = [oracle.encode_plain(workloads.gaussian_matrix(n, k, 0.02, seed=500 + e)) for e in range(E)]
    x = workloads.activations_bf16(3, k, seed=9)
    ids = np.array([[0, 4], [4, 2], [1, 0]], np.int32)
    wts = np.array([[0.7, 0.3], [0.5, 0.5], [0.9, 0.1]], np.float32)
    y = oracle.moe_gateup(experts, x, ids, wts, n, k)
    for t in range(3):
        for s in range(2):
            ref = oracle.gemv(experts[ids[t, s]], x[t:t + 1], n, k)[0]
            assert np.array_equal(y[t, s], ref)
    yw = oracle.moe_gateup(experts, x, ids, wts, n, k, flags=oracle.FLAG_WEIGHT_UP)
    assert np.array_equal(yw[:, :, : n // 2], y[:, :, : n // 2])
    assert np.allclose(yw[:, :, n // 2:], y[:, :, n // 2:] * wts[:, :, None], rtol=1e-15)


def test_route_pairs_is_a_grouping():
    ids = workloads.zipf_topk_ids(64, 256, 8, seed=9)
    counts, offsets, order = oracle.route_pairs(ids, 256)
    flat = ids.reshape(-1)
    assert counts.sum() == 64 * 8 and offsets[-1] == 64 * 8
    for e in range(256):
        seg = order[offsets[e]:offsets[e + 1]]
        assert np.all(flat[seg] == e)
        assert np.all(np.diff(seg) > 0)
    # each token's 8 experts are distinct (drawn without replacement)
    assert all(len(set(r)) == 8 for r in ids.tolist())


# ---------------------------------------------------------------------------
# fp8 activations (E4M3) for the fp8 tile variant
# ---------------------------------------------------------------------------


def test_e4m3_code_table_landmarks():
    # OCP FP8 E4M3 (no infinities): fixed points of the published format
    v = oracle.e4m3_value(np.arange(256))
    assert v[0x00] == 0.0 and v[0x01] == 2.0 ** -9 and v[0x07] == 7 * 2.0 ** -9
    assert v[0x08] == 2.0 ** -6 and v[0x38] == 1.0 and v[0x39] == 1.125 and v[0x7E] == 448.0
    assert np.isnan(v[0x7F]) and np.isnan(v[0xFF])
    assert np.all(np.diff(v[0x00:0x7F]) > 0)                 # 127 ordered non-negative values
    assert np.array_equal(v[0x80:0xFF], -v[0x00:0x7F])       # sign bit mirrors


def _e4m3_brute_force(vals):
    # nearest of the 127 non-negative finite values, ties to the even code,
    # saturating; the sign bit follows the input
    grid = oracle.e4m3_value(np.arange(0x7F))
    out = []
    for x in np.asarray(vals, np.float32).astype(np.float64):
        a = min(abs(x), 448.0)
        dist = np.abs(grid - a)
        best = np.flatnonzero(dist == dist.min())
        code = int(best[0]) if len(best) == 1 else int([c for c in best if c % 2 == 0][0])
        out.append(code | (0x80 if np.signbit(x) else 0))
    return np.array(out, np.uint8)


def test_e4m3_round_is_nearest_with_ties_to_even():
    rng = np.random.default_rng(88)
    grid = oracle.e4m3_value(np.arange(0x7F))
    mids = (grid[:-1] + grid[1:]) / 2                        # exact ties (fp32-representable)
    vals = np.concatenate([
        rng.standard_normal(3000) * 30, rng.uniform(-2.0 ** -6, 2.0 ** -6, 1000),
        rng.uniform(-500, 500, 1000), mids, -mids, grid, [0.0, -0.0, 448.0, 464.0, 465.0, -1e6, 1e-30]])
    vals = vals.astype(np.float32)
    assert np.array_equal(oracle.e4m3_round(vals), _e4m3_brute_force(vals))


def test_e4m3_round_matches_torch_cast():
    torch = pytest.importorskip("torch")
    if not hasattr(torch, "float8_e4m3fn"):
        pytest.skip("torch without float8")
    rng = np.random.default_rng(89)
    vals = np.concatenate([rng.standard_normal(20000) * 40, rng.uniform(-0.02, 0.02, 5000)]).astype(np.float32)
    vals = np.clip(vals, -448, 448)
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_round(vals), ref)


def test_quantize_x_e4m3_scales_each_row_to_the_range():
    x = workloads.activations_bf16(6, 512, seed=90)
    x[3] = 0                                                  # an all-zero row
    x[4, ::7] = 0x8000                                        # some -0.0
    codes, s = oracle.quantize_x_e4m3(x)
    xf = oracle.bf16_to_f64(x)
    for t in range(6):
        amax = np.max(np.abs(xf[t]))
        if amax == 0:
            assert s[t] == 0 and np.all((codes[t] & 0x7F) == 0)
            continue
        assert np.max(codes[t] & 0x7F) == 0x7E                 # the largest element lands on 448
        assert s[t] == np.float32(np.float32(amax) / np.float32(448))
        back = oracle.e4m3_value(codes[t]) * np.float64(s[t])
        # E4M3 has 3 mantissa bits: relative error <= 2^-4 above the subnormal range
        big = np.abs(xf[t]) > amax * 2.0 ** -6
        assert np.all(np.abs(back[big] - xf[t][big]) <= 2.0 ** -4 * np.abs(xf[t][big]) * 1.001)


def test_moe_fp8_is_exact_when_x_is_representable():
    # rows whose values are E4M3 values and whose amax is 448 quantize to themselves
    n, k, E, T, topk = 64, 512, 3, 4, 2
    experts = [oracle.encode_plain(workloads.gaussian_matrix(n, k, 0.02, seed=400 + e)) for e in range(E)]
    rng = np.random.default_rng(91)
    vals = oracle.e4m3_value(rng.integers(0, 0x7F, (T, k)) | (rng.integers(0, 2, (T, k)) << 7))
    vals[:, 0] = 448.0
    x = oracle.bf16_bits_rne(vals.astype(np.float32))
    assert np.array_equal(oracle.bf16_to_f64(x), vals)
    ids = workloads.zipf_topk_ids(T, E, topk, seed=92)
    y8 = oracle.moe_gateup_fp8(experts, x, ids, None, n, k)
    y = oracle.moe_gateup(experts, x, ids, None, n, k)
    assert np.array_equal(y8, y)


@pytest.mark.parametrize("mistake", ["ties_away", "no_saturation", "subnormal_step"])
def test_planted_fp8_mistakes_are_caught(monkeypatch, mistake):
    import oracle.stq1 as o
    grid = oracle.e4m3_value(np.arange(0x7F))
    vals = np.concatenate([grid, (grid[:-1] + grid[1:]) / 2,
                           [470.0, 500.0, 3 * 2.0 ** -10, 5 * 2.0 ** -11]]).astype(np.float32)
    assert np.array_equal(o.e4m3_round(vals), _e4m3_brute_force(vals))
    orig_rint, orig_min, orig_max = np.rint, np.minimum, np.maximum
    if mistake == "ties_away":
        monkeypatch.setattr(o.np, "rint", lambda a: np.floor(np.asarray(a) + 0.5))
    elif mistake == "no_saturation":
        monkeypatch.setattr(o, "E4M3_MAX", 480.0)
    elif mistake == "subnormal_step":
        # the step of the lowest normal binade extended one binade too far up
        monkeypatch.setattr(o.np, "maximum", lambda a, b: orig_max(a, b + 1) if np.isscalar(b) and b == -6 else orig_max(a, b))
    try:
        got = o.e4m3_round(vals)
    finally:
        monkeypatch.undo()
    assert not np.array_equal(got, _e4m3_brute_force(vals))
    assert orig_rint is np.rint and orig_min is np.minimum


# ---------------------------------------------------------------------------
# After gate/up: SwiGLU, combine, the MoE feed-forward chain
# ---------------------------------------------------------------------------


def _bf16_val(bits):
    # bf16 is the top half of an fp32 word (format definition)
    return (np.asarray(bits, np.uint32) << 16).view(np.float32).astype(np.float64)


def test_bf16_from_f64_is_nearest_with_ties_to_even():
    rng = np.random.default_rng(93)
    base = np.concatenate([rng.standard_normal(4000) * 10.0 ** rng.integers(-30, 30, 4000),
                           rng.uniform(-1e-38, 1e-38, 500)])
    # exact ties between neighbouring bf16 values, and values a hair off them
    b = rng.integers(0x0001, 0x7F7F, 500).astype(np.uint32)
    mids = (_bf16_val(b) + _bf16_val(b + 1)) / 2
    vals = np.concatenate([base, mids, -mids, np.nextafter(mids, 0), np.nextafter(mids, np.inf)])
    bits = oracle.bf16_bits_from_f64(vals).astype(np.uint32)
    mag = bits & 0x7FFF
    here = np.abs(np.abs(vals) - _bf16_val(mag))
    lo = np.abs(np.abs(vals) - _bf16_val(np.maximum(mag, 1) - 1))
    hi = np.abs(np.abs(vals) - _bf16_val(mag + 1))
    assert np.all(here <= lo) and np.all(here <= hi)
    tie = (here == hi) | ((here == lo) & (mag > 0))
    assert np.all(mag[tie] % 2 == 0)
    assert np.array_equal(bits >> 15, np.signbit(vals).astype(np.uint32))
    # agrees with the fp32 rounding routine wherever the value is an fp32
    f32 = rng.standard_normal(5000).astype(np.float32)
    assert np.array_equal(oracle.bf16_bits_from_f64(f32.astype(np.float64)), oracle.bf16_bits_rne(f32))


def test_silu_against_logistic_and_identities():
    special = pytest.importorskip("scipy.special")
    v = np.linspace(-40, 40, 4001)
    s = oracle.silu(v)
    assert np.allclose(s, v * special.expit(v), rtol=1e-14, atol=1e-300)
    assert oracle.silu(np.array([0.0]))[0] == 0.0
    assert np.allclose(oracle.silu(-v), s - v, rtol=1e-12, atol=1e-12)   # SiLU(-v) = SiLU(v) - v
    assert abs(oracle.silu(np.array([60.0]))[0] - 60.0) < 1e-20


def test_swiglu_pairs_gate_with_up():
    n = 8
    y = np.zeros((2, n))
    y[0, :4] = [0.0, 30.0, -30.0, 1.0]      # gates
    y[0, 4:] = [5.0, 2.0, 3.0, 4.0]         # ups
    y[1, :4] = 1.0
    y[1, 4:] = [1.0, -1.0, 0.5, 0.0]
    act = oracle.swiglu_bf16(y, n)
    vals = _bf16_val(act)
    s1 = 1.0 / (1.0 + np.exp(-1.0))
    assert vals[0, 0] == 0.0 and vals[0, 1] == 60.0 and abs(vals[0, 2]) < 1e-9
    assert vals[0, 3] == _bf16_val(oracle.bf16_bits_from_f64(np.array([4 * s1])))[0]
    assert np.allclose(vals[1], [s1, -s1, s1 / 2, 0.0], rtol=2 ** -8)


def test_moe_combine_weights_slots():
    yd = np.arange(2 * 3 * 4, dtype=np.float64).reshape(2, 3, 4)
    assert np.array_equal(oracle.moe_combine(yd, None), yd.sum(axis=1))
    w = np.array([[0, 1, 0], [0.5, 0, 0.25]], np.float32)
    got = oracle.moe_combine(yd, w)
    assert np.array_equal(got[0], yd[0, 1]) and np.allclose(got[1], 0.5 * yd[1, 0] + 0.25 * yd[1, 2])


def test_moe_ffn_equals_the_chain_of_single_matmuls():
    # gate/up and down through oracle.gemv per (token, slot) pair instead of the grouped path
    n, hidden, E, T, topk = 512, 256, 3, 3, 2
    gu = [oracle.encode_plain(workloads.gaussian_matrix(n, hidden, 0.05, seed=600 + e)) for e in range(E)]
    dn = [oracle.encode_plain(workloads.gaussian_matrix(hidden, n // 2, 0.05, seed=700 + e)) for e in range(E)]
    x = workloads.activations_bf16(T, hidden, seed=94)
    ids = workloads.zipf_topk_ids(T, E, topk, seed=95)
    wts = workloads.softmax_route_weights(T, topk, seed=96)
    out = oracle.moe_ffn(gu, dn, x, ids, wts, n, hidden)
    ref = np.zeros((T, hidden))
    for t in range(T):
        for s in range(topk):
            e = int(ids[t, s])
            y = oracle.gemv(gu[e], x[t:t + 1], n, hidden)[0]
            act = oracle.swiglu_bf16(y[None, :], n)
            ref[t] += np.float64(np.float32(wts[t, s])) * oracle.gemv(dn[e], act, hidden, n // 2)[0]
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12)
    # weights on the up half instead: SiLU(g) * (w u) = w SiLU(g) u up to the bf16 rounding of act
    # (bf16 rounding of act, up to 2^-9 relative per element, against sum |w W act|)
    out_up = oracle.moe_ffn(gu, dn, x, ids, wts, n, hidden, flags=oracle.FLAG_WEIGHT_UP)
    _, scale = oracle.moe_ffn(gu, dn, x, ids, wts, n, hidden, abs_sum=True)
    assert np.all(np.abs(out_up - out) <= 2 ** -8 * scale + 1e-9)


@pytest.mark.parametrize("mistake", ["swap_gate_up", "silu_sign", "combine_unweighted"])
def test_planted_ffn_mistakes_are_caught(monkeypatch, mistake):
    import oracle.stq1 as o
    def passes():
        try:
            test_silu_against_logistic_and_identities()
            test_swiglu_pairs_gate_with_up()
            test_moe_combine_weights_slots()
        except AssertionError:
            return False
        return True
    assert passes()
    def plant(name, fn):                     # in the module and in the package's re-export
        monkeypatch.setattr(o, name, fn)
        monkeypatch.setattr(oracle, name, fn)
    if mistake == "swap_gate_up":
        orig = o.swiglu_bf16
        plant("swiglu_bf16", lambda y, n: orig(np.concatenate(
            [np.asarray(y, np.float64).reshape(-1, n)[:, n // 2:], np.asarray(y, np.float64).reshape(-1, n)[:, :n // 2]], 1), n))
    elif mistake == "silu_sign":
        plant("silu", lambda v: np.asarray(v, np.float64) / (1.0 + np.exp(np.asarray(v, np.float64))))
    elif mistake == "combine_unweighted":
        plant("moe_combine", lambda yd, w: np.asarray(yd, np.float64).sum(axis=1))
    assert not passes()


# ---------------------------------------------------------------------------
# The pins catch planted mistakes
# ---------------------------------------------------------------------------


def _golden_and_bruteforce_pass():
    """Runs a subset of the pins, returning False on the first failure."""
    try:
        for name in ("plain_uniform_a.txt", "plain_uniform_b.txt"):
            test_golden_plain_uniform(name)
        test_golden_plain_bit_order()
        test_golden_sherry_moves_zero()
        test_plain_encoder_is_the_best_pattern_at_amax_scale()
        test_sherry_zero_choice_matches_brute_force()
        test_gemv_closed_form_all_code_zero()
    except AssertionError:
        return False
    return True


@pytest.mark.parametrize("mistake", ["sign_of_b", "nibble_order", "zero_cost_without_h", "wls_unweighted"])
def test_planted_mistakes_are_caught(monkeypatch, mistake):
    # Each mutation plants a plausible slip into the oracle (on the CPU only);
    # the pins above must notice it.
    import oracle.stq1 as o
    assert _golden_and_bruteforce_pass()
    if mistake == "sign_of_b":
        # the second non-zero lane takes the opposite sign in the decoder
        bad = o.codebook().astype(np.float64)
        for code in range(32):
            z = (code & 0xF) >> 2
            b = [lane for lane in range(4) if lane != z][1]
            bad[code, b] = -bad[code, b]
        monkeypatch.setattr(o, "_CODEBOOK_F64", bad)
    elif mistake == "nibble_order":
        orig = o.pack_blocks
        def bad_pack(d_bits, codes):
            codes = np.asarray(codes, np.uint8).reshape(-1, 64).copy()
            codes[:, 0::2], codes[:, 1::2] = codes[:, 1::2].copy(), codes[:, 0::2].copy()
            return orig(d_bits, codes)
        monkeypatch.setattr(o, "pack_blocks", bad_pack)
    elif mistake == "zero_cost_without_h":
        def bad_choice(aw, h, d):
            B = aw.shape[0]
            a4 = aw.reshape(B, 64, 4)
            dd = d[:, None, None]
            return np.argmin(dd * (2.0 * a4 - dd), axis=2)
        monkeypatch.setattr(o, "zero_lane_choice", bad_choice)
    elif mistake == "wls_unweighted":
        orig_wls = o.wls_scale
        monkeypatch.setattr(o, "wls_scale", lambda aw, h, z: orig_wls(aw, np.ones_like(h), z))
    assert not _golden_and_bruteforce_pass()
