"""The C++ host encoder (stq1_quantize_ref) is bit-exact with the oracle (CPU only)."""

import numpy as np
import pytest

import oracle
import workloads
import sub_bit_sparse_b200 as stq1


def test_plain_matches_oracle_on_single_gemv_weights():
    w, _ = workloads.single_gemv_inputs()
    got = stq1.quantize_ref(w, mode="plain")
    assert np.array_equal(got, oracle.encode_plain(w))


def test_sherry_matches_oracle_on_expert_like_rows():
    w, h, _ = workloads.decode_gemv_inputs()
    rows = np.r_[0:64, 2048:2080, 4064:4096]
    ws = np.ascontiguousarray(w[rows])
    got = stq1.quantize_ref(ws, h, mode="sherry", rounds=3)
    assert np.array_equal(got, oracle.encode_sherry(ws, h, rounds=3))


@pytest.mark.parametrize("rounds", [0, 1, 2, 5])
def test_sherry_round_counts(rounds):
    rng = np.random.default_rng(rounds)
    w = (rng.standard_normal((8, 768)) * 0.02).astype(np.float32)
    h = rng.uniform(0.0, 3.0, 768).astype(np.float32)
    assert np.array_equal(stq1.quantize_ref(w, h, mode="sherry", rounds=rounds),
                          oracle.encode_sherry(w, h, rounds=rounds))


def test_edge_blocks():
    w = np.zeros((6, 256), np.float32)
    w[1] = -0.0                                        # negative zeros count as +
    w[2] = np.tile([1.0, 1.0, -1.0, 1.0], 64)          # ties: lowest lane is zeroed
    w[3] = 1e6                                         # saturates at 65504
    w[4, ::4] = 3e-8                                   # fp16 subnormal scale
    w[5] = np.linspace(-1, 1, 256, dtype=np.float32)
    h0 = np.zeros(256, np.float32)                     # all-zero importance: falls back to h = 1
    h1 = np.tile(np.array([0, 0, 0, 1], np.float32), 64)   # zero on most lanes
    for mode, h in (("plain", None), ("sherry", None), ("sherry", h0), ("sherry", h1)):
        got = stq1.quantize_ref(w, h, mode=mode)
        exp = oracle.encode_plain(w) if mode == "plain" else oracle.encode_sherry(w, h)
        assert np.array_equal(got, exp), (mode, h is None)


def test_golden_blocks_through_the_host_encoder():
    import os
    gdir = os.path.join(os.path.dirname(__file__), "golden")
    kv = {}
    for line in open(os.path.join(gdir, "sherry_moves_zero.txt")):
        line = line.split("#", 1)[0].strip()
        if "=" in line:
            k, v = (s.strip() for s in line.split("=", 1))
            kv[k] = v
    w = np.tile(np.array([float(v) for v in kv["group"].split()], np.float32), 64)[None, :]
    h = np.tile(np.array([float(v) for v in kv["h_group"].split()], np.float32), 64)
    assert stq1.quantize_ref(w, h, mode="sherry").tobytes().hex() == kv["bytes"]
    assert stq1.quantize_ref(w, mode="plain").tobytes().hex() == kv["plain_bytes"]


def test_thread_count_does_not_change_bytes():
    w, h, _ = workloads.decode_gemv_inputs(n=96, k=1024)
    a = stq1.quantize_ref(w, h, mode="sherry", threads=1)
    b = stq1.quantize_ref(w, h, mode="sherry", threads=7)
    assert np.array_equal(a, b)


def test_errors():
    w = np.ones((2, 256), np.float32)
    with pytest.raises(stq1.Stq1Error, match="SHAPE"):
        stq1.quantize_ref(np.ones((2, 300), np.float32))
    bad = w.copy()
    bad[1, 7] = np.nan
    with pytest.raises(stq1.Stq1Error, match="VALUE"):
        stq1.quantize_ref(bad)
    with pytest.raises(stq1.Stq1Error, match="VALUE"):
        stq1.quantize_ref(w, -np.ones(256, np.float32), mode="sherry")
    with pytest.raises(stq1.Stq1Error, match="ARG"):
        stq1.quantize_ref(w, None, mode="sherry", rounds=-1)
