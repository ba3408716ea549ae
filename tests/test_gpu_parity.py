"""CUDA path vs the CPU oracle, through the C ABI (needs a B200).

Bar: packed/dequantized bytes bit-exact; matmul outputs within
|y_gpu - y_oracle| <= 1e-3 * sum_k |W^[j,k] x[t,k]| + 1e-6 elementwise.
"""

import numpy as np
import pytest

import oracle
import workloads

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import sub_bit_sparse_b200 as stq1


def _dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


def _bf16(xbits):
    return _dev(xbits.astype(np.uint16).view(np.int16), None).view(torch.bfloat16)


def _assert_close(y_gpu, y_or, bound, what=""):
    err = np.abs(y_gpu.astype(np.float64) - y_or)
    tol = oracle.tolerance(bound)
    bad = err > tol
    assert not bad.any(), (
        f"{what}: {bad.sum()} of {bad.size} outside tolerance; worst ratio "
        f"{(err / tol).max():.3g}")
    return float((err / tol).max())


# ---------------------------------------------------------------------------
# dequant
# ---------------------------------------------------------------------------


@pytest.mark.parametrize("n,k", [(1, 256), (3, 512), (512, 2048), (37, 7168)])
def test_dequant_bit_exact(n, k):
    w = workloads.gaussian_matrix(n, k, 0.02, seed=n * 7 + k)
    packed = oracle.encode_plain(w)
    got = stq1.dequant(_dev(packed), n, k).view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, oracle.dequant_bf16(packed, n, k))


def test_dequant_all_codes_and_scales():
    d = [0.0, 2.0 ** -24, 1.0, 65504.0, 0.0173, 3.3e-3, 1.5, 0.999]
    d_bits = oracle.fp16_bits(np.array(d))
    codes = np.tile(np.arange(32, dtype=np.uint8), (len(d), 2))
    packed = oracle.pack_blocks(d_bits, codes)
    got = stq1.dequant(_dev(packed), len(d), 256).view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, oracle.dequant_bf16(packed, len(d), 256))


# ---------------------------------------------------------------------------
# GEMV
# ---------------------------------------------------------------------------


def _gemv_case(n, k, b, seed, mode="plain"):
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal((n, k)) * rng.uniform(0.005, 0.05, (n, 1))).astype(np.float32)
    packed = oracle.encode_plain(w) if mode == "plain" else oracle.encode_sherry(w, None)
    x = workloads.activations_bf16(b, k, seed=seed + 1)
    y = stq1.gemv(_dev(packed), _bf16(x), n, k).cpu().numpy()
    return _assert_close(y, oracle.gemv(packed, x, n, k), oracle.gemv_abs(packed, x, n, k),
                         f"gemv n={n} k={k} b={b}")


@pytest.mark.parametrize("n", [1, 3, 64, 130, 512])
@pytest.mark.parametrize("k", [256, 512, 1024, 7168])
@pytest.mark.parametrize("b", [1, 2, 3, 5, 8])
def test_gemv_small_shapes(n, k, b):
    _gemv_case(n, k, b, seed=n * 1000 + k + b)


def test_gemv_single_reference_workload():
    w, x = workloads.single_gemv_inputs()
    packed = stq1.quantize_ref(w, mode="plain")
    assert np.array_equal(packed, oracle.encode_plain(w))
    y = stq1.gemv(_dev(packed), _bf16(x), 512, 2048).cpu().numpy()
    _assert_close(y, oracle.gemv(packed, x, 512, 2048), oracle.gemv_abs(packed, x, 512, 2048), "cfg1")


@pytest.fixture(scope="module")
def decode_workload():
    w, h, x = workloads.decode_gemv_inputs()
    packed = stq1.quantize_ref(w, h, mode="sherry", rounds=3)
    return packed, x


@pytest.mark.parametrize("b", [1, 2, 4, 8])
def test_gemv_decode_workload_full(decode_workload, b):
    packed, x = decode_workload
    n, k = 4096, 7168
    xb = x[:b]
    y = stq1.gemv(_dev(packed), _bf16(xb), n, k).cpu().numpy()
    _assert_close(y, oracle.gemv(packed, xb, n, k), oracle.gemv_abs(packed, xb, n, k), f"cfg2 b={b}")


@pytest.mark.parametrize("b", [1, 2, 8])
def test_gemv_prefetch_leaves_results_unchanged(decode_workload, b):
    # stq1_gemv_prefetch only adds L2 prefetches of another matrix: same bits as
    # stq1_gemv, and the oracle's tolerance; prefetch lengths that are not a
    # multiple of 16, empty, or the matrix itself
    packed, x = decode_workload
    n, k = 4096, 7168
    wd, xd = _dev(packed), _bf16(x[:b])
    other = _dev(np.roll(packed, 4242))
    y0 = stq1.gemv(wd, xd, n, k).clone()
    for nxt in (other, other[: other.numel() - 37], other[:0], wd):
        y = stq1.gemv(wd, xd, n, k, prefetch=nxt)
        assert torch.equal(y, y0)
    assert stq1.status() == 0
    _assert_close(y0.cpu().numpy(), oracle.gemv(packed, x[:b], n, k), oracle.gemv_abs(packed, x[:b], n, k),
                  f"prefetch b={b}")


def test_gemv_repeatable_and_workspace_left_zero(decode_workload):
    packed, x = decode_workload
    wd, xd = _dev(packed), _bf16(x[:1])
    y1 = stq1.gemv(wd, xd, 4096, 7168).clone()
    y2 = stq1.gemv(wd, xd, 4096, 7168)
    # the split-K counters reset themselves: a second call reduces identically
    assert torch.equal(y1, y2)
    assert stq1.status() == 0


def test_gemv_shapes_interleaved_on_one_workspace():
    # calls of different shapes share the cached workspace; split-K counters must
    # stay valid whatever the previous call's shape was
    cases = [(4096, 7168, 1), (64, 1024, 3), (512, 2048, 1), (4096, 7168, 2), (130, 7168, 5), (4096, 7168, 1)]
    for i, (n, k, b) in enumerate(cases):
        _gemv_case(n, k, b, seed=900 + i)


def test_gemv_special_values():
    # zero scale, max scale, all-equal weights, a one-hot activation
    n, k = 8, 512
    codes = np.zeros((n * 2, 64), np.uint8)
    codes[::2] = np.arange(64) % 32
    d = np.array([0.0, 65504.0, 1.0, 2.0 ** -24, 0.5, 0.25, 1.0, 3.0] * 2)
    packed = oracle.pack_blocks(oracle.fp16_bits(d), codes)
    x = np.zeros((2, k), np.float32)
    x[0] = 1.0
    x[1, 5] = 1.0
    xb = workloads.bf16_bits_from_f32(x)
    y = stq1.gemv(_dev(packed), _bf16(xb), n, k).cpu().numpy()
    _assert_close(y, oracle.gemv(packed, xb, n, k), oracle.gemv_abs(packed, xb, n, k), "special")


# ---------------------------------------------------------------------------
# MoE gate/up
# ---------------------------------------------------------------------------


def _moe_check(experts_packed, x, ids, wts, n, k, E, flags=0):
    flat = np.concatenate(experts_packed) if isinstance(experts_packed, list) else experts_packed
    eb = oracle.packed_size(n, k)
    get = lambda e: flat[e * eb:(e + 1) * eb]  # noqa: E731
    y = stq1.moe_gateup(_dev(flat), _bf16(x), _dev(ids.astype(np.int32)), _dev(wts.astype(np.float32)),
                        n, k, E, flags=flags).cpu().numpy()
    y_or, y_abs = oracle.moe_gateup(get, x, ids, wts, n, k, flags=flags, abs_sum=True)
    return _assert_close(y, y_or, y_abs, f"moe n={n} k={k} E={E} flags={flags}")


@pytest.mark.parametrize("flags", [0, 1])
def test_moe_small_encoded_experts(flags):
    n, k, E, T, topk = 256, 1024, 12, 9, 4
    experts = [stq1.quantize_ref(workloads.gaussian_matrix(n, k, 0.02, seed=1000 + e)) for e in range(E)]
    x = workloads.activations_bf16(T, k, seed=3)
    ids = workloads.zipf_topk_ids(T, E, topk, seed=4)
    wts = workloads.softmax_route_weights(T, topk, seed=5)
    _moe_check(experts, x, ids, wts, n, k, E, flags)


def test_moe_skewed_and_duplicate_ids():
    # every token on expert 0 (more tokens than one tile holds), repeated ids in a row
    n, k, E, T, topk = 128, 512, 5, 13, 3
    experts = [stq1.quantize_ref(workloads.gaussian_matrix(n, k, 0.03, seed=77 + e)) for e in range(E)]
    x = workloads.activations_bf16(T, k, seed=8)
    ids = np.zeros((T, topk), np.int32)
    ids[:, 1] = np.arange(T) % E
    ids[:, 2] = 0
    wts = np.full((T, topk), 0.5, np.float32)
    _moe_check(experts, x, ids, wts, n, k, E, flags=1)


@pytest.mark.parametrize("n,k,E", [(130, 512, 5), (6, 1536, 3), (258, 1024, 3)])
def test_moe_expert_rows_straddle_super_rows(n, k, E):
    # With 84 * m bytes per row (m odd: P = 4 rows per 16-byte-aligned super-row;
    # m = 2 mod 4: P = 2) and N not a multiple of P, experts start inside a
    # super-row and the buffer ends in a partial one.
    T, topk = 7, 2
    experts = [stq1.quantize_ref(workloads.gaussian_matrix(n, k, 0.02, seed=500 + e)) for e in range(E)]
    x = workloads.activations_bf16(T, k, seed=21)
    ids = workloads.zipf_topk_ids(T, E, topk, seed=22)
    wts = workloads.softmax_route_weights(T, topk, seed=23)
    _moe_check(experts, x, ids, wts, n, k, E, flags=1)


def test_moe_decode_workload_full():
    # 256 experts x [4096, 7168] (1.23 GB packed), 16 tokens, Zipf(1.1) top-8.
    # Expert bytes are random valid blocks: every 5-bit code is legal, and the
    # kernel's arithmetic does not depend on how the codes were chosen.
    n, k, E = 4096, 7168, 256
    eb = oracle.packed_size(n, k)
    flat = workloads.random_packed_blocks(E * eb // 42, seed=2024)
    x, ids, wts = workloads.moe_decode_inputs()
    _moe_check(flat, x, ids, wts, n, k, E, flags=0)


def test_moe_bad_expert_id_is_flagged_not_trapped():
    n, k, E, T, topk = 64, 512, 4, 3, 2
    experts = np.concatenate([stq1.quantize_ref(workloads.gaussian_matrix(n, k, 0.02, seed=e)) for e in range(E)])
    x = workloads.activations_bf16(T, k, seed=1)
    ids = np.array([[0, 1], [2, 9], [-1, 3]], np.int32)
    y = stq1.moe_gateup(_dev(experts), _bf16(x), _dev(ids), None, n, k, E).cpu().numpy()
    err = stq1.status()
    assert err & stq1.DEV_BAD_EXPERT
    assert np.all(y[1, 1] == 0) and np.all(y[2, 0] == 0)
    good_ids = np.array([[0, 1], [2, 0], [0, 3]], np.int32)
    y_or = oracle.moe_gateup(lambda e: experts[e * oracle.packed_size(n, k):(e + 1) * oracle.packed_size(n, k)],
                             x, good_ids, np.ones((T, topk), np.float32), n, k)
    for t, s in ((0, 0), (0, 1), (1, 0), (2, 1)):
        assert np.allclose(y[t, s], y_or[t, s], rtol=1e-3, atol=1e-5)
    assert stq1.status() == 0   # cleared


def test_bad_arguments_enqueue_nothing():
    w = torch.zeros(42 * 4, dtype=torch.uint8, device="cuda")
    x = torch.zeros((1, 256), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(stq1.Stq1Error, match="SHAPE"):
        stq1.gemv(w, x, 4, 300)
    with pytest.raises(stq1.Stq1Error, match="ALIGN"):
        stq1.gemv(w[1:], x, 3, 256)
    assert stq1.status() == 0


# ---------------------------------------------------------------------------
# Largest sizes and degenerate cases
# ---------------------------------------------------------------------------


@pytest.mark.parametrize("b", [1, 5])
def test_gemv_long_rows(b):
    # K = 65,536: 256 blocks per row (10,752 bytes, a multiple of 16: super-rows of one row)
    n, k = 64, 65536
    w = workloads.gaussian_matrix(n, k, 0.01, seed=4242)
    packed = stq1.quantize_ref(w)
    x = workloads.activations_bf16(b, k, seed=4243)
    y = stq1.gemv(_dev(packed), _bf16(x), n, k).cpu().numpy()
    _assert_close(y, oracle.gemv(packed, x, n, k), oracle.gemv_abs(packed, x, n, k), f"long rows b={b}")


def test_gemv_largest_batch():
    # batch 65,535 (the API's limit) on the tile path
    n, k, b = 128, 256, 65535
    packed = stq1.quantize_ref(workloads.gaussian_matrix(n, k, 0.05, seed=11))
    x = workloads.activations_bf16(b, k, seed=12)
    y = stq1.gemv(_dev(packed), _bf16(x), n, k).cpu().numpy()
    _assert_close(y, oracle.gemv(packed, x, n, k), oracle.gemv_abs(packed, x, n, k), "batch 65535")


def test_gemv_zero_weights_and_zero_activations():
    n, k = 130, 1024
    packed = stq1.quantize_ref(np.zeros((n, k), np.float32))          # every d = 0
    x = workloads.activations_bf16(3, k, seed=5)
    assert np.all(stq1.gemv(_dev(packed), _bf16(x), n, k).cpu().numpy() == 0)
    packed = stq1.quantize_ref(workloads.gaussian_matrix(n, k, 0.02, seed=6))
    z = np.zeros((2, k), np.uint16)
    assert np.all(stq1.gemv(_dev(packed), _bf16(z), n, k).cpu().numpy() == 0)


def test_moe_most_experts_the_library_takes():
    # E = 4096 experts (the routing kernel's limit), a few tokens, top-8
    n, k, E, T, topk = 128, 256, 4096, 3, 8
    bank = workloads.random_packed_blocks(E * oracle.packed_size(n, k) // 42, seed=77)
    x = workloads.activations_bf16(T, k, seed=78)
    ids = workloads.zipf_topk_ids(T, E, topk, seed=79)
    wts = workloads.softmax_route_weights(T, topk, seed=80)
    _moe_check(bank, x, ids, wts, n, k, E, flags=1)


def test_moe_one_token_every_expert():
    n, k, E = 256, 512, 4
    experts = [stq1.quantize_ref(workloads.gaussian_matrix(n, k, 0.02, seed=90 + e)) for e in range(E)]
    x = workloads.activations_bf16(1, k, seed=91)
    ids = np.arange(E, dtype=np.int32).reshape(1, E)
    wts = np.full((1, E), 0.25, np.float32)
    _moe_check(experts, x, ids, wts, n, k, E, flags=0)
