"""Tensor-core decode kernel (mma.sync, few tokens) vs the CPU oracle, through the
C ABI (needs a B200).  The kernel is forced with stq1_set_path(3) so that every
shape, batch and MoE case below runs on it; the lookup-table kernel, which the
library no longer picks for 2..15 tokens, is forced the same way for the
batches it used to serve.

Bar: |y_gpu - y_oracle| <= 1e-3 * sum_k |W^[j,k] x[t,k]| + 1e-6 elementwise.
"""

import numpy as np
import pytest

import oracle
import workloads

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import sub_bit_sparse_b200 as stq1


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _bf16(xbits):
    return _dev(xbits.astype(np.uint16).view(np.int16)).view(torch.bfloat16)


def _assert_close(y_gpu, y_or, bound, what=""):
    err = np.abs(y_gpu.astype(np.float64) - y_or)
    tol = oracle.tolerance(bound)
    bad = err > tol
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} outside tolerance; worst {(err / tol).max():.3g}"


@pytest.fixture
def mma_path():
    stq1.set_path(stq1.PATH_MMA)
    yield
    stq1.set_path(stq1.PATH_AUTO)


@pytest.fixture
def table_path():
    stq1.set_path(stq1.PATH_TABLE)
    yield
    stq1.set_path(stq1.PATH_AUTO)


def _gemv(n, k, b, seed, mode="plain"):
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal((n, k)) * rng.uniform(0.005, 0.05, (n, 1))).astype(np.float32)
    packed = oracle.encode_plain(w) if mode == "plain" else oracle.encode_sherry(w, None)
    x = workloads.activations_bf16(b, k, seed=seed + 1)
    y = stq1.gemv(_dev(packed), _bf16(x), n, k).cpu().numpy()
    _assert_close(y, oracle.gemv(packed, x, n, k), oracle.gemv_abs(packed, x, n, k), f"n={n} k={k} b={b}")
    assert stq1.status() == 0


# K = 512 (one chunk: half a step), 1024 (one step), 1536 (three chunks: the
# last step holds one), 7168 (seven steps); N from one row to several slabs
# with a ragged last one; batches across one and several 8-token tiles.
@pytest.mark.parametrize("n", [1, 3, 64, 130, 512])
@pytest.mark.parametrize("k", [512, 1024, 1536, 7168])
@pytest.mark.parametrize("b", [1, 2, 7, 8, 9, 17])
def test_mma_gemv_shapes(mma_path, n, k, b):
    _gemv(n, k, b, seed=7000 + n * 31 + k + b)


@pytest.mark.parametrize("b", [1, 2, 3, 4, 5, 6, 7, 8, 12, 15])
def test_mma_decode_workload_full(mma_path, b):
    # [4096, 7168], Sherry-encoded with calibration importance (the decode GEMV
    # workload), every output checked
    w, h, x = workloads.decode_gemv_inputs()
    packed = stq1.quantize_ref(w, h, mode="sherry", rounds=3)
    n, k = w.shape
    xb = x[:b] if b <= x.shape[0] else workloads.activations_bf16(b, k, seed=70 + b)
    y = stq1.gemv(_dev(packed), _bf16(xb), n, k).cpu().numpy()
    _assert_close(y, oracle.gemv(packed, xb, n, k), oracle.gemv_abs(packed, xb, n, k), f"decode b={b}")


def test_mma_special_scales_and_activations(mma_path):
    # zero, largest, subnormal scales; every code; a one-hot and an all-ones token
    n, k = 16, 1024
    codes = (np.arange(n * 4 * 64) % 32).astype(np.uint8).reshape(n * 4, 64)
    d = np.tile([0.0, 65504.0, 1.0, 2.0 ** -24, 0.5, 3.0e-3, 7.0, 1.0 / 3], n * 4 // 8)
    packed = oracle.pack_blocks(oracle.fp16_bits(d), codes)
    x = np.zeros((3, k), np.float32)
    x[0, 517] = 1.0
    x[1] = 1.0
    x[2] = np.linspace(-300.0, 300.0, k)
    xb = workloads.bf16_bits_from_f32(x)
    y = stq1.gemv(_dev(packed), _bf16(xb), n, k).cpu().numpy()
    _assert_close(y, oracle.gemv(packed, xb, n, k), oracle.gemv_abs(packed, xb, n, k), "special")


def test_mma_repeatable_split_k(mma_path):
    # few rows: the K range is split over several CTAs and reduced through the
    # workspace; results are deterministic and the counters reset themselves
    n, k, b = 64, 7168, 5
    w = workloads.gaussian_matrix(n, k, 0.02, seed=55)
    packed = stq1.quantize_ref(w)
    x = workloads.activations_bf16(b, k, seed=56)
    wd, xd = _dev(packed), _bf16(x)
    y1 = stq1.gemv(wd, xd, n, k).clone()
    y2 = stq1.gemv(wd, xd, n, k)
    assert torch.equal(y1, y2)
    _assert_close(y1.cpu().numpy(), oracle.gemv(packed, x, n, k), oracle.gemv_abs(packed, x, n, k), "split K")
    assert stq1.status() == 0


def _moe(n, k, E, T, topk, flags, seed, ids=None):
    experts = np.concatenate([stq1.quantize_ref(workloads.gaussian_matrix(n, k, 0.02, seed=seed + e))
                              for e in range(E)])
    x = workloads.activations_bf16(T, k, seed=seed + 100)
    if ids is None:
        ids = workloads.zipf_topk_ids(T, E, topk, seed=seed + 101)
    wts = workloads.softmax_route_weights(T, topk, seed=seed + 102)
    y = stq1.moe_gateup(_dev(experts), _bf16(x), _dev(ids.astype(np.int32)), _dev(wts), n, k, E,
                        flags=flags).cpu().numpy()
    eb = oracle.packed_size(n, k)
    yr, ya = oracle.moe_gateup(lambda e: experts[e * eb:(e + 1) * eb], x, ids, wts, n, k, flags=flags, abs_sum=True)
    _assert_close(y, yr, ya, f"moe n={n} k={k} E={E} T={T} flags={flags}")
    assert stq1.status() == 0


@pytest.mark.parametrize("flags", [0, 1])
def test_mma_moe_small(mma_path, flags):
    _moe(256, 1024, 12, 9, 4, flags, seed=8000)


def test_mma_moe_expert_with_many_tiles(mma_path):
    # 21 tokens all on expert 0 (three 8-pair tiles) plus a second slot elsewhere
    T, E = 21, 5
    ids = np.zeros((T, 2), np.int32)
    ids[:, 1] = 1 + np.arange(T) % (E - 1)
    _moe(128, 512, E, T, 2, 1, seed=8100, ids=ids)


@pytest.mark.parametrize("n,k,E", [(130, 512, 5), (6, 1536, 3), (258, 1024, 3)])
def test_mma_moe_expert_rows_straddle_super_rows(mma_path, n, k, E):
    # experts that start inside a super-row and a buffer that ends in a partial one
    _moe(n, k, E, 7, 2, 1, seed=8200 + n)


def test_mma_moe_decode_workload_full():
    # by size: 16 tokens x top-8 of 256 [4096, 7168] experts takes the
    # tensor-core decode kernel; every output against the oracle
    n, k, E = 4096, 7168, 256
    eb = oracle.packed_size(n, k)
    flat = workloads.random_packed_blocks(E * eb // 42, seed=2024)
    x, ids, wts = workloads.moe_decode_inputs()
    y = stq1.moe_gateup(_dev(flat), _bf16(x), _dev(ids), _dev(wts), n, k, E).cpu().numpy()
    yr, ya = oracle.moe_gateup(lambda e: flat[e * eb:(e + 1) * eb], x, ids, wts, n, k, abs_sum=True)
    _assert_close(y, yr, ya, "moe decode full")
    assert stq1.status() == 0


@pytest.mark.parametrize("b", [2, 3, 4, 5, 8])
@pytest.mark.parametrize("n,k", [(64, 1024), (130, 7168)])
def test_table_kernel_small_batches(table_path, n, k, b):
    _gemv(n, k, b, seed=9000 + n + k + b)


def test_table_kernel_moe(table_path):
    _moe(256, 1024, 12, 9, 4, 1, seed=9100)


def test_table_kernel_one_token_tile_over_many_chunks(table_path):
    # Batch 5 on the table kernel: a four-token tile and a one-token tile.
    # With 112 slabs the split is one piece per unit, so every CTA runs all 14
    # chunks, and the one-token unit alternates two tables (one barrier per
    # chunk, each chunk's copy issued after the previous chunk's barrier).
    # Rows of the first, a middle and the last slab against the oracle.
    n, k, b = 14336, 7168, 5
    rb = k // 256 * 42
    packed = workloads.random_packed_blocks(n * k // 256, seed=9200)
    x = workloads.activations_bf16(b, k, seed=9201)
    y = stq1.gemv(_dev(packed), _bf16(x), n, k).cpu().numpy()
    assert stq1.status() == 0
    for r0 in (0, 7040, n - 128):
        sub = packed[r0 * rb:(r0 + 128) * rb]
        _assert_close(y[:, r0:r0 + 128], oracle.gemv(sub, x, 128, k), oracle.gemv_abs(sub, x, 128, k),
                      f"rows {r0}..{r0 + 127}")
