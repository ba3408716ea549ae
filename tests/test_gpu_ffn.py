"""SwiGLU, top-k combine and the routed MoE feed-forward chain vs the oracle (needs a B200)."""

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


@pytest.mark.parametrize("p,n", [(1, 2), (7, 512), (300, 4096)])
def test_swiglu_bit_exact(p, n):
    # fp64 SiLU rounded once to bf16 on both sides: the bits agree (a 1-ulp fp64
    # difference in exp could flip a rounding only within 2^-45 of a bf16 tie)
    y = workloads.gateup_outputs(p, n, seed=p + n)
    act = stq1.swiglu(_dev(y), n).view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(act, oracle.swiglu_bf16(y, n))


def test_moe_combine_matches_oracle():
    rng = np.random.default_rng(3)
    yd = rng.standard_normal((9, 5, 300)).astype(np.float32)
    w = workloads.softmax_route_weights(9, 5, seed=4)
    for ww in (w, None):
        got = stq1.moe_combine(_dev(yd), None if ww is None else _dev(ww)).cpu().numpy()
        ref = oracle.moe_combine(yd, ww)
        scale = oracle.moe_combine(np.abs(yd), None if ww is None else np.abs(ww))
        assert np.all(np.abs(got - ref) <= oracle.tolerance(scale))


def _ffn_check(gu, dn, x, ids, wts, n, hidden, E, flags, tokens=None):
    flat_gu = np.concatenate(gu) if isinstance(gu, list) else gu
    flat_dn = np.concatenate(dn) if isinstance(dn, list) else dn
    out = stq1.moe_ffn(_dev(flat_gu), _dev(flat_dn), _bf16(x), _dev(ids.astype(np.int32)), _dev(wts), n, hidden, E,
                       flags=flags).cpu().numpy()
    assert stq1.status() == 0
    ebg, ebd = oracle.packed_size(n, hidden), oracle.packed_size(hidden, n // 2)
    getg = lambda e: flat_gu[e * ebg:(e + 1) * ebg]  # noqa: E731
    getd = lambda e: flat_dn[e * ebd:(e + 1) * ebd]  # noqa: E731
    t = slice(None) if tokens is None else tokens
    ref, scale = oracle.moe_ffn(getg, getd, x[t], ids[t], wts[t], n, hidden, flags=flags, abs_sum=True)
    err = np.abs(out[t] - ref)
    tol = oracle.tolerance(scale)
    assert np.all(err <= tol), f"{(err > tol).sum()} outside; worst {(err / tol).max():.3g}"


@pytest.mark.parametrize("flags", [0, 1])
def test_moe_ffn_small(flags):
    n, hidden, E, T, topk = 512, 512, 6, 20, 3
    gu = [stq1.quantize_ref(workloads.gaussian_matrix(n, hidden, 0.05, seed=800 + e)) for e in range(E)]
    dn = [stq1.quantize_ref(workloads.gaussian_matrix(hidden, n // 2, 0.05, seed=900 + e)) for e in range(E)]
    x = workloads.activations_bf16(T, hidden, seed=97)
    ids = workloads.zipf_topk_ids(T, E, topk, seed=98)
    wts = workloads.softmax_route_weights(T, topk, seed=99)
    _ffn_check(gu, dn, x, ids, wts, n, hidden, E, flags)


def test_moe_ffn_decode_workload_sampled_tokens():
    # 256 experts: gate/up [4096, 7168], down [7168, 2048]; 16 tokens, Zipf(1.1)
    # top-8.  Random valid block bytes (every 5-bit code is legal); the oracle
    # recomputes three tokens end to end (24 routed experts).
    n, hidden, E = 4096, 7168, 256
    gu = workloads.random_packed_blocks(E * oracle.packed_size(n, hidden) // 42, seed=31)
    dn = workloads.random_packed_blocks(E * oracle.packed_size(hidden, n // 2) // 42, seed=32, d_sigma=0.004)
    x, ids, wts = workloads.moe_decode_inputs()
    _ffn_check(gu, dn, x, ids, wts, n, hidden, E, flags=0, tokens=[0, 7, 15])
