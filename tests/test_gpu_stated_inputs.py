"""The MoE workloads on their stated inputs, vs the CPU oracle (needs a B200).

The expert matrices are the stated ones: expert e's fused gate+up weights are
N(0, 0.02^2) with seed 1000 + e (workloads.expert_weights), encoded by the
plain amax encoder.  They are encoded on the GPU (stq1_quantize) for the
experts that are read; the GPU encoder's bytes are checked equal to the
oracle's encoder on one expert, so the GEMV checks run on exactly the
encoding the oracle defines.

* MoE decode: 16 tokens, top-8 of 256 (Zipf 1.1): every routed expert
  encoded, all 128 x 4096 outputs checked.
* MoE prefill: 4096 tokens (32,768 pairs): a sample of experts encoded from
  their stated weights and checked -- every expert whose pair count is within
  3 of a multiple of the 128-pair tile, the most and the least loaded, and a
  spread; the other experts hold random valid blocks (read, not checked).
  bf16 against the exact oracle, fp8 against the oracle's fp8 reading.
Bar: |y_gpu - y_oracle| <= 1e-3 * sum_k |W^[j,k] x[t,k]| + 1e-6.
"""

import numpy as np
import pytest

import oracle
import workloads

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import sub_bit_sparse_b200 as stq1

N, K, E = 4096, 7168, 256
EB = N * (K // 256) * 42


def _bank_with_stated_experts(experts, fill_seed=None):
    """A device bank of E experts; `experts` are encoded (plain) on the GPU from
    their stated weights, the rest are zero (fill_seed None) or random valid blocks."""
    bank = torch.zeros(E * EB, dtype=torch.uint8, device="cuda")
    if fill_seed is not None:
        g = torch.Generator(device="cuda")
        g.manual_seed(fill_seed)
        bank.copy_(torch.randint(0, 256, (E * EB,), dtype=torch.uint8, device="cuda", generator=g))
        d = torch.full((E * EB // 42,), 0.058, dtype=torch.float16, device="cuda")
        bank.view(-1, 42)[:, 0:2].copy_(d.view(torch.uint8).view(-1, 2))
    for e in experts:
        w = torch.from_numpy(workloads.expert_weights(int(e))).cuda()
        stq1.quantize_gpu(w, None, mode="plain", out=bank[e * EB:(e + 1) * EB])
        del w
    torch.cuda.synchronize()
    assert stq1.status() == 0
    return bank


def _check(y, ref, bound, what):
    err = np.abs(y.astype(np.float64) - ref)
    tol = oracle.tolerance(bound)
    bad = err > tol
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} outside tolerance; worst {(err / tol).max():.3g}"


def test_gpu_encoder_matches_oracle_on_a_stated_expert():
    e = 0
    w = workloads.expert_weights(e)
    got = stq1.quantize_gpu(torch.from_numpy(w).cuda(), None, mode="plain").cpu().numpy()
    assert np.array_equal(got, oracle.encode_plain(w))


def test_moe_decode_on_stated_experts():
    x, ids, wts = workloads.moe_decode_inputs()
    routed = np.unique(ids)
    bank = _bank_with_stated_experts(routed)
    xd = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    y = stq1.moe_gateup(bank, xd, torch.from_numpy(ids).cuda(), torch.from_numpy(wts).cuda(), N, K, E).cpu().numpy()
    assert stq1.status() == 0
    host = {int(e): bank[e * EB:(e + 1) * EB].cpu().numpy() for e in routed}
    yr, ya = oracle.moe_gateup(lambda e: host[e], x, ids, wts, N, K, abs_sum=True)
    _check(y, yr, ya, "moe decode, stated experts")


def _prefill_sample(ids):
    counts = np.bincount(ids.reshape(-1), minlength=E)
    near = [e for e in range(E) if min(counts[e] % 128, 128 - counts[e] % 128) <= 3]
    spread = [int(e) for e in np.argsort(counts, kind="stable")[::64]]
    return sorted(set(near + [int(np.argmax(counts)), int(np.argmin(counts))] + spread)), counts


@pytest.mark.parametrize("fp8", [False, True])
def test_moe_prefill_on_stated_expert_sample(fp8):
    x, ids, wts = workloads.moe_prefill_inputs()
    sample, counts = _prefill_sample(ids)
    bank = _bank_with_stated_experts(sample, fill_seed=4242)
    xd = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    flags = stq1.MOE_FP8 if fp8 else 0
    y = stq1.moe_gateup(bank, xd, torch.from_numpy(ids).cuda(), torch.from_numpy(wts).cuda(), N, K, E,
                        flags=flags).cpu().numpy()
    assert stq1.status() == 0
    if fp8:
        codes, s = oracle.quantize_x_e4m3(x)
        xf = oracle.e4m3_value(codes) * s.astype(np.float64)[:, None]
    else:
        xf = oracle.bf16_to_f64(x)
    for e in sample:
        w = oracle.decode(bank[e * EB:(e + 1) * EB].cpu().numpy(), N, K)
        tt, ss = np.nonzero(ids == e)
        _check(y[tt, ss], xf[tt] @ w.T, np.abs(xf[tt]) @ np.abs(w).T,
               f"prefill{' fp8' if fp8 else ''} expert {e} ({counts[e]} pairs)")
