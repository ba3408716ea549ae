"""Seeded synthetic inputs for the STQ1_0 matmul workloads.

This module only draws random numbers and shapes them; it holds none of the
STQ1_0 arithmetic (no encoding, decoding or contraction).  Both the CPU oracle
and the CUDA path take their inputs from here, so the two sides see identical
bytes.

Generator: NumPy ``PCG64`` (``numpy.random.default_rng(seed)``), one fixed
seed per quantity.  Activations are bf16 by definition of the workloads; they
are drawn in fp32 and stored as bf16 bit patterns (``uint16``), rounded to
nearest-even.

Workload shapes follow the pages' deployment: 256 routed experts with top-8
routing (lemmy.durstig.online post 66506, "Precision follows weight
sensitivity"; traictory.com "Tencent's 200GB Hy4-preview", "The claim, stated
precisely"), expert gate/up projections in STQ1_0 (same post, "Four weights,
five bits"), hidden size 7168 and a fused gate+up of 2 x 2048 rows.
"""

from __future__ import annotations

import numpy as np

# ---------------------------------------------------------------------------
# bf16 storage of activations (input synthesis, not part of the method)
# ---------------------------------------------------------------------------


def bf16_bits_from_f32(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest, ties to even.

    Non-finite values are not produced by any generator here.
    """
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    rounding = ((u >> 16) & 1) + 0x7FFF
    return ((u + rounding) >> 16).astype(np.uint16)


def f32_from_bf16_bits(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> fp32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------------------
# Building blocks
# ---------------------------------------------------------------------------


def gaussian_matrix(n: int, k: int, sigma: float, seed: int) -> np.ndarray:
    """W ~ N(0, sigma^2), fp32, shape [n, k]."""
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((n, k), dtype=np.float32)
    w *= np.float32(sigma)
    return w


def expert_like_matrix(n: int, k: int, seeds=(3, 4, 5)) -> np.ndarray:
    """Rows N(0, s_r^2) with s_r log-uniform in [0.005, 0.05], plus 0.1% outliers.

    ``seeds = (row-sigma seed, weight seed, outlier seed)``.  Exactly
    ``round(0.001 * n * k)`` positions, drawn uniformly without replacement,
    are set to +/-10 s_r with a random sign.
    """
    s_seed, w_seed, o_seed = seeds
    rs = np.random.default_rng(s_seed)
    sig = np.exp(rs.uniform(np.log(0.005), np.log(0.05), size=n)).astype(np.float32)
    rw = np.random.default_rng(w_seed)
    w = rw.standard_normal((n, k), dtype=np.float32)
    w *= sig[:, None]
    ro = np.random.default_rng(o_seed)
    n_out = int(round(0.001 * n * k))
    pos = ro.choice(n * k, size=n_out, replace=False)
    sign = np.where(ro.integers(0, 2, size=n_out) == 1, np.float32(1), np.float32(-1))
    rows = pos // k
    flat = w.reshape(-1)
    flat[pos] = sign * np.float32(10.0) * sig[rows]
    return w


def calibration_importance(k: int, seed: int, n_vectors: int = 512) -> np.ndarray:
    """Diagonal importance h_k = mean over calibration vectors of x_k^2 (fp32).

    Calibration vectors are tau * N(0, 1) with a per-column tau log-uniform in
    [0.25, 4], so h spans roughly 1/16 .. 16 across columns.
    """
    rng = np.random.default_rng(seed)
    tau = np.exp(rng.uniform(np.log(0.25), np.log(4.0), size=k))
    x = rng.standard_normal((n_vectors, k)) * tau[None, :]
    return np.mean(x * x, axis=0).astype(np.float32)


def activations_bf16(t: int, k: int, seed: int) -> np.ndarray:
    """x ~ N(0, 1) stored as bf16 bits, shape [t, k]."""
    rng = np.random.default_rng(seed)
    return bf16_bits_from_f32(rng.standard_normal((t, k), dtype=np.float32))


def zipf_topk_ids(t: int, n_experts: int, topk: int, seed: int, s: float = 1.1) -> np.ndarray:
    """Per token, ``topk`` distinct expert ids drawn with p_e proportional to (e+1)^-s.

    Draws are sequential without replacement (NumPy ``choice(replace=False)``),
    int32 [t, topk].
    """
    rng = np.random.default_rng(seed)
    p = (np.arange(1, n_experts + 1, dtype=np.float64)) ** (-s)
    p /= p.sum()
    out = np.empty((t, topk), dtype=np.int32)
    for i in range(t):
        out[i] = rng.choice(n_experts, size=topk, replace=False, p=p)
    return out


def softmax_route_weights(t: int, topk: int, seed: int) -> np.ndarray:
    """Routing weights: softmax over the top-k slots of N(0, 1) logits (fp32)."""
    rng = np.random.default_rng(seed)
    z = rng.standard_normal((t, topk))
    z -= z.max(axis=1, keepdims=True)
    e = np.exp(z)
    return (e / e.sum(axis=1, keepdims=True)).astype(np.float32)


def random_fp16_scales(count: int, seed: int, sigma: float = 0.02) -> np.ndarray:
    """|N(0, sigma^2)| values (fp64) to be used as block scales in code sweeps."""
    rng = np.random.default_rng(seed)
    return np.abs(rng.standard_normal(count)) * sigma


# ---------------------------------------------------------------------------
# The five workloads
# ---------------------------------------------------------------------------

HIDDEN = 7168          # K of the expert gate/up projections
GATE_UP = 4096         # fused gate (2048 rows) + up (2048 rows)
N_EXPERTS = 256
TOPK = 8


def single_gemv_inputs():
    """Single GEMV, 512 x 2048, W ~ N(0, 0.02^2) (seed 0), x 1 x 2048 (seed 1)."""
    w = gaussian_matrix(512, 2048, 0.02, seed=0)
    x = activations_bf16(1, 2048, seed=1)
    return w, x


def code_sweep_scales():
    """8 random scales (seed 2) for the 32-code round trip; specials are added by callers."""
    return random_fp16_scales(8, seed=2)


def decode_gemv_inputs(n: int = GATE_UP, k: int = HIDDEN):
    """Expert-shaped decode GEMV: W (seeds 3/4/5), importance h (seed 6), x [8, k] (seed 7)."""
    w = expert_like_matrix(n, k, seeds=(3, 4, 5))
    h = calibration_importance(k, seed=6)
    x = activations_bf16(8, k, seed=7)
    return w, h, x


def expert_weights(e: int, n: int = GATE_UP, k: int = HIDDEN) -> np.ndarray:
    """Expert e's fused gate+up matrix, W ~ N(0, 0.02^2) with seed 1000 + e."""
    return gaussian_matrix(n, k, 0.02, seed=1000 + e)


def moe_decode_inputs(t: int = 16, k: int = HIDDEN):
    """MoE decode: x [16, k] (seed 8), Zipf(1.1) top-8 of 256 ids (seed 9), weights (seed 10)."""
    x = activations_bf16(t, k, seed=8)
    ids = zipf_topk_ids(t, N_EXPERTS, TOPK, seed=9)
    wts = softmax_route_weights(t, TOPK, seed=10)
    return x, ids, wts


def moe_prefill_inputs(t: int = 4096, k: int = HIDDEN):
    """MoE prefill: x [4096, k] (seed 11), ids (seed 12), weights (seed 12 + 10000)."""
    x = activations_bf16(t, k, seed=11)
    ids = zipf_topk_ids(t, N_EXPERTS, TOPK, seed=12)
    wts = softmax_route_weights(t, TOPK, seed=10012)
    return x, ids, wts


def crossover_inputs(n: int = 18432, k: int = HIDDEN, max_batch: int = 1024):
    """Crossover sweep: W with expert-like statistics (seeds 13/14/15), h (16), x (17)."""
    w = expert_like_matrix(n, k, seeds=(13, 14, 15))
    h = calibration_importance(k, seed=16)
    x = activations_bf16(max_batch, k, seed=17)
    return w, h, x


def random_packed_blocks(n_blocks: int, seed: int, d_sigma: float = 0.058) -> np.ndarray:
    """Random but valid STQ1_0 block bytes for speed runs: uniform code bytes, positive
    fp16 scales near ``d_sigma`` (the amax of 256 N(0, 0.02^2) weights is about 0.058).

    Every 5-bit code is valid, so uniform random code bytes are a legal
    encoding with uniformly distributed patterns (as an amax encoder produces
    on Gaussian weights).  Layout of a block: fp16 scale at bytes 0-1, code
    bytes 2-41.
    """
    rng = np.random.default_rng(seed)
    blocks = rng.integers(0, 256, size=(n_blocks, 42), dtype=np.uint8)
    d = (d_sigma * (1.0 + 0.1 * rng.standard_normal(n_blocks))).astype(np.float16)
    blocks[:, 0:2] = d.view(np.uint8).reshape(n_blocks, 2)
    return blocks.reshape(-1)


def gateup_outputs(p: int, n: int, seed: int) -> np.ndarray:
    """fp32 [p, n] stand-ins for fused gate/up outputs: N(0, 1) scaled per row by
    10^U(-3, 2), with a few entries at +/-1e3 (exp underflow / overflow in SiLU)
    and some exact zeros."""
    rng = np.random.default_rng(seed)
    y = rng.standard_normal((p, n)) * 10.0 ** rng.uniform(-3, 2, (p, 1))
    flat = y.reshape(-1)
    idx = rng.choice(flat.size, size=max(1, flat.size // 500), replace=False)
    flat[idx] = rng.choice([-1e3, 1e3, 0.0], size=idx.size)
    return y.astype(np.float32)



# ---------------------------------------------------------------------------
# Mixed-precision allocation study: one [n, k] matrix and n_cal calibration
# rows per layer, with layer-to-layer differences in how strongly the
# calibration channels are correlated and how much of the weights lie along
# the correlated directions (the pages score 77 MoE layers; lemmy.durstig.online
# post 66506, "Full-Hessian scoring").
# ---------------------------------------------------------------------------

MIX_RANK = 16


def mix_layer_params(layer: int, seed: int):
    """(rho, beta) of a layer: correlation strength of the calibration channels
    in [0, 0.9] and weight alignment with the shared directions in [0, 1]."""
    rng = np.random.default_rng([seed, layer, 0])
    return float(rng.uniform(0.0, 0.9)), float(rng.uniform(0.0, 1.0))


def mix_layer(n: int, k: int, n_cal: int, layer: int, seed: int):
    """(w fp32 [n, k], x bf16 bits [n_cal, k]) of one layer (NumPy).

    x = tau * (sqrt(1 - rho^2) z + rho g V): z [n_cal, k] and g [n_cal, 16]
    standard normal, V [16, k] normal with variance 1/16, per-channel tau
    log-uniform in [0.25, 4].  w = s_r * (N(0, 1) + beta A V): per-row s_r
    log-uniform in [0.005, 0.05], A [n, 16] standard normal.
    """
    rho, beta = mix_layer_params(layer, seed)
    rng = np.random.default_rng([seed, layer, 1])
    v = rng.standard_normal((MIX_RANK, k)) / np.sqrt(MIX_RANK)
    tau = np.exp(rng.uniform(np.log(0.25), np.log(4.0), size=k))
    z = rng.standard_normal((n_cal, k))
    g = rng.standard_normal((n_cal, MIX_RANK))
    x = tau[None, :] * (np.sqrt(1.0 - rho * rho) * z + rho * (g @ v))
    s = np.exp(rng.uniform(np.log(0.005), np.log(0.05), size=n))
    a = rng.standard_normal((n, MIX_RANK))
    w = s[:, None] * (rng.standard_normal((n, k)) + beta * (a @ v))
    return w.astype(np.float32), bf16_bits_from_f32(x.astype(np.float32))


def mix_layer_torch(n: int, k: int, n_cal: int, layer: int, seed: int, device):
    """The same recipe drawn on a torch device (torch's generator: other
    numbers than mix_layer, same distributions), for study sizes that NumPy
    would take minutes to draw.  Returns (w fp32 [n, k], x bf16 [n_cal, k])."""
    import torch
    rho, beta = mix_layer_params(layer, seed)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed * 1000003 + layer)
    f32 = torch.float32
    v = torch.randn((MIX_RANK, k), generator=gen, device=device, dtype=f32) / MIX_RANK ** 0.5
    tau = torch.exp(torch.empty(k, device=device, dtype=f32).uniform_(np.log(0.25), np.log(4.0), generator=gen))
    z = torch.randn((n_cal, k), generator=gen, device=device, dtype=f32)
    g = torch.randn((n_cal, MIX_RANK), generator=gen, device=device, dtype=f32)
    x = tau[None, :] * ((1.0 - rho * rho) ** 0.5 * z + rho * (g @ v))
    s = torch.exp(torch.empty(n, device=device, dtype=f32).uniform_(np.log(0.005), np.log(0.05), generator=gen))
    a = torch.randn((n, MIX_RANK), generator=gen, device=device, dtype=f32)
    w = torch.randn((n, k), generator=gen, device=device, dtype=f32)
    w.add_(beta * (a @ v)).mul_(s[:, None])
    return w, x.to(torch.bfloat16)
