"""CPU oracle for the STQ1_0 quantized matmul -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this module.  The
library under ``sub_bit_sparse_b200/`` never imports it and has no CPU
fallback.

Plain, slow and obviously correct: NumPy, fp64 wherever a real number is
involved, no blocking or fusion beyond what the definitions say.  It shares no
code with the CUDA path.

Sources (page title, then the section):

* [LEM] lemmy.durstig.online post 66506 (Tencent Hunyuan quantization
  breakdown): "Four weights, five bits"; "Scale and zero position are fit
  together"; "Runtime".
* [AGI] "Tencent compresses 770B Hunyuan Hy4 Preview into 214 GiB at ~2.38
  bits per weight": "Four weights, five bits"; "Fitting and runtime".
* [TRA] "Tencent's 200GB Hy4-preview: a 7x compression claim that needs a
  second look": "MIX-STQ1_0: where the bits go".
* [ALS] "AngelSlim Shrinks Tencent's 1.5TB Hy4-Preview to 214 GiB at 6x
  Compression": "How STQ1_0 works" and the bullet list at the top.

What the pages fix: every group of four weights takes values in {-d, 0, +d}
with exactly one zero lane; 4 zero positions x 8 sign patterns = 32 patterns
in 5 bits [LEM "Four weights, five bits"]; the 5 bits are a 4-bit code plus a
1-bit table-select into a 32-entry codebook, and one fp16 scale is shared by
256 weights, 42 bytes per block, 1.3125 bits per weight [ALS "How STQ1_0
works"].  The original encoder scales by amax [ALS bullets]; the improved one
alternates a weighted-least-squares fit of d with an importance-weighted
choice of the zero lane, three rounds [LEM "Scale and zero position are fit
together"].

What the pages leave open, and the reading taken here (each is listed in the
design notes):

1. Block layout (little-endian, 42 bytes, no padding): bytes 0-1 the fp16
   scale d; bytes 2-33 ``qs[32]``, the 4-bit code of group g is
   ``(qs[g >> 1] >> 4 * (g & 1)) & 0xF``; bytes 34-41 ``qh[8]``, the select
   bit of group g is ``(qh[g >> 3] >> (g & 7)) & 1``.  Group g covers the
   columns 256 b + 4 g + l, l = 0..3.  Blocks are stored row-major: block
   (j, b) starts at byte (j * K / 256 + b) * 42.
2. Codebook: with n the 4-bit code and t the select bit, the zero lane is
   z = n >> 2; the other lanes in ascending order a < b < c carry +1, then
   -1 if bit 1 of n is set (else +1), then -1 if bit 0 of n is set (else
   +1); table t = 1 is the negation of table t = 0.
3. Plain encoder (E0): d = amax of the block, rounded to fp16; in each
   group the lane of smallest |w| is zeroed (ties: lowest lane) and the
   others take the sign of w (-0.0 counts as +).
4. Sherry encoder (E1): start from E0's zero lanes; each round fits d by
   weighted least squares over the non-zero lanes, then re-picks every
   group's zero lane as the one whose zeroing adds the least weighted error
   h_l * d * (2|w_l| - d) (ties: lowest lane); after the last round d is
   refit for the final zero lanes and rounded to fp16.  All in fp64,
   sums in ascending column order, the unrounded d between rounds.  If the
   importance of a whole block is zero the block uses h = 1; if a fit's
   denominator is zero that fit uses h = 1.
5. fp64 -> fp16 rounding is direct round-to-nearest-even, saturating at
   65504 instead of overflowing to infinity.
6. Matmul: y[t, j] = sum_k W^[j, k] x[t, k] with W^ = pattern * fp32(d).
   MoE gate/up: y[t, s, :] = W^_{ids[t, s]} x_t, unweighted unless flag bit 0
   asks to scale the up half (rows N/2..N-1) by the routing weight.
7. fp8 variant of the tile path (the pages have no fp8 step; the reading is
   this library's): each token row x_t is scaled by one fp32 factor to the
   e4m3 range, inv_t = 448 / amax_t and s_t = amax_t / 448 (both fp32
   divisions; 0 for an all-zero row), each element becomes the e4m3 code of
   the fp32 product x * inv_t, rounded to nearest with ties to the even code
   and saturated at +/-448 (OCP FP8 E4M3: no infinities, 0x7F / 0xFF NaN),
   and y = s_t * W^ q_t with q_t the codes' values.  Weights stay exact
   (+/-1 and 0 are e4m3 values, d is applied in fp32).
8. After gate/up (the pages stop there; the steps below are the plain reading
   of a gated MoE feed-forward): act = SiLU(g) * u with g = y[:, :N/2],
   u = y[:, N/2:] and SiLU(v) = v / (1 + e^-v), evaluated in fp64 and
   rounded once to bf16 (nearest, ties to even) because it is the bf16 input
   of the down projection; the down projection is the same STQ1_0 matmul per
   routed (token, slot) pair; the combine is sum_s w[t, s] * y_down[t, s]
   (or the plain sum when the weights were applied to the up half).
9. Mixed-precision allocation (the pages: per-layer bit widths picked by
   full-Hessian sensitivity, greedily by error reduction per added byte,
   between STQ1_0 and a 2.06-bpw partner format that is third-party): the
   partner here is STQ2, a format of this library at the same rate: per 256
   weights an fp16 scale d and 64 bytes of 2-bit codes (weight k at bits
   2 (k mod 4) of byte k / 4), code q meaning (2q - 3) d / 3, chosen as the
   nearest level (ties: the lower code).  The pages' partner is fitted with
   the importance matrix, so STQ2 is too: d starts at fp16(amax) and is then
   fit like the Sherry scale, by weighted least squares alternating with the
   code choice.  A layer's error under a
   format is tr(D H D^T) with D = W - W^ and H = X^T X over its calibration
   rows x; the diagonal (imatrix) score keeps only H's diagonal.  Greedy:
   start from STQ1_0 everywhere, upgrade layers in order of error reduction
   per added byte (ties: lower layer index) while the total stays within the
   byte budget; byte totals are summed in layer order, then grown one upgrade
   at a time.
"""

from __future__ import annotations

import struct
from typing import Iterable

import numpy as np

BLOCK_WEIGHTS = 256
GROUP = 4
GROUPS_PER_BLOCK = BLOCK_WEIGHTS // GROUP   # 64
BLOCK_BYTES = 42
OFF_D = 0
OFF_QS = 2
OFF_QH = 34
FP16_MAX = 65504.0

FLAG_WEIGHT_UP = 1


class OracleValueError(ValueError):
    """Non-finite weights, negative importance, or a shape the format cannot hold."""


# ---------------------------------------------------------------------------
# Codebook  [LEM "Four weights, five bits"], [ALS "How STQ1_0 works"]
# ---------------------------------------------------------------------------


def code_parts(code: int):
    """5-bit code -> (t, n, z, beta, gamma)."""
    t = (code >> 4) & 1
    n = code & 0xF
    return t, n, n >> 2, (n >> 1) & 1, n & 1


def pattern_of_code(code: int) -> list[int]:
    """The 4-lane pattern in {-1, 0, +1} that code ``code`` (0..31) stands for."""
    t, _, z, beta, gamma = code_parts(code)
    a, b, c = [lane for lane in range(GROUP) if lane != z]
    p = [0, 0, 0, 0]
    p[a] = 1
    p[b] = -1 if beta else 1
    p[c] = -1 if gamma else 1
    if t:
        p = [-v for v in p]
    return p


def codebook() -> np.ndarray:
    """All 32 patterns, int8 [32, 4], row = code."""
    return np.array([pattern_of_code(c) for c in range(32)], dtype=np.int8)


def code_of(z: int, negative: Iterable[bool]) -> int:
    """Encoder side: zero lane z and the sign of each lane (True = negative) -> code.

    t is the sign of the first non-zero lane; bits 1 and 0 of n say whether
    the second and third non-zero lanes differ in sign from the first.
    """
    neg = list(negative)
    a, b, c = [lane for lane in range(GROUP) if lane != z]
    t = 1 if neg[a] else 0
    bit1 = 1 if neg[b] != neg[a] else 0
    bit0 = 1 if neg[c] != neg[a] else 0
    return (t << 4) | (z << 2) | (bit1 << 1) | bit0


def _code_table() -> np.ndarray:
    """[4 zero lanes, 16 sign masks] -> code; sign mask bit l = lane l negative."""
    tab = np.zeros((GROUP, 16), dtype=np.uint8)
    for z in range(GROUP):
        for m in range(16):
            tab[z, m] = code_of(z, [(m >> lane) & 1 == 1 for lane in range(GROUP)])
    return tab


_CODE_TABLE = _code_table()
_CODEBOOK_F64 = codebook().astype(np.float64)


def codes_from_choice(zero_lane: np.ndarray, w_groups: np.ndarray) -> np.ndarray:
    """Vectorised ``code_of``: zero_lane [..., 64] int, w_groups [..., 64, 4] fp -> codes uint8."""
    neg = (w_groups < 0).astype(np.int64)   # -0.0 < 0 is False: counts as +
    mask = neg[..., 0] | (neg[..., 1] << 1) | (neg[..., 2] << 2) | (neg[..., 3] << 3)
    return _CODE_TABLE[zero_lane, mask]


# ---------------------------------------------------------------------------
# fp16 / bf16 rounding
# ---------------------------------------------------------------------------


def fp16_bits(x) -> np.ndarray:
    """fp64 -> fp16 bits, round to nearest even, saturating at +/-65504.

    NumPy's float64 -> float16 cast rounds once, directly from double.  NaN or
    infinite inputs raise ``OracleValueError``.
    """
    x = np.asarray(x, dtype=np.float64)
    if not np.all(np.isfinite(x)):
        raise OracleValueError("non-finite value cannot be stored as an STQ1_0 scale")
    with np.errstate(over="ignore"):
        h = x.astype(np.float16)
    h = np.where(np.isinf(h), np.copysign(np.float16(FP16_MAX), x), h).astype(np.float16)
    return h.view(np.uint16)


def fp16_value(bits) -> np.ndarray:
    """fp16 bits -> fp64 (exact)."""
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def bf16_bits_rne(x32: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bits, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((u + (((u >> 16) & 1) + 0x7FFF)) >> 16).astype(np.uint16)


def bf16_to_f64(bits) -> np.ndarray:
    """bf16 bits -> fp64 (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# Block packing (layout reading 1)
# ---------------------------------------------------------------------------


def pack_blocks(d_bits: np.ndarray, codes: np.ndarray) -> np.ndarray:
    """d_bits uint16 [B], codes uint8 [B, 64] -> bytes uint8 [B * 42]."""
    d_bits = np.asarray(d_bits, dtype=np.uint16).reshape(-1)
    codes = np.asarray(codes, dtype=np.uint8).reshape(-1, GROUPS_PER_BLOCK)
    nb = d_bits.shape[0]
    out = np.zeros((nb, BLOCK_BYTES), dtype=np.uint8)
    out[:, OFF_D] = d_bits & 0xFF
    out[:, OFF_D + 1] = d_bits >> 8
    n = codes & 0xF
    t = (codes >> 4) & 1
    for g in range(GROUPS_PER_BLOCK):
        out[:, OFF_QS + (g >> 1)] |= (n[:, g] << (4 * (g & 1))).astype(np.uint8)
        out[:, OFF_QH + (g >> 3)] |= (t[:, g] << (g & 7)).astype(np.uint8)
    return out.reshape(-1)


def unpack_blocks(packed: np.ndarray):
    """bytes uint8 [B * 42] -> (d_bits uint16 [B], codes uint8 [B, 64])."""
    blk = np.asarray(packed, dtype=np.uint8).reshape(-1, BLOCK_BYTES)
    d_bits = blk[:, OFF_D].astype(np.uint16) | (blk[:, OFF_D + 1].astype(np.uint16) << 8)
    codes = np.zeros((blk.shape[0], GROUPS_PER_BLOCK), dtype=np.uint8)
    for g in range(GROUPS_PER_BLOCK):
        n = (blk[:, OFF_QS + (g >> 1)] >> (4 * (g & 1))) & 0xF
        t = (blk[:, OFF_QH + (g >> 3)] >> (g & 7)) & 1
        codes[:, g] = n | (t << 4)
    return d_bits, codes


def packed_size(n: int, k: int) -> int:
    """Bytes of an [n, k] STQ1_0 matrix."""
    return n * (k // BLOCK_WEIGHTS) * BLOCK_BYTES


def _as_blocks(w: np.ndarray) -> np.ndarray:
    """[N, K] -> [N * K / 256, 64, 4] in block storage order (row-major blocks)."""
    n, k = w.shape
    if k % BLOCK_WEIGHTS:
        raise OracleValueError("K must be a multiple of 256")
    return w.reshape(n * (k // BLOCK_WEIGHTS), GROUPS_PER_BLOCK, GROUP)


# ---------------------------------------------------------------------------
# E0: the plain amax encoder  [ALS bullets], [AGI "Fitting and runtime"]
# ---------------------------------------------------------------------------


def encode_plain(w: np.ndarray) -> np.ndarray:
    """Amax-scaled ternary encoding with the smallest-magnitude lane zeroed."""
    w = np.asarray(w, dtype=np.float32)
    if not np.all(np.isfinite(w)):
        raise OracleValueError("non-finite weight")
    blocks = _as_blocks(w)
    aw = np.abs(blocks)
    amax = aw.reshape(blocks.shape[0], -1).max(axis=1).astype(np.float64)
    d_bits = fp16_bits(amax)
    z = np.argmin(aw, axis=2)              # first minimum: lowest lane on ties
    codes = codes_from_choice(z, blocks)
    return pack_blocks(d_bits, codes)


# ---------------------------------------------------------------------------
# E1: the Sherry encoder  [LEM "Scale and zero position are fit together"]
# ---------------------------------------------------------------------------


def _nonzero_mask(z: np.ndarray) -> np.ndarray:
    """zero lanes [B, 64] -> bool [B, 256], True on the lanes that stay non-zero."""
    lanes = np.arange(GROUP)[None, None, :]
    return (lanes != z[:, :, None]).reshape(z.shape[0], BLOCK_WEIGHTS)


def wls_scale(aw: np.ndarray, h: np.ndarray, z: np.ndarray) -> np.ndarray:
    """Weighted least-squares scale for fixed zero lanes.

    With s_k = sign(w_k) on the non-zero lanes, the minimiser of
    sum_k h_k (w_k - d s_k)^2 is d = sum h_k |w_k| / sum h_k over those lanes.
    Sums run over k in ascending order (sequential fp64).  A zero denominator
    falls back to h = 1 for that fit.  aw, h: fp64 [B, 256]; z: [B, 64].
    """
    nz = _nonzero_mask(z)
    num = np.zeros(aw.shape[0])
    den = np.zeros(aw.shape[0])
    num1 = np.zeros(aw.shape[0])
    for k in range(BLOCK_WEIGHTS):
        m = nz[:, k]
        num = num + np.where(m, h[:, k] * aw[:, k], 0.0)
        den = den + np.where(m, h[:, k], 0.0)
        num1 = num1 + np.where(m, aw[:, k], 0.0)
    zero_den = den == 0.0
    count = float(BLOCK_WEIGHTS - GROUPS_PER_BLOCK)
    safe_den = np.where(zero_den, 1.0, den)
    return np.where(zero_den, num1 / count, num / safe_den)


def zero_lane_choice(aw: np.ndarray, h: np.ndarray, d: np.ndarray) -> np.ndarray:
    """Per group, the lane whose zeroing adds the least weighted error.

    Zeroing lane l instead of giving it sign(w_l) * d raises h_l * w_l^2 -
    h_l * (|w_l| - d)^2 = h_l * d * (2|w_l| - d); evaluated as
    (h_l * d) * (2 |w_l| - d).  Ties go to the lowest lane.
    """
    B = aw.shape[0]
    a4 = aw.reshape(B, GROUPS_PER_BLOCK, GROUP)
    h4 = h.reshape(B, GROUPS_PER_BLOCK, GROUP)
    dd = d[:, None, None]
    delta = (h4 * dd) * (2.0 * a4 - dd)
    return np.argmin(delta, axis=2)


def weighted_error(w_blocks: np.ndarray, h: np.ndarray, d: np.ndarray, z: np.ndarray) -> np.ndarray:
    """sum_k h_k (w_k - d s_k)^2 per block for zero lanes z and s_k = sign(w_k) (fp64)."""
    aw = np.abs(w_blocks.reshape(w_blocks.shape[0], -1).astype(np.float64))
    nz = _nonzero_mask(z)
    r = np.where(nz, aw - d[:, None], aw)
    return np.sum(h * r * r, axis=1)


def encode_sherry(w: np.ndarray, h: np.ndarray | None = None, rounds: int = 3, trace: bool = False):
    """Alternating WLS scale / importance-weighted zero placement, ``rounds`` rounds.

    ``h`` is the per-column importance (diagonal imatrix), shared by all rows;
    ``None`` means h = 1.  With ``trace=True`` also returns the per-round
    scales and zero lanes (for the brute-force checks).
    """
    w = np.asarray(w, dtype=np.float32)
    if not np.all(np.isfinite(w)):
        raise OracleValueError("non-finite weight")
    n, k = w.shape
    blocks = _as_blocks(w)
    B = blocks.shape[0]
    if h is None:
        hcol = np.ones(k)
    else:
        hcol = np.asarray(h, dtype=np.float32).astype(np.float64)
        if hcol.shape != (k,) or not np.all(np.isfinite(hcol)) or np.any(hcol < 0):
            raise OracleValueError("importance must be finite, >= 0, one value per column")
    hb = np.broadcast_to(hcol.reshape(1, k), (n, k)).reshape(B, BLOCK_WEIGHTS).copy()
    all_zero = ~np.any(hb != 0.0, axis=1)
    hb[all_zero] = 1.0
    aw = np.abs(blocks.reshape(B, BLOCK_WEIGHTS).astype(np.float64))

    z = np.argmin(np.abs(blocks), axis=2)     # round 0: E0's zero lanes
    hist = [(None, z.copy())]
    for _ in range(rounds):
        d = wls_scale(aw, hb, z)
        z = zero_lane_choice(aw, hb, d)
        hist.append((d.copy(), z.copy()))
    d_final = wls_scale(aw, hb, z)
    packed = pack_blocks(fp16_bits(d_final), codes_from_choice(z, blocks))
    if trace:
        return packed, {"rounds": hist, "d_final": d_final, "h_blocks": hb}
    return packed


# ---------------------------------------------------------------------------
# Decoder and dequantization
# ---------------------------------------------------------------------------


def decode(packed: np.ndarray, n: int, k: int) -> np.ndarray:
    """STQ1_0 bytes -> W^ fp64 [n, k], W^ = pattern * fp32(d) (exact)."""
    if k % BLOCK_WEIGHTS:
        raise OracleValueError("K must be a multiple of 256")
    d_bits, codes = unpack_blocks(packed)
    if d_bits.shape[0] != n * (k // BLOCK_WEIGHTS):
        raise OracleValueError("packed size does not match the shape")
    d = fp16_value(d_bits)
    pat = _CODEBOOK_F64[codes]                # [B, 64, 4]
    return (pat * d[:, None, None]).reshape(n, k)


def dequant_bf16(packed: np.ndarray, n: int, k: int) -> np.ndarray:
    """W^ as bf16 bits: bf16_RNE(fp32(d)) with the pattern's sign; zero lanes are +0.0."""
    d_bits, codes = unpack_blocks(packed)
    d32 = fp16_value(d_bits).astype(np.float32)
    mag = bf16_bits_rne(d32)                  # d >= 0 for every encoder here; sign kept if not
    pat = codebook()[codes]                   # [B, 64, 4]
    magb = np.broadcast_to(mag[:, None, None], pat.shape)
    out = np.where(pat == 0, np.uint16(0),
                   np.where(pat < 0, magb ^ np.uint16(0x8000), magb)).astype(np.uint16)
    return out.reshape(n, k)


# ---------------------------------------------------------------------------
# Contractions  [LEM "Runtime"]
# ---------------------------------------------------------------------------


def gemv(packed: np.ndarray, x_bits: np.ndarray, n: int, k: int) -> np.ndarray:
    """y [b, n] = W^ x, fp64 (x: bf16 bits [b, k])."""
    w = decode(packed, n, k)
    x = bf16_to_f64(np.asarray(x_bits).reshape(-1, k))
    return x @ w.T


def gemv_abs(packed: np.ndarray, x_bits: np.ndarray, n: int, k: int) -> np.ndarray:
    """sum_k |W^[j, k] x[t, k]|, the scale of the tolerance bound, fp64 [b, n]."""
    w = np.abs(decode(packed, n, k))
    x = np.abs(bf16_to_f64(np.asarray(x_bits).reshape(-1, k)))
    return x @ w.T


def tolerance(abs_sum: np.ndarray) -> np.ndarray:
    """|y_gpu - y_oracle| <= 1e-3 * sum|W x| + 1e-6."""
    return 1e-3 * abs_sum + 1e-6


def route_pairs(ids: np.ndarray, n_experts: int):
    """Token-slot pairs grouped by expert: (counts [E], offsets [E + 1], pairs sorted by
    (expert, pair index)).  Pair index p = t * topk + s."""
    ids = np.asarray(ids, dtype=np.int64)
    if np.any(ids < 0) or np.any(ids >= n_experts):
        raise OracleValueError("expert id out of range")
    flat = ids.reshape(-1)
    counts = np.bincount(flat, minlength=n_experts)
    offsets = np.concatenate([[0], np.cumsum(counts)])
    order = np.argsort(flat, kind="stable")
    return counts, offsets, order


def moe_gateup(expert_packed, x_bits: np.ndarray, ids: np.ndarray, weights: np.ndarray,
               n: int, k: int, flags: int = 0, abs_sum: bool = False):
    """y [T, topk, n] with y[t, s] = W^_{ids[t, s]} x_t (fp64).

    ``expert_packed(e)`` returns expert e's bytes (or pass a list/array indexed by e).
    Flag bit 0 scales the up half (rows n/2 .. n-1) by weights[t, s].
    With ``abs_sum=True`` also returns sum_k |W^ x| for the tolerance.
    """
    x = bf16_to_f64(np.asarray(x_bits).reshape(np.asarray(ids).shape[0], k))
    return _moe_from_f64(expert_packed, x, ids, weights, n, k, flags, abs_sum)


def _moe_from_f64(expert_packed, x: np.ndarray, ids, weights, n: int, k: int, flags: int, abs_sum: bool):
    """MoE gate/up on fp64 activations x [T, k]."""
    ids = np.asarray(ids)
    T, topk = ids.shape
    get = expert_packed if callable(expert_packed) else (lambda e: expert_packed[e])
    y = np.zeros((T, topk, n))
    ya = np.zeros((T, topk, n)) if abs_sum else None
    for e in np.unique(ids):
        tt, ss = np.nonzero(ids == e)
        w = decode(get(int(e)), n, k)
        y[tt, ss] = x[tt] @ w.T
        if abs_sum:
            ya[tt, ss] = np.abs(x[tt]) @ np.abs(w).T
    if flags & FLAG_WEIGHT_UP:
        wt = np.asarray(weights, dtype=np.float32).astype(np.float64)[:, :, None]
        y[:, :, n // 2:] *= wt
        if abs_sum:
            ya[:, :, n // 2:] *= np.abs(wt)
    return (y, ya) if abs_sum else y


# ---------------------------------------------------------------------------
# fp8 (e4m3) activations for the fp8 tile variant (reading 7)
# ---------------------------------------------------------------------------

E4M3_MAX = 448.0


def e4m3_value(codes) -> np.ndarray:
    """OCP FP8 E4M3 code -> fp64: sign bit 7, exponent bits 3-6 (bias 7), mantissa bits 0-2;
    exponent 0 is subnormal (m / 8 * 2^-6); codes 0x7F and 0xFF are NaN."""
    c = np.asarray(codes, dtype=np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    mag = np.where((e == 15) & ((c & 0x7) == 7), np.nan, mag)
    return sign * mag


def e4m3_round(v) -> np.ndarray:
    """fp32 values -> E4M3 codes: nearest value, ties to the even code, magnitudes above 448
    saturate to 448; the sign bit follows the input's (so -0.0 -> 0x80).  Finite inputs."""
    v = np.asarray(v, dtype=np.float32).astype(np.float64)
    a = np.abs(v)
    _, ex = np.frexp(a)                       # a = f * 2^ex with f in [0.5, 1), or a = 0
    e = np.maximum(ex - 1, -6)                # a in [2^e, 2^(e+1)); below 2^-6 one subnormal step
    step = np.exp2(e - 3.0)                   # 8 values per binade
    r = np.rint(a / step)                     # ties to the even multiple = the even mantissa
    q = np.minimum(r * step, E4M3_MAX)
    # q is an E4M3 magnitude: encode it
    _, qx = np.frexp(q)
    qe = qx - 1                               # q in [2^qe, 2^(qe+1)) for q > 0
    normal = q >= 2.0 ** -6
    exp_field = np.where(normal, qe + 7, 0)
    man = np.where(normal, q / np.exp2(qe.astype(np.float64)) * 8.0 - 8.0, q / 2.0 ** -9)
    code = (exp_field.astype(np.int64) << 3) | np.rint(man).astype(np.int64)
    code = np.where(q == 0, 0, code)
    return (code | np.where(np.signbit(v), 0x80, 0)).astype(np.uint8)


def quantize_x_e4m3(x_bits: np.ndarray):
    """bf16 rows [T, K] -> (E4M3 codes uint8 [T, K], scales fp32 [T]) per reading 7."""
    x = bf16_to_f64(np.asarray(x_bits)).astype(np.float32)
    x = x.reshape(x.shape[0], -1)
    amax = np.max(np.abs(x), axis=1)
    with np.errstate(divide="ignore"):
        inv = np.where(amax > 0, np.float32(E4M3_MAX) / amax, np.float32(0.0)).astype(np.float32)
    s = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    v = (x * inv[:, None]).astype(np.float32)
    return e4m3_round(v), s


def moe_gateup_fp8(expert_packed, x_bits: np.ndarray, ids: np.ndarray, weights: np.ndarray,
                   n: int, k: int, flags: int = 0, abs_sum: bool = False):
    """The fp8 variant of ``moe_gateup``: x_t replaced by s_t * q_t (reading 7), fp64."""
    codes, s = quantize_x_e4m3(np.asarray(x_bits).reshape(-1, k))
    xq = e4m3_value(codes) * s.astype(np.float64)[:, None]
    return _moe_from_f64(expert_packed, xq, ids, weights, n, k, flags, abs_sum)


# ---------------------------------------------------------------------------
# After gate/up: SwiGLU, down projection, combine (reading 8)
# ---------------------------------------------------------------------------


def bf16_bits_from_f64(x) -> np.ndarray:
    """fp64 -> bf16 bits directly (no fp32 step): nearest, ties to even; 8 significant
    bits, exponent range of fp32, subnormal quantum 2^-133; overflow to +/-inf."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    sign = np.where(np.signbit(x), 0x8000, 0).astype(np.int64)
    _, ex = np.frexp(a)
    e = np.maximum(ex - 1, -126)               # a in [2^e, 2^(e+1)), subnormals share 2^-126's step
    step = np.exp2(e - 7.0)
    q = np.rint(a / step) * step               # ties to the even multiple
    _, qx = np.frexp(q)
    qe = qx - 1
    normal = q >= 2.0 ** -126
    man = np.where(normal, q / np.exp2(qe.astype(np.float64)) * 128.0 - 128.0, q / 2.0 ** -133)
    bits = np.where(normal, ((qe + 127).astype(np.int64) << 7) | np.rint(man).astype(np.int64),
                    np.rint(man).astype(np.int64))
    bits = np.where(q == 0, 0, bits)
    bits = np.where(q >= 2.0 ** 128, 0x7F80, bits)
    return (bits | sign).astype(np.uint16)


def silu(v) -> np.ndarray:
    """SiLU(v) = v / (1 + e^-v) in fp64."""
    v = np.asarray(v, dtype=np.float64)
    with np.errstate(over="ignore"):
        return v / (1.0 + np.exp(-v))


def swiglu_bf16(y: np.ndarray, n: int) -> np.ndarray:
    """Fused gate/up rows y [P, n] (fp64 or fp32) -> act bf16 bits [P, n/2] = bf16(SiLU(g) * u)."""
    y = np.asarray(y, dtype=np.float64).reshape(-1, n)
    g, u = y[:, : n // 2], y[:, n // 2:]
    return bf16_bits_from_f64(silu(g) * u)


def moe_combine(y_down: np.ndarray, weights) -> np.ndarray:
    """[T, topk, H] -> [T, H]: sum over slots, weighted by weights[t, s] when given (fp64)."""
    yd = np.asarray(y_down, dtype=np.float64)
    if weights is None:
        return yd.sum(axis=1)
    w = np.asarray(weights, dtype=np.float32).astype(np.float64)
    return np.einsum("ts,tsh->th", w, yd)


def moe_ffn(gateup_packed, down_packed, x_bits, ids, weights, n: int, hidden: int, flags: int = 0,
            abs_sum: bool = False):
    """Routed MoE feed-forward: gate/up -> SwiGLU (bf16) -> down -> combine, fp64 (reading 8).

    ``flags`` bit 0 applies the routing weight to the up half (and the combine is then a plain sum);
    otherwise the combine applies it.  With ``abs_sum`` also returns sum|W_down act| * |w| summed
    over slots, the scale of the tolerance for the final output.
    """
    ids = np.asarray(ids)
    T, topk = ids.shape
    y = moe_gateup(gateup_packed, x_bits, ids, weights, n, hidden, flags=flags)
    act = swiglu_bf16(y.reshape(T * topk, n), n)             # [P, n/2] bf16 bits
    flat_ids = ids.reshape(T * topk, 1)
    yd, ya = moe_gateup(down_packed, act, flat_ids, None, hidden, n // 2, abs_sum=True)
    yd = yd.reshape(T, topk, hidden)
    ya = ya.reshape(T, topk, hidden)
    w = None if flags & FLAG_WEIGHT_UP else weights
    out = moe_combine(yd, w)
    if not abs_sum:
        return out
    wa = np.ones((T, topk)) if w is None else np.abs(np.asarray(w, dtype=np.float32).astype(np.float64))
    return out, np.einsum("ts,tsh->th", wa, ya)


# ---------------------------------------------------------------------------
# Mixed-precision allocation (reading 9)
# ---------------------------------------------------------------------------

STQ2_BLOCK_BYTES = 66


def _stq2_levels(d: np.ndarray) -> np.ndarray:
    """[B] fp64 scales -> [B, 4] levels (d * (2q - 3)) / 3."""
    return d[:, None] * (2.0 * np.arange(4) - 3.0)[None, :] / 3.0


def stq2_codes(wb: np.ndarray, d: np.ndarray) -> np.ndarray:
    """Nearest level per weight (ties: the lower code).  wb fp64 [B, 256], d fp64 [B]."""
    dist = np.abs(wb[:, :, None] - _stq2_levels(d)[:, None, :])
    return np.argmin(dist, axis=2)                                           # first minimum


def stq2_wls_scale(wb: np.ndarray, hb: np.ndarray, q: np.ndarray) -> np.ndarray:
    """Weighted least-squares scale for fixed codes: with m_k = 2 q_k - 3 the level
    of weight k is d m_k / 3, and the minimiser of sum_k h_k (w_k - d m_k / 3)^2 is
    d = 3 sum h_k w_k m_k / sum h_k m_k^2, summed over k ascending (sequential fp64)."""
    m = 2.0 * q - 3.0
    num = np.zeros(wb.shape[0])
    den = np.zeros(wb.shape[0])
    for k in range(BLOCK_WEIGHTS):
        num = num + (hb[:, k] * wb[:, k]) * m[:, k]
        den = den + hb[:, k] * (m[:, k] * m[:, k])
    return (3.0 * num) / den


def stq2_weighted_error(wb: np.ndarray, hb: np.ndarray, d: np.ndarray, q: np.ndarray) -> np.ndarray:
    """sum_k h_k (w_k - d m_k / 3)^2 per block (fp64)."""
    lev = np.take_along_axis(_stq2_levels(d), q, axis=1)
    return np.sum(hb * (wb - lev) ** 2, axis=1)


def encode_stq2(w: np.ndarray, h: np.ndarray | None = None, rounds: int = 0, trace: bool = False):
    """[N, K] fp32 -> STQ2 bytes.

    rounds = 0: d = fp16(amax), codes nearest at that d.  rounds > 0: starting
    from those codes, ``rounds`` times fit d by weighted least squares (h per
    column; None means h = 1; a block whose h is all zero uses h = 1) and
    re-pick the nearest levels at that d; then store fp16 of one more fit.
    """
    w = np.asarray(w, dtype=np.float32)
    if not np.all(np.isfinite(w)):
        raise OracleValueError("non-finite weight")
    n, k = w.shape
    wb = w.reshape(-1, BLOCK_WEIGHTS).astype(np.float64)
    B = wb.shape[0]
    if h is None:
        hcol = np.ones(k)
    else:
        hcol = np.asarray(h, dtype=np.float32).astype(np.float64)
        if hcol.shape != (k,) or not np.all(np.isfinite(hcol)) or np.any(hcol < 0):
            raise OracleValueError("importance must be finite, >= 0, one value per column")
    hb = np.broadcast_to(hcol.reshape(1, k), (n, k)).reshape(B, BLOCK_WEIGHTS).copy()
    hb[~np.any(hb != 0.0, axis=1)] = 1.0
    d_bits = fp16_bits(np.max(np.abs(wb), axis=1))
    d = fp16_value(d_bits)
    q = stq2_codes(wb, d)
    hist = [(d.copy(), q.copy())]
    if rounds > 0:
        for _ in range(rounds):
            d = stq2_wls_scale(wb, hb, q)
            q = stq2_codes(wb, d)
            hist.append((d.copy(), q.copy()))
        d_bits = fp16_bits(stq2_wls_scale(wb, hb, q))
    out = np.zeros((B, STQ2_BLOCK_BYTES), dtype=np.uint8)
    out[:, 0] = d_bits & 0xFF
    out[:, 1] = d_bits >> 8
    qq = q.astype(np.uint32).reshape(B, 64, 4)
    out[:, 2:] = (qq[:, :, 0] | (qq[:, :, 1] << 2) | (qq[:, :, 2] << 4) | (qq[:, :, 3] << 6)).astype(np.uint8)
    out = out.reshape(-1)
    if trace:
        return out, {"rounds": hist, "h_blocks": hb}
    return out


def decode_stq2(packed: np.ndarray, n: int, k: int) -> np.ndarray:
    """STQ2 bytes -> [n, k] fp64."""
    b = np.asarray(packed, dtype=np.uint8).reshape(-1, STQ2_BLOCK_BYTES)
    d = fp16_value(b[:, 0].astype(np.uint16) | (b[:, 1].astype(np.uint16) << 8))
    codes = np.stack([(b[:, 2:] >> (2 * i)) & 3 for i in range(4)], axis=2).reshape(-1, BLOCK_WEIGHTS)
    return (d[:, None] * (2.0 * codes - 3.0) / 3.0).reshape(n, k)


def hessian_error(w: np.ndarray, w_hat: np.ndarray, x: np.ndarray) -> float:
    """tr(D H D^T) with D = w - w_hat [N, K] and H = x^T x, x [n_cal, K] (fp64).

    Evaluated as the sum over calibration rows of the squared outputs of D,
    sum_c ||D x_c||^2, which is the same number (tr(D X^T X D^T) = ||X D^T||_F^2)
    without forming the K x K matrix H."""
    d = np.asarray(w, dtype=np.float64) - np.asarray(w_hat, dtype=np.float64)
    y = np.asarray(x, dtype=np.float64) @ d.T
    return float(np.sum(y * y))


def diagonal_error(w: np.ndarray, w_hat: np.ndarray, x: np.ndarray) -> float:
    """The imatrix score: sum_k H_kk D_jk^2 over rows j."""
    d = np.asarray(w, dtype=np.float64) - np.asarray(w_hat, dtype=np.float64)
    hd = np.sum(np.asarray(x, dtype=np.float64) ** 2, axis=0)
    return float(np.sum(d * d * hd[None, :]))


def greedy_allocate(err_low, err_high, bytes_low, bytes_high, budget) -> np.ndarray:
    """Per layer: True = the higher-bit format.  Start all low; upgrade in order of
    (err_low - err_high) / (bytes_high - bytes_low), descending (ties: lower index),
    while the total bytes stay within the budget (a layer that does not fit is skipped)."""
    el, eh = np.asarray(err_low, float), np.asarray(err_high, float)
    bl, bh = np.asarray(bytes_low, float), np.asarray(bytes_high, float)
    gain = (el - eh) / (bh - bl)
    order = sorted(range(len(el)), key=lambda i: (-gain[i], i))
    pick = np.zeros(len(el), dtype=bool)
    total = 0.0
    for v in bl:                         # left to right, one rounding per addition
        total += float(v)
    for i in order:
        if gain[i] <= 0:
            break
        cost = float(bh[i] - bl[i])
        if total + cost <= budget:
            pick[i] = True
            total += cost
    return pick


def half_from_struct(x: float) -> int:
    """IEEE binary16 bits of x via Python's struct (round-half-even), for cross-checks."""
    return struct.unpack("<H", struct.pack("<e", x))[0]
