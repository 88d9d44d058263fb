"""Plain CPU oracle for layer-wise GPTQ / RTN 4-bit weight quantization.

TEST INFRASTRUCTURE ONLY -- see the package docstring.  Float work is fp64
except where the method takes an integer decision (a quantisation code, a
stored 16-bit scale): those decisions are taken in IEEE float32 with the same
operation order as the kernels, so both sides decide in the same precision.

Sources (page title -- section):

* [RTN]  "GPT-2 Quantization Reconstruction Error" -- "What this project
  does": 4-bit symmetric per-channel quantisation, one scale per output row,
  15 discrete levels, dequantised back to float; per-layer output MSE.
* [AFF]  "Model Quantization Mechanics: Precision Reduction and Weight
  Formatting" -- section 1: affine quantisation W_q = round(W/S) + Z,
  W_deq = S (W_q - Z); group-wise quantisation with g = 128.  Section 2.1:
  objective ||WX - W^X||^2; Cholesky decomposition of the inverse Hessian.
* [OBQ]  "GPTQ: Post-Training INT4" -- "OBQ Foundation" (objective),
  "Hessian-Based Weight Update" (H = 2 X X^T, OBS update), "The GPTQ
  Algorithm" (fixed left-to-right order, lazy blocks of B = 128 columns, the
  scaled error and the in-block / trailing updates), "Group Quantization"
  (groups of consecutive weights; 4.25 / 4.125 bits per weight), "Running
  GPTQ with AutoGPTQ" (damp_percent, desc_act, sym).
* [LES]  "GPTQ and AWQ" (Inference and Serving, lesson 17) -- "Your turn"
  (the 0.26 / 0.26 pair) and "Example 1.1" (rounding with the error carried
  forward).

Readings taken where the pages are silent, ambiguous or garbled:

1. H = 2 X^T X with X stored tokens x d_in (the listing's orientation); no
   1/N normalisation.  Codes are invariant to a positive scale of H.
2. Damping: H_jj += damp * mean(diag H) with damp = 0.01 (the AutoGPTQ
   config's damp_percent), not the listing's fixed 1e-6 * I.
3. Dead columns (H_jj == 0): H_jj := 1 and W[:, j] := 0, before damping.
4. The listing's "H_inv" is read as the upper Cholesky factor U of H^-1
   (H^-1 = U^T U): h_inv_jj -> U_jj, H_inv[j, j+1:] -> U[j, j+1:].  This is
   what section 2.1 of the quantisation-mechanics page describes, and only
   this form equals the OBS update (checked against ``obs_quantize``).
5. The OBS update prints H where H_F^-1 is meant: delta_F =
   -(w_q - q^) [H_F^-1]_{F,q} / [H_F^-1]_qq.
6. quantize_to_int on one column: a group's scale (and zero) is computed
   from that group's *current* (already updated) weights when the group's
   first column is reached; for per-channel (group_size = -1) once from the
   initial row.  group_size must divide block_size.
7. Symmetric grid: 15 levels -7..7, s = absmax / 7.  Affine grid: 0..15,
   s = (max' - min') / 15 with min' = min(min, 0), max' = max(max, 0),
   z = rint(-min' / s).  The 16-bit scale is used for quantising and
   dequantising.  A scale that is 0 in fp16 (all-zero group, or underflow)
   becomes 1 with z = 0; a scale above the fp16 range saturates to 65504.
8. Rounding is round-half-to-even.
9. Act-order: perm = stable argsort(-diag H) after damping; groups are
   consecutive columns in permuted order; g_idx[c] is the group of original
   column c; codes are returned in original column order.
10. Activation-aware scaling ("Model Quantization Mechanics", section 2.2;
   "GPT-2 Quantization Reconstruction Error", "Possible extensions"): the
   pages say only that input channel c's weights are multiplied by a
   per-channel s_c chosen from the magnitude of that channel's activations,
   and the activations divided by it.  Read as: magnitude a_c = the RMS of
   x_c, taken from the undamped Hessian (H_cc = 2 sum_t x_tc^2); s_c =
   (a_c / a_bar)^alpha with a_bar the geometric mean of the non-zero a_c
   (s_c = 1 for a dead channel); alpha from the grid k / n_grid, k = 0 ..
   n_grid - 1, the one with the smallest layer MSE (first on ties); the
   quantised weights are RTN(W diag(s)) and the layer's effective weights
   W^ = dequant(RTN(W diag(s))) diag(s)^-1.  alpha = 0 is plain RTN.
"""
from __future__ import annotations

import itertools
from dataclasses import dataclass

import numpy as np

F32 = np.float32
F16_MAX = F32(65504.0)

__all__ = [
    "hessian", "hessian_entries", "damp_hessian", "act_order_perm",
    "upper_factor_of_inverse", "sym_params", "affine_params", "quantize_codes",
    "dequantize_codes", "code_offset", "pack_nibbles", "unpack_nibbles", "rtn_quantize",
    "GptqResult", "gptq_quantize", "dequantize_packed", "recon_sse",
    "recon_sse_trace", "bits_per_weight", "obs_quantize", "bruteforce_row",
    "round_to_grid", "round_error_carried_forward", "gptq_fixed_grid",
    "gptq_layer", "awq_channel_scales", "awq_apply", "awq_rtn_search", "w4a16_matmul",
    "round_to_bf16", "gelu_tanh", "apply_layer", "gptq_sequential", "TIE_TOL", "TIE_REL",
    "QUOT_REL",
]


# --------------------------------------------------------------------------
# Hessian, damping, act-order, inverse factor
# --------------------------------------------------------------------------

def hessian(X) -> np.ndarray:
    """H = 2 X^T X in fp64 ("GPTQ: Post-Training INT4", "Hessian-Based Weight
    Update"; X is tokens x d_in as in the listing of "The GPTQ Algorithm").

    X holds bf16 values (any float dtype that represents them exactly)."""
    X64 = np.asarray(X, dtype=np.float64)
    return 2.0 * (X64.T @ X64)


def hessian_entries(X, rows, cols) -> np.ndarray:
    """The sub-block H[rows][:, cols] of H = 2 X^T X, each entry computed
    straight from its definition (for sampled checks at large sizes)."""
    X64 = np.asarray(X, dtype=np.float64)
    return 2.0 * (X64[:, rows].T @ X64[:, cols])


def damp_hessian(H, damp_percent=0.01):
    """Dead-column fix, then H_jj += damp * mean(diag H).

    Damping follows the damp_percent knob of "GPTQ: Post-Training INT4" --
    "Running GPTQ with AutoGPTQ" (reading 2); dead columns are reading 3.
    Returns (H_damped, dead_mask)."""
    H = np.array(H, dtype=np.float64, copy=True)
    d = H.shape[0]
    diag = np.diag(H).copy()
    dead = diag == 0.0
    idx = np.arange(d)
    H[idx[dead], idx[dead]] = 1.0
    lam = damp_percent * np.mean(np.diag(H))
    H[idx, idx] += lam
    return H, dead


def act_order_perm(H_damped, follow=None, key_tol=1e-6):
    """Columns in order of descending diag H, ties by lower index first
    (desc_act of "Running GPTQ with AutoGPTQ"; reading 9).

    ``follow`` (optional): another implementation's order.  Keys that differ
    by less than ``key_tol`` (relative) are ties at the precision that
    implementation computes H in, and either order of them is correct; the
    other order is adopted when every adjacent pair of it is descending up
    to that tolerance.  Returns the order, or (order, adopted) with
    ``follow``."""
    key = np.diag(np.asarray(H_damped, dtype=np.float64))
    perm = np.argsort(-key, kind="stable").astype(np.int64)
    if follow is None:
        return perm
    f = np.asarray(follow, dtype=np.int64)
    ok = (np.array_equal(np.sort(f), np.arange(len(key)))
          and np.all(key[f[1:]] <= key[f[:-1]] * (1.0 + key_tol)))
    if ok and not np.array_equal(f, perm):
        return f.copy(), True
    return perm, False


def upper_factor_of_inverse(H) -> np.ndarray:
    """U upper triangular with H^-1 = U^T U.

    The route the pages describe: Cholesky of H, its inverse (the listing's
    cholesky_inverse), then the Cholesky factor of H^-1 ("Model Quantization
    Mechanics", section 2.1: "a Cholesky decomposition of the inverse
    Hessian").  Each step is one LAPACK routine in fp64: the Cholesky
    factorisation, the inverse of the triangular factor, the product
    L^-T L^-1, the Cholesky factorisation of that.  Raises
    numpy.linalg.LinAlgError if H is not positive definite."""
    from scipy.linalg import lapack
    H = np.asarray(H, dtype=np.float64)
    L, info = lapack.dpotrf(H, lower=1, clean=1)         # H = L L^T
    if info != 0:
        raise np.linalg.LinAlgError(f"H is not positive definite (pivot {info})")
    Linv, info = lapack.dtrtri(L, lower=1)               # L^-1 (lower triangular)
    if info != 0:
        raise np.linalg.LinAlgError("singular Cholesky factor")
    del L
    Hinv, info = lapack.dlauum(Linv, lower=1)            # lower part of L^-T L^-1 = H^-1
    del Linv
    Hinv = np.tril(Hinv)
    Hinv += np.tril(Hinv, -1).T
    Lh, info = lapack.dpotrf(Hinv, lower=1, clean=1)     # H^-1 = Lh Lh^T
    if info != 0:
        raise np.linalg.LinAlgError("inverse not positive definite")
    return np.ascontiguousarray(Lh.T)                    # U = Lh^T


# --------------------------------------------------------------------------
# Quantisation grid (float32 decisions, see module docstring)
# --------------------------------------------------------------------------

def _to_fp16_scale(s32):
    s32 = np.minimum(np.asarray(s32, dtype=F32), F16_MAX)
    s16 = s32.astype(np.float16)
    degenerate = s16 == np.float16(0)
    s16 = np.where(degenerate, np.float16(1.0), s16)
    return s16, degenerate


def sym_params(vals, bits=4):
    """Symmetric scale per row of ``vals`` (rows x group): s = absmax / qmax,
    qmax = 2^(bits-1) - 1 (7 -> 15 levels, "GPT-2 Quantization
    Reconstruction Error").  Returns (scale fp16, zero fp16 = 0)."""
    v = np.asarray(vals, dtype=F32)
    qmax = F32(2 ** (bits - 1) - 1)
    amax = np.max(np.abs(v), axis=-1)
    s16, _ = _to_fp16_scale(amax / qmax)
    return s16, np.zeros_like(s16)


def affine_params(vals, bits=4):
    """Affine scale and zero per row ("Model Quantization Mechanics",
    section 1): the range [min', max'] always contains 0, s = range / maxq,
    z = rint(-min' / s) clamped to the code range (reading 7)."""
    v = np.asarray(vals, dtype=F32)
    maxq = F32(2 ** bits - 1)
    mn = np.minimum(np.min(v, axis=-1), F32(0))
    mx = np.maximum(np.max(v, axis=-1), F32(0))
    s16, degenerate = _to_fp16_scale((mx - mn) / maxq)
    z = np.rint(-mn / s16.astype(F32)).astype(F32)
    z = np.clip(z, F32(0), maxq)
    z = np.where(degenerate, F32(0), z) + F32(0.0)      # -0 -> +0
    return s16, z.astype(np.float16)


def quantize_codes(w, s16, z16, sym, bits=4):
    """Integer codes c = clamp(rint(w / s) + z) in float32 (RNE)."""
    w32 = np.asarray(w, dtype=F32)
    s = np.asarray(s16).astype(F32)
    z = np.asarray(z16).astype(F32)
    if sym:
        lo, hi = F32(-(2 ** (bits - 1) - 1)), F32(2 ** (bits - 1) - 1)
    else:
        lo, hi = F32(0), F32(2 ** bits - 1)
    c = np.rint(w32 / s) + z
    c = np.clip(c, lo, hi)
    return c.astype(np.int64)


def dequantize_codes(c, s16, z16):
    """W_deq = S (W_q - Z) ("Model Quantization Mechanics", section 1)."""
    return np.asarray(s16).astype(np.float64) * (
        np.asarray(c, dtype=np.float64) - np.asarray(z16).astype(np.float64))


def code_offset(sym, bits=4):
    """Stored value of code 0: symmetric codes -q..q are stored with an
    offset of 2^(bits-1) (8 at 4 bits, so every stored value is >= 1);
    affine codes 0..2^bits - 1 as they are."""
    return 2 ** (bits - 1) if sym else 0


def pack_nibbles(codes, sym, bits=4):
    """Pack [rows, d_in] codes into uint32 words: each row is one little-
    endian bit stream along d_in in which column k occupies bits
    bits*k .. bits*k + bits - 1, cut into 32-bit words (word j holds stream
    bits 32j .. 32j + 31).  At 4 bits, nibble k of word j is column 8j + k;
    at 8 bits, byte k of word j is column 4j + k.  Needs bits * d_in to be a
    multiple of 32."""
    c = np.asarray(codes, dtype=np.int64)
    nib = c + code_offset(sym, bits)
    assert nib.min(initial=0) >= 0 and nib.max(initial=0) <= 2 ** bits - 1
    rows, d_in = nib.shape
    assert (bits * d_in) % 32 == 0
    stream = ((nib[:, :, None] >> np.arange(bits)) & 1).reshape(rows, d_in * bits)
    stream = stream.reshape(rows, -1, 32).astype(np.uint64)
    words = np.zeros(stream.shape[:2], dtype=np.uint64)
    for i in range(32):
        words |= stream[:, :, i] << np.uint64(i)
    return words.astype(np.uint32)


def unpack_nibbles(words, d_in, sym, bits=4):
    """Inverse of ``pack_nibbles``."""
    w = np.asarray(words, dtype=np.uint32).astype(np.uint64)
    rows = w.shape[0]
    stream = ((w[:, :, None] >> np.arange(32, dtype=np.uint64)) & np.uint64(1)).reshape(rows, -1)
    stream = stream[:, :d_in * bits].reshape(rows, d_in, bits).astype(np.int64)
    out = np.zeros((rows, d_in), dtype=np.int64)
    for i in range(bits):
        out |= stream[:, :, i] << i
    return out - code_offset(sym, bits)


def bits_per_weight(d_out, d_in, group_size, sym, act_order=False, bits=4):
    """Storage cost of the packed output in bits per weight: ``bits`` per
    code plus one 16-bit scale (and one 16-bit zero unless symmetric) per
    group ("GPTQ: Post-Training INT4", "Group Quantization"), plus a 32-bit
    group index per input column when the columns are act-ordered."""
    n_groups = 1 if group_size <= 0 else d_in // group_size
    code_bits = bits
    bits = code_bits * d_out * d_in + 16 * d_out * n_groups
    if not sym:
        bits += 16 * d_out * n_groups
    if act_order:
        bits += 32 * d_in
    return bits / (d_out * d_in)


# --------------------------------------------------------------------------
# RTN baseline
# --------------------------------------------------------------------------

def rtn_quantize(W, group_size=-1, sym=True, bits=4):
    """Round-to-nearest on the raw weights, per channel (group_size = -1),
    per tensor (group_size = 0: one scale for the whole matrix, "GPT-2
    Quantization Reconstruction Error", "Possible extensions"; stored once
    per row) or per group of consecutive weights in a row.

    Returns dict(codes [d_out, d_in] int, scales fp16 [d_out, n_groups],
    zeros fp16 [d_out, n_groups], qpacked uint32 [d_out, d_in / 8])."""
    W32 = np.asarray(W, dtype=F32)
    d_out, d_in = W32.shape
    if group_size == 0:
        s, z = (sym_params if sym else affine_params)(W32.reshape(1, -1), bits)
        scales = np.full((d_out, 1), s[0], dtype=np.float16)
        zeros = np.full((d_out, 1), z[0], dtype=np.float16)
        codes = quantize_codes(W32, scales, zeros, sym, bits)
        return dict(codes=codes, scales=scales, zeros=zeros,
                    qpacked=pack_nibbles(codes, sym, bits) if (bits * d_in) % 32 == 0 else None)
    g = d_in if group_size == -1 else group_size
    n_groups = d_in // g
    codes = np.zeros((d_out, d_in), dtype=np.int64)
    scales = np.zeros((d_out, n_groups), dtype=np.float16)
    zeros = np.zeros((d_out, n_groups), dtype=np.float16)
    for gi in range(n_groups):
        blk = W32[:, gi * g:(gi + 1) * g]
        s, z = sym_params(blk, bits) if sym else affine_params(blk, bits)
        scales[:, gi] = s
        zeros[:, gi] = z
        codes[:, gi * g:(gi + 1) * g] = quantize_codes(blk, s[:, None], z[:, None], sym, bits)
    return dict(codes=codes, scales=scales, zeros=zeros,
                qpacked=pack_nibbles(codes, sym, bits) if (bits * d_in) % 32 == 0 else None)


# --------------------------------------------------------------------------
# GPTQ
# --------------------------------------------------------------------------

@dataclass
class GptqResult:
    codes: np.ndarray      # [d_out, d_in] int, original column order
    scales: np.ndarray     # [d_out, n_groups] fp16, group order of the (permuted) columns
    zeros: np.ndarray      # [d_out, n_groups] fp16
    g_idx: np.ndarray      # [d_in] int32, group of each original column
    qpacked: np.ndarray    # [d_out, bits * d_in / 32] uint32 (None unless that divides)
    W_hat: np.ndarray      # [d_out, d_in] fp64 dequantised, original column order
    n_followed: int = 0    # tie decisions adopted from ``follow``
    max_follow_dist: float = 0.0   # largest boundary distance among them
    expected_ties: float = 0.0     # expected number of decisions inside their tie windows


def _tie_dist(x):
    """Distance of x from the nearest rounding boundary k + 1/2."""
    f = np.asarray(x, dtype=np.float64)
    return np.abs(f - np.floor(f) - 0.5)


def _fp16_tie_rel(s32):
    """Relative distance of an fp32 scale from the nearest fp16 rounding
    boundary (the midpoint between the two fp16 values around it)."""
    s = np.asarray(s32, dtype=np.float64)
    lo = s.astype(np.float16).astype(np.float64)
    up = np.nextafter(lo.astype(np.float16), np.float16(np.inf)).astype(np.float64)
    dn = np.nextafter(lo.astype(np.float16), np.float16(-np.inf)).astype(np.float64)
    mid = np.where(s >= lo, (lo + up) / 2, (lo + dn) / 2)
    return np.abs(s - mid) / np.where(s > 0, s, 1.0)


# Width of the rounding-tie window of the replay mode.  The other
# implementation computes each weight at its decision point in fp32: the
# in-block updates are fp32 FMAs, the lazy updates fp32-accuracy products on
# tensor cores (three TF32 products per term, relative error <= ~2^-20 per
# term) accumulated in fp32.  So the weight it decides on differs from the
# fp64 one by about TIE_REL * E, with E = sum over the updates applied to
# that weight of |delta_i U_ij| (tracked alongside, in fp64) and TIE_REL =
# 2^-20, the bound of the split's product error; the measured divergences of
# the column loop at d_in up to 28672 all lie inside this window, at about a
# tenth of the count it predicts (the fp32 accumulation errors mostly
# cancel).  A decision is a tie when w/s lies within max(TIE_TOL,
# QUOT_REL |w/s|, TIE_REL * E/s) steps of k + 1/2: the fp32 weight (one
# rounding, 2^-24 relative) and the correctly rounded quotient (2^-24) put
# w/s within 2^-23 |w/s| steps of the fp64 quotient, covered twice over by
# QUOT_REL = 2^-22 (1.5e-5 steps at |w/s| = 127, the 8-bit range; 2e-6 at
# 4 bits); TIE_TOL = 1e-6 steps is the floor near zero.  A scale is a tie when its fp32 value lies
# within the same relative distance (the window on the group's extreme,
# divided by the extreme) of an fp16 rounding boundary; an affine zero-point
# when -min'/s lies within the window of k + 1/2.
TIE_TOL = 1e-6
TIE_REL = 2.0 ** -20
QUOT_REL = 2.0 ** -22


def gptq_quantize(W, U, bits=4, group_size=-1, block_size=128, sym=True,
                  perm=None, dead=None, follow=None, tie_tol=TIE_TOL,
                  tie_rel=TIE_REL) -> GptqResult:
    """GPTQ on one layer given U (upper, H^-1 = U^T U, in the column order
    the layer is processed in).

    Follows "GPTQ: Post-Training INT4", "The GPTQ Algorithm": columns left
    to right in blocks of ``block_size``; for each column the code from the
    current weights, the scaled error delta = (w - q) / U_jj, the in-block
    update w[j+1:end] -= delta * U[j, j+1:end]; after the block the lazy
    trailing update W[:, end:] -= Err @ U[blk, end:].  Group parameters per
    reading 6.  ``perm`` (act-order) gives the processing order of the
    original columns; ``dead`` columns are zeroed first.

    ``follow`` (optional, dict with "codes" [d_out, d_in] in original column
    order and "scales"/"zeros" [d_out, n_groups]) is the output of another
    implementation.  Where the oracle's own decision is a rounding tie at
    the precision of that implementation -- w/s within max(tie_tol, tie_rel
    E/s) steps of k + 1/2, E the accumulated magnitude of the updates applied
    to w, or the fp32 scale within the same relative distance of an fp16
    rounding boundary (see TIE_REL) -- both roundings are correct, and the
    oracle takes the other implementation's choice so that the rest of the
    row can be checked along it.  Nowhere else does ``follow`` change
    anything; ``n_followed`` counts the adopted decisions and
    ``max_follow_dist`` is the largest distance from a boundary among them
    (steps, or relative for a scale)."""
    W = np.array(W, dtype=np.float64, copy=True)
    d_out, d_in = W.shape
    if dead is not None:
        W[:, np.asarray(dead, dtype=bool)] = 0.0
    if perm is not None:
        perm = np.asarray(perm, dtype=np.int64)
        W = W[:, perm]
    per_tensor = group_size == 0   # one scale from the whole initial matrix
    if per_tensor:
        group_size = -1
    g = d_in if group_size == -1 else group_size
    if group_size != -1:
        assert d_in % g == 0 and block_size % g == 0
    n_groups = d_in // g
    lo = -(2 ** (bits - 1) - 1) if sym else 0
    params = sym_params if sym else affine_params

    codes = np.zeros((d_out, d_in), dtype=np.int64)
    Q = np.zeros((d_out, d_in), dtype=np.float64)
    scales = np.zeros((d_out, n_groups), dtype=np.float16)
    zeros = np.zeros((d_out, n_groups), dtype=np.float16)
    n_followed = 0
    max_dist = 0.0
    expected = 0.0   # sum over decisions of the chance that a decision lands in its window
    if follow is not None:
        f_codes = np.asarray(follow["codes"], dtype=np.int64)
        if perm is not None:
            f_codes = f_codes[:, perm]
        f_scales = np.asarray(follow["scales"], dtype=np.float16)
        f_zeros = (np.asarray(follow["zeros"], dtype=np.float16)
                   if not sym else np.zeros_like(f_scales))

    def group(vals, gi, evals=None):
        nonlocal n_followed, max_dist, expected
        s, z = params(vals, bits)
        if follow is not None:
            v = np.asarray(vals, dtype=F32)
            ev = (np.zeros(len(s)) if evals is None
                  else tie_rel * np.max(np.asarray(evals), axis=-1))   # error of the extremes
            if sym:
                ext = np.max(np.abs(v), axis=-1).astype(np.float64)
                s32 = np.max(np.abs(v), axis=-1) / F32(2 ** (bits - 1) - 1)
                win = np.maximum(tie_tol, ev / np.where(ext > 0, ext, 1.0))
                dist = _fp16_tie_rel(s32)
            else:
                mn = np.minimum(np.min(v, axis=-1), F32(0))
                mx = np.maximum(np.max(v, axis=-1), F32(0))
                ext = (mx - mn).astype(np.float64)
                s32 = (mx - mn) / F32(2 ** bits - 1)
                zr = -mn.astype(np.float64) / s.astype(np.float64)
                zd = _tie_dist(zr)
                win_s = np.maximum(tie_tol, ev / np.where(ext > 0, ext, 1.0))
                win_z = np.maximum(np.maximum(tie_tol, QUOT_REL * np.abs(zr)),
                                   ev / s.astype(np.float64))
                sd = _fp16_tie_rel(s32)
                # compare each distance with its own window: report the one
                # that is a tie (the smaller ratio)
                dist = np.where(sd / win_s <= zd / win_z, sd, zd)
                win = np.where(sd / win_s <= zd / win_z, win_s, win_z)
            # fp16 rounding boundaries are an ulp (2^-11 .. 2^-10 relative) apart
            expected += float(np.sum(np.minimum(1.0, 2.0 * win / 2.0 ** -11)))
            take = (dist < win) & ((f_scales[:, gi] != s) | (f_zeros[:, gi] != z))
            s = np.where(take, f_scales[:, gi], s)
            z = np.where(take, f_zeros[:, gi], z)
            n_followed += int(take.sum())
            if take.any():
                max_dist = max(max_dist, float(dist[take].max()))
        return s, z

    # E: accumulated |update| per weight (only to size the tie windows)
    E = np.zeros_like(W) if follow is not None else None
    if per_tensor:
        s, z = params(W.astype(F32).reshape(1, -1), bits)
        scales[:, 0], zeros[:, 0] = s[0], z[0]
    elif group_size == -1:
        s, z = group(W.astype(F32), 0)
        scales[:, 0], zeros[:, 0] = s, z
    for b0 in range(0, d_in, block_size):
        b1 = min(b0 + block_size, d_in)
        Wb = W[:, b0:b1].copy()
        Eb = E[:, b0:b1].copy() if E is not None else None
        Err = np.zeros_like(Wb)
        for j in range(b1 - b0):
            col = b0 + j
            if group_size != -1 and col % g == 0:
                s, z = group(Wb[:, j:j + g].astype(F32), col // g,
                             None if Eb is None else Eb[:, j:j + g])
                scales[:, col // g], zeros[:, col // g] = s, z
            gi = 0 if group_size == -1 else col // g
            s, z = scales[:, gi], zeros[:, gi]
            w = Wb[:, j]
            c = quantize_codes(w, s, z, sym, bits)
            if follow is not None:
                s64 = s.astype(np.float64)
                r = w.astype(F32).astype(np.float64) / s64
                dist = _tie_dist(r)
                win = np.maximum(np.maximum(tie_tol, QUOT_REL * np.abs(r)),
                                 tie_rel * Eb[:, j] / s64)
                expected += float(np.sum(np.minimum(1.0, 2.0 * win)))
                take = ((dist < win) & (f_codes[:, col] != c)
                        & (np.abs(f_codes[:, col] - c) == 1))
                c = np.where(take, f_codes[:, col], c)
                n_followed += int(take.sum())
                if take.any():
                    max_dist = max(max_dist, float(dist[take].max()))
            q = dequantize_codes(c, s, z)
            codes[:, col] = c
            Q[:, col] = q
            delta = (w - q) / U[col, col]
            Err[:, j] = delta
            Wb[:, j + 1:] -= np.outer(delta, U[col, col + 1:b1])
            if Eb is not None:
                Eb[:, j + 1:] += np.outer(np.abs(delta), np.abs(U[col, col + 1:b1]))
        W[:, b0:b1] = Wb
        W[:, b1:] -= Err @ U[b0:b1, b1:]
        if E is not None:
            E[:, b1:] += np.abs(Err) @ np.abs(U[b0:b1, b1:])

    g_perm = np.arange(d_in) // g
    if perm is not None:
        inv = np.empty_like(perm)
        inv[perm] = np.arange(d_in)
        codes = codes[:, inv]
        Q = Q[:, inv]
        g_idx = g_perm[inv]
    else:
        g_idx = g_perm
    assert codes.min() >= lo
    return GptqResult(codes=codes, scales=scales, zeros=zeros,
                      g_idx=g_idx.astype(np.int32), n_followed=n_followed,
                      max_follow_dist=max_dist, expected_ties=expected,
                      qpacked=pack_nibbles(codes, sym, bits) if (bits * d_in) % 32 == 0 else None,
                      W_hat=Q)


def gptq_layer(W, X, bits=4, group_size=-1, block_size=128, sym=True,
               damp_percent=0.01, act_order=False, follow=None, tie_tol=TIE_TOL,
               tie_rel=TIE_REL):
    """The whole per-layer path: H = 2 X^T X, dead columns and damping,
    optional act-order, U, then GPTQ.  Returns (GptqResult, H_undamped,
    U, perm, dead)."""
    H0 = hessian(X)
    Hd, dead = damp_hessian(H0, damp_percent)
    perm = act_order_perm(Hd) if act_order else None
    Hp = Hd[np.ix_(perm, perm)] if perm is not None else Hd
    U = upper_factor_of_inverse(Hp)
    res = gptq_quantize(W, U, bits=bits, group_size=group_size,
                        block_size=block_size, sym=sym, perm=perm, dead=dead,
                        follow=follow, tie_tol=tie_tol, tie_rel=tie_rel)
    return res, H0, U, perm, dead


def dequantize_packed(qpacked, scales, zeros, d_in, group_size, sym,
                      g_idx=None, bits=4):
    """W^ from packed codes and the stored 16-bit scales / zeros."""
    c = unpack_nibbles(qpacked, d_in, sym, bits)
    if g_idx is None:
        g = d_in if group_size <= 0 else group_size
        g_idx = np.arange(d_in) // g
    g_idx = np.asarray(g_idx, dtype=np.int64)
    s = np.asarray(scales)[:, g_idx]
    z = np.asarray(zeros)[:, g_idx] if not sym else np.zeros_like(s)
    return dequantize_codes(c, s, z)


# --------------------------------------------------------------------------
# Reconstruction error
# --------------------------------------------------------------------------

def recon_sse(W, W_hat, X) -> float:
    """||W X^T - W^ X^T||_F^2 in fp64 -- the layer-wise objective of "GPTQ:
    Post-Training INT4", "OBQ Foundation", with X tokens x d_in.  The MSE is
    this divided by n_tok * d_out."""
    dW = np.asarray(W, dtype=np.float64) - np.asarray(W_hat, dtype=np.float64)
    Y = dW @ np.asarray(X, dtype=np.float64).T
    return float(np.sum(Y * Y))


def recon_sse_trace(W, W_hat, H_undamped) -> float:
    """Second route to the same number: trace(dW H dW^T) / 2 with the
    undamped H = 2 X^T X (pin only)."""
    dW = np.asarray(W, dtype=np.float64) - np.asarray(W_hat, dtype=np.float64)
    return float(np.sum((dW @ H_undamped) * dW) / 2.0)


# --------------------------------------------------------------------------
# Consumer of the packed format
# --------------------------------------------------------------------------

def w4a16_matmul(qpacked, scales, zeros, d_in, group_size, sym, X, g_idx=None, bits=4):
    """Y = W^ X^T in fp64 with W^ = s (c - z) from the packed codes ("GPTQ:
    Post-Training INT4", "Group Quantization": 4-bit codes with 16-bit
    scales are what the quantised model is run from)."""
    What = dequantize_packed(qpacked, scales, zeros, d_in, group_size, sym, g_idx, bits)
    return What @ np.asarray(X, dtype=np.float64).T


def round_to_bf16(x):
    """Round fp64 values to the nearest bf16 value (8 significant bits, ties
    to even), in one rounding step (no intermediate float32)."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                     # x = m 2^e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(m * 256.0) / 256.0, e)


def gelu_tanh(x):
    """GELU in its tanh form, 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715
    x^3))), in fp64 (GPT-2's MLP activation)."""
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * x * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (x + 0.044715 * x ** 3)))


def apply_layer(X, W_hat, act="none", residual=None, follow=None, tie_rel=TIE_REL):
    """The layer applied to its input, as the next layer sees it: Z = act(X
    W^T) (+ residual), fp64, rounded once to bf16.  X [n_tok, d_in], W_hat
    [d_out, d_in].

    ``follow`` (optional, [n_tok, d_out], another implementation's bf16
    values): that implementation computes the value before rounding with an
    error of at most w = tie_rel * (|X| |W|^T + |residual| + |Z|), the
    error bound of an fp32 sum of those terms, so any bf16 value that is
    the rounding of some t in [Z - w, Z + w] is a correct result.  Rounding
    is monotone, so those are exactly the bf16 values between
    round(Z - w) and round(Z + w); the other implementation's value is
    taken where it is one of them (the other neighbour at a rounding tie;
    where Z cancels to far below |X| |W|^T, w can span several bf16 steps).
    Returns Z, or (Z, adopted) with ``follow``."""
    Xa = np.asarray(X, dtype=np.float64)
    Wa = np.asarray(W_hat, dtype=np.float64)
    Y = Xa @ Wa.T
    if act == "relu":
        Y = np.maximum(Y, 0.0)
    elif act == "gelu":
        Y = gelu_tanh(Y)
    if residual is not None:
        Y = Y + np.asarray(residual, dtype=np.float64)
    Z = round_to_bf16(Y)
    if follow is None:
        return Z
    f = np.asarray(follow, dtype=np.float64)
    mag = np.abs(Xa) @ np.abs(Wa).T + np.abs(Y)
    if residual is not None:
        mag = mag + np.abs(np.asarray(residual, dtype=np.float64))
    w = tie_rel * mag
    lo, hi = round_to_bf16(Y - w), round_to_bf16(Y + w)
    take = (f != Z) & (f >= lo) & (f <= hi)
    return np.where(take, f, Z), int(take.sum())


def gptq_sequential(X0, layers, bits=4, group_size=-1, block_size=128, sym=True,
                    damp_percent=0.01, quantized_inputs=True, follow=None, follow_x=None,
                    tie_rel=TIE_REL, x_tie_rel=TIE_REL):
    """Layers quantised one after another, each calibrated on the input it
    actually receives ("GPT-2 Quantization Reconstruction Error", "Key
    findings": the per-layer errors were measured with the whole model
    running, so each layer's input carries the error of the quantised layers
    before it).  ``layers``: list of dicts with W [d_out, d_in], act ("none",
    "relu", "gelu") and residual_from (None, or the index j <= l of an
    earlier input X_j added to layer l's output, e.g. a block's input at the
    end of an MLP block).  For each layer: H from its input X_l, GPTQ, the
    layer error ||(W - W^) X_l^T||^2, then X_{l+1} = apply_layer(X_l, W^ (or
    W when not ``quantized_inputs``), act, X_j).  ``follow``: per-layer
    list of dicts (as for gptq_quantize) or None; ``follow_x``: another
    implementation's X_1 .. X_n (its bf16 roundings are taken at ties, as in
    apply_layer); ``tie_rel``: the GPTQ tie window scale (see TIE_REL), one
    for all layers or a list with one per layer; ``x_tie_rel``: the window
    scale of the activations' replay (apply_layer's tie_rel).  Returns
    (results, sse, xs) with xs the inputs X_0 .. X_n."""
    X = np.asarray(X0, dtype=np.float64)
    results, sse, xs = [], [], [X]
    for li, L in enumerate(layers):
        W = np.asarray(L["W"], dtype=np.float64)
        tr = tie_rel[li] if isinstance(tie_rel, (list, tuple)) else tie_rel
        res, H0, U, perm, dead = gptq_layer(W, X, bits=bits, group_size=group_size,
                                            block_size=block_size, sym=sym,
                                            damp_percent=damp_percent,
                                            follow=None if follow is None else follow[li],
                                            tie_rel=tr)
        results.append(res)
        sse.append(recon_sse(W, res.W_hat, X))
        j = L.get("residual_from")
        X = apply_layer(X, res.W_hat if quantized_inputs else W, L.get("act", "none"),
                        None if j is None else xs[j],
                        follow=None if follow_x is None else follow_x[li], tie_rel=x_tie_rel)
        if follow_x is not None:
            X = X[0]
        xs.append(X)
    return results, sse, xs


# --------------------------------------------------------------------------
# Activation-aware scaling before RTN (reading 10)
# --------------------------------------------------------------------------

def awq_channel_scales(H_diag, alpha) -> np.ndarray:
    """s_c = (a_c / a_bar)^alpha in fp64 with a_c = sqrt(H_cc / 2N): the 2N
    cancels, so s_c = (H_cc / H_bar)^(alpha / 2), H_bar the geometric mean of
    the positive H_cc; s_c = 1 where H_cc <= 0 ("Model Quantization
    Mechanics", section 2.2: per-channel scale from activation magnitude)."""
    h = np.asarray(H_diag, dtype=np.float64)
    pos = h > 0
    s = np.ones_like(h)
    if pos.any():
        logbar = np.mean(np.log(h[pos]))
        s[pos] = np.exp(0.5 * alpha * (np.log(h[pos]) - logbar))
    return s


def awq_apply(W, s32, group_size=-1, sym=True):
    """RTN of W diag(s) (the product taken in fp32, as stored), and the
    effective weights dequant(...) diag(s)^-1 in fp64."""
    s32 = np.asarray(s32, dtype=F32)
    Wp = (np.asarray(W, dtype=F32) * s32[None, :]).astype(F32)
    r = rtn_quantize(Wp, group_size, sym)
    g = Wp.shape[1] if group_size == -1 else group_size
    gi = np.arange(Wp.shape[1]) // g
    What = dequantize_codes(r["codes"], r["scales"][:, gi].astype(np.float64),
                            r["zeros"][:, gi].astype(np.float64))
    return r, What / s32.astype(np.float64)[None, :]


def awq_rtn_search(W, X, group_size=-1, sym=True, n_grid=20):
    """Grid search of alpha (reading 10): for each alpha = k / n_grid the layer
    MSE ||(W - W^) X^T||^2 / (N d_out) of RTN after scaling; returns
    dict(best, alpha, mse [n_grid], s (fp32, of the best alpha), rtn (the
    RTN result of the best alpha: codes, scales, zeros, qpacked), W_hat)."""
    X = np.asarray(X, dtype=np.float64)
    hd = 2.0 * np.sum(X * X, axis=0)
    n, d_out = X.shape[0], np.asarray(W).shape[0]
    mse, keep = [], []
    for k in range(n_grid):
        s32 = awq_channel_scales(hd, k / n_grid).astype(F32)
        r, What = awq_apply(W, s32, group_size, sym)
        mse.append(recon_sse(W, What, X) / (n * d_out))
        keep.append((s32, r, What))
    best = int(np.argmin(mse))
    s32, r, What = keep[best]
    return dict(best=best, alpha=best / n_grid, mse=np.array(mse), s=s32, rtn=r, W_hat=What)


# --------------------------------------------------------------------------
# References used by the pins
# --------------------------------------------------------------------------

def obs_quantize(w, H, quantize):
    """Per-step OBS on one row with the Hessian re-inverted on the remaining
    set F at every step ("GPTQ: Post-Training INT4", "Hessian-Based Weight
    Update", read with H_F^-1 as in reading 5), columns taken left to right.
    ``quantize(col, row) -> dequantised value of row[col]``, where ``row`` is
    the whole current row (entries at col and beyond carry every OBS update
    so far), so that a quantiser can take a group's parameters from the
    group's current weights.  Returns the dequantised row."""
    w = np.array(w, dtype=np.float64, copy=True)
    d = w.shape[0]
    out = np.zeros(d)
    for q in range(d):
        F = np.arange(q, d)
        HinvF = np.linalg.inv(H[np.ix_(F, F)])
        qhat = quantize(q, w.copy())
        out[q] = qhat
        err = w[q] - qhat
        w[F] -= err * HinvF[:, 0] / HinvF[0, 0]
    return out


def bruteforce_row(w, H_undamped, levels_per_col):
    """Exhaustive minimum of (w - q) H (w - q)^T / 2 over every code vector,
    ``levels_per_col[k]`` listing the dequantised values allowed at column
    k.  Returns (best q, best error)."""
    w = np.asarray(w, dtype=np.float64)
    best, best_q = np.inf, None
    for q in itertools.product(*levels_per_col):
        r = w - np.asarray(q)
        e = float(r @ H_undamped @ r) / 2.0
        if e < best:
            best, best_q = e, np.asarray(q)
    return best_q, best


def round_to_grid(w, step):
    """Round each weight alone to the nearest multiple of ``step`` ("GPTQ and
    AWQ", "Part 1. Rounding each weight alone")."""
    return [np.rint(v / step) * step for v in w]


def round_error_carried_forward(w, step):
    """Round left to right so that every partial sum of the rounded weights
    stays as close as the grid allows to the same partial sum of the
    originals ("GPTQ and AWQ", "Example 1.1": the error left by one weight is
    taken off the next before it is rounded).  In closed form, with S_k the
    sum of w_0..w_k and Q_k that of q_0..q_k: q_k = step * rint((S_k -
    Q_{k-1}) / step)."""
    S = np.cumsum(np.asarray(w, dtype=np.float64))
    out = []
    for k in range(len(S)):
        prev = sum(out)
        out.append(np.rint((S[k] - prev) / step) * step)
    return out


def gptq_fixed_grid(w_row, X, step, damp_percent=0.01, block_size=128):
    """GPTQ on a single row with a fixed unbounded grid of spacing ``step``
    (the lesson's setting), same loop as ``gptq_quantize``.  Returns the
    dequantised row."""
    w = np.array(w_row, dtype=np.float64, copy=True)[None, :]
    H, _ = damp_hessian(hessian(X), damp_percent)
    U = upper_factor_of_inverse(H)
    d = w.shape[1]
    Q = np.zeros_like(w)
    for b0 in range(0, d, block_size):
        b1 = min(b0 + block_size, d)
        Wb = w[:, b0:b1].copy()
        Err = np.zeros_like(Wb)
        for j in range(b1 - b0):
            col = b0 + j
            q = np.rint(Wb[:, j] / step) * step
            Q[:, col] = q
            delta = (Wb[:, j] - q) / U[col, col]
            Err[:, j] = delta
            Wb[:, j + 1:] -= np.outer(delta, U[col, col + 1:b1])
        w[:, b0:b1] = Wb
        w[:, b1:] -= Err @ U[b0:b1, b1:]
    return Q[0]
