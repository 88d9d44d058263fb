"""Pins of the CPU oracle to what the pages and the mathematics fix.

Each test ties one oracle function to something other than itself: values
printed on the pages (fixtures under tests/golden/), brute force on tiny
inputs, closed forms, or an independent derivation (per-step OBS with a
re-inverted Hessian, the reversed Cholesky route to U, the trace form of the
reconstruction error).  Chosen so that a dropped term, a wrong sign or index,
or a transposed operand in the oracle fails at least one of them.
"""
import itertools

import numpy as np
import pytest

import oracle as O

F32 = np.float32


# -------------------------------------------------------------- the lesson

def test_lesson_nearest_and_carried_forward(golden):
    g = golden("lesson_example_1_1.txt")
    w, x, step = g["weights"], g["inputs"], g["step"]
    true = sum(a * b for a, b in zip(w, x))
    near = O.round_to_grid(w, step)
    comp = O.round_error_carried_forward(w, step)
    assert [round(v, 1) for v in near] == g["nearest"]
    assert [round(v, 1) for v in comp] == g["compensated"]
    assert round(abs(sum(a * b for a, b in zip(near, x)) - true), 2) == g["nearest_abs_error"]
    assert round(abs(sum(a * b for a, b in zip(comp, x)) - true), 2) == g["compensated_abs_error"]


def test_lesson_gptq_reaches_bruteforce_optimum(golden):
    """GPTQ on the lesson's row (one token, inputs 1.0, grid step 0.1) makes
    the output error 0.04, the same as the best of all code vectors and far
    below round-to-nearest's 0.14."""
    g = golden("lesson_example_1_1.txt")
    w = np.array(g["weights"])
    X = np.array(g["inputs"])[None, :]
    q = O.gptq_fixed_grid(w, X, g["step"], damp_percent=0.01)
    err_gptq = abs(float((q - w) @ X[0]))
    cands = [[np.floor(v / 0.1) * 0.1, np.ceil(v / 0.1) * 0.1] for v in w]
    best = min(abs(float((np.array(c) - w) @ X[0])) for c in itertools.product(*cands))
    assert round(err_gptq, 2) == g["compensated_abs_error"]
    assert round(best, 2) == g["compensated_abs_error"]
    assert err_gptq < g["nearest_abs_error"]


def test_pair_case(golden):
    g = golden("pair_case.txt")
    w, x = np.array(g["weights"]), np.array(g["inputs"])
    outs = {c: float(np.array(c) @ x) for c in itertools.product(g["grid"], repeat=2)}
    best = min(outs.items(), key=lambda kv: abs(kv[1] - w @ x))
    assert round(best[1], 2) == g["best_output"]
    assert round(abs(best[1] - w @ x), 2) == g["best_abs_error"]
    near = O.round_to_grid(w, 0.1)
    assert round(float(np.dot(near, x)), 2) == g["nearest_output"]
    assert round(abs(float(np.dot(near, x)) - w @ x), 2) == g["nearest_abs_error"]
    assert round(abs(0.4 - w @ x), 2) == g["both_down_abs_error"]
    # GPTQ with two equal unit inputs reduces to carrying the error forward
    q = O.gptq_fixed_grid(w, x[None, :], 0.1, damp_percent=0.01)
    assert [round(v, 1) for v in q] == g["carried_forward"]
    assert [round(v, 1) for v in O.round_error_carried_forward(w, 0.1)] == g["carried_forward"]


# -------------------------------------------------------------- Hessian

def test_hessian_bruteforce_definition():
    rng = np.random.default_rng(1)
    X = rng.standard_normal((7, 5))
    H = O.hessian(X)
    for i in range(5):
        for j in range(5):
            ref = 0.0
            for t in range(7):
                ref += 2.0 * X[t, i] * X[t, j]
            assert abs(H[i, j] - ref) < 1e-12
    sub = O.hessian_entries(X, [1, 3], [0, 4])
    assert np.allclose(sub, H[np.ix_([1, 3], [0, 4])], rtol=0, atol=1e-13)


def test_damp_and_dead_columns_closed_form():
    H = np.diag([4.0, 0.0, 2.0])
    H[0, 2] = H[2, 0] = 1.0
    Hd, dead = O.damp_hessian(H, 0.01)
    assert dead.tolist() == [False, True, False]
    lam = 0.01 * (4.0 + 1.0 + 2.0) / 3.0
    assert np.allclose(np.diag(Hd), [4.0 + lam, 1.0 + lam, 2.0 + lam], rtol=0, atol=1e-15)
    assert Hd[0, 2] == 1.0 and Hd[2, 0] == 1.0


def test_act_order_perm_stable_descending():
    H = np.diag([1.0, 5.0, 3.0, 5.0, 0.5])
    assert O.act_order_perm(H).tolist() == [1, 3, 2, 0, 4]


def test_upper_factor_against_reversed_cholesky():
    """U from the pages' route (Cholesky, inverse, Cholesky of the inverse)
    equals the independent reversal identity U = J chol(J H J)^-1 J, and
    U^T U H = I."""
    rng = np.random.default_rng(2)
    for d in (1, 3, 8, 33):
        A = rng.standard_normal((2 * d + 3, d))
        H, _ = O.damp_hessian(O.hessian(A), 0.01)
        U = O.upper_factor_of_inverse(H)
        J = np.eye(d)[::-1]
        Lr = np.linalg.cholesky(J @ H @ J)
        U2 = J @ np.linalg.inv(Lr) @ J
        assert np.allclose(U, np.triu(U), atol=0)
        assert np.max(np.abs(U - U2)) <= 1e-10 * np.max(np.abs(U))
        assert np.max(np.abs(U.T @ U @ H - np.eye(d))) < 1e-9
        assert np.all(np.diag(U) > 0)


def test_not_positive_definite_raises():
    with pytest.raises(np.linalg.LinAlgError):
        O.upper_factor_of_inverse(-np.eye(3))


# -------------------------------------------------------------- grid

def test_sym_grid_has_15_levels(golden):
    g = golden("sym_grid.txt")
    rng = np.random.default_rng(3)
    v = np.concatenate([np.linspace(-1.0, 1.0, 97), rng.uniform(-0.9, 0.9, 4000)])
    v = v[None, :].astype(F32)
    s, z = O.sym_params(v, int(g["bits"]))
    c = O.quantize_codes(v, s[:, None], z[:, None], True, int(g["bits"]))
    assert len(np.unique(c)) == int(g["levels"])
    assert c.min() == -7 and c.max() == 7
    amax_i = np.argmax(np.abs(v[0]))
    assert abs(c[0, amax_i]) == 7
    # negation symmetry of the grid
    c_neg = O.quantize_codes(-v, s[:, None], z[:, None], True)
    assert np.array_equal(c_neg, -c)
    # points on the grid map to themselves
    grid = (np.arange(-7, 8) * s.astype(np.float64)[0])[None, :]
    cg = O.quantize_codes(grid, s[:, None], z[:, None], True)
    assert np.array_equal(cg[0], np.arange(-7, 8))
    assert np.array_equal(O.dequantize_codes(cg, s[:, None], z[:, None]), grid)


def test_affine_grid_formula():
    """W_q = round(W/S) + Z in 0..15, W_deq = S (W_q - Z): zero is exact, the
    range ends map to the end codes, the rounding error is at most half a
    step (plus the fp16 rounding of S at the far end)."""
    rng = np.random.default_rng(4)
    for shift in (0.0, 0.05, -0.05, 0.5):
        v = (rng.standard_normal((16, 128)) * 0.02 + shift).astype(F32)
        s, z = O.affine_params(v)
        c = O.quantize_codes(v, s[:, None], z[:, None], False)
        assert c.min() >= 0 and c.max() <= 15
        deq = O.dequantize_codes(c, s[:, None], z[:, None])
        zero_c = O.quantize_codes(np.zeros((16, 1), F32), s[:, None], z[:, None], False)
        assert np.all(O.dequantize_codes(zero_c, s[:, None], z[:, None]) == 0.0)
        step = s.astype(np.float64)[:, None]
        assert np.all(np.abs(deq - v) <= 0.5 * step * 1.02 + 1e-12)
        mn = np.minimum(v.min(1), 0)
        mx = np.maximum(v.max(1), 0)
        c_mn = O.quantize_codes(mn[:, None], s[:, None], z[:, None], False)[:, 0]
        c_mx = O.quantize_codes(mx[:, None], s[:, None], z[:, None], False)[:, 0]
        assert np.all(c_mn <= 1) and np.all(c_mx >= 14)


def test_degenerate_group():
    v = np.zeros((2, 8), F32)
    for sym in (True, False):
        s, z = O.sym_params(v) if sym else O.affine_params(v)
        assert np.all(s == np.float16(1.0)) and np.all(z == 0)
        c = O.quantize_codes(v, s[:, None], z[:, None], sym)
        assert np.all(c == 0)


def test_pack_layout_and_roundtrip():
    codes = np.arange(16, dtype=np.int64)[None, :]
    words = O.pack_nibbles(codes, sym=False)
    assert words.tolist() == [[0x76543210, 0xFEDCBA98]]
    sym_codes = np.arange(-7, 9, dtype=np.int64)[None, :].clip(-7, 7)
    assert np.array_equal(O.unpack_nibbles(O.pack_nibbles(sym_codes, True), 16, True), sym_codes)
    rng = np.random.default_rng(5)
    c = rng.integers(0, 16, size=(5, 64))
    assert np.array_equal(O.unpack_nibbles(O.pack_nibbles(c, False), 64, False), c)


def test_storage_bits_per_weight(golden):
    g = golden("storage_bits.txt")
    gs = int(g["group_size"])
    assert O.bits_per_weight(8, 1024, gs, sym=True) == g["bits_symmetric"]
    assert O.bits_per_weight(8, 1024, gs, sym=False) == g["bits_affine"]
    W = np.random.default_rng(6).standard_normal((8, 1024)).astype(F32) * 0.02
    for sym, key in ((True, "bits_symmetric"), (False, "bits_affine")):
        r = O.rtn_quantize(W, gs, sym)
        nbytes = r["qpacked"].nbytes + r["scales"].nbytes + (0 if sym else r["zeros"].nbytes)
        assert nbytes * 8 / W.size == g[key]
    assert O.bits_per_weight(8, 768, -1, True) == 4 + 16 / 768


# -------------------------------------------------------------- GPTQ

def _row_quantizer(w_row, sym):
    """Per-channel quantiser for obs_quantize: one scale from the initial row."""
    s, z = O.sym_params(w_row[None].astype(F32)) if sym else O.affine_params(w_row[None].astype(F32))

    def q(col, row):
        c = O.quantize_codes(np.array([[row[col]]]), s[:, None], z[:, None], sym)
        return float(O.dequantize_codes(c, s[:, None], z[:, None])[0, 0])
    return q


def _group_quantizer(g, sym, params_from_initial=None):
    """Group quantiser for obs_quantize written from "Group Quantization":
    when column col starts a group (col % g == 0), the group's scale and zero
    are taken from the row's current values of the group's g columns; later
    columns of the group reuse them.  ``params_from_initial`` (a row) plants
    the mistake of taking them from the initial weights instead."""
    state = {}

    def q(col, row):
        if col % g == 0:
            src = row if params_from_initial is None else params_from_initial
            vals = np.asarray(src[col:col + g], dtype=np.float64)[None].astype(F32)
            state["p"] = O.sym_params(vals) if sym else O.affine_params(vals)
        s, z = state["p"]
        c = O.quantize_codes(np.array([[row[col]]]), s[:, None], z[:, None], sym)
        return float(O.dequantize_codes(c, s[:, None], z[:, None])[0, 0])
    return q


@pytest.mark.parametrize("sym", [True, False])
def test_cholesky_form_equals_per_step_obs(sym):
    """GPTQ's Cholesky form equals OBS with H_F re-inverted at every step,
    for tiny d_in <= 8, with any lazy block size."""
    rng = np.random.default_rng(7 if sym else 8)
    for t in range(40):
        d = int(rng.integers(2, 9))
        n = int(rng.integers(1, 3 * d))
        X = rng.standard_normal((n, d)) * rng.lognormal(0, 0.5, d)
        W = rng.standard_normal((4, d)) * 0.1
        H, _ = O.damp_hessian(O.hessian(X), 0.01)
        U = O.upper_factor_of_inverse(H)
        r = O.gptq_quantize(W, U, group_size=-1, block_size=128, sym=sym)
        for bs in (1, 2, 3):
            rb = O.gptq_quantize(W, U, group_size=-1, block_size=bs, sym=sym)
            assert np.array_equal(rb.codes, r.codes)
        for i in range(4):
            ref = O.obs_quantize(W[i], H, _row_quantizer(W[i], sym))
            assert np.array_equal(ref, r.W_hat[i]), (t, i)


@pytest.mark.parametrize("sym", [True, False])
@pytest.mark.parametrize("g", [2, 4])
def test_grouped_cholesky_form_equals_per_step_obs(g, sym):
    """With groups, GPTQ's Cholesky form equals per-step OBS whose quantiser
    takes each group's parameters from the group's current (OBS-updated)
    weights at the group's first column (reading 6), for d_in <= 8 and every
    lazy block size that the group divides."""
    rng = np.random.default_rng(100 + 10 * g + sym)
    n_diff_groups = 0
    for t in range(40):
        d = g * int(rng.integers(2, 8 // g + 1))
        n = int(rng.integers(1, 3 * d))
        X = rng.standard_normal((n, d)) * rng.lognormal(0, 0.5, d)
        W = rng.standard_normal((6, d)) * 0.1
        H, _ = O.damp_hessian(O.hessian(X), 0.01)
        U = O.upper_factor_of_inverse(H)
        r = O.gptq_quantize(W, U, group_size=g, block_size=128, sym=sym)
        for bs in (g, 2 * g):
            rb = O.gptq_quantize(W, U, group_size=g, block_size=bs, sym=sym)
            assert np.array_equal(rb.codes, r.codes) and np.array_equal(rb.scales, r.scales)
        for i in range(6):
            ref = O.obs_quantize(W[i], H, _group_quantizer(g, sym))
            assert np.array_equal(ref, r.W_hat[i]), (t, i)
            init = O.rtn_quantize(W[i:i + 1].astype(F32), g, sym)["scales"]
            n_diff_groups += int(np.sum(init != r.scales[i]))
    # the later groups' parameters do move with the updates (else this pin
    # could not tell current from initial weights)
    assert n_diff_groups >= 20


def _fixed_scale_levels(s, z, sym, d):
    codes = range(-7, 8) if sym else range(0, 16)
    lv = [float(s) * (c - float(z)) for c in codes]
    return [lv] * d


def test_bruteforce_bounds_gptq():
    """On tiny layers with the scale GPTQ picked: the exhaustive optimum is
    never worse than GPTQ; on correlated inputs (duplicated / near-collinear
    columns) GPTQ beats round-to-nearest."""
    rng = np.random.default_rng(9)
    wins = 0
    for t in range(12):
        d = 4
        base = rng.standard_normal((24, 2))
        X = np.concatenate([base, base + 0.05 * rng.standard_normal((24, 2))], 1)
        W = rng.standard_normal((1, d)) * 0.1
        H0 = O.hessian(X)
        Hd, _ = O.damp_hessian(H0, 0.01)
        U = O.upper_factor_of_inverse(Hd)
        r = O.gptq_quantize(W, U, group_size=-1, sym=True)
        rtn = O.rtn_quantize(W.astype(F32), -1, True)
        assert r.scales[0, 0] == rtn["scales"][0, 0]
        w_rtn = O.dequantize_codes(rtn["codes"], rtn["scales"], rtn["zeros"])
        e_gptq = O.recon_sse(W, r.W_hat, X)
        e_rtn = O.recon_sse(W, w_rtn, X)
        _, e_best = O.bruteforce_row(W[0], H0, _fixed_scale_levels(r.scales[0, 0], 0, True, d))
        assert e_best <= e_gptq * (1 + 1e-12) + 1e-15
        assert e_best <= e_rtn * (1 + 1e-12) + 1e-15
        assert e_gptq <= e_rtn * (1 + 1e-12)
        wins += e_gptq < e_rtn * (1 - 1e-9)
    assert wins >= 3


def test_diagonal_hessian_reduces_to_rtn():
    """Orthogonal inputs give a diagonal H and a diagonal U, so GPTQ has
    nothing to feed forward and equals RTN exactly (codes and scales)."""
    rng = np.random.default_rng(10)
    d = 256
    Q, _ = np.linalg.qr(rng.standard_normal((d, d)))
    X = np.diag(rng.lognormal(0, 0.5, d)) @ np.eye(d)
    W = (rng.standard_normal((16, d)) * 0.02).astype(F32)
    for gs in (-1, 128, 32):
        for sym in (True, False):
            res, H0, U, _, _ = O.gptq_layer(W, X, group_size=gs, sym=sym)
            assert np.count_nonzero(np.triu(U, 1)) == 0
            rtn = O.rtn_quantize(W, gs, sym)
            assert np.array_equal(res.codes, rtn["codes"])
            assert np.array_equal(res.scales, rtn["scales"])
            assert np.array_equal(res.qpacked, rtn["qpacked"])
    del Q


def test_hessian_scale_invariance_and_identity_perm():
    rng = np.random.default_rng(11)
    d = 64
    X = rng.standard_normal((200, d)) * rng.lognormal(0, 0.5, d)
    W = rng.standard_normal((8, d)) * 0.02
    Hd, _ = O.damp_hessian(O.hessian(X), 0.01)
    for gs in (-1, 32):
        a = O.gptq_quantize(W, O.upper_factor_of_inverse(Hd), group_size=gs, block_size=32)
        b = O.gptq_quantize(W, O.upper_factor_of_inverse(7.3 * Hd), group_size=gs, block_size=32)
        c = O.gptq_quantize(W, O.upper_factor_of_inverse(Hd), group_size=gs, block_size=32,
                            perm=np.arange(d))
        assert np.array_equal(a.codes, b.codes)
        assert np.array_equal(a.codes, c.codes) and np.array_equal(a.scales, c.scales)


def test_act_order_groups_and_g_idx():
    rng = np.random.default_rng(12)
    d = 64
    X = rng.standard_normal((300, d)) * rng.lognormal(0, 0.7, d)
    W = rng.standard_normal((8, d)) * 0.02
    res, H0, U, perm, dead = O.gptq_layer(W, X, group_size=16, sym=False, act_order=True)
    assert sorted(perm.tolist()) == list(range(d))
    inv = np.empty(d, int)
    inv[perm] = np.arange(d)
    assert np.array_equal(res.g_idx, inv // 16)
    # dequantising with g_idx reproduces the oracle's W_hat
    Wh = O.dequantize_packed(res.qpacked, res.scales, res.zeros, d, 16, False, g_idx=res.g_idx)
    assert np.array_equal(Wh, res.W_hat)
    # the permuted problem is the plain problem on permuted columns
    plain = O.gptq_quantize(W[:, perm], U, group_size=16, sym=False)
    assert np.array_equal(plain.codes, res.codes[:, perm])


def test_gptq_not_worse_than_rtn_on_correlated_layer():
    rng = np.random.default_rng(13)
    d, n = 128, 400
    base = rng.standard_normal((n, 16))
    X = base @ rng.standard_normal((16, d)) + 0.1 * rng.standard_normal((n, d))
    W = rng.standard_normal((32, d)) * 0.02
    for gs, sym in ((-1, True), (32, True), (32, False)):
        res, *_ = O.gptq_layer(W, X, group_size=gs, sym=sym, block_size=64)
        rtn = O.rtn_quantize(W.astype(F32), gs, sym)
        w_rtn = O.dequantize_packed(rtn["qpacked"], rtn["scales"], rtn["zeros"], d, gs, sym)
        assert O.recon_sse(W, res.W_hat, X) < 0.8 * O.recon_sse(W, w_rtn, X)


def test_mse_two_routes():
    rng = np.random.default_rng(14)
    X = rng.standard_normal((90, 40))
    W = rng.standard_normal((7, 40))
    Wh = W + 0.01 * rng.standard_normal((7, 40))
    a = O.recon_sse(W, Wh, X)
    b = O.recon_sse_trace(W, Wh, O.hessian(X))
    assert abs(a - b) <= 1e-12 * a
    Y = (W - Wh) @ X.T
    assert abs(a - sum(float(v) ** 2 for v in Y.ravel())) <= 1e-12 * a


def test_dead_columns_zeroed():
    rng = np.random.default_rng(15)
    X = rng.standard_normal((50, 16))
    X[:, 3] = 0.0
    W = rng.standard_normal((4, 16)) * 0.02
    res, H0, U, perm, dead = O.gptq_layer(W, X, group_size=-1)
    assert dead.tolist() == [j == 3 for j in range(16)]
    assert np.all(res.W_hat[:, 3] == 0.0)


# -------------------------------------------------------------- planted mistakes

def test_planted_mistakes_are_caught(monkeypatch):
    """Plant plausible mistakes in a copy of the GPTQ loop and check that the
    OBS-equivalence pin rejects each one."""
    rng = np.random.default_rng(16)
    d, rows = 6, 64
    X = rng.standard_normal((10, d)) * rng.lognormal(0, 0.5, d)
    W = rng.standard_normal((rows, d)) * 0.1
    H, _ = O.damp_hessian(O.hessian(X), 0.01)
    U = O.upper_factor_of_inverse(H)
    Hinv = np.linalg.inv(H)
    refs = [O.obs_quantize(W[i], H, _row_quantizer(W[i], True)) for i in range(rows)]

    def matches(Uuse, bs=128):
        r = O.gptq_quantize(W, Uuse, group_size=-1, block_size=bs)
        return all(np.array_equal(refs[i], r.W_hat[i]) for i in range(rows))

    assert matches(U) and matches(U, 2)
    # full inverse instead of its Cholesky factor (the listing read literally)
    assert not matches(np.triu(Hinv))
    # transposed factor (lower instead of upper)
    assert not matches(np.ascontiguousarray(U.T))
    # a wrong sign of the update
    assert not matches(np.diag(np.diag(U)) - np.triu(U, 1))
    # the lazy trailing update dropped (only the 2-column in-block updates kept)
    blockdiag = np.kron(np.eye(d // 2), np.ones((2, 2))) * U
    assert not matches(blockdiag, 2)


@pytest.mark.parametrize("sym", [True, False])
def test_planted_group_params_from_initial_weights_is_caught(sym):
    """Taking each group's scale (and zero) from the initial weights instead
    of the current ones at the group's start is a plausible mistake; the
    grouped OBS pin must tell the two apart.  The mistake is planted in the
    OBS quantiser (a copy of the method on the CPU): the oracle must agree
    with the correct quantiser and disagree with the planted one."""
    rng = np.random.default_rng(18 + sym)
    d, g, rows = 8, 4, 48
    X = rng.standard_normal((12, d)) * rng.lognormal(0, 0.5, d)
    W = rng.standard_normal((rows, d)) * 0.1
    H, _ = O.damp_hessian(O.hessian(X), 0.01)
    U = O.upper_factor_of_inverse(H)
    r = O.gptq_quantize(W, U, group_size=g, block_size=8, sym=sym)
    good = bad = 0
    for i in range(rows):
        good += np.array_equal(O.obs_quantize(W[i], H, _group_quantizer(g, sym)), r.W_hat[i])
        bad += np.array_equal(O.obs_quantize(W[i], H, _group_quantizer(g, sym, W[i])),
                              r.W_hat[i])
    assert good == rows
    assert bad <= rows // 2


def test_tie_follow_only_at_ties():
    """The replay mode adopts another implementation's code only where the
    oracle's own value is a rounding tie; elsewhere it changes nothing."""
    rng = np.random.default_rng(17)
    d = 16
    X = rng.standard_normal((40, d))
    W = (rng.standard_normal((4, d)) * 0.1).astype(np.float64)
    H, _ = O.damp_hessian(O.hessian(X), 0.01)
    U = np.diag(1.0 / np.sqrt(np.diag(H)))         # diagonal: no feedback
    base = O.gptq_quantize(W, U, group_size=-1)
    same = O.gptq_quantize(W, U, group_size=-1, follow=dict(codes=base.codes, scales=base.scales))
    assert same.n_followed == 0 and np.array_equal(same.codes, base.codes)
    other = base.codes.copy()
    other[0, 3] += 1 if other[0, 3] < 7 else -1     # not a tie: must be ignored
    r = O.gptq_quantize(W, U, group_size=-1, follow=dict(codes=other, scales=base.scales))
    assert r.n_followed == 0 and np.array_equal(r.codes, base.codes)
    # plant an exact tie: w = 2.5 s rounds to 2 (half to even); 3 is also correct
    s = float(base.scales[1, 0])
    W2 = W.copy()
    W2[1, 5] = 2.5 * s
    b2 = O.gptq_quantize(W2, U, group_size=-1)
    assert b2.scales[1, 0] == base.scales[1, 0] and b2.codes[1, 5] == 2
    tie = b2.codes.copy()
    tie[1, 5] = 3
    r2 = O.gptq_quantize(W2, U, group_size=-1, follow=dict(codes=tie, scales=b2.scales))
    assert r2.n_followed == 1 and r2.codes[1, 5] == 3
    assert np.array_equal(np.delete(r2.codes.ravel(), 1 * d + 5), np.delete(b2.codes.ravel(), 1 * d + 5))


# ---------------------------------------------------------------- activation-aware scaling

def _awq_case(seed=0, d_in=64, d_out=32, n=512):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((n, d_in))
    X[:, 3] *= 50.0                       # two channels with large activations
    X[:, 10] *= 20.0
    W = rng.standard_normal((d_out, d_in)) * 0.02
    return W, X


def test_awq_scales_closed_form():
    """s_c = (H_cc / H_bar)^(alpha/2): the geometric mean of the scales of the
    live channels is 1, a dead channel gets 1, alpha = 0 gives all ones, and
    the ratio of two channels' scales is (H_aa / H_bb)^(alpha/2)."""
    h = np.array([4.0, 1.0, 0.0, 16.0, 0.25])
    s = O.awq_channel_scales(h, 0.5)
    live = h > 0
    assert abs(np.exp(np.mean(np.log(s[live])))) == pytest.approx(1.0, rel=1e-14)
    assert s[2] == 1.0
    assert s[0] / s[1] == pytest.approx((4.0 / 1.0) ** 0.25, rel=1e-14)
    assert np.all(O.awq_channel_scales(h, 0.0) == 1.0)


def test_awq_alpha_zero_is_rtn():
    """alpha = 0 scales nothing: the codes are plain RTN's and the curve's first
    point is RTN's MSE, computed here by the trace route."""
    W, X = _awq_case()
    H = O.hessian(X)
    for g, sym in ((-1, True), (32, False)):
        res = O.awq_rtn_search(W, X, group_size=g, sym=sym, n_grid=10)
        ref = O.rtn_quantize(W, g, sym)
        Wr = O.dequantize_packed(ref["qpacked"], ref["scales"], ref["zeros"], W.shape[1], g, sym)
        mse_rtn = O.recon_sse_trace(W, Wr, H) / (X.shape[0] * W.shape[0])
        assert res["mse"][0] == pytest.approx(mse_rtn, rel=1e-9)
        r0, _ = O.awq_apply(W, np.ones(W.shape[1], dtype=np.float32), g, sym)
        assert np.array_equal(r0["codes"], ref["codes"])


def test_awq_best_is_consistent_and_helps():
    """The returned effective weights give the curve's minimum (trace route);
    on inputs with outlier channels a positive alpha beats RTN clearly."""
    W, X = _awq_case()
    H = O.hessian(X)
    res = O.awq_rtn_search(W, X, group_size=-1, sym=True, n_grid=10)
    assert res["best"] == int(np.argmin(res["mse"]))
    mse_best = O.recon_sse_trace(W, res["W_hat"], H) / (X.shape[0] * W.shape[0])
    assert mse_best == pytest.approx(res["mse"][res["best"]], rel=1e-9)
    assert res["best"] > 0 and res["mse"][res["best"]] < 0.5 * res["mse"][0]


def test_awq_invariant_to_activation_scale():
    """Scaling every activation by a constant leaves the scales and the choice
    of alpha unchanged and multiplies the MSE curve by the constant squared."""
    W, X = _awq_case(seed=3)
    a = O.awq_rtn_search(W, X, group_size=32, sym=True, n_grid=8)
    b = O.awq_rtn_search(W, 3.0 * X, group_size=32, sym=True, n_grid=8)
    assert a["best"] == b["best"]
    assert np.allclose(a["s"], b["s"], rtol=1e-6)
    assert np.allclose(b["mse"], 9.0 * a["mse"], rtol=1e-6)



# ---------------------------------------------------------------- per-tensor scales

def test_per_tensor_closed_form():
    """group_size 0: one scale s = max |w| / 7 (symmetric) or (max' - min') / 15
    (affine) over the whole matrix, stored in every row; when every row has
    the same extremes it equals the per-channel result, and a single-row
    matrix is per-channel by definition."""
    rng = np.random.default_rng(7)
    W = np.clip(rng.standard_normal((6, 32)) * 0.02, -0.04, 0.04).astype(np.float32)
    W[:, 0] = 0.1                                  # every row's max
    W[:, 1] = -0.05                                # every row's min
    for sym in (True, False):
        pt = O.rtn_quantize(W, 0, sym)
        pc = O.rtn_quantize(W, -1, sym)
        assert np.array_equal(pt["codes"], pc["codes"])
        assert np.array_equal(pt["scales"], pc["scales"])
        one = O.rtn_quantize(W[2:3] * 3.0, 0, sym)
        assert np.array_equal(one["codes"], O.rtn_quantize(W[2:3] * 3.0, -1, sym)["codes"])
    W[4, 7] = 0.7
    pt = O.rtn_quantize(W, 0, True)
    assert np.all(pt["scales"] == np.float16(np.float32(0.7) / np.float32(7)))


def test_per_tensor_gptq_diagonal_is_rtn():
    """With orthogonal inputs (diagonal H) GPTQ with one scale per tensor
    equals RTN with one scale per tensor."""
    d = 64
    X = np.diag(np.linspace(0.5, 3.0, d))
    W = np.random.default_rng(8).standard_normal((10, d)) * 0.02
    for sym in (True, False):
        res, *_ = O.gptq_layer(W, X, group_size=0, sym=sym)
        assert np.array_equal(res.codes, O.rtn_quantize(W, 0, sym)["codes"])


# ---------------------------------------------------------------- W4A16 product

def test_w4a16_grouped_route_and_error_bound():
    """Y = W^ X^T against a second route that never forms W^: per group,
    s (sum_k c_k x_k - z sum_k x_k); and |Y - W X^T| stays within the
    rounding bound sum_k |x_k| s_k / 2 of RTN."""
    rng = np.random.default_rng(9)
    d_out, d_in, n, g = 12, 64, 20, 16
    W = rng.standard_normal((d_out, d_in)) * 0.02
    X = rng.standard_normal((n, d_in))
    for sym in (True, False):
        r = O.rtn_quantize(W, g, sym)
        Y = O.w4a16_matmul(r["qpacked"], r["scales"], r["zeros"], d_in, g, sym, X)
        c = r["codes"].astype(np.float64)
        Y2 = np.zeros((d_out, n))
        for gi in range(d_in // g):
            sl = slice(gi * g, (gi + 1) * g)
            s = r["scales"][:, gi].astype(np.float64)[:, None]
            z = (np.zeros(d_out) if sym else r["zeros"][:, gi].astype(np.float64))[:, None]
            Y2 += s * (c[:, sl] @ X[:, sl].T - z * X[:, sl].sum(axis=1)[None, :])
        assert np.allclose(Y, Y2, rtol=1e-12, atol=1e-12)
        bound = 0.5 * np.abs(X) @ np.repeat(r["scales"].astype(np.float64), g, axis=1).T
        assert np.all(np.abs(Y - W @ X.T) <= bound.T + 1e-12)


# ---------------------------------------------------------------- two-level lazy update

def _gptq_two_level(W, U, S, B=128):
    """Per-channel symmetric GPTQ with the lazy trailing update on two levels
    (the kernels' order): after a block of B columns only the rest of its
    super-block of S columns is updated; after a super-block, every column
    beyond it at once.  Plain numpy, written for this pin."""
    W = np.array(W, dtype=np.float64, copy=True)
    d_out, d_in = W.shape
    s16, z16 = O.sym_params(W.astype(np.float32))
    codes = np.zeros((d_out, d_in), dtype=np.int64)
    for s0 in range(0, d_in, S):
        s1 = min(s0 + S, d_in)
        Err = np.zeros((d_out, s1 - s0))
        for b0 in range(s0, s1, B):
            b1 = min(b0 + B, s1)
            for j in range(b0, b1):
                w = W[:, j]
                c = O.quantize_codes(w, s16, z16, True)
                q = O.dequantize_codes(c, s16, z16)
                codes[:, j] = c
                delta = (w - q) / U[j, j]
                Err[:, j - s0] = delta
                W[:, j + 1:b1] -= np.outer(delta, U[j, j + 1:b1])
            W[:, b1:s1] -= Err[:, b0 - s0:b1 - s0] @ U[b0:b1, b1:s1]
        W[:, s1:] -= Err @ U[s0:s1, s1:]
    return codes


def test_two_level_lazy_update_is_the_same_method():
    """The two-level order of the lazy trailing update (the kernels') gives
    the codes of the one-level form the pages describe: the same terms
    summed in another order."""
    rng = np.random.default_rng(12)
    d_in, d_out, n = 512, 48, 2048
    X = rng.standard_normal((n, d_in)) * np.exp(0.5 * rng.standard_normal(d_in))[None, :]
    W = rng.standard_normal((d_out, d_in)) * 0.02
    H, _ = O.damp_hessian(O.hessian(X), 0.01)
    U = O.upper_factor_of_inverse(H)
    one = O.gptq_quantize(W, U, group_size=-1, block_size=128, sym=True).codes
    for S in (256, 512):
        two = _gptq_two_level(W, U, S)
        assert np.mean(two == one) >= 0.9999
        assert np.max(np.abs(two - one)) <= 1


def test_act_order_follow_only_within_key_ties():
    """The act-order sort adopts another implementation's order only where
    the keys it swaps tie within the stated relative tolerance."""
    key = np.array([5.0, 3.0, 3.0 * (1 + 2e-7), 1.0, 4.0])
    H = np.diag(key)
    own = O.act_order_perm(H)
    assert own.tolist() == [0, 4, 2, 1, 3]
    swapped = np.array([0, 4, 1, 2, 3])            # the near-tie taken the other way
    p, adopted = O.act_order_perm(H, follow=swapped, key_tol=1e-6)
    assert adopted and p.tolist() == swapped.tolist()
    p, adopted = O.act_order_perm(H, follow=swapped, key_tol=1e-8)
    assert not adopted and p.tolist() == own.tolist()
    wrong = np.array([4, 0, 2, 1, 3])               # 4.0 before 5.0: not a tie
    p, adopted = O.act_order_perm(H, follow=wrong)
    assert not adopted and p.tolist() == own.tolist()
    p, adopted = O.act_order_perm(H, follow=own)
    assert not adopted and p.tolist() == own.tolist()


# ---------------------------------------------------------------- other bit widths

@pytest.mark.parametrize("bits,sym_levels", [(2, 3), (3, 7), (4, 15), (8, 255)])
def test_grid_levels_at_other_widths(bits, sym_levels):
    """Symmetric grid -q..q with q = 2^(bits-1) - 1 (2^bits - 1 levels, the
    15 of "GPT-2 Quantization Reconstruction Error" at 4 bits); affine grid
    0..2^bits - 1 (2^bits levels); the absolute maximum maps to the end."""
    rng = np.random.default_rng(30 + bits)
    v = np.concatenate([np.linspace(-1.0, 1.0, 2001), rng.uniform(-1, 1, 20000)])[None].astype(F32)
    s, z = O.sym_params(v, bits)
    c = O.quantize_codes(v, s[:, None], z[:, None], True, bits)
    assert len(np.unique(c)) == sym_levels and c.max() == sym_levels // 2
    s, z = O.affine_params(v, bits)
    c = O.quantize_codes(v, s[:, None], z[:, None], False, bits)
    assert len(np.unique(c)) == 2 ** bits and c.min() == 0 and c.max() == 2 ** bits - 1


def test_packing_bit_positions():
    """Column k of a row occupies stream bits bits*k .. bits*k + bits - 1,
    words little endian: checked against positions worked out by hand."""
    # 8 bits: byte k of word j is column 4j + k
    assert O.pack_nibbles(np.array([[1, 2, 3, 4]]), False, 8).tolist() == [[0x04030201]]
    assert O.pack_nibbles(np.array([[-127, 0, 127, 1]]), True, 8).tolist() == [[0x81FF8001]]
    # 3 bits: column 10 straddles words 0 and 1 (stream bits 30, 31, 32)
    c = np.zeros((1, 32), dtype=np.int64)
    c[0, 10] = 7
    c[0, 0] = 5
    c[0, 31] = 6
    w = O.pack_nibbles(c, False, 3)
    assert w.shape == (1, 3)
    assert w[0, 0] == (5 | (3 << 30)) and w[0, 1] == 1 and w[0, 2] == (6 << 29)
    # 2 bits: column k at bits 2k of word 0 for k < 16 (symmetric zero is stored as 2)
    assert O.pack_nibbles(np.array([[1, 3, 0, 2] + [0] * 12]), False, 2).tolist() == [[1 | 3 << 2 | 2 << 6]]
    sym2 = sum(2 << (2 * k) for k in range(4, 16))
    assert O.pack_nibbles(np.array([[1, -1, 0, 1] + [0] * 12]), True, 2).tolist() == [
        [3 | 1 << 2 | 2 << 4 | 3 << 6 | sym2]]
    rng = np.random.default_rng(31)
    for bits in (2, 3, 4, 8):
        for sym in (True, False):
            lo, hi = (-(2 ** (bits - 1) - 1), 2 ** (bits - 1) - 1) if sym else (0, 2 ** bits - 1)
            codes = rng.integers(lo, hi + 1, size=(5, 64))
            assert np.array_equal(O.unpack_nibbles(O.pack_nibbles(codes, sym, bits), 64, sym, bits),
                                  codes)


@pytest.mark.parametrize("bits", [2, 3, 8])
def test_storage_bits_at_other_widths(bits):
    """bits per code plus 16 bits of scale (and of zero) per group of 128."""
    W = np.random.default_rng(32).standard_normal((8, 1024)).astype(F32) * 0.02
    for sym in (True, False):
        r = O.rtn_quantize(W, 128, sym, bits)
        nbytes = r["qpacked"].nbytes + r["scales"].nbytes + (0 if sym else r["zeros"].nbytes)
        expect = bits + 16 / 128 + (0 if sym else 16 / 128)
        assert nbytes * 8 / W.size == expect == O.bits_per_weight(8, 1024, 128, sym, bits=bits)


@pytest.mark.parametrize("bits", [3, 8])
@pytest.mark.parametrize("sym", [True, False])
def test_cholesky_form_equals_obs_at_other_widths(bits, sym):
    """The OBS equivalence pin does not depend on the grid: it holds at 3
    and 8 bits, per channel and with groups of 4."""
    rng = np.random.default_rng(40 + bits + sym)
    for t in range(20):
        d = 8
        X = rng.standard_normal((int(rng.integers(2, 20)), d)) * rng.lognormal(0, 0.5, d)
        W = rng.standard_normal((4, d)) * 0.1
        H, _ = O.damp_hessian(O.hessian(X), 0.01)
        U = O.upper_factor_of_inverse(H)
        r = O.gptq_quantize(W, U, bits=bits, group_size=-1, sym=sym)
        rg = O.gptq_quantize(W, U, bits=bits, group_size=4, sym=sym)
        for i in range(4):
            s, z = (O.sym_params if sym else O.affine_params)(W[i][None].astype(F32), bits)

            def q(col, row):
                c = O.quantize_codes(np.array([[row[col]]]), s[:, None], z[:, None], sym, bits)
                return float(O.dequantize_codes(c, s[:, None], z[:, None])[0, 0])
            assert np.array_equal(O.obs_quantize(W[i], H, q), r.W_hat[i])

            state = {}

            def qg(col, row):
                if col % 4 == 0:
                    state["p"] = (O.sym_params if sym else O.affine_params)(
                        np.asarray(row[col:col + 4])[None].astype(F32), bits)
                s2, z2 = state["p"]
                c = O.quantize_codes(np.array([[row[col]]]), s2[:, None], z2[:, None], sym, bits)
                return float(O.dequantize_codes(c, s2[:, None], z2[:, None])[0, 0])
            assert np.array_equal(O.obs_quantize(W[i], H, qg), rg.W_hat[i])


def test_eight_bit_error_scales_with_the_step():
    """Rounding error is uniform within half a step, so at a fixed range the
    RTN error variance scales with the squared step: 8-bit against 4-bit
    per channel is (7 / 127)^2 of it, within sampling noise."""
    rng = np.random.default_rng(33)
    W = rng.standard_normal((256, 4096)).astype(F32) * 0.02
    err = {}
    for bits in (4, 8):
        r = O.rtn_quantize(W, -1, True, bits)
        Wh = O.dequantize_packed(r["qpacked"], r["scales"], r["zeros"], 4096, -1, True, bits=bits)
        err[bits] = np.mean((Wh - W) ** 2)
    assert err[8] / err[4] == pytest.approx((7 / 127) ** 2, rel=0.1)


# ---------------------------------------------------------------- sequential pipeline

def test_round_to_bf16_against_library_and_ties():
    """One rounding to 8 significant bits, ties to even: checked at exact
    midpoints and against torch's float32 -> bfloat16 conversion (a single
    rounding for values that float32 holds exactly)."""
    import torch
    assert O.round_to_bf16(1.0 + 2.0 ** -8) == 1.0                  # tie -> even (1.0)
    assert O.round_to_bf16(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6   # tie -> even
    assert O.round_to_bf16(1.0 + 2.0 ** -8 + 2.0 ** -30) == 1.0 + 2.0 ** -7
    assert O.round_to_bf16(-3.0) == -3.0 and O.round_to_bf16(0.0) == 0.0
    v = np.random.default_rng(50).standard_normal(20000).astype(np.float32) * 10.0
    ref = torch.from_numpy(v).to(torch.bfloat16).float().numpy().astype(np.float64)
    assert np.array_equal(O.round_to_bf16(v.astype(np.float64)), ref)


def test_gelu_tanh_closed_forms():
    """gelu(0) = 0; gelu(x) - gelu(-x) = x exactly for the tanh form; the tanh
    form of torch agrees to float32 precision."""
    import torch
    x = np.linspace(-6, 6, 1001)
    assert O.gelu_tanh(0.0) == 0.0
    assert np.allclose(O.gelu_tanh(x) - O.gelu_tanh(-x), x, rtol=0, atol=1e-12)
    t = torch.nn.functional.gelu(torch.from_numpy(x), approximate="tanh").numpy()
    assert np.allclose(O.gelu_tanh(x), t, rtol=1e-12, atol=1e-12)


def test_sequential_pipeline_structure():
    """One layer: the pipeline is gptq_layer plus the layer error.  Two
    layers: the second is calibrated on the first's quantised output, which
    differs from its full-precision output, and the pipeline's errors are
    its layers' errors on the inputs they received."""
    rng = np.random.default_rng(51)
    d, n = 64, 400
    X0 = O.round_to_bf16(rng.standard_normal((n, d)))
    W1 = rng.standard_normal((96, d)) * 0.1
    W2 = rng.standard_normal((d, 96)) * 0.1
    layers = [dict(W=W1, act="gelu"), dict(W=W2, act="none", residual_from=0)]
    res, sse, xs = O.gptq_sequential(X0, layers[:1], group_size=32)
    ref, *_ = O.gptq_layer(W1, X0, group_size=32)
    assert np.array_equal(res[0].codes, ref.codes)
    assert sse[0] == O.recon_sse(W1, ref.W_hat, X0)
    res, sse, xs = O.gptq_sequential(X0, layers, group_size=32)
    X1 = O.apply_layer(X0, res[0].W_hat, "gelu")
    assert np.array_equal(xs[1], X1)
    assert np.array_equal(xs[2], O.apply_layer(X1, res[1].W_hat, "none", X0))
    ref2, *_ = O.gptq_layer(W2, X1, group_size=32)
    assert np.array_equal(res[1].codes, ref2.codes)
    assert sse[1] == O.recon_sse(W2, res[1].W_hat, X1)
    _, _, xs_fp = O.gptq_sequential(X0, layers, group_size=32, quantized_inputs=False)
    assert np.array_equal(xs_fp[1], O.apply_layer(X0, W1, "gelu"))
    assert not np.array_equal(xs_fp[1], xs[1])


def test_tie_window_grows_with_the_updates_a_weight_received():
    """The replay window of a decision is max(TIE_TOL, TIE_REL * E / s) with
    E the accumulated |delta U| applied to the weight: a near-tie inside
    that window is adopted, one just outside it is not."""
    s = 2.0 ** -7                              # fp16-exact scale: absmax 7 s
    # columns 0 and 1 (delta 0.2 s each) update column 2 by -5 s and +5 s:
    # no net change, E = 10 steps
    U = np.eye(4)
    U[0, 2], U[1, 2] = 25.0, -25.0
    win = max(O.TIE_TOL, O.TIE_REL * 10.0)
    assert win > O.TIE_TOL
    for off, adopted in ((0.5 * win, True), (2.0 * win, False)):
        W = np.array([[3.2 * s, 1.2 * s, (2.5 + off) * s, 7 * s]])
        r = O.gptq_quantize(W, U, group_size=-1)
        assert float(r.scales[0, 0]) == s and r.codes[0, 2] == 3
        other = r.codes.copy()
        other[0, 2] = 2
        rf = O.gptq_quantize(W, U, group_size=-1, follow=dict(codes=other, scales=r.scales))
        assert (rf.codes[0, 2] == 2) == adopted, (off, win)
        assert rf.n_followed == int(adopted)


def test_tie_window_scales_with_the_quotient():
    """Near the end of the 8-bit range the fp32 weight and quotient are
    within 2^-23 |w/s| steps of the exact quotient, far more than TIE_TOL:
    the window's floor is QUOT_REL |w/s|.  w/s = 100.5 + off with off one
    fp32 ulp of the quotient (inside 2^-22 * 100.5) is a tie, eight ulps is
    not."""
    s = 2.0 ** -7                              # absmax 127 s: fp16-exact scale s
    U = np.eye(4)
    win = O.QUOT_REL * 100.5
    assert win > O.TIE_TOL
    for off, adopted in ((2.0 ** -17, True), (8 * 2.0 ** -17, False)):
        W = np.array([[127 * s, (100.5 + off) * s, 3 * s, -5 * s]])
        r = O.gptq_quantize(W, U, group_size=-1, bits=8)
        assert float(r.scales[0, 0]) == s and r.codes[0, 1] == 101
        other = r.codes.copy()
        other[0, 1] = 100
        rf = O.gptq_quantize(W, U, group_size=-1, bits=8,
                             follow=dict(codes=other, scales=r.scales))
        assert (rf.codes[0, 1] == 100) == adopted, (off, win)
        assert rf.n_followed == int(adopted)


def test_apply_layer_follow_only_at_rounding_ties():
    """The replay of bf16 roundings takes the other value only where it is
    the rounding of a value within the fp32 error of the fp64 result
    (window 2^-20 * (|X||W| + |Z|) ~ 2^-19 here)."""
    X = np.array([[1.0, 1.0]])
    # Z = 1 + 2^-8 + off: just above the bf16 midpoint between 1 and 1 + 2^-7
    for off, adopted in ((2.0 ** -40, True), (2.0 ** -16, False)):
        W = np.array([[0.5 + 2.0 ** -8 + off, 0.5]])
        Z = O.apply_layer(X, W)
        assert Z[0, 0] == 1.0 + 2.0 ** -7
        Zf, n = O.apply_layer(X, W, follow=np.array([[1.0]]))
        assert (n == 1) == adopted and (Zf[0, 0] == 1.0) == adopted
    # a value two steps away is never taken
    W = np.array([[0.5 + 2.0 ** -8 + 2.0 ** -40, 0.5]])
    Zf, n = O.apply_layer(X, W, follow=np.array([[1.0 + 2.0 ** -6]]))
    assert n == 0 and Zf[0, 0] == 1.0 + 2.0 ** -7
    # cancellation: Z = 2^-30 far below |X||W| = 1, so the window 2^-20 (1 +
    # Z) spans many bf16 steps of Z: any value that rounds some t within it
    # is taken (2^-21, -2^-22), one beyond it is not (2^-19)
    W = np.array([[0.5, -0.5 + 2.0 ** -30]])
    assert O.apply_layer(X, W)[0, 0] == 2.0 ** -30
    for f, adopted in ((2.0 ** -21, True), (-(2.0 ** -22), True), (2.0 ** -19, False)):
        Zf, n = O.apply_layer(X, W, follow=np.array([[f]]))
        assert (n == 1) == adopted and (Zf[0, 0] == f) == adopted
