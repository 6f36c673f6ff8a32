"""Pins of the float64 oracle to facts fixed outside the oracle itself.

Each test ties one oracle function to something it cannot satisfy by
construction: hand-worked examples (tests/golden), closed forms, algebraic
invariants stated on the pages, or a brute-force search written differently
from the oracle's arithmetic.  A plausible slip in the oracle (a dropped factor,
a transposed operand, a wrong sign, a swapped label, a wrong tie rule) fails at
least one of them.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import wush_oracle as O
from workloads import make_inputs, workload, bf16_bits_from_f64

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- Hadamard


def test_hadamard_textbook_order_4():
    # Sylvester construction of order 4, normalised by 1/2 (textbook value).
    H4 = 0.5 * np.array([[1, 1, 1, 1], [1, -1, 1, -1], [1, 1, -1, -1], [1, -1, -1, 1]], float)
    assert np.array_equal(O.sylvester_hadamard(4), H4)


@pytest.mark.parametrize("G", [1, 2, 8, 16, 32, 64])
def test_hadamard_orthonormal_pm_entries(G):
    H = O.sylvester_hadamard(G)
    assert np.allclose(H @ H.T, np.eye(G), atol=1e-15)
    assert np.allclose(np.abs(H), G ** -0.5, atol=0)
    assert np.all(H[0] > 0)


def test_hadamard_rejects_non_power_of_two():
    with pytest.raises(ValueError):
        O.sylvester_hadamard(24)


# ---------------------------------------------------------------- construction invariants


def _tiny_build(lam=0.0, G=32):
    wl = workload("tiny_mxfp4")
    inp = make_inputs(wl)
    return inp, O.build_transforms(inp.w, inp.xcal_bits, G, lam=lam)


def test_inverse_transpose_identity():
    """T_xvsh^T T_wush = I to 1e-9 (unbiasedness constraint T_W = T_X^-T)."""
    _, b = _tiny_build(lam=0.01)
    for Tw, Tx in zip(b["T_wush"], b["T_xvsh"]):
        assert np.max(np.abs(Tx.T @ Tw - np.eye(Tw.shape[0]))) < 1e-9


def test_transformed_second_moments_are_HSH():
    """T_wush Sx T_wush^T = T_xvsh Sw T_xvsh^T = H S H^T, diagonal constant tr(S)/G.

    This also fixes which side gets which transform: with the labels swapped the
    first equality fails."""
    _, b = _tiny_build(lam=0.0)
    G = 32
    H = O.sylvester_hadamard(G)
    for i in range(b["T_wush"].shape[0]):
        Tw, Tx, s = b["T_wush"][i], b["T_xvsh"][i], b["s"][i]
        A = Tw @ b["Sx"][i] @ Tw.T
        B = Tx @ b["Sw"][i] @ Tx.T
        HSH = H @ np.diag(s) @ H.T
        scale = np.max(np.abs(HSH))
        assert np.max(np.abs(A - HSH)) < 1e-9 * scale
        assert np.max(np.abs(B - HSH)) < 1e-9 * scale
        assert np.allclose(np.diag(A), s.sum() / G, rtol=1e-9)
        swapped = Tx @ b["Sx"][i] @ Tx.T
        assert np.max(np.abs(swapped - HSH)) > 1e-3 * scale


def test_inverse_column_norms_equal_mean_singular_value():
    """With T = T_wush W'^-T = H S^-1/2 U^T every column of T^-1 has squared norm tr(S)/G."""
    _, b = _tiny_build(lam=0.01)
    G = 32
    for i in range(b["T_wush"].shape[0]):
        T = b["T_wush"][i] @ np.linalg.inv(b["Wp"][i].T)
        Ti = np.linalg.inv(T)
        norms = np.sum(Ti ** 2, axis=0)
        assert np.allclose(norms, b["s"][i].sum() / G, rtol=1e-9)


def test_singular_values_descending_positive_and_sign_convention():
    _, b = _tiny_build(lam=0.01)
    s = b["s"]
    assert np.all(s > 0)
    assert np.all(np.diff(s, axis=1) <= 0)
    for U in b["U"]:
        j = np.argmax(np.abs(U), axis=0)
        assert np.all(U[j, np.arange(U.shape[1])] > 0)


def test_closed_form_identity_weight_diagonal_activation():
    """Sigma_w = I, Sigma_x = diag(sigma^2), sigma distinct and descending:
    W' = I, X' = diag(sigma), U = V = I, S = diag(sigma), so
    T_wush = H diag(sigma)^-1/2 and T_xvsh = H diag(sigma)^1/2 exactly."""
    G = 16
    sig = np.linspace(3.0, 0.25, G)
    Sw = np.eye(G)[None]
    Sx = np.diag(sig ** 2)[None]
    b = O.transforms_from_moments(Sw, Sx)
    H = O.sylvester_hadamard(G)
    assert np.allclose(b["T_wush"][0], H @ np.diag(sig ** -0.5), atol=1e-12)
    assert np.allclose(b["T_xvsh"][0], H @ np.diag(sig ** 0.5), atol=1e-12)
    assert np.allclose(b["s"][0], sig, atol=1e-12)


def test_closed_form_unsorted_diagonal_uses_sorting_permutation():
    """Unsorted sigma: U = V = P (the permutation sorting sigma descending), so
    T_wush = H P^T diag(sigma)^-1/2 where (P^T)[k, j] = 1 iff j is the k-th largest."""
    G = 8
    sig = np.array([0.5, 2.0, 1.0, 3.0, 0.25, 1.5, 0.75, 4.0])
    b = O.transforms_from_moments(np.eye(G)[None], np.diag(sig ** 2)[None])
    order = np.argsort(-sig)
    Pt = np.zeros((G, G))
    Pt[np.arange(G), order] = 1.0
    H = O.sylvester_hadamard(G)
    assert np.allclose(b["T_wush"][0], H @ Pt @ np.diag(sig ** -0.5), atol=1e-12)
    assert np.allclose(b["T_xvsh"][0], H @ Pt @ np.diag(sig ** 0.5), atol=1e-12)


def test_wus_ablation_is_hadamard_free():
    G = 8
    sig = np.linspace(2, 1, G)
    b = O.transforms_from_moments(np.eye(G)[None], np.diag(sig ** 2)[None], use_hadamard=False)
    assert np.allclose(b["T_wush"][0], np.diag(sig ** -0.5), atol=1e-12)


def test_damping_adds_scaled_identity():
    S = np.array([[[4.0, 1.0], [1.0, 2.0]]])
    D = O.damp(S, 0.5)
    assert np.allclose(D[0], [[5.5, 1.0], [1.0, 3.5]])


def test_second_moments_exact_on_basis_tokens():
    """Tokens that are scaled basis vectors give a diagonal second moment whose entries
    are the mean squared scale per channel; weights with one nonzero per row likewise."""
    G, C = 4, 2
    d = G * C
    x = np.zeros((2 * d, d))
    for j in range(d):
        x[j, j] = 2.0
        x[d + j, j] = -4.0
    w = np.zeros((d, d))
    w[np.arange(d), np.arange(d)] = np.arange(1, d + 1)
    Sw, Sx = O.block_second_moments(w, x, G)
    for i in range(C):
        assert np.allclose(Sx[i], np.eye(G) * (4.0 + 16.0) / (2 * d))
        assert np.allclose(Sw[i], np.diag(np.arange(i * G + 1, i * G + G + 1) ** 2 / d))


def test_transformed_calibration_data_has_HSH_moment():
    """End-to-end pin of second moments + construction + block_transform on data:
    the empirical second moment of y = T_wush x over the calibration tokens is H S H^T,
    and of T_xvsh w over the weight rows likewise (lam = 0, exact algebra)."""
    inp, b = _tiny_build(lam=0.0)
    xcal = O.bf16_to_f64(inp.xcal_bits)
    y = O.block_transform(xcal, b["T_wush"])
    wb = O.block_transform(inp.w.astype(np.float64), b["T_xvsh"])
    G = 32
    H = O.sylvester_hadamard(G)
    for i in range(b["T_wush"].shape[0]):
        HSH = H @ np.diag(b["s"][i]) @ H.T
        yi = y[:, i * G:(i + 1) * G]
        wi = wb[:, i * G:(i + 1) * G]
        assert np.allclose(yi.T @ yi / yi.shape[0], HSH, atol=1e-9 * np.max(np.abs(HSH)))
        assert np.allclose(wi.T @ wi / wi.shape[0], HSH, atol=1e-9 * np.max(np.abs(HSH)))


def test_unquantised_product_preserved():
    """W^T X is unchanged by the transform pair: sum over blocks of (T_xvsh w).(T_wush x) = w.x."""
    inp, b = _tiny_build(lam=0.01)
    x = O.bf16_to_f64(inp.x_bits)
    w = inp.w.astype(np.float64)
    ref = w @ x.T
    got = O.block_transform(w, b["T_xvsh"]) @ O.block_transform(x, b["T_wush"]).T
    assert np.max(np.abs(got - ref)) < 1e-9 * np.max(np.abs(ref))


# ---------------------------------------------------------------- block_transform


def test_block_transform_permutation_and_identity():
    rng = np.random.default_rng(1)
    G, C, n = 4, 3, 5
    x = rng.standard_normal((n, C * G))
    I = np.stack([np.eye(G)] * C)
    assert np.array_equal(O.block_transform(x, I), x)
    # T_i maps channel c to output r = (c + 1) mod G, i.e. T[r, c] = 1 iff r = c + 1 mod G.
    P = np.zeros((G, G))
    P[(np.arange(G) + 1) % G, np.arange(G)] = 1.0
    Ts = np.stack([P, np.eye(G), 2 * np.eye(G)])
    y = O.block_transform(x, Ts)
    xb = x.reshape(n, C, G)
    assert np.array_equal(y.reshape(n, C, G)[:, 0, (np.arange(G) + 1) % G], xb[:, 0, :])
    assert np.array_equal(y.reshape(n, C, G)[:, 1], xb[:, 1])
    assert np.array_equal(y.reshape(n, C, G)[:, 2], 2 * xb[:, 2])


def test_block_transform_basis_vector_gives_column():
    G = 8
    T = np.arange(G * G, dtype=float).reshape(1, G, G)
    for c in range(G):
        e = np.zeros((1, G))
        e[0, c] = 1.0
        assert np.array_equal(O.block_transform(e, T)[0], T[0][:, c])


def test_transform_groups_basis_vectors_and_block_choice():
    """Each sampled group uses its own block's matrix: basis vectors pick its columns,
    and a group of ones gives that block's row sums (exact in float64 for small ints)."""
    G, C = 4, 3
    T = np.arange(C * G * G, dtype=float).reshape(C, G, G)
    for blk in range(C):
        for c in range(G):
            e = np.zeros((1, G))
            e[0, c] = 1.0
            assert np.array_equal(O.transform_groups(e, T, np.array([blk]))[0], T[blk][:, c])
    ones = np.ones((C, G))
    y = O.transform_groups(ones, T, np.array([2, 0, 1]))
    assert np.array_equal(y, np.stack([T[2].sum(axis=1), T[0].sum(axis=1), T[1].sum(axis=1)]))


def test_layer_loss_zero_when_quantisation_is_exact():
    """Identity transforms and values already on the MXFP4 grid (scale 1): q is exact,
    the loss is 0; an INT4 grid input likewise."""
    G, d_in, d_out, n = 32, 64, 3, 4
    I = np.stack([np.eye(G)] * (d_in // G)).astype(np.float32)
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, -0.5, -6.0])
    rng = np.random.default_rng(3)
    w = rng.choice(grid, (d_out, d_in)).astype(np.float32)
    x = rng.choice(grid, (n, d_in))
    w[:, 0] = 6.0                         # every group's amax is 6: scale 2^0
    x[:, ::G] = 6.0
    from workloads import bf16_bits_from_f64
    xb = bf16_bits_from_f64(x)
    assert O.layer_loss(w, xb, I, I, "mxfp4", G) == 0.0
    wi = rng.integers(-7, 8, (d_out, d_in)).astype(np.float32)
    xi = rng.integers(-7, 8, (n, d_in)).astype(np.float64)
    wi[:, ::G] = 7.0
    xi[:, ::G] = 7.0
    assert O.layer_loss(wi, bf16_bits_from_f64(xi), I, I, "int4", G) == 0.0


def test_layer_loss_matches_hand_computed_single_group():
    """One output, one token, one INT4 group of 16: x = (7, 1.4, 0, ...), w = (1, 1, 0, ...).
    s_x = 7/7 = 1, q(x) = (7, 1, 0...); s_w = fl32(1/7), w codes (7, 7, 0...), so the
    quantised product is 7 s_w * 7 + 7 s_w * 1 = 56 s_w; W^T X = 7 + bf16(1.4)."""
    G = 16
    I = np.eye(G, dtype=np.float32)[None]
    x = np.zeros((1, G)); x[0, 0] = 7.0; x[0, 1] = 1.4
    w = np.zeros((1, G), np.float32); w[0, 0] = 1.0; w[0, 1] = 1.0
    from workloads import bf16_bits_from_f64
    xb = bf16_bits_from_f64(x)
    x1 = O.bf16_to_f64(xb)[0, 1]               # 1.4 rounded to bfloat16
    s_w = float(np.float32(1.0) / np.float32(7.0))
    expect = (7.0 + x1 - 56.0 * s_w) ** 2
    assert abs(O.layer_loss(w, xb, I, I, "int4", G) - expect) < 1e-12


def test_scale_atoms_places_bytes_by_the_atom_formula():
    rows, C = 300, 10
    s = (np.arange(rows * C) % 251).astype(np.uint8).reshape(rows, C)
    at = O.scale_atoms(s)
    rows_pad, C_pad = 384, 12
    assert at.shape == (rows_pad * C_pad,)
    for r, c in [(0, 0), (33, 5), (127, 9), (128, 0), (299, 9), (200, 3)]:
        rb, i, j = r // 128, r % 32, (r % 128) // 32
        off = (rb * (C_pad // 4) + c // 4) * 512 + 16 * i + 4 * j + c % 4
        assert at[off] == s[r, c]
    assert at[(2 * 3 + 2) * 512 + 16 * 31 + 4 * 3 + 3] == 0       # padding row 383, column 11
    assert sorted(at[at > 0].tolist()) == sorted(s[s > 0].tolist())


def test_gemm_mx_exact_small_cases():
    """All codes 1.0 at scale 2^0: every output is K.  A at 2^1 and B at 2^-1 with codes
    1.5 and -2: every output is K * 1.5 * -2."""
    M, N, K = 4, 3, 64
    one = O.pack_nibbles(np.full((M, K), 2, np.uint8))               # E2M1 code 2 = 1.0
    oneb = O.pack_nibbles(np.full((N, K), 2, np.uint8))
    d = O.gemm_mx(one, np.full((M, K // 32), 127, np.uint8), oneb, np.full((N, K // 32), 127, np.uint8))
    assert np.array_equal(d, np.full((M, N), float(K)))
    a = O.pack_nibbles(np.full((M, K), 3, np.uint8))                 # 1.5
    b = O.pack_nibbles(np.full((N, K), 0xC, np.uint8))               # -2
    d = O.gemm_mx(a, np.full((M, K // 32), 128, np.uint8), b, np.full((N, K // 32), 126, np.uint8))
    assert np.array_equal(d, np.full((M, N), K * 1.5 * -2.0))


def test_gemm_nv_exact_small_cases():
    """E2M1 1.0 everywhere.  A's E4M3 scales 2.0 (0x40) at tensor scale 0.25, B's 0.5
    (0x30) at 3.0: every product is 0.5 * 1.5, so each output is 0.75 K.  Then A's groups
    alternate 1.0 (0x38) and the smallest subnormal 2^-9 (0x01) with everything else 1:
    each 16-wide group contributes 16 times its scale."""
    M, N, K = 2, 3, 64
    a = O.pack_nibbles(np.full((M, K), 2, np.uint8))
    b = O.pack_nibbles(np.full((N, K), 2, np.uint8))
    d = O.gemm_nv(a, np.full((M, K // 16), 0x40, np.uint8), 0.25, b, np.full((N, K // 16), 0x30, np.uint8), 3.0)
    assert np.array_equal(d, np.full((M, N), 0.75 * K))
    sa = np.tile(np.array([0x38, 0x01], np.uint8), (M, K // 32))
    d = O.gemm_nv(a, sa, 1.0, b, np.full((N, K // 16), 0x38, np.uint8), 1.0)
    assert np.array_equal(d, np.full((M, N), (K // 32) * (16.0 + 16.0 * 2.0 ** -9)))


def test_gptq_block_second_column_takes_the_obs_correction():
    """Two columns, Hb = [[a, b], [b, c]] undamped: after column 0 is rounded, column 1
    moves by (w0 - q0) b / c (the optimal brain surgeon update), then is rounded."""
    a_, b_, c_ = 2.0, 0.7, 1.5
    Hb = np.array([[a_, b_], [b_, c_]])
    Wb = np.array([[1.3, 0.4], [-0.9, 2.2], [0.26, -1.1]])
    Q, codes, sc = O.gptq_block(Wb, Hb, "int4", damp_frac=0.0)
    s = O.fl32(np.max(np.abs(Wb), axis=1) / 7.0)
    inv = O._recip32(s)
    q0 = np.clip(np.rint(O.fl32(Wb[:, 0] * inv)), -7, 7) * s
    w1 = Wb[:, 1] + (Wb[:, 0] - q0) * b_ / c_
    q1 = np.clip(np.rint(O.fl32(w1 * inv)), -7, 7) * s
    assert np.allclose(Q[:, 0], q0, rtol=0, atol=0) and np.allclose(Q[:, 1], q1, rtol=1e-15, atol=0)


def test_gptq_block_with_diagonal_hessian_is_plain_rounding():
    rng = np.random.default_rng(4)
    Wb = rng.standard_normal((6, 32))
    for fmt in ("mxfp4", "int4"):
        Q, codes, sc = O.gptq_block(Wb, np.diag(rng.uniform(0.5, 2.0, 32)), fmt)
        c_ref, s_ref, _ = O.quantize(Wb, fmt, 32)
        assert np.array_equal(codes, c_ref) and np.array_equal(sc, s_ref.reshape(-1))


def test_gptq_wush_rtn_mode_reconstructs_the_target_exactly():
    """RTN mode feeds back the unquantised transformed weights, so the residual target
    vanishes; every block's transforms satisfy T_W^T T_X = I and
    T_X X'_ii X'_ii^T T_X^T = H S H^T."""
    wl = workload("tiny_mxfp4")
    inp = make_inputs(wl)
    r = O.gptq_wush(inp.w, inp.xcal_bits, 32, "mxfp4", gptq=False)
    assert np.linalg.norm(r["Y"]) <= 1e-10 * np.linalg.norm(inp.w.astype(np.float64))
    for i in range(r["T_act"].shape[0]):
        assert np.max(np.abs(r["T_w"][i].T @ r["T_act"][i] - np.eye(32))) < 1e-9


def test_gptq_wush_single_block_agrees_with_the_per_block_construction():
    """With one block the global factor is the block's own Cholesky factor, so up to the
    signs of the singular-vector pairs the transforms and transformed weights are those
    of the per-block WUSH builder: |H^T T| and |H^T W_bar| agree entry by entry."""
    wl = workload("tiny_mxfp4", d_in=32, d_out=64, n_cal=256)
    inp = make_inputs(wl)
    # undamped on both sides (the per-block builder also damps the weight moment)
    r = O.gptq_wush(inp.w, inp.xcal_bits, 32, "mxfp4", gptq=False, lam=0.0)
    b = O.build_transforms(inp.w, inp.xcal_bits, 32, lam=0.0)
    H = O.sylvester_hadamard(32)
    assert np.allclose(np.abs(H.T @ r["T_act"][0]), np.abs(H.T @ b["T_wush"][0]), rtol=1e-7, atol=1e-9)
    wbar_ref = b["T_xvsh"][0] @ inp.w.astype(np.float64).T
    assert np.allclose(np.abs(H.T @ r["W_bar"][0]), np.abs(H.T @ wbar_ref), rtol=1e-7, atol=1e-9)


def test_gptq_error_feedback_lowers_the_layer_loss():
    wl = workload("tiny_mxfp4")
    inp = make_inputs(wl)
    for fmt in ("mxfp4", "int4"):
        losses = {}
        for gq in (False, True):
            r = O.gptq_wush(inp.w, inp.xcal_bits, 32, fmt, gptq=gq)
            losses[gq] = O.layer_loss_prequantised(r["Wq"], inp.w, inp.xcal_bits, r["T_act"].astype(np.float32),
                                                   fmt, 32)
        assert losses[True] < 0.95 * losses[False], (fmt, losses)


# ---------------------------------------------------------------- grids, brute force


def _e2m1_brute(v):
    """Exhaustive nearest-grid search over the eight magnitudes; ties -> even index."""
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    a = abs(v)
    best = None
    for m, g in enumerate(grid):
        d = abs(g - a)
        if best is None or d < best[0] or (d == best[0] and m % 2 == 0):
            best = (d, m)
    return best[1] | (8 if math.copysign(1.0, v) < 0 else 0)


def test_e2m1_matches_brute_force():
    rng = np.random.default_rng(7)
    vals = np.concatenate([rng.uniform(-8, 8, 4000),
                           np.arange(-7.0, 7.01, 0.25),   # every tie point and grid point
                           [6.0000001, -6.5, 100.0, 0.0, -0.0, 1e-30]])
    got = O.e2m1_encode(vals)
    for v, g in zip(vals, got):
        assert int(g) == _e2m1_brute(float(v)), v


def test_e2m1_decode_roundtrip():
    codes = np.arange(16, dtype=np.uint8)
    back = O.e2m1_encode(O.e2m1_decode(codes))
    assert np.array_equal(back, codes)


def _e4m3_value(b):
    s = -1.0 if b & 0x80 else 1.0
    e = (b >> 3) & 0xF
    m = b & 7
    if e == 0:
        return s * m / 512.0
    return s * (8 + m) / 8.0 * 2.0 ** (e - 7)


def _e4m3_brute(r):
    """Nearest over all 127 non-negative finite codes (0x00..0x7E); ties -> even code;
    values beyond 448 saturate."""
    a = abs(r)
    best = None
    for b in range(0x7F):
        d = abs(_e4m3_value(b) - a)
        if best is None or d < best[0] or (d == best[0] and b % 2 == 0):
            best = (d, b)
    return best[1] | (0x80 if r < 0 else 0)


def test_e4m3_matches_brute_force_and_golden():
    rng = np.random.default_rng(3)
    vals = np.concatenate([rng.uniform(0, 460, 300), np.exp(rng.uniform(-9, 6, 700)),
                           [_e4m3_value(b) for b in range(0x7F)],
                           [(_e4m3_value(b) + _e4m3_value(b + 1)) / 2 for b in range(0x7E)]])
    got = O.e4m3_encode(vals)
    for v, g in zip(vals, got):
        assert int(g) == _e4m3_brute(float(v)), v
    with open(os.path.join(GOLDEN, "e4m3_examples.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            v, b = (t.strip() for t in line.split("|"))
            assert int(O.e4m3_encode(np.array([float(v)]))[0]) == int(b, 16), line
    for b in range(0x7F):
        assert O.e4m3_decode(np.array([b], np.uint8))[0] == _e4m3_value(b)


def _mx_exponent_brute(amax):
    if amax == 0:
        return -127
    a = Fraction(amax)
    for e in range(-400, 400):
        if a <= 6 * Fraction(2) ** e:
            return max(-127, min(127, e))
    raise AssertionError


def test_mxfp4_exponent_matches_search():
    rng = np.random.default_rng(11)
    vals = np.concatenate([np.exp(rng.uniform(-100, 80, 500)).astype(np.float32).astype(np.float64),
                           [6.0 * 2.0 ** k for k in range(-20, 20)],
                           [np.nextafter(np.float32(6.0 * 2.0 ** k), np.float32(np.inf)) for k in range(-5, 5)],
                           [3.0, 0.0, 2.0 ** -140, 1e-45]])
    got = O.mxfp4_exponent(vals)
    for v, g in zip(vals, got):
        assert int(g) == _mx_exponent_brute(float(v)), v


def test_int4_rounding_matches_brute_force():
    rng = np.random.default_rng(5)
    y = rng.standard_normal((50, 32)) * rng.uniform(0.01, 10, (50, 1))
    codes, s = O.quant_int4(y, 32)
    q = O.int4_decode(codes)
    for r in range(y.shape[0]):
        sc = np.float32(np.max(np.abs(y[r])) / 7.0)
        inv = np.float32(1.0 / np.float64(sc))
        assert s[r, 0] == sc
        for j in range(32):
            v = float(np.float32(y[r, j] * np.float64(inv)))
            best = min(range(-7, 8), key=lambda k: (abs(k - v), k % 2))
            assert q[r, j] == best


def _read_quant_examples():
    rows = []
    with open(os.path.join(GOLDEN, "quant_examples.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            fmt, ctx, vals, scale, codes = (t.strip() for t in line.split("|"))
            rows.append((fmt, ctx, [float(v) for v in vals.split()], scale,
                         [int(c, 16) for c in codes.split()]))
    return rows


@pytest.mark.parametrize("row", _read_quant_examples(), ids=lambda r: f"{r[0]}:{r[2][:2]}")
def test_hand_worked_examples(row):
    fmt, ctx, vals, scale, codes = row
    g = {"mxfp4": 32, "nvfp4": 16, "int4": 32}[fmt]
    y = np.zeros((1, g))
    y[0, :len(vals)] = vals
    want = np.zeros(g, dtype=np.uint8)
    want[:len(codes)] = codes
    if fmt == "mxfp4":
        c, s = O.quant_mxfp4(y)
        assert int(s[0, 0]) == int(scale, 16)
    elif fmt == "nvfp4":
        st = float(ctx.split("=")[1])
        c, s, _ = O.quant_nvfp4(y, st)
        assert int(s[0, 0]) == int(scale, 16)
    else:
        c, s = O.quant_int4(y, g)
        assert float(s[0, 0]) == float(scale)
    assert np.array_equal(c[0], want), (c[0][:len(codes)], codes)


def test_ocp_floor_rule_differs_on_7():
    """The alternative OCP exponent saturates 7 to 6 while the AbsMax rule keeps 8."""
    y = np.zeros((1, 32))
    y[0, 0] = 7.0
    c_abs, s_abs = O.quant_mxfp4(y)
    c_ocp, s_ocp = O.quant_mxfp4(y, rule="ocp_floor")
    assert O.dequant(c_abs, s_abs, "mxfp4", 32)[0, 0] == 8.0
    assert O.dequant(c_ocp, s_ocp, "mxfp4", 32)[0, 0] == 6.0


def test_nvfp4_tensor_scale_definition():
    assert O.nvfp4_tensor_scale(2688.0) == 1.0
    assert O.nvfp4_tensor_scale(0.0) == 0.0
    # amax / 2688 rounded to float32
    assert O.nvfp4_tensor_scale(1.0) == float(np.float32(1.0 / 2688.0))


def test_nvfp4_zero_and_underflow_groups():
    y = np.zeros((1, 32))
    y[0, 0] = 2688.0          # tensor amax -> s_t = 1
    y[0, 16] = 1e-4           # r = 1e-4/6 < 2^-10 -> E4M3 0 -> whole group zero
    c, s, st = O.quant_nvfp4(y)
    assert st == 1.0 and s[0, 1] == 0 and np.all(c[0, 16:] & 7 == 0)


# ---------------------------------------------------------------- packing


def test_pack_low_nibble_is_even_element():
    c = np.array([[1, 2, 3, 4, 0xF, 0]], dtype=np.uint8)
    p = O.pack_nibbles(c)
    assert p.tolist() == [[0x21, 0x43, 0x0F]]
    assert np.array_equal(O.unpack_nibbles(p), c)


# ---------------------------------------------------------------- composed path


@pytest.mark.parametrize("fmt,G", [("mxfp4", 32), ("nvfp4", 16), ("int4", 32), ("int4", 16)])
def test_quantiser_error_bound_and_amax_code(fmt, G):
    """Every element dequantises to its nearest grid point at the group's scale, the
    block maximum never saturates (MXFP4/INT4) and lands on the top binade."""
    rng = np.random.default_rng(17)
    y = rng.standard_t(3, (200, 4 * G)) * np.exp(rng.uniform(-6, 6, (200, 1)))
    c, s, st = O.quantize(y, fmt, G)
    deq = O.dequant(c, s, fmt, G, st)
    g = y.reshape(200, 4, G)
    dg = deq.reshape(200, 4, G)
    if fmt == "mxfp4":
        sc = np.exp2(s.astype(float) - 127)[:, :, None]
        err = np.abs(dg - g) / sc
        v = np.abs(g) / sc
        half = np.where(v < 2, 0.25, np.where(v < 4, 0.5, 1.0))
        assert np.all(err <= half + 1e-12)
        top = np.abs(g).max(axis=2, keepdims=True) / sc
        assert np.all((top > 3) & (top <= 6))
    elif fmt == "int4":
        sc = s.astype(float)[:, :, None]
        assert np.all(np.abs(dg - g) <= 0.5 * sc * (1 + 1e-6))
        q = O.int4_decode(c).reshape(200, 4, G)
        amax_idx = np.argmax(np.abs(g), axis=2)
        assert np.all(np.abs(np.take_along_axis(q, amax_idx[:, :, None], 2)) == 7)
    else:
        scd = (O.e4m3_decode(s) * st)[:, :, None]
        zero = (s == 0)[:, :, None]                     # block scale underflowed: group is all zero
        assert np.all(np.broadcast_to(zero, g.shape) <= (dg == 0))
        with np.errstate(divide="ignore", invalid="ignore"):
            v = np.where(zero, 0.0, np.abs(g) / np.where(zero, 1.0, scd))
        half = np.where(v < 2, 0.25, np.where(v < 4, 0.5, 1.0)) * scd
        ok = (np.abs(dg - g) <= half * (1 + 1e-6)) | zero
        sat = v > 6.0
        assert np.all(ok | sat)
        # the 3-bit mantissa of a normal E4M3 scale rounds by at most 1/16, so a group
        # maximum can exceed 6 only a little before it saturates
        normal = np.broadcast_to((s >= 0x08)[:, :, None], g.shape)
        assert np.all(v[sat & normal] < 6.0 * (1 + 2 ** -3))


def test_quant_act_tiny_bit_patterns_and_shapes():
    wl = workload("tiny_mxfp4")
    inp = make_inputs(wl)
    b = O.build_transforms(inp.w, inp.xcal_bits, 32)
    codes, scales, st, y = O.quant_act(inp.x_bits, b["T_wush32"], 32, "mxfp4")
    assert codes.shape == (64, 128) and scales.shape == (64, 8) and st is None
    deq = O.dequant(O.unpack_nibbles(codes), scales, "mxfp4", 32)
    # MXFP4 relative error on Gaussian-like data: a few percent, far below 1
    rel = np.linalg.norm(deq - y) / np.linalg.norm(y)
    assert 1e-3 < rel < 0.2


def test_generator_bf16_rounding_is_rne():
    v = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -9, -2.5, 1.0 + 2 ** -7 + 2 ** -8])
    bits = bf16_bits_from_f64(v)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7 -> even (1.0); 1 + 3*2^-9 rounds up to 1 + 2^-7;
    # 1 + 2^-7 + 2^-8 ties between 1+2^-7 (odd) and 1+2^-6 (even) -> 1 + 2^-6.
    assert np.array_equal(O.bf16_to_f64(bits), [1.0, 1.0, 1.0 + 2 ** -7, -2.5, 1.0 + 2 ** -6])


# ---------------------------------------------------------------- grid-step distance (rule 2)


def _read_grid_steps():
    rows = []
    with open(os.path.join(GOLDEN, "grid_steps.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            fmt, a, b, steps, _ = (t.strip() for t in line.split("|"))
            rows.append((fmt, int(a, 16), int(b, 16), int(steps)))
    return rows


@pytest.mark.parametrize("row", _read_grid_steps(), ids=lambda r: f"{r[0]}:{r[1]:x}-{r[2]:x}")
def test_grid_step_distance_hand_worked(row):
    fmt, a, b, steps = row
    ofmt = "mxfp4" if fmt == "e2m1" else "int4"
    assert int(O.grid_step_distance(np.array([a]), np.array([b]), ofmt)[0]) == steps
    assert int(O.grid_step_distance(np.array([b]), np.array([a]), ofmt)[0]) == steps
    if ofmt == "mxfp4":    # NVFP4 shares the E2M1 grid
        assert int(O.grid_step_distance(np.array([a]), np.array([b]), "nvfp4")[0]) == steps


def test_grid_step_distance_is_the_rank_difference_on_the_signed_grid():
    """Brute force over every code pair: the distance equals the difference of the two
    values' ranks in the sorted list of distinct signed grid points (a table written
    here from the E2M1 magnitudes, not the oracle's code arithmetic)."""
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    val = {c: (-mags[c & 7] if c & 8 else mags[c & 7]) for c in range(16)}
    line = sorted(set(v + 0.0 for v in val.values()))           # -0.0 + 0.0 == 0.0
    assert len(line) == 15
    rank = {c: line.index(val[c] + 0.0) for c in range(16)}
    a, b = np.meshgrid(np.arange(16), np.arange(16), indexing="ij")
    d = O.grid_step_distance(a.ravel(), b.ravel(), "mxfp4")
    want = np.array([abs(rank[i] - rank[j]) for i, j in zip(a.ravel(), b.ravel())])
    assert np.array_equal(d, want)
    # INT4: the 15 valid nibbles (0x8 = -8 is never emitted) on the integer line
    codes = [c for c in range(16) if c != 8]
    ival = {c: c if c < 8 else c - 16 for c in codes}
    ia, ib = np.meshgrid(codes, codes, indexing="ij")
    d = O.grid_step_distance(ia.ravel(), ib.ravel(), "int4")
    assert np.array_equal(d, np.array([abs(ival[i] - ival[j]) for i, j in zip(ia.ravel(), ib.ravel())]))


# ---------------------------------------------------------------- Eq. (5) with pre-quantised weights


def test_layer_loss_prequantised_hand_computed():
    """Two outputs, one token, one INT4 group of 16 (T_X = I).  x = (7, 1.4, 0, ...) so
    q(x) = (7, 1, 0, ...) at s = 1 (the 1.4 -> 1 rounding makes q(x) != x).  With
    w rows (1, 1, 0...) and (0, 2, 0...), and given dequantised weights wq rows
    (0.5, 0.25, 0...) and (0, 3, 0...):
      output 0: 7 + x1 - (0.5 * 7 + 0.25 * 1) = 3.25 + x1
      output 1: 2 x1 - 3 * 1                    = 2 x1 - 3
    and Eq. (5) divides the squared sum by d_out * d_batch = 2."""
    G = 16
    I = np.eye(G, dtype=np.float32)[None]
    x = np.zeros((1, G)); x[0, 0] = 7.0; x[0, 1] = 1.4
    xb = bf16_bits_from_f64(x)
    x1 = O.bf16_to_f64(xb)[0, 1]
    w = np.zeros((2, G), np.float32); w[0, 0] = 1.0; w[0, 1] = 1.0; w[1, 1] = 2.0
    wq = np.zeros((2, G)); wq[0, 0] = 0.5; wq[0, 1] = 0.25; wq[1, 1] = 3.0
    expect = ((3.25 + x1) ** 2 + (2 * x1 - 3.0) ** 2) / 2.0
    got = O.layer_loss_prequantised(wq, w, xb, I, "int4", G)
    assert abs(got - expect) < 1e-12
    # swapping the roles of w and wq changes the value (x is not exactly representable)
    swapped = O.layer_loss_prequantised(w.astype(np.float64), wq.astype(np.float32), xb, I, "int4", G)
    assert abs(swapped - expect) > 1e-3


def test_layer_loss_prequantised_equals_layer_loss_on_rtn_weights():
    """With wq = the RTN dequantisation of T_W W, Eq. (5) for pre-quantised weights is
    the plain layerwise loss (the GPTQ-free case of the same objective)."""
    wl = workload("tiny_mxfp4")
    inp = make_inputs(wl)
    b = O.build_transforms(inp.w, inp.xcal_bits, wl.G)
    for fmt, G in (("mxfp4", 32), ("int4", 32)):
        bb = b if G == wl.G else O.build_transforms(inp.w, inp.xcal_bits, G)
        cw, sw, tw, _ = O.quant_weight(inp.w, bb["T_xvsh32"], G, fmt)
        wq = O.dequant(O.unpack_nibbles(cw), sw, fmt, G, tw)
        ref = O.layer_loss(inp.w, inp.x_bits, bb["T_xvsh32"], bb["T_wush32"], fmt, G)
        got = O.layer_loss_prequantised(wq, inp.w, inp.x_bits, bb["T_wush32"], fmt, G)
        assert got == pytest.approx(ref, rel=1e-12)
