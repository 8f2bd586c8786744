"""Pins for the fp64 oracle, checked against things other than itself.

Each test names what fixes the expected value: a hand-computed example,
brute-force loops written in a different association than the oracle, a
closed form, finite differences of a function that is exactly linear in the
perturbed argument, or an invariant stated for the layer (B = 0 gives the
base projection, merged == unmerged, restore-from-pristine is bit-identical
while a bf16 merge/unmerge pair drifts).
"""
import hashlib
import itertools
import json
import os

import numpy as np
import pytest
import torch

import oracle as O
import workloads as WL
from tolerance import lora_tol_check, merge_tol_check

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rng_mats(seed, M, d_in, d_out, r):
    g = np.random.default_rng(seed)
    X = g.standard_normal((M, d_in))
    W = g.standard_normal((d_out, d_in))
    A = g.standard_normal((r, d_in))
    B = g.standard_normal((d_out, r))
    dY = g.standard_normal((M, d_out))
    return X, W, A, B, dY


# ---------------------------------------------------------------- bf16 ------

def test_bf16_known_bit_patterns():
    # IEEE: 1.0 = 0x3F80, -2.0 = 0xC000, 0.5 = 0x3F00, 3.0 = 0x4040, 0 = 0.
    bits = np.array([0x3F80, 0xC000, 0x3F00, 0x4040, 0x0000], dtype=np.uint16)
    vals = O.bf16_bits_to_f64(bits)
    assert vals.tolist() == [1.0, -2.0, 0.5, 3.0, 0.0]
    assert O.f64_to_bf16_bits(vals).tolist() == bits.tolist()


def test_bf16_round_ties_to_even():
    # bf16 spacing on [1, 2) is 2**-7.  1 + 2**-8 is a tie -> even (1.0);
    # 1 + 3*2**-8 is a tie between 1+2**-7 (odd) and 1+2**-6 (even).
    assert O.bf16_round(1 + 2.0 ** -8) == 1.0
    assert O.bf16_round(1 + 3 * 2.0 ** -8) == 1 + 2.0 ** -6
    assert O.bf16_round(-(1 + 3 * 2.0 ** -8)) == -(1 + 2.0 ** -6)
    assert O.bf16_round(1 + 2.0 ** -8 + 2.0 ** -30) == 1 + 2.0 ** -7


def test_bf16_round_matches_torch_cast_on_float32_values():
    # For float32-representable inputs, RNE to bf16 is torch's cast.
    g = torch.Generator().manual_seed(3)
    x = torch.randn(20000, generator=g) * torch.exp(torch.randn(20000, generator=g) * 4)
    ours = O.bf16_round(x.double().numpy())
    ref = x.to(torch.bfloat16).double().numpy()
    assert np.array_equal(ours, ref)


def test_ulp_bf16_values():
    assert O.ulp_bf16(1.0) == 2.0 ** -7
    assert O.ulp_bf16(1.5) == 2.0 ** -7
    assert O.ulp_bf16(2.0) == 2.0 ** -6
    assert O.ulp_bf16(-0.75) == 2.0 ** -8


# ------------------------------------------------------ hand example ------

def test_hand_example():
    with open(os.path.join(GOLDEN, "hand_example.json")) as f:
        g = json.load(f)
    X, W, A, B, dY = (np.array(g[k], dtype=np.float64) for k in ("X", "W", "A", "B", "dY"))
    alpha = g["alpha"]
    assert O.scale_of(alpha, g["r"]) == g["scale"]
    assert np.array_equal(O.lora_down(X, A), np.array(g["intermediates"]["T"]))
    assert np.array_equal(O.lora_forward(X, W, A, B, alpha), np.array(g["Y"]))
    dX, dA, dB = O.lora_backward(X, W, A, B, dY, alpha)
    assert np.array_equal(dX, np.array(g["dX"]))
    assert np.array_equal(dA, np.array(g["dA"]))
    assert np.array_equal(dB, np.array(g["dB"]))
    assert np.array_equal(O.lora_merge(W, A, B, alpha), np.array(g["W_merged"]))


# ----------------------------------------------------------- forward ------

def brute_forward_merged_form(X, W, A, B, s):
    """Y[m][n] = sum_k X[m][k] * (W[n][k] + s * sum_j B[n][j] * A[j][k]).

    The merged association: a different order of operations than the oracle's
    base + scaled up-projection; equal by distributivity."""
    M, d_in = len(X), len(X[0])
    d_out, r = len(B), len(B[0])
    Y = [[0.0] * d_out for _ in range(M)]
    for m in range(M):
        for n in range(d_out):
            acc = 0.0
            for k in range(d_in):
                w = W[n][k]
                for j in range(r):
                    w += s * B[n][j] * A[j][k]
                acc += X[m][k] * w
            Y[m][n] = acc
    return np.array(Y)


@pytest.mark.parametrize("M,d,r", list(itertools.product([1, 3, 17], [8, 24], [1, 2, 8])))
def test_forward_brute_force(M, d, r):
    d_out = d + 8  # non-square, so a transposed W or B cannot pass
    X, W, A, B, _ = rng_mats(M * 1000 + d * 10 + r, M, d, d_out, r)
    alpha = 0.75 * r                       # scale 0.75, not a power of two
    Y = O.lora_forward(X, W, A, B, alpha)
    Yb = brute_forward_merged_form(X.tolist(), W.tolist(), A.tolist(), B.tolist(), alpha / r)
    assert Y.shape == (M, d_out)
    np.testing.assert_allclose(Y, Yb, rtol=1e-12, atol=1e-12 * np.abs(Yb).max())


def test_forward_rows_subset_is_same_definition():
    X, W, A, B, _ = rng_mats(1, 40, 16, 24, 4)
    rows = [0, 7, 39]
    full = O.lora_forward(X, W, A, B, 8.0)
    np.testing.assert_array_equal(O.lora_forward(X, W, A, B, 8.0, rows=rows), full[rows])


def test_forward_identity_input_gives_transposed_merged_weight():
    # Closed form: X = I (M = d_in)  =>  Y = (W + s B A)^T.
    d_in, d_out, r = 12, 20, 3
    _, W, A, B, _ = rng_mats(5, 1, d_in, d_out, r)
    s = 1.25
    Y = O.lora_forward(np.eye(d_in), W, A, B, s * r)
    expect = np.zeros((d_in, d_out))
    for m in range(d_in):
        for n in range(d_out):
            expect[m, n] = W[n, m] + s * sum(B[n, j] * A[j, m] for j in range(r))
    np.testing.assert_allclose(Y, expect, rtol=1e-13, atol=1e-13)


def test_forward_zero_adapter_is_exactly_base():
    X, W, A, B, _ = rng_mats(2, 9, 16, 8, 4)
    base = np.zeros((9, 8))
    for m in range(9):
        for n in range(8):
            base[m, n] = sum(X[m, k] * W[n, k] for k in range(16))
    for A_, B_ in ((A, np.zeros_like(B)), (np.zeros_like(A), B)):
        Y = O.lora_forward(X, W, A_, B_, 8.0)
        np.testing.assert_array_equal(Y, X @ W.T)   # adapter adds exactly 0
        np.testing.assert_allclose(Y, base, rtol=1e-13, atol=1e-13)


def test_degenerate_identity_A_reduces_to_one_gemm():
    # d_in = r and A = I  =>  T = X  =>  Y = X (W + s B)^T, one textbook GEMM.
    M, r, d_out = 7, 8, 12
    X, W, _, B, _ = rng_mats(11, M, r, d_out, r)
    s = 0.5
    Y = O.lora_forward(X, W, np.eye(r), B, s * r)
    Wm = (W + s * B).tolist()
    expect = [[sum(X[m, k] * Wm[n][k] for k in range(r)) for n in range(d_out)] for m in range(M)]
    np.testing.assert_allclose(Y, np.array(expect), rtol=1e-13, atol=1e-13)


def test_bf16_inputs_widen_exactly():
    t = WL.make_layer_inputs(WL.LayerShape(4, 8, 8, 2, 4.0), seed=0)
    bits = WL.bf16_bits(t["X"])
    np.testing.assert_array_equal(O.bf16_bits_to_f64(bits), t["X"].double().numpy())


# ---------------------------------------------------------- backward ------

def _loss(X, W, A, B, dY, alpha):
    return float(np.sum(dY * O.lora_forward(X, W, A, B, alpha)))


@pytest.mark.parametrize("M,d_in,d_out,r", [(3, 5, 4, 2), (6, 8, 10, 3)])
def test_backward_finite_differences_exact_for_linear_arguments(M, d_in, d_out, r):
    # L = <dY, Y> is linear in X, and linear in A and in B separately, so a
    # central difference with h = 1 is exact up to rounding at every entry.
    X, W, A, B, dY = rng_mats(M + d_in, M, d_in, d_out, r)
    alpha = 0.6 * r
    dX, dA, dB = O.lora_backward(X, W, A, B, dY, alpha)
    for name, P, G in (("X", X, dX), ("A", A, dA), ("B", B, dB)):
        fd = np.zeros_like(P)
        for idx in np.ndindex(P.shape):
            Pp, Pm = P.copy(), P.copy()
            Pp[idx] += 1.0
            Pm[idx] -= 1.0
            args = dict(X=X, A=A, B=B)
            args[name] = Pp
            lp = _loss(args["X"], W, args["A"], args["B"], dY, alpha)
            args[name] = Pm
            lm = _loss(args["X"], W, args["A"], args["B"], dY, alpha)
            fd[idx] = (lp - lm) / 2.0
        np.testing.assert_allclose(G, fd, rtol=1e-10, atol=1e-10, err_msg=name)


def test_backward_hand_loops_for_dT_route():
    # dB[n][j] = s sum_m dY[m][n] T[m][j];  dA[j][k] = sum_m dT[m][j] X[m][k]
    M, d_in, d_out, r = 5, 6, 7, 2
    X, W, A, B, dY = rng_mats(21, M, d_in, d_out, r)
    s = 1.5
    dX, dA, dB = O.lora_backward(X, W, A, B, dY, s * r)
    T = [[sum(X[m, k] * A[j, k] for k in range(d_in)) for j in range(r)] for m in range(M)]
    dT = [[s * sum(dY[m, n] * B[n, j] for n in range(d_out)) for j in range(r)] for m in range(M)]
    dB_l = [[s * sum(dY[m, n] * T[m][j] for m in range(M)) for j in range(r)] for n in range(d_out)]
    dA_l = [[sum(dT[m][j] * X[m, k] for m in range(M)) for k in range(d_in)] for j in range(r)]
    dX_l = [[sum(dY[m, n] * W[n, k] for n in range(d_out)) + sum(dT[m][j] * A[j, k] for j in range(r))
             for k in range(d_in)] for m in range(M)]
    np.testing.assert_allclose(dB, np.array(dB_l), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dA, np.array(dA_l), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dX, np.array(dX_l), rtol=1e-12, atol=1e-12)


def test_backward_zero_B_invariants():
    X, W, A, B, dY = rng_mats(4, 6, 8, 5, 3)
    dX, dA, dB = O.lora_backward(X, W, A, np.zeros_like(B), dY, 6.0)
    assert not np.any(dA)                          # dT = 0  =>  dA = 0 exactly
    np.testing.assert_array_equal(dX, dY @ W)      # dX = dY W exactly
    assert np.any(dB)                              # dB still sees T


def test_backward_dx_rows_subset():
    X, W, A, B, dY = rng_mats(8, 30, 8, 6, 2)
    full = O.lora_backward(X, W, A, B, dY, 4.0)
    part = O.lora_backward(X, W, A, B, dY, 4.0, dx_rows=[1, 29])
    np.testing.assert_array_equal(part[0], full[0][[1, 29]])
    np.testing.assert_array_equal(part[1], full[1])
    np.testing.assert_array_equal(part[2], full[2])


# ------------------------------------------------------------- merge ------

def test_merge_brute_force_and_merged_equals_unmerged():
    X, W, A, B, _ = rng_mats(9, 11, 10, 14, 4)
    alpha = 3.0
    s = alpha / 4
    Wm = O.lora_merge(W, A, B, alpha)
    loops = [[W[n, k] + s * sum(B[n, j] * A[j, k] for j in range(4)) for k in range(10)] for n in range(14)]
    np.testing.assert_allclose(Wm, np.array(loops), rtol=1e-13, atol=1e-13)
    # merged forward == unmerged forward (exact arithmetic, fp64 rounding only)
    np.testing.assert_allclose(X @ Wm.T, O.lora_forward(X, W, A, B, alpha), rtol=1e-12, atol=1e-12)


def test_merge_zero_B_is_bitwise_identity_on_bf16_weights():
    t = WL.make_merge_inputs(64, 48, 8, seed=3)
    Wb = WL.bf16_bits(t["W"])
    W = O.bf16_bits_to_f64(Wb)
    out = O.lora_merge_bf16(W, O.bf16_bits_to_f64(WL.bf16_bits(t["A"])), np.zeros((64, 8)), 16.0)
    assert np.array_equal(O.f64_to_bf16_bits(out), Wb)


def _hash(bits):
    return hashlib.sha256(np.ascontiguousarray(bits).tobytes()).hexdigest()


def test_restore_merge_cycles_bit_identical_and_unmerge_drifts():
    """Ten perturb + restore + merge cycles leave the pristine copy unchanged
    and make each merged state a pure function of (pristine, A, B); the bf16
    merge/unmerge protocol (negative control) drifts after one cycle."""
    d_out, d_in, r, alpha = 96, 80, 32, 64.0
    t = WL.make_merge_inputs(d_out, d_in, r, seed=5)
    pristine_bits = WL.bf16_bits(t["W"]).copy()
    h0 = _hash(pristine_bits)
    pristine = O.bf16_bits_to_f64(pristine_bits)
    A, B = t["A"], t["B"]
    merged_history = []
    for cycle in range(10):
        A, B = WL.perturb_adapter(A, B, cycle)
        Af, Bf = O.bf16_bits_to_f64(WL.bf16_bits(A)), O.bf16_bits_to_f64(WL.bf16_bits(B))
        restored, merged = O.restore_and_merge_bf16(pristine, Af, Bf, alpha)
        assert np.array_equal(O.f64_to_bf16_bits(restored), pristine_bits)
        _, merged_again = O.restore_and_merge_bf16(pristine, Af, Bf, alpha)
        assert np.array_equal(merged, merged_again)
        merged_history.append(merged)
    assert _hash(pristine_bits) == h0
    assert np.array_equal(O.f64_to_bf16_bits(pristine), pristine_bits)

    # negative control: merge then unmerge in bf16 does not give W back
    W = pristine
    drifted = 0
    for cycle in range(10):
        A2, B2 = WL.perturb_adapter(t["A"], t["B"], cycle)
        merged, back = O.peft_merge_unmerge_bf16(W, O.bf16_bits_to_f64(WL.bf16_bits(A2)),
                                                 O.bf16_bits_to_f64(WL.bf16_bits(B2)), alpha)
        # each cycle leaks at most one rounding of the merged value and one
        # of the restored value: ULP-sized, but of the merged magnitude
        assert np.all(np.abs(back - W) <= O.ulp_bf16(merged) + O.ulp_bf16(back))
        W = back
        drifted = int(np.sum(W != pristine))
        if cycle == 0:
            assert drifted > 0
    assert drifted > 0


# ---------------------------------------------------------- tolerance ------

def test_tolerance_sees_the_adapter_on_tiny_workload():
    """On the tiny forward workload, the bf16-output tolerance accepts the
    GPU's documented roundings (s*T rounded to bf16, Y rounded to bf16) but
    rejects a dropped adapter term and a halved scale."""
    sh = WL.TINY_FWD
    t = WL.make_layer_inputs(sh, seed=0)
    X, W, A, B = (O.bf16_bits_to_f64(WL.bf16_bits(t[k])) for k in "XWAB")
    s = sh.alpha / sh.r
    ref = O.lora_forward(X, W, A, B, sh.alpha)
    emul = O.bf16_round(X @ W.T + O.bf16_round(s * (X @ A.T)) @ B.T)
    ok, info = lora_tol_check(emul, ref)
    assert ok, info
    ok, _ = lora_tol_check(O.bf16_round(X @ W.T), ref)
    assert not ok
    ok, _ = lora_tol_check(O.bf16_round(X @ W.T + 0.5 * s * (X @ A.T) @ B.T), ref)
    assert not ok
    ok, _ = lora_tol_check(O.bf16_round(X @ W.T + s * (X @ A.T) @ (B.T[::-1])), ref)
    assert not ok                                   # permuted B rows


def test_merge_tolerance_accepts_single_rounding_rejects_double():
    t = WL.make_merge_inputs(128, 96, 32, seed=7)
    W, A, B = (O.bf16_bits_to_f64(WL.bf16_bits(t[k])) for k in "WAB")
    s = 2.0
    exact = O.lora_merge(W, A, B, 64.0)
    ok, info = merge_tol_check(O.bf16_round(exact), exact, W, A, B, s)
    assert ok and info["max_err_in_ulps"] <= 0.5 and info["max_ulps_noncancel"] <= 0.5
    # PEFT-style fp32 delta rounded to bf16 first, then added and rounded:
    # still close, but a wrong scale is not.
    ok, _ = merge_tol_check(O.bf16_round(W + 0.5 * s * (B @ A)), exact, W, A, B, s)
    assert not ok
