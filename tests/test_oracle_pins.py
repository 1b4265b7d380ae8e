"""Pins of the fp64 oracle against facts the pages print and the mathematics fixes.

Each test drives the oracle's sequential scan (or decode step) through a worked example
whose answer does not come from the oracle: the printed numbers of the pages (fixtures
under tests/golden/, each with its citation), closed forms, and independent
implementations (a Hillis-Steele scan over affine pairs, the O(L^2) convolution of a
time-invariant SSM).  The set is chosen so that a dropped term, a wrong sign, a wrong
index or a transposed operand in the oracle fails at least one of them.
"""
import math

import numpy as np
import pytest

import oracle
from tests.conftest import load_golden


def _printed(value, decimals):
    """Tolerance of a number printed with ``decimals`` digits after the point."""
    return 0.5 * 10.0 ** (-decimals) + 1e-12


def _one_state(abar_list, gain_list, x_list, c=1.0, h0=None, zoh=False):
    """Run the oracle scan on one channel with one state.

    The decay Abar_t and the Euler gain Bbar_t are planted through Delta_t and B_t:
    A = -1, Delta_t = -ln(Abar_t), B_t = Bbar_t / Delta_t (so Delta_t B_t = Bbar_t).
    """
    abar = np.asarray(abar_list, dtype=np.float64)
    L = len(x_list)
    delta = -np.log(abar) * np.ones(L)
    B = (np.asarray(gain_list, dtype=np.float64) * np.ones(L)) / delta
    y, hN = oracle.scan(
        x=np.asarray(x_list, dtype=np.float64).reshape(1, 1, L),
        delta=delta.reshape(1, 1, L),
        A=np.array([[-1.0]]),
        B=B.reshape(1, L, 1),
        C=(c * np.ones(L)).reshape(1, L, 1),
        h0=None if h0 is None else np.array(h0, dtype=np.float64).reshape(1, 1, 1),
        zoh_exact=zoh,
    )
    return y[0, 0], hN[0, 0]


def test_toy_recurrence_printed_states():
    g = load_golden("toy_recurrence.json")
    y, _ = _one_state([g["Abar"]] * 4, [g["Bbar"]] * 4, g["x"])
    tol = _printed(None, g["printed_decimals"])
    np.testing.assert_allclose(y, g["h_printed"], atol=tol, rtol=0)
    # the last state, unrounded: 0.8^3 * 1 + 0.2 * 10
    assert abs(y[3] - 2.512) < 1e-12


def test_impulse_response_halves():
    g = load_golden("impulse_response.json")
    y, _ = _one_state([g["Abar"]] * 5, [g["Bbar"]] * 5, g["x"], c=g["C"])
    np.testing.assert_allclose(y, g["y_printed"], atol=_printed(None, g["printed_decimals"]))
    np.testing.assert_allclose(y, [0.5 ** t for t in range(5)], rtol=1e-13)


def test_zoh_decay_percentages():
    g = load_golden("zoh_decay.json")
    for case in g["cases"]:
        # state 1, no input: one step leaves Abar = exp(Delta * A) of it
        y, hN = oracle.scan(x=np.zeros((1, 1, 1)), delta=np.full((1, 1, 1), case["delta"]),
                            A=np.array([[g["A"]]]), B=np.ones((1, 1, 1)), C=np.ones((1, 1, 1)),
                            h0=np.ones((1, 1, 1)))
        kept = 100.0 * hN[0, 0, 0]
        assert abs(kept - case["kept_percent_printed"]) <= 0.5, (case, kept)
        # the sign of A matters: exp(+Delta) would keep more than everything
        assert hN[0, 0, 0] < 1.0


def test_discretize_exact_zoh_printed():
    g = load_golden("discretize_zoh.json")
    N = len(g["A"])
    A = np.array(g["A"]).reshape(1, N)
    tol = _printed(None, g["printed_decimals"])
    # Abar: start from h = 1 with no input, one step
    _, hA = oracle.scan(x=np.zeros((1, 1, 1)), delta=np.full((1, 1, 1), g["delta"]), A=A,
                        B=np.array(g["B"]).reshape(1, 1, N), C=np.zeros((1, 1, N)),
                        h0=np.ones((1, 1, N)), zoh_exact=True)
    np.testing.assert_allclose(hA[0, 0], g["Abar_printed"], atol=tol)
    # Bbar: start from h = 0, input x = 1, one step (exact-ZOH gain mode)
    _, hB = oracle.scan(x=np.ones((1, 1, 1)), delta=np.full((1, 1, 1), g["delta"]), A=A,
                        B=np.array(g["B"]).reshape(1, 1, N), C=np.zeros((1, 1, N)),
                        zoh_exact=True)
    np.testing.assert_allclose(hB[0, 0], g["Bbar_printed"], atol=tol)


def test_exact_over_euler_ratio_table():
    g = load_golden("euler_ratio.json")
    tol = _printed(None, g["printed_decimals"])
    for p, printed in zip(g["p"], g["ratio_printed"]):
        kw = dict(x=np.ones((1, 1, 1)), delta=np.full((1, 1, 1), p), A=np.array([[-1.0]]),
                  B=np.ones((1, 1, 1)), C=np.ones((1, 1, 1)))
        _, h_exact = oracle.scan(zoh_exact=True, **kw)
        _, h_euler = oracle.scan(zoh_exact=False, **kw)
        assert abs(h_euler[0, 0, 0] - p) < 1e-15          # Euler gain is Delta * B
        ratio = h_exact[0, 0, 0] / h_euler[0, 0, 0]
        assert abs(ratio - printed) <= tol, (p, ratio, printed)


def test_affine_scan_printed_by_all_three_routes():
    g = load_golden("affine_scan.json")
    tol = _printed(None, g["printed_decimals"])
    loop = oracle.affine_scan_loop(g["a"], g["b"])
    par = oracle.affine_scan_hillis_steele(g["a"], g["b"])
    np.testing.assert_allclose(loop, g["h_printed"], atol=tol)
    np.testing.assert_allclose(par, g["h_printed"], atol=tol)
    # the C loop, with a_t planted as the decay and b_t as the Euler gain at x = 1
    y, _ = _one_state(g["a"], g["b"], [1.0] * len(g["a"]))
    np.testing.assert_allclose(y, loop, rtol=1e-13, atol=1e-15)


def test_selectivity_toy_percentages():
    g = load_golden("selectivity_toy.json")
    A = np.array([[g["A"]]])

    def survives(deltas):
        # key value 1 at t = 0, fillers carry no input; the last state is what is left of it
        L = len(deltas)
        x = np.zeros((1, 1, L))
        x[0, 0, 0] = 1.0
        _, hN = oracle.scan(x=x, delta=np.array(deltas).reshape(1, 1, L), A=A,
                            B=np.ones((1, L, 1)), C=np.ones((1, L, 1)), zoh_exact=True)
        return 100.0 * hN[0, 0, 0]

    s = g["selective"]
    sel = survives([s["key_delta"]] + [s["filler_delta"]] * s["fillers"])
    assert abs(sel - s["survives_percent_printed"]) <= 0.5, sel
    f = g["fixed"]
    fixed = survives([f["delta"]] * (1 + f["fillers"]))
    assert abs(fixed - f["survives_percent_printed"]) <= 0.05, fixed


def test_lti_kernel_taps_torch_seed0_soft_pin():
    torch = pytest.importorskip("torch")
    g = load_golden("lti_taps.json")
    torch.manual_seed(g["seed"])
    abar = (torch.rand(4) * 0.9 + 0.05).double().numpy()
    bbar = torch.randn(4).double().numpy()
    c = torch.randn(4).double().numpy()
    taps = oracle.lti_kernel(abar, bbar, c, 4)
    np.testing.assert_allclose(taps, g["taps_printed"], atol=_printed(None, g["printed_decimals"]))


def test_recurrence_equals_causal_convolution_when_time_invariant():
    # Delta, B, C fixed over t: the scan is the convolution with K = (C Bbar, C Abar Bbar, ...)
    rng = np.random.default_rng(1)
    N, L = 5, 23
    A = -rng.uniform(0.2, 3.0, size=(1, N))
    delta0 = 0.37
    Bv = rng.normal(size=N)
    Cv = rng.normal(size=N)
    x = rng.normal(size=L)
    y, _ = oracle.scan(x=x.reshape(1, 1, L), delta=np.full((1, 1, L), delta0), A=A,
                       B=np.tile(Bv, (L, 1)).reshape(1, L, N), C=np.tile(Cv, (L, 1)).reshape(1, L, N))
    y_conv = oracle.lti_conv(np.exp(delta0 * A[0]), delta0 * Bv, Cv, x)
    np.testing.assert_allclose(y[0, 0], y_conv, rtol=1e-11, atol=1e-12)


def _random_case(rng, batch=2, dim=3, L=37, N=4):
    return dict(
        x=rng.normal(size=(batch, dim, L)),
        delta=0.5 * rng.normal(size=(batch, dim, L)),
        z=rng.normal(size=(batch, dim, L)),
        B=rng.normal(size=(batch, L, N)),
        C=rng.normal(size=(batch, L, N)),
        A=-rng.uniform(0.5, 4.0, size=(dim, N)),
        D=rng.normal(size=dim),
        delta_bias=np.log(np.expm1(rng.uniform(1e-3, 1e-1, size=dim))),
    )


@pytest.mark.parametrize("shape", [(1, 3, 37, 4), (2, 3, 16, 5), (3, 2, 9, 16)])
def test_loop_equals_bruteforce_parallel_scan(shape):
    batch, dim, L, N = shape
    case = _random_case(np.random.default_rng(sum(shape)), batch, dim, L, N)
    y, hN = oracle.scan(delta_softplus=True, **case)
    y2, h2 = oracle.scan_parallel_reference(delta_softplus=True, **case)
    np.testing.assert_allclose(y, y2, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(hN, h2, rtol=1e-10, atol=1e-12)
    # the distinguishing power of this pin: a transposed B ([b, n, t]) must not agree
    if L != N:
        bad = dict(case)
        bad["B"] = np.ascontiguousarray(case["B"].reshape(batch, N, L).transpose(0, 2, 1))
        yb, _ = oracle.scan(delta_softplus=True, **bad)
        assert np.max(np.abs(yb - y2)) > 1e-3


def test_causality_outputs_before_edit_are_identical():
    rng = np.random.default_rng(7)
    case = _random_case(rng, 2, 3, 40, 4)
    y, _ = oracle.scan(delta_softplus=True, **case)
    t0 = 17
    edited = {k: v.copy() for k, v in case.items()}
    edited["x"][..., t0] += 4.0
    edited["delta"][..., t0] -= 1.0
    edited["z"][..., t0] += 2.0
    edited["B"][:, t0, :] *= -3.0
    edited["C"][:, t0, :] += 1.0
    y2, _ = oracle.scan(delta_softplus=True, **edited)
    assert np.array_equal(y[..., :t0], y2[..., :t0])
    assert not np.array_equal(y[..., t0], y2[..., t0])


def test_skip_and_gate_closed_form():
    # With C = 0 the state contributes nothing: y = D x SiLU(z).  sigmoid(0) = 1/2,
    # sigmoid(ln 3) = 3/4, sigmoid(-ln 3) = 1/4.
    zs = np.array([0.0, math.log(3.0), -math.log(3.0)])
    x = np.array([2.0, 2.0, 2.0])
    L = 3
    y, _ = oracle.scan(x=x.reshape(1, 1, L), delta=np.full((1, 1, L), 0.3), A=np.array([[-1.0]]),
                       B=np.ones((1, L, 1)), C=np.zeros((1, L, 1)), D=np.array([1.5]),
                       z=zs.reshape(1, 1, L))
    expect = 1.5 * x * zs * np.array([0.5, 0.75, 0.25])
    np.testing.assert_allclose(y[0, 0], expect, rtol=1e-14, atol=1e-15)
    # with no gate and no skip the output is the bare readout C h
    y2, h2 = oracle.scan(x=x.reshape(1, 1, L), delta=np.full((1, 1, L), 0.3), A=np.array([[-1.0]]),
                         B=np.ones((1, L, 1)), C=np.full((1, L, 1), 2.0))
    assert abs(y2[0, 0, -1] - 2.0 * h2[0, 0, 0]) < 1e-15


def test_softplus_and_bias_special_values():
    # softplus(0) = ln 2, so with A = -1 one step keeps exp(-ln 2) = 1/2 of the state;
    # softplus(ln 3) = ln 4 keeps 1/4; bias = log(expm1(dt)) gives back Delta = dt.
    def kept(raw, bias):
        _, hN = oracle.scan(x=np.zeros((1, 1, 1)), delta=np.full((1, 1, 1), raw),
                            A=np.array([[-1.0]]), B=np.ones((1, 1, 1)), C=np.ones((1, 1, 1)),
                            delta_bias=np.array([bias]), delta_softplus=True, h0=np.ones((1, 1, 1)))
        return hN[0, 0, 0]

    assert abs(kept(0.0, 0.0) - 0.5) < 1e-15
    assert abs(kept(math.log(3.0), 0.0) - 0.25) < 1e-15
    assert abs(kept(0.25, math.log(3.0) - 0.25) - 0.25) < 1e-14   # bias is added before softplus
    dt = 0.0375
    assert abs(kept(0.0, math.log(math.expm1(dt))) - math.exp(-dt)) < 1e-14
    assert abs(kept(800.0, 0.0)) == 0.0                              # no overflow for large steps


def test_small_step_holds_large_step_resets():
    # Delta -> 0 keeps the state and writes nothing; a large Delta forgets it and
    # writes Bbar x = Delta B x (Euler gain).
    _, h_small = oracle.scan(x=np.full((1, 1, 1), 5.0), delta=np.full((1, 1, 1), 1e-9),
                             A=np.array([[-1.0]]), B=np.ones((1, 1, 1)), C=np.ones((1, 1, 1)),
                             h0=np.full((1, 1, 1), 3.0))
    assert abs(h_small[0, 0, 0] - 3.0) < 1e-8
    _, h_big = oracle.scan(x=np.full((1, 1, 1), 5.0), delta=np.full((1, 1, 1), 60.0),
                           A=np.array([[-1.0]]), B=np.ones((1, 1, 1)), C=np.ones((1, 1, 1)),
                           h0=np.full((1, 1, 1), 3.0))
    assert abs(h_big[0, 0, 0] - 300.0) < 1e-9


def test_decode_step_chaining_equals_scan_from_same_state():
    rng = np.random.default_rng(11)
    batch, dim, L, N = 3, 4, 12, 6
    case = _random_case(rng, batch, dim, L, N)
    h0 = rng.normal(size=(batch, dim, N))
    # the step takes the final Delta: feed the scan the same steps with no bias/softplus
    steps = np.log1p(np.exp(case["delta"] + case["delta_bias"][None, :, None]))
    y, hN = oracle.scan(x=case["x"], delta=steps, A=case["A"], B=case["B"], C=case["C"],
                        D=case["D"], z=case["z"], h0=h0)
    st = h0
    for t in range(L):
        yt, st = oracle.step(st, case["x"][..., t], steps[..., t], case["A"], case["B"][:, t],
                             case["C"][:, t], D=case["D"], z=case["z"][..., t])
        np.testing.assert_allclose(yt, y[..., t], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(st, hN, rtol=1e-13, atol=1e-14)


def test_decode_step_hand_example():
    # one state: h = exp(-0.5 * 2) * 1 + 0.5 * 3 * 2 = e^-1 + 3; y = 0.5 h + 4 * 2 (no gate)
    y, st = oracle.step(np.ones((1, 1, 1)), np.full((1, 1), 2.0), np.full((1, 1), 0.5),
                        np.array([[-2.0]]), np.full((1, 1), 3.0), np.full((1, 1), 0.5),
                        D=np.array([4.0]))
    h = math.exp(-1.0) + 3.0
    assert abs(st[0, 0, 0] - h) < 1e-15
    assert abs(y[0, 0] - (0.5 * h + 8.0)) < 1e-14


def _steps(case):
    return np.log1p(np.exp(case["delta"] + case["delta_bias"][None, :, None]))


def test_end_state_from_zero_is_the_decayed_sum_of_writes():
    # Unrolling h_t = exp(Delta_t A) h_{t-1} + Delta_t B_t x_t ("Module 19", "The Math: The
    # State-Space Recurrence") from h_0 = 0 gives h_L = sum_t exp(A R_t) Delta_t B_t x_t,
    # R_t the sum of the steps after t: evaluated here directly, token by token.
    rng = np.random.default_rng(21)
    batch, dim, L, N = 2, 3, 40, 5
    case = _random_case(rng, batch, dim, L, N)
    steps = _steps(case)
    _, hN = oracle.scan(x=case["x"], delta=steps, A=case["A"], B=case["B"], C=case["C"])
    R = np.cumsum(steps[..., ::-1], axis=-1)[..., ::-1] - steps           # steps after t
    w = steps[..., None] * case["x"][..., None] * case["B"][:, None, :, :]  # [b, d, t, n]
    h = (np.exp(case["A"][None, :, None, :] * R[..., None]) * w).sum(axis=2)
    np.testing.assert_allclose(hN, h, rtol=1e-12, atol=1e-14)


def test_segments_scanned_from_folded_carries_give_the_whole_scan():
    # The affine steps compose ("Module 19", "The Parallel Scan"): a segment maps its carry
    # h to exp(A S) h + h_end, with S its step sum and h_end its end state from zero.
    # Folding the segments in order from the start state gives the carry into each one,
    # and scanning every segment from its carry gives the whole sequence's outputs.
    rng = np.random.default_rng(22)
    batch, dim, L, N = 2, 3, 50, 4
    case = _random_case(rng, batch, dim, L, N)
    steps = _steps(case)
    h0 = rng.normal(size=(batch, dim, N))
    kw = dict(A=case["A"], D=case["D"])
    y_all, h_all = oracle.scan(x=case["x"], delta=steps, B=case["B"], C=case["C"],
                               z=case["z"], h0=h0, **kw)
    h, ys = h0, []
    for a, b in [(0, 13), (13, 29), (29, 50)]:
        seg = dict(x=case["x"][..., a:b], delta=steps[..., a:b], B=case["B"][:, a:b],
                   C=case["C"][:, a:b])
        _, h_end = oracle.scan(**seg, A=case["A"])                        # from zero
        y_seg, h_seg = oracle.scan(**seg, z=case["z"][..., a:b], h0=h, **kw)
        S = steps[..., a:b].sum(axis=-1)
        h = np.exp(case["A"][None] * S[..., None]) * h + h_end
        np.testing.assert_allclose(h, h_seg, rtol=1e-12, atol=1e-13)
        ys.append(y_seg)
    np.testing.assert_allclose(np.concatenate(ys, axis=-1), y_all, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(h, h_all, rtol=1e-12, atol=1e-13)


def test_empty_sequence_keeps_initial_state():
    y, hN = oracle.scan(x=np.zeros((2, 3, 0)), delta=np.zeros((2, 3, 0)), A=-np.ones((3, 4)),
                        B=np.zeros((2, 0, 4)), C=np.zeros((2, 0, 4)))
    assert y.shape == (2, 3, 0)
    assert np.all(hN == 0.0)


# ----------------------------------------------------------------------------------
# the causal depthwise convolution in front of the scan (learnllm "Module 19", "The
# Causal Convolution"; xmarva lesson 10, sections 4 and 7)
# ----------------------------------------------------------------------------------

def _conv_case(rng, batch, dim, L, K):
    return (rng.normal(size=(batch, dim, L)), rng.normal(size=(dim, K)) * 0.5,
            rng.normal(size=dim) * 0.1)


@pytest.mark.parametrize("K", [1, 2, 4])
def test_conv_impulse_returns_reversed_taps(K):
    # output t reads x_{t-K+1..t} with tap i on x_{t-K+1+i}: a spike at t = 0 shows the
    # taps last-first, then only the bias is left
    w = np.arange(1, K + 1, dtype=np.float64).reshape(1, K) * 0.25
    L = K + 3
    x = np.zeros((1, 1, L))
    x[0, 0, 0] = 1.0
    u, _ = oracle.causal_conv1d(x, w, bias=np.array([0.125]), silu=False)
    expect = np.full(L, 0.125)
    expect[:K] += w[0, ::-1]
    np.testing.assert_array_equal(u[0, 0], expect)


def test_conv_first_token_sees_only_its_own_tap():
    rng = np.random.default_rng(3)
    x, w, b = _conv_case(rng, 2, 3, 6, 4)
    u, _ = oracle.causal_conv1d(x, w, bias=b, silu=False)
    np.testing.assert_allclose(u[..., 0], b[None, :] + w[None, :, 3] * x[..., 0], rtol=1e-15)


def test_conv_equals_textbook_full_convolution_cropped():
    rng = np.random.default_rng(5)
    x, w, b = _conv_case(rng, 2, 5, 23, 4)
    u, win = oracle.causal_conv1d(x, w, bias=b, silu=False)
    for bi in range(2):
        for d in range(5):
            full = np.convolve(x[bi, d], w[d, ::-1])       # true convolution, length L + K - 1
            np.testing.assert_allclose(u[bi, d], full[:23] + b[d], rtol=1e-13, atol=1e-14)
    np.testing.assert_array_equal(win, x[..., -3:])


def test_conv_equals_torch_grouped_conv1d_left_padded():
    # the block's own formulation: nn.Conv1d(groups=d_inner, padding=k-1), cropped to L
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(9)
    x, w, b = _conv_case(rng, 3, 6, 17, 4)
    u, _ = oracle.causal_conv1d(x, w, bias=b, silu=True)
    ref = torch.nn.functional.conv1d(torch.from_numpy(x), torch.from_numpy(w)[:, None, :],
                                     torch.from_numpy(b), padding=3, groups=6)[..., :17]
    ref = torch.nn.functional.silu(ref).numpy()
    np.testing.assert_allclose(u, ref, rtol=1e-13, atol=1e-14)


def test_conv_silu_closed_values():
    # pre-activations 0, ln 3, -ln 3 through a single unit tap: SiLU v = v sigmoid(v)
    v = np.array([0.0, math.log(3.0), -math.log(3.0)])
    u, _ = oracle.causal_conv1d(v.reshape(1, 1, 3), np.array([[0.0, 1.0]]), silu=True)
    np.testing.assert_allclose(u[0, 0], v * np.array([0.5, 0.75, 0.25]), rtol=1e-15, atol=0)


def test_conv_is_causal_and_depthwise():
    rng = np.random.default_rng(13)
    x, w, b = _conv_case(rng, 2, 4, 30, 4)
    u, _ = oracle.causal_conv1d(x, w, bias=b)
    t0 = 11
    x2 = x.copy()
    x2[:, 1, t0] += 3.0
    u2, _ = oracle.causal_conv1d(x2, w, bias=b)
    assert np.array_equal(u2[..., :t0], u[..., :t0])           # nothing before the edit moves
    assert np.array_equal(u2[:, [0, 2, 3]], u[:, [0, 2, 3]])   # other channels never mix in
    assert not np.array_equal(u2[:, 1, t0:t0 + 4], u[:, 1, t0:t0 + 4])
    assert np.array_equal(u2[:, 1, t0 + 4:], u[:, 1, t0 + 4:])  # the edit leaves after K taps


@pytest.mark.parametrize("split", [0, 1, 2, 9, 20])
def test_conv_resumes_from_carried_window(split):
    rng = np.random.default_rng(17)
    x, w, b = _conv_case(rng, 2, 3, 20, 4)
    u, win = oracle.causal_conv1d(x, w, bias=b)
    u1, w1 = oracle.causal_conv1d(x[..., :split], w, bias=b)
    u2, w2 = oracle.causal_conv1d(x[..., split:], w, bias=b, hist=w1)
    np.testing.assert_array_equal(np.concatenate([u1, u2], axis=-1), u)
    np.testing.assert_array_equal(w2, win)


def test_conv_decode_steps_chain_to_the_full_convolution():
    rng = np.random.default_rng(19)
    x, w, b = _conv_case(rng, 2, 5, 13, 4)
    hist = rng.normal(size=(2, 5, 3))
    u, win = oracle.causal_conv1d(x, w, bias=b, hist=hist)
    state = hist
    for t in range(13):
        ut, state = oracle.conv1d_step(state, x[..., t], w, bias=b)
        np.testing.assert_allclose(ut, u[..., t], rtol=1e-14, atol=1e-15)
    np.testing.assert_array_equal(state, win)


def test_conv_width_one_is_pointwise():
    rng = np.random.default_rng(23)
    x, w, b = _conv_case(rng, 1, 3, 5, 1)
    u, win = oracle.causal_conv1d(x, w, bias=b, silu=False)
    np.testing.assert_allclose(u, w[None, :, :1] * x + b[None, :, None], rtol=1e-15)
    assert win.shape == (1, 3, 0)


# ----------------------------------------------------------------------------------
# backward of the scan (xmarva lesson 10, section 6: the training half recomputes the
# states): pinned by central finite differences of the forward oracle and closed forms
# ----------------------------------------------------------------------------------

def _bwd_case(rng, batch, dim, L, N, softplus=True):
    case = _random_case(rng, batch, dim, L, N)
    case["h0"] = rng.normal(size=(batch, dim, N))
    if not softplus:
        case["delta"] = np.abs(case["delta"]) * 0.5 + 0.05     # positive steps as given
        case["delta_bias"] = np.abs(case["delta_bias"]) * 0.1
    return case


def _loss(case, dy, dfinal, softplus):
    y, hN = oracle.scan(delta_softplus=softplus, **case)
    return float(np.sum(dy * y) + np.sum(dfinal * hN))


@pytest.mark.parametrize("softplus", [True, False])
def test_scan_bwd_matches_central_differences(softplus):
    rng = np.random.default_rng(29 + softplus)
    batch, dim, L, N = 2, 3, 6, 4
    case = _bwd_case(rng, batch, dim, L, N, softplus)
    dy = rng.normal(size=(batch, dim, L))
    dfinal = rng.normal(size=(batch, dim, N))
    g = oracle.scan_bwd(dy, delta_softplus=softplus, dfinal=dfinal, **case)
    names = dict(x="dx", delta="ddelta", z="dz", A="dA", B="dB", C="dC", D="dD",
                 delta_bias="ddelta_bias", h0="dh0")
    eps = 1e-6
    for key, gname in names.items():
        base = case[key]
        fd = np.empty_like(base)
        for idx in np.ndindex(base.shape):
            plus = {k: v.copy() for k, v in case.items()}
            minus = {k: v.copy() for k, v in case.items()}
            plus[key][idx] += eps
            minus[key][idx] -= eps
            fd[idx] = (_loss(plus, dy, dfinal, softplus) - _loss(minus, dy, dfinal, softplus)) / (2 * eps)
        np.testing.assert_allclose(g[gname], fd, rtol=1e-6, atol=1e-7, err_msg=gname)


def test_scan_bwd_no_decay_closed_form():
    # A = 0: h_t = sum_{s<=t} Delta_s B_s x_s (a running sum).  Loss = y_{L-1} alone, so
    # every earlier token reaches it with weight C_{L-1}.
    rng = np.random.default_rng(31)
    L = 5
    x, step, B, C = (rng.normal(size=L), rng.uniform(0.1, 0.9, size=L), rng.normal(size=L),
                     rng.normal(size=L))
    dy = np.zeros((1, 1, L))
    dy[0, 0, -1] = 1.0
    g = oracle.scan_bwd(dy, x.reshape(1, 1, L), step.reshape(1, 1, L), np.zeros((1, 1)),
                        B.reshape(1, L, 1), C.reshape(1, L, 1))
    cL = C[-1]
    np.testing.assert_allclose(g["dx"][0, 0], cL * step * B, rtol=1e-14)
    np.testing.assert_allclose(g["ddelta"][0, 0], cL * B * x, rtol=1e-14)
    np.testing.assert_allclose(g["dB"][0, :, 0], cL * step * x, rtol=1e-14)
    h = np.cumsum(step * B * x)
    expect_dC = np.zeros(L)
    expect_dC[-1] = h[-1]
    np.testing.assert_allclose(g["dC"][0, :, 0], expect_dC, rtol=1e-14, atol=0)
    hprev = np.concatenate([[0.0], h[:-1]])
    np.testing.assert_allclose(g["dA"][0, 0], cL * np.sum(hprev * step), rtol=1e-13)


def test_scan_bwd_initial_state_gradient_is_the_decay_product():
    # one state, loss = y_{L-1}: dh0 = C_{L-1} prod_t exp(Delta_t a)
    rng = np.random.default_rng(37)
    L, a = 6, -0.7
    step = rng.uniform(0.05, 0.5, size=L)
    C = rng.normal(size=L)
    dy = np.zeros((1, 1, L))
    dy[0, 0, -1] = 1.0
    g = oracle.scan_bwd(dy, rng.normal(size=(1, 1, L)), step.reshape(1, 1, L), np.array([[a]]),
                        rng.normal(size=(1, L, 1)), C.reshape(1, L, 1), h0=np.ones((1, 1, 1)))
    assert abs(g["dh0"][0, 0, 0] - C[-1] * math.exp(a * step.sum())) < 1e-14


def test_scan_bwd_gate_and_skip_closed_form():
    # C = 0, D = 1: y = x SiLU(z); SiLU'(0) = 1/2, SiLU'(z) = s (1 + z (1 - s))
    zs = np.array([0.0, math.log(3.0), -math.log(3.0)])
    x = np.array([2.0, -1.0, 0.5])
    dy = np.array([1.0, 2.0, -1.0])
    L = 3
    g = oracle.scan_bwd(dy.reshape(1, 1, L), x.reshape(1, 1, L), np.full((1, 1, L), 0.3),
                        np.array([[-1.0]]), np.ones((1, L, 1)), np.zeros((1, L, 1)),
                        D=np.array([1.0]), z=zs.reshape(1, 1, L))
    s = np.array([0.5, 0.75, 0.25])
    np.testing.assert_allclose(g["dz"][0, 0], dy * x * s * (1 + zs * (1 - s)), rtol=1e-14)
    assert abs(g["dz"][0, 0, 0] - 0.5 * dy[0] * x[0]) < 1e-15
    # the state never reaches y, so x's gradient is the skip's alone
    np.testing.assert_allclose(g["dx"][0, 0], dy * zs * s, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(g["dD"], [np.sum(dy * zs * s * x)], rtol=1e-14)


# ----------------------------------------------------------------------------------
# Mamba-2 SSD (xmarva lesson 10, section 8): the loop, the chunked form, the attention form
# ----------------------------------------------------------------------------------

def _ssd_case(rng, batch=1, L=150, heads=3, P=8, N=16):
    return (rng.normal(size=(batch, L, heads, P)), -rng.random((batch, L, heads)) * 0.3,
            rng.normal(size=(batch, L, heads, N)), rng.normal(size=(batch, L, heads, N)))


def test_ssd_loop_equals_the_printed_attention_form():
    # y_t = sum_{s<=t} (c_t . b_s) exp(a_{s+1} + ... + a_t) x_s, summed term by term
    rng = np.random.default_rng(41)
    x, a, b, c = _ssd_case(rng, batch=2, L=9, heads=2, P=3, N=4)
    y, _ = oracle.ssd_loop(x, a, b, c)
    brute = np.zeros_like(y)
    for bi in range(2):
        for h in range(2):
            for t in range(9):
                for s in range(t + 1):
                    w = np.dot(c[bi, t, h], b[bi, s, h]) * math.exp(a[bi, s + 1:t + 1, h].sum())
                    brute[bi, t, h] += w * x[bi, s, h]
    np.testing.assert_allclose(y, brute, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("chunk", [16, 32, 64, 150, 256])
def test_ssd_chunked_equals_loop(chunk):
    rng = np.random.default_rng(43)
    x, a, b, c = _ssd_case(rng)
    y, hN = oracle.ssd_loop(x, a, b, c)
    yc, hc = oracle.ssd_chunked(x, a, b, c, chunk=chunk)
    np.testing.assert_allclose(yc, y, rtol=0, atol=1e-11)
    np.testing.assert_allclose(hc, hN, rtol=0, atol=1e-11)


def test_ssd_chunked_fp32_difference_is_of_the_printed_order():
    g = load_golden("ssd_chunk_vs_loop.json")
    rng = np.random.default_rng(47)
    x, a, b, c = (v.astype(np.float32) for v in _ssd_case(rng))
    y, _ = oracle.ssd_loop(x, a, b, c)                      # fp64 of the fp32 inputs
    # the chunked form evaluated in single precision throughout
    y32, _ = oracle.ssd_chunked(x, a, b, c, chunk=g["chunk"], dtype=np.float32)
    diff = float(np.abs(y32 - y).max())
    assert diff < 10 * g["printed_max_abs_difference_fp32"]
    assert diff > 0.0                                        # single precision does round


def test_ssd_loop_is_the_selective_scan_with_one_decay_per_head():
    # per head: channels p share B, C and the decay; the S6 oracle with Delta_t, A = A_h
    # for every (p, n) and input x / Delta gives the same outputs
    rng = np.random.default_rng(53)
    batch, L, heads, P, N = 2, 12, 2, 3, 5
    step = rng.uniform(0.05, 0.6, size=(batch, L, heads))
    A_h = -rng.uniform(0.2, 2.0, size=heads)
    u = rng.normal(size=(batch, L, heads, P))
    b = rng.normal(size=(batch, L, heads, N))
    c = rng.normal(size=(batch, L, heads, N))
    y, hN = oracle.ssd_loop(u * step[..., None], step * A_h, b, c)
    for h in range(heads):
        ys, hs = oracle.scan(x=u[:, :, h, :].transpose(0, 2, 1),
                             delta=np.repeat(step[:, None, :, h], P, axis=1),
                             A=np.full((P, N), A_h[h]), B=b[:, :, h, :], C=c[:, :, h, :])
        np.testing.assert_allclose(ys.transpose(0, 2, 1), y[:, :, h, :], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(hs, hN[:, h], rtol=1e-12, atol=1e-13)


def test_ssd_resumes_from_its_final_state():
    rng = np.random.default_rng(59)
    x, a, b, c = _ssd_case(rng, batch=2, L=40, heads=2, P=4, N=6)
    y, hN = oracle.ssd_loop(x, a, b, c)
    y1, h1 = oracle.ssd_loop(x[:, :17], a[:, :17], b[:, :17], c[:, :17])
    y2, h2 = oracle.ssd_loop(x[:, 17:], a[:, 17:], b[:, 17:], c[:, 17:], h0=h1)
    np.testing.assert_allclose(np.concatenate([y1, y2], axis=1), y, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(h2, hN, rtol=1e-13, atol=1e-14)
    yc, hc = oracle.ssd_chunked(x[:, 17:], a[:, 17:], b[:, 17:], c[:, 17:], chunk=8, h0=h1)
    np.testing.assert_allclose(yc, y2, rtol=0, atol=1e-11)
