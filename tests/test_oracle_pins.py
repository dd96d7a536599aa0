"""Pins for the CPU oracle: checks against things other than the oracle itself.

* hand-worked examples under tests/golden/ (closed forms derived from the
  definitions, each file citing the page and section it follows);
* brute force on tiny inputs in plain Python loops (an O(d^2) rank count for
  top-K, triple loops for the projections), independent of the oracle's sort
  and matmul;
* special cases that reduce to textbook results (K = d is the dense layer,
  K = 0 is zero) and invariants that hold at any size.
"""
import itertools
import math

import numpy as np
import pytest

import oracle
import workloads
from conftest import load_golden

# ---------------------------------------------------------------- brute force


def bf_keep(row, k):
    """Kept set by rank counting: i is kept iff fewer than k entries beat it,
    where j beats i when |x_j| > |x_i|, or |x_j| == |x_i| and j < i."""
    d = len(row)
    mags = [abs(float(v)) for v in row]
    kept = []
    for i in range(d):
        beaters = sum(1 for j in range(d)
                      if mags[j] > mags[i] or (mags[j] == mags[i] and j < i))
        if beaters < k:
            kept.append(i)
    return kept


def bf_matvec(xs_row, wt):
    """y_j = sum_i xs_i * wt[i][j] by plain loops."""
    d_in = len(wt)
    d_out = len(wt[0])
    return [sum(float(xs_row[i]) * float(wt[i][j]) for i in range(d_in)) for j in range(d_out)]


# ---------------------------------------------------------------- top-K pins


def test_topk_golden_hand():
    g = load_golden("topk_hand.json")
    for row in g["rows"]:
        x = np.array([row["x"]], dtype=np.float32)
        for k, want in row["keep"].items():
            got = oracle.topk_keep(x, int(k))[0].tolist()
            assert got == want, (row["x"], k)
    r0 = g["rows"][0]
    keep, m, xs = oracle.topk_mask(np.array([r0["x"]], dtype=np.float32), 4)
    assert m[0].tolist() == r0["mask_k4"]
    assert xs[0].tolist() == r0["xs_k4"]


def test_kept_values_golden_hand():
    """The compacted value list is x at the kept indices, in index order and in
    the input's own dtype (hand values in the golden file; -0.0 keeps its sign)."""
    g = load_golden("topk_hand.json")
    r0, r2 = g["rows"][0], g["rows"][2]
    x0 = np.array([r0["x"]], dtype=np.float32)
    v0 = oracle.kept_values(x0, oracle.topk_keep(x0, 4))
    assert v0.dtype == np.float32 and v0[0].tolist() == r0["vals_k4"]
    x2 = np.array([r2["x"]], dtype=np.float32)
    v2 = oracle.kept_values(x2, oracle.topk_keep(x2, 2))
    assert np.array_equal(np.signbit(v2[0]), np.signbit(np.array(r2["vals_k2"], np.float32)))


@pytest.mark.parametrize("dtype", [np.float32, np.float64, np.int64, np.int8])
def test_kept_values_read_by_loops(dtype):
    """kept_values[t, j] is x[t, keep[t, j]], read here element by element
    (same row, same bits, same dtype) for random keeps of random rows."""
    g = workloads.rng(77)
    x = (g.standard_normal((5, 23)) * 40).astype(dtype)
    for k in (0, 1, 9, 23):
        keep = np.sort(np.stack([g.permutation(23)[:k] for _ in range(5)]), axis=1).astype(np.int64)
        v = oracle.kept_values(x, keep)
        assert v.dtype == x.dtype and v.shape == (5, k)
        for t in range(5):
            for j in range(k):
                assert v[t, j].tobytes() == x[t, keep[t, j]].tobytes()



@pytest.mark.parametrize("seed", range(40))
def test_topk_bruteforce_rank_tiny(seed):
    g = np.random.default_rng(seed)
    d = int(g.integers(1, 13))
    palette = np.array([0.0, -0.0, 0.5, -0.5, 1.0, -1.0, 2.0, -2.0, 3.0], dtype=np.float32)
    if seed % 2:
        row = palette[g.integers(0, palette.size, d)]          # many ties
    else:
        row = g.standard_normal(d).astype(np.float32)           # distinct
    for k in range(d + 1):
        got = oracle.topk_keep(row[None, :], k)[0].tolist()
        assert got == bf_keep(row, k), (row.tolist(), k)


def test_topk_all_equal_and_signed_zero():
    for d in (1, 5, 33):
        for val in (1.25, -1.25, 0.0):
            row = np.full((1, d), val, dtype=np.float32)
            if val == 0.0:
                row[0, ::2] = -0.0
            for k in (0, 1, d // 2, d):
                assert oracle.topk_keep(row, k)[0].tolist() == list(range(k))


def test_topk_rejects_bad_k():
    x = np.zeros((1, 4), np.float32)
    for k in (-1, 5):
        with pytest.raises(ValueError):
            oracle.topk_keep(x, k)


@pytest.mark.parametrize("d,k", [(4096, 2867), (11008, 7705), (4096, 1)])
def test_topk_invariants_config_sizes(d, k):
    x = workloads.normal_f32(workloads.rng(d + k), (3, d))
    keep, m, xs = oracle.topk_mask(x, k)
    assert keep.shape == (3, k)
    assert np.all(m.sum(axis=1) == k)                       # exactly K selected
    for t in range(3):
        kept = np.abs(x[t, keep[t]])
        dropped = np.abs(x[t, m[t] == 0])
        if dropped.size:
            assert kept.min() >= dropped.max()              # every kept >= every dropped
        assert np.all(np.diff(keep[t]) > 0)                 # ascending, distinct
    assert np.array_equal(xs != 0, m.astype(bool))


# ---------------------------------------------------------------- sparse linear


def test_sparse_linear_golden_hand():
    g = load_golden("sparse_linear_hand.json")
    x = np.array([g["x"]], dtype=np.float32)
    wt = np.array(g["wt"], dtype=np.float32)
    for k, want in g["y"].items():
        assert oracle.sparse_linear(x, wt, int(k))[0].tolist() == want


@pytest.mark.parametrize("seed", range(12))
def test_sparse_linear_bruteforce_nonsquare(seed):
    g = np.random.default_rng(100 + seed)
    T, d_in, d_out = int(g.integers(1, 4)), int(g.integers(1, 9)), int(g.integers(1, 7))
    x = g.standard_normal((T, d_in)).astype(np.float32)
    wt = g.standard_normal((d_in, d_out)).astype(np.float32)
    for k in range(d_in + 1):
        y = oracle.sparse_linear(x, wt, k)
        for t in range(T):
            kept = set(bf_keep(x[t], k))
            xs = [x[t, i] if i in kept else 0.0 for i in range(d_in)]
            ref = bf_matvec(xs, wt.tolist())
            assert np.allclose(y[t], ref, rtol=1e-12, atol=1e-12)


def test_sparse_linear_k_eq_d_is_dense_and_k0_is_zero():
    g = np.random.default_rng(7)
    x = g.standard_normal((2, 6)).astype(np.float32)
    wt = g.standard_normal((6, 5)).astype(np.float32)
    dense = [bf_matvec(x[t], wt.tolist()) for t in range(2)]
    assert np.allclose(oracle.sparse_linear(x, wt, 6), dense, rtol=1e-12, atol=1e-12)
    assert np.all(oracle.sparse_linear(x, wt, 0) == 0.0)


def test_sparse_linear_unselected_rows_do_not_matter():
    g = np.random.default_rng(11)
    x = g.standard_normal((1, 64)).astype(np.float32)
    wt = g.standard_normal((64, 16)).astype(np.float32)
    k = 20
    keep = oracle.topk_keep(x, k)[0]
    y0 = oracle.sparse_linear(x, wt, k)
    dropped = np.setdiff1d(np.arange(64), keep)
    wt2 = wt.copy()
    wt2[dropped] = 1e6                        # masked columns contribute nothing
    assert np.array_equal(oracle.sparse_linear(x, wt2, k), y0)
    wt3 = wt.copy()
    wt3[keep[0]] += 1.0                       # a kept row does contribute
    assert not np.array_equal(oracle.sparse_linear(x, wt3, k), y0)


# ---------------------------------------------------------------- STE backward


def test_ste_backward_golden_hand():
    g = load_golden("ste_backward_hand.json")
    x = np.array(g["x"], dtype=np.float32)
    wt = np.array(g["wt"], dtype=np.float32)
    gy = np.array(g["grad_y"], dtype=np.float32)
    for k, want in g["grad_wt"].items():
        r = oracle.sparse_linear_backward_ste(x, wt, int(k), gy)
        assert r["grad_x"].tolist() == g["grad_x"]
        assert r["grad_wt"].tolist() == want


@pytest.mark.parametrize("seed", range(8))
def test_ste_backward_bruteforce(seed):
    """Plain loops: dL/dX[t, i] = sum_j dL/dY[t, j] W^T[i, j] for every K (the
    estimator copies the gradient through the mask); dL/dW^T[i, j] = sum over
    the tokens that kept input i of x[t, i] dL/dY[t, j], zero for inputs no
    token kept."""
    g = np.random.default_rng(300 + seed)
    T, d_in, d_out = int(g.integers(1, 4)), int(g.integers(1, 8)), int(g.integers(1, 6))
    x = g.standard_normal((T, d_in)).astype(np.float32)
    wt = g.standard_normal((d_in, d_out)).astype(np.float32)
    gy = g.standard_normal((T, d_out)).astype(np.float32)
    for k in range(d_in + 1):
        r = oracle.sparse_linear_backward_ste(x, wt, k, gy)
        kept = [set(bf_keep(x[t], k)) for t in range(T)]
        for t in range(T):
            for i in range(d_in):
                ref = sum(float(gy[t, j]) * float(wt[i, j]) for j in range(d_out))
                assert math.isclose(r["grad_x"][t, i], ref, rel_tol=1e-12, abs_tol=1e-12)
        for i in range(d_in):
            for j in range(d_out):
                ref = sum(float(x[t, i]) * float(gy[t, j]) for t in range(T) if i in kept[t])
                assert math.isclose(r["grad_wt"][i, j], ref, rel_tol=1e-12, abs_tol=1e-12)
            if not any(i in kt for kt in kept):
                assert np.all(r["grad_wt"][i] == 0.0)


@pytest.mark.parametrize("seed", range(4))
def test_ste_backward_finite_differences(seed):
    """L = sum(dL/dY * Y) is linear in W^T, so a central difference along any
    direction equals <dL/dW^T, direction> up to rounding; with K = d the mask
    is all ones, the layer is dense, and the estimator's dL/dX is the true
    gradient, checked the same way (Y by plain loops, not the oracle)."""
    g = np.random.default_rng(400 + seed)
    T, d_in, d_out = 3, 7, 5
    x = g.standard_normal((T, d_in))
    wt = g.standard_normal((d_in, d_out))
    gy = g.standard_normal((T, d_out))

    def loss(xx, ww, k):
        total = 0.0
        for t in range(T):
            kept = set(bf_keep(xx[t], k))
            xs = [xx[t, i] if i in kept else 0.0 for i in range(d_in)]
            y = bf_matvec(xs, ww.tolist())
            total += sum(gy[t, j] * y[j] for j in range(d_out))
        return total

    for k in (0, 2, d_in):
        r = oracle.sparse_linear_backward_ste(x, wt, k, gy)
        D = g.standard_normal((d_in, d_out))
        fd = (loss(x, wt + D, k) - loss(x, wt - D, k)) / 2.0
        assert math.isclose(fd, float(np.sum(r["grad_wt"] * D)), rel_tol=1e-9, abs_tol=1e-9)
    r = oracle.sparse_linear_backward_ste(x, wt, d_in, gy)
    E = g.standard_normal((T, d_in))
    fd = (loss(x + E, wt, d_in) - loss(x - E, wt, d_in)) / 2.0
    assert math.isclose(fd, float(np.sum(r["grad_x"] * E)), rel_tol=1e-9, abs_tol=1e-9)
    # the estimator's dL/dX does not depend on K
    for k in range(d_in + 1):
        assert np.array_equal(oracle.sparse_linear_backward_ste(x, wt, k, gy)["grad_x"], r["grad_x"])


# ---------------------------------------------------------------- FFN


def test_ffn_golden_hand_relu2():
    g = load_golden("ffn_hand.json")
    x = np.array([g["x"]], dtype=np.float32)
    c = g["relu2_glu"]
    for k_h, want in c["y"].items():
        r = oracle.sparse_ffn(x, g["wt_up"], g["wt_gate"], g["wt_down"], "relu2_glu",
                              c["k_in"], int(k_h))
        assert r["u"][0].tolist() == c["u"]
        assert r["g"][0].tolist() == c["g"]
        assert r["h"][0].tolist() == c["h"]
        assert r["keep_h"][0].tolist() == c["keep_h"][k_h]
        assert r["y"][0].tolist() == want


def test_ffn_golden_hand_drelu():
    g = load_golden("ffn_hand.json")
    x = np.array([g["x"]], dtype=np.float32)
    c = g["drelu"]
    b = np.full(4, c["bias"])
    r = oracle.sparse_ffn(x, g["wt_up"], g["wt_gate"], g["wt_down"], "drelu", c["k_in"],
                          c["k_h"], b_up=b, b_gate=b)
    assert r["u"][0].tolist() == c["u"]
    assert r["g"][0].tolist() == c["g"]
    assert r["h"][0].tolist() == c["h"]
    assert r["keep_h"][0].tolist() == c["keep_h"]
    assert r["y"][0].tolist() == c["y"]


@pytest.mark.parametrize("act", ["relu2_glu", "drelu"])
@pytest.mark.parametrize("seed", range(6))
def test_ffn_bruteforce_tiny(act, seed):
    g = np.random.default_rng(200 + seed)
    dm, dff = int(g.integers(2, 7)), int(g.integers(2, 9))
    x = g.standard_normal((1, dm)).astype(np.float32)
    up = g.standard_normal((dm, dff))
    gate = g.standard_normal((dm, dff))
    down = g.standard_normal((dff, dm))
    bu = g.standard_normal(dff) * 0.3
    bg = g.standard_normal(dff) * 0.3
    k_in = int(g.integers(0, dm + 1))
    k_h = int(g.integers(0, dff + 1))
    r = oracle.sparse_ffn(x, up, gate, down, act, k_in, k_h, b_up=bu, b_gate=bg)
    kept = set(bf_keep(x[0], k_in))
    xs = [x[0, i] if i in kept else 0.0 for i in range(dm)]
    u = bf_matvec(xs, up.tolist())
    gg = bf_matvec(xs, gate.tolist())
    if act == "relu2_glu":
        h = [max(u[j], 0.0) * max(u[j], 0.0) * gg[j] for j in range(dff)]
    else:
        h = [max(gg[j] + bg[j], 0.0) * max(u[j] + bu[j], 0.0) for j in range(dff)]
    assert np.allclose(r["h"][0], h, rtol=1e-10, atol=1e-12)
    kh = set(bf_keep(r["h"][0], k_h))
    hs = [r["h"][0, j] if j in kh else 0.0 for j in range(dff)]
    assert np.allclose(r["y"][0], bf_matvec(hs, down.tolist()), rtol=1e-10, atol=1e-12)


def test_ffn_relu2_invariants():
    w = workloads.WORKLOADS["ffn_relu2_llama7b"]
    g = np.random.default_rng(5)
    dm, dff = 256, 512
    x = g.standard_normal((2, dm)).astype(np.float32)
    up = g.standard_normal((dm, dff)) / 16
    gate = g.standard_normal((dm, dff)) / 16
    down = g.standard_normal((dff, dm)) / 22
    r = oracle.sparse_ffn(x, up, gate, down, "relu2_glu", 179, 358)
    sq = np.maximum(r["u"], 0) ** 2
    assert np.all(sq >= 0)
    assert np.all(r["h"][r["u"] <= 0] == 0)                 # zeros preserved
    assert np.all(np.sign(r["h"][r["u"] > 0]) == np.sign(r["g"][r["u"] > 0]))
    assert w.k_h == 7705 and w.k == 2867                    # floor(0.7 d)


def test_ffn_drelu_invariants():
    g = np.random.default_rng(6)
    dm, dff = 128, 512
    x = g.standard_normal((2, dm)).astype(np.float32)
    up = g.standard_normal((dm, dff)) / math.sqrt(dm)
    gate = g.standard_normal((dm, dff)) / math.sqrt(dm)
    down = g.standard_normal((dff, dm)) / math.sqrt(dff)
    b = np.full(dff, -0.8)
    r = oracle.sparse_ffn(x, up, gate, down, "drelu", dm, 51, b_up=b, b_gate=b)
    assert np.all(r["h"] >= 0)
    assert np.all(r["h"][(r["u"] - 0.8 <= 0) | (r["g"] - 0.8 <= 0)] == 0)


def test_ffn_drelu_closed_gates_ignore_up():
    """The fact the gate-first dReLU layer rests on: where g + b_gate <= 0, h
    is 0 whatever u is, so replacing u there by any finite values (here huge
    ones) leaves h, and so y, unchanged; changing u at an open gate does not."""
    g = np.random.default_rng(8)
    T, dff = 3, 400
    u = g.standard_normal((T, dff))
    gt = g.standard_normal((T, dff))
    b = np.full(dff, -0.8)
    h = oracle.ffn_hidden(u, gt, "drelu", b_up=b, b_gate=b)
    closed = gt + b <= 0
    u2 = np.where(closed, g.standard_normal((T, dff)) * 1e30, u)
    assert np.array_equal(oracle.ffn_hidden(u2, gt, "drelu", b_up=b, b_gate=b), h)
    t, j = map(int, np.argwhere(~closed & (u + b > 0))[0])
    u3 = u.copy()
    u3[t, j] += 1.0
    assert not np.array_equal(oracle.ffn_hidden(u3, gt, "drelu", b_up=b, b_gate=b), h)


def test_ffn_k_full_is_dense_glu():
    g = np.random.default_rng(8)
    x = g.standard_normal((1, 5)).astype(np.float32)
    up, gate, down = g.standard_normal((5, 7)), g.standard_normal((5, 7)), g.standard_normal((7, 5))
    r = oracle.sparse_ffn(x, up, gate, down, "relu2_glu", 5, 7)
    u = x.astype(np.float64) @ up
    gg = x.astype(np.float64) @ gate
    h = [max(u[0, j], 0) ** 2 * gg[0, j] for j in range(7)]
    assert np.allclose(r["y"][0], bf_matvec(h, down.tolist()), rtol=1e-10)


# ---------------------------------------------------------------- quantizers


def test_absmax_quantize_golden_hand():
    g = load_golden("quant_hand.json")
    for c in g["act_cases"]:
        q, gamma = oracle.absmax_quantize(np.array([c["x"]], dtype=np.float32), g["eps"])
        assert q[0].tolist() == c["q"], c
        if "gamma" in c:
            assert float(gamma[0]) == c["gamma"]


@pytest.mark.parametrize("seed", range(10))
def test_absmax_quantize_properties(seed):
    g = np.random.default_rng(300 + seed)
    x = (g.standard_normal((4, 37)) * 10 ** g.uniform(-3, 3)).astype(np.float32)
    q, gamma = oracle.absmax_quantize(x)
    assert np.all(np.abs(q) <= 127)
    q_neg, _ = oracle.absmax_quantize(-x)
    assert np.array_equal(q_neg, -q)                        # symmetric
    # q is x * 127 / (amax + eps) rounded: within 1/2 (+ float32 slack) in fp64
    ref = x.astype(np.float64) * 127.0 / (np.abs(x).max(axis=1, keepdims=True) + 1e-5)
    assert np.all(np.abs(q - ref) <= 0.5 + 1e-3)
    # the largest |x| of each row lands on |q| = 127 or just under
    am = np.argmax(np.abs(x), axis=1)
    assert np.all(np.abs(q[np.arange(4), am]) >= 126)


def test_ternary_quantize_golden_hand():
    g = load_golden("quant_hand.json")
    for c in g["ternary_cases"]:
        t, alpha = oracle.ternary_quantize(np.array(c["w"], dtype=np.float32), g["eps"])
        assert float(alpha) == c["alpha"]
        assert t.tolist() == c["t"]


def test_ternary_values_and_alpha_is_mean_abs():
    w = workloads.weight_out_major(64, 96, 99)
    t, alpha = oracle.ternary_quantize(w)
    assert set(np.unique(t).tolist()) <= {-1, 0, 1}
    eff = alpha * t.astype(np.float32)                      # weights in {-a, 0, a}
    assert set(np.unique(np.abs(eff)).tolist()) <= {0.0, float(alpha)}
    mean_abs = sum(abs(float(v)) for v in w.reshape(-1)) / w.size
    assert abs(float(alpha) - mean_abs) <= 1e-7 * mean_abs
    # round-clip: |W| >= 1.5 (alpha+eps) -> +-1 ; |W| < 0.5 (alpha+eps) -> 0
    a = float(alpha) + 1e-5
    assert np.all(t[np.abs(w) >= 1.5 * a] == np.sign(w[np.abs(w) >= 1.5 * a]))
    assert np.all(t[np.abs(w) < 0.49 * a] == 0)


def test_ternary_pack_golden_and_roundtrip():
    g = load_golden("quant_hand.json")
    c = g["pack_case"]
    t = np.zeros((16, 2), dtype=np.int8)
    t[:, 0] = c["t_col0"]
    t[:, 1] = c["t_col1_all"]
    p = oracle.ternary_pack(t)
    assert p.tolist() == c["packed"]
    assert np.array_equal(oracle.ternary_unpack(p, 16), t)
    # brute-force bit layout on a random matrix
    gen = np.random.default_rng(3)
    t = gen.integers(-1, 2, size=(48, 5)).astype(np.int8)
    p = oracle.ternary_pack(t)
    for i, j in itertools.product(range(5), range(48)):
        code = (int(p[i, j // 16]) >> (2 * (j % 16))) & 3
        assert code == {0: 0, 1: 1, -1: 2}[int(t[j, i])]
    assert np.array_equal(oracle.ternary_unpack(p, 48), t)


def test_quant_sparse_linear_golden_hand():
    g = load_golden("quant_hand.json")
    c = g["linear_case"]
    r = oracle.quant_sparse_linear(np.array([c["x"]], np.float32), np.array(c["t"]),
                                   np.float32(c["alpha"]), c["k"])
    assert r["keep"][0].tolist() == c["keep"]
    assert r["acc"][0].tolist() == c["acc"]
    assert np.allclose(r["y"][0], c["y_approx"], rtol=2e-7)


def _rne_f32(q):
    """An exact rational rounded to the nearest float32, ties to even (normal
    range), by integer arithmetic: independent of numpy's float32 operations."""
    from fractions import Fraction
    if q == 0:
        return 0.0
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    ulp = Fraction(2) ** (e - 23)
    m = a / ulp
    fl = m.numerator // m.denominator
    rem = m - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return math.copysign(float(fl * ulp), float(q))


def _rint_even(q):
    from fractions import Fraction
    fl = q.numerator // q.denominator
    rem = q - fl
    return fl + (1 if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1) else 0)


def _f32_from_hex(h):
    return np.array([int(h, 16)], dtype=np.uint32).view(np.float32)[0]


def _hex(v):
    return hex(int(np.array([v], dtype=np.float32).view(np.uint32)[0]))


def test_quant_rescale_order_golden_bits():
    """y = float32(acc) * ((alpha * gamma) / 127), each step rounded to float32
    in that order.  The golden case is derived again here with exact rationals
    rounded by hand (not numpy), the oracle must give the same bits, and the
    other grouping alpha * (gamma / 127) must differ in the last bit."""
    from fractions import Fraction as Fr
    g = load_golden("rescale_order_hand.json")
    x = [np.float32(v) for v in g["x"]]
    alpha = _f32_from_hex(g["alpha_bits"])
    eps = _rne_f32(Fr(np.float32(g["eps"]).item()))
    # the hand derivation
    gamma = _rne_f32(Fr(max(abs(float(v)) for v in x)) + Fr(eps))
    s = _rne_f32(Fr(127) / Fr(gamma))
    q = [max(-127, min(127, _rint_even(Fr(_rne_f32(Fr(float(v)) * Fr(s)))))) for v in x]
    r = _rne_f32(Fr(_rne_f32(Fr(float(alpha)) * Fr(gamma))) / 127)
    r_other = _rne_f32(Fr(float(alpha)) * Fr(_rne_f32(Fr(gamma) / 127)))
    keep = sorted(sorted(range(len(q)), key=lambda i: (-abs(q[i]), i))[:g["k"]])
    acc = [sum(q[i] * row[i] for i in keep) for row in g["t"]]
    y = [_rne_f32(Fr(a) * Fr(r)) for a in acc]
    y_other = [_rne_f32(Fr(a) * Fr(r_other)) for a in acc]
    assert _hex(gamma) == g["gamma_bits"] and _hex(s) == g["s_bits"]
    assert q == g["q"] and keep == g["keep"] and acc == g["acc"]
    assert _hex(r) == g["r_bits"] and _hex(r_other) == g["other_order_r_bits"]
    assert [_hex(v) for v in y] == g["y_bits"]
    assert [_hex(v) for v in y_other] == g["other_order_y_bits"]
    assert all(a != b for a, b in zip(g["y_bits"], g["other_order_y_bits"]))
    # the oracle, bit for bit
    res = oracle.quant_sparse_linear(np.array([x], np.float32), np.array(g["t"]), alpha, g["k"],
                                     eps=g["eps"])
    assert _hex(res["gamma"][0]) == g["gamma_bits"]
    assert res["q"][0].tolist() == g["q"] and res["keep"][0].tolist() == g["keep"]
    assert res["acc"][0].tolist() == g["acc"]
    assert _hex(res["r"][0]) == g["r_bits"]
    assert [_hex(v) for v in res["y"][0]] == g["y_bits"]


@pytest.mark.parametrize("seed", range(8))
def test_quant_sparse_linear_bruteforce(seed):
    g = np.random.default_rng(400 + seed)
    T, d_in, d_out = 2, int(g.integers(1, 10)), int(g.integers(1, 6))
    x = g.standard_normal((T, d_in)).astype(np.float32)
    t = g.integers(-1, 2, size=(d_out, d_in))
    k = int(g.integers(0, d_in + 1))
    r = oracle.quant_sparse_linear(x, t, np.float32(0.37), k)
    for tt in range(T):
        kept = set(bf_keep(r["q"][tt], k))              # top-K on |q|, not on |x|
        for j in range(d_out):
            acc = sum(int(r["q"][tt, i]) * int(t[j, i]) for i in range(d_in) if i in kept)
            assert int(r["acc"][tt, j]) == acc
    approx = r["acc"] * (0.37 * r["gamma"].astype(np.float64)[:, None] / 127.0)
    assert np.allclose(r["y"], approx, rtol=1e-6, atol=1e-12)


def test_quant_topk_on_q_ties():
    # many equal |q| near the threshold: lower index first among equals
    x = np.array([[0.5, -0.5, 1.0, 0.5, -0.5, 0.25]], dtype=np.float32)
    r = oracle.quant_sparse_linear(x, np.eye(6, dtype=np.int64), np.float32(1.0), 3)
    assert r["keep"][0].tolist() == [0, 1, 2]


# ---------------------------------------------------------------- error measure


def test_max_rel_err_definition():
    ref = np.array([[1.0, -4.0, 2.0], [0.0, 0.0, 0.0]])
    y = np.array([[1.1, -4.0, 2.0], [0.0, 0.5, 0.0]])
    # row 0: 0.1 / 4 ; row 1 (all-zero reference): 0.5 / 1
    assert oracle.max_rel_err(y, ref) == pytest.approx(0.5)
    assert oracle.max_rel_err(y[:1], ref[:1]) == pytest.approx(0.025)


# ---------------------------------------------------------------- Block Q-Sparse pins


def test_block_topk_golden_hand():
    g = load_golden("block_topk_hand.json")
    x = np.array(g["x"], dtype=np.float32)
    for k, want in g["keep"].items():
        assert oracle.block_topk_keep(x, int(k), g["block"]).tolist() == want, k
    keep3 = oracle.block_topk_keep(x, 3, g["block"])
    xs = x.astype(np.float64) * oracle.mask_from_keep(keep3, *x.shape)
    assert xs[1].tolist() == g["xs_row1_k3"]
    assert oracle.topk_keep(x, 3)[1].tolist() == g["per_row_keep_row1_k3"]
    rows_read = sorted({int(i) for t in (0, 1) for i in keep3[t] if x[t, i] != 0})
    assert rows_read == g["block0_rows_read_k3"]
    assert np.unique(oracle.topk_keep(x[:2], 3)).tolist() == g["per_row_union_block0_k3"]


@pytest.mark.parametrize("seed", range(6))
def test_block_of_one_token_is_per_token_topk(seed):
    g = workloads.rng(600 + seed)
    x = workloads.adversarial_rows(seed, 5, 37) if seed % 2 else \
        workloads.normal_f32(g, (7, 41))
    for k in (0, 1, 5, x.shape[1] // 2, x.shape[1]):
        assert np.array_equal(oracle.block_topk_keep(x, k, 1), oracle.topk_keep(x, k))


@pytest.mark.parametrize("seed", range(12))
def test_block_topk_bruteforce(seed):
    """Block magnitude by loops (max of |x| over the block's rows), kept set by
    the O(d^2) rank count, rows of one block sharing it."""
    g = np.random.default_rng(700 + seed)
    T, d = int(g.integers(1, 9)), int(g.integers(1, 13))
    block = int(g.integers(1, T + 2))
    x = g.integers(-4, 5, size=(T, d)).astype(np.float32) * np.float32(0.5)
    for k in range(d + 1):
        got = oracle.block_topk_keep(x, k, block)
        for b0 in range(0, T, block):
            rows = range(b0, min(T, b0 + block))
            s = [max(abs(float(x[t, i])) for t in rows) for i in range(d)]
            want = bf_keep(s, k)
            for t in rows:
                assert got[t].tolist() == want, (seed, k, block)


def test_block_topk_invariants_at_decode_sizes():
    w = workloads.WORKLOADS["ffn_relu2_llama7b"]
    x = workloads.activations(w, 8)
    for block in (2, 4, 8, 16):
        keep = oracle.block_topk_keep(x, w.k, block)
        for b0 in range(0, 8, block):
            rows = list(range(b0, min(8, b0 + block)))
            assert all(np.array_equal(keep[t], keep[rows[0]]) for t in rows)
            s = np.max(np.abs(x[rows].astype(np.float64)), axis=0)
            kept = np.zeros(x.shape[1], bool)
            kept[keep[rows[0]]] = True
            assert s[kept].min() >= s[~kept].max()
            # the block reads at most k weight rows, fewer than the per-row union
            union = np.unique(oracle.topk_keep(x[rows], w.k))
            assert np.unique(keep[rows]).size == w.k <= union.size


@pytest.mark.parametrize("act", ["relu2_glu", "drelu"])
@pytest.mark.parametrize("seed", range(4))
def test_block_ffn_bruteforce_tiny(act, seed):
    """sparse_ffn with a block selection on x and on h, by plain loops."""
    g = np.random.default_rng(800 + seed)
    T, dm, dff, block = 5, 6, 7, 2
    x = g.standard_normal((T, dm))
    up, gate = g.standard_normal((dm, dff)), g.standard_normal((dm, dff))
    down = g.standard_normal((dff, dm))
    bu = bg = -0.2 if act == "drelu" else None
    r = oracle.sparse_ffn(x, up, gate, down, act, 4, 3, b_up=bu, b_gate=bg, block=block)
    kx = oracle.block_topk_keep(x, 4, block)
    for t in range(T):
        xs = [x[t, i] if i in kx[t] else 0.0 for i in range(dm)]
        u = bf_matvec(xs, up.tolist())
        gg = bf_matvec(xs, gate.tolist())
        if act == "relu2_glu":
            h = [max(u[j], 0.0) ** 2 * gg[j] for j in range(dff)]
        else:
            h = [max(gg[j] - 0.2, 0.0) * max(u[j] - 0.2, 0.0) for j in range(dff)]
        assert np.allclose(r["h"][t], h, rtol=1e-10, atol=1e-12)
    kh = oracle.block_topk_keep(r["h"], 3, block)
    assert np.array_equal(r["keep_h"], kh)
    for t in range(T):
        hs = [r["h"][t, j] if j in kh[t] else 0.0 for j in range(dff)]
        assert np.allclose(r["y"][t], bf_matvec(hs, down.tolist()), rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------- quantized FFN chain pins


def test_ffn_hidden_f32_golden_hand():
    g = load_golden("quant_ffn_hand.json")
    c = g["relu2"]
    assert oracle.ffn_hidden_f32(c["u"], c["g"], "relu2_glu").tolist() == c["h"]
    c = g["drelu"]
    assert oracle.ffn_hidden_f32(c["u"], c["g"], "drelu", b_up=c["b"], b_gate=c["b"]).tolist() == c["h"]
    c = g["rounding"]
    u = _f32_from_hex(c["u_bits"])
    h = oracle.ffn_hidden_f32([u], [c["g"]], "relu2_glu")[0]
    assert _hex(h) == c["h_bits"]
    # the fp64 epilogue is different in the last bits here: the f32 steps are pinned
    assert oracle.ffn_hidden([float(u)], [c["g"]], "relu2_glu")[0] != float(h)


def _bf_quant_ffn(x, t_up, a_up, t_gate, a_gate, t_down, a_down, act, k_in, k_h, b, eps=1e-5):
    """The quantized FFN by loops, every float32 step rounded by hand from an
    exact rational (independent of numpy's float32 arithmetic)."""
    from fractions import Fraction as Fr
    eps32 = _rne_f32(Fr(np.float32(eps).item()))

    def quant(row):
        gamma = _rne_f32(Fr(max(abs(float(v)) for v in row)) + Fr(eps32))
        s = _rne_f32(Fr(127) / Fr(gamma))
        q = [max(-127, min(127, _rint_even(Fr(_rne_f32(Fr(float(v)) * Fr(s)))))) for v in row]
        return q, gamma

    def proj(q, gamma, keep, t, alpha):
        r = _rne_f32(Fr(_rne_f32(Fr(float(alpha)) * Fr(gamma))) / 127)
        out = []
        for j in range(len(t)):
            acc = sum(q[i] * int(t[j][i]) for i in keep)
            out.append(_rne_f32(Fr(acc) * Fr(r)))
        return out

    ys = []
    for row in x:
        q, gamma = quant(row)
        keep = bf_keep([abs(v) for v in q], k_in)
        u = proj(q, gamma, keep, t_up, a_up)
        gg = proj(q, gamma, keep, t_gate, a_gate)
        h = []
        for uj, gj in zip(u, gg):
            if act == "relu2_glu":
                r = max(uj, 0.0)
                h.append(_rne_f32(Fr(_rne_f32(Fr(r) * Fr(r))) * Fr(gj)))
            else:
                ga = max(_rne_f32(Fr(gj) + Fr(float(np.float32(b)))), 0.0)
                ua = max(_rne_f32(Fr(uj) + Fr(float(np.float32(b)))), 0.0)
                h.append(_rne_f32(Fr(ga) * Fr(ua)))
        qh, gh = quant(h)
        keep_h = bf_keep([abs(v) for v in qh], k_h)
        ys.append(proj(qh, gh, keep_h, t_down, a_down))
    return np.array(ys, dtype=np.float32)


@pytest.mark.parametrize("act", ["relu2_glu", "drelu"])
@pytest.mark.parametrize("seed", range(4))
def test_quant_ffn_bruteforce_bits(act, seed):
    g = np.random.default_rng(900 + seed)
    T, dm, dff = 3, 7, 9
    x = (g.standard_normal((T, dm)) * 2).astype(np.float32)
    x[0, 2] = 0.0
    ts = [oracle.ternary_quantize(g.standard_normal(shape).astype(np.float32))
          for shape in ((dff, dm), (dff, dm), (dm, dff))]
    b = -0.1 if act == "drelu" else None
    for k_in, k_h in ((4, 5), (dm, dff), (1, 2)):
        r = oracle.quant_sparse_ffn(x, ts[0][0], ts[0][1], ts[1][0], ts[1][1], ts[2][0], ts[2][1],
                                    act, k_in, k_h, b_up=b, b_gate=b)
        bf = _bf_quant_ffn(x, ts[0][0], ts[0][1], ts[1][0], ts[1][1], ts[2][0], ts[2][1], act, k_in,
                           k_h, b)
        assert np.array_equal(r["y"].view(np.int32), bf.view(np.int32)), (act, k_in, k_h)


def test_quant_ffn_invariants():
    g = np.random.default_rng(990)
    T, dm, dff = 4, 32, 48
    x = g.standard_normal((T, dm)).astype(np.float32)
    ts = [oracle.ternary_quantize(g.standard_normal(shape).astype(np.float32))
          for shape in ((dff, dm), (dff, dm), (dm, dff))]
    r = oracle.quant_sparse_ffn(x, ts[0][0], ts[0][1], ts[1][0], ts[1][1], ts[2][0], ts[2][1],
                                "relu2_glu", 20, 10)
    assert np.all(r["h"][r["u"] <= 0] == 0)                 # squared ReLU zeroes u <= 0
    assert all(np.count_nonzero(r["q_h"][t][r["keep_h"][t]]) <= 10 for t in range(T))
    rd = oracle.quant_sparse_ffn(x, ts[0][0], ts[0][1], ts[1][0], ts[1][1], ts[2][0], ts[2][1],
                                 "drelu", 20, 10, b_up=-0.2, b_gate=-0.2)
    assert np.all(rd["h"] >= 0) and np.all(rd["h"][(rd["g"] - np.float32(0.2)) <= 0] == 0)
    # block = 1 equals the per-token chain; a block of all tokens shares one selection
    rb = oracle.quant_sparse_ffn(x, ts[0][0], ts[0][1], ts[1][0], ts[1][1], ts[2][0], ts[2][1],
                                 "relu2_glu", 20, 10, block=T)
    assert all(np.array_equal(rb["keep_x"][t], rb["keep_x"][0]) for t in range(T))
