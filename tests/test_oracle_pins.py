"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each test ties one oracle function to a worked example printed on the pages
(fixtures under tests/golden/, each with its citation), a closed form, an
exact brute force, a library routine for a special case, or an independent
second route.  A plausible slip in the oracle (dropped term, wrong sign,
wrong index, wrong rounding, wrong tie-break) fails at least one of them;
tests/test_oracle_mutants.py plants such slips in a copy of the oracle and
checks that this file catches each.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synth
from synth import workloads as wl
from conftest import read_golden


def F(v):
    return Fraction(float(v))


# ---- quantizer ---------------------------------------------------------------

def test_absmax_worked_example():
    """2048ai.net s3.1: alpha=10.8 -> s=alpha/127; 3.08 and 3.02 -> 36 -> ~3.06."""
    g = read_golden("absmax_worked_example.txt")
    alpha = float(next(v for k, v in g if k == "alpha")[0])
    s = oracle.scale_from_absmax(alpha)
    # s is the float nearest to alpha/127 (closed form, exact rational check)
    exact = Fraction(alpha) / 127
    assert abs(F(s) - exact) <= abs(F(np.nextafter(s, np.float32(1))) - exact)
    assert abs(F(s) - exact) <= abs(F(np.nextafter(s, np.float32(0))) - exact)
    for key, vals in g:
        if key == "code":
            assert oracle.quantize(float(vals[0]), s) == int(vals[1]), vals
        if key == "dequant":
            q, expect, tol = int(vals[0]), float(vals[1]), float(vals[2])
            assert abs(q * float(s) - expect) <= tol


def test_range_is_symmetric_127():
    """Visual guide: [-127, 127], not [-128, 127]; values beyond clip."""
    s = oracle.scale_from_absmax(1.0)
    assert oracle.quantize(1e6, s) == 127
    assert oracle.quantize(-1e6, s) == -127
    assert oracle.quantize(-1.0, s) == -127
    assert oracle.quantize(1.0, s) == 127
    assert oracle.quantize(0.3, 0.0) == 0       # zero scale -> zero code


@pytest.mark.parametrize("v,s,q", [
    (2.5, 1.0, 3), (-2.5, 1.0, -3), (0.5, 1.0, 1), (-0.5, 1.0, -1), (1.5, 1.0, 2),
    (-1.5, 1.0, -2), (1.25, 0.5, 3), (0.49999999999999994, 1.0, 0), (126.5, 1.0, 127),
    (-126.5, 1.0, -127), (0.0, 1.0, 0), (-0.0, 1.0, 0)])
def test_round_half_away_from_zero(v, s, q):
    assert oracle.quantize(v, s) == q


def _brute_code(r: Fraction, s: Fraction) -> int:
    """argmin over all 255 codes of |r - q*s|, ties to the larger |q|."""
    best, best_err = 0, None
    for q in range(-127, 128):
        err = abs(r - q * s)
        if best_err is None or err < best_err or (err == best_err and abs(q) > abs(best)):
            best, best_err = q, err
    return best


def test_group_codes_brute_force_8x8():
    rng = np.random.default_rng(7)
    r = rng.laplace(0, 0.02, (8, 8))
    r[3, :4] = 0.0                      # an all-zero group
    r[5, 5] = 0.5 * r[5, 4]             # exact half-way structure
    for row in r:
        q, s = oracle.quantize_groups(row, 4)
        for g in range(2):
            blk = row[4 * g:4 * g + 4]
            a = max(abs(float(v)) for v in blk)
            assert (s[g] == 0) == (a == 0)
            for j, v in enumerate(blk):
                expect = 0 if s[g] == 0 else _brute_code(Fraction(float(v)), F(s[g]))
                assert q[4 * g + j] == expect
            if a > 0:  # the group maximum lands on the end of the range
                jm = int(np.argmax(np.abs(blk)))
                assert abs(int(q[4 * g + jm])) == 127


def test_dequant_error_bound():
    """Visual guide e_i = x_i - xhat_i; round-to-nearest bounds it by s/2."""
    W = wl.config1().weights()[:64]
    d = oracle.decompose(W, want_residual=True)
    ng = d["s"].shape[1]
    for r in range(W.shape[0]):
        for g in range(ng):
            s = float(d["s"][r, g])
            blk = slice(128 * g, 128 * g + 128)
            err = np.abs(d["res"][r, blk] - d["q"][r, blk].astype(np.float64) * s)
            assert np.all(err <= s / 2)


def test_group_scaling_example():
    """Visual guide Q4_K section: two blocks of four beat one shared scale."""
    g = dict(read_golden("group_scaling_example.txt"))
    row = np.array([float(v) for v in g["row"]])
    blk = int(g["block"][0])
    qg, sg = oracle.quantize_groups(row, blk)
    qs, ss = oracle.quantize_groups(row, len(row))
    err_g = np.abs(row - qg * np.repeat(sg.astype(np.float64), blk))
    err_s = np.abs(row - qs * float(ss[0]))
    assert err_g.max() < err_s.max()
    # the small-valued first block gains the most from its own scale
    assert err_g[:blk].max() * 10 < err_s[:blk].max()
    assert sg[0] < sg[1] and ss[0] == sg[1]


# ---- threshold, sign and alpha -----------------------------------------------

def test_threshold_is_smallest_value_reaching_the_percentile():
    """Nearest-rank percentile = min{v in |w| : #(|w| <= v) * 100 >= P * K}."""
    rng = np.random.default_rng(3)
    for K in (1, 7, 100, 4096):
        w = rng.laplace(0, 0.02, K).astype(np.float32)
        w[: K // 7] = np.round(w[: K // 7], 2)          # some ties
        a = np.abs(w)
        for P in (1, 50, 60, 80, 100):
            tau = oracle.trunk_threshold(w, P)
            assert tau in a
            assert int((a <= tau).sum()) * 100 >= P * K
            below = a[a < tau]
            if below.size:
                assert int((a <= below.max()).sum()) * 100 < P * K, (K, P)


def test_threshold_closed_form():
    """|W| = 1..10, 60th percentile (nearest rank 6) -> tau 6, trunk {7..10}."""
    w = np.array([1, -2, 3, -4, 5, -6, 7, -8, 9, -10], np.float32)
    assert oracle.trunk_threshold(w, 60) == 6.0
    d = oracle.decompose(w[None, :], G=32, P=60)
    assert d["mask"][0].tolist() == [0] * 6 + [1] * 4
    assert d["alpha"][0] == np.float32(8.5)


def test_sign_tiebreak_zero_is_positive():
    """BitNet weight binarization: non-negative -> +1 (both zeros)."""
    w = np.array([[0.0, -0.0, 1.0, -1.0, 1e-30, -1e-30]], np.float32)
    d = oracle.decompose(w, G=32)
    assert d["sign"][0].tolist() == [1, 1, 1, 0, 1, 0]


def test_alpha_closed_form_full_trunk():
    w = np.array([[0.5, -1.5, 1.5, -0.5, 2.0, -0.0]], np.float32)
    d = oracle.decompose(w, G=32)
    assert d["alpha"][0] == np.float32(1.0)     # (0.5+1.5+1.5+0.5+2+0)/6
    w2 = np.zeros((1, 40), np.float32)
    assert oracle.decompose(w2, G=32)["alpha"][0] == 0.0


def test_empty_trunk_at_100th_percentile():
    w = np.array([[0.25, -0.5, 0.125, 0.5]], np.float32)
    d = oracle.decompose(w, G=32, P=100)
    assert d["mask"].sum() == 0 and d["alpha"][0] == 0.0
    # everything is residual: codes of W itself
    assert d["q"][0].tolist() == [64, -127, 32, 127]


# ---- decomposition identity ----------------------------------------------------

@pytest.mark.parametrize("P", [-1, 60])
def test_residual_plus_trunk_is_W(P):
    """m.lqnn.cn s2.1: W_res = W - alpha*sign(W), exactly, before rounding."""
    W = wl.config1().weights()
    d = oracle.decompose(W, P=P, want_residual=True)
    trunk = d["mask"] * (2.0 * d["sign"] - 1.0) * d["alpha"].astype(np.float64)[:, None]
    recon = d["res"] + trunk
    ok = np.abs(W) >= 2.0 ** -29 * d["alpha"][:, None]
    assert np.all(recon[ok] == W.astype(np.float64)[ok])
    assert ok.all()


# ---- exact end-to-end closed forms ---------------------------------------------

def _exact_row(rng, K, big=None):
    """A row whose decomposition is lossless: alpha exact, residual codes exact.

    Trunk magnitudes come in pairs 1 +- c/1024 (mean exactly 1); every group
    of 128 holds one |c| = 127 so its scale is exactly 2^-10.  With ``big``,
    the trunk entries are ``big +- c/1024`` and the other half of the row
    holds residual-only entries c/1024.
    """
    c = rng.integers(0, 128, K)
    for g0 in range(0, K, 128):
        c[g0] = 127
    sgn = rng.choice([-1.0, 1.0], K)
    w = np.zeros(K)
    if big is None:
        pm = np.ones(K)
        pm[1::2] = -1.0
        if K % 2:
            c[-1] = 0 if K - 1 != (K - 1) // 128 * 128 else c[-1]
            pm[-1] = 1.0 if c[-1] == 0 else pm[-1]
        # pair (2i, 2i+1): +c and -c of the same c keep the mean at 1
        c[1::2] = c[0:K - 1:2][:len(c[1::2])]
        w = sgn * (1.0 + pm * c / 1024.0)
    else:
        in_trunk = np.zeros(K, bool)
        in_trunk[K // 2:] = True
        pm = np.ones(K)
        pm[K // 2 + 1::2] = -1.0
        ct = c.copy()
        ct[K // 2 + 1::2] = ct[K // 2:K - 1:2][:len(ct[K // 2 + 1::2])]
        w = np.where(in_trunk, sgn * (big + pm * ct / 1024.0), sgn * c / 1024.0)
    return w.astype(np.float32)


@pytest.mark.parametrize("K", [128, 130, 256, 384])
def test_lossless_row_gives_exact_dot(K):
    rng = np.random.default_rng(K)
    N = 6
    W = np.stack([_exact_row(rng, K) for _ in range(N)])
    d = oracle.decompose(W, G=128)
    assert np.all(d["alpha"] == 1.0)
    ng = d["s"].shape[1]
    # all groups hold a 127 code except possibly a short tail group
    assert np.all(d["s"][:, :K // 128] == np.float32(2.0 ** -10))
    x = rng.integers(-127, 128, (2, K)).astype(np.float32)
    x[:, 5] = 127.0
    idx = np.array([9, K - 1], np.int32)
    x[0, 9], x[0, K - 1] = 1000.25, -333.5
    x[1, 9], x[1, K - 1] = -4096.0, 0.75
    xq, sx, xout = oracle.quantize_act(x, idx)
    assert np.all(sx == 1.0)                    # absmax excludes the outliers
    y = oracle.linear(d, xq, sx, xout, idx)
    for t in range(2):
        for r in range(N):
            exact = sum(F(W[r, j]) * F(x[t, j]) for j in range(K))
            assert Fraction(y[t, r]) == exact
    assert ng == (K + 127) // 128


def test_lossless_threshold_row_gives_exact_dot():
    rng = np.random.default_rng(11)
    K = 256
    W = np.stack([_exact_row(rng, K, big=4.0) for _ in range(4)])
    d = oracle.decompose(W, G=128, P=50)
    assert np.all(d["mask"][:, K // 2:] == 1) and np.all(d["mask"][:, :K // 2] == 0)
    assert np.all(d["alpha"] == 4.0)
    x = rng.integers(-127, 128, (1, K)).astype(np.float32)
    x[0, 0] = -127.0
    idx = np.array([200], np.int32)
    x[0, 200] = 77.125
    xq, sx, xout = oracle.quantize_act(x, idx)
    y = oracle.linear(d, xq, sx, xout, idx)
    for r in range(4):
        exact = sum(F(W[r, j]) * F(x[0, j]) for j in range(K))
        assert Fraction(y[0, r]) == exact


def test_ternary_select_example():
    """2048ai.net s5.1: weights {+1,-1,-1,+1} give x0 - x1 - x2 + x3."""
    wts = [float(v) for v in dict(read_golden("ternary_example.txt"))["weights"]]
    K = 40
    w = np.full(K, 0.001, np.float32)
    w[1::2] = -0.001
    w[:4] = np.array(wts, np.float32) * 5.0
    d = oracle.decompose(w[None, :], G=32, P=90)   # the 4 large entries only
    assert d["mask"][0, :4].tolist() == [1, 1, 1, 1] and d["mask"][0, 4:].sum() == 0
    xq = np.random.default_rng(5).integers(-127, 128, (3, K)).astype(np.int8)
    T, _ = oracle.accumulate(d, xq)
    x = xq.astype(np.int64)
    assert np.all(T[:, 0] == x[:, 0] - x[:, 1] - x[:, 2] + x[:, 3])


def test_neuron_example_through_quantized_path():
    """Visual guide: W=[0.6,-0.4], b=0.1: x=[2,-1] -> 1.7, x'=[0.2,3] -> -0.98,
    reproduced through the separated path within the quantizers' error bound."""
    g = read_golden("neuron_example.txt")
    W = np.array([[float(v) for v in dict(g)["W"]]], np.float32)
    b = float(dict(g)["b"][0])
    d = oracle.decompose(W, G=32)
    for key, vals in g:
        if key != "case":
            continue
        x = np.array([[float(vals[0]), float(vals[1])]], np.float32)
        z = float(vals[2])
        xq, sx, xout = oracle.quantize_act(x, np.zeros(0, np.int32))
        y = oracle.linear(d, xq, sx, xout, np.zeros(0, np.int32))[0, 0] + b
        # |W.x - What.xhat| <= sum|W| sx/2 + sum|xhat| s_w/2
        bound = np.abs(W).sum() * float(sx[0]) / 2 + np.abs(xq[0] * float(sx[0])).sum() * float(d["s"][0, 0]) / 2
        assert abs(y - z) <= bound + 1e-12, (y, z, bound)


# ---- trunk by popcount and the two output routes ------------------------------

@pytest.mark.parametrize("K,P", [(33, -1), (100, 60), (128, -1), (300, 80)])
def test_popcount_identity(K, P):
    """m.lqnn.cn s2.3 bit trunk: 2*sum_{bit=1} xq - sum xq equals the +-1 sum."""
    rng = np.random.default_rng(K + P)
    W = rng.laplace(0, 0.02, (5, K)).astype(np.float32)
    W[0, :3] = 0.0
    d = oracle.decompose(W, G=32, P=P)
    xq = rng.integers(-127, 128, (3, K)).astype(np.int8)
    T, R = oracle.accumulate(d, xq)
    assert np.array_equal(T, oracle.trunk_popcount(d, xq))
    # and against a numpy +-1 product
    pm = (d["mask"] * (2 * d["sign"].astype(np.int64) - 1))
    assert np.array_equal(T, xq.astype(np.int64) @ pm.T)
    qg = d["q"].astype(np.int64).reshape(5, -1)
    for g in range(R.shape[2]):
        sl = slice(32 * g, min(K, 32 * g + 32))
        assert np.array_equal(R[:, :, g], xq[:, sl].astype(np.int64) @ qg[:, sl].T)


@pytest.mark.parametrize("P", [-1, 60])
def test_factored_equals_naive(P):
    L = wl.config1()
    W = L.weights()[:48]
    x = L.activations(M=3)
    idx = L.planted_channels()
    d = oracle.decompose(W, P=P)
    xq, sx, xout = oracle.quantize_act(x, idx)
    y = oracle.linear(d, xq, sx, xout, idx)
    yn = oracle.linear_naive(d, xq, sx, xout, idx)
    scale = oracle.abs_dot(W, x)
    assert np.all(np.abs(y - yn) <= 1e-12 * scale)
    # and the dequantized product approximates the original W.x
    ref = x.astype(np.float64) @ W.astype(np.float64).T
    assert np.all(np.abs(y - ref) <= 0.05 * scale)


# ---- trunk-only output (residual path skipped, [P1] s3.3) -----------------------

def _xhat(x, xq, sx, idx):
    """Dequantized activations: xq*sx off the outlier set, x itself on it."""
    xh = xq.astype(np.float64) * sx.astype(np.float64)[:, None]
    xh[:, idx] = x[:, idx].astype(np.float64)
    return xh


def test_trunk_only_binary_weights_is_the_exact_product():
    """Rows whose entries are all +-c_r: alpha_r = c_r, the residual vanishes,
    and the trunk-only output is the full output and the plain product W.xhat."""
    rng = np.random.default_rng(41)
    N, K = 24, 700
    c = (rng.integers(1, 64, N) / 1024.0).astype(np.float32)
    W = (np.where(rng.random((N, K)) < 0.5, -1.0, 1.0) * c[:, None]).astype(np.float32)
    x = rng.standard_normal((3, K)).astype(np.float32)
    idx = np.array([5, 311, 699], np.int32)
    x[:, idx] *= 40.0
    d = oracle.decompose(W)
    assert np.array_equal(d["alpha"], c) and not d["q"].any()
    xq, sx, xout = oracle.quantize_act(x, idx)
    yt = oracle.linear_trunk(d, xq, sx, xout, idx)
    ref = _xhat(x, xq, sx, idx) @ W.astype(np.float64).T
    scale = np.abs(_xhat(x, xq, sx, idx)) @ np.abs(W.astype(np.float64)).T
    assert np.all(np.abs(yt - ref) <= 1e-12 * scale)
    assert np.all(np.abs(yt - oracle.linear(d, xq, sx, xout, idx)) <= 1e-12 * scale)


@pytest.mark.parametrize("P", [-1, 60])
def test_trunk_only_plus_residual_path_is_the_full_output(P):
    """y - y_trunk is the residual path alone: the dense dequantized residual
    s_{r,g(j)} * q_rj times xhat, formed here with numpy."""
    L = wl.config1()
    W = L.weights()[:40]
    x = L.activations(M=2)
    idx = L.planted_channels()
    d = oracle.decompose(W, P=P)
    xq, sx, xout = oracle.quantize_act(x, idx)
    xh = _xhat(x, xq, sx, idx)
    y = oracle.linear(d, xq, sx, xout, idx)
    yt = oracle.linear_trunk(d, xq, sx, xout, idx)
    G = d["G"]
    res_hat = d["s"].astype(np.float64)[:, np.arange(W.shape[1]) // G] * d["q"].astype(np.float64)
    trunk_hat = d["mask"] * np.where(d["sign"] == 1, 1.0, -1.0) * d["alpha"].astype(np.float64)[:, None]
    scale = np.abs(xh) @ (np.abs(res_hat) + np.abs(trunk_hat)).T
    assert np.all(np.abs((y - yt) - xh @ res_hat.T) <= 1e-12 * scale)
    # the trunk-only output is the dense trunk weight times xhat: the mask
    # removes entries, outlier channels take the trunk weight, not the full one
    assert np.all(np.abs(yt - xh @ trunk_hat.T) <= 1e-12 * scale)
    if P > 0:
        assert (d["mask"] == 0).any()


# ---- sparse residual ([P1] s3.3, second point) -----------------------------------

@pytest.mark.parametrize("K,Ps", [(300, 60), (128, 50), (1000, 70), (97, 1), (64, 99)])
def test_sparse_residual_keeps_the_largest_entries(K, Ps):
    """Exactly the K - ceil(Ps*K/100) largest |r| survive (continuous values:
    no ties), checked against a sort."""
    r = np.random.default_rng(K + Ps).laplace(0, 0.02, K)
    keep, q, s = oracle.sparsify_residual(r, 32, Ps)
    rank = -(-Ps * K // 100)
    expect = np.zeros(K, np.uint8)
    expect[np.argsort(np.abs(r), kind="stable")[rank:]] = 1
    assert np.array_equal(keep, expect)
    assert not q[keep == 0].any()


def test_sparse_residual_ties_at_the_threshold_are_dropped():
    """|r| sorted: 0.25 x8, 0.5 x8, 1.0 x32, 2.0 x8, 3.0 x8.  Ps = 50 puts the
    rank (32) inside the run of 1.0s: theta = 1.0 and every 1.0 is dropped."""
    r = np.array([0.5, -1.0, 1.0, 1.0, -1.0, 2.0, 3.0, -0.25] * 8)
    keep, q, s = oracle.sparsify_residual(r, 32, 50)
    assert np.array_equal(keep, (np.abs(r) > 1.0).astype(np.uint8)) and keep.sum() == 16


def test_sparse_residual_codes_brute_force():
    """Kept entries take the brute-force nearest code under s = (binary32)
    (max kept |r| / 127); dropped ones 0; a group dropped whole gets s = 0."""
    rng = np.random.default_rng(52)
    r = rng.laplace(0, 0.02, 64)
    r[:32] = np.sign(r[:32]) * (0.01 + np.abs(r[:32]))  # every |r| of group 0 exceeds 0.01
    r[32:] *= 1e-3 / max(1.0, float(np.abs(r[32:]).max()) / 0.005)  # group 1 wholly below
    keep, q, s = oracle.sparsify_residual(r, 32, 50)
    assert not keep[32:].any() and s[1] == 0 and not q[32:].any()
    a = max(abs(float(v)) for v, k in zip(r[:32], keep[:32]) if k)
    assert s[0] == np.float32(a / 127.0)
    for j in range(32):
        assert q[j] == (_brute_code(Fraction(float(r[j])), F(s[0])) if keep[j] else 0)


def test_sparse_residual_at_zero_percent_is_the_dense_quantizer():
    r = np.random.default_rng(53).laplace(0, 0.02, 300)
    keep, q, s = oracle.sparsify_residual(r, 128, 0)
    q2, s2 = oracle.quantize_groups(r, 128)
    assert keep.all() and np.array_equal(q, q2) and np.array_equal(s, s2)


@pytest.mark.parametrize("Ps", [50, 70])
def test_sparse_residual_sparsity_and_output(Ps):
    """[P1] s3.3 quotes 50-70 % residual sparsity: on the stack's weights at
    least that share of the codes is zero (a few more round to zero); the
    output is the dense (trunk + sparse residual) weight times xhat."""
    L = wl.config2_layer(0, 1)
    W = L.weights()[:24]
    x = L.activations(M=2)
    idx = L.planted_channels()
    d = oracle.decompose_sparse(W, Ps=Ps)
    zero = float((d["q"] == 0).mean())
    assert Ps / 100 <= zero <= Ps / 100 + 0.1, zero
    xq, sx, xout = oracle.quantize_act(x, idx)
    xh = _xhat(x, xq, sx, idx)
    G = d["G"]
    res_hat = d["s"].astype(np.float64)[:, np.arange(W.shape[1]) // G] * d["q"].astype(np.float64)
    trunk_hat = d["mask"] * np.where(d["sign"] == 1, 1.0, -1.0) * d["alpha"].astype(np.float64)[:, None]
    y = oracle.linear(d, xq, sx, xout, idx)
    scale = np.abs(xh) @ (np.abs(res_hat) + np.abs(trunk_hat)).T
    assert np.all(np.abs(y - xh @ (trunk_hat + res_hat).T) <= 1e-12 * scale)


# ---- asymmetric residual groups ([P1] s2 pitfalls, [P3] asymmetric quantization) --

def _asym_groups(rng):
    """Groups of 32: centred, all positive, all negative, skewed, with an exact 0."""
    out = [rng.laplace(0, 0.02, 32), rng.uniform(0.1, 0.9, 32), -rng.uniform(0.1, 0.9, 32),
           np.concatenate([rng.uniform(-0.01, 0, 8), rng.uniform(0, 1, 24)])]
    g = rng.laplace(0, 0.02, 32)
    g[7] = 0.0
    out.append(g)
    return out


def test_asym_range_ends_and_zero_point():
    """The group minimum and maximum land on -128 and 127; an exact 0.0 in a
    group that straddles zero lands on the zero-point and dequantizes to 0."""
    rng = np.random.default_rng(61)
    for trial in range(40):
        for g in _asym_groups(rng):
            q, s, z = oracle.quantize_groups_asym(g, 32)
            assert q[int(np.argmin(g))] == -128 and q[int(np.argmax(g))] == 127
            for j in np.flatnonzero(g == 0.0):
                if g.min() <= 0.0 <= g.max():
                    assert q[j] == z[0] and (int(q[j]) - int(z[0])) * float(s[0]) == 0.0


def test_asym_range_example():
    """The pages' range [-7.59, 10.8]: s = (10.8 + 7.59) / 255, z = round(7.59/s - 128)
    = -23 (exact rational arithmetic on the binary32 s)."""
    r = np.zeros(32)
    r[0], r[1] = -7.59, 10.8
    q, s, z = oracle.quantize_groups_asym(r, 32)
    assert s[0] == np.float32((10.8 + 7.59) / 255.0)
    t = Fraction(7.59) / F(s[0]) - 128  # = -22.76...
    assert z[0] == -23 and abs(t - z[0]) < Fraction(1, 2)
    assert q[0] == -128 and q[1] == 127


def test_asym_codes_are_nearest_levels():
    """Each code is a nearest of the 256 levels (q - z) * s (brute force over
    rationals), and a constant group gives s = 0, z = 0, q = 0."""
    rng = np.random.default_rng(62)
    for g in _asym_groups(rng):
        q, s, z = oracle.quantize_groups_asym(g, 32)
        S, Z = F(s[0]), int(z[0])
        for v, c in zip(g, q):
            R = Fraction(float(v))
            best = min(abs(R - (k - Z) * S) for k in range(-128, 128))
            assert abs(R - (int(c) - Z) * S) == best
    q, s, z = oracle.quantize_groups_asym(np.full(32, 0.37), 32)
    assert s[0] == 0 and z[0] == 0 and not q.any()


def test_asym_halves_the_error_on_a_skewed_group():
    """[P3]: the asymmetric form fits a one-sided group better; on values in
    [0, 1] its step is (max - min)/255 against max/127."""
    g = np.random.default_rng(63).uniform(0, 1, 128)
    qa, sa, za = oracle.quantize_groups_asym(g, 128)
    qs, ss = oracle.quantize_groups(g, 128)
    ea = np.abs(g - (qa.astype(np.float64) - za[0]) * sa[0]).max()
    es = np.abs(g - qs.astype(np.float64) * ss[0]).max()
    assert ea <= 0.55 * es


@pytest.mark.parametrize("P", [-1, 60])
def test_asym_linear_is_the_dense_product(P):
    """y = sx*(alpha*T + sum_g s_g*(R_g - z_g*S_g)) + outliers equals the dense
    (trunk + (q - z)*s) weight times xhat, formed with numpy."""
    L = wl.config2_layer(0, 1)
    W = L.weights()[:24]
    x = L.activations(M=2)
    idx = L.planted_channels()
    d = oracle.decompose_asym(W, P=P)
    xq, sx, xout = oracle.quantize_act(x, idx)
    xh = _xhat(x, xq, sx, idx)
    g = np.arange(W.shape[1]) // d["G"]
    res_hat = d["s"].astype(np.float64)[:, g] * (d["q"].astype(np.float64) - d["z"][:, g])
    trunk_hat = d["mask"] * np.where(d["sign"] == 1, 1.0, -1.0) * d["alpha"].astype(np.float64)[:, None]
    y = oracle.linear_asym(d, xq, sx, xout, idx)
    scale = np.abs(xh) @ (np.abs(res_hat) + np.abs(trunk_hat)).T
    assert np.all(np.abs(y - xh @ (trunk_hat + res_hat).T) <= 1e-12 * scale)
    # and it stays within the symmetric residual's accuracy of the original product
    ref = x.astype(np.float64) @ W.astype(np.float64).T
    assert np.all(np.abs(y - ref) <= 0.05 * oracle.abs_dot(W, x))


# ---- calibration and activations ----------------------------------------------

def test_calibration_recovers_planted_channels():
    for L in (wl.config1(), wl.config2_layer(0, 0), wl.config2_layer(0, 3)):
        X = L.calibration()
        idx = oracle.calibrate(X, L.n_out)
        assert np.array_equal(idx, L.planted_channels())


def test_calibration_ties_and_library_order():
    X = np.array([[3.0, -5.0, 5.0, 1.0], [0.0, 2.0, -5.0, -1.0]], np.float32)
    assert oracle.calibrate(X, 1).tolist() == [1]
    assert oracle.calibrate(X, 2).tolist() == [1, 2]
    assert oracle.calibrate(X, 3).tolist() == [0, 1, 2]
    rng = np.random.default_rng(2)
    X = np.round(rng.standard_normal((16, 257)) * 4).astype(np.float32)  # many ties
    mag = np.abs(X).max(axis=0)
    order = np.lexsort((np.arange(257), -mag))
    for k in (1, 5, 40, 257):
        assert oracle.calibrate(X, k).tolist() == sorted(order[:k].tolist())


def test_activation_split():
    x = np.array([[1.0, -254.0, 0.5, 100.0, -0.25]], np.float32)
    xq, sx, xout = oracle.quantize_act(x, np.array([3], np.int32))
    assert sx[0] == np.float32(254.0 / 127.0)      # absmax without channel 3
    assert xq[0].tolist() == [1, -127, 0, 0, 0]     # 0.5/2 = 0.25 -> 0; -0.125 -> 0
    assert xout[0].tolist() == [100.0]
    xq, sx, xout = oracle.quantize_act(np.zeros((2, 7), np.float32), np.array([0], np.int32))
    assert np.all(sx == 0) and np.all(xq == 0)


def test_nonfinite_and_bad_arguments():
    W = np.ones((2, 40), np.float32)
    W[1, 3] = np.nan
    assert oracle.decompose(W, G=32)["status"] == 2
    with pytest.raises(oracle.OracleError):
        oracle.decompose(np.ones((1, 8), np.float32), G=32, P=0)
    with pytest.raises(oracle.OracleError):
        oracle.quantize_act(np.ones((1, 8), np.float32), np.array([3, 2], np.int32))
    with pytest.raises(oracle.OracleError):
        oracle.decompose(np.ones((1, 8), np.float32), G=48)


# ---- per-layer fallback to plain INT8 ---------------------------------------------

def test_fallback_errors_on_binary_rows():
    """Rows of +-c_r: the split is lossless (alpha = c_r, residual 0).  With
    c_r = 127 * 2^-e plain INT8 is lossless too (s = 2^-e exactly, codes
    +-127): both errors are exactly 0, the split gains nothing, and the rule
    falls back.  With c_r = 0.5 the plain scale 0.5/127 rounds, so plain
    INT8 leaves a small error and the split is kept."""
    rng = np.random.default_rng(21)
    signs = rng.choice([-1.0, 1.0], size=(3, 300))
    c = (127.0 * np.array([2.0 ** -8, 2.0 ** -10, 2.0 ** -6]))[:, None]
    W = (c * signs).astype(np.float32)
    assert oracle.layer_sq_error(oracle.decompose(W), W) == 0.0
    assert oracle.plain_sq_error(W) == 0.0
    assert oracle.choose_fallback(W)
    W2 = (0.5 * signs).astype(np.float32)
    assert oracle.layer_sq_error(oracle.decompose(W2), W2) == 0.0
    assert 0.0 < oracle.plain_sq_error(W2) < 1e-12
    assert not oracle.choose_fallback(W2)


def test_fallback_on_grid_aligned_weights():
    """Weights on every group's own INT8 grid (w = s_g * k, |k| <= 127, each
    group reaching 127): plain INT8 is exact, the split is not -> fall back."""
    rng = np.random.default_rng(22)
    N, K, G = 4, 256, 128
    k = rng.integers(-127, 128, size=(N, K))
    k[:, 0] = 127
    k[:, G] = -127
    sg = np.repeat(rng.uniform(1e-3, 1e-2, size=(N, K // G)), G, axis=1)
    W = (sg * k).astype(np.float32)
    # on the grid up to the rounding of s_g*k and of the quantizer's scale
    assert oracle.plain_sq_error(W) < 1e-12 * float((W.astype(np.float64) ** 2).sum())
    assert oracle.layer_sq_error(oracle.decompose(W), W) > 0.0
    assert oracle.choose_fallback(W)


def test_no_fallback_on_the_stack_weights():
    """Laplace weights of the 7B-shaped stack: the residual has the smaller
    range, so the split reconstructs W better and is kept."""
    for mid in range(4):
        W = wl.config2_layer(0, mid).weights(rows=np.arange(8))
        assert oracle.layer_sq_error(oracle.decompose(W), W) < oracle.plain_sq_error(W)
        assert not oracle.choose_fallback(W)


@pytest.mark.parametrize("P", [-1, 60])
def test_fallback_errors_second_route(P):
    """Second route with numpy: What formed from the decomposition's arrays,
    the squared error summed row by row (1e-12 relative); plain INT8 equals
    the split with an empty trunk (100th percentile) bit for bit."""
    rng = np.random.default_rng(23 + P)
    W = rng.laplace(0, 0.02, (7, 300)).astype(np.float32)
    d = oracle.decompose(W, P=P)
    G = 128
    s = np.repeat(d["s"].astype(np.float64), G, axis=1)[:, :300]
    what = d["mask"] * np.where(d["sign"] == 1, 1.0, -1.0) * d["alpha"].astype(np.float64)[:, None] \
        + s * d["q"].astype(np.float64)
    ref = float(((W.astype(np.float64) - what) ** 2).sum(axis=1).sum())
    assert abs(oracle.layer_sq_error(d, W) - ref) <= 1e-12 * ref
    assert oracle.plain_sq_error(W) == oracle.layer_sq_error(oracle.decompose(W, P=100), W)
    da = oracle.decompose_asym(W, P=P)
    sa = np.repeat(da["s"].astype(np.float64), G, axis=1)[:, :300]
    za = np.repeat(da["z"].astype(np.float64), G, axis=1)[:, :300]
    what_a = da["mask"] * np.where(da["sign"] == 1, 1.0, -1.0) * da["alpha"].astype(np.float64)[:, None] \
        + sa * (da["q"].astype(np.float64) - za)
    ref_a = float(((W.astype(np.float64) - what_a) ** 2).sum(axis=1).sum())
    assert abs(oracle.layer_sq_error(da, W) - ref_a) <= 1e-12 * ref_a


# ---- tolerance scale ------------------------------------------------------------

def test_abs_dot_closed_form():
    """sum_j |W_rj x_tj| on weights +-c and activations +-d with random signs
    is K*c*d exactly (every product and partial sum is exact in binary64)."""
    rng = np.random.default_rng(11)
    K, c, d = 37, 0.75, 1.5
    W = (c * rng.choice([-1.0, 1.0], size=(5, K))).astype(np.float32)
    x = (d * rng.choice([-1.0, 1.0], size=(3, K))).astype(np.float32)
    out = oracle.abs_dot(W, x)
    assert out.shape == (3, 5)
    assert np.all(out == K * c * d)


def test_abs_dot_hand_computed():
    """A 2 x 3 weight and two tokens, summed by hand: [[6, 4.5], [5.5, 5]]."""
    W = np.array([[1.0, -2.0, 3.0], [0.5, 0.0, -4.0]], np.float32)
    x = np.array([[1.0, 1.0, 1.0], [-2.0, 0.25, 1.0]], np.float32)
    assert np.array_equal(oracle.abs_dot(W, x), np.array([[6.0, 4.5], [5.5, 5.0]]))


def test_abs_dot_matches_absolute_matrix_product():
    """Second route: the product of the element-wise absolute values (numpy,
    binary64) on the stack's weights and activations, to 1e-12 relative."""
    L = wl.config2_layer(0, 1)
    W = L.weights(rows=np.arange(24))
    x = L.activations(M=2)
    ref = np.abs(x.astype(np.float64)) @ np.abs(W.astype(np.float64)).T
    got = oracle.abs_dot(W, x)
    assert np.allclose(got, ref, rtol=1e-12, atol=0.0)


def test_generator_statistics():
    """The synthetic inputs have the stated distributions (sanity, not a pin)."""
    W = wl.config1().weights()
    assert abs(np.abs(W).mean() - 0.02) < 0.0005          # Laplace mean |W| = b
    x = wl.config2_layer(0, 0).activations(M=64)
    planted = wl.config2_layer(0, 0).planted_channels()
    rest = np.delete(x, planted, axis=1)
    assert abs(rest.std() - 1.0) < 0.02
    assert abs(np.abs(x[:, planted]).mean() / np.abs(rest).mean() - 30.0) < 3.0
    L3 = wl.config3()[0]
    w3 = L3.weights(rows=np.arange(4))
    heavy = np.abs(w3) > 6 * 0.015
    assert 0.0003 < heavy.mean() < 0.003


# ---- NVFP4 prefill format -------------------------------------------------------
# The ISTA-DASLab page on separated quantization (paragraphs 2-4) names NVFP4
# as the prefill format without defining it; the pins below follow from the
# format's bit fields (E2M1: 1 sign, 2 exponent bits with bias 1, 1 mantissa
# bit; UE4M3: 4 exponent bits with bias 7, 3 mantissa bits, code 127 NaN),
# round-to-nearest-even and the two-level scale rule.

def _e2m1_from_fields(code):
    e, m = (code >> 1) & 3, code & 1
    mag = m * 0.5 if e == 0 else (1.0 + m / 2.0) * 2.0 ** (e - 1)
    return -mag if code & 8 else mag


def test_e2m1_values_follow_the_bit_fields():
    for c in range(16):
        assert oracle.e2m1_value(c) == _e2m1_from_fields(c), c
    assert sorted({abs(oracle.e2m1_value(c)) for c in range(16)}) == [0, 0.5, 1, 1.5, 2, 3, 4, 6]


def test_ue4m3_values_known_points_and_spacing():
    """1.0 at 0x38, 448 at 0x7E (largest finite), 2^-9 at 0x01, 2^-6 at 0x08
    (smallest normal); strictly increasing; 8 values per binade above it."""
    assert oracle.ue4m3_value(0x38) == 1.0
    assert oracle.ue4m3_value(0x7E) == 448.0
    assert oracle.ue4m3_value(0x01) == 2.0 ** -9
    assert oracle.ue4m3_value(0x08) == 2.0 ** -6
    assert oracle.ue4m3_value(0x07) == 7 * 2.0 ** -9
    v = [oracle.ue4m3_value(c) for c in range(127)]
    assert all(b > a for a, b in zip(v, v[1:]))
    for e in range(1, 15):
        assert sum(1 for x in v if 2.0 ** (e - 7) <= x < 2.0 ** (e - 6)) == 8


def _nearest_even(v, grid, codes):
    d = np.abs(np.asarray(grid) - v)
    best = np.flatnonzero(d == d.min())
    return [codes[i] for i in best if codes[i] % 2 == 0][0] if len(best) > 1 else codes[best[0]]


def test_e2m1_round_ties_saturation_and_brute_force():
    mags = [abs(_e2m1_from_fields(c)) for c in range(8)]
    # ties: to the even code (mantissa bit 0)
    for v, want in [(0.25, 0), (0.75, 2), (1.25, 2), (1.75, 4), (2.5, 4), (3.5, 6), (5.0, 6)]:
        assert oracle.e2m1_round(v) == want, v
        assert oracle.e2m1_round(-v) == (want | 8 if want else 0), -v
    assert oracle.e2m1_round(100.0) == 7 and oracle.e2m1_round(-6.01) == 15
    assert oracle.e2m1_round(-0.2) == 0 and oracle.e2m1_round(-0.0) == 0  # +0 for a zero result
    rng = np.random.default_rng(5)
    for v in np.concatenate([rng.uniform(-7, 7, 3000), np.array(mags), -np.array(mags)]):
        c = oracle.e2m1_round(float(v))
        want = _nearest_even(abs(v), mags, list(range(8)))
        assert c == (want | 8 if (v < 0 and want) else want), v


def test_ue4m3_round_ties_saturation_and_brute_force():
    vals = [oracle.ue4m3_value(c) for c in range(127)]
    rng = np.random.default_rng(6)
    pts = np.concatenate([np.exp(rng.uniform(np.log(2.0 ** -11), np.log(500.0), 3000)),
                          [(a + b) / 2 for a, b in zip(vals, vals[1:])], vals])
    for v in pts:
        assert oracle.ue4m3_round(float(v)) == _nearest_even(min(v, 1e9), vals, list(range(127))), v
    assert oracle.ue4m3_round(1000.0) == 126
    assert oracle.ue4m3_round(2.0 ** -10) == 0          # the tie between 0 and 2^-9
    assert oracle.ue4m3_round(1.0 + 1.0 / 16) == 0x38   # the tie between 1 and 1.125: even
    assert oracle.ue4m3_round(1.125 + 1.0 / 16) == 0x3A


def _exact_nvfp4_rows(rng, R, nb, g):
    """Rows whose every element is e2m1 * s_b * g exactly, each block holding
    +-6 * s_b * g, and block 0 holding 6 * 448 * g: the quantizer must
    reconstruct them exactly and find exactly these codes."""
    scode = rng.integers(8, 127, size=(R, nb))
    scode[:, 0] = 126
    codes = rng.integers(0, 16, size=(R, nb * 16))
    codes[codes == 8] = 0
    for r in range(R):
        for b in range(nb):
            j = 16 * b + rng.integers(0, 16)
            codes[r, j] = 7 | (8 * int(rng.integers(0, 2)))
    X = np.zeros((R, nb * 16), np.float64)
    for r in range(R):
        for j in range(nb * 16):
            X[r, j] = _e2m1_from_fields(codes[r, j]) * oracle.ue4m3_value(scode[r, j // 16]) * g[r]
    return X.astype(np.float32), codes.astype(np.uint8), scode.astype(np.uint8)


def test_nvfp4_exact_rows_reconstruct_exactly():
    rng = np.random.default_rng(7)
    g = 2.0 ** rng.integers(-12, -2, size=6)
    X, codes, scode = _exact_nvfp4_rows(rng, 6, 5, g)
    d = oracle.nvfp4_quantize(X, per_row=True)
    assert np.array_equal(d["g"], g.astype(np.float32))
    assert np.array_equal(d["scales"], scode)
    assert np.array_equal(d["codes"], codes)
    # per tensor: g is the largest row's, here the same for every row
    Xs = X[:1].repeat(3, axis=0)
    dt = oracle.nvfp4_quantize(Xs, per_row=False)
    assert dt["g"].shape == (1,) and dt["g"][0] == np.float32(g[0])
    assert np.array_equal(dt["codes"], codes[:1].repeat(3, axis=0))


def test_nvfp4_scale_rule_and_block_maximum():
    """g = float(amax / 2688) (per row, and per tensor = the largest row's);
    the block scale is the nearest UE4M3 to amax_b / (6 g); with a normal
    block scale the block's largest |x| gets the code of 6 (amax_b / (s_b g)
    lies within 6 * [1/(1+2^-4), 1/(1-2^-4)], nearer 6 than 4); every code is
    the nearest E2M1 level of x / (s_b g) (ties to even); a ragged last block
    (K = 40) and an all-zero row."""
    rng = np.random.default_rng(8)
    X = (rng.standard_normal((7, 40)) * np.exp(rng.uniform(-3, 3, (7, 1)))).astype(np.float32)
    X[:, 3] *= 20.0
    X[4] = 0.0
    d = oracle.nvfp4_quantize(X, per_row=True)
    dt = oracle.nvfp4_quantize(X, per_row=False)
    amax = np.abs(X.astype(np.float64)).max(axis=1)
    assert np.array_equal(d["g"], (amax / 2688.0).astype(np.float32))
    assert dt["g"][0] == np.float32(amax.max() / 2688.0)
    vals = [oracle.ue4m3_value(c) for c in range(127)]
    mags = [abs(_e2m1_from_fields(c)) for c in range(8)]
    for q, gg in ((d, d["g"].astype(np.float64)), (dt, np.full(7, float(dt["g"][0])))):
        assert q["scales"].shape == (7, 3)
        assert not q["codes"][4].any() and not q["scales"][4].any()
        for r in range(7):
            for b in range(3):
                blk = X[r, 16 * b: 16 * b + 16].astype(np.float64)
                if gg[r] == 0:
                    continue
                ab = np.abs(blk).max()
                sc = q["scales"][r, b]
                assert sc == _nearest_even(ab / (6.0 * gg[r]), vals, list(range(127)))
                step = vals[sc] * gg[r]
                if vals[sc] >= 2.0 ** -6:
                    assert q["codes"][r, 16 * b + int(np.abs(blk).argmax())] & 7 == 7
                for j, v in enumerate(blk):
                    c = int(q["codes"][r, 16 * b + j])
                    want = _nearest_even(abs(v) / step, mags, list(range(8))) if step else 0
                    assert c == (want | 8 if (v < 0 and want) else want)


def test_nvfp4_linear_exact_and_second_route():
    """Exact rows: y equals the exact dot products of the original values
    (Fraction arithmetic).  Random rows: y equals the dequantized operands
    (formed from the bit fields and scales in numpy) multiplied in binary64,
    to 1e-12 of sum |What * xhat|."""
    rng = np.random.default_rng(9)
    gw = np.full(4, 2.0 ** -7)
    Wx, _, _ = _exact_nvfp4_rows(rng, 4, 3, gw)
    gx = 2.0 ** rng.integers(-9, -4, size=3)
    Xx, _, _ = _exact_nvfp4_rows(rng, 3, 3, gx)
    w = oracle.nvfp4_quantize(Wx, per_row=False)
    x = oracle.nvfp4_quantize(Xx, per_row=True)
    y = oracle.nvfp4_linear(w, x)
    for t in range(3):
        for r in range(4):
            exact = sum(F(a) * F(b) for a, b in zip(Wx[r], Xx[t]))
            assert Fraction(y[t, r]) == exact
    L = wl.config2_layer(0, 0)
    W = L.weights(rows=np.arange(12))[:, :300]
    xa = L.activations(M=3)[:, :300]
    w = oracle.nvfp4_quantize(W, per_row=False)
    x = oracle.nvfp4_quantize(xa, per_row=True)
    y = oracle.nvfp4_linear(w, x)
    e2 = np.array([_e2m1_from_fields(c) for c in range(16)])
    u4 = np.array([oracle.ue4m3_value(c) for c in range(127)])
    Wh = e2[w["codes"]] * np.repeat(u4[w["scales"]], 16, axis=1)[:, :300] * float(w["g"][0])
    Xh = e2[x["codes"]] * np.repeat(u4[x["scales"]], 16, axis=1)[:, :300] * \
        x["g"].astype(np.float64)[:, None]
    ref = Xh @ Wh.T
    assert np.all(np.abs(y - ref) <= 1e-12 * (np.abs(Xh) @ np.abs(Wh).T))
    # and it stays near the unquantized product (4-bit elements: a loose bound)
    exact = xa.astype(np.float64) @ W.astype(np.float64).T
    assert np.all(np.abs(y - exact) <= 0.1 * (np.abs(xa.astype(np.float64)) @ np.abs(W.astype(np.float64)).T))
