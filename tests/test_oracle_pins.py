"""Pins for the CPU oracle, against what the pages and the mathematics fix.

None of these tests re-types the oracle's formulas: each checks the oracle
against hand-worked values (tests/golden/), an independent library (numpy's
binary16 conversion and float64 matmul), a closed form, a special case that
reduces to a plain matmul, or an invariant that a plausible mistake breaks
(a dropped term, a wrong sign or index, a transposed operand, a wrong scale).
"""
import math

import numpy as np
import pytest

import oracle
import workloads
from tests import _golden


# --------------------------------------------------------------------------
# binary16 codec, against numpy's independent implementation

def test_half_decode_exhaustive():
    h = np.arange(65536, dtype=np.uint16)
    mine = oracle.half_to_double(h)
    ref = h.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert (np.isnan(mine) == nan).all()
    assert (mine[~nan] == ref[~nan]).all()
    # signed zeros keep their sign
    assert math.copysign(1.0, mine[0x8000]) == -1.0


def test_half_encode_matches_numpy():
    rng = np.random.default_rng(7)
    finite = np.arange(0, 0x7c00, dtype=np.uint16).view(np.float16).astype(np.float64)
    mids = (finite[:-1] + finite[1:]) / 2.0            # exact ties, all ranges
    near = np.concatenate([mids, np.nextafter(mids, 0), np.nextafter(mids, np.inf)])
    rand = np.concatenate([
        rng.standard_normal(200_000) * 10.0 ** rng.uniform(-9, 5, 200_000),
        [0.0, -0.0, 65504.0, 65519.99, 65520.0, 65536.0, 1e9, -65520.0,
         2.0 ** -24, 2.0 ** -25, 2.0 ** -25 * 1.0000001, 3 * 2.0 ** -26, 2.0 ** -14,
         np.inf, -np.inf],
    ])
    v = np.concatenate([finite, -finite, near, -near, rand])
    mine = oracle.double_to_half(v)
    with np.errstate(over="ignore"):
        ref = v.astype(np.float16).view(np.uint16)
    assert (mine == ref).all(), v[mine != ref][:10]
    assert oracle.double_to_half(np.array([np.nan]))[0] & 0x7fff > 0x7c00


# --------------------------------------------------------------------------
# step 1: the outlier test at the threshold (hand-made fixture)

def test_outlier_threshold_golden():
    g = _golden.read("outlier_threshold.txt")
    X = g["X"].astype(np.float16)
    assert (X.astype(np.float64) == g["X"]).all()   # fixture values are exact fp16
    colmax, idx = oracle.outlier_columns(X, float(g["alpha"][0]))
    assert idx.tolist() == g["outliers"].astype(int).tolist()
    assert (colmax == np.abs(g["X"]).max(axis=0)).all()


def test_outlier_is_per_column_not_per_row():
    # one large row spread over many columns must not flag those columns
    # unless an entry exceeds alpha; a single large entry flags its column.
    X = np.zeros((4, 16), np.float16)
    X[1, :] = 5.5
    X[2, 11] = -100
    _, idx = oracle.outlier_columns(X, 6.0)
    assert idx.tolist() == [11]
    _, idx = oracle.outlier_columns(X.T.copy(), 6.0)   # transposed: column 2 only
    assert idx.tolist() == [2]


# --------------------------------------------------------------------------
# steps 1-5 on the hand-worked example

def test_hand_example_golden():
    g = _golden.read("hand_example_m2_k4_n3.txt")
    X = g["X"].astype(np.float16)
    W = g["W"].astype(np.float16)
    assert (X.astype(np.float64) == g["X"]).all() and (W.astype(np.float64) == g["W"]).all()
    r = oracle.decomp_matmul(X, W, float(g["alpha"][0]))
    assert r["idx"].tolist() == g["outliers"].astype(int).tolist()
    assert (r["c_x"] == g["c_x"].astype(np.float32)).all()
    assert (r["qx"] == g["qx"]).all()
    assert (r["c_w"] == g["c_w"].astype(np.float32)).all()
    assert (r["qw"] == g["qw"]).all()
    assert (r["acc"] == g["acc"]).all()
    assert (r["Y"].astype(np.float64) == g["Y"]).all(), (r["Y"], g["Y"])


def test_round_half_to_even_and_clamp():
    q = oracle.quantize_value
    # products that are exact halves go to the even neighbour
    assert [q(2.5, 1.0), q(3.5, 1.0), q(-2.5, 1.0), q(0.5, 1.0), q(-0.5, 1.0)] == [2, 4, -2, 0, 0]
    assert [q(126.5, 1.0), q(-126.5, 1.0)] == [126, -126]
    # never outside [-127, 127] (the page's -128 is never produced)
    assert [q(127.5, 1.0), q(128.0, 1.0), q(-128.0, 1.0), q(-1000.0, 1.0)] == [127, 127, -127, -127]
    # the fp32 product is rounded before the integer rounding:
    # 0.0390625 * 64 = 2.5 exactly -> 2
    assert q(0.0390625, 64.0) == 2
    assert oracle.scale_from_absmax(0.0) == 0.0
    assert oracle.scale_from_absmax(2.0) == np.float32(63.5)
    assert oracle.scale_from_absmax(127.0 / 64.0) == np.float32(64.0)


# --------------------------------------------------------------------------
# T1: in every quantised vector the absmax element maps to +-127

def _check_absmax_maps_to_127(vals, codes, mask):
    # vals [n, L] float, codes [n, L] int8, mask [L] bool of included entries
    for v, c in zip(vals, codes):
        a = np.abs(v) * mask
        if a.max() == 0:
            assert (c == 0).all()
            continue
        j = int(np.argmax(a))
        assert abs(int(c[j])) == 127 and np.sign(c[j]) == np.sign(v[j])
        assert np.abs(c).max() <= 127


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_T1_absmax_element_maps_to_127(seed):
    p = workloads.small(37, 96, 40, 3, seed)
    r = oracle.decomp_matmul(p.X, p.W, p.alpha)
    K = p.X.shape[1]
    mask = np.ones(K, bool)
    mask[r["idx"]] = False
    assert set(r["idx"].tolist()) == set(p.planted.tolist())
    _check_absmax_maps_to_127(p.X.astype(np.float64), r["qx"], mask)
    assert (r["qx"][:, r["idx"]] == 0).all()
    _check_absmax_maps_to_127(p.W.astype(np.float64).T, r["qw"].T, np.ones(K, bool))


# --------------------------------------------------------------------------
# T2: alpha = inf is pure vector-wise int8, within its rounding bound

def test_T2_alpha_inf_is_vectorwise_within_bound():
    p = workloads.small(24, 128, 33, 0, 11, alpha=math.inf)
    r = oracle.decomp_matmul(p.X, p.W, math.inf)
    assert r["idx"].size == 0
    x = p.X.astype(np.float64)
    w = p.W.astype(np.float64)
    exact = x @ w                                   # numpy, independent
    # x = (q_x + e_x)/c_x with |e_x| <= 1/2 (+ fp32 product rounding), same for w:
    # |x.w - acc/(c_x c_w)| <= sum_k (|q_x| |e_w| + |e_x| |q_w| + |e_x e_w|) / (c_x c_w)
    e = 0.5 + 128 * 2.0 ** -24
    qx = np.abs(r["qx"].astype(np.float64))
    qw = np.abs(r["qw"].astype(np.float64))
    bound = (qx @ np.full_like(qw, e) + np.full_like(qx, e) @ qw + e * e * x.shape[1])
    bound /= np.outer(r["c_x"].astype(np.float64), r["c_w"].astype(np.float64))
    err = np.abs(r["Y_exact"] - exact)
    assert (err <= bound * (1 + 1e-9) + 1e-12).all()
    # the bound means something: it sits below the signal, and the actual
    # error is far below it (rounding errors partly cancel over K)
    assert np.median(bound) < 0.5 * np.median(np.abs(exact))
    assert np.linalg.norm(err) < 0.02 * np.linalg.norm(exact)


# --------------------------------------------------------------------------
# T3: alpha = 0 sends every non-zero column to fp16: an exact matmul

def test_T3_alpha_zero_is_exact_fp16_matmul():
    rng = np.random.default_rng(3)
    M, K, N = 9, 40, 17
    # multiples of 2^-6 in [-4, 4): every partial sum is exact in double
    X = (rng.integers(-256, 256, (M, K)) / 64.0).astype(np.float16)
    W = (rng.integers(-256, 256, (K, N)) / 64.0).astype(np.float16)
    X[:, 5] = 0                                     # an all-zero column stays int8
    r = oracle.decomp_matmul(X, W, 0.0)
    assert 5 not in r["idx"].tolist() and r["idx"].size == K - 1
    assert (r["c_x"] == 0).all() and (r["qx"] == 0).all() and (r["acc"] == 0).all()
    ref = (X.astype(np.float64) @ W.astype(np.float64)).astype(np.float16)
    assert (r["Y"].view(np.uint16) == ref.view(np.uint16)).all()


def test_T3_with_bias_adds_before_the_single_rounding():
    # the layer's bias (gartu "Exemple pratique": the int8 layer replacing
    # nn.Linear keeps its bias) joins the exact double sum before the one
    # fp16 rounding: with alpha = 0 the result is fp16(X W + b) bit for bit
    rng = np.random.default_rng(33)
    M, K, N = 9, 40, 17
    X = (rng.integers(-256, 256, (M, K)) / 64.0).astype(np.float16)
    W = (rng.integers(-256, 256, (K, N)) / 64.0).astype(np.float16)
    b = (rng.integers(-4096, 4096, N) / 1024.0 + 1.0 / 4096).astype(np.float16)
    r = oracle.decomp_matmul(X, W, 0.0, bias=b)
    exact = X.astype(np.float64) @ W.astype(np.float64) + b.astype(np.float64)
    assert (r["Y"].view(np.uint16) == exact.astype(np.float16).view(np.uint16)).all()
    assert (r["Y_exact"] == exact).all()
    # and with alpha = inf the bias shifts the unrounded value by exactly b
    r0 = oracle.decomp_matmul(X, W, np.inf)
    r1 = oracle.decomp_matmul(X, W, np.inf, bias=b)
    assert np.allclose(r1["Y_exact"] - r0["Y_exact"], b.astype(np.float64)[None, :], rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# T5: the pages' worked example (estelledc 案例1): 7 outlier channels among
# ordinary ones destroy tensor-wise absmax resolution but not the decomposition

@pytest.mark.parametrize("K", [4102, 4096])
def test_T5_worked_example(K):
    p = workloads.worked_example(K=K, M=256, N=64)
    normal = np.ones(K, bool)
    normal[p.planted] = False
    xa = np.abs(p.X.astype(np.float64))
    # the workload matches the page's statistics
    assert abs(xa[:, normal].mean() - 0.5) < 0.02 and xa[:, normal].max() <= 5.0
    assert xa[:, p.planted].max() == 130.0
    tw = oracle.tensorwise_absmax(p.X, p.W)
    step = 1.0 / float(tw["c_x"])
    assert 1.0 <= step <= 1.03                      # "each step is ~1.0"
    small = np.isin(tw["qx"][:, normal], (-1, 0, 1)).mean()
    assert small > 0.95                             # "squashed to 0 or 1"
    r = oracle.decomp_matmul(p.X, p.W, 6.0)
    assert set(r["idx"].tolist()) == set(p.planted.tolist())
    exact = oracle.matmul_f64(p.X, p.W)
    fro = lambda y: np.linalg.norm(y.astype(np.float64) - exact) / np.linalg.norm(exact)
    e_dec, e_tw = fro(r["Y"]), fro(tw["Y"])
    assert e_dec * 10 < e_tw, (e_dec, e_tw)
    # with the decomposition the ordinary channels keep a real int8 range
    assert np.isin(r["qx"][:, normal], (-1, 0, 1)).mean() < 0.2


# --------------------------------------------------------------------------
# T6: the int32 accumulator bound |acc| <= K * 127^2 holds and is reached

def test_T6_accumulator_bound_reached():
    K = 1024
    X = np.full((2, K), 2.0, np.float16)
    X[1] = -2.0
    W = np.full((K, 3), 0.5, np.float16)
    r = oracle.decomp_matmul(X, W, math.inf)
    assert (r["acc"][0] == K * 127 * 127).all() and (r["acc"][1] == -K * 127 * 127).all()
    assert np.allclose(r["Y"].astype(np.float64), X.astype(np.float64) @ W.astype(np.float64))


# --------------------------------------------------------------------------
# T7: W = identity isolates the outer-product dequantisation

def test_T7_identity_weight():
    p = workloads.small(12, 64, 64, 2, 5)
    W = np.eye(64, dtype=np.float16)
    r = oracle.decomp_matmul(p.X, W, 6.0)
    assert (r["c_w"] == np.float32(127.0)).all()
    x = p.X.astype(np.float64)
    y = r["Y"].astype(np.float64)
    # outlier columns pass through the fp16 path exactly
    assert (y[:, r["idx"]] == x[:, r["idx"]]).all()
    # ordinary columns are x up to half an int8 step of that row, plus fp16 rounding
    normal = np.setdiff1d(np.arange(64), r["idx"])
    step = 1.0 / r["c_x"].astype(np.float64)
    tol = 0.5 * step[:, None] * (1 + 1e-6) + np.abs(x[:, normal]) * 2.0 ** -11
    assert (np.abs(y[:, normal] - x[:, normal]) <= tol).all()


# --------------------------------------------------------------------------
# invariants that catch index, scale and operand mix-ups

def test_joint_permutation_of_K_leaves_Y_unchanged():
    p = workloads.small(20, 128, 24, 4, 21)
    perm = np.random.default_rng(0).permutation(128)
    a = oracle.decomp_matmul(p.X, p.W, 6.0)
    b = oracle.decomp_matmul(np.ascontiguousarray(p.X[:, perm]),
                             np.ascontiguousarray(p.W[perm, :]), 6.0)
    assert (a["acc"] == b["acc"]).all()
    assert (a["c_x"] == b["c_x"]).all() and (a["c_w"] == b["c_w"]).all()
    # the outlier terms are summed in another order: at most 1 fp16 ulp apart
    ua, ub = a["Y"].view(np.int16).astype(np.int64), b["Y"].view(np.int16).astype(np.int64)
    assert np.abs(ua - ub).max() <= 1
    assert sorted(perm[b["idx"]].tolist()) == a["idx"].tolist()


def test_power_of_two_scaling_of_a_row_and_a_column():
    p = workloads.small(8, 64, 16, 2, 31)
    base = oracle.decomp_matmul(p.X, p.W, 6.0)
    X2 = p.X.copy()
    X2[3] = X2[3] * np.float16(0.5)      # outlier entries stay > 6 (>= 10)
    r = oracle.decomp_matmul(X2, p.W, 6.0)
    assert (r["idx"] == base["idx"]).all()
    assert (r["qx"] == base["qx"]).all()
    assert r["c_x"][3] == 2 * base["c_x"][3]
    assert (r["Y"][3].astype(np.float64) == base["Y"][3].astype(np.float64) * 0.5).all()
    W2 = p.W.copy()
    W2[:, 7] = W2[:, 7] * np.float16(2.0)
    r = oracle.decomp_matmul(p.X, W2, 6.0)
    assert (r["qw"] == base["qw"]).all() and r["c_w"][7] == base["c_w"][7] / 2
    assert (r["Y"][:, 7].astype(np.float64) == base["Y"][:, 7].astype(np.float64) * 2).all()
    others = np.arange(16) != 7
    assert (r["Y"][:, others] == base["Y"][:, others]).all()


def test_zero_row_and_zero_column():
    p = workloads.small(6, 48, 10, 1, 41)
    X = p.X.copy()
    X[2, :] = 0
    W = p.W.copy()
    W[:, 4] = 0
    r = oracle.decomp_matmul(X, W, 6.0)
    assert r["c_x"][2] == 0 and (r["qx"][2] == 0).all()
    assert r["c_w"][4] == 0 and (r["qw"][:, 4] == 0).all()
    assert (r["Y"][2].astype(np.float64) == 0).all()
    assert (r["Y"][:, 4].astype(np.float64) == 0).all()


def test_outlier_row_of_W_is_multiplied_by_zero_codes():
    # changing W only in an outlier row moves Y only through the fp16 term
    p = workloads.small(10, 64, 12, 1, 51)
    j = int(p.planted[0])
    base = oracle.decomp_matmul(p.X, p.W, 6.0)
    W2 = p.W.copy()
    W2[j, 3] = np.float16(0.001)
    r = oracle.decomp_matmul(p.X, W2, 6.0)
    ex = r["Y_exact"][:, 3] - base["Y_exact"][:, 3]
    # c_w of column 3 may change (its absmax may have been in row j), but the
    # change in Y is close to X[:, j] * (W2[j,3] - W[j,3]) plus int8 requantisation
    d = p.X[:, j].astype(np.float64) * (float(W2[j, 3]) - float(p.W[j, 3]))
    assert np.abs(ex - d).max() < 0.05 * np.abs(d).max() + 0.02


# --------------------------------------------------------------------------
# the two comparators the harness reports errors against

def test_matmul_f64_matches_numpy():
    rng = np.random.default_rng(8)
    X = (rng.integers(-512, 512, (7, 33)) / 128.0).astype(np.float16)
    W = (rng.integers(-512, 512, (33, 5)) / 128.0).astype(np.float16)
    ref = X.astype(np.float64) @ W.astype(np.float64)   # exact: small dyadic values
    assert (oracle.matmul_f64(X, W) == ref).all()


def test_tensorwise_absmax_hand_example():
    # one scale for all of X (127/8) and one for all of W (127/2), no split:
    # X = [[8, 1], [-4, 0.5]] -> codes [[127, 15.875->16], [-63.5->-64, 7.9375->8]]
    # W = [[2, -1], [0.5, 1]]  -> codes [[127, -63.5->-64], [31.75->32, 63.5->64]]
    X = np.array([[8, 1], [-4, 0.5]], np.float16)
    W = np.array([[2, -1], [0.5, 1]], np.float16)
    r = oracle.tensorwise_absmax(X, W)
    assert r["c_x"] == np.float32(127 / 8) and r["c_w"] == np.float32(63.5)
    assert r["qx"].tolist() == [[127, 16], [-64, 8]]
    assert r["qw"].tolist() == [[127, -64], [32, 64]]
    # acc row 0: [127*127 + 16*32, 127*-64 + 16*64] = [16641, -7104]
    # y = acc / (15.875 * 63.5) = acc / 1008.0625 -> [16.5078.., -7.0472..]
    acc = np.array([[16641, -7104], [-64 * 127 + 8 * 32, -64 * -64 + 8 * 64]], np.float64)
    assert (r["Y"].astype(np.float64) == (acc / (15.875 * 63.5)).astype(np.float16)).all()


# --------------------------------------------------------------------------
# memory-saving weight: rows outside the stored set rebuilt from the codes

def test_rebuilt_weight_rows_exact_on_the_code_grid():
    # columns whose entries lie on their own code grid (absmax / 127 apart)
    # come back exactly: absmax 63.5 (c_w = 2), 127 (c_w = 1), 254 (c_w = 0.5).
    # A scale applied the wrong way (q * c_w) or not at all fails the first
    # and the last column.
    rng = np.random.default_rng(3)
    q = rng.integers(-127, 128, size=(40, 3))
    q[0] = [127, -127, 127]  # every column reaches its absmax
    W = (q * np.array([0.5, 1.0, 2.0])).astype(np.float16)
    qw, c_w = oracle.quantize_cols(W)
    assert c_w.tolist() == [2.0, 1.0, 0.5]
    assert (qw == q).all()
    assert (oracle.rebuild_weight_rows(qw, c_w) == W).all()


def test_rebuilt_weight_rows_within_half_a_code_step():
    # |w~ - w| <= absmax / 254 (half a code step, up to fp32 rounding of the
    # product) + half an fp16 ulp of w~; an all-zero column rebuilds to zeros
    rng = np.random.default_rng(4)
    W = (rng.standard_normal((64, 9)) * 0.02).astype(np.float16)
    W[:, 4] = 0
    qw, c_w = oracle.quantize_cols(W)
    Wr = oracle.rebuild_weight_rows(qw, c_w)
    absmax = np.abs(W.astype(np.float64)).max(axis=0)
    err = np.abs(Wr.astype(np.float64) - W.astype(np.float64))
    bound = absmax / 254 * (1 + 1e-6) + np.spacing(np.abs(Wr)).astype(np.float64) / 2
    assert (err <= bound).all()
    assert (Wr[:, 4] == 0).all() and c_w[4] == 0
    assert err.max() > 0  # the rebuilt rows are the quantised weight, not W


def test_static_weight_keeps_the_stored_rows():
    rng = np.random.default_rng(5)
    W = (rng.standard_normal((12, 7)) * 0.05).astype(np.float16)
    qw, c_w = oracle.quantize_cols(W)
    Ws = oracle.static_weight(W, qw, c_w, [1, 5])
    Wr = oracle.rebuild_weight_rows(qw, c_w)
    assert (Ws[[1, 5]] == W[[1, 5]]).all()
    others = [k for k in range(12) if k not in (1, 5)]
    assert (Ws[others] == Wr[others]).all()
