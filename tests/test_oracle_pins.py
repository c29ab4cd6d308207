"""Pins for the CPU oracle: each check compares the oracle with something other
than itself -- a hand-worked example (tests/golden), a library routine for a
special case, a closed form, an identity of the mathematics, or brute force
over every mask of a tiny layer.  A final test plants plausible mistakes in a
copy of the oracle's C source and checks that some pin rejects each one."""
import itertools
import math
import os
import shutil
import subprocess
import tempfile
from fractions import Fraction

import numpy as np
import pytest

import oracle
from golden_io import ints, mat, read

# ----------------------------------------------------------------------------
# element decoding


def test_half_decode_matches_numpy_for_every_bit_pattern():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.half_to_double(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    # signed zeros keep their sign
    assert math.copysign(1.0, oracle.half_to_double(0x8000)) == -1.0


def test_q4_0_golden_row():
    g = read("q4_0_blocks.txt")
    sc = np.array([int(x, 16) for x in g["scales"].split()], dtype=np.uint16).view(np.float16).reshape(1, -1)
    qs = np.array([int(x, 16) for x in g["qs"].split()], dtype=np.uint8).reshape(1, -1)
    x = mat(g["x"])
    got = oracle.decode_matrix((qs, sc), d=x.size)[0]
    assert np.array_equal(got, x)


# ----------------------------------------------------------------------------
# predictor


def _pred_golden():
    g = read("predictor_d3_r2.txt")
    P1 = mat(g["P1"]).astype(np.float32)
    P2 = mat(g["P2"]).astype(np.float32)
    bp = mat(g["bp"]).astype(np.float32)
    h = mat(g["h"]).astype(np.float32)
    return g, P1, P2, bp, h


def test_predictor_golden_per_token_and_union():
    g, P1, P2, bp, h = _pred_golden()
    thr, n_hot, ffn = float(g["thr"]), int(g["n_hot"]), int(g["ffn"])
    u, s = mat(g["u"]), mat(g["s"])
    for b, key in ((0, "idx_A"), (1, "idx_B")):
        r = oracle.predict(h[b:b + 1], P1, P2, bp, thr, n_hot, ffn)
        assert np.array_equal(r["u"][0], u[b])
        assert np.array_equal(r["s"][0], s[b])
        assert r["idx"].tolist() == ints(g[key])
    r = oracle.predict(h, P1, P2, bp, thr, n_hot, ffn)
    assert r["idx"].tolist() == ints(g["idx_AB"])
    assert r["mask"].tolist() == [1, 1, 0]


def test_predictor_threshold_is_strict_and_bias_optional():
    g, P1, P2, bp, h = _pred_golden()
    n_hot, ffn = int(g["n_hot"]), int(g["ffn"])
    # with thr just below the tied scores, the ties become active
    r = oracle.predict(h[:1], P1, P2, bp, 0.5 - 1e-9, n_hot, ffn)
    assert r["idx"].tolist() == [2, 3, 4]
    # no bias: s = P2 u = [3, -3, 1.5] for token A
    r = oracle.predict(h[:1], P1, P2, None, 0.5, n_hot, ffn)
    assert r["s"][0].tolist() == [3.0, -3.0, 1.5]
    assert r["idx"].tolist() == [2, 4]


def _lowrank_predictor(rng, d, rank, n_cold):
    rh = rank // 2
    U = rng.standard_normal((n_cold, rh))
    V = rng.standard_normal((rh, d)) / math.sqrt(d)
    P1 = np.concatenate([V, -V], 0).astype(np.float32)
    P2 = np.concatenate([U, -U], 1).astype(np.float32)
    return P1, P2


def test_predictor_lowrank_identity():
    """With P1 = [V; -V] and P2 = [U, -U], ReLU(x) - ReLU(-x) = x gives
    s = U (V h) + bp exactly in real arithmetic."""
    rng = np.random.default_rng(3)
    d, rank, n_hot, ffn = 48, 16, 5, 40
    P1, P2 = _lowrank_predictor(rng, d, rank, ffn - n_hot)
    V = P1[: rank // 2].astype(np.float64)
    U = P2[:, : rank // 2].astype(np.float64)
    bp = rng.standard_normal(ffn - n_hot).astype(np.float32)
    h = rng.standard_normal((3, d)).astype(np.float32)
    r = oracle.predict(h, P1, P2, bp, 0.5, n_hot, ffn)
    want = (U @ (V @ h.astype(np.float64).T)).T + bp.astype(np.float64)
    assert np.allclose(r["s"], want, rtol=0, atol=1e-12 * np.abs(want).max())


def test_predictor_compaction_invariants_and_union():
    rng = np.random.default_rng(4)
    d, rank, n_hot, ffn = 40, 12, 7, 97
    P1, P2 = _lowrank_predictor(rng, d, rank, ffn - n_hot)
    bp = (rng.standard_normal(ffn - n_hot) * 0.5).astype(np.float32)
    h = rng.standard_normal((4, d)).astype(np.float32)
    blk = oracle.predict(h, P1, P2, bp, 0.5, n_hot, ffn)
    idx, mask = blk["idx"], blk["mask"]
    assert len(idx) == int(mask.sum())
    assert np.all(np.diff(idx) > 0) and (len(idx) == 0 or (idx[0] >= n_hot and idx[-1] < ffn))
    assert np.array_equal(np.nonzero(mask)[0] + n_hot, idx)
    union = np.zeros(ffn - n_hot, bool)
    for b in range(4):
        one = oracle.predict(h[b:b + 1], P1, P2, bp, 0.5, n_hot, ffn)
        assert np.array_equal(one["s"][0], blk["s"][b])
        union |= one["mask"].astype(bool)
    assert np.array_equal(union, mask.astype(bool))


# ----------------------------------------------------------------------------
# masked FFN


def _golden_ffn(name):
    g = read(name)
    W = {k: (mat(g[k]).astype(np.float32) if k in g else None) for k in ("Wg", "Wu", "WdT")}
    return g, W, mat(g["b1"]).astype(np.float32), mat(g["b2"]).astype(np.float32), mat(g["h"]).astype(np.float32)


@pytest.mark.parametrize("mask", [[], [1], [2], [1, 2]])
def test_ffn_reglu_golden(mask):
    g, W, b1, b2, h = _golden_ffn("ffn_reglu_d2_f3.txt")
    key = "y[%s]" % ",".join(map(str, mask))
    y = oracle.masked_ffn(h, mask, W["Wg"], W["Wu"], W["WdT"], b1, b2, "reglu", int(g["n_hot"]), int(g["ffn"]))
    assert np.array_equal(y, mat(g[key]))
    # every token of the block uses the same list: one token alone gives the same rows
    for b in range(2):
        y1 = oracle.masked_ffn(h[b:b + 1], mask, W["Wg"], W["Wu"], W["WdT"], b1, b2, "reglu", 1, 3)
        assert np.array_equal(y1[0], mat(g[key])[b])


@pytest.mark.parametrize("act", ["relu", "relu2"])
@pytest.mark.parametrize("mask", [[], [1], [2], [1, 2]])
def test_ffn_relu_family_golden(act, mask):
    g, W, b1, b2, h = _golden_ffn("ffn_relu_d2_f3.txt")
    key = "%s y[%s]" % (act, ",".join(map(str, mask)))
    y = oracle.masked_ffn(h, mask, None, W["Wu"], W["WdT"], b1, b2, act, int(g["n_hot"]), int(g["ffn"]))
    assert np.array_equal(y, mat(g[key]))


def test_true_support_golden():
    g, W, b1, _, h = _golden_ffn("ffn_reglu_d2_f3.txt")
    assert np.array_equal(oracle.true_support(h, W["Wg"], W["Wu"], b1, "reglu", 3), mat(g["support"]))
    g, W, b1, _, h = _golden_ffn("ffn_relu_d2_f3.txt")
    assert np.array_equal(oracle.true_support(h, None, W["Wu"], b1, "relu", 3), mat(g["support"]))


def _rand_layer(rng, d, ffn, act, wtype, integer=False):
    def m(rows):
        if integer:
            x = rng.integers(-3, 4, size=(rows, d)) * (rng.random((rows, d)) < 0.3)
            return x.astype(np.float32)
        return (rng.standard_normal((rows, d)) / math.sqrt(d)).astype(np.float32)

    Wg = m(ffn) if act == "reglu" else None
    Wu, WdT = m(ffn), m(ffn)
    if integer:
        b1 = rng.integers(-2, 3, size=ffn).astype(np.float32)
        b2 = rng.integers(-2, 3, size=d).astype(np.float32)
    else:
        b1 = (rng.standard_normal(ffn) * 0.7 - 0.5).astype(np.float32)
        b2 = (rng.standard_normal(d) * 0.1).astype(np.float32)
    if wtype == "f16":
        Wg = None if Wg is None else Wg.astype(np.float16)
        Wu, WdT = Wu.astype(np.float16), WdT.astype(np.float16)
    return Wg, Wu, WdT, b1, b2


def _tokens(rng, B, d, integer=False):
    if integer:
        return rng.integers(-2, 3, size=(B, d)).astype(np.float32)
    h = rng.standard_normal((B, d))
    return (h * math.sqrt(d) / np.linalg.norm(h, axis=1, keepdims=True)).astype(np.float32)


@pytest.mark.parametrize("act", ["relu", "reglu", "relu2"])
@pytest.mark.parametrize("wtype", ["f32", "f16"])
def test_dense_equals_all_ones_mask_and_true_support_is_exact(act, wtype):
    """With the mask forced to all-ones the masked FFN is the dense FFN; with
    the mask equal to the true ReLU support the skipped terms are exact zeros,
    so the output is bit-identical to the dense one."""
    rng = np.random.default_rng(11)
    d, ffn, n_hot, B = 64, 50, 6, 3
    Wg, Wu, WdT, b1, b2 = _rand_layer(rng, d, ffn, act, wtype)
    h = _tokens(rng, B, d)
    dense = oracle.dense_ffn(h, Wg, Wu, WdT, b1, b2, act, n_hot, ffn)
    allm = oracle.masked_ffn(h, np.arange(n_hot, ffn), Wg, Wu, WdT, b1, b2, act, n_hot, ffn)
    assert np.array_equal(dense, allm)
    sup = oracle.true_support(h, Wg, Wu, b1, act, ffn)
    union = np.nonzero(sup.any(axis=0)[n_hot:])[0] + n_hot
    assert 0 < len(union) < ffn - n_hot
    y = oracle.masked_ffn(h, union, Wg, Wu, WdT, b1, b2, act, n_hot, ffn)
    assert np.array_equal(y, dense)
    # dropping any one supported neuron changes the output
    j = union[len(union) // 2]
    y2 = oracle.masked_ffn(h, union[union != j], Wg, Wu, WdT, b1, b2, act, n_hot, ffn)
    assert not np.array_equal(y2, dense)


def _exact_layer_output(h, Wg, Wu, WdT, b1, b2, act, listed):
    """Brute force in exact rational arithmetic, one neuron at a time."""
    B, d = h.shape
    out = []
    for b in range(B):
        hb = [Fraction(float(x)) for x in h[b]]
        y = [Fraction(float(x)) for x in b2]
        for j in listed:
            if act == "reglu":
                g = sum((Fraction(float(Wg[j, i])) * hb[i] for i in range(d)), Fraction(0)) + Fraction(float(b1[j]))
                v = sum((Fraction(float(Wu[j, i])) * hb[i] for i in range(d)), Fraction(0))
                a = max(g, Fraction(0)) * v
            else:
                z = sum((Fraction(float(Wu[j, i])) * hb[i] for i in range(d)), Fraction(0)) + Fraction(float(b1[j]))
                a = max(z, Fraction(0))
                if act == "relu2":
                    a = a * a
            for e in range(d):
                y[e] += a * Fraction(float(WdT[j, e]))
        out.append([float(v) for v in y])
    return np.array(out)


@pytest.mark.parametrize("act", ["relu", "reglu", "relu2"])
def test_brute_force_every_mask_of_a_tiny_layer(act):
    """d = 6, ffn = 10, n_hot = 3: for all 2^7 cold masks the oracle equals an
    exact rational evaluation, and the output is additive over neurons:
    y(M) = y(empty) + sum_{j in M} (y({j}) - y(empty))."""
    rng = np.random.default_rng(5)
    d, ffn, n_hot, B = 6, 10, 3, 2
    Wg, Wu, WdT, b1, b2 = _rand_layer(rng, d, ffn, act, "f32", integer=True)
    h = _tokens(rng, B, d, integer=True)
    cold = list(range(n_hot, ffn))
    y0 = oracle.masked_ffn(h, [], Wg, Wu, WdT, b1, b2, act, n_hot, ffn)
    single = {j: oracle.masked_ffn(h, [j], Wg, Wu, WdT, b1, b2, act, n_hot, ffn) - y0 for j in cold}
    assert np.array_equal(y0, _exact_layer_output(h, Wg, Wu, WdT, b1, b2, act, range(n_hot)))
    for k in range(len(cold) + 1):
        for M in itertools.combinations(cold, k):
            y = oracle.masked_ffn(h, list(M), Wg, Wu, WdT, b1, b2, act, n_hot, ffn)
            want = y0 + sum((single[j] for j in M), np.zeros_like(y0))
            assert np.array_equal(y, want), M
    full = _exact_layer_output(h, Wg, Wu, WdT, b1, b2, act, range(ffn))
    assert np.array_equal(oracle.dense_ffn(h, Wg, Wu, WdT, b1, b2, act, n_hot, ffn), full)


def test_brute_force_predictor_every_neuron():
    rng = np.random.default_rng(6)
    d, rank, n_hot, ffn = 7, 4, 2, 12
    P1 = rng.integers(-2, 3, size=(rank, d)).astype(np.float32)
    P2 = rng.integers(-2, 3, size=(ffn - n_hot, rank)).astype(np.float32)
    bp = (rng.integers(-3, 3, size=ffn - n_hot) + 0.5).astype(np.float32)
    h = rng.integers(-2, 3, size=(3, d)).astype(np.float32)
    r = oracle.predict(h, P1, P2, bp, 0.25, n_hot, ffn)
    act = set()
    for b in range(3):
        u = [max(sum(Fraction(int(P1[k, i])) * int(h[b, i]) for i in range(d)), 0) for k in range(rank)]
        for c in range(ffn - n_hot):
            s = sum(Fraction(int(P2[c, k])) * u[k] for k in range(rank)) + Fraction(float(bp[c]))
            assert r["s"][b, c] == float(s)
            if s > Fraction(1, 4):
                act.add(n_hot + c)
    assert r["idx"].tolist() == sorted(act)


def test_neuron_permutation_invariance():
    """Placing the neurons in another order (the offline hot-first layout and
    its neuron table) does not change y when the list follows the table."""
    rng = np.random.default_rng(7)
    d, ffn, n_hot, B = 32, 40, 0, 2
    for act in ("relu", "reglu"):
        Wg, Wu, WdT, b1, b2 = _rand_layer(rng, d, ffn, act, "f32")
        h = _tokens(rng, B, d)
        M = np.sort(rng.choice(ffn, size=17, replace=False))
        y = oracle.masked_ffn(h, M, Wg, Wu, WdT, b1, b2, act, n_hot, ffn)
        perm = rng.permutation(ffn)           # storage row -> original row
        inv = np.argsort(perm)
        P = lambda A: None if A is None else np.ascontiguousarray(A[perm])
        Mp = np.sort(inv[M])
        yp = oracle.masked_ffn(h, Mp, P(Wg), P(Wu), P(WdT), b1[perm], b2, act, n_hot, ffn)
        assert np.allclose(yp, y, rtol=0, atol=1e-12 * np.abs(y).max())
        assert not np.array_equal(M, Mp)


def test_hot_cold_split_point_invariance():
    rng = np.random.default_rng(8)
    d, ffn, B = 32, 30, 2
    Wg, Wu, WdT, b1, b2 = _rand_layer(rng, d, ffn, "reglu", "f32")
    h = _tokens(rng, B, d)
    union = np.array(sorted(set(range(0, 12)) | {15, 19, 20, 27}))
    ref = oracle.masked_ffn(h, union[union >= 12], Wg, Wu, WdT, b1, b2, "reglu", 12, ffn)
    for H in (0, 3, 7, 12):
        y = oracle.masked_ffn(h, union[union >= H], Wg, Wu, WdT, b1, b2, "reglu", H, ffn)
        assert np.array_equal(y, ref)   # same ascending order -> identical


def _q4_twin(rng, rows, d):
    q = rng.integers(0, 16, size=(rows, d)).astype(np.uint8)
    e = rng.integers(-6, 0, size=(rows, d // 32))
    sc = (2.0 ** e).astype(np.float16) * np.where(rng.random((rows, d // 32)) < 0.5, -1, 1).astype(np.float16)
    blk = q.reshape(rows, d // 32, 32)
    qs = (blk[..., :16] | (blk[..., 16:] << 4)).reshape(rows, d // 2).astype(np.uint8)
    x = (sc.astype(np.float64)[:, :, None] * (blk.astype(np.float64) - 8)).reshape(rows, d)
    return (np.ascontiguousarray(qs), np.ascontiguousarray(sc)), x.astype(np.float16)


@pytest.mark.parametrize("act", ["relu", "reglu"])
def test_q4_0_path_equals_its_fp16_twin(act):
    """Q4_0 weights whose values s * (q - 8) are exact in fp16 give the same y
    through the Q4_0 decoder as through the fp16 decoder."""
    rng = np.random.default_rng(9)
    d, ffn, n_hot = 64, 24, 4
    (gq, gx), (uq, ux), (dq, dx) = _q4_twin(rng, ffn, d), _q4_twin(rng, ffn, d), _q4_twin(rng, ffn, d)
    assert np.array_equal(oracle.decode_matrix(uq, d), ux.astype(np.float64))
    b1 = (rng.standard_normal(ffn) * 0.3).astype(np.float32)
    h = _tokens(rng, 2, d).astype(np.float16)
    M = [5, 9, 10, 17, 23]
    yq = oracle.masked_ffn(h, M, gq if act == "reglu" else None, uq, dq, b1, None, act, n_hot, ffn)
    yx = oracle.masked_ffn(h, M, gx if act == "reglu" else None, ux, dx, b1, None, act, n_hot, ffn)
    assert np.array_equal(yq, yx)


def test_column_subset_matches_full_output():
    rng = np.random.default_rng(10)
    d, ffn, n_hot = 40, 30, 5
    Wg, Wu, WdT, b1, b2 = _rand_layer(rng, d, ffn, "reglu", "f16")
    h = _tokens(rng, 2, d).astype(np.float16)
    M = [6, 8, 29]
    y = oracle.masked_ffn(h, M, Wg, Wu, WdT, b1, b2, "reglu", n_hot, ffn)
    cols = [39, 0, 17, 17]
    ys = oracle.masked_ffn(h, M, Wg, Wu, WdT, b1, b2, "reglu", n_hot, ffn, cols=cols)
    assert np.array_equal(ys, y[:, cols])


def test_empty_list_gives_bias_only():
    rng = np.random.default_rng(12)
    d, ffn = 16, 8
    Wg, Wu, WdT, b1, b2 = _rand_layer(rng, d, ffn, "relu", "f32")
    h = _tokens(rng, 1, d)
    y = oracle.masked_ffn(h, [], Wg, Wu, WdT, b1, b2, "relu", 0, ffn)
    assert np.array_equal(y[0], b2.astype(np.float64))
    y = oracle.masked_ffn(h, [], Wg, Wu, WdT, b1, None, "relu", 0, ffn)
    assert np.array_equal(y[0], np.zeros(d))


# ----------------------------------------------------------------------------
# stack glue


def test_rmsnorm_golden_and_closed_forms():
    g = read("rmsnorm.txt")
    for case in g["case"]:
        hs, ys, eps, want = case.split("|")
        h = mat(hs).astype(np.float32).reshape(1, -1)
        y = mat(ys).reshape(1, -1)
        out = oracle.residual_rmsnorm(h, y, float(eps))
        assert np.allclose(out[0], mat(want), rtol=1e-15, atol=1e-15)
    rng = np.random.default_rng(13)
    h = rng.standard_normal((3, 50)).astype(np.float32)
    y = rng.standard_normal((3, 50))
    out = oracle.residual_rmsnorm(h, y, 0.0)
    assert np.allclose((out ** 2).mean(axis=1), 1.0, rtol=1e-14)   # unit RMS
    out2 = oracle.residual_rmsnorm((h * 4).astype(np.float32), y * 4, 0.0)
    assert np.allclose(out2, out, rtol=1e-14, atol=1e-14)           # scale invariance


# ----------------------------------------------------------------------------
# planted mistakes must be caught

_MUTANTS = {
    "gate bias dropped": ("if (b1) acc += (double)b1[j];", ";"),
    "ReLU on u dropped": ("u[(size_t)b * rank + k] = acc > 0.0 ? acc : 0.0;", "u[(size_t)b * rank + k] = acc;"),
    "threshold not strict": ("(s[(size_t)b * n_cold + c] > thr)", "(s[(size_t)b * n_cold + c] >= thr)"),
    "nibble order swapped": ("int q = (k < 16) ? (byte & 0x0f) : (byte >> 4);",
                             "int q = (k < 16) ? (byte >> 4) : (byte & 0x0f);"),
    "Q4_0 offset missing": ("* (double)(q - 8);", "* (double)(q);"),
    "down projection transposed": ("acc += a[(size_t)b * n_list + p] * orc_elem(wtype, wd, wd_sc, j, e, d);",
                                   "acc += a[(size_t)b * n_list + p] * orc_elem(wtype, wd, wd_sc, e % d, j % d, d);"),
    "gate and up swapped": ("double g = preact(wg, wg_sc, wtype, b1, j, hb, d);",
                            "double g = preact(wu, wu_sc, wtype, b1, j, hb, d);"),
    "hot rows skipped": ("int64_t j = p < n_hot ? p : (int64_t)idx[p - n_hot];\n      a[",
                         "int64_t j = p < n_hot ? p + 1 : (int64_t)idx[p - n_hot];\n      a["),
    "output bias dropped": ("double acc = b2 ? (double)b2[e] : 0.0;", "double acc = 0.0;"),
    "fp16 exponent bias off by one": ("expo - 25", "expo - 24"),
    "squared ReLU not squared": ("return act == ORC_RELU2 ? r * r : r;", "return r;"),
    "rmsnorm mean over d-1": ("sqrt(ss / (double)d + eps)", "sqrt(ss / (double)(d - 1) + eps)"),
}

_PIN_TESTS = [
    test_q4_0_golden_row,
    test_predictor_golden_per_token_and_union,
    lambda: [test_ffn_reglu_golden(m) for m in ([], [1], [2], [1, 2])],
    lambda: [test_ffn_relu_family_golden(a, m) for a in ("relu", "relu2") for m in ([], [2], [1, 2])],
    test_true_support_golden,
    test_rmsnorm_golden_and_closed_forms,
    test_empty_list_gives_bias_only,
    lambda: test_half_decode_matches_numpy_for_every_bit_pattern(),
]


@pytest.mark.parametrize("name", sorted(_MUTANTS))
def test_pins_reject_planted_mistake(name, tmp_path):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "pi_oracle.c"), encoding="utf-8").read()
    old, new = _MUTANTS[name]
    assert src.count(old) == 1, "mutation anchor not found: %s" % name
    path = tmp_path / "mut.c"
    path.write_text(src.replace(old, new), encoding="utf-8")
    so = str(tmp_path / "libmut.so")
    subprocess.check_call(["gcc", "-O1", "-fPIC", "-shared", "-std=c11", "-o", so, str(path), "-lm"])
    caught = False
    with oracle.use_library(so):
        for t in _PIN_TESTS:
            try:
                t()
            except AssertionError:
                caught = True
                break
    assert caught, "no pin rejects the planted mistake: " + name


# ----------------------------------------------------------------------------
# Q4_0 predictor (a smaller predictor; the pages size it per layer)


def _hexrow(s, dtype):
    return np.array([int(x, 16) for x in s.split()], dtype=dtype)


def test_q4_0_predictor_golden():
    """Hand-worked Q4_0 predictor (tests/golden/predictor_q4_0_d32_r32.txt)."""
    g = read("predictor_q4_0_d32_r32.txt")
    d, r, ffn, n_hot, thr = int(g["d"]), int(g["rank"]), int(g["ffn"]), int(g["n_hot"]), float(g["thr"])
    p1_qs = np.tile(_hexrow(g["P1_rest_qs"], np.uint8), (r, 1))
    p1_sc = np.full((r, 1), int(g["P1_rest_scale"], 16), dtype=np.uint16)
    for row in (0, 1):
        p1_qs[row] = _hexrow(g["P1_row%d_qs" % row], np.uint8)
        p1_sc[row, 0] = int(g["P1_row%d_scale" % row], 16)
    p2_qs = np.stack([_hexrow(g["P2_row%d_qs" % c], np.uint8) for c in (0, 1)])
    p2_sc = np.array([[int(g["P2_row%d_scale" % c], 16)] for c in (0, 1)], dtype=np.uint16)
    P1 = (np.ascontiguousarray(p1_qs), np.ascontiguousarray(p1_sc.view(np.float16)))
    P2 = (np.ascontiguousarray(p2_qs), np.ascontiguousarray(p2_sc.view(np.float16)))
    h = np.zeros((1, d), np.float16)
    for i, v in mat(g["h_nonzero"]):
        h[0, int(i)] = v
    u = np.zeros(r)
    for k, v in mat(g["u_nonzero"]):
        u[int(k)] = v
    res = oracle.predict(h, P1, P2, mat(g["bp"]).astype(np.float32), thr, n_hot, ffn)
    assert np.array_equal(res["u"][0], u)
    assert np.array_equal(res["s"][0], mat(g["s"]))
    assert res["idx"].tolist() == ints(g["idx"])


def test_q4_0_predictor_equals_its_fp16_twin():
    """A Q4_0 predictor whose values s * (q - 8) are exact in fp16 gives the
    same u, scores and list as the fp16 predictor holding those values (the
    fp16 path is pinned by the hand-worked fixtures above)."""
    rng = np.random.default_rng(31)
    d, r, ffn, n_hot = 96, 64, 40, 6
    P1q, P1x = _q4_twin(rng, r, d)
    P2q, P2x = _q4_twin(rng, ffn - n_hot, r)
    bp = (rng.standard_normal(ffn - n_hot) * 0.5).astype(np.float32)
    h = _tokens(rng, 3, d).astype(np.float16)
    a = oracle.predict(h, P1q, P2q, bp, 0.5, n_hot, ffn)
    b = oracle.predict(h, P1x, P2x, bp, 0.5, n_hot, ffn)
    assert np.array_equal(a["u"], b["u"]) and np.array_equal(a["s"], b["s"])
    assert np.array_equal(a["idx"], b["idx"]) and 0 < len(a["idx"]) < ffn - n_hot


# ----------------------------------------------------------------------------
# head-sparse decode attention (the self-attention predictor's operator)


def _attn_golden():
    g = read("attention_d4_h2.txt")
    d, H, n = int(g["d"]), int(g["n_heads"]), int(g["len"])
    W = {k: mat(g[k]).astype(np.float32) for k in ("Wq", "Wk", "Wv", "WoT")}
    x = mat(g["x"]).astype(np.float32).reshape(1, d)
    K = np.zeros((1, H, 4, d // H), np.float32)
    V = np.zeros((1, H, 4, d // H), np.float32)
    K[0, :, 0] = mat(g["K0"])
    V[0, :, 0] = mat(g["V0"])
    return g, d, H, n, W, x, K, V


def test_attention_golden_per_head_and_union():
    g, d, H, n, W, x, K, V = _attn_golden()
    r0 = oracle.attention(x, [0], W["Wq"], W["Wk"], W["Wv"], W["WoT"], K, V, n, H, 0)
    assert np.array_equal(r0["y"][0], mat(g["y_head0"]))
    assert np.array_equal(r0["k"][0, 0], mat(g["k_head0"])) and np.array_equal(r0["v"][0, 0], mat(g["v_head0"]))
    r1 = oracle.attention(x, [1], W["Wq"], W["Wk"], W["Wv"], W["WoT"], K, V, n, H, 0)
    assert np.array_equal(r1["y"][0], mat(g["y_head1"]))
    both = oracle.attention(x, [1], W["Wq"], W["Wk"], W["Wv"], W["WoT"], K, V, n, H, 1)   # head 0 hot, 1 listed
    assert np.array_equal(both["y"][0], mat(g["y_both"]))
    assert oracle.attention(x, [], W["Wq"], W["Wk"], W["Wv"], W["WoT"], K, V, n, H, 0)["y"].tolist() == [[0, 0, 0, 0]]


def _attn_rand(rng, B, d, H, s_max, dtype=np.float16):
    W = {k: (rng.standard_normal((d, d)) / np.sqrt(d)).astype(dtype) for k in ("Wq", "Wk", "Wv", "WoT")}
    x = _tokens(rng, B, d).astype(dtype)
    K = rng.standard_normal((B, H, s_max, d // H)).astype(dtype)
    V = rng.standard_normal((B, H, s_max, d // H)).astype(dtype)
    return W, x, K, V


def test_attention_empty_cache_is_the_value_projection():
    """len = 0: the new token attends to itself alone (softmax of one score is
    1), so each head's output is its own v and y = sum_h WoT[h]^T v_h."""
    rng = np.random.default_rng(41)
    B, d, H = 2, 32, 4
    W, x, K, V = _attn_rand(rng, B, d, H, 3)
    r = oracle.attention(x, [1, 3], W["Wq"], W["Wk"], W["Wv"], W["WoT"], K, V, 0, H, 0)
    dh = d // H
    Wv, WoT = W["Wv"].astype(np.float64), W["WoT"].astype(np.float64)
    xd = x.astype(np.float64)
    for b in range(B):
        ref = sum(WoT[h * dh:(h + 1) * dh].T @ (Wv[h * dh:(h + 1) * dh] @ xd[b]) for h in (1, 3))
        assert np.allclose(r["y"][b], ref, rtol=0, atol=1e-12)


def test_attention_equal_scores_average_the_values():
    """Wq = 0: every score is 0, p is uniform over the len + 1 positions, and
    o is the mean of the cached values and the new v."""
    rng = np.random.default_rng(42)
    B, d, H, n = 1, 16, 2, 5
    W, x, K, V = _attn_rand(rng, B, d, H, 8)
    W["Wq"][:] = 0
    r = oracle.attention(x, [0, 1], W["Wq"], W["Wk"], W["Wv"], W["WoT"], K, V, n, H, 0)
    dh = d // H
    for h in range(H):
        o = (V[0, h, :n].astype(np.float64).sum(axis=0) + r["v"][0, h]) / (n + 1)
        y_h = W["WoT"][h * dh:(h + 1) * dh].astype(np.float64).T @ o
        y_one = oracle.attention(x, [h], W["Wq"], W["Wk"], W["Wv"], W["WoT"], K, V, n, H, 0)["y"][0]
        assert np.allclose(y_one, y_h, rtol=0, atol=1e-12)


def test_attention_is_additive_over_heads_and_invariant_to_cache_order():
    """Heads contribute independently (y of a set = sum of single heads, up
    to rounding); permuting the cached positions (K and V together) leaves
    every head's softmax-weighted average unchanged; listing a head as hot
    or as predicted gives the same y."""
    rng = np.random.default_rng(43)
    B, d, H, n = 2, 32, 4, 6
    W, x, K, V = _attn_rand(rng, B, d, H, 9)
    args = (W["Wq"], W["Wk"], W["Wv"], W["WoT"])
    y = oracle.attention(x, [0, 2, 3], *args, K, V, n, H, 0)["y"]
    parts = sum(oracle.attention(x, [h], *args, K, V, n, H, 0)["y"] for h in (0, 2, 3))
    assert np.allclose(y, parts, rtol=0, atol=1e-12)
    perm = rng.permutation(n)
    Kp, Vp = K.copy(), V.copy()
    Kp[:, :, :n] = K[:, :, perm]
    Vp[:, :, :n] = V[:, :, perm]
    assert np.allclose(oracle.attention(x, [0, 2, 3], *args, Kp, Vp, n, H, 0)["y"], y, rtol=0, atol=1e-12)
    assert np.array_equal(oracle.attention(x, [2, 3], *args, K, V, n, H, 1)["y"],
                          oracle.attention(x, [0, 2, 3], *args, K, V, n, H, 0)["y"])
    # positions past len are never read
    K2, V2 = K.copy(), V.copy()
    K2[:, :, n:] = 1e4
    V2[:, :, n:] = -1e4
    assert np.array_equal(oracle.attention(x, [0, 2, 3], *args, K2, V2, n, H, 0)["y"], y)


def test_attention_two_positions_is_a_logistic_of_the_scaled_score():
    """One cached position with key K0 and a new token whose k and v are 0:
    the softmax over two scores reduces to p0 = 1 / (1 + exp(-q.K0 / sqrt(dh))),
    so o = p0 V0 -- this fixes the 1/sqrt(dh) scale."""
    d, H = 8, 2
    dh = d // H
    x = np.zeros((1, d), np.float32)
    x[0, 0] = 1.0
    Wq = np.zeros((d, d), np.float32)
    Wq[0, 0] = 3.0                      # head 0: q = [3, 0, 0, 0]
    Wk = np.zeros((d, d), np.float32)   # k_new = 0
    Wv = np.zeros((d, d), np.float32)   # v_new = 0
    WoT = np.eye(d, dtype=np.float32)   # y = o of head 0 in columns 0..3
    K = np.zeros((1, H, 2, dh), np.float32)
    V = np.zeros((1, H, 2, dh), np.float32)
    K[0, 0, 0] = [1.0, 0, 0, 0]
    V[0, 0, 0] = [2.0, -1.0, 0, 0.5]
    r = oracle.attention(x, [0], Wq, Wk, Wv, WoT, K, V, 1, H, 0)
    p0 = 1.0 / (1.0 + math.exp(-3.0 / math.sqrt(dh)))
    assert np.allclose(r["y"][0, :dh], p0 * V[0, 0, 0].astype(np.float64), rtol=0, atol=1e-15)
    assert np.all(r["y"][0, dh:] == 0)
