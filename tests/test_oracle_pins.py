"""Pins of the CPU oracle to facts outside itself (no GPU needed).

Each ``check_*`` function takes an oracle library handle so that the mutation test at the
bottom can run the same checks against copies of the oracle with a planted mistake: every
planted mistake must make at least one check fail.

Sources of the pinned facts:
  * "A gentle introduction to 8-bit matrix multiplication for transformers at scale"
    (Hugging Face blog, zh translation): the absmax worked example and the x127 scaling
    example (section 模型量化介绍), threshold "6 or more" (section MatMul 内部), the printed
    fp16 / int8 weight rows of nn.Linear(64, 64) (section 用法).
  * "LLM.int8(): 8-Bit Matrix Multiplication for Transformers at Scale" summary
    (azimuth.plus), sections الابتكار الثاني / الصورة الكاملة: outlier columns go through a
    16-bit product, the rest through the int8 product; their sum is the result.
  * Mathematics: threshold = +inf leaves a pure vector-wise int8 product, threshold = 0 a
    plain fp16 matrix product (textbook GEMM, numpy float64 here); round-half-to-even on
    exact ties; permutation and power-of-two scaling invariances; exhaustive binary16 codec
    agreement with numpy; exact brute force on tiny shapes (tests/brute.py).
"""
from __future__ import annotations

import os
import re
import shutil
import subprocess
import tempfile

import numpy as np
import pytest

from oracle import oracle
from int8_quantized_02_b200 import synth

from . import brute

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            out[key] = [float(v) for v in vals]
    return out


def _printed_rows():
    rows = []
    with open(os.path.join(GOLDEN, "printed_weight_rows.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            w, q = line.split("|")
            rows.append(([float(v) for v in w.split()], [int(v) for v in q.split()]))
    return rows


def _ulp16(y: np.ndarray) -> np.ndarray:
    y = np.abs(y.astype(np.float16))
    return (np.nextafter(y, np.float16(np.inf)) - y).astype(np.float64)


# ----------------------------------------------------------------------------- checks ----

def check_absmax_worked_example(lib):
    g = _golden("absmax_worked_example.txt")
    row = np.zeros((1, 16), np.float16)
    row[0, :8] = np.array(g["input"], np.float16)
    # as an activation row: 5.4 < 6, so no outlier column and the row absmax is fp16(5.4)
    Xq, SCA, O = oracle.quantize_rows_and_find_outliers(row, 6.0, lib=lib)
    assert O.size == 0
    assert SCA[0] == np.float32(np.float16(g["absmax"][0]))
    assert Xq[0, :8].tolist() == [int(v) for v in g["quantized"]]
    assert not Xq[0, 8:].any()
    # as a weight row (one output channel)
    CB, SCB = oracle.quantize_weight_colwise(row, lib=lib)
    assert CB[0, :8].tolist() == [int(v) for v in g["quantized"]]
    assert SCB[0] == np.float32(np.float16(g["absmax"][0]))


def check_scaling_worked_example(lib):
    g = _golden("scaling_worked_example.txt")
    w = np.zeros((1, 16), np.float16)
    w[0, 0] = g["range_absmax"][0]
    w[0, 1] = g["value"][0]
    w[0, 2] = -g["range_absmax"][0]
    CB, SCB = oracle.quantize_weight_colwise(w, lib=lib)
    assert SCB[0] == 1.0
    assert CB[0, 1] == int(g["quantized"][0])
    assert CB[0, 0] == 127 and CB[0, 2] == -127
    back = oracle.dequant(CB, SCB, lib=lib)[0, 1]
    # the recovered value 38/127 printed as 0.2992: within one fp16 step (2^-12 near 0.3)
    assert abs(float(back) - g["recovered"][0]) <= 2.0 ** -12
    assert float(back) == float(np.float16(38.0 / 127.0))


def check_printed_rows_are_per_output_channel(lib):
    """Every printed int8 row is reproduced by quantizing its printed fp16 values with one
    absmax of its own (the elided entries hide it, so search the fp16 candidates); no
    single absmax reproduces all rows, which rules out one scale for the whole tensor."""
    rows = _printed_rows()
    cands = np.arange(np.float16(0.04).view(np.uint16), np.float16(0.2).view(np.uint16),
                      dtype=np.uint16).view(np.float16)
    feasible = []
    for w, q in rows:
        w16 = np.array(w, np.float16)
        ok = set()
        for a in cands:
            if a < np.abs(w16).max():
                continue
            W = np.zeros((1, 16), np.float16)
            W[0, :6] = w16
            W[0, 6] = a
            CB, SCB = oracle.quantize_weight_colwise(W, lib=lib)
            if CB[0, :6].tolist() == q:
                ok.add(float(a))
        assert ok, f"no per-row absmax reproduces printed row {q}"
        feasible.append(ok)
    assert not set.intersection(*feasible), "one tensor-wide absmax fits every row"
    # the third printed row shows its own absmax (-0.1227 -> -127)
    assert float(np.float16(0.1227)) in feasible[2]


def check_threshold_inclusive(lib):
    X = np.zeros((3, 32), np.float16)
    X[:, :] = 0.5
    X[1, 4] = 6.0           # exactly the threshold: an outlier ("6 or more")
    X[2, 9] = -6.0          # magnitude counts, not sign
    X[0, 17] = np.nextafter(np.float16(6.0), np.float16(0))  # just below: regular
    Xq, SCA, O = oracle.quantize_rows_and_find_outliers(X, 6.0, lib=lib)
    assert O.tolist() == [4, 9]
    assert not Xq[:, [4, 9]].any()
    # row absmax skips outlier columns: row 1's largest regular value is 0.5
    assert SCA[1] == 0.5
    assert SCA[0] == np.float32(np.nextafter(np.float16(6.0), np.float16(0)))


def check_round_half_even(lib):
    # absmax 127 -> multiplier exactly 1; absmax 254 -> multiplier exactly 0.5
    X = np.array([[127.0, 2.5, 3.5, -2.5, 0.5, 1.5, -3.5, 4.5] + [0.0] * 8,
                  [254.0, 5.0, 7.0, -5.0, 1.0, 3.0, -7.0, 9.0] + [0.0] * 8], np.float16)
    Xq, SCA, O = oracle.quantize_rows_and_find_outliers(X, float("inf"), lib=lib)
    assert O.size == 0
    expect = [127, 2, 4, -2, 0, 2, -4, 4]
    assert Xq[0, :8].tolist() == expect
    assert Xq[1, :8].tolist() == expect


def check_closed_form(lib):
    # X all ones, W all 0.5: Xq = 127, CB = 127, C = 127^2 K, Y = K * 0.5 exactly
    K, N = 16, 3
    X = np.ones((2, K), np.float16)
    W = np.full((N, K), 0.5, np.float16)
    CB, SCB = oracle.quantize_weight_colwise(W, lib=lib)
    Y, C = oracle.linear(X, CB, SCB, threshold=6.0, want_C=True, lib=lib)
    assert (C == 127 * 127 * K).all()
    assert (Y == np.float16(K * 0.5)).all()
    # with a bias and one outlier column of value 8 in row 0
    X[0, 3] = 8.0
    b = np.array([1.0, -2.0, 0.25], np.float16)
    Y = oracle.linear(X, CB, SCB, bias=b, threshold=6.0, lib=lib)
    # row 0: 15 regular ones (exact int path: 127*127*15 * 1 * 0.5 / 127^2 = 7.5) + 8*0.5
    assert Y[0].tolist() == [7.5 + 4.0 + 1.0, 7.5 + 4.0 - 2.0, 7.5 + 4.0 + 0.25]
    # row 1: column 3 is an outlier for every row, so row 1 also splits it off
    assert Y[1].tolist() == [8.0 + 1.0, 8.0 - 2.0, 8.0 + 0.25]


def check_no_outliers_is_pure_int8(lib):
    X, _ = synth.activations(8, 64, 0, seed=3)
    W = synth.weight(24, 64, 0.02, seed=3)
    CB, SCB = oracle.quantize_weight_colwise(W, lib=lib)
    Xq, SCA, O = oracle.quantize_rows_and_find_outliers(X, float("inf"), lib=lib)
    assert O.size == 0
    # vector-wise statistics: per-row absmax of X over all columns
    assert np.array_equal(SCA, np.abs(X.astype(np.float32)).max(axis=1))
    assert np.array_equal(SCB, np.abs(W.astype(np.float32)).max(axis=1))
    Y, C = oracle.linear(X, CB, SCB, threshold=float("inf"), want_C=True, lib=lib)
    C_ref = Xq.astype(np.int64) @ CB.astype(np.int64).T
    assert np.array_equal(C.astype(np.int64), C_ref)
    Y_ref = (C_ref * SCA[:, None].astype(np.float64) * SCB[None, :].astype(np.float64)
             / 16129.0).astype(np.float16)
    assert np.array_equal(Y, Y_ref)


def check_all_outliers_is_fp16_gemm(lib):
    X, _ = synth.activations(6, 48, 0, seed=4)
    W = synth.weight(20, 48, 0.02, seed=4)
    CB, SCB = oracle.quantize_weight_colwise(W, lib=lib)
    Xq, SCA, O = oracle.quantize_rows_and_find_outliers(X, 0.0, lib=lib)
    assert O.tolist() == list(range(48))
    assert not Xq.any() and not SCA.any()
    W_hat = oracle.dequant(CB, SCB, lib=lib)
    for Wsrc, Wkeep in ((W_hat, None), (W, W)):
        Y, C = oracle.linear(X, CB, SCB, W_fp16=Wkeep, threshold=0.0, want_C=True, lib=lib)
        assert not C.any()
        ref = X.astype(np.float64) @ Wsrc.astype(np.float64).T
        ref16 = ref.astype(np.float16)
        diff = np.abs(Y.astype(np.float64) - ref16.astype(np.float64))
        assert (diff <= _ulp16(ref16)).all()
        assert np.mean(Y == ref16) > 0.99


def check_brute_force(lib):
    rng = np.random.default_rng(11)
    cases = []
    for M, K, N in ((1, 16, 1), (3, 16, 5), (4, 32, 8), (2, 32, 3)):
        X = (rng.standard_normal((M, K)) * 2).astype(np.float16)
        W = (rng.standard_normal((N, K)) * 0.05).astype(np.float16)
        cases.append((X, W, 6.0))
    # planted: |x| == t, a zero row, an all-outlier row, exact ties (absmax 127 -> s = 1)
    X = np.zeros((4, 16), np.float16)
    X[0, :] = [127, 2.5, -3.5, 0.5, 1, 6, 2, 2, 2, 2, 2, 2, 2, 2, 2, -127]
    X[2, :] = 7.0
    X[3, :] = [1.5, 2.5, -0.5, 100, 3, 4, 5, 6.5, 0, 0, 0, 0, 1, 1, 1, 1]
    W = (rng.standard_normal((5, 16)) * 0.05).astype(np.float16)
    cases.append((X, W, 200.0))     # no outliers; ties in row 0
    cases.append((X, W, 6.0))       # columns with |x| >= 6 split off; row 2 all outliers
    cases.append((X, W, 0.0))       # everything fp16
    for idx, (X, W, t) in enumerate(cases):
        bias = (rng.standard_normal(W.shape[0]) * 0.1).astype(np.float16)
        for keep in (False, True):
            ref = brute.layer(X, W, t, bias=bias, keep_fp16_weight=keep)
            CB, SCB = oracle.quantize_weight_colwise(W, lib=lib)
            assert np.array_equal(CB, ref["CB"]), idx
            assert np.array_equal(SCB, ref["SCB"]), idx
            Xq, SCA, O = oracle.quantize_rows_and_find_outliers(X, t, lib=lib)
            assert np.array_equal(O, ref["O"]), idx
            assert np.array_equal(Xq, ref["Xq"]), idx
            assert np.array_equal(SCA, ref["SCA"]), idx
            Y, C = oracle.linear(X, CB, SCB, bias=bias, W_fp16=W if keep else None,
                                 threshold=t, want_C=True, lib=lib)
            assert np.array_equal(C.astype(np.int64), ref["C"]), idx
            assert np.array_equal(Y, ref["Y"]), (idx, keep)
            # the sampled form of the layer, every position once in a shuffled order
            M, N = X.shape[0], W.shape[0]
            flat = rng.permutation(M * N)
            rows, cols = flat // N, flat % N
            Ys, Cs = oracle.linear_sampled(X, CB, SCB, rows, cols, bias=bias,
                                           W_fp16=W if keep else None, threshold=t, lib=lib)
            assert np.array_equal(Cs.astype(np.int64), ref["C"][rows, cols]), idx
            assert np.array_equal(Ys, ref["Y"][rows, cols]), (idx, keep)


def check_invariants(lib):
    X, _ = synth.activations(12, 96, 3, lo=6.0, hi=30.0, row_frac=0.5, seed=5)
    W = synth.weight(40, 96, 0.02, seed=5)
    CB, SCB = oracle.quantize_weight_colwise(W, lib=lib)
    Xq, SCA, O = oracle.quantize_rows_and_find_outliers(X, 6.0, lib=lib)
    Y, C = oracle.linear(X, CB, SCB, threshold=6.0, want_C=True, lib=lib)
    assert O.size == 3
    assert not Xq[:, O].any()
    assert np.abs(Xq.astype(np.int32)).max() <= 127
    for i in range(X.shape[0]):
        if SCA[i] > 0:
            assert np.abs(Xq[i].astype(np.int32)).max() == 127
    # row permutation of X permutes Y
    p = np.random.default_rng(0).permutation(X.shape[0])
    Yp = oracle.linear(X[p], CB, SCB, threshold=6.0, lib=lib)
    assert np.array_equal(Yp, Y[p])
    # joint permutation of X's and CB's columns leaves the int32 accumulators unchanged
    q = np.random.default_rng(1).permutation(X.shape[1])
    _, Cq = oracle.linear(np.ascontiguousarray(X[:, q]), np.ascontiguousarray(CB[:, q]), SCB,
                          threshold=6.0, want_C=True, lib=lib)
    assert np.array_equal(Cq, C)
    # scaling X and the threshold by a power of two scales SCA exactly and keeps Xq
    X4 = (X.astype(np.float32) * 4).astype(np.float16)
    Xq4, SCA4, O4 = oracle.quantize_rows_and_find_outliers(X4, 24.0, lib=lib)
    assert np.array_equal(O4, O) and np.array_equal(Xq4, Xq)
    assert np.array_equal(SCA4, SCA * 4)


def check_half_codec(lib):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = bits.view(np.float16).astype(np.float64)
    finite = np.isfinite(vals)
    got = np.array([oracle.half_to_double(int(b), lib=lib) for b in bits[finite]])
    assert np.array_equal(got, vals[finite])
    rng = np.random.default_rng(2)
    xs = np.concatenate([rng.standard_normal(3000) * 10.0 ** rng.integers(-8, 5, 3000),
                         vals[finite] + np.nextafter(0, 1),
                         (vals[finite][:-1] + vals[finite][1:]) / 2])  # midpoints: ties
    xs = xs[np.isfinite(xs)]
    want = xs.astype(np.float16).view(np.uint16)
    got = np.array([oracle.double_to_half(float(x), lib=lib) for x in xs], np.uint16)
    assert np.array_equal(got, want)


def check_int8_accumulate(lib):
    """The stand-alone int8 product against facts outside it: exact Python-integer sums of
    the brute force on tiny shapes, numpy int64 products on larger ones (every int8 code,
    -128 included), and the int32 overflow flag exactly at the first K where all-127
    operands leave the int32 range (INT32_MAX // 127^2 = 133144)."""
    rng = np.random.default_rng(17)
    for M, K, N in ((1, 16, 1), (3, 16, 5), (4, 32, 8)):
        X = (rng.standard_normal((M, K)) * 2).astype(np.float16)
        W = (rng.standard_normal((N, K)) * 0.05).astype(np.float16)
        ref = brute.layer(X, W, 6.0)
        C = oracle.int8_accumulate(ref["Xq"], ref["CB"], lib=lib)
        assert C.dtype == np.int32 and C.shape == (M, N)
        assert np.array_equal(C.astype(np.int64), ref["C"])
    A = rng.integers(-128, 128, (7, 200), dtype=np.int64).astype(np.int8)
    B = rng.integers(-128, 128, (9, 200), dtype=np.int64).astype(np.int8)
    C = oracle.int8_accumulate(A, B, lib=lib)
    assert np.array_equal(C.astype(np.int64), A.astype(np.int64) @ B.astype(np.int64).T)
    # a row against itself and against its negation: the largest and smallest sums
    k_ok = (2**31 - 1) // (127 * 127)
    for K, sign, overflow in ((k_ok, 1, False), (k_ok + 1, 1, True), (k_ok, -1, False),
                              (k_ok + 1, -1, True)):
        a = np.full((1, K), 127, np.int8)
        b = np.full((2, K), 127, np.int8)
        b[1] = 1
        b[0] *= sign
        if overflow:
            with pytest.raises(oracle.OracleError) as e:
                oracle.int8_accumulate(a, b, lib=lib)
            assert e.value.code == oracle.ERR_INT32_OVERFLOW
        else:
            C = oracle.int8_accumulate(a, b, lib=lib)
            assert C[0, 0] == sign * 127 * 127 * K and C[0, 1] == 127 * K


def check_capacity(lib):
    X = np.full((2, 32), 7.0, np.float16)
    with pytest.raises(oracle.OracleError) as e:
        oracle.quantize_rows_and_find_outliers(X, 6.0, cap=5, lib=lib)
    assert e.value.code == oracle.ERR_OUTLIER_CAPACITY


ALL_CHECKS = [check_absmax_worked_example, check_scaling_worked_example,
              check_printed_rows_are_per_output_channel, check_threshold_inclusive,
              check_round_half_even, check_closed_form, check_no_outliers_is_pure_int8,
              check_all_outliers_is_fp16_gemm, check_brute_force, check_invariants,
              check_half_codec, check_int8_accumulate, check_capacity]


@pytest.mark.parametrize("check", ALL_CHECKS, ids=lambda c: c.__name__[6:])
def test_oracle_pin(check, oracle_lib):
    check(oracle_lib)


# ------------------------------------------------------------------- mutation test ----

# Plausible mistakes, planted into a copy of the oracle: (name, pattern, replacement).
MUTANTS = [
    ("threshold_strict", r"\) >= threshold\)", ") > threshold)"),
    ("absmax_over_all_columns", r"if \(is_outlier\[j\]\) continue;", ""),
    ("round_half_away", r"nearbyintf\(scaled\)", "roundf(scaled)"),
    ("outlier_columns_not_zeroed",
     r"xq\[j\] = is_outlier\[j\] \? 0 : absmax_quantize",
     "xq[j] = absmax_quantize"),
    ("reversed_k_index_in_product",
     r"acc \+= \(int64_t\)Xq\[i \* K \+ k\] \* \(int64_t\)CB\[n \* K \+ k\];\n    if \(acc",
     "acc += (int64_t)Xq[i * K + k] * (int64_t)CB[n * K + (K - 1 - k)];\n    if (acc"),
    ("dropped_outlier_term", r"y \+= oracle_half_to_double\(X\[i \* K \+ j\]\)",
     "y += 0.0 * oracle_half_to_double(X[i * K + j])"),
    ("outlier_term_sign", r"y \+= oracle_half_to_double\(X\[i \* K \+ j\]\)",
     "y -= oracle_half_to_double(X[i * K + j])"),
    ("dropped_bias", r"if \(bias\) y \+=", "if (bias) y += 0.0 *"),
    ("scale_not_squared", r"/ 16129\.0", "/ 127.0"),
    ("dequant_without_scale", r"float prod = \(float\)cb \* scb;", "float prod = (float)cb;"),
    ("half_truncates", r"double q = nearbyint\(ldexp\(a, 10 - E\)\);",
     "double q = floor(ldexp(a, 10 - E));"),
    ("half_exponent_bias", r"ldexp\(\(double\)\(m \+ 1024\), e - 25\)",
     "ldexp((double)(m + 1024), e - 24)"),
    ("stores_multiplier_not_absmax", r"SCB\[n\] = amax;", "SCB[n] = 127.0f / amax;"),
    ("accumulate_reversed_k_index",
     r"CB\[n \* K \+ k\];\n            if \(acc > INT32_MAX",
     "CB[n * K + (K - 1 - k)];\n            if (acc > INT32_MAX"),
    ("accumulate_overflow_unflagged",
     r"if \(acc > INT32_MAX \|\| acc < INT32_MIN\) overflow = 1;\n            C\[i \* N \+ n\]",
     "C[i * N + n]"),
    ("accumulate_output_transposed", r"C\[i \* N \+ n\] = \(int32_t\)acc;",
     "C[n * M + i] = (int32_t)acc;"),
    ("sampled_rows_and_cols_swapped", r"Xq, SCA, rows\[s\], cols\[s\],",
     "Xq, SCA, cols[s] % M, rows[s] % N,"),
]


@pytest.fixture(scope="module")
def mutant_dir():
    d = tempfile.mkdtemp(prefix="oracle_mutants_")
    yield d
    shutil.rmtree(d, ignore_errors=True)


@pytest.mark.parametrize("name,pattern,repl", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(name, pattern, repl, mutant_dir):
    with open(os.path.join(os.path.dirname(oracle.__file__), "llmint8_oracle.c")) as f:
        src = f.read()
    mutated, n = re.subn(pattern, repl, src)
    assert n >= 1, f"mutation {name} did not apply"
    path = os.path.join(mutant_dir, f"{name}.c")
    with open(path, "w") as f:
        f.write(mutated)
    so = os.path.join(mutant_dir, f"lib{name}.so")
    subprocess.run(["gcc", *oracle.CFLAGS, "-o", so, path, "-lm"], check=True)
    lib = oracle.load(so)
    caught = []
    for check in ALL_CHECKS:
        try:
            check(lib)
        except (Exception, pytest.fail.Exception):  # noqa: BLE001 - a failed pytest.raises too
            caught.append(check.__name__)
    assert caught, f"no pin catches the planted mistake {name}"
