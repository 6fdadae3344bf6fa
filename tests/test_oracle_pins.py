"""Pins for the CPU oracle: facts fixed by mathematics or printed on the pages.

None of these re-types the oracle's own formula.  Each pin compares the oracle
with something independent of it: numpy's own float16 decoder, a bit
reinterpretation, exact int64 arithmetic, a hand-worked example, closed forms,
invariants of the product, or a different top-k algorithm.  The mutation tests
in ``test_oracle_mutants.py`` check that a plausible slip in ``oracle.c`` makes
at least one of these fail.
"""
import os

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- pin helpers
# Each helper takes an ``Oracle`` so that the mutation tests can run the same
# pins against deliberately broken builds of oracle.c.

def pin_decode_bf16(orc):
    """Every bf16 pattern equals the fp32 with the same top 16 bits (bf16 definition)."""
    bits = np.arange(1 << 16, dtype=np.uint32)
    with np.errstate(invalid="ignore"):
        ref = (bits << np.uint32(16)).view(np.float32).astype(np.float64)
    got = np.array([orc.dec_bf16(int(b)) for b in bits])
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all(), f"bf16 decode differs at {np.flatnonzero(~same)[:5]}"
    assert np.array_equal(np.signbit(got[~np.isnan(got)]), np.signbit(ref[~np.isnan(ref)]))


def pin_decode_f16(orc):
    """Every binary16 pattern equals numpy's own float16 value (IEEE-754 binary16)."""
    bits = np.arange(1 << 16, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([orc.dec_f16(int(b)) for b in bits])
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all(), f"f16 decode differs at {np.flatnonzero(~same)[:5]}"
    assert np.array_equal(np.signbit(got[~np.isnan(got)]), np.signbit(ref[~np.isnan(ref)]))


def _int_case(seed, m, k, n, fmt, lo=-15, hi=15):
    a = synth.integer_bits(seed, (m, k), fmt, lo, hi)
    w = synth.integer_bits(seed + 1, (n, k), fmt, lo, hi)
    ai = synth.bits_to_float32(a, fmt).astype(np.int64)
    wi = synth.bits_to_float32(w, fmt).astype(np.int64)
    return a, w, ai, wi


def pin_integer_bruteforce(orc):
    """Integer-valued inputs: the product is exact, so it must equal int64 A @ W exactly."""
    for fmt in ("bf16", "f16"):
        for (m, k, n) in [(1, 8, 1), (3, 37, 5), (7, 64, 11), (16, 40, 3), (2, 1, 9)]:
            a, w, ai, wi = _int_case(1000 + m * k * n, m, k, n, fmt)
            c, s = orc.matmul(a, fmt, w, fmt)
            assert np.array_equal(c, (ai @ wi.T).astype(np.float64)), (fmt, m, k, n)
            assert np.array_equal(s, (np.abs(ai) @ np.abs(wi).T).astype(np.float64)), (fmt, m, k, n)


def pin_mixed_formats(orc):
    """A in one 16-bit format and W in the other still gives the exact integer product."""
    a, _, ai, _ = _int_case(77, 4, 24, 6, "bf16")
    _, w, _, wi = _int_case(78, 4, 24, 6, "f16")
    c, _ = orc.matmul(a, "bf16", w, "f16")
    assert np.array_equal(c, (ai @ wi.T).astype(np.float64))


def pin_worked_example(orc):
    """The hand-worked 2x3x2 product in tests/golden/worked_2x3x2.txt."""
    rows = {}
    with open(os.path.join(GOLDEN, "worked_2x3x2.txt")) as f:
        for line in f:
            line = line.split("#")[0].split()
            if line:
                rows[line[0]] = line[1:]
    c_ref = np.array(rows["C"], dtype=np.float64).reshape(2, 2)
    s_ref = np.array(rows["S"], dtype=np.float64).reshape(2, 2)
    for fmt in ("bf16", "f16"):
        a = np.array([int(h, 16) for h in rows[f"A_{fmt}"]], dtype=np.uint16).reshape(2, 3)
        w = np.array([int(h, 16) for h in rows[f"Wt_{fmt}"]], dtype=np.uint16).reshape(2, 3)
        c, s = orc.matmul(a, fmt, w, fmt)
        assert np.array_equal(c, c_ref), (fmt, c)
        assert np.array_equal(s, s_ref), (fmt, s)


def pin_identity_and_permutation(orc):
    """W = I gives C = A exactly; a permutation W permutes A's columns."""
    k = 48
    a = synth.normal_bits(5, (6, k), "bf16", 1.0)
    one = synth.to_bits(np.ones(1), "bf16")[0]
    eye = np.zeros((k, k), dtype=np.uint16)
    eye[np.arange(k), np.arange(k)] = one
    c, _ = orc.matmul(a, "bf16", eye, "bf16")
    assert np.array_equal(c, synth.bits_to_float32(a, "bf16").astype(np.float64))
    perm = np.random.default_rng(3).permutation(k)
    pw = np.zeros((k, k), dtype=np.uint16)
    pw[np.arange(k), perm] = one          # row j of Wt picks column perm[j] of A
    c, _ = orc.matmul(a, "bf16", pw, "bf16")
    assert np.array_equal(c, synth.bits_to_float32(a, "bf16").astype(np.float64)[:, perm])


def pin_closed_forms(orc):
    """All-ones gives k; one-hot rows of A select rows of Wt."""
    for fmt in ("bf16", "f16"):
        k = 40
        ones = synth.to_bits(np.ones((3, k)), fmt)
        c, s = orc.matmul(ones, fmt, ones[:2], fmt)
        assert np.array_equal(c, np.full((3, 2), float(k)))
        assert np.array_equal(s, np.full((3, 2), float(k)))
        w = synth.normal_bits(11, (5, k), fmt, 0.3)
        oh = np.zeros((k, k), dtype=np.uint16)
        oh[np.arange(k), np.arange(k)] = synth.to_bits(np.ones(1), fmt)[0]
        c, _ = orc.matmul(oh[[4, 0, 17]], fmt, w, fmt)
        wv = synth.bits_to_float32(w, fmt).astype(np.float64)
        assert np.array_equal(c, wv[:, [4, 0, 17]].T)


def pin_invariants(orc):
    """Row i does not change as m grows; row permutation commutes; W*2 gives C*2 exactly."""
    a, w = synth.gemv_ffn(16, k=128, n=96)
    full, _ = orc.matmul(a, "bf16", w, "bf16")
    for m in (1, 2, 4, 8):
        part, _ = orc.matmul(a[:m], "bf16", w, "bf16")
        assert np.array_equal(part, full[:m])
    perm = np.random.default_rng(1).permutation(16)
    pc, _ = orc.matmul(a[perm], "bf16", w, "bf16")
    assert np.array_equal(pc, full[perm])
    w2 = synth.to_bits(2.0 * synth.bits_to_float32(w, "bf16").astype(np.float64), "bf16")
    c2, _ = orc.matmul(a, "bf16", w2, "bf16")
    assert np.array_equal(c2, 2.0 * full)


def pin_statistics(orc):
    """With W ~ N(0, 1/sqrt(k)) (std reading), C has standard deviation near 1."""
    a, w = synth.gemv_ffn(8, k=896, n=1024)
    c, _ = orc.matmul(a, "bf16", w, "bf16")
    assert abs(c.std() - 1.0) < 0.05
    assert abs(c.mean()) < 0.05


def _cancellation_cases():
    """Cases of tests/golden/cancellation.txt: (name, fmt, A bits, Wt bits, C, S)."""
    out = []
    with open(os.path.join(GOLDEN, "cancellation.txt")) as f:
        for line in f:
            tok = line.split("#")[0].split()
            if not tok:
                continue
            name, fmt, rest = tok[0], tok[1], tok[2:]
            c, s = float(rest[-2]), float(int(rest[-1]))
            bits = []
            for t in rest[:-2]:
                h, _, rep = t.partition("*")
                bits += [int(h, 16)] * (int(rep) if rep else 1)
            k = len(bits) // 2
            a = np.array(bits[:k], dtype=np.uint16).reshape(1, k)
            w = np.array(bits[k:], dtype=np.uint16).reshape(1, k)
            out.append((name, fmt, a, w, c, s))
    return out


def pin_fp64_ascending_accumulation(orc):
    """Cancellation cases worked by hand: they hold only for a binary64 sum in ascending p."""
    cases = _cancellation_cases()
    assert len(cases) == 5
    for name, fmt, a, w, c_ref, s_ref in cases:
        c, s = orc.matmul(a, fmt, w, fmt)
        assert c[0, 0] == c_ref, (name, fmt, c[0, 0], c_ref)
        assert s[0, 0] == s_ref, (name, fmt, s[0, 0], s_ref)


def _brute_topk(row, k):
    """k rounds of a linear scan for the best remaining element (selection, not sort)."""
    taken = np.zeros(row.size, dtype=bool)
    out = []
    for _ in range(k):
        best = -1
        for j in range(row.size):
            if taken[j]:
                continue
            if best < 0:
                best = j
                continue
            x, y = row[j], row[best]
            if np.isnan(x) and not np.isnan(y):
                best = j
            elif not np.isnan(x) and not np.isnan(y) and x > y:
                best = j
            # equal (incl. -0 == +0) or worse: keep the earlier (lower) index
        taken[best] = True
        out.append(best)
    return np.array(out, dtype=np.int32)


def pin_topk_bruteforce(orc):
    """Top-k equals k rounds of linear arg-max, on random, tie-heavy and NaN rows."""
    rows = [
        synth.choice_f32(21, (64,), [-1.0, 0.0, 1.0]),
        synth.choice_f32(22, (64,), [-0.0, 0.0, 2.5, -2.5]),
        synth.bits_to_float32(synth.normal_bits(23, (200,), "bf16", 1.0), "bf16"),
        np.array([1.0, np.nan, 3.0, np.inf, np.nan, -np.inf, 3.0, 0.0, -0.0, 7.0],
                 dtype=np.float32),
    ]
    for row in rows:
        k = min(10, row.size)
        idx, val = orc.topk(row[None, :], k)
        want = _brute_topk(row, k)
        assert np.array_equal(idx[0], want), (row, idx[0], want)
        assert np.array_equal(val[0].view(np.uint32), row[want].view(np.uint32))


def pin_topk_library_sort(orc):
    """Without NaN, top-k equals numpy's stable lexsort by (-value, index)."""
    x = synth.bits_to_float32(synth.choice_bits(31, (16, 512), "bf16",
                                                [-3, -1, -0.5, 0, 0.5, 1, 2, 3]), "bf16")
    idx, _ = orc.topk(x, 10)
    for r in range(x.shape[0]):
        order = np.lexsort((np.arange(x.shape[1]), -x[r].astype(np.float64)))
        assert np.array_equal(idx[r], order[:10])


def pin_ulp(orc):
    """Grid spacing: numpy's float16 spacing, and bf16 spacings worked by hand."""
    xs = np.array([1.0, 1.5, 1.999, 2.0, 3.0, 0.1, 1000.0, 6.1e-5, 1e-6, 5e-8])
    got = orc.ulp(xs, "f16")
    ref = np.spacing(xs.astype(np.float16)).astype(np.float64)
    assert np.array_equal(got, ref), (got, ref)
    hand = {1.0: 2.0 ** -7, 1.5: 2.0 ** -7, 2.0: 2.0 ** -6, 3.0: 2.0 ** -6,
            0.01: 2.0 ** -14, 1e-40: 2.0 ** -133, 300.0: 2.0}
    got = orc.ulp(np.array(list(hand)), "bf16")
    assert np.array_equal(got, np.array(list(hand.values())))


def pin_cast_bf16(orc):
    """fp32 -> bf16 round to nearest even, checked against exact fp64 arithmetic."""
    bits = np.arange(1 << 16, dtype=np.uint32)
    with np.errstate(invalid="ignore"):
        vals = (bits << np.uint32(16)).view(np.float32)
    finite = np.isfinite(vals)
    # (a) every bf16 value is its own image
    got = orc.cast_f32_bf16(vals[finite][None, :])[0]
    assert np.array_equal(got, bits[finite].astype(np.uint16))
    # (b) halfway points go to the even neighbour, (c) just off them to the nearer one
    rng = np.random.default_rng(7)
    lo = bits[finite & (bits & 0x7FFF < 0x7F7F)][rng.choice(30000, 400, replace=False)]
    for b in lo:
        x = float((np.uint32(b) << np.uint32(16)).view(np.float32))
        nb = int(b) + 1 if x >= 0 else int(b) - 1 if (int(b) & 0x7FFF) else int(b) + 1
        xn = float((np.uint32(b + 1) << np.uint32(16)).view(np.float32))
        mid = np.float32((x + xn) / 2.0)          # exact in fp32 (8 more bits)
        even = b if (b & 1) == 0 else b + 1
        assert orc.f32_to_bf16(mid) == even, (hex(b), mid)
        above = np.nextafter(mid, np.float32(np.inf) if xn > x else np.float32(-np.inf))
        below = np.nextafter(mid, np.float32(-np.inf) if xn > x else np.float32(np.inf))
        assert orc.f32_to_bf16(above) == b + 1 and orc.f32_to_bf16(below) == b, hex(b)
    # (d) overflow: half an ulp above the largest finite bf16 rounds to infinity
    big = (np.uint32(0x7F7F8000)).view(np.float32)
    assert orc.f32_to_bf16(big) == 0x7F80 and orc.f32_to_bf16(-big) == 0xFF80
    # (e) NaN stays NaN
    assert (orc.f32_to_bf16(float("nan")) & 0x7F80) == 0x7F80 and (orc.f32_to_bf16(float("nan")) & 0x7F)


def pin_sigmoid(orc):
    """Closed forms of the logistic function."""
    x = np.array([0.0, np.log(3.0), -np.log(3.0), np.log(9.0), 40.0, -40.0, 1.5, -2.25])
    s = orc.sigmoid(x)
    assert s[0] == 0.5
    assert abs(s[1] - 0.75) < 1e-15 and abs(s[2] - 0.25) < 1e-15 and abs(s[3] - 0.9) < 1e-15
    assert 1 - 1e-15 <= s[4] <= 1.0 and 0 < s[5] < 1e-17
    assert np.all(np.abs(orc.sigmoid(x) + orc.sigmoid(-x) - 1.0) < 1e-15)


ALL_PINS = [pin_decode_bf16, pin_decode_f16, pin_integer_bruteforce, pin_mixed_formats,
            pin_worked_example, pin_identity_and_permutation, pin_closed_forms,
            pin_invariants, pin_statistics, pin_fp64_ascending_accumulation, pin_topk_bruteforce,
            pin_topk_library_sort,
            pin_ulp, pin_cast_bf16, pin_sigmoid]


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(oracle.default())


# ------------------------------------------------------- tolerance and facts

def test_ulp_vec_matches_scalar():
    xs = np.concatenate([np.logspace(-9, 4, 300), [0.0, 2.0 ** -14, 2.0 ** -126, 1.0, 2.0]])
    for fmt in ("f16", "bf16"):
        assert np.array_equal(oracle.ulp_vec(xs, fmt), oracle.ulp(xs, fmt))


def test_check_matmul_flags_planted_error():
    c64 = np.array([[1.0, -2.0]])
    s64 = np.array([[10.0, 20.0]])
    ok, r, _ = oracle.check_matmul(c64 + np.array([[0.9e-4, 0.0]]), c64, s64)
    assert ok and r <= 0.9 + 1e-9
    ok, r, where = oracle.check_matmul(c64 + np.array([[0.0, 2.1e-4]]), c64, s64)
    assert not ok and where == (0, 1)
    # f16 output: half an ulp of the output grid is allowed on top of 1e-5*S
    # (2^-11 at |c| in [1,2), 2^-10 at |c| in [2,4)).
    tiny = np.full_like(s64, 1e-12)
    ok, _, _ = oracle.check_matmul(np.array([[1.0 + 2.0 ** -11, -2.0 - 2.0 ** -10]]), c64, tiny, "f16")
    assert ok
    ok, _, where = oracle.check_matmul(np.array([[1.0 + 2.0 ** -10, -2.0]]), c64, tiny, "f16")
    assert not ok and where == (0, 0)


def _facts():
    out = {}
    with open(os.path.join(GOLDEN, "page_facts.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                key, val = (t.strip() for t in line.split("="))
                out[key] = val
    return out


def test_page_facts_fix_the_workload_shapes():
    f = _facts()
    a, w = synth.router(1)
    assert w.shape == (512, 2560) and w.dtype == np.uint16
    assert round(w.nbytes / 1e6, 1) == float(f["router_weight_MB"])
    assert f["router_dq_shape"] == f"{w.shape[1]}x{w.shape[0]}"
    a, w = synth.gemv_ffn(1)
    assert a.shape[1] == int(f["ffn_inner_k"]) == w.shape[1]
    a, w = synth.narrow(4)
    assert w.shape == (int(f["walbe_N"]), int(f["walbe_K"]))
    assert int(f["topk"]) == 10
    assert int(f["walbe_calls"]) == 36


def test_page_roofline_arithmetic():
    """The note's host roofline (491 MB at 9011 MB/s = 54.5 ms) with the bench's helper."""
    import bench
    f = _facts()
    ms = bench.roofline_time_us(float(f["host_model_MB"]) * 1e6, float(f["host_bw_MBps"]) / 1e3) / 1e3
    assert round(ms, 1) == float(f["host_roofline_ms"])
