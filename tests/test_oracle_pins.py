"""Pins for the CPU oracle: each check compares the oracle with something other
than its own arithmetic — values printed on the source pages (tests/golden),
exact-rational brute force, an independent library decode, the trace identity
of the Local-Hessian objective, and its special cases (H = I, one block).
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from conftest import bf16_bits, bits_to_f64, f32_to_bf16_bits

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def read_golden(name):
    rows = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            rows.setdefault(key, []).append(vals)
    return rows


# ------------------------------------------------------------ value sets
def test_e2m1_value_set_matches_page(oracle_mod):
    g = read_golden("e2m1_values.txt")
    mags = [float(v) for v in g["magnitudes"][0]]
    vals = [oracle_mod.e2m1_value(c) for c in range(16)]
    assert len(vals) == int(g["codes"][0][0])
    assert sorted({abs(v) for v in vals}) == sorted(mags)
    assert sorted(set(vals)) == sorted(set(mags) | {-m for m in mags})
    # the sign bit is bit 3 and the magnitude code orders the values
    for c in range(8):
        assert oracle_mod.e2m1_value(c) == mags[c]
        assert oracle_mod.e2m1_value(c | 8) == -mags[c]
        assert math.copysign(1.0, oracle_mod.e2m1_value(8)) == -1.0


def test_e4m3_decode_matches_torch_float8(oracle_mod):
    # independent decode: torch's float8_e4m3fn dtype
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        o = oracle_mod.e4m3_value(c)
        if math.isnan(ref[c]):
            assert math.isnan(o)
        else:
            assert o == ref[c], c


def test_candidate_count_126(oracle_mod):
    g = read_golden("candidates.txt")
    vals = [oracle_mod.e4m3_value(c) for c in range(256)]
    pos = [v for v in vals if math.isfinite(v) and v > 0]
    assert len(pos) == int(g["candidates"][0][0]) == 126
    cand = [oracle_mod.e4m3_value(c) for c in range(1, 127)]
    assert cand == sorted(pos)
    assert all(b > a for a, b in zip(cand, cand[1:]))
    assert cand[0] == 2.0 ** -9 and cand[-1] == 448.0
    assert oracle_mod.e4m3_value(0x56) == 14.0


# ------------------------------------------------------------ E2M1 rounding
E2M1_MAG = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2),
            Fraction(3), Fraction(4), Fraction(6)]


def brute_e2m1(x: float, s: float) -> int:
    """Nearest E2M1 magnitude to |x|/s by enumeration with exact rationals;
    ties to the even magnitude index; s = 0 gives 0; sign kept."""
    sign = 8 if math.copysign(1.0, x) < 0 else 0
    if s == 0:
        return sign
    q = abs(Fraction(x)) / Fraction(s)
    best, best_d = None, None
    for k, v in enumerate(E2M1_MAG):
        d = abs(q - v)
        if best is None or d < best_d or (d == best_d and k % 2 == 0):
            best, best_d = k, d
    return sign | best


def all_finite_bf16():
    u = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    f = bits_to_f64(u)
    return f[np.isfinite(f)]


@pytest.mark.parametrize("s", [1.0, 14.0, 2.0 ** -5, 0.0078125 * 3, 1.1920929e-07 * 1.5,
                               float(np.float32(0.0123456)), float(np.float32(3.3e-3))])
def test_e2m1_encode_brute_force_all_bf16(oracle_mod, s):
    s = float(np.float32(s))
    xs = all_finite_bf16()
    # every finite bf16 at this scale; exact rationals make this the slow reference
    step = 1 if s in (1.0, 14.0) else 7
    for x in xs[::step]:
        assert oracle_mod.e2m1_encode(x, s) == brute_e2m1(float(x), s), (x, s)


def test_e2m1_encode_exact_midpoints_and_saturation(oracle_mod):
    s = float(np.float32(0.75))
    for k in range(7):
        mid = (E2M1_MAG[k] + E2M1_MAG[k + 1]) / 2
        x = float(mid * Fraction(s))
        expect = k if k % 2 == 0 else k + 1
        assert oracle_mod.e2m1_encode(x, s) == expect
        assert oracle_mod.e2m1_encode(-x, s) == 8 | expect
    assert oracle_mod.e2m1_encode(1e30, s) == 7
    assert oracle_mod.e2m1_encode(-0.0, s) == 8
    assert oracle_mod.e2m1_encode(0.0, s) == 0
    assert oracle_mod.e2m1_encode(5.0, 0.0) == 0


# ------------------------------------------------------------ E4M3 rounding
def e4m3_table():
    codes = torch.arange(127, dtype=torch.int32).to(torch.uint8)
    return [Fraction(float(v)) for v in codes.view(torch.float8_e4m3fn).to(torch.float64)]


def brute_e4m3(q: Fraction, table) -> int:
    """Nearest of the 127 non-negative finite E4M3 values (code 0..126),
    ties to the even code, anything above 448 saturates to 448."""
    best, best_d = None, None
    for c, v in enumerate(table):
        d = abs(q - v)
        if best is None or d < best_d or (d == best_d and c % 2 == 0):
            best, best_d = c, d
    return best


def test_e4m3_rounding_brute_force(oracle_mod):
    table = e4m3_table()
    rng = np.random.default_rng(7)
    nums = []
    # every midpoint, exactly, and just around it
    for c in range(126):
        mid = (table[c] + table[c + 1]) / 2
        nums += [mid, mid * (1 + Fraction(1, 2 ** 40)), mid * (1 - Fraction(1, 2 ** 40))]
    nums += [Fraction(float(v)) for v in np.exp2(rng.uniform(-14, 10, 3000))]
    nums += [Fraction(0), Fraction(1, 2 ** 11), Fraction(448), Fraction(464), Fraction(10 ** 6)]
    for q in nums:
        den = 1.0
        num = float(q)
        if Fraction(num) != q:  # keep the quotient exact: scale the denominator instead
            den = float(Fraction(1, 2 ** 50))
            num = float(q * Fraction(1, 2 ** 50))
            assert Fraction(num) / Fraction(den) == q
        assert oracle_mod.e4m3_round_quotient(num, den) == brute_e4m3(q, table), float(q)


# ------------------------------------------------------------ worked example
def test_worked_example_84(oracle_mod):
    g = read_golden("worked_example_84.txt")
    amax = float(g["amax"][0][0])
    scale = float(g["scale"][0][0])
    levels = [float(v) for v in g["levels"][0]]
    zero_below = float(g["zero_below"][0][0])
    blk = np.array([amax, 1, 2, 1.5, 1, 2, 1, 1.25, 2, 1, 1.5, 2, 1, 2, 1, 2], np.float32)
    u = f32_to_bf16_bits(blk)
    s_g = oracle_mod.global_scale(u)
    assert s_g == np.float32(amax / 2688.0) == np.float32(2.0 ** -5)
    code = oracle_mod.max_rule_code(u, s_g)
    assert code == 0x7E
    s_eff = oracle_mod.effective_scale(s_g, code)
    assert s_eff == scale
    # every level is reachable and reproduces itself
    for lv in levels:
        q = oracle_mod.e2m1_encode(lv, s_eff)
        assert oracle_mod.e2m1_value(q) * s_eff == lv
    got = sorted({abs(oracle_mod.e2m1_value(q)) * s_eff for q in range(16)})
    assert got == levels
    # the small values of the example all become 0; 3.5 is the boundary
    for v in [1.0, 1.5, 2.0, zero_below]:
        assert oracle_mod.e2m1_encode(v, s_eff) == 0
    assert oracle_mod.e2m1_encode(float(np.nextafter(np.float32(zero_below), 9)), s_eff) == 1
    # with a unit tensor scale the same block gets FP8 code 0x56 (= 14)
    assert oracle_mod.max_rule_code(u, 1.0) == 0x56
    # dequantised block: 84 stays 84, the rest are 0
    codes = np.array([[code]], np.uint8)
    packed = oracle_mod.quantize_pack(u.reshape(1, 16), s_g, codes)
    deq = bits_to_f64(oracle_mod.dequantize(packed, codes, s_g)).ravel()
    assert deq[0] == amax and np.all(deq[1:] == 0)


def test_global_scale_reading(oracle_mod):
    assert oracle_mod.global_scale(np.zeros(32, np.uint16)) == np.float32(1.0)
    x = f32_to_bf16_bits(np.array([0.5, -3.0, 2.0], np.float32))
    assert oracle_mod.global_scale(x) == np.float32(3.0) / np.float32(2688.0)
    bad = f32_to_bf16_bits(np.array([1.0, np.inf], np.float32))
    with pytest.raises(Exception):
        oracle_mod.global_scale(bad)


def test_effective_scale_is_fp32_product(oracle_mod):
    rng = np.random.default_rng(1)
    for s_g in rng.uniform(1e-4, 1e-1, 20).astype(np.float32):
        for c in (1, 7, 8, 0x38, 0x56, 0x7E):
            e = np.float32(float(torch.tensor([c], dtype=torch.uint8)
                                 .view(torch.float8_e4m3fn).float()))
            assert oracle_mod.effective_scale(s_g, c) == np.float32(s_g * e)


# ------------------------------------------------------------ Local-Hessian
def _tiny_layer(R, C, N, seed):
    g = torch.Generator().manual_seed(seed)
    W = (torch.randn(R, C, generator=g) * 0.02).to(torch.bfloat16)
    X = torch.randn(N, C, generator=g)
    X[:, 3] *= 20.0
    X = X.to(torch.bfloat16)
    return bf16_bits(W), bf16_bits(X)


def test_gram_matches_library_product(oracle_mod):
    W, X = _tiny_layer(8, 48, 40, 3)
    H = oracle_mod.gram(X)
    Xf = bits_to_f64(X)
    for j in range(3):
        Xb = Xf[:, 16 * j:16 * j + 16]
        np.testing.assert_allclose(H[j], Xb.T @ Xb, rtol=1e-15, atol=0)
    # accumulation: two halves add up to the whole
    H2 = oracle_mod.gram(X[20:], oracle_mod.gram(X[:20]))
    np.testing.assert_allclose(H2, H, rtol=1e-15)


def test_lh_objective_equals_output_error_norm(oracle_mod):
    """E(s) = delta H delta^T equals ||X_b delta^T||^2 computed straight from X."""
    W, X = _tiny_layer(6, 64, 48, 5)
    Xf = bits_to_f64(X)
    Wf = bits_to_f64(W)
    H = oracle_mod.gram(X)
    s_g = oracle_mod.global_scale(W)
    for r in range(W.shape[0]):
        for b in range(4):
            blk = W[r, 16 * b:16 * b + 16]
            E = oracle_mod.block_objectives(blk, s_g, H[b])
            for c in (1, 30, 60, 90, 100, 110, 118, 126):
                s = float(oracle_mod.effective_scale(s_g, c))
                q = [oracle_mod.e2m1_encode(w, s) for w in Wf[r, 16 * b:16 * b + 16]]
                delta = Wf[r, 16 * b:16 * b + 16] - np.array([oracle_mod.e2m1_value(k) for k in q]) * s
                direct = float(np.sum((Xf[:, 16 * b:16 * b + 16] @ delta) ** 2))
                assert E[c - 1] == pytest.approx(direct, rel=1e-11, abs=1e-300)


def test_lh_with_identity_hessian_equals_mse(oracle_mod):
    W, _ = _tiny_layer(64, 128, 16, 11)
    s_g = oracle_mod.global_scale(W)
    c_mse, e_mse = oracle_mod.scale_search_mse(W, s_g)
    for alpha in (1.0, 3.7, 1e-3):
        H = np.tile(np.eye(16) * alpha, (8, 1, 1))
        c_lh, e_lh = oracle_mod.scale_search_lh(W, s_g, H)
        assert np.array_equal(c_lh, c_mse)
        np.testing.assert_allclose(e_lh, e_mse * alpha, rtol=1e-12)


def test_lh_single_block_is_exact_full_search(oracle_mod):
    """With C = 16 the block-diagonal approximation is exact: brute force over
    all 126 scales with the full ||delta X||^2 must pick the same scale."""
    W, X = _tiny_layer(40, 16, 64, 13)
    Xf, Wf = bits_to_f64(X), bits_to_f64(W)
    s_g = oracle_mod.global_scale(W)
    codes, _ = oracle_mod.scale_search_lh(W, s_g, oracle_mod.gram(X))
    for r in range(W.shape[0]):
        errs = []
        for c in range(1, 127):
            s = float(oracle_mod.effective_scale(s_g, c))
            v = np.array([oracle_mod.e2m1_value(oracle_mod.e2m1_encode(w, s)) for w in Wf[r]])
            errs.append(float(np.sum((Xf @ (Wf[r] - v * s)) ** 2)))
        errs = np.array(errs)
        best = int(np.argmin(errs)) + 1
        if codes[r, 0] != best:  # only a tie at fp64 resolution may differ
            assert errs[codes[r, 0] - 1] <= errs.min() * (1 + 1e-12)


def test_search_invariants(oracle_mod):
    W, X = _tiny_layer(32, 64, 64, 17)
    s_g = oracle_mod.global_scale(W)
    H = oracle_mod.gram(X)
    c_max = oracle_mod.scale_search_max(W, s_g)
    c_mse, _ = oracle_mod.scale_search_mse(W, s_g)
    c_lh, _ = oracle_mod.scale_search_lh(W, s_g, H)
    for r in range(W.shape[0]):
        for b in range(4):
            blk = W[r, 16 * b:16 * b + 16]
            e_mse = oracle_mod.block_objectives(blk, s_g)
            e_lh = oracle_mod.block_objectives(blk, s_g, H[b])
            assert e_mse[c_mse[r, b] - 1] == e_mse.min()
            assert e_lh[c_lh[r, b] - 1] == e_lh.min()
            # first minimum: no smaller code reaches the minimum
            assert np.all(e_lh[:c_lh[r, b] - 1] > e_lh.min())
            if c_max[r, b]:
                assert e_mse[c_mse[r, b] - 1] <= e_mse[c_max[r, b] - 1]
                assert e_lh[c_lh[r, b] - 1] <= e_lh[c_max[r, b] - 1]
            assert e_lh[c_lh[r, b] - 1] <= e_lh[c_mse[r, b] - 1]


def test_runner_up_objective_is_the_second_smallest(oracle_mod):
    """The searches' runner-up output (used to count near ties) is the second
    smallest of the block's 126 objectives, ties included."""
    W, X = _tiny_layer(6, 48, 40, 29)
    s_g = oracle_mod.global_scale(W)
    W[0, :16] = 0                          # every candidate scores 0: runner-up 0
    H = oracle_mod.gram(X)
    for Hs in (None, H):
        if Hs is None:
            c, b, s2 = oracle_mod.scale_search_mse(W, s_g, runner_up=True)
        else:
            c, b, s2 = oracle_mod.scale_search_lh(W, s_g, Hs, runner_up=True)
        for r in range(6):
            for k in range(3):
                E = oracle_mod.block_objectives(W[r, 16 * k:16 * k + 16], s_g,
                                                None if Hs is None else Hs[k])
                o = np.sort(E)
                assert b[r, k] == o[0] and s2[r, k] == o[1] and E[c[r, k] - 1] == o[0]
        assert s2[0, 0] == 0.0 and c[0, 0] == 1


def test_zero_block_and_zero_hessian(oracle_mod):
    W = np.zeros((2, 32), np.uint16)
    W[1, 16:] = f32_to_bf16_bits(np.linspace(-1, 1, 16, dtype=np.float32))
    s_g = oracle_mod.global_scale(W)
    c_max = oracle_mod.scale_search_max(W, s_g)
    assert c_max[0, 0] == 0 and c_max[1, 0] == 0 and c_max[1, 1] != 0
    c_mse, e = oracle_mod.scale_search_mse(W, s_g)
    assert c_mse[0, 0] == 1 and e[0, 0] == 0
    c_lh, e = oracle_mod.scale_search_lh(W, s_g, np.zeros((2, 16, 16)))
    assert np.all(c_lh == 1) and np.all(e == 0)


# ------------------------------------------------------------ pack / dequant
def test_pack_nibble_order_and_dequant(oracle_mod):
    s_g = np.float32(1.0)
    code = 0x38  # E4M3 value 1.0
    vals = np.array([0.5, -1, 1.5, 6, -6, 0, 2, 3, 4, -0.5, 1, -1.5, 2, -3, -4, 6], np.float32)
    u = f32_to_bf16_bits(vals).reshape(1, 16)
    codes = np.array([[code]], np.uint8)
    packed = oracle_mod.quantize_pack(u, s_g, codes)
    assert packed[0, 0] == (1 | (0xA << 4))      # 0.5 low nibble, -1 high nibble
    assert packed[0, 1] == (3 | (7 << 4))
    assert packed[0, 2] == (0xF | (0 << 4))
    deq = bits_to_f64(oracle_mod.dequantize(packed, codes, s_g))
    np.testing.assert_array_equal(deq.ravel(), vals.astype(np.float64))


def _bf16_nearest_even_exact(f32):
    """bf16 pattern nearest to the finite fp32 value f32, ties to an even bf16
    mantissa, by exact rational distances to the two bf16 values around it
    (overflow past the largest finite bf16 goes to infinity, as IEEE rounding
    does)."""
    b = int(np.float32(f32).view(np.uint32))
    sign, mag = b & 0x80000000, b & 0x7FFFFFFF
    lo = mag & 0xFFFF0000
    if lo == mag:
        return (sign | mag) >> 16
    hi = lo + 0x10000

    def val(bits):
        if bits >= 0x7F800000:  # one step past the largest finite bf16
            return Fraction(2) ** 128
        return Fraction(float(np.uint32(bits).view(np.float32)))
    x = Fraction(float(np.uint32(mag).view(np.float32)))
    dl, dh = x - val(lo), val(hi) - x
    pick = lo if dl < dh else hi if dh < dl else (lo if (lo >> 16) % 2 == 0 else hi)
    return (sign | min(pick, 0x7F800000)) >> 16


def test_bf16_rounding_equals_torch_on_random_patterns(oracle_mod):
    """fp32 -> bf16 rounding of every dequantised and fake-quantised output:
    equal to torch's float32 -> bfloat16 conversion (round to nearest even)
    on 10^7 random bit patterns (every exponent, both signs, subnormals) and
    on every pattern whose low half is a tie (0x8000) or one step either side
    of it, for the upper halves 0x0000..0xFFFF; NaN stays NaN."""
    rng = np.random.default_rng(2024)
    bits = rng.integers(0, 2 ** 32, 10_000_000, dtype=np.uint64).astype(np.uint32)
    hi = np.arange(1 << 16, dtype=np.uint32) << 16
    ties = np.concatenate([hi | 0x8000, hi | 0x7FFF, hi | 0x8001, hi])
    for b in (bits, ties):
        f = b.view(np.float32)
        ours = oracle_mod.floats_to_bf16(f)
        ref = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        nan = np.isnan(f)
        np.testing.assert_array_equal(ours[~nan], ref[~nan])
        assert np.all((ours[nan] & 0x7F80) == 0x7F80) and np.all((ours[nan] & 0x7F) != 0)


def test_bf16_rounding_exact_rationals_on_edge_patterns(oracle_mod):
    """The same rounding against the exact nearest-even bf16 (rational
    arithmetic) on ties of both parities of bit 16, values next to the bf16
    maximum and to the overflow threshold, the smallest subnormals, signed
    zeros and random fp32 values; truncation or round-half-up would fail the
    ties."""
    rng = np.random.default_rng(7)
    pats = [0x3F808000, 0x3F818000, 0xBF808000, 0xBF818000,   # ties, even / odd bit 16
            0x00008000, 0x00018000, 0x80008000, 0x80018000,   # ties among subnormals
            0x7F7F7FFF, 0x7F7F8000, 0x7F7EFFFF, 0x7F7E8000,   # around the largest finite
            0xFF7F8000, 0x00000001, 0x80000001, 0x00007FFF,   # overflow, tiny subnormals
            0x00000000, 0x80000000, 0x3F800000, 0x007F8000]
    pats += list(rng.integers(0, 0x7F800000, 3000, dtype=np.int64) |
                 (rng.integers(0, 2, 3000, dtype=np.int64) << 31))
    f = np.array(pats, np.uint64).astype(np.uint32).view(np.float32)
    ours = oracle_mod.floats_to_bf16(f)
    for x, o in zip(f, ours):
        assert int(o) == _bf16_nearest_even_exact(x), hex(int(np.float32(x).view(np.uint32)))
    # the two ties round to the even neighbour: down for bit 16 = 0, up for 1
    assert list(ours[:4]) == [0x3F80, 0x3F82, 0xBF80, 0xBF82]
    assert ours[9] == 0x7F80 and ours[12] == 0xFF80      # past the overflow threshold
    assert ours[16] == 0x0000 and ours[17] == 0x8000     # signed zeros kept


def test_dequant_of_products_off_the_bf16_grid(oracle_mod):
    """Dequantisation where v * s_eff is not a bf16 value ([QAD] 3.2, the
    quantised value times its scale): every magnitude at tensor scales whose
    fp32 products need rounding to bf16, among them exact ties, against the
    IEEE fp32 product (numpy) rounded by the exact nearest-even rule."""
    mags = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float32)
    for sg_bits in (0x3EAAAAAB, 0x3F808000, 0x3F818000, 0x3DCCCCCD, 0x0071C71C, 0x42F6E979):
        s_g = np.uint32(sg_bits).view(np.float32)
        for code in (0x38, 0x39, 0x5B, 0x01, 0x7E):
            s_eff = np.float32(s_g) * np.float32(oracle_mod.e4m3_value(code))
            assert s_eff == oracle_mod.effective_scale(s_g, code)
            q = np.arange(16, dtype=np.uint8)                 # every E2M1 code once
            packed = (q[0::2] | (q[1::2] << 4)).astype(np.uint8).reshape(1, 8)
            deq = oracle_mod.dequantize(packed, np.array([[code]], np.uint8), s_g).ravel()
            for k in range(16):
                v = mags[k & 7] * (np.float32(-1) if k & 8 else np.float32(1))
                prod = np.float32(v) * np.float32(s_eff)      # one IEEE fp32 multiply
                assert int(deq[k]) == _bf16_nearest_even_exact(prod), (hex(sg_bits), code, k)
    # the tie cases of the fp32 -> bf16 step: s_eff = s_g (code 0x38 = 1.0), v = 1
    for sg_bits, want in ((0x3F808000, 0x3F80), (0x3F818000, 0x3F82)):
        s_g = np.uint32(sg_bits).view(np.float32)
        packed = np.array([[0x22] * 8], np.uint8)             # every element v = 1
        deq = oracle_mod.dequantize(packed, np.array([[0x38]], np.uint8), s_g).ravel()
        assert np.all(deq == want), hex(sg_bits)


def test_quantize_dequantize_idempotent(oracle_mod):
    W, _ = _tiny_layer(16, 64, 1, 19)
    s_g = oracle_mod.global_scale(W)
    codes = oracle_mod.scale_search_max(W, s_g)
    p1 = oracle_mod.quantize_pack(W, s_g, codes)
    y1 = oracle_mod.dequantize(p1, codes, s_g)
    p2 = oracle_mod.quantize_pack(y1, s_g, codes)
    assert np.array_equal(p1, p2)
    # |y| <= 6 s_eff blockwise
    yf = bits_to_f64(y1).reshape(16, 4, 16)
    for r in range(16):
        for b in range(4):
            s = oracle_mod.effective_scale(s_g, codes[r, b])
            assert np.all(np.abs(yf[r, b]) <= 6 * s * (1 + 2 ** -8))


def test_fake_quant_composes_pinned_steps(oracle_mod):
    g = torch.Generator().manual_seed(23)
    X = torch.randn(24, 96, generator=g)
    X[:, 5] *= 40
    Xu = bf16_bits(X.to(torch.bfloat16))
    y, packed, codes, s_g = oracle_mod.fake_quant(Xu)
    assert s_g == oracle_mod.global_scale(Xu)
    assert np.array_equal(codes, oracle_mod.scale_search_max(Xu, s_g))
    assert np.array_equal(packed, oracle_mod.quantize_pack(Xu, s_g, codes))
    assert np.array_equal(y, oracle_mod.dequantize(packed, codes, s_g))


def test_snr_closed_form_arithmetic():
    g = read_golden("snr_closed_form.txt")
    for ratio, _, db in g["m_over_sigma"]:
        est = 20 * math.log10(1.0 / (float(ratio) / 6.0))
        assert est == pytest.approx(float(db), abs=0.06)


def test_grouped_gram_is_per_group_product(oracle_mod):
    g = torch.Generator().manual_seed(29)
    X = torch.randn(50, 32, generator=g).to(torch.bfloat16)
    Xu = bf16_bits(X)
    Xf = bits_to_f64(Xu)
    offsets = np.array([0, 0, 7, 30, 30, 50], np.int64)
    H = oracle_mod.gram_grouped(Xu, offsets, 5)
    for gi in range(5):
        lo, hi = offsets[gi], offsets[gi + 1]
        for j in range(2):
            Xb = Xf[lo:hi, 16 * j:16 * j + 16]
            np.testing.assert_allclose(H[gi, j], Xb.T @ Xb, rtol=1e-15, atol=0)


def test_sampled_search_equals_full_search(oracle_mod):
    W, X = _tiny_layer(20, 64, 32, 31)
    s_g = oracle_mod.global_scale(W)
    H = oracle_mod.gram(X)
    full, fobj = oracle_mod.scale_search_lh(W, s_g, H)
    mfull, mobj = oracle_mod.scale_search_mse(W, s_g)
    rows = np.array([0, 3, 19, 7, 7])
    blocks = np.array([0, 3, 2, 1, 0])
    c, o = oracle_mod.scale_search_sampled(W, s_g, H, rows, blocks)
    assert np.array_equal(c, full[rows, blocks]) and np.array_equal(o, fobj[rows, blocks])
    c, o = oracle_mod.scale_search_sampled(W, s_g, None, rows, blocks)
    assert np.array_equal(c, mfull[rows, blocks]) and np.array_equal(o, mobj[rows, blocks])


# ------------------------------------------------------------ Four Over Six
def _exact_block_mse(vals, s):
    """Exact rational sum of squared errors of a block at scale s (brute-force
    E2M1 codes by enumeration)."""
    e = Fraction(0)
    for x in vals:
        k = brute_e2m1(float(x), float(s)) & 7
        v = E2M1_MAG[k] * Fraction(s)
        e += (abs(Fraction(float(x))) - v) ** 2
    return e


def _brute_four_over_six(vals, s_g, table):
    amax = max(abs(Fraction(float(x))) for x in vals)
    if amax == 0:
        return 0
    sg = Fraction(float(np.float32(s_g)))
    c6 = brute_e4m3(amax / (6 * sg), table)
    c4 = brute_e4m3(amax / (4 * sg), table)
    lo, hi = min(c4, c6), max(c4, c6)
    s_lo = Fraction(float(np.float32(np.float32(s_g) * np.float32(float(table[lo])))))
    s_hi = Fraction(float(np.float32(np.float32(s_g) * np.float32(float(table[hi])))))
    return hi if _exact_block_mse(vals, s_hi) < _exact_block_mse(vals, s_lo) else lo


def test_four_over_six_closed_form_blocks(oracle_mod):
    """Two blocks with tensor scale 1 and amax 48: the candidate scales are
    48/6 = 8 (code 0x50) and 48/4 = 12 (code 0x54).  A block on the grid of
    12 (0, 6, 12, 18, 24, 36, 48) has zero error there and not at 8 (36/8 =
    4.5 rounds to 4): 0x54 wins.  A block on the grid of 8 (0, 4, 8, 12,
    16, 24, 32, 48) with 32 in it (32/12 = 2.67 -> 3) is exact at 8 only:
    0x50 wins."""
    assert oracle_mod.e4m3_value(0x50) == 8.0 and oracle_mod.e4m3_value(0x54) == 12.0
    on12 = [48, 36, 24, 18, 12, 6, 0, -6, -12, -18, -24, -36, 6, 12, 24, 36]
    on8 = [48, 32, 24, 16, 12, 8, 4, 0, -4, -8, -12, -16, -24, -32, 8, 4]
    u12 = f32_to_bf16_bits(np.array(on12, np.float32))
    u8 = f32_to_bf16_bits(np.array(on8, np.float32))
    assert oracle_mod.block_mse(u12, 1.0, 0x54) == 0.0 < oracle_mod.block_mse(u12, 1.0, 0x50)
    assert oracle_mod.block_mse(u8, 1.0, 0x50) == 0.0 < oracle_mod.block_mse(u8, 1.0, 0x54)
    assert oracle_mod.four_over_six_code(u12, 1.0) == 0x54
    assert oracle_mod.four_over_six_code(u8, 1.0) == 0x50
    assert oracle_mod.four_over_six_code(np.zeros(16, np.uint16), 1.0) == 0


def test_four_over_six_brute_force_exact_rationals(oracle_mod):
    """Random blocks (several magnitudes, one saturating the E4M3 range):
    the oracle's choice equals the exact-rational argmin over the two
    candidates."""
    table = e4m3_table()
    rng = np.random.default_rng(21)
    for trial in range(120):
        scale = 10.0 ** rng.uniform(-3, 2)
        vals = rng.standard_normal(16) * scale
        if trial % 10 == 0:
            vals[rng.integers(16)] *= 40
        u = f32_to_bf16_bits(vals.astype(np.float32))
        x = bits_to_f64(u)
        s_g = float(np.float32(np.abs(x).max() * (2.0 if trial % 3 == 0 else 0.4) / 2688.0))
        assert oracle_mod.four_over_six_code(u, s_g) == _brute_four_over_six(x, s_g, table), trial


def test_four_over_six_invariants(oracle_mod):
    """c_46 is the max-rule code or E4M3(amax / (4 s_g)); its MSE is at most
    the max rule's and at least the exhaustive MSE search's."""
    wu, _ = _tiny_layer(32, 128, 8, 5)
    sg = oracle_mod.global_scale(wu)
    c46 = oracle_mod.scale_search_four_over_six(wu, sg)
    cmax = oracle_mod.scale_search_max(wu, sg)
    cmse, emse = oracle_mod.scale_search_mse(wu, sg)
    R, nb = c46.shape
    for r in range(R):
        for b in range(nb):
            blk = wu[r, 16 * b:16 * b + 16]
            amax = np.abs(bits_to_f64(blk)).max()
            c4 = oracle_mod.e4m3_round_quotient(amax, 4.0 * float(np.float32(sg)))
            assert c46[r, b] in (cmax[r, b], c4)
            e46 = oracle_mod.block_mse(blk, sg, int(c46[r, b]))
            assert e46 <= oracle_mod.block_mse(blk, sg, int(cmax[r, b]))
            assert emse[r, b] <= e46 * (1 + 1e-12)


@pytest.mark.parametrize("e", [-100, -60, -24, 24, 60, 110])
def test_every_rule_is_invariant_under_powers_of_two(oracle_mod, e):
    """Scaling the weights by 2^e scales s_g = fl32(amax / 2688) and every
    effective scale fl32(s_g e4m3(c)) by exactly 2^e (all stay normal here),
    every quotient and code is unchanged and every objective scales by
    2^(2e) exactly (fp64, no rounding moves): so every rule picks the same
    codes, pack gives the same bytes, and dequant / fake-quant scale by
    exactly 2^e.  An absolute epsilon or an unscaled tolerance anywhere in
    the path would break this."""
    wu, xu = _tiny_layer(24, 96, 64, 12)
    ws = f32_to_bf16_bits(bits_to_f64(wu) * 2.0 ** e)
    assert np.array_equal(bits_to_f64(ws), bits_to_f64(wu) * 2.0 ** e)
    sg, sgs = oracle_mod.global_scale(wu), oracle_mod.global_scale(ws)
    assert float(sgs) == float(sg) * 2.0 ** e
    for rule in ("scale_search_max", "scale_search_four_over_six"):
        assert np.array_equal(getattr(oracle_mod, rule)(ws, sgs), getattr(oracle_mod, rule)(wu, sg))
    H = oracle_mod.gram(xu)
    for args in ((), (H,)):
        f = oracle_mod.scale_search_lh if args else oracle_mod.scale_search_mse
        c, o = f(wu, sg, *args)
        cs, os_ = f(ws, sgs, *args)
        assert np.array_equal(c, cs)
        assert np.array_equal(os_, o * 2.0 ** (2 * e))
    codes = oracle_mod.scale_search_max(wu, sg)
    p, ps = oracle_mod.quantize_pack(wu, sg, codes), oracle_mod.quantize_pack(ws, sgs, codes)
    assert np.array_equal(p, ps)
    y, ys = oracle_mod.dequantize(p, codes, sg), oracle_mod.dequantize(ps, codes, sgs)
    assert np.array_equal(bits_to_f64(ys), bits_to_f64(y) * 2.0 ** e)
    fy, fp_, fc, fs = oracle_mod.fake_quant(wu)
    gy, gp, gc, gs = oracle_mod.fake_quant(ws)
    assert np.array_equal(fc, gc) and np.array_equal(fp_, gp) and float(gs) == float(fs) * 2.0 ** e
    assert np.array_equal(bits_to_f64(gy), bits_to_f64(fy) * 2.0 ** e)
    Hf = oracle_mod.gram_full(xu)
    assert np.array_equal(oracle_mod.gptq(ws, sgs, codes, Hf), oracle_mod.gptq(wu, sg, codes, Hf))


# ------------------------------------------------------------ W4A4 GEMM
def _decode_nvfp4(packed, codes):
    """Exact values of packed NVFP4 rows, decoded without the oracle: the
    E2M1 magnitudes listed on the pages and torch's float8_e4m3fn decode."""
    lo, hi = packed & 15, packed >> 4
    q = np.stack([lo, hi], -1).reshape(packed.shape[0], -1)
    mag = np.array([float(v) for v in E2M1_MAG])[q & 7]
    v = np.where(q & 8, -mag, mag)
    sf = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    return v * np.repeat(sf, 16, axis=1)


def test_gemm_oracle_equals_library_matmul_of_decoded_operands(oracle_mod):
    rng = np.random.default_rng(31)
    M, N, K = 7, 5, 96
    ap = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    bp = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    ac = rng.integers(0, 127, (M, K // 16), dtype=np.uint8)
    bc = rng.integers(0, 127, (N, K // 16), dtype=np.uint8)
    sa, sb = float(np.float32(0.0123)), float(np.float32(3.5))
    Y, absY = oracle_mod.gemm_nvfp4(ap, ac, sa, bp, bc, sb)
    A, B = _decode_nvfp4(ap, ac), _decode_nvfp4(bp, bc)
    ref = (A @ B.T) * (sa * sb)
    np.testing.assert_allclose(Y, ref, rtol=1e-13, atol=1e-300)
    np.testing.assert_allclose(absY, (np.abs(A) @ np.abs(B).T) * abs(sa * sb), rtol=1e-13)


def test_gemm_oracle_hand_case(oracle_mod):
    """One row of A with codes 1.0 (0x2) everywhere at block scale 2 and one
    row of B with 6.0 (0x7) at block scale 0.5 over K = 32: Y = 32 * 2 * 3."""
    ap = np.full((1, 16), 0x22, np.uint8)
    bp = np.full((1, 16), 0x77, np.uint8)
    two = torch.tensor([2.0]).to(torch.float8_e4m3fn).view(torch.uint8).item()
    half = torch.tensor([0.5]).to(torch.float8_e4m3fn).view(torch.uint8).item()
    ac = np.full((1, 2), two, np.uint8)
    bc = np.full((1, 2), half, np.uint8)
    Y, _ = oracle_mod.gemm_nvfp4(ap, ac, 1.0, bp, bc, 1.0)
    assert Y[0, 0] == 32 * (1.0 * 2.0) * (6.0 * 0.5)


# ------------------------------------------------ activation-range calibration
def _act(seed, n_rows=64, C=256):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(n_rows, C, generator=g)
    x[:, 7] *= 40.0
    x[3, 11] = -900.0
    return bf16_bits(x.to(torch.bfloat16))


def test_abs_histogram_is_magnitude_bincount(oracle_mod):
    x = _act(1)
    h = oracle_mod.abs_histogram(x)
    ref = np.bincount((x & 0x7FFF).astype(np.int64).ravel(), minlength=32768)
    assert np.array_equal(h, ref.astype(np.uint64))
    # accumulates across chunks
    h2 = oracle_mod.abs_histogram(x[32:], oracle_mod.abs_histogram(x[:32]))
    assert np.array_equal(h2, h)


@pytest.mark.parametrize("p", [1.0, 0.9999, 0.999, 0.99, 0.5, 1e-9])
def test_quantile_is_order_statistic(oracle_mod, p):
    x = _act(2)
    mags = np.sort(np.abs(bits_to_f64(x)).ravel())
    k = max(1, math.ceil(p * mags.size))
    assert oracle_mod.quantile_magnitude(oracle_mod.abs_histogram(x), p) == mags[k - 1]


def test_static_scale_at_the_max_is_the_dynamic_scale(oracle_mod):
    x = _act(3)
    amax = np.abs(bits_to_f64(x)).max()
    assert oracle_mod.static_scale(amax) == oracle_mod.global_scale(x)
    y, p, c = oracle_mod.fake_quant_static(x, oracle_mod.global_scale(x))
    ry, rp, rc, _ = oracle_mod.fake_quant(x)
    assert np.array_equal(y, ry) and np.array_equal(p, rp) and np.array_equal(c, rc)


def test_static_scale_clips_outliers(oracle_mod):
    """s_g = 1/64: the largest block scale is 448/64 = 7 (code 0x7E), so a
    value of 100 saturates to 6 * 7 = 42 while the block's small values are
    encoded at scale 7."""
    x = np.zeros((1, 16), np.float32)
    x[0, :4] = [100.0, -3.5, 7.0, 0.0]
    u = f32_to_bf16_bits(x)
    y, p, c = oracle_mod.fake_quant_static(u, np.float32(1 / 64))
    yv = bits_to_f64(y)[0]
    assert c[0, 0] == 0x7E
    assert yv[0] == 42.0 and yv[1] == -3.5 and yv[2] == 7.0 and yv[3] == 0.0


def test_quant_error_is_sum_of_squared_differences(oracle_mod):
    x = _act(4)
    for s_g in (oracle_mod.global_scale(x), np.float32(oracle_mod.global_scale(x) / 8)):
        y, _, _ = oracle_mod.fake_quant_static(x, s_g, want_packed=False)
        ref = float(np.sum((bits_to_f64(x) - bits_to_f64(y)) ** 2))
        assert math.isclose(oracle_mod.quant_error(x, s_g), ref, rel_tol=1e-12)


# ------------------------------------------------------------ full Gram, GPTQ
def _np_e2m1_round(x, s):
    """Independent E2M1 rounding of fp64 values at scale s > 0: nearest grid
    magnitude, ties to the even magnitude index, saturating at 6; returns the
    signed quantised value v(q) * s and the code."""
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    a = np.abs(x)
    k = np.zeros(a.shape, np.int64)
    for i in range(7):
        thr = 0.5 * (grid[i] + grid[i + 1]) * s  # exact in fp64
        up = (a > thr) if i % 2 == 0 else (a >= thr)
        k = np.where(up, i + 1, k)
    code = k | np.where(np.signbit(x), 8, 0)
    return np.where(np.signbit(x), -1.0, 1.0) * grid[k] * s, code


def _gptq_obs_reference(W, S, H, damp):
    """GPTQ in its Optimal-Brain-Surgeon form (the GPTQ paper, before the
    Cholesky reformulation): quantise column j, move the remaining weights by
    -(w_j - q_j) / [H^-1]_jj * [H^-1]_{j,:}, then remove j from the inverse
    Hessian by one step of Gaussian elimination.  S: per-element scales."""
    C = H.shape[0]
    Hd = H + damp * np.mean(np.diag(H)) * np.eye(C)
    Hi = np.linalg.inv(Hd)
    Wc = W.copy()
    codes = np.zeros(W.shape, np.int64)
    at = np.zeros(W.shape)
    for j in range(C):
        at[:, j] = Wc[:, j]
        q, codes[:, j] = _np_e2m1_round(Wc[:, j], S[:, j])
        d = (Wc[:, j] - q) / Hi[j, j]
        Wc[:, j + 1:] -= np.outer(d, Hi[j, j + 1:])
        Hi = Hi - np.outer(Hi[:, j], Hi[j, :]) / Hi[j, j]
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return packed, at


def _gptq_case(oracle_mod, R, C, N, seed):
    W, X = _tiny_layer(R, C, N, seed)
    s_g = oracle_mod.global_scale(W)
    codes = oracle_mod.scale_search_max(W, s_g)
    H = oracle_mod.gram_full(X)
    S = np.repeat(np.array([[oracle_mod.effective_scale(s_g, c) for c in row] for row in codes],
                           np.float64), 16, axis=1)
    return W, X, s_g, codes, H, S


def test_full_gram_is_library_product(oracle_mod):
    W, X = _tiny_layer(4, 64, 40, 11)
    H = oracle_mod.gram_full(X)
    Xf = bits_to_f64(X)
    np.testing.assert_allclose(H, Xf.T @ Xf, rtol=1e-14, atol=0)
    # its 16x16 diagonal blocks are the block-diagonal Gram
    Hb = oracle_mod.gram(X)
    for j in range(4):
        np.testing.assert_array_equal(H[16 * j:16 * j + 16, 16 * j:16 * j + 16], Hb[j])


def test_gptq_factor_is_cholesky_of_inverse(oracle_mod):
    _, X = _tiny_layer(2, 48, 64, 12)
    H = oracle_mod.gram_full(X)
    U = oracle_mod.gptq_factor(H, 0.01)
    Hd = H + 0.01 * np.mean(np.diag(H)) * np.eye(48)
    assert np.all(np.tril(U, -1) == 0) and np.all(np.diag(U) > 0)
    np.testing.assert_allclose(U.T @ U, np.linalg.inv(Hd), rtol=1e-9,
                               atol=1e-12 * np.abs(np.linalg.inv(Hd)).max())


def test_gptq_with_diagonal_hessian_is_plain_rounding(oracle_mod):
    W, X, s_g, codes, _, _ = _gptq_case(oracle_mod, 16, 64, 32, 13)
    rng = np.random.default_rng(13)
    H = np.diag(rng.uniform(0.5, 40.0, 64))
    np.testing.assert_array_equal(oracle_mod.gptq(W, s_g, codes, H, 0.01),
                                  oracle_mod.quantize_pack(W, s_g, codes))


def test_gptq_two_coupled_columns_closed_form(oracle_mod):
    # H couples only columns 0 and 1: after column 0 is rounded, the output
    # error is least when w_1 moves by (w_0 - q_0) H01 / H11 (dampened H);
    # every other column is rounded as it is
    W, X, s_g, codes, _, S = _gptq_case(oracle_mod, 16, 32, 32, 14)
    H = np.eye(32) * 3.0
    H[0, 0], H[1, 1], H[0, 1], H[1, 0] = 5.0, 2.0, 1.5, 1.5
    damp = 0.01
    Hd = H + damp * np.mean(np.diag(H)) * np.eye(32)
    U = oracle_mod.gptq_factor(H, damp)
    packed, at = oracle_mod.gptq_rows(W, s_g, codes, U, np.arange(16))
    Wf = bits_to_f64(W)
    q0, _ = _np_e2m1_round(Wf[:, 0], S[:, 0])
    np.testing.assert_allclose(at[:, 1], Wf[:, 1] + (Wf[:, 0] - q0) * Hd[0, 1] / Hd[1, 1],
                               rtol=1e-12, atol=1e-15)
    np.testing.assert_array_equal(at[:, 2:], Wf[:, 2:])
    np.testing.assert_array_equal(at[:, 0], Wf[:, 0])


@pytest.mark.parametrize("R,C,N,seed", [(12, 48, 80, 15), (7, 64, 30, 16)])
def test_gptq_equals_obs_elimination_form(oracle_mod, R, C, N, seed):
    W, X, s_g, codes, H, S = _gptq_case(oracle_mod, R, C, N, seed)
    ref_packed, ref_at = _gptq_obs_reference(bits_to_f64(W), S, H, 0.01)
    U = oracle_mod.gptq_factor(H, 0.01)
    packed, at = oracle_mod.gptq_rows(W, s_g, codes, U, np.arange(R))
    np.testing.assert_allclose(at, ref_at, rtol=1e-9, atol=1e-12)
    np.testing.assert_array_equal(packed, ref_packed)
    np.testing.assert_array_equal(oracle_mod.gptq(W, s_g, codes, H, 0.01), packed)


def test_gptq_not_positive_definite_is_reported(oracle_mod):
    W, X, s_g, codes, H, _ = _gptq_case(oracle_mod, 4, 32, 16, 17)
    bad = np.eye(32)
    bad[5, 5] = -4.0
    with pytest.raises(Exception):
        oracle_mod.gptq(W, s_g, codes, bad, 0.0)
