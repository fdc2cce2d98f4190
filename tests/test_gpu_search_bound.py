"""The Local-Hessian screen's error bound on the device.

The search screens candidates in fp32 with the 16x16 product on the tensor
cores and re-scores in fp64 whatever its error bound cannot separate (the
exhaustive per-block argmin of the Local-Hessian write-up "4 比特量化到底让模型
笨了多少？", section "A different objective").  The bound rests on one property
of the hardware: a 16x8x16 f16 MMA with fp32 accumulation errs by at most
2^-18 of the sum of the magnitudes of its products and of c.  The first test
checks that property on adversarial tiles through the very instruction the
screen uses; the second runs the search on blocks that lie close to the
E2M1 grid (where the objective is tiny next to ||L^T w||^2 and the screen's
absolute error matters most) and compares every block with the oracle."""
import numpy as np
import pytest
import torch

import oracle
from conftest import bf16_bits, bits_to_f64, f32_to_bf16_bits, record_stat
from parity_util import check_search_codes

pytestmark = pytest.mark.gpu

KAPPA = 2.0 ** -18


@pytest.fixture(scope="module")
def nv():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from scale_calibration_nvfp4_b200 import build, nvfp4
    build.build()
    nvfp4.lib()
    oracle.lib()
    return nvfp4


def _f16(rng, shape, lo_exp, hi_exp):
    """float16 values sign * (1 + m/1024) * 2^e, e uniform in [lo_exp, hi_exp]."""
    e = rng.integers(lo_exp, hi_exp + 1, shape)
    m = rng.integers(0, 1024, shape)
    s = rng.choice([-1.0, 1.0], shape)
    return (s * (1 + m / 1024.0) * np.exp2(e)).astype(np.float16)


def test_mma_accumulation_within_the_screen_bound(nv):
    """d = a b + c through the screen's MMA on tiles built to stress the
    accumulation: products over 30 binades, cancelling sums, one large term
    with many small ones, c far above or near minus the product sum, and the
    screen's own operand shapes (E2M1 values or bf16 weights against the f16
    high and low parts of a factor).  Every output stays within 2^-18 of the
    sum of magnitudes of the 17 addends of the exact fp64 result."""
    rng = np.random.default_rng(123)
    n = 4096
    cases = []
    # wide exponent ranges, random signs
    cases.append((_f16(rng, (n, 16, 16), -14, 7), _f16(rng, (n, 16, 8), -14, 7), None))
    # one dominant product per output, the rest 2^-10..2^-24 of it
    a = _f16(rng, (n, 16, 16), -12, -1)
    a[:, :, 0] = _f16(rng, (n, 16), 6, 8)
    cases.append((a, _f16(rng, (n, 16, 8), -2, 2), None))
    # E2M1 values against a high / low factor split (the screen's u)
    v = rng.choice(np.array([0, .5, 1, 1.5, 2, 3, 4, 6, -.5, -1, -1.5, -2, -3, -4, -6],
                            np.float32), (n, 16, 16)).astype(np.float16)
    L = (np.clip(rng.standard_normal((n, 16, 8)), -3.9, 3.9)
         * np.exp2(rng.integers(0, 14, (n, 1, 1)))).astype(np.float32)
    hi = L.astype(np.float16)
    lo = (L - hi.astype(np.float32)).astype(np.float16)
    cases.append((v, hi, None))
    cases.append((v, lo, None))
    # bf16 weights (exact in f16 at the screen's row scale) against the split
    w = bits_to_f64(f32_to_bf16_bits(rng.standard_normal((n, 16, 16)) * 2.0 ** 13)).astype(np.float16)
    cases.append((w, hi, None))
    worst = 0.0
    for a, b, _ in cases:
        exact_ab = np.einsum("nmk,nkj->nmj", a.astype(np.float64), b.astype(np.float64))
        mag_ab = np.einsum("nmk,nkj->nmj", np.abs(a.astype(np.float64)),
                           np.abs(b.astype(np.float64)))
        for c_kind in range(4):
            if c_kind == 0:
                c = np.zeros((n, 16, 8), np.float32)
            elif c_kind == 1:   # c close to minus the sum: heavy cancellation
                c = (-exact_ab * (1 + rng.standard_normal((n, 16, 8)) * 2.0 ** -12)).astype(np.float32)
            elif c_kind == 2:   # c far above the products
                c = (mag_ab * 2.0 ** rng.integers(4, 20, (n, 16, 8))
                     * rng.choice([-1.0, 1.0], (n, 16, 8))).astype(np.float32)
            else:               # the chained form: c is a first product's result
                c = exact_ab.astype(np.float32)
            d = nv.self_test_mma(torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda(),
                                 torch.from_numpy(c).cuda()).cpu().numpy().astype(np.float64)
            exact = exact_ab + c.astype(np.float64)
            mag = mag_ab + np.abs(c.astype(np.float64))
            ok = mag > 0
            ratio = np.abs(d - exact)[ok] / mag[ok]
            assert np.all(np.abs(d - exact)[~ok] == 0)
            worst = max(worst, float(ratio.max()))
    assert worst <= KAPPA, worst
    record_stat("MMA accumulation (screen's instruction)",
                worst_error_over_sum_of_magnitudes="2^%.2f" % np.log2(max(worst, 2.0 ** -60)),
                assumed="2^-18")


def _near_grid_weights(rng, R, C):
    """bf16 [R, C] whose blocks sit close to the E2M1 grid at one or more
    scales; element [0, 0] = 2688 * 2^-12 makes the tensor scale 2^-12
    exactly, so 6 s_eff and grid values times s_eff are bf16 values."""
    e4m3 = np.array([oracle.e4m3_value(c) for c in range(1, 127)])
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float64)
    sg = 2.0 ** -12
    nb = C // 16
    shape = (R, nb, 16)
    kind = rng.integers(0, 4, (R, nb))[..., None]
    s = (sg * e4m3[rng.integers(40, 100, (R, nb))])[..., None]
    top = rng.integers(0, 16, (R, nb))[..., None] == np.arange(16)   # one element at 6 s
    # kind 0: the others 2^-6 .. 2^-14 of 6 s
    k0 = 6 * s * np.exp2(-rng.integers(6, 15, shape)) * (1 + rng.integers(0, 8, shape) / 8)
    # kind 1: grid values at s, zeros lifted by 2^-10 .. 2^-18 of the maximum
    g1 = grid[rng.integers(0, 8, shape)] * s
    k1 = np.where(g1 == 0, 6 * s * np.exp2(-rng.integers(10, 19, shape)), g1)
    # kind 2: grid values at two related scales
    s2 = s * rng.choice([2.0, 1.5, 0.75], (R, nb, 1))
    k2 = np.where(rng.integers(0, 2, shape).astype(bool), grid[rng.integers(0, 8, shape)] * s,
                  grid[rng.integers(0, 8, shape)] * s2)
    # kind 3: non-zero grid values at s (moved by one or two bf16 ulps below)
    k3 = grid[rng.integers(1, 8, shape)] * s
    W = np.select([kind == 0, kind == 1, kind == 2], [k0, k1, k2], k3)
    W = np.where(top, 6 * s, W) * rng.choice([-1.0, 1.0], shape)
    u = f32_to_bf16_bits(W.reshape(R, C).astype(np.float32))
    move = (kind[..., 0] == 3)[..., None] & (rng.random(shape) < 0.12)
    step = rng.choice(np.array([-2, -1, 1, 2], np.int32), shape)
    u = np.where(move.reshape(R, C), (u.astype(np.int32) + step.reshape(R, C)).astype(np.uint16), u)
    u[0, 0] = f32_to_bf16_bits(np.array([2688.0 * sg], np.float32))[0]
    return np.ascontiguousarray(u)


def test_search_near_grid_blocks_every_block(nv):
    """Every block of a 2048 x 4096 weight built close to the E2M1 grid (one
    element at 6 s_eff and the rest 2^-6..2^-14 of it; grid values with their
    zeros lifted by 2^-10..2^-18 of the block maximum; grid values at two
    related scales; grid values moved by one or two bf16 ulps), searched
    under the dense layer's Gram (eight calibration channels x50) and under
    H = I, against the oracle.  Many of these blocks have a best objective
    between 2^-40 and 2^-16 of ||L^T w||^2, the window where the screen's
    error is largest next to the objective."""
    from scale_calibration_nvfp4_b200 import workloads
    rng = np.random.default_rng(77)
    R, C = 2048, 4096
    wu = _near_grid_weights(rng, R, C)
    W = torch.from_numpy(wu.view(np.int16)).view(torch.bfloat16).cuda()
    _, X = workloads.layer_inputs("dense", "cuda")
    s_g = nv.global_scale(W)
    sg = s_g.item()
    assert sg == 2.0 ** -12 and sg == oracle.global_scale(wu)
    H = torch.zeros(C // 16, 16, 16, device="cuda")
    nv.hessian_accumulate(X, H)
    H64 = H.cpu().numpy().astype(np.float64)
    clh = nv.scale_search_local_hessian(W, s_g, H).cpu().numpy()
    rc, best, second = oracle.scale_search_lh(wu, sg, H64, runner_up=True)
    n_lh = check_search_codes(clh, rc, wu, sg, H64)
    cm = nv.scale_search_mse(W, s_g).cpu().numpy()
    rcm, bm, sm = oracle.scale_search_mse(wu, sg, runner_up=True)
    n_mse = check_search_codes(cm, rcm, wu, sg)
    # how many blocks probe the window: best / ||L^T w||^2 = best / (w H w^T)
    wf = bits_to_f64(wu).reshape(R, C // 16, 16)
    pp = np.einsum("rbi,bij,rbj->rb", wf, H64, wf)
    rel = best / np.where(pp > 0, pp, 1.0)
    window = int(np.count_nonzero((rel > 2.0 ** -40) & (rel < 2.0 ** -16)))
    assert window > 10000, window
    record_stat("near-grid 2048x4096", blocks=R * C // 16, lh_blocks_in_window=window,
                lh_near_ties=int(np.count_nonzero(second - best <= 1e-6 * second)),
                lh_codes_differing=n_lh,
                mse_near_ties=int(np.count_nonzero(sm - bm <= 1e-6 * sm)),
                mse_codes_differing=n_mse)
