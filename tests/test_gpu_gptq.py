"""GPU parity of the full Gram and of GPTQ rounding against the CPU oracle.

Full Gram: fp32 accumulation of exact bf16 products, so every entry lies
within (N - 1) 2^-24 sum_t |x_ta x_tb| of the fp64 value.  GPTQ: the GPU runs
the column loop in fp64 in another (inverse-free, lazily batched) order than
the oracle, so the values at rounding agree to about 1e-13 relative; the
packed codes must be bit-exact on every row whose oracle values at rounding
all stay more than 1e-9 (relative) away from an E2M1 rounding midpoint times
their scale (past column 0, where both sides round w itself)."""
import numpy as np
import pytest
import torch

import oracle
from conftest import bf16_bits, bits_to_f64, record_stat
from parity_util import GRAM_REL, rel_frobenius

pytestmark = pytest.mark.gpu

MIDPOINTS = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)


@pytest.fixture(scope="module")
def nv():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from scale_calibration_nvfp4_b200 import build, nvfp4
    build.build()
    nvfp4.lib()
    oracle.lib()
    return nvfp4


def rand_bf16(shape, seed, std=1.0, outlier_cols=(), factor=1.0):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(*shape, generator=g) * std
    for c in outlier_cols:
        x[..., c] *= factor
    return x.to(torch.bfloat16)


def scales_per_element(s_g, codes):
    S = np.array([[oracle.effective_scale(s_g, int(c)) for c in row] for row in codes], np.float64)
    return np.repeat(S, 16, axis=1)


def near_tie_rows(wq, S, rel=1e-9):
    """Rows holding a value at rounding within rel of a midpoint times its
    scale (past column 0).  A scale of 0 has no midpoint: every value
    encodes to index 0 there, whatever it is."""
    a = np.abs(wq[:, 1:])
    S = S[:, 1:]
    near = np.zeros(wq.shape[0], bool)
    for m in MIDPOINTS:
        thr = m * S
        near |= np.any((np.abs(a - thr) <= rel * thr) & (S > 0), axis=1)
    return near


def compare_gptq(gpu_packed, ref_packed, wq, S, max_near_frac=0.0):
    near = near_tie_rows(wq, S)
    assert near.mean() <= max_near_frac, near.mean()
    ok = ~near
    np.testing.assert_array_equal(np.asarray(gpu_packed)[ok], np.asarray(ref_packed)[ok])
    return int(near.sum())


# ------------------------------------------------------------------ full Gram
@pytest.mark.parametrize("N,C", [(300, 256), (77, 48), (1, 16), (2048, 64), (129, 400)])
def test_full_gram_matches_oracle(nv, N, C):
    x = rand_bf16((N, C), N + C, 1.0, outlier_cols=(3,), factor=30.0)
    g = torch.Generator().manual_seed(5)
    H0 = torch.randn(C, C, generator=g)
    H = H0.clone().cuda()
    nv.hessian_full_accumulate(x.cuda(), H)
    ref = H0.double().numpy() + oracle.gram_full(bf16_bits(x))
    assert rel_frobenius(H.cpu().double().numpy(), ref) <= GRAM_REL
    xa = np.abs(bits_to_f64(bf16_bits(x)))
    bound = (max(N, 2) - 1) * 2.0 ** -24 * (xa.T @ xa) + 2.0 ** -23 * np.abs(ref)
    assert np.all(np.abs(H.cpu().double().numpy() - ref) <= bound * 1.01 + 1e-30)


def test_full_gram_empty_tokens_is_noop(nv):
    H = torch.full((32, 32), 2.5, device="cuda")
    nv.hessian_full_accumulate(torch.empty(0, 32, dtype=torch.bfloat16, device="cuda"), H)
    assert torch.all(H == 2.5)


def test_full_gram_dense_layer_sampled(nv):
    from scale_calibration_nvfp4_b200 import workloads
    _, X = workloads.layer_inputs("dense", "cpu")
    N, C = X.shape
    H = torch.zeros(C, C, device="cuda")
    nv.hessian_full_accumulate(X.cuda(), H)
    Hc = H.cpu().double().numpy()
    Xd = bits_to_f64(bf16_bits(X))
    rng = np.random.default_rng(0)
    a, b = rng.integers(0, C, 3000), rng.integers(0, C, 3000)
    ref = np.einsum("ti,ti->i", Xd[:, a], Xd[:, b])
    absum = np.einsum("ti,ti->i", np.abs(Xd[:, a]), np.abs(Xd[:, b]))
    err = np.abs(Hc[a, b] - ref)
    assert np.all(err <= (N - 1) * 2.0 ** -24 * absum * 1.01 + 2.0 ** -23 * np.abs(ref))


# ----------------------------------------------------------------------- GPTQ
def _case(R, C, N, seed, rule):
    W = rand_bf16((R, C), seed, 0.02)
    X = rand_bf16((N, C), seed + 100, 1.0, outlier_cols=(C // 3,), factor=25.0)
    wu, xu = bf16_bits(W), bf16_bits(X)
    s_g = oracle.global_scale(wu)
    Hf = oracle.gram_full(xu).astype(np.float32)
    if rule == "lh":
        Hb = np.stack([Hf[16 * j:16 * j + 16, 16 * j:16 * j + 16] for j in range(C // 16)])
        codes = oracle.scale_search_lh(wu, s_g, Hb.astype(np.float64))[0]
    else:
        codes = oracle.scale_search_max(wu, s_g)
    return W, wu, s_g, codes, Hf


@pytest.mark.parametrize("R,C,N,seed,rule,damp", [
    (40, 96, 200, 1, "lh", 0.01),     # Local-Hessian scales, three panels
    (130, 80, 64, 2, "max", 0.01),    # ragged rows, a 16-wide last panel, rank-deficient H
    (8, 16, 40, 4, "max", 0.0),       # one block, no dampening
    (300, 512, 512, 5, "lh", 0.01),   # the tiny layer's width
])
def test_gptq_matches_oracle(nv, R, C, N, seed, rule, damp):
    W, wu, s_g, codes, Hf = _case(R, C, N, seed, rule)
    out = nv.gptq(W.cuda(), torch.tensor([s_g]).cuda(), torch.from_numpy(codes).cuda(),
                  torch.from_numpy(Hf).cuda(), damp)
    U = oracle.gptq_factor(Hf.astype(np.float64), damp)
    ref, wq = oracle.gptq_rows(wu, s_g, codes, U, np.arange(R))
    compare_gptq(out.cpu().numpy(), ref, wq, scales_per_element(s_g, codes))
    assert nv.get_device_status() == "NVFP4_OK"


def test_gptq_batch_of_experts(nv):
    cases = [_case(24, 48, 100, 10 + e, "max") for e in range(3)]
    W = torch.stack([c[0] for c in cases])
    s_g = torch.tensor([c[2] for c in cases])
    codes = np.stack([c[3] for c in cases])
    H = np.stack([c[4] for c in cases])
    out = nv.gptq(W.cuda(), s_g.cuda(), torch.from_numpy(codes).cuda(), torch.from_numpy(H).cuda(),
                  0.05).cpu().numpy()
    for e, (_, wu, sg, cd, Hf) in enumerate(cases):
        U = oracle.gptq_factor(Hf.astype(np.float64), 0.05)
        ref, wq = oracle.gptq_rows(wu, sg, cd, U, np.arange(24))
        compare_gptq(out[e], ref, wq, scales_per_element(sg, cd))


def test_gptq_diagonal_hessian_is_plain_rounding(nv):
    W, wu, s_g, codes, _ = _case(64, 128, 10, 20, "max")
    H = torch.diag(torch.linspace(0.5, 9.0, 128))
    sg, cd = torch.tensor([s_g]).cuda(), torch.from_numpy(codes).cuda()
    out = nv.gptq(W.cuda(), sg, cd, H.cuda(), 0.01)
    np.testing.assert_array_equal(out.cpu().numpy(), oracle.quantize_pack(wu, s_g, codes))


def test_gptq_blocks_with_zero_scale(nv):
    """Blocks whose scale code is 0: an all-zero block column, a zero row,
    signed zeros, and blocks about 1e-7 of the tensor maximum, whose max-rule
    code rounds to 0 although their values are not zero.  Every value there
    gets magnitude index 0 with its sign, and all of it is the error carried
    to the later columns; every row against the oracle."""
    R, C = 64, 256
    W = rand_bf16((R, C), 30, 0.02)
    W[:, 16:32] = 0.0
    W[5, :] = 0.0
    W[7, 96:112] = -0.0
    W[:, 64:80] = W[:, 64:80] * 1e-7
    X = rand_bf16((300, C), 130, 1.0, outlier_cols=(C // 3,), factor=25.0)
    wu = bf16_bits(W)
    s_g = oracle.global_scale(wu)
    Hf = oracle.gram_full(bf16_bits(X)).astype(np.float32)
    codes = oracle.scale_search_max(wu, s_g)
    assert np.all(codes[:, 1] == 0) and np.all(codes[:, 4] == 0)
    assert np.count_nonzero(wu.reshape(R, C // 16, 16)[:, 4] & 0x7FFF) > R
    out = nv.gptq(W.cuda(), torch.tensor([s_g]).cuda(), torch.from_numpy(codes).cuda(),
                  torch.from_numpy(Hf).cuda(), 0.01)
    U = oracle.gptq_factor(Hf.astype(np.float64), 0.01)
    ref, wq = oracle.gptq_rows(wu, s_g, codes, U, np.arange(R))
    compare_gptq(out.cpu().numpy(), ref, wq, scales_per_element(s_g, codes), max_near_frac=0.0)
    assert nv.get_device_status() == "NVFP4_OK"


def test_gptq_not_positive_definite_reports(nv):
    W, wu, s_g, codes, _ = _case(16, 32, 10, 21, "max")
    sg, cd = torch.tensor([s_g]).cuda(), torch.from_numpy(codes).cuda()
    H = -torch.eye(32)
    nv.gptq(W.cuda(), sg, cd, H.cuda(), 0.0)
    assert nv.get_device_status() == "NVFP4_ERR_NOT_POSITIVE_DEFINITE"
    # the context stays usable and the status was cleared
    nv.gptq(W.cuda(), sg, cd, torch.eye(32).cuda(), 0.0)
    assert nv.get_device_status() == "NVFP4_OK"


def test_gptq_dense_layer_every_row(nv):
    """The dense projection (W 4096x4096, H from its 2048 calibration tokens)
    in the launch configuration of the benchmark, Local-Hessian block codes;
    every row's GPTQ codes against the oracle, no row screened out."""
    from scale_calibration_nvfp4_b200 import workloads
    W, X = workloads.layer_inputs("dense", "cpu")
    R, C = W.shape
    wu, xd = bf16_bits(W), bits_to_f64(bf16_bits(X))
    Hf = (xd.T @ xd).astype(np.float32)
    s_g = oracle.global_scale(wu)
    Hb = np.stack([Hf[16 * j:16 * j + 16, 16 * j:16 * j + 16] for j in range(C // 16)]).astype(np.float64)
    codes, _ = oracle.scale_search_lh(wu, s_g, Hb)
    out = nv.gptq(W.cuda(), torch.tensor([s_g]).cuda(), torch.from_numpy(codes).cuda(),
                  torch.from_numpy(Hf).cuda(), 0.01).cpu().numpy()
    U = oracle.gptq_factor(Hf.astype(np.float64), 0.01)
    rows = np.arange(R)
    ref, wq = oracle.gptq_rows(wu, s_g, codes, U, rows)
    n = compare_gptq(out, ref, wq, scales_per_element(s_g, codes), max_near_frac=0.0)
    record_stat("gptq dense 4096x4096", rows_checked=R, rows_near_a_midpoint=n)
    assert nv.get_device_status() == "NVFP4_OK"


def test_gptq_moe_experts_every_row(nv):
    """All 128 experts (768 x 2048) in one batched call; four experts (the
    most and fewest routed tokens among them) carry their routed tokens'
    Gram, the rest an identity Hessian; every row of the four against the
    oracle, no row screened out."""
    from scale_calibration_nvfp4_b200 import workloads
    W, X, off = workloads.moe_inputs("cpu")
    G, R, C = W.shape
    wu = bf16_bits(W)
    H = np.broadcast_to(np.eye(C, dtype=np.float32), (G, C, C)).copy()
    s_g = np.array([oracle.global_scale(wu[g]) for g in range(G)], np.float32)
    codes = np.stack([oracle.scale_search_max(wu[g], s_g[g]) for g in range(G)])
    picks = [0, 1, 63, 127]
    for g in picks:
        xd = bits_to_f64(bf16_bits(X[int(off[g]):int(off[g + 1])]))
        H[g] = (xd.T @ xd).astype(np.float32)
    out = nv.gptq(W.cuda(), torch.from_numpy(s_g).cuda(), torch.from_numpy(codes).cuda(),
                  torch.from_numpy(H).cuda(), 0.01).cpu().numpy()
    rows = np.arange(R)
    near = 0
    for g in picks:
        U = oracle.gptq_factor(H[g].astype(np.float64), 0.01)
        ref, wq = oracle.gptq_rows(wu[g], float(s_g[g]), codes[g], U, rows)
        near += compare_gptq(out[g], ref, wq, scales_per_element(float(s_g[g]), codes[g]),
                             max_near_frac=0.0)
    record_stat("gptq moe 4 experts x 768x2048", rows_checked=len(picks) * R,
                rows_near_a_midpoint=near)
    # an identity Hessian leaves the rounding plain
    np.testing.assert_array_equal(out[2], oracle.quantize_pack(wu[2], float(s_g[2]), codes[2]))
    assert nv.get_device_status() == "NVFP4_OK"
