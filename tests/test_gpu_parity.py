"""GPU parity: every C-ABI entry point against the CPU oracle, element by
element, on seeded inputs (small cases that span many tiles with ragged
tails, edge cases, and samples of the full-size workloads)."""
import math

import numpy as np
import pytest
import torch

import oracle
from conftest import bf16_bits, bits_to_f64, f32_to_bf16_bits
from parity_util import GRAM_REL, check_search_codes, rel_frobenius

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from scale_calibration_nvfp4_b200 import build, nvfp4
    build.build()
    nvfp4.lib()
    oracle.lib()
    return nvfp4


def dev_bf16(u16):
    t = torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(torch.bfloat16)
    return t.cuda()


def rand_bf16(shape, seed, std=1.0, outlier_frac=0.0, factor=1.0):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(*shape, generator=g) * std
    n = int(outlier_frac * x.numel())
    if n:
        idx = torch.randperm(x.numel(), generator=g)[:n]
        x.view(-1)[idx] *= factor
    return x.to(torch.bfloat16)


# ------------------------------------------------------------ global scale
def test_global_scale_bitexact(nv):
    x = rand_bf16((5, 4104), 1, 0.02, 0.01, 30.0)
    s = nv.global_scale(x.cuda(), batch=5).cpu().numpy()
    xu = bf16_bits(x)
    for b in range(5):
        assert s[b] == oracle.global_scale(xu[b]), b
    z = torch.zeros(3, 64, dtype=torch.bfloat16, device="cuda")
    assert torch.equal(nv.global_scale(z, batch=3).cpu(), torch.ones(3))
    # one element only, and a subnormal-range maximum
    t = torch.zeros(16, dtype=torch.bfloat16)
    t[7] = -2.0 ** -130
    assert nv.global_scale(t.cuda()).item() == oracle.global_scale(bf16_bits(t))
    assert nv.get_device_status() == "NVFP4_OK"


def test_global_scale_nonfinite_reports(nv):
    x = torch.ones(2, 32, dtype=torch.bfloat16)
    x[1, 5] = float("nan")
    s = nv.global_scale(x.cuda(), batch=2).cpu()
    assert s[0].item() == oracle.global_scale(bf16_bits(x[0]))
    assert torch.isnan(s[1])
    assert nv.get_device_status() == "NVFP4_ERR_NONFINITE"
    assert nv.get_device_status() == "NVFP4_OK"  # cleared by the read


def test_bounded_wait_reports_timeout_and_context_survives(nv):
    """A wait that nothing completes gives up (about one second), the host
    reads NVFP4_ERR_DEVICE_TIMEOUT, and the context still runs kernels.
    While the timeout is on record, Gram calls (pool and no-alloc forms,
    plain and grouped) leave H exactly as it was; after the read clears it,
    they accumulate again."""
    assert nv.get_device_status() == "NVFP4_OK"
    x = rand_bf16((300, 64), 12)
    H0 = torch.randn(4, 16, 16, generator=torch.Generator().manual_seed(3)).cuda()
    nv.self_test_device_timeout()
    H = H0.clone()
    nv.hessian_accumulate(x.cuda(), H)
    nv.hessian_accumulate_noalloc(x.cuda(), H)
    Hg = H0.clone().view(1, 4, 16, 16)
    nv.hessian_accumulate_grouped(x.cuda(), torch.tensor([0, 300]).cuda(), Hg)
    torch.cuda.synchronize()
    assert torch.equal(H, H0) and torch.equal(Hg.view(4, 16, 16), H0)
    assert nv.get_device_status() == "NVFP4_ERR_DEVICE_TIMEOUT"
    assert nv.get_device_status() == "NVFP4_OK"  # cleared by the read
    H = torch.zeros(4, 16, 16, device="cuda")
    nv.hessian_accumulate(x.cuda(), H)
    assert rel_frobenius(H.cpu().numpy().astype(np.float64), oracle.gram(bf16_bits(x))) <= GRAM_REL
    assert nv.get_device_status() == "NVFP4_OK"


# ------------------------------------------------------------ max rule
def test_max_rule_bitexact_with_edge_blocks(nv):
    x = rand_bf16((67, 176), 2, 0.02, 0.01, 20.0)
    x[3, :16] = 0                               # all-zero block
    x[4, 16:32] = 1e-3 * x[4, 16:32]            # small block
    x[5, 32:48] = 0
    x[5, 40] = -1e-7                            # single tiny non-zero: subnormal / zero code
    x[6, 48:64] = x.abs().max()                 # saturating block
    s_g = nv.global_scale(x.cuda())
    codes = nv.scale_search_max(x.cuda(), s_g).cpu().numpy()
    ref = oracle.scale_search_max(bf16_bits(x), s_g.item())
    np.testing.assert_array_equal(codes, ref)
    assert codes[3, 0] == 0 and codes[6, 3] == 0x7E


def test_max_rule_exact_midpoint_ties(nv):
    # block maxima exactly on E4M3 midpoints times 6 s_g (s_g = 2^-5 keeps every
    # product a bf16 value): ties go to the even code
    s_g = np.float32(2.0 ** -5)
    vals = [0.5 * (oracle.e4m3_value(c) + oracle.e4m3_value(c + 1)) * 6 * float(s_g)
            for c in range(0, 126)]
    blocks = np.zeros((len(vals), 16), np.float32)
    blocks[:, 0] = vals
    u = f32_to_bf16_bits(blocks)
    assert np.array_equal(bits_to_f64(u)[:, 0], np.array(vals))
    sg = torch.tensor([s_g], device="cuda")
    codes = nv.scale_search_max(dev_bf16(u), sg).cpu().numpy()
    ref = oracle.scale_search_max(u, s_g)
    np.testing.assert_array_equal(codes, ref)
    assert np.all(ref[:, 0] % 2 == 0)


# ------------------------------------------------------------ E2M1 encode
@pytest.mark.parametrize("s_g,code", [(1.0, 0x38), (1.0, 0x56), (2.0 ** -5, 0x7E),
                                      (0.0123456, 0x31), (3.3e-3, 0x01), (7.1e-4, 0x77),
                                      (1.0, 0x07), (0.5, 0x00),
                                      # scales next to the threshold of the kernels'
                                      # "no quotient near a midpoint" certificate
                                      # (1 + 9 ulp passes it, 1 + 8 ulp does not)
                                      (1.0 + 9 * 2.0 ** -23, 0x38), (1.0 + 8 * 2.0 ** -23, 0x38),
                                      (2.0 - 9 * 2.0 ** -23, 0x38), (1.0 + 9 * 2.0 ** -23, 0x3B)])
def test_encode_every_bf16_pattern(nv, s_g, code):
    """All 65,536 bf16 bit patterns (NaN/Inf replaced by 0) through the
    packed encode at one block scale: bit-exact against the oracle."""
    u = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    exp = (u >> 7) & 0xFF
    u[exp == 0xFF] = 0
    W = u.reshape(256, 256)
    s_g = np.float32(s_g)
    codes = np.full((256, 16), code, np.uint8)
    packed = nv.quantize_pack(dev_bf16(W), torch.tensor([s_g], device="cuda"),
                              torch.from_numpy(codes).cuda()).cpu().numpy()
    ref = oracle.quantize_pack(W, s_g, codes)
    np.testing.assert_array_equal(packed, ref)


def test_encode_exact_midpoints(nv):
    # values exactly on E2M1 midpoints at scale s_eff: the tie rule decides
    s_g = np.float32(1.0)
    codes = np.array([[0x30, 0x38, 0x3A, 0x44]], np.uint8)  # 0.5, 1, 1.25, 2.5
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.5]
    rows = []
    for c in codes[0]:
        s = oracle.effective_scale(s_g, int(c))
        rows += [m * s for m in mids] + [-m * s for m in mids]
    u = f32_to_bf16_bits(np.array(rows, np.float32)).reshape(1, 64)
    assert np.array_equal(bits_to_f64(u).ravel(), np.array(rows))
    packed = nv.quantize_pack(dev_bf16(u), torch.tensor([s_g], device="cuda"),
                              torch.from_numpy(codes).cuda()).cpu().numpy()
    np.testing.assert_array_equal(packed, oracle.quantize_pack(u, s_g, codes))


# ------------------------------------------------------------ pack / dequant
@pytest.mark.parametrize("shape", [(1, 16), (37, 80), (3, 4096), (129, 272)])
def test_pack_dequant_bitexact(nv, shape):
    R, C = shape
    x = rand_bf16(shape, R * 7 + C, 0.02, 0.02, 25.0)
    xu = bf16_bits(x)
    s_g = nv.global_scale(x.cuda())
    assert s_g.item() == oracle.global_scale(xu)
    g = torch.Generator().manual_seed(R + C)
    codes = torch.randint(0, 127, (R, C // 16), generator=g, dtype=torch.int32).to(torch.uint8)
    codes.view(-1)[:4] = torch.tensor([0, 1, 8, 126], dtype=torch.uint8)[: codes.numel()]
    packed = nv.quantize_pack(x.cuda(), s_g, codes.cuda())
    ref_p = oracle.quantize_pack(xu, s_g.item(), codes.numpy())
    np.testing.assert_array_equal(packed.cpu().numpy(), ref_p)
    y = nv.dequantize(packed, codes.cuda(), s_g)
    ref_y = oracle.dequantize(ref_p, codes.numpy(), s_g.item())
    np.testing.assert_array_equal(bf16_bits(y), ref_y)


def test_batched_pack_dequant_per_expert_scale(nv):
    x = rand_bf16((4, 24, 64), 31, 0.02)
    s_g = nv.global_scale(x.cuda(), batch=4)
    codes = nv.scale_search_max(x.cuda(), s_g)
    packed = nv.quantize_pack(x.cuda(), s_g, codes)
    y = nv.dequantize(packed, codes, s_g)
    xu = bf16_bits(x)
    for b in range(4):
        sg = s_g[b].item()
        assert sg == oracle.global_scale(xu[b])
        rc = oracle.scale_search_max(xu[b], sg)
        np.testing.assert_array_equal(codes[b].cpu().numpy(), rc)
        rp = oracle.quantize_pack(xu[b], sg, rc)
        np.testing.assert_array_equal(packed[b].cpu().numpy(), rp)
        np.testing.assert_array_equal(bf16_bits(y[b]), oracle.dequantize(rp, rc, sg))


# ------------------------------------------------------------ fake-quant
@pytest.mark.parametrize("shape", [(333, 96), (1, 16), (64, 8192)])
def test_fake_quant_bitexact(nv, shape):
    x = rand_bf16(shape, shape[0] + shape[1], 1.0)
    if shape[1] > 16:
        x[:, 5] *= 40
    y, packed, codes, s_g = nv.fake_quant(x.cuda(), want_packed=True)
    ry, rp, rc, rs = oracle.fake_quant(bf16_bits(x))
    assert s_g.item() == rs
    np.testing.assert_array_equal(codes.cpu().numpy(), rc)
    np.testing.assert_array_equal(packed.cpu().numpy(), rp)
    np.testing.assert_array_equal(bf16_bits(y), ry)
    y2, p2, c2, _ = nv.fake_quant(x.cuda(), want_packed=False)
    assert p2 is None and torch.equal(y2, y)


@pytest.mark.parametrize("N,C", [(512, 512), (1000, 48), (1, 16), (65, 144), (3000, 1040)])
def test_gram_matches_fp64(nv, N, C):
    x = rand_bf16((N, C), N + C)
    if C > 32:
        x[:, 3] *= 30
    H = torch.zeros(C // 16, 16, 16, device="cuda")
    nv.hessian_accumulate(x.cuda(), H)
    ref = oracle.gram(bf16_bits(x))
    Hc = H.cpu().numpy()
    assert rel_frobenius(Hc, ref) <= GRAM_REL
    for j in range(C // 16):
        assert rel_frobenius(Hc[j], ref[j]) <= GRAM_REL
    np.testing.assert_allclose(Hc, np.transpose(Hc, (0, 2, 1)), rtol=1e-6, atol=1e-6)


def test_gram_accumulates_and_is_deterministic(nv):
    x = rand_bf16((4096, 256), 77).cuda()
    H1 = torch.zeros(16, 16, 16, device="cuda")
    nv.hessian_accumulate(x, H1)
    H2 = torch.zeros(16, 16, 16, device="cuda")
    nv.hessian_accumulate(x, H2)
    assert torch.equal(H1, H2)
    H3 = torch.zeros(16, 16, 16, device="cuda")
    nv.hessian_accumulate(x[:1500], H3)
    nv.hessian_accumulate(x[1500:], H3)
    assert rel_frobenius(H3.cpu().numpy(), H1.cpu().numpy()) <= 1e-6
    H4 = H1.clone()
    nv.hessian_accumulate(x[:0], H4)  # zero tokens: no-op
    assert torch.equal(H4, H1)


def test_gram_grouped(nv):
    C = 96
    counts = [0, 1, 700, 2049, 0, 35, 4100, 17]
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    x = rand_bf16((int(offs[-1]), C), 99)
    H = torch.zeros(len(counts), C // 16, 16, 16, device="cuda")
    nv.hessian_accumulate_grouped(x.cuda(), torch.from_numpy(offs).cuda(), H)
    ref = oracle.gram_grouped(bf16_bits(x), offs, len(counts))
    Hc = H.cpu().numpy()
    for g, n in enumerate(counts):
        if n == 0:
            assert np.all(Hc[g] == 0)
        else:
            assert rel_frobenius(Hc[g], ref[g]) <= GRAM_REL, g


# ------------------------------------------------------------ scale search
def _layer(name):
    from scale_calibration_nvfp4_b200 import workloads
    W, X = workloads.layer_inputs(name, "cuda")
    return W, X


def test_tiny_layer_all_rules(nv):
    """Tiny-layer workload, every block: max, MSE and Local-Hessian codes."""
    W, X = _layer("tiny")
    wu = bf16_bits(W)
    s_g = nv.global_scale(W)
    sg = s_g.item()
    assert sg == oracle.global_scale(wu)
    H = torch.zeros(W.shape[1] // 16, 16, 16, device="cuda")
    nv.hessian_accumulate(X, H)
    H64 = H.cpu().numpy().astype(np.float64)
    assert rel_frobenius(H64, oracle.gram(bf16_bits(X))) <= GRAM_REL

    cmax = nv.scale_search_max(W, s_g).cpu().numpy()
    np.testing.assert_array_equal(cmax, oracle.scale_search_max(wu, sg))

    cmse, omse = nv.scale_search_mse(W, s_g, return_objective=True)
    rc, ro = oracle.scale_search_mse(wu, sg)
    n_tie_mse = check_search_codes(cmse.cpu().numpy(), rc, wu, sg)
    np.testing.assert_allclose(omse.cpu().numpy(), ro, rtol=1e-4, atol=1e-30)

    clh, olh = nv.scale_search_local_hessian(W, s_g, H, return_objective=True)
    rc, ro = oracle.scale_search_lh(wu, sg, H64)
    n_tie_lh = check_search_codes(clh.cpu().numpy(), rc, wu, sg, H64)
    np.testing.assert_allclose(olh.cpu().numpy(), ro, rtol=1e-4, atol=1e-30)
    assert n_tie_mse + n_tie_lh < 10


def test_four_over_six_bitexact(nv):
    """Four Over Six on every block of the tiny layer, a batch of experts
    with their own tensor scales, a ragged shape with zero, saturating,
    on-grid and tiny blocks: equal to the oracle block by block."""
    W, _ = _layer("tiny")
    s_g = nv.global_scale(W)
    c = nv.scale_search_four_over_six(W, s_g).cpu().numpy()
    np.testing.assert_array_equal(c, oracle.scale_search_four_over_six(bf16_bits(W), s_g.item()))
    Wb = rand_bf16((3, 40, 96), 17, 0.02, 0.02, 30.0)
    sb = nv.global_scale(Wb.cuda(), batch=3)
    cb = nv.scale_search_four_over_six(Wb.cuda(), sb).cpu().numpy()
    for e in range(3):
        np.testing.assert_array_equal(cb[e], oracle.scale_search_four_over_six(bf16_bits(Wb[e]), sb[e].item()))
    x = rand_bf16((37, 80), 23, 0.5)
    x[0, :16] = 0
    x[1, 16:32] = x.abs().max()                     # saturating candidate(s)
    x[2, 32:48] = 1e-6 * x[2, 32:48]                # tiny block (codes near 0)
    grid = torch.tensor([48, 36, 24, 18, 12, 6, 0, -6, -12, -18, -24, -36, 6, 12, 24, 36.0])
    x[3, :16] = (grid / 1024).to(torch.bfloat16)    # on the grid of the amax/4 scale
    s = nv.global_scale(x.cuda())
    cx = nv.scale_search_four_over_six(x.cuda(), s).cpu().numpy()
    rx = oracle.scale_search_four_over_six(bf16_bits(x), s.item())
    np.testing.assert_array_equal(cx, rx)
    assert cx[0, 0] == 0


def test_identity_hessian_gives_mse_on_gpu(nv):
    W, _ = _layer("tiny")
    s_g = nv.global_scale(W)
    nb = W.shape[1] // 16
    H = torch.eye(16, device="cuda").repeat(nb, 1, 1) * 2.5
    clh = nv.scale_search_local_hessian(W, s_g, H)
    cmse = nv.scale_search_mse(W, s_g)
    wu = bf16_bits(W)
    rc, _ = oracle.scale_search_mse(wu, s_g.item())
    check_search_codes(clh.cpu().numpy(), rc, wu, s_g.item())
    check_search_codes(cmse.cpu().numpy(), rc, wu, s_g.item())


def test_search_degenerate_blocks(nv):
    """Zero blocks, a zero Hessian block, a rank-deficient Hessian (dead
    channels) and blocks already on the NVFP4 grid (exact-zero ties)."""
    x = rand_bf16((48, 64), 5, 0.02)
    x[0, :16] = 0
    s_g = nv.global_scale(x.cuda())
    codes = nv.scale_search_max(x.cuda(), s_g)
    packed = nv.quantize_pack(x.cuda(), s_g, codes)
    y = nv.dequantize(packed, codes, s_g)
    y[10:20] = x[10:20].cuda()      # half the rows back off the grid
    W = y.contiguous()
    wu = bf16_bits(W)
    sg = s_g.item()
    X = rand_bf16((200, 64), 6)
    X[:, 20:23] = 0                 # dead channels in block 1
    H = torch.zeros(4, 16, 16, device="cuda")
    nv.hessian_accumulate(X.cuda(), H)
    H[3] = 0                        # no calibration signal at all for block 3
    H64 = H.cpu().numpy().astype(np.float64)
    clh = nv.scale_search_local_hessian(W, s_g, H).cpu().numpy()
    rc, _ = oracle.scale_search_lh(wu, sg, H64)
    check_search_codes(clh, rc, wu, sg, H64)
    assert np.all(clh[:, 3] == 1)   # every candidate ties at zero: smallest code
    cm = nv.scale_search_mse(W, s_g).cpu().numpy()
    rc, _ = oracle.scale_search_mse(wu, sg)
    check_search_codes(cm, rc, wu, sg)
    assert cm[0, 0] == 1


def test_signed_zero_weights_every_rule(nv):
    """Weights full of signed zeros (a dequantised or pruned layer holds -0
    wherever a negative value rounded to zero): a quarter of the entries -0,
    some +0, rows that are all -0 or -0 but for one value, under a Gram with
    an outlier channel and dead channels.  Every block's max, Four Over Six,
    MSE and Local-Hessian code against the oracle, and every packed byte and
    dequantised value.  A -0 meets a class reciprocal whose low part is
    negative on many candidates: its class quotient is +0 and the residual
    -0, which must leave the quotient at zero."""
    rng = np.random.default_rng(31)
    R, C = 512, 256
    u = f32_to_bf16_bits((rng.standard_normal((R, C)) * 0.02).astype(np.float32))
    pick = rng.random((R, C))
    u = np.where(pick < 0.25, np.uint16(0x8000), u)
    u = np.where((pick >= 0.25) & (pick < 0.30), np.uint16(0), u)
    u[3] = 0x8000
    u[4] = 0x8000
    u[4, 77] = f32_to_bf16_bits(np.array([-0.03], np.float32))[0]
    u[5, 16:32] = 0x8000
    u = np.ascontiguousarray(u.astype(np.uint16))
    W = dev_bf16(u)
    s_g = nv.global_scale(W)
    sg = s_g.item()
    assert sg == oracle.global_scale(u)
    X = rand_bf16((300, C), 32)
    X[:, 40] *= 30.0
    X[:, 16:19] = 0                 # dead channels in block 1
    H = torch.zeros(C // 16, 16, 16, device="cuda")
    nv.hessian_accumulate(X.cuda(), H)
    H64 = H.cpu().numpy().astype(np.float64)
    np.testing.assert_array_equal(nv.scale_search_max(W, s_g).cpu().numpy(),
                                  oracle.scale_search_max(u, sg))
    np.testing.assert_array_equal(nv.scale_search_four_over_six(W, s_g).cpu().numpy(),
                                  oracle.scale_search_four_over_six(u, sg))
    cm = nv.scale_search_mse(W, s_g).cpu().numpy()
    rc, _ = oracle.scale_search_mse(u, sg)
    check_search_codes(cm, rc, u, sg)
    clh_dev = nv.scale_search_local_hessian(W, s_g, H)
    clh = clh_dev.cpu().numpy()
    rc, _ = oracle.scale_search_lh(u, sg, H64)
    check_search_codes(clh, rc, u, sg, H64)
    assert np.all(clh[3] == 1) and np.all(cm[3] == 1)   # all-zero rows: the smallest code
    packed = nv.quantize_pack(W, s_g, clh_dev)
    rp = oracle.quantize_pack(u, sg, clh)
    np.testing.assert_array_equal(packed.cpu().numpy(), rp)
    y = nv.dequantize(packed, clh_dev, s_g)
    np.testing.assert_array_equal(bf16_bits(y), oracle.dequantize(rp, clh, sg))


def test_search_ragged_rows_mixed_magnitudes(nv):
    """Every block of a ragged 600-row weight (three row groups, the last one
    partly padding) whose rows differ in magnitude by up to 10^5, with zero
    rows, single-spike rows and an outlier calibration channel: rows of very
    different size share tiles, and the candidate walk must still return the
    oracle's choice for each."""
    R, C = 600, 96
    g = torch.Generator().manual_seed(11)
    W = torch.randn(R, C, generator=g) * 0.02
    scale = torch.tensor([1e-3, 0.1, 1.0, 10.0, 100.0])[torch.randint(0, 5, (R,), generator=g)]
    W = W * scale[:, None]
    W[7] = 0
    W[300:310] = 0
    W[311, :] = 0
    W[311, 5] = 0.75
    W[599, 40] = -3.0
    W = W.to(torch.bfloat16)
    X = torch.randn(300, C, generator=g)
    X[:, 17] *= 30.0
    X = X.to(torch.bfloat16)
    wu = bf16_bits(W)
    s_g = nv.global_scale(W.cuda())
    sg = s_g.item()
    H = torch.zeros(C // 16, 16, 16, device="cuda")
    nv.hessian_accumulate(X.cuda(), H)
    H64 = H.cpu().numpy().astype(np.float64)
    clh = nv.scale_search_local_hessian(W.cuda(), s_g, H).cpu().numpy()
    rc, _ = oracle.scale_search_lh(wu, sg, H64)
    check_search_codes(clh, rc, wu, sg, H64)
    cm = nv.scale_search_mse(W.cuda(), s_g).cpu().numpy()
    rc, _ = oracle.scale_search_mse(wu, sg)
    check_search_codes(cm, rc, wu, sg)
    assert np.all(cm[7] == 1) and np.all(clh[300:310] == 1)


@pytest.mark.parametrize("R,C", [(1, 16), (3, 32), (17, 48), (1, 48), (17, 16), (3, 16)])
def test_search_rules_on_tiny_shapes(nv, R, C):
    """Every scale rule on the smallest shapes (one to seventeen rows, one to
    three column blocks): almost every row of a CTA is padding."""
    W = rand_bf16((R, C), R * 100 + C, 0.02, 0.1, 20.0)
    X = rand_bf16((50, C), R + C, 1.0)
    wu = bf16_bits(W)
    s_g = nv.global_scale(W.cuda())
    sg = s_g.item()
    assert sg == oracle.global_scale(wu)
    H = torch.zeros(C // 16, 16, 16, device="cuda")
    nv.hessian_accumulate(X.cuda(), H)
    H64 = H.cpu().numpy().astype(np.float64)
    clh = nv.scale_search_local_hessian(W.cuda(), s_g, H).cpu().numpy()
    check_search_codes(clh, oracle.scale_search_lh(wu, sg, H64)[0], wu, sg, H64)
    cm = nv.scale_search_mse(W.cuda(), s_g).cpu().numpy()
    check_search_codes(cm, oracle.scale_search_mse(wu, sg)[0], wu, sg)
    np.testing.assert_array_equal(nv.scale_search_max(W.cuda(), s_g).cpu().numpy(),
                                  oracle.scale_search_max(wu, sg))
    np.testing.assert_array_equal(nv.scale_search_four_over_six(W.cuda(), s_g).cpu().numpy(),
                                  oracle.scale_search_four_over_six(wu, sg))


def test_search_evaluation_counters(nv):
    """The work statistic: between 1 and 126 evaluations per block searched,
    counted per rule, and zeroed by a reset."""
    W, X = _layer("tiny")
    s_g = nv.global_scale(W)
    H = torch.zeros(W.shape[1] // 16, 16, 16, device="cuda")
    nv.hessian_accumulate(X, H)
    nv.search_evaluations(reset=True)
    assert nv.search_evaluations() == (0, 0)
    blocks = W.numel() // 16
    nv.scale_search_mse(W, s_g)
    m, l = nv.search_evaluations()
    assert blocks <= m <= 126 * blocks and l == 0
    nv.scale_search_local_hessian(W, s_g, H)
    nv.scale_search_local_hessian(W, s_g, H)
    r = nv.search_rescores()
    m2, l2 = nv.search_evaluations(reset=True)
    assert m2 == m and 2 * blocks <= l2 <= 2 * 126 * blocks and l2 % 2 == 0
    assert nv.search_evaluations() == (0, 0) and nv.search_rescores() == (0, 0, 0, 0)
    # re-scored rows: at most every block once per call; the tiny layer has
    # near ties under both rules
    assert 0 < r[0] + r[1] <= blocks and 0 < r[2] + r[3] <= 2 * blocks and r[2] % 2 == 0


def test_four_over_six_dense_layer_every_block(nv):
    """Dense 4096x4096 workload, every block (the oracle's two-candidate
    rule is cheap enough for the full layer)."""
    W, _ = _layer("dense")
    s_g = nv.global_scale(W)
    c = nv.scale_search_four_over_six(W, s_g).cpu().numpy()
    np.testing.assert_array_equal(c, oracle.scale_search_four_over_six(bf16_bits(W), s_g.item()))


# ------------------------------------------------------------ NVFP4 GEMM
def _gemm_operands(nv, X, W):
    """Activations through the dynamic fake-quant (packed outputs), weights
    through the global scale, the max rule and pack."""
    _, ap, ac, asg = nv.fake_quant(X, want_packed=True)
    wsg = nv.global_scale(W)
    wc = nv.scale_search_max(W, wsg)
    wp = nv.quantize_pack(W, wsg, wc)
    return ap, ac, asg, wp, wc, wsg


def _check_gemm(Y, ref, absref, K):
    y = bits_to_f64(bf16_bits(Y))
    # bf16 rounding of the result plus fp32 accumulation over K terms
    tol = 2.0 ** -8 * np.abs(ref) + K * 2.0 ** -23 * absref + 1e-35
    bad = np.argwhere(np.abs(y - ref) > tol)
    assert bad.size == 0, (bad[:5], y[tuple(bad[0])], ref[tuple(bad[0])])


@pytest.mark.parametrize("M,N,K", [(200, 136, 256), (128, 256, 96), (1, 8, 32), (333, 520, 1024)])
def test_gemm_matches_oracle(nv, M, N, K):
    X = rand_bf16((M, K), M + K, 1.0, 0.01, 30.0).cuda()
    W = rand_bf16((N, K), N + K, 0.02, 0.005, 15.0).cuda()
    ap, ac, asg, wp, wc, wsg = _gemm_operands(nv, X, W)
    Y = nv.gemm(ap, ac, asg, wp, wc, wsg)
    ref, absref = oracle.gemm_nvfp4(ap.cpu().numpy(), ac.cpu().numpy(), asg.item(),
                                    wp.cpu().numpy(), wc.cpu().numpy(), wsg.item())
    _check_gemm(Y, ref, absref, K)


def test_gemm_w4a4_full_size_sampled(nv):
    """The W4A4 activations (32768x8192, dynamic fake-quant with packed
    outputs) times an 8192x8192 NVFP4 weight, in one call; 48 rows x 48
    columns of the result against the oracle."""
    from scale_calibration_nvfp4_b200 import workloads
    X = workloads.w4a4_inputs("cuda")
    g = torch.Generator(device="cuda").manual_seed(9)
    W = (torch.randn(8192, 8192, generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    ap, ac, asg, wp, wc, wsg = _gemm_operands(nv, X, W)
    Y = nv.gemm(ap, ac, asg, wp, wc, wsg)
    rng = np.random.default_rng(4)
    rows = np.sort(rng.choice(X.shape[0], 48, replace=False)); rows[-1] = X.shape[0] - 1
    cols = np.sort(rng.choice(W.shape[0], 48, replace=False)); cols[0] = 0
    r_t, c_t = torch.from_numpy(rows).cuda(), torch.from_numpy(cols).cuda()
    ref, absref = oracle.gemm_nvfp4(ap[r_t].cpu().numpy(), ac[r_t].cpu().numpy(), asg.item(),
                                    wp[c_t].cpu().numpy(), wc[c_t].cpu().numpy(), wsg.item())
    _check_gemm(Y[r_t][:, c_t].contiguous(), ref, absref, X.shape[1])


# ------------------------------------------------ activation-range calibration
def test_abs_histogram_and_static_scales(nv):
    x = rand_bf16((301, 96), 41, 1.0, 0.003, 60.0)
    xu = bf16_bits(x)
    flat = x.reshape(-1)
    h = nv.abs_histogram(flat[:10001].contiguous().cuda())       # ragged length
    h = nv.abs_histogram(flat[10001:].contiguous().cuda(), h)    # accumulates
    ref = oracle.abs_histogram(xu)
    assert np.array_equal(h.cpu().numpy().astype(np.uint64), ref)
    for p in (1.0, 0.99999, 0.9999, 0.999, 0.5):
        s = nv.static_scale_from_histogram(h, p).item()
        assert s == oracle.static_scale(oracle.quantile_magnitude(ref, p)), p


def test_fake_quant_static_and_error(nv):
    x = rand_bf16((333, 96), 43, 1.0, 0.003, 60.0)
    xu = bf16_bits(x)
    sg_max = oracle.global_scale(xu)
    for s in (sg_max, np.float32(sg_max / 16), np.float32(sg_max * 3)):
        s_t = torch.tensor([s], dtype=torch.float32, device="cuda")
        y, p, c = nv.fake_quant_static(x.cuda(), s_t, want_packed=True)
        ry, rp, rc = oracle.fake_quant_static(xu, s)
        assert np.array_equal(bf16_bits(y), ry) and np.array_equal(p.cpu().numpy(), rp) \
            and np.array_equal(c.cpu().numpy(), rc)
        e = nv.quant_error(x.cuda(), s_t).item()
        assert math.isclose(e, oracle.quant_error(xu, s), rel_tol=1e-10)
    assert nv.get_device_status() == "NVFP4_OK"


def test_static_scale_on_nonfinite_reports(nv):
    x = torch.ones(64, dtype=torch.bfloat16)
    x[5] = float("inf")
    h = nv.abs_histogram(x.cuda())
    assert math.isnan(nv.static_scale_from_histogram(h, 1.0).item())
    assert nv.get_device_status() == "NVFP4_ERR_NONFINITE"
    assert nv.static_scale_from_histogram(h, 0.5).item() == oracle.static_scale(1.0)
    assert nv.get_device_status() == "NVFP4_OK"


def test_calibration_w4a4_full_size(nv):
    """The W4A4 activations (268 M values): histogram bit-exact, the
    99.99th-percentile static scale bit-exact, the error at it and at the
    maximum within 1e-9 of the oracle."""
    from scale_calibration_nvfp4_b200 import workloads
    X = workloads.w4a4_inputs("cuda")
    xu = bf16_bits(X)
    h = nv.abs_histogram(X)
    ref = oracle.abs_histogram(xu)
    assert np.array_equal(h.cpu().numpy().astype(np.uint64), ref)
    s_p = nv.static_scale_from_histogram(h, 0.9999)
    assert s_p.item() == oracle.static_scale(oracle.quantile_magnitude(ref, 0.9999))
    s_max = nv.static_scale_from_histogram(h, 1.0)
    assert s_max.item() == oracle.global_scale(xu)
    e_p, e_max = nv.quant_error(X, s_p).item(), nv.quant_error(X, s_max).item()
    assert math.isclose(e_p, oracle.quant_error(xu, s_p.item()), rel_tol=1e-9)
    assert math.isclose(e_max, oracle.quant_error(xu, s_max.item()), rel_tol=1e-9)


# ------------------------------------------- tiny and huge tensor scales
@pytest.mark.parametrize("e", [-56, -62, -66, -70, -95, -128, 70, 100, 115])
def test_extreme_tensor_scales_every_rule(nv, e):
    """Weights scaled by 2^e (tensor scale near 2^(e-9)).  Tiny: Four Over
    Six's fp32 block MSEs are subnormal, where the screen's absolute margin
    hands the close calls to the exact fp64 path, and unscaled search
    objectives and bounds would underflow or overflow.  Huge: unscaled MSE
    objectives would overflow fp32.  Beyond [2^-100, 2^100) (e = -95, -128,
    115) the searches re-score every candidate in fp64 and the encodes take
    the exact fp64 path; at e = -128 s_g is a subnormal fp32 and the max
    rule's reciprocal is pre-scaled.  Every rule, pack, dequant and
    fake-quant equal the oracle."""
    W = (rand_bf16((70, 128), 60 - e, 1.0).float() * 2.0 ** e).to(torch.bfloat16)
    X = rand_bf16((200, 128), 41, 1.0, 0.01, 20.0)
    wu = bf16_bits(W)
    Wd = W.cuda()
    s_g = nv.global_scale(Wd)
    sg = s_g.item()
    assert sg == oracle.global_scale(wu)
    assert (2.0 ** -100 <= sg < 2.0 ** 100) == (-90 < e < 110)
    cmax = oracle.scale_search_max(wu, sg)
    np.testing.assert_array_equal(nv.scale_search_max(Wd, s_g).cpu().numpy(), cmax)
    np.testing.assert_array_equal(nv.scale_search_four_over_six(Wd, s_g).cpu().numpy(),
                                  oracle.scale_search_four_over_six(wu, sg))
    rc, _ = oracle.scale_search_mse(wu, sg)
    n_tie = check_search_codes(nv.scale_search_mse(Wd, s_g).cpu().numpy(), rc, wu, sg)
    H = torch.zeros(W.shape[1] // 16, 16, 16, device="cuda")
    nv.hessian_accumulate(X.cuda(), H)
    H64 = H.cpu().numpy().astype(np.float64)
    rc, _ = oracle.scale_search_lh(wu, sg, H64)
    n_tie += check_search_codes(nv.scale_search_local_hessian(Wd, s_g, H).cpu().numpy(), rc,
                                wu, sg, H64)
    assert n_tie < 10
    packed = nv.quantize_pack(Wd, s_g, torch.from_numpy(cmax).cuda())
    ref_p = oracle.quantize_pack(wu, sg, cmax)
    np.testing.assert_array_equal(packed.cpu().numpy(), ref_p)
    y = nv.dequantize(packed, torch.from_numpy(cmax).cuda(), s_g)
    np.testing.assert_array_equal(bf16_bits(y), oracle.dequantize(ref_p, cmax, sg))
    yf, pf, cf, sf = nv.fake_quant(Wd, want_packed=True)
    ry, rp, rcf, rs = oracle.fake_quant(wu)
    assert sf.item() == rs
    np.testing.assert_array_equal(cf.cpu().numpy(), rcf)
    np.testing.assert_array_equal(pf.cpu().numpy(), rp)
    np.testing.assert_array_equal(bf16_bits(yf), ry)
    assert nv.get_device_status() == "NVFP4_OK"


def test_searches_with_a_tensor_scale_far_below_the_weights(nv):
    """A caller-supplied tensor scale far below amax / 2688 (2^-99 for
    weights up to 2^61): rows of ordinary size take the screen's class path,
    rows whose values pass 2^100 s_g (their class quotients would overflow
    fp32) send their tiles to the exact fp64 re-score.  Every block of both
    searches against the oracle."""
    g = torch.Generator().manual_seed(31)
    R, C = 300, 64
    W = torch.randn(R, C, generator=g) * 0.1         # below 2^100 s_g = 2: class path
    big = torch.randperm(R, generator=g)[:70]
    W[big] *= 2.0 ** 63
    W = W.to(torch.bfloat16)
    X = torch.randn(200, C, generator=g).to(torch.bfloat16)
    wu = bf16_bits(W)
    sg = 2.0 ** -99
    s_g = torch.tensor([sg], dtype=torch.float32).cuda()
    H = torch.zeros(C // 16, 16, 16, device="cuda")
    nv.hessian_accumulate(X.cuda(), H)
    H64 = H.cpu().numpy().astype(np.float64)
    clh = nv.scale_search_local_hessian(W.cuda(), s_g, H).cpu().numpy()
    check_search_codes(clh, oracle.scale_search_lh(wu, sg, H64)[0], wu, sg, H64)
    cm = nv.scale_search_mse(W.cuda(), s_g).cpu().numpy()
    check_search_codes(cm, oracle.scale_search_mse(wu, sg)[0], wu, sg)


def test_rows_far_below_their_tile_every_search(nv):
    """Rows scaled by 2^-10, 2^-14, 2^-16 (codes down in E4M3's subnormal
    range) and 2^-40 (every candidate ties at zero) among ordinary rows:
    sorted by magnitude they share the first 16-row tile with ordinary rows,
    and each row's own power-of-two scale keeps its f16 operand and fp32
    objectives at full precision.  MSE and Local-Hessian codes equal the
    oracle."""
    W = rand_bf16((70, 128), 77, 0.02).float()
    for r, e in ((5, -10), (17, -14), (33, -16), (41, -16), (50, -40)):
        W[r] *= 2.0 ** e
    W = W.to(torch.bfloat16)
    X = rand_bf16((300, 128), 78, 1.0, 0.01, 20.0)
    wu = bf16_bits(W)
    Wd = W.cuda()
    s_g = nv.global_scale(Wd)
    sg = s_g.item()
    rc, _ = oracle.scale_search_mse(wu, sg)
    n_tie = check_search_codes(nv.scale_search_mse(Wd, s_g).cpu().numpy(), rc, wu, sg)
    H = torch.zeros(W.shape[1] // 16, 16, 16, device="cuda")
    nv.hessian_accumulate(X.cuda(), H)
    H64 = H.cpu().numpy().astype(np.float64)
    rc, _ = oracle.scale_search_lh(wu, sg, H64)
    n_tie += check_search_codes(nv.scale_search_local_hessian(Wd, s_g, H).cpu().numpy(), rc,
                                wu, sg, H64)
    assert n_tie < 10
    assert nv.get_device_status() == "NVFP4_OK"


@pytest.mark.parametrize("e", [-40, 37])
def test_every_rule_is_invariant_under_powers_of_two_on_gpu(nv, e):
    """W and W 2^e through every rule on the device: s_g scales by 2^e, each
    row's f16 operand, class quotients and certificates are unchanged, and
    every fp32 / fp64 value of the screens scales exactly, so the codes are
    identical bit for bit (near-ties included; no tolerance) and the
    objectives scale by exactly 2^(2e)."""
    W = rand_bf16((130, 256), 91, 0.02, 0.01, 30.0)
    Ws = (W.float() * 2.0 ** e).to(torch.bfloat16)
    assert torch.equal(Ws.float(), W.float() * 2.0 ** e)
    X = rand_bf16((300, 256), 92, 1.0, 0.01, 20.0)
    H = torch.zeros(W.shape[1] // 16, 16, 16, device="cuda")
    nv.hessian_accumulate(X.cuda(), H)
    Hf = torch.zeros(256, 256, device="cuda")
    nv.hessian_full_accumulate(X.cuda(), Hf)
    out = []
    for w in (W.cuda(), Ws.cuda()):
        s_g = nv.global_scale(w)
        cm, om = nv.scale_search_mse(w, s_g, return_objective=True)
        cl, ol = nv.scale_search_local_hessian(w, s_g, H, return_objective=True)
        cmax = nv.scale_search_max(w, s_g)
        out.append(dict(s_g=s_g.item(), cmax=cmax, cm=cm, om=om, cl=cl, ol=ol,
                        c46=nv.scale_search_four_over_six(w, s_g),
                        packed=nv.quantize_pack(w, s_g, cl),
                        gptq=nv.gptq(w, s_g, cl, Hf, 0.01)))
    a, b = out
    assert b["s_g"] == a["s_g"] * 2.0 ** e
    for k in ("cmax", "cm", "cl", "c46", "packed", "gptq"):
        assert torch.equal(a[k], b[k]), k
    for k in ("om", "ol"):
        ref = a[k].double() * 4.0 ** e
        ok = (a[k] > 2.0 ** -100) & (a[k] < 2.0 ** 100) & (ref.abs() > 2.0 ** -120)
        ok &= ref.abs() < 2.0 ** 120
        assert torch.equal(b[k].double()[ok], ref[ok]), k
    assert nv.get_device_status() == "NVFP4_OK"
