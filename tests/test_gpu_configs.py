"""Every-block GPU parity on the five calibration workloads, at their full
sizes and in the launch configuration the benchmark times.

For each workload every 16x16 Gram block is compared with the oracle's fp64
Gram of the same tokens (relative Frobenius error <= 1e-4, per block and
overall), every block's scale code with the oracle's exhaustive search (fed
the GPU's own fp32 H, so the check isolates the search), every packed byte
and every dequantised / fake-quantised value bit for bit.  The number of
blocks whose oracle objectives have their best two within 1e-6 relative
(near ties, where another code is allowed) and the number of codes that
differ there are printed after the run.

Sources: the block-diagonal objective and the 126-candidate search of the
Local-Hessian write-up ("4 比特量化到底让模型笨了多少？", sections "The NVFP4
structure" and "A different objective"), its calibration recipe ("Trying
it": 512 sequences of 2048 tokens, the MLP pair's 16 chunks of 65,536), the
format of "What makes high-quality NVFP4" and the fake-quant forward of
"為什么NVFP4推理精度會掉以及QAD到底在修什么" (section 3.2)."""
import numpy as np
import pytest
import torch

import oracle
from conftest import bf16_bits, record_stat
from parity_util import GRAM_REL, TIE_REL, check_search_codes, rel_frobenius

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


def check_gram_every_block(H_gpu, H_ref):
    """Relative Frobenius error of every 16x16 block and of the whole; returns
    the worst block error."""
    a = np.asarray(H_gpu, np.float64).reshape(-1, 256)
    r = np.asarray(H_ref, np.float64).reshape(-1, 256)
    num = np.linalg.norm(a - r, axis=1)
    den = np.linalg.norm(r, axis=1)
    assert np.all(den > 0)
    worst = float(np.max(num / den))
    assert worst <= GRAM_REL, worst
    assert rel_frobenius(a, r) <= GRAM_REL
    return worst


def near_ties(best, second):
    """Blocks whose best two oracle objectives lie within the tie band."""
    best = np.asarray(best)
    second = np.asarray(second)
    return int(np.count_nonzero(second - best <= TIE_REL * second))


def search_every_block(codes_gpu, w_u16, s_g, H64=None):
    """The oracle's exhaustive search on every block (MSE when H64 is None),
    compared with the GPU's codes; returns (near ties, differing codes)."""
    if H64 is None:
        rc, best, second = oracle.scale_search_mse(w_u16, s_g, runner_up=True)
    else:
        rc, best, second = oracle.scale_search_lh(w_u16, s_g, H64, runner_up=True)
    n_diff = check_search_codes(codes_gpu, rc, w_u16, s_g, H64)
    return near_ties(best, second), n_diff


def pack_dequant_every_element(nv, W, s_g, codes_dev, wu, sg, codes):
    packed = nv.quantize_pack(W, s_g, codes_dev)
    y = nv.dequantize(packed, codes_dev, s_g)
    rp = oracle.quantize_pack(wu, sg, codes)
    np.testing.assert_array_equal(packed.cpu().numpy(), rp)
    np.testing.assert_array_equal(bf16_bits(y), oracle.dequantize(rp, codes, sg))


def single_layer(nv, name, rules):
    from scale_calibration_nvfp4_b200 import workloads
    W, X = workloads.layer_inputs(name, "cuda")
    wu, xu = bf16_bits(W), bf16_bits(X)
    s_g = nv.global_scale(W)
    sg = s_g.item()
    assert sg == oracle.global_scale(wu)
    H = torch.zeros(W.shape[1] // 16, 16, 16, device="cuda")
    nv.hessian_accumulate(X, H)
    H64 = H.cpu().numpy().astype(np.float64)
    stats = {"gram_worst_block_rel": "%.2e" % check_gram_every_block(H64, oracle.gram(xu)),
             "blocks": W.numel() // 16}
    if "max" in rules:
        np.testing.assert_array_equal(nv.scale_search_max(W, s_g).cpu().numpy(),
                                      oracle.scale_search_max(wu, sg))
    if "mse" in rules:
        c = nv.scale_search_mse(W, s_g).cpu().numpy()
        stats["mse_near_ties"], stats["mse_codes_differing"] = search_every_block(c, wu, sg)
    clh = nv.scale_search_local_hessian(W, s_g, H)
    c = clh.cpu().numpy()
    stats["lh_near_ties"], stats["lh_codes_differing"] = search_every_block(c, wu, sg, H64)
    pack_dequant_every_element(nv, W, s_g, clh, wu, sg, c)
    # the W4A4 fake-quant of the calibration activations, every element
    fy, fp, fc, fs = nv.fake_quant(X, want_packed=True)
    ry, rp, rc, rs = oracle.fake_quant(xu)
    assert fs.item() == rs
    np.testing.assert_array_equal(bf16_bits(fy), ry)
    np.testing.assert_array_equal(fp.cpu().numpy(), rp)
    np.testing.assert_array_equal(fc.cpu().numpy(), rc)
    return stats


def test_tiny_layer_every_block(nv):
    """Tiny layer (W 256x512, X 512x512, seed 0): Gram, max, MSE and
    Local-Hessian codes, pack, dequantise and fake-quant, every block."""
    record_stat("tiny 256x512", **single_layer(nv, "tiny", ("max", "mse")))


def test_dense_layer_every_block(nv):
    """Dense projection (W 4096x4096, X 2048x4096, seed 1): every one of its
    1,048,576 blocks under the max, MSE and Local-Hessian rules; every packed
    byte and dequantised value; the fake-quant of X element by element."""
    record_stat("dense 4096x4096", **single_layer(nv, "dense", ("max", "mse")))


def test_mlp_pair_every_block(nv):
    """MLP pair (up 12288x4096, down 4096x12288, Student-t(4) calibration
    tokens streamed in 16 chunks of 65,536): the Gram accumulated chunk by
    chunk on both sides, then every block's Local-Hessian code, packed byte
    and dequantised value."""
    from scale_calibration_nvfp4_b200 import workloads
    up, down = workloads.mlp_weights("cuda")
    chunks = workloads.BY_NAME["mlp_pair"].params["chunks"]
    for which, W in (("up", up), ("down", down)):
        C = W.shape[1]
        H = torch.zeros(C // 16, 16, 16, device="cuda")
        H_ref = np.zeros((C // 16, 16, 16), np.float64)
        for k in range(chunks):
            ch = workloads.mlp_chunk(which, k, "cuda")
            nv.hessian_accumulate(ch, H)
            H_ref = oracle.gram(bf16_bits(ch), H_ref)
            del ch
        H64 = H.cpu().numpy().astype(np.float64)
        worst = check_gram_every_block(H64, H_ref)
        wu = bf16_bits(W)
        s_g = nv.global_scale(W)
        sg = s_g.item()
        assert sg == oracle.global_scale(wu)
        clh = nv.scale_search_local_hessian(W, s_g, H)
        c = clh.cpu().numpy()
        ties, diff = search_every_block(c, wu, sg, H64)
        pack_dequant_every_element(nv, W, s_g, clh, wu, sg, c)
        record_stat("mlp_pair %s %dx%d" % (which, W.shape[0], C), blocks=W.numel() // 16,
                    gram_worst_block_rel="%.2e" % worst, lh_near_ties=ties,
                    lh_codes_differing=diff)


def test_moe_experts_every_block(nv):
    """MoE experts (128 x 768x2048, 262,144 routed tokens sorted by expert):
    the grouped Gram of every expert, per-expert tensor scales, and every
    block's Local-Hessian code, packed byte and dequantised value."""
    from scale_calibration_nvfp4_b200 import workloads
    W, X, offsets = workloads.moe_inputs("cuda")
    G, R, C = W.shape
    nb = C // 16
    s_g = nv.global_scale(W, batch=G)
    H = torch.zeros(G, nb, 16, 16, device="cuda")
    nv.hessian_accumulate_grouped(X, offsets.cuda(), H)
    clh = nv.scale_search_local_hessian(W, s_g, H)
    packed = nv.quantize_pack(W, s_g, clh)
    y = nv.dequantize(packed, clh, s_g)
    Hc = H.cpu().numpy().astype(np.float64)
    worst = check_gram_every_block(Hc, oracle.gram_grouped(bf16_bits(X), offsets.numpy(), G))
    wu_all, codes, pk, yu = bf16_bits(W), clh.cpu().numpy(), packed.cpu().numpy(), bf16_bits(y)
    sgs = s_g.cpu().numpy()
    ties = diff = 0
    for e in range(G):
        sg = float(sgs[e])
        assert sg == oracle.global_scale(wu_all[e]), e
        t, d = search_every_block(codes[e], wu_all[e], sg, Hc[e])
        ties += t
        diff += d
        rp = oracle.quantize_pack(wu_all[e], sg, codes[e])
        np.testing.assert_array_equal(pk[e], rp)
        np.testing.assert_array_equal(yu[e], oracle.dequantize(rp, codes[e], sg))
    record_stat("moe 128x768x2048", blocks=W.numel() // 16, gram_worst_block_rel="%.2e" % worst,
                lh_near_ties=ties, lh_codes_differing=diff)


def test_w4a4_fake_quant_every_element(nv):
    """Dynamic W4A4 fake-quant of X 32768x8192 (seed 4): the tensor scale,
    every block code, every packed byte and every output value."""
    from scale_calibration_nvfp4_b200 import workloads
    X = workloads.w4a4_inputs("cuda")
    fy, fp, fc, fs = nv.fake_quant(X, want_packed=True)
    ry, rp, rc, rs = oracle.fake_quant(bf16_bits(X))
    assert fs.item() == rs
    np.testing.assert_array_equal(fc.cpu().numpy(), rc)
    np.testing.assert_array_equal(fp.cpu().numpy(), rp)
    np.testing.assert_array_equal(bf16_bits(fy), ry)
    record_stat("w4a4 32768x8192", blocks=X.numel() // 16, elements_bit_exact=X.numel())


def test_four_over_six_moe_weights_every_block(nv):
    """Four Over Six on the MoE experts' weights (128 x 768x2048, per-expert
    tensor scales, the benchmark's Four Over Six workload): every block's
    code against the oracle, and the packed bytes of every expert."""
    from scale_calibration_nvfp4_b200 import workloads
    W, _, _ = workloads.moe_inputs("cuda")
    G = W.shape[0]
    s_g = nv.global_scale(W, batch=G)
    c = nv.scale_search_four_over_six(W, s_g)
    packed = nv.quantize_pack(W, s_g, c).cpu().numpy()
    c = c.cpu().numpy()
    wu, sgs = bf16_bits(W), s_g.cpu().numpy()
    for e in range(G):
        ref = oracle.scale_search_four_over_six(wu[e], float(sgs[e]))
        np.testing.assert_array_equal(c[e], ref, err_msg="expert %d" % e)
        np.testing.assert_array_equal(packed[e], oracle.quantize_pack(wu[e], float(sgs[e]), ref))
    record_stat("four_over_six moe 128x768x2048", blocks=W.numel() // 16, codes_differing=0)
