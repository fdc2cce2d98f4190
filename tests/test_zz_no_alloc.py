"""The Gram entry point that allocates nothing (nvfp4_hessian_accumulate_noalloc).

It serves callers that may not allocate device memory — applications that
hand all of HBM to their own allocator or run under a fixed memory budget, and
loops that cannot take an allocation's latency or implicit synchronisation.
Its partial sums live in a fixed device array inside the library, shared by
every call.  This file is collected last so that a run stopping at the first
failure has already run every other test; it also passes alone in a fresh
process (the first call does the one-time address lookup).
"""
import numpy as np
import pytest
import torch

import oracle
from conftest import bf16_bits
from parity_util import GRAM_REL, rel_frobenius

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from scale_calibration_nvfp4_b200 import build, nvfp4
    build.build()
    nvfp4.lib()
    return nvfp4


def _calib(n_tok, C, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(n_tok, C, generator=g)
    x[:, 5] *= 30.0
    return x.to(torch.bfloat16)


def test_noalloc_gram_matches_pool_entry_point_twice(nv):
    # two calls in a row through the shared array, different shapes: the
    # second must not see anything the first left behind
    for call, (n_tok, C) in enumerate([(3000, 1040), (517, 4096)]):
        x = _calib(n_tok, C, 100 + call)
        xd = x.cuda()
        H_ref = torch.zeros(C // 16, 16, 16, device="cuda")
        nv.hessian_accumulate(xd, H_ref)
        H_na = torch.zeros(C // 16, 16, 16, device="cuda")
        nv.hessian_accumulate_noalloc(xd, H_na)
        torch.cuda.synchronize()
        a, r = H_na.cpu().numpy(), H_ref.cpu().numpy()
        assert rel_frobenius(a, r) <= GRAM_REL, call
        for j in range(C // 16):
            assert rel_frobenius(a[j], r[j]) <= GRAM_REL, (call, j)
        # and against the fp64 oracle on a few column blocks
        xu = bf16_bits(x)
        for j in (0, C // 32, C // 16 - 1):
            ref = oracle.gram(np.ascontiguousarray(xu[:, 16 * j:16 * j + 16]))[0]
            assert rel_frobenius(a[j], ref) <= GRAM_REL, (call, j)


def test_noalloc_gram_accumulates_in_place(nv):
    x = _calib(2048, 512, 7).cuda()
    H = torch.zeros(32, 16, 16, device="cuda")
    nv.hessian_accumulate_noalloc(x[:1000], H)
    nv.hessian_accumulate_noalloc(x[1000:], H)
    H_ref = torch.zeros(32, 16, 16, device="cuda")
    nv.hessian_accumulate(x, H_ref)
    assert rel_frobenius(H.cpu().numpy(), H_ref.cpu().numpy()) <= GRAM_REL


def test_noalloc_gram_at_its_channel_limit(nv):
    # C = 262,144: one token range fills the whole array (every partial slot
    # in use, the reduce over a single item), twice in a row
    C = 262144
    for call, n_tok in enumerate((300, 77)):
        x = _calib(n_tok, C, 40 + call)
        xd = x.cuda()
        H_ref = torch.zeros(C // 16, 16, 16, device="cuda")
        nv.hessian_accumulate(xd, H_ref)
        H_na = torch.zeros(C // 16, 16, 16, device="cuda")
        nv.hessian_accumulate_noalloc(xd, H_na)
        torch.cuda.synchronize()
        a, r = H_na.cpu().numpy(), H_ref.cpu().numpy()
        assert rel_frobenius(a, r) <= GRAM_REL, call
        err = np.linalg.norm((a - r).reshape(C // 16, -1), axis=1)
        assert np.all(err <= GRAM_REL * np.linalg.norm(r.reshape(C // 16, -1), axis=1)), call
        xu = bf16_bits(x)
        for j in (0, 1, C // 32, C // 16 - 1):
            ref = oracle.gram(np.ascontiguousarray(xu[:, 16 * j:16 * j + 16]))[0]
            assert rel_frobenius(a[j], ref) <= GRAM_REL, (call, j)


def test_noalloc_gram_rejects_channels_beyond_its_array(nv):
    # checked on the host before anything is launched
    from scale_calibration_nvfp4_b200.nvfp4 import NVFP4Error
    C = 262144 + 16
    x = torch.empty(1, C, dtype=torch.bfloat16, device="cuda")
    H = torch.zeros(C // 16, 16, 16, device="cuda")
    with pytest.raises(NVFP4Error) as ei:
        nv.hessian_accumulate_noalloc(x, H)
    assert ei.value.status == 7  # NVFP4_ERR_TOO_LARGE
