"""Comparison rules shared by the GPU parity tests.

- Integer / byte results (E2M1 codes, packed bytes, max-rule codes, FP32
  tensor scale, dequantised bf16) must be bit-exact.
- A searched scale code must equal the oracle's, except in a near-tie: when
  the oracle's best two objectives lie within 1e-6 relative, the GPU's code
  must reach an oracle objective no worse than the best times (1 + 1e-6).
- The Gram matrix must be within 1e-4 relative Frobenius error of fp64.
"""
import numpy as np

import oracle

TIE_REL = 1e-6
GRAM_REL = 1e-4


def check_search_codes(gpu, ref, w_u16, s_g, H=None, rows=None, blocks=None):
    """gpu/ref: codes of the same blocks; w_u16 [R, C]; rows/blocks give the
    block coordinates when the codes are a sample (else full [R, C/16]).
    H: per-column-block Hessian [C/16, 16, 16] (fp64) or None for MSE.
    Returns the number of tolerated near-tie differences."""
    gpu = np.asarray(gpu).reshape(-1)
    ref = np.asarray(ref).reshape(-1)
    if rows is None:
        R, nb = w_u16.shape[0], w_u16.shape[1] // 16
        rr, bb = np.divmod(np.arange(R * nb), nb)
    else:
        rr, bb = np.asarray(rows), np.asarray(blocks)
    bad = np.nonzero(gpu != ref)[0]
    for i in bad:
        r, b = int(rr[i]), int(bb[i])
        E = oracle.block_objectives(w_u16[r, 16 * b:16 * b + 16], s_g,
                                    None if H is None else H[b])
        order = np.sort(E)
        e1, e2 = order[0], order[1]
        assert e2 - e1 <= TIE_REL * e2, (
            "block (%d,%d): gpu code %d, oracle %d, oracle objectives %.17g / %.17g (no tie)"
            % (r, b, gpu[i], ref[i], E[gpu[i] - 1], e1))
        assert E[gpu[i] - 1] <= e1 * (1 + TIE_REL), (
            "block (%d,%d): gpu code %d objective %.17g vs best %.17g"
            % (r, b, gpu[i], E[gpu[i] - 1], e1))
    return len(bad)


def rel_frobenius(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / den) if den > 0 else float(np.linalg.norm(a))
