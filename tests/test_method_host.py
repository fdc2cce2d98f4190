"""Host checks of the algebra the GPU path is built on (not of the kernels):
each restates, in numpy, a reformulation the CUDA code uses and compares it
with the oracle, which follows the published form."""
import numpy as np
import pytest
import torch

from conftest import bf16_bits, bits_to_f64

MIDS = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _round(x, s):
    a = np.abs(x)
    k = 0 if not s > 0 else int(sum(int(a > m * s) if i % 2 == 0 else int(a >= m * s)
                                    for i, m in enumerate(MIDS)))
    return np.copysign(GRID[k] * s, x), k | (8 if np.signbit(x) else 0)


def _inverse_free_gptq(w, S, H, damp):
    """w'_k = w_k + (1 / T_kk) sum_{j<k} (w_j - q_j) T_jk with H + lambda I =
    T T^T, T upper triangular (the Cholesky factor taken from the last index
    down: T = J chol(J H J) J); no inverse of H."""
    C = H.shape[0]
    Hd = H + damp * np.mean(np.diag(H)) * np.eye(C)
    J = np.eye(C)[::-1]
    T = J @ np.linalg.cholesky(J @ Hd @ J) @ J
    R = w.shape[0]
    codes = np.zeros((R, C), np.int64)
    at = np.zeros((R, C))
    for r in range(R):
        D = np.zeros(C)
        for k in range(C):
            x = w[r, k] + (D[:k] @ T[:k, k]) / T[k, k]
            at[r, k] = x
            q, codes[r, k] = _round(x, S[r, k])
            D[k] = w[r, k] - q
    return (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8), at


@pytest.mark.parametrize("R,C,N,seed,damp", [(6, 48, 80, 1, 0.01), (4, 32, 20, 2, 0.05),
                                              (3, 64, 200, 3, 0.0)])
def test_inverse_free_gptq_equals_the_paper_form(oracle_mod, R, C, N, seed, damp):
    g = torch.Generator().manual_seed(seed)
    W = (torch.randn(R, C, generator=g) * 0.02).to(torch.bfloat16)
    X = torch.randn(N, C, generator=g)
    X[:, 5] *= 20.0
    X = X.to(torch.bfloat16)
    wu, xu = bf16_bits(W), bf16_bits(X)
    s_g = oracle_mod.global_scale(wu)
    codes = oracle_mod.scale_search_max(wu, s_g)
    H = oracle_mod.gram_full(xu)
    S = np.repeat(np.array([[oracle_mod.effective_scale(s_g, int(c)) for c in row]
                            for row in codes], np.float64), 16, axis=1)
    packed, at = _inverse_free_gptq(bits_to_f64(wu), S, H, damp)
    U = oracle_mod.gptq_factor(H, damp)
    ref, ref_at = oracle_mod.gptq_rows(wu, s_g, codes, U, np.arange(R))
    np.testing.assert_allclose(at, ref_at, rtol=1e-9, atol=1e-13)
    np.testing.assert_array_equal(packed, ref)


def test_look_ahead_split_of_the_trailing_update():
    """A panel's trailing update split into the next panel's columns and the
    columns beyond (the lower triangle of each) changes no entry the
    factorisation reads."""
    rng = np.random.default_rng(0)
    C, P0, nw, nw2 = 400, 0, 128, 128
    A = rng.standard_normal((C, C))
    X = rng.standard_normal((C, nw))
    P1, P2 = P0 + nw, P0 + nw + nw2
    full = A.copy()
    full[P1:, P1:] -= X[P1:] @ X[P1:].T
    split = A.copy()
    split[P1:, P1:P2] -= X[P1:] @ X[P1:P2].T
    split[P2:, P2:] -= X[P2:] @ X[P2:].T
    lower = np.tril(np.ones((C, C), bool))
    np.testing.assert_allclose(split[lower], full[lower], rtol=1e-12, atol=1e-12)
