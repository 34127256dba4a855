"""The Gram kernel's inverse of M = lambda I + K^T K, emulated in float32 on
the CPU: a 2 x 2 block inverse over 64 x 64 blocks through the Schur
complement, whose two 64 x 64 inverses are Gauss-Jordan sweeps without
pivoting (M is SPD with eigenvalues >= lambda, so every pivot is >= lambda).
Checked against numpy's LU inverse on the key structures of the workloads:
random keys, the low-rank keys of the hi-res workload (condition number in
the hundreds), a single token (rank one) and no token (M = lambda I)."""
import numpy as np
import pytest


def gj(a):
    """In-place Gauss-Jordan inverse without pivoting, float32."""
    a = np.asarray(a, np.float32).copy()
    for k in range(a.shape[0]):
        p = a[k, k]
        assert p > 0
        ip = np.float32(1) / p
        r, c = a[k].copy() * ip, a[:, k].copy()
        a -= np.outer(c, r).astype(np.float32)
        a[k], a[:, k] = r, -c * ip
        a[k, k] = ip
    return a


def block_inverse(M):
    f = np.float32
    M = np.asarray(M, f)
    A, B, D = M[:64, :64], M[:64, 64:], M[64:, 64:]
    AI = gj(A)
    X = (AI @ B).astype(f)
    SI = gj((D - B.T @ X).astype(f))
    Y = (X @ SI).astype(f)
    return np.block([[AI + Y @ X.T, -Y], [-Y.T, SI]]).astype(f)


def keys(kind, rng):
    if kind == "random":
        K = rng.standard_normal((1008, 128))
    elif kind == "low-rank":
        K = rng.standard_normal((1792, 16)) @ (rng.standard_normal((16, 128)) / 4) \
            + 0.1 * rng.standard_normal((1792, 128))
    elif kind == "one-token":
        K = rng.standard_normal((1, 128))
    else:
        K = np.zeros((0, 128))
    n = np.linalg.norm(K, axis=1, keepdims=True)
    return K / np.maximum(n, 1e-12)


@pytest.mark.parametrize("kind", ["random", "low-rank", "one-token", "none"])
def test_block_inverse_matches_lu(kind):
    K = keys(kind, np.random.default_rng(5))
    M = np.eye(128) + K.T @ K
    ref = np.linalg.inv(M)
    got = block_inverse(M).astype(np.float64)
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < 1e-4
    # the symmetric inverse stays symmetric to rounding
    assert np.abs(got - got.T).max() < 1e-4 * np.abs(ref).max()
