"""Shared helpers for the GPU parity tests (device plumbing and comparisons only)."""
import numpy as np
import torch

TOL_BF16 = 2e-2  # max|err| <= TOL * max|ref| for bf16 (and fp32/tf32) outputs and gradients


def dev():
    return torch.device("cuda", 0)


def np64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def assert_close_rel(got, ref, tol=TOL_BF16, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    scale = float(np.max(np.abs(ref))) if ref.size else 0.0
    err = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    assert err <= tol * max(scale, 1e-30), f"{what}: max|err| {err:.3e} > {tol} * max|ref| {scale:.3e}"
    return err / max(scale, 1e-30)


def routed_buffers(meta, R):
    """Indices (numpy) of the valid rows of each expert in the padded routed buffer."""
    return [(int(meta["poff"][e]), int(meta["counts"][e])) for e in range(len(meta["counts"]))]


def idx_from_counts(counts, T, k, rng):
    """A routing whose per-expert counts are exactly `counts` (sum = T*k), every token choosing k
    distinct experts. Built greedily: token t takes the k experts with the most remaining demand."""
    counts = np.array(counts, dtype=np.int64)
    assert counts.sum() == T * k
    E = len(counts)
    rem = counts.copy()
    idx = np.zeros((T, k), dtype=np.int32)
    for t in range(T):
        # experts with the largest remaining demand (random tie-break) keep the assignment feasible
        order = np.lexsort((rng.random(E), -rem))
        ch = order[:k]
        assert np.all(rem[ch] > 0), "infeasible counts"
        rem[ch] -= 1
        idx[t] = rng.permutation(ch)
    assert np.all(rem == 0)
    return idx
