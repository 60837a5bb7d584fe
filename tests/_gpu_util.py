"""Helpers shared by the GPU parity tests: move seeded bf16 inputs to the
device and compare the CUDA path's outputs with the fp64 oracle."""
import numpy as np

import workloads as W

# Tolerances for bf16 inputs with fp32 accumulation against the fp64 oracle.
O_MAX_ERR = 2e-2
O_MEAN_ERR = 2e-3
LSE_MAX_ERR = 1e-3


def dev_bf16(bits: np.ndarray):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.cuda()


def host_f64(t) -> np.ndarray:
    import torch
    return t.detach().float().cpu().numpy().astype(np.float64)


def compare(o_gpu: np.ndarray, o_ref: np.ndarray, lse_gpu=None, lse_ref=None, what=""):
    """Assert the O / LSE tolerances; -inf LSE entries must match exactly."""
    err = np.abs(o_gpu - o_ref)
    assert np.isfinite(o_gpu).all(), "%s: non-finite O" % what
    mx, mean = float(err.max(initial=0.0)), float(err.mean()) if err.size else 0.0
    assert mx <= O_MAX_ERR, "%s: O max err %.3e" % (what, mx)
    assert mean <= O_MEAN_ERR, "%s: O mean err %.3e" % (what, mean)
    if lse_gpu is not None:
        fin = np.isfinite(lse_ref)
        assert np.array_equal(np.isfinite(lse_gpu), fin), "%s: LSE finiteness differs" % what
        assert (lse_gpu[~fin] == -np.inf).all()
        if fin.any():
            le = float(np.abs(lse_gpu[fin] - lse_ref[fin]).max())
            assert le <= LSE_MAX_ERR, "%s: LSE max err %.3e" % (what, le)
    return mx, mean


def sample_rows(rng, B, Hq, Sq, n, extra_i=()):
    """(b, h, i) rows: n random ones plus the first/last rows and given positions."""
    rows = set()
    for i in list(extra_i) + [0, Sq - 1]:
        if 0 <= i < Sq:
            rows.add((int(rng.integers(B)), int(rng.integers(Hq)), int(i)))
    while len(rows) < n + len(extra_i) + 2 and len(rows) < B * Hq * Sq:
        rows.add((int(rng.integers(B)), int(rng.integers(Hq)), int(rng.integers(Sq))))
    return np.array(sorted(rows), dtype=np.int32)
