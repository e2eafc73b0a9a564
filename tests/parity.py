"""Helpers shared by the GPU parity tests: moving seeded inputs to the device
and comparing the CUDA path's results with the CPU oracle's."""

import numpy as np

# Output tolerance of the float32 result against the oracle's float64 result.
MAX_ABS = 2e-2
MEAN_ABS = 2e-3
MIN_COS = 0.9999


def to_dev(bits):
    import torch

    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def bf16_dev_to_f64(t):
    import torch

    return t.float().cpu().numpy().astype(np.float64)


def compare_out(got: np.ndarray, ref: np.ndarray) -> dict:
    got = np.asarray(got, dtype=np.float64).ravel()
    ref = np.asarray(ref, dtype=np.float64).ravel()
    err = np.abs(got - ref)
    cos = float(np.dot(got, ref) / (np.linalg.norm(got) * np.linalg.norm(ref) + 1e-300))
    return {"max_abs": float(err.max()), "mean_abs": float(err.mean()), "cos": cos, "n": int(got.size)}


def assert_out_ok(stats: dict, what: str = "out") -> None:
    assert stats["max_abs"] <= MAX_ABS, (what, stats)
    assert stats["mean_abs"] <= MEAN_ABS, (what, stats)
    assert stats["cos"] >= MIN_COS, (what, stats)


def mask_mismatch(gpu_idx: np.ndarray, ref_idx: np.ndarray, near_tie: np.ndarray):
    """Rows whose lists differ; every one of them must be a near tie of the oracle."""
    diff = np.any(gpu_idx != ref_idx, axis=-1)
    bad = diff & ~near_tie
    return diff, bad


def mask_record(case: str, near_tie: np.ndarray, diff: np.ndarray, bad: np.ndarray) -> dict:
    """Structured count of the mask comparison of one case."""
    return {"case": case, "rows": int(near_tie.size), "near_tie_rows": int(near_tie.sum()),
            "differing_rows": int(diff.sum()), "differing_off_near_tie": int(bad.sum())}


def sample_items(B, H, nblk, per_head=4, seed=0):
    """Query blocks to check at full size: first, last and a few seeded ones per head."""
    rng = np.random.default_rng(seed)
    items = []
    for b in range(B):
        for h in range(H):
            picks = {0, nblk - 1}
            picks.update(int(x) for x in rng.integers(0, nblk, size=max(0, per_head - 2)))
            items += [(b, h, i) for i in sorted(picks)]
    return items
