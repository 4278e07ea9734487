"""Helpers for the GPU parity tests: device buffers, one selection/attention
pass through the C ABI, and comparisons against the oracle."""
import numpy as np
import torch

ATOL_MAX = 1e-2   # attention: max-abs error bound against the fp64 oracle
ATOL_MEAN = 1e-3  # attention: mean-abs error bound


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def host_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


class Buffers:
    """Device workspace and list buffers for one (B, H, N, d) shape."""

    def __init__(self, sa, B, H, N, d, cap):
        self.sa = sa
        self.B, self.H, self.N, self.d, self.nB, self.cap = B, H, N, d, N // 64, cap
        self.ws_bytes = sa.sa_workspace_size(B, H, N, d)
        self.ws = torch.zeros(self.ws_bytes, dtype=torch.uint8, device="cuda")
        sa.sa_workspace_init(self.ws, self.ws_bytes)
        self.idx = torch.full((B, H, self.nB, cap), -7, dtype=torch.int32, device="cuda")
        self.counts = torch.full((B, H, self.nB), -7, dtype=torch.int32, device="cuda")

    def lists(self):
        return self.idx.cpu().numpy(), self.counts.cpu().numpy()


def compare_lists(idx_a, cnt_a, idx_b, cnt_b):
    """Counts equal and the first `count` entries of every row equal."""
    cnt_a = np.asarray(cnt_a).reshape(-1, cnt_a.shape[-1])
    cnt_b = np.asarray(cnt_b).reshape(-1, cnt_b.shape[-1])
    assert np.array_equal(cnt_a, cnt_b), "counts differ in %d rows" % int(np.sum(cnt_a != cnt_b))
    ia = idx_a.reshape(cnt_a.shape + (-1,))
    ib = idx_b.reshape(cnt_b.shape + (-1,))
    bad = 0
    for r in range(cnt_a.shape[0]):
        for i in range(cnt_a.shape[1]):
            c = cnt_a[r, i]
            if c and not np.array_equal(ia[r, i, :c], ib[r, i, :c]):
                bad += 1
    assert bad == 0, "%d block lists differ" % bad


def check_attention(out_gpu: np.ndarray, out_ref: np.ndarray, live: np.ndarray):
    """out_* [rows, d]; live: bool [rows] rows that have at least one tile."""
    err = np.abs(out_gpu - out_ref)
    if live.any():
        assert err[live].max() <= ATOL_MAX, "max-abs %.3g" % err[live].max()
        assert err[live].mean() <= ATOL_MEAN, "mean-abs %.3g" % err[live].mean()
    assert np.all(out_gpu[~live] == 0.0), "rows without tiles must be exactly zero"
    return float(err[live].max()) if live.any() else 0.0, float(err[live].mean()) if live.any() else 0.0


def sample_rows(B, H, N, frac, seed, must=()):
    rng = np.random.default_rng(seed)
    n = max(1, int(B * H * N * frac))
    rows = set(rng.choice(B * H * N, size=n, replace=False).tolist())
    rows.update(must)
    return np.array(sorted(rows), dtype=np.int64)
