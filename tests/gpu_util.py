"""Helpers for the GPU parity tests: numpy <-> device tensors, comparisons."""
import numpy as np
import torch


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host_bits(t: torch.Tensor) -> np.ndarray:
    """Device tensor -> numpy with the same bytes (bf16 as uint16)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def assert_bits_equal(got, want, what=""):
    got = np.asarray(got)
    want = np.asarray(want)
    assert got.shape == want.shape, f"{what}: shape {got.shape} != {want.shape}"
    if got.dtype == np.float32:
        gb, wb = got.view(np.uint32), want.view(np.uint32)
        # NaN payloads are not part of the contract: compare NaN positions only
        gn, wn = np.isnan(got), np.isnan(want)
        ok = (gb == wb) | (gn & wn)
    else:
        ok = got == want
    if not ok.all():
        idx = np.argwhere(~ok)
        first = tuple(idx[0])
        raise AssertionError(f"{what}: {(~ok).sum()} of {ok.size} differ; first at {first}: "
                             f"got {got[first]!r} want {want[first]!r}")


def sample_rows(rows: int, n: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    pick = rng.choice(rows, size=min(n, rows), replace=False)
    return np.unique(np.concatenate([pick, [0, rows - 1]])).astype(np.int64)
