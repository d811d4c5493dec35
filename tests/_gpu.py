"""Helpers for the GPU parity tests: host<->device moves and fp16 comparison."""
from __future__ import annotations

import numpy as np
import pytest

torch = pytest.importorskip("torch")


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


_VIEW = {np.uint8: torch.uint8, np.int8: torch.int8, np.uint16: torch.int16, np.int16: torch.int16,
         np.uint64: torch.int64, np.int64: torch.int64, np.int32: torch.int32}


def dev(a: np.ndarray | None):
    """numpy -> contiguous CUDA tensor with the same bytes (None stays None)."""
    if a is None:
        return None
    a = np.array(a, copy=True, order="C")
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    elif a.dtype == np.uint64:
        a = a.view(np.int64)
    if a.size == 0:
        return torch.empty(0, dtype=torch.from_numpy(a[:0].copy()).dtype, device="cuda")
    return torch.from_numpy(a).cuda()


def f16_out(n: int, offset_elems: int = 0):
    """fp16 output buffer of n elements; offset_elems > 0 returns a view that
    starts that many elements into a larger buffer (to test unaligned
    outputs)."""
    buf = torch.full((n + offset_elems + 8,), float("nan"), dtype=torch.float16, device="cuda")
    return buf[offset_elems:offset_elems + n]


def host_bits(t) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def status_buf():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def ulp_distance(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """binary16 ulp distance (+0 == -0, NaN == NaN, NaN vs number = huge)."""
    a = a.astype(np.int64)
    b = b.astype(np.int64)
    oa = np.where(a & 0x8000, -(a & 0x7FFF), a)
    ob = np.where(b & 0x8000, -(b & 0x7FFF), b)
    nan_a = ((a & 0x7C00) == 0x7C00) & ((a & 0x3FF) != 0)
    nan_b = ((b & 0x7C00) == 0x7C00) & ((b & 0x3FF) != 0)
    d = np.abs(oa - ob)
    d = np.where(nan_a & nan_b, 0, d)
    d = np.where(nan_a ^ nan_b, 1 << 20, d)
    return d


MAX_ULP = 1  # the tolerance the dequantized outputs must meet (expected 0)


def assert_f16_parity(got: np.ndarray, want: np.ndarray, exact: bool = True, what: str = ""):
    assert got.shape == want.shape, (got.shape, want.shape)
    d = ulp_distance(got, want)
    worst = int(d.max()) if d.size else 0
    assert worst <= MAX_ULP, f"{what}: max ulp {worst}, {int((d > 0).sum())} mismatches, first at {int(np.argmax(d > 0))}"
    if exact:
        assert int((d > 0).sum()) == 0, f"{what}: {int((d > 0).sum())} elements differ by 1 ulp"
