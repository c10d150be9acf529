"""Helpers for the GPU parity tests: host<->device moves and comparisons."""
import numpy as np
import torch


def to_dev_u64(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint64).view(np.int64)).cuda()


def to_dev_u16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).cuda()


def to_dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return to_dev_u16(bits).view(torch.bfloat16)


def to_dev_f32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def host_u64(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.uint64)


def host_u16(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.uint16)


def assert_bits_equal(got: np.ndarray, want: np.ndarray, what: str):
    """Bitwise equality, except that +0.0 and -0.0 compare equal (alpha = 0
    times a negative dot gives -0.0, which is the same value)."""
    assert got.shape == want.shape, (what, got.shape, want.shape)
    if got.dtype.kind == "f":
        same = (got.view(np.uint32 if got.itemsize == 4 else np.uint64) ==
                want.view(np.uint32 if want.itemsize == 4 else np.uint64)) | ((got == 0) & (want == 0))
    else:
        same = got == want
    bad = np.argwhere(~same)
    assert bad.size == 0, f"{what}: {len(bad)} mismatches, first at {bad[:5].tolist()}: " \
                          f"got {got[tuple(bad[0])]!r} want {want[tuple(bad[0])]!r}"


# Ternary tolerance: |y - y_ref| <= TERNARY_REL * mag, where y_ref is the float64
# oracle and mag = scale * sum |x t| (float32 accumulation over k <= 4096 terms
# has a relative error bound of about k * 2^-24 = 2.4e-4 of mag; the stated
# target is 1e-3).
TERNARY_REL = 1e-3


def assert_ternary_close(got: np.ndarray, ref: np.ndarray, mag: np.ndarray, what: str):
    err = np.abs(got.astype(np.float64) - ref)
    lim = TERNARY_REL * mag
    bad = np.argwhere(err > lim)
    assert bad.size == 0, f"{what}: {len(bad)} outside tolerance, first {bad[:3].tolist()}: " \
                          f"got {got[tuple(bad[0])]} ref {ref[tuple(bad[0])]} mag {mag[tuple(bad[0])]}"
    return float((err / np.maximum(mag, 1e-300)).max()) if err.size else 0.0
