"""Helpers shared by the tests: moving BF16 bit patterns between numpy and torch,
reading NVFP4 tensors back, and the floating-point parity bar."""
import numpy as np
import torch


def to_dev(bits: np.ndarray) -> torch.Tensor:
    """uint16 BF16 bit pattern -> CUDA bfloat16 tensor."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def to_bits(t: torch.Tensor) -> np.ndarray:
    """CUDA bfloat16 tensor -> uint16 numpy bit pattern."""
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def nvfp4_host(t):
    """(codes [rows x cols/2], packed scales) of a device NVFP4Tensor as numpy."""
    return t.codes.cpu().numpy(), t.scales.cpu().numpy()


def assert_nvfp4_equal(dev, ref, orc, what=""):
    """Bit-exact comparison of a device NVFP4 tensor with an oracle one (codes and
    the full padded scale buffer, padding included)."""
    codes, scales = nvfp4_host(dev)
    bad = np.argwhere(codes != ref.codes)
    assert bad.size == 0, f"{what}: {len(bad)} code bytes differ, first at {bad[:3].tolist()}"
    want = orc.pack_scales(ref.scales, ref.rows, ref.cols)
    bad = np.nonzero(scales != want)[0]
    assert bad.size == 0, f"{what}: {bad.size} scale bytes differ, first at {bad[:3].tolist()}"


def tol_bound(ref: np.ndarray) -> np.ndarray:
    """|gpu - oracle| <= 8e-3 |oracle| + 1e-3 rms(oracle), elementwise."""
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    return 8e-3 * np.abs(ref) + 1e-3 * rms


def assert_close(got: np.ndarray, ref: np.ndarray, what=""):
    got = np.asarray(got, dtype=np.float64)
    err = np.abs(got - ref)
    bound = tol_bound(ref)
    bad = np.argwhere(~(err <= bound))
    if bad.size:
        i = tuple(bad[0])
        raise AssertionError(f"{what}: {len(bad)}/{ref.size} outside tolerance; first {i}: "
                             f"got {got[i]!r} ref {ref[i]!r} bound {bound[i]!r}; max err/bound "
                             f"{np.max(err / np.maximum(bound, 1e-300)):.3g}")
