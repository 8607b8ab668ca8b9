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


class Guards:
    """Output buffers with canary guard bands.  Each buffer lives inside a larger
    allocation filled with the byte 0xA5: GUARD bytes before and after it and, for
    matrices with a row stride above their width, the columns between rows.  check()
    asserts that no kernel wrote outside the buffer it was given (an out-of-bounds
    store past a ragged edge lands in a band)."""
    GUARD = 4096
    BYTE = 0xA5

    def __init__(self):
        self.bufs = []

    def _raw(self, nbytes):
        raw = torch.full((nbytes + 2 * self.GUARD,), self.BYTE, dtype=torch.uint8, device="cuda")
        return raw

    def matrix(self, rows, cols, dtype=torch.bfloat16, pad_cols=0):
        """[rows x cols] view with row stride cols + pad_cols (elements); pad_cols keeps
        rows 16-byte aligned when it is a multiple of 16 bytes."""
        esz = torch.empty(0, dtype=dtype).element_size()
        ld = cols + pad_cols
        raw = self._raw(rows * ld * esz)
        body = raw[self.GUARD:self.GUARD + rows * ld * esz].view(dtype).view(rows, ld)
        self.bufs.append((raw, rows * ld * esz, (rows, cols, ld, esz)))
        return body[:, :cols]

    def flat(self, nbytes):
        raw = self._raw(nbytes)
        self.bufs.append((raw, nbytes, None))
        return raw[self.GUARD:self.GUARD + nbytes]

    def nvfp4(self, rows, cols):
        import nvfp4_gemm_b200 as P
        codes = self.flat(rows * cols // 2).view(rows, cols // 2)
        scales = self.flat(P.pact_scale_bytes(rows, cols))
        return P.NVFP4Tensor(codes, scales, rows, cols)

    def check(self):
        torch.cuda.synchronize()
        for raw, nbytes, mat in self.bufs:
            host = raw.cpu().numpy()
            g = self.GUARD
            assert np.all(host[:g] == self.BYTE), "write before the start of an output buffer"
            assert np.all(host[g + nbytes:] == self.BYTE), "write past the end of an output buffer"
            if mat is not None:
                rows, cols, ld, esz = mat
                if ld > cols:
                    body = host[g:g + nbytes].reshape(rows, ld * esz)
                    assert np.all(body[:, cols * esz:] == self.BYTE), "write into the padding between rows"
