"""Helpers shared by the GPU parity tests: moving seeded numpy inputs to the
device, guard-byte canaries around outputs, and the comparisons."""
import numpy as np
import torch

GUARD = 4096  # bytes of canary on each side of an output buffer
CANARY = 0xA5


def dev(a: np.ndarray, dtype=None) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


def bf16_dev(bits: np.ndarray) -> torch.Tensor:
    return dev(bits.view(np.int16), torch.int16).view(torch.bfloat16)


class Guarded:
    """A device tensor with canary bytes before and after it."""

    def __init__(self, shape, dtype):
        self.shape = tuple(shape)
        self.dtype = dtype
        nbytes = int(np.prod(self.shape)) * torch.empty(0, dtype=dtype).element_size()
        self.raw = torch.full((GUARD + nbytes + GUARD,), CANARY, dtype=torch.uint8, device="cuda")
        self.tensor = self.raw[GUARD:GUARD + nbytes].view(dtype).view(self.shape) if nbytes else \
            torch.empty(self.shape, dtype=dtype, device="cuda")

    def intact(self) -> bool:
        head = self.raw[:GUARD]
        tail = self.raw[self.raw.numel() - GUARD:]
        return bool((head == CANARY).all().item() and (tail == CANARY).all().item())


def host(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _normwise(got: np.ndarray, ref: np.ndarray, kind: str):
    """The layer's output tolerance: max|y - y_ref| / max|y_ref| <= 2e-3 for
    bf16 output and 1e-5 for fp32.  Returns both sides in float64."""
    if kind == "bf16":
        g, r = bf16_bits_to_f64(got), bf16_bits_to_f64(ref)
        tol = 2e-3
    else:
        g, r = got.astype(np.float64), ref.astype(np.float64)
        tol = 1e-5
    denom = max(np.abs(r).max(), 1e-30) if r.size else 1.0
    err = np.abs(g - r).max() / denom if g.size else 0.0
    assert err <= tol, f"normwise error {err:.3e} > {tol}"
    return g, r


def assert_output_close(got: np.ndarray, ref: np.ndarray, kind: str):
    """The normwise tolerance, and then bit equality, which this library
    claims for the plain epilogue because both sides follow the same fp32
    operation order."""
    _normwise(got, ref, kind)
    mism = int((got != ref).sum())
    assert mism == 0, f"{mism} of {got.size} elements differ from the oracle"


def assert_swiglu_close(got: np.ndarray, ref: np.ndarray, kind: str):
    """SwiGLU outputs: the device computes silu(g) * u in fp32, the oracle in
    double, each rounded once, so they may differ by one unit in the last
    place.  Checked: the normwise tolerance, and elementwise
    |y - y_ref| <= 2^-7 |y_ref| (one bf16 ulp) for bf16 or 4e-6 |y_ref| (a few
    fp32 ulp) for fp32, with an absolute floor far below the output scale."""
    g, r = _normwise(got, ref, kind)
    if not g.size:
        return
    rel = 2.0 ** -7 if kind == "bf16" else 4e-6
    floor = 1e-30 * max(np.abs(r).max(), 1e-30)
    bad = np.abs(g - r) > rel * np.abs(r) + floor
    assert not bad.any(), f"{int(bad.sum())} elements beyond one ulp, e.g. {g[bad][:3]} vs {r[bad][:3]}"
