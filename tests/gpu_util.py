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


def assert_output_close(got: np.ndarray, ref: np.ndarray, kind: str):
    """The benchmark spec's tolerance (normwise: max|y - y_ref| / max|y_ref|, 2e-3 for
    bf16 output and 1e-5 for fp32), and then bit equality, which this library
    claims because both sides follow the same fp32 operation order."""
    if kind == "bf16":
        g, r = bf16_bits_to_f64(got), bf16_bits_to_f64(ref)
        tol = 2e-3
    else:
        g, r = got.astype(np.float64), ref.astype(np.float64)
        tol = 1e-5
    denom = max(np.abs(r).max(), 1e-30)
    err = np.abs(g - r).max() / denom if g.size else 0.0
    assert err <= tol, f"normwise error {err:.3e} > {tol}"
    mism = int((got != ref).sum())
    assert mism == 0, f"{mism} of {got.size} elements differ from the oracle"
