"""Helpers shared by the GPU parity tests (not a test module)."""

import numpy as np
import torch

CANARY_BYTES = 512


class Guarded:
    """An output buffer with canary bytes before and after it, to catch
    out-of-bounds writes (compute-sanitizer is not available on the pool)."""

    def __init__(self, shape, dtype, device="cuda", fill=0x5A):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.n = n
        self.raw = torch.full((n + 2 * CANARY_BYTES,), fill, dtype=torch.uint8, device=device)
        self.fill = fill
        self.tensor = self.raw[CANARY_BYTES:CANARY_BYTES + n].view(dtype).view(*shape)

    def check(self):
        head = self.raw[:CANARY_BYTES]
        tail = self.raw[CANARY_BYTES + self.n:]
        assert bool((head == self.fill).all()), "write before the start of the output"
        assert bool((tail == self.fill).all()), "write past the end of the output"


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def to_cuda_bf16(x) -> torch.Tensor:
    if isinstance(x, torch.Tensor):
        return x.to(torch.bfloat16).cuda().contiguous()
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).cuda()


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |v| (normal range)."""
    a = np.abs(np.asarray(v, np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return np.ldexp(1.0, (e - 7).astype(np.int64))


def assert_codes_close(gpu: np.ndarray, ref: np.ndarray, max_frac: float = 1e-3):
    """int8 codes: every difference at most 1 LSB, on at most `max_frac` of the elements."""
    d = np.abs(gpu.astype(np.int32) - ref.astype(np.int32))
    assert d.max(initial=0) <= 1, f"code differs by {d.max()} LSB"
    frac = np.count_nonzero(d) / max(d.size, 1)
    assert frac <= max_frac, f"{frac:.2e} of codes differ (limit {max_frac})"
    return frac


def sample_rows(M: int, n: int = 256, seed: int = 0) -> np.ndarray:
    """First, last and tail rows plus seeded random ones, sorted and unique."""
    rng = np.random.default_rng(seed)
    fixed = {0, 1, M - 1, M - 2, (M // 128) * 128, max(M - 129, 0)}
    fixed = {r for r in fixed if 0 <= r < M}
    rest = rng.choice(M, size=min(n, M), replace=False)
    return np.array(sorted(fixed | set(int(r) for r in rest)))
