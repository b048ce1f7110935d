"""Helpers of the GPU parity tests: host <-> device copies of bf16 bit
patterns, sentinel-guarded output buffers, and code comparisons."""
import numpy as np
import torch

SENTINEL = 0xA5


def dev_bf16(a: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bit patterns -> bf16 CUDA tensor (same shape)."""
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def dev_f32(a) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def host_u16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def host_u8(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.uint8).cpu().numpy()


class Guarded:
    """A [rows, cols] output view inside a sentinel-filled buffer with guard rows
    above and below and guard columns to the right (row stride cols + pad)."""

    def __init__(self, rows, cols, dtype, pad=16, guard_rows=2):
        self.rows, self.cols, self.pad, self.g = rows, cols, pad, guard_rows
        esz = torch.tensor([], dtype=dtype).element_size()
        self.raw = torch.full(((rows + 2 * guard_rows) * (cols + pad) * esz,), SENTINEL,
                              dtype=torch.uint8, device="cuda")
        full = self.raw.view(dtype).view(rows + 2 * guard_rows, cols + pad)
        self.full = full
        self.view = full[guard_rows:guard_rows + rows, :cols]

    def guards_intact(self) -> bool:
        f = self.full.contiguous().view(torch.uint8).view(self.rows + 2 * self.g, -1)
        esz = f.shape[1] // (self.cols + self.pad)
        top = f[: self.g]
        bot = f[self.g + self.rows:]
        right = f[self.g:self.g + self.rows, self.cols * esz:]
        return bool((top == SENTINEL).all() and (bot == SENTINEL).all() and (right == SENTINEL).all())


def e4m3_rank(codes: np.ndarray) -> np.ndarray:
    c = np.asarray(codes, np.int32)
    mag = c & 0x7F
    return np.where(c & 0x80, -mag, mag)


def e2m1_rank(codes: np.ndarray) -> np.ndarray:
    c = np.asarray(codes, np.int32)
    mag = c & 7
    return np.where(c & 8, -mag, mag)


def same_codes_e4m3(a: np.ndarray, b: np.ndarray) -> bool:
    """Bitwise equal, except that any two NaN codes (0x7F / 0xFF) count as equal."""
    a = np.asarray(a, np.uint8)
    b = np.asarray(b, np.uint8)
    nan_a = (a & 0x7F) == 0x7F
    nan_b = (b & 0x7F) == 0x7F
    return bool(np.array_equal(nan_a, nan_b) and np.array_equal(a[~nan_a], b[~nan_b]))
