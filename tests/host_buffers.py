"""Host buffers for the CPU tests that pass host pointers through the C ABI."""
import numpy as np
import torch


def aligned_zeros(shape, dtype, align=256):
    """A zeroed host tensor whose data starts on an `align`-byte boundary (the library checks it)."""
    n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
    raw = torch.zeros(n + align, dtype=torch.uint8)
    off = (-raw.data_ptr()) % align
    return raw[off:off + n].view(dtype).view(*shape)
