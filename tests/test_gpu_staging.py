"""cskv_copy_segments: the device-side scatter behind the staged upload of a step's new inputs
(16-byte, 4-byte and byte-granular segments; bit-exact)."""

import numpy as np
import pytest
import torch

from compressed_sparse_kv_compress_b200 import api

pytestmark = pytest.mark.gpu


def test_segments_of_every_alignment_land_exactly():
    rng = np.random.default_rng(11)
    src = torch.from_numpy(rng.integers(0, 256, 1 << 16, dtype=np.uint8)).cuda()
    dst = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    # (source offset, destination offset, length): aligned to 16, to 4, and not at all
    segs = [(0, 4096, 512), (16, 8192, 32768), (4, 100, 40), (8, 52, 4), (3, 60001, 13), (1001, 50000, 1)]
    src_off = torch.tensor([s for s, _, _ in segs], dtype=torch.int64, device="cuda")
    dst_ptr = torch.tensor([dst.data_ptr() + d for _, d, _ in segs], dtype=torch.int64, device="cuda")
    lens = torch.tensor([n for _, _, n in segs], dtype=torch.int64, device="cuda")
    api.copy_segments(src, src_off, dst_ptr, lens)
    torch.cuda.synchronize()
    want = np.zeros(1 << 16, np.uint8)
    s_np = src.cpu().numpy()
    for s, d, n in segs:
        want[d:d + n] = s_np[s:s + n]
    assert np.array_equal(dst.cpu().numpy(), want)
