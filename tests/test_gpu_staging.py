"""cskv_copy_segments: the device-side scatter behind the staged upload of a step's new inputs
(16-byte, 4-byte and byte-granular segments; bit-exact), from and to device memory or mapped
page-locked host memory; cskv_mapped_pointer's answers."""

import ctypes

import numpy as np
import pytest
import torch

from compressed_sparse_kv_compress_b200 import _lib, api

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


# (source offset, destination offset, length) in buffers of 128 KiB, destinations disjoint; the
# last takes two batches of loads per thread (2049 16-byte words over 256 threads x 8)
SEGS = [(0, 4096, 512), (16, 8192, 32768), (4, 100, 40), (8, 52, 4), (3, 60001, 13), (1001, 50000, 1),
        (32, 65536, 16 * 2049)]
NBUF = 1 << 17


@pytest.mark.parametrize("src_host,dst_host", [(True, False), (False, True), (True, True)])
def test_segments_between_host_and_device_memory(src_host, dst_host):
    # zero-copy: the kernel reads or writes page-locked host memory through its mapped address
    rng = np.random.default_rng(12)
    data = torch.from_numpy(rng.integers(0, 256, NBUF, dtype=np.uint8))
    src = data.pin_memory() if src_host else data.cuda()
    dst = (torch.zeros(NBUF, dtype=torch.uint8).pin_memory() if dst_host
           else torch.zeros(NBUF, dtype=torch.uint8, device="cuda"))
    src_p, dst_p = api.mapped_pointer(src), api.mapped_pointer(dst)
    if not src_host:
        assert src_p == src.data_ptr()
    src_off = torch.tensor([s for s, _, _ in SEGS], dtype=torch.int64, device="cuda")
    dst_ptr = torch.tensor([dst_p + d for _, d, _ in SEGS], dtype=torch.int64, device="cuda")
    lens = torch.tensor([n for _, _, n in SEGS], dtype=torch.int64, device="cuda")
    api.copy_segments(src_p, src_off, dst_ptr, lens)
    torch.cuda.synchronize()
    want = np.zeros(NBUF, np.uint8)
    s_np = data.numpy()
    for s, d, n in SEGS:
        want[d:d + n] = s_np[s:s + n]
    assert np.array_equal(dst.cpu().numpy(), want)


def test_mapped_pointer_refuses_pageable_host_memory():
    lib = _lib.load()
    out = ctypes.c_void_p(1)
    pageable = torch.zeros(4096, dtype=torch.uint8)
    assert not pageable.is_pinned()
    assert lib.cskv_mapped_pointer(ctypes.c_void_p(pageable.data_ptr()), ctypes.byref(out)) == _lib.ERR_INVALID_ARG
    assert out.value is None
    with pytest.raises(_lib.CskvError):
        api.mapped_pointer(pageable)
    pinned = pageable.pin_memory()
    assert api.mapped_pointer(pinned[16:]) == api.mapped_pointer(pinned) + 16
