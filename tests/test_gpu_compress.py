"""GPU parity of csa_compress / hca_compress (through the C ABI) against the oracle."""

import numpy as np
import pytest
import torch

from oracle import codecs, compress
from oracle import step as ostep
from synth import Workload, spec_by_name

from helpers import bulk_bounds, compress_tol_check, decode_step, dtypes, np_arrays, storage_rows

pytestmark = pytest.mark.gpu


def _bulk(w):
    step, dev = decode_step(w)
    step.bulk_compress(*bulk_bounds(w))
    torch.cuda.synchronize()
    assert int(step.status.item()) == 0
    _, _, new = ostep.compress_step(w.meta, np_arrays(w), dtypes(w), bulk=True)
    return dev, new


@pytest.mark.parametrize("name", ["tiny", "tiny_bias"])
def test_bulk_fp32(name):
    w = Workload(spec_by_name(name))
    dev, new = _bulk(w)
    m = w.meta
    for layer, key, off in (("csa", "cmp_c", "csa_off"), ("hca", "cmp_h", "hca_off")):
        ents, ref = new[(layer, 0)]
        got = storage_rows(dev[key])[m[off][0] + ents]
        compress_tol_check(got, ref, "f32", f"{name}/{layer}")


@pytest.mark.parametrize("seed", [0, 3])
def test_bulk_bf16_ragged_with_biases(seed):
    # lengths that are not multiples of 4 or 128 exercise partial last blocks
    spec = spec_by_name("tiny").replace(batch=3, seq_len=(1001, 4099, 70001), dtype="bf16", heads=8,
                                        biases=True, seed=seed)
    w = Workload(spec)
    dev, new = _bulk(w)
    m = w.meta
    for b in range(3):
        for layer, key, off in (("csa", "cmp_c", "csa_off"), ("hca", "cmp_h", "hca_off")):
            ents, ref = new[(layer, b)]
            got = storage_rows(dev[key])[m[off][b] + ents]
            compress_tol_check(got, ref, "bf16", f"seq{b}/{layer}")


def test_bulk_bf16_more_entries_than_one_grid():
    # 140001 tokens: 35001 CSA entries (more than the 32768 warps of a whole-cache grid) and
    # 1094 HCA entries (more than its 1024), so warps and CTAs loop over entries; checked on
    # entries around the loops' wrap points and at both ends
    spec = spec_by_name("tiny").replace(batch=1, seq_len=(140001,), dtype="bf16", heads=8, biases=True, seed=5)
    w = Workload(spec)
    step, dev = decode_step(w)
    step.bulk_compress(*bulk_bounds(w))
    torch.cuda.synchronize()
    assert int(step.status.item()) == 0
    m, a = w.meta, np_arrays(w)
    n = m["n"][0]
    dec = {k: codecs.decode(a[k], "bf16") for k in ("x_a", "z_a", "x_b", "z_b", "x_h", "z_h")}
    bias = {k: np.asarray(a[k], dtype=np.float64) for k in ("bias_a", "bias_b", "bias_h")}
    csa_ents = np.r_[0:3, 32766:32771, 35000:35001]
    ref = compress.csa_compress(csa_ents, n, dec["x_a"], dec["z_a"], dec["x_b"], dec["z_b"], bias["bias_a"],
                                bias["bias_b"])
    got = storage_rows(dev["cmp_c"])[m["csa_off"][0] + csa_ents]
    compress_tol_check(got, ref, "bf16", "large/csa")
    hca_ents = np.r_[0:2, 1022:1027, 1093:1094]
    ref = compress.hca_compress(hca_ents, n, dec["x_h"], dec["z_h"], bias["bias_h"])
    got = storage_rows(dev["cmp_h"])[m["hca_off"][0] + hca_ents]
    compress_tol_check(got, ref, "bf16", "large/hca")


def test_incremental_tail_compress_touches_only_its_entries():
    spec = spec_by_name("b8_ctx64k").replace(batch=4, seq_len=(70001, 4096, 4097, 129), heads=8)
    w = Workload(spec)
    step, dev = decode_step(w)
    before_c = dev["cmp_c"].clone()
    before_h = dev["cmp_h"].clone()
    step.csa_layer()
    step.hca_layer()
    torch.cuda.synchronize()
    assert int(step.status.item()) == 0
    m = w.meta
    cmp_c, cmp_h, new = ostep.compress_step(m, np_arrays(w), dtypes(w))
    changed_c = np.zeros(len(before_c), bool)
    changed_h = np.zeros(len(before_h), bool)
    for b in range(4):
        ents, ref = new[("csa", b)]
        rows = m["csa_off"][b] + ents
        compress_tol_check(storage_rows(dev["cmp_c"])[rows], ref, "bf16", f"csa seq{b}")
        changed_c[rows] = True
        ents, ref = new[("hca", b)]
        rows = m["hca_off"][b] + ents
        compress_tol_check(storage_rows(dev["cmp_h"])[rows], ref, "bf16", f"hca seq{b}")
        changed_h[rows] = True
    assert torch.equal(dev["cmp_c"][torch.from_numpy(~changed_c).cuda()], before_c[torch.from_numpy(~changed_c).cuda()])
    assert torch.equal(dev["cmp_h"][torch.from_numpy(~changed_h).cuda()], before_h[torch.from_numpy(~changed_h).cuda()])


def test_missing_tail_rows_are_flagged_not_read():
    from compressed_sparse_kv_compress_b200 import api
    spec = spec_by_name("b8_ctx64k").replace(batch=1, seq_len=(4100,), heads=8)
    w = Workload(spec)
    dev = w.device("cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    first = torch.tensor([w.meta["csa_first"][0] - 3], dtype=torch.int64, device="cuda")  # before the tail
    num = torch.tensor([1], dtype=torch.int64, device="cuda")
    before = dev["cmp_c"].clone()
    api.csa_compress(dev["x_a"], dev["z_a"], dev["x_b"], dev["z_b"], dev["csa_x_off"], dev["csa_off"], dev["cmp_c"],
                     max_blocks=1, tok0=dev["csa_t0"], first_block=first, num_blocks=num, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & 2
    assert torch.equal(before, dev["cmp_c"])
