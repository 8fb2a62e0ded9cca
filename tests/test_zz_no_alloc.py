"""hybrid_decode_attn_noalloc: the attention entry point for callers that cannot allocate
device memory (a pool that owns all device memory, a plugin host that forbids allocations
after start-up, a hot path that must not synchronise).  It keeps its split-KV partials in a
fixed array inside the library; here it must reproduce hybrid_decode_attn (the regular
entry point, given its own workspace) on two calls in a row, and refuse a call that needs
more scratch than the array holds.

Collected last on purpose, so a run that stops at the first failure has run every other
test before this one."""

import ctypes

import numpy as np
import pytest
import torch

from compressed_sparse_kv_compress_b200 import _lib, api
from oracle import indexer
from oracle import step as ostep
from synth import Workload, spec_by_name

from helpers import bounds, check_attention, dtypes, np_arrays, to_f64

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(lib, mode, w, dev, idx, out, lse, status):
    m = w.meta
    layer = "c" if mode == api.CSA else "h"
    off = dev["csa_off"] if mode == api.CSA else dev["hca_off"]
    T, H, d = dev["q_" + layer].shape
    return lib.hybrid_decode_attn_noalloc(
        mode, _p(dev["q_" + layer]), _p(dev["cmp_" + layer]), _p(off), _p(idx), 0 if idx is None else idx.shape[1],
        _p(dev["raw_" + layer]), _p(dev["raw_off"]), _p(dev["raw_t0"]), m["W"], _p(dev["sink_" + layer]),
        m["scale"], _p(dev["q_seq"]), _p(dev["q_pos"]), m["B"], T, H, d,
        _lib.BF16 if dev["q_" + layer].dtype == torch.bfloat16 else _lib.F32,
        bounds(w)["max_hca_visible"], _p(out), _p(lse), _p(status), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _regular(mode, w, dev, idx, out, lse):
    m = w.meta
    layer = "c" if mode == api.CSA else "h"
    off = dev["csa_off"] if mode == api.CSA else dev["hca_off"]
    T, H, _ = dev["q_" + layer].shape
    ws = api.attn_workspace(mode, T, H, m["k"], m["W"], bounds(w)["max_hca_visible"])
    api.hybrid_decode_attn(mode, dev["q_" + layer], dev["cmp_" + layer], off, dev["raw_" + layer], dev["raw_off"],
                           dev["q_seq"], dev["q_pos"], out, ws, window=m["W"], idx=idx, raw_tok0=dev["raw_t0"],
                           sink=dev["sink_" + layer], scale=m["scale"], lse=lse,
                           max_entries=bounds(w)["max_hca_visible"])


@pytest.mark.parametrize("kind", ["bf16", "f32"])
def test_noalloc_matches_regular_entry_point_twice(kind):
    """bf16 runs the tensor-core kernel, fp32 the CUDA-core one; both keep their partials in
    the library's array."""
    lib = _lib.load()
    if kind == "bf16":
        w = Workload(spec_by_name("b8_ctx64k").replace(batch=4, seq_len=(65536, 40001, 9000, 300), heads=64))
    else:
        w = Workload(spec_by_name("tiny").replace(batch=3, seq_len=(4096, 2000, 700), heads=16, cache="random"))
    m, a = w.meta, np_arrays(w)
    dev = w.device("cuda")
    rows = np.stack([indexer.topk_select(ostep.query_scores(m, a, dtypes(w), t), m["k"]) for t in range(m["T"])])
    idx = torch.from_numpy(rows.astype(np.int32)).cuda()
    T, H = m["T"], m["H"]
    for mode, use_idx in ((api.CSA, idx), (api.HCA, None)):
        ref = torch.empty(T, H, 128, dtype=torch.float32, device="cuda")
        ref_lse = torch.empty(T, H, dtype=torch.float32, device="cuda")
        _regular(mode, w, dev, use_idx, ref, ref_lse)
        for call in range(2):  # two calls in a row share the library's array
            out = torch.full((T, H, 128), float("nan"), dtype=torch.float32, device="cuda")
            lse = torch.full((T, H), float("nan"), dtype=torch.float32, device="cuda")
            status = torch.zeros(1, dtype=torch.int32, device="cuda")
            rc = _noalloc(lib, mode, w, dev, use_idx, out, lse, status)
            assert rc == _lib.OK, lib.cskv_status_string(rc)
            torch.cuda.synchronize()
            assert int(status.item()) == 0
            for t in range(T):
                check_attention(to_f64(out[t]), to_f64(ref[t]), extra_rel=1e-6, what=f"mode {mode} call {call} q{t}")
            assert torch.allclose(lse, ref_lse, rtol=1e-6, atol=1e-6)


def test_noalloc_refuses_more_scratch_than_it_holds():
    lib = _lib.load()
    # 4096 prefill queries x 64 heads need far more than the built-in array
    w = Workload(spec_by_name("prefill_4k_at_128k").replace(seq_len=(4096 + 2048,), queries_per_seq=4096))
    dev = w.device("cuda")
    T, H = w.meta["T"], w.meta["H"]
    need = api.attn_workspace_size(api.HCA, T, H, 0, w.meta["W"], bounds(w)["max_hca_visible"])
    assert need > _lib.NOALLOC_SCRATCH_BYTES
    out = torch.zeros(T, H, 128, dtype=torch.float32, device="cuda")
    rc = _noalloc(lib, api.HCA, w, dev, None, out, None, None)
    assert rc == _lib.ERR_WORKSPACE
    torch.cuda.synchronize()
    assert int(out.count_nonzero().item()) == 0  # nothing launched


def test_noalloc_reports_bad_arguments_as_such():
    # a bad argument is CSKV_ERR_INVALID_ARG, as from the regular entry point, even when the
    # call would also need more scratch than the array holds; nothing is launched
    lib = _lib.load()
    w = Workload(spec_by_name("b8_ctx64k").replace(batch=2, seq_len=(8192, 5000), heads=64))
    dev = w.device("cuda")
    m = w.meta
    T, H = m["T"], m["H"]
    out = torch.zeros(T, H, 128, dtype=torch.float32, device="cuda")
    idx = torch.zeros(T, m["k"], dtype=torch.int32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    def call(mode=api.CSA, k=m["k"], H_=H, scale=m["scale"], window=m["W"]):
        return lib.hybrid_decode_attn_noalloc(
            mode, _p(dev["q_c"]), _p(dev["cmp_c"]), _p(dev["csa_off"]), _p(idx), k, _p(dev["raw_c"]),
            _p(dev["raw_off"]), _p(dev["raw_t0"]), window, None, scale, _p(dev["q_seq"]), _p(dev["q_pos"]), m["B"],
            T, H_, 128, _lib.BF16, 0, _p(out), None, None, stream)

    assert call(mode=7) == _lib.ERR_INVALID_ARG
    assert call(H_=129) == _lib.ERR_INVALID_ARG
    assert call(k=0) == _lib.ERR_INVALID_ARG
    assert call(scale=-1.0) == _lib.ERR_INVALID_ARG
    assert call(k=(1 << 20) + 1) == _lib.ERR_INVALID_ARG  # also far beyond the array
    torch.cuda.synchronize()
    assert int(out.count_nonzero().item()) == 0
