"""The C-ABI library builds, loads and exports every symbol its header declares;
argument validation rejects bad calls before touching the GPU (no compute here)."""

import ctypes
import os
import re

import pytest

from compressed_sparse_kv_compress_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def _declared():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"CSKV_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)
    return names


def test_header_declares_the_four_operations():
    names = _declared()
    for op in ("csa_compress", "hca_compress", "lindex_score_topk", "hybrid_decode_attn"):
        assert op in names


def test_every_declared_symbol_is_exported(lib):
    for name in _declared():
        assert hasattr(lib, name), name
        assert name in _lib.SIGNATURES, f"binding lacks {name}"


def test_library_is_sm100a_and_in_tree(lib):
    assert os.path.dirname(_lib.LIB_PATH) == os.path.join(ROOT, "compressed_sparse_kv_compress_b200")
    assert lib.cskv_version() >= 100


def test_status_strings(lib):
    for s in range(5):
        assert lib.cskv_status_string(s)
    assert b"INVALID" in lib.cskv_status_string(_lib.ERR_INVALID_ARG)


def _p(v=0x1000):
    return ctypes.c_void_p(v)


def test_compress_validation(lib):
    nul = None

    def csa(x=_p(), z=_p(), xb=nul, zb=nul, out=_p(), in_dt=1, out_dt=1, max_blocks=4, norm=0, gamma=nul, eps=1e-6,
            k_tok=nul, k_dt=1, Di=64, codes=_p(), scale=_p(), flags=0):
        return lib.csa_compress(x, z, xb, zb, nul, nul, _p(), nul, 1, _p(), nul, nul, max_blocks, in_dt, out_dt, out,
                                norm, gamma, eps, k_tok, k_dt, Di, codes, scale, flags, nul, nul)

    def hca(batch=1, in_dt=1, max_blocks=4, norm=0, gamma=nul, eps=1e-6):
        return lib.hca_compress(_p(), _p(), nul, _p(), nul, batch, _p(), nul, nul, max_blocks, in_dt, 1, _p(), norm,
                                gamma, eps, nul, nul)

    assert csa(x=nul) == _lib.ERR_INVALID_ARG               # null rows
    assert csa(xb=_p()) == _lib.ERR_INVALID_ARG             # x_b without z_b
    assert csa(out=_p(0x1004)) == _lib.ERR_INVALID_ARG      # misaligned output
    assert csa(flags=2) == _lib.ERR_INVALID_ARG             # unknown flag bit
    assert csa(flags=1, max_blocks=0) == _lib.OK            # the overlap permission alone is valid
    assert hca(in_dt=2) == _lib.ERR_UNSUPPORTED             # fp8 rows are not a compression input
    assert hca(batch=0) == _lib.ERR_INVALID_ARG             # bad batch / bad enum
    assert hca(in_dt=7) == _lib.ERR_INVALID_ARG
    # RMSNorm arguments
    assert csa(norm=2) == _lib.ERR_INVALID_ARG
    assert hca(norm=1, eps=-1.0) == _lib.ERR_INVALID_ARG
    assert hca(norm=1, eps=float("nan")) == _lib.ERR_INVALID_ARG
    assert hca(norm=1, gamma=_p(0x1002)) == _lib.ERR_INVALID_ARG
    # fused key pooling arguments
    assert csa(k_tok=_p(), codes=nul) == _lib.ERR_INVALID_ARG
    assert csa(k_tok=_p(), Di=96) == _lib.ERR_UNSUPPORTED
    assert csa(k_tok=_p(), k_dt=2) == _lib.ERR_UNSUPPORTED
    assert csa(k_tok=_p(0x1008)) == _lib.ERR_INVALID_ARG
    # the query-side RMSNorm
    assert lib.rmsnorm_heads(_p(), 2, 10, 128, nul, 1e-6, _p(), nul) == _lib.ERR_UNSUPPORTED  # fp8
    assert lib.rmsnorm_heads(_p(), 1, 10, 64, nul, 1e-6, _p(), nul) == _lib.ERR_UNSUPPORTED
    assert lib.rmsnorm_heads(_p(), 1, 10, 128, nul, -1.0, _p(), nul) == _lib.ERR_INVALID_ARG
    assert lib.rmsnorm_heads(_p(0x1008), 1, 10, 128, nul, 1e-6, _p(), nul) == _lib.ERR_INVALID_ARG
    assert lib.rmsnorm_heads(nul, 1, 0, 128, nul, 1e-6, nul, nul) == _lib.OK
    # nothing to do
    assert hca(max_blocks=0) == _lib.OK
    assert csa(max_blocks=0, norm=1, k_tok=_p()) == _lib.OK


def test_indexer_validation(lib):
    nul = None
    args = dict(Hi=8, Di=64, k=16, dtype=_lib.FP8E4M3)

    def call(**kw):
        a = {**args, **kw}
        return lib.lindex_score_topk(_p(), nul, _p(), nul, nul, _p(), _p(), _p(), 1, kw.get("T", 1), a["Hi"], a["Di"],
                                     a["k"], a["dtype"], 100, _p(), nul, kw.get("pf", nul), kw.get("pf_bytes", 0),
                                     _p(), 1 << 20, nul, nul)

    assert call(dtype=9) == _lib.ERR_INVALID_ARG
    assert call(dtype=_lib.BF16) == _lib.ERR_UNSUPPORTED
    assert call(Di=96) == _lib.ERR_UNSUPPORTED
    assert call(Hi=17) == _lib.ERR_UNSUPPORTED
    assert call(k=0) == _lib.ERR_INVALID_ARG
    assert call(T=0) == _lib.OK
    assert call(pf=_p(0x1008), pf_bytes=512) == _lib.ERR_INVALID_ARG  # misaligned prefetch rows
    assert call(pf=_p(), pf_bytes=100) == _lib.ERR_INVALID_ARG  # row size not a multiple of 16
    # the MXFP4 variant
    def fp4(Hi=8, Di=64, k=16, T=1, kbs=_p(), qc=_p()):
        return lib.lindex_score_topk_mxfp4(qc, _p(), nul, _p(), kbs, nul, _p(), _p(), _p(), 1, T, Hi, Di, k, 100,
                                           _p(), nul, nul, 0, _p(), 1 << 20, nul, nul)

    assert fp4(Di=96) == _lib.ERR_UNSUPPORTED
    assert fp4(Hi=17) == _lib.ERR_UNSUPPORTED
    assert fp4(Hi=0) == _lib.ERR_INVALID_ARG
    assert fp4(k=0) == _lib.ERR_INVALID_ARG
    assert fp4(qc=nul) == _lib.ERR_INVALID_ARG
    assert fp4(qc=_p(0x1008)) == _lib.ERR_INVALID_ARG     # codes not 16-byte aligned
    assert fp4(Di=128, kbs=_p(0x1002)) == _lib.ERR_INVALID_ARG  # 4 scale bytes per key: 4-aligned
    assert fp4(T=0) == _lib.OK
    assert lib.lindex_topk_from_scores(nul, 10, _p(), 1, 4, 10, _p(), nul, _p(), 1 << 20, nul,
                                       nul) == _lib.ERR_INVALID_ARG
    assert lib.lindex_topk_from_scores(_p(), 5, _p(), 1, 4, 10, _p(), nul, _p(), 1 << 20, nul,
                                       nul) == _lib.ERR_INVALID_ARG


def test_attention_validation(lib):
    nul = None

    def call(mode=0, d=128, H=16, dtype=1, idx=_p(), k=8, T=1, scale=0.1, noalloc=False):
        if noalloc:  # the allocation-free variant: same arguments minus the workspace
            return lib.hybrid_decode_attn_noalloc(mode, _p(), _p(), _p(), idx, k, _p(), _p(), nul, 128, nul, scale,
                                                  _p(), _p(), 1, T, H, d, dtype, 0, _p(), nul, nul, nul)
        return lib.hybrid_decode_attn(mode, _p(), _p(), _p(), idx, k, _p(), _p(), nul, 128, nul, scale, _p(), _p(), 1,
                                      T, H, d, dtype, 0, _p(), nul, _p(), 1 << 20, nul, nul)

    for na in (False, True):  # both entry points report the same error for the same mistake
        assert call(mode=5, noalloc=na) == _lib.ERR_INVALID_ARG
        assert call(mode=0x400 | 1, noalloc=na) == _lib.ERR_INVALID_ARG  # an unknown flag bit
        assert call(mode=0x800 | _lib.ATTN_KV_FP8, noalloc=na) == _lib.ERR_INVALID_ARG
        assert call(mode=_lib.ATTN_KV_FP8 | 1, T=0, noalloc=na) == _lib.OK  # HCA over FP8 rows: valid
        assert call(mode=_lib.ATTN_PAIRS | 7, noalloc=na) == _lib.ERR_INVALID_ARG
        assert call(mode=_lib.ATTN_PAIRS | 1, T=0, noalloc=na) == _lib.OK  # HCA with pairs: valid
        assert call(d=64, noalloc=na) == _lib.ERR_UNSUPPORTED
        assert call(dtype=_lib.FP8E4M3, noalloc=na) == _lib.ERR_UNSUPPORTED
        assert call(H=0, noalloc=na) == _lib.ERR_INVALID_ARG
        assert call(H=129, noalloc=na) == _lib.ERR_INVALID_ARG
        assert call(idx=nul, noalloc=na) == _lib.ERR_INVALID_ARG
        assert call(k=0, noalloc=na) == _lib.ERR_INVALID_ARG
        # the softmax scale must be positive and finite
        for bad in (0.0, -0.1, float("inf"), float("nan")):
            assert call(scale=bad, noalloc=na) == _lib.ERR_INVALID_ARG
        assert call(T=0, noalloc=na) == _lib.OK


def test_copy_segments_validation(lib):
    # nothing is launched for these (no GPU needed): bad counts and missing arrays are
    # refused on the host, an empty list is a no-op
    nul = None
    assert lib.cskv_copy_segments(_p(), _p(), _p(), _p(), -1, nul) == _lib.ERR_INVALID_ARG
    assert lib.cskv_copy_segments(nul, _p(), _p(), _p(), 3, nul) == _lib.ERR_INVALID_ARG
    assert lib.cskv_copy_segments(_p(), nul, _p(), _p(), 3, nul) == _lib.ERR_INVALID_ARG
    assert lib.cskv_copy_segments(_p(), _p(), nul, _p(), 3, nul) == _lib.ERR_INVALID_ARG
    assert lib.cskv_copy_segments(_p(), _p(), _p(), nul, 3, nul) == _lib.ERR_INVALID_ARG
    assert lib.cskv_copy_segments(nul, nul, nul, nul, 0, nul) == _lib.OK


def test_kv_quantize_fp8_validation(lib):
    # refused on the host before any launch (no GPU needed); n == 0 is a no-op
    nul = None
    assert lib.kv_quantize_fp8(_p(), _lib.F32, -1, _p(), nul) == _lib.ERR_INVALID_ARG
    assert lib.kv_quantize_fp8(_p(), _lib.F32, 8 * (2 ** 31 - 1) + 1, _p(), nul) == _lib.ERR_INVALID_ARG
    assert lib.kv_quantize_fp8(_p(), 7, 4, _p(), nul) == _lib.ERR_INVALID_ARG
    assert lib.kv_quantize_fp8(_p(), _lib.FP8E4M3, 4, _p(), nul) == _lib.ERR_UNSUPPORTED
    assert lib.kv_quantize_fp8(nul, _lib.BF16, 4, _p(), nul) == _lib.ERR_INVALID_ARG
    assert lib.kv_quantize_fp8(_p(), _lib.BF16, 4, nul, nul) == _lib.ERR_INVALID_ARG
    assert lib.kv_quantize_fp8(_p(0x1008), _lib.BF16, 4, _p(), nul) == _lib.ERR_INVALID_ARG  # misaligned
    assert lib.kv_quantize_fp8(nul, _lib.F32, 0, nul, nul) == _lib.OK


def test_mapped_pointer_validation(lib):
    # null arguments are refused before any CUDA query; the out-pointer is cleared
    out = ctypes.c_void_p(1)
    assert lib.cskv_mapped_pointer(None, ctypes.byref(out)) == _lib.ERR_INVALID_ARG
    assert out.value is None
    assert lib.cskv_mapped_pointer(_p(), None) == _lib.ERR_INVALID_ARG


def test_pool_keys_validation(lib):
    nul = None
    # (k_tok, in_dtype, Di, tok_off, tok0, batch, ent_off, first, num, max_blocks, codes, scale, st, stream)
    ok_args = [_p(), 1, 64, _p(), nul, 1, _p(), nul, nul, 4, _p(), _p(), nul, nul]

    def call(**kw):
        a = list(ok_args)
        for i, v in kw.items():
            a[int(i[1:])] = v
        return lib.lindex_pool_keys(*a)

    assert call(a0=nul) == _lib.ERR_INVALID_ARG              # no rows
    assert call(a10=nul) == _lib.ERR_INVALID_ARG             # no output codes
    assert call(a11=nul) == _lib.ERR_INVALID_ARG             # no output scales
    assert call(a1=2) == _lib.ERR_UNSUPPORTED                # fp8 per-token keys
    assert call(a1=9) == _lib.ERR_INVALID_ARG                # bad dtype enum
    assert call(a2=96) == _lib.ERR_UNSUPPORTED               # key width not implemented
    assert call(a2=0) == _lib.ERR_INVALID_ARG
    assert call(a0=_p(0x1008)) == _lib.ERR_INVALID_ARG       # rows not 16-byte aligned
    assert call(a10=_p(0x1004)) == _lib.ERR_INVALID_ARG      # codes not 16-byte aligned
    assert call(a11=_p(0x1002)) == _lib.ERR_INVALID_ARG      # scales not 4-byte aligned
    assert call(a5=0) == _lib.ERR_INVALID_ARG                # empty batch
    assert call(a9=-1) == _lib.ERR_INVALID_ARG
    assert call(a9=0) == _lib.OK                             # nothing to do, nothing launched


def test_indexer_workspace_sizes(lib):
    # many queries: the tensor-core path's candidate lists on top of the scan's workspace;
    # few queries: the scan's alone
    scan = lib.lindex_workspace_size_scan(4096, 33792)  # (0 without a GPU: sized from the device)
    full = lib.lindex_workspace_size(4096, 1024, 33792)
    assert 0 <= scan < full
    assert full >= 4096 * 8192 * 8  # two [T, cap] lists, cap = max(8192, 2k) capped by the entries
    assert lib.lindex_workspace_size(255, 1024, 33792) == lib.lindex_workspace_size_scan(255, 33792)
    # a short cache caps the lists at its entry count
    assert lib.lindex_workspace_size(300, 1024, 2000) < lib.lindex_workspace_size(300, 1024, 20000)
