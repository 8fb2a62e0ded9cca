"""Torch-tensor front end of the cskv C ABI: argument marshalling only.

Every function here turns tensors into pointers, sizes and dtype codes and
calls the C entry point of the same name on the current CUDA stream (or the
one given).  All computation happens in the CUDA library.
"""

from __future__ import annotations

import ctypes
import math

import torch

from . import _lib
from ._lib import ATTN_KV_FP8, ATTN_PAIRS, BF16, CSA, F32, FP8E4M3, HCA, KV8_ROW_BYTES, OVERLAP_PREVIOUS  # noqa: F401

_DT = {torch.float32: F32, torch.bfloat16: BF16, torch.uint8: FP8E4M3, torch.float8_e4m3fn: FP8E4M3}


def _ptr(t):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("cskv expects contiguous tensors")
    return t.data_ptr()


def _dt(t) -> int:
    try:
        return _DT[t.dtype]
    except KeyError:
        raise ValueError(f"unsupported dtype {t.dtype}") from None


def _stream(stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def csa_compress(x_a, z_a, x_b, z_b, tok_off, ent_off, out, *, max_blocks, bias_a=None, bias_b=None, tok0=None,
                 first_block=None, num_blocks=None, rmsnorm=False, norm_gamma=None, norm_eps=1e-6, k_tok=None,
                 k_codes=None, k_scale=None, overlap_previous=False, dev_status=None, stream=None):
    """rmsnorm: normalise each entry's K and V halves (norm_gamma [256] fp32, K then V; None =
    ones).  k_tok [rows, Di] (rows indexed like x_a): also pool the per-token indexer keys of
    the same entries into k_codes [*, Di] uint8 (E4M3) and k_scale [*] fp32.
    overlap_previous: CSKV_OVERLAP_PREVIOUS (the kernel issued just before this call on the
    stream neither writes its inputs nor reads its outputs; see the C header)."""
    lib = _lib.load()
    k_dt = _dt(k_tok) if k_tok is not None else F32
    Di = int(k_tok.shape[-1]) if k_tok is not None else 0
    st = lib.csa_compress(_ptr(x_a), _ptr(z_a), _ptr(x_b), _ptr(z_b), _ptr(bias_a), _ptr(bias_b), _ptr(tok_off),
                          _ptr(tok0), tok_off.numel() - 1, _ptr(ent_off), _ptr(first_block), _ptr(num_blocks),
                          int(max_blocks), _dt(x_a), _dt(out), _ptr(out), int(bool(rmsnorm)), _ptr(norm_gamma),
                          float(norm_eps), _ptr(k_tok), k_dt, Di, _ptr(k_codes), _ptr(k_scale),
                          OVERLAP_PREVIOUS if overlap_previous else 0, _ptr(dev_status), _stream(stream))
    _lib.check("csa_compress", st)
    return out


def hca_compress(x, z, tok_off, ent_off, out, *, max_blocks, bias=None, tok0=None, first_block=None,
                 num_blocks=None, rmsnorm=False, norm_gamma=None, norm_eps=1e-6, dev_status=None, stream=None):
    lib = _lib.load()
    st = lib.hca_compress(_ptr(x), _ptr(z), _ptr(bias), _ptr(tok_off), _ptr(tok0), tok_off.numel() - 1,
                          _ptr(ent_off), _ptr(first_block), _ptr(num_blocks), int(max_blocks), _dt(x), _dt(out),
                          _ptr(out), int(bool(rmsnorm)), _ptr(norm_gamma), float(norm_eps), _ptr(dev_status),
                          _stream(stream))
    _lib.check("hca_compress", st)
    return out


def rmsnorm_heads(x, out=None, *, gamma=None, eps=1e-6, stream=None):
    """RMSNorm of every 128-dimension row of x ([..., 128], fp32 or bf16) into out (default:
    in place): x / sqrt(mean(x^2) + eps) * gamma."""
    out = x if out is None else out
    lib = _lib.load()
    st = lib.rmsnorm_heads(_ptr(x), _dt(x), x.numel() // x.shape[-1], int(x.shape[-1]), _ptr(gamma), float(eps),
                           _ptr(out), _stream(stream))
    _lib.check("rmsnorm_heads", st)
    return out


def lindex_pool_keys(k_tok, tok_off, ent_off, out_codes, out_scale, *, max_blocks, tok0=None, first_block=None,
                     num_blocks=None, dev_status=None, stream=None):
    """Entry keys of the indexer from per-token keys k_tok [rows, Di] (fp32 or bf16): the mean
    of each 4-token block as E4M3 codes (out_codes [*, Di] uint8) with one fp32 scale per
    entry (out_scale [*])."""
    lib = _lib.load()
    st = lib.lindex_pool_keys(_ptr(k_tok), _dt(k_tok), int(k_tok.shape[-1]), _ptr(tok_off), _ptr(tok0),
                              tok_off.numel() - 1, _ptr(ent_off), _ptr(first_block), _ptr(num_blocks),
                              int(max_blocks), _ptr(out_codes), _ptr(out_scale), _ptr(dev_status), _stream(stream))
    _lib.check("lindex_pool_keys", st)
    return out_codes, out_scale


def lindex_workspace_size(T: int, k: int, max_entries: int) -> int:
    return int(_lib.load().lindex_workspace_size(int(T), int(k), int(max_entries)))


def lindex_workspace_size_scan(T: int, max_entries: int) -> int:
    return int(_lib.load().lindex_workspace_size_scan(int(T), int(max_entries)))


def lindex_workspace(T: int, k: int, max_entries: int, device="cuda", scan_only=False) -> torch.Tensor:
    """A zero-filled workspace; calls hand it back zero-filled.  scan_only: the per-query scan's
    size (many-query calls then skip the tensor-core path)."""
    n = lindex_workspace_size_scan(T, max_entries) if scan_only else lindex_workspace_size(T, k, max_entries)
    return torch.zeros(max(16, n), dtype=torch.uint8, device=device)


def lindex_score_topk(q_idx, k_idx, q_seq, q_pos, ent_off, out_idx, workspace, *, max_entries, q_scale=None,
                      k_scale=None, head_w=None, out_score=None, prefetch_rows=None, dev_status=None, stream=None):
    """prefetch_rows: optional [entries, ...] tensor indexed like k_idx (e.g. the compressed
    CSA cache); the rows of the kept entries are prefetched into L2 (a hint)."""
    T, Hi, Di = q_idx.shape
    lib = _lib.load()
    pf_bytes = 0 if prefetch_rows is None else prefetch_rows[0].numel() * prefetch_rows.element_size()
    st = lib.lindex_score_topk(_ptr(q_idx), _ptr(q_scale), _ptr(k_idx), _ptr(k_scale), _ptr(head_w), _ptr(q_seq),
                               _ptr(q_pos), _ptr(ent_off), ent_off.numel() - 1, T, Hi, Di, out_idx.shape[1],
                               _dt(q_idx), int(max_entries), _ptr(out_idx), _ptr(out_score), _ptr(prefetch_rows),
                               pf_bytes, _ptr(workspace), workspace.numel() * workspace.element_size(),
                               _ptr(dev_status), _stream(stream))
    _lib.check("lindex_score_topk", st)
    return out_idx


def lindex_score_topk_mxfp4(q_codes, q_bscale, k_codes, k_bscale, q_seq, q_pos, ent_off, out_idx, workspace, *,
                            max_entries, q_scale=None, head_w=None, out_score=None, prefetch_rows=None,
                            dev_status=None, stream=None):
    """MXFP4 indexer vectors: q_codes [T, Hi, Di/2] / k_codes [Nc, Di/2] uint8 (two E2M1 codes a
    byte) with E8M0 block scales q_bscale [T, Hi, Di/32] / k_bscale [Nc, Di/32] uint8."""
    T, Hi, half = q_codes.shape
    lib = _lib.load()
    pf_bytes = 0 if prefetch_rows is None else prefetch_rows[0].numel() * prefetch_rows.element_size()
    st = lib.lindex_score_topk_mxfp4(_ptr(q_codes), _ptr(q_bscale), _ptr(q_scale), _ptr(k_codes), _ptr(k_bscale),
                                     _ptr(head_w), _ptr(q_seq), _ptr(q_pos), _ptr(ent_off), ent_off.numel() - 1, T,
                                     Hi, 2 * half, out_idx.shape[1], int(max_entries), _ptr(out_idx),
                                     _ptr(out_score), _ptr(prefetch_rows), pf_bytes, _ptr(workspace),
                                     workspace.numel() * workspace.element_size(), _ptr(dev_status),
                                     _stream(stream))
    _lib.check("lindex_score_topk_mxfp4", st)
    return out_idx


def lindex_topk_from_scores(scores, n_valid, out_idx, workspace, *, max_entries, out_score=None, dev_status=None,
                            stream=None):
    T, ld = scores.shape
    lib = _lib.load()
    st = lib.lindex_topk_from_scores(_ptr(scores), ld, _ptr(n_valid), T, out_idx.shape[1], int(max_entries),
                                     _ptr(out_idx), _ptr(out_score), _ptr(workspace),
                                     workspace.numel() * workspace.element_size(), _ptr(dev_status),
                                     _stream(stream))
    _lib.check("lindex_topk_from_scores", st)
    return out_idx


def attn_workspace_size(mode: int, T: int, H: int, k: int, window: int, max_entries: int) -> int:
    return int(_lib.load().hybrid_attn_workspace_size(int(mode), int(T), int(H), 128, int(k), int(window),
                                                      int(max_entries)))


def attn_workspace(mode, T, H, k, window, max_entries, device="cuda") -> torch.Tensor:
    n = attn_workspace_size(mode, T, H, k, window, max_entries)
    return torch.empty(max(16, n), dtype=torch.uint8, device=device)


def hybrid_decode_attn(mode, q, kv_cmp, cmp_off, kv_raw, raw_off, q_seq, q_pos, out, workspace, *, window,
                       idx=None, raw_tok0=None, sink=None, scale=None, lse=None, max_entries=0, adjacent_pairs=False,
                       kv_fp8=False, dev_status=None, stream=None):
    """adjacent_pairs: CSKV_ATTN_PAIRS (queries 2j, 2j + 1 are one sequence's consecutive
    positions; see the C header).  kv_fp8: CSKV_ATTN_KV_FP8, kv_cmp holds FP8 main-KV rows
    ([entries, 336] uint8, from kv_quantize_fp8)."""
    T, H, d = q.shape
    if adjacent_pairs:
        mode = int(mode) | ATTN_PAIRS
    if kv_fp8:
        mode = int(mode) | ATTN_KV_FP8
    k = idx.shape[1] if idx is not None else 0
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    lib = _lib.load()
    st = lib.hybrid_decode_attn(int(mode), _ptr(q), _ptr(kv_cmp), _ptr(cmp_off), _ptr(idx), k, _ptr(kv_raw),
                                _ptr(raw_off), _ptr(raw_tok0), int(window), _ptr(sink), scale, _ptr(q_seq),
                                _ptr(q_pos), cmp_off.numel() - 1, T, H, d, _dt(q), int(max_entries), _ptr(out),
                                _ptr(lse), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                _ptr(dev_status), _stream(stream))
    _lib.check("hybrid_decode_attn", st)
    return out


def copy_segments(src, src_off, dst_ptrs, lens, stream=None):
    """Scatter segments of the byte buffer `src` (int64 device arrays src_off, lens and
    dst_ptrs = destination addresses) with one kernel: the unpacking half of a staged
    host-to-device copy of a step's new inputs, or a read-back into host memory.  `src` is a
    device tensor or an address from mapped_pointer(); host destinations in dst_ptrs must be
    mapped_pointer() addresses too."""
    lib = _lib.load()
    src_p = src if isinstance(src, int) else _ptr(src)
    st = lib.cskv_copy_segments(src_p, _ptr(src_off), _ptr(dst_ptrs), _ptr(lens), int(src_off.numel()),
                                _stream(stream))
    _lib.check("cskv_copy_segments", st)


def kv_quantize_fp8(rows, out=None, stream=None):
    """FP8 main-KV rows ([n, 336] uint8) from K||V rows [n, 256] (fp32 or bf16, device)."""
    assert rows.dim() == 2 and rows.shape[1] == 256
    n = rows.shape[0]
    if out is None:
        out = torch.empty(n, KV8_ROW_BYTES, dtype=torch.uint8, device=rows.device)
    lib = _lib.load()
    st = lib.kv_quantize_fp8(_ptr(rows), _dt(rows), n, _ptr(out), _stream(stream))
    _lib.check("kv_quantize_fp8", st)
    return out


def mapped_pointer(t) -> int:
    """The address at which the current device reaches tensor `t`'s data: its own address for
    device memory, the mapped address for page-locked host memory.  Raises for pageable host
    memory, which the device cannot address."""
    lib = _lib.load()
    out = ctypes.c_void_p()
    st = lib.cskv_mapped_pointer(_ptr(t), ctypes.byref(out))
    _lib.check("cskv_mapped_pointer", st)
    return int(out.value)
