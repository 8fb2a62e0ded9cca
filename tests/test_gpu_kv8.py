"""FP8 main-KV rows ([SW] §十三.4): kv_quantize_fp8 against the exact fp64 quantiser of
oracle/kv8.py (codes equal outside the fp32 error band around an E4M3 rounding boundary, the
neighbouring code allowed inside it; scales within one fp32 rounding; the bf16 RoPE dims and
the padding bit-exact), and hybrid_decode_attn over such rows (CSKV_ATTN_KV_FP8) against the
oracle's attention over the same rows decoded exactly (bf16 queries on the tensor-core
kernel, which decodes the rows to bf16 as it gathers them; fp32 on the CUDA cores)."""

import numpy as np
import pytest
import torch

from oracle import codecs, indexer, kv8
from oracle import step as ostep
from synth import Workload, spec_by_name

from compressed_sparse_kv_compress_b200 import api
from helpers import bounds, check_attention, dtypes, np_arrays, to_f64

pytestmark = pytest.mark.gpu


def _rows(rng, n, dtype):
    x = rng.standard_normal((n, 256)) * np.exp(rng.uniform(-8, 8, (n, 1)))
    x[0] = 0.0                       # all-zero row: both scales 1
    x[1, :64] = 0.0                  # K group zero only
    x[2, 128:] = 0.0                 # V group zero only
    x[3, 7] = 448.0 * 2.0 ** -3      # amax exactly 448 x a power of two
    x[4, :] = 1e-3                   # ties: every value equal to amax
    t = torch.from_numpy(x.astype(np.float32))
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def _f64(t):
    if t.dtype == torch.bfloat16:
        return codecs.bf16_decode(t.view(torch.int16).numpy().view(np.uint16))
    return t.numpy().astype(np.float64)


def _check_group(codes_gpu, q64, tol, codes64, what):
    lo = codecs.e4m3_decode(codecs.e4m3_encode(q64 - tol))
    hi = codecs.e4m3_decode(codecs.e4m3_encode(q64 + tol))
    got = codecs.e4m3_decode(codes_gpu)
    sure = lo == hi
    off = sure & (got != codecs.e4m3_decode(codes64))
    assert not off.any(), f"{what}: {int(off.sum())} codes differ outside the band"
    assert np.all((got >= lo) & (got <= hi)), f"{what}: codes outside the band"
    return int((~sure).sum())


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_quantiser_matches_exact_definition(dtype):
    rng = np.random.default_rng(21 + (dtype == "bf16"))
    rows = _rows(rng, 2053, dtype)   # 256 full CTAs of 8 rows and a ragged tail
    out = api.kv_quantize_fp8(rows.cuda())
    torch.cuda.synchronize()
    b = out.cpu().numpy()
    assert b.shape == (2053, kv8.ROW_BYTES)
    x = _f64(rows)
    kc, rope, vc, s_k, s_v = kv8.quantize_rows_f64(x)
    tk, tv, ts = kv8.quotient_error_bound(x)
    sc = b[:, 320:328].copy().view("<f4").reshape(-1, 2).astype(np.float64)
    assert np.all(np.abs(sc[:, 0] - s_k) <= ts[:, 0]) and np.all(np.abs(sc[:, 1] - s_v) <= ts[:, 1])
    assert sc[0, 0] == 1.0 and sc[0, 1] == 1.0 and sc[1, 0] == 1.0 and sc[2, 1] == 1.0
    ref = kv8.pack_rows(kc, rope, vc, s_k.astype(np.float32), s_v.astype(np.float32))
    assert np.array_equal(b[:, 64:192], ref[:, 64:192]), "RoPE dims"
    assert np.all(b[:, 328:] == 0), "padding"
    band = _check_group(b[:, :64], x[:, :64] / s_k[:, None], tk, kc, "K")
    band += _check_group(b[:, 192:320], x[:, 128:] / s_v[:, None], tv, vc, "V")
    # bf16 rows carry 8 significant bits, so many quotients sit exactly on an E4M3 tie, where
    # either neighbour is within one fp32 rounding: about 0.4 % of the elements here
    assert band < 0.01 * x.size
    # ties: every value of row 4 equals its group's amax -> code 448 (0x7E) everywhere
    assert np.all(b[4, :64] == 0x7E) and np.all(b[4, 192:320] == 0x7E)


def test_quantiser_argument_checks():
    from compressed_sparse_kv_compress_b200 import _lib
    lib = _lib.load()
    x = torch.zeros(4, 256, device="cuda")
    o = torch.zeros(4, 336, dtype=torch.uint8, device="cuda")
    assert lib.kv_quantize_fp8(x.data_ptr(), _lib.F32, -1, o.data_ptr(), None) == _lib.ERR_INVALID_ARG
    assert lib.kv_quantize_fp8(x.data_ptr(), _lib.FP8E4M3, 4, o.data_ptr(), None) == _lib.ERR_UNSUPPORTED
    assert lib.kv_quantize_fp8(x.data_ptr() + 4, _lib.F32, 4, o.data_ptr(), None) == _lib.ERR_INVALID_ARG
    assert lib.kv_quantize_fp8(None, _lib.F32, 0, None, None) == _lib.OK


def _oracle_rows(w, a):
    m = w.meta
    rows = np.full((m["T"], m["k"]), -1, np.int64)
    for t in range(m["T"]):
        rows[t] = indexer.topk_select(ostep.query_scores(m, a, dtypes(w), t), m["k"])
    return rows


def _attend_fp8(w, dev, mode, cache8, idx=None, pairs=False):
    m = w.meta
    b = bounds(w)
    T, H = m["T"], m["H"]
    layer = "c" if mode == api.CSA else "h"
    off = dev["csa_off"] if mode == api.CSA else dev["hca_off"]
    ws = api.attn_workspace(mode, T, H, m["k"], m["W"], b["max_hca_visible"])
    out = torch.empty(T, H, 128, dtype=torch.float32, device="cuda")
    lse = torch.empty(T, H, dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.hybrid_decode_attn(mode, dev["q_" + layer], cache8, off, dev["raw_" + layer], dev["raw_off"], dev["q_seq"],
                           dev["q_pos"], out, ws, window=m["W"], idx=idx, raw_tok0=dev["raw_t0"],
                           sink=dev["sink_" + layer], scale=m["scale"], lse=lse, max_entries=b["max_hca_visible"],
                           adjacent_pairs=pairs, kv_fp8=True, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return to_f64(out), to_f64(lse)


@pytest.mark.parametrize("case", ["tiny_f32", "bf16_h64", "bf16_h128"])
@pytest.mark.parametrize("mode", ["csa", "hca"])
@pytest.mark.parametrize("quantiser", ["oracle", "gpu"])
def test_attention_over_fp8_rows(case, mode, quantiser):
    if case == "tiny_f32":
        spec = spec_by_name("tiny").replace(cache="random")
    else:
        spec = spec_by_name("b8_ctx64k").replace(batch=3, seq_len=(30001, 2000, 300),
                                                 heads=64 if case == "bf16_h64" else 128)
    w = Workload(spec)
    a = np_arrays(w)
    dev = w.device("cuda")
    m = w.meta
    md = api.CSA if mode == "csa" else api.HCA
    layer = "c" if md == api.CSA else "h"
    plain = codecs.decode(a["cmp_" + layer], dtypes(w)["kv"])
    if quantiser == "oracle":
        b8 = kv8.quantize_to_storage_f64(plain)
        cache8 = torch.from_numpy(b8).cuda()
    else:
        cache8 = api.kv_quantize_fp8(dev["cmp_" + layer])
        b8 = cache8.cpu().numpy()
    dec = kv8.decode_rows(b8)
    rows = _oracle_rows(w, a) if md == api.CSA else None
    idx = None if rows is None else torch.from_numpy(rows.astype(np.int32)).cuda()
    o, lse = _attend_fp8(w, dev, md, cache8, idx)
    for t in range(m["T"]):
        if md == api.CSA:
            ent = rows[t][(rows[t] >= 0) & (rows[t] < indexer.visible_entries(m["q_pos"][t], 4))]
        else:
            ent = np.arange(indexer.visible_entries(m["q_pos"][t], 128))
        ro, rl, _ = ostep.query_attention(m, a, dtypes(w), dec, t, layer, ent, cmp_decoded=True)
        check_attention(o[t], ro, 1e-4 if case == "tiny_f32" else None, f"{case} {mode} query {t}")
        fin = np.isfinite(rl)
        assert np.allclose(lse[t][fin], rl[fin], rtol=1e-5, atol=1e-5)


def test_hca_adjacent_pairs_over_fp8_rows():
    # the tensor-core HCA kernel taking adjacent queries in pairs (one pass over the union of
    # their rows) over an FP8 cache; positions straddle 128-token block boundaries
    spec = spec_by_name("prefill_4k_at_128k").replace(seq_len=(20096 + 10,), queries_per_seq=34, heads=64)
    w = Workload(spec)
    a = np_arrays(w)
    dev = w.device("cuda")
    m = w.meta
    cache8 = api.kv_quantize_fp8(dev["cmp_h"])
    dec = kv8.decode_rows(cache8.cpu().numpy())
    o, lse = _attend_fp8(w, dev, api.HCA, cache8, pairs=True)
    for t in range(m["T"]):
        ent = np.arange(indexer.visible_entries(m["q_pos"][t], 128))
        ro, rl, _ = ostep.query_attention(m, a, dtypes(w), dec, t, "h", ent, cmp_decoded=True)
        check_attention(o[t], ro, None, f"pairs query {t}")
        fin = np.isfinite(rl)
        assert np.allclose(lse[t][fin], rl[fin], rtol=1e-5, atol=1e-5)
