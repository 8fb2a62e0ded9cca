"""The compression epilogues and kernel shapes, through the C ABI, against the oracle:

* both kernel shapes (warp per entry for a few entries, the TMA-ring kernel for many) give
  the oracle's entries on the same calls, ragged sequences, partial blocks, provided tails;
* RMSNorm of each entry's K and V halves ([SW] §十四.3) against oracle.norm.norm_packed_rows;
* the per-token indexer keys pooled inside csa_compress ([TR] §4.2): bit for bit the same as
  lindex_pool_keys, and within the fp32 error band of the exact fp64 definition;
* missing tail rows are flagged and not read by the TMA-ring kernels either."""

import numpy as np
import pytest
import torch

from compressed_sparse_kv_compress_b200 import api
from oracle import codecs, compress, norm

from helpers import check_pooled_keys, compress_tol_check, storage_rows

pytestmark = pytest.mark.gpu

CSA_BULK_MIN, HCA_BULK_MIN = 512, 128  # the host switches to the TMA-ring kernels at these bounds


def _i64(v):
    return torch.tensor(np.asarray(v, dtype=np.int64), dtype=torch.int64, device="cuda")


def _rows(rng, n, width, dtype, scale):
    x = torch.from_numpy((rng.standard_normal((n, width)) * scale).astype(np.float32))
    return x.to(torch.bfloat16) if dtype == "bf16" else x


def _dec(t):
    return storage_rows(t.cpu())


class Case:
    """Ragged sequences with provided tails (tok0) and partial last blocks; per-token rows of
    the CSA layer (x_a, z_a, x_b, z_b, indexer keys) and of the HCA layer (x, z)."""

    def __init__(self, seed, lengths, tails, dtype, Di=64, biases=False):
        rng = np.random.default_rng(seed)
        self.n, self.t0, self.dtype, self.Di = list(lengths), list(tails), dtype, Di
        B = len(lengths)
        rows = [n - t for n, t in zip(lengths, tails)]
        self.tok_off = np.concatenate([[0], np.cumsum(rows)])
        self.csa_n = [(n + 3) // 4 for n in lengths]
        self.hca_n = [(n + 127) // 128 for n in lengths]
        self.csa_off = np.concatenate([[0], np.cumsum(self.csa_n)])
        self.hca_off = np.concatenate([[0], np.cumsum(self.hca_n)])
        # entries whose tokens (and, for CSA, the previous block's) lie in the provided tail
        self.csa_first = [0 if t == 0 else t // 4 + 1 for t in tails]
        self.hca_first = [(t + 127) // 128 for t in tails]
        R = int(self.tok_off[-1])
        s = 128 ** -0.5
        self.cpu = {k: _rows(rng, R, 256, dtype, sc) for k, sc in
                    (("x_a", s), ("z_a", 1.0), ("x_b", s), ("z_b", 1.0), ("x_h", s), ("z_h", 1.0))}
        self.cpu["k_tok"] = _rows(rng, R, Di, dtype, Di ** -0.5)
        self.bias = None
        if biases:
            self.bias = {"a": torch.from_numpy(rng.standard_normal((4, 256)).astype(np.float32)),
                         "b": torch.from_numpy(rng.standard_normal((4, 256)).astype(np.float32)),
                         "h": torch.from_numpy(rng.standard_normal((128, 256)).astype(np.float32))}
        self.gamma = torch.from_numpy(rng.uniform(0.5, 1.5, 256).astype(np.float32))
        self.dev = {k: v.cuda() for k, v in self.cpu.items()}
        self.B = B

    def seq_rows(self, key, b):
        return codecs.decode(self._np(key)[self.tok_off[b]:self.tok_off[b + 1]], self.dtype)

    def _np(self, key):
        t = self.cpu[key]
        return t.view(torch.int16).numpy().view(np.uint16) if t.dtype == torch.bfloat16 else t.numpy()

    def bias_np(self, k):
        return None if self.bias is None else self.bias[k].numpy().astype(np.float64)

    def bias_dev(self, k):
        return None if self.bias is None else self.bias[k].cuda()


def _csa_call(c, out, max_blocks, *, rmsnorm=False, pool=False, codes=None, scales=None, status=None,
              first=None, num=None):
    first = c.csa_first if first is None else first
    num = [c.csa_n[b] - first[b] for b in range(c.B)] if num is None else num
    api.csa_compress(c.dev["x_a"], c.dev["z_a"], c.dev["x_b"], c.dev["z_b"], _i64(c.tok_off), _i64(c.csa_off), out,
                     max_blocks=max_blocks, bias_a=c.bias_dev("a"), bias_b=c.bias_dev("b"), tok0=_i64(c.t0),
                     first_block=_i64(first), num_blocks=_i64(num), rmsnorm=rmsnorm,
                     norm_gamma=c.gamma.cuda() if rmsnorm else None, norm_eps=1e-6,
                     k_tok=c.dev["k_tok"] if pool else None, k_codes=codes, k_scale=scales, dev_status=status)
    return first, num


def _csa_ref(c, b, first, num, rmsnorm):
    ents = np.arange(first[b], first[b] + num[b])
    ref = compress.csa_compress(ents, c.n[b], c.seq_rows("x_a", b), c.seq_rows("z_a", b), c.seq_rows("x_b", b),
                                c.seq_rows("z_b", b), c.bias_np("a"), c.bias_np("b"), tok0=c.t0[b])
    if rmsnorm:
        g = c.gamma.numpy().astype(np.float64)
        ref = norm.norm_packed_rows(ref, g[:128], g[128:], 1e-6)
    return ents, ref


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("rmsnorm", [False, True])
def test_csa_both_shapes_with_and_without_rmsnorm(dtype, rmsnorm):
    c = Case(1 + (dtype == "f32") + 2 * rmsnorm, lengths=[1999, 1026, 301], tails=[0, 412, 0], dtype=dtype,
             biases=True)
    torch_dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    for max_blocks in (max(c.csa_n), CSA_BULK_MIN):  # warp per entry, then the TMA-ring kernel
        out = torch.full((int(c.csa_off[-1]), 256), float("nan"), dtype=torch_dt, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        first, num = _csa_call(c, out, max_blocks, rmsnorm=rmsnorm, status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        got = _dec(out)
        for b in range(c.B):
            ents, ref = _csa_ref(c, b, first, num, rmsnorm)
            compress_tol_check(got[c.csa_off[b] + ents], ref, dtype, f"max_blocks {max_blocks} seq{b}")
            # entries before the tail's first complete pair were not asked for: untouched
            assert np.all(np.isnan(got[c.csa_off[b]:c.csa_off[b] + first[b]]))
        if rmsnorm:  # unit RMS times the gains, per half
            g = c.gamma.numpy().astype(np.float64)
            rows = got[c.csa_off[0] + first[0]: c.csa_off[0] + first[0] + 50]
            for h in (slice(0, 128), slice(128, 256)):
                rms = np.sqrt(np.mean((rows[:, h] / g[h]) ** 2, axis=1))
                assert np.allclose(rms, 1.0, rtol=2e-2)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_hca_both_shapes_and_rmsnorm(dtype):
    c = Case(7 + (dtype == "f32"), lengths=[15000, 4097, 129], tails=[0, 1280, 0], dtype=dtype, biases=True)
    torch_dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    first = c.hca_first
    num = [c.hca_n[b] - first[b] for b in range(c.B)]
    g = c.gamma.numpy().astype(np.float64)
    for max_blocks, rmsnorm in ((max(c.hca_n), False), (HCA_BULK_MIN, False), (max(c.hca_n), True)):
        out = torch.full((int(c.hca_off[-1]), 256), float("nan"), dtype=torch_dt, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        api.hca_compress(c.dev["x_h"], c.dev["z_h"], _i64(c.tok_off), _i64(c.hca_off), out, max_blocks=max_blocks,
                         bias=c.bias_dev("h"), tok0=_i64(c.t0), first_block=_i64(first), num_blocks=_i64(num),
                         rmsnorm=rmsnorm, norm_gamma=c.gamma.cuda() if rmsnorm else None, norm_eps=1e-6,
                         dev_status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        got = _dec(out)
        for b in range(c.B):
            ents = np.arange(first[b], first[b] + num[b])
            ref = compress.hca_compress(ents, c.n[b], c.seq_rows("x_h", b), c.seq_rows("z_h", b), c.bias_np("h"),
                                        tok0=c.t0[b])
            if rmsnorm:
                ref = norm.norm_packed_rows(ref, g[:128], g[128:], 1e-6)
            compress_tol_check(got[c.hca_off[b] + ents], ref, dtype, f"max_blocks {max_blocks} norm {rmsnorm} seq{b}")


@pytest.mark.parametrize("Di", [64, 128])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_csa_fused_key_pooling(Di, dtype):
    c = Case(11 + Di + (dtype == "f32"), lengths=[1999, 1026, 301], tails=[0, 412, 0], dtype=dtype, Di=Di)
    torch_dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    V = int(c.csa_off[-1])
    # the separate pooling call is the reference for the codes (the same fp32 steps)
    ref_codes = torch.full((V, Di), 0xAA, dtype=torch.uint8, device="cuda")
    ref_scale = torch.full((V,), -1.0, dtype=torch.float32, device="cuda")
    first = c.csa_first
    num = [c.csa_n[b] - first[b] for b in range(c.B)]
    api.lindex_pool_keys(c.dev["k_tok"], _i64(c.tok_off), _i64(c.csa_off), ref_codes, ref_scale,
                         max_blocks=max(num), tok0=_i64(c.t0), first_block=_i64(first), num_blocks=_i64(num))
    for max_blocks in (max(c.csa_n), CSA_BULK_MIN):
        out = torch.empty(V, 256, dtype=torch_dt, device="cuda")
        codes = torch.full((V, Di), 0xAA, dtype=torch.uint8, device="cuda")
        scales = torch.full((V,), -1.0, dtype=torch.float32, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        _csa_call(c, out, max_blocks, pool=True, codes=codes, scales=scales, status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        assert torch.equal(codes, ref_codes) and torch.equal(scales, ref_scale), f"max_blocks {max_blocks}"
        cn, sn = codes.cpu().numpy(), scales.cpu().numpy()
        for b in range(c.B):
            e0 = c.csa_off[b] + first[b]
            tok = c.seq_rows("k_tok", b)[4 * first[b] - c.t0[b]:]
            check_pooled_keys(cn[e0:e0 + num[b]], sn[e0:e0 + num[b]], tok, 4, what=f"seq{b}")
        # the entries themselves are unchanged by the extra epilogue
        got = _dec(out)
        for b in range(c.B):
            ents, ref = _csa_ref(c, b, first, num, False)
            compress_tol_check(got[c.csa_off[b] + ents], ref, dtype, f"seq{b}")


def test_bulk_kernels_flag_missing_tail_rows():
    c = Case(21, lengths=[3000], tails=[800], dtype="bf16")
    out_c = torch.zeros(int(c.csa_off[-1]), 256, dtype=torch.bfloat16, device="cuda")
    out_h = torch.zeros(int(c.hca_off[-1]), 256, dtype=torch.bfloat16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    # CSA entries 150..249: tokens 596.. lie before the tail (token 800)
    _csa_call(c, out_c, CSA_BULK_MIN, first=[150], num=[100], status=st)
    # HCA entries 5..9: entry 5 starts at token 640, before the tail
    api.hca_compress(c.dev["x_h"], c.dev["z_h"], _i64(c.tok_off), _i64(c.hca_off), out_h, max_blocks=HCA_BULK_MIN,
                     tok0=_i64(c.t0), first_block=_i64([5]), num_blocks=_i64([5]), dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & 2  # CSKV_DEV_TAIL_MISSING
    got_c, got_h = _dec(out_c), _dec(out_h)
    # entries with missing rows stay untouched; the ones after them are computed
    assert np.all(got_c[150:201] == 0) and np.all(got_h[5:7] == 0)
    ents, ref = _csa_ref(c, 0, [201], [49], False)
    compress_tol_check(got_c[ents], ref, "bf16", "csa after the gap")
    ents = np.arange(7, 10)
    ref = compress.hca_compress(ents, c.n[0], c.seq_rows("x_h", 0), c.seq_rows("z_h", 0), None, tok0=c.t0[0])
    compress_tol_check(got_h[ents], ref, "bf16", "hca after the gap")


def test_bulk_capacity_flag():
    c = Case(22, lengths=[4000], tails=[0], dtype="bf16")
    out = torch.zeros(int(c.csa_off[-1]), 256, dtype=torch.bfloat16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    _csa_call(c, out, CSA_BULK_MIN, first=[0], num=[1000], status=st)  # 1000 > the bound 512
    torch.cuda.synchronize()
    assert int(st.item()) & 4
    got = _dec(out)
    ents, ref = _csa_ref(c, 0, [0], [CSA_BULK_MIN], False)
    compress_tol_check(got[ents], ref, "bf16", "entries within the bound")
    assert np.all(got[CSA_BULK_MIN:] == 0)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_rmsnorm_heads_query_side(dtype):
    # the query-side pass: every 128-dimension head vector, gains and eps, in place and not
    rng = np.random.default_rng(31)
    q = torch.from_numpy((rng.standard_normal((37, 16, 128)) / np.sqrt(128)).astype(np.float32))
    q[3, 5] = 0.0  # a zero head: stays zero
    q = q.to(torch.bfloat16) if dtype == "bf16" else q
    gamma = torch.from_numpy(rng.uniform(0.5, 1.5, 128).astype(np.float32))
    ref = norm.rmsnorm(storage_rows(q.reshape(-1, 128)), gamma.numpy().astype(np.float64), 1e-6)
    out = torch.empty_like(q).cuda()
    qd = q.cuda()
    api.rmsnorm_heads(qd, out, gamma=gamma.cuda(), eps=1e-6)
    torch.cuda.synchronize()
    compress_tol_check(storage_rows(out.cpu().reshape(-1, 128)), ref, dtype, "rmsnorm_heads")
    assert torch.all(out[3, 5] == 0)
    api.rmsnorm_heads(qd, gamma=gamma.cuda(), eps=1e-6)  # in place
    torch.cuda.synchronize()
    assert torch.equal(qd, out)
