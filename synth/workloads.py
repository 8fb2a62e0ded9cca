"""Named workloads and their seeded input tensors.

Every tensor is drawn on the CPU from numpy's PCG64, one stream per
(seed, tensor name, row chunk), so any chunk can be regenerated on its own
and the draw does not depend on the number of threads used.

Storage forms of the returned CPU tensors:
  * ``bf16`` rows   -> ``torch.bfloat16``
  * ``f32`` rows    -> ``torch.float32``
  * ``fp8`` indexer -> ``torch.uint8`` holding OCP E4M3 codes, plus a
    ``torch.float32`` scale per row (entry) or per (query, head).
The fp8 codes are produced by torch's own ``float8_e4m3fn`` cast; the
scale of a row is ``amax / 448`` (448 is the largest finite E4M3 value).

Layout (all row-major, sequences concatenated in order):
  * compressed caches ``cmp_c`` [sum ceil(n/4), 256] and ``cmp_h``
    [sum ceil(n/128), 256]; each row is K (cols 0..127) then V (128..255);
  * per-token compression rows ``x_a z_a x_b z_b`` (CSA layer) and
    ``x_h z_h`` (HCA layer) hold only the tail of every sequence that the
    step needs, starting at token ``csa_t0[b]`` / ``hca_t0[b]``;
  * raw window rows ``raw_c`` / ``raw_h`` hold the tail from ``raw_t0[b]``;
  * indexer keys ``k_idx`` [sum ceil(n/4), 64] with ``k_scale``;
  * queries ``q_c`` / ``q_h`` [T, H, 128], indexer queries ``q_idx``
    [T, Hi, 64] with ``q_scale`` [T, Hi];
  * with ``pool_keys``: per-token indexer keys ``k_tok`` [rows, 64] bf16 of the CSA
    tail rows (indexed like ``x_a``), from which the step pools its entries' keys.
"""

from __future__ import annotations

import dataclasses
import math
import zlib
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

ROW = 256          # packed K||V width
HEAD_DIM = 128
E4M3_MAX = 448.0
_CHUNK_ELEMS = 1 << 22


@dataclasses.dataclass(frozen=True)
class Spec:
    name: str
    batch: int
    seq_len: tuple = ()            # explicit per-sequence token counts n_b
    len_range: tuple = ()          # (lo, hi) inclusive: n_b ~ U[lo, hi]
    queries_per_seq: int = 1       # queries at the last Q positions of each sequence
    heads: int = 64
    idx_heads: int = 8
    idx_dim: int = 64
    topk: int = 1024
    window: int = 128
    dtype: str = "bf16"            # KV / query / compression-row storage: f32 | bf16
    idx_dtype: str = "fp8"         # indexer storage: f32 | fp8
    sink: str = "per_head"         # one | per_head | none
    biases: bool = False           # position biases ~N(0,1) instead of 0
    cache: str = "random"          # random: cache state drawn directly; compress: built from full rows
    needles: int = 0
    pool_keys: bool = False        # the step pools its entries' indexer keys from per-token keys (k_tok)
    seed: int = 0

    def replace(self, **kw) -> "Spec":
        return dataclasses.replace(self, **kw)


SPECS = {
    s.name: s
    for s in [
        # batch 1, 4096 tokens, 16 heads, fp32, indexer 4x64 fp32, top-64, one sink logit
        Spec("tiny", batch=1, seq_len=(4096,), heads=16, idx_heads=4, topk=64,
             dtype="f32", idx_dtype="f32", sink="one", cache="compress"),
        Spec("tiny_bias", batch=1, seq_len=(4096,), heads=16, idx_heads=4, topk=64,
             dtype="f32", idx_dtype="f32", sink="one", cache="compress", biases=True, seed=1),
        # batch 8 x 65536 tokens, 64 heads, bf16, indexer 8x64 fp8, top-1024
        Spec("b8_ctx64k", batch=8, seq_len=(65536,) * 8, heads=64),
        # batch 1 x 2^20 tokens, 128 heads, 16 planted needle entries
        Spec("b1_ctx1m", batch=1, seq_len=(1 << 20,), heads=128, needles=16),
        # 4096 new query tokens appended to a 131072-token cache, 64 heads
        Spec("prefill_4k_at_128k", batch=1, seq_len=(131072 + 4096,), queries_per_seq=4096, heads=64),
        # batch 64, n_b ~ U[32768, 262144], 64 heads
        Spec("ragged_b64", batch=64, len_range=(32768, 262144), heads=64),
    ]
}


def spec_by_name(name: str) -> Spec:
    return SPECS[name]


def _ceil_div(a: int, b: int) -> int:
    return -(-a // b)


def _stream(seed: int, tag: str, chunk: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, zlib.crc32(tag.encode()), chunk])))


def _normal(seed: int, tag: str, rows: int, cols: int, std: float) -> np.ndarray:
    """[rows, cols] float32 of N(0, std^2), drawn chunk by chunk in parallel."""
    out = np.empty((rows, cols), dtype=np.float32)
    if rows == 0 or cols == 0:
        return out
    crows = max(1, _CHUNK_ELEMS // cols)
    nchunks = _ceil_div(rows, crows)

    def fill(c: int) -> None:
        r0, r1 = c * crows, min(rows, (c + 1) * crows)
        blk = out[r0:r1]
        _stream(seed, tag, c).standard_normal(out=blk, dtype=np.float32)
        if std != 1.0:
            blk *= np.float32(std)

    if nchunks == 1:
        fill(0)
    else:
        with ThreadPoolExecutor(8) as ex:
            list(ex.map(fill, range(nchunks)))
    return out


def _to_storage(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(x)
    if dtype == "bf16":
        return t.to(torch.bfloat16)
    if dtype == "f32":
        return t.clone()
    raise ValueError(dtype)


def _quant_e4m3(x: np.ndarray) -> tuple[torch.Tensor, torch.Tensor]:
    """Per-row symmetric E4M3 codes (torch cast) and fp32 scales amax/448."""
    t = torch.from_numpy(x)
    amax = t.abs().amax(dim=-1, keepdim=True)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    codes = (t / scale).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.contiguous(), scale.squeeze(-1).contiguous()


def mxfp4_random(seed: int, tag: str, rows: int, di: int, exp_lo: int = 121, exp_hi: int = 126):
    """Random MXFP4 vectors: E2M1 codes drawn uniformly over all 16 codes, packed two per byte
    (element 2j in the low nibble), and E8M0 block exponents drawn uniformly in
    [exp_lo, exp_hi] (scales 2^-6 .. 2^-1), one per 32 elements.  Returns
    (codes uint8 [rows, di/2], scales uint8 [rows, di/32]) as torch tensors."""
    g = _stream(seed, tag, 0)
    nib = g.integers(0, 16, size=(rows, di), dtype=np.uint8)
    codes = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    scales = g.integers(exp_lo, exp_hi + 1, size=(rows, di // 32), dtype=np.uint8)
    return torch.from_numpy(codes), torch.from_numpy(scales)


class Workload:
    """Host-side tensors and sizes of one named workload.

    ``meta`` holds python ints / lists; ``arrays`` holds CPU tensors.  Query t
    belongs to sequence ``q_seq[t]`` and sits at position ``q_pos[t]``; the
    step compresses, for every sequence, the CSA and HCA entries that contain
    the positions of its queries (``csa_first/csa_num``, ``hca_first/hca_num``).
    """

    def __init__(self, spec: Spec):
        self.spec = spec
        s = spec
        if s.seq_len:
            n = [int(v) for v in s.seq_len]
            assert len(n) == s.batch
        else:
            lo, hi = s.len_range
            n = [int(v) for v in _stream(s.seed, "seq_len", 0).integers(lo, hi + 1, size=s.batch)]
        Q = s.queries_per_seq
        assert all(v >= Q for v in n)
        W = s.window
        ncsa = [_ceil_div(v, 4) for v in n]
        nhca = [_ceil_div(v, 128) for v in n]
        first = [v - Q for v in n]
        if s.cache == "compress":
            csa_t0 = [0] * s.batch
            hca_t0 = [0] * s.batch
        else:
            csa_t0 = [max(0, 4 * (f // 4 - 1)) for f in first]
            hca_t0 = [128 * (f // 128) for f in first]
        raw_t0 = [max(0, f - W + 1) for f in first]

        def offs(sizes):
            o = [0]
            for v in sizes:
                o.append(o[-1] + v)
            return o

        T = s.batch * Q
        self.meta = dict(
            n=n, B=s.batch, T=T, Q=Q, H=s.heads, d=HEAD_DIM, D=ROW, Hi=s.idx_heads, di=s.idx_dim,
            k=s.topk, W=W, ncsa=ncsa, nhca=nhca,
            csa_off=offs(ncsa), hca_off=offs(nhca),
            csa_t0=csa_t0, hca_t0=hca_t0, raw_t0=raw_t0,
            csa_x_off=offs([v - t for v, t in zip(n, csa_t0)]),
            hca_x_off=offs([v - t for v, t in zip(n, hca_t0)]),
            raw_off=offs([v - t for v, t in zip(n, raw_t0)]),
            csa_first=[f // 4 for f in first], csa_num=[c - f // 4 for c, f in zip(ncsa, first)],
            hca_first=[f // 128 for f in first], hca_num=[c - f // 128 for c, f in zip(nhca, first)],
            q_seq=[b for b in range(s.batch) for _ in range(Q)],
            q_pos=[n[b] - Q + j for b in range(s.batch) for j in range(Q)],
            scale=1.0 / math.sqrt(HEAD_DIM),
        )
        self.arrays = self._generate()

    # ------------------------------------------------------------------
    def _generate(self) -> dict:
        s, m = self.spec, self.meta
        seed, kv_std, dt = s.seed, 1.0 / math.sqrt(HEAD_DIM), s.dtype
        a = {}
        T, H, Hi, di = m["T"], m["H"], m["Hi"], m["di"]
        ncsa_tot, nhca_tot = m["csa_off"][-1], m["hca_off"][-1]
        rows_c, rows_h, rows_r = m["csa_x_off"][-1], m["hca_x_off"][-1], m["raw_off"][-1]

        for name in ("x_a", "x_b"):
            a[name] = _to_storage(_normal(seed, name, rows_c, ROW, kv_std), dt)
        for name in ("z_a", "z_b"):
            a[name] = _to_storage(_normal(seed, name, rows_c, ROW, 1.0), dt)
        a["x_h"] = _to_storage(_normal(seed, "x_h", rows_h, ROW, kv_std), dt)
        a["z_h"] = _to_storage(_normal(seed, "z_h", rows_h, ROW, 1.0), dt)
        a["raw_c"] = _to_storage(_normal(seed, "raw_c", rows_r, ROW, kv_std), dt)
        a["raw_h"] = _to_storage(_normal(seed, "raw_h", rows_r, ROW, kv_std), dt)

        qc = _normal(seed, "q_c", T * H, HEAD_DIM, kv_std).reshape(T, H, HEAD_DIM)
        a["q_h"] = _to_storage(_normal(seed, "q_h", T * H, HEAD_DIM, kv_std), dt).reshape(T, H, HEAD_DIM)
        qi = _normal(seed, "q_idx", T * Hi, di, 1.0 / math.sqrt(di)).reshape(T, Hi, di)
        ki = _normal(seed, "k_idx", ncsa_tot, di, 1.0 / math.sqrt(di))

        if s.cache == "random":
            cc = _normal(seed, "cmp_c", ncsa_tot, ROW, kv_std)
            a["cmp_h"] = _to_storage(_normal(seed, "cmp_h", nhca_tot, ROW, kv_std), dt)
        else:
            cc = np.zeros((ncsa_tot, ROW), np.float32)
            a["cmp_h"] = _to_storage(np.zeros((nhca_tot, ROW), np.float32), dt)

        needles = []
        if s.needles:
            # Plant needles for query 0 (sequence 0): entries visible to it, not recompressed by the step.
            vis = (m["q_pos"][0] + 1) // 4
            cand = min(vis, m["csa_first"][0])
            pick = _stream(seed, "needles", 0).choice(cand, size=s.needles, replace=False)
            needles = sorted(int(e) for e in pick)
            g = qi[0].sum(axis=0)
            g = g / np.linalg.norm(g)
            u = qc[0].mean(axis=0)
            u = u / np.linalg.norm(u)
            for e in needles:
                ki[m["csa_off"][0] + e] += np.float32(3.0) * g.astype(np.float32)
                cc[m["csa_off"][0] + e, :HEAD_DIM] += np.float32(3.0) * u.astype(np.float32)
        self.needles = needles

        a["q_c"] = _to_storage(qc.reshape(T * H, HEAD_DIM), dt).reshape(T, H, HEAD_DIM)
        a["cmp_c"] = _to_storage(cc, dt)
        if s.idx_dtype == "fp8":
            a["k_idx"], a["k_scale"] = _quant_e4m3(ki)
            codes, sc = _quant_e4m3(qi.reshape(T * Hi, di))
            a["q_idx"], a["q_scale"] = codes.reshape(T, Hi, di), sc.reshape(T, Hi)
        else:
            a["k_idx"], a["k_scale"] = torch.from_numpy(ki).clone(), None
            a["q_idx"], a["q_scale"] = torch.from_numpy(qi).clone(), None

        if s.pool_keys:
            # per-token indexer keys of the CSA tail rows (rows indexed like x_a), bf16
            a["k_tok"] = _normal(seed, "k_tok", rows_c, di, 1.0 / math.sqrt(di))
            a["k_tok"] = _to_storage(a["k_tok"], "bf16")
        a["head_w"] = torch.ones(Hi, dtype=torch.float32)
        if s.sink == "one":
            v = _normal(seed, "sink", 1, 1, 1.0)[0, 0]
            a["sink_c"] = torch.full((H,), float(v), dtype=torch.float32)
            a["sink_h"] = a["sink_c"].clone()
        elif s.sink == "per_head":
            a["sink_c"] = torch.from_numpy(_normal(seed, "sink_c", 1, H, 1.0)[0]).clone()
            a["sink_h"] = torch.from_numpy(_normal(seed, "sink_h", 1, H, 1.0)[0]).clone()
        else:
            a["sink_c"] = a["sink_h"] = None

        if s.biases:
            a["bias_a"] = torch.from_numpy(_normal(seed, "bias_a", 4, ROW, 1.0)).clone()
            a["bias_b"] = torch.from_numpy(_normal(seed, "bias_b", 4, ROW, 1.0)).clone()
            a["bias_h"] = torch.from_numpy(_normal(seed, "bias_h", 128, ROW, 1.0)).clone()
        else:
            a["bias_a"] = a["bias_b"] = a["bias_h"] = None

        for key in ("csa_off", "hca_off", "csa_t0", "hca_t0", "raw_t0", "csa_x_off", "hca_x_off",
                    "raw_off", "csa_first", "csa_num", "hca_first", "hca_num", "q_pos"):
            a[key] = torch.tensor(m[key], dtype=torch.int64)
        a["q_seq"] = torch.tensor(m["q_seq"], dtype=torch.int32)
        return a

    # ------------------------------------------------------------------
    def numpy(self, name: str) -> np.ndarray | None:
        """Storage-form numpy view: bf16 as uint16 codes, fp8 as uint8 codes."""
        t = self.arrays[name]
        if t is None:
            return None
        if t.dtype == torch.bfloat16:
            return t.view(torch.int16).numpy().view(np.uint16)
        return t.numpy()

    def device(self, dev) -> dict:
        return {k: (None if v is None else v.to(dev)) for k, v in self.arrays.items()}

    def host_bytes(self) -> int:
        return sum(v.numel() * v.element_size() for v in self.arrays.values() if v is not None)
