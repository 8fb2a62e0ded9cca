"""lindex_pool_keys: the indexer's entry keys pooled from per-token keys and stored as E4M3
codes with per-entry scales, on ragged sequences with partial blocks and provided tails, and
on sampled entries of a 1M-token sequence.

Two checks per case: (1) against the exact fp64 definition -- codes equal except inside the
fp32 error band around an E4M3 rounding boundary, where the neighbouring code is allowed and
counted; (2) a second, labelled check: bit for bit against the oracle's fp32 restatement of
the same steps (the kernel's precision)."""

import numpy as np
import pytest
import torch

from compressed_sparse_kv_compress_b200 import api
from oracle import codecs, indexer

from helpers import check_pooled_keys

pytestmark = pytest.mark.gpu


def _rows(rng, n, Di, dtype):
    x = torch.from_numpy(rng.standard_normal((n, Di)).astype(np.float32) / 8.0)
    if dtype == "bf16":
        x = x.to(torch.bfloat16)
    return x


def _as_f32(x: torch.Tensor) -> np.ndarray:
    if x.dtype == torch.bfloat16:
        return codecs.bf16_decode(x.view(torch.int16).numpy().view(np.uint16)).astype(np.float32)
    return x.numpy().astype(np.float32)


def _i64(v):
    return torch.tensor(v, dtype=torch.int64, device="cuda")


@pytest.mark.parametrize("dtype,Di", [("bf16", 64), ("f32", 64), ("bf16", 128), ("f32", 128)])
def test_ragged_sequences_with_tails_bit_exact(dtype, Di):
    rng = np.random.default_rng(Di + (dtype == "bf16"))
    n = [4097, 30, 1, 4 * 700, 2 * 240 + 3]          # lengths; partial last blocks
    t0 = [0, 0, 0, 1200, 8]                           # sequence 3 and 4 provide a tail only
    toks = [_rows(rng, n[b] - t0[b], Di, dtype) for b in range(len(n))]
    nent = [(x + 3) // 4 for x in n]
    ent_off = np.concatenate([[0], np.cumsum(nent)])
    tok_off = np.concatenate([[0], np.cumsum([len(t) for t in toks])])
    first = [0, 0, 0, t0[3] // 4, t0[4] // 4]        # entries whose tokens are all provided
    num = [nent[b] - first[b] for b in range(len(n))]
    k_tok = torch.cat(toks).cuda()
    codes = torch.full((ent_off[-1], Di), 0xAA, dtype=torch.uint8, device="cuda")
    scale = torch.full((ent_off[-1],), -1.0, dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.lindex_pool_keys(k_tok, _i64(tok_off), _i64(ent_off), codes, scale, max_blocks=max(num),
                         tok0=_i64(t0), first_block=_i64(first), num_blocks=_i64(num), dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    codes, scale = codes.cpu().numpy(), scale.cpu().numpy()
    for b in range(len(n)):
        # the oracle over the whole sequence, with the rows before the tail absent: pool the
        # provided tokens (the tail starts on a block boundary) and compare the computed entries
        f32 = _as_f32(toks[b])
        e0 = ent_off[b] + first[b]
        banded = check_pooled_keys(codes[e0:e0 + num[b]], scale[e0:e0 + num[b]], f32.astype(np.float64), 4,
                                   what=f"sequence {b}")
        assert banded <= max(8, f32.size // 200)  # a narrow band: well under 1 % of the codes
        # second check: the fp32 restatement, bit for bit
        want_c, want_s = indexer.quantize_keys(indexer.pool_keys(f32, 4))
        assert np.array_equal(codes[e0:e0 + num[b]], want_c), f"codes, sequence {b}"
        assert np.array_equal(scale[e0:e0 + num[b]], want_s), f"scales, sequence {b}"
        # entries not asked for are untouched
        assert np.all(codes[ent_off[b]:e0] == 0xAA) and np.all(scale[ent_off[b]:e0] == -1.0)


def test_zero_key_and_saturation_edges():
    Di = 64
    x = np.zeros((12, Di), np.float32)
    x[4:8] = 3.0                      # a constant block: every element lands on 448
    x[8, 0], x[9, 0] = 1e-30, -1e-30  # a block whose mean is exactly zero in dim 0
    x[8, 1] = 5.0
    k_tok = torch.from_numpy(x).cuda()
    codes = torch.empty(3, Di, dtype=torch.uint8, device="cuda")
    scale = torch.empty(3, dtype=torch.float32, device="cuda")
    api.lindex_pool_keys(k_tok, _i64([0, 12]), _i64([0, 3]), codes, scale, max_blocks=3)
    torch.cuda.synchronize()
    check_pooled_keys(codes.cpu().numpy(), scale.cpu().numpy(), x.astype(np.float64), 4, what="edges")
    want_c, want_s = indexer.quantize_keys(indexer.pool_keys(x, 4))
    assert np.array_equal(codes.cpu().numpy(), want_c) and np.array_equal(scale.cpu().numpy(), want_s)
    assert scale[0].item() == 1.0 and torch.all(codes[0] == 0)
    assert torch.all(codes[1] == 0x7E)


def test_device_checks_flag_and_skip():
    Di = 64
    k_tok = torch.zeros(40, Di, device="cuda")
    codes = torch.full((16, Di), 0x11, dtype=torch.uint8, device="cuda")
    scale = torch.zeros(16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    # entry 10 lies past the 40-token sequence: skipped and flagged
    api.lindex_pool_keys(k_tok, _i64([0, 40]), _i64([0, 16]), codes, scale, max_blocks=1,
                         first_block=_i64([10]), num_blocks=_i64([1]), dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & 1 and torch.all(codes == 0x11)
    # the tail starts at token 8: entry 1 (tokens 4..7) is missing
    st.zero_()
    api.lindex_pool_keys(k_tok[:32], _i64([0, 32]), _i64([0, 16]), codes, scale, max_blocks=1,
                         tok0=_i64([8]), first_block=_i64([1]), num_blocks=_i64([1]), dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & 2 and torch.all(codes == 0x11)
    # more entries asked for than the bound
    st.zero_()
    api.lindex_pool_keys(k_tok, _i64([0, 40]), _i64([0, 16]), codes, scale, max_blocks=2,
                         num_blocks=_i64([10]), dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & 4


def test_million_token_sequence_sampled_entries():
    # the whole-cache call (bounded grid, warps looping over 262,144 entries), sampled entries
    n, Di = 1 << 20, 64
    g = torch.Generator(device="cuda")
    g.manual_seed(7)
    k_tok = (torch.randn(n, Di, generator=g, device="cuda") / 8).to(torch.bfloat16)
    V = n // 4
    codes = torch.empty(V, Di, dtype=torch.uint8, device="cuda")
    scale = torch.empty(V, dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.lindex_pool_keys(k_tok, _i64([0, n]), _i64([0, V]), codes, scale, max_blocks=V, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rng = np.random.default_rng(3)
    sample = np.unique(np.concatenate([[0, 1, V - 1], rng.integers(0, V, 2000)]))
    rows = k_tok.view(V, 4, Di)[torch.from_numpy(sample).cuda()].cpu()
    f32 = codecs.bf16_decode(rows.view(torch.int16).numpy().view(np.uint16)).astype(np.float32)
    banded = check_pooled_keys(codes.cpu().numpy()[sample], scale.cpu().numpy()[sample],
                               f32.reshape(-1, Di).astype(np.float64), 4, what="1M sample")
    assert banded <= max(8, f32.size // 200)
    want_c, want_s = indexer.quantize_keys(indexer.pool_keys(f32.reshape(-1, Di), 4))
    assert np.array_equal(codes.cpu().numpy()[sample], want_c)
    assert np.array_equal(scale.cpu().numpy()[sample], want_s)
