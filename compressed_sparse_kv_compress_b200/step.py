"""One hybrid decode step through the C ABI: compress, index + top-k, attend.

``DecodeStep`` holds the caller's device tensors (caches, tails, queries) and
the workspaces, and issues, in the pages' order ([SW] §三-§十二, [TR] §4.2-4.3
as cited in the C header):

  CSA layer: csa_compress (the entries the new tokens complete)
             -> lindex_score_topk -> hybrid_decode_attn(CSA)
  HCA layer: hca_compress -> hybrid_decode_attn(HCA)

Inside the CSA layer the indexer reads the entry keys, not the compressed
cache, so it is issued first and the compression of the newest entries runs
beside it as a dependent launch (CSKV_OVERLAP_PREVIOUS); the attention waits
for both.  The HCA layer does not depend on the CSA layer, so with
``two_streams`` it runs on a side stream that forks from and joins the
caller's stream.  The whole step can be captured into a CUDA graph and
replayed.

Tensor names (all device tensors, int64 offsets unless noted):
  CSA rows  x_a z_a x_b z_b [rows, 256], csa_x_off [B+1], csa_t0 [B],
            bias_a bias_b [4, 256] fp32 or None, csa_first csa_num [B]
  HCA rows  x_h z_h, hca_x_off, hca_t0, bias_h [128, 256] or None, hca_first hca_num
  caches    cmp_c [sum ceil(n/4), 256] + csa_off [B+1]; cmp_h + hca_off
  indexer   k_idx [entries, Di] (+ k_scale), q_idx [T, Hi, Di] (+ q_scale), head_w;
            optional k_tok [rows, Di] bf16 per-token keys (rows like x_a): the step pools
            its entries' keys from them inside the CSA compression
  window    raw_c raw_h [rows, 256], raw_off [B+1], raw_t0 [B]
  queries   q_c q_h [T, H, 128], sink_c sink_h [H] or None, q_seq [T] int32, q_pos [T]
"""

from __future__ import annotations

import torch

from . import api


class DecodeStep:
    def __init__(self, t: dict, *, k: int, window: int, scale: float, max_csa_blocks: int, max_hca_blocks: int,
                 max_csa_visible: int, max_hca_visible: int, two_streams: bool = False,
                 adjacent_pairs: bool = False):
        """adjacent_pairs: queries 2j and 2j + 1 are one sequence's consecutive positions (a
        prefill chunk): the HCA attention takes them in pairs (CSKV_ATTN_PAIRS)."""
        self.t = t
        self.adjacent_pairs = bool(adjacent_pairs)
        self.k, self.W, self.scale = int(k), int(window), float(scale)
        self.max_csa_blocks, self.max_hca_blocks = int(max_csa_blocks), int(max_hca_blocks)
        self.max_csa_visible, self.max_hca_visible = int(max_csa_visible), int(max_hca_visible)
        dev = t["q_c"].device
        T, H, _ = t["q_c"].shape
        self.T, self.H = T, H
        self.idx = torch.empty(T, self.k, dtype=torch.int32, device=dev)
        self.score = torch.empty(T, self.k, dtype=torch.float32, device=dev)
        # both layers' outputs in one buffer, so a read-back is a single copy
        self.o_all = torch.empty(2, T, H, 128, dtype=torch.float32, device=dev)
        self.o_c, self.o_h = self.o_all[0], self.o_all[1]
        self.lse_c = torch.empty(T, H, dtype=torch.float32, device=dev)
        self.lse_h = torch.empty_like(self.lse_c)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.ws_idx = api.lindex_workspace(T, self.k, self.max_csa_visible, dev)
        self.ws_c = api.attn_workspace(api.CSA, T, H, self.k, self.W, 0, dev)
        self.ws_h = api.attn_workspace(api.HCA, T, H, 0, self.W, self.max_hca_visible, dev)
        self.two_streams = two_streams
        self.side = torch.cuda.Stream(device=dev) if two_streams else None
        self.graph = None

    # ------------------------------------------------------------------
    def bulk_compress(self, max_csa_entries: int, max_hca_entries: int, stream=None):
        """Compress every entry of both caches from the rows provided (a cache built from scratch).

        max_*_entries bound ceil(n/4) and ceil(n/128) over the sequences."""
        t = self.t
        api.csa_compress(t["x_a"], t["z_a"], t["x_b"], t["z_b"], t["csa_x_off"], t["csa_off"], t["cmp_c"],
                         max_blocks=max_csa_entries, bias_a=t.get("bias_a"), bias_b=t.get("bias_b"),
                         tok0=t["csa_t0"], dev_status=self.status, stream=stream)
        api.hca_compress(t["x_h"], t["z_h"], t["hca_x_off"], t["hca_off"], t["cmp_h"],
                         max_blocks=max_hca_entries, bias=t.get("bias_h"), tok0=t["hca_t0"],
                         dev_status=self.status, stream=stream)

    def csa_compress(self, stream=None, after_select=False):
        """The CSA entries the new tokens complete; with per-token indexer keys (k_tok) the
        same kernel also pools those entries' indexer keys into k_idx / k_scale.
        after_select: issued right after csa_select on the same stream, which writes none of its
        inputs and reads none of its outputs (no key pooling): it then runs beside the indexer."""
        t = self.t
        pool = t.get("k_tok") is not None
        api.csa_compress(t["x_a"], t["z_a"], t["x_b"], t["z_b"], t["csa_x_off"], t["csa_off"], t["cmp_c"],
                         max_blocks=self.max_csa_blocks, bias_a=t.get("bias_a"), bias_b=t.get("bias_b"),
                         tok0=t["csa_t0"], first_block=t["csa_first"], num_blocks=t["csa_num"],
                         k_tok=t["k_tok"] if pool else None, k_codes=t["k_idx"] if pool else None,
                         k_scale=t["k_scale"] if pool else None, overlap_previous=after_select and not pool,
                         dev_status=self.status, stream=stream)

    def csa_select(self, stream=None):
        # no L2 prefetch of the kept rows (prefetch_rows): issuing it lengthens the indexer's
        # tail by more than it saves the attention's gather (measured 0.4 us a step at
        # b1_ctx1m and b8_ctx64k, 4 us at ragged_b64)
        t = self.t
        api.lindex_score_topk(t["q_idx"], t["k_idx"], t["q_seq"], t["q_pos"], t["csa_off"], self.idx, self.ws_idx,
                              max_entries=self.max_csa_visible, q_scale=t.get("q_scale"), k_scale=t.get("k_scale"),
                              head_w=t.get("head_w"), out_score=self.score, dev_status=self.status, stream=stream)

    def csa_attend(self, stream=None):
        t = self.t
        api.hybrid_decode_attn(api.CSA, t["q_c"], t["cmp_c"], t["csa_off"], t["raw_c"], t["raw_off"], t["q_seq"],
                               t["q_pos"], self.o_c, self.ws_c, window=self.W, idx=self.idx, raw_tok0=t["raw_t0"],
                               sink=t.get("sink_c"), scale=self.scale, lse=self.lse_c, dev_status=self.status,
                               stream=stream)

    def csa_layer(self, stream=None):
        """Compression, indexer and attention of the CSA layer on one stream.  The indexer reads
        the entry keys, not the compressed cache, so it goes first and the compression of the
        newest entries runs beside it (a dependent launch that waits for the indexer only at its
        end); the attention waits for both.  With per-token keys (k_tok) the compression pools
        the keys the indexer reads, so it goes first."""
        if self.t.get("k_tok") is not None:
            self.csa_compress(stream)
            self.csa_select(stream)
        else:
            self.csa_select(stream)
            self.csa_compress(stream, after_select=True)
        self.csa_attend(stream)

    def hca_layer(self, stream=None):
        t = self.t
        api.hca_compress(t["x_h"], t["z_h"], t["hca_x_off"], t["hca_off"], t["cmp_h"],
                         max_blocks=self.max_hca_blocks, bias=t.get("bias_h"), tok0=t["hca_t0"],
                         first_block=t["hca_first"], num_blocks=t["hca_num"], dev_status=self.status,
                         stream=stream)
        api.hybrid_decode_attn(api.HCA, t["q_h"], t["cmp_h"], t["hca_off"], t["raw_h"], t["raw_off"], t["q_seq"],
                               t["q_pos"], self.o_h, self.ws_h, window=self.W, raw_tok0=t["raw_t0"],
                               sink=t.get("sink_h"), scale=self.scale, lse=self.lse_h,
                               max_entries=self.max_hca_visible, adjacent_pairs=self.adjacent_pairs,
                               dev_status=self.status, stream=stream)

    def run(self, stream=None):
        """Issue the whole step on `stream` (default: the current stream)."""
        main = stream if stream is not None else torch.cuda.current_stream()
        if not self.two_streams:
            self.csa_layer(main)
            self.hca_layer(main)
            return
        # The HCA layer runs on a side stream beside the CSA layer, which it does not depend on.
        # The CSA layer is issued first, so that in a captured graph the indexer (the longest
        # kernel) is the first node to launch; its kernels chain by dependent launches alone.
        self.side.wait_stream(main)
        self.csa_layer(main)
        self.hca_layer(self.side)
        main.wait_stream(self.side)

    # ------------------------------------------------------------------
    def capture(self):
        """Capture run() into a CUDA graph (replay with replay())."""
        s = torch.cuda.Stream(device=self.o_c.device)
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.run(s)  # warm-up outside capture (sets kernel attributes)
        torch.cuda.current_stream().wait_stream(s)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.run()
        self.graph = g
        return g

    # transfers up to this size per direction go zero-copy by default: the pieces' CTAs reach
    # the pinned host buffer in one bus round trip each, where a copy node costs a fixed few
    # microseconds more (measured at 0.07-6.6 MB a step); larger ones, a prefill chunk's queries
    # and outputs, go through the copy engines
    ZERO_COPY_MAX_BYTES = 8 << 20
    # a segment is split into pieces of at most this size, one CTA each: 256 threads x 8 loads
    # of 16 bytes, so a piece costs one round trip over the bus
    PIECE_BYTES = 32 << 10

    def capture_io(self, h2d=(), d2h=(), zero_copy=None):
        """Capture, into one CUDA graph, the upload of this step's new inputs, the step, and the
        read-back of its results; replay with replay_io().

        h2d: (host, device) pairs.  The host sides are packed into one pinned staging buffer:
        the returned host tensors (views into it, initialised from the given ones) are where
        the caller writes each step's new inputs.  d2h: (device, host pinned) pairs copied back
        after the step.  Zero copy: one cskv_copy_segments launch reads the staging buffer over
        the bus and spreads it to the device tensors (which must be contiguous), and one more
        writes the results straight into the host tensors.  Otherwise a host-to-device copy of
        the buffer precedes the spreading launch and each result comes back by a
        device-to-host copy.  zero_copy: True / False for both directions; None (default)
        chooses zero copy for a direction whose bytes are at most ZERO_COPY_MAX_BYTES.  A
        replay costs one launch on the host, whatever the number of tensors."""
        views = self.prepare_io(h2d, d2h, zero_copy)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.run_io()
        self.graph_io = g
        return views

    def prepare_io(self, h2d=(), d2h=(), zero_copy=None):
        """The pinned staging buffer and copy tables of capture_io (returns the host views);
        run_io() then issues upload, step and read-back on the current stream."""
        if self.graph is None:
            self.capture()  # sets kernel attributes and warms up outside capture
        dev = self.o_c.device

        def i64(vals):
            return torch.tensor(list(vals), dtype=torch.int64, device=dev)

        def nbytes(t):
            return t.numel() * t.element_size()

        sizes = [nbytes(d) for _, d in h2d]
        offs, total = [], 0
        for nb in sizes:
            offs.append(total)
            total += (nb + 15) // 16 * 16
        stage_h = torch.empty(max(total, 16), dtype=torch.uint8, pin_memory=True)
        views = []
        for (h, d), o, nb in zip(h2d, offs, sizes):
            assert d.is_contiguous()
            v = stage_h[o:o + nb].view(d.dtype).view(d.shape)
            v.copy_(h)
            views.append(v)
        down_bytes = sum(nbytes(d) for d, _ in d2h)
        up_zc = zero_copy if zero_copy is not None else total <= self.ZERO_COPY_MAX_BYTES
        down_zc = zero_copy if zero_copy is not None else down_bytes <= self.ZERO_COPY_MAX_BYTES

        def pieces(segs):
            """(src_off, dst, len) segments cut into PIECE_BYTES pieces (16-byte boundaries
            inside a segment stay 16-byte boundaries), as three int64 device arrays."""
            so, da, ln = [], [], []
            for o, d, n in segs:
                for c in range(0, n, self.PIECE_BYTES):
                    so.append(o + c)
                    da.append(d + c)
                    ln.append(min(self.PIECE_BYTES, n - c))
            return i64(so), i64(da), i64(ln)

        up = None  # (staging buffer to fill first or None, copy_segments arguments)
        if h2d:
            segs = [(o, d.data_ptr(), nb) for o, (_, d), nb in zip(offs, h2d, sizes)]
            if up_zc:
                up = (None, (api.mapped_pointer(stage_h), *pieces(segs)))
            else:
                stage_d = torch.empty(stage_h.shape, dtype=torch.uint8, device=dev)
                up = (stage_d, (stage_d, *pieces(segs)))
        down = None
        if d2h and down_zc:
            for d, h in d2h:
                assert d.is_contiguous() and h.is_contiguous() and h.is_pinned()
                assert nbytes(d) == nbytes(h)
            base = min(d.data_ptr() for d, _ in d2h)
            down = (base, *pieces([(d.data_ptr() - base, api.mapped_pointer(h), nbytes(d)) for d, h in d2h]))
        # the host tensors stay referenced for as long as the captured graph may touch them
        self._io = (stage_h, up, down, list(d2h))
        self.io_zero_copy = (up_zc if h2d else None, down_zc if d2h else None)
        return views

    def run_io(self):
        """Upload, the step, the read-back (prepare_io first)."""
        stage_h, up, down, d2h = self._io
        if up is not None:
            stage_d, args = up
            if stage_d is not None:
                stage_d.copy_(stage_h, non_blocking=True)
            api.copy_segments(*args)
        self.run()
        if down is not None:
            api.copy_segments(*down)
        else:
            for d, h in d2h:
                h.copy_(d, non_blocking=True)

    def replay_io(self):
        self.graph_io.replay()

    def replay(self):
        self.graph.replay()
