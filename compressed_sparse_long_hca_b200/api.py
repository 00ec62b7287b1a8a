"""Thin Python binding over the C ABI (include/csa.h).

PyTorch supplies device memory and streams; every step of the decode path
runs in libcsa's CUDA kernels.  Functions here only check tensor shapes,
dtypes and devices and pass raw pointers.
"""
from __future__ import annotations

import ctypes

import numpy as np
import torch

from . import _lib
from ._lib import CsaCfg, check

VARIANTS = {"auto": _lib.VARIANT_AUTO, "high": _lib.VARIANT_HIGH_OCC, "low": _lib.VARIANT_LOW_OCC}
STATE_READY = _lib.ATTN_STATE_READY
FORMATS = {"mixed": _lib.FMT_MIXED, "f32": _lib.FMT_F32}


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream or None


def _need(t, dtype, shape=None, name="tensor"):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


class Cache:
    """A CSA/HCA cache living in one caller-owned device buffer (the arena).

    Pool pages hold 512 raw tokens (4 classic-cache blocks) of one request.

    Layers 0 .. n_csa-1 are CSA layers, n_csa .. n_csa+n_hca-1 HCA layers."""

    def __init__(self, *, n_csa: int, n_hca: int, H: int, D: int, D_rope: int, H_I: int, d_I: int,
                 max_requests: int, max_pages_per_request: int, pool_pages: int,
                 b_pos_csa=None, b_pos_idx=None, b_pos_hca=None, rope_base: float = 10000.0,
                 fmt: str = "mixed", device: str | torch.device = "cuda"):
        """fmt: "mixed" (FP8 + BF16 rows, MXFP4 index keys, BF16 q and out) or
        "f32" (fp32 rows, keys, q and out)."""
        self.lib = _lib.load()
        if fmt not in FORMATS:
            raise ValueError(f"fmt must be one of {sorted(FORMATS)}")
        self.fmt = fmt
        self.qdtype = torch.float32 if fmt == "f32" else torch.bfloat16
        self.cfg = CsaCfg(n_csa, n_hca, H, D, D_rope, H_I if n_csa else 0, d_I if n_csa else 0, 128,
                          max_requests, max_pages_per_request, pool_pages, rope_base, FORMATS[fmt])
        nbytes = self.lib.csa_cache_required_bytes(ctypes.byref(self.cfg))
        if nbytes == 0:
            raise ValueError("invalid cache configuration")
        self.nbytes = nbytes
        self.arena = torch.empty(nbytes + 256, dtype=torch.uint8, device=device)
        base = self.arena.data_ptr()
        aligned = (base + 255) // 256 * 256
        self.n_csa, self.n_hca = n_csa, n_hca
        self.H, self.D, self.D_rope, self.H_I, self.d_I = H, D, D_rope, H_I, d_I

        def host(a, shape):
            if a is None:
                return None, None
            arr = np.ascontiguousarray(np.asarray(a, dtype=np.float32).reshape(shape))
            return arr, arr.ctypes.data

        self._bkv, p_bkv = host(b_pos_csa, (n_csa, 8, D)) if n_csa else (None, None)
        self._bix, p_bix = host(b_pos_idx, (n_csa, 8, d_I)) if n_csa else (None, None)
        self._bh, p_bh = host(b_pos_hca, (n_hca, 128, D)) if n_hca else (None, None)
        handle = ctypes.c_void_p()
        torch.cuda.synchronize()
        check(self.lib.csa_cache_init(ctypes.byref(self.cfg), aligned, nbytes, p_bkv, p_bix, p_bh,
                                      ctypes.byref(handle)), "csa_cache_init")
        self.handle = handle

    def __del__(self):
        h = getattr(self, "handle", None)
        if h is not None and h.value:
            self.lib.csa_cache_destroy(h)
            self.handle = None

    # ------------------------------------------------------------ requests
    def request_alloc(self, req: int, capacity_tokens: int) -> None:
        check(self.lib.csa_request_alloc(self.handle, req, capacity_tokens), "csa_request_alloc")

    def request_free(self, req: int) -> None:
        check(self.lib.csa_request_free(self.handle, req), "csa_request_free")

    # ------------------------------------------------------------ the path
    def compress_append(self, layer: int, req_ids: torch.Tensor, kv_cand, kv_gate,
                        idx_cand=None, idx_gate=None, stream=None) -> None:
        n = req_ids.numel()
        _need(req_ids, torch.int32, name="req_ids")
        n_tok = kv_cand.shape[1] if n else 0
        _need(kv_cand, torch.float32, (n, n_tok, self.D), "kv_cand")
        _need(kv_gate, torch.float32, (n, n_tok, self.D), "kv_gate")
        if layer < self.n_csa:
            _need(idx_cand, torch.float32, (n, n_tok, self.d_I), "idx_cand")
            _need(idx_gate, torch.float32, (n, n_tok, self.d_I), "idx_gate")
        check(self.lib.csa_compress_append(self.handle, layer, n, _ptr(req_ids), n_tok, _ptr(kv_cand),
                                           _ptr(kv_gate), _ptr(idx_cand), _ptr(idx_gate),
                                           _stream(stream)), "csa_compress_append")

    def index_scores(self, layer: int, req_ids, q_idx, w, scores, n_valid, variant="auto",
                     stream=None) -> None:
        n = req_ids.numel()
        _need(req_ids, torch.int32, name="req_ids")
        _need(q_idx, torch.float32, (n, self.H_I, self.d_I), "q_idx")
        _need(w, torch.float32, (n, self.H_I), "w")
        _need(scores, torch.float32, name="scores")
        _need(n_valid, torch.int32, (n,), "n_valid")
        if scores.dim() != 2 or scores.shape[0] != n:
            raise ValueError("scores must be [n, ld]")
        check(self.lib.csa_index_scores(self.handle, layer, n, _ptr(req_ids), _ptr(q_idx), _ptr(w),
                                        _ptr(scores), scores.shape[1], _ptr(n_valid),
                                        VARIANTS[variant], _stream(stream)), "csa_index_scores")

    def index_topk(self, layer: int, req_ids, q_idx, w, scores, n_valid, k: int, idx_out, variant="auto",
                   stream=None, workspace: torch.Tensor | None = None) -> None:
        """Index scores and top-k in one launch (csa_index_topk): the same
        results as index_scores followed by topk.  Unless `workspace` is
        given, a buffer owned by this Cache object is grown to the size the
        library asks for."""
        n = req_ids.numel()
        _need(req_ids, torch.int32, name="req_ids")
        _need(q_idx, torch.float32, (n, self.H_I, self.d_I), "q_idx")
        _need(w, torch.float32, (n, self.H_I), "w")
        _need(scores, torch.float32, name="scores")
        _need(n_valid, torch.int32, (n,), "n_valid")
        _need(idx_out, torch.int32, (n, k), "idx_out")
        if scores.dim() != 2 or scores.shape[0] != n:
            raise ValueError("scores must be [n, ld]")
        ws_ptr, ws_bytes = None, 0
        if n > 0:
            need = self.index_topk_workspace_bytes(n, scores.shape[1])
            if workspace is None:
                ws = getattr(self, "_tk_ws", None)
                if ws is None or ws.numel() < need + 256 or ws.device != q_idx.device:
                    ws = torch.empty(need + 256, dtype=torch.uint8, device=q_idx.device)
                    self._tk_ws = ws
                workspace = ws
            _need(workspace, torch.uint8, name="workspace")
            ws_ptr = (workspace.data_ptr() + 255) // 256 * 256
            ws_bytes = workspace.numel() - (ws_ptr - workspace.data_ptr())
        check(self.lib.csa_index_topk(self.handle, layer, n, _ptr(req_ids), _ptr(q_idx), _ptr(w), _ptr(scores),
                                      scores.shape[1], _ptr(n_valid), k, _ptr(idx_out), ws_ptr, ws_bytes,
                                      VARIANTS[variant], _stream(stream)), "csa_index_topk")

    def index_topk_workspace_bytes(self, n: int, ld: int) -> int:
        return int(self.lib.csa_index_topk_workspace_bytes(self.handle, n, ld))

    def attn_workspace_bytes(self, layer: int, n: int, k: int = 0) -> int:
        return int(self.lib.csa_attn_workspace_bytes(self.handle, layer, n, k))

    def _workspace(self, nbytes: int, device) -> torch.Tensor:
        ws = getattr(self, "_ws", None)
        if ws is None or ws.numel() < nbytes or ws.device != device:
            ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)
            self._ws = ws
        return ws

    def decode_attn(self, layer: int, req_ids, q, topk_idx, sink, out, scale=None,
                    variant="auto", stream=None, workspace: torch.Tensor | None = None,
                    state_ready: bool = False) -> None:
        """Attention of each query over its rows.  The split (low-occupancy)
        launch needs scratch; unless `workspace` is given, a buffer owned by
        this Cache object is grown to the size the library asks for.
        state_ready (CSA_ATTN_STATE_READY): the call directly follows this
        step's index_topk on the stream, so the lengths, window rows and q
        may be read before that kernel ends."""
        n = req_ids.numel()
        _need(req_ids, torch.int32, name="req_ids")
        _need(q, self.qdtype, (n, self.H, self.D), "q")
        _need(out, self.qdtype, (n, self.H, self.D), "out")
        _need(sink, torch.float32, (self.H,), "sink")
        k = 0
        if topk_idx is not None:
            _need(topk_idx, torch.int32, name="topk_idx")
            k = topk_idx.shape[1]
        if scale is None:
            scale = 1.0 / float(np.sqrt(self.D))
        ws_ptr, ws_bytes = None, 0
        if variant != "high" and n > 0:
            need = self.attn_workspace_bytes(layer, n, k)
            if workspace is None:
                workspace = self._workspace(need, q.device)
            _need(workspace, torch.uint8, name="workspace")
            ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel()
        flags = STATE_READY if state_ready else 0
        check(self.lib.csa_hca_decode_attn(self.handle, layer, n, _ptr(req_ids), _ptr(q), _ptr(topk_idx),
                                           k, _ptr(sink), scale, _ptr(out), ws_ptr, ws_bytes,
                                           VARIANTS[variant] | flags, _stream(stream)), "csa_hca_decode_attn")

    def prefill_workspace_bytes(self, layer: int, n: int, n_tok: int, k: int = 0, variant="auto") -> int:
        return int(self.lib.csa_prefill_workspace_bytes(self.handle, layer, n, n_tok, k, VARIANTS[variant]))

    def prefill_chunk(self, layer: int, req_ids, kv_cand, kv_gate, idx_cand, idx_gate, q, q_idx, w, k: int,
                      sink, out, topk_out=None, scale=None, variant="auto", stream=None,
                      workspace: torch.Tensor | None = None) -> None:
        """A chunk of n_tok (1 .. 128) new tokens per request, each also a
        query with causal visibility (csa_prefill_chunk): the tokens are
        appended, and query j of request b (at position len - n_tok + j)
        attends to what a decode query there would.  kv_cand, kv_gate
        [n, n_tok, D] fp32; idx_cand, idx_gate [n, n_tok, d_I] fp32, q_idx
        [n, n_tok, H_I, d_I] and w [n, n_tok, H_I] fp32 (CSA layers, else
        None); q and out [n, n_tok, H, D] (BF16, fp32 in the fp32 format);
        topk_out [n, n_tok, k] int32 or None.  Unless `workspace` is given, a
        buffer owned by this Cache object is grown to the size the library
        asks for."""
        n = req_ids.numel()
        _need(req_ids, torch.int32, name="req_ids")
        n_tok = kv_cand.shape[1] if kv_cand.dim() == 3 else -1
        _need(kv_cand, torch.float32, (n, n_tok, self.D), "kv_cand")
        _need(kv_gate, torch.float32, (n, n_tok, self.D), "kv_gate")
        _need(q, self.qdtype, (n, n_tok, self.H, self.D), "q")
        _need(out, self.qdtype, (n, n_tok, self.H, self.D), "out")
        _need(sink, torch.float32, (self.H,), "sink")
        csa = layer < self.n_csa
        if csa:
            _need(idx_cand, torch.float32, (n, n_tok, self.d_I), "idx_cand")
            _need(idx_gate, torch.float32, (n, n_tok, self.d_I), "idx_gate")
            _need(q_idx, torch.float32, (n, n_tok, self.H_I, self.d_I), "q_idx")
            _need(w, torch.float32, (n, n_tok, self.H_I), "w")
            if topk_out is not None:
                _need(topk_out, torch.int32, (n, n_tok, k), "topk_out")
        else:
            k = 0
        if scale is None:
            scale = 1.0 / float(np.sqrt(self.D))
        need = self.prefill_workspace_bytes(layer, n, n_tok, k, variant)
        if need == 0:
            raise ValueError("invalid chunk shape (n_tok must be in [1, 128], n * n_tok <= 65535)")
        if workspace is None:
            ws = getattr(self, "_pf_ws", None)
            if ws is None or ws.numel() < need + 256 or ws.device != q.device:
                ws = torch.empty(need + 256, dtype=torch.uint8, device=q.device)
                self._pf_ws = ws
            workspace = ws
        _need(workspace, torch.uint8, name="workspace")
        ws_ptr = (workspace.data_ptr() + 255) // 256 * 256
        ws_bytes = workspace.numel() - (ws_ptr - workspace.data_ptr())
        check(self.lib.csa_prefill_chunk(self.handle, layer, n, _ptr(req_ids), n_tok, _ptr(kv_cand), _ptr(kv_gate),
                                         _ptr(idx_cand), _ptr(idx_gate), _ptr(q), _ptr(q_idx), _ptr(w), k,
                                         _ptr(sink), scale, _ptr(out), _ptr(topk_out), ws_ptr, ws_bytes,
                                         VARIANTS[variant], _stream(stream)), "csa_prefill_chunk")

    def check_device_error(self, stream=None) -> None:
        check(self.lib.csa_check_device_error(self.handle, _stream(stream)), "device")

    # ------------------------------------------------------------ test helpers
    def row_bytes(self, region: int) -> int:
        return self.lib.csa_debug_row_bytes(self.handle, region)

    def read_rows(self, layer: int, req: int, region: int, first: int, count: int) -> np.ndarray:
        buf = np.zeros((count, self.row_bytes(region)), dtype=np.uint8)
        check(self.lib.csa_debug_rows(self.handle, layer, req, region, first, count,
                                      buf.ctypes.data, 0), "csa_debug_rows(read)")
        return buf

    def write_rows(self, layer: int, req: int, region: int, first: int, rows: np.ndarray) -> None:
        rows = np.ascontiguousarray(rows, dtype=np.uint8)
        assert rows.shape[1] == self.row_bytes(region)
        check(self.lib.csa_debug_rows(self.handle, layer, req, region, first, rows.shape[0],
                                      rows.ctypes.data, 1), "csa_debug_rows(write)")

    def set_length(self, layer: int, req: int, length: int) -> None:
        check(self.lib.csa_debug_set_length(self.handle, layer, req, length), "csa_debug_set_length")

    def get_length(self, layer: int, req: int) -> int:
        return int(self.lib.csa_debug_get_length(self.handle, layer, req))


def topk(scores: torch.Tensor, n_valid: torch.Tensor, k: int, out: torch.Tensor,
         variant="auto", stream=None) -> None:
    lib = _lib.load()
    _need(scores, torch.float32, name="scores")
    _need(n_valid, torch.int32, name="n_valid")
    n = scores.shape[0]
    _need(out, torch.int32, (n, k), "out")
    check(lib.csa_topk(_ptr(scores), scores.shape[1], _ptr(n_valid), n, k, _ptr(out),
                       VARIANTS[variant], _stream(stream)), "csa_topk")


# ---------------------------------------------------------------- one decode step, replayed

def decode_step_fields(n: int, H: int, D: int, H_I: int, d_I: int, csa: bool, align: int = 256,
                       qdtype=torch.bfloat16):
    """Packed layout of one decode step's inputs: a list of (name, dtype,
    shape, byte offset, bytes) with every field starting on an `align`-byte
    boundary, and the buffer's total size.  The attention query q (BF16, or
    fp32 for an fp32 cache) comes last, so that everything before it is one
    contiguous copy."""
    fields = [("c", torch.float32, (n, 1, D)), ("z", torch.float32, (n, 1, D))]
    if csa:
        fields += [("ci", torch.float32, (n, 1, d_I)), ("zi", torch.float32, (n, 1, d_I)),
                   ("q_idx", torch.float32, (n, H_I, d_I)), ("w", torch.float32, (n, H_I))]
    fields.append(("q", qdtype, (n, H, D)))
    out, off = [], 0
    for name, dtype, shape in fields:
        nbytes = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        out.append((name, dtype, shape, off, nbytes))
        off += (nbytes + align - 1) // align * align
    return out, off


class DecodeStep:
    """One decode step of a fixed batch of requests on one layer, captured
    once as a CUDA graph and replayed every step.

    The step is the C ABI's csa_decode_step (host input copy, append, index
    scores and top-k, attention, output copy, on one stream, the query's copy
    on a second one); with fused_select=True it is composed here from
    csa_compress_append, csa_index_topk (one launch) and csa_hca_decode_attn
    instead.  The attention may start while the selection finishes.

    Inputs of a step, packed in the pinned host buffer `host_in` (owned by
    the step) and filled through `views(step.host_in)`: c and z [n, 1, D] fp32
    (the token's KV candidate and gate logits), on a CSA layer also ci and zi
    [n, 1, d_I] fp32, q_idx [n, H_I, d_I] fp32 and w [n, H_I] fp32, and last
    q [n, H, D] (bf16, fp32 in the fp32 format).  Each field starts on a
    256-byte boundary.

    Host transfers are nodes of the graph: the fields before q in one copy
    ahead of the append; q, which only the attention reads, in one copy on a
    forked branch that runs beside the append and the selection and that the
    attention waits for; the output [n, H, D] in one copy into `host_out`
    (pinned) at the end.

    The graph holds device and host pointers, so the batch (req_ids), k, the
    sink logits and the two host buffers are fixed at construction.  On a CSA
    layer construction runs the selection once (it changes nothing in the
    cache) so that its one-time launch set-up happens before the capture."""

    def __init__(self, cache: Cache, layer: int, req_ids, k: int, sink, variant: str = "auto",
                 device: str | torch.device = "cuda", fused_select: bool = False):
        self.cache, self.layer, self.k, self.variant = cache, layer, int(k), variant
        self.fused_select = bool(fused_select)
        self.csa = layer < cache.n_csa
        ids = [int(r) for r in req_ids]
        n = self.n = len(ids)
        if n == 0:
            raise ValueError("a decode step needs at least one request")
        if self.csa and self.k <= 0:
            raise ValueError("a CSA layer needs k > 0")
        H, D = cache.H, cache.D
        self._fields, off = decode_step_fields(n, H, D, cache.H_I, cache.d_I, self.csa, qdtype=cache.qdtype)
        if int(cache.lib.csa_decode_step_input_bytes(cache.handle, layer, n)) != off:
            raise RuntimeError("packed input layout differs from the library's")
        self.input_bytes = off
        self._q_off = next(f[3] for f in self._fields if f[0] == "q")
        dev = self.device = torch.device(device)
        self._dev_in = torch.zeros(off, dtype=torch.uint8, device=dev)
        self.host_in = torch.zeros(off, dtype=torch.uint8).pin_memory()
        self._req = torch.tensor(ids, dtype=torch.int32, device=dev)
        self._sink = (sink if isinstance(sink, torch.Tensor) else torch.from_numpy(np.asarray(sink, np.float32)))
        self._sink = self._sink.to(device=dev, dtype=torch.float32).contiguous()
        self.out = torch.empty((n, H, D), dtype=cache.qdtype, device=dev)
        self.host_out = torch.empty((n, H, D), dtype=cache.qdtype).pin_memory()
        self._ws = torch.empty(max(cache.attn_workspace_bytes(layer, n, self.k if self.csa else 0), 16),
                               dtype=torch.uint8, device=dev)
        self._side = torch.cuda.Stream(device=dev)
        self._done = torch.cuda.Event()
        self._dev_buf = None
        if not self.fused_select:
            nbytes = int(cache.lib.csa_decode_step_dev_bytes(cache.handle, layer, n, self.k if self.csa else 0))
            if nbytes == 0:
                raise ValueError("invalid decode step shape")
            self._dev_buf = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
            # the C step holds its own copies of the inputs and the output
            self._dev_in = None
            self.out = None
            if self.csa:
                # one eager pass of the selection kernels on the C step's own
                # scratch (it changes nothing in the cache) does their one-time
                # launch set-up (cluster-size query) outside the capture
                d = self.views(self._dev_buf[: self.input_bytes])
                ld = max(cache.cfg.max_pages_per_request * 128, 128)
                o = self.input_bytes
                scores = self._dev_buf[o: o + n * ld * 4].view(torch.float32).view(n, ld)
                o += (n * ld * 4 + 255) // 256 * 256
                nv = self._dev_buf[o: o + n * 4].view(torch.int32)
                cache.index_scores(layer, self._req, d["q_idx"], d["w"], scores, nv)
                topk(scores, nv, self.k, self.topk_idx)
                torch.cuda.synchronize(dev)
                cache.check_device_error()
        if self.csa and self.fused_select:
            n_max = max(cache.cfg.max_pages_per_request * 128, 128)   # 512 tokens = 128 entries per page
            self._scores = torch.empty((n, n_max), dtype=torch.float32, device=dev)
            self._nv = torch.empty(n, dtype=torch.int32, device=dev)
            self._idx = torch.empty((n, self.k), dtype=torch.int32, device=dev)
            self._tk_ws = torch.empty(cache.index_topk_workspace_bytes(n, n_max) + 256, dtype=torch.uint8,
                                      device=dev)
            # one eager pass of the selection kernels (valid on any cache
            # state, an empty request included) does their one-time launch
            # set-up (cluster-size query) outside the capture
            self._select(self.views(self._dev_in))
            torch.cuda.synchronize(dev)
            cache.check_device_error()
        self.graph = self._capture(None)
        self.marks = None
        self._graph_marked = None
        torch.cuda.synchronize(dev)

    def _select(self, d) -> None:
        cache, layer, variant = self.cache, self.layer, self.variant
        if self.fused_select:           # index scores and top-k in one launch (csa_index_topk)
            cache.index_topk(layer, self._req, d["q_idx"], d["w"], self._scores, self._nv, self.k, self._idx,
                             variant, workspace=self._tk_ws)
        else:                           # csa_index_scores, then csa_topk
            cache.index_scores(layer, self._req, d["q_idx"], d["w"], self._scores, self._nv, variant)
            topk(self._scores, self._nv, self.k, self._idx, variant)

    def _step_c(self, stream) -> None:
        c = self.cache
        check(c.lib.csa_decode_step(c.handle, self.layer, self.n, self._req.data_ptr(), self.k if self.csa else 0,
                                    self._sink.data_ptr(), 1.0 / float(np.sqrt(c.D)), self.host_in.data_ptr(),
                                    self.host_out.data_ptr(), self._dev_buf.data_ptr(), self._dev_buf.numel(),
                                    stream.cuda_stream), "csa_decode_step")

    def _capture(self, marks):
        """The step as one graph; `marks` (two external timing events) are
        recorded after the inputs are on the device and after the attention
        (the composed step) or before and after the whole C step."""
        cache, layer = self.cache, self.layer
        if not self.fused_select:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                main = torch.cuda.current_stream(self.device)
                if marks is not None:
                    marks[0].record(main)
                self._step_c(main)
                if marks is not None:
                    marks[1].record(main)
            return g
        d = self.views(self._dev_in)
        qo = self._q_off
        ev_fork, ev_q = torch.cuda.Event(), torch.cuda.Event()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            main = torch.cuda.current_stream(self.device)
            ev_fork.record(main)
            self._side.wait_event(ev_fork)
            with torch.cuda.stream(self._side):
                self._dev_in[qo:].copy_(self.host_in[qo:], non_blocking=True)
                ev_q.record(self._side)
            self._dev_in[:qo].copy_(self.host_in[:qo], non_blocking=True)
            if marks is not None:
                marks[0].record(main)
            cache.compress_append(layer, self._req, d["c"], d["z"], d.get("ci"), d.get("zi"))
            if self.csa:
                self._select(d)
            main.wait_event(ev_q)
            cache.decode_attn(layer, self._req, d["q"], self._idx if self.csa else None, self._sink, self.out,
                              variant=self.variant, workspace=self._ws, state_ready=self.csa)
            if marks is not None:
                marks[1].record(main)
            self.host_out.copy_(self.out, non_blocking=True)
        return g

    def views(self, buf: torch.Tensor) -> dict:
        """Typed views of the step's input fields inside a packed buffer."""
        if buf.dtype != torch.uint8 or buf.numel() < self.input_bytes or not buf.is_contiguous():
            raise ValueError(f"a packed input buffer is {self.input_bytes} contiguous bytes")
        return {name: buf[off: off + nbytes].view(dtype).view(shape)
                for name, dtype, shape, off, nbytes in self._fields}

    def new_host_inputs(self) -> torch.Tensor:
        """A pinned host buffer for one step's packed inputs (for callers
        that keep their own buffers; see __call__)."""
        return torch.zeros(self.input_bytes, dtype=torch.uint8).pin_memory()

    def __call__(self, host_inputs: torch.Tensor | None = None, timed: bool = False) -> torch.Tensor:
        """Enqueue one step on the current stream and return `host_out` (the
        output [n, H, D], valid once the stream has reached the end of the
        step; the next call overwrites it).

        The step reads its inputs from `host_in`: fill it through
        `views(step.host_in)` and call with no argument.  It must not change
        until the step's copy has run (`ready()`).  A caller's own pinned
        buffer may be passed instead: the call then waits for the previous
        step and copies it into `host_in` on the host first.

        timed=True replays a second capture of the step that records the
        events `marks` (after the input copy, after the attention) for
        timing the phases."""
        if host_inputs is not None and host_inputs.data_ptr() != self.host_in.data_ptr():
            if host_inputs.device.type != "cpu" or host_inputs.dtype != torch.uint8 \
                    or host_inputs.numel() != self.input_bytes:
                raise ValueError(f"host_inputs must be {self.input_bytes} bytes on the host")
            self._done.synchronize()
            self.host_in.copy_(host_inputs)
        if timed:
            if self._graph_marked is None:
                self.marks = (torch.cuda.Event(enable_timing=True, external=True),
                              torch.cuda.Event(enable_timing=True, external=True))
                self._graph_marked = self._capture(self.marks)
            self._graph_marked.replay()
        else:
            self.graph.replay()
        self._done.record(torch.cuda.current_stream(self.device))
        return self.host_out

    def ready(self) -> bool:
        """Whether the last step has finished (host_in may be refilled)."""
        return self._done.query()

    @property
    def topk_idx(self) -> torch.Tensor | None:
        """The last step's selected entries [n, k] (CSA layers)."""
        if not self.csa:
            return None
        if self.fused_select:
            return self._idx
        off = self._step_dev_offsets()["idx"]
        return self._dev_buf[off: off + self.n * self.k * 4].view(torch.int32).view(self.n, self.k)

    def _step_dev_offsets(self) -> dict:
        """Byte offsets in the C step's device scratch (csa_decode_step's
        layout: the inputs, scores [n][ld], counts [n], indices [n][k], the
        attention workspace, the output; each on a 256-byte boundary)."""
        al = lambda x: (x + 255) // 256 * 256
        c = self.cache
        o = self.input_bytes
        ld = max(c.cfg.max_pages_per_request * 128, 128) if self.csa else 0
        o += al(self.n * ld * 4)                 # scores
        o += al(self.n * 4)                      # counts
        return {"idx": o}


# ---------------------------------------------------------------- host row formats

def pack_kv_rows(fp8: np.ndarray, rope_bf16_bits: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """Packed host rows for REGION_KV / REGION_WINDOW: codes | BF16 | fp32 scale."""
    n = fp8.shape[0]
    return np.concatenate([fp8.astype(np.uint8).reshape(n, -1),
                           np.ascontiguousarray(rope_bf16_bits.astype(np.uint16)).view(np.uint8).reshape(n, -1),
                           np.ascontiguousarray(scale.astype(np.float32)).view(np.uint8).reshape(n, 4)], axis=1)


def unpack_kv_rows(rows: np.ndarray, D: int, R: int):
    fp8 = rows[:, : D - R].copy()
    bf = np.ascontiguousarray(rows[:, D - R: D - R + 2 * R]).view(np.uint16).reshape(-1, R)
    sc = np.ascontiguousarray(rows[:, D + R: D + R + 4]).view(np.float32).reshape(-1)
    return fp8, bf, sc


def pack_index_rows(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Packed host rows for REGION_INDEX: E2M1 pairs (element 2i low nibble) | E8M0."""
    c = codes.astype(np.uint8)
    packed = (c[:, 0::2] & 0xF) | ((c[:, 1::2] & 0xF) << 4)
    return np.concatenate([packed.astype(np.uint8), scales.astype(np.uint8)], axis=1)


def unpack_index_rows(rows: np.ndarray, d_I: int):
    packed = rows[:, : d_I // 2]
    codes = np.empty((rows.shape[0], d_I), dtype=np.uint8)
    codes[:, 0::2] = packed & 0xF
    codes[:, 1::2] = packed >> 4
    return codes, rows[:, d_I // 2:].copy()


# ---------------------------------------------------------------- batch-invariant projection GEMM

def bf16_bits(a) -> np.ndarray:
    """BF16 bit patterns (uint16) of a host array (torch's round-to-nearest-even cast)."""
    t = torch.from_numpy(np.ascontiguousarray(np.asarray(a, dtype=np.float32)))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


class Linear:
    """A BF16 weight packed once for the batch-invariant projection GEMM
    (csa_gemm_bf16): Y[t][o] = sum_k X[t][k] W[o][k], fp32 accumulation.

    w: host array [n_out][k_in // groups] (BF16 bit patterns as uint16, or
    real values, rounded to BF16 here).  With groups > 1 the weight is block
    diagonal: group g's rows (n_out / groups, a multiple of 128) read the
    columns [g k_in / groups, (g + 1) k_in / groups) of X."""

    def __init__(self, w, groups: int = 1, device: str | torch.device = "cuda"):
        self.lib = _lib.load()
        w = np.ascontiguousarray(w)
        if w.dtype != np.uint16:
            w = bf16_bits(w)
        self.n_out, kg = w.shape
        self.groups = int(groups)
        self.k_in = kg * self.groups
        nbytes = self.lib.csa_gemm_weight_bytes(self.n_out, self.k_in, self.groups)
        if nbytes == 0:
            raise ValueError("invalid GEMM weight shape")
        self.packed = torch.empty(nbytes, dtype=torch.uint8, device=device)
        check(self.lib.csa_gemm_pack_weight(w.ctypes.data, self.n_out, self.k_in, self.groups,
                                            self.packed.data_ptr(), nbytes), "csa_gemm_pack_weight")
        self._ws = None

    def workspace_bytes(self, n_tok: int) -> int:
        return int(self.lib.csa_gemm_workspace_bytes(self.n_out, self.k_in, self.groups, n_tok))

    MAX_TOKENS = 256        # tokens per csa_gemm_bf16 call

    def __call__(self, x: torch.Tensor, outs, workspace: torch.Tensor | None = None, stream=None):
        """x: CUDA BF16 [n_tok][k_in].  outs: one tensor or a list of CUDA
        tensors [n_tok][rows_s] (BF16 or fp32, contiguous) whose rows add up
        to n_out: rows [r_s, r_s + rows_s) of Y go to outs[s].  More than
        MAX_TOKENS tokens are projected in consecutive calls of MAX_TOKENS
        (a token's result does not depend on its batch).  Returns outs."""
        single = isinstance(outs, torch.Tensor)
        segs = [outs] if single else list(outs)
        n = x.shape[0] if x.dim() == 2 else -1
        _need(x, torch.bfloat16, (n, self.k_in), "x")
        for s, t in enumerate(segs):
            if t.dtype not in (torch.bfloat16, torch.float32):
                raise ValueError("outputs must be BF16 or fp32")
            _need(t, t.dtype, (n, t.shape[1] if t.dim() == 2 else -1), f"outs[{s}]")
        for t0 in range(0, max(n, 1), self.MAX_TOKENS):
            t1 = min(t0 + self.MAX_TOKENS, n)
            self._call(x[t0:t1], [t[t0:t1] for t in segs], t1 - t0, workspace, stream)
        return outs

    def _call(self, x, segs, n, workspace, stream):
        arr = (_lib.GemmOut * len(segs))()
        for s, t in enumerate(segs):
            arr[s] = _lib.GemmOut(t.shape[1], 1 if t.dtype == torch.bfloat16 else 0, t.data_ptr())
        need = self.workspace_bytes(n) if n > 0 else 0
        if workspace is None:
            if self._ws is None or self._ws.numel() < need + 256 or self._ws.device != x.device:
                self._ws = torch.empty(need + 256, dtype=torch.uint8, device=x.device)
            workspace = self._ws
        ws_ptr = (workspace.data_ptr() + 255) // 256 * 256
        ws_bytes = workspace.numel() - (ws_ptr - workspace.data_ptr())
        check(self.lib.csa_gemm_bf16(self.packed.data_ptr(), self.n_out, self.k_in, self.groups, _ptr(x), n,
                                     len(segs), arr, ws_ptr, ws_bytes, _stream(stream)), "csa_gemm_bf16")

    @staticmethod
    def check_device_error(stream=None) -> None:
        check(_lib.load().csa_gemm_check_device_error(_stream(stream)), "gemm device")


class LayerProjections:
    """The projections that feed one layer's decode step, from the token's
    hidden state h (BF16 [n, d]) through the batch-invariant GEMM:

      first call, one fused weight [W_c; W_z; (W_cI; W_zI; W_w;) W_dq]:
        c, z [n, 1, D] fp32 (compressor candidate and gate logits),
        on a CSA layer c_I, z_I [n, 1, d_I] and w [n, H_I] fp32,
        c_q [n, d_c] BF16 (the query latent);
      second call, [W_uq; (W_uqI)] on c_q:
        q [n, H, D] BF16 (before RoPE), on a CSA layer q_I [n, H_I, d_I] fp32.

    Weights are host arrays [out, in] (rounded to BF16 when packed)."""

    def __init__(self, *, csa: bool, W_c, W_z, W_dq, W_uq, W_cI=None, W_zI=None, W_w=None, W_uqI=None,
                 device: str | torch.device = "cuda"):
        self.csa = bool(csa)
        self.D = W_c.shape[0]
        self.d = W_c.shape[1]
        self.d_c = W_dq.shape[0]
        first = [W_c, W_z] + ([W_cI, W_zI, W_w] if csa else []) + [W_dq]
        self.rows1 = [int(w.shape[0]) for w in first]
        self.W1 = Linear(np.concatenate([np.asarray(w, np.float32) for w in first]), device=device)
        second = [W_uq] + ([W_uqI] if csa else [])
        self.rows2 = [int(w.shape[0]) for w in second]
        self.W2 = Linear(np.concatenate([np.asarray(w, np.float32) for w in second]), device=device)
        self.d_I = int(W_cI.shape[0]) if csa else 0
        self.H_I = int(W_w.shape[0]) if csa else 0
        self.HD = int(W_uq.shape[0])

    def new_outputs(self, n: int, H: int, device="cuda") -> dict:
        f32, bf = torch.float32, torch.bfloat16
        o = {"c": torch.empty((n, 1, self.D), dtype=f32, device=device),
             "z": torch.empty((n, 1, self.D), dtype=f32, device=device),
             "c_q": torch.empty((n, self.d_c), dtype=bf, device=device),
             "q": torch.empty((n, H, self.HD // H), dtype=bf, device=device)}
        if self.csa:
            o.update(ci=torch.empty((n, 1, self.d_I), dtype=f32, device=device),
                     zi=torch.empty((n, 1, self.d_I), dtype=f32, device=device),
                     w=torch.empty((n, self.H_I), dtype=f32, device=device),
                     q_idx=torch.empty((n, self.H_I, self.rows2[1] // self.H_I), dtype=f32, device=device))
        return o

    def __call__(self, h: torch.Tensor, outs: dict, stream=None) -> dict:
        n = h.shape[0]
        seg1 = [outs["c"].view(n, -1), outs["z"].view(n, -1)]
        if self.csa:
            seg1 += [outs["ci"].view(n, -1), outs["zi"].view(n, -1), outs["w"]]
        seg1.append(outs["c_q"])
        self.W1(h, seg1, stream=stream)
        seg2 = [outs["q"].view(n, -1)] + ([outs["q_idx"].view(n, -1)] if self.csa else [])
        self.W2(outs["c_q"], seg2, stream=stream)
        return outs


class OutputProjection:
    """The grouped output projection after the attention: the H heads x D
    output (BF16 [n, H, D]) is projected per group of H / groups heads by a
    block-diagonal weight W_g [groups * d_g, (H / groups) * D] to a BF16
    intermediate [n, groups * d_g], then to the model width by W_o
    [d_model, groups * d_g] (fp32 output [n, d_model])."""

    def __init__(self, W_g, W_o, groups: int, device: str | torch.device = "cuda"):
        self.groups = int(groups)
        self.Wg = Linear(W_g, groups=self.groups, device=device)
        self.Wo = Linear(W_o, device=device)

    def __call__(self, attn_out: torch.Tensor, mid: torch.Tensor, out: torch.Tensor, stream=None) -> torch.Tensor:
        n = attn_out.shape[0]
        self.Wg(attn_out.view(n, -1), mid, stream=stream)
        self.Wo(mid, out, stream=stream)
        return out
