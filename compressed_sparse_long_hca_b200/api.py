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

    def attn_workspace_bytes(self, layer: int, n: int, k: int = 0) -> int:
        return int(self.lib.csa_attn_workspace_bytes(self.handle, layer, n, k))

    def _workspace(self, nbytes: int, device) -> torch.Tensor:
        ws = getattr(self, "_ws", None)
        if ws is None or ws.numel() < nbytes or ws.device != device:
            ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)
            self._ws = ws
        return ws

    def decode_attn(self, layer: int, req_ids, q, topk_idx, sink, out, scale=None,
                    variant="auto", stream=None, workspace: torch.Tensor | None = None) -> None:
        """Attention of each query over its rows.  The split (low-occupancy)
        launch needs scratch; unless `workspace` is given, a buffer owned by
        this Cache object is grown to the size the library asks for."""
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
        check(self.lib.csa_hca_decode_attn(self.handle, layer, n, _ptr(req_ids), _ptr(q), _ptr(topk_idx),
                                           k, _ptr(sink), scale, _ptr(out), ws_ptr, ws_bytes,
                                           VARIANTS[variant], _stream(stream)), "csa_hca_decode_attn")

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
    once as two CUDA graphs and replayed every step.

    The step appends each request's new token (csa_compress_append), then on
    a CSA layer scores the index keys (csa_index_scores) and selects the top
    k (csa_topk) -- the first graph -- and attends (csa_hca_decode_attn) --
    the second graph; on an HCA layer the first graph only appends and the
    attention covers every compressed entry.

    Inputs of a step, packed in a buffer from `new_host_inputs()` and filled
    through `views(buf)`: c and z [n, 1, D] fp32 (the token's KV candidate
    and gate logits), on a CSA layer also ci and zi [n, 1, d_I] fp32, q_idx
    [n, H_I, d_I] fp32 and w [n, H_I] fp32, and last q [n, H, D] bf16.  Each
    field starts on a 256-byte boundary.

    Host transfers: the fields before q travel in one copy on the caller's
    stream ahead of the first graph; q, which only the attention reads,
    travels in one copy on a side stream while the first graph runs, and the
    second graph waits for it; the output returns in one copy.

    The graphs hold device pointers, so the batch (req_ids), k and the sink
    logits are fixed at construction.  On a CSA layer construction runs the
    index and top-k kernels once (they change nothing in the cache) so that
    their one-time launch set-up happens before the capture."""

    def __init__(self, cache: Cache, layer: int, req_ids, k: int, sink, variant: str = "auto",
                 device: str | torch.device = "cuda"):
        self.cache, self.layer, self.k, self.variant = cache, layer, int(k), variant
        self.csa = layer < cache.n_csa
        ids = [int(r) for r in req_ids]
        n = self.n = len(ids)
        if n == 0:
            raise ValueError("a decode step needs at least one request")
        if self.csa and self.k <= 0:
            raise ValueError("a CSA layer needs k > 0")
        H, D = cache.H, cache.D
        self._fields, off = decode_step_fields(n, H, D, cache.H_I, cache.d_I, self.csa, qdtype=cache.qdtype)
        self.input_bytes = off
        self._q_off = next(f[3] for f in self._fields if f[0] == "q")
        dev = self.device = torch.device(device)
        self._dev_in = torch.zeros(off, dtype=torch.uint8, device=dev)
        d = self.views(self._dev_in)
        self._req = torch.tensor(ids, dtype=torch.int32, device=dev)
        self._sink = (sink if isinstance(sink, torch.Tensor) else torch.from_numpy(np.asarray(sink, np.float32)))
        self._sink = self._sink.to(device=dev, dtype=torch.float32).contiguous()
        self.out = torch.empty((n, H, D), dtype=cache.qdtype, device=dev)
        self.host_out = torch.empty((n, H, D), dtype=cache.qdtype).pin_memory()
        self._ws = torch.empty(max(cache.attn_workspace_bytes(layer, n, self.k if self.csa else 0), 16),
                               dtype=torch.uint8, device=dev)
        self._side = torch.cuda.Stream(device=dev)
        self._ev_start, self._ev_q = torch.cuda.Event(), torch.cuda.Event()
        if self.csa:
            n_max = max(cache.cfg.max_pages_per_request * 128, 128)   # 512 tokens = 128 entries per page
            self._scores = torch.empty((n, n_max), dtype=torch.float32, device=dev)
            self._nv = torch.empty(n, dtype=torch.int32, device=dev)
            self._idx = torch.empty((n, self.k), dtype=torch.int32, device=dev)

        def select():
            cache.index_scores(layer, self._req, d["q_idx"], d["w"], self._scores, self._nv, variant)
            topk(self._scores, self._nv, self.k, self._idx, variant)

        if self.csa:
            # one eager pass of the selection kernels (valid on any cache
            # state, an empty request included) does their one-time launch
            # set-up (cluster-size query) outside the capture
            select()
            torch.cuda.synchronize(dev)
            cache.check_device_error()
        self.graph_select = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph_select):
            cache.compress_append(layer, self._req, d["c"], d["z"], d.get("ci"), d.get("zi"))
            if self.csa:
                select()
        self.graph_attn = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph_attn):
            cache.decode_attn(layer, self._req, d["q"], self._idx if self.csa else None, self._sink, self.out,
                              variant=variant, workspace=self._ws)
        torch.cuda.synchronize(dev)

    def views(self, buf: torch.Tensor) -> dict:
        """Typed views of the step's input fields inside a packed buffer."""
        if buf.dtype != torch.uint8 or buf.numel() < self.input_bytes or not buf.is_contiguous():
            raise ValueError(f"a packed input buffer is {self.input_bytes} contiguous bytes")
        return {name: buf[off: off + nbytes].view(dtype).view(shape)
                for name, dtype, shape, off, nbytes in self._fields}

    def new_host_inputs(self) -> torch.Tensor:
        """A pinned host buffer for one step's packed inputs."""
        return torch.zeros(self.input_bytes, dtype=torch.uint8).pin_memory()

    def __call__(self, host_inputs: torch.Tensor, marks=None) -> torch.Tensor:
        """Enqueue one step on the current stream: copy the packed inputs in,
        replay the step, copy the output [n, H, D] bf16 to `host_out` (pinned),
        which is returned and is valid once the stream has reached this point
        (the next call overwrites it).  The copies are asynchronous:
        `host_inputs` must not change until the stream has passed them.
        `marks`, two torch.cuda.Events, are recorded on the current stream
        after the first input copy and after the second graph (to time the
        three phases; the query's copy overlaps the first graph)."""
        if host_inputs.device.type != "cpu" or not host_inputs.is_pinned():
            raise ValueError("host_inputs must be a pinned host buffer (new_host_inputs())")
        if host_inputs.dtype != torch.uint8 or host_inputs.numel() != self.input_bytes:
            raise ValueError(f"host_inputs must be {self.input_bytes} bytes")
        main = torch.cuda.current_stream(self.device)
        qo = self._q_off
        # the query's copy starts once everything queued before this step
        # (the previous step's attention reads the same buffer) has run
        self._ev_start.record(main)
        self._side.wait_event(self._ev_start)
        with torch.cuda.stream(self._side):
            self._dev_in[qo:].copy_(host_inputs[qo:], non_blocking=True)
            self._ev_q.record(self._side)
        self._dev_in[:qo].copy_(host_inputs[:qo], non_blocking=True)
        if marks is not None:
            marks[0].record(main)
        self.graph_select.replay()
        main.wait_event(self._ev_q)
        self.graph_attn.replay()
        if marks is not None:
            marks[1].record(main)
        self.host_out.copy_(self.out, non_blocking=True)
        return self.host_out

    @property
    def topk_idx(self) -> torch.Tensor | None:
        """The last step's selected entries [n, k] (CSA layers)."""
        return self._idx if self.csa else None


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
