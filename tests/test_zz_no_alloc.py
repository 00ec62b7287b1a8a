"""csa_hca_decode_attn_noalloc: attention for callers that cannot allocate
device memory (an engine whose memory planner owns every device buffer, a
plugin that only receives device pointers).  It keeps its scratch in an array
built into the library; its results must match csa_hca_decode_attn's.

Called through the C ABI twice in a row on different queries, so the second
call runs over whatever the first left in the shared array."""
import ctypes
import math

import numpy as np
import pytest

from compressed_sparse_long_hca_b200 import _lib
from compressed_sparse_long_hca_b200 import inputs as I
from compressed_sparse_long_hca_b200.api import pack_kv_rows
from oracle import csa_oracle as O
from tests import helpers as Hp

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _lib_built(cuda_lib):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return cuda_lib


def _t(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t.to(dtype) if dtype is not None else t


def _fill(pair, layer, req, T, rng, csa):
    wl = pair.wl
    N = T // 4 if csa else T // 128
    pair.cache.set_length(layer, req, T)
    ent = O.quantize_kv(rng.standard_normal((N, wl.D)) * 0.5, wl.R)
    pair.cache.write_rows(layer, req, 0, 0, pack_kv_rows(ent.fp8, ent.rope, ent.scale))
    wp = O.window_positions(T - 1)
    win = O.quantize_kv(rng.standard_normal((len(wp), wl.D)), wl.R)
    pair.cache.write_rows(layer, req, 2, wp[0], pack_kv_rows(win.fp8, win.rope, win.scale))
    return N


def _noalloc(pair, layer, rid, q, idx, k, sink, out):
    lib = _lib.load()
    st = lib.csa_hca_decode_attn_noalloc(pair.cache.handle, layer, rid.numel(), rid.data_ptr(), q.data_ptr(),
                                         idx.data_ptr() if idx is not None else None, k, sink.data_ptr(),
                                         1.0 / math.sqrt(pair.wl.D), out.data_ptr(),
                                         torch.cuda.current_stream().cuda_stream or None)
    return st


def test_noalloc_matches_workspace_entry_point_twice():
    wl = I.Workload("noalloc", "csa", H=64, D=512, R=64, H_I=4, d_I=32, k=300, W=128, context=0,
                    batch=0, seed=777)
    lens = [2000, 9001, 130]
    n = len(lens)
    pair = Hp.Pair(wl, 1, 1, max_req=n, capacity=max(lens) + 8)
    rng = np.random.default_rng(5)
    for i, T in enumerate(lens):
        pair.cache.request_alloc(i, T + 8)
    for layer in (0, 1):
        csa = layer == 0
        sink = _t(pair.params[layer]["sink"])
        sels = np.full((n, wl.k), -1, np.int32)
        for i, T in enumerate(lens):
            N = _fill(pair, layer, i, T, rng, csa)
            if csa:
                pick = np.sort(rng.choice(N, size=min(N, wl.k), replace=False))
                sels[i, : len(pick)] = pick
        rid = _t(np.arange(n, dtype=np.int32))
        idx = _t(sels) if csa else None
        for call in range(2):
            q = _t(I.bf16_grid(rng.standard_normal((n, wl.H, wl.D)).astype(np.float32)), torch.bfloat16)
            ref = torch.empty((n, wl.H, wl.D), dtype=torch.bfloat16, device="cuda")
            pair.cache.decode_attn(layer, rid, q, idx, sink, ref)
            got = torch.full((n, wl.H, wl.D), float("nan"), dtype=torch.bfloat16, device="cuda")
            st = _noalloc(pair, layer, rid, q, idx, wl.k if csa else 0, sink, got)
            assert st == _lib.CSA_OK, _lib.load().csa_last_error()
            pair.cache.check_device_error()
            g, r = got.float().cpu().numpy(), ref.float().cpu().numpy()
            for i in range(n):
                Hp.check_attention(g[i], r[i], f"layer {layer} call {call} query {i}")
            assert np.array_equal(g, r), f"layer {layer} call {call}: differs from csa_hca_decode_attn"


def test_noalloc_rejects_batches_beyond_its_scratch():
    wl = I.Workload("noalloc-big", "csa", H=128, D=512, R=64, H_I=4, d_I=32, k=8192, W=128, context=0,
                    batch=0, seed=778)
    pair = Hp.Pair(wl, 1, 0, max_req=2, capacity=600)
    n = 8
    need = pair.cache.attn_workspace_bytes(0, n, wl.k)
    assert need > 16 << 20
    rid = torch.zeros(n, dtype=torch.int32, device="cuda")
    q = torch.zeros((n, wl.H, wl.D), dtype=torch.bfloat16, device="cuda")
    idx = torch.full((n, wl.k), -1, dtype=torch.int32, device="cuda")
    sink = torch.zeros(wl.H, device="cuda")
    out = torch.zeros((n, wl.H, wl.D), dtype=torch.bfloat16, device="cuda")
    st = _noalloc(pair, 0, rid, q, idx, wl.k, sink, out)
    assert st == -2, "expected CSA_ERR_CAPACITY"
    assert b"scratch" in _lib.load().csa_last_error()


def test_noalloc_hca_limit_follows_the_cache_capacity():
    """On an HCA layer a query's tiles are cut into chunks of
    max(1, tiles / 8), at most 15 chunks for any length, one partial each,
    so at H = 128, D = 512 the scratch fits 4 queries and not 5 whatever the
    cache's capacity (2048 pages = 1M tokens, or 16,128); a batch that does
    not fit is refused before any launch."""
    wl = I.Workload("noalloc-hca", "hca", H=128, D=512, R=64, H_I=0, d_I=0, k=0, W=128, context=0,
                    batch=0, seed=779)
    sink = torch.zeros(wl.H, device="cuda")
    for pages, n, expect in ((2048, 4, True), (2048, 5, False), (16128, 4, True), (16128, 5, False)):
        pair = Hp.Pair(wl, 0, 1, max_req=1, capacity=pages * 512)
        fits = pair.cache.attn_workspace_bytes(0, n, 0) <= 16 << 20
        assert fits == expect, (pages, n, pair.cache.attn_workspace_bytes(0, n, 0))
        if not expect:
            q = torch.zeros((n, wl.H, wl.D), dtype=torch.bfloat16, device="cuda")
            out = torch.zeros((n, wl.H, wl.D), dtype=torch.bfloat16, device="cuda")
            rid = torch.zeros(n, dtype=torch.int32, device="cuda")
            st = _noalloc(pair, 0, rid, q, None, 0, sink, out)
            assert st == -2, "expected CSA_ERR_CAPACITY"
            assert b"scratch" in _lib.load().csa_last_error()
