"""Chunks of queries with causal visibility (csa_prefill_chunk): every token
of a chunk is also a query and sees what a decode query at its position
sees.  The chunk's outputs and top-k lists must be bit-identical to
appending the same tokens one at a time and running the decode calls after
each, on a second cache filled identically (batch invariance), for chunks of
1 .. 128 tokens that start at position 0, cross CSA entries and HCA blocks
and overwrite the window ring, in every launch variant and both storage
formats; a chunk is also checked against the oracle's chunk of queries."""
import numpy as np
import pytest

from compressed_sparse_long_hca_b200 import _lib
from compressed_sparse_long_hca_b200 import inputs as I
from compressed_sparse_long_hca_b200.api import topk
from oracle import csa_oracle as O
from tests import helpers as Hp

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _lib_loaded(cuda_lib):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return cuda_lib


CHUNKS = [1, 37, 128, 5]                 # 171 tokens per request
VARIANTS = ["auto", "low", "high", "auto"]


def _workload(fmt):
    if fmt == "f32":
        return I.Workload("chunk-f32", "csa", H=8, D=64, R=16, H_I=4, d_I=32, k=16, W=128, context=0, batch=0,
                          seed=6161)
    return I.Workload("chunk", "csa", H=16, D=128, R=32, H_I=8, d_I=64, k=40, W=128, context=0, batch=0,
                      seed=6060)


def _queries(wl, n_tok, n_req, seed, fmt):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((n_req, n_tok, wl.H, wl.D)).astype(np.float32)
    if fmt != "f32":
        q = I.bf16_grid(q)
    qi = rng.standard_normal((n_req, n_tok, wl.H_I, wl.d_I)).astype(np.float32)
    w = rng.standard_normal((n_req, n_tok, wl.H_I)).astype(np.float32)
    return q, qi, w


@pytest.mark.parametrize("layer,fmt", [(0, "mixed"), (1, "mixed"), (0, "f32"), (1, "f32")])
def test_chunk_matches_token_by_token_decode(layer, fmt):
    wl = _workload(fmt)
    csa = layer == 0
    lens = [0, 250, 1021]
    reqs = [1, 2, 0]                     # batch order differs from request order
    total = sum(CHUNKS)
    pairs = [Hp.Pair(wl, 1, 1, max_req=3, capacity=max(lens) + total + 64, fmt=fmt) for _ in range(2)]
    for pair in pairs:
        for r, T in enumerate(lens):
            pair.cache.request_alloc(r, T + total + 64)
            if T:
                pair.append(layer, [r], {r: pair.gen_tokens(layer, r, 0, T)}, T, oracle=pair is pairs[0])
    torch.cuda.synchronize()
    qdt = torch.float32 if fmt == "f32" else torch.bfloat16
    sink = pairs[0].params[layer]["sink"]
    sink_d = torch.from_numpy(sink).cuda()
    toks = {r: pairs[0].gen_tokens(layer, r, lens[r], total) for r in reqs}
    q, qi, w = _queries(wl, total, len(reqs), 99 + layer, fmt)
    rid = torch.tensor(reqs, dtype=torch.int32, device="cuda")
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    A, B = pairs[0].cache, pairs[1].cache
    t0 = 0
    last = None
    for n_tok, variant in zip(CHUNKS, VARIANTS):
        sl = slice(t0, t0 + n_tok)
        field = lambda x: dev(np.stack([toks[r][x][sl] for r in reqs]))
        c, z = field(0), field(1)
        ci, zi = (field(2), field(3)) if csa else (None, None)
        qd = dev(q[:, sl]).to(qdt)
        qid, wd = (dev(qi[:, sl]), dev(w[:, sl])) if csa else (None, None)
        out = torch.empty((3, n_tok, wl.H, wl.D), dtype=qdt, device="cuda")
        idx = torch.full((3, n_tok, wl.k), -7, dtype=torch.int32, device="cuda") if csa else None
        A.prefill_chunk(layer, rid, c, z, ci, zi, qd, qid, wd, wl.k, sink_d, out, topk_out=idx, variant=variant)
        torch.cuda.synchronize()
        A.check_device_error()
        got = out.cpu()
        got_idx = idx.cpu() if csa else None
        # the same tokens one at a time through the decode calls
        for j in range(n_tok):
            B.compress_append(layer, rid, c[:, j:j + 1].contiguous(), z[:, j:j + 1].contiguous(),
                              ci[:, j:j + 1].contiguous() if csa else None,
                              zi[:, j:j + 1].contiguous() if csa else None)
            ref_idx = None
            if csa:
                ld = max(B.get_length(layer, r) for r in reqs) // 4 + 1
                scores = torch.empty((3, ld), device="cuda")
                nv = torch.empty(3, dtype=torch.int32, device="cuda")
                B.index_scores(layer, rid, qid[:, j].contiguous(), wd[:, j].contiguous(), scores, nv)
                ref_idx = torch.empty((3, wl.k), dtype=torch.int32, device="cuda")
                topk(scores, nv, wl.k, ref_idx)
            ref = torch.empty((3, wl.H, wl.D), dtype=qdt, device="cuda")
            B.decode_attn(layer, rid, qd[:, j].contiguous(), ref_idx, sink_d, ref)
            torch.cuda.synchronize()
            B.check_device_error()
            bits = torch.int32 if fmt == "f32" else torch.int16
            assert torch.equal(got[:, j].view(bits), ref.cpu().view(bits)), \
                f"chunk of {n_tok} ({variant}), token {j}: output differs"
            if csa:
                assert torch.equal(got_idx[:, j], ref_idx.cpu()), f"chunk of {n_tok}, token {j}: top-k differs"
        for r in reqs:
            assert A.get_length(layer, r) == lens[r] + t0 + n_tok
        last = (sl, got, got_idx)
        t0 += n_tok
    # the last chunk against the oracle's chunk of queries
    sl, got, got_idx = last
    p = pairs[0].oracle_params(layer)
    for b, r in enumerate(reqs):
        st = pairs[0].states.setdefault((layer, r), O.RequestState())
        pre = toks[r]
        O.append_tokens(st, pre[0][:sl.start], pre[1][:sl.start], pre[2][:sl.start] if csa else None,
                        pre[3][:sl.start] if csa else None)
        res = O.chunk_queries(p, st, pre[0][sl], pre[1][sl], pre[2][sl] if csa else None,
                              pre[3][sl] if csa else None, q=q[b, sl], sink=sink, k=wl.k if csa else None,
                              q_idx=qi[b, sl] if csa else None, w=w[b, sl] if csa else None)
        for j, rj in enumerate(res):
            t = lens[r] + sl.start + j
            g = got[b, j].float().numpy()
            if csa:
                Hp.check_topk(got_idx[b, j].numpy(), rj["scores"], wl.k, (t + 1) // 4,
                              what=f"request {r} position {t}")
                same = set(got_idx[b, j].numpy().tolist()) == set(rj["topk"].tolist())
            else:
                same = True
            if same:
                Hp.check_attention(g, rj["out"], f"request {r} position {t}", fmt=fmt)
        # the chunk's last query: its whole window is in the ring, so also
        # the attention over the rows the GPU stored and selected
        t = st.T - 1
        sel = got_idx[b, -1].numpy() if csa else np.arange(st.T // 128)
        Hp.check_attention(got[b, -1].float().numpy(),
                           Hp.attention_over_stored_rows(A, layer, r, t, sel, q[b, sl][-1], sink, wl.D, wl.R),
                           f"request {r} (stored rows)", fmt=fmt)


def test_chunk_rejects_bad_shapes():
    wl = _workload("mixed")
    pair = Hp.Pair(wl, 1, 1, max_req=1, capacity=512)
    A = pair.cache
    A.request_alloc(0, 512)
    lib = _lib.load()
    assert A.prefill_workspace_bytes(0, 1, 129, wl.k) == 0          # more than the window
    assert A.prefill_workspace_bytes(0, 1, 0, wl.k) == 0
    assert A.prefill_workspace_bytes(0, 1, 16, 0) == 0              # CSA needs k
    assert A.prefill_workspace_bytes(1, 1, 16, 0) > 0               # HCA does not
    assert A.prefill_workspace_bytes(0, 600, 128, wl.k) == 0        # n * n_tok > 65535
    rid = torch.zeros(1, dtype=torch.int32, device="cuda")
    n_tok = 4
    c = torch.zeros((1, n_tok, wl.D), device="cuda")
    ci = torch.zeros((1, n_tok, wl.d_I), device="cuda")
    q = torch.zeros((1, n_tok, wl.H, wl.D), dtype=torch.bfloat16, device="cuda")
    qi = torch.zeros((1, n_tok, wl.H_I, wl.d_I), device="cuda")
    w = torch.zeros((1, n_tok, wl.H_I), device="cuda")
    out = torch.empty_like(q)
    sink = torch.zeros(wl.H, device="cuda")
    need = A.prefill_workspace_bytes(0, 1, n_tok, wl.k)
    small = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(_lib.CsaError):
        A.prefill_chunk(0, rid, c, c, ci, ci, q, qi, w, wl.k, sink, out, workspace=small)
    # nothing was launched: the request is still empty
    assert A.get_length(0, 0) == 0
    status = lib.csa_prefill_chunk(A.handle, 0, 1, rid.data_ptr(), 129, c.data_ptr(), c.data_ptr(), ci.data_ptr(),
                                   ci.data_ptr(), q.data_ptr(), qi.data_ptr(), w.data_ptr(), wl.k, sink.data_ptr(),
                                   0.1, out.data_ptr(), None, small.data_ptr(), small.numel(), 0, None)
    assert status == -1
    A.check_device_error()
