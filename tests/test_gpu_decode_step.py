"""DecodeStep: the decode step captured as one CUDA graph, fed from one packed
pinned host buffer.  Its results must be bit-identical to the same step run
through the individual calls (compress_append, index_scores, topk,
decode_attn) on a second cache filled identically, step after step, while
entries (every 4th token) and HCA blocks (every 128th) complete; the last
step is also checked against the oracle."""
import numpy as np
import pytest

from compressed_sparse_long_hca_b200 import inputs as I
from oracle import csa_oracle as O
from tests import helpers as Hp

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_lib):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return cuda_lib


def _eager(pair, layer, reqs, k, sink, v):
    """The same step through the individual calls; returns (out, idx)."""
    from compressed_sparse_long_hca_b200.api import topk
    cache, wl = pair.cache, pair.wl
    n = len(reqs)
    rid = torch.tensor(reqs, dtype=torch.int32, device="cuda")
    dv = {name: t.cuda() for name, t in v.items()}
    csa = layer < pair.n_csa
    cache.compress_append(layer, rid, dv["c"], dv["z"], dv.get("ci"), dv.get("zi"))
    out = torch.empty((n, wl.H, wl.D), dtype=torch.bfloat16, device="cuda")
    idx = None
    if csa:
        ld = max(cache.get_length(layer, r) for r in reqs) // 4 + 1
        scores = torch.empty((n, ld), device="cuda")
        nv = torch.empty(n, dtype=torch.int32, device="cuda")
        cache.index_scores(layer, rid, dv["q_idx"], dv["w"], scores, nv)
        idx = torch.empty((n, k), dtype=torch.int32, device="cuda")
        topk(scores, nv, k, idx)
    cache.decode_attn(layer, rid, dv["q"], idx, torch.from_numpy(sink).cuda(), out)
    cache.check_device_error()
    return out.cpu(), (idx.cpu() if idx is not None else None)


@pytest.mark.parametrize("layer,fused", [(0, False), (1, False), (0, True)])
def test_decode_step_graph_matches_individual_calls(layer, fused):
    """fused=False: the graph of one csa_decode_step call (host buffers);
    fused=True: the step composed from csa_compress_append, csa_index_topk
    and csa_hca_decode_attn."""
    from compressed_sparse_long_hca_b200.api import DecodeStep
    wl = I.Workload("step", "csa", H=16, D=128, R=32, H_I=8, d_I=64, k=40, W=128, context=0, batch=0,
                    seed=4242)
    lens = [701, 2045, 125]          # HCA blocks complete at 2048 and 128 during the steps
    reqs = [2, 0, 1]                 # batch order differs from request order
    n_steps = 6
    pairs = [Hp.Pair(wl, 1, 1, max_req=3, capacity=max(lens) + 64) for _ in range(2)]
    for pair in pairs:
        for r, T in enumerate(lens):
            pair.cache.request_alloc(r, T + 64)
            pair.append(layer, [r], {r: pair.gen_tokens(layer, r, 0, T)}, T, oracle=pair is pairs[0])
    torch.cuda.synchronize()
    csa = layer == 0
    sink = pairs[0].params[layer]["sink"]
    step = DecodeStep(pairs[0].cache, layer, reqs, wl.k if csa else 0, sink, fused_select=fused)
    rng = np.random.default_rng(17)
    for s in range(n_steps):
        # even steps: a caller's own pinned buffer (copied into the step's on
        # the host); odd steps: the step's own buffer, filled in place, and
        # the replay that records the phase marks
        own = s % 2 == 1
        buf = step.host_in if own else step.new_host_inputs()
        v = step.views(buf)
        q = I.bf16_grid(rng.standard_normal((3, wl.H, wl.D)).astype(np.float32))
        v["q"].copy_(torch.from_numpy(q).to(torch.bfloat16))
        toks = {r: pairs[0].gen_tokens(layer, r, lens[r] + s, 1) for r in reqs}
        v["c"].copy_(torch.from_numpy(np.stack([toks[r][0] for r in reqs])))
        v["z"].copy_(torch.from_numpy(np.stack([toks[r][1] for r in reqs])))
        if csa:
            v["ci"].copy_(torch.from_numpy(np.stack([toks[r][2] for r in reqs])))
            v["zi"].copy_(torch.from_numpy(np.stack([toks[r][3] for r in reqs])))
            v["q_idx"].copy_(torch.from_numpy(rng.standard_normal((3, wl.H_I, wl.d_I)).astype(np.float32)))
            v["w"].copy_(torch.from_numpy(rng.standard_normal((3, wl.H_I)).astype(np.float32)))
        got = step(None, timed=True) if own else step(buf)
        torch.cuda.synchronize()
        if own:
            assert step.marks[0].elapsed_time(step.marks[1]) > 0
        got_idx = step.topk_idx.cpu() if csa else None
        pairs[0].cache.check_device_error()
        got = got.clone()
        ref, ref_idx = _eager(pairs[1], layer, reqs, wl.k, sink, {nm: t.clone() for nm, t in v.items()})
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16)), f"step {s}: output differs"
        if csa:
            assert torch.equal(got_idx, ref_idx), f"step {s}: top-k differs"
        for r in reqs:
            assert pairs[0].cache.get_length(layer, r) == lens[r] + s + 1
            st = pairs[0].states[(layer, r)]
            cc, zz, cci, zzi = toks[r]
            O.append_tokens(st, cc, zz, cci if csa else None, zzi if csa else None)
    # the last step against the oracle
    p = pairs[0].oracle_params(layer)
    for i, r in enumerate(reqs):
        st = pairs[0].states[(layer, r)]
        t = st.T - 1
        if csa:
            res = O.decode_query(p, st, q[i], sink, k=wl.k, q_idx=v["q_idx"][i].numpy(), w=v["w"][i].numpy())
            N = st.T // 4
            Hp.check_topk(got_idx[i].numpy(), res["scores"], wl.k, N, what=f"request {r}")
            sel = got_idx[i].numpy()
        else:
            res = O.decode_query(p, st, q[i], sink)
            sel = np.arange(st.T // 128)
        # the attention over the rows the GPU selected and stored, always
        Hp.check_attention(got[i].float().numpy(),
                           Hp.attention_over_stored_rows(pairs[0].cache, layer, r, t, sel, q[i], sink, wl.D, wl.R),
                           f"request {r} (stored rows)")
        if not csa or set(sel.tolist()) == set(res["topk"].tolist()):
            # and end to end against the oracle's own rows (a tie-zone swap
            # changes the rows legitimately, which the check above covers)
            Hp.check_attention(got[i].float().numpy(), res["out"], f"request {r}")


def test_decode_step_rejects_mis_sized_or_device_inputs():
    from compressed_sparse_long_hca_b200.api import DecodeStep
    wl = I.Workload("step-args", "hca", H=8, D=64, R=16, H_I=0, d_I=0, k=0, W=128, context=0, batch=0,
                    seed=4243)
    pair = Hp.Pair(wl, 0, 1, max_req=1, capacity=256)
    pair.cache.request_alloc(0, 256)
    step = DecodeStep(pair.cache, 0, [0], 0, pair.params[0]["sink"])
    with pytest.raises(ValueError):
        step(torch.zeros(step.input_bytes, dtype=torch.uint8, device="cuda"))   # not a host buffer
    with pytest.raises(ValueError):
        step(torch.zeros(step.input_bytes + 16, dtype=torch.uint8).pin_memory())
    step(torch.zeros(step.input_bytes, dtype=torch.uint8))                    # pageable: copied on the host
    torch.cuda.synchronize()
    with pytest.raises(ValueError):
        DecodeStep(pair.cache, 0, [], 0, pair.params[0]["sink"])


@pytest.mark.parametrize("layer", [0, 1])
def test_c_decode_step_pageable_and_pinned_buffers_agree(layer):
    """csa_decode_step called through the C ABI: with page-locked host
    buffers the step's kernels read the inputs and write the output over the
    bus directly; with pageable host memory (numpy arrays) it copies them
    through the copy engine.  Both, on two caches filled identically, give
    the same bits, step after step."""
    from compressed_sparse_long_hca_b200 import _lib
    from compressed_sparse_long_hca_b200.api import decode_step_fields
    lib = _lib.load()
    wl = I.Workload("step-c", "csa", H=16, D=128, R=32, H_I=8, d_I=64, k=40, W=128, context=0, batch=0,
                    seed=4343)
    lens = [900, 131]
    reqs = [1, 0]
    pairs = [Hp.Pair(wl, 1, 1, max_req=2, capacity=max(lens) + 64) for _ in range(2)]
    for pair in pairs:
        for r, T in enumerate(lens):
            pair.cache.request_alloc(r, T + 64)
            pair.append(layer, [r], {r: pair.gen_tokens(layer, r, 0, T)}, T, oracle=False)
    torch.cuda.synchronize()
    csa = layer == 0
    k = wl.k if csa else 0
    sink = torch.from_numpy(pairs[0].params[layer]["sink"]).cuda()
    rid = torch.tensor(reqs, dtype=torch.int32, device="cuda")
    fields, in_bytes = decode_step_fields(2, wl.H, wl.D, wl.H_I, wl.d_I, csa)
    assert lib.csa_decode_step_input_bytes(pairs[0].cache.handle, layer, 2) == in_bytes
    dev_bytes = lib.csa_decode_step_dev_bytes(pairs[0].cache.handle, layer, 2, k)
    bufs = [torch.zeros(dev_bytes, dtype=torch.uint8, device="cuda") for _ in range(2)]
    pinned_in = torch.zeros(in_bytes, dtype=torch.uint8).pin_memory()
    pinned_out = torch.zeros((2, wl.H, wl.D), dtype=torch.bfloat16).pin_memory()
    page_in = np.zeros(in_bytes, dtype=np.uint8)
    page_out = np.zeros(2 * wl.H * wl.D, dtype=np.uint16)
    rng = np.random.default_rng(29)
    scale = 1.0 / float(np.sqrt(wl.D))
    stream = torch.cuda.current_stream().cuda_stream
    for s in range(4):
        page_in[:] = rng.integers(0, 256, in_bytes, dtype=np.uint8)
        # sane values: fp32 fields from N(0, 1), the bf16 q from the bf16 grid
        for name, dtype, shape, off, nbytes in fields:
            if dtype == torch.float32:
                page_in[off: off + nbytes] = rng.standard_normal(nbytes // 4).astype(np.float32).view(np.uint8)
            else:
                q = I.bf16_grid(rng.standard_normal(nbytes // 2).astype(np.float32))
                page_in[off: off + nbytes] = torch.from_numpy(q).to(torch.bfloat16).view(torch.uint8).numpy()
        pinned_in.copy_(torch.from_numpy(page_in))
        st = lib.csa_decode_step(pairs[0].cache.handle, layer, 2, rid.data_ptr(), k, sink.data_ptr(), scale,
                                 pinned_in.data_ptr(), pinned_out.data_ptr(), bufs[0].data_ptr(), dev_bytes, stream)
        assert st == 0, _lib.load().csa_last_error()
        st = lib.csa_decode_step(pairs[1].cache.handle, layer, 2, rid.data_ptr(), k, sink.data_ptr(), scale,
                                 page_in.ctypes.data, page_out.ctypes.data, bufs[1].data_ptr(), dev_bytes, stream)
        assert st == 0, _lib.load().csa_last_error()
        torch.cuda.synchronize()
        pairs[0].cache.check_device_error()
        pairs[1].cache.check_device_error()
        assert np.array_equal(pinned_out.view(torch.int16).numpy().reshape(-1).view(np.uint16), page_out), \
            f"step {s}: output differs"
        assert np.any(page_out != 0)
