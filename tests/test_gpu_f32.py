"""GPU parity of the fp32 storage format (CSA_FMT_F32): the tiny CSA
configuration as its description states it -- fp32 throughout, from hidden
states through the stored rows and keys to the output -- and the fp32
indexer and attention on oracle-written rows across several tiles, ragged
tails, empty rows, both launch variants and other batch compositions."""
import math

import numpy as np
import pytest

from compressed_sparse_long_hca_b200 import inputs as I
from compressed_sparse_long_hca_b200.api import topk
from oracle import csa_oracle as O
from tests import helpers as Hp

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_lib):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return cuda_lib


def _t(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t.to(dtype) if dtype is not None else t


def _c1_weights(seed):
    d = I.C1.hidden
    W = lambda shape, fan, f: I.normal(shape, seed, 99, f).astype(np.float64) / math.sqrt(fan)
    return dict(kv=W((64, d), d, 1), z=W((64, d), d, 2), ik=W((32, d), d, 3), iz=W((32, d), d, 4),
                q=W((8 * 64, d), d, 5), dq=W((64, d), d, 6), uq=W((4 * 32, 64), 64, 7), w=W((4, d), d, 8))


def _read_path(pair, reqs, q, qi, w, sink, k, variant="auto"):
    """Index, top-k and attention for the requests in `reqs` (rows of q, qi,
    w in request order); returns (scores, n_valid, idx, out) in batch order."""
    n = len(reqs)
    rid = _t(np.array(reqs, np.int32))
    ld = max(pair.cache.get_length(0, r) for r in reqs) // 4 + 9
    scores = torch.full((n, ld), float("nan"), device="cuda")
    nv = torch.zeros(n, dtype=torch.int32, device="cuda")
    pair.cache.index_scores(0, rid, _t(qi[reqs]), _t(w[reqs]), scores, nv, variant=variant)
    idx = torch.empty((n, k), dtype=torch.int32, device="cuda")
    topk(scores, nv, k, idx, variant=variant)
    out = torch.empty((n, pair.wl.H, pair.wl.D), dtype=torch.float32, device="cuda")
    pair.cache.decode_attn(0, rid, _t(q[reqs]), idx, _t(sink), out, variant=variant)
    pair.cache.check_device_error()
    return scores.cpu().numpy(), nv.cpu().numpy(), idx.cpu().numpy(), out.cpu().numpy()


def test_c1_fp32_end_to_end_from_hidden_states():
    """Tiny CSA decode in fp32 (hidden 256, 8 heads x 64, RoPE 16, indexer
    4 x 32, top-16, context 1024): hidden states -> projections (fp64, test
    side, rounded to fp32) -> CUDA path with an fp32 cache vs the oracle in
    the fp32 format, stage by stage; both variants and two batch
    compositions give the same bits."""
    wl = I.C1
    Wt = _c1_weights(wl.seed)
    T = wl.context
    h = I.normal((T + 1, wl.hidden), wl.seed, 0, 0, 77).astype(np.float64)
    proj = lambda M: O.f32(h @ M.T)
    c, z, ci, zi = proj(Wt["kv"]), proj(Wt["z"]), proj(Wt["ik"]), proj(Wt["iz"])
    pair = Hp.Pair(wl, 1, 0, max_req=2, capacity=T + 64, fmt="f32")
    pair.cache.request_alloc(1, T + 64)
    pos = 0
    for n_tok in [1, 2, 5, 3, 117, 4, 128, 256, 500, 7, 1]:
        n_tok = min(n_tok, T - pos)
        if n_tok == 0:
            break
        pair.append(0, [1], {1: (c[pos:pos + n_tok], z[pos:pos + n_tok], ci[pos:pos + n_tok],
                                 zi[pos:pos + n_tok])}, n_tok)
        pos += n_tok
    pair.append(0, [1], {1: (c[T:T + 1], z[T:T + 1], ci[T:T + 1], zi[T:T + 1])}, 1)
    # a second request (another context) to vary the batch around request 1
    pair.cache.request_alloc(0, T + 64)
    T0 = 701
    pair.append(0, [0], {0: pair.gen_tokens(0, 0, 0, T0)}, T0)
    hq = h[T]
    q1 = O.f32(Wt["q"] @ hq).reshape(8, 64)
    qi1 = O.f32(Wt["uq"] @ (Wt["dq"] @ hq)).reshape(4, 32)
    w1 = O.f32(Wt["w"] @ hq)
    rng = np.random.default_rng(3)
    q = np.stack([rng.standard_normal((8, 64)).astype(np.float32), q1])
    qi = np.stack([rng.standard_normal((4, 32)).astype(np.float32), qi1])
    w = np.stack([rng.standard_normal(4).astype(np.float32), w1])
    sink = pair.params[0]["sink"]
    s_b, nv_b, idx_b, out_b = _read_path(pair, [1], q, qi, w, sink, wl.k)
    N = (T + 1) // 4
    assert int(nv_b[0]) == N and pair.cache.get_length(0, 1) == T + 1
    # ---- stored rows against the oracle (fp32 pooling vs fp64)
    p = pair.oracle_params(0)
    st = pair.states[(0, 1)]
    kv_ref, key_ref = O.csa_entries_all(np.array(st.c), np.array(st.z), np.array(st.ci),
                                        np.array(st.zi), p.b_kv, p.b_idx, p.R)
    Hp.check_f32_rows(pair.cache.read_rows(0, 1, 0, 0, N), kv_ref, "entries")
    Hp.check_f32_rows(pair.cache.read_rows(0, 1, 1, 0, N), key_ref, "index keys")
    wp = O.window_positions(T)
    win_ref = np.stack([O.raw_token_row(st.c[t], t, wl.R) for t in wp])
    Hp.check_f32_rows(pair.cache.read_rows(0, 1, 2, wp[0], len(wp)), win_ref, "window")
    # ---- scores on the stored keys, top-k, attention
    kd = Hp.f32_rows_value(pair.cache.read_rows(0, 1, 1, 0, N), wl.d_I)
    qd = O.store_f32(qi1)
    ref_s = O.index_scores(qd, w1, kd)
    mag = np.abs(kd @ qd.T) @ np.abs(w1)
    assert np.all(np.abs(s_b[0, :N] - ref_s) <= 1e-5 * mag + 1e-7), "index scores"
    assert np.isnan(s_b[0, N:]).all(), "scores written past N"
    Hp.check_topk(idx_b[0], ref_s, wl.k, N, what="top-k on the stored keys")
    res = O.decode_query(p, st, q1, sink, k=wl.k, q_idx=qi1, w=w1)
    Hp.check_topk(idx_b[0], res["scores"], wl.k, N, what="top-k vs the oracle's own keys")
    Hp.check_attention(out_b[0], Hp.attention_over_stored_rows(pair.cache, 0, 1, T, idx_b[0], q1, sink, 64, 16),
                       "c1 fp32 attention (stored rows)", fmt="f32")
    if set(idx_b[0].tolist()) == set(res["topk"].tolist()):
        Hp.check_attention(out_b[0], res["out"], "c1 fp32 attention", fmt="f32")
    # ---- both variants and other batches: identical bits for request 1
    for reqs, variant in (([0, 1], "high"), ([1, 0], "low"), ([1], "low"), ([0, 1], "auto")):
        s2, nv2, idx2, out2 = _read_path(pair, reqs, q, qi, w, sink, wl.k, variant)
        x = reqs.index(1)
        assert np.array_equal(s2[x, :N].view(np.uint32), s_b[0, :N].view(np.uint32)), (reqs, variant)
        assert np.array_equal(idx2[x], idx_b[0]), (reqs, variant)
        assert np.array_equal(out2[x].view(np.uint32), out_b[0].view(np.uint32)), (reqs, variant)


@pytest.mark.parametrize("H,D,R,HI,dI", [(8, 64, 16, 4, 32), (16, 128, 32, 8, 64)])
def test_f32_index_and_attention_on_written_rows(H, D, R, HI, dI):
    """fp32 rows and keys written from host values (several 128-row tiles,
    ragged tails, a context of one token, -1 holes in the lists): index
    scores, CSA and HCA attention against the oracle; both variants
    bit-identical."""
    wl = I.Workload("f32", "csa", H=H, D=D, R=R, H_I=HI, d_I=dI, k=40, W=128, context=0, batch=0, seed=556)
    lens = [1, 5, 130, 1000, 4000]
    n = len(lens)
    pair = Hp.Pair(wl, 1, 1, max_req=n, capacity=max(lens) + 8, fmt="f32")
    rng = np.random.default_rng(H + D)
    q = rng.standard_normal((n, H, D)).astype(np.float32)
    for layer in (0, 1):
        csa = layer == 0
        sink = pair.params[layer]["sink"]
        ents, wins, keys = [], [], []
        sels = np.full((n, wl.k), -1, np.int32)
        for i, T in enumerate(lens):
            if layer == 0:
                pair.cache.request_alloc(i, T + 8)
            pair.cache.set_length(layer, i, T)
            N = T // 4 if csa else T // 128
            e = rng.standard_normal((N, D)).astype(np.float32) * 0.5
            if N:
                pair.cache.write_rows(layer, i, 0, 0, e.view(np.uint8).reshape(N, -1))
            wp = O.window_positions(T - 1)
            wv = rng.standard_normal((len(wp), D)).astype(np.float32)
            pair.cache.write_rows(layer, i, 2, wp[0], wv.view(np.uint8).reshape(len(wp), -1))
            ents.append(e.astype(np.float64))
            wins.append(wv.astype(np.float64))
            if csa:
                kk = rng.standard_normal((N, dI)).astype(np.float32)
                if N:
                    pair.cache.write_rows(layer, i, 1, 0, kk.view(np.uint8).reshape(N, -1))
                keys.append(kk.astype(np.float64))
                if N:
                    pick = np.sort(rng.choice(N, size=min(N, wl.k - 3), replace=False))
                    sels[i, : len(pick)] = pick
        rid = _t(np.arange(n, dtype=np.int32))
        if csa:
            qi = rng.standard_normal((n, HI, dI)).astype(np.float32)
            w = rng.standard_normal((n, HI)).astype(np.float32)
            ld = max(lens) // 4 + 5
            got = []
            for variant in ("high", "low"):
                scores = torch.full((n, ld), float("nan"), device="cuda")
                nv = torch.zeros(n, dtype=torch.int32, device="cuda")
                pair.cache.index_scores(0, rid, _t(qi), _t(w), scores, nv, variant=variant)
                pair.cache.check_device_error()
                got.append(scores.cpu().numpy())
            assert np.array_equal(np.nan_to_num(got[0], nan=7.0).view(np.uint32),
                                  np.nan_to_num(got[1], nan=7.0).view(np.uint32)), "index variants differ"
            for i, T in enumerate(lens):
                N = T // 4
                ref = O.index_scores(qi[i].astype(np.float64), w[i], keys[i])
                mag = np.abs(keys[i] @ qi[i].T.astype(np.float64)) @ np.abs(w[i])
                assert np.all(np.abs(got[0][i, :N] - ref) <= 1e-5 * mag + 1e-7), f"scores len {T}"
                assert np.isnan(got[0][i, N:]).all()
        outs = []
        for variant in ("high", "low"):
            out = torch.empty((n, H, D), dtype=torch.float32, device="cuda")
            pair.cache.decode_attn(layer, rid, _t(q), _t(sels) if csa else None, _t(sink), out, variant=variant)
            pair.cache.check_device_error()
            outs.append(out.cpu().numpy())
        assert np.array_equal(outs[0].view(np.uint32), outs[1].view(np.uint32)), "attention variants differ"
        for i, T in enumerate(lens):
            rows = ents[i][sels[i][sels[i] >= 0]] if csa else ents[i]
            rows = np.concatenate([rows, wins[i]], axis=0)
            ref = O.mqa_attention(O.rope(q[i].astype(np.float64), T - 1, R), rows, sink, 1.0 / math.sqrt(D))
            Hp.check_attention(outs[0][i], ref, f"layer {layer} len {T}", fmt="f32")


@pytest.mark.parametrize("layer", [0, 1])
def test_f32_decode_step_host_buffers_match_individual_calls(layer):
    """csa_decode_step (through api.DecodeStep) on an fp32-format cache: fp32
    q in the packed host buffer and an fp32 output, bit-identical to the
    individual calls on a second cache filled the same way, step after step,
    while CSA entries (every 4th token) and an HCA block (at 1024) complete."""
    from compressed_sparse_long_hca_b200.api import DecodeStep
    wl = I.Workload("f32-step", "csa", H=8, D=64, R=16, H_I=4, d_I=32, k=16, W=128, context=0, batch=0,
                    seed=5151)
    lens = [300, 1021]
    reqs = [1, 0]
    pairs = [Hp.Pair(wl, 1, 1, max_req=2, capacity=max(lens) + 64, fmt="f32") for _ in range(2)]
    for pair in pairs:
        for r, T in enumerate(lens):
            pair.cache.request_alloc(r, T + 64)
            pair.append(layer, [r], {r: pair.gen_tokens(layer, r, 0, T)}, T, oracle=False)
    torch.cuda.synchronize()
    csa = layer == 0
    sink = pairs[0].params[layer]["sink"]
    sink_d = _t(sink)
    step = DecodeStep(pairs[0].cache, layer, reqs, wl.k if csa else 0, sink)
    c2 = pairs[1].cache
    rid = _t(np.array(reqs, np.int32))
    rng = np.random.default_rng(23)
    for s in range(6):
        v = step.views(step.host_in)
        v["q"].copy_(torch.from_numpy(rng.standard_normal((2, wl.H, wl.D)).astype(np.float32)))
        toks = {r: pairs[0].gen_tokens(layer, r, lens[r] + s, 1) for r in reqs}
        for x, name in enumerate(("c", "z", "ci", "zi")):
            if name in v:
                v[name].copy_(torch.from_numpy(np.stack([toks[r][x] for r in reqs])))
        if csa:
            v["q_idx"].copy_(torch.from_numpy(rng.standard_normal((2, wl.H_I, wl.d_I)).astype(np.float32)))
            v["w"].copy_(torch.from_numpy(rng.standard_normal((2, wl.H_I)).astype(np.float32)))
        got = step()
        torch.cuda.synchronize()
        pairs[0].cache.check_device_error()
        assert got.dtype == torch.float32
        got = got.clone()
        got_idx = step.topk_idx.cpu() if csa else None
        # the same step through the individual calls on the second cache
        dv = {name: t.cuda() for name, t in v.items()}
        c2.compress_append(layer, rid, dv["c"], dv["z"], dv.get("ci"), dv.get("zi"))
        idx = None
        if csa:
            ld = max(c2.get_length(layer, r) for r in reqs) // 4 + 1
            scores = torch.empty((2, ld), device="cuda")
            nv = torch.empty(2, dtype=torch.int32, device="cuda")
            c2.index_scores(layer, rid, dv["q_idx"], dv["w"], scores, nv)
            idx = torch.empty((2, wl.k), dtype=torch.int32, device="cuda")
            topk(scores, nv, wl.k, idx)
        out = torch.empty((2, wl.H, wl.D), dtype=torch.float32, device="cuda")
        c2.decode_attn(layer, rid, dv["q"], idx, sink_d, out)
        torch.cuda.synchronize()
        c2.check_device_error()
        assert torch.equal(got.view(torch.int32), out.cpu().view(torch.int32)), f"step {s}: output differs"
        if csa:
            assert torch.equal(got_idx, idx.cpu()), f"step {s}: top-k differs"
