"""GPU parity: every step of the CUDA path against the fp64 oracle on the same
seeded inputs (through the C ABI), plus batch invariance and launch-variant
identity."""
import math

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


def _t(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t.to(dtype) if dtype is not None else t


# ---------------------------------------------------------------- tiny CSA from hidden states

def _c1_weights(seed):
    d = I.C1.hidden
    W = lambda shape, fan, f: I.normal(shape, seed, 99, f).astype(np.float64) / math.sqrt(fan)
    return dict(kv=W((64, d), d, 1), z=W((64, d), d, 2), ik=W((32, d), d, 3), iz=W((32, d), d, 4),
                q=W((8 * 64, d), d, 5), dq=W((64, d), d, 6), uq=W((4 * 32, 64), 64, 7), w=W((4, d), d, 8))


def test_c1_end_to_end_from_hidden_states():
    """Tiny CSA decode (hidden 256, 8 heads x 64, RoPE 16, indexer 4 x 32,
    top-16, context 1024, batch 1): hidden states -> projections (fp64, test
    side) -> CUDA path vs oracle, stage by stage."""
    wl = I.C1
    W = _c1_weights(wl.seed)
    T = wl.context
    h = I.normal((T + 1, wl.hidden), wl.seed, 0, 0, 77).astype(np.float64)
    proj = lambda M: O.f32(h @ M.T)
    c, z, ci, zi = proj(W["kv"]), proj(W["z"]), proj(W["ik"]), proj(W["iz"])
    pair = Hp.Pair(wl, 1, 0, max_req=2, capacity=T + 64)
    pair.cache.request_alloc(1, T + 64)
    # ragged chunking of the prefix exercises tails that straddle calls
    pos = 0
    for n_tok in [1, 2, 5, 3, 117, 4, 128, 256, 500, 7, 1]:
        n_tok = min(n_tok, T - pos)
        if n_tok == 0:
            break
        pair.append(0, [1], {1: (c[pos:pos + n_tok], z[pos:pos + n_tok], ci[pos:pos + n_tok],
                                 zi[pos:pos + n_tok])}, n_tok)
        pos += n_tok
    assert pos == T
    # decode step: append token T, then index -> top-k -> attention
    pair.append(0, [1], {1: (c[T:T + 1], z[T:T + 1], ci[T:T + 1], zi[T:T + 1])}, 1)
    hq = h[T]
    q = I.bf16_grid(O.f32(W["q"] @ hq).reshape(8, 64))
    qi = O.f32(W["uq"] @ (W["dq"] @ hq)).reshape(4, 32)
    w = O.f32(W["w"] @ hq)
    sink = pair.params[0]["sink"]
    rid = _t(np.array([1], np.int32))
    N = (T + 1) // 4
    ld = N + 37
    scores = torch.full((1, ld), float("nan"), device="cuda")
    nv = torch.zeros(1, dtype=torch.int32, device="cuda")
    pair.cache.index_scores(0, rid, _t(qi[None]), _t(w[None]), scores, nv)
    idx = torch.empty((1, wl.k), dtype=torch.int32, device="cuda")
    from compressed_sparse_long_hca_b200.api import topk
    topk(scores, nv, wl.k, idx)
    out = torch.empty((1, 8, 64), dtype=torch.bfloat16, device="cuda")
    pair.cache.decode_attn(0, rid, _t(q[None], torch.bfloat16), idx, _t(sink), out)
    pair.cache.check_device_error()
    assert pair.cache.get_length(0, 1) == T + 1
    assert int(nv[0]) == N
    # ---- oracle, stage by stage
    p = pair.oracle_params(0)
    st = pair.states[(0, 1)]
    kv_ref, key_ref = O.csa_entries_all(np.array(st.c), np.array(st.z), np.array(st.ci),
                                        np.array(st.zi), p.b_kv, p.b_idx, p.R)
    same_kv = Hp.check_kv_rounding(pair.cache.read_rows(0, 1, 0, 0, N), kv_ref, 64, 16, "entries")
    same_key = Hp.check_index_rounding(pair.cache.read_rows(0, 1, 1, 0, N), key_ref, 32, "keys")
    win_pos = O.window_positions(T)
    win_ref = np.stack([O.raw_token_row(st.c[t], t, 16) for t in win_pos])
    Hp.check_kv_rounding(pair.cache.read_rows(0, 1, 2, win_pos[0], len(win_pos)), win_ref, 64, 16, "window")
    res = O.decode_query(p, st, q, sink, k=wl.k, q_idx=qi, w=w)
    s_gpu = scores[0, :N].double().cpu().numpy()
    assert np.isnan(scores[0, N:].cpu().numpy()).all(), "scores written past N"
    qd = O.dequantize_mxfp4(O.quantize_mxfp4(qi))
    keyd = O.dequantize_mxfp4(O.quantize_mxfp4(key_ref))
    mag = np.abs(keyd @ qd.T) @ np.abs(w)
    ok = same_key
    assert np.all(np.abs(s_gpu - res["scores"])[ok] <= 1e-5 * mag[ok] + 1e-6)
    Hp.check_topk(idx[0].cpu().numpy(), res["scores"], wl.k, N, excused=np.where(~ok)[0])
    got_out = out[0].float().cpu().numpy()
    # the attention over the rows the GPU selected and stored, whatever the selection
    Hp.check_attention(got_out, Hp.attention_over_stored_rows(pair.cache, 0, 1, T, idx[0].cpu().numpy(), q, sink,
                                                              64, 16), "c1 attention (stored rows)")
    if set(idx[0].cpu().numpy().tolist()) == set(res["topk"].tolist()):
        # and end to end against the oracle's own rows
        Hp.check_attention(got_out, res["out"], "c1 attention")
    # scales are fp32 divisions of amax values that differ by fp32 rounding only
    from compressed_sparse_long_hca_b200.api import unpack_kv_rows
    sc_gpu = unpack_kv_rows(pair.cache.read_rows(0, 1, 0, 0, N), 64, 16)[2]
    sc_ref = O.quantize_kv(kv_ref, 16).scale
    assert np.all(np.abs(sc_gpu / sc_ref - 1) <= 2.0 ** -20)
    assert same_kv.mean() > 0.2


# ---------------------------------------------------------------- stage: index scores

@pytest.mark.parametrize("HI,dI", [(4, 32), (64, 128), (7, 96)])
def test_index_scores_on_oracle_written_keys(HI, dI):
    """Scores over keys written from oracle codes: only the indexer runs."""
    wl = I.Workload("idx", "csa", H=8, D=64, R=16, H_I=HI, d_I=dI, k=8, W=128, context=0, batch=0,
                    seed=4242)
    lens = [1, 3, 4, 129 * 4 + 3, 1000, 4096 + 17]          # ragged, tile tails, tiny
    pair = Hp.Pair(wl, 1, 0, max_req=len(lens), capacity=max(lens) + 8)
    r = np.random.default_rng(7)
    ref_scores = {}
    for i, T in enumerate(lens):
        pair.cache.request_alloc(i, T + 8)
        pair.cache.set_length(0, i, T)
        N = T // 4
        keys = O.quantize_mxfp4(r.standard_normal((max(N, 1), dI)) * np.exp2(r.integers(-3, 3, (max(N, 1), 1))))
        if N:
            from compressed_sparse_long_hca_b200.api import pack_index_rows
            pair.cache.write_rows(0, i, 1, 0, pack_index_rows(keys.codes[:N], keys.scales[:N]))
        ref_scores[i] = keys
    n = len(lens)
    qi = r.standard_normal((n, HI, dI)).astype(np.float32)
    w = r.standard_normal((n, HI)).astype(np.float32)
    ld = max(lens) // 4 + 5
    for variant in ("high", "low"):
        scores = torch.full((n, ld), float("nan"), device="cuda")
        nv = torch.zeros(n, dtype=torch.int32, device="cuda")
        pair.cache.index_scores(0, _t(np.arange(n, dtype=np.int32)), _t(qi), _t(w), scores, nv, variant=variant)
        pair.cache.check_device_error()
        got = scores.double().cpu().numpy()
        for i, T in enumerate(lens):
            N = T // 4
            assert int(nv[i]) == N
            if N == 0:
                continue
            kd = O.dequantize_mxfp4(ref_scores[i])[:N]
            qd = O.dequantize_mxfp4(O.quantize_mxfp4(qi[i]))
            ref = O.index_scores(qd, w[i], kd)
            mag = np.abs(kd @ qd.T) @ np.abs(w[i])
            assert np.all(np.abs(got[i, :N] - ref) <= 1e-5 * mag + 1e-6), f"len {T} variant {variant}"
            assert np.isnan(got[i, N:]).all()
        if variant == "high":
            first = got.copy()
        else:
            assert np.array_equal(np.nan_to_num(first, nan=7.0), np.nan_to_num(got, nan=7.0))
    # the same queries in smaller batches and other positions: the same bits
    for sub in ([5, 3, 0], [4, 5, 1, 2], [5], [3, 4, 5, 0]):
        scores = torch.full((len(sub), ld), float("nan"), device="cuda")
        nv = torch.zeros(len(sub), dtype=torch.int32, device="cuda")
        pair.cache.index_scores(0, _t(np.array(sub, np.int32)), _t(qi[sub]), _t(w[sub]), scores, nv)
        pair.cache.check_device_error()
        got = scores.double().cpu().numpy()
        assert np.array_equal(np.nan_to_num(first[sub], nan=7.0), np.nan_to_num(got, nan=7.0)), f"batch {sub}"


# ---------------------------------------------------------------- stage: top-k

def _topk_case(scores_list, k):
    from compressed_sparse_long_hca_b200.api import topk
    n = len(scores_list)
    ld = max(len(s) for s in scores_list) + 3
    S = np.full((n, ld), np.float32(-1e30))
    for i, s in enumerate(scores_list):
        S[i, : len(s)] = s
    nv = np.array([len(s) for s in scores_list], np.int32)
    outs = []
    for variant in ("high", "low"):
        out = torch.full((n, k), 12345, dtype=torch.int32, device="cuda")
        topk(_t(S), _t(nv), k, out, variant=variant)
        torch.cuda.synchronize()
        outs.append(out.cpu().numpy())
    assert np.array_equal(outs[0], outs[1])
    for i, s in enumerate(scores_list):
        ref = O.topk(np.asarray(s, np.float64), k)
        assert np.array_equal(outs[0][i], ref), f"row {i} (n={len(s)}, k={k})"


def test_topk_exact_on_shared_scores():
    r = np.random.default_rng(11)
    rows = [
        r.standard_normal(5000).astype(np.float32),
        r.integers(-4, 5, 3000).astype(np.float32),                  # heavy ties
        np.zeros(700, np.float32) * np.where(r.random(700) < 0.5, -1, 1),   # +-0 only
        r.standard_normal(10).astype(np.float32),                    # N < k
        r.standard_normal(64).astype(np.float32),                    # N == k
        r.standard_normal(65).astype(np.float32),                    # N == k + 1
        np.array([], np.float32),                                    # empty
        np.concatenate([np.full(100, 3.0, np.float32), np.full(100, -np.inf, np.float32)]),
    ]
    rows[2][::3] = -0.0
    _topk_case(rows, 64)
    _topk_case(rows[:2], 1)


@pytest.mark.parametrize("N,k", [(32768, 512), (262144, 1024)])
def test_topk_exact_large(N, k):
    r = np.random.default_rng(N)
    a = (r.standard_normal(N) * 10).astype(np.float32)
    b = np.round(r.standard_normal(N) * 3).astype(np.float32)     # many exact ties at the k-th
    _topk_case([a, b], k)


def test_topk_rows_that_defeat_or_stress_the_sample_filter():
    """The selector estimates a threshold from a sample of the scores (64
    evenly spaced runs of 64 consecutive scores).  Rows whose sample lies
    about the top k must still come out exact: a sample made of the largest
    scores (too few pass the threshold), a top k hidden outside the sample,
    and a tie class at the k-th score."""
    N, k = 262144, 1024
    x = np.arange(4096)
    sampled = (x // 64) * (N // 64) + x % 64
    unsampled = (x // 64) * (N // 64) + 64 + x % 64
    r = np.random.default_rng(99)
    base = r.standard_normal(N).astype(np.float32)
    lying = base.copy()
    lying[sampled] = 100.0 + np.arange(4096, dtype=np.float32)        # the sample sees only these
    hidden = base.copy()
    hidden[unsampled[:k]] = 50.0 + r.random(k).astype(np.float32)     # never sampled
    ties = base.copy()
    ties[r.choice(N, 3000, replace=False)] = 3.0                       # the k-th score is a 3000-way tie
    _topk_case([lying, hidden, ties], k)


# ---------------------------------------------------------------- stage: attention

def _write_cache_rows(pair, layer, req, T, rng, csa=True):
    """Write oracle-quantised random entries and window rows; return their
    dequantised values (entries, window)."""
    from compressed_sparse_long_hca_b200.api import pack_kv_rows
    wl = pair.wl
    N = T // 4 if csa else T // 128
    pair.cache.set_length(layer, req, T)
    ent = O.quantize_kv(rng.standard_normal((max(N, 1), wl.D)) * 0.5, wl.R)
    if N:
        pair.cache.write_rows(layer, req, 0, 0, pack_kv_rows(ent.fp8[:N], ent.rope[:N], ent.scale[:N]))
    wp = O.window_positions(T - 1)
    win = O.quantize_kv(rng.standard_normal((len(wp), wl.D)), wl.R)
    pair.cache.write_rows(layer, req, 2, wp[0], pack_kv_rows(win.fp8, win.rope, win.scale))
    return O.dequantize_kv(ent)[:N], O.dequantize_kv(win)


@pytest.mark.parametrize("H,D,R", [(8, 64, 16), (64, 512, 64), (128, 512, 64)])
def test_attention_on_oracle_written_rows(H, D, R):
    wl = I.Workload("att", "csa", H=H, D=D, R=R, H_I=4, d_I=32, k=40, W=128, context=0, batch=0,
                    seed=555)
    lens = [1, 5, 130, 1000, 4000]
    pair = Hp.Pair(wl, 1, 1, max_req=len(lens), capacity=max(lens) + 8)
    rng = np.random.default_rng(H + D)
    n = len(lens)
    q = I.bf16_grid(rng.standard_normal((n, H, D)).astype(np.float32))
    sink = pair.params[0]["sink"]
    sink_h = pair.params[1]["sink"]
    for layer in (0, 1):
        csa = layer == 0
        ents, wins, sels = [], [], np.full((n, wl.k), -1, np.int32)
        for i, T in enumerate(lens):
            pair.cache.request_alloc(i, T + 8) if layer == 0 else None
            e, wv = _write_cache_rows(pair, layer, i, T, rng, csa)
            ents.append(e)
            wins.append(wv)
            N = e.shape[0]
            if csa and N:
                pick = np.sort(rng.choice(N, size=min(N, wl.k - 3), replace=False))
                sels[i, : len(pick)] = pick
        outs = []
        for variant in ("high", "low"):
            out = torch.empty((n, H, D), dtype=torch.bfloat16, device="cuda")
            pair.cache.decode_attn(layer, _t(np.arange(n, dtype=np.int32)), _t(q, torch.bfloat16),
                                   _t(sels) if csa else None, _t(sink if csa else sink_h), out,
                                   variant=variant)
            pair.cache.check_device_error()
            outs.append(out.float().cpu().numpy())
        assert np.array_equal(outs[0], outs[1]), "variants differ"
        for i, T in enumerate(lens):
            rows = ents[i][sels[i][sels[i] >= 0]] if csa else ents[i]
            rows = np.concatenate([rows, wins[i]], axis=0)
            ref = O.mqa_attention(O.rope(q[i].astype(np.float64), T - 1, R), rows,
                                  sink if csa else sink_h, 1.0 / math.sqrt(D))
            Hp.check_attention(outs[0][i], ref, f"layer {layer} len {T}")


@pytest.mark.parametrize("H,D,R", [(32, 160, 32), (128, 512, 64)])
def test_attention_many_tiles_and_empty_rows(H, D, R):
    """Rows spanning many 128-row tiles, -1 holes inside the list, tiles with
    no row at all, and a padded head dim; every launch variant returns the
    same bits and matches the oracle."""
    wl = I.Workload("att-tiles", "csa", H=H, D=D, R=R, H_I=4, d_I=32, k=700, W=128, context=0, batch=0,
                    seed=556)
    lens = [3000, 40000, 9001]
    pair = Hp.Pair(wl, 1, 1, max_req=len(lens), capacity=max(lens) + 8)
    rng = np.random.default_rng(H * D)
    n = len(lens)
    q = I.bf16_grid(rng.standard_normal((n, H, D)).astype(np.float32))
    for layer in (0, 1):
        csa = layer == 0
        sink = pair.params[layer]["sink"]
        ents, wins, sels = [], [], np.full((n, wl.k), -1, np.int32)
        for i, T in enumerate(lens):
            if layer == 0:
                pair.cache.request_alloc(i, T + 8)
            e, wv = _write_cache_rows(pair, layer, i, T, rng, csa)
            ents.append(e)
            wins.append(wv)
            if csa:
                N = e.shape[0]
                pick = np.sort(rng.choice(N, size=min(N, wl.k), replace=False)).astype(np.int32)
                sels[i, : len(pick)] = pick
        if csa:
            sels[0, rng.random(wl.k) < 0.3] = -1               # holes inside the list
            sels[2, :384] = -1                                 # three tiles without a row
        outs = []
        for variant in ("high", "low", "auto"):
            out = torch.empty((n, H, D), dtype=torch.bfloat16, device="cuda")
            pair.cache.decode_attn(layer, _t(np.arange(n, dtype=np.int32)), _t(q, torch.bfloat16),
                                   _t(sels) if csa else None, _t(sink), out, variant=variant)
            pair.cache.check_device_error()
            outs.append(out.float().cpu().numpy())
        assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[0], outs[2]), "variants differ"
        for i, T in enumerate(lens):
            rows = ents[i][sels[i][sels[i] >= 0]] if csa else ents[i]
            rows = np.concatenate([rows, wins[i]], axis=0)
            ref = O.mqa_attention(O.rope(q[i].astype(np.float64), T - 1, R), rows, sink, 1.0 / math.sqrt(D))
            Hp.check_attention(outs[0][i], ref, f"layer {layer} len {T}")


# ---------------------------------------------------------------- HCA end to end

def test_hca_end_to_end_small():
    wl = I.Workload("hca-small", "hca", H=8, D=64, R=16, H_I=0, d_I=0, k=0, W=128, context=0,
                    batch=0, seed=9090)
    pair = Hp.Pair(wl, 0, 1, max_req=3, capacity=1200)
    sink = pair.params[0]["sink"]
    lens = {0: [1, 127, 1], 1: [300, 5, 400], 2: [128, 128, 1]}
    for r in lens:
        pair.cache.request_alloc(r, 1200)
    for step in range(3):
        for r, chunks in lens.items():
            start = pair.cache.get_length(0, r) if (0, r) in pair.states else 0
            n_tok = chunks[step]
            pair.append(0, [r], {r: pair.gen_tokens(0, r, start, n_tok)}, n_tok)
    reqs = [0, 1, 2]
    q = I.bf16_grid(np.random.default_rng(3).standard_normal((3, 8, 64)).astype(np.float32))
    out = torch.empty((3, 8, 64), dtype=torch.bfloat16, device="cuda")
    pair.cache.decode_attn(0, _t(np.array(reqs, np.int32)), _t(q, torch.bfloat16), None, _t(sink), out)
    pair.cache.check_device_error()
    p = pair.oracle_params(0)
    for i, r in enumerate(reqs):
        st = pair.states[(0, r)]
        T = st.T
        assert pair.cache.get_length(0, r) == T
        ent_ref = O.hca_entries_all(np.array(st.c), np.array(st.z), p.b_kv, 16)
        if ent_ref.shape[0]:
            Hp.check_kv_rounding(pair.cache.read_rows(0, r, 0, 0, ent_ref.shape[0]), ent_ref, 64, 16, "hca entries")
        res = O.decode_query(p, st, q[i], sink)
        Hp.check_attention(out[i].float().cpu().numpy(), res["out"], f"hca req {r}")


# ---------------------------------------------------------------- batch invariance

def test_batch_invariance_and_variants():
    """A query's bits do not depend on batch size, position in the batch or
    co-batched requests, nor on the launch variant."""
    wl = I.Workload("bi", "csa", H=16, D=128, R=32, H_I=8, d_I=64, k=24, W=128, context=0, batch=0,
                    seed=31337)
    lens = [700, 33, 2000, 129, 1500]
    pair = Hp.Pair(wl, 1, 1, max_req=len(lens), capacity=max(lens) + 8)
    for r, T in enumerate(lens):
        pair.cache.request_alloc(r, T + 8)
        for layer in (0, 1):
            pair.append(layer, [r], {r: pair.gen_tokens(layer, r, 0, T)}, T, oracle=False)
    rng = np.random.default_rng(5)
    n = len(lens)
    q = I.bf16_grid(rng.standard_normal((n, 16, 128)).astype(np.float32))
    qi = rng.standard_normal((n, 8, 64)).astype(np.float32)
    w = rng.standard_normal((n, 8)).astype(np.float32)
    sink = pair.params[0]["sink"]

    def run(order, variant, fused=False):
        """fused: index_topk, then the attention directly after it with
        state_ready (its lengths, window and q read before the top-k ends)."""
        order = list(order)
        rid = _t(np.array(order, np.int32))
        m = len(order)
        ld = max(lens) // 4 + 1
        scores = torch.zeros((m, ld), device="cuda")
        nv = torch.zeros(m, dtype=torch.int32, device="cuda")
        idx = torch.empty((m, wl.k), dtype=torch.int32, device="cuda")
        qd = _t(q[order], torch.bfloat16)
        if fused:
            pair.cache.index_topk(0, rid, _t(qi[order]), _t(w[order]), scores, nv, wl.k, idx, variant=variant)
        else:
            pair.cache.index_scores(0, rid, _t(qi[order]), _t(w[order]), scores, nv, variant=variant)
            from compressed_sparse_long_hca_b200.api import topk
            topk(scores, nv, wl.k, idx, variant=variant)
        out = torch.empty((m, 16, 128), dtype=torch.bfloat16, device="cuda")
        pair.cache.decode_attn(0, rid, qd, idx, _t(sink), out, variant=variant, state_ready=fused)
        out_h = torch.empty((m, 16, 128), dtype=torch.bfloat16, device="cuda")
        pair.cache.decode_attn(1, rid, _t(q[order], torch.bfloat16), None, _t(sink), out_h, variant=variant)
        pair.cache.check_device_error()
        return {r: (scores[i, : lens[r] // 4].cpu().numpy().tobytes(), idx[i].cpu().numpy().tobytes(),
                    out[i].view(torch.int16).cpu().numpy().tobytes(),
                    out_h[i].view(torch.int16).cpu().numpy().tobytes())
                for i, r in enumerate(order)}

    base = run(range(n), "high")
    for order, variant, fused in [([2], "low", False), ([4, 2, 0], "high", False), ([1, 3, 0, 4, 2], "low", False),
                                  ([3, 3, 1], "auto", False), ([1, 3, 0, 4, 2], "low", True), ([4, 2, 0], "high", True)]:
        got = run(order, variant, fused)
        for r in order:
            assert got[r] == base[r], f"request {r} differs in batch {order} ({variant})"


# ---------------------------------------------------------------- device-side errors

def test_device_errors_are_reported_not_trapped():
    from compressed_sparse_long_hca_b200._lib import CsaError
    wl = I.Workload("err", "csa", H=8, D=64, R=16, H_I=4, d_I=32, k=8, W=128, context=0, batch=0, seed=1)
    pair = Hp.Pair(wl, 1, 0, max_req=2, capacity=256)
    pair.cache.request_alloc(0, 256)
    # request id out of range: recorded on the device, reported by the check
    scores = torch.zeros((1, 100), device="cuda")
    nv = torch.zeros(1, dtype=torch.int32, device="cuda")
    pair.cache.index_scores(0, _t(np.array([7], np.int32)), _t(np.zeros((1, 4, 32), np.float32)),
                            _t(np.zeros((1, 4), np.float32)), scores, nv)
    with pytest.raises(CsaError) as e:
        pair.cache.check_device_error()
    assert e.value.status == -5
    pair.cache.check_device_error()          # the word was cleared
    # capacity: one 512-token page allowed, appending 600 is refused on the device
    toks = pair.gen_tokens(0, 0, 0, 600)
    pair.append(0, [0], {0: toks}, 600, oracle=False)
    with pytest.raises(CsaError) as e:
        pair.cache.check_device_error()
    assert e.value.status == -2
    assert pair.cache.get_length(0, 0) == 0
    # score row too short
    pair.append(0, [0], {0: pair.gen_tokens(0, 0, 0, 200)}, 200, oracle=False)
    small = torch.zeros((1, 10), device="cuda")
    pair.cache.index_scores(0, _t(np.array([0], np.int32)), _t(np.zeros((1, 4, 32), np.float32)),
                            _t(np.zeros((1, 4), np.float32)), small, nv)
    with pytest.raises(CsaError):
        pair.cache.check_device_error()
    # host-side argument errors never launch
    with pytest.raises(CsaError) as e:
        pair.cache.decode_attn(0, _t(np.array([0], np.int32)), torch.zeros((1, 8, 64), dtype=torch.bfloat16,
                               device="cuda"), None, _t(np.zeros(8, np.float32)),
                               torch.zeros((1, 8, 64), dtype=torch.bfloat16, device="cuda"))
    assert e.value.status == -1
    # a top-k index beyond the request's entries is a bounds error, not a fault
    bad = _t(np.array([[0, 1, 99999, -1, -1, -1, -1, -1]], np.int32))
    out = torch.zeros((1, 8, 64), dtype=torch.bfloat16, device="cuda")
    pair.cache.decode_attn(0, _t(np.array([0], np.int32)), torch.zeros((1, 8, 64), dtype=torch.bfloat16,
                           device="cuda"), bad, _t(np.zeros(8, np.float32)), out)
    with pytest.raises(CsaError) as e:
        pair.cache.check_device_error()
    assert e.value.status == -5


# ---------------------------------------------------------------- stage: fused index + top-k

def _fused_vs_separate(pair, qi, w, k, reqs, ld, variant="auto"):
    """csa_index_topk against csa_index_scores + csa_topk on the same inputs:
    returns (scores, n_valid, idx) of the fused call after checking bits."""
    from compressed_sparse_long_hca_b200.api import topk
    n = len(reqs)
    rid = _t(np.array(reqs, np.int32))
    s1 = torch.full((n, ld), float("nan"), device="cuda")
    nv1 = torch.zeros(n, dtype=torch.int32, device="cuda")
    pair.cache.index_scores(0, rid, _t(qi[reqs]), _t(w[reqs]), s1, nv1, variant=variant)
    i1 = torch.full((n, k), 777, dtype=torch.int32, device="cuda")
    topk(s1, nv1, k, i1, variant=variant)
    s2 = torch.full((n, ld), float("nan"), device="cuda")
    nv2 = torch.zeros(n, dtype=torch.int32, device="cuda")
    i2 = torch.full((n, k), 777, dtype=torch.int32, device="cuda")
    pair.cache.index_topk(0, rid, _t(qi[reqs]), _t(w[reqs]), s2, nv2, k, i2, variant=variant)
    pair.cache.check_device_error()
    a1, a2 = s1.cpu().numpy(), s2.cpu().numpy()
    assert np.array_equal(np.nan_to_num(a1, nan=7.0).view(np.uint32), np.nan_to_num(a2, nan=7.0).view(np.uint32))
    assert torch.equal(nv1, nv2)
    assert torch.equal(i1, i2), f"fused top-k differs from csa_topk (k={k}, reqs={reqs})"
    return a2, nv2.cpu().numpy(), i2.cpu().numpy()


@pytest.mark.parametrize("k", [1, 16, 512, 1024])
def test_fused_index_topk_equals_separate_calls(k):
    """csa_index_topk = csa_index_scores + csa_topk, bit for bit, on keys
    written from oracle codes: ragged lengths (tile tails, N < k, N = 0), heavy
    exact ties (integer-valued scores), an all-zero row (w = 0: one tie class
    of 33,793 keys, which sends the selection to its radix path), and other
    batch compositions; indices also against the oracle's top-k."""
    from compressed_sparse_long_hca_b200.api import pack_index_rows
    HI, dI = 64, 128
    wl = I.Workload("fused", "csa", H=8, D=64, R=16, H_I=HI, d_I=dI, k=k, W=128, context=0, batch=0, seed=4243)
    lens = [1, 3, 4, 517 * 4 + 1, 4000, 40000, 33 * 4096 + 5, 20000, 12345]
    pair = Hp.Pair(wl, 1, 0, max_req=len(lens), capacity=max(lens) + 8)
    r = np.random.default_rng(k + 7)
    keys = {}
    for i, T in enumerate(lens):
        pair.cache.request_alloc(i, T + 8)
        pair.cache.set_length(0, i, T)
        N = T // 4
        if i == 7:      # integer-valued dots: every element +-1 at scale 2^0
            x = np.where(r.random((max(N, 1), dI)) < 0.5, -1.0, 1.0)
        else:
            x = r.standard_normal((max(N, 1), dI)) * np.exp2(r.integers(-3, 3, (max(N, 1), 1)))
        kq = O.quantize_mxfp4(x)
        if N:
            pair.cache.write_rows(0, i, 1, 0, pack_index_rows(kq.codes[:N], kq.scales[:N]))
        keys[i] = kq
    n = len(lens)
    qi = r.standard_normal((n, HI, dI)).astype(np.float32)
    qi[7] = np.where(r.random((HI, dI)) < 0.5, -1.0, 1.0).astype(np.float32)
    w = r.standard_normal((n, HI)).astype(np.float32)
    w[5] = 0.0                         # all scores 0: one tie class of N = 33793 keys
    w[7] = 1.0
    ld = max(lens) // 4 + 5
    allr = list(range(n))
    sc, nv, idx = _fused_vs_separate(pair, qi, w, k, allr, ld)
    for i, T in enumerate(lens):
        N = T // 4
        assert int(nv[i]) == N
        if N == 0:
            assert (idx[i] == -1).all()
            continue
        kd = O.dequantize_mxfp4(keys[i])[:N]
        ref = O.index_scores(O.dequantize_mxfp4(O.quantize_mxfp4(qi[i])), w[i], kd)
        Hp.check_topk(idx[i], ref, k, N, what=f"fused top-k len {T}")
        # exactly the top-k of the GPU's own scores
        assert np.array_equal(idx[i], O.topk(sc[i, :N].astype(np.float64), k)), f"len {T}"
    for sub, variant in (([6, 2, 5], "high"), ([5], "low"), ([8, 7, 0, 3], "auto"), (allr[::-1], "low")):
        _, _, idx2 = _fused_vs_separate(pair, qi, w, k, sub, ld, variant)
        for x_, i in enumerate(sub):
            assert np.array_equal(idx2[x_], idx[i]), (sub, i)
