"""GPU parity at the workloads' full sizes, in the launch configuration that
bench.py times (AUTO variants, the same batch shapes).

Caches are filled through csa_compress_append with device-generated inputs,
then one decode step runs (append -> index -> top-k -> attention).  The
oracle checks every index score against the keys read back from the cache,
the top-k index set against its own top-k of its own scores, and every
attention output over the rows the GPU selected (read back); the same step is
re-run in another batch order and with both launch variants, bit-exact.

A bounded ragged sweep (Pro-like CSA and HCA layers, contexts log-uniform in
[4K, 256K]) checks that a request's bits do not depend on the batch it is in.
"""
import math

import numpy as np
import pytest

from compressed_sparse_long_hca_b200 import inputs as I
from compressed_sparse_long_hca_b200.api import topk, unpack_index_rows, unpack_kv_rows
from oracle import csa_oracle as O
from tests import helpers as Hp

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_lib):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return cuda_lib


def _fill(cache, layer, reqs, lengths, seed, D, dI):
    """Append tokens 0 .. lengths[r]-1 of every request (chunks of 4096;
    requests that are already full drop out of later calls)."""
    t = 0
    chunk, gen = -1, {}
    while True:
        live = [r for r in reqs if lengths[r] > t]
        if not live:
            break
        n_tok = min(min(lengths[r] for r in live) - t, I.CHUNK - t % I.CHUNK)
        if t // I.CHUNK != chunk:          # each request's chunk is generated once
            chunk, gen = t // I.CHUNK, {}
        for r in live:
            if r not in gen:
                gen[r] = I.device_token_inputs(seed, layer, r, chunk, D, dI)
        parts = [gen[r] for r in live]
        lo = t % I.CHUNK
        st = lambda k: (torch.stack([p[k][lo:lo + n_tok] for p in parts]).contiguous()
                        if parts[0][k] is not None else None)
        cache.compress_append(layer, torch.tensor(live, dtype=torch.int32, device="cuda"), st(0), st(1), st(2), st(3))
        t += n_tok
    torch.cuda.synchronize()
    cache.check_device_error()


def _compressor_check(cache, wl, layer, r, seed, T0, c_dec, csa):
    """The compressor at the workload's shapes against the oracle, on the
    device-generated inputs the fill appended (copied back to the host): the
    first entries, an entry whose 8-token window straddles two fill calls
    (CSA), the last entries before the decode token (positions near T0), and
    the window rows including the decode token's own (host-generated) row."""
    dI = wl.d_I if csa else 0
    m = 4 if csa else 128
    N = T0 // m
    chunks = {}

    def tokens(lo, hi):
        """c, z, ci, zi of positions lo .. hi-1 (hi <= T0), fp64 on the host."""
        parts = {k: [] for k in range(4)}
        for ch in range(lo // I.CHUNK, (hi - 1) // I.CHUNK + 1):
            if ch not in chunks:
                g = I.device_token_inputs(seed, layer, r, ch, wl.D, dI)
                chunks[ch] = [x.double().cpu().numpy() if x is not None else None for x in g]
            a, b = max(lo, ch * I.CHUNK) - ch * I.CHUNK, min(hi, (ch + 1) * I.CHUNK) - ch * I.CHUNK
            for k in range(4):
                if chunks[ch][k] is not None:
                    parts[k].append(chunks[ch][k][a:b])
        return [np.concatenate(parts[k]) if parts[k] else None for k in range(4)]

    params = _PARAMS[(wl.name, layer)]
    ents = [0, 1, N - 2, N - 1]
    if csa and T0 >= 2 * I.CHUNK:
        ents.append((T0 // I.CHUNK - 1) * (I.CHUNK // 4))     # window [4096c - 4, 4096c + 4)
    ents = sorted(set(e for e in ents if 0 <= e < N))
    got_kv = np.concatenate([cache.read_rows(layer, r, 0, j, 1) for j in ents])
    ref_kv, ref_key = [], []
    for j in ents:
        lo = max(0, m * j - (4 if csa else 0))
        c, z, ci, zi = tokens(lo, m * j + m)
        if csa:
            kv, key = O.csa_entry_vectors(c, z, ci, zi, params["b_kv"], params["b_idx"], j, wl.D, wl.R, offset=lo)
            ref_key.append(key)
        else:
            kv = O.hca_entry_vector(c, z, params["b_kv"], j, wl.D, wl.R, offset=lo)
        ref_kv.append(kv)
    Hp.check_kv_rounding(got_kv, np.stack(ref_kv), wl.D, wl.R, f"{wl.name} entries {ents}", min_exact=0.998)
    if csa:
        got_key = np.concatenate([cache.read_rows(layer, r, 1, j, 1) for j in ents])
        Hp.check_index_rounding(got_key, np.stack(ref_key), wl.d_I, f"{wl.name} index keys {ents}", min_exact=0.998)
    # window: positions T0-127 .. T0, the last one the decode token
    wp = O.window_positions(T0)
    c = tokens(wp[0], T0)[0]
    c = np.concatenate([c, np.asarray(c_dec, np.float64).reshape(1, -1)])
    win_ref = np.stack([O.raw_token_row(c[x], wp[x], wl.R) for x in range(len(wp))])
    Hp.check_kv_rounding(cache.read_rows(layer, r, 2, wp[0], len(wp)), win_ref, wl.D, wl.R,
                         f"{wl.name} window", min_exact=0.998)


_PARAMS = {}


def _host(seed, *shape):
    return np.random.default_rng(seed).standard_normal(shape).astype(np.float32)


def _step(cache, wl, layer, order, q, qi, w, sink, variant="auto"):
    """Index, top-k and attention for the requests in `order`; results are
    returned in request order (dicts keyed by request)."""
    csa = wl.kind == "csa"
    n = len(order)
    rid = torch.tensor(order, dtype=torch.int32, device="cuda")
    dq = torch.from_numpy(q[order]).cuda().to(torch.bfloat16)
    out = torch.empty((n, wl.H, wl.D), dtype=torch.bfloat16, device="cuda")
    res = {}
    if csa:
        ld = max(cache.get_length(layer, r) for r in order) // 4 + 128
        scores = torch.full((n, ld), float("nan"), device="cuda")
        nv = torch.zeros(n, dtype=torch.int32, device="cuda")
        cache.index_scores(layer, rid, torch.from_numpy(qi[order]).cuda(), torch.from_numpy(w[order]).cuda(), scores,
                           nv, variant=variant)
        idx = torch.empty((n, wl.k), dtype=torch.int32, device="cuda")
        topk(scores, nv, wl.k, idx, variant=variant)
        cache.decode_attn(layer, rid, dq, idx, torch.from_numpy(sink).cuda(), out, variant=variant)
        # the fused index + top-k (the launch the bench times) gives the same bits
        s2 = torch.full((n, ld), float("nan"), device="cuda")
        nv2 = torch.zeros(n, dtype=torch.int32, device="cuda")
        i2 = torch.empty((n, wl.k), dtype=torch.int32, device="cuda")
        cache.index_topk(layer, rid, torch.from_numpy(qi[order]).cuda(), torch.from_numpy(w[order]).cuda(), s2, nv2,
                         wl.k, i2, variant=variant)
        cache.check_device_error()
        assert torch.equal(i2, idx), "fused top-k differs"
        assert torch.equal(nv2, nv)
        assert torch.equal(torch.nan_to_num(s2, nan=7.0).view(torch.int32), torch.nan_to_num(scores, nan=7.0).view(torch.int32))
        sc, nvh, ih = scores.cpu().numpy(), nv.cpu().numpy(), idx.cpu().numpy()
        for x, r in enumerate(order):
            res[r] = dict(scores=sc[x, : nvh[x]].copy(), idx=ih[x].copy())
    else:
        cache.decode_attn(layer, rid, dq, None, torch.from_numpy(sink).cuda(), out, variant=variant)
        cache.check_device_error()
    oh = out.cpu()
    for x, r in enumerate(order):
        res.setdefault(r, {})["out"] = oh[x].view(torch.int16).numpy().copy()
        res[r]["out_f"] = oh[x].float().numpy()
    return res


def _oracle_check(cache, wl, layer, r, T, q, qi, w, sink, got):
    """Oracle parity of one request's decode step (T tokens stored)."""
    csa = wl.kind == "csa"
    t = T - 1
    N = T // 4 if csa else T // 128
    if csa:
        codes, scales = unpack_index_rows(cache.read_rows(layer, r, 1, 0, N), wl.d_I)
        kd = O.dequantize_mxfp4(O.MXFP4(codes=codes, scales=scales))
        qd = O.dequantize_mxfp4(O.quantize_mxfp4(qi[r]))
        ref = O.index_scores(qd, w[r], kd)
        mag = np.abs(kd @ qd.T) @ np.abs(w[r])
        assert got["scores"].shape[0] == N
        assert np.all(np.abs(got["scores"].astype(np.float64) - ref) <= 1e-5 * mag + 1e-6), f"scores, request {r}"
        Hp.check_topk(got["idx"], ref, wl.k, N, what=f"topk request {r}")
        sel = got["idx"][got["idx"] >= 0]
    else:
        sel = np.arange(N)
    kv = cache.read_rows(layer, r, 0, 0, N) if N else np.zeros((0, cache.row_bytes(0)), np.uint8)
    fp8, bf, sc = unpack_kv_rows(kv[sel] if len(sel) else kv[:0], wl.D, wl.R)
    ent = O.dequantize_kv(O.KVRow(fp8=fp8, rope=bf, scale=sc))
    wp = O.window_positions(t)
    fp8, bf, sc = unpack_kv_rows(cache.read_rows(layer, r, 2, wp[0], len(wp)), wl.D, wl.R)
    win = O.dequantize_kv(O.KVRow(fp8=fp8, rope=bf, scale=sc))
    rows = np.concatenate([ent, win], axis=0)
    ref_out = O.mqa_attention(O.rope(q[r].astype(np.float64), t, wl.R), rows, sink, 1.0 / math.sqrt(wl.D))
    Hp.check_attention(got["out_f"], ref_out, f"attention request {r}")


@pytest.mark.parametrize("name", ["csa-pro-1m", "csa-flash-128k", "hca-128k"])
def test_full_size_decode_step(name):
    wl = I.WORKLOADS[name]
    csa = wl.kind == "csa"
    B, T0 = wl.batch, wl.context
    pair = Hp.Pair(wl, 1 if csa else 0, 0 if csa else 1, max_req=B, capacity=T0 + 512)
    cache = pair.cache
    for r in range(B):
        cache.request_alloc(r, T0 + 512)
    dI = wl.d_I if csa else 0
    _fill(cache, 0, list(range(B)), {r: T0 for r in range(B)}, wl.seed, wl.D, dI)
    # the decode step's own token (host-generated), then the read path
    c, z = _host(wl.seed + 1, B, 1, wl.D), _host(wl.seed + 2, B, 1, wl.D)
    ci = _host(wl.seed + 3, B, 1, dI) if csa else None
    zi = _host(wl.seed + 4, B, 1, dI) if csa else None
    dev = lambda a: torch.from_numpy(a).cuda() if a is not None else None
    cache.compress_append(0, torch.arange(B, dtype=torch.int32, device="cuda"), dev(c), dev(z), dev(ci), dev(zi))
    q = I.bf16_grid(_host(wl.seed + 5, B, wl.H, wl.D))
    qi = _host(wl.seed + 6, B, wl.H_I, wl.d_I) if csa else None
    w = _host(wl.seed + 7, B, wl.H_I) if csa else None
    sink = pair.params[0]["sink"]
    # the compressor at these shapes (D = 512, R = 64, d_I = 128), against
    # the oracle on the same inputs, for the first and the last request
    _PARAMS[(wl.name, 0)] = pair.params[0]
    for r in (0, B - 1):
        _compressor_check(cache, wl, 0, r, wl.seed, T0, c[r], csa)
    base = _step(cache, wl, 0, list(range(B)), q, qi, w, sink)
    # oracle parity: every request of the small batches, four of the large ones
    check = list(range(B)) if B <= 4 else [0, 7, 18, B - 1]
    for r in check:
        _oracle_check(cache, wl, 0, r, T0 + 1, q, qi, w, sink, base[r])
    # the same requests in another order, and both launch variants: bit-exact
    order = list(np.random.default_rng(wl.seed).permutation(B))
    for variant in ("high", "low"):
        again = _step(cache, wl, 0, [int(x) for x in order], q, qi, w, sink, variant)
        for r in range(B):
            assert np.array_equal(again[r]["out"], base[r]["out"]), f"request {r} ({variant})"
            if csa:
                assert np.array_equal(again[r]["idx"], base[r]["idx"]), f"request {r} ({variant})"
                assert np.array_equal(again[r]["scores"].view(np.uint32), base[r]["scores"].view(np.uint32))


def test_ragged_sweep_batch_invariance():
    """Pro-like CSA (top-1024) and HCA layers, 16 requests with contexts
    log-uniform in [4K, 1M], three decode steps; each step runs the whole
    batch and sampled sub-batches (sizes 1 .. 16, shuffled positions, both
    variants): every request's bits agree across all of them."""
    wl_c, wl_h = I.C5_CSA, I.C5_HCA
    n_req = 16
    ctx = I.sweep_contexts(wl_c.seed, n_req, lo=4096, hi=1 << 20)
    cap = int(ctx.max()) + 512
    pair = Hp.Pair(wl_c, 1, 1, max_req=n_req, capacity=cap)
    cache = pair.cache
    for r in range(n_req):
        cache.request_alloc(r, int(ctx[r]) + 512)
    lens = {r: int(ctx[r]) for r in range(n_req)}
    _fill(cache, 0, list(range(n_req)), lens, wl_c.seed, wl_c.D, wl_c.d_I)
    _fill(cache, 1, list(range(n_req)), lens, wl_c.seed + 1, wl_c.D, 0)
    rng = np.random.default_rng(55)
    allr = list(range(n_req))
    for step in range(3):
        for layer, wl in ((0, wl_c), (1, wl_h)):
            csa = layer == 0
            c, z = _host(900 + step * 2 + layer, n_req, 1, wl.D), _host(950 + step * 2 + layer, n_req, 1, wl.D)
            ci = _host(990 + step, n_req, 1, wl.d_I) if csa else None
            zi = _host(995 + step, n_req, 1, wl.d_I) if csa else None
            dev = lambda a: torch.from_numpy(a).cuda() if a is not None else None
            cache.compress_append(layer, torch.arange(n_req, dtype=torch.int32, device="cuda"), dev(c), dev(z),
                                  dev(ci), dev(zi))
            q = I.bf16_grid(_host(700 + step * 2 + layer, n_req, wl.H, wl.D))
            qi = _host(800 + step, n_req, wl.H_I, wl.d_I) if csa else None
            w = _host(850 + step, n_req, wl.H_I) if csa else None
            sink = pair.params[layer]["sink"]
            base = _step(cache, wl, layer, allr, q, qi, w, sink)
            if step == 0:   # oracle parity on the shortest request of each layer
                r = int(np.argmin(ctx))
                _oracle_check(cache, wl, layer, r, lens[r] + 1, q, qi, w, sink, base[r])
            for size in (1, 3, 7, 16):
                sub = [int(x) for x in rng.choice(n_req, size=size, replace=False)]
                variant = ("high", "low", "auto")[int(rng.integers(0, 3))]
                again = _step(cache, wl, layer, sub, q, qi, w, sink, variant)
                for r in sub:
                    assert np.array_equal(again[r]["out"], base[r]["out"]), f"step {step} layer {layer} req {r}"
                    if csa:
                        assert np.array_equal(again[r]["idx"], base[r]["idx"])
        for r in allr:
            lens[r] += 1


def test_batch_larger_than_the_indexer_query_table():
    """300 requests in one batch (the indexer keeps per-query tile counts in
    shared memory for the first 256 and recomputes them beyond), Pro-like CSA
    and HCA layers, contexts log-uniform in [600, 20K]: the whole batch, its
    reverse and sub-batches agree bit for bit per request, and three requests
    (shortest, median, longest) match the oracle."""
    wl_c, wl_h = I.C5_CSA, I.C5_HCA
    n_req = 300
    ctx = I.sweep_contexts(wl_c.seed + 300, n_req, lo=600, hi=20000)
    cap = int(ctx.max()) + 64
    pair = Hp.Pair(wl_c, 1, 1, max_req=n_req, capacity=cap)
    cache = pair.cache
    for r in range(n_req):
        cache.request_alloc(r, int(ctx[r]) + 64)
    lens = {r: int(ctx[r]) for r in range(n_req)}
    _fill(cache, 0, list(range(n_req)), lens, wl_c.seed + 300, wl_c.D, wl_c.d_I)
    _fill(cache, 1, list(range(n_req)), lens, wl_c.seed + 301, wl_c.D, 0)
    allr = list(range(n_req))
    order_ctx = [int(x) for x in np.argsort(ctx, kind="stable")]
    probes = [order_ctx[0], order_ctx[n_req // 2], order_ctx[-1]]
    rng = np.random.default_rng(300)
    for layer, wl in ((0, wl_c), (1, wl_h)):
        csa = layer == 0
        c, z = _host(1300 + layer, n_req, 1, wl.D), _host(1350 + layer, n_req, 1, wl.D)
        ci = _host(1390, n_req, 1, wl.d_I) if csa else None
        zi = _host(1395, n_req, 1, wl.d_I) if csa else None
        dev = lambda a: torch.from_numpy(a).cuda() if a is not None else None
        cache.compress_append(layer, torch.arange(n_req, dtype=torch.int32, device="cuda"), dev(c), dev(z),
                              dev(ci), dev(zi))
        q = I.bf16_grid(_host(1400 + layer, n_req, wl.H, wl.D))
        qi = _host(1450, n_req, wl.H_I, wl.d_I) if csa else None
        w = _host(1460, n_req, wl.H_I) if csa else None
        sink = pair.params[layer]["sink"]
        base = _step(cache, wl, layer, allr, q, qi, w, sink)
        for r in probes:
            _oracle_check(cache, wl, layer, r, lens[r] + 1, q, qi, w, sink, base[r])
        subs = [allr[::-1], [int(x) for x in rng.choice(n_req, size=40, replace=False)], probes]
        for sub, variant in zip(subs, ("high", "low", "auto")):
            again = _step(cache, wl, layer, sub, q, qi, w, sink, variant)
            for r in sub:
                assert np.array_equal(again[r]["out"], base[r]["out"]), f"layer {layer} req {r} ({variant})"
                if csa:
                    assert np.array_equal(again[r]["idx"], base[r]["idx"]), f"layer {layer} req {r}"
                    assert np.array_equal(again[r]["scores"].view(np.uint32), base[r]["scores"].view(np.uint32))


def _pool_fill(cache, layer, reqs, lengths, pool, dI, group=32):
    """Append tokens 0 .. lengths[r]-1 of every request: the inputs of
    request r's chunk c (4096 tokens) are pool chunk (131 r + 7 c) mod P.
    Requests go in groups so that one call's stacked inputs stay small."""
    P = pool[0].shape[0]
    for g0 in range(0, len(reqs), group):
        grp = reqs[g0:g0 + group]
        t = 0
        while True:
            live = [r for r in grp if lengths[r] > t]
            if not live:
                break
            n_tok = min(min(lengths[r] for r in live) - t, I.CHUNK - t % I.CHUNK)
            c, lo = t // I.CHUNK, t % I.CHUNK
            idx = torch.tensor([(131 * r + 7 * c) % P for r in live], device="cuda")
            st = lambda k: pool[k][idx, lo:lo + n_tok].contiguous() if pool[k] is not None else None
            cache.compress_append(layer, torch.tensor(live, dtype=torch.int32, device="cuda"), st(0), st(1),
                                  st(2) if dI else None, st(3) if dI else None)
            t += n_tok
    torch.cuda.synchronize()
    cache.check_device_error()


def test_c5_ragged_sweep_at_scale():
    """The ragged batch-invariance sweep at its stated scale: interleaved
    CSA (top-1024) and HCA layers with Pro-like shapes, 256 requests with
    contexts log-uniform in [4K, 1M], 64 decode steps, each appending a token
    to every request (entries complete every 4th / 128th token).  Every step
    runs the whole batch, then sub-batches whose sizes span 1 .. 256 in
    shuffled order with random launch variants: every request's scores,
    indices and outputs must equal its whole-batch bits.  Eight probe
    requests (shortest, longest, quantiles) are checked against the oracle on
    the last step."""
    wl_c, wl_h = I.C5_CSA, I.C5_HCA
    n_req, n_steps = 256, 64
    ctx = I.sweep_contexts(wl_c.seed, n_req, lo=4096, hi=1 << 20)
    cap = int(ctx.max()) + n_steps + 512
    pair = Hp.Pair(wl_c, 1, 1, max_req=n_req, capacity=cap,
                   pool_blocks=int(sum((int(c) + n_steps + 8 + 511) // 512 for c in ctx)))
    cache = pair.cache
    for r in range(n_req):
        cache.request_alloc(r, int(ctx[r]) + n_steps + 8)
    lens = {r: int(ctx[r]) for r in range(n_req)}
    g = torch.Generator(device="cuda")
    g.manual_seed(5005)
    P = 24
    pool_c = [torch.randn((P, I.CHUNK, wl_c.D), generator=g, device="cuda") for _ in range(2)]
    pool_i = [torch.randn((P, I.CHUNK, wl_c.d_I), generator=g, device="cuda") for _ in range(2)]
    _pool_fill(cache, 0, list(range(n_req)), lens, (pool_c[0], pool_c[1], pool_i[0], pool_i[1]), wl_c.d_I)
    _pool_fill(cache, 1, list(range(n_req)), lens, (pool_c[1], pool_c[0], None, None), 0)
    del pool_c, pool_i
    order_ctx = [int(x) for x in np.argsort(ctx, kind="stable")]
    probes = [order_ctx[int(round(qq * (n_req - 1)))] for qq in (0, 1 / 7, 2 / 7, 3 / 7, 4 / 7, 5 / 7, 6 / 7, 1)]
    rng = np.random.default_rng(5)
    allr = list(range(n_req))
    sizes_seen = set()
    for step in range(n_steps):
        for layer, wl in ((0, wl_c), (1, wl_h)):
            csa = layer == 0
            gs = torch.Generator(device="cuda")
            gs.manual_seed(10_000 + 2 * step + layer)
            mk = lambda *shape: torch.randn(shape, generator=gs, device="cuda")
            c, z = mk(n_req, 1, wl.D), mk(n_req, 1, wl.D)
            ci = mk(n_req, 1, wl.d_I) if csa else None
            zi = mk(n_req, 1, wl.d_I) if csa else None
            cache.compress_append(layer, torch.arange(n_req, dtype=torch.int32, device="cuda"), c, z, ci, zi)
            q = mk(n_req, wl.H, wl.D).to(torch.bfloat16)
            qi = mk(n_req, wl.H_I, wl.d_I) if csa else None
            w = mk(n_req, wl.H_I) if csa else None
            sink = torch.from_numpy(pair.params[layer]["sink"]).cuda()

            def run(sub, variant):
                rid = torch.tensor(sub, dtype=torch.int32, device="cuda")
                ix = torch.tensor(sub, device="cuda")
                out = torch.empty((len(sub), wl.H, wl.D), dtype=torch.bfloat16, device="cuda")
                res = {"out": out}
                if csa:
                    ld = max(lens[r] + 1 for r in sub) // 4 + 128
                    sc = torch.full((len(sub), ld), float("nan"), device="cuda")
                    nv = torch.zeros(len(sub), dtype=torch.int32, device="cuda")
                    idx = torch.empty((len(sub), wl.k), dtype=torch.int32, device="cuda")
                    cache.index_topk(layer, rid, qi[ix].contiguous(), w[ix].contiguous(), sc, nv, wl.k, idx,
                                     variant=variant)
                    cache.decode_attn(layer, rid, q[ix].contiguous(), idx, sink, out, variant=variant)
                    res.update(sc=sc, nv=nv, idx=idx)
                else:
                    cache.decode_attn(layer, rid, q[ix].contiguous(), None, sink, out, variant=variant)
                cache.check_device_error()
                return res

            base = run(allr, "auto")
            n_sub = 3
            for s_ in range(n_sub):
                size = int([rng.integers(1, 9), rng.integers(9, 65), rng.integers(65, 257)][s_])
                if step == 0 and s_ == 0:
                    size = 1
                sizes_seen.add(size)
                sub = [int(x) for x in rng.choice(n_req, size=size, replace=False)]
                variant = ("high", "low", "auto")[int(rng.integers(0, 3))]
                got = run(sub, variant)
                pos = torch.tensor(sub, device="cuda")
                assert torch.equal(got["out"].view(torch.int16), base["out"][pos].view(torch.int16)), \
                    f"step {step} layer {layer} size {size} {variant}: outputs differ"
                if csa:
                    assert torch.equal(got["idx"], base["idx"][pos]), f"step {step}: indices differ"
                    assert torch.equal(got["nv"], base["nv"][pos])
                    ldm = min(got["sc"].shape[1], base["sc"].shape[1])
                    a_ = torch.nan_to_num(got["sc"][:, :ldm], nan=7.0).view(torch.int32)
                    b_ = torch.nan_to_num(base["sc"][pos][:, :ldm], nan=7.0).view(torch.int32)
                    assert torch.equal(a_, b_), f"step {step}: scores differ"
            if step == n_steps - 1:
                qh = q.float().cpu().numpy()
                qih = qi.cpu().numpy() if csa else None
                wh = w.cpu().numpy() if csa else None
                got_h = {}
                for r in probes:
                    x = allr.index(r)
                    d = {"out_f": base["out"][x].float().cpu().numpy()}
                    if csa:
                        nvr = int(base["nv"][x])
                        d.update(scores=base["sc"][x, :nvr].cpu().numpy(), idx=base["idx"][x].cpu().numpy())
                    got_h[r] = d
                for r in probes:
                    _oracle_check(cache, wl, layer, r, lens[r] + 1, qh, qih, wh, pair.params[layer]["sink"], got_h[r])
        for r in allr:
            lens[r] += 1
    assert 1 in sizes_seen and max(sizes_seen) > 64


@pytest.mark.parametrize("name", ["csa-pro-1m", "hca-pro-1m"])
def test_full_size_prefill_chunk_matches_decode(name):
    """A chunk of 128 queries per request (csa_prefill_chunk) at the
    production shapes (H = 128, D = 512, R = 64; CSA: H_I = 64, d_I = 128,
    k = 1024) equals, bit for bit, the same 128 tokens appended one at a time
    with a decode step after each, on a second cache filled identically;
    contexts of 5,000 to 131,071 tokens, so the chunk crosses CSA entries, an
    HCA block and (for the longest) the 2^17 boundary.  The chunk's last query
    of every request is also checked against the oracle over the stored rows."""
    wl = I.WORKLOADS[name]
    csa = wl.kind == "csa"
    lens = [70000, 131071, 5000]
    reqs = [1, 2, 0]
    n_tok = 128
    cap = max(lens) + n_tok + 64
    pairs = [Hp.Pair(wl, 1 if csa else 0, 0 if csa else 1, max_req=3, capacity=cap) for _ in range(2)]
    dI = wl.d_I if csa else 0
    for pair in pairs:
        for r in range(3):
            pair.cache.request_alloc(r, cap)
        _fill(pair.cache, 0, list(range(3)), {r: lens[r] for r in range(3)}, wl.seed, wl.D, dI)
    A, B = pairs[0].cache, pairs[1].cache
    sink = pairs[0].params[0]["sink"]
    sink_d = torch.from_numpy(sink).cuda()
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    c, z = _host(wl.seed + 11, 3, n_tok, wl.D), _host(wl.seed + 12, 3, n_tok, wl.D)
    ci = _host(wl.seed + 13, 3, n_tok, dI) if csa else None
    zi = _host(wl.seed + 14, 3, n_tok, dI) if csa else None
    q = I.bf16_grid(_host(wl.seed + 15, 3, n_tok, wl.H, wl.D))
    qi = _host(wl.seed + 16, 3, n_tok, wl.H_I, wl.d_I) if csa else None
    w = _host(wl.seed + 17, 3, n_tok, wl.H_I) if csa else None
    rid = torch.tensor(reqs, dtype=torch.int32, device="cuda")
    # the batch rows follow `reqs`
    sel = lambda a: a[reqs] if a is not None else None
    out = torch.empty((3, n_tok, wl.H, wl.D), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((3, n_tok, wl.k), dtype=torch.int32, device="cuda") if csa else None
    A.prefill_chunk(0, rid, dev(sel(c)), dev(sel(z)), dev(sel(ci)) if csa else None, dev(sel(zi)) if csa else None,
                    dev(sel(q)).to(torch.bfloat16), dev(sel(qi)) if csa else None, dev(sel(w)) if csa else None,
                    wl.k, sink_d, out, topk_out=idx)
    torch.cuda.synchronize()
    A.check_device_error()
    got = out.cpu().view(torch.int16)
    got_idx = idx.cpu() if csa else None
    for j in range(n_tok):
        B.compress_append(0, rid, dev(sel(c)[:, j:j + 1]), dev(sel(z)[:, j:j + 1]),
                          dev(sel(ci)[:, j:j + 1]) if csa else None, dev(sel(zi)[:, j:j + 1]) if csa else None)
        ref_idx = None
        if csa:
            ld = max(B.get_length(0, r) for r in reqs) // 4 + 128
            scores = torch.empty((3, ld), device="cuda")
            nv = torch.empty(3, dtype=torch.int32, device="cuda")
            B.index_scores(0, rid, dev(sel(qi)[:, j]), dev(sel(w)[:, j]), scores, nv)
            ref_idx = torch.empty((3, wl.k), dtype=torch.int32, device="cuda")
            topk(scores, nv, wl.k, ref_idx)
        ref = torch.empty((3, wl.H, wl.D), dtype=torch.bfloat16, device="cuda")
        B.decode_attn(0, rid, dev(sel(q)[:, j]).to(torch.bfloat16), ref_idx, sink_d, ref)
        torch.cuda.synchronize()
        B.check_device_error()
        assert torch.equal(got[:, j], ref.cpu().view(torch.int16)), f"token {j}: output differs"
        if csa:
            assert torch.equal(got_idx[:, j], ref_idx.cpu()), f"token {j}: top-k differs"
    # the oracle on the chunk's last query of every request, over the rows
    # the GPU stored (its whole window is in the ring after the chunk)
    for b, r in enumerate(reqs):
        T = lens[r] + n_tok
        last = dict(out_f=out[b, -1].float().cpu().numpy())
        qq = {r: q[r, -1]}
        if csa:
            N = T // 4
            nvv = torch.empty(1, dtype=torch.int32, device="cuda")
            sc = torch.empty((1, N + 128), device="cuda")
            B.index_scores(0, torch.tensor([r], dtype=torch.int32, device="cuda"), dev(qi[r, -1][None]),
                           dev(w[r, -1][None]), sc, nvv)
            torch.cuda.synchronize()
            last.update(scores=sc[0, :N].cpu().numpy(), idx=got_idx[b, -1].numpy())
            _oracle_check(A, wl, 0, r, T, qq, {r: qi[r, -1]}, {r: w[r, -1]}, sink, last)
        else:
            _oracle_check(A, wl, 0, r, T, qq, None, None, sink, last)
