"""Pin of the oracle's chunk of queries (prefill with causal visibility)
against a second, independent formulation: the whole context's entries
computed once, and each query's visible set cut out by an explicit causal
mask (entries completed by its own token; window max(0, t - 127) .. t;
RoPE at t).  A planted off-by-one in the oracle's visibility (the chunk
appended before its queries run) must fail the pin."""
import math

import numpy as np
import pytest

from compressed_sparse_long_hca_b200 import inputs as I
from oracle import csa_oracle as O

D, R, H, H_I, d_I, K = 64, 16, 4, 2, 32, 6
T0, N_TOK = 248, 12          # the chunk covers positions 248 .. 259: CSA entries at 251, 255, 259; HCA at 255


def _setup(kind, seed=31):
    b_kv, b_idx, sink = I.layer_params(seed, 0, kind, D, d_I, H)
    p = O.LayerParams(kind, D, R, b_kv, b_idx if kind == "csa" else None, m=4 if kind == "csa" else 128)
    tok = I.token_inputs(seed, 0, 0, 0, T0 + N_TOK, D, d_I if kind == "csa" else 0)
    rng = np.random.default_rng(seed)
    q = I.bf16_grid(rng.standard_normal((N_TOK, H, D)).astype(np.float32))
    qi = rng.standard_normal((N_TOK, H_I, d_I)).astype(np.float32)
    w = rng.standard_normal((N_TOK, H_I)).astype(np.float32)
    return p, tok, q, qi, w, sink


def _masked(p, tok, q, qi, w, sink):
    """Each query over the full context with an explicit causal mask."""
    full = O.RequestState()
    csa = p.kind == "csa"
    O.append_tokens(full, tok[0], tok[1], tok[2] if csa else None, tok[3] if csa else None)
    kvq, keyq = O.stored_entries(p, full)
    kv_all = O.dequantize_kv(kvq)
    n_all = kv_all.shape[0]
    scale = 1.0 / math.sqrt(D)
    outs, sels = [], []
    for j in range(N_TOK):
        t = T0 + j
        m = 4 if csa else 128
        visible = np.arange(n_all) * m + m - 1 <= t          # entry e is complete once token e m + m - 1 exists
        if csa:
            s = O.index_scores(O.dequantize_mxfp4(O.quantize_mxfp4(qi[j])), w[j], O.dequantize_mxfp4(keyq))
            cand = np.where(visible)[0]
            order = sorted(cand.tolist(), key=lambda e: (-s[e], e))[:K]
            sel = np.array(sorted(order), dtype=np.int64)
            sels.append(sel)
            rows = kv_all[sel]
        else:
            rows = kv_all[visible]
        win_pos = np.arange(max(0, t - 127), t + 1)
        win = O.dequantize_kv(O.quantize_kv(np.stack([O.raw_token_row(tok[0][tau], tau, R) for tau in win_pos]), R))
        qr = O.rope(q[j].astype(np.float64), t, R)
        outs.append(O.mqa_attention(qr, np.concatenate([rows, win]), sink, scale))
    return outs, sels


def _prefix_state(p, tok):
    st = O.RequestState()
    csa = p.kind == "csa"
    O.append_tokens(st, tok[0][:T0], tok[1][:T0], tok[2][:T0] if csa else None, tok[3][:T0] if csa else None)
    return st


def _chunk(tok, a, b):
    return [None if x is None else x[a:b] for x in tok]


@pytest.mark.parametrize("kind", ["csa", "hca"])
def test_chunk_queries_match_causal_mask(kind):
    p, tok, q, qi, w, sink = _setup(kind)
    csa = kind == "csa"
    st = _prefix_state(p, tok)
    c, z, ci, zi = _chunk(tok, T0, T0 + N_TOK)
    res = O.chunk_queries(p, st, c, z, ci if csa else None, zi if csa else None, q=q, sink=sink,
                          k=K if csa else None, q_idx=qi if csa else None, w=w if csa else None)
    ref, sels = _masked(p, tok, q, qi, w, sink)
    assert st.T == T0 + N_TOK
    for j in range(N_TOK):
        assert np.allclose(res[j]["out"], ref[j], rtol=1e-12, atol=1e-12), f"query {j}"
        if csa:
            assert np.array_equal(res[j]["topk"][res[j]["topk"] >= 0], sels[j]), f"query {j} selection"
    # the chunk's last query is the decode query after the whole chunk
    last = O.decode_query(p, st, q[-1], sink, k=K if csa else None, q_idx=qi[-1] if csa else None,
                          w=w[-1] if csa else None)
    assert np.array_equal(last["out"], res[-1]["out"])


@pytest.mark.parametrize("kind", ["csa", "hca"])
def test_planted_visibility_mistake_fails_the_pin(kind):
    """Plant the mistake in the oracle (on the CPU): every query of the chunk
    sees the whole chunk (the chunk appended first).  The causal-mask
    formulation must disagree for the early queries."""
    p, tok, q, qi, w, sink = _setup(kind)
    csa = kind == "csa"
    st = _prefix_state(p, tok)
    c, z, ci, zi = _chunk(tok, T0, T0 + N_TOK)
    O.append_tokens(st, c, z, ci if csa else None, zi if csa else None)
    ref, _ = _masked(p, tok, q, qi, w, sink)
    wrong = [O.decode_query(p, st, q[j], sink, k=K if csa else None, q_idx=qi[j] if csa else None,
                            w=w[j] if csa else None, T=T0 + j + 1, window=None) for j in range(N_TOK)]
    # with T given the window and RoPE follow position t, but the entries are
    # those of the whole chunk: queries before the last completed entry differ
    differs = [not np.allclose(wrong[j]["out"], ref[j], rtol=1e-9, atol=1e-9) for j in range(N_TOK)]
    assert any(differs[:N_TOK - 1])
    assert not differs[-1]
