"""Pins of the oracle's RoPE, compressor, indexer, top-k and attention against
closed forms, library routines and brute force on tiny inputs."""
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

from oracle import csa_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(s=0):
    return np.random.default_rng(s)


# ---------------------------------------------------------------- RoPE

def test_rope_matches_complex_rotation():
    r = _rng(1)
    D, R = 64, 16
    x = r.standard_normal((5, D))
    pos = np.array([0, 1, 17, 4096, 1048575])
    y = O.rope(x, pos, R)
    z = x[:, D - R::2] + 1j * x[:, D - R + 1::2]
    theta = 10000.0 ** (-np.arange(R // 2) * 2.0 / R)
    zr = z * np.exp(1j * pos[:, None] * theta[None, :])
    assert np.allclose(y[:, D - R::2], zr.real, atol=1e-12)
    assert np.allclose(y[:, D - R + 1::2], zr.imag, atol=1e-12)
    assert np.array_equal(y[:, : D - R], x[:, : D - R])          # no position on the rest
    assert np.array_equal(O.rope(x, 0, R), x)                   # identity at position 0
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1))


def test_rope_relative_position():
    r = _rng(2)
    q, k = r.standard_normal(32), r.standard_normal(32)
    a = O.rope(q, 100, 16) @ O.rope(k, 37, 16)
    b = O.rope(q, 100 + 5000, 16) @ O.rope(k, 37 + 5000, 16)
    assert abs(a - b) < 1e-9


# ---------------------------------------------------------------- compressor

def test_entry_counts_match_page_figures():
    # golden: figures printed on the pages, with their citations
    rows = {}
    for line in open(os.path.join(GOLDEN, "page_counts.txt"), encoding="utf-8"):
        if line.strip() and not line.startswith("#"):
            key, val = line.split("|")[0].split("=")
            rows[key.strip()] = int(val)
    T = rows["context_tokens"]
    assert O.n_csa_entries(T) == rows["csa_entries_exact"]
    assert abs(O.n_csa_entries(T) - rows["csa_entries_printed"]) / rows["csa_entries_printed"] < 0.05
    assert O.n_hca_entries(T) == rows["hca_entries_exact"]
    assert O.n_csa_entries(rows["block_tokens"]) == rows["csa_entries_per_block"]
    assert O.n_hca_entries(rows["block_tokens"]) == rows["hca_entries_per_block"]
    assert rows["block_tokens"] == math.lcm(4, 128)


def test_uniform_gate_gives_mean():
    r = _rng(3)
    T, D, dI = 40, 16, 32
    c, ci = r.standard_normal((T, D)), r.standard_normal((T, dI))
    z, zi = np.zeros((T, D)), np.zeros((T, dI))
    kv, key = O.csa_entries_all(c, z, ci, zi, np.zeros((8, D)), np.zeros((8, dI)), R=4)
    kv = O.rope(kv, -4 * np.arange(T // 4), 4)                  # undo the rotation
    assert np.allclose(kv[0], c[0:4].mean(0))                    # entry 0: its own 4 tokens
    assert np.allclose(key[0], ci[0:4].mean(0))
    for j in range(1, T // 4):
        assert np.allclose(kv[j], c[4 * j - 4: 4 * j + 4].mean(0))
        assert np.allclose(key[j], ci[4 * j - 4: 4 * j + 4].mean(0))
    h = O.hca_entries_all(np.repeat(c, 8, axis=0)[:256], np.zeros((256, D)),
                          np.zeros((128, D)), R=4)
    h = O.rope(h, -128 * np.arange(2), 4)
    assert np.allclose(h[1], np.repeat(c, 8, axis=0)[128:256].mean(0))


def test_one_hot_gate_copies_token():
    r = _rng(4)
    T, D = 16, 8
    c = r.standard_normal((T, D))
    z = np.zeros((T, D))
    z[6] = 1e4                        # token 6 is in the windows of entries 1 and 2
    kv, _ = O.csa_entries_all(c, z, c, z, np.zeros((8, D)), np.zeros((8, D)), R=2)
    kv = O.rope(kv, -4 * np.arange(T // 4), 2)
    assert np.allclose(kv[1], c[6]) and np.allclose(kv[2], c[6])


def test_scalar_gate_is_scipy_softmax():
    r = _rng(5)
    T, D = 12, 6
    c = r.standard_normal((T, D))
    zs = r.standard_normal(T)
    z = np.repeat(zs[:, None], D, axis=1)
    b = np.repeat(r.standard_normal(8)[:, None], D, axis=1)
    kv, _ = O.csa_entries_all(c, z, c, z, b, b, R=2)
    kv = O.rope(kv, -4 * np.arange(3), 2)
    g = scipy.special.softmax(zs[0:8] + b[:, 0])
    assert np.allclose(kv[1], g @ c[0:8])


def _brute_entry(c, z, b, taus, slots):
    """Per-channel softmax pooling written with explicit loops."""
    D = len(c[0])
    out = []
    for d in range(D):
        logits = [z[t][d] + b[s][d] for t, s in zip(taus, slots)]
        mx = max(logits)
        ws = [math.exp(v - mx) for v in logits]
        tot = sum(ws)
        out.append(sum(w / tot * c[t][d] for w, t in zip(ws, taus)))
    return out


def _brute_rope(x, pos, R):
    x = list(x)
    D = len(x)
    for i in range(R // 2):
        ang = pos * 10000.0 ** (-2.0 * i / R)
        a, b = x[D - R + 2 * i], x[D - R + 2 * i + 1]
        x[D - R + 2 * i] = a * math.cos(ang) - b * math.sin(ang)
        x[D - R + 2 * i + 1] = a * math.sin(ang) + b * math.cos(ang)
    return x


def test_compressor_brute_force_csa_and_hca():
    r = _rng(6)
    T, D, dI, R = 22, 6, 4, 2
    c, z = r.standard_normal((T, D)).tolist(), r.standard_normal((T, D)).tolist()
    ci, zi = r.standard_normal((T, dI)).tolist(), r.standard_normal((T, dI)).tolist()
    b, bi = r.standard_normal((8, D)).tolist(), r.standard_normal((8, dI)).tolist()
    kv, key = O.csa_entries_all(np.array(c), np.array(z), np.array(ci), np.array(zi),
                                np.array(b), np.array(bi), R=R)
    assert kv.shape[0] == T // 4
    for j in range(T // 4):
        taus = [t for t in range(4 * j - 4, 4 * j + 4) if t >= 0]
        slots = [t - (4 * j - 4) for t in taus]
        assert np.allclose(kv[j], _brute_rope(_brute_entry(c, z, b, taus, slots), 4 * j, R))
        assert np.allclose(key[j], _brute_entry(ci, zi, bi, taus, slots))
        kv1, key1 = O.csa_entry_vectors(np.array(c), np.array(z), np.array(ci), np.array(zi),
                                        np.array(b), np.array(bi), j, D, R)
        assert np.allclose(kv1, kv[j]) and np.allclose(key1, key[j])
    T2 = 300
    c2, z2 = r.standard_normal((T2, D)), r.standard_normal((T2, D))
    bh = r.standard_normal((128, D))
    h = O.hca_entries_all(c2, z2, bh, R=R)
    assert h.shape[0] == 2
    for j in range(2):
        taus = list(range(128 * j, 128 * j + 128))
        ref = _brute_rope(_brute_entry(c2.tolist(), z2.tolist(), bh.tolist(), taus,
                                       list(range(128))), 128 * j, R)
        assert np.allclose(h[j], ref)


# ---------------------------------------------------------------- indexer

def test_index_scores_brute_force():
    r = _rng(7)
    N, HI, dI = 30, 3, 8
    q, w, k = r.standard_normal((HI, dI)), r.standard_normal(HI), r.standard_normal((N, dI))
    s = O.index_scores(q, w, k)
    for j in range(N):
        ref = 0.0
        for h in range(HI):
            dot = sum(q[h][i] * k[j][i] for i in range(dI))
            ref += w[h] * (dot if dot > 0 else 0.0)
        assert abs(s[j] - ref) < 1e-12


def test_index_single_head_is_relu_dot():
    r = _rng(8)
    q, k = r.standard_normal((1, 16)), r.standard_normal((50, 16))
    assert np.allclose(O.index_scores(q, np.ones(1), k), np.maximum(k @ q[0], 0))


# ---------------------------------------------------------------- top-k

def test_topk_brute_force_with_ties():
    r = _rng(9)
    for trial in range(30):
        n = int(r.integers(1, 80))
        k = int(r.integers(1, 90))
        s = r.integers(-3, 4, n).astype(np.float64)             # many exact ties
        got = O.topk(s, k)
        ref = sorted(sorted(range(n), key=lambda j: (-s[j], j))[:k])
        ref = ref + [-1] * (k - len(ref))
        assert list(got) == ref


def test_topk_selects_all_when_k_exceeds_n():
    assert list(O.topk(np.array([0.5, 2.0, -1.0]), 5)) == [0, 1, 2, -1, -1]


# ---------------------------------------------------------------- attention

def _sdpa(q, rows):
    qt = torch.from_numpy(q)[None, :, None, :]                 # [1, H, 1, D]
    kt = torch.from_numpy(rows)[None, None].expand(1, q.shape[0], -1, -1)
    return torch.nn.functional.scaled_dot_product_attention(
        qt, kt, kt, scale=1.0 / math.sqrt(q.shape[1]))[0, :, 0].numpy()


def test_attention_without_sink_is_sdpa():
    r = _rng(10)
    q, rows = r.standard_normal((4, 32)), r.standard_normal((20, 32))
    o = O.mqa_attention(q, rows, np.full(4, -np.inf), 1.0 / math.sqrt(32))
    assert np.allclose(o, _sdpa(q, rows), atol=1e-12)


def test_attention_sink_is_extra_zero_value_key():
    # a sink logit in the denominator equals attending to one extra key whose
    # logit is the sink and whose value is zero
    r = _rng(11)
    H, D, n = 3, 16, 9
    q, rows, sink = r.standard_normal((H, D)), r.standard_normal((n, D)), r.standard_normal(H)
    scale = 1.0 / math.sqrt(D)
    o = O.mqa_attention(q, rows, sink, scale)
    for h in range(H):
        qa = np.concatenate([q[h], [sink[h] / scale]])
        K = np.concatenate([np.concatenate([rows, np.zeros((n, 1))], 1),
                            np.concatenate([np.zeros((1, D)), [[1.0]]], 1)], 0)
        V = np.concatenate([rows, np.zeros((1, D))], 0)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(qa)[None, None], torch.from_numpy(K)[None],
            torch.from_numpy(V)[None], scale=scale)[0, 0].numpy()
        assert np.allclose(o[h], ref, atol=1e-12)


def test_attention_single_row_closed_form():
    r = _rng(12)
    q, v, sink = r.standard_normal((2, 8)), r.standard_normal((1, 8)), np.array([0.3, -2.0])
    o = O.mqa_attention(q, v, sink, 0.5)
    u = 0.5 * q @ v[0]
    ref = v[0][None] * (np.exp(u) / (np.exp(u) + np.exp(sink)))[:, None]
    assert np.allclose(o, ref)


def test_attention_brute_force_loops():
    r = _rng(13)
    H, D, n = 2, 5, 7
    q, rows, sink = r.standard_normal((H, D)), r.standard_normal((n, D)), r.standard_normal(H)
    o = O.mqa_attention(q, rows, sink, 0.7)
    for h in range(H):
        u = [0.7 * sum(q[h][d] * rows[i][d] for d in range(D)) for i in range(n)]
        den = sum(math.exp(x) for x in u) + math.exp(sink[h])
        for d in range(D):
            assert abs(o[h][d] - sum(math.exp(u[i]) * rows[i][d] for i in range(n)) / den) < 1e-12


# ---------------------------------------------------------------- whole step

def _tiny_layer(kind, r, D=32, R=8, dI=32):
    if kind == "csa":
        return O.LayerParams("csa", D, R, r.standard_normal((8, D)), r.standard_normal((8, dI)))
    return O.LayerParams("hca", D, R, r.standard_normal((128, D)), None, m=128)


def test_csa_with_k_at_least_entries_is_dense():
    r = _rng(14)
    p = _tiny_layer("csa", r)
    st = O.RequestState()
    T = 203
    O.append_tokens(st, r.standard_normal((T, 32)), r.standard_normal((T, 32)),
                    r.standard_normal((T, 32)), r.standard_normal((T, 32)))
    q = O.bf16_round(r.standard_normal((4, 32)))
    sink = r.standard_normal(4)
    res = O.decode_query(p, st, q, sink, k=T // 4 + 7, q_idx=r.standard_normal((2, 32)),
                         w=r.standard_normal(2))
    assert list(res["topk"][: T // 4]) == list(range(T // 4))
    assert np.all(res["topk"][T // 4:] == -1)
    kvq, _ = O.stored_entries(p, st)
    rows = np.concatenate([O.dequantize_kv(kvq), O.dequantize_kv(O.stored_window(p, st, T - 1))])
    dense = O.mqa_attention(O.rope(q, T - 1, 8), rows, sink, 1.0 / math.sqrt(32))
    assert np.allclose(res["out"], dense)
    assert res["n_rows"] == T // 4 + 128


def test_window_visibility():
    assert O.window_positions(0) == [0]
    assert O.window_positions(127) == list(range(128))
    assert O.window_positions(1000) == list(range(873, 1001))


def _stored_value(x, R, fmt):
    """What a stored vector stands for: its fp32 rounding (fp32 format), or
    its FP8 + BF16 quantisation (mixed format)."""
    x = np.asarray(x, np.float64)[None]
    if fmt == "f32":
        return np.array([float(np.float32(v)) for v in x[0]])
    return O.dequantize_kv(O.quantize_kv(x, R))[0]


@pytest.mark.parametrize("fmt", ["mixed", "f32"])
def test_decode_brute_force_tiny(fmt):
    """The whole CSA step, written out with loops over positions for a tiny
    context, against decode_query, in both storage formats (fp32: stored
    vectors and the index query rounded to fp32, no quantiser)."""
    r = _rng(15)
    D, R, dI, H, HI, k, T = 32, 8, 32, 2, 2, 3, 45
    p = _tiny_layer("csa", r, D, R, dI)
    p.W = 8
    p.fmt = fmt
    st = O.RequestState()
    c, z = r.standard_normal((T, D)), r.standard_normal((T, D))
    ci, zi = r.standard_normal((T, dI)), r.standard_normal((T, dI))
    O.append_tokens(st, c, z, ci, zi)
    q = O.bf16_round(r.standard_normal((H, D)))
    qi, w, sink = r.standard_normal((HI, dI)), r.standard_normal(HI), r.standard_normal(H)
    res = O.decode_query(p, st, q, sink, k=k, q_idx=qi, w=w)
    t = T - 1
    # entries, one by one
    keys, kvs = [], []
    for j in range((t + 1) // 4):
        taus = [x for x in range(4 * j - 4, 4 * j + 4) if x >= 0]
        slots = [x - (4 * j - 4) for x in taus]
        kv = _brute_rope(_brute_entry(c.tolist(), z.tolist(), p.b_kv.tolist(), taus, slots), 4 * j, R)
        kvs.append(_stored_value(kv, R, fmt))
        kk = _brute_entry(ci.tolist(), zi.tolist(), p.b_idx.tolist(), taus, slots)
        if fmt == "f32":
            keys.append(np.array([float(np.float32(v)) for v in kk]))
        else:
            keys.append(O.dequantize_mxfp4(O.quantize_mxfp4(np.array(kk)[None]))[0])
    if fmt == "f32":
        qd = np.array([[float(np.float32(v)) for v in row] for row in qi])
    else:
        qd = O.dequantize_mxfp4(O.quantize_mxfp4(qi))
    scores = []
    for j in range(len(keys)):
        s = 0.0
        for h in range(HI):
            s += w[h] * max(0.0, float(np.dot(qd[h], keys[j])))
        scores.append(s)
    assert np.allclose(res["scores"], scores)
    sel = sorted(sorted(range(len(scores)), key=lambda j: (-scores[j], j))[:k])
    assert list(res["topk"]) == sel
    rows = [kvs[j] for j in sel]
    for tau in range(max(0, t - p.W + 1), t + 1):
        rows.append(_stored_value(_brute_rope(c[tau], tau, R), R, fmt))
    qr = np.array([_brute_rope(q[h], t, R) for h in range(H)])
    for h in range(H):
        u = [qr[h] @ row / math.sqrt(D) for row in rows]
        mu = max(max(u), sink[h])
        den = sum(math.exp(x - mu) for x in u) + math.exp(sink[h] - mu)
        o = sum(math.exp(u[i] - mu) * rows[i] for i in range(len(rows))) / den
        assert np.allclose(res["out"][h], o)


def _hca_brute_step(c, z, bh, q, sink, T, D, R, W, fmt="mixed"):
    """The HCA step written out with loops: every completed 128-token entry
    pooled per channel (softmax over the block's tokens), rotated at its
    first token and stored; the window's raw tokens rotated at their own
    positions and stored; attention of every head over entries then window,
    with the sink in the denominator."""
    t = T - 1
    rows = []
    for j in range(T // 128):                      # only blocks whose 128 tokens have all arrived
        taus = list(range(128 * j, 128 * j + 128))
        kv = _brute_rope(_brute_entry(c.tolist(), z.tolist(), bh.tolist(), taus, list(range(128))), 128 * j, R)
        rows.append(_stored_value(kv, R, fmt))
    n_ent = len(rows)
    for tau in range(max(0, t - W + 1), t + 1):
        rows.append(_stored_value(_brute_rope(c[tau], tau, R), R, fmt))
    out = np.zeros((q.shape[0], D))
    for h in range(q.shape[0]):
        qr = np.array(_brute_rope(q[h], t, R))
        u = [float(qr @ row) / math.sqrt(D) for row in rows]
        mu = max(max(u), sink[h])
        den = sum(math.exp(x - mu) for x in u) + math.exp(sink[h] - mu)
        out[h] = sum(math.exp(u[i] - mu) * rows[i] for i in range(len(rows))) / den
    return out, n_ent


@pytest.mark.parametrize("fmt", ["mixed", "f32"])
@pytest.mark.parametrize("T", [130, 255, 256, 300])
def test_hca_decode_brute_force_tiny(T, fmt):
    """The HCA branch of decode_query (dense over every completed 128:1 entry,
    then the window) against loops: a block counts only once all its 128
    tokens have arrived (T = 255 sees one entry, T = 256 two), and the window
    is the last W raw tokens."""
    r = _rng(16)
    D, R, H = 16, 4, 2
    p = _tiny_layer("hca", r, D, R)
    p.W = 8
    p.fmt = fmt
    c, z = r.standard_normal((T, D)), r.standard_normal((T, D))
    st = O.RequestState()
    O.append_tokens(st, c, z)
    q = O.bf16_round(r.standard_normal((H, D)))
    sink = r.standard_normal(H)
    res = O.decode_query(p, st, q, sink)
    ref, n_ent = _hca_brute_step(c, z, p.b_kv, q, sink, T, D, R, p.W, fmt)
    assert n_ent == T // 128
    assert res["n_rows"] == n_ent + min(T, p.W)
    assert np.allclose(res["out"], ref, atol=1e-12)


def test_hca_equals_csa_with_k_at_least_entries():
    """With the same stored entries and window, the HCA branch (dense) gives
    exactly what the CSA branch gives when k >= the number of entries (every
    entry selected, in index order)."""
    r = _rng(17)
    D, R, H, dI = 32, 8, 4, 32
    N, T = 37, 37 * 128 + 50
    ent = O.quantize_kv(r.standard_normal((N, D)), R)
    win = O.quantize_kv(r.standard_normal((128, D)), R)
    keys = O.quantize_mxfp4(r.standard_normal((N, dI)))
    q = O.bf16_round(r.standard_normal((H, D)))
    sink = r.standard_normal(H)
    ph = _tiny_layer("hca", r, D, R)
    pc = _tiny_layer("csa", r, D, R, dI)
    oh = O.decode_query(ph, None, q, sink, entries=(ent, None), window=win, T=T)
    for k in (N, N + 5):
        oc = O.decode_query(pc, None, q, sink, k=k, q_idx=r.standard_normal((2, dI)), w=r.standard_normal(2),
                            entries=(ent, keys), window=win, T=T)
        assert list(oc["topk"][:N]) == list(range(N))
        assert np.array_equal(oh["out"], oc["out"])
        assert oh["n_rows"] == oc["n_rows"] == N + 128


# ---------------------------------------------------------------- projections

def test_linear_brute_force_and_one_hot():
    r = _rng(18)
    x, W = r.standard_normal((3, 7)), r.standard_normal((5, 7))
    y = O.linear(x, W)
    for t in range(3):
        for o in range(5):
            assert abs(y[t, o] - sum(x[t][k] * W[o][k] for k in range(7))) < 1e-12
    P = np.zeros((4, 7))
    for o, k in enumerate([6, 0, 3, 3]):
        P[o, k] = 1.0                      # one-hot rows copy columns exactly
    assert np.array_equal(O.linear(x, P), x[:, [6, 0, 3, 3]])


def test_grouped_linear_is_block_diagonal_dense():
    r = _rng(19)
    groups, rg, kg = 4, 3, 5
    x, W = r.standard_normal((2, groups * kg)), r.standard_normal((groups * rg, kg))
    dense = np.zeros((groups * rg, groups * kg))
    for g in range(groups):
        dense[g * rg:(g + 1) * rg, g * kg:(g + 1) * kg] = W[g * rg:(g + 1) * rg]
    assert np.allclose(O.grouped_linear(x, W, groups), O.linear(x, dense), atol=1e-12)
    assert np.allclose(O.grouped_linear(x, W, 1)[:, :rg], O.linear(x[:, :kg], W[:rg]))
