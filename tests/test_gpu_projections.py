"""A decode step fed by the batch-invariant projections and followed by the
grouped output projection, on the tiny configuration's shapes (hidden 256,
8 heads x 64, RoPE 16, indexer 4 x 32, top-16) with one CSA and one HCA
layer: hidden states -> projections (csa_gemm_bf16) -> append -> fused index
+ top-k -> attention -> grouped output projection, each stage against the
oracle on the GPU's own inputs to that stage (read back), so a wrong stage
fails at that stage."""
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


def _w(seed, rows, cols, f):
    return I.bf16_grid(I.normal((rows, cols), seed, 98, f) / np.float32(math.sqrt(cols)))


def _gemm_ok(gpu, x, W, what, bf16_out=False, groups=1):
    """fp32 accumulation over K: |gpu - ref| <= 2e-5 sum_k |x_k w_k|, plus
    half a BF16 ulp of the result for a BF16 output."""
    lin = (lambda a, b: O.grouped_linear(a, b, groups)) if groups > 1 else O.linear
    ref = lin(x, W)
    mag = lin(np.abs(x), np.abs(W))
    bound = 2e-5 * mag + (np.abs(ref) * 2.0 ** -8 if bf16_out else 0.0) + 1e-30
    err = np.abs(np.asarray(gpu, np.float64).reshape(ref.shape) - ref)
    assert np.all(err <= bound), f"{what}: worst {float((err / (mag + 1e-30)).max()):.3e}"


def test_projected_decode_step_stage_by_stage():
    from compressed_sparse_long_hca_b200.api import LayerProjections, Linear, OutputProjection
    wl = I.C1
    d, D, R, H, H_I, d_I, d_c, k = wl.hidden, wl.D, wl.R, wl.H, wl.H_I, wl.d_I, 64, wl.k
    T = wl.context
    seed = wl.seed + 7
    pair = Hp.Pair(wl, 1, 1, max_req=1, capacity=T + 64)
    pair.cache.request_alloc(0, T + 64)
    h = I.bf16_grid(I.normal((T + 1, d), seed, 0, 0, 5))
    hd = torch.from_numpy(h).cuda().to(torch.bfloat16)
    rid = torch.zeros(1, dtype=torch.int32, device="cuda")
    outs = []
    for layer in (0, 1):
        csa = layer == 0
        f = 10 * layer
        Wd = dict(W_c=_w(seed, D, d, f + 1), W_z=_w(seed, D, d, f + 2), W_dq=_w(seed, d_c, d, f + 3),
                  W_uq=_w(seed, H * D, d_c, f + 4))
        if csa:
            Wd.update(W_cI=_w(seed, d_I, d, f + 5), W_zI=_w(seed, d_I, d, f + 6), W_w=_w(seed, H_I, d, f + 7),
                      W_uqI=_w(seed, H_I * d_I, d_c, f + 8))
        P = LayerProjections(csa=csa, **Wd)
        # ---- projections + append, in ragged chunks of the prefix and the decode token alone
        got = []
        bounds = [0, 1, 250, 251, 700, T, T + 1]
        for t0, t1 in zip(bounds[:-1], bounds[1:]):
            n = t1 - t0
            o = P.new_outputs(n, H)
            P(hd[t0:t1].contiguous(), o)
            v = lambda x: x.view(1, n, -1)
            pair.cache.compress_append(layer, rid, v(o["c"]), v(o["z"]), v(o["ci"]) if csa else None,
                                       v(o["zi"]) if csa else None)
            got.append({key: t.float().cpu().numpy().reshape(n, -1) for key, t in o.items()})
        torch.cuda.synchronize()
        Linear.check_device_error()
        pair.cache.check_device_error()
        cat = {key: np.concatenate([g[key] for g in got]) for key in got[0]}
        _gemm_ok(cat["c"], h, Wd["W_c"], f"layer {layer} c")
        _gemm_ok(cat["z"], h, Wd["W_z"], f"layer {layer} z")
        _gemm_ok(cat["c_q"], h, Wd["W_dq"], f"layer {layer} c_q", bf16_out=True)
        _gemm_ok(cat["q"], cat["c_q"], Wd["W_uq"], f"layer {layer} q", bf16_out=True)
        if csa:
            _gemm_ok(cat["ci"], h, Wd["W_cI"], "c_I")
            _gemm_ok(cat["zi"], h, Wd["W_zI"], "z_I")
            _gemm_ok(cat["w"], h, Wd["W_w"], "w")
            _gemm_ok(cat["q_idx"], cat["c_q"], Wd["W_uqI"], "q_I")
        # batch invariance: the decode token's projections computed alone
        # equal, bit for bit, the same token's projections inside a batch
        o_big = P.new_outputs(300, H)
        P(hd[T - 299:T + 1].contiguous(), o_big)
        for key in got[-1]:
            assert np.array_equal(o_big[key][-1:].float().cpu().numpy().reshape(1, -1), got[-1][key]), key
        # ---- the oracle on the GPU's projected inputs
        p = pair.oracle_params(layer)
        st = O.RequestState()
        O.append_tokens(st, cat["c"], cat["z"], cat["ci"] if csa else None, cat["zi"] if csa else None)
        q = cat["q"][T].reshape(H, D)
        sink = pair.params[layer]["sink"]
        out = torch.empty((1, H, D), dtype=torch.bfloat16, device="cuda")
        qd = torch.from_numpy(q[None]).cuda().to(torch.bfloat16)
        if csa:
            N = (T + 1) // 4
            kv_ref, key_ref = O.csa_entries_all(cat["c"], cat["z"], cat["ci"], cat["zi"], p.b_kv, p.b_idx, R)
            Hp.check_kv_rounding(pair.cache.read_rows(0, 0, 0, 0, N), kv_ref, D, R, "projected entries")
            same_key = Hp.check_index_rounding(pair.cache.read_rows(0, 0, 1, 0, N), key_ref, d_I, "projected keys")
            qi, w = cat["q_idx"][T].reshape(H_I, d_I), cat["w"][T]
            scores = torch.full((1, N + 9), float("nan"), device="cuda")
            nv = torch.zeros(1, dtype=torch.int32, device="cuda")
            idx = torch.empty((1, k), dtype=torch.int32, device="cuda")
            pair.cache.index_topk(0, rid, torch.from_numpy(qi[None]).cuda(), torch.from_numpy(w[None]).cuda(),
                                  scores, nv, k, idx)
            pair.cache.decode_attn(0, rid, qd, idx, torch.from_numpy(sink).cuda(), out)
            pair.cache.check_device_error()
            res = O.decode_query(p, st, q, sink, k=k, q_idx=qi, w=w)
            assert int(nv[0]) == N
            Hp.check_topk(idx[0].cpu().numpy(), res["scores"], k, N, excused=np.where(~same_key)[0],
                          what="projected top-k")
            sel = idx[0].cpu().numpy()
        else:
            N = (T + 1) // 128
            kv_ref = O.hca_entries_all(cat["c"], cat["z"], p.b_kv, R)
            Hp.check_kv_rounding(pair.cache.read_rows(1, 0, 0, 0, N), kv_ref, D, R, "projected HCA entries")
            pair.cache.decode_attn(1, rid, qd, None, torch.from_numpy(sink).cuda(), out)
            pair.cache.check_device_error()
            res = O.decode_query(p, st, q, sink)
            sel = np.arange(N)
        got_out = out[0].float().cpu().numpy()
        Hp.check_attention(got_out, Hp.attention_over_stored_rows(pair.cache, layer, 0, T, sel, q, sink, D, R),
                           f"layer {layer} attention (stored rows)")
        if not csa or set(sel.tolist()) == set(res["topk"].tolist()):
            Hp.check_attention(got_out, res["out"], f"layer {layer} attention")
        outs.append(out)
    # ---- grouped output projection of both layers' outputs (batch of 2)
    groups, d_model = 2, 384
    W_g = _w(seed, groups * 128, (H // groups) * D, 31)
    W_o = _w(seed, d_model, groups * 128, 32)
    op = OutputProjection(W_g, W_o, groups)
    a = torch.cat(outs).contiguous()
    mid = torch.empty((2, groups * 128), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((2, d_model), device="cuda")
    op(a, mid, y)
    Linear.check_device_error()
    a_h = a.float().cpu().numpy().reshape(2, -1)
    mid_h = mid.float().cpu().numpy()
    _gemm_ok(mid_h, a_h, W_g, "grouped projection", bf16_out=True, groups=groups)
    _gemm_ok(y.cpu().numpy(), mid_h, W_o, "output projection")
