"""Shared test helpers: build caches, drive both the CUDA library and the
oracle from the same seeded inputs, and compare their results.

Test infrastructure: imports the oracle; nothing on the product path imports
this module."""
from __future__ import annotations

import math

import numpy as np

from compressed_sparse_long_hca_b200 import inputs as I
from oracle import csa_oracle as O

# ---------------------------------------------------------------- tolerances
# Attention output (BF16).  Outputs are compared after scaling them to O(1)
# by the reference's RMS sigma, elementwise in the allclose form
#     |gpu - ref| <= ATT_ATOL * sigma + ATT_RTOL * |ref|.
ATT_ATOL = 1e-2
ATT_RTOL = 2e-2
TOPK_TIE_REL = 1e-3     # oracle scores within this of the k-th score are a tie zone
# Attention output in the fp32 storage format: fp32 operands and fp32 FMA
# chains.  A logit's error is about D * 2^-24 * sum|q_d k_d| (< 1e-5 for the
# tiny configuration), which moves an output by ~1e-5 relative; the bound
# below leaves a factor of about 10.
F32_ATT_ATOL = 1e-4
F32_ATT_RTOL = 1e-4


def check_attention(gpu: np.ndarray, ref: np.ndarray, what: str = "attention", fmt: str = "mixed") -> float:
    """Returns the largest |gpu - ref| / sigma seen."""
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    sigma = math.sqrt(float(np.mean(ref ** 2))) or 1.0
    err = np.abs(gpu - ref)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite output"
    atol, rtol = (F32_ATT_ATOL, F32_ATT_RTOL) if fmt == "f32" else (ATT_ATOL, ATT_RTOL)
    bad = err > atol * sigma + rtol * np.abs(ref)
    assert not bad.any(), (f"{what}: {int(bad.sum())} elements outside tolerance; worst "
                           f"|err|/sigma {err.max() / sigma:.3e}")
    return float(err.max() / sigma)


def check_kv_rounding(gpu_rows: np.ndarray, ref_vals: np.ndarray, D: int, R: int, what="kv",
                      min_exact=0.999, ref_codes: O.KVRow | None = None) -> None:
    """Stored KV rows must be a valid rounding of the oracle's fp64 vectors;
    the codes must equal the oracle's own codes almost everywhere (they can
    differ only where fp32 and fp64 pooling fall on two sides of a rounding
    midpoint)."""
    from compressed_sparse_long_hca_b200.api import unpack_kv_rows
    fp8, bf, sc = unpack_kv_rows(gpu_rows, D, R)
    v = O.dequantize_kv(O.KVRow(fp8=fp8, rope=bf, scale=sc))
    x = np.asarray(ref_vals, np.float64)
    ref = ref_codes if ref_codes is not None else O.quantize_kv(x, R)
    nope_err = np.abs(v[:, : D - R] - x[:, : D - R])
    bound = (np.abs(x[:, : D - R]) * 2.0 ** -4 + ref.scale.astype(np.float64)[:, None] * 2.0 ** -10) * 1.001 + 1e-30
    assert np.all(nope_err <= bound), f"{what}: FP8 part outside the rounding bound"
    rope_err = np.abs(v[:, D - R:] - x[:, D - R:])
    # BF16 rounds to half an ulp (2^-9 relative; 2^-8 allowed).  The kernels
    # pool in fp32 and the oracle in fp64, so a pooled or rotated value near
    # zero (cancellation) also carries an absolute error of a few fp32 ulps
    # of the row's magnitudes: 2^-18 x the row's RMS covers it (simulated
    # worst case on 25.6M values: 2.7e-7 x RMS).
    rms = np.sqrt(np.mean(x ** 2, axis=1, keepdims=True))
    assert np.all(rope_err <= np.abs(x[:, D - R:]) * 2.0 ** -8 * 1.001 + 2.0 ** -18 * rms + 1e-30), \
        f"{what}: BF16 part outside bound"
    same = (fp8 == ref.fp8).all(1) & (bf == ref.rope).all(1) & (sc == ref.scale)
    frac_elem = ((fp8 == ref.fp8).mean() + (bf == ref.rope).mean()) / 2
    assert frac_elem >= min_exact, f"{what}: only {frac_elem:.5f} of codes equal the oracle's"
    return same


def check_index_rounding(gpu_rows: np.ndarray, ref_vals: np.ndarray, d_I: int, what="index",
                         min_exact=0.999):
    from compressed_sparse_long_hca_b200.api import unpack_index_rows
    codes, scales = unpack_index_rows(gpu_rows, d_I)
    v = O.dequantize_mxfp4(O.MXFP4(codes=codes, scales=scales))
    x = np.asarray(ref_vals, np.float64)
    ref = O.quantize_mxfp4(x)
    e = np.repeat(np.exp2(ref.scales.astype(np.float64) - 127), 32, axis=1)
    err = np.abs(v - x)
    assert np.all(err <= np.maximum(0.25 * np.abs(x), 0.25 * e) * 1.001 + 1e-30), f"{what}: outside bound"
    frac = (codes == ref.codes).mean()
    assert frac >= min_exact, f"{what}: only {frac:.5f} of codes equal the oracle's"
    same = (codes == ref.codes).all(1) & (scales == ref.scales).all(1)
    return same


def check_topk(gpu_idx: np.ndarray, ref_scores: np.ndarray, k: int, n_valid: int,
               excused=None, what="topk") -> bool:
    """GPU top-k vs the oracle's: identical except for entries whose oracle
    score lies within TOPK_TIE_REL of the k-th score (or entries listed in
    `excused`).  Also checks the output's form.  Returns True when the two
    index sets are identical."""
    g = [int(x) for x in gpu_idx]
    sel = [x for x in g if x >= 0]
    assert all(x == -1 for x in g[len(sel):]), f"{what}: -1 padding not at the end"
    assert sel == sorted(sel) and len(set(sel)) == len(sel), f"{what}: not ascending/unique"
    assert len(sel) == min(k, n_valid), f"{what}: wrong count"
    assert all(0 <= x < n_valid for x in sel)
    ref = O.topk(ref_scores[:n_valid], k)
    rset = set(int(x) for x in ref if x >= 0)
    gset = set(sel)
    if gset == rset:
        return True
    kth = np.sort(ref_scores[:n_valid])[::-1][min(k, n_valid) - 1]
    zone = TOPK_TIE_REL * abs(kth) + 1e-6
    ex = set(excused or ())
    for j in gset ^ rset:
        assert abs(ref_scores[j] - kth) <= zone or j in ex, \
            f"{what}: entry {j} (score {ref_scores[j]:.6g}, k-th {kth:.6g}) differs outside the tie zone"
    return False


# ---------------------------------------------------------------- driving both sides

class Pair:
    """One CUDA cache plus the oracle's state for the same requests."""

    def __init__(self, wl: I.Workload, n_csa: int, n_hca: int, max_req: int, capacity: int,
                 pool_blocks: int | None = None, fmt: str = "mixed"):
        import torch
        from compressed_sparse_long_hca_b200.api import Cache
        self.wl = wl
        self.fmt = fmt
        self.n_csa, self.n_hca = n_csa, n_hca
        self.params = []
        bkv, bix, bh = [], [], []
        for layer in range(n_csa + n_hca):
            kind = "csa" if layer < n_csa else "hca"
            b, bi, sink = I.layer_params(wl.seed, layer, kind, wl.D, wl.d_I or 32, wl.H)
            self.params.append(dict(kind=kind, b_kv=b, b_idx=bi, sink=sink))
            if kind == "csa":
                bkv.append(b)
                bix.append(bi)
            else:
                bh.append(b)
        nb = (capacity + 511) // 512
        self.cache = Cache(n_csa=n_csa, n_hca=n_hca, H=wl.H, D=wl.D, D_rope=wl.R,
                           H_I=wl.H_I or 1, d_I=wl.d_I or 32, max_requests=max_req,
                           max_pages_per_request=nb, pool_pages=pool_blocks or nb * max_req,
                           b_pos_csa=np.stack(bkv) if bkv else None,
                           b_pos_idx=np.stack(bix) if bix else None,
                           b_pos_hca=np.stack(bh) if bh else None, fmt=fmt)
        self.torch = torch
        self.states = {}   # (layer, req) -> O.RequestState

    def oracle_params(self, layer: int) -> O.LayerParams:
        p = self.params[layer]
        if p["kind"] == "csa":
            return O.LayerParams("csa", self.wl.D, self.wl.R, p["b_kv"], p["b_idx"], fmt=self.fmt)
        return O.LayerParams("hca", self.wl.D, self.wl.R, p["b_kv"], None, m=128, fmt=self.fmt)

    def append(self, layer: int, reqs, tokens: dict, n_tok: int, stream=None, oracle=True):
        """Append n_tok tokens to each request in `reqs`; tokens[req] = (c, z, ci, zi)."""
        torch = self.torch
        csa = layer < self.n_csa
        dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
        c = dev(np.stack([tokens[r][0] for r in reqs]))
        z = dev(np.stack([tokens[r][1] for r in reqs]))
        ci = dev(np.stack([tokens[r][2] for r in reqs])) if csa else None
        zi = dev(np.stack([tokens[r][3] for r in reqs])) if csa else None
        rid = torch.tensor(reqs, dtype=torch.int32, device="cuda")
        self.cache.compress_append(layer, rid, c, z, ci, zi, stream=stream)
        if oracle:
            for r in reqs:
                st = self.states.setdefault((layer, r), O.RequestState())
                cc, zz, cci, zzi = tokens[r]
                O.append_tokens(st, cc, zz, cci if csa else None, zzi if csa else None)

    def gen_tokens(self, layer: int, req: int, start: int, count: int):
        return I.token_inputs(self.wl.seed, layer, req, start, count, self.wl.D,
                              self.wl.d_I if layer < self.n_csa else 0)


def attention_over_stored_rows(cache, layer: int, req: int, t: int, sel, q, sink, D: int, R: int,
                               scale: float | None = None) -> np.ndarray:
    """The oracle's attention for the query at position t over the rows the
    GPU path attends to: the stored entries listed in `sel` (the GPU's own
    top-k, -1 = none; for HCA every entry) and the stored window, read back
    from the cache.  Checks the attention kernel whatever the selection
    (also when a tie-zone swap makes the GPU's selection differ from the
    oracle's)."""
    from compressed_sparse_long_hca_b200.api import unpack_kv_rows

    def value(packed):
        if cache.fmt == "f32":
            return f32_rows_value(packed, D)
        fp8, bf, sc = unpack_kv_rows(packed, D, R)
        return O.dequantize_kv(O.KVRow(fp8=fp8, rope=bf, scale=sc))

    sel = np.asarray(sel)
    sel = sel[sel >= 0]
    rows = []
    if len(sel):
        rows.append(value(np.concatenate([cache.read_rows(layer, req, 0, int(j), 1) for j in sel])))
    wp = O.window_positions(t)
    rows.append(value(cache.read_rows(layer, req, 2, wp[0], len(wp))))
    rows = np.concatenate(rows, axis=0)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    return O.mqa_attention(O.rope(np.asarray(q, np.float64), t, R), rows, sink, scale)


def check_f32_rows(gpu_rows: np.ndarray, ref_vals: np.ndarray, what="rows") -> None:
    """fp32 storage format: stored rows (packed fp32 bytes) against the
    oracle's fp64 values.  The kernels pool in fp32 (a few ulps; near-zero
    values after cancellation carry a few ulps of the row's magnitudes), so
    |gpu - ref| <= 2^-20 |ref| + 2^-18 rms(row)."""
    g = np.ascontiguousarray(gpu_rows).view(np.float32).astype(np.float64).reshape(np.asarray(ref_vals).shape)
    x = np.asarray(ref_vals, np.float64)
    rms = np.sqrt(np.mean(x ** 2, axis=1, keepdims=True))
    err = np.abs(g - x)
    bad = err > 2.0 ** -20 * np.abs(x) + 2.0 ** -18 * rms + 1e-30
    assert not bad.any(), f"{what}: {int(bad.sum())} values outside the fp32 bound; worst {err.max():.3e}"


def f32_rows_value(gpu_rows: np.ndarray, d: int) -> np.ndarray:
    return np.ascontiguousarray(gpu_rows).view(np.float32).astype(np.float64).reshape(-1, d)

