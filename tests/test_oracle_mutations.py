"""The oracle's pins catch plausible mistakes.  Each case plants one mistake
in the oracle on the CPU (a rotation the wrong way, a dropped bias, a
window one token off, a missing ReLU or sink, ties to the wrong index, a
wrong format constant, a transposed group), by replacing one oracle
function for the duration of the case, and checks that a named pin of
test_oracle_math / test_oracle_formats then fails with an assertion.  The
oracle's own functions call each other through the module, so a planted
mistake reaches every path that uses the function."""
import numpy as np
import pytest

from oracle import csa_oracle as O
from tests import test_oracle_formats as TF
from tests import test_oracle_math as TM

_ORIG = {name: getattr(O, name) for name in (
    "rope", "pool", "csa_window", "csa_entries_all", "stored_window", "index_scores", "topk", "mqa_attention", "window_positions",
    "e4m3_value", "bf16_bits_from_f32", "quantize_mxfp4", "e2m1_code", "grouped_linear", "linear",
    "quantize_kv", "n_csa_entries", "n_hca_entries")}


# ---------------------------------------------------------------- the mistakes

def rope_wrong_direction(x, pos, R, base=10000.0):
    return _ORIG["rope"](x, -np.asarray(pos, np.float64), R, base)


def rope_first_dims(x, pos, R, base=10000.0):
    """Rotates the first R dims instead of the last R."""
    x = np.asarray(x, np.float64)
    moved = np.concatenate([x[..., R:], x[..., :R]], axis=-1)
    y = _ORIG["rope"](moved, pos, R, base)
    return np.concatenate([y[..., -R:], y[..., :-R]], axis=-1)


def rope_half_frequency(x, pos, R, base=10000.0):
    """theta_i = base^(-i/R) instead of base^(-2i/R)."""
    return _ORIG["rope"](x, pos, R, base ** 0.5)


def pool_without_bias(cands, gates, bias):
    return _ORIG["pool"](cands, gates, np.zeros_like(np.asarray(bias, np.float64)))


def pool_softmax_over_channels(cands, gates, bias):
    logits = np.asarray(gates, np.float64) + np.asarray(bias, np.float64)
    w = np.exp(logits - logits.max(axis=-1, keepdims=True))
    w = w / w.sum(axis=-1, keepdims=True)
    return np.sum(w * np.asarray(cands, np.float64), axis=-2)


def csa_window_shifted(j, m=4):
    """Window [m j - m - 1, m j + m - 1): one token early (each token paired
    with its neighbour's bias slot)."""
    taus, slots = _ORIG["csa_window"](j, m)
    pairs = [(t - 1, s) for t, s in zip(taus, slots) if t - 1 >= 0]
    return [t for t, _ in pairs], [s for _, s in pairs]


def csa_window_not_overlapping(j, m=4):
    """Only the entry's own block [m j, m j + m)."""
    taus = list(range(m * j, m * j + m))
    return taus, [t - (m * j - m) for t in taus]


def csa_entries_own_block_only(c, z, ci, zi, b_kv, b_idx, R, m=4, base=10000.0):
    """Every entry pooled over its own m tokens (the previous block left out)."""
    T, D = c.shape
    N = T // m
    kv = O.pool(c[: N * m].reshape(N, m, D), z[: N * m].reshape(N, m, D), b_kv[None, m:])
    key = O.pool(ci[: N * m].reshape(N, m, -1), zi[: N * m].reshape(N, m, -1), b_idx[None, m:])
    return O.rope(kv, m * np.arange(N), R, base), key


def stored_window_last_row_only(p, st, t):
    w = _ORIG["stored_window"](p, st, t)
    if isinstance(w, O.KVRow):
        return O.KVRow(fp8=w.fp8[-1:], rope=w.rope[-1:], scale=w.scale[-1:])
    return w[-1:]                                # fp32 format: plain rows


def index_scores_without_relu(q_idx, w, keys):
    dots = np.asarray(keys, np.float64) @ np.asarray(q_idx, np.float64).T
    return dots @ np.asarray(w, np.float64)


def index_scores_weight_inside_relu(q_idx, w, keys):
    dots = np.asarray(keys, np.float64) @ np.asarray(q_idx, np.float64).T
    return np.maximum(dots * np.asarray(w, np.float64)[None, :], 0.0).sum(axis=1)


def topk_ties_to_higher_index(scores, k):
    s = np.asarray(scores, np.float64)
    n = s.shape[0]
    order = np.lexsort((-np.arange(n), -s))
    sel = np.sort(order[: min(k, n)])
    out = np.full(k, -1, dtype=np.int64)
    out[: sel.shape[0]] = sel
    return out


def topk_in_score_order(scores, k):
    s = np.asarray(scores, np.float64)
    n = s.shape[0]
    order = np.lexsort((np.arange(n), -s))[: min(k, n)]
    out = np.full(k, -1, dtype=np.int64)
    out[: order.shape[0]] = order
    return out


def attention_without_sink(q, rows, sink, scale):
    return _ORIG["mqa_attention"](q, rows, np.full(np.shape(sink), -np.inf), scale)


def attention_without_scale(q, rows, sink, scale):
    return _ORIG["mqa_attention"](q, rows, sink, 1.0)


def window_one_too_many(t, W=128):
    return list(range(max(0, t - W), t + 1))


def e4m3_bias_8(codes):
    """Exponent bias 8 instead of 7 (every normal value halved)."""
    v = _ORIG["e4m3_value"](codes)
    e = (np.asarray(codes, dtype=np.uint8).astype(np.int64) >> 3) & 0xF
    return np.where(e > 0, v / 2.0, v)


def bf16_truncated(x32):
    u = np.asarray(x32, dtype=np.float32).view(np.uint32)
    return (u >> np.uint32(16)).astype(np.uint16)


def mxfp4_exponent_off_by_one(x):
    """Shared exponent floor(log2 amax) - 1 instead of - 2."""
    x32 = O.f32(x).astype(np.float64)
    d = x32.shape[-1]
    blocks = x32.reshape(x32.shape[:-1] + (d // 32, 32))
    amax = np.max(np.abs(blocks), axis=-1)
    _, ex = np.frexp(np.where(amax > 0, amax, 1.0))
    e = np.clip(np.where(amax > 0, ex - 1 - 1, 0), -127, 127)
    codes = O.e2m1_code(blocks / np.exp2(e)[..., None]).reshape(x32.shape)
    return O.MXFP4(codes=codes, scales=(e + 127).astype(np.uint8))


def e2m1_ties_away_from_zero(y):
    y = np.asarray(y, dtype=np.float64)
    return _ORIG["e2m1_code"](y + np.sign(y) * 1e-9)


def kv_scale_for_224(x, R):
    """FP8 scale amax / 224 instead of amax / 448 (half the code range used)."""
    x32 = O.f32(x)
    nope = x32[..., :-R]
    amax = np.max(np.abs(nope), axis=-1).astype(np.float32)
    s = np.where(amax > 0, amax / np.float32(224.0), np.float32(1.0)).astype(np.float32)
    y = (nope / s[..., None]).astype(np.float32)
    return O.KVRow(fp8=O.e4m3_code(y), rope=O.bf16_bits_from_f32(x32[..., -R:]), scale=s)


def kv_fp8_truncated(x, R):
    """FP8 codes by truncation toward zero instead of to nearest."""
    row = _ORIG["quantize_kv"](x, R)
    y = (O.f32(x)[..., :-R] / row.scale[..., None]).astype(np.float64)
    v = O.e4m3_value(row.fp8)
    over = np.abs(v) > np.abs(y)                 # rounded away from zero: step one code down
    codes = np.where(over & ((row.fp8 & 0x7F) > 0), row.fp8 - 1, row.fp8).astype(np.uint8)
    return O.KVRow(fp8=codes, rope=row.rope, scale=row.scale)


def kv_rope_truncated(x, R):
    row = _ORIG["quantize_kv"](x, R)
    u = O.f32(x)[..., -R:].view(np.uint32)
    return O.KVRow(fp8=row.fp8, rope=(u >> np.uint32(16)).astype(np.uint16), scale=row.scale)


def csa_count_partial_entry(T, m=4):
    return T // m + 1


def hca_count_ratio_127(T, m=128):
    return T // (m - 1)


def grouped_linear_groups_reversed(x, W, groups):
    """Row group g reads column block groups - 1 - g."""
    x = np.asarray(x, np.float64)
    W = np.asarray(W, np.float64)
    n_out, kg = W.shape
    rg = n_out // groups
    return np.concatenate([x[:, (groups - 1 - g) * kg:(groups - g) * kg] @ W[g * rg:(g + 1) * rg].T
                           for g in range(groups)], axis=1)


def linear_drops_last_column(x, W):
    return np.asarray(x, np.float64)[:, :-1] @ np.asarray(W, np.float64)[:, :-1].T


# ---------------------------------------------------------------- the cases

# (oracle function, planted mistake, pin that must fail, the pin's arguments)
CASES = [
    ("rope", rope_wrong_direction, TM.test_rope_matches_complex_rotation, ()),
    ("rope", rope_first_dims, TM.test_rope_matches_complex_rotation, ()),
    ("rope", rope_half_frequency, TM.test_rope_matches_complex_rotation, ()),
    ("rope", rope_wrong_direction, TM.test_compressor_brute_force_csa_and_hca, ()),
    ("pool", pool_without_bias, TM.test_scalar_gate_is_scipy_softmax, ()),
    ("pool", pool_without_bias, TM.test_compressor_brute_force_csa_and_hca, ()),
    ("pool", pool_softmax_over_channels, TM.test_uniform_gate_gives_mean, ()),
    ("csa_window", csa_window_shifted, TM.test_compressor_brute_force_csa_and_hca, ()),
    ("csa_window", csa_window_not_overlapping, TM.test_compressor_brute_force_csa_and_hca, ()),
    ("csa_entries_all", csa_entries_own_block_only, TM.test_uniform_gate_gives_mean, ()),
    ("csa_entries_all", csa_entries_own_block_only, TM.test_decode_brute_force_tiny, ("mixed",)),
    ("stored_window", stored_window_last_row_only, TM.test_hca_decode_brute_force_tiny, (300, "mixed")),
    ("stored_window", stored_window_last_row_only, TM.test_decode_brute_force_tiny, ("f32",)),
    ("index_scores", index_scores_without_relu, TM.test_index_single_head_is_relu_dot, ()),
    ("index_scores", index_scores_weight_inside_relu, TM.test_index_scores_brute_force, ()),
    ("index_scores", index_scores_without_relu, TM.test_decode_brute_force_tiny, ("mixed",)),
    ("topk", topk_ties_to_higher_index, TM.test_topk_brute_force_with_ties, ()),
    ("topk", topk_in_score_order, TM.test_topk_brute_force_with_ties, ()),
    ("mqa_attention", attention_without_sink, TM.test_attention_sink_is_extra_zero_value_key, ()),
    ("mqa_attention", attention_without_sink, TM.test_hca_decode_brute_force_tiny, (255, "f32")),
    ("mqa_attention", attention_without_scale, TM.test_attention_without_sink_is_sdpa, ()),
    ("window_positions", window_one_too_many, TM.test_window_visibility, ()),
    ("e4m3_value", e4m3_bias_8, TF.test_e4m3_decode_all_codes_matches_torch, ()),
    ("bf16_bits_from_f32", bf16_truncated, TF.test_bf16_matches_torch_cast, ()),
    ("quantize_mxfp4", mxfp4_exponent_off_by_one, TF.test_mxfp4_scale_rule_and_brute_force, ()),
    ("e2m1_code", e2m1_ties_away_from_zero, TF.test_e2m1_ties_to_even_and_saturation, (0.25, 0.0)),
    ("e2m1_code", e2m1_ties_away_from_zero, TF.test_e2m1_ties_to_even_and_saturation, (2.5, 2.0)),
    ("quantize_kv", kv_scale_for_224, TF.test_kv_row_quantiser, ()),
    ("quantize_kv", kv_fp8_truncated, TF.test_kv_row_quantiser, ()),
    ("quantize_kv", kv_rope_truncated, TF.test_kv_row_rope_dims_are_torch_bf16, ()),
    ("n_csa_entries", csa_count_partial_entry, TM.test_entry_counts_match_page_figures, ()),
    ("n_hca_entries", hca_count_ratio_127, TM.test_entry_counts_match_page_figures, ()),
    ("grouped_linear", grouped_linear_groups_reversed, TM.test_grouped_linear_is_block_diagonal_dense, ()),
    ("linear", linear_drops_last_column, TM.test_linear_brute_force_and_one_hot, ()),
]


@pytest.mark.parametrize("name,mutant,pin,args", CASES,
                         ids=[f"{c[1].__name__}->{c[2].__name__}{list(c[3]) if c[3] else ''}" for c in CASES])
def test_planted_mistake_fails_its_pin(monkeypatch, name, mutant, pin, args):
    pin(*args)                                   # the pin passes on the oracle as it is
    monkeypatch.setattr(O, name, mutant)
    with pytest.raises(AssertionError):
        pin(*args)
