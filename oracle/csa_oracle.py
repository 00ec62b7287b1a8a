"""Plain fp64 CPU oracle for the CSA / HCA compressed-attention decode step.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only the tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may call it.  It shares no code, no
table and no constant generator with the CUDA library; both sides only share
the seeded input generators.

Every function restates, in the most direct form numpy allows, one step that
the source pages describe.  The pages are five web articles about the
DeepSeek-V4 technical report; they are cited by title and section:

* [V4-来了]  "V4终于终于终于终于是来了", sections "CSA——压缩稀疏注意力" and
  "HCA——重度压缩注意力" (the most precise data-flow description: compressor,
  lightning indexer, top-k selector, MQA core, 128-token window, sink logit,
  RoPE on the last 64 dims, FP8 + BF16 KV cache, state cache / classic cache).
* [深度解读]  "深度解读DeepSeek V4 看清Benchmark以外的三个范式创新",
  section "01", sub-sections "混合注意力的精细解剖" (HCA 128:1 and CSA 4:1 with
  overlap, indexer picks top 1024) and "「精度补偿」的无限套娃游戏" (head dim 512,
  sliding window of 128 raw tokens).
* [播客摘要]  the podcast summary page, sections "1.1 混合注意力架构（CSA 与
  HCA）" (CSA = compression then sparse attention over k entries; HCA dense)
  and "2.1 推理与计算效率" (FP4 on the indexer path).
* [全解析]  "DeepSeek V4 底层逻辑全解析：从 V3 到 V4，真正升级了什么？",
  section "二、升级点 1：CSA + HCA" (m=4 with overlap, FP4 indexer, top-512 /
  top-1024, MQA over the selected entries).

Where the pages leave a step open the oracle takes the reading written in the
repository's design notes (gating form, overlap geometry, FP4 / FP8 scaling,
RoPE pairing and positions, K = V, visibility, tie-break); each such reading
is named in the docstring of the function that applies it.

Parity status: every function below is pinned by tests in ``tests/`` against
closed forms, library routines (torch dtype casts, scipy softmax, torch
scaled-dot-product attention, numpy complex rotation) or brute force.  No
function is "parity unpinned".

Precision: arithmetic is fp64.  Where a floating-point value decides an
integer (a quantised code) the decision is taken in fp32, the precision the
kernels use: the fp64 value is rounded to fp32 first and the code is chosen
from that fp32 value by the formats' own definitions.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

# ---------------------------------------------------------------------------
# Number formats.
#
# [V4-来了] section "HCA——重度压缩注意力": the KV cache keeps the RoPE dims in
# BF16 and the other dims in FP8.  [播客摘要] section "2.1 推理与计算效率":
# the indexer path is FP4.  The bit layouts follow the public OCP 8-bit
# floating point specification (E4M3: bias 7, no infinities, max 448) and the
# OCP microscaling (MX) specification (E2M1 elements, E8M0 shared scale).
# ---------------------------------------------------------------------------

E4M3_MAX = 448.0
E2M1_MAX = 6.0


def f32(x):
    """Round fp64 values to the nearest fp32 value (ties to even)."""
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def bf16_bits_from_f32(x32) -> np.ndarray:
    """BF16 bit pattern of fp32 values, round to nearest, ties to even."""
    u = np.asarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_value(bits) -> np.ndarray:
    """fp64 value of BF16 bit patterns (exact)."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def e4m3_value(codes) -> np.ndarray:
    """fp64 value of FP8 E4M3 codes (sign, 4-bit exponent bias 7, 3-bit mantissa).

    Exponent field 0 is subnormal: m/8 * 2^-6.  Code S.1111.111 is NaN."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return s * mag


def e4m3_code(y) -> np.ndarray:
    """E4M3 code of real values: round to nearest, ties to even, saturate at 448."""
    y = np.asarray(y, dtype=np.float64)
    sign = np.signbit(y).astype(np.int64) << 7
    a = np.abs(y)
    out = np.zeros(a.shape, dtype=np.int64)
    sub = a < 2.0 ** -6
    # subnormal range: integer multiples of 2^-9 (a count of 8 is the smallest normal)
    out = np.where(sub, np.rint(a / 2.0 ** -9).astype(np.int64), out)
    with np.errstate(divide="ignore"):
        _, ex = np.frexp(np.where(sub, 1.0, a))
    E = ex - 1                                          # a = 2^E * (1 + f)
    q = np.rint((np.where(sub, 1.0, a) / np.exp2(E) - 1.0) * 8.0).astype(np.int64)
    E = np.where(q == 8, E + 1, E)
    q = np.where(q == 8, 0, q)
    normal_code = ((E + 7) << 3) | q
    normal_code = np.minimum(normal_code, 0x7E)         # 0x7E = 448; 0x7F is NaN
    out = np.where(sub, out, normal_code)
    return (out | sign).astype(np.uint8)


_E2M1_MAGS = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e2m1_value(codes) -> np.ndarray:
    """fp64 value of 4-bit E2M1 codes (sign, 2-bit exponent bias 1, 1-bit mantissa)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    e = (c >> 1) & 0x3
    m = c & 0x1
    mag = np.where(e == 0, m * 0.5, (1.0 + m / 2.0) * np.exp2(e - 1.0))
    return np.where(c & 0x8, -mag, mag)


def e2m1_code(y) -> np.ndarray:
    """E2M1 code of real values: round to nearest, ties to even, saturate at 6."""
    y = np.asarray(y, dtype=np.float64)
    sign = np.signbit(y).astype(np.int64) << 3
    a = np.abs(y)
    sub = a < 1.0
    out_sub = np.rint(a / 0.5).astype(np.int64)          # 0, 1 or 2 (2 == 1.0)
    _, ex = np.frexp(np.where(sub, 1.0, a))
    E = ex - 1
    q = np.rint((np.where(sub, 1.0, a) / np.exp2(E) - 1.0) * 2.0).astype(np.int64)
    E = np.where(q == 2, E + 1, E)
    q = np.where(q == 2, 0, q)
    out_norm = np.minimum(((E + 1) << 1) | q, 0x7)       # 0x7 = 6.0
    out = np.where(sub, out_sub, out_norm)
    return (out | sign).astype(np.uint8)


def ue8m0_value(codes) -> np.ndarray:
    """fp64 value of unsigned E8M0 scale codes: 2^(code - 127)."""
    return np.exp2(np.asarray(codes, dtype=np.float64) - 127.0)


# ---------------------------------------------------------------------------
# Row quantisers.
# ---------------------------------------------------------------------------

@dataclass
class KVRow:
    """One stored KV vector: FP8 E4M3 codes for the non-RoPE dims, BF16 bits for
    the RoPE dims, and one fp32 scale for the FP8 part."""
    fp8: np.ndarray      # uint8 [.., D - R]
    rope: np.ndarray     # uint16 [.., R]  (BF16 bit patterns)
    scale: np.ndarray    # float32 [..]


def quantize_kv(x, R: int) -> KVRow:
    """Store a KV vector as [V4-来了] section "HCA——重度压缩注意力" describes:
    BF16 for the last R (RoPE) dims and FP8 for the rest.

    Reading (the pages fix no FP8 scale): one fp32 scale per row,
    s = amax / 448 over the FP8 dims (s = 1 when amax = 0); code =
    E4M3(x / s).  Both divisions are fp32 divisions of the fp32-rounded value."""
    x32 = f32(x)
    nope = x32[..., :-R]
    amax = np.max(np.abs(nope), axis=-1).astype(np.float32)
    s = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    y = (nope / s[..., None]).astype(np.float32)
    return KVRow(fp8=e4m3_code(y), rope=bf16_bits_from_f32(x32[..., -R:]), scale=s)


def dequantize_kv(row: KVRow) -> np.ndarray:
    """fp64 vector that a stored KV row stands for (K = V = this vector)."""
    nope = e4m3_value(row.fp8) * row.scale.astype(np.float64)[..., None]
    return np.concatenate([nope, bf16_value(row.rope)], axis=-1)


@dataclass
class MXFP4:
    """MXFP4 vector: E2M1 element codes and one E8M0 scale per 32 elements."""
    codes: np.ndarray    # uint8 [.., d]  (one 4-bit code per byte, unpacked)
    scales: np.ndarray   # uint8 [.., d / 32]


def quantize_mxfp4(x) -> MXFP4:
    """MXFP4 quantiser for the indexer path ([播客摘要] section "2.1 推理与计算效率";
    [全解析] section "二、升级点 1": the indexer scores in FP4).

    Reading: OCP MX block of 32 elements; shared exponent
    e = floor(log2(amax)) - 2 (2 is the largest E2M1 exponent), clamped to
    [-127, 127]; element code = E2M1(x / 2^e) with saturation at 6; an all-zero
    block takes e = 0.  The decision is taken on the fp32-rounded value."""
    x32 = f32(x).astype(np.float64)
    d = x32.shape[-1]
    assert d % 32 == 0
    blocks = x32.reshape(x32.shape[:-1] + (d // 32, 32))
    amax = np.max(np.abs(blocks), axis=-1)
    _, ex = np.frexp(np.where(amax > 0, amax, 1.0))
    e = np.where(amax > 0, ex - 1 - 2, 0)
    e = np.clip(e, -127, 127)
    y = blocks / np.exp2(e)[..., None]
    codes = e2m1_code(y).reshape(x32.shape)
    return MXFP4(codes=codes, scales=(e + 127).astype(np.uint8))


def dequantize_mxfp4(v: MXFP4) -> np.ndarray:
    d = v.codes.shape[-1]
    vals = e2m1_value(v.codes).reshape(v.codes.shape[:-1] + (d // 32, 32))
    return (vals * ue8m0_value(v.scales)[..., None]).reshape(v.codes.shape)


# ---------------------------------------------------------------------------
# Partial RoPE.  [V4-来了] section "HCA——重度压缩注意力": queries and KV get RoPE
# on their last 64 dims only; the other dims carry no position.
# Reading: rotation pairs (2i, 2i+1) inside the last R dims, frequency
# base^(-2i/R) with base 10000.
# ---------------------------------------------------------------------------

def rope(x, pos, R: int, base: float = 10000.0) -> np.ndarray:
    """Rotate the last R dims of x (fp64) by position pos (scalar or per row)."""
    x = np.array(x, dtype=np.float64, copy=True)
    D = x.shape[-1]
    pos = np.asarray(pos, dtype=np.float64)
    for i in range(R // 2):
        theta = base ** (-2.0 * i / R)
        ang = pos * theta
        c, s = np.cos(ang), np.sin(ang)
        a = x[..., D - R + 2 * i].copy()
        b = x[..., D - R + 2 * i + 1].copy()
        x[..., D - R + 2 * i] = a * c - b * s
        x[..., D - R + 2 * i + 1] = a * s + b * c
    return x


# ---------------------------------------------------------------------------
# Token-level compressor.  [V4-来了] section "CSA——压缩稀疏注意力": every 4
# tokens' KV become one entry; [深度解读] "混合注意力的精细解剖": CSA uses
# overlapping windows so meaning is not cut at block edges, HCA folds 128
# consecutive tokens into one entry; [深度解读] "再行界说「压缩」" describes the
# entry as an importance-weighted sum of the tokens' feature vectors.
#
# Readings: per-channel softmax gating over the window's tokens,
# g = softmax_tau(z_tau + b_pos[slot]); CSA entry j covers tokens
# [4j - 4, 4j + 4) (the previous block and its own), tokens before 0 are left
# out of the softmax; HCA entry j covers [128j, 128j + 128); RoPE is applied
# after pooling, at the position of the entry's own first token (4j or 128j).
# ---------------------------------------------------------------------------

def pool(cands, gates, bias) -> np.ndarray:
    """Importance-weighted sum over the token axis (axis -2), per channel:
    sum_tau softmax_tau(gates + bias)[tau] * cands[tau]."""
    logits = np.asarray(gates, np.float64) + np.asarray(bias, np.float64)
    mx = np.max(logits, axis=-2, keepdims=True)
    w = np.exp(logits - mx)
    w = w / np.sum(w, axis=-2, keepdims=True)
    return np.sum(w * np.asarray(cands, np.float64), axis=-2)


def csa_window(j: int, m: int = 4):
    """Token positions and bias slots of CSA entry j (overlapping 2m window)."""
    first = m * j - m
    taus = [t for t in range(first, m * j + m) if t >= 0]
    slots = [t - first for t in taus]
    return taus, slots


def hca_window(j: int, m: int = 128):
    taus = list(range(m * j, m * j + m))
    return taus, [t - m * j for t in taus]


def n_csa_entries(T: int, m: int = 4) -> int:
    """Completed CSA entries after T tokens ([深度解读] "混合注意力的精细解剖":
    1M tokens leave about 250K blocks)."""
    return T // m


def n_hca_entries(T: int, m: int = 128) -> int:
    """Completed HCA entries after T tokens (1M tokens leave under 8000)."""
    return T // m


def csa_entry_vectors(c, z, ci, zi, b_kv, b_idx, j: int, D: int, R: int,
                      m: int = 4, base: float = 10000.0, offset: int = 0):
    """Pooled fp64 KV vector (after RoPE at 4j) and pooled index-key vector of
    CSA entry j.  c, z: [T, D]; ci, zi: [T, d_I]; b_kv: [2m, D]; b_idx: [2m, d_I].
    Row x of c, z, ci, zi holds token position offset + x."""
    taus, slots = csa_window(j, m)
    rows = [t - offset for t in taus]
    kv = pool(c[rows], z[rows], b_kv[slots])
    kv = rope(kv, m * j, R, base)
    key = pool(ci[rows], zi[rows], b_idx[slots])
    return kv, key


def hca_entry_vector(c, z, b_kv, j: int, D: int, R: int, m: int = 128,
                     base: float = 10000.0, offset: int = 0):
    """Pooled fp64 KV vector of HCA entry j (after RoPE at 128j); row x of c, z
    holds token position offset + x."""
    taus, slots = hca_window(j, m)
    rows = [t - offset for t in taus]
    kv = pool(c[rows], z[rows], b_kv[slots])
    return rope(kv, m * j, R, base)


def csa_entries_all(c, z, ci, zi, b_kv, b_idx, R: int, m: int = 4,
                    base: float = 10000.0):
    """All completed CSA entries of a context, vectorised over j (same
    arithmetic as csa_entry_vectors, one entry per row)."""
    T, D = c.shape
    N = T // m
    kv = np.empty((N, D))
    key = np.empty((N, ci.shape[1]))
    if N == 0:
        return kv, key
    cb = c[: N * m].reshape(N, m, D)
    zb = z[: N * m].reshape(N, m, D)
    cib = ci[: N * m].reshape(N, m, -1)
    zib = zi[: N * m].reshape(N, m, -1)
    # entry 0 has no previous block: softmax over its own m tokens only
    kv[0] = pool(cb[0], zb[0], b_kv[m:])
    key[0] = pool(cib[0], zib[0], b_idx[m:])
    if N > 1:
        kv[1:] = pool(np.concatenate([cb[:-1], cb[1:]], axis=1),
                      np.concatenate([zb[:-1], zb[1:]], axis=1), b_kv[None])
        key[1:] = pool(np.concatenate([cib[:-1], cib[1:]], axis=1),
                       np.concatenate([zib[:-1], zib[1:]], axis=1), b_idx[None])
    kv = rope(kv, m * np.arange(N), R, base)
    return kv, key


def hca_entries_all(c, z, b_kv, R: int, m: int = 128, base: float = 10000.0):
    T, D = c.shape
    N = T // m
    if N == 0:
        return np.empty((0, D))
    kv = pool(c[: N * m].reshape(N, m, D), z[: N * m].reshape(N, m, D), b_kv[None])
    return rope(kv, m * np.arange(N), R, base)


def raw_token_row(c_tau, tau, R: int, base: float = 10000.0) -> np.ndarray:
    """Uncompressed KV of token tau for the sliding window: RoPE at tau
    ([V4-来了]: both CSA and HCA keep the latest 128 tokens' raw KV)."""
    return rope(c_tau, tau, R, base)


# ---------------------------------------------------------------------------
# Projections around the path.  [V4-来了] section "CSA——压缩稀疏注意力": the
# token's hidden state is projected to the compressor's inputs, and the query
# side down to a latent of width d_c (1024 in the Flash-like configuration)
# and up to the (index) query heads.  [深度解读] section 01, "「精度补偿」的无限
# 套娃游戏": the 128 heads x 512 attention output is projected in 16 groups
# first, then to the model width.  A projection is a plain matrix product;
# the grouped one is the same product with a block-diagonal weight.
# ---------------------------------------------------------------------------

def linear(x, W) -> np.ndarray:
    """y = x W^T in fp64: x [n, K], W [n_out, K]."""
    return np.asarray(x, np.float64) @ np.asarray(W, np.float64).T


def grouped_linear(x, W, groups: int) -> np.ndarray:
    """Block-diagonal projection: W [n_out, K / groups]; the rows of group g
    (n_out / groups of them) see the columns [g K / groups, (g + 1) K / groups)
    of x.  y[:, rows of g] = x[:, columns of g] W[rows of g]^T."""
    x = np.asarray(x, np.float64)
    W = np.asarray(W, np.float64)
    n_out, kg = W.shape
    rg = n_out // groups
    return np.concatenate([x[:, g * kg:(g + 1) * kg] @ W[g * rg:(g + 1) * rg].T for g in range(groups)], axis=1)


# ---------------------------------------------------------------------------
# Lightning indexer.  [V4-来了] section "CSA——压缩稀疏注意力": the query's hidden
# state is projected down and up to multi-head index queries, passed through
# ReLU and scored against the compressed index keys.  Reading: the score is
# the head-weighted sum of ReLU(q_h . k_j) (per-query head weights w_h, any
# sign, no scale, no RoPE), with q and k both MXFP4.
# ---------------------------------------------------------------------------

def index_scores(q_idx, w, keys) -> np.ndarray:
    """s_j = sum_h w_h * max(0, q_h . k_j).  q_idx: [H_I, d_I] dequantised;
    w: [H_I]; keys: [N, d_I] dequantised.  Returns fp64 [N]."""
    dots = np.asarray(keys, np.float64) @ np.asarray(q_idx, np.float64).T   # [N, H_I]
    return np.maximum(dots, 0.0) @ np.asarray(w, np.float64)


# ---------------------------------------------------------------------------
# Top-k selector.  [V4-来了] section "CSA——压缩稀疏注意力": keep the 512 (Flash)
# or 1024 (Pro) most relevant compressed entries.  Readings: equal scores go
# to the lower index; output ascending; k > N pads with -1.
# ---------------------------------------------------------------------------

def topk(scores, k: int) -> np.ndarray:
    s = np.asarray(scores, dtype=np.float64)
    n = s.shape[0]
    order = np.lexsort((np.arange(n), -s))       # primary: score desc; then index asc
    sel = np.sort(order[: min(k, n)])
    out = np.full(k, -1, dtype=np.int64)
    out[: sel.shape[0]] = sel
    return out


# ---------------------------------------------------------------------------
# Core MQA with sliding window and sink.  [V4-来了]: the selected compressed
# entries and the window's 128 raw tokens are fed together to multi-query
# attention; each head has a learnable sink logit added to the softmax
# denominator.  Readings: K = V = the stored vector; scale 1/sqrt(D); the max
# is taken over the logits and the sink; q gets RoPE at the query position.
# ---------------------------------------------------------------------------

def mqa_attention(q, rows, sink, scale: float) -> np.ndarray:
    """o_h = sum_r e^{u_hr - mu} V_r / (sum_r e^{u_hr - mu} + e^{sink_h - mu}),
    u = scale * q K^T, mu = max(max_r u_hr, sink_h).  q: [H, D] (already
    rotated), rows: [n, D], sink: [H]."""
    q = np.asarray(q, np.float64)
    rows = np.asarray(rows, np.float64)
    sink = np.asarray(sink, np.float64)
    u = scale * (q @ rows.T)                                   # [H, n]
    mu = np.maximum(np.max(u, axis=1) if rows.shape[0] else -np.inf, sink)
    e = np.exp(u - mu[:, None])
    den = np.sum(e, axis=1) + np.exp(sink - mu)
    return (e @ rows) / den[:, None]


def window_positions(t: int, W: int = 128):
    """Raw tokens visible to the query at position t: max(0, t - W + 1) .. t."""
    return list(range(max(0, t - W + 1), t + 1))


# ---------------------------------------------------------------------------
# One layer's cache, held the way the pages split it ([V4-来了] section
# "HCA——重度压缩注意力"): compressed entries (classic cache) and the raw
# window plus unfinished tails (state cache).  The oracle keeps the raw token
# inputs of the whole context, which is simpler to check by eye than a ring.
# ---------------------------------------------------------------------------

@dataclass
class LayerParams:
    kind: str                 # "csa" or "hca"
    D: int
    R: int
    b_kv: np.ndarray          # [2m, D] (CSA) or [128, D] (HCA)
    b_idx: np.ndarray | None  # [2m, d_I] (CSA)
    m: int = 4
    W: int = 128
    base: float = 10000.0
    fmt: str = "mixed"        # "mixed": FP8 + BF16 rows, MXFP4 keys; "f32": fp32 storage


@dataclass
class RequestState:
    c: list = field(default_factory=list)
    z: list = field(default_factory=list)
    ci: list = field(default_factory=list)
    zi: list = field(default_factory=list)

    @property
    def T(self) -> int:
        return len(self.c)


def append_tokens(st: RequestState, c, z, ci=None, zi=None) -> None:
    for i in range(np.asarray(c).shape[0]):
        st.c.append(np.asarray(c[i], np.float64))
        st.z.append(np.asarray(z[i], np.float64))
        if ci is not None:
            st.ci.append(np.asarray(ci[i], np.float64))
            st.zi.append(np.asarray(zi[i], np.float64))


def store_f32(x) -> np.ndarray:
    """fp32 storage format (the tiny configuration is described as fp32):
    a stored vector is its value rounded to fp32, with no other quantiser."""
    return f32(x).astype(np.float64)


def stored_entries(p: LayerParams, st: RequestState):
    """Stored compressed entries of the context: KV rows and (CSA) index keys,
    quantised (mixed format) or rounded to fp32 (fp32 format)."""
    c = np.array(st.c)
    z = np.array(st.z)
    if p.kind == "csa":
        kv, key = csa_entries_all(c, z, np.array(st.ci), np.array(st.zi),
                                  p.b_kv, p.b_idx, p.R, p.m, p.base)
        if p.fmt == "f32":
            return store_f32(kv), store_f32(key)
        return quantize_kv(kv, p.R), quantize_mxfp4(key)
    kv = hca_entries_all(c, z, p.b_kv, p.R, p.m, p.base)
    if p.fmt == "f32":
        return store_f32(kv), None
    return quantize_kv(kv, p.R), None


def stored_window(p: LayerParams, st: RequestState, t: int):
    pos = window_positions(t, p.W)
    rows = np.stack([raw_token_row(st.c[tau], tau, p.R, p.base) for tau in pos])
    return store_f32(rows) if p.fmt == "f32" else quantize_kv(rows, p.R)


def bf16_round(x) -> np.ndarray:
    """Value of x after rounding to fp32 and then to BF16."""
    return bf16_value(bf16_bits_from_f32(f32(x)))


def decode_query(p: LayerParams, st: RequestState | None, q, sink, k: int | None = None,
                 q_idx=None, w=None, scale: float | None = None,
                 entries=None, window=None, T: int | None = None):
    """Full decode step for the query at position t = T - 1 (the token just
    appended): index scores, top-k and attention for CSA; dense attention
    over all entries for HCA.  q: [H, D] before RoPE (BF16 values in the
    mixed format, fp32 values in the fp32 format, where the index query is
    used as given instead of through MXFP4).
    `entries` / `window` may hand in stored rows directly (then `st` may be
    None and T gives the context length).  Returns a dict with the
    intermediate results."""
    t = (st.T if T is None else T) - 1
    if scale is None:
        scale = 1.0 / math.sqrt(p.D)
    if entries is None:
        entries = stored_entries(p, st)
    kvq, keyq = entries
    win = window if window is not None else stored_window(p, st, t)
    f32_fmt = p.fmt == "f32"
    value = (lambda rows: np.asarray(rows, np.float64)) if f32_fmt else dequantize_kv
    out = {}
    if p.kind == "csa":
        if f32_fmt:
            s = index_scores(store_f32(q_idx), w, keyq)
        else:
            qi = dequantize_mxfp4(quantize_mxfp4(q_idx))
            s = index_scores(qi, w, dequantize_mxfp4(keyq))
        out["scores"] = s
        # the kernels select on fp32 scores; the oracle selects on its fp64
        # scores (comparison tolerance covers the difference)
        sel = topk(s, k)
        out["topk"] = sel
        j = sel[sel >= 0]
        rows = kvq[j] if f32_fmt else dequantize_kv(KVRow(fp8=kvq.fp8[j], rope=kvq.rope[j], scale=kvq.scale[j]))
    else:
        rows = value(kvq)
    rows = np.concatenate([rows, value(win)], axis=0)
    qr = rope(np.asarray(q, np.float64), t, p.R, p.base)
    out["out"] = mqa_attention(qr, rows, sink, scale)
    out["n_rows"] = rows.shape[0]
    return out


def chunk_queries(p: LayerParams, st: RequestState, c, z, ci=None, zi=None, q=None, sink=None,
                  k: int | None = None, q_idx=None, w=None, scale: float | None = None):
    """A chunk of n new tokens that are also queries (prefill).  The pages
    describe the decode step ([V4-来了] section "CSA——压缩稀疏注意力": the
    data flow for the latest token); the reading taken for a chunk is causal
    visibility: the query at position t sees what a decode query at t sees,
    i.e. the tokens 0 .. t and nothing after.  Written as that definition:
    append the chunk's tokens one at a time and run the decode step after
    each.  c, z: [n, D]; ci, zi: [n, d_I]; q: [n, H, D]; q_idx: [n, H_I, d_I];
    w: [n, H_I].  Returns one decode_query result per token, in order."""
    res = []
    for j in range(np.asarray(c).shape[0]):
        append_tokens(st, c[j:j + 1], z[j:j + 1], None if ci is None else ci[j:j + 1],
                      None if zi is None else zi[j:j + 1])
        res.append(decode_query(p, st, q[j], sink, k=k, q_idx=None if q_idx is None else q_idx[j],
                                w=None if w is None else w[j], scale=scale))
    return res
