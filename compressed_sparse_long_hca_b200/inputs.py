"""Seeded synthetic inputs and workload shapes.

This module holds no arithmetic of the method: it only draws random numbers
and names shapes.  Both the CUDA library's callers (tests, bench) and the
fp64 oracle take their inputs from here.

Distributions: every projected vector that feeds the decode step (KV
candidate c, gate logits z, index-key candidate and gate, query q, index
query q_I, index head weights w), every position bias b_pos and every sink
logit is drawn N(0, 1).  Hidden states N(0, 1) with weights N(0, 1/d) give
projected coordinates of unit variance, so drawing the projections directly
keeps the same distribution at a fraction of the cost.

Two generator families:

* ``host``: numpy PCG64, one stream per (seed, layer, request, chunk of
  4096 tokens); any token range can be regenerated on its own.
* ``device``: torch's CUDA Philox generator with the same keying, used only to
  fill large caches quickly; a test that needs such inputs on the host copies
  the generated tensors back.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

CHUNK = 4096

# field ids of the counter key
F_C, F_Z, F_CI, F_ZI, F_Q, F_QI, F_W = 1, 2, 3, 4, 5, 6, 7
F_BKV, F_BIDX, F_BHCA, F_SINK = 11, 12, 13, 14


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "csa" or "hca"
    H: int               # query heads (one shared KV head)
    D: int               # head dim
    R: int               # RoPE dims (the last R)
    H_I: int             # indexer heads
    d_I: int             # index dim
    k: int               # top-k
    W: int               # sliding window
    context: int         # tokens already in the cache before the decode step
    batch: int
    seed: int
    hidden: int = 0


# The five workloads the method is measured on (see the design notes).
C1 = Workload("tiny-csa", "csa", H=8, D=64, R=16, H_I=4, d_I=32, k=16, W=128,
              context=1024, batch=1, seed=1001, hidden=256)
C2 = Workload("hca-128k", "hca", H=64, D=512, R=64, H_I=0, d_I=0, k=0, W=128,
              context=131072, batch=32, seed=1002, hidden=4096)
C3 = Workload("csa-flash-128k", "csa", H=64, D=512, R=64, H_I=64, d_I=128, k=512,
              W=128, context=131072, batch=32, seed=1003, hidden=4096)
C4 = Workload("csa-pro-1m", "csa", H=128, D=512, R=64, H_I=64, d_I=128, k=1024,
              W=128, context=1048576, batch=4, seed=1004, hidden=7168)
# C5: interleaved CSA (top-1024) and HCA layers with Pro-like shapes, ragged
# batches of 1..256 requests with context ~ log-uniform(4K, 1M).
C5_CSA = Workload("sweep-csa", "csa", H=128, D=512, R=64, H_I=64, d_I=128, k=1024,
                  W=128, context=0, batch=0, seed=1005, hidden=7168)
C5_HCA = Workload("sweep-hca", "hca", H=128, D=512, R=64, H_I=0, d_I=0, k=0,
                  W=128, context=0, batch=0, seed=1005, hidden=7168)
# The sweep's HCA layer at its longest context (1M tokens: 8192 compressed
# entries + the window per query), batch 4: the attention over every entry is
# the one contraction-heavy case of the path (about 430 flops per byte).
C5_HCA_1M = Workload("hca-pro-1m", "hca", H=128, D=512, R=64, H_I=0, d_I=0, k=0, W=128,
                     context=1048576, batch=4, seed=1006, hidden=7168)
WORKLOADS = {w.name: w for w in (C1, C2, C3, C4, C5_HCA_1M)}


def _rng(*key) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(key))))


def normal(shape, *key, dtype=np.float32) -> np.ndarray:
    """N(0,1) array for one counter key."""
    return _rng(*key).standard_normal(shape).astype(dtype)


def token_inputs(seed: int, layer: int, req: int, start: int, count: int,
                 D: int, d_I: int):
    """c, z [count, D] and ci, zi [count, d_I] (fp32) for tokens
    start .. start+count-1 of one request of one layer."""
    out = {f: [] for f in ("c", "z", "ci", "zi")}
    t = start
    end = start + count
    while t < end:
        ch = t // CHUNK
        lo = t - ch * CHUNK
        hi = min(CHUNK, end - ch * CHUNK)
        out["c"].append(normal((CHUNK, D), seed, layer, req, ch, F_C)[lo:hi])
        out["z"].append(normal((CHUNK, D), seed, layer, req, ch, F_Z)[lo:hi])
        if d_I:
            out["ci"].append(normal((CHUNK, d_I), seed, layer, req, ch, F_CI)[lo:hi])
            out["zi"].append(normal((CHUNK, d_I), seed, layer, req, ch, F_ZI)[lo:hi])
        t = ch * CHUNK + hi
    cat = lambda xs, d: np.concatenate(xs) if xs else np.zeros((0, d), np.float32)
    return cat(out["c"], D), cat(out["z"], D), cat(out["ci"], d_I), cat(out["zi"], d_I)


def layer_params(seed: int, layer: int, kind: str, D: int, d_I: int, H: int, m: int = 4):
    """Position biases and sink logits of one layer."""
    if kind == "csa":
        b_kv = normal((2 * m, D), seed, layer, F_BKV)
        b_idx = normal((2 * m, d_I), seed, layer, F_BIDX)
    else:
        b_kv = normal((128, D), seed, layer, F_BHCA)
        b_idx = None
    sink = normal((H,), seed, layer, F_SINK)
    return b_kv, b_idx, sink


def bf16_grid(x: np.ndarray) -> np.ndarray:
    """Snap fp32 values to BF16-representable values (ties to even), so that the
    same numbers can be handed to a BF16 kernel argument and to the oracle.
    This is input preparation, not a step of the method."""
    u = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    u = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return u.astype(np.uint32).view(np.float32)


def query_inputs(seed: int, layer: int, step: int, n: int, H: int, D: int,
                 H_I: int, d_I: int):
    """Per-query inputs of one decode step: q [n, H, D] (BF16-representable
    fp32), q_I [n, H_I, d_I], w [n, H_I]."""
    q = bf16_grid(normal((n, H, D), seed, layer, step, F_Q))
    qi = normal((n, H_I, d_I), seed, layer, step, F_QI) if H_I else None
    w = normal((n, H_I), seed, layer, step, F_W) if H_I else None
    return q, qi, w


def sweep_contexts(seed: int, n: int, lo: int = 4096, hi: int = 1 << 20) -> np.ndarray:
    """Per-request contexts ~ log-uniform(lo, hi) for the ragged sweep."""
    u = _rng(seed, 0xC5).random(n)
    return np.floor(np.exp(np.log(lo) + u * (np.log(hi) - np.log(lo)))).astype(np.int64)


def device_token_inputs(seed: int, layer: int, req: int, chunk: int, D: int, d_I: int,
                        device="cuda"):
    """Device-side N(0,1) inputs for one 4096-token chunk (torch Philox), for
    filling long contexts quickly.  Returns c, z, ci, zi as fp32 tensors."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed((((seed * 1_000_003 + layer) * 1_000_033 + req) * 1_000_037 + chunk) % (2**62))
    c = torch.randn((CHUNK, D), generator=g, device=device)
    z = torch.randn((CHUNK, D), generator=g, device=device)
    if d_I:
        ci = torch.randn((CHUNK, d_I), generator=g, device=device)
        zi = torch.randn((CHUNK, d_I), generator=g, device=device)
    else:
        ci = zi = None
    return c, z, ci, zi
