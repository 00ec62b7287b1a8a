"""Host-side checks of the C ABI that need no GPU: the library builds and
loads, exports every function include/csa.h declares, and validates
configurations on the host."""
import ctypes
import os
import re

import pytest

from compressed_sparse_long_hca_b200 import _lib

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "csa.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^[A-Za-z_][\w\s\*]*?\b(csa_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_path():
    names = declared_functions()
    for f in ("csa_compress_append", "csa_index_scores", "csa_topk", "csa_hca_decode_attn",
              "csa_cache_required_bytes", "csa_cache_init"):
        assert f in names


def test_library_exports_every_declared_symbol(cuda_lib):
    for name in declared_functions():
        assert hasattr(cuda_lib, name), name
        assert name in _lib.SIGNATURES, f"{name} has no Python binding"


def _cfg(**kw):
    base = dict(n_csa_layers=1, n_hca_layers=1, H=128, D=512, D_rope=64, H_I=64, d_I=128, window=128,
                max_requests=4, max_pages_per_request=2048, pool_pages=4 * 2048, rope_base=10000.0)
    base.update(kw)
    return _lib.CsaCfg(**base)


def test_required_bytes_and_validation(cuda_lib):
    c = _cfg()
    nbytes = cuda_lib.csa_cache_required_bytes(ctypes.byref(c))
    # 32768 blocks of (32 CSA rows + 32 index keys + 1 HCA row) at least
    assert nbytes >= 32768 * (32 * 580 + 32 * 68 + 580)
    assert nbytes < 32768 * 24000 + 64 * 2**20
    for bad in (dict(D=500), dict(D_rope=15), dict(window=64), dict(d_I=48), dict(H=0),
                dict(H_I=65), dict(n_csa_layers=0, n_hca_layers=0), dict(pool_pages=0)):
        assert cuda_lib.csa_cache_required_bytes(ctypes.byref(_cfg(**bad))) == 0, bad


def test_init_rejects_bad_arguments_without_launching(cuda_lib):
    c = _cfg()
    h = ctypes.c_void_p()
    # unaligned pointer and too-small arena are refused before any CUDA call
    assert cuda_lib.csa_cache_init(ctypes.byref(c), 0x1001, 1 << 40, None, None, None, ctypes.byref(h)) == -1
    assert cuda_lib.csa_cache_init(ctypes.byref(c), 0x10000, 16, None, None, None, ctypes.byref(h)) == -2
    assert h.value is None
    assert b"256-byte" in cuda_lib.csa_last_error() or True
    # compute calls on a NULL handle fail on the host
    assert cuda_lib.csa_compress_append(None, 0, 1, None, 1, None, None, None, None, None) == -1
    assert cuda_lib.csa_topk(None, 1, None, 1, 1, None, 0, None) == -1


def test_decode_step_packed_input_layout():
    """DecodeStep's packed host buffer: the fields in order (the attention
    query last, copied on its own), each on a 256-byte boundary, sized by
    shape and dtype, none overlapping."""
    import math

    import torch

    from compressed_sparse_long_hca_b200.api import decode_step_fields
    for csa, names in ((True, ["c", "z", "ci", "zi", "q_idx", "w", "q"]), (False, ["c", "z", "q"])):
        fields, total = decode_step_fields(4, 128, 512, 64, 128, csa)
        assert [f[0] for f in fields] == names
        end = 0
        for name, dtype, shape, off, nbytes in fields:
            assert off % 256 == 0 and off >= end, name
            assert nbytes == math.prod(shape) * torch.empty((), dtype=dtype).element_size(), name
            end = off + nbytes
        assert total >= end and total % 256 == 0
    fields, _ = decode_step_fields(4, 128, 512, 64, 128, True)
    f = {x[0]: x for x in fields}
    assert f["q"][4] == 4 * 128 * 512 * 2 and f["q"][1] == torch.bfloat16
    assert f["q_idx"][2] == (4, 64, 128) and f["w"][2] == (4, 64)
    assert f["c"][2] == (4, 1, 512) and f["ci"][2] == (4, 1, 128)


def test_topk_argument_errors_are_returned_before_any_launch(cuda_lib):
    """csa_topk needs no cache: every argument error comes back as
    CSA_ERR_ARG from the host checks (the pointer below is never touched)."""
    P = 0x10000
    cases = [
        ((P, 10, P, -1, 4, P, 0, None), b"n must be"),
        ((P, 10, P, 70000, 4, P, 0, None), b"n must be"),
        ((None, 10, P, 1, 4, P, 0, None), b"NULL"),
        ((P, 10, None, 1, 4, P, 0, None), b"NULL"),
        ((P, 10, P, 1, 4, None, 0, None), b"NULL"),
        ((P, 10, P, 1, 0, P, 0, None), b"k and ld"),
        ((P, 0, P, 1, 4, P, 0, None), b"k and ld"),
        ((P, 10, P, 1, 4, P, 3, None), b"variant"),
    ]
    for args, msg in cases:
        assert cuda_lib.csa_topk(*args) == -1, args
        assert msg in cuda_lib.csa_last_error(), (args, cuda_lib.csa_last_error())
    assert cuda_lib.csa_topk(P, 10, P, 0, 4, P, 0, None) == 0        # an empty batch is a no-op


def test_cache_calls_on_a_null_handle_fail_on_the_host(cuda_lib):
    P = 0x10000
    assert cuda_lib.csa_index_scores(None, 0, 1, P, P, P, P, 8, P, 0, None) == -1
    assert cuda_lib.csa_hca_decode_attn(None, 0, 1, P, P, P, 4, P, 1.0, P, P, 1 << 20, 0, None) == -1
    assert cuda_lib.csa_hca_decode_attn_noalloc(None, 0, 1, P, P, P, 4, P, 1.0, P, None) == -1
    assert cuda_lib.csa_attn_workspace_bytes(None, 0, 1, 4) == 0
    assert cuda_lib.csa_request_alloc(None, 0, 16) == -1
    assert cuda_lib.csa_request_free(None, 0) == -1
    assert cuda_lib.csa_check_device_error(None, None) == -1
    assert cuda_lib.csa_debug_wait_timeout(None, 1000, None) == -1
    assert cuda_lib.csa_decode_step_input_bytes(None, 0, 1) == 0
    assert cuda_lib.csa_decode_step_dev_bytes(None, 0, 1, 16) == 0
    assert cuda_lib.csa_decode_step(None, 0, 1, P, 16, P, 1.0, P, P, P, 1 << 20, None) == -1
    assert cuda_lib.csa_prefill_workspace_bytes(None, 0, 1, 16, 16, 0) == 0
    assert cuda_lib.csa_prefill_chunk(None, 0, 1, P, 16, P, P, P, P, P, P, P, 16, P, 1.0, P, None, P, 1 << 20, 0,
                                      None) == -1


def test_gemm_shapes_and_argument_errors_on_the_host(cuda_lib):
    """The projection GEMM's size function and its argument checks run on the
    host: packed weight bytes are 128-row x 64-column tiles of 16 KB, a bad
    shape gives 0 bytes, and csa_gemm_bf16 returns CSA_ERR_ARG for every bad
    argument before any CUDA call (the pointers below are never touched)."""
    wb = cuda_lib.csa_gemm_weight_bytes
    tile = 128 * 64 * 2
    assert wb(300, 1000, 1) == 3 * 16 * tile                    # ceil(300 / 128) row tiles x ceil(1000 / 64)
    assert wb(16 * 128, 16 * 64, 16) == 16 * 1 * tile           # block diagonal: each row tile reads its group
    for bad in ((0, 64, 1), (256, 0, 1), (256, 64, 0), (256, 63, 1), (300, 64, 2), (256, 96, 3),
                (128 * 70000, 64 * 70000, 70000)):
        assert wb(*bad) == 0, bad
    P = 0x10000
    seg = (_lib.GemmOut * 2)()
    seg[0].rows, seg[0].bf16, seg[0].y = 100, 1, P
    seg[1].rows, seg[1].bf16, seg[1].y = 156, 0, P
    segs = ctypes.cast(seg, ctypes.c_void_p)
    g = cuda_lib.csa_gemm_bf16
    cases = [
        ((P, 256, 63, 1, P, 4, 2, segs, P, 1 << 30, None), b"multiple of 8"),
        ((P, 256, 64, 1, P, 257, 2, segs, P, 1 << 30, None), b"n_tok"),
        ((P, 256, 64, 1, P, 4, 0, segs, P, 1 << 30, None), b"n_seg"),
        ((P, 256, 64, 1, P, 4, 9, segs, P, 1 << 30, None), b"n_seg"),
        ((P, 300, 64, 1, P, 4, 2, segs, P, 1 << 30, None), b"add up"),
        ((None, 256, 64, 1, P, 4, 2, segs, P, 1 << 30, None), b"NULL"),
        ((P, 256, 64, 1, P, 4, 2, segs, P + 16, 1 << 30, None), b"aligned"),
    ]
    for args, msg in cases:
        assert g(*args) == -1, args
        assert msg in cuda_lib.csa_last_error(), (args, cuda_lib.csa_last_error())
    assert g(P, 256, 64, 1, P, 0, 2, segs, P, 1 << 30, None) == 0     # no tokens: nothing to do
    seg[1].y = None
    assert g(P, 256, 64, 1, P, 4, 2, segs, P, 1 << 30, None) == -1    # a segment without an output
