"""Device-side failure path without a GPU fault: a bounded wait that runs out.

One thread block waits, through the bounded-wait routine the tensor-core
kernels use for their mbarriers, on a barrier that nothing arrives on.  The
wait must give up after its limit, the block must record
CSA_ERR_DEVICE_TIMEOUT in the device error word and return, and the context
must stay usable: the error is read once and cleared, and a normal call
afterwards returns correct results."""
import time

import numpy as np
import pytest

from compressed_sparse_long_hca_b200 import _lib
from compressed_sparse_long_hca_b200 import inputs as I
from oracle import csa_oracle as O
from tests import helpers as Hp

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _lib_built(cuda_lib):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return cuda_lib


def test_bounded_wait_gives_up_and_reports_a_timeout():
    wl = I.Workload("wait", "hca", H=8, D=64, R=16, H_I=0, d_I=0, k=0, W=128, context=0, batch=0, seed=31)
    pair = Hp.Pair(wl, 0, 1, max_req=1, capacity=512)
    lib = _lib.load()
    stream = torch.cuda.current_stream().cuda_stream or None
    for limit_us in (1000, 20000):
        t0 = time.perf_counter()
        assert lib.csa_debug_wait_timeout(pair.cache.handle, limit_us, stream) == 0
        st = lib.csa_check_device_error(pair.cache.handle, stream)
        el = time.perf_counter() - t0
        assert st == -4, f"expected CSA_ERR_DEVICE_TIMEOUT, got {st}: {lib.csa_last_error()}"
        assert b"bounded wait" in lib.csa_last_error()
        assert el >= limit_us * 1e-6 * 0.9, "the wait ended before its limit"
        assert el < 5.0, "the wait did not end near its limit"
        # the error word was cleared by the read, and the context still works
        assert lib.csa_check_device_error(pair.cache.handle, stream) == 0
    assert lib.csa_debug_wait_timeout(pair.cache.handle, 0, stream) == -1
    assert lib.csa_debug_wait_timeout(pair.cache.handle, 2_000_000, stream) == -1
    # a normal attention call after the timeouts is correct
    rng = np.random.default_rng(3)
    pair.cache.request_alloc(0, 512)
    T = 300
    pair.cache.set_length(0, 0, T)
    from compressed_sparse_long_hca_b200.api import pack_kv_rows
    ent = O.quantize_kv(rng.standard_normal((T // 128, wl.D)), wl.R)
    pair.cache.write_rows(0, 0, 0, 0, pack_kv_rows(ent.fp8, ent.rope, ent.scale))
    wp = O.window_positions(T - 1)
    win = O.quantize_kv(rng.standard_normal((len(wp), wl.D)), wl.R)
    pair.cache.write_rows(0, 0, 2, wp[0], pack_kv_rows(win.fp8, win.rope, win.scale))
    q = I.bf16_grid(rng.standard_normal((1, wl.H, wl.D)).astype(np.float32))
    sink = pair.params[0]["sink"]
    out = torch.empty((1, wl.H, wl.D), dtype=torch.bfloat16, device="cuda")
    pair.cache.decode_attn(0, torch.zeros(1, dtype=torch.int32, device="cuda"),
                           torch.from_numpy(q).cuda().to(torch.bfloat16), None, torch.from_numpy(sink).cuda(), out)
    pair.cache.check_device_error()
    ref = Hp.attention_over_stored_rows(pair.cache, 0, 0, T - 1, np.arange(T // 128), q[0], sink, wl.D, wl.R)
    Hp.check_attention(out[0].float().cpu().numpy(), ref, "attention after the timeouts")
