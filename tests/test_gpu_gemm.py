"""GPU parity of the batch-invariant projection GEMM (csa_gemm_bf16) against
the oracle's projections, through the C ABI: dense weights with and without
a fixed K split, a grouped (block-diagonal) weight, several output segments
in BF16 and fp32, and batch invariance -- a token's output bits do not
depend on the batch size, its position in the batch or the other tokens."""
import numpy as np
import pytest

from compressed_sparse_long_hca_b200 import inputs as I
from oracle import csa_oracle as O

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_lib):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return cuda_lib


def _bf16(a):
    return I.bf16_grid(np.asarray(a, np.float32))


def _check(gpu, ref_x, ref_w, groups, what, bf16_out=False):
    """|gpu - ref| <= 2e-5 sum_k |x_k w_k| (fp32 accumulation over K), plus
    half a BF16 ulp of the result for BF16 outputs."""
    ref = O.grouped_linear(ref_x, ref_w, groups) if groups > 1 else O.linear(ref_x, ref_w)
    mag = O.grouped_linear(np.abs(ref_x), np.abs(ref_w), groups) if groups > 1 else O.linear(np.abs(ref_x), np.abs(ref_w))
    bound = 2e-5 * mag + 1e-30 + (np.abs(ref) * 2.0 ** -8 if bf16_out else 0.0)
    err = np.abs(np.asarray(gpu, np.float64) - ref)
    assert np.all(err <= bound), f"{what}: {int((err > bound).sum())} outside; worst {float((err / (mag + 1e-30)).max()):.3e}"


@pytest.mark.parametrize("n_out,k_in,groups,n_tok", [
    (72, 200, 1, 5),             # ragged everything, one row tile, few K tiles
    (2368, 7168, 1, 4),          # hidden -> [c | z | c_I | z_I | w | c_q]: few row tiles, K split
    (9216, 1024, 1, 33),         # latent -> query heads: many row tiles, two token chunks
    (2048, 4096, 16, 7),         # grouped: 16 groups of 128 rows over 256 columns each
])
def test_gemm_matches_oracle(n_out, k_in, groups, n_tok):
    from compressed_sparse_long_hca_b200.api import Linear
    rng = np.random.default_rng(n_out + k_in)
    W = _bf16(rng.standard_normal((n_out, k_in // groups)) / np.sqrt(k_in // groups))
    x = _bf16(rng.standard_normal((n_tok, k_in)))
    lin = Linear(W, groups=groups)
    xd = torch.from_numpy(x).cuda().to(torch.bfloat16)
    y = torch.full((n_tok, n_out), float("nan"), device="cuda")
    lin(xd, y)
    Linear.check_device_error()
    _check(y.cpu().numpy(), x, W, groups, f"gemm {n_out}x{k_in}/{groups}")


def test_gemm_segments_bf16_and_fp32():
    """One fused weight writing several outputs: [c | z | c_I | z_I | w] in
    fp32 and the query latent in BF16, from one call."""
    from compressed_sparse_long_hca_b200.api import Linear
    rng = np.random.default_rng(7)
    rows = [512, 512, 128, 128, 64, 1024]
    n_out, k_in, n_tok = sum(rows), 1536, 6
    W = _bf16(rng.standard_normal((n_out, k_in)) / np.sqrt(k_in))
    x = _bf16(rng.standard_normal((n_tok, k_in)))
    lin = Linear(W)
    outs = [torch.full((n_tok, r), float("nan"), device="cuda") for r in rows[:-1]]
    outs.append(torch.zeros((n_tok, rows[-1]), dtype=torch.bfloat16, device="cuda"))
    lin(torch.from_numpy(x).cuda().to(torch.bfloat16), outs)
    Linear.check_device_error()
    r0 = 0
    for s, (r, t) in enumerate(zip(rows, outs)):
        _check(t.float().cpu().numpy(), x, W[r0:r0 + r], 1, f"segment {s}", bf16_out=t.dtype == torch.bfloat16)
        r0 += r


@pytest.mark.parametrize("n_out,k_in,groups", [(2368, 7168, 1), (9216, 1024, 1), (2048, 4096, 16)])
def test_gemm_batch_invariance(n_out, k_in, groups):
    """The same tokens in batches of 1, 5, 33 and 200 at shuffled positions:
    every token's output row is bit-identical."""
    from compressed_sparse_long_hca_b200.api import Linear
    rng = np.random.default_rng(11)
    W = _bf16(rng.standard_normal((n_out, k_in // groups)) / np.sqrt(k_in // groups))
    pool = _bf16(rng.standard_normal((200, k_in)))
    lin = Linear(W, groups=groups)
    xd = torch.from_numpy(pool).cuda().to(torch.bfloat16)
    base = torch.empty((200, n_out), device="cuda")
    lin(xd, base)
    for size in (1, 5, 33, 200):
        pick = rng.choice(200, size=size, replace=False)
        y = torch.empty((size, n_out), device="cuda")
        lin(xd[torch.from_numpy(pick).cuda()].contiguous(), y)
        assert torch.equal(y.view(torch.int32), base[torch.from_numpy(pick).cuda()].view(torch.int32)), size
    Linear.check_device_error()
