"""The NVFP4 block scale on E4M3 rounding points ("NVFP4 与 MXFP4 格式"
section 3: b = Q_E4M3(A_b / (6a))).  Inputs are built so that A_b / (6g)
lands on an E4M3 value or on the midpoint between two, or one fp32 step
beside one.  With A = 2688, g = 1 and A_b = 6 P is exact, so the quotient is
exactly P (exact ties at the midpoints).  With A = 308, g = fl32(11/96) and
6g is within an fp32 step of 11/16: A_b = fl32(6 g P) puts the quotient a
tiny nonzero distance from P (near ties, the case of an input like the GEMM
workload's activation).  The kernels decide both by an fma comparison
instead of a division; codes, scale bytes, g and losses must equal the
oracle's bit for bit, for the quantiser and for the search and four over
six, which round the same quotient (and A_b / (4g))."""
import numpy as np
import pytest
import torch

import block_scaled_fp4_reduce_b200 as fp4
import oracle
from test_gpu_parity import assert_same, odata

pytestmark = pytest.mark.gpu
DEV = "cuda"


def tie_tensor(dtype: torch.dtype, A: float) -> torch.Tensor:
    """One block per target: the block maximum at fl32(6 g P) or one fp32
    step below or above it, for every E4M3 value and midpoint P of the
    normal range; the block's other elements uniform in (-0.9, 0.9) A_b; the
    tensor maximum A in the first block."""
    g = float(np.float32(A / 2688.0))
    targets = []
    for c in range(8, 126):
        v, w = oracle.e4m3_value(c), oracle.e4m3_value(c + 1)
        for p in (v, (v + w) / 2):
            a = np.float32(6.0 * g * p)
            targets += [a, np.nextafter(a, np.float32(0)), np.nextafter(a, np.float32(1e9))]
    rng = np.random.default_rng(11)
    n_blocks = -(-(len(targets) + 1) // 16) * 16
    x = np.zeros((n_blocks, 16), np.float32)
    amaxes = [np.float32(A)] + targets
    amaxes += [np.float32(rng.uniform(0.01, 0.95) * A) for _ in range(n_blocks - len(amaxes))]
    for b, a in enumerate(amaxes):
        row = (rng.uniform(-0.9, 0.9, 16) * a).astype(np.float32)
        row[rng.integers(16)] = a * (1 if rng.random() < 0.5 else -1)
        x[b] = row
    return torch.from_numpy(x.reshape(-1, 256)).to(dtype)


def exact_ties(x: torch.Tensor) -> int:
    """Blocks whose A_b / (6g) is exactly an E4M3 midpoint."""
    ab = x.float().abs().reshape(-1, 16).amax(dim=1).double().numpy()
    t = ab / (6.0 * float(np.float32(x.float().abs().max().item() / 2688.0)))
    mids = {(oracle.e4m3_value(c) + oracle.e4m3_value(c + 1)) / 2 for c in range(126)}
    return int(sum(1 for v in t if v in mids))


@pytest.mark.parametrize("A", [2688.0, 308.0])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_block_scale_at_e4m3_midpoints(dtype, A):
    x = tie_tensor(dtype, A)
    if dtype == torch.float32 and A == 2688.0:
        assert exact_ties(x) >= 100
    xo, xd = odata(x), x.to(DEV)
    q = fp4.nvfp4_quantize(xd)
    ss = fp4.scale_search(xd)
    fo = fp4.nvfp4_quantize_four_over_six(xd)
    torch.cuda.synchronize()
    for r in (q, ss, fo):
        r.check("ties")
    p, s, g = oracle.nvfp4_quantize(xo)
    assert q.global_scale.item() == g == np.float32(A / 2688.0)
    assert_same(q.scales, s, f"NVFP4 scales at E4M3 midpoints ({dtype})")
    assert_same(q.packed, p, f"NVFP4 codes at E4M3 midpoints ({dtype})")
    p, s, g, loss = oracle.nvfp4_scale_search(xo)
    assert_same(ss.scales, s, f"search scales ({dtype})")
    assert_same(ss.packed, p, f"search codes ({dtype})")
    assert_same(ss.block_loss, loss.astype(np.float32), f"search loss ({dtype})")
    p, s, g, loss = oracle.nvfp4_quantize_four_over_six(xo)
    assert_same(fo.scales, s, f"four over six scales ({dtype})")
    assert_same(fo.packed, p, f"four over six codes ({dtype})")
