"""The row-sharded step's device calls on one GPU: the shards of a tensor
run the bench's pre-bound calls one after another -- each shard's amax, then
the max of those amaxes (what the all-reduce of the multi-GPU mode gives
every rank), then the shard's NVFP4 quantiser and search with that amax and
its MXFP4 quantiser and dequantisers -- and every output equals the
unsharded step's rows bit for bit (g belongs to the whole tensor, "NVFP4 与
MXFP4 格式" section 3; the blocks are independent).  No shard waits on
another: the ranks' exchange is replaced by a sequential max on the host
side of the calls."""
import pytest
import torch

import bench
import workloads

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run_calls(path, idx):
    for i in idx:
        fn, args = path.calls[i]
        assert fn(*args) == 0, fn.__name__


@pytest.mark.parametrize("world", [2, 3])
def test_row_shards_reproduce_the_whole_tensor(world):
    w = workloads.with_shape(workloads.ACT_8K, 301, 2048, 60)
    x = workloads.generate(w).to(DEV)
    full = bench.Path(x)
    run_calls(full, range(len(full.calls)))
    shards = []
    for rank in range(world):
        r0, r1 = bench.shard_rows(x.shape[0], world, rank)
        shards.append((r0, r1, bench.Path(x[r0:r1])))
    for _, _, p in shards:
        run_calls(p, [0])                                      # local amax
    a = torch.stack([p.amax for _, _, p in shards]).max()      # the all-reduce(MAX)
    for _, _, p in shards:
        p.amax.copy_(a.reshape(1))
        run_calls(p, range(1, len(p.calls)))                   # the rest with the shared A
    torch.cuda.synchronize()
    assert int(full.status.item()) == 0
    for r0, r1, p in shards:
        assert int(p.status.item()) == 0
        assert torch.equal(p.amax, full.amax)
        assert torch.equal(p.nv_g, full.nv_g) and torch.equal(p.ss_g, full.ss_g)
        for got, want in ((p.nv_p, full.nv_p), (p.nv_s, full.nv_s), (p.mx_p, full.mx_p), (p.mx_s, full.mx_s),
                          (p.ss_p, full.ss_p), (p.ss_s, full.ss_s)):
            assert torch.equal(got, want[r0:r1])
        for got, want in ((p.y_nv, full.y_nv), (p.y_mx, full.y_mx)):
            assert torch.equal(got.view(torch.int16), want[r0:r1].view(torch.int16))
