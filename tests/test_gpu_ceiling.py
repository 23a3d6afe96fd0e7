"""The tensor-core ceiling probe runs to completion on every SM and reports
a pipe time per block-scaled FP4 MMA in a plausible range (the MMA of
M=128, N=256, K=64 is 4.19 MFLOP; at the B200's nominal 9 PFLOP/s dense FP4
over 148 SMs and 1.965 GHz that is about 136 cycles)."""
import pytest
import torch

from nvfp4_moe_expert_topk_b200 import nvfp4_fp4_mma_ceiling

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("bn", [256, 128])
def test_ceiling_probe(bn):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    cycles = torch.full((sms,), -7, dtype=torch.int64, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    iters = 500
    nvfp4_fp4_mma_ceiling(bn, iters, cycles, err)
    torch.cuda.synchronize()
    assert err.item() == 0
    per_mma = cycles.double() / (iters * 4)
    assert (per_mma > 30).all() and (per_mma < 2000).all(), per_mma


@pytest.mark.parametrize("rows,stages", [(256, 2), (16384, 4), (262144, 6)])
def test_tma_stream_probe(rows, stages):
    """The TMA streaming probe completes without a timeout on every SM, for a
    one-tile matrix (every block re-reads it), an L2-resident one and one of
    0.9 GB, and moves its bytes at a plausible rate."""
    from nvfp4_moe_expert_topk_b200 import nvfp4_tma_stream_ceiling
    m = torch.randint(0, 256, (rows, 3584), dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    work = max(rows // 256, 296)
    nvfp4_tma_stream_ceiling(m, work, stages, err)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    nvfp4_tma_stream_ceiling(m, work, stages, err)
    b.record()
    torch.cuda.synchronize()
    assert err.item() == 0
    gbs = work * 256 * 3584 / (a.elapsed_time(b) * 1e-3) / 1e9
    assert 500 < gbs < 40000, gbs
