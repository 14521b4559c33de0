"""A decode step captured as a CUDA graph and replayed (how bench.py times the headline) gives
the bits of the same step run as eager calls: outputs, the cache bytes the fused append writes,
the abort flags and the status word."""
import numpy as np
import pytest
import torch

from synth.workloads import get_workload, small_variant

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from store_kv_attention_b200 import build_lib
    build_lib.build()


@pytest.mark.parametrize("name,split", [("int4_2b", 0), ("fp16_407m", 128), ("int8_b16", 512)])
def test_graph_replay_equals_eager_step(name, split):
    import store_kv_attention_b200 as tl
    from synth.device import DeviceWorkload
    w = small_variant(get_workload(name), ctx=[0, 130, 1025, 2100], loops=[8, 3, 8, 5], name=name + "_graph")
    eager = DeviceWorkload(w, split_rows=split, flag_mix=True)
    graphed = DeviceWorkload(w, split_rows=split, flag_mix=True, fill=False)
    # the same bytes everywhere, the positions no step writes included
    graphed.cache.codes.copy_(eager.cache.codes)
    if eager.cache.scales is not None:
        graphed.cache.scales.copy_(eager.cache.scales)
    eager.step(fused_append=True)
    # capture on a side stream after a warm-up there, as CUDA graphs require
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        graphed.step(fused_append=True)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graphed.reset_flags()
    graphed.out.fill_(float("nan"))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        graphed.step(fused_append=True)
    g.replay()
    torch.cuda.synchronize()
    a, b = eager.out.cpu().numpy(), graphed.out.cpu().numpy()
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    assert torch.equal(eager.cache.codes, graphed.cache.codes)
    if eager.cache.scales is not None:
        assert torch.equal(eager.cache.scales, graphed.cache.scales)
    assert torch.equal(eager.flags, graphed.flags) and torch.equal(eager.first, graphed.first)
    assert tl.poll_status(eager.cache) == tl.TL_OK and tl.poll_status(graphed.cache) == tl.TL_OK
    # a second replay over the same buffers gives the same bits again
    g.replay()
    torch.cuda.synchronize()
    assert np.array_equal(a.view(np.uint32), graphed.out.cpu().numpy().view(np.uint32))
