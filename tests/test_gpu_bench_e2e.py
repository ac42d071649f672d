"""The benchmark's end-to-end leg overlaps copies in, the chain and copies
out on three streams with two device buffer sets.  Its outputs must be the
ones a plain single-stream run of the chain gives on the same inputs: a
missing wait between the streams would show as a changed output here while
the timing still looked fine."""
import pytest
import torch

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from dit_block_pass_b200 import build
    build.build()


def test_pipelined_e2e_outputs_equal_a_single_stream_run():
    import bench
    from dit_block_pass_b200 import workloads as W
    wl = W.CONFIGS["small"]
    chain = bench.Chain(wl, DEV)
    ms, h2d, d2h, host_in, host_out = bench.time_e2e(chain, 5, 2, 1, keep_outputs=True)
    assert ms > 0 and h2d > 0 and d2h > 0
    # the same inputs through the chain on one stream
    for name, h in host_in.items():
        getattr(chain, name).copy_(h)
    for op in chain.ops():
        op()
    torch.cuda.synchronize()
    for name, h in host_out.items():
        ref = getattr(chain, name).cpu()
        assert torch.equal(h.view(torch.uint8), ref.view(torch.uint8)), name
