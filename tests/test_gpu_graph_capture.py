"""The decode entry points can be captured in a CUDA graph (as a decode loop replays a step) and the
replay gives the eager result bit for bit: pa_decode on an independent batch, pa_decode_shared_prefix
(whose per-sequence kernel is a programmatic dependent of the joint kernel) on a forked one."""
import pytest

from paged_kv_cache_356_b200 import binding as pa
from paged_kv_cache_356_b200 import workloads
from paged_kv_cache_356_b200.runner import TraceRunner

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("make,shared", [
    (lambda: workloads.llama8b(num_seqs=12, lo=100, hi=2500), False),
    (lambda: workloads.beam32k(num_beams=4, prompt_len=2600, own=30), True),
    (lambda: workloads.prefix(num_seqs=20, prefix_len=1800, max_tail=300), True),
], ids=["independent", "beam", "prefix"])
def test_step_replays_from_a_graph(make, shared):
    import torch
    w = make()
    run = TraceRunner(w, shared_prefix=shared)
    eager = run.run().clone()
    assert run.status() == 0
    run.out.zero_()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        run.step(stream=side)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    run.out.zero_()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        run.step(stream=torch.cuda.current_stream())
    for _ in range(3):
        run.out.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(run.out.view(torch.int16), eager.view(torch.int16))
    assert run.status() == 0
    del graph
