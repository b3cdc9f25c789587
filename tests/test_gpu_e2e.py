"""The end-to-end decode step the benchmark times (bench.end_to_end_decode): host allocator work,
incremental block-table updates applied on the device, one CUDA graph per step with the batch cut
into slices whose copies overlap the kernels.  The function checks its own result (device tables
against the full export, the last output bit for bit against one device-resident call on the same
state) and raises on a mismatch; these tests run it on small batches."""
import importlib.util
import os
import types

import numpy as np
import pytest

from paged_kv_cache_356_b200 import binding as pa
from paged_kv_cache_356_b200 import workloads
from paged_kv_cache_356_b200.runner import TraceRunner

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("slices", [1, 3, 5])
@pytest.mark.parametrize("num_seqs,bs", [(24, 16), (9, 32)])
def test_end_to_end_decode_matches_a_device_resident_call(num_seqs, bs, slices):
    import torch
    bench = _bench()
    w = workloads.llama8b(num_seqs=num_seqs, block_size=bs)
    run = TraceRunner(w)
    run.run(decode=False)
    torch.cuda.synchronize()
    before = {b: run.alloc.num_tokens(b) for b in range(w.num_seqs)}
    kd, vd, _ = run.step_write
    args = types.SimpleNamespace(steps=6)
    e2e = bench.end_to_end_decode(args, torch, pa, run, w, 1, None, (run.q, kd, vd), slices)
    # 3 warm-up steps and the timed ones each grew every sequence by one token
    assert all(run.alloc.num_tokens(b) == before[b] + 3 + 6 for b in range(w.num_seqs))
    assert e2e["value"] > 0 and e2e["slices"] == slices
    q_bytes = run.q.numel() * run.q.element_size()
    assert e2e["d2h_bytes_per_step"] == q_bytes
    assert e2e["h2d_bytes_per_step"] >= q_bytes
    assert np.isfinite(e2e["ms_per_step"])
