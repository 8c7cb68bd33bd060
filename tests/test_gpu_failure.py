"""Failure detection on the GPU without a fault: the bounded device wait of the tensor-core
pipeline gives up on a barrier that nothing completes and reports a timeout through the
status word, leaving the context usable; and the library's per-thread resources can be
released and recreated between calls."""
import pytest
import torch

from kv_cache_compression_group_b200 import jolt as J
from kv_cache_compression_group_b200 import synth

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_reports_timeout():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    J.wait_selftest(True, 200_000, status)          # arrival: the wait completes
    assert status.item() == 0
    with pytest.raises(J.JoltError) as e:           # no arrival: gives up after 50 ms
        J.wait_selftest(False, 50_000, status)
    assert e.value.name == "TIMEOUT"
    assert status.item() == 32                      # the timeout bit, set by the kernel
    # the context is still usable: a real call runs and agrees with itself
    J.wait_selftest(True, 200_000, status)
    x = torch.arange(10, device="cuda", dtype=torch.float32)
    assert float(x.sum()) == 45.0


def test_release_then_compress_again():
    w = synth.WORKLOADS["tiny"]
    K, V = (t.cuda() for t in synth.make_cache(w, 0))
    opts = J.Options((4, 8, 16, 32), (4, 8, 16), (0, 2, 3, 4), "randomized")
    comp = J.Compressor(w.n_layers, w.n_heads, w.T, w.D, w.layers_per_group, K.dtype, opts)
    budget = w.bf16_bytes() // 2
    blobs = [comp.compress(K, V, budget, 0) for _ in range(3)]   # direct, captured, replayed
    torch.cuda.synchronize()
    J.release()
    again = comp.compress(K, V, budget, 0)
    _, total, _ = J.read_header(again)
    for b in blobs:
        assert torch.equal(b[:total], again[:total])
    J.release()
