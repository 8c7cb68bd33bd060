"""The allocation-free Frobenius entry point (for callers that cannot allocate device memory,
e.g. programs whose device memory is owned by another allocator) must return what the
workspace-taking entry point returns, call after call, although all its calls share one
scratch array inside the library.  Named to run last in the suite."""
import pytest
import torch

from kv_cache_compression_group_b200 import jolt as J
from kv_cache_compression_group_b200 import synth

pytestmark = pytest.mark.gpu


def test_noalloc_matches_workspace_entry_point_twice():
    w = synth.small_workload("mistral7b", n_layers=8, n_heads=2, T=256)
    K, V = (t.cuda() for t in synth.make_cache(w, 3))
    Kh = (K.float() * 1.01).contiguous()
    Vh = (V.float() - 0.02).contiguous()
    want = J.frobenius(K, V, Kh, Vh, w.layers_per_group)
    for _ in range(2):
        got = J.frobenius_noalloc(K, V, Kh, Vh, w.layers_per_group)
        torch.cuda.synchronize()
        assert torch.allclose(got, want, rtol=1e-12, atol=0.0)
    # without the second operand: only the squared norms
    want0 = J.frobenius(K, V, None, None, w.layers_per_group)
    for _ in range(2):
        got0 = J.frobenius_noalloc(K, V, None, None, w.layers_per_group)
        assert torch.allclose(got0, want0, rtol=1e-12, atol=0.0)


def test_noalloc_rejects_too_many_units():
    w = synth.small_workload("mistral7b", n_layers=66, n_heads=1, T=16)
    K, V = (t.cuda() for t in synth.make_cache(w, 0))
    with pytest.raises(J.JoltError) as e:
        J.frobenius_noalloc(K, V, None, None, 1)
    assert e.value.name == "WORKSPACE_TOO_SMALL" and "64" in str(e.value)


def test_noalloc_largest_accepted_unit_count_and_fp32_cache():
    """64 units (the limit: the highest slots of the compiled-in array) and an fp32 cache
    with an fp32 second operand, each against the workspace entry point, twice in a row."""
    w = synth.small_workload("mistral7b", n_layers=32, n_heads=1, T=32)
    K, V = (t.cuda() for t in synth.make_cache(w, 5))
    Kh, Vh = (K.float() * 0.99).contiguous(), (V.float() + 0.01).contiguous()
    want = J.frobenius(K, V, Kh, Vh, 1)
    assert want.shape[0] == 64
    for _ in range(2):
        got = J.frobenius_noalloc(K, V, Kh, Vh, 1)
        assert torch.allclose(got, want, rtol=1e-12, atol=0.0)
    Kf, Vf = K.float().contiguous(), V.float().contiguous()
    want = J.frobenius(Kf, Vf, Kh, Vh, 2)
    for _ in range(2):
        got = J.frobenius_noalloc(Kf, Vf, Kh, Vh, 2)
        assert torch.allclose(got, want, rtol=1e-12, atol=0.0)
