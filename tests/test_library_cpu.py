"""Host-side checks of libjolt.so that need no GPU: the library loads, exports every symbol
include/jolt.h declares, and its host logic (argument validation, workspace plan, byte
accounting) behaves as documented."""
import ctypes
import os
import re

import pytest

import oracle as O
from kv_cache_compression_group_b200 import jolt as J
from kv_cache_compression_group_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    text = open(os.path.join(ROOT, "include", "jolt.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(jolt_[a-z0-9_]+)\s*\(", text)))


def test_library_loads_and_exports_every_declared_symbol():
    L = J.lib()
    declared = _declared_symbols()
    assert len(declared) >= 13
    for name in declared:
        assert hasattr(L, name), name
    assert set(declared) == set(J.EXPORTED)
    assert b"sm_100a" in L.jolt_version()


def _shape(w):
    return J.CShape(w.n_layers, w.n_heads, w.T, w.D, w.layers_per_group, J.JOLT_BF16 if w.dtype == "bf16" else J.JOLT_F32)


@pytest.mark.parametrize("name", ["tiny", "mistral7b", "llama2_13b", "llama31_8b_64k"])
@pytest.mark.parametrize("method", ["exact", "randomized"])
def test_workspace_plan_on_host(name, method):
    w = synth.WORKLOADS[name]
    opts = (J.Options((4, 8, 16, 32), (4, 8, 16), (0, 2, 3, 4), method) if name == "tiny"
            else J.default_options(w.T, w.D, method))
    ws, blob, dws = J.sizes(_shape(w), opts)
    assert ws > 0 and dws > 0
    nu, nc = J.counts(_shape(w), opts)
    assert nu == 2 * w.n_groups and nc == opts.n_choices
    # the largest blob: headers + every unit at its largest choice
    S = w.layers_per_group * w.n_heads
    mx = max(O.unit_payload_bytes(w.T, w.D, S, rt, rd, b)
             for rt in opts.token_ranks for rd in opts.feature_ranks for b in opts.bits)
    assert blob == O.header_bytes(nu) + nu * mx


@pytest.mark.parametrize("name", ["tiny", "mistral7b", "llama2_13b"])
def test_choice_bytes_match_oracle(name):
    w = synth.WORKLOADS[name]
    opts = (J.Options((4, 8, 16, 32), (4, 8, 16), (0, 2, 3, 4)) if name == "tiny"
            else J.default_options(w.T, w.D))
    got = J.choice_bytes(_shape(w), opts)
    oo = O.Options(opts.token_ranks, opts.feature_ranks, opts.bits)
    want = O.bytes_table(w.T, w.D, w.layers_per_group * w.n_heads, oo).reshape(-1)
    assert list(want) == got


def _status(f):
    try:
        f()
    except J.JoltError as e:
        return e.name
    return "OK"


def test_argument_errors_on_host():
    w = synth.WORKLOADS["tiny"]
    good = J.Options((4, 8, 16, 32), (4, 8, 16), (0, 2, 3, 4))
    sh = _shape(w)
    assert _status(lambda: J.sizes(sh, good)) == "OK"
    bad_d = J.CShape(2, 2, 64, 24, 2, J.JOLT_F32)
    assert _status(lambda: J.sizes(bad_d, good)) == "UNSUPPORTED_SHAPE"
    bad_t = J.CShape(2, 2, 60, 16, 2, J.JOLT_F32)
    assert _status(lambda: J.sizes(bad_t, good)) == "UNSUPPORTED_SHAPE"
    bad_g = J.CShape(3, 2, 64, 16, 2, J.JOLT_F32)
    assert _status(lambda: J.sizes(bad_g, good)) == "UNSUPPORTED_SHAPE"
    assert _status(lambda: J.sizes(sh, J.Options((8, 4), (4,), (0,)))) == "INVALID_ARG"        # not ascending
    assert _status(lambda: J.sizes(sh, J.Options((4, 8, 16, 65), (4,), (0,)))) == "INVALID_ARG"  # > min(T, M)
    assert _status(lambda: J.sizes(sh, J.Options((8,), (4, 17), (0,)))) == "INVALID_ARG"       # > D
    assert _status(lambda: J.sizes(sh, J.Options((8,), (8,), (0, 9)))) == "INVALID_ARG"        # > 8 bits
    assert _status(lambda: J.sizes(sh, J.Options((4, 12), (8,), (0,)))) == "UNSUPPORTED_SHAPE"  # max % 8
    assert _status(lambda: J.sizes(sh, J.Options((8,), (8,), (0,), "randomized", oversample=60))) == "UNSUPPORTED_SHAPE"
    bad_dtype = J.CShape(2, 2, 64, 16, 2, 7)
    assert _status(lambda: J.sizes(bad_dtype, good)) == "INVALID_ARG"


def test_null_pointer_calls_fail_before_any_launch():
    """Calls with null device pointers are rejected by the host checks (no GPU touched)."""
    L = J.lib()
    w = synth.WORKLOADS["tiny"]
    sh = _shape(w)
    o = J.Options((4, 8, 16, 32), (4, 8, 16), (0, 2, 3, 4)).c()
    ws, blob, _ = J.sizes(sh, J.Options((4, 8, 16, 32), (4, 8, 16), (0, 2, 3, 4)))
    st = L.jolt_compress(ctypes.byref(sh), None, None, ctypes.byref(o), 8192, 0, None, blob, None, ws, None)
    assert J.STATUS_NAMES[st] == "INVALID_ARG"
    st = L.jolt_compress(ctypes.byref(sh), ctypes.c_void_p(256), ctypes.c_void_p(256), ctypes.byref(o), 8192, 0,
                         ctypes.c_void_p(256), blob, ctypes.c_void_p(256), 16, None)
    assert J.STATUS_NAMES[st] == "WORKSPACE_TOO_SMALL"
    st = L.jolt_allocate(None, None, 0, 0, 0, None, None, None, None)
    assert J.STATUS_NAMES[st] == "INVALID_ARG"
    st = L.jolt_decompress(None, 3, None, None, None, 0, None)
    assert J.STATUS_NAMES[st] == "INVALID_ARG"
    assert b"out_dtype" in L.jolt_last_error()


def test_struct_layouts():
    assert ctypes.sizeof(J.CShape) == 24
    assert ctypes.sizeof(J.COptions) == 4 * (3 + 3 * J.MAXC + 4)   # + method, oversample, power_iters, unit_offset
    assert ctypes.sizeof(J.CUnitRecord) == 64


def test_build_tracks_every_source_file():
    """A kernel header missing from the rebuild check would leave a stale library in place."""
    import os
    from kv_cache_compression_group_b200 import build
    on_disk = sorted(f for f in os.listdir(build.CSRC) if f.endswith((".cu", ".cuh")))
    assert sorted(build.DEPS) == on_disk
    assert all(s in build.DEPS for s in build.SOURCES)
