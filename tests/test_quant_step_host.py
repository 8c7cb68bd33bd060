"""The library's block quantiser compiled for the host from the same source the kernels use,
against the oracle:

* the exact fp16 block scales (lo = fp16 round-down of the block minimum, step = smallest
  fp16 s with s * (2^b - 1) >= max - lo), bit for bit, on random and adversarial blocks, in
  the branching form, the select form and the bracketed conversion form
  (values at and next to fp16 numbers, steps landing exactly on fp16 numbers, the fp16
  subnormal range, overflow, equal minimum and maximum);
* the packed code bytes, bit for bit with the oracle's packing of the same codes, and their
  unpacking;
* the codes themselves: the library rounds (x - lo) * fp32(1/step), the oracle rounds
  (x - lo) / step in float64, so they may differ only where the quotient lies within fp32
  rounding of a half-integer."""
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "kv_cache_compression_group_b200", "csrc")
BITS = (1, 2, 3, 4, 8)


def _cases(rng):
    f32 = np.float32
    mn, mx = [], []
    # random blocks at many scales
    for scale in (1e-7, 1e-5, 3e-4, 1e-2, 1.0, 37.0, 1e3, 3e4):
        x = (rng.standard_normal((4000, 16)) * scale).astype(f32)
        mn.append(x.min(1))
        mx.append(x.max(1))
    # minima on fp16 numbers and one fp32 ulp either side
    h = rng.uniform(-6e4, 6e4, 3000).astype(np.float16).astype(f32)
    for m in (h, np.nextafter(h, f32(np.inf)), np.nextafter(h, f32(-np.inf))):
        mn.append(m)
        mx.append(m + np.abs(rng.standard_normal(m.size)).astype(f32) * f32(3.0))
    # maxima that put (max - lo) / levels exactly on an fp16 number, and one ulp either side
    lo = O.fp16_rd(rng.standard_normal(3000) * 4.0).astype(f32)
    for b in BITS:
        s = np.abs(rng.standard_normal(3000) * 0.5).astype(np.float16).astype(f32)
        exact = (lo.astype(np.float64) + s.astype(np.float64) * ((1 << b) - 1)).astype(f32)
        for m in (exact, np.nextafter(exact, f32(np.inf)), np.nextafter(exact, f32(-np.inf))):
            mn.append(lo)
            mx.append(np.maximum(m, lo))
    # fp16 subnormal range, overflow, degenerate blocks
    t = (rng.standard_normal((2000, 16)) * 2e-6).astype(f32)
    mn.append(t.min(1))
    mx.append(t.max(1))
    big = rng.uniform(-7e4, 7e4, (2000, 2)).astype(f32)
    mn.append(big.min(1))
    mx.append(big.max(1))
    eq = rng.standard_normal(500).astype(f32)
    mn.append(eq)
    mx.append(eq)
    return np.concatenate(mn), np.concatenate(mx)


@pytest.fixture(scope="module")
def host_prog(tmp_path_factory):
    nvcc = shutil.which("nvcc")
    if nvcc is None:
        pytest.skip("nvcc not available")
    exe = str(tmp_path_factory.mktemp("qstep") / "quant_step_host")
    subprocess.run([nvcc, "-std=c++17", "-O2", "-Wno-deprecated-gpu-targets", "-I", CSRC, "-o", exe, os.path.join(ROOT, "tests", "quant_step_host.cu")],
                   check=True, capture_output=True)
    return exe


def _compile(tmp_path_factory, name):
    nvcc = shutil.which("nvcc")
    if nvcc is None:
        pytest.skip("nvcc not available")
    exe = str(tmp_path_factory.mktemp(name) / name)
    subprocess.run([nvcc, "-std=c++17", "-O2", "-Wno-deprecated-gpu-targets", "-I", CSRC, "-o", exe,
                    os.path.join(ROOT, "tests", name + ".cu")], check=True, capture_output=True)
    return exe


@pytest.fixture(scope="module")
def codes_prog(tmp_path_factory):
    return _compile(tmp_path_factory, "quant_codes_host")


@pytest.mark.parametrize("b", BITS)
def test_codes_and_packing(codes_prog, b):
    rng = np.random.default_rng(100 + b)
    blocks = [(rng.standard_normal((3000, 16)) * s) for s in (1e-4, 0.05, 1.0, 30.0)]
    # blocks whose values sit on and next to the quantiser's half-integer levels
    lo = O.fp16_rd(rng.standard_normal(2000))
    step = O.fp16_ru(np.abs(rng.standard_normal(2000)) * 0.1 + 1e-3)
    k = rng.integers(0, (1 << b) - 1, (2000, 16)) + 0.5
    x = lo[:, None] + k * step[:, None]
    x[:, 0] = lo
    x[:, 1] = lo + ((1 << b) - 1) * step
    blocks.append(x)
    v = np.concatenate(blocks).astype(np.float32)
    out = subprocess.run([codes_prog], input=np.int32(b).tobytes() + v.tobytes(), capture_output=True,
                         check=True).stdout
    rec = np.frombuffer(out, dtype=np.dtype([("lo", "<f4"), ("step", "<f4"), ("codes", "u1", 16),
                                             ("bytes", "u1", 16), ("back", "u1", 16)]))
    assert rec.shape[0] == v.shape[0]
    codes = rec["codes"].astype(np.int64)
    nbytes = 2 * b
    # packing: bit for bit the oracle's packing of the same codes; unpacking inverts it
    np.testing.assert_array_equal(rec["bytes"][:, :nbytes], O.pack_codes(codes[:, None, :], b))
    assert not rec["bytes"][:, nbytes:].any()
    np.testing.assert_array_equal(rec["back"].astype(np.int64), codes)
    np.testing.assert_array_equal(O.unpack_codes(rec["bytes"][:, :nbytes], b)[:, 0, :], codes)
    # codes: the oracle's quantiser on the same fp32 block; differences only at ties
    ref_codes, ref_lo, ref_step, _, ok = O.quantize(v.astype(np.float64), b)
    ref_codes, ref_lo, ref_step, ok = ref_codes[:, 0, :], ref_lo[:, 0], ref_step[:, 0], ok[:, 0]
    assert ok.all()
    np.testing.assert_array_equal(rec["lo"].astype(np.float64), ref_lo)
    np.testing.assert_array_equal(rec["step"].astype(np.float64), ref_step)
    diff = codes != ref_codes
    q = (v.astype(np.float64) - ref_lo[:, None]) / np.where(ref_step > 0, ref_step, 1.0)[:, None]
    near_tie = np.abs(q - np.floor(q) - 0.5) <= 4 * np.finfo(np.float32).eps * np.maximum(np.abs(q), 1.0)
    assert np.all(near_tie[diff])
    assert np.all(np.abs(codes - ref_codes) <= 1)
    # the stated bound on random blocks (the constructed blocks above are ties on purpose)
    n_random = sum(x.shape[0] for x in blocks[:-1])
    assert diff[:n_random].mean() <= 1e-4


def test_block_scales_match_the_oracle_bit_for_bit(host_prog):
    rng = np.random.default_rng(7)
    mn, mx = _cases(rng)
    pairs = np.stack([mn, mx], 1).astype(np.float32)
    out = subprocess.run([host_prog], input=pairs.tobytes(), capture_output=True, check=True).stdout
    got = np.frombuffer(out, dtype=np.float32).reshape(-1, 16).astype(np.float64)
    assert got.shape[0] == pairs.shape[0]
    lo = O.fp16_rd(mn.astype(np.float64))
    np.testing.assert_array_equal(got[:, 0], lo)
    for j, b in enumerate(BITS):
        levels = (1 << b) - 1
        with np.errstate(invalid="ignore", over="ignore"):
            ref = np.where(mx.astype(np.float64) > lo, O.fp16_ru((mx.astype(np.float64) - lo) / levels), 0.0)
        np.testing.assert_array_equal(got[:, 1 + j], ref, err_msg=f"b = {b}")
        # the branch-free form and the bracketed conversion form: the same value in every case
        np.testing.assert_array_equal(got[:, 6 + j], ref, err_msg=f"b = {b} (select form)")
        np.testing.assert_array_equal(got[:, 11 + j], ref, err_msg=f"b = {b} (conversion form)")
    # the cases reach every branch: ties on fp16 numbers, subnormal steps, overflow, zero step
    steps = got[:, 1:]
    assert np.any(steps == 0.0) and np.any(np.isinf(steps)) and np.any((steps > 0) & (steps < 6.103515625e-05))
