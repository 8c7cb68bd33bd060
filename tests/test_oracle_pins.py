"""Pins of the float64 oracle against facts that do not come from the oracle itself:
published test vectors, hand-worked examples, library routines (LAPACK SVD, scipy's
Hadamard matrix, ml_dtypes / numpy float16 tables), closed forms and brute force."""
import itertools
import math
import os

import numpy as np
import pytest
import scipy.linalg
import scipy.stats

import oracle as O


def _read_golden(golden_dir, name):
    rows = []
    with open(os.path.join(golden_dir, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line)
    return rows


# ------------------------------------------------------------------ random numbers
def test_splitmix64_published_vector(golden_dir):
    want = [int(x) for x in _read_golden(golden_dir, "splitmix64_seed0.txt")]
    # the generator's state advances by the golden gamma before each output; our mix
    # function adds the gamma itself, so output n is mix(n * gamma)
    states = np.array([(n * O.GOLDEN_GAMMA) & ((1 << 64) - 1) for n in range(3)], dtype=np.uint64)
    got = [int(x) for x in O.splitmix64_mix(states)]
    assert got == want


def test_gaussian_is_standard_normal():
    z = O.gaussian(7, O.stream_id(O.STREAM_OMEGA, 3, 1), np.arange(200_000, dtype=np.uint64))
    assert np.all(np.isfinite(z))
    ks = scipy.stats.kstest(z, "norm")
    assert ks.pvalue > 1e-3
    assert abs(z.mean()) < 0.01 and abs(z.var() - 1) < 0.02


def test_signs_balanced_and_stream_dependent():
    s0 = O.rotation_signs(0, 0, 0, 4096)
    s1 = O.rotation_signs(0, 0, 1, 4096)
    assert set(np.unique(s0)) == {-1.0, 1.0}
    assert abs(s0.mean()) < 0.1
    assert np.mean(s0 != s1) > 0.4


# ------------------------------------------------------------------ rounding
def test_bf16_rn_matches_ml_dtypes_on_f32_inputs():
    import ml_dtypes
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(100_000) * np.exp(rng.uniform(-30, 30, 100_000))).astype(np.float32)
    ref = x.astype(ml_dtypes.bfloat16).astype(np.float64)
    got = O.bf16_rn(x.astype(np.float64))
    assert np.array_equal(ref, got)


def _all_fp16_finite():
    v = np.arange(65536, dtype=np.uint32).astype(np.uint16).view(np.float16).astype(np.float64)
    return np.unique(v[np.isfinite(v)])


def test_fp16_directed_rounding_brute_force():
    tab = _all_fp16_finite()
    rng = np.random.default_rng(2)
    x = rng.standard_normal(50_000) * np.exp(rng.uniform(-20, 12, 50_000))
    x = np.concatenate([x, tab[::97], [0.0, 65504.0, -65504.0, 65519.0, 1e-9, -1e-9]])
    x = x[np.abs(x) <= 65504.0]
    rd = tab[np.searchsorted(tab, x, side="right") - 1]       # largest fp16 <= x
    ru = tab[np.searchsorted(tab, x, side="left")]             # smallest fp16 >= x
    assert np.array_equal(O.fp16_rd(x), rd)
    assert np.array_equal(O.fp16_ru(x), ru)
    assert O.fp16_ru(70000.0) == np.inf and O.fp16_rd(70000.0) == 65504.0
    assert O.fp16_rd(-70000.0) == -np.inf and O.fp16_ru(-70000.0) == -65504.0


# ------------------------------------------------------------------ rotation
@pytest.mark.parametrize("D", [16, 64, 128])
def test_fwht_is_sylvester_hadamard(D):
    H = scipy.linalg.hadamard(D).astype(np.float64)
    x = np.random.default_rng(D).standard_normal((5, D))
    assert np.allclose(O.fwht(x), x @ H.T, atol=1e-12, rtol=0)


def test_rotation_orthogonal_and_invertible():
    rng = np.random.default_rng(3)
    R = rng.standard_normal((3, 7, 128))
    sig = O.rotation_signs(5, 1, 0, 128)
    rho = O.rotate(R, sig)
    assert np.allclose(np.linalg.norm(rho, axis=-1), np.linalg.norm(R, axis=-1), rtol=1e-14, atol=0)
    assert np.allclose(O.unrotate(rho, sig), R, atol=1e-13, rtol=0)
    # dense matrix form of the same map
    Phi = np.diag(sig) @ scipy.linalg.hadamard(128) / math.sqrt(128)
    assert np.allclose(rho, R @ Phi, atol=1e-13, rtol=0)


# ------------------------------------------------------------------ Tucker factors
def _rand_cache(rng, Lg, H, T, D):
    return rng.standard_normal((Lg, H, T, D)) * np.exp(-np.arange(D) / D)[None, None, None, :]


def test_full_rank_tucker_reconstructs_exactly():
    rng = np.random.default_rng(4)
    X = _rand_cache(rng, 2, 2, 24, 16)          # T=24 <= M=64
    _, W = O.feature_factor(X)
    U = O.token_factor_exact(X, 24)
    C = O.tucker_core(X, U, W)
    err = np.linalg.norm(X - O.tucker_reconstruct(U, C, W)) / np.linalg.norm(X)
    assert err < 1e-12


@pytest.mark.parametrize("method", ["exact", "randomized"])
@pytest.mark.parametrize("rT,rD", [(4, 4), (8, 12), (20, 3)])
def test_energy_split(method, rT, rD):
    rng = np.random.default_rng(5 + rT)
    X = _rand_cache(rng, 2, 2, 40, 16)
    _, W = O.feature_factor(X)
    if method == "exact":
        U = O.token_factor_exact(X, rT)
    else:
        U = O.token_factor_randomized(X, rT, 6, 2, 11, 0, 0)
    W = W[:, :rD]
    C = O.tucker_core(X, U, W)
    lhs = np.sum(X * X)
    rhs = np.sum(C * C) + np.sum((X - O.tucker_reconstruct(U, C, W)) ** 2)
    assert abs(lhs - rhs) <= 1e-12 * lhs
    assert np.allclose(U.T @ U, np.eye(rT), atol=1e-12)


@pytest.mark.parametrize("r", [1, 3, 7])
def test_eckart_young_single_slice(r):
    """One layer, one head: the factors are the matrix's singular vectors and the
    truncation error is the tail of the squared singular values (LAPACK SVD)."""
    rng = np.random.default_rng(6)
    A = rng.standard_normal((30, 16)) @ np.diag(np.exp(-np.arange(16) / 3.0))
    X = A[None, None]
    _, W = O.feature_factor(X)
    U = O.token_factor_exact(X, r)
    C = O.tucker_core(X, U, W[:, :r])
    err = np.sum((X - O.tucker_reconstruct(U, C, W[:, :r])) ** 2)
    s = np.linalg.svd(A, compute_uv=False)
    assert abs(err - np.sum(s[r:] ** 2)) <= 1e-10 * np.sum(s ** 2)
    Ul, _, Vt = np.linalg.svd(A)
    assert np.allclose(np.abs(U.T @ Ul[:, :r]), np.eye(r), atol=1e-8)
    assert np.allclose(np.abs(W[:, :r].T @ Vt[:r].T), np.eye(r), atol=1e-8)


def _tucker_exact_cache(rng, Lg, H, T, D, k):
    """Shared token / feature bases, per-slice k x k coefficients, no noise: exact
    multilinear rank (k, k) on the token and feature modes."""
    A = np.linalg.qr(rng.standard_normal((T, k)))[0]
    B = np.linalg.qr(rng.standard_normal((D, k)))[0]
    Cs = rng.standard_normal((Lg, H, k, k))
    return np.einsum("tk,lhkj,dj->lhtd", A, Cs, B)


def test_tucker_exact_generator_zero_truncation_error():
    rng = np.random.default_rng(7)
    X = _tucker_exact_cache(rng, 2, 3, 48, 16, 5)
    _, W = O.feature_factor(X)
    U = O.token_factor_exact(X, 5)
    C = O.tucker_core(X, U, W[:, :5])
    assert np.linalg.norm(X - O.tucker_reconstruct(U, C, W[:, :5])) <= 1e-10 * np.linalg.norm(X)
    Ur = O.token_factor_randomized(X, 5, 4, 1, 3, 0, 1)
    assert np.linalg.norm(U @ U.T - Ur @ Ur.T) < 1e-8


def _sin_theta(U1, U2):
    """Largest principal-angle sine between span(U1) and span(U2) (orthonormal columns):
    the spectral norm of the part of U2 outside span(U1)."""
    return float(np.linalg.norm(U2 - U1 @ (U1.T @ U2), 2))


def test_token_factor_m_side_equals_t_side():
    """T > M route (eigen of X^T X, back-projection, QR) spans the same space as the
    left singular vectors from LAPACK's SVD of the unfolding."""
    rng = np.random.default_rng(8)
    X = _rand_cache(rng, 1, 2, 50, 16) * np.exp(-np.arange(50) / 10)[None, None, :, None]  # M = 32 < T
    U = O.token_factor_exact(X, 6)
    Ul = np.linalg.svd(O.token_unfolding(X), full_matrices=False)[0][:, :6]
    assert _sin_theta(U, Ul) < 1e-8
    assert np.allclose(U.T @ U, np.eye(6), atol=1e-12)


def test_randomized_matches_exact_with_gap():
    rng = np.random.default_rng(9)
    X = _tucker_exact_cache(rng, 2, 2, 64, 16, 6) + 1e-6 * rng.standard_normal((2, 2, 64, 16))
    Ue = O.token_factor_exact(X, 6)
    Ur = O.token_factor_randomized(X, 6, 4, 2, 123, 0, 0)
    assert _sin_theta(Ue, Ur) < 1e-8


def test_sign_convention():
    rng = np.random.default_rng(10)
    X = _rand_cache(rng, 2, 2, 32, 16)
    _, W = O.feature_factor(X)
    piv = np.argmax(np.abs(W), axis=0)
    assert np.all(W[piv, np.arange(16)] > 0)


# ------------------------------------------------------------------ quantiser
def test_quant_worked_example(golden_dir):
    g = dict((r.split()[0], r.split()[1:]) for r in _read_golden(golden_dir, "quant_worked_example.txt"))
    b = int(g["b"][0])
    rho = np.arange(16, dtype=np.float64)[None]
    codes, lo, step, rhat, ok = O.quantize(rho, b)
    assert lo[0] == float(g["lo"][0]) and step[0] == float(g["step"][0])
    assert list(codes.ravel()) == [int(c) for c in g["codes"]]
    assert O.quant_error(rho, b) == float(g["sqerr"][0])
    assert list(O.pack_codes(codes, b).ravel()) == [int(c) for c in g["packed"]]


def test_quant_ties_to_even():
    rho = np.array([[0.0, 0.5, 1.5, 2.5, 3.0] + [1.0] * 11])
    codes, lo, step, _, _ = O.quantize(rho, 2)
    assert lo[0] == 0.0 and step[0] == 1.0
    assert list(codes.ravel()[:5]) == [0, 0, 2, 2, 3]


@pytest.mark.parametrize("b", [1, 2, 3, 4, 8])
def test_quant_nearest_level_brute_force(b):
    rng = np.random.default_rng(b)
    rho = rng.standard_normal((300, 32)) * rng.uniform(0.01, 5, (300, 1))
    codes, lo, step, rhat, ok = O.quantize(rho, b)
    assert ok.all()
    x = rho.reshape(300, 2, 16)
    levels = lo[..., None] + np.arange(1 << b)[None, None, :] * step[..., None]   # (300,2,L)
    assert np.all(levels[..., 0] <= x.min(-1)) and np.all(levels[..., -1] >= x.max(-1))
    d = np.abs(x[..., :, None] - levels[..., None, :])                             # (300,2,16,L)
    best = d.min(-1, keepdims=True)
    cand = d == best
    c = codes
    # the code is a nearest level; where two are nearest, it is the even one
    assert np.all(np.take_along_axis(cand, c[..., None], -1))
    two = cand.sum(-1) == 2
    assert np.all(c[two] % 2 == 0)
    assert np.allclose(rhat.reshape(x.shape), np.take_along_axis(levels, c, -1), rtol=0, atol=0)


def test_quant_constant_and_overflow_blocks():
    rho = np.full((1, 16), 0.25)
    codes, lo, step, rhat, ok = O.quantize(rho, 3)
    assert step[0] == 0 and np.all(codes == 0) and np.all(rhat == 0.25)
    big = np.linspace(-1e5, 1e5, 16)[None]
    assert O.quant_error(big, 4) == math.inf
    assert O.quant_error(big, 0) == float(np.sum(big * big))


@pytest.mark.parametrize("b", [1, 2, 3, 4, 5, 8])
def test_pack_bit_layout(b):
    rng = np.random.default_rng(b + 100)
    codes = rng.integers(0, 1 << b, size=(7, 3, 16))
    packed = O.pack_codes(codes, b)
    assert packed.shape == (7, 3 * 2 * b)
    for r in range(7):
        for blk in range(3):
            bits = 0
            for j in range(16):
                bits |= int(codes[r, blk, j]) << (j * b)
            want = bits.to_bytes(2 * b, "little")
            assert bytes(packed[r, blk * 2 * b:(blk + 1) * 2 * b]) == want
    assert np.array_equal(O.unpack_codes(packed, b), codes)


def test_payload_bytes_count_the_arrays():
    T, D, S = 64, 16, 4
    for rT, rD, b in [(4, 4, 0), (8, 16, 3), (32, 8, 8), (5, 3, 1)]:
        n = O.pad16(T * rT * 2) + O.pad16(D * rD * 2) + O.pad16(S * rT * rD * 2)
        if b:
            codes = np.zeros((S * T, D // 16, 16), dtype=np.int64)
            n += O.pad16(O.pack_codes(codes, b).nbytes) + O.pad16(np.zeros((S * T, D // 16), np.float16).nbytes * 2)
        assert O.unit_payload_bytes(T, D, S, rT, rD, b) == n


# ------------------------------------------------------------------ allocation
def _exhaustive(Dt, Bt, budget):
    best = None
    for combo in itertools.product(*[range(Dt.shape[1])] * Dt.shape[0]):
        B = sum(Bt[u, c] for u, c in enumerate(combo))
        if B <= budget:
            Dsum = sum(Dt[u, c] for u, c in enumerate(combo))
            if best is None or Dsum < best[0]:
                best = (Dsum, combo)
    return best


@pytest.mark.parametrize("seed", range(12))
def test_allocation_against_exhaustive(seed):
    rng = np.random.default_rng(seed)
    nu = int(rng.integers(2, 4))
    nc = int(rng.integers(3, 9))
    Bt = rng.integers(10, 200, size=(nu, nc)).astype(np.int64)
    Dt = 1000.0 / Bt * rng.uniform(0.5, 2.0, size=(nu, nc))
    budget = int(Bt.min(1).sum() + rng.integers(0, int(Bt.max(1).sum() - Bt.min(1).sum()) + 1))
    al = O.allocate(Dt, Bt, budget)
    assert al.status == "ok"
    assert al.bytes <= budget                         # never over budget
    # Everett: the Lagrangian answer is optimal for the budget equal to its own bytes
    opt = _exhaustive(Dt, Bt, al.bytes)
    got = sum(Dt[u, c] for u, c in enumerate(al.choice))
    assert got <= opt[0] + 1e-9 * abs(opt[0])
    # and never better than the true constrained optimum at the given budget
    assert got >= _exhaustive(Dt, Bt, budget)[0] - 1e-9 * abs(got)


def test_allocation_special_cases():
    Bt = np.array([[10, 20, 30], [15, 25, 35]], dtype=np.int64)
    Dt = np.array([[3.0, 2.0, 1.0], [6.0, 4.0, 2.0]])
    al = O.allocate(Dt, Bt, 1000)
    assert al.lam == 0.0 and list(al.choice) == [2, 2]
    assert O.allocate(Dt, Bt, 24).status == "infeasible"
    al = O.allocate(Dt, Bt, 25)
    assert list(al.choice) == [0, 0] and al.bytes == 25


# ------------------------------------------------------------------ whole method
@pytest.mark.parametrize("method", ["exact", "randomized"])
def test_round_trip_equals_table_entry(method):
    from kv_cache_compression_group_b200 import synth
    w = synth.WORKLOADS["tiny"]
    K, V = (synth.to_f64(t) for t in synth.make_cache(w, 0))
    opts = O.Options((4, 8, 16, 32), (4, 8, 16), (0, 2, 3, 4), method=method)
    budget = w.bf16_bytes() // 2
    res = O.compress(K, V, 2, opts, budget, 0)
    assert res.status == "ok" and res.total_bytes <= budget
    Kh, Vh = O.decompress(res)
    for rec in res.units:
        X = K if rec.kv == 0 else V
        Xh = Kh if rec.kv == 0 else Vh
        sl = slice(rec.group * 2, rec.group * 2 + 2)
        e = np.sum((X[sl] - Xh[sl]) ** 2)
        assert abs(e - rec.distortion) <= 1e-12 * np.sum(X[sl] ** 2)


# ------------------------------------------------------------------ stored format
# The stored core, the rotated reconstruction operator and the decoder are pinned against
# hand-worked examples, exact column selections and the textbook Tucker forms above
# (tucker_core / tucker_reconstruct, themselves pinned by the closed forms of this file),
# never against themselves.  Each check is also run on a copy of the oracle function with
# one plausible mistake planted, and must reject it.
import oracle.jolt_ref as JR

_U8 = 2.0 ** -8     # unit roundoff of bf16 (8 significant bits)


def _golden_map(golden_dir, name):
    return dict((r.split()[0], [float(v) for v in r.split()[1:]]) for r in _read_golden(golden_dir, name))


def _core_worked_example(stored_core_fn, golden_dir):
    g = _golden_map(golden_dir, "stored_core_worked_example.txt")
    t = int(g["t"][0])
    X = np.tile(np.array(g["x_row"]), (t, 1))[None, None]        # (1, 1, T, 2)
    W_s = np.ones((2, 1))
    U_s = np.ones((t, 1))
    return float(stored_core_fn(X, U_s, W_s)[0, 0, 0, 0]), g


def test_stored_core_worked_example(golden_dir):
    got, g = _core_worked_example(O.stored_core, golden_dir)
    assert got == g["core"][0]
    # the unrounded Tucker core of the same slice is the textbook value
    X = np.tile(np.array(g["x_row"]), (int(g["t"][0]), 1))[None, None]
    assert float(O.tucker_core(X, np.ones((X.shape[2], 1)), np.ones((2, 1)))[0, 0, 0, 0]) == g["core_unrounded"][0]


def _core_by_selection(stored_core_fn):
    """U_s, W_s that pick rows / columns (exact in bf16): the core of a bf16-exact slice is
    then the selected sub-block, C[l,h][r, q] = X[l,h][rows[r], cols[q]], with no rounding.
    Returns the largest deviation."""
    rng = np.random.default_rng(21)
    Lg, H, T, D = 2, 3, 12, 16
    X = O.bf16_rn(rng.standard_normal((Lg, H, T, D)))
    rows = np.array([7, 2, 11, 0])
    cols = np.array([5, 14, 3, 9])
    U_s = np.zeros((T, 4))
    U_s[rows, np.arange(4)] = 1.0
    W_s = np.zeros((D, 4))
    W_s[cols, np.arange(4)] = 1.0
    want = X[:, :, rows][:, :, :, cols]
    got = stored_core_fn(X, U_s, W_s)
    if got.shape != want.shape:
        return math.inf
    return float(np.max(np.abs(got - want)))


def test_stored_core_selects_the_sub_block():
    assert _core_by_selection(O.stored_core) == 0.0


def _core_vs_tucker(stored_core_fn):
    """stored_core against the unrounded Tucker core U_s^T X W_s: two bf16 roundings, so
    |C_s - C| <= u (|U_s|^T |X W_s|) (1 + u) + u |C| (1 + u)^2 entry by entry.  Returns the
    largest ratio of the deviation to that bound."""
    rng = np.random.default_rng(22)
    X = O.bf16_rn(_rand_cache(rng, 2, 2, 40, 16) * 3.0)
    _, W = O.feature_factor(X)
    U = O.token_factor_exact(X, 10)
    U_s, W_s = O.bf16_rn(U), O.bf16_rn(W[:, :6])
    C = O.tucker_core(X, U_s, W_s)
    Cs = stored_core_fn(X, U_s, W_s)
    if Cs.shape != C.shape:
        return math.inf
    Z = np.abs(np.einsum("lhtd,dq->lhtq", X, W_s))
    bound = _U8 * np.einsum("tr,lhtq->lhrq", np.abs(U_s), Z) * (1 + _U8) + _U8 * np.abs(C) * (1 + _U8) ** 2
    return float(np.max(np.abs(Cs - C) / (bound + 1e-300)))


def test_stored_core_within_two_bf16_roundings_of_tucker_core():
    assert _core_vs_tucker(O.stored_core) <= 1.0


def test_recon_operator_worked_example(golden_dir):
    g = _golden_map(golden_dir, "recon_operator_worked_example.txt")
    P = O.recon_operator(np.ones((1, 1, 1, 1)), np.ones((2, 1)), np.array(g["sigma"]), 1)
    assert list(P.ravel()) == g["p_rot"]


def _decode_vs_tucker(monkeypatch=None):
    """At b = 0 the decoder over the stored bytes is the Tucker reconstruction of the stored
    factors, U_s C_s W_s^T, up to the bf16 rounding of P' (Phi is orthogonal):
    ||decode - U_s C_s W_s^T||_F <= ||U_s||_2 u ||C_s W_s^T||_F per slice.  Returns the
    largest ratio of the deviation to that bound over several (r_T, r_D)."""
    from kv_cache_compression_group_b200 import synth
    w = synth.WORKLOADS["tiny"]
    K, V = (synth.to_f64(t) for t in synth.make_cache(w, 3))
    X = K[:2]
    opts = O.Options((4, 8, 16, 32), (4, 8, 16), (0, 2), method="exact")
    f = O.unit_factors(X, 0, 0, opts, 5)
    worst = 0.0
    for rT in (4, 16, 32):
        for rD in (4, 8, 16):
            c = opts.token_ranks.index(rT) * len(opts.feature_ranks) * len(opts.bits) \
                + opts.feature_ranks.index(rD) * len(opts.bits)        # b = 0
            rec = O.encode_unit(X, f, opts, c, 0.0)
            assert rec.b == 0 and rec.r_T == rT and rec.r_D == rD
            got = O.decode_unit(rec)
            want = O.tucker_reconstruct(f.U_s[:, :rT], f.C_s[:, :, :rT, :rD], f.W_s[:, :rD])
            P = np.einsum("lhrq,dq->lhrd", f.C_s[:, :, :rT, :rD], f.W_s[:, :rD])
            nU = np.linalg.norm(f.U_s[:, :rT], 2)
            for l in range(X.shape[0]):
                for h in range(X.shape[1]):
                    dev = np.linalg.norm(got[l, h] - want[l, h])
                    bound = nU * _U8 * np.linalg.norm(P[l, h]) * (1 + 1e-12) + 1e-300
                    worst = max(worst, dev / bound)
    return worst


def test_decode_b0_is_tucker_reconstruction_of_stored_factors():
    assert _decode_vs_tucker() <= 1.0


def test_full_rank_unrounded_table_entry_is_zero(monkeypatch):
    """With r_T = T, r_D = D and every storage rounding replaced by the identity, the
    stored-format pipeline (core, rotated operator, rotated residual) reconstructs X
    exactly: the b = 0 table entry is ||rho||^2 = 0 (full-rank Tucker is exact)."""
    monkeypatch.setattr(JR, "bf16_rn", lambda x: np.asarray(x, dtype=np.float64))
    rng = np.random.default_rng(23)
    X = _rand_cache(rng, 2, 2, 24, 16)          # T = 24 <= M = 64
    _, W = O.feature_factor(X)
    U = O.token_factor_exact(X, 24)
    C_s = O.stored_core(X, U, W)
    sigma = O.rotation_signs(1, 0, 0, 16)
    opts = O.Options((8, 24), (4, 16), (0, 3))
    tab = O.distortion_table(X, U, W, C_s, sigma, opts)
    assert tab[1, 1, 0] <= 1e-12 * np.sum(X * X)
    assert tab[0, 0, 0] > 1e-3 * np.sum(X * X)          # a truncated choice is not exact


# --- planted mistakes: each must be caught by one of the pins above --------------------
def _core_transposed(X, U_s, W_s):
    Z = O.bf16_rn(np.einsum("lhtd,dq->lhtq", X, W_s))
    return O.bf16_rn(np.einsum("tr,lhtq->lhqr", U_s, Z))


def _core_unrounded_z(X, U_s, W_s):
    Z = np.einsum("lhtd,dq->lhtq", X, W_s)
    return O.bf16_rn(np.einsum("tr,lhtq->lhrq", U_s, Z))


def _core_token_side_first(X, U_s, W_s):
    Y = O.bf16_rn(np.einsum("tr,lhtd->lhrd", U_s, X))
    return O.bf16_rn(np.einsum("lhrd,dq->lhrq", Y, W_s))


def _recon_phi_transposed(C_s, W_s, sigma, r_D):
    P = np.einsum("lhrq,dq->lhrd", C_s[..., :r_D], W_s[:, :r_D])
    return O.bf16_rn(O.fwht(P) / math.sqrt(P.shape[-1]) * sigma)


def _recon_unrotated(C_s, W_s, sigma, r_D):
    return O.bf16_rn(np.einsum("lhrq,dq->lhrd", C_s[..., :r_D], W_s[:, :r_D]))


def test_planted_core_mistakes_are_caught(golden_dir):
    assert _core_by_selection(_core_transposed) > 0          # transposed core einsum
    got, g = _core_worked_example(_core_unrounded_z, golden_dir)
    assert got == g["core_without_z_rounding"][0] != g["core"][0]   # Z left unrounded
    got, _ = _core_worked_example(_core_token_side_first, golden_dir)
    assert got != g["core"][0]                                      # rounded on the token side first


def test_planted_operator_mistakes_are_caught(golden_dir, monkeypatch):
    g = _golden_map(golden_dir, "recon_operator_worked_example.txt")
    P = _recon_phi_transposed(np.ones((1, 1, 1, 1)), np.ones((2, 1)), np.array(g["sigma"]), 1)
    assert list(P.ravel()) == g["p_rot_transposed"] != g["p_rot"]
    for mutant in (_recon_phi_transposed, _recon_unrotated):
        with monkeypatch.context() as m:
            m.setattr(JR, "recon_operator", mutant)
            assert _decode_vs_tucker() > 100.0
