"""The library at the full workload sizes, in the launch configuration the benchmark times.

At these sizes the float64 checker cannot redo whole compress calls, so every case checks
  * properties that hold at any size: the byte budget is never exceeded; every unit's
    measured round-trip error equals the distortion-table entry it was chosen by (table,
    encoder and decoder agree); decompression is deterministic in its dtype;
  * sampled outputs the checker computes one by one: for two sampled units the library's
    rotated reconstruction operator (from the stored core and feature factor) against the
    checker's; then, for a range of token rows of every slice, the checker's decoder
    formula over the stored bytes against the library's decompression, and the checker's
    quantiser on the residual of those rows against the stored scales and codes (both on
    the library's bf16 operator, as in the small-size tests);
  * on the Mistral-shaped cache (cheap enough for the checker's own factor step) the
    token and feature factors of the sampled units against the checker's, with the same
    randomized sketch, as in the small-size parity tests.
Tolerances are the ones of the small-size parity tests.
"""
import numpy as np
import pytest
import torch

import oracle as O
from kv_cache_compression_group_b200 import jolt as J
from kv_cache_compression_group_b200 import synth
from blob_helpers import add_counts, as_record, assert_code_counts, blob_unit, check_codes

pytestmark = pytest.mark.gpu

FULL = [
    ("mistral7b", "randomized", (2.0, 3.0)),
    ("mistral7b", "exact", (2.0,)),
    ("llama2_13b", "randomized", (2.0, 3.0, 4.0)),
    ("llama31_8b_64k", "randomized", (2.0, 3.0, 4.0, 5.0)),
    # the compression-time sweep on the Mistral-shaped generator
    ("sweep_T512", "exact", (2.0,)), ("sweep_T512", "randomized", (3.0,)),
    ("sweep_T2048", "exact", (3.0,)), ("sweep_T2048", "randomized", (2.0,)),
    ("sweep_T8192", "randomized", (2.0, 3.0)), ("sweep_T32768", "randomized", (2.0,)),
]


def _workload(name):
    if name.startswith("sweep_T"):
        return synth.sweep_workload(int(name[len("sweep_T"):]))
    return synth.WORKLOADS[name]
SEED = 0
ROWS = 64  # token rows of every slice checked per sampled unit


def _unit_x(K, V, w, u, rows=None):
    """Unit u of the CPU caches in float64 (only token rows [t0, t1) if given)."""
    g, kv = u // 2, u % 2
    src = (K if kv == 0 else V)[g * w.layers_per_group:(g + 1) * w.layers_per_group]
    if rows is not None:
        src = src[:, :, rows[0]:rows[1]]
    return synth.to_f64(src.contiguous())


def _library_operator(comp, opts, w, u, g_full):
    """The library's rotated reconstruction operator P' of unit u for its stored (r_T, r_D),
    computed by the library from the stored core and feature factor (S x r_T x D, float64)."""
    S, D = w.layers_per_group * w.n_heads, w.D
    rT, rD = g_full["C"].shape[1], g_full["C"].shape[2]
    core = torch.zeros((comp.n_units, S, max(opts.token_ranks), max(opts.feature_ranks)), dtype=torch.bfloat16)
    Wf = torch.zeros((comp.n_units, D, max(opts.feature_ranks)), dtype=torch.bfloat16)
    core[u, :, :rT, :rD] = torch.from_numpy(g_full["C"]).to(torch.bfloat16)
    Wf[u, :, :rD] = torch.from_numpy(g_full["W"]).to(torch.bfloat16)
    P = comp.recon_operator(core.cuda(), Wf.cuda(), SEED)
    return P[opts.feature_ranks.index(rD), u, :, :rT, :].double().cpu().numpy()


def _sampled_rows_check(blob_np, rec, w, u, K, V, comp, opts):
    """Decode and re-encode token rows [t0, t0 + ROWS) of every slice with the checker, on
    the library's own bf16 operator P' (whose agreement with the checker's is checked too)."""
    g, kv = u // 2, u % 2
    t0 = (w.T - ROWS) if u % 4 == 3 else (u * 37) % (w.T - ROWS + 1)
    gb = blob_unit(blob_np, rec, w, rows=(t0, t0 + ROWS))
    r = as_record(gb, w, rec, g, kv, SEED)
    Pl = _library_operator(comp, opts, w, u, gb)
    Po = O.recon_operator(r.C_s, r.W_s, r.sigma, r.r_D).reshape(Pl.shape)
    diff = Pl != Po
    assert diff.mean() <= 1e-6, diff.mean()   # fp64 operator, one rounding: equal but for fp64 ties
    step = np.abs(Po) * 2.0 ** -7 * 1.0001 + 2.0 ** -16 * np.abs(Po).max(-1, keepdims=True)
    assert np.all(np.abs(Pl - Po)[diff] <= step[diff])
    Xrows = _unit_x(K, V, w, u, (t0, t0 + ROWS))
    xr = O.rotated_input(Xrows, r.sigma)
    Pg = Pl.reshape(w.layers_per_group, w.n_heads, r.r_T, w.D)
    recon = np.einsum("tr,lhrd->lhtd", r.U_s, Pg, optimize=True)
    rho = xr - recon
    rho_o = xr - np.einsum("tr,lhrd->lhtd", r.U_s, Po.reshape(Pg.shape), optimize=True)
    counts = check_codes(gb, rho, xr, r.b, rho_oracle=rho_o) if r.b else {}
    # the checker's decoder formula over the stored bytes and the library's operator
    rhat = (r.lo[..., None] + r.codes * r.step[..., None]).reshape(recon.shape) if r.b else 0.0
    Xo = O.unrotate(recon + rhat, r.sigma)
    return t0, Xrows, Xo, counts


@pytest.mark.parametrize("name,method,ratios", FULL)
def test_full_size(name, method, ratios):
    w = _workload(name)
    K, V = synth.make_cache(w, SEED)
    Kd, Vd = K.cuda(), V.cuda()
    opts = J.default_options(w.T, w.D, method)
    comp = J.Compressor(w.n_layers, w.n_heads, w.T, w.D, w.layers_per_group, K.dtype, opts)
    nu = comp.n_units
    sample = (0, nu - 1)
    acc = {}
    for ratio in ratios:
        budget = int(w.bf16_bytes() / ratio)
        blob = comp.compress(Kd, Vd, budget, SEED)
        _, total, recs = J.read_header(blob)
        assert total <= budget
        Kh, Vh = comp.decompress(blob, torch.float32)
        sq = J.frobenius(Kd, Vd, Kh, Vh, w.layers_per_group).cpu().numpy()
        for u, r in enumerate(recs):
            assert abs(sq[u, 1] - r["distortion"]) <= 1e-5 * max(sq[u, 1], 1e-30) + 1e-9 * sq[u, 0], (u, ratio)
        Kb, _ = comp.decompress(blob, torch.bfloat16)
        assert torch.equal(Kb, Kh.to(torch.bfloat16))
        del Kb
        blob_np = blob[:total].cpu().numpy()
        for u in sample:
            t0, X, Xo, counts = _sampled_rows_check(blob_np, recs[u], w, u, K, V, comp, opts)
            add_counts(acc, counts)
            g, kv = u // 2, u % 2
            Xl = (Kh if kv == 0 else Vh)[g * w.layers_per_group:(g + 1) * w.layers_per_group, :, t0:t0 + ROWS]
            Xl = Xl.double().cpu().numpy()
            # fp32 decoder against the float64 one over the same stored bytes
            assert np.abs(Xl - Xo).max() <= 2.0 ** -18 * (np.abs(Xo).max() + np.abs(X).max()), (u, ratio)
        del Kh, Vh
    assert_code_counts(acc, f"{name} {method}")


def test_full_size_factors_mistral():
    """Token and feature factors of sampled units of the full Mistral-shaped cache against
    the checker's (same seed, so the same Gaussian sketch for FlashJoLT)."""
    w = synth.WORKLOADS["mistral7b"]
    K, V = synth.make_cache(w, SEED)
    Kd, Vd = K.cuda(), V.cuda()
    for method in ("randomized", "exact"):
        opts = J.default_options(w.T, w.D, method)
        oo = O.Options(opts.token_ranks, opts.feature_ranks, opts.bits, method)
        comp = J.Compressor(w.n_layers, w.n_heads, w.T, w.D, w.layers_per_group, K.dtype, opts)
        U, W = comp.factor(Kd, Vd, SEED)
        U, W = U.double().cpu().numpy(), W.double().cpu().numpy()
        checked = 0
        for u in (0, comp.n_units - 1):
            X = _unit_x(K, V, w, u)
            f = O.unit_factors(X, u // 2, u % 2, oo, SEED)
            A = O.token_unfolding(X)
            gt = np.linalg.eigvalsh(A @ A.T)[::-1]
            for r in oo.token_ranks:
                gap = (gt[r - 1] - gt[r]) / gt[0]
                if gap >= 1e-4:
                    s = np.linalg.norm(f.U[:, :r] - U[u][:, :r] @ (U[u][:, :r].T @ f.U[:, :r]), 2)
                    assert s <= 1e-3, (method, u, r, s)
                    checked += 1
            wv = np.sort(f.w_eigvals)[::-1]
            for r in oo.feature_ranks:
                gap = (wv[r - 1] - wv[r]) / wv[0] if r < len(wv) else 1.0
                if gap >= 1e-4:
                    s = np.linalg.norm(f.W[:, :r] - W[u][:, :r] @ (W[u][:, :r].T @ f.W[:, :r]), 2)
                    assert s <= 1e-3, (method, u, r, s)
                    checked += 1
        print(f"\n[mistral7b {method}] {checked} subspace cuts checked")
        assert checked >= 4, (method, checked)


def test_free_zone_flashjolt_matches_jolt():
    """Budget sweep 2x..5x on the Mistral-shaped cache, JoLT (exact token SVD) against FlashJoLT
    (randomized): the randomized sketch must lose nothing measurable in the free zone ("A JoLT
    for the KV cache ... Joint Rank-bit Allocation", abstract: FlashJoLT matches JoLT at a
    fraction of the compression cost).  Criterion: FlashJoLT's relative Frobenius error of K and
    of V at most 1.05 x JoLT's + 1e-4 at every budget."""
    w = synth.WORKLOADS["mistral7b"]
    K, V = synth.make_cache(w, SEED)
    Kd, Vd = K.cuda(), V.cuda()
    comps = {m: J.Compressor(w.n_layers, w.n_heads, w.T, w.D, w.layers_per_group, K.dtype,
                             J.default_options(w.T, w.D, m)) for m in ("exact", "randomized")}
    for ratio in (2.0, 3.0, 4.0, 5.0):
        budget = int(w.bf16_bytes() / ratio)
        err = {}
        for m, comp in comps.items():
            blob = comp.compress(Kd, Vd, budget, SEED)
            _, total, _ = J.read_header(blob)
            assert total <= budget
            Kh, Vh = comp.decompress(blob, torch.float32)
            err[m] = J.relative_errors(Kd, Vd, Kh, Vh, w.layers_per_group)
        print(f"\n[free zone {ratio:g}x] JoLT K/V {err['exact']}, FlashJoLT K/V {err['randomized']}")
        for kv in (0, 1):
            assert err["randomized"][kv] <= 1.05 * err["exact"][kv] + 1e-4, (ratio, kv, err)
