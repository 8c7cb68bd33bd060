"""Parity of the CUDA library (through the C ABI) with the float64 oracle on the same
seeded inputs.  Tolerances:
  factor subspaces        : largest principal-angle sine <= 1e-3 where the relative eigengap
                            at the cut is >= 1e-4 (elsewhere the subspace is not determined)
  stored core             : <= 5e-2 of entries differ, each by at most one bf16 step plus four
                            flips of a bf16 rounding of Z = bf16(X W) (two rounding points of
                            fp32 vs fp64 sums; entries near cancellation flip)
  reconstruction operator : formed in fp64 and rounded once: equal to the oracle's except at a
                            tie closer than fp64 resolution (<= 1e-6 of entries, one bf16 step)
  distortion table        : 1e-6 relative + 2 sqrt(entry) * 64 u_32 ||X|| (fp32 residual vs fp64)
  block scales            : equal, except where the oracle's block minimum / maximum lies within
                            w = 2^-17 (max|x'| + max|x_hat|) of an fp16 rounding boundary (the
                            fp32 residual's absolute error); then the library's scale must be
                            the rounding of a value inside that window
  codes                   : <= 1e-4 of codes differ from the oracle's own codes (its scales,
                            its operator); under the library's scales every differing code lies
                            within w / step of a rounding tie
  allocation              : bit-exact choices and lambda given identical tables
  end to end              : relative Frobenius error within 1e-4 absolute of the oracle's
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from kv_cache_compression_group_b200 import jolt as J
from kv_cache_compression_group_b200 import synth
from blob_helpers import add_counts, assert_code_counts, blob_unit, check_codes

pytestmark = pytest.mark.gpu

TINY_OPTS = ((4, 8, 16, 32), (4, 8, 16), (0, 2, 3, 4))


def _case(name):
    if name.startswith("tiny"):
        w = synth.WORKLOADS["tiny"]
        rt, rd, bits = TINY_OPTS
        ratio = 2.0
    elif name.startswith("mistral4"):
        w = synth.small_workload("mistral7b", n_layers=4)
        o = J.default_options(w.T, w.D)
        rt, rd, bits = o.token_ranks, o.feature_ranks, o.bits
        ratio = 2.0
    elif name.startswith("mistral8"):
        w = synth.small_workload("mistral7b", n_layers=8, n_heads=4)
        o = J.default_options(w.T, w.D)
        rt, rd, bits = o.token_ranks, o.feature_ranks, o.bits
        ratio = 3.0
    elif name.startswith("mstm"):
        # more tokens than unfolded columns: T = 1024 > M = 4 layers x 1 head x 128 = 512, so the
        # exact token factor takes the M x M Gram route (back-projection + re-orthonormalisation)
        w = synth.small_workload("mistral7b", n_layers=4, n_heads=1)
        o = J.default_options(w.T, w.D)
        rt, rd, bits = o.token_ranks, o.feature_ranks, o.bits
        ratio = 2.0
    method = "randomized" if name.endswith("rand") else "exact"
    return w, J.Options(rt, rd, bits, method), O.Options(rt, rd, bits, method), ratio


CASES = ["tiny-exact", "tiny-rand", "mistral4-exact", "mistral4-rand", "mistral8-rand", "mstm-exact", "mstm-rand"]
_cache = {}


def _setup(name):
    if name in _cache:
        return _cache[name]
    w, jo, oo, ratio = _case(name)
    K, V = synth.make_cache(w, 0)
    Kn, Vn = synth.to_f64(K), synth.to_f64(V)
    budget = int(w.bf16_bytes() / ratio)
    res = O.compress(Kn, Vn, w.layers_per_group, oo, budget, 0)
    comp = J.Compressor(w.n_layers, w.n_heads, w.T, w.D, w.layers_per_group, K.dtype, jo)
    units = list(O.units_of(Kn, Vn, w.layers_per_group))
    d = dict(w=w, jo=jo, oo=oo, K=K.cuda(), V=V.cuda(), Kn=Kn, Vn=Vn, budget=budget, res=res, comp=comp,
             units=units)
    _cache[name] = d
    return d


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).cuda()


def _sin_theta(U1, U2):
    return float(np.linalg.norm(U2 - U1 @ (U1.T @ U2), 2))


def _relgaps(vals, cuts):
    v = np.sort(np.asarray(vals))[::-1]
    out = []
    for r in cuts:
        out.append((v[r - 1] - v[r]) / v[0] if r < len(v) else 1.0)
    return out


@pytest.mark.parametrize("name", CASES)
def test_factor_subspaces(name):
    d = _setup(name)
    U, W = d["comp"].factor(d["K"], d["V"], 0)
    U = U.double().cpu().numpy()
    W = W.double().cpu().numpy()
    checked = n_cuts = 0
    for u, f in enumerate(d["res"].factors):
        X = d["units"][u][2]
        A = O.token_unfolding(X)
        gt = np.linalg.eigvalsh(A @ A.T if A.shape[0] <= A.shape[1] else A.T @ A)
        for r, g in zip(d["oo"].token_ranks, _relgaps(gt, d["oo"].token_ranks)):
            s = _sin_theta(f.U[:, :r], U[u][:, :r])
            n_cuts += 1
            if g >= 1e-4:
                assert s <= 1e-3, (u, r, s, g)
                checked += 1
        for r, g in zip(d["oo"].feature_ranks, _relgaps(f.w_eigvals, d["oo"].feature_ranks)):
            s = _sin_theta(f.W[:, :r], W[u][:, :r])
            n_cuts += 1
            if g >= 1e-4:
                assert s <= 1e-3, (u, r, s, g)
                checked += 1
        assert np.abs(U[u].T @ U[u] - np.eye(U.shape[2])).max() < 1e-4
        assert np.abs(W[u].T @ W[u] - np.eye(W.shape[2])).max() < 1e-4
    # cuts under the eigengap threshold are skipped: at least a quarter of them must be checked
    print(f"\n[{name}] {checked} of {n_cuts} subspace cuts checked")
    assert checked >= max(2, n_cuts // 4), (checked, n_cuts)


def _oracle_factors(d):
    facs = d["res"].factors
    Us = _bf16(np.stack([f.U_s for f in facs]))
    Ws = _bf16(np.stack([f.W_s for f in facs]))
    return facs, Us, Ws


def _ulp_close(got, want, slack):
    """fraction of entries that differ, and whether every difference is within one bf16 step
    of the value plus `slack` (the absolute error the fp32 sums before the rounding may carry)."""
    diff = got != want
    frac = diff.mean()
    step = np.abs(want) * 2.0 ** -7 * 1.0001 + slack
    ok = np.all(np.abs(got - want)[diff] <= np.broadcast_to(step, want.shape)[diff])
    return frac, ok


@pytest.mark.parametrize("name", CASES)
def test_core_table_and_operator(name):
    d = _setup(name)
    facs, Us, Ws = _oracle_factors(d)
    core, tab = d["comp"].table(d["K"], d["V"], Us, Ws, 0)
    core = core.double().cpu().numpy()
    tab = tab.cpu().numpy()
    P = d["comp"].recon_operator(torch.from_numpy(core).to(torch.bfloat16).cuda(), Ws, 0).double().cpu().numpy()
    Lg, H = d["w"].layers_per_group, d["w"].n_heads
    for u, f in enumerate(facs):
        X = d["units"][u][2]
        want = O.stored_core(X, f.U_s, f.W_s).reshape(core[u].shape)
        # two bf16 rounding points (Z = bf16(X W), C = bf16(U^T Z)): fp32 sums flip a rounding
        # of Z now and then (one bf16 step, 2^-8 relative), and a flipped Z entry moves every
        # core sum that uses it by up to 2^-8 max|U| max|Z|; allow four such flips per sum
        Z = O.bf16_rn(np.einsum("lhtd,dq->lhtq", X, f.W_s)).reshape(-1, X.shape[2], f.W_s.shape[1])
        slack = 4 * 2.0 ** -8 * np.abs(f.U_s).max(0)[None, :, None] * np.abs(Z).max(1)[:, None, :]
        frac, ok = _ulp_close(core[u], want, slack)
        # every difference is a rounding flip within the bound; how many entries flip depends
        # on how many sit near cancellation (about 2 % with 4 slices per unit)
        assert frac <= 5e-2 and ok, (u, frac)
        Cg = core[u].reshape(Lg, H, *core[u].shape[1:])
        for iD, rD in enumerate(d["oo"].feature_ranks):
            # the library forms P' in fp64 and rounds once: equal to the oracle's operator
            # except at a tie closer than fp64 resolution
            Pw = O.recon_operator(Cg, f.W_s, f.sigma, rD).reshape(P[iD, u].shape)
            frac, ok = _ulp_close(P[iD, u], Pw, 0.0)
            assert frac <= 1e-6 and ok, (u, rD, frac)
        # the table kernel against the oracle's table built from the same stored core.
        # The library forms rho in fp32: |d rho| <= c u_32 |x| per element, so an entry
        # sum_i e_i^2 moves by at most 2 sqrt(entry) ||d rho|| (+ ties, which move e^2 by
        # the same order); c = 64 covers the accumulation depth of the reconstruction.
        tw = O.distortion_table(X, f.U_s, f.W_s, Cg, f.sigma, d["oo"]).reshape(-1)
        fin = np.isfinite(tw)
        assert np.array_equal(fin, np.isfinite(tab[u]))
        xnorm = float(np.linalg.norm(X))
        tol = 1e-6 * tw[fin] + 2 * np.sqrt(tw[fin]) * 64 * 2.0 ** -24 * xnorm
        assert np.all(np.abs(tab[u][fin] - tw[fin]) <= tol), (u, np.max(np.abs(tab[u][fin] - tw[fin]) / tol))


@pytest.mark.parametrize("seed", range(6))
def test_allocation_bit_exact(seed):
    rng = np.random.default_rng(seed)
    nu = int(rng.integers(2, 21))
    nc = int(rng.integers(8, 97))
    B = rng.integers(1000, 10_000_000, size=(nu, nc)).astype(np.int64)
    D = 1e9 / B * rng.uniform(0.2, 5.0, size=(nu, nc))
    if seed % 2:
        D[rng.random((nu, nc)) < 0.1] = np.inf      # unstorable choices
        D[:, 0] = 1e12                              # fewest-bytes choice always finite
        B[:, 0] = B.min() // 2
    lo, hi = int(B.min(1).sum()), int(B.max(1).sum())
    for budget in (lo, (lo + hi) // 3, (lo + hi) // 2, hi, hi * 2):
        al = O.allocate(D, B, budget)
        ch, lam, st = J.allocate(torch.from_numpy(D).cuda(), torch.from_numpy(B).cuda(), budget)
        assert st.item() == 0
        assert list(ch.cpu().numpy()) == list(al.choice), budget
        assert lam.cpu().numpy()[0].tobytes() == np.float64(al.lam).tobytes(), (lam.item(), al.lam)
    ch, lam, st = J.allocate(torch.from_numpy(D).cuda(), torch.from_numpy(B).cuda(), lo - 1)
    assert st.item() == 4 and math.isinf(lam.item())


def test_allocation_bit_exact_on_oracle_tables():
    for name in ("tiny-exact", "mistral4-exact"):
        d = _setup(name)
        res = d["res"]
        avail = d["budget"] - O.header_bytes(res.table.shape[0])
        for frac in (0.6, 0.8, 1.0, 1.3):
            b = int(avail * frac)
            al = O.allocate(res.table, res.bytes, b)
            ch, lam, st = J.allocate(torch.from_numpy(res.table).cuda(), torch.from_numpy(res.bytes).cuda(), b)
            if al.status == "infeasible":
                assert st.item() == 4
                continue
            assert list(ch.cpu().numpy()) == list(al.choice)
            assert lam.cpu().numpy()[0].tobytes() == np.float64(al.lam).tobytes()


@pytest.mark.parametrize("name", CASES)
def test_encode_codes_and_factors(name):
    d = _setup(name)
    res, w = d["res"], d["w"]
    facs, Us, Ws = _oracle_factors(d)
    core = _bf16(np.stack([f.C_s.reshape(-1, f.C_s.shape[-2], f.C_s.shape[-1]) for f in facs]))
    choice = torch.tensor([r.choice for r in res.units], dtype=torch.int32)
    dist = torch.from_numpy(res.table)
    blob = d["comp"].encode(d["K"], d["V"], Us, Ws, core, choice, dist, 0)
    _, total, recs = J.read_header(blob)
    assert total == res.total_bytes
    P = d["comp"].recon_operator(core, Ws, 0).double().cpu().numpy()
    bnp = blob.cpu().numpy()
    acc = {}
    for u, (rec_o, rec_g) in enumerate(zip(res.units, recs)):
        assert (rec_g["r_T"], rec_g["r_D"], rec_g["bits"]) == (rec_o.r_T, rec_o.r_D, rec_o.b)
        g = blob_unit(bnp, rec_g, w)
        assert np.array_equal(g["U"], rec_o.U_s) and np.array_equal(g["W"], rec_o.W_s)
        assert np.array_equal(g["C"], rec_o.C_s.reshape(g["C"].shape))
        if not rec_o.b:
            continue
        # residual with the library's own reconstruction operator (same bf16 operands on both sides)
        iD = d["oo"].feature_ranks.index(rec_o.r_D)
        X = d["units"][u][2]
        Pg = P[iD, u][:, :rec_o.r_T, :].reshape(w.layers_per_group, w.n_heads, rec_o.r_T, w.D)
        xr = O.rotated_input(X, rec_o.sigma)
        rho = xr - np.einsum("tr,lhrd->lhtd", rec_o.U_s, Pg)
        # strict: the oracle's own codes (its operator, its scales) of the same choice
        rho_o = xr - np.einsum("tr,lhrd->lhtd", rec_o.U_s,
                               O.recon_operator(rec_o.C_s, rec_o.W_s, rec_o.sigma, rec_o.r_D))
        add_counts(acc, check_codes(g, rho, xr, rec_o.b, rho_oracle=rho_o))
        assert np.count_nonzero(g["codes"] != rec_o.codes.reshape(-1, 16)) == \
            np.count_nonzero(g["codes"] != O.quantize(rho_o, rec_o.b)[0].reshape(-1, 16))
    assert_code_counts(acc, name)
    # The library's decompression of this blob against the oracle's decompression of its own
    # compress result, element by element.  Factors, core and choices are the same, so row t
    # of a slice can differ only through (a) the bf16 operator P' (library vs oracle rounding:
    # U_s (P'_lib - P'_o)), (b) the dequantised residual where a code or a scale differs
    # (rho_hat_lib - rho_hat_o), both un-rotated by Phi^T whose entries are +-1/sqrt(D), and
    # (c) fp32 sums in the decoder.  So |X_lib - X_o| <= (|U_s||dP'| + |d rho_hat|) 1 / sqrt(D)
    # + 2^-18 (row magnitudes), entry by entry.
    Kh, Vh = d["comp"].decompress(blob, torch.float32)
    Kh, Vh = Kh.double().cpu().numpy(), Vh.double().cpu().numpy()
    Ko, Vo = O.decompress(res)
    Lg, D = w.layers_per_group, w.D
    n_far = n_all = 0
    for u, (rec_o, rec_g) in enumerate(zip(res.units, recs)):
        sl = slice(rec_o.group * Lg, (rec_o.group + 1) * Lg)
        Xl = (Kh if rec_o.kv == 0 else Vh)[sl]
        Xo = (Ko if rec_o.kv == 0 else Vo)[sl]
        Xn = d["units"][u][2]
        iD = d["oo"].feature_ranks.index(rec_o.r_D)
        Pl = P[iD, u][:, :rec_o.r_T, :].reshape(Lg, w.n_heads, rec_o.r_T, D)
        Po = O.recon_operator(rec_o.C_s, rec_o.W_s, rec_o.sigma, rec_o.r_D)
        spread = np.einsum("tr,lhrd->lht", np.abs(rec_o.U_s), np.abs(Pl - Po))
        if rec_o.b:
            g = blob_unit(bnp, rec_g, w)
            shp = rec_o.codes.shape
            rl = g["lo"].reshape(shp[:-1])[..., None] + g["codes"].reshape(shp) * g["step"].reshape(shp[:-1])[..., None]
            ro = rec_o.lo[..., None] + rec_o.codes * rec_o.step[..., None]
            spread = spread + np.abs(rl - ro).reshape(Xo.shape).sum(-1)
        bound = spread[..., None] / math.sqrt(D) + 2.0 ** -18 * (np.abs(Xo).max(-1, keepdims=True)
                                                                 + np.abs(Xn).max(-1, keepdims=True))
        assert np.all(np.abs(Xl - Xo) <= bound), (u, np.max(np.abs(Xl - Xo) / bound))
        n_far += np.count_nonzero(np.abs(Xl - Xo) > 2.0 ** -18 * (np.abs(Xo).max(-1, keepdims=True)
                                                                   + np.abs(Xn).max(-1, keepdims=True)))
        n_all += Xo.size
    print(f"[{name}] decompress: {n_far / n_all:.2e} of elements differ from the oracle's by more than "
          f"2^-18 of the row magnitude (operator roundings, differing codes)")


@pytest.mark.parametrize("name", CASES)
def test_end_to_end_against_oracle(name):
    d = _setup(name)
    comp, res, w = d["comp"], d["res"], d["w"]
    blob = comp.compress(d["K"], d["V"], d["budget"], 0)
    _, total, recs = J.read_header(blob)
    assert total <= d["budget"]
    assert [(r["r_T"], r["r_D"], r["bits"]) for r in recs] == [(u.r_T, u.r_D, u.b) for u in res.units]
    Kh, Vh = comp.decompress(blob, torch.float32)
    ek, ev = J.relative_errors(d["K"], d["V"], Kh, Vh, w.layers_per_group)
    Ko, Vo = O.decompress(res)
    assert abs(ek - O.relative_error(d["Kn"], Ko)) <= 1e-4
    assert abs(ev - O.relative_error(d["Vn"], Vo)) <= 1e-4
    # round trip: the measured error of every unit is the table entry it was chosen by
    sq = J.frobenius(d["K"], d["V"], Kh, Vh, w.layers_per_group).cpu().numpy()
    for u, r in enumerate(recs):
        assert abs(sq[u, 1] - r["distortion"]) <= 1e-5 * max(sq[u, 1], 1e-30) + 1e-9 * sq[u, 0]
    # bf16 output is the bf16 rounding of the fp32 output
    Kb, Vb = comp.decompress(blob, torch.bfloat16)
    assert torch.equal(Kb, Kh.to(torch.bfloat16)) and torch.equal(Vb, Vh.to(torch.bfloat16))
    # deterministic: a second compress gives the same bytes
    blob2 = comp.compress(d["K"], d["V"], d["budget"], 0)
    assert torch.equal(blob[:total], blob2[:total])


def test_device_side_errors():
    d = _setup("tiny-exact")
    comp, w = d["comp"], d["w"]
    blob = comp.compress(d["K"], d["V"], O.header_bytes(comp.n_units) + 16, 0)
    with pytest.raises(J.JoltError) as e:
        J.read_header(blob)
    assert e.value.name == "BUDGET_INFEASIBLE"
    K = d["K"].clone()
    K[0, 0, 3, 5] = float("nan")
    blob = comp.compress(K, d["V"], d["budget"], 0)
    with pytest.raises(J.JoltError) as e:
        J.read_header(blob)
    assert e.value.name == "NUMERIC"
    with pytest.raises(J.JoltError) as e:
        comp.compress(d["K"], d["V"], d["budget"], 0, blob=torch.empty(100, dtype=torch.uint8, device="cuda"))
    assert e.value.name == "OUTPUT_TOO_SMALL"
    bad = torch.zeros(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(J.JoltError) as e:
        comp.decompress(bad)
    assert e.value.name == "BAD_BLOB"


def test_edge_candidate_sets():
    """Residual-free (bits {0}) and full-rank feature factor (r_D = D) choices."""
    w = synth.WORKLOADS["tiny"]
    K, V = synth.make_cache(w, 1)
    Kn, Vn = synth.to_f64(K), synth.to_f64(V)
    for rt, rd, bits, ratio in (((8, 32), (8, 16), (0,), 1.5), ((32,), (16,), (0, 8), 0.6)):
        jo, oo = J.Options(rt, rd, bits), O.Options(rt, rd, bits)
        budget = int(w.bf16_bytes() / ratio)
        res = O.compress(Kn, Vn, w.layers_per_group, oo, budget, 1)
        comp = J.Compressor(w.n_layers, w.n_heads, w.T, w.D, w.layers_per_group, K.dtype, jo)
        blob = comp.compress(K.cuda(), V.cuda(), budget, 1)
        _, total, recs = J.read_header(blob)
        assert [(r["r_T"], r["r_D"], r["bits"]) for r in recs] == [(u.r_T, u.r_D, u.b) for u in res.units]
        Kh, Vh = comp.decompress(blob, torch.float32)
        ek, ev = J.relative_errors(K.cuda(), V.cuda(), Kh, Vh, w.layers_per_group)
        Ko, Vo = O.decompress(res)
        assert abs(ek - O.relative_error(Kn, Ko)) <= 1e-4 and abs(ev - O.relative_error(Vn, Vo)) <= 1e-4


def test_graph_replay_identical():
    """Repeated compress calls with the same arguments replay a captured CUDA graph (the first
    runs directly, the second is captured, later ones replay): every call gives the bytes of
    a direct call, also after the inputs change in place and for a second budget."""
    d = _setup("mistral4-rand")
    comp, w = d["comp"], d["w"]
    J.set_graphs(False)
    ref = comp.compress(d["K"], d["V"], d["budget"], 0)
    _, total, _ = J.read_header(ref)
    K2 = d["K"].clone()
    K2[0, 0, :7] *= 1.5
    ref2 = comp.compress(K2, d["V"], d["budget"] // 2, 0)
    _, total2, _ = J.read_header(ref2)
    J.set_graphs(True)
    try:
        blob = torch.zeros_like(ref)
        Kbuf = d["K"].clone()
        for i in range(4):
            comp.compress(Kbuf, d["V"], d["budget"], 0, blob=blob)
            assert torch.equal(blob[:total], ref[:total]), i
        n0 = J.launch_count()
        comp.compress(Kbuf, d["V"], d["budget"], 0, blob=blob)
        assert J.launch_count() - n0 > 10      # a replay counts the kernels it runs
        Kbuf.copy_(K2)                          # same buffers, new contents
        blob2 = torch.zeros_like(ref)
        for i in range(3):
            comp.compress(Kbuf, d["V"], d["budget"] // 2, 0, blob=blob2)
            assert torch.equal(blob2[:total2], ref2[:total2]), i
    finally:
        J.set_graphs(True)
