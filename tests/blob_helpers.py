"""Host-side readers of the library's compressed blob for the GPU parity tests: pull one
unit's stored factors, codes and scales out of the bytes (optionally only a range of token
rows of every slice) and wrap them as the float64 checker's unit record."""
import numpy as np
import torch

import oracle as O


def blob_unit(blob_np, rec, w, rows=None, block=16):
    """Stored U, W, C and (for b > 0) codes, lo, step of one unit record.  ``rows`` =
    (t0, t1) restricts U and the residual to those token rows of every slice."""
    S = w.layers_per_group * w.n_heads
    T, D = w.T, w.D
    t0, t1 = rows if rows is not None else (0, T)
    nb_row = D // block

    def bf(off, n):
        return torch.from_numpy(blob_np[off:off + 2 * n].copy()).view(torch.bfloat16).double().numpy()

    Ub = bf(rec["off_U"], T * rec["r_T"]).reshape(T, rec["r_T"])[t0:t1]
    Wb = bf(rec["off_W"], D * rec["r_D"]).reshape(D, rec["r_D"])
    Cb = bf(rec["off_C"], S * rec["r_T"] * rec["r_D"]).reshape(S, rec["r_T"], rec["r_D"])
    out = dict(U=Ub, W=Wb, C=Cb)
    b = rec["bits"]
    if b:
        # block index of (slice s, row t, block j) is (s * T + t) * nb_row + j
        blk = (np.arange(S)[:, None] * T + np.arange(t0, t1)[None, :]).reshape(-1)
        blk = (blk[:, None] * nb_row + np.arange(nb_row)[None, :]).reshape(-1)
        cbytes = 2 * b
        allc = blob_np[rec["off_codes"]:rec["off_codes"] + S * T * nb_row * cbytes].reshape(-1, cbytes)
        out["codes"] = O.unpack_codes(allc[blk], b).reshape(-1, block)
        sc = blob_np[rec["off_scales"]:rec["off_scales"] + S * T * nb_row * 4].reshape(-1, 4)[blk]
        sc = sc.copy().view(np.float16).astype(np.float64).reshape(-1, 2)
        out["lo"], out["step"] = sc[:, 0], sc[:, 1]
    return out


def as_record(g, w, rec, group, kv, seed, block=16):
    """The float64 checker's UnitRecord for the rows held in ``g`` (from blob_unit)."""
    Lg, H, D = w.layers_per_group, w.n_heads, w.D
    rows = g["U"].shape[0]
    b = rec["bits"]
    shp = (Lg, H, rows, D // block)
    if b:
        codes = g["codes"].reshape(shp + (block,))
        lo, step = g["lo"].reshape(shp), g["step"].reshape(shp)
    else:
        codes = np.zeros(shp + (block,), dtype=np.int64)
        lo = step = np.zeros(shp)
    return O.UnitRecord(group, kv, -1, rec["r_T"], rec["r_D"], b, g["U"], g["W"],
                        g["C"].reshape(Lg, H, rec["r_T"], rec["r_D"]), O.rotation_signs(seed, group, kv, D),
                        codes, lo, step, rec["distortion"])


def check_codes(g, rho, xr, b, rho_oracle=None):
    """Scales and codes of the library against the oracle's quantiser on the same rho.

    The library forms rho in fp32 from x' and the reconstruction: its error is absolute,
    bounded per block by w = 2^-17 (max |x'| + max |x_hat|).  A differing scale must be the
    rounding of a block minimum / maximum inside that window; codes are compared under the
    library's own scales and may differ only where the oracle's scaled value lies within
    w / step of a rounding tie.  A
    differing scale is only possible in a block whose window straddles an fp16 rounding
    boundary, and their number is asserted not to exceed the number of such blocks.

    ``rho_oracle`` (the residual on the oracle's own reconstruction operator) adds the strict
    count: codes that differ from the oracle's own codes (its scales, its operator), which is
    the quantity the 1e-4 target bounds.  Returns a dict of counts."""
    codes, lo, step, _, _ = O.quantize(rho, b)
    codes, lo, step = codes.reshape(-1, 16), lo.reshape(-1), step.reshape(-1)
    rb = rho.reshape(-1, 16)
    xr = xr.reshape(-1, 16)
    win = 2.0 ** -17 * (np.abs(xr).max(1) + np.abs(xr - rb).max(1))
    same = (g["lo"] == lo) & (g["step"] == step)
    bad = np.nonzero(~same)[0]
    # blocks whose window straddles an fp16 rounding boundary of lo or of step
    L = (1 << b) - 1
    mn_all, mx_all = rb.min(1), rb.max(1)
    st_lo_all = O.fp16_rd(mn_all - win) != O.fp16_rd(mn_all + win)
    st_st_all = O.fp16_ru(np.maximum(mx_all - win - lo, 0) / L) != O.fp16_ru((mx_all + win - lo) / L)
    n_straddle = int(np.count_nonzero(st_lo_all | st_st_all))
    if bad.size:
        L = (1 << b) - 1
        mn, mx, wb = rb[bad].min(1), rb[bad].max(1), win[bad]
        lo_ok = (g["lo"][bad] >= O.fp16_rd(mn - wb)) & (g["lo"][bad] <= O.fp16_rd(mn + wb))
        st_lo = O.fp16_ru(np.maximum(mx - wb - g["lo"][bad], 0) / L)
        st_hi = O.fp16_ru((mx + wb - g["lo"][bad]) / L)
        st_ok = (g["step"][bad] >= st_lo) & (g["step"][bad] <= st_hi)
        assert np.all(lo_ok & st_ok), bad[~(lo_ok & st_ok)][:5]
    assert bad.size <= n_straddle, (bad.size, n_straddle)
    gl, gs = g["lo"][:, None], g["step"][:, None]
    q = (rb - gl) / np.where(gs > 0, gs, 1.0)
    want = np.where(gs > 0, np.clip(np.rint(q), 0, (1 << b) - 1), 0)
    diff = g["codes"] != want
    if diff.any():
        tie = np.abs(q - np.floor(q) - 0.5)
        tw = (win[:, None] / np.where(gs > 0, gs, 1.0)) + 1e-6
        assert np.all(tie[diff] <= np.broadcast_to(tw, tie.shape)[diff]), tie[diff].max()
    out = dict(scales=lo.size, scale_bad=int(bad.size), codes=want.size, code_bad=int(diff.sum()),
               code_vs_oracle=int(np.count_nonzero(g["codes"] != codes)))
    if rho_oracle is not None:
        oc = O.quantize(rho_oracle, b)[0].reshape(-1, 16)
        out["code_vs_oracle"] = int(np.count_nonzero(g["codes"] != oc))
    return out


def add_counts(acc, c):
    for k, v in c.items():
        acc[k] = acc.get(k, 0) + v
    return acc


def assert_code_counts(acc, label=""):
    """Report both code-mismatch fractions and bound them by the 1e-4 target: the codes the
    library stored against the oracle's own codes (strict), and against the oracle's quantiser
    evaluated under the library's scales."""
    n = acc.get("codes", 0)
    if not n:
        return
    print(f"\n[codes {label}] {n} codes: {acc['code_vs_oracle']} differ from the oracle's own codes "
          f"({acc['code_vs_oracle'] / n:.2e}), {acc['code_bad']} under the library's scales "
          f"({acc['code_bad'] / n:.2e}); {acc['scale_bad']} of {acc['scales']} block scales differ")
    assert acc["code_bad"] <= max(1, 1e-4 * n), acc
    assert acc["code_vs_oracle"] <= max(1, 1e-4 * n), acc
