"""Float64 restatement of the JoLT / FlashJoLT compressor (test infrastructure only).

Sources, cited below by short name:
  [Abstract] "A JoLT for the KV cache: Near-Lossless KV Cache Compression via Joint
             Rank-bit Allocation", abstract (research.draconitic.com).
  [Intro]    "A JoLT for the KV Cache: Near-Lossless KV Cache Compression via Joint
             Tucker and JL-Residual Allocation for LLMs", introduction (catalyzex author page).
  [Blog]     "JoLT: nearly lossless KV cache loss compression for LLMs" (q2bstudio blog).
  [Wiki]     AI-Wiki paper summary, "Key Contributions" and "Methodology".
  [Radio]    AI Radio episode on the paper, "The Core Mechanism".

What the pages fix: per layer group and separately for K and V, a grouped prefill
cache (layers x heads x tokens x features) gets a partial Tucker decomposition on
the token and feature modes only; the truncation residual is rotated by a random
orthogonal (Johnson-Lindenstrauss) rotation and quantised to a few bits; one
Lagrangian dual picks the Tucker ranks and residual bit-widths of every group
under one global byte budget; FlashJoLT replaces the exact token-mode SVD by a
randomized one.  Everything else below is a stated reading: the Gram/eigen factor
route, the random-sign Walsh-Hadamard rotation along the features, 16-wide min-max
blocks with fp16 scales, bf16 factor storage, the byte formula and the bisection rule.

Every step runs in float64 except at the storage rounding points the format
defines (bf16 factors and reconstruction operator, fp16 block scales).  No
blocking, fusion or reordering is done beyond what each definition states.

Parity status (what pins each function, see tests/test_oracle_*.py):
  splitmix64 / gaussian / signs  -- published splitmix64 test vectors; moments.
  bf16_rn / fp16_rd / fp16_ru    -- ml_dtypes round-trip, brute force over neighbours.
  fwht / rotate / unrotate       -- scipy.linalg.hadamard dense product; norm; inverse.
  feature_factor, token_factor_* -- full-rank exactness, energy split, Eckart-Young,
                                    exact Tucker generator, T-side vs M-side route,
                                    randomized == exact when the sketch covers the rank.
  tucker_core / tucker_reconstruct -- full-rank exactness, energy split, Eckart-Young.
  stored_core                    -- hand-worked example of both bf16 roundings; exact
                                    sub-block under row / column selections; within two
                                    bf16 roundings of tucker_core.
  recon_operator / decode_unit   -- hand-worked example of the rotated operator; at b = 0
                                    the decoder equals tucker_reconstruct of the stored
                                    factors within the bf16 rounding of P'; full rank with
                                    roundings removed reconstructs exactly.
  quantize / pack_codes          -- brute-force nearest level on tiny blocks, tie cases,
                                    bit-level unpack, hand-worked block.
  unit_payload_bytes             -- byte count of the actual packed arrays.
  distortion_table / encode_unit -- round trip error equals the table entry; zero at full
                                    rank without roundings.
  allocate                       -- exhaustive enumeration (Everett), budget never exceeded,
                                    lambda = 0 and infeasible special cases.
  compress / decompress          -- round trip error equals the table entry.
  slice_attention_factored       -- equals softmax attention over the decompressed cache
                                    (dense route) for every bit-width and both methods.
Planted mistakes (a transposed core, an unrounded Z, Phi^T for Phi, an unrotated
operator) are each shown to fail one of these pins.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

# ----------------------------------------------------------------------------------------
# Counter-based random numbers: splitmix64 (Steele, Lea & Flood, "Fast splittable
# pseudorandom number generators", OOPSLA 2014).  The rotation signs and the FlashJoLT
# sketch matrix are drawn from it so that any implementation can regenerate them from
# (seed, stream, index) alone.
# ----------------------------------------------------------------------------------------
_MASK = (1 << 64) - 1
GOLDEN_GAMMA = 0x9E3779B97F4A7C15
INDEX_MULT = 0xD1B54A32D192ED03
STREAM_OMEGA = 1
STREAM_SIGN = 2


def splitmix64_mix(z: np.ndarray) -> np.ndarray:
    """splitmix64 output function on a uint64 array: add the golden gamma, then mix."""
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = z + np.uint64(GOLDEN_GAMMA)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
    return z ^ (z >> np.uint64(31))


def stream_id(kind: int, group: int, kv: int) -> int:
    """Stream of one unit: kind in the high word, unit index 2*group+kv in the low word."""
    return (kind << 32) | ((2 * group + kv) & 0xFFFFFFFF)


def hash64(seed: int, stream: int, idx: np.ndarray) -> np.ndarray:
    """h(seed, stream, i) = mix((seed XOR stream*gamma) + i*INDEX_MULT), all mod 2^64."""
    key = (seed ^ ((stream * GOLDEN_GAMMA) & _MASK)) & _MASK
    idx = np.asarray(idx, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(key) + idx * np.uint64(INDEX_MULT)
    return splitmix64_mix(z)


def rotation_signs(seed: int, group: int, kv: int, D: int) -> np.ndarray:
    """sigma_d in {+1,-1}: -1 where the low bit of h(seed, SIGN stream, d) is set."""
    h = hash64(seed, stream_id(STREAM_SIGN, group, kv), np.arange(D, dtype=np.uint64))
    return np.where((h & np.uint64(1)) != 0, -1.0, 1.0)


def gaussian(seed: int, stream: int, idx: np.ndarray) -> np.ndarray:
    """Box-Muller normal deviate for counter ``idx``.

    u1 = ((h(i) >> 11) + 1) 2^-53 in (0, 1],  u2 = (h(i | 2^63) >> 11) 2^-53 in [0, 1),
    z = sqrt(-2 ln u1) cos(2 pi u2), all in float64.
    """
    idx = np.asarray(idx, dtype=np.uint64)
    h1 = hash64(seed, stream, idx)
    h2 = hash64(seed, stream, idx | np.uint64(1 << 63))
    u1 = ((h1 >> np.uint64(11)).astype(np.float64) + 1.0) * 2.0 ** -53
    u2 = (h2 >> np.uint64(11)).astype(np.float64) * 2.0 ** -53
    return np.sqrt(-2.0 * np.log(u1)) * np.cos((2.0 * math.pi) * u2)


def sketch_matrix(seed: int, group: int, kv: int, M: int, k: int) -> np.ndarray:
    """FlashJoLT test matrix Omega (M x k): bf16-rounded Gaussians, entry (m, j) <- counter m*k + j."""
    idx = np.arange(M * k, dtype=np.uint64)
    g = gaussian(seed, stream_id(STREAM_OMEGA, group, kv), idx)
    return bf16_rn(g).reshape(M, k)


# ----------------------------------------------------------------------------------------
# Rounding to the storage formats (bf16: 8 significant bits; fp16: 11 significant bits,
# smallest subnormal 2^-24, largest finite 65504).
# ----------------------------------------------------------------------------------------
def _round_sig(x: np.ndarray, sig_bits: int, min_exp: int, mode: str) -> np.ndarray:
    """Round float64 ``x`` to ``sig_bits`` significant bits with quantum >= 2^min_exp."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                       # x = m 2^e, 0.5 <= |m| < 1
    q = np.ldexp(1.0, np.maximum(e - sig_bits, min_exp))
    y = x / q                                # exact: q is a power of two
    if mode == "rn":
        r = np.rint(y)                       # round half to even
    elif mode == "rd":
        r = np.floor(y)
    elif mode == "ru":
        r = np.ceil(y)
    else:
        raise ValueError(mode)
    out = r * q
    return np.where(x == 0, x, out)


BF16_MAX = float.fromhex("0x1.fep127")
FP16_MAX = 65504.0


def bf16_rn(x):
    """Round to nearest-even bf16 (float64 in, float64 holding bf16 values out)."""
    x = np.asarray(x, dtype=np.float64)
    y = _round_sig(x, 8, -133, "rn")
    return np.where(np.abs(y) > BF16_MAX, np.copysign(np.inf, x), y)


def fp16_rd(x):
    """Round toward -inf to fp16; below -65504 gives -inf, above gives 65504."""
    x = np.asarray(x, dtype=np.float64)
    y = _round_sig(x, 11, -24, "rd")
    y = np.where(y > FP16_MAX, FP16_MAX, y)
    return np.where(y < -FP16_MAX, -np.inf, y)


def fp16_ru(x):
    """Round toward +inf to fp16; above 65504 gives +inf, below -65504 gives -65504."""
    x = np.asarray(x, dtype=np.float64)
    y = _round_sig(x, 11, -24, "ru")
    y = np.where(y < -FP16_MAX, -FP16_MAX, y)
    return np.where(y > FP16_MAX, np.inf, y)


# ----------------------------------------------------------------------------------------
# Options and shapes
# ----------------------------------------------------------------------------------------
@dataclass
class Options:
    """Candidate sets and the token-factor method ([Abstract]: JoLT exact vs FlashJoLT)."""

    token_ranks: tuple
    feature_ranks: tuple
    bits: tuple
    method: str = "exact"           # "exact" (JoLT) or "randomized" (FlashJoLT)
    oversample: int = 10
    power_iters: int = 2
    block: int = 16

    @property
    def n_choices(self) -> int:
        return len(self.token_ranks) * len(self.feature_ranks) * len(self.bits)

    def choice(self, c: int):
        """(i_T, i_D, i_b) of choice index c = (i_T * |R_D| + i_D) * |B| + i_b."""
        nb, nd = len(self.bits), len(self.feature_ranks)
        return c // (nd * nb), (c // nb) % nd, c % nb


GLOBAL_HEADER_BYTES = 64
UNIT_HEADER_BYTES = 64


def pad16(n: int) -> int:
    return (n + 15) // 16 * 16


def unit_payload_bytes(T: int, D: int, S: int, r_T: int, r_D: int, b: int, block: int = 16) -> int:
    """Stored bytes of one unit: U (T x r_T), W (D x r_D), core (S x r_T x r_D) in bf16,
    plus, when b > 0, the packed b-bit codes (block*b/8 bytes per block) and one fp16
    (lo, step) pair per block.  Every array starts on a 16-byte boundary and the padding
    counts against the global byte limit ([Abstract])."""
    n = 2 * T * r_T
    n = pad16(n) + pad16(2 * D * r_D) + pad16(2 * S * r_T * r_D)
    if b > 0:
        nblocks = S * T * (D // block)
        n += pad16(nblocks * block * b // 8) + pad16(nblocks * 4)
    return n


def header_bytes(n_units: int) -> int:
    return GLOBAL_HEADER_BYTES + UNIT_HEADER_BYTES * n_units


# ----------------------------------------------------------------------------------------
# Tensor views: the grouped prefill cache of one unit u = (group g, K or V) is the
# fourth-order tensor X[l, h, t, d] over its L_g layers ([Abstract]: the grouped prefill
# cache is handled as a fourth-order tensor; [Blog], [Intro]: keys and values separately).
# ----------------------------------------------------------------------------------------
def units_of(K: np.ndarray, V: np.ndarray, layers_per_group: int):
    """Yield (g, kv, X_unit[L_g, H, T, D]) in unit order u = 2 g + kv."""
    n_layers = K.shape[0]
    for g in range(n_layers // layers_per_group):
        sl = slice(g * layers_per_group, (g + 1) * layers_per_group)
        yield g, 0, np.asarray(K[sl], dtype=np.float64)
        yield g, 1, np.asarray(V[sl], dtype=np.float64)


def token_unfolding(X: np.ndarray) -> np.ndarray:
    """X_(T): T x (L_g H D), column index (l*H + h)*D + d."""
    Lg, H, T, D = X.shape
    return X.transpose(2, 0, 1, 3).reshape(T, Lg * H * D)


def feature_unfolding(X: np.ndarray) -> np.ndarray:
    """X_(D): (L_g H T) x D, rows in (l, h, t) order."""
    return X.reshape(-1, X.shape[-1])


# ----------------------------------------------------------------------------------------
# Partial Tucker factors on the token and feature modes only ([Abstract], [Intro],
# [Radio] "The Core Mechanism"; head and layer modes are left intact, i.e. their
# factors are the identity).  Reading: truncated HOSVD, each factor = leading
# eigenvectors of its mode-unfolding Gram matrix.
# ----------------------------------------------------------------------------------------
def sort_and_fix_signs(vals: np.ndarray, vecs: np.ndarray):
    """Order eigenpairs by descending eigenvalue (ties: lower original index first) and
    make the entry of largest magnitude in every eigenvector positive (ties: lowest row)."""
    order = np.argsort(-vals, kind="stable")
    vals = vals[order]
    vecs = vecs[:, order].copy()
    piv = np.argmax(np.abs(vecs), axis=0)
    sgn = np.sign(vecs[piv, np.arange(vecs.shape[1])])
    sgn[sgn == 0] = 1.0
    return vals, vecs * sgn


def feature_factor(X: np.ndarray):
    """W: eigenvectors of G_D = X_(D)^T X_(D) (D x D), descending.  Returns (eigvals, W)."""
    A = feature_unfolding(X)
    G = A.T @ A
    vals, vecs = np.linalg.eigh(G)
    return sort_and_fix_signs(vals, vecs)


def qr_positive(Y: np.ndarray) -> np.ndarray:
    """Thin QR factor Q with a positive diagonal in R (the unique one for full column rank)."""
    Q, R = np.linalg.qr(Y)
    d = np.sign(np.diag(R))
    d[d == 0] = 1.0
    return Q * d


def token_factor_exact(X: np.ndarray, r: int) -> np.ndarray:
    """JoLT: leading r left singular vectors of X_(T) (the exact token-mode SVD, [Abstract]).

    T <= M: eigenvectors of G_T = X_(T) X_(T)^T.  T > M: eigenpairs (lam, v) of
    X_(T)^T X_(T), u = X_(T) v / sqrt(lam), then re-orthonormalised by QR."""
    A = token_unfolding(X)
    T, M = A.shape
    if T <= M:
        vals, vecs = np.linalg.eigh(A @ A.T)
        vals, vecs = sort_and_fix_signs(vals, vecs)
        return vecs[:, :r]
    vals, vecs = np.linalg.eigh(A.T @ A)
    vals, vecs = sort_and_fix_signs(vals, vecs)
    if not np.all(vals[:r] > 0):
        raise FloatingPointError("token Gram is rank deficient below the requested rank")
    U = (A @ vecs[:, :r]) / np.sqrt(vals[:r])
    U = qr_positive(U)
    _, U = sort_and_fix_signs(np.arange(r, 0, -1, dtype=np.float64), U)
    return U


def token_factor_randomized(X: np.ndarray, r: int, oversample: int, power_iters: int,
                            seed: int, group: int, kv: int) -> np.ndarray:
    """FlashJoLT: randomized token-mode SVD in place of the exact one ([Abstract]).
    Randomized subspace iteration in the form of
    Halko, Martinsson & Tropp (SIAM Review 2011), Algorithm 4.4: sketch Y = X_(T) Omega,
    orthonormalise after every product, then a Rayleigh-Ritz step (small SVD of
    B = Q^T X_(T) through the eigenvectors of B B^T)."""
    A = token_unfolding(X)
    T, M = A.shape
    k = r + oversample
    if k > min(T, M):
        raise ValueError("sketch width exceeds min(T, M)")
    Omega = sketch_matrix(seed, group, kv, M, k)
    Q = qr_positive(A @ Omega)
    for _ in range(power_iters):
        Qz = qr_positive(A.T @ Q)
        Q = qr_positive(A @ Qz)
    B = Q.T @ A
    vals, vecs = np.linalg.eigh(B @ B.T)
    vals, vecs = sort_and_fix_signs(vals, vecs)
    U = Q @ vecs[:, :r]
    _, U = sort_and_fix_signs(np.arange(r, 0, -1, dtype=np.float64), U)
    return U


def tucker_core(X: np.ndarray, U: np.ndarray, W: np.ndarray) -> np.ndarray:
    """Unrounded core C[l,h] = U^T X[l,h] W (r_T x r_D per slice)."""
    return np.einsum("tr,lhtd,dq->lhrq", U, X, W, optimize=True)


def tucker_reconstruct(U: np.ndarray, C: np.ndarray, W: np.ndarray) -> np.ndarray:
    """U C[l,h] W^T, the Tucker approximation of every slice."""
    return np.einsum("tr,lhrq,dq->lhtd", U, C, W, optimize=True)


# ----------------------------------------------------------------------------------------
# Stored factors (bf16) and the canonical decoder
# ----------------------------------------------------------------------------------------
def stored_core(X: np.ndarray, U_s: np.ndarray, W_s: np.ndarray) -> np.ndarray:
    """Stored core: Z = bf16(X[l,h] W_s), C_s = bf16(U_s^T Z) per slice, [L_g,H,r_T,r_D]."""
    Z = bf16_rn(np.einsum("lhtd,dq->lhtq", X, W_s, optimize=True))
    return bf16_rn(np.einsum("tr,lhtq->lhrq", U_s, Z, optimize=True))


# ----------------------------------------------------------------------------------------
# Johnson-Lindenstrauss rotation of the residual ([Intro], [Blog], [Wiki] "Methodology": a
# random orthogonal rotation is applied before the few-bit quantiser).
# Reading: along the feature axis of every row, rho = r diag(sigma) H_D / sqrt(D) with
# H_D the Sylvester Hadamard matrix and sigma random signs; Phi = diag(sigma) H_D/sqrt(D)
# is orthogonal, so the rotation preserves the residual's energy.
# ----------------------------------------------------------------------------------------
def fwht(x: np.ndarray) -> np.ndarray:
    """Unnormalised Walsh-Hadamard transform (Sylvester / natural order) along the last axis."""
    x = np.array(x, dtype=np.float64, copy=True)
    n = x.shape[-1]
    if n & (n - 1):
        raise ValueError("length must be a power of two")
    lead = x.shape[:-1]
    h = 1
    while h < n:
        y = x.reshape(lead + (n // (2 * h), 2, h))
        a = y[..., 0, :].copy()
        b = y[..., 1, :]
        y[..., 0, :] = a + b
        y[..., 1, :] = a - b
        x = y.reshape(lead + (n,))
        h *= 2
    return x


def rotate(R: np.ndarray, sigma: np.ndarray) -> np.ndarray:
    """rho = R Phi: flip signs, Walsh-Hadamard along features, scale by 1/sqrt(D)."""
    return fwht(R * sigma) / math.sqrt(R.shape[-1])


def unrotate(rho: np.ndarray, sigma: np.ndarray) -> np.ndarray:
    """R = rho Phi^T = sigma * (H rho) / sqrt(D)."""
    return fwht(rho) / math.sqrt(rho.shape[-1]) * sigma


def recon_operator(C_s: np.ndarray, W_s: np.ndarray, sigma: np.ndarray, r_D: int) -> np.ndarray:
    """Rotated reconstruction operator P' = bf16((C_s[..., :r_D] W_s[:, :r_D]^T) Phi).

    Storage reading: the decoder forms the reconstruction U P' in the rotated basis, where
    the residual lives; un-rotating the sum recovers U C W^T + residual.  Rows of P'
    depend only on the same rows of C_s, so a token-rank prefix of P' is the operator of
    the matching core prefix."""
    P = np.einsum("lhrq,dq->lhrd", C_s[..., :r_D], W_s[:, :r_D], optimize=True)
    return bf16_rn(rotate(P, sigma))


# ----------------------------------------------------------------------------------------
# Low-bit residual quantiser ([Abstract]: the truncation residual is stored by a rotated
# few-bit quantiser).  Reading: asymmetric min-max round-to-nearest per block of 16
# consecutive rotated features; lo = fp16 round-down of the block minimum, step =
# fp16 round-up of (max - lo)/(2^b - 1); code = round-half-even((rho - lo)/step).
# ----------------------------------------------------------------------------------------
def quantize(rho: np.ndarray, b: int, block: int = 16):
    """Quantise rows of rho (..., D).  Returns (codes, lo, step, rho_hat, ok).

    codes: (..., D//block, block) int64; lo, step: (..., D//block) float64 holding fp16
    values; ok is False where a scale overflowed fp16 (that block cannot be stored)."""
    shp = rho.shape[:-1] + (rho.shape[-1] // block, block)
    x = rho.reshape(shp)
    if b == 0:
        z = np.zeros(shp[:-1])
        return (np.zeros(shp, dtype=np.int64), z, z, np.zeros_like(rho), np.ones(shp[:-1], bool))
    mn = x.min(axis=-1)
    mx = x.max(axis=-1)
    lo = fp16_rd(mn)
    levels = (1 << b) - 1
    with np.errstate(invalid="ignore", over="ignore"):
        step = np.where(mx > lo, fp16_ru((mx - lo) / levels), 0.0)
        ok = np.isfinite(lo) & np.isfinite(step)
        safe = np.where(ok & (step > 0), step, 1.0)
        q = np.rint((x - lo[..., None]) / safe[..., None])
    codes = np.where((step > 0)[..., None] & ok[..., None], np.clip(q, 0, levels), 0).astype(np.int64)
    lo_s = np.where(ok, lo, 0.0)
    rhat = np.where(ok[..., None], lo_s[..., None] + codes * np.where(ok, step, 0.0)[..., None], 0.0)
    return codes, lo, step, rhat.reshape(rho.shape), ok


def quant_error(rho: np.ndarray, b: int, block: int = 16) -> float:
    """Sum of squared quantisation errors; +inf if any block's scale overflows fp16."""
    if b == 0:
        return float(np.sum(rho * rho))
    _, _, _, rhat, ok = quantize(rho, b, block)
    if not np.all(ok):
        return math.inf
    e = rho - rhat
    return float(np.sum(e * e))


def pack_codes(codes: np.ndarray, b: int) -> np.ndarray:
    """Pack b-bit codes: code j of a block occupies bits [j b, (j+1) b) of the block's
    little-endian bit string (block*b/8 bytes per block).  Returns uint8 (..., nblk*block*b/8)."""
    shp = codes.shape
    blk = shp[-1]
    flat = codes.reshape(-1, blk).astype(np.uint64)
    nbytes = blk * b // 8
    out = np.zeros((flat.shape[0], nbytes), dtype=np.uint8)
    for j in range(blk):
        for bit in range(b):
            pos = j * b + bit
            v = ((flat[:, j] >> np.uint64(bit)) & np.uint64(1)).astype(np.uint8)
            out[:, pos // 8] |= (v << np.uint8(pos % 8)).astype(np.uint8)
    return out.reshape(shp[:-2] + (shp[-2] * nbytes,))


def unpack_codes(packed: np.ndarray, b: int, block: int = 16) -> np.ndarray:
    """Inverse of pack_codes."""
    nbytes = block * b // 8
    flat = packed.reshape(-1, nbytes)
    out = np.zeros((flat.shape[0], block), dtype=np.int64)
    for j in range(block):
        for bit in range(b):
            pos = j * b + bit
            out[:, j] |= ((flat[:, pos // 8] >> (pos % 8)) & 1).astype(np.int64) << bit
    return out.reshape(packed.shape[:-1] + (packed.shape[-1] // nbytes, block))


# ----------------------------------------------------------------------------------------
# Distortion table and the single Lagrangian dual ([Abstract]: one dual sets the Tucker
# ranks and residual bit-widths of every group under a single global byte limit; [Intro]:
# per layer group, keys and values separately, one budget; [Radio] "The Core Mechanism":
# bytes can move between the K and V sides).
# ----------------------------------------------------------------------------------------
def rotated_input(X: np.ndarray, sigma: np.ndarray) -> np.ndarray:
    return rotate(X, sigma)


def distortion_table(X: np.ndarray, U_s: np.ndarray, W_s: np.ndarray, C_s: np.ndarray,
                     sigma: np.ndarray, opts: Options) -> np.ndarray:
    """D[i_T, i_D, i_b] = || rho - Q_b(rho) ||^2 with rho = X Phi - U_s[:, :r_T] P'(r_D)[:r_T].

    Because Phi is orthogonal this is exactly || X - decode(encode(X)) ||^2 for that choice."""
    Xr = rotated_input(X, sigma)
    out = np.zeros((len(opts.token_ranks), len(opts.feature_ranks), len(opts.bits)))
    for iD, rD in enumerate(opts.feature_ranks):
        P = recon_operator(C_s, W_s, sigma, rD)
        for iT, rT in enumerate(opts.token_ranks):
            Xhat = np.einsum("tr,lhrd->lhtd", U_s[:, :rT], P[:, :, :rT, :], optimize=True)
            rho = Xr - Xhat
            for ib, b in enumerate(opts.bits):
                out[iT, iD, ib] = quant_error(rho, b, opts.block)
    return out


def bytes_table(T: int, D: int, S: int, opts: Options) -> np.ndarray:
    out = np.zeros((len(opts.token_ranks), len(opts.feature_ranks), len(opts.bits)), dtype=np.int64)
    for iT, rT in enumerate(opts.token_ranks):
        for iD, rD in enumerate(opts.feature_ranks):
            for ib, b in enumerate(opts.bits):
                out[iT, iD, ib] = unit_payload_bytes(T, D, S, rT, rD, b, opts.block)
    return out


BISECT_STEPS = 200
MAX_DOUBLINGS = 2100


def lagrangian_choice(Dtab: np.ndarray, Btab: np.ndarray, lam: float) -> np.ndarray:
    """Per unit: argmin_c D[c] + lam * B[c] (two separate roundings, no fused multiply-add),
    ties to fewer bytes, then to the lower choice index."""
    n_units, n_ch = Dtab.shape
    out = np.zeros(n_units, dtype=np.int64)
    for u in range(n_units):
        best = None
        for c in range(n_ch):
            with np.errstate(invalid="ignore", over="ignore"):
                v = float(np.float64(Dtab[u, c]) + np.float64(np.float64(lam) * np.float64(Btab[u, c])))
            key = (v, int(Btab[u, c]), c)
            if best is None or key < best:
                best = key
        out[u] = best[2]
    return out


def total_bytes(Btab: np.ndarray, choice: np.ndarray) -> int:
    return int(sum(int(Btab[u, c]) for u, c in enumerate(choice)))


@dataclass
class Allocation:
    status: str                 # "ok" or "infeasible"
    choice: np.ndarray
    lam: float
    bytes: int


def allocate(Dtab: np.ndarray, Btab: np.ndarray, budget: int) -> Allocation:
    """Bisection on lambda for the single Lagrangian dual.

    F(lam) = sum_u B_u(c_u(lam)).  Infeasible if every unit at its fewest-bytes choice
    still exceeds the budget.  lam = 0 if the distortion-minimising choices fit.
    Otherwise lo = 0, hi = 1 doubled until F(hi) <= budget, then exactly 200 halvings of
    [lo, hi] (mid = lo + (hi - lo)/2; F(mid) <= budget -> hi = mid, else lo = mid); the
    answer is c(hi).  No greedy refill of leftover bytes."""
    Dtab = np.asarray(Dtab, dtype=np.float64)
    Btab = np.asarray(Btab, dtype=np.int64)
    minB = sum(int(Btab[u].min()) for u in range(Btab.shape[0]))
    if minB > budget:
        return Allocation("infeasible", np.zeros(Btab.shape[0], dtype=np.int64), math.inf, minB)
    c0 = lagrangian_choice(Dtab, Btab, 0.0)
    if total_bytes(Btab, c0) <= budget:
        return Allocation("ok", c0, 0.0, total_bytes(Btab, c0))
    lo, hi = 0.0, 1.0
    for _ in range(MAX_DOUBLINGS):
        if total_bytes(Btab, lagrangian_choice(Dtab, Btab, hi)) <= budget:
            break
        hi = hi * 2.0
    for _ in range(BISECT_STEPS):
        mid = lo + (hi - lo) / 2.0
        if total_bytes(Btab, lagrangian_choice(Dtab, Btab, mid)) <= budget:
            hi = mid
        else:
            lo = mid
    c = lagrangian_choice(Dtab, Btab, hi)
    return Allocation("ok", c, hi, total_bytes(Btab, c))


# ----------------------------------------------------------------------------------------
# Whole compress / decompress
# ----------------------------------------------------------------------------------------
@dataclass
class UnitFactors:
    group: int
    kv: int
    U_s: np.ndarray        # T x max r_T, bf16 values
    W_s: np.ndarray        # D x max r_D, bf16 values
    C_s: np.ndarray        # L_g x H x max r_T x max r_D, bf16 values
    sigma: np.ndarray      # D rotation signs
    U: np.ndarray = None   # unrounded factors (for subspace checks)
    W: np.ndarray = None
    w_eigvals: np.ndarray = None


@dataclass
class UnitRecord:
    group: int
    kv: int
    choice: int
    r_T: int
    r_D: int
    b: int
    U_s: np.ndarray
    W_s: np.ndarray
    C_s: np.ndarray
    sigma: np.ndarray
    codes: np.ndarray      # (L_g, H, T, D//16, 16) int64, empty when b == 0
    lo: np.ndarray         # (L_g, H, T, D//16) fp16 values
    step: np.ndarray
    distortion: float


@dataclass
class CompressResult:
    status: str
    shape: tuple            # (n_layers, H, T, D, L_g)
    opts: Options
    seed: int
    budget: int
    table: np.ndarray       # n_units x n_choices
    bytes: np.ndarray       # n_units x n_choices
    lam: float
    units: list = field(default_factory=list)
    factors: list = field(default_factory=list)
    total_bytes: int = 0


def unit_factors(X: np.ndarray, g: int, kv: int, opts: Options, seed: int) -> UnitFactors:
    """Token and feature factors, stored core and rotation signs of one unit."""
    rT, rD = max(opts.token_ranks), max(opts.feature_ranks)
    wvals, W = feature_factor(X)
    W = W[:, :rD]
    if opts.method == "exact":
        U = token_factor_exact(X, rT)
    elif opts.method == "randomized":
        U = token_factor_randomized(X, rT, opts.oversample, opts.power_iters, seed, g, kv)
    else:
        raise ValueError(opts.method)
    U_s, W_s = bf16_rn(U), bf16_rn(W)
    C_s = stored_core(X, U_s, W_s)
    sigma = rotation_signs(seed, g, kv, X.shape[-1])
    return UnitFactors(g, kv, U_s, W_s, C_s, sigma, U, W, wvals)


def encode_unit(X: np.ndarray, f: UnitFactors, opts: Options, choice: int, dist: float) -> UnitRecord:
    iT, iD, ib = opts.choice(choice)
    rT, rD, b = opts.token_ranks[iT], opts.feature_ranks[iD], opts.bits[ib]
    P = recon_operator(f.C_s[:, :, :rT, :], f.W_s, f.sigma, rD)
    rho = rotated_input(X, f.sigma) - np.einsum("tr,lhrd->lhtd", f.U_s[:, :rT], P, optimize=True)
    codes, lo, step, _, _ = quantize(rho, b, opts.block)
    return UnitRecord(f.group, f.kv, choice, rT, rD, b, f.U_s[:, :rT].copy(), f.W_s[:, :rD].copy(),
                      f.C_s[:, :, :rT, :rD].copy(), f.sigma, codes, lo, step, dist)


def decode_unit(rec: UnitRecord, block: int = 16) -> np.ndarray:
    """X_hat = (U_s P' + dequant(codes)) Phi^T  -- the decoder over the stored factors."""
    P = recon_operator(rec.C_s, rec.W_s, rec.sigma, rec.r_D)
    Xr = np.einsum("tr,lhrd->lhtd", rec.U_s, P, optimize=True)
    if rec.b > 0:
        rhat = rec.lo[..., None] + rec.codes * rec.step[..., None]
        Xr = Xr + rhat.reshape(Xr.shape)
    return unrotate(Xr, rec.sigma)


def compress(K, V, layers_per_group: int, opts: Options, budget: int, seed: int) -> CompressResult:
    """JoLT / FlashJoLT compress of K and V [n_layers, H, T, D] under one byte budget."""
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    nL, H, T, D = K.shape
    S = layers_per_group * H
    units = list(units_of(K, V, layers_per_group))
    Btab_u = bytes_table(T, D, S, opts).reshape(-1)
    facs, Drows = [], []
    for g, kv, X in units:
        f = unit_factors(X, g, kv, opts, seed)
        facs.append(f)
        Drows.append(distortion_table(X, f.U_s, f.W_s, f.C_s, f.sigma, opts).reshape(-1))
    Dtab = np.stack(Drows)
    Btab = np.stack([Btab_u] * len(units))
    avail = budget - header_bytes(len(units))
    res = CompressResult("ok", (nL, H, T, D, layers_per_group), opts, seed, budget, Dtab, Btab, 0.0,
                         factors=facs)
    if avail < 0:
        res.status = "infeasible"
        return res
    al = allocate(Dtab, Btab, avail)
    res.status, res.lam = al.status, al.lam
    if al.status != "ok":
        return res
    for (g, kv, X), f, c in zip(units, facs, al.choice):
        res.units.append(encode_unit(X, f, opts, int(c), float(Dtab[2 * g + kv, c])))
    res.total_bytes = header_bytes(len(units)) + al.bytes
    return res


def decompress(res: CompressResult):
    """Reconstruct K_hat, V_hat [n_layers, H, T, D] in float64 from the stored records."""
    nL, H, T, D, Lg = res.shape
    K = np.zeros((nL, H, T, D))
    V = np.zeros((nL, H, T, D))
    for rec in res.units:
        sl = slice(rec.group * Lg, (rec.group + 1) * Lg)
        (K if rec.kv == 0 else V)[sl] = decode_unit(rec, res.opts.block)
    return K, V


# ----------------------------------------------------------------------------------------
# Decode-side attention over the stored factors ([Abstract]: the decode path evaluates
# attention directly over the stored factors, without forming dense K and V tensors).
# Reading: one decode step of queries q against every cached token of one (layer, head)
# slice of a layer group.  With Phi = diag(sigma) H / sqrt(D), the decoder above stores the
# slice as X_hat = (U_s P' + rho_hat) Phi^T, so
#   scores:  X_hat q = U_s (P' q') + rho_hat q',   q' = Phi^T q  (rotate(q) as a row),
#   values:  p^T X_hat = (p^T U_s P' + p^T rho_hat) Phi^T,
# and rho_hat q' sums, per 16-wide block, lo * (sum of q' over the block) + step * (codes . q').
# Scores are scaled by 1 / sqrt(D) before the softmax.
# ----------------------------------------------------------------------------------------
def softmax(s: np.ndarray) -> np.ndarray:
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / e.sum(axis=-1, keepdims=True)


def slice_scores_factored(rec: UnitRecord, l: int, h: int, q: np.ndarray, block: int = 16) -> np.ndarray:
    """X_hat[l, h] q for queries q (nq, D) from the stored factors and codes: (nq, T)."""
    D = q.shape[-1]
    P = recon_operator(rec.C_s, rec.W_s, rec.sigma, rec.r_D)[l, h]      # (r_T, D), rotated
    qr = rotate(np.asarray(q, dtype=np.float64), rec.sigma)             # q' as rows
    s = (rec.U_s @ (P @ qr.T)).T                                        # (nq, T)
    if rec.b > 0:
        nb = D // block
        qb = qr.reshape(qr.shape[0], nb, block)
        s = s + np.einsum("tb,qb->qt", rec.lo[l, h], qb.sum(-1), optimize=True)
        s = s + np.einsum("tb,tbj,qbj->qt", rec.step[l, h], rec.codes[l, h].astype(np.float64), qb,
                          optimize=True)
    return s


def slice_values_factored(rec: UnitRecord, l: int, h: int, p: np.ndarray, block: int = 16) -> np.ndarray:
    """p^T X_hat[l, h] for attention weights p (nq, T) from the stored factors: (nq, D)."""
    P = recon_operator(rec.C_s, rec.W_s, rec.sigma, rec.r_D)[l, h]
    y = (np.asarray(p, dtype=np.float64) @ rec.U_s) @ P                 # rotated basis
    if rec.b > 0:
        rhat = rec.lo[l, h][..., None] + rec.codes[l, h] * rec.step[l, h][..., None]   # (T, nb, block)
        y = y + p @ rhat.reshape(rhat.shape[0], -1)
    return unrotate(y, rec.sigma)


def slice_attention_factored(recK: UnitRecord, recV: UnitRecord, l: int, h: int, q: np.ndarray,
                             block: int = 16):
    """One decode step over the stored factors: (softmax weights (nq, T), output (nq, D))."""
    D = q.shape[-1]
    p = softmax(slice_scores_factored(recK, l, h, q, block) / math.sqrt(D))
    return p, slice_values_factored(recV, l, h, p, block)


def relative_error(X: np.ndarray, Xhat: np.ndarray) -> float:
    """|| X - X_hat ||_F / || X ||_F ([Intro]: relative Frobenius error, reported per K and V)."""
    X = np.asarray(X, dtype=np.float64)
    return float(np.linalg.norm((X - Xhat).ravel()) / np.linalg.norm(X.ravel()))


def budget_for_ratio(n_layers: int, H: int, T: int, D: int, ratio: float) -> int:
    """Byte budget for an x-fold compression of K plus V measured against their bf16 size."""
    return int((2 * 2 * n_layers * H * T * D) / ratio)
