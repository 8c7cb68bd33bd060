"""Python binding of libjolt.so (argument marshalling only).

Every step of the compress / allocate / decompress path runs in the library's CUDA
kernels; torch is used here for device memory and the current stream.  The binding
raises if the library is missing: there is no other implementation behind it.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libjolt.so")

MAXC = 8
JOLT_BF16, JOLT_F32 = 0, 1
JOLT_EXACT, JOLT_RANDOMIZED = 0, 1

STATUS_NAMES = {
    0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED_SHAPE", 3: "WORKSPACE_TOO_SMALL", 4: "OUTPUT_TOO_SMALL",
    5: "BUDGET_INFEASIBLE", 6: "NUMERIC", 7: "TIMEOUT", 8: "CUDA", 9: "BAD_BLOB",
}

EXPORTED = [
    "jolt_version", "jolt_last_error", "jolt_workspace_size", "jolt_counts", "jolt_choice_bytes",
    "jolt_compress", "jolt_factor", "jolt_table", "jolt_allocate", "jolt_encode", "jolt_read_header",
    "jolt_decompress", "jolt_frobenius", "jolt_profile_begin", "jolt_profile_end", "jolt_recon_operator",
    "jolt_launch_count", "jolt_frobenius_noalloc", "jolt_set_graphs", "jolt_release", "jolt_fp32_rate_probe",
    "jolt_wait_selftest", "jolt_attend_prepare", "jolt_attend_scratch_size", "jolt_attend", "jolt_quant_baseline",
]


class JoltError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status
        self.name = STATUS_NAMES.get(status, str(status))


class CShape(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int32), ("n_heads", ctypes.c_int32), ("n_tokens", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("layers_per_group", ctypes.c_int32), ("dtype", ctypes.c_int32)]


class COptions(ctypes.Structure):
    _fields_ = [("n_token_ranks", ctypes.c_int32), ("token_ranks", ctypes.c_int32 * MAXC),
                ("n_feature_ranks", ctypes.c_int32), ("feature_ranks", ctypes.c_int32 * MAXC),
                ("n_bits", ctypes.c_int32), ("bits", ctypes.c_int32 * MAXC),
                ("method", ctypes.c_int32), ("oversample", ctypes.c_int32), ("power_iters", ctypes.c_int32),
                ("unit_offset", ctypes.c_int32)]


class CUnitRecord(ctypes.Structure):
    _fields_ = [("r_T", ctypes.c_int32), ("r_D", ctypes.c_int32), ("bits", ctypes.c_int32),
                ("choice", ctypes.c_int32), ("off_U", ctypes.c_uint64), ("off_W", ctypes.c_uint64),
                ("off_C", ctypes.c_uint64), ("off_codes", ctypes.c_uint64), ("off_scales", ctypes.c_uint64),
                ("distortion", ctypes.c_double)]


_lib = None


def lib():
    """Load libjolt.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with kv_cache_compression_group_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        vp, sz, i32, u64, pS, pO = (ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_uint64,
                                    ctypes.POINTER(CShape), ctypes.POINTER(COptions))
        L.jolt_version.restype = ctypes.c_char_p
        L.jolt_last_error.restype = ctypes.c_char_p
        sigs = {
            "jolt_workspace_size": [pS, pO, ctypes.POINTER(sz), ctypes.POINTER(sz), ctypes.POINTER(sz)],
            "jolt_counts": [pS, pO, ctypes.POINTER(i32), ctypes.POINTER(i32)],
            "jolt_choice_bytes": [pS, pO, ctypes.POINTER(u64)],
            "jolt_compress": [pS, vp, vp, pO, u64, u64, vp, sz, vp, sz, vp],
            "jolt_factor": [pS, vp, vp, pO, u64, vp, ctypes.c_int64, vp, ctypes.c_int64, vp, sz, vp],
            "jolt_table": [pS, vp, vp, pO, u64, vp, ctypes.c_int64, vp, ctypes.c_int64, vp, vp, vp, sz, vp],
            "jolt_allocate": [vp, vp, i32, i32, u64, vp, vp, vp, vp],
            "jolt_encode": [pS, vp, vp, pO, u64, vp, ctypes.c_int64, vp, ctypes.c_int64, vp, vp, vp, vp, sz, vp,
                            sz, vp],
            "jolt_read_header": [vp, pS, ctypes.POINTER(u64), ctypes.POINTER(CUnitRecord), i32, vp],
            "jolt_decompress": [vp, i32, vp, vp, vp, sz, vp],
            "jolt_frobenius": [pS, vp, vp, vp, vp, i32, vp, vp, sz, vp],
            "jolt_frobenius_noalloc": [pS, vp, vp, vp, vp, i32, vp, vp],
            "jolt_recon_operator": [pS, pO, u64, vp, vp, ctypes.c_int64, vp, vp, sz, vp],
            "jolt_profile_begin": [],
            "jolt_profile_end": [ctypes.c_char_p, sz],
            "jolt_release": [],
            "jolt_fp32_rate_probe": [i32, i32, vp, ctypes.POINTER(u64), vp],
            "jolt_wait_selftest": [i32, ctypes.c_uint32, vp, vp],
            "jolt_attend_prepare": [vp, vp, sz, vp],
            "jolt_attend_scratch_size": [pS, i32, i32, ctypes.POINTER(sz)],
            "jolt_attend": [vp, vp, sz, i32, vp, i32, vp, vp, sz, vp],
            "jolt_quant_baseline": [pS, vp, vp, i32, vp, vp, vp, vp, sz, vp],
        }
        L.jolt_launch_count.argtypes = []
        L.jolt_launch_count.restype = ctypes.c_uint64
        L.jolt_set_graphs.argtypes = [i32]
        L.jolt_set_graphs.restype = None
        for name, args in sigs.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        _lib = L
    return _lib


def _check(status: int):
    if status != 0:
        raise JoltError(status, lib().jolt_last_error().decode())


def _stream(stream=None):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


# ------------------------------------------------------------------------------------------
@dataclass
class Options:
    """Candidate sets and token-factor method (choice c = (i_T*|R_D| + i_D)*|B| + i_b)."""

    token_ranks: tuple
    feature_ranks: tuple
    bits: tuple
    method: str = "exact"
    oversample: int = 10
    power_iters: int = 2
    unit_offset: int = 0    # global index of the first unit (a shard of a larger cache)

    def c(self) -> COptions:
        o = COptions()
        for name, vals in (("token_ranks", self.token_ranks), ("feature_ranks", self.feature_ranks),
                           ("bits", self.bits)):
            if len(vals) > MAXC:
                raise ValueError(f"at most {MAXC} {name}")
            setattr(o, "n_" + name, len(vals))
            arr = getattr(o, name)
            for i, v in enumerate(vals):
                arr[i] = int(v)
        o.method = {"exact": JOLT_EXACT, "randomized": JOLT_RANDOMIZED}[self.method]
        o.oversample = self.oversample
        o.power_iters = self.power_iters
        o.unit_offset = self.unit_offset
        return o

    @property
    def n_choices(self):
        return len(self.token_ranks) * len(self.feature_ranks) * len(self.bits)


def default_options(T: int, D: int, method: str = "exact", bits=(0, 1, 2, 3, 4, 8)) -> Options:
    """Candidate sets used for the Mistral / LLaMA shaped workloads: token ranks T/32, T/16, T/8
    and 15T/64 (128..960 from 4096 tokens on: 128, 256, 512, 960), feature ranks D/4..D.

    The largest token rank is 15T/64 rather than T/4 so that FlashJoLT's sketch (largest rank
    + 10 = 250 at 1024 tokens) stays within 256 columns, where the batched eigen solver of the
    Rayleigh-Ritz step runs at about half the time it needs at 266."""
    if T <= 4096:
        rt = tuple(max(8, T // d) for d in (32, 16, 8)) + (max(8, (15 * T // 64) // 8 * 8),)
    else:
        rt = (128, 256, 512, 960)
    rd = (D // 4, D // 2, 3 * D // 4, D)
    return Options(rt, rd, tuple(bits), method)


def make_shape(K: torch.Tensor, layers_per_group: int) -> CShape:
    if K.dim() != 4:
        raise ValueError("cache must be [n_layers, n_heads, n_tokens, head_dim]")
    s = CShape()
    s.n_layers, s.n_heads, s.n_tokens, s.head_dim = K.shape
    s.layers_per_group = layers_per_group
    if K.dtype == torch.bfloat16:
        s.dtype = JOLT_BF16
    elif K.dtype == torch.float32:
        s.dtype = JOLT_F32
    else:
        raise ValueError("cache dtype must be bf16 or fp32")
    return s


def sizes(shape: CShape, opts: Options):
    ws, blob, dws = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().jolt_workspace_size(ctypes.byref(shape), ctypes.byref(opts.c()), ctypes.byref(ws),
                                     ctypes.byref(blob), ctypes.byref(dws)))
    return ws.value, blob.value, dws.value


def counts(shape: CShape, opts: Options):
    nu, nc = ctypes.c_int32(), ctypes.c_int32()
    _check(lib().jolt_counts(ctypes.byref(shape), ctypes.byref(opts.c()), ctypes.byref(nu), ctypes.byref(nc)))
    return nu.value, nc.value


def choice_bytes(shape: CShape, opts: Options):
    n = opts.n_choices
    arr = (ctypes.c_uint64 * n)()
    _check(lib().jolt_choice_bytes(ctypes.byref(shape), ctypes.byref(opts.c()), arr))
    return [int(x) for x in arr]


def _check_cache(K, V):
    if K.shape != V.shape or K.dtype != V.dtype:
        raise ValueError("K and V must have the same shape and dtype")
    if not (K.is_cuda and V.is_cuda and K.is_contiguous() and V.is_contiguous()):
        raise ValueError("K and V must be contiguous CUDA tensors")


class Compressor:
    """Holds the workspace for one cache shape and candidate set; compress / decompress
    calls reuse it.  All buffers are torch device tensors owned by this object."""

    def __init__(self, n_layers, n_heads, n_tokens, head_dim, layers_per_group, dtype, opts: Options,
                 device="cuda"):
        self.shape = CShape(n_layers, n_heads, n_tokens, head_dim, layers_per_group,
                            JOLT_BF16 if dtype == torch.bfloat16 else JOLT_F32)
        self.opts = opts
        self._copts = opts.c()
        self.ws_bytes, self.blob_max, self.dws_bytes = sizes(self.shape, opts)
        self.n_units, self.n_choices = counts(self.shape, opts)
        self.device = torch.device(device)
        self.ws = torch.empty(self.ws_bytes + 256, dtype=torch.uint8, device=self.device)
        self.dws = None

    def _ws_ptr(self, t):
        p = t.data_ptr()
        return ctypes.c_void_p((p + 255) // 256 * 256)

    def compress(self, K, V, budget: int, seed: int = 0, blob: torch.Tensor | None = None, stream=None):
        """Compress K, V under `budget` total bytes; returns the blob (uint8 device tensor of
        capacity max(budget, needed)).  Asynchronous; errors found on the device surface in
        read_header / decompress."""
        _check_cache(K, V)
        cap = min(int(budget), self.blob_max) if blob is None else blob.numel()
        if blob is None:
            blob = torch.empty(max(cap, 64 + 64 * self.n_units), dtype=torch.uint8, device=K.device)
        _check(lib().jolt_compress(ctypes.byref(self.shape), _ptr(K), _ptr(V), ctypes.byref(self._copts),
                                   int(budget), int(seed), _ptr(blob), blob.numel(), self._ws_ptr(self.ws),
                                   self.ws_bytes, _stream(stream)))
        return blob

    def factor(self, K, V, seed: int = 0, stream=None):
        _check_cache(K, V)
        o = self.opts
        rT, rD = max(o.token_ranks), max(o.feature_ranks)
        U = torch.zeros((self.n_units, self.shape.n_tokens, rT), dtype=torch.float32, device=K.device)
        W = torch.zeros((self.n_units, self.shape.head_dim, rD), dtype=torch.float32, device=K.device)
        _check(lib().jolt_factor(ctypes.byref(self.shape), _ptr(K), _ptr(V), ctypes.byref(self._copts), int(seed),
                                 _ptr(U), rT, _ptr(W), rD, self._ws_ptr(self.ws), self.ws_bytes, _stream(stream)))
        return U, W

    def table(self, K, V, U_bf16, W_bf16, seed: int = 0, stream=None):
        """Core (bf16) and distortion table (fp64) from given bf16 factors [units, T, r_T], [units, D, r_D]."""
        _check_cache(K, V)
        o = self.opts
        rT, rD = max(o.token_ranks), max(o.feature_ranks)
        S = self.shape.layers_per_group * self.shape.n_heads
        core = torch.zeros((self.n_units, S, rT, rD), dtype=torch.bfloat16, device=K.device)
        tab = torch.zeros((self.n_units, self.n_choices), dtype=torch.float64, device=K.device)
        U_bf16 = U_bf16.contiguous()
        W_bf16 = W_bf16.contiguous()
        _check(lib().jolt_table(ctypes.byref(self.shape), _ptr(K), _ptr(V), ctypes.byref(self._copts), int(seed),
                                _ptr(U_bf16), U_bf16.shape[-1], _ptr(W_bf16), W_bf16.shape[-1], _ptr(core),
                                _ptr(tab), self._ws_ptr(self.ws), self.ws_bytes, _stream(stream)))
        return core, tab

    def recon_operator(self, core, W_bf16, seed: int = 0, stream=None):
        """Rotated reconstruction operators P' [n_feature_ranks, units, S, max r_T, D] (bf16)."""
        o = self.opts
        S = self.shape.layers_per_group * self.shape.n_heads
        P = torch.zeros((len(o.feature_ranks), self.n_units, S, max(o.token_ranks), self.shape.head_dim),
                        dtype=torch.bfloat16, device=core.device)
        W_bf16 = W_bf16.contiguous()
        _check(lib().jolt_recon_operator(ctypes.byref(self.shape), ctypes.byref(self._copts), int(seed),
                                         _ptr(core.contiguous()), _ptr(W_bf16), W_bf16.shape[-1], _ptr(P),
                                         self._ws_ptr(self.ws), self.ws_bytes, _stream(stream)))
        return P

    def encode(self, K, V, U_bf16, W_bf16, core, choice, dist, seed: int = 0, cap: int | None = None, stream=None):
        _check_cache(K, V)
        cap = self.blob_max if cap is None else cap
        blob = torch.zeros(cap, dtype=torch.uint8, device=K.device)
        choice = choice.to(device=K.device, dtype=torch.int32).contiguous()
        dist = dist.to(device=K.device, dtype=torch.float64).contiguous()
        _check(lib().jolt_encode(ctypes.byref(self.shape), _ptr(K), _ptr(V), ctypes.byref(self._copts), int(seed),
                                 _ptr(U_bf16.contiguous()), U_bf16.shape[-1], _ptr(W_bf16.contiguous()),
                                 W_bf16.shape[-1], _ptr(core.contiguous()), _ptr(choice), _ptr(dist), _ptr(blob),
                                 blob.numel(), self._ws_ptr(self.ws), self.ws_bytes, _stream(stream)))
        return blob

    def decompress(self, blob, out_dtype=None, K_out=None, V_out=None, stream=None):
        if out_dtype is None:
            out_dtype = torch.bfloat16 if self.shape.dtype == JOLT_BF16 else torch.float32
        shp = (self.shape.n_layers, self.shape.n_heads, self.shape.n_tokens, self.shape.head_dim)
        if K_out is None:
            K_out = torch.empty(shp, dtype=out_dtype, device=blob.device)
            V_out = torch.empty(shp, dtype=out_dtype, device=blob.device)
        if self.dws is None:
            self.dws = torch.empty(self.dws_bytes + 256, dtype=torch.uint8, device=blob.device)
        _check(lib().jolt_decompress(_ptr(blob), JOLT_F32 if out_dtype == torch.float32 else JOLT_BF16,
                                     _ptr(K_out), _ptr(V_out), self._ws_ptr(self.dws), self.dws_bytes,
                                     _stream(stream)))
        return K_out, V_out


class Attention:
    """Decode-side attention over one compressed blob: prepare once (the aligned factors and
    rotated operators in a workspace it owns), then attend(layer, q) for any layer."""

    def __init__(self, comp: "Compressor", blob: torch.Tensor, n_q_heads: int, stream=None):
        self.blob = blob
        self.nq = int(n_q_heads)
        self.D = comp.shape.head_dim
        self.ws = torch.empty(comp.dws_bytes + 256, dtype=torch.uint8, device=blob.device)
        self.ws_ptr = comp._ws_ptr(self.ws)
        self.ws_bytes = comp.dws_bytes
        nbytes = ctypes.c_size_t()
        _check(lib().jolt_attend_scratch_size(ctypes.byref(comp.shape), max(comp.opts.token_ranks), self.nq,
                                              ctypes.byref(nbytes)))
        self.scratch = torch.empty(nbytes.value, dtype=torch.uint8, device=blob.device)
        _check(lib().jolt_attend_prepare(_ptr(blob), self.ws_ptr, self.ws_bytes, _stream(stream)))

    def attend(self, layer: int, q: torch.Tensor, out: torch.Tensor | None = None, stream=None):
        """q [n_q_heads, head_dim] fp32 on the device; returns the attention output (same shape)."""
        q = q.to(torch.float32).contiguous()
        if q.shape != (self.nq, self.D):
            raise ValueError(f"q must be [{self.nq}, {self.D}]")
        if out is None:
            out = torch.empty_like(q)
        _check(lib().jolt_attend(_ptr(self.blob), self.ws_ptr, self.ws_bytes, int(layer), _ptr(q), self.nq, _ptr(out),
                                 _ptr(self.scratch), self.scratch.numel(), _stream(stream)))
        return out


def read_header(blob: torch.Tensor, stream=None):
    """(shape dict, total bytes, list of unit records); synchronises.  Raises on a device-side
    error recorded in the blob (infeasible budget, non-finite input, ...)."""
    sh = CShape()
    tot = ctypes.c_uint64()
    n = 4096
    recs = (CUnitRecord * n)()
    _check(lib().jolt_read_header(_ptr(blob), ctypes.byref(sh), ctypes.byref(tot), recs, n, _stream(stream)))
    G = sh.n_layers // sh.layers_per_group
    units = [dict(r_T=r.r_T, r_D=r.r_D, bits=r.bits, choice=r.choice, off_U=r.off_U, off_W=r.off_W,
                  off_C=r.off_C, off_codes=r.off_codes, off_scales=r.off_scales, distortion=r.distortion)
             for r in recs[:2 * G]]
    shape = dict(n_layers=sh.n_layers, n_heads=sh.n_heads, n_tokens=sh.n_tokens, head_dim=sh.head_dim,
                 layers_per_group=sh.layers_per_group, dtype=sh.dtype)
    return shape, tot.value, units


def allocate(dist: torch.Tensor, nbytes: torch.Tensor, budget: int, stream=None):
    """Lagrangian dual on device tables [units, choices]: returns (choice int32, lambda, status)."""
    nu, nc = dist.shape
    dist = dist.to(torch.float64).contiguous()
    nbytes = nbytes.to(torch.int64).contiguous()
    choice = torch.zeros(nu, dtype=torch.int32, device=dist.device)
    lam = torch.zeros(1, dtype=torch.float64, device=dist.device)
    status = torch.zeros(1, dtype=torch.int32, device=dist.device)
    _check(lib().jolt_allocate(_ptr(dist), _ptr(nbytes), nu, nc, int(budget), _ptr(choice), _ptr(lam), _ptr(status),
                               _stream(stream)))
    return choice, lam, status


def frobenius(K, V, K_hat=None, V_hat=None, layers_per_group=1, stream=None):
    """Per-unit [||X_u||^2, ||X_u - Y_u||^2] (fp64, device) for units u = 2 g + kv."""
    shape = make_shape(K, layers_per_group)
    G = K.shape[0] // layers_per_group
    sq = torch.zeros(2 * 2 * G, dtype=torch.float64, device=K.device)
    ws = torch.empty(2 * G * 64 * 16, dtype=torch.uint8, device=K.device)
    yd = JOLT_F32 if (K_hat is not None and K_hat.dtype == torch.float32) else JOLT_BF16
    _check(lib().jolt_frobenius(ctypes.byref(shape), _ptr(K), _ptr(V), _ptr(K_hat), _ptr(V_hat), yd, _ptr(sq),
                                _ptr(ws), ws.numel(), _stream(stream)))
    return sq.view(2 * G, 2)


def launch_count() -> int:
    """Kernels launched by the library in this process so far."""
    return int(lib().jolt_launch_count())


def set_graphs(enable: bool):
    """CUDA graphs of repeated compress calls on this thread (on by default)."""
    lib().jolt_set_graphs(1 if enable else 0)


def profile_begin():
    """Start recording CUDA events around every library stage on this thread."""
    _check(lib().jolt_profile_begin())


def profile_end():
    """Stop recording; returns {stage: (total_ms, launches, units)} (synchronises)."""
    buf = ctypes.create_string_buffer(1 << 16)
    _check(lib().jolt_profile_end(buf, len(buf)))
    out = {}
    for line in buf.value.decode().splitlines():
        name, ms, n, u = line.split()
        out[name] = (float(ms), int(n), int(u))
    return out


def release():
    """Release this thread's library-owned streams, events, cached graphs and solver handles."""
    _check(lib().jolt_release())


def fp32_rate_probe(packed: bool, iters: int, sink: torch.Tensor, stream=None) -> int:
    """Launch the FP32-pipe rate probe on the stream; returns the FMAs the launch performs."""
    ops = ctypes.c_uint64()
    _check(lib().jolt_fp32_rate_probe(1 if packed else 0, int(iters), _ptr(sink), ctypes.byref(ops),
                                      _stream(stream)))
    return int(ops.value)


def wait_selftest(arrive: bool, limit_us: int, status: torch.Tensor, stream=None):
    """Bounded device wait self-test (synchronises); raises JoltError TIMEOUT when it gives up."""
    _check(lib().jolt_wait_selftest(1 if arrive else 0, int(limit_us), _ptr(status), _stream(stream)))


def frobenius_noalloc(K, V, K_hat=None, V_hat=None, layers_per_group=1, stream=None):
    """As frobenius(), through the entry point that needs no workspace (its scratch is a
    fixed array inside the library; calls whose GPU work overlaps must not be mixed)."""
    shape = make_shape(K, layers_per_group)
    G = K.shape[0] // layers_per_group
    sq = torch.zeros(2 * 2 * G, dtype=torch.float64, device=K.device)
    yd = JOLT_F32 if (K_hat is not None and K_hat.dtype == torch.float32) else JOLT_BF16
    _check(lib().jolt_frobenius_noalloc(ctypes.byref(shape), _ptr(K), _ptr(V), _ptr(K_hat), _ptr(V_hat), yd,
                                        _ptr(sq), _stream(stream)))
    return sq.view(2 * G, 2)


def quant_baseline(K, V, bits: int, layers_per_group: int, keep_codes: bool = False, stream=None):
    """Per-block b-bit quantisation of K and V themselves: per-unit [||X_u||^2, ||X_u - Q(X_u)||^2]
    (fp64, device), and (keep_codes) the codes and fp16 scales."""
    shape = make_shape(K, layers_per_group)
    G = K.shape[0] // layers_per_group
    nblk_all = 2 * K.numel() // 16
    sq = torch.zeros(2 * 2 * G, dtype=torch.float64, device=K.device)
    ws = torch.empty(2 * G * 148 * 16, dtype=torch.uint8, device=K.device)
    codes = torch.empty(nblk_all * 2 * bits, dtype=torch.uint8, device=K.device) if keep_codes else None
    scales = torch.empty(nblk_all * 2, dtype=torch.float16, device=K.device) if keep_codes else None
    _check(lib().jolt_quant_baseline(ctypes.byref(shape), _ptr(K), _ptr(V), int(bits), _ptr(codes), _ptr(scales),
                                     _ptr(sq), _ptr(ws), ws.numel(), _stream(stream)))
    return sq.view(2 * G, 2), codes, scales


def relative_errors(K, V, K_hat, V_hat, layers_per_group):
    """Relative Frobenius error of K and of V over all their units."""
    sq = frobenius(K, V, K_hat, V_hat, layers_per_group).cpu()
    k, v = sq[0::2], sq[1::2]
    return float((k[:, 1].sum() / k[:, 0].sum()).sqrt()), float((v[:, 1].sum() / v[:, 0].sum()).sqrt())
