"""Python binding of libmuon.so (ctypes).

Argument marshalling only: every step of the computation runs in the CUDA
library. PyTorch supplies device memory (outputs and workspaces are torch
tensors) and the current CUDA stream. If the library is missing, loading it
raises: there is no fallback.
"""

from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass, field

HERE = os.path.dirname(os.path.abspath(__file__))
# MUON_BOUNDS_CHECK=1 loads the bounds-checked debug build (built by
# `python -m newton_schulz_10_b200.build --debug`): the same library with
# device-side index checks that report MUON_ERR_INVALID_ARG.
LIB_PATH = os.path.join(HERE, "libmuon_check.so" if os.environ.get("MUON_BOUNDS_CHECK") == "1" else "libmuon.so")
MAX_T = 16

# muon_status
OK, ERR_INVALID_ARG, ERR_SHAPE, ERR_DTYPE, ERR_ALIGN, ERR_WORKSPACE, ERR_CUDA, ERR_NONFINITE, \
    ERR_TIMEOUT, ERR_UNSUPPORTED = range(10)
# muon_dtype
F32, BF16, F16 = 0, 1, 2
# muon_norm
NORM_L1, NORM_L2 = 0, 1

EXPORTS = ("muon_set_wait_timeout_ns", "muon_set_gemm_cta_pair", "muon_status_str", "muon_rows_for_fraction", "muon_ns_params_default",
           "muon_ns_workspace_size", "ns_polar", "gram_ns_polar", "normuon_scale", "muon_select_workspace_size",
           "select_rows", "muon_workspace_size", "muon_step", "muon_step_profiled", "muon_kernel_launch_count",
           "select_rows_noalloc", "muon_step_events", "muon_set_gemm_chain", "muon_momentum",
           "muon_orthogonalize", "muon_apply_update")


class NsParams(C.Structure):
    _fields_ = [("T", C.c_int32), ("coeffs", (C.c_float * 3) * MAX_T), ("norm_eps", C.c_float),
                ("gram", C.c_int32), ("restart_at", C.c_int32), ("compute", C.c_int32)]


class Matrix(C.Structure):
    _fields_ = [("W", C.c_void_p), ("M", C.c_void_p), ("G", C.c_void_p), ("v", C.c_void_p),
                ("rows", C.c_int64), ("cols", C.c_int64)]


class Params(C.Structure):
    _fields_ = [("mu", C.c_float), ("lr", C.c_float), ("ns", NsParams), ("normuon", C.c_int32),
                ("beta2", C.c_float), ("normuon_eps", C.c_float), ("dion3", C.c_int32),
                ("frac_num", C.c_int32), ("frac_den", C.c_int32), ("select_norm", C.c_int32),
                ("dev_status", C.c_void_p)]


class StepProfile(C.Structure):
    _fields_ = [("ms_total", C.c_float), ("ms_prologue", C.c_float), ("ms_ns", C.c_float),
                ("ms_normuon", C.c_float), ("ms_update", C.c_float), ("kernel_launches", C.c_int64),
                ("gemm_launches", C.c_int64), ("ns_flops", C.c_double), ("ns_flops_dense", C.c_double),
                ("ns_flops_executed", C.c_double), ("bytes_prologue", C.c_double), ("bytes_update", C.c_double)]

    def as_dict(self):
        return {name: getattr(self, name) for name, _ in self._fields_}


class MuonError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_str(code)}")


_lib = None


def lib() -> C.CDLL:
    """Load libmuon.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m newton_schulz_10_b200.build`")
        L = C.CDLL(LIB_PATH)
        vp, i32, i64, sz, f32 = C.c_void_p, C.c_int32, C.c_int64, C.c_size_t, C.c_float
        L.muon_set_wait_timeout_ns.argtypes = [C.c_uint64]
        L.muon_set_wait_timeout_ns.restype = None
        L.muon_set_gemm_cta_pair.argtypes = [i32]
        L.muon_set_gemm_cta_pair.restype = None
        L.muon_set_gemm_chain.argtypes = [i32]
        L.muon_set_gemm_chain.restype = None
        L.muon_status_str.argtypes = [i32]
        L.muon_status_str.restype = C.c_char_p
        L.muon_rows_for_fraction.argtypes = [i64, i32, i32]
        L.muon_rows_for_fraction.restype = i64
        L.muon_ns_params_default.argtypes = [C.POINTER(NsParams)]
        L.muon_ns_params_default.restype = None
        L.muon_ns_workspace_size.argtypes = [i64, i64, C.POINTER(NsParams)]
        L.muon_ns_workspace_size.restype = sz
        for name in ("ns_polar", "gram_ns_polar"):
            fn = getattr(L, name)
            fn.argtypes = [vp, i32, vp, i32, i64, i64, C.POINTER(NsParams), vp, sz, vp]
            fn.restype = i32
        L.normuon_scale.argtypes = [vp, i32, i64, i64, vp, vp, f32, f32, vp, vp, vp]
        L.normuon_scale.restype = i32
        L.muon_select_workspace_size.argtypes = [i64]
        L.muon_select_workspace_size.restype = sz
        L.select_rows.argtypes = [vp, i64, i64, i64, i32, vp, vp, sz, vp]
        L.select_rows.restype = i32
        L.select_rows_noalloc.argtypes = [vp, i64, i64, i64, i32, vp, vp, vp]
        L.select_rows_noalloc.restype = i32
        L.muon_workspace_size.argtypes = [C.POINTER(Matrix), i32, C.POINTER(Params)]
        L.muon_workspace_size.restype = sz
        L.muon_step.argtypes = [C.POINTER(Matrix), i32, C.POINTER(Params), vp, sz, vp]
        L.muon_step.restype = i32
        L.muon_step_profiled.argtypes = [C.POINTER(Matrix), i32, C.POINTER(Params), vp, sz, vp,
                                         C.POINTER(StepProfile)]
        L.muon_step_profiled.restype = i32
        L.muon_step_events.argtypes = [C.POINTER(Matrix), i32, C.POINTER(Params), vp, sz, vp, C.POINTER(vp)]
        L.muon_step_events.restype = i32
        L.muon_momentum.argtypes = [C.POINTER(Matrix), i32, C.POINTER(Params), vp]
        L.muon_momentum.restype = i32
        L.muon_orthogonalize.argtypes = [C.POINTER(Matrix), i32, C.POINTER(Params), C.POINTER(vp), C.POINTER(vp),
                                         C.POINTER(vp), vp, sz, vp]
        L.muon_orthogonalize.restype = i32
        L.muon_apply_update.argtypes = [C.POINTER(Matrix), i32, C.POINTER(Params), C.POINTER(vp), C.POINTER(vp),
                                        C.POINTER(vp), vp]
        L.muon_apply_update.restype = i32
        L.muon_kernel_launch_count.argtypes = []
        L.muon_kernel_launch_count.restype = i64
        _lib = L
    return _lib


def status_str(code: int) -> str:
    return lib().muon_status_str(code).decode()


def _check(code: int, where: str) -> None:
    if code != OK:
        raise MuonError(code, where)


# ---------------------------------------------------------------------------
# parameters
# ---------------------------------------------------------------------------

WORKLOAD_COEFFS = (3.4445, -4.7750, 2.0315)


def ns_params(T: int = 5, coeffs=None, norm_eps: float = 1e-7, gram: bool = False, restart_at: int = 3,
              compute: int = BF16) -> NsParams:
    p = NsParams()
    lib().muon_ns_params_default(C.byref(p))
    p.T = T
    if coeffs is not None:
        coeffs = list(coeffs)
        if len(coeffs) == 3 and not hasattr(coeffs[0], "__len__"):
            coeffs = [coeffs] * T
        for t, (a, b, c) in enumerate(coeffs[:MAX_T]):
            p.coeffs[t][0], p.coeffs[t][1], p.coeffs[t][2] = a, b, c
    p.norm_eps = norm_eps
    p.gram = int(gram)
    p.restart_at = restart_at
    p.compute = compute
    return p


def step_params(mu=0.95, lr=0.02, ns: NsParams | None = None, normuon=False, beta2=0.95, normuon_eps=1e-8,
                dion3=False, frac=(1, 1), select_norm=NORM_L1, dev_status=None) -> Params:
    p = Params()
    p.mu, p.lr = mu, lr
    p.ns = ns if ns is not None else ns_params()
    p.normuon, p.beta2, p.normuon_eps = int(normuon), beta2, normuon_eps
    p.dion3 = int(dion3)
    p.frac_num, p.frac_den = frac
    p.select_norm = select_norm
    p.dev_status = None if dev_status is None else _ptr(dev_status)
    return p


# ---------------------------------------------------------------------------
# tensor helpers
# ---------------------------------------------------------------------------


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int | None:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


def _dtype_code(t) -> int:
    import torch
    return {torch.float32: F32, torch.bfloat16: BF16, torch.float16: F16}[t.dtype]


def workspace(nbytes: int, device=None):
    """A caller-owned workspace tensor of at least nbytes (256-byte aligned)."""
    import torch
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")


def kernel_launch_count() -> int:
    """Kernels this library queued from the calling thread so far."""
    return lib().muon_kernel_launch_count()


def set_gemm_cta_pair(enable: bool) -> None:
    """True (default): CTA-pair tensor-core GEMM; False: single-CTA kernel."""
    lib().muon_set_gemm_cta_pair(int(bool(enable)))


def set_gemm_chain(enable: bool) -> None:
    """True: each Newton-Schulz chain runs as one fused persistent launch;
    False (default): one launch per product."""
    lib().muon_set_gemm_chain(int(bool(enable)))


def set_wait_timeout_ns(ns: int) -> None:
    lib().muon_set_wait_timeout_ns(int(ns))


def rows_for_fraction(n: int, f_num: int, f_den: int) -> int:
    return lib().muon_rows_for_fraction(n, f_num, f_den)


def ns_workspace_size(rows: int, cols: int, p: NsParams) -> int:
    return lib().muon_ns_workspace_size(rows, cols, C.byref(p))


def _polar(name, X, p: NsParams, out_dtype, ws, stream):
    import torch
    assert X.dim() == 2 and X.is_contiguous()
    O = torch.empty(X.shape, dtype=out_dtype or X.dtype, device=X.device)
    if ws is None:
        ws = workspace(ns_workspace_size(X.shape[0], X.shape[1], p), X.device)
    code = getattr(lib(), name)(_ptr(X), _dtype_code(X), _ptr(O), _dtype_code(O), X.shape[0], X.shape[1],
                                C.byref(p), _ptr(ws), ws.numel(), _stream(stream))
    _check(code, name)
    return O, ws


def ns_polar(X, p: NsParams | None = None, out_dtype=None, ws=None, stream=None):
    """O ~= polar(X) by standard (or, with p.gram, Gram) Newton-Schulz.
    Returns (O, workspace); the first 4 workspace bytes hold the device status."""
    return _polar("ns_polar", X, p or ns_params(), out_dtype, ws, stream)


def gram_ns_polar(X, p: NsParams | None = None, out_dtype=None, ws=None, stream=None):
    return _polar("gram_ns_polar", X, p or ns_params(gram=True, compute=F16), out_dtype, ws, stream)


def normuon_scale(O, v, beta2=0.95, eps=1e-8, rows=None, dev_status=None, stream=None):
    """Row scales of Eq. (2) for O (k x m); updates v in place."""
    import torch
    k, m = O.shape
    out = torch.empty(k, dtype=torch.float32, device=O.device)
    code = lib().normuon_scale(_ptr(O), _dtype_code(O), k, m, _ptr(v), _ptr(rows), beta2, eps, _ptr(out),
                               _ptr(dev_status), _stream(stream))
    _check(code, "normuon_scale")
    return out


def select_rows(M, k: int, norm: int = NORM_L1, ws=None, stream=None):
    import torch
    n, m = M.shape
    idx = torch.empty(k, dtype=torch.int32, device=M.device)
    if ws is None:
        ws = workspace(lib().muon_select_workspace_size(n), M.device)
    code = lib().select_rows(_ptr(M), n, m, k, norm, _ptr(idx), _ptr(ws), ws.numel(), _stream(stream))
    _check(code, "select_rows")
    return idx


def select_rows_noalloc(M, k: int, norm: int = NORM_L1, idx=None, dev_status=None, stream=None):
    """select_rows without a workspace (fixed scratch inside the library; at
    most 65536 rows; calls that overlap on the GPU race). idx may be passed
    in to avoid allocating the output here too."""
    import torch
    n, m = M.shape
    if idx is None:
        idx = torch.empty(k, dtype=torch.int32, device=M.device)
    code = lib().select_rows_noalloc(_ptr(M), n, m, k, norm, _ptr(idx), _ptr(dev_status), _stream(stream))
    _check(code, "select_rows_noalloc")
    return idx


def _matrices(mats):
    arr = (Matrix * max(len(mats), 1))()
    for i, m in enumerate(mats):
        W, M, G = m[0], m[1], m[2]
        v = m[3] if len(m) > 3 else None
        shape = next(t for t in (W, M, G) if t is not None).shape
        arr[i] = Matrix(_ptr(W), _ptr(M), _ptr(G), _ptr(v), shape[0], shape[1])
    return arr


def workspace_size(mats, p: Params) -> int:
    return lib().muon_workspace_size(_matrices(mats), len(mats), C.byref(p))


@dataclass
class Step:
    """A prepared optimizer step: the matrix table and a workspace, reused
    across calls (allocation happens once, in __init__)."""
    mats: list
    params: Params
    ws: object = None
    _table: object = field(default=None, repr=False)

    def __post_init__(self):
        self._table = _matrices(self.mats)
        if self.ws is None:
            n = lib().muon_workspace_size(self._table, len(self.mats), C.byref(self.params))
            if n == 0 and len(self.mats) > 0:
                raise MuonError(ERR_INVALID_ARG, "muon_workspace_size")
            device = self.mats[0][0].device if self.mats else "cuda"
            self.ws = workspace(n, device)

    def __call__(self, stream=None) -> None:
        code = lib().muon_step(self._table, len(self.mats), C.byref(self.params), _ptr(self.ws), self.ws.numel(),
                               _stream(stream))
        _check(code, "muon_step")

    def profiled(self, stream=None) -> StepProfile:
        """Run the step with per-phase CUDA events (synchronises)."""
        prof = StepProfile()
        code = lib().muon_step_profiled(self._table, len(self.mats), C.byref(self.params), _ptr(self.ws),
                                        self.ws.numel(), _stream(stream), C.byref(prof))
        _check(code, "muon_step_profiled")
        return prof

    def timed(self, events, stream=None) -> None:
        """Run the step, recording the five torch.cuda.Event objects in
        `events` (enable_timing=True) at its phase boundaries on the stream:
        start, NS chain start, NS chain end, NorMuon end, update end. Does not
        synchronise."""
        import torch
        ts = stream if stream is not None else torch.cuda.current_stream()
        for e in events:
            if not e.cuda_event:  # torch creates the CUDA event at its first record
                e.record(ts)
        handles = (C.c_void_p * 5)(*[e.cuda_event for e in events])
        code = lib().muon_step_events(self._table, len(self.mats), C.byref(self.params), _ptr(self.ws),
                                      self.ws.numel(), _stream(stream), handles)
        _check(code, "muon_step_events")

    def device_status(self) -> int:
        """Deferred device status of the last step (synchronises)."""
        import torch
        if self.params.dev_status:
            raise RuntimeError("status goes to the caller's dev_status")
        return int(self.ws[:4].view(torch.int32).item())


def _ptrs(ts):
    arr = (C.c_void_p * max(len(ts), 1))()
    for i, t in enumerate(ts):
        arr[i] = _ptr(t)
    return arr


def operand_dtype(p: Params):
    """torch dtype of the orthogonalised rows muon_orthogonalize writes."""
    import torch
    return {F32: torch.float32, BF16: torch.bfloat16, F16: torch.float16}[p.ns.compute]


def momentum(mats, p: Params, stream=None) -> None:
    """M <- mu M + G (M <- M + G for Dion3) on every (W, M, G[, v]) of mats."""
    _check(lib().muon_momentum(_matrices(mats), len(mats), C.byref(p), _stream(stream)), "muon_momentum")


def orthogonalize(mats, p: Params, O, row_scale, selected=None, ws=None, stream=None):
    """Norms / selection, Newton-Schulz and NorMuon on the momentum of mats;
    writes O[i] (rows x cols, operand dtype), row_scale[i] (rows) and, for
    Dion3, selected[i] (rows, int32). Returns the workspace."""
    table = _matrices(mats)
    if ws is None:
        ws = workspace(lib().muon_workspace_size(table, len(mats), C.byref(p)), mats[0][1].device if mats else None)
    code = lib().muon_orthogonalize(table, len(mats), C.byref(p), _ptrs(O), _ptrs(row_scale),
                                    _ptrs(selected) if selected is not None else None, _ptr(ws), ws.numel(),
                                    _stream(stream))
    _check(code, "muon_orthogonalize")
    return ws


def apply_update(mats, p: Params, O, row_scale, selected=None, stream=None) -> None:
    """W -= lr * row_scale * O per row (Dion3: M *= mu on the selected rows)."""
    code = lib().muon_apply_update(_matrices(mats), len(mats), C.byref(p), _ptrs(O), _ptrs(row_scale),
                                   _ptrs(selected) if selected is not None else None, _stream(stream))
    _check(code, "muon_apply_update")


def muon_step(mats, p: Params | None = None, ws=None, stream=None) -> Step:
    """One optimizer step over mats = [(W, M, G[, v]), ...] (fp32 CUDA
    tensors, updated in place). Returns the Step (reusable)."""
    s = Step(list(mats), p or step_params(), ws)
    s(stream)
    return s
