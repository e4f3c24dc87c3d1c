"""ctypes binding of libmpq.so (argument marshalling only).

Every step of the solve runs in the library's CUDA kernels; this module only
checks tensor shapes/dtypes/devices, passes raw pointers and the current CUDA
stream, and turns status codes into exceptions.  There is no fallback: if the
shared library is missing, importing this module raises.
"""
from __future__ import annotations

import ctypes as C
import math
import os
from typing import Optional

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmpq.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"libmpq.so not found at {LIB_PATH}; build it with "
        "`python -c 'import __graft_entry__ as g; g.build()'` or "
        "`python post_weight_quantization_row_b200/build.py`")

lib = C.CDLL(LIB_PATH)

STATUS = {0: "MPQ_OK", 1: "MPQ_ERR_INVALID_ARG", 2: "MPQ_ERR_CUDA", 3: "MPQ_ERR_OOM",
          4: "MPQ_ERR_NONFINITE", 5: "MPQ_ERR_RANK", 6: "MPQ_ERR_TIMEOUT",
          7: "MPQ_ERR_UNSUPPORTED"}


class MPQError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str):
        super().__init__(f"{where}: {STATUS.get(status, status)}: {msg}")
        self.status = status


class Params(C.Structure):
    _fields_ = [("d", C.c_int32), ("K", C.c_int32), ("codebook", C.c_void_p),
                ("beta0", C.c_double), ("damping", C.c_double), ("tau", C.c_double),
                ("gamma_lo_rel", C.c_double), ("gamma_hi_rel", C.c_double),
                ("alpha_min", C.c_double), ("alpha_max", C.c_double),
                ("vec_engine", C.c_int32), ("cd_panel", C.c_int32),
                ("group_size", C.c_int32), ("solve_graphs", C.c_int32),
                ("cd_skip_precision", C.c_double),
                ("greedy_init", C.c_int32),
                ("greedy_damp", C.c_double)]


class RowStats(C.Structure):
    _fields_ = [("gamma1", C.c_void_p), ("beta", C.c_void_p), ("clamps", C.c_void_p),
                ("cd_changes", C.c_void_p)]


P = C.c_void_p
I64 = C.c_int64
I32 = C.c_int32
ST = C.c_int


def _sig(name, res, *args):
    f = getattr(lib, name)
    f.restype = res
    f.argtypes = list(args)
    return f


_sig("mpq_params_default", None, C.POINTER(Params), I32, I32)
_sig("mpq_plan_create_from_spectrum", ST, P, P, I64, I64, C.POINTER(Params), P, C.POINTER(P))
_sig("mpq_plan_create_from_x", ST, P, I64, I64, C.POINTER(Params), P, C.POINTER(P))
_sig("mpq_plan_destroy", ST, P)
_sig("mpq_gram_create", ST, I64, P, C.POINTER(P))
_sig("mpq_gram_accumulate", ST, P, P, I64, P)
_sig("mpq_gram_info", ST, P, C.POINTER(I64), C.POINTER(I64))
_sig("mpq_gram_get", ST, P, P, P)
_sig("mpq_gram_destroy", ST, P)
_sig("mpq_plan_create_from_gram", ST, P, C.POINTER(Params), P, C.POINTER(P))
_sig("mpq_rht", ST, P, I64, I64, P, P)
_sig("mpq_plan_info", ST, P, C.POINTER(I64), C.POINTER(I64), C.POINTER(I32), C.POINTER(I32))
_sig("mpq_plan_get_spectrum", ST, P, P, P, P)
_sig("mpq_plan_status", ST, P, P)
_sig("mpq_plan_workspace_bytes", I64, P, I64)
_sig("mpq_plan_set_workspace_cap", ST, P, I64)
_sig("mpq_solve", ST, P, P, I64, P, P, I32, I32, P, P, P, C.POINTER(RowStats), P)
_sig("mpq_solve_host", ST, P, P, I64, I32, I32, P, P, P, P)
_sig("mpq_stage_init", ST, P, P, I64, I32, P, P, P, P, P)
_sig("mpq_stage_denoise", ST, P, P, P, P, P, I64, P, P, P, P, P, P, P)
_sig("mpq_stage_linear", ST, P, P, I64, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P)
_sig("mpq_stage_vamp_scalar", ST, P, P, I64, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P)
_sig("mpq_stage_cd", ST, P, P, I64, P, P, P, I32, P, P)
_sig("mpq_stage_energy", ST, P, P, I64, P, P, P, P, P, P)
_sig("mpq_stage_energy_noalloc", ST, P, P, I64, P, P, P, P, P, P)
_sig("mpq_profile_start", ST)
_sig("mpq_profile_stop", ST, C.c_char_p, I64)
_sig("mpq_last_error", C.c_char_p)
_sig("mpq_kernel_launch_count", I64)

EXPORTED = ["mpq_params_default", "mpq_plan_create_from_spectrum", "mpq_plan_create_from_x",
            "mpq_plan_destroy", "mpq_gram_create", "mpq_gram_accumulate", "mpq_gram_info",
            "mpq_gram_get", "mpq_gram_destroy", "mpq_plan_create_from_gram", "mpq_rht",
            "mpq_plan_info", "mpq_plan_get_spectrum", "mpq_plan_status",
            "mpq_plan_workspace_bytes", "mpq_plan_set_workspace_cap", "mpq_solve",
            "mpq_solve_host", "mpq_stage_init", "mpq_stage_denoise", "mpq_stage_linear",
            "mpq_stage_vamp_scalar",
            "mpq_stage_cd", "mpq_stage_energy", "mpq_stage_energy_noalloc",
            "mpq_profile_start", "mpq_profile_stop",
            "mpq_last_error", "mpq_kernel_launch_count"]


def check(status: int, where: str):
    if status != 0:
        raise MPQError(status, where, lib.mpq_last_error().decode())


def kernel_launch_count() -> int:
    return int(lib.mpq_kernel_launch_count())


def profile_start():
    check(lib.mpq_profile_start(), "mpq_profile_start")


def profile_stop() -> dict:
    """{kernel name: (launches, total ms)} for launches since profile_start."""
    buf = C.create_string_buffer(1 << 16)
    check(lib.mpq_profile_stop(buf, len(buf)), "mpq_profile_stop")
    out = {}
    for line in buf.value.decode().splitlines():
        name, cnt, ms = line.split()
        out[name] = (int(cnt), float(ms))
    return out


def _stream():
    return P(torch.cuda.current_stream().cuda_stream)


def _ptr(t: Optional[torch.Tensor], dtype=None, shape=None, name="tensor"):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return P(t.data_ptr())


def make_params(d: int, K: int, codebook=None, **kw) -> tuple:
    p = Params()
    lib.mpq_params_default(C.byref(p), d, K)
    keep = None
    if codebook is not None:
        cb = np.ascontiguousarray(np.asarray(codebook, dtype=np.float32))
        if cb.shape != (K, d):
            raise ValueError(f"codebook must be {K} x {d}")
        keep = cb
        p.codebook = cb.ctypes.data
    for k, v in kw.items():
        if not hasattr(p, k):
            raise ValueError(f"unknown parameter {k}")
        setattr(p, k, v)
    return p, keep


class Gram:
    """Streamed calibration: G = sum over chunks of X_c^T X_c (n x n, fp64, on
    the device); Plan.from_gram takes the spectrum from it."""

    def __init__(self, n: int):
        self._h = P()
        check(lib.mpq_gram_create(int(n), _stream(), C.byref(self._h)), "mpq_gram_create")
        self.n = int(n)

    def accumulate(self, X: torch.Tensor):
        if X.dim() != 2 or X.shape[1] != self.n:
            raise ValueError(f"X must be rows x {self.n}")
        check(lib.mpq_gram_accumulate(self._h, _ptr(X, torch.float32, name="X"), X.shape[0],
                                      _stream()), "mpq_gram_accumulate")
        return self

    @property
    def rows(self) -> int:
        n, r = I64(), I64()
        check(lib.mpq_gram_info(self._h, C.byref(n), C.byref(r)), "mpq_gram_info")
        return r.value

    def matrix(self) -> torch.Tensor:
        G = torch.empty((self.n, self.n), dtype=torch.float64, device="cuda")
        check(lib.mpq_gram_get(self._h, _ptr(G), _stream()), "mpq_gram_get")
        return G

    def close(self):
        if self._h is not None and self._h.value:
            lib.mpq_gram_destroy(self._h)
        self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def rht(X: torch.Tensor, signs: torch.Tensor) -> torch.Tensor:
    """In place: every row x of X becomes (x .* signs) H_n / sqrt(n)."""
    if X.dim() != 2:
        raise ValueError("X must be 2-D")
    rows, n = X.shape
    check(lib.mpq_rht(_ptr(X, torch.float32, name="X"), rows, n,
                      _ptr(signs, torch.float32, (n,), name="signs"), _stream()), "mpq_rht")
    return X


class Plan:
    """A solver plan: the spectrum of X and the codebook tables, on one GPU."""

    def __init__(self, handle, group_size: int = 0):
        self._h = P(handle)
        n, r, d, K = I64(), I64(), I32(), I32()
        check(lib.mpq_plan_info(self._h, C.byref(n), C.byref(r), C.byref(d), C.byref(K)), "info")
        self.n, self.r, self.d, self.K = n.value, r.value, d.value, K.value
        self.B = self.n // self.d
        self.G = int(group_size)                      # scalar grid group (0: per row)
        self.ng = self.n // self.G if self.G else 1   # grids per row
        self.device = torch.cuda.current_device()

    def _sshape(self, m):
        """Shape of a scale/offset array for m rows."""
        return (m,) if self.ng == 1 else (m, self.ng)

    # ------------------------------------------------------------ creation --
    @classmethod
    def from_spectrum(cls, s: torch.Tensor, V: torch.Tensor, d: int, K: int, codebook=None, **kw):
        if s.dtype != torch.float64 or V.dtype != torch.float64:
            raise ValueError("s and V must be float64")
        n, r = V.shape
        if s.shape != (r,):
            raise ValueError("s must have shape (r,)")
        prm, keep = make_params(d, K, codebook, **kw)
        h = P()
        check(lib.mpq_plan_create_from_spectrum(_ptr(s, name="s"), _ptr(V, name="V"), n, r,
                                                C.byref(prm), _stream(), C.byref(h)),
              "mpq_plan_create_from_spectrum")
        del keep
        return cls(h.value, kw.get("group_size", 0))

    @classmethod
    def from_x(cls, X: torch.Tensor, d: int, K: int, codebook=None, **kw):
        m, n = X.shape
        prm, keep = make_params(d, K, codebook, **kw)
        h = P()
        check(lib.mpq_plan_create_from_x(_ptr(X, torch.float32, name="X"), m, n, C.byref(prm),
                                         _stream(), C.byref(h)), "mpq_plan_create_from_x")
        del keep
        return cls(h.value, kw.get("group_size", 0))

    @classmethod
    def from_gram(cls, gram: "Gram", d: int, K: int, codebook=None, **kw):
        prm, keep = make_params(d, K, codebook, **kw)
        h = P()
        check(lib.mpq_plan_create_from_gram(gram._h, C.byref(prm), _stream(), C.byref(h)),
              "mpq_plan_create_from_gram")
        del keep
        return cls(h.value, kw.get("group_size", 0))

    def close(self):
        if self._h is not None and self._h.value:
            lib.mpq_plan_destroy(self._h)
        self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    # --------------------------------------------------------------- misc --
    def spectrum(self):
        s = torch.empty(self.r, dtype=torch.float64, device="cuda")
        V = torch.empty(self.n, self.r, dtype=torch.float64, device="cuda")
        check(lib.mpq_plan_get_spectrum(self._h, _ptr(s), _ptr(V), _stream()), "get_spectrum")
        torch.cuda.current_stream().synchronize()
        return s, V

    def status(self):
        check(lib.mpq_plan_status(self._h, _stream()), "mpq_plan_status")

    def workspace_bytes(self, m: int) -> int:
        return int(lib.mpq_plan_workspace_bytes(self._h, m))

    def set_workspace_cap(self, cap: int):
        check(lib.mpq_plan_set_workspace_cap(self._h, cap), "set_workspace_cap")

    # -------------------------------------------------------------- solve --
    def solve(self, W: torch.Tensor, T_vamp: int, cd_sweeps: int, row_scale=None,
              row_offset=None, stats: bool = False, check_status: bool = True, out=None):
        m = W.shape[0]
        _ptr(W, torch.float32, (m, self.n), "W")
        dev = W.device
        if out is None:
            out = {"idx": torch.empty(m, self.B, dtype=torch.int16, device=dev),
                   "w_hat": torch.empty(m, self.n, dtype=torch.float32, device=dev),
                   "energy": torch.empty(m, dtype=torch.float32, device=dev)}
        st = None
        if stats:
            out["gamma1"] = torch.empty(m, dtype=torch.float64, device=dev)
            out["beta"] = torch.empty(m, dtype=torch.float64, device=dev)
            out["clamps"] = torch.empty(m, dtype=torch.int32, device=dev)
            out["cd_changes"] = torch.zeros(m, max(cd_sweeps, 1), dtype=torch.int32, device=dev)
            st = RowStats(out["gamma1"].data_ptr(), out["beta"].data_ptr(),
                          out["clamps"].data_ptr(), out["cd_changes"].data_ptr())
        check(lib.mpq_solve(self._h, _ptr(W), m, _ptr(row_scale, torch.float32, self._sshape(m), "row_scale"),
                            _ptr(row_offset, torch.float32, self._sshape(m), "row_offset"), T_vamp, cd_sweeps,
                            _ptr(out["idx"], torch.int16, (m, self.B), "idx"),
                            _ptr(out.get("w_hat"), torch.float32, None, "w_hat"),
                            _ptr(out.get("energy"), torch.float32, None, "energy"),
                            C.byref(st) if st is not None else None, _stream()), "mpq_solve")
        if check_status:
            self.status()
        return out

    def solve_host(self, W: torch.Tensor, T_vamp: int, cd_sweeps: int, out=None):
        """W: CPU float32 tensor (pinned for fast copies); results on the CPU."""
        if W.is_cuda or W.dtype != torch.float32 or not W.is_contiguous():
            raise ValueError("W must be a contiguous CPU float32 tensor")
        m = W.shape[0]
        if out is None:
            pin = W.is_pinned()
            out = {"idx": torch.empty(m, self.B, dtype=torch.int16, pin_memory=pin),
                   "w_hat": torch.empty(m, self.n, dtype=torch.float32, pin_memory=pin),
                   "energy": torch.empty(m, dtype=torch.float32, pin_memory=pin)}
        check(lib.mpq_solve_host(self._h, P(W.data_ptr()), m, T_vamp, cd_sweeps,
                                 P(out["idx"].data_ptr()), P(out["w_hat"].data_ptr()),
                                 P(out["energy"].data_ptr()), _stream()), "mpq_solve_host")
        return out

    # ------------------------------------------------------------- stages --
    def stage_init(self, W, scale=None, offset=None):
        m = W.shape[0]
        dev = W.device
        given = scale is not None
        if given:
            scale = scale.clone()
            offset = offset.clone()
        else:
            scale = torch.empty(self._sshape(m), dtype=torch.float32, device=dev)
            offset = torch.empty(self._sshape(m), dtype=torch.float32, device=dev)
        idx = torch.empty(m, self.B, dtype=torch.int16, device=dev)
        g0 = torch.empty(m, dtype=torch.float64, device=dev)
        check(lib.mpq_stage_init(self._h, _ptr(W, torch.float32, (m, self.n), "W"), m, int(given),
                                 _ptr(scale), _ptr(offset), _ptr(idx), _ptr(g0), _stream()),
              "mpq_stage_init")
        return {"scale": scale, "offset": offset, "idx": idx, "gamma1_0": g0}

    def stage_denoise(self, R1, gamma1, scale, offset, W=None, gamma1_0=None):
        m = R1.shape[0]
        dev = R1.device
        xhat = torch.empty(m, self.n, dtype=torch.float32, device=dev)
        vblock = torch.empty(m, self.B, dtype=torch.float32, device=dev)
        vsum = torch.empty(m, dtype=torch.float64, device=dev)
        idx = torch.empty(m, self.B, dtype=torch.int16, device=dev)
        check(lib.mpq_stage_denoise(self._h, _ptr(R1, torch.float32, (m, self.n), "R1"),
                                    _ptr(gamma1, torch.float64, (m,), "gamma1"),
                                    _ptr(scale, torch.float32, self._sshape(m), "scale"),
                                    _ptr(offset, torch.float32, self._sshape(m), "offset"), m,
                                    _ptr(W, torch.float32, None, "W"),
                                    _ptr(gamma1_0, torch.float64, None, "gamma1_0"), _ptr(xhat),
                                    _ptr(vblock), _ptr(vsum), _ptr(idx), _stream()),
              "mpq_stage_denoise")
        return {"xhat": xhat, "vblock": vblock, "vsum": vsum, "idx": idx}

    def stage_linear(self, W, R1, gamma1, xhat1, vsum, gamma1_0, beta):
        m = W.shape[0]
        dev = W.device
        beta = beta.clone()
        o = {"R1": torch.empty(m, self.n, dtype=torch.float32, device=dev),
             "gamma1": torch.empty(m, dtype=torch.float64, device=dev),
             "R2": torch.empty(m, self.n, dtype=torch.float32, device=dev),
             "gamma2": torch.empty(m, dtype=torch.float64, device=dev),
             "Uprime": torch.empty(m, self.r, dtype=torch.float32, device=dev),
             "xhat2": torch.empty(m, self.n, dtype=torch.float32, device=dev),
             "alpha2": torch.empty(m, dtype=torch.float64, device=dev),
             "beta_hat": torch.empty(m, dtype=torch.float64, device=dev),
             "clamps": torch.zeros(m, dtype=torch.int32, device=dev)}
        check(lib.mpq_stage_linear(self._h, _ptr(W, torch.float32, (m, self.n), "W"), m,
                                   _ptr(R1, torch.float32, (m, self.n), "R1"),
                                   _ptr(gamma1, torch.float64, (m,), "gamma1"),
                                   _ptr(xhat1, torch.float32, (m, self.n), "xhat1"),
                                   _ptr(vsum, torch.float64, (m,), "vsum"),
                                   _ptr(gamma1_0, torch.float64, (m,), "gamma1_0"), _ptr(beta),
                                   _ptr(o["R1"]), _ptr(o["gamma1"]), _ptr(o["R2"]),
                                   _ptr(o["gamma2"]), _ptr(o["Uprime"]), _ptr(o["xhat2"]),
                                   _ptr(o["alpha2"]), _ptr(o["beta_hat"]), _ptr(o["clamps"]),
                                   _stream()), "mpq_stage_linear")
        o["beta"] = beta
        return o

    def stage_vamp_scalar(self, W, scale, offset, R1, gamma1, gamma1_0, beta, next_pass=True,
                          map_pass=True):
        """mpq_stage_vamp_scalar: one iteration of the fused scalar row kernel
        and the linear module on an injected cavity (R1, gamma1)."""
        m = W.shape[0]
        dev = W.device
        beta = beta.clone()
        f32 = lambda *sh: torch.empty(*sh, dtype=torch.float32, device=dev)
        f64 = lambda *sh: torch.empty(*sh, dtype=torch.float64, device=dev)
        o = {"R2": f32(m, self.n), "gamma2": f64(m), "gamma1": f64(m),
             "clamps": torch.zeros(m, dtype=torch.int32, device=dev)}
        if map_pass:
            o["idx"] = torch.empty(m, self.n, dtype=torch.int16, device=dev)
        if next_pass:
            o.update({"R1": f32(m, self.n), "R2_next": f32(m, self.n), "gamma2_next": f64(m)})
        check(lib.mpq_stage_vamp_scalar(
            self._h, _ptr(W, torch.float32, (m, self.n), "W"), m,
            _ptr(scale, torch.float32, self._sshape(m), "scale"),
            _ptr(offset, torch.float32, self._sshape(m), "offset"),
            _ptr(R1, torch.float32, (m, self.n), "R1"), _ptr(gamma1, torch.float64, (m,), "gamma1"),
            _ptr(gamma1_0, torch.float64, (m,), "gamma1_0"), _ptr(beta), _ptr(o["R2"]),
            _ptr(o["gamma2"]), _ptr(o.get("R1")), _ptr(o["gamma1"]), _ptr(o.get("idx")),
            _ptr(o.get("R2_next")), _ptr(o.get("gamma2_next")), _ptr(o["clamps"]), _stream()),
            "mpq_stage_vamp_scalar")
        o["beta"] = beta
        return o

    def stage_cd(self, W, scale, offset, idx, sweeps: int):
        m = W.shape[0]
        idx = idx.clone()
        changes = torch.zeros(m, max(sweeps, 1), dtype=torch.int32, device=W.device)
        check(lib.mpq_stage_cd(self._h, _ptr(W, torch.float32, (m, self.n), "W"), m,
                               _ptr(scale, torch.float32, self._sshape(m), "scale"),
                               _ptr(offset, torch.float32, self._sshape(m), "offset"),
                               _ptr(idx, torch.int16, (m, self.B), "idx"), sweeps, _ptr(changes),
                               _stream()), "mpq_stage_cd")
        return {"idx": idx, "changes": changes}

    def stage_energy(self, W, scale, offset, idx):
        m = W.shape[0]
        w_hat = torch.empty(m, self.n, dtype=torch.float32, device=W.device)
        energy = torch.empty(m, dtype=torch.float32, device=W.device)
        check(lib.mpq_stage_energy(self._h, _ptr(W, torch.float32, (m, self.n), "W"), m,
                                   _ptr(scale, torch.float32, self._sshape(m), "scale"),
                                   _ptr(offset, torch.float32, self._sshape(m), "offset"),
                                   _ptr(idx, torch.int16, (m, self.B), "idx"), _ptr(w_hat),
                                   _ptr(energy), _stream()), "mpq_stage_energy")
        return {"w_hat": w_hat, "energy": energy}


    def stage_energy_noalloc(self, W, scale, offset, idx, w_hat=None, energy=None):
        """mpq_stage_energy_noalloc: the energy stage without any allocation in
        the library (its scratch is a static device array).  Output tensors
        are allocated here by the caller side unless given."""
        m = W.shape[0]
        if w_hat is None:
            w_hat = torch.empty(m, self.n, dtype=torch.float32, device=W.device)
        if energy is None:
            energy = torch.empty(m, dtype=torch.float32, device=W.device)
        check(lib.mpq_stage_energy_noalloc(self._h, _ptr(W, torch.float32, (m, self.n), "W"), m,
                                           _ptr(scale, torch.float32, self._sshape(m), "scale"),
                                           _ptr(offset, torch.float32, self._sshape(m), "offset"),
                                           _ptr(idx, torch.int16, (m, self.B), "idx"),
                                           _ptr(w_hat), _ptr(energy), _stream()),
              "mpq_stage_energy_noalloc")
        return {"w_hat": w_hat, "energy": energy}


NOALLOC_SCRATCH_BYTES = 16 << 20


def idx_to_numpy(idx: torch.Tensor) -> np.ndarray:
    """uint16 codeword indices stored in an int16 tensor -> int64 numpy."""
    return idx.cpu().numpy().view(np.uint16).astype(np.int64)
