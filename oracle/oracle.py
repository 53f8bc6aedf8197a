"""fp64 CPU oracle for causal alpha-entmax attention -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` import this
module.  The CUDA library never does, and this module imports nothing from it.

The arithmetic lives in ``entmax_oracle.c`` (plain C, fp64, OpenMP over rows); this file only
compiles it with gcc on first use and marshals numpy arrays through ctypes.  What it computes,
with the passages it follows, is described at the top of that file:

* ``entmax_vec``          -- exact alpha-entmax of one vector (tau by sort + closed form / root).
* ``tau_halley``          -- the fixed-iteration bracketed Halley + bisection search for tau
                             ("Triton Entmax (Optimized Entmax Activation)" section of the AdaSplash
                             page), in fp64.
* ``attention_rows``      -- tau, output rows and per-key-tile max p for chosen query rows of an
                             attention problem ("AdaSplash with Block Masking", "Variable Length
                             Sequences", "Causal and Non-causal Masking").
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "entmax_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libentmax_oracle.so")
TILE = 128  # edge of the query and key tiles of the block mask

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (fp64, OpenMP, no fast-math).  Returns the .so path."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    os.makedirs(_BUILD_DIR, exist_ok=True)
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
           "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    dp = ctypes.POINTER(ctypes.c_double)
    lib.oracle_entmax_vec.argtypes = [dp, ctypes.c_int, ctypes.c_double, ctypes.c_int, dp, dp]
    lib.oracle_entmax_vec.restype = ctypes.c_int
    lib.oracle_tau_halley.argtypes = [dp, ctypes.c_int, ctypes.c_double, ctypes.c_int]
    lib.oracle_tau_halley.restype = ctypes.c_double
    lib.oracle_entmax_attn_rows.argtypes = [
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        ctypes.c_double, ctypes.c_int, ctypes.c_void_p, ctypes.c_int,
        ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int]
    lib.oracle_entmax_attn_rows.restype = ctypes.c_int
    lib.oracle_max_threads.argtypes = []
    lib.oracle_max_threads.restype = ctypes.c_int
    _lib = lib
    return lib


def host_threads() -> int:
    """Threads the oracle uses by default: every core this process may run on."""
    return len(os.sched_getaffinity(0))


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def alpha_as_float32(alpha: float) -> float:
    """alpha as the fp32 value both sides compute with (1.333 is taken literally)."""
    return float(np.float32(alpha))


def entmax_vec(z, alpha: float, force_general: bool = False):
    """Exact alpha-entmax of a 1-D vector z.  Returns (p, tau) in fp64."""
    z = _f64(z).ravel()
    p = np.empty_like(z)
    tau = ctypes.c_double()
    rc = _load().oracle_entmax_vec(z.ctypes.data_as(ctypes.POINTER(ctypes.c_double)), z.size,
                                   float(alpha), int(force_general),
                                   p.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
                                   ctypes.byref(tau))
    if rc != 0:
        raise ValueError(f"oracle_entmax_vec failed ({rc})")
    return p, tau.value


def tau_halley(z, alpha: float, n_iter: int) -> float:
    """tau after n_iter steps of the bracketed Halley + bisection search, fp64."""
    z = _f64(z).ravel()
    return _load().oracle_tau_halley(z.ctypes.data_as(ctypes.POINTER(ctypes.c_double)), z.size,
                                     float(alpha), int(n_iter))


def _as_f32(x) -> np.ndarray:
    """Exact fp32 copy of a numpy array or torch tensor (bf16 widens exactly)."""
    if hasattr(x, "detach"):  # torch tensor, without importing torch here
        x = x.detach().cpu().float().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def attention_rows(q, k, v, alpha: float, causal: bool = True, cu_seqlens=None, rows=None,
                   tau_given=None, want_out: bool = True, want_maxp: bool = True,
                   nthreads: int | None = None):
    """Oracle forward for selected query rows.

    q: [B, Hq, T, d] (fixed length) or [Hq, T, d] (varlen with cu_seqlens); k, v likewise with
    Hkv heads.  rows: flat row ids ((b*Hq + h)*T + t, or h*T + t for varlen); None = all rows.
    alpha is used exactly as given (callers pass the fp32-rounded value).
    Returns dict(rows, tau [n], out [n, d] or None, maxp [n, nKt] or None, nkt).
    """
    qf, kf, vf = _as_f32(q), _as_f32(k), _as_f32(v)
    if cu_seqlens is None:
        B, Hq, T, d = qf.shape
        Hkv = kf.shape[1]
        cu = None
        nseq = 0
        longest = T
        total_rows = B * Hq * T
    else:
        Hq, T, d = qf.shape
        Hkv = kf.shape[0]
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
        nseq = cu.size - 1
        B = nseq
        longest = int(np.max(np.diff(cu)))
        total_rows = Hq * T
    if rows is None:
        rows = np.arange(total_rows, dtype=np.int64)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    n = rows.size
    nkt = (longest + TILE - 1) // TILE
    tau = np.empty(n, dtype=np.float64)
    out = np.empty((n, d), dtype=np.float64) if want_out else None
    maxp = np.empty((n, nkt), dtype=np.float64) if want_maxp else None
    tg = None if tau_given is None else _f64(tau_given).ravel()
    if tg is not None and tg.size != n:
        raise ValueError("tau_given must have one entry per row")
    rc = _load().oracle_entmax_attn_rows(
        _ptr(qf), _ptr(kf), _ptr(vf), B, Hq, Hkv, T, d, float(alpha), int(bool(causal)),
        _ptr(cu), nseq, _ptr(rows), n, _ptr(tg), _ptr(tau), _ptr(out), _ptr(maxp), nkt,
        int(nthreads or host_threads()))
    if rc != 0:
        raise ValueError(f"oracle_entmax_attn_rows failed ({rc})")
    return {"rows": rows, "tau": tau, "out": out, "maxp": maxp, "nkt": nkt}
