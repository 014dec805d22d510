"""ctypes front end of the C oracle (``gdn_oracle.c``).  TEST INFRASTRUCTURE.

``build()`` compiles ``gdn_oracle.c`` (double) and ``gdn_oracle_ld.c`` (long
double) with gcc into ``liboracle.so`` beside this file, when the library is
missing or older than its sources.  ``oracle_fwd`` / ``oracle_bidir`` take
numpy arrays in the library's layouts (q, k [B,T,H,Dk]; v [B,T,H,Dv];
g, beta [B,T,H]; state [B,H,Dk,Dv]) and return ``(out, state_out)`` in fp64
(or long double with ``precision="long double"``).

The recurrence itself lives in the C file; see its header for the definition
and for the passages of the pages it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SOURCES = [os.path.join(_HERE, "gdn_oracle.c"), os.path.join(_HERE, "gdn_oracle_ld.c")]
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O3, no fast-math) if it is stale."""
    stale = force or not os.path.exists(_LIB_PATH)
    if not stale:
        lib_mtime = os.path.getmtime(_LIB_PATH)
        stale = any(os.path.getmtime(s) > lib_mtime for s in _SOURCES)
    if stale:
        tmp = _LIB_PATH + ".tmp.%d" % os.getpid()
        cmd = ["gcc", "-O3", "-std=c11", "-D_GNU_SOURCE", "-fPIC", "-shared",
               "-o", tmp, _SOURCES[0], _SOURCES[1], "-lpthread", "-lm"]
        subprocess.run(cmd, check=True, cwd=_HERE)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        fp = ctypes.POINTER(ctypes.c_float)
        for suffix, real in (("", ctypes.c_double), ("_ld", ctypes.c_longdouble)):
            rp = ctypes.POINTER(real)
            for name in ("gdn_oracle_fwd", "gdn_oracle_bidir", "gdn_oracle_fwd_logits",
                         "gdn_oracle_bidir_logits"):
                fn = getattr(lib, name + suffix)
                fn.restype = ctypes.c_int
                fn.argtypes = [fp, fp, fp, fp, fp, rp, rp, rp] + [ctypes.c_int] * 6
        lib.gdn_oracle_online_cores.restype = ctypes.c_int
        _lib = lib
    return _lib


def online_cores() -> int:
    """Host cores the oracle's thread pool uses by default."""
    return int(_load().gdn_oracle_online_cores())


def _f32(x, shape, name):
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    if a.shape != shape:
        raise ValueError(f"{name}: expected shape {shape}, got {a.shape}")
    return a


def _run(bidir, q, k, v, g, beta, state_in, nthreads, precision, logits=False):
    q = np.asarray(q)
    B, T, H, Dk = q.shape
    Dv = np.asarray(v).shape[-1]
    q = _f32(q, (B, T, H, Dk), "q")
    k = _f32(k, (B, T, H, Dk), "k")
    v = _f32(v, (B, T, H, Dv), "v")
    g = _f32(g, (B, T, H), "g")
    beta = _f32(beta, (B, T, H), "beta")
    if precision == "double":
        real_np, real_c, suffix = np.float64, ctypes.c_double, ""
    elif precision == "long double":
        real_np, real_c, suffix = np.longdouble, ctypes.c_longdouble, "_ld"
    else:
        raise ValueError("precision must be 'double' or 'long double'")
    if state_in is not None:
        s_in = np.ascontiguousarray(np.asarray(state_in, dtype=real_np))
        if s_in.shape != (B, H, Dk, Dv):
            raise ValueError(f"state_in: expected {(B, H, Dk, Dv)}, got {s_in.shape}")
    else:
        s_in = None
    s_out = np.zeros((B, H, Dk, Dv), dtype=real_np)
    out = np.zeros((B, T, H, Dv), dtype=real_np)
    lib = _load()
    name = ("gdn_oracle_bidir" if bidir else "gdn_oracle_fwd") + ("_logits" if logits else "")
    fn = getattr(lib, name + suffix)
    fp = ctypes.POINTER(ctypes.c_float)
    rp = ctypes.POINTER(real_c)
    rc = fn(q.ctypes.data_as(fp), k.ctypes.data_as(fp), v.ctypes.data_as(fp),
            g.ctypes.data_as(fp), beta.ctypes.data_as(fp),
            s_in.ctypes.data_as(rp) if s_in is not None else None,
            s_out.ctypes.data_as(rp), out.ctypes.data_as(rp),
            B, T, H, Dk, Dv, int(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle returned {rc}")
    return out, s_out


def oracle_fwd(q, k, v, g, beta, state_in=None, nthreads=0, precision="double"):
    """Forward (causal) scan from ``state_in`` (None = zero state)."""
    return _run(False, q, k, v, g, beta, state_in, nthreads, precision)


def oracle_bidir(q, k, v, g, beta, state_in=None, nthreads=0, precision="double"):
    """Forward scan from ``state_in`` plus reverse scan from zero, summed;
    the state returned is the forward scan's."""
    return _run(True, q, k, v, g, beta, state_in, nthreads, precision)


def oracle_fwd_logits(q, k, v, g_logit, beta_logit, state_in=None, nthreads=0,
                      precision="double"):
    """Forward scan whose gates come from the gate layer's logits:
    g = -softplus(g_logit), beta = sigmoid(beta_logit), both evaluated in the
    oracle's precision (``gdn_oracle.c``, gate-logit mode)."""
    return _run(False, q, k, v, g_logit, beta_logit, state_in, nthreads, precision, logits=True)


def oracle_bidir_logits(q, k, v, g_logit, beta_logit, state_in=None, nthreads=0,
                        precision="double"):
    """Bidirectional scan with gates from logits (as ``oracle_fwd_logits``)."""
    return _run(True, q, k, v, g_logit, beta_logit, state_in, nthreads, precision, logits=True)
