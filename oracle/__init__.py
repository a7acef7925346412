"""ctypes front end of the fp64 CPU oracle (``lf_oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()``
and by the benchmark's CPU-baseline leg, never by the library.  The oracle
is plain C compiled with gcc (with OpenMP across rows when available); it
shares no code with the CUDA path.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lf_oracle.c")
_LIB = os.path.join(_HERE, "liblforacle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/liblforacle.so`` (gcc, -O2, OpenMP)."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    tmp = _LIB + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.lf_oracle_rows.argtypes = [P, P, P, I, I, I, I, I, P, P, I, P, ctypes.c_double,
                                       P, ctypes.c_long, P, I]
        lib.lf_oracle_rows.restype = I
        lib.lf_oracle_fwd.argtypes = [P, P, P, P, I, I, I, I, I, P, P, I, P, ctypes.c_double, I]
        lib.lf_oracle_fwd.restype = I
        lib.lf_oracle_fwd_rand.argtypes = [P, P, P, P, I, I, I, I, I, P, P, I, P, ctypes.c_double, I, P, I]
        lib.lf_oracle_fwd_rand.restype = I
        lib.lf_oracle_key_set.argtypes = [I, I, I, I, P, I, P, P]
        lib.lf_oracle_key_set.restype = I
        lib.lf_oracle_key_total.argtypes = [I, I, I, P, I, P]
        lib.lf_oracle_key_total.restype = ctypes.c_long
        lib.lf_oracle_row_probs.argtypes = [P, P, P, I, I, I, I, I, P, P, I, P, ctypes.c_double,
                                            I, I, I, P, P]
        lib.lf_oracle_row_probs.restype = I
        lib.lf_oracle_max_threads.argtypes = []
        lib.lf_oracle_max_threads.restype = I
        _lib = lib
    return _lib


def _f32(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor (fp32, bf16 or f16): the 16-bit types widen exactly to fp32
        import torch
        x = x.detach().to("cpu", torch.float32).numpy()
    return np.ascontiguousarray(x, dtype=np.float32)


def _i32(x) -> Optional[np.ndarray]:
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(x, dtype=np.int32)


def _u8(x) -> Optional[np.ndarray]:
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(x, dtype=np.uint8)


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _dil(dil, H):
    if dil is None:
        return np.ones(H, dtype=np.int32)
    if isinstance(dil, int):
        return np.full(H, dil, dtype=np.int32)
    return _i32(dil)


def fwd(q, k, v, r: int, dil=None, global_idx=None, key_pad_mask=None, scale: float = None,
        nthreads: int = 0, rand_blocks=None) -> np.ndarray:
    """All rows.  q, k, v: [B, H, T, d]; returns fp64 [B, H, T, d].
    rand_blocks (the BigBird variant): int [B, H, ceil(T / 64), n_rand], the
    random key blocks of every 64-row query block (see lf_oracle.c)."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    B, H, T, d = q.shape
    gi = _i32(global_idx)
    n_global = 0 if gi is None else gi.shape[1]
    pad = _u8(key_pad_mask)
    dl = _dil(dil, H)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = np.empty((B, H, T, d), dtype=np.float64)
    rb = _i32(rand_blocks)
    n_rand = 0
    if rb is not None:
        assert rb.shape[:3] == (B, H, (T + 63) // 64), rb.shape
        n_rand = rb.shape[3]
    st = _load().lf_oracle_fwd_rand(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, T, d, int(r), _ptr(dl),
                                    _ptr(gi), n_global, _ptr(pad), float(scale), int(nthreads),
                                    _ptr(rb) if n_rand else None, n_rand)
    if st != 0:
        raise RuntimeError("oracle failed with status %d" % st)
    return out


def rows(q, k, v, r: int, rows_bhi, dil=None, global_idx=None, key_pad_mask=None,
         scale: float = None, nthreads: int = 0) -> np.ndarray:
    """Sampled rows: rows_bhi int [n, 3] of (b, h, i); returns fp64 [n, d]."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    B, H, T, d = q.shape
    gi = _i32(global_idx)
    n_global = 0 if gi is None else gi.shape[1]
    pad = _u8(key_pad_mask)
    dl = _dil(dil, H)
    rb = _i32(np.asarray(rows_bhi).reshape(-1, 3))
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = np.empty((rb.shape[0], d), dtype=np.float64)
    st = _load().lf_oracle_rows(_ptr(q), _ptr(k), _ptr(v), B, H, T, d, int(r), _ptr(dl), _ptr(gi),
                                n_global, _ptr(pad), float(scale), _ptr(rb), rb.shape[0], _ptr(out),
                                int(nthreads))
    if st != 0:
        raise RuntimeError("oracle failed with status %d" % st)
    return out


def key_set(T: int, r: int, dil: int, i: int, globals_b=None, pad_b=None) -> np.ndarray:
    """Sorted K(i) of one row of one sample."""
    G = _i32(np.asarray([] if globals_b is None else globals_b))
    pad = _u8(pad_b)
    keys = np.empty(T, dtype=np.int32)
    n = _load().lf_oracle_key_set(T, r, dil, i, _ptr(G) if G.size else None, int(G.size),
                                  _ptr(pad), _ptr(keys))
    if n < 0:
        raise RuntimeError("bad arguments")
    return keys[:n].copy()


def key_total(T: int, r: int, dil: int, globals_b=None, pad_b=None) -> int:
    """Sum over rows of |K(i)| for one sample and one head dilation."""
    G = _i32(np.asarray([] if globals_b is None else globals_b))
    pad = _u8(pad_b)
    n = _load().lf_oracle_key_total(T, r, dil, _ptr(G) if G.size else None, int(G.size), _ptr(pad))
    if n < 0:
        raise RuntimeError("bad arguments")
    return int(n)


def row_probs(q, k, v, r: int, b: int, h: int, i: int, dil=None, global_idx=None,
              key_pad_mask=None, scale: float = None):
    """(probs [T], y [d]) of one row; probs holds p_j / l on K(i), 0 elsewhere."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    B, H, T, d = q.shape
    gi = _i32(global_idx)
    n_global = 0 if gi is None else gi.shape[1]
    pad = _u8(key_pad_mask)
    dl = _dil(dil, H)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    probs = np.empty(T, dtype=np.float64)
    y = np.empty(d, dtype=np.float64)
    st = _load().lf_oracle_row_probs(_ptr(q), _ptr(k), _ptr(v), B, H, T, d, int(r), _ptr(dl),
                                     _ptr(gi), n_global, _ptr(pad), float(scale), b, h, i,
                                     _ptr(probs), _ptr(y))
    if st != 0:
        raise RuntimeError("oracle failed with status %d" % st)
    return probs, y


def max_threads() -> int:
    return int(_load().lf_oracle_max_threads())


def bwd(q, k, v, dy, r: int, dil=None, global_idx=None, key_pad_mask=None, scale: float = None):
    """Gradients (dq, dk, dv), fp64 numpy [B, H, T, d], of sum(y * dy) for the
    forward's y.  Follows the forward's definition step by step in fp64 torch
    on the CPU -- the mask view of the "Longformer" note (section "Mask
    View": A = scale Q K^T + M, M = -inf off K(i), y = softmax(A) V) with
    K(i) from this oracle's key_set -- and lets autograd form the gradients.
    Rows with an empty K(i) give y = 0 and no gradient."""
    import torch
    qd, kd, vd, gd = (torch.from_numpy(_f32(x).astype(np.float64)) for x in (q, k, v, dy))
    B, H, T, d = qd.shape
    dl = _dil(dil, H)
    gi = _i32(global_idx)
    pad = _u8(key_pad_mask)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    qd.requires_grad_(True)
    kd.requires_grad_(True)
    vd.requires_grad_(True)
    total = 0.0
    for b in range(B):
        G = None if gi is None else gi[b]
        pb = None if pad is None else pad[b]
        for h in range(H):
            mask = torch.zeros((T, T), dtype=torch.bool)
            for i in range(T):
                mask[i, torch.from_numpy(key_set(T, r, int(dl[h]), i, G, pb).astype(np.int64))] = True
            A = scale * (qd[b, h] @ kd[b, h].T)
            A = torch.where(mask, A, torch.full_like(A, -np.inf))
            has = mask.any(dim=1, keepdim=True)
            P = torch.softmax(torch.where(has, A, torch.zeros_like(A)), dim=1) * has
            y = P @ vd[b, h]
            total = total + (y * gd[b, h]).sum()
    total.backward()
    return qd.grad.numpy(), kd.grad.numpy(), vd.grad.numpy()
