"""ctypes binding of liblfattn (``include/lf_attn.h``): argument marshalling only.

Every step of the forward runs in the library's CUDA kernels.  There is no
fallback: if the shared library is missing or cannot be loaded, the calls
raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "liblfattn.so")

LF_F32, LF_BF16, LF_F16 = 0, 1, 2
STATUS = {0: "LF_OK", 1: "LF_ERR_INVALID_ARG", 2: "LF_ERR_UNSUPPORTED", 3: "LF_ERR_CUDA",
          4: "LF_ERR_NO_MEMORY", 5: "LF_ERR_DEVICE_CHECK", 6: "LF_ERR_SCRATCH_TOO_SMALL"}
EXPORTS = ("lf_attn_fwd", "lf_attn_fwd_rand", "lf_attn_bwd", "lf_attn_rows_partial", "lf_attn_merge_rows",
           "lf_attn_fwd_stages", "lf_attn_fwd_host", "lf_attn_device_status", "lf_attn_strerror",
           "lf_attn_release", "lf_attn_workspace_bytes", "lf_attn_last_launch_count",
           "lf_attn_fwd_static", "lf_attn_band_plan", "lf_attn_test_hooks")

_lib = None


class LfAttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__("%s failed: %s (%s)" % (what, STATUS.get(status, status), strerror(status)))


def load():
    """Load liblfattn.so (built in-tree by build.py); raises if it is absent."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("liblfattn.so is not built (run sparse_long_sequence_fwd_b200/build.py)")
        lib = ctypes.CDLL(LIB_PATH)
        P, I = ctypes.c_void_p, ctypes.c_int
        sig = [P, P, P, P, I, I, I, I, I, P, P, I, P, ctypes.c_float, I, P]
        lib.lf_attn_fwd.argtypes = sig
        lib.lf_attn_fwd.restype = I
        lib.lf_attn_fwd_rand.argtypes = sig[:15] + [P, I, P]
        lib.lf_attn_fwd_rand.restype = I
        lib.lf_attn_bwd.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, P, P, I, P, ctypes.c_float, I, P]
        lib.lf_attn_bwd.restype = I
        lib.lf_attn_rows_partial.argtypes = [P, P, P, I, I, I, I, I, P, ctypes.c_float, I, P, P, P]
        lib.lf_attn_rows_partial.restype = I
        lib.lf_attn_merge_rows.argtypes = [P, P, I, I, I, I, I, P, P, I, I, P]
        lib.lf_attn_merge_rows.restype = I
        lib.lf_attn_fwd_stages.argtypes = sig + [ctypes.c_uint32]
        lib.lf_attn_fwd_stages.restype = I
        lib.lf_attn_fwd_host.argtypes = sig
        lib.lf_attn_fwd_host.restype = I
        lib.lf_attn_device_status.argtypes = [P, ctypes.POINTER(ctypes.c_uint32)]
        lib.lf_attn_device_status.restype = I
        lib.lf_attn_strerror.argtypes = [I]
        lib.lf_attn_strerror.restype = ctypes.c_char_p
        lib.lf_attn_release.argtypes = []
        lib.lf_attn_release.restype = None
        lib.lf_attn_workspace_bytes.argtypes = [I, I, I, I, I, I]
        lib.lf_attn_workspace_bytes.restype = ctypes.c_uint64
        lib.lf_attn_last_launch_count.argtypes = []
        lib.lf_attn_last_launch_count.restype = I
        lib.lf_attn_fwd_static.argtypes = sig
        lib.lf_attn_fwd_static.restype = I
        lib.lf_attn_band_plan.argtypes = [I, I, I, I, P, I, I, P, I]
        lib.lf_attn_band_plan.restype = I
        lib.lf_attn_test_hooks.argtypes = [ctypes.c_uint32, ctypes.c_uint64]
        lib.lf_attn_test_hooks.restype = None

        _lib = lib
    return _lib


def strerror(status: int) -> str:
    try:
        return load().lf_attn_strerror(int(status)).decode()
    except Exception:  # library absent: still format the error
        return STATUS.get(status, "unknown")


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return LF_F32
    if t.dtype == torch.bfloat16:
        return LF_BF16
    if t.dtype == torch.float16:
        return LF_F16
    raise TypeError("q/k/v must be float32, bfloat16 or float16, got %s" % t.dtype)


def _dil_array(dil, H):
    if dil is None:
        return None
    if isinstance(dil, int):
        dil = [dil] * H
    vals = [int(x) for x in (dil.tolist() if hasattr(dil, "tolist") else dil)]
    if len(vals) != H:
        raise ValueError("dil must have H entries")
    return (ctypes.c_int32 * H)(*vals)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check_qkv(q, k, v):
    if q.dim() != 4 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must all be [B, H, T, d]")
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k, v must share a dtype")
    for t in (q, k, v):
        if not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous")


def fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, r: int, dil=None,
        global_idx: Optional[torch.Tensor] = None, key_pad_mask: Optional[torch.Tensor] = None,
        scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
        stream: Optional[torch.cuda.Stream] = None, stages: int = 7,
        rand_blocks: Optional[torch.Tensor] = None) -> torch.Tensor:
    """lf_attn_fwd on CUDA tensors, queued on ``stream`` (default: current stream).

    ``stages`` != 7 calls lf_attn_fwd_stages (per-kernel timing).  ``rand_blocks``
    (int32 [B, H, ceil(T / 64), n_rand], on the device) calls lf_attn_fwd_rand,
    the BigBird variant."""
    _check_qkv(q, k, v)
    B, H, T, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    n_global = 0
    if global_idx is not None:
        if global_idx.dtype != torch.int32 or not global_idx.is_contiguous() or global_idx.dim() != 2:
            raise ValueError("global_idx must be a contiguous int32 [B, n_global] tensor")
        n_global = global_idx.shape[1]
        if n_global == 0:
            global_idx = None
    if key_pad_mask is not None and (key_pad_mask.dtype != torch.uint8 or not key_pad_mask.is_contiguous()):
        raise ValueError("key_pad_mask must be a contiguous uint8 [B, T] tensor")
    if scale is None:
        scale = d ** -0.5
    s = stream if stream is not None else torch.cuda.current_stream(q.device)
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, T, d, int(r), _dil_array(dil, H),
            _ptr(global_idx), n_global, _ptr(key_pad_mask), float(scale), _dtype_code(q),
            ctypes.c_void_p(s.cuda_stream))
    if rand_blocks is not None:
        if rand_blocks.dtype != torch.int32 or not rand_blocks.is_contiguous() or rand_blocks.dim() != 4 or \
                tuple(rand_blocks.shape[:3]) != (B, H, (T + 63) // 64) or stages != 7:
            raise ValueError("rand_blocks must be a contiguous int32 [B, H, ceil(T / 64), n_rand] tensor")
        n_rand = rand_blocks.shape[3]
        st = load().lf_attn_fwd_rand(*args[:15], _ptr(rand_blocks) if n_rand else None, n_rand, args[15])
        if st != 0:
            raise LfAttnError(st, "lf_attn_fwd_rand")
        return out
    if stages == 7:
        st = load().lf_attn_fwd(*args)
    else:
        st = load().lf_attn_fwd_stages(*args, ctypes.c_uint32(stages))
    if st != 0:
        raise LfAttnError(st, "lf_attn_fwd")
    return out


def bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, y: torch.Tensor, dy: torch.Tensor, r: int, dil=None,
        global_idx: Optional[torch.Tensor] = None, key_pad_mask: Optional[torch.Tensor] = None,
        scale: Optional[float] = None, stream: Optional[torch.cuda.Stream] = None):
    """lf_attn_bwd on CUDA tensors: (dq, dk, dv) fp32 [B, H, T, d] for the forward output y and
    its gradient dy."""
    _check_qkv(q, k, v)
    _check_qkv(y, dy, dy)
    if y.shape != q.shape or y.dtype != q.dtype or dy.dtype != q.dtype:
        raise ValueError("y and dy must match q's shape and dtype")
    B, H, T, d = q.shape
    dq, dk, dv = (torch.empty(q.shape, dtype=torch.float32, device=q.device) for _ in range(3))
    n_global = 0 if global_idx is None else global_idx.shape[1]
    if n_global == 0:
        global_idx = None
    if scale is None:
        scale = d ** -0.5
    s = stream if stream is not None else torch.cuda.current_stream(q.device)
    st = load().lf_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(y), _ptr(dy), _ptr(dq), _ptr(dk), _ptr(dv), B, H, T, d,
                            int(r), _dil_array(dil, H), _ptr(global_idx), n_global, _ptr(key_pad_mask), float(scale),
                            _dtype_code(q), ctypes.c_void_p(s.cuda_stream))
    if st != 0:
        raise LfAttnError(st, "lf_attn_bwd")
    return dq, dk, dv


def rows_partial(q_rows: torch.Tensor, k: torch.Tensor, v: torch.Tensor, key_pad_mask: Optional[torch.Tensor],
                 scale: float, stream: Optional[torch.cuda.Stream] = None):
    """lf_attn_rows_partial: (ml fp32 [B, H, n_rows, 2], acc fp32 [B, H, n_rows, d]) of the rows
    q_rows [B, H, n_rows, d] over the keys k, v [B, H, T, d] (CUDA tensors)."""
    _check_qkv(k, k, v)
    B, H, T, d = k.shape
    if q_rows.dim() != 4 or tuple(q_rows.shape[:2]) != (B, H) or q_rows.shape[3] != d or \
            q_rows.dtype != k.dtype or not q_rows.is_contiguous():
        raise ValueError("q_rows must be a contiguous [B, H, n_rows, d] tensor of k's dtype")
    n = q_rows.shape[2]
    ml = torch.empty((B, H, n, 2), dtype=torch.float32, device=k.device)
    acc = torch.empty((B, H, n, d), dtype=torch.float32, device=k.device)
    if key_pad_mask is not None and (key_pad_mask.dtype != torch.uint8 or not key_pad_mask.is_contiguous()):
        raise ValueError("key_pad_mask must be a contiguous uint8 [B, T] tensor")
    s = stream if stream is not None else torch.cuda.current_stream(k.device)
    st = load().lf_attn_rows_partial(_ptr(q_rows), _ptr(k), _ptr(v), B, H, n, T, d, _ptr(key_pad_mask),
                                     float(scale), _dtype_code(k), _ptr(ml), _ptr(acc), ctypes.c_void_p(s.cuda_stream))
    if st != 0:
        raise LfAttnError(st, "lf_attn_rows_partial")
    return ml, acc


def merge_rows(ml: torch.Tensor, acc: torch.Tensor, out_pos: torch.Tensor, out: torch.Tensor,
               stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """lf_attn_merge_rows: ml [P, B, H, n, 2], acc [P, B, H, n, d] (fp32); row a of sample b
    goes to out[b, :, out_pos[b, a]] (skipped where out_pos < 0); out [B, H, T_out, d]."""
    P_, B, H, n, d = acc.shape
    if ml.shape != (P_, B, H, n, 2) or ml.dtype != torch.float32 or acc.dtype != torch.float32 or \
            not (ml.is_contiguous() and acc.is_contiguous()):
        raise ValueError("ml / acc must be contiguous fp32 [P, B, H, n, 2] / [P, B, H, n, d]")
    if out_pos.shape != (B, n) or out_pos.dtype != torch.int32 or not out_pos.is_contiguous():
        raise ValueError("out_pos must be a contiguous int32 [B, n] tensor")
    if not out.is_contiguous() or tuple(out.shape[:2]) != (B, H) or out.shape[3] != d:
        raise ValueError("out must be a contiguous [B, H, T_out, d] tensor")
    s = stream if stream is not None else torch.cuda.current_stream(out.device)
    st = load().lf_attn_merge_rows(_ptr(ml), _ptr(acc), P_, B, H, n, d, _ptr(out_pos), _ptr(out), out.shape[2],
                                   _dtype_code(out), ctypes.c_void_p(s.cuda_stream))
    if st != 0:
        raise LfAttnError(st, "lf_attn_merge_rows")
    return out


def fwd_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, r: int, dil=None,
             global_idx: Optional[torch.Tensor] = None, key_pad_mask: Optional[torch.Tensor] = None,
             scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
             stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """lf_attn_fwd_host on CPU tensors (pinned for full copy bandwidth); returns when ``out`` is ready."""
    _check_qkv(q, k, v)
    B, H, T, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    n_global = 0 if global_idx is None else global_idx.shape[1]
    if n_global == 0:
        global_idx = None
    if scale is None:
        scale = d ** -0.5
    s = stream if stream is not None else torch.cuda.current_stream()
    st = load().lf_attn_fwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, T, d, int(r), _dil_array(dil, H),
                                 _ptr(global_idx), n_global, _ptr(key_pad_mask), float(scale), _dtype_code(q),
                                 ctypes.c_void_p(s.cuda_stream))
    if st != 0:
        raise LfAttnError(st, "lf_attn_fwd_host")
    return out


def fwd_static(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, r: int, dil=None,
               global_idx: Optional[torch.Tensor] = None, key_pad_mask: Optional[torch.Tensor] = None,
               scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
               stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """lf_attn_fwd_static on CUDA tensors: the forward on the library's fixed
    32 MiB scratch array, for callers that cannot allocate device memory
    (graph capture in global mode, fixed budgets, own pool allocators).  Such
    callers pass ``out`` in (otherwise torch allocates it here)."""
    _check_qkv(q, k, v)
    B, H, T, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    n_global = 0 if global_idx is None else global_idx.shape[1]
    if n_global == 0:
        global_idx = None
    if scale is None:
        scale = d ** -0.5
    s = stream if stream is not None else torch.cuda.current_stream(q.device)
    st = load().lf_attn_fwd_static(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, T, d, int(r), _dil_array(dil, H),
                                   _ptr(global_idx), n_global, _ptr(key_pad_mask), float(scale), _dtype_code(q),
                                   ctypes.c_void_p(s.cuda_stream))
    if st != 0:
        raise LfAttnError(st, "lf_attn_fwd_static")
    return out


def device_status(stream: Optional[torch.cuda.Stream] = None):
    """(status, flags): synchronises the stream, reads and clears the device status word."""
    s = stream if stream is not None else torch.cuda.current_stream()
    flags = ctypes.c_uint32(0)
    st = load().lf_attn_device_status(ctypes.c_void_p(s.cuda_stream), ctypes.byref(flags))
    return st, flags.value


def release() -> None:
    load().lf_attn_release()


def workspace_bytes(B, H, T, d, n_global, dtype_code) -> int:
    return int(load().lf_attn_workspace_bytes(B, H, T, d, n_global, dtype_code))


def last_launch_count() -> int:
    return int(load().lf_attn_last_launch_count())


def band_plan(B: int, H: int, T: int, r: int, dil=None, n_global: int = 0, max_ctas: int = 296):
    """The band kernel's split of its work over at most ``max_ctas`` pipelines
    (computed on the host, no device needed): an int32 array [pieces, 10] of
    (pipeline, tile, first block, end block, blocks of the tile, first and
    last pipeline of the tile, partial-state slot, b*H + h, class*65536 + t)."""
    import numpy as np
    d = _dil_array(dil, H)
    n = load().lf_attn_band_plan(B, H, T, int(r), d, int(n_global), int(max_ctas), None, 0)
    if n < 0:
        raise ValueError("lf_attn_band_plan rejected these sizes")
    out = np.zeros((max(n, 1), 10), dtype=np.int32)
    m = load().lf_attn_band_plan(B, H, T, int(r), d, int(n_global), int(max_ctas),
                                 ctypes.c_void_p(out.ctypes.data), n)
    assert m == n
    return out[:n]


def test_hooks(flags: int = 0, wait_ns: int = 0) -> None:
    """Test hook of the band kernel's failure path (see lf_attn_test_hooks)."""
    load().lf_attn_test_hooks(int(flags), int(wait_ns))


def raw_call(name: str, *args) -> int:
    """Calls an entry point with raw arguments (used by the error-path tests)."""
    return getattr(load(), name)(*args)
