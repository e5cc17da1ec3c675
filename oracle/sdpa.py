"""ctypes front end of the fp64 attention oracle (``sdpa_oracle.c``).

TEST INFRASTRUCTURE ONLY (see the package docstring).

Inputs are widened exactly to float64 before the call, so the oracle sees the
same rounded bf16/fp32 values the device sees.  Layouts follow the two forms of
the pages:

  * dense  -- "Core 注意力", example section: q ``[B, Hq, Lq, Dqk]``,
    k ``[B, Hkv, Lk, Dqk]``, v ``[B, Hkv, Lk, Dv]``, out ``[B, Hq, Lq, Dv]``;
  * packed -- "MLA Prefill", parameter table: q ``[nTokens, headNum, Dqk]``,
    qRope ``[nTokens, headNum, 64]``, k/kRope/v ``[sum kv, kvHeadNum, *]``,
    ``qSeqLen``/``kvSeqLen`` int32 ``[batch]``, attenOut ``[nTokens, headNum, Dv]``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_BUILD = os.path.join(_HERE, "_build")
_SRC = os.path.join(_HERE, "sdpa_oracle.c")

MASK_KINDS = {"none": 0, "causal": 1, "keep": 2, "add": 3}


class _Tensor(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("sb", ctypes.c_int64),
                ("sh", ctypes.c_int64), ("si", ctypes.c_int64)]


class _Args(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("head_num", ctypes.c_int32), ("kv_head_num", ctypes.c_int32),
        ("dqk", ctypes.c_int32), ("drope", ctypes.c_int32), ("dv", ctypes.c_int32),
        ("varlen", ctypes.c_int32),
        ("lq", ctypes.c_int64), ("lk", ctypes.c_int64),
        ("q_seqlen", ctypes.c_void_p), ("kv_seqlen", ctypes.c_void_p),
        ("q", _Tensor), ("qrope", _Tensor), ("k", _Tensor), ("krope", _Tensor), ("v", _Tensor),
        ("out", ctypes.c_void_p), ("out_t", _Tensor),
        ("mask_kind", ctypes.c_int32),
        ("keep", ctypes.c_void_p), ("add", ctypes.c_void_p),
        ("mb", ctypes.c_int64), ("mh", ctypes.c_int64), ("mi", ctypes.c_int64), ("mj", ctypes.c_int64),
        ("qk_scale", ctypes.c_double),
        ("lse", ctypes.c_void_p), ("lse_ld", ctypes.c_int64),
    ]


_libs: dict[int, ctypes.CDLL] = {}
_lock = threading.Lock()


def _lib_path(plant: int) -> str:
    return os.path.join(_BUILD, "liboracle.so" if plant == 0 else f"liboracle_plant{plant}.so")


def build_oracle(plant: int = 0, force: bool = False) -> str:
    """Compile the oracle with gcc (OpenMP).  ``plant`` > 0 builds a copy with one
    deliberately planted mistake, used only by the pin-strength tests."""
    os.makedirs(_BUILD, exist_ok=True)
    out = _lib_path(plant)
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(_SRC):
        tmp = out + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11", _SRC, "-o", tmp, "-lm"]
        if plant:
            cmd.insert(1, f"-DORACLE_PLANT={plant}")
        subprocess.run(cmd, check=True)
        os.replace(tmp, out)
    return out


def _load(plant: int = 0) -> ctypes.CDLL:
    with _lock:
        if plant not in _libs:
            lib = ctypes.CDLL(build_oracle(plant))
            lib.ora_sdpa_fwd.argtypes = [ctypes.POINTER(_Args)]
            lib.ora_sdpa_fwd.restype = ctypes.c_int
            lib.ora_sdpa_fwd_rows.argtypes = [ctypes.POINTER(_Args), ctypes.c_void_p, ctypes.c_int64,
                                              ctypes.c_void_p, ctypes.c_void_p]
            lib.ora_sdpa_fwd_rows.restype = ctypes.c_int
            lib.ora_num_threads.restype = ctypes.c_int
            _libs[plant] = lib
        return _libs[plant]


def oracle_threads() -> int:
    """OpenMP threads the oracle runs with on this host."""
    return int(_load().ora_num_threads())


def _f64(x) -> np.ndarray:
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: widen exactly on the CPU
        import torch
        x = x.detach().to("cpu")
        if x.dtype in (torch.bfloat16, torch.float16):
            x = x.to(torch.float32)
        x = x.numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _i32(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _tensor(a: np.ndarray, varlen: bool) -> _Tensor:
    es = a.itemsize
    if varlen:      # [T, H, D]
        return _Tensor(a.ctypes.data, 0, a.strides[1] // es, a.strides[0] // es)
    return _Tensor(a.ctypes.data, a.strides[0] // es, a.strides[1] // es, a.strides[2] // es)


def _prepare(q, k, v, qrope, krope, q_seqlen, kv_seqlen, mask, mask_kind,
             head_num, kv_head_num, qk_scale, full_out=True):
    keep_alive = []
    q, k, v = _f64(q), _f64(k), _f64(v)
    qrope, krope = _f64(qrope), _f64(krope)
    if (qrope is None) != (krope is None):
        raise ValueError("qRope and kRope come together")
    varlen = q_seqlen is not None
    if varlen != (kv_seqlen is not None):
        raise ValueError("qSeqLen and kvSeqLen come together")
    kind = MASK_KINDS[mask_kind]
    a = _Args()
    a.head_num, a.kv_head_num = int(head_num), int(kv_head_num)
    a.dqk, a.dv = q.shape[-1], v.shape[-1]
    a.drope = 0 if qrope is None else qrope.shape[-1]
    a.varlen = int(varlen)
    a.qk_scale = float(qk_scale)
    a.mask_kind = kind
    if varlen:
        qs, ks = _i32(q_seqlen), _i32(kv_seqlen)
        keep_alive += [qs, ks]
        a.batch = qs.shape[0]
        a.q_seqlen, a.kv_seqlen = qs.ctypes.data, ks.ctypes.data
        out_shape = q.shape[:2] + (a.dv,)
        a.lq = a.lk = 0
    else:
        a.batch = q.shape[0]
        a.lq, a.lk = q.shape[2], k.shape[2]
        out_shape = q.shape[:3] + (a.dv,)
    out = np.zeros(out_shape if full_out else (1,) * len(out_shape), dtype=np.float64)
    a.q, a.k, a.v = _tensor(q, varlen), _tensor(k, varlen), _tensor(v, varlen)
    if qrope is not None:
        a.qrope, a.krope = _tensor(qrope, varlen), _tensor(krope, varlen)
    a.out = out.ctypes.data
    a.out_t = _tensor(out, varlen)
    if kind in (2, 3):
        if varlen:
            raise ValueError("explicit masks are defined for the dense layout only")
        B, Hq, Lq, Lk = q.shape[0], q.shape[1], q.shape[2], k.shape[2]
        m = mask.detach().cpu().numpy() if hasattr(mask, "detach") else np.asarray(mask)
        m = m.astype(np.uint8) if kind == 2 else m.astype(np.float64)
        while m.ndim < 4:
            m = m[None]
        mb = np.broadcast_to(m, (B, Hq, Lq, Lk))
        es = mb.itemsize
        a.mb, a.mh, a.mi, a.mj = (s // es for s in mb.strides)
        keep_alive.append(m)
        if kind == 2:
            a.keep = mb.ctypes.data
        else:
            a.add = mb.ctypes.data
    keep_alive += [q, k, v, qrope, krope]
    return a, out, keep_alive, varlen


def sdpa(q, k, v, *, qrope=None, krope=None, q_seqlen=None, kv_seqlen=None,
         mask=None, mask_kind="none", head_num=None, kv_head_num=None,
         qk_scale=None, with_lse=False, plant=0):
    """Full fp64 attention forward; returns ``out`` (and ``lse``, natural log)."""
    varlen = q_seqlen is not None
    hq = q.shape[1] if head_num is None else head_num
    hk = k.shape[1] if kv_head_num is None else kv_head_num
    if qk_scale is None:
        raise ValueError("qk_scale is required")
    a, out, keep_alive, varlen = _prepare(q, k, v, qrope, krope, q_seqlen, kv_seqlen, mask,
                                          mask_kind, hq, hk, qk_scale)
    lse = None
    if with_lse:
        if varlen:
            lse = np.full((hq, q.shape[0]), -np.inf)
            a.lse_ld = q.shape[0]
        else:
            lse = np.full((q.shape[0], hq, q.shape[2]), -np.inf)
        a.lse = lse.ctypes.data
    rc = _load(plant).ora_sdpa_fwd(ctypes.byref(a))
    if rc != 0:
        raise ValueError(f"oracle rejected the arguments (code {rc})")
    del keep_alive
    return (out, lse) if with_lse else out


def sdpa_rows(q, k, v, rows, *, qrope=None, krope=None, q_seqlen=None, kv_seqlen=None,
              mask=None, mask_kind="none", head_num=None, kv_head_num=None, qk_scale=None,
              with_lse=False, plant=0):
    """fp64 output for selected rows only.  ``rows`` is an int array ``[n, 3]`` of
    (sequence or batch index, query head, row within the sequence).  Each row is
    evaluated over its full key range.  Returns ``[n, Dv]`` (and ``[n]`` LSE)."""
    hq = q.shape[1] if head_num is None else head_num
    hk = k.shape[1] if kv_head_num is None else kv_head_num
    if qk_scale is None:
        raise ValueError("qk_scale is required")
    a, _, keep_alive, _ = _prepare(q, k, v, qrope, krope, q_seqlen, kv_seqlen, mask,
                                   mask_kind, hq, hk, qk_scale, full_out=False)
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    res = np.zeros((r.shape[0], a.dv), dtype=np.float64)
    lse = np.full((r.shape[0],), -np.inf) if with_lse else None
    rc = _load(plant).ora_sdpa_fwd_rows(ctypes.byref(a), r.ctypes.data, r.shape[0],
                                        res.ctypes.data, None if lse is None else lse.ctypes.data)
    if rc != 0:
        raise ValueError(f"oracle rejected the arguments (code {rc})")
    del keep_alive
    return (res, lse) if with_lse else res
