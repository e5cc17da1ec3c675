"""Python front end: torch tensors in, C-ABI calls out.

Every function here only marshals arguments (pointers, shapes, strides, the
current CUDA stream) into ``libwfattn.so``; all computation runs in its
kernels.  Tensors must live on a CUDA device: there is no CPU path.

Mirrors the pages' API surface:
  * :func:`attn_fwd` -- the attention forward of "Core 注意力" (section
    "选择最窄的入口", PyTorch SDPA contract with GQA) and of "MLA Prefill"
    (packed layout, qSeqLen/kvSeqLen, QRope/kRope, headNum/kvHeadNum/qkScale).
  * :func:`scaled_dot_product_attention` -- the same forward under the
    PyTorch SDPA signature itself, for callers of that entry.
  * :class:`BlockKVCache` -- the rolling cache of "Core 注意力", section
    "Block KV cache 的调用顺序" (before_update -> update -> cached_k/cached_v
    -> after_update).
"""
from __future__ import annotations

import ctypes
import enum
import math

import torch

from . import _lib as L


class WfError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{L.STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class MaskType(enum.IntEnum):
    NONE = L.WF_MASK_NONE
    CAUSAL = L.WF_MASK_CAUSAL
    BOOL_KEEP = L.WF_MASK_BOOL_KEEP
    ADDITIVE = L.WF_MASK_ADDITIVE
    CAUSAL_TOP_LEFT = L.WF_MASK_CAUSAL_TOP_LEFT


_DTYPES = {torch.float32: L.WF_F32, torch.bfloat16: L.WF_BF16, torch.float16: L.WF_F16,
           torch.uint8: L.WF_U8, torch.bool: L.WF_U8, torch.int32: L.WF_I32}


def _check(status: int) -> None:
    if status != L.WF_OK:
        msg = L.load().wf_last_error_message()
        raise WfError(status, msg.decode() if msg else "")


def describe(t: torch.Tensor | None) -> L.WfTensor | None:
    """C descriptor of a tensor (no copy; the tensor must outlive the call)."""
    if t is None:
        return None
    if t.dim() > 4:
        raise ValueError("at most 4 dims")
    d = L.WfTensor()
    d.data = t.data_ptr() if t.numel() else None
    d.dtype = _DTYPES[t.dtype]
    d.ndim = t.dim()
    for i in range(t.dim()):
        d.shape[i] = t.shape[i]
        d.stride[i] = t.stride(i)
    return d


def _ref(d):
    return ctypes.byref(d) if d is not None else None


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _require_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise WfError(L.WF_ERR_INVALID_ARG,
                          "tensors must be on a CUDA device (this library has no CPU path)")


def attn_fwd(q, k, v, *, qrope=None, krope=None, q_seqlen=None, kv_seqlen=None, mask=None,
             mask_type=None, head_num=None, kv_head_num=None, qk_scale=None, out=None,
             return_lse=False, lse=None, num_splits=None, kv_layout=None, stream=None,
             debug_flags=0, timeout_cycles=0):
    """out = softmax(q k^T * qk_scale + mask) v, see ``include/wf_attn.h``.

    Dense: q [B,Hq,Lq,D], k/v [B,Hkv,Lk,D].  Packed: q [T,Hq,D], k/v [Tk,Hkv,D]
    with int32 ``q_seqlen`` / ``kv_seqlen`` on the device.  ``mask_type``
    defaults to BOOL_KEEP for a bool mask, ADDITIVE for a float mask, NONE
    otherwise.  ``qk_scale`` defaults to 1/sqrt(Dqk + Drope).

    ``return_lse`` (or a given fp32 ``lse`` tensor of out's shape without the
    last dim) also returns the natural-log LSE of every row: ``(out, lse)``.
    ``num_splits``: None/0 automatic split-KV, 1 none, n > 1 forced
    (``wf_attn_fwd_ex``).

    Packed layout extras ("MLA Prefill" parameter table): q / qrope may be
    given flattened as [T, Hq * D] (then ``head_num`` is required), and K /
    kRope / V padded as [batch, max_seq, Hkv, D] or, with
    ``kv_layout="padded"``, flattened as [batch, max_seq, Hkv * D] (then
    ``kv_head_num`` is required).  These are views, no copies.
    """
    _require_cuda(q, k, v, qrope, krope, q_seqlen, kv_seqlen, mask, out, lse)
    varlen = q_seqlen is not None
    if varlen and q.dim() == 2:
        if head_num is None:
            raise ValueError("flattened q [T, Hq*D] needs head_num")
        q = q.view(q.shape[0], head_num, -1)
        if qrope is not None:
            qrope = qrope.view(qrope.shape[0], head_num, -1)
    if varlen and kv_layout == "padded" and k.dim() == 3:
        if kv_head_num is None:
            raise ValueError("flattened padded k/v [B, S, Hkv*D] needs kv_head_num")
        k, v = (t.view(t.shape[0], t.shape[1], kv_head_num, -1) for t in (k, v))
        if krope is not None:
            krope = krope.view(krope.shape[0], krope.shape[1], kv_head_num, -1)
    if head_num is None:
        head_num = q.shape[1]
    if kv_head_num is None:
        kv_head_num = k.shape[2] if (varlen and k.dim() == 4) else k.shape[1]
    if mask_type is None:
        if mask is None:
            mask_type = MaskType.NONE
        else:
            mask_type = MaskType.BOOL_KEEP if mask.dtype in (torch.bool, torch.uint8) else MaskType.ADDITIVE
    if qk_scale is None:
        qk_scale = 1.0 / math.sqrt(q.shape[-1] + (qrope.shape[-1] if qrope is not None else 0))
    if out is None:
        shape = (q.shape[0], head_num, v.shape[-1]) if varlen else \
            (q.shape[0], head_num, q.shape[2], v.shape[-1])
        out = torch.empty(shape, dtype=q.dtype, device=q.device)
    if mask is not None and mask.dtype == torch.bool:
        mask = mask.view(torch.uint8)
    if mask is not None:
        while mask.dim() < 4:
            mask = mask.unsqueeze(0)
    want_lse = return_lse or lse is not None
    if want_lse and lse is None:
        lse = torch.empty(out.shape[:-1], dtype=torch.float32, device=q.device)
    descs = [describe(x) for x in (q, qrope, k, krope, v, q_seqlen, kv_seqlen, mask)]
    od = describe(out)
    lib = L.load()
    with torch.cuda.device(q.device):
        if want_lse or num_splits is not None:
            if debug_flags or timeout_cycles:
                raise ValueError("debug switches do not combine with lse / num_splits")
            ld = describe(lse) if want_lse else None
            st = lib.wf_attn_fwd_ex(*[_ref(d) for d in descs], int(head_num), int(kv_head_num),
                                    float(qk_scale), int(mask_type), ctypes.byref(od), _ref(ld),
                                    int(num_splits or 0), _stream(stream))
        elif debug_flags or timeout_cycles:
            st = lib.wf_attn_fwd_debug(*[_ref(d) for d in descs], int(head_num), int(kv_head_num),
                                       float(qk_scale), int(mask_type), ctypes.byref(od),
                                       _stream(stream), int(debug_flags), int(timeout_cycles))
        else:
            st = lib.wf_attn_fwd(*[_ref(d) for d in descs], int(head_num), int(kv_head_num),
                                 float(qk_scale), int(mask_type), ctypes.byref(od), _stream(stream))
    _check(st)
    return (out, lse) if want_lse else out


def scaled_dot_product_attention(query, key, value, attn_mask=None, dropout_p=0.0, is_causal=False,
                                 scale=None, enable_gqa=False, *, backend=None, out=None, stream=None):
    """The ``torch.nn.functional.scaled_dot_product_attention`` contract that
    "Core 注意力" (section "选择最窄的入口") gives its entry, for inference,
    on this library's kernels (argument mapping onto :func:`attn_fwd`).

    ``query`` [B, Hq, L, E] or [Hq, L, E]; ``key`` / ``value`` [B, Hkv, S, E]
    / [B, Hkv, S, Ev] (same rank as ``query``).  ``attn_mask``: bool (True =
    the key takes part) or float (added to the scaled scores), broadcastable
    to [B, Hq, L, S].  ``is_causal``: query i sees keys j <= i, aligned at the
    top-left as in torch; with L == S that is the library's causal mask,
    otherwise an explicit keep-mask is passed.  ``scale`` defaults to
    1/sqrt(E).  ``enable_gqa``: Hq may be a multiple of Hkv (consecutive query
    heads share a key head).  ``dropout_p`` must be 0.  ``backend`` is
    accepted for call compatibility with the page's entry, which selects a
    provider with it; this library has one provider, its sm_100a kernels,
    whatever is named.

    One difference from torch: a row whose keys are all masked gives zeros
    (torch gives NaN).
    """
    if dropout_p != 0.0:
        raise ValueError("dropout_p must be 0: this is the inference forward")
    if is_causal and attn_mask is not None:
        raise ValueError("attn_mask and is_causal cannot both be given (as in torch)")
    squeeze = query.dim() == 3
    if squeeze:
        query, key, value = query.unsqueeze(0), key.unsqueeze(0), value.unsqueeze(0)
    if query.dim() != 4 or key.dim() != 4 or value.dim() != 4:
        raise ValueError("query / key / value must all be [B, H, L, E] or all [H, L, E]")
    hq, hk = query.shape[1], key.shape[1]
    if hq != hk and not enable_gqa:
        raise ValueError(f"{hq} query heads against {hk} key heads needs enable_gqa=True (as in torch)")
    lq, lk = query.shape[2], key.shape[2]
    mask, mask_type = None, MaskType.NONE
    if is_causal:
        # torch's is_causal is top-left aligned (key j visible to query i iff
        # j <= i); the kernel generates it, as it does the bottom-right form
        mask_type = MaskType.CAUSAL if lq == lk else MaskType.CAUSAL_TOP_LEFT
    elif attn_mask is not None:
        mask = attn_mask
        if mask.dtype == torch.bool:
            mask_type = MaskType.BOOL_KEEP
        else:
            if mask.dtype not in (torch.float32, query.dtype):
                mask = mask.float()
            mask_type = MaskType.ADDITIVE
    if mask is not None:
        if mask.dim() > 4:
            raise ValueError("attn_mask must be broadcastable to [B, H, L, S]")
        while mask.dim() < 4:
            mask = mask.unsqueeze(0)
    if out is not None and squeeze:
        out = out.unsqueeze(0)
    res = attn_fwd(query, key, value, mask=mask, mask_type=mask_type, qk_scale=scale, out=out,
                   stream=stream)
    return res.squeeze(0) if squeeze else res


def merge(out_parts, lse_parts, *, out=None, lse=None, stream=None):
    """Combine results over disjoint key sets (``wf_attn_merge``).

    ``out_parts`` [S, ..., Dv] (fp32 or bf16), ``lse_parts`` [S, ...] fp32
    (natural log).  Returns ``(out, lse)``; ``out`` defaults to the parts'
    dtype.  The row dims are flattened by views, so they must be viewable as
    one dim.
    """
    _require_cuda(out_parts, lse_parts, out, lse)
    S, dv = out_parts.shape[0], out_parts.shape[-1]
    rows_shape = tuple(out_parts.shape[1:-1])
    if tuple(lse_parts.shape) != (S,) + rows_shape:
        raise ValueError(f"lse_parts {tuple(lse_parts.shape)} does not match out_parts {tuple(out_parts.shape)}")
    if out is None:
        out = torch.empty(rows_shape + (dv,), dtype=out_parts.dtype, device=out_parts.device)
    if lse is None:
        lse = torch.empty(rows_shape, dtype=torch.float32, device=out_parts.device)
    pd = describe(out_parts.view(S, -1, dv))
    ld = describe(lse_parts.view(S, -1))
    od = describe(out.view(-1, dv))
    ed = describe(lse.view(-1))
    with torch.cuda.device(out_parts.device):
        _check(L.load().wf_attn_merge(ctypes.byref(pd), ctypes.byref(ld), ctypes.byref(od),
                                      ctypes.byref(ed), _stream(stream)))
    return out, lse


def dca(q_intra, q_succ, q_inter, k, v, chunk_size, *, qk_scale=None, out=None, return_lse=False,
        stream=None):
    """Dual chunk attention (``wf_attn_dca``): query i of chunk c attends
    causally, scoring keys of chunk c with ``q_intra``, of chunk c - 1 with
    ``q_succ`` and of earlier chunks with ``q_inter`` (each [B, H, L, D],
    rotated by the caller for its position map); k / v [B, Hkv, L, D]."""
    _require_cuda(q_intra, q_succ, q_inter, k, v, out)
    if qk_scale is None:
        qk_scale = 1.0 / math.sqrt(q_intra.shape[-1])
    if out is None:
        out = torch.empty(q_intra.shape[:3] + (v.shape[-1],), dtype=q_intra.dtype, device=q_intra.device)
    lse = torch.empty(q_intra.shape[:3], dtype=torch.float32, device=q_intra.device) if return_lse else None
    ds = [describe(x) for x in (q_intra, q_succ, q_inter, k, v)]
    od, ld = describe(out), describe(lse)
    with torch.cuda.device(q_intra.device):
        _check(L.load().wf_attn_dca(*[ctypes.byref(d) for d in ds], int(chunk_size), int(q_intra.shape[1]),
                                    int(k.shape[1]), float(qk_scale), ctypes.byref(od), _ref(ld),
                                    _stream(stream)))
    return (out, lse) if return_lse else out


def device_status(stream=None) -> None:
    """Synchronize the stream and raise if a kernel recorded a device-side error."""
    _check(L.load().wf_get_device_status(_stream(stream)))


class BlockKVCache:
    """Rolling sink + window KV cache over caller-owned buffers.

    ``k_buf``/``v_buf``: [B, H, L, D] (seq_dim 2) or [B, L, H, D] (seq_dim 1) on a
    CUDA device.  ``sink_size + window_size == L``; both multiples of
    ``chunk_size``.  State transitions are checked by the library; a call out
    of order raises :class:`WfError` with status ``WF_ERR_ORDER``.

    The constructor form of "Core 注意力" ("Block KV cache 的调用顺序") is
    accepted too: ``BlockKVCache(k_shape=..., v_shape=..., seq_dim=...,
    chunk_size=..., window_size=..., device=..., dtype=...)`` allocates zeroed
    buffers (``device`` must be a CUDA device).
    """

    def __init__(self, k_buf=None, v_buf=None, *, seq_dim=2, chunk_size, window_size, sink_size=0,
                 k_shape=None, v_shape=None, device="cuda", dtype=torch.bfloat16):
        bufs = (k_buf is not None, v_buf is not None)
        shapes = (k_shape is not None, v_shape is not None)
        if not ((all(bufs) and not any(shapes)) or (all(shapes) and not any(bufs))):
            raise ValueError("give either k_buf and v_buf, or k_shape and v_shape")
        if all(shapes):
            if torch.device(device).type != "cuda":
                raise WfError(L.WF_ERR_INVALID_ARG,
                              "tensors must be on a CUDA device (this library has no CPU path)")
            k_buf = torch.zeros(k_shape, dtype=dtype, device=device)
            v_buf = torch.zeros(v_shape, dtype=dtype, device=device)
        _require_cuda(k_buf, v_buf)
        self.k_buf, self.v_buf = k_buf, v_buf
        self.seq_dim = seq_dim
        h = ctypes.c_void_p()
        self._kd, self._vd = describe(k_buf), describe(v_buf)
        _check(L.load().wf_kvcache_create(ctypes.byref(self._kd), ctypes.byref(self._vd), seq_dim,
                                          chunk_size, sink_size, window_size, ctypes.byref(h)))
        self._h = h

    @classmethod
    def allocate(cls, k_shape, v_shape, *, seq_dim=2, chunk_size, window_size, sink_size=0,
                 device="cuda", dtype=torch.bfloat16):
        """Allocate zeroed buffers of the given shapes and wrap them."""
        return cls(k_shape=k_shape, v_shape=v_shape, seq_dim=seq_dim, chunk_size=chunk_size,
                   window_size=window_size, sink_size=sink_size, device=device, dtype=dtype)

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value:
            L.load().wf_kvcache_destroy(h)
            self._h = None

    def before_update(self, chunk_idx: int) -> None:
        _check(L.load().wf_kvcache_before_update(self._h, int(chunk_idx)))

    def update(self, k, v, stream=None) -> None:
        _require_cuda(k, v)
        kd, vd = describe(k), describe(v)
        with torch.cuda.device(self.k_buf.device):
            _check(L.load().wf_kvcache_update(self._h, ctypes.byref(kd), ctypes.byref(vd),
                                              _stream(stream)))

    def _views(self):
        kd, vd, vis = L.WfTensor(), L.WfTensor(), ctypes.c_int64()
        _check(L.load().wf_kvcache_cached(self._h, ctypes.byref(kd), ctypes.byref(vd),
                                          ctypes.byref(vis)))
        kv = torch.as_strided(self.k_buf, tuple(kd.shape[:4]), tuple(kd.stride[:4]))
        vv = torch.as_strided(self.v_buf, tuple(vd.shape[:4]), tuple(vd.stride[:4]))
        return kv, vv

    def cached_k(self):
        """Visible keys, [B, H, vis, D] view of the buffer (physical ring order)."""
        return self._views()[0]

    def cached_v(self):
        """Visible values, [B, H, vis, D] view of the buffer (physical ring order)."""
        return self._views()[1]

    def update_attend(self, k, v, q, *, qk_scale=None, head_num=None, out=None, stream=None):
        """The chunk's update, cached views and attention of ``q`` over the
        visible keys in one call (``wf_kvcache_update_attend``); returns out
        [B, Hq, Lq, Dv].  Call after ``before_update``, then ``after_update``."""
        _require_cuda(k, v, q, out)
        if head_num is None:
            head_num = q.shape[1]
        if qk_scale is None:
            qk_scale = 1.0 / math.sqrt(q.shape[-1])
        if out is None:
            out = torch.empty(q.shape[:3] + (self.v_buf.shape[-1],), dtype=q.dtype, device=q.device)
        kd, vd, qd, od = describe(k), describe(v), describe(q), describe(out)
        with torch.cuda.device(self.k_buf.device):
            _check(L.load().wf_kvcache_update_attend(self._h, ctypes.byref(kd), ctypes.byref(vd),
                                                     ctypes.byref(qd), int(head_num), float(qk_scale),
                                                     ctypes.byref(od), _stream(stream)))
        return out

    def after_update(self, chunk_idx: int) -> None:
        _check(L.load().wf_kvcache_after_update(self._h, int(chunk_idx)))

    def state(self):
        """(current index, committed index, write slot, visible length, phase)."""
        cur, com, slot, vis = (ctypes.c_int64() for _ in range(4))
        ph = ctypes.c_int32()
        _check(L.load().wf_kvcache_get_state(self._h, ctypes.byref(cur), ctypes.byref(com),
                                             ctypes.byref(slot), ctypes.byref(vis),
                                             ctypes.byref(ph)))
        return cur.value, com.value, slot.value, vis.value, ph.value

    def set_state(self, committed_idx: int) -> None:
        """Resume at chunk ``committed_idx`` (-1: none) as the last committed
        chunk, for buffers restored by the caller (``wf_kvcache_set_state``)."""
        _check(L.load().wf_kvcache_set_state(self._h, int(committed_idx)))

    def gather_logical(self, stream=None):
        """Copy of the visible tokens in logical chunk order (buffer layout)."""
        vis = self.state()[3]
        ks = list(self.k_buf.shape)
        vs = list(self.v_buf.shape)
        ks[self.seq_dim] = vis
        vs[self.seq_dim] = vis
        ko = torch.empty(ks, dtype=self.k_buf.dtype, device=self.k_buf.device)
        vo = torch.empty(vs, dtype=self.v_buf.dtype, device=self.v_buf.device)
        kd, vd = describe(ko), describe(vo)
        with torch.cuda.device(self.k_buf.device):
            _check(L.load().wf_kvcache_gather_logical(self._h, ctypes.byref(kd), ctypes.byref(vd),
                                                      _stream(stream)))
        return ko, vo
