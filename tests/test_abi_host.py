"""The C-ABI library on the host (no GPU): it loads, exports every declared
symbol, rejects bad arguments before touching a device, and enforces the
BlockKVCache call order."""
import ctypes
import glob
import os
import re

import pytest

from attention_forward_tmem_b200 import _lib as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ALIGNED = 0x10000          # fake, 16-byte aligned addresses: never dereferenced on the host


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"\b(wf_[a-z_0-9]+)\s*\(", src):
            names.add(m.group(1))
    return names


@pytest.fixture(scope="module")
def lib():
    return L.load()


def test_every_declared_symbol_is_exported(lib):
    declared = _declared_functions()
    assert "wf_attn_fwd" in declared and "wf_kvcache_update" in declared
    for name in declared:
        assert hasattr(lib, name), f"{name} is declared in include/ but not exported"
    assert set(L.SIGNATURES) >= declared


def test_version(lib):
    assert lib.wf_version() == 1


def _t(shape, dtype=L.WF_BF16, data=ALIGNED, strides=None):
    d = L.WfTensor()
    d.data = data
    d.dtype = dtype
    d.ndim = len(shape)
    if strides is None:
        strides, acc = [], 1
        for s in reversed(shape):
            strides.insert(0, acc)
            acc *= s
    for i, (s, st) in enumerate(zip(shape, strides)):
        d.shape[i] = s
        d.stride[i] = st
    return d


def _call(lib, q, k, v, out, *, qr=None, kr=None, ql=None, kl=None, mask=None, hq=None, hk=None,
          scale=0.125, mt=L.WF_MASK_NONE):
    r = lambda x: ctypes.byref(x) if x is not None else None
    hq = q.shape[1] if hq is None else hq
    hk = k.shape[1] if hk is None else hk
    return lib.wf_attn_fwd(r(q), r(qr), r(k), r(kr), r(v), r(ql), r(kl), r(mask), hq, hk, scale, mt,
                           ctypes.byref(out), None)


def _dense(B=2, Hq=8, Hk=2, Lq=100, Lk=120, D=128, Dv=128, dtype=L.WF_BF16):
    return (_t([B, Hq, Lq, D], dtype), _t([B, Hk, Lk, D], dtype), _t([B, Hk, Lk, Dv], dtype),
            _t([B, Hq, Lq, Dv], dtype))


def test_valid_call_reaches_device_check(lib):
    """Everything valid: the only thing left to fail on a CPU host is the device."""
    q, k, v, o = _dense()
    st = _call(lib, q, k, v, o, mt=L.WF_MASK_CAUSAL)
    assert st in (L.WF_ERR_NO_DEVICE, L.WF_OK)   # WF_OK only where a B200 is present
    q, k, v, o = _dense(dtype=L.WF_F16)
    st = _call(lib, q, k, v, o, mt=L.WF_MASK_ADDITIVE, mask=_t([2, 8, 100, 120], L.WF_F16))
    assert st in (L.WF_ERR_NO_DEVICE, L.WF_OK)
    # packed q, padded k / v with rope
    q, o, qr = _t([300, 8, 128]), _t([300, 8, 128]), _t([300, 8, 64])
    k, v, kr = _t([3, 160, 2, 128]), _t([3, 160, 2, 128]), _t([3, 160, 2, 64])
    st = _call(lib, q, k, v, o, qr=qr, kr=kr, ql=_t([3], L.WF_I32), kl=_t([3], L.WF_I32), hk=2,
               mt=L.WF_MASK_CAUSAL)
    assert st in (L.WF_ERR_NO_DEVICE, L.WF_OK), lib.wf_last_error_message()


@pytest.mark.parametrize("case,expect", [
    ("i32_inputs", L.WF_ERR_UNSUPPORTED),
    ("mask_f16_with_bf16", L.WF_ERR_INVALID_ARG),
    ("padded_batch_mismatch", L.WF_ERR_INVALID_ARG),
    ("padded_head_mismatch", L.WF_ERR_INVALID_ARG),
    ("padded_f32", L.WF_ERR_UNSUPPORTED),
    ("padded_rope_mismatch", L.WF_ERR_INVALID_ARG),
    ("heads_not_divisible", L.WF_ERR_INVALID_ARG),
    ("head_count_mismatch", L.WF_ERR_INVALID_ARG),
    ("dtype_mix", L.WF_ERR_INVALID_ARG),
    ("dv_unsupported", L.WF_ERR_UNSUPPORTED),
    ("unaligned_ptr", L.WF_ERR_INVALID_ARG),
    ("unaligned_stride", L.WF_ERR_INVALID_ARG),
    ("noncontig_last", L.WF_ERR_INVALID_ARG),
    ("mask_missing", L.WF_ERR_INVALID_ARG),
    ("mask_with_causal", L.WF_ERR_INVALID_ARG),
    ("mask_with_varlen", L.WF_ERR_UNSUPPORTED),
    ("f32_varlen", L.WF_ERR_UNSUPPORTED),
    ("mask_bad_shape", L.WF_ERR_INVALID_ARG),
    ("mask_bad_dtype", L.WF_ERR_INVALID_ARG),
    ("rope_one_side", L.WF_ERR_INVALID_ARG),
    ("rope_bad_width", L.WF_ERR_UNSUPPORTED),
    ("seqlen_one_side", L.WF_ERR_INVALID_ARG),
    ("seqlen_len_mismatch", L.WF_ERR_INVALID_ARG),
    ("bad_mask_type", L.WF_ERR_INVALID_ARG),
    ("nan_scale", L.WF_ERR_INVALID_ARG),
    ("batch_mismatch", L.WF_ERR_INVALID_ARG),
])
def test_argument_errors(lib, case, expect):
    q, k, v, o = _dense()
    kw = {}
    if case == "i32_inputs":
        q, k, v, o = _dense(dtype=L.WF_I32)
    elif case == "mask_f16_with_bf16":
        kw.update(mt=L.WF_MASK_ADDITIVE, mask=_t([2, 8, 100, 120], L.WF_F16))
    elif case in ("padded_batch_mismatch", "padded_head_mismatch", "padded_f32", "padded_rope_mismatch"):
        dt = L.WF_F32 if case == "padded_f32" else L.WF_BF16
        q, o = _t([300, 8, 128], dt), _t([300, 8, 128], dt)
        kb = 4 if case == "padded_batch_mismatch" else 3
        kh = 4 if case == "padded_head_mismatch" else 2
        k, v = _t([kb, 160, kh, 128], dt), _t([kb, 160, kh, 128], dt)
        kw.update(ql=_t([3], L.WF_I32), kl=_t([3], L.WF_I32), hk=2)
        if case == "padded_rope_mismatch":
            kw.update(qr=_t([300, 8, 64]), kr=_t([3, 150, 2, 64]))
    elif case == "heads_not_divisible":
        q, k, v, o = _dense(Hq=6, Hk=4)
    elif case == "head_count_mismatch":
        kw["hq"] = 4
    elif case == "dtype_mix":
        v = _t([2, 2, 120, 128], L.WF_F32)
    elif case == "dv_unsupported":
        q, k, v, o = _dense(Dv=80)
    elif case == "unaligned_ptr":
        q = _t([2, 8, 100, 128], data=ALIGNED + 2)
    elif case == "unaligned_stride":
        q = _t([2, 8, 100, 128], strides=[8 * 100 * 132, 100 * 132, 132 - 4 + 1, 1])
    elif case == "noncontig_last":
        q = _t([2, 8, 100, 128], strides=[8 * 100 * 256, 100 * 256, 256, 2])
    elif case == "mask_missing":
        kw["mt"] = L.WF_MASK_BOOL_KEEP
    elif case == "mask_with_causal":
        kw.update(mt=L.WF_MASK_CAUSAL, mask=_t([2, 8, 100, 120], L.WF_U8))
    elif case == "mask_with_varlen":
        q, k, v, o = _t([300, 8, 128]), _t([300, 2, 128]), _t([300, 2, 128]), _t([300, 8, 128])
        kw.update(ql=_t([3], L.WF_I32), kl=_t([3], L.WF_I32), mask=_t([1, 1, 300, 300], L.WF_U8),
                  mt=L.WF_MASK_BOOL_KEEP)
    elif case == "f32_varlen":
        f = L.WF_F32
        q, k, v, o = _t([300, 8, 128], f), _t([300, 2, 128], f), _t([300, 2, 128], f), _t([300, 8, 128], f)
        kw.update(ql=_t([3], L.WF_I32), kl=_t([3], L.WF_I32))
    elif case == "mask_bad_shape":
        kw.update(mt=L.WF_MASK_BOOL_KEEP, mask=_t([2, 3, 100, 120], L.WF_U8))
    elif case == "mask_bad_dtype":
        kw.update(mt=L.WF_MASK_BOOL_KEEP, mask=_t([2, 8, 100, 120], L.WF_F32))
    elif case == "rope_one_side":
        kw.update(qr=_t([2, 8, 100, 64]))
    elif case == "rope_bad_width":
        kw.update(qr=_t([2, 8, 100, 32]), kr=_t([2, 2, 120, 32]))
    elif case == "seqlen_one_side":
        q, k, v, o = _t([300, 8, 128]), _t([300, 2, 128]), _t([300, 2, 128]), _t([300, 8, 128])
        kw.update(ql=_t([3], L.WF_I32))
    elif case == "seqlen_len_mismatch":
        q, k, v, o = _t([300, 8, 128]), _t([300, 2, 128]), _t([300, 2, 128]), _t([300, 8, 128])
        kw.update(ql=_t([3], L.WF_I32), kl=_t([4], L.WF_I32))
    elif case == "bad_mask_type":
        kw["mt"] = 7
    elif case == "nan_scale":
        kw["scale"] = float("nan")
    elif case == "batch_mismatch":
        k = _t([3, 2, 120, 128])
    assert _call(lib, q, k, v, o, **kw) == expect
    assert lib.wf_last_error_message()


def test_empty_input_is_a_no_op(lib):
    q, k, v, o = _dense(Lq=0)
    q.data = None
    o.data = None
    assert _call(lib, q, k, v, o) == L.WF_OK


def _call_ex(lib, q, k, v, out, lse, splits, *, ql=None, kl=None, mt=L.WF_MASK_NONE):
    r = lambda x: ctypes.byref(x) if x is not None else None
    return lib.wf_attn_fwd_ex(r(q), None, r(k), None, r(v), r(ql), r(kl), None, q.shape[1],
                              k.shape[1], 0.125, mt, ctypes.byref(out), r(lse), splits, None)


@pytest.mark.parametrize("case,expect", [
    ("ok", None),
    ("lse_wrong_rank", L.WF_ERR_INVALID_ARG),
    ("lse_wrong_shape", L.WF_ERR_INVALID_ARG),
    ("lse_bf16", L.WF_ERR_INVALID_ARG),
    ("lse_misaligned", L.WF_ERR_INVALID_ARG),
    ("splits_negative", L.WF_ERR_INVALID_ARG),
    ("splits_too_many", L.WF_ERR_INVALID_ARG),
    ("packed_lse_shape", L.WF_ERR_INVALID_ARG),
])
def test_attn_fwd_ex_argument_errors(lib, case, expect):
    q, k, v, o = _dense()
    lse, splits, kw = _t([2, 8, 100], L.WF_F32), 0, {}
    if case == "lse_wrong_rank":
        lse = _t([2, 8, 100, 1], L.WF_F32)
    elif case == "lse_wrong_shape":
        lse = _t([2, 8, 101], L.WF_F32)
    elif case == "lse_bf16":
        lse = _t([2, 8, 100], L.WF_BF16)
    elif case == "lse_misaligned":
        lse = _t([2, 8, 100], L.WF_F32, data=ALIGNED + 2)
    elif case == "splits_negative":
        splits = -1
    elif case == "splits_too_many":
        splits = 129
    elif case == "packed_lse_shape":
        q, k, v, o = _t([300, 8, 128]), _t([300, 2, 128]), _t([300, 2, 128]), _t([300, 8, 128])
        kw.update(ql=_t([3], L.WF_I32), kl=_t([3], L.WF_I32))
        lse = _t([8, 300], L.WF_F32)              # head-major must be passed transposed
    st = _call_ex(lib, q, k, v, o, lse, splits, **kw)
    if expect is None:
        assert st in (L.WF_ERR_NO_DEVICE, L.WF_OK)
    else:
        assert st == expect
        assert lib.wf_last_error_message()


@pytest.mark.parametrize("case,expect", [
    ("ok", None),
    ("lse_parts_shape", L.WF_ERR_INVALID_ARG),
    ("out_shape", L.WF_ERR_INVALID_ARG),
    ("lse_shape", L.WF_ERR_INVALID_ARG),
    ("dv_not_mult4", L.WF_ERR_UNSUPPORTED),
    ("int_parts", L.WF_ERR_UNSUPPORTED),
    ("parts_rank", L.WF_ERR_INVALID_ARG),
    ("parts_unaligned_stride", L.WF_ERR_INVALID_ARG),
])
def test_merge_argument_errors(lib, case, expect):
    S, R, dv = 3, 50, 128
    parts, lp, out, lse = _t([S, R, dv], L.WF_F32), _t([S, R], L.WF_F32), _t([R, dv]), _t([R], L.WF_F32)
    if case == "lse_parts_shape":
        lp = _t([S, R + 1], L.WF_F32)
    elif case == "out_shape":
        out = _t([R, dv + 8])
    elif case == "lse_shape":
        lse = _t([R - 1], L.WF_F32)
    elif case == "dv_not_mult4":
        parts, out = _t([S, R, 10], L.WF_F32, strides=[R * 12, 12, 1]), _t([R, 10], strides=[16, 1])
    elif case == "int_parts":
        parts = _t([S, R, dv], L.WF_I32)
    elif case == "parts_rank":
        parts = _t([S, 2, R // 2, dv], L.WF_F32)
    elif case == "parts_unaligned_stride":
        parts = _t([S, R, dv], L.WF_F32, strides=[R * 130, 130, 1])
    st = lib.wf_attn_merge(ctypes.byref(parts), ctypes.byref(lp), ctypes.byref(out), ctypes.byref(lse), None)
    if expect is None:
        assert st in (L.WF_ERR_NO_DEVICE, L.WF_OK)
    else:
        assert st == expect
        assert lib.wf_last_error_message()


@pytest.mark.parametrize("case,expect", [
    ("ok", None),
    ("fp32", L.WF_ERR_UNSUPPORTED),
    ("chunk_zero", L.WF_ERR_INVALID_ARG),
    ("q_forms_differ", L.WF_ERR_INVALID_ARG),
    ("kv_len", L.WF_ERR_INVALID_ARG),
    ("out_shape", L.WF_ERR_INVALID_ARG),
])
def test_dca_argument_errors(lib, case, expect):
    dt = L.WF_F32 if case == "fp32" else L.WF_BF16
    qi, qs, qe = _t([1, 4, 300, 128], dt), _t([1, 4, 300, 128], dt), _t([1, 4, 300, 128], dt)
    k, v, o = _t([1, 2, 300, 128], dt), _t([1, 2, 300, 128], dt), _t([1, 4, 300, 128], dt)
    chunk = 0 if case == "chunk_zero" else 128
    if case == "q_forms_differ":
        qe = _t([1, 4, 299, 128], dt)
    elif case == "kv_len":
        k = _t([1, 2, 301, 128], dt)
    elif case == "out_shape":
        o = _t([1, 4, 300, 64], dt)
    r = ctypes.byref
    st = lib.wf_attn_dca(r(qi), r(qs), r(qe), r(k), r(v), chunk, 4, 2, 0.1, r(o), None, None)
    if expect is None:
        assert st in (L.WF_ERR_NO_DEVICE, L.WF_OK)
    else:
        assert st == expect
        assert lib.wf_last_error_message()


# ------------------------------------------------------------------ BlockKVCache

def _cache(lib, L_=8, chunk=2, window=6, sink=2, seq_dim=2):
    shape = [1, 2, L_, 4] if seq_dim == 2 else [1, L_, 2, 4]
    h = ctypes.c_void_p()
    st = lib.wf_kvcache_create(ctypes.byref(_t(shape, L.WF_F32)), ctypes.byref(_t(shape, L.WF_F32)),
                               seq_dim, chunk, sink, window, ctypes.byref(h))
    return st, h


@pytest.mark.parametrize("L_,chunk,window,sink", [(8, 3, 8, 0), (8, 2, 4, 2), (8, 4, 6, 2),
                                                  (8, 2, 0, 8), (8, 0, 8, 0)])
def test_cache_bad_sizes(lib, L_, chunk, window, sink):
    st, h = _cache(lib, L_, chunk, window, sink)
    assert st == L.WF_ERR_INVALID_ARG and not h.value


def test_cache_order_errors_on_host(lib):
    st, h = _cache(lib)
    assert st == L.WF_OK
    state = lambda: _state(lib, h)
    s0 = state()
    assert s0 == (-1, -1, -1, 0, 0)
    assert lib.wf_kvcache_before_update(h, 1) == L.WF_ERR_ORDER        # first must be 0
    assert state() == s0
    kv = _t([1, 2, 2, 4], L.WF_F32)
    assert lib.wf_kvcache_update(h, ctypes.byref(kv), ctypes.byref(kv), None) == L.WF_ERR_ORDER
    qd = _t([1, 2, 2, 4], L.WF_F32)
    assert lib.wf_kvcache_update_attend(h, ctypes.byref(kv), ctypes.byref(kv), ctypes.byref(qd), 2, 0.5,
                                        ctypes.byref(qd), None) == L.WF_ERR_ORDER
    assert lib.wf_kvcache_cached(h, None, None, None) == L.WF_ERR_ORDER
    assert lib.wf_kvcache_after_update(h, 0) == L.WF_ERR_ORDER
    assert state() == s0
    assert lib.wf_kvcache_before_update(h, 0) == L.WF_OK
    assert state() == (0, -1, 0, 0, 1)
    assert lib.wf_kvcache_before_update(h, 0) == L.WF_ERR_ORDER        # twice
    assert lib.wf_kvcache_cached(h, None, None, None) == L.WF_ERR_ORDER  # before update
    assert lib.wf_kvcache_after_update(h, 0) == L.WF_ERR_ORDER         # before cached
    bad = _t([1, 2, 3, 4], L.WF_F32)                                   # not chunk_size positions
    assert lib.wf_kvcache_update(h, ctypes.byref(bad), ctypes.byref(bad), None) == L.WF_ERR_INVALID_ARG
    assert state() == (0, -1, 0, 0, 1)
    lib.wf_kvcache_destroy(h)


def test_cache_set_state_resumes_the_rolling_order(lib):
    """set_state(c) leaves the handle as after_update(c): the next legal
    chunk indices are c (overwrite) and c + 1, the write slot and visible
    length follow the ring; refused while a chunk is in progress."""
    st, h = _cache(lib)                    # L 8, chunk 2, sink 2, window 6: 4 slots
    assert st == L.WF_OK
    assert lib.wf_kvcache_set_state(h, -2) == L.WF_ERR_INVALID_ARG
    assert lib.wf_kvcache_set_state(h, 5) == L.WF_OK
    assert _state(lib, h) == (5, 5, 1 + (5 - 1) % 3, 8, 0)
    assert lib.wf_kvcache_before_update(h, 7) == L.WF_ERR_ORDER
    assert lib.wf_kvcache_before_update(h, 6) == L.WF_OK
    assert _state(lib, h) == (6, 5, 1 + (6 - 1) % 3, 8, 1)
    assert lib.wf_kvcache_set_state(h, 2) == L.WF_ERR_ORDER          # chunk 6 in progress
    assert _state(lib, h) == (6, 5, 1 + (6 - 1) % 3, 8, 1)
    lib.wf_kvcache_destroy(h)
    st, h = _cache(lib)
    assert lib.wf_kvcache_set_state(h, 0) == L.WF_OK
    assert _state(lib, h) == (0, 0, 0, 2, 0)
    assert lib.wf_kvcache_set_state(h, -1) == L.WF_OK                # back to the empty cache
    assert _state(lib, h) == (-1, -1, -1, 0, 0)
    assert lib.wf_kvcache_before_update(h, 1) == L.WF_ERR_ORDER
    assert lib.wf_kvcache_before_update(h, 0) == L.WF_OK
    lib.wf_kvcache_destroy(h)


def _state(lib, h):
    cur, com, slot, vis = (ctypes.c_int64() for _ in range(4))
    ph = ctypes.c_int32()
    assert lib.wf_kvcache_get_state(h, ctypes.byref(cur), ctypes.byref(com), ctypes.byref(slot),
                                    ctypes.byref(vis), ctypes.byref(ph)) == L.WF_OK
    return cur.value, com.value, slot.value, vis.value, ph.value
