"""fp64 CPU oracle for packed-varlen / paged attention (TEST INFRASTRUCTURE).

Only the tests, ``__graft_entry__.smoke()`` and the bench's CPU-baseline leg
import this package.  The product library never loads it, and it shares no
code with the CUDA path.  The arithmetic lives in ``oracle.c`` (plain C,
double precision); this module only marshals arrays into it.

Parity pins for every function here live in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

MASK_NONE, MASK_ALIBI, MASK_ALIBI_SQRT, MASK_ALIBI_LEFT, MASK_CAUSAL = 0, 3, 4, 5, 9

_DTYPE_CODE = {torch.float16: 0, torch.bfloat16: 1, torch.float32: 2, torch.int8: 3}


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", _SRC, "-o", _LIB, "-lm"]
        )
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P, I32, I64, D = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_double
        _lib.oracle_attention.argtypes = [P, ctypes.c_int, P, P, ctypes.c_int, P, I64, I32, P, P, I32, P,
                                          ctypes.c_int, I32, I32, I32, I32, D, P, I64, P, P]
        _lib.oracle_build_mask.argtypes = [ctypes.c_int, P, I32, I64, I64, P]
        _lib.oracle_attention_explicit.argtypes = [P, ctypes.c_int, P, P, ctypes.c_int, I64, I64, I32, I32,
                                                   I32, I32, D, P, P, P]
        _lib.oracle_expand_causal_compressed.argtypes = [P, I64, I64, P]
        _lib.oracle_mla.argtypes = [P, P, P, P, ctypes.c_int, P, I64, I32, P, P, I32, I32, I32, I32, D, P, I64,
                                    P, P]
        _lib.oracle_mla_dequant.argtypes = [P, ctypes.c_int, P, ctypes.c_int, P, ctypes.c_int, P, P, P, P, I64,
                                            I32, P, P, I32, I32, I32, I32, D, P, ctypes.c_int, I64, P, I64, P, P]
        _lib.oracle_lse_merge.argtypes = [I32, I64, I32, P, P, P, P]
        _lib.oracle_decode.argtypes = [P, ctypes.c_int, I64, P]
        for f in ("oracle_attention", "oracle_build_mask", "oracle_attention_explicit",
                  "oracle_expand_causal_compressed", "oracle_mla", "oracle_mla_dequant", "oracle_lse_merge",
                  "oracle_decode"):
            getattr(_lib, f).restype = ctypes.c_int
    return _lib


def _raw(t: torch.Tensor):
    """Stored bits of a CPU tensor as a contiguous numpy array plus its dtype code."""
    t = t.detach().cpu().contiguous()
    code = _DTYPE_CODE[t.dtype]
    arr = t.view(torch.int16).numpy() if t.dtype in (torch.float16, torch.bfloat16) else t.numpy()
    return np.ascontiguousarray(arr), code


_F64 = 4


def _decoded(t: torch.Tensor):
    """The stored elements of a CPU tensor decoded to float64 by oracle.c (exact), with the F64 code."""
    raw, code = _raw(t)
    out = np.empty(raw.size, dtype=np.float64)
    _load().oracle_decode(raw.ctypes.data_as(ctypes.c_void_p), code, raw.size, out.ctypes.data_as(ctypes.c_void_p))
    return out, _F64


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _i32(x):
    return None if x is None else np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def attention(q, k, v, seq_len, kv_seq_len, mask_type, heads, kv_heads, qk_scale, slopes=None,
              block_tables=None, block_size=0, rows=None):
    """Rule-based masked attention in fp64.

    q: [nTokens, heads, d_qk]; k, v: contiguous [nKvTokens, kv_heads, d] or paged
    [numBlocks, blockSize, kv_heads, d] with ``block_tables`` [batch, maxBlockNum].
    Returns (out [n, d_v] float64, lse [n] float64) where n = len(rows) or
    nTokens*heads (row index = token*heads + head).
    """
    lib = _load()
    assert k.dtype == v.dtype
    qa, qc = _decoded(q)
    ka, kc = _decoded(k)
    va, vc = _decoded(v)
    d_qk, d_v = q.shape[-1], v.shape[-1]
    sl, kl = _i32(seq_len), _i32(kv_seq_len)
    bt = _i32(block_tables)
    max_blocks = 0 if bt is None else bt.shape[1]
    sp = None if slopes is None else np.ascontiguousarray(np.asarray(slopes, dtype=np.float32))
    rw = None if rows is None else np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    n = len(rw) if rw is not None else int(sl.sum()) * heads
    out = np.zeros((n, d_v), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    rc = lib.oracle_attention(_ptr(qa), qc, _ptr(ka), _ptr(va), kc, _ptr(bt), max_blocks, block_size,
                              _ptr(sl), _ptr(kl), len(sl), _ptr(sp), mask_type, heads, kv_heads, d_qk, d_v,
                              float(qk_scale), _ptr(rw), 0 if rw is None else len(rw), _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_attention: inconsistent arguments")
    return out, lse


def build_mask(mask_type, slopes, heads, seq_len, kv_len):
    """Full mask M [heads, seq_len, kv_len] (float64, -inf where masked) from the rule."""
    lib = _load()
    m = np.zeros((heads, seq_len, kv_len), dtype=np.float64)
    sp = None if slopes is None else np.ascontiguousarray(np.asarray(slopes, dtype=np.float32))
    if lib.oracle_build_mask(mask_type, _ptr(sp), heads, seq_len, kv_len, _ptr(m)) != 0:
        raise ValueError("oracle_build_mask: kv_len < seq_len")
    return m


def attention_explicit(q, k, v, mask, heads, kv_heads, qk_scale):
    """softmax(qk_scale*QK^T + M)V for one contiguous sequence and a full mask M."""
    lib = _load()
    qa, qc = _raw(q)
    ka, kc = _raw(k)
    va, _ = _raw(v)
    L, Lkv = q.shape[0], k.shape[0]
    d_qk, d_v = q.shape[-1], v.shape[-1]
    m = np.ascontiguousarray(mask, dtype=np.float64)
    out = np.zeros((L * heads, d_v), dtype=np.float64)
    lse = np.zeros((L * heads,), dtype=np.float64)
    rc = lib.oracle_attention_explicit(_ptr(qa), qc, _ptr(ka), _ptr(va), kc, L, Lkv, heads, kv_heads, d_qk, d_v,
                                       float(qk_scale), _ptr(m), _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_attention_explicit: bad heads")
    return out, lse


def expand_causal_compressed(tri, seq_len, kv_len):
    """Expand a 128x128 compressed causal triangle into the [seq_len, kv_len] mask."""
    lib = _load()
    t = np.ascontiguousarray(tri, dtype=np.float64)
    assert t.shape == (128, 128)
    m = np.zeros((seq_len, kv_len), dtype=np.float64)
    if lib.oracle_expand_causal_compressed(_ptr(t), seq_len, kv_len, _ptr(m)) != 0:
        raise ValueError("kv_len < seq_len")
    return m


def mla(q_nope, q_rope, ct_kv, k_rope, block_tables, block_size, context_lens, q_seq_len, heads, qk_scale,
        rows=None, mask=None):
    """MLA decode/spec attention in fp64: key=[ctKV;kRope], value=ctKV, spec-causal rule.

    With ``mask`` ([tokens, max_seq_len] fp16/bf16 tensor, the MLA page's MASK_TYPE_SPEC mask) every key
    j < contextLens of a token's batch is considered and mask[token, j] is added to its scaled score."""
    if mask is not None:
        return mla_dequant(q_nope, q_rope, ct_kv, k_rope, None, None, block_tables, block_size, context_lens,
                           q_seq_len, heads, qk_scale, rows=rows, mask=mask)
    lib = _load()
    assert q_nope.dtype == q_rope.dtype == ct_kv.dtype == k_rope.dtype
    qn, c1 = _decoded(q_nope)
    qr, _ = _decoded(q_rope)
    ck, _ = _decoded(ct_kv)
    kr, _ = _decoded(k_rope)
    bt = _i32(block_tables)
    cl = _i32(context_lens)
    qs = _i32(q_seq_len) if q_seq_len is not None else np.ones_like(cl)
    d_nope, d_rope = q_nope.shape[-1], q_rope.shape[-1]
    rw = None if rows is None else np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    n = len(rw) if rw is not None else int(qs.sum()) * heads
    out = np.zeros((n, d_nope), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    rc = lib.oracle_mla(_ptr(qn), _ptr(qr), _ptr(ck), _ptr(kr), c1, _ptr(bt), bt.shape[1], block_size, _ptr(cl),
                        _ptr(qs), len(cl), heads, d_nope, d_rope, float(qk_scale), _ptr(rw),
                        0 if rw is None else len(rw), _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_mla: inconsistent arguments")
    return out, lse


def mla_dequant(q_nope, q_rope, ct_kv, k_rope, qk_descale, pv_descale, block_tables, block_size, context_lens,
                q_seq_len, heads, qk_scale, rows=None, mask=None):
    """MLA over an int8 latent cache in fp64 (the MLA page's qkDescale / pvDescale rows):
    s = qkScale * (qkDescale[h] * qNope.ctKV + qRope.kRope), O = pvDescale[h] * softmax(s) ctKV,
    qNope and ctKV taken as stored (int8 or float); a None descale means 1.  ``mask`` as in ``mla``."""
    lib = _load()
    assert q_rope.dtype == k_rope.dtype
    qn, cq = _decoded(q_nope)
    qr, cr = _decoded(q_rope)
    ck, ckv = _decoded(ct_kv)
    kr, _ = _decoded(k_rope)
    qd = None if qk_descale is None else np.ascontiguousarray(np.asarray(qk_descale, dtype=np.float32))
    pd = None if pv_descale is None else np.ascontiguousarray(np.asarray(pv_descale, dtype=np.float32))
    for d in (qd, pd):
        assert d is None or d.shape == (heads,)
    bt = _i32(block_tables)
    cl = _i32(context_lens)
    qs = _i32(q_seq_len) if q_seq_len is not None else np.ones_like(cl)
    d_nope, d_rope = q_nope.shape[-1], q_rope.shape[-1]
    rw = None if rows is None else np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    n = len(rw) if rw is not None else int(qs.sum()) * heads
    out = np.zeros((n, d_nope), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    ma, mc, mcols = None, 0, 0
    if mask is not None:
        assert mask.dim() == 2 and mask.shape[0] == int(qs.sum()) and mask.dtype in (torch.float16, torch.bfloat16)
        ma, mc = _raw(mask)
        mcols = mask.shape[1]
    rc = lib.oracle_mla_dequant(_ptr(qn), cq, _ptr(qr), cr, _ptr(ck), ckv, _ptr(kr), _ptr(qd), _ptr(pd), _ptr(bt),
                                bt.shape[1], block_size, _ptr(cl), _ptr(qs), len(cl), heads, d_nope, d_rope,
                                float(qk_scale), _ptr(ma), mc, mcols, _ptr(rw), 0 if rw is None else len(rw),
                                _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_mla_dequant: inconsistent arguments")
    return out, lse


def lse_merge(o_parts, lse_parts):
    """Combine partial (O_p, lse_p) over disjoint key ranges: o_parts [P, n, d], lse_parts [P, n]."""
    lib = _load()
    o = np.ascontiguousarray(o_parts, dtype=np.float64)
    s = np.ascontiguousarray(lse_parts, dtype=np.float64)
    P, n, d = o.shape
    out = np.zeros((n, d), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    lib.oracle_lse_merge(P, n, d, _ptr(o), _ptr(s), _ptr(out), _ptr(lse))
    return out, lse
