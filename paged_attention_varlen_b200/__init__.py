"""Python binding of libala.so: packed-varlen / paged attention on B200 (sm_100a).

Argument marshalling only.  Every step of the computation runs in the CUDA
kernels behind the C ABI declared in ``include/ala.h``; there is no CPU or
PyTorch fallback.  If the shared library is missing the calls raise.

Entry points (names as in the C ABI):
  * ``varlen_attention``         contiguous packed K/V, mask types 0/3/4/5/9
  * ``atb_like_prefix_encoder``  paged K/V through blockTables, mask types 3/4/5/9
  * ``atb_like_mla``             MLA decode / speculative decode over a paged latent cache

Each returns an ``Op`` that owns the workspace and can be executed again on
the current CUDA stream (``op()``), which is what the bench does.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# ALA_LIBRARY=debug selects libala_debug.so: the same kernels with every block-table entry range-checked
LIB_PATH = os.path.join(_HERE, "libala_debug.so" if os.environ.get("ALA_LIBRARY") == "debug" else "libala.so")

F16, BF16, F32, I32, I8 = 0, 1, 2, 3, 4
MASK_NONE, MASK_ALIBI, MASK_ALIBI_SQRT, MASK_ALIBI_LEFT, MASK_CAUSAL = 0, 3, 4, 5, 9
MLA_MASK_UNDEFINED, MLA_MASK_SPEC, MLA_MASK_FREE = 0, 1, 2
MLA_CALC_UNDEFINED, MLA_CALC_SPEC, MLA_CALC_RING, MLA_CALC_PREFILL = 0, 1, 2, 3
MLA_CACHE_KVCACHE, MLA_CACHE_KROPE_CTKV, MLA_CACHE_INT8_NZ, MLA_CACHE_NZ = 0, 1, 2, 3

STATUS = {0: "OK", 1: "NULL_REQUIRED", 2: "INVALID_SHAPE", 3: "INVALID_DTYPE", 4: "INVALID_PARAM",
          5: "UNSUPPORTED", 6: "WORKSPACE_TOO_SMALL", 7: "CUDA_ERROR", 8: "DEVICE_TIMEOUT"}

_TORCH_DTYPE = {torch.float16: F16, torch.bfloat16: BF16, torch.float32: F32, torch.int32: I32, torch.int8: I8}
_NP_DTYPE = {np.dtype(np.int32): I32, np.dtype(np.float32): F32}


class AlaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


class AlaTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("ndim", ctypes.c_int32),
                ("dims", ctypes.c_int64 * 4)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libala.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m paged_attention_varlen_b200.build`"
                               " (add --debug-bounds for libala_debug.so)")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.c_void_p
        T = ctypes.POINTER(AlaTensor)
        OPP = ctypes.POINTER(ctypes.c_void_p)
        U64P = ctypes.POINTER(ctypes.c_uint64)
        L.ala_last_error.restype = ctypes.c_char_p
        L.ala_op_destroy.argtypes = [P]
        L.ala_op_destroy.restype = None
        L.ala_workspace_status.argtypes = [P, P, P, ctypes.POINTER(ctypes.c_int32)]
        L.atb_like_prefix_encoder_get_workspace_size.argtypes = [T, T, T, T, T, T, T, T, ctypes.c_int, ctypes.c_int32,
                                                                 ctypes.c_int32, ctypes.c_float, T, U64P, OPP]
        L.varlen_attention_get_workspace_size.argtypes = [T, T, T, T, T, T, ctypes.c_int, ctypes.c_int32,
                                                          ctypes.c_int32, ctypes.c_float, T, T, U64P, OPP]
        L.atb_like_mla_get_workspace_size.argtypes = [T, T, T, T, T, T, T, T, T, T, ctypes.c_int32, ctypes.c_float,
                                                      ctypes.c_int32, ctypes.c_int, ctypes.c_int, ctypes.c_uint8, T, T,
                                                      U64P, OPP]
        L.varlen_attention_noalloc.argtypes = [T, T, T, T, T, T, ctypes.c_int, ctypes.c_int32, ctypes.c_int32,
                                               ctypes.c_float, T, T, P]
        L.varlen_attention_noalloc.restype = ctypes.c_int
        L.varlen_attention_noalloc_status.argtypes = [P, ctypes.POINTER(ctypes.c_int32)]
        L.varlen_attention_noalloc_status.restype = ctypes.c_int
        L.atb_like_prefix_encoder_lse_get_workspace_size.argtypes = [T, T, T, T, T, T, T, T, ctypes.c_int,
                                                                     ctypes.c_int32, ctypes.c_int32, ctypes.c_float,
                                                                     T, T, U64P, OPP]
        L.atb_like_prefix_encoder_lse_get_workspace_size.restype = ctypes.c_int
        L.ala_op_bind_workspace.argtypes = [P, P, ctypes.c_uint64, P]
        L.ala_op_bind_workspace.restype = ctypes.c_int
        L.ala_lse_merge.argtypes = [T, T, T, T, T, T, P]
        L.ala_lse_merge.restype = ctypes.c_int
        for f in ("atb_like_prefix_encoder", "varlen_attention", "atb_like_mla"):
            getattr(L, f).argtypes = [P, ctypes.c_uint64, P, P]
        for f in ("ala_workspace_status", "atb_like_prefix_encoder_get_workspace_size",
                  "varlen_attention_get_workspace_size", "atb_like_mla_get_workspace_size",
                  "atb_like_prefix_encoder", "varlen_attention", "atb_like_mla"):
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


def _check(status: int):
    if status != 0:
        raise AlaError(status, lib().ala_last_error().decode())


def tensor(x) -> AlaTensor | None:
    """Describe a torch tensor or numpy array (contiguous) as an ala_tensor; None -> NULL."""
    if x is None:
        return None
    if isinstance(x, np.ndarray):
        assert x.flags["C_CONTIGUOUS"]
        dt, ptr, shape = _NP_DTYPE[x.dtype], x.ctypes.data, x.shape
    else:
        assert x.is_contiguous(), "tensors passed to libala must be contiguous"
        dt, ptr, shape = _TORCH_DTYPE[x.dtype], x.data_ptr(), tuple(x.shape)
    assert 1 <= len(shape) <= 4
    t = AlaTensor()
    t.data = ptr
    t.dtype = dt
    t.ndim = len(shape)
    for i, s in enumerate(shape):
        t.dims[i] = s
    return t


def _ref(t):
    return None if t is None else ctypes.byref(t)


def _host_i32(x) -> np.ndarray:
    if isinstance(x, torch.Tensor):
        x = x.cpu().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


class Op:
    """A planned call: owns the op handle, its workspace and references to its tensors."""

    def __init__(self, handle, ws_size, execute_fn, device, keep):
        self._handle = handle
        self._execute = execute_fn
        self.workspace = torch.empty(max(int(ws_size), 256), dtype=torch.uint8, device=device)
        self.workspace_size = int(ws_size)
        self._keep = keep
        self._bound = False

    def __call__(self, stream: torch.cuda.Stream | None = None):
        s = stream if stream is not None else torch.cuda.current_stream(self.workspace.device)
        ws = ctypes.c_void_p(self.workspace.data_ptr())
        if not self._bound:
            # the workspace belongs to this Op alone: the schedule is copied into it once (ala_op_bind_workspace)
            _check(lib().ala_op_bind_workspace(self._handle, ws, self.workspace_size, ctypes.c_void_p(s.cuda_stream)))
            self._bound = True
        _check(self._execute(ws, self.workspace_size, self._handle, ctypes.c_void_p(s.cuda_stream)))
        return self

    def device_status(self) -> int:
        code = ctypes.c_int32(0)
        s = torch.cuda.current_stream(self.workspace.device)
        _check(lib().ala_workspace_status(self._handle, ctypes.c_void_p(self.workspace.data_ptr()),
                                          ctypes.c_void_p(s.cuda_stream), ctypes.byref(code)))
        if code.value != 0:
            self._bound = False  # a recorded failure stays in a bound workspace: the next call binds it afresh
        return code.value

    def __del__(self):
        if getattr(self, "_handle", None) and _lib is not None:
            _lib.ala_op_destroy(self._handle)
            self._handle = None


def plan_varlen_attention(q, k, v, seq_len, kv_seq_len, mask_type, heads, kv_heads, qk_scale, slopes=None,
                          out=None, lse=None) -> tuple[Op, torch.Tensor]:
    """Plan contiguous packed-varlen attention; returns (op, out).  Call op() to run."""
    L = lib()
    out = torch.empty_like(q) if out is None else out
    sl, kl = _host_i32(seq_len), _host_i32(kv_seq_len)
    ts = [tensor(q), tensor(k), tensor(v), tensor(sl), tensor(kl), tensor(slopes)]
    to, tl = tensor(out), tensor(lse)
    ws = ctypes.c_uint64(0)
    h = ctypes.c_void_p(0)
    _check(L.varlen_attention_get_workspace_size(*[_ref(t) for t in ts], int(mask_type), int(heads), int(kv_heads),
                                                 float(qk_scale), _ref(to), _ref(tl), ctypes.byref(ws),
                                                 ctypes.byref(h)))
    return Op(h, ws.value, L.varlen_attention, q.device, (q, k, v, sl, kl, slopes, out, lse)), out


def varlen_attention(q, k, v, seq_len, kv_seq_len, mask_type, heads, kv_heads, qk_scale, slopes=None,
                     return_lse=False):
    """O (and optionally the fp32 lse [nTokens, heads]) for contiguous packed K/V."""
    lse = torch.empty((q.shape[0], heads), dtype=torch.float32, device=q.device) if return_lse else None
    op, out = plan_varlen_attention(q, k, v, seq_len, kv_seq_len, mask_type, heads, kv_heads, qk_scale, slopes,
                                    lse=lse)
    op()
    return (out, lse) if return_lse else out


def varlen_attention_noalloc(q, k, v, seq_len, kv_seq_len, mask_type, heads, kv_heads, qk_scale, slopes=None,
                             out=None, lse=None, stream=None):
    """varlen_attention through the entry point that allocates nothing on the device.

    For callers that cannot allocate device memory: no workspace is passed; the
    library's fixed device scratch holds the schedule.  ``out`` (and ``lse``)
    must be supplied by the caller or are created here with torch.  A stream
    that is being captured is refused (AlaError, UNSUPPORTED).
    """
    L = lib()
    out = torch.empty_like(q) if out is None else out
    sl, kl = _host_i32(seq_len), _host_i32(kv_seq_len)
    s = stream if stream is not None else torch.cuda.current_stream(q.device)
    ts = [tensor(q), tensor(k), tensor(v), tensor(sl), tensor(kl), tensor(slopes)]
    to, tl = tensor(out), tensor(lse)
    _check(L.varlen_attention_noalloc(*[_ref(t) for t in ts], int(mask_type), int(heads), int(kv_heads),
                                      float(qk_scale), _ref(to), _ref(tl), ctypes.c_void_p(s.cuda_stream)))
    return out


def varlen_attention_noalloc_status(stream=None, device=None) -> int:
    """Status word of the last varlen_attention_noalloc call (0: every kernel wait completed)."""
    s = stream if stream is not None else torch.cuda.current_stream(device)
    code = ctypes.c_int32(0)
    _check(lib().varlen_attention_noalloc_status(ctypes.c_void_p(s.cuda_stream), ctypes.byref(code)))
    return code.value


def plan_prefix_encoder(q, k, v, block_tables, seq_len, kv_seq_len, mask_type, heads, kv_heads, qk_scale,
                        slopes=None, mask=None, out=None, lse=None) -> tuple[Op, torch.Tensor]:
    """Plan the paged PrefixEncoder call; returns (op, out).  With ``lse`` ([nTokens, heads] fp32) the
    lse-returning entry point is used."""
    L = lib()
    out = torch.empty_like(q) if out is None else out
    sl, kl = _host_i32(seq_len), _host_i32(kv_seq_len)
    ts = [tensor(q), tensor(k), tensor(v), tensor(block_tables), tensor(mask), tensor(sl), tensor(kl),
          tensor(slopes)]
    to = tensor(out)
    ws = ctypes.c_uint64(0)
    h = ctypes.c_void_p(0)
    if lse is None:
        _check(L.atb_like_prefix_encoder_get_workspace_size(*[_ref(t) for t in ts], int(mask_type), int(heads),
                                                            int(kv_heads), float(qk_scale), _ref(to),
                                                            ctypes.byref(ws), ctypes.byref(h)))
    else:
        _check(L.atb_like_prefix_encoder_lse_get_workspace_size(*[_ref(t) for t in ts], int(mask_type), int(heads),
                                                                int(kv_heads), float(qk_scale), _ref(to),
                                                                _ref(tensor(lse)), ctypes.byref(ws), ctypes.byref(h)))
    return Op(h, ws.value, L.atb_like_prefix_encoder, q.device,
              (q, k, v, block_tables, mask, sl, kl, slopes, out, lse)), out


def atb_like_prefix_encoder(q, k, v, block_tables, seq_len, kv_seq_len, mask_type, heads, kv_heads, qk_scale,
                            slopes=None, mask=None):
    op, out = plan_prefix_encoder(q, k, v, block_tables, seq_len, kv_seq_len, mask_type, heads, kv_heads,
                                  qk_scale, slopes, mask)
    op()
    return out


def plan_mla(q_nope, q_rope, ct_kv, k_rope, block_tables, context_lens, q_seq_len, heads, qk_scale,
             mask_type=MLA_MASK_UNDEFINED, calc_type=MLA_CALC_UNDEFINED, cache_mode=None,
             lse=None, out=None, kv_heads=1, qk_descale=None, pv_descale=None, mask=None) -> tuple[Op, torch.Tensor]:
    """Plan the MLA decode/spec call; returns (op, attenOut).

    An int8 ``ct_kv`` selects the int8 latent cache (cacheMode INT8_NZCACHE, ND layout) and needs
    ``qk_descale`` / ``pv_descale`` ([heads] fp32 on the device); ``q_nope`` may then be int8 too.
    ``mask`` ([tokens, maxSeqLen] fp16/bf16 on the device, maskType SPEC) is added to the scaled scores
    of every key below contextLens in place of the generated speculative rule.
    """
    L = lib()
    if cache_mode is None:
        cache_mode = MLA_CACHE_INT8_NZ if ct_kv.dtype == torch.int8 else MLA_CACHE_KROPE_CTKV
    out = (torch.empty(q_rope.shape[:-1] + (q_nope.shape[-1],), dtype=q_rope.dtype, device=q_rope.device)
           if out is None else out)
    cl = _host_i32(context_lens)
    qs = None if q_seq_len is None else _host_i32(q_seq_len)
    ts = [tensor(q_nope), tensor(q_rope), tensor(ct_kv), tensor(k_rope), tensor(block_tables), tensor(cl),
          tensor(mask), tensor(qs), tensor(qk_descale), tensor(pv_descale)]
    to, tl = tensor(out), tensor(lse)
    ws = ctypes.c_uint64(0)
    h = ctypes.c_void_p(0)
    _check(L.atb_like_mla_get_workspace_size(*[_ref(t) for t in ts], int(heads), float(qk_scale), int(kv_heads),
                                             int(mask_type), int(calc_type), int(cache_mode), _ref(to), _ref(tl),
                                             ctypes.byref(ws), ctypes.byref(h)))
    return Op(h, ws.value, L.atb_like_mla, q_nope.device,
              (q_nope, q_rope, ct_kv, k_rope, block_tables, cl, qs, out, lse, qk_descale, pv_descale, mask)), out


def atb_like_mla(q_nope, q_rope, ct_kv, k_rope, block_tables, context_lens, q_seq_len, heads, qk_scale,
                 mask_type=MLA_MASK_UNDEFINED, calc_type=MLA_CALC_UNDEFINED, return_lse=False, qk_descale=None,
                 pv_descale=None, mask=None):
    return_lse = return_lse or calc_type == MLA_CALC_RING  # ring mode always returns the lse
    lse = (torch.empty((q_nope.shape[0], heads, 1), dtype=torch.float32, device=q_nope.device)
           if return_lse else None)
    op, out = plan_mla(q_nope, q_rope, ct_kv, k_rope, block_tables, context_lens, q_seq_len, heads, qk_scale,
                       mask_type, calc_type, lse=lse, qk_descale=qk_descale, pv_descale=pv_descale, mask=mask)
    op()
    return (out, lse) if return_lse else out


def lse_merge(out_a, lse_a, out_b, lse_b, out=None, lse=None, stream=None):
    """Merge two partial results over disjoint key ranges by their lse (ala_lse_merge).

    ``out`` / ``lse`` default to new tensors; passing ``out_a`` / ``lse_a`` merges in place.
    Returns (out, lse).
    """
    L = lib()
    out = torch.empty_like(out_a) if out is None else out
    lse = torch.empty_like(lse_a) if lse is None else lse
    s = stream if stream is not None else torch.cuda.current_stream(out_a.device)
    ts = [tensor(out_a), tensor(lse_a), tensor(out_b), tensor(lse_b), tensor(out), tensor(lse)]
    _check(L.ala_lse_merge(*[_ref(t) for t in ts], ctypes.c_void_p(s.cuda_stream)))
    return out, lse
