"""The C ABI without a GPU: the library loads, exports every declared symbol, and
rejects bad arguments with the documented status before touching the device."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import paged_attention_varlen_b200 as ala

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    from paged_attention_varlen_b200 import build
    build.build()


def _declared():
    text = open(os.path.join(ROOT, "include", "ala.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:ALA_API\s+)?(?:const\s+)?\w+\*?\s+\**(\w+)\s*\(", text, flags=re.M)))


def test_every_declared_symbol_is_exported():
    names = _declared()
    assert {"atb_like_prefix_encoder", "atb_like_mla", "varlen_attention", "ala_last_error"} <= set(names)
    L = ctypes.CDLL(ala.LIB_PATH)
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/ala.h but not exported"


def _varlen_args(**over):
    a = dict(q=torch.zeros(10, 4, 128, dtype=torch.bfloat16), k=torch.zeros(14, 2, 128, dtype=torch.bfloat16),
             v=torch.zeros(14, 2, 128, dtype=torch.bfloat16), seq_len=[4, 6], kv_seq_len=[6, 8], mask_type=9,
             heads=4, kv_heads=2, qk_scale=0.1, slopes=None)
    a.update(over)
    return a


def _plan_varlen(**over):
    a = _varlen_args(**over)
    return ala.plan_varlen_attention(a["q"], a["k"], a["v"], a["seq_len"], a["kv_seq_len"], a["mask_type"],
                                     a["heads"], a["kv_heads"], a["qk_scale"], a["slopes"])


def test_valid_plan_needs_no_gpu():
    op, out = _plan_varlen()
    assert op.workspace_size > 0 and out.shape == (10, 4, 128)


def test_bind_workspace_refusals_need_no_gpu():
    op, _ = _plan_varlen()
    L = ala.lib()
    fake = ctypes.c_void_p(1 << 20)
    assert L.ala_op_bind_workspace(None, fake, op.workspace_size, None) == 1           # op NULL
    assert L.ala_op_bind_workspace(op._handle, fake, op.workspace_size - 1, None) == 6  # too small
    assert L.ala_op_bind_workspace(op._handle, ctypes.c_void_p((1 << 20) + 8), op.workspace_size, None) == 4
    assert L.ala_op_bind_workspace(op._handle, None, 0, None) == 0                     # unbinding is host-only


def test_output_must_be_32_byte_aligned():
    # the kernel writes output rows in 32-byte pieces: a 16-byte-aligned output is refused on the host
    a = _varlen_args()
    q = a["q"]
    buf = torch.zeros(q.numel() + 8, dtype=q.dtype)
    out = buf[8:].view(q.shape)  # 16 bytes past a 256-byte boundary
    assert out.data_ptr() % 32 == 16
    with pytest.raises(ala.AlaError) as e:
        ala.plan_varlen_attention(q, a["k"], a["v"], a["seq_len"], a["kv_seq_len"], a["mask_type"], a["heads"],
                                  a["kv_heads"], a["qk_scale"], a["slopes"], out=out)
    assert e.value.status == 4 and "32-byte" in str(e.value)


@pytest.mark.parametrize("over,status", [
    (dict(heads=0), 4),                                          # headNum must be > 0
    (dict(kv_heads=3), 4),                                       # kvHeadNum must divide headNum
    (dict(mask_type=7), 4),                                      # maskType not in {0,3,4,5,9}
    (dict(kv_seq_len=[3, 8]), 4),                                # kvSeqLen < seqLen
    (dict(seq_len=[4, 5], kv_seq_len=[6, 8]), 2),                # sum(seqLen) != nTokens
    (dict(kv_seq_len=[6, 9]), 2),                                # sum(kvSeqLen) != nKvTokens
    (dict(mask_type=3), 1),                                      # ALiBi needs slopes
    (dict(slopes=np.ones(4, np.float32)), 4),                    # causal forbids slopes
    (dict(mask_type=3, slopes=np.ones(3, np.float32)), 2),       # slopes must be [headNum]
    (dict(k=torch.zeros(14, 2, 128, dtype=torch.float16)), 3),   # dtype mismatch
    (dict(q=torch.zeros(10, 4, 68, dtype=torch.bfloat16), k=torch.zeros(14, 2, 68, dtype=torch.bfloat16),
          v=torch.zeros(14, 2, 68, dtype=torch.bfloat16)), 5),     # headSize not a multiple of 8
    (dict(q=torch.zeros(10, 4, 272, dtype=torch.bfloat16), k=torch.zeros(14, 2, 272, dtype=torch.bfloat16),
          v=torch.zeros(14, 2, 272, dtype=torch.bfloat16)), 5),    # headSize > 256 is not built
    (dict(q=torch.zeros(10, 4, 96, dtype=torch.float32), k=torch.zeros(14, 2, 96, dtype=torch.float32),
          v=torch.zeros(14, 2, 96, dtype=torch.float32)), 5),      # fp32 up to 64
    (dict(q=torch.zeros(10, 4, 256, dtype=torch.bfloat16), k=torch.zeros(14, 2, 256, dtype=torch.bfloat16),
          v=torch.zeros(14, 2, 256, dtype=torch.bfloat16), mask_type=3, slopes=np.ones(4, np.float32)), 4),
    (dict(q=torch.zeros(10, 4, 128), k=torch.zeros(14, 2, 128), v=torch.zeros(14, 2, 128)), 5),  # f32 d=128
])
def test_varlen_rejects(over, status):
    with pytest.raises(ala.AlaError) as e:
        _plan_varlen(**over)
    assert e.value.status == status, str(e.value)


def _prefix_args():
    bs, nb = 16, 8
    return dict(q=torch.zeros(10, 4, 128, dtype=torch.float16), k=torch.zeros(nb, bs, 2, 128, dtype=torch.float16),
                v=torch.zeros(nb, bs, 2, 128, dtype=torch.float16),
                block_tables=torch.zeros(2, 2, dtype=torch.int32), seq_len=[4, 6], kv_seq_len=[20, 30],
                mask_type=3, heads=4, kv_heads=2, qk_scale=0.1, slopes=torch.ones(4), mask=None)


def _plan_prefix(**over):
    a = _prefix_args()
    a.update(over)
    return ala.plan_prefix_encoder(a["q"], a["k"], a["v"], a["block_tables"], a["seq_len"], a["kv_seq_len"],
                                   a["mask_type"], a["heads"], a["kv_heads"], a["qk_scale"], a["slopes"], a["mask"])


def test_prefix_plan_ok_and_mask_tensor_accepted():
    _plan_prefix()
    for bs in (48, 80, 144):  # any multiple of 16 (K/V boxes of gcd(blockSize, 128) rows)
        _plan_prefix(k=torch.zeros(8, bs, 2, 128, dtype=torch.float16), v=torch.zeros(8, bs, 2, 128, dtype=torch.float16))
    _plan_prefix(mask=torch.zeros(256, 256, dtype=torch.float16))
    _plan_prefix(mask=torch.zeros(4, 4, 128, dtype=torch.float16), mask_type=4)


@pytest.mark.parametrize("over,status", [
    (dict(mask_type=0, slopes=None), 4),                                      # PrefixEncoder: 3/4/5/9 only
    (dict(mask_type=9), 4),                                                   # slopes must be NULL for causal
    (dict(mask_type=5, mask=torch.zeros(256, 256, dtype=torch.float16)), 4),  # mask NULL for 5/9
    (dict(mask=torch.zeros(128, 128, dtype=torch.float16)), 2),               # mask shape
    (dict(kv_seq_len=[20, 40]), 4),                                           # needs 3 blocks > maxBlockNum 2
    (dict(block_tables=torch.zeros(3, 2, dtype=torch.int32)), 2),             # rows != batch
    (dict(k=torch.zeros(8, 24, 2, 128, dtype=torch.float16), v=torch.zeros(8, 24, 2, 128, dtype=torch.float16)), 5),
    (dict(q=torch.zeros(10, 4, 128), k=torch.zeros(8, 16, 2, 128), v=torch.zeros(8, 16, 2, 128)), 3),  # f32
    (dict(block_tables=None), 1),
])
def test_prefix_rejects(over, status):
    with pytest.raises(ala.AlaError) as e:
        _plan_prefix(**over)
    assert e.value.status == status, str(e.value)


def _mla_args():
    nb, bs, H = 6, 64, 128
    return dict(q_nope=torch.zeros(3, H, 512, dtype=torch.bfloat16), q_rope=torch.zeros(3, H, 64, dtype=torch.bfloat16),
                ct_kv=torch.zeros(nb, bs, 1, 512, dtype=torch.bfloat16),
                k_rope=torch.zeros(nb, bs, 1, 64, dtype=torch.bfloat16),
                block_tables=torch.zeros(3, 2, dtype=torch.int32), context_lens=[5, 100, 128], q_seq_len=None,
                heads=H, qk_scale=0.04, mask_type=0, calc_type=0, cache_mode=1, kv_heads=1)


def _plan_mla(**over):
    a = _mla_args()
    a.update(over)
    return ala.plan_mla(a["q_nope"], a["q_rope"], a["ct_kv"], a["k_rope"], a["block_tables"], a["context_lens"],
                        a["q_seq_len"], a["heads"], a["qk_scale"], a["mask_type"], a["calc_type"], a["cache_mode"],
                        kv_heads=a["kv_heads"], lse=a.get("lse"), qk_descale=a.get("qk_descale"),
                        pv_descale=a.get("pv_descale"), mask=a.get("mask"))


def _int8_cache(**over):
    # the int8 latent cache (cacheMode 2): int8 ctKV (and qNope) with per-head fp32 descales
    d = dict(ct_kv=torch.zeros(6, 64, 1, 512, dtype=torch.int8), q_nope=torch.zeros(3, 128, 512, dtype=torch.int8),
             cache_mode=2, qk_descale=torch.ones(128), pv_descale=torch.ones(128))
    d.update(over)
    return d


def test_mla_plan_ok():
    _plan_mla()
    for bs in (80, 112, 144):  # any multiple of 16 (cache boxes of gcd(blockSize, 64) rows)
        _plan_mla(ct_kv=torch.zeros(6, bs, 1, 512, dtype=torch.bfloat16),
                  k_rope=torch.zeros(6, bs, 1, 64, dtype=torch.bfloat16))
    _plan_mla(q_nope=torch.zeros(6, 128, 512, dtype=torch.bfloat16), q_rope=torch.zeros(6, 128, 64, dtype=torch.bfloat16),
              q_seq_len=[2, 2, 2], mask_type=1, calc_type=1)


def test_mla_prefill_plans_with_qseqlen():
    _plan_mla(q_nope=torch.zeros(9, 128, 512, dtype=torch.bfloat16), q_rope=torch.zeros(9, 128, 64, dtype=torch.bfloat16),
              q_seq_len=[1, 5, 3], calc_type=3)
    _plan_mla(q_nope=torch.zeros(9, 128, 512, dtype=torch.bfloat16), q_rope=torch.zeros(9, 128, 64, dtype=torch.bfloat16),
              q_seq_len=[1, 5, 3], calc_type=3, mask_type=1)


def test_mla_int8_cache_plans():
    _plan_mla(**_int8_cache())
    _plan_mla(**_int8_cache(q_nope=torch.zeros(3, 128, 512, dtype=torch.bfloat16)))  # float qNope
    _plan_mla(**_int8_cache(q_nope=torch.zeros(6, 128, 512, dtype=torch.int8),
                            q_rope=torch.zeros(6, 128, 64, dtype=torch.bfloat16), q_seq_len=[2, 2, 2], mask_type=1,
                            calc_type=1))


@pytest.mark.parametrize("over,status", [
    (dict(qk_descale=None), 1),                                          # both descales are required
    (dict(pv_descale=None), 1),
    (dict(qk_descale=torch.ones(64)), 2),                                # one per head
    (dict(pv_descale=torch.ones(128, dtype=torch.float16)), 3),          # fp32
    (dict(ct_kv=torch.zeros(6, 64, 1, 512, dtype=torch.bfloat16)), 3),   # cacheMode 2 holds int8 codes
    (dict(q_nope=torch.zeros(3, 128, 512, dtype=torch.float16)), 3),     # qNope: int8 or qRope's dtype
    (dict(cache_mode=1), 4),                                             # descales only with cacheMode 2
])
def test_mla_int8_cache_rejects(over, status):
    with pytest.raises(ala.AlaError) as e:
        _plan_mla(**_int8_cache(**over))
    assert e.value.status == status, str(e.value)


def test_mla_int8_codes_need_cache_mode_2():
    with pytest.raises(ala.AlaError) as e:
        _plan_mla(ct_kv=torch.zeros(6, 64, 1, 512, dtype=torch.int8))
    assert e.value.status == 3
    with pytest.raises(ala.AlaError) as e:
        _plan_mla(q_nope=torch.zeros(3, 128, 512, dtype=torch.int8))
    assert e.value.status == 3


def test_mla_ring_plans_with_lse():
    # ring mode computes the same attention and requires the lse it is merged with
    lse = torch.zeros(3, 128, 1, dtype=torch.float32)
    _plan_mla(calc_type=2, lse=lse)
    _plan_mla(q_nope=torch.zeros(6, 128, 512, dtype=torch.bfloat16), q_rope=torch.zeros(6, 128, 64, dtype=torch.bfloat16),
              q_seq_len=[2, 2, 2], mask_type=1, calc_type=2, lse=torch.zeros(6, 128, 1, dtype=torch.float32))


def test_prefix_encoder_lse_entry_requires_lse():
    L = ala.lib()
    q = torch.zeros(4, 2, 128, dtype=torch.float16)
    kv = torch.zeros(2, 64, 2, 128, dtype=torch.float16)
    bt = torch.zeros(1, 2, dtype=torch.int32)
    sl = np.array([4], dtype=np.int32)
    kl = np.array([70], dtype=np.int32)
    ts = [ala.tensor(x) for x in (q, kv, kv, bt)] + [None] + [ala.tensor(sl), ala.tensor(kl), None]
    ws = ctypes.c_uint64(0)
    h = ctypes.c_void_p(0)
    args = [ala._ref(t) for t in ts] + [9, 2, 2, ctypes.c_float(0.1), ala._ref(ala.tensor(q))]
    st = L.atb_like_prefix_encoder_lse_get_workspace_size(*args, None, ctypes.byref(ws), ctypes.byref(h))
    assert st == 1
    lse = torch.zeros(4, 2, dtype=torch.float32)
    st = L.atb_like_prefix_encoder_lse_get_workspace_size(*args, ala._ref(ala.tensor(lse)), ctypes.byref(ws),
                                                          ctypes.byref(h))
    assert st == 0, L.ala_last_error().decode()
    L.ala_op_destroy(h)
    bad = torch.zeros(4, 3, dtype=torch.float32)  # one value per (token, head)
    st = L.atb_like_prefix_encoder_lse_get_workspace_size(*args, ala._ref(ala.tensor(bad)), ctypes.byref(ws),
                                                          ctypes.byref(h))
    assert st == 2


def _merge_args(n=4, d=512, dtype=torch.bfloat16):
    return dict(out_a=torch.zeros(n, 2, d, dtype=dtype), lse_a=torch.zeros(n, 2, 1), out_b=torch.zeros(n, 2, d, dtype=dtype),
                lse_b=torch.zeros(n, 2, 1), out=torch.zeros(n, 2, d, dtype=dtype), lse=torch.zeros(n, 2, 1))


@pytest.mark.parametrize("over,status", [
    (dict(out_b=torch.zeros(4, 2, 256, dtype=torch.bfloat16)), 2),   # shapes differ
    (dict(out=torch.zeros(4, 2, 512, dtype=torch.float16)), 3),      # dtypes differ
    (dict(lse_b=torch.zeros(4, 2, 1, dtype=torch.float16)), 3),      # lse must be fp32
    (dict(lse=torch.zeros(4, 3, 1)), 2),                             # one lse per row
    (dict(out_a=torch.zeros(4, 2, 2048, dtype=torch.bfloat16), out_b=torch.zeros(4, 2, 2048, dtype=torch.bfloat16),
          out=torch.zeros(4, 2, 2048, dtype=torch.bfloat16)), 2),    # d <= 1024
    (dict(out_a=torch.zeros(4, 2, 512, dtype=torch.int32), out_b=torch.zeros(4, 2, 512, dtype=torch.int32),
          out=torch.zeros(4, 2, 512, dtype=torch.int32)), 3),        # outputs are floating point
])
def test_lse_merge_rejects(over, status):
    # all checks run before any GPU work, so host tensors are enough here
    a = _merge_args()
    a.update(over)
    L = ala.lib()
    ts = [ala.tensor(a[k]) for k in ("out_a", "lse_a", "out_b", "lse_b", "out", "lse")]
    st = L.ala_lse_merge(*[ala._ref(t) for t in ts], None)
    assert st == status, ala.lib().ala_last_error().decode()


def test_lse_merge_null_tensor():
    a = _merge_args()
    L = ala.lib()
    ts = [ala.tensor(a[k]) for k in ("out_a", "lse_a", "out_b", "lse_b", "out")]
    assert L.ala_lse_merge(*[ala._ref(t) for t in ts], None, None) == 1


@pytest.mark.parametrize("over,status", [
    (dict(cache_mode=0), 5), (dict(cache_mode=3), 5),
    (dict(cache_mode=2), 1),                       # the int8 cache needs its descales
    (dict(calc_type=2), 1),                        # RING needs lse
    (dict(calc_type=3), 1),                        # PREFILL needs qseqlen
    (dict(calc_type=3, q_seq_len=[1, 1, 1], mask_type=2), 4),  # PREFILL is causal: UNDEFINED or SPEC only
    (dict(mask_type=3), 4),                        # ALiBi only on the encoder paths
    (dict(kv_heads=2), 5),
    (dict(context_lens=[5, 100, 129]), 4),         # needs 3 blocks > 2
    (dict(calc_type=1), 1),                        # SPEC needs qseqlen
    (dict(q_seq_len=[1, 1, 1]), 4),                # qseqlen only with SPEC
    (dict(q_rope=torch.zeros(3, 128, 32, dtype=torch.bfloat16)), 2),
    (dict(heads=0), 4),
])
def test_mla_rejects(over, status):
    with pytest.raises(ala.AlaError) as e:
        _plan_mla(**over)
    assert e.value.status == status, str(e.value)


def test_last_error_is_text():
    with pytest.raises(ala.AlaError) as e:
        _plan_varlen(heads=0)
    assert "headNum" in str(e.value)


def _fake(shape, dtype_code, addr=1 << 20):
    """An ala_tensor over a dummy address: the checks below run before any data is touched."""
    t = ala.AlaTensor()
    t.data = addr
    t.dtype = dtype_code
    t.ndim = len(shape)
    for i, s in enumerate(shape):
        t.dims[i] = s
    return t


def _noalloc_raw(n_tokens, heads, kv_heads, d, seq_len, lse_shape=None):
    L = ala.lib()
    sl = np.asarray(seq_len, dtype=np.int32)
    q = _fake((n_tokens, heads, d), ala.BF16)
    kv = _fake((n_tokens, kv_heads, d), ala.BF16)
    out = _fake((n_tokens, heads, d), ala.BF16)
    lse = None if lse_shape is None else _fake(lse_shape, ala.F32)
    st = L.varlen_attention_noalloc(ctypes.byref(q), ctypes.byref(kv), ctypes.byref(kv),
                                    ala._ref(ala.tensor(sl)), ala._ref(ala.tensor(sl)), None, 9, heads, kv_heads,
                                    ctypes.c_float(0.1), ctypes.byref(out), ala._ref(lse), None)
    return st, L.ala_last_error().decode()


def test_noalloc_refuses_more_work_units_than_its_scratch_holds():
    # one 2M-token sequence over 8 heads without grouping: 8 x 7813 units of two 128-row blocks, more than
    # the fixed scratch holds; refused on the host before the device is touched
    st, msg = _noalloc_raw(2_000_000, 8, 8, 64, [2_000_000])
    assert st == 5 and "work units" in msg


@pytest.mark.parametrize("lse_shape", [(10,), (10, 1), (10, 4, 2), (9, 4)])
def test_noalloc_refuses_an_lse_of_the_wrong_shape(lse_shape):
    st, msg = _noalloc_raw(10, 4, 4, 64, [10], lse_shape)
    assert st == 2 and "lse" in msg


def test_mla_explicit_mask_plans():
    # the MASK_TYPE_SPEC mask [tokens, maxSeqLen] (fp16 or bf16) with maskType SPEC, one or more tokens per batch
    _plan_mla(mask_type=1, mask=torch.zeros(3, 128, dtype=torch.bfloat16))
    _plan_mla(mask_type=1, mask=torch.zeros(3, 200, dtype=torch.float16))
    _plan_mla(q_nope=torch.zeros(6, 128, 512, dtype=torch.bfloat16), q_rope=torch.zeros(6, 128, 64, dtype=torch.bfloat16),
              q_seq_len=[2, 2, 2], mask_type=1, calc_type=1, mask=torch.zeros(6, 130, dtype=torch.bfloat16))


@pytest.mark.parametrize("over,status", [
    (dict(mask=torch.zeros(3, 128, dtype=torch.bfloat16)), 4),                    # maskType UNDEFINED takes no mask
    (dict(mask_type=1, mask=torch.zeros(3, 127, dtype=torch.bfloat16)), 2),       # shorter than contextLens 128
    (dict(mask_type=1, mask=torch.zeros(4, 128, dtype=torch.bfloat16)), 2),       # one row per token
    (dict(mask_type=1, mask=torch.zeros(3, 128, dtype=torch.float32)), 3),        # fp16 / bf16 only
    (dict(mask_type=1, mask=torch.zeros(3, 2, 128, dtype=torch.bfloat16)), 2),    # 2-D
    (dict(q_seq_len=[1, 1, 1], calc_type=3, mask_type=1, mask=torch.zeros(3, 128, dtype=torch.bfloat16)), 4),
])
def test_mla_explicit_mask_rejects(over, status):
    with pytest.raises(ala.AlaError) as e:
        _plan_mla(**over)
    assert e.value.status == status, str(e.value)


@pytest.mark.parametrize("d,dtype", [(16, torch.bfloat16), (80, torch.float16), (96, torch.bfloat16),
                                     (112, torch.bfloat16), (40, torch.float32), (144, torch.float16),
                                     (192, torch.bfloat16), (256, torch.bfloat16), (8, torch.bfloat16),
                                     (72, torch.float16), (200, torch.bfloat16)])
def test_head_sizes_plan(d, dtype):
    op, out = _plan_varlen(q=torch.zeros(10, 4, d, dtype=dtype), k=torch.zeros(14, 2, d, dtype=dtype),
                           v=torch.zeros(14, 2, d, dtype=dtype))
    assert out.shape == (10, 4, d)
