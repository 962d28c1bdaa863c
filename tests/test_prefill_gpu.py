"""GPU parity of the prefill kernel (varlen_attention / atb_like_prefix_encoder)
against the fp64 oracle on the same seeded inputs.

Every test compares every output element and every lse value with the
oracle, the full-size workloads included.  Outputs and lse buffers start out
as NaN, so a row the kernel never writes fails the comparison.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import paged_attention_varlen_b200 as ala
import synth
from parity import LSE_REL, LSE_REL_TF32, check_lse, check_out, nan_lse, nan_out

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from paged_attention_varlen_b200 import build
    build.build()


def _dev(case):
    d = "cuda"
    return (case.q.to(d), case.k.to(d), case.v.to(d),
            None if case.slopes is None else torch.from_numpy(case.slopes).to(d),
            None if case.block_tables is None else torch.from_numpy(case.block_tables).to(d))


def _run(case, want_lse=True):
    q, k, v, slopes, bt = _dev(case)
    lse = nan_lse(q.shape[0], case.heads) if want_lse else None
    out = nan_out(q)
    if case.paged:
        # the lse-returning PrefixEncoder entry point (the plain one shares everything else)
        op, out = ala.plan_prefix_encoder(q, k, v, bt, case.seq_len, case.kv_seq_len, case.mask_type, case.heads,
                                          case.kv_heads, case.qk_scale, slopes, out=out, lse=lse)
    else:
        op, out = ala.plan_varlen_attention(q, k, v, case.seq_len, case.kv_seq_len, case.mask_type, case.heads,
                                            case.kv_heads, case.qk_scale, slopes, out=out, lse=lse)
    op()
    torch.cuda.synchronize()
    assert op.device_status() == 0, f"device status {op.device_status():#x}"
    return out, lse


def _oracle(case, rows=None):
    return oracle.attention(case.q, case.k, case.v, case.seq_len, case.kv_seq_len, case.mask_type, case.heads,
                            case.kv_heads, case.qk_scale, slopes=case.slopes, block_tables=case.block_tables,
                            block_size=case.block_size, rows=rows)


def _full_check(case, lse_rel=LSE_REL):
    out, lse = _run(case)
    ref, lref = _oracle(case)
    check_out(out.reshape(-1, out.shape[-1]), ref)
    if lse is not None:
        check_lse(lse.reshape(-1), lref, rel_bound=lse_rel)
    return out


def test_tiny_causal_fp32_tf32():
    _full_check(synth.tiny_causal_fp32())


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_ragged_varlen_causal_gqa(d, dtype):
    L = [1, 127, 128, 129, 300, 0, 5, 257]
    case = synth.make_prefill("ragged", L, L, 8, 2, d, dtype, synth.MASK_CAUSAL, 7)
    _full_check(case)


@pytest.mark.parametrize("mask_type", [0, 3, 4, 5, 9])
def test_prefix_offset_masks_contiguous(mask_type):
    L = [3, 130, 64, 200]
    pre = [0, 77, 256, 1000]
    case = synth.make_prefill("prefix", L, [a + b for a, b in zip(L, pre)], 8, 4, 128, torch.bfloat16, mask_type, 11)
    _full_check(case)


@pytest.mark.parametrize("block_size", [16, 32, 48, 64, 96, 128, 160, 256])
@pytest.mark.parametrize("mask_type", [3, 4, 5, 9])
def test_paged_prefix_encoder(block_size, mask_type):
    # block sizes that neither divide nor are multiples of the 128-key tile gather in gcd-high boxes
    L = [64, 1, 333, 129]
    pre = [256, 40, 512, 0]
    case = synth.make_prefill("paged", L, [a + b for a, b in zip(L, pre)], 8, 2, 128, torch.float16, mask_type, 13,
                              paged=True, block_size=block_size)
    _full_check(case)


@pytest.mark.parametrize("d,dtype,mask_type,paged", [
    (16, torch.bfloat16, 9, False), (48, torch.float16, 3, False), (80, torch.bfloat16, 9, False),
    (96, torch.bfloat16, 4, False), (112, torch.float16, 0, False), (96, torch.float16, 3, True),
    (80, torch.float16, 5, True), (40, torch.float32, 9, False), (8, torch.float32, 0, False),
    (8, torch.bfloat16, 9, False), (40, torch.float16, 3, False), (72, torch.bfloat16, 9, True),
    (120, torch.float16, 4, False)])
def test_head_sizes_between_the_kernel_sizes(d, dtype, mask_type, paged):
    # head sizes run on the next kernel instance up (64 or 128) with the extra dimensions zero-filled
    L = [1, 127, 128, 129, 300, 5]
    pre = [0, 40, 0, 77, 129, 3]
    case = synth.make_prefill(f"d{d}", L, [a + b for a, b in zip(L, pre)], 8, 2, d, dtype, mask_type, 95 + d,
                              paged=paged, block_size=64)
    _full_check(case, LSE_REL_TF32 if dtype == torch.float32 else LSE_REL)


@pytest.mark.parametrize("d,dtype,mask_type,paged,block_size", [
    (256, torch.bfloat16, 9, False, 128), (256, torch.float16, 0, False, 128), (256, torch.bfloat16, 9, True, 16),
    (256, torch.float16, 9, True, 128), (192, torch.bfloat16, 9, True, 64), (144, torch.float16, 0, False, 128),
    (256, torch.bfloat16, 9, True, 48), (160, torch.float16, 9, True, 80), (200, torch.bfloat16, 0, False, 128),
    (136, torch.float16, 9, True, 16)])
def test_large_head_sizes(d, dtype, mask_type, paged, block_size):
    # head sizes above 128 run on the D = 256 kernel (one 128-row block per CTA, 64-key tiles); GQA group 4
    L = [1, 63, 64, 65, 128, 129, 400, 7]
    pre = [0, 0, 1, 200, 64, 77, 129, 3]
    case = synth.make_prefill(f"d{d}", L, [a + b for a, b in zip(L, pre)], 8, 2, d, dtype, mask_type, 311 + d,
                              paged=paged, block_size=block_size)
    _full_check(case)


def test_paged_equals_contiguous_on_gpu():
    L, pre = [100, 250], [300, 17]
    kv = [a + b for a, b in zip(L, pre)]
    c = synth.make_prefill("c", L, kv, 8, 2, 128, torch.float16, 3, 17)
    p = synth.make_prefill("p", L, kv, 8, 2, 128, torch.float16, 3, 17, paged=True, block_size=64)
    oc, _ = _run(c, want_lse=False)
    op, _ = _run(p, want_lse=False)
    assert torch.equal(oc, op)


def test_padded_run_matches_packed_on_valid_rows():
    case = synth.varlen_causal_bf16(seed=21, batch=4, lo=20, hi=400)
    pad = synth.padded_from(case)
    out, _ = _run(case, want_lse=False)
    outp, _ = _run(pad, want_lse=False)
    Lmax = pad.meta["Lmax"]
    pos = 0
    for b, L in enumerate(case.seq_len.tolist()):
        assert torch.equal(out[pos:pos + L], outp[b * Lmax:b * Lmax + L])
        pos += L


def test_bound_workspace_equals_fresh_upload():
    # Op executions bind their own workspace (the schedule is copied once, later calls clear the status only);
    # an execution into a second, unbound workspace copies the schedule and must give the same bits
    case = synth.make_prefill("bind", [300, 1, 129], [400, 1, 200], 8, 2, 128, torch.bfloat16, 9, 29)
    q, k, v, slopes, _ = _dev(case)
    op, out = ala.plan_varlen_attention(q, k, v, case.seq_len, case.kv_seq_len, 9, 8, 2, case.qk_scale, slopes)
    for _ in range(3):
        op()
    torch.cuda.synchronize()
    assert op.device_status() == 0
    bound = out.clone()
    other = torch.full((max(op.workspace_size, 256),), 0xFF, dtype=torch.uint8, device="cuda")
    out.fill_(float("nan"))
    s = torch.cuda.current_stream()
    L = ala.lib()
    assert L.varlen_attention(ctypes.c_void_p(other.data_ptr()), op.workspace_size, op._handle,
                              ctypes.c_void_p(s.cuda_stream)) == 0
    torch.cuda.synchronize()
    assert torch.equal(bound, out)
    # unbinding makes the Op's own workspace take the copying path again
    assert L.ala_op_bind_workspace(op._handle, None, 0, None) == 0
    out.fill_(float("nan"))
    assert L.varlen_attention(ctypes.c_void_p(op.workspace.data_ptr()), op.workspace_size, op._handle,
                              ctypes.c_void_p(s.cuda_stream)) == 0
    torch.cuda.synchronize()
    assert torch.equal(bound, out)


def test_repeat_is_deterministic_and_status_clean():
    case = synth.make_prefill("rep", [300, 50], [400, 50], 8, 2, 128, torch.bfloat16, 4, 23)
    q, k, v, slopes, _ = _dev(case)
    op, out = ala.plan_varlen_attention(q, k, v, case.seq_len, case.kv_seq_len, 4, 8, 2, case.qk_scale, slopes)
    op()
    first = out.clone()
    for _ in range(3):
        op()
    torch.cuda.synchronize()
    assert torch.equal(first, out)
    assert op.device_status() == 0


# ---------------------------------------------------------------------------- full-size workloads, every element

def test_full_varlen_causal_bf16():
    _full_check(synth.varlen_causal_bf16())


def test_full_varlen_causal_bf16_padded_twin():
    """The same batch padded to its longest sequence: every row (padding rows included) against the oracle."""
    _full_check(synth.padded_from(synth.varlen_causal_bf16()))


def test_full_prefix_paged_alibi_fp16():
    _full_check(synth.prefix_paged_alibi_fp16())


@pytest.mark.parametrize("variant", [synth.MASK_ALIBI_SQRT, synth.MASK_ALIBI_LEFT])
def test_full_long_alibi_bf16(variant):
    _full_check(synth.long_alibi_bf16(variant))


@pytest.mark.parametrize("mask_type", [0, 3, 9])
def test_negative_qk_scale(mask_type):
    """A negative qkScale reverses the score order; the max must be taken after scaling."""
    L = [70, 200]
    case = synth.make_prefill("neg", L, [a + 30 for a in L], 8, 4, 128, torch.bfloat16, mask_type, 29,
                              qk_scale=-0.06)
    _full_check(case)
