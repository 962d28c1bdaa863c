"""GPU parity of MLA over an int8 latent cache (atb_like_mla with cacheMode 2 and
qkDescale / pvDescale) against the fp64 oracle on the same seeded inputs:
small ragged cases element by element, int8 and float qNope, bf16 and fp16,
the conversion of every int8 code, ring mode's lse, and the full-size decode
workload, every element of the output and the lse.  Output buffers start out
as NaN, so an unwritten row fails."""
import numpy as np
import pytest
import torch

import oracle
import paged_attention_varlen_b200 as ala
import synth
from parity import check_lse, check_out, nan_lse, nan_out

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from paged_attention_varlen_b200 import build
    build.build()


def _run(case, calc_type=None, mask=None):
    d = "cuda"
    ct = case.calc_type if calc_type is None else calc_type
    qn, qr = case.q_nope.to(d), case.q_rope.to(d)
    ck, kr = case.ct_kv.to(d), case.k_rope.to(d)
    bt = torch.from_numpy(case.block_tables).to(d)
    qkd = torch.from_numpy(case.qk_descale).to(d)
    pvd = torch.from_numpy(case.pv_descale).to(d)
    lse = nan_lse(case.n_tokens, case.heads, 1)
    out = nan_out(qr, (case.n_tokens, case.heads, 512))
    qs = case.q_seq_len if (ct in (synth.MLA_CALC_SPEC, ala.MLA_CALC_PREFILL) or
                            (ct == ala.MLA_CALC_RING and (case.q_seq_len > 1).any())) else None
    op, out = ala.plan_mla(qn, qr, ck, kr, bt, case.context_lens, qs, case.heads, case.qk_scale, case.mask_type, ct,
                           lse=lse, out=out, qk_descale=qkd, pv_descale=pvd,
                           mask=None if mask is None else mask.to(d))
    op()
    torch.cuda.synchronize()
    assert op.device_status() == 0, f"device status {op.device_status():#x}"
    return out, lse, op


def _oracle(case, rows=None, mask=None):
    return oracle.mla_dequant(case.q_nope, case.q_rope, case.ct_kv, case.k_rope, case.qk_descale, case.pv_descale,
                              case.block_tables, case.block_size, case.context_lens, case.q_seq_len, case.heads,
                              case.qk_scale, rows=rows, mask=mask)


@pytest.mark.parametrize("qn_int8", [True, False])
@pytest.mark.parametrize("qs", [1, 4])
@pytest.mark.parametrize("block_size", [16, 64, 128])
def test_mla_int8_small_ragged(qs, block_size, qn_int8):
    ctx = np.array([qs, 63, 64, 65, 700, 1100], dtype=np.int32)
    case = synth.make_mla_int8("small", ctx, qs, 128, 11 + qs, block_size=block_size, qnope_int8=qn_int8)
    out, lse, _ = _run(case)
    ref, lref = _oracle(case)
    check_out(out.reshape(-1, 512), ref)
    check_lse(lse.reshape(-1), lref)


def test_mla_int8_fp16_and_64_heads():
    ctx = np.array([300, 5, 900], dtype=np.int32)
    case = synth.make_mla_int8("f16", ctx, 2, 64, 33, block_size=32, dtype=torch.float16)
    out, lse, _ = _run(case)
    ref, lref = _oracle(case)
    check_out(out.reshape(-1, 512), ref)
    check_lse(lse.reshape(-1), lref)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_mla_int8_every_code_converts_exactly(dtype):
    """One cached key per batch: the softmax weight is exactly 1, so with pvDescale = 1 the output row
    is the key's ctKV codes themselves, every code -128..127 of them, each exact in bf16 and fp16.
    The lse is that key's score, which carries every qNope code through the QK product."""
    rng = np.random.Generator(np.random.PCG64(47))
    codes = np.tile(np.arange(-128, 128, dtype=np.int16), 2)
    case = synth.make_mla_int8("codes", np.ones(4, dtype=np.int32), 1, 64, 47, rng=rng, block_size=16, dtype=dtype)
    for b in range(4):
        blk = int(case.block_tables[b, 0])
        case.ct_kv[blk, 0, 0] = torch.from_numpy(np.roll(codes, 37 * b).astype(np.int8))
        case.q_nope[b] = torch.from_numpy(np.roll(codes, 11 * b).astype(np.int8)).expand(64, 512)
    case.pv_descale[:] = 1.0
    out, lse, _ = _run(case)
    for b in range(4):
        want = torch.from_numpy(np.roll(codes, 37 * b).astype(np.float32)).to(dtype)
        assert torch.equal(out[b].cpu(), want.expand(64, 512)), f"batch {b}: codes not reproduced exactly"
    _, lref = _oracle(case)
    check_lse(lse.reshape(-1), lref)


def test_mla_int8_spec_mixed_qseqlen():
    ctx = np.array([50, 700, 1300, 20], dtype=np.int32)
    qs = np.array([1, 3, 4, 2], dtype=np.int32)
    case = synth.make_mla_int8("mixed", ctx, qs, 128, 45, block_size=64)
    out, lse, _ = _run(case)
    ref, lref = _oracle(case)
    check_out(out.reshape(-1, 512), ref)
    check_lse(lse.reshape(-1), lref)


def test_mla_int8_ring_returns_the_lse():
    ctx = np.array([200, 1500, 77], dtype=np.int32)
    case = synth.make_mla_int8("ring", ctx, 1, 128, 49, block_size=128, qnope_int8=False)
    out, lse, _ = _run(case, calc_type=ala.MLA_CALC_RING)
    ref, lref = _oracle(case)
    check_out(out.reshape(-1, 512), ref)
    check_lse(lse.reshape(-1), lref)


def test_mla_int8_repeat_deterministic():
    case = synth.make_mla_int8("rep", np.array([2000, 40], dtype=np.int32), 1, 128, 51, block_size=128)
    out, _, op = _run(case)
    first = out.clone()
    for _ in range(3):
        op()
    torch.cuda.synchronize()
    assert torch.equal(first, out)
    assert op.device_status() == 0


def test_mla_int8_full_size():
    case = synth.mla_decode_int8()
    out, lse, _ = _run(case)
    ref, lref = _oracle(case)
    check_out(out.reshape(-1, 512), ref)
    check_lse(lse.reshape(-1), lref)


@pytest.mark.parametrize("heads,qs,block_size,qn_int8", [(256, 1, 256, True), (128, 2, 32, False), (64, 4, 128, True)])
def test_mla_int8_row_block_shapes(heads, qs, block_size, qn_int8):
    # rows per CTA = tokens per chunk x heads per group: 1 x 64 (four groups of a 256-head token, whole
    # 256-key pages), 2 x 32 (64 heads of two tokens, pages of 32 keys) and 4 x 16
    ctx = np.array([90, 640, 1500, qs + 3], dtype=np.int32)
    case = synth.make_mla_int8(f"rows8_{heads}_{qs}", ctx, qs, heads, 53 + qs, block_size=block_size,
                               qnope_int8=qn_int8)
    out, lse, _ = _run(case)
    ref, lref = _oracle(case)
    check_out(out.reshape(-1, 512), ref)
    check_lse(lse.reshape(-1), lref)


def test_mla_int8_negative_qk_scale():
    case = synth.make_mla_int8("neg8", np.array([100, 700], dtype=np.int32), 2, 128, 55, block_size=64)
    case.qk_scale = -0.03
    out, lse, _ = _run(case)
    ref, lref = _oracle(case)
    check_out(out.reshape(-1, 512), ref)
    check_lse(lse.reshape(-1), lref)


def test_mla_int8_prefill_is_causal_within_each_batch():
    # calcType PREFILL over the int8 cache: all new tokens of a batch attend causally
    ctx = np.array([100, 300, 520], dtype=np.int32)
    qs = np.array([37, 300, 64], dtype=np.int32)
    case = synth.make_mla_int8("prefill8", ctx, qs, 64, 57, block_size=64)
    out, lse, _ = _run(case, calc_type=ala.MLA_CALC_PREFILL)
    ref, lref = _oracle(case)
    check_out(out.reshape(-1, 512), ref)
    check_lse(lse.reshape(-1), lref)


def test_mla_int8_explicit_mask():
    # the MASK_TYPE_SPEC mask tensor over the int8 cache: a non-causal additive mask per token
    ctx = np.array([700, 1100, 65], dtype=np.int32)
    case = synth.make_mla_int8("mask8", ctx, 2, 128, 59, block_size=64)
    case.calc_type, case.mask_type = synth.MLA_CALC_SPEC, synth.MLA_MASK_SPEC
    rng = np.random.Generator(np.random.PCG64(59))
    m = (rng.standard_normal((case.n_tokens, 1100)) * 2.0).astype(np.float32)
    m[rng.random(m.shape) < 0.3] = -np.inf
    m[:, 0] = 0.0
    mask = torch.from_numpy(m).to(torch.float16)
    out, lse, _ = _run(case, mask=mask)
    ref, lref = _oracle(case, mask=mask)
    check_out(out.reshape(-1, 512), ref)
    check_lse(lse.reshape(-1), lref)
