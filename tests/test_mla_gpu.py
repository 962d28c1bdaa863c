"""GPU parity of the MLA decode / speculative-decode path (atb_like_mla) against
the fp64 oracle on the same seeded inputs: small ragged cases element by
element (key ranges long enough to be split, so the lse merge runs), and the
full-size workload on sampled rows."""
import numpy as np
import pytest
import torch

import oracle
import paged_attention_varlen_b200 as ala
import synth
from parity import check_lse, check_out

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from paged_attention_varlen_b200 import build
    build.build()


def _run(case):
    d = "cuda"
    qn, qr = case.q_nope.to(d), case.q_rope.to(d)
    ck, kr = case.ct_kv.to(d), case.k_rope.to(d)
    bt = torch.from_numpy(case.block_tables).to(d)
    lse = torch.empty((case.n_tokens, case.heads, 1), dtype=torch.float32, device=d)
    qs = case.q_seq_len if case.calc_type == synth.MLA_CALC_SPEC else None
    op, out = ala.plan_mla(qn, qr, ck, kr, bt, case.context_lens, qs, case.heads, case.qk_scale, case.mask_type,
                           case.calc_type, lse=lse)
    op()
    torch.cuda.synchronize()
    assert op.device_status() == 0, f"device status {op.device_status():#x}"
    return out, lse, op


def _oracle(case, rows=None):
    return oracle.mla(case.q_nope, case.q_rope, case.ct_kv, case.k_rope, case.block_tables, case.block_size,
                      case.context_lens, case.q_seq_len, case.heads, case.qk_scale, rows=rows)


@pytest.mark.parametrize("qs", [1, 4])
@pytest.mark.parametrize("block_size", [16, 32, 64, 128])
def test_mla_small_ragged(qs, block_size):
    ctx = np.array([qs, 63, 64, 65, 700, 1100], dtype=np.int32)
    case = synth.make_mla("small", ctx, qs, 128, 5 + qs, block_size=block_size)
    out, lse, _ = _run(case)
    ref, lref = _oracle(case)
    check_out(out.reshape(-1, 512), ref)
    check_lse(lse.reshape(-1), lref)


def test_mla_fp16_and_64_heads():
    ctx = np.array([300, 5, 900], dtype=np.int32)
    case = synth.make_mla("f16", ctx, 2, 64, 31, block_size=64, dtype=torch.float16)
    out, lse, _ = _run(case)
    ref, lref = _oracle(case)
    check_out(out.reshape(-1, 512), ref)
    check_lse(lse.reshape(-1), lref)


def test_mla_mixed_qseqlen():
    # qseqlen 1, 3, 4, 2: one query token per CTA row block, 64 heads of it
    ctx = np.array([50, 700, 1300, 20], dtype=np.int32)
    qs = np.array([1, 3, 4, 2], dtype=np.int32)
    case = synth.make_mla("mixed", ctx, qs, 128, 43, block_size=32)
    out, lse, _ = _run(case)
    ref, lref = _oracle(case)
    check_out(out.reshape(-1, 512), ref)
    check_lse(lse.reshape(-1), lref)


def test_mla_spec_range_past_some_rows():
    # four speculative tokens share each CTA; the second batch's key range is cut just before its
    # last 32-key tile (keys 128..), which only its last token may see, so three of the four tokens
    # have no allowed key in that range and their partial carries lse = -inf
    ctx = np.array([100, 129, 300], dtype=np.int32)
    case = synth.make_mla("spec_cut", ctx, 4, 128, 44, block_size=32)
    out, lse, _ = _run(case)
    ref, lref = _oracle(case)
    check_out(out.reshape(-1, 512), ref)
    check_lse(lse.reshape(-1), lref)


def test_mla_repeat_deterministic():
    ctx = np.array([2000, 40], dtype=np.int32)
    case = synth.make_mla("rep", ctx, 1, 128, 37, block_size=128)
    out, lse, op = _run(case)
    first = out.clone()
    for _ in range(3):
        op()
    torch.cuda.synchronize()
    assert torch.equal(first, out)
    assert op.device_status() == 0


@pytest.mark.parametrize("qs", [1, 4])
def test_mla_full_size_sampled(qs):
    case = synth.mla_decode_bf16(qs)
    out, lse, _ = _run(case)
    rng = np.random.Generator(np.random.PCG64(qs))
    n = case.n_tokens * case.heads
    rows = np.unique(np.concatenate([rng.choice(n, 160, replace=False), [0, n - 1]])).astype(np.int64)
    ref, lref = _oracle(case, rows)
    idx = torch.from_numpy(rows).cuda()
    check_out(out.reshape(-1, 512)[idx], ref)
    check_lse(lse.reshape(-1)[idx], lref)
    assert torch.isfinite(out.float()).all()


def test_mla_negative_qk_scale():
    ctx = np.array([100, 700], dtype=np.int32)
    case = synth.make_mla("neg", ctx, 2, 128, 41, block_size=64)
    case.qk_scale = -0.03
    out, lse, _ = _run(case)
    ref, lref = _oracle(case)
    check_out(out.reshape(-1, 512), ref)
    check_lse(lse.reshape(-1), lref)
