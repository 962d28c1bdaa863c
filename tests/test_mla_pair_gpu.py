"""GPU parity of the CTA-pair MLA decode kernel (M = 128 rows per CTA, two CTAs per 128 heads
splitting the latent dimensions, scores exchanged through distributed shared memory) against the
fp64 oracle.  The kernel serves a request only when ALA_MLA_PAIR=1 is set while it is planned."""
import os

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
    os.environ["ALA_MLA_PAIR"] = "1"
    try:
        op, out = ala.plan_mla(qn, qr, ck, kr, bt, case.context_lens, None, case.heads, case.qk_scale,
                               case.mask_type, case.calc_type, lse=lse)
    finally:
        del os.environ["ALA_MLA_PAIR"]
    op()
    torch.cuda.synchronize()
    assert op.device_status() == 0, f"device status {op.device_status():#x}"
    return out, lse, op


def _oracle(case, rows=None):
    return oracle.mla(case.q_nope, case.q_rope, case.ct_kv, case.k_rope, case.block_tables, case.block_size,
                      case.context_lens, case.q_seq_len, case.heads, case.qk_scale, rows=rows)


@pytest.mark.parametrize("block_size", [16, 64, 128])
def test_mla_pair_small_ragged(block_size):
    ctx = np.array([1, 63, 64, 65, 700, 1100], dtype=np.int32)
    case = synth.make_mla("pair", ctx, 1, 128, 61, block_size=block_size)
    out, lse, _ = _run(case)
    ref, lref = _oracle(case)
    check_out(out.reshape(-1, 512), ref)
    check_lse(lse.reshape(-1), lref)


def test_mla_pair_fp16_256_heads():
    ctx = np.array([300, 5, 900, 2000], dtype=np.int32)
    case = synth.make_mla("pair16", ctx, 1, 256, 63, block_size=64, dtype=torch.float16)
    out, lse, _ = _run(case)
    ref, lref = _oracle(case)
    check_out(out.reshape(-1, 512), ref)
    check_lse(lse.reshape(-1), lref)


def test_mla_pair_full_size_sampled():
    case = synth.mla_decode_bf16(1)
    out, lse, _ = _run(case)
    rng = np.random.Generator(np.random.PCG64(9))
    n = case.n_tokens * case.heads
    rows = np.unique(np.concatenate([rng.choice(n, 160, replace=False), [0, n - 1]])).astype(np.int64)
    ref, lref = _oracle(case, rows)
    idx = torch.from_numpy(rows).cuda()
    check_out(out.reshape(-1, 512)[idx], ref)
    check_lse(lse.reshape(-1)[idx], lref)
    assert torch.isfinite(out.float()).all()
