"""GPU parity of the MLA decode / speculative-decode path (atb_like_mla) against
the fp64 oracle on the same seeded inputs: small ragged cases element by
element (key ranges long enough to be split, so the lse merge runs), and the
full-size decode and speculative workloads, every element of the output and
the lse.  Output buffers start out as NaN, so an unwritten row fails."""
import ctypes

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


def _run(case, mask=None):
    d = "cuda"
    qn, qr = case.q_nope.to(d), case.q_rope.to(d)
    ck, kr = case.ct_kv.to(d), case.k_rope.to(d)
    bt = torch.from_numpy(case.block_tables).to(d)
    lse = nan_lse(case.n_tokens, case.heads, 1)
    out = nan_out(qr, (case.n_tokens, case.heads, 512))
    qs = case.q_seq_len if case.calc_type in (synth.MLA_CALC_SPEC, ala.MLA_CALC_PREFILL) else None
    op, out = ala.plan_mla(qn, qr, ck, kr, bt, case.context_lens, qs, case.heads, case.qk_scale, case.mask_type,
                           case.calc_type, lse=lse, out=out, mask=None if mask is None else mask.to(d))
    op()
    torch.cuda.synchronize()
    assert op.device_status() == 0, f"device status {op.device_status():#x}"
    return out, lse, op


def _oracle(case, rows=None, mask=None):
    return oracle.mla(case.q_nope, case.q_rope, case.ct_kv, case.k_rope, case.block_tables, case.block_size,
                      case.context_lens, case.q_seq_len, case.heads, case.qk_scale, rows=rows, mask=mask)


def test_mla_bound_workspace_equals_fresh_upload():
    # the Op binds its workspace (schedule copied once); an execution into another workspace copies it again,
    # with split key ranges so the partials and the combine are exercised, and must give the same bits
    ctx = np.array([1, 700, 3000, 65], dtype=np.int32)
    case = synth.make_mla("bind", ctx, 1, 128, 31, block_size=64)
    out, lse, op = _run(case)
    op()
    torch.cuda.synchronize()
    ref_out, ref_lse = out.clone(), lse.clone()
    other = torch.full((max(op.workspace_size, 256),), 0xFF, dtype=torch.uint8, device="cuda")
    out.fill_(float("nan"))
    lse.fill_(float("nan"))
    s = torch.cuda.current_stream()
    assert ala.lib().atb_like_mla(ctypes.c_void_p(other.data_ptr()), op.workspace_size, op._handle,
                                  ctypes.c_void_p(s.cuda_stream)) == 0
    torch.cuda.synchronize()
    assert torch.equal(ref_out, out) and torch.equal(ref_lse, lse)


@pytest.mark.parametrize("qs", [1, 4])
@pytest.mark.parametrize("block_size", [16, 32, 48, 64, 80, 128, 192])
def test_mla_small_ragged(qs, block_size):
    ctx = np.array([qs, 63, 64, 65, 700, 1100], dtype=np.int32)
    case = synth.make_mla("small", ctx, qs, 128, 5 + qs, block_size=block_size)
    out, lse, _ = _run(case)
    ref, lref = _oracle(case)
    check_out(out.reshape(-1, 512), ref)
    check_lse(lse.reshape(-1), lref)


@pytest.mark.parametrize("heads,dtype", [(64, torch.bfloat16), (128, torch.float16), (384, torch.bfloat16)])
def test_mla_decode_row_kernels(heads, dtype):
    # one token per batch: 64-row blocks of one token's heads (384 heads: six head groups per key range)
    ctx = np.array([1, 64, 65, 700, 2500, 129], dtype=np.int32)
    case = synth.make_mla(f"rows_{heads}", ctx, 1, heads, 89, block_size=64, dtype=dtype)
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
def test_mla_full_size(qs):
    case = synth.mla_decode_bf16(qs)
    out, lse, _ = _run(case)
    ref, lref = _oracle(case)
    check_out(out.reshape(-1, 512), ref)
    check_lse(lse.reshape(-1), lref)


def test_mla_negative_qk_scale():
    ctx = np.array([100, 700], dtype=np.int32)
    case = synth.make_mla("neg", ctx, 2, 128, 41, block_size=64)
    case.qk_scale = -0.03
    out, lse, _ = _run(case)
    ref, lref = _oracle(case)
    check_out(out.reshape(-1, 512), ref)
    check_lse(lse.reshape(-1), lref)


def _ring_ranges(case, bs):
    """Each batch's keys cut at a page boundary into [0, cut) and [cut, ctx): two block tables over the same cache."""
    ctx = case.context_lens
    cut = np.maximum(ctx // (2 * bs), 1) * bs
    assert (cut < ctx).all()
    bt = case.block_tables
    bt_a = np.full_like(bt, -1)
    bt_b = np.full_like(bt, -1)
    for b in range(len(ctx)):
        pa = cut[b] // bs
        nb = (ctx[b] - cut[b] + bs - 1) // bs
        bt_a[b, :pa] = bt[b, :pa]
        bt_b[b, :nb] = bt[b, pa:pa + nb]
    return (cut.astype(np.int32), bt_a), ((ctx - cut).astype(np.int32), bt_b)


def test_mla_ring_ranges_merged_equal_the_whole_context():
    # calcType RING over two disjoint key ranges, merged by lse (ala_lse_merge), against the oracle over all keys
    bs = 64
    ctx = np.array([700, 1100, 300, 129], dtype=np.int32)
    case = synth.make_mla("ring", ctx, 1, 128, 45, block_size=bs)
    d = "cuda"
    qn, qr = case.q_nope.to(d), case.q_rope.to(d)
    ck, kr = case.ct_kv.to(d), case.k_rope.to(d)
    parts = []
    for cl, bt in _ring_ranges(case, bs):
        lse = nan_lse(case.n_tokens, case.heads, 1)
        op, out = ala.plan_mla(qn, qr, ck, kr, torch.from_numpy(bt).to(d), cl, None, case.heads, case.qk_scale,
                               synth.MLA_MASK_UNDEFINED, ala.MLA_CALC_RING, lse=lse,
                               out=nan_out(qr, (case.n_tokens, case.heads, 512)))
        op()
        parts.append((out, lse, op))
    (oa, la, opa), (ob, lb, opb) = parts
    out, lse = ala.lse_merge(oa, la, ob, lb, out=nan_out(oa), lse=nan_lse(*la.shape))
    torch.cuda.synchronize()
    ref, lref = _oracle(case)
    check_out(out.reshape(-1, 512), ref)
    check_lse(lse.reshape(-1), lref)
    # in place over the first range's buffers gives the same result
    ala.lse_merge(oa, la, ob, lb, out=oa, lse=la)
    torch.cuda.synchronize()
    assert torch.equal(oa, out) and torch.equal(la, lse)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_lse_merge_matches_the_oracle(dtype):
    rng = np.random.Generator(np.random.PCG64(46))
    n, heads, dv = 96, 3, 512
    oa = torch.from_numpy(rng.standard_normal((n, heads, dv)).astype(np.float32)).to(dtype)
    ob = torch.from_numpy(rng.standard_normal((n, heads, dv)).astype(np.float32)).to(dtype)
    la = (rng.standard_normal((n, heads, 1)) * 4).astype(np.float32)
    lb = (rng.standard_normal((n, heads, 1)) * 4).astype(np.float32)
    la[5, 0, 0] = -np.inf                           # one side saw no allowed key
    lb[7, 1, 0] = -np.inf
    la[9, 2, 0] = lb[9, 2, 0] = -np.inf             # neither side: lse -inf, output 0
    ref, lref = oracle.lse_merge(np.stack([oa.double().numpy().reshape(-1, dv), ob.double().numpy().reshape(-1, dv)]),
                                 np.stack([la.reshape(-1), lb.reshape(-1)]).astype(np.float64))
    out, lse = ala.lse_merge(oa.cuda(), torch.from_numpy(la).cuda(), ob.cuda(), torch.from_numpy(lb).cuda(),
                             out=nan_out(oa.cuda()), lse=nan_lse(*la.shape))
    torch.cuda.synchronize()
    got = out.reshape(-1, dv).double().cpu().numpy()
    gl = lse.reshape(-1).double().cpu().numpy()
    both = 9 * heads + 2
    assert gl[both] == -np.inf and lref[both] == -np.inf
    assert (got[both] == 0).all() and (ref[both] == 0).all()
    keep = np.arange(n * heads) != both
    tol = 2e-2 if dtype == torch.bfloat16 else 1e-5
    assert np.abs(got[keep] - ref[keep]).max() <= tol
    assert (np.abs(gl[keep] - lref[keep]) / np.maximum(1, np.abs(lref[keep]))).max() <= 1e-5


@pytest.mark.parametrize("heads,qs,block_size", [(256, 1, 128), (128, 2, 64), (64, 4, 128)])
def test_mla_row_block_shapes(heads, qs, block_size):
    # rows per CTA = tokens per chunk x heads per group: 1 x 64 (four groups of a 256-head token),
    # 2 x 32 and 4 x 16 (64 heads: four groups of 16)
    ctx = np.array([90, 640, 1500, qs + 3], dtype=np.int32)
    case = synth.make_mla(f"rows_{heads}_{qs}", ctx, qs, heads, 47 + qs, block_size=block_size)
    out, lse, _ = _run(case)
    ref, lref = _oracle(case)
    check_out(out.reshape(-1, 512), ref)
    check_lse(lse.reshape(-1), lref)


def test_mla_prefill_is_causal_within_each_batch():
    # calcType PREFILL: all new tokens of a batch (one batch without a prefix) attend causally
    ctx = np.array([100, 300, 520], dtype=np.int32)
    qs = np.array([37, 300, 64], dtype=np.int32)
    case = synth.make_mla("prefill", ctx, qs, 64, 49, block_size=64)
    case.calc_type = ala.MLA_CALC_PREFILL
    case.mask_type = synth.MLA_MASK_UNDEFINED
    out, lse, _ = _run(case)
    ref, lref = _oracle(case)
    check_out(out.reshape(-1, 512), ref)
    check_lse(lse.reshape(-1), lref)


# ---------------------------------------------------------------------------- explicit MASK_TYPE_SPEC mask tensor

def _random_mask(case, cols, seed, dtype, p_masked=0.3):
    """[tokens, cols] additive mask: N(0, 2) values, a share of -inf, key 0 always open."""
    rng = np.random.Generator(np.random.PCG64(seed))
    m = (rng.standard_normal((case.n_tokens, cols)) * 2.0).astype(np.float32)
    m[rng.random(m.shape) < p_masked] = -np.inf
    m[:, 0] = 0.0
    return torch.from_numpy(m).to(dtype)


def _spec_mask(case, cols, dtype):
    rows = []
    for c, q in zip(case.context_lens.tolist(), case.q_seq_len.tolist()):
        for t in range(q):
            r = torch.full((cols,), torch.finfo(dtype).min, dtype=torch.float32)
            r[:c - q + t + 1] = 0.0
            rows.append(r)
    return torch.stack(rows).to(dtype)


def _with_mask(case):
    case.calc_type = synth.MLA_CALC_SPEC
    case.mask_type = synth.MLA_MASK_SPEC
    return case


@pytest.mark.parametrize("qs,block_size,cols", [(1, 128, 1104), (4, 16, 1100), ([1, 3, 4, 2], 64, 1107)])
def test_mla_explicit_random_mask(qs, block_size, cols):
    # a non-causal additive mask per token; key ranges long enough to be cut across CTAs (partials merged)
    ctx = np.array([700, 1100, 65, 300], dtype=np.int32)
    case = _with_mask(synth.make_mla("emask", ctx, qs, 128, 83, block_size=block_size))
    mask = _random_mask(case, cols, 83, torch.bfloat16)
    out, lse, _ = _run(case, mask)
    ref, lref = _oracle(case, mask=mask)
    check_out(out.reshape(-1, 512), ref)
    check_lse(lse.reshape(-1), lref)


def test_mla_explicit_mask_of_the_rule_matches_the_rule_fp16():
    ctx = np.array([90, 640, 1500, 7], dtype=np.int32)
    case = _with_mask(synth.make_mla("rule_mask", ctx, 4, 128, 85, block_size=32, dtype=torch.float16))
    mask = _spec_mask(case, 1504, torch.float16)
    out, lse, _ = _run(case, mask)
    ref, lref = _oracle(case)  # the generated rule
    check_out(out.reshape(-1, 512), ref)
    check_lse(lse.reshape(-1), lref)


def test_mla_explicit_mask_rows_without_an_allowed_key():
    # token 1 is masked everywhere (output 0, lse -inf), token 2 only beyond key 900 (the row's whole key
    # range is cut across CTAs, so empty partials meet in the merge)
    ctx = np.array([1200], dtype=np.int32)
    case = _with_mask(synth.make_mla("empty_rows", ctx, 4, 128, 87, block_size=64))
    mask = _random_mask(case, 1200, 87, torch.bfloat16, p_masked=0.1)
    mask[1, :] = -float("inf")
    mask[2, :900] = -float("inf")
    out, lse, _ = _run(case, mask)
    ref, lref = _oracle(case, mask=mask)
    assert (ref[128:256] == 0).all() and (lref[128:256] == -np.inf).all()
    check_out(out.reshape(-1, 512), ref)
    check_lse(lse.reshape(-1), lref)
