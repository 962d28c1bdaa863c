"""The allocation-free entry point varlen_attention_noalloc, on the GPU.

It exists for callers that cannot call cudaMalloc (runtimes that only hand out
fixed arenas, hosts whose device allocator belongs to another component):
instead of a caller-supplied workspace it uses a fixed 1 MiB array in device
memory owned by the library.

The tests call it through the C ABI twice in a row, on two different
workloads, and compare each result element by element with the fp64 oracle
and with the regular varlen_attention entry point on the same inputs, within
the parity tolerance; the status word read back through
varlen_attention_noalloc_status must be 0 after each call.  They also cover a
call without lse (mask type 0, fp32 inputs on tf32), a head size of 256, and
the refusals: a schedule larger than the fixed scratch, an lse of the wrong
shape, and a stream that is being captured.  This file is collected last so that, if it
fails, a run that stops at the first failure has already run every other
test; it passes alone in a fresh process as well.
"""
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


def _dev(case):
    d = "cuda"
    slopes = None if case.slopes is None else torch.from_numpy(case.slopes).to(d)
    return case.q.to(d), case.k.to(d), case.v.to(d), slopes


def _noalloc(case, with_lse=True):
    q, k, v, slopes = _dev(case)
    out = nan_out(q)
    lse = nan_lse(q.shape[0], case.heads) if with_lse else None
    ala.varlen_attention_noalloc(q, k, v, case.seq_len, case.kv_seq_len, case.mask_type, case.heads, case.kv_heads,
                                 case.qk_scale, slopes, out=out, lse=lse)
    assert ala.varlen_attention_noalloc_status() == 0
    return out, lse


def _workspace_entry(case):
    q, k, v, slopes = _dev(case)
    lse = nan_lse(q.shape[0], case.heads)
    op, out = ala.plan_varlen_attention(q, k, v, case.seq_len, case.kv_seq_len, case.mask_type, case.heads,
                                        case.kv_heads, case.qk_scale, slopes, out=nan_out(q), lse=lse)
    op()
    torch.cuda.synchronize()
    assert op.device_status() == 0
    return out, lse


def _oracle(case):
    return oracle.attention(case.q, case.k, case.v, case.seq_len, case.kv_seq_len, case.mask_type, case.heads,
                            case.kv_heads, case.qk_scale, slopes=case.slopes)


def test_noalloc_matches_the_oracle_and_the_workspace_entry_point_two_calls_in_a_row():
    first = synth.make_prefill("na1", [1, 127, 300, 0, 129], [1, 200, 300, 0, 400], 8, 2, 128, torch.bfloat16,
                               synth.MASK_ALIBI_SQRT, 71)
    second = synth.make_prefill("na2", [64, 513], [64, 513], 4, 4, 64, torch.float16, synth.MASK_CAUSAL, 72)
    for case in (first, second):
        out, lse = _noalloc(case)
        ref, lref = _oracle(case)
        check_out(out.reshape(-1, out.shape[-1]), ref)
        check_lse(lse.reshape(-1), lref)
        wout, wlse = _workspace_entry(case)
        err = (out.double() - wout.double()).abs()
        assert err.max().item() <= 2e-2 and err.mean().item() <= 2e-3
        rel = (lse.double() - wlse.double()).abs() / wlse.double().abs().clamp(min=1.0)
        assert rel.max().item() <= 1e-3


def test_noalloc_without_lse_fp32_no_mask():
    case = synth.make_prefill("na3", [70, 5], [90, 5], 2, 1, 64, torch.float32, synth.MASK_NONE, 73)
    out, _ = _noalloc(case, with_lse=False)
    ref, _ = _oracle(case)
    check_out(out.reshape(-1, 64), ref)


def test_noalloc_head_size_256_causal():
    # the D = 256 kernel: one 128-row block per unit, 64-key K/V tiles
    case = synth.make_prefill("na6", [1, 200, 129], [30, 200, 300], 4, 2, 256, torch.bfloat16, synth.MASK_CAUSAL, 76)
    out, lse = _noalloc(case)
    ref, lref = _oracle(case)
    check_out(out.reshape(-1, 256), ref)
    check_lse(lse.reshape(-1), lref)


def test_noalloc_refuses_a_schedule_larger_than_its_scratch():
    # 5000 sequences exceed the 4096 the fixed scratch holds; refused before any GPU work
    L = np.ones(5000, dtype=np.int32)
    q = torch.zeros((5000, 2, 64), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((5000, 2, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ala.AlaError) as e:
        ala.varlen_attention_noalloc(q, kv, kv, L, L, synth.MASK_CAUSAL, 2, 2, 0.125)
    assert e.value.status == 5 and "4096" in str(e.value)


def test_noalloc_refuses_an_lse_of_the_wrong_shape():
    case = synth.make_prefill("na4", [10], [10], 4, 4, 64, torch.bfloat16, synth.MASK_CAUSAL, 74)
    q, k, v, _ = _dev(case)
    with pytest.raises(ala.AlaError) as e:
        ala.varlen_attention_noalloc(q, k, v, case.seq_len, case.kv_seq_len, case.mask_type, 4, 4, case.qk_scale,
                                     out=nan_out(q), lse=nan_lse(q.shape[0]))
    assert e.value.status == 2


def test_noalloc_refuses_a_stream_being_captured():
    case = synth.make_prefill("na5", [40], [40], 4, 4, 64, torch.bfloat16, synth.MASK_CAUSAL, 75)
    q, k, v, _ = _dev(case)
    out = nan_out(q)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    refused = None
    with torch.cuda.stream(side):
        graph.capture_begin()
        try:
            ala.varlen_attention_noalloc(q, k, v, case.seq_len, case.kv_seq_len, case.mask_type, 4, 4,
                                         case.qk_scale, out=out, stream=side)
        except ala.AlaError as e:
            refused = e
        finally:
            graph.capture_end()
    torch.cuda.synchronize()
    assert refused is not None and refused.status == 5 and "captured" in str(refused)
    # the refusal left nothing behind: an ordinary call afterwards works
    out2, _ = _noalloc(case, with_lse=False)
    ref, _ = _oracle(case)
    check_out(out2.reshape(-1, 64), ref)
