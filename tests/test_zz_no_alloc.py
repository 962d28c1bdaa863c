"""The allocation-free entry point varlen_attention_noalloc, on the GPU.

It exists for callers that cannot call cudaMalloc (code running while another
component builds a CUDA graph, runtimes that only hand out fixed arenas, hosts
whose device allocator belongs to someone else): instead of a caller-supplied
workspace it uses a fixed 1 MiB array in device memory owned by the library.

The test calls it through the C ABI twice in a row, on two different workloads,
and compares each result with the regular varlen_attention entry point on the
same inputs within the parity tolerance.  It also checks that a call too large
for the fixed scratch is refused with a clear message.  This file is collected
last so that, if it fails, a run that stops at the first failure has already run
every other test; it passes alone in a fresh process as well.
"""
import numpy as np
import pytest
import torch

import paged_attention_varlen_b200 as ala
import synth
from parity import LSE_REL, MAX_ABS, MEAN_ABS

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from paged_attention_varlen_b200 import build
    build.build()


def _both(case):
    d = "cuda"
    q, k, v = case.q.to(d), case.k.to(d), case.v.to(d)
    slopes = None if case.slopes is None else torch.from_numpy(case.slopes).to(d)
    lse_ref = torch.empty((q.shape[0], case.heads), dtype=torch.float32, device=d)
    op, ref = ala.plan_varlen_attention(q, k, v, case.seq_len, case.kv_seq_len, case.mask_type, case.heads,
                                        case.kv_heads, case.qk_scale, slopes, lse=lse_ref)
    op()
    out = torch.full_like(q, float("nan"))
    lse = torch.full((q.shape[0], case.heads), float("nan"), dtype=torch.float32, device=d)
    ala.varlen_attention_noalloc(q, k, v, case.seq_len, case.kv_seq_len, case.mask_type, case.heads, case.kv_heads,
                                 case.qk_scale, slopes, out=out, lse=lse)
    torch.cuda.synchronize()
    return out, lse, ref, lse_ref


def _close(out, lse, ref, lse_ref):
    err = (out.double() - ref.double()).abs()
    assert torch.isfinite(out).all()
    assert err.max().item() <= MAX_ABS and err.mean().item() <= MEAN_ABS
    rel = (lse.double() - lse_ref.double()).abs() / lse_ref.double().abs().clamp(min=1.0)
    assert rel.max().item() <= LSE_REL


def test_noalloc_matches_workspace_entry_point_two_calls_in_a_row():
    first = synth.make_prefill("na1", [1, 127, 300, 0, 129], [1, 200, 300, 0, 400], 8, 2, 128, torch.bfloat16,
                               synth.MASK_ALIBI_SQRT, 71)
    second = synth.make_prefill("na2", [64, 513], [64, 513], 4, 4, 64, torch.float16, synth.MASK_CAUSAL, 72)
    for case in (first, second):
        _close(*_both(case))


def test_noalloc_refuses_a_schedule_larger_than_its_scratch():
    # 5000 sequences exceed the 4096 the fixed scratch holds; refused before any GPU work
    L = np.ones(5000, dtype=np.int32)
    q = torch.zeros((5000, 2, 64), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((5000, 2, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ala.AlaError) as e:
        ala.varlen_attention_noalloc(q, kv, kv, L, L, synth.MASK_CAUSAL, 2, 2, 0.125)
    assert e.value.status == 5 and "4096" in str(e.value)
