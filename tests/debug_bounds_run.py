"""Runs small paged calls on the range-checking library (ALA_LIBRARY=debug, libala_debug.so) and prints
one JSON line per case: the device status word and the largest error against the fp64 oracle.  Started as a
child process by tests/test_debug_bounds_gpu.py, so the library choice stays out of the main test process."""
import json
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import paged_attention_varlen_b200 as ala  # noqa: E402
import synth  # noqa: E402


def prefill(case, bt):
    d = "cuda"
    slopes = None if case.slopes is None else torch.from_numpy(case.slopes).to(d)
    op, out = ala.plan_prefix_encoder(case.q.to(d), case.k.to(d), case.v.to(d), torch.from_numpy(bt).to(d),
                                      case.seq_len, case.kv_seq_len, case.mask_type, case.heads, case.kv_heads,
                                      case.qk_scale, slopes)
    op()
    torch.cuda.synchronize()
    return op.device_status(), out


def mla(case, bt):
    d = "cuda"
    op, out = ala.plan_mla(case.q_nope.to(d), case.q_rope.to(d), case.ct_kv.to(d), case.k_rope.to(d),
                           torch.from_numpy(bt).to(d), case.context_lens, None, case.heads, case.qk_scale)
    op()
    torch.cuda.synchronize()
    return op.device_status(), out


def main():
    assert ala.LIB_PATH.endswith("libala_debug.so"), ala.LIB_PATH
    res = {}
    # paged prefix encoder: unused block-table entries are -1 and never read -> status 0, parity
    case = synth.make_prefill("dbg", [64, 1, 333], [320, 41, 845], 8, 2, 128, torch.float16, synth.MASK_CAUSAL, 91,
                              paged=True, block_size=64)
    st, out = prefill(case, case.block_tables)
    ref, _ = oracle.attention(case.q, case.k, case.v, case.seq_len, case.kv_seq_len, case.mask_type, case.heads,
                              case.kv_heads, case.qk_scale, block_tables=case.block_tables, block_size=64)
    res["prefill_ok"] = {"status": st, "max_err": float(np.abs(out.float().cpu().double().numpy().reshape(ref.shape)
                                                               - ref).max())}
    # one used entry past the cache: the kernel records the bad index and reads zeros instead
    bad = case.block_tables.copy()
    bad[2, 3] = case.k.shape[0] + 7
    st, _ = prefill(case, bad)
    res["prefill_bad_entry"] = {"status": st}
    # MLA decode (128 heads: the 128-row kernel) with 16-key pages, then one negative entry in use
    m = synth.make_mla("dbg_mla", np.array([100, 700, 33], dtype=np.int32), 1, 128, 93, block_size=16)
    st, out = mla(m, m.block_tables)
    ref, _ = oracle.mla(m.q_nope, m.q_rope, m.ct_kv, m.k_rope, m.block_tables, 16, m.context_lens, m.q_seq_len,
                        128, m.qk_scale)
    res["mla_ok"] = {"status": st, "max_err": float(np.abs(out.float().cpu().double().numpy().reshape(ref.shape)
                                                           - ref).max())}
    bad = m.block_tables.copy()
    bad[1, 5] = -3
    st, _ = mla(m, bad)
    res["mla_bad_entry"] = {"status": st}
    print(json.dumps(res))


if __name__ == "__main__":
    main()
