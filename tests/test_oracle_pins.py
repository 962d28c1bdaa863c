"""Pins of the fp64 oracle to facts the pages and the mathematics fix (CPU only).

Each test checks the oracle against something other than itself: a worked
example derived by hand (tests/golden), a closed form, a library routine the
case reduces to (torch's scaled_dot_product_attention in float64), or an
invariant the pages state (packing, paging, masked pairs contributing nothing).
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, dtype=torch.float32, seed=0, sigma=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * sigma).to(dtype)


def _seq_case(L, Lkv, H, Hkv, d, mask_type, dtype=torch.float32, seed=0, slopes=None, dv=None):
    q = _rand((L, H, d), dtype, seed)
    k = _rand((Lkv, Hkv, d), dtype, seed + 1)
    v = _rand((Lkv, Hkv, dv or d), dtype, seed + 2)
    return q, k, v


# --------------------------------------------------------------------------
# hand-derived worked examples
# --------------------------------------------------------------------------

def _read_kv(path):
    vals = {}
    for line in open(path):
        if line.startswith("#") or not line.strip():
            continue
        key, *rest = line.split()
        vals[key] = [float(x) for x in rest]
    return vals


def test_two_key_worked_example():
    g = _read_kv(os.path.join(GOLDEN, "two_key_softmax.txt"))
    q = torch.tensor(g["q"], dtype=torch.float32).view(1, 1, 1)
    k = torch.tensor(g["k"], dtype=torch.float32).view(2, 1, 1)
    v = torch.tensor(g["v"], dtype=torch.float32).view(2, 1, 1)
    out, lse = oracle.attention(q, k, v, [1], [2], oracle.MASK_NONE, 1, 1, g["qk_scale"][0])
    assert abs(out[0, 0] - g["out"][0]) < 1e-6
    assert abs(lse[0] - g["lse"][0]) < 1e-6


def test_mask_rule_matches_hand_derived_masks():
    rows = {}
    for line in open(os.path.join(GOLDEN, "alibi_masks_L2_Lkv4.txt")):
        if line.startswith("#") or not line.strip():
            continue
        parts = line.split()
        rows[(int(parts[0]), int(parts[1]))] = [float(x) for x in parts[2:]]
    for mt in (0, 3, 4, 5, 9):
        m = oracle.build_mask(mt, np.array([0.5], np.float32), 1, 2, 4)
        for i in range(2):
            np.testing.assert_allclose(m[0, i], rows[(mt, i)], rtol=0, atol=1e-15)


# --------------------------------------------------------------------------
# closed forms
# --------------------------------------------------------------------------

@pytest.mark.parametrize("mask_type", [0, 3, 4, 5, 9])
def test_single_key_returns_v0(mask_type):
    q, k, v = _seq_case(1, 1, 2, 1, 8, mask_type, seed=3)
    slopes = np.array([0.25, 0.5], np.float32)
    out, lse = oracle.attention(q, k, v, [1], [1], mask_type, 2, 1, 0.3, slopes=slopes)
    for h in range(2):
        np.testing.assert_array_equal(out[h], v[0, 0].double().numpy())
        dot = float((q[0, h].double() * k[0, 0].double()).sum())
        assert abs(lse[h] - 0.3 * dot) < 1e-12  # bias is 0 at distance 0 for 3/4; j=0 for 5


@pytest.mark.parametrize("mask_type", [0, 9])
def test_zero_query_gives_mean_of_allowed_values(mask_type):
    L, Lkv = 5, 9  # prefix of 4 tokens
    q = torch.zeros((L, 2, 4))
    _, k, v = _seq_case(L, Lkv, 2, 2, 4, mask_type, seed=5)
    out, lse = oracle.attention(q, k, v, [L], [Lkv], mask_type, 2, 2, 0.7)
    out = out.reshape(L, 2, 4)
    lse = lse.reshape(L, 2)
    for i in range(L):
        n_allowed = Lkv if mask_type == 0 else i + (Lkv - L) + 1
        for h in range(2):
            np.testing.assert_allclose(out[i, h], v[:n_allowed, h].double().mean(0).numpy(), rtol=0, atol=1e-12)
            assert abs(lse[i, h] - math.log(n_allowed)) < 1e-12


@pytest.mark.parametrize("mask_type", [0, 3, 4, 5, 9])
def test_constant_values_give_that_constant(mask_type):
    L, Lkv = 6, 10
    q, k, _ = _seq_case(L, Lkv, 4, 2, 8, mask_type, seed=7)
    c = torch.linspace(-2.0, 3.0, 8)
    v = c.expand(Lkv, 2, 8).contiguous()
    out, _ = oracle.attention(q, k, v, [L], [Lkv], mask_type, 4, 2, 0.35,
                              slopes=synth.alibi_slopes(4))
    np.testing.assert_allclose(out, np.broadcast_to(c.double().numpy(), out.shape), rtol=0, atol=1e-12)


def test_right_aligned_alibi_geometric_closed_form():
    """q = 0, d = 1, v_j = j: weights r^(iabs-j) with r = exp(-slope) -> a geometric-series mean."""
    L, Lkv, slope = 4, 11, 0.37
    q = torch.zeros((L, 1, 1))
    k = _rand((Lkv, 1, 1), seed=11)
    v = torch.arange(Lkv, dtype=torch.float32).view(Lkv, 1, 1)
    out, lse = oracle.attention(q, k, v, [L], [Lkv], oracle.MASK_ALIBI, 1, 1, 1.0,
                                slopes=np.array([slope], np.float32))
    s = float(np.float32(slope))
    r = math.exp(-s)
    for i in range(L):
        n = i + (Lkv - L)  # iabs; keys 0..n allowed
        s0 = (1 - r ** (n + 1)) / (1 - r)                                     # sum_k r^k
        s1 = r * (1 - (n + 1) * r ** n + n * r ** (n + 1)) / (1 - r) ** 2     # sum_k k r^k
        assert abs(out[i, 0] - (n * s0 - s1) / s0) < 1e-12                  # sum_j j r^(n-j) / s0
        assert abs(lse[i] - math.log(s0)) < 1e-12


# --------------------------------------------------------------------------
# library routine the cases reduce to: torch SDPA (math path, float64)
# --------------------------------------------------------------------------

def _sdpa(q, k, v, scale, attn_mask=None, is_causal=False):
    qq = q.double().permute(1, 0, 2).unsqueeze(0)
    kk = k.double().permute(1, 0, 2).unsqueeze(0)
    vv = v.double().permute(1, 0, 2).unsqueeze(0)
    o = F.scaled_dot_product_attention(qq, kk, vv, attn_mask=attn_mask, is_causal=is_causal, scale=scale,
                                       enable_gqa=True)
    return o.squeeze(0).permute(1, 0, 2).reshape(-1, v.shape[-1]).numpy()


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
def test_no_mask_and_causal_match_sdpa_with_gqa(dtype):
    L, H, Hkv, d = 37, 8, 2, 16
    q, k, v = _seq_case(L, L, H, Hkv, d, 0, dtype=dtype, seed=13)
    for mt, causal in ((oracle.MASK_NONE, False), (oracle.MASK_CAUSAL, True)):
        out, _ = oracle.attention(q, k, v, [L], [L], mt, H, Hkv, 0.25)
        ref = _sdpa(q, k, v, 0.25, is_causal=causal)
        np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("mask_type", [3, 4, 5, 9])
def test_prefix_offset_masks_match_sdpa_with_additive_bias(mask_type):
    """Bias built from the page rules as a float mask; SDPA adds it after scaling."""
    L, Lkv, H, Hkv, d = 7, 19, 4, 4, 8
    q, k, v = _seq_case(L, Lkv, H, Hkv, d, mask_type, seed=17)
    slopes = synth.alibi_slopes(H)
    out, _ = oracle.attention(q, k, v, [L], [Lkv], mask_type, H, Hkv, 0.5, slopes=slopes)
    bias = torch.full((H, L, Lkv), float("-inf"), dtype=torch.float64)
    for h in range(H):
        sl = float(slopes[h])
        for i in range(L):
            iabs = i + Lkv - L
            for j in range(iabs + 1):
                bias[h, i, j] = {3: sl * (j - iabs), 4: -sl * math.sqrt(iabs - j), 5: sl * j, 9: 0.0}[mask_type]
    ref = _sdpa(q, k, v, 0.5, attn_mask=bias.unsqueeze(0))
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# invariants the pages state
# --------------------------------------------------------------------------

@pytest.mark.parametrize("mask_type", [0, 3, 4, 5, 9])
def test_rule_equals_explicit_full_mask(mask_type):
    L, Lkv, H, Hkv, d = 9, 14, 4, 2, 8
    q, k, v = _seq_case(L, Lkv, H, Hkv, d, mask_type, seed=19)
    slopes = synth.alibi_slopes(H)
    out, lse = oracle.attention(q, k, v, [L], [Lkv], mask_type, H, Hkv, 0.4, slopes=slopes)
    m = oracle.build_mask(mask_type, slopes, H, L, Lkv)
    out2, lse2 = oracle.attention_explicit(q, k, v, m, H, Hkv, 0.4)
    np.testing.assert_allclose(out, out2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse2, rtol=0, atol=1e-12)


def test_compressed_causal_triangle_expands_to_rule():
    tri = np.where(np.arange(128)[None, :] > np.arange(128)[:, None], -np.inf, 0.0)
    for L, Lkv in ((5, 5), (40, 300), (200, 200), (130, 400)):
        m = oracle.expand_causal_compressed(tri, L, Lkv)
        ref = oracle.build_mask(oracle.MASK_CAUSAL, None, 1, L, Lkv)[0]
        np.testing.assert_array_equal(m, ref)


def test_zero_slopes_equal_causal():
    L, Lkv, H = 8, 13, 3
    q, k, v = _seq_case(L, Lkv, H, H, 8, 3, seed=23)
    ref, lref = oracle.attention(q, k, v, [L], [Lkv], oracle.MASK_CAUSAL, H, H, 0.5)
    for mt in (3, 4, 5):
        out, lse = oracle.attention(q, k, v, [L], [Lkv], mt, H, H, 0.5, slopes=np.zeros(H, np.float32))
        np.testing.assert_array_equal(out, ref)
        np.testing.assert_array_equal(lse, lref)


def test_left_aligned_equals_right_aligned_up_to_row_shift():
    L, Lkv, H = 6, 15, 4
    q, k, v = _seq_case(L, Lkv, H, H, 8, 3, seed=29)
    slopes = synth.alibi_slopes(H)
    o3, l3 = oracle.attention(q, k, v, [L], [Lkv], 3, H, H, 0.5, slopes=slopes)
    o5, l5 = oracle.attention(q, k, v, [L], [Lkv], 5, H, H, 0.5, slopes=slopes)
    np.testing.assert_allclose(o3, o5, rtol=0, atol=1e-12)
    for i in range(L):
        for h in range(H):
            iabs = i + Lkv - L
            assert abs(l5[i * H + h] - l3[i * H + h] - float(slopes[h]) * iabs) < 1e-12


def test_sqrt_equals_linear_on_unit_distances():
    q, k, v = _seq_case(2, 2, 2, 2, 8, 4, seed=31)
    slopes = synth.alibi_slopes(2)
    o3, l3 = oracle.attention(q, k, v, [2], [2], 3, 2, 2, 0.5, slopes=slopes)
    o4, l4 = oracle.attention(q, k, v, [2], [2], 4, 2, 2, 0.5, slopes=slopes)
    np.testing.assert_allclose(o3, o4, rtol=0, atol=1e-15)
    np.testing.assert_allclose(l3, l4, rtol=0, atol=1e-15)


@pytest.mark.parametrize("mask_type", [0, 4, 9])
def test_packed_equals_each_sequence_alone(mask_type):
    rng = np.random.Generator(np.random.PCG64(37))
    L = rng.integers(1, 40, size=4).astype(np.int32)
    pre = rng.integers(0, 30, size=4).astype(np.int32)
    case = synth.make_prefill("t", L, L + pre, 4, 2, 8, torch.bfloat16, mask_type, 37)
    out, lse = oracle.attention(case.q, case.k, case.v, case.seq_len, case.kv_seq_len, mask_type, 4, 2, 0.3,
                                slopes=case.slopes)
    qo = ko = 0
    for b in range(4):
        Lb, Lkvb = int(L[b]), int(L[b] + pre[b])
        o1, l1 = oracle.attention(case.q[qo:qo + Lb], case.k[ko:ko + Lkvb], case.v[ko:ko + Lkvb], [Lb], [Lkvb],
                                  mask_type, 4, 2, 0.3, slopes=case.slopes)
        np.testing.assert_array_equal(out[qo * 4:(qo + Lb) * 4], o1)
        np.testing.assert_array_equal(lse[qo * 4:(qo + Lb) * 4], l1)
        qo += Lb
        ko += Lkvb


def test_packed_equals_padded_layout_on_valid_rows():
    case = synth.varlen_causal_bf16(seed=41, batch=3, lo=5, hi=30)
    case.heads, case.kv_heads = 32, 8
    pad = synth.padded_from(case)
    out, _ = oracle.attention(case.q, case.k, case.v, case.seq_len, case.kv_seq_len, 9, 32, 8, case.qk_scale)
    outp, _ = oracle.attention(pad.q, pad.k, pad.v, pad.seq_len, pad.kv_seq_len, 9, 32, 8, pad.qk_scale)
    Lmax = pad.meta["Lmax"]
    pos = 0
    for b, L in enumerate(case.seq_len.tolist()):
        np.testing.assert_array_equal(out[pos * 32:(pos + L) * 32], outp[b * Lmax * 32:(b * Lmax + L) * 32])
        pos += L
    assert pad.meta["padding_positions"] == 3 * Lmax - int(case.seq_len.sum())


@pytest.mark.parametrize("block_size", [16, 64, 128])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_paged_equals_contiguous(block_size, dtype):
    rng = np.random.Generator(np.random.PCG64(43 + block_size))
    L = rng.integers(1, 50, size=3).astype(np.int32)
    Lkv = L + rng.integers(0, 300, size=3).astype(np.int32)
    contig = synth.make_prefill("c", L, Lkv, 4, 2, 16, dtype, 3, 43)
    paged = synth.make_prefill("p", L, Lkv, 4, 2, 16, dtype, 3, 43, paged=True, block_size=block_size)
    assert (paged.block_tables >= -1).all()
    o1, l1 = oracle.attention(contig.q, contig.k, contig.v, L, Lkv, 3, 4, 2, 0.25, slopes=contig.slopes)
    o2, l2 = oracle.attention(paged.q, paged.k, paged.v, L, Lkv, 3, 4, 2, 0.25, slopes=paged.slopes,
                              block_tables=paged.block_tables, block_size=block_size)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_masked_keys_and_values_do_not_contribute():
    L, Lkv, H = 6, 10, 2
    q, k, v = _seq_case(L, Lkv, H, H, 8, 9, seed=47)
    out, lse = oracle.attention(q, k, v, [L], [Lkv], 9, H, H, 0.5)
    # row 0 sits at iabs 4: keys 5.. are masked for it; row L-1 sees all
    k2, v2 = k.clone(), v.clone()
    k2[5:] = 1e4
    v2[5:] = -1e4
    out2, lse2 = oracle.attention(q, k2, v2, [L], [Lkv], 9, H, H, 0.5)
    np.testing.assert_array_equal(out[:H], out2[:H])
    np.testing.assert_array_equal(lse[:H], lse2[:H])
    assert not np.allclose(out[-H:], out2[-H:])


def test_lse_merge_of_disjoint_key_ranges_equals_whole():
    """Split the keys in two ranges, attend to each alone, merge by lse: equals attending to all."""
    L, Lkv, H, d = 3, 50, 2, 8
    q, k, v = _seq_case(L, Lkv, H, H, d, 0, seed=53)
    whole, lw = oracle.attention(q, k, v, [L], [Lkv], 0, H, H, 0.3)
    a = 21
    o1, l1 = oracle.attention(q, k[:a], v[:a], [L], [a], 0, H, H, 0.3)
    o2, l2 = oracle.attention(q, k[a:], v[a:], [L], [Lkv - a], 0, H, H, 0.3)
    mo, ml = oracle.lse_merge(np.stack([o1, o2]), np.stack([l1, l2]))
    np.testing.assert_allclose(mo, whole, rtol=0, atol=1e-12)
    np.testing.assert_allclose(ml, lw, rtol=0, atol=1e-12)
    # lse normalises the weights: sum_j exp(s_j - lse) = 1 with s_j from an independent dot product
    s = 0.3 * torch.einsum("lhd,jhd->lhj", q.double(), k.double())
    np.testing.assert_allclose(torch.exp(s - torch.tensor(lw).view(L, H, 1)).sum(-1).numpy(), 1.0, atol=1e-12)


# --------------------------------------------------------------------------
# MLA entry point
# --------------------------------------------------------------------------

@pytest.mark.parametrize("qs", [1, 4])
def test_mla_equals_generic_with_concatenated_key(qs):
    rng = np.random.Generator(np.random.PCG64(59))
    ctx = rng.integers(qs, 300, size=3).astype(np.int32)
    case = synth.make_mla("m", ctx, qs, 4, 59, rng=rng, block_size=64, d_nope=32, d_rope=8)
    out, lse = oracle.mla(case.q_nope, case.q_rope, case.ct_kv, case.k_rope, case.block_tables, 64,
                          case.context_lens, case.q_seq_len, 4, case.qk_scale)
    q = torch.cat([case.q_nope, case.q_rope], dim=-1)
    kcat = torch.cat([case.ct_kv, case.k_rope], dim=-1)
    o2, l2 = oracle.attention(q, kcat, case.ct_kv, case.q_seq_len, case.context_lens, oracle.MASK_CAUSAL, 4, 1,
                              case.qk_scale, block_tables=case.block_tables, block_size=64)
    np.testing.assert_allclose(out, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, l2, rtol=0, atol=1e-12)


def test_mla_spec_last_token_equals_decode_over_full_context():
    rng = np.random.Generator(np.random.PCG64(61))
    ctx = rng.integers(8, 200, size=2).astype(np.int32)
    case = synth.make_mla("m", ctx, 4, 2, 61, rng=rng, block_size=16, d_nope=16, d_rope=8)
    out, lse = oracle.mla(case.q_nope, case.q_rope, case.ct_kv, case.k_rope, case.block_tables, 16,
                          case.context_lens, case.q_seq_len, 2, case.qk_scale)
    for b in range(2):
        t = b * 4 + 3
        o1, l1 = oracle.mla(case.q_nope[t:t + 1], case.q_rope[t:t + 1], case.ct_kv, case.k_rope,
                            case.block_tables[b:b + 1], 16, case.context_lens[b:b + 1], [1], 2, case.qk_scale)
        np.testing.assert_array_equal(out[t * 2:t * 2 + 2], o1)
        np.testing.assert_array_equal(lse[t * 2:t * 2 + 2], l1)


def test_row_subset_equals_full_run():
    case = synth.make_prefill("r", [20, 33], [50, 33], 4, 2, 16, torch.bfloat16, 4, 67)
    full, lf = oracle.attention(case.q, case.k, case.v, case.seq_len, case.kv_seq_len, 4, 4, 2, 0.25,
                                slopes=case.slopes)
    rows = np.array([0, 5, 79, 80, 150, 211], dtype=np.int64)
    sub, ls = oracle.attention(case.q, case.k, case.v, case.seq_len, case.kv_seq_len, 4, 4, 2, 0.25,
                               slopes=case.slopes, rows=rows)
    np.testing.assert_array_equal(sub, full[rows])
    np.testing.assert_array_equal(ls, lf[rows])


# --------------------------------------------------------------------------
# MLA over an int8 latent cache (MLA page, qkDescale / pvDescale rows)
# --------------------------------------------------------------------------

def _int8_two_key_case():
    """Two heads, two cached keys, d_nope 16, d_rope 4, one page (physical block 1 of 2).

    Stored numbers: qNope head 0 = -3, head 1 = 5 (every element); ctKV key 0 = 2, key 1 = -1;
    qRope head 0 = 0.5, head 1 = -0.25; kRope key 0 = 1, key 1 = 2.  qkDescale = (1/64, 1/32),
    pvDescale = (0.5, 3), qkScale = 0.5.  By hand:
      head 0: nope dots 16*(-3*2) = -96 and 16*(-3*-1) = 48; rope dots 4*0.5*1 = 2 and 4*0.5*2 = 4
              s = 0.5*(-96/64 + 2) = 0.25 and 0.5*(48/64 + 4) = 2.375
      head 1: nope dots 16*(5*2) = 160 and 16*(5*-1) = -80; rope dots -1 and -2
              s = 0.5*(160/32 - 1) = 2 and 0.5*(-80/32 - 2) = -2.25
    The output is pvDescale * (p0 * 2 + p1 * (-1)) in every column, p1 = 1/(1 + exp(s0 - s1)),
    and lse = s0 + log(1 + exp(s1 - s0))."""
    qn = torch.tensor([-3, 5], dtype=torch.int8).view(1, 2, 1).expand(1, 2, 16).contiguous()
    qr = torch.tensor([0.5, -0.25], dtype=torch.bfloat16).view(1, 2, 1).expand(1, 2, 4).contiguous()
    ck = torch.full((2, 16, 1, 16), 99, dtype=torch.int8)  # block 0 is not referenced
    ck[1, 0] = 2
    ck[1, 1] = -1
    kr = torch.full((2, 16, 1, 4), 7.0, dtype=torch.bfloat16)
    kr[1, 0] = 1.0
    kr[1, 1] = 2.0
    return qn, qr, ck, kr, np.array([[1]], dtype=np.int32)


def test_mla_int8_two_key_worked_example():
    qn, qr, ck, kr, bt = _int8_two_key_case()
    out, lse = oracle.mla_dequant(qn, qr, ck, kr, [1 / 64, 1 / 32], [0.5, 3.0], bt, 16, [2], [1], 2, 0.5)
    for h, (s0, s1, pv) in enumerate([(0.25, 2.375, 0.5), (2.0, -2.25, 3.0)]):
        p1 = 1.0 / (1.0 + math.exp(s0 - s1))
        expect = pv * ((1.0 - p1) * 2.0 + p1 * -1.0)
        np.testing.assert_allclose(out[h], np.full(16, expect), rtol=0, atol=1e-13)
        assert abs(lse[h] - (s0 + math.log1p(math.exp(s1 - s0)))) < 1e-13


@pytest.mark.parametrize("qn_int8", [True, False])
@pytest.mark.parametrize("qs", [1, 3])
def test_mla_int8_equals_sdpa_with_prescaled_operands(qn_int8, qs):
    """The dequantised scores are qkScale * [qkDescale*qNope ; qRope] . [ctKV ; kRope]: torch's float64
    scaled_dot_product_attention on those concatenated operands, with the speculative causal mask,
    times pvDescale, must give the same rows."""
    rng = np.random.Generator(np.random.PCG64(71))
    heads, d_nope, d_rope, bs = 3, 24, 8, 16
    ctx = np.array([5, 40, 33], dtype=np.int32)
    case = synth.make_mla_int8("q8", ctx, qs, heads, 71, rng=rng, block_size=bs, d_nope=d_nope, d_rope=d_rope,
                               qnope_int8=qn_int8)
    out, lse = oracle.mla_dequant(case.q_nope, case.q_rope, case.ct_kv, case.k_rope, case.qk_descale,
                                  case.pv_descale, case.block_tables, bs, case.context_lens, case.q_seq_len, heads,
                                  case.qk_scale)
    qkd = torch.from_numpy(case.qk_descale.astype(np.float64))
    pvd = torch.from_numpy(case.pv_descale.astype(np.float64))
    t0 = 0
    for b, L in enumerate(ctx.tolist()):
        keys = []
        for j in range(L):
            blk = int(case.block_tables[b, j // bs])
            keys.append((case.ct_kv[blk, j % bs, 0].double(), case.k_rope[blk, j % bs, 0].double()))
        kn = torch.stack([k[0] for k in keys])                      # [L, d_nope]
        kcat = torch.cat([kn, torch.stack([k[1] for k in keys])], dim=-1)
        for t in range(qs):
            allow = torch.arange(L) <= L - qs + t
            for h in range(heads):
                q = torch.cat([case.q_nope[t0 + t, h].double() * qkd[h], case.q_rope[t0 + t, h].double()])
                o = F.scaled_dot_product_attention(q.view(1, 1, 1, -1), kcat.view(1, 1, L, -1), kn.view(1, 1, L, -1),
                                                   attn_mask=allow.view(1, 1, 1, L), scale=case.qk_scale)
                row = (t0 + t) * heads + h
                np.testing.assert_allclose(out[row], (o.view(-1) * pvd[h]).numpy(), rtol=1e-12, atol=1e-12)
                s = case.qk_scale * (kcat[allow] @ q)
                assert abs(lse[row] - torch.logsumexp(s, 0).item()) < 1e-12
        t0 += qs


def test_mla_int8_output_is_linear_in_pv_descale_and_lse_ignores_it():
    rng = np.random.Generator(np.random.PCG64(73))
    case = synth.make_mla_int8("q8", np.array([70], dtype=np.int32), 1, 2, 73, rng=rng, block_size=32, d_nope=16,
                               d_rope=8, qnope_int8=True)
    args = (case.block_tables, 32, case.context_lens, case.q_seq_len, 2, case.qk_scale)
    o1, l1 = oracle.mla_dequant(case.q_nope, case.q_rope, case.ct_kv, case.k_rope, case.qk_descale,
                                np.ones(2, np.float32), *args)
    o2, l2 = oracle.mla_dequant(case.q_nope, case.q_rope, case.ct_kv, case.k_rope, case.qk_descale,
                                np.array([0.25, 4.0], np.float32), *args)
    np.testing.assert_array_equal(l1, l2)
    np.testing.assert_array_equal(o2[0], o1[0] * 0.25)
    np.testing.assert_array_equal(o2[1], o1[1] * 4.0)


# --------------------------------------------------------------------------
# MLA with the explicit MASK_TYPE_SPEC mask tensor (MLA page, rows mask / maskType)
# --------------------------------------------------------------------------

def _spec_rule_mask(ctx, qs, cols, dtype, masked_value):
    """[tokens, cols] mask holding 0 where the speculative rule allows key j (j <= ctx - qs + t) and
    `masked_value` elsewhere."""
    rows = []
    for c, q in zip(ctx.tolist(), qs.tolist()):
        for t in range(q):
            r = torch.full((cols,), masked_value, dtype=torch.float64)
            r[:c - q + t + 1] = 0.0
            rows.append(r)
    return torch.stack(rows).to(dtype)


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("masked_value", [-math.inf, "lowest"])
def test_mla_explicit_mask_of_the_spec_rule_equals_the_rule(dtype, masked_value):
    rng = np.random.Generator(np.random.PCG64(77))
    ctx = np.array([9, 70, 33], dtype=np.int32)
    qs = np.array([3, 1, 4], dtype=np.int32)
    case = synth.make_mla("mm", ctx, qs, 3, 77, rng=rng, block_size=16, d_nope=24, d_rope=8, dtype=dtype)
    mv = torch.finfo(dtype).min if masked_value == "lowest" else masked_value
    mask = _spec_rule_mask(ctx, qs, 80, dtype, mv)
    args = (case.q_nope, case.q_rope, case.ct_kv, case.k_rope, case.block_tables, 16, ctx, qs, 3, case.qk_scale)
    o_rule, l_rule = oracle.mla(*args)
    o_mask, l_mask = oracle.mla(*args, mask=mask)
    np.testing.assert_allclose(o_mask, o_rule, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l_mask, l_rule, rtol=0, atol=1e-12)


def test_mla_explicit_mask_equals_sdpa_with_the_additive_mask():
    """A random, non-causal additive mask (finite values and some -inf) per packed token: torch's float64
    scaled_dot_product_attention over the concatenated key with the token's mask row as attn_mask."""
    rng = np.random.Generator(np.random.PCG64(79))
    heads, d_nope, d_rope, bs, cols = 2, 16, 8, 16, 48
    ctx = np.array([7, 40, 21], dtype=np.int32)
    qs = np.array([2, 3, 1], dtype=np.int32)
    case = synth.make_mla("ms", ctx, qs, heads, 79, rng=rng, block_size=bs, d_nope=d_nope, d_rope=d_rope,
                          dtype=torch.bfloat16)
    m = rng.standard_normal((int(qs.sum()), cols)).astype(np.float32) * 2.0
    m[rng.random(m.shape) < 0.3] = -np.inf
    m[:, 0] = 0.0  # every row keeps at least key 0
    mask = torch.from_numpy(m).to(torch.bfloat16)
    out, lse = oracle.mla(case.q_nope, case.q_rope, case.ct_kv, case.k_rope, case.block_tables, bs, ctx, qs, heads,
                          case.qk_scale, mask=mask)
    t0 = 0
    for b, L in enumerate(ctx.tolist()):
        keys = [(case.ct_kv[int(case.block_tables[b, j // bs]), j % bs, 0].double(),
                 case.k_rope[int(case.block_tables[b, j // bs]), j % bs, 0].double()) for j in range(L)]
        kn = torch.stack([k[0] for k in keys])
        kcat = torch.cat([kn, torch.stack([k[1] for k in keys])], dim=-1)
        for t in range(int(qs[b])):
            bias = mask[t0 + t, :L].double()
            for h in range(heads):
                q = torch.cat([case.q_nope[t0 + t, h].double(), case.q_rope[t0 + t, h].double()])
                o = F.scaled_dot_product_attention(q.view(1, 1, 1, -1), kcat.view(1, 1, L, -1), kn.view(1, 1, L, -1),
                                                   attn_mask=bias.view(1, 1, 1, L), scale=case.qk_scale)
                row = (t0 + t) * heads + h
                np.testing.assert_allclose(out[row], o.view(-1).numpy(), rtol=1e-12, atol=1e-12)
                s = case.qk_scale * (kcat @ q) + bias
                assert abs(lse[row] - torch.logsumexp(s, 0).item()) < 1e-12
        t0 += int(qs[b])


def test_mla_explicit_mask_fully_masked_row_gives_zero_and_minus_inf():
    rng = np.random.Generator(np.random.PCG64(81))
    ctx = np.array([20], dtype=np.int32)
    case = synth.make_mla("mz", ctx, 2, 2, 81, rng=rng, block_size=16, d_nope=16, d_rope=8, dtype=torch.float16)
    mask = torch.zeros((2, 32), dtype=torch.float16)
    mask[1, :] = -math.inf  # the second token sees no key at all
    out, lse = oracle.mla(case.q_nope, case.q_rope, case.ct_kv, case.k_rope, case.block_tables, 16, ctx, [2], 2,
                          case.qk_scale, mask=mask)
    assert (out[2:] == 0).all() and (lse[2:] == -np.inf).all()
    assert np.isfinite(out[:2]).all() and np.isfinite(lse[:2]).all()
