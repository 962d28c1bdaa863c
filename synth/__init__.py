"""Seeded synthetic workloads shared by the tests, the bench and the smoke check.

This module only draws inputs: sequence lengths, Q/K/V values, block tables
and per-head ALiBi slopes.  It holds none of the attention arithmetic, so both
the CUDA path and the CPU oracle can consume its output without sharing code.

Recipe (fixed for every workload):
  * numpy PCG64 generator seeded with ``seed``;
  * draw order: lengths -> Q -> K -> V -> block permutation;
  * values drawn as float32 normals with the workload's standard deviation and
    rounded to the workload dtype by ``torch.Tensor.to``;
  * paged caches hold Sum ceil(kvSeqLen/blockSize) used blocks plus 10 % spare
    blocks; the block table is a random permutation, entries past a sequence's
    last block are -1, and every unused cache slot (spare blocks and the tail
    of each sequence's last block) is filled with a large finite poison value
    (+-6e4 for fp16, +-1e30 for bf16/fp32) that must never contribute.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

MASK_NONE, MASK_ALIBI, MASK_ALIBI_SQRT, MASK_ALIBI_LEFT, MASK_CAUSAL = 0, 3, 4, 5, 9
MLA_CALC_UNDEFINED, MLA_CALC_SPEC = 0, 1
MLA_MASK_UNDEFINED, MLA_MASK_SPEC = 0, 1

_POISON = {torch.float16: 6.0e4, torch.bfloat16: 1.0e30, torch.float32: 1.0e30, torch.int8: 127}


def alibi_slopes(heads: int) -> np.ndarray:
    """Geometric per-head ALiBi coefficients 2^(-8(h+1)/heads), float32."""
    return np.array([2.0 ** (-8.0 * (h + 1) / heads) for h in range(heads)], dtype=np.float32)


@dataclass
class PrefillCase:
    name: str
    dtype: torch.dtype
    q: torch.Tensor            # [nTokens, heads, d]
    k: torch.Tensor            # contiguous [nKvTokens, kvHeads, d] or paged [numBlocks, blockSize, kvHeads, d]
    v: torch.Tensor
    seq_len: np.ndarray        # [batch] int32 (host)
    kv_seq_len: np.ndarray     # [batch] int32 (host)
    heads: int
    kv_heads: int
    head_size: int
    qk_scale: float
    mask_type: int
    slopes: np.ndarray | None = None
    block_tables: np.ndarray | None = None   # [batch, maxBlockNum] int32, -1 = unused
    block_size: int = 0
    meta: dict = field(default_factory=dict)

    @property
    def paged(self) -> bool:
        return self.block_tables is not None

    @property
    def n_tokens(self) -> int:
        return int(self.seq_len.sum())

    def valid_pairs(self) -> int:
        """Allowed (i, j) pairs per head (integer bookkeeping of the mask rule's extent)."""
        tot = 0
        for L, Lkv in zip(self.seq_len.tolist(), self.kv_seq_len.tolist()):
            if self.mask_type == MASK_NONE:
                tot += L * Lkv
            else:
                off = Lkv - L
                tot += L * off + L * (L + 1) // 2
        return tot


def _normal(rng, shape, sigma, dtype):
    a = rng.standard_normal(size=shape, dtype=np.float32)
    if sigma != 1.0:
        a *= np.float32(sigma)
    return torch.from_numpy(a).to(dtype)


def _page(rng, kv_seq_len, block_size, k_logical, v_logical, dtype, spare_frac=0.1):
    """Scatter logical per-sequence K/V rows into a randomly permuted paged cache."""
    kv_heads, d = k_logical.shape[1], k_logical.shape[2]
    dv = v_logical.shape[2]
    nblk = [(int(x) + block_size - 1) // block_size for x in kv_seq_len]
    used = sum(nblk)
    num_blocks = used + max(1, int(math.ceil(used * spare_frac)))
    perm = rng.permutation(num_blocks).astype(np.int32)
    max_blocks = max(1, max(nblk) if nblk else 1)
    bt = np.full((len(kv_seq_len), max_blocks), -1, dtype=np.int32)
    poison = _POISON[dtype]
    # poison pattern: alternating sign so both large positive and negative scores appear
    sign = torch.where(torch.arange(d) % 2 == 0, 1.0, -1.0)
    k_cache = (sign * poison).to(dtype).repeat(num_blocks, block_size, kv_heads, 1)
    signv = torch.where(torch.arange(dv) % 2 == 0, 1.0, -1.0)
    v_cache = (signv * poison).to(dtype).repeat(num_blocks, block_size, kv_heads, 1)
    pos, nxt = 0, 0
    for b, L in enumerate(kv_seq_len.tolist()):
        for p in range(nblk[b]):
            blk = int(perm[nxt])
            nxt += 1
            bt[b, p] = blk
            lo = p * block_size
            n = min(block_size, L - lo)
            k_cache[blk, :n] = k_logical[pos + lo: pos + lo + n]
            v_cache[blk, :n] = v_logical[pos + lo: pos + lo + n]
        pos += L
    return k_cache, v_cache, bt


def make_prefill(name, seq_len, kv_seq_len, heads, kv_heads, head_size, dtype, mask_type, seed,
                 paged=False, block_size=128, sigma=1.0, qk_scale=None, rng=None) -> PrefillCase:
    """Build a packed varlen prefill case from already drawn lengths (rng continues the stream)."""
    rng = rng if rng is not None else np.random.Generator(np.random.PCG64(seed))
    seq_len = np.asarray(seq_len, dtype=np.int32)
    kv_seq_len = np.asarray(kv_seq_len, dtype=np.int32)
    n_tok, n_kv = int(seq_len.sum()), int(kv_seq_len.sum())
    q = _normal(rng, (n_tok, heads, head_size), sigma, dtype)
    k = _normal(rng, (n_kv, kv_heads, head_size), sigma, dtype)
    v = _normal(rng, (n_kv, kv_heads, head_size), sigma, dtype)
    bt = None
    if paged:
        k, v, bt = _page(rng, kv_seq_len, block_size, k, v, dtype)
    slopes = alibi_slopes(heads) if mask_type in (MASK_ALIBI, MASK_ALIBI_SQRT, MASK_ALIBI_LEFT) else None
    return PrefillCase(name=name, dtype=dtype, q=q, k=k, v=v, seq_len=seq_len, kv_seq_len=kv_seq_len,
                       heads=heads, kv_heads=kv_heads, head_size=head_size,
                       qk_scale=qk_scale if qk_scale is not None else 1.0 / math.sqrt(head_size),
                       mask_type=mask_type, slopes=slopes, block_tables=bt,
                       block_size=block_size if paged else 0)


# ---------------------------------------------------------------------------
# The five workloads, full size, with their seeds (1000 + index).
# ---------------------------------------------------------------------------

def tiny_causal_fp32(seed=1000) -> PrefillCase:
    """1 sequence, L=128, 2 heads, d=64, fp32, causal, contiguous."""
    return make_prefill("tiny_causal_fp32_L128_h2_d64", [128], [128], 2, 2, 64, torch.float32, MASK_CAUSAL,
                        seed, qk_scale=1.0 / 8.0)


def varlen_causal_bf16(seed=1001, batch=8, lo=64, hi=2048, heads=32, kv_heads=8, head_size=128) -> PrefillCase:
    """batch 8, seqLen ~ U{64..2048}, H=32, Hkv=8, d=128, bf16, causal, contiguous (heads and head size
    adjustable: the d=256 variant keeps the lengths and takes H=16, Hkv=4)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    L = rng.integers(lo, hi + 1, size=batch).astype(np.int32)
    return make_prefill(f"varlen_causal_bf16_b{batch}_h{heads}kv{kv_heads}_d{head_size}", L, L, heads, kv_heads,
                        head_size, torch.bfloat16, MASK_CAUSAL, seed, rng=rng)


def padded_from(case: PrefillCase) -> PrefillCase:
    """The same batch laid out padded: every sequence extended to Lmax with zero rows.

    Valid rows of sequence b keep their values; padding rows follow them.  Under the
    causal rule valid rows never see padding keys (they come later), so the valid
    outputs are unchanged while the work grows to B*Lmax rows.
    """
    assert not case.paged
    B = len(case.seq_len)
    Lmax = int(case.seq_len.max())
    H, Hkv, d = case.heads, case.kv_heads, case.head_size
    q = torch.zeros((B * Lmax, H, d), dtype=case.dtype)
    k = torch.zeros((B * Lmax, Hkv, d), dtype=case.dtype)
    v = torch.zeros((B * Lmax, Hkv, d), dtype=case.dtype)
    pos = 0
    for b, L in enumerate(case.seq_len.tolist()):
        q[b * Lmax: b * Lmax + L] = case.q[pos: pos + L]
        k[b * Lmax: b * Lmax + L] = case.k[pos: pos + L]
        v[b * Lmax: b * Lmax + L] = case.v[pos: pos + L]
        pos += L
    full = np.full(B, Lmax, dtype=np.int32)
    return PrefillCase(name=case.name + "_padded", dtype=case.dtype, q=q, k=k, v=v, seq_len=full,
                       kv_seq_len=full.copy(), heads=H, kv_heads=Hkv, head_size=d, qk_scale=case.qk_scale,
                       mask_type=case.mask_type, slopes=case.slopes,
                       meta={"padding_positions": int(B * Lmax - case.seq_len.sum()), "Lmax": Lmax})


def prefix_paged_alibi_fp16(seed=1002, batch=16, block_size=128, prefix_max=4096, new_lo=64, new_hi=1024
                            ) -> PrefillCase:
    """batch 16, prefix ~ U{256,384,..,4096}, new ~ U{64..1024}, paged bs=128, H=32/Hkv=8, fp16, ALiBi right."""
    rng = np.random.Generator(np.random.PCG64(seed))
    prefix = 128 * rng.integers(2, prefix_max // 128 + 1, size=batch)
    new = rng.integers(new_lo, new_hi + 1, size=batch)
    return make_prefill(f"prefix_paged_alibi_fp16_b{batch}_bs{block_size}", new, prefix + new, 32, 8, 128,
                        torch.float16, MASK_ALIBI, seed, paged=True, block_size=block_size, rng=rng)


def long_alibi_bf16(variant: int, seed=1003, batch=2, L=8192, heads=40) -> PrefillCase:
    """batch 2, L=8192, H=Hkv=40, d=128, bf16, sqrt right-aligned (4) or left-aligned (5) ALiBi."""
    assert variant in (MASK_ALIBI_SQRT, MASK_ALIBI_LEFT)
    rng = np.random.Generator(np.random.PCG64(seed))
    Ls = np.full(batch, L, dtype=np.int32)
    return make_prefill(f"long_alibi{variant}_bf16_b{batch}_L{L}_h{heads}", Ls, Ls, heads, heads, 128,
                        torch.bfloat16, variant, seed, rng=rng)


@dataclass
class MlaCase:
    name: str
    dtype: torch.dtype
    q_nope: torch.Tensor        # [tokens, heads, 512]
    q_rope: torch.Tensor        # [tokens, heads, 64]
    ct_kv: torch.Tensor         # [numBlocks, blockSize, 1, 512]
    k_rope: torch.Tensor        # [numBlocks, blockSize, 1, 64]
    block_tables: np.ndarray    # [batch, maxBlocks] int32
    context_lens: np.ndarray    # [batch] int32
    q_seq_len: np.ndarray       # [batch] int32
    heads: int
    qk_scale: float
    calc_type: int
    mask_type: int
    block_size: int
    qk_descale: np.ndarray | None = None  # [heads] float32, int8 latent cache only
    pv_descale: np.ndarray | None = None  # [heads] float32, int8 latent cache only

    @property
    def n_tokens(self) -> int:
        return int(self.q_seq_len.sum())

    def valid_pairs(self) -> int:
        tot = 0
        for c, qs in zip(self.context_lens.tolist(), self.q_seq_len.tolist()):
            tot += sum(c - qs + t + 1 for t in range(qs))
        return tot


def make_mla(name, context_lens, qs, heads, seed, rng=None, block_size=128, d_nope=512, d_rope=64, sigma=0.5,
             dtype=torch.bfloat16) -> MlaCase:
    rng = rng if rng is not None else np.random.Generator(np.random.PCG64(seed))
    context_lens = np.asarray(context_lens, dtype=np.int32)
    batch = len(context_lens)
    q_seq_len = np.broadcast_to(np.asarray(qs, dtype=np.int32), (batch,)).copy()  # one count or one per batch
    tokens = int(q_seq_len.sum())
    spec = bool((q_seq_len > 1).any())
    q_nope = _normal(rng, (tokens, heads, d_nope), sigma, dtype)
    q_rope = _normal(rng, (tokens, heads, d_rope), sigma, dtype)
    n_kv = int(context_lens.sum())
    ckv = _normal(rng, (n_kv, 1, d_nope), sigma, dtype)
    kr = _normal(rng, (n_kv, 1, d_rope), sigma, dtype)
    ct_kv, k_rope, bt = _page(rng, context_lens, block_size, ckv, kr, dtype)
    return MlaCase(name=name, dtype=dtype, q_nope=q_nope, q_rope=q_rope, ct_kv=ct_kv, k_rope=k_rope,
                   block_tables=bt, context_lens=context_lens, q_seq_len=q_seq_len, heads=heads,
                   qk_scale=1.0 / math.sqrt(d_nope + d_rope),
                   calc_type=MLA_CALC_SPEC if spec else MLA_CALC_UNDEFINED,
                   mask_type=MLA_MASK_SPEC if spec else MLA_MASK_UNDEFINED, block_size=block_size)


def mla_decode_bf16(qs: int, seed=1004, batch=64, lo=1024, hi=16384, heads=128) -> MlaCase:
    """batch 64, contextLens ~ U{1024..16384}, 128 heads, 512+64, paged bs=128, bf16 N(0,0.5), qs 1 or 4."""
    rng = np.random.Generator(np.random.PCG64(seed))
    ctx = rng.integers(lo, hi + 1, size=batch).astype(np.int32)
    return make_mla(f"mla_qs{qs}_bf16_b{batch}_h{heads}", ctx, qs, heads, seed, rng=rng)


def _quantize(x: np.ndarray, scale) -> torch.Tensor:
    """Symmetric int8 codes of float samples: round(x / scale) clipped to [-127, 127]."""
    return torch.from_numpy(np.clip(np.rint(x / scale), -127, 127).astype(np.int8))


def make_mla_int8(name, context_lens, qs, heads, seed, rng=None, block_size=128, d_nope=512, d_rope=64, sigma=0.5,
                  dtype=torch.bfloat16, qnope_int8=True) -> MlaCase:
    """An MLA case over an int8 latent cache: ctKV holds int8 codes of N(0, sigma) samples at one scale
    (4 sigma / 127); qNope is int8 codes at a per-head scale (or plain `dtype` samples); qRope and kRope
    stay `dtype`.  qk_descale[h] = qNope scale x cache scale (cache scale alone, with a per-head factor in
    [0.75, 1.25), for a float qNope) and pv_descale[h] = cache scale x a per-head factor in [0.75, 1.25)."""
    rng = rng if rng is not None else np.random.Generator(np.random.PCG64(seed))
    context_lens = np.asarray(context_lens, dtype=np.int32)
    batch = len(context_lens)
    q_seq_len = np.broadcast_to(np.asarray(qs, dtype=np.int32), (batch,)).copy()
    tokens = int(q_seq_len.sum())
    spec = bool((q_seq_len > 1).any())
    kv_scale = 4.0 * sigma / 127.0
    head_f = (0.75 + 0.5 * rng.random(heads)).astype(np.float32)
    qn = rng.standard_normal(size=(tokens, heads, d_nope), dtype=np.float32) * np.float32(sigma)
    if qnope_int8:
        q_scale = (kv_scale * head_f).astype(np.float32)
        q_nope = _quantize(qn, q_scale[None, :, None])
        qk_descale = (q_scale * np.float32(kv_scale)).astype(np.float32)
    else:
        q_nope = torch.from_numpy(qn).to(dtype)
        qk_descale = (np.float32(kv_scale) * head_f).astype(np.float32)
    pv_descale = (np.float32(kv_scale) * (0.75 + 0.5 * rng.random(heads))).astype(np.float32)
    q_rope = _normal(rng, (tokens, heads, d_rope), sigma, dtype)
    n_kv = int(context_lens.sum())
    ckv = _quantize(rng.standard_normal(size=(n_kv, 1, d_nope), dtype=np.float32) * np.float32(sigma), kv_scale)
    kr = _normal(rng, (n_kv, 1, d_rope), sigma, dtype)
    ct_kv, _, bt = _page(rng, context_lens, block_size, ckv, ckv[:, :, :1], torch.int8)
    # kRope goes through the same block table: page it again with the table just drawn
    k_rope = (torch.where(torch.arange(d_rope) % 2 == 0, 1.0, -1.0) * _POISON[dtype]).to(dtype).repeat(
        ct_kv.shape[0], block_size, 1, 1)
    pos = 0
    for b, L in enumerate(context_lens.tolist()):
        for p_ in range((L + block_size - 1) // block_size):
            lo, n = p_ * block_size, min(block_size, L - p_ * block_size)
            k_rope[int(bt[b, p_]), :n] = kr[pos + lo: pos + lo + n]
        pos += L
    return MlaCase(name=name, dtype=dtype, q_nope=q_nope, q_rope=q_rope, ct_kv=ct_kv, k_rope=k_rope,
                   block_tables=bt, context_lens=context_lens, q_seq_len=q_seq_len, heads=heads,
                   qk_scale=1.0 / math.sqrt(d_nope + d_rope),
                   calc_type=MLA_CALC_SPEC if spec else MLA_CALC_UNDEFINED,
                   mask_type=MLA_MASK_SPEC if spec else MLA_MASK_UNDEFINED, block_size=block_size,
                   qk_descale=qk_descale, pv_descale=pv_descale)


def mla_decode_int8(seed=1004, batch=64, lo=1024, hi=16384, heads=128, qs=1) -> MlaCase:
    """The MLA decode workload over an int8 latent cache: batch 64, contextLens ~ U{1024..16384}, 128 heads,
    512 + 64, paged bs = 128, int8 qNope and ctKV, bf16 qRope / kRope."""
    rng = np.random.Generator(np.random.PCG64(seed))
    ctx = rng.integers(lo, hi + 1, size=batch).astype(np.int32)
    return make_mla_int8(f"mla_qs{qs}_int8_b{batch}_h{heads}", ctx, qs, heads, seed, rng=rng)
