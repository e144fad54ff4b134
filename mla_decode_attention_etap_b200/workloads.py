"""Seeded synthetic inputs for MLA decode (shared by the CUDA path's tests/bench and the oracle's tests).

This module only draws inputs: it holds none of the attention arithmetic.  Both
the oracle and the CUDA library receive the tensors it returns.

Shapes follow the DeepSeek-R1 MLA decode shape the FlashMLA-ETAP pages evaluate
("FlashMLA-ETAP", Results: DeepSeek-R1, 16 heads per GPU, head dimension 576,
sequence length up to 64K, batch 16/32):

* ``q``      bf16 ``[B, q_len, h, 576]``  (query tokens; all heads share one latent KV head)
* ``kv``     bf16 contiguous ``[B, L_max, 576]`` or paged ``[num_blocks, 64, 576]``
             (the latent cache; V is the first 512 columns of each row)
* ``seqlens`` int32 ``[B]``
* ``block_table`` int32 ``[B, max_blocks]`` (paged only; unused entries are -1)

Recipe (one ``torch.Generator`` seeded with ``seed``, drawn in this order):
  1. per-sequence lengths, when drawn (``randint`` inclusive range),
  2. Q  ~ N(0,1) fp32, rounded to bf16 (round-to-nearest-even),
  3. KV ~ N(0,1) fp32, rounded to bf16,
  4. the physical block permutation (paged layouts),
  5. the "spike" rows: a fraction of each sequence's KV rows (chosen by a
     per-sequence permutation) multiplied by ``spike_scale`` (exact in bf16 for
     powers of two).

FP8 caches (``kv_dtype="e4m3"``) quantise that bf16 cache row by row (no further
random draws): scale[r] = max_k |kv[r, k]| / 448 in fp32 (1 for an all-zero row)
and code[r, k] = E4M3(kv[r, k] / scale[r]) rounded to nearest-even, so every
row uses the full E4M3 range.  ``kv8`` holds the codes (uint8, same layout as
``kv``) and ``kv_scale`` the fp32 scales ([B, L_max] or [num_blocks, 64]).
"""

from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Optional, Sequence

import torch

D_QK = 576
D_V = 512
PAGE = 64


@dataclass
class Workload:
    q: torch.Tensor
    kv: torch.Tensor
    seqlens: torch.Tensor
    block_table: Optional[torch.Tensor]
    q_len: int
    num_heads: int
    causal: bool
    softmax_scale: float
    q_lens: Optional[torch.Tensor] = None  # ragged batch: real query tokens per sequence (int32 [B])
    kv8: Optional[torch.Tensor] = None      # FP8 cache: E4M3 codes, uint8, laid out like kv
    kv_scale: Optional[torch.Tensor] = None  # FP8 cache: fp32 scale per cache row

    @property
    def fp8(self) -> bool:
        return self.kv8 is not None

    @property
    def batch(self) -> int:
        return int(self.q.shape[0])

    @property
    def paged(self) -> bool:
        return self.block_table is not None

    def kv_rows(self, b: int, rows: Optional[slice] = None) -> torch.Tensor:
        """Logical KV rows of sequence ``b`` ([L_b, 576]) gathered through the block table."""
        L = int(self.seqlens[b])
        if self.block_table is None:
            out = self.kv[b, :L]
        else:
            nb = (L + PAGE - 1) // PAGE
            blocks = self.block_table[b, :nb].long().to(self.kv.device)
            out = self.kv[blocks].reshape(nb * PAGE, D_QK)[:L]
        return out if rows is None else out[rows]


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn_bf16(shape, g, device) -> torch.Tensor:
    # bf16 conversion of an fp32 normal draw is round-to-nearest-even.
    return torch.randn(*shape, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


def draw_seqlens(batch: int, lo: int, hi: int, seed: int) -> list[int]:
    """Per-sequence lengths uniform in [lo, hi] (inclusive), from ``seed``."""
    g = _gen(seed, "cpu")
    return [int(x) for x in torch.randint(lo, hi + 1, (batch,), generator=g)]


def make_workload(
    batch: int,
    num_heads: int,
    seqlens: Sequence[int],
    *,
    q_len: int = 1,
    paged: bool = False,
    causal: bool = False,
    seed: int = 0,
    device="cpu",
    spike_frac: float = 0.0,
    spike_scale: float = 8.0,
    l_max: Optional[int] = None,
    softmax_scale: Optional[float] = None,
    extra_blocks: int = 0,
    q_lens: Optional[Sequence[int]] = None,
    kv_dtype: str = "bf16",
) -> Workload:
    """Draw one synthetic MLA decode batch.

    ``l_max`` (contiguous layout) defaults to ``max(seqlens)``; rows past a
    sequence's length are filled with N(0,1) too.  ``extra_blocks`` adds unused
    physical blocks to the paged pool (they join the permutation).
    """
    assert len(seqlens) == batch
    g = _gen(seed, device)
    seqlens_t = torch.tensor(list(seqlens), dtype=torch.int32)
    q = _randn_bf16((batch, q_len, num_heads, D_QK), g, device)
    if not paged:
        lm = int(l_max if l_max is not None else max(max(seqlens), 1))
        kv = _randn_bf16((batch, lm, D_QK), g, device)
        block_table = None
    else:
        nblk = [(int(L) + PAGE - 1) // PAGE for L in seqlens]
        total = sum(nblk) + extra_blocks
        kv = _randn_bf16((max(total, 1), PAGE, D_QK), g, device)
        perm = torch.randperm(max(total, 1), generator=_gen(seed + 1, "cpu"))
        max_blocks = max(max(nblk), 1)
        block_table = torch.full((batch, max_blocks), -1, dtype=torch.int32)
        off = 0
        for b, nb in enumerate(nblk):
            block_table[b, :nb] = perm[off:off + nb].to(torch.int32)
            off += nb
    if spike_frac > 0.0:
        gs = _gen(seed + 2, "cpu")
        for b, L in enumerate(seqlens):
            L = int(L)
            n_spike = int(round(spike_frac * L))
            if n_spike == 0:
                continue
            rows = torch.randperm(L, generator=gs)[:n_spike]
            if block_table is None:
                kv[b, rows.to(kv.device)] = (kv[b, rows.to(kv.device)].float() * spike_scale).to(torch.bfloat16)
            else:
                blk = block_table[b, (rows // PAGE)].long().to(kv.device)
                off_in = (rows % PAGE).to(kv.device)
                kv[blk, off_in] = (kv[blk, off_in].float() * spike_scale).to(torch.bfloat16)
    scale = softmax_scale if softmax_scale is not None else 1.0 / math.sqrt(D_QK)
    ql = None
    if q_lens is not None:
        assert len(q_lens) == batch and all(0 <= int(x) <= q_len for x in q_lens)
        ql = torch.tensor([int(x) for x in q_lens], dtype=torch.int32)
    kv8 = kv_scale = None
    if kv_dtype == "e4m3":
        kv8, kv_scale = quantize_e4m3_rows(kv)
    else:
        assert kv_dtype == "bf16", kv_dtype
    return Workload(q=q, kv=kv, seqlens=seqlens_t, block_table=block_table, q_len=q_len,
                    num_heads=num_heads, causal=causal, softmax_scale=scale, q_lens=ql, kv8=kv8,
                    kv_scale=kv_scale)


E4M3_MAX = 448.0


def quantize_e4m3_rows(kv: torch.Tensor):
    """Per-row E4M3 quantisation of a [..., 576] cache -> (codes uint8 [..., 576], scale fp32 [...])."""
    x = kv.float()
    amax = x.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    y = (x / scale[..., None]).clamp(-E4M3_MAX, E4M3_MAX)
    codes = y.to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.contiguous(), scale.contiguous()


# The five synthetic workloads (sizes follow the DeepSeek-R1 MLA decode shape).
def workload_b1_h16_l1024(seed: int = 0, device="cpu") -> Workload:
    """B=1, 16 heads, one query token, 1024 contiguous KV rows."""
    return make_workload(1, 16, [1024], seed=seed, device=device)


def workload_b16_h16(seqlen: int, seed: int = 0, device="cpu") -> Workload:
    """B=16, 16 heads, one query token, equal contiguous lengths (4K/16K/32K/64K)."""
    return make_workload(16, 16, [seqlen] * 16, seed=seed, device=device)


def workload_b64_h16_paged(seed: int = 0, device="cpu", batch: int = 64, lmax: int = 65536) -> Workload:
    """B=64, 16 heads, lengths uniform in [1, 65536], 64-token pages in a random permutation."""
    lens = draw_seqlens(batch, 1, lmax, seed)
    return make_workload(batch, 16, lens, paged=True, seed=seed, device=device)


def workload_b32_h128_paged(seed: int = 0, device="cpu", batch: int = 32, lo: int = 8192, hi: int = 32768) -> Workload:
    """B=32, 128 heads, lengths uniform in [8192, 32768], 64-token pages."""
    lens = draw_seqlens(batch, lo, hi, seed)
    return make_workload(batch, 128, lens, paged=True, seed=seed, device=device)


def workload_b16_h16_q4_causal(seed: int = 0, device="cpu", seqlen: int = 32768, batch: int = 16) -> Workload:
    """B=16, 16 heads, 4 causal query tokens at the end of a 32768-row cache, 5% of rows scaled x8."""
    return make_workload(batch, 16, [seqlen] * batch, q_len=4, causal=True, seed=seed, device=device,
                         spike_frac=0.05, spike_scale=8.0)


def workload_b16_h16_ragged_q4_causal(seed: int = 0, device="cpu", seqlen: int = 32768,
                                      batch: int = 16) -> Workload:
    """Ragged speculative verify: B=16, 16 heads, 1..4 causal query tokens per sequence (uniform,
    from ``seed + 3``) at the end of a 32768-row cache, 5% of rows scaled x8."""
    q_lens = draw_seqlens(batch, 1, 4, seed + 3)
    return make_workload(batch, 16, [seqlen] * batch, q_len=4, causal=True, seed=seed, device=device,
                         spike_frac=0.05, spike_scale=8.0, q_lens=q_lens)


def workload_b16_h16_append_q16(seed: int = 0, device="cpu", seqlen: int = 32768, batch: int = 16) -> Workload:
    """Append attention: B=16, 16 heads, 16 new causal tokens at the end of a 32768-row cache
    (256 query columns per sequence)."""
    return make_workload(batch, 16, [seqlen] * batch, q_len=16, causal=True, seed=seed, device=device)


def workload_b16_h16_fp8(seqlen: int, seed: int = 0, device="cpu") -> Workload:
    """B=16, 16 heads, one query token, equal contiguous lengths, FP8 (E4M3 + row scale) cache."""
    return make_workload(16, 16, [seqlen] * 16, seed=seed, device=device, kv_dtype="e4m3")


def workload_b64_h16_paged_fp8(seed: int = 0, device="cpu", batch: int = 64, lmax: int = 65536) -> Workload:
    """The B=64 paged workload with an FP8 (E4M3 + row scale) cache."""
    lens = draw_seqlens(batch, 1, lmax, seed)
    return make_workload(batch, 16, lens, paged=True, seed=seed, device=device, kv_dtype="e4m3")


def bf16_bits(t: torch.Tensor):
    """uint16 numpy view of a bf16 tensor (CPU), for the oracle's C interface."""
    import numpy as np
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def algorithmic_kv_bytes(seqlens: Sequence[int], fp8: bool = False) -> int:
    """KV bytes a decode step must read once: 576 bf16 values per cached token, or 576 E4M3
    codes and one fp32 scale."""
    per_token = D_QK + 4 if fp8 else D_QK * 2
    return sum(int(L) for L in seqlens) * per_token


def algorithmic_flops(seqlens: Sequence[int], q_len: int, num_heads: int, causal: bool,
                      q_lens: Optional[Sequence[int]] = None) -> int:
    """2*(576+512) flops per visible (query column, KV token) pair (padding tokens of a ragged
    batch see no pair)."""
    total = 0
    for b, L in enumerate(seqlens):
        L = int(L)
        qb = q_len if q_lens is None else int(q_lens[b])
        for t in range(qb):
            vis = (L - qb + t + 1) if causal else L
            total += max(vis, 0) * num_heads
    return total * 2 * (D_QK + D_V)
