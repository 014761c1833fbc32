"""Seeded synthetic inputs for paged GQA/MQA decode attention.

This module only builds inputs: sequence lengths, a shuffled page pool, block
tables and bf16 tensors drawn from N(0, 1).  It contains none of the attention
arithmetic, so both the CPU oracle and the CUDA path may use it.

Layouts (row-major, contiguous):
  q, out              [num_seqs, num_heads, head_dim]           bf16
  k_pages, v_pages    [num_pages, num_kv_heads, page_size, head_dim] bf16
  block_table         [num_seqs, max_blocks_per_seq]            int32 (-1 = unused)
  seq_lens            [num_seqs]                                int32
  positions           [num_seqs]                                int32 (kv_append slot)
  k_new, v_new        [num_seqs, num_kv_heads, head_dim]        bf16

Token t of sequence b lives in page block_table[b][t // page_size], slot
t % page_size; query head h reads kv head h // (num_heads // num_kv_heads).

The five workloads follow the decode-attention problem described on the page
"TensorRT对Multi-Query Attention的专项优化支持" (MQA: every query head shares one
K/V head; paged KV cache in fixed-size pages) and the GQA / paged-KV notes of the
tiny-llm "优化" page (num_kv_heads may differ from num_heads; block table +
scatter/gather).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

__all__ = [
    "WORKLOADS",
    "WorkloadSpec",
    "PagedDecodeInputs",
    "make_inputs",
    "make_custom_inputs",
    "make_shrunk_inputs",
    "bf16_bits",
]


@dataclass(frozen=True)
class WorkloadSpec:
    """Static description of one synthetic decode workload."""

    index: int
    name: str
    num_seqs: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    page_size: int
    description: str


# The five decode workloads.  Index 1 is the tiny MQA case the oracle runs in
# milliseconds; index 2 is the GQA serving batch the throughput figure is
# quoted on.
WORKLOADS = {
    1: WorkloadSpec(1, "tiny_mqa", 2, 4, 1, 64, 16,
                    "2 seqs (17, 40 tokens), H=4, Hk=1, D=64, ps=16, 8-page pool"),
    2: WorkloadSpec(2, "gqa_decode", 32, 32, 8, 128, 16,
                    "B=32, H=32, Hk=8, D=128, ps=16, L~U[512,4096], pool 1.25x needed"),
    3: WorkloadSpec(3, "mqa_decode", 64, 96, 1, 128, 64,
                    "B=64, H=96, Hk=1, D=128, ps=64, L=8192, pool exactly needed"),
    4: WorkloadSpec(4, "long_context", 4, 64, 8, 128, 16,
                    "B=4, H=64, Hk=8, D=128, ps=16, L=131072, K x4 on 1% of positions"),
    5: WorkloadSpec(5, "continuous_batch", 256, 32, 8, 128, 16,
                    "B=256, H=32, Hk=8, D=128, ps=16, L log-uniform [1,32768], kv_append"),
}


@dataclass
class PagedDecodeInputs:
    """One batch of decode-step inputs (torch tensors, CPU or CUDA)."""

    name: str
    num_seqs: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    page_size: int
    num_pages: int
    max_blocks_per_seq: int
    scale: float
    seq_lens: torch.Tensor
    block_table: torch.Tensor
    q: torch.Tensor
    k_pages: torch.Tensor
    v_pages: torch.Tensor
    positions: Optional[torch.Tensor] = None
    k_new: Optional[torch.Tensor] = None
    v_new: Optional[torch.Tensor] = None
    meta: dict = field(default_factory=dict)

    @property
    def has_append(self) -> bool:
        return self.positions is not None

    def to(self, device) -> "PagedDecodeInputs":
        def mv(t):
            return None if t is None else t.to(device)

        return PagedDecodeInputs(
            self.name, self.num_seqs, self.num_heads, self.num_kv_heads,
            self.head_dim, self.page_size, self.num_pages,
            self.max_blocks_per_seq, self.scale,
            mv(self.seq_lens), mv(self.block_table), mv(self.q),
            mv(self.k_pages), mv(self.v_pages), mv(self.positions),
            mv(self.k_new), mv(self.v_new), dict(self.meta))

    def total_context_tokens(self) -> int:
        return int(self.seq_lens.to(torch.int64).sum().item())


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Raw bf16 bit patterns of a tensor as a uint16 numpy array (host copy)."""
    assert t.dtype == torch.bfloat16
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _seq_lens_for(spec: WorkloadSpec, gen: torch.Generator) -> torch.Tensor:
    if spec.index == 1:
        return torch.tensor([17, 40], dtype=torch.int32)
    if spec.index == 2:
        return torch.randint(512, 4096 + 1, (spec.num_seqs,), generator=gen,
                             dtype=torch.int64).to(torch.int32)
    if spec.index == 3:
        return torch.full((spec.num_seqs,), 8192, dtype=torch.int32)
    if spec.index == 4:
        return torch.full((spec.num_seqs,), 131072, dtype=torch.int32)
    if spec.index == 5:
        u = torch.rand(spec.num_seqs, generator=gen, dtype=torch.float64)
        lens = torch.round(torch.exp(u * math.log(32768.0)))
        return lens.clamp(1, 32768).to(torch.int32)
    raise ValueError(spec.index)


def _pool_pages_for(spec: WorkloadSpec, needed: int) -> int:
    if spec.index == 1:
        return 8
    if spec.index == 2:
        return int(math.ceil(1.25 * needed))
    return needed  # workloads 3, 4, 5: exactly the needed pages


def _randn_bf16(shape, gen: torch.Generator, device) -> torch.Tensor:
    return torch.randn(shape, generator=gen, dtype=torch.float32,
                       device=device).to(torch.bfloat16)


def _build(name, num_seqs, num_heads, num_kv_heads, head_dim, page_size,
           seq_lens, num_pages, scale, gen_small, gen_big, device,
           poison, append, spike_fraction=0.0, spike_factor=4.0,
           max_blocks_per_seq=None):
    """Assemble the page pool, block table and tensors for given lengths."""
    seq_lens = seq_lens.to(torch.int32)
    B = num_seqs
    pages_per_seq = [(int(L) + page_size - 1) // page_size for L in seq_lens.tolist()]
    needed = sum(pages_per_seq)
    if num_pages < needed:
        raise ValueError("page pool smaller than needed pages")
    mb = max(1, max(pages_per_seq) if pages_per_seq else 1)
    if max_blocks_per_seq is not None:
        mb = max(mb, max_blocks_per_seq)
    perm = torch.randperm(num_pages, generator=gen_small).to(torch.int32)
    block_table = torch.full((B, mb), -1, dtype=torch.int32)
    off = 0
    for b, n in enumerate(pages_per_seq):
        block_table[b, :n] = perm[off:off + n]
        off += n

    q = _randn_bf16((B, num_heads, head_dim), gen_big, device)
    k_pages = _randn_bf16((num_pages, num_kv_heads, page_size, head_dim), gen_big, device)
    v_pages = _randn_bf16((num_pages, num_kv_heads, page_size, head_dim), gen_big, device)

    if spike_fraction > 0.0:
        # Peaked softmax: multiply K by spike_factor (a power of two, so the
        # bf16 product is exact) on a random spike_fraction of each sequence's
        # positions, for every kv head and dimension.
        for b in range(B):
            L = int(seq_lens[b])
            n = int(round(spike_fraction * L))
            if n == 0:
                continue
            pos = torch.randperm(L, generator=gen_small)[:n].to(torch.int64)
            pages = block_table[b].to(torch.int64)[pos // page_size].to(device)
            slots = (pos % page_size).to(device)
            k_pages[pages, :, slots, :] = k_pages[pages, :, slots, :] * spike_factor

    positions = k_new = v_new = None
    if append:
        positions = (seq_lens - 1).clamp(min=0).to(torch.int32)
        k_new = _randn_bf16((B, num_kv_heads, head_dim), gen_big, device)
        v_new = _randn_bf16((B, num_kv_heads, head_dim), gen_big, device)

    if poison:
        # Slots the attention must never read hold NaN: every unused pool page,
        # every slot at or beyond seq_len in a sequence's last page, and (when
        # the step appends) the slot kv_append is about to fill.
        used = torch.zeros(num_pages, dtype=torch.bool)
        for b, n in enumerate(pages_per_seq):
            used[block_table[b, :n].to(torch.int64)] = True
        unused = (~used).nonzero().flatten().to(device)
        nan = float("nan")
        k_pages[unused] = nan
        v_pages[unused] = nan
        for b, n in enumerate(pages_per_seq):
            L = int(seq_lens[b])
            if n == 0:
                continue
            last = int(block_table[b, n - 1])
            first_dead = L - (n - 1) * page_size
            if append and L > 0:
                first_dead -= 1  # the new token's slot is written by kv_append
            if first_dead < page_size:
                k_pages[last, :, first_dead:, :] = nan
                v_pages[last, :, first_dead:, :] = nan

    return PagedDecodeInputs(
        name=name, num_seqs=B, num_heads=num_heads, num_kv_heads=num_kv_heads,
        head_dim=head_dim, page_size=page_size, num_pages=num_pages,
        max_blocks_per_seq=mb, scale=float(scale),
        seq_lens=seq_lens.to(device), block_table=block_table.to(device),
        q=q, k_pages=k_pages, v_pages=v_pages,
        positions=None if positions is None else positions.to(device),
        k_new=k_new, v_new=v_new,
        meta={"pages_needed": needed})


def make_inputs(index: int, seed: Optional[int] = None, device="cpu",
                poison: bool = True) -> PagedDecodeInputs:
    """Inputs of workload `index` (1..5) drawn from a seeded generator.

    Recipe: a CPU torch.Generator seeded with `seed` (default 1000 + index)
    draws, in order, the sequence lengths, the page-pool permutation and any
    spike positions.  The large tensors (q, K/V pool, k_new, v_new) come from a
    second generator on `device` seeded with seed + 1: N(0, 1) in fp32, rounded
    to bf16 (round-to-nearest-even).  Generating on CPU or on CUDA therefore
    gives identical lengths and block tables but different tensor values.
    """
    spec = WORKLOADS[index]
    if seed is None:
        seed = 1000 + index
    gen_small = torch.Generator().manual_seed(seed)
    gen_big = torch.Generator(device=device).manual_seed(seed + 1)
    seq_lens = _seq_lens_for(spec, gen_small)
    pages = [(int(L) + spec.page_size - 1) // spec.page_size for L in seq_lens.tolist()]
    num_pages = _pool_pages_for(spec, sum(pages))
    inp = _build(spec.name, spec.num_seqs, spec.num_heads, spec.num_kv_heads,
                 spec.head_dim, spec.page_size, seq_lens, num_pages,
                 1.0 / math.sqrt(spec.head_dim), gen_small, gen_big, device,
                 poison=poison, append=(index == 5),
                 spike_fraction=0.01 if index == 4 else 0.0)
    inp.meta["workload"] = index
    return inp


def make_shrunk_inputs(index: int, shrink: int, seed: Optional[int] = None, device="cpu",
                       poison: bool = True) -> PagedDecodeInputs:
    """Workload `index` with every context length divided by `shrink` (rounded up): the
    same shapes, page size, length recipe and spike fraction on fewer tokens, for
    profiler captures of a smaller case of the same kernel."""
    spec = WORKLOADS[index]
    if seed is None:
        seed = 1000 + index
    lens = _seq_lens_for(spec, torch.Generator().manual_seed(seed))
    lens = [(int(L) + shrink - 1) // shrink for L in lens.tolist()]
    inp = make_custom_inputs(lens, spec.num_heads, spec.num_kv_heads, spec.head_dim, spec.page_size,
                             seed=seed, device=device, poison=poison,
                             spike_fraction=0.01 if index == 4 else 0.0)
    inp.meta["workload"] = index
    inp.meta["shrink"] = shrink
    return inp


def make_custom_inputs(seq_lens, num_heads, num_kv_heads, head_dim, page_size,
                       seed=0, device="cpu", poison=True, append=False,
                       extra_pages=0, scale=None, spike_fraction=0.0,
                       max_blocks_per_seq=None) -> PagedDecodeInputs:
    """Inputs with caller-chosen lengths and shapes (small parity cases)."""
    gen_small = torch.Generator().manual_seed(seed)
    gen_big = torch.Generator(device=device).manual_seed(seed + 1)
    seq_lens = torch.as_tensor(list(seq_lens), dtype=torch.int32)
    pages = [(int(L) + page_size - 1) // page_size for L in seq_lens.tolist()]
    num_pages = max(1, sum(pages) + extra_pages)
    if scale is None:
        scale = 1.0 / math.sqrt(head_dim)
    return _build("custom", len(seq_lens), num_heads, num_kv_heads, head_dim,
                  page_size, seq_lens, num_pages, scale, gen_small, gen_big,
                  device, poison=poison, append=append,
                  spike_fraction=spike_fraction,
                  max_blocks_per_seq=max_blocks_per_seq)
