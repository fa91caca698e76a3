"""Seeded synthetic decode batches for paged FP8-KV decode attention.

This module only draws inputs: sequence lengths, page pools, page tables,
page tags, queries and new K/V tokens.  It holds none of the method's
arithmetic (no quantisation, no attention, no tag comparison); the CUDA path
and the CPU oracle each compute everything from these inputs on their own.

Structure (lengths, page assignment, tags) comes from numpy's PCG64 seeded
with the workload's seed.  Bulk values (queries, K/V pools, new tokens) come
from a torch generator seeded with the same seed on the device that will hold
them, so a workload drawn on the GPU and one drawn on the CPU share structure
but not bulk values; a test that compares two implementations draws once and
copies.

Value recipe, as the workloads state it: Q ~ N(0, 1); K and V ~ N(0, 1) with
each element independently multiplied by 20 with probability 0.01; every
value is drawn in fp32 and rounded to bf16 (the activation dtype a model
produces).  The per-tensor FP8 scales are amax / 448 over the whole generated
K (resp. V) pool, as the workloads prescribe; they are inputs of the method.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

E4M3_MAX = 448.0          # largest finite E4M3 value (OCP E4M3), used for the scale recipe
OUTLIER_P = 0.01
OUTLIER_MUL = 20.0


@dataclass
class DecodeBatch:
    """One decode step's inputs.  Caches are laid out [NP][Hkv][P][D]."""
    name: str
    seed: int
    page_size: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    num_pages: int
    seq_lens: np.ndarray           # int32 [B], counts the new token
    page_table: np.ndarray         # int32 [B][MP], -1 past the used entries
    page_tags: np.ndarray          # uint32 [NP]
    expected_tags: np.ndarray      # uint32 [B][MP]
    q: torch.Tensor                # bf16 [B][Hq][D]
    k_pool: torch.Tensor           # bf16 [NP][Hkv][P][D]
    v_pool: torch.Tensor           # bf16 [NP][Hkv][P][D]
    k_new: torch.Tensor            # bf16 [B][Hkv][D]
    v_new: torch.Tensor            # bf16 [B][Hkv][D]
    k_scale: float                 # fp32 value, amax(K pool) / 448
    v_scale: float                 # fp32 value, amax(V pool) / 448
    sm_scale: float                # fp32 value of 1/sqrt(D)
    stale_entries: list = field(default_factory=list)   # (b, j) given a stale expected tag
    notes: str = ""

    @property
    def batch(self) -> int:
        return int(self.seq_lens.shape[0])

    @property
    def max_pages(self) -> int:
        return int(self.page_table.shape[1])

    def used_pages(self, b: int) -> int:
        L = int(self.seq_lens[b])
        return (L + self.page_size - 1) // self.page_size

    def logical_tokens(self) -> int:
        return int(self.seq_lens.astype(np.int64).sum())

    def unique_pages(self) -> int:
        s = set()
        for b in range(self.batch):
            s.update(self.page_table[b, : self.used_pages(b)].tolist())
        return len(s)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _draw_kv(shape, gen, device, chunk=1 << 26) -> torch.Tensor:
    """N(0,1) with 1% of elements x20, drawn in fp32 chunks, rounded to bf16."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(-1)
    n = flat.numel()
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        x = torch.randn(e - s, generator=gen, device=device, dtype=torch.float32)
        u = torch.rand(e - s, generator=gen, device=device, dtype=torch.float32)
        x = torch.where(u < OUTLIER_P, x * OUTLIER_MUL, x)
        flat[s:e] = x.to(torch.bfloat16)
    return out


def _draw_q(shape, gen, device) -> torch.Tensor:
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)


def _amax_scale(pool: torch.Tensor) -> float:
    amax = float(pool.abs().amax().float().item())
    if amax == 0.0:
        return 1.0
    return float(np.float32(amax) / np.float32(E4M3_MAX))


def _sm_scale(head_dim: int) -> float:
    return float(np.float32(1.0 / math.sqrt(head_dim)))


def _finish(name, seed, rng, lens, page_table, num_pages, P, Hq, Hkv, D, device,
            tags=None, notes="") -> DecodeBatch:
    lens = np.asarray(lens, dtype=np.int32)
    B = lens.shape[0]
    if tags is None:
        tags = rng.integers(0, 2**32, size=num_pages, dtype=np.uint64).astype(np.uint32)
    expected = np.zeros_like(page_table, dtype=np.uint32)
    for b in range(B):
        n = (int(lens[b]) + P - 1) // P
        expected[b, :n] = tags[page_table[b, :n]]
    gen = _gen(seed, device)
    q = _draw_q((B, Hq, D), gen, device)
    k_pool = _draw_kv((num_pages, Hkv, P, D), gen, device)
    v_pool = _draw_kv((num_pages, Hkv, P, D), gen, device)
    k_new = _draw_kv((B, Hkv, D), gen, device)
    v_new = _draw_kv((B, Hkv, D), gen, device)
    return DecodeBatch(name=name, seed=seed, page_size=P, num_q_heads=Hq, num_kv_heads=Hkv,
                       head_dim=D, num_pages=num_pages, seq_lens=lens,
                       page_table=page_table.astype(np.int32), page_tags=tags.astype(np.uint32),
                       expected_tags=expected, q=q, k_pool=k_pool, v_pool=v_pool,
                       k_new=k_new, v_new=v_new, k_scale=_amax_scale(k_pool),
                       v_scale=_amax_scale(v_pool), sm_scale=_sm_scale(D), notes=notes)


def _contiguous_tables(rng, lens, P, spare_pages=0, max_pages=None):
    """Each sequence gets its own pages, drawn from a seeded permutation."""
    need = [(int(L) + P - 1) // P for L in lens]
    num_pages = sum(need) + spare_pages
    perm = rng.permutation(num_pages).astype(np.int32)
    MP = max(need) if max_pages is None else max_pages
    table = np.full((len(lens), max(MP, 1)), -1, dtype=np.int32)
    off = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[off: off + n]
        off += n
    return table, num_pages


def custom(lens, page_size=64, num_q_heads=64, num_kv_heads=8, head_dim=128, seed=0,
           device="cpu", spare_pages=0, max_pages=None, name="custom") -> DecodeBatch:
    """Any lengths and shapes, each sequence on private pages."""
    rng = np.random.Generator(np.random.PCG64(seed))
    table, NP = _contiguous_tables(rng, lens, page_size, spare_pages, max_pages)
    return _finish(name, seed, rng, lens, table, NP, page_size, num_q_heads, num_kv_heads,
                   head_dim, device)


def from_table(lens, page_table, num_pages, page_size=64, num_q_heads=64, num_kv_heads=8,
               head_dim=128, seed=0, device="cpu", name="from_table") -> DecodeBatch:
    """Given lengths and page table (pages may be shared between rows); the
    contents of the pools, queries and new tokens are drawn as everywhere."""
    rng = np.random.Generator(np.random.PCG64(seed))
    table = np.asarray(page_table, dtype=np.int32)
    return _finish(name, seed, rng, lens, table, num_pages, page_size, num_q_heads, num_kv_heads,
                   head_dim, device)


def tiny_decode(seed=1, device="cpu") -> DecodeBatch:
    """2 sequences of 37 and 100 tokens, P=16, Hq=4, Hkv=1, D=64, a pool of 16
    pages assigned by a seeded permutation, random tags with one stale
    expected tag at a seeded page of sequence 1."""
    rng = np.random.Generator(np.random.PCG64(seed))
    P, NP = 16, 16
    lens = np.array([37, 100], dtype=np.int32)
    perm = rng.permutation(NP).astype(np.int32)
    table = np.full((2, 7), -1, dtype=np.int32)
    table[0, :3] = perm[:3]
    table[1, :7] = perm[3:10]
    wl = _finish("tiny_decode", seed, rng, lens, table, NP, P, 4, 1, 64, device)
    j = int(rng.integers(0, 7))
    wl.expected_tags[1, j] = np.uint32((int(wl.expected_tags[1, j]) - 1) % 2**32)
    wl.stale_entries = [(1, j)]
    return wl


def concurrency_sweep(batch, seed=2, device="cpu", context=8192) -> DecodeBatch:
    """`batch` sequences at `context` tokens, P=64, Hq=64, Hkv=8, D=128."""
    rng = np.random.Generator(np.random.PCG64(seed * 1000 + batch))
    lens = np.full(batch, context, dtype=np.int32)
    table, NP = _contiguous_tables(rng, lens, 64)
    return _finish(f"concurrency_sweep_b{batch}", seed, rng, lens, table, NP, 64, 64, 8, 128,
                   device)


CAPACITY_TOKENS_FP8 = 1_372_160
CAPACITY_TOKENS_BF16 = 686_080


def capacity(kv_dtype="fp8", seed=3, device="cpu") -> DecodeBatch:
    """One layer's byte budget of 1,372,160 FP8 tokens = 686,080 BF16 tokens
    (8 KV heads x D=128, P=64): 64 FP8 or 32 BF16 sequences of 21,440 tokens."""
    rng = np.random.Generator(np.random.PCG64(seed))
    B = 64 if kv_dtype == "fp8" else 32
    lens = np.full(B, 21_440, dtype=np.int32)
    table, NP = _contiguous_tables(rng, lens, 64)
    return _finish(f"capacity_{kv_dtype}", seed, rng, lens, table, NP, 64, 64, 8, 128, device)


def integrity_stress(seed=4, stale_fraction=0.001, device="cpu", batch=256,
                     lo=1024, hi=16384, rounds=3) -> DecodeBatch:
    """256 sequences, L ~ U[1024, 16384], P=64; a pool of exactly the pages
    needed, freed, shuffled and reallocated for `rounds` seeded rounds with
    every reassigned page's tag bumped by one; then a fraction of the used
    page-table entries get a stale expected tag (tag - 1)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    P = 64
    lens = rng.integers(lo, hi + 1, size=batch).astype(np.int32)
    need = [(int(L) + P - 1) // P for L in lens]
    NP = sum(need)
    tags = rng.integers(0, 2**32, size=NP, dtype=np.uint64).astype(np.uint32)
    table = np.full((batch, max(need)), -1, dtype=np.int32)
    for _ in range(rounds):
        order = rng.permutation(NP).astype(np.int32)
        off = 0
        for b, n in enumerate(need):
            table[b, :n] = order[off: off + n]
            off += n
        tags = (tags.astype(np.uint64) + 1).astype(np.uint32)   # every page was reassigned
    wl = _finish("integrity_stress", seed, rng, lens, table, NP, P, 64, 8, 128, device, tags=tags)
    total = sum(need)
    n_stale = int(round(stale_fraction * total))
    flat = rng.choice(total, size=n_stale, replace=False) if n_stale else []
    starts = np.concatenate([[0], np.cumsum(need)])
    for f in sorted(int(x) for x in flat):
        b = int(np.searchsorted(starts, f, side="right") - 1)
        j = f - int(starts[b])
        wl.expected_tags[b, j] = np.uint32((int(wl.expected_tags[b, j]) - 1) % 2**32)
        wl.stale_entries.append((b, j))
    return wl


def ragged_prefix(seed=5, device="cpu", batch=512, group=8, prefix_pages=64) -> DecodeBatch:
    """512 sequences, L ~ LogNormal(ln 2048, 1.2) clipped to [16, 131072], P=64.
    Groups of 8 consecutive sequences share the physical pages of a common
    4,096-token prefix: sequence b maps its first min(64, (L_b - 1) // 64)
    entries to the group's shared pages, so the page holding its newest
    token is always private."""
    rng = np.random.Generator(np.random.PCG64(seed))
    P = 64
    lens = np.clip(np.rint(rng.lognormal(mean=math.log(2048.0), sigma=1.2, size=batch)),
                   16, 131072).astype(np.int32)
    need = [(int(L) + P - 1) // P for L in lens]
    shared = [min(prefix_pages, (int(L) - 1) // P) for L in lens]
    n_groups = (batch + group - 1) // group
    private = sum(n - s for n, s in zip(need, shared))
    NP = n_groups * prefix_pages + private
    perm = rng.permutation(NP).astype(np.int32)
    table = np.full((batch, max(need)), -1, dtype=np.int32)
    off = 0
    group_pages = []
    for gi in range(n_groups):
        group_pages.append(perm[off: off + prefix_pages])
        off += prefix_pages
    for b in range(batch):
        s, n = shared[b], need[b]
        table[b, :s] = group_pages[b // group][:s]
        table[b, s:n] = perm[off: off + (n - s)]
        off += n - s
    return _finish("ragged_prefix", seed, rng, lens, table, NP, P, 64, 8, 128, device,
                   notes="prefix pages shared within groups of 8")


# --------------------------------------------------------------------------
# INT4 weight dequantisation GEMV (decode)
# --------------------------------------------------------------------------

INT4_GROUP = 128          # columns of one row sharing a scale
INT4_N = 32768            # output features of the synthetic projection
INT4_K = 8192             # input features
INT4_BATCHES = (1, 8, 16, 32, 64)   # the concurrency levels the pages tabulate


@dataclass
class Int4Gemv:
    """Inputs of one decode-time INT4 GEMV y = x W^T.

    ``w_tiles`` holds the codes in the tiled layout ([n/128][k/256] tiles of
    128 rows x 128 bytes); it is filled with uniformly random bytes, and
    every byte is a valid pair of signed 4-bit codes, so the codes are
    uniform over -8..7 and this module packs nothing.  ``scales``
    [n/128][k/group][128] are bf16 values drawn log-uniformly in
    [2^-10, 2^-4]; x ~ N(0, 1) rounded to bf16.
    """
    name: str
    seed: int
    group: int
    x: torch.Tensor          # bf16 [B][k]
    w_tiles: torch.Tensor    # uint8 [n/128][k/256][128][128]
    scales: torch.Tensor     # bf16 [n/128][k/group][128]

    @property
    def batch(self) -> int:
        return int(self.x.shape[0])

    @property
    def n(self) -> int:
        return int(self.w_tiles.shape[0]) * 128

    @property
    def k(self) -> int:
        return int(self.x.shape[1])


def int4_gemv_case(batch, n=INT4_N, k=INT4_K, group=INT4_GROUP, seed=6, device="cpu",
                   w_tiles=None, scales=None) -> Int4Gemv:
    """A seeded INT4 GEMV case.  ``w_tiles``/``scales`` may be passed in to
    share one weight matrix between several batch sizes."""
    g = _gen(seed, device)
    if w_tiles is None:
        w_tiles = torch.randint(0, 256, (n // 128, k // 256, 128, 128), generator=g, device=device,
                                dtype=torch.int32).to(torch.uint8)
    if scales is None:
        e = torch.rand((n // 128, k // group, 128), generator=g, device=device, dtype=torch.float32)
        scales = torch.exp2(-10.0 + 6.0 * e).to(torch.bfloat16)
    gx = _gen(seed * 1000 + batch, device)
    x = _draw_q((batch, k), gx, device)
    return Int4Gemv(f"int4_gemv_b{batch}", seed, group, x, w_tiles, scales)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Raw uint16 bit patterns of a bf16 tensor, on the host."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
