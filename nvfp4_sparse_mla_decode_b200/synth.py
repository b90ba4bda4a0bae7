"""Seeded synthetic inputs for NVFP4 sparse MLA decode.

This module only draws random numbers and lays them out (BF16 cache source
rows, FP16 queries, paged slot tables, index lists).  It holds none of the
method's arithmetic -- no quantization, no attention -- so both the CUDA path
and the CPU oracle can be fed from it without sharing any method code.

The value distributions follow the workloads used on the pages' deployment
(page "Prime Intellect Launches Prime Inference, Serving 600B Tokens Daily",
sections "Why agents strain inference servers" -- a ~6K-token turn on a
140K-token prompt -- and "Four-bit caches make room" -- 2,048-position sparse
lists, a 35-token decode launch):

* cache source rows: BF16 N(0,1) times one per-channel scale vector
  U[0.25, 4] of length 576 (512 latent + 64 RoPE) per workload;
* queries: FP16 N(0,1);
* caches are paged (page size 64); each request owns a random set of pages;
* index lists hold slot ids (page * 64 + offset), -1 for an empty entry.

Row content is a function of (seed, slot chunk), so any subset of rows can be
regenerated on the same device for the oracle without keeping the whole
BF16 source resident.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Iterator, Optional, Sequence

import torch

PAGE_SIZE = 64
LATENT = 512
ROPE = 64
TOPK = 2048
CHUNK_ROWS = 1 << 19


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & ((1 << 63) - 1))
    return g


def channel_scale(seed: int, device) -> torch.Tensor:
    """One per-channel scale vector U[0.25, 4] of length 576 (float32)."""
    g = _gen(device, seed * 1_000_003 + 17)
    return 0.25 + 3.75 * torch.rand(LATENT + ROPE, generator=g, device=device)


@dataclasses.dataclass
class SlotRows:
    """Deterministic BF16 source content for every slot of a cache.

    Rows are produced in chunks of ``chunk_rows`` slots; chunk c is drawn
    from a generator seeded by (seed, c) on ``device``.  ``special`` adds the
    append-workload patterns (1% all-zero groups, 1% groups holding a +-448
    outlier) when set.
    """
    seed: int
    num_slots: int
    device: str
    chunk_rows: int = CHUNK_ROWS
    special: bool = False

    def __post_init__(self):
        self.scale = channel_scale(self.seed, self.device)

    def chunk(self, c: int) -> tuple[torch.Tensor, torch.Tensor]:
        lo = c * self.chunk_rows
        n = min(self.chunk_rows, self.num_slots - lo)
        return source_rows(n, self.scale, self.seed * 7919 + 101 * c + 3, self.device, self.special)

    def chunks(self) -> Iterator[tuple[int, torch.Tensor, torch.Tensor]]:
        for c in range(math.ceil(self.num_slots / self.chunk_rows)):
            lat, rope = self.chunk(c)
            yield c * self.chunk_rows, lat, rope

    def rows(self, slots: torch.Tensor) -> tuple[torch.Tensor, torch.Tensor]:
        """BF16 source rows for the given slot ids (any order, repeats ok)."""
        slots = slots.to(device=self.device, dtype=torch.int64)
        lat = torch.empty(slots.numel(), LATENT, dtype=torch.bfloat16, device=self.device)
        rope = torch.empty(slots.numel(), ROPE, dtype=torch.bfloat16, device=self.device)
        which = torch.div(slots, self.chunk_rows, rounding_mode="floor")
        for c in torch.unique(which).tolist():
            sel = (which == c).nonzero().flatten()
            clat, crope = self.chunk(int(c))
            off = slots[sel] - c * self.chunk_rows
            lat[sel] = clat[off]
            rope[sel] = crope[off]
        return lat, rope


def source_rows(n: int, scale: torch.Tensor, seed: int, device, special: bool = False):
    """n BF16 rows N(0,1)*scale -> (latent [n,512], rope [n,64]).

    With ``special``: 1% of the 32 latent groups of 16 are all zero and 1% of
    groups carry one element set to +-448 (exactly representable in BF16 and
    the largest finite E4M3 value)."""
    g = _gen(device, seed)
    x = torch.randn(n, LATENT + ROPE, generator=g, device=device) * scale
    if special and n:
        grp = x[:, :LATENT].view(n, LATENT // 16, 16)
        u = torch.rand(n, LATENT // 16, generator=g, device=device)
        zero = u < 0.01
        outl = (u >= 0.01) & (u < 0.02)
        grp[zero] = 0.0
        pos = torch.randint(0, 16, (n, LATENT // 16), generator=g, device=device)
        sign = torch.where(torch.rand(n, LATENT // 16, generator=g, device=device) < 0.5, -448.0, 448.0)
        rows_i, grp_i = outl.nonzero(as_tuple=True)
        grp[rows_i, grp_i, pos[rows_i, grp_i]] = sign[rows_i, grp_i]
    x = x.to(torch.bfloat16)
    return x[:, :LATENT].contiguous(), x[:, LATENT:].contiguous()


def queries(T: int, H: int, seed: int, device):
    """FP16 N(0,1) queries: (q_nope [T,H,512], q_rope [T,H,64])."""
    g = _gen(device, seed * 31 + 7)
    q = torch.randn(T, H, LATENT + ROPE, generator=g, device=device).to(torch.float16)
    return q[..., :LATENT].contiguous(), q[..., LATENT:].contiguous()


def page_tables(ctx_lens: Sequence[int], num_pages: int, seed: int, device) -> list[torch.Tensor]:
    """Give each request ceil(ctx/64) distinct pages drawn at random from
    [0, num_pages)."""
    need = [math.ceil(c / PAGE_SIZE) for c in ctx_lens]
    assert sum(need) <= num_pages
    g = _gen("cpu", seed * 131 + 5)
    perm = torch.randperm(num_pages, generator=g)
    out, at = [], 0
    for k in need:
        out.append(perm[at:at + k].to(device))
        at += k
    return out


def positions_to_slots(pos: torch.Tensor, table: torch.Tensor) -> torch.Tensor:
    """Context positions -> slot ids through a page table (-1 stays -1)."""
    valid = pos >= 0
    p = pos.clamp(min=0).to(torch.int64)
    slot = table[torch.div(p, PAGE_SIZE, rounding_mode="floor")] * PAGE_SIZE + p % PAGE_SIZE
    return torch.where(valid, slot, torch.full_like(slot, -1)).to(torch.int32)


def draw_positions(limits: torch.Tensor, k: int, seed: int, device, batch: int = 128) -> torch.Tensor:
    """For each row i, min(k, limits[i]) distinct positions drawn uniformly
    from [0, limits[i]), in random order, padded with -1 to width k.  Random
    keys + top-k: the k largest of iid uniform keys over the allowed
    positions are a uniform k-subset in uniformly random order."""
    T = limits.numel()
    out = torch.full((T, k), -1, dtype=torch.int32, device=device)
    g = _gen(device, seed * 977 + 11)
    lim = limits.to(device=device, dtype=torch.int64)
    for t0 in range(0, T, batch):
        t1 = min(T, t0 + batch)
        n = int(lim[t0:t1].max().item())
        keys = torch.rand(t1 - t0, n, generator=g, device=device)
        ar = torch.arange(n, device=device)
        keys = torch.where(ar[None, :] < lim[t0:t1, None], keys, torch.full_like(keys, -1.0))
        kk = min(k, n)
        val, idx = torch.topk(keys, kk, dim=1)
        idx = torch.where(val >= 0, idx, torch.full_like(idx, -1)).to(torch.int32)
        out[t0:t1, :kk] = idx
    return out


@dataclasses.dataclass
class Workload:
    """A decode workload: cache geometry + per-token index lists + queries.

    ``indices`` is int32 [T, 2048] of slot ids (-1 = empty); the cache has
    ``num_slots`` rows whose BF16 source is ``rows`` (and, for the append
    workload, ``new_rows`` placed at ``new_slots``)."""
    name: str
    T: int
    H: int
    num_slots: int
    indices: torch.Tensor
    q_nope: torch.Tensor
    q_rope: torch.Tensor
    rows: SlotRows
    sm_scale: float = 1.0 / math.sqrt(LATENT + ROPE)
    new_lat: Optional[torch.Tensor] = None
    new_rope: Optional[torch.Tensor] = None
    new_slots: Optional[torch.Tensor] = None
    ctx_lens: Optional[list] = None
    tables: Optional[list] = None
    positions: Optional[torch.Tensor] = None  # [T, 2048] request-local positions behind ``indices``

    def source_rows(self, slots: torch.Tensor):
        """BF16 source of the given slots as the cache holds them after any
        append (new rows override the base content of their slots)."""
        lat, rope = self.rows.rows(slots)
        if self.new_slots is not None:
            ns = self.new_slots.to(device=lat.device, dtype=torch.int64)
            slots_d = slots.to(device=lat.device, dtype=torch.int64)
            order = torch.argsort(ns)
            ns_sorted = ns[order]
            loc = torch.searchsorted(ns_sorted, slots_d).clamp(max=ns.numel() - 1)
            hit = ns_sorted[loc] == slots_d
            src = order[loc[hit]]
            lat[hit] = self.new_lat.to(lat.device)[src]
            rope[hit] = self.new_rope.to(lat.device)[src]
        return lat, rope


def tiny(device, T=1, H=16, num_slots=8192, nvalid=1500, seed=0) -> Workload:
    """One request over an 8192-row cache (page 64); each token's list holds
    ``nvalid`` distinct uniform rows first, then -1 entries."""
    tables = page_tables([num_slots], num_slots // PAGE_SIZE, seed, device)
    lim = torch.full((T,), num_slots, dtype=torch.int64)
    pos = draw_positions(lim, nvalid, seed, device)
    idx = torch.full((T, TOPK), -1, dtype=torch.int32, device=device)
    idx[:, :nvalid] = positions_to_slots(pos, tables[0])
    qn, qr = queries(T, H, seed, device)
    return Workload("tiny", T, H, num_slots, idx, qn, qr, SlotRows(seed, num_slots, device))


def per_request(device, ctx_lens: Sequence[int], H: int, seed: int, name: str,
                pad_lists: bool = False, sort_half: bool = False) -> Workload:
    """One query token per request; request t owns ctx_lens[t] rows in a
    shared paged cache and draws min(ctx, 2048) distinct positions.  With
    ``pad_lists`` the rest of each list is -1; ``sort_half`` sorts the first
    half of the lists ascending (so their -1 entries lead) and leaves the
    other half in random order."""
    T = len(ctx_lens)
    pages = sum(math.ceil(c / PAGE_SIZE) for c in ctx_lens)
    num_slots = pages * PAGE_SIZE
    tables = page_tables(ctx_lens, pages, seed, device)
    lim = torch.tensor(list(ctx_lens), dtype=torch.int64)
    pos = draw_positions(lim, TOPK, seed, device)
    idx = torch.empty(T, TOPK, dtype=torch.int32, device=device)
    for t in range(T):
        idx[t] = positions_to_slots(pos[t], tables[t])
    if pad_lists:
        g = _gen(device, seed * 13 + 1)
        for t in range(T):
            if sort_half and t < T // 2:
                idx[t] = torch.sort(idx[t]).values
            else:
                idx[t] = idx[t][torch.randperm(TOPK, generator=g, device=device)]
    qn, qr = queries(T, H, seed, device)
    return Workload(name, T, H, num_slots, idx, qn, qr, SlotRows(seed, num_slots, device),
                    ctx_lens=list(ctx_lens), tables=tables, positions=None if pad_lists else pos)


def block_table(w: Workload, width: Optional[int] = None) -> torch.Tensor:
    """The requests' page tables as one int32 [T, width] tensor, -1 padded."""
    assert w.tables is not None
    width = width or max(int(tb.numel()) for tb in w.tables)
    out = torch.full((w.T, width), -1, dtype=torch.int32, device=w.indices.device)
    for t, tb in enumerate(w.tables):
        out[t, :tb.numel()] = tb.to(torch.int32)
    return out


def redraw(w: Workload, seed: int) -> tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """A fresh (indices, q_nope, q_rope) for the same requests, contexts and
    cache as ``w`` (one request per token, full 2048-entry lists)."""
    assert w.ctx_lens is not None and w.tables is not None
    device = w.indices.device
    lim = torch.tensor(list(w.ctx_lens), dtype=torch.int64)
    pos = draw_positions(lim, w.indices.shape[1], seed, device)
    idx = torch.empty_like(w.indices)
    for t in range(w.T):
        idx[t] = positions_to_slots(pos[t], w.tables[t])
    qn, qr = queries(w.T, w.H, seed, device)
    return idx, qn, qr


INDEX_HEADS = 64
INDEX_DIM = 128


def indexer_keys(num_slots: int, seed: int, device, chunk_rows: int = CHUNK_ROWS) -> torch.Tensor:
    """Indexer key cache, uint8 [num_slots, 128]: the E4M3 bytes (torch's
    float8_e4m3fn conversion) of N(0,1) draws, chunk c drawn from a generator
    seeded by (seed, c)."""
    out = torch.empty(num_slots, INDEX_DIM, dtype=torch.uint8, device=device)
    for c, lo in enumerate(range(0, num_slots, chunk_rows)):
        n = min(chunk_rows, num_slots - lo)
        g = _gen(device, seed * 6151 + 37 * c + 1)
        x = torch.randn(n, INDEX_DIM, generator=g, device=device)
        out[lo:lo + n] = x.to(torch.float8_e4m3fn).view(torch.uint8)
    return out


def indexer_queries(T: int, seed: int, device) -> tuple[torch.Tensor, torch.Tensor]:
    """Indexer queries uint8 [T, 64, 128] (E4M3 bytes of N(0,1) draws) and
    head weights float32 [T, 64] (N(0,1) / 8, both signs)."""
    g = _gen(device, seed * 389 + 23)
    q = torch.randn(T, INDEX_HEADS, INDEX_DIM, generator=g, device=device)
    w = torch.randn(T, INDEX_HEADS, generator=g, device=device) / 8
    return q.to(torch.float8_e4m3fn).view(torch.uint8).contiguous(), w.contiguous()


def decode35(device, seed=1, ctx=140_000, T=35, H=64) -> Workload:
    """35 query tokens from 35 requests, each with a 140,000-row context."""
    return per_request(device, [ctx] * T, H, seed, "decode35x64")


def sweep(device, T: int, seed=2, H=128, lo=134_000, hi=146_000) -> Workload:
    """One token per request, contexts uniform in [lo, hi], H=128."""
    g = _gen("cpu", seed * 41 + T)
    ctx = torch.randint(lo, hi + 1, (T,), generator=g).tolist()
    return per_request(device, ctx, H, seed, "sweep%dx%d" % (T, H))


def padded(device, T=256, H=64, seed=3, lo=16, hi=4096) -> Workload:
    """Contexts log-uniform in [lo, hi]; lists hold min(ctx, 2048) rows and
    -1 elsewhere; half the lists sorted ascending, half in random order."""
    g = _gen("cpu", seed * 43 + 9)
    u = torch.rand(T, generator=g, dtype=torch.float64)
    ctx = torch.exp(math.log(lo) + u * (math.log(hi) - math.log(lo))).round().to(torch.int64)
    ctx = ctx.clamp(lo, hi).tolist()
    return per_request(device, ctx, H, seed, "padded%dx%d" % (T, H), pad_lists=True, sort_half=True)


def append_prefill(device, T=4000, H=64, history=146_000, seed=4, extra_pages=64) -> Workload:
    """A 4000-row chunk appended into scattered free pages of a cache that
    holds a 146,000-row history; token i attends to 2048 distinct positions
    of history + new rows 0..i (causal)."""
    hist_pages = math.ceil(history / PAGE_SIZE)
    new_pages = math.ceil(T / PAGE_SIZE)
    num_pages = hist_pages + new_pages + extra_pages
    num_slots = num_pages * PAGE_SIZE
    g = _gen("cpu", seed * 131 + 5)
    perm = torch.randperm(num_pages, generator=g)
    hist_table = perm[:hist_pages].to(device)
    new_table = perm[hist_pages:hist_pages + new_pages].to(device)
    new_pos = torch.arange(T, device=device)
    new_slots = positions_to_slots(new_pos, new_table)
    rows = SlotRows(seed, num_slots, device)
    new_lat, new_rope = source_rows(T, rows.scale, seed * 7919 + 999_983, device, special=True)
    lim = history + 1 + torch.arange(T, dtype=torch.int64)
    pos = draw_positions(lim, TOPK, seed, device)
    p = pos.to(torch.int64)
    hist_slot = positions_to_slots(p.clamp(max=history - 1), hist_table).to(torch.int64)
    new_slot = new_slots.to(torch.int64)[(p - history).clamp(min=0, max=T - 1)]
    idx = torch.where(p < history, hist_slot, new_slot).to(torch.int32)
    qn, qr = queries(T, H, seed, device)
    return Workload("append_prefill%dx%d" % (T, H), T, H, num_slots, idx, qn, qr, rows,
                    new_lat=new_lat, new_rope=new_rope, new_slots=new_slots)
