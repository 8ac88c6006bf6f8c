"""Seeded synthetic decode workloads (inputs only).

This module builds the tensors that both the CUDA library and the CPU oracle consume: queries,
a paged GQA KV cache, page tables, context lengths and per-request k.  It contains none of the
method's arithmetic (no scores, no selection, no softmax); it only draws random numbers and
writes planted structure into the cache.  It imports nothing from the library or the oracle.

Cache layout (NHD pages): K and V are bf16 ``[num_pages, P, Hkv, d]``; logical position ``p`` of
request ``b`` sits at ``[page_table[b, p // P], p % P]``.  Query head ``h`` reads KV head
``h // G`` with ``G = Hq // Hkv``.

Named workloads (shapes from the long-context decode study; the pages' own model tables give the
head counts, e.g. Llama-3.1-8B 32/8 and 70B 64/8, "The Sparse Frontier" review, Table 5):

``tiny``      B=1, Hq/Hkv=8/2, N=4096, k=82; per query head 16 planted keys set to 4*q_h at
              positions disjoint within the group; contiguous (identity) page table.
``llama8b``   B=8, 32/8, N=32768, k=655; 1% heavy-hitter keys per (b, kv head) shifted by 2*mean
              of the group's queries; shuffled page table.
``long128k``  B=4, 64/8, N=131072, k=2621; attention-sink rows 0-3 of K scaled by 3; shuffled
              page table.
``sweep128k`` B=16, 32/8, N=131072, k in {N/10, N/50, N/100, N}; random page table.
``ragged``    B=32, 32/8, N_b ~ U[8192, 163840], k_b = round(N_b/50); pages from a shuffled free
              list, sized for 64 appended decode steps (one K/V row per request per step).

k for a sparsity ratio r is ``max(1, round_half_up(N / r))``: 4096 -> 82, 32768 -> 655,
131072 -> 2621 at r = 50.
"""
from __future__ import annotations

import dataclasses

import torch

HEAD_DIM = 128
PAGE_SIZE = 16

CONFIG_IDS = {"tiny": 1, "llama8b": 2, "long128k": 3, "sweep128k": 4, "ragged": 5}
SWEEP_RATIOS = (10, 50, 100, 1)  # k = N/10, N/50, N/100, N (dense)


def k_for_ratio(n: int, ratio: int) -> int:
    """Selected rows for a sparsity ratio: round half up of n/ratio, at least 1."""
    return max(1, (2 * n + ratio) // (2 * ratio))


@dataclasses.dataclass
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    P: int
    max_pages: int
    num_pages: int
    k_max: int
    q: torch.Tensor            # bf16 [B, Hq, d]
    K: torch.Tensor            # bf16 [num_pages, P, Hkv, d]
    V: torch.Tensor            # bf16 [num_pages, P, Hkv, d]
    page_table: torch.Tensor   # int32 [B, max_pages]
    lens: torch.Tensor         # int32 [B]
    k: torch.Tensor            # int32 [B]
    meta: dict = dataclasses.field(default_factory=dict)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def shape(self) -> dict:
        return dict(B=self.B, Hq=self.Hq, Hkv=self.Hkv, d=self.d, P=self.P, max_pages=self.max_pages,
                    k_max=self.k_max, num_pages=self.num_pages)

    def to(self, device) -> "Workload":
        moved = {}
        for f in dataclasses.fields(self):
            v = getattr(self, f.name)
            moved[f.name] = v.to(device) if isinstance(v, torch.Tensor) else v
        return Workload(**moved)


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _randn_bf16(shape, g: torch.Generator, device, chunk_rows: int = 1 << 14) -> torch.Tensor:
    """bf16 N(0,1) tensor, drawn in chunks of the leading dimension to bound fp32 scratch."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    n0 = shape[0]
    for s in range(0, n0, chunk_rows):
        e = min(n0, s + chunk_rows)
        out[s:e] = torch.randn((e - s,) + tuple(shape[1:]), generator=g, device=device).to(torch.bfloat16)
    return out


def _page_table(B: int, pages_per_req: list[int], max_pages: int, order: str, g, device):
    total = sum(pages_per_req)
    if order == "identity":
        phys = torch.arange(total, dtype=torch.int32, device=device)
    else:
        phys = torch.randperm(total, generator=g, device=device).to(torch.int32)
    pt = torch.full((B, max_pages), -1, dtype=torch.int32, device=device)
    off = 0
    for b, n in enumerate(pages_per_req):
        pt[b, :n] = phys[off:off + n]
        off += n
    return pt, total


def rows_of(w_pt: torch.Tensor, P: int, b: int, positions: torch.Tensor):
    """(page, slot) of logical positions of request b: pure addressing, no arithmetic of the method."""
    pages = w_pt[b].long()[positions // P]
    return pages, positions % P


def make_workload(B: int, Hq: int, Hkv: int, lens, k, *, seed: int = 0, page_order: str = "shuffled",
                  d: int = HEAD_DIM, P: int = PAGE_SIZE, k_max: int | None = None, extra_pages: int = 0,
                  device="cpu", name: str = "custom", structure: str | None = None) -> Workload:
    """Generic seeded workload.

    lens: int or list of per-request context lengths.  k: int or list of per-request k.
    page_order: "shuffled" (random permutation of physical pages) or "identity" (contiguous).
    extra_pages: pages reserved per request beyond ceil(N_b/P) (page-table room for appends).
    structure: None, "planted16", "heavy1pct" or "sinks3" (see module docstring).
    """
    device = torch.device(device)
    g = _gen(device, seed)
    lens_l = [int(lens)] * B if isinstance(lens, int) else [int(x) for x in lens]
    k_l = [int(k)] * B if isinstance(k, int) else [int(x) for x in k]
    assert len(lens_l) == B and len(k_l) == B
    pages_per_req = [(n + P - 1) // P + extra_pages for n in lens_l]
    max_pages = max(max(pages_per_req), 1)
    pt, num_pages = _page_table(B, pages_per_req, max_pages, page_order, g, device)
    num_pages = max(num_pages, 1)
    q = _randn_bf16((B, Hq, d), g, device)
    K = _randn_bf16((num_pages, P, Hkv, d), g, device)
    V = _randn_bf16((num_pages, P, Hkv, d), g, device)
    if k_max is None:
        k_max = max(1, max(min(kk, n) for kk, n in zip(k_l, lens_l)) if B else 1)
    w = Workload(name=name, B=B, Hq=Hq, Hkv=Hkv, d=d, P=P, max_pages=max_pages, num_pages=num_pages,
                 k_max=int(k_max), q=q, K=K, V=V, page_table=pt,
                 lens=torch.tensor(lens_l, dtype=torch.int32, device=device),
                 k=torch.tensor(k_l, dtype=torch.int32, device=device), meta={"seed": seed})
    if structure == "planted16":
        _plant_keys(w, g, per_head=16, scale=4.0)
    elif structure == "heavy1pct":
        _heavy_hitters(w, g, frac=0.01, shift=2.0)
    elif structure == "sinks3":
        _sinks(w, n_sinks=4, scale=3.0)
    elif structure is not None:
        raise ValueError(f"unknown structure {structure!r}")
    return w


def _plant_keys(w: Workload, g, per_head: int, scale: float):
    """Per query head h: `per_head` positions of KV head h//G (disjoint within the group) get
    K <- bf16(scale * q_h)."""
    planted = {}
    G = w.G
    for b in range(w.B):
        n = int(w.lens[b])
        for kvh in range(w.Hkv):
            perm = torch.randperm(n, generator=g, device=w.K.device)[: G * per_head]
            for gi in range(G):
                h = kvh * G + gi
                pos = perm[gi * per_head:(gi + 1) * per_head].sort().values
                pages, slots = rows_of(w.page_table, w.P, b, pos)
                w.K[pages, slots, kvh] = (scale * w.q[b, h].float()).to(torch.bfloat16)
                planted[(b, h)] = pos.cpu()
    w.meta["planted"] = planted


def _heavy_hitters(w: Workload, g, frac: float, shift: float):
    """Per (b, kv head): round(frac*N) positions get K <- bf16(K + shift * mean of the group's q)."""
    G = w.G
    hh = {}
    for b in range(w.B):
        n = int(w.lens[b])
        cnt = max(1, int(frac * n + 0.5))
        for kvh in range(w.Hkv):
            qbar = w.q[b, kvh * G:(kvh + 1) * G].float().mean(dim=0)
            pos = torch.randperm(n, generator=g, device=w.K.device)[:cnt].sort().values
            pages, slots = rows_of(w.page_table, w.P, b, pos)
            w.K[pages, slots, kvh] = (w.K[pages, slots, kvh].float() + shift * qbar).to(torch.bfloat16)
            hh[(b, kvh)] = pos.cpu()
    w.meta["heavy"] = hh


def _sinks(w: Workload, n_sinks: int, scale: float):
    """K rows at logical positions 0..n_sinks-1 of every (b, kv head) multiplied by `scale`."""
    for b in range(w.B):
        n = min(n_sinks, int(w.lens[b]))
        if n == 0:
            continue
        pos = torch.arange(n, device=w.K.device)
        pages, slots = rows_of(w.page_table, w.P, b, pos)
        w.K[pages, slots] = (w.K[pages, slots].float() * scale).to(torch.bfloat16)


def named(name: str, *, device="cpu", seed: int | None = None, ratio: int = 50, steps: int = 64) -> Workload:
    """The five named workloads; `ratio` picks the k of `sweep128k` (10, 50, 100 or 1 = dense)."""
    if seed is None:
        seed = 1234 + CONFIG_IDS[name]
    if name == "tiny":
        return make_workload(1, 8, 2, 4096, k_for_ratio(4096, 50), seed=seed, page_order="identity",
                             device=device, name=name, structure="planted16")
    if name == "llama8b":
        return make_workload(8, 32, 8, 32768, k_for_ratio(32768, 50), seed=seed, device=device, name=name,
                             structure="heavy1pct")
    if name == "long128k":
        return make_workload(4, 64, 8, 131072, k_for_ratio(131072, 50), seed=seed, device=device, name=name,
                             structure="sinks3")
    if name == "sweep128k":
        n = 131072
        w = make_workload(16, 32, 8, n, k_for_ratio(n, ratio), seed=seed, device=device, name=name)
        w.meta["ratio"] = ratio
        return w
    if name == "ragged":
        return ragged(device=device, seed=seed, steps=steps)
    raise KeyError(name)


def ragged(*, B: int = 32, Hq: int = 32, Hkv: int = 8, lo: int = 8192, hi: int = 163840, steps: int = 64,
           ratio: int = 50, seed: int = 1239, device="cpu", d: int = HEAD_DIM, P: int = PAGE_SIZE) -> Workload:
    """Ragged agentic batch.  Pages come from one shuffled free list: each request first takes the
    pages of its initial context, then during the `steps` appended decode steps a request takes the
    next free page whenever its length crosses a page boundary (len % P == 0).  The whole page
    table is planned here, so the per-step append only writes rows."""
    device = torch.device(device)
    g = _gen(device, seed)
    lens0 = torch.randint(lo, hi + 1, (B,), generator=g, device=device).tolist()
    final_pages = [(n + steps + P - 1) // P for n in lens0]
    total = sum(final_pages)
    free = torch.randperm(total, generator=g, device=device).to(torch.int32).tolist()
    max_pages = max(final_pages)
    pt = [[-1] * max_pages for _ in range(B)]
    nxt = 0
    for b, n in enumerate(lens0):
        for p in range((n + P - 1) // P):
            pt[b][p] = free[nxt]
            nxt += 1
    for t in range(steps):
        for b, n in enumerate(lens0):
            pos = n + t
            if pos % P == 0:
                pt[b][pos // P] = free[nxt]
                nxt += 1
    page_table = torch.tensor(pt, dtype=torch.int32, device=device)
    q = _randn_bf16((B, Hq, d), g, device)
    K = _randn_bf16((total, P, Hkv, d), g, device)
    V = _randn_bf16((total, P, Hkv, d), g, device)
    k = [k_for_ratio(n, ratio) for n in lens0]
    k_max = k_for_ratio(max(lens0) + steps, ratio)
    w = Workload(name="ragged", B=B, Hq=Hq, Hkv=Hkv, d=d, P=P, max_pages=max_pages, num_pages=total,
                 k_max=k_max, q=q, K=K, V=V, page_table=page_table,
                 lens=torch.tensor(lens0, dtype=torch.int32, device=device),
                 k=torch.tensor(k, dtype=torch.int32, device=device),
                 meta={"seed": seed, "steps": steps, "ratio": ratio})
    # Per-step fresh queries and the K/V rows each step appends.
    w.meta["q_steps"] = _randn_bf16((steps, B, Hq, d), g, device)
    w.meta["k_new"] = _randn_bf16((steps, B, Hkv, d), g, device)
    w.meta["v_new"] = _randn_bf16((steps, B, Hkv, d), g, device)
    return w
