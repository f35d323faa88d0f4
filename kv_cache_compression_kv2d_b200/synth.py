"""Seeded synthetic inputs shaped like long-context decode workloads.

This module holds no step of the compression method: it only draws keys,
values and queries.  Both the CUDA path and the CPU oracle are fed from it.

Distribution (one attention layer):
  * K, V ~ N(0, 1).
  * 4 outlier key channels per KV head, scaled x8 (the pages observe that
    large-magnitude outliers sit in a few channels: MosaicKV, Fig. 2 text,
    "Channel Compression").
  * mu_h ~ N(0, I_d) per KV head; window and decode queries are
    mu_h + N(0, I_d) for each of the G query heads of that KV head.
  * planted high-affinity tokens: k_t += 4 * mu_h / |mu_h| for a fraction of
    the tokens (uniform without replacement, or one per stratum).
  * optional segment classes (mix4) so that every strategy wins somewhere:
    3% dense-mass segments (half their tokens planted), 5% dense-mass
    segments whose keys keep their energy in c channels (the others x0.02),
    30% few-heavy segments (1..r planted) and 62% plain segments.
Everything is generated in fp32 with a seeded torch.Generator on the target
device and rounded to fp16 once.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Optional

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    num_kv_heads: int
    group: int              # query heads per KV head
    head_dim: int
    seq_len: int            # prompt length (max length for ragged batches)
    segment_len: int
    window: int
    budget: float
    keep_tokens: int = 0    # 0 -> S/8
    keep_channels: int = 0  # 0 -> d/4
    planted_frac: float = 0.01
    planted_layout: str = "uniform"     # "uniform" | "stratified"
    segment_mix: bool = False           # mix4 segment classes
    ragged_min: int = 0                 # >0: lengths uniform in [ragged_min, seq_len]
    block_size: int = 0                 # >0: paged dense view
    decode_steps: int = 0
    recompress_every: int = 0
    outliers: int = 4
    outlier_scale: float = 8.0
    planted_gain: float = 4.0

    @property
    def num_q_heads(self) -> int:
        return self.num_kv_heads * self.group

    @property
    def r(self) -> int:
        return self.keep_tokens or max(1, self.segment_len // 8)

    @property
    def c(self) -> int:
        return self.keep_channels or max(1, self.head_dim // 4)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    # 1 layer, 1 KV head, GQA 4, d=128, 2048 tokens, S=64, W=32, budget 25%.
    "tiny": Workload("tiny", 1, 1, 4, 128, 2048, 64, 32, 0.25),
    # Llama-3-8B-shaped layer: 32 q / 8 KV heads, batch 1, 32K context.
    "llama3_8b_32k": Workload("llama3_8b_32k", 1, 8, 4, 128, 32768, 64, 64, 0.20),
    # same layer, batch 16 x 128K, budget 15%, all four strategies, 256 steps.
    "llama3_8b_b16_128k_mix": Workload("llama3_8b_b16_128k_mix", 16, 8, 4, 128, 131072, 64, 64,
                                       0.15, segment_mix=True, decode_steps=256),
    # the same batch at 16K tokens per sequence (1.1 GB dense K/V, 160 MB
    # packed): a size that a full hardware-counter capture of decode can hold
    "llama3_8b_b16_16k_mix": Workload("llama3_8b_b16_16k_mix", 16, 8, 4, 128, 16384, 64, 64,
                                      0.15, segment_mix=True),
    # same layer, batch 1, 1M tokens, S=W=128, budget 10%, 0.1% planted.
    "llama3_8b_1m": Workload("llama3_8b_1m", 1, 8, 4, 128, 1 << 20, 128, 128, 0.10,
                             planted_frac=0.001, planted_layout="stratified"),
    # ragged batch of 32 in [4K, 128K], paged 16-token blocks, re-compress
    # the trailing region every 128 decode steps.
    "ragged32_paged": Workload("ragged32_paged", 32, 8, 4, 128, 131072, 64, 64, 0.20,
                               ragged_min=4096, block_size=16, decode_steps=512,
                               recompress_every=128),
}


@dataclass
class Batch:
    wl: Workload
    seq_len: torch.Tensor            # [B] int32 (host)
    k: torch.Tensor                  # contiguous [B][Hkv][cap][d] or paged pool
    v: torch.Tensor
    qw: torch.Tensor                 # [B][Hq][W][d] fp16
    q: torch.Tensor                  # [B][Hq][d] fp16
    capacity: int                    # tokens per sequence the dense view holds
    block_table: Optional[torch.Tensor] = None   # [B][max_blocks] int32 (paged)
    mu: Optional[torch.Tensor] = None
    extra: dict = field(default_factory=dict)


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _normal(shape, g, device):
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32)


def lengths(wl: Workload, seed: int = 0) -> torch.Tensor:
    if wl.ragged_min > 0:
        g = _gen("cpu", seed + 7919)
        return torch.randint(wl.ragged_min, wl.seq_len + 1, (wl.batch,), generator=g,
                             dtype=torch.int64).to(torch.int32)
    return torch.full((wl.batch,), wl.seq_len, dtype=torch.int32)


def _keys_for_sequence(wl, T, mu_dir, outl, g, device, b):
    """K rows [Hkv][T][d] in fp32 for one sequence."""
    H, d = wl.num_kv_heads, wl.head_dim
    k = _normal((H, T, d), g, device)
    for h in range(H):
        k[h][:, outl[h]] *= wl.outlier_scale
    n_pl = int(round(wl.planted_frac * T))
    if wl.segment_mix:
        S = wl.segment_len
        nseg = T // S
        # class per (h, j): 0 dense-mass (half the tokens planted), 1 dense-mass
        # with every key's energy in c channels, 2 few-heavy (1..r planted),
        # 3 plain.  3% / 5% / 30% / 62%.
        u = torch.rand((H, max(nseg, 1)), generator=g, device=device)
        cls = torch.full_like(u, 3, dtype=torch.int64)
        cls[u < 0.38] = 2
        cls[u < 0.08] = 1
        cls[u < 0.03] = 0
        ar = torch.arange(S, device=device)
        for h in range(H):
            segs = torch.nonzero(cls[h, :nseg] == 2).flatten()
            if segs.numel():
                cnt = torch.randint(1, wl.r + 1, (segs.numel(),), generator=g, device=device)
                off = torch.rand((segs.numel(), S), generator=g, device=device).argsort(dim=1)
                pos = (segs[:, None] * S + off)[ar[None, :] < cnt[:, None]]
                k[h, pos] += wl.planted_gain * mu_dir[h]
            segs = torch.nonzero(cls[h, :nseg] == 0).flatten()
            if segs.numel():
                off = torch.rand((segs.numel(), S), generator=g, device=device).argsort(dim=1)
                pos = (segs[:, None] * S + off[:, : S // 2]).flatten()
                k[h, pos] += wl.planted_gain * mu_dir[h]
            segs = torch.nonzero(cls[h, :nseg] == 1).flatten()
            if segs.numel():
                n1 = segs.numel()
                ch = torch.rand((n1, d), generator=g, device=device).argsort(dim=1)[:, : wl.c]
                mask = torch.zeros((n1, d), device=device)
                mask.scatter_(1, ch, 1.0)
                rows = segs[:, None] * S + ar[None, :]                     # [n1][S]
                k[h, rows] = k[h, rows] * (0.02 + 0.98 * mask)[:, None, :]
                dirc = mu_dir[h][None, :] * mask
                dirc = dirc / dirc.norm(dim=1, keepdim=True)
                off = torch.rand((n1, S), generator=g, device=device).argsort(dim=1)[:, : S // 2]
                pos = segs[:, None] * S + off                               # [n1][S/2]
                k[h, pos] += 2.0 * wl.planted_gain * dirc[:, None, :]
    if n_pl > 0 and not wl.segment_mix:
        for h in range(H):
            if wl.planted_layout == "stratified":
                stride = T / n_pl
                base = (torch.arange(n_pl, device=device, dtype=torch.float64) * stride)
                jit = torch.rand((n_pl,), generator=g, device=device, dtype=torch.float64) * stride
                pos = (base + jit).long().clamp_(0, T - 1)
            else:
                pos = torch.randperm(T, generator=g, device=device)[:n_pl]
            k[h, pos] += wl.planted_gain * mu_dir[h]
    return k


def generate(wl: Workload, seed: int = 0, device="cpu", extra_capacity: int = 0,
             seq_lens: Optional[torch.Tensor] = None) -> Batch:
    """Draws one layer's dense K/V view, window queries and decode queries.

    extra_capacity: room for tokens appended during decode.
    """
    device = torch.device(device)
    g = _gen(device, seed)
    H, G, d = wl.num_kv_heads, wl.group, wl.head_dim
    B = wl.batch
    lens = seq_lens if seq_lens is not None else lengths(wl, seed)
    Tmax = int(lens.max())
    cap = Tmax + extra_capacity
    mu = _normal((H, d), g, device)
    mu_dir = mu / mu.norm(dim=1, keepdim=True)
    outl = [torch.randperm(d, generator=g, device=device)[: wl.outliers] for _ in range(H)]

    paged = wl.block_size > 0
    if paged:
        bs = wl.block_size
        nblk = [int(math.ceil((int(lens[b]) + extra_capacity) / bs)) for b in range(B)]
        total = sum(nblk)
        perm = torch.randperm(total, generator=g, device=device).to(torch.int32)
        maxb = max(nblk)
        table = torch.full((B, maxb), -1, dtype=torch.int32, device=device)
        kpool = torch.zeros((total, H, bs, d), dtype=torch.float16, device=device)
        vpool = torch.zeros((total, H, bs, d), dtype=torch.float16, device=device)
        cur = 0
        for b in range(B):
            table[b, : nblk[b]] = perm[cur: cur + nblk[b]]
            cur += nblk[b]
    else:
        kc = torch.zeros((B, H, cap, d), dtype=torch.float16, device=device)
        vc = torch.zeros((B, H, cap, d), dtype=torch.float16, device=device)

    for b in range(B):
        T = int(lens[b])
        kb = _keys_for_sequence(wl, T, mu_dir, outl, g, device, b).to(torch.float16)
        vb = _normal((H, T, d), g, device).to(torch.float16)
        if paged:
            bs = wl.block_size
            nb_used = int(math.ceil(T / bs))
            pad = nb_used * bs - T
            if pad:
                kb = torch.cat([kb, torch.zeros((H, pad, d), dtype=kb.dtype, device=device)], 1)
                vb = torch.cat([vb, torch.zeros((H, pad, d), dtype=vb.dtype, device=device)], 1)
            phys = table[b, :nb_used].long()
            kpool[phys] = kb.view(H, nb_used, bs, d).transpose(0, 1)
            vpool[phys] = vb.view(H, nb_used, bs, d).transpose(0, 1)
        else:
            kc[b, :, :T] = kb
            vc[b, :, :T] = vb
        del kb, vb

    mu_q = mu.repeat_interleave(G, dim=0)                       # [Hq][d]
    qw = (mu_q[None, :, None, :] + _normal((B, H * G, wl.window, d), g, device)).to(torch.float16)
    q = (mu_q[None, :, :] + _normal((B, H * G, d), g, device)).to(torch.float16)
    if paged:
        return Batch(wl, lens, kpool, vpool, qw, q, cap, block_table=table, mu=mu)
    return Batch(wl, lens, kc, vc, qw, q, cap, mu=mu)


def decode_tokens(wl: Workload, step: int, seed: int = 0, device="cpu", mu=None):
    """New (k, v, q) for one decode step: k, v ~ N(0,1) [B][Hkv][d];
    q = mu_h + N(0, I) [B][Hq][d]."""
    device = torch.device(device)
    g = _gen(device, seed * 1000003 + 17 + step)
    B, H, G, d = wl.batch, wl.num_kv_heads, wl.group, wl.head_dim
    k = _normal((B, H, d), g, device).to(torch.float16)
    v = _normal((B, H, d), g, device).to(torch.float16)
    base = torch.zeros((H, d), device=device) if mu is None else mu.to(device)
    q = (base.repeat_interleave(G, dim=0)[None] + _normal((B, H * G, d), g, device)).to(torch.float16)
    return k, v, q


def dense_rows(batch: Batch, b: int, h: int, t0: int, t1: int):
    """Rows [t0, t1) of (b, h) of the dense view, as fp16 tensors [n][d]
    (reads either layout; used to hand the same inputs to the oracle)."""
    if batch.block_table is None:
        return batch.k[b, h, t0:t1], batch.v[b, h, t0:t1]
    bs = batch.wl.block_size
    ks, vs = [], []
    t = t0
    while t < t1:
        blk = t // bs
        off = t % bs
        n = min(bs - off, t1 - t)
        phys = int(batch.block_table[b, blk])
        ks.append(batch.k[phys, h, off: off + n])
        vs.append(batch.v[phys, h, off: off + n])
        t += n
    if not ks:
        d = batch.wl.head_dim
        z = torch.zeros((0, d), dtype=torch.float16, device=batch.k.device)
        return z, z
    return torch.cat(ks), torch.cat(vs)
