"""Seeded synthetic inputs for query-aware block-sparse attention.

This module only draws inputs: random normals, rotary position embedding applied to the
draws (the method itself takes already-rotated q and k), planted "needle" blocks, active
masks and cached outputs.  It contains none of the method's arithmetic (no summaries,
scores, selection or attention) and is the one module that both the CUDA library's tests
and the oracle's tests draw their inputs from.

Recipes (the shapes are those of the five workloads the pages motivate):

* q, k, v ~ N(0, 1) drawn in fp32 from ``torch.Generator().manual_seed(seed)``;
* rotary embedding in fp64, rotate-half pairing (j, j + D/2), frequency
  theta^(-2j/D), angle = position * frequency; key t sits at position t; a decode query
  at position T_b - 1 (the cache already holds the current token); a block-query token i
  at T_prefix + i; a prefill token i at i;
* needle blocks (decode): u_g = unit vector of the mean of group g's rotated query heads;
  every key of a needle block is sqrt(D) * u_g + 0.5 * N(0, I) (so |key| ~ |N(0,1) key|);
  needle blocks are distinct, uniform over the non-forced blocks, independent per (b, g);
  they are planted after the rotation; v is left N(0, 1);
* LoSA steps: the previous step's queries are the current ones plus 0.02 * N(0, I) for a
  stable token and a fresh rotated N(0, 1) draw for an active one; the block's own keys
  and values sit at cache rows T_prefix .. T_prefix + Tq - 1;
* the result is rounded once (round-to-nearest-even) to the case dtype;
* optional poison: cache positions at or beyond a sequence's length are filled with NaN,
  so that any kernel that lets them into a result is caught.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

BLK = 64


def _gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def rope(x: torch.Tensor, pos: torch.Tensor, theta: float) -> torch.Tensor:
    """Rotate-half rotary embedding in fp64.  x [..., T, D]; pos [T] (or broadcastable)."""
    D = x.shape[-1]
    half = D // 2
    j = torch.arange(half, dtype=torch.float64, device=x.device)
    freq = theta ** (-2.0 * j / D)
    ang = pos.to(torch.float64).unsqueeze(-1) * freq  # [T, half]
    c, s = torch.cos(ang), torch.sin(ang)
    x = x.to(torch.float64)
    x1, x2 = x[..., :half], x[..., half:]
    return torch.cat([x1 * c - x2 * s, x1 * s + x2 * c], dim=-1)


@dataclass
class DecodeCase:
    q: torch.Tensor          # [B, Hq, D]
    k: torch.Tensor          # [B, Hkv, T_cap, D]
    v: torch.Tensor          # [B, Hkv, T_cap, D]
    seqlens: torch.Tensor    # [B] int32
    topk: int
    n_sink: int
    n_local: int
    blk: int = BLK
    needles: list = field(default_factory=list)  # [(b, g, [blocks])]

    @property
    def shape(self):
        B, Hkv, T_cap, D = self.k.shape
        return B, Hkv, self.q.shape[1] // Hkv, D, T_cap


def decode_case(B, Hkv, G, D, T_cap, seqlens, dtype, topk, n_sink, n_local, n_needles=0,
                theta=1e4, seed=0, poison_tail=False, device="cpu") -> DecodeCase:
    """Draw one decode batch.  seqlens: int, list or tensor of per-sequence lengths."""
    if isinstance(seqlens, int):
        seqlens = [seqlens] * B
    sl = torch.as_tensor(seqlens, dtype=torch.int32)
    assert sl.numel() == B and int(sl.max()) <= T_cap
    gen = _gen(seed, device)
    Hq = Hkv * G
    q = torch.randn(B, Hq, D, generator=gen, device=device)
    k = torch.empty(B, Hkv, T_cap, D, dtype=dtype, device=device)
    v = torch.empty(B, Hkv, T_cap, D, dtype=dtype, device=device)
    pos_k = torch.arange(T_cap, device=device)
    qr = torch.empty(B, Hq, D, dtype=torch.float64, device=device)
    for b in range(B):  # one sequence at a time keeps the fp64 temporaries small
        kb = torch.randn(Hkv, T_cap, D, generator=gen, device=device)
        k[b] = rope(kb, pos_k, theta).to(dtype)
        del kb
        v[b] = torch.randn(Hkv, T_cap, D, generator=gen, device=device).to(dtype)
        qpos = torch.full((1,), int(sl[b]) - 1, device=device)
        qr[b] = rope(q[b].unsqueeze(-2), qpos, theta).squeeze(-2)
    needles = []
    if n_needles > 0:
        for b in range(B):
            T = int(sl[b])
            NB = -(-T // BLK)
            forced = set(range(min(n_sink, NB))) | set(range(max(0, NB - n_local), NB))
            # the needle block must be full-length so every key is a needle key
            free = [j for j in range(NB) if j not in forced and (j + 1) * BLK <= T]
            for g in range(Hkv):
                u = qr[b, g * G:(g + 1) * G].mean(dim=0)
                u = u / u.norm()
                perm = torch.randperm(len(free), generator=gen, device=device)[:n_needles]
                blocks = sorted(free[int(i)] for i in perm)
                for j in blocks:
                    eps = torch.randn(BLK, D, generator=gen, device=device).to(torch.float64)
                    key = math.sqrt(D) * u.unsqueeze(0) + 0.5 * eps
                    k[b, g, j * BLK:(j + 1) * BLK] = key.to(dtype)
                needles.append((b, g, blocks))
    if poison_tail:
        for b in range(B):
            T = int(sl[b])
            k[b, :, T:] = float("nan")
            v[b, :, T:] = float("nan")
    return DecodeCase(q=qr.to(dtype), k=k, v=v, seqlens=sl.to(device), topk=topk,
                      n_sink=n_sink, n_local=n_local, needles=needles)


# ---- the five workloads -------------------------------------------------------------

def tiny_decode(seed=1001, device="cpu") -> DecodeCase:
    """Tiny fp32 decode: 1 x (1 KV head, 4 q heads), D 64, 2048 tokens, top-8 incl. block 0
    and the last 2 blocks, RoPE theta 1e4, one query token."""
    return decode_case(B=1, Hkv=1, G=4, D=64, T_cap=2048, seqlens=2048, dtype=torch.float32,
                       topk=8, n_sink=1, n_local=2, n_needles=0, theta=1e4, seed=seed,
                       device=device)


def gqa_decode_64k(seed=1002, device="cpu", n_needles=16) -> DecodeCase:
    """64K-context GQA decode, bf16: 8 KV heads x 8 q heads, D 128, top-16 (block 0 and the
    last 2 blocks forced) shared per group, 16 needle blocks per group."""
    return decode_case(B=1, Hkv=8, G=8, D=128, T_cap=65536, seqlens=65536,
                       dtype=torch.bfloat16, topk=16, n_sink=1, n_local=2,
                       n_needles=n_needles, theta=1e4, seed=seed, device=device)


def batched_decode(seed=1003, device="cpu", B=16, T_lo=8192, T_hi=32768,
                   poison_tail=False) -> DecodeCase:
    """Batched varlen decode, bf16: 16 sequences with lengths uniform in [8192, 32768],
    8 KV heads x 4 q heads, D 128, top-16 with sink + 2 local, 8 needles per (b, g)."""
    gen = _gen(seed + 7919)
    sl = torch.randint(T_lo, T_hi + 1, (B,), generator=gen, dtype=torch.int64).to(torch.int32)
    return decode_case(B=B, Hkv=8, G=4, D=128, T_cap=T_hi, seqlens=sl, dtype=torch.bfloat16,
                       topk=16, n_sink=1, n_local=2, n_needles=8, theta=1e4, seed=seed,
                       poison_tail=poison_tail, device=device)


@dataclass
class BlockQueryCase:
    q: torch.Tensor          # [B, Hq, Tq, D]
    k: torch.Tensor          # [B, Hkv, T_cap, D]
    v: torch.Tensor
    active: torch.Tensor     # [B, Tq] uint8
    o_cache: torch.Tensor    # [B, Hq, Tq, D]
    lse_cache: torch.Tensor  # [B, Hq, Tq] fp32
    T_prefix: int
    topk: int
    n_sink: int = 0
    n_local: int = 0
    blk: int = BLK


def blockquery_case(B=1, Hkv=8, G=4, D=128, Tq=32, T_prefix=32768, T_cap=None, n_active=8,
                    topk=8, n_sink=0, n_local=0, dtype=torch.bfloat16, theta=1e4, seed=1004,
                    device="cpu", same_query=False) -> BlockQueryCase:
    """Diffusion-LM block-query step: Tq query tokens, n_active of them active (seeded
    choice per sequence), prefix of T_prefix cached tokens; o_cache ~ N(0,1),
    lse_cache ~ N(0,1) + 10.  same_query=True gives every token the same query."""
    T_cap = T_cap or T_prefix
    gen = _gen(seed, device)
    Hq = Hkv * G
    if same_query:
        q = torch.randn(B, Hq, 1, D, generator=gen, device=device).expand(B, Hq, Tq, D)
    else:
        q = torch.randn(B, Hq, Tq, D, generator=gen, device=device)
    q = rope(q, torch.arange(T_prefix, T_prefix + Tq, device=device), theta)
    if same_query:  # identical after rotation too
        q = q[:, :, :1].expand(B, Hq, Tq, D)
    k = torch.empty(B, Hkv, T_cap, D, dtype=dtype, device=device)
    v = torch.empty(B, Hkv, T_cap, D, dtype=dtype, device=device)
    pos = torch.arange(T_cap, device=device)
    for b in range(B):
        k[b] = rope(torch.randn(Hkv, T_cap, D, generator=gen, device=device), pos,
                    theta).to(dtype)
        v[b] = torch.randn(Hkv, T_cap, D, generator=gen, device=device).to(dtype)
    active = torch.zeros(B, Tq, dtype=torch.uint8, device=device)
    for b in range(B):
        pick = torch.randperm(Tq, generator=gen, device=device)[:n_active]
        active[b, pick] = 1
    o_cache = torch.randn(B, Hq, Tq, D, generator=gen, device=device).to(dtype)
    lse_cache = torch.randn(B, Hq, Tq, generator=gen, device=device) + 10.0
    return BlockQueryCase(q=q.to(dtype).contiguous(), k=k, v=v, active=active,
                          o_cache=o_cache, lse_cache=lse_cache.float(), T_prefix=T_prefix,
                          topk=topk, n_sink=n_sink, n_local=n_local)


def diffusion_blockquery(seed=1004, device="cpu") -> BlockQueryCase:
    """32 query tokens per block, 8 KV heads x 4 q heads, D 128, prefix 32768, per-token
    top-8 blocks of 64, 25% (8 of 32) tokens active."""
    return blockquery_case(seed=seed, device=device)


@dataclass
class LosaCase(BlockQueryCase):
    q_prev: torch.Tensor = None  # [B, Hq, Tq, D]: the block's queries one denoising step earlier


def losa_case(B=1, Hkv=8, G=4, D=128, Tq=32, T_prefix=32768, n_active=8, topk=8, n_sink=0,
              n_local=0, dtype=torch.bfloat16, theta=1e4, stable_noise=0.02, seed=1006,
              device="cpu") -> LosaCase:
    """A LoSA denoising step: the block-query case with the block's own keys and values at
    cache rows T_prefix .. T_prefix + Tq - 1 (T_cap = T_prefix + Tq), plus the previous
    step's queries.  A stable token's previous query is its query plus
    stable_noise * N(0, I); an active token's is an independent rotated N(0, 1) draw, so
    that the change separates the two kinds (expected squared change per element
    stable_noise^2 against 2).  `active` is the planted set."""
    c = blockquery_case(B=B, Hkv=Hkv, G=G, D=D, Tq=Tq, T_prefix=T_prefix, T_cap=T_prefix + Tq,
                        n_active=n_active, topk=topk, n_sink=n_sink, n_local=n_local,
                        dtype=dtype, theta=theta, seed=seed, device=device)
    gen = _gen(seed + 7919, device)
    Hq = Hkv * G
    fresh = rope(torch.randn(B, Hq, Tq, D, generator=gen, device=device),
                 torch.arange(T_prefix, T_prefix + Tq, device=device), theta).float()
    near = c.q.float() + stable_noise * torch.randn(B, Hq, Tq, D, generator=gen, device=device)
    on = c.active.bool()[:, None, :, None]
    q_prev = torch.where(on, fresh, near).to(dtype).contiguous()
    return LosaCase(q=c.q, k=c.k, v=c.v, active=c.active, o_cache=c.o_cache,
                    lse_cache=c.lse_cache, T_prefix=c.T_prefix, topk=c.topk, n_sink=c.n_sink,
                    n_local=c.n_local, q_prev=q_prev)


def diffusion_losa_step(seed=1006, device="cpu") -> LosaCase:
    """The diffusion block-query workload as a whole LoSA step: 32 query tokens (8 of them
    changing), 8 KV heads x 4 q heads, D 128, prefix 32768, per-token top-8 blocks."""
    return losa_case(seed=seed, device=device)


@dataclass
class PrefillCase:
    q: torch.Tensor  # [B, Hq, L, D]
    k: torch.Tensor  # [B, Hkv, L, D]
    v: torch.Tensor
    lam: float


def prefill_case(B=1, Hq=32, Hkv=8, L=32768, D=128, lam=1e-3, dtype=torch.bfloat16,
                 theta=1e4, q_scale=1.0, sink=0.0, sink_tokens=64, seed=1005,
                 device="cpu") -> PrefillCase:
    """Causal prefill: q, k, v ~ N(0,1) with rotary embedding; q_scale multiplies q after
    the rotation (a larger q sharpens the softmax).  sink > 0 plants an attention sink:
    a common unit direction u gets weight sqrt(sink * sqrt(D)) in every query and in the
    keys of the first sink_tokens positions, which raises those logits by ~sink, so that
    later tiles whose logits trail by more than -ln(lambda) become negligible."""
    gen = _gen(seed, device)
    pos = torch.arange(L, device=device)
    u = None
    if sink > 0:
        u = torch.randn(D, generator=gen, device=device, dtype=torch.float32).double()
        u = u / u.norm() * math.sqrt(sink * math.sqrt(D))
    q = torch.empty(B, Hq, L, D, dtype=dtype, device=device)
    k = torch.empty(B, Hkv, L, D, dtype=dtype, device=device)
    v = torch.empty(B, Hkv, L, D, dtype=dtype, device=device)
    for b in range(B):
        for h in range(Hq):
            qh = rope(torch.randn(L, D, generator=gen, device=device), pos, theta) * q_scale
            if u is not None:
                qh = qh + u
            q[b, h] = qh.to(dtype)
        for h in range(Hkv):
            kh = rope(torch.randn(L, D, generator=gen, device=device), pos, theta)
            if u is not None:
                kh[:sink_tokens] += u
            k[b, h] = kh.to(dtype)
            v[b, h] = torch.randn(L, D, generator=gen, device=device).to(dtype)
    return PrefillCase(q=q, k=k, v=v, lam=lam)


def blasst_prefill_32k(seed=1005, device="cpu") -> PrefillCase:
    """Causal prefill, bf16: 32 q heads / 8 KV heads, D 128, L 32768, lambda 1e-3."""
    return prefill_case(seed=seed, device=device)
