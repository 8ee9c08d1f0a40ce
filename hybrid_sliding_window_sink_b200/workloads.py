"""Seeded synthetic inputs and workload shapes.

This module draws random numbers and describes shapes; it holds none of the
attention arithmetic. Tests, the smoke check and the benchmark use it to build
the same inputs for the CUDA library and for the CPU oracle (which receives the
exact bf16 values, upcast).

Shapes follow the MiMo-V2 layer configuration ("39层滑窗+9层全局注意力 ...
MiMo-V2.6-Flash-MOPD", §3-§5): SWA layers 64 Q / 8 KV heads with window 128 and
RoPE base 1e4; GA layers 64 Q / 4 KV heads with RoPE base 1e7; QK head dim 192,
V head dim 128, RoPE on the first 64 dims. The token-level sparse workload
follows "小米MiMo-V3的核心架构HySparse2" §四.3 (recent 128 + 1,024 selected).
Values are N(0, 1) drawn in fp32 and cast to bf16; sinks are fp32 N(0, 1).
"""

from __future__ import annotations

from dataclasses import dataclass

import torch

DQK = 192
DV = 128
ROT_DIMS = 64
SWA_WINDOW = 128
SWA_THETA = 1.0e4
GA_THETA = 1.0e7

#: GA layer indices of the 48-layer hybrid stack (0 = GA, the rest SWA):
#: 9 GA + 39 SWA layers, pwwt.cn page §2.
GA_LAYERS = (0, 6, 12, 18, 24, 30, 36, 42, 47)
NUM_LAYERS = 48


def layer_pattern() -> list[int]:
    """hybrid_layer_pattern: 1 = SWA, 0 = GA, one entry per layer."""
    return [0 if l in GA_LAYERS else 1 for l in range(NUM_LAYERS)]


@dataclass(frozen=True)
class PrefillCase:
    name: str
    batch: int
    seqlen: int
    hq: int
    hkv: int
    window: int          # <= 0: full causal (GA)
    theta: float
    k_scale: float = 1.0
    seed: int = 0


@dataclass(frozen=True)
class DecodeCase:
    name: str
    batch: int
    hq: int
    hkv: int
    kind: str            # "ring" | "linear"
    capacity: int
    min_len: int
    max_len: int
    seed: int = 0


@dataclass(frozen=True)
class SparseCase:
    name: str
    batch: int
    context: int
    hq: int
    hkv: int
    recent: int
    n_sel: int
    seed: int = 0


#: The five workloads the library is measured and checked on.
TINY_SWA_PREFILL = PrefillCase("tiny SWA+sink prefill n=1024 8Q/1KV W=128", 1, 1024, 8, 1,
                               SWA_WINDOW, SWA_THETA, seed=1001)
SWA_PREFILL = PrefillCase("SWA layer prefill n=32768 64Q/8KV W=128", 1, 32768, 64, 8,
                          SWA_WINDOW, SWA_THETA, seed=1002)
GA_PREFILL = PrefillCase("GA layer prefill n=32768 causal 64Q/4KV", 1, 32768, 64, 4,
                         0, GA_THETA, k_scale=0.5, seed=1003)
HYBRID_DECODE_SWA = DecodeCase("hybrid decode SWA layer B=64 ring128 64Q/8KV", 64, 64, 8,
                               "ring", SWA_WINDOW, 4096, 131072, seed=1004)
HYBRID_DECODE_GA = DecodeCase("hybrid decode GA layer B=64 linear 64Q/4KV", 64, 64, 4,
                              "linear", 131072, 4096, 131072, seed=1004)
SPARSE_DECODE = SparseCase("token-sparse decode B=8 L=262144 64Q/4KV 128+1024", 8, 262144,
                           64, 4, 128, 1024, seed=1005)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _randn_bf16(shape, g, device, scale=1.0):
    x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if scale != 1.0:
        x.mul_(scale)
    return x.to(torch.bfloat16)


def prefill_inputs(batch, seqlen, hq, hkv, *, seed, device="cpu", k_scale=1.0,
                   dqk=DQK, dv=DV, with_sink=True):
    """q [B,n,Hq,dqk], k [B,n,Hkv,dqk], v [B,n,Hkv,dv] bf16; sink [Hq] fp32.
    Draw order: Q, K, V, sink."""
    g = _gen(seed, device)
    q = _randn_bf16((batch, seqlen, hq, dqk), g, device)
    k = _randn_bf16((batch, seqlen, hkv, dqk), g, device, k_scale)
    v = _randn_bf16((batch, seqlen, hkv, dv), g, device)
    sink = torch.randn(hq, generator=g, device=device, dtype=torch.float32)
    return {"q": q, "k": k, "v": v, "sink": sink if with_sink else None}


def case_prefill_inputs(case: PrefillCase, device="cpu"):
    return prefill_inputs(case.batch, case.seqlen, case.hq, case.hkv, seed=case.seed,
                          device=device, k_scale=case.k_scale)


def lengths_uniform(batch, lo, hi, *, seed, device="cpu"):
    """Per-sequence context lengths, integers uniform in [lo, hi]."""
    g = _gen(seed + 7, "cpu")
    L = torch.randint(lo, hi + 1, (batch,), generator=g, dtype=torch.int32)
    return L.to(device)


def decode_inputs(batch, hq, hkv, capacity, lengths, *, seed, device="cpu",
                  dqk=DQK, dv=DV, seq_stride=None):
    """q [B,Hq,dqk]; k_cache [B,stride,Hkv,dqk]; v_cache [B,stride,Hkv,dv] bf16;
    sink [Hq] fp32. ``lengths`` is stored as int32. Draw order: Q, K, V, sink."""
    stride = capacity if seq_stride is None else seq_stride
    g = _gen(seed, device)
    q = _randn_bf16((batch, hq, dqk), g, device)
    kc = _randn_bf16((batch, stride, hkv, dqk), g, device)
    vc = _randn_bf16((batch, stride, hkv, dv), g, device)
    sink = torch.randn(hq, generator=g, device=device, dtype=torch.float32)
    return {"q": q, "k_cache": kc, "v_cache": vc, "sink": sink,
            "lengths": torch.as_tensor(lengths, dtype=torch.int32).to(device)}


def decode_mq_inputs(batch, q_len, hq, hkv, capacity, lengths, *, seed, device="cpu",
                     dqk=DQK, dv=DV):
    """Multi-query decode inputs: those of decode_inputs (same draws) plus
    ``q_mq`` [B, q_len, Hq, dqk] bf16 for the q_len newest tokens, drawn after them."""
    inp = decode_inputs(batch, hq, hkv, capacity, lengths, seed=seed, device=device, dqk=dqk, dv=dv)
    g = _gen(seed + 29, device)
    inp["q_mq"] = _randn_bf16((batch, q_len, hq, dqk), g, device)
    return inp


def fp8_cache(x):
    """Quantizes a bf16/fp32 cache [B, S, Hkv, D] to E4M3 bytes with one fp32 scale per
    (token, KV head) row (amax / 448, 1 for an all-zero row), the way a serving stack would
    write it. Returns (bytes uint8 [B, S, Hkv, D], scale fp32 [B, S, Hkv])."""
    xf = x.float()
    amax = xf.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    q = (xf / scale[..., None]).to(torch.float8_e4m3fn)
    return q.view(torch.uint8), scale.contiguous()


def decode_fp8_inputs(batch, hq, hkv, capacity, lengths, *, seed, device="cpu"):
    """decode_inputs (same draws) plus k8/v8 E4M3 caches and k_scale/v_scale from fp8_cache."""
    inp = decode_inputs(batch, hq, hkv, capacity, lengths, seed=seed, device=device)
    inp["k8"], inp["k_scale"] = fp8_cache(inp["k_cache"])
    inp["v8"], inp["v_scale"] = fp8_cache(inp["v_cache"])
    return inp


def integer_qk(batch, hq, hkv, capacity, *, seed, device="cpu", lo=-2, hi=2):
    """q [B,Hq,192] and k_cache [B,cap,Hkv,192] bf16 with integer entries uniform in [lo, hi]:
    every dot product is an integer, exact in fp32 and float64 alike (ties included).
    Drawn on ``device`` (a CUDA device avoids a host copy of a large cache)."""
    g = _gen(seed + 17, device)
    q = torch.randint(lo, hi + 1, (batch, hq, DQK), generator=g, device=device).to(torch.bfloat16)
    k = torch.randint(lo, hi + 1, (batch, capacity, hkv, DQK), generator=g,
                      device=device, dtype=torch.int8).to(torch.bfloat16)
    return q, k


def random_e4m3(shape, g, device):
    """Uniformly random E4M3 bytes with the two NaN patterns replaced by 0 (a cache holds
    no NaN), drawn with generator ``g`` on ``device``."""
    b = torch.randint(0, 256, shape, generator=g, device=device, dtype=torch.uint8)
    return b.masked_fill_((b & 0x7F) == 0x7F, 0)


def random_fp8_cache(batch, capacity, hkv, *, seed, device="cpu", scale_lo=0.002, scale_hi=0.01):
    """An FP8 KV cache drawn directly as bytes (no bf16 source): k8 [B,cap,Hkv,192] and
    v8 [B,cap,Hkv,128] random E4M3 bytes, k_scale / v_scale [B,cap,Hkv] fp32 uniform in
    [scale_lo, scale_hi]. Draw order: k8, v8, k_scale, v_scale."""
    g = _gen(seed, device)
    k8 = random_e4m3((batch, capacity, hkv, DQK), g, device)
    v8 = random_e4m3((batch, capacity, hkv, DV), g, device)
    ks = torch.empty(batch, capacity, hkv, device=device).uniform_(scale_lo, scale_hi, generator=g)
    vs = torch.empty(batch, capacity, hkv, device=device).uniform_(scale_lo, scale_hi, generator=g)
    return k8, v8, ks, vs


def sorted_unique_indices(batch, hkv, n_sel, hi_excl, *, seed):
    """[B, Hkv, n_sel] int32, each row sorted unique uniform in [0, hi_excl[b])."""
    g = _gen(seed + 13, "cpu")
    out = torch.empty(batch, hkv, n_sel, dtype=torch.int32)
    for b in range(batch):
        hi = int(hi_excl[b]) if hasattr(hi_excl, "__len__") else int(hi_excl)
        if hi < n_sel:
            raise ValueError("not enough tokens outside the recent window")
        for h in range(hkv):
            if hi > 8 * n_sel:
                # rejection-free draw for a large range: oversample then dedup
                while True:
                    c = torch.randint(0, hi, (n_sel * 2,), generator=g)
                    u = torch.unique(c)
                    if u.numel() >= n_sel:
                        perm = torch.randperm(u.numel(), generator=g)[:n_sel]
                        out[b, h] = torch.sort(u[perm]).values.to(torch.int32)
                        break
            else:
                perm = torch.randperm(hi, generator=g)[:n_sel]
                out[b, h] = torch.sort(perm).values.to(torch.int32)
    return out


def to_f64(t):
    """Exact float64 numpy copy of a (bf16 or fp32) tensor."""
    import numpy as np
    return t.detach().to("cpu", torch.float64).numpy().astype(np.float64, copy=False)
