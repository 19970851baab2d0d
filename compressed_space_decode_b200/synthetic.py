"""Seeded synthetic inputs for the IsoQuant compressed-space attention path.

This module only draws random numbers; it holds none of the method's
arithmetic and imports neither the CUDA binding nor the oracle, so that both
sides can be fed from it.  The pages measure on trained models with unnamed
datasets (RotaryQuant, Abstract); these generators stand in for them with the
shapes and value distributions listed per workload below.

Distributions
-------------
* ``gaussian``: iid N(0,1) fp32 with four seeded outlier channels scaled by
  10 (the same channels for K, V and q).
* ``heavy``: per (head, channel) Student-t with 4 degrees of freedom,
  Z / sqrt(chi2_4 / 4) with chi2_4 = -2 ln(U1 U2), times a per-channel scale
  drawn log-uniformly in [0.1, 10]; four seeded outlier channels per head are
  multiplied by a further 20.  K and V have independent scales.  Values are
  rounded to bf16.  Queries are iid N(0,1).
* rotation parameters: sign vector of fair coins (+1/-1, int8) and raw
  quaternion 4-vectors drawn N(0, I) (each consumer normalises them).
"""
from dataclasses import dataclass, field
from typing import List, Optional

import torch

D = 128


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & 0x7FFFFFFFFFFFFFFF)
    return g


def stream_seed(seed: int, *ids: int) -> int:
    """Deterministic sub-seed for an independent stream (no method arithmetic)."""
    s = (int(seed) * 0x9E3779B97F4A7C15) & 0xFFFFFFFFFFFFFFFF
    for i in ids:
        s ^= (int(i) + 0x632BE59BD9B4E019 + ((s << 6) & 0xFFFFFFFFFFFFFFFF) + (s >> 2))
        s &= 0xFFFFFFFFFFFFFFFF
    return s & 0x7FFFFFFFFFFFFFFF


def rotation_params(seed: int, num_kv_heads: int):
    """signs int8 [H][128] (+-1) and raw quaternions float32 [H][32][2][4]."""
    g = _gen(stream_seed(seed, 1), "cpu")
    bits = torch.randint(0, 2, (num_kv_heads, D), generator=g, dtype=torch.int8)
    signs = (bits * 2 - 1).to(torch.int8)
    quats = torch.randn((num_kv_heads, 32, 2, 4), generator=g, dtype=torch.float32)
    return signs.contiguous(), quats.contiguous()


def outlier_channels(seed: int, num_heads: int, count: int = 4) -> torch.Tensor:
    """[H][count] distinct channel indices per head."""
    g = _gen(stream_seed(seed, 2), "cpu")
    return torch.stack([torch.randperm(D, generator=g)[:count] for _ in range(num_heads)])


def channel_scales(seed: int, which: int, num_heads: int, outlier_factor: float = 20.0) -> torch.Tensor:
    """Per (head, channel) scales, log-uniform in [0.1, 10], outliers x factor.

    ``which`` selects an independent draw (0 for K, 1 for V)."""
    g = _gen(stream_seed(seed, 3, which), "cpu")
    u = torch.rand((num_heads, D), generator=g, dtype=torch.float64)
    lo, hi = torch.log(torch.tensor(0.1, dtype=torch.float64)), torch.log(torch.tensor(10.0, dtype=torch.float64))
    sc = torch.exp(lo + (hi - lo) * u)
    idx = outlier_channels(stream_seed(seed, 4, which), num_heads)
    for h in range(num_heads):
        sc[h, idx[h]] *= outlier_factor
    return sc.to(torch.float32)


def heavy_tailed(seed: int, stream: int, n_tok: int, scales: torch.Tensor, device="cpu",
                 dtype=torch.bfloat16) -> torch.Tensor:
    """[n_tok][H][128] Student-t(4) x scales, rounded to ``dtype``.

    ``stream`` names an independent chunk so that long caches can be drawn
    (and re-drawn) chunk by chunk."""
    H = scales.shape[0]
    g = _gen(stream_seed(seed, 5, stream), device)
    z = torch.randn((n_tok, H, D), generator=g, device=device, dtype=torch.float32)
    u1 = 1.0 - torch.rand((n_tok, H, D), generator=g, device=device, dtype=torch.float32)
    u2 = 1.0 - torch.rand((n_tok, H, D), generator=g, device=device, dtype=torch.float32)
    chi2_over_4 = (-(torch.log(u1) + torch.log(u2)) * 0.5).clamp_min(1e-30)
    t = z / torch.sqrt(chi2_over_4)
    return (t * scales.to(device)[None]).to(dtype)


def gaussian(seed: int, stream: int, shape, device="cpu", dtype=torch.float32) -> torch.Tensor:
    g = _gen(stream_seed(seed, 6, stream), device)
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(dtype)


def gaussian_with_outliers(seed: int, stream: int, n_tok: int, H: int, factor: float = 10.0,
                           device="cpu") -> torch.Tensor:
    """fp32 N(0,1) [n_tok][H][128]; the seed's four outlier channels x factor."""
    x = gaussian(seed, stream, (n_tok, H, D), device=device)
    idx = outlier_channels(stream_seed(seed, 7), 1)[0]
    x[..., idx.to(device)] *= factor
    return x


def ragged_lengths(seed: int, batch: int, lo: int, hi: int) -> List[int]:
    g = _gen(stream_seed(seed, 8), "cpu")
    return [int(v) for v in torch.randint(lo, hi + 1, (batch,), generator=g)]


def shuffled_pages(seed: int, num_pages: int) -> torch.Tensor:
    g = _gen(stream_seed(seed, 9), "cpu")
    return torch.randperm(num_pages, generator=g).to(torch.int32)


@dataclass
class Workload:
    """One synthetic workload; ``name`` states what it is and its sizes."""
    name: str
    batch: int
    q_heads: int
    kv_heads: int
    seq_lens: List[int]
    nq: int = 1
    causal: bool = False
    page_size: int = 256
    kind: str = "heavy"          # "heavy" (bf16 Student-t) or "gaussian" (fp32, x10 outliers)
    seed: int = 1000
    shuffle_pages: bool = True
    layers: int = 1
    note: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def group(self) -> int:
        return self.q_heads // self.kv_heads

    @property
    def kv_token_heads(self) -> int:
        return sum(self.seq_lens) * self.kv_heads


def workloads(small: bool = False) -> dict:
    """The workloads (sizes as stated in their names): the five the method is
    measured on, plus causal prefill attention over a packed prompt.

    ``small`` shrinks contexts (and the prefill) to sizes the fp64 oracle
    checks in seconds while keeping several pages, split boundaries and a
    ragged tail."""
    w = {}
    w["single_head_d128_L1024"] = Workload(
        "single_head_d128_L1024", 1, 1, 1, [1024], kind="gaussian", seed=1000, shuffle_pages=False,
        note="fp32 N(0,1), 4 outlier channels x10; compress whole cache then one decode")
    w["gqa_b1_q32_kv8_L4096"] = Workload(
        "gqa_b1_q32_kv8_L4096", 1, 32, 8, [4096 if not small else 1000], seed=1001,
        note="bf16 Student-t(4) x log-uniform channel scales, 4 outliers x20")
    w["gqa_b16_q32_kv4_L32768_paged"] = Workload(
        "gqa_b16_q32_kv4_L32768_paged", 16, 32, 4, [32768 if not small else 700] * 16, seed=1002,
        note="256-token pages, shuffled page table; each step appends one token per sequence, then attends")
    lens = ragged_lengths(1003, 4, 65536, 131072) if not small else ragged_lengths(1003, 4, 300, 900)
    w["long_b4_q64_kv8_L64k_128k_ragged"] = Workload(
        "long_b4_q64_kv8_L64k_128k_ragged", 4, 64, 8, lens, seed=1003,
        note="ragged lengths uniform in [65536, 131072]; only the packed cache is resident")
    w["verify_b8_nq16_q32_kv8_L16384"] = Workload(
        "verify_b8_nq16_q32_kv8_L16384", 8, 32, 8, [16384 if not small else 600] * 8, nq=16, causal=True,
        seed=1004, note="16 consecutive query positions per sequence, causal within the chunk")
    w["prefill_attend_b1_q32_kv8_L32768"] = Workload(
        "prefill_attend_b1_q32_kv8_L32768", 1, 32, 8, [32768 if not small else 600], nq=32768 if not small else 600,
        causal=True, seed=1006, shuffle_pages=False,
        note="causal self-attention of a 32768-token prompt over its own packed K/V: each step compresses the "
             "prompt's K/V into the cache, rotates its 32768 x 32 queries and attends")
    w["prefill_attend_b1_q32_kv8_L8192"] = Workload(
        "prefill_attend_b1_q32_kv8_L8192", 1, 32, 8, [8192 if not small else 400], nq=8192 if not small else 400,
        causal=True, seed=1007, shuffle_pages=False,
        note="the same at an 8192-token prompt (the profiling case of the prefill attention kernel)")
    w["prefill_32768_kv8_layers48"] = Workload(
        "prefill_32768_kv8_layers48", 1, 32, 8, [32768 if not small else 2048], seed=1005,
        layers=48 if not small else 2, shuffle_pages=False,
        note="bulk compression of a 32768-token prompt x 8 KV heads x 48 layers (K and V)")
    return w


# ------------------------------------------------------- workload streams
CHUNK = 4096  # tokens per independently seeded K/V chunk


def workload_scales(wl):
    """(K scales, V scales) of a heavy-tailed workload, or (None, None)."""
    if wl.kind != "heavy":
        return None, None
    return channel_scales(wl.seed, 0, wl.kv_heads), channel_scales(wl.seed, 1, wl.kv_heads)


def workload_kv_chunk(wl, b, c, device="cpu", scales=None):
    """K, V [CHUNK][H][128] of tokens [c*CHUNK, (c+1)*CHUNK) of sequence b."""
    sid = (b * 100003 + c) * 2
    if wl.kind == "heavy":
        ks, vs = scales if scales is not None else workload_scales(wl)
        return (heavy_tailed(wl.seed, sid, CHUNK, ks, device=device),
                heavy_tailed(wl.seed, sid + 1, CHUNK, vs, device=device))
    return (gaussian_with_outliers(wl.seed, sid, CHUNK, wl.kv_heads, device=device),
            gaussian_with_outliers(wl.seed, sid + 1, CHUNK, wl.kv_heads, device=device))


def workload_kv_tokens(wl, b, t0, t1, device="cpu", scales=None):
    """K, V of tokens [t0, t1) of sequence b, chunk by chunk."""
    ks, vs = [], []
    t = t0
    while t < t1:
        c = t // CHUNK
        k, v = workload_kv_chunk(wl, b, c, device=device, scales=scales)
        a, e = t - c * CHUNK, min(t1 - c * CHUNK, CHUNK)
        ks.append(k[a:e])
        vs.append(v[a:e])
        t = c * CHUNK + e
    if not ks:
        shape = (0, wl.kv_heads, D)
        dt = torch.bfloat16 if wl.kind == "heavy" else torch.float32
        return torch.empty(shape, dtype=dt, device=device), torch.empty(shape, dtype=dt, device=device)
    return torch.cat(ks), torch.cat(vs)


def workload_queries(wl, step, device="cpu", nq=None):
    """Queries [B][nq][Hq][128] of decode step `step` (N(0,1); fp32 with the
    x10 outlier channels for the Gaussian workload, bf16 otherwise)."""
    nq = nq or wl.nq
    if wl.kind == "gaussian":
        return gaussian_with_outliers(wl.seed, 10_000_000 + step, wl.batch * nq, wl.q_heads,
                                      device=device).reshape(wl.batch, nq, wl.q_heads, D)
    return gaussian(wl.seed, 10_000_000 + step, (wl.batch, nq, wl.q_heads, D), device=device, dtype=torch.bfloat16)
