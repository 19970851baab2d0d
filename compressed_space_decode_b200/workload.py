"""Device-side set-up of a synthetic workload: context, paged cache, page
table, and the compressed prefix of every sequence.

Only the library's own calls touch the data (isoquant_compress_kv writes the
cache); PyTorch allocates memory and draws the seeded inputs.
"""
import math

import torch

from . import (PagedCache, alloc_workspace, isoquant_compress_kv, isoquant_init, synthetic)
from .synthetic import CHUNK

class DecodeState:
    """Packed cache holding ``wl.seq_lens`` tokens per sequence, plus room for
    ``growth`` appended tokens per sequence."""

    def __init__(self, wl, growth=0, device="cuda", fill=True, page_size=None, bits=3):
        self.wl = wl
        self.bits = bits
        self.device = device
        self.H = wl.kv_heads
        self.Hq = wl.q_heads
        self.G = wl.group
        self.B = wl.batch
        self.ps = page_size or wl.page_size
        self.signs, self.quats = synthetic.rotation_params(wl.seed, self.H)
        self.ctx = isoquant_init(self.signs, self.quats, bits=bits)
        self.seq_lens = list(wl.seq_lens)
        cap = [L + growth for L in self.seq_lens]
        self.max_pages = max(1, max(math.ceil(c / self.ps) for c in cap))
        pages = [max(1, math.ceil(c / self.ps)) for c in cap]
        total = sum(pages)
        perm = synthetic.shuffled_pages(wl.seed, total) if wl.shuffle_pages else torch.arange(total, dtype=torch.int32)
        pt = torch.zeros((self.B, self.max_pages), dtype=torch.int32)
        off = 0
        for b in range(self.B):
            pt[b, :pages[b]] = perm[off:off + pages[b]]
            off += pages[b]
        self.page_table_cpu = pt
        self.page_table = pt.to(device)
        self.cache = PagedCache.allocate(self.H, total, self.ps, device=device, bits=bits)
        self.scales = synthetic.workload_scales(wl)
        if fill:
            for b in range(self.B):
                self.fill_sequence(b, 0, self.seq_lens[b])
        self.seq_lens_dev = torch.tensor(self.seq_lens, dtype=torch.int32, device=device)

    # -------------------------------------------------------------- inputs
    def kv_chunk(self, b, c):
        """K, V of tokens [c*CHUNK, (c+1)*CHUNK) of sequence b (device)."""
        return synthetic.workload_kv_chunk(self.wl, b, c, device=self.device, scales=self.scales)

    def kv_tokens(self, b, t0, t1):
        """K, V of tokens [t0, t1) of sequence b (device)."""
        return synthetic.workload_kv_tokens(self.wl, b, t0, t1, device=self.device, scales=self.scales)

    def slots(self, b, t0, t1):
        t = torch.arange(t0, t1, dtype=torch.int64)
        pages = self.page_table_cpu[b, (t // self.ps)].to(torch.int64)
        return (pages * self.ps + t % self.ps).to(self.device)

    def fill_sequence(self, b, t0, t1, stream=None):
        for c0 in range(t0, t1, CHUNK):
            c1 = min(t1, (c0 // CHUNK + 1) * CHUNK)
            k, v = self.kv_tokens(b, c0, c1)
            isoquant_compress_kv(self.ctx, self.cache, k.contiguous(), v.contiguous(), self.slots(b, c0, c1),
                                 stream=stream)

    def queries(self, step, nq=None):
        return synthetic.workload_queries(self.wl, step, device=self.device, nq=nq)

    def slot_matrix(self, starts, n):
        """int64 [n][B]: slot of token starts[b] + s of every sequence b."""
        t = torch.tensor(starts, dtype=torch.int64)[None, :] + torch.arange(n, dtype=torch.int64)[:, None]
        pages = self.page_table_cpu.to(torch.int64).gather(1, (t // self.ps).T).T
        return (pages * self.ps + t % self.ps).to(self.device)

    def workspace(self, nq=None):
        return alloc_workspace(self.ctx, self.B, nq or self.wl.nq, self.Hq, device=self.device, page_size=self.ps)

    # ----------------------------------------------------- canonical views
    def gather(self, b, h, kv, t0, t1):
        """Canonical packed vectors of tokens [t0, t1): (uint32 words [n][W]
        as int64, fp16 norm bits [n] as int64), read back from the cache."""
        t = torch.arange(t0, t1, dtype=torch.int64)
        pages = self.page_table_cpu[b, t // self.ps].to(torch.int64).to(self.device)
        off = (t % self.ps).to(self.device)
        codes = self.cache.codes[pages, kv, h][torch.arange(t1 - t0, device=self.device), :, off]
        norms = self.cache.norms[pages, kv, h, off]
        return (codes.to(torch.int64).cpu() & 0xFFFFFFFF), norms.view(torch.int16).to(torch.int64).cpu() & 0xFFFF
