"""Seeded synthetic inputs and named workload shapes.

This module holds no step of the method: it only draws q, k, v (and nothing else)
from seeded generators.  Both the CUDA path and the CPU oracle take their inputs from
here, so they see the same bf16 values.

Recipe: every tensor is viewed as rows of d values ([b, h, N, d] flattened to
[b*h*N, d]) and split into chunks of 2^17 rows; chunk c of stream s (0: q, 1: k, 2: v,
3: the key offsets, 4: the upstream gradient of the backward) is drawn as float32 N(0, 1) from its own
``torch.Generator('cpu').manual_seed(seed * 2^32 + s * 2^24 + c)``, so the chunks are
independent and are drawn in parallel threads.  q is [b, hq, N, d], k and v are
[b, hkv, N, d].  For the MoBA workloads one offset vector per (batch, kv-head, block),
N(0, 0.5^2) of shape [b, hkv, ceil(N/B), d] (stream 3), is added to every key of its
block (so that the pooled keys separate and the gate's choices are not near-ties);
all three are then cast to bf16.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    hq: int
    hkv: int
    seqlen: int
    d: int
    block: int = 0          # MoBA block size B (0 for pure sliding-window attention)
    topk: int = 0           # blocks kept per query, the own block included
    window: int = 0         # causal window (0 = none)
    key_offset_std: float = 0.0
    sampled_rows: bool = False   # the oracle checks sampled rows only
    q_len: int = 0               # chunked prefill: the queries are the last q_len positions
    gate: str = "mean"           # block selection: "mean" (MoBA), "minmax" (min/max pooled
                                 # blocks) or "static" (own block, `sink` first blocks and the
                                 # most recent ones, no scores)
    sink: int = 0
    note: str = ""

    @property
    def kind(self) -> str:
        return "moba" if self.block > 0 else "swa"

    @property
    def nblocks(self) -> int:
        return -(-self.seqlen // self.block) if self.block else 0

    @property
    def nq(self) -> int:
        """Query rows: q_len for a chunked prefill, else all seqlen positions."""
        return self.q_len or self.seqlen

    @property
    def q_off(self) -> int:
        """Position of query row 0 among the keys."""
        return self.seqlen - self.nq


# The five workloads the method is measured and checked on.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 1, 1024, 64, block=128, topk=3,
                     note="1 head, 8 blocks of 128, top-3"),
    "gqa32k": Workload("gqa32k", 1, 32, 8, 32768, 128, block=512, topk=3, key_offset_std=0.5,
                       note="GQA 32 q / 8 kv heads, 64 blocks of 512, top-3"),
    "swa16k": Workload("swa16k", 1, 32, 32, 16384, 80, window=4096,
                       note="sliding window 4096, 32 heads, d=80"),
    "hybrid64k": Workload("hybrid64k", 2, 8, 4, 65536, 128, block=2048, topk=16, window=512,
                          key_offset_std=0.5, sampled_rows=True,
                          note="GQA 8/4, 32 blocks of 2048, top-16 unioned with window 512"),
    "moba1m": Workload("moba1m", 1, 32, 8, 1 << 20, 128, block=4096, topk=12, key_offset_std=0.5,
                       sampled_rows=True, note="1M tokens, 256 blocks of 4096, top-12"),
    "moba1m_4h": Workload("moba1m_4h", 1, 4, 1, 1 << 20, 128, block=4096, topk=12,
                          key_offset_std=0.5, sampled_rows=True,
                          note="one KV head of the 1M-token workload (4 q-heads): the same "
                               "256 blocks and top-12 at an eighth of the size"),
    "gqa32k_chunk8k": Workload("gqa32k_chunk8k", 1, 32, 8, 32768, 128, block=512, topk=3,
                               key_offset_std=0.5, q_len=8192,
                               note="chunked prefill: the last 8192 queries of the gqa32k "
                                    "context against all 32768 keys"),
    "gqa32k_minmax": Workload("gqa32k_minmax", 1, 32, 8, 32768, 128, block=512, topk=3,
                              key_offset_std=0.5, gate="minmax",
                              note="gqa32k with min/max pooled blocks"),
    "gqa32k_sink": Workload("gqa32k_sink", 1, 32, 8, 32768, 128, block=512, topk=3,
                            key_offset_std=0.5, gate="static", sink=1,
                            note="gqa32k with a static gate: the first block, the most recent "
                                 "block and the own block"),
}


_CHUNK_ROWS = 1 << 17


def _seed(seed: int, stream: int, chunk: int) -> int:
    return seed * (1 << 32) + stream * (1 << 24) + chunk


def _draw_rows(shape, seed: int, stream: int, pool, row_fn=None) -> torch.Tensor:
    """bf16 tensor of ``shape`` (last dim d) drawn chunk by chunk: chunk c holds rows
    [c * 2^17, (c + 1) * 2^17) of the [rows, d] view, float32 N(0, 1) from its own
    generator; ``row_fn(r0, r1, x)`` may adjust the float32 chunk before the cast."""
    d = shape[-1]
    out = torch.empty(shape, dtype=torch.bfloat16)
    flat = out.view(-1, d)
    rows = flat.shape[0]

    def one(c):
        r0, r1 = c * _CHUNK_ROWS, min(rows, (c + 1) * _CHUNK_ROWS)
        g = torch.Generator("cpu").manual_seed(_seed(seed, stream, c))
        x = torch.randn((r1 - r0, d), generator=g, dtype=torch.float32)
        if row_fn is not None:
            row_fn(r0, r1, x)
        flat[r0:r1] = x.to(torch.bfloat16)

    list(pool.map(one, range(-(-rows // _CHUNK_ROWS))))
    return out


def make_inputs(w: Workload, seed: int = 0, device: str = "cpu"):
    """q [b,hq,N,d], k, v [b,hkv,N,d] as bf16 tensors on ``device`` (drawn on the CPU)."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    b, N, d = w.batch, w.seqlen, w.d
    with ThreadPoolExecutor(max_workers=min(32, os.cpu_count() or 1)) as pool:
        q = _draw_rows((b, w.hq, N, d), seed, 0, pool)
        row_fn = None
        if w.key_offset_std > 0:
            # One offset per block, the partial last block (when block does not divide
            # N) included; row r of the [b*hkv*N, d] view sits at position r mod N of
            # plane r div N.
            nb = -(-N // w.block)
            g = torch.Generator("cpu").manual_seed(_seed(seed, 3, 0))
            off = (w.key_offset_std *
                   torch.randn((b * w.hkv * nb, d), generator=g, dtype=torch.float32))

            def row_fn(r0, r1, x):
                r = torch.arange(r0, r1, dtype=torch.int64)
                x += off[(r // N) * nb + (r % N) // w.block]
        k = _draw_rows((b, w.hkv, N, d), seed, 1, pool, row_fn)
        v = _draw_rows((b, w.hkv, N, d), seed, 2, pool)
    return q.to(device), k.to(device), v.to(device)


def make_grad(w: Workload, seed: int = 0, device: str = "cpu"):
    """An upstream gradient dO for the backward, [b, hq, nq, d] bf16: float32 N(0, 1)
    draws of stream 4 (chunked like the inputs), cast to bf16."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(max_workers=min(32, os.cpu_count() or 1)) as pool:
        g = _draw_rows((w.batch, w.hq, w.nq, w.d), seed, 4, pool)
    return g.to(device)


def small_moba(batch=1, hq=2, hkv=1, seqlen=1024, d=64, block=128, topk=3, window=0,
               key_offset_std=0.5, name="small"):
    """A MoBA workload of arbitrary (small) shape with the standard recipe."""
    return Workload(name, batch, hq, hkv, seqlen, d, block=block, topk=topk, window=window,
                    key_offset_std=key_offset_std)


def small_swa(batch=1, hq=2, hkv=2, seqlen=1000, d=80, window=300, name="small_swa"):
    return Workload(name, batch, hq, hkv, seqlen, d, window=window)


def sampled_rows(w: Workload, seed: int = 0) -> np.ndarray:
    """Query positions the oracle checks on the large workloads: the first and last
    row of every 8th block, the first and last 64 rows of 4 random blocks (tile and
    block edges), and 256 uniform rows; drawn with seed + 1000.  Sorted, unique."""
    rng = np.random.default_rng(seed + 1000)
    N = w.seqlen
    B = w.block if w.block else 4096
    n = N // B
    rows = []
    for j in range(0, n, 8):
        rows += [j * B, j * B + B - 1]
    for j in rng.choice(n, size=min(4, n), replace=False):
        rows += list(range(j * B, j * B + min(64, B)))
        rows += list(range(j * B + B - min(64, B), j * B + B))
    rows += list(rng.integers(0, N, size=256))
    return np.unique(np.asarray(rows, dtype=np.int32))
