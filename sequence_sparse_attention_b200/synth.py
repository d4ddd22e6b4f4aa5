"""Seeded synthetic prefill inputs shaped like long-video LMM prefill.

This module only draws random numbers and lays out chunk boundaries; it holds
none of the attention arithmetic, so both the CUDA library's callers and the
CPU oracle can take their inputs from it.

Stand-in for the video benchmarks the method is evaluated on (LongVideoBench,
VNBench; "Riepilogo Tecnico: APB-V", section "Risultati Sperimentali"), which
are not available here: visual tokens come in frames of ``frame`` tokens, and
every key of a frame carries the same per-frame, per-KV-head offset vector,
which gives keys the frame-level correlation of video embeddings.

Recipe (all draws from one ``torch.Generator`` seeded with ``seed``, in this
order, in token slabs of 8192 so large layers need no huge temporaries):
  Q ~ N(0, 1)                                   [N, Hq, d]
  K = z + o[frame(t), g],  z ~ N(0, 1),  o ~ N(0, sigma^2)   [N, Hkv, d]
      frame(t) = floor(t / frame) over absolute positions
  V ~ N(0, 1)                                   [N, Hkv, d]
  heavy hitters: a seeded permutation picks ``heavy_frac`` of the context
      positions [a, N-q); their K rows (all KV heads) are multiplied by
      ``heavy_mult`` after the offset is added.
All values are drawn in float32 and rounded to bf16 (round to nearest even).

Chunk boundaries: the context [a, N-q) is split into 2H chunks.  Equal split
gives the first ``C mod 2H`` chunks one extra token.  With ``jitter > 0`` the
context is counted in frames: chunk v gets F(1+delta_v) frames, delta_v ~
U[-jitter, jitter], rounded by largest remainder (ties to the lower v) so the
frame counts add up, i.e. uneven per-host frame counts as the visual load
balancer would hand over.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    H: int          # physical hosts = virtual-host pairs; 2H chunks
    Hq: int
    Hkv: int
    d: int
    N: int
    a: int          # anchor length
    q: int          # query-block length
    l: int          # passing-block size per KV head per chunk
    frame: int = 256
    sigma: float = 0.5
    heavy_frac: float = 0.0
    heavy_mult: float = 4.0
    jitter: float = 0.0
    seed: int = 0
    local_pair_full: int = 1
    score_norm: int = 0     # selection variants (see spava_config)
    score_pool: int = 0
    # Uneven frames: token counts of the context's frames in order (the anchor
    # and the query block count as one frame each); () = frames of `frame`
    # tokens over absolute positions.
    frame_tokens: tuple = ()
    # Explicit chunk offsets off[0..2H], e.g. from the visual load balancer
    # (spava_plan_chunks); () = the split chunk_offsets() draws.
    offsets: tuple = ()

    @property
    def n_chunks(self) -> int:
        return 2 * self.H

    @property
    def context(self) -> int:
        return self.N - self.a - self.q

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five layer shapes of the long-video prefill study.
WORKLOADS = {
    "tiny": Workload("tiny", H=2, Hq=4, Hkv=2, d=64, N=2048, a=64, q=32, l=32,
                     frame=64, seed=0),
    "16k": Workload("16k", H=4, Hq=28, Hkv=4, d=128, N=16384, a=1024, q=128, l=1024,
                    seed=1),
    "64k": Workload("64k", H=8, Hq=28, Hkv=4, d=128, N=65536, a=2048, q=256, l=2048,
                    seed=2),
    "128k": Workload("128k", H=8, Hq=28, Hkv=4, d=128, N=131072, a=4096, q=256, l=4096,
                     heavy_frac=0.05, seed=3),
    "256k": Workload("256k", H=16, Hq=32, Hkv=8, d=128, N=262144, a=4096, q=512, l=2048,
                     jitter=0.10, seed=4),
}


def chunk_offsets(w: Workload) -> np.ndarray:
    """Chunk boundaries ``off[0..2H]`` (int64): off[0] = a, off[2H] = N - q."""
    nc, C = w.n_chunks, w.context
    if w.offsets:
        off = np.asarray(w.offsets, dtype=np.int64)
        if len(off) != nc + 1 or off[0] != w.a or off[-1] != w.N - w.q or (np.diff(off) < 1).any():
            raise ValueError("explicit offsets do not split the context into 2H chunks")
        return off
    if C < nc:
        raise ValueError("context shorter than the number of chunks")
    if w.jitter <= 0.0:
        sizes = np.full(nc, C // nc, dtype=np.int64)
        sizes[: C % nc] += 1
    else:
        if C % w.frame:
            raise ValueError("jittered split needs the context to be whole frames")
        frames = C // w.frame
        g = torch.Generator().manual_seed(w.seed)
        delta = (torch.rand(nc, generator=g, dtype=torch.float64) * 2 - 1) * w.jitter
        want = (frames / nc) * (1.0 + delta.numpy())
        want *= frames / want.sum()
        base = np.floor(want).astype(np.int64)
        rem = frames - int(base.sum())
        frac = want - base
        order = sorted(range(nc), key=lambda v: (-frac[v], v))
        for v in order[:rem]:
            base[v] += 1
        if (base < 1).any():
            raise ValueError("jitter left a chunk without frames")
        sizes = base * w.frame
    off = np.empty(nc + 1, dtype=np.int64)
    off[0] = w.a
    off[1:] = w.a + np.cumsum(sizes)
    assert off[-1] == w.N - w.q
    return off


def _randn_slabs(g: torch.Generator, shape, device, slab=8192) -> torch.Tensor:
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    for t0 in range(0, shape[0], slab):
        t1 = min(shape[0], t0 + slab)
        out[t0:t1] = torch.randn((t1 - t0,) + tuple(shape[1:]), generator=g,
                                 device=device, dtype=torch.float32).to(torch.bfloat16)
    return out


def make_inputs(w: Workload, device: str | torch.device = "cpu"):
    """Q, K, V (bf16, token-major, contiguous) and the chunk offsets.

    The same (workload, device) always gives the same bytes.  CPU and CUDA
    generators draw different streams, so a comparison must hand the SAME
    tensors (copied) to both sides.
    """
    device = torch.device(device)
    g = torch.Generator(device=device).manual_seed(w.seed)
    Q = _randn_slabs(g, (w.N, w.Hq, w.d), device)
    if w.frame_tokens:
        if sum(w.frame_tokens) != w.context:
            raise ValueError("frame_tokens must add up to the context length")
        # frame boundaries: the anchor, each context frame, the query block
        bounds = torch.tensor(np.cumsum([w.a] + list(w.frame_tokens) + [w.q]), device=device)
        n_frames = len(w.frame_tokens) + 2
    else:
        n_frames = (w.N + w.frame - 1) // w.frame
    K = torch.empty((w.N, w.Hkv, w.d), dtype=torch.bfloat16, device=device)
    z = _randn_slabs(g, (w.N, w.Hkv, w.d), device)
    o = torch.randn((n_frames, w.Hkv, w.d), generator=g, device=device,
                    dtype=torch.float32) * w.sigma
    slab = 8192
    for t0 in range(0, w.N, slab):
        t1 = min(w.N, t0 + slab)
        pos = torch.arange(t0, t1, device=device)
        fr = torch.bucketize(pos, bounds, right=True) if w.frame_tokens else pos // w.frame
        K[t0:t1] = (z[t0:t1].float() + o[fr]).to(torch.bfloat16)
    del z
    V = _randn_slabs(g, (w.N, w.Hkv, w.d), device)
    if w.heavy_frac > 0:
        C = w.context
        perm = torch.randperm(C, generator=g, device=device)
        pos = perm[: int(round(w.heavy_frac * C))] + w.a
        K[pos] = (K[pos].float() * w.heavy_mult).to(torch.bfloat16)
    return Q, K, V, chunk_offsets(w)


def uneven_frames(n_frames: int, lo: int, hi: int, seed: int) -> tuple:
    """Token counts of ``n_frames`` frames drawn uniformly from [lo, hi)
    (seeded): frames of uneven resolution for the visual load balancer."""
    g = torch.Generator().manual_seed(seed)
    return tuple(int(x) for x in torch.randint(lo, hi, (n_frames,), generator=g))


def bf16_bits(x: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (host copy, contiguous)."""
    return x.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
