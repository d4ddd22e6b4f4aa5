"""PyTorch-facing wrappers of the libspava C ABI (same names as include/spava.h).

Argument marshalling only: shapes and dtypes are checked, pointers and the
current CUDA stream are handed to the library, and every step of the
computation runs in the library's kernels.  PyTorch provides device memory and
streams.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass, field

import numpy as np
import torch

from . import native
from .native import SpavaConfig


@dataclass
class Layout:
    """One prefill attention layer: [anchor a | 2H chunks | query q]."""
    H: int
    Hq: int
    Hkv: int
    d: int
    N: int
    a: int
    q: int
    offsets: np.ndarray
    l: int
    scale: float = 0.0
    local_pair_full: int = 1
    score_norm: int = 0
    score_pool: int = 0
    _keep: list = field(default_factory=list, repr=False)

    @classmethod
    def from_workload(cls, w, offsets=None) -> "Layout":
        from .synth import chunk_offsets
        off = chunk_offsets(w) if offsets is None else offsets
        return cls(w.H, w.Hq, w.Hkv, w.d, w.N, w.a, w.q, np.asarray(off, dtype=np.int64), w.l,
                   0.0, w.local_pair_full, w.score_norm, w.score_pool)

    def c(self) -> SpavaConfig:
        off = np.ascontiguousarray(self.offsets, dtype=np.int64)
        self._keep = [off]
        return SpavaConfig(self.H, self.Hq, self.Hkv, self.d, self.N, self.a, self.q,
                           off.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), self.l,
                           float(self.scale), int(self.local_pair_full), int(self.score_norm),
                           int(self.score_pool))

    @property
    def n_chunks(self) -> int:
        return 2 * self.H

    @property
    def context(self) -> int:
        return self.N - self.a - self.q


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _check(t: torch.Tensor, shape, dtype, name):
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name}: expected contiguous {dtype} {tuple(shape)}, got "
                         f"{t.dtype} {tuple(t.shape)} contiguous={t.is_contiguous()}")
    if not t.is_cuda:
        raise ValueError(f"{name}: expected a CUDA tensor")


def workspace_size(lay: Layout) -> int:
    n = ctypes.c_size_t()
    cfg = lay.c()
    native.call("spava_workspace_size", ctypes.byref(cfg), ctypes.byref(n))
    return n.value


def packed_len(lay: Layout) -> int:
    n = ctypes.c_int64()
    cfg = lay.c()
    native.call("spava_packed_len", ctypes.byref(cfg), ctypes.byref(n))
    return n.value


def attended_pairs(lay: Layout):
    """(anchor, context, query) attended (row, key) pairs per head, and the
    context pairs per physical host."""
    pairs = (ctypes.c_int64 * 3)()
    per_host = (ctypes.c_int64 * lay.H)()
    cfg = lay.c()
    native.call("spava_attended_pairs", ctypes.byref(cfg), pairs, per_host)
    return tuple(pairs), list(per_host)


def plan_chunks(H: int, frame_tokens, anchor_len: int) -> np.ndarray:
    """Chunk offsets [2H+1] spreading the frames evenly over the 2H virtual
    hosts (whole frames, consecutive, counts differing by at most one)."""
    ft = np.ascontiguousarray(frame_tokens, dtype=np.int64)
    off = np.empty(2 * H + 1, dtype=np.int64)
    P = ctypes.POINTER(ctypes.c_int64)
    native.call("spava_plan_chunks", int(H), ft.ctypes.data_as(P), len(ft), int(anchor_len),
                off.ctypes.data_as(P))
    return off


def new_workspace(lay: Layout, device) -> torch.Tensor:
    """A zeroed workspace (the status word must start at zero)."""
    return torch.zeros(workspace_size(lay), dtype=torch.uint8, device=device)


class Spava:
    """A layer layout plus its workspace on one device."""

    def __init__(self, lay: Layout, device="cuda", workspace: torch.Tensor | None = None):
        self.lay = lay
        self.device = torch.device(device)
        self.cfg = lay.c()
        self.ws = new_workspace(lay, self.device) if workspace is None else workspace
        self.L = packed_len(lay)

    # -- shapes
    def _qkv(self, q, k, v=None):
        lay = self.lay
        _check(q, (lay.N, lay.Hq, lay.d), torch.bfloat16, "q")
        _check(k, (lay.N, lay.Hkv, lay.d), torch.bfloat16, "k")
        if v is not None:
            _check(v, (lay.N, lay.Hkv, lay.d), torch.bfloat16, "v")

    def _args(self):
        return ctypes.byref(self.cfg)

    # -- steps
    def score(self, q, k, scores=None):
        self._qkv(q, k)
        lay = self.lay
        if scores is None:
            scores = torch.zeros((lay.Hkv, lay.context), dtype=torch.float32, device=self.device)
        native.call("spava_score", self._args(), _ptr(q), _ptr(k), _ptr(scores), _ptr(self.ws),
                    self.ws.numel(), _stream(self.device))
        return scores

    def topk_select(self, scores, idx=None):
        lay = self.lay
        _check(scores, (lay.Hkv, lay.context), torch.float32, "scores")
        if idx is None:
            idx = torch.empty((lay.n_chunks - 1, lay.Hkv, lay.l), dtype=torch.int32, device=self.device)
        native.call("spava_topk_select", self._args(), _ptr(scores), _ptr(idx), _stream(self.device))
        return idx

    def pack_passing(self, k, v, idx, pk=None, pv=None):
        lay = self.lay
        shape = (lay.Hkv, self.L, lay.d)
        pk = torch.empty(shape, dtype=torch.bfloat16, device=self.device) if pk is None else pk
        pv = torch.empty(shape, dtype=torch.bfloat16, device=self.device) if pv is None else pv
        native.call("spava_pack_passing", self._args(), _ptr(k), _ptr(v), _ptr(idx), _ptr(pk),
                    _ptr(pv), _stream(self.device))
        return pk, pv

    def attn(self, q, k, v, pk, pv, o=None, lse=None, want_lse=True):
        self._qkv(q, k, v)
        lay = self.lay
        o = torch.empty_like(q) if o is None else o
        if lse is None and want_lse:
            lse = torch.empty((lay.Hq, lay.N), dtype=torch.float32, device=self.device)
        native.call("spava_attn", self._args(), _ptr(q), _ptr(k), _ptr(v), _ptr(pk), _ptr(pv),
                    _ptr(o), _ptr(lse), _ptr(self.ws), self.ws.numel(), _stream(self.device))
        return o, lse

    def prefill_attention(self, q, k, v, o=None, lse=None, idx_out=None, want_lse=True,
                          want_idx=False):
        self._qkv(q, k, v)
        lay = self.lay
        o = torch.empty_like(q) if o is None else o
        if lse is None and want_lse:
            lse = torch.empty((lay.Hq, lay.N), dtype=torch.float32, device=self.device)
        if idx_out is None and want_idx:
            idx_out = torch.empty((lay.n_chunks - 1, lay.Hkv, lay.l), dtype=torch.int32,
                                  device=self.device)
        native.call("spava_prefill_attention", self._args(), _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                    _ptr(lse), _ptr(idx_out), _ptr(self.ws), self.ws.numel(), _stream(self.device))
        return o, lse, idx_out

    def prefill_attention_host(self, q_host, k_host, v_host, o_host, lse_host, q, k, v, o, lse,
                               copy_stream=None):
        """Host (pinned) buffers in and out; device buffers are the caller's.
        With a ``torch.cuda.Stream`` as ``copy_stream`` the copies overlap the
        kernels (run on the current stream) group by group."""
        cs = copy_stream.cuda_stream if copy_stream is not None else None
        native.call("spava_prefill_attention_host", self._args(), _ptr(q_host), _ptr(k_host),
                    _ptr(v_host), _ptr(o_host), _ptr(lse_host), _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                    _ptr(lse), _ptr(self.ws), self.ws.numel(), _stream(self.device), cs)

    def device_status(self) -> int:
        """Synchronises, returns and clears the kernels' status word (0 = clean)."""
        flags = ctypes.c_int32()
        lib = native.load()
        lib.spava_device_status(_ptr(self.ws), self.ws.numel(), _stream(self.device),
                                ctypes.byref(flags))
        return flags.value


# ------------------------------------------------------------------ shards
def shard_layout(lay: Layout, rank: int, world: int):
    """Local layout of rank ``rank`` of ``world``: (first local row of each
    region [2H+2] -- anchor, chunk 0..2H-1, query block; -1 if not held --,
    rows of the local buffers, the chunks of its message slots)."""
    first = np.empty(2 * lay.H + 2, dtype=np.int64)
    n_local = ctypes.c_int64()
    m = lay.H // world if world > 0 and lay.H % world == 0 else 0
    slots = np.empty(max(1, 2 * m), dtype=np.int32)
    cfg = lay.c()
    P = ctypes.POINTER
    native.call("spava_shard_layout", ctypes.byref(cfg), int(rank), int(world),
                first.ctypes.data_as(P(ctypes.c_int64)), ctypes.byref(n_local),
                slots.ctypes.data_as(P(ctypes.c_int32)))
    return first, n_local.value, slots[:2 * m].copy()


def shard_sizes(lay: Layout, world: int):
    """(workspace bytes, pass message bytes, partial message bytes) per rank."""
    ws, pm, qm = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    cfg = lay.c()
    native.call("spava_shard_sizes", ctypes.byref(cfg), int(world), ctypes.byref(ws),
                ctypes.byref(pm), ctypes.byref(qm))
    return ws.value, pm.value, qm.value


def local_positions(lay: Layout, first: np.ndarray) -> np.ndarray:
    """Global token position of every local row, from a shard layout."""
    off = np.asarray(lay.offsets, dtype=np.int64)
    bounds = [(0, lay.a)] + [(int(off[v]), int(off[v + 1])) for v in range(2 * lay.H)] + \
             [(lay.N - lay.q, lay.N)]
    parts = [None] * len(bounds)
    for r, (lo, hi) in enumerate(bounds):
        if first[r] >= 0:
            parts[r] = (int(first[r]), np.arange(lo, hi, dtype=np.int64))
    held = sorted((p for p in parts if p is not None), key=lambda x: x[0])
    return np.concatenate([x for _, x in held]) if held else np.zeros(0, dtype=np.int64)


class SpavaShard:
    """One rank of the ZigZag sequence-parallel layer: rank ``rank`` of
    ``world`` GPUs holds the physical hosts p in [rank*m, (rank+1)*m),
    m = H/world (chunks p and 2H-1-p of each), in local buffers laid out
    [anchor | its chunks in increasing order | query block].  The two
    exchanges -- every rank's passing blocks, every rank's query-row partials
    -- are all-gathers of fixed-size byte messages between the calls."""

    def __init__(self, lay: Layout, rank: int, world: int, device="cuda"):
        self.lay, self.rank, self.world = lay, rank, world
        self.device = torch.device(device)
        self.cfg = lay.c()
        self.first, self.n_local, self.slots = shard_layout(lay, rank, world)
        self.positions = local_positions(lay, self.first)
        ws, pm, qm = shard_sizes(lay, world)
        self.ws = torch.zeros(ws, dtype=torch.uint8, device=self.device)
        self.pass_send = torch.zeros(pm, dtype=torch.uint8, device=self.device)
        self.part_send = torch.zeros(qm, dtype=torch.uint8, device=self.device)
        self.pass_all = torch.zeros(world * pm, dtype=torch.uint8, device=self.device)
        self.part_all = torch.zeros(world * qm, dtype=torch.uint8, device=self.device)

    def _args(self):
        return ctypes.byref(self.cfg), int(self.rank), int(self.world)

    def check_local(self, q, k, v=None):
        lay = self.lay
        _check(q, (self.n_local, lay.Hq, lay.d), torch.bfloat16, "q")
        _check(k, (self.n_local, lay.Hkv, lay.d), torch.bfloat16, "k")
        if v is not None:
            _check(v, (self.n_local, lay.Hkv, lay.d), torch.bfloat16, "v")

    def front(self, q, k, v):
        self.check_local(q, k, v)
        native.call("spava_shard_front", *self._args(), _ptr(q), _ptr(k), _ptr(v),
                    _ptr(self.pass_send), _ptr(self.ws), self.ws.numel(), _stream(self.device))

    def check_out(self, o, lse):
        lay = self.lay
        _check(o, (self.n_local, lay.Hq, lay.d), torch.bfloat16, "o")
        if lse is not None:
            _check(lse, (lay.Hq, self.n_local), torch.float32, "lse")

    def local_attn(self, q, k, v, o, lse):
        self.check_local(q, k, v)
        self.check_out(o, lse)
        native.call("spava_shard_local_attn", *self._args(), _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                    _ptr(lse), _ptr(self.part_send), _ptr(self.ws), self.ws.numel(),
                    _stream(self.device))

    def context_attn(self, q, k, v, o, lse, idx_out=None):
        self.check_local(q, k, v)
        self.check_out(o, lse)
        if idx_out is not None:
            lay = self.lay
            _check(idx_out, (2 * lay.H - 1, lay.Hkv, lay.l), torch.int32, "idx_out")
        native.call("spava_shard_context_attn", *self._args(), _ptr(q), _ptr(k), _ptr(v),
                    _ptr(self.pass_all), _ptr(o), _ptr(lse), _ptr(idx_out), _ptr(self.ws),
                    self.ws.numel(), _stream(self.device))

    def merge(self, o, lse):
        self.check_out(o, lse)
        native.call("spava_shard_merge", *self._args(), _ptr(self.part_all), _ptr(o), _ptr(lse),
                    _ptr(self.ws), self.ws.numel(), _stream(self.device))

    def new_outputs(self, want_lse=True):
        lay = self.lay
        o = torch.empty((self.n_local, lay.Hq, lay.d), dtype=torch.bfloat16, device=self.device)
        lse = (torch.empty((lay.Hq, self.n_local), dtype=torch.float32, device=self.device)
               if want_lse else None)
        return o, lse

    def layer(self, q, k, v, o, lse, all_gather, comm_stream=None, idx_out=None):
        """One sharded layer.  ``all_gather(out, inp)`` gathers every rank's
        ``inp`` bytes into ``out`` (rank-major) on the current stream, e.g.
        ``torch.distributed.all_gather_into_tensor``.  With ``comm_stream``
        the gathers run there: the passing blocks travel while this rank's
        anchor rows and query partials compute, the partials while its
        context rows compute."""
        cur = torch.cuda.current_stream(self.device)
        cs = comm_stream or cur
        self.front(q, k, v)
        if cs is not cur:
            cs.wait_stream(cur)
        with torch.cuda.stream(cs):
            all_gather(self.pass_all, self.pass_send)
        e_pass = cs.record_event() if cs is not cur else None
        self.local_attn(q, k, v, o, lse)
        if cs is not cur:
            cs.wait_stream(cur)
        with torch.cuda.stream(cs):
            all_gather(self.part_all, self.part_send)
        e_part = cs.record_event() if cs is not cur else None
        if e_pass is not None:
            cur.wait_event(e_pass)
        self.context_attn(q, k, v, o, lse, idx_out)
        if e_part is not None:
            cur.wait_event(e_part)
        self.merge(o, lse)
