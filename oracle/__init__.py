"""CPU oracle for the APB-V / Spava approximate-attention prefill (fp64).

TEST INFRASTRUCTURE ONLY: imported by the test suite, the smoke check and the
benchmark's CPU-baseline leg.  The product library never imports, links or
calls anything here, and nothing here imports the product package.

The arithmetic lives in ``spava_oracle.c`` (plain C, double precision,
OpenMP); this module only builds it and marshals numpy arrays.  Inputs are
bf16 bit patterns (``numpy.uint16``) laid out token-major: Q ``[N, Hq, d]``,
K and V ``[N, Hkv, d]``.

Method source: "Riepilogo Tecnico: APB-V" (gist.science), section
"Metodologia: APB-V" (sequence split, ZigZag layout, anchor block, passing
blocks, computation) and section "Ottimizzazioni a Livello di Sistema"
("Forward Fuso di Contesto e Query").
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "spava_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

# Plain x86-64 code (no -march=native): the library is built on one machine and
# may run on another; no fast-math and no FMA contraction, so results do not
# depend on the build host.
CFLAGS = ["-O3", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off", "-std=c11"]


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` next to its source if it is missing or stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Cfg(ctypes.Structure):
    _fields_ = [
        ("H", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
        ("d", ctypes.c_int32), ("N", ctypes.c_int64), ("a", ctypes.c_int64),
        ("q", ctypes.c_int64), ("off", ctypes.POINTER(ctypes.c_int64)),
        ("l", ctypes.c_int32), ("scale", ctypes.c_double),
        ("local_pair_full", ctypes.c_int32), ("score_norm", ctypes.c_int32),
        ("score_pool", ctypes.c_int32),
    ]


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.POINTER
        c_u16p, c_i32p, c_i64p, c_dp = (P(ctypes.c_uint16), P(ctypes.c_int32),
                                        P(ctypes.c_int64), P(ctypes.c_double))
        lib.oracle_validate.argtypes = [P(_Cfg)]
        lib.oracle_chunk_scores.argtypes = [P(_Cfg), c_u16p, c_u16p, ctypes.c_int, ctypes.c_int, c_dp]
        lib.oracle_select_top_l.argtypes = [c_dp, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32, c_i32p]
        lib.oracle_key_set.argtypes = [P(_Cfg), c_i32p, ctypes.c_int64, ctypes.c_int, c_i64p]
        lib.oracle_key_set.restype = ctypes.c_int64
        lib.oracle_prefill_rows.argtypes = [P(_Cfg), c_u16p, c_u16p, c_u16p, c_i32p, c_i64p,
                                            ctypes.c_int64, c_i32p, ctypes.c_int32, c_dp, c_dp]
        lib.oracle_pair.argtypes = [ctypes.c_int, ctypes.c_int]
        lib.oracle_pool_sums.argtypes = [c_dp, ctypes.c_int64, ctypes.c_int32, c_dp]
        lib.oracle_pool_sums_f32.argtypes = [ctypes.POINTER(ctypes.c_float), ctypes.c_int64,
                                             ctypes.c_int32, ctypes.POINTER(ctypes.c_float)]
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_attended_pairs.argtypes = [P(_Cfg), c_i64p]
        lib.oracle_plan_chunks.argtypes = [ctypes.c_int32, c_i64p, ctypes.c_int64, ctypes.c_int64, c_i64p]
        _lib = lib
    return _lib


@dataclass
class Problem:
    """Shape of one prefill layer (the oracle's own copy of the parameters)."""
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
    score_norm: int = 0     # 0: softmax over the chunk; 1: over the row's whole key set
    score_pool: int = 0     # 0/1: none; odd w >= 3: select on w-key window sums
    _keep: list = field(default_factory=list, repr=False)

    def c(self) -> _Cfg:
        off = np.ascontiguousarray(self.offsets, dtype=np.int64)
        self._keep = [off]
        return _Cfg(self.H, self.Hq, self.Hkv, self.d, self.N, self.a, self.q,
                    off.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), self.l,
                    float(self.scale), int(self.local_pair_full), int(self.score_norm),
                    int(self.score_pool))

    @property
    def n_chunks(self) -> int:
        return 2 * self.H


def _u16(x: np.ndarray) -> ctypes.POINTER(ctypes.c_uint16):
    assert x.dtype == np.uint16 and x.flags.c_contiguous
    return x.ctypes.data_as(ctypes.POINTER(ctypes.c_uint16))


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def pair(H: int, v: int) -> int:
    return int(_load().oracle_pair(H, v))


def plan_chunks(H: int, frame_tokens, anchor_len: int) -> np.ndarray:
    """Chunk offsets ``[2H+1]`` of the visual load balancing: whole,
    consecutive frames, frame counts dealt out evenly over the 2H virtual
    hosts (the first hosts take the extra ones)."""
    ft = np.ascontiguousarray(frame_tokens, dtype=np.int64)
    off = np.empty(2 * H + 1, dtype=np.int64)
    P = ctypes.POINTER(ctypes.c_int64)
    rc = _load().oracle_plan_chunks(int(H), ft.ctypes.data_as(P), len(ft), int(anchor_len),
                                    off.ctypes.data_as(P))
    if rc != 0:
        raise ValueError(f"oracle_plan_chunks failed ({rc})")
    return off


def validate(p: Problem) -> bool:
    cfg = p.c()
    return _load().oracle_validate(ctypes.byref(cfg)) == 0


def chunk_scores(p: Problem, Q: np.ndarray, K: np.ndarray, u: int, g: int) -> np.ndarray:
    """Scores S_u[g, j] of the keys of chunk u (length n_u, float64)."""
    cfg = p.c()
    n = int(p.offsets[u + 1] - p.offsets[u])
    S = np.empty(n, dtype=np.float64)
    rc = _load().oracle_chunk_scores(ctypes.byref(cfg), _u16(Q), _u16(K), u, g,
                                     S.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
    if rc != 0:
        raise ValueError(f"oracle_chunk_scores failed ({rc})")
    return S


def select_top_l(S: np.ndarray, base: int, l: int) -> np.ndarray:
    """Top-l positions (absolute, ascending, -1 padded) of one score vector."""
    S = np.ascontiguousarray(S, dtype=np.float64)
    out = np.empty(l, dtype=np.int32)
    rc = _load().oracle_select_top_l(S.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
                                     len(S), base, l,
                                     out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)))
    if rc != 0:
        raise ValueError(f"oracle_select_top_l failed ({rc})")
    return out


def pool_sums(S: np.ndarray, w: int) -> np.ndarray:
    """Window sums of the pooled-score variant, in the dtype of ``S`` (float64
    or float32, the latter in the GPU's order and precision)."""
    if S.dtype == np.float32:
        S = np.ascontiguousarray(S)
        out = np.empty_like(S)
        fp = ctypes.POINTER(ctypes.c_float)
        rc = _load().oracle_pool_sums_f32(S.ctypes.data_as(fp), len(S), int(w), out.ctypes.data_as(fp))
    else:
        S = np.ascontiguousarray(S, dtype=np.float64)
        out = np.empty_like(S)
        dp = ctypes.POINTER(ctypes.c_double)
        rc = _load().oracle_pool_sums(S.ctypes.data_as(dp), len(S), int(w), out.ctypes.data_as(dp))
    if rc != 0:
        raise ValueError(f"oracle_pool_sums failed ({rc})")
    return out


def selection_scores(p: Problem, scores: np.ndarray) -> np.ndarray:
    """The values the selection ranks: the scores, or with ``score_pool`` > 1
    their window sums taken chunk by chunk."""
    if p.score_pool <= 1:
        return scores
    out = np.array(scores, copy=True)
    for u in range(p.n_chunks - 1):
        s0, s1 = int(p.offsets[u] - p.a), int(p.offsets[u + 1] - p.a)
        for g in range(out.shape[0]):
            if not np.isnan(out[g, s0]):
                out[g, s0:s1] = pool_sums(scores[g, s0:s1], p.score_pool)
    return out


def scores_and_select(p: Problem, Q: np.ndarray, K: np.ndarray, groups=None):
    """Scores and passing blocks of every producing chunk u < 2H-1.

    Returns ``(scores, idx)``: ``scores[g]`` is the float64 vector over the
    context tokens (chunk u at ``offsets[u]-a``; raw scores, before any
    pooling the selection applies), ``idx`` is int32
    ``[2H-1, Hkv, l]``.  KV heads not in ``groups`` are left as NaN / -2
    (not computed) so that a caller cannot use them by accident.
    """
    groups = range(p.Hkv) if groups is None else list(groups)
    C = int(p.offsets[-1] - p.offsets[0])
    scores = np.full((p.Hkv, C), np.nan)
    idx = np.full((p.n_chunks - 1, p.Hkv, p.l), -2, dtype=np.int32)
    for g in groups:
        for u in range(p.n_chunks - 1):
            S = chunk_scores(p, Q, K, u, g)
            s0 = int(p.offsets[u] - p.a)
            scores[g, s0:s0 + len(S)] = S
            ranked = pool_sums(S, p.score_pool) if p.score_pool > 1 else S
            idx[u, g] = select_top_l(ranked, int(p.offsets[u]), p.l)
    return scores, idx


def key_set(p: Problem, idx: np.ndarray, t: int, g: int) -> np.ndarray:
    cfg = p.c()
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    keys = np.empty(t + 1, dtype=np.int64)
    n = _load().oracle_key_set(ctypes.byref(cfg),
                               idx.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), t, g,
                               keys.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)))
    if n < 0:
        raise ValueError(f"oracle_key_set failed ({n})")
    return keys[:n].copy()


def attended_pairs(p: Problem):
    """(anchor, context, query) attended (row, key) pairs per query head,
    counted from the key-set definition without listing keys."""
    cfg = p.c()
    out = (ctypes.c_int64 * 3)()
    rc = _load().oracle_attended_pairs(ctypes.byref(cfg), out)
    if rc != 0:
        raise ValueError(f"oracle_attended_pairs failed ({rc})")
    return tuple(int(x) for x in out)


def prefill_rows(p: Problem, Q, K, V, idx, rows, heads):
    """Outputs (float64 ``O[len(rows), len(heads), d]``, ``lse[len(rows), len(heads)]``)."""
    cfg = p.c()
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    heads = np.ascontiguousarray(heads, dtype=np.int32)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    O = np.empty((len(rows), len(heads), p.d), dtype=np.float64)
    lse = np.empty((len(rows), len(heads)), dtype=np.float64)
    P = ctypes.POINTER
    rc = _load().oracle_prefill_rows(
        ctypes.byref(cfg), _u16(Q), _u16(K), _u16(V),
        idx.ctypes.data_as(P(ctypes.c_int32)), rows.ctypes.data_as(P(ctypes.c_int64)),
        len(rows), heads.ctypes.data_as(P(ctypes.c_int32)), len(heads),
        O.ctypes.data_as(P(ctypes.c_double)), lse.ctypes.data_as(P(ctypes.c_double)))
    if rc != 0:
        raise ValueError(f"oracle_prefill_rows failed ({rc})")
    return O, lse
