"""Seeded synthetic inputs for the QSA sparse-attention step.

This module only draws random numbers and shapes them into the tensors the
step consumes (a quantized K/V cell cache, indexer keys, queries, weights).
It computes no part of the method itself: no score, selection, softmax,
merge or quantization happens here.  Both the CPU oracle and the CUDA path
are fed from it, so neither can leak into the other through their inputs.

Generator: SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014) used counter-style, so the value at position
i of a stream is a pure function of (stream seed, i).  Uniform doubles take
the top 53 bits; normals use the Box-Muller transform.  Every tensor draws
from its own sub-stream whose seed mixes the workload seed with the tensor's
name, so adding a tensor never shifts the values of another.

Shapes follow the model the pages describe: 24 query heads x 256 (the
prompt path's ``qcur`` row of 6144 floats), 2 KV heads x 256 (``kcur`` and
``vcur`` rows of 512 floats per token), an indexer of 4 heads x 64 in fp16,
int8 K/V with one fp16 scale per 32 values, and top-k 2048 (the 2051-word
``qids`` row per token) -- see "Round 5 Track C Report: Direct FP16 qcurh in
qsa_prep ...", section 1, Target 2, and "opus r20 track A ...", section 3.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

HQ = 24          # query heads
D = 256          # head dim
HKV = 2          # KV heads (GQA 12:1)
G = 32           # values per fp16 scale
NG = D // G      # scale groups per head row
HI = 4           # indexer heads
DI = 64          # indexer dim

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 22


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def splitmix64(seed: int, start: int, count: int) -> np.ndarray:
    """Values start..start+count-1 of the SplitMix64 sequence seeded with ``seed``."""
    with np.errstate(over="ignore"):
        i = np.arange(start + 1, start + count + 1, dtype=np.uint64)
        return _mix(np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + i * _GOLDEN)


def _fnv1a(name: str) -> int:
    h = 0xCBF29CE484222325
    for b in name.encode():
        h = ((h ^ b) * 0x100000001B3) & 0xFFFFFFFFFFFFFFFF
    return h


class Stream:
    """One named sub-stream of a seeded workload."""

    def __init__(self, seed: int, name: str):
        self.seed = int(splitmix64(seed ^ _fnv1a(name), 0, 1)[0])
        self.pos = 0

    def u64(self, n: int) -> np.ndarray:
        out = splitmix64(self.seed, self.pos, n)
        self.pos += n
        return out

    def uniform(self, n: int, lo: float = 0.0, hi: float = 1.0) -> np.ndarray:
        out = np.empty(n, dtype=np.float64)
        for s in range(0, n, _CHUNK):
            m = min(_CHUNK, n - s)
            u = (self.u64(m) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
            out[s:s + m] = lo + (hi - lo) * u
        return out

    def normal(self, n: int) -> np.ndarray:
        out = np.empty(n, dtype=np.float64)
        for s in range(0, n, _CHUNK):
            m = min(_CHUNK, n - s)
            h = (m + 1) // 2
            r = self.u64(2 * h)
            u1 = ((r[:h] >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)
            u2 = (r[h:] >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
            rad = np.sqrt(-2.0 * np.log(u1))
            z = np.concatenate([rad * np.cos(2 * np.pi * u2), rad * np.sin(2 * np.pi * u2)])
            out[s:s + m] = z[:m]
        return out

    def int8_sym(self, n: int) -> np.ndarray:
        """Integers uniform on [-127, 127] (four 16-bit lanes per draw)."""
        out = np.empty(n, dtype=np.int8)
        for s in range(0, n, 4 * _CHUNK):
            m = min(4 * _CHUNK, n - s)
            r = self.u64((m + 3) // 4)
            lanes = np.stack([(r >> np.uint64(16 * j)) & np.uint64(0xFFFF) for j in range(4)], 1)
            v = ((lanes.reshape(-1)[:m] * np.uint64(255)) >> np.uint64(16)).astype(np.int16) - 127
            out[s:s + m] = v.astype(np.int8)
        return out

    def integers(self, n: int, hi: int) -> np.ndarray:
        """Integers uniform on [0, hi)."""
        return (self.uniform(n) * hi).astype(np.int64).clip(0, hi - 1)


@dataclass
class Cache:
    """Host copy of a QSA cell cache (layouts match include/qsa.h)."""
    k: np.ndarray        # int8    [cells][HKV][D]
    v: np.ndarray        # int8    [cells][HKV][D]
    ks: np.ndarray       # float16 [cells][HKV][NG]
    vs: np.ndarray       # float16 [cells][HKV][NG]
    idx_key: np.ndarray  # float16 [cells][DI]

    @property
    def cells(self) -> int:
        return self.k.shape[0]


@dataclass
class Workload:
    name: str
    kind: str            # "decode" or "prefill"
    cache: Cache
    L: int               # decode: cache length seen by the last token; prefill: pos0 + T
    rows: int            # n (decode) or T (prefill)
    pos0: int            # prefill chunk offset (decode: L - n)
    top_k: int
    nsplit: int
    scale: float
    q: np.ndarray        # float32 [rows][HQ][D]
    iq: np.ndarray       # float16 [rows][HI][DI]
    iw: np.ndarray       # float32 [rows][HI]
    meta: dict = field(default_factory=dict)

    def vis0(self) -> int:
        """Cells visible to row 0; row r sees vis0 + r cells."""
        return self.L - self.rows + 1 if self.kind == "decode" else self.pos0 + 1


def make_cache(seed: int, cells: int, ks_range=(0.005, 0.02), vs_range=(0.005, 0.02),
               outlier_frac: float = 0.0, dup_frac: float = 0.0) -> Cache:
    k = Stream(seed, "k").int8_sym(cells * HKV * D).reshape(cells, HKV, D)
    v = Stream(seed, "v").int8_sym(cells * HKV * D).reshape(cells, HKV, D)
    ks = Stream(seed, "ks").uniform(cells * HKV * NG, *ks_range).astype(np.float16).reshape(cells, HKV, NG)
    vs = Stream(seed, "vs").uniform(cells * HKV * NG, *vs_range).astype(np.float16).reshape(cells, HKV, NG)
    key = Stream(seed, "idx_key").normal(cells * DI).reshape(cells, DI)
    if outlier_frac > 0:
        nout = max(1, int(round(outlier_frac * cells)))
        which = np.unique(Stream(seed, "outliers").integers(nout, cells))
        key[which] *= 8.0
    key = key.astype(np.float16)
    if dup_frac > 0:
        ndup = int(round(dup_frac * cells))
        perm = np.argsort(Stream(seed, "dup_pick").uniform(cells), kind="stable")
        dups = np.sort(perm[:ndup])
        sources = np.sort(perm[ndup:])
        src = sources[Stream(seed, "dup_src").integers(ndup, sources.size)]
        key[dups] = key[src]
    return Cache(k=k, v=v, ks=ks, vs=vs, idx_key=key)


def make_queries(seed: int, rows: int):
    q = Stream(seed, "q").normal(rows * HQ * D).astype(np.float32).reshape(rows, HQ, D)
    iq = Stream(seed, "iq").normal(rows * HI * DI).astype(np.float16).reshape(rows, HI, DI)
    iw = Stream(seed, "iw").uniform(rows * HI).astype(np.float32).reshape(rows, HI)
    return q, iq, iw


def make_new_cells(seed: int, n: int):
    """fp32 K/V rows and fp16 indexer keys for n cells appended by a cache write."""
    k = Stream(seed, "new_k").normal(n * HKV * D).astype(np.float32).reshape(n, HKV, D)
    v = Stream(seed, "new_v").normal(n * HKV * D).astype(np.float32).reshape(n, HKV, D)
    key = Stream(seed, "new_key").normal(n * DI).astype(np.float16).reshape(n, DI)
    return k, v, key


# The five workloads: decode at 4K/64K/256K cells, prefill chunks at 64K/256K.
CONFIGS = {
    0: dict(kind="decode", L=4096, n=1, top_k=512, nsplit=0),
    1: dict(kind="decode", L=65536, n=8, top_k=2048, nsplit=0, outlier_frac=0.01),
    2: dict(kind="decode", L=262144, n=1, top_k=2048, nsplit=64, outlier_frac=0.01),
    3: dict(kind="prefill", L=65536, T=2048, pos0=63488, top_k=2048, nsplit=1),
    4: dict(kind="prefill", L=262144, T=1024, pos0=261120, top_k=2048, nsplit=1,
            dup_frac=0.10, vs_range=(1e-4, 0.05)),
}

CONFIG_NAMES = {
    0: "decode n=1 L=4096 top_k=512",
    1: "decode n=1..8 (MTP) L=65536 top_k=2048",
    2: "decode n=1 L=262144 top_k=2048 nsplit=64",
    3: "prefill T=2048 pos0=63488 L=65536 top_k=2048",
    4: "prefill T=1024 pos0=261120 L=262144 top_k=2048 dup-keys",
}


def make_workload(cfg: int, n: int | None = None, cells: int | None = None, rows: int | None = None,
                  seed: int | None = None) -> Workload:
    """Build workload ``cfg``; ``n``/``rows``/``cells`` shrink it for fast tests."""
    c = CONFIGS[cfg]
    seed = 1000 + cfg if seed is None else seed
    L = c["L"] if cells is None else cells
    cache = make_cache(seed, L, vs_range=c.get("vs_range", (0.005, 0.02)),
                       outlier_frac=c.get("outlier_frac", 0.0), dup_frac=c.get("dup_frac", 0.0))
    if c["kind"] == "decode":
        nr = c["n"] if n is None else n
        q, iq, iw = make_queries(seed, nr)
        return Workload(CONFIG_NAMES[cfg], "decode", cache, L, nr, L - nr, c["top_k"], c["nsplit"],
                        1.0 / 16.0, q, iq, iw, dict(cfg=cfg))
    T = c["T"] if rows is None else rows
    pos0 = L - T if (cells is not None or rows is not None) else c["pos0"]
    q, iq, iw = make_queries(seed, T)
    return Workload(CONFIG_NAMES[cfg], "prefill", cache, pos0 + T, T, pos0, c["top_k"], c["nsplit"],
                    1.0 / 16.0, q, iq, iw, dict(cfg=cfg))


def quantizer_patterns(seed: int, ngroups: int) -> dict:
    """Five fp32 input patterns for the cache-write quantizer (seeded random,
    signed zeros, mixed powers of two, alternating signs, tiny values), after
    the pattern set of the CPU bit-pattern harness in "round 4 track b: mtp
    input and hyper-connection fusion", section "checks actually run", item 2."""
    n = ngroups * G
    st = Stream(seed, "qpat")
    rnd = (st.normal(n) * 3.0).astype(np.float32)
    zeros = np.where(st.uniform(n) < 0.5, np.float32(0.0), np.float32(-0.0)).astype(np.float32)
    exps = st.integers(n, 40) - 20
    sgn = np.where(st.uniform(n) < 0.5, -1.0, 1.0)
    pow2 = (sgn * np.ldexp(1.0, exps)).astype(np.float32)
    alt = (np.where(np.arange(n) % 2 == 0, 1.0, -1.0) * (1.0 + st.uniform(n))).astype(np.float32)
    tiny = (st.normal(n) * 3e-6).astype(np.float32)
    return dict(random=rnd, signed_zeros=zeros, pow2=pow2, alternating=alt, tiny=tiny)
