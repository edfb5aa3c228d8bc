"""Counter-based seeded input streams and the five workload shapes.

Random numbers
--------------
Every tensor draws from its own SplitMix64 stream (Steele, Lea and Flood,
"Fast splittable pseudorandom number generators", OOPSLA 2014).  Output ``i``
of a stream with key ``K`` is ``mix64(K + (i + 1) * GAMMA)``, so any index
range can be generated on its own.  ``mix64`` is the published finaliser
(shift 30 / 27 / 31, multipliers 0xbf58476d1ce4e5b9 and 0x94d049bb133111eb).

* uniform in [0, 1):   ``(z >> 11) * 2**-53``
* normal N(0, 1):      Box-Muller in fp64 on the pair (u1, u2) taken from
  outputs (2i, 2i+1): ``r = sqrt(-2 ln(1 - u1))``, ``n[2i] = r cos(2 pi u2)``,
  ``n[2i+1] = r sin(2 pi u2)``.
* fp32 tensors are the fp64 values rounded to nearest even; bf16 tensors are
  those fp32 values rounded to nearest even once more (torch's conversion).

Workloads (DeepSeek-V3 / DeepSeek-MoE shapes named by the DeepEP V2 README's
benchmark setting: 8K tokens per batch, hidden 7168, top-8, FP8 dispatch and
BF16 combine) are listed in ``CONFIGS``.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# stream ids: one per tensor kind
STREAM_X = 1
STREAM_LOGITS = 2
STREAM_BIAS = 3
STREAM_Y = 4
STREAM_PERM = 5

_CHUNK = 1 << 22  # values per numpy chunk (bounds temporary memory)


def _mix64(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, stream: int) -> np.uint64:
    """Key of the stream ``stream`` under ``seed`` (two mix64 rounds)."""
    with np.errstate(over="ignore"):
        a = _mix64(np.array([seed & 0xFFFFFFFFFFFFFFFF], dtype=np.uint64))
        b = _mix64(a + np.uint64(stream))
    return b[0]


def splitmix64_stream(key: np.uint64, start: int, count: int) -> np.ndarray:
    """Outputs ``start .. start+count-1`` of the SplitMix64 stream ``key``."""
    idx = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix64(np.uint64(key) + idx * GAMMA)


def uniforms(key: np.uint64, start: int, count: int) -> np.ndarray:
    """fp64 uniforms in [0, 1) from stream outputs ``start ..``."""
    z = splitmix64_stream(key, start, count)
    return (z >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def normals(key: np.uint64, start: int, count: int) -> np.ndarray:
    """fp64 N(0,1) values ``start .. start+count-1`` of the normal stream."""
    out = np.empty(count, dtype=np.float64)
    pos = 0
    while pos < count:
        n = min(_CHUNK, count - pos)
        first = start + pos
        p0 = first // 2
        p1 = (first + n - 1) // 2 + 1
        u = uniforms(key, 2 * p0, 2 * (p1 - p0))
        u1 = u[0::2]
        u2 = u[1::2]
        r = np.sqrt(-2.0 * np.log1p(-u1))
        th = (2.0 * math.pi) * u2
        pair = np.empty(2 * (p1 - p0), dtype=np.float64)
        pair[0::2] = r * np.cos(th)
        pair[1::2] = r * np.sin(th)
        off = first - 2 * p0
        out[pos:pos + n] = pair[off:off + n]
        pos += n
    return out


def _to_bf16(v64: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(v64.astype(np.float32)).to(torch.bfloat16)


def expert_permutation(seed: int, E: int) -> np.ndarray:
    """A seeded permutation pi of the experts: pi[e] = popularity rank of e."""
    u = uniforms(stream_key(seed, STREAM_PERM), 0, E)
    order = np.argsort(u, kind="stable")
    pi = np.empty(E, dtype=np.int64)
    pi[order] = np.arange(E)
    return pi


def redundant_expert_map(pi: np.ndarray, R: int, slots_per_rank: int,
                         n_hot: int, zipf_s: float):
    """Greedy replica placement for the skewed workload (an input, not a step).

    The predicted load of logical expert e is its Zipf prior
    ``(pi[e] + 1) ** -zipf_s``.  The ``n_hot`` most loaded experts get one
    extra replica; a replica carries load / n_rep.  Replicas, ordered by
    (load desc, logical id asc, replica index asc), go one by one to the rank
    with the least accumulated load that still has a free slot (ties to the
    lower rank); a replica's physical id is rank * slots_per_rank + its arrival
    order on that rank.  This is the "global" replicate-then-pack policy the
    DeepSeek EPLB description gives in words.

    Returns ``phys_of`` int32 [E, 2] (unused entries -1, each row ascending)
    and ``n_rep`` int32 [E].
    """
    E = pi.shape[0]
    P = R * slots_per_rank
    n_rep = np.where(pi < n_hot, 2, 1).astype(np.int32)
    if int(n_rep.sum()) != P:
        raise ValueError("replica count does not fill the physical slots")
    load = (pi.astype(np.float64) + 1.0) ** (-zipf_s)
    replicas = []
    for e in range(E):
        for r in range(int(n_rep[e])):
            replicas.append((-load[e] / n_rep[e], e, r))
    replicas.sort()
    acc = [0.0] * R
    used = [0] * R
    phys = [[] for _ in range(E)]
    for neg_l, e, _r in replicas:
        best = -1
        for rank in range(R):
            if used[rank] >= slots_per_rank:
                continue
            if best < 0 or acc[rank] < acc[best]:
                best = rank
        phys[e].append(best * slots_per_rank + used[best])
        used[best] += 1
        acc[best] += -neg_l
    phys_of = np.full((E, 2), -1, dtype=np.int32)
    for e in range(E):
        ids = sorted(phys[e])
        phys_of[e, :len(ids)] = ids
    return phys_of, n_rep


@dataclasses.dataclass(frozen=True)
class WorkloadConfig:
    name: str
    T: int
    H: int
    E: int
    R: int
    n_group: int
    topk_group: int
    topk: int
    fp8: bool
    routed_scale: float
    renorm: bool
    bias: str  # "zero" | "uniform" | "zipf"
    P: Optional[int] = None  # physical expert slots (redundant experts)
    n_hot: int = 0
    zipf_s: float = 1.2
    zipf_beta: float = 0.05
    inter: int = 2048        # expert intermediate width I (gate and up halves)

    @property
    def n_phys(self) -> int:
        return self.P if self.P is not None else self.E

    def scaled(self, T: int) -> "WorkloadConfig":
        return dataclasses.replace(self, T=T)


CONFIGS = {
    "tiny": WorkloadConfig("tiny", T=128, H=256, E=16, R=4, n_group=1,
                           topk_group=1, topk=2, fp8=False, routed_scale=1.0,
                           renorm=True, bias="zero", inter=128),
    "ds16b": WorkloadConfig("ds16b", T=4096, H=2048, E=64, R=8, n_group=1,
                            topk_group=1, topk=6, fp8=True, routed_scale=1.0,
                            renorm=True, bias="uniform", inter=1408),
    "v3": WorkloadConfig("v3", T=8192, H=7168, E=256, R=8, n_group=8,
                         topk_group=4, topk=8, fp8=True, routed_scale=2.5,
                         renorm=True, bias="uniform"),
    "v3_decode": WorkloadConfig("v3_decode", T=256, H=7168, E=256, R=32,
                                n_group=8, topk_group=4, topk=8, fp8=True,
                                routed_scale=2.5, renorm=True, bias="uniform"),
    "skew": WorkloadConfig("skew", T=16384, H=7168, E=256, R=32, n_group=8,
                           topk_group=4, topk=8, fp8=True, routed_scale=2.5,
                           renorm=True, bias="zipf", P=288, n_hot=32),
}


class Workload:
    """Materialises one configuration's inputs on the host (CPU tensors).

    ``x`` bf16 [T, H], ``logits`` fp32 [T, E], ``bias`` fp32 [E] and, for the
    redundant-expert workload, ``phys_of`` int32 [E, 2] and ``n_rep`` int32
    [E].  ``y_rows(first, n)`` gives rows of the stand-in expert output
    (bf16 N(0,1), [T*k, H]) without materialising the whole tensor.
    """

    def __init__(self, cfg: WorkloadConfig, seed: int = 0):
        self.cfg = cfg
        self.seed = seed
        T, E = cfg.T, cfg.E
        self._x = None
        self.logits = torch.from_numpy(
            normals(stream_key(seed, STREAM_LOGITS), 0, T * E).astype(np.float32)
        ).view(T, E)
        self.phys_of = None
        self.n_rep = None
        if cfg.bias == "zero":
            b = np.zeros(E, dtype=np.float64)
        elif cfg.bias == "uniform":
            b = -0.1 + 0.2 * uniforms(stream_key(seed, STREAM_BIAS), 0, E)
        elif cfg.bias == "zipf":
            pi = expert_permutation(seed, E)
            b = cfg.zipf_beta * (-cfg.zipf_s) * np.log(pi.astype(np.float64) + 1.0)
            self.pi = pi
        else:
            raise ValueError(cfg.bias)
        self.bias = torch.from_numpy(b.astype(np.float32))
        if cfg.P is not None:
            pi = self.pi if cfg.bias == "zipf" else expert_permutation(seed, E)
            self.phys_of, self.n_rep = (torch.from_numpy(a) for a in redundant_expert_map(
                pi, cfg.R, cfg.P // cfg.R, cfg.n_hot, cfg.zipf_s))

    @property
    def x(self) -> torch.Tensor:
        if self._x is None:
            T, H = self.cfg.T, self.cfg.H
            self._x = _to_bf16(normals(stream_key(self.seed, STREAM_X), 0, T * H)).view(T, H)
        return self._x

    def x_rows(self, first: int, n: int) -> torch.Tensor:
        H = self.cfg.H
        return _to_bf16(normals(stream_key(self.seed, STREAM_X), first * H, n * H)).view(n, H)

    def y_rows(self, first: int, n: int) -> torch.Tensor:
        H = self.cfg.H
        v = normals(stream_key(self.seed, STREAM_Y), first * H, n * H)
        return _to_bf16(v).view(n, H)

    def y(self) -> torch.Tensor:
        return self.y_rows(0, self.cfg.T * self.cfg.topk)


def device_normal_bf16(rows: int, cols: int, seed: int, device="cuda") -> torch.Tensor:
    """bf16 N(0,1) [rows, cols] drawn on the device by torch's seeded Philox
    generator: a large stand-in input (e.g. expert outputs) that would take
    too long to draw on the host.  Both the GPU path and the oracle read the
    same bytes (the oracle after a copy to the host)."""
    g = torch.Generator(device=device)
    g.manual_seed(0x5EED0000 + seed)
    out = torch.empty((rows, cols), device=device, dtype=torch.bfloat16)
    step = max(1, (1 << 26) // max(cols, 1))
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        out[r0:r1] = torch.randn((r1 - r0, cols), generator=g, device=device,
                                 dtype=torch.float32).to(torch.bfloat16)
    return out
