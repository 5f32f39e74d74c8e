"""Seeded synthetic inputs for PISA attention (shared by the tests, the oracle's
callers and the benchmark).

This module only *makes inputs*: shapes, seeds, value distributions and the
bf16 rounding of the generated values. It holds none of the attention
arithmetic, so both the CUDA path and the CPU oracle can be fed from it without
sharing any of the method.

Workloads (the shapes follow the diffusion-transformer workloads that the PISA
explainer evaluates -- image latents of 64x64 tokens and video latents of
8x64x64 and 21x60x60 tokens; "PISA: Piecewise Sparse Attention Is Wiser for
Efficient Diffusion Transformers", technical summary section 4, Experimental
results):

=====  ============================  ====  =====  =====  =======================
name   [B, H, N, d]                  b     top-k  order  values
=====  ============================  ====  =====  =====  =======================
tiny   [1, 1, 256, 64]               64    2      1      N(0,1) (+ clustered keys)
image  [2, 24, 4096, 128]            64    16     1      N(0,1)/d^1/4 + 2-D waves
video  [1, 24, 32768, 128]           64    64     1      3-D waves + 0.3 N(0,1)
dense  [1, 16, 16384, 64]            128   128/8  0/1    N(0,1)
long   [1, 40, 75600, 128]           128   60     1      3-D waves + 0.3 N(0,1)
=====  ============================  ====  =====  =====  =======================

Every (batch, head, tensor) slice is drawn from its own counter-based seed
(``SeedSequence([seed, b, h, tensor])``), so any single head can be regenerated
alone -- that is how the oracle is run on sampled heads of the large workloads.
Values are generated in fp32 and rounded to bf16 (round to nearest even); the
GPU receives the bf16 bits and the oracle the same values upcast to fp64.
"""
from __future__ import annotations

import concurrent.futures
import dataclasses
import math
import os

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "get", "to_bf16_bits", "bf16_bits_to_f32",
    "make_head", "make_inputs", "make_clustered_keys", "grid_of",
]

_TENSOR_ID = {"q": 0, "k": 1, "v": 2}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    block: int
    topk: int
    order: int
    scale: float
    kind: str            # "normal" | "image" | "video"
    grid: tuple = ()     # token grid for the smooth generators
    seed: int = 0
    route_lambda: float = 0.0   # covariance-aware routing weight (0: plain relevance)
    select_group: int = 1       # query blocks per proxy query (1: every block is its own)
    select_cand: int = 0        # proxy candidate-list length (0: every key block)
    reuse_idx: bool = False     # the step reuses the indices of an earlier call

    @property
    def nB(self) -> int:
        return -(-self.N // self.block)

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def _ceil_keep(keep: float, nB: int) -> int:
    return int(math.ceil(keep * nB - 1e-9))


WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 256, 64, 64, 2, 1, 1.0 / 8.0, "normal", (), 1001),
    "image": Workload("image", 2, 24, 4096, 128, 64, _ceil_keep(0.25, 64), 1, 1.0,
                      "image", (64, 64), 1002),
    "video": Workload("video", 1, 24, 32768, 128, 64, _ceil_keep(0.125, 512), 1,
                      1.0 / math.sqrt(128), "video", (8, 64, 64), 1003),
    "dense": Workload("dense", 1, 16, 16384, 64, 128, 128, 1, 1.0 / 8.0, "normal", (), 1004),
    "dense_k8_o0": Workload("dense_k8_o0", 1, 16, 16384, 64, 128, 8, 0, 1.0 / 8.0,
                            "normal", (), 1004),
    "dense_k8_o1": Workload("dense_k8_o1", 1, 16, 16384, 64, 128, 8, 1, 1.0 / 8.0,
                            "normal", (), 1004),
    "long": Workload("long", 1, 40, 75600, 128, 128, _ceil_keep(0.10, 591), 1,
                     1.0 / math.sqrt(128), "video", (21, 60, 60), 1005),
}
# the video workloads under the hybrid order (global Hbar) and keep-or-drop
WORKLOADS["video_hybrid"] = WORKLOADS["video"].with_(name="video_hybrid", order=2)
WORKLOADS["video_drop"] = WORKLOADS["video"].with_(name="video_drop", order=-1)
WORKLOADS["long_hybrid"] = WORKLOADS["long"].with_(name="long_hybrid", order=2)
# the hybrid order with covariance-aware routing; the weight puts lambda * std(M_j)
# at about half the spread between a row's best and k-th pooled score
WORKLOADS["video_routed"] = WORKLOADS["video"].with_(name="video_routed", order=2, route_lambda=0.015)
# selection amortisation at the hybrid order: one proxy per 4 query blocks keeping 2k
# candidates refined per member (grouped proxies), and indices reused from an earlier
# call with no selection in the step (index reuse across layers)
WORKLOADS["video_grouped"] = WORKLOADS["video"].with_(name="video_grouped", order=2, select_group=4,
                                                      select_cand=128)
WORKLOADS["video_reuse"] = WORKLOADS["video"].with_(name="video_reuse", order=2, reuse_idx=True)


def get(name: str) -> Workload:
    return WORKLOADS[name]


# ----------------------------------------------------------------------------
# bf16 rounding of generated values (input preparation, not the method)
# ----------------------------------------------------------------------------
def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest, ties to even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ----------------------------------------------------------------------------
# generators
# ----------------------------------------------------------------------------
def grid_of(wl: Workload) -> np.ndarray:
    """Integer token coordinates [N, len(grid)], row-major over the grid.

    When the grid has more cells than N the first N cells are used; when it has
    fewer (never for the named workloads) the coordinates wrap.
    """
    dims = wl.grid
    n = np.arange(wl.N)
    coords = []
    rem = n % int(np.prod(dims))
    for ext in reversed(dims):
        coords.append(rem % ext)
        rem = rem // ext
    return np.stack(coords[::-1], axis=1).astype(np.float32)


def _rng(wl: Workload, b: int, h: int, tensor: str) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([wl.seed, b, h, _TENSOR_ID[tensor]]))


def _image_slice(wl: Workload, rng, tensor: str, coords) -> np.ndarray:
    d = wl.d
    amp = 1.0 / d ** 0.25
    if tensor == "v":
        return rng.standard_normal((wl.N, d), dtype=np.float32)
    noise = rng.standard_normal((wl.N, d), dtype=np.float32) * np.float32(amp)
    fy = rng.uniform(0.0, 3.0, d).astype(np.float32)
    fx = rng.uniform(0.0, 3.0, d).astype(np.float32)
    ph = rng.uniform(0.0, 2 * np.pi, d).astype(np.float32)
    H, W = wl.grid
    arg = (2 * np.pi) * (coords[:, 0:1] * fy[None, :] / H + coords[:, 1:2] * fx[None, :] / W) + ph[None, :]
    return noise + np.float32(amp) * np.sin(arg, dtype=np.float32)


def _video_slice(wl: Workload, rng, coords) -> np.ndarray:
    d = wl.d
    T, Hh, W = wl.grid
    out = np.zeros((wl.N, d), dtype=np.float32)
    for _ in range(3):
        ft = rng.uniform(0.0, 4.0, d).astype(np.float32)
        fy = rng.uniform(0.0, 4.0, d).astype(np.float32)
        fx = rng.uniform(0.0, 4.0, d).astype(np.float32)
        ph = rng.uniform(0.0, 2 * np.pi, d).astype(np.float32)
        arg = (2 * np.pi) * (coords[:, 0:1] * ft / T + coords[:, 1:2] * fy / Hh
                             + coords[:, 2:3] * fx / W) + ph
        out += np.sin(arg, dtype=np.float32)
    out *= np.float32(1.0 / math.sqrt(3.0))
    out += np.float32(0.3) * rng.standard_normal((wl.N, d), dtype=np.float32)
    return out


def make_head(wl: Workload, b: int, h: int, tensor: str, coords=None) -> np.ndarray:
    """bf16 bits [N, d] (uint16) of one (batch, head) slice of q, k or v."""
    rng = _rng(wl, b, h, tensor)
    if wl.kind == "normal":
        x = rng.standard_normal((wl.N, wl.d), dtype=np.float32)
    elif wl.kind == "image":
        x = _image_slice(wl, rng, tensor, grid_of(wl) if coords is None else coords)
    elif wl.kind == "video":
        x = _video_slice(wl, rng, grid_of(wl) if coords is None else coords)
    else:
        raise ValueError(wl.kind)
    return to_bf16_bits(x)


def make_inputs(wl: Workload, heads=None, batch_offset: int = 0):
    """Q, K, V as bf16 bits, each uint16 [B, H, N, d] (or [B, len(heads), N, d]).

    ``heads`` selects a subset of (batch-independent) head indices; the values
    of a head do not depend on which other heads are generated. ``batch_offset``
    shifts the batch indices (one process per GPU draws its own batch).
    """
    heads = list(range(wl.H)) if heads is None else list(heads)
    coords = grid_of(wl) if wl.kind != "normal" else None
    out = [np.empty((wl.B, len(heads), wl.N, wl.d), dtype=np.uint16) for _ in range(3)]
    jobs = [(ti, t, b, hi, h) for ti, t in enumerate(("q", "k", "v"))
            for b in range(wl.B) for hi, h in enumerate(heads)]

    def fill(job):
        ti, t, b, hi, h = job
        out[ti][b, hi] = make_head(wl, b + batch_offset, h, t, coords)

    # every slice has its own seed, so the result does not depend on the thread schedule
    workers = min(len(jobs), max(1, min(16, os.cpu_count() or 1)))
    if workers > 1:
        with concurrent.futures.ThreadPoolExecutor(workers) as ex:
            list(ex.map(fill, jobs))
    else:
        for job in jobs:
            fill(job)
    return tuple(out)


def make_clustered_keys(wl: Workload, spread: float, seed_offset: int = 0) -> np.ndarray:
    """Keys whose block j is c_j + spread * N(0,1), c_j ~ N(0,1) (bf16 bits).

    ``spread = 0`` gives blocks of identical keys. Used for the order-0/order-1
    convergence checks on the tiny workload.
    """
    rng = np.random.default_rng(np.random.SeedSequence([wl.seed, 7, seed_offset]))
    K = np.empty((wl.B, wl.H, wl.N, wl.d), dtype=np.float32)
    for j in range(wl.nB):
        s, e = j * wl.block, min((j + 1) * wl.block, wl.N)
        c = rng.standard_normal((wl.B, wl.H, 1, wl.d), dtype=np.float32)
        z = rng.standard_normal((wl.B, wl.H, e - s, wl.d), dtype=np.float32)
        K[:, :, s:e] = c + np.float32(spread) * z
    return to_bf16_bits(K)
