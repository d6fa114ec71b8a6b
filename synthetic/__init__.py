"""Seeded synthetic inputs for the VSA2 hot path (router -> TopK -> block-sparse attention).

This module is shared by the CPU oracle tests, the GPU parity tests and the benchmark. It holds
no arithmetic of the method itself: it only draws random fields, rounds them to the storage
dtype and lays them out in cube-major token order, the input contract of the library.

Workload shapes follow "Improving Video Sparse Attention with Fine-grained Router and Sparse
Rebasing" (arXiv 2609.32882), Fig. 8 (batch 1, 20 heads, head dim 128, top64) and §4 setup
(480p / 720p 10-second latents). Tiles are 4x4x4 = 64 tokens; the router pools 2x2x4 = 16-token
sub-cubes, so each tile holds G = 4 sub-cubes.

Value recipe (the pages print no data; this is the stated stand-in):
  * per tensor X in {Q, K, V} and per (b, h): white N(0,1) of shape (T, H, W, D) in fp32,
    smoothed along T, H and W by a normalised Gaussian (sigma = 2 cells, radius 6, periodic
    boundary), rescaled to unit variance, plus 0.5 * N(0,1) white noise;
  * dO (upstream gradient) is plain N(0,1);
  * generator: numpy default_rng([seed, tensor_id, b, h]) with tensor_id Q=0, K=1, V=2, dO=3,
    so any single (b, h) slice can be regenerated alone;
  * values are rounded once to the storage dtype (round-to-nearest-even for bf16) before both
    the GPU path and the oracle see them.
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ProcessPoolExecutor
import multiprocessing as mp

import numpy as np

TENSOR_ID = {"q": 0, "k": 1, "v": 2, "do": 3}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    heads: int
    head_dim: int
    grid: tuple  # (T, H, W) latent token grid
    topk: int
    dtype: str  # "bf16" or "fp32"
    backward: bool = False
    tile: tuple = (4, 4, 4)
    pool: tuple = (2, 2, 4)
    seed: int = 0

    @property
    def tokens(self) -> int:
        t, h, w = self.grid
        return t * h * w

    @property
    def tile_tokens(self) -> int:
        return int(np.prod(self.tile))

    @property
    def pool_tokens(self) -> int:
        return int(np.prod(self.pool))

    @property
    def num_tiles(self) -> int:
        return self.tokens // self.tile_tokens

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 64, (8, 16, 16), 8, "fp32"),
    "480p_top64": Workload("480p_top64", 1, 20, 128, (28, 32, 52), 64, "bf16"),
    "480p_top128": Workload("480p_top128", 1, 20, 128, (28, 32, 52), 128, "bf16"),
    "720p_top64": Workload("720p_top64", 1, 20, 128, (56, 48, 80), 64, "bf16"),
    "480p_train_top64": Workload("480p_train_top64", 1, 20, 128, (28, 32, 52), 64, "bf16", backward=True),
}


def round_to_dtype(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round fp32 values to the storage dtype and return them as fp32 (exactly representable)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "fp32":
        return x
    if dtype != "bf16":
        raise ValueError(dtype)
    u = x.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def _gauss_weights(sigma: float = 2.0, radius: int = 6) -> np.ndarray:
    t = np.arange(-radius, radius + 1, dtype=np.float64)
    w = np.exp(-0.5 * (t / sigma) ** 2)
    return (w / w.sum()).astype(np.float32)


def smoothed_field(rng: np.random.Generator, grid: tuple, d: int) -> np.ndarray:
    """Unit-variance periodic Gaussian-smoothed white noise plus 0.5*N(0,1), shape (T,H,W,D) fp32."""
    from scipy import ndimage

    w = _gauss_weights()
    x = rng.standard_normal((*grid, d), dtype=np.float32)
    for ax in range(3):
        x = ndimage.convolve1d(x, w, axis=ax, mode="wrap")
    x *= np.float32(1.0 / np.sqrt(float(np.sum(w.astype(np.float64) ** 2)) ** 3))
    x += np.float32(0.5) * rng.standard_normal((*grid, d), dtype=np.float32)
    return x


def raster_to_cube_major(x: np.ndarray, tile: tuple, pool: tuple) -> np.ndarray:
    """(T,H,W,D) raster -> (L,D) cube-major: tiles in raster order, inside a tile the pooling
    sub-cubes in raster order, inside a sub-cube the tokens in raster order."""
    T, H, W, D = x.shape
    bt, bh, bw = tile
    rt, rh, rw = pool
    nt, nh, nw = T // bt, H // bh, W // bw
    st, sh, sw = bt // rt, bh // rh, bw // rw
    y = x.reshape(nt, st, rt, nh, sh, rh, nw, sw, rw, D)
    y = y.transpose(0, 3, 6, 1, 4, 7, 2, 5, 8, 9)
    return np.ascontiguousarray(y.reshape(T * H * W, D))


def cube_major_to_raster(y: np.ndarray, grid: tuple, tile: tuple, pool: tuple) -> np.ndarray:
    T, H, W = grid
    D = y.shape[-1]
    bt, bh, bw = tile
    rt, rh, rw = pool
    nt, nh, nw = T // bt, H // bh, W // bw
    st, sh, sw = bt // rt, bh // rh, bw // rw
    z = y.reshape(nt, nh, nw, st, sh, sw, rt, rh, rw, D)
    z = z.transpose(0, 3, 6, 1, 4, 7, 2, 5, 8, 9)
    return np.ascontiguousarray(z.reshape(T, H, W, D))


def make_slice(wl: Workload, name: str, b: int, h: int) -> np.ndarray:
    """One (b, h) slice of tensor `name` in cube-major order, (L, D) fp32 rounded to wl.dtype."""
    rng = np.random.default_rng([wl.seed, TENSOR_ID[name], b, h])
    if name == "do":
        x = rng.standard_normal((*wl.grid, wl.head_dim), dtype=np.float32)
    else:
        x = smoothed_field(rng, wl.grid, wl.head_dim)
    return round_to_dtype(raster_to_cube_major(x, wl.tile, wl.pool), wl.dtype)


def _slice_job(args):
    wl, name, b, h = args
    return make_slice(wl, name, b, h)


def make_tensor(wl: Workload, name: str, heads=None, workers: int | None = None) -> np.ndarray:
    """Tensor `name` as (batch, len(heads), L, D) fp32 in cube-major token order.

    Slices are generated in worker processes started with the 'spawn' method, so this is safe
    to call after CUDA has been initialised in the parent process.
    """
    heads = list(range(wl.heads)) if heads is None else list(heads)
    jobs = [(wl, name, b, h) for b in range(wl.batch) for h in heads]
    if workers is None:
        workers = min(len(jobs), max(1, len(os.sched_getaffinity(0))), 16)
    if workers <= 1 or wl.tokens * wl.head_dim < (1 << 20):
        parts = [_slice_job(j) for j in jobs]
    else:
        with ProcessPoolExecutor(max_workers=workers, mp_context=mp.get_context("spawn")) as ex:
            parts = list(ex.map(_slice_job, jobs))
    out = np.stack(parts).reshape(wl.batch, len(heads), wl.tokens, wl.head_dim)
    return out
