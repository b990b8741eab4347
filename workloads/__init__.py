"""Seeded synthetic inputs for residual vector quantization (RVQ) of visual features.

This module only draws random numbers and lays them out; it holds none of the
RVQ arithmetic (no distances, no argmin, no residual update).  Both the fp64
oracle (tests, CPU baseline) and the CUDA path (tests, bench) take their inputs
from here, so the two sides always see bit-identical data.

The pages that describe the method (LongCat-2.5 release notes, "Visual Primitive
Modeling" / "Discrete Native Resolution Vision Transformer" and "Offline Visual
Preprocessing") fix no codebook size, depth, feature width or data set.  The five
workloads below are synthetic stand-ins shaped like native-resolution image
patch features:

  tiny    N=256,  D=64,   L=2, K=256,   fp32 features, fp32 codebooks
  image   N=4096 (64x64 patch grid), D=1024, L=4, K=8192, bf16 features, fp32 codebooks
  packed  64 images, patch grids h,w ~ U{16..96}, D=1024, L=8, K=16384, bf16 / fp32
  offline N=2^20, D=256, L=4, K=65536, bf16 features (Gaussian mixture + tail), fp32 codebooks
  detok   ids [2^20, 8] (level 0 Zipf(1.1), others uniform over 16384), bf16 codebooks [8,16384,1024]

Every array is returned as float32 whose values are exactly representable in the
stored dtype (bf16 values are rounded once, round-to-nearest-even, here), plus the
dtype tag; `as_bf16_bits` gives the 16-bit payload for upload.
"""
from __future__ import annotations

import dataclasses

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "spec", "generate", "round_bf16", "as_bf16_bits",
    "bf16_bits_to_f32", "zipf_ids", "sample_rows",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    N: int            # number of feature vectors (tokens); packed: realised after drawing grids
    D: int            # feature width
    L: int            # RVQ levels
    K: int            # codewords per level
    f_dtype: str      # "f32" | "bf16" storage type of features
    cb_dtype: str     # "f32" | "bf16" storage type of codebooks
    seed: int
    description: str


WORKLOADS = {
    "tiny": Workload("tiny", 256, 64, 2, 256, "f32", "f32", 0,
                     "N=256 fp32 vectors, D=64, L=2, K=256; level-l codebook ~N(0,(0.5^l)^2) "
                     "with codeword 0 zero at every level; features = level-0 codeword (uniform id) "
                     "+ N(0,0.3^2) noise; seed 0"),
    "image": Workload("image", 4096, 1024, 4, 8192, "bf16", "f32", 1,
                      "single native-resolution image: 64x64 patch grid -> N=4096 bf16 features, "
                      "D=1024, L=4, K=8192 fp32 codebooks ~N(0,(0.5^l)^2); features = sum over "
                      "levels of uniformly drawn codewords + N(0,0.05^2)"),
    "packed": Workload("packed", -1, 1024, 8, 16384, "bf16", "f32", 2,
                       "64 images with patch grids h,w ~ U{16..96} concatenated (offsets[65]); "
                       "D=1024, L=8, K=16384; same generative model as 'image'"),
    "offline": Workload("offline", 1 << 20, 256, 4, 65536, "bf16", "f32", 3,
                        "N=2^20 bf16 vectors, D=256, L=4, K=65536; level-0 codebook = 65536 "
                        "mixture centres ~N(0,I); level l>=1 ~N(0,(0.1*0.5^(l-1))^2); features = "
                        "centre + N(0,0.1^2) and, on a seeded 1% of rows, + N(0,0.5^2) tail"),
    "detok": Workload("detok", 1 << 20, 1024, 8, 16384, "f32", "bf16", 4,
                      "ids [2^20, 8]: level 0 Zipf(1.1) over 16384 ranks, levels 1..7 uniform; "
                      "bf16 codebooks [8,16384,1024] ~N(0,(0.5^l)^2); decode -> fp32 recon, "
                      "which is re-encoded"),
}


def spec(name: str) -> Workload:
    return WORKLOADS[name]


# ---------------------------------------------------------------- bf16 storage

def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returns float32.

    Storage conversion of generated inputs only.  NaN/Inf never occur here."""
    a = np.array(a, dtype=np.float32, copy=True, order="C")
    u = a.view(np.uint32)
    # finite inputs only: the largest finite pattern plus 0x8000 stays below 2^32
    lsb = u >> np.uint32(16)
    lsb &= np.uint32(1)
    lsb += np.uint32(0x7FFF)
    u += lsb
    u &= np.uint32(0xFFFF0000)
    return a


def as_bf16_bits(a: np.ndarray) -> np.ndarray:
    """uint16 payload of float32 values that are already bf16-representable."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    bits = a.view(np.uint32)
    if np.any(bits & np.uint32(0xFFFF)):
        raise ValueError("array holds values that are not bf16-representable")
    return (bits >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _store(a: np.ndarray, dtype: str) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.float32)
    return round_bf16(a) if dtype == "bf16" else a


# ---------------------------------------------------------------- generators

def _normal(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    out = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        out *= np.float32(std)
    return out


def zipf_ids(rng: np.random.Generator, n: int, K: int, s: float) -> np.ndarray:
    """Draw n ids in [0,K) with P(id = r-1) proportional to r^-s (truncated Zipf)."""
    w = np.arange(1, K + 1, dtype=np.float64) ** (-s)
    cdf = np.cumsum(w)
    cdf /= cdf[-1]
    u = rng.random(n)
    ids = np.searchsorted(cdf, u, side="right")
    return np.minimum(ids, K - 1).astype(np.int32)


def _planted_sum(cb: np.ndarray, ids: np.ndarray, chunk: int = 16384) -> np.ndarray:
    """features[n] = sum_l cb[l, ids[n,l]] in float32, ascending l (data synthesis)."""
    N, L = ids.shape
    D = cb.shape[2]
    out = np.empty((N, D), dtype=np.float32)
    for s in range(0, N, chunk):
        e = min(N, s + chunk)
        acc = cb[0][ids[s:e, 0]].copy()
        for l in range(1, L):
            acc += cb[l][ids[s:e, l]]
        out[s:e] = acc
    return out


def generate(name: str, batch: int = 0, n_override: int | None = None) -> dict:
    """Build one workload.

    Returns a dict with
      spec      the Workload record (N realised for 'packed')
      x         float32 [N, D] features (values representable in spec.f_dtype); None for 'detok'
      codebooks float32 [L, K, D] (values representable in spec.cb_dtype)
      offsets   int64 [B+1] image boundaries ('packed'; [0, N] otherwise)
      planted   int32 [N, L] ids used to synthesise the features (or the decode ids for 'detok')
    `batch` selects an independent feature draw with the same codebooks (one per data-parallel
    rank); `n_override` shrinks N for quick tests (same recipe, fewer rows).
    """
    w = WORKLOADS[name]
    cb_rng = np.random.Generator(np.random.PCG64(w.seed))
    x_rng = np.random.Generator(np.random.PCG64([w.seed, 1 + batch]))
    L, K, D = w.L, w.K, w.D

    cb = np.empty((L, K, D), dtype=np.float32)
    if name == "offline":
        cb[0] = _normal(cb_rng, (K, D), 1.0)
        for l in range(1, L):
            cb[l] = _normal(cb_rng, (K, D), 0.1 * 0.5 ** (l - 1))
    else:
        for l in range(L):
            cb[l] = _normal(cb_rng, (K, D), 0.5 ** l)
    if name == "tiny":
        cb[:, 0, :] = 0.0
    cb = _store(cb, w.cb_dtype)

    offsets = None
    if name == "tiny":
        N = n_override or w.N
        planted = x_rng.integers(0, K, size=(N, 1), dtype=np.int64).astype(np.int32)
        x = cb[0][planted[:, 0]] + _normal(x_rng, (N, D), 0.3)
        planted = np.concatenate([planted, np.zeros((N, L - 1), np.int32)], axis=1)
    elif name in ("image", "packed"):
        if name == "packed":
            hw = x_rng.integers(16, 97, size=(64, 2))
            sizes = (hw[:, 0] * hw[:, 1]).astype(np.int64)
            if n_override:
                sizes = np.maximum(1, (sizes * n_override) // int(sizes.sum()))
            offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
            N = int(offsets[-1])
        else:
            N = n_override or w.N
        planted = x_rng.integers(0, K, size=(N, L), dtype=np.int64).astype(np.int32)
        x = _planted_sum(cb, planted)
        x += _normal(x_rng, (N, D), 0.05)
    elif name == "offline":
        N = n_override or w.N
        z = x_rng.integers(0, K, size=N, dtype=np.int64).astype(np.int32)
        x = cb[0][z]
        x += _normal(x_rng, (N, D), 0.1)
        tail = x_rng.random(N) < 0.01
        nt = int(tail.sum())
        x[tail] += _normal(x_rng, (nt, D), 0.5)
        planted = np.zeros((N, L), np.int32)
        planted[:, 0] = z
    elif name == "detok":
        N = n_override or w.N
        planted = np.empty((N, L), np.int32)
        planted[:, 0] = zipf_ids(x_rng, N, K, 1.1)
        planted[:, 1:] = x_rng.integers(0, K, size=(N, L - 1), dtype=np.int64).astype(np.int32)
        x = None
    else:
        raise KeyError(name)

    if x is not None:
        x = _store(x, w.f_dtype)
    if offsets is None:
        offsets = np.array([0, N], dtype=np.int64)
    return {"spec": dataclasses.replace(w, N=N), "x": x, "codebooks": cb,
            "offsets": offsets, "planted": planted}


def sample_rows(N: int, count: int, seed: int, offsets: np.ndarray | None = None) -> np.ndarray:
    """Seeded row sample that always includes the first and last rows and, when given,
    the first and last row of every image; sorted, unique, int64."""
    rng = np.random.Generator(np.random.PCG64([seed, 7]))
    must = [0, N - 1]
    if offsets is not None:
        for a, b in zip(offsets[:-1], offsets[1:]):
            if b > a:
                must += [int(a), int(b) - 1]
    pick = rng.choice(N, size=min(N, max(0, count)), replace=False) if N > 0 else np.array([], np.int64)
    rows = np.unique(np.concatenate([np.asarray(must, np.int64), pick.astype(np.int64)]))
    return rows[(rows >= 0) & (rows < N)]
