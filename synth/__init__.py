"""Seeded synthetic inputs for the Dense-and-Sparse quantized GEMV.

This module only draws random numbers and lays them out in the storage
format's containers; it holds none of the method's arithmetic (no unpacking,
no table lookups, no dot products).  Both the CUDA path's tests/benchmark and
the CPU oracle's tests take their inputs from here.

Workloads follow the shapes of the SqueezeLLM experiments (LLaMA-7B/13B/65B
linear layers; "SqueezeLLM: Dense-and-Sparse Quantization", §5 Experimental
Analysis, Tables 1 and 3).  No model weights or datasets are used: every
tensor is drawn from the distributions below.

* LUT: per output row, 2**bits draws from N(0, 0.02), rounded to fp16
  (round-to-nearest-even), sorted ascending ("sorted k-means-like"
  centroids).
* Codes: uniform in [0, 2**bits).  The packed format is a contiguous
  LSB-first bitstream along K with no padding, so a stream of uniformly
  random 32-bit words *is* a stream of i.i.d. uniform codes; the words are
  drawn directly and never packed here.
* Outliers: round(p*N*K) distinct positions drawn uniformly without
  replacement, stored in CSR order (row-major, ascending column); values
  are +-U(0.1, 0.5) (fair sign) or 0.1*t(df=3) clamped to the fp16 range,
  rounded to fp16.  The "skew" distribution draws the same number of
  outliers with +-U(0.1, 0.5) values but concentrates them on few rows: row
  counts are multinomial with Zipf weights 1/r over a random order of the
  rows (capped at K, so the heaviest rows are entirely outliers), columns
  uniform without replacement within a row -- a stress case for the
  balanced sparse scheme (the pages state that outliers are unevenly
  spread over rows).
* Activations: x ~ N(0, 1) rounded to fp16.

Every tensor comes from its own PCG64 stream keyed by (seed, workload id,
instance, tensor name), so a layer is reproducible in isolation.
"""
from __future__ import annotations

import dataclasses
import zlib
from typing import Dict, List, Optional, Tuple

import numpy as np

FP16_MAX = 65504.0

_TENSOR_IDS = {"lut": 1, "codes": 2, "pos": 3, "sign": 4, "mag": 5, "x": 6, "rows": 7, "w": 8}


def _rng(seed: int, key: str, instance: int, tensor: str) -> np.random.Generator:
    """Independent PCG64 stream for one tensor of one layer instance."""
    wid = zlib.crc32(key.encode("utf-8"))
    ss = np.random.SeedSequence(entropy=int(seed), spawn_key=(wid, int(instance), _TENSOR_IDS[tensor]))
    return np.random.Generator(np.random.PCG64(ss))


def words_per_row(k_in: int, bits: int) -> int:
    """Number of 32-bit words holding one row of K b-bit codes (no padding)."""
    if (k_in * bits) % 32:
        raise ValueError(f"K={k_in} x {bits} bits is not a whole number of 32-bit words")
    return k_in * bits // 32


def nnz_for(n_out: int, k_in: int, density: float) -> int:
    return int(round(density * n_out * k_in))


@dataclasses.dataclass
class Layer:
    """Host copy of one quantized layer in the canonical storage format.

    codes  uint32 [n_out, k_in*bits/32]  LSB-first bitstream per row
    lut    uint16 [n_out, 2**bits]       fp16 bit patterns
    rowptr int32  [n_out+1]
    col    int32  [nnz]
    val    uint16 [nnz]                  fp16 bit patterns
    """

    n_out: int
    k_in: int
    bits: int
    codes: np.ndarray
    lut: np.ndarray
    rowptr: np.ndarray
    col: np.ndarray
    val: np.ndarray

    @property
    def nnz(self) -> int:
        return int(self.col.shape[0])

    def nbytes(self) -> int:
        return int(self.codes.nbytes + self.lut.nbytes + self.rowptr.nbytes + self.col.nbytes + self.val.nbytes)


def draw_lut(rng: np.random.Generator, n_out: int, bits: int, std: float = 0.02) -> np.ndarray:
    lut = rng.normal(0.0, std, size=(n_out, 1 << bits)).astype(np.float16)
    lut.sort(axis=1)
    return lut.view(np.uint16)


def draw_codes(rng: np.random.Generator, n_out: int, k_in: int, bits: int) -> np.ndarray:
    wpr = words_per_row(k_in, bits)
    return rng.integers(0, 1 << 32, size=(n_out, wpr), dtype=np.uint64).astype(np.uint32)


def draw_outliers(seed: int, key: str, instance: int, n_out: int, k_in: int, density: float,
                  dist: str = "uniform") -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    nnz = nnz_for(n_out, k_in, density)
    if nnz and dist == "skew":
        rr = _rng(seed, key, instance, "rows")
        order = rr.permutation(n_out)
        w = 1.0 / np.arange(1, n_out + 1)
        counts = np.zeros(n_out, dtype=np.int64)
        counts[order] = rr.multinomial(nnz, w / w.sum())
        counts = np.minimum(counts, k_in)
        pr = _rng(seed, key, instance, "pos")
        parts = [i * k_in + np.sort(pr.choice(k_in, size=int(c), replace=False)) for i, c in enumerate(counts) if c]
        pos = np.concatenate(parts).astype(np.int64) if parts else np.zeros(0, dtype=np.int64)
        nnz = int(pos.shape[0])
    elif nnz:
        pos = _rng(seed, key, instance, "pos").choice(n_out * k_in, size=nnz, replace=False)
        pos = np.sort(pos.astype(np.int64))
    else:
        pos = np.zeros(0, dtype=np.int64)
    rows = pos // k_in
    col = (pos % k_in).astype(np.int32)
    rowptr = np.zeros(n_out + 1, dtype=np.int64)
    np.cumsum(np.bincount(rows, minlength=n_out), out=rowptr[1:])
    if dist in ("uniform", "skew"):
        sign = _rng(seed, key, instance, "sign").integers(0, 2, size=nnz) * 2 - 1
        mag = _rng(seed, key, instance, "mag").uniform(0.1, 0.5, size=nnz)
        v = sign * mag
    elif dist == "t3":
        v = 0.1 * _rng(seed, key, instance, "mag").standard_t(3, size=nnz)
        v = np.clip(v, -FP16_MAX, FP16_MAX)
    else:
        raise ValueError(f"unknown outlier distribution {dist!r}")
    val = v.astype(np.float16).view(np.uint16)
    return rowptr.astype(np.int32), col, val


def make_layer(n_out: int, k_in: int, bits: int, density: float, *, seed: int = 0, key: str = "layer",
               instance: int = 0, dist: str = "uniform") -> Layer:
    lut = draw_lut(_rng(seed, key, instance, "lut"), n_out, bits)
    codes = draw_codes(_rng(seed, key, instance, "codes"), n_out, k_in, bits)
    rowptr, col, val = draw_outliers(seed, key, instance, n_out, k_in, density, dist)
    return Layer(n_out, k_in, bits, codes, lut, rowptr, col, val)


def make_weights(n_out: int, k_in: int, *, seed: int = 0, key: str = "weights", instance: int = 0,
                 scale: float = 0.02, df: float = 4.0) -> np.ndarray:
    """Dense fp16 weights for the encoder: scale * Student-t(df) per entry,
    rounded to fp16 (bits as uint16).  Heavy tails give the few extreme
    values per layer that the Dense-and-Sparse split is for."""
    w = scale * _rng(seed, key, instance, "w").standard_t(df, size=(n_out, k_in))
    return w.astype(np.float16).view(np.uint16)


def make_x(batch: int, k_in: int, *, seed: int = 0, key: str = "layer", instance: int = 0) -> np.ndarray:
    x = _rng(seed, key, instance, "x").standard_normal(size=(batch, k_in)).astype(np.float16)
    return x.view(np.uint16)


# --------------------------------------------------------------------------
# Workloads: the layer shapes of the experiments, with the sparsity levels
# and batch sizes the experiments sweep.


@dataclasses.dataclass(frozen=True)
class Shape:
    name: str
    n_out: int
    k_in: int
    bits: int
    density: float
    batch: int = 1
    dist: str = "uniform"

    @property
    def key(self) -> str:
        return f"{self.name}/{self.n_out}x{self.k_in}/b{self.bits}/p{self.density:g}/{self.dist}"


def workloads() -> Dict[str, List[Shape]]:
    """The synthetic workloads (LLaMA-7B/13B/65B linear-layer shapes)."""
    w: Dict[str, List[Shape]] = {}
    w["llama7b-q-4bit"] = [Shape("q_proj", 4096, 4096, 4, 0.0045)]
    w["llama7b-up-3bit"] = [Shape("up_proj", 11008, 4096, 3, 0.0045)]
    sweep = []
    for bits in (3, 4):
        for p in (0.0, 0.0005, 0.0045):
            for nm, n, k in (("qkvo", 4096, 4096), ("gate_up", 11008, 4096), ("down", 4096, 11008)):
                sweep.append(Shape(nm, n, k, bits, p))
    w["llama7b-sweep"] = sweep
    w["llama65b-3bit-t3"] = [Shape(nm, n, k, 3, 0.0005, 1, "t3") for nm, n, k in
                             (("qkvo", 8192, 8192), ("gate_up", 22016, 8192), ("down", 8192, 22016))]
    w["llama13b-batch"] = [Shape(nm, n, k, 3, 0.0045, b) for nm, n, k in
                           (("qkvo", 5120, 5120), ("gate_up", 13824, 5120), ("down", 5120, 13824))
                           for b in (1, 2, 4, 8, 16)]
    # skewed outliers (same counts as the uniform 0.45 % layers, Zipf rows)
    w["llama7b-skew"] = [Shape("up_proj", 11008, 4096, 3, 0.0045, 1, "skew"),
                         Shape("q_proj", 4096, 4096, 4, 0.0045, 1, "skew")]
    return w


def layer_for(shape: Shape, *, seed: int = 0, instance: int = 0) -> Layer:
    return make_layer(shape.n_out, shape.k_in, shape.bits, shape.density, seed=seed, key=shape.key,
                      instance=instance, dist=shape.dist)


def x_for(shape: Shape, *, seed: int = 0, instance: int = 0, batch: Optional[int] = None) -> np.ndarray:
    return make_x(shape.batch if batch is None else batch, shape.k_in, seed=seed, key=shape.key, instance=instance)
