"""Seeded synthetic inputs for the CSA / HCA workloads.

This module serves both the CUDA path and the FP64 oracle and holds none of
the method's arithmetic: it only draws random numbers and rounds them to the
storage type. numpy only.

Recipe. Every tensor is viewed as rows of its last dimension. Rows are drawn
in chunks of ``CHUNK_ROWS``; chunk j of tensor ``name`` uses the PCG64 stream
``numpy.random.default_rng([seed, tag(name), j])`` and
``standard_normal(dtype=float32)``, multiplied by the tensor's standard
deviation in FP32, then rounded once to BF16 (nearest, ties to even) for BF16
tensors. Any subset of rows can thus be regenerated without drawing the rest.
``N(0, v)`` in the workload descriptions is read with v the variance.
"""
from __future__ import annotations

import math
import os
import zlib
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

CHUNK_ROWS = 4096


def _tag(name: str) -> int:
    return zlib.crc32(name.encode()) & 0x7FFFFFFF


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round FP32 values to BF16 (nearest, ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclass
class Spec:
    """One synthetic tensor: name, shape, standard deviation, storage type."""
    name: str
    shape: tuple
    std: float
    dtype: str  # "bf16" or "f32"
    seed: int

    @property
    def width(self) -> int:
        return int(self.shape[-1])

    @property
    def nrows(self) -> int:
        return int(np.prod(self.shape[:-1], dtype=np.int64)) if len(self.shape) > 1 else 1

    def _chunk(self, j: int) -> np.ndarray:
        r0 = j * CHUNK_ROWS
        n = min(CHUNK_ROWS, self.nrows - r0)
        rng = np.random.default_rng([self.seed, _tag(self.name), j])
        v = rng.standard_normal((n, self.width), dtype=np.float32)
        v *= np.float32(self.std)
        if self.dtype == "bf16":
            v = bf16_bits_to_f32(f32_to_bf16_bits(v))
        return v

    def _fill(self, out: np.ndarray, convert) -> np.ndarray:
        n = self.nrows
        nchunks = math.ceil(n / CHUNK_ROWS)

        def one(j):
            out[j * CHUNK_ROWS:(j + 1) * CHUNK_ROWS] = convert(self._chunk(j))

        if nchunks > 4:
            with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
                list(ex.map(one, range(nchunks)))
        else:
            for j in range(nchunks):
                one(j)
        return out.reshape(self.shape)

    def values(self) -> np.ndarray:
        """All values as float32 (exactly representable in the storage type)."""
        return self._fill(np.empty((self.nrows, self.width), np.float32), lambda v: v)

    def rows(self, flat_rows) -> np.ndarray:
        """Values of the given flat row indices (rows of the last dim)."""
        flat_rows = np.asarray(flat_rows, dtype=np.int64)
        out = np.empty((flat_rows.size, self.width), np.float32)
        chunks = flat_rows // CHUNK_ROWS
        for j in np.unique(chunks):
            sel = np.nonzero(chunks == j)[0]
            out[sel] = self._chunk(int(j))[flat_rows[sel] - j * CHUNK_ROWS]
        return out

    def storage(self) -> np.ndarray:
        """Stored representation: uint16 BF16 bits or float32 values."""
        if self.dtype == "bf16":
            return self._fill(np.empty((self.nrows, self.width), np.uint16),
                              lambda v: (v.view(np.uint32) >> 16).astype(np.uint16))
        return self.values()


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------
@dataclass
class Workload:
    name: str
    kind: str            # "csa_prefill", "csa_decode", "hca_prefill"
    seed: int
    dtype: str           # "f32" or "bf16"
    d: int = 4096
    c: int = 512
    c_I: int = 128
    H_I: int = 64
    H_q: int = 64
    rope_dims: int = 64
    m: int = 4
    k: int = 1024
    n_win: int = 128
    T: int = 0           # prefill tokens
    B: int = 0           # decode batch
    L: int = 0           # decode context (query position)
    kv_mixed: bool = False
    extra: dict = field(default_factory=dict)

    # ---- derived sizes ----
    @property
    def overlap(self) -> int:
        return 1 if self.kind != "hca_prefill" else 0

    @property
    def n_entries(self) -> int:
        if self.kind == "csa_decode":
            return self.L // self.m
        return self.T // self.m

    def spec(self, name, shape, std, dtype=None) -> Spec:
        return Spec(name, tuple(int(s) for s in shape), float(std), dtype or self.dtype, self.seed)

    def specs(self) -> dict:
        """All input tensors of the workload, keyed by name."""
        d, c, cI, HI, Hq, m = self.d, self.c, self.c_I, self.H_I, self.H_q, self.m
        wstd = 1.0 / math.sqrt(d)
        bstd = math.sqrt(0.02)
        s = {}
        if self.kind == "csa_prefill":
            T = self.T
            s["H"] = self.spec("H", (T, d), 1.0)
            for nm in ("W_aKV", "W_bKV", "W_aZ", "W_bZ"):
                s[nm] = self.spec(nm, (d, c), wstd)
            s["bias"] = self.spec("bias", (2 * m, c), bstd, "f32")
            for nm in ("WI_aKV", "WI_bKV", "WI_aZ", "WI_bZ"):
                s[nm] = self.spec(nm, (d, cI), wstd)
            s["biasI"] = self.spec("biasI", (2 * m, cI), bstd, "f32")
            s["qI"] = self.spec("qI", (T, HI, cI), 1.0)
            s["w"] = self.spec("w", (T, HI), 1.0, "f32")
            s["q"] = self.spec("q", (T, Hq, c), 1.0)
            s["kv_win"] = self.spec("kv_win", (T, c), 1.0)
            s["sink"] = self.spec("sink", (Hq,), 1.0, "f32")
        elif self.kind == "hca_prefill":
            T = self.T
            s["H"] = self.spec("H", (T, d), 1.0)
            s["W_KV"] = self.spec("W_KV", (d, c), wstd)
            s["W_Z"] = self.spec("W_Z", (d, c), wstd)
            s["bias"] = self.spec("bias", (m, c), 1.0, "f32")
            s["q"] = self.spec("q", (T, Hq, c), 1.0)
            s["kv_win"] = self.spec("kv_win", (T, c), 1.0)
            s["sink"] = self.spec("sink", (Hq,), 1.0, "f32")
        elif self.kind == "csa_decode":
            B, N = self.B, self.n_entries
            s["E_raw"] = self.spec("E_raw", (B, N, c), 1.0, "bf16")
            s["KI"] = self.spec("KI", (B, N, cI), 1.0)
            s["win_raw"] = self.spec("win_raw", (B, self.n_win, c), 1.0)
            s["q"] = self.spec("q", (B, Hq, c), 1.0)
            s["qI"] = self.spec("qI", (B, HI, cI), 1.0)
            s["w"] = self.spec("w", (B, HI), 1.0, "f32")
            s["sink"] = self.spec("sink", (Hq,), 1.0, "f32")
            # decode-time compressor of the new token (main and index keys)
            s["h"] = self.spec("h", (B, d), 1.0)
            for nm in ("W_aKV", "W_bKV", "W_aZ", "W_bZ"):
                s[nm] = self.spec(nm, (d, c), wstd)
            s["bias"] = self.spec("bias", (2 * m, c), bstd, "f32")
            for nm in ("WI_aKV", "WI_bKV", "WI_aZ", "WI_bZ"):
                s[nm] = self.spec(nm, (d, cI), wstd)
            s["biasI"] = self.spec("biasI", (2 * m, cI), bstd, "f32")
        else:
            raise ValueError(self.kind)
        return s

    def positions(self) -> np.ndarray:
        if self.kind == "csa_decode":
            return np.full(self.B, self.L, np.int64)
        return np.arange(self.T, dtype=np.int64)


def tiny_csa_fp32(**kw) -> Workload:
    """Tiny CSA, FP32, T=1024, d=256, c=128, c_I=32, 4 indexer heads,
    8 query heads, RoPE 32, top-k 32, window 128, seed 0."""
    a = dict(name="tiny_csa_fp32", kind="csa_prefill", seed=0, dtype="f32", T=1024, d=256,
             c=128, c_I=32, H_I=4, H_q=8, rope_dims=32, m=4, k=32, n_win=128)
    a.update(kw)
    return Workload(**a)


def csa_prefill_bf16(**kw) -> Workload:
    """CSA prefill, BF16, T=8192, d=4096, c=512, 64x128 indexer, 64 query
    heads x 512, top-k 1024, window 128, seed 1."""
    a = dict(name="csa_prefill_bf16", kind="csa_prefill", seed=1, dtype="bf16", T=8192)
    a.update(kw)
    return Workload(**a)


def csa_decode_bf16(**kw) -> Workload:
    """CSA decode, BF16, 32 sequences at position 131072 (32768 entries
    each), 64 query heads x 512, 64x128 indexer, top-k 1024, seed 2."""
    a = dict(name="csa_decode_bf16", kind="csa_decode", seed=2, dtype="bf16", B=32, L=131072)
    a.update(kw)
    return Workload(**a)


def hca_prefill_bf16(**kw) -> Workload:
    """HCA prefill, BF16, T=65536, m'=128 without overlap, 512 entries of
    width 512, 64 query heads, seed 3."""
    a = dict(name="hca_prefill_bf16", kind="hca_prefill", seed=3, dtype="bf16", T=65536, m=128)
    a.update(kw)
    return Workload(**a)


def csa_decode_long_mixed(**kw) -> Workload:
    """Long-context CSA decode: 4 sequences at position 1,048,576 (262,144
    entries each) stored as FP8 E4M3 + per-row scale + BF16 RoPE dims;
    BF16 index keys, seed 4."""
    a = dict(name="csa_decode_long_mixed", kind="csa_decode", seed=4, dtype="bf16", B=4,
             L=1048576, kv_mixed=True)
    a.update(kw)
    return Workload(**a)


WORKLOADS = {
    "tiny_csa_fp32": tiny_csa_fp32,
    "csa_prefill_bf16": csa_prefill_bf16,
    "csa_decode_bf16": csa_decode_bf16,
    "hca_prefill_bf16": hca_prefill_bf16,
    "csa_decode_long_mixed": csa_decode_long_mixed,
}


def random_topk_indices(rng: np.random.Generator, n_vis: np.ndarray, k: int,
                        hole_frac: float = 0.0) -> np.ndarray:
    """A valid top-k index input: per row, min(k, n_vis) distinct entries of
    [0, n_vis) in ascending order, padded with -1; ``hole_frac`` of the kept
    slots are then replaced by -1 (entries a caller chose not to read)."""
    n_vis = np.asarray(n_vis, dtype=np.int64)
    out = np.full((n_vis.size, k), -1, np.int32)
    for i, nv in enumerate(n_vis):
        ke = int(min(k, nv))
        if ke <= 0:
            continue
        sel = np.sort(rng.choice(int(nv), size=ke, replace=False)).astype(np.int32)
        if hole_frac > 0:
            sel[rng.random(ke) < hole_frac] = -1
        out[i, :ke] = sel
    return out
