"""The algorithmic work that bench.py's rooflines divide by (CPU): the
prefill indexer's FLOPs against the oracle's own visibility rule, the decode
indexer's bytes against the workload's tensors."""
import sys
from pathlib import Path

import numpy as np

ROOT = Path(__file__).resolve().parents[1]
if str(ROOT) not in sys.path:
    sys.path.insert(0, str(ROOT))

import bench  # noqa: E402
import compressed_sparse_attention_17_b200 as csa  # noqa: E402
from compressed_sparse_attention_17_b200 import synth  # noqa: E402


def test_prefill_indexer_flops_follow_visibility(orc):
    w = synth.csa_prefill_bf16()
    pre = bench.Prefill.__new__(bench.Prefill)  # the count needs no device buffers
    pre.w, pre.g = w, csa.geom(c=w.c, rope_dims=w.rope_dims)
    pairs = sum(orc.visible_entries(t, w.m, 1, w.T // w.m) for t in range(w.T))
    # token t sees floor((t + 1) / 4) entries: sum over u = 1..8192 of floor(u / 4)
    assert pairs == 4 * (2047 * 2048 // 2) + 2048
    assert pre.index_flops() == pairs * 2 * w.H_I * w.c_I  # one multiply-add per (head, dim)


def test_decode_indexer_bytes_are_the_tensors_read():
    w = synth.csa_decode_bf16()
    dec = bench.Decode.__new__(bench.Decode)
    dec.w = w
    s = w.specs()
    keys = int(np.prod(s["KI"].shape)) * 2          # every cached index key, BF16
    queries = int(np.prod(s["qI"].shape)) * 2       # q^I, BF16
    weights = int(np.prod(s["w"].shape)) * 4        # w, FP32
    selected = w.B * w.k * 4                        # the int32 indices written
    assert dec.index_bytes() == keys + queries + weights + selected
    assert keys == 32 * 32768 * 128 * 2


def test_decode_attention_bytes_are_the_rows_read():
    w = synth.csa_decode_bf16()
    dec = bench.Decode.__new__(bench.Decode)
    dec.w = w
    # 32 queries x (1024 selected + 128 window) rows of 512 BF16, queries in and outputs out
    assert dec.attend_bytes() == 32 * 1152 * 1024 + 2 * (32 * 64 * 512 * 2)
    mixed = synth.csa_decode_long_mixed()
    dec.w = mixed
    # selected rows in the 592-byte mixed format, window rows in BF16
    assert dec.attend_bytes() == 4 * (1024 * 592 + 128 * 1024) + 2 * (4 * 64 * 512 * 2)
