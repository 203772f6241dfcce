"""Pins for the oracle's 4-bit embedding lookup (reading R11), CPU only.

"mps-bitsandbytes 0.4.7", Quantized Embeddings: Embedding4bit.from_embedding
quantizes an embedding table (NF4 by default).  The [V, D] table is quantized
as one flat array; looking up indices returns the dequantized rows.  Pinned
against the exact rational restatement (oracle.bruteforce) of quantize and
dequantize followed by a plain row gather, with row widths that hold whole
blocks and widths whose rows start inside a byte and inside a block.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import bruteforce as bf
import synthetic


def _to_fracs(arr, dtype):
    if dtype == "f32":
        return [Fraction(float(v)) for v in arr]
    conv = bf.f16_bits_to_fraction if dtype == "f16" else bf.bf16_bits_to_fraction
    return [conv(int(v)) for v in arr]


@pytest.mark.parametrize("q", ["nf4", "fp4"])
@pytest.mark.parametrize("D,B", [(12, 4), (13, 4), (64, 64), (24, 8)])
def test_matches_exact_rationals(q, D, B):
    V = 6
    table = synthetic.normal((V * D,), D + B, 0.02, "f32").numpy()
    packed, absmax = oracle.quantize(table, "f32", B, q)
    _, amax_exact, idxs = bf.quantize([Fraction(float(v)) for v in table], B, q)
    idx = np.array([5, 0, 3, 3, 1, 5, 2], np.int64)        # repeats, first and last rows
    for out in ("f32", "f16", "bf16"):
        got = oracle.embedding_4bit(packed, absmax, V, D, B, q, idx, out)
        flat = bf.dequantize(idxs, amax_exact, B, q, out)
        want = [flat[r * D + k] for r in idx for k in range(D)]
        assert got.shape == (idx.size, D)
        assert _to_fracs(got.reshape(-1), out) == want, out


def test_index_checks():
    V, D, B = 4, 8, 4
    packed, absmax = oracle.quantize(synthetic.normal((V * D,), 1, 1.0, "f32").numpy(), "f32", B, "nf4")
    assert oracle.embedding_4bit(packed, absmax, V, D, B, "nf4", np.zeros(0, np.int64), "bf16").shape == (0, D)
    last = oracle.embedding_4bit(packed, absmax, V, D, B, "nf4", [V - 1], "f32")
    assert np.array_equal(last[0], oracle.dequantize(packed, absmax, V * D, B, "nf4", "f32")[-D:])
    for bad in ([V], [-1], [0, V + 3]):
        with pytest.raises(ValueError):
            oracle.embedding_4bit(packed, absmax, V, D, B, "nf4", bad, "f32")


def test_rows_follow_the_indices():
    """Any index list gives the rows of the identity lookup in that order."""
    V, D, B = 50, 64, 64
    packed, absmax = oracle.quantize(synthetic.normal((V * D,), 2, 1.0, "f32").numpy(), "f32", B, "fp4")
    full = oracle.embedding_4bit(packed, absmax, V, D, B, "fp4", np.arange(V), "bf16")
    idx = np.random.default_rng(0).integers(0, V, 300)
    assert np.array_equal(oracle.embedding_4bit(packed, absmax, V, D, B, "fp4", idx, "bf16"), full[idx])
