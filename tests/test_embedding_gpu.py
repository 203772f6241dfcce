"""embedding_4bit on the GPU against the CPU oracle: bit-exact.

"mps-bitsandbytes 0.4.7", Quantized Embeddings (Embedding4bit): rows of a
[V, D] table quantized as one flat array, dequantized.  Row widths with
D % 16 == 0 take the vector path; others (rows starting inside a byte) the
per-element path.  An index out of range gives zeros and is reported by
bnb4_device_status.
"""
import numpy as np
import pytest
import torch

import bit_blockwise_weight_b200 as bnb4
import oracle
import synthetic

from gpu_util import to_host

pytestmark = pytest.mark.gpu

INDEX = 10  # BNB4_ERR_INDEX


@pytest.mark.parametrize("q", ["nf4", "fp4"])
@pytest.mark.parametrize("out", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("V,D,B", [(1000, 64, 64), (300, 4096, 64), (500, 48, 64), (97, 13, 64),
                                   (200, 100, 128), (64, 1024, 1024)])
def test_matches_oracle(q, out, V, D, B):
    table = synthetic.normal((V * D,), V + D, 0.02, "f32").numpy()
    packed, absmax = oracle.quantize(table, "f32", B, q)
    idx = np.random.default_rng(D).integers(0, V, 777).astype(np.int64)
    idx[:3] = [0, V - 1, 0]
    got = bnb4.embedding_4bit(torch.from_numpy(packed).cuda(), torch.from_numpy(absmax).cuda(), V, D,
                              torch.from_numpy(idx).cuda(), B, q, dtype=synthetic.TORCH_DTYPES[out])
    want = oracle.embedding_4bit(packed, absmax, V, D, B, q, idx, out)
    g = to_host(got).reshape(want.shape)
    assert g.dtype == want.dtype and np.array_equal(g.view(np.uint8), want.view(np.uint8))
    assert bnb4.device_status() == bnb4.STATUS_OK


def test_out_of_range_index_is_reported():
    V, D, B = 50, 64, 64
    table = synthetic.normal((V * D,), 3, 0.02, "f32").numpy()
    packed, absmax = oracle.quantize(table, "f32", B, "nf4")
    idx = torch.tensor([1, V, 2, -1], dtype=torch.int64, device="cuda")
    assert bnb4.device_status() == bnb4.STATUS_OK
    got = to_host(bnb4.embedding_4bit(torch.from_numpy(packed).cuda(), torch.from_numpy(absmax).cuda(), V, D,
                                      idx, B, "nf4", dtype=torch.float32))
    assert bnb4.device_status() == INDEX
    assert bnb4.device_status() == bnb4.STATUS_OK   # cleared by the read
    assert np.all(got[1] == 0) and np.all(got[3] == 0)
    want = oracle.embedding_4bit(packed, absmax, V, D, B, "nf4", [1, 2], "f32")
    assert np.array_equal(got[[0, 2]], want)
