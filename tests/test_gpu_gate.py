"""GPU parity of the decompressed-space gate (ic_decompress_gate) against the
float64 oracle: per-head wv_b up-projection of the latent attention output,
then the sigmoid gate. Error per (b, h) row: max |gpu - ref| / max |ref|."""
import numpy as np
import pytest
import torch

from oracle import gate_oracle as G
from lightning_indexer_cross_b200 import workloads as W

pytestmark = pytest.mark.gpu

# bf16 inputs, fp32 accumulation over 512 products: far below 1e-4 of the
# row's largest value; a bf16 output adds its rounding (2^-9)
TOL = {torch.float32: 1e-4, torch.bfloat16: 6e-3}


def _row_err(out, ref):
    got = out.double().cpu().numpy()
    scale = np.maximum(np.abs(ref).max(axis=-1), 1e-30)
    return float((np.abs(got - ref).max(axis=-1) / scale).max())


@pytest.mark.parametrize("B,H", [(1, 1), (32, 128), (200, 8), (129, 3)])
@pytest.mark.parametrize("odt", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("gate", [True, False])
def test_decompress_gate_matches_oracle(cuda_dev, B, H, odt, gate):
    from lightning_indexer_cross_b200 import ops
    o, w, g = W.gate_case(B, H, gate=gate, seed=80 + B + H, device=cuda_dev)
    out = ops.decompress_gate(o, w, g, out_dtype=odt)
    torch.cuda.synchronize()
    ref = G.decompressed_gate(o, w, g)
    assert _row_err(out, ref) <= TOL[odt]
