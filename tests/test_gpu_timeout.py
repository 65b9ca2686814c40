"""Device failure path: a bounded wait that gives up.

Every wait inside the kernels is bounded (ic_set_wait_limit_ns, 2 s by
default). With the bound set to 0 a wait that is not already satisfied gives
up at once, so the kernel takes its failure path: it records IC_ERR_TIMEOUT,
writes nothing, lets its own copies and MMAs in flight finish and frees its
tensor memory. The call must still return (the stream synchronises), the
status word must read IC_ERR_TIMEOUT, and a following call with the default
bound and a freshly zeroed workspace must be correct against the oracle. No
GPU fault is involved: the failure is a wait that the host told to give up.

The decompressed-space gate kernel is the one run here (the simplest
producer / MMA / epilogue pipeline; its abort path was checked by reading:
every role leaves its loop on the abort flag, the producer drains the loads
it issued, and the accumulator is freed after the issuer's final commit)."""
import numpy as np
import pytest
import torch

from oracle import gate_oracle as G
from lightning_indexer_cross_b200 import workloads as W

pytestmark = pytest.mark.gpu


def test_wait_limit_zero_gives_timeout_status_and_the_next_call_is_correct(cuda_dev):
    from lightning_indexer_cross_b200 import _abi, ops
    o, w, g = W.gate_case(256, 16, gate=True, seed=501, device=cuda_dev)
    ws = ops.new_workspace(_abi.ic_decompress_gate_workspace_size(), cuda_dev)
    out = torch.full((256, 16, 128), 7.0, dtype=torch.float32, device=cuda_dev)
    default = _abi.ic_wait_limit_ns()
    assert default == 2_000_000_000
    try:
        _abi.ic_set_wait_limit_ns(0)
        ops.decompress_gate(o, w, g, out=out, workspace=ws)
    finally:
        _abi.ic_set_wait_limit_ns(default)
    # synchronises the stream (the kernel returned) and reads the status word
    assert _abi.ic_last_device_status(ops._ptr(ws), ops._stream_ptr()) == _abi.IC_ERR_TIMEOUT
    torch.cuda.synchronize()
    ws.zero_()
    out.fill_(7.0)
    ops.decompress_gate(o, w, g, out=out, workspace=ws)
    assert _abi.ic_last_device_status(ops._ptr(ws), ops._stream_ptr()) == _abi.IC_OK
    ref = G.decompressed_gate(o, w, g)
    got = out.double().cpu().numpy()
    scale = np.maximum(np.abs(ref).max(axis=-1), 1e-30)
    assert float((np.abs(got - ref).max(axis=-1) / scale).max()) <= 1e-4
