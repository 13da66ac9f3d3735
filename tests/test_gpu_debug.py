"""Failure detection without a fault, on the GPU: a bounded mbarrier wait that
nothing satisfies expires, records SSA_ERR_TIMEOUT in the device error word,
and the context stays usable for the next calls.
"""
import pytest
import torch

from parity import BF16_MAX_ABS, out_errors
from workloads import planted_prefill, to_f64

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def test_bounded_wait_expires_and_context_survives():
    import block_sparse_top_summary_b200 as ssa
    assert ssa.ssa_device_error() == 0
    ssa.ssa_debug_wait_timeout(2000)  # 2 ms
    assert ssa.ssa_device_error() == 4  # SSA_ERR_TIMEOUT, then reset
    assert ssa.ssa_device_error() == 0
    # the context still runs the hot path correctly
    Q, K, V = planted_prefill(1, 8, 2, 64 * 6, 128, 64, 2, seed=4, dtype="bf16")
    out, _, idx, cnt, _ = ssa.prefill(Q.cuda(), K.cuda(), V.cuda(), 64, 2)
    import oracle as O
    ref, _ = O.sparse_attention(to_f64(Q), to_f64(K), to_f64(V), idx.cpu().numpy(),
                                cnt.cpu().numpy(), 64)
    ma, _ = out_errors(to_f64(out), ref)
    assert ma <= BF16_MAX_ABS
    assert ssa.ssa_device_error() == 0


def test_stream_ordered_error_check():
    # The same expired wait, read back in the order of the stream it ran on,
    # waiting for that stream only.
    import block_sparse_top_summary_b200 as ssa
    assert ssa.ssa_device_error() == 0
    side = torch.cuda.Stream()
    ssa.ssa_debug_wait_timeout(2000, stream=side)
    assert ssa.ssa_check_device_error(side) == 4  # SSA_ERR_TIMEOUT, then reset
    assert ssa.ssa_check_device_error(side) == 0
    assert ssa.ssa_check_device_error() == 0  # the current stream
    assert ssa.ssa_device_error() == 0
