"""The bounded waits on the GPU: a wait that cannot complete (an mbarrier
nothing arrives on) gives up after its limit, the kernel returns, the
device status word reports the timeout, and the context keeps working."""
import time

import pytest
import torch

import sparse_decode_attention_basiskv_b200 as bkv
from sparse_decode_attention_basiskv_b200 import synth

from harness import gpu_layer, status_clean

pytestmark = pytest.mark.gpu


def test_wait_that_cannot_complete_times_out_and_context_survives():
    status_clean()
    t0 = time.perf_counter()
    bkv.basiskv_selftest_bounded_wait(2_000_000)  # 2 ms
    flags = bkv.read_device_status()
    elapsed = time.perf_counter() - t0
    assert flags & bkv.DEV_TIMEOUT, f"status {flags:#x}"
    assert elapsed < 5.0
    assert bkv.read_device_status() == 0  # reading cleared it
    # the context still runs a decode step
    wl = synth.with_sizes(synth.TINY, B=2)
    pb, layer = gpu_layer(wl)
    y = layer.decode(pb.q, max_seq_len=wl.T)
    torch.cuda.synchronize()
    status_clean()
    assert torch.isfinite(y.float()).all()
