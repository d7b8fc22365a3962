"""The bounded-wait failure path on the GPU, without a fault: a wait that
nothing completes gives up after its budget, the timeout reaches the host
through the status word, and the context keeps working afterwards."""
from __future__ import annotations

import numpy as np
import pytest
import torch

SA_ERR_TIMEOUT = -6


@pytest.mark.gpu
def test_bounded_wait_times_out_and_context_survives():
    import banded_log_domain_b200 as sa
    from tests import parity

    ws = torch.zeros(64, dtype=torch.int32, device="cuda")  # a 256-byte status header
    assert sa.sinkhorn_attn_poll(ws) == 0
    assert sa.sinkhorn_attn_debug_timeout(ws, 200_000) == 0
    assert sa.sinkhorn_attn_poll(ws) == SA_ERR_TIMEOUT
    assert sa.sinkhorn_attn_poll(ws) == 0  # poll resets the word

    # the same context still runs the path and matches the oracle
    x = parity.draw_case(1, 2, 200, dtype="f32", seed=5, mask_kind="holes")
    g = parity.gpu_run(x, W=17, eps=1.0, T=4, R=2)
    r = parity.oracle_run(x, W=17, eps=1.0, T=4, R=2)
    parity.compare(x, g, r, dtype="f32", dustbin=False, label="after timeout")


def test_timeout_hook_rejects_bad_workspace():
    import ctypes

    import banded_log_domain_b200 as sa

    lib = sa.load()
    # misaligned, and plain host memory (not device memory of the current device)
    assert lib.sinkhorn_attn_debug_timeout(ctypes.c_void_p(0x1001), 1000, None) == -1
    buf = ctypes.create_string_buffer(512)
    addr = (ctypes.addressof(buf) + 15) & ~15
    assert lib.sinkhorn_attn_debug_timeout(ctypes.c_void_p(addr), 1000, None) == -1
