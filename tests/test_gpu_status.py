"""Failure detection without a GPU fault: a bounded device wait that nothing
satisfies gives up, the status word records it, the host reads
I8_ERR_TIMEOUT, and the context keeps working."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from int8_mixed_precision_column_b200 import build, native, workloads

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    assert torch.cuda.is_available()
    build.build()
    lib = native.lib()
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    st = lib.int8_selftest_wait_timeout(ws.data_ptr(), ws.numel(), 20000, torch.cuda.current_stream().cuda_stream)
    assert st == 0
    status, where = native.int8_check_status(ws)
    assert status == 4 and where == 0x5E1F  # I8_ERR_TIMEOUT at the self-test's wait
    assert native.int8_check_status(ws)[0] == 0  # the read cleared it
    # the context is still usable: a normal forward runs and reports OK
    p = workloads.toy(seed=0)
    CB, SCB = native.int8_quantize_weight(p.W.cuda())
    Y, idx, n_out, wsf = native.int8_linear_forward(p.X.cuda(), CB, SCB, p.bias.cuda(), 6.0)
    assert native.int8_check_status(wsf)[0] == 0
    assert int(n_out.item()) == 2 and np.isfinite(Y.float().cpu().numpy()).all()


def test_selftest_rejects_bad_arguments():
    lib = native.lib()
    assert lib.int8_selftest_wait_timeout(None, 0, 10, None) == 2
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    assert lib.int8_selftest_wait_timeout(ws.data_ptr(), 256, 0, None) == 1
    assert lib.int8_selftest_wait_timeout(ws.data_ptr(), 256, 3000000, None) == 1
