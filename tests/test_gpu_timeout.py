"""Failure detection without a GPU fault: every device-side wait in the kernels
is bounded (about one second of %globaltimer), after which the block raises
its abort flag, records GMLA_ERR_TIMEOUT in the workspace status word and
leaves through its abort path (copies in flight drained, tensor memory freed,
every warp at the final barrier). A test hook makes one decode block wait on a
barrier that nothing completes; the test checks the status, then that the same
device and workspace give a correct decode right after the status is cleared."""
import time

import numpy as np
import pytest
import torch

import oracle
from gpu_pipeline import BF16_TOL, assert_close, run_decode, small_decode

pytestmark = pytest.mark.gpu


def test_decode_wait_that_runs_out_reports_timeout_and_the_device_recovers():
    from gated_mla_b200 import _lib
    inp = small_decode("decode_b32", 4, [300, 1000, 129, 2000])
    gpu = run_decode(inp)
    model, cache = gpu["model"], gpu["cache"]
    q = torch.from_numpy(gpu["q"]).to("cuda", torch.bfloat16)
    g = torch.from_numpy(gpu["glogit"]).to("cuda")
    lens = torch.tensor(inp["lengths"], dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream

    _lib.check(_lib.gmla_test_stall_next_decode(1), "arm the stall")
    t0 = time.perf_counter()
    model.decode(q, g, cache, lens)
    ws = model._ws["decode"]
    st = _lib.gmla_sync_status(ws.data_ptr(), stream)
    waited = time.perf_counter() - t0
    assert st == _lib.GMLA_ERR_TIMEOUT, st
    assert waited >= 0.9, waited          # the bound, not an early exit

    # the context is intact: clear the word and decode again on the same workspace
    _lib.check(_lib.gmla_clear_status(ws.data_ptr(), stream), "clear")
    o = model.decode(q, g, cache, lens)
    model.sync_status()
    o = o.float().cpu().numpy()
    np.testing.assert_array_equal(o, gpu["o"])
    ref = oracle.decode(oracle.params(inp), inp["x"], inp["past"])
    assert_close(o, ref["gated"], BF16_TOL, "gated o after recovery")
