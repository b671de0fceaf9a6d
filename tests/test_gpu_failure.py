"""Failure reporting on the GPU, without a fault: a bounded device wait that
runs out ends its kernel normally, records the timeout in the device status
word, and the next cg_sync_status reports CG_ERR_TIMEOUT; the device stays
usable and the status is cleared once read."""
import numpy as np
import pytest
import torch

from quantization_cg_encode_b200 import cg, synth
from tests.gpu_util import bf16_np, block_uniform_np, need_gpu, oracle_quantize_own, run_encode

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_reports():
    need_gpu()
    cg.cg_sync_status()  # nothing pending before the test
    result = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    cg.cg_selftest_wait_timeout(50_000_000, result)  # 50 ms limit on a barrier nothing completes
    with pytest.raises(cg.CgError) as e:
        cg.cg_sync_status()
    assert e.value.status == cg.CG_ERR_TIMEOUT
    assert int(result.item()) == 0, "the wait must give up, not complete"
    cg.cg_sync_status()  # cleared once reported

    # the context is intact: a normal encode runs and matches the oracle
    kv = synth.kv_cache(1, 1, 2, 256, 128, seed=2, device="cuda")
    G = synth.identity_gauge(1, 2, 8, 16, device="cuda")
    codec = cg.codec_desc(g=16, bits=4)
    codes, scales, zeros, gauged = run_encode(kv, G, codec)
    ref = oracle_quantize_own(gauged.cpu().numpy().astype(np.float64), 4, 16)
    c, s, z = block_uniform_np(codes, scales, zeros, kv.shape, codec)
    assert np.array_equal(c, ref["codes"])
    assert np.array_equal(gauged.cpu().numpy(), bf16_np(kv))


def test_timeout_reported_on_its_own_stream():
    """The status word is read after synchronizing the given stream."""
    need_gpu()
    st = torch.cuda.Stream()
    result = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    cg.cg_selftest_wait_timeout(5_000_000, result, stream=st)
    with pytest.raises(cg.CgError) as e:
        cg.cg_sync_status(stream=st)
    assert e.value.status == cg.CG_ERR_TIMEOUT
    cg.cg_sync_status(stream=st)
