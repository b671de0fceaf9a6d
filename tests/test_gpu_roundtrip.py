"""cg_roundtrip_host: the layer-pipelined encode + decode of a host-resident cache gives,
bit for bit, the codes, steps, zero points and decoded cache of cg_encode followed by
cg_decode on the whole cache in device memory (the same kernels on one-layer views).
Layer counts 1, 3 and 5 run the two-buffer ring with and without wrapping; block-uniform
(g = 16, 4 bits; g = 8, 16 x d ranges, 3 bits), KIVI (3 bits) and the full-head gauge
(g = 128) each take the pipelined path."""
import numpy as np
import pytest
import torch

from quantization_cg_encode_b200 import cg, synth
from tests.gpu_util import need_gpu

pytestmark = pytest.mark.gpu

CODECS = [
    dict(g=16, bits=4),
    dict(g=8, bits=3, range_cols=128),
    dict(g=16, bits=3, mode=cg.KIVI),
    dict(g=128, bits=4, range_cols=128),
]


def _gauges(L, H, d, g, seed):
    A = synth.gauge_params(L, H, d // g, g, sigma=0.1, seed=seed).cuda()
    G = torch.empty_like(A)
    cg.cg_gauge_build(A, G)
    return G


@pytest.mark.parametrize("L", [1, 3, 5])
@pytest.mark.parametrize("ci", range(len(CODECS)))
def test_roundtrip_host_equals_device_path(L, ci):
    need_gpu()
    B, H, T, d = 1, 2, 256, 128
    codec = cg.codec_desc(**CODECS[ci])
    kvd = cg.kv_desc(L, B, H, T, d)
    kv = synth.kv_cache(L, B, H, T, d, seed=L + 7 * ci, device="cuda", n_outliers=2)
    G = _gauges(L, H, d, codec.g, seed=ci)
    cb, sc = cg.cg_sizes_for(kvd, codec)

    codes = torch.zeros(cb, dtype=torch.uint8, device="cuda")
    scales = torch.zeros(sc, dtype=torch.float16, device="cuda")
    zeros = torch.zeros(sc, dtype=torch.float16, device="cuda")
    out = torch.zeros_like(kv)
    cg.cg_encode(kvd, codec, kv, G, 0, T, codes, scales, zeros)
    cg.cg_decode(kvd, codec, codes, scales, zeros, G, 0, T, out)

    kv_host = kv.cpu().pin_memory()
    out_host = torch.zeros(kv.shape, dtype=torch.bfloat16).pin_memory()
    codes2 = torch.full_like(codes, 0xAB)
    scales2 = torch.full_like(scales, 7.0)
    zeros2 = torch.full_like(zeros, 7.0)
    ws = torch.empty(cg.cg_roundtrip_workspace_size(kvd), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.Stream()
    cg.cg_roundtrip_host(kvd, codec, kv_host, G, codes2, scales2, zeros2, out_host, ws, stream=stream)
    stream.synchronize()
    cg.cg_sync_status()

    assert torch.equal(codes2, codes)
    assert torch.equal(scales2.view(torch.int16), scales.view(torch.int16))
    assert torch.equal(zeros2.view(torch.int16), zeros.view(torch.int16))
    assert torch.equal(out_host.view(torch.int16), out.cpu().view(torch.int16))


def test_roundtrip_host_pageable_buffers_and_stream_order():
    """Pageable host buffers still give the exact result (the copies just do not overlap),
    and work queued on the caller's stream after the call sees the decoded output."""
    need_gpu()
    L, B, H, T, d = 4, 2, 2, 128, 128
    codec = cg.codec_desc(g=16, bits=4)
    kvd = cg.kv_desc(L, B, H, T, d)
    kv = synth.kv_cache(L, B, H, T, d, seed=3, device="cuda", n_outliers=2)
    G = _gauges(L, H, d, 16, seed=3)
    cb, sc = cg.cg_sizes_for(kvd, codec)
    codes = torch.empty(cb, dtype=torch.uint8, device="cuda")
    scales = torch.empty(sc, dtype=torch.float16, device="cuda")
    zeros = torch.empty(sc, dtype=torch.float16, device="cuda")
    ref = torch.empty_like(kv)
    cg.cg_encode(kvd, codec, kv, G, 0, T, codes, scales, zeros)
    cg.cg_decode(kvd, codec, codes, scales, zeros, G, 0, T, ref)

    kv_host = kv.cpu()
    out_host = torch.zeros(kv.shape, dtype=torch.bfloat16)
    ws = torch.empty(cg.cg_roundtrip_workspace_size(kvd), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.Stream()
    codes2 = torch.zeros_like(codes)
    cg.cg_roundtrip_host(kvd, codec, kv_host, G, codes2, scales, zeros, out_host, ws, stream=stream)
    with torch.cuda.stream(stream):
        again = torch.empty_like(kv)
        cg.cg_decode(kvd, codec, codes2, scales, zeros, G, 0, T, again, stream=stream)  # ordered after the call
    stream.synchronize()
    cg.cg_sync_status()
    assert torch.equal(codes2, codes)
    assert np.array_equal(out_host.view(torch.int16).numpy(), ref.cpu().view(torch.int16).numpy())
    assert torch.equal(again.view(torch.int16), ref.view(torch.int16))
