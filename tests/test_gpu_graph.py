"""CUDA-graph capture of the codec calls: a rolling-append decode step (KIVI
encode of one 128-token chunk, then decode of the cache) and a block-uniform
encode + decode round trip are captured once and replayed on new input data;
every replay must give bit-identical outputs to the same calls made eagerly.
The entry points are called once before capture (their first call on a device
looks up device addresses and the tensor-map encoder)."""
import pytest
import torch

from quantization_cg_encode_b200 import cg, synth
from tests.gpu_util import need_gpu

pytestmark = pytest.mark.gpu


def _gauge(L, H, g=16, seed=0):
    A = synth.gauge_params(L, H, 128 // g, g, sigma=0.1, seed=seed).cuda()
    G = torch.empty_like(A)
    cg.cg_gauge_build(A, G)
    return G


def test_captured_kivi_append_step_replays_exactly():
    need_gpu()
    L, B, H, T, d = 4, 1, 8, 2048, 128
    kvd = cg.kv_desc(L, B, H, T, d)
    codec = cg.codec_desc(g=16, bits=3, mode=cg.KIVI)
    G = _gauge(L, H, seed=1)
    kv = synth.kv_cache(L, B, H, T, d, seed=1, device="cuda")
    codes, scales, zeros = cg.alloc_encoded(kvd, codec)
    out = torch.empty_like(kv)
    t0 = T - 128
    cg.cg_encode(kvd, codec, kv, G, 0, T, codes, scales, zeros)  # history, and first (uncaptured) calls

    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        cg.cg_encode(kvd, codec, kv, G, t0, 128, codes, scales, zeros)
        cg.cg_decode(kvd, codec, codes, scales, zeros, G, 0, T, out)
    for step in range(3):
        new = synth.kv_cache(L, B, H, T, d, seed=10 + step, device="cuda")
        kv[..., t0:, :].copy_(new[..., t0:, :])  # the new chunk lands in the captured input buffer
        graph.replay()
        torch.cuda.synchronize()
        cg.cg_sync_status()
        got = (codes.clone(), scales.clone(), zeros.clone(), out.clone())
        # the same step, eagerly
        cg.cg_encode(kvd, codec, kv, G, t0, 128, codes, scales, zeros)
        cg.cg_decode(kvd, codec, codes, scales, zeros, G, 0, T, out)
        cg.cg_sync_status()
        for a, b in zip(got, (codes, scales, zeros, out)):
            assert torch.equal(a, b), "replay differs from the eager step %d" % step
    del graph


def test_captured_block_uniform_round_trip_replays_exactly():
    need_gpu()
    L, B, H, T, d = 4, 1, 8, 1024, 128
    kvd = cg.kv_desc(L, B, H, T, d)
    codec = cg.codec_desc(g=16, bits=4)
    G = _gauge(L, H, seed=2)
    kv = synth.kv_cache(L, B, H, T, d, seed=2, device="cuda")
    codes, scales, zeros = cg.alloc_encoded(kvd, codec)
    out = torch.empty_like(kv)
    cg.cg_encode(kvd, codec, kv, G, 0, T, codes, scales, zeros)
    cg.cg_decode(kvd, codec, codes, scales, zeros, G, 0, T, out)
    cg.cg_sync_status()
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        cg.cg_encode(kvd, codec, kv, G, 0, T, codes, scales, zeros)
        cg.cg_decode(kvd, codec, codes, scales, zeros, G, 0, T, out)
    kv.copy_(synth.kv_cache(L, B, H, T, d, seed=3, device="cuda"))
    graph.replay()
    torch.cuda.synchronize()
    cg.cg_sync_status()
    got = (codes.clone(), scales.clone(), zeros.clone(), out.clone())
    cg.cg_encode(kvd, codec, kv, G, 0, T, codes, scales, zeros)
    cg.cg_decode(kvd, codec, codes, scales, zeros, G, 0, T, out)
    cg.cg_sync_status()
    for a, b in zip(got, (codes, scales, zeros, out)):
        assert torch.equal(a, b)
    del graph
