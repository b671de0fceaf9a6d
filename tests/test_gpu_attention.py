"""GPU parity of decode-step attention read from the encoded cache
(cg_decode_attention) against the oracle: the oracle decodes the same codes in
fp64 (G^T (s q + z)) and runs plain softmax attention; the device folds the
gauge into the query and the output.  Tolerance: per (layer, batch, query head)
output vector, norm-relative 1e-4 (fp32 sums over up to 4096 tokens).

Launch geometry: one CTA per (layer, batch, KV head, run of chunks), then one
per (layer, batch, query head) for the merge; the cases cover
one chunk, a last chunk of 16 or 240 tokens, several chunks in one CTA, a layer
range inside the cache, every GQA group size and the 8B-shaped cache (32 layers,
32 query heads over 8 KV heads, 4096 tokens: 1024 CTAs, four partials merged per
query head) on sampled slices.  The launcher picks the chunk size: the small cases
fit one wave of 256-token chunks; the 8B-shaped cache and a ragged 10-layer call
(two 128-token chunks per CTA, a last chunk of 80 tokens) take 128-token chunks."""
import numpy as np
import pytest
import torch

from oracle import attention as oa
from oracle import codec as oc
from quantization_cg_encode_b200 import cg, synth
from tests.gpu_util import bf16_np, block_uniform_np, need_gpu, run_encode

pytestmark = pytest.mark.gpu


def _encoded(L, B, H, T, d, bits, seed):
    kv = synth.kv_cache(L, B, H, T, d, seed=seed, device="cuda", n_outliers=2)
    A = synth.gauge_params(L, H, d // 16, 16, sigma=0.1, seed=seed).cuda()
    G = torch.empty_like(A)
    cg.cg_gauge_build(A, G)
    codec = cg.codec_desc(g=16, bits=bits)
    codes, scales, zeros, _ = run_encode(kv, G, codec, want_gauged=False)
    return kv, G, codec, codes, scales, zeros


def _attend(kv, G, codec, codes, scales, zeros, q, n_tokens, layer0, scale):
    kvd = cg.kv_desc_of(kv)
    at = cg.AttnDesc(q.shape[2], n_tokens, layer0, q.shape[0], scale)
    ws = torch.empty(cg.cg_decode_attention_workspace_size(kvd, at), dtype=torch.uint8, device="cuda")
    out = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
    cg.cg_decode_attention(kvd, codec, at, q, codes, scales, zeros, G, out, ws)
    cg.cg_sync_status()
    return out.cpu().numpy().astype(np.float64)


def _close(got, ref, what):
    g = got.reshape(-1, got.shape[-1])
    r = ref.reshape(g.shape)
    rel = np.sqrt(((g - r) ** 2).sum(-1) / (r ** 2).sum(-1))
    assert rel.max() <= 1e-4, "%s: worst norm-relative error %.3g" % (what, rel.max())


@pytest.mark.parametrize("d,bits,gq,T,n,l0,nl", [
    (128, 4, 4, 512, 512, 0, 2), (128, 4, 4, 1024, 272, 1, 1), (128, 3, 2, 512, 16, 0, 2),
    (128, 8, 1, 768, 768, 0, 1), (64, 4, 8, 512, 496, 0, 2), (64, 6, 2, 256, 256, 1, 1), (128, 2, 4, 512, 512, 0, 2)])
def test_decode_attention_matches_oracle(d, bits, gq, T, n, l0, nl):
    need_gpu()
    L, B, H = 2, 2, 2
    kv, G, codec, codes, scales, zeros = _encoded(L, B, H, T, d, bits, seed=bits + gq + d)
    q = (torch.randn((nl, B, H * gq, d), generator=torch.Generator().manual_seed(3)) * 2).to(torch.bfloat16).cuda()
    scale = 1.0 / np.sqrt(d)
    got = _attend(kv, G, codec, codes, scales, zeros, q, n, l0, scale)
    c, s, z = block_uniform_np(codes, scales, zeros, kv.shape, codec)
    zf = z.view(np.float16).astype(np.float64)
    sf = s.view(np.float16).astype(np.float64)
    ref = oa.decode_attention(bf16_np(q), c, zf, sf, G.cpu().numpy(), bits, n, float(np.float32(scale)), layer0=l0)
    _close(got, ref, "d=%d b=%d gq=%d n=%d" % (d, bits, gq, n))


def test_decode_attention_8b_shaped_cache_sampled():
    need_gpu()
    L, B, H, T, d, Hq = 32, 1, 8, 4096, 128, 32
    kv, G, codec, codes, scales, zeros = _encoded(L, B, H, T, d, 4, seed=9)
    q = torch.randn((L, B, Hq, d), generator=torch.Generator().manual_seed(4)).to(torch.bfloat16).cuda()
    scale = 1.0 / np.sqrt(d)
    got = _attend(kv, G, codec, codes, scales, zeros, q, T, 0, scale)
    c, s, z = block_uniform_np(codes, scales, zeros, kv.shape, codec)
    Gn = G.cpu().numpy().astype(np.float64)
    qn = bf16_np(q)
    rng = np.random.default_rng(5)
    for _ in range(3):
        l, h = int(rng.integers(L)), int(rng.integers(H))
        x = oc.decode_block_uniform(c[l:l + 1, :, :, h:h + 1], z[l:l + 1, :, :, h:h + 1].view(np.float16).astype(np.float64),
                                    s[l:l + 1, :, :, h:h + 1].view(np.float16).astype(np.float64),
                                    Gn[l:l + 1, :, h:h + 1], 4)           # [1, 2, B, 1, T, d]
        ref = oa.softmax_attention(qn[l, :, 4 * h:4 * h + 4], x[0, 0], x[0, 1], float(np.float32(scale)))
        _close(got[l, :, 4 * h:4 * h + 4], ref, "8B slice %s" % ((l, h),))


def test_decode_attention_small_chunks_ragged_sampled():
    """A call too large for one wave of 256-token chunks: 10 layers x 2 batches x 8 KV
    heads over 2000 of 2048 tokens takes 128-token chunks, two per CTA (1280 CTAs),
    with a last chunk of 80 tokens; sampled (layer, batch, KV head) slices against
    the oracle."""
    need_gpu()
    L, B, H, T, d, Hq, n = 10, 2, 8, 2048, 128, 32, 2000
    kv, G, codec, codes, scales, zeros = _encoded(L, B, H, T, d, 4, seed=12)
    q = torch.randn((L, B, Hq, d), generator=torch.Generator().manual_seed(6)).to(torch.bfloat16).cuda()
    scale = 1.0 / np.sqrt(d)
    got = _attend(kv, G, codec, codes, scales, zeros, q, n, 0, scale)
    c, s, z = block_uniform_np(codes, scales, zeros, kv.shape, codec)
    Gn = G.cpu().numpy().astype(np.float64)
    qn = bf16_np(q)
    rng = np.random.default_rng(7)
    for _ in range(3):
        l, h = int(rng.integers(L)), int(rng.integers(H))
        x = oc.decode_block_uniform(c[l:l + 1, :, :, h:h + 1], z[l:l + 1, :, :, h:h + 1].view(np.float16).astype(np.float64),
                                    s[l:l + 1, :, :, h:h + 1].view(np.float16).astype(np.float64),
                                    Gn[l:l + 1, :, h:h + 1], 4)           # [1, 2, B, 1, T, d]
        for b in range(B):
            ref = oa.softmax_attention(qn[l, b:b + 1, 4 * h:4 * h + 4], x[0, 0, b:b + 1, :, :n], x[0, 1, b:b + 1, :, :n],
                                       float(np.float32(scale)))
            _close(got[l, b:b + 1, 4 * h:4 * h + 4], ref, "slice %s" % ((l, b, h),))
