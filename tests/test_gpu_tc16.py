"""GPU parity of the chain-exact tensor-core g = 16 encoder (engine
CG_ENGINE_CHAIN_TENSOR; d_head = 128, 16 x 16 ranges).

The tensor cores contract with G split exactly into three bf16 terms, and the
encoder re-evaluates the fp32 FMA chain wherever the tensor-core value could
change a zero point, a step or a code.  So codes, steps and zero points must
equal the oracle's (the chain) bit for bit, and equal those of the CUDA-core
engine; the gauged values it reports must lie within 2^-16 max|y| of the chain
over every 16 x 16 block, and equal it wherever it re-evaluated the chain.
"""
import numpy as np
import pytest
import torch

from oracle import codec as oc
from oracle import gauge as og
from quantization_cg_encode_b200 import cg, synth
from tests.gpu_util import assert_close_bf16, bf16_np, block_uniform_np, need_gpu, run_decode, run_encode

pytestmark = pytest.mark.gpu

BOUND = 2.0 ** -16   # documented: |y_tc - y_chain| <= 2^-16 max|y| over the block


def _oracle_G(L, H, sigma=0.1, seed=0):
    A = synth.gauge_params(L, H, 8, 16, sigma=sigma, seed=seed)
    return og.gauge_from_A(A.numpy().astype(np.float64)).astype(np.float32)


def _check(kv, G32, bits, t0=0, nt=None, engine=cg.ENGINE_CHAIN_TENSOR):
    """Encode on the GPU and compare with the oracle; returns (codes, scales, zeros, ref, y_gpu)."""
    T = kv.shape[4]
    nt = T - t0 if nt is None else nt
    G = torch.from_numpy(G32).cuda()
    codec = cg.codec_desc(g=16, bits=bits, engine=engine)
    codes, scales, zeros, gauged = run_encode(kv, G, codec, t0, nt)
    x = bf16_np(kv)
    ref = oc.encode_block_uniform(x, G32.astype(np.float64), bits, t0=t0, nt=nt)
    c, s, z = block_uniform_np(codes, scales, zeros, kv.shape, codec)
    tb0, tb1 = t0 // 16, (t0 + nt) // 16
    assert np.array_equal(z[..., tb0:tb1, :], np.asarray(ref["z"]).astype(np.float16).view(np.uint16)), "zero points"
    assert np.array_equal(s[..., tb0:tb1, :], np.asarray(ref["s"]).astype(np.float16).view(np.uint16)), "steps"
    assert np.array_equal(c[..., tb0:tb1, :, :], ref["codes"]), "codes"
    assert not c[..., :tb0, :, :].any() and not c[..., tb1:, :, :].any(), "codes written outside the range"
    y = gauged.cpu().numpy().astype(np.float64)
    assert np.all(np.isnan(y[..., :t0, :])) and np.all(np.isnan(y[..., t0 + nt:, :])), "gauged written outside"
    return codes, scales, zeros, ref, y[..., t0:t0 + nt, :]


def _block_error(y_gpu, y_ref):
    """max over 16 x 16 blocks of |y_gpu - y_ref| / max|y_ref| (0 for all-zero blocks)."""
    from oracle import quant as oq
    d = oq.block_uniform_view(np.abs(y_gpu - y_ref), 16, 16).max(-1)
    m = oq.block_uniform_view(np.abs(y_ref), 16, 16).max(-1)
    assert np.all(d[m == 0] == 0)
    return float((d[m > 0] / m[m > 0]).max()) if (m > 0).any() else 0.0


@pytest.mark.parametrize("bits", [2, 3, 4, 6, 8])
def test_codes_equal_chain_and_cuda_core_engine(bits):
    need_gpu()
    kv = synth.kv_cache(2, 2, 2, 512, 128, seed=bits, device="cuda", n_outliers=4)
    G32 = _oracle_G(2, 2, seed=bits)
    c_tc, s_tc, z_tc, ref, y_tc = _check(kv, G32, bits)
    err = _block_error(y_tc, ref["y"])
    assert err <= BOUND, "tensor-core gauged values %.3g of the block max from the chain" % err
    c_cc, s_cc, z_cc, _, y_cc = _check(kv, G32, bits, engine=cg.ENGINE_CUDA_CORES)
    assert np.array_equal(y_cc, ref["y"]), "CUDA-core engine must report the chain itself"
    assert torch.equal(c_tc, c_cc) and torch.equal(s_tc, s_cc) and torch.equal(z_tc, z_cc)
    out = run_decode(kv.shape, torch.from_numpy(G32).cuda(), cg.codec_desc(g=16, bits=bits), c_tc, s_tc, z_tc)
    xr = oc.decode_block_uniform(ref["codes"], ref["z"], ref["s"], G32.astype(np.float64), bits)
    assert_close_bf16(bf16_np(out), xr, what="decode of tensor-core codes")


@pytest.mark.parametrize("t0,nt", [(0, 16), (48, 176), (16, 240), (128, 128), (0, 400)])
def test_ragged_token_ranges(t0, nt):
    """Partial 128-token blocks at the end of every head slice; only [t0, t0+nt) is written."""
    need_gpu()
    kv = synth.kv_cache(1, 1, 3, 416, 128, seed=7, device="cuda", n_outliers=2)
    _check(kv, _oracle_G(1, 3, seed=7), 4, t0, nt)


def test_many_blocks_per_cta_and_slice_changes():
    """512 blocks of 128 tokens over 148 SMs: each CTA crosses head slices (G restaged,
    its four TMEM accumulators reused by the three epilogue warpgroups), with a ragged
    tail per slice."""
    need_gpu()
    kv = synth.kv_cache(2, 1, 4, 4096, 128, seed=11, device="cuda", n_outliers=4)
    _, _, _, ref, y = _check(kv, _oracle_G(2, 4, seed=11), 4, 0, 4096 - 48)
    assert _block_error(y, ref["y"]) <= BOUND


def test_rounding_ties_and_degenerate_blocks():
    """Identity gauge with values on the half-step grid (every code an exact tie between
    two integers, so every code is re-evaluated), constant and zero blocks, blocks whose
    minimum is near zero while the maximum is large (zero point undecidable from the
    tensor-core value alone), and large magnitudes."""
    need_gpu()
    L, B, H, T, d = 1, 1, 2, 256, 128
    rng = np.random.default_rng(3)
    x = np.zeros((L, 2, B, H, T, d), np.float32)
    # 4-bit grid: z = -1, s = 0.25 over a 16 x 16 block needs min -1 and max -1 + 15 * 0.25 = 2.75
    k = rng.integers(0, 30, size=(T, d)).astype(np.float32)
    x[0, 0, 0, 0] = -1.0 + 0.125 * k          # ties at every odd k
    x[0, 0, 0, 0, ::16, :] = -1.0             # pin every block's range
    x[0, 0, 0, 0, 1::16, :] = 2.75
    x[0, 0, 0, 1, :16, :] = 1.5               # constant block
    x[0, 0, 0, 1, 16:32, :] = 0.0             # zero block
    x[0, 1, 0, 0] = rng.standard_normal((T, d)).astype(np.float32) * 1e-3
    x[0, 1, 0, 0, 5::16, :] = 40.0            # min near 0, max large
    x[0, 1, 0, 1] = rng.standard_normal((T, d)).astype(np.float32) * 3000.0
    kv = torch.from_numpy(x).to(torch.bfloat16).cuda()
    G32 = np.broadcast_to(np.eye(16, dtype=np.float32), (L, 2, H, 8, 16, 16)).copy()
    for bits in (3, 4):
        _, _, _, ref, y = _check(kv, G32, bits)
        assert np.array_equal(y, ref["y"]), "identity gauge: the tensor cores see every value exactly"


def test_non_orthogonal_gauge_is_evaluated_exactly():
    """A gauge whose rows are not orthonormal voids the error bound; the encoder then
    evaluates the chain everywhere and still matches the oracle bit for bit."""
    need_gpu()
    kv = synth.kv_cache(1, 1, 2, 256, 128, seed=13, device="cuda", n_outliers=2)
    G32 = _oracle_G(1, 2, seed=13)
    G32[0, 0] *= 1.5
    G32[0, 1] = np.random.default_rng(13).standard_normal(G32[0, 1].shape).astype(np.float32) * 0.3
    _, _, _, ref, y = _check(kv, G32, 4)
    assert np.array_equal(y, ref["y"]), "non-orthogonal gauge: every value from the chain"


@pytest.mark.parametrize("bits", [3, 4])
def test_inputs_built_against_the_error_bound(bits):
    """Inputs built to attack the assumed accumulation bound (|y_tc - x.G_i| <= 2^-20
    sum_j |G_ij x_j|): rows whose gauged values cancel heavily (x = bf16(G^T v) with one
    large entry in v, so sum |G_ij x_j| is about 2^9 times most |y_i|); bf16 values whose
    exponents span 2^-20 .. 2^20 inside one 16-vector; a near-identity gauge with tiny
    off-diagonals; and outlier channels at 10^3 times the rest.  Codes, steps and zero
    points must equal the oracle's chain bit for bit, and no re-evaluated value may lie
    outside the bound (cg_sync_status, called by run_encode, would report CG_ERR_BOUND)."""
    need_gpu()
    L, B, H, T, d = 1, 1, 4, 256, 128
    rng = np.random.default_rng(100 + bits)
    G32 = _oracle_G(L, H, sigma=0.1, seed=bits)
    G32[0, :, 2] = _oracle_G(L, H, sigma=1e-4, seed=7)[0, :, 2]        # near identity, tiny off-diagonals
    x = np.zeros((L, 2, B, H, T, d), np.float32)
    # head 0: heavy cancellation, y = G x close to a one-hot v per 16-vector
    for s in range(2):
        for r in range(8):
            v = rng.standard_normal((T, 16)) * 1e-3
            v[np.arange(T), rng.integers(0, 16, T)] = rng.choice([-1.0, 1.0], T) * 10.0 ** rng.uniform(0, 3, T)
            x[0, s, 0, 0, :, 16 * r:16 * r + 16] = v @ G32[0, s, 0, r].astype(np.float64)   # x = G^T v per row
    # head 1: exponents spread over 2^-20 .. 2^20 inside each 16-vector, random signs
    x[0, :, 0, 1] = rng.choice([-1.0, 1.0], (2, T, d)) * 2.0 ** rng.uniform(-20, 20, (2, T, d))
    # head 2: near-identity gauge on ordinary data; head 3: outlier channels at 10^3 x
    x[0, :, 0, 2] = rng.standard_normal((2, T, d))
    x[0, :, 0, 3] = rng.standard_normal((2, T, d))
    x[0, :, 0, 3, :, [5, 40, 77, 126]] *= 1000.0
    kv = torch.from_numpy(x).to(torch.bfloat16).cuda()
    _, _, _, ref, y = _check(kv, G32, bits)
    cg.cg_sync_status()
    err = _block_error(y, np.asarray(ref["y"], dtype=np.float64))
    assert err <= BOUND, err
