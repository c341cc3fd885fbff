"""Parity of the decode step (through the C ABI) with the fp64 oracle.

One new token per sequence at position L-1 of a KV cache of L tokens: the
gate row without query pooling, the mask row, and the token's block-sparse
attention.  Tolerances are the prefill ones (see test_gpu_parity.py): gate
scores |x - x_ref| <= 1e-2 |x_ref| + 1e-12; O max abs <= 2e-2 and mean abs
<= 2e-3; LSE abs <= 1e-3; the mask bit-exact (decided by the oracle from the
GPU's own fp32 scores).
"""
import numpy as np
import pytest
import torch

import long_context_prefill_attngate_b200 as seer
from long_context_prefill_attngate_b200 import build as seer_build
from long_context_prefill_attngate_b200 import synthetic as syn

pytestmark = pytest.mark.gpu

BLOCK = 64
O_MAX, O_MEAN, REL = 2e-2, 2e-3, 1e-2


@pytest.fixture(scope="module", autouse=True)
def gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    seer_build.build()
    seer.lib()
    yield
    seer.seer_check_status()


def bits(t):
    return syn.bf16_bits(t.cpu().contiguous())


def dev(t):
    return t.cuda().contiguous()


def decode_inputs(B, Hq, Hkv, L, d, dg, number):
    w = syn.custom("decode", B, Hq, Hkv, L, d, number=number, d_gate=dg)
    x = syn.make_inputs(w)
    return w, x["q"][:, :, L - 1].contiguous(), x["k"], x["v"], x["wq"], x["wk"]


def check_rel(x, ref, what):
    x = np.asarray(x, np.float64)
    bad = np.abs(x - ref) > REL * np.abs(ref) + 1e-12
    assert not bad.any(), f"{what}: {bad.sum()} entries off, e.g. {x[bad][:3]} vs {ref[bad][:3]}"


def check_o(o, o_ref, what):
    err = np.abs(o.double().cpu().numpy() - o_ref)
    assert np.isfinite(err).all(), what
    assert err.max() <= O_MAX, f"{what}: max abs err {err.max():.3e}"
    assert err.mean() <= O_MEAN, f"{what}: mean abs err {err.mean():.3e}"


@pytest.mark.parametrize("B,Hq,Hkv,L,d,dg,maxmin", [
    (1, 8, 2, 4096, 128, 128, False),
    (2, 4, 1, 9 * BLOCK + 17, 64, 64, True),   # ragged cache, max+min K pooling
    (1, 4, 2, 37, 128, 64, False),            # one partial block
    (1, 32, 8, 32768, 128, 128, False),       # the Llama-3.1-8B layer at 32k
])
def test_decode_gate_parity(oracle, B, Hq, Hkv, L, d, dg, maxmin):
    w, q, k, v, wq, wk = decode_inputs(B, Hq, Hkv, L, d, dg, 301 + L)
    if maxmin:
        g = torch.Generator().manual_seed(L)
        wk = (torch.randn((Hkv, 2 * d, dg), generator=g) * 0.08).to(torch.bfloat16)
    s = seer.seer_decode_gate_scores(dev(q), dev(k), dev(wq), dev(wk), rope_theta=w.rope_theta, k_maxmin=maxmin)
    seer.seer_check_status()
    ref = oracle.decode_gate_scores(bits(q), bits(k), bits(wq), bits(wk), theta=w.rope_theta, k_maxmin=maxmin)
    assert s.shape == (B, Hq, -(-L // BLOCK))
    check_rel(s.cpu().numpy(), ref, "decode scores")


@pytest.mark.parametrize("L", [4096, 5 * BLOCK + 3])
def test_decode_mask_bit_exact(oracle, L):
    B, Hq, Hkv, d = 2, 8, 2, 128
    w, q, k, v, wq, wk = decode_inputs(B, Hq, Hkv, L, d, 128, 311 + L)
    s = seer.seer_decode_gate_scores(dev(q), dev(k), dev(wq), dev(wk), rope_theta=w.rope_theta)
    nb = s.shape[-1]
    sc = s.cpu().numpy()
    for density in (0.1, 0.3, 1.0):
        m = seer.seer_decode_block_mask(s, "topk", density=density)
        seer.seer_check_status()
        kk = int(np.ceil(density * nb))
        ref = oracle.decode_mask(sc, "topk", k=kk)
        assert np.array_equal(m.cpu().numpy(), ref), f"topk density {density}"
    m = seer.seer_decode_block_mask(s, "topk", k_fixed=5)
    assert np.array_equal(m.cpu().numpy(), oracle.decode_mask(sc, "topk", k=5))
    thr = float(np.quantile(sc, 0.8))
    m = seer.seer_decode_block_mask(s, "threshold", threshold=thr)
    assert np.array_equal(m.cpu().numpy(), oracle.decode_mask(sc, "threshold", threshold=np.float32(thr)))


@pytest.mark.parametrize("B,Hq,Hkv,L,d,p", [
    (1, 8, 2, 4096, 128, 0.1),
    (2, 4, 4, 3000, 64, 0.5),                 # ragged cache, g = 1
    (1, 5, 1, 64 * 33 + 1, 128, 0.3),          # a one-token last block, g = 5
    (1, 4, 2, 50, 128, 1.0),                  # shorter than one block
    (1, 6, 2, 2048, 128, 1.0),                # dense decode
    (1, 16, 1, 1500, 64, 0.4),                # g = 16: the per-head form (groups above 8)
])
def test_decode_attention_parity(oracle, B, Hq, Hkv, L, d, p):
    w, q, k, v, wq, wk = decode_inputs(B, Hq, Hkv, L, d, 128, 321 + L)
    nb = -(-L // BLOCK)
    g = torch.Generator().manual_seed(L + 7)
    mask = (torch.rand((B, Hq, nb), generator=g) < p).to(torch.uint8)
    mask[..., 0] = 1
    mask[..., nb - 1] = 1
    o, lse = seer.seer_block_sparse_decode(dev(q), dev(k), dev(v), dev(mask), return_lse=True)
    seer.seer_check_status()
    o_ref, lse_ref = oracle.decode_attention(bits(q), bits(k), bits(v), mask.numpy())
    check_o(o, o_ref, "decode O")
    assert np.abs(lse.cpu().double().numpy() - lse_ref).max() <= 1e-3


def test_decode_attention_empty_row(oracle):
    B, Hq, Hkv, L, d = 1, 4, 2, 1024, 128
    w, q, k, v, wq, wk = decode_inputs(B, Hq, Hkv, L, d, 128, 331)
    mask = torch.zeros((B, Hq, L // BLOCK), dtype=torch.uint8)
    mask[0, 1, 3] = 1                          # one head with a single active block
    o, lse = seer.seer_block_sparse_decode(dev(q), dev(k), dev(v), dev(mask), return_lse=True)
    seer.seer_check_status()
    o_ref, lse_ref = oracle.decode_attention(bits(q), bits(k), bits(v), mask.numpy())
    assert torch.all(o[0, [0, 2, 3]] == 0) and torch.all(torch.isinf(lse[0, [0, 2, 3]]))
    check_o(o[0, 1:2], o_ref[0, 1:2], "single block")


def test_decode_step_full_size(oracle):
    """Gate -> TopK mask -> sparse decode for the last token of a 32k Llama
    layer (all 32 heads checked against the oracle on the GPU's own mask)."""
    B, Hq, Hkv, L, d = 1, 32, 8, 32768, 128
    w, q, k, v, wq, wk = decode_inputs(B, Hq, Hkv, L, d, 128, 341)
    qd, kd, vd = dev(q), dev(k), dev(v)
    s = seer.seer_decode_gate_scores(qd, kd, dev(wq), dev(wk), rope_theta=w.rope_theta)
    m = seer.seer_decode_block_mask(s, "topk", density=0.1)
    o, lse = seer.seer_block_sparse_decode(qd, kd, vd, m, return_lse=True)
    seer.seer_check_status()
    assert int(m.sum()) == B * Hq * int(np.ceil(0.1 * (L // BLOCK)))
    o_ref, lse_ref = oracle.decode_attention(bits(q), bits(k), bits(v), m.cpu().numpy())
    check_o(o, o_ref, "decode O (32k)")
    assert np.abs(lse.cpu().double().numpy() - lse_ref).max() <= 1e-3


@pytest.mark.parametrize("maxmin", [False, True])
def test_decode_gate_key_cache(oracle, maxmin):
    """Key rows kept across decode steps: the cached row equals the one-call
    gate bit for bit, and refreshing only from the last partial block on after
    the cache grew equals recomputing every row."""
    B, Hq, Hkv, d, dg = 2, 8, 2, 128, 64
    L1, L2 = 5 * BLOCK + 10, 6 * BLOCK + 3
    w, q, k, v, wq, wk = decode_inputs(B, Hq, Hkv, L2, d, dg, 361)
    if maxmin:
        g = torch.Generator().manual_seed(361)
        wk = (torch.randn((Hkv, 2 * d, dg), generator=g) * 0.08).to(torch.bfloat16)
    kd, wqd, wkd, qd = dev(k), dev(wq), dev(wk), dev(q)
    k1 = kd[:, :, :L1].contiguous()
    kt1 = seer.seer_gate_key_cache(k1, wkd, rope_theta=w.rope_theta, k_maxmin=maxmin)
    s_c = seer.seer_decode_gate_scores_cached(qd, kt1, wqd, L1, Hkv, rope_theta=w.rope_theta)
    s_f = seer.seer_decode_gate_scores(qd, k1, wqd, wkd, rope_theta=w.rope_theta, k_maxmin=maxmin)
    seer.seer_check_status()
    assert torch.equal(s_c, s_f)
    ref = oracle.decode_gate_scores(bits(q), bits(k[:, :, :L1]), bits(wq), bits(wk), theta=w.rope_theta,
                                    k_maxmin=maxmin)
    check_rel(s_c.cpu().numpy(), ref, "cached decode scores")
    # the cache grows to L2: keep the complete blocks, refresh from block 5 (was partial) on
    nb1, nb2 = -(-L1 // BLOCK), -(-L2 // BLOCK)
    kt2 = torch.full((B, Hkv, nb2, dg), float("nan"), dtype=torch.float32, device="cuda")
    kt2[:, :, : nb1 - 1] = kt1[:, :, : nb1 - 1]
    seer.seer_gate_key_cache(kd, wkd, kt=kt2, first_block=nb1 - 1, rope_theta=w.rope_theta, k_maxmin=maxmin)
    full = seer.seer_gate_key_cache(kd, wkd, rope_theta=w.rope_theta, k_maxmin=maxmin)
    seer.seer_check_status()
    assert torch.equal(kt2, full)
