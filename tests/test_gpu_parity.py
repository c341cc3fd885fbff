"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Tolerances (fixed by the benchmark spec of the hot path, restated here):
  * O: bf16 inputs, fp32 accumulation -> max |O - O_ref| <= 2e-2 and
    mean |O - O_ref| <= 2e-3 against the fp64 oracle;
  * gate scores and the pooled map A: |x - x_ref| <= 1e-2 |x_ref| + 1e-12;
  * LSE: |lse - lse_ref| <= 1e-3 (fp32 log-sum-exp of exact fp32 dot products);
  * block mask and compaction: bit-exact (the oracle decides the mask from the
    GPU's own fp32 scores, in the same precision).
Small cases are compared element by element; the full-size layers are
compared on sampled query blocks, each of which the oracle computes exactly.
"""
import math

import numpy as np
import pytest
import torch

import long_context_prefill_attngate_b200 as seer
from long_context_prefill_attngate_b200 import build as seer_build
from long_context_prefill_attngate_b200 import synthetic as syn

pytestmark = pytest.mark.gpu

BLOCK = 64
O_MAX, O_MEAN = 2e-2, 2e-3
REL = 1e-2


@pytest.fixture(scope="module", autouse=True)
def gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    seer_build.build()
    seer.lib()
    torch.cuda.init()
    yield
    seer.seer_check_status()


def bits(t):
    return syn.bf16_bits(t.cpu())


def dev(t):
    return t.cuda().contiguous()


def check_o(o_gpu, o_ref, what=""):
    o = o_gpu.double().cpu().numpy()
    err = np.abs(o - o_ref)
    assert np.isfinite(o).all(), f"{what}: non-finite output"
    assert err.max() <= O_MAX, f"{what}: max abs err {err.max():.3e}"
    assert err.mean() <= O_MEAN, f"{what}: mean abs err {err.mean():.3e}"


def check_rel(x, ref, what=""):
    x = np.asarray(x, np.float64)
    bad = np.abs(x - ref) > REL * np.abs(ref) + 1e-12
    assert not bad.any(), f"{what}: {bad.sum()} entries off, worst at {np.argwhere(bad)[:3]}: " \
                          f"{x[bad][:3]} vs {ref[bad][:3]}"


def units_all(B, H, nb):
    import oracle
    return oracle.all_units(B, H, nb)


def gather_units(t, units, fill=0.0):
    """Rows [n, 64, ...] of a [B,H,S,...] tensor for (b, h, i) units; the rows
    a ragged last block lacks (past S) are filled with `fill`, as the oracle
    reports them."""
    out = []
    for b, h, i in units:
        r = t[b, h, i * BLOCK:(i + 1) * BLOCK]
        if r.shape[0] < BLOCK:
            r = torch.cat([r, torch.full((BLOCK - r.shape[0],) + tuple(r.shape[1:]), fill, dtype=r.dtype)])
        out.append(r)
    return torch.stack(out)


def sample_units(B, H, nb, n_blocks, seed):
    rng = np.random.default_rng(seed)
    blocks = sorted(set([0, nb - 1, nb // 2] + list(rng.integers(0, nb, size=max(0, n_blocks - 3)))))
    return np.array([(b, h, i) for b in range(B) for h in range(H) for i in blocks], np.int32)


def run_prefill_case(oracle, q, k, v, mask, units=None, scale=0.0, lse=True):
    qd, kd, vd, md = dev(q), dev(k), dev(v), dev(mask)
    o, l = seer.seer_block_sparse_prefill(qd, kd, vd, md, softmax_scale=scale, return_lse=lse)
    seer.seer_check_status()
    B, Hq, S, d = q.shape
    if units is None:
        units = units_all(B, Hq, -(-S // BLOCK))
    o_ref, lse_ref = oracle.masked_attention(bits(q), bits(k), bits(v), mask.numpy(),
                                             scale=(scale if scale > 0 else None), units=units)
    check_o(gather_units(o.cpu(), units), o_ref, "O")
    if lse:
        lg = gather_units(l.cpu(), units, fill=float("-inf")).double().numpy()
        fin = np.isfinite(lse_ref)
        assert np.array_equal(np.isfinite(lg), fin)
        assert np.abs(lg[fin] - lse_ref[fin]).max() <= 1e-3
    return o


# ------------------------------------------------------------------ prefill
def test_prefill_tiny_workload(oracle):
    w = syn.WORKLOADS["tiny"]
    x = syn.make_inputs(w)
    run_prefill_case(oracle, x["q"], x["k"], x["v"], x["mask"])


@pytest.mark.parametrize("B,Hq,Hkv,S,d,p,ff,fd", [
    (1, 8, 2, 1024, 128, 0.3, True, True),     # GQA g=4: head pairs
    (2, 4, 4, 640, 64, 0.5, True, True),       # g=1: block pairs, nb=10
    (1, 5, 1, 576, 128, 0.4, True, True),      # g=5: pairs + leftover head, odd nb
    (1, 6, 2, 768, 128, 1.0, True, True),      # g=3, dense causal
    (1, 4, 2, 512, 128, 0.2, False, False),    # rows with no active block
    (1, 2, 2, 64, 64, 1.0, True, True),        # a single block
    (1, 3, 3, 1984, 64, 0.15, True, False),    # g=1, odd nb=31, no diagonal forcing
])
def test_prefill_shapes(oracle, B, Hq, Hkv, S, d, p, ff, fd):
    w = syn.custom("case", B, Hq, Hkv, S, d, number=7 + S + Hq)
    x = syn.make_inputs(w)
    mask = syn.random_mask(B, Hq, S // BLOCK, p, seed=S + Hq, force_first=ff, force_diag=fd)
    run_prefill_case(oracle, x["q"], x["k"], x["v"], mask)


@pytest.mark.parametrize("d", [128, 64])
def test_prefill_odd_counts_and_single_block_rows(oracle, d):
    """Rows whose active count is odd (the kernel ends them with a one-block
    step), rows holding a single block (the diagonal alone, or block 0 alone
    with no diagonal), and even counts, all in one layer."""
    B, Hq, Hkv, nb = 1, 4, 2, 24
    S = nb * BLOCK
    w = syn.custom("odd", B, Hq, Hkv, S, d, number=91 + d)
    x = syn.make_inputs(w)
    rng = np.random.default_rng(5 + d)
    mask = np.zeros((B, Hq, nb, nb), np.uint8)
    for h in range(Hq):
        for i in range(nb):
            kind = (h + i) % 5
            if kind == 0:
                sel = [i]                                   # the diagonal alone
            elif kind == 1:
                sel = [0]                                   # block 0 alone (no diagonal for i > 0)
            elif kind == 2:
                sel = rng.choice(i + 1, size=min(i + 1, 3), replace=False)
            elif kind == 3:
                n_odd = (i + 1) if (i + 1) % 2 else i       # the largest odd count <= i + 1
                sel = rng.choice(i + 1, size=n_odd, replace=False)
            else:
                sel = rng.choice(i + 1, size=min(i + 1, 2), replace=False)
            mask[0, h, i, sel] = 1
    counts = mask.sum(-1)
    assert (counts % 2 == 1).sum() > nb and (counts == 1).sum() >= 2 * Hq
    run_prefill_case(oracle, x["q"], x["k"], x["v"], torch.from_numpy(mask))


@pytest.mark.parametrize("B,Hq,Hkv,S,d,p", [
    (1, 4, 2, 5 * BLOCK + 17, 128, 0.5),      # ragged last block, head pairs
    (2, 3, 1, 3 * BLOCK + 1, 64, 0.6),        # a one-token last block, leftover head
    (1, 8, 2, 9 * BLOCK + 63, 128, 0.3),      # 63 of 64
    (1, 2, 2, 37, 64, 1.0),                   # S < 64: one partial block
    (1, 6, 2, 20 * BLOCK + 40, 128, 1.0),     # dense causal, ragged
])
def test_prefill_ragged_sequence(oracle, B, Hq, Hkv, S, d, p):
    """S not a multiple of 64: rows past S are never written, keys past S never
    attended (TMA fills them with zeros; the causal mask of the last block
    excludes them)."""
    w = syn.custom("ragged", B, Hq, Hkv, S, d, number=211 + S)
    x = syn.make_inputs(w)
    nb = -(-S // BLOCK)
    mask = syn.random_mask(B, Hq, nb, p, seed=S + 5)
    qd, kd, vd = dev(x["q"]), dev(x["k"]), dev(x["v"])
    # O as a view at the front of a larger buffer: rows a kernel wrote past S
    # of the last head would land in the sentinel tail.
    n = B * Hq * S * d
    flat = torch.full((n + BLOCK * d,), 7.0, dtype=torch.bfloat16, device="cuda")
    seer.seer_block_sparse_prefill(qd, kd, vd, dev(mask), o=flat[:n].view(B, Hq, S, d))
    seer.seer_check_status()
    assert torch.all(flat[n:] == 7.0)
    run_prefill_case(oracle, x["q"], x["k"], x["v"], mask)


def test_pooled_map_ragged_sequence(oracle):
    B, Hq, Hkv, S, d = 1, 4, 2, 7 * BLOCK + 29, 128
    w = syn.custom("rmap", B, Hq, Hkv, S, d, number=223)
    x = syn.make_inputs(w)
    o, A = seer.seer_attn_pooled_map(dev(x["q"]), dev(x["k"]), dev(x["v"]))
    seer.seer_check_status()
    nb = -(-S // BLOCK)
    units = units_all(B, Hq, nb)
    o_ref, A_ref = oracle.pooled_map(bits(x["q"]), bits(x["k"]), bits(x["v"]), units=units)
    check_o(gather_units(o.cpu(), units), o_ref, "O(map, ragged)")
    check_rel(A.cpu().numpy().reshape(-1, nb), A_ref, "A(ragged)")


@pytest.mark.parametrize("S,maxmin", [(4 * BLOCK + 3, False), (9 * BLOCK + 50, True), (50, False)])
def test_gate_scores_ragged_sequence(oracle, S, maxmin):
    B, Hq, Hkv, d, dg = 1, 4, 2, 128, 64
    w = syn.custom("rgate", B, Hq, Hkv, S, d, number=227 + S, d_gate=dg)
    x = syn.make_inputs(w)
    wk = x["wk"]
    if maxmin:
        g = torch.Generator().manual_seed(S)
        wk = (torch.randn((Hkv, 2 * d, dg), generator=g) * 0.08).to(torch.bfloat16)
    s = seer.seer_gate_scores(dev(x["q"]), dev(x["k"]), dev(x["wq"]), dev(wk), rope_theta=w.rope_theta,
                              k_maxmin=maxmin)
    seer.seer_check_status()
    ref = oracle.gate_scores(bits(x["q"]), bits(x["k"]), bits(x["wq"]), bits(wk), theta=w.rope_theta,
                             k_maxmin=maxmin)
    assert s.shape[-1] == -(-S // BLOCK)
    check_rel(s.cpu().numpy(), ref, "scores(ragged)")


def test_prefill_all_zero_mask_gives_zero_output(oracle):
    w = syn.custom("zero", 1, 4, 2, 256, 128, number=3)
    x = syn.make_inputs(w)
    mask = torch.zeros((1, 4, 4, 4), dtype=torch.uint8)
    o, l = seer.seer_block_sparse_prefill(dev(x["q"]), dev(x["k"]), dev(x["v"]), dev(mask), return_lse=True)
    seer.seer_check_status()
    assert torch.all(o == 0)
    assert torch.all(torch.isinf(l)) and torch.all(l < 0)


def test_prefill_custom_scale_and_long_rows(oracle):
    w = syn.custom("long", 1, 2, 1, 8192, 128, number=11)
    x = syn.make_inputs(w)
    mask = syn.random_mask(1, 2, 128, 0.1, seed=5)
    units = sample_units(1, 2, 128, 8, 3)
    run_prefill_case(oracle, x["q"], x["k"], x["v"], mask, units=units, scale=0.05)


def test_prefill_repeatable():
    w = syn.custom("rep", 1, 8, 2, 2048, 128, number=12)
    x = syn.make_inputs(w)
    mask = dev(syn.random_mask(1, 8, 32, 0.3, seed=9))
    q, k, v = dev(x["q"]), dev(x["k"]), dev(x["v"])
    o1 = seer.seer_block_sparse_prefill(q, k, v, mask)
    o2 = seer.seer_block_sparse_prefill(q, k, v, mask)
    seer.seer_check_status()
    assert torch.equal(o1, o2)


def test_prefill_concurrent_streams_and_counter_ring():
    """Launches on different streams take tiles from different counters: two
    concurrent calls give exactly their one-at-a-time results, and more calls
    than the counter ring holds (256) in a row stay exact."""
    w1 = syn.custom("cs1", 1, 8, 2, 4096, 128, number=41)
    w2 = syn.custom("cs2", 2, 4, 1, 2048, 64, number=42)
    x1, x2 = syn.make_inputs(w1), syn.make_inputs(w2)
    m1 = dev(syn.random_mask(1, 8, 64, 0.3, seed=43))
    m2 = dev(syn.random_mask(2, 4, 32, 0.5, seed=44))
    a = [dev(x1[n]) for n in ("q", "k", "v")]
    b = [dev(x2[n]) for n in ("q", "k", "v")]
    ref1 = seer.seer_block_sparse_prefill(*a, m1)
    ref2 = seer.seer_block_sparse_prefill(*b, m2)
    torch.cuda.synchronize()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    o1, o2 = torch.empty_like(ref1), torch.empty_like(ref2)
    for _ in range(5):
        o1.zero_()
        o2.zero_()
        torch.cuda.synchronize()
        with torch.cuda.stream(s1):
            seer.seer_block_sparse_prefill(*a, m1, o=o1, stream=s1)
        with torch.cuda.stream(s2):
            seer.seer_block_sparse_prefill(*b, m2, o=o2, stream=s2)
        torch.cuda.synchronize()
        assert torch.equal(o1, ref1) and torch.equal(o2, ref2)
    o = torch.empty_like(ref2)
    for _ in range(300):
        seer.seer_block_sparse_prefill(*b, m2, o=o)
    torch.cuda.synchronize()
    seer.seer_check_status()
    assert torch.equal(o, ref2)


@pytest.mark.parametrize("d", [64, 128])
def test_prefill_max_sequence(oracle, d):
    """S = 2^20 (the largest nb the library accepts): first + diagonal blocks only.
    At d = 128 the kernel's shared-memory layout leaves almost no room under the
    227 KB cap, so this also covers the window-fit check passing."""
    B, Hq, Hkv, S = 1, 2, 1, 1 << 20
    nb = S // BLOCK
    g = torch.Generator().manual_seed(77)
    q = torch.randn((B, Hq, S, d), generator=g).to(torch.bfloat16)
    k = torch.randn((B, Hkv, S, d), generator=g).to(torch.bfloat16)
    v = torch.randn((B, Hkv, S, d), generator=g).to(torch.bfloat16)
    scores = torch.zeros((B, Hq, nb, nb), dtype=torch.float32, device="cuda")
    mask = seer.seer_block_mask(scores, "topk", k_fixed=2, Hkv=Hkv, d=d)
    for _, h, i in [(0, h, i) for h in range(Hq) for i in (0, 1, 5000, nb - 1)]:
        row = mask[0, h, i].cpu().numpy()
        want = np.zeros(nb, np.uint8)
        want[0] = 1
        want[i] = 1
        assert np.array_equal(row, want)
    if d == 128:
        mask[0, 0, nb - 1].fill_(1)    # one full row: a 16384-entry key-block list
    o = seer.seer_block_sparse_prefill(dev(q), dev(k), dev(v), mask)
    seer.seer_check_status()
    units = np.array([(0, h, i) for h in range(Hq) for i in (0, 1, 5000, nb - 1)], np.int32)
    mask_rows = torch.zeros((B, Hq, nb, nb), dtype=torch.uint8)
    del scores
    # Only the sampled rows are needed by the oracle; build a mask holding them.
    for _, h, i in units:
        mask_rows[0, h, i] = mask[0, h, i].cpu()
    o_ref, _ = oracle.masked_attention(bits(q), bits(k), bits(v), mask_rows.numpy(), units=units)
    check_o(gather_units(o.cpu(), units), o_ref, f"O@1M d={d}")


# ------------------------------------------------------------------ pooled map
@pytest.mark.parametrize("B,Hq,Hkv,S,d", [
    (1, 2, 2, 512, 64),      # the tiny workload's shape (g=1)
    (1, 5, 1, 576, 128),     # g=5, odd nb
    (2, 4, 2, 1024, 64),     # g=2
])
def test_pooled_map_small(oracle, B, Hq, Hkv, S, d):
    w = syn.WORKLOADS["tiny"] if (S == 512 and d == 64) else syn.custom("map", B, Hq, Hkv, S, d, number=31 + S)
    x = syn.make_inputs(w)
    o, A = seer.seer_attn_pooled_map(dev(x["q"]), dev(x["k"]), dev(x["v"]))
    seer.seer_check_status()
    units = units_all(B, Hq, S // BLOCK)
    o_ref, A_ref = oracle.pooled_map(bits(x["q"]), bits(x["k"]), bits(x["v"]), units=units)
    check_o(gather_units(o.cpu(), units), o_ref, "O(map)")
    check_rel(A.cpu().numpy().reshape(-1, S // BLOCK), A_ref, "A")
    An = A.cpu().double().numpy()
    assert np.all(An[..., 0, 0] == pytest.approx(1.0, rel=1e-2))
    assert np.all(np.triu(An, 1) == 0)


# ------------------------------------------------------------------ gate / mask / compaction
@pytest.mark.parametrize("B,Hq,Hkv,S,d,dg", [(1, 2, 2, 512, 64, 64), (1, 8, 2, 4096, 128, 128),
                                             (2, 5, 1, 1152, 128, 64)])
def test_gate_scores(oracle, B, Hq, Hkv, S, d, dg):
    w = syn.custom("gate", B, Hq, Hkv, S, d, number=41 + S, d_gate=dg)
    x = syn.make_inputs(w)
    s = seer.seer_gate_scores(dev(x["q"]), dev(x["k"]), dev(x["wq"]), dev(x["wk"]), rope_theta=w.rope_theta)
    seer.seer_check_status()
    ref = oracle.gate_scores(bits(x["q"]), bits(x["k"]), bits(x["wq"]), bits(x["wk"]), theta=w.rope_theta)
    check_rel(s.cpu().numpy(), ref, "scores")


@pytest.mark.parametrize("B,Hq,Hkv,S,d,dg", [(1, 4, 2, 1000, 128, 256), (2, 3, 3, 700, 64, 12),
                                             (1, 2, 1, 37 * BLOCK + 5, 128, 4)])
def test_gate_scores_dgate_range(oracle, B, Hq, Hkv, S, d, dg):
    """d_gate above one 64-feature stage of the logits kernel (256: four stages,
    the projection's second column pass), below one warp's rotation pairs
    (12, 4); block counts 16 (the 16-byte load path), 11 and 38 (not multiples
    of 4: the element-wise path)."""
    w = syn.custom("gatedg", B, Hq, Hkv, S, d, number=53 + S + dg, d_gate=dg)
    x = syn.make_inputs(w)
    s = seer.seer_gate_scores(dev(x["q"]), dev(x["k"]), dev(x["wq"]), dev(x["wk"]), rope_theta=w.rope_theta)
    seer.seer_check_status()
    ref = oracle.gate_scores(bits(x["q"]), bits(x["k"]), bits(x["wq"]), bits(x["wk"]), theta=w.rope_theta)
    check_rel(s.cpu().numpy(), ref, f"scores(d_gate={dg})")


@pytest.mark.parametrize("B,Hq,Hkv,S,d,dg", [(1, 2, 2, 512, 64, 64), (1, 8, 2, 4096, 128, 128),
                                             (2, 5, 1, 1152, 128, 64)])
def test_gate_scores_maxmin_k(oracle, B, Hq, Hkv, S, d, dg):
    """K pooled by [max | min] (2d features, W_k [Hkv, 2d, dg])."""
    w = syn.custom("gatemm", B, Hq, Hkv, S, d, number=47 + S, d_gate=dg)
    x = syn.make_inputs(w)
    g = torch.Generator().manual_seed(4700 + S)
    wk = (torch.randn((Hkv, 2 * d, dg), generator=g) * (2.0 / (2 * d + dg)) ** 0.5).to(torch.bfloat16)
    s = seer.seer_gate_scores(dev(x["q"]), dev(x["k"]), dev(x["wq"]), dev(wk), rope_theta=w.rope_theta,
                              k_maxmin=True)
    seer.seer_check_status()
    ref = oracle.gate_scores(bits(x["q"]), bits(x["k"]), bits(x["wq"]), bits(wk), theta=w.rope_theta,
                             k_maxmin=True)
    check_rel(s.cpu().numpy(), ref, "scores(max+min K)")
    # the same inputs through the average path must differ (the flag is honoured)
    s_avg = seer.seer_gate_scores(dev(x["q"]), dev(x["k"]), dev(x["wq"]), dev(wk[:, :d].contiguous()),
                                  rope_theta=w.rope_theta)
    assert not torch.allclose(s_avg, s)


def test_gate_scores_strong_logits(oracle):
    """Larger weights so the softmax is far from uniform (exercises exp range)."""
    w = syn.custom("gate2", 1, 4, 2, 2048, 128, number=43)
    x = syn.make_inputs(w)
    wq = (x["wq"].float() * 40).to(torch.bfloat16)
    wk = (x["wk"].float() * 40).to(torch.bfloat16)
    s = seer.seer_gate_scores(dev(x["q"]), dev(x["k"]), dev(wq), dev(wk))
    seer.seer_check_status()
    ref = oracle.gate_scores(bits(x["q"]), bits(x["k"]), bits(wq), bits(wk))
    assert ref.max() > 0.5
    check_rel(s.cpu().numpy(), ref, "scores")


def _scores_with_ties(B, H, nb, seed):
    g = torch.Generator().manual_seed(seed)
    s = torch.rand((B, H, nb, nb), generator=g)
    s = torch.round(s * 16) / 16          # many exact ties
    s[0, 0, nb - 1, :] = 0.25
    return s.contiguous()


@pytest.mark.parametrize("nb,density,ff,fd", [(40, 0.3, True, True), (257, 0.1, True, True),
                                              (64, 0.5, False, False), (33, 0.0, True, True),
                                              (700, 0.2, True, True), (1100, 0.05, False, True)])
def test_topk_mask_bit_exact(oracle, nb, density, ff, fd):
    s = _scores_with_ties(2, 3, nb, nb)
    m = seer.seer_block_mask(dev(s), "topk", density=density, force_first=ff, force_diag=fd)
    seer.seer_check_status()
    k_row = np.array([math.ceil(density * (i + 1)) for i in range(nb)], np.int32)
    ref = oracle.block_mask(s.numpy(), "topk", k_row=k_row, force_first=ff, force_diag=fd)
    assert np.array_equal(m.cpu().numpy(), ref)


def test_topk_mask_k_per_row_and_fixed(oracle):
    nb = 50
    s = _scores_with_ties(1, 2, nb, 3)
    kr = torch.tensor([(i * 7) % 11 for i in range(nb)], dtype=torch.int32)
    m = seer.seer_block_mask(dev(s), "topk", k_per_row=kr.cuda())
    ref = oracle.block_mask(s.numpy(), "topk", k_row=kr.numpy())
    assert np.array_equal(m.cpu().numpy(), ref)
    m = seer.seer_block_mask(dev(s), "topk", k_fixed=5)
    ref = oracle.block_mask(s.numpy(), "topk", k_row=np.full(nb, 5, np.int32))
    assert np.array_equal(m.cpu().numpy(), ref)


@pytest.mark.parametrize("thr,ff,fd", [(0.5, True, True), (0.8125, False, False), (-1.0, True, False)])
def test_threshold_mask_bit_exact(oracle, thr, ff, fd):
    s = _scores_with_ties(2, 2, 70, 5)
    m = seer.seer_block_mask(dev(s), "threshold", threshold=thr, force_first=ff, force_diag=fd)
    seer.seer_check_status()
    ref = oracle.block_mask(s.numpy(), "threshold", thr, force_first=ff, force_diag=fd)
    assert np.array_equal(m.cpu().numpy(), ref)


def test_compact_bit_exact(oracle):
    m = syn.random_mask(2, 3, 70, 0.3, seed=4)
    lists, counts = seer.seer_compact_mask(dev(m))
    seer.seer_check_status()
    rl, rc = oracle.compact(m.numpy())
    assert np.array_equal(counts.cpu().numpy(), rc)
    gl = lists.cpu().numpy()
    for b in range(2):
        for h in range(3):
            for i in range(70):
                off = i * (i + 1) // 2
                n = rc[b, h, i]
                assert np.array_equal(gl[b, h, off:off + n], rl[b, h, off:off + n])


# ------------------------------------------------------------------ full-size layers (sampled)
def _gate_mask(w, x, mode, **kw):
    s = seer.seer_gate_scores(dev(x["q"]), dev(x["k"]), dev(x["wq"]), dev(x["wk"]), rope_theta=w.rope_theta)
    m = seer.seer_block_mask(s, mode, Hkv=w.Hkv, d=w.d, **kw)
    seer.seer_check_status()
    return s, m


def test_llama8k_threshold_layer(oracle):
    w = syn.WORKLOADS["llama8b_8k"]
    x = syn.make_inputs(w)
    s, m = _gate_mask(w, x, "threshold", threshold=w.threshold)
    ref_s = oracle.gate_scores(bits(x["q"]), bits(x["k"]), bits(x["wq"]), bits(x["wk"]), theta=w.rope_theta)
    check_rel(s.cpu().numpy(), ref_s, "scores@8k")
    ref_m = oracle.block_mask(s.cpu().numpy(), "threshold", w.threshold)
    assert np.array_equal(m.cpu().numpy(), ref_m)
    run_prefill_case(oracle, x["q"], x["k"], x["v"], m.cpu(), units=sample_units(1, w.Hq, w.nb, 4, 1))


@pytest.fixture(scope="module")
def llama32k(oracle):
    w = syn.WORKLOADS["llama8b_32k"]
    x = syn.make_inputs(w)
    ref_rows = oracle.gate_scores(bits(x["q"]), bits(x["k"]), bits(x["wq"]), bits(x["wk"]), theta=w.rope_theta)
    return w, x, ref_rows


@pytest.mark.parametrize("density", [1.0, 0.5, 0.3, 0.2, 0.1])
def test_llama32k_topk_layer(oracle, llama32k, density):
    """The benchmark's launch configuration: 32k, every TopK density of the
    sweep (1.0 is the dense causal point).  Scores within rel 1e-2, the mask
    bit-exact, O on sampled query blocks of every head."""
    w, x, ref_rows = llama32k
    s, m = _gate_mask(w, x, "topk", density=density)
    k_row = oracle.topk_counts(density, w.nb)
    sc = s.cpu().numpy()
    ref_m = oracle.block_mask(sc, "topk", k_row=k_row)
    assert np.array_equal(m.cpu().numpy(), ref_m)
    check_rel(sc, ref_rows, "scores@32k")
    del sc, ref_m
    n_blocks = 3 if density >= 0.5 else 4
    run_prefill_case(oracle, x["q"], x["k"], x["v"], m.cpu(),
                     units=sample_units(1, w.Hq, w.nb, n_blocks, 2 + int(density * 10)))


def test_llama128k_threshold_layer(oracle):
    w = syn.WORKLOADS["llama8b_128k"]
    x = syn.make_inputs(w)
    s = seer.seer_gate_scores(dev(x["q"]), dev(x["k"]), dev(x["wq"]), dev(x["wk"]), rope_theta=w.rope_theta)
    # Threshold tuned for ~0.17 density: a quantile of the causal scores.
    nb = w.nb
    tri = torch.tril(torch.ones(nb, nb, dtype=torch.bool, device="cuda"))
    vals = s[0, 0][tri]
    thr = float(torch.quantile(vals[torch.randperm(vals.numel(), device="cuda")[:1 << 20]].float(), 0.83))
    m = seer.seer_block_mask(s, "threshold", threshold=thr, Hkv=w.Hkv, d=w.d)
    seer.seer_check_status()
    units = sample_units(1, w.Hq, nb, 3, 3)[::4]
    sc = s.cpu().numpy()
    ref_m = oracle.block_mask(sc, "threshold", thr)
    assert np.array_equal(m.cpu().numpy(), ref_m)
    del sc, ref_m
    run_prefill_case(oracle, x["q"], x["k"], x["v"], m.cpu(), units=units)


def test_qwen64k_pooled_map_sampled(oracle):
    w = syn.WORKLOADS["qwen14b_64k_map"]
    x = syn.make_inputs(w)
    o, A = seer.seer_attn_pooled_map(dev(x["q"]), dev(x["k"]), dev(x["v"]))
    seer.seer_check_status()
    units = np.array([(0, 0, 0), (0, 7, 3), (0, 39, 1023), (0, 12, 517), (0, 4, 64), (0, 25, 901)], np.int32)
    o_ref, A_ref = oracle.pooled_map(bits(x["q"]), bits(x["k"]), bits(x["v"]), units=units)
    check_o(gather_units(o.cpu(), units), o_ref, "O(map)@64k")
    Ag = np.stack([A[b, h, i].cpu().numpy() for b, h, i in units])
    check_rel(Ag, A_ref, "A@64k")


def test_prefill_repeated_calls_block_attribution(oracle):
    """V one-hot in the key block: column j of O is the attention weight on block j,
    so a PV result read before it is complete, or a stale V tile, shows up as a
    wrong column while the all-ones column stays 1.  Repeated calls catch races
    (g=1, odd nb, sparse rows without a forced diagonal)."""
    B, Hq, Hkv, S, d = 1, 3, 3, 1984, 64
    nb = S // BLOCK
    w = syn.custom("onehot", B, Hq, Hkv, S, d, number=7 + S + Hq)
    x = syn.make_inputs(w)
    v = torch.zeros((B, Hkv, S, d))
    v[:, :, torch.arange(S), torch.arange(S) // BLOCK] = 1.0
    v[:, :, :, 40] = 1.0
    v = v.to(torch.bfloat16)
    mask = syn.random_mask(B, Hq, nb, 0.15, seed=S + 3, force_first=True, force_diag=False)
    o_ref, _ = oracle.masked_attention(bits(x["q"]), bits(x["k"]), bits(v), mask.numpy())
    q, k, vd, md = dev(x["q"]), dev(x["k"]), dev(v), dev(mask)
    for _ in range(12):
        o = seer.seer_block_sparse_prefill(q, k, vd, md)
        seer.seer_check_status()
        check_o(o.cpu().reshape(-1, BLOCK, d), o_ref, "O(one-hot V)")


# ------------------------------------------------------------------ distillation target and loss
@pytest.mark.parametrize("name", ["tiny", "map"])
def test_distill_loss(oracle, name):
    if name == "tiny":
        w = syn.WORKLOADS["tiny"]
    else:
        w = syn.custom("distill", 1, 5, 1, 2048, 128, number=81)
    x = syn.make_inputs(w)
    q, k, v = dev(x["q"]), dev(x["k"]), dev(x["v"])
    G = seer.seer_gate_scores(q, k, dev(x["wq"]), dev(x["wk"]), rope_theta=w.rope_theta)
    _, A = seer.seer_attn_pooled_map(q, k, v)
    loss, rows, an = seer.seer_distill_loss(G, A, want_norm=True, Hkv=w.Hkv, d=w.d)
    seer.seer_check_status()
    ahat_ref, rows_ref, heads_ref = oracle.distill_loss(G.cpu().numpy(), A.cpu().numpy())
    check_rel(an.cpu().numpy(), ahat_ref, "A_norm")
    check_rel(rows.cpu().numpy(), rows_ref, "loss rows")
    check_rel(loss.cpu().numpy(), heads_ref, "loss")
    # reproducible
    loss2, _, _ = seer.seer_distill_loss(G, A, Hkv=w.Hkv, d=w.d)
    assert torch.equal(loss, loss2)
    # and the whole chain against the oracle's own gate and map (fp64)
    if name == "tiny":
        Go = oracle.gate_scores(bits(x["q"]), bits(x["k"]), bits(x["wq"]), bits(x["wk"]), theta=w.rope_theta)
        _, Ao = oracle.pooled_map(bits(x["q"]), bits(x["k"]), bits(x["v"]))
        _, _, heads_o = oracle.distill_loss(Go.astype(np.float32), Ao.reshape(Go.shape).astype(np.float32))
        check_rel(loss.cpu().numpy(), heads_o, "loss (oracle chain)")


# ------------------------------------------------------------------ host-memory pipeline
@pytest.mark.parametrize("B,Hq,Hkv,S,d", [(1, 8, 2, 4096, 128), (2, 4, 1, 2000, 64)])
def test_host_prefill_matches_whole_layer_calls(oracle, B, Hq, Hkv, S, d):
    """Group-by-group processing with overlapped copies gives the same bits as
    one whole-layer call of each entry point."""
    w = syn.custom("hostpipe", B, Hq, Hkv, S, d, number=401 + S)
    x = syn.make_inputs(w)
    hq, hk, hv, hwq, hwk = (x[n].pin_memory() for n in ("q", "k", "v", "wq", "wk"))
    ho = torch.empty(hq.shape, dtype=torch.bfloat16).pin_memory()
    hp = seer.HostPrefill(B, Hq, Hkv, S, d, w.d_gate)
    for _ in range(2):                    # the second call reuses the buffers
        ho.zero_()
        hp.run(hq, hk, hv, hwq, hwk, ho, density=0.2, rope_theta=w.rope_theta)
        torch.cuda.synchronize()
    seer.seer_check_status()
    s = seer.seer_gate_scores(dev(x["q"]), dev(x["k"]), dev(x["wq"]), dev(x["wk"]), rope_theta=w.rope_theta)
    m = seer.seer_block_mask(s, "topk", density=0.2, Hkv=Hkv, d=d)
    o = seer.seer_block_sparse_prefill(dev(x["q"]), dev(x["k"]), dev(x["v"]), m)
    torch.cuda.synchronize()
    assert torch.equal(hp.mask.cpu(), m.cpu())
    assert torch.equal(ho, o.cpu())


# ------------------------------------------------------------------ every output element written
def test_outputs_fully_written_over_poison():
    """Outputs pre-filled with NaN (0xFF for the mask) come back finite and equal
    to the results of calls on zero-filled outputs: no tile, row or tail block of
    any output is left unwritten (ragged S, GQA, decode included)."""
    B, Hq, Hkv, S, d = 1, 4, 2, 7 * BLOCK + 29, 128
    nb = -(-S // BLOCK)
    w = syn.custom("poison", B, Hq, Hkv, S, d, number=431)
    x = syn.make_inputs(w)
    q, k, v, wq, wk = (dev(x[n]) for n in ("q", "k", "v", "wq", "wk"))
    nan = float("nan")

    s_p = torch.full((B, Hq, nb, nb), nan, dtype=torch.float32, device="cuda")
    seer.seer_gate_scores(q, k, wq, wk, rope_theta=w.rope_theta, scores=s_p)
    s_z = seer.seer_gate_scores(q, k, wq, wk, rope_theta=w.rope_theta)
    m_p = torch.full((B, Hq, nb, nb), 255, dtype=torch.uint8, device="cuda")
    seer.seer_block_mask(s_z, "topk", density=0.3, mask=m_p, Hkv=Hkv, d=d)
    m_z = seer.seer_block_mask(s_z, "topk", density=0.3, Hkv=Hkv, d=d)
    o_p = torch.full_like(q, nan)
    lse_p = torch.full((B, Hq, S), nan, dtype=torch.float32, device="cuda")
    seer.seer_block_sparse_prefill(q, k, v, m_z, o=o_p, lse=lse_p)
    o_z, lse_z = seer.seer_block_sparse_prefill(q, k, v, m_z, return_lse=True)
    om_p = torch.full_like(q, nan)
    A_p = torch.full((B, Hq, nb, nb), nan, dtype=torch.float32, device="cuda")
    seer.seer_attn_pooled_map(q, k, v, o=om_p, A=A_p)
    om_z, A_z = seer.seer_attn_pooled_map(q, k, v)
    q_tok = q[:, :, -1].contiguous()
    ds = seer.seer_decode_gate_scores(q_tok, k, wq, wk, rope_theta=w.rope_theta)
    dm = seer.seer_decode_block_mask(ds, "topk", density=0.3)
    do_p = torch.full_like(q_tok, nan)
    dl_p = torch.full((B, Hq), nan, dtype=torch.float32, device="cuda")
    seer.seer_block_sparse_decode(q_tok, k, v, dm, o=do_p, lse=dl_p)
    do_z, dl_z = seer.seer_block_sparse_decode(q_tok, k, v, dm, return_lse=True)
    torch.cuda.synchronize()
    seer.seer_check_status()

    assert torch.isfinite(s_p).all() and torch.equal(s_p, s_z)
    assert int(m_p.max()) <= 1 and torch.equal(m_p, m_z)
    assert not torch.triu(m_p.view(-1, nb, nb).to(torch.int32), diagonal=1).any()
    assert torch.isfinite(o_p.float()).all() and torch.equal(o_p, o_z)
    assert torch.isfinite(lse_p).all() and torch.equal(lse_p, lse_z)
    assert torch.isfinite(om_p.float()).all() and torch.equal(om_p, om_z)
    assert torch.isfinite(A_p).all() and torch.equal(A_p, A_z)
    assert torch.isfinite(do_p.float()).all() and torch.equal(do_p, do_z)
    assert torch.isfinite(dl_p).all() and torch.equal(dl_p, dl_z)
