"""Host-side checks of the C ABI: the library loads, exports every symbol
include/seer.h declares, and rejects bad arguments before touching a GPU.
No test here launches a kernel."""
import ctypes
import os
import re

import pytest

import long_context_prefill_attngate_b200 as seer
from long_context_prefill_attngate_b200 import build as seer_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "seer.h")


@pytest.fixture(scope="module")
def L():
    seer_build.build()
    return seer.lib()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"SEER_API\s+[\w\s\*]+?\b(seer_\w+)\s*\(", text)))


def test_header_declares_expected_calls():
    names = declared_symbols()
    for want in ("seer_gate_scores", "seer_block_mask", "seer_block_sparse_prefill", "seer_attn_pooled_map",
                 "seer_compact_mask", "seer_workspace_bytes", "seer_check_status", "seer_last_error"):
        assert want in names
    assert sorted(names) == sorted(seer.EXPORTS)


def test_library_exports_every_declared_symbol(L):
    for name in declared_symbols():
        assert hasattr(L, name), name
    assert seer.seer_version().startswith("seer-b200")


def test_workspace_sizes(L):
    sh = seer.seer_shape(1, 32, 8, 32768, 128)
    nb = 512
    gate = seer.seer_workspace_bytes(seer.SEER_CALL_GATE_SCORES, sh)
    assert gate >= 4 * 40 * nb * (128 + 128)
    assert seer.seer_workspace_bytes(seer.SEER_CALL_BLOCK_SPARSE_PREFILL, sh) == 0
    assert seer.seer_workspace_bytes(seer.SEER_CALL_ATTN_POOLED_MAP, sh) == 4 * 296 * nb * 128
    assert seer.seer_workspace_bytes(7, sh) == 0
    assert "unknown call" in seer.seer_last_error()


@pytest.mark.parametrize("shape,status,msg", [
    ((1, 2, 2, 64 * 16384 + 1, 64), seer.SEER_ERR_UNSUPPORTED, "exceeds"),
    ((1, 32, 8, 4096, 96), seer.SEER_ERR_UNSUPPORTED, "head dim"),
    ((1, 30, 8, 4096, 128), seer.SEER_ERR_INVALID_ARG, "multiple of Hkv"),
    ((0, 32, 8, 4096, 128), seer.SEER_ERR_INVALID_ARG, "positive"),
    ((1, 2, 2, 64 * 20000, 64), seer.SEER_ERR_UNSUPPORTED, "exceeds"),
    ((2048, 32, 8, 64, 64), seer.SEER_ERR_UNSUPPORTED, "exceeds 65535"),
])
def test_shape_rejections(L, shape, status, msg):
    sh = seer.seer_shape(*shape)
    fake = ctypes.c_void_p(0x10000)
    st = L.seer_block_sparse_prefill(ctypes.byref(sh), fake, fake, fake, fake, 0.0, fake, None, None, 0, None)
    assert st == status
    assert msg in seer.seer_last_error()


def test_null_and_misaligned_pointers_rejected(L):
    sh = seer.seer_shape(1, 2, 2, 512, 64)
    good = ctypes.c_void_p(0x10000)
    odd = ctypes.c_void_p(0x10008)
    st = L.seer_block_sparse_prefill(ctypes.byref(sh), None, good, good, good, 0.0, good, None, None, 0, None)
    assert st == seer.SEER_ERR_INVALID_ARG
    st = L.seer_block_sparse_prefill(ctypes.byref(sh), odd, good, good, good, 0.0, good, None, None, 0, None)
    assert st == seer.SEER_ERR_INVALID_ARG and "aligned" in seer.seer_last_error()
    st = L.seer_block_sparse_prefill(ctypes.byref(sh), good, good, good, None, 0.0, good, None, None, 0, None)
    assert st == seer.SEER_ERR_INVALID_ARG and "mask" in seer.seer_last_error()
    st = L.seer_attn_pooled_map(ctypes.byref(sh), good, good, good, 0.0, good, None, None, 0, None)
    assert st == seer.SEER_ERR_INVALID_ARG
    st = L.seer_attn_pooled_map(ctypes.byref(sh), good, good, good, 0.0, good, good, None, 0, None)
    assert st == seer.SEER_ERR_WORKSPACE or st == seer.SEER_ERR_CUDA


def test_gate_and_mask_argument_checks(L):
    sh = seer.seer_shape(1, 2, 2, 512, 64)
    p = ctypes.c_void_p(0x10000)
    gp = seer.seer_gate_params(63, 5e5, 64 * 63, 64 * 63)
    assert L.seer_gate_scores(ctypes.byref(sh), p, p, p, p, ctypes.byref(gp), p, p, 1 << 30, None) == \
        seer.SEER_ERR_UNSUPPORTED
    gp = seer.seer_gate_params(64, -1.0, 0, 0)
    assert L.seer_gate_scores(ctypes.byref(sh), p, p, p, p, ctypes.byref(gp), p, p, 1 << 30, None) == \
        seer.SEER_ERR_INVALID_ARG
    gp = seer.seer_gate_params(64, 5e5, 0, 0)
    assert L.seer_gate_scores(ctypes.byref(sh), p, p, p, p, ctypes.byref(gp), p, p, 16, None) == \
        seer.SEER_ERR_WORKSPACE
    mp = seer.seer_mask_params(9, 0.0, 0.0, 0, None, 1, 1)
    assert L.seer_block_mask(ctypes.byref(sh), p, ctypes.byref(mp), p, None) == seer.SEER_ERR_INVALID_ARG
    mp = seer.seer_mask_params(seer.SEER_MASK_TOPK, 0.0, float("nan"), 0, None, 1, 1)
    assert L.seer_block_mask(ctypes.byref(sh), p, ctypes.byref(mp), p, None) == seer.SEER_ERR_INVALID_ARG
    assert L.seer_compact_mask(ctypes.byref(sh), None, p, p, None) == seer.SEER_ERR_INVALID_ARG


@pytest.mark.parametrize("ff,fd", [(True, True), (True, False), (False, True), (False, False)])
def test_topk_from_density_matches_oracle(oracle, ff, fd):
    """The C library's per-row TopK counts equal the oracle's k_i rule for
    densities across [0, 1] (including values whose products are exact
    integers, where ceil is most fragile), above 1, and nb up to the maximum."""
    densities = [0.0, 1e-6, 0.1, 0.17, 0.2, 0.25, 0.3, 1.0 / 3.0, 0.5, 0.7, 0.9, 0.999, 1.0, 1.5]
    for nb in (1, 2, 33, 512, 16384):
        for density in densities:
            got = seer.seer_topk_from_density(density, nb, ff, fd)
            if nb <= 512 or density in (0.1, 1.0 / 3.0, 1.0):
                want = oracle.topk_counts(density, nb, force_first=ff, force_diag=fd)
                assert got == list(want), (nb, density)
            assert all(1 <= k <= i + 1 for i, k in enumerate(got)) or not (ff or fd)


def test_topk_from_density_rejects_bad_arguments(L):
    out = (ctypes.c_int32 * 4)(7, 7, 7, 7)
    for density, nb in ((float("nan"), 4), (-0.5, 4), (float("inf"), 4), (0.5, 0), (0.5, 16385)):
        assert L.seer_topk_from_density(ctypes.c_double(density), nb, 1, 1, out) == seer.SEER_ERR_INVALID_ARG
    assert list(out) == [7, 7, 7, 7]
    assert L.seer_topk_from_density(ctypes.c_double(0.5), 4, 1, 1, None) == seer.SEER_ERR_INVALID_ARG


def test_ragged_sequence_accepted(L):
    """S that is not a multiple of 64: nb = ceil(S/64), the gate workspace
    covers that many blocks and the shape passes the argument checks."""
    sh = seer.seer_shape(1, 4, 2, 100, 64)
    ws = seer.seer_workspace_bytes(seer.SEER_CALL_GATE_SCORES, sh)
    assert ws >= 4 * (4 * 2 * (64 + 256) + 2 * 2 * (128 + 256))
    assert seer.seer_workspace_bytes(seer.SEER_CALL_ATTN_POOLED_MAP, sh) == 4 * 296 * 2 * 128
