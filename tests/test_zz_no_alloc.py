"""seer_gate_scores_noalloc, the gate-scores call for callers that cannot
allocate device memory (an application whose memory pool owns the device, or
a path that must not call cudaMalloc): it takes only inputs and outputs and
uses a fixed scratch array inside the library.  This file is collected last
so that a run stopping at the first failure has run everything else first.
"""
import ctypes

import numpy as np
import pytest
import torch

import long_context_prefill_attngate_b200 as seer
from long_context_prefill_attngate_b200 import build as seer_build
from long_context_prefill_attngate_b200 import synthetic as syn

pytestmark = pytest.mark.gpu

REL = 1e-2      # the gate-score tolerance used by the parity tests


def test_gate_scores_noalloc_matches_workspace_call():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    seer_build.build()
    L = seer.lib()
    w = syn.custom("noalloc", 1, 8, 2, 4096, 128, number=61)
    x = syn.make_inputs(w)
    q, k, wq, wk = (x[n].cuda().contiguous() for n in ("q", "k", "wq", "wk"))
    ref = seer.seer_gate_scores(q, k, wq, wk, rope_theta=w.rope_theta)   # caller-provided workspace
    seer.seer_check_status()
    ref_np = ref.cpu().numpy()
    sh = seer.shape_of(q, k)
    gp = seer.seer_gate_params(w.d_gate, w.rope_theta, w.d * w.d_gate, w.d * w.d_gate)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):          # two calls in a row share the library's scratch
        out = torch.full_like(ref, float("nan"))
        st = L.seer_gate_scores_noalloc(ctypes.byref(sh), q.data_ptr(), k.data_ptr(), wq.data_ptr(),
                                        wk.data_ptr(), ctypes.byref(gp), out.data_ptr(), stream)
        assert st == seer.SEER_OK, seer.seer_last_error()
        seer.seer_check_status()
        got = out.cpu().numpy()
        assert np.isfinite(got).all()
        assert np.all(np.abs(got - ref_np) <= REL * np.abs(ref_np) + 1e-12)


def test_gate_scores_noalloc_rejects_oversized_shape():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    L = seer.lib()
    big = seer.seer_shape(1, 32, 8, 131072, 128)      # needs ~84 MB of gate scratch
    gp = seer.seer_gate_params(128, 5e5, 128 * 128, 128 * 128)
    fake = ctypes.c_void_p(0x10000)
    # scores = NULL as well: even if the size check were missing, nothing could launch.
    st = L.seer_gate_scores_noalloc(ctypes.byref(big), fake, fake, fake, fake, ctypes.byref(gp), None, None)
    assert st == seer.SEER_ERR_UNSUPPORTED
    assert "scratch" in seer.seer_last_error()


def test_gate_scores_noalloc_maxmin_k_matches_workspace_call():
    """K pooled by [max | min]: the K workspace region is 2d wide."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    w = syn.custom("noallocmm", 1, 4, 2, 2048, 128, number=53)
    x = syn.make_inputs(w)
    g = torch.Generator().manual_seed(53)
    wk = (torch.randn((2, 256, 128), generator=g) * 0.07).to(torch.bfloat16).cuda()
    q, k, wq = (x[n].cuda().contiguous() for n in ("q", "k", "wq"))
    a = seer.seer_gate_scores(q, k, wq, wk, rope_theta=w.rope_theta, k_maxmin=True)
    b = seer.seer_gate_scores_noalloc(q, k, wq, wk, rope_theta=w.rope_theta, k_maxmin=True)
    seer.seer_check_status()
    assert torch.equal(a, b)
