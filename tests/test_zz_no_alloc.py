"""dg_vocab_attention_static: vocabulary attention with the library's own scratch.

Callers that cannot call cudaMalloc (a host callback, a plugin whose framework
owns all device memory, a process that must not grow its device footprint)
use this entry point; it takes its scratch from a fixed device array inside
libdg.so. Its outputs must match what a CUDA-core context computes for the same
hidden state through dg_denoise_step_h, on two calls in a row (the second call
finds the first call's leftovers in the shared array), and the second call
must leave the device's free memory exactly as it found it.
"""
import numpy as np
import pytest
import torch

import synthetic
import uniform_state_text_b200 as dg
from parity import H_ATOL, SC_RTOL, sc_rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from uniform_state_text_b200 import build
    build.build()
    dg.lib()


def _static(w, scale, E, h, stream):
    """One call of the allocation-free entry point; returns its outputs and the
    change of the device's free memory across the call (outputs allocated and
    the device synchronised before the first reading)."""
    H = torch.empty(w.C, dtype=torch.float32, device="cuda")
    amax = torch.empty(w.C, dtype=torch.int32, device="cuda")
    sc = torch.empty(w.C, w.d, dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    dg.dg_vocab_attention_static(w.C, w.V, w.d, dg.DG_BF16 if w.dtype == "bf16" else dg.DG_F32,
                                 scale, E.data_ptr(), h.data_ptr(), H.data_ptr(), amax.data_ptr(),
                                 sc.data_ptr(), stream.cuda_stream)
    stream.synchronize()
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    return H.cpu().numpy(), amax.cpu().numpy(), sc.cpu().numpy().astype(np.float64), free0 - free1


@pytest.mark.parametrize("shape", [(128, 8192, 512, "bf16"), (16, 512, 64, "f32")])
def test_static_scratch_matches_workspace_path(shape):
    C, V, d, dt = shape
    w = synthetic.SMALL.replace(C=C, V=V, d=d, dtype=dt, tau=0.5 * C * np.log(2), max_steps=2,
                                coef_target=1.0, coef_canvas=0.5, logit_scale=2.0)
    E = synthetic.make_embedding(w).cuda()
    den = dg.Denoiser(w, E, impl=dg.DG_IMPL_SIMT)
    den.step()                                     # a stand-in hidden state to work on
    h = den.read(dg.DG_HIDDEN).contiguous()
    den.begin_block(0)
    den.step_h(h)                                  # the existing entry point, step 0
    H_ref = den.read(dg.DG_ENTROPY).cpu().numpy()
    a_ref = den.read(dg.DG_ARGMAX).cpu().numpy()
    sc_ref = den.read(dg.DG_SC).cpu().numpy().astype(np.float64)
    scale = float(np.float32(w.logit_scale / w.T_start))
    stream = torch.cuda.Stream()
    for call in range(2):
        H, amax, sc, grew = _static(w, scale, E, h, stream)
        if call == 1:                              # the first call may load the module
            assert grew == 0, f"device memory in use grew by {grew} bytes"
        assert np.abs(H - H_ref).max() <= H_ATOL, call
        assert np.array_equal(amax, a_ref), call
        assert sc_rel_err(sc, sc_ref).max() <= SC_RTOL, call
    den.close()


def test_static_scratch_rejects_oversized_problems():
    w = synthetic.HEADLINE
    with pytest.raises(dg.DgError) as e:
        dg.dg_vocab_attention_static(w.C, w.V, w.d, dg.DG_BF16, 1.0, 1, 1, 1, 1, 1, 0)
    assert e.value.code == dg.DG_EUNSUPPORTED
    assert "scratch" in dg.dg_last_error(None)
