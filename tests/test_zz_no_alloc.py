"""The allocation-free routed FFN (qrx_expert_ffn_noalloc) against qrx_expert_ffn.

Some callers cannot allocate device memory when they call in (a host whose
allocator owns the whole device budget, a plug-in given no allocator), so they
cannot pass a workspace.  qrx_expert_ffn_noalloc keeps its scratch in a fixed
array inside the library instead.  This file checks, through the C ABI, that
two calls in a row give the same result as the workspace version on the same
inputs, and that a size above the array's limit is refused before any launch.
It is named to be collected last and builds everything it needs itself, so it
passes both alone in a fresh process and after the other GPU tests.
"""
import numpy as np
import pytest
import torch

from quantized_routed_expert_tc_b200 import build as qbuild, qrx, workloads as W
from quantized_routed_expert_tc_b200.layer import (GpuLayer, activations, router_weights,
                                                   to_device_act)
from tests.harness import TOL, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    qbuild.build(check=qrx.lib_path() == qbuild.CHECK_LIB)    # the library the binding loads
    torch.cuda.set_device(0)
    return torch.device("cuda:0")


def _routed_inputs(glay, wl, batch):
    """Route one batch and build its permutation (through the library)."""
    c = qrx.cfg_of(wl)
    T = wl.T
    x = to_device_act(wl, activations(wl, T, batch=batch))
    _, bias = router_weights(wl)
    idx = torch.empty((T, wl.top_k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, wl.top_k), dtype=torch.float32, device="cuda")
    ws = qrx.workspace(c, T)
    qrx.qrx_route(c, x, glay.Wr, torch.from_numpy(bias).cuda(), idx, w, ws)
    perm = qrx.Perm.empty(T, wl.top_k, wl.n_experts)
    qrx.qrx_permute(c, idx, perm)
    kw = dict(x=x)
    if wl.afmt == W.A_Q8:
        xq = torch.empty((T, wl.hidden), dtype=torch.int8, device="cuda")
        xd = torch.empty((T, wl.hidden // 32), dtype=torch.float32, device="cuda")
        qrx.qrx_quantize_act_q8(x, xq, xd)
        kw = dict(xq=xq, xd=xd)
    return c, perm, kw, ws


@pytest.mark.parametrize("wl", [W.TINY, W.TINY.with_(afmt=W.A_Q8, T=5),
                                W.GLM_DECODE_T1.with_(n_experts=16, T=4)],
                         ids=["tiny_f32", "tiny_q8_t5", "glm_shaped_e16_t4"])
def test_noalloc_matches_workspace_version(dev, wl):
    glay = GpuLayer(wl)
    routed = glay.routed[wl.wbits]
    A = wl.T * wl.top_k
    for batch in (0, 1):                   # two calls in a row, different routing
        c, perm, kw, ws = _routed_inputs(glay, wl, batch)
        y_ref = torch.empty((A, wl.hidden), dtype=torch.float32, device="cuda")
        qrx.qrx_expert_ffn(c, routed, perm, wl.T, y_ref, ws, **kw)
        y = torch.full((A, wl.hidden), float("nan"), dtype=torch.float32, device="cuda")
        qrx.qrx_expert_ffn_noalloc(c, routed, perm, wl.T, y, **kw)
        torch.cuda.synchronize()
        assert qrx.qrx_last_error() == qrx.QRX_OK
        got, ref = y.cpu().numpy(), y_ref.cpu().numpy()
        assert np.isfinite(got).all()
        assert rel_err(got, ref) <= TOL


def test_noalloc_refuses_sizes_above_its_array(dev):
    wl = W.GLM_DECODE_T1.with_(n_experts=16, T=97)      # 97 * (65536 + 21504) B > 8 MiB
    c = qrx.cfg_of(wl)
    ex = qrx.Experts.empty(16, wl.hidden, wl.inter, 4)
    perm = qrx.Perm.empty(wl.T, wl.top_k, wl.n_experts)
    x = torch.zeros((wl.T, wl.hidden), dtype=torch.float32, device="cuda")
    y = torch.empty((wl.T * wl.top_k, wl.hidden), dtype=torch.float32, device="cuda")
    with pytest.raises(qrx.QrxError) as ei:
        qrx.qrx_expert_ffn_noalloc(c, ex, perm, wl.T, y, x=x)
    assert ei.value.code == qrx.QRX_ENOSPACE
