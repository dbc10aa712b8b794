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


def _noalloc_bytes(wl) -> int:
    """Scratch the allocation-free call needs, by the rule its header states: h
    (T*k*I f32, rounded up to 256 bytes), then T records of x rounded up to 256
    bytes, then T*k records of h; a record of a row of K values takes
    3K + 4(K/32) + 12(K/32) bytes (f32: three digit planes, a scale and three
    corrections per 32-block, each part rounded up to 16 bytes)."""
    a256 = lambda v: (v + 255) // 256 * 256
    a16 = lambda v: (v + 15) // 16 * 16
    rec = lambda K: 3 * K + a16(4 * (K // 32)) + a16(12 * (K // 32))
    A = wl.T * wl.top_k
    return a256(A * wl.inter * 4) + a256(wl.T * rec(wl.hidden)) + A * rec(wl.inter)


LIMIT = 8 << 20          # the library's fixed array
GLM16 = W.GLM_DECODE_T1.with_(n_experts=16)


@pytest.mark.parametrize("wl", [W.TINY, W.TINY.with_(afmt=W.A_Q8, T=5), W.TINY.with_(T=1),
                                GLM16.with_(T=4), GLM16.with_(T=58)],
                         ids=["tiny_f32", "tiny_q8_t5", "tiny_t1", "glm_shaped_e16_t4",
                              "glm_shaped_e16_t58_largest"])
def test_noalloc_matches_workspace_version(dev, wl):
    """Two calls in a row, with different routing, give exactly the workspace
    version's bytes: both run the same kernels on the same inputs, so any
    difference would be a scratch aliasing or offset error.  T = 58 is the
    largest batch the array takes at this shape (the scratch then fills all but
    14 KB of it), so an offset error there would run past its end; the
    bounds-checked build (QRX_CHECK=1) checks those runs too."""
    if wl.T == 58:
        assert _noalloc_bytes(wl) <= LIMIT < _noalloc_bytes(wl.with_(T=59))
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
        assert np.array_equal(got.view(np.uint32), ref.view(np.uint32)), batch


def test_noalloc_refuses_sizes_above_its_array(dev):
    """T = 59 at the GLM shape needs more than the 8 MiB array (h: 59*8*2048*4 B,
    x records: 59*21504 B, h records: 472*7168 B, 8,518,656 B in all): the call
    returns QRX_ENOSPACE before any launch."""
    wl = GLM16.with_(T=59)
    assert _noalloc_bytes(wl) > LIMIT
    c = qrx.cfg_of(wl)
    ex = qrx.Experts.empty(16, wl.hidden, wl.inter, 4)
    perm = qrx.Perm.empty(wl.T, wl.top_k, wl.n_experts)
    x = torch.zeros((wl.T, wl.hidden), dtype=torch.float32, device="cuda")
    y = torch.empty((wl.T * wl.top_k, wl.hidden), dtype=torch.float32, device="cuda")
    with pytest.raises(qrx.QrxError) as ei:
        qrx.qrx_expert_ffn_noalloc(c, ex, perm, wl.T, y, x=x)
    assert ei.value.code == qrx.QRX_ENOSPACE
