"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Rules: integer, index and byte results bit-exact (expert indices up to counted
near-ties, where the oracle's selection is then fed to the later stages); f32
outputs max|gpu - oracle| <= 1e-3 * max|oracle|.  Sizes span the tiny layer
(every format and activation mode, ragged T) and the full GLM-shaped layer
(decode, Q8_0 decode batch, verify and prefill batches, the format sweep), at
full size on sampled tokens the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

import oracle
from quantized_routed_expert_tc_b200 import build as qbuild, qrx, synth, workloads as W
from quantized_routed_expert_tc_b200.layer import (GpuLayer, activations, router_weights,
                                                   to_device_act)
from tests.harness import TOL, OracleLayer, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="session")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    qbuild.build(check=qrx.lib_path() == qbuild.CHECK_LIB)    # the library the binding loads
    torch.cuda.set_device(0)
    assert qrx.qrx_last_error() == qrx.QRX_OK
    return torch.device("cuda:0")


@pytest.fixture(scope="session")
def tiny(dev):
    return GpuLayer(W.TINY, formats=(8, 4, 2)), OracleLayer(W.TINY)


@pytest.fixture(scope="session")
def small_tc(dev):
    return GpuLayer(W.SMALL_TC, formats=(4,)), OracleLayer(W.SMALL_TC)


@pytest.fixture(scope="session")
def glm(dev):
    return GpuLayer(W.GLM_DECODE_T1, formats=(4, 8, 2)), OracleLayer(W.GLM_DECODE_T1)


def cu(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def np_(t):
    return t.detach().cpu().numpy()


def check_routing(r, idx_gpu, w_gpu):
    """Expert indices bit-exact except counted near-ties; weights of matching tokens."""
    idx_gpu, w_gpu = np.asarray(idx_gpu), np.asarray(w_gpu)
    ties = []
    for t in range(idx_gpu.shape[0]):
        if np.array_equal(idx_gpu[t], r["idx"][t]):
            assert np.allclose(w_gpu[t], r["w"][t], rtol=2e-7, atol=0), t
        else:
            assert r["ties"][t] != 0, f"token {t}: selection differs without a near-tie"
            ties.append(t)
    return ties


def gpu_layer(glay, wl, x_np, bias=None, bits=None, topp=0.0, usage=None):
    """Whole layer through qrx_moe_forward; returns (idx, w, out) on the host."""
    bits = wl.wbits if bits is None else bits
    cfg = qrx.cfg_of(wl.with_(wbits=bits))
    T = x_np.shape[0]
    x = to_device_act(wl, x_np)
    idx = torch.empty((T, wl.top_k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, wl.top_k), dtype=torch.float32, device="cuda")
    out = torch.empty((T, wl.hidden), dtype=torch.float32, device="cuda")
    ws = qrx.workspace(cfg, T)
    qrx.qrx_moe_forward(cfg, x, glay.Wr, glay.bias if bias is None else bias,
                        glay.routed[bits], glay.shared[bits], idx, w, out, ws, topp=topp, usage=usage)
    torch.cuda.synchronize()
    assert qrx.qrx_last_error() == qrx.QRX_OK
    return np_(idx), np_(w), np_(out)


def gpu_staged(glay, wl, x_np, idx_np, w_np, bits=None):
    """The layer by stages from a given selection (used to resolve near-ties)."""
    bits = wl.wbits if bits is None else bits
    c = qrx.cfg_of(wl.with_(wbits=bits))
    T = x_np.shape[0]
    ws = qrx.workspace(c, T)
    perm = qrx.Perm.empty(T, wl.top_k, wl.n_experts)
    qrx.qrx_permute(c, cu(idx_np.astype(np.int32)), perm)
    x = to_device_act(wl, x_np)
    kw = dict(x=x)
    if wl.afmt == W.A_Q8:
        xq = torch.empty((T, wl.hidden), dtype=torch.int8, device="cuda")
        xd = torch.empty((T, wl.hidden // 32), dtype=torch.float32, device="cuda")
        qrx.qrx_quantize_act_q8(x, xq, xd)
        kw = dict(xq=xq, xd=xd)
    A = T * wl.top_k
    ys = torch.empty((A, wl.hidden), dtype=torch.float32, device="cuda")
    ysh = torch.empty((T, wl.hidden), dtype=torch.float32, device="cuda")
    qrx.qrx_expert_ffn(c, glay.routed[bits], perm, T, ys, ws, **kw)
    qrx.qrx_shared_ffn(c, glay.shared[bits], T, ysh, ws, **kw)
    out = torch.empty((T, wl.hidden), dtype=torch.float32, device="cuda")
    qrx.qrx_combine(c, ys, ysh, cu(w_np.astype(np.float32)), perm.inv, out)
    torch.cuda.synchronize()
    assert qrx.qrx_last_error() == qrx.QRX_OK
    return np_(out)


def check_layer(glay, olay, wl, x_np, tokens, bits=None, bias_np=None, topp=0.0):
    """Whole-layer parity on the listed tokens (near-ties resolved by the oracle)."""
    bits = wl.wbits if bits is None else bits
    wlb = wl.with_(wbits=bits)
    bias_np = router_weights(wl)[1] if bias_np is None else bias_np
    idx, w, out = gpu_layer(glay, wlb, x_np, bias=cu(bias_np), bits=bits, topp=topp)
    r, ref = olay.forward_tokens(wlb, x_np, tokens, bias=bias_np, topp=topp)
    ties = check_routing(r, idx, w)
    got = out[list(tokens)]
    if ties:
        staged = gpu_staged(glay, wlb, x_np, r["idx"], r["w"], bits)
        got = staged[list(tokens)]
    e = rel_err(got, ref)
    assert e <= TOL, f"{wl.name} int{bits}: rel err {e:.3g}"
    return dict(rel_err=e, ties=len(ties), idx=idx, out=out)


# ------------------------------------------------------------------ bit-exact kernels
@pytest.mark.parametrize("bits", [8, 4, 2])
def test_quantize_weights_bitexact(dev, bits):
    for K in (256, 6144):
        w = synth.normal_f32(71, bits, 40 * K, 0.0, 0.02).reshape(40, K)
        w[1] = 0.0
        w[2] = (np.arange(K) % 16 - 7.5).astype(np.float32) * 2 ** -4   # exact halves
        w[3, :] = 1e-30
        w[3, 5] = -3e-30
        q_ref, s_ref = oracle.quantize_rows(w, bits)
        q = torch.zeros((40, K * bits // 8), dtype=torch.uint8, device="cuda")
        s = torch.zeros(40, dtype=torch.float32, device="cuda")
        qrx.qrx_quantize_weights(cu(w), bits, q, K * bits // 8, s, 1)
        torch.cuda.synchronize()
        assert np.array_equal(np_(q), q_ref)
        assert np.array_equal(np_(s).view(np.uint32), s_ref.view(np.uint32))


def test_quantize_act_q8_bitexact(dev):
    T, H = 33, 6144
    x = synth.normal_f32(72, 0, T * H).reshape(T, H)
    x[0, :32] = 0.0
    x[1, 32:64] = 1e-38
    x[2, :32] = np.arange(32, dtype=np.float32) * 0.0625 - 1.0    # exact multiples
    q_ref, d_ref = oracle.quantize_q8(x)
    xq = torch.empty((T, H), dtype=torch.int8, device="cuda")
    xd = torch.empty((T, H // 32), dtype=torch.float32, device="cuda")
    qrx.qrx_quantize_act_q8(cu(x), xq, xd)
    torch.cuda.synchronize()
    assert np.array_equal(np_(xq), q_ref)
    assert np.array_equal(np_(xd).view(np.uint32), d_ref.view(np.uint32))


@pytest.mark.parametrize("bits", [8, 4, 2])
def test_block_dots_bitexact(dev, bits):
    rng = np.random.default_rng(bits)
    for K in (256, 2048, 6144):
        w = synth.normal_f32(73, bits, 24 * K, 0.0, 0.02).reshape(24, K)
        q_ref, _ = oracle.quantize_rows(w, bits)
        xq = rng.integers(-127, 128, size=K).astype(np.int8)
        acc_ref = oracle.block_dots_q8(q_ref, K, bits, xq)
        acc = torch.empty((24, K // 32), dtype=torch.int32, device="cuda")
        qrx.qrx_block_dots_q8(bits, cu(q_ref), K, cu(xq), acc)
        torch.cuda.synchronize()
        assert np.array_equal(np_(acc), acc_ref)


# ------------------------------------------------------------------ exact Q8_0 accumulators
def _q8_block_sums_case(glay, olay, wl, batch):
    """The decode engine's int32 block accumulators of gate/up (from the
    library's Q8_0 codes of x, which equal the oracle's) and of down (from the
    oracle's h, re-quantised by the kernel) against the oracle's exact sums."""
    T, k, H, I, bits = wl.T, wl.top_k, wl.hidden, wl.inter, wl.wbits
    x = activations(wl, T, batch=batch)
    _, bias = router_weights(wl)
    r = oracle.router(wl, x, olay.Wr, bias)
    p = oracle.permute(r["idx"], wl.n_experts)
    xq_o, xd_o = oracle.quantize_q8(x)
    ex = olay.experts(r["idx"].ravel(), bits)
    h_o, _ = oracle.expert_ffn(wl, ex, p, x)
    c = qrx.cfg_of(wl)
    ws = qrx.workspace(c, T)
    perm = qrx.Perm.empty(T, k, wl.n_experts)
    qrx.qrx_permute(c, cu(r["idx"]), perm)
    xq = torch.empty((T, H), dtype=torch.int8, device="cuda")
    xd = torch.empty((T, H // 32), dtype=torch.float32, device="cuda")
    qrx.qrx_quantize_act_q8(cu(x), xq, xd)
    A = T * k
    hs = torch.empty((A, I), dtype=torch.float32, device="cuda")
    acc_gu = torch.full((A, 2, I, H // 32), -7, dtype=torch.int32, device="cuda")
    qrx.qrx_expert_gateup_q8_sums(c, glay.routed[bits], perm, T, hs, acc_gu, ws, xq, xd)
    ys = torch.empty((A, H), dtype=torch.float32, device="cuda")
    acc_d = torch.full((A, H, I // 32), -7, dtype=torch.int32, device="cuda")
    qrx.qrx_expert_down_q8_sums(c, glay.routed[bits], perm, cu(h_o), T, ys, acc_d, ws)
    torch.cuda.synchronize()
    assert qrx.qrx_last_error() == qrx.QRX_OK
    assert np.array_equal(np_(xq), xq_o) and np.array_equal(np_(xd), xd_o)
    acc_gu, acc_d = np_(acc_gu), np_(acc_d)
    flat = r["idx"].ravel()
    for pos in range(A):
        a = int(p["sorted"][pos])
        e, t = int(flat[a]), a // k
        o = ex[e]
        assert np.array_equal(acc_gu[pos, 0], oracle.block_dots_q8(o.gate_q, H, bits, xq_o[t])), (pos, "gate")
        assert np.array_equal(acc_gu[pos, 1], oracle.block_dots_q8(o.up_q, H, bits, xq_o[t])), (pos, "up")
        hq, _ = oracle.quantize_q8(h_o[pos:pos + 1])
        assert np.array_equal(acc_d[pos], oracle.block_dots_q8(o.down_q, I, bits, hq[0])), (pos, "down")
    assert rel_err(np_(hs), h_o) <= TOL


@pytest.mark.parametrize("bits", [8, 4, 2])
@pytest.mark.parametrize("T", [1, 4])
def test_q8_block_sums_bitexact_tiny(tiny, bits, T):
    glay, olay = tiny
    _q8_block_sums_case(glay, olay, W.TINY.with_(wbits=bits, afmt=W.A_Q8, T=T), 40 + T)


@pytest.mark.parametrize("bits", [8, 4, 2])
@pytest.mark.parametrize("T", [1, 4])
def test_q8_block_sums_bitexact_glm(glm, bits, T):
    """At the GLM shape: 2I x 192 gate/up and H x 64 down block sums per position."""
    glay, olay = glm
    _q8_block_sums_case(glay, olay, W.GLM_DECODE_T1.with_(wbits=bits, afmt=W.A_Q8, T=T), 50 + T)


# ------------------------------------------------------------------ router and permutation
def _route_gpu(glay, wl, x_np, bias_np):
    c = qrx.cfg_of(wl)
    T = x_np.shape[0]
    idx = torch.empty((T, wl.top_k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, wl.top_k), dtype=torch.float32, device="cuda")
    ws = qrx.workspace(c, T)
    qrx.qrx_route(c, to_device_act(wl, x_np), glay.Wr, cu(bias_np), idx, w, ws)
    torch.cuda.synchronize()
    return np_(idx), np_(w)


def test_route_tiny(tiny):
    glay, olay = tiny
    for T in (1, 5, 8, 64):
        wl = W.TINY.with_(T=T)
        x = activations(wl, T)
        _, bias = router_weights(wl)
        idx, w = _route_gpu(glay, wl, x, bias)
        check_routing(oracle.router(wl, x, olay.Wr, bias), idx, w)


@pytest.mark.parametrize("wl", [W.GLM_DECODE_T1, W.GLM_DECODE_T32_Q8, W.GLM_VERIFY_T4_BF16,
                                W.GLM_PREFILL_T2048_BF16], ids=lambda w: w.name)
def test_route_glm(glm, wl):
    glay, olay = glm
    x = activations(wl)
    _, bias = router_weights(wl)
    idx, w = _route_gpu(glay, wl, x, bias)
    r = oracle.router(wl, x, olay.Wr, bias)
    ties = check_routing(r, idx, w)
    assert len(ties) <= max(2, wl.T // 50)


def _perm_gpu(idx_np, E):
    T, k = idx_np.shape
    wl = W.TINY.with_(n_experts=E, n_group=1, topk_group=1, top_k=k)
    perm = qrx.Perm.empty(T, k, E)
    qrx.qrx_permute(qrx.cfg_of(wl), cu(idx_np.astype(np.int32)), perm)
    torch.cuda.synchronize()
    return {k_: np_(getattr(perm, k_)) for k_ in ("counts", "offsets", "sorted", "inv",
                                                  "union_ids", "n_union")}


def test_permute_bitexact(dev):
    rng = np.random.default_rng(9)
    for T, k, E in [(1, 8, 256), (7, 4, 16), (64, 8, 256), (2048, 8, 256), (33, 3, 1024),
                    (5, 1, 2)]:
        idx = rng.integers(0, E, size=(T, k)).astype(np.int32)
        if T == 2048:
            idx = (rng.zipf(1.5, size=(T, k)) % E).astype(np.int32)   # skewed load
        ref = oracle.permute(idx, E)
        got = _perm_gpu(idx, E)
        for key in ("counts", "offsets", "sorted", "inv"):
            assert np.array_equal(got[key], ref[key]), (T, k, E, key)
        n = int(got["n_union"][0])
        assert n == ref["n_union"]
        assert np.array_equal(got["union_ids"][:n], ref["union_ids"])


def test_permute_bad_index_sets_device_flag(dev):
    idx = np.array([[0, 3], [16, 1]], dtype=np.int32)        # 16 is outside [0, 16)
    _perm_gpu(idx, 16)
    assert qrx.qrx_last_error() == qrx.QRX_EDEVICE
    assert qrx.qrx_last_error() == qrx.QRX_OK                # the flag was cleared


# ------------------------------------------------------------------ FFN stages, tiny layer
@pytest.mark.parametrize("bits", [8, 4, 2])
@pytest.mark.parametrize("afmt", [W.A_F32, W.A_Q8, W.A_BF16], ids=["f32", "q8", "bf16"])
@pytest.mark.parametrize("T", [1, 5, 8])
def test_stages_tiny(tiny, bits, afmt, T):
    glay, olay = tiny
    wl = W.TINY.with_(wbits=bits, afmt=afmt, T=T)
    x = activations(wl, T)
    _, bias = router_weights(wl)
    r = oracle.router(wl, x, olay.Wr, bias)
    p = oracle.permute(r["idx"], wl.n_experts)
    ex = olay.experts(r["idx"].ravel(), bits)
    h_o, y_o = oracle.expert_ffn(wl, ex, p, x)
    hsh_o, ysh_o = oracle.shared_ffn(wl, olay.shared(bits), x)
    out_o = oracle.combine(wl, y_o, ysh_o, r["w"], p["inv"])

    c = qrx.cfg_of(wl)
    ws = qrx.workspace(c, T)
    perm = qrx.Perm.empty(T, wl.top_k, wl.n_experts)
    qrx.qrx_permute(c, cu(r["idx"]), perm)
    xt = to_device_act(wl, x)
    kw = dict(x=xt)
    if afmt == W.A_Q8:
        xq = torch.empty((T, wl.hidden), dtype=torch.int8, device="cuda")
        xd = torch.empty((T, wl.hidden // 32), dtype=torch.float32, device="cuda")
        qrx.qrx_quantize_act_q8(xt, xq, xd)
        q_ref, d_ref = oracle.quantize_q8(x)
        torch.cuda.synchronize()
        assert np.array_equal(np_(xq), q_ref) and np.array_equal(np_(xd), d_ref)
        kw = dict(xq=xq, xd=xd)
    A = T * wl.top_k
    hs = torch.empty((A, wl.inter), dtype=torch.float32, device="cuda")
    ys = torch.empty((A, wl.hidden), dtype=torch.float32, device="cuda")
    qrx.qrx_expert_ffn(c, glay.routed[bits], perm, T, ys, ws, h_sorted=hs, **kw)
    hsh = torch.empty((T, wl.inter), dtype=torch.float32, device="cuda")
    ysh = torch.empty((T, wl.hidden), dtype=torch.float32, device="cuda")
    qrx.qrx_shared_ffn(c, glay.shared[bits], T, ysh, ws, h_sh=hsh, **kw)
    # down stage fed the oracle's h
    yd = torch.empty((A, wl.hidden), dtype=torch.float32, device="cuda")
    qrx.qrx_expert_down(c, glay.routed[bits], perm, cu(h_o), T, yd, ws)
    # combine fed the oracle's expert outputs
    oc = torch.empty((T, wl.hidden), dtype=torch.float32, device="cuda")
    qrx.qrx_combine(c, cu(y_o), cu(ysh_o), cu(r["w"]), perm.inv, oc)
    torch.cuda.synchronize()
    assert qrx.qrx_last_error() == qrx.QRX_OK
    assert np.array_equal(np_(perm.sorted), p["sorted"])
    for name, got, ref in [("h", hs, h_o), ("y", ys, y_o), ("h_sh", hsh, hsh_o),
                           ("y_sh", ysh, ysh_o), ("down(h_oracle)", yd, y_o)]:
        assert rel_err(np_(got), ref) <= TOL, name
    assert rel_err(np_(oc), out_o) <= 1e-6
    # the whole layer
    check_layer(glay, olay, wl, x, range(T), bits)


def test_tiny_zero_input_gives_zero(tiny):
    glay, _ = tiny
    wl = W.TINY
    _, _, out = gpu_layer(glay, wl, np.zeros((8, wl.hidden), np.float32))
    assert not out.any()


def test_tiny_large_batch_many_token_groups(tiny):
    """T = 300 tokens at the tiny size: every expert serves many tokens."""
    glay, olay = tiny
    for afmt in (W.A_F32, W.A_Q8):
        wl = W.TINY.with_(T=300, afmt=afmt)
        x = activations(wl, 300, batch=3)
        check_layer(glay, olay, wl, x, [0, 77, 299])


def test_tiny_bf16_many_tokens_gemv(tiny):
    """bf16 with many tokens but inter = 128 (not a multiple of 256): the GEMV engine."""
    glay, olay = tiny
    wl = W.TINY.with_(T=300, afmt=W.A_BF16)
    assert qrx.qrx_ffn_engine(qrx.cfg_of(wl), 300) == qrx.QRX_ENGINE_GEMV
    check_layer(glay, olay, wl, activations(wl, 300, batch=4), [0, 131, 299])


def test_small_bf16_tensor_cores_all_tokens(small_tc):
    """tcgen05 grouped GEMMs: every token of ragged batches, expert tiles split in N."""
    glay, olay = small_tc
    for T in (256, 300, 517):
        wl = W.SMALL_TC.with_(T=T)
        assert qrx.qrx_ffn_engine(qrx.cfg_of(wl), T) == qrx.QRX_ENGINE_TC
        assert qrx.qrx_ffn_engine(qrx.cfg_of(wl), 255) == qrx.QRX_ENGINE_GEMV
        check_layer(glay, olay, wl, activations(wl, T, batch=4 + T), range(T))


def test_small_bf16_tensor_cores_skewed_routing(small_tc):
    """A bias that sends every token to experts 0..3: 300 tokens per expert, three
    N tiles each, 12 of 16 experts idle."""
    glay, olay = small_tc
    wl = W.SMALL_TC
    bias = np.zeros(wl.n_experts, np.float32)
    bias[:4] = 10.0
    res = check_layer(glay, olay, wl, activations(wl, 300, batch=9), [0, 100, 299], bias_np=bias)
    assert sorted(np.unique(res["idx"]).tolist()) == [0, 1, 2, 3]


def test_small_bf16_tensor_cores_stages(small_tc):
    """Stage isolation on the tensor-core engine: h and y of the routed FFN, and the
    down projection alone from the oracle's h."""
    glay, olay = small_tc
    wl = W.SMALL_TC
    T = wl.T
    x = activations(wl, T, batch=4)
    _, bias = router_weights(wl)
    r = oracle.router(wl, x, olay.Wr, bias)
    p = oracle.permute(r["idx"], wl.n_experts)
    ex = olay.experts(r["idx"].ravel(), wl.wbits)
    h_o, y_o = oracle.expert_ffn(wl, ex, p, x)
    c = qrx.cfg_of(wl)
    ws = qrx.workspace(c, T)
    perm = qrx.Perm.empty(T, wl.top_k, wl.n_experts)
    qrx.qrx_permute(c, cu(r["idx"]), perm)
    A = T * wl.top_k
    hs = torch.empty((A, wl.inter), dtype=torch.float32, device="cuda")
    ys = torch.empty((A, wl.hidden), dtype=torch.float32, device="cuda")
    qrx.qrx_expert_ffn(c, glay.routed[4], perm, T, ys, ws, x=to_device_act(wl, x), h_sorted=hs)
    ys2 = torch.full((A, wl.hidden), float("nan"), dtype=torch.float32, device="cuda")
    qrx.qrx_expert_ffn(c, glay.routed[4], perm, T, ys2, ws, x=to_device_act(wl, x))
    yd = torch.empty((A, wl.hidden), dtype=torch.float32, device="cuda")
    qrx.qrx_expert_down(c, glay.routed[4], perm, cu(h_o), T, yd, ws)
    torch.cuda.synchronize()
    assert qrx.qrx_last_error() == qrx.QRX_OK
    assert rel_err(np_(hs), h_o) <= TOL
    assert rel_err(np_(ys), y_o) <= TOL
    assert np.array_equal(np_(ys2), np_(ys))          # without h_sorted: same y
    assert rel_err(np_(yd), y_o) <= TOL


# ------------------------------------------------------------------ adaptive top-p, usage
@pytest.mark.parametrize("p", [0.3, 0.5, 0.7, 0.9])
def test_topp_prune_bitexact(tiny, p):
    """qrx_topp_prune on the oracle router's output: idx and w bit-exact."""
    glay, olay = tiny
    wl = W.TINY.with_(T=300)
    x = activations(wl, 300, batch=11)
    _, bias = router_weights(wl)
    r = oracle.router(wl, x, olay.Wr, bias)
    i_ref, w_ref, _ = oracle.topp_prune(r["idx"], r["w"], p, wl.rsf)
    idx, w = cu(r["idx"]), cu(r["w"])
    qrx.qrx_topp_prune(qrx.cfg_of(wl), idx, w, p)
    torch.cuda.synchronize()
    assert qrx.qrx_last_error() == qrx.QRX_OK
    assert np.array_equal(np_(idx), i_ref)
    assert np.array_equal(np_(w).view(np.uint32), w_ref.view(np.uint32))


@pytest.mark.parametrize("afmt", [W.A_F32, W.A_Q8])
def test_tiny_layer_topp(tiny, afmt):
    """The whole layer with top-p 0.7 fused into the router: every token."""
    glay, olay = tiny
    wl = W.TINY.with_(T=40, afmt=afmt)
    res = check_layer(glay, olay, wl, activations(wl, 40, batch=12), range(40), topp=0.7)
    dropped = int((res["idx"] < 0).sum())
    assert 0 < dropped < 40 * wl.top_k


def test_small_tc_layer_topp(small_tc):
    """Top-p on the tensor-core engine: fewer positions than T*k in every expert tile."""
    glay, olay = small_tc
    wl = W.SMALL_TC
    check_layer(glay, olay, wl, activations(wl, 300, batch=13), range(0, 300, 7), topp=0.7)


def test_usage_counters(tiny):
    """Usage counters from the fused permutation equal the routed assignments per
    expert, summed over calls; qrx_usage_accumulate adds a permutation's counts."""
    glay, olay = tiny
    wl = W.TINY.with_(T=50)
    usage = torch.zeros(wl.n_experts, dtype=torch.int64, device="cuda")
    ref = np.zeros(wl.n_experts, np.uint64)
    for b, p in enumerate([0.0, 0.7, 0.0]):
        x = activations(wl, 50, batch=20 + b)
        idx, _, _ = gpu_layer(glay, wl, x, topp=p, usage=usage)
        ref += oracle.usage(idx, wl.n_experts)
    torch.cuda.synchronize()
    assert np.array_equal(np_(usage).astype(np.uint64), ref)
    # the stage entry point
    c = qrx.cfg_of(wl)
    perm = qrx.Perm.empty(50, wl.top_k, wl.n_experts)
    qrx.qrx_permute(c, cu(idx), perm)
    u2 = torch.zeros(wl.n_experts, dtype=torch.int64, device="cuda")
    qrx.qrx_usage_accumulate(c, perm, u2)
    qrx.qrx_usage_accumulate(c, perm, u2)
    torch.cuda.synchronize()
    assert np.array_equal(np_(u2).astype(np.uint64), 2 * oracle.usage(idx, wl.n_experts))


@pytest.mark.parametrize("bits", [8, 4, 2])
def test_requant_fp8_bitexact(dev, bits):
    """FP8 (128x128 block scales) -> packed per-row codes: every byte value (NaN and
    subnormal codes included), ragged blocks (300 x 224), a padded row stride, and one
    GLM down-projection matrix (6144 x 2048); codes and scales bit-exact."""
    rng = np.random.default_rng(40 + bits)
    for rows, K, ld in ((300, 224, 224), (300, 224, 260), (6144, 2048, 2048)):
        w8 = rng.integers(0, 256, size=(rows, ld), dtype=np.uint8)
        bs = (rng.random(((rows + 127) // 128, (K + 127) // 128)) * 0.01 + 1e-4).astype(np.float32)
        q_ref, s_ref = oracle.requant_fp8(np.ascontiguousarray(w8[:, :K]), bs, bits)
        w8_d = cu(w8)[:, :K]
        q = torch.zeros((rows, K * bits // 8), dtype=torch.uint8, device="cuda")
        sc = torch.zeros(rows, dtype=torch.float32, device="cuda")
        qrx.qrx_requant_fp8(w8_d, cu(bs), bits, q, sc)
        torch.cuda.synchronize()
        assert qrx.qrx_last_error() == qrx.QRX_OK
        assert np.array_equal(np_(q), q_ref), (rows, K, ld)
        assert np.array_equal(np_(sc).view(np.uint32), s_ref.view(np.uint32)), (rows, K, ld)


def test_requant_fp8_exact_halves(dev):
    """Values whose quotient by the row scale lands on (or next to) a half-integer:
    e4m3 7.0 (0x4E) sets the row maximum, 3.5 / -3.5 / 2.5 / 0.5 (0x46 / 0xC6 / 0x42 /
    0x30) divide to exact halves at int4 (s = 1) and to near-halves at int8 and int2."""
    rows, K = 128, 256
    pattern = np.array([0x4E, 0x46, 0xC6, 0x42, 0x30, 0xB0, 0x00, 0x38], np.uint8)
    w8 = np.tile(pattern, (rows, K // pattern.size))
    w8[::3, 0] = 0x46                        # rows whose maximum is 3.5 instead
    bs = np.ones((1, 2), np.float32)
    bs[0, 1] = 0.5
    for bits in (8, 4, 2):
        q_ref, s_ref = oracle.requant_fp8(w8, bs, bits)
        q = torch.zeros((rows, K * bits // 8), dtype=torch.uint8, device="cuda")
        sc = torch.zeros(rows, dtype=torch.float32, device="cuda")
        qrx.qrx_requant_fp8(cu(w8), cu(bs), bits, q, sc)
        torch.cuda.synchronize()
        assert np.array_equal(np_(q), q_ref), bits
        assert np.array_equal(np_(sc).view(np.uint32), s_ref.view(np.uint32)), bits


@pytest.mark.parametrize("rho", [0.0, 0.6, 0.95])
def test_verify_batch_union(glm, rho):
    """Union size of correlated verify batches through the library's router and
    permutation equals the oracle's (batches without router near-ties)."""
    from quantized_routed_expert_tc_b200.layer import activations_correlated
    glay, olay = glm
    for T in (2, 4, 16):
        wl = W.GLM_DECODE_T1.with_(T=T)
        c = qrx.cfg_of(wl)
        x = activations_correlated(wl, T, rho, batch=7)
        r = oracle.router(wl, x, olay.Wr, olay.bias)
        nu_ref = oracle.permute(r["idx"], wl.n_experts)["n_union"]
        idx = torch.empty((T, wl.top_k), dtype=torch.int32, device="cuda")
        w = torch.empty((T, wl.top_k), dtype=torch.float32, device="cuda")
        ws = qrx.workspace(c, T)
        qrx.qrx_route(c, to_device_act(wl, x), glay.Wr, glay.bias, idx, w, ws)
        perm = qrx.Perm.empty(T, wl.top_k, wl.n_experts)
        qrx.qrx_permute(c, idx, perm)
        torch.cuda.synchronize()
        assert qrx.qrx_last_error() == qrx.QRX_OK
        if not r["ties"].any():
            assert int(perm.n_union.item()) == nu_ref, (T, rho)


# ------------------------------------------------------------------ GLM-shaped layer, full size
def test_glm_decode_t1(glm):
    glay, olay = glm
    wl = W.GLM_DECODE_T1
    for b in range(3):
        check_layer(glay, olay, wl, activations(wl, 1, batch=b), [0])


def test_glm_decode_t32_q8(glm):
    """Every token of the skewed 32-token Q8_0 batch."""
    glay, olay = glm
    wl = W.GLM_DECODE_T32_Q8
    res = check_layer(glay, olay, wl, activations(wl), range(32))
    n_union = len(np.unique(res["idx"]))
    assert n_union < 256                       # skewed bias: the union is below E


def test_glm_decode_t32_q8_topp(glm):
    """Top-p 0.7 at the GLM shape: sampled tokens match, and the union shrinks."""
    glay, olay = glm
    wl = W.GLM_DECODE_T32_Q8
    x = activations(wl)
    res = check_layer(glay, olay, wl, x, range(32), topp=0.7)
    idx0, _, _ = gpu_layer(glay, wl, x)
    nu_p = len(np.unique(res["idx"][res["idx"] >= 0]))
    assert nu_p < len(np.unique(idx0))


def test_glm_verify_t4_bf16(glm):
    glay, olay = glm
    wl = W.GLM_VERIFY_T4_BF16
    check_layer(glay, olay, wl, activations(wl), range(4))


def test_glm_prefill_t2048_bf16(glm):
    """128 tokens spread over the 2048-token batch (every 16th, and the last): on
    the tensor-core engine each expert's token tiles are hit, on the ~1,100 work
    items that 148 persistent CTAs take about seven at a time, so every CTA's
    later items (second accumulator buffer, later ring phases) are compared."""
    glay, olay = glm
    wl = W.GLM_PREFILL_T2048_BF16
    check_layer(glay, olay, wl, activations(wl), list(range(0, 2048, 16)) + [2047])


@pytest.mark.parametrize("wl", W.sweep(), ids=lambda w: w.name)
def test_glm_sweep(glm, wl):
    """Every token of each format-sweep batch (1 or 64 tokens)."""
    glay, olay = glm
    check_layer(glay, olay, wl, activations(wl), range(wl.T), bits=wl.wbits)


def test_glm_all_tokens_one_expert_set(glm):
    """Degenerate routing: a bias that sends all 64 tokens to experts 0..7 (union = 8)."""
    glay, olay = glm
    wl = W.GLM_DECODE_T1.with_(T=64)
    bias = np.zeros(wl.n_experts, np.float32)
    bias[:8] = 10.0
    x = activations(wl, 64, batch=5)
    res = check_layer(glay, olay, wl, x, [0, 63], bias_np=bias)
    assert sorted(np.unique(res["idx"]).tolist()) == list(range(8))


def test_glm_deterministic(glm):
    glay, _ = glm
    wl = W.GLM_DECODE_T32_Q8
    x = activations(wl)
    bias = cu(router_weights(wl)[1])
    a = gpu_layer(glay, wl, x, bias=bias)[2]
    b = gpu_layer(glay, wl, x, bias=bias)[2]
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))


def test_hostio_matches_device_call(glm):
    glay, _ = glm
    wl = W.GLM_DECODE_T1
    x = activations(wl, 1, batch=7)
    _, _, out = gpu_layer(glay, wl, x)
    c = qrx.cfg_of(wl)
    xh = torch.from_numpy(x).pin_memory()
    oh = torch.empty((1, wl.hidden), dtype=torch.float32).pin_memory()
    ws = qrx.workspace(c, 1)
    qrx.qrx_moe_forward_hostio(c, xh, glay.Wr, glay.bias, glay.routed[4], glay.shared[4], oh, ws)
    assert np.array_equal(oh.numpy(), out)


# ------------------------------------------------------------------ maximum sizes
# The largest routing the library accepts (E = 1024 experts, top-32, 32 groups of
# 32 with 8 kept) on a small expert (H = I = 256, which the tensor-core engine also
# takes), through qrx_moe_forward in every activation mode and every engine: the
# one-token fused decode path (T = 1), the multi-token mma GEMV (T = 4, 33) and the
# tensor-core engine (bf16, T = 300).
MAX_WL = W.TINY.with_(name="max_e1024_k32", n_experts=1024, n_group=32, topk_group=8,
                      top_k=32, inter=256)


@pytest.fixture(scope="session")
def max_layer(dev):
    return GpuLayer(MAX_WL, formats=(4, 8, 2)), OracleLayer(MAX_WL)


@pytest.mark.parametrize("T", [1, 4, 33])
@pytest.mark.parametrize("afmt", [W.A_F32, W.A_Q8, W.A_BF16], ids=["f32", "q8", "bf16"])
def test_max_sizes_layer(max_layer, afmt, T):
    glay, olay = max_layer
    wl = MAX_WL.with_(afmt=afmt, T=T)
    res = check_layer(glay, olay, wl, activations(wl, batch=T), range(T))
    assert res["idx"].shape == (T, 32) and (res["idx"] >= 0).all()
    assert all(len(set(row.tolist())) == 32 for row in res["idx"])


@pytest.mark.parametrize("bits", [8, 2])
@pytest.mark.parametrize("T", [1, 33])
def test_max_sizes_formats(max_layer, bits, T):
    glay, olay = max_layer
    wl = MAX_WL.with_(T=T)
    check_layer(glay, olay, wl, activations(wl, batch=T), range(T), bits=bits)


@pytest.mark.parametrize("T", [4, 33])
@pytest.mark.parametrize("afmt", [W.A_F32, W.A_BF16], ids=["f32", "bf16"])
def test_max_sizes_int2_multi_token(max_layer, afmt, T):
    """int2 weights with fixed-point activations on the multi-token mma GEMV."""
    glay, olay = max_layer
    wl = MAX_WL.with_(afmt=afmt, T=T)
    check_layer(glay, olay, wl, activations(wl, batch=T + 7), range(T), bits=2)


def test_max_sizes_tensor_core(max_layer):
    glay, olay = max_layer
    wl = MAX_WL.with_(afmt=W.A_BF16, T=300)
    assert qrx.qrx_ffn_engine(qrx.cfg_of(wl), 300) == qrx.QRX_ENGINE_TC
    check_layer(glay, olay, wl, activations(wl), list(range(0, 300, 13)) + [299])


def test_max_sizes_topp(max_layer):
    glay, olay = max_layer
    wl = MAX_WL.with_(afmt=W.A_Q8, T=33)
    check_layer(glay, olay, wl, activations(wl, batch=5), range(33), topp=0.6)


# ------------------------------------------------------------------ repeat runs
def _same_bits(a, b):
    return all(np.array_equal(np.asarray(u).view(np.uint32), np.asarray(v).view(np.uint32))
               for u, v in zip(a, b))


@pytest.mark.parametrize("wl", [W.GLM_DECODE_T1, W.GLM_DECODE_T1.with_(afmt=W.A_Q8),
                                W.GLM_VERIFY_T4_BF16, W.GLM_DECODE_T32_Q8,
                                W.GLM_PREFILL_T2048_BF16], ids=lambda w: f"{w.name}_a{w.afmt}")
def test_glm_repeat_runs_bit_identical(glm, wl):
    """Three runs of the same call give the same indices, weights and output bits
    on every engine (fused decode, mma GEMV, tensor core): no atomics decide an
    order of floating-point additions."""
    glay, _ = glm
    x = activations(wl)
    bias = cu(router_weights(wl)[1])
    first = gpu_layer(glay, wl, x, bias=bias)
    for _ in range(2):
        assert _same_bits(first, gpu_layer(glay, wl, x, bias=bias))


@pytest.mark.parametrize("T,afmt", [(1, W.A_F32), (33, W.A_Q8), (300, W.A_BF16)])
def test_max_sizes_repeat_runs_bit_identical(max_layer, T, afmt):
    glay, _ = max_layer
    wl = MAX_WL.with_(afmt=afmt, T=T)
    x = activations(wl)
    first = gpu_layer(glay, wl, x)
    assert _same_bits(first, gpu_layer(glay, wl, x))
