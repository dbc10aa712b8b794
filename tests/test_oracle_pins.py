"""Pins of the CPU oracle to things other than itself (no GPU needed).

Each test ties one oracle function to a hand-derived fixture (tests/golden),
brute force on tiny inputs, a closed form, an invariant, or an independent
numpy / torch recomputation in float64, chosen so that a dropped term, a wrong
sign or index, or a transposed operand fails at least one of them.
"""
import itertools

import numpy as np
import pytest

import oracle
from quantized_routed_expert_tc_b200 import synth, workloads as W
from tests.conftest import read_golden

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


def ints(s):
    return [int(v) for v in s.split(",")]


def floats(s):
    return [float(v) for v in s.split(",")]


def np_codes(q: np.ndarray, K: int, bits: int) -> np.ndarray:
    """Independent numpy decode of packed rows (two's-complement fields)."""
    q = q.astype(np.int32)
    per = 8 // bits
    fields = [(q >> (bits * i)) & ((1 << bits) - 1) for i in range(per)]
    codes = np.stack(fields, axis=-1).reshape(q.shape[0], -1)[:, :K]
    return np.where(codes >= (1 << (bits - 1)), codes - (1 << bits), codes).astype(np.int64)


# --------------------------------------------------------------------------- packing
def test_pack_fixture():
    for fmt, codes, hexbytes in read_golden("pack_codes.txt"):
        bits, codes = int(fmt), ints(codes)
        want = bytes(int(h, 16) for h in hexbytes.split())
        # pack through the quantiser: a row whose values are the codes and whose
        # absmax equals qmax quantises to exactly those codes with scale 1
        qmax = oracle._load().qo_qmax(bits)
        row = np.array(codes + [qmax], dtype=np.float32)
        pad = (-row.size) % (8 // bits)
        row = np.concatenate([row, np.zeros(pad, np.float32)])
        if np.abs(row).max() > qmax:   # codes at qmin: scale differs, test unpack only
            continue
        q, s = oracle.quantize_rows(row[None, :], bits)
        assert s[0] == 1.0
        assert bytes(q[0, :len(want)]) == want, (bits, codes)


def test_unpack_fixture_and_exhaustive():
    for fmt, codes, hexbytes in read_golden("pack_codes.txt"):
        bits, codes = int(fmt), ints(codes)
        b = np.array([[int(h, 16) for h in hexbytes.split()]], dtype=np.uint8)
        got = oracle.unpack_rows(b, len(codes), bits)[0].tolist()
        assert got == codes
    allb = np.arange(256, dtype=np.uint8)[:, None]
    for bits in (8, 4, 2):
        K = 8 // bits
        got = oracle.unpack_rows(allb, K, bits).astype(np.int64)
        assert np.array_equal(got, np_codes(allb, K, bits))
        lo, hi = -(1 << (bits - 1)), (1 << (bits - 1)) - 1
        assert got.min() == lo and got.max() == hi
        # every byte decodes to a distinct code tuple: the map is a bijection
        assert len({tuple(r) for r in got.tolist()}) == 256


def test_int4_is_bit_consistent_with_int8_container():
    """README '已实现的功能': packing verified bit-consistent with the int8 container.
    The same codes held as int4 and as int8 give identical integer block dots and
    identical FFN outputs with the same scales."""
    rng = np.random.default_rng(7)
    K, rows = 128, 16
    codes = rng.integers(-8, 8, size=(rows, K)).astype(np.int64)
    q4 = np.zeros((rows, K // 2), np.uint8)
    q4[:] = ((codes[:, 0::2] & 0xF) | ((codes[:, 1::2] & 0xF) << 4)).astype(np.uint8)
    q8 = (codes & 0xFF).astype(np.uint8)
    xq = rng.integers(-127, 128, size=K).astype(np.int8)
    a4 = oracle.block_dots_q8(q4, K, 4, xq)
    a8 = oracle.block_dots_q8(q8, K, 8, xq)
    assert np.array_equal(a4, a8)
    ref = (codes.reshape(rows, K // 32, 32) * xq.astype(np.int64).reshape(K // 32, 32)).sum(-1)
    assert np.array_equal(a4, ref)
    # FFN through both containers
    wl = W.TINY.with_(hidden=K, inter=64, n_experts=1, n_group=1, topk_group=1, top_k=1, T=2)
    g = rng.integers(-8, 8, size=(64, K)); u = rng.integers(-8, 8, size=(64, K))
    d = rng.integers(-8, 8, size=(K, 64))

    def pack(c, bits):
        c = np.asarray(c)
        if bits == 8:
            return (c & 0xFF).astype(np.uint8)
        return ((c[:, 0::2] & 0xF) | ((c[:, 1::2] & 0xF) << 4)).astype(np.uint8)
    sc = lambda n: (rng.random(n).astype(np.float32) * 0.01 + 0.001)
    gs, us, ds = sc(64), sc(64), sc(K)
    x = rng.standard_normal((2, K)).astype(np.float32)
    outs = []
    for bits in (4, 8):
        ex = oracle.Expert(pack(g, bits), gs, pack(u, bits), us, pack(d, bits), ds)
        for af in (W.A_F32, W.A_Q8):
            h, y = oracle.shared_ffn(wl.with_(wbits=bits, afmt=af), ex, x)
            outs.append((bits, af, h, y))
    for af in (W.A_F32, W.A_Q8):
        r4 = [o for o in outs if o[0] == 4 and o[1] == af][0]
        r8 = [o for o in outs if o[0] == 8 and o[1] == af][0]
        assert np.array_equal(r4[2], r8[2]) and np.array_equal(r4[3], r8[3])


# --------------------------------------------------------------------------- quantiser
def test_quantize_fixture():
    for fmt, wv, scale, codes in read_golden("quantize_rows.txt"):
        bits = int(fmt)
        w = np.array([floats(wv)], np.float32)
        q, s = oracle.quantize_rows(w, bits)
        assert s[0] == np.float32(float(scale))
        assert oracle.unpack_rows(q, w.shape[1], bits)[0].tolist() == ints(codes)


@pytest.mark.parametrize("bits", [8, 4, 2])
def test_quantize_is_nearest_code(bits):
    """Brute force: each code is the nearest of all codes in [qmin, qmax] to w/s
    (halves away from zero), the scale maps absmax to qmax, qmin never emitted."""
    w = synth.normal_f32(11, bits, 64 * 96, 0.0, 0.02).reshape(64, 96)
    w[3] = 0.0
    q, s = oracle.quantize_rows(w, bits)
    codes = oracle.unpack_rows(q, 96, bits).astype(np.int64)
    qmax = (1 << (bits - 1)) - 1
    qmin = -(1 << (bits - 1))
    absmax = np.abs(w).max(axis=1)
    assert s[3] == 0 and not codes[3].any()
    nz = absmax > 0
    assert np.allclose(s[nz].astype(np.float64) * qmax, absmax[nz], rtol=1e-6)
    cand = np.arange(qmin, qmax + 1)
    for r in np.nonzero(nz)[0]:
        v = (w[r] / s[r]).astype(np.float64)            # the f32 quotient, widened
        dist = np.abs(v[:, None] - cand[None, :])
        best = dist.min(axis=1)
        ok = np.isclose(dist, best[:, None], rtol=0, atol=1e-12)
        # among equally near codes, the one farther from zero
        pick = np.array([cand[o][np.argmax(np.abs(cand[o]))] for o in ok])
        assert np.array_equal(codes[r], pick)
        assert codes[r].min() >= -qmax          # qmin is never emitted
        # reconstruction error at most half a step
        assert np.all(np.abs(w[r] - s[r] * codes[r]) <= s[r] * 0.5 * (1 + 1e-6))


# --------------------------------------------------------------------------- Q8_0
def test_q8_fixture():
    for xs, d, qs in read_golden("q8_block.txt"):
        x = np.array(floats(xs), np.float32)
        q, dd = oracle.quantize_q8(x)
        assert dd[0] == np.float32(float(d))
        assert q.tolist() == ints(qs)


def test_q8_properties():
    x = synth.normal_f32(12, 1, 32 * 64, 0.0, 1.0).reshape(64, 32)
    x[5] = 0.0
    x[6, 3] = 1e-30
    x[7] = 0.0
    x[7, :3] = [1e-38, -5e-39, 2e-39]   # amax below 127/FLT_MAX: 127/amax overflows
    q, d = oracle.quantize_q8(x)
    q = q.astype(np.int64)
    for b in range(64):
        amax = np.abs(x[b]).max()
        if amax == 0:
            assert d[b, 0] == 0 and not q[b].any()
            continue
        if d[b, 0] < np.finfo(np.float32).tiny:
            # subnormal scale: 127/amax overflowed; the clamp on the product still
            # gives +-127 with the sign of x, and 0 for zeros
            assert np.array_equal(q[b], np.sign(x[b]).astype(np.int64) * 127)
            continue
        assert np.isclose(float(d[b, 0]) * 127, amax, rtol=1e-6)
        assert np.abs(q[b]).max() == 127 and np.abs(q[b]).max() <= 127
        assert np.all(np.abs(x[b] - d[b, 0] * q[b]) <= d[b, 0] * 0.5 * (1 + 1e-5))


def test_block_dots_exact():
    rng = np.random.default_rng(3)
    for bits in (8, 4, 2):
        K = 256
        w = synth.normal_f32(13, bits, 8 * K, 0.0, 0.02).reshape(8, K)
        q, _ = oracle.quantize_rows(w, bits)
        xq = rng.integers(-127, 128, size=K).astype(np.int8)
        acc = oracle.block_dots_q8(q, K, bits, xq)
        codes = np_codes(q, K, bits)
        ref = (codes.reshape(8, K // 32, 32) * xq.astype(np.int64).reshape(K // 32, 32)).sum(-1)
        assert np.array_equal(acc, ref)


def test_bf16_rounding_matches_torch():
    torch = pytest.importorskip("torch")
    v = np.concatenate([synth.normal_f32(14, 1, 4000), np.array(
        [1.0, 1.00390625, 1.0 + 2**-8 + 2**-20, 1.0 + 2**-9, 1.0 + 3 * 2**-9, -2.5, 0.0, 65504.0,
         3.0e38, 1e-40], np.float32)])
    ours = oracle.f32_to_bf16(v)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


# --------------------------------------------------------------------------- router
def _router_case(E, G, Gk, k, rsf, s, bias):
    wl = W.TINY.with_(hidden=1, n_experts=E, n_group=G, topk_group=Gk, top_k=k, rsf=rsf, T=1)
    s = np.array(s, np.float64)
    Wr = np.log(s / (1 - s)).astype(np.float32)[:, None]
    x = np.ones((1, 1), np.float32)
    return wl, oracle.router(wl, x, Wr, np.array(bias, np.float32))


def test_router_fixture():
    for case, shape, sv, bias, idx, wv in read_golden("router_tiny.txt"):
        E, G, Gk, k = ints(shape.rsplit(",", 1)[0])
        rsf = float(shape.rsplit(",", 1)[1])
        wl, r = _router_case(E, G, Gk, k, rsf, floats(sv), floats(bias))
        assert r["idx"][0].tolist() == ints(idx), case
        assert np.allclose(r["w"][0], floats(wv), rtol=0, atol=2e-6), case
        assert r["ties"][0] == 0


def _brute_router(sc, s, G, Gk, k, rsf):
    """Enumerate every kept-group set and every k-subset of its experts."""
    E = sc.size
    gs = E // G
    gscore = [np.sort(sc[g * gs:(g + 1) * gs])[::-1][:2].sum() for g in range(G)]
    best_groups = max(itertools.combinations(range(G), Gk),
                      key=lambda c: (sum(gscore[g] for g in c), [-g for g in c]))
    cand = [e for e in range(E) if e // gs in best_groups]
    best = max(itertools.combinations(cand, k), key=lambda c: (sum(sc[e] for e in c), [-e for e in c]))
    chosen = sorted(best, key=lambda e: (-sc[e], e))
    w = np.array([s[e] for e in chosen]) / sum(s[e] for e in chosen) * rsf
    return chosen, w


@pytest.mark.parametrize("E,G,Gk,k", [(16, 4, 2, 4), (12, 3, 2, 3), (8, 1, 1, 3), (8, 8, 4, 4),
                                      (16, 2, 1, 5)])
def test_router_brute_force(E, G, Gk, k):
    H, T = 24, 24
    wl = W.TINY.with_(hidden=H, n_experts=E, n_group=G, topk_group=Gk, top_k=k, T=T)
    x = synth.normal_f32(21, E, T * H).reshape(T, H)
    Wr = synth.normal_f32(22, E, E * H, 0, 0.3).reshape(E, H)
    bias = synth.normal_f32(23, E, E, 0, 0.1)
    r = oracle.router(wl, x, Wr, bias)
    # logits: independent f64 matmul, rounded to f32
    lg = (x.astype(np.float64) @ Wr.astype(np.float64).T).astype(np.float32)
    assert np.array_equal(lg, r["logits"])
    s = r["scores"].astype(np.float64)
    assert np.allclose(s, 1 / (1 + np.exp(-lg.astype(np.float64))), rtol=1e-7, atol=0)
    for t in range(T):
        sc = (r["scores"][t] + bias).astype(np.float32).astype(np.float64)
        chosen, w = _brute_router(sc, s[t], G, Gk, k, wl.rsf)
        if r["ties"][t]:
            continue
        assert r["idx"][t].tolist() == chosen
        assert np.allclose(r["w"][t], w, rtol=1e-6)
        assert abs(float(r["w"][t].astype(np.float64).sum()) - wl.rsf) <= 1e-6 * wl.rsf


def test_router_special_cases():
    E, H, T, k = 16, 32, 16, 4
    x = synth.normal_f32(31, 0, T * H).reshape(T, H)
    Wr = synth.normal_f32(32, 0, E * H, 0, 0.3).reshape(E, H)
    # one group: plain top-k of sc;  zero bias: top-k of logits (sigmoid is monotone)
    wl = W.TINY.with_(hidden=H, n_experts=E, n_group=1, topk_group=1, top_k=k, T=T)
    r = oracle.router(wl, x, Wr, np.zeros(E, np.float32))
    lg = (x.astype(np.float64) @ Wr.astype(np.float64).T)
    for t in range(T):
        ref = sorted(range(E), key=lambda e: (-lg[t, e], e))[:k]
        assert r["idx"][t].tolist() == ref
    # G = Gk: group limiting keeps every group, same as one group
    wl2 = wl.with_(n_group=4, topk_group=4)
    r2 = oracle.router(wl2, x, Wr, np.zeros(E, np.float32))
    assert np.array_equal(r["idx"], r2["idx"]) and np.array_equal(r["w"], r2["w"])
    # the bias moves selection but never the weights' formula: weights are s/sum(s)*rsf
    bias = synth.normal_f32(33, 0, E, 0, 0.5)
    r3 = oracle.router(wl, x, Wr, bias)
    for t in range(T):
        s_sel = r3["scores"][t, r3["idx"][t]].astype(np.float64)
        assert np.allclose(r3["w"][t], s_sel / s_sel.sum() * wl.rsf, rtol=1e-6)
    # routed scaling factor scales the weights linearly
    r4 = oracle.router(wl.with_(rsf=5.0), x, Wr, bias)
    assert np.array_equal(r3["idx"], r4["idx"])
    assert np.allclose(r4["w"], 2 * r3["w"], rtol=1e-6)


def test_router_tie_flags():
    # two candidates whose sc differ by 5e-6 straddle the k-th place
    wl, r = _router_case(4, 1, 1, 1, 1.0, [0.6, 0.6, 0.1, 0.2], [0, 5e-6, 0, 0])
    assert r["ties"][0] & 1
    wl, r = _router_case(4, 1, 1, 1, 1.0, [0.6, 0.5, 0.1, 0.2], [0, 0, 0, 0])
    assert r["ties"][0] == 0
    # two groups whose scores differ by less than 1e-5
    wl, r = _router_case(4, 2, 1, 1, 1.0, [0.6, 0.4, 0.5, 0.5], [0, 0, 0, 2e-6])
    assert r["ties"][0] & 2


def test_router_bf16_input():
    E, H, T = 16, 64, 4
    xb = synth.normal_bf16(41, 0, T * H).reshape(T, H)
    Wr = synth.normal_f32(42, 0, E * H, 0, 0.3).reshape(E, H)
    wl = W.TINY.with_(hidden=H, afmt=W.A_BF16, T=T)
    r = oracle.router(wl, xb, Wr, np.zeros(E, np.float32))
    xf = synth.bf16_bits_to_f32(xb)
    r2 = oracle.router(wl.with_(afmt=W.A_F32), xf, Wr, np.zeros(E, np.float32))
    assert np.array_equal(r["logits"], r2["logits"]) and np.array_equal(r["idx"], r2["idx"])


# --------------------------------------------------------------------------- permutation
def test_permute_fixture():
    rows = {r[0]: r[1] for r in read_golden("permute_tiny.txt")}
    E, k = int(rows["E"]), int(rows["k"])
    idx = np.array(ints(rows["idx"]), np.int32).reshape(-1, k)
    p = oracle.permute(idx, E)
    for key in ("counts", "offsets", "sorted", "inv"):
        assert p[key].tolist() == ints(rows[key]), key
    assert p["union_ids"].tolist() == ints(rows["union"])


def test_permute_against_numpy():
    rng = np.random.default_rng(5)
    for T, k, E in [(1, 8, 256), (37, 4, 16), (512, 8, 256), (64, 2, 3)]:
        idx = rng.integers(0, E, size=(T, k)).astype(np.int32)
        p = oracle.permute(idx, E)
        flat = idx.ravel()
        assert np.array_equal(p["counts"], np.bincount(flat, minlength=E))
        assert p["counts"].sum() == T * k
        assert np.array_equal(p["sorted"], np.argsort(flat, kind="stable"))
        assert np.array_equal(p["inv"][p["sorted"]], np.arange(T * k))
        assert np.array_equal(p["union_ids"], np.unique(flat))
        assert np.array_equal(p["offsets"], np.concatenate([[0], np.cumsum(p["counts"])]))


# --------------------------------------------------------------------------- FFN
def _tiny_layer(bits=4, afmt=W.A_F32, T=6, H=64, I=32, E=8, k=2):
    wl = W.TINY.with_(hidden=H, inter=I, n_experts=E, n_group=2, topk_group=1, top_k=k, T=T,
                      wbits=bits, afmt=afmt)
    ex = {}
    for e in range(E + 1):
        g = synth.normal_f32(51, W.stream(W.K_GATE, e), I * H, 0, 0.02).reshape(I, H)
        u = synth.normal_f32(51, W.stream(W.K_UP, e), I * H, 0, 0.02).reshape(I, H)
        d = synth.normal_f32(51, W.stream(W.K_DOWN, e), H * I, 0, 0.02).reshape(H, I)
        ex[e] = oracle.quantize_expert(g, u, d, bits)
    shared = ex.pop(E)
    if afmt == W.A_BF16:
        x = synth.normal_bf16(52, 0, T * H).reshape(T, H)
    else:
        x = synth.normal_f32(52, 0, T * H).reshape(T, H)
    Wr = synth.normal_f32(53, 0, E * H, 0, 0.1).reshape(E, H)
    bias = synth.normal_f32(54, 0, E, 0, 0.1)
    return wl, ex, shared, x, Wr, bias


def _deq(q, s, K, bits):
    return np_codes(q, K, bits).astype(np.float64) * s.astype(np.float64)[:, None]


def _np_bf16(v):
    torch = pytest.importorskip("torch")
    import torch as T_
    b = T_.from_numpy(np.ascontiguousarray(v, np.float32)).to(T_.bfloat16).to(T_.float32)
    return b.numpy().astype(np.float64)


def _dense_ffn(wl, ex, xrow):
    """Independent f64 dense dequantised reference of one token through one expert,
    with the f32 roundings the definition states (g, u, h stored as f32)."""
    H, I, bits = wl.hidden, wl.inter, wl.wbits
    Wg, Wu, Wd = _deq(ex.gate_q, ex.gate_s, H, bits), _deq(ex.up_q, ex.up_s, H, bits), \
        _deq(ex.down_q, ex.down_s, I, bits)
    if wl.afmt == W.A_Q8:
        xq, xd = oracle.quantize_q8(xrow.astype(np.float32))
        xv = (xq.astype(np.float64).reshape(-1, 32) * xd.astype(np.float64)[:, None]).ravel()
    elif wl.afmt == W.A_BF16:
        xv = synth.bf16_bits_to_f32(xrow).astype(np.float64)
    else:
        xv = xrow.astype(np.float64)
    g = (Wg @ xv).astype(np.float32).astype(np.float64)
    u = (Wu @ xv).astype(np.float32).astype(np.float64)
    h = (g / (1 + np.exp(-g)) * u).astype(np.float32)
    if wl.afmt == W.A_Q8:
        hq, hd = oracle.quantize_q8(h)
        hv = (hq.astype(np.float64).reshape(-1, 32) * hd.astype(np.float64)[:, None]).ravel()
    elif wl.afmt == W.A_BF16:
        hv = _np_bf16(h)
    else:
        hv = h.astype(np.float64)
    y = (Wd @ hv).astype(np.float32)
    return h, y


@pytest.mark.parametrize("bits,afmt", [(4, W.A_F32), (8, W.A_F32), (2, W.A_F32), (4, W.A_Q8),
                                       (2, W.A_Q8), (8, W.A_Q8), (4, W.A_BF16)])
def test_ffn_against_dense_f64(bits, afmt):
    wl, ex, shared, x, Wr, bias = _tiny_layer(bits, afmt)
    for t in range(wl.T):
        for e in (0, 3):
            h, y = oracle.ffn_token(wl, ex[e], x, t)
            hr, yr = _dense_ffn(wl, ex[e], x[t])
            assert np.allclose(h, hr, rtol=2.5e-7, atol=1e-30)
            assert np.allclose(y, yr, rtol=2.5e-7, atol=1e-9 * np.abs(yr).max())


def test_ffn_zero_cases():
    wl, ex, shared, x, Wr, bias = _tiny_layer()
    h, y = oracle.ffn_token(wl, ex[0], np.zeros_like(x), 0)
    assert not h.any() and not y.any()
    z = oracle.Expert(np.zeros_like(ex[0].gate_q), ex[0].gate_s, ex[0].up_q, ex[0].up_s,
                      ex[0].down_q, ex[0].down_s)
    h, y = oracle.ffn_token(wl, z, x, 0)
    assert not h.any() and not y.any()


@pytest.mark.parametrize("afmt", [W.A_F32, W.A_Q8, W.A_BF16])
def test_union_equals_per_token(afmt):
    wl, ex, shared, x, Wr, bias = _tiny_layer(afmt=afmt, T=9)
    r = oracle.router(wl, x, Wr, bias)
    p = oracle.permute(r["idx"], wl.n_experts)
    h_u, y_u = oracle.expert_ffn(wl, ex, p, x)
    y_t = oracle.expert_ffn_per_token(wl, ex, r["idx"], p, x)
    assert np.array_equal(y_u, y_t)
    y_d = oracle.expert_down(wl, ex, p, h_u)
    assert np.array_equal(y_d, y_u)


def test_combine_and_layer():
    wl, ex, shared, x, Wr, bias = _tiny_layer(T=7)
    idx, wt, out = oracle.moe_forward(wl, x, Wr, bias, ex, shared)
    r = oracle.router(wl, x, Wr, bias)
    assert np.array_equal(idx, r["idx"]) and np.array_equal(wt, r["w"])
    p = oracle.permute(idx, wl.n_experts)
    _, ys = oracle.expert_ffn(wl, ex, p, x)
    _, ysh = oracle.shared_ffn(wl, shared, x)
    # combine against numpy f64
    ref = ysh.astype(np.float64).copy()
    for t in range(wl.T):
        for j in range(wl.top_k):
            ref[t] += float(wt[t, j]) * ys[p["inv"][t * wl.top_k + j]].astype(np.float64)
    assert np.allclose(out, ref.astype(np.float32), rtol=2.5e-7, atol=1e-12)
    # layer through per-token dense references
    for t in range(wl.T):
        acc = _dense_ffn(wl, shared, x[t])[1].astype(np.float64)
        for j in range(wl.top_k):
            acc += float(wt[t, j]) * _dense_ffn(wl, ex[idx[t, j]], x[t])[1].astype(np.float64)
        assert np.allclose(out[t], acc, rtol=1e-6, atol=1e-7 * np.abs(acc).max())
    # doubling rsf doubles the routed part exactly up to rounding
    _, wt2, out2 = oracle.moe_forward(wl.with_(rsf=2 * wl.rsf), x, Wr, bias, ex, shared)
    assert np.allclose(out2 - ysh, 2 * (out - ysh), rtol=1e-5, atol=1e-6 * np.abs(out).max())
    # x = 0: every expert output is 0, so the layer output is 0
    _, _, out0 = oracle.moe_forward(wl, np.zeros_like(x), Wr, bias, ex, shared)
    assert not out0.any()


def test_combine_stage_properties():
    """The combine stage alone (README "JustVugg/colibri", "已实现的功能": routed
    experts plus the shared expert), by properties that fix it:
    - one-hot weights (1 on one slot) with no shared term return that slot's row;
    - a dropped slot (inv -1) counts as nothing, whatever its weight: it equals
      the same call with that slot kept at weight 0;
    - every slot dropped leaves the shared term;
    - relabelling the sorted positions (rows moved, inv remapped) changes nothing."""
    rng = np.random.default_rng(5)
    wl = W.TINY
    T, k, H = 5, wl.top_k, wl.hidden
    A = T * k
    ys = rng.standard_normal((A, H)).astype(np.float32)
    ysh = rng.standard_normal((T, H)).astype(np.float32)
    wt = rng.uniform(0.1, 1.0, (T, k)).astype(np.float32)
    inv = rng.permutation(A).astype(np.int32)
    out = oracle.combine(wl, ys, ysh, wt, inv)
    for t in range(T):
        for j in range(k):
            oh = np.zeros((T, k), np.float32)
            oh[t, j] = 1.0
            sel = oracle.combine(wl, ys, None, oh, inv)
            assert np.array_equal(sel[t], ys[inv[t * k + j]])
            assert not np.delete(sel, t, axis=0).any()
    drop = inv.copy()
    dropped = [1, 6, 7, 12]
    drop[dropped] = -1
    w0 = wt.copy().ravel()
    w0[dropped] = 0.0
    assert np.array_equal(oracle.combine(wl, ys, ysh, wt, drop),
                          oracle.combine(wl, ys, ysh, w0.reshape(T, k), inv))
    assert np.array_equal(oracle.combine(wl, ys, ysh, wt, np.full(A, -1, np.int32)), ysh)
    relabel = rng.permutation(A)                    # row p moves to relabel[p]
    ys2 = np.empty_like(ys)
    ys2[relabel] = ys
    assert np.array_equal(oracle.combine(wl, ys2, ysh, wt, relabel[inv].astype(np.int32)), out)


# --------------------------------------------------------------------------- adaptive top-p
def test_topp_fixture():
    """Hand-derived cases: README "JustVugg/colibri", "快速开始" (--topp)."""
    for case, rsf, p, T, k, idx_in, w_in, idx_out, w_out in read_golden("topp_prune.txt"):
        T, k = int(T), int(k)
        idx = np.array(ints(idx_in), np.int32).reshape(T, k)
        wt = np.array(floats(w_in), np.float32).reshape(T, k)
        i2, w2, kept = oracle.topp_prune(idx, wt, float(p), float(rsf))
        assert i2.ravel().tolist() == ints(idx_out), case
        assert w2.ravel().tolist() == floats(w_out), case
        assert kept == sum(v >= 0 for v in ints(idx_out)), case


@pytest.mark.parametrize("p", [0.3, 0.7, 0.9])
def test_topp_minimal_prefix_brute_force(p):
    """On real router outputs: the kept set reaches p * rsf, and no smaller set of
    slots does (every subset of one fewer slots is checked), and among sets of its
    size it holds the largest weights."""
    wl, ex, shared, x, Wr, bias = _tiny_layer(T=40)
    r = oracle.router(wl, x, Wr, bias)
    i2, w2, kept = oracle.topp_prune(r["idx"], r["w"], p, wl.rsf)
    thr = float(np.float32(p)) * float(np.float32(wl.rsf))
    total = 0
    for t in range(wl.T):
        keep = [j for j in range(wl.top_k) if i2[t, j] >= 0]
        drop = [j for j in range(wl.top_k) if i2[t, j] < 0]
        total += len(keep)
        assert keep, "at least one slot kept"
        assert all(i2[t, j] == r["idx"][t, j] and w2[t, j] == r["w"][t, j] for j in keep)
        assert all(w2[t, j] == 0.0 for j in drop)
        wts = [float(r["w"][t, j]) for j in range(wl.top_k)]
        if drop:
            assert sum(wts[j] for j in keep) >= thr * (1 - 1e-12)
        for sub in itertools.combinations(range(wl.top_k), len(keep) - 1):
            assert sum(wts[j] for j in sub) < thr * (1 + 1e-12)
        assert min(wts[j] for j in keep) >= max([wts[j] for j in drop], default=0.0)
    assert total == kept


def test_topp_bounds_and_layer():
    """p outside (0,1) changes nothing; top-p feeds a permutation without the dropped
    slots, and the layer's routed part sums only the kept experts."""
    wl, ex, shared, x, Wr, bias = _tiny_layer(T=9)
    r = oracle.router(wl, x, Wr, bias)
    for p in (0.0, 1.0, 1.5, -0.1):
        i2, w2, kept = oracle.topp_prune(r["idx"], r["w"], p, wl.rsf)
        assert np.array_equal(i2, r["idx"]) and np.array_equal(w2, r["w"]) and kept == wl.T * wl.top_k
    i2, w2, kept = oracle.topp_prune(r["idx"], r["w"], 0.5, wl.rsf)
    assert kept < wl.T * wl.top_k
    perm = oracle.permute(i2, wl.n_experts)
    assert int(perm["counts"].sum()) == kept == int(perm["offsets"][-1])
    flat = i2.ravel()
    assert all(perm["inv"][a] == -1 for a in range(flat.size) if flat[a] < 0)
    # the kept slots keep their stable (expert, slot) order
    order = sorted((int(flat[a]), a) for a in range(flat.size) if flat[a] >= 0)
    assert perm["sorted"][:kept].tolist() == [a for _, a in order]
    assert np.array_equal(oracle.usage(i2, wl.n_experts),
                          perm["counts"].astype(np.uint64))
    # the layer with top-p = the kept experts' weighted outputs plus the shared expert
    idx_l, wt_l, out = oracle.moe_forward(wl, x, Wr, bias, ex, shared, topp=0.5)
    assert np.array_equal(idx_l, i2) and np.array_equal(wt_l, w2)
    for t in range(wl.T):
        acc = _dense_ffn(wl, shared, x[t])[1].astype(np.float64)
        for j in range(wl.top_k):
            if idx_l[t, j] >= 0:
                acc += float(wt_l[t, j]) * _dense_ffn(wl, ex[idx_l[t, j]], x[t])[1].astype(np.float64)
        assert np.allclose(out[t], acc, rtol=1e-6, atol=1e-7 * np.abs(acc).max())
    # top-p off through the options entry: bit-identical to the plain layer
    _, _, out_off = oracle.moe_forward(wl, x, Wr, bias, ex, shared, topp=0.0)
    _, _, out_plain = oracle.moe_forward(wl, x, Wr, bias, ex, shared)
    assert np.array_equal(out_off, out_plain)


# --------------------------------------------------------------------------- FP8 requantisation
def test_fp8_decode_matches_torch():
    """Every e4m3 code decodes to torch's float8_e4m3fn value (NaN codes to NaN)."""
    import torch
    f = oracle.fp8_e4m3_to_f32(np.arange(256))
    t = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    nan = np.isnan(t)
    assert np.array_equal(np.isnan(f), nan) and nan.sum() == 2
    assert np.array_equal(f[~nan].view(np.uint32), t[~nan].view(np.uint32))


def _fixture_fp8():
    w8 = np.zeros((2, 256), np.uint8)
    w8[0, :128], w8[0, 128:] = 0x38, 0x40
    w8[1, 0], w8[1, 5], w8[1, 200] = 0xC8, 0x7F, 0x30
    return w8, np.array([[0.5, 0.25]], np.float32)


def test_requant_fixture():
    w8, bs = _fixture_fp8()
    for bits, row, amax, c0, c5, c200, rest in read_golden("requant_fp8.txt"):
        bits, row = int(bits), int(row)
        q, s = oracle.requant_fp8(w8, bs, bits)
        codes = np_codes(q, 256, bits)[row]
        qmax = {8: 127, 4: 7, 2: 1}[bits]
        assert s[row] == np.float32(float(amax)) / np.float32(qmax)
        assert (codes[0], codes[5], codes[200]) == (int(c0), int(c5), int(c200))
        others = np.delete(codes, [0, 5, 200])
        assert (others == int(rest)).all()


@pytest.mark.parametrize("bits", [8, 4, 2])
def test_requant_against_torch_dequant(bits):
    """Random codes (every byte value, NaN and subnormals included) and block scales on
    a ragged 300 x 224 matrix: the result equals quantising the dequantised matrix,
    the dequantisation done here with torch's float8 decode and one f32 multiply."""
    import torch
    rng = np.random.default_rng(5)
    rows, K = 300, 224
    w8 = rng.integers(0, 256, size=(rows, K), dtype=np.uint8)
    bs = (rng.random((3, 2)) * 0.01 + 1e-4).astype(np.float32)
    q, s = oracle.requant_fp8(w8, bs, bits)
    f = torch.from_numpy(w8).view(torch.float8_e4m3fn).float().numpy()
    f = np.where(np.isnan(f), np.float32(0), f)
    scale = np.repeat(np.repeat(bs, 128, axis=0), 128, axis=1)[:rows, :K]
    deq = (f * scale).astype(np.float32)
    q2, s2 = oracle.quantize_rows(deq, bits)
    assert np.array_equal(q, q2) and np.array_equal(s.view(np.uint32), s2.view(np.uint32))


def test_requant_power_of_two_scales():
    """Scaling every block scale by 2^m scales each row scale by 2^m exactly and leaves
    the codes unchanged (multiplication by a power of two is exact)."""
    rng = np.random.default_rng(6)
    w8 = rng.integers(0, 126, size=(130, 256), dtype=np.uint8)   # finite codes only
    bs = (rng.random((2, 2)) + 0.5).astype(np.float32)
    for bits in (8, 4, 2):
        q, s = oracle.requant_fp8(w8, bs, bits)
        for m in (-3, 5):
            q2, s2 = oracle.requant_fp8(w8, bs * np.float32(2.0 ** m), bits)
            assert np.array_equal(q, q2)
            assert np.array_equal(s2, s * np.float32(2.0 ** m))


# --------------------------------------------------------------------------- verify-batch union
def test_union_of_correlated_batches():
    """Union size of a verify batch (README "JustVugg/colibri", "已实现的功能": MTP
    verification routes extra experts): identical tokens (rho = 1) route to exactly k
    experts; independent tokens (rho = 0) are the plain draws; the union never exceeds
    min(E, T*k) and grows with T."""
    from quantized_routed_expert_tc_b200.layer import activations_correlated, router_weights
    wl = W.TINY
    Wr, bias = router_weights(wl)
    x1 = activations_correlated(wl, 6, 1.0, batch=3)
    assert (x1 == x1[0]).all()
    r = oracle.router(wl, x1, Wr, bias)
    assert oracle.permute(r["idx"], wl.n_experts)["n_union"] == wl.top_k
    x0 = activations_correlated(wl, 6, 0.0, batch=3)
    from quantized_routed_expert_tc_b200 import synth as S
    assert np.array_equal(x0, S.normal_f32(wl.seed, W.stream(W.K_X, 3), 6 * wl.hidden).reshape(6, -1))
    last = 0
    for T in (1, 2, 4, 8):
        x = activations_correlated(wl, T, 0.5, batch=4)
        nu = oracle.permute(oracle.router(wl, x, Wr, bias)["idx"], wl.n_experts)["n_union"]
        assert wl.top_k <= nu <= min(wl.n_experts, T * wl.top_k) and nu >= last
        last = nu


# --------------------------------------------------------------------------- layer closed form
def test_layer_closed_form():
    """The whole layer against a closed form.  Structured inputs make every stage
    collapse to a few scalar operations:
    - token t is one-hot at input column t (values 1, 2, -0.5), so each logit is one
      chosen router entry times that value (exact);
    - the logits are chosen so that each token's kept groups and top-4 experts follow
      by hand (well separated: no near-ties);
    - every gate/up/down row has one nonzero entry, 7 * (e + 1) / 2^m times a sign,
      which int4 per-row quantisation represents exactly (scale (e + 1) / 2^m, code 7).
    Expected values are formed here in double from those constants."""
    import math
    wl = W.TINY.with_(T=3, bias_std=0.0)                       # H 256, E 16, I 128, G 4, Gk 2, k 4
    H, E, I, k, rsf = wl.hidden, wl.n_experts, wl.inter, wl.top_k, wl.rsf
    xv = [1.0, 2.0, -0.5]
    x = np.zeros((3, H), np.float32)
    for t in range(3):
        x[t, t] = xv[t]
    # wanted logits per token (unlisted experts: -4, far below)
    want = [{0: 3.0, 1: 2.5, 2: 2.0, 3: 1.5, 4: 1.0, 5: 0.5, 6: 0.0, 7: -0.5},
            {15: 3.0, 14: 2.0, 11: 2.5, 8: 1.0},
            {5: 4.0, 0: 1.0, 6: 0.5, 2: 0.25}]
    Wr = np.zeros((E, H), np.float32)
    for t in range(3):
        for e in range(E):
            Wr[e, t] = want[t].get(e, -4.0) / xv[t]
    bias = np.zeros(E, np.float32)
    sel = [[0, 1, 2, 3], [15, 11, 14, 8], [5, 0, 6, 2]]          # by hand from the logits above

    def val(e, r, m):              # the one nonzero of row r of a matrix of expert e
        return (1 if (r + e) % 2 == 0 else -1) * 7.0 * (e + 1) / 2.0 ** m

    ex = {}
    for e in range(E + 1):         # e == E: the shared expert
        g = np.zeros((I, H), np.float32)
        u = np.zeros((I, H), np.float32)
        d = np.zeros((H, I), np.float32)
        for i in range(I):
            g[i, i % 3] = val(e, i, 6)
            u[i, i % 3] = val(e, i + 1, 7)
        for r in range(H):
            d[r, r % I] = val(e, r, 8)
        ex[e] = oracle.quantize_expert(g, u, d, 4)
    shared = ex.pop(E)
    idx, wt, out = oracle.moe_forward(wl, x, Wr, bias, ex, shared)

    sig = lambda z: 1.0 / (1.0 + math.exp(-z))
    for t in range(3):
        assert idx[t].tolist() == sel[t]
        s = [sig(want[t][e]) for e in sel[t]]
        for j in range(k):
            assert abs(wt[t, j] - s[j] / sum(s) * rsf) <= 1e-6 * rsf

    def expert_out(e, t):          # y[r] of expert e for token t, in double
        h = np.zeros(I)
        for i in range(I):
            if i % 3 == t:
                gi, ui = val(e, i, 6) * xv[t], val(e, i + 1, 7) * xv[t]
                h[i] = gi * sig(gi) * ui
        return np.array([val(e, r, 8) * h[r % I] for r in range(H)])

    for t in range(3):
        ref = expert_out(E, t)
        for j, e in enumerate(sel[t]):
            s = [sig(want[t][q]) for q in sel[t]]
            ref = ref + (s[j] / sum(s) * rsf) * expert_out(e, t)
        scale = np.abs(ref).max()
        assert scale > 0
        assert np.abs(out[t].astype(np.float64) - ref).max() <= 1e-6 * scale, t


def _bf16_rne(v: float) -> tuple[float, float]:
    """v rounded to bf16 (8 significant bits, ties to even), and the distance of
    v's scaled mantissa from the nearest rounding tie."""
    import math
    if v == 0.0:
        return 0.0, 0.5
    m, ex = math.frexp(v)                      # |m| in [0.5, 1)
    z = m * 256.0
    return math.ldexp(round(z), ex - 8), abs(abs(z - math.trunc(z)) - 0.5)


@pytest.mark.parametrize("afmt", [W.A_F32, W.A_Q8, W.A_BF16])
def test_layer_closed_form_h_rounding(afmt):
    """The whole layer in each activation mode against a closed form that includes
    the rounding of h before the down projection (Q8_0 re-quantisation per
    32-block, or bf16 nearest-even).
    - Tokens are one-hot (values 1, 2, -0.5), routed as in test_layer_closed_form.
    - Each gate/up row has one nonzero, in a column that belongs to one token, so
      token t's h has three nonzeros of different sizes in every 32-block of I
      (rows 32b + t, +3, +6); every int4 row is exact (scale c, code 7).
    - Q8_0: x's block is one-hot, so its code is +-127 and d = f32(|x|/127);
      h's blocks hold three values, so two of them move by the quantisation.
    The closed form checks its own guards: no value near a rounding tie, and the
    rounding of h must change the result by far more than the tolerance."""
    import math
    wl = W.TINY.with_(T=3, bias_std=0.0, afmt=afmt)
    H, E, I, k, rsf = wl.hidden, wl.n_experts, wl.inter, wl.top_k, wl.rsf
    xv = [1.0, 2.0, -0.5]
    x = np.zeros((3, H), np.float32)
    for t in range(3):
        x[t, t] = xv[t]
    want = [{0: 3.0, 1: 2.5, 2: 2.0, 3: 1.5, 4: 1.0, 5: 0.5, 6: 0.0, 7: -0.5},
            {15: 3.0, 14: 2.0, 11: 2.5, 8: 1.0},
            {5: 4.0, 0: 1.0, 6: 0.5, 2: 0.25}]
    Wr = np.zeros((E, H), np.float32)
    for t in range(3):
        for e in range(E):
            Wr[e, t] = want[t].get(e, -4.0) / xv[t]
    bias = np.zeros(E, np.float32)
    sel = [[0, 1, 2, 3], [15, 11, 14, 8], [5, 0, 6, 2]]

    def val(e, r, m):              # the one nonzero of row r: +-7 * (e + 1) * mag / 2^m
        mag = 1 + (r + r // 32 + r // 128) % 4
        return (1 if (r + e) % 2 == 0 else -1) * 7.0 * (e + 1) * mag / 2.0 ** m

    def col(i):                    # input column of gate/up row i; columns >= 3 are zero in x
        j = i % 32
        return j % 3 if j < 9 else 3 + i % 5

    ex = {}
    for e in range(E + 1):
        g = np.zeros((I, H), np.float32)
        u = np.zeros((I, H), np.float32)
        d = np.zeros((H, I), np.float32)
        for i in range(I):
            g[i, col(i)] = val(e, i, 6)
            u[i, col(i)] = val(e, i + 1, 7)
        for r in range(H):
            d[r, r % I] = val(e, r, 8)
        ex[e] = oracle.quantize_expert(g, u, d, 4)
    shared = ex.pop(E)
    act = x
    if afmt == W.A_BF16:           # 1, 2 and -0.5 are exact in bf16: the top half of the f32
        act = (x.view(np.uint32) >> 16).astype(np.uint16)
    idx, wt, out = oracle.moe_forward(wl, act, Wr, bias, ex, shared)

    sig = lambda z: 1.0 / (1.0 + math.exp(-z))
    if afmt == W.A_Q8:             # one-hot block: code +-127, d = f32(|v| / 127)
        xe = [math.copysign(127.0 * float(np.float32(abs(v)) / np.float32(127.0)), v) for v in xv]
    else:
        xe = xv
    guard = []                     # distances from a rounding tie

    def h_of(e, t):
        h = np.zeros(I)
        for i in range(I):
            if col(i) == t:
                gi, ui = val(e, i, 6) * xe[t], val(e, i + 1, 7) * xe[t]
                h[i] = gi * sig(gi) * ui
        return h

    def h_rounded(h):
        if afmt == W.A_F32:
            return h
        hr = np.zeros(I)
        if afmt == W.A_BF16:
            for i in range(I):
                hr[i], dist = _bf16_rne(h[i])
                if h[i] != 0.0:
                    guard.append(dist)
            return hr
        for b in range(I // 32):   # Q8_0 per 32-block of I
            blk = h[b * 32:(b + 1) * 32]
            amax = np.abs(blk).max()
            dq = float(np.float32(amax) / np.float32(127.0))
            for j, v in enumerate(blk):
                z = v * 127.0 / amax
                guard.append(abs(abs(z - math.trunc(z)) - 0.5))
                hr[b * 32 + j] = math.copysign(math.floor(abs(z) + 0.5), z) * dq
        return hr

    def layer(t, rounded):
        s = [sig(want[t][q]) for q in sel[t]]
        def y(e):
            h = h_of(e, t)
            h = h_rounded(h) if rounded else h
            return np.array([val(e, r, 8) * h[r % I] for r in range(H)])
        ref = y(E)
        for j, e in enumerate(sel[t]):
            ref = ref + (s[j] / sum(s) * rsf) * y(e)
        return ref, s

    for t in range(3):
        assert idx[t].tolist() == sel[t]
        ref, s = layer(t, True)
        for j in range(k):
            assert abs(wt[t, j] - s[j] / sum(s) * rsf) <= 1e-6 * rsf
        scale = np.abs(ref).max()
        assert scale > 0
        assert np.abs(out[t].astype(np.float64) - ref).max() <= 1e-6 * scale, t
        if afmt != W.A_F32:        # the rounding of h is visible at this tolerance
            plain, _ = layer(t, False)
            assert np.abs(plain - ref).max() > 100 * 1e-6 * scale, t
    if afmt != W.A_F32:            # the oracle's f32 h is within a few ulps (~2.4e-7 relative)
        # of the double h here, which moves a scaled mantissa (< 256) or a Q8_0 ratio
        # (<= 127) by < 7e-5: a tie distance of 2e-4 leaves every rounding decided alike
        assert min(guard) > 2e-4, min(guard)


def test_layer_at_maximum_sizes():
    """The largest configuration the library accepts: E = 1024 experts, top-32,
    32 groups of 32 with 8 kept.  Each token gets 32 distinct experts, all inside
    the 8 groups with the largest group scores (sum of the top-2 sc); the weights
    sum to rsf; the permutation places every assignment once; and the layer equals
    the dense per-token reference."""
    E, k, G, Gk, H, I, T = 1024, 32, 32, 8, 64, 64, 3
    wl = W.TINY.with_(hidden=H, inter=I, n_experts=E, n_group=G, topk_group=Gk, top_k=k, T=T)
    ex = {}
    for e in range(E + 1):
        g = synth.normal_f32(61, W.stream(W.K_GATE, e), I * H, 0, 0.02).reshape(I, H)
        u = synth.normal_f32(61, W.stream(W.K_UP, e), I * H, 0, 0.02).reshape(I, H)
        d = synth.normal_f32(61, W.stream(W.K_DOWN, e), H * I, 0, 0.02).reshape(H, I)
        ex[e] = oracle.quantize_expert(g, u, d, 4)
    shared = ex.pop(E)
    x = synth.normal_f32(62, 0, T * H).reshape(T, H)
    Wr = synth.normal_f32(63, 0, E * H, 0, 0.1).reshape(E, H)
    bias = synth.normal_f32(64, 0, E, 0, 0.1)
    r = oracle.router(wl, x, Wr, bias)
    gs = E // G
    for t in range(T):
        sel = r["idx"][t]
        assert len(set(sel.tolist())) == k and sel.min() >= 0 and sel.max() < E
        s = (1.0 / (1.0 + np.exp(-r["logits"][t].astype(np.float64)))).astype(np.float32)
        sc = (s + bias).astype(np.float32)
        top2 = np.sort(sc.reshape(G, gs), axis=1)[:, -2:]
        gscore = (top2[:, 0] + top2[:, 1]).astype(np.float32)
        best = set(np.argsort(-gscore.astype(np.float64), kind="stable")[:Gk].tolist())
        assert set((sel // gs).tolist()) <= best
        cand = np.array([e for e in range(E) if e // gs in best])
        order = cand[np.lexsort((cand, -sc[cand].astype(np.float64)))]   # sc descending, then index
        assert sel.tolist() == order[:k].tolist()
        assert abs(float(r["w"][t].astype(np.float64).sum()) - wl.rsf) <= 1e-5 * wl.rsf
    p = oracle.permute(r["idx"], E)
    A = T * k
    assert int(p["counts"].sum()) == A and sorted(p["sorted"].tolist()) == list(range(A))
    assert all(p["sorted"][p["inv"][a]] == a for a in range(A))
    idx, wt, out = oracle.moe_forward(wl, x, Wr, bias, ex, shared)
    assert np.array_equal(idx, r["idx"])
    for t in range(T):
        acc = _dense_ffn(wl, shared, x[t])[1].astype(np.float64)
        for j in range(k):
            acc += float(wt[t, j]) * _dense_ffn(wl, ex[idx[t, j]], x[t])[1].astype(np.float64)
        assert np.allclose(out[t], acc, rtol=1e-6, atol=1e-7 * np.abs(acc).max())
