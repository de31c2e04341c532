"""Pins for the oracle's attention (decode over the hybrid cache, hybrid prefill), CPU only.

Special cases reduce to a library routine (torch's scaled_dot_product_attention
in float64 on the CPU), brute-force loops check the vectorised code on tiny
inputs, and the planted generator checks the orderings the pages report.
"""
import numpy as np
import torch

from oracle import attention, formats, hybrid, select
from hybrid_precision_attention_b200 import synth

SM = 1 / np.sqrt(128)


def _sdpa(q, k, v, causal=False):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(np.asarray(a, np.float64)))
    return torch.nn.functional.scaled_dot_product_attention(t(q)[None], t(k)[None], t(v)[None], is_causal=causal, scale=SM)[0].numpy()


def test_attend_matches_loops():
    rng = np.random.default_rng(0)
    for N in (1, 3, 16):
        q = rng.standard_normal((2, 6)); k = rng.standard_normal((N, 6)); v = rng.standard_normal((N, 6))
        assert np.allclose(attention.attend(q, k, v, 0.4), attention.attend_loops(q, k, v, 0.4), rtol=1e-12, atol=1e-14)


def test_identical_keys_give_mean_of_values():
    rng = np.random.default_rng(1)
    k = np.repeat(rng.standard_normal((1, 128)), 50, axis=0)
    v = rng.standard_normal((50, 128))
    o = attention.attend(rng.standard_normal((4, 128)), k, v, SM)
    assert np.allclose(o, v.mean(axis=0)[None], rtol=1e-12, atol=1e-13)


def _run_decode(W, rho_bp, L=300, steps=3, seed=3, B=1, Hq=4, Hkv=1):
    lay = synth.planted_layer(seed, B, Hq, Hkv, L)
    qd, kd, vd = synth.decode_tokens(seed, B, Hq, Hkv, steps)
    c = hybrid.HybridCacheRef(B, Hq, Hkv, W, rho_bp, cap=L + steps)
    c.init_from_prefix(lay.k, lay.v, lay.q_tail)
    outs = [c.decode(qd[t], kd[t], vd[t]) for t in range(steps)]
    return lay, (qd, kd, vd), outs, c


def test_decode_all_fp16_equals_sdpa():
    # window covering the whole prefix, and rho = 100 % with no window: both keep every key FP16
    for W, rho in ((400, 10000), (0, 10000)):
        lay, (qd, kd, vd), outs, _ = _run_decode(W, rho)
        for t, o in enumerate(outs):
            K = np.concatenate([lay.k[0, 0], kd[:t + 1, 0, 0]]).astype(np.float64)
            V = np.concatenate([lay.v[0, 0], vd[:t + 1, 0, 0]]).astype(np.float64)
            assert np.allclose(o[0], _sdpa(qd[t, 0], K, V), rtol=1e-11, atol=1e-13), (W, rho, t)


def test_decode_strict_low_bit_equals_dequantise_then_attend():
    # rho = 0, W = 0: every prefix position is K4V4 (the strict d_k4v4 mode); new tokens are staged in FP16
    lay, (qd, kd, vd), outs, _ = _run_decode(0, 0)
    c, s, z = formats.pack_k4v4(lay.k[0, 0]); Kd = formats.dequant_k4v4(c, s, z)
    c, s, z = formats.pack_k4v4(lay.v[0, 0]); Vd = formats.dequant_k4v4(c, s, z)
    for t, o in enumerate(outs):
        K = np.concatenate([Kd, kd[:t + 1, 0, 0].astype(np.float64)])
        V = np.concatenate([Vd, vd[:t + 1, 0, 0].astype(np.float64)])
        assert np.allclose(o[0], _sdpa(qd[t, 0], K, V), rtol=1e-11, atol=1e-13)


def _mse(a, b):
    return float(np.mean((np.asarray(a) - np.asarray(b)) ** 2))


def test_hybrid_error_below_uniform_int4_and_monotone():
    """Hybrid decode error vs full FP16 is below strict 4-bit, and falls as W or rho grows."""
    L = 2048
    full = _run_decode(L + 10, 0, L=L, steps=2, Hq=8, Hkv=2)[2]
    err = {}
    for W, rho in ((0, 0), (128, 0), (512, 0), (128, 500), (128, 2000), (0, 500)):
        err[(W, rho)] = _mse(_run_decode(W, rho, L=L, steps=2, Hq=8, Hkv=2)[2], full)
    assert err[(128, 500)] < err[(0, 0)]            # hybrid beats uniform INT4
    assert err[(512, 0)] < err[(128, 0)] < err[(0, 0)]
    assert err[(128, 2000)] < err[(128, 500)] < err[(128, 0)]
    assert err[(0, 500)] < err[(0, 0)]


# ------------------------------------------------------------------ prefill

def _prefill_loops(q16, k16, v16, is_vl, W, sm):
    """Explicit per-(i, j) classification, for tiny L."""
    L, D = q16.shape
    sq = formats.fp8_block_scales(q16); qt = formats.fp8_dequant(formats.fp8_quantize(q16, sq), sq)
    sk = formats.fp8_block_scales(k16); kt = formats.fp8_dequant(formats.fp8_quantize(k16, sk), sk)
    sv = formats.fp8_block_scales(v16); vt = formats.fp8_dequant(formats.fp8_quantize(v16, sv), sv)
    out = np.zeros((L, D))
    for i in range(L):
        logits, vals = [], []
        for j in range(i + 1):
            if j > i - W or is_vl[j]:
                logits.append(float(q16[i].astype(np.float64) @ k16[j].astype(np.float64)) * sm)
                vals.append(v16[j].astype(np.float64))
            else:
                logits.append(float(qt[i] @ kt[j]) * sm)
                vals.append(vt[j])
        mx = max(logits)
        w = np.exp(np.array(logits) - mx)
        out[i] = (w[:, None] * np.array(vals)).sum(0) / w.sum()
    return out


def test_prefill_matches_loops():
    rng = np.random.default_rng(4)
    L = 16
    q, k, v = [(rng.standard_normal((L, 128)) * 2).astype(np.float16) for _ in range(3)]
    is_vl = np.zeros(L, bool); is_vl[[0, 5, 9]] = True
    for W in (0, 3, 20):
        got = attention.prefill_head(q, k, v, is_vl, W, SM)
        assert np.allclose(got, _prefill_loops(q, k, v, is_vl, W, SM), rtol=1e-11, atol=1e-13)


def test_prefill_special_cases():
    rng = np.random.default_rng(5)
    L = 300
    q, k, v = [rng.standard_normal((L, 128)).astype(np.float16) for _ in range(3)]
    none = np.zeros(L, bool)
    # window >= L: exact FP16 causal attention
    assert np.allclose(attention.prefill_head(q, k, v, none, L, SM), _sdpa(q, k, v, causal=True), rtol=1e-11, atol=1e-13)
    # every key a vertical line: also exact FP16 attention
    assert np.allclose(attention.prefill_head(q, k, v, ~none, 0, SM), _sdpa(q, k, v, causal=True), rtol=1e-11, atol=1e-13)
    # no window, no lines: plain causal attention over the FP8-represented tensors
    f = lambda x: formats.fp8_dequant(formats.fp8_quantize(x, formats.fp8_block_scales(x)), formats.fp8_block_scales(x))
    assert np.allclose(attention.prefill_head(q, k, v, none, 0, SM), _sdpa(f(q), f(k), f(v), causal=True), rtol=1e-11, atol=1e-13)
    # a vertical line inside the window is counted once: same result with or without the flag
    vl = none.copy(); vl[[250, 260, 299]] = True
    a = attention.prefill_head(q, k, v, vl, 64, SM)
    vl2 = vl.copy(); vl2[[260, 299]] = False
    rows = np.arange(290, 300)   # for these rows 260 and 299 are window keys
    assert np.allclose(a[rows], attention.prefill_head(q, k, v, vl2, 64, SM)[rows], rtol=1e-13, atol=1e-15)


def test_prefill_hybrid_error_below_uniform_fp8():
    L = 1024
    lay = synth.planted_layer(11, 1, 4, 1, L)
    Q = synth.full_queries(11, 1, 4, 1, L)
    ref = _sdpa(Q[0, 0], lay.k[0, 0], lay.v[0, 0], causal=True)
    n = L - 128
    qs = Q[0, :, L - 64:].reshape(-1, 128).astype(np.float64)
    vl, _ = select.select_vlines(lay.k[0, 0].astype(np.float64), qs, np.tile(np.arange(L - 64, L), 4), n, 500, SM)
    is_vl = np.zeros(L, bool); is_vl[vl] = True
    hyb = attention.prefill_head(Q[0, 0], lay.k[0, 0], lay.v[0, 0], is_vl, 128, SM)
    uni = attention.prefill_head(Q[0, 0], lay.k[0, 0], lay.v[0, 0], np.zeros(L, bool), 0, SM)
    wide = attention.prefill_head(Q[0, 0], lay.k[0, 0], lay.v[0, 0], is_vl, 256, SM)
    assert _mse(hyb, ref) < _mse(uni, ref)
    assert _mse(wide, ref) < _mse(hyb, ref)


def test_prefill_ref_maps_query_heads_to_their_kv_head():
    """The multi-head driver: query head hq of batch b reads kv head hq // G of
    the same batch (GQA groups of consecutive query heads) with that kv head's
    own vertical lines.  Checked head by head against the per-(i, j) loops on
    inputs where every kv head and batch differs."""
    rng = np.random.default_rng(6)
    B, Hq, Hkv, L, W = 2, 4, 2, 20, 3
    G = Hq // Hkv
    Q = (rng.standard_normal((B, Hq, L, 128)) * 2).astype(np.float16)
    K = (rng.standard_normal((B, Hkv, L, 128)) * 2).astype(np.float16)
    V = rng.standard_normal((B, Hkv, L, 128)).astype(np.float16)
    vl = [[np.array([0, 4, 11]), np.array([2, 7])], [np.array([1, 5, 6, 13]), np.array([3])]]
    got = attention.prefill_ref(Q, K, V, vl, W, SM)
    assert sorted(got) == [(b, h) for b in range(B) for h in range(Hq)]
    for b in range(B):
        for hq in range(Hq):
            kv = hq // G
            is_vl = np.zeros(L, bool)
            is_vl[vl[b][kv]] = True
            want = _prefill_loops(Q[b, hq], K[b, kv], V[b, kv], is_vl, W, SM)
            assert np.allclose(got[(b, hq)], want, rtol=1e-11, atol=1e-13), (b, hq)
    # a subset of heads and rows gives the same rows
    sub = attention.prefill_ref(Q, K, V, vl, W, SM, rows=np.arange(8, 20), heads=[(1, 3), (0, 1)])
    assert np.array_equal(sub[(1, 3)], got[(1, 3)][8:]) and np.array_equal(sub[(0, 1)], got[(0, 1)][8:])


def test_code_widths_strict_mode_and_error_order():
    """The other code widths (README Mode reference: K8V8, K4V2, K2V4): with no
    window and no lines the cache reduces to dequantise-then-attend at those
    widths (torch SDPA in float64 on the dequantised rows), and the error
    against FP16 falls as bits are added."""
    L, steps = 400, 2
    lay = synth.planted_layer(9, 1, 4, 1, L)
    qd, kd, vd = synth.decode_tokens(9, 1, 4, 1, steps)
    full = None
    errs = {}
    for kb, vb in ((8, 8), (4, 4), (4, 2), (2, 4), (16, 16)):
        if kb == 16:
            c = hybrid.HybridCacheRef(1, 4, 1, L + 10, 0, cap=L + steps)
        else:
            c = hybrid.HybridCacheRef(1, 4, 1, 0, 0, cap=L + steps, k_bits=kb, v_bits=vb)
        c.init_from_prefix(lay.k, lay.v, lay.q_tail)
        outs = [c.decode(qd[t], kd[t], vd[t]) for t in range(steps)]
        if kb == 16:
            full = outs
            continue
        ck, sk, zk = formats.pack_bits(lay.k[0, 0], kb)
        cv, sv, zv = formats.pack_bits(lay.v[0, 0], vb)
        Kd, Vd = formats.dequant_bits(ck, sk, zk, kb), formats.dequant_bits(cv, sv, zv, vb)
        for t, o in enumerate(outs):
            K = np.concatenate([Kd, kd[:t + 1, 0, 0].astype(np.float64)])
            V = np.concatenate([Vd, vd[:t + 1, 0, 0].astype(np.float64)])
            assert np.allclose(o[0], _sdpa(qd[t, 0], K, V), rtol=1e-11, atol=1e-13), (kb, vb, t)
        errs[(kb, vb)] = outs
    e = {key: _mse(v, full) for key, v in errs.items()}
    assert e[(8, 8)] < e[(4, 4)] < e[(4, 2)] and e[(4, 4)] < e[(2, 4)]


def test_prefill_int8_qk_format():
    """INT8-QK / FP16-PV (README: INT8 Q.K with FP16 P.V): per-(i, j) loops on a
    tiny case; without window or lines it is causal SDPA over the INT8 values
    of Q and K with V in FP16; with W >= L it is exact FP16 attention."""
    rng = np.random.default_rng(12)
    L = 16
    q, k, v = [(rng.standard_normal((L, 128)) * 2).astype(np.float16) for _ in range(3)]
    is_vl = np.zeros(L, bool); is_vl[[1, 7]] = True
    qt = attention.low_precision(q, "int8"); kt = attention.low_precision(k, "int8")
    for W in (0, 4):
        got = attention.prefill_head(q, k, v, is_vl, W, SM, qk_format="int8")
        want = np.zeros((L, 128))
        for i in range(L):
            lg, vals = [], []
            for j in range(i + 1):
                fp = j > i - W or is_vl[j]
                lg.append(float((q[i].astype(np.float64) @ k[j].astype(np.float64)) if fp else (qt[i] @ kt[j])) * SM)
                vals.append(v[j].astype(np.float64))
            w = np.exp(np.array(lg) - max(lg))
            want[i] = (w[:, None] * np.array(vals)).sum(0) / w.sum()
        assert np.allclose(got, want, rtol=1e-11, atol=1e-13), W
    L = 300
    q, k, v = [rng.standard_normal((L, 128)).astype(np.float16) for _ in range(3)]
    none = np.zeros(L, bool)
    got = attention.prefill_head(q, k, v, none, 0, SM, qk_format="int8")
    f = lambda x: attention.low_precision(x, "int8")
    assert np.allclose(got, _sdpa(f(q), f(k), v, causal=True), rtol=1e-11, atol=1e-13)
    assert np.allclose(attention.prefill_head(q, k, v, none, L, SM, qk_format="int8"), _sdpa(q, k, v, causal=True),
                       rtol=1e-11, atol=1e-13)
    # INT8 keeps more of Q.K than e4m3: lower error against exact attention on the planted generator
    lay = synth.planted_layer(13, 1, 4, 1, 1024)
    Q = synth.full_queries(13, 1, 4, 1, 1024)
    ref = _sdpa(Q[0, 0], lay.k[0, 0], lay.v[0, 0], causal=True)
    none = np.zeros(1024, bool)
    e8 = _mse(attention.prefill_head(Q[0, 0], lay.k[0, 0], lay.v[0, 0], none, 0, SM, qk_format="e4m3"), ref)
    ei = _mse(attention.prefill_head(Q[0, 0], lay.k[0, 0], lay.v[0, 0], none, 0, SM, qk_format="int8"), ref)
    assert ei < e8
