"""GPU parity of the hybrid-precision causal prefill (tcgen05 kernel) against
the float64 oracle, through the C ABI.

Tolerance: rel-L2 <= 2e-2 of the whole output (or of the sampled rows).  Both
sides use the same e4m3 codes (checked bit-exactly below); the kernel rounds P
to fp16 and stores V's e4m3 value times its block scale as fp16, each a
relative error near 2^-11, far inside the bound.
"""
import numpy as np
import pytest
import torch

from hybrid_precision_attention_b200 import synth
from oracle import attention as oatt, formats, select as osel
from tests._gpu import dev, hq

pytestmark = pytest.mark.gpu
PF_RELL2 = 2e-2
SM = 1 / np.sqrt(128)


def _vl_sets(lay_k, Q, W, rho_bp, G):
    """Vertical lines from the column mass of the last 64 queries (oracle selection)."""
    B, Hkv, L, D = lay_k.shape
    n = max(L - W, 0)
    nq = min(64, L)
    qpos = np.tile(np.arange(L - nq, L), G)
    out = []
    for b in range(B):
        row = []
        for h in range(Hkv):
            qs = Q[b, h * G:(h + 1) * G, L - nq:].reshape(-1, D).astype(np.float64)
            idx, _ = osel.select_vlines(lay_k[b, h].astype(np.float64), qs, qpos, n, rho_bp, SM)
            row.append(idx)
        out.append(row)
    return out


def _vl_tensor(vl, B, Hkv):
    stride = max(16, max((len(v) for r in vl for v in r), default=0))
    t = np.zeros((B, Hkv, stride), np.int32)
    n = len(vl[0][0])
    for b in range(B):
        for h in range(Hkv):
            assert len(vl[b][h]) == n
            t[b, h, :n] = vl[b][h]
    return t, n


FORMATS = {"e4m3": 0, "int8": 1}   # hq.PREFILL_E4M3, hq.PREFILL_INT8_QK


def _run(B, Hq, Hkv, L, W, rho_bp, seed, rows=None, heads=None, fmt="e4m3"):
    H = hq()
    lay = synth.planted_layer(seed, B, Hq, Hkv, L)
    Q = synth.full_queries(seed, B, Hq, Hkv, L)
    G = Hq // Hkv
    vl = _vl_sets(lay.k, Q, W, rho_bp, G)
    vlt, n_vl = _vl_tensor(vl, B, Hkv)
    out = H.hq_prefill_attn(dev(Q), dev(lay.k), dev(lay.v), dev(vlt), n_vl, W, qk_format=FORMATS[fmt])
    torch.cuda.synchronize()
    got = out.float().cpu().numpy().astype(np.float64)
    ref = oatt.prefill_ref(Q, lay.k, lay.v, vl, W, SM, rows=rows, heads=heads, qk_format=fmt)
    return got, ref


@pytest.mark.parametrize("B,Hq,Hkv,L,W,rho", [
    (1, 4, 1, 128, 128, 500),     # one tile: window only
    (1, 4, 1, 300, 64, 500),      # ragged tiles, FP8 + VL + window
    (1, 8, 2, 1000, 128, 500),    # GQA 4, several FP8 tiles
    (2, 2, 2, 520, 100, 700),     # GQA 1, batch 2, window not a tile multiple
    (1, 8, 1, 400, 0, 500),       # no window: FP8 and VL only
    (1, 4, 1, 200, 500, 500),     # window longer than the prompt: plain FP16 causal
    (1, 4, 1, 384, 32, 0),        # no vertical lines
    (1, 4, 1, 1, 128, 500),       # a one-token prompt
    (1, 4, 2, 17, 4, 10000),      # rho = 100 %: every key outside the window is a vertical line
])
@pytest.mark.parametrize("fmt", ["e4m3", "int8"])
def test_prefill_matches_oracle(B, Hq, Hkv, L, W, rho, fmt):
    got, ref = _run(B, Hq, Hkv, L, W, rho, seed=L + W, fmt=fmt)
    assert np.all(np.isfinite(got))
    for (b, h), r in ref.items():
        g = got[b, h]
        rel = np.linalg.norm(g - r) / np.linalg.norm(r)
        assert rel <= PF_RELL2, (b, h, rel)


def _e4m3_decode(codes):
    """Real values of e4m3 bytes from the OCP bit layout (bias 7, 3 mantissa bits)."""
    codes = codes.astype(np.int64)
    sign = np.where(codes & 0x80, -1.0, 1.0)
    e = (codes >> 3) & 0xF
    m = codes & 0x7
    return sign * np.where(e == 0, m / 8.0 * 2.0 ** -6, (1 + m / 8.0) * 2.0 ** (e - 7))


def test_prefill_fp8_pre_pass_matches_oracle():
    """The pre-pass outputs the workspace exposes (include/hq.h, prefill
    workspace regions): the e4m3 codes of Q and K, bit-exact against the
    oracle's per-block rounding, and V's fp16 values fp16(fp32(e4m3) * scale),
    bit-exact against the same rounding of the oracle's codes and scales."""
    H = hq()
    B, Hq, Hkv, L = 2, 4, 2, 300
    lay = synth.planted_layer(3, B, Hq, Hkv, L)
    Q = synth.full_queries(3, B, Hq, Hkv, L)
    vlt = np.zeros((B, Hkv, 16), np.int32)
    ws = torch.zeros(H.hq_prefill_workspace_bytes(B, Hq, Hkv, L, 16), dtype=torch.uint8, device="cuda")
    H.hq_prefill_attn(dev(Q), dev(lay.k), dev(lay.v), dev(vlt), 0, 64, ws=ws)
    torch.cuda.synchronize()
    r = H.prefill_ws_regions(B, Hq, Hkv, L)
    Lp = r["Lp"]
    w = ws.cpu().numpy()
    assert w[:4].view(np.uint32)[0] == 0
    q8 = w[r["q8"]:r["q8"] + B * Hq * Lp * 128].reshape(B, Hq, Lp, 128)
    k8 = w[r["k8"]:r["k8"] + B * Hkv * Lp * 128].reshape(B, Hkv, Lp, 128)
    v16 = w[r["v16"]:r["v16"] + B * Hkv * Lp * 128 * 2].view(np.float16).reshape(B, Hkv, Lp, 128)
    for name, x, got in (("Q", Q, q8), ("K", lay.k, k8)):
        for b in range(B):
            for h in range(x.shape[1]):
                want = formats.fp8_quantize(x[b, h], formats.fp8_block_scales(x[b, h]))
                assert np.array_equal(_e4m3_decode(got[b, h, :L]), want), (name, b, h)
                assert not got[b, h, L:].any(), (name, b, h)
    for b in range(B):
        for h in range(Hkv):
            sv = formats.fp8_block_scales(lay.v[b, h])
            code = formats.fp8_quantize(lay.v[b, h], sv)
            blk = np.repeat(sv.astype(np.float32), 128)[:L]
            want = (code.astype(np.float32) * blk[:, None]).astype(np.float16)
            assert np.array_equal(v16[b, h, :L].view(np.uint16), want.view(np.uint16)), (b, h)
            assert not v16[b, h, L:].view(np.uint16).any(), (b, h)


def test_prefill_int8_codes_match_oracle():
    """INT8-QK format: the pre-pass INT8 codes of Q and K are bit-exact against
    the oracle's per-block rounding (the workspace's code regions)."""
    H = hq()
    B, Hq, Hkv, L = 1, 4, 2, 300
    lay = synth.planted_layer(4, B, Hq, Hkv, L)
    Q = synth.full_queries(4, B, Hq, Hkv, L)
    vlt = np.zeros((B, Hkv, 16), np.int32)
    ws = torch.zeros(H.hq_prefill_workspace_bytes(B, Hq, Hkv, L, 16), dtype=torch.uint8, device="cuda")
    H.hq_prefill_attn(dev(Q), dev(lay.k), dev(lay.v), dev(vlt), 0, 64, ws=ws, qk_format=1)
    torch.cuda.synchronize()
    r = H.prefill_ws_regions(B, Hq, Hkv, L)
    Lp = r["Lp"]
    w = ws.cpu().numpy()
    assert w[:4].view(np.uint32)[0] == 0
    q8 = w[r["q8"]:r["q8"] + B * Hq * Lp * 128].view(np.int8).reshape(B, Hq, Lp, 128)
    k8 = w[r["k8"]:r["k8"] + B * Hkv * Lp * 128].view(np.int8).reshape(B, Hkv, Lp, 128)
    for name, x, got in (("Q", Q, q8), ("K", lay.k, k8)):
        for h in range(x.shape[1]):
            want = formats.int8_quantize(x[0, h], formats.int8_block_scales(x[0, h]))
            assert np.array_equal(got[0, h, :L].astype(np.float64), want), (name, h)
            assert not got[0, h, L:].any(), (name, h)


@pytest.mark.slow
@pytest.mark.parametrize("fmt", ["e4m3", "int8"])
def test_prefill_full_size_32k(fmt):
    """The 32K prefill layer (B=1, Hq=32, Hkv=8): sampled rows of a few heads against the oracle."""
    L = 32768
    rows = np.unique(np.concatenate([np.arange(0, 64, 7), np.linspace(64, L - 1, 40).astype(np.int64), [L - 1]]))
    got, ref = _run(1, 32, 8, L, 128, 500, seed=0, rows=rows, heads=[(0, 0), (0, 13), (0, 31)], fmt=fmt)
    for (b, h), r in ref.items():
        g = got[b, h, rows]
        rel = np.linalg.norm(g - r) / np.linalg.norm(r)
        assert rel <= PF_RELL2, (b, h, rel)
