"""Full-size multi-layer decode through the C ABI, checked on sampled units.

Two workloads of the method's evaluation shapes, every layer resident at once:
  * Qwen3-8B-shaped KV: 36 layers, B=16, Hq=32, Hkv=8, prefix 32768;
  * Qwen3-32B-shaped capacity case: 64 layers, B=32, Hq=64, Hkv=8, prefix 32768
    (about 100 GB of hybrid cache on one GPU).
Each layer is drawn on the device with the planted-vertical-line recipe, its
vertical lines are selected from its own last 64 queries and the prefix is
packed; then one decode step runs over every layer.  Sampled (layer, b, kv head)
units are checked against the oracle: the unit's column-mass scores against the
oracle's float64 column mass of the same keys and queries (and the selected set
against its stable top-k, outside the tie band); then, on a cache the oracle
rebuilds from the dense prefix and the GPU's vertical-line set, the K4V4
records bit-exactly, the VL rows bit-exactly, and the decode output within the
decode tolerances.
"""
import numpy as np
import pytest
import torch

from hybrid_precision_attention_b200 import synth
from oracle import formats, hybrid, select as osel
from tests._gpu import check_decode, check_selection, hq, sz_words

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _run_layers(n_layers, B, Hq, Hkv, L, W, samples, seed0):
    H = hq()
    G = Hq // Hkv
    cap = L + 128
    caches, kept = [], {}
    for layer in range(n_layers):
        k, v, q_tail, _ = synth.planted_layer_device(seed0 + layer, B, Hq, Hkv, L, "cuda")
        c = H.HybridCache(B, Hq, Hkv, cap, W, 500)
        mine = [(ly, b, h) for (ly, b, h) in samples if ly == layer]
        scores = torch.zeros((B, Hkv, c.cap), dtype=torch.float32, device="cuda") if mine else None
        H.hq_select_vlines(c, k, q_tail, scores_out=scores)
        H.hq_pack_merge(c, k, v)
        for (ly, b, h) in mine:
            kept[(ly, b, h)] = (k[b, h].cpu().numpy(), v[b, h].cpu().numpy(),
                                q_tail[b, h * G:(h + 1) * G].cpu().numpy(), scores[b, h].cpu().numpy())
        del scores
        del k, v, q_tail
        caches.append(c)
    torch.cuda.synchronize()
    for c in caches:
        st = c.state()
        assert st["err"] == 0 and st["T"] == L and st["n_packed"] == L - W, st
    # one decode step over every layer
    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed0 + 99)
    steps = []
    for layer, c in enumerate(caches):
        q = torch.randn((B, Hq, 128), generator=gen, device="cuda").to(torch.float16)
        kn = torch.randn((B, Hkv, 128), generator=gen, device="cuda").to(torch.float16)
        vn = torch.randn((B, Hkv, 128), generator=gen, device="cuda").to(torch.float16)
        out = H.hq_decode_attn(c, q, kn, vn)
        steps.append((q, kn, vn, out))
    torch.cuda.synchronize()
    for c in caches:
        assert c.state()["err"] == 0 and c.state()["T"] == L + 1
    return caches, kept, steps


def _check_unit(c, kept, step, ly, b, h, L, W, G):
    k16, v16, qg, gsc = kept[(ly, b, h)]
    n_vl = c.state()["n_vl"]
    vl = c.vl_pos[b, h, :n_vl].cpu().numpy().astype(np.int64)
    assert np.all(np.diff(vl) > 0) and vl.max() < L - W
    # the unit's column mass (the last 64 prefix queries of its G heads, keys in FP16) and its selection
    n = L - W
    nq = qg.shape[1]
    ref = osel.column_mass(k16.astype(np.float64), qg.reshape(-1, 128).astype(np.float64),
                           np.tile(np.arange(L - nq, L), G), n, 1 / np.sqrt(128))
    assert n_vl == osel.k_of(n, 500)
    check_selection(gsc, vl, ref, n_vl, f"layer {ly} unit ({b},{h}) selection")
    # K4V4 records of the packed prefix, bit-exact (this unit's pages only)
    H = hq()
    pg = c.pages[b, h].cpu().numpy()
    npg = pg.shape[0]
    take = lambda off, width: pg[:, off:off + 64 * width].reshape(npg * 64, width)
    n_packed = L - W
    for which, x16, off_c, off_s in (("k", k16, H.PAGE_KCODES, H.PAGE_KSZ), ("v", v16, H.PAGE_VCODES, H.PAGE_VSZ)):
        codes, scale, zero = formats.pack_k4v4(x16[:n_packed])
        assert np.array_equal(take(off_c, 64)[:n_packed], codes), f"layer {ly} ({b},{h}) {which} codes"
        words = take(off_s, 16).copy().view(np.uint32)[:n_packed]
        assert np.array_equal(words, sz_words(scale, zero)), f"layer {ly} ({b},{h}) {which} scale/zero"
    bits = np.unpackbits(pg[:, H.PAGE_VLMASK:H.PAGE_VLMASK + 8].copy(), axis=-1, bitorder="little").reshape(-1).astype(bool)
    assert np.array_equal(np.nonzero(bits[:n_packed])[0], vl)
    # VL rows: the dense prefix rows of those positions
    assert np.array_equal(c.kf[b, h, :n_vl].cpu().numpy(), k16[vl])
    assert np.array_equal(c.vf[b, h, :n_vl].cpu().numpy(), v16[vl])
    # decode output of the unit's G query heads against the oracle cache
    q, kn, vn, out = step
    ref = hybrid.HybridCacheRef(1, G, 1, W, 500, c.cap)
    ref.install_prefix(k16[None, None], v16[None, None], [[vl]])
    want = ref.decode(q[b, h * G:(h + 1) * G].cpu().numpy()[None], kn[b, h].cpu().numpy()[None, None],
                      vn[b, h].cpu().numpy()[None, None])
    check_decode(out[b, h * G:(h + 1) * G], want[0], f"layer {ly} unit ({b},{h})")


def test_qwen3_8b_shape_36_layers_b16():
    B, Hq, Hkv, L, W, layers = 16, 32, 8, 32768, 128, 36
    samples = [(0, 0, 0), (17, 9, 3), (35, 15, 7)]
    caches, kept, steps = _run_layers(layers, B, Hq, Hkv, L, W, samples, seed0=800)
    for (ly, b, h) in samples:
        _check_unit(caches[ly], kept, steps[ly], ly, b, h, L, W, Hq // Hkv)


def test_qwen3_32b_shape_64_layers_b32_capacity():
    B, Hq, Hkv, L, W, layers = 32, 64, 8, 32768, 128, 64
    free, _ = torch.cuda.mem_get_info()
    # cache bytes of the 64 layers plus one layer's dense prefix while it is installed
    probe = hq().HybridCache(1, Hq, Hkv, L + 128, W, 500)
    per_unit = probe.nbytes()
    del probe
    # (+ each layer's selection / merge workspaces, about 0.3 GB at this size)
    need = layers * (B * per_unit + 300 * 2**20) + 3 * B * Hkv * L * 128 * 2 * 2
    if need > free:
        pytest.skip(f"needs {need / 1e9:.0f} GB of device memory, {free / 1e9:.0f} GB free")
    samples = [(0, 0, 0), (40, 31, 5)]
    caches, kept, steps = _run_layers(layers, B, Hq, Hkv, L, W, samples, seed0=900)
    for (ly, b, h) in samples:
        _check_unit(caches[ly], kept, steps[ly], ly, b, h, L, W, Hq // Hkv)
