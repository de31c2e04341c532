"""GPU parity: K4V4 pack, VL selection, staging merge and decode attention
against the CPU oracle, through the C ABI (libhq.so)."""
import numpy as np
import pytest
import torch

from hybrid_precision_attention_b200 import synth
from oracle import hybrid
from tests._gpu import Pair, check_decode, dev, hq

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,Hq,Hkv,L,W,rho", [
    (1, 32, 8, 1024, 128, 500),     # the 1K decode layer (Llama-3.1-8B attention shape)
    (2, 8, 2, 1000, 100, 500),      # ragged: L, L - W not multiples of any tile
    (1, 8, 8, 333, 64, 700),        # GQA 1
    (1, 16, 2, 700, 128, 500),      # GQA 8
    (1, 4, 2, 200, 0, 0),           # strict 4-bit: no window, no lines
    (1, 4, 1, 150, 200, 500),       # window longer than the prefix: nothing packed
    (1, 4, 1, 70, 16, 10000),       # every non-window position a line
    (8, 32, 8, 300, 64, 500),       # 64 (b, kv head) units: the narrow CTA shape (3 per SM)
])
def test_prefix_init_and_decode(B, Hq, Hkv, L, W, rho):
    p = Pair(B, Hq, Hkv, L, W, rho, cap=L + 200, seed=L)
    p.init()
    q, k, v = synth.decode_tokens(L, B, Hq, Hkv, 5)
    for t in range(5):
        out, ref = p.decode(q[t], k[t], v[t])
        check_decode(out, ref, f"step {t}")
    assert p.g.state()["T"] == L + 5 and p.g.state()["n_q"] == 5


def test_decode_loop_with_reselection():
    """64 decode steps, staging full, reselect + merge, 64 more, reselect + merge."""
    B, Hq, Hkv, L, W = 1, 32, 8, 1024, 128
    p = Pair(B, Hq, Hkv, L, W, 500, cap=L + 256, seed=5)
    p.init()
    q, k, v = synth.decode_tokens(5, B, Hq, Hkv, 140)
    t = 0
    for rnd in range(2):
        for _ in range(64):
            out, ref = p.decode(q[t], k[t], v[t])
            check_decode(out, ref, f"step {t}")
            t += 1
        # staging full: the kernel refuses the step and flags it
        H = hq()
        sentinel = torch.full((B, Hq, 128), 7.0, dtype=torch.float16, device="cuda")
        H.hq_decode_attn(p.g, dev(q[t]), dev(k[t]), dev(v[t]), out=sentinel)
        torch.cuda.synchronize()
        st = p.g.state()
        assert st["err"] & H.DEVERR_STAGING_FULL and st["T"] == L + t
        assert torch.all(sentinel == 7.0)
        p.g.state_t[:, H.STATE_ERR] = 0
        p.reselect_merge()
        assert p.g.state()["n_packed"] == L + t - W
    for _ in range(3):
        out, ref = p.decode(q[t], k[t], v[t])
        check_decode(out, ref, f"step {t}")
        t += 1


def test_decode_from_an_empty_cache():
    """No prefix at all: the first step attends to its own token alone; the cache
    then grows by decode steps only, and the first reselection + merge (over
    decoded positions, with the query buffer just filled) packs what left the
    window; decoding continues over packed, VL and ring positions."""
    B, Hq, Hkv, W = 2, 8, 2, 32
    p = Pair(B, Hq, Hkv, 64, W, 500, cap=256, seed=21)  # the drawn prefix is never installed
    assert p.g.state()["T"] == 0
    q, k, v = synth.decode_tokens(21, B, Hq, Hkv, W + 64 + 5)
    out, ref = p.decode(q[0], k[0], v[0])
    check_decode(out, ref, "first step")
    G = Hq // Hkv
    want = np.repeat(v[0].astype(np.float32), G, axis=1)  # softmax over one key: the new V row
    assert np.allclose(out.float().cpu().numpy(), want, atol=2e-3)
    for t in range(1, W + 64):
        out, ref = p.decode(q[t], k[t], v[t])
        check_decode(out, ref, f"step {t}")
    p.reselect_merge()
    assert p.g.state()["n_packed"] == 64
    for t in range(W + 64, W + 69):
        out, ref = p.decode(q[t], k[t], v[t])
        check_decode(out, ref, f"step {t}")


def test_reselect_before_staging_is_full():
    """A merge with fewer than 64 staged tokens packs only what left the window.
    The second reselection's buffer holds queries from before the first merge
    (which saw other keys), so the decode steps' stored log-sum-exps are not
    used for them and the selection's own first pass runs."""
    p = Pair(1, 8, 2, 500, 64, 500, cap=800, seed=9)
    p.init()
    q, k, v = synth.decode_tokens(9, 1, 8, 2, 25)
    for t in range(10):
        out, ref = p.decode(q[t], k[t], v[t])
        check_decode(out, ref)
    p.reselect_merge()        # every buffered query is fresh: row sums from the decode steps
    assert p.g.state()["n_packed"] == 510 - 64
    for t in range(10, 20):
        out, ref = p.decode(q[t], k[t], v[t])
        check_decode(out, ref)
    p.reselect_merge()        # 10 queries from before the last merge: the first pass runs
    assert p.g.state()["n_packed"] == 520 - 64
    for t in range(20, 25):
        out, ref = p.decode(q[t], k[t], v[t])
        check_decode(out, ref)


def test_capacity_flag():
    H = hq()
    p = Pair(1, 4, 1, 120, 8, 500, cap=128, seed=3)
    p.init()
    q, k, v = synth.decode_tokens(3, 1, 4, 1, 10)
    for t in range(8):
        out, ref = p.decode(q[t], k[t], v[t])
        check_decode(out, ref)
    H.hq_decode_attn(p.g, dev(q[8]), dev(k[8]), dev(v[8]))
    torch.cuda.synchronize()
    assert p.g.state()["err"] & H.DEVERR_CAPACITY and p.g.state()["T"] == 128


@pytest.mark.slow
def test_full_size_32k_layer():
    """The 32K decode layer (B=1, Hq=32, Hkv=8): init, one step, a 64-step period
    (every 8th step checked, so the ring's wrap at this geometry is covered),
    reselect + merge, one step."""
    B, Hq, Hkv, L, W = 1, 32, 8, 32768, 128
    p = Pair(B, Hq, Hkv, L, W, 500, cap=L + 128, seed=0)
    p.init()
    q, k, v = synth.decode_tokens(0, B, Hq, Hkv, 65)
    out, ref = p.decode(q[0], k[0], v[0])
    check_decode(out, ref, "first step")
    for t in range(1, 64):
        if t % 8 == 0 or t == 63:   # every 8th step (and the last, with the ring full) against the oracle
            out, ref = p.decode(q[t], k[t], v[t])
            check_decode(out, ref, f"step {t}")
        else:
            hq().hq_decode_attn(p.g, dev(q[t]), dev(k[t]), dev(v[t]))
            p.r.append(q[t], k[t], v[t])
    p.reselect_merge()
    out, ref = p.decode(q[64], k[64], v[64])
    check_decode(out, ref, "after merge")


def test_running_scores_over_three_periods():
    """Running (accumulated) column-mass scores: each reselection adds its
    column mass to the stored sums and ranks the sums; scores and selections
    against the oracle's running scores over three 64-token periods (the
    1K layer, B=2), decode checked after every merge."""
    B, Hq, Hkv, L, W = 2, 32, 8, 1024, 128
    p = Pair(B, Hq, Hkv, L, W, 500, cap=L + 4 * 64 + 64, seed=13, running=True)
    p.init()
    acc0 = p.g.score_acc.cpu().numpy()
    n0 = L - W
    for b in range(B):
        for h in range(Hkv):
            want = p.r.acc[b, h, :n0]
            assert np.allclose(acc0[b, h, :n0], want, rtol=5e-4, atol=0), (b, h)
            assert not acc0[b, h, n0:].any()
    q, k, v = synth.decode_tokens(13, B, Hq, Hkv, 3 * 64 + 1)
    t = 0
    for period in range(3):
        for i in range(64):   # the first step of a period follows a merge
            if i % 16 == 0:
                out, ref = p.decode(q[t], k[t], v[t])
                check_decode(out, ref, f"step {t}")
            else:
                hq().hq_decode_attn(p.g, dev(q[t]), dev(k[t]), dev(v[t]))
                p.r.append(q[t], k[t], v[t])
            t += 1
        p.reselect_merge()
        acc = p.g.score_acc.cpu().numpy()
        n = p.r.T - W
        for b in range(B):
            for h in range(Hkv):
                assert np.allclose(acc[b, h, :n], p.r.acc[b, h, :n], rtol=5e-4, atol=0), (period, b, h)
    out, ref = p.decode(q[t], k[t], v[t])
    check_decode(out, ref, "after the last merge")


def test_reset_then_reinstall_with_running_scores():
    """hq_cache_reset empties a used cache: every state row zero, every VL
    bitmap cleared, the running scores zero; a different prefix installed
    afterwards through the same buffers then matches a fresh oracle cache
    (selection, records, decode, reselection and merge)."""
    p = Pair(2, 8, 2, 700, 64, 500, cap=1000, seed=81, running=True)
    p.init()
    q, k, v = synth.decode_tokens(81, 2, 8, 2, 64)
    for t in range(64):
        hq().hq_decode_attn(p.g, dev(q[t]), dev(k[t]), dev(v[t]))
        p.r.append(q[t], k[t], v[t])
    p.reselect_merge()
    hq().hq_cache_reset(p.g)
    torch.cuda.synchronize()
    assert not p.g.state_t.any()
    assert not p.g.packed()["vl_bits"].any()
    assert not p.g.score_acc.any()
    # a shorter, different prefix through the same cache
    p.lay = synth.planted_layer(82, 2, 8, 2, 400)
    p.L = 400
    p.r = hybrid.HybridCacheRef(2, 8, 2, 64, 500, p.g.cap, accumulate=True)
    p.init()
    q, k, v = synth.decode_tokens(83, 2, 8, 2, 66)
    for t in range(64):
        if t % 16 == 0:
            out, ref = p.decode(q[t], k[t], v[t])
            check_decode(out, ref, f"after reset, step {t}")
        else:
            hq().hq_decode_attn(p.g, dev(q[t]), dev(k[t]), dev(v[t]))
            p.r.append(q[t], k[t], v[t])
    p.reselect_merge()
    out, ref = p.decode(q[64], k[64], v[64])
    check_decode(out, ref, "after reset and a merge")


def test_reselection_after_decode_steps_at_another_scale():
    """Decode steps run at a scale other than 1/sqrt(D) store no usable
    log-sum-exp (NaN), so the reselection computes its own row normalisers
    (its first pass) and still matches the oracle's column mass."""
    p = Pair(1, 8, 2, 700, 64, 500, cap=900, seed=95)
    p.init()
    q, k, v = synth.decode_tokens(95, 1, 8, 2, 64)
    for t in range(64):
        hq().hq_decode_attn(p.g, dev(q[t]), dev(k[t]), dev(v[t]), sm_scale=0.05)
        p.r.append(q[t], k[t], v[t])
    torch.cuda.synchronize()
    assert torch.isnan(p.g.qlse).all()
    p.reselect_merge()
