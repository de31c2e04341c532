"""Seeded random combinations of the cache's options, each through install,
decode, a full 64-token period, reselection and merge, every sequence against
its own oracle cache (bit-exact records and VL store, decode within its
tolerances, selections against the oracle's column mass).

The draws cover batch sizes 1-3 with ragged lengths (1 .. 900 tokens),
GQA 1-8, windows that are not multiples of the 16-row tile (0 .. 128), line
ratios from 0 to 100 %, the four code widths, and dense or shuffled paged
stores."""
import numpy as np
import pytest

from tests.test_gpu_varlen import Ragged, _tokens

pytestmark = pytest.mark.gpu

WIDTHS = [(4, 4), (8, 8), (4, 2), (2, 4)]


def _draw(case):
    rng = np.random.default_rng(1000 + case)
    B = int(rng.integers(1, 4))
    Hkv = int(rng.choice([1, 2]))
    G = int(rng.choice([1, 2, 4, 8]))
    W = int(rng.choice([0, 5, 16, 33, 64, 100, 128]))
    rho = int(rng.choice([0, 100, 500, 2500, 10000]))
    kb, vb = WIDTHS[int(rng.integers(0, 4))]
    paged = bool(rng.integers(0, 2))
    lengths = [int(x) for x in rng.integers(1, 901, size=B)]
    return B, Hkv, G, W, rho, kb, vb, paged, lengths


@pytest.mark.parametrize("case", range(48))
def test_random_option_combinations(case):
    B, Hkv, G, W, rho, kb, vb, paged, lengths = _draw(case)
    Hq = G * Hkv
    rg = Ragged(lengths, Hq, Hkv, W, rho, cap=max(lengths) + 200, seed=2000 + case, paged=paged, k_bits=kb, v_bits=vb)
    for b in range(B):
        rg.install(b, check=True)
        rg.check_store(b)
    q, k, v = _tokens(3000 + case, B, Hq, Hkv, 67)
    for t in range(64):
        rg.decode(q[t], k[t], v[t], check=(t % 9 == 0 or t == 63))
    rg.reselect_merge()
    for t in range(64, 67):
        rg.decode(q[t], k[t], v[t])


@pytest.mark.parametrize("case", range(24))
def test_random_prefill_shapes(case):
    """Seeded random prefill shapes (L 1 .. 700, GQA 1-8, batch 1-2, window
    0 .. 300, line ratio 0 .. 100 %), both Q.K formats, whole output against
    the oracle within the prefill bound."""
    from tests.test_gpu_prefill import PF_RELL2, _run
    rng = np.random.default_rng(4000 + case)
    B = int(rng.integers(1, 3))
    Hkv = int(rng.choice([1, 2]))
    G = int(rng.choice([1, 2, 4, 8]))
    L = int(rng.integers(1, 701))
    W = int(rng.choice([0, 7, 64, 128, 300]))
    rho = int(rng.choice([0, 250, 500, 10000]))
    fmt = "int8" if case % 2 else "e4m3"
    got, ref = _run(B, G * Hkv, Hkv, L, W, rho, seed=5000 + case, fmt=fmt)
    assert np.all(np.isfinite(got))
    for (b, h), r in ref.items():
        g = got[b, h]
        rel = np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30)
        assert rel <= PF_RELL2, (case, b, h, rel, (B, G * Hkv, Hkv, L, W, rho, fmt))


@pytest.mark.parametrize("case", range(8))
def test_random_large_ragged_batches(case):
    """Seeded random batches of 10 .. 40 sequences with 4 or 8 kv heads (more
    than 37 units: the stream-K decode grid), ragged lengths 1 .. 2000, a
    random code width, dense or paged: installs, a period with checked steps,
    reselection and merge, against per-sequence oracles."""
    rng = np.random.default_rng(6000 + case)
    B = int(rng.integers(10, 41))
    Hkv = int(rng.choice([4, 8]))
    G = int(rng.choice([1, 4]))
    W = int(rng.choice([16, 64, 128]))
    kb, vb = WIDTHS[int(rng.integers(0, 4))]
    paged = bool(rng.integers(0, 2))
    lengths = [int(x) for x in rng.integers(1, 2001, size=B)]
    rg = Ragged(lengths, G * Hkv, Hkv, W, 500, cap=max(lengths) + 200, seed=7000 + case, paged=paged,
                k_bits=kb, v_bits=vb)
    for b in range(B):
        rg.install(b, check=(b % 8 == 0))
    q, k, v = _tokens(8000 + case, B, G * Hkv, Hkv, 66)
    for t in range(64):
        rg.decode(q[t], k[t], v[t], check=(t % 21 == 0 or t == 63))
    rg.reselect_merge()
    for t in range(64, 66):
        rg.decode(q[t], k[t], v[t])
