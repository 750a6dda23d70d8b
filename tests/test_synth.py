"""The seeded synthetic adapters follow their stated recipes (CPU): the Walsh-Hadamard
adapter's budget, per-row floor and index list, and the LoRDBA carriers and scales."""
import numpy as np
import pytest

from quantized_base_rank_b200 import synth


@pytest.mark.parametrize("N,K,r", [(4096, 4096, 16), (11008, 4096, 64), (64, 192, 8), (8, 64, 64)])
def test_qwha_inputs_recipe(N, K, r):
    ad = synth.qwha_inputs(N, K, r, seed=2)
    rp = ad["row_ptr"].numpy().astype(np.int64)
    col = ad["col"].numpy().astype(np.int64)
    c = ad["c"].float().numpy()
    p = min(r * (N + K), N * K)
    cnt = np.diff(rp)
    assert rp[0] == 0 and rp[-1] == col.size == c.size
    # the budget is spent exactly unless rows saturate at K
    assert rp[-1] == p or np.any(cnt == K)
    assert np.all(cnt >= min(max(1, p // (4 * N)), K)) and np.all(cnt <= K)
    for n in range(0, N, max(1, N // 64)):
        seg = col[rp[n]:rp[n + 1]]
        assert np.all(np.diff(seg) > 0) and (seg.size == 0 or (seg[0] >= 0 and seg[-1] < K))
    assert np.all(np.isfinite(c)) and abs(np.std(c) - 0.02) < 0.005


def test_qwha_inputs_are_seeded():
    a = synth.qwha_inputs(256, 512, 8, seed=5)
    b = synth.qwha_inputs(256, 512, 8, seed=5)
    d = synth.qwha_inputs(256, 512, 8, seed=6)
    assert all(np.array_equal(a[k].numpy(), b[k].numpy()) for k in ("row_ptr", "col"))
    assert np.array_equal(a["c"].float().numpy(), b["c"].float().numpy())
    assert not np.array_equal(a["col"].numpy(), d["col"].numpy())


def test_lordba_inputs_recipe():
    ad = synth.lordba_inputs(96, 128, 16, 3, seed=1)
    for k in ("B1", "B2"):
        assert set(np.unique(ad[k].numpy())) <= {-1.0, 1.0}
    assert ad["B1"].shape == (96, 16) and ad["B2"].shape == (16, 128)
    a = ad["alpha"].float().numpy()
    assert a.shape == (3, 96) and np.all((a >= 0.5 * 0.02 / 4 * 0.999) & (a <= 0.02 / 4 * 1.001))
    for k, shape in (("beta", (3, 16)), ("gamma", (3, 128))):
        v = ad[k].float().numpy()
        assert v.shape == shape and np.all((v >= 0.5 * 0.999) & (v <= 1.0))
