"""The V-skip counters of the two-pass q8 path against the oracle's record of the skip test.

Page "La Elegancia de la Omision": row j leaves head g's numerator when exp(s_j - m'_t) < tau,
m'_t the split's running maximum after row j's tile.  The device counts, per (batch, kv head,
split), the rows left out for every head of the group and the tiles whose rows all were (their
V is not read at all).  The oracle records p / tau per (head, row) in double precision; a row
whose largest ratio over the group lies within WINDOW of 1 may go either way (the device decides
in fp32 on log2-domain scores), so each count must lie between the oracle's certain count and
the certain plus the undecided ones.  The outputs themselves are checked by the parity tests.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import kv_cache_early_split_b200 as K  # noqa: E402
from kv_cache_early_split_b200 import capi  # noqa: E402
from kv_cache_early_split_b200 import inputs as I  # noqa: E402
from helpers import TOL  # noqa: E402

import oracle  # noqa: E402

pytestmark = pytest.mark.gpu
WINDOW = 1e-3


def oracle_counts(w, tau, S):
    r = oracle.decode(kind=oracle.KV_Q8, q=w.q, k=w.k, v=w.v, k_scale=w.k_scale, v_scale=w.v_scale,
                      seq_lens=w.seq_lens, tile=w.tile, num_splits=S, tau=tau, want_vskip=True, n_threads=8)
    G = w.Hq // w.Hkv
    lo = np.zeros((w.B, w.Hkv, S, 2), np.int64)
    hi = np.zeros_like(lo)
    for b in range(w.B):
        L = int(w.seq_lens[b])
        n = -(-L // w.tile)
        for kvh in range(w.Hkv):
            ratio = r.vskip[b, kvh * G:(kvh + 1) * G, :L].max(axis=0)  # the group's largest p / tau per row
            sure = ratio < 1.0 - WINDOW
            maybe = ratio < 1.0 + WINDOW
            for s in range(S):
                t0, t1 = (s * n) // S, ((s + 1) * n) // S
                rows = slice(t0 * w.tile, min(t1 * w.tile, L))
                lo[b, kvh, s, 0], hi[b, kvh, s, 0] = sure[rows].sum(), maybe[rows].sum()
                for t in range(t0, t1):
                    tr = slice(t * w.tile, min((t + 1) * w.tile, L))
                    lo[b, kvh, s, 1] += int(sure[tr].all())
                    hi[b, kvh, s, 1] += int(maybe[tr].all())
    return r, lo, hi


@pytest.mark.parametrize("tau", [1e-6, 1e-3, 1e-2])
@pytest.mark.parametrize("S", [1, 3])
def test_vskip_counts_match_oracle(tau, S):
    w = I.make_workload(kind="q8", B=2, Hq=8, Hkv=2, d=128, L_max=4096, tile=64, num_splits=S,
                        seq_lens=[4096, 2777], seed=61, sink=8.0, gumbel_scale=2.0, lognormal_v=True, tau=tau)
    dp = K.upload(w)
    assert K.kernel_name(dp, "q8") == "q8_pv_mma_kernel"
    K.decode(dp, "q8", tau=tau, q8_path="two_pass")
    assert K.device_status(dp) == capi.ART_OK
    got = dp.vskip_counts().cpu().numpy().astype(np.int64)
    r, lo, hi = oracle_counts(w, tau, S)
    assert float(np.max(np.abs(dp.o.cpu().numpy() - r.o))) <= TOL["q8"]
    assert np.all(got >= lo) and np.all(got <= hi), (got.tolist(), lo.tolist(), hi.tolist())
    if tau >= 1e-3:
        assert got[..., 0].sum() > 0, "the case must skip rows"
    print(f"tau {tau:g} S {S}: rows left out {int(got[..., 0].sum())}, V tiles not read {int(got[..., 1].sum())}")


def test_vskip_counts_zero_without_skip():
    w = I.make_workload(kind="q8", B=1, Hq=4, Hkv=1, d=128, L_max=2048, tile=64, seed=62, tau=0.0)
    dp = K.upload(w)
    off = capi.art_workspace_vskip_offset(dp.shape)
    dp.ws[off:off + 8 * w.B * w.Hkv].fill_(0x7F)  # the counters must be written, not left over
    K.decode(dp, "q8", tau=0.0, q8_path="two_pass")
    assert K.device_status(dp) == capi.ART_OK
    assert np.all(dp.vskip_counts().cpu().numpy() == 0)
