"""The tensor-core kernel's bounded waits, driven to their limit on the GPU without a hung copy.

The short-wait test build (libart_decode_shortwait.so: the same sources with the tensor-core
kernel's wait limit set to 1000 SM cycles instead of about a second) gives up on the first wait
that outlasts 1000 cycles -- waiting for the first K/V block to arrive from HBM already does.
The CTA then sets the timeout bit of the workspace status word and aborts: every role leaves its
loop, the copies and tensor-core operations it issued are waited for (the drains keep the long
limit), and every CTA of a cluster still reaches the cluster barriers.  Each call must return,
report ART_ERR_TIMEOUT (or ART_OK with oracle-correct outputs when no wait outlasted the limit),
and leave the context usable: the regular library then decodes the same problem correctly.

Cases run single-CTA clusters first (128 units fill the GPU), then 8-CTA clusters, for bf16 full
attention, bf16 ART and q8 ART (the q8 tensor-core variant and its converter warpgroup).
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import kv_cache_early_split_b200 as K  # noqa: E402
from kv_cache_early_split_b200 import build, capi  # noqa: E402
from kv_cache_early_split_b200 import inputs as I  # noqa: E402
from helpers import TOL, oracle_run  # noqa: E402

pytestmark = pytest.mark.gpu

ART = dict(eps_scale=1e-3, eps_dir=1e-4, patience=1, lanes=I.probe_lanes_strided(128, 16))

CASES = [
    # name, workload kwargs, mode
    ("bf16-full-cluster1", dict(kind="bf16", B=16, Hq=32, Hkv=8, L_max=512), "full"),
    ("bf16-art-cluster1", dict(kind="bf16", B=16, Hq=32, Hkv=8, L_max=512), "art"),
    ("bf16-art-cluster8", dict(kind="bf16", B=1, Hq=4, Hkv=1, L_max=4096), "art"),
    ("q8-art-cluster8", dict(kind="q8", B=1, Hq=4, Hkv=1, L_max=4096, tau=1e-6), "q8_art"),
]

_short = {}


def short_wait_lib():
    if "L" not in _short:
        _short["L"] = capi.load_variant(build.build_short_wait())
    return _short["L"]


def call(L, dp, mode, stream):
    p = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    sh = ctypes.byref(dp.shape)
    params = capi.make_params(ART["eps_scale"], ART["eps_dir"], ART["patience"], ART["lanes"])
    if mode == "full":
        return L.art_decode_attn_full(sh, capi.ART_BF16, p(dp.q), p(dp.k), p(dp.v), p(dp.seq_lens), p(dp.o),
                                      p(dp.tiles), p(dp.ws), dp.ws_bytes, stream)
    if mode == "art":
        return L.art_decode_attn_terminate(sh, capi.ART_BF16, p(dp.q), p(dp.k), p(dp.v), p(dp.seq_lens),
                                           ctypes.byref(params), p(dp.o), p(dp.tiles), p(dp.ws), dp.ws_bytes, stream)
    return L.art_decode_attn_q8_skipv_path(sh, p(dp.q), p(dp.k), p(dp.k_scale), p(dp.v), p(dp.v_scale),
                                           p(dp.seq_lens), dp.tau, ctypes.byref(params), p(dp.o), p(dp.tiles),
                                           p(dp.ws), dp.ws_bytes, capi.ART_Q8_TENSOR_CORE, stream)


def check_against_oracle(w, dp, mode):
    used = dp.split_tiles().cpu().numpy()
    base = "q8" if mode == "q8_art" else "full"
    ref = oracle_run(w, base, forced_used=used)
    err = float(np.max(np.abs(dp.o.cpu().numpy() - ref.o)))
    assert err <= TOL[w.kind], err


def test_short_waits_time_out_and_leave_the_context_usable():
    L = short_wait_lib()
    stream = torch.cuda.current_stream().cuda_stream
    timed_out = []
    for name, kw, mode in CASES:
        w = I.make_workload(d=128, tile=64, seed=31, sink=6.0, art=dict(ART), **kw)
        # (q8: the decode kernel is pinned by path below; the query names the default, the two-pass rule)
        assert K.kernel_name(K.upload(w), mode) == ("q8_pv_mma_kernel" if mode == "q8_art" else "art_decode_tc_kernel"), name
        dp = K.upload(w)
        dp.o.fill_(float("nan"))
        rc = call(L, dp, mode, stream)
        assert rc == capi.ART_OK, (name, capi.art_status_string(rc))
        st = L.art_read_device_status(dp.ws.data_ptr(), stream)  # synchronises
        assert st in (capi.ART_ERR_TIMEOUT, capi.ART_OK), (name, capi.art_status_string(st))
        if st == capi.ART_ERR_TIMEOUT:
            timed_out.append(name)
        else:
            check_against_oracle(w, dp, mode)
        # the context is intact: the regular library decodes the same buffers correctly
        K.decode(dp, mode)
        assert K.device_status(dp) == capi.ART_OK, name
        check_against_oracle(w, dp, mode)
    assert timed_out, "no call reached the short wait limit"
    print("timed out:", timed_out)
