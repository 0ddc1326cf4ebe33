"""The allocation-free entry point art_decode_attn_terminate_noalloc.

It serves callers that cannot allocate device memory (a host framework that
hands a plugin only its input and output buffers, or a hot path that must not
call cudaMalloc): its workspace is a 4 MiB device array inside the library.
This test calls it through the C ABI twice in a row and checks both results
against the regular art_decode_attn_terminate (caller-provided workspace) with
the tolerances the parity tests use; it also checks the size limit.  The file
is named so that pytest collects it last.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import kv_cache_early_split_b200 as K  # noqa: E402
from kv_cache_early_split_b200 import capi  # noqa: E402
from kv_cache_early_split_b200 import inputs as I  # noqa: E402
from helpers import TOL  # noqa: E402

pytestmark = pytest.mark.gpu


def _noalloc(dp, art, stream):
    params = capi.make_params(art["eps_scale"], art["eps_dir"], art["patience"], art["lanes"])
    dtype = capi.ART_F32 if dp.kind == "f32" else capi.ART_BF16
    return capi.art_decode_attn_terminate_noalloc(
        dp.shape, dtype, dp.q.data_ptr(), dp.k.data_ptr(), dp.v.data_ptr(), dp.seq_lens.data_ptr(), params,
        dp.o.data_ptr(), dp.tiles.data_ptr(), stream)


@pytest.mark.parametrize("S", [1, 4])
def test_noalloc_matches_workspace_entry_point(S):
    w = I.make_workload(kind="bf16", B=3, Hq=16, Hkv=4, d=128, L_max=4096, tile=64, num_splits=S,
                        seq_lens=[4096, 2500, 777], seed=77, sink=8.0)
    art = dict(eps_scale=5e-2, eps_dir=1e-2, patience=2, lanes=I.probe_lanes_strided(128, 16))
    stream = torch.cuda.current_stream().cuda_stream

    ref = K.upload(w)
    K.decode(ref, "art", art=art)
    assert K.device_status(ref) == capi.ART_OK
    o_ref = ref.o.cpu().numpy()
    t_ref = ref.tiles.cpu().numpy()
    assert np.all(t_ref >= 1)

    dp = K.upload(w)
    for call in range(2):  # the second call reuses the scratch the first one left behind
        dp.o.fill_(float("nan"))
        dp.tiles.fill_(-1)
        rc = _noalloc(dp, art, stream)
        assert rc == capi.ART_OK, capi.art_status_string(rc)
        torch.cuda.synchronize()
        o = dp.o.cpu().numpy()
        t = dp.tiles.cpu().numpy()
        assert np.array_equal(t, t_ref), (call, t, t_ref)
        assert np.max(np.abs(o - o_ref)) <= TOL["bf16"], call


def test_noalloc_rejects_oversized_workspace():
    # 64 x 64 heads x 8 splits x 130 floats > 4 MiB: refused before any work is enqueued
    shape = capi.art_shape(64, 64, 8, 128, 4096, 64, 8)
    assert capi.art_workspace_bytes(shape) > (4 << 20)
    params = capi.make_params(1e-3, 1e-4, 1, [0, 8])
    a = 0x100000
    rc = capi.art_decode_attn_terminate_noalloc(shape, capi.ART_BF16, a, a, a, a, params, a, a, None)
    assert rc == capi.ART_ERR_WORKSPACE
