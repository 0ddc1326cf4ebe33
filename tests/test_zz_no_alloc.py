"""The allocation-free entry point art_decode_attn_terminate_noalloc.

It serves callers that cannot allocate device memory (a host framework that
hands a plugin only its input and output buffers, or a hot path that must not
call cudaMalloc): its workspace is a 4 MiB device array inside the library.
These tests call it through the C ABI and check its results against the
regular art_decode_attn_terminate (caller-provided workspace) with the
tolerances the parity tests use:

* on the tensor-core kernel (bf16, d = 128, G = 4) and on the CUDA-core kernel
  (fp32, d = 64, one head, the small fp32 workload's shape), each with one and
  with four KV splits;
* twice in a row, with a call of the other shape in between, so that the
  second checked call starts from the other shape's leftovers in the array;
* with one sequence given an invalid length: its outputs are NaN and its
  tiles 0, the other sequences are unaffected;
* and the size limit.

The file is named so that pytest collects it last.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import kv_cache_early_split_b200 as K  # noqa: E402
from kv_cache_early_split_b200 import capi  # noqa: E402
from kv_cache_early_split_b200 import inputs as I  # noqa: E402
from helpers import TOL  # noqa: E402

pytestmark = pytest.mark.gpu

ART_BF16 = dict(eps_scale=5e-2, eps_dir=1e-2, patience=2, lanes=I.probe_lanes_strided(128, 16))
ART_F32 = dict(eps_scale=1e-2, eps_dir=1e-3, patience=1, lanes=list(range(8)))


def _bf16_case(S):
    return I.make_workload(kind="bf16", B=3, Hq=16, Hkv=4, d=128, L_max=4096, tile=64, num_splits=S,
                           seq_lens=[4096, 2500, 777], seed=77, sink=8.0), ART_BF16


def _f32_case(S):
    return I.make_workload(kind="f32", B=1, Hq=1, Hkv=1, d=64, L_max=4096, tile=64, num_splits=S,
                           seed=78), ART_F32


def _noalloc(dp, art, stream):
    params = capi.make_params(art["eps_scale"], art["eps_dir"], art["patience"], art["lanes"])
    dtype = capi.ART_F32 if dp.kind == "f32" else capi.ART_BF16
    return capi.art_decode_attn_terminate_noalloc(
        dp.shape, dtype, dp.q.data_ptr(), dp.k.data_ptr(), dp.v.data_ptr(), dp.seq_lens.data_ptr(), params,
        dp.o.data_ptr(), dp.tiles.data_ptr(), stream)


def _reference(w, art):
    ref = K.upload(w)
    K.decode(ref, "art", art=art)
    assert K.device_status(ref) == capi.ART_OK
    t_ref = ref.tiles.cpu().numpy()
    assert np.all(t_ref >= 1)
    return ref.o.cpu().numpy(), t_ref


@pytest.mark.parametrize("S", [1, 4])
@pytest.mark.parametrize("case,other", [(_bf16_case, _f32_case), (_f32_case, _bf16_case)],
                         ids=["bf16_d128_tensor_core", "f32_d64_cuda_core"])
def test_noalloc_matches_workspace_entry_point(case, other, S):
    w, art = case(S)
    w2, art2 = other(5 - S)  # the other kernel, with the other split count
    stream = torch.cuda.current_stream().cuda_stream
    o_ref, t_ref = _reference(w, art)

    dp = K.upload(w)
    dp2 = K.upload(w2)
    for call in range(2):
        dp.o.fill_(float("nan"))
        dp.tiles.fill_(-1)
        rc = _noalloc(dp, art, stream)
        assert rc == capi.ART_OK, capi.art_status_string(rc)
        torch.cuda.synchronize()
        o = dp.o.cpu().numpy()
        t = dp.tiles.cpu().numpy()
        assert np.array_equal(t, t_ref), (call, t, t_ref)
        assert np.max(np.abs(o - o_ref)) <= TOL[w.kind], call
        # a call of the other shape leaves its own contents in the shared array before the next call
        rc = _noalloc(dp2, art2, stream)
        assert rc == capi.ART_OK, capi.art_status_string(rc)
        torch.cuda.synchronize()


@pytest.mark.parametrize("S", [1, 4])
@pytest.mark.parametrize("bad_len", [0, 4097])
def test_noalloc_invalid_length_gives_nan_and_zero_tiles(bad_len, S):
    w, art = _bf16_case(S)
    o_ref, t_ref = _reference(w, art)
    dp = K.upload(w)
    dp.seq_lens[1] = bad_len  # sequence 1: outside [1, L_max]
    rc = _noalloc(dp, art, torch.cuda.current_stream().cuda_stream)
    assert rc == capi.ART_OK, capi.art_status_string(rc)
    torch.cuda.synchronize()
    o = dp.o.cpu().numpy()
    t = dp.tiles.cpu().numpy()
    assert np.all(np.isnan(o[1])) and np.all(t[1] == 0)
    for b in (0, 2):
        assert np.array_equal(t[b], t_ref[b])
        assert np.max(np.abs(o[b] - o_ref[b])) <= TOL["bf16"]


def test_noalloc_rejects_oversized_workspace():
    # 64 x 64 heads x 8 splits x 130 floats > 4 MiB: refused before any work is enqueued
    shape = capi.art_shape(64, 64, 8, 128, 4096, 64, 8)
    assert capi.art_workspace_bytes(shape) > (4 << 20)
    params = capi.make_params(1e-3, 1e-4, 1, [0, 8])
    a = 0x100000
    rc = capi.art_decode_attn_terminate_noalloc(shape, capi.ART_BF16, a, a, a, a, params, a, a, None)
    assert rc == capi.ART_ERR_WORKSPACE
