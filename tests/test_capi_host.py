"""Host-side checks of the C ABI (no GPU): the library loads, exports every
symbol include/art_decode.h declares, sizes its workspace, and rejects invalid
arguments synchronously without touching the device (fake, never-dereferenced
pointer values are passed)."""
import ctypes
import re
import os

import pytest

from kv_cache_early_split_b200 import build, capi

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "art_decode.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return capi.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(art_\w+)\s*\(", text)))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 8
    assert sorted(capi.EXPORTS) == names
    for n in names:
        assert hasattr(L, n), n


def test_status_strings(L):
    for code in range(0, -7, -1):
        assert capi.art_status_string(code).startswith("ART_")
    assert capi.art_status_string(-99) == "ART_ERR_UNKNOWN"


def shape(**kw):
    d = dict(B=4, Hq=32, Hkv=8, d=128, L_max=32768, tile=64, num_splits=1)
    d.update(kw)
    return capi.art_shape(**d)


def test_workspace_sizes(L):
    s = shape()
    ws = capi.art_workspace_bytes(s)
    off_r = capi.art_workspace_tiles_read_offset(s)
    off_u = capi.art_workspace_split_tiles_offset(s)
    assert off_r >= 4 and off_r % 16 == 0
    assert off_u >= off_r + 4 * 4 * 8
    assert ws >= off_u + 4 * 4 * 32 + 4 * 4 * 32 * 130
    s8 = shape(num_splits=8)
    assert capi.art_workspace_bytes(s8) > ws
    assert capi.art_workspace_bytes(shape(B=0)) == 0
    assert capi.art_workspace_bytes(shape(num_splits=0)) == 0


def test_q8_workspace_sizes(L):
    """The two-pass q8 workspace extends the common one: scores [B, Hkv, L_max, G] fp32, tile and
    chunk maxima, a (2 + d)-float state per query head and chunk of every split, and for ART a
    34-float probe record per query head and tile plus a stop tile per query head and split."""
    for kw in (dict(), dict(num_splits=3), dict(d=64, tile=16), dict(Hq=8, Hkv=8, tile=256), dict(B=1, L_max=1)):
        s = shape(**kw)
        base, q8 = capi.art_workspace_bytes(s), capi.art_q8_workspace_bytes(s)
        n_max = -(-s.L_max // s.tile)
        assert q8 >= base + 4 * s.B * s.Hq * s.L_max + 4 * s.B * s.Hq * n_max
        chunks = -(-n_max // s.num_splits)  # chunks of at least one tile per split
        ct = min(32, 8 * max(1, 128 // s.tile))
        assert q8 >= base + 4 * s.B * s.Hq * s.num_splits * -(-chunks // ct) * (s.d + 2)
        assert q8 >= base + 4 * s.B * s.Hq * n_max * 34 + 4 * s.B * s.Hq * s.num_splits
    assert capi.art_q8_workspace_bytes(shape(B=0)) == 0
    # the default q8 workload: 2 x 8 kv heads x 32768 positions x 4 heads of scores = 8 MiB, and
    # 2 x 32 heads x 512 tiles of 136-byte probe records = 4.25 MiB, and change
    s = shape(B=2)
    assert capi.art_q8_workspace_bytes(s) - capi.art_workspace_bytes(s) < 15 << 20


A = 0x100000  # fake 16-byte aligned device addresses (never dereferenced)


def full(s, **kw):
    args = dict(dtype=capi.ART_BF16, q=A, k=A * 2, v=A * 3, seq=A * 4, o=A * 5, tiles=A * 6, ws=A * 7,
                ws_bytes=capi.art_workspace_bytes(s) if capi.art_workspace_bytes(s) else 1 << 20)
    args.update(kw)
    return capi.art_decode_attn_full(s, args["dtype"], args["q"], args["k"], args["v"], args["seq"], args["o"],
                                     args["tiles"], args["ws"], args["ws_bytes"], None)


def term(s, params, **kw):
    wsb = capi.art_workspace_bytes(s) or (1 << 20)
    return capi.art_decode_attn_terminate(s, kw.get("dtype", capi.ART_BF16), A, A * 2, A * 3, A * 4, params, A * 5,
                                          A * 6, A * 7, kw.get("ws_bytes", wsb), None)


def q8(s, params=None, tau=1e-6, **kw):
    wsb = kw.get("ws_bytes", capi.art_workspace_bytes(s) or (1 << 20))
    return capi.art_decode_attn_q8_skipv(s, A, A * 2, kw.get("ks", A * 8), A * 3, kw.get("vs", A * 9), A * 4, tau,
                                         params, A * 5, A * 6, A * 7, wsb, None)


def test_invalid_arguments_full(L):
    s = shape()
    assert full(s, q=None) == capi.ART_ERR_INVALID_ARG
    assert full(s, o=None) == capi.ART_ERR_INVALID_ARG
    assert full(s, seq=None) == capi.ART_ERR_INVALID_ARG
    assert full(s, q=A + 4) == capi.ART_ERR_INVALID_ARG  # misaligned
    assert full(s, dtype=7) == capi.ART_ERR_INVALID_ARG
    assert full(s, ws=None) == capi.ART_ERR_WORKSPACE
    assert full(s, ws_bytes=capi.art_workspace_bytes(s) - 1) == capi.ART_ERR_WORKSPACE
    assert full(shape(Hq=30)) == capi.ART_ERR_INVALID_ARG  # Hq % Hkv
    assert full(shape(B=0)) == capi.ART_ERR_INVALID_ARG
    assert full(shape(d=96)) == capi.ART_ERR_UNSUPPORTED
    assert full(shape(tile=48)) == capi.ART_ERR_UNSUPPORTED
    assert full(shape(Hq=128, Hkv=8)) == capi.ART_ERR_UNSUPPORTED  # 16 query heads per kv head


def test_invalid_arguments_terminate(L):
    s = shape()
    ok = capi.make_params(1e-3, 1e-4, 1, list(range(0, 128, 8)))
    assert term(s, None) == capi.ART_ERR_INVALID_ARG
    assert term(s, capi.make_params(1e-3, 1e-4, 0, [0])) == capi.ART_ERR_INVALID_ARG  # patience 0
    assert term(s, capi.make_params(1e-3, 1e-4, 1, [])) == capi.ART_ERR_INVALID_ARG  # no lanes
    assert term(s, capi.make_params(1e-3, 1e-4, 1, list(range(33)))) == capi.ART_ERR_INVALID_ARG
    assert term(s, capi.make_params(1e-3, 1e-4, 1, [0, 128])) == capi.ART_ERR_INVALID_ARG  # lane >= d
    assert term(s, capi.make_params(1e-3, 1e-4, 1, [-1])) == capi.ART_ERR_INVALID_ARG
    assert term(s, capi.make_params(1e-3, 1e-4, 1, [3, 3])) == capi.ART_ERR_INVALID_ARG  # duplicate
    assert term(s, capi.make_params(1e-3, 1e-4, 1, [0], max_spec_tiles=-1)) == capi.ART_ERR_INVALID_ARG
    assert term(shape(d=64), capi.make_params(1e-3, 1e-4, 1, [64])) == capi.ART_ERR_INVALID_ARG
    assert term(s, ok, ws_bytes=16) == capi.ART_ERR_WORKSPACE


def test_invalid_arguments_q8(L):
    s = shape()
    assert q8(s, ks=None) == capi.ART_ERR_INVALID_ARG
    assert q8(s, vs=A + 2) == capi.ART_ERR_INVALID_ARG
    assert q8(s, tau=float("nan")) == capi.ART_ERR_INVALID_ARG
    assert q8(shape(L_max=32767)) == capi.ART_ERR_UNSUPPORTED  # scale rows not 16-byte granular
    assert q8(s, params=capi.make_params(1e-3, 1e-4, 1, [200])) == capi.ART_ERR_INVALID_ARG
    # the same checks, synchronously and before any launch, with a two-pass workspace
    big = capi.art_q8_workspace_bytes(s)
    assert q8(s, ks=None, ws_bytes=big) == capi.ART_ERR_INVALID_ARG
    assert q8(s, vs=A + 2, ws_bytes=big) == capi.ART_ERR_INVALID_ARG
    assert q8(s, tau=float("nan"), ws_bytes=big) == capi.ART_ERR_INVALID_ARG
    s2 = shape(L_max=32767)
    assert q8(s2, ws_bytes=capi.art_q8_workspace_bytes(s2)) == capi.ART_ERR_UNSUPPORTED
    assert q8(s, ws_bytes=capi.art_workspace_bytes(s) - 16) == capi.ART_ERR_WORKSPACE
    # ART on the two passes: the rule's settings are checked before any launch, and shapes outside the
    # tensor-core passes (d = 64, tile 16, 8 heads per kv head) are refused on that path
    art = capi.make_params(1e-3, 1e-4, 2, [0, 8, 16])
    assert q8(s, params=capi.make_params(1e-3, 1e-4, 1, [200]), ws_bytes=big) == capi.ART_ERR_INVALID_ARG
    assert q8(s, params=capi.make_params(1e-3, 1e-4, 0, [0]), ws_bytes=big) == capi.ART_ERR_INVALID_ARG

    def two_pass(sh):
        return capi.art_decode_attn_q8_skipv_path(sh, A, A * 2, A * 8, A * 3, A * 9, A * 4, 1e-6, art, A * 5, A * 6,
                                                  A * 7, capi.art_q8_workspace_bytes(sh), capi.ART_Q8_TWO_PASS, None)
    assert two_pass(shape(d=64)) == capi.ART_ERR_UNSUPPORTED
    assert two_pass(shape(tile=16)) == capi.ART_ERR_UNSUPPORTED
    assert two_pass(shape(Hq=64, Hkv=8)) == capi.ART_ERR_UNSUPPORTED


def test_read_status_rejects_null(L):
    assert capi.art_read_device_status(None, None) == capi.ART_ERR_INVALID_ARG


def test_kernel_name_query(L):
    """The selection query follows the documented tensor-core eligibility rule."""
    tc = shape(Hq=32, Hkv=8, d=128, tile=64)
    assert capi.art_kernel_name(tc, capi.ART_BF16, False, True) == "art_decode_tc_kernel"
    assert capi.art_kernel_name(tc, capi.ART_BF16, False, False) == "art_decode_tc_kernel"
    assert capi.art_kernel_name(shape(Hq=32, Hkv=8, d=128, tile=128), capi.ART_BF16, 0, 1) == "art_decode_tc_kernel"
    assert capi.art_kernel_name(tc, capi.ART_F32, False, True) == "art_decode_kernel"
    # q8 ART with 3 or 4 heads per kv head, d = 128, tile 64 / 128, even L_max: the tensor cores;
    # q8 full attention: two streaming passes (the second named) given the q8 workspace
    assert capi.art_kernel_name(tc, capi.ART_BF16, True, True) == "q8_pv_mma_kernel"  # (given the q8 workspace)
    assert capi.art_kernel_name(tc, capi.ART_BF16, True, False) == "q8_pv_mma_kernel"
    assert capi.art_kernel_name(shape(Hq=24, Hkv=8, d=128, tile=64), capi.ART_BF16, True, False) == "q8_pv_mma_kernel"
    # (the tensor-core passes move 32-row steps: tiles of 16 take the CUDA-core passes)
    assert capi.art_kernel_name(shape(Hq=32, Hkv=8, d=128, tile=16), capi.ART_BF16, True, False) == "q8_pv_kernel"
    assert capi.art_kernel_name(shape(Hq=32, Hkv=8, d=128, tile=32), capi.ART_BF16, True, False) == "q8_pv_mma_kernel"
    assert capi.art_kernel_name(shape(Hq=24, Hkv=8, d=128, tile=128), capi.ART_BF16, 1, 1) == "q8_pv_mma_kernel"
    # other q8 shapes: full attention as two streaming passes (the second named), ART one pass
    q8o = shape(Hq=16, Hkv=8, d=128, tile=64)
    assert capi.art_kernel_name(q8o, capi.ART_BF16, True, False) == "q8_pv_kernel"
    assert capi.art_kernel_name(q8o, capi.ART_BF16, True, True) == "art_decode_kernel"
    assert capi.art_kernel_name(shape(Hq=24, Hkv=8, d=64, tile=16), capi.ART_BF16, 1, 0) == "q8_pv_kernel"
    assert capi.art_kernel_name(shape(Hq=32, Hkv=8, d=64, tile=64), capi.ART_BF16, 0, 1) == "art_decode_kernel"
    assert capi.art_kernel_name(shape(Hq=32, Hkv=8, d=128, tile=32), capi.ART_BF16, 0, 1) == "art_decode_kernel"
    assert capi.art_kernel_name(shape(Hq=32, Hkv=8, d=96, tile=64), capi.ART_BF16, 0, 1) is None
    assert capi.art_kernel_name(shape(Hq=32, Hkv=2, d=128, tile=64), capi.ART_BF16, 0, 1) is None
    assert capi.art_kernel_name(shape(B=0), capi.ART_BF16, 0, 1) is None


def test_status_strings_new_codes(L):
    assert capi.art_status_string(capi.ART_ERR_ORDER) == "ART_ERR_ORDER"
    assert capi.art_status_string(capi.ART_ERR_PAGE) == "ART_ERR_PAGE"
    assert capi.art_status_string(capi.ART_ERR_INDEX) == "ART_ERR_INDEX"


def test_invalid_arguments_orders(L):
    s = shape()
    assert capi.art_tile_order_recency(s, None, A, None) == capi.ART_ERR_INVALID_ARG
    assert capi.art_tile_order_recency(shape(B=0), A, A * 2, None) == capi.ART_ERR_INVALID_ARG
    assert capi.art_tile_key_summary(s, capi.ART_BF16, None, A, A * 2, None) == capi.ART_ERR_INVALID_ARG
    assert capi.art_tile_key_summary(shape(d=96), capi.ART_BF16, A, A * 2, A * 3, None) == capi.ART_ERR_UNSUPPORTED
    assert capi.art_tile_key_summary(s, 7, A, A * 2, A * 3, None) == capi.ART_ERR_INVALID_ARG
    assert capi.art_tile_order_importance(shape(Hq=30), capi.ART_BF16, A, A * 2, A * 3, A * 4,
                                          None) == capi.ART_ERR_INVALID_ARG
    assert capi.art_tile_order_importance(s, 7, A, A * 2, A * 3, A * 4, None) == capi.ART_ERR_INVALID_ARG
    big = shape(L_max=1 << 26, tile=16)  # 4M tiles of scores would not fit one block's shared memory
    assert capi.art_tile_order_importance(big, capi.ART_BF16, A, A * 2, A * 3, A * 4,
                                          None) == capi.ART_ERR_UNSUPPORTED
    ok = capi.make_params(1e-3, 1e-4, 1, [0, 8])
    wsb = capi.art_workspace_bytes(s)

    def ordered(params, order):
        return capi.art_decode_attn_terminate_ordered(s, capi.ART_BF16, A, A * 2, A * 3, A * 4, params, order,
                                                      A * 5, A * 6, A * 7, wsb, None)

    assert ordered(None, A * 8) == capi.ART_ERR_INVALID_ARG
    assert ordered(ok, None) == capi.ART_ERR_INVALID_ARG
    assert ordered(ok, A * 8 + 2) == capi.ART_ERR_INVALID_ARG  # misaligned sequence array


def test_invalid_arguments_paged(L):
    s = shape(L_max=4096, tile=64)
    wsb = capi.art_workspace_bytes(s)

    def paged(pages, params=None, order=None):
        return capi.art_decode_attn_paged(s, capi.ART_BF16, A, A * 2, A * 3, pages, A * 4, params, order, A * 5,
                                          A * 6, A * 7, wsb, None)

    good = capi.art_paged_kv(128, 200, 32, A * 8)
    assert paged(None) == capi.ART_ERR_INVALID_ARG
    assert paged(capi.art_paged_kv(128, 200, 32, None)) == capi.ART_ERR_INVALID_ARG
    assert paged(capi.art_paged_kv(96, 200, 64, A * 8)) == capi.ART_ERR_UNSUPPORTED  # not a multiple of the tile
    assert paged(capi.art_paged_kv(128, 200, 16, A * 8)) == capi.ART_ERR_INVALID_ARG  # 16 * 128 < L_max
    assert paged(capi.art_paged_kv(128, 0, 32, A * 8)) == capi.ART_ERR_INVALID_ARG
    assert paged(capi.art_paged_kv(128, 1 << 30, 32, A * 8)) == capi.ART_ERR_UNSUPPORTED  # pool index overflow
    assert paged(good, params=None, order=A * 9) == capi.ART_ERR_INVALID_ARG  # a sequence needs ART
    assert capi.art_decode_attn_q8_skipv_paged(s, A, A * 2, None, A * 3, A * 4, good, A * 5, 1e-6, None, A * 6,
                                               A * 7, A * 9, wsb, None) == capi.ART_ERR_INVALID_ARG


def test_invalid_arguments_eviction(L):
    s = shape(L_max=4096)
    assert capi.art_evict_random_select(s, A, None, 4, 8, 64, A * 2, A * 3, None) == capi.ART_ERR_INVALID_ARG
    assert capi.art_evict_random_select(s, A, A * 2, 40, 40, 64, A * 3, A * 4, None) == capi.ART_ERR_INVALID_ARG
    assert capi.art_evict_random_select(s, A, A * 2, -1, 8, 64, A * 3, A * 4, None) == capi.ART_ERR_INVALID_ARG
    assert capi.art_evict_random_select(s, A, A * 2, 0, 0, 0, A * 3, A * 4, None) == capi.ART_ERR_INVALID_ARG
    assert capi.art_evict_compact(s, 7, A, None, A * 2, 64, A * 3, None, None) == capi.ART_ERR_INVALID_ARG
    assert capi.art_evict_compact(s, capi.ART_KV_Q8, A, None, A * 2, 64, A * 3, None,
                                  None) == capi.ART_ERR_INVALID_ARG  # q8 needs its scales
    assert capi.art_evict_compact(s, capi.ART_KV_BF16, A, A * 4, A * 2, 64, A * 3, A * 5,
                                  None) == capi.ART_ERR_INVALID_ARG  # scales only with q8
    assert capi.art_evict_compact(s, capi.ART_KV_BF16, A, None, A * 2, 64, A * 3 + 8, None,
                                  None) == capi.ART_ERR_INVALID_ARG  # misaligned destination
    assert capi.art_evict_compact(shape(d=4), capi.ART_KV_BF16, A, None, A * 2, 64, A * 3, None,
                                  None) == capi.ART_ERR_UNSUPPORTED  # 8-byte rows


def test_missing_library_fails_loudly(tmp_path):
    """No fallback: with the CUDA library absent, the first call raises instead of computing anything."""
    import subprocess
    import sys

    code = (
        "import sys; sys.path.insert(0, %r)\n"
        "from kv_cache_early_split_b200 import capi\n"
        "capi.LIB_PATH = %r\n"
        "try:\n"
        "    capi.art_workspace_bytes(capi.art_shape(1, 1, 1, 64, 64, 64, 1))\n"
        "except OSError as e:\n"
        "    print('raised', 'no fallback' in str(e))\n"
    ) % (os.path.dirname(os.path.dirname(os.path.abspath(__file__))), str(tmp_path / "absent.so"))
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=120)
    assert r.stdout.strip() == "raised True", r.stdout + r.stderr
