"""ctypes binding of the C ABI in include/art_decode.h (argument marshalling only).

Every function here has the name of the C entry point it forwards to and takes
raw pointers (ints) and sizes, exactly like the C signature.  There is no
fallback: if libart_decode.so cannot be loaded, the first call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libart_decode.so")

ART_OK = 0
ART_ERR_INVALID_ARG = -1
ART_ERR_UNSUPPORTED = -2
ART_ERR_WORKSPACE = -3
ART_ERR_CUDA = -4
ART_ERR_TIMEOUT = -5
ART_ERR_SEQLEN = -6
ART_ERR_ORDER = -7
ART_ERR_PAGE = -8
ART_ERR_INDEX = -9  # debug build (-DART_DEBUG) only
ART_F32 = 0
ART_BF16 = 1
ART_KV_F32, ART_KV_BF16, ART_KV_Q8 = 0, 1, 2
ART_Q8_AUTO, ART_Q8_TENSOR_CORE, ART_Q8_TWO_PASS, ART_Q8_CLUSTER = 0, 1, 2, 3

# every symbol the header declares
EXPORTS = (
    "art_workspace_bytes",
    "art_q8_workspace_bytes",
    "art_workspace_tiles_read_offset",
    "art_workspace_split_tiles_offset",
    "art_workspace_vskip_offset",
    "art_decode_attn_full",
    "art_decode_attn_terminate",
    "art_decode_attn_terminate_noalloc",
    "art_decode_attn_q8_skipv",
    "art_decode_attn_q8_skipv_path",
    "art_read_device_status",
    "art_status_string",
    "art_kernel_name",
    "art_tile_order_recency",
    "art_tile_key_summary",
    "art_tile_order_importance",
    "art_decode_attn_terminate_ordered",
    "art_decode_attn_paged",
    "art_decode_attn_q8_skipv_paged",
    "art_evict_random_select",
    "art_evict_compact",
)


class art_shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "Hq", "Hkv", "d", "L_max", "tile", "num_splits")]


class art_params(ctypes.Structure):
    _fields_ = [
        ("eps_scale", ctypes.c_float),
        ("eps_dir", ctypes.c_float),
        ("patience", ctypes.c_int32),
        ("probe_lanes", ctypes.POINTER(ctypes.c_int32)),
        ("n_probe", ctypes.c_int32),
        ("max_spec_tiles", ctypes.c_int32),
    ]


class art_paged_kv(ctypes.Structure):
    _fields_ = [
        ("page_size", ctypes.c_int32),
        ("num_pages", ctypes.c_int32),
        ("max_pages_per_seq", ctypes.c_int32),
        ("block_table", ctypes.c_void_p),
    ]


class ArtError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {art_status_string(code)} ({code})")
        self.code = code


_lock = threading.Lock()
_lib = None

_P = ctypes.c_void_p
_SH = ctypes.POINTER(art_shape)
_PA = ctypes.POINTER(art_params)
_PG = ctypes.POINTER(art_paged_kv)


def lib() -> ctypes.CDLL:
    """Load libart_decode.so (built in-tree by kv_cache_early_split_b200.build)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise OSError(
                    f"{LIB_PATH} is missing: build it with `python -m kv_cache_early_split_b200.build` "
                    "(there is no fallback implementation)"
                )
            _lib = _bind(ctypes.CDLL(LIB_PATH))
    return _lib


def load_variant(path: str) -> ctypes.CDLL:
    """A separately built copy of the library (for instance the short-wait test build), with the
    same signatures bound; its symbols stay local to it."""
    return _bind(ctypes.CDLL(path))


def _bind(L: ctypes.CDLL) -> ctypes.CDLL:
    """Declare the C signatures on a loaded copy of the library."""
    L.art_workspace_bytes.restype = ctypes.c_size_t
    L.art_workspace_bytes.argtypes = [_SH]
    L.art_q8_workspace_bytes.restype = ctypes.c_size_t
    L.art_q8_workspace_bytes.argtypes = [_SH]
    L.art_workspace_tiles_read_offset.restype = ctypes.c_size_t
    L.art_workspace_tiles_read_offset.argtypes = [_SH]
    L.art_workspace_split_tiles_offset.restype = ctypes.c_size_t
    L.art_workspace_split_tiles_offset.argtypes = [_SH]
    L.art_workspace_vskip_offset.restype = ctypes.c_size_t
    L.art_workspace_vskip_offset.argtypes = [_SH]
    L.art_decode_attn_full.restype = ctypes.c_int
    L.art_decode_attn_full.argtypes = [_SH, ctypes.c_int, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
    L.art_decode_attn_terminate.restype = ctypes.c_int
    L.art_decode_attn_terminate.argtypes = [
        _SH, ctypes.c_int, _P, _P, _P, _P, _PA, _P, _P, _P, ctypes.c_size_t, _P]
    L.art_decode_attn_terminate_noalloc.restype = ctypes.c_int
    L.art_decode_attn_terminate_noalloc.argtypes = [
        _SH, ctypes.c_int, _P, _P, _P, _P, _PA, _P, _P, _P]
    L.art_decode_attn_q8_skipv.restype = ctypes.c_int
    L.art_decode_attn_q8_skipv.argtypes = [
        _SH, _P, _P, _P, _P, _P, _P, ctypes.c_float, _PA, _P, _P, _P, ctypes.c_size_t, _P]
    L.art_decode_attn_q8_skipv_path.restype = ctypes.c_int
    L.art_decode_attn_q8_skipv_path.argtypes = [
        _SH, _P, _P, _P, _P, _P, _P, ctypes.c_float, _PA, _P, _P, _P, ctypes.c_size_t, ctypes.c_int32, _P]
    L.art_read_device_status.restype = ctypes.c_int
    L.art_read_device_status.argtypes = [_P, _P]
    L.art_status_string.restype = ctypes.c_char_p
    L.art_status_string.argtypes = [ctypes.c_int]
    L.art_tile_order_recency.restype = ctypes.c_int
    L.art_tile_order_recency.argtypes = [_SH, _P, _P, _P]
    L.art_tile_key_summary.restype = ctypes.c_int
    L.art_tile_key_summary.argtypes = [_SH, ctypes.c_int, _P, _P, _P, _P]
    L.art_tile_order_importance.restype = ctypes.c_int
    L.art_tile_order_importance.argtypes = [_SH, ctypes.c_int, _P, _P, _P, _P, _P]
    L.art_decode_attn_terminate_ordered.restype = ctypes.c_int
    L.art_decode_attn_terminate_ordered.argtypes = [_SH, ctypes.c_int, _P, _P, _P, _P, _PA, _P, _P, _P, _P,
                                                    ctypes.c_size_t, _P]
    L.art_decode_attn_paged.restype = ctypes.c_int
    L.art_decode_attn_paged.argtypes = [_SH, ctypes.c_int, _P, _P, _P, _PG, _P, _PA, _P, _P, _P, _P,
                                        ctypes.c_size_t, _P]
    L.art_decode_attn_q8_skipv_paged.restype = ctypes.c_int
    L.art_decode_attn_q8_skipv_paged.argtypes = [_SH, _P, _P, _P, _P, _P, _PG, _P, ctypes.c_float, _PA, _P,
                                                 _P, _P, ctypes.c_size_t, _P]
    L.art_evict_random_select.restype = ctypes.c_int
    L.art_evict_random_select.argtypes = [_SH, _P, _P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, _P, _P,
                                          _P]
    L.art_evict_compact.restype = ctypes.c_int
    L.art_evict_compact.argtypes = [_SH, ctypes.c_int, _P, _P, _P, ctypes.c_int32, _P, _P, _P]
    L.art_kernel_name.restype = ctypes.c_char_p
    L.art_kernel_name.argtypes = [_SH, ctypes.c_int, ctypes.c_int32, ctypes.c_int32]
    return L


def _ref(x):
    return None if x is None else ctypes.byref(x)


def art_workspace_bytes(shape: art_shape) -> int:
    return int(lib().art_workspace_bytes(ctypes.byref(shape)))


def art_q8_workspace_bytes(shape: art_shape) -> int:
    return int(lib().art_q8_workspace_bytes(ctypes.byref(shape)))


def art_workspace_tiles_read_offset(shape: art_shape) -> int:
    return int(lib().art_workspace_tiles_read_offset(ctypes.byref(shape)))


def art_workspace_split_tiles_offset(shape: art_shape) -> int:
    return int(lib().art_workspace_split_tiles_offset(ctypes.byref(shape)))


def art_workspace_vskip_offset(shape: art_shape) -> int:
    return int(lib().art_workspace_vskip_offset(ctypes.byref(shape)))


def art_decode_attn_full(shape, dtype, q, k, v, seq_lens, o, tiles, ws, ws_bytes, stream) -> int:
    return int(lib().art_decode_attn_full(ctypes.byref(shape), dtype, q, k, v, seq_lens, o, tiles, ws, ws_bytes, stream))


def art_decode_attn_terminate(shape, dtype, q, k, v, seq_lens, params, o, tiles, ws, ws_bytes, stream) -> int:
    return int(lib().art_decode_attn_terminate(
        ctypes.byref(shape), dtype, q, k, v, seq_lens, _ref(params), o, tiles, ws, ws_bytes, stream))


def art_decode_attn_terminate_noalloc(shape, dtype, q, k, v, seq_lens, params, o, tiles, stream) -> int:
    """Allocation-free art_decode_attn_terminate (library-held 4 MiB device scratch; see the header)."""
    return int(lib().art_decode_attn_terminate_noalloc(
        ctypes.byref(shape), dtype, q, k, v, seq_lens, _ref(params), o, tiles, stream))


def art_decode_attn_q8_skipv(shape, q_bf16, k_q, k_scale_f16, v_q, v_scale_f16, seq_lens, tau, params, o, tiles,
                             ws, ws_bytes, stream) -> int:
    return int(lib().art_decode_attn_q8_skipv(
        ctypes.byref(shape), q_bf16, k_q, k_scale_f16, v_q, v_scale_f16, seq_lens, float(tau), _ref(params), o,
        tiles, ws, ws_bytes, stream))


def art_decode_attn_q8_skipv_path(shape, q_bf16, k_q, k_scale_f16, v_q, v_scale_f16, seq_lens, tau, params, o,
                                  tiles, ws, ws_bytes, path, stream) -> int:
    return int(lib().art_decode_attn_q8_skipv_path(
        ctypes.byref(shape), q_bf16, k_q, k_scale_f16, v_q, v_scale_f16, seq_lens, float(tau), _ref(params), o,
        tiles, ws, ws_bytes, int(path), stream))


def art_read_device_status(ws, stream) -> int:
    return int(lib().art_read_device_status(ws, stream))


def art_status_string(code: int) -> str:
    return lib().art_status_string(int(code)).decode()


def art_tile_order_recency(shape, seq_lens, tile_order, stream) -> int:
    return int(lib().art_tile_order_recency(ctypes.byref(shape), seq_lens, tile_order, stream))


def art_tile_key_summary(shape, dtype, k, seq_lens, summary, stream) -> int:
    return int(lib().art_tile_key_summary(ctypes.byref(shape), dtype, k, seq_lens, summary, stream))


def art_tile_order_importance(shape, dtype, q, summary, seq_lens, tile_order, stream) -> int:
    return int(lib().art_tile_order_importance(ctypes.byref(shape), dtype, q, summary, seq_lens, tile_order, stream))


def art_decode_attn_terminate_ordered(shape, dtype, q, k, v, seq_lens, params, tile_order, o, tiles, ws, ws_bytes,
                                      stream) -> int:
    return int(lib().art_decode_attn_terminate_ordered(
        ctypes.byref(shape), dtype, q, k, v, seq_lens, _ref(params), tile_order, o, tiles, ws, ws_bytes, stream))


def art_decode_attn_paged(shape, dtype, q, k_pages, v_pages, pages, seq_lens, params, tile_order, o, tiles, ws,
                          ws_bytes, stream) -> int:
    return int(lib().art_decode_attn_paged(
        ctypes.byref(shape), dtype, q, k_pages, v_pages, _ref(pages), seq_lens, _ref(params), tile_order, o, tiles,
        ws, ws_bytes, stream))


def art_decode_attn_q8_skipv_paged(shape, q_bf16, k_q_pages, k_scale_pages, v_q_pages, v_scale_pages, pages, seq_lens,
                                   tau, params, o, tiles, ws, ws_bytes, stream) -> int:
    return int(lib().art_decode_attn_q8_skipv_paged(
        ctypes.byref(shape), q_bf16, k_q_pages, k_scale_pages, v_q_pages, v_scale_pages, _ref(pages), seq_lens,
        float(tau), _ref(params), o, tiles, ws, ws_bytes, stream))


def art_evict_random_select(shape, seq_lens, rand_keys, n_sink, n_recent, budget, kept, kept_lens, stream) -> int:
    return int(lib().art_evict_random_select(ctypes.byref(shape), seq_lens, rand_keys, int(n_sink), int(n_recent),
                                             int(budget), kept, kept_lens, stream))


def art_evict_compact(shape, fmt, src, src_scale, kept, budget, dst, dst_scale, stream) -> int:
    return int(lib().art_evict_compact(ctypes.byref(shape), int(fmt), src, src_scale, kept, int(budget), dst,
                                       dst_scale, stream))


def art_kernel_name(shape, dtype, kv_q8, with_art):
    """Base name of the main kernel a call with this shape launches, or None if unsupported."""
    r = lib().art_kernel_name(ctypes.byref(shape), int(dtype), int(bool(kv_q8)), int(bool(with_art)))
    return None if r is None else r.decode()


def make_params(eps_scale: float, eps_dir: float, patience: int, lanes, max_spec_tiles: int = 0) -> art_params:
    """art_params with its own HOST copy of the lane list (kept alive on the object)."""
    arr = (ctypes.c_int32 * len(lanes))(*[int(x) for x in lanes])
    p = art_params(float(eps_scale), float(eps_dir), int(patience),
                   ctypes.cast(arr, ctypes.POINTER(ctypes.c_int32)), len(lanes), int(max_spec_tiles))
    p._lanes_keepalive = arr
    return p
