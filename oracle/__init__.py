"""CPU oracle for ART decode attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it, and it
imports nothing from the CUDA side: the two share only the seeded input
generators (``kv_cache_early_split_b200.inputs``), which hold none of the
method's arithmetic.

The arithmetic lives in ``art_oracle.c`` (plain C, double precision); this
module compiles it on demand with gcc and marshals numpy arrays into it.

Sources (web pages, cited by title and section):
  "Resumen Tecnico: ART (Terminacion de la Atencion en Tiempo de Ejecucion)"
  (gist.science, arXiv 2606.00024), S2.1-S2.4 -- tile-wise attention, the
  probe, d_scale / d_direction, the conjunctive thresholds, patience and the
  mandatory block 0.
  "La paradoja de la eficiencia: como omitir redefine la velocidad de los LLM"
  (puntofijo.es), "La Elegancia de la Omision" -- skipping V dequantisation
  where the softmax weight is negligible.

Pins: every function here is pinned by ``tests/test_oracle_pins.py`` against
brute-force softmax attention in extended precision, closed forms, invariants
and a hand-worked two-tile probe example (``tests/golden/``).  The ART stop
tiles on the large synthetic workloads have no value printed on the pages:
parity unpinned there beyond the rule itself and those invariants.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "art_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libart_oracle.so")

KV_F32, KV_BF16, KV_Q8 = 0, 1, 2
_lock = threading.Lock()
_lib = None


class _Shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("B", "Hq", "Hkv", "d", "L_max", "tile", "num_splits")]


class _Art(ctypes.Structure):
    _fields_ = [
        ("enabled", ctypes.c_int),
        ("eps_scale", ctypes.c_double),
        ("eps_dir", ctypes.c_double),
        ("patience", ctypes.c_int),
        ("lanes", ctypes.POINTER(ctypes.c_int32)),
        ("n_probe", ctypes.c_int),
    ]


def build(force: bool = False) -> str:
    """Compile art_oracle.c into libart_oracle.so (plain -O2, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-std=c11", "-O2", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.oracle_decode.restype = ctypes.c_int
            lib.oracle_decode.argtypes = [
                ctypes.POINTER(_Shape), ctypes.c_int,
                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                ctypes.POINTER(_Art), ctypes.c_double, ctypes.c_void_p, ctypes.c_int,
                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
            ]
            lib.oracle_decode_ordered.restype = ctypes.c_int
            lib.oracle_decode_ordered.argtypes = lib.oracle_decode.argtypes[:12] + [ctypes.c_void_p] + \
                lib.oracle_decode.argtypes[12:]
            lib.oracle_decode_vskip.restype = ctypes.c_int
            lib.oracle_decode_vskip.argtypes = lib.oracle_decode_ordered.argtypes + [ctypes.c_void_p]
            lib.oracle_bf16_to_double.restype = ctypes.c_double
            lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
            lib.oracle_f16_to_double.restype = ctypes.c_double
            lib.oracle_f16_to_double.argtypes = [ctypes.c_uint16]
            _lib = lib
    return _lib


def bf16_to_double(bits: int) -> float:
    return _load().oracle_bf16_to_double(int(bits))


def f16_to_double(bits: int) -> float:
    return _load().oracle_f16_to_double(int(bits))


def _ptr(a):
    return None if a is None else a.ctypes.data


class OracleResult:
    """o [B,Hq,d] float64; tiles [B,Hq]; used [B,Hq,S]; metrics [B,Hq,n,2] or None;
    vskip [B,Hq,L_max] or None: p / tau of every row weighed with the V skip on (NaN elsewhere)."""

    def __init__(self, o, tiles, used, metrics, vskip=None):
        self.o, self.tiles, self.used, self.metrics, self.vskip = o, tiles, used, metrics, vskip


def decode(
    *,
    kind: int,
    q: np.ndarray,
    k: np.ndarray,
    v: np.ndarray,
    seq_lens: np.ndarray,
    tile: int,
    num_splits: int = 1,
    k_scale: np.ndarray | None = None,
    v_scale: np.ndarray | None = None,
    art: dict | None = None,
    tau: float = 0.0,
    forced_used: np.ndarray | None = None,
    no_break: bool = False,
    want_metrics: bool = False,
    n_threads: int = 1,
    tile_order: np.ndarray | None = None,
    want_vskip: bool = False,
) -> OracleResult:
    """Run the oracle.

    q: float32 [B,Hq,d] (KV_F32) or uint16 bf16 bits [B,Hq,d].
    k, v: float32 / uint16 bf16 bits / int8, [B,Hkv,L_max,d].
    k_scale, v_scale: uint16 fp16 bits [B,Hkv,L_max,d/32] (KV_Q8 only).
    art: None for plain attention, else dict(eps_scale, eps_dir, patience, lanes).
    tile_order: None (natural order) or int32 [B,Hkv,ceil(L_max/tile)]: each (batch, kv head)'s
      traversal sequence; split s walks positions [s*n/S, (s+1)*n/S) of it (see orders.py).
    want_vskip: also return, for the q8 V skip (tau > 0), p / tau of every row each head weighed
      (the row left that head's numerator iff the value is below 1).
    """
    lib = _load()
    B, Hq, d = q.shape
    _, Hkv, L_max, d2 = k.shape
    assert d2 == d and v.shape == k.shape
    dt = {KV_F32: np.float32, KV_BF16: np.uint16, KV_Q8: np.int8}[kind]
    qdt = np.float32 if kind == KV_F32 else np.uint16
    q = np.ascontiguousarray(q, dtype=qdt)
    k = np.ascontiguousarray(k, dtype=dt)
    v = np.ascontiguousarray(v, dtype=dt)
    if kind == KV_Q8:
        k_scale = np.ascontiguousarray(k_scale, dtype=np.uint16)
        v_scale = np.ascontiguousarray(v_scale, dtype=np.uint16)
    seq = np.ascontiguousarray(seq_lens, dtype=np.int32)
    sh = _Shape(B, Hq, Hkv, d, L_max, tile, num_splits)
    art_s = None
    lanes = None
    if art is not None:
        lanes = np.ascontiguousarray(art["lanes"], dtype=np.int32)
        art_s = _Art(
            1, float(art["eps_scale"]), float(art["eps_dir"]), int(art["patience"]),
            lanes.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), len(lanes),
        )
    fu = None if forced_used is None else np.ascontiguousarray(forced_used, dtype=np.int32)
    o = np.zeros((B, Hq, d), np.float64)
    used = np.zeros((B, Hq, num_splits), np.int32)
    tiles = np.zeros((B, Hq), np.int32)
    n_tiles_max = (L_max + tile - 1) // tile
    metrics = np.zeros((B, Hq, n_tiles_max, 2), np.float64) if want_metrics else None
    order = None
    if tile_order is not None:
        order = np.ascontiguousarray(tile_order, dtype=np.int32)
        assert order.shape == (B, Hkv, n_tiles_max), order.shape
    vskip = np.zeros((B, Hq, L_max), np.float64) if want_vskip else None
    rc = lib.oracle_decode_vskip(
        ctypes.byref(sh), kind, _ptr(q), _ptr(k), _ptr(v), _ptr(k_scale), _ptr(v_scale), _ptr(seq),
        ctypes.byref(art_s) if art_s is not None else None, float(tau), _ptr(fu), int(no_break), _ptr(order),
        _ptr(o), _ptr(used), _ptr(tiles), _ptr(metrics), int(n_threads), _ptr(vskip),
    )
    if rc != 0:
        raise ValueError(f"oracle_decode failed with code {rc}")
    return OracleResult(o, tiles, used, metrics, vskip)
