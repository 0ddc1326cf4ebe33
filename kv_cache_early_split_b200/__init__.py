"""B200 (sm_100a) single-token decode attention with ART (runtime attention
termination) and the q8 V-dequantisation skip.

The computation lives in CUDA kernels behind the C ABI of
``include/art_decode.h`` (``libart_decode.so``).  ``capi`` is the ctypes
binding with the C names; this module adds tensor-level helpers that only
allocate outputs / workspace with PyTorch and marshal pointers.
"""
from __future__ import annotations

from dataclasses import dataclass

from . import capi
from .capi import ArtError

__all__ = ["capi", "ArtError", "DeviceProblem", "upload", "decode", "kernel_name", "tile_order", "key_summary",
           "evict_random", "evict_random_into"]


@dataclass
class DeviceProblem:
    """A workload resident on the GPU (torch tensors), plus its output buffers."""

    kind: str
    shape: "capi.art_shape"
    q: object
    k: object
    v: object
    k_scale: object
    v_scale: object
    seq_lens: object
    o: object
    tiles: object
    ws: object
    art: dict
    tau: float
    pages: object = None  # paged cache: capi.art_paged_kv (k, v, scales are then page pools)
    block_table: object = None

    @property
    def ws_bytes(self) -> int:
        return int(self.ws.numel())

    def tiles_read(self):
        """int32 [B, Hkv, S]: KV tiles fetched by the last call (device tensor view)."""
        import torch

        off = capi.art_workspace_tiles_read_offset(self.shape)
        s = self.shape
        n = s.B * s.Hkv * s.num_splits
        return self.ws[off:off + 4 * n].view(torch.int32).view(s.B, s.Hkv, s.num_splits)


    def vskip_counts(self):
        """int32 [B, Hkv, S, 2]: V rows left out of every head's numerator and V tiles not read,
        by the last two-pass q8 call (device tensor view; needs the q8 workspace)."""
        import torch

        off = capi.art_workspace_vskip_offset(self.shape)
        s = self.shape
        n = s.B * s.Hkv * s.num_splits * 2
        return self.ws[off:off + 4 * n].view(torch.int32).view(s.B, s.Hkv, s.num_splits, 2)

    def split_tiles(self):
        """int32 [B, Hq, S]: KV tiles consumed per split by the last call (device tensor view)."""
        import torch

        off = capi.art_workspace_split_tiles_offset(self.shape)
        s = self.shape
        n = s.B * s.Hq * s.num_splits
        return self.ws[off:off + 4 * n].view(torch.int32).view(s.B, s.Hq, s.num_splits)


def _t(torch, arr, device, dtype=None):
    import numpy as np

    if arr is None:
        return None
    a = np.ascontiguousarray(arr)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    t = torch.from_numpy(a)
    if dtype is not None:
        t = t.to(dtype)
    return t.to(device)


def _ws_bytes(kind: str, shape, paged: bool, q8_two_pass: bool) -> int:
    """Workspace for a problem: the q8 two-pass arrays too for a contiguous q8 cache."""
    if kind == "q8" and not paged and q8_two_pass:
        return capi.art_q8_workspace_bytes(shape)
    return capi.art_workspace_bytes(shape)


def upload(w, device="cuda", num_splits=None, tile=None, paged=None, q8_two_pass=True):
    """Copy a kv_cache_early_split_b200.inputs.Workload to the GPU and allocate o / tiles / workspace.
    paged: None, or an inputs.PagedKV of the same workload: its page pools and block table are
    uploaded instead of the contiguous K/V.  q8_two_pass: for a contiguous q8 cache, size the
    workspace for the two-pass full-attention path (False: the one-pass cluster kernel)."""
    import torch

    S = w.num_splits if num_splits is None else int(num_splits)
    T = w.tile if tile is None else int(tile)
    shape = capi.art_shape(w.B, w.Hq, w.Hkv, w.d, w.L_max, T, S)
    wsb = _ws_bytes(w.kind, shape, paged is not None, q8_two_pass)
    if wsb == 0:
        raise ArtError(capi.ART_ERR_INVALID_ARG, "art_workspace_bytes")
    src = w if paged is None else paged
    bt = None
    pg = None
    if paged is not None:
        bt = _t(torch, paged.block_table, device, torch.int32)
        pg = capi.art_paged_kv(paged.page_size, paged.num_pages, paged.block_table.shape[1], bt.data_ptr())
    return DeviceProblem(
        kind=w.kind, shape=shape,
        q=_t(torch, w.q, device), k=_t(torch, src.k, device), v=_t(torch, src.v, device),
        k_scale=_t(torch, src.k_scale, device), v_scale=_t(torch, src.v_scale, device),
        pages=pg, block_table=bt,
        seq_lens=_t(torch, w.seq_lens, device, torch.int32),
        o=torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=device),
        tiles=torch.empty((w.B, w.Hq), dtype=torch.int32, device=device),
        ws=torch.zeros(wsb, dtype=torch.uint8, device=device),
        art=dict(w.art), tau=float(w.tau),
    )


def _ptr(t):
    return None if t is None else t.data_ptr()


Q8_PATHS = {"auto": capi.ART_Q8_AUTO, "tensor_core": capi.ART_Q8_TENSOR_CORE, "two_pass": capi.ART_Q8_TWO_PASS,
            "cluster": capi.ART_Q8_CLUSTER}


def decode(dp: DeviceProblem, mode: str, *, art: dict | None = None, tau: float | None = None, stream=None,
           check: bool = True, order=None, q8_path: str = "auto") -> int:
    """Launch one decode call on dp's buffers.

    mode: "full" | "art" (art_decode_attn_terminate) | "q8" (q8_skipv without ART) |
          "q8_art" (q8_skipv with ART).  order: None, or an int32 device tensor
    [B, Hkv, ceil(L_max/tile)] of tile traversal sequences (mode "art" only:
    art_decode_attn_terminate_ordered).  q8_path: for the q8 modes, "auto" (the library's choice)
    or one implementation, "tensor_core" / "two_pass" / "cluster"
    (art_decode_attn_q8_skipv_path).  Returns the C status code; raises ArtError on a non-zero
    code when check is True.
    """
    import torch

    if order is not None and mode != "art":
        raise ValueError("a traversal order applies to mode 'art' only")
    st = torch.cuda.current_stream().cuda_stream if stream is None else stream
    a = dp.art if art is None else art
    dtype = capi.ART_F32 if dp.kind == "f32" else capi.ART_BF16
    if dp.pages is not None:
        return _decode_paged(dp, mode, a, tau, st, check, order)
    if mode == "full":
        rc = capi.art_decode_attn_full(dp.shape, dtype, _ptr(dp.q), _ptr(dp.k), _ptr(dp.v), _ptr(dp.seq_lens),
                                       _ptr(dp.o), _ptr(dp.tiles), _ptr(dp.ws), dp.ws_bytes, st)
        name = "art_decode_attn_full"
    elif mode == "art" and order is not None:
        params = capi.make_params(a["eps_scale"], a["eps_dir"], a["patience"], a["lanes"], a.get("max_spec_tiles", 0))
        rc = capi.art_decode_attn_terminate_ordered(
            dp.shape, dtype, _ptr(dp.q), _ptr(dp.k), _ptr(dp.v), _ptr(dp.seq_lens), params, _ptr(order),
            _ptr(dp.o), _ptr(dp.tiles), _ptr(dp.ws), dp.ws_bytes, st)
        name = "art_decode_attn_terminate_ordered"
    elif mode == "art":
        params = capi.make_params(a["eps_scale"], a["eps_dir"], a["patience"], a["lanes"], a.get("max_spec_tiles", 0))
        rc = capi.art_decode_attn_terminate(dp.shape, dtype, _ptr(dp.q), _ptr(dp.k), _ptr(dp.v), _ptr(dp.seq_lens),
                                            params, _ptr(dp.o), _ptr(dp.tiles), _ptr(dp.ws), dp.ws_bytes, st)
        name = "art_decode_attn_terminate"
    elif mode in ("q8", "q8_art"):
        params = None
        if mode == "q8_art":
            params = capi.make_params(a["eps_scale"], a["eps_dir"], a["patience"], a["lanes"], a.get("max_spec_tiles", 0))
        rc = capi.art_decode_attn_q8_skipv_path(
            dp.shape, _ptr(dp.q), _ptr(dp.k), _ptr(dp.k_scale), _ptr(dp.v), _ptr(dp.v_scale), _ptr(dp.seq_lens),
            dp.tau if tau is None else tau, params, _ptr(dp.o), _ptr(dp.tiles), _ptr(dp.ws), dp.ws_bytes,
            Q8_PATHS[q8_path], st)
        name = "art_decode_attn_q8_skipv_path"
    else:
        raise ValueError(mode)
    if check and rc != capi.ART_OK:
        raise ArtError(rc, name)
    return rc


def _decode_paged(dp, mode, a, tau, st, check, order):
    params = None
    if mode in ("art", "q8_art"):
        params = capi.make_params(a["eps_scale"], a["eps_dir"], a["patience"], a["lanes"], a.get("max_spec_tiles", 0))
    if mode in ("full", "art"):
        dtype = capi.ART_F32 if dp.kind == "f32" else capi.ART_BF16
        rc = capi.art_decode_attn_paged(dp.shape, dtype, _ptr(dp.q), _ptr(dp.k), _ptr(dp.v), dp.pages,
                                        _ptr(dp.seq_lens), params, _ptr(order), _ptr(dp.o), _ptr(dp.tiles),
                                        _ptr(dp.ws), dp.ws_bytes, st)
        name = "art_decode_attn_paged"
    elif mode in ("q8", "q8_art"):
        rc = capi.art_decode_attn_q8_skipv_paged(
            dp.shape, _ptr(dp.q), _ptr(dp.k), _ptr(dp.k_scale), _ptr(dp.v), _ptr(dp.v_scale), dp.pages,
            _ptr(dp.seq_lens), dp.tau if tau is None else tau, params, _ptr(dp.o), _ptr(dp.tiles), _ptr(dp.ws),
            dp.ws_bytes, st)
        name = "art_decode_attn_q8_skipv_paged"
    else:
        raise ValueError(mode)
    if check and rc != capi.ART_OK:
        raise ArtError(rc, name)
    return rc


def tile_order(dp: DeviceProblem, kind: str, *, stream=None, summary=None):
    """Build tile traversal sequences on the GPU: kind "recency" or "importance" (the latter from dp's
    query and a per-tile key summary, computed here unless given).  Returns int32 [B, Hkv, n_max]."""
    import torch

    s = dp.shape
    st = torch.cuda.current_stream().cuda_stream if stream is None else stream
    n_max = -(-s.L_max // s.tile)
    out = torch.empty((s.B, s.Hkv, n_max), dtype=torch.int32, device=dp.k.device)
    if kind == "recency":
        rc = capi.art_tile_order_recency(s, _ptr(dp.seq_lens), _ptr(out), st)
        name = "art_tile_order_recency"
    elif kind == "importance":
        if dp.kind not in ("f32", "bf16"):
            raise ValueError("importance order needs fp32 or bf16 keys")
        dtype = capi.ART_F32 if dp.kind == "f32" else capi.ART_BF16
        if summary is None:
            summary = key_summary(dp, stream=st)
        rc = capi.art_tile_order_importance(s, dtype, _ptr(dp.q), _ptr(summary), _ptr(dp.seq_lens), _ptr(out), st)
        name = "art_tile_order_importance"
    else:
        raise ValueError(kind)
    if rc != capi.ART_OK:
        raise ArtError(rc, name)
    return out


def evict_random(dp: DeviceProblem, rand_keys, n_sink: int, n_recent: int, budget: int, *, stream=None):
    """Random eviction on the GPU (art_evict_random_select + art_evict_compact): returns (the
    DeviceProblem of the packed cache, L_max = budget, seq_lens = kept lengths; kept positions
    int32 [B, Hkv, budget]).  rand_keys: device tensor of 32-bit keys [B, Hkv, L_max] (int32 or
    uint32 bits)."""
    import torch

    if dp.pages is not None:
        raise ValueError("eviction packs a contiguous cache")
    s = dp.shape
    dev = dp.k.device
    shape2 = capi.art_shape(s.B, s.Hq, s.Hkv, s.d, budget, s.tile, s.num_splits)

    def like(x, rows_last):
        return None if x is None else torch.empty((s.B, s.Hkv, budget, rows_last), dtype=x.dtype, device=dev)

    dp2 = DeviceProblem(
        kind=dp.kind, shape=shape2, q=dp.q, k=like(dp.k, s.d), v=like(dp.v, s.d),
        k_scale=like(dp.k_scale, s.d // 32), v_scale=like(dp.v_scale, s.d // 32),
        seq_lens=torch.empty((s.B,), dtype=torch.int32, device=dev), o=torch.empty_like(dp.o),
        tiles=torch.empty_like(dp.tiles),
        ws=torch.zeros(_ws_bytes(dp.kind, shape2, False, dp.ws_bytes > capi.art_workspace_bytes(s)),
                       dtype=torch.uint8, device=dev),
        art=dict(dp.art), tau=dp.tau)
    kept = torch.empty((s.B, s.Hkv, budget), dtype=torch.int32, device=dev)
    evict_random_into(dp, dp2, kept, rand_keys, n_sink, n_recent, stream=stream)
    return dp2, kept


def evict_random_into(dp: DeviceProblem, dp2: DeviceProblem, kept, rand_keys, n_sink: int, n_recent: int, *,
                      stream=None) -> None:
    """evict_random into the buffers of an existing packed problem (no allocation): kept positions
    into `kept`, kept lengths into dp2.seq_lens, packed rows into dp2.k / dp2.v (and scales)."""
    import torch

    s = dp.shape
    budget = dp2.shape.L_max
    st = torch.cuda.current_stream().cuda_stream if stream is None else stream
    rc = capi.art_evict_random_select(s, _ptr(dp.seq_lens), _ptr(rand_keys), n_sink, n_recent, budget, _ptr(kept),
                                      _ptr(dp2.seq_lens), st)
    if rc != capi.ART_OK:
        raise ArtError(rc, "art_evict_random_select")
    fmt = {"f32": capi.ART_KV_F32, "bf16": capi.ART_KV_BF16, "q8": capi.ART_KV_Q8}[dp.kind]
    for name in ("k", "v"):
        rc = capi.art_evict_compact(s, fmt, _ptr(getattr(dp, name)), _ptr(getattr(dp, name + "_scale")), _ptr(kept),
                                    budget, _ptr(getattr(dp2, name)), _ptr(getattr(dp2, name + "_scale")), st)
        if rc != capi.ART_OK:
            raise ArtError(rc, "art_evict_compact")


def key_summary(dp: DeviceProblem, *, stream=None):
    """Mean key per tile, fp32 [B, Hkv, n_max, d] (art_tile_key_summary; contiguous K only)."""
    import torch

    if dp.pages is not None:
        raise ValueError("the key summary reads a contiguous cache")

    s = dp.shape
    st = torch.cuda.current_stream().cuda_stream if stream is None else stream
    n_max = -(-s.L_max // s.tile)
    out = torch.empty((s.B, s.Hkv, n_max, s.d), dtype=torch.float32, device=dp.k.device)
    dtype = capi.ART_F32 if dp.kind == "f32" else capi.ART_BF16
    rc = capi.art_tile_key_summary(s, dtype, _ptr(dp.k), _ptr(dp.seq_lens), _ptr(out), st)
    if rc != capi.ART_OK:
        raise ArtError(rc, "art_tile_key_summary")
    return out


def kernel_name(dp: DeviceProblem, mode: str) -> str:
    """Base name of the main CUDA kernel decode(dp, mode) launches (art_kernel_name)."""
    dtype = capi.ART_F32 if dp.kind == "f32" else capi.ART_BF16
    name = capi.art_kernel_name(dp.shape, dtype, mode.startswith("q8"), mode in ("art", "q8_art"))
    if name is None:
        raise ArtError(capi.ART_ERR_UNSUPPORTED, "art_kernel_name")
    if dp.pages is not None and dp.pages.page_size % 64 and name == "art_decode_tc_kernel":
        name = "art_decode_kernel"  # the tensor-core path takes pages of a multiple of 64 positions
    return name


def device_status(dp: DeviceProblem, stream=None) -> int:
    """Synchronise and return (and clear) the sticky device status of dp's workspace."""
    import torch

    st = torch.cuda.current_stream().cuda_stream if stream is None else stream
    return capi.art_read_device_status(_ptr(dp.ws), st)
