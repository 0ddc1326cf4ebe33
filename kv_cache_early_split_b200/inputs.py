"""Seeded synthetic inputs for decode attention (numpy only).

This module is shared by the tests, the benchmark and the oracle harness.  It
holds no step of the attention method itself: it draws random tensors, rounds
them to their storage formats (bf16, fp16, q8 blocks) and builds the five
synthetic workloads, nothing more.  It imports neither the CUDA binding nor the
oracle.

Every tensor slab is drawn from its own ``numpy.random.default_rng`` stream,
keyed by (seed, tensor id, batch, kv head), so a slab is identical whether the
whole workload or a single (batch, kv head) slice is generated.

Workload recipes (shapes from the long-context decode settings the pages
discuss, 32K-128K positions; the pages' own benchmark suites are not used):
  fp32_b1_h1_d64_L4k        fp32, B=1, Hq=Hkv=1, d=64, L=4096, tile 64, N(0,1)
  gqa_b4_h32x8_d128_L32k    bf16, B=4, Hq=32, Hkv=8, d=128, L=32768, tile 64,
                            N(0,1); key 0 of each group moved 8 units along the
                            group's mean query direction (attention sink)
  gqa_b1_h32x8_d128_L128k   bf16, B=1, Hq=32, Hkv=8, d=128, L=131072, tile 128;
                            keys shifted along the mean query direction by
                            Gumbel(0, 2) offsets; V rows = unit directions times
                            LogNormal(0, 1) norms
  split_b16_h32x8_d128_Lvar bf16, B=16, Hq=32, Hkv=8, d=128, L_b ~ U{8192..65536},
                            L_max=65536, tile 64, 8 KV splits, N(0,1)
  q8_b2_h32x8_d128_L32k     q8 K/V (32-element blocks, fp16 scale), bf16 Q,
                            B=2, Hq=32, Hkv=8, d=128, L=32768, tile 64, N(0,1)
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

# tensor ids for the per-slab random streams
_T_Q, _T_K, _T_V, _T_LEN, _T_GUMBEL, _T_VNORM = 1, 2, 3, 4, 6, 7


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest even; NaN kept quiet."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    out = rounded.astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float32 (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> IEEE fp16 bit patterns (numpy's round to nearest even)."""
    return np.asarray(x, dtype=np.float32).astype(np.float16).view(np.uint16)


def quantize_q8(x: np.ndarray, block: int = 32):
    """q8_0-style blocks along the last axis.

    scale = amax/127 rounded to fp16; q = round-half-even(x/scale) clamped to
    [-127, 127] (0 where the block is all zeros).  Returns (int8 codes, uint16
    fp16-scale bits with shape [..., d/block]).
    """
    x = np.asarray(x, dtype=np.float32)
    d = x.shape[-1]
    assert d % block == 0
    xb = x.reshape(*x.shape[:-1], d // block, block)
    amax = np.abs(xb).max(axis=-1)
    scale_h = (amax / np.float32(127.0)).astype(np.float16)
    s = scale_h.astype(np.float32)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        qf = np.where(s > 0, np.rint(xb / np.where(s > 0, s, 1)), 0)
    qi = np.clip(qf, -127, 127).astype(np.int8).reshape(x.shape)
    return qi, scale_h.view(np.uint16)


def _rng(seed: int, tensor: int, *idx: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(tensor), *[int(i) for i in idx]])


@dataclass
class Workload:
    """A decode-attention problem in its storage formats.

    kind: "f32" | "bf16" | "q8".  q is float32 (f32) or bf16 bits (bf16, q8).
    k, v: float32 / bf16 bits (uint16) / int8 codes, [B, Hkv, L_max, d].
    k_scale, v_scale: fp16 bits [B, Hkv, L_max, d/32] for q8, else None.
    art: dict(eps_scale, eps_dir, patience, lanes) -- ART settings of the workload.
    """

    name: str
    kind: str
    B: int
    Hq: int
    Hkv: int
    d: int
    L_max: int
    tile: int
    num_splits: int
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    seq_lens: np.ndarray
    art: dict
    tau: float = 0.0
    k_scale: np.ndarray | None = None
    v_scale: np.ndarray | None = None
    meta: dict = field(default_factory=dict)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def kv_bytes_full(self) -> int:
        """Bytes of K and V inside the sequence lengths (what full attention reads)."""
        row = self.d * {"f32": 4, "bf16": 2, "q8": 1}[self.kind]
        if self.kind == "q8":
            row += 2 * (self.d // 32)
        return int(2 * row * self.Hkv * int(np.sum(self.seq_lens)))


def probe_lanes_strided(d: int, n: int) -> list[int]:
    """n lanes evenly spaced over [0, d): 0, d/n, 2d/n, ..."""
    return [i * (d // n) for i in range(n)]


def _normal_slab(seed, tensor, b, h, rows, d):
    return _rng(seed, tensor, b, h).standard_normal((rows, d), dtype=np.float32)


def make_workload(
    *,
    name: str = "custom",
    kind: str = "bf16",
    B: int = 1,
    Hq: int = 4,
    Hkv: int = 1,
    d: int = 128,
    L_max: int = 1024,
    tile: int = 64,
    num_splits: int = 1,
    seq_lens=None,
    seed: int = 0,
    sink: float = 0.0,
    gumbel_scale: float = 0.0,
    lognormal_v: bool = False,
    q_scale: float = 1.0,
    art: dict | None = None,
    tau: float = 0.0,
    keys_b=None,
    keys_h=None,
) -> Workload:
    """General seeded generator.

    seq_lens: None (all L_max), an int array [B], or ("uniform", lo, hi).
    sink: move key 0 of each (b, kv head) `sink` units along the unit mean of
          the group's queries.
    gumbel_scale: > 0 shifts every key along that direction by Gumbel(0, scale).
    lognormal_v: V rows = uniform random unit directions times LogNormal(0, 1).
    keys_b, keys_h: stream keys of the batches / kv heads to build (default
           range(B), range(Hkv)).  A sub-list builds exactly those slabs of the
           full problem, so a test can take one (batch, kv head) slice of a
           large workload without generating the rest.  B and Hkv are the full
           problem's sizes; Hq is scaled to the kept kv heads.
    """
    G = Hq // Hkv
    assert Hq % Hkv == 0
    kb = list(range(B)) if keys_b is None else [int(x) for x in keys_b]
    kh = list(range(Hkv)) if keys_h is None else [int(x) for x in keys_h]
    if seq_lens is None:
        lens_full = np.full(B, L_max, np.int32)
    elif isinstance(seq_lens, tuple) and seq_lens[0] == "uniform":
        lens_full = _rng(seed, _T_LEN, 0, 0).integers(seq_lens[1], seq_lens[2] + 1, size=B).astype(np.int32)
    else:
        lens_full = np.asarray(seq_lens, dtype=np.int32).reshape(B)
    lens = lens_full[kb].copy()
    B, Hkv = len(kb), len(kh)
    Hq = Hkv * G
    # Queries: one stream per (b, kv head) group.
    qf = np.zeros((B, Hq, d), np.float32)
    for bi, b in enumerate(kb):
        for hi, h in enumerate(kh):
            qf[bi, hi * G:(hi + 1) * G] = _normal_slab(seed, _T_Q, b, h, G, d) * np.float32(q_scale)
    if kind == "f32":
        q = qf
        q_used = qf
    else:
        q = bf16_bits(qf)
        q_used = bf16_to_f32(q)
    if kind not in ("f32", "bf16", "q8"):
        raise ValueError(kind)
    store = {"f32": np.float32, "bf16": np.uint16, "q8": np.int8}[kind]
    k = np.zeros((B, Hkv, L_max, d), store)
    v = np.zeros((B, Hkv, L_max, d), store)
    k_scale = v_scale = None
    if kind == "q8":
        k_scale = np.zeros((B, Hkv, L_max, d // 32), np.uint16)
        v_scale = np.zeros((B, Hkv, L_max, d // 32), np.uint16)
    def build_slab(bi, b, hi, h):
        kf = _normal_slab(seed, _T_K, b, h, L_max, d)
        if lognormal_v:
            vf = _normal_slab(seed, _T_V, b, h, L_max, d)
            vf /= np.linalg.norm(vf, axis=1, keepdims=True)
            vf *= _rng(seed, _T_VNORM, b, h).lognormal(0.0, 1.0, size=(L_max, 1)).astype(np.float32)
        else:
            vf = _normal_slab(seed, _T_V, b, h, L_max, d)
        if sink or gumbel_scale:
            mean_q = q_used[bi, hi * G:(hi + 1) * G].mean(axis=0)
            nrm = float(np.linalg.norm(mean_q))
            u = mean_q / nrm if nrm > 0 else np.zeros(d, np.float32)
            if gumbel_scale:
                g = _rng(seed, _T_GUMBEL, b, h).gumbel(0.0, gumbel_scale, size=(L_max, 1)).astype(np.float32)
                kf += g * u[None, :]
            if sink:
                kf[0] += np.float32(sink) * u
        # storage format of this slab
        if kind == "f32":
            k[bi, hi], v[bi, hi] = kf, vf
        elif kind == "bf16":
            k[bi, hi], v[bi, hi] = bf16_bits(kf), bf16_bits(vf)
        else:
            k[bi, hi], k_scale[bi, hi] = quantize_q8(kf)
            v[bi, hi], v_scale[bi, hi] = quantize_q8(vf)

    # Every slab has its own random stream and its own output rows, so the slabs are built in
    # parallel threads (numpy's generators and array kernels release the GIL); the result is the
    # same as building them one after another.
    slabs = [(bi, b, hi, h) for bi, b in enumerate(kb) for hi, h in enumerate(kh)]
    if len(slabs) > 1 and L_max * d >= (1 << 16):
        with ThreadPoolExecutor(max_workers=min(len(slabs), os.cpu_count() or 1)) as ex:
            list(ex.map(lambda a: build_slab(*a), slabs))
    else:
        for a in slabs:
            build_slab(*a)
    if art is None:
        art = dict(eps_scale=1e-3, eps_dir=1e-4, patience=1, lanes=probe_lanes_strided(d, 16 if d >= 128 else 8))
    return Workload(
        name=name, kind=kind, B=B, Hq=Hq, Hkv=Hkv, d=d, L_max=L_max, tile=tile, num_splits=num_splits,
        q=q, k=k, v=v, seq_lens=lens, art=art, tau=tau, k_scale=k_scale, v_scale=v_scale,
        meta=dict(seed=seed, sink=sink, gumbel_scale=gumbel_scale, lognormal_v=lognormal_v, keys_b=kb, keys_h=kh),
    )


ART_C2 = dict(eps_scale=1e-3, eps_dir=1e-4, patience=1, lanes=list(range(0, 128, 8)))

WORKLOADS = (
    "fp32_b1_h1_d64_L4k",
    "gqa_b4_h32x8_d128_L32k",
    "gqa_b1_h32x8_d128_L128k",
    "split_b16_h32x8_d128_Lvar",
    "q8_b2_h32x8_d128_L32k",
)


# Variants used by the benchmark's sweeps (not among the five workloads):
#   q8_b2_h32x8_d128_L32k_skewed  the q8 workload's shape with skewed logits: attention sink
#                                 (key 0 moved 8 units along the group's mean query), keys shifted
#                                 along that direction by Gumbel(0, 2), V rows = unit directions
#                                 times LogNormal(0, 1) norms -- so that many softmax weights fall
#                                 below the V-skip threshold.
VARIANTS = ("q8_b2_h32x8_d128_L32k_skewed",)


def workload(name: str, *, keys_b=None, keys_h=None) -> Workload:
    """The five named synthetic workloads (seed 20260000 + index), or a variant of VARIANTS.

    keys_b / keys_h select a slice (batches, kv heads) of the same problem; the
    selected slabs are bit-identical to those of the full workload.
    """
    if name == VARIANTS[0]:
        return make_workload(
            name=name, kind="q8", B=2, Hq=32, Hkv=8, d=128, L_max=32768, tile=64, tau=1e-6, sink=8.0,
            gumbel_scale=2.0, lognormal_v=True, art=dict(ART_C2), seed=20260104, keys_b=keys_b, keys_h=keys_h,
        )
    i = WORKLOADS.index(name)
    seed = 20260000 + i
    kw = dict(name=name, seed=seed, keys_b=keys_b, keys_h=keys_h)
    if i == 0:
        return make_workload(
            kind="f32", B=1, Hq=1, Hkv=1, d=64, L_max=4096, tile=64,
            art=dict(eps_scale=1e-3, eps_dir=1e-4, patience=1, lanes=list(range(8))), **kw,
        )
    if i == 1:
        return make_workload(
            kind="bf16", B=4, Hq=32, Hkv=8, d=128, L_max=32768, tile=64, sink=8.0, art=dict(ART_C2), **kw,
        )
    if i == 2:
        return make_workload(
            kind="bf16", B=1, Hq=32, Hkv=8, d=128, L_max=131072, tile=128, gumbel_scale=2.0, lognormal_v=True,
            art=dict(ART_C2), **kw,
        )
    if i == 3:
        return make_workload(
            kind="bf16", B=16, Hq=32, Hkv=8, d=128, L_max=65536, tile=64, num_splits=8,
            seq_lens=("uniform", 8192, 65536), art=dict(ART_C2), **kw,
        )
    if i == 4:
        return make_workload(
            kind="q8", B=2, Hq=32, Hkv=8, d=128, L_max=32768, tile=64, tau=1e-6, art=dict(ART_C2), **kw,
        )
    raise ValueError(name)


# ----------------------------------------------------------------------------- paged layout
@dataclass
class PagedKV:
    """A workload's K/V (and q8 scales) scattered into a page pool [num_pages, Hkv, page_size, ...].

    block_table[b, i] is the page holding positions [i*page_size, (i+1)*page_size) of sequence b;
    entries past the sequence are -1.  Pages that no sequence uses hold NaN (fp16 NaN scales for q8),
    so a read of a wrong page shows up in the output."""

    page_size: int
    num_pages: int
    block_table: np.ndarray  # int32 [B, max_pages]
    k: np.ndarray
    v: np.ndarray
    k_scale: np.ndarray | None
    v_scale: np.ndarray | None


def paginate(w: Workload, page_size: int, seed: int = 0, spare_pages: int = 3) -> PagedKV:
    B, Hkv, L_max = w.B, w.Hkv, w.L_max
    max_pages = -(-L_max // page_size)
    need = [-(-int(L) // page_size) for L in w.seq_lens]
    num_pages = sum(need) + spare_pages
    perm = np.random.default_rng(seed).permutation(num_pages).astype(np.int32)
    table = np.full((B, max_pages), -1, np.int32)
    nxt = 0
    for b in range(B):
        table[b, :need[b]] = perm[nxt:nxt + need[b]]
        nxt += need[b]

    def scatter(x, fill):
        if x is None:
            return None
        tail = x.shape[3:]
        pool = np.empty((num_pages, Hkv, page_size) + tail, dtype=x.dtype)
        pool[...] = fill
        for b in range(B):
            for i in range(need[b]):
                j0 = i * page_size
                j1 = min(j0 + page_size, L_max)
                pool[table[b, i], :, :j1 - j0] = x[b, :, j0:j1]
        return pool

    nan = {np.dtype(np.float32): np.float32(np.nan), np.dtype(np.uint16): np.uint16(0x7FC0),
           np.dtype(np.int8): np.int8(0)}[w.k.dtype]
    return PagedKV(page_size=page_size, num_pages=num_pages, block_table=table,
                   k=scatter(w.k, nan), v=scatter(w.v, nan),
                   k_scale=scatter(w.k_scale, np.uint16(0x7E00)), v_scale=scatter(w.v_scale, np.uint16(0x7E00)))
