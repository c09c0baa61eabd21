"""Seeded synthetic inputs for varlen GQA decode / short-query attention.

This module is shared by the tests, the benchmark and the smoke check.  It
holds none of the attention arithmetic: it draws sequence lengths, builds the
cumulative-offset arrays (cu_seqlens) and draws iid N(0, 1) values rounded to
bf16.  Both the CUDA path and the fp64 oracle receive the same bytes from here.

Workloads (sizes, length laws and the readings behind them are recorded in the
design notes):

  tiny        B=2, q_len=1, Hq=4, Hkv=1, D=64, kv lengths {37, 100}, s_max=128
  long        B=1, q_len=1, Hq=64, Hkv=8, D=128, kv length 32768
  ragged      B=64, q_len=1, Hq=32, Hkv=8, D=128, kv ~ U{0..8192}, s_max=8192
  continuous  B=256, q_len=1, Hq=64, Hkv=8, D=128, s_max=16384, 100 steps,
              kv ~ round(lognormal(mean 2048, sigma 1)) clamped to [1, 16384]
  shortq      B=32, q_len ~ U{1..16}, Hq=32, Hkv=4, D=128, kv ~ U{q_len..4096},
              tail-aligned causal mask
  prefill     B=4, q_len = kv ~ U{512..2048}, Hq=32, Hkv=4, D=128, causal (queries
              longer than one 128-row tile; not one of the method's five
              workloads)

Random streams: lengths come from ``numpy.random.default_rng(seed)`` (PCG64),
one stream per workload, drawn in step order.  Values come from a
``torch.Generator`` seeded with ``seed`` on the device named by ``gen_device``,
drawing q, then k, then v; the byte stream depends on that device (CPU:
Mersenne Twister, CUDA: Philox), so a check always hands the same tensors to
both sides instead of regenerating them.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

# lognormal with arithmetic mean 2048 and sigma 1: mu = ln(2048) - sigma^2 / 2
LOGNORMAL_MEAN = 2048.0
LOGNORMAL_SIGMA = 1.0


@dataclasses.dataclass
class Shape:
    name: str
    B: int          # B_max: sequences the plan is sized for (cu arrays hold B+1 entries)
    Hq: int
    Hkv: int
    D: int
    max_q: int      # largest query length per sequence
    s_max: int      # largest key length per sequence
    causal: bool = True

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv


SHAPES = {
    "tiny": Shape("tiny", B=2, Hq=4, Hkv=1, D=64, max_q=1, s_max=128),
    "long": Shape("long", B=1, Hq=64, Hkv=8, D=128, max_q=1, s_max=32768),
    "ragged": Shape("ragged", B=64, Hq=32, Hkv=8, D=128, max_q=1, s_max=8192),
    "continuous": Shape("continuous", B=256, Hq=64, Hkv=8, D=128, max_q=1, s_max=16384),
    "shortq": Shape("shortq", B=32, Hq=32, Hkv=4, D=128, max_q=16, s_max=4096),
    # longer queries than one 128-row tile (G = 8: 16 tokens per row tile):
    # causal prefill of whole sequences, q_len = kv_len ~ U{512..2048}
    "prefill": Shape("prefill", B=4, Hq=32, Hkv=4, D=128, max_q=2048, s_max=2048),
}

CONTINUOUS_STEPS = 100


def lengths(name: str, seed: int = 0, steps: int | None = None):
    """Draw (lens_q, lens_k) for a workload.

    Returns a list with one (lens_q, lens_k) pair of int64 arrays of length B
    per step: 1 step for every workload except ``continuous``, which draws
    ``steps`` (default 100) steps from one stream, step s after step s-1.
    """
    sh = SHAPES[name]
    rng = np.random.default_rng(seed)
    if name == "tiny":
        return [(np.ones(2, np.int64), np.array([37, 100], np.int64))]
    if name == "long":
        return [(np.ones(1, np.int64), np.array([32768], np.int64))]
    if name == "ragged":
        lk = rng.integers(0, 8192, size=sh.B, endpoint=True)
        return [(np.ones(sh.B, np.int64), lk.astype(np.int64))]
    if name == "continuous":
        n = CONTINUOUS_STEPS if steps is None else steps
        mu = math.log(LOGNORMAL_MEAN) - LOGNORMAL_SIGMA ** 2 / 2.0
        out = []
        for _ in range(n):
            x = rng.lognormal(mean=mu, sigma=LOGNORMAL_SIGMA, size=sh.B)
            lk = np.clip(np.rint(x), 1, sh.s_max).astype(np.int64)
            out.append((np.ones(sh.B, np.int64), lk))
        return out
    if name == "shortq":
        lq = rng.integers(1, 16, size=sh.B, endpoint=True)
        lk = np.array([rng.integers(int(a), 4096, endpoint=True) for a in lq], np.int64)
        return [(lq.astype(np.int64), lk)]
    if name == "prefill":
        lq = rng.integers(512, 2048, size=sh.B, endpoint=True).astype(np.int64)
        return [(lq, lq.copy())]
    raise KeyError(name)


def cu_from_lengths(lens, entries: int | None = None) -> np.ndarray:
    """Cumulative offsets [0, l0, l0+l1, ...] as int32.

    ``entries`` (>= len(lens)+1) pads the array by repeating the last offset,
    i.e. appending zero-length sequences up to a plan's B_max."""
    lens = np.asarray(lens, dtype=np.int64)
    cu = np.zeros(len(lens) + 1, dtype=np.int64)
    np.cumsum(lens, out=cu[1:])
    if entries is not None:
        if entries < cu.size:
            raise ValueError("entries must be >= len(lens) + 1")
        cu = np.concatenate([cu, np.full(entries - cu.size, cu[-1], np.int64)])
    if cu[-1] > np.iinfo(np.int32).max:
        raise ValueError("offsets overflow int32")
    return cu.astype(np.int32)


def bf16_normal(shape, generator: torch.Generator, device) -> torch.Tensor:
    """iid N(0, 1) drawn in fp32, rounded to bf16 (round to nearest even)."""
    x = torch.randn(shape, generator=generator, device=device, dtype=torch.float32)
    return x.to(torch.bfloat16)


def make_generator(seed: int, gen_device) -> torch.Generator:
    g = torch.Generator(device=gen_device)
    g.manual_seed(seed)
    return g


@dataclasses.dataclass
class Batch:
    """One set of inputs: packed q [T_q, Hq, D], k / v [T_kv, Hkv, D] (bf16)
    and cu arrays with B_max+1 int32 entries (host numpy)."""
    shape: Shape
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    cu_q: np.ndarray
    cu_k: np.ndarray
    lens_q: np.ndarray
    lens_k: np.ndarray

    @property
    def kv_tokens(self) -> int:
        return int(self.cu_k[-1])

    @property
    def q_tokens(self) -> int:
        return int(self.cu_q[-1])


def make_batch(shape: Shape, lens_q, lens_k, seed: int = 0, gen_device="cpu",
               kv_capacity: int | None = None, q_capacity: int | None = None) -> Batch:
    """Draw q, k, v for the given lengths.

    ``kv_capacity`` / ``q_capacity`` (tokens) allocate larger packed buffers
    than this step needs, so later steps can reuse them with other lengths."""
    lens_q = np.asarray(lens_q, np.int64)
    lens_k = np.asarray(lens_k, np.int64)
    cu_q = cu_from_lengths(lens_q, shape.B + 1)
    cu_k = cu_from_lengths(lens_k, shape.B + 1)
    T_q = max(int(cu_q[-1]), q_capacity or 0)
    T_kv = max(int(cu_k[-1]), kv_capacity or 0)
    g = make_generator(seed, gen_device)
    q = bf16_normal((T_q, shape.Hq, shape.D), g, gen_device)
    k = bf16_normal((T_kv, shape.Hkv, shape.D), g, gen_device)
    v = bf16_normal((T_kv, shape.Hkv, shape.D), g, gen_device)
    return Batch(shape, q, k, v, cu_q, cu_k, lens_q, lens_k)


def workload(name: str, seed: int = 0, gen_device="cpu", step: int = 0) -> Batch:
    """The named workload's inputs (for ``continuous``: one step's lengths)."""
    sh = SHAPES[name]
    lq, lk = lengths(name, seed)[step]
    return make_batch(sh, lq, lk, seed=seed, gen_device=gen_device)


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> host numpy uint16 bit patterns (no value change)."""
    if t.dtype != torch.bfloat16:
        raise TypeError("expected a bf16 tensor")
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def from_bits(a: np.ndarray) -> torch.Tensor:
    """host numpy uint16 bit patterns -> CPU bf16 tensor (no value change)."""
    a = np.ascontiguousarray(a, dtype=np.uint16)
    return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16)


def bf16_bits_to_f64(a: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64 (for checks)."""
    a = np.asarray(a, dtype=np.uint16)
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float64 values to bf16 bit patterns (via fp32, nearest even).

    Used to build special-case inputs (constant keys, ramps); finite values
    only."""
    f = np.asarray(x, dtype=np.float32)
    return bits(torch.from_numpy(np.ascontiguousarray(f)).to(torch.bfloat16))


# ------------------------------------------------------------ paged K/V caches

@dataclasses.dataclass
class PagedCache:
    """A batch's keys and values scattered into a paged cache.

    k_cache / v_cache: [num_pages, page_size, Hkv, D] (views of one
    [num_pages, 2, page_size, Hkv, D] buffer when fused); block_table:
    [B_max, cols] int32, row b listing sequence b's pages in key order, every
    entry past the sequence's pages set to `unused`."""
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    block_table: torch.Tensor
    page_size: int


def paginate(k: torch.Tensor, v: torch.Tensor, cu_k, B_max: int, page_size: int, s_max: int, *,
             seed: int = 0, spare_pages: int = 3, fill: float = float("nan"), fused: bool = False,
             extra_cols: int = 0, unused: int = -7) -> PagedCache:
    """Place key j of sequence b (packed token cu_k[b] + j) at slot j % page_size
    of a randomly chosen distinct page; slots no key uses hold `fill` (NaN by
    default, so a kernel that lets them into its result fails loudly).
    `spare_pages` pages belong to no sequence."""
    cu_k = np.asarray(cu_k, dtype=np.int64)
    lens = np.diff(cu_k[: B_max + 1])
    Hkv, D = k.shape[1], k.shape[2]
    n_pages_b = (lens + page_size - 1) // page_size
    total = int(n_pages_b.sum()) + spare_pages
    rng = np.random.default_rng(seed)
    phys = rng.permutation(total)                  # logical page -> physical page
    cols = (s_max + page_size - 1) // page_size + extra_cols
    bt = np.full((B_max, cols), unused, dtype=np.int32)
    first = np.concatenate([[0], np.cumsum(n_pages_b)])
    rows = []                                       # physical row of each packed key
    for b in range(B_max):
        n = int(n_pages_b[b])
        bt[b, :n] = phys[first[b]: first[b] + n]
        j = np.arange(int(lens[b]))
        rows.append(phys[first[b] + j // page_size] * page_size + j % page_size)
    rows = np.concatenate(rows) if rows else np.zeros(0, np.int64)
    dev = k.device
    if fused:
        buf = torch.full((total, 2, page_size, Hkv, D), fill, dtype=torch.bfloat16, device=dev)
        kc, vc = buf[:, 0], buf[:, 1]
    else:
        kc = torch.full((total, page_size, Hkv, D), fill, dtype=torch.bfloat16, device=dev)
        vc = torch.full((total, page_size, Hkv, D), fill, dtype=torch.bfloat16, device=dev)
    idx = torch.from_numpy(rows).to(dev)
    src = slice(int(cu_k[0]), int(cu_k[0]) + len(rows))
    # scatter through a flat [pages * page_size, Hkv, D] view of each cache
    for cache, data in ((kc, k), (vc, v)):
        flat = cache.reshape(total * page_size, Hkv, D) if cache.is_contiguous() else None
        if flat is not None:
            flat[idx] = data[src]
        else:
            pg, sl = idx // page_size, idx % page_size
            cache[pg, sl] = data[src]
    return PagedCache(kc, vc, torch.from_numpy(bt).to(dev), page_size)
