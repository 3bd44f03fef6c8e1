"""Seeded synthetic workloads for paged MLA decode.

This module only draws random numbers and casts them to the storage types; it holds
none of the attention arithmetic, so the CUDA library and the float64 oracle can both
consume its output without sharing any of the method.

The shapes mirror the agentic decode regime the TokenSpeed pages describe: batches
4/8/16 with speculative query lengths 4-16 over long prefixes (more than 50K tokens),
and an fp8 batch-decode case ("TokenSpeed launch digest", MLA kernel paragraphs;
"Faster kernels, slower engine", fp8 KV cache note).  Those pages evaluate on agent
trajectories that are not available here; these seeded inputs stand in for them.

Recipe (per workload, one ``numpy.random.SeedSequence(seed)`` spawned into five
independent PCG64 streams, so chunking one stream never shifts another):
  stream 0  sequence lengths (fixed, uniform integers, or clipped log-normal)
  stream 1  physical page permutation (identity for the tiny case)
  stream 2  cache values N(0, 1), drawn as float32 page chunk by page chunk
  stream 3  per-token row-norm scales U[0.5, 2] (only where the workload asks)
  stream 4  query values N(0, 1)
Values are rounded to bfloat16 (round to nearest even) or encoded to e4m3 with one
per-tensor scale amax / 448.  Rows past a request's length inside its last page, and
the spare pages no request references, hold NaN so that any over-read shows.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

PAGE = 64
DQK = 576
DV = 512
KV_BF16 = 0
KV_E4M3 = 1
BF16_NAN = 0x7FC0
E4M3_NAN = 0x7F
E4M3_MAX = 448.0


@dataclasses.dataclass
class WorkloadSpec:
    name: str
    B: int
    s_q: int
    H: int
    seq: tuple            # ("fixed", T) | ("uniform", lo, hi) | ("lognormal", median, sigma, lo, hi)
    kv_dtype: int = KV_BF16
    causal: bool = True
    identity_pages: bool = False
    row_scale: Optional[tuple] = None   # (lo, hi) per-token multiplier
    seed: int = 0
    spare_pages: int = 2

    @property
    def M(self) -> int:
        return self.s_q * self.H

    @property
    def scale(self) -> float:
        # 1/sqrt(128 + 64): the un-absorbed head dimension of a DeepSeek-style MLA
        return 1.0 / math.sqrt(192.0)


# The five workloads (tiny, agent spec-decode, ragged, long, fp8 batch).
WORKLOADS = {
    "tiny": WorkloadSpec("tiny", B=1, s_q=1, H=16, seq=("fixed", 256), identity_pages=True, seed=0),
    "agent_spec": WorkloadSpec("agent_spec", B=4, s_q=4, H=16, seq=("fixed", 65536), seed=1),
    "ragged_rownorm": WorkloadSpec("ragged_rownorm", B=8, s_q=8, H=32, seq=("uniform", 32768, 65536),
                                   row_scale=(0.5, 2.0), seed=2),
    "long_m256": WorkloadSpec("long_m256", B=16, s_q=16, H=16, seq=("fixed", 131072), seed=3),
    "fp8_batch": WorkloadSpec("fp8_batch", B=32, s_q=2, H=128, seq=("lognormal", 8192, 1.0, 512, 65536),
                              kv_dtype=KV_E4M3, seed=4),
}
WORKLOAD_ORDER = ["tiny", "agent_spec", "ragged_rownorm", "long_m256", "fp8_batch"]


@dataclasses.dataclass
class Workload:
    spec: WorkloadSpec
    q: np.ndarray            # uint16 bf16 bits [B, s_q, H, 576]
    kv: np.ndarray           # uint16 bf16 bits or uint8 e4m3 [P, 64, 576]
    kv_scale: float
    block_table: np.ndarray  # int32 [B, max_pages], -1 past each request's pages
    seq_lens: np.ndarray     # int32 [B]
    scale: float
    causal: bool

    @property
    def B(self):
        return self.spec.B

    @property
    def s_q(self):
        return self.spec.s_q

    @property
    def H(self):
        return self.spec.H

    @property
    def kv_dtype(self):
        return self.spec.kv_dtype

    @property
    def num_pages(self):
        return int(self.kv.shape[0])

    def kv_bytes(self) -> int:
        """Bytes of cache rows a decode must read: sum of lengths x 576 x element size."""
        return int(self.seq_lens.astype(np.int64).sum()) * DQK * (2 if self.kv_dtype == KV_BF16 else 1)

    def flops(self) -> int:
        """Algorithmic FLOPs 2 * (s_q * H) * T * (576 + 512) summed over requests."""
        return int(2 * self.spec.M * int(self.seq_lens.astype(np.int64).sum()) * (DQK + DV))


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _e4m3_bytes(x: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy()


def draw_seq_lens(spec: WorkloadSpec, rng: np.random.Generator) -> np.ndarray:
    kind = spec.seq[0]
    if kind == "fixed":
        return np.full(spec.B, spec.seq[1], dtype=np.int32)
    if kind == "uniform":
        return rng.integers(spec.seq[1], spec.seq[2] + 1, size=spec.B).astype(np.int32)
    if kind == "lognormal":
        _, median, sigma, lo, hi = spec.seq
        z = rng.standard_normal(spec.B)
        t = np.rint(np.exp(math.log(median) + sigma * z))
        return np.clip(t, lo, hi).astype(np.int32)
    raise ValueError(kind)


def make_workload(spec, seed: Optional[int] = None, seq_lens=None, chunk_pages: int = 512,
                  **overrides) -> Workload:
    """Build the host arrays of one workload.

    ``spec`` is a WorkloadSpec or a key of WORKLOADS; keyword overrides replace spec
    fields (e.g. a shorter ``seq`` for a parity-size case); ``seq_lens`` forces the
    lengths outright.
    """
    if isinstance(spec, str):
        spec = WORKLOADS[spec]
    if overrides or seed is not None:
        kw = dict(overrides)
        if seed is not None:
            kw["seed"] = seed
        spec = dataclasses.replace(spec, **kw)
    streams = [np.random.Generator(np.random.PCG64(s)) for s in np.random.SeedSequence(spec.seed).spawn(5)]
    r_len, r_perm, _, r_scale, r_q = streams  # stream 2 is re-created per pass in chunks()

    lens = np.asarray(seq_lens, dtype=np.int32) if seq_lens is not None else draw_seq_lens(spec, r_len)
    assert lens.shape == (spec.B,)
    npages = (lens.astype(np.int64) + PAGE - 1) // PAGE
    used = int(npages.sum())
    P = used + int(spec.spare_pages)
    max_pages = int(max(1, npages.max()))
    perm = np.arange(P, dtype=np.int64) if spec.identity_pages else r_perm.permutation(P)
    bt = np.full((spec.B, max_pages), -1, dtype=np.int32)
    k = 0
    for b in range(spec.B):
        n = int(npages[b])
        bt[b, :n] = perm[k:k + n]
        k += n
    spare = perm[used:]

    rows_total = P * PAGE
    rs = None
    if spec.row_scale is not None:
        rs = r_scale.uniform(spec.row_scale[0], spec.row_scale[1], size=rows_total).astype(np.float32)

    def chunks():
        # the value stream is drawn in fixed page chunks so the result is independent of memory
        kv_rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence(spec.seed).spawn(5)[2]))
        for p0 in range(0, P, chunk_pages):
            p1 = min(P, p0 + chunk_pages)
            x = kv_rng.standard_normal((p1 - p0) * PAGE * DQK, dtype=np.float32).reshape(p1 - p0, PAGE, DQK)
            if rs is not None:
                x *= rs[p0 * PAGE:p1 * PAGE].reshape(p1 - p0, PAGE, 1)
            yield p0, p1, x

    kv_scale = 1.0
    if spec.kv_dtype == KV_BF16:
        kv = np.empty((P, PAGE, DQK), dtype=np.uint16)
        for p0, p1, x in chunks():
            kv[p0:p1] = _bf16_bits(x)
        nan_code = BF16_NAN
    else:
        amax = 0.0
        for _, _, x in chunks():
            amax = max(amax, float(np.abs(x).max()))
        kv_scale = float(np.float32(amax / E4M3_MAX))
        kv = np.empty((P, PAGE, DQK), dtype=np.uint8)
        for p0, p1, x in chunks():
            kv[p0:p1] = _e4m3_bytes(np.clip(x / np.float32(kv_scale), -E4M3_MAX, E4M3_MAX))
        nan_code = E4M3_NAN
    # canaries: the tail of each request's last page and every spare page
    for b in range(spec.B):
        T = int(lens[b])
        if T % PAGE:
            kv[bt[b, T // PAGE], T % PAGE:, :] = nan_code
    for p in spare:
        kv[int(p)] = nan_code

    q = _bf16_bits(r_q.standard_normal((spec.B, spec.s_q, spec.H, DQK), dtype=np.float32))
    return Workload(spec=spec, q=q, kv=kv, kv_scale=kv_scale, block_table=bt, seq_lens=lens,
                    scale=spec.scale, causal=spec.causal)


def bf16_bits_to_float32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
