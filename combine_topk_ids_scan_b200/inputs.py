"""Seeded synthetic inputs for MoE dispatch / combine.

This module only draws random inputs (token ids, gate weights, hidden rows,
synthetic expert outputs).  It holds none of the dispatch or combine
arithmetic, so both the CUDA path and the CPU oracle can be fed from it
without sharing any of the method's code.

Workloads (shapes and routing structure of the MoE dispatch / combine pages;
seed = 1000 + index):

  0 tiny            N=512   H=1024 E=8   k=2 S=4  uniform distinct ids, C=N*k
  1 mid_zipf        N=4096  H=4096 E=64  k=6 S=8  Zipf(s=1) over a seeded
                                                  expert permutation, C=N*6
  2 fp8_metric      N=8192  H=7168 E=256 k=8 S=8  uniform distinct ids; 1% of
                                                  rows scaled x100; C=N*k;
                                                  expert outputs ~N(0,1)
  3 nvfp4_hot       N=16384 H=7168 E=256 k=8 S=8  10% of tokens include expert
                                                  0; global scale amax/2688
  4 decode_capacity N=128   H=7168 E=256 k=8 S=8  capacity layout [E,Ce,H],
                                                  Ce = ceil(1.25*N*k/E) = 5
  5 balanced_static N=8192  H=7168 E=256 k=8 S=8  expert (t*k+j) mod E

Distinct ids per token are drawn by Gumbel-top-k (sampling without
replacement, in router order).  Gates are a float32 softmax over k N(0,1)
logits.  Hidden rows are N(0,1) float32 rounded to bfloat16 by torch.
Everything is returned as numpy arrays (bf16 data as uint16 bit patterns).
"""
from __future__ import annotations

import concurrent.futures as cf
import dataclasses
import os

import numpy as np

CONFIG_NAMES = ["tiny", "mid_zipf", "fp8_metric", "nvfp4_hot", "decode_capacity",
                "balanced_static"]

_ROWS_PER_CHUNK = 1024


@dataclasses.dataclass
class Workload:
    name: str
    N: int
    H: int
    E: int
    k: int
    S: int
    recv_capacity: int          # C rows in packed mode (0 in capacity mode)
    expert_capacity: int        # Ce > 0 selects the [E, Ce, H] layout
    ids: np.ndarray             # int32 [N, k]
    gates: np.ndarray           # float32 [N, k]
    hidden: np.ndarray          # uint16 [N, H] (bf16 bits)
    expert_out: np.ndarray | None  # uint16 [rows, H] (bf16 bits) or None
    global_scale: float         # NVFP4 decode global scale (float32 value)
    seed: int

    @property
    def rows(self) -> int:
        return self.E * self.expert_capacity if self.expert_capacity > 0 else self.recv_capacity

    @property
    def P(self) -> int:
        return self.N * self.k


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def normal_bf16(seed_seq: np.random.SeedSequence, rows: int, H: int,
                threads: int | None = None) -> np.ndarray:
    """rows x H bf16 bit patterns of N(0,1) draws; chunked by rows with
    spawned child seeds, so the result does not depend on the thread count."""
    out = np.empty((rows, H), np.uint16)
    n_chunks = (rows + _ROWS_PER_CHUNK - 1) // _ROWS_PER_CHUNK
    children = seed_seq.spawn(n_chunks)

    def work(c):
        r0 = c * _ROWS_PER_CHUNK
        r1 = min(rows, r0 + _ROWS_PER_CHUNK)
        g = np.random.Generator(np.random.PCG64(children[c]))
        out[r0:r1] = _bf16_bits(g.standard_normal((r1 - r0, H), dtype=np.float32))

    threads = threads or min(16, os.cpu_count() or 1)
    if n_chunks <= 1 or threads <= 1:
        for c in range(n_chunks):
            work(c)
    else:
        with cf.ThreadPoolExecutor(threads) as ex:
            list(ex.map(work, range(n_chunks)))
    return out


def gumbel_topk(rng: np.random.Generator, log_w: np.ndarray, N: int, k: int) -> np.ndarray:
    """k distinct ids per row by Gumbel-top-k over log-weights log_w[E]."""
    g = rng.gumbel(size=(N, log_w.size)) + log_w[None, :]
    return np.argsort(-g, axis=1, kind="stable")[:, :k].astype(np.int32)


def softmax_gates(rng: np.random.Generator, N: int, k: int) -> np.ndarray:
    logits = rng.standard_normal((N, k), dtype=np.float32)
    z = np.exp(logits - logits.max(axis=1, keepdims=True), dtype=np.float32)
    return (z / z.sum(axis=1, keepdims=True, dtype=np.float32)).astype(np.float32)


def make_workload(name_or_index, seed: int | None = None, n_tokens: int | None = None,
                  with_expert_out: bool = True, with_hidden: bool = True) -> Workload:
    """Build one workload.  ``n_tokens`` overrides N (a sub-batch with the
    same routing distribution; packed capacity stays N*k-proportional)."""
    idx = (CONFIG_NAMES.index(name_or_index) if isinstance(name_or_index, str)
           else int(name_or_index))
    name = CONFIG_NAMES[idx]
    seed = 1000 + idx if seed is None else seed
    ss = np.random.SeedSequence(seed)
    s_route, s_gate, s_hidden, s_out, s_extra = ss.spawn(5)
    rng = np.random.Generator(np.random.PCG64(s_route))

    if name == "tiny":
        N, H, E, k, S = 512, 1024, 8, 2, 4
    elif name == "mid_zipf":
        N, H, E, k, S = 4096, 4096, 64, 6, 8
    elif name in ("fp8_metric", "balanced_static"):
        N, H, E, k, S = 8192, 7168, 256, 8, 8
    elif name == "nvfp4_hot":
        N, H, E, k, S = 16384, 7168, 256, 8, 8
    elif name == "decode_capacity":
        N, H, E, k, S = 128, 7168, 256, 8, 8
    else:  # pragma: no cover
        raise ValueError(name)
    if n_tokens is not None:
        N = int(n_tokens)

    # ---- routing
    if name == "mid_zipf":
        perm = rng.permutation(E)
        log_w = np.empty(E)
        log_w[perm] = -1.0 * np.log(np.arange(1, E + 1))   # weight ~ 1/rank^s, s=1
        ids = gumbel_topk(rng, log_w, N, k)
    elif name == "nvfp4_hot":
        ids = gumbel_topk(rng, np.zeros(E), N, k)
        n_hot = int(round(0.10 * N))
        hot = rng.choice(N, size=n_hot, replace=False)
        others = gumbel_topk(rng, np.zeros(E - 1), n_hot, k - 1) + 1  # from 1..E-1
        pos = rng.integers(0, k, size=n_hot)
        for i, t in enumerate(hot):
            row = list(others[i])
            row.insert(int(pos[i]), 0)
            ids[t] = row
    elif name == "balanced_static":
        t = np.arange(N, dtype=np.int64)[:, None]
        j = np.arange(k, dtype=np.int64)[None, :]
        ids = ((t * k + j) % E).astype(np.int32)
    else:
        ids = gumbel_topk(rng, np.zeros(E), N, k)
    ids = np.ascontiguousarray(ids, dtype=np.int32)

    gates = softmax_gates(np.random.Generator(np.random.PCG64(s_gate)), N, k)

    # ---- capacities
    if name == "decode_capacity":
        recv_capacity = 0
        expert_capacity = (5 * N * k + 4 * E - 1) // (4 * E)   # ceil(1.25*N*k/E)
    elif name == "mid_zipf":
        recv_capacity = N * min(k, 8)
        expert_capacity = 0
    else:
        recv_capacity = N * k
        expert_capacity = 0
    rows = E * expert_capacity if expert_capacity > 0 else recv_capacity

    # ---- hidden rows
    hidden = np.zeros((N, H), np.uint16)
    global_scale = 1.0
    if with_hidden:
        if name == "fp8_metric":
            g = np.random.Generator(np.random.PCG64(s_hidden))
            xf = g.standard_normal((N, H), dtype=np.float32)
            n_out = int(round(0.01 * N))
            sel = np.random.Generator(np.random.PCG64(s_extra)).choice(N, size=n_out, replace=False)
            xf[sel] *= np.float32(100.0)
            hidden = _bf16_bits(xf)
            del xf
        else:
            hidden = normal_bf16(s_hidden, N, H)
        # NVFP4 decode global scale: tensor amax / (448 * 6), 1 when amax == 0
        hv = (hidden.astype(np.uint32) << 16).view(np.float32)
        amax = np.float32(np.max(np.abs(hv))) if hv.size else np.float32(0)
        global_scale = float(amax / np.float32(2688.0)) if amax > 0 else 1.0

    expert_out = normal_bf16(s_out, rows, H) if with_expert_out else None

    return Workload(name=name, N=N, H=H, E=E, k=k, S=S, recv_capacity=recv_capacity,
                    expert_capacity=expert_capacity, ids=ids, gates=gates, hidden=hidden,
                    expert_out=expert_out, global_scale=float(np.float32(global_scale)),
                    seed=seed)
