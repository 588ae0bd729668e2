"""Decode-time state of one sequence, token by token (oracle).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import anything under ``oracle/``.

kwkr.cn notes 4.4 (FP4 QAT 与 KV Cache 层级): besides the classical KV cache
(here: the compressed entries) a sequence keeps a *state cache*: the
sliding window's raw tokens and the compressor's tokens that do not yet form
a complete entry; the state can be checkpointed periodically (every 1024
tokens) so that a sequence can resume from a checkpoint.

Readings (the page names the parts, not their contents):

* The window state at position P (after P tokens) is the packed KV rows of
  tokens max(0, P-W) .. P-1, packed like a compressed entry (the mixed
  layout: FP8 E4M3 non-RoPE dims with scale amax/448, BF16 RoPE dims).
* The compressor state at P (P a multiple of m) is the stream rows and gate
  logits of tokens P-m .. P-1: entry P/m merges stream a over tokens
  P .. P+m-1 with stream b over these (kwkr.cn notes 3.1: adjacent blocks
  overlap), so they are all a resumed sequence needs.
* Entries are the compressor's output for every complete block, exactly
  as ``oracle.csa.compress`` computes them over the whole sequence.
* A checkpoint taken at P holds both states at P; checkpoint slot
  (P / every - 1) mod n_slots.
"""

from __future__ import annotations

import numpy as np

from . import csa


def window_row(v, r: int, kv_fmt: str):
    """One token's window row in the cache layout: (codes, scale, rope bits)
    for the fp8 format, the f64 vector itself for f32."""
    if kv_fmt == "f32":
        return np.asarray(v, dtype=np.float64)
    return csa.pack_entry(v, r)


def window_state(kv, P: int, W: int, r: int, kv_fmt: str):
    """{position: row} of the window state after P tokens."""
    return {p: window_row(kv[p], r, kv_fmt) for p in range(max(0, P - W), P)}


def stream_state(a, b, gate, P: int, m: int):
    """{position: (a row, b row, gate pair)} of the compressor state at P."""
    assert P % m == 0
    return {p: (a[p], b[p], gate[p]) for p in range(max(0, P - m), P)}


def entries_after(a, b, gate, P: int, m: int, r: int, theta: float, eps: float):
    """The entries complete after P tokens (entry e needs tokens up to
    m(e+1) - 1): compress over the whole prefix."""
    n = P // m
    if n == 0:
        return np.zeros((0, np.asarray(a).shape[-1])), np.zeros(0, np.int64)
    return csa.compress(a[:n * m], b[:n * m], gate[:n * m], m, r, theta, eps, None, e_begin=0, e_end=n)


def checkpoints(P_from: int, P_to: int, every: int):
    """Checkpoint positions crossed by appending tokens P_from .. P_to-1:
    every multiple of ``every`` in (P_from, P_to]."""
    first = (P_from // every + 1) * every
    return list(range(first, P_to + 1, every))
