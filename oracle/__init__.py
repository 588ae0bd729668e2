"""fp64 CPU oracle for the CSA/HCA hot path.

TEST INFRASTRUCTURE, not part of the product.  Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU baseline leg of ``bench.py`` may
import, call or execute anything under ``oracle/``.  The oracle shares no
code with the CUDA library: no kernels, headers, helpers, tables or
constants; neither imports the other.  Both read workloads from ``synth``,
which holds none of the method's arithmetic.

Modules:
  codecs    FP8 E4M3, BF16, E2M1, UE8M0 decoders/encoders from the specs
  csa       the method, step by step (compress, pack, index, top-k, attend)
  pipeline  the five library calls run over a workload's stored bytes

Parity status: every function is pinned by the ``-m "not gpu"`` tests
(closed forms, invariants, hand-worked fixtures under ``tests/golden``,
brute force on tiny inputs, library codecs).  The compressor's reading of the
pages (which blocks overlap, gate granularity, softmax scope) has no
external worked example to pin against; its pins are internal consistency
and the hand-worked fixture of that reading.
"""
