"""Device-resident workloads driven through the five library calls.

A workload is a dict of host (numpy) arrays in the storage layouts that
``include/csa.h`` documents (the keys are listed in ``DeviceWorkload``).
``DeviceWorkload`` uploads it once, allocates outputs and workspaces with
torch (torch is only the allocator and stream provider here) and runs the
CSA or HCA step through the binding.  It never computes anything itself.
"""

from __future__ import annotations

import numpy as np
import torch

from . import (ACT_BF16, ACT_F32, IDX_F32, IDX_MXFP4, KV_F32, KV_FP8_BF16, SCORE_BF16, SCORE_F32, csa_compress,
               csa_index_topk, csa_index_topk_workspace_bytes, csa_sparse_attn,
               csa_sparse_attn_workspace_bytes, hca_compress, hca_dense_attn,
               hca_dense_attn_workspace_bytes, make_params)

_KV = {"f32": KV_F32, "fp8": KV_FP8_BF16}
_IDX = {"f32": IDX_F32, "mxfp4": IDX_MXFP4}
_ACT = {"f32": ACT_F32, "bf16": ACT_BF16}

# per-step inputs (copied host->device every step in the end-to-end path)
STEP_INPUTS = ("a", "b", "gate", "q_idx", "q_idx_sf", "w_idx", "q")


def params_of(p):
    """csa_params from a workload's parameter record (attribute names of
    ``synth.Params``)."""
    return make_params(B=p.B, d=p.d, r=p.r, m=p.m, n_idx_heads=p.H_I, idx_dim=p.c_I,
                       topk=max(p.k, 1), n_heads=p.n_h, window=p.W, kv_fmt=_KV[p.kv_fmt],
                       idx_fmt=_IDX[p.idx_fmt], act_fmt=_ACT[p.act_fmt], softmax_scale=p.tau,
                       rope_theta=p.theta, eps=p.eps,
                       score_fmt=SCORE_BF16 if getattr(p, "score_fmt", "f32") == "bf16" else SCORE_F32)


def _t(x, device):
    return torch.from_numpy(np.ascontiguousarray(x)).to(device)


class DeviceWorkload:
    """Keys used: params, T, Ncap, q_pos0, S, a, b, gate, tok_base, e_begin,
    e_end, kv, kv_scale, Wcap, win, win_scale, q_idx, q_idx_sf, w_idx, k_idx,
    k_idx_sf, q, sink."""

    def __init__(self, w, device="cuda", kinds=None):
        p = w["params"]
        self.p, self.w, self.device = p, w, device
        self.params = params_of(p)
        self.T = int(w["T"])
        self.Ncap = int(w["Ncap"])
        B = p.B
        dev = lambda k: _t(w[k], device) if k in w and w[k] is not None else None
        self.q_pos0 = dev("q_pos0")
        self.S = int(w["S"])
        self.a, self.b, self.gate = dev("a"), dev("b"), dev("gate")
        self.tok_base, self.e_begin, self.e_end = dev("tok_base"), dev("e_begin"), dev("e_end")
        self.max_entries = int((np.asarray(w["e_end"]) - np.asarray(w["e_begin"])).max()) if self.S else 0
        self.kv, self.kv_scale = dev("kv"), dev("kv_scale")
        self.win, self.win_scale = dev("win"), dev("win_scale")
        self.q_idx, self.q_idx_sf, self.w_idx = dev("q_idx"), dev("q_idx_sf"), dev("w_idx")
        self.k_idx, self.k_idx_sf = dev("k_idx"), dev("k_idx_sf")
        self.q, self.sink = dev("q"), dev("sink")
        self.kv_pos = torch.zeros((B, self.Ncap), dtype=torch.int32, device=device)
        self.err = torch.zeros(4, dtype=torch.int32, device=device)
        # n_t bound over the batch
        q_end = np.asarray(w["q_pos0"], dtype=np.int64) + self.T
        self.n_max = int(min(self.Ncap, (q_end // p.m).max()))
        self.idx = torch.full((B, self.T, max(p.k, 1)), -2, dtype=torch.int32, device=device)
        out_dt = torch.float32 if p.act_fmt == "f32" else torch.uint16
        self.out = torch.zeros((B, self.T, p.n_h, p.d), dtype=out_dt, device=device)
        nb_idx = csa_index_topk_workspace_bytes(self.params, self.T, self.n_max) if p.k > 0 else 0
        nb_sp = csa_sparse_attn_workspace_bytes(self.params, self.T) if p.k > 0 else 0
        nb_de = hca_dense_attn_workspace_bytes(self.params, self.T, self.n_max)
        self.ws_idx = torch.empty(max(nb_idx, 16), dtype=torch.uint8, device=device)
        self.ws_attn = torch.empty(max(nb_sp, nb_de, 16), dtype=torch.uint8, device=device)

    # ---- the five calls ----------------------------------------------------
    def compress(self, stream=None):
        if not self.S:
            return
        fn = hca_compress if self.p.m >= 64 else csa_compress
        fn(self.params, self.a, self.b, self.gate, self.tok_base, self.e_begin, self.e_end,
           self.max_entries, self.kv, self.kv_scale, self.kv_pos, None, self.err, stream)

    def index_topk(self, stream=None):
        csa_index_topk(self.params, self.q_idx, self.q_idx_sf, self.w_idx, self.k_idx, self.k_idx_sf,
                       self.q_pos0, self.T, self.n_max, self.idx, self.ws_idx, self.err, stream)

    def sparse_attn(self, stream=None):
        csa_sparse_attn(self.params, self.q, self.kv, self.kv_scale, self.idx, self.win, self.win_scale,
                        self.sink, self.q_pos0, self.T, self.out, self.ws_attn, self.err, stream)

    def dense_attn(self, stream=None):
        hca_dense_attn(self.params, self.q, self.kv, self.kv_scale, self.win, self.win_scale, self.sink,
                       self.q_pos0, self.T, self.n_max, self.out, self.ws_attn, self.err, stream)

    def csa_step(self, stream=None, side=None):
        """compress -> index + top-k -> sparse attention.  With a `side`
        stream the compressor runs concurrently with the indexer (they are
        independent; only the attention reads the new entry)."""
        if side is None or not self.S:
            self.compress(stream)
            self.index_topk(stream)
            self.sparse_attn(stream)
            return
        main = stream if stream is not None else torch.cuda.current_stream()
        side.wait_stream(main)
        with torch.cuda.stream(side):
            self.compress(side)
        self.index_topk(main)
        main.wait_stream(side)
        self.sparse_attn(main)

    def hca_step(self, stream=None):
        self.compress(stream)
        self.dense_attn(stream)

    def step(self, stream=None):
        if self.p.k > 0:
            self.csa_step(stream)
        else:
            self.hca_step(stream)

    # ---- host views of the results -------------------------------------------
    def out_f64(self):
        o = self.out.cpu().numpy()
        if self.p.act_fmt == "f32":
            return o.astype(np.float64)
        return (o.astype(np.uint32) << 16).view(np.float32).astype(np.float64)

    def err_bits(self):
        return int(self.err.cpu()[0])
