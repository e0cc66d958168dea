"""Helpers that run one problem through the CUDA path (test support, not a test).

Builds the cache by appending the cached segments' K/V with the library's
append kernel, builds and uploads the metadata, and calls the attention
forward, all through the C ABI binding.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import cache as ocache
from segment_causal_masked_b200 import sca
from segment_causal_masked_b200 import workloads as W


class GpuSession:
    """``int8``: the cache stores int8 codes and per-row scales (the append
    kernel quantises)."""

    def __init__(self, problem: W.Problem, inputs: dict, capacity: int = None,
                 device: str = "cuda:0", int8: bool = False):
        self.p = problem
        self.dev = torch.device(device)
        h = problem.heads
        nc, nq = problem.n_cache_tokens, problem.n_query_tokens
        self.capacity = capacity or max(nc + nq, 1)
        if int8:
            self.capacity = (self.capacity + 3) // 4 * 4
        cap_pad = (self.capacity + 127) // 128 * 128
        self.desc = torch.zeros(cap_pad, dtype=torch.int32, device=self.dev)
        if int8:
            # codes are stored offset-binary (code + 128)
            self.k_buf = torch.zeros(h, self.capacity, 128, dtype=torch.uint8, device=self.dev)
            self.v_buf = torch.zeros_like(self.k_buf)
            self.k_scale = torch.zeros(h, self.capacity, dtype=torch.float32, device=self.dev)
            self.v_scale = torch.zeros_like(self.k_scale)
            self.cache = sca.KVCache(h, self.capacity, self.k_buf, self.v_buf, self.desc,
                                     self.k_scale, self.v_scale)
        else:
            self.k_buf = torch.zeros(h, self.capacity, 128, dtype=torch.bfloat16, device=self.dev)
            self.v_buf = torch.zeros_like(self.k_buf)
            self.cache = sca.KVCache(h, self.capacity, self.k_buf, self.v_buf, self.desc)
        ck = inputs["cache_k"].to(self.dev)
        cv = inputs["cache_v"].to(self.dev)
        pos = 0
        for seg in problem.cached:
            n = seg.n_tokens
            self.cache.append(seg, ck[pos:pos + n].contiguous(), cv[pos:pos + n].contiguous())
            pos += n
        self.q = inputs["q"].to(self.dev).contiguous()
        self.k_cur = inputs["k_cur"].to(self.dev).contiguous()
        self.v_cur = inputs["v_cur"].to(self.dev).contiguous()
        self.md = sca.build_for(problem).upload()
        self.status = torch.zeros(1, dtype=torch.int32, device=self.dev)

    def forward(self, q=None, k_cur=None, v_cur=None, workspace=True):
        """One attention call; with ``workspace`` the split plan's scratch is
        passed (so the key-split tail and the merge kernel run when planned)."""
        q = self.q if q is None else q
        k_cur = self.k_cur if k_cur is None else k_cur
        v_cur = self.v_cur if v_cur is None else v_cur
        nq, h = self.p.n_query_tokens, self.p.heads
        o = torch.empty(nq, h, 128, dtype=torch.bfloat16, device=self.dev)
        lse = torch.empty(h, nq, dtype=torch.float32, device=self.dev)
        ws = None
        if workspace:
            nbytes = sca.attn_workspace_bytes(self.md, h)
            ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=self.dev)
        sca.action_causal_attn_fwd(self.cache if self.p.cached else None, self.md, h, q, k_cur,
                                   v_cur, o, lse, self.p.softmax_scale, ws, None, self.status)
        torch.cuda.synchronize(self.dev)
        assert int(self.status.item()) == 0, f"device status {int(self.status.item())}"
        return o, lse


def oracle_inputs(inputs: dict, int8: bool = False):
    """float32 numpy views (exact copies of the bf16 values) for the oracle;
    with ``int8`` the cached keys and values are the oracle's INT8 round trip
    (codes times scales, float64)."""
    q = inputs["q"].float().numpy()
    ck, cv = inputs["cache_k"].float().numpy(), inputs["cache_v"].float().numpy()
    if int8:
        ck = ocache.dequantize_rows(*ocache.quantize_rows(ck))
        cv = ocache.dequantize_rows(*ocache.quantize_rows(cv))
    k = np.concatenate([ck, inputs["k_cur"].float().numpy()])
    v = np.concatenate([cv, inputs["v_cur"].float().numpy()])
    return q, k, v


def compare(o_gpu, lse_gpu, o_ref, lse_ref, atol=2e-2, rel=1e-2, lse_tol=1e-2):
    """The parity bar: max |dO| <= atol (bf16 in/out, fp32 accumulate), relative
    L2 error <= rel, |dLSE| <= lse_tol; returns the measured errors."""
    o = o_gpu.float().cpu().numpy().astype(np.float64)
    d = np.abs(o - o_ref)
    max_abs = float(d.max())
    rel_l2 = float(np.linalg.norm(o - o_ref) / max(np.linalg.norm(o_ref), 1e-30))
    finite = np.isfinite(lse_ref)
    l = lse_gpu.float().cpu().numpy().astype(np.float64)
    assert np.array_equal(np.isfinite(l), finite)
    lse_err = float(np.abs(l[finite] - lse_ref[finite]).max()) if finite.any() else 0.0
    assert max_abs <= atol, f"max |dO| = {max_abs}"
    assert rel_l2 <= rel, f"relative L2 = {rel_l2}"
    assert lse_err <= lse_tol, f"max |dLSE| = {lse_err}"
    return max_abs, rel_l2, lse_err
