"""Helpers shared by the GPU tests: move a workload to the device, run the CUDA
path through the C-ABI binding, and compare with the fp64 oracle."""
from __future__ import annotations

import numpy as np
import torch

import decode_attention_paged_split_b200 as apd

# Per bf16 output element: |gpu - ref| <= ATOL + RTOL * |ref|, ref = fp64 oracle.
ATOL = 1e-2
RTOL = 1e-2


class DeviceProblem:
    """A workload's tensors on the GPU (same logical views and strides as on the host)."""

    def __init__(self, w, device="cuda"):
        self.w = w
        self.q = w.q.to(device)
        # keep the storage order (NHD/blhd, or HND/bhld) of the host cache
        heads_outer = w.layout in ("HND", "bhld")
        ks = w.k_cache.permute(0, 2, 1, 3) if heads_outer else w.k_cache
        vs = w.v_cache.permute(0, 2, 1, 3) if heads_outer else w.v_cache
        ks = ks.contiguous().to(device)
        vs = vs.contiguous().to(device)
        self.k = ks.permute(0, 2, 1, 3) if heads_outer else ks
        self.v = vs.permute(0, 2, 1, 3) if heads_outer else vs
        self.contig = w.meta.get("kv_policy") == "contig"
        self.page_table = w.page_table.to(device)
        self.seq_lens = w.seq_lens.to(device)
        self.out = torch.full_like(self.q, float("nan"))
        self.workspace = None

    def run(self, num_splits: int | None = None, stream=None, workspace=None) -> torch.Tensor:
        s = self.w.num_splits if num_splits is None else num_splits
        if workspace is None:
            workspace = apd.alloc_workspace(self.q.shape[0], self.q.shape[1], self.k.shape[2], self.q.shape[2], s)
        self.workspace = workspace
        if self.contig:
            apd.attn_contig_decode(self.q, self.k, self.v, self.seq_lens, self.out, self.w.scale, s, workspace,
                                   stream=stream)
        else:
            apd.attn_paged_decode(self.q, self.k, self.v, self.page_table, self.seq_lens, self.out, self.w.scale, s,
                                  workspace, stream=stream)
        return self.out


def check_close(got: torch.Tensor, ref: np.ndarray, what: str = "") -> dict:
    """Element-wise tolerance check of a bf16 GPU result against the fp64 oracle."""
    g = got.detach().to("cpu", torch.float64).numpy()
    assert g.shape == ref.shape, (g.shape, ref.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite output at {np.argwhere(~np.isfinite(g))[:5].tolist()}"
    err = np.abs(g - ref)
    bound = ATOL + RTOL * np.abs(ref)
    bad = err > bound
    if bad.any():
        idx = np.argwhere(bad)[:5].tolist()
        raise AssertionError(f"{what}: {int(bad.sum())} elements outside |gpu-ref| <= {ATOL} + {RTOL}|ref|; "
                             f"max err {err.max():.3e}; first at {idx}")
    return {"max_abs_err": float(err.max()), "max_err_over_bound": float((err / bound).max())}
