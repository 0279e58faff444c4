"""Convenience wrapper: workspaces held in torch device memory, plan/fwd/bwd calls.

The library itself never allocates; this wrapper allocates the three
workspaces once per problem with torch and passes them to the C entry points.
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np


class BranchAttention:
    def __init__(self, problem, device="cuda"):
        import torch
        from . import ba_workspace_size
        self.problem = problem
        self.device = torch.device(device)
        plan_b, fwd_b, bwd_b = ba_workspace_size(problem)
        self.plan_ws = torch.empty(plan_b, dtype=torch.uint8, device=self.device)
        self.fwd_ws = torch.empty(fwd_b, dtype=torch.uint8, device=self.device) if fwd_b else None
        self.bwd_ws = torch.empty(bwd_b, dtype=torch.uint8, device=self.device)

    # -- calls ---------------------------------------------------------------
    def plan(self, stream=None):
        from . import ba_plan
        ba_plan(self.problem, self.plan_ws, stream)

    def plan_status(self, stream=None) -> int:
        from . import ba_plan_status
        return ba_plan_status(self.plan_ws, stream)

    def alloc_outputs(self):
        import torch
        sh = self.problem.shapes()
        kw = dict(device=self.device)
        return {"o_m": torch.empty(sh["q_m"], dtype=torch.bfloat16, **kw),
                "o_b": torch.empty(sh["q_b"], dtype=torch.bfloat16, **kw),
                "lse_m": torch.empty(sh["lse_m"], dtype=torch.float32, **kw),
                "lse_b": torch.empty(sh["lse_b"], dtype=torch.float32, **kw)}

    def alloc_grads(self):
        import torch
        sh = self.problem.shapes()
        return {f"d{k}": torch.empty(sh[k], dtype=torch.bfloat16, device=self.device)
                for k in ("q_m", "k_m", "v_m", "q_b", "k_b", "v_b")}

    def forward(self, t: Dict, out: Optional[Dict] = None, stream=None) -> Dict:
        from . import branch_attn_fwd
        out = out if out is not None else self.alloc_outputs()
        branch_attn_fwd(self.problem, self.plan_ws, self.fwd_ws, t["q_m"], t["k_m"], t["v_m"],
                        t["q_b"], t["k_b"], t["v_b"], out["o_m"], out["o_b"], out["lse_m"],
                        out["lse_b"], stream)
        return out

    def backward(self, t: Dict, out: Dict, grads: Optional[Dict] = None, stream=None) -> Dict:
        from . import branch_attn_bwd
        grads = grads if grads is not None else self.alloc_grads()
        branch_attn_bwd(self.problem, self.plan_ws, self.bwd_ws, t["q_m"], t["k_m"], t["v_m"],
                        t["q_b"], t["k_b"], t["v_b"], out["o_m"], out["o_b"], out["lse_m"],
                        out["lse_b"], t["do_m"], t["do_b"], grads["dq_m"], grads["dk_m"],
                        grads["dv_m"], grads["dq_b"], grads["dk_b"], grads["dv_b"], stream)
        return grads

    # -- inspection ----------------------------------------------------------
    def read_plan(self) -> Dict[str, np.ndarray]:
        """Copy the plan metadata back to the host as int64 numpy arrays."""
        from . import ba_plan_layout_query
        L = ba_plan_layout_query(self.problem)
        raw = self.plan_ws.cpu().numpy().view(np.int32)
        c = self.problem.c
        n_qt = L["n_qtiles_main"] + L["n_qtiles_branch"]
        n_kv = L["n_kv_main"] + L["n_kv_branch"]
        rows = c.n_main + c.n_branch_tokens

        def arr(off, n, width=1):
            a = raw[off // 4: off // 4 + n * width].astype(np.int64)
            return a.reshape(n, width) if width > 1 else a

        out = {
            "status": int(raw[L["off_status"] // 4]),
            "walk": int(raw[L["off_status"] // 4 + 2]),
            "cu_branch": arr(L["off_cu_branch"], c.n_branches + 1),
            "branch_seq": arr(L["off_branch_seq"], c.n_branches),
            "row_iv": arr(L["off_row_iv"], rows, 4),
            "qtile": arr(L["off_qtile"], n_qt, 6),
            "kv_main": arr(L["off_kv_main"], L["n_kv_main"], 4),
            "kv_branch": arr(L["off_kv_branch"], L["n_kv_branch"], 2),
            "fwd_order": arr(L["off_fwd_order"], n_qt),
            "bwd_order": arr(L["off_bwd_order"], n_kv),
            "key_iv": arr(L["off_key_iv"], rows, 4),
            "bwd_prefix": arr(L["off_bwd_prefix"], n_kv),
        }
        if c.zigzag_C > 1:
            out["zz_tiles"] = arr(L["off_zz_tiles"], c.zigzag_C * n_qt, 4).reshape(
                c.zigzag_C, n_qt, 4)
        return out
