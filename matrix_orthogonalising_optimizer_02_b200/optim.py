"""torch.optim front-ends over the C ABI (argument marshalling only).

``Muon`` mirrors the constructor of the ``Muon`` class on the "Muon优化器" page
(linsight.cn/f25d614e.html, "Muon 算法伪代码与 PyTorch 实现"): lr, momentum,
weight_decay, nesterov, ns_steps, scale_mode.  ``MuonCayley`` mirrors the optimizer of
the Stiefel-manifold page (mlqm.cn/news/1339166, §4.3) for its Cayley branch.  Both hand
every matrix of a parameter group to one library call per step; grouping parameters
into Muon matrices and AdamW tensors stays with the caller, as the pages advise, so
these classes accept 2-D parameters only.
"""
from __future__ import annotations

import torch

from . import binding as mb

KJ_COEFFS = (3.4445, -4.7750, 2.0315)


def _check_matrix(p):
    if p.dim() != 2:
        raise ValueError(f"Muon handles 2-D weight matrices only, got shape {tuple(p.shape)}; "
                         "give embeddings, heads, biases and norms to AdamW")
    if p.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError(f"unsupported parameter dtype {p.dtype}")


class _Workspaces:
    """One workspace per device, grown to the largest request: the library's calls are
    ordered on the current stream, so successive calls can share it."""

    def __init__(self):
        self.bufs = {}

    def get(self, nbytes, device):
        ws = self.bufs.get(device)
        if ws is None or ws.numel() < nbytes:
            ws = mb.workspace(nbytes, device=device)
            self.bufs[device] = ws
        return ws


class Muon(torch.optim.Optimizer):
    """Momentum orthogonalised by Newton-Schulz, one grouped CUDA step per param group."""

    def __init__(self, params, lr=1e-3, momentum=0.95, weight_decay=0.01, nesterov=True, ns_steps=5,
                 scale_mode="moonlight", coeffs=None, n_split_iters=0, fp32_mode=False, eps=1e-7):
        if scale_mode not in mb.SCALE_MODES:
            raise ValueError(f"scale_mode must be one of {sorted(mb.SCALE_MODES)}")
        defaults = dict(lr=lr, momentum=momentum, weight_decay=weight_decay, nesterov=nesterov, ns_steps=ns_steps,
                        scale_mode=scale_mode, coeffs=coeffs, n_split_iters=n_split_iters, fp32_mode=fp32_mode,
                        eps=eps)
        super().__init__(params, defaults)
        for g in self.param_groups:
            for p in g["params"]:
                _check_matrix(p)
        self._ws = _Workspaces()

    @torch.no_grad()
    def step(self, closure=None):
        loss = None
        if closure is not None:
            with torch.enable_grad():
                loss = closure()
        for group in self.param_groups:
            mats = []
            for p in group["params"]:
                if p.grad is None:
                    continue
                state = self.state[p]
                if "momentum_buffer" not in state:
                    state["momentum_buffer"] = torch.zeros(p.shape, dtype=torch.float32, device=p.device)
                mats.append(mb.Matrix(p.data, p.grad.contiguous(), state["momentum_buffer"]))
            if not mats:
                continue
            coeffs = group["coeffs"] or [KJ_COEFFS] * group["ns_steps"]
            sch = mb.Schedule(coeffs, n_split_iters=group["n_split_iters"], fp32_mode=group["fp32_mode"],
                              eps=group["eps"])
            hp = mb.hyper(group["lr"], group["momentum"], group["weight_decay"], group["nesterov"],
                          group["scale_mode"], sch)
            ws = self._ws.get(mb.muon_step_workspace_size(mats, hp), mats[0].W.device)
            mb.muon_step_batched(mats, hp, ws)
        return loss


class MuonCayley(torch.optim.Optimizer):
    """Stiefel-manifold Muon: EMA momentum, column centering, tangent projection and the
    Cayley retraction in Woodbury form.  Parameters are fp32 and orthonormal along their
    shorter side: a tall n x k parameter has orthonormal columns, a wide one orthonormal
    rows and is updated as its transpose inside the library (page §4.4)."""

    def __init__(self, params, lr=3e-3, momentum=0.9, center=True):
        super().__init__(params, dict(lr=lr, momentum=momentum, center=center))
        for g in self.param_groups:
            for p in g["params"]:
                _check_matrix(p)
                if p.dtype != torch.float32:
                    raise ValueError("MuonCayley needs fp32 parameters")
        self._ws = _Workspaces()

    @torch.no_grad()
    def step(self, closure=None):
        loss = None
        if closure is not None:
            with torch.enable_grad():
                loss = closure()
        for group in self.param_groups:
            for p in group["params"]:
                if p.grad is None:
                    continue
                state = self.state[p]
                if "momentum_buffer" not in state:
                    state["momentum_buffer"] = torch.zeros_like(p)
                n, k = p.shape
                ws = self._ws.get(mb.muon_cayley_workspace_size(1, n, k), p.device)
                mb.muon_cayley_step(p.data, p.grad.contiguous(), state["momentum_buffer"], group["lr"],
                                    group["momentum"], ws, center=group["center"])
        return loss
