"""A ``torch.optim`` optimizer with the DMuon training guide's interface
("第 4 步：创建优化器"): Muon for the matrix parameters and AdamW for the
others in one optimizer, on one GPU, each path one batched library call per
parameter group and step.

* Group routing: 2-D parameters take the Muon path; every other parameter,
  and matrices whose name ``adamw_filter`` accepts (by default embeddings and
  output heads, which Muon practice leaves to AdamW), take the AdamW path.
* Semantic groups (the guide's ``param_groups``, "语义参数组"): every user
  group ``name`` becomes two optimizer groups, ``name/muon`` and
  ``name/adamw``; each trainable parameter must appear in exactly one user
  group, or construction fails.
* Per-group keys the guide names: ``lr`` (both paths unless overridden),
  ``muon_lr``, ``adamw_lr``, ``weight_decay``/``muon_weight_decay``,
  ``adamw_weight_decay``, ``momentum``, ``adamw_betas``, ``adamw_eps``.

Everything runs in the library's kernels; this module only sorts parameters
and keeps their state (momentum buffers, AdamW moments and step counts) in
``self.state`` so that schedulers and ``state_dict`` work as for any
``torch.optim`` optimizer.
"""
from __future__ import annotations

from typing import Callable, Iterable, List, Optional

import torch

from . import dmuon_adamw_step_batched, dmuon_muon_step_batched_opts


def _default_adamw_filter(name: str) -> bool:
    n = name.lower()
    return "embed" in n or "lm_head" in n


class Muon(torch.optim.Optimizer):
    def __init__(self, model_or_params, lr: float = 0.02, momentum: float = 0.95, ns_steps: int = 5,
                 nesterov: bool = True, weight_decay: float = 0.0, adamw_lr: float = 1e-3,
                 adamw_betas=(0.9, 0.999), adamw_weight_decay: float = 0.01, adamw_eps: float = 1e-8,
                 param_groups: Optional[List[dict]] = None, ns_coefficients=(1.5, -0.5),
                 lr_scale: str = "plain", max_grad_norm: float = 0.0,
                 adamw_filter: Optional[Callable[[str], bool]] = None):
        adamw_filter = adamw_filter or _default_adamw_filter
        if isinstance(model_or_params, torch.nn.Module):
            named = [(n, p) for n, p in model_or_params.named_parameters() if p.requires_grad]
        else:
            named = [(f"param{i}", p) for i, p in enumerate(model_or_params) if p.requires_grad]
        names = {id(p): n for n, p in named}
        if len(names) != len(named):
            raise ValueError("a parameter appears twice")
        defaults = dict(lr=lr, momentum=momentum, nesterov=nesterov, weight_decay=weight_decay,
                        ns_steps=ns_steps, ns_coefficients=tuple(ns_coefficients), lr_scale=lr_scale,
                        adamw_betas=tuple(adamw_betas), adamw_eps=adamw_eps,
                        adamw_weight_decay=adamw_weight_decay, max_grad_norm=max_grad_norm)
        user_groups = param_groups if param_groups is not None else [
            {"params": [p for _, p in named], "group_name": "default", "lr": lr, "adamw_lr": adamw_lr}]
        seen = set()
        groups = []
        for ug in user_groups:
            ps = list(ug["params"])
            gname = ug.get("group_name", f"group{len(groups) // 2}")
            for p in ps:
                if id(p) not in names:
                    raise ValueError(f"group {gname!r}: a parameter that is not a trainable parameter "
                                     "of the model (an old or foreign tensor)")
                if id(p) in seen:
                    raise ValueError(f"group {gname!r}: parameter {names[id(p)]!r} is in more than one group")
                seen.add(id(p))
            muon = [p for p in ps if p.dim() == 2 and not adamw_filter(names[id(p)])]
            adamw = [p for p in ps if not (p.dim() == 2 and not adamw_filter(names[id(p)]))]
            glr = ug.get("lr", lr)
            common = {k: v for k, v in ug.items() if k not in ("params", "group_name")}
            groups.append(dict(common, params=muon, group_name=f"{gname}/muon", route="muon",
                               lr=ug.get("muon_lr", glr),
                               weight_decay=ug.get("muon_weight_decay", ug.get("weight_decay", weight_decay))))
            groups.append(dict(common, params=adamw, group_name=f"{gname}/adamw", route="adamw",
                               lr=ug.get("adamw_lr", glr if param_groups is not None else adamw_lr),
                               weight_decay=ug.get("adamw_weight_decay", adamw_weight_decay)))
        missing = [names[id(p)] for _, p in named if id(p) not in seen]
        if missing:
            raise ValueError(f"trainable parameters in no group: {missing[:5]}")
        for g in groups:
            g.setdefault("momentum", momentum)
        super().__init__(groups, defaults)

    def load_state_dict(self, state_dict) -> None:
        """As torch.optim's, except that the momentum buffers and AdamW
        moments stay fp32 (the base class would cast them to each
        parameter's dtype, e.g. bf16, and lose bits)."""
        super().load_state_dict(state_dict)
        saved = state_dict["state"]
        for g, sg in zip(self.param_groups, state_dict["param_groups"]):
            for p, pid in zip(g["params"], sg["params"]):
                for k, v in saved.get(pid, {}).items():
                    if torch.is_tensor(v) and k != "step":
                        self.state[p][k] = v.to(device=p.device, dtype=torch.float32).clone()

    @torch.no_grad()
    def step(self, closure=None):
        loss = None
        if closure is not None:
            with torch.enable_grad():
                loss = closure()
        for g in self.param_groups:
            ps = [p for p in g["params"] if p.grad is not None]
            if not ps:
                continue
            if g["route"] == "muon":
                bufs = []
                for p in ps:
                    st = self.state[p]
                    if "momentum_buffer" not in st:
                        st["momentum_buffer"] = torch.zeros(p.shape, dtype=torch.float32, device=p.device)
                    bufs.append(st["momentum_buffer"])
                dmuon_muon_step_batched_opts(
                    ps, [p.grad for p in ps], bufs, lr=g["lr"], momentum=g["momentum"],
                    nesterov=g["nesterov"], weight_decay=g["weight_decay"], ns_steps=g["ns_steps"],
                    ns_coefficients=g["ns_coefficients"], lr_scale=g["lr_scale"],
                    max_grad_norm=g["max_grad_norm"])
            else:
                ms, vs = [], []
                for p in ps:
                    st = self.state[p]
                    if "exp_avg" not in st:
                        st["exp_avg"] = torch.zeros(p.shape, dtype=torch.float32, device=p.device)
                        st["exp_avg_sq"] = torch.zeros(p.shape, dtype=torch.float32, device=p.device)
                        st["step"] = 0
                    ms.append(st["exp_avg"])
                    vs.append(st["exp_avg_sq"])
                # one call per distinct step count (parameters that joined later)
                by_step: dict = {}
                for p, m, v in zip(ps, ms, vs):
                    self.state[p]["step"] += 1
                    by_step.setdefault(self.state[p]["step"], []).append((p, m, v))
                for step, items in sorted(by_step.items()):
                    dmuon_adamw_step_batched([p for p, _, _ in items], [p.grad for p, _, _ in items],
                                             [m for _, m, _ in items], [v for _, _, v in items],
                                             lr=g["lr"], betas=g["adamw_betas"], eps=g["adamw_eps"],
                                             weight_decay=g["weight_decay"], step=step)
        return loss


def route_names(opt: Muon) -> Iterable[str]:
    """The optimizer's group names, e.g. ``base/muon``, ``base/adamw``."""
    return [g["group_name"] for g in opt.param_groups]
