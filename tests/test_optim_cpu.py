"""The Muon optimizer's construction on CPU (no kernel runs): routing of
parameters to the Muon and AdamW paths, semantic groups split into
<name>/muon and <name>/adamw, and the construction errors the training guide
describes (duplicate, missing or foreign parameters)."""
import pytest
import torch

from newton_schulz_09_b200 import Muon
from newton_schulz_09_b200.optim import route_names


class Tiny(torch.nn.Module):
    def __init__(self):
        super().__init__()
        self.embed_tokens = torch.nn.Embedding(32, 16)
        self.proj = torch.nn.Linear(16, 24)
        self.norm = torch.nn.LayerNorm(24)
        self.action_head = torch.nn.Linear(24, 8, bias=False)
        self.lm_head = torch.nn.Linear(24, 32, bias=False)


def _names(model, params):
    by_id = {id(p): n for n, p in model.named_parameters()}
    return sorted(by_id[id(p)] for p in params)


def test_default_routing():
    m = Tiny()
    opt = Muon(m, lr=0.02, adamw_lr=1e-3)
    assert list(route_names(opt)) == ["default/muon", "default/adamw"]
    muon, adamw = opt.param_groups
    assert _names(m, muon["params"]) == ["action_head.weight", "proj.weight"]
    assert _names(m, adamw["params"]) == ["embed_tokens.weight", "lm_head.weight", "norm.bias",
                                          "norm.weight", "proj.bias"]
    assert muon["lr"] == 0.02 and adamw["lr"] == 1e-3
    assert muon["weight_decay"] == 0.0 and adamw["weight_decay"] == 0.01
    assert muon["momentum"] == 0.95 and muon["nesterov"] and muon["ns_steps"] == 5


def test_semantic_groups():
    m = Tiny()
    action = [m.action_head.weight]
    base = [p for n, p in m.named_parameters() if not n.startswith("action_head")]
    opt = Muon(m, lr=5e-5, adamw_lr=5e-5, param_groups=[
        {"params": base, "lr": 5e-5, "group_name": "base"},
        {"params": action, "lr": 1e-4, "group_name": "action", "adamw_weight_decay": 0.0}])
    assert list(route_names(opt)) == ["base/muon", "base/adamw", "action/muon", "action/adamw"]
    g = {x["group_name"]: x for x in opt.param_groups}
    assert g["action/muon"]["lr"] == 1e-4 and _names(m, g["action/muon"]["params"]) == ["action_head.weight"]
    assert g["action/adamw"]["params"] == [] and g["action/adamw"]["weight_decay"] == 0.0
    assert g["base/adamw"]["lr"] == 5e-5
    # per-path overrides
    opt = Muon(m, param_groups=[{"params": list(m.parameters()), "group_name": "all", "muon_lr": 0.03,
                                 "adamw_lr": 2e-3, "muon_weight_decay": 0.1}])
    g = {x["group_name"]: x for x in opt.param_groups}
    assert g["all/muon"]["lr"] == 0.03 and g["all/adamw"]["lr"] == 2e-3 and g["all/muon"]["weight_decay"] == 0.1


def test_construction_errors():
    m = Tiny()
    ps = list(m.parameters())
    with pytest.raises(ValueError, match="more than one group"):
        Muon(m, param_groups=[{"params": ps, "group_name": "a"}, {"params": ps[:1], "group_name": "b"}])
    with pytest.raises(ValueError, match="in no group"):
        Muon(m, param_groups=[{"params": ps[1:], "group_name": "a"}])
    with pytest.raises(ValueError, match="not a trainable parameter"):
        Muon(m, param_groups=[{"params": ps + [torch.nn.Parameter(torch.zeros(3))], "group_name": "a"}])
    # frozen parameters are not managed
    m.norm.weight.requires_grad_(False)
    opt = Muon(m)
    assert all(p is not m.norm.weight for g in opt.param_groups for p in g["params"])
