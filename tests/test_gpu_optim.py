"""The Muon optimizer on a B200: its steps equal the direct batched calls bit
for bit (Muon for the matrices, AdamW for the rest), a learning-rate
scheduler reaches both paths, and state_dict / load_state_dict resume."""
import copy

import pytest
import torch

from tests.test_optim_cpu import Tiny

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _set_grads(model, step):
    g = torch.Generator(device=DEV)
    g.manual_seed(100 + step)
    for p in model.parameters():
        p.grad = (torch.randn(p.shape, generator=g, device=DEV) * 1e-3).to(p.dtype)


def _split(model):
    muon = [model.proj.weight, model.action_head.weight]
    adamw = [model.embed_tokens.weight, model.proj.bias, model.norm.weight, model.norm.bias,
             model.lm_head.weight]
    return muon, adamw


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
def test_optimizer_equals_direct_calls(cuda_lib, dtype):
    dm = cuda_lib
    torch.manual_seed(0)
    m = Tiny().to(DEV, dtype)
    ref = copy.deepcopy(m)
    opt = dm.Muon(m, lr=0.02, weight_decay=0.01, adamw_lr=1e-3, adamw_weight_decay=0.01)
    sched = torch.optim.lr_scheduler.LambdaLR(opt, lambda e: 0.5 ** e)
    rm, ra = _split(ref)
    bufs = [torch.zeros(p.shape, dtype=torch.float32, device=DEV) for p in rm]
    ms = [torch.zeros(p.shape, dtype=torch.float32, device=DEV) for p in ra]
    vs = [torch.zeros(p.shape, dtype=torch.float32, device=DEV) for p in ra]
    for step in range(1, 4):
        _set_grads(m, step)
        _set_grads(ref, step)
        opt.step()
        scale = 0.5 ** (step - 1)
        dm.dmuon_muon_step_batched_opts(rm, [p.grad for p in rm], bufs, lr=0.02 * scale, weight_decay=0.01)
        dm.dmuon_adamw_step_batched(ra, [p.grad for p in ra], ms, vs, lr=1e-3 * scale, betas=(0.9, 0.999),
                                    eps=1e-8, weight_decay=0.01, step=step)
        sched.step()
        torch.cuda.synchronize()
        for (n, a), b in zip(m.named_parameters(), ref.parameters()):
            assert torch.equal(a, b), (step, n)
    assert dm.dmuon_device_status() == 0


def test_state_dict_resume(cuda_lib):
    dm = cuda_lib
    torch.manual_seed(1)
    m = Tiny().to(DEV, torch.bfloat16)
    m2 = copy.deepcopy(m)
    opt = dm.Muon(m)
    _set_grads(m, 1)
    opt.step()
    saved = copy.deepcopy(opt.state_dict())
    m2.load_state_dict(m.state_dict())
    opt2 = dm.Muon(m2)
    opt2.load_state_dict(saved)
    for step in (2, 3):
        _set_grads(m, step)
        _set_grads(m2, step)
        opt.step()
        opt2.step()
    torch.cuda.synchronize()
    for a, b in zip(m.parameters(), m2.parameters()):
        assert torch.equal(a, b)
