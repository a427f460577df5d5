"""ZeroAdamW on a small bf16 model: autograd writes into the plan's gradient
buffer through the .grad views, the step writes the model's parameters
through the parameter buffer, and three steps equal the oracle's step on
the same gradients (fp32 state bit for bit, bf16 parameters within 1 ulp)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_harness import DEV, assert_state_close, bf16_ulp_distance, bits32
from sharded_optimizer_step_zr_b200.optim import ZeroAdamW

pytestmark = pytest.mark.gpu


def make_model(seed):
    torch.manual_seed(seed)
    return torch.nn.Sequential(torch.nn.Linear(64, 128), torch.nn.GELU(), torch.nn.Linear(128, 24),
                               torch.nn.LayerNorm(24)).to(DEV).to(torch.bfloat16)


def flat_u16(tensors):
    return torch.cat([t.detach().reshape(-1) for t in tensors]).cpu().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("partition, clip, overlap", [("flat", 0.0, False), ("whole", 1.0, False),
                                                     ("flat", 0.0, True), ("whole", 1.0, True),
                                                     ("flat", 0.05, True)])
def test_zero_adamw_one_rank_matches_the_oracle(partition, clip, overlap):
    """overlap=True steps each 10 KB bucket on a side stream as the backward
    fills it (the rest of the backward runs beside it): the same steps."""
    model = make_model(5)
    params = list(model.parameters())
    hp = (1e-3, 0.9, 0.999, 1e-8, 0.1, clip)
    init = flat_u16(params)
    opt = ZeroAdamW(params, lr=hp[0], betas=hp[1:3], eps=hp[3], weight_decay=hp[4], max_grad_norm=clip,
                    partition=partition, bucket_cap_mb=0.01, overlap=overlap)
    if overlap:
        assert opt.plan.n_buckets >= 2
    assert np.array_equal(flat_u16(params), init)          # rebinding kept the values
    N = init.size
    o_master = (init.astype(np.uint32) << 16).view(np.float32)      # bf16 -> fp32 is exact
    o_m, o_v = np.zeros(N, np.float32), np.zeros(N, np.float32)
    o_out = np.zeros(N, np.uint16)
    gen = torch.Generator(device=DEV).manual_seed(11)
    lo, hi = opt.grad_buffer.data_ptr(), opt.grad_buffer.data_ptr() + 2 * opt.grad_buffer.numel()
    for t in (1, 2, 3):
        x = torch.randn(32, 64, device=DEV, generator=gen).to(torch.bfloat16)
        loss = model(x).float().pow(2).mean()
        loss.backward()
        for p in params:                                      # autograd wrote into the buffer
            assert lo <= p.grad.data_ptr() < hi
        grads = flat_u16([p.grad for p in params])
        c = None
        if clip > 0:
            g = oracle.reduce([grads])
            c = oracle.clip_coef(oracle.sumsq(g), clip)
        oracle.ddp_step([grads], o_master, o_m, o_v, o_out, hp, t, clip=c)
        opt.step()
        opt.zero_grad()
        torch.cuda.synchronize()
        got = flat_u16(params)
        assert bf16_ulp_distance(got, o_out).max() <= 1, t
        if clip == 0:
            assert np.array_equal(got, o_out), t
            # one rank: owned order is the global order
            assert np.array_equal(bits32(opt.master[:N].cpu().numpy()), bits32(o_master))
    opt.close()


def test_zero_adamw_save_and_resume(tmp_path):
    """Two steps, save, a fresh model and optimizer loaded from the shard,
    a third step: equal to three uninterrupted steps bit for bit."""
    import os

    def batches():
        gen = torch.Generator(device=DEV).manual_seed(7)
        return [torch.randn(32, 64, device=DEV, generator=gen).to(torch.bfloat16) for _ in range(3)]

    xs = batches()
    ref_model = make_model(3)
    ref = ZeroAdamW(list(ref_model.parameters()), lr=1e-3)
    for x in xs:
        ref_model(x).float().pow(2).mean().backward()
        ref.step()
        ref.zero_grad()
    model = make_model(3)
    opt = ZeroAdamW(list(model.parameters()), lr=1e-3)
    for x in xs[:2]:
        model(x).float().pow(2).mean().backward()
        opt.step()
        opt.zero_grad()
    path = os.path.join(str(tmp_path), "rank0.zrs")
    opt.save(path)
    model2 = make_model(99)                                   # other initial weights: replaced by the load
    opt2 = ZeroAdamW(list(model2.parameters()), lr=1e-3)
    opt2.load(path)
    assert opt2.step_count == 2
    model2(xs[2]).float().pow(2).mean().backward()
    opt2.step()
    torch.cuda.synchronize()
    assert np.array_equal(flat_u16(model2.parameters()), flat_u16(ref_model.parameters()))
    for a, b in ((opt2.master, ref.master), (opt2.m, ref.m), (opt2.v, ref.v)):
        assert np.array_equal(bits32(a.cpu().numpy()), bits32(b.cpu().numpy()))
    for o in (ref, opt, opt2):
        o.close()


def make_deep_model(seed):
    torch.manual_seed(seed)
    return torch.nn.Sequential(torch.nn.Linear(64, 128), torch.nn.GELU(), torch.nn.Linear(128, 128), torch.nn.GELU(),
                               torch.nn.Linear(128, 96), torch.nn.LayerNorm(96), torch.nn.Linear(96, 24)
                               ).to(DEV).to(torch.bfloat16)


@pytest.mark.parametrize("partition", ["flat", "whole"])
def test_zero3_trains_like_zero_adamw(partition):
    """Zero3 (each module's parameters gathered from the shard before its
    forward and again before its backward, two rotating slots) takes the
    same steps as ZeroAdamW with every parameter resident: after each of
    three steps the gathered model equals the other one bit for bit, and so
    do the losses."""
    from sharded_optimizer_step_zr_b200.optim import Zero3
    a, b = make_deep_model(8), make_deep_model(8)
    z2 = ZeroAdamW(list(a.parameters()), lr=1e-3, partition=partition)
    z3 = Zero3(b, lr=1e-3, partition=partition)
    N = sum(p.numel() for p in a.parameters())
    big = max(sum(p.numel() for p in m.parameters(recurse=False)) for m in b.modules())
    assert all(s.numel() == max(big, 8) for s in z3.slots)          # two slots of the largest module
    gen = torch.Generator(device=DEV).manual_seed(21)
    for t in (1, 2, 3):
        x = torch.randn(32, 64, device=DEV, generator=gen).to(torch.bfloat16)
        la = a(x).float().pow(2).mean()
        la.backward()
        z2.step()
        z2.zero_grad()
        lb = b(x).float().pow(2).mean()
        lb.backward()
        z3.step()
        z3.zero_grad()
        torch.cuda.synchronize()
        assert la.item() == lb.item(), t
        full = torch.empty(N, dtype=torch.bfloat16, device=DEV)
        z3.gather_all(full)
        torch.cuda.synchronize()
        assert np.array_equal(full.cpu().view(torch.int16).numpy(), flat_u16(a.parameters()).view(np.int16)), t
    z2.close()
    z3.close()


def test_zero3_save_and_resume(tmp_path):
    import os
    from sharded_optimizer_step_zr_b200.optim import Zero3
    gen = torch.Generator(device=DEV).manual_seed(9)
    xs = [torch.randn(32, 64, device=DEV, generator=gen).to(torch.bfloat16) for _ in range(3)]
    ref_model = make_deep_model(4)
    ref = Zero3(ref_model, lr=1e-3)
    for x in xs:
        ref_model(x).float().pow(2).mean().backward()
        ref.step()
        ref.zero_grad()
    model = make_deep_model(4)
    z = Zero3(model, lr=1e-3)
    for x in xs[:2]:
        model(x).float().pow(2).mean().backward()
        z.step()
        z.zero_grad()
    path = os.path.join(str(tmp_path), "z3_rank0.zrs")
    z.save(path)
    model2 = make_deep_model(77)
    z2 = Zero3(model2, lr=1e-3)
    z2.load(path)
    model2(xs[2]).float().pow(2).mean().backward()
    z2.step()
    N = sum(p.numel() for p in ref_model.parameters())
    a = torch.empty(N, dtype=torch.bfloat16, device=DEV)
    b = torch.empty(N, dtype=torch.bfloat16, device=DEV)
    ref.gather_all(a)
    z2.gather_all(b)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    for o in (ref, z, z2):
        o.close()


def test_zero3_accumulation_and_evaluation():
    """Two forward / backward passes per step (gradient accumulation) and a
    no-grad evaluation forward between steps: Zero3's hooks gather for every
    pass, and the steps equal ZeroAdamW's bit for bit."""
    from sharded_optimizer_step_zr_b200.optim import Zero3
    a, b = make_deep_model(12), make_deep_model(12)
    z2 = ZeroAdamW(list(a.parameters()), lr=1e-3)
    z3 = Zero3(b, lr=1e-3)
    gen = torch.Generator(device=DEV).manual_seed(5)
    N = sum(p.numel() for p in a.parameters())
    for t in (1, 2):
        xs = [torch.randn(16, 64, device=DEV, generator=gen).to(torch.bfloat16) for _ in range(3)]
        for m, opt in ((a, z2), (b, z3)):
            for x in xs[:2]:
                m(x).float().pow(2).mean().backward()
            opt.step()
            opt.zero_grad()
        with torch.no_grad():
            ea, eb = a(xs[2]), b(xs[2])
        torch.cuda.synchronize()
        assert torch.equal(ea.view(torch.int16), eb.view(torch.int16)), t
        full = torch.empty(N, dtype=torch.bfloat16, device=DEV)
        z3.gather_all(full)
        torch.cuda.synchronize()
        assert np.array_equal(full.cpu().view(torch.int16).numpy(), flat_u16(a.parameters()).view(np.int16)), t
    z2.close()
    z3.close()


@pytest.mark.parametrize("partition", ["flat", "whole"])
def test_zero3_reduce_in_backward_with_clipping(partition):
    """reduce_in_backward with a global-norm clip small enough to bite: the
    backward's per-module calls reduce and sum the squares (the fp32
    averaged gradient kept), step() applies the clipped update.  The
    modules' buckets cut the tiles differently from the byte-cap plan, so
    the norm's fp64 sum runs in another order: the parameters equal
    ordinary Zero3's within 1 bf16 ulp over three steps, not bit for bit."""
    from sharded_optimizer_step_zr_b200.optim import Zero3
    a, b = make_deep_model(9), make_deep_model(9)
    za = Zero3(a, lr=1e-3, partition=partition, max_grad_norm=0.01)
    zb = Zero3(b, lr=1e-3, partition=partition, max_grad_norm=0.01, reduce_in_backward=True)
    N = sum(p.numel() for p in a.parameters())
    gen = torch.Generator(device=DEV).manual_seed(29)
    for t in (1, 2, 3):
        x = torch.randn(32, 64, device=DEV, generator=gen).to(torch.bfloat16)
        a(x).float().pow(2).mean().backward()
        za.step()
        za.zero_grad()
        b(x).float().pow(2).mean().backward()
        zb.step()
        torch.cuda.synchronize()
        assert all(not s_.view(torch.int16).any() for s_ in zb.grad_slots)
        fa = torch.empty(N, dtype=torch.bfloat16, device=DEV)
        fb = torch.empty(N, dtype=torch.bfloat16, device=DEV)
        za.gather_all(fa)
        zb.gather_all(fb)
        torch.cuda.synchronize()
        ua = fa.cpu().view(torch.int16).numpy().view(np.uint16)
        ub = fb.cpu().view(torch.int16).numpy().view(np.uint16)
        assert bf16_ulp_distance(ua, ub).max() <= 1, t
        assert_state_close(zb.master[:zb.plan.owned_numel].cpu().numpy(),
                           za.master[:za.plan.owned_numel].cpu().numpy(), f"master step {t}")
    # the clip did bite: the coefficient is below 1
    S = float(zb.plan.partials.sum().item())
    assert 0.01 / (S ** 0.5 + 1e-6) < 1.0
    za.close()
    zb.close()


@pytest.mark.parametrize("partition", ["flat", "whole"])
def test_zero3_reduce_in_backward_takes_the_same_steps(partition):
    """The gradient side of stage 3: each module's gradients accumulate into
    one of two rotating slots and are reduced and applied (zr_step_bucket on
    the module's bucket) as soon as the module's backward is done; no
    full-model gradient buffer exists.  Three steps equal Zero3's ordinary
    step (and so ZeroAdamW's) bit for bit, weights and losses; a second
    backward before step() is refused."""
    from sharded_optimizer_step_zr_b200.optim import Zero3
    a, b = make_deep_model(8), make_deep_model(8)
    za = Zero3(a, lr=1e-3, partition=partition)
    zb = Zero3(b, lr=1e-3, partition=partition, reduce_in_backward=True)
    assert zb.grad_buffer is None and len(zb.grad_slots) == 2
    big = max(sum(p.numel() for p in m.parameters(recurse=False)) for m in b.modules())
    assert all(s.numel() <= big + 8 for s in zb.grad_slots)     # one module's gradients per slot
    N = sum(p.numel() for p in a.parameters())
    gen = torch.Generator(device=DEV).manual_seed(23)
    for t in (1, 2, 3):
        x = torch.randn(32, 64, device=DEV, generator=gen).to(torch.bfloat16)
        la = a(x).float().pow(2).mean()
        la.backward()
        za.step()
        za.zero_grad()
        lb = b(x).float().pow(2).mean()
        lb.backward()
        zb.step()
        zb.zero_grad()
        torch.cuda.synchronize()
        assert la.item() == lb.item(), t
        fa = torch.empty(N, dtype=torch.bfloat16, device=DEV)
        fb = torch.empty(N, dtype=torch.bfloat16, device=DEV)
        za.gather_all(fa)
        zb.gather_all(fb)
        torch.cuda.synchronize()
        assert torch.equal(fa.view(torch.int16), fb.view(torch.int16)), t
        assert all(not s.view(torch.int16).any() for s in zb.grad_slots)   # cleared after every module
    x = torch.randn(32, 64, device=DEV, generator=gen).to(torch.bfloat16)
    b(x).float().pow(2).mean().backward()
    with pytest.raises(RuntimeError, match="second backward"):
        b(x).float().pow(2).mean().backward()
    za.close()
    zb.close()
