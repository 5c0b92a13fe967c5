"""The optimizer step overlapped with a (synthetic) backward pass, group by group.

Gradients are produced on the main stream group after group, as a backward
pass would; each group's step starts on a side stream as soon as its
gradients are final. The result must be exactly one plain call of the
library on every bank with the same gradients, eagerly and replayed from a
CUDA graph that holds the backward pass and the overlapped step together.
The first (eager) overlapped step is also checked against the CPU oracle:
every momentum element, the parameter step of sampled matrices and, with
fp32 parameters, the orthogonalised update and its singular values.
"""
import pytest
import torch

from _oracle_checks import check_anvil_step, check_muon_step, hp_dict

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
SHAPES = [(4, 768, 768), (2, 768, 3072), (2, 3072, 768), (3, 512, 1024)]
GROUPS = [[3], [1, 2], [0]]          # the order the backward pass finishes them


def _setup(seed, dtype):
    g = torch.Generator(device=DEV).manual_seed(seed)
    params = [(torch.randn(c, r, k, generator=g, device=DEV) * 0.02).to(dtype)
              for c, r, k in SHAPES]
    # per bank: activations and output gradients whose product is the weight gradient
    acts = [(torch.randn(c, 64, r, generator=g, device=DEV), torch.randn(c, 64, k, generator=g, device=DEV))
            for c, r, k in SHAPES]
    return params, acts


def _grad(acts, b, out):
    x, dy = acts[b]
    torch.bmm(x.transpose(1, 2), dy, out=out)   # [c, r, k] = x^T dy


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("variant", ["muon", "anvil"])
def test_overlapped_step_equals_one_call_eager_and_in_a_graph(variant, dtype):
    import muon_newton_schulz_05_b200 as mb
    from muon_newton_schulz_05_b200.overlap import OverlappedStep
    if variant == "anvil":
        hp = mb.Hparams(lr=0.05, weight_decay=0.1, coeffs=[(3.4445, -4.7750, 2.0315)] * 6,
                        beta_fast=0.9, beta_slow=0.99)
    else:
        hp = mb.Hparams(lr=0.02, mu=0.95, weight_decay=0.01, nesterov=True)
    step_fn = mb.anvil_step if variant == "anvil" else mb.muon_step

    def banks_for(params, grads):
        out = []
        for p, gr in zip(params, grads):
            m = torch.zeros(p.shape, device=DEV)
            out.append(mb.Bank(p, gr, m, torch.zeros_like(m) if variant == "anvil" else None))
        return out

    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    params, acts = _setup(5, tdt)
    params0 = [p.clone() for p in params]
    grads = [torch.empty(c, r, k, device=DEV) for c, r, k in SHAPES]
    banks = banks_for(params, grads)
    ov = OverlappedStep([[banks[b] for b in grp] for grp in GROUPS], hp, variant=variant)

    def train_step():
        for grp in GROUPS:            # the backward pass, group after group
            for b in grp:
                _grad(acts, b, grads[b])
            ov.grad_ready(GROUPS.index(grp))
        ov.wait()

    # reference: the same gradients, one plain call over every bank
    r_params = [p.clone() for p in params]
    r_grads = [torch.empty_like(g) for g in grads]
    r_banks = banks_for(r_params, r_grads)
    r_ws = mb.alloc_workspace([b.shape for b in r_banks])

    def ref_step():
        for b in range(len(SHAPES)):
            _grad(acts, b, r_grads[b])
        step_fn(r_banks, hp, r_ws)

    train_step()                      # eager
    ref_step()
    torch.cuda.synchronize()
    assert ov.device_status() == 0 and mb.device_status(r_ws) == 0
    for a, r in zip(banks, r_banks):
        assert torch.equal(a.param, r.param)
        assert torch.equal(a.momentum, r.momentum)
    # the first step against the oracle (zero momenta before it)
    ohp = hp_dict(hp)
    for b, bk in enumerate(banks):
        picks = [0, SHAPES[b][0] - 1]
        zero = torch.zeros(bk.momentum.shape)
        if variant == "anvil":
            check_anvil_step(params0[b], bk.param, grads[b], zero, bk.momentum, zero,
                             bk.momentum_slow, ohp, picks, dtype)
        else:
            check_muon_step(params0[b], bk.param, grads[b], zero, bk.momentum, ohp, picks, dtype)

    graph = torch.cuda.CUDAGraph()    # backward + overlapped step in one graph
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        graph.capture_begin()
        train_step()
        graph.capture_end()
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(2):
        graph.replay()
        ref_step()
    torch.cuda.synchronize()
    assert ov.device_status() == 0
    for a, r in zip(banks, r_banks):
        assert torch.equal(a.param, r.param)
        assert torch.equal(a.momentum, r.momentum)
        if variant == "anvil":
            assert torch.equal(a.momentum_slow, r.momentum_slow)


def test_overlapped_step_rejects_misuse():
    import muon_newton_schulz_05_b200 as mb
    from muon_newton_schulz_05_b200.overlap import OverlappedStep
    p = torch.zeros(1, 256, 256, dtype=torch.bfloat16, device=DEV)
    bank = mb.Bank(p, torch.zeros_like(p), torch.zeros(1, 256, 256, device=DEV))
    with pytest.raises(ValueError):
        OverlappedStep([[]], mb.Hparams())
    ov = OverlappedStep([[bank]], mb.Hparams())
    with pytest.raises(RuntimeError):
        ov.wait()                     # group 0 was never stepped
    ov.grad_ready(0)
    with pytest.raises(RuntimeError):
        ov.grad_ready(0)              # twice in one step
    ov.wait()
    assert ov.device_status() == 0
