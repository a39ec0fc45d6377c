"""GPU tests of the two halves of a step whose update is exchanged in bf16:
muon_update_bf16 (momentum and NS5, O rounded to bf16, W untouched) against
the oracle and against the fp32 step's own O, and muon_apply_bf16 (W -= lr*O)
against the same arithmetic on the host."""

import numpy as np
import pytest
import torch

import muon_newton_schulz_02_b200 as muon
from oracle import muon_oracle

from gpu_helpers import REL_BUF, check_o, o_from_w, relF

pytestmark = pytest.mark.gpu

# every path: fused single-CTA (128x512), CTA pair (200x256), chained launch,
# one launch per phase (1100x2000), ragged and odd element counts
SHAPES = [(128, 512), (200, 256), (768, 3072), (3072, 768), (300, 701), (1100, 2000), (5, 3)]


@pytest.fixture(scope="module", autouse=True)
def _built():
    import __graft_entry__
    __graft_entry__.build()


def _inputs(seed=11):
    gen = torch.Generator().manual_seed(seed)
    W = [(torch.randn(*s, generator=gen) * 0.02) for s in SHAPES]
    g = [torch.randn(*s, generator=gen) for s in SHAPES]
    b = [(torch.randn(*s, generator=gen) * 0.1) for s in SHAPES]
    return W, g, b


def test_update_bf16_matches_the_oracle_and_the_fp32_step():
    dev = torch.device("cuda:0")
    W, g, b = _inputs()
    gd = [x.to(dev) for x in g]
    bd = [x.to(dev) for x in b]
    O = muon.update_bf16(gd, bd, 0.95)
    torch.cuda.synchronize()
    assert muon.sync_status() == 0, muon.last_error()
    # the fp32 step on the same inputs: its O rounded to bf16 must be the same bits
    Wd = [x.to(dev) for x in W]
    bd2 = [x.to(dev) for x in b]
    muon.step(Wd, gd, bd2, lr=1.0, mu=0.95)
    torch.cuda.synchronize()
    for i, s in enumerate(SHAPES):
        assert O[i].dtype == torch.bfloat16 and tuple(O[i].shape) == s
        assert torch.equal(bd[i], bd2[i])
        Oh = O[i].float().cpu().numpy()
        _, b_ref, O_ref = muon_oracle.muon_update(W[i].numpy(), g[i].numpy(), b[i].numpy(), 0.02, 0.95)
        check_o(Oh, O_ref, f"{s}")
        assert relF(bd[i].cpu().numpy(), b_ref) <= REL_BUF
        # W - 1*O from the fp32 step carries O to within the rounding of W's subtraction
        O32 = o_from_w(W[i].numpy(), Wd[i].cpu().numpy(), 1.0)
        assert relF(Oh, O32) < 5e-3, s


def test_apply_bf16_is_one_fused_multiply_add():
    dev = torch.device("cuda:0")
    gen = torch.Generator().manual_seed(12)
    shapes = SHAPES + [(1, 1), (3, 8), (64, 64)]
    W = [torch.randn(*s, generator=gen) for s in shapes]
    O = [torch.randn(*s, generator=gen).to(torch.bfloat16) for s in shapes]
    Wd = [x.to(dev) for x in W]
    muon.apply_bf16(Wd, [o.to(dev) for o in O], 0.02)
    torch.cuda.synchronize()
    lr = np.float64(np.float32(0.02))
    for i in range(len(shapes)):
        exact = W[i].double().numpy() - lr * O[i].double().numpy()      # then one rounding to fp32
        got = Wd[i].cpu().numpy()
        assert np.array_equal(got, exact.astype(np.float32)) or \
            np.max(np.abs(got - exact) / np.maximum(np.abs(exact), 1e-30)) < 1.2e-7, shapes[i]


def test_misaligned_bf16_views_take_the_scalar_path():
    dev = torch.device("cuda:0")
    gen = torch.Generator().manual_seed(13)
    W = torch.randn(64, 96, generator=gen)
    flat = torch.randn(64 * 96 + 1, generator=gen).to(torch.bfloat16)
    O = flat[1:].view(64, 96)                                  # 2-byte offset: not 16-byte aligned
    Wd = W.to(dev)
    muon.apply_bf16([Wd], [flat.to(dev)[1:].view(64, 96)], 0.5)
    torch.cuda.synchronize()
    exact = (W.double() - 0.5 * O.double()).float()
    assert torch.allclose(Wd.cpu(), exact, rtol=2e-7, atol=0)


def test_rejects_fp32_updates():
    dev = torch.device("cuda:0")
    W = [torch.zeros(8, 8, device=dev)]
    with pytest.raises(ValueError):
        muon.apply_bf16(W, [torch.zeros(8, 8, device=dev)], 0.1)
