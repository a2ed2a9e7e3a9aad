"""The autograd wrapper ``sinkhorn_attention``: it appends the dustbin token and the inactive
fillers ("Blockwise Differentiable Sinkhorn Attention" §2.3), runs the forward and the exact
tail adjoint through the C ABI (§2.1-§2.2), slices the real rows out of O, and folds the
per-batch dustbin gradients back onto the learned per-head dustbin parameters.  Checked
against the float64 oracle on the extended problem, through ``.backward()``."""
import numpy as np
import pytest

import eot_inputs
from harness import TOL, oracle_run, rel_err

pytestmark = pytest.mark.gpu


def _ragged(B, N, seed):
    rng = np.random.default_rng(seed)
    lengths = rng.integers(N // 2, N, size=B, endpoint=True)
    return (np.arange(N)[None, :] < lengths[:, None]).astype(np.uint8)


@pytest.mark.parametrize("with_dustbin", [True, False])
def test_sinkhorn_attention_autograd_matches_oracle(with_dustbin):
    import torch
    from entropic_ot_attention_b200 import sinkhorn_attention
    B, H, N, d, W, T, R = 2, 3, 200, 64, 48, 6, 2
    mask = _ragged(B, N, 5)
    if with_dustbin:
        case = eot_inputs.dustbin_case(B, H, N, d, W, T, R, "bf16", seed=31, mass=0.1, mask=mask,
                                       name="autograd_dustbin")
    else:
        L = 256
        full = np.zeros((B, L), np.uint8)
        full[:, :N] = mask
        case = eot_inputs.dense_case(B, H, L, d, W, T, R, "bf16", seed=32, mask=full, name="autograd_plain")
    dev = torch.device("cuda:0")
    as_t = lambda x, grad=True: torch.tensor(x, dtype=torch.bfloat16, device=dev, requires_grad=grad)
    q, k, v = (as_t(x[:, :, :N]) for x in (case.Q, case.K, case.V))
    dO = as_t(case.dO[:, :, :N], grad=False)
    m = torch.from_numpy(mask).to(dev)
    dustbin = None
    if with_dustbin:
        dustbin = tuple(as_t(x[0, :, N]) for x in (case.Q, case.K, case.V))
    O = sinkhorn_attention(q, k, v, W, T, R, mask=m, dustbin=dustbin, dustbin_mass=0.1)
    (O.float() * dO.float()).sum().backward()
    torch.cuda.synchronize()

    orc = oracle_run(case)
    f = lambda t: t.detach().float().cpu().numpy().astype(np.float64)
    tol = TOL["bf16"]
    assert O.shape == (B, H, N, d)
    assert rel_err(f(O), orc["O"][:, :, :N]) <= tol
    for got, key in ((q.grad, "dQ"), (k.grad, "dK"), (v.grad, "dV")):
        assert rel_err(f(got), orc[key][:, :, :N]) <= tol, key
    if with_dustbin:
        for p_, key in zip(dustbin, ("dQ", "dK", "dV")):
            want = orc[key][:, :, N].sum(axis=0)   # one learned token shared by the batch
            assert p_.grad.shape == (H, d)
            assert rel_err(f(p_.grad), want) <= tol, key
    # inactive real rows have zero outputs and zero gradients
    inactive = mask == 0
    for t in (O, q.grad, k.grad, v.grad):
        assert np.all(f(t).transpose(0, 2, 1, 3)[inactive] == 0.0)
