"""Transformer-XL adapter: output and parameter gradients through the CUDA
path against dense fp32 PyTorch attention written from the Transformer-XL
score (content term (q + u).k plus position term (q + v).W_r R_(j - i)),
autograd on both sides, the same fp16 inputs and the same fp16-rounded
relation table."""
import math

import pytest
import torch

from exact_relative_position_b200.adapters import TransformerXLRelPos, sinusoid_table

pytestmark = pytest.mark.gpu


def _relf(a, b):
    return (a.double() - b.double()).norm().item() / max(b.double().norm().item(), 1e-30)


def _dense_reference(q, k, v, W_r, u, vb, causal, tau):
    """Dense [N, N] scores in fp32, cell by cell from the Transformer-XL form."""
    B, H, N, d = q.shape
    R = sinusoid_table(N, W_r.shape[1], device=q.device)                 # row r <-> offset r - (N - 1)
    rel = torch.einsum("rc,hcd->hrd", R, W_r.float()).half().float()     # the table the kernel sees
    i = torch.arange(N, device=q.device)
    idx = (i[None, :] - i[:, None]) + (N - 1)                            # [i, j] -> row of offset j - i
    relg = rel[:, idx]                                                   # [H, N, N, d]
    qf, kf, vf = q.float(), k.float(), v.float()
    content = torch.einsum("bhid,bhjd->bhij", qf + u.half().float()[None, :, None, :], kf)
    pos = torch.einsum("bhid,hijd->bhij", qf + vb.float()[None, :, None, :], relg)
    s = tau * (content + pos)
    if causal:
        s = s.masked_fill(i[None, :] > i[:, None], float("-inf"))
    return torch.softmax(s, dim=-1) @ vf


@pytest.mark.parametrize("causal", [True, False])
def test_transformer_xl_adapter_matches_dense(causal):
    torch.manual_seed(0)
    B, H, N, d = 1, 2, 200, 64
    layer = TransformerXLRelPos(H, d, causal=causal).cuda()
    q, k, v = (torch.randn(B, H, N, d, device="cuda").half().requires_grad_() for _ in range(3))
    do = torch.randn(B, H, N, d, device="cuda").half()

    o = layer(q, k, v)
    o.backward(do)
    got = [o.detach().float(), q.grad.clone(), k.grad.clone(), v.grad.clone(),
           layer.W_r.grad.clone(), layer.u.grad.clone(), layer.v.grad.clone()]

    ref_layer_params = [p.detach().clone().requires_grad_() for p in (layer.W_r, layer.u, layer.v)]
    q2, k2, v2 = (t.detach().clone().requires_grad_() for t in (q, k, v))
    o_ref = _dense_reference(q2, k2, v2, *ref_layer_params, causal, layer.tau)
    o_ref.backward(do.float())
    want = [o_ref.detach(), q2.grad, k2.grad, v2.grad] + [p.grad for p in ref_layer_params]

    assert _relf(got[0], want[0]) <= 2e-3
    for name, g, w in zip(("dq", "dk", "dv", "dW_r", "du", "dv_bias"), got[1:], want[1:]):
        assert _relf(g, w) <= 1e-2, name
