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


def _deberta_dense(q, k, v, E, W_kr, W_qr, tau, span, md, key_len):
    """Dense fp32 DeBERTa attention: c2p gathered at the log-bucket row of i - j
    from q . K^r, p2c gathered key-major at the row of the negated relative
    position from k . Q^r and transposed; the fp16-rounded tables the kernel sees."""
    import oracle as orc
    B, H, N, d = q.shape
    Kr = torch.einsum("rc,hcd->hrd", E.float(), W_kr.float()).half().float()
    Qr = torch.einsum("rc,hcd->hrd", E.float(), W_qr.float()).half().float()
    i = torch.arange(N)
    rel = (i[:, None] - i[None, :]).numpy()
    c2p_idx = torch.as_tensor(orc.log_bucket(rel, span, md), device=q.device)
    p2c_idx = torch.as_tensor(orc.log_bucket(-rel, span, md), device=q.device)
    qf, kf, vf = q.float(), k.float(), v.float()
    c2p = torch.gather(torch.einsum("bhid,hrd->bhir", qf, Kr), 3, c2p_idx.expand(B, H, N, N))
    p2c = torch.gather(torch.einsum("bhjd,hrd->bhjr", kf, Qr), 3, p2c_idx.expand(B, H, N, N)).transpose(-1, -2)
    s = tau * (torch.einsum("bhid,bhjd->bhij", qf, kf) + c2p + p2c)
    if key_len is not None:
        keep = i.to(q.device)[None, :] < key_len.to(q.device)[:, None]          # [B, N] keys
        s = s.masked_fill(~keep[:, None, None, :], float("-inf"))
    return torch.softmax(s, dim=-1) @ vf


@pytest.mark.parametrize("key_len", [None, [300, 187]])
def test_deberta_adapter_matches_dense(key_len):
    from exact_relative_position_b200.adapters import DebertaRelPos
    torch.manual_seed(0)
    B, H, N, d, span, md = 2, 2, 300, 64, 64, 256
    layer = DebertaRelPos(H, d, span=span, max_position=md).cuda()
    q, k, v = (torch.randn(B, H, N, d, device="cuda").half().requires_grad_() for _ in range(3))
    do = torch.randn(B, H, N, d, device="cuda").half()
    kl = None if key_len is None else torch.tensor(key_len, dtype=torch.int32, device="cuda")

    o = layer(q, k, v, key_len=kl)
    o.backward(do)
    got = [o.detach().float(), q.grad.clone(), k.grad.clone(), v.grad.clone(), layer.rel_embeddings.grad.clone(),
           layer.W_kr.grad.clone(), layer.W_qr.grad.clone()]

    params = [p.detach().clone().requires_grad_() for p in (layer.rel_embeddings, layer.W_kr, layer.W_qr)]
    q2, k2, v2 = (t.detach().clone().requires_grad_() for t in (q, k, v))
    o_ref = _deberta_dense(q2, k2, v2, *params, layer.tau, span, md, kl)
    o_ref.backward(do.float())
    want = [o_ref.detach(), q2.grad, k2.grad, v2.grad] + [p.grad for p in params]

    assert _relf(got[0], want[0]) <= 2e-3
    for name, g, w in zip(("dq", "dk", "dv", "dE", "dW_kr", "dW_qr"), got[1:], want[1:]):
        assert _relf(g, w) <= 1e-2, name
