"""The Transformer-XL adapter's re-parameterisation, on CPU in fp64: the
unified score q'.k + q'.aQ[phi(i, j)] + b[phi(i, j)] with q' = q + u,
aQ = R W_r, b = (v - u).aQ equals (q + u).k + (q + v).W_r R_(j - i) in every
cell (identity map: phi = j - i + N - 1)."""
import torch

from exact_relative_position_b200.adapters import TransformerXLRelPos, sinusoid_table


def test_sinusoid_rows_are_offsets():
    N, dim = 7, 8
    R = sinusoid_table(N, dim).double()
    assert R.shape == (2 * N - 1, dim)
    # offset 0 sits at row N - 1: sin(0) = 0, cos(0) = 1
    assert torch.all(R[N - 1, : dim // 2] == 0) and torch.all(R[N - 1, dim // 2:] == 1)
    # sin is odd, cos is even in the offset
    assert torch.allclose(R[N - 1 + 3, : dim // 2], -R[N - 1 - 3, : dim // 2])
    assert torch.allclose(R[N - 1 + 3, dim // 2:], R[N - 1 - 3, dim // 2:])


def test_unified_score_equals_transformer_xl_score():
    torch.manual_seed(0)
    H, N, d = 2, 9, 4
    layer = TransformerXLRelPos(H, d, d_model=6, init_std=0.5).double().requires_grad_(False)
    q, k = torch.randn(1, H, N, d, dtype=torch.float64), torch.randn(1, H, N, d, dtype=torch.float64)
    R = sinusoid_table(N, 6).double()
    rel = torch.einsum("rc,hcd->hrd", R, layer.W_r)                       # [H, 2N - 1, d]
    # unified inputs, computed here in fp64 with the adapter's formulas
    qp = q + layer.u[None, :, None, :]
    b = torch.einsum("hd,hrd->hr", layer.v - layer.u, rel)
    for h in range(H):
        for i in range(N):
            for j in range(N):
                r = j - i + N - 1
                unified = qp[0, h, i] @ k[0, h, j] + qp[0, h, i] @ rel[h, r] + b[h, r]
                txl = (q[0, h, i] + layer.u[h]) @ k[0, h, j] + (q[0, h, i] + layer.v[h]) @ rel[h, r]
                assert abs(float(unified - txl)) < 1e-12


def test_deberta_unified_score_equals_disentangled_score():
    """The DeBERTa adapter's tables in the unified score, q.k + q.aQ[phi] + k.aK[phi]
    with phi = 'log_rev', equal DeBERTa's c2c + c2p + p2c in every cell, c2p and
    p2c read at the log-bucket row of the query-minus-key position i - j."""
    import oracle as orc
    from exact_relative_position_b200.adapters import DebertaRelPos
    torch.manual_seed(1)
    H, N, d, span, md = 2, 23, 4, 4, 12
    layer = DebertaRelPos(H, d, d_model=6, span=span, max_position=md, init_std=0.5).double()
    q, k = torch.randn(1, H, N, d, dtype=torch.float64), torch.randn(1, H, N, d, dtype=torch.float64)
    with torch.no_grad():
        Kr = torch.einsum("rc,hcd->hrd", layer.rel_embeddings, layer.W_kr)
        Qr = torch.einsum("rc,hcd->hrd", layer.rel_embeddings, layer.W_qr)
        aq, ak = layer.unified_inputs(torch.float64)
    m = layer.rel_map()
    phi = orc.phi_matrix(orc.MapDesc(m.kind, num_buckets=m.num_buckets, max_distance=m.max_distance), N)
    for h in range(H):
        for i in range(N):
            for j in range(N):
                row = int(orc.log_bucket(i - j, span, md))
                deberta = q[0, h, i] @ k[0, h, j] + q[0, h, i] @ Kr[h, row] + k[0, h, j] @ Qr[h, row]
                unified = q[0, h, i] @ k[0, h, j] + q[0, h, i] @ aq[h, phi[i, j]] + k[0, h, j] @ ak[h, phi[i, j]]
                assert abs(float(unified - deberta)) < 1e-12
