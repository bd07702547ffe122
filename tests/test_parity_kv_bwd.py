"""Parity of the K/V recomputation gradients against the fp64 oracle:
dW_k = y^T dK, dW_v = y^T dV, dy = dK W_k^T + dV W_v^T.

Integer-valued inputs make every product and every fp32 partial sum exact,
so the small cases must match the oracle rounded once to the output dtype,
bit for bit.  The full-size visual-feature workload (y [65536, 4096],
W [4096, 1024]) is compared on sampled rows of dy and sampled rows of dW
(row e of dW depends only on column e of y, so the oracle runs on those
columns alone).  The weight gradients are sums of 65536 products, so they
are compared after dividing both sides by the oracle's RMS, against the same
bar as the attention outputs.
"""

import numpy as np
import pytest
import torch

import oracle
from blockwise_long_context_b200 import inputs
from blockwise_long_context_b200 import binding as lvx
from tests._parity import compare, sample_rows

pytestmark = pytest.mark.gpu


def _run(y, wk, wv, dk, dv):
    dy = torch.full_like(y, float("nan"), device="cuda")
    dwk = torch.full_like(wk, float("nan"), device="cuda")
    dwv = torch.full_like(wv, float("nan"), device="cuda")
    lvx.lvx_kv_recompute_bwd(y.cuda(), wk.cuda(), wv.cuda(), dk.cuda(), dv.cuda(), dy, dwk, dwv)
    torch.cuda.synchronize()
    lvx.lvx_last_device_error()
    return dy.cpu(), dwk.cpu(), dwv.cpu()


def _rounded(x: np.ndarray, dtype) -> np.ndarray:
    return torch.from_numpy(x).to(dtype).double().numpy()


@pytest.mark.parametrize("dtype,B,S,E,H_kv,d", [
    (torch.bfloat16, 1, 200, 512, 2, 128),   # tensor cores; S not a multiple of the 64-row K step
    (torch.bfloat16, 2, 64, 256, 1, 256),    # two batches flattened into one K loop / row range
    (torch.bfloat16, 1, 1, 256, 4, 64),      # a single row of y
    (torch.bfloat16, 1, 77, 40, 3, 8),       # CUDA-core path (sizes off the tensor-core tiles)
    (torch.float32, 2, 50, 64, 2, 32),       # fp32: CUDA-core path
])
def test_kv_recompute_bwd_exact_integers(dtype, B, S, E, H_kv, d):
    g = torch.Generator().manual_seed(11)
    N = H_kv * d
    # sparse {-1, 0, 1} entries: the sums stay small, every partial sum is exact in fp32
    def tern(*shape):
        x = torch.randint(-1, 2, shape, generator=g) * (torch.rand(shape, generator=g) < 0.5)
        return x.to(dtype)
    y, wk, wv = tern(B, S, E), tern(E, N), tern(E, N)
    dk, dv = tern(B, S, H_kv, d), tern(B, S, H_kv, d)
    dy, dwk, dwv = _run(y, wk, wv, dk, dv)
    rdy, rdwk, rdwv = oracle.kv_recompute_bwd(y.double().numpy(), wk.double().numpy(),
                                              wv.double().numpy(),
                                              dk.double().numpy().reshape(B, S, N),
                                              dv.double().numpy().reshape(B, S, N))
    np.testing.assert_array_equal(dwk.double().numpy(), _rounded(rdwk, dtype))
    np.testing.assert_array_equal(dwv.double().numpy(), _rounded(rdwv, dtype))
    np.testing.assert_array_equal(dy.double().numpy().reshape(B, S, E), _rounded(rdy, dtype))


def test_kv_recompute_bwd_gaussian_small():
    """Non-integer inputs on the tensor-core path, every output element."""
    w = inputs.WORKLOADS["C2"].scaled(S_KV=640, d_embed=512, H_kv=2, d=128)
    host = inputs.make(w, tensors=("y", "w_k", "w_v", "dk", "dv"))
    dy, dwk, dwv = _run(host["y"], host["w_k"], host["w_v"], host["dk"], host["dv"])
    flat = lambda t: t.double().numpy().reshape(w.B, w.S_KV, -1)
    ref = oracle.kv_recompute_bwd(flat(host["y"]), host["w_k"].double().numpy(),
                                  host["w_v"].double().numpy(), flat(host["dk"]), flat(host["dv"]))
    for got, r, what in zip((dy, dwk, dwv), ref, ("dy", "dW_k", "dW_v")):
        r = r.reshape(got.shape)
        s = float(np.sqrt(np.mean(r * r)))
        compare(got.double().numpy() / s, r / s, "bf16", what)


def test_kv_recompute_bwd_full_size_sampled():
    w = inputs.WORKLOADS["C2"]
    host = inputs.make(w, tensors=("y", "w_k", "w_v", "dk", "dv"))
    dy, dwk, dwv = _run(host["y"], host["w_k"], host["w_v"], host["dk"], host["dv"])
    y64 = host["y"][0].double().numpy()
    wk64, wv64 = host["w_k"].double().numpy(), host["w_v"].double().numpy()
    dk64 = host["dk"].double().numpy().reshape(w.B, w.S_KV, -1)
    dv64 = host["dv"].double().numpy().reshape(w.B, w.S_KV, -1)
    rows = sample_rows(w.S_KV, w.n_blocks, count=256)
    rdy, _, _ = oracle.kv_recompute_bwd(y64, wk64, wv64, dk64[0], dv64[0], rows=rows)
    s = float(np.sqrt(np.mean(rdy * rdy)))
    compare(dy[0, rows].double().numpy() / s, rdy / s, "bf16", "dy (sampled rows)")
    e_sel = sample_rows(w.d_embed, 4, count=48, seed=1)
    _, rdwk, rdwv = oracle.kv_recompute_bwd(y64[:, e_sel], wk64[e_sel], wv64[e_sel], dk64[0],
                                            dv64[0], rows=rows[:1])
    for got, r, what in ((dwk, rdwk, "dW_k"), (dwv, rdwv, "dW_v")):
        s = float(np.sqrt(np.mean(r * r)))
        compare(got[e_sel].double().numpy() / s, r / s, "bf16", f"{what} (sampled rows)")
    for t in (dy, dwk, dwv):
        assert torch.isfinite(t.float()).all()
