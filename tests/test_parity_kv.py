"""K/V recomputation parity: K = y W_k, V = y W_v against the fp64 oracle.

Integer-valued inputs are exact in bf16 and in fp32 accumulation, so the
small case must match bit for bit; the full-size visual-feature workload is
compared on sampled rows.
"""

import numpy as np
import pytest
import torch

import oracle
from blockwise_long_context_b200 import inputs
from blockwise_long_context_b200 import binding as lvx
from tests._parity import compare, sample_rows

pytestmark = pytest.mark.gpu


def _run(y, wk, wv, H_kv, d):
    B, S, _ = y.shape
    k = torch.empty(B, S, H_kv, d, dtype=y.dtype, device="cuda")
    v = torch.empty_like(k)
    lvx.lvx_kv_recompute(y.cuda(), wk.cuda(), wv.cuda(), k, v, H_kv, d)
    torch.cuda.synchronize()
    return k, v


@pytest.mark.parametrize("dtype,S,E,H_kv,d", [
    (torch.bfloat16, 300, 256, 2, 128),     # tensor-core tiles with a ragged row tail
    (torch.bfloat16, 129, 192, 1, 128),
    (torch.bfloat16, 77, 40, 3, 8),         # CUDA-core path
    (torch.float32, 100, 64, 2, 64),
])
def test_kv_recompute_exact_integers(dtype, S, E, H_kv, d):
    g = torch.Generator().manual_seed(5)
    y = torch.randint(-2, 3, (2, S, E), generator=g).to(dtype)
    wk = torch.randint(-2, 3, (E, H_kv * d), generator=g).to(dtype)
    wv = torch.randint(-2, 3, (E, H_kv * d), generator=g).to(dtype)
    k, v = _run(y, wk, wv, H_kv, d)
    K, V = oracle.kv_recompute(y.double().numpy(), wk.double().numpy(), wv.double().numpy())
    # |entries| <= 4*E <= 1024 is exact in bf16 only below 256; compare after rounding the oracle
    Kr = torch.from_numpy(K).to(dtype).double().numpy().reshape(2, S, H_kv, d)
    Vr = torch.from_numpy(V).to(dtype).double().numpy().reshape(2, S, H_kv, d)
    np.testing.assert_array_equal(k.double().cpu().numpy(), Kr)
    np.testing.assert_array_equal(v.double().cpu().numpy(), Vr)


def test_kv_recompute_full_size_sampled_rows():
    w = inputs.WORKLOADS["C2"]
    host = inputs.make(w, tensors=("y", "w_k", "w_v"))
    k, v = _run(host["y"], host["w_k"], host["w_v"], w.H_kv, w.d)
    rows = sample_rows(w.S_KV, w.n_blocks, count=512)
    K, V = oracle.kv_recompute(host["y"][0].double().numpy(), host["w_k"].double().numpy(),
                               host["w_v"].double().numpy(), rows=rows)
    compare(k[0, rows].reshape(len(rows), -1), K, "bf16", "K (sampled rows)")
    compare(v[0, rows].reshape(len(rows), -1), V, "bf16", "V (sampled rows)")
    assert torch.isfinite(k.float()).all() and torch.isfinite(v.float()).all()
