"""Expansion parity: hd_expand_embed (CUDA, through the C ABI) vs the oracle, bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import structured_causal_attention_b200 as hd
from structured_causal_attention_b200 import synthetic as syn
from tests.gpu_util import need_gpu

pytestmark = pytest.mark.gpu


def _bits(t):
    """Raw bytes of a tensor as an integer array (exact comparison)."""
    return t.contiguous().view(torch.uint8).cpu().numpy() if t.element_size() == 1 else \
        t.contiguous().view({2: torch.int16, 4: torch.int32, 8: torch.int64}[t.element_size()]).cpu().numpy()


def test_expand_tiny_workload_bit_exact():
    """B1, L64, n4, V1000, d256 fp32 tables ~N(0, 0.02)."""
    need_gpu()
    w = syn.WORKLOADS["tiny"]
    inp = syn.expand_inputs(w["B"], w["L"], w["n"], w["V"], w["d"], seed=1)
    out = hd.expand_embed(inp["ids"].cuda(), inp["tables"].cuda())
    torch.cuda.synchronize()
    want = oracle.expand_embed(inp["ids"].numpy(), inp["tables"].numpy())
    assert (_bits(out) == want.view(np.int32)).all()
    assert hd.hd_device_status() == hd.HD_OK


@pytest.mark.parametrize("B,L,n,V,d,dtype", [
    (2, 33, 3, 50, 7, torch.float32),     # 28-byte rows: 4-byte path
    (1, 17, 5, 9, 3, torch.bfloat16),     # 6-byte rows: 2-byte path
    (3, 5, 1, 4, 64, torch.bfloat16),     # n = 1: plain lookup
    (1, 1, 8, 2, 4096, torch.float32),    # one token, wide rows
    (4, 100, 4, 300, 520, torch.float16),
])
def test_expand_shapes_bit_exact(B, L, n, V, d, dtype):
    need_gpu()
    inp = syn.expand_inputs(B, L, n, V, d, seed=B + L, dtype=dtype)
    out = hd.expand_embed(inp["ids"].cuda(), inp["tables"].cuda())
    torch.cuda.synchronize()
    want = torch.from_numpy(oracle.expand_embed(inp["ids"].numpy(), inp["tables"].view(torch.int16 if
                            dtype != torch.float32 else torch.int32).numpy()))
    assert (_bits(out) == want.numpy()).all()


def test_expand_out_of_range_id_zero_row_and_status():
    need_gpu()
    inp = syn.expand_inputs(1, 6, 3, 10, 8, seed=4)
    inp["ids"][0, 2] = 10
    inp["ids"][0, 4] = -1
    hd.hd_device_status(clear=True)
    out = hd.expand_embed(inp["ids"].cuda(), inp["tables"].cuda()).cpu()
    assert hd.hd_device_status(clear=True) == hd.HD_ERR_DEVICE_INDEX
    assert (out[0, 2 * 3:3 * 3] == 0).all() and (out[0, 4 * 3:5 * 3] == 0).all()
    ok = [0, 1, 3, 5]
    for t in ok:
        for s in range(3):
            assert torch.equal(out[0, t * 3 + s], inp["tables"][s, inp["ids"][0, t]])


def test_expand_large_sampled_bit_exact():
    """B4, L8192, n4, V32000, d4096 fp32 (4.3 GB moved): 512 sampled tokens, bit exact."""
    need_gpu()
    B, L, n, V, d = 4, 8192, 4, 32000, 4096
    ids = syn.token_ids(B, L, V, seed=77)
    tables = torch.empty((n, V, d), dtype=torch.float32, device="cuda")
    g = torch.Generator(device="cuda")
    g.manual_seed(78)
    tables.normal_(0.0, 0.02, generator=g)
    out = hd.expand_embed(ids.cuda(), tables)
    torch.cuda.synchronize()
    rng = np.random.default_rng(79)
    bt = np.unique(np.concatenate([[0, B * L - 1], rng.integers(0, B * L, 510)]))
    want = oracle.expand_embed(ids.numpy().reshape(-1)[bt][None, :], tables.cpu().numpy())[0]
    rows = (bt[:, None] * n + np.arange(n)[None, :]).reshape(-1)
    got = out.view(-1, d)[torch.from_numpy(rows).cuda()].cpu().numpy()
    assert (got.view(np.int32) == want.view(np.int32)).all()
