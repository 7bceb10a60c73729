"""GPU parity of the dense per-head attention baseline (12 x 128 keys and values per token, the
layout the VideoMLA paper page replaces) against the oracle's textbook multi-head attention.
Same bar as the latent path: relative L2 <= 1e-2 and max-abs <= 3e-2 x RMS."""
import math

import numpy as np
import pytest
import torch

import mla_synth
from oracle import dense_mha
from tests.harness import assert_close

pytestmark = pytest.mark.gpu


def _qkv(B, nq, nkv, H, seed):
    q = mla_synth.normal_bf16((B, nq, H, 128), 1.0, seed)
    k = mla_synth.normal_bf16((B, nkv, H, 128), 1.0, seed + 1)
    v = mla_synth.normal_bf16((B, nkv, H, 128), 1.0, seed + 2)
    return q, k, v


def _run(q, k, v, scale=0.0, split=True):
    """split: hand the kernel the workspace the library asks for (key ranges merged by a second
    kernel where the shape has too few items to fill the GPU), else one pass per item."""
    import mla_latent_kv_window_b200 as M
    out = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    B, nq, H, _ = q.shape
    ws = None
    if split:
        ws = torch.empty(M.mla_dense_workspace_bytes(B, nq, k.shape[1], H), dtype=torch.uint8, device="cuda")
    M.mla_dense_attention(q.cuda(), k.cuda(), v.cuda(), out, scale, workspace=ws)
    assert M.mla_dense_sync() == 0
    return out.cpu()


@pytest.mark.parametrize("split", [True, False])
@pytest.mark.parametrize("B,nq,nkv,H", [(2, 200, 1000, 3), (1, 5, 130, 2), (1, 128, 128, 1), (3, 300, 77, 4),
                                        (1, 130, 1281, 2)])
def test_dense_small_every_element(B, nq, nkv, H, split):
    q, k, v = _qkv(B, nq, nkv, H, 10 * nq + nkv)
    out = _run(q, k, v, split=split)
    for b in range(B):
        ref = dense_mha(q[b], k[b], v[b], 1 / math.sqrt(128))
        assert_close(out[b], ref, f"dense B={B} nq={nq} nkv={nkv} H={H} split={split} stream {b}")


def test_dense_split_is_chosen_where_items_are_few():
    import mla_latent_kv_window_b200 as M
    # 12 items over 8 key tiles, and the 21-frame window (156 items on 148 SMs): split;
    # one key tile: nothing to split.
    assert M.mla_dense_workspace_bytes(2, 200, 1000, 3) > 0
    assert M.mla_dense_workspace_bytes(1, 1560, 21 * 1560 + 1560, 12) > 0
    assert M.mla_dense_workspace_bytes(1, 128, 128, 1) == 0
    assert M.mla_dense_workspace_bytes(1, 40, 1, 2) == 0


def test_dense_single_key_returns_value():
    q, k, v = _qkv(1, 40, 1, 2, 7)
    out = _run(q, k, v)
    np.testing.assert_array_equal(out[0].float().numpy(), np.broadcast_to(v[0].float().numpy(), out[0].shape))


def test_dense_custom_scale():
    q, k, v = _qkv(1, 64, 300, 2, 8)
    out = _run(q, k, v, scale=0.3)
    assert_close(out[0], dense_mha(q[0], k[0], v[0], 0.3), "dense scale 0.3")


def test_dense_full_size_layout_baseline_sampled():
    # The 21-frame Wan-1.3B window plus a 1,560-token query frame: 34,320 keys, 12 heads.
    nq, nkv, H = 1560, 21 * 1560 + 1560, 12
    q, k, v = _qkv(1, nq, nkv, H, 4000)
    rows = np.sort(np.random.default_rng(0).choice(nq, 64, replace=False))
    ref = dense_mha(q[0][rows], k[0], v[0], 1 / math.sqrt(128))
    for split in (True, False):
        out = _run(q, k, v, split=split)
        assert_close(out[0][rows], ref, f"dense full size, sampled rows, split={split}")
        assert torch.isfinite(out.float()).all()
