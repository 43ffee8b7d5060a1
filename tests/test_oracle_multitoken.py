"""Pins for the multi-token decode oracle (several query tokens per
sequence, each with its own top-k index list), on the CPU: torch float64
scaled-dot-product attention with a query length above one, independence
of the tokens, and the single-token case."""
import numpy as np
import torch

from oracle import sparse_mla_ref as ref


def bf16(x) -> np.ndarray:
    return torch.as_tensor(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _as_t(bits):
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double()


def test_shared_full_list_equals_torch_attention_with_several_queries():
    rng = np.random.default_rng(1)
    B, T, H, D, N, dv = 2, 3, 4, 24, 40, 16
    q = bf16(rng.standard_normal((B, T, H, D)))
    kv = bf16(rng.standard_normal((N, D)))
    idx = np.broadcast_to(np.stack([rng.permutation(N) for _ in range(B)])[:, None, :], (B, T, N)).astype(np.int32)
    out, lse = ref.sparse_mla_decode_multi_token(q, kv, idx, 0.2, d_v=dv)
    kt = _as_t(kv)
    for b in range(B):
        qt = _as_t(q[b]).permute(1, 0, 2)                     # [H, T, D]: heads as batch, tokens as queries
        want = torch.nn.functional.scaled_dot_product_attention(qt, kt[None].expand(H, N, D),
                                                                kt[None, :, :dv].expand(H, N, dv), scale=0.2)
        np.testing.assert_allclose(out[b], want.permute(1, 0, 2).numpy(), atol=1e-12, rtol=0)
        np.testing.assert_allclose(lse[b], torch.logsumexp(0.2 * qt @ kt.T, -1).T.numpy(), rtol=1e-12)


def test_tokens_are_independent_and_padding_only_tokens_are_empty():
    rng = np.random.default_rng(2)
    B, T, H, D, N = 1, 3, 2, 16, 30
    q = bf16(rng.standard_normal((B, T, H, D)))
    kv = bf16(rng.standard_normal((N, D)))
    idx = np.stack([rng.permutation(N)[:10] for _ in range(T)])[None].astype(np.int32)
    out, lse = ref.sparse_mla_decode_multi_token(q, kv, idx, 0.3, d_v=8)
    idx2 = idx.copy()
    idx2[0, 1] = -1                                           # token 1 loses every entry
    out2, lse2 = ref.sparse_mla_decode_multi_token(q, kv, idx2, 0.3, d_v=8)
    assert np.array_equal(out2[0, 0], out[0, 0]) and np.array_equal(out2[0, 2], out[0, 2])
    assert np.all(out2[0, 1] == 0) and np.all(np.isneginf(lse2[0, 1]))


def test_one_token_is_the_single_token_decode():
    rng = np.random.default_rng(3)
    q = bf16(rng.standard_normal((2, 1, 4, 16)))
    kv = bf16(rng.standard_normal((64 * 3, 16)))
    pt = np.array([[2, 0], [1, 2]], np.int32)
    idx = rng.integers(-1, 128, size=(2, 1, 20)).astype(np.int32)
    o, l = ref.sparse_mla_decode_multi_token(q, kv, idx, 0.25, d_v=8, page_table=pt, page_size=64)
    o1, l1 = ref.sparse_mla_decode(q[:, 0], kv, idx[:, 0], 0.25, d_v=8, page_table=pt, page_size=64)
    assert np.array_equal(o[:, 0], o1) and np.array_equal(l[:, 0], l1)
