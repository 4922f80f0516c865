"""Pins for the text-query half of joint attention (global tokens as
queries over all image and global keys): it is full attention, so a library
routine over the concatenated keys is the closed form; permutation of the
image tokens and a single global token are checked as well."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from workloads import bf16_bits_to_f64, f64_to_bf16_bits


def rnd(rng, shape):
    return f64_to_bf16_bits(rng.standard_normal(shape))


@pytest.mark.parametrize("B,heads,H,W,d,G", [(1, 2, 6, 5, 16, 7), (2, 1, 4, 9, 32, 1), (1, 3, 8, 8, 16, 33)])
def test_equals_library_attention_over_all_keys(B, heads, H, W, d, G):
    rng = np.random.default_rng(G)
    gq, k, v = rnd(rng, (B, heads, G, d)), rnd(rng, (B, heads, H * W, d)), rnd(rng, (B, heads, H * W, d))
    gk, gv = rnd(rng, (B, heads, G, d)), rnd(rng, (B, heads, G, d))
    got = oracle.global_query_attention(gq, k, v, gk, gv, B=B, heads=heads, H=H, W=W, d=d, G=G)
    K = np.concatenate([k, gk], 2)
    V = np.concatenate([v, gv], 2)
    ref = F.scaled_dot_product_attention(*(torch.from_numpy(bf16_bits_to_f64(x)) for x in (gq, K, V))).numpy()
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_image_token_permutation_invariance_and_subset():
    rng = np.random.default_rng(9)
    B, heads, H, W, d, G = 1, 2, 5, 6, 16, 11
    gq, k, v = rnd(rng, (B, heads, G, d)), rnd(rng, (B, heads, H * W, d)), rnd(rng, (B, heads, H * W, d))
    gk, gv = rnd(rng, (B, heads, G, d)), rnd(rng, (B, heads, G, d))
    a = oracle.global_query_attention(gq, k, v, gk, gv, B=B, heads=heads, H=H, W=W, d=d, G=G)
    perm = rng.permutation(H * W)
    b = oracle.global_query_attention(gq, k[:, :, perm], v[:, :, perm], gk, gv, B=B, heads=heads, H=H, W=W,
                                      d=d, G=G)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-13)
    qs = np.array([[0, 1, 10], [0, 0, 3]], dtype=np.int32)
    sub = oracle.global_query_attention(gq, k, v, gk, gv, B=B, heads=heads, H=H, W=W, d=d, G=G, queries=qs)
    np.testing.assert_array_equal(sub[0], a[0, 1, 10])
    np.testing.assert_array_equal(sub[1], a[0, 0, 3])
