"""Synthetic needle-in-a-haystack retrieval on the compressed cache.

The ai-muninn benchmark page reports a synthetic needle test
("Needle-in-Haystack（Synthetic）" section): exact retrieval at 2, 3 and 4 bits
for 512, 2048 and 8192 tokens. It does not say how its needles were made.
This is our own construction with the same grid:
* One kv head holds N random keys: random directions with log-normal norms
  (σ = 0.5). Eight query heads read it.
* Head h has a seeded query q_h and a needle at a seeded position. The
  needle's key has cosine 0.8 with q_h plus an orthogonal random remainder:
  a token that matches the query, as a retrieved fact does.
* Its norm is set so that its unquantized logit beats the largest
  haystack logit of that head by MARGIN standard deviations of the haystack
  logits. The difficulty is therefore stated, and the same in every cell of
  the grid.
* Each head's needle is haystack for the other heads.
* Retrieval is exact when the argmax over positions of the estimated logits
  is the needle, for every head. The test checks this for the GPU's tq_scores
  and for the oracle's logits, after checking that the unquantized fp64
  logits retrieve it too.
"""
import math

import numpy as np
import pytest
import torch

import kv_cache_vector_04_b200 as tq
from kv_cache_vector_04_b200 import inputs
from oracle import oracle as O
from tests import parity as P
from tests.test_parity_gpu import ctx_for

pytestmark = pytest.mark.gpu

D, HQ, MARGIN = 128, 8, 6.0


def haystack_with_needles(N, seed):
    k = inputs.kv_tensor((1, 1, N, D), "lognormal_norm", seed)[0, 0].double()
    v = inputs.kv_tensor((1, 1, N, D), "lognormal_norm", seed + 1)[0, 0]
    g = torch.Generator().manual_seed(seed + 2)
    q = torch.randn((HQ, D), generator=g, dtype=torch.float64).to(torch.bfloat16).double()
    pos = torch.randperm(N, generator=g)[:HQ]
    hay = k @ q.T / math.sqrt(D)                                  # [N, HQ] haystack logits
    for h in range(HQ):
        qh = q[h] / q[h].norm()
        r = torch.randn(D, generator=g, dtype=torch.float64)
        r = r - (r @ qh) * qh
        r = r / r.norm()
        target = hay[:, h].max() + MARGIN * hay[:, h].std()
        norm = target * math.sqrt(D) / (0.8 * q[h].norm())
        k[pos[h]] = norm * (0.8 * qh + 0.6 * r)
    return k.to(torch.float16), v, q.to(torch.bfloat16), pos.numpy()


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("N", [512, 2048, 8192])
def test_needle_is_retrieved_exactly(bits, N):
    k, v, q, pos = haystack_with_needles(N, seed=7000 + N + bits)
    exact = (k.double() @ q.double().T / math.sqrt(D)).numpy()          # [N, HQ]
    assert np.array_equal(exact.argmax(axis=0), pos)                      # the needle is there

    ctx, tab = ctx_for(D, bits)
    cache = P.quantize_on_gpu(ctx, k[None, None], v[None, None], capacity=N)
    seq = torch.tensor([N], dtype=torch.int32, device="cuda")
    s = tq.tq_scores(ctx, q[None].cuda(), cache, seq, N)
    torch.cuda.synchronize()
    assert tq.tq_status(ctx) == 0
    got = s[0].cpu().numpy()                                              # [HQ, N]
    assert np.array_equal(got.argmax(axis=1), pos), (got.argmax(axis=1), pos)

    codes = O.quantize(tab, k.numpy(), v.numpy())
    qb = P.q_bits(q)
    for h in range(HQ):
        _, lg = O.attend_head(tab, qb[h], True, codes, N)
        assert int(np.argmax(lg)) == pos[h]
