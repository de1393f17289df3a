"""General block-causal attention (several query units over a shared prefix)
through the C ABI against the oracle's masked attention.

Query i (unit i // U) sees the prefix -- the first n_kv - n_q keys -- and the
keys of units <= its own; the mask on the oracle side is built from that
definition with the oracle's block-causal rule (prefix keys in unit -1).  Cases
span units that are not a multiple of the 128-row tiles (the mask changes inside
a tile and inside a warp), key splits in which some rows see no key at all,
ragged tails, one unit (must equal the every-key-visible result bit for bit),
and the fp32 mode.  Tolerances: relative L2 <= 2e-2 (bf16), <= 1e-5 (fp32).
"""
import numpy as np
import pytest
import torch

import sfm_synth as S
from oracle import sfm_oracle as O
from tests._gpu_util import BF16_TOL, FP32_TOL, rel_l2

pytestmark = pytest.mark.gpu


def _visible(n_q, n_kv, unit, rows=None):
    rows = np.arange(n_q) if rows is None else np.asarray(rows)
    prefix = n_kv - n_q
    k_units = np.concatenate([np.full(prefix, -1), np.arange(n_q) // unit])
    return O.block_causal_visible(rows // unit, k_units)


@pytest.mark.parametrize("n_q,prefix,unit,heads", [
    (2772, 4800, 924, 2),     # three 640x368 units over a cached prefix; key splits > 1
    (300, 0, 100, 3),         # no prefix: the first unit sees only itself
    (257, 129, 64, 2),        # ragged query and key tails
    (512, 1000, 128, 2),      # unit = one query tile
    (200, 50, 7, 2),          # many short units: the limit changes every few rows
])
def test_block_causal_bf16_matches_oracle(cuda_device, n_q, prefix, unit, heads):
    from streaming_flow_matching_b200 import attention
    n_kv = n_q + prefix
    q, k, v = S.make_qkv(n_q, n_kv, heads, 128)
    o = attention(q.cuda(), k.cuda(), v.cuda(), unit_tokens=unit)
    torch.cuda.synchronize()
    ref = O.attention(q, k, v, _visible(n_q, n_kv, unit))
    e = rel_l2(o.float().cpu().numpy(), ref)
    assert e <= BF16_TOL, e
    # the rows of the first unit must not see the second unit: compare against
    # attention restricted to their visible keys
    first = min(unit, n_q)
    ref0 = O.attention(q[:first], k[:prefix + first], v[:prefix + first])
    assert rel_l2(o[:first].float().cpu().numpy(), ref0) <= BF16_TOL


def test_block_causal_long_prefix_sampled_rows(cuda_device):
    # four 924-token units over a 57,600-token prefix, 24 heads; sampled rows
    # around the unit boundaries against the oracle
    from streaming_flow_matching_b200 import attention
    n_q, prefix, unit, H = 4 * 924, 57600, 924, 24
    q, k, v = S.make_qkv(n_q, n_q + prefix, H, 128, device="cuda")
    o = attention(q, k, v, unit_tokens=unit)
    torch.cuda.synchronize()
    rows = [0, 923, 924, 1023, 1024, 1847, 1848, 2771, 2772, 3695]
    qc, kc, vc = q[rows].cpu(), k.cpu(), v.cpu()
    ref = O.attention(qc, kc, vc, _visible(n_q, n_q + prefix, unit, rows))
    e = rel_l2(o[rows].float().cpu().numpy(), ref)
    assert e <= BF16_TOL, e


@pytest.mark.parametrize("n_q,n_kv", [(924, 5724), (300, 300), (1030, 3000)])
def test_single_unit_equals_every_key_visible(cuda_device, n_q, n_kv):
    from streaming_flow_matching_b200 import attention
    q, k, v = S.make_qkv(n_q, n_kv, 3, 128, device="cuda")
    a = attention(q, k, v)
    for unit in (n_q, n_q + 5):
        b = attention(q, k, v, unit_tokens=unit)
        torch.cuda.synchronize()
        assert torch.equal(a, b)


def test_block_causal_fp32_matches_oracle(cuda_device):
    from streaming_flow_matching_b200 import attention
    n_q, prefix, unit = 90, 37, 16
    q, k, v = S.make_qkv(n_q, n_q + prefix, 4, 64, dtype="fp32")
    o = attention(q.cuda(), k.cuda(), v.cuda(), unit_tokens=unit)
    torch.cuda.synchronize()
    ref = O.attention(q, k, v, _visible(n_q, n_q + prefix, unit))
    assert rel_l2(o.cpu().numpy(), ref) <= FP32_TOL


def test_block_causal_argument_errors(cuda_device):
    from streaming_flow_matching_b200 import _lib as L, attention
    q, k, v = S.make_qkv(64, 32, 2, 128, device="cuda")
    with pytest.raises(L.SfmError) as e:          # fewer keys than queries
        attention(q, k, v, unit_tokens=16)
    assert e.value.status == L.SFM_EINVAL
    q, k, v = S.make_qkv(64, 80, 2, 128, device="cuda")
    with pytest.raises(L.SfmError) as e:
        attention(q, k, v, unit_tokens=0)
    assert e.value.status == L.SFM_EINVAL
