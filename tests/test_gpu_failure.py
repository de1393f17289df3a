"""Failure detection without a GPU fault: every wait inside the tensor-core kernels is
bounded.  A test-only fault makes a kernel's TMA producer issue no loads, with a
1 ms bound on the waits, so the roles waiting for those loads give up, record
their wait site and unwind; the context stays usable.  The handle then refuses
f_theta calls (SFM_EDEVICE) until the error is cleared, and the next call is
correct against the oracle."""
import ctypes as C

import numpy as np
import pytest
import torch

import sfm_synth as S
from oracle import sfm_oracle as O
from streaming_flow_matching_b200 import SfmError, _lib as L
from tests._gpu_util import BF16_TOL, SMALL_BF16, ocfg, oracle_cache_layers, rel_l2, to_cuda

pytestmark = pytest.mark.gpu

BOUND_NS = 1_000_000          # 1 ms


def _setup(w):
    from streaming_flow_matching_b200 import Performer
    weights_cpu = S.make_weights(w)
    k, v = S.make_kv_slices(w, w.cache_units)
    p = Performer.from_workload(w, to_cuda(weights_cpu))
    s = p.open_session(w.cache_units)
    p.kvcache_append(s, k.cuda(), v.cuda())
    ck, cv = oracle_cache_layers(k, v, w.cache_units, w.unit_kv_tokens, w.cache_units)
    return weights_cpu, ck, cv, p, s


@pytest.mark.parametrize("fault,kernel", [(L.SFM_FAULT_ATTN_NO_LOADS, 0x2),
                                          (L.SFM_FAULT_GEMM_NO_LOADS, 0x1)],
                         ids=["attention", "projections"])
@pytest.mark.parametrize("graphs", [True, False], ids=["graph", "direct"])
def test_timed_out_wait_is_reported_refused_and_recovered(cuda_device, fault, kernel, graphs):
    w = SMALL_BF16
    weights_cpu, ck, cv, p, s = _setup(w)
    p.set_graph_mode(graphs)
    _, eps = S.make_latents(w)
    taus = S.uniform_taus(w.n_steps)
    p.test_fault(fault, BOUND_NS)
    z = eps[0].cuda().clone()
    p.fm_solve(s, z, taus)                  # launches; the kernels give up and unwind
    code = p.check_device_error()
    assert code >> 8 == kernel, hex(code)   # a wait of the faulted kernel recorded its site
    # once the solve's copy of the error word has landed, f_theta calls are refused
    z2 = eps[0].cuda().clone()
    with pytest.raises(SfmError) as e:
        p.fm_solve(s, z2, taus)
    assert e.value.status == L.SFM_EDEVICE
    with pytest.raises(SfmError):
        p.denoise_step(s, z2, 1.0, 0.5)
    # clear the fault and the error: the same handle computes the right answer again
    p.test_fault(L.SFM_FAULT_NONE, 0)
    p.clear_device_error()
    assert p.check_device_error() == 0
    z = eps[0].cuda().clone()
    p.fm_solve(s, z, taus)
    torch.cuda.synchronize()
    valid = w.cache_units * w.unit_kv_tokens
    ref = O.denoise_solve(ocfg(w), eps[0], taus, weights_cpu, ck, cv, valid, valid)
    e_z = rel_l2(z.cpu().numpy(), ref)
    assert p.check_device_error() == 0
    assert e_z <= BF16_TOL, e_z
    p.close()


def test_standalone_attention_reports_a_timed_out_wait(cuda_device):
    from streaming_flow_matching_b200 import attention
    q, k, v = S.make_qkv(300, 2000, 3, 128, device="cuda")
    assert L.check_call_error() == 0
    L.set_call_fault(L.SFM_FAULT_ATTN_NO_LOADS, BOUND_NS)
    try:
        attention(q, k, v)
        code = L.check_call_error()
    finally:
        L.set_call_fault(L.SFM_FAULT_NONE, 0)
    assert code >> 8 == 0x2, hex(code)
    assert L.check_call_error() == 0        # reading the word cleared it
    o = attention(q, k, v)
    torch.cuda.synchronize()
    assert L.check_call_error() == 0
    assert rel_l2(o.float().cpu().numpy(), O.attention(q.cpu(), k.cpu(), v.cpu())) <= BF16_TOL


def test_standalone_pair_projection_reports_a_timed_out_wait(cuda_device):
    # 7392 x 3072 runs on CTA pairs (cta_group::2): both CTAs of a pair unwind
    from streaming_flow_matching_b200 import linear
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    x = torch.randn(7392, 3072, generator=g, device="cuda").to(torch.bfloat16)
    wt = (0.02 * torch.randn(3072, 3072, generator=g, device="cuda")).to(torch.bfloat16)
    L.set_call_fault(L.SFM_FAULT_GEMM_NO_LOADS, BOUND_NS)
    try:
        linear(x, wt)
        code = L.check_call_error()
    finally:
        L.set_call_fault(L.SFM_FAULT_NONE, 0)
    assert code >> 8 == 0x1, hex(code)
    y = linear(x, wt)
    torch.cuda.synchronize()
    assert L.check_call_error() == 0
    ref = x.float() @ wt.float().T
    assert rel_l2(y.cpu().numpy(), ref.cpu().numpy()) <= 5e-5


def test_fault_arguments_are_checked(cuda_device):
    assert L.lib.sfm_test_fault(None, 4, 0) == L.SFM_EINVAL
    assert L.lib.sfm_test_fault(None, 1, 10) == L.SFM_EINVAL          # bound below 10 us
    assert L.lib.sfm_test_fault(None, 1, 10 ** 11) == L.SFM_EINVAL    # above 10 s
    assert L.lib.sfm_test_fault(None, 0, 0) == L.SFM_OK
    code = C.c_int(-1)
    assert L.lib.sfm_check_call_error(C.byref(code)) == L.SFM_OK and code.value == 0
    assert L.lib.sfm_clear_device_error(None) == L.SFM_EINVAL
