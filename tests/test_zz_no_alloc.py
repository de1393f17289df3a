"""The allocation-free attention entry point, for callers that cannot allocate
device memory (hard-deadline serving loops, hosts whose allocator owns all
device memory): through the C ABI it must give the same result as the
allocating entry point, call after call, and refuse shapes that need more
scratch than its fixed array holds.  Collected last on purpose."""
import ctypes as C

import pytest
import torch

import sfm_synth as S
from streaming_flow_matching_b200 import _lib as L
from tests._gpu_util import BF16_TOL, FP32_TOL, rel_l2

pytestmark = pytest.mark.gpu


def _noalloc(q, k, v, o, dtype):
    n_q, H, D = q.shape
    return L.lib.sfm_attention_noalloc(
        C.c_void_p(q.data_ptr()), C.c_void_p(k.data_ptr()), C.c_void_p(v.data_ptr()),
        C.c_void_p(o.data_ptr()), n_q, k.shape[0], H, D, dtype,
        C.c_void_p(torch.cuda.current_stream().cuda_stream))


def _allocating(q, k, v, dtype):
    n_q, H, D = q.shape
    o = torch.empty_like(q)
    need = L.lib.sfm_attention_workspace_bytes(n_q, k.shape[0], H, D, dtype)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    rc = L.lib.sfm_attention(C.c_void_p(q.data_ptr()), C.c_void_p(k.data_ptr()),
                             C.c_void_p(v.data_ptr()), C.c_void_p(o.data_ptr()), n_q, k.shape[0],
                             H, D, dtype, C.c_void_p(ws.data_ptr()), need,
                             C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == L.SFM_OK
    return o, need


def test_noalloc_matches_allocating_entry_point_on_consecutive_calls(cuda_device):
    # split-KV shapes (they use the scratch array) with different split counts, so a
    # merge reads a different-sized part of what the previous call left there; then
    # the first shape again, and an fp32 call that needs no scratch at all: stale
    # contents of the shared array must not leak into a later call
    cases = [(924, 17724, 24, "bf16"), (128, 20000, 2, "bf16"), (924, 17724, 24, "bf16"),
             (512, 9000, 8, "bf16"), (204, 704, 3, "bf16"), (68, 452, 4, "fp32")]
    splits = set()
    for n_q, n_kv, H, dt in cases:
        dtype = L.SFM_DTYPE_BF16 if dt == "bf16" else L.SFM_DTYPE_FP32
        q, k, v = S.make_qkv(n_q, n_kv, H, 128 if dt == "bf16" else 64, dtype=dt, device="cuda",
                             seed=n_kv)
        ref, need = _allocating(q, k, v, dtype)
        if dt == "bf16":
            # the partials of every split: [splits][n_q][H][128 + 1] fp32
            assert need > 0 and need % (n_q * H * 129 * 4) == 0, (n_q, n_kv, H, need)
            splits.add(need // (n_q * H * 129 * 4))
        o = torch.full_like(q, float("nan"))
        assert _noalloc(q, k, v, o, dtype) == L.SFM_OK
        torch.cuda.synchronize()
        e = rel_l2(o.float().cpu().numpy(), ref.float().cpu().numpy())
        assert e <= (BF16_TOL if dt == "bf16" else FP32_TOL), (n_q, n_kv, H, e)
    assert len(splits) >= 3, splits
    assert L.check_call_error() == 0


def test_noalloc_rejects_shapes_beyond_its_scratch(cuda_device):
    cap = L.SFM_NOALLOC_SCRATCH_BYTES
    big = None
    for H in (8, 12, 16, 24, 32, 48, 64):
        for n_q in range(64, 8192, 64):
            if L.lib.sfm_attention_workspace_bytes(n_q, 1 << 17, H, 128, L.SFM_DTYPE_BF16) > cap:
                big = (n_q, H)
                break
        if big:
            break
    if big is None:
        pytest.skip("no shape in the search range needs more scratch than the array holds")
    n_q, H = big
    # real-sized buffers, so the call would stay in bounds even if it were accepted
    q = torch.zeros(n_q, H, 128, dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros(1 << 17, H, 128, dtype=torch.bfloat16, device="cuda")
    o = torch.zeros_like(q)
    assert _noalloc(q, kv, kv, o, L.SFM_DTYPE_BF16) == L.SFM_ECAPACITY
    torch.cuda.synchronize()
    assert int(torch.count_nonzero(o)) == 0
