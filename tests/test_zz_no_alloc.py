"""The allocation-free attention entry point, tpl_attn_decode_static.

It serves callers that cannot allocate device memory themselves (a plugin in
a host application that owns the whole device budget, a serving loop that
must never enter the allocator): it takes no workspace and keeps its split
partials in a fixed array of the library's static device memory.  This test
calls it through the C-ABI and checks it against tpl_attn_decode, which uses
a caller-provided workspace, on two calls in a row.  It lives in a file that
pytest collects last, and passes both alone in a fresh process and after the
other tests.
"""
import ctypes

import pytest

from tests.conftest import has_gpu

pytestmark = pytest.mark.gpu


def test_attn_decode_static_matches_workspace_variant(gpu):
    import torch

    from megatron_tensor_transformer_plan_b200 import synth, tpl
    from tests.gpu_util import TOL, assert_close_rel, to_np

    # the attention step of the 70B-shaped stack: t = 8, batch 4, KV length 4096
    H, nq, nkv, d, F, t, B, S = 8192, 64, 8, 128, 28672, 8, 4, 4096
    plan = tpl.Plan(tpl.make_dims(H, nq, nkv, d, F, 1), t)
    kl, vl = synth.kv_cache((B, nkv, S + 1, d), seed=7, device=gpu)
    k, v = plan.pack_kv(kl), plan.pack_kv(vl)
    kv = tpl.Plan.kv(k, v, B, S + 1)
    q = torch.empty((B, nq, d), dtype=torch.float32, device=gpu)
    synth.normal_(q, 1.8, seed=11)
    k_new = torch.empty((B, nkv, d), dtype=torch.float32, device=gpu)
    v_new = torch.empty_like(k_new)
    synth.normal_(k_new, 1.8, seed=12)
    synth.normal_(v_new, 1.8, seed=13)
    ws = plan.workspace(B, S, device=gpu)
    o_ref = torch.empty((B, nq * d), dtype=torch.bfloat16, device=gpu)
    plan.attn_decode(kv, q, S, o_ref, ws, k_new, v_new)
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        o = torch.full_like(o_ref, float("nan"))
        rc = tpl.tpl_attn_decode_static(plan.handle, ctypes.byref(kv), q.data_ptr(), k_new.data_ptr(),
                                        v_new.data_ptr(), B, S, o.data_ptr(), stream)
        assert rc == tpl.TPL_OK, tpl.tpl_status_string(rc)
        torch.cuda.synchronize()
        assert_close_rel(to_np(o), to_np(o_ref), tol=TOL, what=f"static call {call}")
    assert plan.last_device_error() == tpl.TPL_OK

    # a problem larger than the fixed scratch is refused before any launch
    # 64 kv heads x 16 sequences = 1024 (sequence, kv head) pairs, 16 query
    # heads per kv head: ~8.6 MB of split partials
    big = tpl.Plan(tpl.make_dims(8192, 1024, 64, 128, 28672, 1), 1)
    kv_big = tpl.tpl_kv(k.data_ptr(), v.data_ptr(), 16, 8193)
    rc = tpl.tpl_attn_decode_static(big.handle, ctypes.byref(kv_big), q.data_ptr(), None, None, 16, 8192,
                                    o.data_ptr(), stream)
    assert rc == tpl.TPL_ENOMEM
