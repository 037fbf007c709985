"""sa_bwd_no_alloc, the backward for callers that cannot allocate device memory
(a plugin whose host framework owns all device memory and forbids allocation
while it runs, or a loop that cannot absorb an allocation's synchronisation).

It runs the backward on the library's fixed scratch array instead of a
caller-supplied workspace.  Its outputs must match the workspace entry point
sa_bwd within the parity tolerance, on two calls in a row (the second call
reuses the scratch the first one left behind).  This file is collected last,
so a run that stops at the first failure has already run every other test.
"""

import ctypes

import numpy as np
import pytest
import torch

from gen import get_workload, make_inputs, scaled
from gpu_harness import check_close, device_problem, grads_to_host, widen
from top_sparse_attention_attn_b200 import _lib as L

pytestmark = pytest.mark.gpu


def _io(o, lse, d_o, g):
    ptr = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    return L.SaBwdIo(o=ptr(o), d_o=ptr(d_o), lse=ptr(lse), dq=ptr(g["dq"]), dk=ptr(g.get("dk")),
                     dv=ptr(g.get("dv")), dkv=ptr(g.get("dkv")), dcmp_kv=ptr(g.get("dcmp")),
                     dsinks=ptr(g.get("dsinks")))


@pytest.mark.parametrize("w", [
    get_workload("cfg1"),                                                    # bucketed key-stationary index
    scaled("cfg2", "noalloc", S=700, Hq=16, Hkv=2, seed=42),                 # count / scan / fill index
    scaled("cfg4", "noalloc", seqlens=(100, 60), Hq=16, cmp_topk=32, cmp_len_range=(8, 32), seed=41),
], ids=["cfg1", "cfg2_small", "cfg4_small"])
def test_no_alloc_backward_matches_workspace_backward(w):
    if not torch.cuda.is_available():
        pytest.fail("a CUDA GPU is required for -m gpu tests")
    inputs = make_inputs(w)
    sa, t = device_problem(w, inputs)
    o, lse = sa.forward()
    ref = grads_to_host(sa.backward(o, lse, t["do"]))       # existing entry point, own workspace
    torch.cuda.synchronize()
    assert L.sa_bwd_get_workspace_size(sa.args()) <= L.sa_bwd_no_alloc_max_workspace()
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        g = sa.alloc_bwd()
        for v in g.values():
            v.fill_(float("nan"))                            # every output must be overwritten
        L.sa_bwd_no_alloc(sa.args(), _io(o, lse, t["do"], g), stream)
        torch.cuda.synchronize()
        assert L.sa_bwd_no_alloc_read_status(stream) == L.SA_OK
        got = grads_to_host(g)
        assert set(got) == set(ref)
        for key in ref:
            if key == "dsinks":
                check_close(f"call{call}:{key}", got[key], ref[key])
            else:
                check_close(f"call{call}:{key}", widen(got[key]), widen(ref[key]))
