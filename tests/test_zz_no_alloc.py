"""The decode entry point that allocates nothing (B200).

pkv_paged_attention_decode_static serves callers that cannot allocate device
memory while they decode (a runtime that has reserved nearly all of HBM for
its KV pool, a plugin whose host owns every allocation, a hot loop that must
not pay a synchronising cudaMalloc).  Its scratch is a static array inside the
library.  Here it is called through the C ABI twice in a row, on different
inputs, and each result must equal the workspace-taking entry point's on the
same inputs bit for bit (both run the same kernels); sizes whose scratch exceeds the
static array are refused before launch.  This file is collected last so that a
run stopping at the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from helpers import Case

pytestmark = pytest.mark.gpu


def _static_call(lib, d, case, out, pt=0):
    B, hq, D = d["q"].shape
    return lib.pkv_paged_attention_decode_static(
        d["q"].data_ptr(), d["k_pool"].data_ptr(), d["v_pool"].data_ptr(), d["block_tables"].data_ptr(),
        d["seq_lens"].data_ptr(), B, hq, case.hkv, D, case.nb, d["block_tables"].shape[1], case.bs,
        ctypes.c_float(case.scale), 1 if case.dtype == "bf16" else 2, pt, out.data_ptr(),
        torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("dtype,g,bs", [("bf16", 4, 16), ("f16", 1, 16), ("bf16", 2, 8)])
def test_static_workspace_matches_workspace_entry_point(native, dtype, g, bs):
    import paged_kv_cache_406_b200 as P
    for call in range(2):  # two calls in a row share (and overwrite) the static scratch
        lens = [1, 17, 300, 777, 1500, 2049][call:] + [64 + 100 * call]
        case = Case(lens, 2 * g, 2, 128, bs, dtype, seed=100 + call)
        d = case.device()
        want = P.pkv_paged_attention_decode(d["q"], d["k_pool"], d["v_pool"], d["block_tables"], d["seq_lens"],
                                            case.scale)
        got = torch.full_like(want, float("nan"))
        rc = _static_call(native, d, case, got)
        assert rc == 0, native.pkv_last_error_string()
        torch.cuda.synchronize()
        assert P.pkv_device_status(clear=True) == 0
        # the same kernels on the same inputs: bit-identical, not merely within tolerance
        assert torch.isfinite(got).all()
        assert torch.equal(got, want), float((got - want).abs().max())


def test_static_workspace_refuses_sizes_beyond_its_limit(native):
    limit = native.pkv_static_workspace_bytes()
    assert limit == 64 << 20
    need = ctypes.c_size_t(0)
    # 4096 sequences of up to 8192 tokens in 16-token partitions: far beyond the limit
    assert native.pkv_decode_workspace_size(4096, 32, 8, 128, 512, 16, 16, ctypes.byref(need)) == 0
    assert need.value > limit
    fake = 1 << 20  # never dereferenced: the size check comes first
    rc = native.pkv_paged_attention_decode_static(fake, fake, fake, fake, fake, 4096, 32, 8, 128, 1000, 512, 16,
                                                  ctypes.c_float(0.1), 1, 16, fake, None)
    assert rc == -1
    assert b"static workspace" in native.pkv_last_error_string()
