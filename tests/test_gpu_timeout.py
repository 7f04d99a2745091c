"""The decode kernels' bounded waits, made to run out on purpose (B200).

Every wait of a decode consumer for a K/V chunk gives up after a limit (1 s),
records PKV_ERR_DEVICE_TIMEOUT in the device status word and lets its CTA
finish.  Here that path runs without any fault or hang: through
pkv_debug_stall_decode the producer of CTA 0 skips the copies of its first
work unit, so that unit's consumers wait for chunks that never arrive; they
give up after the limit, the producer stops and, having issued no copy,
exits at once.  The call must end within the limit plus a margin, with the
timeout recorded, and the next normal call on the same pools must match the
oracle.
"""
import time

import pytest
import torch

from helpers import Case, assert_close

pytestmark = pytest.mark.gpu

PKV_ERR_DEVICE_TIMEOUT = -6


# bf16 with G = 4: the tensor-core kernel; f32 (G = 4) and f16 with G = 1: the CUDA-core kernel
@pytest.mark.parametrize("dtype,g", [("bf16", 4), ("f32", 4), ("f16", 1)])
def test_stalled_unit_times_out_and_next_call_is_correct(native, dtype, g):
    import paged_kv_cache_406_b200 as P
    # 4 sequences x 4 partitions of 512 tokens x 2 KV heads = 32 work units, one
    # per CTA; a unit spans 32 chunks, more than any ring has stages, so the
    # stalled producer issues no copy at all before it gives up
    case = Case([2048] * 4, 2 * g, 2, 128, 16, dtype, seed=404 + g)
    d = case.device()
    args = (d["q"], d["k_pool"], d["v_pool"], d["block_tables"], d["seq_lens"], case.scale)
    P.pkv_paged_attention_decode(*args)  # first launch: module load and tensor maps outside the timing
    assert P.pkv_device_status(clear=True) == 0
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    P.pkv_debug_stall_decode(0)
    try:
        t0 = time.perf_counter()
        e0.record()
        P.pkv_paged_attention_decode(*args)
        e1.record()
        status = P.pkv_device_status(clear=True)
        wall = time.perf_counter() - t0
    finally:
        P.pkv_debug_stall_decode(-1)
    assert status == PKV_ERR_DEVICE_TIMEOUT
    ms = e0.elapsed_time(e1)
    # one wait limit (1 s) for the stalled consumers, then every role leaves;
    # no second limit is waited out (the producer issued no copy to drain)
    assert 900.0 < ms < 1600.0, f"the stalled call took {ms:.1f} ms on the device"
    assert wall < 10.0
    out = P.pkv_paged_attention_decode(*args)
    assert P.pkv_device_status(clear=True) == 0
    assert_close(out, case.oracle(), dtype, f"{dtype} G={g} after the timed-out call")


def test_stalled_unit_times_out_e4m3_kernel(native):
    """The same on the tcgen05 e4m3 kernel: the stalled CTA's MMA warp gives up
    waiting for its first chunk's tiles, raises the abort flag, and the
    softmax warps and the producer (blocked on a stage that never frees)
    leave with it."""
    import numpy as np
    import paged_kv_cache_406_b200 as P
    from test_gpu_fp8 import Fp8Case
    # 4 sequences x 4 partitions of 512 tokens x 2 KV heads = 32 units, one per
    # CTA; a unit spans 4 chunks of 128 tokens, more than the ring's 2 stages
    case = Fp8Case([2048] * 4, 8, 2, 16, seed=406)
    ref = case.oracle()
    case.gpu()  # first launch: module load and tensor maps outside the timing
    assert P.pkv_device_status(clear=True) == 0
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    P.pkv_debug_stall_decode(0)
    try:
        t0 = time.perf_counter()
        e0.record()
        case.gpu()
        e1.record()
        status = P.pkv_device_status(clear=True)
        wall = time.perf_counter() - t0
    finally:
        P.pkv_debug_stall_decode(-1)
    assert status == PKV_ERR_DEVICE_TIMEOUT
    ms = e0.elapsed_time(e1)
    assert 900.0 < ms < 1600.0, f"the stalled call took {ms:.1f} ms on the device"
    assert wall < 10.0
    out = case.gpu()
    assert P.pkv_device_status(clear=True) == 0
    assert_close(out, ref, "f16", "e4m3 after the timed-out call")
    assert np.isfinite(out.cpu().numpy()).all()


def test_stall_setting_is_off_by_default(native):
    import paged_kv_cache_406_b200 as P
    case = Case([700, 1500], 8, 2, 128, 16, "bf16", seed=405)
    d = case.device()
    P.pkv_debug_stall_decode(-1)
    out = P.pkv_paged_attention_decode(d["q"], d["k_pool"], d["v_pool"], d["block_tables"], d["seq_lens"],
                                       case.scale)
    assert P.pkv_device_status(clear=True) == 0
    assert_close(out, case.oracle(), "bf16", "stall off")


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_stalled_prefill_times_out_and_next_call_is_correct(native, dtype):
    """The prefill kernel's bounded waits: through pkv_debug_stall_prefill the
    K producer of CTA 0 skips its first chunk of K, the MMA warp gives up
    after the limit, the CTA's abort flag sends every role out of its tile
    loop, and the producers drain only the copies they issued.  The other
    CTAs finish their tiles.  The call ends within the limit plus a margin
    with the timeout recorded, and the next call matches the oracle (bf16:
    the staged path, whose f16 instance is the one that stalls)."""
    import paged_kv_cache_406_b200 as P
    from test_gpu_prefill import PrefillCase
    # 8 sequences x 16 tiles of 64 tokens x 2 KV heads = 256 tiles, every one
    # with rows to compute, more than there are persistent CTAs: CTA 0 draws
    # work (with tiles past a short chunk's end it could draw only those)
    case = PrefillCase([1536] * 8, [1024] * 8, 8, 2, 16, dtype, seed=405)
    case.run()  # first call: module load and tensor maps outside the timing
    assert P.pkv_device_status(clear=True) == 0
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    P.pkv_debug_stall_prefill(0)
    try:
        t0 = time.perf_counter()
        e0.record()
        case.run()
        e1.record()
        status = P.pkv_device_status(clear=True)
        wall = time.perf_counter() - t0
    finally:
        P.pkv_debug_stall_prefill(-1)
    assert status == PKV_ERR_DEVICE_TIMEOUT
    ms = e0.elapsed_time(e1)
    # one wait limit (1 s) for the MMA warp, then every role of the CTA leaves;
    # the skipped fill is not waited for again in the drain
    assert 900.0 < ms < 1600.0, f"the stalled call took {ms:.1f} ms on the device"
    assert wall < 10.0
    out = case.run()
    assert P.pkv_device_status(clear=True) == 0
    assert_close(out, case.oracle(), dtype, f"{dtype} prefill after the timed-out call")


def test_prefill_stall_setting_is_off_by_default(native):
    """Without the test call, no prefill launch stalls: a normal call records
    no timeout."""
    import paged_kv_cache_406_b200 as P
    from test_gpu_prefill import PrefillCase
    case = PrefillCase([300, 129], [77, 1], 8, 2, 16, "bf16", seed=406)
    out = case.run()
    assert P.pkv_device_status(clear=True) == 0
    assert_close(out, case.oracle(), "bf16", "prefill with the stall setting off")
