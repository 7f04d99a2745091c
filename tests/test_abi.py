"""The C-ABI library loads, exports every entry point the header declares,
and rejects bad arguments on the host before anything is launched (CPU only:
no call here reaches a kernel launch)."""
import ctypes
import os
import re

import pytest

from paged_kv_cache_406_b200 import _native as N

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "paged_kv.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(pkv_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_documented_entry_points():
    names = declared_functions()
    for must in ("pkv_kv_append", "pkv_paged_attention_decode", "pkv_copy_blocks", "pkv_alloc_create",
                 "pkv_seq_append_slots", "pkv_seq_free", "pkv_seq_fork", "pkv_decode_workspace_size"):
        assert must in names


def test_library_exports_every_declared_symbol(native):
    for name in declared_functions():
        assert hasattr(native, name), f"{name} declared in include/paged_kv.h but not exported"
        assert name in N.SIGNATURES, f"{name} has no binding signature"


def test_version_and_error_string(native):
    assert native.pkv_version().decode() == "1.0.0"
    rc = native.pkv_alloc_create(0, 16, None, ctypes.byref(ctypes.c_void_p()))
    assert rc == N.PKV_ERR_INVALID_ARG
    assert b"num_blocks" in native.pkv_last_error_string()


def _ws(native, *args):
    out = ctypes.c_size_t(0)
    rc = native.pkv_decode_workspace_size(*args, ctypes.byref(out))
    return rc, out.value


def test_workspace_size_host_only(native):
    rc, a = _ws(native, 64, 32, 8, 128, 257, 16, 256)
    assert rc == 0 and a > 0
    rc, b = _ws(native, 64, 32, 8, 128, 257, 16, 512)
    assert rc == 0 and b < a  # fewer partitions, smaller partials
    rc, c = _ws(native, 64, 32, 8, 128, 257, 16, 0)  # automatic: 512-token partitions
    assert rc == 0 and c == b
    rc, _ = _ws(native, 64, 32, 8, 128, 257, 16, 100)  # not a multiple of the block size
    assert rc == N.PKV_ERR_INVALID_ARG
    rc, _ = _ws(native, -1, 32, 8, 128, 257, 16, 0)
    assert rc == N.PKV_ERR_INVALID_ARG


FAKE = 1 << 20  # an aligned non-null address; every call below fails validation before using it


@pytest.mark.parametrize("kw,code", [
    (dict(dtype=7), N.PKV_ERR_UNSUPPORTED),
    (dict(head_dim=96), N.PKV_ERR_UNSUPPORTED),
    (dict(block_size=12), N.PKV_ERR_UNSUPPORTED),
    (dict(hq=24, hkv=8), N.PKV_ERR_UNSUPPORTED),        # group size 3
    (dict(hq=30, hkv=8), N.PKV_ERR_INVALID_ARG),        # not a multiple
    (dict(pt=100), N.PKV_ERR_INVALID_ARG),
    (dict(ws_bytes=16), N.PKV_ERR_INVALID_ARG),         # workspace too small
    (dict(q=FAKE + 4), N.PKV_ERR_INVALID_ARG),          # misaligned q
    (dict(ws=FAKE + 16), N.PKV_ERR_INVALID_ARG),        # workspace not 256-aligned
    (dict(q=0), N.PKV_ERR_INVALID_ARG),
    (dict(scale=float("nan")), N.PKV_ERR_INVALID_ARG),
])
def test_decode_rejects_bad_arguments_before_launch(native, kw, code):
    a = dict(q=FAKE, k=FAKE, v=FAKE, t=FAKE, l=FAKE, B=4, hq=32, hkv=8, head_dim=128, nb=64, maxb=8,
             block_size=16, scale=0.1, dtype=N.PKV_BF16, pt=0, ws=FAKE, ws_bytes=1 << 30, out=FAKE)
    a.update(kw)
    rc = native.pkv_paged_attention_decode(a["q"], a["k"], a["v"], a["t"], a["l"], a["B"], a["hq"], a["hkv"],
                                           a["head_dim"], a["nb"], a["maxb"], a["block_size"], a["scale"],
                                           a["dtype"], a["pt"], a["ws"], a["ws_bytes"], a["out"], None)
    assert rc == code, native.pkv_last_error_string()


@pytest.mark.parametrize("kw,code", [
    (dict(dtype=9), N.PKV_ERR_UNSUPPORTED),
    (dict(head_dim=80), N.PKV_ERR_UNSUPPORTED),
    (dict(kn=FAKE + 8), N.PKV_ERR_INVALID_ARG),
    (dict(n=-1), N.PKV_ERR_INVALID_ARG),
    (dict(slots=0), N.PKV_ERR_INVALID_ARG),
])
def test_append_rejects_bad_arguments_before_launch(native, kw, code):
    a = dict(kn=FAKE, vn=FAKE, slots=FAKE, n=3, kp=FAKE, vp=FAKE, nb=8, hkv=8, head_dim=128, bs=16,
             dtype=N.PKV_BF16)
    a.update(kw)
    rc = native.pkv_kv_append(a["kn"], a["vn"], a["slots"], a["n"], a["kp"], a["vp"], a["nb"], a["hkv"],
                              a["head_dim"], a["bs"], a["dtype"], None)
    assert rc == code


def test_zero_sized_calls_are_no_ops(native):
    assert native.pkv_kv_append(None, None, None, 0, None, None, 8, 8, 128, 16, N.PKV_BF16, None) == 0
    assert native.pkv_copy_blocks(None, None, None, 0, 8, 8, 128, 16, N.PKV_BF16, None) == 0
    assert native.pkv_paged_attention_decode(None, None, None, None, None, 0, 32, 8, 128, 8, 8, 16, 0.1,
                                             N.PKV_BF16, 0, None, 0, None, None) == 0


def test_copy_blocks_rejects_bad_arguments_before_launch(native):
    assert native.pkv_copy_blocks(FAKE, FAKE, FAKE, 2, 8, 8, 128, 16, 5, None) == N.PKV_ERR_UNSUPPORTED
    assert native.pkv_copy_blocks(FAKE + 4, FAKE, FAKE, 2, 8, 8, 128, 16, N.PKV_F16, None) == N.PKV_ERR_INVALID_ARG
    assert native.pkv_copy_blocks(FAKE, FAKE, 0, 2, 8, 8, 128, 16, N.PKV_F16, None) == N.PKV_ERR_INVALID_ARG


def test_step_meta_bytes_and_step_argument_checks(native):
    """pkv_step_meta_bytes is the documented layout (slots, lengths, copy
    pairs, tables: n * (4 + max_blocks) int32); the one-call step refuses bad
    arguments before it touches the allocator or the GPU."""
    assert native.pkv_step_meta_bytes(64, 256) == 64 * (4 + 256) * 4
    assert native.pkv_step_meta_bytes(0, 256) == 0 and native.pkv_step_meta_bytes(-1, 8) == 0
    buf = N.StepBuffers()
    assert native.pkv_decode_step_host(None, None, 1, ctypes.byref(buf), FAKE, FAKE, 8, 32, 8, 128, 16, 4, 0.1,
                                       N.PKV_BF16, 1.0, 1.0, 0, FAKE, 0, None) == N.PKV_ERR_INVALID_ARG
    a = ctypes.c_void_p()
    assert native.pkv_alloc_create(16, 16, None, ctypes.byref(a)) == 0
    ids = (ctypes.c_int64 * 1)(0)
    try:
        # a NULL staging buffer: refused, and nothing reserved
        assert native.pkv_seq_add(a, 0, 5) == 0
        rc = native.pkv_decode_step_host(a, ids, 1, ctypes.byref(buf), FAKE, FAKE, 16, 32, 8, 128, 16, 4, 0.1,
                                         N.PKV_BF16, 1.0, 1.0, 0, FAKE, 0, None)
        assert rc == N.PKV_ERR_INVALID_ARG
        n = ctypes.c_int32()
        assert native.pkv_seq_len(a, 0, ctypes.byref(n)) == 0 and n.value == 5
        assert native.pkv_decode_step_host(a, ids, 0, ctypes.byref(buf), FAKE, FAKE, 16, 32, 8, 128, 16, 4, 0.1,
                                           N.PKV_BF16, 1.0, 1.0, 0, FAKE, 0, None) == 0
    finally:
        native.pkv_alloc_destroy(a)


@pytest.mark.parametrize("kw,code", [
    (dict(dtype=7), N.PKV_ERR_UNSUPPORTED),
    (dict(n=-1), N.PKV_ERR_INVALID_ARG),
    (dict(kn=FAKE + 8), N.PKV_ERR_INVALID_ARG),         # misaligned new rows
    (dict(slots=0), N.PKV_ERR_INVALID_ARG),
    (dict(hq=24, hkv=8), N.PKV_ERR_UNSUPPORTED),        # group size 3: the decode half refuses
    (dict(scale=float("nan")), N.PKV_ERR_INVALID_ARG),
    (dict(ws_bytes=16), N.PKV_ERR_INVALID_ARG),
    (dict(pt=100), N.PKV_ERR_INVALID_ARG),
])
def test_append_and_decode_rejects_bad_arguments_before_launch(native, kw, code):
    """The one-call append + decode checks both halves' arguments before it
    launches anything (nothing here reaches the GPU)."""
    a = dict(kn=FAKE, vn=FAKE, slots=FAKE, n=4, q=FAKE, k=FAKE, v=FAKE, t=FAKE, l=FAKE, B=4, hq=32, hkv=8,
             head_dim=128, nb=64, maxb=8, block_size=16, scale=0.1, dtype=N.PKV_BF16, pt=0, ws=FAKE,
             ws_bytes=1 << 30, out=FAKE)
    a.update(kw)
    rc = native.pkv_append_and_decode(a["kn"], a["vn"], a["slots"], a["n"], a["q"], a["k"], a["v"], a["t"], a["l"],
                                      a["B"], a["hq"], a["hkv"], a["head_dim"], a["nb"], a["maxb"], a["block_size"],
                                      a["scale"], a["dtype"], a["pt"], a["ws"], a["ws_bytes"], a["out"], None)
    assert rc == code, native.pkv_last_error_string()


@pytest.mark.parametrize("kw,code", [
    (dict(src=7), N.PKV_ERR_UNSUPPORTED),
    (dict(k_scale=0.0), N.PKV_ERR_INVALID_ARG),
    (dict(v_scale=float("inf")), N.PKV_ERR_INVALID_ARG),
    (dict(head_dim=64), N.PKV_ERR_UNSUPPORTED),         # e4m3 pools need head_dim 128
    (dict(pt=264), N.PKV_ERR_INVALID_ARG),              # not a multiple of 16
])
def test_append_and_decode_fp8_rejects_bad_arguments_before_launch(native, kw, code):
    a = dict(kn=FAKE, vn=FAKE, src=N.PKV_F16, slots=FAKE, n=4, q=FAKE, k=FAKE, v=FAKE, t=FAKE, l=FAKE, B=4,
             hq=32, hkv=8, head_dim=128, nb=64, maxb=64, block_size=8, scale=0.1, k_scale=0.5, v_scale=0.5,
             pt=0, ws=FAKE, ws_bytes=1 << 30, out=FAKE)
    a.update(kw)
    rc = native.pkv_append_and_decode_fp8(a["kn"], a["vn"], a["src"], a["slots"], a["n"], a["q"], a["k"], a["v"],
                                          a["t"], a["l"], a["B"], a["hq"], a["hkv"], a["head_dim"], a["nb"],
                                          a["maxb"], a["block_size"], a["scale"], a["k_scale"], a["v_scale"],
                                          a["pt"], a["ws"], a["ws_bytes"], a["out"], None)
    assert rc == code, native.pkv_last_error_string()


@pytest.mark.parametrize("kw,code", [
    (dict(dtype=N.PKV_F32), N.PKV_ERR_UNSUPPORTED),    # the tensor-core prefill takes 16-bit K/V
    (dict(head_dim=64), N.PKV_ERR_UNSUPPORTED),
    (dict(hq=24, hkv=8), N.PKV_ERR_UNSUPPORTED),
    (dict(hq=30, hkv=8), N.PKV_ERR_INVALID_ARG),
    (dict(scale=0.0), N.PKV_ERR_INVALID_ARG),
    (dict(scale=float("nan")), N.PKV_ERR_INVALID_ARG),
    (dict(q=FAKE + 4), N.PKV_ERR_INVALID_ARG),
    (dict(qs=0), N.PKV_ERR_INVALID_ARG),
    (dict(T=-1), N.PKV_ERR_INVALID_ARG),
    (dict(ws=FAKE + 16, ws_bytes=1 << 30), N.PKV_ERR_INVALID_ARG),  # the V staging area: 256-byte aligned
    (dict(ws=FAKE, ws_bytes=4096), N.PKV_ERR_INVALID_ARG),          # and large enough
])
def test_prefill_rejects_bad_arguments_before_launch(native, kw, code):
    a = dict(q=FAKE, k=FAKE, v=FAKE, t=FAKE, l=FAKE, qs=FAKE, B=2, T=64, maxq=32, hq=32, hkv=8, head_dim=128,
             nb=64, maxb=8, block_size=16, scale=0.1, dtype=N.PKV_BF16, ws=None, ws_bytes=0, out=FAKE)
    a.update(kw)
    rc = native.pkv_paged_attention_prefill(a["q"], a["k"], a["v"], a["t"], a["l"], a["qs"], a["B"], a["T"],
                                            a["maxq"], a["hq"], a["hkv"], a["head_dim"], a["nb"], a["maxb"],
                                            a["block_size"], a["scale"], a["dtype"], a["ws"], a["ws_bytes"], a["out"],
                                            None)
    assert rc == code, native.pkv_last_error_string()


def test_prefill_empty_batch_is_a_no_op(native):
    assert native.pkv_paged_attention_prefill(None, None, None, None, None, None, 0, 0, 0, 32, 8, 128, 64, 8, 16,
                                              0.1, N.PKV_BF16, None, 0, None, None) == 0


def test_prefill_workspace_size(native):
    out = ctypes.c_size_t(0)
    # bf16: a 256-byte record + [num_seqs][max_blocks][Hkv][block_size][128] f16
    assert native.pkv_prefill_workspace_size(16, 8, 128, 256, 16, N.PKV_BF16, ctypes.byref(out)) == 0
    assert out.value == 256 + 16 * 256 * 8 * 16 * 128 * 2
    assert native.pkv_prefill_workspace_size(16, 8, 128, 256, 16, N.PKV_F16, ctypes.byref(out)) == 0
    assert out.value == 0  # f16 pools need no staging
    assert native.pkv_prefill_workspace_size(-1, 8, 128, 256, 16, N.PKV_BF16, ctypes.byref(out)) == N.PKV_ERR_INVALID_ARG


def _pools(*specs):
    """pkv_pool_t array from (num_blocks, block_size, max_blocks, num_seqs); fake pointers (never read)."""
    arr = (N.pkv_pool_t * len(specs))()
    for c, (nb, bs, maxb, n) in enumerate(specs):
        arr[c] = N.pkv_pool_t(FAKE, FAKE, FAKE, nb, bs, maxb, n)
    return arr


def test_pools_workspace_size_matches_the_single_pool_layout(native):
    out, ref = ctypes.c_size_t(0), ctypes.c_size_t(0)
    # 50 + 13 + 1 sequences; the largest capacity is 256 blocks of 16 = 512 blocks of 8 = 4096 tokens
    pools = _pools((1000, 32, 32, 50), (2000, 16, 256, 13), (3000, 8, 512, 1))
    assert native.pkv_decode_pools_workspace_size(pools, 3, 32, 8, 128, 0, ctypes.byref(out)) == 0
    assert native.pkv_decode_workspace_size(64, 32, 8, 128, 256, 16, 0, ctypes.byref(ref)) == 0
    assert out.value == ref.value


@pytest.mark.parametrize("specs,kw,code", [
    ((), {}, N.PKV_ERR_INVALID_ARG),                                                   # no pool
    (((64, 16, 8, 1),) * 4, {}, N.PKV_ERR_INVALID_ARG),                               # four pools
    (((64, 24, 8, 1),), {}, N.PKV_ERR_UNSUPPORTED),                                   # block size 24
    (((64, 32, 8, 1),), dict(pt=48), N.PKV_ERR_INVALID_ARG),                         # 48 % 32 != 0
    (((64, 16, 8, 1),), dict(pt=24), N.PKV_ERR_INVALID_ARG),                         # not a multiple of 16
    (((64, 16, 8, 1),), dict(dtype=N.PKV_F32), N.PKV_ERR_UNSUPPORTED),               # tensor cores only
    (((64, 16, 8, 1),), dict(hq=8, hkv=8), N.PKV_ERR_UNSUPPORTED),                   # one query head per KV head
    (((64, 16, 8, 1),), dict(head_dim=64), N.PKV_ERR_UNSUPPORTED),
    (((64, 16, 8, 1),), dict(ws_bytes=256), N.PKV_ERR_INVALID_ARG),                  # workspace too small
    (((64, 16, 8, 1),), dict(q=FAKE + 8), N.PKV_ERR_INVALID_ARG),                    # misaligned q
    (((64, 16, 8, -1),), {}, N.PKV_ERR_INVALID_ARG),                                  # negative count
])
def test_pools_call_rejects_bad_arguments_before_launch(native, specs, kw, code):
    a = dict(q=FAKE, hq=32, hkv=8, head_dim=128, scale=0.1, dtype=N.PKV_BF16, pt=0, ws_bytes=1 << 30)
    a.update(kw)
    pools = _pools(*specs) if specs else None
    rc = native.pkv_append_and_decode_pools(pools, len(specs), FAKE, FAKE, FAKE, a["q"], FAKE, a["hq"], a["hkv"],
                                            a["head_dim"], a["scale"], a["dtype"], a["pt"], FAKE, a["ws_bytes"], FAKE,
                                            None)
    assert rc == code, native.pkv_last_error_string()


def test_pools_call_with_no_sequences_is_a_no_op(native):
    pools = _pools((64, 16, 8, 0), (64, 8, 8, 0))
    assert native.pkv_append_and_decode_pools(pools, 2, None, None, None, None, None, 32, 8, 128, 0.1, N.PKV_BF16,
                                              0, None, 0, None, None) == 0
