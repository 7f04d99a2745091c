"""GPU parity on the five seeded workloads at their full sizes (B200).

Every step's slot mapping must equal the allocator model's; sampled sequences'
pool blocks must equal the oracle's byte for byte, and their attention output
must be within tolerance of the fp64 oracle.
"""
import pytest

from paged_kv_cache_406_b200 import workloads as W
from workload_driver import run_workload

pytestmark = pytest.mark.gpu


def test_llama3_8b_decode_layer(native):
    w = W.WORKLOADS["llama3_8b"]
    lens = W.seq_lens(w)
    order = sorted(range(w.num_seqs), key=lambda b: lens[b])
    sample = {order[0], order[1], order[len(order) // 2], order[-2], order[-1], 7}
    st = run_workload(w, sample, check=lambda step, b: True)
    assert st["num_seqs"] == 64


@pytest.mark.parametrize("bs", [8, 16, 32])
@pytest.mark.parametrize("prefix", [1024, 1021])
def test_prefix_shared_batch(native, bs, prefix):
    """1024-token prefix as specified (block-aligned for 8/16/32: no copy);
    1021 tokens leaves the last shared block partial, so the first tail token
    of every sharer but the last copies it."""
    w = W.WORKLOADS[f"prefix_shared_bs{bs}"]
    st = run_workload(w, None, check=lambda step, b: True, prefix_tokens=prefix)
    assert st["cow_copies"] == (w.num_seqs - 1 if prefix % bs else 0)


def test_long_context_split_k(native):
    w = W.WORKLOADS["long_splitk"]
    run_workload(w, {0, 7}, check=lambda step, b: True, heads=[0, 5])


def test_mha_7b_fifty_steps(native):
    """Steps 0 and 49 checked for four sequences (the longest among them),
    and one sequence at every step."""
    w = W.WORKLOADS["mha_7b"]
    lens = W.seq_lens(w)
    longest = int(lens.argmax())
    sample = {0, 100, 200, longest}
    run_workload(w, sample, check=lambda step, b: step in (0, w.steps - 1) or b == 100, heads=[0, 13, 31])
