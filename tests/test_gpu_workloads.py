"""GPU parity on the five seeded workloads at their full sizes (B200).

Every step's slot mapping must equal the allocator model's; the checked
sequences' pool blocks must equal the oracle's byte for byte, and their
attention output, for every KV head, must be within tolerance of the fp64
oracle.  The Llama-3-8B-shaped, prefix-shared and long split-K batches are
checked in full (every sequence, every head); the 50-step MHA batch in full at
its first and last step and on a rotating eighth of its sequences at every
step in between, so a work-assignment slip that touches only some (sequence,
partition, head) units cannot hide.
"""
import pytest

from paged_kv_cache_406_b200 import workloads as W
from workload_driver import run_workload

pytestmark = pytest.mark.gpu


def test_llama3_8b_decode_layer(native):
    w = W.WORKLOADS["llama3_8b"]
    st = run_workload(w, None, check=lambda step, b: True)
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
    run_workload(w, None, check=lambda step, b: True)


def test_mha_7b_fifty_steps(native):
    """All 256 sequences and 32 heads at steps 0 and 49; at every step in
    between, the sequences b with b % 8 == step % 8 (each sequence checked
    six times over the run)."""
    w = W.WORKLOADS["mha_7b"]
    last = w.steps - 1
    run_workload(w, None, check=lambda step, b: step in (0, last) or b % 8 == step % 8)
