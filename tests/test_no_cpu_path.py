"""The binding has no CPU path: every compute call handed host tensors
refuses them (ValueError) before the library sees a pointer, so nothing can
fall back to running on the host."""
import numpy as np
import pytest
import torch

import paged_kv_cache_segment_b200 as tf

BF = torch.bfloat16


def bf(*shape):
    return torch.zeros(shape, dtype=BF)


def f32(*shape):
    return torch.zeros(shape, dtype=torch.float32)


def u8(*shape):
    return torch.zeros(shape, dtype=torch.uint8)


def i32(*shape):
    return torch.zeros(shape, dtype=torch.int32)


SEGS = np.array([[0, 1, 16, 0, 1]], np.int32)


def partial_kw():
    return dict(scale=0.125, split_keys=16, n_splits_max=1, part_o=f32(1, 8, 1, 64), part_m=f32(1, 8, 1),
                part_l=f32(1, 8, 1), part_flag=u8(1, 8, 1), status=i32(1))


CALLS = {
    "tf_paged_attn_decode": lambda: tf.tf_paged_attn_decode(bf(1, 8, 64), bf(2, 2, 16, 64), bf(2, 2, 16, 64), i32(2),
                                                            torch.from_numpy(SEGS.copy()), **partial_kw()),
    "tf_paged_attn_block": lambda: tf.tf_paged_attn_block(bf(1, 8, 64), bf(2, 2, 16, 64), bf(2, 2, 16, 64), i32(2),
                                                          torch.from_numpy(SEGS.copy()), **partial_kw()),
    "tf_verify_round": lambda: tf.tf_verify_round(bf(1, 8, 64), bf(2, 2, 16, 64), bf(2, 2, 16, 64), i32(2),
                                                  torch.from_numpy(SEGS.copy()), out=f32(1, 8, 64), flags=u8(1, 8),
                                                  **partial_kw()),
    "tf_attn_merge": lambda: tf.tf_attn_merge(f32(1, 8, 2, 64), f32(1, 8, 2), f32(1, 8, 2), u8(1, 8, 2),
                                              f32(1, 8, 64), u8(1, 8)),
    "tf_paged_attn_prompt": lambda: tf.tf_paged_attn_prompt(bf(1, 8, 64), bf(2, 2, 16, 64), bf(2, 2, 16, 64), i32(2),
                                                            SEGS, scale=0.125, out=f32(1, 8, 64), status=i32(1)),
    "tf_kv_append": lambda: tf.tf_kv_append(bf(1, 2, 64), bf(1, 2, 64), bf(2, 2, 16, 64), bf(2, 2, 16, 64), i32(2),
                                            torch.from_numpy(SEGS.copy()), status=i32(1)),
    "tf_argmax_rows": lambda: tf.tf_argmax_rows(bf(2, 100), i32(2), u8(2)),
    "tf_ring_attn": lambda: tf.tf_ring_attn(bf(1, 8, 64), bf(40, 2, 64), bf(40, 2, 64), u8(24), scale=0.125,
                                            split_slots=16, n_splits_max=3, workspace=u8(4096), out=f32(1, 8, 64),
                                            flags=u8(1, 8), status=i32(1)),
    "tf_ring_tree_attn": lambda: tf.tf_ring_tree_attn(bf(3, 8, 64), bf(40, 2, 64), bf(40, 2, 64), u8(32), i32(3),
                                                      scale=0.125, split_slots=64, n_splits_max=2,
                                                      workspace=u8(1 << 16), out=f32(3, 8, 64), flags=u8(3, 8),
                                                      status=i32(1)),
    "tf_ring_attn_noalloc": lambda: tf.tf_ring_attn_noalloc(bf(1, 8, 64), bf(40, 2, 64), bf(40, 2, 64), u8(24),
                                                            scale=0.125, split_slots=16, n_splits_max=3,
                                                            out=f32(1, 8, 64), flags=u8(1, 8), status=i32(1)),
}


@pytest.mark.parametrize("name", sorted(CALLS))
def test_host_tensors_are_refused(name):
    with pytest.raises(ValueError, match="CUDA device"):
        CALLS[name]()


def test_every_compute_call_is_covered():
    host_only = ("tf_status_str", "tf_abi_version", "tf_ring_workspace_bytes", "tf_ring_tree_workspace_bytes",
                 "tf_choose_split_keys", "tf_wait_limit_test")
    compute = {n for n in tf.EXPORTS if n not in host_only}
    assert compute == set(CALLS)
