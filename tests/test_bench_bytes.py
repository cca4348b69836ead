"""The algorithmic bytes behind bench.py's roofline, against the call's tensors.

For each step of the path, the bytes a kernel must move are its inputs read
once plus its outputs written once.  Here they are summed from the shapes and
element sizes of the tensors each C-ABI call takes and fills (the same
allocation the binding makes), and compared with bench.algorithmic_bytes."""
import os
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _nbytes(*shapes_dtypes):
    return sum(int(torch.empty(s, dtype=d, device="meta").numel()) *
               torch.empty((), dtype=d).element_size() for s, d in shapes_dtypes)


@pytest.mark.parametrize("T,H,k,E,n_rows", [(65536, 2048, 8, 128, 431022),   # headline, dedup
                                            (65536, 2048, 8, 128, 65536 * 8),  # conventional
                                            (262144, 2048, 8, 256, 1513400),
                                            (4096, 2048, 6, 64, 4096 * 6)])
def test_algorithmic_bytes_match_the_calls_tensors(T, H, k, E, n_rows):
    import bench
    i32, f32, bf16 = torch.int32, torch.float32, torch.bfloat16
    want = {
        # logits in; top-k indices and gates out
        "route_topk": _nbytes(((T, E), f32), ((T, k), i32), ((T, k), f32)),
        # top-k in; assign_row, row_of_slot out; row_token, row_mask for each row
        "dispatch_layout": _nbytes(((T, k), i32), ((T, k), i32), ((T, k), i32),
                                   ((n_rows,), i32), ((n_rows,), i32)),
        # x and row_of_slot in; one bf16 row out per dispatch row
        "dispatch_permute": _nbytes(((T, H), bf16), ((T, k), i32), ((n_rows, H), bf16)),
        # expert outputs, assign_row, idx, gates in; one bf16 row out per token
        "combine": _nbytes(((T * k, H), bf16), ((T, k), i32), ((T, k), i32), ((T, k), f32),
                           ((T, H), bf16)),
    }
    assert bench.algorithmic_bytes(T, H, k, E, n_rows) == want


def test_headline_combine_bytes_per_token():
    import bench
    # the headline workload: T=262144, H=2048, E=256, k=8;
    # 2H(k+1) + 12k = 36,960 B per token
    assert bench.WORKLOAD == "full_e256_k8"
    assert bench.algorithmic_bytes(262144, 2048, 8, 256, 0)["combine"] == 262144 * 36960
