"""Parity at the full workload sizes the benchmark runs, in the same launch
configuration: the whole output is checked for finiteness and sampled rows
(every head, or a head sample for the largest cases) are compared with the
float64 oracle computed row by row."""
import numpy as np
import pytest

import workloads
from parity_util import check_workload, sample_rows

pytestmark = pytest.mark.gpu


def test_config1_tiny_exact_f32_full():
    check_workload(workloads.CONFIGS[1])


def test_config2_llama7b_prefill_sampled():
    w = workloads.CONFIGS[2]
    check_workload(w, rows=sample_rows(w, n_random=128), heads=[0, 7, 19, 31])


def test_config3_gqa_prefill_sampled():
    w = workloads.CONFIGS[3]
    check_workload(w, rows=sample_rows(w, n_random=64), heads=[0, 3, 4, 30, 31])


def test_config4_prefill_1m_sampled():
    w = workloads.CONFIGS[4]
    rows = np.array(sorted(set(range(0, 130)) | {16383, 16384, 16385, 524287, 524288, 1048447}
                           | set(range(1048576 - 8, 1048576))), dtype=np.int64)
    check_workload(w, rows=rows, heads=[0, 5])


def test_config5_cache_idx_sampled():
    w = workloads.CONFIGS[5]
    rows = np.array(list(range(0, 40)) + list(range(250, 260)) + list(range(490, 512)), dtype=np.int64)
    check_workload(w, rows=rows, heads=[0, 4, 13, 31])


@pytest.mark.parametrize("key", ["5d1", "5d8"])
def test_config5_decode_shapes(key):
    w = workloads.CONFIGS[key]
    check_workload(w, rows=np.arange(w.N_q), heads=[0, 1, 2, 3, 17, 31])


# The benchmark's end-to-end line runs the bf16 forward through the
# host-buffer entry point (KV-head groups streamed through the device).
def test_config2_host_path_sampled():
    w = workloads.CONFIGS[2]
    check_workload(w, rows=sample_rows(w, n_random=64), heads=[0, 2, 3, 17, 30, 31], host=True)


def test_config5_host_path_sampled():
    w = workloads.CONFIGS[5]
    rows = np.array(list(range(0, 24)) + list(range(500, 512)), dtype=np.int64)
    check_workload(w, rows=rows, heads=[0, 3, 4, 31], host=True)
