"""Host checks of the seeded workloads (no GPU): every benchmark workload has
a full-size GPU parity test of its own kind, and the generators are
deterministic."""

import os

import torch

from token_dynamic_quantization_b200 import workloads

TESTS = os.path.dirname(os.path.abspath(__file__))


def test_every_workload_has_a_full_size_gpu_test():
    import test_parity_gpu

    kinds = {n: workloads.make(n, rows=128).kind for n in workloads.WORKLOADS}
    # the quantizer workloads run through the parametrized full-size test
    assert set(test_parity_gpu.DQ_WORKLOADS) == {n for n, k in kinds.items() if k == "dynamic_quant"}
    # every other workload is named by a full-size test of its own
    gpu_sources = "".join(open(os.path.join(TESTS, f)).read() for f in os.listdir(TESTS)
                          if f.startswith("test_") and f.endswith("_gpu.py"))
    for n, k in kinds.items():
        if k != "dynamic_quant":
            assert f'workloads.make("{n}")' in gpu_sources, n


def test_generators_are_deterministic():
    for n in workloads.WORKLOADS:
        a = workloads.make(n, rows=64).tensors
        b = workloads.make(n, rows=64).tensors
        assert a.keys() == b.keys()
        for key in a:
            if isinstance(a[key], torch.Tensor):
                assert torch.equal(a[key], b[key]), (n, key)
