"""GPU parity of the routing variants against the fp64 oracle: raw softmax
gates (Switch), the selection-only bias, sigmoid affinities normalised over the
chosen experts with group-limited selection (DeepSeek-V3)."""
import pytest
import torch

from sparse_mixture_experts_aux_b200.inputs import DEEPSEEK_V3, Workload
from tests.parity_util import check_workload

pytestmark = pytest.mark.gpu

CASES = [
    Workload("raw top-1 capacity zipf", 2048, 256, 16, 256, 1, capacity_factor=1.25,
             zipf_bias=True, gate_mode=1, seed=61),
    Workload("raw top-2", 777, 256, 32, 256, 2, gate_mode=1, seed=62),
    Workload("selection bias renorm", 600, 256, 16, 192, 2, selection_bias=True, seed=63),
    Workload("sigmoid 8 groups of 8, top-4 groups, shared", 700, 256, 64, 128, 8, d_s=128,
             gate_mode=2, selection_bias=True, n_group=8, topk_group=4, seed=64),
    Workload("sigmoid E=256 groups 8/4", 512, 256, 256, 64, 8, gate_mode=2, selection_bias=True,
             n_group=8, topk_group=4, seed=65),
    Workload("raw groups capacity", 900, 192, 16, 128, 2, gate_mode=1, n_group=4, topk_group=2,
             capacity_factor=0.9, seed=66),
    Workload("fp32 sigmoid groups", 200, 128, 16, 64, 4, "f32", gate_mode=2, n_group=4,
             topk_group=2, seed=67),
]


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_variant_parity(w):
    check_workload(w)


def test_deepseek_v3_workload_with_its_routing_sampled():
    w = DEEPSEEK_V3.with_(gate_mode=2, selection_bias=True, n_group=8, topk_group=4)
    check_workload(w, sample=256)
