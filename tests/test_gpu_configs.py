"""Every case of the five benchmark configurations at full size, in the
launch configuration the benchmark times.  Small problems are checked on
every output; large ones on sampled weight rows (all activation rows), with
the GPU quantizer's codes/absmax checked bit-exact on the same rows."""
import pytest

from bit_weight_dequant_b200 import inputs
from parity import run_case, run_case_sampled

pytestmark = pytest.mark.gpu

CASES = [(name, wl.index, c) for name, wl in inputs.workloads().items() for c in wl.cases]
FULL_CHECK_MAX_NK = 20_000_000      # host-generated W and every output checked below this size


@pytest.mark.parametrize("name,index,case", CASES, ids=[f"{n}-{c.tag}" for n, _, c in CASES])
def test_config_case(cuda_device, name, index, case):
    seed = inputs.seed_for(index, case.M)
    if case.N * case.K <= FULL_CHECK_MAX_NK:
        run_case(case, seed, cuda_device)
    else:
        run_case_sampled(case, seed, cuda_device)
