"""The largest sequence the attention kernel accepts: 6,144 64-token blocks
(a 96x64x64 grid, 393,216 tokens), the size of its on-chip step table and
close to on-chip selection's limit, checked like every full-size workload
(layout maps, permuted rows, pooled means, every index list, sampled
attention outputs against fp64).  The file name sorts last so that it runs
after the other GPU tests."""
import pytest

from test_parity_full_gpu import check_full_size

pytestmark = pytest.mark.gpu

MAX_GRID = {"B": 1, "heads": 2, "T": 96, "H": 64, "W": 64, "T_valid": 96, "H_valid": 64,
            "W_valid": 64}


@pytest.fixture(scope="module", autouse=True)
def built(cuda_ok):
    from block_sparse_attention_47_b200 import build
    build.build()


def test_maximum_block_count():
    check_full_size("720p", MAX_GRID)
