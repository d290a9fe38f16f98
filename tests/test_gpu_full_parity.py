"""Full GPU-oracle comparison on the Wan2.1-1.3B-480p-shaped layer (12 heads, 21x30x52 tokens = 32760 padded to
32768, head_dim 128, bf16, 128 x 128 blocks): every one of the 3072 (head, query block) items, in the launch
configuration the benchmark times. Dense O and lse, every block mass M(i, j), the selection of every row bit for bit,
and the sparse output at tau = 0.99 on the retained lists. Definitions: "LoSA: Near-Lossless Sparse Attention for
Training-Free Video Diffusion Acceleration", Motivation Summary (A and M(i, j)) and Methodology Summary ("One-time
pattern construction"; "Sparse attention with a frozen pattern"). The fp64 oracle takes a few minutes here."""
import dataclasses

import pytest

from losa_synth import CONFIGS
from tests.gpu_util import require_gpu
from tests.test_gpu_attention import _pipeline

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def test_wan480_every_item(oracle_mod):
    cfg = dataclasses.replace(CONFIGS["wan1.3b480"], taus=(0.99,))
    buf, _ = _pipeline(cfg, None, oracle_mod)
    assert buf.rows == 12 * 256
