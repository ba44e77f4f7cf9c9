"""A multi-image document (images and text runs of seeded random length, many short segments):
index sets against the oracle's (near-tie rule) and outputs against the oracle run with the
GPU's index sets; the small layout on every row, the 64K layout on sampled rows."""
import pytest

import oracle
from helpers import compare_outputs
from test_gpu_estimate import _check_head
from test_gpu_fullsize import check_rows, one_head_per_kind, run, sample_rows
import workload

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)


def small():
    return workload.mixed_image_text(L=3072, image=144, width=12, text=(16, 200), Hq=8, Hkv=2, k_v=60,
                                     k_s=200, name="mixed-image-text-3k")


def test_mixed_image_text_small_all_rows():
    p = small()
    Q, K, V, idx, o, _, _ = run(p, seed=2)
    for h in range(p.Hq):
        _check_head(p, h, idx[h], oracle.estimate_head(p, h, Q, K))
    Oref, _ = oracle.attention(p, Q, K, V, idx)
    got = o.float().cpu().numpy()
    for h in range(p.Hq):
        compare_outputs(got[h], Oref[h], f"{p.name} head {h}")


def test_mixed_image_text_64k_sampled():
    p = workload.mixed_image_text(L=65536)
    Q, K, V, idx, o, _, _ = run(p)
    for h in one_head_per_kind(p):
        _check_head(p, h, idx[h], oracle.estimate_head(p, h, Q, K))
    check_rows(p, Q, K, V, idx, o, range(p.Hq), sample_rows(p, 8))
