"""GPU parity of the alternative partitions behind sparsepr_partition against
the oracle's partition modes:
  * semantic: the comparison partition of "Partition the Support, Reconstruct
    the Residual" section 4 (ablations), keys and queries each clustered by
    plain Euclidean k-means on their own rows;
  * co-clustering: the bidirectional QK co-clustering of "Attention Sparsity
    is Input-Stable" (online co-clustering), rounds of key assignment in the
    query centres' affinity space and query assignment in the key centres'.
Labels and round counts bit for bit, then the rest of the call (permutation,
routes, attention, probe fit) on those partitions, integers bit-exact and
outputs within max-abs 2e-2 / mean-abs 2e-3."""
import numpy as np
import pytest

from free_block_sparse_eigenbasis_b200 import synth
from tests.parity import compare_head, gpu_run, np_, oracle_head

pytestmark = pytest.mark.gpu

CASES = [
    # bf16: both sides on the tensor cores
    synth.custom("small_bf16_d128", 2, (4, 16, 32), 128, "bf16", Ck=64, Cq=16, Ms=256,
                 n_eig=8, M=64, r=16, keep=(0.25, 0.4), seed=11),
    # fp32: both sides in fp64 on the CUDA cores
    synth.custom("small_f32_d64", 1, (3, 7, 11), 64, "f32", Ck=12, Cq=5, Ms=64, n_eig=4,
                 M=20, r=8, keep=0.3, seed=5),
    # many key groups: the keys' centroid planes exceed shared memory (fp64 path),
    # the queries stay on the tensor cores
    synth.custom("bf16_many_keys", 1, (4, 16, 32), 128, "bf16", Ck=700, Cq=24, Ms=256,
                 n_eig=8, M=32, r=8, keep=0.1, seed=13),
    # text tokens: outside every partition
    synth.custom("text_bf16_d128", 2, (3, 8, 16), 128, "bf16", n_text=40, Ck=24, Cq=6, Ms=128,
                 n_eig=8, M=32, r=8, keep=(0.2, 0.3), seed=21),
]


def _S():
    from free_block_sparse_eigenbasis_b200 import sparsepr as S
    return S


@pytest.mark.parametrize("mode", ["semantic", "coclustering"])
@pytest.mark.parametrize("w0", CASES, ids=[x.name for x in CASES])
def test_partition_mode_matches_oracle(w0, mode):
    w = w0.with_params(partition=mode)
    b, (q, k, v) = gpu_run(w, fill=0xFF)
    st = _S().sparsepr_read_stats(b.ws)
    assert st["status"] == 0
    for h in range(w.H):
        res = oracle_head(w, q, k, v, h)
        assert st["key_passes"][h] == res.info["key_passes"], (h, st["key_passes"])
        assert st["query_passes"][h] == res.info["query_passes"], (h, st["query_passes"])
        compare_head(b, res, w, h, None)
