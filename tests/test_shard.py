"""Host side of the leaf-partitioned search (no GPU): shard arrays partition
the points by leaf, and two gloo ranks gather their candidates in rank order."""
import os
import socket
import subprocess
import sys
import textwrap

import numpy as np
import pytest
import torch

from mips_ivf_centroid_b200 import datagen

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def ix():
    w = datagen.WORKLOADS["glove"].scaled(n=4000, d=16, num_leaves=25, nq=4, n_means=10,
                                          training_sample_size=4000)
    return datagen.build_index(w, datagen.make_data(w), "cpu")


@pytest.mark.parametrize("G", [1, 2, 3, 7])
def test_shards_partition_points_by_leaf(ix, G):
    from mips_ivf_centroid_b200.shard import shard_arrays
    sizes = np.diff(ix.leaf_offsets.numpy())
    seen = []
    for g in range(G):
        sh = shard_arrays(ix, G, g)
        ss = np.diff(sh.leaf_offsets.numpy())
        owned = np.arange(len(sizes)) % G == g
        np.testing.assert_array_equal(ss[owned], sizes[owned])
        assert (ss[~owned] == 0).all()
        assert sh.slot_ids.shape[0] == sh.codes.shape[0] == sh.reorder_vecs.shape[0] == ss.sum()
        assert torch.equal(sh.centroids, ix.centroids) and torch.equal(sh.codebook, ix.codebook)
        # each kept slot carries its original code row and vector
        pos = {int(s): i for i, s in enumerate(ix.slot_ids.numpy())}
        for i, s in enumerate(sh.slot_ids.numpy()[:50]):
            j = pos[int(s)]
            assert torch.equal(sh.codes[i], ix.codes[j]) and torch.equal(sh.reorder_vecs[i], ix.reorder_vecs[j])
        seen.append(sh.slot_ids.numpy())
    allids = np.concatenate(seen)
    assert np.array_equal(np.sort(allids), np.sort(ix.slot_ids.numpy()))


def test_bad_shard_index(ix):
    from mips_ivf_centroid_b200 import AhError
    from mips_ivf_centroid_b200.shard import shard_arrays
    with pytest.raises(AhError):
        shard_arrays(ix, 2, 2)


WORKER = textwrap.dedent("""
    import os, sys, json
    sys.path.insert(0, {root!r})
    import torch, torch.distributed as dist
    from datetime import timedelta
    from mips_ivf_centroid_b200.shard import gather_candidates
    dist.init_process_group("gloo", timeout=timedelta(seconds=60))
    r = dist.get_rank()
    ids = torch.full((3, 5), 100 * r, dtype=torch.int32) + torch.arange(5, dtype=torch.int32)
    approx = torch.full((3, 5), float(r))
    exact = None if {no_exact} else torch.full((3, 5), 10.0 + r)
    g_ids, g_approx, g_exact = gather_candidates((ids, approx, exact))
    out = dict(shape=list(g_ids.shape), ids0=g_ids[0, 0].tolist(), ids1=g_ids[1, 0].tolist(),
               approx=g_approx[:, 0, 0].tolist(), exact=None if g_exact is None else g_exact[:, 0, 0].tolist())
    with open(os.path.join({tmp!r}, f"r{{r}}.json"), "w") as f:
        json.dump(out, f)
    dist.destroy_process_group()
""")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("no_exact", [False, True])
def test_two_ranks_gather_in_rank_order(tmp_path, no_exact):
    import json
    script = tmp_path / "w.py"
    script.write_text(WORKER.format(root=ROOT, tmp=str(tmp_path), no_exact=no_exact))
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={_free_port()}", str(script)]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300,
                       env=dict(os.environ, CUDA_VISIBLE_DEVICES=""))
    assert r.returncode == 0, r.stderr[-2000:]
    for i in range(2):
        out = json.loads((tmp_path / f"r{i}.json").read_text())
        assert out["shape"] == [2, 3, 5]
        assert out["ids0"] == [0, 1, 2, 3, 4] and out["ids1"] == [100, 101, 102, 103, 104]
        assert out["approx"] == [0.0, 1.0]
        assert out["exact"] == (None if no_exact else [10.0, 11.0])
