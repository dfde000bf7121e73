"""The Full indexer has two complete implementations: a single launch per
query cluster (used whenever a query's entries fit its shared memory) and a
multi-launch path (scan, then per target a collecting pass and a per-query
select, used for longer sequences). This runs the Full-indexer parity tests once more with
the multi-launch path forced (CSA2_FULL_PATH=multipass, read by the library
at load time, hence the separate process); there the score keys left in the
workspace are also compared with the oracle's exact scores."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def test_full_indexer_multipass_path(cuda_device):
    env = dict(os.environ, CSA2_FULL_PATH="multipass")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-m", "gpu", "-p", "no:cacheprovider",
                        os.path.join(HERE, "test_indexer_gpu.py"), "-k", "full"],
                       env=env, cwd=os.path.dirname(HERE), capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]


def test_reindex_cluster_path(cuda_device):
    """The Reindex parity tests once more on the one-launch cluster kernel
    (CSA2_REINDEX=cluster) instead of the default two-launch path."""
    env = dict(os.environ, CSA2_REINDEX="cluster")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-m", "gpu", "-p", "no:cacheprovider",
                        os.path.join(HERE, "test_indexer_gpu.py"), "-k", "reindex"],
                       env=env, cwd=os.path.dirname(HERE), capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]


@pytest.mark.parametrize("mode", ["exact", "redo"])
def test_batched_full_modes(cuda_device, mode):
    """The batched Full parity tests once more with the exact two-pass path
    alone (CSA2_BATCH_MODE=exact) and with every query handed from the sampled
    threshold path to the exact passes (=redo), the fallback the sampled path
    takes when its threshold leaves too few candidates."""
    env = dict(os.environ, CSA2_BATCH_MODE=mode)
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-m", "gpu", "-p", "no:cacheprovider",
                        os.path.join(HERE, "test_indexer_gpu.py"), "-k", "batched"],
                       env=env, cwd=os.path.dirname(HERE), capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
