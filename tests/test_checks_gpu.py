"""The debug build (-DPOEM_CHECKS, libpoem_checks.so): the same kernels with
device-side bounds checks on the packed score writes, the sampled-query
workspace and the selection scratch.  It stands in for a memory checker: a
small exact layer, a chunked call and the practical path run through it in a
child process (the binding picks the library at import) and must match the
oracle with every bounds check silent."""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


def test_checks_build_runs_small_layers_without_a_bounds_fault():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    sys.path.insert(0, os.path.dirname(HERE))
    from block_sparse_attention_poem_b200 import build

    build.build(variant="checks")
    env = dict(os.environ, POEM_LIBRARY_VARIANT="checks")
    r = subprocess.run([sys.executable, os.path.join(HERE, "_checks_layer.py")], env=env, capture_output=True,
                       text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert "checks build ok" in r.stdout
