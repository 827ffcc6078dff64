"""The append kernel's work split against the oracle at other group counts.

A multi-token append gives each CTA up to KVQ_APPEND_GROUPS_PER_CTA of a
sequence-head's completed 32-token groups (default 8), staging the next group's
rows while it quantizes one. The count is read once per process, so each
setting runs the page-parity tests in a child process: 1 (every group its own
CTA, nothing staged ahead), 3 (strided groups, a ragged last round) and 64
(one CTA per sequence-head). The pages must stay bit-identical to the oracle's.
"""

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


@pytest.mark.parametrize("groups_per_cta", [1, 3, 64])
def test_append_parity_at_group_count(groups_per_cta):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    env = dict(os.environ, KVQ_APPEND_GROUPS_PER_CTA=str(groups_per_cta))
    cmd = [sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider", "-m", "gpu",
           os.path.join(HERE, "test_gpu_parity.py"),
           "-k", "append_and_decode_small or fp32_inputs or window_boundaries or chunking_invariance "
                 "or full_llama_k4v4_layer"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
    assert " passed" in r.stdout and "failed" not in r.stdout
