"""The device status word: a code recorded in one workspace survives the
switch to another, and reading it clears it.  The code is planted on the
host side of the test by writing the workspace header through torch (no
kernel is made to time out)."""
import pytest

from gpu_env import require_gpu

pytestmark = pytest.mark.gpu


def test_status_word_carried_to_new_workspace():
    require_gpu()
    import torch
    from matrix_aware_optimizers_muon_b200 import Context, build
    build.build()
    ctx = Context(0)
    ctx.attach_workspace(1 << 20)
    assert ctx.device_status() == 0
    ctx.workspace[:4].view(torch.int32).fill_(7)     # as a timed-out wait would leave it
    old = ctx.workspace
    ctx.attach_workspace(2 << 20)                    # a different buffer
    assert ctx.workspace.data_ptr() != old.data_ptr()
    assert ctx.device_status() == 7
    assert ctx.device_status() == 0                  # cleared by the read


def test_status_word_kept_when_workspace_detached():
    """Dropping the workspace (ctx.workspace = None) detaches it in the
    library after reading its status word, which the next read reports."""
    require_gpu()
    import torch
    from matrix_aware_optimizers_muon_b200 import Context, build
    build.build()
    ctx = Context(0)
    ctx.attach_workspace(1 << 20)
    ctx.workspace[:4].view(torch.int32).fill_(5)
    ctx.workspace = None
    torch.cuda.empty_cache()                         # the buffer may be unmapped now
    assert ctx.device_status() == 5
    ctx.attach_workspace(1 << 20)                    # a fresh buffer after the detach: no copy from the old one
    assert ctx.device_status() == 0
