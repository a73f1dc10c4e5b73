"""Memory-safety checks of the CUDA path without a sanitizer.

  * Guard bands: every parameter, gradient and momentum tensor, and the
    workspace, sit inside a larger buffer whose bytes on either side hold a
    known canary pattern; after a step the canaries must be intact, so no
    kernel wrote outside the memory it was given.
  * Poisoned workspace: the workspace needs no initialisation, so a step on a
    workspace filled with NaN bytes must give bitwise the same parameters and
    momentum as one on a zeroed workspace; a kernel that read scratch memory
    before writing it would change the result.

Shapes cover both orientations, ragged tiles and rows whose length is not a
multiple of 4 (scalar update paths); flags cover each variant of the step.
"""
import pytest
import torch

from muon_polar_orthogonalized_b200 import _native as N
from muon_polar_orthogonalized_b200 import api
from tests.test_gpu_parity import FIXED, STEP_FLAGS, dev, make_state  # noqa: F401  (dev: fixture)

pytestmark = pytest.mark.gpu

GUARD_BYTES = 4096
CANARY = 0xA5
SHAPES = [(256, 1024), (1024, 256), (130, 200), (200, 130), (100, 300), (300, 100)]
VARIANTS = [0, N.MUON_UNFUSED_UPDATE, N.MUON_NORMUON, N.MUON_ROW_EQUILIBRATE, N.MUON_FP32_DEBUG,
            N.MUON_TC_NARROW_TILES, N.MUON_TC_WIDE_TILES]


def guarded_copy(t: torch.Tensor):
    """(buffer, view): a copy of t at byte GUARD_BYTES of a canary-filled buffer."""
    nbytes = t.numel() * t.element_size()
    buf = torch.full((2 * GUARD_BYTES + nbytes,), CANARY, dtype=torch.uint8, device=t.device)
    view = buf[GUARD_BYTES:GUARD_BYTES + nbytes].view(t.dtype).view(t.shape)
    view.copy_(t)
    return buf, view


def canaries_intact(buf: torch.Tensor, nbytes: int) -> bool:
    return bool((buf[:GUARD_BYTES] == CANARY).all()) and bool((buf[GUARD_BYTES + nbytes:] == CANARY).all())


@pytest.mark.parametrize("extra", VARIANTS)
def test_step_writes_nothing_outside_its_tensors_and_workspace(dev, extra):
    flags = STEP_FLAGS | extra
    groups, W, G, M, _, _ = make_state(dev, SHAPES, "bf16", 31)
    bands = []
    lists = []
    for src in (W, G, M):
        views = []
        for t in src:
            buf, view = guarded_copy(t)
            bands.append((buf, t.numel() * t.element_size()))
            views.append(view)
        lists.append(views)
    need = api.muon_workspace_size(groups, flags)
    wbuf = torch.full((2 * GUARD_BYTES + need,), CANARY, dtype=torch.uint8, device=dev)
    ws = wbuf[GUARD_BYTES:GUARD_BYTES + need]
    for _ in range(2):
        api.muon_step(*lists, groups, 0.02, 0.95, 0.01, 5, FIXED, flags, ws)
    torch.cuda.synchronize()
    assert api.muon_query_status(ws) == N.MUON_OK
    for k, (buf, nbytes) in enumerate(bands + [(wbuf, need)]):
        assert canaries_intact(buf, nbytes), f"guard band {k} overwritten"


@pytest.mark.parametrize("extra", [0, N.MUON_UNFUSED_UPDATE, N.MUON_NORMUON, N.MUON_ROW_EQUILIBRATE])
def test_step_never_reads_unwritten_workspace(dev, extra):
    flags = STEP_FLAGS | extra
    results = []
    for fill in (0x00, 0xFF):   # 0xFF bytes are NaN as fp32 and as bf16
        groups, W, G, M, _, _ = make_state(dev, SHAPES, "bf16", 32)
        ws = torch.full((api.muon_workspace_size(groups, flags),), fill, dtype=torch.uint8, device=dev)
        api.muon_step(W, G, M, groups, 0.02, 0.95, 0.01, 5, FIXED, flags, ws)
        torch.cuda.synchronize()
        assert api.muon_query_status(ws) == N.MUON_OK
        results.append([t.clone() for t in W + M])
    for a, b in zip(*results):
        assert torch.equal(a, b)


def test_orthogonalize_and_adamw_write_nothing_outside(dev):
    """The orthogonaliser on the edge shapes (including 1-row and 1-column
    matrices) and AdamW on tensors whose lengths are not multiples of 4."""
    from tests.test_gpu_parity import EDGE_SHAPES
    bands = []

    def guard(t):
        buf, view = guarded_copy(t)
        bands.append((buf, t.numel() * t.element_size()))
        return view

    groups = [(r, c, 1, k, N.MUON_BF16, 1.0) for k, (r, c) in enumerate(EDGE_SHAPES)]
    inputs = [guard(torch.randn(r, c, device=dev).to(torch.bfloat16)) for r, c in EDGE_SHAPES]
    outs = [guard(torch.zeros(r, c, device=dev)) for r, c in EDGE_SHAPES]
    need = api.muon_workspace_size(groups, 0)
    wbuf = torch.full((2 * GUARD_BYTES + need,), CANARY, dtype=torch.uint8, device=dev)
    ws = wbuf[GUARD_BYTES:GUARD_BYTES + need]
    api.muon_orthogonalize(inputs, outs, groups, 5, FIXED, 0, ws)

    numels = [17, 1000, 4099, 65539]
    P = [guard(torch.randn(n, device=dev) * 0.02) for n in numels]
    Gr = [guard(torch.randn(n, device=dev).to(torch.bfloat16)) for n in numels]
    Ma = [guard(torch.zeros(n, device=dev)) for n in numels]
    Va = [guard(torch.zeros(n, device=dev)) for n in numels]
    spec = api.AdamWSpec(P, Gr, Ma, Va, 3e-4, 0.9, 0.95, 1e-8, 0.1)
    for t in (1, 2):
        api.adamw_step([spec], t)
    torch.cuda.synchronize()
    assert api.muon_query_status(ws) == N.MUON_OK
    assert all(bool(torch.isfinite(o).all()) for o in outs)
    for k, (buf, nbytes) in enumerate(bands + [(wbuf, need)]):
        assert canaries_intact(buf, nbytes), f"guard band {k} overwritten"
