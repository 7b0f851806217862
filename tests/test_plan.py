"""Host-side planning of the chunk forward (no GPU): how a sequence of NC
chunks over B*H heads is split into waves for a given workspace, and when the
segment-parallel state pass is used.  The planner is the library's own
(`gdn_chunk_fwd_plan`, the rule the launcher follows); these tests check its
contract against the workspace sizes the library reports."""
import math

import pytest
import torch

import gated_delta_rule_94_b200 as gdn
from gated_delta_rule_94_b200._lib import GDN_ERR_WORKSPACE

BF16, SCALAR, PERDIM = torch.bfloat16, gdn.GDN_GATE_SCALAR, gdn.GDN_GATE_PER_DIM
D = 128


def full(B, T, H, gate=SCALAR):
    return gdn.gdn_chunk_fwd_workspace_bytes(B, T, H, D, D, 64, BF16, gate)


def least(B, T, H, gate=SCALAR):
    return gdn.gdn_chunk_fwd_workspace_min_bytes(B, T, H, D, D, 64, BF16, gate)


def plan(B, T, H, ws, gate=SCALAR):
    return gdn.gdn_chunk_fwd_plan(B, T, H, D, D, 64, BF16, gate, ws)


def counter_bytes(NC):
    return (NC * 4 + 255) // 256 * 256


# one chunk of one head's step image: the least workspace of a one-chunk,
# one-head forward, less its 256-byte item counter
IMG = least(1, 64, 1) - counter_bytes(1)

SHAPES = [(1, 64, 1), (1, 256, 1), (1, 320, 1), (2, 6000, 2), (8, 300, 3), (4, 2048, 16),
          (3, 1000, 7), (1, 65536, 4), (1, 65536, 32), (2, 4096, 20)]


def sizes_between(B, T, H):
    lo, hi = least(B, T, H), full(B, T, H)
    return sorted({lo, (3 * lo + hi) // 4, (lo + hi) // 2, (lo + 3 * hi) // 4, hi, 2 * hi})


def test_image_size_is_a_whole_number_of_16_byte_units():
    assert IMG > 0 and IMG % 16 == 0


@pytest.mark.parametrize("B,T,H", SHAPES)
def test_waves_cover_the_sequence(B, T, H):
    NC = math.ceil(T / 64)
    for ws in sizes_between(B, T, H):
        p = plan(B, T, H, ws)
        assert p["chunks_per_wave"] >= 1
        assert p["waves"] == math.ceil(NC / p["chunks_per_wave"])
        assert p["segments"] >= 1


@pytest.mark.parametrize("B,T,H", SHAPES)
def test_plan_fits_its_workspace(B, T, H):
    """Without segment buffers, the images of the chosen waves (two alternating
    buffers and the carried state when there is more than one wave) and the
    item counters fit the workspace."""
    NC, nbh = math.ceil(T / 64), B * H
    for ws in sizes_between(B, T, H):
        p = plan(B, T, H, ws)
        if p["segments"] > 1:
            continue
        cw, nw = p["chunks_per_wave"], p["waves"]
        need = nbh * cw * IMG * (2 if nw > 1 else 1) + counter_bytes(NC)
        if nw > 1:
            need += nbh * D * D * 4
        assert need <= ws


@pytest.mark.parametrize("B,T,H", SHAPES)
def test_more_workspace_never_shortens_the_waves(B, T, H):
    cws = [plan(B, T, H, ws)["chunks_per_wave"] for ws in sizes_between(B, T, H)]
    assert cws == sorted(cws)


@pytest.mark.parametrize("B,T,H", SHAPES)
def test_least_workspace_runs_one_chunk_waves_and_less_is_refused(B, T, H):
    NC = math.ceil(T / 64)
    p = plan(B, T, H, least(B, T, H))
    assert p["segments"] == 1
    if NC > 1 and least(B, T, H) < NC * B * H * IMG + counter_bytes(NC):
        assert p["chunks_per_wave"] == 1 and p["waves"] == NC
    with pytest.raises(gdn.GdnError) as e:
        plan(B, T, H, least(B, T, H) - 1)
    assert e.value.status == GDN_ERR_WORKSPACE


@pytest.mark.parametrize("B,T,H", SHAPES)
def test_waves_overlap_and_respect_the_buffer_cap(B, T, H):
    """With the full-speed workspace: short sequences (up to four chunks) run as
    one wave; longer ones take at most half the chunks a wave, so that one
    wave's chain overlaps the next wave's prep, and a wave's image buffer stays
    within 160 MiB (unless a single chunk a wave already exceeds it)."""
    NC, nbh = math.ceil(T / 64), B * H
    p = plan(B, T, H, full(B, T, H))
    cw = p["chunks_per_wave"]
    if NC <= 4:
        assert p["waves"] == 1
    else:
        assert cw <= (NC + 1) // 2
        assert cw == 1 or cw * nbh * IMG <= 160 << 20


@pytest.mark.parametrize("B,T,H", SHAPES)
def test_segments_only_for_few_heads(B, T, H):
    nbh = B * H
    for ws in sizes_between(B, T, H):
        p = plan(B, T, H, ws)
        if nbh > 16:
            assert p["segments"] == 1
        if p["segments"] > 1:
            # every segment holds at least 8 chunks of the wave
            assert p["chunks_per_wave"] >= 8 * (p["segments"] - 1)


def test_few_head_long_sequences_use_segments_at_full_speed():
    assert plan(1, 65536, 4, full(1, 65536, 4))["segments"] > 1
    assert plan(2, 6000, 2, full(2, 6000, 2))["segments"] > 1


@pytest.mark.parametrize("B,T,H,gate,expect", [
    (4, 2048, 16, SCALAR, {"waves": 3, "chunks_per_wave": 13, "segments": 1}),
    (4, 4096, 16, PERDIM, {"waves": 3, "chunks_per_wave": 27, "segments": 1}),
    (1, 65536, 32, SCALAR, {"waves": 19, "chunks_per_wave": 55, "segments": 1}),
    (1, 65536, 4, SCALAR, {"waves": 3, "chunks_per_wave": 444, "segments": 18}),
])
def test_plans_of_the_measured_workloads(B, T, H, gate, expect):
    """The plans the bench's figures were measured with (full-speed workspace)."""
    assert plan(B, T, H, full(B, T, H, gate), gate) == expect


@pytest.mark.parametrize("dtype,dk", [(torch.float32, 128), (torch.bfloat16, 64)])
def test_cuda_core_path_runs_one_wave_without_workspace(dtype, dk):
    assert gdn.gdn_chunk_fwd_workspace_bytes(2, 200, 2, dk, dk, 64, dtype, SCALAR) == 0
    assert gdn.gdn_chunk_fwd_plan(2, 200, 2, dk, dk, 64, dtype, SCALAR, 0) == \
        {"waves": 1, "chunks_per_wave": 4, "segments": 1}
