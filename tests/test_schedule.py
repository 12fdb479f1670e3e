"""The timestep-aware cube schedule (DeltaQuant note: 16-token cubes 4x1x4 for
the first quarter to 30 % of denoising steps, 64-token cubes 4x2x8 after; an
amortised cube size of 33 against a uniform 32)."""
import pytest

from video_diffusion_w4a4_b200 import schedule


def test_schedule_switches_once():
    cubes = [schedule.cube_for_step(s, 50) for s in range(50)]
    assert cubes[:15] == [(4, 1, 4)] * 15 and cubes[15:] == [(4, 2, 8)] * 35
    assert [schedule.cube_for_step(s, 40, 0.25) for s in (9, 10)] == [(4, 1, 4), (4, 2, 8)]


def test_amortized_size_matches_the_note():
    # the kernel path's cost is proportional to the number of cubes: harmonic mean of the sizes
    a30 = schedule.amortized_cube_tokens(50, 0.3)
    assert a30 == pytest.approx(1.0 / (0.3 / 16 + 0.7 / 64))
    # the note's "amortised cube size 33" lies between the 25 % and 30 % schedules
    assert schedule.amortized_cube_tokens(40, 0.3) < 34 < schedule.amortized_cube_tokens(40, 0.25)
    assert schedule.amortized_cube_tokens(10, 0.0) == 64 and schedule.amortized_cube_tokens(10, 1.0) == 16


@pytest.mark.parametrize("args", [(-1, 10), (10, 10), (0, 0)])
def test_rejects_steps_outside_the_loop(args):
    with pytest.raises(ValueError):
        schedule.cube_for_step(*args)
