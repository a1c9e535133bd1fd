"""Host-side planning of the host-fed step pipeline (no device work)."""
import pytest

from paged_kv_cache_370_b200.step import HostStepPipeline


@pytest.mark.parametrize("k", list(range(1, 70)) + [100, 500])
def test_ramp_sizes_cover_the_steps_and_keep_copies_hidden(k):
    kernel, up, down = 55.0, 16.0, 10.0
    sizes = HostStepPipeline.ramp_sizes(k, kernel_us=kernel, upload_us=up, download_us=down)
    assert sum(sizes) == k and all(1 <= s <= 16 for s in sizes)
    for a, b in zip(sizes, sizes[1:]):
        assert b * up <= a * kernel, f"uploads of a round of {b} not under a round of {a}"
        assert a * down <= b * kernel, f"downloads of a round of {a} not under a round of {b}"


def test_ramp_sizes_short_runs_start_and_end_small():
    # only the first round's uploads and the last round's downloads are exposed
    assert HostStepPipeline.ramp_sizes(20) == [1, 3, 10, 5, 1]
    assert HostStepPipeline.ramp_sizes(1) == [1]
    assert HostStepPipeline.ramp_sizes(0) == []
